// Memory-bound kernels: per-branch RMSNorm + beta + average, SWA cache finalisation,
// decode-step attention (RoPE, ring write, split-K over keys), conv/SSM decode step,
// split-K finalisation.
#pragma once
#include "common.cuh"

namespace hymba {

__device__ __forceinline__ float block_sum_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x < 32) {
    t = (l < (int)(blockDim.x >> 5)) ? red[l] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (l == 0) red[0] = t;
  }
  __syncthreads();
  return red[0];
}

__device__ __forceinline__ void unpack8(const uint4& r, float* f) {
  const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&r);
#pragma unroll
  for (int e = 0; e < 8; ++e) f[e] = __bfloat162float(h[e]);
}
__device__ __forceinline__ void unpack8h(const uint4& r, float* f) {
  const __half* h = reinterpret_cast<const __half*>(&r);
#pragma unroll
  for (int e = 0; e < 8; ++e) f[e] = __half2float(h[e]);
}

// ----------------------------------------------------------------------------------------
// u = 1/2 [ g_attn * rms(O) ; g_ssm * rms(y * SiLU(z)) ] ([JJ] §数学表示 5), z == nullptr
// meaning y is already gated.  O fp32 [rows, ld_o] (attn_w columns); y [rows, ld_y] bf16 or
// fp32; z bf16 [rows, ld_z] (di columns) -> u fp16 [rows, ld_u].  fp16 holds the normalised
// values with 8x finer rounding than bf16 and cannot overflow: after the RMSNorm
// |value| <= sqrt(width) * |gain| / 2.
// Persistent CTAs of 128 threads walk the rows; each row's O, y and z arrive as three
// untiled bulk copies into a NORM_STAGES-deep shared-memory ring (completed on mbarriers),
// so several rows per SM are in flight while one is reduced.  The row is pulled into
// registers, both sums of squares are reduced across the CTA, the stage is handed back to
// the copy engine and the scaled row leaves as 16-byte (y) / 8-byte (O) fp16 stores.
// Requirements (checked by the host): attn_w % 4 == 0, di % 8 == 0, attn_w <= 2048,
// di <= 4096, 16-byte aligned rows.
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ void load8(const float* p, float* f) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f) {
  unpack8(*reinterpret_cast<const uint4*>(p), f);
}
constexpr int NORM_THREADS = 128;
constexpr int NORM_STAGES = 3;
constexpr int NORM_MAXO = 4;          // float4 chunks of O per thread (attn_w <= 2048)
constexpr int NORM_MAXY = 4;          // 8-element chunks of y per thread (d_inner <= 4096)

__host__ __device__ constexpr int norm_stage_bytes(int attn_w, int di, int y_bytes, bool has_z) {
  return attn_w * 4 + di * y_bytes + (has_z ? di * 2 : 0);
}

template <typename YT>
__global__ void __launch_bounds__(NORM_THREADS)
    branch_norm_avg_kernel(const float* __restrict__ O, int ld_o, int attn_w, const YT* __restrict__ y, int ld_y,
                           const __nv_bfloat16* __restrict__ z, int ld_z, int di, const float* __restrict__ g_attn,
                           const float* __restrict__ g_ssm, float eps, __half* __restrict__ u, int ld_u, int rows,
                           DevStatus* status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t norm_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(norm_smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t full[NORM_STAGES];
  __shared__ float red[2][4][2];   // double-buffered by row parity: one barrier per row
  __shared__ int abort_flag;
  const bool has_z = z != nullptr;
  const int o_bytes = attn_w * 4, y_bytes = di * (int)sizeof(YT), z_bytes = has_z ? di * 2 : 0;
  const int stage_bytes = (o_bytes + y_bytes + z_bytes + 127) & ~127;
  const int t = threadIdx.x, wr = t >> 5, ln = t & 31;
  const int n_mine = blockIdx.x < rows ? (rows - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (t == 0) {
    for (int i = 0; i < NORM_STAGES; ++i) mbar_init(&full[i], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int i) {   // one thread: the copies of this CTA's i-th row
    const size_t row = (size_t)blockIdx.x + (size_t)i * gridDim.x;
    uint8_t* st = base + (i % NORM_STAGES) * stage_bytes;
    uint64_t* bar = &full[i % NORM_STAGES];
    mbar_arrive_expect_tx(bar, (uint32_t)(o_bytes + y_bytes + z_bytes));
    bulk_load(st, O + row * ld_o, (uint32_t)o_bytes, bar);
    bulk_load(st + o_bytes, y + row * ld_y, (uint32_t)y_bytes, bar);
    if (has_z) bulk_load(st + o_bytes + y_bytes, z + row * ld_z, (uint32_t)z_bytes, bar);
  };
  int issued = 0;
  if (t == 0)
    for (; issued < NORM_STAGES && issued < n_mine; ++issued) issue(issued);
  const float inv_a = 1.f / (float)attn_w, inv_s = 1.f / (float)di;
  int i = 0;
  for (; i < n_mine; ++i) {
    const size_t row = (size_t)blockIdx.x + (size_t)i * gridDim.x;
    const bool ok = mbar_wait(&full[i % NORM_STAGES], (uint32_t)(i / NORM_STAGES) & 1u, &abort_flag, status, 401);
    const uint8_t* st = base + (i % NORM_STAGES) * stage_bytes;
    const float* so = reinterpret_cast<const float*>(st);
    const YT* sy = reinterpret_cast<const YT*>(st + o_bytes);
    const __nv_bfloat16* sz = reinterpret_cast<const __nv_bfloat16*>(st + o_bytes + y_bytes);
    float fo[NORM_MAXO][4], fy[NORM_MAXY][8];
    float sa = 0.f, ss = 0.f;
#pragma unroll
    for (int k = 0; k < NORM_MAXO; ++k) {
      const int c = (t + k * NORM_THREADS) * 4;
      if (c < attn_w) {
        const float4 v = *reinterpret_cast<const float4*>(so + c);
        fo[k][0] = v.x; fo[k][1] = v.y; fo[k][2] = v.z; fo[k][3] = v.w;
        sa += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
      }
    }
#pragma unroll
    for (int k = 0; k < NORM_MAXY; ++k) {
      const int c = (t + k * NORM_THREADS) * 8;
      if (c < di) {
        load8(sy + c, fy[k]);
        if (has_z) {
          float fz[8];
          unpack8(*reinterpret_cast<const uint4*>(sz + c), fz);
#pragma unroll
          for (int e = 0; e < 8; ++e) fy[k][e] *= silu_f(fz[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) ss += fy[k][e] * fy[k][e];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sa += __shfl_xor_sync(0xffffffffu, sa, o);
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
    }
    float (*rd)[2] = red[i & 1];
    if (ln == 0) {
      rd[wr][0] = sa;
      rd[wr][1] = ss;
    }
    const int bad = __syncthreads_or(ok ? 0 : 1);   // stage i fully read; partial sums visible
    sa = rd[0][0] + rd[1][0] + rd[2][0] + rd[3][0];
    ss = rd[0][1] + rd[1][1] + rd[2][1] + rd[3][1];
    if (bad) break;
    if (t == 0 && issued < n_mine) issue(issued++);   // refill this stage with a later row
    const float ra = 0.5f / sqrtf(sa * inv_a + eps);
    const float rs = 0.5f / sqrtf(ss * inv_s + eps);
    __half* u_r = u + row * ld_u;
#pragma unroll
    for (int k = 0; k < NORM_MAXO; ++k) {
      const int c = (t + k * NORM_THREADS) * 4;
      if (c < attn_w) {
        const float4 g = *reinterpret_cast<const float4*>(g_attn + c);
        *reinterpret_cast<uint2*>(u_r + c) = make_uint2(pack_f16x2(fo[k][0] * ra * g.x, fo[k][1] * ra * g.y),
                                                        pack_f16x2(fo[k][2] * ra * g.z, fo[k][3] * ra * g.w));
      }
    }
#pragma unroll
    for (int k = 0; k < NORM_MAXY; ++k) {
      const int c = (t + k * NORM_THREADS) * 8;
      if (c < di) {
        float g[8];
        load8(g_ssm + c, g);
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) pk[e / 2] = pack_f16x2(fy[k][e] * rs * g[e], fy[k][e + 1] * rs * g[e + 1]);
        *reinterpret_cast<uint4*>(u_r + attn_w + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }
  if (i < n_mine && t == 0)   // gave up: let the copies in flight land before the CTA exits
    for (int j = i; j < issued; ++j)
      mbar_wait(&full[j % NORM_STAGES], (uint32_t)(j / NORM_STAGES) & 1u, nullptr, status, 402);
}

// ----------------------------------------------------------------------------------------
// SWA cache after prefill: meta rows [0, M) -> meta_k/v; rows [max(M, T-W), T) -> ring slot
// (pos - M) mod W.  view_k/v [B, Lmax, Hkv*D]; meta [B, M, Hkv*D]; ring [B, W, Hkv*D].
// ----------------------------------------------------------------------------------------
__global__ void swa_cache_finalize_kernel(const __half* __restrict__ vk, const __half* __restrict__ vv,
                                          int Lmax, int T, int M, int W, int row_elems,
                                          __half* __restrict__ meta_k, __half* __restrict__ meta_v,
                                          __half* __restrict__ ring_k, __half* __restrict__ ring_v) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int first_win = max(M, T - W);
  const int n_rows = M + (T - first_win);
  const int vec_per_row = row_elems / 8;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_rows * vec_per_row; i += gridDim.x * blockDim.x) {
    const int rr = i / vec_per_row, cv = (i % vec_per_row) * 8;
    int pos;
    __half *dk, *dv;
    if (rr < M) {
      pos = rr;
      dk = meta_k + ((size_t)b * M + pos) * row_elems;
      dv = meta_v + ((size_t)b * M + pos) * row_elems;
    } else {
      pos = first_win + (rr - M);
      const int slot = (pos - M) % W;
      dk = ring_k + ((size_t)b * W + slot) * row_elems;
      dv = ring_v + ((size_t)b * W + slot) * row_elems;
    }
    const size_t src = ((size_t)b * Lmax + pos) * row_elems + cv;
    *reinterpret_cast<uint4*>(dk + cv) = *reinterpret_cast<const uint4*>(vk + src);
    *reinterpret_cast<uint4*>(dv + cv) = *reinterpret_cast<const uint4*>(vv + src);
  }
}

// ----------------------------------------------------------------------------------------
// Decode step, before attention: the conv step of the SSM input (blocks [0, conv_blocks))
// and RoPE of the new token's query heads and key heads at position p (the other blocks).
// Rotated queries, pre-scaled by log2(e)/sqrt(D), go to qrot [B, Hq, 64]; an own/producer
// layer writes the rotated k and v of position p into its cache (ring slot (p - M) mod W, or
// row p of a global cache), so that attention reads every key, the new one included, from
// the cache.  Conv: window [state(3), x_new] -> xc = SiLU(b + w . window), the state shifts;
// x from proj [B, ld_proj] fp32 at column off_x; xc [B, Di] bf16; state [B, Di, 3] fp32.
// ----------------------------------------------------------------------------------------
struct DecPrepParams {
  const float* proj;
  int ld_proj, B, Di, off_x, conv_blocks;
  const float* conv_w;
  const float* conv_b;
  float* conv_state;
  __nv_bfloat16* xc;
  int Hq, Hkv, p, write_kv, is_global, M, W, Lmax;
  __half *ring_k, *ring_v, *full_k, *full_v;
  float* qrot;
  float scale_log2;
  double rope_theta[32];
};

__global__ void __launch_bounds__(256) decode_prep_kernel(const __grid_constant__ DecPrepParams p) {
  pdl_wait();
  pdl_trigger();
  if ((int)blockIdx.x < p.conv_blocks) {
    const int i = blockIdx.x * 256 + threadIdx.x;
    if (i >= p.B * p.Di) return;
    const int b = i / p.Di, c = i % p.Di;
    float* st = p.conv_state + (size_t)i * 3;
    const float x0 = st[0], x1 = st[1], x2 = st[2];
    const float xn = p.proj[(size_t)b * p.ld_proj + p.off_x + c];
    const float4 wv = *reinterpret_cast<const float4*>(p.conv_w + (size_t)c * 4);
    const float acc = p.conv_b[c] + wv.x * x0 + wv.y * x1 + wv.z * x2 + wv.w * xn;
    p.xc[i] = __float2bfloat16_rn(silu_f(acc));
    st[0] = x1;
    st[1] = x2;
    st[2] = xn;
    return;
  }
  const int n_heads = p.Hq + (p.write_kv ? p.Hkv : 0);
  const int i = (blockIdx.x - p.conv_blocks) * 256 + threadIdx.x;
  if (i >= p.B * n_heads * 32) return;
  const int j = i & 31, hh = (i >> 5) % n_heads, b = (i >> 5) / n_heads;
  // angle p * theta_j reduced mod 2 pi in double precision, then the fp32 sincos
  double a = (double)p.p * p.rope_theta[j];
  a -= 6.283185307179586 * rint(a * 0.15915494309189535);
  float sn, cs;
  sincosf((float)a, &sn, &cs);
  const float* pr = p.proj + (size_t)b * p.ld_proj;
  if (hh < p.Hq) {
    const float x1 = pr[hh * 64 + j], x2 = pr[hh * 64 + j + 32];
    float* q = p.qrot + ((size_t)b * p.Hq + hh) * 64;
    q[j] = (x1 * cs - x2 * sn) * p.scale_log2;
    q[j + 32] = (x2 * cs + x1 * sn) * p.scale_log2;
    return;
  }
  const int g = hh - p.Hq;
  const int kvw = p.Hkv * 64;
  const float* kp = pr + p.Hq * 64 + g * 64;
  const float* vp = kp + kvw;
  const float k1 = kp[j], k2 = kp[j + 32];
  size_t row;
  __half *dk, *dv;
  if (p.is_global) {
    row = ((size_t)b * p.Lmax + p.p) * kvw + g * 64;
    dk = p.full_k + row;
    dv = p.full_v + row;
  } else {
    row = ((size_t)b * p.W + (p.p - p.M) % p.W) * kvw + g * 64;
    dk = p.ring_k + row;
    dv = p.ring_v + row;
  }
  dk[j] = __float2half_rn(k1 * cs - k2 * sn);
  dk[j + 32] = __float2half_rn(k2 * cs + k1 * sn);
  dv[j] = __float2half_rn(vp[j]);
  dv[j + 32] = __float2half_rn(vp[j + 32]);
}

// ----------------------------------------------------------------------------------------
// Decode attention ([JJ] eq. (1) for the one new query per sequence), split over keys.
// Keys of (sequence b, kv head g): the meta tiles (SWA) then the ring slots, or rows 0..p of
// a global cache; a key is visible iff it is stored (meta row < M, ring slot < number of
// filled slots, global row <= p): the window of an SWA layer is exactly the ring, so keys
// are visited in slot order (the softmax does not depend on the order).  Work item =
// (b, g, split of DA_TPS tiles of 64 keys); persistent CTAs walk their items while one
// thread keeps DA_STAGES K/V tile pairs in flight by TMA (128-byte swizzled boxes of the
// [rows, Hkv*64] caches), so loads of the next item overlap the current one.  The query
// heads of group g share each K/V tile: scores (thread = key, 3 heads), an online softmax
// per head across the item's tiles, PV (thread = dim pair x key quarter).  Partial (m, l,
// o[64]) per (b, head, split) go to part [B, Hq, n_splits, 66]; the combine kernel merges.
// ----------------------------------------------------------------------------------------
constexpr int DA_KT = 64;               // keys per tile
constexpr int DA_STAGES = 4;
constexpr int DA_TPS = 2;               // tiles per split
constexpr int DA_THREADS = 128;
constexpr int DA_TILE_BYTES = DA_KT * 128;
constexpr int DEC_MAXG = 6;             // max query heads per KV head
constexpr int DA_SMEM = DA_STAGES * 2 * DA_TILE_BYTES + 1024;

struct DecAttnParams {
  const float* qrot;       // [B, Hq, 64] rotated, pre-scaled queries
  int Hq, Hkv, M, is_global;
  int n_meta_tiles;        // SWA: cdiv(M, 64); global: 0
  int n_tiles;             // tiles per (b, g)
  int n_main_valid;        // SWA: filled ring slots; global: p + 1
  int rows_main;           // rows per sequence in the main cache (W or Lmax)
  int n_splits, n_items;
  float* part;
  DevStatus* status;
};

// element (key r, dim d) of a 64 x 64 fp16 tile stored with the 128-byte swizzle
__device__ __forceinline__ const __half* sw128_row_chunk(const uint8_t* tile, int r, int chunk) {
  return reinterpret_cast<const __half*>(tile + r * 128 + ((chunk ^ (r & 7)) << 4));
}

__global__ void __launch_bounds__(DA_THREADS)
    decode_attn_kernel(const __grid_constant__ CUtensorMap mapMK, const __grid_constant__ CUtensorMap mapMV,
                       const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                       const __grid_constant__ DecAttnParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t da_smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(da_smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[DA_STAGES];
  __shared__ __align__(16) float qs[DEC_MAXG][64];
  __shared__ __align__(16) float ps[DEC_MAXG][DA_KT];
  __shared__ float mrun[DEC_MAXG], lrun[DEC_MAXG], alph[DEC_MAXG];
  __shared__ __align__(16) float opart[4][DEC_MAXG][64];
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.Hq / p.Hkv;
  if (tid == 0) {
    for (int i = 0; i < DA_STAGES; ++i) mbar_init(&full[i], 1);
    abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapMK);
    tma_prefetch_desc(&mapMV);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  __syncthreads();

  auto item_tiles = [&](int w) { return min(DA_TPS, p.n_tiles - (w % p.n_splits) * DA_TPS); };
  // producer state (thread 0): the next (item, tile) of this CTA's sequence
  int pw = blockIdx.x, pt = 0, issued = 0;
  auto issue_next = [&]() {
    while (pw < p.n_items && pt >= item_tiles(pw)) {
      pw += gridDim.x;
      pt = 0;
    }
    if (pw >= p.n_items) return;
    const int split = pw % p.n_splits, bg = pw / p.n_splits;
    const int g = bg % p.Hkv, b = bg / p.Hkv;
    const int ti = split * DA_TPS + pt;
    const int stg = issued % DA_STAGES;
    uint8_t* kt = tiles + stg * 2 * DA_TILE_BYTES;
    mbar_arrive_expect_tx(&full[stg], 2 * DA_TILE_BYTES);
    if (ti < p.n_meta_tiles) {
      tma_load_2d(kt, &mapMK, &full[stg], g * 64, b * p.M + ti * DA_KT);
      tma_load_2d(kt + DA_TILE_BYTES, &mapMV, &full[stg], g * 64, b * p.M + ti * DA_KT);
    } else {
      const int r0 = b * p.rows_main + (ti - p.n_meta_tiles) * DA_KT;
      tma_load_2d(kt, &mapK, &full[stg], g * 64, r0);
      tma_load_2d(kt + DA_TILE_BYTES, &mapV, &full[stg], g * 64, r0);
    }
    ++pt;
    ++issued;
  };
  if (tid == 0)
    for (int k = 0; k < DA_STAGES - 1; ++k) issue_next();

  int ct = 0;   // tiles consumed
  bool ok = true;
  for (int w = blockIdx.x; w < p.n_items; w += gridDim.x) {
    const int split = w % p.n_splits, bg = w / p.n_splits;
    const int g = bg % p.Hkv, b = bg / p.Hkv;
    const int nt = item_tiles(w);
    for (int i = tid; i < G * 64; i += DA_THREADS)
      qs[i >> 6][i & 63] = p.qrot[((size_t)b * p.Hq + g * G + (i >> 6)) * 64 + (i & 63)];
    if (tid < G) {
      mrun[tid] = -INFINITY;
      lrun[tid] = 0.f;
    }
    float acc[DEC_MAXG][2];
#pragma unroll
    for (int hh = 0; hh < DEC_MAXG; ++hh) acc[hh][0] = acc[hh][1] = 0.f;
    __syncthreads();
    for (int t = 0; t < nt; ++t, ++ct) {
      if (tid == 0) issue_next();   // the stage of tile ct-1 was released by the last barrier
      const int stg = ct % DA_STAGES;
      if (!mbar_wait(&full[stg], (uint32_t)(ct / DA_STAGES) & 1u, &abort_flag, p.status, 501)) ok = false;
      const uint8_t* kt = tiles + stg * 2 * DA_TILE_BYTES;
      const uint8_t* vt = kt + DA_TILE_BYTES;
      const int ti = split * DA_TPS + t;
      const bool meta = ti < p.n_meta_tiles;
      const int key0 = meta ? ti * DA_KT : (ti - p.n_meta_tiles) * DA_KT;
      const int lim = meta ? p.M : p.n_main_valid;
      {  // scores: thread = (key kk, heads hg, hg+2, hg+4)
        const int kk = tid & 63, hg = tid >> 6;
        float kf[64];
#pragma unroll
        for (int c = 0; c < 8; ++c) unpack8h(*reinterpret_cast<const uint4*>(sw128_row_chunk(kt, kk, c)), kf + c * 8);
        const bool vis = key0 + kk < lim;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const int hh = hg + 2 * j;
          if (hh < G) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int d = 0; d < 64; d += 8) {
              const float4 q0 = *reinterpret_cast<const float4*>(&qs[hh][d]);
              const float4 q1 = *reinterpret_cast<const float4*>(&qs[hh][d + 4]);
              a0 = fmaf(q0.x, kf[d], a0); a1 = fmaf(q0.y, kf[d + 1], a1);
              a0 = fmaf(q0.z, kf[d + 2], a0); a1 = fmaf(q0.w, kf[d + 3], a1);
              a0 = fmaf(q1.x, kf[d + 4], a0); a1 = fmaf(q1.y, kf[d + 5], a1);
              a0 = fmaf(q1.z, kf[d + 6], a0); a1 = fmaf(q1.w, kf[d + 7], a1);
            }
            ps[hh][kk] = vis ? a0 + a1 : -INFINITY;
          }
        }
      }
      __syncthreads();
      // online softmax per head (warp per head)
      for (int hh = warp; hh < G; hh += 4) {
        const float v0 = ps[hh][lane], v1 = ps[hh][lane + 32];
        float tm = fmaxf(v0, v1);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, o));
        const float m_old = mrun[hh];
        const float m_new = fmaxf(m_old, tm);        // finite: every tile holds a visible key
        const float al = m_old == -INFINITY ? 0.f : ex2_approx(m_old - m_new);
        const float e0 = ex2_approx(v0 - m_new), e1 = ex2_approx(v1 - m_new);
        ps[hh][lane] = e0;
        ps[hh][lane + 32] = e1;
        float sm = e0 + e1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
        __syncwarp();
        if (lane == 0) {
          lrun[hh] = lrun[hh] * al + sm;
          mrun[hh] = m_new;
          alph[hh] = al;
        }
      }
      __syncthreads();
      {  // PV: thread = (dims 2*lane, 2*lane+1; keys 16*warp ..)
        const int kq = warp;
#pragma unroll
        for (int hh = 0; hh < DEC_MAXG; ++hh)
          if (hh < G) {
            const float al = alph[hh];
            acc[hh][0] *= al;
            acc[hh][1] *= al;
          }
#pragma unroll 4
        for (int k = kq * 16; k < kq * 16 + 16; ++k) {
          const __half2 v2 = *reinterpret_cast<const __half2*>(sw128_row_chunk(vt, k, lane >> 2) + (lane & 3) * 2);
          const float v0 = __low2float(v2), v1 = __high2float(v2);
#pragma unroll
          for (int hh = 0; hh < DEC_MAXG; ++hh)
            if (hh < G) {
              const float pv = ps[hh][k];
              acc[hh][0] = fmaf(pv, v0, acc[hh][0]);
              acc[hh][1] = fmaf(pv, v1, acc[hh][1]);
            }
        }
      }
      if (__syncthreads_or(ok ? 0 : 1)) {   // a wait gave up: every thread leaves together
        ok = false;
        break;
      }
    }
    if (!ok) break;
    // the item's partial: sum the four key quarters
#pragma unroll
    for (int hh = 0; hh < DEC_MAXG; ++hh)
      if (hh < G) {
        opart[warp][hh][2 * lane] = acc[hh][0];
        opart[warp][hh][2 * lane + 1] = acc[hh][1];
      }
    __syncthreads();
    for (int i = tid; i < G * 64; i += DA_THREADS) {
      const int hh = i >> 6, d = i & 63;
      float* dst = p.part + (((size_t)b * p.Hq + g * G + hh) * p.n_splits + split) * 66;
      dst[2 + d] = opart[0][hh][d] + opart[1][hh][d] + opart[2][hh][d] + opart[3][hh][d];
      if (d == 0) {
        dst[0] = mrun[hh];
        dst[1] = lrun[hh];
      }
    }
    __syncthreads();   // qs, mrun, opart are rewritten by the next item
  }
  if (!ok && tid == 0)   // let the loads in flight land before the CTA exits
    for (int j = ct; j < issued; ++j)
      mbar_wait(&full[j % DA_STAGES], (uint32_t)(j / DA_STAGES) & 1u, nullptr, p.status, 502);
}

__global__ void decode_attn_combine_kernel(const float* __restrict__ part, int n_splits, int Hq,
                                           float* __restrict__ out, int ld_out) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;   // 64 threads
  const float* pp = part + ((size_t)b * Hq + h) * n_splits * 66;
  float M = -1e30f;
  for (int i = 0; i < n_splits; ++i) M = fmaxf(M, pp[i * 66]);
  float L = 0.f, O = 0.f;
  for (int i = 0; i < n_splits; ++i) {
    const float w = exp2f(pp[i * 66] - M);
    L += w * pp[i * 66 + 1];
    O += w * pp[i * 66 + 2 + d];
  }
  out[(size_t)b * ld_out + h * 64 + d] = O / L;
}

// ----------------------------------------------------------------------------------------
// decode SSM step ([JJ] §数学表示 4, one step of eq. (2)): dt = softplus(dt_low . W_dt[c] +
// bias), h = exp(dt A) h + dt B x, y = (C . h) * SiLU(z).  CTA = 16 channels x 16 states
// and DSSM_NB sequences: each W_dt element is read once per CTA and used for all its
// sequences, and every sequence's state is loaded before the dt dot products.
//   xbc [B, ld_xbc] fp32: dt_low at 0..R-1, B at R.., C at R+16..; W_dt [Di, ld_dt] fp32;
//   xc [B, Di] bf16; z from proj at column off_z; state [B, Di, 16] in place; y [B, Di] fp32.
//   R + 32 <= 256.
// ----------------------------------------------------------------------------------------
constexpr int DSSM_NB = 8;

__global__ void __launch_bounds__(256)
    decode_ssm_kernel(const float* __restrict__ xbc, int ld_xbc, int R, const float* __restrict__ w_dt, int ld_dt,
                      const float* __restrict__ dt_bias, const float* __restrict__ A,
                      const __nv_bfloat16* __restrict__ xc, const float* __restrict__ proj, int ld_proj,
                      int off_z, float* __restrict__ state, float* __restrict__ y, int Di, int B) {
  pdl_wait();
  pdl_trigger();
  __shared__ float dl[DSSM_NB][224];
  __shared__ float bcs[DSSM_NB][32];
  const int tid = threadIdx.x;
  const int cl = tid >> 4, s = tid & 15;
  const int c = blockIdx.x * 16 + cl;
  const int b0 = blockIdx.y * DSSM_NB;
  const int nb = min(DSSM_NB, B - b0);
  // this lane's state of every sequence first (the loads overlap the dot products)
  float h[DSSM_NB];
#pragma unroll
  for (int bi = 0; bi < DSSM_NB; ++bi)
    h[bi] = bi < nb ? state[((size_t)(b0 + bi) * Di + c) * 16 + s] : 0.f;
  for (int i = tid; i < DSSM_NB * R; i += 256) {
    const int bi = i / R, r = i - bi * R;
    dl[bi][r] = bi < nb ? xbc[(size_t)(b0 + bi) * ld_xbc + r] : 0.f;
  }
  for (int i = tid; i < DSSM_NB * 32; i += 256) {
    const int bi = i >> 5;
    bcs[bi][i & 31] = bi < nb ? xbc[(size_t)(b0 + bi) * ld_xbc + R + (i & 31)] : 0.f;
  }
  __syncthreads();
  float acc[DSSM_NB];
#pragma unroll
  for (int bi = 0; bi < DSSM_NB; ++bi) acc[bi] = 0.f;
  const float* wr = w_dt + (size_t)c * ld_dt;
  for (int r = s; r < R; r += 16) {
    const float wv = wr[r];
#pragma unroll
    for (int bi = 0; bi < DSSM_NB; ++bi) acc[bi] = fmaf(dl[bi][r], wv, acc[bi]);
  }
#pragma unroll
  for (int bi = 0; bi < DSSM_NB; ++bi)
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) acc[bi] += __shfl_xor_sync(0xffffffffu, acc[bi], o);
  const float bias = dt_bias[c];
  const float Acs = A[(size_t)c * 16 + s];
#pragma unroll
  for (int bi = 0; bi < DSSM_NB; ++bi) {
    if (bi >= nb) break;
    const int b = b0 + bi;
    const float dt = softplus_f(acc[bi] + bias);
    const float x = __bfloat162float(xc[(size_t)b * Di + c]);
    const float hn = fmaf(expf(dt * Acs), h[bi], dt * bcs[bi][s] * x);
    state[((size_t)b * Di + c) * 16 + s] = hn;
    float yv = bcs[bi][16 + s] * hn;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) yv += __shfl_xor_sync(0xffffffffu, yv, o);
    if (s == 0) y[(size_t)b * Di + c] = yv * silu_f(proj[(size_t)b * ld_proj + off_z + c]);
  }
}

// RoPE angles: tab[pos][j] = (cos, sin) of pos * base^(-2j/64), the angle reduced mod 2*pi
// in double precision before the fp32 sincos.
struct RopeThetas {
  double t[32];
};
__global__ void rope_table_kernel(float2* __restrict__ tab, int n_pos, const __grid_constant__ RopeThetas th) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pos * 32) return;
  const int pos = i >> 5, j = i & 31;
  double a = (double)pos * th.t[j];
  a -= 6.283185307179586 * rint(a * 0.15915494309189535);
  float s, c;
  sincosf((float)a, &s, &c);
  tab[i] = make_float2(c, s);
}

// out[r, :] = x[r, :] / sqrt(mean(x[r, :]^2) + eps) * gain  (one row per CTA, 256 threads)
__global__ void __launch_bounds__(256)
    rmsnorm_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ gain, int d, float eps,
                   __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  const size_t row = blockIdx.x;
  const __nv_bfloat16* xr = x + row * d;
  float ss = 0.f;
  for (int c = threadIdx.x * 8; c < d; c += 256 * 8) {
    float f[8];
    unpack8(*reinterpret_cast<const uint4*>(xr + c), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) ss += f[e] * f[e];
  }
  ss = block_sum_256(ss, red);
  const float r = 1.f / sqrtf(ss / (float)d + eps);
  for (int c = threadIdx.x * 8; c < d; c += 256 * 8) {
    float f[8];
    unpack8(*reinterpret_cast<const uint4*>(xr + c), f);
    uint32_t pk[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) pk[e / 2] = pack_bf16x2(f[e] * r * gain[c + e], f[e + 1] * r * gain[c + e + 1]);
    *reinterpret_cast<uint4*>(out + row * d + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

// out[b] = [meta; x[b]] : meta [M, d], x [B, N, d] -> out [B, M+N, d] (16-byte pieces)
__global__ void prepend_meta_kernel(const __nv_bfloat16* __restrict__ meta, const __nv_bfloat16* __restrict__ x,
                                    int B, int M, int N, int d, __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int vec = d / 8;
  const long long total = (long long)B * (M + N) * vec;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int v = (int)(i % vec);
    const long long rowg = i / vec;
    const int t = (int)(rowg % (M + N));
    const int b = (int)(rowg / (M + N));
    const __nv_bfloat16* src = t < M ? meta + (size_t)t * d : x + ((size_t)b * N + (t - M)) * d;
    *reinterpret_cast<uint4*>(out + rowg * d + v * 8) = *reinterpret_cast<const uint4*>(src + v * 8);
  }
}

// Waits on a barrier that nothing arrives at, through the same bounded wait the pipelined
// kernels use; the wait runs out and records DEV_ERR_TIMEOUT.
__global__ void wait_timeout_selftest_kernel(DevStatus* st) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, nullptr, st, 900);
}

// Fixed-order sum of split-K partial slices: out[i] = sum_s part[s*stride + i] (+ residual),
// as fp32 or bf16; n is a multiple of 4.  The order never changes, so results are
// identical from run to run.
// When bcT is set, columns [tr_col0, tr_col0 + 32) of the [rows, ld] result (rows = b*T + t)
// are also written time-major to bcT [B][32][Tp] (the scan's B/C input).
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int n_split, long long stride, int n,
                                     const __nv_bfloat16* __restrict__ residual, void* __restrict__ out,
                                     int out_bf16, float* __restrict__ bcT = nullptr, int ld = 0, int T = 0,
                                     int Tp = 0, int tr_col0 = 0) {
  pdl_wait();
  pdl_trigger();
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= n) return;
  float4 acc = *reinterpret_cast<const float4*>(part + i);
  for (int s = 1; s < n_split; ++s) {
    const float4 q = *reinterpret_cast<const float4*>(part + (size_t)s * stride + i);
    acc.x += q.x; acc.y += q.y; acc.z += q.z; acc.w += q.w;
  }
  if (residual != nullptr) {
    const __nv_bfloat162 r0 = *reinterpret_cast<const __nv_bfloat162*>(residual + i);
    const __nv_bfloat162 r1 = *reinterpret_cast<const __nv_bfloat162*>(residual + i + 2);
    acc.x += __low2float(r0); acc.y += __high2float(r0); acc.z += __low2float(r1); acc.w += __high2float(r1);
  }
  if (out_bf16) {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + i;
    *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + i) = acc;
  }
  if (bcT != nullptr) {
    const int row = i / ld, col = i % ld;       // 4 columns of one row (ld % 4 == 0)
    const int b = row / T, t = row % T;
    const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int cc = col + e - tr_col0;
      if (cc >= 0 && cc < 32) bcT[((size_t)b * 32 + cc) * Tp + t] = vals[e];
    }
  }
}

// out[r, c] = bf16(acc[r, c] + residual[r, c])
__global__ void f32_to_bf16_residual_kernel(const float* __restrict__ acc, const __nv_bfloat16* __restrict__ res,
                                            __nv_bfloat16* __restrict__ out, int n) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float v = acc[i];
  if (res != nullptr) v += __bfloat162float(res[i]);
  out[i] = __float2bfloat16_rn(v);
}

}  // namespace hymba
