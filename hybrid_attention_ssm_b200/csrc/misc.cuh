// Memory-bound kernels: per-branch RMSNorm + beta + average, the decode step (conv step and
// RoPE with the cache write, attention split over key tiles and its merge, the SSM step),
// split-K finalisation, RoPE tables, the stack's RMSNorm and the meta prepend.
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
  uint8_t* base = align_smem<128>(norm_smem_raw);
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
  // this thread's columns are the same in every row: their gains stay in registers
  float ga[NORM_MAXO][4], gs[NORM_MAXY][8];
#pragma unroll
  for (int k = 0; k < NORM_MAXO; ++k) {
    const int c = (t + k * NORM_THREADS) * 4;
    if (c < attn_w) {
      const float4 g = *reinterpret_cast<const float4*>(g_attn + c);
      ga[k][0] = g.x; ga[k][1] = g.y; ga[k][2] = g.z; ga[k][3] = g.w;
    }
  }
#pragma unroll
  for (int k = 0; k < NORM_MAXY; ++k) {
    const int c = (t + k * NORM_THREADS) * 8;
    if (c < di) load8(g_ssm + c, gs[k]);
  }
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
      if (c < attn_w)
        *reinterpret_cast<uint2*>(u_r + c) =
            make_uint2(pack_f16x2(fo[k][0] * ra * ga[k][0], fo[k][1] * ra * ga[k][1]),
                       pack_f16x2(fo[k][2] * ra * ga[k][2], fo[k][3] * ra * ga[k][3]));
    }
#pragma unroll
    for (int k = 0; k < NORM_MAXY; ++k) {
      const int c = (t + k * NORM_THREADS) * 8;
      if (c < di) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2)
          pk[e / 2] = pack_f16x2(fy[k][e] * rs * gs[k][e], fy[k][e + 1] * rs * gs[k][e + 1]);
        *reinterpret_cast<uint4*>(u_r + attn_w + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }
  if (i < n_mine && t == 0)   // gave up: let the copies in flight land before the CTA exits
    for (int j = i; j < issued; ++j)
      mbar_wait(&full[j % NORM_STAGES], (uint32_t)(j / NORM_STAGES) & 1u, nullptr, status, 402);
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
// Sum of the n <= NMAX split-K slices of an fp32 projection, in slice order (deterministic).
// The bound is a compile-time constant so that every load is issued before the first add.
template <int NMAX>
__device__ __forceinline__ float sum_slices(const float* p, long long stride, int n) {
  float v[NMAX];
#pragma unroll
  for (int i = 0; i < NMAX; ++i) v[i] = i < n ? p[i * stride] : 0.f;
  float s = v[0];
#pragma unroll
  for (int i = 1; i < NMAX; ++i) s += v[i];
  return s;
}
constexpr int DEC_MAX_IN_SPLIT = 4;     // in_proj split-K slices (the layout caps them)
constexpr int DEC_MAX_XPROJ_SPLIT = 8;  // x_proj split-K slices (the layout caps them)

struct DecPrepParams {
  const float* proj;          // in_proj output: n_slices split-K slices [B, ld_proj], slice stride proj_stride
  int n_slices;
  long long proj_stride;
  int ld_proj, B, Di, off_x, conv_blocks;
  const float* conv_w;
  const float* conv_b;
  float* conv_state;
  __nv_bfloat16* xc;
  int Hq, Hkv, p, write_kv, is_global, M, W, Lmax;
  const int* positions;       // per-sequence positions [B] (device), or NULL: every sequence at p
  int max_position;           // with positions: the caller's bound on them
  __half *ring_k, *ring_v, *full_k, *full_v;
  float* qrot;
  float scale_log2;
  DevStatus* status;
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
    const float xn = sum_slices<DEC_MAX_IN_SPLIT>(p.proj + (size_t)b * p.ld_proj + p.off_x + c, p.proj_stride, p.n_slices);
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
  int pos = p.p;
  if (p.positions != nullptr) {
    pos = p.positions[b];
    // a position the cache cannot hold: record it and leave this sequence's cache alone
    if (pos < p.M || pos > p.max_position || (p.is_global && pos >= p.Lmax)) {
      if (j == 0) report_error(p.status, DEV_ERR_BOUNDS, 232);
      return;
    }
  }
  // angle pos * theta_j reduced mod 2 pi in double precision, then the fp32 sincos
  double a = (double)pos * p.rope_theta[j];
  a -= 6.283185307179586 * rint(a * 0.15915494309189535);
  float sn, cs;
  sincosf((float)a, &sn, &cs);
  const float* pr = p.proj + (size_t)b * p.ld_proj;
  auto P = [&](int col) { return sum_slices<DEC_MAX_IN_SPLIT>(pr + col, p.proj_stride, p.n_slices); };
  if (hh < p.Hq) {
    const float x1 = P(hh * 64 + j), x2 = P(hh * 64 + j + 32);
    float* q = p.qrot + ((size_t)b * p.Hq + hh) * 64;
    const float qv[2] = {(x1 * cs - x2 * sn) * p.scale_log2, (x2 * cs + x1 * sn) * p.scale_log2};
    f16_range_guard<2>(qv, p.status, 230);   // the attention reads q as fp16
    q[j] = qv[0];
    q[j + 32] = qv[1];
    return;
  }
  const int g = hh - p.Hq;
  const int kvw = p.Hkv * 64;
  const int kc = p.Hq * 64 + g * 64, vc = kc + kvw;
  const float k1 = P(kc + j), k2 = P(kc + j + 32);
  size_t row;
  __half *dk, *dv;
  if (p.is_global) {
    row = ((size_t)b * p.Lmax + pos) * kvw + g * 64;
    dk = p.full_k + row;
    dv = p.full_v + row;
  } else {
    row = ((size_t)b * p.W + (pos - p.M) % p.W) * kvw + g * 64;
    dk = p.ring_k + row;
    dv = p.ring_v + row;
  }
  const float kv[4] = {k1 * cs - k2 * sn, k2 * cs + k1 * sn, P(vc + j), P(vc + j + 32)};
  f16_range_guard<4>(kv, p.status, 231);
  dk[j] = __float2half_rn(kv[0]);
  dk[j + 32] = __float2half_rn(kv[1]);
  dv[j] = __float2half_rn(kv[2]);
  dv[j + 32] = __float2half_rn(kv[3]);
}

// ----------------------------------------------------------------------------------------
// Decode attention ([JJ] eq. (1) for the one new query per sequence), split over keys.
// Keys of (sequence b, kv head g): the meta tiles (SWA) then the ring slots, or rows 0..p of
// a global cache; a key is visible iff it is stored (meta row < M, ring slot < number of
// filled slots, global row <= p): the window of an SWA layer is exactly the ring, so keys
// are visited in slot order (the softmax does not depend on the order).  Work item =
// (b, g, split of DA_TPS tiles of 64 keys); persistent CTAs walk their items while one
// thread keeps DA_STAGES K/V tile pairs in flight by TMA (128-byte swizzled boxes of the
// [rows, Hkv*64] caches), so loads of the next item overlap the current one.
// The G <= 6 query heads of group g form the rows of 16 x 16 fp16 tensor-core fragments
// (mma.sync m16n8k16, fp32 accumulation; rows >= G are zero): a tcgen05 tile would need
// at least 64 query rows, and this kernel is bound by the K/V bytes, not by the math.  Each
// of the 4 warps takes 16 keys of every tile: S = Q K^T from ldmatrix fragments of the
// swizzled K tile, an online softmax in registers, O += P V with P reused from the S
// accumulators and V fragments from ldmatrix.trans.  At the end of an item the 4 warps'
// (m, l, O) are merged; the partial (m, l, o[64]) per (b, head, split) goes to
// part [B, Hq, n_splits, 66] and decode_attn_combine_kernel merges the splits in split
// order.  Each item's queries arrive by bulk copy together with its first K/V tile.
// ----------------------------------------------------------------------------------------
constexpr int DA_KT = 64;               // keys per tile
constexpr int DA_STAGES = 3;
constexpr int DA_TPS = 3;               // tiles per split
constexpr int DA_CONSUMERS = 128;      // 4 consumer warps
constexpr int DA_THREADS = DA_CONSUMERS + 32;   // + the producer warp
constexpr int DA_TILE_BYTES = DA_KT * 128;
constexpr int DEC_MAXG = 6;             // max query heads per KV head
constexpr int DA_Q_BYTES = DEC_MAXG * 64 * 4;   // an item's queries ride with its first tile
constexpr int DA_SMEM = DA_STAGES * 2 * DA_TILE_BYTES + 1024;

struct DecAttnParams {
  const float* qrot;       // [B, Hq, 64] rotated, pre-scaled queries
  int Hq, Hkv, M, is_global;
  int n_meta_tiles;        // SWA: cdiv(M, 64); global: 0
  int n_tiles;             // tiles per (b, g) (with positions: the most any sequence has)
  int n_main_valid;        // SWA: filled ring slots; global: p + 1
  int rows_main;           // rows per sequence in the main cache (W or Lmax)
  int n_splits, n_items;
  const int* positions;    // per-sequence positions [B] (device), or NULL: n_main_valid for all
  int W, max_position;
  float* part;
  DevStatus* status;
};

// Keys of sequence b in the main cache (ring slots filled, or global rows 0..pos); 0 for a
// position the cache cannot hold (the prep kernel reports it).
__device__ __forceinline__ int da_main_valid(const DecAttnParams& p, int b) {
  if (p.positions == nullptr) return p.n_main_valid;
  const int pos = p.positions[b];
  if (pos < p.M || pos > p.max_position || (p.is_global && pos >= p.rows_main)) return 0;
  return p.is_global ? pos + 1 : min(pos - p.M + 1, p.W);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}
// d (16x8 fp32) += a (16x16 fp16, row-major) * b (16x8 fp16, column-major)
__device__ __forceinline__ void mma_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
               "{%0, %1, %2, %3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// shared address of the 16-byte chunk `chunk` of row r in a 64 x 64 fp16 tile stored with
// the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128_addr(uint32_t tile, int r, int chunk) {
  return tile + r * 128 + ((chunk ^ (r & 7)) << 4);
}

__device__ __forceinline__ void da_consumer_sync() {   // the four consumer warps only
  asm volatile("bar.sync 1, %0;" ::"n"(DA_CONSUMERS) : "memory");
}

__global__ void __launch_bounds__(DA_THREADS, 3)
    decode_attn_kernel(const __grid_constant__ CUtensorMap mapMK, const __grid_constant__ CUtensorMap mapMV,
                       const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                       const __grid_constant__ DecAttnParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t da_smem_raw[];
  uint8_t* tiles = align_smem<1024>(da_smem_raw);
  __shared__ uint64_t full[DA_STAGES], empty[DA_STAGES];
  __shared__ __align__(16) float qbuf[DA_STAGES][DEC_MAXG * 64];
  __shared__ float cm[4][8], cl[4][8];
  __shared__ __align__(16) float co[4][8][64];
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.Hq / p.Hkv;
  if (tid == 0) {
    for (int i = 0; i < DA_STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], DA_CONSUMERS / 32);
    }
    abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapMK);
    tma_prefetch_desc(&mapMV);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  __syncthreads();
  // tiles of item w: its split's share of the (b, g) tiles (none when the split lies past
  // them, as it can for a sequence shorter than the batch's longest)
  auto item_tiles = [&](int w, int main_valid) {
    const int nt = p.n_meta_tiles + (main_valid + DA_KT - 1) / DA_KT;
    return max(0, min(DA_TPS, nt - (w % p.n_splits) * DA_TPS));
  };

  if (warp == DA_CONSUMERS / 32) {
    // ------------------------------ producer warp ------------------------------
    // Streams this CTA's (item, tile) sequence through the ring; a stage is refilled once
    // the four consumer warps have released it.
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x) {
        const int split = w % p.n_splits, bg = w / p.n_splits;
        const int g = bg % p.Hkv, b = bg / p.Hkv;
        const int nt = item_tiles(w, da_main_valid(p, b));
        for (int t = 0; t < nt; ++t, ++issued) {
          const int stg = issued % DA_STAGES;
          if (issued >= DA_STAGES &&
              !mbar_wait(&empty[stg], (uint32_t)(issued / DA_STAGES - 1) & 1u, &abort_flag, p.status, 503)) {
            ok = false;
            break;
          }
          const int ti = split * DA_TPS + t;
          uint8_t* kt = tiles + stg * 2 * DA_TILE_BYTES;
          const uint32_t q_bytes = t == 0 ? (uint32_t)(G * 64 * 4) : 0u;
          mbar_arrive_expect_tx(&full[stg], 2 * DA_TILE_BYTES + q_bytes);
          if (t == 0) bulk_load(&qbuf[stg][0], p.qrot + ((size_t)b * p.Hq + g * G) * 64, q_bytes, &full[stg]);
          if (ti < p.n_meta_tiles) {
            tma_load_2d(kt, &mapMK, &full[stg], g * 64, b * p.M + ti * DA_KT);
            tma_load_2d(kt + DA_TILE_BYTES, &mapMV, &full[stg], g * 64, b * p.M + ti * DA_KT);
          } else {
            const int r0 = b * p.rows_main + (ti - p.n_meta_tiles) * DA_KT;
            tma_load_2d(kt, &mapK, &full[stg], g * 64, r0);
            tma_load_2d(kt + DA_TILE_BYTES, &mapV, &full[stg], g * 64, r0);
          }
        }
      }
      // the last fills may still be in flight (all of them, if the consumers gave up): let
      // them land before the CTA can exit
      for (int j = issued > DA_STAGES ? issued - DA_STAGES : 0; j < issued; ++j)
        mbar_wait(&full[j % DA_STAGES], (uint32_t)(j / DA_STAGES) & 1u, nullptr, p.status, 504);
    }
    return;
  }

  // ------------------------------ consumer warps ------------------------------
  const int gq = lane >> 2, tq = lane & 3;   // fragment row (query head) and column pair
  const uint32_t tiles_u32 = smem_u32(tiles);
  // ldmatrix row of this lane: K fragments (keys x dims), V fragments (.trans)
  const int k_row = warp * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
  const int k_chk = (lane >> 3) & 1;
  const int v_row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
  const int v_chk = (lane >> 4) & 1;
  int ct = 0;   // tiles consumed
  bool ok = true;
  for (int w = blockIdx.x; w < p.n_items; w += gridDim.x) {
    const int split = w % p.n_splits, bg = w / p.n_splits;
    const int g = bg % p.Hkv, b = bg / p.Hkv;
    const int main_valid = da_main_valid(p, b);
    const int nt = item_tiles(w, main_valid);
    uint32_t qa[4][2];   // Q fragments (fp16): row gq = query head (zero beyond G), 4 x 16 dims
    float m_run = -INFINITY, l_run = 0.f;
    float o[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    for (int t = 0; t < nt; ++t, ++ct) {
      const int stg = ct % DA_STAGES;
      // after a wait has given up, the warps keep walking the items (so that every one of
      // them reaches the same merge barriers) without waiting or releasing stages
      if (ok) ok = mbar_wait(&full[stg], (uint32_t)(ct / DA_STAGES) & 1u, &abort_flag, p.status, 501);
      ok = __all_sync(0xffffffffu, ok);   // one decision per warp: the shuffles below need all lanes
      if (!ok) continue;
      if (t == 0) {   // the item's queries arrived with its first tile
        const float* q = &qbuf[stg][gq * 64];
#pragma unroll
        for (int st = 0; st < 4; ++st) {
          float2 lo = make_float2(0.f, 0.f), hi = make_float2(0.f, 0.f);
          if (gq < G) {
            lo = *reinterpret_cast<const float2*>(q + st * 16 + 2 * tq);
            hi = *reinterpret_cast<const float2*>(q + st * 16 + 8 + 2 * tq);
          }
          qa[st][0] = pack_f16x2(lo.x, lo.y);
          qa[st][1] = pack_f16x2(hi.x, hi.y);
        }
      }
      const uint32_t kt = tiles_u32 + stg * 2 * DA_TILE_BYTES;
      const uint32_t vt = kt + DA_TILE_BYTES;
      const int ti = split * DA_TPS + t;
      const bool meta = ti < p.n_meta_tiles;
      const int key0 = meta ? ti * DA_KT : (ti - p.n_meta_tiles) * DA_KT;
      const int lim = meta ? p.M : main_valid;
      // S = Q K^T for this warp's 16 keys (two n-tiles of 8)
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sw128_addr(kt, k_row, 2 * st + k_chk), b0, b1, b2, b3);
        mma_16816(s0, qa[st][0], 0u, qa[st][1], 0u, b0, b1);
        mma_16816(s1, qa[st][0], 0u, qa[st][1], 0u, b2, b3);
      }
      // keys of this lane: tile columns warp*16 + 2tq + {0,1} (s0) and + 8 (s1)
      const int kb = key0 + warp * 16 + 2 * tq;
      float v[4] = {kb < lim ? s0[0] : -INFINITY, kb + 1 < lim ? s0[1] : -INFINITY,
                    kb + 8 < lim ? s1[0] : -INFINITY, kb + 9 < lim ? s1[1] : -INFINITY};
      float tm = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
      tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 1));
      tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 2));
      const float m_new = fmaxf(m_run, tm);
      float al = 1.f, e[4] = {0.f, 0.f, 0.f, 0.f};
      if (m_new != -INFINITY) {          // some key of this warp visible so far
        al = ex2_approx(m_run - m_new);  // 0 while nothing was accumulated
#pragma unroll
        for (int i = 0; i < 4; ++i) e[i] = ex2_approx(v[i] - m_new);
      }
      float rs = (e[0] + e[1]) + (e[2] + e[3]);
      rs += __shfl_xor_sync(0xffffffffu, rs, 1);
      rs += __shfl_xor_sync(0xffffffffu, rs, 2);
      l_run = l_run * al + rs;
      m_run = m_new;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        o[j][0] *= al;
        o[j][1] *= al;
      }
      // O += P V: P is the A fragment of the warp's 16 keys (rows >= 8 zero)
      const uint32_t pa0 = pack_f16x2(e[0], e[1]), pa2 = pack_f16x2(e[2], e[3]);
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sw128_addr(vt, v_row, j + v_chk), b0, b1, b2, b3);
        mma_16816(o[j], pa0, 0u, pa2, 0u, b0, b1);
        mma_16816(o[j + 1], pa0, 0u, pa2, 0u, b2, b3);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stg]);   // this warp is done with the stage
    }
    // merge the 4 warps' states for rows (heads) < G
    if (gq < 8) {
      if (tq == 0) {
        cm[warp][gq] = m_run;
        cl[warp][gq] = l_run;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float2*>(&co[warp][gq][8 * j + 2 * tq]) = make_float2(o[j][0], o[j][1]);
    }
    da_consumer_sync();
    if (ok) {
      for (int i = tid; i < G * 64; i += DA_CONSUMERS) {
        const int hh = i >> 6, d = i & 63;
        float M = cm[0][hh];
#pragma unroll
        for (int k = 1; k < 4; ++k) M = fmaxf(M, cm[k][hh]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float wk = cm[k][hh] == -INFINITY ? 0.f : ex2_approx(cm[k][hh] - M);
          L += wk * cl[k][hh];
          O += wk * co[k][hh][d];
        }
        float* dst = p.part + (((size_t)b * p.Hq + g * G + hh) * p.n_splits + split) * 66;
        dst[2 + d] = O;
        if (d == 0) {
          dst[0] = M;
          dst[1] = L;
        }
      }
    }
    da_consumer_sync();   // cm, cl, co are rewritten by the next item
  }
}

// merge of the decode attention splits: out[b, h*64 + d] = sum_s w_s o_s / sum_s w_s l_s,
// w_s = 2^(m_s - max m), in split order (64 threads per (head, sequence))
__global__ void decode_attn_combine_kernel(const float* __restrict__ part, int n_splits, int Hq,
                                           float* __restrict__ out, int ld_out) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;   // 64 threads
  const float* pp = part + ((size_t)b * Hq + h) * n_splits * 66;
  float M = -1e30f;
  for (int i0 = 0; i0 < n_splits; i0 += 8) {   // 8 splits' loads in flight at a time
    float mv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) mv[k] = i0 + k < n_splits ? pp[(i0 + k) * 66] : -1e30f;
#pragma unroll
    for (int k = 0; k < 8; ++k) M = fmaxf(M, mv[k]);
  }
  float L = 0.f, O = 0.f;
  for (int i0 = 0; i0 < n_splits; i0 += 8) {
    float mv[8], lv[8], ov[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const bool in = i0 + k < n_splits;
      mv[k] = in ? pp[(i0 + k) * 66] : -INFINITY;
      lv[k] = in ? pp[(i0 + k) * 66 + 1] : 0.f;
      ov[k] = in ? pp[(i0 + k) * 66 + 2 + d] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float w = exp2f(mv[k] - M);   // 0 for the padding
      L += w * lv[k];
      O += w * ov[k];
    }
  }
  out[(size_t)b * ld_out + h * 64 + d] = O / L;
}

// ----------------------------------------------------------------------------------------
// decode SSM step ([JJ] §数学表示 4, one step of eq. (2)): dt = softplus(dt_low . W_dt[c] +
// bias), h = exp(dt A) h + dt B x, y = (C . h) * SiLU(z).
// CTA = 64 channels x NB sequences, 256 threads; thread = one channel x BPT sequences
// (NB = 4 BPT), their BPT x 16 states in registers.  Everything the CTA reads arrives in one
// round: bulk copies bring the x_proj slices of its sequences and the W_dt rows of its
// channels into shared memory while every thread loads its states, x, z and A row; the
// slices are then added in slice order in shared memory.
//   xbc: n_xbc split-K slices [B, ld_xbc] fp32 (stride xbc_stride): dt_low at 0..R-1, B at
//   R.., C at R+16..; W_dt [Di, ld_dt] fp32; xc [B, Di] bf16; z from the in_proj slices
//   (stride proj_stride) at column off_z; state [B, Di, 16] in place; y [B, Di] fp32.
//   R % 4 == 0, ld_xbc % 4 == 0, Di % 64 == 0; 16-byte aligned rows.
// ----------------------------------------------------------------------------------------
constexpr int DSSM_NC = 64;        // channels per CTA
constexpr int DSSM_THREADS = 256;
// dynamic shared memory: the x_proj slices [n_xbc][NB][ld_xbc], W_dt rows [64][R], mbarrier
__host__ __device__ constexpr size_t dssm_smem_bytes(int bpt, int n_xbc, int ld_xbc, int R) {
  return ((size_t)n_xbc * 4 * bpt * ld_xbc + (size_t)DSSM_NC * R) * sizeof(float) + 16;
}

template <int BPT>
__global__ void __launch_bounds__(DSSM_THREADS, BPT == 1 ? 3 : 2)
    decode_ssm_kernel(const float* __restrict__ xbc, long long xbc_stride, int n_xbc, int ld_xbc, int R,
                      const float* __restrict__ w_dt, int ld_dt,
                      const float* __restrict__ dt_bias, const float* __restrict__ A,
                      const __nv_bfloat16* __restrict__ xc, const float* __restrict__ proj, int ld_proj,
                      long long proj_stride, int n_slices, int off_z, float* __restrict__ state,
                      float* __restrict__ y, int Di, int B, DevStatus* status) {
  constexpr int NB = 4 * BPT;   // sequences per CTA
  // Unlike the other kernels, this one reads part of its input before pdl_wait(): the
  // states (written only by this kernel, in an earlier step), A, dt_bias and W_dt.  Its
  // launch implies that the kernel two places before it on the stream has completed (each
  // kernel lets the next one launch only after its own wait, or, the x_proj GEMM before
  // this one, after its launch), so every earlier writer of the states is done; the reads
  // overlap the x_proj GEMM.  What that GEMM and the prep kernel write (the x_proj slices,
  // x and z) is read after the wait.
  extern __shared__ __align__(128) float dssm_sh[];
  float* xs = dssm_sh;                                  // slice k, sequence bl: xs[(k * NB + bl) * ld_xbc]
  float* wsh = xs + (size_t)n_xbc * NB * ld_xbc;        // W_dt row cl: wsh[cl * R]
  uint64_t* bar = reinterpret_cast<uint64_t*>(wsh + DSSM_NC * R);
  __shared__ int ok_sh;
  const int tid = threadIdx.x;
  const int cl = tid & (DSSM_NC - 1), bq = tid / DSSM_NC;
  const int c0 = blockIdx.x * DSSM_NC, b0 = blockIdx.y * NB;
  const int c = c0 + cl;
  const int nb = min(NB, B - b0);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, (uint32_t)(((size_t)n_xbc * nb * ld_xbc + (size_t)DSSM_NC * R) * sizeof(float)));
  }
  __syncthreads();   // the expected byte count is set before any copy can complete
  if (tid < DSSM_NC)
    bulk_load(wsh + tid * R, w_dt + (size_t)(c0 + tid) * ld_dt, (uint32_t)(R * sizeof(float)), bar);
  float h[BPT][16];
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    const int b = b0 + bq * BPT + j;
    if (b < B) {
      const float* hp = state + ((size_t)b * Di + c) * 16;
#pragma unroll
      for (int k = 0; k < 16; k += 4) {
        const float4 v = *reinterpret_cast<const float4*>(hp + k);
        h[j][k] = v.x; h[j][k + 1] = v.y; h[j][k + 2] = v.z; h[j][k + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) h[j][k] = 0.f;
    }
  }
  float a2[16];   // A[c] * log2(e): exp(dt A) = 2^(dt A log2 e)
#pragma unroll
  for (int k = 0; k < 16; k += 4) {
    const float4 v = *reinterpret_cast<const float4*>(A + (size_t)c * 16 + k);
    a2[k] = v.x * 1.4426950408889634f; a2[k + 1] = v.y * 1.4426950408889634f;
    a2[k + 2] = v.z * 1.4426950408889634f; a2[k + 3] = v.w * 1.4426950408889634f;
  }
  const float bias = dt_bias[c];
  pdl_wait();
  pdl_trigger();
  if (tid >= DSSM_NC && tid < DSSM_NC + n_xbc) {
    const int k = tid - DSSM_NC;
    bulk_load(xs + (size_t)k * NB * ld_xbc, xbc + k * xbc_stride + (size_t)b0 * ld_xbc,
              (uint32_t)((size_t)nb * ld_xbc * sizeof(float)), bar);
  }
  float xv[BPT], zv[BPT];
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    const int b = b0 + bq * BPT + j;
    xv[j] = b < B ? __bfloat162float(xc[(size_t)b * Di + c]) : 0.f;
    zv[j] = b < B ? sum_slices<DEC_MAX_IN_SPLIT>(proj + (size_t)b * ld_proj + off_z + c, proj_stride, n_slices) : 0.f;
  }
  if (tid == 0) ok_sh = mbar_wait(bar, 0, nullptr, status, 250) ? 1 : 0;
  __syncthreads();
  if (!ok_sh) return;
  // add the slices in slice order into slice 0 (16-byte pieces of the [nb][ld_xbc] block)
  {
    const int n4 = nb * ld_xbc / 4;
    const size_t sstride = (size_t)NB * ld_xbc;
    for (int i = tid; i < n4; i += DSSM_THREADS) {
      float4 acc = reinterpret_cast<const float4*>(xs)[i];
      for (int k = 1; k < n_xbc; ++k) {
        const float4 v = reinterpret_cast<const float4*>(xs + k * sstride)[i];
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      reinterpret_cast<float4*>(xs)[i] = acc;
    }
  }
  __syncthreads();
  // dt_low . W_dt[c] for the thread's sequences (the warp's lanes share the sequences, so
  // the dt_low reads are broadcasts)
  float dt[BPT], dtx[BPT], yv[2][BPT];
  {
    float acc[BPT][2];
#pragma unroll
    for (int j = 0; j < BPT; ++j) acc[j][0] = acc[j][1] = 0.f;
    const float* wr = wsh + cl * R;
#pragma unroll 2
    for (int r = 0; r < R; r += 4) {
      const float4 w = *reinterpret_cast<const float4*>(wr + r);
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        const float4 d = *reinterpret_cast<const float4*>(xs + (bq * BPT + j) * ld_xbc + r);
        acc[j][0] = fmaf(d.x, w.x, acc[j][0]);
        acc[j][1] = fmaf(d.y, w.y, acc[j][1]);
        acc[j][0] = fmaf(d.z, w.z, acc[j][0]);
        acc[j][1] = fmaf(d.w, w.w, acc[j][1]);
      }
    }
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      dt[j] = softplus_f(acc[j][0] + acc[j][1] + bias);
      dtx[j] = dt[j] * xv[j];
      yv[0][j] = yv[1][j] = 0.f;
    }
  }
#pragma unroll
  for (int k = 0; k < 16; k += 4) {
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      const float* row = xs + (bq * BPT + j) * ld_xbc + R;
      const float4 b4 = *reinterpret_cast<const float4*>(row + k);
      const float4 c4 = *reinterpret_cast<const float4*>(row + 16 + k);
      const float bv[4] = {b4.x, b4.y, b4.z, b4.w}, cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int s = k + e;
        h[j][s] = fmaf(ex2_approx(dt[j] * a2[s]), h[j][s], dtx[j] * bv[e]);
        yv[s & 1][j] = fmaf(cv[e], h[j][s], yv[s & 1][j]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    const int b = b0 + bq * BPT + j;
    if (b >= B) continue;
    float* hp = state + ((size_t)b * Di + c) * 16;
#pragma unroll
    for (int k = 0; k < 16; k += 4) *reinterpret_cast<float4*>(hp + k) = make_float4(h[j][k], h[j][k + 1], h[j][k + 2], h[j][k + 3]);
    y[(size_t)b * Di + c] = (yv[0][j] + yv[1][j]) * silu_f(zv[j]);
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

// The split-K sum of a decode projection with its residual, followed in the same pass by the
// RMSNorm of the result (the input norm of the block's next sublayer), one CTA per row and one
// 16-byte piece of the row per thread (blockDim.x * 4 >= d), the slices' loads 16 at a time:
//   out_sum[r, :]  = bf16(residual[r, :] + the slices in slice order), exactly as
//                    splitk_reduce_kernel stores it;
//   out_norm[r, :] = bf16(s / sqrt(mean(s^2) + eps) * gain) with s = out_sum[r, :] as stored,
//                    as rmsnorm_kernel computes it from the stored row.
// d % 4 == 0, d <= 4096.
constexpr int SNORM_MAX_D = 4096;
__global__ void __launch_bounds__(1024)
    splitk_sum_rmsnorm_kernel(const float* __restrict__ part, int n_split, long long stride, int d,
                              const __nv_bfloat16* __restrict__ residual, __nv_bfloat16* __restrict__ out_sum,
                              const float* __restrict__ gain, float eps, __nv_bfloat16* __restrict__ out_norm) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  const int c = threadIdx.x * 4;
  const size_t i = (size_t)blockIdx.x * d + c;
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (c < d) {
    __nv_bfloat162 r0, r1;
    if (residual != nullptr) {
      r0 = *reinterpret_cast<const __nv_bfloat162*>(residual + i);
      r1 = *reinterpret_cast<const __nv_bfloat162*>(residual + i + 2);
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < n_split; s0 += 16) {
      float4 q[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)
        q[j] = s0 + j < n_split ? *reinterpret_cast<const float4*>(part + (size_t)(s0 + j) * stride + i)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        acc.x += q[j].x; acc.y += q[j].y; acc.z += q[j].z; acc.w += q[j].w;
      }
    }
    if (residual != nullptr) {
      acc.x += __low2float(r0); acc.y += __high2float(r0); acc.z += __low2float(r1); acc.w += __high2float(r1);
    }
    const uint32_t p0 = pack_bf16x2(acc.x, acc.y), p1 = pack_bf16x2(acc.z, acc.w);
    *reinterpret_cast<uint2*>(out_sum + i) = make_uint2(p0, p1);
    const __nv_bfloat162 b0 = *reinterpret_cast<const __nv_bfloat162*>(&p0);
    const __nv_bfloat162 b1 = *reinterpret_cast<const __nv_bfloat162*>(&p1);
    v = make_float4(__low2float(b0), __high2float(b0), __low2float(b1), __high2float(b1));
  }
  const float ss = block_sum_256(v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w, red);
  const float r = 1.f / sqrtf(ss / (float)d + eps);
  if (c < d) {
    const float4 g = *reinterpret_cast<const float4*>(gain + c);
    *reinterpret_cast<uint2*>(out_norm + i) =
        make_uint2(pack_bf16x2(v.x * r * g.x, v.y * r * g.y), pack_bf16x2(v.z * r * g.z, v.w * r * g.w));
  }
}

// The same, one warp per row (8 rows per 256-thread CTA), the row held in registers between
// the sum of squares and the store: for many rows of up to 4096 elements, where one CTA per
// row leaves each CTA too little work to cover its own memory latency.
constexpr int RMSW_MAXV = 16;   // 16-byte pieces per lane: d <= 32 * 8 * 16 = 4096
__global__ void __launch_bounds__(256)
    rmsnorm_warp_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ gain, int rows, int d,
                        float eps, __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const __nv_bfloat16* xr = x + row * d;
  uint4 v[RMSW_MAXV];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < RMSW_MAXV; ++k) {
    const int c = (lane + 32 * k) * 8;
    if (c < d) {
      v[k] = *reinterpret_cast<const uint4*>(xr + c);
      float f[8];
      unpack8(v[k], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += f[e] * f[e];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = 1.f / sqrtf(ss / (float)d + eps);
#pragma unroll
  for (int k = 0; k < RMSW_MAXV; ++k) {
    const int c = (lane + 32 * k) * 8;
    if (c < d) {
      float f[8];
      unpack8(v[k], f);
      const float4 g0 = *reinterpret_cast<const float4*>(gain + c), g1 = *reinterpret_cast<const float4*>(gain + c + 4);
      *reinterpret_cast<uint4*>(out + row * d + c) =
          make_uint4(pack_bf16x2(f[0] * r * g0.x, f[1] * r * g0.y), pack_bf16x2(f[2] * r * g0.z, f[3] * r * g0.w),
                     pack_bf16x2(f[4] * r * g1.x, f[5] * r * g1.y), pack_bf16x2(f[6] * r * g1.z, f[7] * r * g1.w));
    }
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

// The meta positions' K/V of a precomputed prefix ([M, Hkv*64] fp16 each, the same for every
// sequence) copied into rows 0..M-1 of each sequence's prefill view [B, Lmax, Hkv*64] and,
// when meta_k is set, into an SWA cache's meta rows [B, M, Hkv*64].  One 16-byte piece per
// thread; row_vec pieces per position.
__global__ void __launch_bounds__(256)
    prefix_kv_kernel(const __half* __restrict__ pk, const __half* __restrict__ pv, int B, int M, int row_vec,
                     __half* __restrict__ vk, __half* __restrict__ vv, int Lmax, __half* __restrict__ mk,
                     __half* __restrict__ mv) {
  pdl_wait();
  pdl_trigger();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)B * M * row_vec) return;
  const int q = (int)(i % row_vec);
  const long long br = i / row_vec;
  const int r = (int)(br % M);
  const int b = (int)(br / M);
  const size_t src = ((size_t)r * row_vec + q) * 8;
  const uint4 kq = *reinterpret_cast<const uint4*>(pk + src);
  const uint4 vq = *reinterpret_cast<const uint4*>(pv + src);
  const size_t dv = (((size_t)b * Lmax + r) * row_vec + q) * 8;
  *reinterpret_cast<uint4*>(vk + dv) = kq;
  *reinterpret_cast<uint4*>(vv + dv) = vq;
  if (mk != nullptr) {
    const size_t dm = (((size_t)b * M + r) * row_vec + q) * 8;
    *reinterpret_cast<uint4*>(mk + dm) = kq;
    *reinterpret_cast<uint4*>(mv + dm) = vq;
  }
}

// SwiGLU of a decode FFN's gate/up projection: act[r, f] = SiLU(g) * u, with g and u the
// sums, in slice order, of n_split fp32 slices [rows, 2F] whose columns interleave gate and
// up in blocks of 32 (gate f at column 64 (f / 32) + f % 32, up 32 columns later); fp16 out.
__global__ void __launch_bounds__(256)
    swiglu_slices_kernel(const float* __restrict__ part, int n_split, long long stride, int rows, int F,
                         __half* __restrict__ act, DevStatus* status) {
  pdl_wait();
  pdl_trigger();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)rows * F) return;
  const int r = (int)(i / F), f = (int)(i % F);
  const size_t gc = (size_t)r * 2 * F + (size_t)(f >> 5) * 64 + (f & 31);
  float g = 0.f, u = 0.f;
  for (int s = 0; s < n_split; ++s) {
    g += part[(size_t)s * stride + gc];
    u += part[(size_t)s * stride + gc + 32];
  }
  const float a[1] = {silu_f(g) * u};
  f16_range_guard<1>(a, status, 240);
  act[i] = __float2half_rn(a[0]);
}

// Fixed-order sum of split-K partial slices: out[i] = sum_s part[s*stride + i] (+ residual),
// as fp32 or bf16; n is a multiple of 4.  The order never changes, so results are
// identical from run to run.
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int n_split, long long stride, int n,
                                     const __nv_bfloat16* __restrict__ residual, void* __restrict__ out,
                                     int out_bf16) {
  pdl_wait();
  pdl_trigger();
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= n) return;
  // slices in order, 8 loads in flight at a time (a runtime-bounded loop would wait for each)
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < n_split; s0 += 8) {
    float4 q[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      q[k] = s0 + k < n_split ? *reinterpret_cast<const float4*>(part + (size_t)(s0 + k) * stride + i)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      acc.x += q[k].x; acc.y += q[k].y; acc.z += q[k].z; acc.w += q[k].w;
    }
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
}

// ---------------------------------------------------------------------------------------
// L2 prefetch of read-only ranges (weights a later kernel of the same step streams).  One
// thread per 32 KB chunk issues a bulk prefetch and exits: the copy engine brings the chunk
// into L2 while the latency-bound kernels before its consumer run.  A hint only: nothing
// waits for it, and a range's last partial 16 bytes are not prefetched.
// ---------------------------------------------------------------------------------------
constexpr int L2PF_MAX_RANGES = 8;
constexpr unsigned L2PF_CHUNK = 32768;
constexpr int L2PF_THREADS = 128;
struct L2Ranges {
  const char* ptr[L2PF_MAX_RANGES];
  unsigned long long bytes[L2PF_MAX_RANGES];
  int n;
};

__global__ void __launch_bounds__(L2PF_THREADS) l2_prefetch_kernel(L2Ranges r) {
  long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long stride = (long long)gridDim.x * blockDim.x;
  long long first = 0;   // chunk index of range k's first chunk
  for (int k = 0; k < r.n; ++k) {
    const long long nch = (long long)((r.bytes[k] + L2PF_CHUNK - 1) / L2PF_CHUNK);
    for (; g < first + nch; g += stride) {
      const unsigned long long off = (unsigned long long)(g - first) * L2PF_CHUNK;
      const unsigned long long left = r.bytes[k] - off;
      const unsigned size = (unsigned)(left < L2PF_CHUNK ? left : L2PF_CHUNK) & ~15u;
      if (size > 0)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(r.ptr[k] + off), "r"(size) : "memory");
    }
    first += nch;
  }
}

}  // namespace hymba
