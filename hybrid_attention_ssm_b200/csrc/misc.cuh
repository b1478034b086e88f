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
// u = 1/2 [ g_attn * rms(O) ; g_ssm * rms(y * SiLU(z)) ], one row per CTA (256 threads);
// z == nullptr means y is already gated.  O fp32 [rows, ld_o] (attn_w columns); y [rows,
// ld_y] bf16 or fp32; z bf16 [rows, ld_z] (di columns) -> u fp16 [rows, ld_u].  fp16 holds
// the normalised values with 8x finer rounding than bf16 and cannot overflow: after the
// RMSNorm |value| <= sqrt(width) * |gain| / 2.  Widths are multiples of 8.
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ void load8(const float* p, float* f) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f) {
  unpack8(*reinterpret_cast<const uint4*>(p), f);
}
constexpr int NORM_ROWS = 2;          // rows per CTA, 128 threads each
constexpr int NORM_MAXO = 2;          // 8-element chunks of O per thread (attn_w <= 2048)
constexpr int NORM_MAXY = 4;          // 8-element chunks of y per thread (d_inner <= 4096)

template <typename YT>
__global__ void __launch_bounds__(128 * NORM_ROWS)
    branch_norm_avg_kernel(const float* __restrict__ O, int ld_o, int attn_w, const YT* __restrict__ y, int ld_y,
                           const __nv_bfloat16* __restrict__ z, int ld_z, int di, const float* __restrict__ g_attn,
                           const float* __restrict__ g_ssm, float eps, __half* __restrict__ u, int ld_u, int rows) {
  __shared__ float red[NORM_ROWS][4][2];
  const int sub = threadIdx.x >> 7;                 // row within the CTA
  const int t = threadIdx.x & 127;
  const int wr = t >> 5, ln = t & 31;
  const size_t row = (size_t)blockIdx.x * NORM_ROWS + sub;
  const bool live = row < (size_t)rows;
  const float* o_r = O + row * ld_o;
  const YT* y_r = y + row * ld_y;
  const __nv_bfloat16* z_r = z != nullptr ? z + row * ld_z : nullptr;
  __half* u_r = u + row * ld_u;
  // the whole row in registers: every load is issued before the first use
  float fo[NORM_MAXO][8], fy[NORM_MAXY][8];
  uint4 rz[NORM_MAXY];
#pragma unroll
  for (int k = 0; k < NORM_MAXO; ++k) {
    const int c = (t + k * 128) * 8;
    if (live && c < attn_w) load8(o_r + c, fo[k]);
  }
#pragma unroll
  for (int k = 0; k < NORM_MAXY; ++k) {
    const int c = (t + k * 128) * 8;
    if (live && c < di) {
      load8(y_r + c, fy[k]);
      if (z != nullptr) rz[k] = *reinterpret_cast<const uint4*>(z_r + c);
    }
  }
  float sa = 0.f, ss = 0.f;
#pragma unroll
  for (int k = 0; k < NORM_MAXY; ++k) {
    const int c = (t + k * 128) * 8;
    if (live && c < di && z != nullptr) {
      float fz[8];
      unpack8(rz[k], fz);
#pragma unroll
      for (int e = 0; e < 8; ++e) fy[k][e] *= silu_f(fz[e]);
    }
  }
#pragma unroll
  for (int k = 0; k < NORM_MAXO; ++k) {
    const int c = (t + k * 128) * 8;
    if (live && c < attn_w)
#pragma unroll
      for (int e = 0; e < 8; ++e) sa += fo[k][e] * fo[k][e];
  }
#pragma unroll
  for (int k = 0; k < NORM_MAXY; ++k) {
    const int c = (t + k * 128) * 8;
    if (live && c < di)
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += fy[k][e] * fy[k][e];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sa += __shfl_xor_sync(0xffffffffu, sa, o);
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  if (ln == 0) {
    red[sub][wr][0] = sa;
    red[sub][wr][1] = ss;
  }
  __syncthreads();
  sa = red[sub][0][0] + red[sub][1][0] + red[sub][2][0] + red[sub][3][0];
  ss = red[sub][0][1] + red[sub][1][1] + red[sub][2][1] + red[sub][3][1];
  if (!live) return;
  const float ra = 0.5f / sqrtf(sa / (float)attn_w + eps);
  const float rs = 0.5f / sqrtf(ss / (float)di + eps);
#pragma unroll
  for (int k = 0; k < NORM_MAXO; ++k) {
    const int c = (t + k * 128) * 8;
    if (c < attn_w) {
      float g[8];
      load8(g_attn + c, g);
      uint32_t pk[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) pk[e / 2] = pack_f16x2(fo[k][e] * ra * g[e], fo[k][e + 1] * ra * g[e + 1]);
      *reinterpret_cast<uint4*>(u_r + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
#pragma unroll
  for (int k = 0; k < NORM_MAXY; ++k) {
    const int c = (t + k * 128) * 8;
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

// ----------------------------------------------------------------------------------------
// SWA cache after prefill: meta rows [0, M) -> meta_k/v; rows [max(M, T-W), T) -> ring slot
// (pos - M) mod W.  view_k/v [B, Lmax, Hkv*D]; meta [B, M, Hkv*D]; ring [B, W, Hkv*D].
// ----------------------------------------------------------------------------------------
__global__ void swa_cache_finalize_kernel(const __half* __restrict__ vk, const __half* __restrict__ vv,
                                          int Lmax, int T, int M, int W, int row_elems,
                                          __half* __restrict__ meta_k, __half* __restrict__ meta_v,
                                          __half* __restrict__ ring_k, __half* __restrict__ ring_v) {
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
// Decode attention, split-K over keys.  CTA = (split, kv head g, sequence b), 128 threads,
// 128 keys per split.  Keys: meta [0, M) then window positions [max(M, p-W+1), p] for SWA
// (ring slot (pos-M) mod W), or [0, p] for a global cache.  The query heads of group g
// (Hq/Hkv of them) share the K/V reads.
// An own/producer layer takes k, v of the new token from the in_proj output, applies RoPE
// to k, writes it into the cache (split 0 only) and uses the in-register copy for position
// p, so no split reads a slot another split is writing.  A consumer reads everything from
// the cache (its producer already wrote position p).
// Partial results per (b, h, split): m (log2 domain), l, o[64] unnormalised.
// ----------------------------------------------------------------------------------------
struct DecAttnParams {
  const float* proj;          // [B, ld_proj] fp32: q at 0, k at q_w, v at q_w + kv_w (when present)
  int ld_proj;
  int Hq, Hkv, M, W, is_global, write_kv, p, n_keys, n_splits;
  __half *meta_k, *meta_v, *ring_k, *ring_v;  // SWA cache (fp16)
  __half *full_k, *full_v;                    // global cache [B, Lmax, Hkv*D] (fp16)
  int Lmax;
  float scale_log2;
  double rope_theta[32];
  float* part;                // [B, Hq, n_splits, 66]
};

constexpr int DEC_KT = 128;
constexpr int DEC_MAXG = 6;     // max query heads per KV head

__device__ __forceinline__ void rope64_smem(float* v, int pos, const double* theta) {
  // rotate pairs (v[j], v[j+32]) of a 64-vector in place; called by 32 threads (j = lane)
  const int j = threadIdx.x & 31;
  double a = (double)pos * theta[j];
  a -= 6.283185307179586 * rint(a * 0.15915494309189535);
  float s, c;
  sincosf((float)a, &s, &c);
  const float x1 = v[j], x2 = v[j + 32];
  v[j] = x1 * c - x2 * s;
  v[j + 32] = x2 * c + x1 * s;
}

__global__ void __launch_bounds__(128) decode_attn_kernel(const __grid_constant__ DecAttnParams p) {
  __shared__ __align__(16) __half ks[DEC_KT][72];   // padded rows (144 B)
  __shared__ __align__(16) __half vs[DEC_KT][64];
  __shared__ __align__(16) float qs[DEC_MAXG][64];
  __shared__ __align__(16) float knew[64], vnew[64];
  __shared__ __align__(16) float ps[DEC_MAXG][DEC_KT];
  __shared__ float red[DEC_MAXG][4];
  __shared__ __align__(16) float opart[4][DEC_MAXG][64];
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.Hq / p.Hkv;
  const int kvw = p.Hkv * 64;
  const int k_first = split * DEC_KT;
  const int nk = min(DEC_KT, p.n_keys - k_first);
  const int n_meta_keys = p.is_global ? 0 : p.M;
  const int win0 = p.is_global ? 0 : max(p.M, p.p - p.W + 1);

  // key index -> (cache row pointer) ; position p is the last key
  auto key_row = [&](int kidx, bool is_v) -> const __half* {
    if (p.is_global) {
      const __half* base = is_v ? p.full_v : p.full_k;
      return base + ((size_t)b * p.Lmax + kidx) * kvw + g * 64;
    }
    if (kidx < n_meta_keys) {
      const __half* base = is_v ? p.meta_v : p.meta_k;
      return base + ((size_t)b * p.M + kidx) * kvw + g * 64;
    }
    const int pos = win0 + (kidx - n_meta_keys);
    const int slot = (pos - p.M) % p.W;
    const __half* base = is_v ? p.ring_v : p.ring_k;
    return base + ((size_t)b * p.W + slot) * kvw + g * 64;
  };
  const bool last_is_new = p.write_kv != 0;   // position p comes from registers

  // async K/V tile loads (16 B pieces); the new token's row is filled later
  for (int i = tid; i < nk * 16; i += 128) {
    const int kk = i >> 4, piece = i & 15;
    const int kidx = k_first + kk;
    if (last_is_new && kidx == p.n_keys - 1) continue;
    if (piece < 8) cp_async16(&ks[kk][piece * 8], key_row(kidx, false) + piece * 8, 16);
    else cp_async16(&vs[kk][(piece - 8) * 8], key_row(kidx, true) + (piece - 8) * 8, 16);
  }
  cp_async_commit();

  // queries of this group with RoPE at position p, pre-scaled
  const float* pr = p.proj + (size_t)b * p.ld_proj;
  for (int i = tid; i < G * 64; i += 128) {
    const int hh = i >> 6, d = i & 63;
    qs[hh][d] = pr[(g * G + hh) * 64 + d];
  }
  if (last_is_new && tid < 64) {
    knew[tid] = pr[p.Hq * 64 + g * 64 + tid];
    vnew[tid] = pr[p.Hq * 64 + kvw + g * 64 + tid];
  }
  __syncthreads();
  for (int i = warp; i < G + (last_is_new ? 1 : 0); i += 4) rope64_smem(i < G ? qs[i] : knew, p.p, p.rope_theta);
  __syncthreads();
  for (int i = tid; i < G * 64; i += 128) qs[i >> 6][i & 63] *= p.scale_log2;
  if (last_is_new && split == 0 && tid < 64) {
    __half *dk, *dv;
    if (p.is_global) {
      dk = p.full_k + ((size_t)b * p.Lmax + p.p) * kvw + g * 64;
      dv = p.full_v + ((size_t)b * p.Lmax + p.p) * kvw + g * 64;
    } else {
      const int slot = (p.p - p.M) % p.W;
      dk = p.ring_k + ((size_t)b * p.W + slot) * kvw + g * 64;
      dv = p.ring_v + ((size_t)b * p.W + slot) * kvw + g * 64;
    }
    dk[tid] = __float2half_rn(knew[tid]);
    dv[tid] = __float2half_rn(vnew[tid]);
  }
  cp_async_wait<0>();
  __syncthreads();
  // the new token's row (rounded to fp16 like the cached copy)
  if (last_is_new && p.n_keys - 1 >= k_first && p.n_keys - 1 < k_first + nk && tid < 64) {
    const int kk = p.n_keys - 1 - k_first;
    ks[kk][tid] = __float2half_rn(knew[tid]);
    vs[kk][tid] = __float2half_rn(vnew[tid]);
  }
  __syncthreads();

  // scores: thread = key
  float sc[DEC_MAXG];
  {
    const int kk = tid;
    float kf[64];
    if (kk < nk) {
#pragma unroll
      for (int d = 0; d < 64; d += 8) unpack8h(*reinterpret_cast<const uint4*>(&ks[kk][d]), kf + d);
    }
#pragma unroll
    for (int hh = 0; hh < DEC_MAXG; ++hh) {
      float a = -1e30f;
      if (hh < G && kk < nk) {
        a = 0.f;
#pragma unroll
        for (int d = 0; d < 64; ++d) a = fmaf(qs[hh][d], kf[d], a);
      }
      sc[hh] = a;
    }
  }
  // per-head max and exp over the 128 keys
  float mh[DEC_MAXG];
#pragma unroll
  for (int hh = 0; hh < DEC_MAXG; ++hh) {
    float m = sc[hh];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[hh][warp] = m;
  }
  __syncthreads();
#pragma unroll
  for (int hh = 0; hh < DEC_MAXG; ++hh)
    mh[hh] = fmaxf(fmaxf(red[hh][0], red[hh][1]), fmaxf(red[hh][2], red[hh][3]));
#pragma unroll
  for (int hh = 0; hh < DEC_MAXG; ++hh) {
    const float e = (tid < nk && hh < G) ? exp2f(sc[hh] - mh[hh]) : 0.f;
    ps[hh][tid] = e;
  }
  __syncthreads();
  // PV: thread = (dim pair, key quarter)
  {
    const int dp = lane, kq = warp;
    float acc[DEC_MAXG][2];
#pragma unroll
    for (int hh = 0; hh < DEC_MAXG; ++hh) acc[hh][0] = acc[hh][1] = 0.f;
    for (int kk = kq * 32; kk < kq * 32 + 32; ++kk) {
      const __half2 v2 = *reinterpret_cast<const __half2*>(&vs[kk][dp * 2]);
      const float v0 = __low2float(v2), v1 = __high2float(v2);
#pragma unroll
      for (int hh = 0; hh < DEC_MAXG; ++hh) {
        const float pv = ps[hh][kk];
        acc[hh][0] = fmaf(pv, v0, acc[hh][0]);
        acc[hh][1] = fmaf(pv, v1, acc[hh][1]);
      }
    }
#pragma unroll
    for (int hh = 0; hh < DEC_MAXG; ++hh) {
      opart[kq][hh][dp * 2] = acc[hh][0];
      opart[kq][hh][dp * 2 + 1] = acc[hh][1];
    }
  }
  // row sums
  float lsum[DEC_MAXG];
#pragma unroll
  for (int hh = 0; hh < DEC_MAXG; ++hh) {
    float v = ps[hh][tid];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    lsum[hh] = v;
  }
  __syncthreads();
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < DEC_MAXG; ++hh) red[hh][warp] = lsum[hh];
  }
  __syncthreads();
  for (int i = tid; i < G * 64; i += 128) {
    const int hh = i >> 6, d = i & 63;
    const float o = opart[0][hh][d] + opart[1][hh][d] + opart[2][hh][d] + opart[3][hh][d];
    float* dst = p.part + (((size_t)b * p.Hq + g * G + hh) * p.n_splits + split) * 66;
    dst[2 + d] = o;
    if (d == 0) {
      dst[0] = mh[hh];
      dst[1] = red[hh][0] + red[hh][1] + red[hh][2] + red[hh][3];
    }
  }
}

// merge the split partials of one (b, h): O = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i
__global__ void decode_attn_combine_kernel(const float* __restrict__ part, int n_splits, int Hq,
                                           float* __restrict__ out, int ld_out) {
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
// decode conv step: window [state(3), x_new] -> xc = SiLU(b + w . window); state shifts.
// x from proj [B, ld_proj] fp32 at column off_x; xc [B, Di] bf16; state [B, Di, 3] fp32 in place.
// ----------------------------------------------------------------------------------------
__global__ void decode_conv_kernel(const float* __restrict__ proj, int ld_proj, int off_x, int Di,
                                   const float* __restrict__ w, const float* __restrict__ bias,
                                   float* __restrict__ state, __nv_bfloat16* __restrict__ xc, int B) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * Di) return;
  const int b = i / Di, c = i % Di;
  float* st = state + (size_t)i * 3;
  const float x0 = st[0], x1 = st[1], x2 = st[2];
  const float xn = proj[(size_t)b * ld_proj + off_x + c];
  const float4 wv = *reinterpret_cast<const float4*>(w + (size_t)c * 4);
  const float acc = bias[c] + wv.x * x0 + wv.y * x1 + wv.z * x2 + wv.w * xn;
  xc[i] = __float2bfloat16_rn(silu_f(acc));
  st[0] = x1;
  st[1] = x2;
  st[2] = xn;
}

// ----------------------------------------------------------------------------------------
// decode SSM step: dt = softplus(dt_low . W_dt[c] + bias), h = exp(dt A) h + dt B x,
// y = (C . h) * SiLU(z).  CTA = 16 channels x 16 states of one sequence.
//   xbc [B, ld_xbc] fp32: dt_low at 0..R-1, B at R.., C at R+16..; W_dt [Di, ld_dt] fp32;
//   xc [B, Di] bf16; z from proj at column off_z; state [B, Di, 16] in place; y [B, Di] fp32.
// ----------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    decode_ssm_kernel(const float* __restrict__ xbc, int ld_xbc, int R, const float* __restrict__ w_dt, int ld_dt,
                      const float* __restrict__ dt_bias, const float* __restrict__ A,
                      const __nv_bfloat16* __restrict__ xc, const float* __restrict__ proj, int ld_proj,
                      int off_z, float* __restrict__ state, float* __restrict__ y, int Di) {
  __shared__ float dl[256];
  __shared__ float bcs[32];
  const int b = blockIdx.y;
  const int tid = threadIdx.x;
  const int cl = tid >> 4, s = tid & 15;
  const int c = blockIdx.x * 16 + cl;
  const float* row = xbc + (size_t)b * ld_xbc;
  for (int i = tid; i < R; i += 256) dl[i] = row[i];
  if (tid < 32) bcs[tid] = row[R + tid];
  __syncthreads();
  float acc = 0.f;
  const float* wr = w_dt + (size_t)c * ld_dt;
  for (int r = s; r < R; r += 16) acc = fmaf(dl[r], wr[r], acc);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  const float dt = softplus_f(acc + dt_bias[c]);
  const float x = __bfloat162float(xc[(size_t)b * Di + c]);
  float* hp = state + ((size_t)b * Di + c) * 16 + s;
  const float a = expf(dt * A[(size_t)c * 16 + s]);
  const float hn = fmaf(a, *hp, dt * bcs[s] * x);
  *hp = hn;
  float yv = bcs[16 + s] * hn;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) yv += __shfl_xor_sync(0xffffffffu, yv, o);
  if (s == 0) {
    const float zz = proj[(size_t)b * ld_proj + off_z + c];
    y[(size_t)b * Di + c] = yv * silu_f(zz);
  }
}

// RoPE angles: tab[pos][j] = (cos, sin) of pos * base^(-2j/64), the angle reduced mod 2*pi
// in double precision before the fp32 sincos.
struct RopeThetas {
  double t[32];
};
__global__ void rope_table_kernel(float2* __restrict__ tab, int n_pos, const __grid_constant__ RopeThetas th) {
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
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float v = acc[i];
  if (res != nullptr) v += __bfloat162float(res[i]);
  out[i] = __float2bfloat16_rn(v);
}

}  // namespace hymba
