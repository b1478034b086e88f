// SSM branch kernels (prefill): causal depthwise conv1d + SiLU, and the selective scan.
#pragma once
#include "common.cuh"

namespace hymba {

// ----------------------------------------------------------------------------------------
// conv1d (kernel width 4) + SiLU over time, per channel.
//   x      [B*T, ld_x] bf16, channel c at column c (the x part of the in_proj output)
//   xc     [B*T, Di]   bf16 row-major (A operand of x_proj)
//   xcT    [B, Di, Tp] bf16 time-major (input of the scan), row stride Tp (multiple of 8)
//   state  [B, Di, 3]  fp32: the last 3 inputs x[T-3..T-1] (zero before the start)
// CTA: 64 channels x 64 time steps, 256 threads.
// ----------------------------------------------------------------------------------------
constexpr int CONV_K = 4;
constexpr int CONV_RUN = 8;      // time steps per thread

// Thread = (channel pair, run of 8 time steps): the 3-step history stays in registers,
// loads and row-major stores are 4 bytes per lane (128 B per warp), the time-major store
// is 16 contiguous bytes per channel.
__global__ void __launch_bounds__(256)
    conv1d_silu_kernel(const __nv_bfloat16* __restrict__ x, int ld_x, const float* __restrict__ w,
                       const float* __restrict__ bias, __nv_bfloat16* __restrict__ xc,
                       __nv_bfloat16* __restrict__ xcT, float* __restrict__ state, int T, int Tp, int Di) {
  const int pairs = Di >> 1;
  const int gid = blockIdx.x * blockDim.x + threadIdx.x;
  const int cp = gid % pairs;
  const int run = gid / pairs;
  const int b = blockIdx.y;
  const int t0 = run * CONV_RUN;
  if (t0 >= T) return;
  const int c = cp * 2;
  const float4 w0 = *reinterpret_cast<const float4*>(w + (size_t)c * 4);
  const float4 w1 = *reinterpret_cast<const float4*>(w + (size_t)(c + 1) * 4);
  const float b0 = bias[c], b1 = bias[c + 1];
  const __nv_bfloat16* xb = x + (size_t)b * T * ld_x + c;
  float h0[3], h1[3];          // x[t-3], x[t-2], x[t-1] of both channels
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int t = t0 - 3 + k;
    float2 f = make_float2(0.f, 0.f);
    if (t >= 0) f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(xb + (size_t)t * ld_x));
    h0[k] = f.x;
    h1[k] = f.y;
  }
  const int n = min(CONV_RUN, T - t0);
  float2 xv[CONV_RUN];
#pragma unroll
  for (int i = 0; i < CONV_RUN; ++i)
    if (i < n) xv[i] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(xb + (size_t)(t0 + i) * ld_x));
  __align__(16) __nv_bfloat16 o0[CONV_RUN], o1[CONV_RUN];
#pragma unroll
  for (int i = 0; i < CONV_RUN; ++i) {
    if (i < n) {
      const float a0 = b0 + w0.x * h0[0] + w0.y * h0[1] + w0.z * h0[2] + w0.w * xv[i].x;
      const float a1 = b1 + w1.x * h1[0] + w1.y * h1[1] + w1.z * h1[2] + w1.w * xv[i].y;
      h0[0] = h0[1]; h0[1] = h0[2]; h0[2] = xv[i].x;
      h1[0] = h1[1]; h1[1] = h1[2]; h1[2] = xv[i].y;
      const __nv_bfloat162 y2 = __floats2bfloat162_rn(silu_f(a0), silu_f(a1));
      *reinterpret_cast<__nv_bfloat162*>(xc + ((size_t)b * T + t0 + i) * Di + c) = y2;
      o0[i] = y2.x;
      o1[i] = y2.y;
    } else {
      o0[i] = __float2bfloat16_rn(0.f);
      o1[i] = __float2bfloat16_rn(0.f);
    }
  }
  __nv_bfloat16* d0 = xcT + ((size_t)b * Di + c) * Tp + t0;
  __nv_bfloat16* d1 = d0 + Tp;
  if (n == CONV_RUN) {
#pragma unroll
    for (int i = 0; i < CONV_RUN; i += 8) {
      *reinterpret_cast<uint4*>(d0 + i) = *reinterpret_cast<const uint4*>(o0 + i);
      *reinterpret_cast<uint4*>(d1 + i) = *reinterpret_cast<const uint4*>(o1 + i);
    }
  } else {
    for (int i = 0; i < n; ++i) {
      d0[i] = o0[i];
      d1[i] = o1[i];
    }
  }
  // conv state: the last 3 inputs x[T-3..T-1] (zero when T < 3), from the last run
  if (t0 + n == T) {
    float* s0 = state + ((size_t)b * Di + c) * 3;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const bool valid = T - 3 + k >= 0;
      s0[k] = valid ? h0[k] : 0.f;
      s0[3 + k] = valid ? h1[k] : 0.f;
    }
  }
}

// ----------------------------------------------------------------------------------------
// Selective scan, time-sequential per (channel, state) thread.
//   h_t = exp(delta_t * A[c,s]) h_{t-1} + delta_t * B_t[s] * x_t ;  y_t = sum_s C_t[s] h_t[s]
// CTA = 8 channels x 16 states.  The fp32 state stays in a register for the whole
// sequence.  Inputs go through shared memory in chunks of 64 steps, 3 stages deep: delta,
// delta*x (formed once per step and channel while staging) and B/C transposed to
// [state][t] so each thread reads 4 steps per 128-bit load.  Each thread writes its
// C_t[s] h_t[s] terms to a swizzled buffer; after the chunk, one thread per (4 steps,
// channel) sums the 16 states (bank-conflict-free on both sides) and the y rows leave as
// 16-byte stores.
//   xcT [B, Di, Tp] bf16; dT [B, Di, Tp] fp32 (Tp: row stride, multiple of 8; steps at or
//   beyond T read as zero, so delta = 0 leaves the state unchanged); bc [B*T, ld_bc] fp32
//   (B at col 0..15, C at 16..31 of the pointer); A [Di, 16]; y [B*T, Di] bf16 (not gated);
//   state [B, Di, 16].
// ----------------------------------------------------------------------------------------
constexpr int SCAN_CH = 8;            // channels per CTA
constexpr int SCAN_TC = 64;           // time steps per chunk
constexpr int SCAN_NST = 3;           // pipeline stages
constexpr int SCAN_THREADS = SCAN_CH * 16;

struct ScanStage {
  float d[SCAN_CH][SCAN_TC];          // delta
  float dx[SCAN_CH][SCAN_TC];         // delta * x
  float bcT[32][SCAN_TC + 4];         // [state (B 0..15, C 16..31)][t]
};
struct ScanSmem {
  ScanStage st[SCAN_NST];
  float part[SCAN_TC / 4][16][SCAN_CH][4];   // C*h terms: [t/4][state][channel ^ (state&7)][t%4]
  __nv_bfloat16 ys[SCAN_TC][SCAN_CH];
};

__global__ void __launch_bounds__(SCAN_THREADS)
    selective_scan_kernel(const __nv_bfloat16* __restrict__ xcT, const float* __restrict__ dT,
                          const float* __restrict__ bc, int ld_bc, const float* __restrict__ A,
                          __nv_bfloat16* __restrict__ y, float* __restrict__ state, int T, int Tp, int Di) {
  extern __shared__ __align__(16) uint8_t scan_smem_raw[];
  ScanSmem& sm = *reinterpret_cast<ScanSmem*>(scan_smem_raw);
  const int tid = threadIdx.x;
  const int cl = tid >> 4;         // channel within CTA
  const int s = tid & 15;          // state
  const int c0 = blockIdx.x * SCAN_CH;
  const int b = blockIdx.y;
  const int c = c0 + cl;
  const int n_chunks = (T + SCAN_TC - 1) / SCAN_TC;
  const float A2 = A[(size_t)c * 16 + s] * 1.4426950408889634f;   // exp(d*A) = 2^(d*A*log2 e)

  // staging of chunk k through registers: thread -> (channel lch, 4 steps lq*4..) for
  // delta and x, and (row, 16 of B|C) for the B/C rows
  const int lch = tid >> 4, lq = tid & 15;
  float4 rd;
  uint2 rx;
  float rbc[16];
  auto load_chunk = [&](int k) {
    const int t = k * SCAN_TC + lq * 4;
    const size_t row = ((size_t)b * Di + c0 + lch) * Tp;
    rd = make_float4(0.f, 0.f, 0.f, 0.f);
    rx = make_uint2(0u, 0u);
    if (t + 4 <= T) {
      rd = *reinterpret_cast<const float4*>(dT + row + t);
      rx = *reinterpret_cast<const uint2*>(xcT + row + t);
    } else {
      float dd[4] = {0.f, 0.f, 0.f, 0.f};
      __nv_bfloat16 xx[4] = {__float2bfloat16_rn(0.f), __float2bfloat16_rn(0.f), __float2bfloat16_rn(0.f),
                             __float2bfloat16_rn(0.f)};
      for (int e = 0; e < 4; ++e)
        if (t + e < T) {
          dd[e] = dT[row + t + e];
          xx[e] = xcT[row + t + e];
        }
      rd = make_float4(dd[0], dd[1], dd[2], dd[3]);
      rx = *reinterpret_cast<const uint2*>(xx);
    }
    const int brow = tid >> 1, half = (tid & 1) * 16;
    const int tb = k * SCAN_TC + brow;
#pragma unroll
    for (int e = 0; e < 16; e += 4) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (tb < T) v = *reinterpret_cast<const float4*>(bc + ((size_t)b * T + tb) * ld_bc + half + e);
      rbc[e] = v.x; rbc[e + 1] = v.y; rbc[e + 2] = v.z; rbc[e + 3] = v.w;
    }
  };
  auto store_chunk = [&](int k) {
    ScanStage& S = sm.st[k % SCAN_NST];
    const __nv_bfloat16* xh = reinterpret_cast<const __nv_bfloat16*>(&rx);
    *reinterpret_cast<float4*>(&S.d[lch][lq * 4]) = rd;
    *reinterpret_cast<float4*>(&S.dx[lch][lq * 4]) =
        make_float4(rd.x * __bfloat162float(xh[0]), rd.y * __bfloat162float(xh[1]), rd.z * __bfloat162float(xh[2]),
                    rd.w * __bfloat162float(xh[3]));
    const int brow = tid >> 1, half = (tid & 1) * 16;
#pragma unroll
    for (int e = 0; e < 16; ++e) S.bcT[half + e][brow] = rbc[e];
  };

  // prologue: chunks 0 .. NST-2
  for (int k = 0; k < SCAN_NST - 1 && k < n_chunks; ++k) {
    load_chunk(k);
    store_chunk(k);
  }
  float h = 0.f;
  const int sw = s & 7;
  for (int k = 0; k < n_chunks; ++k) {
    const int kn = k + SCAN_NST - 1;
    __syncthreads();                       // chunk k staged; its part/ys buffers free
    if (kn < n_chunks) load_chunk(kn);     // in flight during the compute below
    const ScanStage& S = sm.st[k % SCAN_NST];
#pragma unroll 2
    for (int tt = 0; tt < SCAN_TC; tt += 8) {
      const float4 d0 = *reinterpret_cast<const float4*>(&S.d[cl][tt]);
      const float4 d1 = *reinterpret_cast<const float4*>(&S.d[cl][tt + 4]);
      const float4 q0 = *reinterpret_cast<const float4*>(&S.dx[cl][tt]);
      const float4 q1 = *reinterpret_cast<const float4*>(&S.dx[cl][tt + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&S.bcT[s][tt]);
      const float4 b1 = *reinterpret_cast<const float4*>(&S.bcT[s][tt + 4]);
      const float4 e0 = *reinterpret_cast<const float4*>(&S.bcT[16 + s][tt]);
      const float4 e1 = *reinterpret_cast<const float4*>(&S.bcT[16 + s][tt + 4]);
      const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
      const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      const float cv[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
      float a[8], v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) a[u] = ex2_approx(dv[u] * A2);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        h = fmaf(a[u], h, qv[u] * bv[u]);
        v[u] = cv[u] * h;
      }
      *reinterpret_cast<float4*>(&sm.part[tt >> 2][s][cl ^ sw][0]) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4*>(&sm.part[(tt >> 2) + 1][s][cl ^ sw][0]) = make_float4(v[4], v[5], v[6], v[7]);
    }
    if (kn < n_chunks) store_chunk(kn);
    __syncthreads();
    // sum over the 16 states: thread -> (4 steps tg, channel ch)
    {
      const int tg = tid >> 3, ch = tid & 7;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int st = 0; st < 16; ++st) {
        const float4 q = *reinterpret_cast<const float4*>(&sm.part[tg][st][ch ^ (st & 7)][0]);
        acc.x += q.x; acc.y += q.y; acc.z += q.z; acc.w += q.w;
      }
      sm.ys[tg * 4 + 0][ch] = __float2bfloat16_rn(acc.x);
      sm.ys[tg * 4 + 1][ch] = __float2bfloat16_rn(acc.y);
      sm.ys[tg * 4 + 2][ch] = __float2bfloat16_rn(acc.z);
      sm.ys[tg * 4 + 3][ch] = __float2bfloat16_rn(acc.w);
    }
    __syncthreads();
    if (tid < SCAN_TC) {
      const int t = k * SCAN_TC + tid;
      if (t < T)
        *reinterpret_cast<uint4*>(y + ((size_t)b * T + t) * Di + c0) = *reinterpret_cast<const uint4*>(&sm.ys[tid][0]);
    }
  }
  state[((size_t)b * Di + c) * 16 + s] = h;
}

}  // namespace hymba
