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
// 16 lanes of a warp hold the 16 states of one channel; the sum over states is a
// reduce-scatter through 8 shuffles per 8 time steps.  The fp32 state stays in registers
// for the whole sequence.  Inputs are staged through shared memory in chunks of 64 steps
// (cp.async for the time-major x and delta, register transpose for B/C), 3 stages deep.
//   xcT [B, Di, Tp] bf16; dT [B, Di, Tp] fp32 (Tp: row stride, multiple of 8; steps at or
//   beyond T read as zero, so delta = 0 leaves the state unchanged); bc [B*T, ld_bc] fp32 (B at col 0..15, C at
//   16..31 of the pointer); A [Di, 16]; y [B*T, Di] bf16 (not gated); state [B, Di, 16].
// ----------------------------------------------------------------------------------------
constexpr int SCAN_CH = 8;            // channels per CTA
constexpr int SCAN_TC = 64;           // time steps per chunk
constexpr int SCAN_NST = 3;           // pipeline stages
constexpr int SCAN_THREADS = SCAN_CH * 16;

struct ScanStage {
  __nv_bfloat16 x[SCAN_CH][SCAN_TC];  // 8 x 128 B
  float d[SCAN_CH][SCAN_TC];          // 8 x 256 B
  float bcT[32][SCAN_TC + 4];         // [state (B 0..15, C 16..31)][t]
};

__global__ void __launch_bounds__(SCAN_THREADS)
    selective_scan_kernel(const __nv_bfloat16* __restrict__ xcT, const float* __restrict__ dT,
                          const float* __restrict__ bc, int ld_bc, const float* __restrict__ A,
                          __nv_bfloat16* __restrict__ y, float* __restrict__ state, int T, int Tp, int Di) {
  __shared__ __align__(16) ScanStage st[SCAN_NST];
  __shared__ __align__(16) __nv_bfloat16 ys[SCAN_TC][SCAN_CH];
  const int tid = threadIdx.x;
  const int cl = tid >> 4;         // channel within CTA
  const int s = tid & 15;          // state
  const int c0 = blockIdx.x * SCAN_CH;
  const int b = blockIdx.y;
  const int c = c0 + cl;
  const int n_chunks = (T + SCAN_TC - 1) / SCAN_TC;
  const float A2 = A[(size_t)c * 16 + s] * 1.4426950408889634f;   // exp(d*A) = 2^(d*A*log2 e)

  // async loads of the time-major x / delta rows of chunk k into stage k % NST
  auto load_xd = [&](int k) {
    ScanStage& S = st[k % SCAN_NST];
    const int t0 = k * SCAN_TC;
    // x: 8 channels x 8 pieces of 16 B; delta: 8 channels x 16 pieces
    for (int i = tid; i < SCAN_CH * 24; i += SCAN_THREADS) {
      const int ch = i / 24, piece = i % 24;
      if (piece < 8) {
        const int t = t0 + piece * 8;
        const int nbytes = t >= T ? 0 : min(16, (T - t) * 2);
        const __nv_bfloat16* src = xcT + ((size_t)b * Di + c0 + ch) * Tp + (t >= T ? 0 : t);
        cp_async16(&S.x[ch][piece * 8], src, nbytes);
      } else {
        const int t = t0 + (piece - 8) * 4;
        const int nbytes = t >= T ? 0 : min(16, (T - t) * 4);
        const float* src = dT + ((size_t)b * Di + c0 + ch) * Tp + (t >= T ? 0 : t);
        cp_async16(&S.d[ch][(piece - 8) * 4], src, nbytes);
      }
    }
  };
  // B/C of chunk k: 64 rows x 32 floats, loaded into registers (16 per thread) ...
  float bcr[16];
  auto load_bc = [&](int k) {
    const int t0 = k * SCAN_TC;
    const int row = tid >> 1, half = (tid & 1) * 16;
    const int t = t0 + row;
#pragma unroll
    for (int e = 0; e < 16; e += 4) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < T) v = *reinterpret_cast<const float4*>(bc + ((size_t)b * T + t) * ld_bc + half + e);
      bcr[e] = v.x; bcr[e + 1] = v.y; bcr[e + 2] = v.z; bcr[e + 3] = v.w;
    }
  };
  // ... and stored transposed ([state][t]) into the stage
  auto store_bc = [&](int k) {
    ScanStage& S = st[k % SCAN_NST];
    const int row = tid >> 1, half = (tid & 1) * 16;
#pragma unroll
    for (int e = 0; e < 16; ++e) S.bcT[half + e][row] = bcr[e];
  };

  // prologue: chunks 0 .. NST-2
  for (int k = 0; k < SCAN_NST - 1; ++k) {
    if (k < n_chunks) {
      load_xd(k);
      load_bc(k);
      store_bc(k);
    }
    cp_async_commit();
  }

  float h = 0.f;
  const int l = tid & 15;
  const int my_step = ((l >> 3) & 1) * 4 + ((l >> 2) & 1) * 2 + ((l >> 1) & 1);
  for (int k = 0; k < n_chunks; ++k) {
    const int kn = k + SCAN_NST - 1;
    cp_async_wait<SCAN_NST - 2>();
    __syncthreads();                       // chunk k visible; stage of chunk k-1 free
    if (kn < n_chunks) {
      load_xd(kn);
      load_bc(kn);
    }
    cp_async_commit();
    const ScanStage& S = st[k % SCAN_NST];
    // Software pipeline over the 8 blocks of 8 steps: block q's recurrence runs while the
    // state-sum of block q-1 goes through its shuffles, so the two latency chains overlap.
    float vprev[8];
    auto block_inputs = [&](int tt, float* dv, float* xv, float* bv, float* cv) {
      const uint4 xr = *reinterpret_cast<const uint4*>(&S.x[cl][tt]);
      const __nv_bfloat16* xh = reinterpret_cast<const __nv_bfloat16*>(&xr);
      const float4 d0 = *reinterpret_cast<const float4*>(&S.d[cl][tt]);
      const float4 d1 = *reinterpret_cast<const float4*>(&S.d[cl][tt + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&S.bcT[s][tt]);
      const float4 b1 = *reinterpret_cast<const float4*>(&S.bcT[s][tt + 4]);
      const float4 e0 = *reinterpret_cast<const float4*>(&S.bcT[16 + s][tt]);
      const float4 e1 = *reinterpret_cast<const float4*>(&S.bcT[16 + s][tt + 4]);
      dv[0] = d0.x; dv[1] = d0.y; dv[2] = d0.z; dv[3] = d0.w; dv[4] = d1.x; dv[5] = d1.y; dv[6] = d1.z; dv[7] = d1.w;
      bv[0] = b0.x; bv[1] = b0.y; bv[2] = b0.z; bv[3] = b0.w; bv[4] = b1.x; bv[5] = b1.y; bv[6] = b1.z; bv[7] = b1.w;
      cv[0] = e0.x; cv[1] = e0.y; cv[2] = e0.z; cv[3] = e0.w; cv[4] = e1.x; cv[5] = e1.y; cv[6] = e1.z; cv[7] = e1.w;
#pragma unroll
      for (int u = 0; u < 8; ++u) xv[u] = __bfloat162float(xh[u]);
    };
    auto recur = [&](const float* dv, const float* xv, const float* bv, const float* cv, float* v) {
      float a[8], q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        a[u] = ex2_approx(dv[u] * A2);
        q[u] = dv[u] * xv[u] * bv[u];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        h = fmaf(a[u], h, q[u]);
        v[u] = cv[u] * h;
      }
    };
    // reduce-scatter of v[0..7] over the 16 state lanes: lane l ends with the full sum of
    // step my_step (lanes l and l^1 hold the same step)
    auto reduce_store = [&](const float* v, int tt) {
      const bool q3 = l & 8, q2 = l & 4, q1 = l & 2;
      float w4[4];
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const float send = q3 ? v[k4] : v[k4 + 4];
        const float keep = q3 ? v[k4 + 4] : v[k4];
        w4[k4] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
      }
      float w2[2];
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2) {
        const float send = q2 ? w4[k2] : w4[k2 + 2];
        const float keep = q2 ? w4[k2 + 2] : w4[k2];
        w2[k2] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
      }
      float w1;
      {
        const float send = q1 ? w2[0] : w2[1];
        const float keep = q1 ? w2[1] : w2[0];
        w1 = keep + __shfl_xor_sync(0xffffffffu, send, 2);
      }
      w1 += __shfl_xor_sync(0xffffffffu, w1, 1);
      if ((l & 1) == 0) ys[tt + my_step][cl] = __float2bfloat16_rn(w1);
    };
    {
      float dv[8], xv[8], bv[8], cv[8];
      block_inputs(0, dv, xv, bv, cv);
      recur(dv, xv, bv, cv, vprev);
    }
#pragma unroll 1
    for (int tt = 8; tt < SCAN_TC; tt += 8) {
      float dv[8], xv[8], bv[8], cv[8], v[8];
      block_inputs(tt, dv, xv, bv, cv);
      recur(dv, xv, bv, cv, v);
      reduce_store(vprev, tt - 8);
#pragma unroll
      for (int u = 0; u < 8; ++u) vprev[u] = v[u];
    }
    reduce_store(vprev, SCAN_TC - 8);
    if (kn < n_chunks) store_bc(kn);
    __syncthreads();
    // flush y rows of this chunk: 64 rows x 16 B
    if (tid < SCAN_TC) {
      const int t = k * SCAN_TC + tid;
      if (t < T)
        *reinterpret_cast<uint4*>(y + ((size_t)b * T + t) * Di + c0) = *reinterpret_cast<const uint4*>(&ys[tid][0]);
    }
  }
  state[((size_t)b * Di + c) * 16 + s] = h;
}

}  // namespace hymba
