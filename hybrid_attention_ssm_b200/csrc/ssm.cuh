// SSM branch kernels (prefill): causal depthwise conv1d + SiLU, and the selective scan.
#pragma once
#include <type_traits>
#include "common.cuh"

namespace hymba {

// ----------------------------------------------------------------------------------------
// conv1d (kernel width 4) + SiLU over time, per channel.
//   x      [B*T, ld_x] bf16, channel c at column c (the x part of the in_proj output)
//   xc     [B*T, Di]   bf16 row-major (A operand of x_proj and input of the scan)
//   state  [B, Di, 3]  fp32: the last 3 inputs x[T-3..T-1] (zero before the start)
// Rows t_begin .. T-1 are computed; inputs before t_begin come from hist [Di, 3] (the
// inputs t_begin-3 .. t_begin-1, the same for every sequence), or are zero when hist is
// NULL.
// ----------------------------------------------------------------------------------------
constexpr int CONV_K = 4;
constexpr int CONV_TT = 64;      // time steps per CTA
constexpr int CONV_TC = 64;      // channels per CTA
constexpr int CONV_P = CONV_TC + 8;   // smem row pitch (16-byte aligned rows)

// CTA = 64 channels x 64 time steps, 256 threads.  The x tile (plus the 3 rows before it)
// comes in as 128-byte row pieces; a thread walks 16 steps of one channel with the 3-step
// history in registers and writes its outputs into a [t][c] shared tile, from which they
// leave as 128-byte rows.
__global__ void __launch_bounds__(256)
    conv1d_silu_kernel(const __nv_bfloat16* __restrict__ x, int ld_x, const float* __restrict__ w,
                       const float* __restrict__ bias, __nv_bfloat16* __restrict__ xc,
                       float* __restrict__ state, int T, int Di, int t_begin, const float* __restrict__ hist) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) __nv_bfloat16 xs[CONV_TT + CONV_K - 1][CONV_P];   // rows t0-3 .. t0+63
  __shared__ __align__(16) __nv_bfloat16 orow[CONV_TT][CONV_P];               // [t][c]
  const int c0 = blockIdx.x * CONV_TC, t0 = t_begin + blockIdx.y * CONV_TT, b = blockIdx.z;
  const int tid = threadIdx.x;
  const __nv_bfloat16* xb = x + (size_t)b * T * ld_x + c0;
  for (int i = tid; i < (CONV_TT + CONV_K - 1) * 8; i += 256) {
    const int r = i >> 3, q = i & 7, t = t0 - (CONV_K - 1) + r;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (t >= t_begin && t < T) {
      v = *reinterpret_cast<const uint4*>(xb + (size_t)t * ld_x + q * 8);
    } else if (t < t_begin && t >= t_begin - 3 && hist != nullptr) {
      __nv_bfloat16 hv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) hv[e] = __float2bfloat16_rn(hist[(size_t)(c0 + q * 8 + e) * 3 + (t - t_begin + 3)]);
      v = *reinterpret_cast<const uint4*>(hv);
    }
    *reinterpret_cast<uint4*>(&xs[r][q * 8]) = v;
  }
  __syncthreads();
  {
    const int cc = tid & 63, tq = (tid >> 6) * 16;   // channel, first of 16 steps
    const float4 wv = *reinterpret_cast<const float4*>(w + (size_t)(c0 + cc) * 4);
    const float bb = bias[c0 + cc];
    float h0 = __bfloat162float(xs[tq][cc]), h1 = __bfloat162float(xs[tq + 1][cc]);
    float h2 = __bfloat162float(xs[tq + 2][cc]);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float xa = __bfloat162float(xs[tq + 3 + i][cc]);
      const float ya = bb + wv.x * h0 + wv.y * h1 + wv.z * h2 + wv.w * xa;
      const float xb2 = __bfloat162float(xs[tq + 4 + i][cc]);
      const float yb = bb + wv.x * h1 + wv.y * h2 + wv.z * xa + wv.w * xb2;
      h0 = h2; h1 = xa; h2 = xb2;
      const __nv_bfloat162 o2 = __floats2bfloat162_rn(silu_f(ya), silu_f(yb));
      orow[tq + i][cc] = o2.x;
      orow[tq + i + 1][cc] = o2.y;
    }
  }
  __syncthreads();
  // row-major xc, 128-byte rows (8 threads x 16 bytes)
  for (int i = tid; i < CONV_TT * 8; i += 256) {
    const int r = i >> 3, q = i & 7, t = t0 + r;
    if (t < T)
      *reinterpret_cast<uint4*>(xc + ((size_t)b * T + t) * Di + c0 + q * 8) =
          *reinterpret_cast<const uint4*>(&orow[r][q * 8]);
  }
  // conv state: the last 3 inputs x[T-3..T-1] (zero before the start), from the last tile
  // (the rows before it are in xs too, history included)
  if (t0 + CONV_TT >= T && tid < CONV_TC) {
    float* s0 = state + ((size_t)b * Di + c0 + tid) * 3;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const int t = T - 3 + k;
      s0[k] = t >= 0 ? __bfloat162float(xs[t - t0 + CONV_K - 1][tid]) : 0.f;
    }
  }
}

// ----------------------------------------------------------------------------------------
// Chunked selective scan ([JJ] §数学表示 4, eq. (2), Euler form):
//   h_t[s] = exp(delta_t A[s]) h_{t-1}[s] + delta_t B_t[s] x_t,   y_t = sum_s C_t[s] h_t[s]
// The recurrence is linear in h, so a stretch of steps acts on its start state as the
// affine map h -> D h + e with D[s] = prod_t exp(delta_t A[s]) = exp(A[s] sum_t delta_t) and
// e = the stretch's end state from a zero start; these maps compose associatively.  T is cut
// into n_chunks chunks of L steps, which makes B*Di*n_chunks independent lanes instead of
// B*Di*16 serial chains, enough to fill the GPU at batch 1:
//   pass 1  scan_chunk_kernel<false>: chunks 0..n-2 from a zero state -> e (end state) and
//           sum(delta) per (sequence, chunk, channel);
//   carry   scan_carry_kernel: per (sequence, channel, state), chunks in order:
//           start[k+1] = exp(A sum_k(delta)) start[k] + e_k  (start[0] = 0);
//   pass 2  scan_chunk_kernel<true>: every chunk from its true start; writes y and, from the
//           last chunk, the final state.
// A lane owns one (sequence, channel, chunk) and the channel's 16 states in registers, so
// y_t = C_t . h_t is a sum inside the lane and B_t, C_t are the same for every lane of the
// CTA (shared-memory broadcasts).  CTA = 64 channels (two warps) of one chunk; dt_pre
// [rows, Di] bf16 (dt_low W_dt^T), x [rows, Di] bf16 and (B | C) [rows, 32] fp32 stream in by
// TMA, 8 steps per stage, all in their row-major producer layouts.  dt_proj's bias and
// softplus are applied here, as each step is read: delta = softplus(dt_pre + dt_bias), in
// both passes, instead of a pass of their own over [rows, Di].
// The 16 decays exp(delta A[s]) take 16 MUFU ex2 per step.  When a warp's A rows are the
// progression A[s] = (s + 1) A[0] (the S4D-real initialisation -[1..16] of the workloads),
// exp(delta A[s]) = exp(delta A[0])^(s+1): one ex2 and a multiplication tree give all 16.
//   y [rows, Di] bf16 (ungated: the branch norm applies SiLU(z)); state [B, Di, 16] fp32;
//   carry [B][n_chunks-1][Di][16] fp32 and sumd [B][n_chunks-1][Di] fp32 (workspace).
// ----------------------------------------------------------------------------------------
constexpr int SC_CH = 64;      // channels per CTA, one lane each
constexpr int SC_SUB = 8;      // steps per TMA stage
constexpr int SC_NST = 4;      // ring stages
constexpr int SC_THREADS = SC_CH;
constexpr int SC_PER_SM = 10;  // CTAs resident per SM (the register budget of __launch_bounds__)

struct ScStage {
  __nv_bfloat16 d[SC_SUB][SC_CH];    // dt_pre rows   (box {64, 8} bf16, 1024 B)
  __nv_bfloat16 x[SC_SUB][SC_CH];    // x rows        (box {64, 8} bf16, 1024 B)
  float bc[SC_SUB][32];              // B | C rows    (box {32, 8} fp32, 1024 B)
};
static_assert(sizeof(ScStage) == 3072, "stage layout must match the TMA boxes");

struct ScSmem {
  ScStage st[SC_NST];
  uint64_t full[SC_NST];
  int abort;
};
constexpr int SC_SMEM = (int)sizeof(ScSmem) + 128;   // + alignment slack

struct ScanParams {
  int T, Di, L, n_chunks;
  int t_begin;           // first row scanned (the chunks cover rows t_begin .. T-1)
  const float* h0;       // [Di, 16] state before row t_begin, the same for every sequence, or NULL (zero)
  const float* A;        // [Di, 16]
  const float* dt_bias;  // [Di]
  float* carry;          // [B][n_chunks-1][Di][16]
  float* sumd;           // [B][n_chunks-1][Di]
  __nv_bfloat16* y;      // [B*T, Di]
  float* state;          // [B, Di, 16]
  DevStatus* status;
};

// The 16 decays of one step as (state 2j, state 2j+1) pairs: a[j] = exp2(d * A2[s]), A2 = A log2 e.
__device__ __forceinline__ void scan_decays_general(float d, const uint64_t* A2, uint64_t* a) {
  const uint64_t dd = f2_pack(d, d);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint64_t arg = f2_mul(dd, A2[j]);
    a[j] = f2_pack(ex2_approx(f2_lo(arg)), ex2_approx(f2_hi(arg)));
  }
}
// The same when A[s] = (s + 1) A[0]: e_k = e_1^k from e_1 = exp2(d * A2[0]) by a product
// tree of depth 4 (e_2 = e_1 e_1, e_4 = e_2 e_2, e_8 = e_4 e_4, e_16 = e_8 e_8).
__device__ __forceinline__ void scan_decays_pow(float d, float A20, uint64_t* a) {
  const float e1 = ex2_approx(d * A20);
  const float e2 = e1 * e1;
  a[0] = f2_pack(e1, e2);                           // (e1, e2)
  a[1] = f2_mul(a[0], f2_pack(e2, e2));             // (e3, e4)
  const float e4 = f2_hi(a[1]);
  const uint64_t p4 = f2_pack(e4, e4);
  a[2] = f2_mul(a[0], p4);                          // (e5, e6)
  a[3] = f2_mul(a[1], p4);                          // (e7, e8)
  const float e8 = f2_hi(a[3]);
  const uint64_t p8 = f2_pack(e8, e8);
#pragma unroll
  for (int j = 0; j < 4; ++j) a[4 + j] = f2_mul(a[j], p8);   // (e9, e10) .. (e15, e16)
}

template <bool OUT>
__global__ void __launch_bounds__(SC_THREADS, SC_PER_SM)
    scan_chunk_kernel(const __grid_constant__ CUtensorMap mapD, const __grid_constant__ CUtensorMap mapX,
                      const __grid_constant__ CUtensorMap mapBC, const __grid_constant__ ScanParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t sc_smem_raw[];
  ScSmem& sm = *reinterpret_cast<ScSmem*>(align_smem<128>(sc_smem_raw));
  const int tid = threadIdx.x;
  const int g = blockIdx.x, k = blockIdx.y, b = blockIdx.z;
  const int c = g * SC_CH + tid;
  const int t0 = p.t_begin + k * p.L;
  const int t1 = min(t0 + p.L, p.T);
  const int n_sub = (t1 - t0 + SC_SUB - 1) / SC_SUB;
  const int row0 = b * p.T + t0;

  if (tid == 0) {
    for (int i = 0; i < SC_NST; ++i) mbar_init(&sm.full[i], 1);
    sm.abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mapD);
    tma_prefetch_desc(&mapX);
    tma_prefetch_desc(&mapBC);
  }
  __syncthreads();
  auto issue = [&](int j) {    // one thread: the three loads of sub-chunk j
    ScStage& S = sm.st[j % SC_NST];
    uint64_t* bar = &sm.full[j % SC_NST];
    mbar_arrive_expect_tx(bar, (uint32_t)sizeof(ScStage));
    tma_load_2d(&S.d[0][0], &mapD, bar, g * SC_CH, row0 + j * SC_SUB);
    tma_load_2d(&S.x[0][0], &mapX, bar, g * SC_CH, row0 + j * SC_SUB);
    tma_load_2d(&S.bc[0][0], &mapBC, bar, 0, row0 + j * SC_SUB);
  };
  int issued = 0;
  if (tid == 0)
    for (; issued < SC_NST - 1 && issued < n_sub; ++issued) issue(issued);

  // A in log2 units, and whether this warp's channels all have A[s] = (s + 1) A[0]
  uint64_t A2[8];
  bool prog = true;
  {
    const float4* ar = reinterpret_cast<const float4*>(p.A + (size_t)c * 16);
    float a[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = ar[q];
      a[4 * q] = v.x; a[4 * q + 1] = v.y; a[4 * q + 2] = v.z; a[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int s = 1; s < 16; ++s) prog = prog && (a[s] == (float)(s + 1) * a[0]);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      A2[j] = f2_pack(a[2 * j] * 1.4426950408889634f, a[2 * j + 1] * 1.4426950408889634f);
  }
  const bool pow_path = __all_sync(0xffffffffu, prog);
  const float A20 = f2_lo(A2[0]);
  const float bias = p.dt_bias[c];

  uint64_t h[8];
  if (OUT && k > 0) {
    const float4* hs = reinterpret_cast<const float4*>(p.carry + (((size_t)b * (p.n_chunks - 1) + k - 1) * p.Di + c) * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = hs[q];
      h[2 * q] = f2_pack(v.x, v.y);
      h[2 * q + 1] = f2_pack(v.z, v.w);
    }
  } else if (OUT && p.h0 != nullptr) {   // chunk 0 of the output pass from the given state
    const float4* hs = reinterpret_cast<const float4*>(p.h0 + (size_t)c * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = hs[q];
      h[2 * q] = f2_pack(v.x, v.y);
      h[2 * q + 1] = f2_pack(v.z, v.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) h[j] = 0ull;
  }
  float sumd = 0.f;
  __nv_bfloat16* yrow = p.y + (size_t)row0 * p.Di + c;

  // one step: decays, h = a h + dx B, and (output pass) y = C . h with two independent
  // accumulators; B and C are read as (state 2q, state 2q+1) pairs straight into 64-bit
  // registers
  // POW: the decay path, a template argument so that a stage's unrolled steps hold no branch
  // and the scheduler can overlap one step's softplus and decays with the previous step's
  // state update
  auto step = [&](auto pow_c, const ScStage& S, int i, __nv_bfloat16* yp) {
    constexpr bool POW = decltype(pow_c)::value;
    const float d = softplus_sel(__bfloat162float(S.d[i][tid]) + bias);   // delta of this step and channel
    const float dx = d * __bfloat162float(S.x[i][tid]);
    uint64_t a[8];
    if constexpr (POW) scan_decays_pow(d, A20, a);
    else scan_decays_general(d, A2, a);
    const uint64_t dxp = f2_pack(dx, dx);
    const ulonglong2* bc = reinterpret_cast<const ulonglong2*>(&S.bc[i][0]);   // the same address in every lane
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const ulonglong2 bv = bc[q];   // (B[4q], B[4q+1]), (B[4q+2], B[4q+3])
      h[2 * q] = f2_fma(a[2 * q], h[2 * q], f2_mul(dxp, bv.x));
      h[2 * q + 1] = f2_fma(a[2 * q + 1], h[2 * q + 1], f2_mul(dxp, bv.y));
    }
    if constexpr (OUT) {
      uint64_t acc0 = 0ull, acc1 = 0ull;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const ulonglong2 cv = bc[4 + q];   // C[4q .. 4q+3]
        acc0 = f2_fma(cv.x, h[2 * q], acc0);
        acc1 = f2_fma(cv.y, h[2 * q + 1], acc1);
      }
      const uint64_t acc = f2_add(acc0, acc1);
      *yp = __float2bfloat16_rn(f2_lo(acc) + f2_hi(acc));
    } else {
      sumd += d;
    }
  };

  int j = 0;
  for (; j < n_sub; ++j) {
    // the stage of sub-chunk j-1 is free (barrier at the end of the previous iteration)
    if (tid == 0 && issued < n_sub) issue(issued++);
    const bool ok = mbar_wait(&sm.full[j % SC_NST], (uint32_t)(j / SC_NST) & 1u, &sm.abort, p.status, 311);
    if (ok) {
      const ScStage& S = sm.st[j % SC_NST];
      __nv_bfloat16* yj = yrow + (size_t)(j * SC_SUB) * p.Di;
      const int n_steps = t1 - t0 - j * SC_SUB;
      using pow_t = std::integral_constant<bool, true>;
      using gen_t = std::integral_constant<bool, false>;
      if (n_steps >= SC_SUB) {
        if (pow_path) {
#pragma unroll
          for (int i = 0; i < SC_SUB; ++i) step(pow_t{}, S, i, yj + (size_t)i * p.Di);
        } else {
#pragma unroll
          for (int i = 0; i < SC_SUB; ++i) step(gen_t{}, S, i, yj + (size_t)i * p.Di);
        }
      } else {
        for (int i = 0; i < n_steps; ++i) {
          if (pow_path) step(pow_t{}, S, i, yj + (size_t)i * p.Di);
          else step(gen_t{}, S, i, yj + (size_t)i * p.Di);
        }
      }
    }
    if (__syncthreads_or(ok ? 0 : 1)) break;   // a wait gave up: every thread leaves together
  }
  if (j < n_sub) {
    // gave up: wait (bounded) for the loads still in flight before the CTA exits
    if (tid == 0)
      for (int q = j; q < issued; ++q)
        mbar_wait(&sm.full[q % SC_NST], (uint32_t)(q / SC_NST) & 1u, nullptr, p.status, 312);
    return;
  }
  float* dst = nullptr;
  if constexpr (OUT) {
    if (k == p.n_chunks - 1) dst = p.state + ((size_t)b * p.Di + c) * 16;
  } else {
    const size_t ci = ((size_t)b * (p.n_chunks - 1) + k) * p.Di + c;
    dst = p.carry + ci * 16;
    p.sumd[ci] = sumd;
  }
  if (dst != nullptr) {
    float4* o = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      o[q] = make_float4(f2_lo(h[2 * q]), f2_hi(h[2 * q]), f2_lo(h[2 * q + 1]), f2_hi(h[2 * q + 1]));
  }
}

// Carry across chunks, one thread per (sequence, channel, state): replaces each chunk's
// zero-start end state by the true start state of the next chunk, in chunk order.
__global__ void __launch_bounds__(256)
    scan_carry_kernel(const __grid_constant__ ScanParams p, int B) {
  pdl_wait();
  pdl_trigger();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)B * p.Di * 16) return;
  const int s = (int)(i & 15);
  const long long bc = i >> 4;               // b * Di + c
  const int c = (int)(bc % p.Di);
  const long long b = bc / p.Di;
  const float a2 = p.A[(size_t)c * 16 + s] * 1.4426950408889634f;
  const int nk = p.n_chunks - 1;
  float* e = p.carry + ((size_t)b * nk * p.Di + c) * 16 + s;
  const float* sd = p.sumd + (size_t)b * nk * p.Di + c;
  const size_t es = (size_t)p.Di * 16;
  float h = p.h0 != nullptr ? p.h0[(size_t)c * 16 + s] : 0.f;
  for (int k0 = 0; k0 < nk; k0 += 8) {
    float ev[8], dv[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {   // eight chunks' loads in flight before the chain uses them
      ev[q] = k0 + q < nk ? e[(size_t)(k0 + q) * es] : 0.f;
      dv[q] = k0 + q < nk ? sd[(size_t)(k0 + q) * p.Di] : 0.f;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (k0 + q < nk) {
        h = fmaf(ex2_approx(a2 * dv[q]), h, ev[q]);
        e[(size_t)(k0 + q) * es] = h;
      }
    }
  }
}

}  // namespace hymba
