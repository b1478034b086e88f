// tcgen05 GEMM for sm_100a: D[m, n] = sum_k A[m, k] * B[n, k] (both operands K-major),
// bf16 or fp16 (kind::f16) or fp32 (kind::tf32) inputs, fp32 accumulation in TMEM, TMA-fed.
//
// Persistent warp-specialised kernel, 192 threads:
//   warp 0      TMA producer (one elected lane), STAGES-deep smem ring
//   warp 1      TMEM allocator + MMA issuer (one elected lane)
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (thread = accumulator row),
//               fused epilogue math, global stores
// The accumulator is double-buffered in TMEM so the epilogue of tile i overlaps the
// mainloop of tile i+1.  No TMA multicast, no clusters.
#pragma once
#include "common.cuh"

namespace hymba {

enum EpiMode : int {
  EPI_PROJ = 0,         // segmented bf16 stores with RoPE on marked segments (in_proj)
  EPI_BF16 = 1,         // bf16 store, optional bf16 residual add
  EPI_ATOMIC_F32 = 2,   // fp32 atomic add (split-K partial sums)
  EPI_SOFTPLUS = 3,     // fp32 store of softplus(acc + bias[col])
  EPI_BF16_T = 4,       // transposed bf16 store: out[n][m] (weights as the M operand)
  EPI_ATOMIC_F32_T = 5, // transposed fp32 atomic add
  EPI_SWIGLU = 6,       // columns interleaved [gate(32) | up(32)] -> bf16 SiLU(gate)*up
  EPI_SOFTPLUS_T = 7,   // fp32 softplus(acc + bias[col]) stored time-major: out[(b*N + col)*T_out + row]
  EPI_F32_T = 8,        // transposed fp32 store: out[n][m]
};

struct Segment {
  int col_begin, col_end;   // columns of D this segment covers (multiples of 64)
  void* ptr;                // destination (bf16 or fp16)
  long long bstride;        // batch stride in elements
  int ld;                   // row stride in elements
  int rope;                 // apply RoPE (head dim 64) to this segment
  int f16;                  // 1: store fp16, 0: store bf16
};

struct GemmParams {
  // rows of A come from two sources:
  //   source 0: 2-D map [rows0, K], shared by every batch (the meta-token prefix)
  //   source 1: 3-D map [nb1, rows1, K]
  int tiles0, rows0;
  int nb1, rows1, tiles1;
  int N, K, n_tiles_n, k_blocks, split_k, m_tiles, total_tiles;
  // output row mapping: a source-0 row r goes to rows {b*T_out + r}, b < out_batches;
  // a source-1 row (b, r) goes to b*T_out + row_off1 + r (position row_off1 + r)
  int out_batches, T_out, row_off1;
  int mode;
  void* out;
  int ld_out;
  int n_valid;              // columns (or, transposed, rows of out) that exist
  int m_valid;              // for transposed stores: valid M rows (output columns)
  const __nv_bfloat16* residual;
  int ld_res;
  const float* bias;
  int nseg;
  Segment seg[5];
  double rope_theta[32];    // base^(-2j/64), j < 32
  DevStatus* status;
};

constexpr int GEMM_THREADS = 192;
constexpr int GEMM_BM = 128;

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr int A_BYTES = GEMM_BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_OFFSET = STAGES * STAGE_BYTES;
  static constexpr int TOTAL = BAR_OFFSET + 256 + 1024;   // + barriers + alignment slack
};

__device__ __forceinline__ void rope_pair_rotate(float* v, int pos, const double* theta) {
  // v[0..31] are the first halves x_j, v[32..63] the second halves x_{j+32}.
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    double a = (double)pos * theta[j];
    a -= 6.283185307179586 * rint(a * 0.15915494309189535);
    float s, c;
    sincosf((float)a, &s, &c);
    const float x1 = v[j], x2 = v[j + 32];
    v[j] = x1 * c - x2 * s;
    v[j + 32] = x2 * c + x1 * s;
  }
}

// element types of both operands: bf16, fp16 (kind::f16) or fp32 read as tf32 (kind::tf32)
enum : int { ET_BF16 = 0, ET_F16 = 1, ET_TF32 = 2 };

template <int BN, int STAGES, int ET>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA0, const __grid_constant__ CUtensorMap mapA1,
                   const __grid_constant__ CUtensorMap mapB, const __grid_constant__ GemmParams p) {
  using L = GemmSmem<BN, STAGES>;
  constexpr int ACC_STRIDE = BN <= 128 ? 128 : 256;       // TMEM columns per accumulator
  constexpr uint32_t TMEM_COLS = 2 * ACC_STRIDE;
  constexpr bool TF32 = ET == ET_TF32;
  constexpr uint32_t IDESC = make_idesc(GEMM_BM, BN, ET == ET_TF32 ? 2u : (ET == ET_BF16 ? 1u : 0u), false, false);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFFSET);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapA0);
    tma_prefetch_desc(&mapA1);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < p.total_tiles && !*abort_flag; tile += gridDim.x) {
        const int ks = tile % p.split_k;
        const int t2 = tile / p.split_k;
        const int m = t2 % p.m_tiles;
        const int n = t2 / p.m_tiles;
        const int kb0 = (int)((long long)ks * p.k_blocks / p.split_k);
        const int kb1 = (int)((long long)(ks + 1) * p.k_blocks / p.split_k);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, 101)) break;
          uint8_t* sa = smem + s * L::STAGE_BYTES;
          uint8_t* sb = sa + L::A_BYTES;
          mbar_arrive_expect_tx(&full[s], L::STAGE_BYTES);
          const int kc = kb * (TF32 ? 32 : 64);
          if (m < p.tiles0) {
            tma_load_2d(sa, &mapA0, &full[s], kc, m * GEMM_BM);
          } else {
            const int idx = m - p.tiles0;
            tma_load_3d(sa, &mapA1, &full[s], kc, (idx % p.tiles1) * GEMM_BM, idx / p.tiles1);
          }
          tma_load_2d(sb, &mapB, &full[s], kc, n * BN);
        }
      }
      // Drain: wait until every load issued has landed (their consumer may have given up).
      for (uint32_t j = (it > (uint32_t)STAGES ? it - STAGES : 0u); j < it; ++j) {
        mbar_wait(&full[j % STAGES], (j / STAGES) & 1u, nullptr, p.status, 102);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      uint32_t it = 0;
      int lt = 0;
      for (int tile = blockIdx.x; tile < p.total_tiles && !*abort_flag; tile += gridDim.x, ++lt) {
        const int ks = tile % p.split_k;
        const int kb0 = (int)((long long)ks * p.k_blocks / p.split_k);
        const int kb1 = (int)((long long)(ks + 1) * p.k_blocks / p.split_k);
        const int ab = lt & 1;
        const uint32_t aph = (lt >> 1) & 1u;
        if (!mbar_wait(&acc_empty[ab], aph ^ 1u, abort_flag, p.status, 103)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * ACC_STRIDE;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag, p.status, 104)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * L::STAGE_BYTES);
          const uint32_t sb = sa + L::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_sdesc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = make_sdesc_sw128(sb + kk * 32, 16, 1024);
            const uint32_t acc = (kb > kb0 || kk > 0) ? 1u : 0u;
            if (TF32) umma_tf32(d_tmem, ad, bd, IDESC, acc);
            else umma_f16(d_tmem, ad, bd, IDESC, acc);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int quad = warp & 3;               // TMEM lanes this warp may access
    const int r = quad * 32 + lane;          // accumulator row of this thread
    int lt = 0;
    for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++lt) {
      const int t2 = tile / p.split_k;
      const int m = t2 % p.m_tiles;
      const int n = t2 / p.m_tiles;
      const int ab = lt & 1;
      const uint32_t aph = (lt >> 1) & 1u;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&acc_full[ab], aph, abort_flag, p.status, 105) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);   // keep the warp converged for tcgen05.ld
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + ab * ACC_STRIDE;

      // which output row(s) this accumulator row feeds
      int src0 = m < p.tiles0;
      int b1 = 0, rr;
      if (src0) {
        rr = m * GEMM_BM + r;
      } else {
        const int idx = m - p.tiles0;
        b1 = idx / p.tiles1;
        rr = (idx % p.tiles1) * GEMM_BM + r;
      }
      const bool row_ok = src0 ? (rr < p.rows0) : (rr < p.rows1);
      const int col_base = n * BN;

      if (p.mode == EPI_PROJ) {
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 64) {
          float v[64];
          tmem_ld32(tbase + c0, v);
          tmem_ld32(tbase + c0 + 32, v + 32);
          const int gc = col_base + c0;
          if (!row_ok || gc >= p.N) continue;
          int si = 0;
#pragma unroll 1
          while (si < p.nseg - 1 && gc >= p.seg[si].col_end) ++si;
          const Segment sg = p.seg[si];
          const int pos = src0 ? rr : p.row_off1 + rr;
          if (sg.rope) rope_pair_rotate(v, pos, p.rope_theta);
          __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(sg.ptr) + (gc - sg.col_begin);
          const int b_lo = src0 ? 0 : b1, b_hi = src0 ? p.out_batches : b1 + 1;
          for (int b = b_lo; b < b_hi; ++b) {
            __nv_bfloat16* dst = base + b * sg.bstride + (size_t)pos * sg.ld;
            if (sg.f16) store_f16_row(dst, v, 64);
            else store_bf16_row(dst, v, 64);
          }
        }
      } else if (p.mode == EPI_BF16_T || p.mode == EPI_ATOMIC_F32_T || p.mode == EPI_F32_T) {
        // accumulator row = output column (weight row), accumulator column = output row
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          float v[32];
          tmem_ld32(tbase + c0, v);
          if (!row_ok || rr >= p.m_valid) continue;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int orow = col_base + c0 + e;
            if (orow < p.n_valid) {
              if (p.mode == EPI_BF16_T)
                reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)orow * p.ld_out + rr] = __float2bfloat16_rn(v[e]);
              else if (p.mode == EPI_F32_T)
                reinterpret_cast<float*>(p.out)[(size_t)orow * p.ld_out + rr] = v[e];
              else
                atomicAdd(reinterpret_cast<float*>(p.out) + (size_t)orow * p.ld_out + rr, v[e]);
            }
          }
        }
      } else if (p.mode == EPI_SWIGLU) {
        // B rows interleave 32 gate rows and 32 up rows; each 64-column chunk gives 32
        // outputs SiLU(gate) * up at output columns (col_base + c0) / 2.
        const size_t orow = (size_t)b1 * p.rows1 + rr;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 64) {
          float v[64];
          tmem_ld32(tbase + c0, v);
          tmem_ld32(tbase + c0 + 32, v + 32);
          const int gc = col_base + c0;
          if (!row_ok || gc >= p.N) continue;
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = silu_f(v[e]) * v[e + 32];
          store_bf16_row(reinterpret_cast<__nv_bfloat16*>(p.out) + orow * p.ld_out + gc / 2, v, 32);
        }
      } else {
        const size_t orow = (size_t)b1 * p.rows1 + rr;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          float v[32];
          tmem_ld32(tbase + c0, v);
          const int gc = col_base + c0;
          if (!row_ok || gc >= p.n_valid) continue;
          if (p.mode == EPI_BF16) {
            if (p.residual != nullptr) {
              const __nv_bfloat16* res = p.residual + orow * p.ld_res + gc;
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (gc + e < p.n_valid) v[e] += __bfloat162float(res[e]);
            }
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + orow * p.ld_out + gc;
            const int nv = min(32, p.n_valid - gc);
            if (nv == 32) {
              store_bf16_row(dst, v, 32);
            } else {
              for (int e = 0; e < nv; ++e) dst[e] = __float2bfloat16_rn(v[e]);
            }
          } else if (p.mode == EPI_ATOMIC_F32) {
            // vector fp32 reductions (ld_out and n_valid are multiples of 4)
            float* dst = reinterpret_cast<float*>(p.out) + orow * p.ld_out + gc;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              if (gc + e < p.n_valid)
                atomicAdd(reinterpret_cast<float4*>(dst + e), make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]));
          } else if (p.mode == EPI_SOFTPLUS) {
            float* dst = reinterpret_cast<float*>(p.out) + orow * p.ld_out + gc;
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (gc + e < p.n_valid) dst[e] = softplus_fast(v[e] + p.bias[gc + e]);
          } else {  // EPI_SOFTPLUS_T: lanes hold consecutive rows -> coalesced along time
            float* dst = reinterpret_cast<float*>(p.out) + ((size_t)b1 * p.N + gc) * p.T_out + rr;
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (gc + e < p.n_valid) dst[(size_t)e * p.T_out] = softplus_fast(v[e] + p.bias[gc + e]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace hymba
