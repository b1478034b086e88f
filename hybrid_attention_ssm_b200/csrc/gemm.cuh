// tcgen05 GEMM for sm_100a: D[m, n] = sum_k A[m, k] * B[n, k] (both operands K-major),
// bf16 or fp16 (kind::f16) or fp32 (kind::tf32) inputs, fp32 accumulation in TMEM, TMA-fed.
//
// Persistent warp-specialised kernel, 320 threads:
//   warp 0      TMA producer (one elected lane), STAGES-deep smem ring
//   warp 1      TMEM allocator + MMA issuer (one elected lane)
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (thread = accumulator row),
//               fused epilogue math, global stores.  A warp may only read the TMEM lane
//               quadrant warp%4, so two warps share each quadrant and split the tile's
//               column chunks between them (two epilogue warps per SM sub-partition).
// The accumulator is double-buffered in TMEM so the epilogue of tile i overlaps the
// mainloop of tile i+1.  The epilogue is a template parameter, so each instance carries
// only its own code.
//
// PAIR: the CTAs run as clusters of two on two SMs, and one tcgen05.mma.cta_group::2 of
// M = 256 covers both CTAs' 128-row A tiles against a BN-wide B tile of which each CTA holds
// one half: per k-block an SM then moves 16 KB of A and BN/2 x 128 B of B into shared memory
// instead of 16 KB + BN x 128 B, for the same MMA work.  Each CTA loads its own tiles into
// its own shared memory; the loads of both complete on the even CTA's barrier, whose single MMA
// thread issues the pair's MMAs and commits them to both CTAs' barriers.  Each CTA's
// epilogue reads its own TMEM rows, as in the single-CTA form.
#pragma once
#include "common.cuh"

namespace hymba {

enum EpiMode : int {
  EPI_PROJ = 0,         // segmented bf16/fp16 stores with RoPE on marked segments (in_proj)
  EPI_BF16 = 1,         // bf16 store, optional bf16 residual add
  EPI_SWIGLU = 2,       // columns interleaved [gate(32) | up(32)] -> fp16 SiLU(gate)*up
  // 3: unused (formerly an fp32 row store)
  EPI_F32_T = 4,        // transposed fp32 store: out[n][m] (weights as the M operand)
  EPI_F32_PART = 5,     // fp32 store of split ks's partial sum at out + ks*split_stride (row-major)
  EPI_F32_T_PART = 6,   // the same, transposed
};

struct Segment {
  int col_begin, col_end;   // columns of D this segment covers (multiples of 64)
  void* ptr;                // destination (bf16 or fp16)
  long long bstride;        // batch stride in elements
  int ld;                   // row stride in elements
  int rope;                 // apply RoPE (head dim 64) to this segment
  int f16;                  // 1: store fp16, 0: store bf16
  // optional second home of fp16 rows in an SWA decode cache ([B, M, ld] meta rows and a
  // [B, W, ld] ring): position < M goes to meta[b][pos], position >= win0 to
  // ring[b][(pos - M) mod W]
  void* meta;
  void* ring;
  int M, W, win0;
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
  int m_pairs;              // PAIR: cdiv(m_tiles, 2); total_tiles counts pair tiles
  // 1: the column tiles of one row tile (or pair) are consecutive in the tile order, so the
  // CTAs at work at any moment share a few A row tiles and sweep the whole B operand (the
  // weights, 15-35 MB, which stay in L2); for an A operand too large to stay in L2 next to
  // them.  0: row tiles inner (each B column tile is shared by the CTAs at work).
  int n_inner;
  // 1: only the epilogue warps wait for the previous kernel on the stream.  For a GEMM whose
  // operands no kernel of the same call writes (the caller's input and the weights), so the
  // mainloop overlaps a previous kernel that only prepares what the epilogue reads.
  int wait_late;
  // 1: the A operand (weights) is read-only for the whole stream: the producer issues the A
  // tiles of its first tile's first STAGES k-blocks before it waits for the previous kernel,
  // so the weight stream starts while that kernel runs (decode GEMMs, weights as M operand).
  int prefetch_a;
  // with prefetch_a, 1: the producer also lets the next kernel launch before its own wait,
  // so that kernel's CTAs are resident (and waiting) before this one starts its mainloop;
  // for a next kernel whose launch latency is on the critical path and no other stream's
  // kernel needs the SM room meanwhile.  0: only the warps that have waited trigger it.
  int trigger_early;
  void* out;
  long long split_stride;   // elements between the partial-sum slices of two splits
  int ld_out;
  int n_valid;              // columns (or, transposed, rows of out) that exist
  int m_valid;              // for transposed stores: valid M rows (output columns)
  const __nv_bfloat16* residual;
  int ld_res;
  const float* bias;
  int nseg;
  Segment seg[5];
  const float2* rope_tab;   // [positions][32] (cos, sin) of pos * base^(-2j/64)
  DevStatus* status;
};

constexpr int GEMM_EPI_WARPS = 8;
constexpr int GEMM_THREADS = 64 + 32 * GEMM_EPI_WARPS;
constexpr int GEMM_BM = 128;

// Shared memory an epilogue stages its output through: EPI_BF16 exchanges each warp's
// 32 x 32 bf16 block (rows of 64 bytes padded to 80) so that four lanes load or store one
// row's 64 bytes (two whole 32-byte sectors) instead of each lane touching 16 bytes of its
// own row.
constexpr int GEMM_BF16_TILE_WORDS = 20;   // words per staged row
__host__ __device__ constexpr int gemm_epi_bytes(int mode) {
  return mode == 1 /* EPI_BF16 */ ? GEMM_EPI_WARPS * 32 * GEMM_BF16_TILE_WORDS * 4 : 0;
}

template <int BN, int STAGES, int EPI_BYTES = 0, bool PAIR = false>
struct GemmSmem {
  static constexpr int A_BYTES = GEMM_BM * 128;
  static constexpr int B_BYTES = (PAIR ? BN / 2 : BN) * 128;   // PAIR: this CTA's half of the B tile
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_OFFSET = STAGES * STAGE_BYTES;
  static constexpr int EPI_OFFSET = BAR_OFFSET + 256;
  static constexpr int TOTAL = EPI_OFFSET + EPI_BYTES + 1024;   // + barriers, staging, alignment slack
};

// Rotate the pairs (v[j], v[j+32]) of one 64-wide head by the angles of position pos.
__device__ __forceinline__ void rope_pair_rotate(float* v, const float2* __restrict__ tab_row) {
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const float4 cs = *reinterpret_cast<const float4*>(tab_row + j);   // (c_j, s_j, c_j+1, s_j+1)
    float x1 = v[j], x2 = v[j + 32];
    v[j] = x1 * cs.x - x2 * cs.y;
    v[j + 32] = x2 * cs.x + x1 * cs.y;
    x1 = v[j + 1], x2 = v[j + 33];
    v[j + 1] = x1 * cs.z - x2 * cs.w;
    v[j + 33] = x2 * cs.z + x1 * cs.w;
  }
}

// tcgen05.ld of 32 columns without waiting, and the wait that orders later uses of the
// registers after the load (every register is an operand of the wait).
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t* r) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;\n"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]),
        "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]),
        "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
        "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// element types of both operands: bf16, fp16 (kind::f16) or fp32 read as tf32 (kind::tf32)
enum : int { ET_BF16 = 0, ET_F16 = 1, ET_TF32 = 2 };

template <int BN, int STAGES, int ET, int MODE, bool PAIR = false>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA0, const __grid_constant__ CUtensorMap mapA1,
                   const __grid_constant__ CUtensorMap mapB, const __grid_constant__ GemmParams p) {
  using L = GemmSmem<BN, STAGES, gemm_epi_bytes(MODE), PAIR>;
  static_assert(L::TOTAL <= 232448, "shared memory of one CTA");
  static_assert(!PAIR || (ET != ET_TF32 && BN % 32 == 0), "pair tiles: 16-bit operands, BN / 2 a multiple of 16");
  static_assert(L::STAGE_BYTES % 1024 == 0, "stage buffers keep the 1024-byte swizzle alignment");
  constexpr int ACC_STRIDE = BN <= 128 ? 128 : 256;       // TMEM columns per accumulator
  constexpr uint32_t TMEM_COLS = 2 * ACC_STRIDE;
  constexpr bool TF32 = ET == ET_TF32;
  constexpr uint32_t IDESC =
      make_idesc(PAIR ? 2 * GEMM_BM : GEMM_BM, BN, ET == ET_TF32 ? 2u : (ET == ET_BF16 ? 1u : 0u), false, false);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem<1024>(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFFSET);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // PAIR: rank in the pair (its M tile is 2 * pair + rank) and the pair's tile stream
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int tile0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int tile_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int m_count = PAIR ? p.m_pairs : p.m_tiles;   // row tiles, or pairs of them
  // Tile order (GemmParams::n_inner): row tiles (or pairs) inner, or column tiles inner.
  auto tile_m = [&](int t2) {
    const int mi = p.n_inner ? t2 / p.n_tiles_n : t2 % m_count;
    return PAIR ? 2 * mi + (int)rank : mi;
  };
  auto tile_n = [&](int t2) { return p.n_inner ? t2 % p.n_tiles_n : t2 / m_count; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], PAIR ? 2 * GEMM_EPI_WARPS : GEMM_EPI_WARPS);   // PAIR: both CTAs' epilogues
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
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // both CTAs' barriers and TMEM exist before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The set-up above touches only this CTA's shared memory, its TMEM and the kernel
  // parameters, so it overlaps the previous kernel's tail.  Every access to global memory
  // comes after the wait.  A CTA launched early can only meet TMEM held by CTAs of the
  // previous kernel, which are all running by then and free it when they finish.
  // With prefetch_a the producer warp waits in its own branch, after its early A loads, and
  // (unless trigger_early) leaves the launch of the next kernel to the warps that have
  // waited: a dependent launched before this kernel's own predecessor has finished holds SM
  // room that a kernel on another stream (the decode attention) may need.
  const bool early_a = p.prefetch_a && warp == 0;
  if ((!p.wait_late && !early_a) || warp >= 2) pdl_wait();
  if (!early_a || p.trigger_early) pdl_trigger();

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      auto load_a = [&](uint8_t* sa, uint64_t* bar, int m, int kc) {
        if (m < p.tiles0) {
          tma_load_2d(sa, &mapA0, bar, kc, m * GEMM_BM);
        } else {
          const int idx = m - p.tiles0;
          tma_load_3d(sa, &mapA1, bar, kc, (idx % p.tiles1) * GEMM_BM, idx / p.tiles1);
        }
      };
      // k-blocks (counted from the CTA's first) whose A tile is already in flight: stages
      // 0..pre-1 of the first tile, loaded before the wait with the stage's full byte count
      // expected, so their B loads below complete them
      uint32_t pre = 0;
      if (!PAIR && p.prefetch_a) {
        if ((int)blockIdx.x < p.total_tiles) {
          const int tile = blockIdx.x;
          const int ks = tile % p.split_k;
          const int m = tile_m(tile / p.split_k);
          const int kb0 = (int)((long long)ks * p.k_blocks / p.split_k);
          const int kb1 = (int)((long long)(ks + 1) * p.k_blocks / p.split_k);
          pre = (uint32_t)min(kb1 - kb0, STAGES);
          for (uint32_t j = 0; j < pre; ++j) {
            mbar_arrive_expect_tx(&full[j], L::STAGE_BYTES);
            load_a(smem + j * L::STAGE_BYTES, &full[j], m, (kb0 + (int)j) * (TF32 ? 32 : 64));
          }
        }
        pdl_wait();
      }
      uint32_t it = 0;
      // the first tile is always entered when it has A tiles in flight: their stages get
      // their B loads before any wait, so the drain below finds every issued stage complete
      for (int tile = tile0; tile < p.total_tiles && (it < pre || !*abort_flag); tile += tile_step) {
        const int ks = tile % p.split_k;
        const int t2 = tile / p.split_k;
        const int m = tile_m(t2);
        const int n = tile_n(t2);
        const int kb0 = (int)((long long)ks * p.k_blocks / p.split_k);
        const int kb1 = (int)((long long)(ks + 1) * p.k_blocks / p.split_k);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          uint8_t* sa = smem + s * L::STAGE_BYTES;
          uint8_t* sb = sa + L::A_BYTES;
          const int kc = kb * (TF32 ? 32 : 64);
          if constexpr (PAIR) {
            // both CTAs' A tiles and B halves complete on the even CTA's full[s]; that CTA
            // expects the bytes of both
            if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, 101)) break;
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * L::STAGE_BYTES);
            const uint32_t bar = smem_cluster_addr(&full[s], 0);
            if (m < p.tiles0) {
              tma_load_2d_pair(sa, &mapA0, bar, kc, m * GEMM_BM);
            } else {
              const int idx = m - p.tiles0;   // past the last tile (odd count): a zero-filled tile
              tma_load_3d_pair(sa, &mapA1, bar, kc, (idx % p.tiles1) * GEMM_BM, idx / p.tiles1);
            }
            tma_load_2d_pair(sb, &mapB, bar, kc, n * BN + (int)rank * (BN / 2));
          } else {
            if (it >= pre) {
              if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, 101)) break;
              mbar_arrive_expect_tx(&full[s], L::STAGE_BYTES);
              load_a(sa, &full[s], m, kc);
            }
            tma_load_2d(sb, &mapB, &full[s], kc, n * BN);
          }
        }
      }
      // Drain: wait until every load issued has landed (their consumer may have given up).
      // PAIR: the loads complete on the even CTA's barriers, which that CTA drains; the odd
      // CTA's last loads have landed once the even CTA's MMAs have consumed them, before the
      // closing cluster barrier.
      if (!PAIR || rank == 0) {
        for (uint32_t j = (it > (uint32_t)STAGES ? it - STAGES : 0u); j < it; ++j) {
          mbar_wait(&full[j % STAGES], (j / STAGES) & 1u, nullptr, p.status, 102);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    // PAIR: the even CTA's thread issues the pair's MMAs; the odd CTA's warp 1 only holds TMEM
    if (lane == 0 && (!PAIR || rank == 0)) {
      uint32_t it = 0;
      int lt = 0;
      for (int tile = tile0; tile < p.total_tiles && !*abort_flag; tile += tile_step, ++lt) {
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
            if constexpr (PAIR) umma_f16_pair(d_tmem, ad, bd, IDESC, acc);
            else if (TF32) umma_tf32(d_tmem, ad, bd, IDESC, acc);
            else umma_f16(d_tmem, ad, bd, IDESC, acc);
          }
          if constexpr (PAIR) {   // both CTAs' stage s is free
            umma_commit_pair(smem_cluster_addr(&empty[s], 0));
            umma_commit_pair(smem_cluster_addr(&empty[s], 1));
          } else {
            umma_commit(&empty[s]);
          }
        }
        if (!ok) break;
        if constexpr (PAIR) {
          umma_commit_pair(smem_cluster_addr(&acc_full[ab], 0));
          umma_commit_pair(smem_cluster_addr(&acc_full[ab], 1));
        } else {
          umma_commit(&acc_full[ab]);
        }
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int quad = warp & 3;               // TMEM lanes this warp may access
    const int half = (warp - 2) >> 2;        // which of the quadrant's two warps (column chunks)
    const int r = quad * 32 + lane;          // accumulator row of this thread
    int lt = 0;
    for (int tile = tile0; tile < p.total_tiles; tile += tile_step, ++lt) {
      const int ks = tile % p.split_k;
      const int t2 = tile / p.split_k;
      const int m = tile_m(t2);
      const int n = tile_n(t2);
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
      const bool row_ok = m < p.m_tiles && (src0 ? (rr < p.rows0) : (rr < p.rows1));
      const int col_base = n * BN;

      if constexpr (MODE == EPI_PROJ || MODE == EPI_SWIGLU) {
        // 64-column chunks (both 32-column halves loaded before one wait); the two warps
        // of a quadrant take alternate chunks
        static_assert(BN % 64 == 0, "64-column epilogue needs BN % 64 == 0");
        const size_t orow = (size_t)b1 * p.rows1 + rr;
#pragma unroll 1
        for (int c0 = 64 * half; c0 < BN; c0 += 128) {
          uint32_t r[64];
          tmem_ld32_async(tbase + c0, r);
          tmem_ld32_async(tbase + c0 + 32, r + 32);
          tmem_wait_ld_regs(r);
          tmem_wait_ld_regs(r + 32);
          float* v = reinterpret_cast<float*>(r);
          const int gc = col_base + c0;
          if (!row_ok || gc >= p.N) continue;
          if constexpr (MODE == EPI_SWIGLU) {   // fp16 activations (the down projection runs in fp16)
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = silu_f(v[e]) * v[e + 32];
            f16_range_guard<32>(v, p.status, 121);
            store_f16_row(reinterpret_cast<__half*>(p.out) + orow * p.ld_out + gc / 2, v, 32);
          } else {
            int si = 0;
#pragma unroll 1
            while (si < p.nseg - 1 && gc >= p.seg[si].col_end) ++si;
            const Segment& sg = p.seg[si];
            const int pos = src0 ? rr : p.row_off1 + rr;
            if (sg.rope) rope_pair_rotate(v, p.rope_tab + (size_t)pos * 32);
            if (sg.f16) f16_range_guard<64>(v, p.status, 120);
            __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(sg.ptr) + (gc - sg.col_begin);
            const int b_lo = src0 ? 0 : b1, b_hi = src0 ? p.out_batches : b1 + 1;
            for (int b = b_lo; b < b_hi; ++b) {
              __nv_bfloat16* dst = base + b * sg.bstride + (size_t)pos * sg.ld;
              if (sg.f16) store_f16_row(dst, v, 64);
              else store_bf16_row(dst, v, 64);
            }
            if (sg.meta != nullptr && (pos < sg.M || pos >= sg.win0)) {
              const int col = gc - sg.col_begin;
              for (int b = b_lo; b < b_hi; ++b) {
                __half* dst = pos < sg.M
                                  ? reinterpret_cast<__half*>(sg.meta) + ((size_t)b * sg.M + pos) * sg.ld + col
                                  : reinterpret_cast<__half*>(sg.ring) + ((size_t)b * sg.W + (pos - sg.M) % sg.W) * sg.ld + col;
                store_f16_row(dst, v, 64);
              }
            }
          }
        }
      } else {
        // 32-column chunks j = half, half+2, ...; the next chunk's TMEM load is in flight
        // while this one is processed
        static_assert(BN % 32 == 0, "BN % 32 == 0");
        constexpr int NCH = BN / 32;
        const size_t orow = (size_t)b1 * p.rows1 + rr;
        auto process = [&](uint32_t* r, int c0) {
          float* v = reinterpret_cast<float*>(r);
          const int gc = col_base + c0;
          if constexpr (MODE == EPI_F32_T || MODE == EPI_F32_T_PART) {
            // accumulator row = output column (weight row), accumulator column = output row
            if (!row_ok || rr >= p.m_valid) return;
            float* outf = reinterpret_cast<float*>(p.out) + (MODE == EPI_F32_T_PART ? ks * p.split_stride : 0);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int orow_t = gc + e;
              if (orow_t < p.n_valid) outf[(size_t)orow_t * p.ld_out + rr] = v[e];
            }
            return;
          }
          if constexpr (MODE == EPI_BF16) {
            // whole 32-column chunks: the residual comes in and the result goes out through
            // this warp's staging block, rows read and written by four lanes each (all lanes
            // take part; rows past the tile's valid rows are neither read nor written)
            if (gc >= p.n_valid) return;          // the same for the whole warp
            if (gc + 32 <= p.n_valid) {
              uint32_t* tile = reinterpret_cast<uint32_t*>(smem + L::EPI_OFFSET) + (warp - 2) * (32 * GEMM_BF16_TILE_WORDS);
              const int rows_valid = src0 ? p.rows0 : p.rows1;
              const int rr0 = rr - lane;            // accumulator row of lane 0
              const size_t orow0 = (size_t)b1 * p.rows1 + rr0;
              const int pr = lane >> 2, pc = lane & 3;   // row in a group of 8, 16-byte piece
              const bool tile_ok = m < p.m_tiles;
              if (p.residual != nullptr) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int j = pr + 8 * i;
                  if (tile_ok && rr0 + j < rows_valid)
                    *reinterpret_cast<uint4*>(tile + j * GEMM_BF16_TILE_WORDS + pc * 4) =
                        *reinterpret_cast<const uint4*>(p.residual + (orow0 + j) * p.ld_res + gc + pc * 8);
                }
                __syncwarp();
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                  const uint4 raw = *reinterpret_cast<const uint4*>(tile + lane * GEMM_BF16_TILE_WORDS + e / 2);
                  const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
                  for (int k = 0; k < 8; ++k) v[e + k] += __bfloat162float(hv[k]);
                }
                __syncwarp();
              }
#pragma unroll
              for (int e = 0; e < 32; e += 8)
                *reinterpret_cast<uint4*>(tile + lane * GEMM_BF16_TILE_WORDS + e / 2) =
                    make_uint4(pack_bf16x2(v[e], v[e + 1]), pack_bf16x2(v[e + 2], v[e + 3]),
                               pack_bf16x2(v[e + 4], v[e + 5]), pack_bf16x2(v[e + 6], v[e + 7]));
              __syncwarp();
              __nv_bfloat16* outb = reinterpret_cast<__nv_bfloat16*>(p.out);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int j = pr + 8 * i;
                if (tile_ok && rr0 + j < rows_valid) {
                  const uint4 w = *reinterpret_cast<const uint4*>(tile + j * GEMM_BF16_TILE_WORDS + pc * 4);
                  st_global_v4(outb + (orow0 + j) * p.ld_out + gc + pc * 8, w.x, w.y, w.z, w.w);
                }
              }
              __syncwarp();
              return;
            }
          }
          if (!row_ok || gc >= p.n_valid) return;
          const bool whole = gc + 32 <= p.n_valid;
          if constexpr (MODE == EPI_BF16) {
            if (p.residual != nullptr) {
              const __nv_bfloat16* res = p.residual + orow * p.ld_res + gc;
              if (whole) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                  float f[8];
                  const uint4 raw = *reinterpret_cast<const uint4*>(res + e);
                  const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
                  for (int k = 0; k < 8; ++k) f[k] = __bfloat162float(hv[k]);
#pragma unroll
                  for (int k = 0; k < 8; ++k) v[e + k] += f[k];
                }
              } else {
                for (int e = 0; e < 32; ++e)
                  if (gc + e < p.n_valid) v[e] += __bfloat162float(res[e]);
              }
            }
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + orow * p.ld_out + gc;
            if (whole) store_bf16_row(dst, v, 32);
            else
              for (int e = 0; e < 32; ++e)
                if (gc + e < p.n_valid) dst[e] = __float2bfloat16_rn(v[e]);
          } else if constexpr (MODE == EPI_F32_PART) {
            // fp32 partial sums, 4-wide (ld_out and n_valid are multiples of 4)
            float* dst = reinterpret_cast<float*>(p.out) + ks * p.split_stride + orow * p.ld_out + gc;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              if (gc + e < p.n_valid)
                *reinterpret_cast<float4*>(dst + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
          }
        };
        uint32_t ra[32], rb[32];
        if (half < NCH) {
          tmem_ld32_async(tbase + 32 * half, ra);
          tmem_wait_ld_regs(ra);
        }
#pragma unroll 1
        for (int j = half; j < NCH; j += 4) {
          const bool has_b = j + 2 < NCH;
          if (has_b) tmem_ld32_async(tbase + 32 * (j + 2), rb);
          process(ra, 32 * j);
          if (has_b) {
            tmem_wait_ld_regs(rb);
            const bool has_a = j + 4 < NCH;
            if (has_a) tmem_ld32_async(tbase + 32 * (j + 4), ra);
            process(rb, 32 * (j + 2));
            if (has_a) tmem_wait_ld_regs(ra);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(smem_cluster_addr(&acc_empty[ab], 0));
        else mbar_arrive(&acc_empty[ab]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // no CTA leaves while the other may still signal or read it
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace hymba
