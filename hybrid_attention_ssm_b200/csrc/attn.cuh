// Prefill attention on tcgen05 for sm_100a: head dim 64, GQA, RoPE already applied, fp16
// Q/K/V/P (keys, values and probabilities sit far inside fp16's range, where it rounds 8x
// finer than bf16), fp32 scores and accumulators.
//
// Persistent: two CTAs per SM (256 TMEM columns and 113 KB of shared memory each), so one
// CTA's softmax overlaps the other's MMAs, loop over the (query tile of 128 rows, query head,
// sequence) work items, heaviest first and dealt in a snake order over the CTAs
// (attn_slot_item), so that no CTA is left with a much longer list than the rest.  The TMA
// warp prefetches the next item's Q and K/V while the current item finishes.  The key tiles
// a CTA visits are the meta-token tiles plus the tiles that intersect the sliding window of
// its rows (every causal tile for a global layer): block skipping, no dense mask.  Only
// tiles that straddle the causal diagonal or the window edge apply an element mask.
//
// 192 threads:
//   warp 0      TMA: Q once, K/V tiles through a 3-stage ring
//   warp 1      TMEM allocation and MMA issue: S = Q K^T (M128 N128 K64) into TMEM, and
//               O += P V with P read straight from TMEM (the "A in tensor memory" form).
//               S(i+1) is issued as soon as the softmax has read S(i), so it runs on the
//               tensor core while the softmax of tile i is still computing P(i).
//   warps 2..5  softmax, one query row per thread: the whole S row comes into registers
//               with one wait, P = 2^(s - m) is packed to fp16 into its own TMEM columns;
//               O stays in TMEM and is rescaled only when the running max grows by more
//               than 2^8 (P <= 256 otherwise), then divided by the row sum at the end.
// TMEM columns: S 0..127, P 128..191 (fp16 pairs), O 192..255.
#pragma once
#include "common.cuh"

namespace hymba {

struct AttnParams {
  int T;              // rows per sequence (meta included)
  int q_off;          // first query row (M when the meta rows come from a precomputed prefix)
  int Hq, Hkv;
  int n_meta, window, is_global;
  int q_tiles;        // tiles of 128 query rows over rows q_off .. T-1
  int n_items;        // q_tiles * Hq * B work items
  float scale_log2;   // log2(e) / sqrt(head_dim)
  float* out;         // O [B*T, ld_out] fp32, head h at columns h*64
  int ld_out;
  DevStatus* status;
};

constexpr int ATT_THREADS = 192;
constexpr int ATT_Q_BYTES = 128 * 128;
constexpr int ATT_KV_BYTES = 128 * 128;          // one K or V tile: 128 keys x 64 dims fp16
// Shared-memory layout for a K/V ring of STAGES tile pairs: Q, K ring, V ring, barriers.
template <int STAGES>
struct AttnLayout {
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + ATT_Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * ATT_KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * ATT_KV_BYTES;
  static constexpr int USED = OFF_BAR + 160;
  // requested dynamic shared memory: the tiles and barriers plus up to 1 KB to align the
  // window.  3 stages: 113 KB, the most two CTAs can each take on one SM (228 KB, 1 KB
  // reserved per CTA), which also keeps a third CTA (which would wait for TMEM) off the
  // SM.  2 stages: 82 KB, for a prefill that runs this kernel beside the selective scan
  // (one attention CTA and three scan CTAs per SM).
  static constexpr int SMEM = STAGES == 3 ? 113 * 1024 : (USED + 1023 + 1023) / 1024 * 1024;
};
// (the kernel checks at run time that the aligned window holds the layout)
static_assert(AttnLayout<3>::USED <= AttnLayout<3>::SMEM, "3-stage layout fits");
static_assert(AttnLayout<2>::USED + 1023 <= AttnLayout<2>::SMEM, "2-stage layout fits");
constexpr uint32_t ATT_TMEM_COLS = 256;
constexpr float ATT_RESCALE_LOG2 = 8.f;          // lazy rescale threshold (P <= 2^8)

// Key tiles (128 keys each) visited by query tile qt, in order: meta tiles first, then the
// window.
struct KeyTiles {
  int n_meta_tiles;   // leading meta tiles that precede the window range
  int lo, hi;         // window tile range [lo, hi]
  __device__ __forceinline__ int count() const { return n_meta_tiles + (hi - lo + 1); }
  __device__ __forceinline__ int tile(int i) const { return i < n_meta_tiles ? i : lo + (i - n_meta_tiles); }
};

__device__ __forceinline__ KeyTiles key_tiles(const AttnParams& p, int qt) {
  KeyTiles kt;
  const int t0 = p.q_off + qt * 128;
  const int t1 = min(t0 + 127, p.T - 1);
  kt.hi = t1 >> 7;
  if (p.is_global) {
    kt.lo = 0;
    kt.n_meta_tiles = 0;
  } else {
    const int first = t0 - p.window + 1;
    kt.lo = first <= 0 ? 0 : (first >> 7);
    const int meta_tiles = (p.n_meta + 127) >> 7;
    kt.n_meta_tiles = min(meta_tiles, kt.lo);
  }
  return kt;
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 128 fp32 columns of TMEM into registers with a single completion wait.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float* v) {
  uint32_t r[128];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
        : "=r"(r[c * 32 + 0]), "=r"(r[c * 32 + 1]), "=r"(r[c * 32 + 2]), "=r"(r[c * 32 + 3]), "=r"(r[c * 32 + 4]),
          "=r"(r[c * 32 + 5]), "=r"(r[c * 32 + 6]), "=r"(r[c * 32 + 7]), "=r"(r[c * 32 + 8]), "=r"(r[c * 32 + 9]),
          "=r"(r[c * 32 + 10]), "=r"(r[c * 32 + 11]), "=r"(r[c * 32 + 12]), "=r"(r[c * 32 + 13]),
          "=r"(r[c * 32 + 14]), "=r"(r[c * 32 + 15]), "=r"(r[c * 32 + 16]), "=r"(r[c * 32 + 17]),
          "=r"(r[c * 32 + 18]), "=r"(r[c * 32 + 19]), "=r"(r[c * 32 + 20]), "=r"(r[c * 32 + 21]),
          "=r"(r[c * 32 + 22]), "=r"(r[c * 32 + 23]), "=r"(r[c * 32 + 24]), "=r"(r[c * 32 + 25]),
          "=r"(r[c * 32 + 26]), "=r"(r[c * 32 + 27]), "=r"(r[c * 32 + 28]), "=r"(r[c * 32 + 29]),
          "=r"(r[c * 32 + 30]), "=r"(r[c * 32 + 31])
        : "r"(taddr + c * 32)
        : "memory");
  }
  // the wait takes every loaded register as an operand so no use can move above it
#pragma unroll
  for (int i = 0; i < 128; i += 32) {
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;\n"
        : "+r"(r[i + 0]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]), "+r"(r[i + 5]),
          "+r"(r[i + 6]), "+r"(r[i + 7]), "+r"(r[i + 8]), "+r"(r[i + 9]), "+r"(r[i + 10]), "+r"(r[i + 11]),
          "+r"(r[i + 12]), "+r"(r[i + 13]), "+r"(r[i + 14]), "+r"(r[i + 15]), "+r"(r[i + 16]), "+r"(r[i + 17]),
          "+r"(r[i + 18]), "+r"(r[i + 19]), "+r"(r[i + 20]), "+r"(r[i + 21]), "+r"(r[i + 22]), "+r"(r[i + 23]),
          "+r"(r[i + 24]), "+r"(r[i + 25]), "+r"(r[i + 26]), "+r"(r[i + 27]), "+r"(r[i + 28]), "+r"(r[i + 29]),
          "+r"(r[i + 30]), "+r"(r[i + 31])
        :
        : "memory");
  }
#pragma unroll
  for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 32 columns of 32-bit values from registers into TMEM (completion is awaited
// with tmem_wait_st before the data is handed to the tensor core).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// The work item a CTA takes on its k-th pass over the grid: passes go through the items in
// order (longest query tiles first), the odd passes in reverse CTA order, so the CTAs whose
// first item was among the shortest of its pass get the longest of the next (a snake order).
// Item indices grow with k for every CTA, so the first index past the end ends the loop.
__device__ __forceinline__ int attn_slot_item(int k, int grid, int cta) {
  return k * grid + ((k & 1) ? grid - 1 - cta : cta);
}

// work item w -> (query tile, head, sequence); longest query tiles first
__device__ __forceinline__ void attn_item(const AttnParams& p, int w, int B, int& qt, int& h, int& b) {
  const int per_qt = p.Hq * B;
  qt = p.q_tiles - 1 - w / per_qt;
  const int r = w % per_qt;
  h = r % p.Hq;
  b = r / p.Hq;
}

template <int ATT_STAGES>
__global__ void __launch_bounds__(ATT_THREADS, 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                    const __grid_constant__ CUtensorMap mapV, const __grid_constant__ AttnParams p, int B) {
  using AL = AttnLayout<ATT_STAGES>;
  constexpr int ATT_OFF_Q = AL::OFF_Q, ATT_OFF_K = AL::OFF_K, ATT_OFF_V = AL::OFF_V, ATT_OFF_BAR = AL::OFF_BAR;
  constexpr int ATT_USED = AL::USED, ATT_SMEM = AL::SMEM;
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem<1024>(smem_raw);
  if ((size_t)(smem - smem_raw) + ATT_USED > (size_t)ATT_SMEM) {   // cannot happen with a 1 KB-aligned window
    if (threadIdx.x == 0) report_error(p.status, DEV_ERR_BOUNDS, 299);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ATT_OFF_BAR);
  uint64_t* q_full = bars;                   // Q of the current item loaded
  uint64_t* q_empty = bars + 1;              // every S of the current item issued and done
  uint64_t* kv_full = bars + 2;              // ATT_STAGES
  uint64_t* kv_empty = kv_full + ATT_STAGES; // ATT_STAGES
  uint64_t* s_full = kv_empty + ATT_STAGES;  // S(i) in TMEM
  uint64_t* s_free = s_full + 1;             // softmax has read S(i)
  uint64_t* p_full = s_free + 1;             // P(i) in TMEM (and O rescaled)
  uint64_t* o_done = p_full + 1;             // PV(i) complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < ATT_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, ATT_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t TM_S = tmem, TM_P = tmem + 128, TM_O = tmem + 192;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      int gi = 0, it = 0;                    // tiles and items issued by this CTA
      bool ok = true;
      for (int k = 0, w = attn_slot_item(0, gridDim.x, blockIdx.x); ok && w < p.n_items;
           ++k, w = attn_slot_item(k, gridDim.x, blockIdx.x), ++it) {
        int qt, h, b;
        attn_item(p, w, B, qt, h, b);
        const int g = (h * p.Hkv) / p.Hq;
        const KeyTiles kts = key_tiles(p, qt);
        if (it > 0 && !mbar_wait(q_empty, (it - 1) & 1u, abort_flag, p.status, 200)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, ATT_Q_BYTES);
        tma_load_3d(smem + ATT_OFF_Q, &mapQ, q_full, h * 64, p.q_off + qt * 128, b);
        for (int i = 0; i < kts.count(); ++i, ++gi) {
          const int s = gi % ATT_STAGES;
          if (!mbar_wait(&kv_empty[s], ((gi / ATT_STAGES) & 1u) ^ 1u, abort_flag, p.status, 201)) {
            ok = false;
            break;
          }
          const int kt = kts.tile(i);
          mbar_arrive_expect_tx(&kv_full[s], 2 * ATT_KV_BYTES);
          tma_load_3d(smem + ATT_OFF_K + s * ATT_KV_BYTES, &mapK, &kv_full[s], g * 64, kt * 128, b);
          tma_load_3d(smem + ATT_OFF_V + s * ATT_KV_BYTES, &mapV, &kv_full[s], g * 64, kt * 128, b);
        }
      }
      // drain every load still in flight
      if (it > 0) mbar_wait(q_full, (it - 1) & 1u, nullptr, p.status, 202);
      for (int j = max(0, gi - ATT_STAGES); j < gi; ++j)
        mbar_wait(&kv_full[j % ATT_STAGES], (j / ATT_STAGES) & 1u, nullptr, p.status, 203);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t IDESC_S = make_idesc(128, 128, 0u, false, false);   // fp16 Q, K (K-major)
      constexpr uint32_t IDESC_O = make_idesc(128, 64, 0u, false, true);     // fp16 P (TMEM), V MN-major
      const uint32_t sq = smem_u32(smem + ATT_OFF_Q);
      // O (+)= P(gj) V(gj): P in its TMEM columns, 8 steps of 16 keys (8 columns each)
      auto issue_pv = [&](int gj, bool first) -> bool {
        if (!mbar_wait(p_full, gj & 1u, abort_flag, p.status, 205)) return false;
        tc_fence_after();
        const int s = gj % ATT_STAGES;
        const uint32_t sv = smem_u32(smem + ATT_OFF_V + s * ATT_KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = make_sdesc_sw128(sv + kk * 2048, 8192, 1024);
          umma_f16_tmem_a(TM_O, TM_P + kk * 8, bd, IDESC_O, (!first || kk > 0) ? 1u : 0u);
        }
        umma_commit(o_done);
        umma_commit(&kv_empty[s]);
        return true;
      };
      int gi = 0, it = 0;
      bool ok = true;
      for (int k = 0, w = attn_slot_item(0, gridDim.x, blockIdx.x); ok && w < p.n_items;
           ++k, w = attn_slot_item(k, gridDim.x, blockIdx.x), ++it) {
        int qt, h, b;
        attn_item(p, w, B, qt, h, b);
        const int n_tiles = key_tiles(p, qt).count();
        if (!mbar_wait(q_full, it & 1u, abort_flag, p.status, 204)) { ok = false; break; }
        for (int i = 0; i < n_tiles; ++i, ++gi) {
          const int s = gi % ATT_STAGES;
          if (!mbar_wait(&kv_full[s], (gi / ATT_STAGES) & 1u, abort_flag, p.status, 206)) { ok = false; break; }
          if (gi >= 1 && !mbar_wait(s_free, (gi - 1) & 1u, abort_flag, p.status, 209)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sk = smem_u32(smem + ATT_OFF_K + s * ATT_KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_sdesc_sw128(sq + kk * 32, 16, 1024);
            const uint64_t bd = make_sdesc_sw128(sk + kk * 32, 16, 1024);
            umma_f16(TM_S, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(s_full);
          if (i == n_tiles - 1) umma_commit(q_empty);          // Q no longer read
          if (i >= 1 && !issue_pv(gi - 1, i == 1)) { ok = false; break; }
        }
        if (ok && n_tiles > 0 && !issue_pv(gi - 1, n_tiles == 1)) ok = false;
      }
    }
  } else {
    // ------------------------------ softmax warps ------------------------------
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;

    auto wait_bar = [&](uint64_t* bar, int j, unsigned site) -> bool {   // warp-uniform
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar, j & 1u, abort_flag, p.status, site) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok) tc_fence_after();
      return ok != 0;
    };

    int gi = 0;
    bool ok = true;
    for (int k = 0, w = attn_slot_item(0, gridDim.x, blockIdx.x); ok && w < p.n_items;
         ++k, w = attn_slot_item(k, gridDim.x, blockIdx.x)) {
      int qt, h, b;
      attn_item(p, w, B, qt, h, b);
      const KeyTiles kts = key_tiles(p, qt);
      const int n_tiles = kts.count();
      const int t0 = p.q_off + qt * 128;
      const int qi = t0 + r;                     // absolute query position
      float m_run = -INFINITY, l_run = 0.f;
      for (int i = 0; i < n_tiles; ++i, ++gi) {
        if (!wait_bar(s_full, gi, 208)) { ok = false; break; }
        const int j0 = kts.tile(i) * 128;
        const bool causal_full = j0 + 127 <= t0;
        const bool window_full = p.is_global || j0 + 127 < p.n_meta || (t0 + 127) - j0 < p.window;
        float s[128];
        tmem_ld128(TM_S + lane_off, s);
        tc_fence_before();
        mbar_arrive(s_free);                     // the tensor core may compute S(i+1) now
        // row max of the raw scores (the positive scale keeps the order), 8 independent
        // partial maxima; invisible keys become -inf (tile kinds: full, diagonal only,
        // window edge only, both)
        float mxp[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mxp[k] = -INFINITY;
        const int e_hi = qi - j0;                          // causal: e <= e_hi
        const int e_lo = qi - p.window + 1 - j0;           // window: e >= e_lo
        const int e_meta = p.n_meta - j0;                  // meta: e < e_meta
        if (causal_full && window_full) {
#pragma unroll
          for (int e = 0; e < 128; e += 16)
#pragma unroll
            for (int k = 0; k < 8; ++k) mxp[k] = fmax3(mxp[k], s[e + k], s[e + 8 + k]);
        } else if (window_full) {
#pragma unroll
          for (int e = 0; e < 128; ++e) {
            s[e] = e <= e_hi ? s[e] : -INFINITY;
            mxp[e & 7] = fmaxf(mxp[e & 7], s[e]);
          }
        } else if (causal_full) {
#pragma unroll
          for (int e = 0; e < 128; ++e) {
            s[e] = (e >= e_lo || e < e_meta) ? s[e] : -INFINITY;
            mxp[e & 7] = fmaxf(mxp[e & 7], s[e]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 128; ++e) {
            s[e] = (e <= e_hi && (e >= e_lo || e < e_meta)) ? s[e] : -INFINITY;
            mxp[e & 7] = fmaxf(mxp[e & 7], s[e]);
          }
        }
        const float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                               fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]))) * p.scale_log2;
        // running max (log2 units): rescale O (in TMEM) only when it grows by more than 2^8
        float alpha = 1.f;
        bool resc = false;
        if (m_run == -INFINITY) {
          m_run = mx;                             // nothing accumulated for this row yet
        } else if (mx > m_run + ATT_RESCALE_LOG2) {
          alpha = exp2f(m_run - mx);
          m_run = mx;
          resc = true;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        float rsp[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) rsp[k] = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int e = 0; e < 128; e += 2) {
          const float p0 = ex2_approx(fmaf(s[e], p.scale_log2, -m_use));
          const float p1 = ex2_approx(fmaf(s[e + 1], p.scale_log2, -m_use));
          rsp[(e >> 1) & 7] += p0 + p1;
          pk[e >> 1] = pack_f16x2(p0, p1);
        }
        // the sum so far was taken against the old maximum: rescale it before this tile's
        // terms (taken against the new one) are added (alpha = 1 without a rescale)
        l_run = fmaf(l_run, alpha, ((rsp[0] + rsp[1]) + (rsp[2] + rsp[3])) + ((rsp[4] + rsp[5]) + (rsp[6] + rsp[7])));
        // PV of the previous tile must be done before P is replaced and O rescaled
        if (i >= 1 && !wait_bar(o_done, gi - 1, 207)) { ok = false; break; }
        if (__any_sync(0xffffffffu, resc)) {
          float o[32];
#pragma unroll
          for (int hcol = 0; hcol < 64; hcol += 32) {
            tmem_ld32(TM_O + lane_off + hcol, o);
#pragma unroll
            for (int d = 0; d < 32; ++d) o[d] *= alpha;
            tmem_st32(TM_O + lane_off + hcol, reinterpret_cast<const uint32_t*>(o));
          }
        }
        tmem_st32(TM_P + lane_off, pk);
        tmem_st32(TM_P + lane_off + 32, pk + 32);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full);
      }
      if (!ok || n_tiles == 0) break;
      if (!wait_bar(o_done, gi - 1, 210)) { ok = false; break; }
      float o[64];
      tmem_ld32(TM_O + lane_off, o);
      tmem_ld32(TM_O + lane_off + 32, o + 32);
      tc_fence_before();
      if (qi < p.T) {
        const float inv = 1.f / l_run;
        float* dst = p.out + ((size_t)b * p.T + qi) * p.ld_out + h * 64;
#pragma unroll
        for (int d = 0; d < 64; d += 4)
          *reinterpret_cast<float4*>(dst + d) = make_float4(o[d] * inv, o[d + 1] * inv, o[d + 2] * inv, o[d + 3] * inv);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, ATT_TMEM_COLS);
  }
}

}  // namespace hymba
