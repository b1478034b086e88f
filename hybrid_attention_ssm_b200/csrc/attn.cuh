// Prefill attention on tcgen05 for sm_100a, head dim 64, GQA, RoPE already applied.
// Q, K, V and the probabilities P are fp16 (P in [0, 1] and the normalised-input
// activations sit well inside fp16's range, where it rounds 8x finer than bf16); scores and
// the output accumulate in fp32.
//
// One CTA per (query tile of 128 rows, query head, sequence).  The key tiles a CTA visits
// are the meta-token tiles plus the tiles that intersect the sliding window of its rows
// (or every causal tile for a global layer): block skipping, no dense mask.  Only tiles
// that straddle the causal diagonal or the window edge apply an element mask.
//
// 192 threads: warp 0 issues TMA loads (Q once, K/V tiles through a 2-stage ring),
// warp 1 allocates TMEM and issues the MMAs (S = Q K^T into a double-buffered TMEM tile,
// O_j = P_j V_j into a double-buffered TMEM tile), warps 2..5 run the online softmax with
// one query row per thread, write P (fp16) into 128B-swizzled shared memory for the PV
// MMA, and accumulate O in registers.
#pragma once
#include "common.cuh"

namespace hymba {

struct AttnParams {
  int T;              // rows per sequence (meta included)
  int Hq, Hkv;
  int n_meta, window, is_global;
  int q_tiles;
  float scale_log2;   // log2(e) / sqrt(head_dim)
  float* out;         // O [B*T, ld_out] fp32, head h at columns h*64
  int ld_out;
  DevStatus* status;
};

constexpr int ATT_THREADS = 192;
constexpr int ATT_STAGES = 2;
constexpr int ATT_Q_BYTES = 128 * 128;
constexpr int ATT_KV_BYTES = 128 * 128;          // one K or V tile: 128 keys x 64 dims fp16
constexpr int ATT_P_BYTES = 128 * 256;           // P tile: 128 rows x 128 keys fp16
constexpr int ATT_OFF_Q = 0;
constexpr int ATT_OFF_K = ATT_OFF_Q + ATT_Q_BYTES;
constexpr int ATT_OFF_V = ATT_OFF_K + ATT_STAGES * ATT_KV_BYTES;
constexpr int ATT_OFF_P = ATT_OFF_V + ATT_STAGES * ATT_KV_BYTES;
constexpr int ATT_OFF_BAR = ATT_OFF_P + 2 * ATT_P_BYTES;
constexpr int ATT_SMEM = ATT_OFF_BAR + 256 + 1024;

// Key tiles (128 keys each) visited by query tile qt, in order: meta tiles first, then the
// window.  Returns the count; tile(i) gives the i-th key-tile index.
struct KeyTiles {
  int n_meta_tiles;   // leading meta tiles that precede the window range
  int lo, hi;         // window tile range [lo, hi]
  __device__ __forceinline__ int count() const { return n_meta_tiles + (hi - lo + 1); }
  __device__ __forceinline__ int tile(int i) const { return i < n_meta_tiles ? i : lo + (i - n_meta_tiles); }
};

__device__ __forceinline__ KeyTiles key_tiles(const AttnParams& p, int qt) {
  KeyTiles kt;
  const int t0 = qt * 128;
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

__global__ void __launch_bounds__(ATT_THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                    const __grid_constant__ CUtensorMap mapV, const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ATT_OFF_BAR);
  uint64_t* q_full = bars;                 // 1
  uint64_t* kv_full = bars + 1;            // ATT_STAGES
  uint64_t* kv_empty = kv_full + ATT_STAGES;
  uint64_t* s_full = kv_empty + ATT_STAGES;  // 2
  uint64_t* p_full = s_full + 2;             // 2
  uint64_t* o_full = p_full + 2;             // 2
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_full + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = p.q_tiles - 1 - blockIdx.x;     // longest rows first
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int g = (h * p.Hkv) / p.Hq;
  const KeyTiles kts = key_tiles(p, qt);
  const int n_tiles = kts.count();

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < ATT_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_full[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;   // S0: +0, S1: +128, O0: +256, O1: +320

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      mbar_arrive_expect_tx(q_full, ATT_Q_BYTES);
      tma_load_3d(smem + ATT_OFF_Q, &mapQ, q_full, h * 64, qt * 128, b);
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % ATT_STAGES;
        const uint32_t ph = (i / ATT_STAGES) & 1u;
        if (!mbar_wait(&kv_empty[s], ph ^ 1u, abort_flag, p.status, 201)) break;
        const int kt = kts.tile(i);
        mbar_arrive_expect_tx(&kv_full[s], 2 * ATT_KV_BYTES);
        tma_load_3d(smem + ATT_OFF_K + s * ATT_KV_BYTES, &mapK, &kv_full[s], g * 64, kt * 128, b);
        tma_load_3d(smem + ATT_OFF_V + s * ATT_KV_BYTES, &mapV, &kv_full[s], g * 64, kt * 128, b);
        issued = i + 1;
      }
      // drain every load still in flight
      mbar_wait(q_full, 0, nullptr, p.status, 202);
      for (int j = max(0, issued - ATT_STAGES); j < issued; ++j)
        mbar_wait(&kv_full[j % ATT_STAGES], (j / ATT_STAGES) & 1u, nullptr, p.status, 203);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC_S = make_idesc(128, 128, 0u, false, false);   // fp16 Q, K
      constexpr uint32_t IDESC_O = make_idesc(128, 64, 0u, false, true);     // fp16 P, V (MN-major)
      const uint32_t sq = smem_u32(smem + ATT_OFF_Q);
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status, 204);
      // PV of tile j: O[j%2] = P[j%2] * V[stage of j]
      auto issue_pv = [&](int j) -> bool {
        const int pb = j & 1;
        if (!mbar_wait(&p_full[pb], (j >> 1) & 1u, abort_flag, p.status, 205)) return false;
        tc_fence_after();
        const int s = j % ATT_STAGES;
        const uint32_t sp = smem_u32(smem + ATT_OFF_P + pb * ATT_P_BYTES);
        const uint32_t sv = smem_u32(smem + ATT_OFF_V + s * ATT_KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = make_sdesc_sw128(sp + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = make_sdesc_sw128(sv + kk * 2048, 8192, 1024);
          umma_f16(tmem + 256 + pb * 64, ad, bd, IDESC_O, kk > 0 ? 1u : 0u);
        }
        umma_commit(&o_full[pb]);
        umma_commit(&kv_empty[s]);
        return true;
      };
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int s = i % ATT_STAGES;
        if (!mbar_wait(&kv_full[s], (i / ATT_STAGES) & 1u, abort_flag, p.status, 206)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sk = smem_u32(smem + ATT_OFF_K + s * ATT_KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = make_sdesc_sw128(sq + kk * 32, 16, 1024);
          const uint64_t bd = make_sdesc_sw128(sk + kk * 32, 16, 1024);
          umma_f16(tmem + (i & 1) * 128, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[i & 1]);
        if (i >= 1 && !issue_pv(i - 1)) { ok = false; break; }
      }
      if (ok && n_tiles > 0) issue_pv(n_tiles - 1);
    }
  } else {
    // ------------------------------ softmax warps ------------------------------
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int t0 = qt * 128;
    const int qi = t0 + r;                         // absolute query position
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    float m_run = -1e30f, l_run = 0.f, alpha_prev = 1.f;
    float o_acc[64];
#pragma unroll
    for (int d = 0; d < 64; ++d) o_acc[d] = 0.f;

    auto consume_o = [&](int j) -> bool {
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&o_full[j & 1], (j >> 1) & 1u, abort_flag, p.status, 207) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) return false;
      tc_fence_after();
      float ot[32];
      const uint32_t ob = tmem + lane_off + 256 + (j & 1) * 64;
      tmem_ld32(ob, ot);
#pragma unroll
      for (int d = 0; d < 32; ++d) o_acc[d] = o_acc[d] * alpha_prev + ot[d];
      tmem_ld32(ob + 32, ot);
#pragma unroll
      for (int d = 0; d < 32; ++d) o_acc[32 + d] = o_acc[32 + d] * alpha_prev + ot[d];
      return true;
    };

    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int sb = i & 1;
      int w_ok = 1;
      if (lane == 0) w_ok = mbar_wait(&s_full[sb], (i >> 1) & 1u, abort_flag, p.status, 208) ? 1 : 0;
      w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
      if (!w_ok) { ok = false; break; }
      tc_fence_after();
      const int kt = kts.tile(i);
      const int j0 = kt * 128;
      const bool full = (j0 + 127 <= t0) &&
                        (p.is_global || j0 + 127 < p.n_meta || (t0 + 127) - j0 < p.window);
      const uint32_t sbase = tmem + lane_off + sb * 128;
      // pass 1: row max of the scaled, masked scores
      float mx = -1e30f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(sbase + c * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float sc = v[e] * p.scale_log2;
          if (!full) {
            const int j = j0 + c * 32 + e;
            const bool vis = (j <= qi) && (p.is_global || j < p.n_meta || qi - j < p.window);
            sc = vis ? sc : -1e30f;
          }
          mx = fmaxf(mx, sc);
        }
      }
      const float m_new = fmaxf(m_run, mx);
      const float alpha = exp2f(m_run - m_new);
      // pass 2: P = exp2(s - m_new) -> bf16 in 128B-swizzled smem, row sums
      float rs = 0.f;
      uint8_t* prow = smem + ATT_OFF_P + sb * ATT_P_BYTES + r * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(sbase + c * 32, v);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float s0 = v[e] * p.scale_log2, s1 = v[e + 1] * p.scale_log2;
          if (!full) {
            const int j = j0 + c * 32 + e;
            const bool v0 = (j <= qi) && (p.is_global || j < p.n_meta || qi - j < p.window);
            const bool v1 = (j + 1 <= qi) && (p.is_global || j + 1 < p.n_meta || qi - j - 1 < p.window);
            s0 = v0 ? s0 : -1e30f;
            s1 = v1 ? s1 : -1e30f;
          }
          const float p0 = exp2f(s0 - m_new), p1 = exp2f(s1 - m_new);
          rs += p0 + p1;
          pk[e >> 1] = pack_f16x2(p0, p1);
        }
        uint8_t* sub = prow + (c >> 1) * 16384;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = ((c & 1) * 4 + q) ^ (r & 7);
          *reinterpret_cast<uint4*>(sub + chunk * 16) =
              make_uint4(pk[q * 4 + 0], pk[q * 4 + 1], pk[q * 4 + 2], pk[q * 4 + 3]);
        }
      }
      l_run = l_run * alpha + rs;
      m_run = m_new;
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&p_full[sb]);
      if (i >= 1 && !consume_o(i - 1)) { ok = false; break; }
      alpha_prev = alpha;
    }
    if (ok && n_tiles > 0 && consume_o(n_tiles - 1) && qi < p.T) {
      const float inv = 1.f / l_run;
      float* dst = p.out + ((size_t)b * p.T + qi) * p.ld_out + h * 64;
#pragma unroll
      for (int d = 0; d < 64; d += 4)
        *reinterpret_cast<float4*>(dst + d) =
            make_float4(o_acc[d] * inv, o_acc[d + 1] * inv, o_acc[d + 2] * inv, o_acc[d + 3] * inv);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace hymba
