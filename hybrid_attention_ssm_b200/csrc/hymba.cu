// libhymba.so: the C ABI declared in include/hymba.h.  Host code validates arguments,
// carves the workspace, encodes TMA tensor maps and enqueues the sm_100a kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/hymba.h"
#include "attn.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "misc.cuh"
#include "ssm.cuh"

using namespace hymba;

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define HY_CUDA(call)                                                                     \
  do {                                                                                    \
    cudaError_t e_ = (call);                                                              \
    if (e_ != cudaSuccess) return fail(HYMBA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

#define HY_TRY(expr)            \
  do {                          \
    int rc_ = (expr);           \
    if (rc_ != HYMBA_OK) return rc_; \
  } while (0)

// Launches a kernel with programmatic stream serialisation: the grid may be launched while
// the previous kernel on the stream drains; every kernel starts with pdl_wait().
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
// threads of splitk_sum_rmsnorm_kernel for rows of d: one 16-byte piece each, whole warps
inline int snorm_threads(int d) { return ((d / 4 + 31) / 32) * 32; }
inline int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ----------------------------------------------------------------------------------------
// device properties and TMA descriptor encoding
// ----------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceInfo {
  int sms = 0;
  int major = 0;
  bool ok = false;
};
DeviceInfo g_dev[64];
std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;

int device_info(DeviceInfo** out) {
  int dev = 0;
  HY_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(HYMBA_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ok) {
    HY_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    HY_CUDA(cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev));
    d.ok = true;
  }
  if (d.major != 10) return fail(HYMBA_ERR_UNSUPPORTED, "needs an sm_100 device (found major %d)", d.major);
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    HY_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
    if (fn == nullptr || q != cudaDriverEntryPointSuccess)
      return fail(HYMBA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  *out = &d;
  return HYMBA_OK;
}

// A 2-D or 3-D tiled map with 128-byte swizzle; dims/strides innermost first, strides in
// bytes for dims 1.. ; box inner extent must be 128 bytes.
int make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int rank, const uint64_t* dims,
             const uint64_t* strides_bytes, const uint32_t* box,
             CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  if (!aligned16(base)) return fail(HYMBA_ERR_INVALID_ARG, "tensor base %p not 16-byte aligned", base);
  cuuint64_t d[3], s[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) {
    s[i] = strides_bytes[i];
    if (s[i] % 16 != 0) return fail(HYMBA_ERR_INVALID_ARG, "tensor stride %llu not a multiple of 16", (unsigned long long)s[i]);
  }
  CUresult r = g_encode(m, dt, rank, const_cast<void*>(base), d, s, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HYMBA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return HYMBA_OK;
}

// ----------------------------------------------------------------------------------------
// kernel-level profiling: a CUDA event pair around every launch while enabled
// ----------------------------------------------------------------------------------------
struct ProfState {
  bool on = false;
  int cap = 0, n = 0;
  cudaEvent_t* ev = nullptr;   // 2 * cap events
  char (*names)[24] = nullptr;
};
ProfState g_prof;

// ----------------------------------------------------------------------------------------
// A library-owned side stream per (host thread, device) for the attention branch of a
// decode step: it forks from the caller's stream after the decode prep kernel and joins
// before the branch norm through two events, so the attention runs beside x_proj and the
// SSM step.  Event fork/join is also how stream capture follows work onto another stream,
// so a captured decode step becomes a graph with two parallel branches.
// ----------------------------------------------------------------------------------------
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
int side_stream(SideStream** out) {
  thread_local SideStream per_dev[64];
  int dev = 0;
  HY_CUDA(cudaGetDevice(&dev));
  SideStream& ss = per_dev[dev & 63];
  if (ss.s == nullptr) {
    HY_CUDA(cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking));
    HY_CUDA(cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming));
    HY_CUDA(cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming));
  }
  *out = &ss;
  return HYMBA_OK;
}

// Between a fork and its join, an error return would leave work on the side stream outside
// the caller's stream (and a stream capture with an unjoined branch).  The guard joins the
// side stream back into the caller's stream when it goes out of scope still open.
struct ForkGuard {
  SideStream* side;
  cudaStream_t st;
  bool open = false;
  ForkGuard(SideStream* s, cudaStream_t stream) : side(s), st(stream) {}
  ForkGuard(const ForkGuard&) = delete;
  ForkGuard& operator=(const ForkGuard&) = delete;
  ~ForkGuard() {
    if (!open) return;
    cudaEventRecord(side->join, side->s);   // best effort: the call is already failing
    cudaStreamWaitEvent(st, side->join, 0);
  }
};

// Inside a stream capture the events become event-record nodes of the graph (the external
// flag), so every replay re-records them.
inline void prof_record(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  if (cs == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  else cudaEventRecord(ev, st);
}
inline void prof_begin(const char* name, cudaStream_t st) {
  if (!g_prof.on || g_prof.n >= g_prof.cap) return;
  strncpy(g_prof.names[g_prof.n], name, 23);
  g_prof.names[g_prof.n][23] = 0;
  prof_record(g_prof.ev[2 * g_prof.n], st);
}
inline void prof_end(cudaStream_t st) {
  if (!g_prof.on || g_prof.n >= g_prof.cap) return;
  prof_record(g_prof.ev[2 * g_prof.n + 1], st);
  ++g_prof.n;
}

// ----------------------------------------------------------------------------------------
// GEMM launcher
// ----------------------------------------------------------------------------------------
struct GemmCall {
  const char* name = "gemm";
  // A source 0 (optional): [rows0, K] row stride lda0 elements
  const void* a0 = nullptr;
  int rows0 = 0;
  long long lda0 = 0;
  // A source 1: [nb1, rows1, K], row stride lda1, batch stride a1_bstride (elements)
  const void* a1 = nullptr;
  int nb1 = 1, rows1 = 0;
  long long lda1 = 0, a1_bstride = 0;
  // B: [N, K] row stride ldb
  const void* b = nullptr;
  int N = 0;
  long long ldb = 0;
  int K = 0;
  int etype = ET_BF16;
  int mode = EPI_BF16;
  int bn = 256;
  int split_k = 1;
  // CTA pairs (cta_group::2, clusters of two): 256-row pair tiles, each CTA loading half of
  // the B tile.  Instantiated for the large prefill GEMMs only.
  bool pair = false;
  GemmParams p{};
};

template <int BN, int STAGES, int ET, int MODE, bool PAIR = false>
int launch_gemm_inst(const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& mb, const GemmParams& p,
                     int grid, cudaStream_t st, const char* name) {
  static bool attr_set[64] = {false};
  static int max_pairs[64] = {0};   // PAIR: clusters of two that fit on the device at once
  int dev = 0;
  cudaGetDevice(&dev);
  constexpr int smem = GemmSmem<BN, STAGES, gemm_epi_bytes(MODE), PAIR>::TOTAL;
  auto kern = gemm_tc_kernel<BN, STAGES, ET, MODE, PAIR>;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  if (!attr_set[dev & 63]) {
    HY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    if constexpr (PAIR) {
      // A persistent grid of pairs must be resident at once: a GPC with an odd number of free
      // SMs leaves one out, so ask the occupancy calculator rather than halving the SM count.
      cudaLaunchConfig_t q{};
      q.gridDim = dim3(2);
      q.blockDim = dim3(GEMM_THREADS);
      q.dynamicSmemBytes = smem;
      q.attrs = attr + 1;
      q.numAttrs = 1;
      int n = 0;
      HY_CUDA(cudaOccupancyMaxActiveClusters(&n, kern, &q));
      if (n < 1) return fail(HYMBA_ERR_UNSUPPORTED, "no SM pair can hold a %d-byte GEMM CTA", smem);
      max_pairs[dev & 63] = n;
    }
    attr_set[dev & 63] = true;
  }
  prof_begin(name, st);
  if constexpr (PAIR) {
    const int pairs = p.total_tiles < max_pairs[dev & 63] ? p.total_tiles : max_pairs[dev & 63];
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(GEMM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    HY_CUDA(cudaLaunchKernelEx(&cfg, kern, m0, m1, mb, p));
  } else {
    (void)attr;
    HY_CUDA(launch_pdl(kern, dim3(grid), dim3(GEMM_THREADS), smem, st, m0, m1, mb, p));
  }
  prof_end(st);
  return HYMBA_OK;
}

// Pair tiles are 256 x 256: a CTA's stage holds its 16 KB A tile and 128 rows of B, six
// stages.  (Measured on the Hymba layer shapes: 6 stages beat 7, and narrower pair tiles lose
// to the single-CTA tiles of the same width.)
template <int ET, int MODE>
int launch_gemm_bn_pair(int bn, const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& mb,
                        const GemmParams& p, cudaStream_t st, const char* name) {
  if (bn == 256) return launch_gemm_inst<256, 6, ET, MODE, true>(m0, m1, mb, p, 0, st, name);
  return fail(HYMBA_ERR_UNSUPPORTED, "no pair GEMM instance for tile width %d, type %d, epilogue %d", bn, ET, MODE);
}

// Tile widths instantiated per (epilogue, operand type); anything else is rejected.
template <int ET, int MODE>
int launch_gemm_bn(int bn, const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& mb, const GemmParams& p,
                   int grid, cudaStream_t st, const char* name) {
  constexpr bool any_bn = MODE == EPI_F32_PART || MODE == EPI_F32_T || MODE == EPI_F32_T_PART;
  if constexpr (ET == ET_TF32) {   // dt_proj: short K (dt_rank), 4 stages hold a whole tile's K
    if (bn == 256) return launch_gemm_inst<256, 4, ET, MODE>(m0, m1, mb, p, grid, st, name);
    return fail(HYMBA_ERR_UNSUPPORTED, "no tf32 GEMM instance for tile width %d", bn);
  } else {
    if (bn == 256) return launch_gemm_inst<256, 4, ET, MODE>(m0, m1, mb, p, grid, st, name);
    if constexpr (MODE != EPI_PROJ) {
      if (bn == 128) return launch_gemm_inst<128, 6, ET, MODE>(m0, m1, mb, p, grid, st, name);
    }
    if constexpr ((MODE == EPI_PROJ || MODE == EPI_SWIGLU) && ET == ET_BF16) {
      if (bn == 192) return launch_gemm_inst<192, 5, ET, MODE>(m0, m1, mb, p, grid, st, name);
    }
    if constexpr (MODE == EPI_BF16) {
      if (bn == 224) return launch_gemm_inst<224, 4, ET, MODE>(m0, m1, mb, p, grid, st, name);
    }
    if constexpr (any_bn && ET != ET_TF32) {
      if (bn == 160) return launch_gemm_inst<160, 5, ET, MODE>(m0, m1, mb, p, grid, st, name);
      if (bn == 64) return launch_gemm_inst<64, 8, ET, MODE>(m0, m1, mb, p, grid, st, name);
    }
    return fail(HYMBA_ERR_UNSUPPORTED, "no GEMM instance for tile width %d, type %d, epilogue %d", bn, ET, MODE);
  }
}

int launch_gemm_mode(const GemmCall& c, const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& mb,
                     const GemmParams& p, int grid, cudaStream_t st) {
  if (c.pair) {
    if (c.mode == EPI_PROJ && c.etype == ET_BF16) return launch_gemm_bn_pair<ET_BF16, EPI_PROJ>(c.bn, m0, m1, mb, p, st, c.name);
    if (c.mode == EPI_BF16 && c.etype == ET_F16) return launch_gemm_bn_pair<ET_F16, EPI_BF16>(c.bn, m0, m1, mb, p, st, c.name);
    if (c.mode == EPI_SWIGLU && c.etype == ET_BF16) return launch_gemm_bn_pair<ET_BF16, EPI_SWIGLU>(c.bn, m0, m1, mb, p, st, c.name);
    return fail(HYMBA_ERR_UNSUPPORTED, "no pair GEMM for epilogue %d with operand type %d", c.mode, c.etype);
  }
  switch (c.mode) {
    case EPI_PROJ:
      if (c.etype == ET_BF16) return launch_gemm_bn<ET_BF16, EPI_PROJ>(c.bn, m0, m1, mb, p, grid, st, c.name);
      break;
    case EPI_BF16:
      if (c.etype == ET_BF16) return launch_gemm_bn<ET_BF16, EPI_BF16>(c.bn, m0, m1, mb, p, grid, st, c.name);
      if (c.etype == ET_F16) return launch_gemm_bn<ET_F16, EPI_BF16>(c.bn, m0, m1, mb, p, grid, st, c.name);
      if (c.etype == ET_TF32) return launch_gemm_bn<ET_TF32, EPI_BF16>(c.bn, m0, m1, mb, p, grid, st, c.name);
      break;
    case EPI_SWIGLU:
      if (c.etype == ET_BF16) return launch_gemm_bn<ET_BF16, EPI_SWIGLU>(c.bn, m0, m1, mb, p, grid, st, c.name);
      break;
    case EPI_F32_T:
      if (c.etype == ET_BF16) return launch_gemm_bn<ET_BF16, EPI_F32_T>(c.bn, m0, m1, mb, p, grid, st, c.name);
      break;
    case EPI_F32_PART:
      if (c.etype == ET_BF16) return launch_gemm_bn<ET_BF16, EPI_F32_PART>(c.bn, m0, m1, mb, p, grid, st, c.name);
      break;
    case EPI_F32_T_PART:
      if (c.etype == ET_BF16) return launch_gemm_bn<ET_BF16, EPI_F32_T_PART>(c.bn, m0, m1, mb, p, grid, st, c.name);
      if (c.etype == ET_F16) return launch_gemm_bn<ET_F16, EPI_F32_T_PART>(c.bn, m0, m1, mb, p, grid, st, c.name);
      break;
    default:
      break;
  }
  return fail(HYMBA_ERR_UNSUPPORTED, "no GEMM instance for epilogue %d with operand type %d", c.mode, c.etype);
}

// Branch norm + average: persistent CTAs, rows streamed through a bulk-copy ring.
template <typename YT>
int launch_branch_norm(const float* O, int ld_o, int attn_w, const YT* y, int ld_y, const __nv_bfloat16* z, int ld_z,
                       int di, const float* g_attn, const float* g_ssm, float eps, __half* u, int ld_u, int rows,
                       DevStatus* status, int sms, cudaStream_t st) {
  if (rows <= 0) return HYMBA_OK;
  if (attn_w % 4 || di % 8 || attn_w > 4 * NORM_THREADS * NORM_MAXO || di > 8 * NORM_THREADS * NORM_MAXY)
    return fail(HYMBA_ERR_UNSUPPORTED, "branch norm widths %d/%d unsupported", attn_w, di);
  const bool rows_ok = aligned16(O) && aligned16(y) && (z == nullptr || aligned16(z)) && aligned16(u) &&
                       (ld_o * 4) % 16 == 0 && (ld_y * (int)sizeof(YT)) % 16 == 0 && (ld_z * 2) % 16 == 0 &&
                       (ld_u * 2) % 16 == 0 && (attn_w * 2) % 16 == 0;
  if (!rows_ok) return fail(HYMBA_ERR_INVALID_ARG, "branch norm rows must be 16-byte aligned");
  const int stage = (norm_stage_bytes(attn_w, di, (int)sizeof(YT), z != nullptr) + 127) & ~127;
  const int smem = NORM_STAGES * stage + 128;
  static bool attr_set[2][64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  bool& set = attr_set[sizeof(YT) == 4][dev & 63];
  if (!set) {
    HY_CUDA(cudaFuncSetAttribute(branch_norm_avg_kernel<YT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 NORM_STAGES * ((norm_stage_bytes(2048, 4096, 4, true) + 127) & ~127) + 128));
    set = true;
  }
  int per_sm = (200 * 1024) / smem;
  if (per_sm < 1) per_sm = 1;
  if (per_sm > 8) per_sm = 8;
  const int grid = rows < sms * per_sm ? rows : sms * per_sm;
  HY_CUDA(launch_pdl(branch_norm_avg_kernel<YT>, dim3(grid), dim3(NORM_THREADS), smem, st, O, ld_o, attn_w, y, ld_y,
                     z, ld_z, di, g_attn, g_ssm, eps, u, ld_u, rows, status));
  return HYMBA_OK;
}

template <int STAGES>
int launch_attention(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnParams& ap,
                     int B, int grid, cudaStream_t s) {
  static bool attr[64] = {false};
  int d = 0;
  cudaGetDevice(&d);
  auto kern = attn_fwd_kernel<STAGES>;
  constexpr int smem = AttnLayout<STAGES>::SMEM;
  if (!attr[d & 63]) {
    HY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    attr[d & 63] = true;
  }
  prof_begin("attention", s);
  HY_CUDA(launch_pdl(kern, dim3(grid), dim3(ATT_THREADS), smem, s, mq, mk, mv, ap, B));
  prof_end(s);
  return HYMBA_OK;
}

int run_gemm(GemmCall& c, const DeviceInfo& dev, cudaStream_t st) {
  const bool tf32 = c.etype == ET_TF32;
  const CUtensorMapDataType dt = tf32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                      : (c.etype == ET_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                           : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  const int esz = tf32 ? 4 : 2;
  const uint32_t kbox = tf32 ? 32 : 64;
  CUtensorMap m0, m1, mb;
  {
    const uint64_t dims[3] = {(uint64_t)c.K, (uint64_t)c.rows1, (uint64_t)c.nb1};
    const uint64_t str[2] = {(uint64_t)c.lda1 * esz, (uint64_t)c.a1_bstride * esz};
    const uint32_t box[3] = {kbox, (uint32_t)GEMM_BM, 1};
    HY_TRY(make_map(&m1, c.a1, dt, 3, dims, str, box));
  }
  if (c.a0 != nullptr && c.rows0 > 0) {
    const uint64_t dims[2] = {(uint64_t)c.K, (uint64_t)c.rows0};
    const uint64_t str[1] = {(uint64_t)c.lda0 * esz};
    const uint32_t box[2] = {kbox, (uint32_t)GEMM_BM};
    HY_TRY(make_map(&m0, c.a0, dt, 2, dims, str, box));
  } else {
    m0 = m1;
  }
  {
    const uint64_t dims[2] = {(uint64_t)c.K, (uint64_t)c.N};
    const uint64_t str[1] = {(uint64_t)c.ldb * esz};
    const uint32_t box[2] = {kbox, (uint32_t)(c.pair ? c.bn / 2 : c.bn)};   // a pair CTA loads half the B tile
    HY_TRY(make_map(&mb, c.b, dt, 2, dims, str, box));
  }
  GemmParams& p = c.p;
  p.tiles0 = (c.a0 != nullptr && c.rows0 > 0) ? cdiv(c.rows0, GEMM_BM) : 0;
  p.rows0 = c.rows0;
  p.nb1 = c.nb1;
  p.rows1 = c.rows1;
  p.tiles1 = cdiv(c.rows1, GEMM_BM);
  p.N = c.N;
  p.K = c.K;
  p.n_tiles_n = cdiv(c.N, c.bn);
  p.k_blocks = cdiv(c.K, kbox);
  p.split_k = c.split_k < 1 ? 1 : (c.split_k > p.k_blocks ? p.k_blocks : c.split_k);
  p.m_tiles = p.tiles0 + c.nb1 * p.tiles1;
  p.m_pairs = (p.m_tiles + 1) / 2;
  p.total_tiles = (c.pair ? p.m_pairs : p.m_tiles) * p.n_tiles_n * p.split_k;
  // column tiles inner once A no longer fits in a quarter of L2 beside the weights
  // (measured: in_proj at batch 4 x 8320 rows, 106 MB of A, 802 -> 718 us, out_proj 479 ->
  // 415 us; at 2176 rows, 7 MB of A, row tiles inner stay faster, 63 against 70 us)
  const double a_bytes = ((double)p.rows0 + (double)c.nb1 * c.rows1) * c.K * esz;
  p.n_inner = (p.n_tiles_n > 1 && a_bytes > 32.0 * (1 << 20)) ? 1 : 0;
  if (p.total_tiles <= 0) return HYMBA_OK;
  const int grid = p.total_tiles < dev.sms ? p.total_tiles : dev.sms;
  return launch_gemm_mode(c, m0, m1, mb, p, grid, st);
}

// smallest supported tile width covering n (for skinny N), else 256
int pick_bn_cover(int n) {
  if (n <= 64) return 64;
  if (n <= 128) return 128;
  if (n <= 160) return 160;
  return 256;
}
// Tile width among `cands` minimising (rounds of the persistent grid) x (operand bytes per
// k-block): the mainloops run at the rate shared memory is fed, so a round of tiles costs
// k_blocks times those bytes whether or not every SM has a tile.
int pick_bn_rounds(int m_tiles, int N, int sms, std::initializer_list<int> cands) {
  int best = *cands.begin();
  double best_cost = 1e300;
  for (int bn : cands) {
    const long long tiles = (long long)m_tiles * cdiv(N, bn);
    const long long rounds = (tiles + sms - 1) / sms;
    const double cost = (double)rounds * (GEMM_BM + bn);
    if (cost < best_cost * 0.999) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}
// Single-CTA tiles of width bn_single, or 256 x 256 pair tiles (cta_group::2)?  A round of
// pair tiles (sms / 2 pairs) took 0.9 of the time of a round of 128 x 256 tiles on the
// Hymba layer shapes (half the B tile per SM; the mainloop is bound by the operand feed from
// L2, not by the MMAs); a round of narrower single tiles costs in proportion to its operand
// bytes.  So pairs win at large M, and lose where they add a round (e.g. 17 row tiles x 34
// column tiles: 4 single rounds, 5 pair rounds).
bool pair_tiles_pay(int m_tiles, int N, int sms, int bn_single) {
  const long long rounds_s = cdiv((long long)m_tiles * cdiv(N, bn_single), sms);
  const long long rounds_p = cdiv((long long)cdiv(m_tiles, 2) * cdiv(N, 256), sms / 2);
  return 0.9 * (double)rounds_p < (double)rounds_s * (GEMM_BM + bn_single) / (GEMM_BM + 256);
}

void fill_rope_theta(double* theta, float base) {
  for (int j = 0; j < 32; ++j) theta[j] = std::pow((double)base, -2.0 * j / 64.0);
}

// ----------------------------------------------------------------------------------------
// validation and workspace layout
// ----------------------------------------------------------------------------------------
int check_cfg(const hymba_layer_cfg* c) {
  if (c == nullptr) return fail(HYMBA_ERR_INVALID_ARG, "cfg is NULL");
  if (c->head_dim != 64) return fail(HYMBA_ERR_UNSUPPORTED, "head_dim %d (only 64)", c->head_dim);
  if (c->d_state != 16) return fail(HYMBA_ERR_UNSUPPORTED, "d_state %d (only 16)", c->d_state);
  if (c->d_conv != 4) return fail(HYMBA_ERR_UNSUPPORTED, "d_conv %d (only 4)", c->d_conv);
  if (c->d_model < 8 || c->d_model % 8) return fail(HYMBA_ERR_UNSUPPORTED, "d_model %d (multiple of 8)", c->d_model);
  // the branch norm holds a row in registers: 8-element chunks of y, 4-element chunks of O
  if (c->d_inner < 64 || c->d_inner % 64 || c->d_inner > 8 * NORM_THREADS * NORM_MAXY)
    return fail(HYMBA_ERR_UNSUPPORTED, "d_inner %d (multiple of 64, at most %d)", c->d_inner,
                8 * NORM_THREADS * NORM_MAXY);
  if (c->n_q_heads * c->head_dim > 4 * NORM_THREADS * NORM_MAXO)
    return fail(HYMBA_ERR_UNSUPPORTED, "n_q_heads * head_dim above %d", 4 * NORM_THREADS * NORM_MAXO);
  if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_q_heads % c->n_kv_heads)
    return fail(HYMBA_ERR_UNSUPPORTED, "heads %d/%d", c->n_q_heads, c->n_kv_heads);
  if (c->n_q_heads / c->n_kv_heads > DEC_MAXG)
    return fail(HYMBA_ERR_UNSUPPORTED, "more than %d query heads per KV head", DEC_MAXG);
  if (c->dt_rank < 4 || c->dt_rank % 4 || c->dt_rank + 2 * c->d_state > 256)
    return fail(HYMBA_ERR_UNSUPPORTED, "dt_rank %d", c->dt_rank);
  if (c->window < 1 || c->n_meta < 0) return fail(HYMBA_ERR_INVALID_ARG, "window %d / n_meta %d", c->window, c->n_meta);
  if (c->kv_role < 0 || c->kv_role > 2) return fail(HYMBA_ERR_INVALID_ARG, "kv_role %d", c->kv_role);
  if (c->kv_role == HYMBA_KV_CONSUMER && c->is_global)
    return fail(HYMBA_ERR_INVALID_ARG, "a global layer cannot consume a shared SWA cache");
  if (!(c->rope_base > 1.f) || !(c->norm_eps >= 0.f)) return fail(HYMBA_ERR_INVALID_ARG, "rope_base/norm_eps");
  return HYMBA_OK;
}

struct Dims {
  int d, Hq, Hkv, D, Di, S, R, M, W;
  int qw, kvw, P, xz_off, uw, ld_xbc;
};
Dims dims_of(const hymba_layer_cfg* c) {
  Dims x;
  x.d = c->d_model; x.Hq = c->n_q_heads; x.Hkv = c->n_kv_heads; x.D = c->head_dim; x.Di = c->d_inner;
  x.S = c->d_state; x.R = c->dt_rank; x.M = c->n_meta; x.W = c->window;
  x.qw = x.Hq * x.D;
  x.kvw = x.Hkv * x.D;
  const bool kv = c->kv_role != HYMBA_KV_CONSUMER;
  x.P = x.qw + (kv ? 2 * x.kvw : 0) + 2 * x.Di;
  x.xz_off = x.qw + (kv ? 2 * x.kvw : 0);
  x.uw = x.qw + x.Di;
  x.ld_xbc = (x.R + 2 * x.S + 3) & ~3;
  return x;
}

// Split-K factors depend only on the shapes (never on the device), so workspace sizes and
// results are reproducible: enough splits to cover ~160 SMs, capped.
// split-K factor: as many splits as keep every tile's splits within one round of a B200's
// 148 SMs (fixed here so that workspace sizes do not depend on the device)
int splits_for(int tiles, int k_blocks, int cap) {
  int s = 148 / tiles;
  if (s > cap) s = cap;
  if (s > k_blocks) s = k_blocks;
  return s < 1 ? 1 : s;
}
// Split-K for the decode GEMMs (a few activation rows, the weights streamed as the M
// operand): the split that gives the busiest of 148 persistent CTAs the fewest k-blocks,
// ceil(tiles * s / 148) tiles of ceil(k_blocks / s) each; on a tie the smaller split (fewer
// slices to add).  E.g. 86 weight tiles of 25 k-blocks: s = 1 streams on 86 SMs only (25
// k-blocks each), s = 5 on all of them (3 tiles of 5).
int splits_balanced(int tiles, int k_blocks, int cap) {
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= cap && s <= k_blocks; ++s) {
    const long long cost = (long long)cdiv((long long)tiles * s, 148) * cdiv(k_blocks, s);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

struct PrefillWs {
  size_t q, xz, xc, xbc, xbc_part, dt_pre, carry, sumd, y, o, u, sstate, cstate, rope, total;
  int T, xproj_split, scan_L, scan_chunks;
};
// Time chunks of the selective scan.  Every chunk of a pass runs at once: the CTAs of the
// output pass, (Di / 64) x n_chunks x B, must fit in one wave of a B200's 148 SMs, else a
// second wave doubles the time of the serial walk over a chunk.  An SM holds SC_PER_SM scan
// CTAs (registers).  Within that, as many chunks as fit: shorter chunks, shorter walk.
// Fixed to 148 SMs so that workspace sizes do not depend on the device; the chunk length
// is a multiple of the scan's TMA stage.
// *cap is the most chunks any row count up to T gets (the chunk buffers are sized for it).
void scan_chunking(int B, int Di, int T, int* L, int* n_chunks, int* cap = nullptr) {
  const long long per_sm = SC_PER_SM;
  const long long groups = (long long)B * (Di / SC_CH);
  long long c = 148LL * per_sm / groups;
  const long long cmax = (T + SC_SUB - 1) / SC_SUB;
  if (c > cmax) c = cmax;
  if (c < 1) c = 1;
  const int len = SC_SUB * cdiv(cdiv(T, c), SC_SUB);
  *L = len;
  *n_chunks = cdiv(T, len);
  if (cap != nullptr) *cap = (int)c;
}
// scan_from: the first row the scan walks (M when the meta rows come from a precomputed
// prefix); the chunk buffers come last, so the other offsets do not depend on it.
PrefillWs prefill_layout(const Dims& m, int B, int n_tokens, int x_has_meta, int scan_from = 0) {
  PrefillWs w;
  w.T = x_has_meta ? n_tokens : m.M + n_tokens;
  int cap = 1;
  scan_chunking(B, m.Di, w.T, &w.scan_L, &w.scan_chunks, &cap);   // cap: for any rows <= T
  if (scan_from > 0) scan_chunking(B, m.Di, w.T - scan_from, &w.scan_L, &w.scan_chunks);
  const size_t rows = (size_t)B * w.T;
  size_t off = 256;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  w.q = take(rows * m.qw * 2);
  w.xz = take(rows * 2 * m.Di * 2);
  w.xc = take(rows * m.Di * 2);
  w.xbc = take(rows * m.ld_xbc * 4);
  w.xproj_split = splits_for(cdiv((long long)rows, GEMM_BM), cdiv(m.Di, 64), 16);
  w.xbc_part = take((size_t)w.xproj_split * rows * m.ld_xbc * 4);
  w.dt_pre = take(rows * m.Di * 2);
  w.y = take(rows * m.Di * 2);
  w.o = take(rows * m.qw * 4);
  w.u = take(rows * m.uw * 2);
  w.sstate = take((size_t)B * m.Di * 16 * 4);
  w.cstate = take((size_t)B * m.Di * 3 * 4);
  w.rope = take((size_t)w.T * 32 * 8);
  w.carry = take((size_t)B * (cap - 1) * m.Di * 16 * 4);
  w.sumd = take((size_t)B * (cap - 1) * m.Di * 4);
  w.total = off;
  return w;
}

// Device copies of a host prefill's input and output, after the prefill's own workspace.
struct HostStaging {
  size_t x, out, x_bytes, out_bytes, total;
};
HostStaging host_staging(const PrefillWs& L, const Dims& m, int B, int n_tokens) {
  HostStaging h;
  h.x_bytes = (size_t)B * n_tokens * m.d * 2;
  h.out_bytes = (size_t)B * L.T * m.d * 2;
  h.x = align256(L.total);
  h.out = align256(h.x + h.x_bytes);
  h.total = align256(h.out + h.out_bytes);
  return h;
}

struct DecodeWs {
  size_t proj, qrot, part, o, xc, xbc, xbc_part, y, u, acc_part, total;
  int n_splits, xproj_split, oproj_split, in_split;
};
// Key tiles of one (sequence, kv head) in decode: SWA reads the meta tiles and the ring,
// a global layer rows 0..p of its cache (p < n_keys_max).
int decode_key_tiles(const Dims& m, bool global, int n_keys_max) {
  return global ? cdiv(n_keys_max, DA_KT) : cdiv(m.M, DA_KT) + cdiv(m.W, DA_KT);
}
DecodeWs decode_layout(const Dims& m, int B, bool global, int n_keys_max) {
  DecodeWs w;
  w.n_splits = cdiv(decode_key_tiles(m, global, n_keys_max), DA_TPS);
  size_t off = 256;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  // in_proj split-K: enough weight tiles in flight for every SM of a B200 (148); the
  // consumers add the slices
  {
    const int bn0 = B <= 64 ? 64 : (B <= 128 ? 128 : 256);
    w.in_split = splits_balanced(cdiv(m.P, GEMM_BM) * cdiv(B, bn0), cdiv(m.d, 64), DEC_MAX_IN_SPLIT);
  }
  w.proj = take((size_t)w.in_split * B * m.P * 4);
  w.qrot = take((size_t)B * m.Hq * 64 * 4);
  w.part = take((size_t)B * m.Hq * w.n_splits * 66 * 4);
  w.o = take((size_t)B * m.qw * 4);
  w.xc = take((size_t)B * m.Di * 2);
  w.xbc = take((size_t)B * m.ld_xbc * 4);
  const int bn = B <= 64 ? 64 : (B <= 128 ? 128 : 256);
  const int n_tiles = cdiv(B, bn);
  w.xproj_split = splits_balanced(cdiv(m.R + 2 * m.S, GEMM_BM) * n_tiles, cdiv(m.Di, 64), DEC_MAX_XPROJ_SPLIT);
  w.xbc_part = take((size_t)w.xproj_split * B * m.ld_xbc * 4);
  w.y = take((size_t)B * m.Di * 4);
  w.u = take((size_t)B * m.uw * 2);
  w.oproj_split = splits_balanced(cdiv(m.d, GEMM_BM) * n_tiles, cdiv(m.uw, 64), 32);
  w.acc_part = take((size_t)w.oproj_split * B * m.d * 4);
  w.total = off;
  return w;
}

// Decode keys: SWA reads at most M + W keys; a global layer up to max_tokens.
int decode_max_keys(const hymba_layer_cfg* c, int max_tokens) {
  return c->is_global ? max_tokens : c->n_meta + c->window;
}

int check_weights(const hymba_layer_weights* w, const Dims& m, bool need_meta) {
  if (w == nullptr) return fail(HYMBA_ERR_INVALID_ARG, "weights is NULL");
  const void* ptrs[] = {w->w_in, w->conv_w, w->conv_b, w->w_x, w->w_dt, w->dt_bias, w->A, w->g_attn, w->g_ssm, w->w_out};
  for (const void* q : ptrs)
    if (q == nullptr || !aligned16(q)) return fail(HYMBA_ERR_INVALID_ARG, "weight pointer NULL or not 16-byte aligned");
  if (need_meta && m.M > 0 && (w->meta == nullptr || !aligned16(w->meta)))
    return fail(HYMBA_ERR_INVALID_ARG, "meta tokens pointer");
  if (w->w_dt_ld < m.R || w->w_dt_ld % 4) return fail(HYMBA_ERR_INVALID_ARG, "w_dt_ld %d", w->w_dt_ld);
  return HYMBA_OK;
}

}  // namespace

// ========================================================================================
// C ABI
// ========================================================================================
extern "C" {

int hymba_version(void) { return 10000; }

int hymba_profile_begin(int max_records) {
  if (max_records < 1) return fail(HYMBA_ERR_INVALID_ARG, "max_records < 1");
  if (g_prof.cap < max_records) {
    for (int i = 0; i < 2 * g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
    delete[] g_prof.ev;
    delete[] g_prof.names;
    g_prof.ev = new cudaEvent_t[2 * max_records];
    g_prof.names = new char[max_records][24];
    for (int i = 0; i < 2 * max_records; ++i) HY_CUDA(cudaEventCreate(&g_prof.ev[i]));
    g_prof.cap = max_records;
  }
  g_prof.n = 0;
  g_prof.on = true;
  return HYMBA_OK;
}

int hymba_profile_read(hymba_prof_record* out, int max_records, int* n_records) {
  if (out == nullptr || n_records == nullptr) return fail(HYMBA_ERR_INVALID_ARG, "NULL argument");
  g_prof.on = false;
  const int n = g_prof.n < max_records ? g_prof.n : max_records;
  for (int i = 0; i < n; ++i) {
    HY_CUDA(cudaEventSynchronize(g_prof.ev[2 * i + 1]));
    float ms = 0.f;
    HY_CUDA(cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]));
    memcpy(out[i].name, g_prof.names[i], 24);
    out[i].ms = ms;
  }
  *n_records = n;
  return HYMBA_OK;
}

int hymba_profile_end(hymba_prof_record* out, int max_records, int* n_records) {
  if (out == nullptr || n_records == nullptr) return fail(HYMBA_ERR_INVALID_ARG, "NULL argument");
  g_prof.on = false;
  const int n = g_prof.n < max_records ? g_prof.n : max_records;
  for (int i = 0; i < n; ++i) {
    HY_CUDA(cudaEventSynchronize(g_prof.ev[2 * i + 1]));
    float ms = 0.f;
    HY_CUDA(cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]));
    memcpy(out[i].name, g_prof.names[i], 24);
    out[i].ms = ms;
  }
  *n_records = n;
  g_prof.n = 0;
  return HYMBA_OK;
}

const char* hymba_last_error(void) { return g_err.c_str(); }

int hymba_set_wait_limit_ns(unsigned long long ns) {
  HY_CUDA(cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns)));
  return HYMBA_OK;
}

int hymba_mixer_workspace_size(const hymba_layer_cfg* cfg, int batch, int n_tokens, int x_has_meta, int mode,
                               size_t* bytes) {
  HY_TRY(check_cfg(cfg));
  if (bytes == nullptr || batch < 1) return fail(HYMBA_ERR_INVALID_ARG, "bytes NULL or batch < 1");
  const Dims m = dims_of(cfg);
  if (mode == HYMBA_MODE_PREFILL || mode == HYMBA_MODE_PREFILL_HOST) {
    if (n_tokens < 1) return fail(HYMBA_ERR_INVALID_ARG, "n_tokens < 1");
    const PrefillWs L = prefill_layout(m, batch, n_tokens, x_has_meta);
    *bytes = mode == HYMBA_MODE_PREFILL ? L.total : host_staging(L, m, batch, n_tokens).total;
  } else if (mode == HYMBA_MODE_DECODE) {
    // for a global layer n_tokens is the cache's max_tokens (keys read per step)
    const int mk = cfg->is_global ? (n_tokens > 0 ? n_tokens : 1) : decode_max_keys(cfg, 0);
    *bytes = decode_layout(m, batch, cfg->is_global != 0, mk).total;
  } else {
    return fail(HYMBA_ERR_INVALID_ARG, "mode %d", mode);
  }
  return HYMBA_OK;
}

int hymba_mixer_stage_layout(const hymba_layer_cfg* cfg, int batch, int n_tokens, int x_has_meta,
                             hymba_stage_layout* out) {
  HY_TRY(check_cfg(cfg));
  if (out == nullptr || batch < 1 || n_tokens < 1) return fail(HYMBA_ERR_INVALID_ARG, "stage layout args");
  const Dims m = dims_of(cfg);
  const PrefillWs w = prefill_layout(m, batch, n_tokens, x_has_meta);
  out->q = w.q; out->xz = w.xz; out->xc = w.xc; out->xbc = w.xbc; out->dt_pre = w.dt_pre;
  out->y = w.y; out->o = w.o; out->u = w.u;
  out->ld_xbc = m.ld_xbc;
  out->scan_chunks = w.scan_chunks;
  out->scan_chunk_len = w.scan_L;
  return HYMBA_OK;
}

int hymba_decode_stage_layout(const hymba_layer_cfg* cfg, int batch, int max_tokens, hymba_decode_stages* out) {
  HY_TRY(check_cfg(cfg));
  if (out == nullptr || batch < 1) return fail(HYMBA_ERR_INVALID_ARG, "decode stage layout args");
  const Dims m = dims_of(cfg);
  const int mk = cfg->is_global ? (max_tokens > 0 ? max_tokens : 1) : decode_max_keys(cfg, 0);
  const DecodeWs w = decode_layout(m, batch, cfg->is_global != 0, mk);
  out->proj = w.proj; out->xc = w.xc; out->xbc_part = w.xbc_part; out->y = w.y;
  out->proj_slice_stride = (long long)batch * m.P;
  out->xbc_slice_stride = (long long)batch * m.ld_xbc;
  out->in_split = w.in_split;
  out->xproj_split = w.xproj_split;
  out->ld_proj = m.P;
  out->ld_xbc = m.ld_xbc;
  return HYMBA_OK;
}

int hymba_workspace_init(void* ws, size_t ws_bytes, hymba_stream stream) {
  if (ws == nullptr || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(HYMBA_ERR_INVALID_ARG, "workspace NULL, < 256 bytes or not 256-byte aligned");
  HY_CUDA(cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream));
  return HYMBA_OK;
}

int hymba_status_read(void* ws, hymba_stream stream, int* status) {
  if (ws == nullptr || status == nullptr) return fail(HYMBA_ERR_INVALID_ARG, "NULL argument");
  DevStatus h;
  HY_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  HY_CUDA(cudaMemcpy(&h, ws, sizeof(unsigned) * 2, cudaMemcpyDeviceToHost));
  HY_CUDA(cudaMemset(ws, 0, 256));
  *status = (h.flags & DEV_ERR_TIMEOUT)      ? HYMBA_ERR_TIMEOUT
            : (h.flags & DEV_ERR_FP16_RANGE) ? HYMBA_ERR_FP16_RANGE
            : (h.flags & DEV_ERR_BOUNDS)     ? HYMBA_ERR_INVALID_ARG
                                             : HYMBA_OK;
  if (h.flags != 0) fail(*status, "device status flags 0x%x at site %u", h.flags, h.site);
  return HYMBA_OK;
}

int hymba_kv_share_alloc(const hymba_layer_cfg* base, int n_layers, const uint8_t* is_global, int batch,
                         int max_tokens, void* dev_buf, size_t buf_bytes, size_t* bytes_needed,
                         int* layer_cache_id, int* layer_kv_role, hymba_kv_cache* caches, int max_caches,
                         int* n_caches) {
  if (base == nullptr || is_global == nullptr || layer_cache_id == nullptr || layer_kv_role == nullptr ||
      bytes_needed == nullptr || n_caches == nullptr)
    return fail(HYMBA_ERR_INVALID_ARG, "NULL argument");
  if (n_layers < 1 || batch < 1 || max_tokens < 1) return fail(HYMBA_ERR_INVALID_ARG, "sizes");
  if (base->head_dim < 1 || base->n_kv_heads < 1 || base->n_meta < 0 || base->window < 1)
    return fail(HYMBA_ERR_INVALID_ARG, "cache sizes in base cfg");
  // plan
  int nc = 0;
  int i = 0;
  bool any_swa = false;
  while (i < n_layers) {
    if (is_global[i]) {
      layer_cache_id[i] = nc++;
      layer_kv_role[i] = HYMBA_KV_OWN;
      i += 1;
    } else if (i + 1 < n_layers && !is_global[i + 1]) {
      layer_cache_id[i] = layer_cache_id[i + 1] = nc++;
      layer_kv_role[i] = HYMBA_KV_PRODUCER;
      layer_kv_role[i + 1] = HYMBA_KV_CONSUMER;
      any_swa = true;
      i += 2;
    } else {
      layer_cache_id[i] = nc++;
      layer_kv_role[i] = HYMBA_KV_OWN;
      any_swa = true;
      i += 1;
    }
  }
  *n_caches = nc;
  const size_t row = (size_t)base->n_kv_heads * base->head_dim * 2;       // bytes per position
  const size_t full = align256((size_t)batch * max_tokens * row);
  const size_t meta = align256((size_t)batch * (base->n_meta > 0 ? base->n_meta : 1) * row);
  const size_t ring = align256((size_t)batch * base->window * row);
  size_t need = any_swa ? 2 * full : 0;     // shared prefill view
  for (int l = 0; l < n_layers; ++l) {
    const bool first = (l == 0) || layer_cache_id[l] != layer_cache_id[l - 1];
    if (!first) continue;
    need += is_global[l] ? 2 * full : 2 * (meta + ring);
  }
  *bytes_needed = need;
  if (dev_buf == nullptr) return HYMBA_OK;
  if (caches == nullptr || max_caches < nc) return fail(HYMBA_ERR_INVALID_ARG, "caches array too small (%d)", nc);
  if (buf_bytes < need) return fail(HYMBA_ERR_WORKSPACE, "cache buffer %zu < %zu bytes", buf_bytes, need);
  if (reinterpret_cast<uintptr_t>(dev_buf) & 255u) return fail(HYMBA_ERR_INVALID_ARG, "cache buffer not 256-byte aligned");
  uint8_t* p = static_cast<uint8_t*>(dev_buf);
  hymba_f16 *view_k = nullptr, *view_v = nullptr;
  if (any_swa) {
    view_k = reinterpret_cast<hymba_f16*>(p); p += full;
    view_v = reinterpret_cast<hymba_f16*>(p); p += full;
  }
  for (int l = 0; l < n_layers; ++l) {
    const bool first = (l == 0) || layer_cache_id[l] != layer_cache_id[l - 1];
    if (!first) continue;
    hymba_kv_cache& c = caches[layer_cache_id[l]];
    memset(&c, 0, sizeof(c));
    c.batch = batch;
    c.n_kv_heads = base->n_kv_heads;
    c.head_dim = base->head_dim;
    c.n_meta = base->n_meta;
    c.window = base->window;
    c.max_tokens = max_tokens;
    if (is_global[l]) {
      c.kind = HYMBA_CACHE_GLOBAL;
      c.k = reinterpret_cast<hymba_f16*>(p); p += full;
      c.v = reinterpret_cast<hymba_f16*>(p); p += full;
    } else {
      c.kind = HYMBA_CACHE_SWA;
      c.meta_k = reinterpret_cast<hymba_f16*>(p); p += meta;
      c.meta_v = reinterpret_cast<hymba_f16*>(p); p += meta;
      c.ring_k = reinterpret_cast<hymba_f16*>(p); p += ring;
      c.ring_v = reinterpret_cast<hymba_f16*>(p); p += ring;
      c.k = view_k;
      c.v = view_v;
    }
  }
  return HYMBA_OK;
}

// The prefill.  prefix == NULL: every row, meta rows included.  Otherwise the meta rows come
// from `prefix` (x holds only the input rows, x_has_meta == 0): their K/V are copied into the
// cache, the conv and the scan start from the prefix states, and only rows M..T-1 are
// computed; out and residual then hold those rows only, [B, n_tokens, d].
static int prefill_impl(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x,
                        int x_has_meta, int B, int n_tokens, const hymba_meta_prefix* prefix, hymba_kv_cache* kv,
                        float* ssm_state_out, float* conv_state_out, const hymba_bf16* residual, hymba_bf16* out,
                        void* ws, size_t ws_bytes, hymba_stream stream) {
  HY_TRY(check_cfg(cfg));
  DeviceInfo* dev = nullptr;
  HY_TRY(device_info(&dev));
  const Dims m = dims_of(cfg);
  if (B < 1 || n_tokens < 1) return fail(HYMBA_ERR_INVALID_ARG, "batch %d / n_tokens %d", B, n_tokens);
  HY_TRY(check_weights(w, m, !x_has_meta && prefix == nullptr));
  if (x == nullptr || out == nullptr || kv == nullptr || !aligned16(x) || !aligned16(out))
    return fail(HYMBA_ERR_INVALID_ARG, "x/out/kv pointer");
  if (residual != nullptr && !aligned16(residual)) return fail(HYMBA_ERR_INVALID_ARG, "residual alignment");
  const int P0 = prefix != nullptr ? m.M : 0;   // first row computed
  if (prefix != nullptr) {
    if (x_has_meta) return fail(HYMBA_ERR_INVALID_ARG, "a precomputed prefix needs x without the meta rows");
    if (prefix->ssm_state == nullptr || prefix->conv_state == nullptr || !aligned16(prefix->ssm_state) ||
        (m.M > 0 && (prefix->k == nullptr || prefix->v == nullptr || !aligned16(prefix->k) || !aligned16(prefix->v))))
      return fail(HYMBA_ERR_INVALID_ARG, "meta prefix pointers");
  }
  const PrefillWs L = prefill_layout(m, B, n_tokens, x_has_meta, P0);
  const int T = L.T;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return fail(HYMBA_ERR_INVALID_ARG, "workspace");
  if (ws_bytes < L.total) return fail(HYMBA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
  if (kv->k == nullptr || kv->v == nullptr || kv->max_tokens < T || kv->batch < B || kv->n_kv_heads != m.Hkv ||
      kv->head_dim != m.D)
    return fail(HYMBA_ERR_INVALID_ARG, "kv cache view (k/v, max_tokens >= %d, batch, heads)", T);
  const bool own_kv = cfg->kv_role != HYMBA_KV_CONSUMER;
  if (own_kv && !cfg->is_global && kv->kind == HYMBA_CACHE_SWA &&
      (kv->meta_k == nullptr && m.M > 0 || kv->ring_k == nullptr || kv->window != m.W || kv->n_meta != m.M))
    return fail(HYMBA_ERR_INVALID_ARG, "SWA cache meta/ring buffers");
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  DevStatus* status = reinterpret_cast<DevStatus*>(ws);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(wsb + off); };
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(wsb + off); };
  auto h16 = [&](size_t off) { return reinterpret_cast<__half*>(wsb + off); };
  const size_t rows = (size_t)B * T;
  const int Lmax = kv->max_tokens;

  // 0. RoPE angle table for the T positions
  {
    RopeThetas th;
    fill_rope_theta(th.t, cfg->rope_base);
    const int n = T * 32;
    prof_begin("rope_table", st);
    HY_CUDA(launch_pdl(rope_table_kernel, dim3(cdiv(n, 256)), dim3(256), 0, st, reinterpret_cast<float2*>(wsb + L.rope), T, th));
    prof_end(st);
    HY_CUDA(cudaGetLastError());
  }
  // the meta rows' K/V from the prefix: into the prefill view and, for an SWA cache, its meta rows
  if (prefix != nullptr && own_kv && m.M > 0) {
    const bool swa = !cfg->is_global && kv->kind == HYMBA_CACHE_SWA;
    const int row_vec = m.kvw / 8;   // 16-byte pieces per position
    const long long n = (long long)B * m.M * row_vec;
    prof_begin("prefix_kv", st);
    HY_CUDA(launch_pdl(prefix_kv_kernel, dim3(cdiv(n, 256)), dim3(256), 0, st,
                       reinterpret_cast<const __half*>(prefix->k), reinterpret_cast<const __half*>(prefix->v), B, m.M,
                       row_vec, reinterpret_cast<__half*>(kv->k), reinterpret_cast<__half*>(kv->v), Lmax,
                       swa ? reinterpret_cast<__half*>(kv->meta_k) : (__half*)nullptr,
                       swa ? reinterpret_cast<__half*>(kv->meta_v) : (__half*)nullptr));
    prof_end(st);
  }
  // 1. in_proj with RoPE on Q/K, scattering Q, K, V, x|z
  {
    GemmCall c;
    if (prefix != nullptr) {   // the input rows only, at positions M..T-1
      c.a1 = x; c.nb1 = B; c.rows1 = n_tokens; c.lda1 = m.d; c.a1_bstride = (long long)n_tokens * m.d;
      c.p.row_off1 = m.M;
    } else if (!x_has_meta && m.M > 0) {
      c.a0 = w->meta; c.rows0 = m.M; c.lda0 = m.d;
      c.a1 = x; c.nb1 = B; c.rows1 = n_tokens; c.lda1 = m.d; c.a1_bstride = (long long)n_tokens * m.d;
      c.p.row_off1 = m.M;
    } else {
      c.a1 = x; c.nb1 = B; c.rows1 = T; c.lda1 = m.d; c.a1_bstride = (long long)T * m.d;
      c.p.row_off1 = 0;
    }
    c.b = w->w_in; c.N = m.P; c.ldb = m.d; c.K = m.d;
    {
      const int m_tiles = (c.a0 != nullptr ? cdiv(c.rows0, GEMM_BM) : 0) + c.nb1 * cdiv(c.rows1, GEMM_BM);
      c.bn = pick_bn_rounds(m_tiles, m.P, dev->sms, {256, 192});
      c.pair = pair_tiles_pay(m_tiles, m.P, dev->sms, c.bn);
      if (c.pair) c.bn = 256;
    }
    c.name = "in_proj";
    c.mode = EPI_PROJ;
    c.p.out_batches = B;
    c.p.T_out = T;
    c.p.status = status;
    int ns = 0;
    c.p.seg[ns++] = Segment{0, m.qw, bf(L.q), (long long)T * m.qw, m.qw, 1, 1};
    if (own_kv) {
      Segment sk{m.qw, m.qw + m.kvw, kv->k, (long long)Lmax * m.kvw, m.kvw, 1, 1};
      Segment sv{m.qw + m.kvw, m.qw + 2 * m.kvw, kv->v, (long long)Lmax * m.kvw, m.kvw, 0, 1};
      if (!cfg->is_global && kv->kind == HYMBA_CACHE_SWA) {
        // the decode cache of an SWA layer: meta rows and the last W positions, written by
        // the epilogue next to the prefill view
        const int win0 = T - m.W > m.M ? T - m.W : m.M;
        sk.meta = kv->meta_k; sk.ring = kv->ring_k;
        sv.meta = kv->meta_v; sv.ring = kv->ring_v;
        sk.M = sv.M = m.M; sk.W = sv.W = m.W; sk.win0 = sv.win0 = win0;
      }
      c.p.seg[ns++] = sk;
      c.p.seg[ns++] = sv;
    }
    c.p.seg[ns++] = Segment{m.xz_off, m.xz_off + 2 * m.Di, bf(L.xz), (long long)T * 2 * m.Di, 2 * m.Di, 0, 0};
    c.p.nseg = ns;
    c.p.rope_tab = reinterpret_cast<const float2*>(wsb + L.rope);
    // x and W_in are inputs of the call: the mainloop may start while the RoPE table (read
    // only by the epilogue) is still being written.  A kernel before the table kernel has
    // completed by then: the table kernel waits for it before it lets this one launch.
    c.p.wait_late = 1;
    HY_TRY(run_gemm(c, *dev, st));
  }
  // 2. conv1d + SiLU (writes xc and the conv state)
  float* cstate = conv_state_out != nullptr ? conv_state_out : f32(L.cstate);
  {
    dim3 grid(m.Di / CONV_TC, cdiv(T - P0, CONV_TT), B);
    prof_begin("conv1d_silu", st);
    HY_CUDA(launch_pdl(conv1d_silu_kernel, grid, dim3(256), 0, st, bf(L.xz), 2 * m.Di, w->conv_w, w->conv_b, bf(L.xc),
                       cstate, T, m.Di, P0, prefix != nullptr ? prefix->conv_state : (const float*)nullptr));
    prof_end(st);
    HY_CUDA(cudaGetLastError());
  }
  // 3. x_proj (split-K into per-split slices, then a fixed-order sum): [dt_low | B | C]
  {
    GemmCall c;
    c.name = "x_proj";
    c.a1 = bf(L.xc); c.nb1 = 1; c.rows1 = (int)rows; c.lda1 = m.Di; c.a1_bstride = (long long)rows * m.Di;
    c.b = w->w_x; c.N = m.R + 2 * m.S; c.ldb = m.Di; c.K = m.Di;
    c.bn = pick_bn_cover(c.N);
    c.split_k = L.xproj_split;
    c.mode = EPI_F32_PART;
    c.p.out = f32(L.xbc_part);
    c.p.split_stride = (long long)rows * m.ld_xbc;
    c.p.ld_out = m.ld_xbc;
    c.p.n_valid = c.N;
    c.p.status = status;
    HY_TRY(run_gemm(c, *dev, st));
    const int n = (int)(rows * m.ld_xbc);
    prof_begin("splitk_reduce", st);
    HY_CUDA(launch_pdl(splitk_reduce_kernel, dim3(cdiv(n / 4, 256)), dim3(256), 0, st, f32(L.xbc_part),
                       L.xproj_split, (long long)n, n, nullptr, f32(L.xbc), 0));
    prof_end(st);
    HY_CUDA(cudaGetLastError());
  }
  // 4. dt_proj (tf32): dt_pre = dt_low W_dt^T [B*T, Di], stored bf16 (the scan adds dt_bias
  //    and applies the softplus in fp32 as it reads it).  The GEMM is bound by its stores
  //    (K = dt_rank is short), so the 16-bit rows halve its time and the scan's reads.
  {
    GemmCall c;
    c.etype = ET_TF32;
    c.a1 = f32(L.xbc); c.nb1 = B; c.rows1 = T; c.lda1 = m.ld_xbc; c.a1_bstride = (long long)T * m.ld_xbc;
    c.b = w->w_dt; c.N = m.Di; c.ldb = w->w_dt_ld; c.K = m.R;
    c.bn = 256;   // (measured: 128-wide tiles the same at 2176 rows, 124 against 97 us at 33280)
    c.name = "dt_proj";
    c.mode = EPI_BF16;
    c.p.out = bf(L.dt_pre);
    c.p.ld_out = m.Di;
    c.p.n_valid = m.Di;
    c.p.status = status;
    HY_TRY(run_gemm(c, *dev, st));
  }
  // 5. attention (block-skipped SWA + meta, or global causal), 3-stage ring, two CTAs per
  //    SM.  (Run beside the scan on a second stream instead, it gained nothing: the two
  //    compete for the same registers, and the scan then needed two waves.)
  {
    CUtensorMap mq, mk, mv;
    const uint32_t box[3] = {64, 128, 1};
    {
      const uint64_t dims[3] = {(uint64_t)m.qw, (uint64_t)T, (uint64_t)B};
      const uint64_t str[2] = {(uint64_t)m.qw * 2, (uint64_t)T * m.qw * 2};
      HY_TRY(make_map(&mq, bf(L.q), CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, dims, str, box));
    }
    {
      const uint64_t dims[3] = {(uint64_t)m.kvw, (uint64_t)T, (uint64_t)B};
      const uint64_t str[2] = {(uint64_t)m.kvw * 2, (uint64_t)Lmax * m.kvw * 2};
      HY_TRY(make_map(&mk, kv->k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, dims, str, box));
      HY_TRY(make_map(&mv, kv->v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, dims, str, box));
    }
    AttnParams ap;
    ap.T = T; ap.Hq = m.Hq; ap.Hkv = m.Hkv; ap.n_meta = m.M; ap.window = m.W; ap.is_global = cfg->is_global;
    ap.q_off = P0;
    ap.q_tiles = cdiv(T - P0, 128);
    ap.n_items = ap.q_tiles * m.Hq * B;
    ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)m.D));
    ap.out = f32(L.o);
    ap.ld_out = m.qw;
    ap.status = status;
    HY_TRY(launch_attention<3>(mq, mk, mv, ap, B, ap.n_items < 2 * dev->sms ? ap.n_items : 2 * dev->sms, st));
  }
  // 6. selective scan in time chunks: chunk end states, carry, outputs
  float* sstate = ssm_state_out != nullptr ? ssm_state_out : f32(L.sstate);
  {
    // row-major inputs through tensor maps of B*T rows (zero fill past the last row)
    CUtensorMap md, mx, mbc;
    {
      const uint64_t dims[2] = {(uint64_t)m.Di, (uint64_t)rows};
      const uint64_t str[1] = {(uint64_t)m.Di * 2};
      const uint32_t box[2] = {SC_CH, SC_SUB};
      HY_TRY(make_map(&md, bf(L.dt_pre), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE));
    }
    {
      const uint64_t dims[2] = {(uint64_t)m.Di, (uint64_t)rows};
      const uint64_t str[1] = {(uint64_t)m.Di * 2};
      const uint32_t box[2] = {SC_CH, SC_SUB};
      HY_TRY(make_map(&mx, bf(L.xc), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE));
    }
    {   // the B | C columns of the x_proj output (column offset dt_rank, a multiple of 4)
      const uint64_t dims[2] = {32, (uint64_t)rows};
      const uint64_t str[1] = {(uint64_t)m.ld_xbc * 4};
      const uint32_t box[2] = {32, SC_SUB};
      HY_TRY(make_map(&mbc, f32(L.xbc) + m.R, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, dims, str, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE));
    }
    ScanParams sp;
    sp.T = T; sp.Di = m.Di; sp.L = L.scan_L; sp.n_chunks = L.scan_chunks;
    sp.t_begin = P0;
    sp.h0 = prefix != nullptr ? prefix->ssm_state : nullptr;
    sp.A = w->A;
    sp.dt_bias = w->dt_bias;
    sp.carry = f32(L.carry);
    sp.sumd = f32(L.sumd);
    sp.y = bf(L.y);
    sp.state = sstate;
    sp.status = status;
    static bool attr_scan[64] = {false};
    int dcur = 0;
    cudaGetDevice(&dcur);
    if (!attr_scan[dcur & 63]) {
      HY_CUDA(cudaFuncSetAttribute(scan_chunk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SC_SMEM));
      HY_CUDA(cudaFuncSetAttribute(scan_chunk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SC_SMEM));
      attr_scan[dcur & 63] = true;
    }
    if (L.scan_chunks > 1) {
      prof_begin("scan_chunk_end", st);
      HY_CUDA(launch_pdl(scan_chunk_kernel<false>, dim3(m.Di / SC_CH, L.scan_chunks - 1, B), dim3(SC_THREADS), SC_SMEM,
                         st, md, mx, mbc, sp));
      prof_end(st);
      const long long n = (long long)B * m.Di * 16;
      prof_begin("scan_carry", st);
      HY_CUDA(launch_pdl(scan_carry_kernel, dim3(cdiv(n, 256)), dim3(256), 0, st, sp, B));
      prof_end(st);
    }
    prof_begin("selective_scan", st);
    HY_CUDA(launch_pdl(scan_chunk_kernel<true>, dim3(m.Di / SC_CH, L.scan_chunks, B), dim3(SC_THREADS), SC_SMEM, st,
                       md, mx, mbc, sp));
    prof_end(st);
  }
  // 7. per-branch RMSNorm, gate, beta, average
  {
    prof_begin("norm_avg", st);
    HY_TRY(launch_branch_norm<__nv_bfloat16>(f32(L.o), m.qw, m.qw, bf(L.y), m.Di, bf(L.xz) + m.Di, 2 * m.Di, m.Di,
                                             w->g_attn, w->g_ssm, cfg->norm_eps, h16(L.u), m.uw, (int)rows, status,
                                             dev->sms, st));
    prof_end(st);
    HY_CUDA(cudaGetLastError());
  }
  // 8. out_proj (+ residual); with a prefix, rows M..T-1 of each sequence into out [B, N, d]
  {
    GemmCall c;
    if (prefix != nullptr) {
      c.a1 = h16(L.u) + (size_t)P0 * m.uw; c.nb1 = B; c.rows1 = n_tokens; c.lda1 = m.uw;
      c.a1_bstride = (long long)T * m.uw;
    } else {
      c.a1 = h16(L.u); c.nb1 = 1; c.rows1 = (int)rows; c.lda1 = m.uw; c.a1_bstride = (long long)rows * m.uw;
    }
    c.b = w->w_out; c.N = m.d; c.ldb = m.uw; c.K = m.uw;
    c.etype = ET_F16;
    c.name = "out_proj";
    c.bn = pick_bn_rounds(c.nb1 * cdiv(c.rows1, GEMM_BM), m.d, dev->sms, {256, 224, 128});
    c.pair = pair_tiles_pay(c.nb1 * cdiv(c.rows1, GEMM_BM), m.d, dev->sms, c.bn);
    if (c.pair) c.bn = 256;
    c.mode = EPI_BF16;
    c.p.out = out;
    c.p.ld_out = m.d;
    c.p.n_valid = m.d;
    c.p.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
    c.p.ld_res = m.d;
    c.p.status = status;
    HY_TRY(run_gemm(c, *dev, st));
  }
  return HYMBA_OK;
}

int hymba_mixer_prefill(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x,
                        int x_has_meta, int B, int n_tokens, hymba_kv_cache* kv, float* ssm_state_out,
                        float* conv_state_out, const hymba_bf16* residual, hymba_bf16* out, void* ws,
                        size_t ws_bytes, hymba_stream stream) {
  return prefill_impl(cfg, w, x, x_has_meta, B, n_tokens, nullptr, kv, ssm_state_out, conv_state_out, residual, out,
                      ws, ws_bytes, stream);
}

int hymba_mixer_prefill_prefix(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x, int B,
                               int n_tokens, const hymba_meta_prefix* prefix, hymba_kv_cache* kv,
                               float* ssm_state_out, float* conv_state_out, const hymba_bf16* residual,
                               hymba_bf16* out, void* ws, size_t ws_bytes, hymba_stream stream) {
  if (prefix == nullptr) return fail(HYMBA_ERR_INVALID_ARG, "prefix is NULL");
  return prefill_impl(cfg, w, x, 0, B, n_tokens, prefix, kv, ssm_state_out, conv_state_out, residual, out, ws,
                      ws_bytes, stream);
}

int hymba_meta_prefix_size(const hymba_layer_cfg* cfg, size_t* bytes) {
  HY_TRY(check_cfg(cfg));
  if (bytes == nullptr) return fail(HYMBA_ERR_INVALID_ARG, "bytes is NULL");
  const Dims m = dims_of(cfg);
  const size_t kv = align256((size_t)(m.M > 0 ? m.M : 1) * m.kvw * 2);
  *bytes = 2 * kv + align256((size_t)m.Di * 16 * 4) + align256((size_t)m.Di * 3 * 4);
  return HYMBA_OK;
}

int hymba_meta_prefix_build(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* meta_rows,
                            void* buf, size_t buf_bytes, const hymba_meta_prefix* producer,
                            hymba_meta_prefix* prefix, hymba_bf16* meta_out, void* ws, size_t ws_bytes,
                            hymba_stream stream) {
  HY_TRY(check_cfg(cfg));
  const Dims m = dims_of(cfg);
  if (m.M < 1) return fail(HYMBA_ERR_INVALID_ARG, "n_meta is 0: there is no prefix");
  if (meta_rows == nullptr || buf == nullptr || prefix == nullptr || meta_out == nullptr ||
      (reinterpret_cast<uintptr_t>(buf) & 255u))
    return fail(HYMBA_ERR_INVALID_ARG, "meta_rows/buf/prefix/meta_out NULL or buf not 256-byte aligned");
  size_t need = 0;
  HY_TRY(hymba_meta_prefix_size(cfg, &need));
  if (buf_bytes < need) return fail(HYMBA_ERR_WORKSPACE, "prefix buffer %zu < %zu bytes", buf_bytes, need);
  const bool consumer = cfg->kv_role == HYMBA_KV_CONSUMER;
  if (consumer && (producer == nullptr || producer->k == nullptr || producer->v == nullptr))
    return fail(HYMBA_ERR_INVALID_ARG, "a consumer layer's prefix needs its producer's prefix K/V");
  uint8_t* p = static_cast<uint8_t*>(buf);
  const size_t kvb = align256((size_t)m.M * m.kvw * 2);
  prefix->k = reinterpret_cast<hymba_f16*>(p);
  prefix->v = reinterpret_cast<hymba_f16*>(p + kvb);
  prefix->ssm_state = reinterpret_cast<float*>(p + 2 * kvb);
  prefix->conv_state = reinterpret_cast<float*>(p + 2 * kvb + align256((size_t)m.Di * 16 * 4));
  // the M meta rows alone, as one sequence: their K/V go straight into the prefix (a
  // one-sequence cache of M positions; a consumer reads its producer's), the states after
  // them into the prefix, their outputs to meta_out
  hymba_kv_cache c;
  memset(&c, 0, sizeof(c));
  c.kind = HYMBA_CACHE_GLOBAL;
  c.batch = 1;
  c.n_kv_heads = m.Hkv;
  c.head_dim = m.D;
  c.n_meta = m.M;
  c.window = m.W;
  c.max_tokens = m.M;
  c.k = consumer ? const_cast<hymba_f16*>(producer->k) : prefix->k;
  c.v = consumer ? const_cast<hymba_f16*>(producer->v) : prefix->v;
  if (consumer) {
    prefix->k = producer->k;
    prefix->v = producer->v;
  }
  return prefill_impl(cfg, w, meta_rows, 1, 1, m.M, nullptr, &c, prefix->ssm_state, prefix->conv_state, nullptr,
                      meta_out, ws, ws_bytes, stream);
}

int hymba_mixer_prefill_host(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x_host,
                             int x_has_meta, int B, int n_tokens, hymba_kv_cache* kv, float* ssm_state_out,
                             float* conv_state_out, hymba_bf16* out_host, void* ws, size_t ws_bytes,
                             hymba_stream stream) {
  HY_TRY(check_cfg(cfg));
  if (x_host == nullptr || out_host == nullptr || B < 1 || n_tokens < 1)
    return fail(HYMBA_ERR_INVALID_ARG, "x_host/out_host NULL, batch or n_tokens < 1");
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return fail(HYMBA_ERR_INVALID_ARG, "workspace");
  const Dims m = dims_of(cfg);
  const PrefillWs L = prefill_layout(m, B, n_tokens, x_has_meta);
  const HostStaging h = host_staging(L, m, B, n_tokens);
  if (ws_bytes < h.total) return fail(HYMBA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, h.total);
  const cudaStream_t st = (cudaStream_t)stream;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  HY_CUDA(cudaMemcpyAsync(wsb + h.x, x_host, h.x_bytes, cudaMemcpyHostToDevice, st));
  HY_TRY(hymba_mixer_prefill(cfg, w, reinterpret_cast<const hymba_bf16*>(wsb + h.x), x_has_meta, B, n_tokens, kv,
                             ssm_state_out, conv_state_out, nullptr, reinterpret_cast<hymba_bf16*>(wsb + h.out), ws,
                             L.total, stream));
  HY_CUDA(cudaMemcpyAsync(out_host, wsb + h.out, h.out_bytes, cudaMemcpyDeviceToHost, st));
  return HYMBA_OK;
}

// The decode step; positions == NULL: every sequence at `position`; otherwise sequence b at
// positions[b] (device memory), each <= `position`, which sizes the attention's key splits.
// norm_out != NULL: the final split-K sum also writes norm_out = RMSNorm(out) * norm_gain.
static int decode_impl(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x, int B,
                       int position, const int* positions, hymba_kv_cache* kv, float* ssm_state,
                       float* conv_state, const hymba_bf16* residual, hymba_bf16* out, void* ws, size_t ws_bytes,
                       hymba_stream stream, const float* norm_gain = nullptr, float norm_eps = 0.f,
                       hymba_bf16* norm_out = nullptr) {
  HY_TRY(check_cfg(cfg));
  DeviceInfo* dev = nullptr;
  HY_TRY(device_info(&dev));
  const Dims m = dims_of(cfg);
  if (B < 1) return fail(HYMBA_ERR_INVALID_ARG, "batch %d", B);
  HY_TRY(check_weights(w, m, false));
  if (x == nullptr || out == nullptr || kv == nullptr || ssm_state == nullptr || conv_state == nullptr ||
      !aligned16(x) || !aligned16(out) || !aligned16(conv_state) || !aligned16(ssm_state))
    return fail(HYMBA_ERR_INVALID_ARG, "x/out/kv/state pointer");
  if (position < m.M) return fail(HYMBA_ERR_INVALID_ARG, "position %d < n_meta %d", position, m.M);
  if (kv->batch < B || kv->n_kv_heads != m.Hkv || kv->head_dim != m.D)
    return fail(HYMBA_ERR_INVALID_ARG, "kv cache shape");
  const bool global = cfg->is_global != 0;
  if (global) {
    if (kv->kind != HYMBA_CACHE_GLOBAL || kv->k == nullptr || position >= kv->max_tokens)
      return fail(HYMBA_ERR_INVALID_ARG, "global cache / position %d >= max_tokens", position);
  } else {
    if (kv->kind != HYMBA_CACHE_SWA || kv->ring_k == nullptr || (m.M > 0 && kv->meta_k == nullptr) ||
        kv->window != m.W || kv->n_meta != m.M)
      return fail(HYMBA_ERR_INVALID_ARG, "SWA cache");
  }
  const int max_keys = decode_max_keys(cfg, kv->max_tokens);
  const DecodeWs L = decode_layout(m, B, global, max_keys);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return fail(HYMBA_ERR_INVALID_ARG, "workspace");
  if (ws_bytes < L.total) return fail(HYMBA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  DevStatus* status = reinterpret_cast<DevStatus*>(ws);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(wsb + off); };
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(wsb + off); };
  auto h16 = [&](size_t off) { return reinterpret_cast<__half*>(wsb + off); };
  const bool own_kv = cfg->kv_role != HYMBA_KV_CONSUMER;

  // 1. in_proj, weights as the M operand (swap-AB), transposed store -> proj [B, P]
  {
    GemmCall c;
    c.a1 = w->w_in; c.nb1 = 1; c.rows1 = m.P; c.lda1 = m.d; c.a1_bstride = (long long)m.P * m.d;
    c.p.prefetch_a = 1;   // weights: their first stages load before the wait
    c.b = x; c.N = B; c.ldb = m.d; c.K = m.d;
    c.bn = pick_bn_cover(B);
    c.name = "decode_in_proj";
    c.mode = EPI_F32_T_PART;
    c.split_k = L.in_split;
    c.p.out = f32(L.proj);
    c.p.split_stride = (long long)B * m.P;
    c.p.ld_out = m.P;
    c.p.m_valid = m.P;
    c.p.n_valid = B;
    c.p.status = status;
    HY_TRY(run_gemm(c, *dev, st));
  }
  // 2. conv step, RoPE of q and the new k, the new k/v into the cache
  {
    DecPrepParams pp;
    pp.proj = f32(L.proj);
    pp.n_slices = L.in_split;
    pp.proj_stride = (long long)B * m.P;
    pp.ld_proj = m.P;
    pp.B = B;
    pp.Di = m.Di;
    pp.off_x = m.xz_off;
    pp.conv_blocks = cdiv(B * m.Di, 256);
    pp.conv_w = w->conv_w;
    pp.conv_b = w->conv_b;
    pp.conv_state = conv_state;
    pp.xc = bf(L.xc);
    pp.Hq = m.Hq; pp.Hkv = m.Hkv; pp.p = position; pp.write_kv = own_kv ? 1 : 0;
    pp.positions = positions;
    pp.max_position = position;
    pp.is_global = global ? 1 : 0; pp.M = m.M; pp.W = m.W; pp.Lmax = kv->max_tokens;
    pp.ring_k = reinterpret_cast<__half*>(kv->ring_k);
    pp.ring_v = reinterpret_cast<__half*>(kv->ring_v);
    pp.full_k = reinterpret_cast<__half*>(kv->k);
    pp.full_v = reinterpret_cast<__half*>(kv->v);
    pp.qrot = f32(L.qrot);
    pp.status = status;
    pp.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)m.D));
    fill_rope_theta(pp.rope_theta, cfg->rope_base);
    const int n_rope = B * (m.Hq + (own_kv ? m.Hkv : 0)) * 32;
    prof_begin("decode_prep", st);
    HY_CUDA(launch_pdl(decode_prep_kernel, dim3(pp.conv_blocks + cdiv(n_rope, 256)), dim3(256), 0, st, pp));
    prof_end(st);
  }
  // 3. attention over meta + window (or rows 0..p), split over key tiles, then combine.
  //    The two branches are independent from here to the norm: the attention runs on the
  //    side stream beside x_proj and the SSM step (both chains are latency-bound kernels
  //    that leave most of the GPU idle), joined before the norm.
  SideStream* side = nullptr;
  HY_TRY(side_stream(&side));
  ForkGuard fork_guard(side, st);
  int attn_items = 0;   // the attention's work items (its grid is min(items, 3 per SM))
  {
    const cudaStream_t ast = side->s;
    DecAttnParams ap;
    ap.qrot = f32(L.qrot);
    ap.Hq = m.Hq; ap.Hkv = m.Hkv; ap.M = m.M; ap.is_global = global ? 1 : 0;
    const int kvw = m.Hkv * m.D;
    CUtensorMap mmk, mmv, mk, mv;
    auto map_rows = [&](CUtensorMap* mp, const void* base, long long rows) {
      const uint64_t dims[2] = {(uint64_t)kvw, (uint64_t)rows};
      const uint64_t str[1] = {(uint64_t)kvw * 2};
      const uint32_t box[2] = {64, DA_KT};
      return make_map(mp, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, dims, str, box);
    };
    if (global) {
      ap.n_meta_tiles = 0;
      ap.n_main_valid = position + 1;
      ap.rows_main = kv->max_tokens;
      HY_TRY(map_rows(&mk, kv->k, (long long)B * kv->max_tokens));
      HY_TRY(map_rows(&mv, kv->v, (long long)B * kv->max_tokens));
      mmk = mk;
      mmv = mv;
    } else {
      ap.n_meta_tiles = cdiv(m.M, DA_KT);
      const int filled = position - m.M + 1;
      ap.n_main_valid = filled < m.W ? filled : m.W;
      ap.rows_main = m.W;
      HY_TRY(map_rows(&mk, kv->ring_k, (long long)B * m.W));
      HY_TRY(map_rows(&mv, kv->ring_v, (long long)B * m.W));
      if (m.M > 0) {
        HY_TRY(map_rows(&mmk, kv->meta_k, (long long)B * m.M));
        HY_TRY(map_rows(&mmv, kv->meta_v, (long long)B * m.M));
      } else {
        mmk = mk;
        mmv = mv;
      }
    }
    ap.positions = positions;
    ap.W = m.W;
    ap.max_position = position;
    ap.n_tiles = ap.n_meta_tiles + cdiv(ap.n_main_valid, DA_KT);
    ap.n_splits = cdiv(ap.n_tiles, DA_TPS);
    if (ap.n_splits > L.n_splits) return fail(HYMBA_ERR_WORKSPACE, "decode workspace sized for fewer keys");
    ap.n_items = B * m.Hkv * ap.n_splits;
    ap.part = f32(L.part);
    ap.status = status;
    static bool attr_da[64] = {false};
    int dcur = 0;
    cudaGetDevice(&dcur);
    if (!attr_da[dcur & 63]) {
      HY_CUDA(cudaFuncSetAttribute(decode_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DA_SMEM));
      attr_da[dcur & 63] = true;
    }
    // three CTAs per SM (four would fit).  (Measured: this order, with x_proj and the SSM
    // step queued behind the attention on the caller's stream, beat both x_proj first with
    // two attention CTAs per SM and a single stream.)
    attn_items = ap.n_items;
    const int grid = ap.n_items < 3 * dev->sms ? ap.n_items : 3 * dev->sms;
    HY_CUDA(cudaEventRecord(side->fork, st));   // every host-side check has passed
    HY_CUDA(cudaStreamWaitEvent(ast, side->fork, 0));
    fork_guard.open = true;
    prof_begin("decode_attn", ast);
    HY_CUDA(launch_pdl(decode_attn_kernel, dim3(grid), dim3(DA_THREADS), DA_SMEM, ast, mmk, mmv, mk, mv, ap));
    prof_end(ast);
    prof_begin("decode_attn_combine", ast);
    HY_CUDA(launch_pdl(decode_attn_combine_kernel, dim3(m.Hq, B), dim3(64), 0, ast, f32(L.part), ap.n_splits, m.Hq,
                       f32(L.o), m.qw));
    prof_end(ast);
    HY_CUDA(cudaEventRecord(side->join, ast));
  }
  // 4. x_proj (swap-AB, split-K into per-split slices, fixed-order sum)
  {
    GemmCall c;
    c.a1 = w->w_x; c.nb1 = 1; c.rows1 = m.R + 2 * m.S; c.lda1 = m.Di; c.a1_bstride = (long long)c.rows1 * m.Di;
    c.p.prefetch_a = 1;   // weights: their first stages load before the wait
    // when the attention grid leaves SM room (fewer items than its CTA slots), the SSM step's
    // CTAs may take it early: their launch latency is then on the step's critical path
    c.p.trigger_early = attn_items < 3 * dev->sms ? 1 : 0;
    c.b = bf(L.xc); c.N = B; c.ldb = m.Di; c.K = m.Di;
    c.bn = pick_bn_cover(B);
    c.name = "decode_x_proj";
    c.split_k = L.xproj_split;
    c.mode = EPI_F32_T_PART;
    c.p.out = f32(L.xbc_part);
    c.p.split_stride = (long long)B * m.ld_xbc;
    c.p.ld_out = m.ld_xbc;
    c.p.m_valid = c.rows1;
    c.p.n_valid = B;
    c.p.status = status;
    HY_TRY(run_gemm(c, *dev, st));   // the SSM step adds the slices (fixed order)
  }
  // 5. dt_proj + softplus + state update + C.h + gate
  {
    // four sequences per thread from 64 sequences on (each W_dt row read feeds four dot
    // products); below that one, so that a small batch still spreads over the SMs
    static size_t attr_ssm[64][2] = {};   // dynamic shared memory allowed so far
    int dcur = 0;
    HY_CUDA(cudaGetDevice(&dcur));
    const int wide = B >= 64 ? 1 : 0;
    auto kern = wide ? decode_ssm_kernel<4> : decode_ssm_kernel<1>;
    const int nb = wide ? 16 : 4;
    const size_t smem = dssm_smem_bytes(nb / 4, L.xproj_split, m.ld_xbc, m.R);
    if (smem > attr_ssm[dcur & 63][wide]) {
      HY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
      attr_ssm[dcur & 63][wide] = smem;
    }
    dim3 grid(m.Di / DSSM_NC, cdiv(B, nb));
    prof_begin("decode_ssm", st);
    HY_CUDA(launch_pdl(kern, grid, dim3(DSSM_THREADS), smem, st,
                       f32(L.xbc_part), (long long)B * m.ld_xbc, L.xproj_split, m.ld_xbc, m.R, w->w_dt, w->w_dt_ld,
                       w->dt_bias, w->A, bf(L.xc), f32(L.proj), m.P, (long long)B * m.P, L.in_split,
                       m.xz_off + m.Di, ssm_state, f32(L.y), m.Di, B, status));
    prof_end(st);
    HY_CUDA(cudaGetLastError());
  }
  // 6. norm + average (y already gated); the attention branch joins here
  HY_CUDA(cudaStreamWaitEvent(st, side->join, 0));
  fork_guard.open = false;
  {
    prof_begin("decode_norm_avg", st);
    HY_TRY(launch_branch_norm<float>(f32(L.o), m.qw, m.qw, f32(L.y), m.Di, nullptr, 0, m.Di, w->g_attn, w->g_ssm,
                                     cfg->norm_eps, h16(L.u), m.uw, B, status, dev->sms, st));
    prof_end(st);
    HY_CUDA(cudaGetLastError());
  }
  // 7. out_proj (swap-AB, split-K into per-split slices), then the fixed-order sum with the
  //    residual and the bf16 store
  {
    GemmCall c;
    c.a1 = w->w_out; c.nb1 = 1; c.rows1 = m.d; c.lda1 = m.uw; c.a1_bstride = (long long)m.d * m.uw;
    c.p.prefetch_a = 1;   // weights: their first stages load before the wait
    c.b = h16(L.u); c.N = B; c.ldb = m.uw; c.K = m.uw;
    c.etype = ET_F16;
    c.bn = pick_bn_cover(B);
    c.name = "decode_out_proj";
    c.split_k = L.oproj_split;
    c.mode = EPI_F32_T_PART;
    c.p.out = f32(L.acc_part);
    c.p.split_stride = (long long)B * m.d;
    c.p.ld_out = m.d;
    c.p.m_valid = m.d;
    c.p.n_valid = B;
    c.p.status = status;
    HY_TRY(run_gemm(c, *dev, st));
    const int n = B * m.d;
    prof_begin("decode_out_store", st);
    if (norm_out != nullptr) {
      HY_CUDA(launch_pdl(splitk_sum_rmsnorm_kernel, dim3(B), dim3(snorm_threads(m.d)), 0, st, (const float*)f32(L.acc_part),
                         L.oproj_split, (long long)n, m.d, reinterpret_cast<const __nv_bfloat16*>(residual),
                         reinterpret_cast<__nv_bfloat16*>(out), norm_gain, norm_eps,
                         reinterpret_cast<__nv_bfloat16*>(norm_out)));
    } else {
      HY_CUDA(launch_pdl(splitk_reduce_kernel, dim3(cdiv(n / 4, 256)), dim3(256), 0, st, f32(L.acc_part), L.oproj_split, (long long)n, n,
                                                              reinterpret_cast<const __nv_bfloat16*>(residual), out, 1));
    }
    prof_end(st);
    HY_CUDA(cudaGetLastError());
  }
  return HYMBA_OK;
}

int hymba_mixer_decode(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x, int B,
                       int position, hymba_kv_cache* kv, float* ssm_state, float* conv_state,
                       const hymba_bf16* residual, hymba_bf16* out, void* ws, size_t ws_bytes,
                       hymba_stream stream) {
  return decode_impl(cfg, w, x, B, position, nullptr, kv, ssm_state, conv_state, residual, out, ws, ws_bytes,
                     stream);
}

int hymba_mixer_decode_norm(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x, int B,
                            int position, hymba_kv_cache* kv, float* ssm_state, float* conv_state,
                            const hymba_bf16* residual, hymba_bf16* out, const float* norm_gain, float norm_eps,
                            hymba_bf16* norm_out, void* ws, size_t ws_bytes, hymba_stream stream) {
  if (norm_gain == nullptr || norm_out == nullptr || !aligned16(norm_gain) || !aligned16(norm_out) || norm_out == out ||
      norm_out == x)
    return fail(HYMBA_ERR_INVALID_ARG, "norm gain / output NULL, misaligned, or aliasing out or x");
  if (cfg != nullptr && cfg->d_model > SNORM_MAX_D)
    return fail(HYMBA_ERR_UNSUPPORTED, "d_model %d above %d for the fused norm", cfg->d_model, SNORM_MAX_D);
  return decode_impl(cfg, w, x, B, position, nullptr, kv, ssm_state, conv_state, residual, out, ws, ws_bytes, stream,
                     norm_gain, norm_eps, norm_out);
}

int hymba_mixer_decode_ragged(const hymba_layer_cfg* cfg, const hymba_layer_weights* w, const hymba_bf16* x, int B,
                              const int* positions, int max_position, hymba_kv_cache* kv, float* ssm_state,
                              float* conv_state, const hymba_bf16* residual, hymba_bf16* out, void* ws,
                              size_t ws_bytes, hymba_stream stream) {
  if (positions == nullptr || (reinterpret_cast<uintptr_t>(positions) & 3u))
    return fail(HYMBA_ERR_INVALID_ARG, "positions pointer NULL or not 4-byte aligned");
  return decode_impl(cfg, w, x, B, max_position, positions, kv, ssm_state, conv_state, residual, out, ws,
                     ws_bytes, stream);
}

int hymba_gemm_bf16(const hymba_bf16* A, const hymba_bf16* Bm, const hymba_bf16* residual, hymba_bf16* C, int M,
                    int N, int K, void* status_ws, hymba_stream stream) {
  DeviceInfo* dev = nullptr;
  HY_TRY(device_info(&dev));
  if (A == nullptr || Bm == nullptr || C == nullptr || M < 1 || N < 8 || K < 8 || N % 8 || K % 8 || !aligned16(C))
    return fail(HYMBA_ERR_INVALID_ARG, "gemm arguments");
  GemmCall c;
  c.a1 = A; c.nb1 = 1; c.rows1 = M; c.lda1 = K; c.a1_bstride = (long long)M * K;
  c.b = Bm; c.N = N; c.ldb = K; c.K = K;
  c.bn = pick_bn_rounds(cdiv(M, GEMM_BM), N, dev->sms, {256, 224, 128});
  c.mode = EPI_BF16;
  c.p.out = C;
  c.p.ld_out = N;
  c.p.n_valid = N;
  c.p.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
  c.p.ld_res = N;
  c.p.status = reinterpret_cast<DevStatus*>(status_ws);
  return run_gemm(c, *dev, (cudaStream_t)stream);
}

int hymba_rmsnorm(const hymba_bf16* x, const float* gain, int rows, int d, float eps, hymba_bf16* out,
                  hymba_stream stream) {
  if (x == nullptr || gain == nullptr || out == nullptr || rows < 1 || d < 8 || d % 8 || !aligned16(x) ||
      !aligned16(out))
    return fail(HYMBA_ERR_INVALID_ARG, "rmsnorm arguments");
  prof_begin("rmsnorm", (cudaStream_t)stream);
  if (d <= 32 * 8 * RMSW_MAXV && aligned16(gain)) {   // a warp per row
    HY_CUDA(launch_pdl(rmsnorm_warp_kernel, dim3(cdiv(rows, 8)), dim3(256), 0, (cudaStream_t)stream,
                       reinterpret_cast<const __nv_bfloat16*>(x), gain, rows, d, eps, reinterpret_cast<__nv_bfloat16*>(out)));
  } else {
    HY_CUDA(launch_pdl(rmsnorm_kernel, dim3(rows), dim3(256), 0, (cudaStream_t)stream, reinterpret_cast<const __nv_bfloat16*>(x), gain, d, eps,
                       reinterpret_cast<__nv_bfloat16*>(out)));
  }
  prof_end((cudaStream_t)stream);
  HY_CUDA(cudaGetLastError());
  return HYMBA_OK;
}

int hymba_ffn_swiglu(const hymba_bf16* h, const hymba_bf16* w_gate_up, const hymba_f16* w_down, int rows, int d,
                     int F, hymba_f16* act, const hymba_bf16* residual, hymba_bf16* out, void* status_ws,
                     hymba_stream stream) {
  DeviceInfo* dev = nullptr;
  HY_TRY(device_info(&dev));
  if (h == nullptr || w_gate_up == nullptr || w_down == nullptr || act == nullptr || out == nullptr || rows < 1 ||
      d < 8 || d % 8 || F < 64 || F % 64 || !aligned16(act) || !aligned16(out))
    return fail(HYMBA_ERR_INVALID_ARG, "ffn arguments");
  cudaStream_t st = (cudaStream_t)stream;
  {
    GemmCall c;
    c.a1 = h; c.nb1 = 1; c.rows1 = rows; c.lda1 = d; c.a1_bstride = (long long)rows * d;
    c.b = w_gate_up; c.N = 2 * F; c.ldb = d; c.K = d;
    c.bn = pick_bn_rounds(cdiv(rows, GEMM_BM), 2 * F, dev->sms, {256, 192, 128});
    c.pair = pair_tiles_pay(cdiv(rows, GEMM_BM), 2 * F, dev->sms, c.bn);
    if (c.pair) c.bn = 256;
    c.name = "ffn_gate_up";
    c.mode = EPI_SWIGLU;
    c.p.out = act;
    c.p.ld_out = F;
    c.p.n_valid = 2 * F;
    c.p.status = reinterpret_cast<DevStatus*>(status_ws);
    HY_TRY(run_gemm(c, *dev, st));
  }
  {
    GemmCall c;
    c.a1 = act; c.nb1 = 1; c.rows1 = rows; c.lda1 = F; c.a1_bstride = (long long)rows * F;
    c.b = w_down; c.N = d; c.ldb = F; c.K = F;
    c.etype = ET_F16;
    c.name = "ffn_down";
    c.bn = pick_bn_rounds(cdiv(rows, GEMM_BM), d, dev->sms, {256, 224, 128});
    c.pair = pair_tiles_pay(cdiv(rows, GEMM_BM), d, dev->sms, c.bn);
    if (c.pair) c.bn = 256;
    c.mode = EPI_BF16;
    c.p.out = out;
    c.p.ld_out = d;
    c.p.n_valid = d;
    c.p.residual = reinterpret_cast<const __nv_bfloat16*>(residual);
    c.p.ld_res = d;
    c.p.status = reinterpret_cast<DevStatus*>(status_ws);
    HY_TRY(run_gemm(c, *dev, st));
  }
  return HYMBA_OK;
}

// Decode-shaped FFN: the weights as the M operand (swap-AB) so that their rows, not the few
// token rows, spread the work over the SMs, split over K into fp32 slices summed in a fixed
// order.
namespace {
struct FfnDecWs {
  size_t part1, act, part2, total;
  int s1, s2;
};
FfnDecWs ffn_dec_layout(int rows, int d, int F) {
  FfnDecWs w;
  const int bn = rows <= 64 ? 64 : (rows <= 128 ? 128 : 256);
  const int nt = cdiv(rows, bn);
  w.s1 = splits_balanced(cdiv(2 * F, GEMM_BM) * nt, cdiv(d, 64), 8);
  w.s2 = splits_balanced(cdiv(d, GEMM_BM) * nt, cdiv(F, 64), 16);
  size_t off = 256;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  w.part1 = take((size_t)w.s1 * rows * 2 * F * 4);
  w.act = take((size_t)rows * F * 2);
  w.part2 = take((size_t)w.s2 * rows * d * 4);
  w.total = off;
  return w;
}
}  // namespace

int hymba_ffn_workspace_size(int rows, int d, int F, size_t* bytes) {
  if (bytes == nullptr || rows < 1 || rows > 256 || d < 8 || d % 8 || F < 64 || F % 64)
    return fail(HYMBA_ERR_INVALID_ARG, "ffn workspace arguments (rows 1..256, d a multiple of 8, F of 64)");
  *bytes = ffn_dec_layout(rows, d, F).total;
  return HYMBA_OK;
}

int hymba_l2_prefetch(const void* const* ranges, const size_t* bytes, int n_ranges, hymba_stream stream) {
  if (ranges == nullptr || bytes == nullptr || n_ranges < 1 || n_ranges > L2PF_MAX_RANGES)
    return fail(HYMBA_ERR_INVALID_ARG, "l2_prefetch: 1..8 ranges");
  L2Ranges r{};
  long long chunks = 0;
  for (int i = 0; i < n_ranges; ++i) {
    if (ranges[i] == nullptr || !aligned16(ranges[i])) return fail(HYMBA_ERR_INVALID_ARG, "l2_prefetch: range pointer");
    r.ptr[i] = static_cast<const char*>(ranges[i]);
    r.bytes[i] = bytes[i];
    chunks += (long long)((bytes[i] + L2PF_CHUNK - 1) / L2PF_CHUNK);
  }
  r.n = n_ranges;
  if (chunks == 0) return HYMBA_OK;
  const int grid = (int)std::min<long long>(cdiv(chunks, (long long)L2PF_THREADS), 148);
  prof_begin("l2_prefetch", (cudaStream_t)stream);
  l2_prefetch_kernel<<<grid, L2PF_THREADS, 0, (cudaStream_t)stream>>>(r);
  prof_end((cudaStream_t)stream);
  HY_CUDA(cudaGetLastError());
  return HYMBA_OK;
}

namespace {
// norm_out != NULL: the final split-K sum also writes norm_out = RMSNorm(out) * norm_gain.
int ffn_decode_impl(const hymba_bf16* h, const hymba_bf16* w_gate_up, const hymba_f16* w_down, int rows, int d, int F,
                    const hymba_bf16* residual, hymba_bf16* out, const float* norm_gain, float norm_eps,
                    hymba_bf16* norm_out, void* ws, size_t ws_bytes, hymba_stream stream) {
  DeviceInfo* dev = nullptr;
  HY_TRY(device_info(&dev));
  size_t need = 0;
  HY_TRY(hymba_ffn_workspace_size(rows, d, F, &need));
  if (h == nullptr || w_gate_up == nullptr || w_down == nullptr || out == nullptr || !aligned16(h) ||
      !aligned16(out) || (residual != nullptr && !aligned16(residual)))
    return fail(HYMBA_ERR_INVALID_ARG, "ffn decode pointers");
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return fail(HYMBA_ERR_INVALID_ARG, "workspace");
  if (ws_bytes < need) return fail(HYMBA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  const FfnDecWs L = ffn_dec_layout(rows, d, F);
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  DevStatus* status = reinterpret_cast<DevStatus*>(ws);
  float* part1 = reinterpret_cast<float*>(wsb + L.part1);
  float* part2 = reinterpret_cast<float*>(wsb + L.part2);
  __half* act = reinterpret_cast<__half*>(wsb + L.act);
  {  // [gate | up] slices, transposed: part1[s][r][2F]
    GemmCall c;
    c.a1 = w_gate_up; c.nb1 = 1; c.rows1 = 2 * F; c.lda1 = d; c.a1_bstride = (long long)2 * F * d;
    c.p.prefetch_a = 1;   // weights: their first stages load before the wait
    c.b = h; c.N = rows; c.ldb = d; c.K = d;
    c.bn = pick_bn_cover(rows);
    c.name = "ffn_dec_gate_up";
    c.split_k = L.s1;
    c.mode = EPI_F32_T_PART;
    c.p.out = part1;
    c.p.split_stride = (long long)rows * 2 * F;
    c.p.ld_out = 2 * F;
    c.p.m_valid = 2 * F;
    c.p.n_valid = rows;
    c.p.status = status;
    HY_TRY(run_gemm(c, *dev, st));
  }
  {
    const long long n = (long long)rows * F;
    prof_begin("ffn_dec_swiglu", st);
    HY_CUDA(launch_pdl(swiglu_slices_kernel, dim3(cdiv(n, 256)), dim3(256), 0, st, (const float*)part1, L.s1,
                       (long long)rows * 2 * F, rows, F, act, status));
    prof_end(st);
  }
  {  // down projection slices part2[s][r][d], then their sum with the residual
    GemmCall c;
    c.a1 = w_down; c.nb1 = 1; c.rows1 = d; c.lda1 = F; c.a1_bstride = (long long)d * F;
    c.p.prefetch_a = 1;   // weights: their first stages load before the wait
    c.b = act; c.N = rows; c.ldb = F; c.K = F;
    c.etype = ET_F16;
    c.bn = pick_bn_cover(rows);
    c.name = "ffn_dec_down";
    c.split_k = L.s2;
    c.mode = EPI_F32_T_PART;
    c.p.out = part2;
    c.p.split_stride = (long long)rows * d;
    c.p.ld_out = d;
    c.p.m_valid = d;
    c.p.n_valid = rows;
    c.p.status = status;
    HY_TRY(run_gemm(c, *dev, st));
    const int n = rows * d;
    prof_begin("ffn_dec_out", st);
    if (norm_out != nullptr) {
      HY_CUDA(launch_pdl(splitk_sum_rmsnorm_kernel, dim3(rows), dim3(snorm_threads(d)), 0, st, (const float*)part2, L.s2,
                         (long long)n, d, reinterpret_cast<const __nv_bfloat16*>(residual),
                         reinterpret_cast<__nv_bfloat16*>(out), norm_gain, norm_eps,
                         reinterpret_cast<__nv_bfloat16*>(norm_out)));
    } else {
      HY_CUDA(launch_pdl(splitk_reduce_kernel, dim3(cdiv(n / 4, 256)), dim3(256), 0, st, (const float*)part2, L.s2,
                         (long long)n, n, reinterpret_cast<const __nv_bfloat16*>(residual), out, 1));
    }
    prof_end(st);
  }
  return HYMBA_OK;
}
}  // namespace

int hymba_ffn_swiglu_decode(const hymba_bf16* h, const hymba_bf16* w_gate_up, const hymba_f16* w_down, int rows,
                            int d, int F, const hymba_bf16* residual, hymba_bf16* out, void* ws, size_t ws_bytes,
                            hymba_stream stream) {
  return ffn_decode_impl(h, w_gate_up, w_down, rows, d, F, residual, out, nullptr, 0.f, nullptr, ws, ws_bytes, stream);
}

int hymba_ffn_swiglu_decode_norm(const hymba_bf16* h, const hymba_bf16* w_gate_up, const hymba_f16* w_down, int rows,
                                 int d, int F, const hymba_bf16* residual, hymba_bf16* out, const float* norm_gain,
                                 float norm_eps, hymba_bf16* norm_out, void* ws, size_t ws_bytes, hymba_stream stream) {
  if (norm_gain == nullptr || norm_out == nullptr || !aligned16(norm_gain) || !aligned16(norm_out) || norm_out == out ||
      norm_out == h)
    return fail(HYMBA_ERR_INVALID_ARG, "norm gain / output NULL, misaligned, or aliasing out or h");
  if (d > SNORM_MAX_D) return fail(HYMBA_ERR_UNSUPPORTED, "d %d above %d for the fused norm", d, SNORM_MAX_D);
  return ffn_decode_impl(h, w_gate_up, w_down, rows, d, F, residual, out, norm_gain, norm_eps, norm_out, ws, ws_bytes,
                         stream);
}

int hymba_prepend_meta(const hymba_bf16* meta, const hymba_bf16* x, int batch, int n_meta, int n_tokens, int d,
                       hymba_bf16* out, hymba_stream stream) {
  if ((n_meta > 0 && meta == nullptr) || x == nullptr || out == nullptr || batch < 1 || n_meta < 0 ||
      n_tokens < 0 || d < 8 || d % 8 || (meta != nullptr && !aligned16(meta)) || !aligned16(x) || !aligned16(out))
    return fail(HYMBA_ERR_INVALID_ARG, "prepend_meta arguments");
  const long long total = (long long)batch * (n_meta + n_tokens) * (d / 8);
  if (total == 0) return HYMBA_OK;
  const int grid = (int)((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
  prof_begin("prepend_meta", (cudaStream_t)stream);
  HY_CUDA(launch_pdl(prepend_meta_kernel, dim3(grid), dim3(256), 0, (cudaStream_t)stream, reinterpret_cast<const __nv_bfloat16*>(meta),
                                                               reinterpret_cast<const __nv_bfloat16*>(x), batch,
                                                               n_meta, n_tokens, d,
                                                               reinterpret_cast<__nv_bfloat16*>(out)));
  prof_end((cudaStream_t)stream);
  HY_CUDA(cudaGetLastError());
  return HYMBA_OK;
}

int hymba_selftest_wait_timeout(void* ws, size_t ws_bytes, hymba_stream stream) {
  if (ws == nullptr || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(HYMBA_ERR_INVALID_ARG, "workspace");
  HY_CUDA(launch_pdl(wait_timeout_selftest_kernel, dim3(1), dim3(32), 0, (cudaStream_t)stream, reinterpret_cast<DevStatus*>(ws)));
  HY_CUDA(cudaGetLastError());
  return HYMBA_OK;
}

}  // extern "C"

// ========================================================================================
// Decode step without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run a decode step:
// serving loops that must not hit cudaMalloc's implicit device synchronisation between
// tokens, and plugins whose host runtime owns every device allocation and hands them only
// inputs and outputs.  For them the scratch memory of the
// decode step lives in this file-scope device array instead of a workspace argument.
// ========================================================================================
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;   // 32 MiB, held by every GPU that loads the library
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_noalloc_ptr[64] = {nullptr};
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device (host code only sees a host
// stand-in for the symbol, which must never be handed to a kernel).
int noalloc_scratch(void** out) {
  int dev = 0;
  HY_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(HYMBA_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(HYMBA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return HYMBA_OK;
}

}  // namespace

extern "C" int hymba_mixer_decode_noalloc(const hymba_layer_cfg* cfg, const hymba_layer_weights* w,
                                          const hymba_bf16* x, int batch, int position, hymba_kv_cache* kv,
                                          float* ssm_state, float* conv_state, const hymba_bf16* residual,
                                          hymba_bf16* out, hymba_stream stream) {
  if (kv == nullptr) return fail(HYMBA_ERR_INVALID_ARG, "kv cache is NULL");
  size_t need = 0;
  HY_TRY(hymba_mixer_workspace_size(cfg, batch, kv->max_tokens, 0, HYMBA_MODE_DECODE, &need));
  if (need > kNoAllocScratchBytes)
    return fail(HYMBA_ERR_WORKSPACE,
                "decode step needs %zu bytes of scratch, more than the %zu-byte built-in scratch; "
                "use hymba_mixer_decode with a workspace",
                need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  HY_TRY(noalloc_scratch(&scratch));
  // The array keeps the previous call's contents: the status word must start at zero (the
  // other buffers the step reads are either fully written first or cleared by the step).
  HY_CUDA(cudaMemsetAsync(scratch, 0, 256, (cudaStream_t)stream));
  return hymba_mixer_decode(cfg, w, x, batch, position, kv, ssm_state, conv_state, residual, out, scratch,
                            kNoAllocScratchBytes, stream);
}
