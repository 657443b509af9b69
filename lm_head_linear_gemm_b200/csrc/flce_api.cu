// C ABI of the fused LM-head linear + softcapped cross-entropy (include/flce.h):
// argument validation, workspace layout, tensor maps and the launch sequence.
//
// Launch sequence of one fused forward + backward (flce_forward with want_grads = 1):
//   prep_targets                                  targets -> effective ids, Nv, status
//   for each chunk of Nc rows:
//     logits GEMM   z = X_c W^T  (tcgen05 on SM pairs, fused softcap / sum-exp / target /
//                   gradient-operand epilogue)
//     row_finish    lse, per-row loss, r = 1/(Nv S), target patch of A', Xs = r . X_c
//     grad GEMMs    one balanced launch of both contractions:
//                     dX_c = r . (A' W)     (A' K-major, W MN-major)
//                     dW (+)= A'^T Xs       (both MN-major)
//   loss          deterministic mean over rows in the loss
// The logits of a chunk exist only as the bf16 operand A' [Nc, Vpad]; nothing of size N x Vpad
// is ever allocated.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/flce.h"
#include "gemm.cuh"
#include "rowwise.cuh"

using namespace flce;

namespace {

// Contraction tiles: pairs of SMs (cta_group::2), 256-row tiles, shared-memory rings of
// 32 KB stages.  Build-time tuning constants (measured defaults).
#ifndef FLCE_LOGITS_BN
#define FLCE_LOGITS_BN 256
#endif
#ifndef FLCE_LOGITS_STAGES
#define FLCE_LOGITS_STAGES 3
#endif
// k-blocks per ring slot of the logits kernels (slots of 64 KB)
#ifndef FLCE_LOGITS_KSUB
#define FLCE_LOGITS_KSUB 2
#endif
#ifndef FLCE_GRAD_STAGES
#define FLCE_GRAD_STAGES 6
#endif
#ifndef FLCE_EPI_WARPS
#define FLCE_EPI_WARPS 8
#endif
// L2 priorities of the operand streams (0 normal, 1 evict first, 2 evict last): the logits
// keep their X rows, which every W slab meets (last); the gradient launch keeps Xs, which
// every dW tile re-reads (last).  Marking W or A' evict-first measured slower.
#ifndef FLCE_L2_LOGITS_X
#define FLCE_L2_LOGITS_X 2
#endif
#ifndef FLCE_L2_LOGITS_W
#define FLCE_L2_LOGITS_W 0
#endif
#ifndef FLCE_L2_DX_A
#define FLCE_L2_DX_A 0
#endif
#ifndef FLCE_L2_DX_W
#define FLCE_L2_DX_W 0
#endif
#ifndef FLCE_L2_DW_A
#define FLCE_L2_DW_A 0
#endif
#ifndef FLCE_L2_DW_XS
#define FLCE_L2_DW_XS 2
#endif
// ring slots per MMA-issue round in the logits kernels
#ifndef FLCE_LOGITS_ROUND
#define FLCE_LOGITS_ROUND 1
#endif
// the gradient contractions run over each chunk's rows in the loss only (compacted)
#ifndef FLCE_COMPACT
#define FLCE_COMPACT 1
#endif
// padding of the gradient operand's rows (elements; a multiple of 16): the row stride of A'
#ifndef FLCE_A_PAD
#define FLCE_A_PAD 0
#endif
// dW tiles alternate their K direction from one wave to the next (the dX tiles keep theirs, so
// that a row's dX does not depend on the tile it lands in); measured within box-to-box noise,
// so off by default
#ifndef FLCE_SERPENTINE
#define FLCE_SERPENTINE 0
#endif
// dW tiles in groups of d-columns (all vocabulary tiles of one group before the next), so the
// dW tiles running at one time read only that group's columns of Xs
#ifndef FLCE_DW_GROUPS
#define FLCE_DW_GROUPS 1
#endif
// dX in wide tiles (256 x 512 per SM pair, two accumulators sharing each staged A' k-block)
#ifndef FLCE_DX_WIDE
#define FLCE_DX_WIDE 1
#endif
// gradient epilogues write (and, accumulating dW, read) whole 32-byte sectors when aligned
#ifndef FLCE_EPI_SECTOR32
#define FLCE_EPI_SECTOR32 1
#endif
using Cfg = PairCfg<256, FLCE_GRAD_STAGES, FLCE_EPI_WARPS>;
// epilogue warps of the logits kernels (the gradient kernels keep FLCE_EPI_WARPS)
#ifndef FLCE_LOGITS_EPI_WARPS
#define FLCE_LOGITS_EPI_WARPS FLCE_EPI_WARPS
#endif
using CfgL = PairCfg<FLCE_LOGITS_BN, FLCE_LOGITS_STAGES, FLCE_LOGITS_EPI_WARPS, 2, FLCE_LOGITS_KSUB>;
// logits: A = X (K-major), B = W (K-major)
constexpr auto kLogitsKernel =
    gemm_pair_kernel<CfgL, LogitsEpi, LogitsEpi, Major::K, Major::K, Major::K, Major::K, false,
                     FLCE_LOGITS_ROUND>;
// the same with the final RMSNorm's row sums in the epilogue (flce_forward_rmsnorm)
constexpr auto kLogitsFoldKernel =
    gemm_pair_kernel<CfgL, LogitsFoldEpi, LogitsFoldEpi, Major::K, Major::K, Major::K, Major::K,
                     false, FLCE_LOGITS_ROUND>;
// logits from e4m3 operands (kind::f8f6f4, tensorwise scales applied in the epilogue)
#ifndef FLCE_LOGITS8_STAGES
#define FLCE_LOGITS8_STAGES FLCE_LOGITS_STAGES
#endif
#ifndef FLCE_LOGITS8_KSUB
#define FLCE_LOGITS8_KSUB FLCE_LOGITS_KSUB
#endif
using Cfg8 = PairCfg<FLCE_LOGITS_BN, FLCE_LOGITS8_STAGES, FLCE_LOGITS_EPI_WARPS, 1,
                     FLCE_LOGITS8_KSUB>;
constexpr auto kLogitsKernel8 =
    gemm_pair_kernel<Cfg8, LogitsEpi, LogitsEpi, Major::K, Major::K, Major::K, Major::K, false,
                     FLCE_LOGITS_ROUND>;
static_assert(CfgL::BN == Cfg8::BN && CfgL::COL_SPLIT == Cfg8::COL_SPLIT,
              "both logits kernels fill the same per-row partial slots");
// gradients in one launch: dX = A' W (A' K-major, W MN-major), dW = A'^T Xs (both MN-major)
constexpr auto kGradKernel = gemm_pair_kernel<Cfg, DxEpi, DwEpi, Major::K, Major::MN, Major::MN,
                                             Major::MN, FLCE_DX_WIDE != 0>;
// gradients from 8-bit operands: dX = dz8 W8 (dz8 e5m2 K-major, W8 e4m3 MN-major) and
// dW = dz8^T Xs8 (dz8 e5m2 MN-major, Xs8 e4m3 MN-major), kind::f8f6f4
using CfgG8 = PairCfg<256, FLCE_GRAD_STAGES, FLCE_EPI_WARPS, 1, 1>;
constexpr auto kGradKernel8 =
    gemm_pair_kernel<CfgG8, DxEpi, DwEpi, Major::K, Major::MN, Major::MN, Major::MN,
                     FLCE_DX_WIDE != 0, 1, F8_A0 | F8_A1>;

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s bound on every in-kernel wait
constexpr float kFixedRefMaxCap = 32.f;           // exp(s - cap) >= e^{-64}: no underflow in fp32
constexpr int64_t kAutoChunkRows = 8192;   // rows per chunk when chunk_rows = 0
constexpr int kRmsRowsPerPart = 128;       // rows per dgamma partial of the RMSNorm backward
constexpr int kLogitsRows = 4096;          // rows per logits launch (launch_logits)
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Layout {
  int64_t chunk;      // rows per pass
  int64_t a_ld;       // row stride of A' (elements)
  int n_chunks;
  int n_slabs;        // per-row partial slots of the logits pass
  bool fixed_ref;
  bool compact;       // gradients over each chunk's rows in the loss only
  size_t hdr, tgt, s_t, der_t, e_t, row_loss, partial, r, A, Xs, pos, orig, cnt, bad, gsc, total;
  // final RMSNorm in front of the head (flce_forward_rmsnorm): the normalised rows and rstd;
  // with gradients either the folded backward's pieces (fixed reference) or a dX buffer and
  // dgamma partials for the separate backward kernels
  bool rms;
  size_t Xn, rstd, qpart, zt, cdot, dgpart, dXtmp, rmspart;
};

bool shape_ok(const flce_shape* s) {
  if (s == nullptr) return false;
  if (s->N < 0 || s->d <= 0 || s->Vpad <= 0 || s->Vreal <= 0 || s->Vreal > s->Vpad) return false;
  if (s->chunk_rows < 0) return false;
  if (!std::isfinite(s->cap)) return false;
  // 32-bit tile and row indices inside the kernels
  if (s->N > (int64_t(1) << 31) - 1 || s->d > (int64_t(1) << 24) || s->Vpad > (int64_t(1) << 28))
    return false;
  return true;
}

Layout make_layout(const flce_shape* s, int want_grads, int rms = 0) {
  Layout L{};
  const int64_t N = s->N;
  int64_t nc = s->chunk_rows > 0 ? s->chunk_rows : kAutoChunkRows;
  if (nc > N) nc = N;
  if (nc < 1) nc = 1;
  L.chunk = nc;
  L.a_ld = s->Vpad + FLCE_A_PAD;
  L.n_chunks = static_cast<int>(N > 0 ? (N + nc - 1) / nc : 1);
  L.fixed_ref = s->cap > 0.f && s->cap <= kFixedRefMaxCap;
  L.compact = want_grads && FLCE_COMPACT;
  const int64_t vtiles = (s->Vpad + CfgL::BN - 1) / CfgL::BN;
  L.n_slabs = static_cast<int>(vtiles * CfgL::COL_SPLIT);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  const size_t n = static_cast<size_t>(N > 0 ? N : 1);
  L.hdr = take(sizeof(DevHeader));
  L.tgt = take(n * sizeof(int));
  L.s_t = take(n * sizeof(float));
  L.der_t = take(n * sizeof(float));
  L.e_t = take(n * sizeof(float));
  L.row_loss = take(n * sizeof(float));
  L.partial = take(static_cast<size_t>(nc) * L.n_slabs * 2 * sizeof(float));
  if (want_grads) {
    L.r = take(static_cast<size_t>(nc) * sizeof(float));
    L.A = take(static_cast<size_t>(nc) * L.a_ld * sizeof(__nv_bfloat16));
    L.Xs = take(static_cast<size_t>(nc) * s->d * sizeof(__nv_bfloat16));
    if (L.compact) {
      L.pos = take(n * sizeof(int));
      L.orig = take(n * sizeof(int));
      L.cnt = take(static_cast<size_t>(L.n_chunks) * sizeof(int));
      L.bad = take(static_cast<size_t>(L.n_chunks) * sizeof(int));
      L.gsc = take(2 * sizeof(float));
    }
  }
  if (rms) {
    L.rms = true;
    L.Xn = take(n * static_cast<size_t>(s->d) * sizeof(__nv_bfloat16));
    L.rstd = take(n * sizeof(float));
    if (want_grads && L.fixed_ref) {
      L.qpart = take(static_cast<size_t>(nc) * L.n_slabs * sizeof(float));
      L.zt = take(n * sizeof(float));
      L.cdot = take(static_cast<size_t>(nc) * sizeof(float));
      // one row of partials per 32 rows of the chunk's 256-row tiles
      L.dgpart = take(static_cast<size_t>((nc + 255) / 256 * 8) * s->d * sizeof(float));
    } else if (want_grads) {
      L.dXtmp = take(n * static_cast<size_t>(s->d) * sizeof(__nv_bfloat16));
      L.rmspart = take(static_cast<size_t>((n + kRmsRowsPerPart - 1) / kRmsRowsPerPart) * s->d *
                       sizeof(float));
    }
  }
  L.total = off;
  return L;
}

// ------------------------------------------------------------------------------ device facts
struct DeviceInfo {
  bool checked = false;
  bool ok = false;
  int sms = 0;
  bool attrs_set = false;
};
std::mutex g_mu;
DeviceInfo g_dev[64];

int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FLCE_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.checked) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FLCE_ERR_CUDA;
    di.ok = (major == 10 && minor == 0);
    di.sms = sms;
    di.checked = true;
  }
  if (!di.ok) return FLCE_ERR_DEVICE;
  if (!di.attrs_set) {
    if (cudaFuncSetAttribute(kLogitsKernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             CfgL::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(kLogitsFoldKernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             CfgL::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(kGradKernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(kLogitsKernel8, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg8::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(kGradKernel8, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             CfgG8::SMEM_BYTES) != cudaSuccess)
      return FLCE_ERR_CUDA;
    di.attrs_set = true;
  }
  *out = &di;
  return FLCE_OK;
}

// ------------------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Matrix [outer][inner] of bf16 (elem_bytes 2) or e4m3 (elem_bytes 1, described as bytes),
// row-major with row stride `ld` elements, in 128-byte swizzled boxes of {128 bytes of inner
// elements, box_outer rows}.  Out-of-range box elements read as zero.
int make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
             uint32_t box_outer, int elem_bytes = 2) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return FLCE_ERR_CUDA;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {ld * static_cast<uint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem_bytes), box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FLCE_OK : FLCE_ERR_CUDA;
}

// ------------------------------------------------------------------------------ instrumentation
struct TimedLaunch {
  int kind;
  double flop;
  cudaEvent_t start, stop;
};
std::atomic<int> g_instr{0};
std::atomic<long long> g_launches{0};
std::mutex g_instr_mu;
std::vector<TimedLaunch> g_timed;      // recorded since the last reset
std::vector<cudaEvent_t> g_event_pool; // reusable events
double g_done_ms[3] = {0, 0, 0};
double g_done_flop[3] = {0, 0, 0};
long long g_done_n[3] = {0, 0, 0};

void count_launch() {
  if (g_instr.load(std::memory_order_relaxed)) g_launches.fetch_add(1, std::memory_order_relaxed);
}

cudaEvent_t pooled_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

template <class CF>
long long pair_tiles(const PairProblem& p) {
  if (p.M <= 0 || p.N <= 0) return 0;
  return static_cast<long long>((p.M + CF::BM - 1) / CF::BM) * ((p.N + CF::BN - 1) / CF::BN);
}

// Launch one persistent pair kernel over one or two problems; `kind` labels the launch for the
// instrumentation counters (0: logits, 1: dX + dW).
template <class E0, class E1, class CF = Cfg, class K>
int launch_pair(K kernel, const DeviceInfo* di, const CUtensorMap& a0, const CUtensorMap& b0,
                const CUtensorMap& a1, const CUtensorMap& b1, const PairProblem& p0,
                const PairProblem& p1, uint32_t* status, const typename E0::Params& e0,
                const typename E1::Params& e1, cudaStream_t st, int kind,
                const int* dyn = nullptr) {
  const long long tiles = pair_tiles<CF>(p0) + pair_tiles<CF>(p1);
  if (tiles <= 0) return FLCE_OK;
  const long long units = di->sms / 2;   // one CTA pair per SM pair, persistent
  const int grid = static_cast<int>(2 * (tiles < units ? tiles : units));
  PairArgs args{{p0, p1}, status, kWaitLimitNs, dyn};
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  const bool timed = g_instr.load(std::memory_order_relaxed) != 0;
  if (timed) {
    std::lock_guard<std::mutex> lock(g_instr_mu);
    ev0 = pooled_event();
    ev1 = pooled_event();
    if (ev0 != nullptr) cudaEventRecord(ev0, st);
  }
  kernel<<<grid, CF::THREADS, CF::SMEM_BYTES, st>>>(a0, b0, a1, b1, args, e0, e1);
  const bool ok = cudaGetLastError() == cudaSuccess;
  count_launch();
  if (timed && ev0 != nullptr && ev1 != nullptr) {
    cudaEventRecord(ev1, st);
    const double flop = 2.0 * p0.M * p0.N * static_cast<double>(p0.K) +
                        (p1.M > 0 ? 2.0 * p1.M * p1.N * static_cast<double>(p1.K) : 0.0);
    std::lock_guard<std::mutex> lock(g_instr_mu);
    g_timed.push_back(TimedLaunch{kind, flop, ev0, ev1});
  }
  return ok ? FLCE_OK : FLCE_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

#define FLCE_TRY(expr)             \
  do {                             \
    const int _rc = (expr);        \
    if (_rc != FLCE_OK) return _rc; \
  } while (0)

int launch_ok() {
  count_launch();
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

// Operands of the logits contraction when they are e4m3 (otherwise the bf16 X and W are used):
// x ~ X8 * (*scale_x), w ~ W8 * (*scale_w).
struct Fp8Logits {
  const uint8_t* X8 = nullptr;
  const uint8_t* W8 = nullptr;
  const float* scale_x = nullptr;
  const float* scale_w = nullptr;
};

// The final RMSNorm x = h rstd gamma in front of the head, and where its gradients go.
struct RmsFold {
  const __nv_bfloat16* H;
  const __nv_bfloat16* gamma;
  float eps;
  __nv_bfloat16* dH;
  float* dgamma;
  int accumulate;            // dgamma += (else =)
};

struct Ctx {
  const flce_shape* s;
  Fp8Logits fp8;
  const RmsFold* rms = nullptr;          // RMSNorm backward folded into the dX epilogue
  const long long* nv_total = nullptr;   // data-parallel normaliser (null: this call's rows)
  int dW_bf16 = 0;                       // dW element type: 0 fp32, 1 bf16
  int grad_fp8 = 0;                      // gradient contractions from e5m2 / e4m3 operands
  Layout L;
  uint8_t* ws;
  DevHeader* hdr;
  const DeviceInfo* di;
  cudaStream_t st;
  template <class T>
  T* at(size_t off) const {
    return reinterpret_cast<T*>(ws + off);
  }
};

// Logits contraction of rows [row0, row0 + rows) with the given epilogue parameters, from the
// bf16 X/W or, when the context carries them, from the e4m3 operands.
int launch_logits_rows(const Ctx& c, int64_t row0, int rows, const __nv_bfloat16* X,
                       const __nv_bfloat16* W, LogitsParams lp) {
  const flce_shape* s = c.s;
  const int d = static_cast<int>(s->d), Vpad = static_cast<int>(s->Vpad);
  const PairProblem logits{rows, Vpad, d, 1, 0, FLCE_L2_LOGITS_X, FLCE_L2_LOGITS_W};
  const PairProblem none{0, 0, 0, 0, 0, 0, 0};
  CUtensorMap mX, mW;
  if (c.fp8.X8 != nullptr) {
    FLCE_TRY(make_map(&mX, c.fp8.X8 + row0 * s->d, d, rows, d, Cfg8::BM_CTA, 1));
    FLCE_TRY(make_map(&mW, c.fp8.W8, d, Vpad, d, Cfg8::BN_CTA, 1));
    lp.scale_a = c.fp8.scale_x;
    lp.scale_b = c.fp8.scale_w;
    return launch_pair<LogitsEpi, LogitsEpi, Cfg8>(kLogitsKernel8, c.di, mX, mW, mX, mW, logits,
                                                    none, &c.hdr->status, lp, lp, c.st, 0);
  }
  FLCE_TRY(make_map(&mX, X + row0 * s->d, d, rows, d, CfgL::BM_CTA));
  FLCE_TRY(make_map(&mW, W, d, Vpad, d, CfgL::BN_CTA));
  lp.scale_a = lp.scale_b = nullptr;
  if (lp.q_partial != nullptr)
    return launch_pair<LogitsFoldEpi, LogitsFoldEpi, CfgL>(kLogitsFoldKernel, c.di, mX, mW, mX,
                                                          mW, logits, none, &c.hdr->status, lp,
                                                          lp, c.st, 0);
  return launch_pair<LogitsEpi, LogitsEpi, CfgL>(kLogitsKernel, c.di, mX, mW, mX, mW, logits,
                                                  none, &c.hdr->status, lp, lp, c.st, 0);
}

// The logits of rows [row0, row0 + rows) in launches of at most kLogitsRows rows: a launch walks
// the row blocks of one W slab before the next, so its X rows must stay in L2 next to the W
// slabs and the A' stream; past 4096 rows (25 MB of X at d = 3072) they start to fall out.
int launch_logits(const Ctx& c, int64_t row0, int rows, const __nv_bfloat16* X,
                  const __nv_bfloat16* W, const LogitsParams& lp) {
  const int per_row = lp.fixed_ref ? 1 : 2;   // partial words per (row, slab)
  for (int r0 = 0; r0 < rows; r0 += kLogitsRows) {
    const int rr = rows - r0 < kLogitsRows ? rows - r0 : kLogitsRows;
    LogitsParams q = lp;
    q.rows = rr;
    q.tgt = lp.tgt + r0;
    q.ref = lp.ref != nullptr ? lp.ref + r0 : nullptr;
    q.partial = lp.partial + static_cast<size_t>(r0) * lp.n_slabs * per_row;
    q.s_t = lp.s_t + r0;
    q.der_t = lp.der_t + r0;
    q.e_t = lp.e_t + r0;
    if (lp.q_partial != nullptr) {
      q.q_partial = lp.q_partial + static_cast<size_t>(r0) * lp.n_slabs;
      q.z_t = lp.z_t + r0;
    }
    // compacted rows index A from the chunk's first row: only pos moves with the launch
    q.pos = lp.pos != nullptr ? lp.pos + r0 : nullptr;
    q.A = lp.A != nullptr && lp.pos == nullptr ? lp.A + static_cast<size_t>(r0) * lp.a_ld : lp.A;
    FLCE_TRY(launch_logits_rows(c, row0 + r0, rr, X, W, q));
  }
  return FLCE_OK;
}

// One chunk of the gradient path: logits GEMM (mode FUSED or RECOMPUTE), row finish, and the
// dX / dW contractions in one launch.
// Vocabulary buckets of a chunk's dW (data-parallel exchange): after the launch that completes
// bucket b the library records events[b] (when not NULL) on the call's stream and writes the
// bucket's dW rows [bounds[b], bounds[b + 1]).
struct Buckets {
  int n;
  void* const* events;
  int64_t* bounds;
};

int grad_chunk(const Ctx& c, int64_t row0, int rows, const __nv_bfloat16* X,
               const __nv_bfloat16* W, const float* lse_in, float* lse_out, const float* grad_out,
               __nv_bfloat16* dX, void* dW, int accumulate, int mode,
               const Buckets* buckets = nullptr) {
  const flce_shape* s = c.s;
  const int d = static_cast<int>(s->d), Vpad = static_cast<int>(s->Vpad);
  const __nv_bfloat16* Xc = X + row0 * s->d;
  __nv_bfloat16* Abuf = c.at<__nv_bfloat16>(c.L.A);
  __nv_bfloat16* Xs = c.at<__nv_bfloat16>(c.L.Xs);
  float* r = c.at<float>(c.L.r);

  CUtensorMap mA_k, mW_mn, mA_mn, mXs_mn;
  uint8_t* Xs8 = reinterpret_cast<uint8_t*>(Xs);
  if (c.grad_fp8) {
    // e5m2 gradient rows in place of the bf16 rows of A (row stride 2 Vpad bytes), e4m3 W8 and
    // compacted X8 rows; boxes of 128 bytes x 128 rows
    FLCE_TRY(make_map(&mA_k, Abuf, Vpad, rows, 2 * static_cast<uint64_t>(c.L.a_ld),
                      CfgG8::BM_CTA, 1));
    FLCE_TRY(make_map(&mW_mn, c.fp8.W8, d, Vpad, d, CfgG8::BK, 1));
    FLCE_TRY(make_map(&mA_mn, Abuf, Vpad, rows, 2 * static_cast<uint64_t>(c.L.a_ld), CfgG8::BK,
                      1));
    FLCE_TRY(make_map(&mXs_mn, Xs8, d, rows, d, CfgG8::BK, 1));
  } else {
    FLCE_TRY(make_map(&mA_k, Abuf, Vpad, rows, c.L.a_ld, Cfg::BM_CTA));
    FLCE_TRY(make_map(&mW_mn, W, d, Vpad, d, 64));
    FLCE_TRY(make_map(&mA_mn, Abuf, Vpad, rows, c.L.a_ld, 64));
    FLCE_TRY(make_map(&mXs_mn, Xs, d, rows, d, 64));
  }

  LogitsParams lp{};
  lp.rows = rows;
  lp.Vreal = static_cast<int>(s->Vreal);
  lp.Vpad = Vpad;
  lp.a_ld = static_cast<int>(c.L.a_ld);
  lp.mode = mode;
  lp.fixed_ref = c.L.fixed_ref ? 1 : 0;
  lp.cap = s->cap;
  lp.k_u = s->cap > 0.f ? 2.0f / s->cap * 1.4426950408889634f : 0.f;
  lp.m2c_log2e = -2.0f * s->cap * 1.4426950408889634f;
  lp.tgt = c.at<int>(c.L.tgt) + row0;
  lp.ref = lse_in ? lse_in + row0 : nullptr;
  lp.partial = c.at<float>(c.L.partial);
  lp.n_slabs = c.L.n_slabs;
  lp.s_t = c.at<float>(c.L.s_t) + row0;
  lp.der_t = c.at<float>(c.L.der_t) + row0;
  lp.e_t = c.at<float>(c.L.e_t) + row0;
  lp.A = Abuf;
  const int chunk_index = static_cast<int>(row0 / c.L.chunk);
  const int* cnt = c.L.compact ? c.at<int>(c.L.cnt) + chunk_index : nullptr;
  lp.pos = c.L.compact ? c.at<int>(c.L.pos) + row0 : nullptr;
  const bool fold = c.rms != nullptr;
  if (fold) {
    lp.q_partial = c.at<float>(c.L.qpart);
    lp.z_t = c.at<float>(c.L.zt) + row0;
  }
  FLCE_TRY(launch_logits(c, row0, rows, X, W, lp));

  RowFinishParams rp{};
  rp.rows = rows;
  rp.d = d;
  rp.Vpad = Vpad;
  rp.a_ld = lp.a_ld;
  rp.n_slabs = c.L.n_slabs;
  rp.cap = s->cap;
  rp.fixed_ref = lp.fixed_ref;
  rp.from_partials = mode == LOGITS_FUSED ? 1 : 0;
  rp.want_grads = 1;
  rp.partial = lp.partial;
  rp.tgt = lp.tgt;
  rp.s_t = lp.s_t;
  rp.der_t = lp.der_t;
  rp.e_t = lp.e_t;
  rp.lse_in = lse_in ? lse_in + row0 : nullptr;
  rp.lse_out = lse_out ? lse_out + row0 : nullptr;
  rp.row_loss = c.at<float>(c.L.row_loss) + row0;
  rp.hdr = c.hdr;
  rp.nv_total = c.nv_total;
  rp.grad_out = grad_out;
  rp.r = r;
  rp.A = Abuf;
  rp.X = Xc;
  rp.Xs = Xs;
  __nv_bfloat16* dXc = dX + row0 * s->d;
  rp.pos = lp.pos;
  rp.cnt = cnt;
  rp.dX = dXc;
  rp.fp8 = c.grad_fp8;
  rp.X8 = c.grad_fp8 ? c.fp8.X8 + row0 * s->d : nullptr;
  rp.Xs8 = Xs8;
  rp.ktail = c.grad_fp8 ? CfgG8::KSLOT : Cfg::KSLOT;
  if (fold) {
    rp.q_partial = lp.q_partial;
    rp.z_t = lp.z_t;
    rp.cdot = c.at<float>(c.L.cdot);
  }
  const int finish_warps = rows + (c.L.compact ? rp.ktail : 0);
  row_finish_kernel<<<(finish_warps + 7) / 8, 256, 0, c.st>>>(rp);
  FLCE_TRY(launch_ok());

  // dX (long tiles: K = Vpad) and dW (short tiles: K = rows) share one balanced launch; with
  // compaction both run over the chunk's rows in the loss only (a device-side count: dX's M
  // and dW's K), dX rows scattered back to their places
  const int dx32 = FLCE_EPI_SECTOR32 && (d % 16) == 0 && aligned32(dXc);
  const float* gsc = c.grad_fp8 ? c.at<float>(c.L.gsc) : nullptr;
  DxParams xp{rows, d, dx32, r, dXc, c.L.compact ? c.at<int>(c.L.orig) + row0 : nullptr, cnt,
              gsc};
  if (fold) {
    xp.H = c.rms->H + row0 * s->d;
    xp.gamma = c.rms->gamma;
    xp.rstd = c.at<float>(c.L.rstd) + row0;
    xp.cdot = c.at<float>(c.L.cdot);
    xp.dg_part = c.at<float>(c.L.dgpart);
  }
  const int dyn_x = c.L.compact ? DYN_M : 0, dyn_w = c.L.compact ? DYN_K : 0;
  const PairProblem pdx{rows, d, Vpad, 0, FLCE_DX_WIDE, FLCE_L2_DX_A, FLCE_L2_DX_W, dyn_x};
  const PairProblem none{0, 0, 0, 0, 0, 0, 0, 0};
  const int nb = buckets != nullptr ? buckets->n : 1;
  const int vtiles = (Vpad + Cfg::BM - 1) / Cfg::BM;
  for (int b = 0; b < nb; ++b) {
    // Bucket b: the dW rows of vocabulary tiles [b vtiles / nb, (b + 1) vtiles / nb); the dX
    // tiles ride with the last bucket, so earlier buckets are final (and can be exchanged)
    // while dX still runs.  One bucket is the plain combined launch.
    const int v0 = static_cast<int>(static_cast<int64_t>(b) * vtiles / nb) * Cfg::BM;
    const int v1 = b + 1 == nb ? Vpad
                               : static_cast<int>(static_cast<int64_t>(b + 1) * vtiles / nb) * Cfg::BM;
    void* dWb = static_cast<uint8_t*>(dW) +
                static_cast<size_t>(v0) * s->d * (c.dW_bf16 ? 2 : 4);
    const int dw32 = FLCE_EPI_SECTOR32 && aligned32(dWb) && (!c.dW_bf16 || (d % 16) == 0);
    DwParams wp{v1 - v0, d, accumulate, dw32, c.dW_bf16, dWb, gsc != nullptr ? gsc + 1 : nullptr};
    const PairProblem pdw{v1 - v0, d, rows, 0, 0, FLCE_L2_DW_A, FLCE_L2_DW_XS, dyn_w,
                          FLCE_SERPENTINE, v0 / Cfg::BM, FLCE_DW_GROUPS};
    CUtensorMap mA_mn_b = mA_mn;
    if (v0 > 0) {
      if (c.grad_fp8)
        FLCE_TRY(make_map(&mA_mn_b, reinterpret_cast<uint8_t*>(Abuf) + v0, Vpad - v0, rows,
                          2 * static_cast<uint64_t>(c.L.a_ld), CfgG8::BK, 1));
      else
        FLCE_TRY(make_map(&mA_mn_b, Abuf + v0, Vpad - v0, rows, c.L.a_ld, 64));
    }
    if (v1 > v0 || b + 1 == nb) {
      if (c.grad_fp8)
        FLCE_TRY((launch_pair<DxEpi, DwEpi, CfgG8>(kGradKernel8, c.di, mA_k, mW_mn, mA_mn_b,
                                                   mXs_mn, b + 1 == nb ? pdx : none,
                                                   v1 > v0 ? pdw : none, &c.hdr->status, xp, wp,
                                                   c.st, 1, cnt)));
      else
        FLCE_TRY((launch_pair<DxEpi, DwEpi>(kGradKernel, c.di, mA_k, mW_mn, mA_mn_b, mXs_mn,
                                             b + 1 == nb ? pdx : none, v1 > v0 ? pdw : none,
                                             &c.hdr->status, xp, wp, c.st, 1, cnt)));
    }
    if (buckets != nullptr && buckets->events[b] != nullptr) {
      if (cudaEventRecord(static_cast<cudaEvent_t>(buckets->events[b]), c.st) != cudaSuccess)
        return FLCE_ERR_CUDA;
    }
    if (buckets != nullptr && buckets->bounds != nullptr) {
      buckets->bounds[b] = v0;
      buckets->bounds[b + 1] = v1;
    }
  }
  if (fold) {
    rmsnorm_dgamma_chunk_kernel<<<(d + 31) / 32, dim3(32, 8), 0, c.st>>>(
        xp.dg_part, d, rows, cnt, c.rms->dgamma, (row0 > 0 || c.rms->accumulate) ? 1 : 0);
    FLCE_TRY(launch_ok());
  }
  return FLCE_OK;
}

// Statistics-only pass over all rows: lse and per-row loss terms.
int stats_pass(const Ctx& c, const __nv_bfloat16* X, const __nv_bfloat16* W, float* lse) {
  const flce_shape* s = c.s;
  const int d = static_cast<int>(s->d), Vpad = static_cast<int>(s->Vpad);
  for (int64_t row0 = 0; row0 < s->N; row0 += c.L.chunk) {
    const int rows = static_cast<int>(s->N - row0 < c.L.chunk ? s->N - row0 : c.L.chunk);
    LogitsParams lp{};
    lp.rows = rows;
    lp.Vreal = static_cast<int>(s->Vreal);
    lp.Vpad = Vpad;
    lp.a_ld = Vpad;
    lp.mode = LOGITS_STATS;
    lp.fixed_ref = c.L.fixed_ref ? 1 : 0;
    lp.cap = s->cap;
    lp.k_u = s->cap > 0.f ? 2.0f / s->cap * 1.4426950408889634f : 0.f;
    lp.m2c_log2e = -2.0f * s->cap * 1.4426950408889634f;
    lp.tgt = c.at<int>(c.L.tgt) + row0;
    lp.partial = c.at<float>(c.L.partial);
    lp.n_slabs = c.L.n_slabs;
    lp.s_t = c.at<float>(c.L.s_t) + row0;
    lp.der_t = c.at<float>(c.L.der_t) + row0;
    lp.e_t = c.at<float>(c.L.e_t) + row0;
    FLCE_TRY(launch_logits(c, row0, rows, X, W, lp));
    RowFinishParams rp{};
    rp.rows = rows;
    rp.d = d;
    rp.Vpad = Vpad;
    rp.a_ld = Vpad;
    rp.n_slabs = c.L.n_slabs;
    rp.cap = s->cap;
    rp.fixed_ref = lp.fixed_ref;
    rp.from_partials = 1;
    rp.want_grads = 0;
    rp.partial = lp.partial;
    rp.tgt = lp.tgt;
    rp.s_t = lp.s_t;
    rp.der_t = lp.der_t;
    rp.e_t = lp.e_t;
    rp.lse_out = lse + row0;
    rp.row_loss = c.at<float>(c.L.row_loss) + row0;
    rp.hdr = c.hdr;
    row_finish_kernel<<<(rows + 7) / 8, 256, 0, c.st>>>(rp);
    FLCE_TRY(launch_ok());
  }
  return FLCE_OK;
}

__global__ void fill_zero_f32_kernel(float* p, long long n) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += stride)
    p[i] = 0.f;
}

int zero_dW(const Ctx& c, void* dW) {
  // fp32: Vpad * d words; bf16: half as many (d is even)
  const long long n = c.s->Vpad * c.s->d / (c.dW_bf16 ? 2 : 1);
  fill_zero_f32_kernel<<<4 * c.di->sms, 256, 0, c.st>>>(static_cast<float*>(dW), n);
  return launch_ok();
}

// The RMSNorm backward as row kernels, for a dX already formed: dH per row, dgamma in two
// deterministic stages (partials of kRmsRowsPerPart rows, then summed in order).
int rmsnorm_backward_kernels(const __nv_bfloat16* H, const __nv_bfloat16* gamma,
                             const float* rstd, const __nv_bfloat16* dX, int64_t N, int d,
                             __nv_bfloat16* dH, float* dgamma, int accumulate, float* partial,
                             cudaStream_t st) {
  int parts = 0;
  if (N > 0) {
    rmsnorm_bwd_rows_kernel<<<static_cast<unsigned>((N + 7) / 8), 256, 0, st>>>(H, gamma, rstd,
                                                                                dX, N, d, dH);
    FLCE_TRY(launch_ok());
    parts = static_cast<int>((N + kRmsRowsPerPart - 1) / kRmsRowsPerPart);
    rmsnorm_dgamma_partial_kernel<<<dim3((d / 2 + 255) / 256, parts), 256, 0, st>>>(
        H, rstd, dX, N, d, kRmsRowsPerPart, partial);
    FLCE_TRY(launch_ok());
  }
  rmsnorm_dgamma_final_kernel<<<(d + 255) / 256, 256, 0, st>>>(partial, parts, d, dgamma,
                                                                accumulate);
  return launch_ok();
}

// Targets -> effective ids, the count of rows in the loss and the status word; with compaction
// also each chunk's positions of its rows in the loss (prep_chunks_kernel).
int prep(const Ctx& c, const int64_t* targets) {
  const flce_shape* s = c.s;
  const auto* t = reinterpret_cast<const long long*>(targets);
  if (!c.L.compact) {
    prep_targets_kernel<<<1, 1024, 0, c.st>>>(t, s->N, s->Vreal, s->ignore_index,
                                              c.at<int>(c.L.tgt), c.hdr);
    return launch_ok();
  }
  prep_chunks_kernel<<<c.L.n_chunks, 1024, 0, c.st>>>(
      t, s->N, c.L.chunk, s->Vreal, s->ignore_index, c.at<int>(c.L.tgt), c.at<int>(c.L.pos),
      c.at<int>(c.L.orig), c.at<int>(c.L.cnt), c.at<int>(c.L.bad));
  FLCE_TRY(launch_ok());
  prep_total_kernel<<<1, 256, 0, c.st>>>(c.at<int>(c.L.cnt), c.at<int>(c.L.bad), c.L.n_chunks,
                                         c.hdr);
  return launch_ok();
}

int common_checks(const flce_shape* s, const void* X, const void* W, const int64_t* targets,
                  void* workspace, size_t ws_bytes, int want_grads) {
  if (!shape_ok(s)) return FLCE_ERR_ARG;
  if ((s->d % 8) != 0 || (s->Vpad % 8) != 0) return FLCE_ERR_ALIGN;
  // X and targets may be NULL only when there are no rows.
  if ((s->N > 0 && (X == nullptr || targets == nullptr)) || W == nullptr || workspace == nullptr)
    return FLCE_ERR_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(targets) ||
      (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return FLCE_ERR_ALIGN;
  if (ws_bytes < make_layout(s, want_grads).total) return FLCE_ERR_WORKSPACE;
  return FLCE_OK;
}

// ------------------------------------------------------------------------------ no-alloc scratch
// Scratch of flce_forward_noalloc.  In host code this name is only a stand-in for the device
// object: its device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FLCE_NOALLOC_SCRATCH_BYTES];
std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {};

int noalloc_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FLCE_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return FLCE_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return FLCE_OK;
}

// Forward (and, with want_grads, the gradients of the mean loss) from bf16 X/W, or from e4m3
// operands for the logits when fp8.X8 is set (X/W then only feed the gradient contractions).
int forward_impl(const flce_shape* s, const void* X, const void* W, const Fp8Logits& fp8,
                 const int64_t* targets, float* loss, float* lse, int want_grads,
                 const float* grad_scale, void* dX, void* dW, int dW_dtype, int accumulate_dW,
                 void* workspace, size_t workspace_bytes, void* stream,
                 const int64_t* nv_total = nullptr, const Buckets* buckets = nullptr,
                 int grad_fp8 = 0, const RmsFold* rms = nullptr) {
  want_grads = want_grads ? 1 : 0;
  if (loss == nullptr || (s->N > 0 && lse == nullptr)) return FLCE_ERR_ARG;
  if (!aligned4(loss) || !aligned4(lse)) return FLCE_ERR_ALIGN;
  if (want_grads) {
    if ((s->N > 0 && dX == nullptr) || dW == nullptr) return FLCE_ERR_ARG;
    if (dW_dtype != FLCE_DTYPE_F32 && dW_dtype != FLCE_DTYPE_BF16) return FLCE_ERR_ARG;
    if (!aligned16(dX) || !aligned16(dW)) return FLCE_ERR_ALIGN;
    if (grad_scale != nullptr && !aligned4(grad_scale)) return FLCE_ERR_ALIGN;
  }
  DeviceInfo* di = nullptr;
  FLCE_TRY(device_info(&di));
  Ctx c{};
  c.s = s;
  c.fp8 = fp8;
  c.nv_total = reinterpret_cast<const long long*>(nv_total);
  c.dW_bf16 = want_grads && dW_dtype == FLCE_DTYPE_BF16 ? 1 : 0;
  c.grad_fp8 = want_grads && grad_fp8 ? 1 : 0;
  c.L = make_layout(s, want_grads, rms != nullptr ? 1 : 0);
  // 8-bit gradients need the fixed exp reference and the compacted rows (rows not in the loss
  // must not enter the e5m2 operand)
  if (c.grad_fp8 && (!c.L.fixed_ref || !c.L.compact || fp8.X8 == nullptr)) return FLCE_ERR_ARG;
  c.ws = static_cast<uint8_t*>(workspace);
  c.di = di;
  c.st = static_cast<cudaStream_t>(stream);
  c.hdr = c.at<DevHeader>(c.L.hdr);
  const auto* Xb = static_cast<const __nv_bfloat16*>(X);
  const auto* Wb = static_cast<const __nv_bfloat16*>(W);
  // With the final RMSNorm in front, the head reads the normalised rows written here.  Its
  // backward is folded into the dX epilogue on the fixed-reference path (dX is then never
  // formed: the epilogue writes dH), else dX goes to a buffer and the RMSNorm backward kernels
  // follow the head.
  const bool fold = rms != nullptr && want_grads && c.L.fixed_ref;
  auto* dXout = static_cast<__nv_bfloat16*>(dX);
  if (rms != nullptr) {
    if (s->N > 0) {
      auto* Xn = c.at<__nv_bfloat16>(c.L.Xn);
      rmsnorm_fwd_kernel<<<static_cast<unsigned>((s->N + 7) / 8), 256, 0, c.st>>>(
          rms->H, rms->gamma, rms->eps, s->N, static_cast<int>(s->d), Xn,
          c.at<float>(c.L.rstd));
      FLCE_TRY(launch_ok());
      Xb = Xn;
    }
    if (fold) {
      c.rms = rms;
      dXout = rms->dH;
    } else if (want_grads) {
      dXout = c.at<__nv_bfloat16>(c.L.dXtmp);
    }
  }

  FLCE_TRY(prep(c, targets));
  if (c.grad_fp8) {
    fp8_grad_scales_kernel<<<1, 1, 0, c.st>>>(c.hdr, c.nv_total, grad_scale, fp8.scale_w,
                                              fp8.scale_x, c.at<float>(c.L.gsc));
    FLCE_TRY(launch_ok());
  }
  if (s->N == 0) {
    zero_loss_kernel<<<1, 1, 0, c.st>>>(loss);
    FLCE_TRY(launch_ok());
    if (want_grads && !accumulate_dW) FLCE_TRY(zero_dW(c, dW));
    if (want_grads && rms != nullptr && !rms->accumulate) {
      fill_zero_f32_kernel<<<1, 256, 0, c.st>>>(rms->dgamma, s->d);
      FLCE_TRY(launch_ok());
    }
    if (buckets != nullptr) {
      // nothing to wait for: every bucket is final now
      for (int b = 0; b < buckets->n; ++b) {
        if (buckets->events[b] != nullptr &&
            cudaEventRecord(static_cast<cudaEvent_t>(buckets->events[b]), c.st) != cudaSuccess)
          return FLCE_ERR_CUDA;
        if (buckets->bounds != nullptr) {
          const int vtiles = static_cast<int>((s->Vpad + Cfg::BM - 1) / Cfg::BM);
          buckets->bounds[b] = static_cast<int64_t>(b) * vtiles / buckets->n * Cfg::BM;
          buckets->bounds[b + 1] =
              b + 1 == buckets->n ? s->Vpad
                                  : static_cast<int64_t>(b + 1) * vtiles / buckets->n * Cfg::BM;
        }
      }
    }
    return FLCE_OK;
  }
  if (want_grads && c.L.fixed_ref) {
    for (int64_t row0 = 0; row0 < s->N; row0 += c.L.chunk) {
      const int rows = static_cast<int>(s->N - row0 < c.L.chunk ? s->N - row0 : c.L.chunk);
      const bool last = row0 + rows >= s->N;
      FLCE_TRY(grad_chunk(c, row0, rows, Xb, Wb, nullptr, lse, grad_scale, dXout, dW,
                          (row0 > 0 || accumulate_dW) ? 1 : 0, LOGITS_FUSED,
                          last ? buckets : nullptr));
    }
  } else {
    FLCE_TRY(stats_pass(c, Xb, Wb, lse));
  }
  loss_kernel<<<1, 1024, 0, c.st>>>(c.at<float>(c.L.row_loss), s->N, c.hdr, c.nv_total, loss);
  FLCE_TRY(launch_ok());
  if (want_grads && !c.L.fixed_ref) {
    // Without a fixed exp reference the gradient needs lse first: recompute with it.
    for (int64_t row0 = 0; row0 < s->N; row0 += c.L.chunk) {
      const int rows = static_cast<int>(s->N - row0 < c.L.chunk ? s->N - row0 : c.L.chunk);
      const bool last = row0 + rows >= s->N;
      FLCE_TRY(grad_chunk(c, row0, rows, Xb, Wb, lse, nullptr, grad_scale, dXout, dW,
                          (row0 > 0 || accumulate_dW) ? 1 : 0, LOGITS_RECOMPUTE,
                          last ? buckets : nullptr));
    }
  }
  if (rms != nullptr && want_grads && !fold)
    FLCE_TRY(rmsnorm_backward_kernels(rms->H, rms->gamma, c.at<float>(c.L.rstd), dXout, s->N,
                                      static_cast<int>(s->d), rms->dH, rms->dgamma,
                                      rms->accumulate, c.at<float>(c.L.rmspart), c.st));
  return FLCE_OK;
}

}  // namespace

extern "C" {

size_t flce_workspace_bytes(const flce_shape* shape, int want_grads) {
  if (!shape_ok(shape)) return 0;
  return make_layout(shape, want_grads ? 1 : 0).total;
}

int flce_forward(const flce_shape* s, const void* X, const void* W, const int64_t* targets,
                 float* loss, float* lse, int want_grads, const float* grad_scale, void* dX,
                 void* dW, int dW_dtype, int accumulate_dW, void* workspace,
                 size_t workspace_bytes, void* stream) {
  FLCE_TRY(common_checks(s, X, W, targets, workspace, workspace_bytes, want_grads ? 1 : 0));
  return forward_impl(s, X, W, Fp8Logits{}, targets, loss, lse, want_grads, grad_scale, dX, dW,
                      dW_dtype, accumulate_dW, workspace, workspace_bytes, stream);
}

int flce_count_valid(const flce_shape* s, const int64_t* targets, int64_t* n_valid_out,
                     void* stream) {
  if (!shape_ok(s) || n_valid_out == nullptr || (s->N > 0 && targets == nullptr))
    return FLCE_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(n_valid_out) & 7u) != 0 || !aligned16(targets))
    return FLCE_ERR_ALIGN;
  DeviceInfo* di = nullptr;
  FLCE_TRY(device_info(&di));
  count_valid_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const long long*>(targets), s->N, s->Vreal, s->ignore_index,
      reinterpret_cast<long long*>(n_valid_out));
  return launch_ok();
}

int flce_forward_dp(const flce_shape* s, const void* X, const void* W, const int64_t* targets,
                    const int64_t* n_valid_total, float* loss, float* lse, int want_grads,
                    const float* grad_scale, void* dX, void* dW, int dW_dtype,
                    int accumulate_dW, void* workspace, size_t workspace_bytes, void* stream) {
  FLCE_TRY(common_checks(s, X, W, targets, workspace, workspace_bytes, want_grads ? 1 : 0));
  if (n_valid_total == nullptr) return FLCE_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(n_valid_total) & 7u) != 0) return FLCE_ERR_ALIGN;
  return forward_impl(s, X, W, Fp8Logits{}, targets, loss, lse, want_grads, grad_scale, dX, dW,
                      dW_dtype, accumulate_dW, workspace, workspace_bytes, stream,
                      n_valid_total);
}

int flce_forward_dp_bucketed(const flce_shape* s, const void* X, const void* W,
                             const int64_t* targets, const int64_t* n_valid_total, float* loss,
                             float* lse, const float* grad_scale, void* dX, void* dW,
                             int dW_dtype, int accumulate_dW, int n_buckets,
                             void* const* bucket_events, int64_t* bucket_bounds,
                             void* workspace, size_t workspace_bytes, void* stream) {
  FLCE_TRY(common_checks(s, X, W, targets, workspace, workspace_bytes, 1));
  if (n_valid_total == nullptr || bucket_events == nullptr || bucket_bounds == nullptr)
    return FLCE_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(n_valid_total) & 7u) != 0) return FLCE_ERR_ALIGN;
  const int64_t vtiles = (s->Vpad + Cfg::BM - 1) / Cfg::BM;
  if (n_buckets < 1 || n_buckets > 64 || n_buckets > vtiles) return FLCE_ERR_ARG;
  for (int b = 0; b < n_buckets; ++b)
    if (bucket_events[b] == nullptr) return FLCE_ERR_ARG;
  const Buckets bk{n_buckets, bucket_events, bucket_bounds};
  return forward_impl(s, X, W, Fp8Logits{}, targets, loss, lse, 1, grad_scale, dX, dW,
                      dW_dtype, accumulate_dW, workspace, workspace_bytes, stream,
                      n_valid_total, &bk);
}

int flce_forward_fp8(const flce_shape* s, const void* X8, const void* W8, const float* scale_x,
                     const float* scale_w, const void* X, const void* W, const int64_t* targets,
                     float* loss, float* lse, int want_grads, int grad_fp8,
                     const float* grad_scale, void* dX, void* dW, int dW_dtype,
                     int accumulate_dW, void* workspace, size_t workspace_bytes, void* stream) {
  if (!shape_ok(s)) return FLCE_ERR_ARG;
  if ((s->d % 16) != 0 || (s->Vpad % 8) != 0) return FLCE_ERR_ALIGN;  // 16-byte e4m3 rows
  if ((s->N > 0 && (X8 == nullptr || targets == nullptr)) || W8 == nullptr ||
      scale_x == nullptr || scale_w == nullptr || workspace == nullptr)
    return FLCE_ERR_ARG;
  // the bf16 copies feed the gradient contractions unless those read the 8-bit operands
  if (want_grads && !grad_fp8 && ((s->N > 0 && X == nullptr) || W == nullptr))
    return FLCE_ERR_ARG;
  // 8-bit gradients: the exp reference is the cap (0 < cap <= 32), the rows are compacted
  if (want_grads && grad_fp8 && (!(s->cap > 0.f && s->cap <= kFixedRefMaxCap) || !FLCE_COMPACT))
    return FLCE_ERR_ARG;
  if (!aligned16(X8) || !aligned16(W8) || !aligned16(X) || !aligned16(W) || !aligned16(targets) ||
      (reinterpret_cast<uintptr_t>(scale_x) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(scale_w) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return FLCE_ERR_ALIGN;
  if (workspace_bytes < make_layout(s, want_grads ? 1 : 0).total) return FLCE_ERR_WORKSPACE;
  Fp8Logits fp8;
  fp8.X8 = static_cast<const uint8_t*>(X8);
  fp8.W8 = static_cast<const uint8_t*>(W8);
  fp8.scale_x = scale_x;
  fp8.scale_w = scale_w;
  return forward_impl(s, X, W, fp8, targets, loss, lse, want_grads, grad_scale, dX, dW,
                      dW_dtype, accumulate_dW, workspace, workspace_bytes, stream, nullptr,
                      nullptr, grad_fp8);
}

int flce_quantize_e4m3(const void* src, int64_t n, void* dst, float* scale_out, void* stream) {
  if (n < 0 || (n > 0 && (src == nullptr || dst == nullptr)) || scale_out == nullptr)
    return FLCE_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(scale_out) & 3u) != 0) return FLCE_ERR_ALIGN;
  DeviceInfo* di = nullptr;
  FLCE_TRY(device_info(&di));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* amax_bits = reinterpret_cast<uint32_t*>(scale_out);
  const int grid = 4 * di->sms;
  zero_u32_kernel<<<1, 1, 0, st>>>(amax_bits);
  FLCE_TRY(launch_ok());
  if (n > 0) {
    amax_bf16_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(src), n, amax_bits);
    FLCE_TRY(launch_ok());
    quantize_e4m3_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(src), n,
                                                 static_cast<uint8_t*>(dst), amax_bits);
    FLCE_TRY(launch_ok());
  }
  finish_scale_kernel<<<1, 1, 0, st>>>(amax_bits);
  return launch_ok();
}

int flce_backward(const flce_shape* s, const void* X, const void* W, const int64_t* targets,
                  const float* lse, const float* grad_out, void* dX, void* dW, int dW_dtype,
                  int accumulate_dW, int grads_precomputed, void* workspace,
                  size_t workspace_bytes, void* stream) {
  if (!shape_ok(s)) return FLCE_ERR_ARG;
  if ((s->N > 0 && dX == nullptr) || dW == nullptr) return FLCE_ERR_ARG;
  if (dW_dtype != FLCE_DTYPE_F32 && dW_dtype != FLCE_DTYPE_BF16) return FLCE_ERR_ARG;
  if (!aligned16(dX) || !aligned16(dW)) return FLCE_ERR_ALIGN;
  if (grad_out != nullptr && (reinterpret_cast<uintptr_t>(grad_out) & 3u) != 0)
    return FLCE_ERR_ALIGN;
  const int dW_bf16 = dW_dtype == FLCE_DTYPE_BF16 ? 1 : 0;
  if (grads_precomputed) {
    // Scaling after the fact is only right for gradients this call's forward wrote; a dW that
    // holds earlier micro-batches must get g through the forward's grad_scale instead.
    if (accumulate_dW) return FLCE_ERR_ARG;
    if ((s->d % 8) != 0) return FLCE_ERR_ALIGN;
    DeviceInfo* di = nullptr;
    FLCE_TRY(device_info(&di));
    if (grad_out == nullptr) return FLCE_OK;
    const long long nX8 = s->N * s->d / 8;
    const long long nW = s->Vpad * s->d / (dW_bf16 ? 8 : 4);
    scale_grads_kernel<<<4 * di->sms, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<__nv_bfloat16*>(dX), nX8, dW, nW, dW_bf16, grad_out);
    return launch_ok();
  }
  FLCE_TRY(common_checks(s, X, W, targets, workspace, workspace_bytes, 1));
  if (s->N > 0 && lse == nullptr) return FLCE_ERR_ARG;
  if (!aligned4(lse)) return FLCE_ERR_ALIGN;
  DeviceInfo* di = nullptr;
  FLCE_TRY(device_info(&di));
  Ctx c{};
  c.s = s;
  c.dW_bf16 = dW_bf16;
  c.L = make_layout(s, 1);
  c.ws = static_cast<uint8_t*>(workspace);
  c.di = di;
  c.st = static_cast<cudaStream_t>(stream);
  c.hdr = c.at<DevHeader>(c.L.hdr);
  FLCE_TRY(prep(c, targets));
  if (s->N == 0) {
    if (!accumulate_dW) FLCE_TRY(zero_dW(c, dW));
    return FLCE_OK;
  }
  for (int64_t row0 = 0; row0 < s->N; row0 += c.L.chunk) {
    const int rows = static_cast<int>(s->N - row0 < c.L.chunk ? s->N - row0 : c.L.chunk);
    FLCE_TRY(grad_chunk(c, row0, rows, static_cast<const __nv_bfloat16*>(X),
                        static_cast<const __nv_bfloat16*>(W), lse, nullptr, grad_out,
                        static_cast<__nv_bfloat16*>(dX), dW, (row0 > 0 || accumulate_dW) ? 1 : 0,
                        LOGITS_RECOMPUTE));
  }
  return FLCE_OK;
}

int flce_forward_noalloc(const flce_shape* shape, const void* X, const void* W,
                         const int64_t* targets, float* loss, float* lse, void* stream) {
  if (!shape_ok(shape)) return FLCE_ERR_ARG;
  flce_shape s = *shape;
  if (s.chunk_rows == 0) {
    s.chunk_rows = 128;
    for (int64_t c = 4096; c >= 128; c /= 2) {
      flce_shape t = s;
      t.chunk_rows = c;
      if (make_layout(&t, 0).total <= FLCE_NOALLOC_SCRATCH_BYTES) {
        s.chunk_rows = c;
        break;
      }
    }
  }
  if (make_layout(&s, 0).total > FLCE_NOALLOC_SCRATCH_BYTES) return FLCE_ERR_WORKSPACE;
  DeviceInfo* di = nullptr;
  FLCE_TRY(device_info(&di));
  void* scratch = nullptr;
  FLCE_TRY(noalloc_scratch_address(&scratch));
  return flce_forward(&s, X, W, targets, loss, lse, 0, nullptr, nullptr, nullptr,
                      FLCE_DTYPE_F32, 0, scratch, FLCE_NOALLOC_SCRATCH_BYTES, stream);
}


static int rms_args_ok(const void* H, const void* gamma, int64_t N, int64_t d) {
  if (N < 0 || d <= 0 || d > (int64_t(1) << 24) || gamma == nullptr || (N > 0 && H == nullptr))
    return FLCE_ERR_ARG;
  if ((d % 8) != 0 || !aligned16(H) || !aligned16(gamma)) return FLCE_ERR_ALIGN;
  return FLCE_OK;
}

int flce_rmsnorm_forward(const void* H, const void* gamma, float eps, int64_t N, int64_t d,
                         void* X, float* rstd, void* stream) {
  FLCE_TRY(rms_args_ok(H, gamma, N, d));
  if (!(eps >= 0.f) || (N > 0 && (X == nullptr || rstd == nullptr))) return FLCE_ERR_ARG;
  if (!aligned16(X) || (reinterpret_cast<uintptr_t>(rstd) & 3u) != 0) return FLCE_ERR_ALIGN;
  DeviceInfo* di = nullptr;
  FLCE_TRY(device_info(&di));
  if (N == 0) return FLCE_OK;
  rmsnorm_fwd_kernel<<<static_cast<unsigned>((N + 7) / 8), 256, 0,
                       static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(H), static_cast<const __nv_bfloat16*>(gamma), eps, N,
      static_cast<int>(d), static_cast<__nv_bfloat16*>(X), rstd);
  return launch_ok();
}

size_t flce_rmsnorm_workspace_bytes(int64_t N, int64_t d) {
  if (N < 0 || d <= 0) return 0;
  const int64_t parts = N > 0 ? (N + kRmsRowsPerPart - 1) / kRmsRowsPerPart : 1;
  return align_up(static_cast<size_t>(parts) * static_cast<size_t>(d) * sizeof(float));
}

int flce_rmsnorm_backward(const void* H, const void* gamma, const float* rstd, const void* dX,
                          int64_t N, int64_t d, void* dH, float* dgamma, int accumulate_dgamma,
                          void* workspace, size_t workspace_bytes, void* stream) {
  FLCE_TRY(rms_args_ok(H, gamma, N, d));
  if (dgamma == nullptr || workspace == nullptr ||
      (N > 0 && (rstd == nullptr || dX == nullptr || dH == nullptr)))
    return FLCE_ERR_ARG;
  if (!aligned16(dX) || !aligned16(dH) || (reinterpret_cast<uintptr_t>(dgamma) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(rstd) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
    return FLCE_ERR_ALIGN;
  if (workspace_bytes < flce_rmsnorm_workspace_bytes(N, d)) return FLCE_ERR_WORKSPACE;
  DeviceInfo* di = nullptr;
  FLCE_TRY(device_info(&di));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return rmsnorm_backward_kernels(
      static_cast<const __nv_bfloat16*>(H), static_cast<const __nv_bfloat16*>(gamma), rstd,
      static_cast<const __nv_bfloat16*>(dX), N, static_cast<int>(d),
      static_cast<__nv_bfloat16*>(dH), dgamma, accumulate_dgamma,
      static_cast<float*>(workspace), st);
}

size_t flce_workspace_bytes_rmsnorm(const flce_shape* shape, int want_grads) {
  if (!shape_ok(shape)) return 0;
  return make_layout(shape, want_grads ? 1 : 0, 1).total;
}

static int forward_rmsnorm_impl(const flce_shape* s, const void* H, const void* gamma, float eps,
                                const void* W, const int64_t* targets,
                                const int64_t* n_valid_total, float* loss, float* lse,
                                int want_grads, const float* grad_scale, void* dH, float* dgamma,
                                void* dW, int dW_dtype, int accumulate, void* workspace,
                                size_t workspace_bytes, void* stream) {
  want_grads = want_grads ? 1 : 0;
  if (!shape_ok(s)) return FLCE_ERR_ARG;
  FLCE_TRY(rms_args_ok(H, gamma, s->N, s->d));
  if (!(eps >= 0.f)) return FLCE_ERR_ARG;
  if ((s->Vpad % 8) != 0) return FLCE_ERR_ALIGN;
  if ((s->N > 0 && targets == nullptr) || W == nullptr || workspace == nullptr)
    return FLCE_ERR_ARG;
  if (!aligned16(W) || !aligned16(targets) ||
      (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 ||
      (reinterpret_cast<uintptr_t>(n_valid_total) & 7u) != 0)
    return FLCE_ERR_ALIGN;
  if (workspace_bytes < make_layout(s, want_grads, 1).total) return FLCE_ERR_WORKSPACE;
  if (want_grads) {
    if (dgamma == nullptr) return FLCE_ERR_ARG;
    if (!aligned4(dgamma)) return FLCE_ERR_ALIGN;
  }
  const RmsFold rf{static_cast<const __nv_bfloat16*>(H), static_cast<const __nv_bfloat16*>(gamma),
                   eps, static_cast<__nv_bfloat16*>(dH), dgamma, accumulate ? 1 : 0};
  // the head's input is the normalised rows forward_impl writes; dH takes dX's place
  return forward_impl(s, nullptr, W, Fp8Logits{}, targets, loss, lse, want_grads, grad_scale, dH,
                      dW, dW_dtype, accumulate, workspace, workspace_bytes, stream, n_valid_total,
                      nullptr, 0, &rf);
}

int flce_forward_rmsnorm(const flce_shape* s, const void* H, const void* gamma, float eps,
                         const void* W, const int64_t* targets, float* loss, float* lse,
                         int want_grads, const float* grad_scale, void* dH, float* dgamma,
                         void* dW, int dW_dtype, int accumulate, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return forward_rmsnorm_impl(s, H, gamma, eps, W, targets, nullptr, loss, lse, want_grads,
                              grad_scale, dH, dgamma, dW, dW_dtype, accumulate, workspace,
                              workspace_bytes, stream);
}

int flce_forward_rmsnorm_dp(const flce_shape* s, const void* H, const void* gamma, float eps,
                            const void* W, const int64_t* targets, const int64_t* n_valid_total,
                            float* loss, float* lse, int want_grads, const float* grad_scale,
                            void* dH, float* dgamma, void* dW, int dW_dtype, int accumulate,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (n_valid_total == nullptr) return FLCE_ERR_ARG;
  return forward_rmsnorm_impl(s, H, gamma, eps, W, targets, n_valid_total, loss, lse, want_grads,
                              grad_scale, dH, dgamma, dW, dW_dtype, accumulate, workspace,
                              workspace_bytes, stream);
}

int flce_scale_grads_rmsnorm(const flce_shape* s, const float* grad_out, void* dH, float* dgamma,
                             void* dW, int dW_dtype, void* stream) {
  if (!shape_ok(s) || dgamma == nullptr || dW == nullptr || (s->N > 0 && dH == nullptr))
    return FLCE_ERR_ARG;
  if (dW_dtype != FLCE_DTYPE_F32 && dW_dtype != FLCE_DTYPE_BF16) return FLCE_ERR_ARG;
  if ((s->d % 8) != 0 || !aligned16(dH) || !aligned16(dW) || !aligned4(dgamma) ||
      !aligned4(grad_out))
    return FLCE_ERR_ALIGN;
  DeviceInfo* di = nullptr;
  FLCE_TRY(device_info(&di));
  if (grad_out == nullptr) return FLCE_OK;
  const int dW_bf16 = dW_dtype == FLCE_DTYPE_BF16 ? 1 : 0;
  scale_grads_kernel<<<4 * di->sms, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<__nv_bfloat16*>(dH), s->N * s->d / 8, dW, s->Vpad * s->d / (dW_bf16 ? 8 : 4),
      dW_bf16, grad_out, dgamma, s->d);
  return launch_ok();
}

int flce_selftest_wait_timeout(void* workspace, uint64_t limit_ns, void* stream) {
  if (workspace == nullptr) return FLCE_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return FLCE_ERR_ALIGN;
  if (limit_ns == 0 || limit_ns > 10000000000ull) return FLCE_ERR_ARG;   // at most 10 s
  DeviceInfo* di = nullptr;
  FLCE_TRY(device_info(&di));
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      &static_cast<DevHeader*>(workspace)->status, limit_ns);
  return launch_ok();
}

int flce_check_pair_schedule(int pairs, int T0, int c0, int T1, int c1, int64_t* max_cost,
                             int64_t* min_cost) {
  if (pairs < 1 || pairs > 4096 || T0 < 0 || T1 < 0 || T0 > (1 << 24) || T1 > (1 << 24) ||
      c0 < 1 || c1 < 1)
    return FLCE_ERR_ARG;
  std::vector<uint8_t> seen0(static_cast<size_t>(T0), 0), seen1(static_cast<size_t>(T1), 0);
  int64_t hi = 0, lo = INT64_MAX;
  for (int p = 0; p < pairs; ++p) {
    const PairSchedule ps = pair_schedule(p, pairs, T0, c0, T1, c1);
    if (ps.n0 < 0 || ps.qa < 0 || ps.qb < 0) return FLCE_ERR_ARG;
    const int total = ps.n0 + ps.qa + ps.qb;
    int64_t cost = 0;
    for (int i = 0; i < total; ++i) {
      const PairTile pt = pair_tile(ps, p, pairs, i);
      std::vector<uint8_t>& seen = pt.prob == 0 ? seen0 : seen1;
      if (pt.t < 0 || pt.t >= static_cast<int>(seen.size()) || seen[pt.t]) return FLCE_ERR_ARG;
      seen[pt.t] = 1;
      cost += pt.prob == 0 ? c0 : c1;
    }
    hi = cost > hi ? cost : hi;
    lo = cost < lo ? cost : lo;
  }
  for (uint8_t v : seen0)
    if (!v) return FLCE_ERR_ARG;
  for (uint8_t v : seen1)
    if (!v) return FLCE_ERR_ARG;
  if (max_cost) *max_cost = hi;
  if (min_cost) *min_cost = lo;
  return FLCE_OK;
}

int flce_read_status(const void* workspace, uint32_t* dev_status_out, int64_t* n_valid_out,
                     void* stream) {
  if (workspace == nullptr) {
    // the fixed scratch of flce_forward_noalloc on the current device
    void* scratch = nullptr;
    FLCE_TRY(noalloc_scratch_address(&scratch));
    workspace = scratch;
  }
  DevHeader h;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return FLCE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FLCE_ERR_CUDA;
  if (dev_status_out) *dev_status_out = h.status;
  if (n_valid_out) *n_valid_out = h.n_valid;
  return FLCE_OK;
}

int flce_instrument(int enable) {
  std::lock_guard<std::mutex> lock(g_instr_mu);
  if (enable) {
    for (auto& t : g_timed) {
      g_event_pool.push_back(t.start);
      g_event_pool.push_back(t.stop);
    }
    g_timed.clear();
    for (int k = 0; k < 3; ++k) g_done_ms[k] = g_done_flop[k] = 0, g_done_n[k] = 0;
    g_launches.store(0);
  }
  g_instr.store(enable ? 1 : 0);
  return FLCE_OK;
}

int flce_instrument_read(flce_kernel_stats* out) {
  if (out == nullptr) return FLCE_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_instr_mu);
  for (auto& t : g_timed) {
    if (cudaEventSynchronize(t.stop) != cudaSuccess) return FLCE_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, t.start, t.stop) != cudaSuccess) return FLCE_ERR_CUDA;
    g_done_ms[t.kind] += ms;
    g_done_flop[t.kind] += t.flop;
    g_done_n[t.kind] += 1;
    g_event_pool.push_back(t.start);
    g_event_pool.push_back(t.stop);
  }
  g_timed.clear();
  out->launches_total = g_launches.load();
  for (int k = 0; k < 3; ++k) {
    out->gemm_launches[k] = g_done_n[k];
    out->gemm_ms[k] = g_done_ms[k];
    out->gemm_flop[k] = g_done_flop[k];
  }
  return FLCE_OK;
}

const char* flce_status_string(int status) {
  switch (status) {
    case FLCE_OK: return "FLCE_OK";
    case FLCE_ERR_ARG: return "FLCE_ERR_ARG: invalid argument";
    case FLCE_ERR_ALIGN: return "FLCE_ERR_ALIGN: pointer or row stride not 16-byte aligned";
    case FLCE_ERR_WORKSPACE: return "FLCE_ERR_WORKSPACE: workspace too small";
    case FLCE_ERR_DEVICE: return "FLCE_ERR_DEVICE: device is not compute capability 10.0";
    case FLCE_ERR_CUDA: return "FLCE_ERR_CUDA: CUDA runtime error";
    case FLCE_ERR_TIMEOUT: return "FLCE_ERR_TIMEOUT: a device wait ran out";
    default: return "unknown flce status";
  }
}

}  // extern "C"
