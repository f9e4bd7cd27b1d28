// C ABI of the predictor-gated sparse FFN (declared in include/pi.h).
//
// Host side: argument validation, workspace layout, kernel selection and
// launches.  Every kernel is launched with programmatic stream serialization
// so its prologue (barrier set-up, weight prefetch) overlaps the tail of the
// kernel before it; each kernel waits (griddepcontrol.wait) before it touches
// that kernel's results.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <set>
#include <utility>
#include <cstring>
#include <string>

#include "../../include/pi.h"
#include "pi_generic.cuh"
#include "pi_umma.cuh"

using namespace pi;

// Fixed device scratch of pi_sparse_ffn_static: the per-CTA partial sums of y
// (and, on the batched path, the activations h).  It is part of the module
// image, so the call never allocates; every device the library runs on
// carries one copy, and concurrent calls on one device share it.
static __device__ __align__(256) uint8_t g_static_scratch[PI_STATIC_SCRATCH_BYTES];

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};

int32_t fail(int32_t status, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int32_t fail(int32_t status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

#define PI_CUDA(call)                                                                    \
  do {                                                                                   \
    cudaError_t e_ = (call);                                                             \
    if (e_ != cudaSuccess)                                                               \
      return fail(PI_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));          \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
  static thread_local int cached_dev = -1, cached = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev != cached_dev) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cached = v;
    cached_dev = dev;
  }
  return cached;
}

constexpr size_t kSmemMax = 227 * 1024;
constexpr size_t kSmemPred1 = 96 * 1024;
#ifndef PI_SMEM_PRED2_KB
#define PI_SMEM_PRED2_KB 160
#endif
constexpr size_t kSmemPred2 = PI_SMEM_PRED2_KB * 1024;
constexpr size_t kSmemFfn = 220 * 1024;  // shared by the CTAs on one SM
constexpr size_t kPartCap = 64ull << 20;  // bytes of batched down partials

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

// The fused FFN kernel runs ffn_cps(B) CTAs of 256 threads per SM: two at
// batch 1 (registers allow it, and two independent block-reduction domains
// per SM keep more copies in flight), one for larger batches.
#ifndef PI_LDG_CPS
#define PI_LDG_CPS 2
#endif
int ffn_cps(int B) { return B == 1 ? PI_LDG_CPS : 1; }
// up to this many partial planes are summed by k_reduce_few
constexpr int kReduceFew = 16;
int ffn_grid(int B);

// ------------------------------------------------------------ workspace
struct WsLayout {
  size_t bar, a, mask, umask, idx, count, xl, part, h, total;
};

int down_slices(int d, int B, int nsm) {
  const int ndc = (d / 8 + 255) / 256;
  int S = std::max(1, 2 * nsm / ndc);
  const size_t per = (size_t)B * d * 4;
  S = (int)std::min<size_t>((size_t)S, std::max<size_t>(1, kPartCap / per));
  return S;
}

WsLayout ws_layout(int d, int F, int r, int B) {
  const int nsm = num_sms();
  WsLayout w{};
  size_t o = 0;
  w.bar = o;   o += 256;
  w.a = o;     o += al256((size_t)kAReplicas * B * r * 4);
  w.mask = o;  o += al256((size_t)B * (F / 32) * 4);
  w.umask = o; o += al256((size_t)(F / 32) * 4);
  w.idx = o;   o += al256((size_t)F * 4);
  w.count = o; o += 256;
  w.xl = o;    o += al256((size_t)B * d * 2);
  const int G = std::max(ffn_cps(B) * nsm, down_slices(d, B, nsm));
  w.part = o;  o += al256((size_t)G * B * d * 4);
  w.h = o;     o += al256((size_t)F * B * 4);
  w.total = o;
  return w;
}

// ------------------------------------------------------------ launching
cudaError_t allow_large_smem(const void* kern) {
  // once per (device, kernel): allow the large dynamic shared memory carve-out
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const auto key = std::make_pair(dev, kern);
  std::lock_guard<std::mutex> lock(mu);
  if (!done.count(key)) {
    // the carve-out is shared with the kernel's static shared memory
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(kSmemMax - fa.sharedSizeBytes));
    if (e != cudaSuccess) return e;
    done.insert(key);
  }
  return cudaSuccess;
}

template <typename Kern, typename... Args>
cudaError_t launch(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   Args... args) {
  if (smem > 48 * 1024) {
    const cudaError_t e = allow_large_smem(reinterpret_cast<const void*>(kern));
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}

// ------------------------------------------------------------ validation
int check_act_dtype(int dt) { return dt == PI_F16 || dt == PI_BF16; }

int32_t validate_predictor(const pi_predictor* p) {
  if (!p) return fail(PI_ERR_INVALID_ARG, "predictor is NULL");
  if (!check_act_dtype(p->dtype))
    return fail(PI_ERR_UNSUPPORTED, "predictor dtype must be PI_F16 or PI_BF16 (got %d)", p->dtype);
  if (p->d_model < 32 || p->d_model > 8192 || p->d_model % 32)
    return fail(PI_ERR_UNSUPPORTED, "d_model %d: need 32 <= d_model <= 8192, multiple of 32",
                p->d_model);
  if (p->d_ff < 32 || p->d_ff > 65536 || p->d_ff % 32)
    return fail(PI_ERR_UNSUPPORTED, "d_ff %d: need 32 <= d_ff <= 65536, multiple of 32", p->d_ff);
  if (p->rank < 8 || p->rank > 2048 || p->rank % 8)
    return fail(PI_ERR_UNSUPPORTED, "rank %d: need 8 <= rank <= 2048, multiple of 8", p->rank);
  if (!p->w1 || !p->w2 || !p->b2) return fail(PI_ERR_INVALID_ARG, "predictor w1, w2 and b2 are required");
  if (!aligned16(p->w1) || !aligned16(p->w2) || !aligned16(p->b2) || (p->b1 && !aligned16(p->b1)))
    return fail(PI_ERR_INVALID_ARG, "predictor pointers must be 16-byte aligned");
  return PI_OK;
}

int32_t validate_layer(const pi_layer* L) {
  if (!L) return fail(PI_ERR_INVALID_ARG, "layer is NULL");
  if (int32_t s = validate_predictor(&L->pred)) return s;
  if (L->d_model != L->pred.d_model || L->d_ff != L->pred.d_ff)
    return fail(PI_ERR_INVALID_ARG, "layer and predictor disagree on d_model/d_ff");
  if (!check_act_dtype(L->adtype) || L->adtype != L->pred.dtype)
    return fail(PI_ERR_UNSUPPORTED, "adtype must be PI_F16/PI_BF16 and equal the predictor dtype");
  if (L->act != PI_RELU && L->act != PI_REGLU && L->act != PI_SQRELU)
    return fail(PI_ERR_UNSUPPORTED, "act must be PI_RELU, PI_REGLU or PI_SQRELU");
  if (L->wdtype == PI_F16 || L->wdtype == PI_BF16) {
    if (L->wdtype != L->adtype)
      return fail(PI_ERR_UNSUPPORTED, "16-bit weights must have the activation dtype");
  } else if (L->wdtype == PI_Q4_0) {
    if (L->adtype != PI_F16) return fail(PI_ERR_UNSUPPORTED, "Q4_0 weights need fp16 activations");
    if (L->d_model % 256)
      return fail(PI_ERR_UNSUPPORTED, "Q4_0 needs d_model %% 256 == 0 (16-byte aligned rows)");
  } else {
    return fail(PI_ERR_UNSUPPORTED, "wdtype %d unknown", L->wdtype);
  }
  if (!L->w_up || !L->w_down_t) return fail(PI_ERR_INVALID_ARG, "w_up and w_down_t are required");
  if ((L->act == PI_REGLU) != (L->w_gate != nullptr))
    return fail(PI_ERR_INVALID_ARG, "w_gate must be given exactly for ReGLU");
  if (L->act != PI_REGLU && L->b_gate)
    return fail(PI_ERR_INVALID_ARG, "b_gate is only meaningful for ReGLU");
  if (L->act == PI_REGLU && L->b_up)
    return fail(PI_ERR_INVALID_ARG, "ReGLU has no up-projection bias (use b_gate)");
  const void* ps[] = {L->w_up, L->w_gate, L->w_down_t, L->b_up, L->b_gate};
  for (const void* q : ps)
    if (q && !aligned16(q)) return fail(PI_ERR_INVALID_ARG, "layer pointers must be 16-byte aligned");
  return PI_OK;
}

int32_t validate_batch(int B) {
  if (B < 1 || B > kMaxBatch)
    return fail(PI_ERR_UNSUPPORTED, "batch %d: need 1 <= batch <= %d", B, kMaxBatch);
  return PI_OK;
}

int32_t check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return PI_OK;
  if (!ws) return fail(PI_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
  if (!aligned16(ws)) return fail(PI_ERR_WORKSPACE, "workspace must be 16-byte aligned");
  if (have < need) return fail(PI_ERR_WORKSPACE, "workspace has %zu bytes, need %zu", have, need);
  return PI_OK;
}

// ------------------------------------------------- tensor-core batched path
// Batches of at least kUmmaMinBatch tokens that the fused batch-1/2/4
// kernels do not take run the gathered up and down projections as tcgen05
// GEMMs (pi_umma.cuh), N = the batch rounded up to 16: the rows are read
// once either way, and the tensor cores leave the CUDA cores' FMA issue
// (half the issue slots of the batch-5 row kernels) out of the path.  Their
// operands are described to the copy engine by tensor maps built here.
constexpr int kUmmaMinBatch = 3;

PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

// A row-major [rows x inner] tensor of 16-bit values, read in boxes of
// box_inner x box_rows with the 128-byte swizzle; rows and columns outside the
// tensor read as zeros.
bool make_tmap16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows) {
  auto enc = tmap_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool umma_ok(const pi_layer* L, int B) {
  return B >= kUmmaMinBatch && B <= 64 && L->d_model % kUmmaM == 0 && tmap_encoder() != nullptr;
}

// Pipeline stages (at least 2, at most 6) within a shared-memory budget
// that keeps two CTAs on an SM.  16-bit operands arrive by asynchronous
// copies, which land in the stage buffers: the whole budget goes to stages.
// Q4_0 operands are loaded through the L1 and decoded in registers, and
// fewer stages leave the L1 more room for loads in flight (measured: 75 KB
// beats 110 KB by 12-15% there, and loses by as much on 16-bit rows).
constexpr int umma_ns(int stage_bytes, bool q4 = false) {
  const int budget = (q4 ? 75 : 110) * 1024;
  return budget / stage_bytes < 2 ? 2 : budget / stage_bytes > 6 ? 6 : budget / stage_bytes;
}

// ------------------------------------------------------------ predictor
template <int DT, int B, int CPT>
cudaError_t launch_pred1(const pi_predictor* P, const uint16_t* x, const float* xr,
                         uint16_t* xo, float* a, cudaStream_t st) {
  const int nsm = num_sms();
  Pred1Params p{};
  p.w1 = static_cast<const uint8_t*>(P->w1);
  p.b1 = P->b1;
  p.x = x;
  p.x_resid = xr;
  p.x_out = xo;
  p.a = a;
  p.d = P->d_model;
  p.r = P->rank;
  const int G = std::min(nsm, P->rank);
  p.rows_per_cta = (P->rank + G - 1) / G;
  const size_t row = (size_t)P->d_model * 2;
  const size_t xb = ((size_t)B * P->d_model * 2 + 127) & ~size_t(127);
  const size_t avail = kSmemPred1 > 2048 + xb ? kSmemPred1 - 2048 - xb : 0;
  p.nstages = (int)std::max<size_t>(kRowGroup, std::min<size_t>(std::max(p.rows_per_cta, kRowGroup),
                                                                std::min<size_t>(32, avail / row)));
  const size_t smem = 2048 + xb + (size_t)p.nstages * row;
  return launch(k_pred1<DT, B, CPT>, dim3(G), dim3(kThreads), smem, st, p);
}

// x held in registers: B x CPT 16-byte chunks per thread (B * CPT <= 16)
bool pred1_fused_ok(int B, int d) {
  const int cpt = (d / 8 + kConsumers - 1) / kConsumers;
  return (B == 1 || B == 2 || B == 4) && cpt <= 4 && B * cpt <= 8;
}

template <int DT, int B>
cudaError_t pred1_cpt(const pi_predictor* P, const uint16_t* x, const float* xr, uint16_t* xo,
                      float* a, cudaStream_t st) {
  const int cpt = (P->d_model / 8 + kConsumers - 1) / kConsumers;
  if (cpt <= 1) return launch_pred1<DT, B, 1>(P, x, xr, xo, a, st);
  if (cpt <= 2) return launch_pred1<DT, B, 2>(P, x, xr, xo, a, st);
  if constexpr (B <= 2) return launch_pred1<DT, B, 4>(P, x, xr, xo, a, st);
  return cudaErrorInvalidValue;
}

template <int DT>
cudaError_t pred1_dispatch(const pi_predictor* P, int B, const uint16_t* x, const float* xr,
                           uint16_t* xo, float* a, cudaStream_t st) {
  switch (B) {
    case 1: return pred1_cpt<DT, 1>(P, x, xr, xo, a, st);
    case 2: return pred1_cpt<DT, 2>(P, x, xr, xo, a, st);
    default: return pred1_cpt<DT, 4>(P, x, xr, xo, a, st);
  }
}

int cpl_for(int r) {
  const int need = (r / 8 + 31) / 32;
  for (int c : {1, 2, 4, 6, 8})
    if (c >= need) return c;
  return 0;
}

bool pred2_fused_ok(int B, int r) {
  const int c = cpl_for(r);
  return c > 0 && (B == 1 || B == 2) && B * c <= 8;
}

template <int DT, int B, int CPL>
cudaError_t launch_pred2(const pi_predictor* P, const float* a, uint32_t* mask, float* logits,
                         cudaStream_t st) {
  const int nsm = num_sms();
  Pred2Params p{};
  p.w2 = static_cast<const uint8_t*>(P->w2);
  p.b2 = P->b2;
  p.a = a;
  p.mask = mask;
  p.logits = logits;
  p.threshold = P->threshold;
  p.F = P->d_ff;
  p.r = P->rank;
  const int nunits = P->d_ff / 32;
  p.units_per_cta = (nunits + nsm - 1) / nsm;
  const int G = (nunits + p.units_per_cta - 1) / p.units_per_cta;
  const size_t stage = (size_t)8 * P->rank * 2;
  const size_t fixed = 1024 + (((size_t)p.units_per_cta * 32 * 4 + 127) & ~size_t(127));
  const size_t avail = kSmemPred2 > fixed ? kSmemPred2 - fixed : 0;
  // a unit's four stages go to four warp pairs; with fewer than four stages a
  // pair could wait on a stage phase ahead of the one in progress
  p.nstages = (int)std::min<size_t>((size_t)4 * p.units_per_cta, std::min<size_t>(32, avail / stage));
  if (p.nstages < 4 && p.nstages < 4 * p.units_per_cta) return cudaErrorInvalidValue;
  const size_t smem = fixed + (size_t)p.nstages * stage;
  return launch(k_pred2<DT, B, CPL>, dim3(G), dim3(kThreads), smem, st, p);
}

template <int DT, int B>
cudaError_t pred2_cpl(const pi_predictor* P, const float* a, uint32_t* mask, float* logits,
                      cudaStream_t st) {
  switch (cpl_for(P->rank)) {
    case 1: return launch_pred2<DT, B, 1>(P, a, mask, logits, st);
    case 2: return launch_pred2<DT, B, 2>(P, a, mask, logits, st);
    case 4: return launch_pred2<DT, B, 4>(P, a, mask, logits, st);
    case 6: if constexpr (B == 1) return launch_pred2<DT, B, 6>(P, a, mask, logits, st); break;
    case 8: if constexpr (B == 1) return launch_pred2<DT, B, 8>(P, a, mask, logits, st); break;
  }
  return cudaErrorInvalidValue;
}

// batches of 8+ with 16-bit rows: tensor-core tiles of 16 rows x 8 tokens
template <int MODE, int WDT, int ACT, int NT>
cudaError_t launch_rows_mma_nt(const RowsParams& p, int tiles, int Y, cudaStream_t st) {
  constexpr int NUP = (MODE == kModeUp && ACT == 1) ? 2 : 1;
  const size_t smem = (size_t)kMmaWarps * NUP * NT * 4 * 32 * sizeof(float);
  return launch(k_rows_mma<MODE, WDT, ACT, NT>, dim3(tiles, Y), dim3(32 * kMmaWarps), smem, st, p);
}

// one CTA per tile of 16 rows (the upper bound nrows_work; CTAs past the
// device-side row count return at once) and slice of the contraction (Y > 1:
// predictor layer 1 only, raw sums to p.part)
template <int MODE, int WDT, int ACT>
cudaError_t launch_rows_mma(const RowsParams& p, int nrows_work, cudaStream_t st, int Y = 1) {
  const int tiles = std::max(1, (nrows_work + 15) / 16);
  const int nt = (p.B + 7) / 8;
  if (nt <= 1) return launch_rows_mma_nt<MODE, WDT, ACT, 1>(p, tiles, Y, st);
  if (nt <= 2) return launch_rows_mma_nt<MODE, WDT, ACT, 2>(p, tiles, Y, st);
  if (nt <= 4) return launch_rows_mma_nt<MODE, WDT, ACT, 4>(p, tiles, Y, st);
  return launch_rows_mma_nt<MODE, WDT, ACT, 8>(p, tiles, Y, st);
}

template <int DT, int MODE, int BB>
cudaError_t launch_rows(const RowsParams& p, int nrows_work, cudaStream_t st) {
  const int nsm = num_sms();
  const int warps = std::max(1, nrows_work);
  const int blocks = std::min((warps + 7) / 8, nsm * 8);
  return launch(k_rows<MODE, DT, 0, BB>, dim3(blocks), dim3(256), 0, st, p);
}

template <int DT, int MODE>
cudaError_t rows_bb(const RowsParams& p, int nrows_work, cudaStream_t st) {
  if (MODE == kModePred1 && p.B >= 8) return launch_rows_mma<kModePred1, DT, 0>(p, nrows_work, st);
  if (p.B <= 8) return launch_rows<DT, MODE, 8>(p, nrows_work, st);
  if (p.B <= 32) return launch_rows<DT, MODE, 32>(p, nrows_work, st);
  return launch_rows<DT, MODE, 64>(p, nrows_work, st);
}

// Both predictor layers in one kernel (batch 1-2): chunks per thread of a W1
// row (CPT) and per lane of a W2 row (CPL).
int pred_cpt(int d) {
  const int need = (d / 8 + kPredThreads - 1) / kPredThreads;
  for (int c : {1, 2, 4})
    if (c >= need) return c;
  return 0;
}
int pred_cpl(int r) {
  const int need = (r / 8 + 31) / 32;
  for (int c : {1, 2, 4, 8})
    if (c >= need) return c;
  return 0;
}

template <int DT, int B, int CPT, int CPL>
cudaError_t launch_predict(const pi_predictor* P, const uint16_t* x, const float* xr,
                           uint16_t* xo, float* a, uint32_t* mask, float* logits, uint32_t* bar,
                           cudaStream_t st) {
  auto kern = k_predict<DT, B, CPT, CPL>;
  // every CTA must be resident at once for the grid barrier
  int occ = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kPredThreads, 0);
  if (e != cudaSuccess) return e;
  // the grid barrier's ticket counter needs one grid size for every launch
  if (occ < 2) return cudaErrorInvalidConfiguration;
  const int G = num_sms() * 2;
  if ((P->d_ff / 8 + G - 1) / G > kPredMaxUnits || (P->rank + G - 1) / G > kPredMaxRows1)
    return cudaErrorInvalidValue;
  PredParams p{};
  p.w1 = static_cast<const uint8_t*>(P->w1);
  p.b1 = P->b1;
  p.x = x;
  p.x_resid = xr;
  p.x_out = xo;
  p.a = a;
  p.w2 = static_cast<const uint8_t*>(P->w2);
  p.b2 = P->b2;
  p.mask = reinterpret_cast<uint8_t*>(mask);
  p.logits = logits;
  p.bar = bar;
  p.threshold = P->threshold;
  p.d = P->d_model;
  p.r = P->rank;
  p.F = P->d_ff;
  return launch(kern, dim3(G), dim3(kPredThreads), 0, st, p);
}

bool predict_fused_ok(int B, const pi_predictor* P) {
  if (B != 1 && B != 2) return false;
  const int cpt = pred_cpt(P->d_model), cpl = pred_cpl(P->rank);
  if (cpt == 0 || cpl == 0 || B * cpt > 4 || B * cpl > 8) return false;
  return (P->d_ff / 8 + num_sms() - 1) / num_sms() <= kPredMaxUnits &&
         (P->rank + num_sms() - 1) / num_sms() <= kPredMaxRows1;
}

template <int DT, int B, int CPT>
cudaError_t predict_cpl(const pi_predictor* P, const uint16_t* x, const float* xr, uint16_t* xo,
                        float* a, uint32_t* mask, float* logits, uint32_t* bar, cudaStream_t st) {
  switch (pred_cpl(P->rank)) {
    case 1: return launch_predict<DT, B, CPT, 1>(P, x, xr, xo, a, mask, logits, bar, st);
    case 2: return launch_predict<DT, B, CPT, 2>(P, x, xr, xo, a, mask, logits, bar, st);
    case 4: return launch_predict<DT, B, CPT, 4>(P, x, xr, xo, a, mask, logits, bar, st);
    case 8: if constexpr (B == 1) return launch_predict<DT, B, CPT, 8>(P, x, xr, xo, a, mask, logits, bar, st); break;
  }
  return cudaErrorInvalidValue;
}

template <int DT, int B>
cudaError_t predict_cpt(const pi_predictor* P, const uint16_t* x, const float* xr, uint16_t* xo,
                        float* a, uint32_t* mask, float* logits, uint32_t* bar, cudaStream_t st) {
  switch (pred_cpt(P->d_model)) {
    case 1: return predict_cpl<DT, B, 1>(P, x, xr, xo, a, mask, logits, bar, st);
    case 2: return predict_cpl<DT, B, 2>(P, x, xr, xo, a, mask, logits, bar, st);
    case 4: if constexpr (B == 1) return predict_cpl<DT, B, 4>(P, x, xr, xo, a, mask, logits, bar, st); break;
  }
  return cudaErrorInvalidValue;
}

// Predictor layer 2 on the tensor cores (batches of 16 or more, ranks that
// are a multiple of 64): a as hi + lo 16-bit parts from layer 1, the mask
// written whole by the kernel's ballots.
constexpr int kUmmaPredMinBatch = 16;

bool umma_pred_ok(int B, const pi_predictor* P) {
  return B >= kUmmaPredMinBatch && B <= 64 && P->rank % kUmmaK == 0 &&
         P->d_model % kUmmaK == 0 && tmap_encoder() != nullptr;
}

template <bool L1, int DT, int N>
cudaError_t launch_umma_pred_n(int rows, int S, const CUtensorMap& t0, const CUtensorMap& t1,
                               const UmmaPredParams& p, cudaStream_t st) {
  constexpr int STAGE = kUmmaM * kUmmaK * 2 + (L1 ? 1 : 2) * N * kUmmaK * 2;
  constexpr int NS = umma_ns(STAGE);
  return launch(k_umma_pred<L1, DT, N, NS>, dim3((rows + kUmmaM - 1) / kUmmaM, S),
                dim3(kUmmaThreads), (size_t)NS * STAGE + 1024, st, t0, t1, p);
}

template <bool L1, int DT>
cudaError_t umma_pred_n(int N, int rows, int S, const CUtensorMap& t0, const CUtensorMap& t1,
                        const UmmaPredParams& p, cudaStream_t st) {
  switch (N) {
    case 16: return launch_umma_pred_n<L1, DT, 16>(rows, S, t0, t1, p, st);
    case 32: return launch_umma_pred_n<L1, DT, 32>(rows, S, t0, t1, p, st);
    case 48: return launch_umma_pred_n<L1, DT, 48>(rows, S, t0, t1, p, st);
    default: return launch_umma_pred_n<L1, DT, 64>(rows, S, t0, t1, p, st);
  }
}

// Layer 1 (split over the contraction into `part`, then finished into the
// hi + lo parts of a) and layer 2 with the threshold.  part_bytes bounds the
// number of slices.
template <int DT>
cudaError_t umma_predict(const pi_predictor* P, int B, const uint16_t* x, uint16_t* ah,
                         uint16_t* al, float* part, size_t part_bytes, uint32_t* mask,
                         uint32_t* umask, float* logits, cudaStream_t st) {
  const int N = (B + 15) / 16 * 16, r = P->rank, d = P->d_model;
  CUtensorMap tx{}, th{}, tl{};
  if (!make_tmap16(&tx, x, d, B, (uint64_t)d * 2, kUmmaK, N) ||
      !make_tmap16(&th, ah, r, B, (uint64_t)r * 2, kUmmaK, N) ||
      !make_tmap16(&tl, al, r, B, (uint64_t)r * 2, kUmmaK, N))
    return cudaErrorInvalidValue;
  // layer 1: about two CTAs per SM, at least 8 stages each
  const int tiles1 = (r + kUmmaM - 1) / kUmmaM;
  int S = std::max(1, std::min((2 * num_sms()) / tiles1, (d / kUmmaK) / 8));
  S = (int)std::max<size_t>(1, std::min<size_t>(S, part_bytes / ((size_t)B * r * 4)));
  UmmaPredParams p1{};
  p1.w = static_cast<const uint8_t*>(P->w1);
  p1.part = part;
  p1.len = d;
  p1.nrows = r;
  p1.B = B;
  cudaError_t e = umma_pred_n<true, DT>(N, r, S, tx, tx, p1, st);
  if (e != cudaSuccess) return e;
  e = launch(k_pred1_finish<DT>, dim3((B * r + 255) / 256), dim3(256), 0, st, (const float*)part,
             S, B, r, P->b1, ah, al, (float*)nullptr);
  if (e != cudaSuccess) return e;
  UmmaPredParams p2{};
  p2.w = static_cast<const uint8_t*>(P->w2);
  p2.bias = P->b2;
  p2.mask = mask;
  p2.umask = umask;
  p2.logits = logits;
  p2.threshold = P->threshold;
  p2.len = r;
  p2.nrows = P->d_ff;
  p2.B = B;
  return umma_pred_n<false, DT>(N, P->d_ff, 1, th, tl, p2, st);
}

// x16: 16-bit input, or null with xr (residual) given; xo receives x_l then.
// bar: the workspace's grid-barrier words, zeroed by the API call beforehand.
// umask (optional): receives the OR of the batch's mask rows when the
// tensor-core layer 2 runs (returns whether it was written).
// part / part_bytes: scratch for the tensor-core layer 1's partial sums.
template <int DT>
int32_t predict_impl(const pi_predictor* P, int B, const uint16_t* x16, const float* xr,
                     uint16_t* xo, uint32_t* mask, float* logits, float* a, uint32_t* bar,
                     cudaStream_t st, float* part, size_t part_bytes,
                     uint32_t* umask = nullptr, bool* umask_written = nullptr) {
  if (umask_written) *umask_written = false;
  if (umma_pred_ok(B, P)) {
    // both layers on the tensor cores; a as 16-bit hi + lo parts in the
    // workspace's a region (which holds several copies of a)
    if (xr) {
      PI_CUDA((launch(k_cast_rms<DT>, dim3(B), dim3(256), 0, st, xr, xo, P->d_model)));
      x16 = xo;
    }
    uint16_t* ah = reinterpret_cast<uint16_t*>(a);
    uint16_t* al = ah + (size_t)B * P->rank;
    const cudaError_t e =
        umma_predict<DT>(P, B, x16, ah, al, part, part_bytes, mask, umask, logits, st);
    if (e != cudaSuccess)
      return fail(PI_ERR_CUDA, "tensor-core predictor launch failed: %s", cudaGetErrorString(e));
    if (umask_written) *umask_written = umask != nullptr;
    return PI_OK;
  }
  const int d = P->d_model;
  if (predict_fused_ok(B, P)) {
    const cudaError_t e = B == 1 ? predict_cpt<DT, 1>(P, x16, xr, xo, a, mask, logits, bar, st)
                                 : predict_cpt<DT, 2>(P, x16, xr, xo, a, mask, logits, bar, st);
    if (e != cudaSuccess) return fail(PI_ERR_CUDA, "predictor launch failed: %s", cudaGetErrorString(e));
    return PI_OK;
  }
  if (pred1_fused_ok(B, d)) {
    PI_CUDA((pred1_dispatch<DT>(P, B, x16, xr, xo, a, st)));
  } else {
    if (xr) {
      PI_CUDA((launch(k_cast_rms<DT>, dim3(B), dim3(256), 0, st, xr, xo, d)));
      x16 = xo;
    }
    RowsParams p{};
    p.w = static_cast<const uint8_t*>(P->w1);
    p.bias = P->b1;
    p.x16 = x16;
    p.out = a;
    p.nrows = P->rank;
    p.len = d;
    p.B = B;
    // batch 8-15: the r/16 row tiles leave most SMs idle, so the contraction
    // is also split (about two CTAs per SM), the raw sums go to the scratch
    // and k_pred1_finish adds them in slice order with b1 and the ReLU
    const int tiles = P->rank / 16;
    int Y = std::min(8, std::max(1, 2 * num_sms() / std::max(1, tiles)));
    Y = (int)std::min<size_t>((size_t)Y, part_bytes / ((size_t)B * P->rank * 4));
    if (B >= 8 && part && Y > 1) {
      p.part = part;
      PI_CUDA((launch_rows_mma<kModePred1, DT, 0>(p, P->rank, st, Y)));
      PI_CUDA((launch(k_pred1_finish<DT>, dim3((B * P->rank + 255) / 256), dim3(256), 0, st,
                      (const float*)part, Y, B, P->rank, P->b1, (uint16_t*)nullptr,
                      (uint16_t*)nullptr, a)));
    } else {
      PI_CUDA((rows_bb<DT, kModePred1>(p, P->rank, st)));
    }
  }
  if (pred2_fused_ok(B, P->rank)) {
    if (B == 1) PI_CUDA((pred2_cpl<DT, 1>(P, a, mask, logits, st)));
    else PI_CUDA((pred2_cpl<DT, 2>(P, a, mask, logits, st)));
  } else {
    // one CTA per mask word and 8 tokens; the rank in 4 (rank <= 1024) or 8
    // warp groups, so a lane's slice of a stays in registers
    Pred2WordsParams p{};
    p.w2 = static_cast<const uint8_t*>(P->w2);
    p.b2 = P->b2;
    p.a = a;
    p.mask = mask;
    p.logits = logits;
    p.threshold = P->threshold;
    p.F = P->d_ff;
    p.r = P->rank;
    p.B = B;
    // units of a mask word, or of half a word when that spreads them more
    // evenly over the two CTAs per SM; each CTA loops over its units
    const int slots = 2 * num_sms(), w32 = P->d_ff / 32, w16 = P->d_ff / 16;
    const double e32 = (double)w32 / (slots * ((w32 + slots - 1) / slots));
    const double e16 = (double)w16 / (slots * ((w16 + slots - 1) / slots));
    const bool half = e16 > e32 + 0.05;
    const dim3 grid(std::min(half ? w16 : w32, slots), (B + 7) / 8);
    if (P->rank <= 1024) {
      if (half) PI_CUDA((launch(k_pred2_words<DT, 4, 16>, grid, dim3(256), 0, st, p)));
      else PI_CUDA((launch(k_pred2_words<DT, 4, 32>, grid, dim3(256), 0, st, p)));
    } else {
      if (half) PI_CUDA((launch(k_pred2_words<DT, 8, 16>, grid, dim3(256), 0, st, p)));
      else PI_CUDA((launch(k_pred2_words<DT, 8, 32>, grid, dim3(256), 0, st, p)));
    }
  }
  return PI_OK;
}

// ------------------------------------------------------------ gathered FFN
int ffn_grid(int B) { return ffn_cps(B) * num_sms(); }

size_t ffn_row_bytes(const pi_layer* L) {
  return L->wdtype == PI_Q4_0 ? (size_t)L->d_model / 32 * 18 : (size_t)L->d_model * 2;
}


int ffn_list_cap(const pi_layer* L, int B) {
  return (L->d_ff + ffn_grid(B) - 1) / ffn_grid(B) + 1;
}

// 16-bit weights (k_ffn_ldg): down-phase column chunks per thread
int ldg_cpt(int d) {
  const int need = (d / 8 + kLdgThreads - 1) / kLdgThreads;
  for (int c : {1, 2, 4})
    if (c >= need) return c;
  return 0;
}

size_t ldg_smem(const pi_layer* L, int B) {
  return 256 + (size_t)ffn_list_cap(L, B) * (8 + 4 * B) + (size_t)L->d_ff / 4 + 16;
}

bool ffn_fused_ok(const pi_layer* L, int B) {
  if (!(B == 1 || B == 2 || B == 4)) return false;
  if (L->wdtype == PI_Q4_0) {
    // one 32-element block per thread (d <= 8192)
    if (L->d_model / 32 > kQ4Threads || B > 2) return false;
    return ldg_smem(L, B) <= kSmemFfn / ffn_cps(B);
  }
  const int c = ldg_cpt(L->d_model);
  if (c == 0 || B * c > 8) return false;
  return ldg_smem(L, B) <= kSmemFfn / ffn_cps(B);
}

struct FfnSrc {            // where the fused kernel takes its neuron list from
  const int32_t* idx;      // explicit list ...
  const int32_t* count;
  const uint32_t* mask;    // ... or the predictor's mask bits
  int mask_rows;
  int32_t* idx_out;        // mask mode: write the ascending list / count here
  int32_t* count_out;
  const pi_predictor* next;  // predictor the stream runs next (L2 prefetch), or null
};

FfnParams ffn_params(const pi_layer* L, int B, const uint16_t* x, const FfnSrc& src, float* part) {
  FfnParams p{};
  const bool reglu = L->act == PI_REGLU;
  p.w_act = static_cast<const uint8_t*>(reglu ? L->w_gate : L->w_up);
  p.w_up = static_cast<const uint8_t*>(L->w_up);
  p.w_dn = static_cast<const uint8_t*>(L->w_down_t);
  p.b_act = reglu ? L->b_gate : L->b_up;
  p.x = x;
  p.idx = src.idx;
  p.count = src.count;
  p.mask = src.mask;
  p.mask_rows = src.mask_rows;
  p.idx_out = src.idx_out;
  p.count_out = src.count_out;
  p.part = part;
  p.d = L->d_model;
  p.F = L->d_ff;
  p.row_bytes = (uint32_t)ffn_row_bytes(L);
  p.list_cap = ffn_list_cap(L, B);
  if (src.next) {
    const pi_predictor* N = src.next;
    p.pf_base[0] = static_cast<const uint8_t*>(N->w1);
    p.pf_bytes[0] = (size_t)N->rank * N->d_model * 2;
    p.pf_base[1] = static_cast<const uint8_t*>(N->w2);
    p.pf_bytes[1] = (size_t)N->d_ff * N->rank * 2;
  }
  return p;
}

template <int WDT, int ACT, int B, int CPT>
cudaError_t launch_ffn_ldg(const pi_layer* L, const uint16_t* x, const FfnSrc& src, float* part,
                           cudaStream_t st) {
  const FfnParams p = ffn_params(L, B, x, src, part);
  constexpr int CPS = B == 1 ? PI_LDG_CPS : 1;
  return launch(k_ffn_ldg<WDT, ACT, B, CPT, CPS>, dim3(ffn_grid(B)), dim3(kLdgThreads),
                ldg_smem(L, B), st, p);
}

template <int WDT, int ACT, int B>
cudaError_t ffn_ldg_cpt(const pi_layer* L, const uint16_t* x, const FfnSrc& src, float* part,
                        cudaStream_t st) {
  switch (ldg_cpt(L->d_model)) {
    case 1: return launch_ffn_ldg<WDT, ACT, B, 1>(L, x, src, part, st);
    case 2: return launch_ffn_ldg<WDT, ACT, B, 2>(L, x, src, part, st);
    case 4: if constexpr (B <= 2) return launch_ffn_ldg<WDT, ACT, B, 4>(L, x, src, part, st); break;
  }
  return cudaErrorInvalidValue;
}

template <int WDT, int ACT>
cudaError_t ffn_ldg(const pi_layer* L, int B, const uint16_t* x, const FfnSrc& src, float* part,
                    cudaStream_t st) {
  if (B == 1) return ffn_ldg_cpt<WDT, ACT, 1>(L, x, src, part, st);
  if (B == 2) return ffn_ldg_cpt<WDT, ACT, 2>(L, x, src, part, st);
  return ffn_ldg_cpt<WDT, ACT, 4>(L, x, src, part, st);
}

// Q4_0 weights: k_ffn_q4, block t of every row on thread t
template <int ACT>
cudaError_t ffn_q4(const pi_layer* L, int B, const uint16_t* x, const FfnSrc& src, float* part,
                   cudaStream_t st) {
  const FfnParams p = ffn_params(L, B, x, src, part);
  if (B == 1)
    return launch(k_ffn_q4<ACT, 1>, dim3(ffn_grid(1)), dim3(kQ4Threads), ldg_smem(L, 1), st, p);
  if (B == 2)
    return launch(k_ffn_q4<ACT, 2>, dim3(ffn_grid(2)), dim3(kQ4Threads), ldg_smem(L, 2), st, p);
  return cudaErrorInvalidValue;
}

template <int WDT, int ACT>
cudaError_t launch_up_generic(const pi_layer* L, int B, const uint16_t* x, const int32_t* idx,
                              const int32_t* count, float* h, cudaStream_t st) {
  RowsParams p{};
  p.w = static_cast<const uint8_t*>(ACT == 1 ? L->w_gate : L->w_up);
  p.w2nd = static_cast<const uint8_t*>(L->w_up);
  p.bias = ACT == 1 ? L->b_gate : L->b_up;
  p.x16 = x;
  p.idx = idx;
  p.count = count;
  p.out = h;
  p.nrows = L->d_ff;
  p.len = L->d_model;
  p.B = B;
  const int nsm = num_sms();
  if constexpr (WDT != 2)
    if (B >= 8) return launch_rows_mma<kModeUp, WDT, ACT>(p, L->d_ff, st);
  const int blocks = std::min((L->d_ff + 7) / 8, nsm * 8);
  if (B <= 8) return launch(k_rows<kModeUp, WDT, ACT, 8>, dim3(blocks), dim3(256), 0, st, p);
  if (B <= 32) return launch(k_rows<kModeUp, WDT, ACT, 32>, dim3(blocks), dim3(256), 0, st, p);
  return launch(k_rows<kModeUp, WDT, ACT, 64>, dim3(blocks), dim3(256), 0, st, p);
}

template <int WDT>
cudaError_t up_generic_act(const pi_layer* L, int B, const uint16_t* x, const int32_t* idx,
                           const int32_t* count, float* h, cudaStream_t st) {
  if (L->act == PI_REGLU) return launch_up_generic<WDT, 1>(L, B, x, idx, count, h, st);
  if (L->act == PI_SQRELU) return launch_up_generic<WDT, 2>(L, B, x, idx, count, h, st);
  return launch_up_generic<WDT, 0>(L, B, x, idx, count, h, st);
}

// The up projection (grid: p.ucap units or the tiles of all F neurons,
// whichever is more) and, when its contraction may be split, the kernel
// that completes split tiles.
template <int DT, int ACT, int N>
cudaError_t launch_umma_up_n(const pi_layer* L, const CUtensorMap& tx, const UmmaParams& p,
                             cudaStream_t st) {
  constexpr int NMAT = ACT == 1 ? 2 : 1;
  constexpr int STAGE = umma_up_stage<NMAT, N>();
  constexpr int NS = umma_ns(STAGE, DT == 2);
  const int tiles = (L->d_ff + kUmmaM - 1) / kUmmaM;
  cudaError_t e = launch(k_umma_up<DT, ACT, N, NS>, dim3(std::max(tiles, p.ucap)),
                         dim3(kUmmaThreads), (size_t)NS * STAGE + 1024, st, tx, p);
  if (e != cudaSuccess || p.ucap < 2) return e;
  return launch(k_umma_up_finish<DT, ACT>, dim3(2 * num_sms()), dim3(256), 0, st, p);
}

template <int DT, int N>
cudaError_t launch_umma_down_n(const pi_layer* L, int S, const CUtensorMap& th,
                               const CUtensorMap& tl, const UmmaParams& p, cudaStream_t st) {
  constexpr int STAGE = umma_down_stage<N>();
  constexpr int NS = umma_ns(STAGE, DT == 2);
  return launch(k_umma_down<DT, N, NS>, dim3(L->d_model / kUmmaM, S), dim3(kUmmaDownThreads),
                (size_t)NS * STAGE + 1024, st, th, tl, p);
}

template <int DT, int ACT>
cudaError_t umma_up_act(const pi_layer* L, int N, const CUtensorMap& tx, const UmmaParams& p,
                        cudaStream_t st) {
  switch (N) {
    case 16: return launch_umma_up_n<DT, ACT, 16>(L, tx, p, st);
    case 32: return launch_umma_up_n<DT, ACT, 32>(L, tx, p, st);
    case 48: return launch_umma_up_n<DT, ACT, 48>(L, tx, p, st);
    default: return launch_umma_up_n<DT, ACT, 64>(L, tx, p, st);
  }
}

// DT: 0 fp16, 1 bf16, 2 Q4_0 weights (pi_umma.cuh).
template <int DT>
cudaError_t umma_ffn(const pi_layer* L, int B, const uint16_t* x, const FfnSrc& src, uint16_t* hh,
                     uint16_t* hl, float* part, size_t part_bytes, int S, cudaStream_t st) {
  const int d = L->d_model, F = L->d_ff;
  const int N = (B + 15) / 16 * 16;
  const bool reglu = L->act == PI_REGLU;
  CUtensorMap tx{}, th{}, tl{};
  if (!make_tmap16(&tx, x, d, B, (uint64_t)d * 2, kUmmaK, N) ||
      !make_tmap16(&th, hh, F, B, (uint64_t)F * 2, kUmmaK, N) ||
      !make_tmap16(&tl, hl, F, B, (uint64_t)F * 2, kUmmaK, N))
    return cudaErrorInvalidValue;
  UmmaParams p{};
  p.idx = src.idx;
  p.count = src.count;
  p.mask = src.mask;
  p.mask_rows = src.mask_rows;
  p.idx_out = src.idx_out;
  p.count_out = src.count_out;
  p.wa = static_cast<const uint8_t*>(reglu ? L->w_gate : L->w_up);
  p.wa2 = static_cast<const uint8_t*>(L->w_up);
  p.wd = static_cast<const uint8_t*>(L->w_down_t);
  p.rb = (uint32_t)ffn_row_bytes(L);
  p.bias = reglu ? L->b_gate : L->b_up;
  p.hh = hh;
  p.hl = hl;
  p.part = part;
  // a split up projection keeps its slices' sums in the partial-sum scratch,
  // which the down projection overwrites only after they have been added
  const int nsm = num_sms();
  const size_t unit_bytes = (size_t)(reglu ? 2 : 1) * B * kUmmaM * 4;
  p.pu = part;
  p.slots = 2 * nsm;
  p.ucap = (int)std::min<size_t>((size_t)(4 * nsm), part_bytes / unit_bytes);
  p.d = d;
  p.F = F;
  p.B = B;
  cudaError_t e = L->act == PI_REGLU ? umma_up_act<DT, 1>(L, N, tx, p, st)
                : L->act == PI_SQRELU ? umma_up_act<DT, 2>(L, N, tx, p, st)
                                      : umma_up_act<DT, 0>(L, N, tx, p, st);
  if (e != cudaSuccess) return e;
  if (src.mask) {  // the down projection reads the list the up kernel wrote
    p.idx = src.idx_out;
    p.count = src.count_out;
  }
  switch (N) {
    case 16: return launch_umma_down_n<DT, 16>(L, S, th, tl, p, st);
    case 32: return launch_umma_down_n<DT, 32>(L, S, th, tl, p, st);
    case 48: return launch_umma_down_n<DT, 48>(L, S, th, tl, p, st);
    default: return launch_umma_down_n<DT, 64>(L, S, th, tl, p, st);
  }
}

// neuron slices of the tensor-core down projection: about two CTAs per SM
int umma_slices(int d, int B, int nsm) {
  const int tiles = d / kUmmaM;
  return std::max(1, std::min(down_slices(d, B, nsm), (2 * nsm) / tiles));
}

// Records a caller's timing event on the stream; under stream capture it
// becomes an external event-record node, so every graph launch records it.
cudaError_t record_event(void* ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  if (cs == cudaStreamCaptureStatusActive)
    return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(ev), st, cudaEventRecordExternal);
  return cudaEventRecord(static_cast<cudaEvent_t>(ev), st);
}

// The gathered FFN: mode 0 writes y = FFN(x), mode 1 adds FFN(x) into out.
// The neuron list is src.idx/src.count, or (fused path only) src.mask.
// ev (optional): two events recorded right before and after the FFN kernel(s).
int32_t ffn_impl(const pi_layer* L, int B, const uint16_t* x, const FfnSrc& src, float* out,
                 int mode, const WsLayout& w, uint8_t* ws, cudaStream_t st,
                 void* const* ev = nullptr) {
  float* part = reinterpret_cast<float*>(ws + w.part);
  const int d = L->d_model;
  const int n4 = B * d / 4;
  int G;
  if (ev) PI_CUDA(record_event(ev[0], st));
  if (ffn_fused_ok(L, B)) {
    cudaError_t e = cudaErrorInvalidValue;
    const int act = L->act;
    switch (L->wdtype) {
      case PI_F16:
        e = act == PI_REGLU ? ffn_ldg<0, 1>(L, B, x, src, part, st)
          : act == PI_SQRELU ? ffn_ldg<0, 2>(L, B, x, src, part, st)
                             : ffn_ldg<0, 0>(L, B, x, src, part, st);
        break;
      case PI_BF16:
        e = act == PI_REGLU ? ffn_ldg<1, 1>(L, B, x, src, part, st)
          : act == PI_SQRELU ? ffn_ldg<1, 2>(L, B, x, src, part, st)
                             : ffn_ldg<1, 0>(L, B, x, src, part, st);
        break;
      case PI_Q4_0:
        e = act == PI_REGLU ? ffn_q4<1>(L, B, x, src, part, st)
          : act == PI_SQRELU ? ffn_q4<2>(L, B, x, src, part, st)
                             : ffn_q4<0>(L, B, x, src, part, st);
        break;
    }
    if (e != cudaSuccess) return fail(PI_ERR_CUDA, "fused FFN launch failed: %s", cudaGetErrorString(e));
    G = ffn_grid(B);
  } else if (umma_ok(L, B)) {
    uint16_t* hh = reinterpret_cast<uint16_t*>(ws + w.h);
    uint16_t* hl = hh + (size_t)L->d_ff * B;
    G = umma_slices(d, B, num_sms());
    const size_t pb = w.h - w.part;
    const cudaError_t e =
        L->wdtype == PI_BF16  ? umma_ffn<1>(L, B, x, src, hh, hl, part, pb, G, st)
        : L->wdtype == PI_Q4_0 ? umma_ffn<2>(L, B, x, src, hh, hl, part, pb, G, st)
                               : umma_ffn<0>(L, B, x, src, hh, hl, part, pb, G, st);
    if (e != cudaSuccess)
      return fail(PI_ERR_CUDA, "tensor-core FFN launch failed: %s", cudaGetErrorString(e));
  } else {
    if (src.mask) return fail(PI_ERR_UNSUPPORTED, "mask-driven FFN needs the fused kernel");
    float* h = reinterpret_cast<float*>(ws + w.h);
    cudaError_t e = cudaErrorInvalidValue;
    switch (L->wdtype) {
      case PI_F16: e = up_generic_act<0>(L, B, x, src.idx, src.count, h, st); break;
      case PI_BF16: e = up_generic_act<1>(L, B, x, src.idx, src.count, h, st); break;
      case PI_Q4_0: e = up_generic_act<2>(L, B, x, src.idx, src.count, h, st); break;
    }
    if (e != cudaSuccess) return fail(PI_ERR_CUDA, "batched up launch failed: %s", cudaGetErrorString(e));
    DownParams dp{};
    dp.w_dn = static_cast<const uint8_t*>(L->w_down_t);
    dp.idx = src.idx;
    dp.count = src.count;
    dp.h = h;
    dp.part = part;
    dp.d = d;
    dp.F = L->d_ff;
    dp.B = B;
    G = down_slices(d, B, num_sms());
    if (L->wdtype != PI_Q4_0 && B % 4 == 0) {
      // one pass over the rows per 32 tokens: 64 / BB columns per thread
      const int BB = B <= 8 ? 8 : B <= 16 ? 16 : 32;
      const int units = d / (64 / BB);
      const int gx = (units + 255) / 256;
      G = std::max(1, std::min(G, 2 * num_sms() / gx));
      dim3 grid(gx, G);
      const bool bf = L->wdtype == PI_BF16;
      for (int b0 = 0; b0 < B && e == cudaSuccess; b0 += BB) {
        dp.b0 = b0;
        switch (BB) {
          case 8: e = bf ? launch(k_down2<1, 8>, grid, dim3(256), 0, st, dp) : launch(k_down2<0, 8>, grid, dim3(256), 0, st, dp); break;
          case 16: e = bf ? launch(k_down2<1, 16>, grid, dim3(256), 0, st, dp) : launch(k_down2<0, 16>, grid, dim3(256), 0, st, dp); break;
          default: e = bf ? launch(k_down2<1, 32>, grid, dim3(256), 0, st, dp) : launch(k_down2<0, 32>, grid, dim3(256), 0, st, dp); break;
        }
      }
    } else {
      dim3 grid((d / 8 + 255) / 256, G);
      switch (L->wdtype) {
        case PI_F16: e = launch(k_down<0>, grid, dim3(256), 0, st, dp); break;
        case PI_BF16: e = launch(k_down<1>, grid, dim3(256), 0, st, dp); break;
        default: e = launch(k_down<2>, grid, dim3(256), 0, st, dp); break;
      }
    }
    if (e != cudaSuccess) return fail(PI_ERR_CUDA, "batched down launch failed: %s", cudaGetErrorString(e));
  }
  if (ev) PI_CUDA(record_event(ev[1], st));
  if (G <= kReduceFew) {
    const dim3 rg((n4 + 255) / 256);
    if (mode == 0) PI_CUDA((launch(k_reduce_few<0>, rg, dim3(256), 0, st, (const float*)part, G, n4, out)));
    else PI_CUDA((launch(k_reduce_few<1>, rg, dim3(256), 0, st, (const float*)part, G, n4, out)));
    return PI_OK;
  }
  const dim3 rg((n4 + kRedCols - 1) / kRedCols);
  const dim3 rt(kRedCols * kRedSlices);
  if (mode == 0) PI_CUDA((launch(k_reduce<0>, rg, rt, 0, st, (const float*)part, G, n4, out)));
  else PI_CUDA((launch(k_reduce<1>, rg, rt, 0, st, (const float*)part, G, n4, out)));
  return PI_OK;
}

// One neuron-indexed tensor of a layer permuted into dst (see pi_permute_layer).
cudaError_t gather_rows(const void* src, void* dst, const int32_t* perm, int n, size_t row_bytes,
                        cudaStream_t st) {
  const int nsm = num_sms();
  if (row_bytes % 16 == 0) {
    const int units = (int)(row_bytes / 16);
    const long long total = (long long)n * units;
    const int blocks = (int)std::min<long long>((total + 255) / 256, 8ll * nsm);
    return launch(k_gather_rows<16>, dim3(blocks), dim3(256), 0, st,
                  static_cast<const uint8_t*>(src), static_cast<uint8_t*>(dst), perm, n, units);
  }
  const int units = (int)(row_bytes / 4);
  const long long total = (long long)n * units;
  const int blocks = (int)std::min<long long>((total + 255) / 256, 8ll * nsm);
  return launch(k_gather_rows<4>, dim3(blocks), dim3(256), 0, st,
                static_cast<const uint8_t*>(src), static_cast<uint8_t*>(dst), perm, n, units);
}

bool overlaps(const void* a, const void* b, size_t bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + bytes && y < x + bytes;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

const char* pi_status_string(int32_t s) {
  switch (s) {
    case PI_OK: return "success";
    case PI_ERR_INVALID_ARG: return "invalid argument";
    case PI_ERR_UNSUPPORTED: return "unsupported shape, dtype or batch";
    case PI_ERR_WORKSPACE: return "workspace missing or too small";
    case PI_ERR_CUDA: return "CUDA runtime error";
    default: return "unknown status";
  }
}

const char* pi_last_error(void) { return g_last_error.c_str(); }

uint64_t pi_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int32_t pi_device_error(int32_t* code_out) {
  if (!code_out) return fail(PI_ERR_INVALID_ARG, "code_out is NULL");
  PI_CUDA(cudaDeviceSynchronize());
  int v = 0;
  PI_CUDA(cudaMemcpyFromSymbol(&v, g_dev_error, sizeof v));
  const int zero = 0;
  PI_CUDA(cudaMemcpyToSymbol(g_dev_error, &zero, sizeof zero));
  *code_out = v;
  return PI_OK;
}

size_t pi_workspace_size(const pi_layer* layers, int32_t n_layers, int32_t batch) {
  if (!layers || n_layers < 1 || validate_batch(batch)) return 0;
  int d = 0, F = 0, r = 0;
  for (int l = 0; l < n_layers; ++l) {
    if (validate_layer(&layers[l])) return 0;
    d = std::max(d, layers[l].d_model);
    F = std::max(F, layers[l].d_ff);
    r = std::max(r, layers[l].pred.rank);
  }
  return ws_layout(d, F, r, batch).total;
}

int32_t pi_predict(const pi_predictor* pred, const void* x, int32_t batch, uint32_t* mask_bits,
                   float* logits, void* workspace, size_t workspace_bytes, void* stream) {
  if (int32_t s = validate_predictor(pred)) return s;
  if (int32_t s = validate_batch(batch)) return s;
  if (!x || !mask_bits) return fail(PI_ERR_INVALID_ARG, "x and mask_bits are required");
  if (!aligned16(x) || !aligned16(mask_bits) || (logits && !aligned16(logits)))
    return fail(PI_ERR_INVALID_ARG, "x, mask_bits and logits must be 16-byte aligned");
  const WsLayout w = ws_layout(pred->d_model, pred->d_ff, pred->rank, batch);
  if (int32_t s = check_ws(workspace, workspace_bytes, w.total)) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* a = reinterpret_cast<float*>(ws + w.a);
  float* part = reinterpret_cast<float*>(ws + w.part);
  uint32_t* bar = reinterpret_cast<uint32_t*>(ws + w.bar);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  PI_CUDA(cudaMemsetAsync(bar, 0, 8, st));
  const uint16_t* x16 = static_cast<const uint16_t*>(x);
  if (pred->dtype == PI_F16)
    return predict_impl<0>(pred, batch, x16, nullptr, nullptr, mask_bits, logits, a, bar, st, part,
                           w.h - w.part);
  return predict_impl<1>(pred, batch, x16, nullptr, nullptr, mask_bits, logits, a, bar, st, part,
                         w.h - w.part);
}

int32_t pi_compact(const uint32_t* mask_bits, int32_t batch, int32_t d_ff, int32_t* idx,
                   int32_t* count, void* workspace, size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (int32_t s = validate_batch(batch)) return s;
  if (d_ff < 32 || d_ff > 65536 || d_ff % 32)
    return fail(PI_ERR_UNSUPPORTED, "d_ff %d: need 32 <= d_ff <= 65536, multiple of 32", d_ff);
  if (!mask_bits || !idx || !count) return fail(PI_ERR_INVALID_ARG, "mask_bits, idx and count are required");
  if (!aligned16(mask_bits) || !aligned16(idx) || (reinterpret_cast<uintptr_t>(count) & 3u))
    return fail(PI_ERR_INVALID_ARG, "mask_bits and idx must be 16-byte aligned, count 4-byte aligned");
  PI_CUDA((launch(k_compact, dim3(1), dim3(kCompactThreads), 0, static_cast<cudaStream_t>(stream),
                  mask_bits, (int)batch, (int)d_ff, idx, count)));
  return PI_OK;
}

int32_t pi_sparse_ffn(const pi_layer* layer, const void* x, int32_t batch, const int32_t* idx,
                      const int32_t* count, float* y, void* workspace, size_t workspace_bytes,
                      void* stream) {
  if (int32_t s = validate_layer(layer)) return s;
  if (int32_t s = validate_batch(batch)) return s;
  if (!x || !idx || !count || !y) return fail(PI_ERR_INVALID_ARG, "x, idx, count and y are required");
  if (!aligned16(x) || !aligned16(idx) || !aligned16(y) || (reinterpret_cast<uintptr_t>(count) & 3u))
    return fail(PI_ERR_INVALID_ARG, "x, idx and y must be 16-byte aligned, count 4-byte aligned");
  const WsLayout w = ws_layout(layer->d_model, layer->d_ff, layer->pred.rank, batch);
  if (int32_t s = check_ws(workspace, workspace_bytes, w.total)) return s;
  FfnSrc src{idx, count, nullptr, 0, nullptr, nullptr};
  return ffn_impl(layer, batch, static_cast<const uint16_t*>(x), src, y, 0, w,
                  static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream));
}

int32_t pi_ffn_stack(const pi_layer* layers, int32_t n_layers, float* x_resid, int32_t batch,
                     int32_t* idx_out, int32_t* count_out, void* workspace, size_t workspace_bytes,
                     void* stream) {
  return pi_ffn_stack_timed(layers, n_layers, x_resid, batch, idx_out, count_out, workspace,
                            workspace_bytes, stream, nullptr);
}

int32_t pi_ffn_stack_timed(const pi_layer* layers, int32_t n_layers, float* x_resid,
                           int32_t batch, int32_t* idx_out, int32_t* count_out, void* workspace,
                           size_t workspace_bytes, void* stream, void* const* ffn_events) {
  if (!layers || n_layers < 1) return fail(PI_ERR_INVALID_ARG, "need at least one layer");
  if (int32_t s = validate_batch(batch)) return s;
  if (!x_resid || !aligned16(x_resid)) return fail(PI_ERR_INVALID_ARG, "x_resid must be a 16-byte aligned pointer");
  if ((idx_out && !aligned16(idx_out)) || (count_out && (reinterpret_cast<uintptr_t>(count_out) & 3u)))
    return fail(PI_ERR_INVALID_ARG, "idx_out must be 16-byte aligned, count_out 4-byte aligned");
  int d = 0, F = 0, r = 0;
  for (int l = 0; l < n_layers; ++l) {
    if (int32_t s = validate_layer(&layers[l])) return s;
    if (layers[l].d_model != layers[0].d_model || layers[l].adtype != layers[0].adtype)
      return fail(PI_ERR_INVALID_ARG, "all layers of a stack need the same d_model and adtype");
    if (idx_out && layers[l].d_ff != layers[0].d_ff)
      return fail(PI_ERR_INVALID_ARG, "idx_out needs the same d_ff in every layer");
    d = std::max(d, layers[l].d_model);
    F = std::max(F, layers[l].d_ff);
    r = std::max(r, layers[l].pred.rank);
  }
  const WsLayout w = ws_layout(d, F, r, batch);
  if (int32_t s = check_ws(workspace, workspace_bytes, w.total)) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint16_t* xl = reinterpret_cast<uint16_t*>(ws + w.xl);
  float* a = reinterpret_cast<float*>(ws + w.a);
  uint32_t* mask = reinterpret_cast<uint32_t*>(ws + w.mask);
  uint32_t* bar = reinterpret_cast<uint32_t*>(ws + w.bar);
  PI_CUDA(cudaMemsetAsync(bar, 0, 8, st));
  for (int l = 0; l < n_layers; ++l) {
    const pi_layer* L = &layers[l];
    int32_t* idx = idx_out ? idx_out + (size_t)l * L->d_ff : reinterpret_cast<int32_t*>(ws + w.idx);
    int32_t* cnt = count_out ? count_out + l : reinterpret_cast<int32_t*>(ws + w.count);
    uint32_t* umask = reinterpret_cast<uint32_t*>(ws + w.umask);
    bool have_union = false;
    float* part = reinterpret_cast<float*>(ws + w.part);
    int32_t s = (L->adtype == PI_F16)
                    ? predict_impl<0>(&L->pred, batch, nullptr, x_resid, xl, mask, nullptr, a, bar,
                                      st, part, w.h - w.part, umask, &have_union)
                    : predict_impl<1>(&L->pred, batch, nullptr, x_resid, xl, mask, nullptr, a, bar,
                                      st, part, w.h - w.part, umask, &have_union);
    if (s) return s;
    if (ffn_events && (!ffn_events[2 * l] || !ffn_events[2 * l + 1]))
      return fail(PI_ERR_INVALID_ARG, "ffn_events[%d..%d] must be events", 2 * l, 2 * l + 1);
    FfnSrc src{idx, cnt, nullptr, 0, nullptr, nullptr};
    if (ffn_fused_ok(L, batch)) {
      // compaction fused into the FFN kernel: it reads the mask bits directly
      src = FfnSrc{nullptr, nullptr, mask, (int)batch, idx_out ? idx : nullptr,
                   count_out ? cnt : nullptr, &layers[(l + 1) % n_layers].pred};
    } else if (umma_ok(L, batch)) {
      // compaction fused into the tensor-core up kernel: every CTA scans the
      // union (ORed by the predictor, or the batch's mask rows) for its tile
      src = FfnSrc{nullptr, nullptr, have_union ? umask : mask, have_union ? 1 : (int)batch, idx,
                   cnt, nullptr};
    } else {
      PI_CUDA((launch(k_compact, dim3(1), dim3(kCompactThreads), 0, st, (const uint32_t*)mask,
                      (int)batch, L->d_ff, idx, cnt)));
    }
    if ((s = ffn_impl(L, batch, xl, src, x_resid, 1, w, ws, st,
                      ffn_events ? ffn_events + 2 * l : nullptr)))
      return s;
  }
  return PI_OK;
}

// Callers that cannot allocate -- a host framework whose allocator owns the
// whole device, a latency-bound loop in which an allocation (which may wait
// for the device) is not allowed, or code that only holds weights and
// activations -- get the gathered FFN without supplying a workspace.
// The scratch lives in g_static_scratch; its address is looked up at set-up
// (the first call on a device, which must come before any stream capture) and
// refreshed on every uncaptured call.  Nothing in the scratch has to start at zero: every CTA writes its
// whole partial plane, and h is written for every listed neuron before it is
// read.  Calls whose work overlaps on one device race on the scratch.
int32_t pi_sparse_ffn_static(const pi_layer* layer, const void* x, int32_t batch,
                             const int32_t* idx, const int32_t* count, float* y, void* stream) {
  if (int32_t s = validate_layer(layer)) return s;
  if (int32_t s = validate_batch(batch)) return s;
  if (!x || !idx || !count || !y) return fail(PI_ERR_INVALID_ARG, "x, idx, count and y are required");
  if (!aligned16(x) || !aligned16(idx) || !aligned16(y) || (reinterpret_cast<uintptr_t>(count) & 3u))
    return fail(PI_ERR_INVALID_ARG, "x, idx and y must be 16-byte aligned, count 4-byte aligned");
  // the same scratch ffn_impl uses, packed from offset 0: partials, then h
  const int d = layer->d_model;
  const bool fused = ffn_fused_ok(layer, batch);
  const int G = fused ? ffn_grid(batch) : down_slices(d, batch, num_sms());
  WsLayout w{};
  w.part = 0;
  w.h = al256((size_t)G * batch * d * 4);
  w.total = fused ? w.h : w.h + al256((size_t)layer->d_ff * batch * 4);
  if (w.total > (size_t)PI_STATIC_SCRATCH_BYTES)
    return fail(PI_ERR_WORKSPACE,
                "pi_sparse_ffn_static: this shape needs %zu bytes of scratch, the fixed scratch "
                "holds %zu; use pi_sparse_ffn with a workspace",
                w.total, (size_t)PI_STATIC_SCRATCH_BYTES);
  int dev = 0;
  PI_CUDA(cudaGetDevice(&dev));
  constexpr int kMaxDevices = 64;
  if (dev < 0 || dev >= kMaxDevices)
    return fail(PI_ERR_UNSUPPORTED, "device ordinal %d: the fixed scratch supports 0..%d", dev,
                kMaxDevices - 1);
  // The address is looked up with this device current: at set-up (the first
  // call on the device), and again on every call made outside stream capture,
  // so a device reset (which reloads the module at another address) cannot
  // leave a stale pointer behind.  Under capture the set-up value is used.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  PI_CUDA(cudaStreamIsCapturing(st, &cs));
  static std::mutex mu;
  static uint8_t* base[kMaxDevices] = {};
  uint8_t* ws = nullptr;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (cs == cudaStreamCaptureStatusNone || !base[dev]) {
      if (cs != cudaStreamCaptureStatusNone)
        return fail(PI_ERR_INVALID_ARG,
                    "pi_sparse_ffn_static: the first call on a device must not be captured");
      void* ptr = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
      if (e != cudaSuccess)
        return fail(PI_ERR_CUDA, "cudaGetSymbolAddress(fixed scratch) failed: %s",
                    cudaGetErrorString(e));
      base[dev] = static_cast<uint8_t*>(ptr);
    }
    ws = base[dev];
  }
  FfnSrc src{idx, count, nullptr, 0, nullptr, nullptr};
  return ffn_impl(layer, batch, static_cast<const uint16_t*>(x), src, y, 0, w, ws, st);
}

// Hot-row ordering: the layer with its neurons renumbered (dst neuron i =
// src neuron perm[i]).  Every neuron-indexed tensor is gathered row by row
// into the caller's dst buffers; W1, b1 and the threshold are not touched.
int32_t pi_permute_layer(const pi_layer* src, const int32_t* perm, const pi_layer* dst,
                         void* stream) {
  if (int32_t s = validate_layer(src)) return s;
  if (int32_t s = validate_layer(dst)) return s;
  if (!perm || !aligned16(perm)) return fail(PI_ERR_INVALID_ARG, "perm must be a 16-byte aligned device pointer");
  if (src->d_model != dst->d_model || src->d_ff != dst->d_ff || src->wdtype != dst->wdtype ||
      src->adtype != dst->adtype || src->act != dst->act || src->pred.rank != dst->pred.rank)
    return fail(PI_ERR_INVALID_ARG, "src and dst must have the same shapes, dtypes and activation");
  if ((src->b_up == nullptr) != (dst->b_up == nullptr) ||
      (src->b_gate == nullptr) != (dst->b_gate == nullptr))
    return fail(PI_ERR_INVALID_ARG, "src and dst must both have, or both lack, each bias");
  const int F = src->d_ff;
  const size_t rb = ffn_row_bytes(src);
  const size_t rb2 = (size_t)src->pred.rank * 2;
  struct T { const void* s; void* d; size_t row; };
  const T ts[] = {
      {src->w_up, const_cast<void*>(dst->w_up), rb},
      {src->w_gate, const_cast<void*>(dst->w_gate), rb},
      {src->w_down_t, const_cast<void*>(dst->w_down_t), rb},
      {src->pred.w2, const_cast<void*>(dst->pred.w2), rb2},
      {src->pred.b2, const_cast<float*>(dst->pred.b2), 4},
      {src->b_up, const_cast<float*>(dst->b_up), 4},
      {src->b_gate, const_cast<float*>(dst->b_gate), 4},
  };
  for (const T& t : ts)
    if (t.s && (t.d == t.s || overlaps(t.s, t.d, t.row * F)))
      return fail(PI_ERR_INVALID_ARG, "a permuted dst tensor overlaps its src tensor");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (const T& t : ts)
    if (t.s) PI_CUDA(gather_rows(t.s, t.d, perm, F, t.row, st));
  return PI_OK;
}

}  // extern "C"
