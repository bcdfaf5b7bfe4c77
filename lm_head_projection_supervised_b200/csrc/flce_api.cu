// C ABI of libflce.so: argument validation, workspace carving, TMA tensor
// maps and the launch sequence of the forward and backward passes.
//
// Forward  (one stream, no host synchronisation):
//   compact -> gather H_c -> gemm<fwd> (Z tiles + online (m, s) + target)
//   -> merge partials per row -> fixed-order loss reduction
// Backward, with P vocabulary panels of Vc columns and three panel buffers:
//   compact -> gather H_c (skipped when reusing the forward's) ->
//   for L = 0 .. P:   gemm<bwd> with
//                       grad units of panel L     (if L < P) -> buffer L % 3
//                         (+ the bias gradient's fixed-point column sums)
//                       dW, dH units of panel L-1 (if L > 0) <- buffer (L-1) % 3
//                     launches L >= 1 may start while launch L-1 runs
//                     (programmatic dependent launch): their set-up overlaps
//                     its tail, their dW / dH units wait for it; the third
//                     panel buffer keeps a gradient unit from overwriting a
//                     panel the previous launch may still read
//   -> db from the column sums (bias only)
//   -> rows grouped by label (stable radix sort, own kernels) -> dW target
//      terms in fp32
//   -> scatter dH_c to dH with its target terms (zero rows for unsupervised
//      positions)
//   with row scales s_k = S r_k computed first (row_scale_kernel); the panels
//   hold r_k (p - onehot) sigma and the dW / dH epilogues multiply by S / sigma.
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/flce.h"
#include "../../include/flce_diag.h"
#include "aux_kernels.cuh"
#include "gemm.cuh"
#include "fused_bwd.cuh"

using namespace flce;

namespace {

constexpr int64_t kMaxN = int64_t(1) << 24;
constexpr int64_t kMaxD = int64_t(1) << 16;
constexpr int64_t kMaxV = int64_t(1) << 24;
constexpr int kMaxShards = 4096;  // vocabulary slices merged by one combine
#ifndef FLCE_PANEL_COLS
#define FLCE_PANEL_COLS 8192
#endif
constexpr int64_t kPanelCols = FLCE_PANEL_COLS;  // vocabulary columns per gradient panel
constexpr float kFp16Log2Sigma = 15.f;  // fp16 panels hold (p - onehot) * 2^15
#ifndef FLCE_POLY_EXP_MAX_D
#define FLCE_POLY_EXP_MAX_D 256
#endif
// Up to this hidden size the forward epilogue, not the tensor core, bounds
// the score tiles: one exponential in four then goes to the FMA pipe
// (ex2_poly).  Measured: 6 % off the forward at D = 64 .. 256, nothing in the
// gradient epilogue (which is not bound by the exponentials), a loss at 512.
constexpr int64_t kPolyExpMaxD = FLCE_POLY_EXP_MAX_D;
constexpr size_t kCounterOffset = 64;   // work counters follow the error word

int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t roundup64(int64_t a, int64_t b) { return cdiv64(a, b) * b; }

constexpr int kPanelBufs = 3;  // panel buffers: written, read, and one of slack for the overlap

struct Layout {
  size_t ctrl, ctrl_bytes, C, idx, yc, hc, part, tgt, loss_rows, fwd_total;
  size_t pos, rs, resid, skeys[2], svals[2], rscount, dbacc, keep, keep_bytes, dhc, twin;
  size_t gpanel[kPanelBufs], dwp, dhp, total;
  int64_t Np, nvt, vc, gld, panels;
  bool fused;   // the single-kernel backward applies (D <= 64)
  int64_t Vp;   // its dW partials: FB_NG_MAX slabs of Vp rows
};


// Workspace carve-up.  The control block (error word, then one work counter
// per GEMM launch) sits at offset 0 for every size.  The regions the forward
// pass uses come first (fwd_total bytes); the backward's follow.
Layout make_layout(int64_t N, int64_t D, int64_t V) {
  Layout L{};
  L.Np = roundup64(N > 0 ? N : 1, PAIR_M);  // every half-tile of a CTA pair starts inside
  L.nvt = cdiv64(V, BN);  // forward (m, s) partials per row: one per vocabulary tile
  L.vc = roundup64(V, BN) < kPanelCols ? roundup64(V, BN) : kPanelCols;
  L.panels = cdiv64(V, L.vc);
  L.gld = L.vc;  // gradient-panel row pitch in elements
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += static_cast<size_t>(roundup64(static_cast<int64_t>(bytes), 1024));
    return o;
  };
  L.ctrl_bytes = kCounterOffset + 4 * static_cast<size_t>(L.panels + 2);
  L.ctrl = take(L.ctrl_bytes);
  L.C = take(256);
  L.idx = take(static_cast<size_t>(L.Np) * 4);
  L.yc = take(static_cast<size_t>(L.Np) * 4);
  L.hc = take(static_cast<size_t>(L.Np) * D * 2);
  L.part = take(static_cast<size_t>(L.Np) * L.nvt * 8);  // tile-major [nvt][Np]
  L.tgt = take(static_cast<size_t>(L.Np) * 4);
  L.loss_rows = take(static_cast<size_t>(L.Np) * 4);
  L.pos = take(static_cast<size_t>(L.Np) * 4);
  L.fwd_total = off;
  L.rs = take(static_cast<size_t>(L.Np) * 4);
  L.resid = take(static_cast<size_t>(L.Np) * 4);
  // rows grouped by label (stable radix sort: ping-pong buffers, digit counts per tile)
  for (int i = 0; i < 2; ++i) {
    L.skeys[i] = take(static_cast<size_t>(L.Np) * 4);
    L.svals[i] = take(static_cast<size_t>(L.Np) * 4);
  }
  L.rscount = take(static_cast<size_t>(RS_DIGITS) * cdiv64(L.Np, RS_TILE) * 4);
  L.dbacc = take(static_cast<size_t>(V) * 8);  // bias gradient, fixed point per vocabulary id
  L.dhc = take(static_cast<size_t>(L.Np) * D * 4);
  // dW target terms: two partial sums per window of TW label-sorted rows
  L.twin = take(static_cast<size_t>(cdiv64(L.Np, TW)) * 2 * D * 4);
  // What follows is used by one of the two backward forms only: the panel
  // backward's flags and panels, or the single-kernel backward's partials.
  const size_t shared_base = off;
  // gradient filtering: one keep flag per 128-row x 64-column box of each panel buffer
  L.keep_bytes = static_cast<size_t>(L.Np / BM) * static_cast<size_t>(L.gld / 64);
  L.keep = take(L.keep_bytes * kPanelBufs);
  for (int i = 0; i < kPanelBufs; ++i) L.gpanel[i] = take(static_cast<size_t>(L.Np) * L.gld * 2);
  const size_t panel_end = off;
  L.Vp = roundup64(V, FB_COLS);
  // (the partials' TMA coordinates are 32-bit)
  L.fused = D <= FB_MAX_D && FB_NG_MAX * L.Vp < (int64_t(1) << 31) &&
            FB_NCH_MAX * L.Np < (int64_t(1) << 31);
  if (L.fused) {
    off = shared_base;
    L.dwp = take(static_cast<size_t>(FB_NG_MAX * L.Vp * D) * 4);
    L.dhp = take(static_cast<size_t>(FB_NCH_MAX) * static_cast<size_t>(L.Np) * D * 4);
    if (off < panel_end) off = panel_end;
  }
  L.total = off;
  return L;
}

// Workspace of flce_shard_combine: error word, C, idx [N], per-row losses [N].
struct CombineLayout {
  size_t C, idx, loss_rows, total;
};

CombineLayout combine_layout(int64_t N) {
  CombineLayout L{};
  const size_t n = static_cast<size_t>(roundup64(N > 0 ? N : 1, 64)) * 4;
  L.C = 256;
  L.idx = 512;
  L.loss_rows = L.idx + n;
  L.total = L.loss_rows + n;
  return L;
}

bool shape_ok(int64_t N, int64_t D, int64_t V) {
  return N >= 0 && N <= kMaxN && D >= 8 && D <= kMaxD && V >= 1 && V <= kMaxV;
}
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---- driver entry point for tensor-map encoding (no link against libcuda)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

enum MapType { kMapBF16, kMapFP16, kMapF32 };

// 2-D map over a row-major matrix [outer x inner] with row pitch `pitch`
// bytes, 128-byte swizzle, zero fill outside the extents.
bool make_map(CUtensorMap* m, const void* base, MapType t, uint64_t inner, uint64_t outer,
              uint64_t pitch, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t es[2] = {1, 1};
  const CUtensorMapDataType dt = t == kMapBF16   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : t == kMapFP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- the GEMM kernel's instantiations: one per mode and combination of the
// optional features that mode can use (bias, rounding of the logits, and the
// forward's polynomial exponentials or the backward's gradient filtering)
using GemmKernel = void (*)(GemmArgs);
// (at D <= kPolyExpMaxD the forward takes the polynomial exponentials and four
// epilogue warpgroups together)
constexpr int kFeatSmallD = kFeatPolyExp | kFeatWide;
using FwdFeats = std::integer_sequence<int, 0, kFeatBias, kFeatSmallD, kFeatBias | kFeatSmallD,
                                       kFeatRound, kFeatRound | kFeatBias,
                                       kFeatRound | kFeatSmallD,
                                       kFeatRound | kFeatBias | kFeatSmallD>;
using BwdFeats = std::integer_sequence<int, 0, kFeatBias, kFeatFilter, kFeatBias | kFeatFilter,
                                       kFeatRound, kFeatRound | kFeatBias,
                                       kFeatRound | kFeatFilter,
                                       kFeatRound | kFeatBias | kFeatFilter>;
using PlainFeats = std::integer_sequence<int, 0>;

// an instantiation with its launch shape
struct GemmKernelInfo {
  GemmKernel fn;
  int threads;
  size_t smem;
};
template <int MODE, int... F>
GemmKernelInfo pick_kernel(int feat, std::integer_sequence<int, F...>) {
  GemmKernelInfo k{nullptr, 0, 0};
  ((feat == F ? (k = GemmKernelInfo{flce_gemm_kernel<MODE, F>, Shape<MODE, F>::THREADS,
                                    Shape<MODE, F>::Cfg::SMEM_BYTES},
                 0)
              : 0),
   ...);
  return k;
}
template <int MODE>
GemmKernelInfo gemm_kernel(int feat) {
  if constexpr (MODE == kModeFwd) return pick_kernel<MODE>(feat, FwdFeats{});
  else if constexpr (MODE == kModeBwd) return pick_kernel<MODE>(feat, BwdFeats{});
  else return pick_kernel<MODE>(feat, PlainFeats{});
}
template <int MODE, int... F, class Fn>
void each_kernel(std::integer_sequence<int, F...>, Fn&& fn) {
  (fn(reinterpret_cast<const void*>(flce_gemm_kernel<MODE, F>),
      Shape<MODE, F>::Cfg::SMEM_BYTES, Shape<MODE, F>::REGS_AT_LAUNCH),
   ...);
}
// the single-kernel backward: bias and rounding of the logits
using FusedFeats = std::integer_sequence<int, 0, kFeatBias, kFeatRound, kFeatBias | kFeatRound>;
using FusedKernel = void (*)(FusedArgs);
template <int... F>
FusedKernel pick_fused(int feat, std::integer_sequence<int, F...>) {
  FusedKernel k = nullptr;
  ((feat == F ? (k = flce_fused_bwd_kernel<F>, 0) : 0), ...);
  return k;
}
template <int... F, class Fn>
void each_fused(std::integer_sequence<int, F...>, Fn&& fn) {
  (fn(reinterpret_cast<const void*>(flce_fused_bwd_kernel<F>), FB_SMEM_BYTES, FB_REGS_AT_LAUNCH),
   ...);
}

// ---- per-device set-up
struct DevInfo {
  bool init = false;
  bool ok = false;
  int sms = 0;
  int pairs = 0;  // CTA pairs of the GEMM kernel that fit on the device at once
};
std::mutex g_mu;
DevInfo g_dev[64];

flce_status device_setup(DevInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FLCE_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FLCE_ERR_CUDA;
    d.ok = (major == 10 && minor == 0) && encode_fn() != nullptr;
    if (d.ok) {
      bool fail = false;
      auto setup = [&](const void* fn, size_t smem, uint32_t regs_needed) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess) {
          fail = true;
          return;
        }
        // The GEMM kernels split registers between warpgroups with setmaxnreg;
        // the split only fits if the block was launched with enough of them.
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) fail = true;
        else if (fa.numRegs < static_cast<int>(regs_needed)) d.ok = false;
      };
      each_kernel<kModeFwd>(FwdFeats{}, setup);
      each_kernel<kModeBwd>(BwdFeats{}, setup);
      each_kernel<kModePlain>(PlainFeats{}, setup);
      each_fused(FusedFeats{}, setup);
      if (fail) return FLCE_ERR_CUDA;
    }
    if (d.ok) {
      // how many CTA pairs can be resident together (one CTA per SM)
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1));
      cfg.blockDim = dim3(NUM_THREADS);
      cfg.dynamicSmemBytes = GEMM_SMEM_BYTES;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, flce_gemm_kernel<kModeBwd>, &cfg) !=
              cudaSuccess ||
          clusters < 1)
        return FLCE_ERR_CUDA;
      d.pairs = clusters;
    }
    d.sms = sms;
    d.init = true;
  }
  *out = d;
  return d.ok ? FLCE_OK : FLCE_ERR_DEVICE;
}

#define FLCE_CK(expr)                               \
  do {                                              \
    if ((expr) != cudaSuccess) return FLCE_ERR_CUDA; \
  } while (0)

// ---- optional per-launch timing (diagnostic; off unless profile_begin)
struct ProfRec {
  int kind;
  int launches;  // kernels between the two events
  cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;

enum ProfKind : int { kProfFwd = 0, kProfBwd = 1, kProfPlain = 2, kProfAux = 3 };

// Runs `launch` (which enqueues one kernel on s); when profiling is on, the
// launch is bracketed by two events on the same stream.
template <class F>
cudaError_t timed_launch(int kind, cudaStream_t s, F&& launch) {
  bool on;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    on = g_prof_on;
  }
  if (!on) {
    launch();
    return cudaGetLastError();
  }
  ProfRec r{kind, 1, nullptr, nullptr};
  if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess)
    return cudaErrorUnknown;
  cudaEventRecord(r.start, s);
  launch();
  const cudaError_t e = cudaGetLastError();
  cudaEventRecord(r.stop, s);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof.push_back(r);
  return e;
}

// A timed span of several launches that overlap one another (the backward's
// chain of GEMM launches): one event before the first and one after the last,
// none in between.  begin returns false when profiling is off.
bool prof_span_begin(ProfRec* r, int kind, cudaStream_t s) {
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_prof_on) return false;
  }
  *r = ProfRec{kind, 0, nullptr, nullptr};
  if (cudaEventCreate(&r->start) != cudaSuccess || cudaEventCreate(&r->stop) != cudaSuccess)
    return false;
  cudaEventRecord(r->start, s);
  return true;
}
void prof_span_end(ProfRec* r, int launches, cudaStream_t s) {
  r->launches = launches;
  cudaEventRecord(r->stop, s);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof.push_back(*r);
}

// Persistent launch of CTA pairs: min(work units, resident pairs) clusters of 2.
// pdl: the launch may start before the previous kernel of the stream ends
// (programmatic stream serialisation; the kernel waits where it must).
// timed: wrap the launch in profiling events (off inside a timed span).
template <int MODE>
cudaError_t launch_gemm(const GemmArgs& a, int feat, int64_t units_upper, int pairs,
                        cudaStream_t s, bool pdl = false, bool timed = true) {
  const GemmKernelInfo kernel = gemm_kernel<MODE>(feat);
  if (kernel.fn == nullptr) return cudaErrorInvalidValue;
  if (units_upper <= 0) return cudaSuccess;
  const int npairs = static_cast<int>(units_upper < pairs ? units_upper : pairs);
  const int kind = MODE == kModeFwd ? kProfFwd : MODE == kModeBwd ? kProfBwd : kProfPlain;
  auto launch = [&] {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * npairs));
    cfg.blockDim = dim3(static_cast<unsigned>(kernel.threads));
    cfg.dynamicSmemBytes = kernel.smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    cudaLaunchKernelEx(&cfg, kernel.fn, a);
  };
  if (!timed) {
    launch();
    return cudaGetLastError();
  }
  return timed_launch(kind, s, launch);
}

struct WsPtrs {
  uint32_t* err;
  int* counters;
  int* C;
  float* scal;  // backward: S = max_k |s_k|
  int* idx;
  int* yc;
  int* pos;
  uint16_t* hc;
  float2* part;
  float* tgt;
  float* loss_rows;
  float* rs;
  float* resid;
  uint32_t* skeys[2];
  int* svals[2];
  int* rscount;
  unsigned long long* dbacc;
  uint8_t* keep;
  float* dhc;
  float* twin;
  uint16_t* gpanel[kPanelBufs];
  float* dwp;  // single-kernel backward: dW partials [FB_NG_MAX][Vp][D]
  float* dhp;  //   and dH partials [FB_NCH_MAX][Np][D]
};

WsPtrs carve(void* ws, const Layout& L) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  WsPtrs p;
  p.err = reinterpret_cast<uint32_t*>(w + L.ctrl);
  p.counters = reinterpret_cast<int*>(w + L.ctrl + kCounterOffset);
  p.C = reinterpret_cast<int*>(w + L.C);
  p.scal = reinterpret_cast<float*>(w + L.C + 64);
  p.idx = reinterpret_cast<int*>(w + L.idx);
  p.yc = reinterpret_cast<int*>(w + L.yc);
  p.pos = reinterpret_cast<int*>(w + L.pos);
  p.hc = reinterpret_cast<uint16_t*>(w + L.hc);
  p.part = reinterpret_cast<float2*>(w + L.part);
  p.tgt = reinterpret_cast<float*>(w + L.tgt);
  p.loss_rows = reinterpret_cast<float*>(w + L.loss_rows);
  p.rs = reinterpret_cast<float*>(w + L.rs);
  p.resid = reinterpret_cast<float*>(w + L.resid);
  for (int i = 0; i < 2; ++i) {
    p.skeys[i] = reinterpret_cast<uint32_t*>(w + L.skeys[i]);
    p.svals[i] = reinterpret_cast<int*>(w + L.svals[i]);
  }
  p.rscount = reinterpret_cast<int*>(w + L.rscount);
  p.dbacc = reinterpret_cast<unsigned long long*>(w + L.dbacc);
  p.keep = w + L.keep;
  p.dhc = reinterpret_cast<float*>(w + L.dhc);
  p.twin = reinterpret_cast<float*>(w + L.twin);
  for (int i = 0; i < kPanelBufs; ++i) p.gpanel[i] = reinterpret_cast<uint16_t*>(w + L.gpanel[i]);
  p.dwp = L.fused ? reinterpret_cast<float*>(w + L.dwp) : nullptr;
  p.dhp = L.fused ? reinterpret_cast<float*>(w + L.dhp) : nullptr;
  return p;
}

// control block reset + compaction + gather of the supervised rows.  With
// `reuse` (a forward on this workspace already did both) only the work
// counters are reset; the error word keeps what the forward recorded.
flce_status prologue(const void* H, const int64_t* labels, const uint8_t* mask, int64_t ignore,
                     int64_t N, int64_t D, int64_t V, int64_t v0, int64_t V_slice,
                     const Layout& L, const WsPtrs& p,
                     float* m_out, float* logs_out, int* pos, float* lossvec,
                     cudaStream_t s, bool reuse = false) {
  if (reuse) {
    FLCE_CK(cudaMemsetAsync(p.counters, 0, L.ctrl_bytes - kCounterOffset, s));
    return FLCE_OK;
  }
  FLCE_CK(cudaMemsetAsync(p.err, 0, L.ctrl_bytes, s));
  FLCE_CK(timed_launch(kProfAux, s, [&] {
    compact_kernel<<<1, COMPACT_THREADS, 0, s>>>(labels, mask, ignore, N, V, v0, V_slice, p.idx,
                                                 p.yc, p.C,
                                                 p.err, m_out, logs_out, pos, lossvec);
  }));
  const int64_t vec = D / 8;
  FLCE_CK(timed_launch(kProfAux, s, [&] {
    gather_rows_kernel<<<static_cast<unsigned>(cdiv64(L.Np, 8)), 256, 0, s>>>(
        static_cast<const uint4*>(H), p.idx, p.C, L.Np, vec, reinterpret_cast<uint4*>(p.hc));
  }));
  return FLCE_OK;
}

// Forward of the full vocabulary (shard false) or of the slice [v0, v0 + V)
// of a vocabulary of V_total ids (shard true: per-row partial statistics in
// `stats` instead of the loss; see flce_shard_forward).
flce_status forward_impl(const void* H, const void* W, const void* b, const int64_t* labels,
                         const uint8_t* mask, int64_t ignore_index, int64_t N, int64_t D,
                         int64_t V, int64_t v0, int64_t V_total, int dtype, const float* weight,
                         int reduction, float denom, unsigned flags, float* loss,
                         float* loss_rows, float* m, float* logs, bool shard, float4* stats,
                         void* ws, size_t ws_bytes, cudaStream_t s) {
  if ((reduction != FLCE_REDUCE_MEAN && reduction != FLCE_REDUCE_SUM &&
       reduction != FLCE_REDUCE_NONE) ||
      (flags & ~FLCE_FLAG_ROUND_LOGITS) != 0)
    return FLCE_ERR_ARG;
  const bool none = !shard && reduction == FLCE_REDUCE_NONE;
  if (shard) {
    if ((N > 0 && (H == nullptr || labels == nullptr || stats == nullptr)) || W == nullptr ||
        ws == nullptr)
      return FLCE_ERR_NULL;
  } else if ((N > 0 && (H == nullptr || labels == nullptr || m == nullptr || logs == nullptr ||
                        (none && loss_rows == nullptr))) ||
             W == nullptr || (!none && loss == nullptr) || ws == nullptr) {
    return FLCE_ERR_NULL;
  }
  if (dtype != FLCE_BF16 && dtype != FLCE_FP16) return FLCE_ERR_DTYPE;
  if (!shape_ok(N, D, V) || v0 < 0 || V_total > kMaxV || v0 + V > V_total)
    return FLCE_ERR_SHAPE;
  if (D % 8 != 0 || !aligned(H, 16) || !aligned(W, 16) || (b != nullptr && !aligned(b, 16)) ||
      !aligned(ws, 256) || !aligned(m, 4) || !aligned(logs, 4) || !aligned(loss, 4) ||
      !aligned(weight, 4) || !aligned(loss_rows, 4) || !aligned(stats, 16))
    return FLCE_ERR_ALIGN;
  const Layout L = make_layout(N, D, V);
  if (ws_bytes < L.fwd_total) return FLCE_ERR_WORKSPACE;
  DevInfo di;
  flce_status st = device_setup(&di);
  if (st != FLCE_OK) return st;
  const WsPtrs p = carve(ws, L);
  const bool bf16 = dtype == FLCE_BF16;
  const MapType mt = bf16 ? kMapBF16 : kMapFP16;

  float* lossvec = none ? loss_rows : nullptr;
  // the row map (pos) is kept for a backward that reuses this compaction
  st = prologue(H, labels, mask, ignore_index, N, D, V_total, v0, V, L, p, shard ? nullptr : m,
                shard ? nullptr : logs, p.pos, lossvec, s);
  if (st != FLCE_OK) return st;

  GemmArgs a{};
  if (!make_map(&a.tmA[0], p.hc, mt, D, L.Np, D * 2, BK, BM) ||
      !make_map(&a.tmB[0], W, mt, D, V, D * 2, BK, BN_HALF))
    return FLCE_ERR_CUDA;
  a.is_bf16 = bf16;
  a.C_dev = p.C;
  a.counter = p.counters;
  a.ncols = static_cast<int>(V);
  a.K = static_cast<int>(D);
  a.D = static_cast<int>(D);
  a.V = static_cast<int>(V);
  a.y_c = p.yc;
  a.idx = p.idx;
  a.bias = static_cast<const uint16_t*>(b);
  a.part = p.part;
  a.part_ld = static_cast<int>(L.Np);
  a.tgt = p.tgt;
  a.err = p.err;
  const int feat = (b != nullptr ? kFeatBias : 0) |
                   ((flags & FLCE_FLAG_ROUND_LOGITS) ? kFeatRound : 0) |
                   (D <= kPolyExpMaxD ? kFeatSmallD : 0);
  FLCE_CK(launch_gemm<kModeFwd>(a, feat, cdiv64(N, PAIR_M) * L.nvt, di.pairs, s));

  // 32 rows per block pass, at most 8 blocks per SM
  const int64_t blocks =
      cdiv64(N, MERGE_ROWS) < 8LL * di.sms ? cdiv64(N, MERGE_ROWS) : 8LL * di.sms;
  if (shard) {
    if (N > 0) {
      FLCE_CK(timed_launch(kProfAux, s, [&] {
        shard_stats_kernel<<<static_cast<unsigned>(blocks), MERGE_ROWS * MERGE_SPLIT, 0, s>>>(
            p.part, L.Np, static_cast<int>(L.nvt), p.tgt, p.yc, p.pos, N, static_cast<int>(V),
            stats, p.err);
      }));
    }
    return FLCE_OK;
  }
  if (N > 0) {
    FLCE_CK(timed_launch(kProfAux, s, [&] {
      merge_stats_kernel<<<static_cast<unsigned>(blocks), MERGE_ROWS * MERGE_SPLIT, 0, s>>>(
          p.part, L.Np, static_cast<int>(L.nvt), p.tgt, p.C, p.idx, m, logs, p.loss_rows, weight,
          lossvec, p.err);
    }));
  }
  if (!none) {
    FLCE_CK(timed_launch(kProfAux, s, [&] {
      loss_reduce_kernel<<<1, 1024, 0, s>>>(p.loss_rows, p.C,
                                            reduction == FLCE_REDUCE_MEAN ? 1 : 0, denom, p.err,
                                            loss);
    }));
  }
  return FLCE_OK;
}

// Backward of the full vocabulary (v0 = 0, V_total = V) or of the slice
// [v0, v0 + V): dW, db are the slice's rows and dH its term of the sum.
flce_status backward_impl(const void* H, const void* W, const void* b, const int64_t* labels,
                          const uint8_t* mask, int64_t ignore_index, int64_t N, int64_t D,
                          int64_t V, int64_t v0, int64_t V_total, int dtype, const float* m,
                          const float* logs, const float* weight, int reduction, float denom,
                          unsigned flags, float lambda, const float* lambda_dev,
                          const float* grad_rows, float filter_eps, float* dH, float* dW,
                          float* db, void* ws, size_t ws_bytes, cudaStream_t s) {
  if (!(filter_eps >= 0.f) || !isfinite(filter_eps)) return FLCE_ERR_ARG;
  if ((reduction != FLCE_REDUCE_MEAN && reduction != FLCE_REDUCE_SUM &&
       reduction != FLCE_REDUCE_NONE) ||
      (flags & ~(FLCE_FLAG_ROUND_LOGITS | FLCE_FLAG_ACCUMULATE_DH | FLCE_FLAG_REUSE_FORWARD |
                 FLCE_FLAG_PANEL_BACKWARD)) != 0)
    return FLCE_ERR_ARG;
  const bool none = reduction == FLCE_REDUCE_NONE;
  if ((N > 0 && (H == nullptr || labels == nullptr || m == nullptr || logs == nullptr ||
                 dH == nullptr || (none && grad_rows == nullptr))) ||
      W == nullptr || dW == nullptr || ws == nullptr || (b != nullptr && db == nullptr))
    return FLCE_ERR_NULL;
  if (dtype != FLCE_BF16 && dtype != FLCE_FP16) return FLCE_ERR_DTYPE;
  if (!shape_ok(N, D, V) || v0 < 0 || V_total > kMaxV || v0 + V > V_total)
    return FLCE_ERR_SHAPE;
  if (D % 8 != 0 || !aligned(H, 16) || !aligned(W, 16) || (b != nullptr && !aligned(b, 16)) ||
      !aligned(ws, 256) || !aligned(dH, 16) || !aligned(dW, 16) ||
      (db != nullptr && !aligned(db, 8)) || !aligned(m, 4) || !aligned(logs, 4) ||
      !aligned(weight, 4) || !aligned(grad_rows, 4))
    return FLCE_ERR_ALIGN;
  const Layout L = make_layout(N, D, V);
  if (ws_bytes < L.total) return FLCE_ERR_WORKSPACE;
  DevInfo di;
  flce_status st = device_setup(&di);
  if (st != FLCE_OK) return st;
  const WsPtrs p = carve(ws, L);
  const bool bf16 = dtype == FLCE_BF16;
  const MapType mt = bf16 ? kMapBF16 : kMapFP16;
  const float log2_sigma = bf16 ? 0.f : kFp16Log2Sigma;
  const float sigma = exp2f(log2_sigma);

  int end_bit = 1;
  while ((int64_t(1) << end_bit) <= V) ++end_bit;  // sort keys are 0 .. V
  st = prologue(H, labels, mask, ignore_index, N, D, V_total, v0, V, L, p, nullptr, nullptr,
                p.pos, nullptr, s, (flags & FLCE_FLAG_REUSE_FORWARD) != 0);
  if (st != FLCE_OK) return st;
  FLCE_CK(timed_launch(kProfAux, s, [&] {
    row_scale_kernel<<<1, 1024, 0, s>>>(p.C, p.idx, weight, none ? grad_rows : nullptr,
                                        reduction, denom, lambda, lambda_dev, p.rs, p.scal);
  }));
  // rows whose label another vocabulary slice holds keep a zero residual
  FLCE_CK(cudaMemsetAsync(p.resid, 0, static_cast<size_t>(L.Np) * 4, s));

  // maps that do not depend on the panel
  CUtensorMap hcK, wK, hcMN, wMN, dwMap, dhMap;
  if (!make_map(&hcK, p.hc, mt, D, L.Np, D * 2, BK, BM) ||
      !make_map(&wK, W, mt, D, V, D * 2, BK, BN_HALF) ||
      !make_map(&hcMN, p.hc, mt, D, L.Np, D * 2, 64, BK) ||
      !make_map(&wMN, W, mt, D, V, D * 2, 64, BK) ||
      !make_map(&dwMap, dW, kMapF32, D, V, D * 4, 32, BM) ||
      !make_map(&dhMap, p.dhc, kMapF32, D, L.Np, D * 4, 32, BM))
    return FLCE_ERR_CUDA;

  const bool fused =
      L.fused && filter_eps == 0.f && (flags & FLCE_FLAG_PANEL_BACKWARD) == 0;
  if (b != nullptr) FLCE_CK(cudaMemsetAsync(p.dbacc, 0, static_cast<size_t>(V) * 8, s));
  if (fused) {
    // single kernel: scores, gradient and both contractions per tile, then
    // the fixed-order sums of the dW and dH slabs
    FusedArgs fa{};
    GemmArgs& a = fa.g;
    a.tmA[0] = hcK;
    a.tmB[0] = wK;
    if (!make_map(&a.tmDW, p.dwp, kMapF32, D, FB_NG_MAX * L.Vp, D * 4, 32, 32) ||
        !make_map(&a.tmDH, p.dhp, kMapF32, D, FB_NCH_MAX * L.Np, D * 4, 32, 32))
      return FLCE_ERR_CUDA;
    a.is_bf16 = bf16;
    a.C_dev = p.C;
    a.counter = p.counters + 1;
    a.D = static_cast<int>(D);
    a.V = static_cast<int>(V);
    a.y_c = p.yc;
    a.idx = p.idx;
    a.bias = static_cast<const uint16_t*>(b);
    a.m_saved = m;
    a.logs_saved = logs;
    a.log2_sigma = log2_sigma;
    a.sigma = sigma;
    a.row_scale = p.rs;
    a.tgt_resid = p.resid;
    a.scal = p.scal;
    a.inv_sigma = 1.f / sigma;
    a.db_acc = b != nullptr ? p.dbacc : nullptr;
    a.db_fx_scale = 0x1p32f / sigma;
    a.err = p.err;
    fa.Vp = static_cast<int>(L.Vp);
    fa.Np = static_cast<int>(L.Np);
    fa.nctas = di.sms;
    const FusedKernel kern = pick_fused(
        (b != nullptr ? kFeatBias : 0) | ((flags & FLCE_FLAG_ROUND_LOGITS) ? kFeatRound : 0),
        FusedFeats{});
    if (kern == nullptr) return FLCE_ERR_ARG;
    FLCE_CK(timed_launch(kProfBwd, s, [&] {
      kern<<<static_cast<unsigned>(di.sms), FB_THREADS, FB_SMEM_BYTES, s>>>(fa);
    }));
    const int64_t D4 = D / 4;
    const int64_t dw_blocks =
        cdiv64(V * D4, 256) < 8LL * di.sms ? cdiv64(V * D4, 256) : 8LL * di.sms;
    FLCE_CK(timed_launch(kProfAux, s, [&] {
      fused_reduce_dw_kernel<<<static_cast<unsigned>(dw_blocks), 256, 0, s>>>(
          reinterpret_cast<const float4*>(p.dwp), L.Vp * D4, static_cast<int>(V),
          static_cast<int>(D4), p.C, di.sms, p.scal, 1.f / sigma, reinterpret_cast<float4*>(dW));
    }));
    const int64_t dh_blocks =
        cdiv64(L.Np * D4, 256) < 8LL * di.sms ? cdiv64(L.Np * D4, 256) : 8LL * di.sms;
    FLCE_CK(timed_launch(kProfAux, s, [&] {
      fused_reduce_dh_kernel<<<static_cast<unsigned>(dh_blocks), 256, 0, s>>>(
          reinterpret_cast<const float4*>(p.dhp), L.Np * D4, static_cast<int>(D4), p.C,
          static_cast<int>(V), di.sms, p.scal, 1.f / sigma, reinterpret_cast<float4*>(p.dhc));
    }));
  }

  const int64_t nT_max = cdiv64(N, PAIR_M);
  const int bn_wh = D <= 128 ? 128 : BN;  // dW / dH tile width along D
  const int64_t nD = cdiv64(D, bn_wh);
  // The GEMM launches form one timed span: with programmatic dependent launch
  // they overlap, so events between them would measure nothing useful (and
  // would hold the next launch back).
  ProfRec span;
  const bool timed = !fused && prof_span_begin(&span, kProfBwd, s);
  int launched = 0;
  for (int64_t Lp = 0; !fused && Lp <= L.panels; ++Lp) {
    const bool has_g = Lp < L.panels;
    const bool has_wh = Lp > 0;
    const int64_t vp_g = Lp * L.vc;
    const int64_t w_g = has_g ? ((V - vp_g) < L.vc ? (V - vp_g) : L.vc) : 0;
    const int64_t vp_wh = (Lp - 1) * L.vc;
    const int64_t w_wh = has_wh ? ((V - vp_wh) < L.vc ? (V - vp_wh) : L.vc) : 0;

    GemmArgs a{};
    a.tmA[kClsGrad] = hcK;
    a.tmB[kClsGrad] = wK;
    a.tmB[kClsDW] = hcMN;
    a.tmB[kClsDH] = wMN;
    a.tmDW = dwMap;
    a.tmDH = dhMap;
    if (has_g &&
        !make_map(&a.tmG, p.gpanel[Lp % kPanelBufs], mt, w_g, L.Np, L.gld * 2, 64, BM))
      return FLCE_ERR_CUDA;
    if (has_wh) {
      const uint16_t* gp = p.gpanel[(Lp - 1) % kPanelBufs];
      if (!make_map(&a.tmA[kClsDW], gp, mt, w_wh, L.Np, L.gld * 2, 64, BK) ||
          !make_map(&a.tmA[kClsDH], gp, mt, w_wh, L.Np, L.gld * 2, BK, BM))
        return FLCE_ERR_CUDA;
    }
    a.is_bf16 = bf16;
    a.C_dev = p.C;
    a.counter = p.counters + 1 + Lp;
    a.D = static_cast<int>(D);
    a.V = static_cast<int>(V);
    a.has_wh = has_wh;
    a.vp_wh = static_cast<int>(vp_wh);
    a.w_wh = static_cast<int>(w_wh);
    a.dh_accumulate = Lp > 1;
    a.bn_wh = bn_wh;
    a.has_g = has_g;
    a.vp_g = static_cast<int>(vp_g);
    a.w_g = static_cast<int>(w_g);
    a.y_c = p.yc;
    a.idx = p.idx;
    a.bias = static_cast<const uint16_t*>(b);
    a.m_saved = m;
    a.logs_saved = logs;
    a.log2_sigma = log2_sigma;
    a.sigma = sigma;
    a.row_scale = p.rs;
    a.tgt_resid = p.resid;
    a.scal = p.scal;
    a.inv_sigma = 1.f / sigma;
    a.db_acc = b != nullptr ? p.dbacc : nullptr;
    a.db_fx_scale = 0x1p32f / sigma;
    if (filter_eps > 0.f) {
      a.filter_eps_sigma = filter_eps * sigma;
      a.keep_ld = static_cast<int>(L.gld / 64);
      a.keep_g = has_g ? p.keep + L.keep_bytes * (Lp % kPanelBufs) : nullptr;
      a.keep_wh = has_wh ? p.keep + L.keep_bytes * ((Lp - 1) % kPanelBufs) : nullptr;
      // a launch without gradient units still reads flags: keep_g stays null
      // there, so the kernel tests keep_wh for the consumers
    }
    a.err = p.err;
    const int64_t units = (has_wh ? cdiv64(w_wh, PAIR_M) * nD + nT_max * nD : 0) +
                          (has_g ? nT_max * cdiv64(w_g, BN) : 0);
    // every launch after the first may overlap its predecessor
    const int feat = (b != nullptr ? kFeatBias : 0) | (filter_eps > 0.f ? kFeatFilter : 0) |
                     ((flags & FLCE_FLAG_ROUND_LOGITS) ? kFeatRound : 0);
    FLCE_CK(launch_gemm<kModeBwd>(a, feat, units, di.pairs, s, /*pdl=*/launched > 0,
                                  /*timed=*/false));
    launched += units > 0 ? 1 : 0;
  }
  if (timed) prof_span_end(&span, launched, s);
  if (b != nullptr) {
    FLCE_CK(timed_launch(kProfAux, s, [&] {
      bias_finish_kernel<<<static_cast<unsigned>(cdiv64(V, 256)), 256, 0, s>>>(
          p.dbacc, static_cast<int>(V), p.C, p.scal, db);
    }));
  }
  if (N > 0) {
    // dW's target terms in fp32: group the rows by label (stable sort), then
    // add each group's residuals times its H rows to the label's dW row
    const int64_t pblocks = cdiv64(L.Np, 256) < 4LL * di.sms ? cdiv64(L.Np, 256) : 4LL * di.sms;
    FLCE_CK(timed_launch(kProfAux, s, [&] {
      label_sort_prep_kernel<<<static_cast<unsigned>(pblocks), 256, 0, s>>>(
          p.C, p.yc, L.Np, static_cast<int>(V), p.skeys[0], p.svals[0]);
    }));
    int cur = 0;
    const unsigned tiles = static_cast<unsigned>(cdiv64(L.Np, RS_TILE));
    for (int shift = 0; shift < end_bit; shift += RS_BITS) {
      FLCE_CK(timed_launch(kProfAux, s, [&] {
        radix_count_kernel<<<tiles, RS_TILE, 0, s>>>(p.skeys[cur], L.Np, shift, p.rscount);
      }));
      FLCE_CK(timed_launch(kProfAux, s, [&] {
        radix_scan_kernel<<<1, 1024, 0, s>>>(p.rscount, static_cast<int64_t>(RS_DIGITS) * tiles);
      }));
      FLCE_CK(timed_launch(kProfAux, s, [&] {
        radix_scatter_kernel<<<tiles, RS_TILE, 0, s>>>(p.skeys[cur], p.svals[cur], L.Np, shift,
                                                       p.rscount, p.skeys[cur ^ 1],
                                                       p.svals[cur ^ 1]);
      }));
      cur ^= 1;
    }
    // one warp per (window of TW sorted rows, 128 columns), both passes
    const int64_t rwarps = cdiv64(L.Np, TW) * cdiv64(D / 4, 32);
    const int64_t rblocks = cdiv64(rwarps, 8);
    FLCE_CK(timed_launch(kProfAux, s, [&] {
      dw_target_window_kernel<<<static_cast<unsigned>(rblocks), 256, 0, s>>>(
          p.skeys[cur], p.svals[cur], L.Np, static_cast<int>(V),
          reinterpret_cast<const uint2*>(p.hc), D / 4, bf16 ? 1 : 0, p.resid, p.scal,
          1.f / sigma, reinterpret_cast<float4*>(p.twin), reinterpret_cast<float4*>(dW));
    }));
    FLCE_CK(timed_launch(kProfAux, s, [&] {
      dw_target_chain_kernel<<<static_cast<unsigned>(rblocks), 256, 0, s>>>(
          p.skeys[cur], L.Np, static_cast<int>(V), D / 4,
          reinterpret_cast<const float4*>(p.twin), p.scal, 1.f / sigma,
          reinterpret_cast<float4*>(dW));
    }));
    FLCE_CK(timed_launch(kProfAux, s, [&] {
      scatter_dh_kernel<<<static_cast<unsigned>(cdiv64(N, 8)), 256, 0, s>>>(
          reinterpret_cast<const float4*>(p.dhc), p.pos, N, D / 4, reinterpret_cast<float4*>(dH),
          p.resid, p.yc, static_cast<const uint2*>(W), bf16 ? 1 : 0, static_cast<int>(V), p.scal,
          1.f / sigma, (flags & FLCE_FLAG_ACCUMULATE_DH) ? 1 : 0);
    }));
  }
  return FLCE_OK;
}

}  // namespace

extern "C" {

size_t flce_workspace_bytes(int64_t N, int64_t D, int64_t V, int dtype) {
  if (!shape_ok(N, D, V) || (dtype != FLCE_BF16 && dtype != FLCE_FP16)) return 0;
  return make_layout(N, D, V).total;
}

const char* flce_status_string(int status) {
  switch (status) {
    case FLCE_OK: return "FLCE_OK";
    case FLCE_ERR_NULL: return "FLCE_ERR_NULL: a required pointer is NULL";
    case FLCE_ERR_SHAPE: return "FLCE_ERR_SHAPE: N, D or V out of range";
    case FLCE_ERR_DTYPE: return "FLCE_ERR_DTYPE: dtype must be FLCE_BF16 or FLCE_FP16";
    case FLCE_ERR_ALIGN: return "FLCE_ERR_ALIGN: misaligned pointer or D not a multiple of 8";
    case FLCE_ERR_WORKSPACE: return "FLCE_ERR_WORKSPACE: workspace too small";
    case FLCE_ERR_CUDA: return "FLCE_ERR_CUDA: a CUDA runtime call failed";
    case FLCE_ERR_LABEL: return "FLCE_ERR_LABEL: supervised label outside [0, V)";
    case FLCE_ERR_TIMEOUT: return "FLCE_ERR_TIMEOUT: a device pipeline wait ran out";
    case FLCE_ERR_NONFINITE: return "FLCE_ERR_NONFINITE: non-finite per-row statistic";
    case FLCE_ERR_DEVICE: return "FLCE_ERR_DEVICE: current device is not sm_100";
    case FLCE_ERR_ARG: return "FLCE_ERR_ARG: invalid argument value";
    case FLCE_ERR_SHARD:
      return "FLCE_ERR_SHARD: a supervised label is held by no vocabulary slice or by several";
    default: return "FLCE_ERR_UNKNOWN";
  }
}

flce_status flce_compact(const int64_t* labels, const uint8_t* mask, int64_t ignore_index,
                         int64_t N, int64_t V, int32_t* idx, int32_t* C_out, void* ws,
                         size_t ws_bytes, flce_stream stream) {
  if ((N > 0 && (labels == nullptr || idx == nullptr)) || C_out == nullptr || ws == nullptr)
    return FLCE_ERR_NULL;
  if (N < 0 || N > kMaxN || V < 1 || V > kMaxV) return FLCE_ERR_SHAPE;
  if (!aligned(ws, 256)) return FLCE_ERR_ALIGN;
  if (ws_bytes < 256) return FLCE_ERR_WORKSPACE;
  DevInfo di;
  const flce_status st = device_setup(&di);
  if (st != FLCE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(ws);
  FLCE_CK(cudaMemsetAsync(err, 0, 256, s));
  FLCE_CK(timed_launch(kProfAux, s, [&] {
    compact_kernel<<<1, COMPACT_THREADS, 0, s>>>(labels, mask, ignore_index, N, V, 0, V, idx,
                                                 nullptr,
                                                 C_out, err, nullptr, nullptr, nullptr, nullptr);
  }));
  return FLCE_OK;
}

flce_status flce_forward(const void* H, const void* W, const void* b, const int64_t* labels,
                         const uint8_t* mask, int64_t ignore_index, int64_t N, int64_t D,
                         int64_t V, int dtype, float* loss, float* m, float* logs, void* ws,
                         size_t ws_bytes, flce_stream stream) {
  return flce_forward_ex(H, W, b, labels, mask, ignore_index, N, D, V, dtype, nullptr,
                         FLCE_REDUCE_MEAN, 0.f, 0u, loss, nullptr, m, logs, ws, ws_bytes,
                         stream);
}

flce_status flce_forward_ex(const void* H, const void* W, const void* b, const int64_t* labels,
                            const uint8_t* mask, int64_t ignore_index, int64_t N, int64_t D,
                            int64_t V, int dtype, const float* weight, int reduction, float denom,
                            unsigned flags, float* loss, float* loss_rows, float* m, float* logs,
                            void* ws,
                            size_t ws_bytes, flce_stream stream) {
  return forward_impl(H, W, b, labels, mask, ignore_index, N, D, V, 0, V, dtype, weight,
                      reduction, denom, flags, loss, loss_rows, m, logs, false, nullptr, ws,
                      ws_bytes, static_cast<cudaStream_t>(stream));
}

flce_status flce_shard_forward(const void* H, const void* W_slice, const void* b_slice,
                               const int64_t* labels, const uint8_t* mask, int64_t ignore_index,
                               int64_t N, int64_t D, int64_t V_slice, int64_t v0,
                               int64_t V_total, int dtype, unsigned flags, float* stats,
                               void* ws, size_t ws_bytes, flce_stream stream) {
  return forward_impl(H, W_slice, b_slice, labels, mask, ignore_index, N, D, V_slice, v0,
                      V_total, dtype, nullptr, FLCE_REDUCE_MEAN, 0.f, flags, nullptr, nullptr,
                      nullptr, nullptr, true, reinterpret_cast<float4*>(stats), ws, ws_bytes,
                      static_cast<cudaStream_t>(stream));
}

size_t flce_shard_combine_workspace_bytes(int64_t N) {
  if (N < 0 || N > kMaxN) return 0;
  return combine_layout(N).total;
}

flce_status flce_shard_combine(const float* stats_all, int P, const int64_t* labels,
                               const uint8_t* mask, int64_t ignore_index, int64_t N,
                               const float* weight, int reduction, float denom, float* loss,
                               float* loss_rows, float* m, float* logs, void* ws,
                               size_t ws_bytes, flce_stream stream) {
  if (reduction != FLCE_REDUCE_MEAN && reduction != FLCE_REDUCE_SUM &&
      reduction != FLCE_REDUCE_NONE)
    return FLCE_ERR_ARG;
  const bool none = reduction == FLCE_REDUCE_NONE;
  if ((N > 0 && (stats_all == nullptr || labels == nullptr || m == nullptr || logs == nullptr ||
                 (none && loss_rows == nullptr))) ||
      (!none && loss == nullptr) || ws == nullptr)
    return FLCE_ERR_NULL;
  if (N < 0 || N > kMaxN || P < 1 || P > kMaxShards) return FLCE_ERR_SHAPE;
  if (!aligned(stats_all, 16) || !aligned(ws, 256) || !aligned(m, 4) || !aligned(logs, 4) ||
      !aligned(loss, 4) || !aligned(weight, 4) || !aligned(loss_rows, 4))
    return FLCE_ERR_ALIGN;
  const CombineLayout L = combine_layout(N);
  if (ws_bytes < L.total) return FLCE_ERR_WORKSPACE;
  DevInfo di;
  const flce_status st = device_setup(&di);
  if (st != FLCE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint32_t* err = reinterpret_cast<uint32_t*>(w);
  int* C = reinterpret_cast<int*>(w + L.C);
  int* idx = reinterpret_cast<int*>(w + L.idx);
  float* rows = reinterpret_cast<float*>(w + L.loss_rows);
  float* lossvec = none ? loss_rows : nullptr;
  FLCE_CK(cudaMemsetAsync(err, 0, 256, s));
  // labels were range-checked by the slices' forwards; V here only bounds them again
  FLCE_CK(timed_launch(kProfAux, s, [&] {
    compact_kernel<<<1, COMPACT_THREADS, 0, s>>>(labels, mask, ignore_index, N, kMaxV, 0, kMaxV,
                                                 idx, nullptr, C, err, m, logs, nullptr, lossvec);
  }));
  if (N > 0) {
    const int64_t blocks = cdiv64(N, 256) < 4LL * di.sms ? cdiv64(N, 256) : 4LL * di.sms;
    FLCE_CK(timed_launch(kProfAux, s, [&] {
      shard_combine_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
          reinterpret_cast<const float4*>(stats_all), P, N, C, idx, m, logs, rows, weight,
          lossvec, err);
    }));
  }
  if (!none) {
    FLCE_CK(timed_launch(kProfAux, s, [&] {
      loss_reduce_kernel<<<1, 1024, 0, s>>>(rows, C, reduction == FLCE_REDUCE_MEAN ? 1 : 0,
                                            denom, err, loss);
    }));
  }
  return FLCE_OK;
}

flce_status flce_backward(const void* H, const void* W, const void* b, const int64_t* labels,
                          const uint8_t* mask, int64_t ignore_index, int64_t N, int64_t D,
                          int64_t V, int dtype, const float* m, const float* logs, float lambda,
                          const float* lambda_dev, float* dH, float* dW, float* db, void* ws,
                          size_t ws_bytes, flce_stream stream) {
  return flce_backward_ex(H, W, b, labels, mask, ignore_index, N, D, V, dtype, m, logs, nullptr,
                          FLCE_REDUCE_MEAN, 0.f, 0u, lambda, lambda_dev, nullptr, dH, dW, db, ws,
                          ws_bytes, stream);
}

flce_status flce_backward_ex(const void* H, const void* W, const void* b, const int64_t* labels,
                             const uint8_t* mask, int64_t ignore_index, int64_t N, int64_t D,
                             int64_t V, int dtype, const float* m, const float* logs,
                             const float* weight, int reduction, float denom, unsigned flags,
                             float lambda,
                             const float* lambda_dev, const float* grad_rows, float* dH,
                             float* dW, float* db, void* ws, size_t ws_bytes,
                             flce_stream stream) {
  return backward_impl(H, W, b, labels, mask, ignore_index, N, D, V, 0, V, dtype, m, logs, weight,
                       reduction, denom, flags, lambda, lambda_dev, grad_rows, 0.f, dH, dW, db,
                       ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

flce_status flce_backward_filtered(const void* H, const void* W, const void* b,
                                   const int64_t* labels, const uint8_t* mask,
                                   int64_t ignore_index, int64_t N, int64_t D, int64_t V,
                                   int dtype, const float* m, const float* logs,
                                   const float* weight, int reduction, float denom,
                                   unsigned flags, float lambda, const float* lambda_dev,
                                   const float* grad_rows, float filter_eps, float* dH, float* dW,
                                   float* db, void* ws, size_t ws_bytes, flce_stream stream) {
  return backward_impl(H, W, b, labels, mask, ignore_index, N, D, V, 0, V, dtype, m, logs, weight,
                       reduction, denom, flags, lambda, lambda_dev, grad_rows, filter_eps, dH,
                       dW, db, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

flce_status flce_shard_backward(const void* H, const void* W_slice, const void* b_slice,
                                const int64_t* labels, const uint8_t* mask, int64_t ignore_index,
                                int64_t N, int64_t D, int64_t V_slice, int64_t v0,
                                int64_t V_total, int dtype, const float* m, const float* logs,
                                const float* weight, int reduction, float denom, unsigned flags,
                                float lambda, const float* lambda_dev, const float* grad_rows,
                                float* dH, float* dW_slice, float* db_slice, void* ws,
                                size_t ws_bytes, flce_stream stream) {
  return backward_impl(H, W_slice, b_slice, labels, mask, ignore_index, N, D, V_slice, v0,
                       V_total, dtype, m, logs, weight, reduction, denom, flags, lambda,
                       lambda_dev, grad_rows, 0.f, dH, dW_slice, db_slice, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream));
}

flce_status flce_device_status(const void* ws, flce_stream stream) {
  if (ws == nullptr) return FLCE_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FLCE_ERR_CUDA;
  uint32_t e = 0;
  if (cudaMemcpy(&e, ws, sizeof(e), cudaMemcpyDeviceToHost) != cudaSuccess) return FLCE_ERR_CUDA;
  if (e & kErrBitLabel) return FLCE_ERR_LABEL;
  if (e & kErrBitTimeout) return FLCE_ERR_TIMEOUT;
  if (e & kErrBitShard) return FLCE_ERR_SHARD;
  if (e & kErrBitNonfinite) return FLCE_ERR_NONFINITE;
  if (e != 0) return FLCE_ERR_CUDA;
  return FLCE_OK;
}

flce_status flce_diag_gemm(const void* A, const void* B, float* out, int64_t M, int64_t N,
                           int64_t K, int dtype, int a_mn, int b_mn, float scale, void* ws,
                           size_t ws_bytes, flce_stream stream) {
  if (A == nullptr || B == nullptr || out == nullptr || ws == nullptr) return FLCE_ERR_NULL;
  if (dtype != FLCE_BF16 && dtype != FLCE_FP16) return FLCE_ERR_DTYPE;
  if (M < 1 || N < 1 || K < 1 || M > kMaxN || N > kMaxV || K > kMaxN) return FLCE_ERR_SHAPE;
  if ((a_mn ? M : K) % 8 != 0 || (b_mn ? N : K) % 8 != 0 || !aligned(A, 16) ||
      !aligned(B, 16) || !aligned(ws, 256))
    return FLCE_ERR_ALIGN;
  if (ws_bytes < 256) return FLCE_ERR_WORKSPACE;
  DevInfo di;
  const flce_status st = device_setup(&di);
  if (st != FLCE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const MapType mt = dtype == FLCE_BF16 ? kMapBF16 : kMapFP16;
  GemmArgs a{};
  const bool okA = a_mn ? make_map(&a.tmA[0], A, mt, M, K, M * 2, 64, BK)
                        : make_map(&a.tmA[0], A, mt, K, M, K * 2, BK, BM);
  const bool okB = b_mn ? make_map(&a.tmB[0], B, mt, N, K, N * 2, 64, BK)
                        : make_map(&a.tmB[0], B, mt, K, N, K * 2, BK, BN_HALF);
  if (!okA || !okB) return FLCE_ERR_CUDA;
  a.a_mn = a_mn ? 1 : 0;
  a.b_mn = b_mn ? 1 : 0;
  a.is_bf16 = dtype == FLCE_BF16;
  a.M = static_cast<int>(M);
  a.ncols = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.out = out;
  a.scale = scale;
  a.err = static_cast<uint32_t*>(ws);
  a.counter = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + kCounterOffset);
  FLCE_CK(cudaMemsetAsync(ws, 0, 256, s));
  FLCE_CK(launch_gemm<kModePlain>(a, 0, cdiv64(M, PAIR_M) * cdiv64(N, BN), di.pairs, s));
  return FLCE_OK;
}

flce_status flce_diag_exp2(const float* x, float* y_poly, float* y_sfu, int64_t n,
                           flce_stream stream) {
  if (n > 0 && (x == nullptr || y_poly == nullptr || y_sfu == nullptr)) return FLCE_ERR_NULL;
  if (n < 0 || n > (int64_t(1) << 31)) return FLCE_ERR_SHAPE;
  if (n == 0) return FLCE_OK;
  DevInfo di;
  const flce_status st = device_setup(&di);
  if (st != FLCE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FLCE_CK(timed_launch(kProfAux, s, [&] {
    exp2_probe_kernel<<<static_cast<unsigned>(cdiv64(n, 256)), 256, 0, s>>>(x, y_poly, y_sfu, n);
  }));
  return FLCE_OK;
}

flce_status flce_diag_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns, flce_stream stream) {
  if (ws == nullptr) return FLCE_ERR_NULL;
  if (!aligned(ws, 256)) return FLCE_ERR_ALIGN;
  if (ws_bytes < 256) return FLCE_ERR_WORKSPACE;
  DevInfo di;
  const flce_status st = device_setup(&di);
  if (st != FLCE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FLCE_CK(cudaMemsetAsync(ws, 0, 256, s));
  FLCE_CK(timed_launch(kProfAux, s, [&] {
    timeout_probe_kernel<<<1, 32, 0, s>>>(static_cast<uint32_t*>(ws), limit_ns);
  }));
  return FLCE_OK;
}

flce_status flce_diag_profile_begin(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof) {
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  g_prof.clear();
  g_prof_on = true;
  return FLCE_OK;
}

flce_status flce_diag_profile_end(double* ms, int64_t* launches, int nkinds) {
  if (ms == nullptr || launches == nullptr) return FLCE_ERR_NULL;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = false;
  for (int k = 0; k < nkinds; ++k) {
    ms[k] = 0.0;
    launches[k] = 0;
  }
  flce_status st = FLCE_OK;
  for (auto& r : g_prof) {
    float t = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
      st = FLCE_ERR_CUDA;
    if (r.kind < nkinds) {
      ms[r.kind] += t;
      launches[r.kind] += r.launches;
    }
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  g_prof.clear();
  return st;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward with the library's own fixed scratch, for callers that cannot
// allocate device memory (see flce_forward_noalloc in flce.h).
// ---------------------------------------------------------------------------
namespace {
static __device__ __align__(256) uint8_t g_noalloc_scratch[FLCE_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device (host code cannot
// use the symbol itself as a device pointer).  Looked up on every call, with
// the device current: the lookup allocates nothing, and an address kept from
// an earlier call could be stale after a reset of the device's primary context
// (the module, and with it the array, is loaded again).
flce_status noalloc_scratch(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return FLCE_ERR_CUDA;
  *out = p;
  return FLCE_OK;
}
}  // namespace

extern "C" flce_status flce_forward_noalloc(const void* H, const void* W, const void* b,
                                            const int64_t* labels, const uint8_t* mask,
                                            int64_t ignore_index, int64_t N, int64_t D,
                                            int64_t V, int dtype, float* loss, float* m,
                                            float* logs, flce_stream stream) {
  if (dtype != FLCE_BF16 && dtype != FLCE_FP16) return FLCE_ERR_DTYPE;
  if (!shape_ok(N, D, V)) return FLCE_ERR_SHAPE;
  if (make_layout(N, D, V).fwd_total > FLCE_NOALLOC_SCRATCH_BYTES) return FLCE_ERR_WORKSPACE;
  void* scratch = nullptr;
  const flce_status st = noalloc_scratch(&scratch);
  if (st != FLCE_OK) return st;
  return flce_forward(H, W, b, labels, mask, ignore_index, N, D, V, dtype, loss, m, logs, scratch,
                      FLCE_NOALLOC_SCRATCH_BYTES, stream);
}
