// Persistent, warp-specialised tcgen05 GEMM for sm_100a with the fused
// epilogues of exact linear cross-entropy.
//
// CTAs run in pairs (clusters of 2), one CTA per SM; a work unit is a
// 256 x 256 output tile.  Each CTA holds half of the unit's A rows (128) and
// half of its B rows (128) in a STAGES-deep ring of 32 KiB stages loaded by
// TMA, and half of the accumulator (128 rows x 256 f32 columns) in its TMEM.
// The even CTA of the pair takes work units from a global counter (longest
// units first) and broadcasts each unit id into both CTAs' unit rings; its
// warp 1 issues tcgen05.mma.cta_group::2.kind::f16 (M=256, N=256, K=16),
// which reads both CTAs' stages and writes both CTAs' TMEM, into one of two
// accumulators (512 columns).  In each CTA, warp 0 streams that CTA's halves
// of the operands (in the backward warp 0 the A boxes and warp 2 the B
// boxes), and two epilogue warpgroups (warps 4..7 and 8..11, each on half of
// the columns; four in the small-D forward) read a finished accumulator with
// tcgen05.ld (thread = TMEM lane = tile row) and run the epilogue while the
// next unit accumulates in the other.
//
// Modes (one launch = one mode; each mode is instantiated once per
// combination of its optional features FEAT, see Feature):
//   kModeFwd   Z = H_c W^T (+ b) per 128 x 256 tile; the epilogue keeps the
//              running max / rescaled exp-sum over the tile's columns and
//              captures the target logit from the tile that holds it
//              ("分块交叉熵" page, §02); the two warpgroups' halves of a row
//              are merged in shared memory and one (m, s) partial per row and
//              tile is stored, tile-major (a warp's 32 rows are contiguous).
//   kModeBwd   three unit classes in one launch, with no dependency between
//              them, longest first.  The launch may start while the previous
//              one still runs (programmatic dependent launch): its producers
//              wait for it before their first dW / dH unit.
//              class 2 (grad): the tile of vocabulary panel p recomputed; the
//                 epilogue rebuilds p = exp((Z - m) - log s) from the saved
//                 statistics, subtracts the one-hot target (§04), rounds to
//                 the 16-bit input type, stages 128 x 64 boxes in shared
//                 memory and stores them with TMA into gradient buffer p % 2,
//                 and records what the rounding took off each row's target
//                 entry (added back in fp32 to dH and dW later); with a bias,
//                 the fp32 column sums of its rows go to the bias gradient
//                 as 64-bit fixed-point integer additions (order-free, so
//                 deterministic);
//              The panel holds r_k (p - onehot) sigma with the row scale
//              s_k = S r_k (S = max |s_k|), the contractions multiply by S / sigma.
//              class 0 (dW): dW[panel p-1 rows] = G^T H_c  (K = C), stored by TMA;
//              class 1 (dH): dH_c (+)= G W[panel p-1]      (K = panel width),
//                 stored (first panel) or added with a TMA reduction (later
//                 panels).
//              Every output tile is owned by one unit and panels run in
//              order, so dW, dH and the panel buffers are deterministic.
//   kModePlain diagnostic: out = scale * A B^T with a plain store.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace flce {

constexpr int BM = 128;                          // rows per CTA
constexpr int PAIR_M = 2 * BM;                   // rows per work unit (CTA pair)
constexpr int BN = 256;                          // columns per work unit
constexpr int BN_HALF = BN / 2;                  // B rows held by each CTA
constexpr int BK = 64;
constexpr int UQ = 4;                            // depth of the unit-id ring
constexpr uint32_t A_STAGE_BYTES = BM * BK * 2;       // 16 KiB
constexpr uint32_t B_STAGE_BYTES = BN_HALF * BK * 2;  // 16 KiB
// bytes both CTAs' loads bring per k-block for a tile of bn columns
__host__ __device__ constexpr uint32_t pair_tx_bytes(int bn) {
  return 2 * (A_STAGE_BYTES + static_cast<uint32_t>(bn / 2) * BK * 2);
}
constexpr uint32_t MN_BOX_BYTES = 64 * BK * 2;   // 8 KiB: 64 MN-elements x 64 K rows
constexpr uint32_t STG_BYTES = BM * 128;         // 16 KiB: 128 rows x 128 bytes
// Warps 0-3 form the first warpgroup: scheduler + producer (warp 0), MMA
// issuer (warp 1), two idle warps.  Warps 4-11 are the epilogue: two
// warpgroups, each draining half of the accumulator's columns (warp w reads
// TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31, the rows of its quadrant).  The
// small-D forward has four epilogue warpgroups, warps 4-19, a quarter of the
// columns each (see Shape).
constexpr int NUM_THREADS = 384;
constexpr int EPI_WARP0 = 4;
constexpr int NUM_EPI_WG = 2;
constexpr int EPI_WG_THREADS = 128;
constexpr int NUM_EPI_THREADS = NUM_EPI_WG * EPI_WG_THREADS;
// Registers per thread after the split: the first warpgroup gives up what the
// epilogue takes.  The block is launched with at least kRegsAtLaunch per
// thread (checked on the host before any launch), which covers the split.
// 80 / 208 is the split at which no instantiation spills: 72 / 216 spilled
// in the plain forward and backward variants, 56 in the producers.
constexpr uint32_t kRegsLow = 80;
constexpr uint32_t kRegsHigh = 208;
constexpr uint32_t kRegsAtLaunch =
    (128 * kRegsLow + NUM_EPI_THREADS * kRegsHigh + NUM_THREADS - 1) / NUM_THREADS;
static_assert(128 * kRegsLow + NUM_EPI_THREADS * kRegsHigh <= 65536, "register split");
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr float kLog2e = 1.4426950408889634f;
enum GemmMode : int { kModeFwd = 0, kModeBwd = 1, kModePlain = 2 };

// Ring depth per mode: the backward epilogue stages TMA stores through one
// 16 KiB box per epilogue warpgroup, the other modes use that shared memory
// for a 7th stage (6 with four epilogue warpgroups, whose (m, s) merge takes
// more room).
template <int MODE, bool WIDE = false>
struct ModeCfg {
  static constexpr int STAGES = (MODE == kModeBwd || WIDE) ? 6 : 7;
  static constexpr uint32_t STAGING = (MODE == kModeBwd) ? NUM_EPI_WG * STG_BYTES : 0;
  // forward: one (m, s) pair per row of the CTA's half tile from each
  // epilogue warpgroup but the first, to merge their column slices
  static constexpr uint32_t MERGE = (MODE == kModeFwd) ? (WIDE ? 3 : 1) * BM * 8 : 0;
  static constexpr size_t SMEM_BYTES =
      1024 + STAGES * (A_STAGE_BYTES + B_STAGE_BYTES) + STAGING + 512 + MERGE;
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};
constexpr size_t GEMM_SMEM_BYTES = ModeCfg<kModeBwd>::SMEM_BYTES;  // the largest
enum UnitClass : int { kClsDW = 0, kClsDH = 1, kClsGrad = 2 };
// Optional work, chosen when the kernel is compiled (one instantiation per
// combination), so that the common path carries none of its code: measured,
// the runtime-switched form cost the backward 3-4 %.  Both passes: the bias
// (its add to the logits, and in the backward its column sums) and the
// rounding of the logits to the input type.  Backward: gradient filtering.
// Forward: one exponential in four on the FMA pipe.
enum Feature : int {
  kFeatBias = 1,
  kFeatFilter = 2,
  kFeatPolyExp = 4,
  kFeatRound = 8,
  kFeatWide = 16  // forward: four epilogue warpgroups (small D, where the epilogue is the bound)
};

// Thread layout of an instantiation: the first warpgroup (scheduler,
// producers, MMA issuer) and two epilogue warpgroups, or four for kFeatWide
// (640 threads; registers 64 / 104 after the split, 96 at launch).
template <int MODE, int FEAT>
struct Shape {
  static constexpr bool WIDE = MODE == kModeFwd && (FEAT & kFeatWide) != 0;
  static constexpr int EPI_WG = WIDE ? 4 : NUM_EPI_WG;
  static constexpr int EPI_THREADS = EPI_WG * EPI_WG_THREADS;
  static constexpr int THREADS = EPI_WARP0 * 32 + EPI_THREADS;
  static constexpr int CHUNKS = BN / 32 / EPI_WG;  // 32-column chunks per epilogue warpgroup
  static constexpr uint32_t REGS_LOW = WIDE ? 64 : kRegsLow;
  static constexpr uint32_t REGS_HIGH = WIDE ? 104 : kRegsHigh;
  static constexpr uint32_t REGS_AT_LAUNCH =
      (128 * REGS_LOW + EPI_THREADS * REGS_HIGH + THREADS - 1) / THREADS;
  static_assert(128 * REGS_LOW + EPI_THREADS * REGS_HIGH <= 65536, "register split");
  using Cfg = ModeCfg<MODE, WIDE>;
};

struct GemmArgs {
  CUtensorMap tmA[3];  // A operand map per unit class (fwd / plain use [0])
  CUtensorMap tmB[3];  // B operand map per unit class
  CUtensorMap tmG;     // bwd: store map of the gradient panel being produced
  CUtensorMap tmDW;    // bwd: fp32 dW [V x D], 128 x 32 boxes
  CUtensorMap tmDH;    // bwd: fp32 compact dH [Np x D], 128 x 32 boxes
  int a_mn;            // plain: A is MN-major
  int b_mn;            // plain: B is MN-major
  int is_bf16;
  const int* C_dev;    // supervised-row count (device); unused in plain mode
  int* counter;        // work-unit counter of this launch, zero at launch
  int M;               // plain: rows of out
  int ncols;           // fwd: V; plain: N
  int K;               // fwd: D; plain: K
  int D;
  int V;
  // bwd: the dW/dH part works on panel [vp_wh, vp_wh + w_wh), the gradient
  // part produces panel [vp_g, vp_g + w_g)
  int has_wh, vp_wh, w_wh, dh_accumulate;
  int bn_wh;               // bwd: columns (hidden dimension) of a dW / dH tile: BN, or 128
                           //      when D <= 128, so that small D does not pay for padding
  int has_g, vp_g, w_g;
  // epilogue data
  const int* y_c;          // compact labels
  const int* idx;          // compact row -> original row
  const uint16_t* bias;    // 16-bit bias [V] or null
  float2* part;            // fwd: (m, s) partials [tiles][part_ld], part_ld >= rows
  int part_ld;
  float* tgt;              // fwd: target logits [rows]
  const float* m_saved;    // bwd: saved statistics [N]
  const float* logs_saved;
  float log2_sigma;        // bwd: the panel holds (p - onehot) * sigma
  float sigma;
  const float* row_scale;  // bwd: r_k, relative row scale of compact row k, in [-1, 1]
  float* tgt_resid;        // bwd: per compact row, the target entry's value minus its 16-bit
                           //      panel value (written by the tile that holds the label)
  const float* scal;       // bwd: S (device scalar); G = S r_k (p - onehot)
  float inv_sigma;
  unsigned long long* db_acc;  // bwd, bias only (else null): per vocabulary id, the sum of
                               //      the column's r_k (p - onehot) in 2^-32 fixed point
  float db_fx_scale;           // bwd: 2^32 / sigma (panel units -> fixed point)
  // bwd, gradient filtering (keep_g / keep_wh null when off): a 128-row x
  // 64-column box of the panel whose every |p - onehot| sigma is below
  // filter_eps_sigma is dropped: stored as zeros and flagged 0, and the dW /
  // dH units skip the k-blocks whose boxes are all dropped.
  float filter_eps_sigma;
  uint8_t* keep_g;             // flags of the panel being produced [Np / 128][keep_ld]
  const uint8_t* keep_wh;      // flags of the panel being read
  int keep_ld;                 // boxes per 128-row half (panel pitch / 64)
  float* out;              // plain
  float scale;             // plain
  uint32_t* err;
};

struct Unit {
  int cls;
  int m0;
  int n0;
  int nk;
  int bn;  // columns of the unit's tile: BN, or GemmArgs::bn_wh for dW / dH units
};

__device__ __forceinline__ int cdiv_i(int a, int b) { return (a + b - 1) / b; }

// Work units of one launch, grouped by class and ordered longest-first.
// Fields are scalars (no arrays) so that they stay in registers.
struct UnitSpace {
  int n0, n1, n2;     // units per class
  int k0, k1, k2;     // K-blocks per unit of each class
  int o0, o1, o2;     // classes, longest first
  int total;
};

__device__ __forceinline__ int pick3(int c, int a, int b, int d) {
  return c == 0 ? a : (c == 1 ? b : d);
}

template <int MODE>
__device__ __forceinline__ UnitSpace make_unit_space(const GemmArgs& g, int C) {
  UnitSpace s;
  if (MODE == kModeBwd) {
    const int nT = cdiv_i(C, PAIR_M), nD = cdiv_i(g.D, g.bn_wh);
    s.n0 = g.has_wh ? cdiv_i(g.w_wh, PAIR_M) * nD : 0;   // dW
    s.n1 = g.has_wh ? nT * nD : 0;                       // dH
    s.n2 = g.has_g ? nT * cdiv_i(g.w_g, BN) : 0;         // grad
    s.k0 = cdiv_i(C, BK);
    s.k1 = cdiv_i(g.w_wh, BK);
    s.k2 = cdiv_i(g.D, BK);
    // Longest units first (dW, dH, then the short gradient units), so that a
    // launch ends on short units (a short tail), and the panel the gradient
    // units write at the end of a launch is still in L2 when the next
    // launch's dW / dH units read it at its start.  Measured against
    // gradient-units-first (which lets them overlap the previous launch's
    // tail): about 1 % faster.
    {
      int a = 0, b = 1, c = 2;
      int ka = s.k0, kb = s.k1, kc = s.k2;
      if (ka < kb) { int t = a; a = b; b = t; t = ka; ka = kb; kb = t; }
      if (kb < kc) { int t = b; b = c; c = t; t = kb; kb = kc; kc = t; }
      if (ka < kb) { int t = a; a = b; b = t; t = ka; ka = kb; kb = t; }
      s.o0 = a;
      s.o1 = b;
      s.o2 = c;
    }
    s.total = s.n0 + s.n1 + s.n2;
  } else {
    const int rows = (MODE == kModePlain) ? g.M : C;
    s.n0 = cdiv_i(rows, PAIR_M) * cdiv_i(g.ncols, BN);
    s.n1 = s.n2 = 0;
    s.k0 = cdiv_i(g.K, BK);
    s.k1 = s.k2 = 0;
    s.o0 = 0;
    s.o1 = 1;
    s.o2 = 2;
    s.total = s.n0;
  }
  return s;
}

// Unit u -> 256 x 256 tile (m0, n0) of the pair.  For the forward, gradient and
// plain tiles, row (token) tiles vary fastest so that units running at
// the same time share the W / G columns they read through L2.
template <int MODE>
__device__ __forceinline__ Unit decode_unit(const GemmArgs& g, const UnitSpace& s, int C, int u) {
  Unit un;
  int cls = s.o0;
  const int c0 = pick3(s.o0, s.n0, s.n1, s.n2);
  if (u >= c0) {
    u -= c0;
    cls = s.o1;
    const int c1 = pick3(s.o1, s.n0, s.n1, s.n2);
    if (u >= c1) {
      u -= c1;
      cls = s.o2;
    }
  }
  un.cls = cls;
  un.nk = pick3(cls, s.k0, s.k1, s.k2);
  if (MODE == kModeBwd && cls != kClsGrad) {
    // dW / dH: the hidden-dimension block varies fastest, so the units that
    // read the same block of the gradient panel (a column strip for dW, a
    // row block for dH) run side by side and share it through L2
    const int nD = cdiv_i(g.D, g.bn_wh);
    un.m0 = (u / nD) * PAIR_M;
    un.n0 = (u % nD) * g.bn_wh;
    un.bn = g.bn_wh;
  } else {
    const int rows = (MODE == kModePlain) ? g.M : C;
    const int nT = cdiv_i(rows, PAIR_M);
    un.m0 = (u % nT) * PAIR_M;
    un.n0 = (u / nT) * BN;
    un.bn = BN;
  }
  return un;
}

template <int MODE>
__device__ __forceinline__ bool unit_a_mn(const GemmArgs& g, const Unit& un) {
  if (MODE == kModeBwd) return un.cls == kClsDW;
  if (MODE == kModePlain) return g.a_mn != 0;
  return false;
}
template <int MODE>
__device__ __forceinline__ bool unit_b_mn(const GemmArgs& g, const Unit& un) {
  if (MODE == kModeBwd) return un.cls != kClsGrad;
  if (MODE == kModePlain) return g.b_mn != 0;
  return false;
}

// Gradient filtering: which k-blocks of a dW / dH unit read any kept box of
// the panel (all of them without filtering).  dH: rows [m0, m0 + 256) are row
// halves m0 / 128 and the next; k-block kb is column box kb.  dW: vocabulary
// ids [m0, m0 + 256) of the panel are boxes m0 / 64 .. + 3; k-block kb covers
// rows [64 kb, 64 kb + 64) of row half kb / 2.  Computed for k-blocks
// kb0 .. kb0 + 31 at once, as a bit mask (bit j: k-block kb0 + j; bits past nk
// are 0): the flags are read with independent loads issued back to back.
template <int MODE, int FEAT>
__device__ __forceinline__ uint32_t active_mask32(const GemmArgs& g, const Unit& un, int kb0) {
  if (MODE != kModeBwd || !(FEAT & kFeatFilter) || un.cls == kClsGrad) return 0xffffffffu;
  uint32_t m = 0;
  if (un.cls == kClsDH) {
    // 32 flag bytes of each of the two row halves, read as 32-bit words (a row
    // holds a multiple of 4 flags, and a word that starts before nk ends
    // inside the row); flag byte k of a word becomes bit k
    const uint32_t* r0 = reinterpret_cast<const uint32_t*>(
        g.keep_wh + static_cast<size_t>(un.m0 / BM) * g.keep_ld + kb0);
    const uint32_t* r1 = reinterpret_cast<const uint32_t*>(
        reinterpret_cast<const uint8_t*>(r0) + g.keep_ld);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t w = (kb0 + 4 * i < un.nk) ? (r0[i] | r1[i]) : 0u;
      const uint32_t b4 = (w & 1u) | ((w >> 7) & 2u) | ((w >> 14) & 4u) | ((w >> 21) & 8u);
      m |= b4 << (4 * i);
    }
    if (un.nk - kb0 < 32) m &= (1u << (un.nk - kb0)) - 1u;
  } else {
    // two k-blocks per row half; four flag bytes (one 32-bit word) per row half
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      w[i] = (kb0 + 2 * i < un.nk)
                 ? *reinterpret_cast<const uint32_t*>(
                       g.keep_wh + static_cast<size_t>((kb0 >> 1) + i) * g.keep_ld + (un.m0 >> 6))
                 : 0u;
#pragma unroll
    for (int i = 0; i < 16; ++i) m |= (w[i] != 0 ? 3u : 0u) << (2 * i);
    if (un.nk - kb0 < 32) m &= (1u << (un.nk - kb0)) - 1u;
  }
  return m;
}

// TMA loads of k-block kb of unit `un` into this CTA's ring stage: its 128
// A rows (16 KiB) and its 128 of the 256 B rows (16 KiB).  Completion is
// counted on the even CTA's barrier `bar_cluster`.
// Which operand boxes a producer thread issues: the backward splits A and B
// between two threads, because issuing a stage's 2-4 boxes from one thread
// takes about as long as the stage's MMAs.
enum LoadPart : int { kLoadA = 0, kLoadB = 1, kLoadAB = 2 };
template <int MODE>
struct LoadSplit {
  static constexpr bool kSplit = MODE == kModeBwd;
};

template <int MODE>
__device__ __forceinline__ void issue_stage_loads(const GemmArgs& g, const Unit& un, int kb,
                                                  uint32_t rank, uint32_t sa, uint32_t sb,
                                                  uint32_t bar_cluster, int part) {
  const int mapi = (MODE == kModeBwd) ? un.cls : 0;
  const CUtensorMap* tA = &g.tmA[mapi];
  const CUtensorMap* tB = &g.tmB[mapi];
  const int k0 = kb * BK;
  const int am0 = un.m0 + static_cast<int>(rank) * BM;       // this CTA's A rows
  const int bn0 = un.n0 + static_cast<int>(rank) * (un.bn / 2);  // this CTA's B rows
  if (part != kLoadB) {
    if (unit_a_mn<MODE>(g, un)) {
      tma_load_2d_pair(sa, tA, bar_cluster, am0, k0);
      tma_load_2d_pair(sa + MN_BOX_BYTES, tA, bar_cluster, am0 + 64, k0);
    } else {
      tma_load_2d_pair(sa, tA, bar_cluster, k0, am0);
    }
  }
  if (part == kLoadA) return;
  if (unit_b_mn<MODE>(g, un)) {
    // dH: the k index is a vocabulary id of the panel
    const int kB = (MODE == kModeBwd && un.cls == kClsDH) ? g.vp_wh + k0 : k0;
    tma_load_2d_pair(sb, tB, bar_cluster, bn0, kB);
    if (un.bn / 2 > 64) tma_load_2d_pair(sb + MN_BOX_BYTES, tB, bar_cluster, bn0 + 64, kB);
  } else {
    // fwd / grad: the row index is a vocabulary id
    const int nrow = (MODE == kModeBwd) ? g.vp_g + bn0 : bn0;
    tma_load_2d_pair(sb, tB, bar_cluster, k0, nrow);
  }
}

// 32 bias values for vocabulary ids col0 .. col0+31 (0 past V).
__device__ __forceinline__ void load_bias32(const uint16_t* b, int col0, int V, bool bf16,
                                            float (&bv)[32]) {
  if (col0 + 32 <= V) {
    const uint4* p = reinterpret_cast<const uint4*>(b + col0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 w = __ldg(p + q);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const uint16_t lo = static_cast<uint16_t>(ws[h] & 0xFFFFu);
        const uint16_t hi = static_cast<uint16_t>(ws[h] >> 16);
        if (bf16) {
          bv[q * 8 + 2 * h] = __uint_as_float(static_cast<uint32_t>(lo) << 16);
          bv[q * 8 + 2 * h + 1] = __uint_as_float(static_cast<uint32_t>(hi) << 16);
        } else {
          bv[q * 8 + 2 * h] = __half2float(__ushort_as_half(lo));
          bv[q * 8 + 2 * h + 1] = __half2float(__ushort_as_half(hi));
        }
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float v = 0.f;
      if (col0 + j < V) {
        const uint16_t u = __ldg(b + col0 + j);
        v = bf16 ? __uint_as_float(static_cast<uint32_t>(u) << 16)
                 : __half2float(__ushort_as_half(u));
      }
      bv[j] = v;
    }
  }
}

// Logits rounded to the 16-bit input type (round to nearest even).
__device__ __forceinline__ void round_to_input_type(const GemmArgs& g, float (&x)[32]) {
  if (g.is_bf16) {
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = __bfloat162float(__float2bfloat16_rn(x[j]));
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = __half2float(__float2half_rn(x[j]));
  }
}

// ---------------------------------------------------------------------------
// Epilogue: forward statistics of one 32-column chunk.
// ---------------------------------------------------------------------------
struct FwdRowState {
  float m;
  float s;
  float tgt;
  bool have_tgt;
};

// 2^x for element j of a chunk: with POLY every fourth on the FMA pipe.
template <bool POLY>
__device__ __forceinline__ float ex2_elem(float x, int j) {
  return (POLY && (j & 3) == 3) ? ex2_poly(x) : ex2_approx(x);
}

template <int FEAT>
__device__ __forceinline__ void fwd_chunk(const GemmArgs& g, uint32_t (&z)[32], int cb, int vglob0,
                                          int vlim, int yl, FwdRowState& st) {
  constexpr bool POLY = (FEAT & kFeatPolyExp) != 0;
  float x[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(z[j]);
  if (FEAT & kFeatBias) {
    float bv[32];
    load_bias32(g.bias, vglob0 + cb, g.V, g.is_bf16 != 0, bv);
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] += bv[j];
  }
  if (FEAT & kFeatRound) round_to_input_type(g, x);
  if (cb + 32 > vlim) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (cb + j >= vlim) x[j] = -INFINITY;
  }
  // chunk max as a tree of three-input maxima (17 operations, depth 4)
  float t[11];
#pragma unroll
  for (int j = 0; j < 10; ++j) t[j] = fmax3(x[3 * j], x[3 * j + 1], x[3 * j + 2]);
  t[10] = fmaxf(x[30], x[31]);
  const float u0 = fmax3(t[0], t[1], t[2]), u1 = fmax3(t[3], t[4], t[5]),
              u2 = fmax3(t[6], t[7], t[8]), u3 = fmaxf(t[9], t[10]);
  const float cm = fmaxf(fmax3(u0, u1, u2), u3);
  const float mn = fmaxf(st.m, cm);
  // nothing seen yet and this chunk is all padding (a half tile past V): the
  // state stays (-inf, 0) instead of exp(-inf + inf)
  if (mn == -INFINITY) return;
  const float nb = -mn * kLog2e;
  // four running sums, two per packed pair
  const float2 l2 = make_float2(kLog2e, kLog2e), nb2 = make_float2(nb, nb);
  float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float2 y01 = ffma2(make_float2(x[j], x[j + 1]), l2, nb2);
    const float2 y23 = ffma2(make_float2(x[j + 2], x[j + 3]), l2, nb2);
    a01 = fadd2(a01, make_float2(ex2_approx(y01.x), ex2_approx(y01.y)));
    a23 = fadd2(a23, make_float2(ex2_approx(y23.x), ex2_elem<POLY>(y23.y, j + 3)));
  }
  // first chunk: st.m = -inf, the old sum is scaled by exp(-inf) = 0
  st.s = st.s * ex2_approx((st.m - mn) * kLog2e) + ((a01.x + a01.y) + (a23.x + a23.y));
  st.m = mn;
  const int jt = yl - cb;
  if (static_cast<unsigned>(jt) < 32u) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j == jt) st.tgt = x[j];
    st.have_tgt = true;
  }
}

// Column sums over a warp's 32 rows of a 32-column chunk: a butterfly that
// halves the columns a lane holds at each step, so that lane j ends with
// column j's sum.  The order of the additions is fixed.
__device__ __forceinline__ float warp_column_sums(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

// ---------------------------------------------------------------------------
// Epilogue: gradient-panel values of one 32-column chunk, packed to 16 bits.
// ---------------------------------------------------------------------------
// krow is log2(sigma) - (log s) log2(e) - m log2(e) for the row, so that
// sigma p = 2^(z log2(e) + krow) takes one FMA per entry.  FOLDED: the row is
// supervised and its scale r positive, and krow already holds log2(r) as
// well, so that the entry is r sigma p at once (no selection on `valid`, no
// product with r) and the one-hot term is r sigma.
template <int FEAT, bool FOLDED = false>
__device__ __forceinline__ void grad_chunk(const GemmArgs& g, uint32_t (&z)[32], int cb,
                                           int vglob0, int vlim, int yl, bool valid,
                                           float krow, float rrow, int row, int lane,
                                           uint32_t (&packed)[16], bool& big) {
  float x[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(z[j]);
  if (FEAT & kFeatBias) {
    float bv[32];
    load_bias32(g.bias, vglob0 + cb, g.V, g.is_bf16 != 0, bv);
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] += bv[j];
  }
  if (FEAT & kFeatRound) round_to_input_type(g, x);
  float gv[32];
  // sigma * p = 2^( ((z - m) - log s) * log2(e) + log2(sigma) )
  if (FOLDED) {
    const float2 l2 = make_float2(kLog2e, kLog2e), k2 = make_float2(krow, krow);
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const float2 y = ffma2(make_float2(x[j], x[j + 1]), l2, k2);
      gv[j] = ex2_approx(y.x);
      gv[j + 1] = ex2_approx(y.y);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) gv[j] = ex2_approx(fmaf(x[j], kLog2e, krow));
  }
  if (!FOLDED && !valid) {
#pragma unroll
    for (int j = 0; j < 32; ++j) gv[j] = 0.f;
  }
  if (cb + 32 > vlim) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (cb + j >= vlim) gv[j] = 0.f;
  }
  const int jt = yl - cb;
  if (static_cast<unsigned>(jt) < 32u) {
    const float onehot = FOLDED ? g.sigma * rrow : g.sigma;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j == jt) gv[j] -= onehot;
  }
  if (FEAT & kFeatFilter) {
    // gradient filtering: does this row hold an entry that is not negligible?
#pragma unroll
    for (int j = 0; j < 32; ++j) big |= fabsf(gv[j]) >= g.filter_eps_sigma;
  }
  if (!FOLDED) {
#pragma unroll
    for (int j = 0; j < 32; ++j) gv[j] *= rrow;  // the row's scale relative to S
  }
  // The target entry r (p - 1) sigma dominates its row of dH; keep what the
  // 16-bit rounding takes off it so that dH can add it back in fp32.
  if (valid && static_cast<unsigned>(jt) < 32u) {
    float resid = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j == jt)
        resid = gv[j] - (g.is_bf16 ? __bfloat162float(__float2bfloat16_rn(gv[j]))
                                   : __half2float(__float2half_rn(gv[j])));
    g.tgt_resid[row] = resid;
  }
  if (g.is_bf16) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(gv[2 * j], gv[2 * j + 1]);
      packed[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const __half2 h = __floats2half2_rn(gv[2 * j], gv[2 * j + 1]);
      packed[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  if (FEAT & kFeatBias) {
    // bias gradient: this warp's 32 rows of the chunk, in fp32 (target
    // entries included exactly), added as 2^-32 fixed-point integers
    const float cs = warp_column_sums(gv, lane);
    if (cb + lane < vlim) {
      const long long q = __float2ll_rn(cs * g.db_fx_scale);
      atomicAdd(g.db_acc + vglob0 + cb + lane, static_cast<unsigned long long>(q));
    }
  }
}

// Writes 128 bytes of this thread's row into a 128-row staging box laid out
// as the 128-byte-swizzled TMA box (16-byte chunk j of row r sits at chunk
// j ^ (r & 7)).
template <int NW>
__device__ __forceinline__ void stage_row128(uint8_t* stg, int r, int chunk0,
                                             const uint32_t (&w)[NW]) {
  uint8_t* rowp = stg + r * 128;
#pragma unroll
  for (int j = 0; j < NW / 4; ++j) {
    const int c = (chunk0 + j) ^ (r & 7);
    *reinterpret_cast<uint4*>(rowp + c * 16) =
        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  }
}

// ---------------------------------------------------------------------------
// The kernel (launched as clusters of 2 CTAs)
// ---------------------------------------------------------------------------
template <int MODE, int FEAT = 0>
__global__ void __launch_bounds__((Shape<MODE, FEAT>::THREADS), 1)
    flce_gemm_kernel(const __grid_constant__ GemmArgs g) {
  using SH = Shape<MODE, FEAT>;
  using CFG = typename SH::Cfg;
  constexpr int STAGES = CFG::STAGES;
  constexpr int EPI_THREADS = SH::EPI_THREADS;
  constexpr int CHUNKS = SH::CHUNKS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_STAGE_BYTES;
  uint8_t* sStg = sB + STAGES * B_STAGE_BYTES;
  float2* sMerge = reinterpret_cast<float2*>(sStg + CFG::STAGING);  // forward only
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + CFG::STAGING + CFG::MERGE);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* uq_full = tempty + 2;
  uint64_t* uq_empty = uq_full + UQ;
  uint64_t* done_bar = uq_empty + UQ;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* decision = abort_flag + 1;  // [2]
  volatile int* s_unit = decision + 2;      // [UQ]
  volatile int* s_keep = s_unit + UQ;       // [EPI_THREADS / 32]: filtering votes per warp

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that schedules and issues MMAs
  const bool leader = rank == 0;
  // Barriers that only the even CTA uses are counted there; the odd CTA
  // reaches them through shared::cluster addresses.
  auto leader_addr = [&](const void* p) -> uint32_t {
    return leader ? smem_addr(p) : mapa_shared(smem_addr(p), 0);
  };
  auto arrive_on_leader = [&](uint64_t* bar) {
    if (leader)
      mbar_arrive(bar);
    else
      mbar_arrive_cluster_release_cta(mapa_shared(smem_addr(bar), 0));
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // even CTA: its expect_tx arrival + both CTAs' bytes
      mbar_init(&empty[s], 1);  // one multicast MMA commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);                           // one multicast MMA commit
      mbar_init(&tempty[a], 2 * EPI_THREADS / 32);   // one lane per epilogue warp, both CTAs
    }
    for (int q = 0; q < UQ; ++q) {
      mbar_init(&uq_full[q], 1);
      // even CTA: its MMA lane and epilogue warps; odd CTA: its producer and epilogue warps
      // + the second producer of each CTA when the loads are split
      mbar_init(&uq_empty[q], 2 * (1 + EPI_THREADS / 32) + (LoadSplit<MODE>::kSplit ? 2 : 0));
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    decision[0] = 0;
    decision[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    const int nmaps = (MODE == kModeBwd) ? 3 : 1;
    for (int i = 0; i < nmaps; ++i) {
      tma_prefetch_map(&g.tmA[i]);
      tma_prefetch_map(&g.tmB[i]);
    }
    if (MODE == kModeBwd) {
      tma_prefetch_map(&g.tmG);
      tma_prefetch_map(&g.tmDW);
      tma_prefetch_map(&g.tmDH);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int C = (MODE == kModePlain) ? g.M : *g.C_dev;
  const UnitSpace us = make_unit_space<MODE>(g, C);

  if (warp < EPI_WARP0) {
    setmaxnreg_dec<SH::REGS_LOW>();  // the whole first warpgroup
    if (warp == 0 || (LoadSplit<MODE>::kSplit && warp == 2)) {
      // ------------------------------------------------------------ scheduler + producers
      // warp 0: the scheduler (even CTA) and the A loads (all loads when not split);
      // warp 2: the B loads when split
      const int part = !LoadSplit<MODE>::kSplit ? kLoadAB : (warp == 0 ? kLoadA : kLoadB);
      const bool scheduler = leader && warp == 0;
      if (lane == 0) {
        uint32_t n_issued = 0;
        bool ok = true;
        // backward: whether this thread has waited for the previous launch
        // (which may still run) and let the next one start
        bool dep_done = MODE != kModeBwd;
        const uint32_t full_c0 = leader_addr(&full[0]);
        for (int it = 0; ok; ++it) {
          const int slot = it % UQ;
          const uint32_t ph = (it / UQ) & 1;
          int u;
          if (scheduler) {
            if (!mbar_wait(&uq_empty[slot], ph ^ 1u, abort_flag, g.err)) break;
            u = atomicAdd(g.counter, 1);
            if (u >= us.total) u = -1;
            s_unit[slot] = u;
            st_shared_cluster_u32(mapa_shared(smem_addr(const_cast<int*>(&s_unit[slot])), 1),
                                  static_cast<uint32_t>(u));
            mbar_arrive(&uq_full[slot]);
            mbar_arrive_cluster(mapa_shared(smem_addr(&uq_full[slot]), 1));
          } else {
            const bool got = leader ? mbar_wait(&uq_full[slot], ph, abort_flag, g.err)
                                    : mbar_wait_cluster(&uq_full[slot], ph, abort_flag, g.err);
            if (!got) break;
            u = s_unit[slot];
            arrive_on_leader(&uq_empty[slot]);
          }
          if (u < 0) break;
          const Unit un = decode_unit<MODE>(g, us, C, u);
          if (MODE == kModeBwd && !dep_done && un.cls != kClsGrad) {
            // dW / dH read the panel the previous launch wrote and add to the
            // dH tiles it added to: wait for it to complete.  Only then may
            // the next launch start (its gradient units overwrite the panel
            // buffer that the launch before the previous one read).
            griddep_wait();
            griddep_launch_dependents();
            dep_done = true;
          }
          uint32_t act = 0;
          for (int kb = 0; kb < un.nk; ++kb) {
            if (FEAT & kFeatFilter) {
              if ((kb & 31) == 0) act = active_mask32<MODE, FEAT>(g, un, kb);
              if (!((act >> (kb & 31)) & 1u)) continue;
            }
            const uint32_t stage = n_issued % STAGES;
            const uint32_t phase = (n_issued / STAGES) & 1u;
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, g.err)) {
              ok = false;
              break;
            }
            // one arrival (with both CTAs' bytes) per stage, from the scheduler
            if (scheduler) mbar_arrive_expect_tx(&full[stage], pair_tx_bytes(un.bn));
            issue_stage_loads<MODE>(g, un, kb, rank, smem_addr(sA + stage * A_STAGE_BYTES),
                                    smem_addr(sB + stage * B_STAGE_BYTES),
                                    full_c0 + stage * static_cast<uint32_t>(sizeof(uint64_t)),
                                    part);
            ++n_issued;
          }
        }
        if (!dep_done) {
          griddep_wait();
          griddep_launch_dependents();
        }
        // The even CTA lets every copy still in flight (its own and its peer's,
        // both producers') land before the pair can exit.
        if (scheduler) {
          const uint32_t first = n_issued > STAGES ? n_issued - STAGES : 0u;
          for (uint32_t i = first; i < n_issued; ++i)
            mbar_wait(&full[i % STAGES], (i / STAGES) & 1u, nullptr, nullptr, kDrainLimitNs);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer (even CTA)
      if (lane == 0 && leader) {
        uint32_t n_used = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int it = 0;; ++it) {
          const int slot = it % UQ;
          if (!mbar_wait(&uq_full[slot], (it / UQ) & 1, abort_flag, g.err)) break;
          const int u = s_unit[slot];
          mbar_arrive(&uq_empty[slot]);
          if (u < 0) break;
          const Unit un = decode_unit<MODE>(g, us, C, u);
          // the filtering flags of the panel being read come from the previous launch
          if (MODE == kModeBwd && (FEAT & kFeatFilter) && un.cls != kClsGrad) griddep_wait();
          if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, g.err)) break;
          tc_fence_after();
          const bool a_mn = unit_a_mn<MODE>(g, un);
          const bool b_mn = unit_b_mn<MODE>(g, un);
          const uint32_t idesc = make_idesc_f16(g.is_bf16 != 0, a_mn, b_mn, PAIR_M, un.bn);
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
          const uint32_t a_lbo = a_mn ? MN_BOX_BYTES : 16u;
          const uint32_t b_lbo = b_mn ? MN_BOX_BYTES : 16u;
          const uint32_t a_step = a_mn ? 16u * 128u : 32u;  // bytes per K=16 slice
          const uint32_t b_step = b_mn ? 16u * 128u : 32u;
          bool ok = true;
          bool first = true;  // the first k-block issued overwrites the accumulator
          uint32_t act = 0;
          for (int kb = 0; kb < un.nk; ++kb) {
            if (FEAT & kFeatFilter) {
              if ((kb & 31) == 0) act = active_mask32<MODE, FEAT>(g, un, kb);
              if (!((act >> (kb & 31)) & 1u)) continue;
            }
            const uint32_t stage = n_used % STAGES;
            const uint32_t phase = (n_used / STAGES) & 1u;
            if (!mbar_wait(&full[stage], phase, abort_flag, g.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_addr(sA + stage * A_STAGE_BYTES);
            const uint32_t sb = smem_addr(sB + stage * B_STAGE_BYTES);
  #pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = smem_desc_sw128(sa + kk * a_step, a_lbo, 1024u);
              const uint64_t bd = smem_desc_sw128(sb + kk * b_step, b_lbo, 1024u);
              umma_f16_pair(d_tmem, ad, bd, idesc, (!first || kk > 0) ? 1u : 0u);
            }
            first = false;
            umma_commit_pair_mc(&empty[stage], 0x3);  // frees the stage in both CTAs
            ++n_used;
          }
          if (!ok) break;
          umma_commit_pair_mc(&tfull[acc], 0x3);  // accumulator ready in both CTAs
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
        // All pair MMAs complete before either CTA releases its TMEM.
        umma_commit_pair_mc(done_bar, 0x1);
        mbar_wait(done_bar, 0, nullptr, nullptr, kDrainLimitNs);
      }
    }
  } else {
    setmaxnreg_inc<SH::REGS_HIGH>();  // each epilogue warpgroup
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;         // row within this CTA's half of the tile
    const int rbase = static_cast<int>(rank) * BM;
    const int epi_tid = threadIdx.x - EPI_WARP0 * 32;
    const int wg = epi_tid / EPI_WG_THREADS;   // epilogue warpgroup: its CHUNKS 32-column chunks
    const int wtid = epi_tid % EPI_WG_THREADS;
    const int c0 = wg * CHUNKS;                // first 32-column chunk of this warpgroup
    const uint32_t wg_bar = 2 + static_cast<uint32_t>(wg);  // named barrier of this warpgroup
    uint8_t* stg = sStg + wg * STG_BYTES;      // this warpgroup's staging box (backward)
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int acc = 0;
    uint32_t acc_phase = 0;
    float wh_scale = 0.f;
    if (MODE == kModeBwd) wh_scale = (C > 0) ? *g.scal * g.inv_sigma : 0.f;
    // Shared decision of the epilogue warps (they pass named barriers
    // together, so they leave the loop together).
    int round = 0;
    auto decide_abort = [&]() -> bool {
      named_bar_sync(1, EPI_THREADS);
      if (epi_tid == 0) decision[round & 1] = *abort_flag;
      named_bar_sync(1, EPI_THREADS);
      return decision[(round++) & 1] != 0;
    };
    // Stages one 128 x 128-byte box in this warpgroup's staging buffer and
    // hands it to the TMA engine.
    auto emit_box = [&](const uint32_t (&w)[32], const CUtensorMap* map, int x, int y,
                        bool reduce, bool issue) {
      if (wtid == 0) bulk_wait_group_read<0>();  // the previous box has left the buffer
      named_bar_sync(wg_bar, EPI_WG_THREADS);
      stage_row128(stg, r, 0, w);
      fence_proxy_async_smem();
      named_bar_sync(wg_bar, EPI_WG_THREADS);
      if (wtid == 0) {
        if (issue) {
          if (reduce)
            tma_reduce_add_2d(map, smem_addr(stg), x, y);
          else
            tma_store_2d(map, smem_addr(stg), x, y);
        }
        bulk_commit_group();
      }
    };

    for (int it = 0;; ++it) {
      const int slot = it % UQ;
      const bool got = leader ? mbar_wait(&uq_full[slot], (it / UQ) & 1, abort_flag, g.err)
                              : mbar_wait_cluster(&uq_full[slot], (it / UQ) & 1, abort_flag, g.err);
      const int u = got ? s_unit[slot] : -1;
      __syncwarp();
      if (lane == 0) arrive_on_leader(&uq_empty[slot]);
      if (decide_abort() || u < 0) break;
      const Unit un = decode_unit<MODE>(g, us, C, u);
      const int tm0 = un.m0 + rbase;  // first row of this CTA's half

      // per-row data, fetched before waiting for the accumulator
      const int row = tm0 + r;
      bool valid = false;
      int yl = -1000000;
      float mrow = 0.f, krow = 0.f, rrow = 0.f;
      int vglob0 = 0, vlim = 0;
      if (MODE == kModeFwd || (MODE == kModeBwd && un.cls == kClsGrad)) {
        valid = row < C;
        vglob0 = (MODE == kModeBwd ? g.vp_g : 0) + un.n0;
        vlim = g.V - vglob0;
        if (valid) yl = __ldg(g.y_c + row) - vglob0;
        if (MODE == kModeBwd && valid) {
          const int o = __ldg(g.idx + row);
          mrow = __ldg(g.m_saved + o);
          krow = fmaf(-mrow, kLog2e, g.log2_sigma - __ldg(g.logs_saved + o) * kLog2e);
          rrow = __ldg(g.row_scale + row);
        }
      } else if (MODE == kModePlain) {
        valid = row < g.M;
      }

      mbar_wait(&tfull[acc], acc_phase, abort_flag, g.err);
      // The small-D forward, bound by its epilogue, decides once per unit (a
      // wait that gives up raises the abort flag; the warps finish the unit
      // with whatever TMEM holds and leave together at the next unit's
      // decision): measured 3-8 % off that forward, and within the noise
      // elsewhere, where the second decision stays.
      if constexpr (!SH::WIDE) {
        if (decide_abort()) break;
      }
      tc_fence_after();
      const uint32_t t_acc = lane_base + static_cast<uint32_t>(acc * BN);

      if (MODE == kModeFwd) {
        // (m, s) of this warpgroup's columns.  Chunks stream out of TMEM
        // two at a time (one loading while the other is reduced); the
        // accumulator goes back to the MMA issuer after the last chunk's
        // arithmetic.  (Measured slower: reading all four chunks first, 8 %
        // on the forward at D = 64 and 128; releasing the accumulator right
        // after its last read, 2 % here and 2 % on the backward.)
        FwdRowState st{-INFINITY, 0.f, 0.f, false};
        uint32_t za[32];
        if constexpr (SH::WIDE) {
          // four warpgroups: one chunk in flight per thread (the other warps
          // hide the load), which keeps the epilogue within its registers
#pragma unroll 1
          for (int c = c0; c < c0 + CHUNKS; ++c) {
            tmem_ld32(t_acc + c * 32, za);
            tmem_wait_ld(za);
            fwd_chunk<FEAT>(g, za, c * 32, vglob0, vlim, yl, st);
          }
        } else {
          uint32_t zb[32];
          tmem_ld32(t_acc + c0 * 32, za);
          tmem_wait_ld(za);
#pragma unroll 1
          for (int c = c0; c < c0 + CHUNKS; c += 2) {
            tmem_ld32(t_acc + (c + 1) * 32, zb);
            fwd_chunk<FEAT>(g, za, c * 32, vglob0, vlim, yl, st);
            tmem_wait_ld(zb);
            if (c + 2 < c0 + CHUNKS) tmem_ld32(t_acc + (c + 2) * 32, za);
            fwd_chunk<FEAT>(g, zb, (c + 1) * 32, vglob0, vlim, yl, st);
            if (c + 2 < c0 + CHUNKS) tmem_wait_ld(za);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_on_leader(&tempty[acc]);
        if (valid && st.have_tgt) g.tgt[row] = st.tgt;
        // the other warpgroups' slices of the row join the first's, in
        // warpgroup order: one partial per row and tile, stored tile-major
        // (coalesced per warp).  The buffer is reused only after the next
        // unit's decide_abort, which all warpgroups pass together.
        if (wg > 0) sMerge[(wg - 1) * BM + r] = make_float2(st.m, st.s);
        named_bar_sync(8, EPI_THREADS);
        if (wg == 0) {
#pragma unroll
          for (int k = 0; k < SH::EPI_WG - 1; ++k) {
            const float2 o = sMerge[k * BM + r];
            const float mn = fmaxf(st.m, o.x);
            if (mn != -INFINITY) {
              st.s = st.s * ex2_approx((st.m - mn) * kLog2e) +
                     o.y * ex2_approx((o.x - mn) * kLog2e);
              st.m = mn;
            }
          }
          if (valid)
            g.part[static_cast<size_t>(un.n0 / BN) * g.part_ld + row] = make_float2(st.m, st.s);
        }
      } else if (MODE == kModeBwd && un.cls == kClsGrad) {
        // Chunks stream out of TMEM two at a time (registers allow no more);
        // the accumulator is handed back after the last box.
        uint32_t za[32], zb[32];
        tmem_ld32(t_acc + c0 * 32, za);
        tmem_wait_ld(za);
#pragma unroll 1
        for (int c = c0; c < c0 + CHUNKS; c += 2) {
          // chunks c, c+1 form one 64-column box of the 16-bit panel
          if (wtid == 0) bulk_wait_group_read<0>();  // the previous box has left the buffer
          named_bar_sync(wg_bar, EPI_WG_THREADS);
          tmem_ld32(t_acc + (c + 1) * 32, zb);
          uint32_t pk[16];
          bool big = false;
          grad_chunk<FEAT>(g, za, c * 32, vglob0, vlim, yl, valid, krow, rrow, row, lane, pk, big);
          stage_row128(stg, r, 0, pk);
          tmem_wait_ld(zb);
          if (c + 2 < c0 + CHUNKS) tmem_ld32(t_acc + (c + 2) * 32, za);
          grad_chunk<FEAT>(g, zb, (c + 1) * 32, vglob0, vlim, yl, valid, krow, rrow, row, lane, pk,
                     big);
          stage_row128(stg, r, 4, pk);
          if (c + 2 < c0 + CHUNKS) tmem_wait_ld(za);
          fence_proxy_async_smem();
          if (FEAT & kFeatFilter) {
            const bool any = __any_sync(0xffffffffu, big);
            if (lane == 0) s_keep[wg * 4 + q] = any ? 1 : 0;
          }
          named_bar_sync(wg_bar, EPI_WG_THREADS);
          if (FEAT & kFeatFilter) {
            // gradient filtering: the box (this warpgroup's 128 rows x 64
            // columns) is kept when any of its entries is not negligible;
            // a dropped box is stored as zeros, and the target entries it
            // holds lose their fp32 residual as well
            const int* sk = const_cast<const int*>(s_keep) + wg * 4;
            const bool keep = (sk[0] | sk[1] | sk[2] | sk[3]) != 0;
            if (!keep) {
              const uint32_t zw[32] = {};
              stage_row128(stg, r, 0, zw);
              if (valid && static_cast<unsigned>(yl - c * 32) < 64u) g.tgt_resid[row] = 0.f;
              fence_proxy_async_smem();
              named_bar_sync(wg_bar, EPI_WG_THREADS);
            }
            if (wtid == 0)
              g.keep_g[static_cast<size_t>(tm0 / BM) * g.keep_ld + (un.n0 + c * 32) / 64] =
                  keep ? 1 : 0;
          }
          if (wtid == 0) {
            // a box that starts past the panel's last column holds only padding
            if (un.n0 + c * 32 < g.w_g) tma_store_2d(&g.tmG, smem_addr(stg), un.n0 + c * 32, tm0);
            bulk_commit_group();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_on_leader(&tempty[acc]);
      } else if (MODE == kModeBwd) {
        // dW (class 0) or dH (class 1): fp32, scaled by lambda / (C sigma)
        const bool is_dw = un.cls == kClsDW;
        const CUtensorMap* map = is_dw ? &g.tmDW : &g.tmDH;
        const int y = is_dw ? g.vp_wh + tm0 : tm0;
        const bool reduce = !is_dw && g.dh_accumulate;
        bool zero = (un.nk == 0);
        if ((FEAT & kFeatFilter) && !zero) {
          // with filtering, no MMA ran when every k-block was skipped: the
          // warp scans the unit's flags (from the previous launch)
          griddep_wait();
          bool any = false;
          for (int kb0 = 32 * lane; kb0 < un.nk && !any; kb0 += 32 * 32)
            any = active_mask32<MODE, FEAT>(g, un, kb0) != 0;
          zero = !__any_sync(0xffffffffu, any);
        }
        // a dW half that starts past the panel's last row has nothing to store;
        // adding a zero tile to dH changes nothing
        const bool issue = (!is_dw || tm0 < g.w_wh) && !(zero && reduce);
        // this warpgroup's chunks [c0, ce) of the ones inside D
        const int ce = min(c0 + CHUNKS, cdiv_i(g.D - un.n0, 32));
        const int nch = ce;
        uint32_t za[32], zb[32], w[32];
        if (!zero && c0 < ce) {
          tmem_ld32(t_acc + c0 * 32, za);
          tmem_wait_ld(za);
        }
#pragma unroll 1
        for (int c = c0; c < ce; c += 2) {
          // za holds chunk c; chunk c+1 loads into zb meanwhile
          if (!zero && c + 1 < nch) tmem_ld32(t_acc + (c + 1) * 32, zb);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            w[j] = zero ? 0u : __float_as_uint(__uint_as_float(za[j]) * wh_scale);
          emit_box(w, map, un.n0 + c * 32, y, reduce, issue);
          if (c + 1 < nch) {
            if (!zero) tmem_wait_ld(zb);
            if (!zero && c + 2 < nch) tmem_ld32(t_acc + (c + 2) * 32, za);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              w[j] = zero ? 0u : __float_as_uint(__uint_as_float(zb[j]) * wh_scale);
            emit_box(w, map, un.n0 + (c + 1) * 32, y, reduce, issue);
            if (!zero && c + 2 < nch) tmem_wait_ld(za);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_on_leader(&tempty[acc]);
      } else {  // kModePlain
#pragma unroll 1
        for (int c = c0; c < c0 + CHUNKS; ++c) {
          const int col0 = un.n0 + c * 32;
          if (col0 >= g.ncols) break;
          uint32_t z[32];
          tmem_ld32(t_acc + c * 32, z);
          tmem_wait_ld(z);
          if (valid) {
            float* dst = g.out + static_cast<size_t>(row) * g.ncols + col0;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < g.ncols) dst[j] = __uint_as_float(z[j]) * g.scale;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_on_leader(&tempty[acc]);
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (MODE == kModeBwd && wtid == 0) bulk_wait_group<0>();
  }

  // Neither CTA frees its TMEM (or exits) while the pair still uses it.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace flce
