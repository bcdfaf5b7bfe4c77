// Persistent, warp-specialised tcgen05 GEMM for sm_100a with the fused
// epilogues of exact linear cross-entropy.
//
// One CTA per SM.  Warp 0 (one lane) streams operand tiles with TMA into a
// STAGES-deep shared-memory ring; warp 1 (one lane) issues
// tcgen05.mma.kind::f16 (M=128, N=256, K=16) into one of two 128x256 f32
// accumulators in TMEM (512 columns); warps 4..7 read the finished
// accumulator back with tcgen05.ld (thread = TMEM lane = tile row) and run
// the epilogue while the next tile accumulates in the other buffer.
//
// Modes (one launch = one mode):
//   kModeFwd   Z = H_c W^T (+ b) per 128 x 256 tile; the epilogue keeps the
//              running max / rescaled exp-sum over the tile's columns and
//              captures the target logit from the tile that holds it
//              ("分块交叉熵" page, §02), writing one (m, s) partial per row
//              and vocabulary tile.
//   kModeGrad  the same tile recomputed for the backward; the epilogue
//              rebuilds p = exp((Z - m) - log s) from the saved statistics,
//              subtracts the one-hot target (§04), rounds to the 16-bit
//              input type, stages the tile in shared memory and stores it
//              with TMA into a C x Vc gradient panel.
//   kModeWH    one launch with two unit classes fed by the same panel:
//              class 0: dW[panel rows] = G_panel^T H_c   (K = C)
//              class 1: dH[idx] (+)= G_panel W[panel]    (K = panel width)
//              every output tile is owned by one unit, so both are
//              deterministic; dH accumulates over panels in panel order.
//   kModePlain diagnostic: out = scale * A B^T with a plain store.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace flce {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr uint32_t A_STAGE_BYTES = BM * BK * 2;  // 16 KiB
constexpr uint32_t B_STAGE_BYTES = BN * BK * 2;  // 32 KiB
constexpr uint32_t MN_BOX_BYTES = 64 * BK * 2;   // 8 KiB: 64 MN-elements x 64 K rows
constexpr uint32_t STG_BYTES = BM * 64 * 2;      // 16 KiB: 128 rows x 64 16-bit columns
constexpr int NUM_THREADS = 256;
constexpr int EPI_WARP0 = 4;
constexpr int NUM_EPI_THREADS = 128;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr float kLog2e = 1.4426950408889634f;
constexpr size_t GEMM_SMEM_BYTES =
    1024 + STAGES * (A_STAGE_BYTES + B_STAGE_BYTES) + 2 * STG_BYTES + 256;

enum GemmMode : int { kModeFwd = 0, kModeGrad = 1, kModeWH = 2, kModePlain = 3 };

struct GemmArgs {
  CUtensorMap tmA[2];  // A operand map of unit class 0 / 1
  CUtensorMap tmB[2];  // B operand map of unit class 0 / 1
  CUtensorMap tmOut;   // gradient panel store map (kModeGrad)
  int a_mn;            // kModePlain: A is MN-major
  int b_mn;            // kModePlain: B is MN-major
  int is_bf16;
  const int* C_dev;    // supervised-row count (device); unused in kModePlain
  int M;               // kModePlain: rows of out
  int ncols;           // fwd: V; grad: panel width; plain: N
  int K;               // fwd/grad: D; plain: K; wh: panel width
  int D;
  int V;
  int vp;              // first vocabulary id of the panel (grad, wh); 0 for fwd
  int nDW;             // wh: number of dW units
  int nVb;             // wh: 128-row blocks in the panel
  // epilogue data
  const int* y_c;              // compact labels
  const int* idx;              // compact row -> original row
  const uint16_t* bias;        // 16-bit bias [V] or null
  float2* part;                // fwd: (m, s) partials [rows][part_ld]
  int part_ld;
  float* tgt;                  // fwd: target logits [rows]
  const float* m_saved;        // grad: saved statistics [N]
  const float* logs_saved;
  float log2_sigma;            // grad: the panel holds (p - onehot) * sigma
  float sigma;
  float lam;                   // wh: upstream gradient
  const float* lam_dev;        //     (device copy, overrides lam when set)
  float inv_sigma;
  float* dW;
  float* dH;
  float* out;                  // plain
  float scale;                 // plain
  uint32_t* err;
};

struct Unit {
  int cls;
  int m0;
  int n0;
  int nk;
};

__device__ __forceinline__ int cdiv_i(int a, int b) { return (a + b - 1) / b; }

template <int MODE>
__device__ __forceinline__ int num_units(const GemmArgs& g, int C) {
  if (MODE == kModeWH) return g.nDW + cdiv_i(C, BM) * cdiv_i(g.D, BN);
  const int rows = (MODE == kModePlain) ? g.M : C;
  return cdiv_i(rows, BM) * cdiv_i(g.ncols, BN);
}

// Unit u -> tile.  Token (row) tiles vary fastest so that CTAs running at the
// same time share the W / G columns they read through L2.
template <int MODE>
__device__ __forceinline__ Unit decode_unit(const GemmArgs& g, int C, int u) {
  Unit un;
  if (MODE == kModeWH) {
    if (u < g.nDW) {
      un.cls = 0;
      un.m0 = (u % g.nVb) * BM;
      un.n0 = (u / g.nVb) * BN;
      un.nk = cdiv_i(C, BK);
    } else {
      const int v = u - g.nDW;
      const int nT = cdiv_i(C, BM);
      un.cls = 1;
      un.m0 = (v % nT) * BM;
      un.n0 = (v / nT) * BN;
      un.nk = cdiv_i(g.K, BK);
    }
  } else {
    const int rows = (MODE == kModePlain) ? g.M : C;
    const int nT = cdiv_i(rows, BM);
    un.cls = 0;
    un.m0 = (u % nT) * BM;
    un.n0 = (u / nT) * BN;
    un.nk = cdiv_i(g.K, BK);
  }
  return un;
}

template <int MODE>
__device__ __forceinline__ bool unit_a_mn(const GemmArgs& g, const Unit& un) {
  if (MODE == kModeWH) return un.cls == 0;
  if (MODE == kModePlain) return g.a_mn != 0;
  return false;
}
template <int MODE>
__device__ __forceinline__ bool unit_b_mn(const GemmArgs& g, const Unit& un) {
  if (MODE == kModeWH) return true;
  if (MODE == kModePlain) return g.b_mn != 0;
  return false;
}

// TMA loads of k-block kb of unit `un` into one ring stage (48 KiB in total).
template <int MODE>
__device__ __forceinline__ void issue_stage_loads(const GemmArgs& g, const Unit& un, int kb,
                                                  uint32_t sa, uint32_t sb, uint64_t* bar) {
  const CUtensorMap* tA = &g.tmA[un.cls];
  const CUtensorMap* tB = &g.tmB[un.cls];
  const int k0 = kb * BK;
  const bool a_mn = unit_a_mn<MODE>(g, un);
  const bool b_mn = unit_b_mn<MODE>(g, un);
  // A: 128 rows x 64 k
  if (a_mn) {
    tma_load_2d(sa, tA, bar, un.m0, k0);
    tma_load_2d(sa + MN_BOX_BYTES, tA, bar, un.m0 + 64, k0);
  } else {
    tma_load_2d(sa, tA, bar, k0, un.m0);
  }
  // B: 256 rows x 64 k.  In the wh mode's dH class the k index is a vocabulary
  // id of the panel; in fwd/grad the row index is.
  const int kB = (MODE == kModeWH && un.cls == 1) ? g.vp + k0 : k0;
  if (b_mn) {
#pragma unroll
    for (int j = 0; j < 4; ++j) tma_load_2d(sb + j * MN_BOX_BYTES, tB, bar, un.n0 + 64 * j, kB);
  } else {
    const int nrow = (MODE == kModeFwd || MODE == kModeGrad) ? g.vp + un.n0 : un.n0;
    tma_load_2d(sb, tB, bar, k0, nrow);
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

// ---------------------------------------------------------------------------
// Epilogue: forward statistics of one 32-column chunk.
// ---------------------------------------------------------------------------
struct FwdRowState {
  float m;
  float s;
  float tgt;
  bool have_tgt;
};

__device__ __forceinline__ void fwd_chunk(const GemmArgs& g, uint32_t (&z)[32], int cb, int vglob0,
                                          int vlim, int yl, FwdRowState& st) {
  float x[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(z[j]);
  if (g.bias != nullptr) {
    float bv[32];
    load_bias32(g.bias, vglob0 + cb, g.V, g.is_bf16 != 0, bv);
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] += bv[j];
  }
  if (cb + 32 > vlim) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (cb + j >= vlim) x[j] = -INFINITY;
  }
  float cm = x[0];
#pragma unroll
  for (int j = 1; j < 32; ++j) cm = fmaxf(cm, x[j]);
  const float mn = fmaxf(st.m, cm);
  const float nb = -mn * kLog2e;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    a0 += ex2_approx(fmaf(x[j], kLog2e, nb));
    a1 += ex2_approx(fmaf(x[j + 1], kLog2e, nb));
    a2 += ex2_approx(fmaf(x[j + 2], kLog2e, nb));
    a3 += ex2_approx(fmaf(x[j + 3], kLog2e, nb));
  }
  // first chunk: st.m = -inf, the old sum is scaled by exp(-inf) = 0
  st.s = st.s * ex2_approx((st.m - mn) * kLog2e) + ((a0 + a1) + (a2 + a3));
  st.m = mn;
  const int jt = yl - cb;
  if (static_cast<unsigned>(jt) < 32u) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j == jt) st.tgt = x[j];
    st.have_tgt = true;
  }
}

// ---------------------------------------------------------------------------
// Epilogue: gradient-panel values of one 32-column chunk, packed to 16 bits.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void grad_chunk(const GemmArgs& g, uint32_t (&z)[32], int cb,
                                           int vglob0, int vlim, int yl, bool valid, float mrow,
                                           float krow, uint32_t (&packed)[16]) {
  float x[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(z[j]);
  if (g.bias != nullptr) {
    float bv[32];
    load_bias32(g.bias, vglob0 + cb, g.V, g.is_bf16 != 0, bv);
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] += bv[j];
  }
  float gv[32];
  // sigma * p = 2^( ((z - m) - log s) * log2(e) + log2(sigma) )
#pragma unroll
  for (int j = 0; j < 32; ++j) gv[j] = ex2_approx(fmaf(x[j] - mrow, kLog2e, krow));
  if (!valid) {
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
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j == jt) gv[j] -= g.sigma;
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
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1) flce_gemm_kernel(const __grid_constant__ GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_STAGE_BYTES;
  uint8_t* sStg = sB + STAGES * B_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + 2 * STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* done_bar = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* decision = abort_flag + 1;  // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], NUM_EPI_THREADS);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    decision[0] = 0;
    decision[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&g.tmA[0]);
    tma_prefetch_map(&g.tmB[0]);
    if (MODE == kModeWH) {
      tma_prefetch_map(&g.tmA[1]);
      tma_prefetch_map(&g.tmB[1]);
    }
    if (MODE == kModeGrad) tma_prefetch_map(&g.tmOut);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int C = (MODE == kModePlain) ? g.M : *g.C_dev;
  const int nunits = num_units<MODE>(g, C);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t n_issued = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
        const Unit un = decode_unit<MODE>(g, C, u);
        for (int kb = 0; kb < un.nk; ++kb) {
          const uint32_t stage = n_issued % STAGES;
          const uint32_t phase = (n_issued / STAGES) & 1u;
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, g.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], A_STAGE_BYTES + B_STAGE_BYTES);
          issue_stage_loads<MODE>(g, un, kb, smem_addr(sA + stage * A_STAGE_BYTES),
                                  smem_addr(sB + stage * B_STAGE_BYTES), &full[stage]);
          ++n_issued;
        }
      }
      // Let every copy still in flight land before the CTA can exit.
      const uint32_t first = n_issued > STAGES ? n_issued - STAGES : 0u;
      for (uint32_t i = first; i < n_issued; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1u, nullptr, nullptr, kDrainLimitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t n_used = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
        const Unit un = decode_unit<MODE>(g, C, u);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, g.err)) break;
        tc_fence_after();
        const bool a_mn = unit_a_mn<MODE>(g, un);
        const bool b_mn = unit_b_mn<MODE>(g, un);
        const uint32_t idesc = make_idesc_f16(g.is_bf16 != 0, a_mn, b_mn, BM, BN);
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        const uint32_t a_lbo = a_mn ? MN_BOX_BYTES : 16u;
        const uint32_t b_lbo = b_mn ? MN_BOX_BYTES : 16u;
        const uint32_t a_step = a_mn ? 16u * 128u : 32u;  // bytes per K=16 slice
        const uint32_t b_step = b_mn ? 16u * 128u : 32u;
        for (int kb = 0; kb < un.nk; ++kb) {
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
            umma_f16(d_tmem, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);  // frees the stage once these MMAs are done
          ++n_used;
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);  // accumulator ready (immediately when nk == 0)
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // All MMAs of this CTA complete before TMEM is released.
      umma_commit(done_bar);
      mbar_wait(done_bar, 0, nullptr, nullptr, kDrainLimitNs);
    }
  } else if (warp >= EPI_WARP0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;         // row within the tile
    const int epi_tid = threadIdx.x - EPI_WARP0 * 32;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t nstore = 0;  // grad: 64-column boxes stored so far by this CTA
    float wh_scale = 0.f;
    if (MODE == kModeWH) {
      const float lam = (g.lam_dev != nullptr) ? *g.lam_dev : g.lam;
      wh_scale = (C > 0) ? lam / static_cast<float>(C) * g.inv_sigma : 0.f;
    }
    int it = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
      const Unit un = decode_unit<MODE>(g, C, u);
      // per-row data, fetched before waiting for the accumulator
      const int row = un.m0 + r;
      bool valid = false;
      int yl = -1;
      float mrow = 0.f, krow = 0.f;
      int orow = 0;
      int vglob0 = 0, vlim = 0;
      if (MODE == kModeFwd || MODE == kModeGrad) {
        valid = row < C;
        vglob0 = g.vp + un.n0;
        vlim = g.V - vglob0;
        const int y = valid ? __ldg(g.y_c + row) : -1;
        yl = valid ? y - vglob0 : -1000000;
        if (MODE == kModeGrad && valid) {
          const int o = __ldg(g.idx + row);
          mrow = __ldg(g.m_saved + o);
          krow = g.log2_sigma - __ldg(g.logs_saved + o) * kLog2e;
        }
      } else if (MODE == kModeWH) {
        if (un.cls == 0) {
          valid = (un.m0 + r) < g.K;
          orow = g.vp + un.m0 + r;  // dW row (vocabulary id)
        } else {
          valid = row < C;
          orow = valid ? __ldg(g.idx + row) : 0;  // dH row (original position)
        }
      } else {
        valid = row < g.M;
      }

      mbar_wait(&tfull[acc], acc_phase, abort_flag, g.err);
      named_bar_sync(1, NUM_EPI_THREADS);
      if (epi_tid == 0) decision[it & 1] = *abort_flag;
      named_bar_sync(1, NUM_EPI_THREADS);
      if (decision[it & 1]) break;
      tc_fence_after();
      const uint32_t t_acc = lane_base + static_cast<uint32_t>(acc * BN);

      if (MODE == kModeFwd) {
        FwdRowState st{-INFINITY, 0.f, 0.f, false};
        uint32_t za[32], zb[32];
        tmem_ld32(t_acc, za);
        tmem_wait_ld(za);
#pragma unroll 1
        for (int c = 0; c < BN / 32; c += 2) {
          tmem_ld32(t_acc + (c + 1) * 32, zb);
          fwd_chunk(g, za, c * 32, vglob0, vlim, yl, st);
          tmem_wait_ld(zb);
          if (c + 2 < BN / 32) tmem_ld32(t_acc + (c + 2) * 32, za);
          fwd_chunk(g, zb, (c + 1) * 32, vglob0, vlim, yl, st);
          if (c + 2 < BN / 32) tmem_wait_ld(za);
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        if (valid) {
          g.part[static_cast<size_t>(row) * g.part_ld + un.n0 / BN] = make_float2(st.m, st.s);
          if (st.have_tgt) g.tgt[row] = st.tgt;
        }
      } else if (MODE == kModeGrad) {
        uint32_t za[32], zb[32];
        tmem_ld32(t_acc, za);
        tmem_wait_ld(za);
#pragma unroll 1
        for (int c = 0; c < BN / 32; c += 2) {
          // chunks c, c+1 form one 64-column box staged in buffer (nstore & 1)
          uint8_t* stg = sStg + (nstore & 1u) * STG_BYTES;
          if (epi_tid == 0) bulk_wait_group_read<1>();  // the box stored 2 boxes ago left smem
          named_bar_sync(1, NUM_EPI_THREADS);
          tmem_ld32(t_acc + (c + 1) * 32, zb);
          uint32_t pk[16];
          grad_chunk(g, za, c * 32, vglob0, vlim, yl, valid, mrow, krow, pk);
          uint8_t* rowp = stg + r * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int chunk16 = j ^ (r & 7);
            *reinterpret_cast<uint4*>(rowp + chunk16 * 16) =
                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
          tmem_wait_ld(zb);
          if (c + 2 < BN / 32) tmem_ld32(t_acc + (c + 2) * 32, za);
          grad_chunk(g, zb, (c + 1) * 32, vglob0, vlim, yl, valid, mrow, krow, pk);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int chunk16 = (4 + j) ^ (r & 7);
            *reinterpret_cast<uint4*>(rowp + chunk16 * 16) =
                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
          if (c + 2 < BN / 32) tmem_wait_ld(za);
          fence_proxy_async_smem();
          named_bar_sync(1, NUM_EPI_THREADS);
          if (epi_tid == 0) {
            // a box that starts past the panel's last column holds only padding
            if (un.n0 + c * 32 < g.ncols) tma_store_2d(&g.tmOut, smem_addr(stg), un.n0 + c * 32, un.m0);
            bulk_commit_group();
          }
          ++nstore;
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
      } else if (MODE == kModeWH) {
        float* dst = (un.cls == 0 ? g.dW : g.dH) + static_cast<size_t>(orow) * g.D;
        const bool accumulate = (un.cls == 1) && (g.vp > 0);
        const bool zero = (un.nk == 0);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          const int d0 = un.n0 + c * 32;
          if (d0 >= g.D) break;
          uint32_t z[32];
          if (!zero) {
            tmem_ld32(t_acc + c * 32, z);
            tmem_wait_ld(z);
          }
          if (valid) {
            const int nv = min(32, g.D - d0);  // multiple of 8
            float4* p = reinterpret_cast<float4*>(dst + d0);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              if (q4 * 4 < nv) {
                float4 v;
                if (zero) {
                  v = make_float4(0.f, 0.f, 0.f, 0.f);
                } else {
                  v = make_float4(__uint_as_float(z[4 * q4]) * wh_scale,
                                  __uint_as_float(z[4 * q4 + 1]) * wh_scale,
                                  __uint_as_float(z[4 * q4 + 2]) * wh_scale,
                                  __uint_as_float(z[4 * q4 + 3]) * wh_scale);
                }
                if (accumulate) {
                  const float4 o = p[q4];
                  v.x += o.x;
                  v.y += o.y;
                  v.z += o.z;
                  v.w += o.w;
                }
                p[q4] = v;
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
      } else {  // kModePlain
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          const int c0 = un.n0 + c * 32;
          if (c0 >= g.ncols) break;
          uint32_t z[32];
          tmem_ld32(t_acc + c * 32, z);
          tmem_wait_ld(z);
          if (valid) {
            float* dst = g.out + static_cast<size_t>(row) * g.ncols + c0;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c0 + j < g.ncols) dst[j] = __uint_as_float(z[j]) * g.scale;
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (MODE == kModeGrad && epi_tid == 0) bulk_wait_group<0>();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace flce
