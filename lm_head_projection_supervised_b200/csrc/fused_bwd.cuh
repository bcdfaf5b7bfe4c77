// Single-kernel backward for small hidden sizes (D <= 64): the literal fused
// form of the "分块交叉熵" page, §04 — per tile, the scores are recomputed, the
// gradient of the logits is formed on chip, and both contractions consume it
// at once; dH of a row block accumulates across vocabulary tiles in TMEM,
// beside the score tile, and dW is summed per group of row blocks in one
// slab of partials, the slabs then added up by a second kernel (every sum in
// a fixed order: deterministic).
//
// One CTA per SM, no clusters (tcgen05 cta_group::1, M = 128).  A work item is
// (vocabulary chunk ch, group g of row blocks); for each row block rb of the
// group in turn (256 rows = two 128-row halves), the CTA sweeps the chunk's
// 128-id tiles t:
//   Z_h   = H_h W_t^T                  h = 0, 1   M=128 rows, N=128 ids, K=64
//   G_h   = r (p - onehot) sigma        epilogue, 16-bit, into shared memory
//   dH_h += G_h W_t                               M=128 rows, N=64,      K=128 ids
//   dW_t  = G_0^T H_0 + G_1^T H_1                 M=128 ids,  N=64,      K=256 rows
// with G, W_t and H_h read from shared memory as laid out by TMA / the
// epilogue (128-byte swizzle; the same tile serves as a K-major operand of
// one product and an MN-major operand of another).  dW_t goes to slab g: a TMA
// store for the group's first row block, a TMA reduction (an f32 add in L2)
// for the next ones, each pass over the chunk starting after the previous
// pass's writes have completed, so the additions come in row-block order; the
// chunk's slice of the slab (about 0.4 MB) stays in L2 meanwhile.  After each
// row block dH_h goes to the slab of chunk ch.  TMEM (512 columns): Z of both
// halves [0, 256), dH of both halves [256, 384), dW in two buffers [384, 512)
// so that the epilogue drains one while the next accumulates.  D > 64 does
// not fit: dH of 256 rows and a dW tile need 2 D + D columns beside the 256
// of the scores.
//
// Roles (640 threads): warp 0 schedules items and loads H (once per row
// block) and the W tiles (a ring); warp 1 issues the MMAs; warps 4..19 are
// four epilogue warpgroups, warpgroup (h, s) on row half h and the 64 ids s
// of the tile (thread = TMEM lane = row): the epilogue is bound by its
// per-entry arithmetic and latency, and four warps per scheduler hide more
// of it than two.  They also drain the dW tiles (lane = vocabulary id; the
// two warpgroups of row half t % 2 take tile t, 32 columns each) and the dH
// halves, each warp its 32 TMEM lanes through its own 4 KiB staging box and
// TMA, so that the epilogue warps meet only once per row block.  Every wait
// is bounded (see mbar_wait).
#pragma once

#include "gemm.cuh"

namespace flce {

constexpr int FB_MAX_D = 64;        // hidden sizes the fused backward takes
constexpr int FB_ROWS = 256;        // rows per row block (two 128-row halves)
constexpr int FB_COLS = 128;        // vocabulary ids per tile
constexpr int FB_WSTAGES = 2;       // W tile ring depth (a tile lasts thousands of cycles)
constexpr int FB_EPI_WG = 4;        // epilogue warpgroups
constexpr int FB_EPI_THREADS = FB_EPI_WG * EPI_WG_THREADS;
constexpr int FB_THREADS = EPI_WARP0 * 32 + FB_EPI_THREADS;
// registers per thread after the split (the first warpgroup only schedules,
// loads and issues), and at launch
constexpr uint32_t FB_REGS_LOW = 64;
constexpr uint32_t FB_REGS_HIGH = 104;
static_assert(128 * FB_REGS_LOW + FB_EPI_THREADS * FB_REGS_HIGH <= 65536, "register split");
constexpr uint32_t FB_REGS_AT_LAUNCH =
    (128 * FB_REGS_LOW + FB_EPI_THREADS * FB_REGS_HIGH + FB_THREADS - 1) / FB_THREADS;
constexpr uint32_t FB_STG_BYTES = 32 * 128;  // 4 KiB staging box per epilogue warp
constexpr int FB_NCH_MAX = 160;     // vocabulary chunks (slabs of dH partials) at most
constexpr int FB_NG_MAX = 8;        // groups of row blocks (slabs of dW partials) at most
constexpr uint32_t FB_H_BYTES = BM * 64 * 2;        // 16 KiB: one 128-row half of H
constexpr uint32_t FB_HB_BYTES = 2 * FB_H_BYTES;    // 32 KiB: one H buffer (a row block)
constexpr uint32_t FB_W_BYTES = FB_COLS * 64 * 2;   // 16 KiB: one W tile
constexpr uint32_t FB_G_BYTES = 2 * STG_BYTES;      // 32 KiB: 128 rows x 128 ids, two 64-id boxes
constexpr uint32_t FB_TM_Z = 0;     // TMEM column of Z_0 (Z_1 at +128)
constexpr uint32_t FB_TM_DH = 256;  // dH_0 (dH_1 at +64)
constexpr uint32_t FB_TM_DW = 384;  // dW buffer 0 (buffer 1 at +64)
constexpr size_t FB_SMEM_BYTES = 1024 + 2 * FB_HB_BYTES + FB_WSTAGES * FB_W_BYTES +
                                 2 * FB_G_BYTES + (FB_EPI_THREADS / 32) * FB_STG_BYTES + 512;
static_assert(FB_SMEM_BYTES <= 232448, "shared memory per CTA");
// The MMA issuer adds operand offsets to a descriptor's 14-bit start-address
// field (desc_sw128_sbo1k): every shared-memory address of the CTA (this
// kernel's dynamic shared memory after at most 1 KiB reserved ahead of it),
// in 16-byte units, stays below 2^14.
static_assert(1024 + FB_SMEM_BYTES <= (size_t(1) << 18), "descriptor start-address field");

// The split of the work: nch vocabulary chunks (one per CTA or more, at most
// FB_NCH_MAX: a chunk's dW slice stays small enough for L2) times ng groups
// of R row blocks (about four items per CTA in all, at most FB_NG_MAX).  With
// no supervised row there is still one (empty) row block, so that dW is
// written.  The fused kernel and both reductions derive it from (C, V, CTAs).
struct FusedPlan {
  int nrb, nv, nch, ng, R;
};
__host__ __device__ inline FusedPlan fused_plan(int C, int V, int nctas) {
  FusedPlan p;
  p.nrb = C > 0 ? (C + FB_ROWS - 1) / FB_ROWS : 1;
  p.nv = (V + FB_COLS - 1) / FB_COLS;
  p.nch = p.nv < FB_NCH_MAX ? p.nv : FB_NCH_MAX;
  int ng = (4 * nctas + p.nch - 1) / p.nch;
  if (ng > p.nrb) ng = p.nrb;
  if (ng > FB_NG_MAX) ng = FB_NG_MAX;
  if (ng < 1) ng = 1;
  p.R = (p.nrb + ng - 1) / ng;
  p.ng = (p.nrb + p.R - 1) / p.R;
  return p;
}

struct FusedArgs {
  // tmA[0]: H_c, K-major 64 x 128 boxes; tmB[0]: W, K-major 64 x 128 boxes;
  // tmDW: dW partials [FB_NG_MAX * Vp][D] f32; tmDH: dH partials
  // [FB_NCH_MAX * Np][D] f32 (32 x 32 boxes); the rest as for the backward's
  // gradient units
  GemmArgs g;
  int Vp;     // rows per dW slab (V rounded up to a tile)
  int Np;     // rows per dH slab
  int nctas;  // CTAs of the launch (fixes the chunking)
};

template <int FEAT>
__global__ void __launch_bounds__(FB_THREADS, 1)
    flce_fused_bwd_kernel(const __grid_constant__ FusedArgs fa) {
  const GemmArgs& g = fa.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sH = smem;                              // [2 buffers][2 halves][16 KiB]
  uint8_t* sW = sH + 2 * FB_HB_BYTES;              // [FB_WSTAGES][16 KiB]
  uint8_t* sG = sW + FB_WSTAGES * FB_W_BYTES;      // [2 halves][2 boxes][16 KiB]
  uint8_t* sStg = sG + 2 * FB_G_BYTES;             // [16 epilogue warps][4 KiB]
  uint64_t* w_full =
      reinterpret_cast<uint64_t*>(sStg + (FB_EPI_THREADS / 32) * FB_STG_BYTES);
  uint64_t* w_empty = w_full + FB_WSTAGES;
  uint64_t* h_full = w_empty + FB_WSTAGES;  // [2]
  uint64_t* h_empty = h_full + 2;           // [2]
  uint64_t* z_full = h_empty + 2;
  uint64_t* z_empty = z_full + 1;
  uint64_t* g_full = z_empty + 1;
  uint64_t* g_empty = g_full + 1;
  uint64_t* dw_full = g_empty + 1;   // [2]
  uint64_t* dw_empty = dw_full + 2;  // [2]
  uint64_t* dh_full = dw_empty + 2;
  uint64_t* dh_empty = dh_full + 1;
  uint64_t* uq_full = dh_empty + 1;  // [UQ]
  uint64_t* uq_empty = uq_full + UQ;
  uint64_t* done_bar = uq_empty + UQ;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* decision = abort_flag + 1;  // [2]
  volatile int* s_unit = decision + 2;      // [UQ]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr uint32_t kEpiWarps = FB_EPI_THREADS / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < FB_WSTAGES; ++s) {
      mbar_init(&w_full[s], 1);   // the producer's expect_tx arrival + the tile's bytes
      mbar_init(&w_empty[s], 1);  // one MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&h_full[b], 1);
      mbar_init(&h_empty[b], 1);
    }
    mbar_init(z_full, 1);
    mbar_init(z_empty, kEpiWarps);
    mbar_init(g_full, kEpiWarps);
    mbar_init(g_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&dw_full[b], 1);
      mbar_init(&dw_empty[b], kEpiWarps / 2);  // the eight warps that drain the tile
    }
    mbar_init(dh_full, 1);
    mbar_init(dh_empty, kEpiWarps);
    for (int q = 0; q < UQ; ++q) {
      mbar_init(&uq_full[q], 1);
      mbar_init(&uq_empty[q], 1 + kEpiWarps);  // the MMA lane and the epilogue warps
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
    tma_prefetch_map(&g.tmDW);
    tma_prefetch_map(&g.tmDH);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int C = *g.C_dev;
  const FusedPlan pl = fused_plan(C, g.V, fa.nctas);
  const int total = pl.ng * pl.nch;
  // item u -> group (fastest, so that concurrent items share W tiles in L2),
  // its row blocks [rb0, rb1) and the chunk's tiles [t0, t1)
  struct Item {
    int g, ch, rb0, rb1, t0, t1;
  };
  auto decode = [&](int u) {
    Item it;
    it.g = u % pl.ng;
    it.ch = u / pl.ng;
    it.rb0 = it.g * pl.R;
    it.rb1 = min(pl.nrb, it.rb0 + pl.R);
    it.t0 = static_cast<int>(static_cast<int64_t>(it.ch) * pl.nv / pl.nch);
    it.t1 = static_cast<int>(static_cast<int64_t>(it.ch + 1) * pl.nv / pl.nch);
    return it;
  };

  if (warp < EPI_WARP0) {
    setmaxnreg_dec<FB_REGS_LOW>();
    if (warp == 0) {
      // ------------------------------------------------------------ scheduler + loads
      if (lane == 0) {
        uint32_t n_w = 0;
        int n_item = 0;
        bool ok = true;
        for (int it = 0; ok; ++it) {
          const int slot = it % UQ;
          if (!mbar_wait(&uq_empty[slot], ((it / UQ) & 1) ^ 1u, abort_flag, g.err)) break;
          int u = atomicAdd(g.counter, 1);
          if (u >= total) u = -1;
          s_unit[slot] = u;
          mbar_arrive(&uq_full[slot]);
          if (u < 0) break;
          const Item itm = decode(u);
          for (int rb = itm.rb0; ok && rb < itm.rb1; ++rb) {
            // the row block's rows into H buffer n_item % 2, once the MMAs of
            // the row block before the previous one are done with it
            const int hb = n_item & 1;
            if (!mbar_wait(&h_empty[hb], ((n_item >> 1) & 1) ^ 1, abort_flag, g.err)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&h_full[hb], FB_HB_BYTES);
            tma_load_2d(smem_addr(sH + hb * FB_HB_BYTES), &g.tmA[0], &h_full[hb], 0,
                        rb * FB_ROWS);
            tma_load_2d(smem_addr(sH + hb * FB_HB_BYTES + FB_H_BYTES), &g.tmA[0], &h_full[hb], 0,
                        rb * FB_ROWS + BM);
            ++n_item;
            for (int t = itm.t0; t < itm.t1; ++t) {
              const uint32_t stage = n_w % FB_WSTAGES;
              if (!mbar_wait(&w_empty[stage], ((n_w / FB_WSTAGES) & 1u) ^ 1u, abort_flag,
                             g.err)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(&w_full[stage], FB_W_BYTES);
              tma_load_2d(smem_addr(sW + stage * FB_W_BYTES), &g.tmB[0], &w_full[stage], 0,
                          t * FB_COLS);
              ++n_w;
            }
          }
        }
        // every copy still in flight lands before the CTA can exit
        const uint32_t first = n_w > FB_WSTAGES ? n_w - FB_WSTAGES : 0u;
        for (uint32_t i = first; i < n_w; ++i)
          mbar_wait(&w_full[i % FB_WSTAGES], (i / FB_WSTAGES) & 1u, nullptr, nullptr,
                    kDrainLimitNs);
        for (int i = n_item > 2 ? n_item - 2 : 0; i < n_item; ++i)
          mbar_wait(&h_full[i & 1], (i >> 1) & 1, nullptr, nullptr, kDrainLimitNs);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const bool bf16 = g.is_bf16 != 0;
        const uint32_t idesc_z = make_idesc_f16(bf16, false, false, BM, FB_COLS);
        const uint32_t idesc_dh = make_idesc_f16(bf16, false, true, BM, 64);
        const uint32_t idesc_dw = make_idesc_f16(bf16, true, true, BM, 64);
        const uint32_t sg = smem_addr(sG);
        uint32_t sh = smem_addr(sH);  // H buffer of the current row block
        uint32_t n_w = 0, n_t = 0;
        int n_item = 0;
        // Z of the tile with global index ti, from W tile wi of the ring.  The
        // scores of tile t + 1 are issued as soon as the epilogue has read
        // those of tile t (while it still forms G of tile t), ahead of tile
        // t's contractions, so that they are ready when it moves on.
        auto issue_z = [&](uint32_t wi, uint32_t ti) -> bool {
          if (!mbar_wait(&w_full[wi % FB_WSTAGES], (wi / FB_WSTAGES) & 1u, abort_flag, g.err) ||
              !mbar_wait(z_empty, (ti & 1) ^ 1, abort_flag, g.err))
            return false;
          tc_fence_after();
          const uint32_t sw = smem_addr(sW + (wi % FB_WSTAGES) * FB_W_BYTES);
          // descriptors: the low words once, each MMA adds its offset (40 MMAs
          // a tile, issued by one thread that shares its scheduler with four
          // epilogue warps: the issue cost is on the tile's critical path)
          const uint32_t za = desc_lo_sw128(sh, 16), zb = desc_lo_sw128(sw, 16);
          // K = 64 (the hidden size, zero-padded)
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f16(tmem_base + FB_TM_Z + 128 * h,
                       desc_sw128_sbo1k(za + ((h * FB_H_BYTES + kk * 32) >> 4)),
                       desc_sw128_sbo1k(zb + ((kk * 32) >> 4)), idesc_z, kk > 0 ? 1u : 0u);
          umma_commit(z_full);
          return true;
        };
        bool ok = true;
        for (int it = 0; ok; ++it) {
          const int slot = it % UQ;
          if (!mbar_wait(&uq_full[slot], (it / UQ) & 1, abort_flag, g.err)) break;
          const int u = s_unit[slot];
          mbar_arrive(&uq_empty[slot]);
          if (u < 0) break;
          const Item itm = decode(u);
          const int t0 = itm.t0, t1 = itm.t1;
          for (int rb = itm.rb0; ok && rb < itm.rb1; ++rb) {
            // the row block's H is in; its first scores go ahead of the wait
            // for the previous row block's dH to leave TMEM (before the first
            // dH product, which overwrites it)
            const int hb = n_item & 1;
            sh = smem_addr(sH + hb * FB_HB_BYTES);
            ok = mbar_wait(&h_full[hb], (n_item >> 1) & 1, abort_flag, g.err) &&
                 issue_z(n_w, n_t);
            for (int t = t0; ok && t < t1; ++t) {
              const uint32_t stage = n_w % FB_WSTAGES;
              // the next tile's scores as soon as this tile's have been read
              // (the epilogue is still forming G)
              if (t + 1 < t1 && !(ok = issue_z(n_w + 1, n_t + 1))) break;
              if (!mbar_wait(g_full, n_t & 1, abort_flag, g.err)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t sw = smem_addr(sW + stage * FB_W_BYTES);
              const uint32_t buf = n_t & 1;
              if (t == t0 && !(ok = mbar_wait(dh_empty, (n_item & 1) ^ 1, abort_flag, g.err)))
                break;
              const uint32_t ga = desc_lo_sw128(sg, 16), wb = desc_lo_sw128(sw, 8192);
              const uint32_t acc0 = t > t0 ? 1u : 0u;
              // dH_h += G_h W_t: G K-major (rows x ids), W_t MN-major (ids x D)
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                  for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem_base + FB_TM_DH + 64 * h,
                             desc_sw128_sbo1k(ga + ((h * FB_G_BYTES + j * STG_BYTES + kk * 32) >> 4)),
                             desc_sw128_sbo1k(wb + ((j * 8192 + kk * 2048) >> 4)), idesc_dh,
                             (j > 0 || kk > 0) ? 1u : acc0);
              if (!mbar_wait(&dw_empty[buf], ((n_t >> 1) & 1) ^ 1, abort_flag, g.err)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t gm = desc_lo_sw128(sg, STG_BYTES), hm = desc_lo_sw128(sh, 8192);
              const uint32_t tdw = tmem_base + FB_TM_DW + 64 * buf;
              // dW_t = sum_h G_h^T H_h: G MN-major (ids x rows), H_h MN-major (D x rows)
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                  umma_f16(tdw, desc_sw128_sbo1k(gm + ((h * FB_G_BYTES + kk * 2048) >> 4)),
                           desc_sw128_sbo1k(hm + ((h * FB_H_BYTES + kk * 2048) >> 4)), idesc_dw,
                           (h > 0 || kk > 0) ? 1u : 0u);
              umma_commit(&dw_full[buf]);
              umma_commit(g_empty);
              umma_commit(&w_empty[stage]);
              ++n_t;
              ++n_w;
            }
            if (!ok) break;
            umma_commit(dh_full);
            umma_commit(&h_empty[hb]);
            ++n_item;
          }
        }
        // every MMA completes before TMEM is released
        umma_commit(done_bar);
        mbar_wait(done_bar, 0, nullptr, nullptr, kDrainLimitNs);
      }
    }
  } else {
    setmaxnreg_inc<FB_REGS_HIGH>();
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;  // TMEM lane: a row of the half, or a vocabulary id of a dW tile
    const int epi_tid = threadIdx.x - EPI_WARP0 * 32;
    const int wg = epi_tid / EPI_WG_THREADS;
    const int hh = wg >> 1;  // row half: Z_hh, G_hh, dH_hh; drains the dW tiles t with t % 2 == hh
    const int ss = wg & 1;   // ids [64 ss, 64 ss + 64) of a tile (G box ss); columns
                             // [32 ss, 32 ss + 32) of the dW tiles and of dH_hh
    uint8_t* stg = sStg + (epi_tid / 32) * FB_STG_BYTES;  // this warp's 32 x 128-byte box
    uint8_t* gbox = sG + hh * FB_G_BYTES + ss * STG_BYTES;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int round = 0;
    auto decide_abort = [&]() -> bool {
      named_bar_sync(1, FB_EPI_THREADS);
      if (epi_tid == 0) decision[round & 1] = *abort_flag;
      named_bar_sync(1, FB_EPI_THREADS);
      return decision[(round++) & 1] != 0;
    };
    // this warp's 32 rows x 32 f32 columns through its staging box, stored
    // or added (TMA reduction) to global memory.  The box is reused once the
    // previous one has been read from it; with `order`, once everything this
    // warp sent before has been written.
    auto emit_box = [&](const uint32_t (&w)[32], const CUtensorMap* map, int x, int y,
                        bool issue, bool add, bool order) {
      if (lane == 0) {
        if (order)
          bulk_wait_group<0>();
        else
          bulk_wait_group_read<0>();
      }
      __syncwarp();
      stage_row128(stg, lane, 0, w);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (issue) {
          if (add)
            tma_reduce_add_2d(map, smem_addr(stg), x, y);
          else
            tma_store_2d(map, smem_addr(stg), x, y);
        }
        bulk_commit_group();
      }
    };
    // dW of tile t (TMEM buffer buf) -> slab sg, stored or added: this warp's
    // 32 vocabulary ids x its 32 columns.  TMEM is handed back as soon as it
    // has been read.  A warp drains the same ids and columns of a tile in
    // every pass, so waiting for its own earlier additions orders them.
    bool first_drain = false;
    auto drain_dw = [&](uint32_t buf, int sg, int t, bool add) {
      uint32_t w[32];
      tmem_ld32(lane_base + FB_TM_DW + 64 * buf + 32 * ss, w);
      tmem_wait_ld(w);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dw_empty[buf]);
      emit_box(w, &g.tmDW, 32 * ss, sg * fa.Vp + t * FB_COLS + 32 * q, 32 * ss < g.D, add,
               add && first_drain);
      first_drain = false;
    };

    uint32_t n_t = 0;
    int n_item = 0;
    for (int it = 0;; ++it) {
      const int slot = it % UQ;
      const bool got = mbar_wait(&uq_full[slot], (it / UQ) & 1, abort_flag, g.err);
      const int u = got ? s_unit[slot] : -1;
      __syncwarp();
      if (lane == 0) mbar_arrive(&uq_empty[slot]);
      if (decide_abort() || u < 0) break;
      const Item itm = decode(u);
      const int t0 = itm.t0, t1 = itm.t1;
      bool aborted = false;
      for (int rb = itm.rb0; !aborted && rb < itm.rb1; ++rb) {
        // dW: the group's later row blocks add to the slab, each warp's first
        // addition of a pass after its additions of the previous pass have
        // all been written, so that every element receives its terms in
        // row-block order
        const bool add = rb > itm.rb0;
        first_drain = true;
        const int row = rb * FB_ROWS + hh * BM + r;
        const bool valid = row < C;
        int yabs = 0;
        float krow = 0.f, rrow = 0.f;
        if (valid) {
          yabs = __ldg(g.y_c + row);
          const int o = __ldg(g.idx + row);
          krow = fmaf(-__ldg(g.m_saved + o), kLog2e,
                      g.log2_sigma - __ldg(g.logs_saved + o) * kLog2e);
          rrow = __ldg(g.row_scale + row);
        }
        // a warp whose 32 rows are all supervised with a positive scale takes
        // the scale into the exponent (two operations an entry fewer); the
        // bias variants keep the general form, which needs fewer registers
        const bool fold =
            (FEAT & kFeatBias) == 0 && __all_sync(0xffffffffu, valid && rrow > 0.f);
        const float krow_f = fold ? krow + log2f(rrow) : krow;
        // The epilogue warps decide together whether to stop once per row
        // block (at its end): a wait that gives up raises the abort flag and
        // returns, the later waits return at once, and the warps run on to
        // the decision with whatever TMEM and shared memory hold.
        for (int t = t0; t < t1; ++t, ++n_t) {
          // Z_t is in TMEM
          mbar_wait(z_full, n_t & 1, abort_flag, g.err);
          tc_fence_after();
          const int vglob0 = t * FB_COLS;
          const int vlim = g.V - vglob0;
          const int yl = valid ? yabs - vglob0 : -1000000;
          const uint32_t t_z = lane_base + FB_TM_Z + 128 * hh + 64 * ss;
          // both 32-id chunks are formed before the wait for the previous
          // tile's contractions to release G, so that only the stores into
          // shared memory wait for them
          uint32_t za[32], pk0[16], pk1[16];
          bool big = false;
          tmem_ld32(t_z, za);
          tmem_wait_ld(za);
          if (fold)
            grad_chunk<FEAT, true>(g, za, 64 * ss, vglob0, vlim, yl, true, krow_f, rrow, row, lane,
                                   pk0, big);
          else
            grad_chunk<FEAT>(g, za, 64 * ss, vglob0, vlim, yl, valid, krow, rrow, row, lane, pk0,
                             big);
          tmem_ld32(t_z + 32, za);
          tmem_wait_ld(za);
          // Z read: its TMEM is free for the next tile's scores
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(z_empty);
          if (fold)
            grad_chunk<FEAT, true>(g, za, 64 * ss + 32, vglob0, vlim, yl, true, krow_f, rrow, row,
                                   lane, pk1, big);
          else
            grad_chunk<FEAT>(g, za, 64 * ss + 32, vglob0, vlim, yl, valid, krow, rrow, row, lane,
                             pk1, big);
          // G of tile t - 1 has been read by its contractions
          mbar_wait(g_empty, (n_t & 1) ^ 1, abort_flag, g.err);
          stage_row128(gbox, r, 0, pk0);
          stage_row128(gbox, r, 4, pk1);
          // G written (visible to the tensor core's reads)
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(g_full);
          if (t > t0 && ((t - 1) & 1) == hh) {
            const uint32_t np = n_t - 1;
            mbar_wait(&dw_full[np & 1], (np >> 1) & 1, abort_flag, g.err);
            tc_fence_after();
            drain_dw(np & 1, itm.g, t - 1, add);
          }
        }
        // the last dW tile, then the row block's dH halves -> the slab of chunk ch
        const uint32_t nl = n_t - 1;
        if (((t1 - 1) & 1) == hh) {
          mbar_wait(&dw_full[nl & 1], (nl >> 1) & 1, abort_flag, g.err);
          tc_fence_after();
          drain_dw(nl & 1, itm.g, t1 - 1, add);
        }
        mbar_wait(dh_full, n_item & 1, abort_flag, g.err);
        tc_fence_after();
        uint32_t w0[32];
        tmem_ld32(lane_base + FB_TM_DH + 64 * hh + 32 * ss, w0);
        tmem_wait_ld(w0);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dh_empty);
        const int ydh = itm.ch * fa.Np + rb * FB_ROWS + hh * BM + 32 * q;
        emit_box(w0, &g.tmDH, 32 * ss, ydh, 32 * ss < g.D, false, false);
        ++n_item;
        if (decide_abort()) {
          aborted = true;
          break;
        }
      }
      if (aborted) break;
    }
    if (lane == 0) bulk_wait_group<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// dW[v][d] = (S / sigma) * sum over the groups of row blocks of the slabs
// [g][v][d], in order of g.  Vectors of 4 f32 (D % 4 == 0).
__global__ void fused_reduce_dw_kernel(const float4* __restrict__ part, int64_t slab4, int V,
                                       int D4, const int* __restrict__ C_dev, int nctas,
                                       const float* __restrict__ scal, float inv_sigma,
                                       float4* __restrict__ dW) {
  const int C = *C_dev;
  const int ng = fused_plan(C, V, nctas).ng;
  const float sc = C > 0 ? *scal * inv_sigma : 0.f;
  const int64_t n = static_cast<int64_t>(V) * D4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 a = __ldcs(part + i);
    for (int k = 1; k < ng; ++k) {
      const float4 v = __ldcs(part + k * slab4 + i);
      a.x += v.x;
      a.y += v.y;
      a.z += v.z;
      a.w += v.w;
    }
    dW[i] = make_float4(a.x * sc, a.y * sc, a.z * sc, a.w * sc);
  }
}

// dH_c[k][d] = (S / sigma) * sum over the vocabulary chunks of the slabs
// [ch][k][d], in order of ch, for the supervised rows k < C.
__global__ void fused_reduce_dh_kernel(const float4* __restrict__ part, int64_t slab4, int D4,
                                       const int* __restrict__ C_dev, int V, int nctas,
                                       const float* __restrict__ scal, float inv_sigma,
                                       float4* __restrict__ dhc) {
  const int C = *C_dev;
  const int nch = fused_plan(C, V, nctas).nch;
  const float sc = C > 0 ? *scal * inv_sigma : 0.f;
  const int64_t n = static_cast<int64_t>(C) * D4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int ch = 0; ch < nch; ++ch) {
      const float4 v = __ldcs(part + ch * slab4 + i);
      a.x += v.x;
      a.y += v.y;
      a.z += v.z;
      a.w += v.w;
    }
    dhc[i] = make_float4(a.x * sc, a.y * sc, a.z * sc, a.w * sc);
  }
}

}  // namespace flce
