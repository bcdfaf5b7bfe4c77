// Memory-bound helper kernels around the tensor-core GEMMs: supervised-row
// compaction, row gather, merge of per-tile statistics, the deterministic
// loss mean, bias-gradient column sums and the scatter of dH to all rows.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace flce {

constexpr int COMPACT_THREADS = 1024;
constexpr int kNoColumn = -(1 << 30);  // y_c of a label that another vocabulary slice holds

__device__ __forceinline__ bool is_supervised(const int64_t* labels, const uint8_t* mask,
                                              int64_t ignore, int64_t i) {
  return labels[i] != ignore && (mask == nullptr || mask[i] != 0);
}

// a_i = 1[mask_i] 1[y_i != ignore]; idx = supervised rows ascending (stable),
// y_c = their labels (optional), C = count ("分块交叉熵" page §01; the supervised-row
// filter of "ChunkedLinearCrossEntropy").  One block walks the rows in
// batches of COMPACT_BATCH chunks of COMPACT_THREADS consecutive rows (thread t
// takes row base + k * COMPACT_THREADS + t, so loads are coalesced and a batch's
// loads are all in flight at once); within a chunk a warp ballot and a scan of
// the 32 warp counts give each supervised row its output slot, chunks follow
// one another, so the order is ascending.  Labels outside [0, V) on
// supervised rows set the label error bit and are clamped to 0 so later
// indexing stays in range.  y_c holds y - v0, the label's column in the
// vocabulary slice [v0, v0 + V_slice) (the whole vocabulary unsharded), or
// kNoColumn when another slice holds it, so that no column of this slice ever
// matches it.  Unsupervised rows get m = log s = -inf when m_out is given.
// pos (optional) is the inverse map: pos[i] = compact row of i, or -1.
// lossvec (optional) gets 0 on unsupervised rows (per-row loss output).
constexpr int COMPACT_BATCH = 4;
__global__ void __launch_bounds__(COMPACT_THREADS)
    compact_kernel(const int64_t* __restrict__ labels, const uint8_t* __restrict__ mask,
                   int64_t ignore, int64_t N, int64_t V, int64_t v0, int64_t V_slice,
                   int* __restrict__ idx,
                   int* __restrict__ y_c, int* __restrict__ C_out, uint32_t* err,
                   float* __restrict__ m_out, float* __restrict__ logs_out,
                   int* __restrict__ pos, float* __restrict__ lossvec) {
  constexpr int NW = COMPACT_THREADS / 32;
  static_assert(NW == 32 && COMPACT_BATCH <= NW, "one scanning warp per chunk of the batch");
  __shared__ int warp_cnt[COMPACT_BATCH][NW];
  __shared__ int warp_off[COMPACT_BATCH][NW];
  __shared__ int chunk_tot[COMPACT_BATCH];
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  const unsigned lanes_below = (1u << lane) - 1u;
  int running = 0;  // rows written by the previous batches (the same in every thread)
  bool bad = false;
  for (int64_t base = 0; base < N; base += static_cast<int64_t>(COMPACT_THREADS) * COMPACT_BATCH) {
    int64_t y[COMPACT_BATCH];
    bool sup[COMPACT_BATCH];
    unsigned bal[COMPACT_BATCH];
#pragma unroll
    for (int k = 0; k < COMPACT_BATCH; ++k) {
      const int64_t i = base + static_cast<int64_t>(k) * COMPACT_THREADS + t;
      sup[k] = i < N && is_supervised(labels, mask, ignore, i);
      y[k] = sup[k] ? labels[i] : 0;
    }
#pragma unroll
    for (int k = 0; k < COMPACT_BATCH; ++k) {
      bal[k] = __ballot_sync(0xffffffffu, sup[k]);
      if (lane == 0) warp_cnt[k][warp] = __popc(bal[k]);
    }
    __syncthreads();
    if (warp < COMPACT_BATCH) {  // warp k: exclusive scan of chunk k's warp counts
      const int c = warp_cnt[warp][lane];
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      warp_off[warp][lane] = incl - c;
      if (lane == 31) chunk_tot[warp] = incl;
    }
    __syncthreads();
    int off = running;
#pragma unroll
    for (int k = 0; k < COMPACT_BATCH; ++k) {
      const int64_t i = base + static_cast<int64_t>(k) * COMPACT_THREADS + t;
      if (sup[k]) {
        const int o = off + warp_off[k][warp] + __popc(bal[k] & lanes_below);
        int64_t yy = y[k];
        if (yy < 0 || yy >= V) {
          bad = true;
          yy = 0;
        }
        idx[o] = static_cast<int>(i);
        if (y_c != nullptr)
          y_c[o] = (yy >= v0 && yy < v0 + V_slice) ? static_cast<int>(yy - v0) : kNoColumn;
        if (pos != nullptr) pos[i] = o;
      } else if (i < N) {
        if (m_out != nullptr) {
          m_out[i] = -INFINITY;
          logs_out[i] = -INFINITY;
        }
        if (pos != nullptr) pos[i] = -1;
        if (lossvec != nullptr) lossvec[i] = 0.f;
      }
      off += chunk_tot[k];
    }
    running = off;
    __syncthreads();  // the next batch reuses warp_cnt / warp_off / chunk_tot
  }
  if (t == 0) *C_out = running;
  if (bad) atomicOr(err, kErrBitLabel);
}

// H_c[k] = H[idx[k]] for k < C, zero rows for C <= k < Np (16-byte vectors,
// one warp per row).
__global__ void gather_rows_kernel(const uint4* __restrict__ H, const int* __restrict__ idx,
                                   const int* __restrict__ C_dev, int64_t Np, int64_t vec_per_row,
                                   uint4* __restrict__ Hc) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= Np) return;
  const int lane = threadIdx.x & 31;
  const int C = *C_dev;
  uint4* dst = Hc + row * vec_per_row;
  if (row < C) {
    const uint4* src = H + static_cast<int64_t>(idx[row]) * vec_per_row;
    for (int64_t k = lane; k < vec_per_row; k += 32) dst[k] = __ldg(src + k);
  } else {
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int64_t k = lane; k < vec_per_row; k += 32) dst[k] = z;
  }
}

// Online-softmax merge of two partial states (m, s): the running update of
// the "分块交叉熵" page §02, in the two-state form of the maths-basics page
// (online softmax block merge).  -inf marks an empty state.
__device__ __forceinline__ void merge_state(float& m, float& s, float om, float os) {
  if (om == -INFINITY) return;
  if (m == -INFINITY) {
    m = om;
    s = os;
    return;
  }
  const float mn = fmaxf(m, om);
  s = s * expf(m - mn) + os * expf(om - mn);
  m = mn;
}

// Per supervised row: merge the per-vocabulary-tile partials (lane-strided,
// then a butterfly of warp shuffles, symmetric so that every lane ends with
// the same state), then m_i, log s_i and l_i = (m_i - target_i) + log s_i.
// loss_rows[i] = w_i l_i (compact order); lossvec[orig] = w_i l_i if given.
__global__ void merge_stats_kernel(const float2* __restrict__ part, int part_ld, int nvt,
                                   const float* __restrict__ tgt, const int* __restrict__ C_dev,
                                   const int* __restrict__ idx, float* __restrict__ m_out,
                                   float* __restrict__ logs_out, float* __restrict__ loss_rows,
                                   const float* __restrict__ weight,
                                   float* __restrict__ lossvec, uint32_t* err) {
  const int C = *C_dev;
  const int lane = threadIdx.x & 31;
  const int warps = (blockDim.x >> 5) * gridDim.x;
  for (int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < C; i += warps) {
    const float2* pr = part + static_cast<size_t>(i) * part_ld;
    float m = -INFINITY, s = 0.f;
    for (int v = lane; v < nvt; v += 32) {
      const float2 ps = pr[v];
      merge_state(m, s, ps.x, ps.y);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float om = __shfl_xor_sync(0xffffffffu, m, o);
      const float os = __shfl_xor_sync(0xffffffffu, s, o);
      merge_state(m, s, om, os);
    }
    if (lane == 0) {
      const float logs = logf(s);
      const float li = (m - tgt[i]) + logs;
      const int o = idx[i];
      m_out[o] = m;
      logs_out[o] = logs;
      const float wl = (weight != nullptr) ? weight[o] * li : li;
      loss_rows[i] = wl;
      if (lossvec != nullptr) lossvec[o] = wl;
      if (!isfinite(li) || !isfinite(m) || !isfinite(logs)) atomicOr(err, kErrBitNonfinite);
    }
  }
}

// Vocabulary slice [v0, v0 + V_slice): per ORIGINAL row i the partial
// statistics (m_r, log s_r, t_r, o_r) of the slice's columns: the merged
// tile partials, the target logit when the slice holds the label (y_c in
// [0, V_slice)) else 0, and the ownership flag.  Unsupervised rows (pos < 0)
// get the recurrence's initial state (-inf, -inf, 0, 0).  One warp per row.
__global__ void shard_stats_kernel(const float2* __restrict__ part, int part_ld, int nvt,
                                   const float* __restrict__ tgt, const int* __restrict__ y_c,
                                   const int* __restrict__ pos, int64_t N, int V_slice,
                                   float4* __restrict__ stats, uint32_t* err) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(blockDim.x >> 5) * gridDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       i < N; i += warps) {
    const int k = pos[i];
    if (k < 0) {
      if (lane == 0) stats[i] = make_float4(-INFINITY, -INFINITY, 0.f, 0.f);
      continue;
    }
    const float2* pr = part + static_cast<size_t>(k) * part_ld;
    float m = -INFINITY, s = 0.f;
    for (int v = lane; v < nvt; v += 32) {
      const float2 ps = pr[v];
      merge_state(m, s, ps.x, ps.y);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float om = __shfl_xor_sync(0xffffffffu, m, o);
      const float os = __shfl_xor_sync(0xffffffffu, s, o);
      merge_state(m, s, om, os);
    }
    if (lane == 0) {
      const float logs = logf(s);
      const bool own = static_cast<unsigned>(y_c[k]) < static_cast<unsigned>(V_slice);
      stats[i] = make_float4(m, logs, own ? tgt[k] : 0.f, own ? 1.f : 0.f);
      if (!isfinite(m) || !isfinite(logs)) atomicOr(err, kErrBitNonfinite);
    }
  }
}

// Merge of the slices' partial statistics stats[r * N + i], r < P (the
// two-state online-softmax merge, maths-basics page worked example 9.4, in
// log form): M = max_r m_r, log S = log sum_r exp((m_r - M) + log s_r),
// target = the owning slice's t_r, l = (M - target) + log S ("分块交叉熵"
// §02).  Per supervised row k (original row o = idx[k]): m_out[o], logs_out[o],
// loss_rows[k] = w_o l and lossvec[o] = w_o l when given.  A row owned by no
// slice or by several sets the shard error bit.  One thread per row.
__global__ void shard_combine_kernel(const float4* __restrict__ stats, int P, int64_t N,
                                     const int* __restrict__ C_dev, const int* __restrict__ idx,
                                     float* __restrict__ m_out, float* __restrict__ logs_out,
                                     float* __restrict__ loss_rows,
                                     const float* __restrict__ weight,
                                     float* __restrict__ lossvec, uint32_t* err) {
  const int C = *C_dev;
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < C; k += blockDim.x * gridDim.x) {
    const int o = idx[k];
    float M = -INFINITY;
    for (int r = 0; r < P; ++r) M = fmaxf(M, stats[static_cast<int64_t>(r) * N + o].x);
    float S = 0.f, t = 0.f;
    int owners = 0;
    for (int r = 0; r < P; ++r) {
      const float4 q = stats[static_cast<int64_t>(r) * N + o];
      if (q.x != -INFINITY) S += expf((q.x - M) + q.y);
      if (q.w != 0.f) {
        t = q.z;
        ++owners;
      }
    }
    const float logs = logf(S);
    const float li = (M - t) + logs;
    m_out[o] = M;
    logs_out[o] = logs;
    const float wl = (weight != nullptr) ? weight[o] * li : li;
    loss_rows[k] = wl;
    if (lossvec != nullptr) lossvec[o] = wl;
    if (owners != 1) atomicOr(err, kErrBitShard);
    if (!isfinite(li) || !isfinite(M) || !isfinite(logs)) atomicOr(err, kErrBitNonfinite);
  }
}

// L = sum_i loss_rows[i] / den in a fixed order (per-thread strided sums in
// double, then a fixed tree), den = C for the mean and `denom` (or 1) for the
// sum; 0 when C = 0; NaN when the label, timeout or shard bit is set.
__global__ void __launch_bounds__(1024)
    loss_reduce_kernel(const float* __restrict__ loss_rows, const int* __restrict__ C_dev,
                       int is_mean, float denom, const uint32_t* err, float* __restrict__ loss) {
  __shared__ double red[1024];
  const int C = *C_dev;
  double acc = 0.0;
  for (int i = threadIdx.x; i < C; i += blockDim.x) acc += static_cast<double>(loss_rows[i]);
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double den = is_mean ? static_cast<double>(C) : (denom > 0.f ? denom : 1.0);
    float L = (C > 0) ? static_cast<float>(red[0] / den) : 0.f;
    if (*err & (kErrBitLabel | kErrBitTimeout | kErrBitShard)) L = __int_as_float(0x7fc00000);
    *loss = L;
  }
}

// Backward row scales: s_k = lambda w_o / den (mean, sum) or g_o w_o (per-row
// upstream gradients), o = idx[k].  Stores r_k = s_k / S and *scal = S with
// S = max_k |s_k| (r = 0 when S = 0), so that the 16-bit gradient panel holds
// r_k (p - onehot) sigma in range and the contractions multiply by S / sigma.
// One block, fixed-order reduction.
__global__ void __launch_bounds__(1024)
    row_scale_kernel(const int* __restrict__ C_dev, const int* __restrict__ idx,
                     const float* __restrict__ weight, const float* __restrict__ grad_rows,
                     int reduction, float denom, float lam, const float* __restrict__ lam_dev,
                     float* __restrict__ r, float* __restrict__ scal) {
  __shared__ float red[1024];
  const int C = *C_dev;
  float base = 0.f;
  if (grad_rows == nullptr) {
    const float l = (lam_dev != nullptr) ? *lam_dev : lam;
    const float den = (reduction == 0) ? static_cast<float>(C) : (denom > 0.f ? denom : 1.f);
    base = (C > 0) ? l / den : 0.f;
  }
  float mx = 0.f;
  for (int k = threadIdx.x; k < C; k += blockDim.x) {
    const int o = idx[k];
    float sk = (grad_rows != nullptr) ? grad_rows[o] : base;
    if (weight != nullptr) sk *= weight[o];
    r[k] = sk;
    mx = fmaxf(mx, fabsf(sk));
  }
  red[threadIdx.x] = mx;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] = fmaxf(red[threadIdx.x], red[threadIdx.x + w]);
    __syncthreads();
  }
  const float S = red[0];
  for (int k = threadIdx.x; k < C; k += blockDim.x) r[k] = (S > 0.f) ? r[k] / S : 0.f;
  if (threadIdx.x == 0) *scal = S;
}

// db[vp + j] = (S / sigma) * sum_{i < C} (Gp[i][j] + [y_i = vp + j] e_i) for the
// panel's columns, in two passes with a fixed order.  e_i is what the 16-bit
// rounding took off row i's target entry (recorded by the gradient units), so
// the target terms enter db exactly.
// Pass 1: block (x, s) sums 256 columns over the rows of split s (rows
// s * ceil(C / gridDim.y) ...): warp g takes rows g, g + 8, ... of the split
// (four rows' 16-byte loads in flight per lane, 8 columns each); the 8 warps'
// sums are added in warp order into bpart[s][j].  A lane reads up to 7
// columns past the panel width, inside the panel row (whose pitch is a
// multiple of 256 columns); those columns are never written out.
constexpr int BIAS_SPLITS = 32;
__global__ void __launch_bounds__(256)
    bias_partial_kernel(const uint16_t* __restrict__ Gp, int64_t ldg, int w,
                        const int* __restrict__ C_dev, int is_bf16, int vp,
                        const int* __restrict__ y_c, const float* __restrict__ tgt_resid,
                        float* __restrict__ bpart) {
  __shared__ float part[8][256];
  const int C = *C_dev;
  const int lane = threadIdx.x & 31, grp = threadIdx.x >> 5;
  const int j0 = blockIdx.x * 256 + lane * 8;  // this lane's 8 columns
  const int per = (C + static_cast<int>(gridDim.y) - 1) / static_cast<int>(gridDim.y);
  const int r0 = static_cast<int>(blockIdx.y) * per;
  const int r1 = min(C, r0 + per);
  float acc[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) acc[t] = 0.f;
  auto add_row = [&](const uint4& v, int i) {
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    float g[8];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      if (is_bf16) {
        g[2 * h] = __uint_as_float(wv[h] << 16);
        g[2 * h + 1] = __uint_as_float(wv[h] & 0xFFFF0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[h]));
        g[2 * h] = f.x;
        g[2 * h + 1] = f.y;
      }
    }
    const int yc = __ldg(y_c + i) - vp - j0;  // the row's label among this lane's columns
    if (static_cast<unsigned>(yc) < 8u) {
      const float e = __ldg(tgt_resid + i);
#pragma unroll
      for (int t = 0; t < 8; ++t)
        if (t == yc) g[t] += e;
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] += g[t];
  };
  if (j0 < w) {
    int i = r0 + grp;
    for (; i + 24 < r1; i += 32) {  // four rows per step, loads first
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = __ldg(reinterpret_cast<const uint4*>(Gp + static_cast<int64_t>(i + 8 * u) * ldg + j0));
#pragma unroll
      for (int u = 0; u < 4; ++u) add_row(v[u], i + 8 * u);
    }
    for (; i < r1; i += 8)
      add_row(__ldg(reinterpret_cast<const uint4*>(Gp + static_cast<int64_t>(i) * ldg + j0)), i);
  }
#pragma unroll
  for (int t = 0; t < 8; ++t) part[grp][lane * 8 + t] = acc[t];
  __syncthreads();
  const int j = blockIdx.x * 256 + threadIdx.x;
  if (j < w) {
    float t = part[0][threadIdx.x];
#pragma unroll
    for (int k = 1; k < 8; ++k) t += part[k][threadIdx.x];
    bpart[static_cast<int64_t>(blockIdx.y) * w + j] = t;
  }
}

// Pass 2: db[vp + j] = (S / sigma) * sum_s bpart[s][j], splits in order.
__global__ void bias_finish_kernel(const float* __restrict__ bpart, int splits, int w,
                                   const int* __restrict__ C_dev, const float* __restrict__ scal,
                                   float inv_sigma, int vp, float* __restrict__ db) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= w) return;
  float t = 0.f;
  for (int sp = 0; sp < splits; ++sp) t += bpart[static_cast<int64_t>(sp) * w + j];
  const float scale = (*C_dev > 0) ? *scal * inv_sigma : 0.f;
  db[vp + j] = t * scale;
}

// dH[i] = dH_c[pos[i]] + (S / sigma) e_k W[y_k] for supervised rows (k =
// pos[i]), 0 for the others.  e_k is what the 16-bit rounding took off the
// row's target entry of the gradient panel, so this adds back the exact
// target term in fp32; labels of another vocabulary slice (y_k outside
// [0, V_slice)) carry none.  accumulate != 0: dH[i] += that value instead
// (unsupervised rows unchanged).  One warp per row, 16-byte vectors of dH.
__global__ void scatter_dh_kernel(const float4* __restrict__ dHc, const int* __restrict__ pos,
                                  int64_t N, int64_t vec_per_row, float4* __restrict__ dH,
                                  const float* __restrict__ tgt_resid,
                                  const int* __restrict__ y_c, const uint2* __restrict__ W,
                                  int is_bf16, int V_slice, const float* __restrict__ scal,
                                  float inv_sigma, int accumulate) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= N) return;
  const int lane = threadIdx.x & 31;
  const int p = pos[row];
  float4* dst = dH + row * vec_per_row;
  if (p >= 0) {
    const float4* src = dHc + static_cast<int64_t>(p) * vec_per_row;
    const int y = y_c[p];
    const float c = tgt_resid[p] * (*scal) * inv_sigma;
    if (c != 0.f && static_cast<unsigned>(y) < static_cast<unsigned>(V_slice)) {
      const uint2* wr = W + static_cast<int64_t>(y) * vec_per_row;
      for (int64_t k = lane; k < vec_per_row; k += 32) {
        const uint2 wv = __ldg(wr + k);
        float w0, w1, w2, w3;
        if (is_bf16) {
          w0 = __uint_as_float(wv.x << 16);
          w1 = __uint_as_float(wv.x & 0xFFFF0000u);
          w2 = __uint_as_float(wv.y << 16);
          w3 = __uint_as_float(wv.y & 0xFFFF0000u);
        } else {
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&wv.x));
          const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&wv.y));
          w0 = a.x;
          w1 = a.y;
          w2 = b.x;
          w3 = b.y;
        }
        float4 h = src[k];
        if (accumulate) {
          const float4 o = dst[k];
          h = make_float4(h.x + o.x, h.y + o.y, h.z + o.z, h.w + o.w);
        }
        dst[k] = make_float4(fmaf(c, w0, h.x), fmaf(c, w1, h.y), fmaf(c, w2, h.z),
                             fmaf(c, w3, h.w));
      }
    } else if (accumulate) {
      for (int64_t k = lane; k < vec_per_row; k += 32) {
        const float4 h = src[k], o = dst[k];
        dst[k] = make_float4(h.x + o.x, h.y + o.y, h.z + o.z, h.w + o.w);
      }
    } else {
      for (int64_t k = lane; k < vec_per_row; k += 32) dst[k] = src[k];
    }
  } else if (!accumulate) {
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t k = lane; k < vec_per_row; k += 32) dst[k] = z;
  }
}

// Sort keys for grouping the supervised rows by label: key = the row's label
// as a column of this vocabulary slice, or V_slice (sorts last, ignored) for
// padding rows and labels another slice holds; value = the compact row.
__global__ void label_sort_prep_kernel(const int* __restrict__ C_dev, const int* __restrict__ y_c,
                                       int64_t Np, int V_slice, uint32_t* __restrict__ keys,
                                       int* __restrict__ vals) {
  const int C = *C_dev;
  for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < Np;
       k += static_cast<int64_t>(blockDim.x) * gridDim.x) {
    const int y = k < C ? y_c[k] : -1;
    keys[k] = (y >= 0 && y < V_slice) ? static_cast<uint32_t>(y) : static_cast<uint32_t>(V_slice);
    vals[k] = static_cast<int>(k);
  }
}

// dW[v] += (S / sigma) sum_{k: y_k = v} e_k H_c[k], over the rows grouped by
// label (keys sorted stably, so each group's rows are in ascending order):
// the fp32 residuals of the 16-bit target entries (see scatter_dh_kernel),
// added once per label after every panel's dW is written.  One warp per
// (group start, 128-column chunk): a lane owns 4 columns; the group's row
// ids and residuals are read 32 at a time (one step ahead) and broadcast by
// shuffles, so the H loads of consecutive rows are independent.  Fixed
// order: deterministic.
__global__ void dw_target_resid_kernel(const uint32_t* __restrict__ keys,
                                       const int* __restrict__ rows, int64_t Np, int V_slice,
                                       const uint2* __restrict__ Hc, int64_t vec_per_row,
                                       int is_bf16, const float* __restrict__ tgt_resid,
                                       const float* __restrict__ scal, float inv_sigma,
                                       float4* __restrict__ dW) {
  const int lane = threadIdx.x & 31;
  const int64_t nchunk = (vec_per_row + 31) / 32;
  const int64_t warps = static_cast<int64_t>(blockDim.x >> 5) * gridDim.x;
  const float scale = (*scal) * inv_sigma;
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       w < Np * nchunk; w += warps) {
    const int64_t p = w / nchunk;
    const int64_t c = (w % nchunk) * 32 + lane;  // this lane's 4-column group
    const uint32_t v = keys[p];
    if (v >= static_cast<uint32_t>(V_slice) || (p > 0 && keys[p - 1] == v)) continue;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    // up to 32 rows of the group per step: row id and residual in lane order;
    // the next step's are fetched while this step's H rows load
    bool in = p + lane < Np && keys[p + lane] == v;
    int k = in ? rows[p + lane] : 0;
    float e = in ? tgt_resid[k] : 0.f;
    for (int64_t q0 = p;; q0 += 32) {
      const unsigned live = __ballot_sync(0xffffffffu, in);
      const int n = __popc(live);  // the group's rows are contiguous from q0
      bool in_next = false;
      int k_next = 0;
      float e_next = 0.f;
      if (n == 32) {
        const int64_t qn = q0 + 32 + lane;
        in_next = qn < Np && keys[qn] == v;
        k_next = in_next ? rows[qn] : 0;
        e_next = in_next ? tgt_resid[k_next] : 0.f;
      }
      for (int j0 = 0; j0 < n; j0 += 16) {
        // sixteen rows' loads in flight, then their terms in row order
        uint2 hv[16];
        float ej[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int kj = __shfl_sync(0xffffffffu, k, j0 + u);
          ej[u] = __shfl_sync(0xffffffffu, e, j0 + u);
          hv[u] = (j0 + u < n && c < vec_per_row)
                      ? __ldg(Hc + static_cast<int64_t>(kj) * vec_per_row + c)
                      : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          if (j0 + u >= n) break;
          float h0, h1, h2, h3;
          if (is_bf16) {
            h0 = __uint_as_float(hv[u].x << 16);
            h1 = __uint_as_float(hv[u].x & 0xFFFF0000u);
            h2 = __uint_as_float(hv[u].y << 16);
            h3 = __uint_as_float(hv[u].y & 0xFFFF0000u);
          } else {
            const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&hv[u].x));
            const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&hv[u].y));
            h0 = lo.x;
            h1 = lo.y;
            h2 = hi.x;
            h3 = hi.y;
          }
          a0 = fmaf(ej[u], h0, a0);
          a1 = fmaf(ej[u], h1, a1);
          a2 = fmaf(ej[u], h2, a2);
          a3 = fmaf(ej[u], h3, a3);
        }
      }
      if (n < 32) break;
      in = in_next;
      k = k_next;
      e = e_next;
    }
    if (c < vec_per_row) {
      float4* dst = dW + static_cast<int64_t>(v) * vec_per_row + c;
      const float4 o = *dst;
      *dst = make_float4(fmaf(scale, a0, o.x), fmaf(scale, a1, o.y), fmaf(scale, a2, o.z),
                         fmaf(scale, a3, o.w));
    }
  }
}

// Failure-path check: waits on a barrier nothing completes, with a short
// limit; the bounded wait records the timeout bit and the kernel returns.
__global__ void timeout_probe_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(&bar, 0, &abort_flag, err, limit_ns);
    if (ok) atomicOr(err, 1u << 31);  // impossible: nothing arrives on `bar`
  }
}

}  // namespace flce
