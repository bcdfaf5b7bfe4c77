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
// (online softmax block merge).  -inf marks an empty state.  Only the
// smaller state is rescaled, so one exponential per merge.
__device__ __forceinline__ void merge_state(float& m, float& s, float om, float os) {
  if (om == -INFINITY) return;
  if (m == -INFINITY) {
    m = om;
    s = os;
    return;
  }
  if (om <= m) {
    s += os * expf(om - m);
  } else {
    s = s * expf(m - om) + os;
    m = om;
  }
}

// Per-tile forward partials are stored tile-major: part[v * ld + k] is the
// (m, s) of compact row k over vocabulary tile v.  A block of 512 threads
// merges the partials of 32 rows: thread (t, r) = (threadIdx.x / 32,
// threadIdx.x % 32) takes tiles t, t + 16, ... of row r (each warp reads 32
// consecutive rows of one tile: 256 contiguous bytes), eight loads in
// flight, then thread (0, r) merges the 16 lane states in t order.  Fixed
// order: deterministic.  (Latency-bound: 8 splits with 4 loads in flight
// took 35 us for 970 tiles x 11472 rows.)
constexpr int MERGE_ROWS = 32;
constexpr int MERGE_SPLIT = 16;

__device__ __forceinline__ float2 merge_row_tiles(const float2* __restrict__ part, int64_t ld,
                                                  int nvt, int k, bool live,
                                                  float2 (&sh)[MERGE_SPLIT][MERGE_ROWS]) {
  const int r = threadIdx.x & 31, t = threadIdx.x >> 5;
  float m = -INFINITY, s = 0.f;
  if (live) {
    int v = t;
    for (; v + 7 * MERGE_SPLIT < nvt; v += 8 * MERGE_SPLIT) {  // eight loads in flight
      float2 q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) q[u] = part[static_cast<int64_t>(v + u * MERGE_SPLIT) * ld + k];
#pragma unroll
      for (int u = 0; u < 8; ++u) merge_state(m, s, q[u].x, q[u].y);
    }
    for (; v < nvt; v += MERGE_SPLIT) {
      const float2 q = part[static_cast<int64_t>(v) * ld + k];
      merge_state(m, s, q.x, q.y);
    }
  }
  sh[t][r] = make_float2(m, s);
  __syncthreads();
  float2 out = make_float2(-INFINITY, 0.f);
  if (t == 0) {
    float mm = -INFINITY, ss = 0.f;
#pragma unroll
    for (int j = 0; j < MERGE_SPLIT; ++j) merge_state(mm, ss, sh[j][r].x, sh[j][r].y);
    out = make_float2(mm, ss);
  }
  __syncthreads();
  return out;
}

// Per supervised row: merge the per-vocabulary-tile partials, then m_i,
// log s_i and l_i = (m_i - target_i) + log s_i.  loss_rows[i] = w_i l_i
// (compact order); lossvec[orig] = w_i l_i if given.
__global__ void __launch_bounds__(MERGE_ROWS * MERGE_SPLIT)
    merge_stats_kernel(const float2* __restrict__ part, int64_t ld, int nvt,
                       const float* __restrict__ tgt, const int* __restrict__ C_dev,
                       const int* __restrict__ idx, float* __restrict__ m_out,
                       float* __restrict__ logs_out, float* __restrict__ loss_rows,
                       const float* __restrict__ weight, float* __restrict__ lossvec,
                       uint32_t* err) {
  __shared__ float2 sh[MERGE_SPLIT][MERGE_ROWS];
  const int C = *C_dev;
  for (int base = blockIdx.x * MERGE_ROWS; base < C; base += gridDim.x * MERGE_ROWS) {
    const int i = base + (threadIdx.x & 31);
    const float2 ms = merge_row_tiles(part, ld, nvt, i, i < C, sh);
    if (threadIdx.x < 32 && i < C) {
      const float m = ms.x;
      const float logs = logf(ms.y);
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
// get the recurrence's initial state (-inf, -inf, 0, 0).  32 rows per block
// pass, as in merge_stats_kernel.
__global__ void __launch_bounds__(MERGE_ROWS * MERGE_SPLIT)
    shard_stats_kernel(const float2* __restrict__ part, int64_t ld, int nvt,
                       const float* __restrict__ tgt, const int* __restrict__ y_c,
                       const int* __restrict__ pos, int64_t N, int V_slice,
                       float4* __restrict__ stats, uint32_t* err) {
  __shared__ float2 sh[MERGE_SPLIT][MERGE_ROWS];
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * MERGE_ROWS; base < N;
       base += static_cast<int64_t>(gridDim.x) * MERGE_ROWS) {
    const int64_t i = base + (threadIdx.x & 31);
    const int k = i < N ? pos[i] : -1;
    const float2 ms = merge_row_tiles(part, ld, nvt, k, k >= 0, sh);
    if (threadIdx.x < 32 && i < N) {
      if (k < 0) {
        stats[i] = make_float4(-INFINITY, -INFINITY, 0.f, 0.f);
      } else {
        const float logs = logf(ms.y);
        const bool own = static_cast<unsigned>(y_c[k]) < static_cast<unsigned>(V_slice);
        stats[i] = make_float4(ms.x, logs, own ? tgt[k] : 0.f, own ? 1.f : 0.f);
        if (!isfinite(ms.x) || !isfinite(logs)) atomicOr(err, kErrBitNonfinite);
      }
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

// db[j] = S * acc[j] * 2^-32: the bias gradient from the fixed-point column
// sums that the gradient units added (acc[j] = 2^32 sum_i r_i (p_ij -
// 1[j = y_i]), exact integer additions, so the result does not depend on
// their order); 0 when C = 0.
__global__ void bias_finish_kernel(const unsigned long long* __restrict__ acc, int V,
                                   const int* __restrict__ C_dev, const float* __restrict__ scal,
                                   float* __restrict__ db) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= V) return;
  const double q = static_cast<double>(static_cast<long long>(acc[j]));
  db[j] = (*C_dev > 0) ? static_cast<float>(q * 0x1p-32 * static_cast<double>(*scal)) : 0.f;
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

// Stable least-significant-digit radix sort of (key, row) pairs by key, used to
// group the supervised rows by label: 8-bit digits, one pass per digit, each
// pass three kernels -- per-tile digit counts, one exclusive scan over the
// counts (digit-major, so that tiles keep their order inside a digit), and a
// scatter in which every element's rank among the equal digits of its tile
// comes from warp match masks and per-warp counts.  All ranks are fixed by the
// input order, so the result is the stable sort whatever the schedule.
constexpr int RS_BITS = 8;
constexpr int RS_DIGITS = 1 << RS_BITS;
constexpr int RS_TILE = 1024;  // one element per thread

__global__ void __launch_bounds__(RS_TILE)
    radix_count_kernel(const uint32_t* __restrict__ keys, int64_t n, int shift,
                       int* __restrict__ counts) {
  __shared__ int h[RS_DIGITS];
  for (int d = threadIdx.x; d < RS_DIGITS; d += blockDim.x) h[d] = 0;
  __syncthreads();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * RS_TILE + threadIdx.x;
  if (i < n) atomicAdd(&h[(keys[i] >> shift) & (RS_DIGITS - 1)], 1);
  __syncthreads();
  for (int d = threadIdx.x; d < RS_DIGITS; d += blockDim.x)
    counts[static_cast<int64_t>(d) * gridDim.x + blockIdx.x] = h[d];
}

// In-place exclusive scan of `total` ints with one block: each thread scans a
// contiguous run, then the runs' sums are scanned across the block.
__global__ void __launch_bounds__(1024) radix_scan_kernel(int* __restrict__ a, int64_t total) {
  __shared__ int sums[1024];
  const int t = threadIdx.x;
  const int64_t per = (total + blockDim.x - 1) / blockDim.x;
  const int64_t b0 = t * per, b1 = min(total, b0 + per);
  int run = 0;
  for (int64_t i = b0; i < b1; ++i) run += a[i];
  sums[t] = run;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {  // inclusive scan of the run sums
    const int v = t >= off ? sums[t - off] : 0;
    __syncthreads();
    sums[t] += v;
    __syncthreads();
  }
  int acc = sums[t] - run;
  for (int64_t i = b0; i < b1; ++i) {
    const int v = a[i];
    a[i] = acc;
    acc += v;
  }
}

__global__ void __launch_bounds__(RS_TILE)
    radix_scatter_kernel(const uint32_t* __restrict__ keys, const int* __restrict__ vals,
                         int64_t n, int shift, const int* __restrict__ offsets,
                         uint32_t* __restrict__ keys_out, int* __restrict__ vals_out) {
  constexpr int NW = RS_TILE / 32;
  __shared__ int cnt[NW][RS_DIGITS];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int j = threadIdx.x; j < NW * RS_DIGITS; j += blockDim.x) (&cnt[0][0])[j] = 0;
  __syncthreads();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * RS_TILE + threadIdx.x;
  const bool live = i < n;
  const uint32_t k = live ? keys[i] : 0u;
  const int d = live ? static_cast<int>((k >> shift) & (RS_DIGITS - 1)) : RS_DIGITS;
  const unsigned peers = __match_any_sync(0xffffffffu, d);
  const int below = __popc(peers & ((1u << lane) - 1u));
  if (live && below == 0) cnt[warp][d] = __popc(peers);
  __syncthreads();
  if (threadIdx.x < RS_DIGITS) {  // per digit: counts of the earlier warps
    int run = 0;
    for (int w = 0; w < NW; ++w) {
      const int c = cnt[w][threadIdx.x];
      cnt[w][threadIdx.x] = run;
      run += c;
    }
  }
  __syncthreads();
  if (live) {
    const int64_t dst = offsets[static_cast<int64_t>(d) * gridDim.x + blockIdx.x] +
                        cnt[warp][d] + below;
    keys_out[dst] = k;
    vals_out[dst] = vals[i];
  }
}

// dW[v] += (S / sigma) sum_{k: y_k = v} e_k H_c[k], over the rows grouped by
// label (keys sorted stably, so each group's rows are in ascending order):
// the fp32 residuals of the 16-bit target entries (see scatter_dh_kernel),
// added once per label after every panel's dW is written.  A segmented sum
// in two passes over windows of 32 sorted positions, so that no warp walks a
// long group (the hottest label of a Zipf batch holds about a tenth of the
// rows):
//   pass 1 (dw_target_window_kernel), a warp per (window, 128-column chunk):
//     the window's runs of equal labels, each summed in row order; a run
//     that is a whole group is added to dW; otherwise its sum is kept in the
//     window's slot 0 (the run that begins at the window's start) or slot 1
//     (the run that begins inside the window and goes on past its end);
//   pass 2 (dw_target_chain_kernel), a warp per (window, chunk) whose last
//     run opens a group that goes on: the group's window sums in window
//     order, added to dW.
// Fixed order everywhere: deterministic.  A lane owns 4 columns.
constexpr int TW = 32;  // sorted positions per window

__device__ __forceinline__ void h4_to_f32(uint2 hv, bool bf16, float& h0, float& h1, float& h2,
                                          float& h3) {
  if (bf16) {
    h0 = __uint_as_float(hv.x << 16);
    h1 = __uint_as_float(hv.x & 0xFFFF0000u);
    h2 = __uint_as_float(hv.y << 16);
    h3 = __uint_as_float(hv.y & 0xFFFF0000u);
  } else {
    const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&hv.x));
    const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&hv.y));
    h0 = lo.x;
    h1 = lo.y;
    h2 = hi.x;
    h3 = hi.y;
  }
}

__global__ void dw_target_window_kernel(const uint32_t* __restrict__ keys,
                                        const int* __restrict__ rows, int64_t Np, int V_slice,
                                        const uint2* __restrict__ Hc, int64_t vec_per_row,
                                        int is_bf16, const float* __restrict__ tgt_resid,
                                        const float* __restrict__ scal, float inv_sigma,
                                        float4* __restrict__ win_sums, float4* __restrict__ dW) {
  const int lane = threadIdx.x & 31;
  const int64_t nchunk = (vec_per_row + 31) / 32;
  const int64_t nwin = (Np + TW - 1) / TW;
  const int64_t warps = static_cast<int64_t>(blockDim.x >> 5) * gridDim.x;
  const float scale = (*scal) * inv_sigma;
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       w < nwin * nchunk; w += warps) {
    const int64_t win = w / nchunk;
    const int64_t c = (w % nchunk) * 32 + lane;  // this lane's 4-column group
    const int64_t base = win * TW;
    const int n = static_cast<int>(Np - base < TW ? Np - base : TW);
    const uint32_t none = 0xFFFFFFFFu;
    const uint32_t key = lane < n ? keys[base + lane] : none;
    const bool counted = key < static_cast<uint32_t>(V_slice);
    const int k = counted ? rows[base + lane] : 0;
    const float e = counted ? tgt_resid[k] : 0.f;
    const uint32_t prev_key = base > 0 ? keys[base - 1] : none;
    const uint32_t next_key = base + TW < Np ? keys[base + TW] : none;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int run0 = 0;  // first window position of the current run
    // the current run [run0, j] ends at j: whole group or window slot
    auto flush = [&](uint32_t kv, bool ends_group) {
      if (kv < static_cast<uint32_t>(V_slice) && c < vec_per_row) {
        const bool starts_group = !(run0 == 0 && prev_key == kv);
        if (starts_group && ends_group) {
          float4* dst = dW + static_cast<int64_t>(kv) * vec_per_row + c;
          const float4 o = *dst;
          *dst = make_float4(fmaf(scale, a0, o.x), fmaf(scale, a1, o.y), fmaf(scale, a2, o.z),
                             fmaf(scale, a3, o.w));
        } else {
          win_sums[(win * 2 + (run0 == 0 ? 0 : 1)) * vec_per_row + c] =
              make_float4(a0, a1, a2, a3);
        }
      }
      a0 = a1 = a2 = a3 = 0.f;
    };
    for (int j0 = 0; j0 < n; j0 += 16) {
      // sixteen rows' loads in flight, then their terms in row order
      // (measured: all 32 at once needs more registers and ran slower)
      uint2 hv[16];
      float ej[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int kj = __shfl_sync(0xffffffffu, k, j0 + u);
        ej[u] = __shfl_sync(0xffffffffu, e, j0 + u);
        hv[u] = (j0 + u < n && c < vec_per_row && ej[u] != 0.f)
                    ? __ldg(Hc + static_cast<int64_t>(kj) * vec_per_row + c)
                    : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int j = j0 + u;
        const uint32_t kv = __shfl_sync(0xffffffffu, key, j);
        const uint32_t nk = __shfl_sync(0xffffffffu, key, (j + 1) & 31);
        if (j >= n) break;
        float h0, h1, h2, h3;
        h4_to_f32(hv[u], is_bf16 != 0, h0, h1, h2, h3);
        a0 = fmaf(ej[u], h0, a0);
        a1 = fmaf(ej[u], h1, a1);
        a2 = fmaf(ej[u], h2, a2);
        a3 = fmaf(ej[u], h3, a3);
        const uint32_t after = j + 1 < n ? nk : next_key;  // label of the next sorted position
        if (after != kv) {
          flush(kv, true);
          run0 = j + 1;
        } else if (j + 1 == n) {
          flush(kv, false);  // the group goes on in the next window
        }
      }
    }
  }
}

__global__ void dw_target_chain_kernel(const uint32_t* __restrict__ keys, int64_t Np,
                                       int V_slice, int64_t vec_per_row,
                                       const float4* __restrict__ win_sums,
                                       const float* __restrict__ scal, float inv_sigma,
                                       float4* __restrict__ dW) {
  const int lane = threadIdx.x & 31;
  const int64_t nchunk = (vec_per_row + 31) / 32;
  const int64_t nwin = (Np + TW - 1) / TW;
  const int64_t warps = static_cast<int64_t>(blockDim.x >> 5) * gridDim.x;
  const float scale = (*scal) * inv_sigma;
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       w < nwin * nchunk; w += warps) {
    const int64_t win = w / nchunk;
    const int64_t c = (w % nchunk) * 32 + lane;
    const int64_t base = win * TW;
    const int n = static_cast<int>(Np - base < TW ? Np - base : TW);
    const uint32_t v = keys[base + n - 1];  // label of the window's last run
    if (v >= static_cast<uint32_t>(V_slice)) continue;
    if (!(base + TW < Np && keys[base + TW] == v)) continue;  // the run ends here: pass 1 had it
    // where the last run begins: after the last position (below n) with another label
    const uint32_t key = lane < n ? keys[base + lane] : v;
    const unsigned other = __ballot_sync(0xffffffffu, key != v);
    const int run0 = other ? 32 - __clz(other) : 0;
    if (run0 == 0 && base > 0 && keys[base - 1] == v) continue;  // a window before opens it
    if (c >= vec_per_row) continue;
    float4 t = win_sums[(win * 2 + (run0 == 0 ? 0 : 1)) * vec_per_row + c];
    // the following windows eight at a time (loads in flight together); a
    // window's sum is added when the group reaches it, in window order
    bool go = true;
    for (int64_t w0 = win + 1; go && w0 < nwin; w0 += 8) {
      float4 u[8];
      bool cont[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int64_t ww = w0 + i;
        const int64_t nb = (ww + 1) * TW;
        u[i] = ww < nwin ? win_sums[(ww * 2) * vec_per_row + c] : make_float4(0.f, 0.f, 0.f, 0.f);
        cont[i] = nb < Np && keys[nb] == v;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (!go || w0 + i >= nwin) {
          go = false;
          break;
        }
        t.x += u[i].x;
        t.y += u[i].y;
        t.z += u[i].z;
        t.w += u[i].w;
        go = cont[i];
      }
    }
    float4* dst = dW + static_cast<int64_t>(v) * vec_per_row + c;
    const float4 o = *dst;
    *dst = make_float4(fmaf(scale, t.x, o.x), fmaf(scale, t.y, o.y), fmaf(scale, t.z, o.z),
                       fmaf(scale, t.w, o.w));
  }
}

// Accuracy check of the two exponentials the epilogues use: y_poly = ex2_poly(x),
// y_sfu = ex2.approx(x), element-wise.
__global__ void exp2_probe_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                  float* __restrict__ y_sfu, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  y_poly[i] = ex2_poly(x[i]);
  y_sfu[i] = ex2_approx(x[i]);
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
