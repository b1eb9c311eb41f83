// Token-level top-k selection with the forced recent window.
//
// Scores are non-negative fp32 values, so their bit patterns order like the
// values.  The k-th largest pattern tau is found digit by digit from three
// histograms (bits [30:20] -- built by attn_score --, [19:9], [8:0]); then one
// ordered pass keeps every candidate above tau and the first `need` equal to
// tau (ties go to the lower position), writing positions in ascending order,
// followed by the window positions i-window+1 .. i.
#pragma once

#include "hs2_common.cuh"

namespace hs2 {

constexpr int kSelThreads = 1024;

struct SelectParams {
  const float* score;     // [B*T][L]
  const unsigned* hist;   // [B*T][2048]  level-1 counts
  int32_t* idx;           // [B*T][slots]
  int32_t* n_sel;         // [B*T]
  int T;
  long long L;
  int topk, window, slots;
};

// Exclusive prefix sum over the block (1024 threads); returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int& excl, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
    int s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_tot[32 + lane] = s - w;  // exclusive prefix of warp totals
    if (lane == 31) warp_tot[64] = s;
  }
  __syncthreads();
  excl = x - v + warp_tot[32 + warp];
  const int total = warp_tot[64];
  __syncthreads();
  return total;
}

// Given counts hist[0..nbins) and k >= 1, finds the bin `sel` holding the
// k-th largest element: count(bins > sel) < k <= count(bins >= sel).
// Writes sel and need = k - count(bins > sel) to out[0], out[1].
__device__ __forceinline__ void find_kth_bin(const unsigned* hist, int nbins, int k, int* out,
                                             int* warp_tot) {
  const int per = (nbins + kSelThreads - 1) / kSelThreads;
  // thread 0 owns the highest bins
  const int hi = nbins - threadIdx.x * per;  // exclusive upper bin
  const int lo = max(0, hi - per);
  int local = 0;
  for (int bb = lo; bb < hi; ++bb) local += (int)hist[bb];
  int excl;
  block_exclusive_scan(local, excl, warp_tot);
  if (excl < k && k <= excl + local) {
    int above = excl;
    for (int bb = hi - 1; bb >= lo; --bb) {
      const int cnt = (int)hist[bb];
      if (above + cnt >= k) {
        out[0] = bb;
        out[1] = k - above;
        break;
      }
      above += cnt;
    }
  }
  __syncthreads();
}

// SMEM = true: the candidate scores of the row are first copied to dynamic
// shared memory (rows of at most kSelSmemMax candidates), and every later pass
// reads them there.  SMEM = false: passes read the row in global memory.
constexpr int kSelSmemMax = 48 * 1024;

template <bool SMEM>
__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(const SelectParams p) {
  __shared__ unsigned hist[2048];
  __shared__ int warp_tot[72];
  __shared__ int res[2];
  extern __shared__ unsigned row_s[];
  const long long row = blockIdx.x;
  const int t = (int)(row % p.T);
  const long long i = p.L - p.T + t;
  const long long nc = i - p.window + 1;  // candidates 0 .. nc-1
  int32_t* out = p.idx + row * p.slots;

  if (nc <= p.topk) {  // every candidate is taken: S = {0 .. i}
    const long long n = i + 1;
    for (long long j = threadIdx.x; j < p.slots; j += kSelThreads) out[j] = j < n ? (int32_t)j : -1;
    if (threadIdx.x == 0) p.n_sel[row] = (int32_t)n;
    return;
  }
  const unsigned* srow_u = reinterpret_cast<const unsigned*>(p.score + row * p.L);
  if (SMEM) {
    // 16-byte copies where the row start allows it (p.L % 4 == 0), else words
    if ((p.L & 3) == 0) {
      const uint4* g4 = reinterpret_cast<const uint4*>(srow_u);
      uint4* s4 = reinterpret_cast<uint4*>(row_s);
      for (long long j = threadIdx.x; j < nc / 4; j += kSelThreads) s4[j] = g4[j];
      for (long long j = (nc / 4) * 4 + threadIdx.x; j < nc; j += kSelThreads) row_s[j] = srow_u[j];
    } else {
      for (long long j = threadIdx.x; j < nc; j += kSelThreads) row_s[j] = srow_u[j];
    }
    __syncthreads();
    srow_u = row_s;
  }
  int need = p.topk;
  unsigned prefix = 0;
  if (need > 0) {
    // level 1: bits [30:20]
    find_kth_bin(p.hist + row * 2048, 2048, need, res, warp_tot);
    prefix = (unsigned)res[0];
    need = res[1];
    // level 2: bits [19:9] among elements with bits[30:20] == prefix
    for (int u = threadIdx.x; u < 2048; u += kSelThreads) hist[u] = 0u;
    __syncthreads();
    for (long long j = threadIdx.x; j < nc; j += kSelThreads) {
      const unsigned v = srow_u[j];
      if ((v >> 20) == prefix) atomicAdd(&hist[(v >> 9) & 2047u], 1u);
    }
    __syncthreads();
    find_kth_bin(hist, 2048, need, res, warp_tot);
    prefix = (prefix << 11) | (unsigned)res[0];
    need = res[1];
    // level 3: bits [8:0] among elements with bits[30:9] == prefix
    for (int u = threadIdx.x; u < 512; u += kSelThreads) hist[u] = 0u;
    __syncthreads();
    for (long long j = threadIdx.x; j < nc; j += kSelThreads) {
      const unsigned v = srow_u[j];
      if ((v >> 9) == prefix) atomicAdd(&hist[v & 511u], 1u);
    }
    __syncthreads();
    find_kth_bin(hist, 512, need, res, warp_tot);
    prefix = (prefix << 9) | (unsigned)res[0];
    need = res[1];
  }
  const unsigned tau = prefix;
  // Ordered compaction of {v > tau} and the first `need` of {v == tau}.  Warp w
  // owns the contiguous segment [w*seg, (w+1)*seg) of the candidates: a first
  // pass counts its survivors (ballots), one block scan orders the warps, and a
  // second pass writes each warp's survivors at its offset, in index order.
  if (p.topk > 0) {
    __shared__ int wsel[32], weq[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long seg = (nc + 31) / 32;
    const long long s0 = warp * seg, s1 = min(nc, s0 + seg);
    int n_gt = 0, n_eq = 0;
    for (long long base = s0; base < s1; base += 32) {
      const long long j = base + lane;
      const unsigned v = j < s1 ? srow_u[j] : 0u;
      n_gt += __popc(__ballot_sync(0xffffffffu, j < s1 && v > tau));
      n_eq += __popc(__ballot_sync(0xffffffffu, j < s1 && v == tau));
    }
    if (lane == 0) {
      wsel[warp] = n_gt;
      weq[warp] = n_eq;
    }
    __syncthreads();
    int gt_before = 0, eq_before = 0;
    for (int w = 0; w < warp; ++w) {
      gt_before += wsel[w];
      eq_before += weq[w];
    }
    // equal elements taken by this warp: those of rank < need overall
    int pos = gt_before + min(eq_before, need);
    int eq_rank = eq_before;
    for (long long base = s0; base < s1; base += 32) {
      const long long j = base + lane;
      const unsigned v = j < s1 ? srow_u[j] : 0u;
      const bool gt = j < s1 && v > tau;
      const bool eq = j < s1 && v == tau;
      const unsigned eqm = __ballot_sync(0xffffffffu, eq);
      const int my_eq_rank = eq_rank + __popc(eqm & ((1u << lane) - 1u));
      const bool sel = gt || (eq && my_eq_rank < need);
      const unsigned selm = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const int o = pos + __popc(selm & ((1u << lane) - 1u));
        if (o < p.topk) out[o] = (int32_t)j;
      }
      pos += __popc(selm);
      eq_rank += __popc(eqm);
    }
    if (warp == 31 && lane == 0 && pos != p.topk) raise_status(kStatusBadIndex);
  }
  const long long w0 = i - p.window + 1;
  for (int w = threadIdx.x; w < p.window; w += kSelThreads) out[p.topk + w] = (int32_t)(w0 + w);
  for (int s = p.topk + p.window + threadIdx.x; s < p.slots; s += kSelThreads) out[s] = -1;
  if (threadIdx.x == 0) p.n_sel[row] = p.topk + p.window;
}

}  // namespace hs2
