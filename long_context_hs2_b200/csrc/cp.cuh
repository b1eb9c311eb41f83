// Context parallelism for the full-attention layer and its selection: the
// merge steps that follow each exchange between the G ranks that hold
// contiguous slices of a long context (the 1M-token chunk the pages analyse:
// dpshk.com explainer, section 05; cnyes.com article, cost paragraph).
//
// Each rank r holds positions [a_r, a_r + L_r) of every sequence and all the
// queries.  Per query row and head it computes the partial normaliser lse_r
// and the output O_r normalised over its slice (hs2_cp_attn_partial).  Then:
//   lse   = log sum_r exp(lse_r)                          (cp_lse_combine)
//   O     = sum_r exp(lse_r - lse) O_r                    (cp_rescale, then a sum
//                                                          all-reduce across ranks)
// With the global lse every rank scores its own candidates exactly as one
// device would, and keeps its top-k by (score descending, position ascending)
// (hs2_cp_select_local).  The global top-k is contained in the union of the
// ranks' lists, and the ranks' slices ascend, so the lists concatenated in
// rank order ascend too: cp_merge_select picks the top-k of the union in that
// order (ties to the lower position) and appends the window.
#pragma once

#include "select.cuh"

namespace hs2 {

// lse[n] = log sum_r exp(parts[r][n]) (natural log; -inf parts contribute nothing).
__global__ void __launch_bounds__(256) cp_lse_combine_kernel(const float* parts, int G, long long n,
                                                             float* lse) {
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    float m = -INFINITY;
    for (int r = 0; r < G; ++r) m = fmaxf(m, parts[(long long)r * n + e]);
    float s = 0.f;
    if (m != -INFINITY)
      for (int r = 0; r < G; ++r) s += __expf(parts[(long long)r * n + e] - m);
    lse[e] = m == -INFINITY ? m : m + __logf(s);
  }
}

// o[n][d] *= exp(lse_part[n] - lse[n]) (0 when the slice saw no key of row n).
__global__ void __launch_bounds__(256) cp_rescale_kernel(float* o, const float* lse_part,
                                                         const float* lse, long long n, int D) {
  const long long total = n * D;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long row = e / D;
    const float lp = lse_part[row];
    o[e] = lp == -INFINITY ? 0.f : o[e] * __expf(lp - lse[row]);
  }
}

constexpr int kCpThreads = 256;

struct CpMergeParams {
  const float* cand_score;  // [G][rows][topk]; -1 where cand_idx is -1
  const int32_t* cand_idx;  // [G][rows][topk] global positions, ascending per list, -1 padded
  int32_t* idx;             // [rows][topk + window]
  int32_t* n_sel;           // [rows]
  long long rows;
  int G, T, topk, window;
  long long qpos0;          // global position of query 0
};

// One CTA per query row.  Keys: score bit pattern + 1 for a valid candidate
// (scores are >= 0, so patterns order like the values), 0 for padding.
__global__ void __launch_bounds__(kCpThreads) cp_merge_select_kernel(const CpMergeParams p) {
  __shared__ unsigned h[2048];
  __shared__ int tmp[kCpThreads / 32];
  __shared__ int res[2];
  __shared__ int wsel[kCpThreads / 32];
  extern __shared__ unsigned key_s[];  // [G * topk]

  const long long row = blockIdx.x;
  const int t = (int)(row % p.T);
  const long long i = p.qpos0 + t;
  const int M = p.G * p.topk;
  const int slots = p.topk + p.window;
  int32_t* out = p.idx + row * slots;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int W = kCpThreads / 32;
  auto at = [&](int e) { return ((long long)(e / p.topk) * p.rows + row) * p.topk + e % p.topk; };

  int nv = 0;
  for (int e = threadIdx.x; e < M; e += kCpThreads) {
    const long long g = at(e);
    const bool valid = p.cand_idx[g] >= 0;
    key_s[e] = valid ? __float_as_uint(p.cand_score[g]) + 1u : 0u;
    nv += valid;
  }
  int nv_ex;
  nv = sel_block_scan<kCpThreads>(nv, nv_ex, tmp);
  const int keep = min(p.topk, nv);
  int need = keep;
  unsigned tau = 1u;   // keep every valid key when all fit
  if (nv > p.topk) {
    for (int b = threadIdx.x; b < 2048; b += kCpThreads) h[b] = 0u;
    __syncthreads();
    for (int e = threadIdx.x; e < M; e += kCpThreads)
      if (key_s[e]) atomicAdd(&h[key_s[e] >> 20], 1u);
    __syncthreads();
    sel_find_bin<kCpThreads>(h, 2048, need, res, tmp);
    unsigned prefix = (unsigned)res[0];
    need = res[1];
    for (int b = threadIdx.x; b < 2048; b += kCpThreads) h[b] = 0u;
    __syncthreads();
    for (int e = threadIdx.x; e < M; e += kCpThreads)
      if (key_s[e] && (key_s[e] >> 20) == prefix) atomicAdd(&h[(key_s[e] >> 9) & 2047u], 1u);
    __syncthreads();
    sel_find_bin<kCpThreads>(h, 2048, need, res, tmp);
    prefix = (prefix << 11) | (unsigned)res[0];
    need = res[1];
    for (int b = threadIdx.x; b < 512; b += kCpThreads) h[b] = 0u;
    __syncthreads();
    for (int e = threadIdx.x; e < M; e += kCpThreads)
      if (key_s[e] && (key_s[e] >> 9) == prefix) atomicAdd(&h[key_s[e] & 511u], 1u);
    __syncthreads();
    sel_find_bin<kCpThreads>(h, 512, need, res, tmp);
    tau = (prefix << 9) | (unsigned)res[0];
    need = res[1];
  } else {
    need = 0;   // every valid key is above tau - 1 ... kept through "gt" below
    tau = 0u;
  }
  // ordered compaction over the concatenated lists (ascending positions)
  const int wseg = (M + W - 1) / W;
  const int w0 = min(M, warp * wseg), w1 = min(M, w0 + wseg);
  int n_gt = 0, n_eq = 0;
  for (int base = w0; base < w1; base += 32) {
    const int e = base + lane;
    const unsigned v = e < w1 ? key_s[e] : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, e < w1 && v > tau));
    n_eq += __popc(__ballot_sync(0xffffffffu, e < w1 && v == tau && tau != 0u));
  }
  if (lane == 0) {
    wsel[warp] = n_gt;
    tmp[warp] = n_eq;
  }
  __syncthreads();
  int gt_before = 0, eq_before = 0;
  for (int w = 0; w < warp; ++w) {
    gt_before += wsel[w];
    eq_before += tmp[w];
  }
  int pos = gt_before + min(eq_before, need);
  int eq_rank = eq_before;
  for (int base = w0; base < w1; base += 32) {
    const int e = base + lane;
    const unsigned v = e < w1 ? key_s[e] : 0u;
    const bool gt = e < w1 && v > tau;
    const bool eq = e < w1 && v == tau && tau != 0u;
    const unsigned eqm = __ballot_sync(0xffffffffu, eq);
    const bool sel = gt || (eq && eq_rank + __popc(eqm & ((1u << lane) - 1u)) < need);
    const unsigned selm = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int o = pos + __popc(selm & ((1u << lane) - 1u));
      if (o < keep) out[o] = p.cand_idx[at(e)];
    }
    pos += __popc(selm);
    eq_rank += __popc(eqm);
  }
  if (warp == W - 1 && lane == 0 && pos != keep) raise_status(kStatusBadIndex);
  // the window, padding and count
  const long long w_lo = max(0LL, i - p.window + 1);
  const int nw = (int)(i - w_lo + 1);
  for (int w = threadIdx.x; w < nw; w += kCpThreads) out[keep + w] = (int32_t)(w_lo + w);
  for (int s = keep + nw + threadIdx.x; s < slots; s += kCpThreads) out[s] = -1;
  if (threadIdx.x == 0) p.n_sel[row] = keep + nw;
}

}  // namespace hs2
