// Block-level selection: the granularity of the HySparse generation before
// HySparse2, kept as the comparison variant of the token-level selection
// (dpshk.com explainer, section 03: history was chosen in blocks of 64 tokens,
// so a block with one useful token still takes 64 positions of the budget;
// cnyes.com article, section "檢索精確到token": the ablation keeps the same
// backbone and budget and compares the two granularities).
//
// Per query position i (candidates C = {0 .. i-window}, as for tokens): block
// b holds positions b*block .. b*block+block-1 and is a candidate when it holds
// a candidate position; its score is the sum of the head-summed scores of its
// candidate positions; the topk/block blocks of largest score (ties to the
// lower block) are kept, and S = their candidate positions, then the window
// positions i-window+1 .. i, in ascending order (-1 padded).  When there are
// no more candidate blocks than that, every position 0 .. i is taken.
//
// One CTA per query row.  The block sums (fp32, non-negative, so their bit
// patterns order like the values) are built from the row's scores into shared
// memory by the warps; the (topk/block)-th largest pattern tau is found from
// three digit histograms (bits [30:20], [19:9], [8:0]) as in the token-level
// selection; an ordered compaction in block order keeps every block above tau
// and the first `need` equal to tau; the kept blocks are expanded to
// positions.
#pragma once

#include "select.cuh"

namespace hs2 {

constexpr int kBlkThreads = 256;
constexpr int kBlkMaxBlocks = 48 * 1024;   // candidate blocks of one row held in shared memory
constexpr int kBlkMaxKeep = 4096;          // kept blocks (topk / block <= topk <= 4095)

struct BlockSelectParams {
  const float* score;   // [B*T][L] head-summed scores (candidates written)
  int32_t* idx;         // [B*T][slots]
  int32_t* n_sel;       // [B*T]
  int T;
  long long L;
  int topk, window, slots, block;
  int block_shift;      // log2(block) when block is a power of two, else -1
  long long qpos0;      // query t sits at position qpos0 + t
};

__global__ void __launch_bounds__(kBlkThreads) select_blocks_kernel(const BlockSelectParams p) {
  __shared__ unsigned h[2048];
  __shared__ int tmp[kBlkThreads / 32];
  __shared__ int res[2];
  __shared__ int wsel[kBlkThreads / 32];
  extern __shared__ unsigned bsum_s[];   // [nblk] block-sum patterns, then [keep] kept blocks

  pdl_launch_dependents();  // a following sparse layer may place its CTAs on idle SMs
  const long long row = blockIdx.x;
  const int t = (int)(row % p.T);
  const long long i = p.qpos0 + t;
  const long long last = i - p.window;                 // last candidate position
  const int nblk = last < 0 ? 0 : (int)(last / p.block) + 1;
  const int keep = p.topk / p.block;
  int32_t* out = p.idx + row * p.slots;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int W = kBlkThreads / 32;

  if (nblk <= keep) {  // every candidate block is kept: S = {0 .. i}
    const long long n = i + 1;
    for (long long j = threadIdx.x; j < p.slots; j += kBlkThreads) out[j] = j < n ? (int32_t)j : -1;
    if (threadIdx.x == 0) p.n_sel[row] = (int32_t)n;
    return;
  }
  // block sums: the row's candidate scores are streamed in coalesced passes of
  // kBlkUnroll independent loads per thread (the row was just written, so the
  // loads hit L2; what bounds this loop is how many are in flight) and added
  // into shared-memory sums -- per warp first when a warp's 32 positions lie in
  // one block (block a multiple of 32), else one shared atomic per position
  float* bsum_f = reinterpret_cast<float*>(bsum_s);
  for (int b = threadIdx.x; b < nblk; b += kBlkThreads) bsum_f[b] = 0.f;
  for (int b = threadIdx.x; b < 2048; b += kBlkThreads) h[b] = 0u;
  __syncthreads();
  const float* srow = p.score + row * p.L;
  const bool warp_blocks = (p.block & 31) == 0;
  constexpr int kBlkUnroll = 16;
  // positions fit 31 bits (L < 2^31): 32-bit block indices, a shift for a
  // power-of-two block
  auto block_of = [&](int j) { return p.block_shift >= 0 ? j >> p.block_shift : j / p.block; };
  const int last32 = (int)last;
  for (int base = 0; base <= last32; base += kBlkThreads * kBlkUnroll) {
    float x[kBlkUnroll];
#pragma unroll
    for (int u = 0; u < kBlkUnroll; ++u) {
      const int j = base + u * kBlkThreads + (int)threadIdx.x;
      x[u] = j <= last32 ? __ldcg(srow + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kBlkUnroll; ++u) {
      const int j = base + u * kBlkThreads + (int)threadIdx.x;
      if (warp_blocks) {
        float v = x[u];
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        const int j0 = j - lane;   // the warp's first position: same block for all lanes
        if (lane == 0 && j0 <= last32) atomicAdd(&bsum_f[block_of(j0)], v);
      } else if (j <= last32) {
        atomicAdd(&bsum_f[block_of(j)], x[u]);
      }
    }
  }
  __syncthreads();   // the sums are non-negative floats: their patterns order like the values

  // tau: the keep-th largest pattern, digit by digit
  int need = keep;
  unsigned prefix = 0;
  if (need > 0) {
    for (int b = threadIdx.x; b < nblk; b += kBlkThreads) atomicAdd(&h[bsum_s[b] >> 20], 1u);
    __syncthreads();
    sel_find_bin<kBlkThreads>(h, 2048, need, res, tmp);
    prefix = (unsigned)res[0];
    need = res[1];
    for (int b = threadIdx.x; b < 2048; b += kBlkThreads) h[b] = 0u;
    __syncthreads();
    for (int b = threadIdx.x; b < nblk; b += kBlkThreads) {
      const unsigned v = bsum_s[b];
      if ((v >> 20) == prefix) atomicAdd(&h[(v >> 9) & 2047u], 1u);
    }
    __syncthreads();
    sel_find_bin<kBlkThreads>(h, 2048, need, res, tmp);
    prefix = (prefix << 11) | (unsigned)res[0];
    need = res[1];
    for (int b = threadIdx.x; b < 512; b += kBlkThreads) h[b] = 0u;
    __syncthreads();
    for (int b = threadIdx.x; b < nblk; b += kBlkThreads) {
      const unsigned v = bsum_s[b];
      if ((v >> 9) == prefix) atomicAdd(&h[v & 511u], 1u);
    }
    __syncthreads();
    sel_find_bin<kBlkThreads>(h, 512, need, res, tmp);
    prefix = (prefix << 9) | (unsigned)res[0];
    need = res[1];
  }
  const unsigned tau = prefix;

  // ordered compaction of the kept blocks (warp w owns a contiguous range)
  int* kept = reinterpret_cast<int*>(bsum_s + nblk);
  const int wseg = (nblk + W - 1) / W;
  const int w0 = min(nblk, warp * wseg), w1 = min(nblk, w0 + wseg);
  int n_gt = 0, n_eq = 0;
  if (keep > 0)
    for (int base = w0; base < w1; base += 32) {
      const int b = base + lane;
      const unsigned v = b < w1 ? bsum_s[b] : 0u;
      n_gt += __popc(__ballot_sync(0xffffffffu, b < w1 && v > tau));
      n_eq += __popc(__ballot_sync(0xffffffffu, b < w1 && v == tau));
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
  if (keep > 0) {
    int pos = gt_before + min(eq_before, need);
    int eq_rank = eq_before;
    for (int base = w0; base < w1; base += 32) {
      const int b = base + lane;
      const unsigned v = b < w1 ? bsum_s[b] : 0u;
      const bool gt = b < w1 && v > tau;
      const bool eq = b < w1 && v == tau;
      const unsigned eqm = __ballot_sync(0xffffffffu, eq);
      const bool sel = gt || (eq && eq_rank + __popc(eqm & ((1u << lane) - 1u)) < need);
      const unsigned selm = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const int o = pos + __popc(selm & ((1u << lane) - 1u));
        if (o < keep) kept[o] = b;
      }
      pos += __popc(selm);
      eq_rank += __popc(eqm);
    }
    if (warp == W - 1 && lane == 0 && pos != keep) raise_status(kStatusBadIndex);
  }
  __syncthreads();
  // expansion: kept blocks ascend, and only the last candidate block can be
  // partial (it is then the last kept one), so kept block q starts at slot
  // q * block
  const int full_n = keep > 0 && kept[keep - 1] == nblk - 1
                         ? (keep - 1) * p.block + (int)(last + 1 - (long long)(nblk - 1) * p.block)
                         : keep * p.block;
  for (int e = threadIdx.x; e < full_n; e += kBlkThreads) {
    const int q = e / p.block;
    out[e] = (int32_t)((long long)kept[q] * p.block + (e - q * p.block));
  }
  const long long wstart = i - p.window + 1;
  for (int w = threadIdx.x; w < p.window; w += kBlkThreads) out[full_n + w] = (int32_t)(wstart + w);
  for (int s = full_n + p.window + threadIdx.x; s < p.slots; s += kBlkThreads) out[s] = -1;
  if (threadIdx.x == 0) p.n_sel[row] = full_n + p.window;
}

}  // namespace hs2
