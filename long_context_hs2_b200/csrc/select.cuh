// Token-level top-k selection with the forced recent window.
//
// Scores are non-negative fp32 values, so their bit patterns order like the
// values.  For each query the k-th largest pattern tau is found digit by
// digit from three histograms (bits [30:20] -- built by the score pass --,
// then [19:9] and [8:0] over the row); an ordered compaction then keeps every
// candidate above tau and the first `need` equal to tau (ties go to the lower
// position), writing positions in ascending order, followed by the window
// positions i-window+1 .. i.
//
// A query's candidates are split into contiguous segments over a thread-block
// cluster of CS CTAs (CS = 1 when there are many queries).  Each CTA keeps
// its segment in shared memory when it fits (else reads it from global
// memory), the digit histograms are summed across the cluster through
// distributed shared memory, and the compaction offsets each CTA by the
// survivors of the CTAs before it.  All cross-CTA steps use hardware cluster
// barriers.
#pragma once

#include "hs2_common.cuh"

namespace hs2 {

constexpr int kSelThreads = 256;
constexpr int kSelSmemMax = 48 * 1024;   // candidates of one CTA kept in shared memory

struct SelectParams {
  const float* score;     // [B*T][L]
  const unsigned* hist;   // [B*T][2048]  level-1 counts
  int32_t* idx;           // [B*T][slots]
  int32_t* n_sel;         // [B*T]
  int T;
  long long L;
  int topk, window, slots, cs;
  long long qpos0;       // query t sits at position qpos0 + t (L - T for a whole cache)
  // context-parallel slice: only the slice's candidates are selected (no
  // window), written as global positions (+ key_off) with their scores
  int cp;
  long long key_off;
  float* cand_score;     // [B*T][topk] when cp
};

__device__ __forceinline__ uint32_t sel_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void sel_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t sel_mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ unsigned ld_dsmem_u32(uint32_t addr) {
  unsigned v;
  asm("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void red_dsmem_add_u32(uint32_t addr, unsigned v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint4 ld_dsmem_u32x4(uint32_t addr) {
  uint4 v;
  asm("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "r"(addr));
  return v;
}
// Copies rank 0's histogram h (nbins, a multiple of 4) into the local out.
__device__ __forceinline__ void copy_rank0_hist(const unsigned* h, int nbins, unsigned* out) {
  const uint32_t base = sel_mapa(smem_u32(h), 0);
  for (int b = 4 * threadIdx.x; b < nbins; b += 4 * kSelThreads)
    *reinterpret_cast<uint4*>(out + b) = ld_dsmem_u32x4(base + b * 4);
}

// Exclusive prefix sum over the CTA (kThreads threads); returns the total.
template <int kThreads = kSelThreads>
__device__ __forceinline__ int sel_block_scan(int v, int& excl, int* tmp) {
  constexpr int W = kThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const int t = tmp[w];
    if (w < warp) before += t;
    total += t;
  }
  excl = before + x - v;
  __syncthreads();
  return total;
}

// Bin `sel` holding the k-th largest element of hist[0..nbins) (k >= 1):
// count(bins > sel) < k <= count(bins >= sel); need = k - count(bins > sel).
// With kGlobal, hist is global memory that may have been written earlier in
// the same grid, and is read through L2 (ld.global.cg); else shared memory.
template <int kThreads = kSelThreads, bool kGlobal = false>
__device__ __forceinline__ void sel_find_bin(const unsigned* hist, int nbins, int k, int* res,
                                             int* tmp) {
  const int per = (nbins + kThreads - 1) / kThreads;
  const int hi = max(0, nbins - (int)threadIdx.x * per);  // thread 0 owns the highest bins
  const int lo = max(0, hi - per);
  int local = 0;
  for (int b = lo; b < hi; ++b) local += (int)(kGlobal ? __ldcg(hist + b) : hist[b]);
  int excl;
  sel_block_scan<kThreads>(local, excl, tmp);
  if (excl < k && k <= excl + local) {
    int above = excl;
    for (int b = hi - 1; b >= lo; --b) {
      const int c = (int)(kGlobal ? __ldcg(hist + b) : hist[b]);
      if (above + c >= k) {
        res[0] = b;
        res[1] = k - above;
        break;
      }
      above += c;
    }
  }
  __syncthreads();
}

// Bin holding the k-th largest element of a global histogram of NB bins
// (k >= 1), read through L2 (it may have been written earlier in the same
// grid): each thread loads its bins into registers with independent loads,
// then a block scan finds the owner.  res[0] = bin, res[1] = k - count(bins
// above it).  Whole CTA (kThreads threads).
template <int kThreads, int NB>
__device__ __forceinline__ void sel_find_bin_global(const unsigned* hist, int k, int* res,
                                                    int* tmp) {
  constexpr int PER = (NB + kThreads - 1) / kThreads;
  const int hi = NB - (int)threadIdx.x * PER;  // thread 0 owns the highest bins
  unsigned c[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int bin = hi - 1 - e;
    c[e] = bin >= 0 && hi > 0 ? __ldcg(hist + bin) : 0u;
  }
  int local = 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) local += (int)c[e];
  int excl;
  sel_block_scan<kThreads>(local, excl, tmp);
  if (excl < k && k <= excl + local) {
    int above = excl;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      if (above + (int)c[e] >= k) {
        res[0] = hi - 1 - e;
        res[1] = k - above;
        break;
      }
      above += (int)c[e];
    }
  }
  __syncthreads();
}

// The same search over a shared-memory histogram by one warp (all 32 lanes;
// a block barrier must follow before res is read), in short loops: the code
// runs once per launch, when it is not in the instruction caches.  Lane l sums
// the NB/32 bins below NB - l*NB/32 (16-byte loads), a warp scan from the top
// finds the owner lane, and the whole warp then searches the owner's bins,
// NB/1024 (at least one) per lane.
template <int NB>
__device__ __forceinline__ void sel_find_bin_warp(const unsigned* hist, int k, int* res) {
  constexpr int PER = NB / 32;
  constexpr int R = PER >= 32 ? PER / 32 : 1;
  static_assert(PER % 4 == 0, "whole 16-byte groups per lane");
  const int lane = threadIdx.x & 31;
  const int lo = NB - (lane + 1) * PER;
  int local = 0;
#pragma unroll 1
  for (int e = 0; e < PER; e += 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(hist + lo + e);
    local += (int)(v.x + v.y + v.z + v.w);
  }
  int incl = local;  // lane 0 holds the highest bins
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned own = __ballot_sync(0xffffffffu, incl - local < k && k <= incl);
  if (own == 0u) return;  // k above the histogram's total: res is left as it was
  const int ol = __ffs((int)own) - 1;
  const int above = __shfl_sync(0xffffffffu, incl - local, ol);
  const int top = NB - 1 - ol * PER;  // the owner's highest bin
  // lane j: the owner's bins top - j*R - r, r < R
  int cnt = 0;
#pragma unroll
  for (int r = 0; r < R; ++r)
    if (lane * R + r < PER) cnt += (int)hist[top - lane * R - r];
  int inc2 = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc2, o);
    if (lane >= o) inc2 += y;
  }
  if (above + inc2 - cnt < k && k <= above + inc2) {
    int acc = above + inc2 - cnt;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int bin = top - lane * R - r;
      const int c = (int)hist[bin];
      if (acc + c >= k) {
        res[0] = bin;
        res[1] = k - acc;
        break;
      }
      acc += c;
    }
  }
}

template <bool SMEM>
__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(const SelectParams p) {
  __shared__ unsigned h2[2048];       // this CTA's level-2 histogram
  __shared__ unsigned h3[512];        // this CTA's level-3 histogram
  __shared__ unsigned hs[2048];       // cluster sum of the current level
  __shared__ int tmp[kSelThreads / 32];
  __shared__ int res[2];
  __shared__ int cnt[2];              // this CTA's (count above tau, count equal to tau)
  __shared__ int wsel[kSelThreads / 32], weq[kSelThreads / 32];
  extern __shared__ unsigned seg_s[];

  pdl_launch_dependents();  // a following sparse layer may place its CTAs on idle SMs
  const int cs = p.cs;
  const uint32_t rank = cs > 1 ? sel_cluster_rank() : 0u;
  const long long row = blockIdx.x / cs;
  const int t = (int)(row % p.T);
  const long long i = p.qpos0 + t;
  // candidates 0 .. nc-1 (a context-parallel slice holds positions 0 .. L-1 of them)
  const long long nc = p.cp ? max(0LL, min(i - p.window + 1, p.L)) : i - p.window + 1;
  int32_t* out = p.idx + row * p.slots;

  if (nc <= p.topk) {  // every candidate is taken: S = {0 .. i}, or the slice's candidates
    if (rank == 0) {
      if (p.cp) {
        const float* srow = p.score + row * p.L;
        for (long long j = threadIdx.x; j < p.slots; j += kSelThreads) {
          out[j] = j < nc ? (int32_t)(j + p.key_off) : -1;
          p.cand_score[row * p.slots + j] = j < nc ? srow[j] : -1.f;
        }
      } else {
        const long long n = i + 1;
        for (long long j = threadIdx.x; j < p.slots; j += kSelThreads) out[j] = j < n ? (int32_t)j : -1;
        if (threadIdx.x == 0) p.n_sel[row] = (int32_t)n;
      }
    }
    return;  // the same branch for every CTA of the cluster: no cluster barrier follows
  }
  // this CTA's segment [s0, s1) of the candidates (s0 a multiple of 4)
  const long long seg = ((nc + cs - 1) / cs + 3) / 4 * 4;
  const long long s0 = min(nc, (long long)rank * seg), s1 = min(nc, s0 + seg);
  const unsigned* src = reinterpret_cast<const unsigned*>(p.score + row * p.L) + s0;
  const int n = (int)(s1 - s0);
  if (SMEM) {
    if ((p.L & 3) == 0) {  // 16-byte copies: the row start and s0 are multiples of 4 words
      const uint4* g4 = reinterpret_cast<const uint4*>(src);
      uint4* s4 = reinterpret_cast<uint4*>(seg_s);
      for (int j = threadIdx.x; j < n / 4; j += kSelThreads) s4[j] = g4[j];
      for (int j = (n / 4) * 4 + threadIdx.x; j < n; j += kSelThreads) seg_s[j] = src[j];
    } else {
      for (int j = threadIdx.x; j < n; j += kSelThreads) seg_s[j] = src[j];
    }
    src = seg_s;
  }
  for (int b = threadIdx.x; b < 2048; b += kSelThreads) h2[b] = 0u;
  for (int b = threadIdx.x; b < 512; b += kSelThreads) h3[b] = 0u;
  __syncthreads();
  // fn(v) for every candidate of the segment, in no particular order.  From
  // global memory (rows too long for shared memory) with 16-byte loads,
  // kBatch of them in flight per thread: one 4-byte load per thread at a time
  // leaves a row pass bound by memory latency, not bandwidth.
  const bool vec = !SMEM && (((uintptr_t)src) & 15u) == 0;
  auto each = [&](auto&& fn) {
    if (vec) {
      constexpr int kBatch = 4;
      const uint4* s4 = reinterpret_cast<const uint4*>(src);
      const int n4 = n >> 2;
      for (int j0 = threadIdx.x; j0 < n4; j0 += kBatch * kSelThreads) {
        uint4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int j = j0 + u * kSelThreads;
          v[u] = j < n4 ? s4[j] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
          if (j0 + u * kSelThreads < n4) {
            fn(v[u].x);
            fn(v[u].y);
            fn(v[u].z);
            fn(v[u].w);
          }
      }
      for (int j = 4 * n4 + threadIdx.x; j < n; j += kSelThreads) fn(src[j]);
    } else {
      for (int j = threadIdx.x; j < n; j += kSelThreads) fn(src[j]);
    }
  };

  int need = p.topk;
  unsigned prefix = 0;
  if (need > 0) {
    // level 1: bits [30:20], counted by the score pass
    sel_find_bin<kSelThreads, true>(p.hist + row * 2048, 2048, need, res, tmp);
    prefix = (unsigned)res[0];
    need = res[1];
    // level 2: bits [19:9] among elements with bits[30:20] == prefix.  With a
    // cluster, every CTA counts straight into rank 0's histogram (distributed
    // shared-memory atomics); after a cluster barrier each CTA copies it.
    const uint32_t h2_0 = cs > 1 ? sel_mapa(smem_u32(h2), 0) : 0u;
    if (cs > 1) sel_cluster_sync();  // rank 0's histograms are cleared
    each([&](unsigned v) {
      if ((v >> 20) == prefix) {
        if (cs > 1) red_dsmem_add_u32(h2_0 + ((v >> 9) & 2047u) * 4, 1u);
        else atomicAdd(&h2[(v >> 9) & 2047u], 1u);
      }
    });
    const unsigned* h = h2;
    if (cs > 1) {
      sel_cluster_sync();
      copy_rank0_hist(h2, 2048, hs);
      h = hs;
    }
    __syncthreads();
    sel_find_bin(h, 2048, need, res, tmp);
    prefix = (prefix << 11) | (unsigned)res[0];
    need = res[1];
    // level 3: bits [8:0] among elements with bits[30:9] == prefix
    const uint32_t h3_0 = cs > 1 ? sel_mapa(smem_u32(h3), 0) : 0u;
    each([&](unsigned v) {
      if ((v >> 9) == prefix) {
        if (cs > 1) red_dsmem_add_u32(h3_0 + (v & 511u) * 4, 1u);
        else atomicAdd(&h3[v & 511u], 1u);
      }
    });
    h = h3;
    if (cs > 1) {
      sel_cluster_sync();
      copy_rank0_hist(h3, 512, hs);
      h = hs;
    }
    __syncthreads();
    sel_find_bin(h, 512, need, res, tmp);
    prefix = (prefix << 9) | (unsigned)res[0];
    need = res[1];
  }
  const unsigned tau = prefix;

  // Ordered compaction of {v > tau} and the first `need` of {v == tau}: warp w
  // of the CTA owns the contiguous sub-segment [w*wseg, (w+1)*wseg).
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wseg = (n + kSelThreads / 32 - 1) / (kSelThreads / 32);
  const int w0 = min(n, warp * wseg), w1 = min(n, w0 + wseg);
  int n_gt = 0, n_eq = 0;
  constexpr int kChunks = 4;  // 32-candidate chunks loaded together (in order afterwards)
  if (p.topk > 0) {
    for (int base = w0; base < w1; base += 32 * kChunks) {
      unsigned v[kChunks];
#pragma unroll
      for (int u = 0; u < kChunks; ++u) {
        const int j = base + 32 * u + lane;
        v[u] = j < w1 ? src[j] : 0u;
      }
#pragma unroll
      for (int u = 0; u < kChunks; ++u) {
        const int j = base + 32 * u + lane;
        n_gt += __popc(__ballot_sync(0xffffffffu, j < w1 && v[u] > tau));
        n_eq += __popc(__ballot_sync(0xffffffffu, j < w1 && v[u] == tau));
      }
    }
  }
  if (lane == 0) {
    wsel[warp] = n_gt;
    weq[warp] = n_eq;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0, e = 0;
    for (int w = 0; w < kSelThreads / 32; ++w) {
      a += wsel[w];
      e += weq[w];
    }
    cnt[0] = a;
    cnt[1] = e;
  }
  if (cs > 1) sel_cluster_sync();
  else __syncthreads();
  // survivors of the CTAs before this one (lane q of every warp reads rank q's
  // counts; a warp sum adds them), then of the warps before this one
  int gt_before = 0, eq_before = 0;
  if (cs > 1) {
    const uint32_t caddr = smem_u32(cnt);
    int g = 0, e = 0;
    if (lane < (int)rank) {
      g = (int)ld_dsmem_u32(sel_mapa(caddr, lane));
      e = (int)ld_dsmem_u32(sel_mapa(caddr + 4, lane));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, o);
      e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    gt_before = g;
    eq_before = e;
  }
  for (int w = 0; w < warp; ++w) {
    gt_before += wsel[w];
    eq_before += weq[w];
  }
  if (p.topk > 0) {
    int pos = gt_before + min(eq_before, need);
    int eq_rank = eq_before;
    for (int base = w0; base < w1; base += 32 * kChunks) {
      unsigned vc[kChunks];
#pragma unroll
      for (int u = 0; u < kChunks; ++u) {
        const int j = base + 32 * u + lane;
        vc[u] = j < w1 ? src[j] : 0u;
      }
#pragma unroll
      for (int u = 0; u < kChunks; ++u) {
        const int j = base + 32 * u + lane;
        const unsigned v = vc[u];
        const bool gt = j < w1 && v > tau;
        const bool eq = j < w1 && v == tau;
        const unsigned eqm = __ballot_sync(0xffffffffu, eq);
        const int my_eq_rank = eq_rank + __popc(eqm & ((1u << lane) - 1u));
        const bool sel = gt || (eq && my_eq_rank < need);
        const unsigned selm = __ballot_sync(0xffffffffu, sel);
        if (sel) {
          const int o = pos + __popc(selm & ((1u << lane) - 1u));
          if (o < p.topk) {
            out[o] = (int32_t)(s0 + j + p.key_off);
            if (p.cp) p.cand_score[row * p.slots + o] = __uint_as_float(v);
          }
        }
        pos += __popc(selm);
        eq_rank += __popc(eqm);
      }
    }
    if (rank == (uint32_t)(cs - 1) && warp == kSelThreads / 32 - 1 && lane == 0 && pos != p.topk)
      raise_status(kStatusBadIndex);
  }
  if (rank == 0 && !p.cp) {
    const long long wstart = i - p.window + 1;
    for (int w = threadIdx.x; w < p.window; w += kSelThreads) out[p.topk + w] = (int32_t)(wstart + w);
    for (int s = p.topk + p.window + threadIdx.x; s < p.slots; s += kSelThreads) out[s] = -1;
    if (threadIdx.x == 0) p.n_sel[row] = p.topk + p.window;
  }
  if (cs > 1) sel_cluster_sync();  // no CTA leaves while others may still read its shared memory
}

}  // namespace hs2
