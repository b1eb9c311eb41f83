// Full-attention layer of a hybrid block (dense causal MQA attention over the
// shared cache) and the head-summed selection score.
//
// Work unit: a "row group" = G = 32/H consecutive queries of one sequence x
// all H heads = 32 query rows sharing one K/V stream (MQA), and a contiguous
// split of that group's causal key range.  Warps 0-3 each take 16 keys of
// every 64-key tile; warp 4 issues the TMA loads of the tile ring.
//   attn_partial : per (group, split) the base-2 running max m, sum l and the
//                  un-normalised O of the split (flash-decoding partials); the
//                  group's first split also clears its level-1 histograms.
//   attn_score   : merges the splits into lse (every CTA, for its group) and O
//                  (each row by one CTA of the group), then makes a second pass
//                  over K (L2-resident when it fits): for every candidate
//                  j <= i - window, score_j = sum_h exp(s_hj - lse_h), written as
//                  fp32, plus a histogram of the score's top bits.
#pragma once

#include "attn_warp.cuh"

namespace hs2 {

constexpr int kTile = 64;         // keys per pipeline stage
constexpr int kRows = 32;         // query rows per group
constexpr int kConsumers = 4;     // MMA warps
constexpr int kHistBins = 2048;   // level-1 radix digit: score bits [30:20]
constexpr int kHistShift = 20;

struct FullAttnParams {
  const __nv_bfloat16* q;   // [B][T][H][D]
  const float* k_scale;     // [B][L] (E4M3) or null
  const float* v_scale;
  float* part_o;            // [groups][splits][32][D]
  float2* part_ml;          // [groups][splits][32] (m, l), base 2
  float* lse;               // [B][T][H] natural log (workspace)
  float* lse_out;           // optional copy for the caller
  float* o;                 // [B][T][H][D]
  float* score;             // [B][T][L]
  unsigned* hist;           // [B][T][kHistBins]
  int B, T, H, D;
  long long L;
  int G, groups_per_seq, n_splits, split_keys, window;
  int score_splits, score_keys;  // split of the score pass (finer than the partials')
  float scale_log2;
  // fused tcgen05 pass only: per-group arrival counters (zeroed before the
  // launch), and the selection outputs when the selection is fused too
  unsigned* grp_sync;            // [groups][8]
  unsigned* sel_list;            // [B*T][splits][split_keys] candidate scores in the level-1 bin
  int2* sel_cnt;                 // [B*T][splits] candidates above / in the level-1 bin per split
  int32_t* idx;                  // [B*T][slots]
  int32_t* n_sel;                // [B*T]
  int topk, slots, fuse_select;
  // the group barriers' wait limit, and arrivals they wait for beyond the
  // group's CTA count (non-zero only under fault injection)
  unsigned long long wait_limit_ns;
  unsigned barrier_extra;
  // fused kernel: kPhases global-timer stamps per CTA b < phase_ctas (null: off)
  unsigned long long* phase_stamps;
  int phase_ctas;
  // query t sits at local key position qpos0 + t (L - T when the cache holds
  // the whole context; with a context-parallel slice, the queries' position
  // relative to the slice's first key, which may exceed L)
  long long qpos0;
  // context-parallel score pass: the global natural-log normaliser [B][T][H]
  // replaces the merge of this slice's partials (O and lse are not written)
  const float* lse_in;
  int no_score;   // merge the partials into O and lse only (no score pass)
};

template <int D, bool FP8>
struct FullAttnSmem {
  static constexpr int kElem = FP8 ? 1 : 2;
  static constexpr int kTileBytes = kTile * D * kElem;          // one of K or V
  static constexpr int kStages = FP8 ? 4 : 3;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStagingBytes = FP8 ? kConsumers * 2 * 16 * D * 2 : 0;
  static constexpr int kObufBytes = kConsumers * kRows * (D + 8) * 4;
  static constexpr int kRingBytes = kStages * kStageBytes + kStagingBytes;
  static constexpr int kMainBytes = kRingBytes > kObufBytes ? kRingBytes : kObufBytes;
  static constexpr int kQOff = kMainBytes;
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kMlOff = kQOff + kQBytes;
  static constexpr int kBarOff = kMlOff + kConsumers * kRows * 8;
  static constexpr int kBytes = kBarOff + 2 * kStages * 8 + 1024;  // + alignment slack
  // score pass: K only
  static constexpr int kScoreStageBytes = kTileBytes;
  static constexpr int kScoreStagingBytes = FP8 ? kConsumers * 16 * D * 2 : 0;
  static constexpr int kScoreStages = 4;
  static constexpr int kScoreHistOff = kScoreStages * kScoreStageBytes + kScoreStagingBytes;
  static constexpr int kScoreQOff = kScoreHistOff + 4 * kHistBins * 4;
  static constexpr int kScoreLseOff = kScoreQOff + kQBytes;
  static constexpr int kScoreBarOff = kScoreLseOff + kRows * 4;
  static constexpr int kScoreBytes = kScoreBarOff + 2 * kScoreStages * 8 + 1024;
};

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
}

// Loads the group's 32 query rows (row r = query t0 + r/H, head r%H) into a
// swizzled bf16 tile; rows of queries past T are zero.  Consumer threads only.
template <int D>
__device__ __forceinline__ void load_q_tile(const FullAttnParams& p, int b, int t0, uint8_t* qs) {
  constexpr int kChunks = D * 2 / 16;
  for (int u = threadIdx.x; u < kRows * kChunks; u += kConsumers * 32) {
    const int r = u / kChunks, ch = u % kChunks;
    const int t = t0 + r / p.H, h = r % p.H;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (t < p.T)
      v = *reinterpret_cast<const uint4*>(p.q + (((long long)b * p.T + t) * p.H + h) * D + ch * 8);
    *reinterpret_cast<uint4*>(qs + sw128_offset(r, ch * 16, kRows)) = v;
  }
}

// Issues the TMA loads of one K or V tile (kTile rows starting at global row
// `row`) into a swizzled tile at dst.
template <int D, bool FP8>
__device__ __forceinline__ void tma_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                         long long row, uint64_t pol) {
  if (FP8) {
    tma_load_2d(dst, map, bar, 0, (int)row, pol);
  } else {
#pragma unroll
    for (int h = 0; h < D / 64; ++h) tma_load_2d(dst + h * kTile * 128, map, bar, h * 64, (int)row, pol);
  }
}

template <int D, bool FP8>
__global__ void __launch_bounds__(160) attn_partial_kernel(const __grid_constant__ CUtensorMap kmap,
                                                           const __grid_constant__ CUtensorMap vmap,
                                                           const FullAttnParams p) {
  using SM = FullAttnSmem<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* qs = smem + SM::kQOff;
  float2* ml_s = reinterpret_cast<float2*>(smem + SM::kMlOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint64_t* empty = full + SM::kStages;

  const int split = blockIdx.x % p.n_splits;
  const int grp = blockIdx.x / p.n_splits;
  const int b = grp / p.groups_per_seq;
  const int t0 = (grp % p.groups_per_seq) * p.G;
  const int t_last = min(p.T, t0 + p.G) - 1;
  const long long i_last = p.qpos0 + t_last;
  const long long k_lo = (long long)split * p.split_keys;
  const long long k_hi = min(min(k_lo + p.split_keys, i_last + 1), p.L);
  const long long part = (long long)grp * p.n_splits + split;

  if (split == 0) {  // clear the group's level-1 selection histograms
    for (int u = threadIdx.x; u < p.G * kHistBins; u += blockDim.x) {
      const int t = t0 + u / kHistBins;
      if (t < p.T) p.hist[((long long)b * p.T + t) * kHistBins + (u % kHistBins)] = 0u;
    }
  }
  if (k_lo >= k_hi) {  // empty split: neutral partial
    for (int u = threadIdx.x; u < kRows * D; u += blockDim.x) p.part_o[part * kRows * D + u] = 0.f;
    if (threadIdx.x < kRows) p.part_ml[part * kRows + threadIdx.x] = make_float2(kNegInf, 0.f);
    return;
  }
  const int n_tiles = (int)((k_hi - k_lo + kTile - 1) / kTile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SM::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumers) {  // ---------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      const uint64_t pol_k = policy_evict_normal(), pol_v = policy_evict_first();
      for (int n = 0; n < n_tiles; ++n) {
        const int s = n % SM::kStages;
        if (n >= SM::kStages && !mbar_wait(&empty[s], ((n / SM::kStages) - 1) & 1)) break;
        uint8_t* st = smem + s * SM::kStageBytes;
        mbar_arrive_expect_tx(&full[s], SM::kStageBytes);
        const long long row = (long long)b * p.L + k_lo + (long long)n * kTile;
        tma_tile<D, FP8>(st, &kmap, &full[s], row, pol_k);
        tma_tile<D, FP8>(st + SM::kTileBytes, &vmap, &full[s], row, pol_v);
      }
    }
    return;
  }

  // ----------------------------------------------------------- consumers
  load_q_tile<D>(p, b, t0, qs);
  consumer_sync();

  const int g = lane >> 2, c = lane & 3;
  long long i_row[2][2];
  bool row_ok[2][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = mt * 16 + g + 8 * h;
      const int t = t0 + r / p.H;
      row_ok[mt][h] = t < p.T;
      i_row[mt][h] = p.qpos0 + t;
    }
  const float* ksc = FP8 ? p.k_scale + (long long)b * p.L : nullptr;
  const float* vsc = FP8 ? p.v_scale + (long long)b * p.L : nullptr;

  WarpAttn<2, D> st;
  st.init();
  const uint32_t q_base = smem_u32(qs);
  uint8_t* stg_k = smem + SM::kStages * SM::kStageBytes + warp * 2 * 16 * D * 2;
  uint8_t* stg_v = stg_k + 16 * D * 2;

  for (int n = 0; n < n_tiles; ++n) {
    const int s = n % SM::kStages;
    if (!mbar_wait(&full[s], (n / SM::kStages) & 1)) break;
    uint8_t* stage = smem + s * SM::kStageBytes;
    const long long kbase = k_lo + (long long)n * kTile + warp * 16;
    uint32_t kt, vt;
    int key0, rows;
    if (FP8) {
      warp_fp8_rows_to_bf16(stage, warp * 16, 16, stg_k, 16);
      warp_fp8_rows_to_bf16(stage + SM::kTileBytes, warp * 16, 16, stg_v, 16);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      kt = smem_u32(stg_k);
      vt = smem_u32(stg_v);
      key0 = 0;
      rows = 16;
    } else {
      kt = smem_u32(stage);
      vt = smem_u32(stage + SM::kTileBytes);
      key0 = warp * 16;
      rows = kTile;
    }
    float x[2][2][4];
    warp_qk<2, D>(q_base, kt, key0, rows, x);
    float pvs[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const long long key = kbase + nt * 8 + 2 * c + j;
        const bool in = key < k_hi;
        const float ks = (FP8 && in) ? ksc[key] : 1.f;
        pvs[nt][j] = (FP8 && in) ? vsc[key] : 1.f;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const bool ok = in && row_ok[mt][h] && key <= i_row[mt][h];
            x[mt][nt][2 * h + j] = ok ? x[mt][nt][2 * h + j] * (p.scale_log2 * ks) : kNegInf;
          }
      }
    warp_softmax_pv<2, D>(st, x, vt, key0, rows, pvs);
    if (!FP8) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }

  // ------------------------------------------- merge the 4 warps' partials
  float lf[2][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      lf[mt][h] = quad_sum(st.l[mt][h]);
      if (c == 0) ml_s[warp * kRows + mt * 16 + g + 8 * h] = make_float2(st.m[mt][h], lf[mt][h]);
    }
  consumer_sync();
  float f[2][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = mt * 16 + g + 8 * h;
      float M = kNegInf;
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, ml_s[w * kRows + r].x);
      f[mt][h] = (M == kNegInf) ? 0.f : fast_exp2(st.m[mt][h] - M);
    }
  float* obuf = reinterpret_cast<float*>(smem);
  warp_store_o<2, D>(st, f, obuf + warp * kRows * (D + 8));
  consumer_sync();
  for (int u = threadIdx.x; u < kRows * D; u += kConsumers * 32) {
    const int r = u / D, d = u % D;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) acc += obuf[(w * kRows + r) * (D + 8) + d];
    p.part_o[(part * kRows + r) * D + d] = acc;
  }
  if (threadIdx.x < kRows) {
    const int r = threadIdx.x;
    float M = kNegInf;
    for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, ml_s[w * kRows + r].x);
    float lt = 0.f;
    if (M != kNegInf)
      for (int w = 0; w < kConsumers; ++w) {
        const float2 v = ml_s[w * kRows + r];
        lt += v.y * fast_exp2(v.x - M);
      }
    p.part_ml[part * kRows + r] = make_float2(M, lt);
  }
}

template <int D, bool FP8, int G>
__global__ void __launch_bounds__(160) attn_score_kernel(const __grid_constant__ CUtensorMap kmap,
                                                         const FullAttnParams p) {
  using SM = FullAttnSmem<D, FP8>;
  constexpr int kStages = SM::kScoreStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  unsigned* hist_s = reinterpret_cast<unsigned*>(smem + SM::kScoreHistOff);
  uint8_t* qs = smem + SM::kScoreQOff;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kScoreBarOff);
  uint64_t* empty = full + kStages;

  const int split = blockIdx.x % p.score_splits;
  const int grp = blockIdx.x / p.score_splits;
  const int b = grp / p.groups_per_seq;
  const int t0 = (grp % p.groups_per_seq) * G;
  const int t_last = min(p.T, t0 + G) - 1;
  const long long i_last = p.qpos0 + t_last;
  const long long k_lo = (long long)split * p.score_keys;
  const long long k_hi = min(min(k_lo + p.score_keys, i_last - p.window + 1), p.L);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* lse2_s = reinterpret_cast<float*>(smem + SM::kScoreLseOff);

  // ---- merge of the splits: lse of the group's rows (base 2) in every CTA;
  //      O of row r in the CTA whose score-split index is r mod score_splits.
  if (warp < kConsumers) {
    for (int r = warp; r < kRows; r += kConsumers) {
      const int t = t0 + r / p.H;
      const float2* ml = p.part_ml + (long long)grp * p.n_splits * kRows + r;
      float M = kNegInf;
      for (int sp = lane; sp < p.n_splits; sp += 32) M = fmaxf(M, ml[(long long)sp * kRows].x);
#pragma unroll
      for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      float lt = 0.f;
      if (M != kNegInf)
        for (int sp = lane; sp < p.n_splits; sp += 32) {
          const float2 v = ml[(long long)sp * kRows];
          lt += v.x == kNegInf ? 0.f : v.y * fast_exp2(v.x - M);
        }
#pragma unroll
      for (int o = 16; o; o >>= 1) lt += __shfl_xor_sync(0xffffffffu, lt, o);
      const float l2 = M + log2f(lt);
      if (lane == 0) lse2_s[r] = l2;
      if (t < p.T && (r % p.score_splits) == split) {
        const long long li = ((long long)b * p.T + t) * p.H + r % p.H;
        if (lane == 0) {
          p.lse[li] = l2 * 0.69314718055994531f;
          if (p.lse_out) p.lse_out[li] = l2 * 0.69314718055994531f;
        }
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        float acc[D / 32];
#pragma unroll
        for (int k = 0; k < D / 32; ++k) acc[k] = 0.f;
        const float* po = p.part_o + ((long long)grp * p.n_splits * kRows + r) * D;
#pragma unroll 4
        for (int sp = 0; sp < p.n_splits; ++sp) {
          const float2 v = ml[(long long)sp * kRows];
          const float f = (v.x == kNegInf) ? 0.f : fast_exp2(v.x - M) * inv;
#pragma unroll
          for (int k = 0; k < D / 32; ++k) acc[k] += f * po[(long long)sp * kRows * D + lane + 32 * k];
        }
        float* out = p.o + li * D;
#pragma unroll
        for (int k = 0; k < D / 32; ++k) out[lane + 32 * k] = acc[k];
      }
    }
  }
  if (k_lo >= k_hi) return;
  const int n_tiles = (int)((k_hi - k_lo + kTile - 1) / kTile);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumers) {
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      const uint64_t pol = policy_evict_first();
      for (int n = 0; n < n_tiles; ++n) {
        const int s = n % kStages;
        if (n >= kStages && !mbar_wait(&empty[s], ((n / kStages) - 1) & 1)) break;
        mbar_arrive_expect_tx(&full[s], SM::kScoreStageBytes);
        tma_tile<D, FP8>(smem + s * SM::kScoreStageBytes, &kmap, &full[s],
                         (long long)b * p.L + k_lo + (long long)n * kTile, pol);
      }
    }
    return;
  }

  load_q_tile<D>(p, b, t0, qs);
  for (int u = threadIdx.x; u < G * kHistBins; u += kConsumers * 32) hist_s[u] = 0u;
  consumer_sync();

  const int g = lane >> 2, c = lane & 3;
  long long i_row[2][2];
  float lse2[2][2];
  int qry[2][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = mt * 16 + g + 8 * h;
      const int tl = r / p.H;
      const int t = t0 + tl;
      qry[mt][h] = tl;
      i_row[mt][h] = (t < p.T) ? p.qpos0 + t : -1;  // -1: no candidates
      lse2[mt][h] = (t < p.T) ? lse2_s[r] : 0.f;
    }
  const float* ksc = FP8 ? p.k_scale + (long long)b * p.L : nullptr;
  const uint32_t q_base = smem_u32(qs);
  uint8_t* stg_k = smem + kStages * SM::kScoreStageBytes + warp * 16 * D * 2;

  for (int n = 0; n < n_tiles; ++n) {
    const int s = n % kStages;
    if (!mbar_wait(&full[s], (n / kStages) & 1)) break;
    uint8_t* stage = smem + s * SM::kScoreStageBytes;
    const long long kbase = k_lo + (long long)n * kTile + warp * 16;
    uint32_t kt;
    int key0, rows;
    if (FP8) {
      warp_fp8_rows_to_bf16(stage, warp * 16, 16, stg_k, 16);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      kt = smem_u32(stg_k);
      key0 = 0;
      rows = 16;
    } else {
      kt = smem_u32(stage);
      key0 = warp * 16;
      rows = kTile;
    }
    float x[2][2][4];
    warp_qk<2, D>(q_base, kt, key0, rows, x);
    if (!FP8) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // acc[tl][nt][j]: head-sum of query tl (rows tl*H .. tl*H+H-1) for key nt*8 + 2c + j.
    // Thread rows are mt*16 + g + 8h, so query tl = (mt*16 + 8h + g) / H.
    float acc[G][2][2];
#pragma unroll
    for (int q = 0; q < G; ++q)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) acc[q][nt][0] = acc[q][nt][1] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const long long key = kbase + nt * 8 + 2 * c + j;
        const float ks = (FP8 && key < k_hi) ? ksc[key] : 1.f;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const bool ok = key <= i_row[mt][h] - p.window;
            const float pr = ok ? fast_exp2(x[mt][nt][2 * h + j] * (p.scale_log2 * ks) - lse2[mt][h]) : 0.f;
            if (G == 1) {
              acc[0][nt][j] += pr;
            } else {
              // rows of this thread: mt*16 + 8h + g; with H = 32/G, query = row / H
              constexpr int kH = 32 / G;
#pragma unroll
              for (int q = 0; q < G; ++q)
                if (((mt * 16 + 8 * h) / kH == q && kH >= 16) ||
                    (kH == 8 && (mt * 16 + 8 * h) / 8 == q))
                  acc[q][nt][j] += pr;
            }
          }
      }
#pragma unroll
    for (int q = 0; q < G; ++q)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float v = acc[q][nt][j];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          acc[q][nt][j] = v;
        }
    if (g == 0) {
#pragma unroll
      for (int q = 0; q < G; ++q) {
        const int t = t0 + q;
        if (t >= p.T) break;
        const long long i_q = p.qpos0 + t;
        float* srow = p.score + ((long long)b * p.T + t) * p.L;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const long long key = kbase + nt * 8 + 2 * c + j;
            const bool cand = key <= i_q - p.window;
            const float v = acc[q][nt][j];
            if (cand) srow[key] = v;
            hist_inc(hist_s + q * kHistBins, __float_as_uint(v) >> kHistShift, cand);
          }
      }
    }
  }
  consumer_sync();
  for (int u = threadIdx.x; u < G * kHistBins; u += kConsumers * 32) {
    const unsigned cnt = hist_s[u];
    const int q = u / kHistBins;
    const int t = t0 + q;
    if (cnt && t < p.T) atomicAdd(&p.hist[((long long)b * p.T + t) * kHistBins + (u % kHistBins)], cnt);
  }
}

}  // namespace hs2
