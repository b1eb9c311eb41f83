// Full-attention layer on the 5th-generation tensor cores (tcgen05), for
// head_dim 128 and a bf16 or E4M3 cache.
//
// MQA: every query row of a group -- N rows = N/H queries x H heads -- reads
// the same K/V stream.  Each 128-key tile is processed transposed:
//   S^T[128 keys][N rows] = K_tile[128 x 128] . Q^T        (M = 128 keys)
//   O^T[128 d][N rows]   += V_tile^T[128 d x 128 keys] . P (M = 128 d)
// with fp32 accumulators in tensor memory (TMEM).  In S^T, TMEM lane = key, so
// the thread that owns a lane holds one key's logits for all N rows: the
// head-sum of the selection score needs no cross-thread step, and the softmax
// exponentials are element-wise.  The softmax normaliser uses a lazily
// refreshed per-row reference max (raised, and O and the row sums rescaled,
// only when some logit exceeds it by more than 2^8), so the common tile needs
// no cross-thread max; each thread keeps its keys' partial row sums in a TMEM
// column block.
//
// Warp roles: warp 0 issues the TMA loads of the K/V tile ring; warp 1
// allocates TMEM and one of its threads issues every tcgen05.mma; the softmax
// (or score) warps own one TMEM lane = one key each.
//
// E4M3 cache: TMA brings the 128-byte E4M3 rows; converter warps rewrite each
// K and V tile as f16 (E4M3 -> f16 is exact) in the same 128B-swizzled layout
// a bf16 tile has, and the MMAs run kind::f16 with f16 operands (Q is staged
// as f16: exact for bf16 values of magnitude >= 2^-14, and P is written as
// f16).  The per-token scales need no extra pass: the thread that owns key j
// multiplies its logits by k_scale[j] and its P values by v_scale[j].
//   attn_tc_fused   : decode shapes (32 rows per group): the partial pass of
//                     a (group, split), a group barrier, the score pass over
//                     the same split (from logits kept in TMEM when the split
//                     has at most 15 tiles, else recomputed from K), and the
//                     group's top-k selection -- one cooperative launch.
//   attn_tc_partial : other shapes, per (group, split): reference max m, sum
//                     l and un-normalised O of the split.
//   attn_tc_score   : merges the splits into lse and O, then recomputes S^T per
//                     tile and writes score_j = sum over a query's heads of
//                     exp(s - lse), with the level-1 selection histogram.
#pragma once

#include "full_attn.cuh"
#include "select.cuh"
#include "tc_common.cuh"

namespace hs2 {

constexpr int kTcKeys = 128;          // keys per tile (M of the score MMA)
constexpr int kTcTileBytes = kTcKeys * 128 * 2;   // one 16-bit K or V tile: 32 KB
constexpr int kTcTile8Bytes = kTcKeys * 128;      // one E4M3 K or V tile: 16 KB
constexpr float kRescaleAbove = 8.f;  // base-2 logits may exceed the reference by this

// Shared-memory plan.  Partial kernel: K/V tile ring (16-bit, or E4M3 plus
// f16 K and V tiles), Q, P^T (double-buffered for N = 32), per-row reference
// max / correction / partial maxima and sums.  Score kernel: K ring (plus two
// f16 K tiles for E4M3), staged (m, l) partials of the group, Q, histograms.
template <int N, bool FP8>
struct TcSmem {
  // E4M3 32-row groups: a 2-stage E4M3 ring (the f16 tiles buffer two more)
  static constexpr int kStages = N == 32 ? (FP8 ? 2 : 3) : 2;
  static constexpr int kNP = N == 32 ? 2 : 1;            // P^T buffers
  static constexpr int kStageBytes = 2 * (FP8 ? kTcTile8Bytes : kTcTileBytes);  // K then V
  // E4M3 only: converted f16 K tiles, then f16 V tiles -- two of each for
  // 32-row groups, so the converters write tile n+1 while the tensor cores
  // read tile n
  static constexpr int kNK16 = (FP8 && N == 32) ? 2 : 1;
  static constexpr int kNV16 = (FP8 && N == 32) ? 2 : 1;
  static constexpr int kK16Off = kStages * kStageBytes;
  static constexpr int kV16Off = kK16Off + kNK16 * kTcTileBytes;
  static constexpr int kQOff = kK16Off + (FP8 ? (kNK16 + kNV16) * kTcTileBytes : 0);
  static constexpr int kQBytes = N * 256;
  static constexpr int kPOff = kQOff + kQBytes;  // P^T [N rows][128 keys] (N = 128: P MN-major), 16-bit
  static constexpr int kPBytes = N * 256;
  static constexpr int kMrefOff = kPOff + kNP * kPBytes; // float [N]
  static constexpr int kCorrOff = kMrefOff + N * 4;      // float [N]
  static constexpr int kTmaxOff = kCorrOff + N * 4;      // float [4][N] (also the row sums)
  static constexpr int kBarOff = kTmaxOff + 4 * N * 4;
  // + V arrival per stage, second f16 K and V tiles
  static constexpr int kNumBars = 3 * kStages + 13 + 2 * kNP;
  static constexpr int kSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kBar2Off = kSlotOff + 16;         // fused kernel: score-pass barriers
  static constexpr int kNumBars2 = 16;
  // retained tiles' references (16-byte aligned: read as float4)
  static constexpr int kMhistOff = (kBar2Off + kNumBars2 * 8 + 15) / 16 * 16;
  static constexpr int kMhistBytes = N == 32 ? 15 * N * 4 : 0;
  static constexpr int kBytes = kMhistOff + kMhistBytes + 1024;
  // fused kernel: the score pass reuses the partial pass's tile ring for its
  // K ring, the group's (m, l) partials float2 [N][splits] and the
  // histograms unsigned [G][2048] (<= 32 KB each): after the K ring, or for
  // E4M3 in the two f16 V tiles (idle in the score pass, whose two f16 K tiles
  // are the partial pass's).  The fused selection then uses everything below Q
  // for the row's candidate scores and its counters.
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kS2Stages = 4;
  static constexpr int kS2TileBytes = FP8 ? kTcTile8Bytes : kTcTileBytes;
  static constexpr bool kHistInV16 = FP8 && N == 32;
  static constexpr int kS2MlOff = kHistInV16 ? kV16Off + 32 * 1024 : kS2Stages * kS2TileBytes;
  static constexpr int kS2HistOff = kHistInV16 ? kV16Off : kS2MlOff + 32 * 1024;
  static constexpr bool kFusable =
      kHistInV16 ? (kS2Stages * kS2TileBytes <= kRingBytes && kNV16 * kTcTileBytes >= 64 * 1024)
                 : kS2HistOff + 32 * 1024 <= kRingBytes;
  // counters (2048), list offsets, the lower splits' counters (2048 + 512)
  static constexpr int kSelWorkOff = kQOff - 24 * 1024;
  static constexpr int kSelCap = kSelWorkOff / 4;        // list entries held in smem
  // score kernel
  static constexpr int kSStages = (FP8 || N == 32) ? 4 : 3;
  static constexpr int kSStageBytes = FP8 ? kTcTile8Bytes : kTcTileBytes;
  static constexpr int kSK16Off = kSStages * kSStageBytes;
  static constexpr int kSMlOff = kSK16Off + (FP8 ? 2 * kTcTileBytes : 0);
  static constexpr int kSMlBytes = 32 * 1024;            // rows x splits x 8 bytes
  static constexpr int kSQOff = kSMlOff + kSMlBytes;
  static constexpr int kSHistOff = kSQOff + kQBytes;
  static constexpr int kSHistBytes = 4 * kHistBins * 4;
  static constexpr int kSLseOff = kSHistOff + kSHistBytes;
  static constexpr int kSBarOff = kSLseOff + N * 4;
  static constexpr int kSSlotOff = kSBarOff + (2 * kSStages + 9) * 8;
  static constexpr int kSBytes = kSSlotOff + 16 + 1024;
};

// Rows [row0, row0 + nrows) of an E4M3 tile (TMA layout: 128-byte rows, 16-byte
// chunks swizzled by row & 7) rewritten as f16 rows of a 128B-swizzled 16-bit
// tile of 128 rows per column half.  E4M3 -> f16 is exact.
__device__ __forceinline__ void fp8_rows_to_f16(const uint8_t* src, int row0, int nrows,
                                                int tid, int nthreads, uint8_t* dst) {
#pragma unroll 4  // independent 16-byte chunks in flight: the loop is latency-bound otherwise
  for (int u = tid; u < nrows * 8; u += nthreads) {
    const int r = row0 + (u >> 3), ch = u & 7;  // codes 16ch .. 16ch+15 of row r
    const uint4 raw = *reinterpret_cast<const uint4*>(src + r * 128 + ((ch ^ (r & 7)) << 4));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t h[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[k] & 0xFFFFu), __NV_E4M3);
      const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[k] >> 16), __NV_E4M3);
      h[2 * k] = (uint32_t)lo.x | ((uint32_t)lo.y << 16);
      h[2 * k + 1] = (uint32_t)hi.x | ((uint32_t)hi.y << 16);
    }
    *reinterpret_cast<uint4*>(dst + sw128_offset(r, ch * 32, kTcKeys)) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(dst + sw128_offset(r, ch * 32 + 16, kTcKeys)) =
        make_uint4(h[4], h[5], h[6], h[7]);
  }
}

// Stages the group's N query rows (row r = query t0 + r/H, head r%H) into a
// K-major 128B-swizzled 16-bit tile (bf16, or f16 for an E4M3 cache); rows of
// queries past T are zero.
template <int N, bool FP8>
__device__ __forceinline__ void tc_stage_q(const FullAttnParams& p, int b, int t0, uint8_t* qs,
                                           int tid, int nthreads) {
  for (int u = tid; u < N * 16; u += nthreads) {
    const int r = u >> 4, ch = u & 15;
    const int t = t0 + r / p.H, h = r % p.H;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (t < p.T)
      v = *reinterpret_cast<const uint4*>(p.q + (((long long)b * p.T + t) * p.H + h) * 128 + ch * 8);
    if (FP8) {
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __nv_bfloat162 bb = *reinterpret_cast<const __nv_bfloat162*>(&w[k]);
        const float2 f = __bfloat1622float2(bb);
        const __half2 hh = __floats2half2_rn(f.x, f.y);
        w[k] = *reinterpret_cast<const uint32_t*>(&hh);
      }
      v = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *reinterpret_cast<uint4*>(qs + sw128_offset(r, ch * 16, N)) = v;
  }
}

// Barrier, and block-wide OR, over the softmax warps (named barrier 1).
template <int kThreads>
__device__ __forceinline__ void softmax_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
}
template <int kThreads>
__device__ __forceinline__ bool softmax_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kThreads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Issues the 8 MMAs of S^T[128 x N] = K_tile . Q^T into TMEM at tmem_d.
template <int N, bool F16>
__device__ __forceinline__ void tc_issue_qk(uint32_t tmem_d, uint32_t k_addr, uint32_t q_addr) {
  constexpr uint32_t idesc = tc_idesc_f16(128, N, F16 ? kTcF16 : kTcBF16, false, false);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
    tc_mma_f16(tmem_d, sw128_kmajor_desc(k_addr + half * (kTcKeys * 128) + koff),
               sw128_kmajor_desc(q_addr + half * (N * 128) + koff), idesc, ks > 0);
  }
}

// P operand layout of the PV product: 128-row groups store P MN-major (each
// key's rows contiguous, so a softmax thread writes 16-byte chunks), 32-row
// groups P^T K-major (a key's 16 rows would fill only a quarter of a row).
__host__ __device__ constexpr bool tc_p_mn_major(int N) { return N == 128; }

// Issues the 8 MMAs of O^T[128 x N] (+)= V_tile^T . P, V read MN-major from its
// TMA tile (d contiguous within a 64-d half, halves 16 KB apart); P MN-major
// in the same geometry (64-row halves 16 KB apart) or P^T K-major.
template <int N, bool F16>
__device__ __forceinline__ void tc_issue_pv(uint32_t tmem_d, uint32_t v_addr, uint32_t p_addr,
                                            bool accumulate) {
  constexpr bool kPMN = tc_p_mn_major(N);
  constexpr uint32_t idesc = tc_idesc_f16(128, N, F16 ? kTcF16 : kTcBF16, true, kPMN);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
    tc_mma_f16(tmem_d, sw128_mnmajor_desc(v_addr + ks * 16 * 128, kTcKeys * 128),
               kPMN ? sw128_mnmajor_desc(p_addr + ks * 16 * 128, kTcKeys * 128)
                    : sw128_kmajor_desc(p_addr + half * (N * 128) + koff),
               idesc, accumulate || ks > 0);
  }
}

// Partial kernel: warps 0 (TMA), 1 (MMA) and 8 softmax warps 2-9 (plus, for
// an E4M3 cache, K converter warps 10-12 and V converter warps 13-15).
// Softmax warp w reads TMEM lane quarter w%4 (keys, or d for O^T) and the
// column half (w-2)/4 of the N rows, so two warps share each scheduler and
// each thread handles one key x N/2 rows per tile.
constexpr int kTcSoftmax = 256;
// Three converter warps per tensor: with two, the E4M3 -> f16 conversion set the
// per-tile time (measured on B200: 256K decode call 0.215 -> 0.207 ms, 1M chunk
// 238 -> 226 ms with three).
constexpr int kTcConvert = 96;  // threads per converted tensor (K or V)
__host__ __device__ constexpr int tc_partial_threads(bool fp8) {
  return 64 + kTcSoftmax + (fp8 ? 2 * kTcConvert : 0);
}
// Score kernel: warps 0 (TMA), 1 (MMA), two groups of four score warps (2-5
// take the even tiles, 6-9 the odd ones, each its own S^T buffer), and for an
// E4M3 cache converter warps 10-13.
__host__ __device__ constexpr int tc_score_threads(bool fp8) { return fp8 ? 448 : 320; }

// Barrier initialisation and per-row state of the partial pass (all threads;
// a block barrier must follow before the body runs).
template <int N, bool FP8>
__device__ __forceinline__ void tc_partial_setup(uint8_t* smem) {
  using SM = TcSmem<N, FP8>;
  constexpr int S = SM::kStages;
  constexpr int NP = SM::kNP;
  float* m_ref = reinterpret_cast<float*>(smem + SM::kMrefOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  if (threadIdx.x < N) m_ref[threadIdx.x] = kNegInf;
  if (threadIdx.x == 0) {
    uint64_t* kv_full = bars;
    uint64_t* kv_empty = kv_full + S;
    uint64_t* s_full = kv_empty + S;
    uint64_t* s_empty = s_full + 2;
    uint64_t* p_full = s_empty + 2;
    uint64_t* pv_done = p_full + NP;
    uint64_t* q_ready = pv_done + NP;
    for (int s = 0; s < S; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], FP8 ? 2 * kTcConvert / 32 : 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kTcSoftmax / 32);
    }
    for (int i = 0; i < NP; ++i) {
      mbar_init(&p_full[i], kTcSoftmax / 32);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(q_ready, kTcSoftmax / 32);
    mbar_init(q_ready + 1, kTcConvert / 32);  // k16_full
    mbar_init(q_ready + 2, 1);                // k16_free
    mbar_init(q_ready + 3, kTcConvert / 32);  // v16_full
    mbar_init(q_ready + 4, 1);                // v16_free
    for (int s = 0; s < S; ++s) mbar_init(q_ready + 5 + s, 1);  // v_full (bf16: V of stage s)
    mbar_init(q_ready + 5 + S, kTcConvert / 32);  // k16_full of the second f16 K tile
    mbar_init(q_ready + 6 + S, 1);                // its k16_free
    mbar_init(q_ready + 7 + S, kTcConvert / 32);  // v16_full of the second f16 V tile
    mbar_init(q_ready + 8 + S, 1);                // its v16_free
    fence_mbar_init();
  }
}

// Tiles whose logits stay in tensor memory in a retaining partial pass (32
// columns each beside the 32 of O^T: all 512 columns).
constexpr int kTcRetainTiles = 15;

// Phase stamps per CTA of the fused kernel (tracing).
constexpr int kPhases = 8;


// The partial pass of one (group, split) work item: every role's work, with
// the barriers of tc_partial_setup initialised and the TMEM columns at `tmem`
// (4N; 512 when RETAIN).  TMEM layout: S^T double buffer at columns 0 and N,
// O^T at 2N, per-key row sums at 3N (16-column rows: in registers); with
// RETAIN (N = 32, at most kTcRetainTiles tiles) O^T at 0 and the S^T of tile n
// kept at N + n*N for a later score pass.
// Returns in every thread once its role is done (no trailing barrier).
template <int N, int G, bool FP8, bool RETAIN = false>
__device__ __forceinline__ void tc_partial_body(const CUtensorMap& kmap, const CUtensorMap& vmap,
                                                const FullAttnParams& p, uint8_t* smem,
                                                uint32_t tmem) {
  static_assert(!RETAIN || N == 32, "retained logits: 32 rows per group");
  using SM = TcSmem<N, FP8>;
  constexpr uint32_t kOCol = RETAIN ? 0 : 2 * N;
  auto s_col = [](int n) -> uint32_t { return RETAIN ? N + n * N : (n & 1) * N; };
  constexpr int S = SM::kStages;
  constexpr int NP = SM::kNP;
  constexpr int kH = N / G;     // heads per query
  constexpr int NC = N / 2;     // columns per softmax warp
  constexpr int kTileIn = FP8 ? kTcTile8Bytes : kTcTileBytes;  // one K or V tile as loaded
  float* m_ref = reinterpret_cast<float*>(smem + SM::kMrefOff);
  float* corr = reinterpret_cast<float*>(smem + SM::kCorrOff);
  float* tmax = reinterpret_cast<float*>(smem + SM::kTmaxOff);
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint64_t* kv_empty = kv_full + S;
  uint64_t* s_full = kv_empty + S;   // [2]
  uint64_t* s_empty = s_full + 2;    // [2]
  uint64_t* p_full = s_empty + 2;    // [NP]
  uint64_t* pv_done = p_full + NP;   // [NP]
  uint64_t* q_ready = pv_done + NP;
  uint64_t* k16_full = q_ready + 1;  // E4M3 only: converted K / V tile handshakes
  uint64_t* k16_free = k16_full + 1;
  uint64_t* v16_full = k16_free + 1;
  uint64_t* v16_free = v16_full + 1;
  uint64_t* v_full = v16_free + 1;   // [S] bf16: V of a stage (kv_full then means K)
  // E4M3: f16 K tile n sits in buffer n % kNK16, V tile n in buffer n % kNV16,
  // each buffer with its own full/free pair
  constexpr int NK = SM::kNK16;
  constexpr int NV = SM::kNV16;
  auto k16_full_of = [&](int n) { return (NK == 2 && (n & 1)) ? v_full + S : k16_full; };
  auto k16_free_of = [&](int n) { return (NK == 2 && (n & 1)) ? v_full + S + 1 : k16_free; };
  auto k16_use = [&](int n) { return (uint32_t)((n / NK) & 1); };   // phase of tile n's use
  auto v16_full_of = [&](int n) { return (NV == 2 && (n & 1)) ? v_full + S + 2 : v16_full; };
  auto v16_free_of = [&](int n) { return (NV == 2 && (n & 1)) ? v_full + S + 3 : v16_free; };
  auto v16_use = [&](int n) { return (uint32_t)((n / NV) & 1); };

  const int split = blockIdx.x % p.n_splits;
  const int grp = blockIdx.x / p.n_splits;
  const int b = grp / p.groups_per_seq;
  const int t0 = (grp % p.groups_per_seq) * G;
  const int t_last = min(p.T, t0 + G) - 1;
  const long long i_last = p.qpos0 + t_last;
  const long long k_lo = (long long)split * p.split_keys;
  const long long k_hi = min(min(k_lo + p.split_keys, i_last + 1), p.L);
  const long long part = (long long)grp * p.n_splits + split;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (k_lo >= k_hi) {  // empty split: neutral partial
    if (split == 0)
      for (int u = threadIdx.x; u < G * kHistBins; u += blockDim.x) {
        const int t = t0 + u / kHistBins;
        if (t < p.T) p.hist[((long long)b * p.T + t) * kHistBins + (u % kHistBins)] = 0u;
      }
    for (int u = threadIdx.x; u < N * 128; u += blockDim.x) p.part_o[part * N * 128 + u] = 0.f;
    if (threadIdx.x < N) p.part_ml[part * N + threadIdx.x] = make_float2(kNegInf, 0.f);
    return;
  }
  const int n_tiles = (int)((k_hi - k_lo + kTcKeys - 1) / kTcKeys);
  const uint32_t q_addr = smem_u32(smem + SM::kQOff);
  const uint32_t p_addr = smem_u32(smem + SM::kPOff);

  if (warp == 0) {
    // -------------------------------------------------------------- TMA
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      const uint64_t pol_k = policy_evict_normal(), pol_v = policy_evict_first();
      for (int n = 0; n < n_tiles; ++n) {
        const int s = n % S;
        if (n >= S && !mbar_wait(&kv_empty[s], ((n / S) - 1) & 1)) break;
        uint8_t* st = smem + s * SM::kStageBytes;
        const int row = (int)((long long)b * p.L + k_lo + (long long)n * kTcKeys);
        if (FP8) {  // 128-byte E4M3 rows: one box per tensor, both on kv_full
          mbar_arrive_expect_tx(&kv_full[s], SM::kStageBytes);
          tma_load_2d(st, &kmap, &kv_full[s], 0, row, pol_k);
          tma_load_2d(st + kTileIn, &vmap, &kv_full[s], 0, row, pol_v);
        } else {  // K on kv_full, V on v_full: QK(n) need not wait for V(n)
          mbar_arrive_expect_tx(&kv_full[s], kTileIn);
          tma_load_2d(st, &kmap, &kv_full[s], 0, row, pol_k);
          tma_load_2d(st + 16384, &kmap, &kv_full[s], 64, row, pol_k);
          mbar_arrive_expect_tx(&v_full[s], kTileIn);
          tma_load_2d(st + kTileIn, &vmap, &v_full[s], 0, row, pol_v);
          tma_load_2d(st + kTileIn + 16384, &vmap, &v_full[s], 64, row, pol_v);
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t k16_addr = smem_u32(smem + SM::kK16Off);
      const uint32_t v16_addr = smem_u32(smem + SM::kV16Off);
      bool ok = true;
      auto pv = [&](int m) {
        if (!mbar_wait(&p_full[m % NP], (m / NP) & 1)) return false;
        if (FP8 && !mbar_wait(v16_full_of(m), v16_use(m))) return false;
        if (!FP8 && !mbar_wait(&v_full[m % S], (m / S) & 1)) return false;
        tc_fence_after();
        tc_issue_pv<N, FP8>(tmem + kOCol,
                            FP8 ? v16_addr + (uint32_t)((m % NV) * kTcTileBytes)
                                : smem_u32(smem + (m % S) * SM::kStageBytes + kTileIn),
                            p_addr + (m % NP) * SM::kPBytes, m > 0);
        tc_commit(&pv_done[m % NP]);
        tc_commit(FP8 ? v16_free_of(m) : &kv_empty[m % S]);
        return true;
      };
      ok = mbar_wait(q_ready, 0);  // Q staged by the softmax warps
      for (int n = 0; n < n_tiles && ok; ++n) {
        const int s = n % S, bb = n & 1;
        if (!mbar_wait(FP8 ? k16_full_of(n) : &kv_full[s], FP8 ? k16_use(n) : (n / S) & 1)) break;
        if (!RETAIN && n >= 2 && !mbar_wait(&s_empty[bb], ((n - 2) >> 1) & 1)) break;
        tc_fence_after();
        tc_issue_qk<N, FP8>(tmem + s_col(n),
                            FP8 ? k16_addr + (uint32_t)((n % NK) * kTcTileBytes)
                                : smem_u32(smem + s * SM::kStageBytes),
                            q_addr);
        tc_commit(&s_full[bb]);
        if (FP8) tc_commit(k16_free_of(n));
        if (n >= 1) ok = pv(n - 1);
      }
      if (ok) pv(n_tiles - 1);
    }
  } else if (FP8 && warp >= 2 + kTcSoftmax / 32) {
    // ----------------------------------------------- E4M3 -> f16 converters
    const int ct = threadIdx.x - (64 + kTcSoftmax);  // 0..127
    const bool is_v = ct >= kTcConvert;
    const int cid = ct % kTcConvert;
    const int nbuf = is_v ? NV : NK;   // f16 buffers of this tensor
    for (int n = 0; n < n_tiles; ++n) {
      const int s = n % S;
      uint8_t* dst = smem + (is_v ? SM::kV16Off : SM::kK16Off) + (n % nbuf) * kTcTileBytes;
      uint64_t* full16 = is_v ? v16_full_of(n) : k16_full_of(n);
      uint64_t* free16 = is_v ? v16_free_of(n) : k16_free_of(n);
      if (!mbar_wait(&kv_full[s], (n / S) & 1)) break;
      // the MMAs are done with the tile this buffer held before (tile n - nbuf)
      if (n >= nbuf && !mbar_wait(free16, ((n - nbuf) / nbuf) & 1)) break;
      fp8_rows_to_f16(smem + s * SM::kStageBytes + (is_v ? kTileIn : 0), 0, kTcKeys, cid,
                      kTcConvert, dst);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&kv_empty[s]);
        mbar_arrive(full16);
      }
    }
  } else {
    // ---------------------------------------------------------- softmax
    // stage Q (read by the tensor cores: fence to the async proxy, then publish)
    tc_stage_q<N, FP8>(p, b, t0, smem + SM::kQOff, threadIdx.x - 64, kTcSoftmax);
    fence_proxy_async_smem();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(q_ready);
    if (split == 0)  // clear the group's level-1 selection histograms
      for (int u = threadIdx.x - 64; u < G * kHistBins; u += kTcSoftmax) {
        const int t = t0 + u / kHistBins;
        if (t < p.T) p.hist[((long long)b * p.T + t) * kHistBins + (u % kHistBins)] = 0u;
      }
    const int wq = warp & 3;                 // TMEM lane quarter
    const int c0 = ((warp - 2) >> 2) * NC;   // first of this warp's NC columns
    const int st = threadIdx.x - 64;         // softmax thread 0..255
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const int keyrow = wq * 32 + lane;       // row of S^T (key) / of O^T (d)
    // P^T store address of (row c0 + c, this key): base + c*128 + (the 16-byte
    // chunk of this key's 8-key group, swizzled by the row) + 2 * (key & 7)
    // (K-major P^T); for 128-row groups P is stored MN-major instead: this
    // key's 128-byte row of the 64-row half c0/64, 16-byte chunks swizzled by key
    constexpr bool kPMN = tc_p_mn_major(N);
    uint8_t* p_base = smem + SM::kPOff + (keyrow >> 6) * (N * 128) + c0 * 128;
    uint8_t* pmn_row = smem + SM::kPOff + (c0 / 64) * (kTcKeys * 128) + keyrow * 128;
    const uint32_t kchunk = (uint32_t)(keyrow & 63) >> 3;  // this key's 16-byte chunk of a row
    const uint32_t kpair = (uint32_t)(keyrow & 6) * 2;     // its lane pair's byte in the chunk
    bool failed = false;
    // this key's row sums: in registers for 16-column rows, else in TMEM at 3N
    constexpr bool kLReg = NC <= 16;
    static_assert(!RETAIN || kLReg, "a retaining pass keeps the row sums in registers");
    float lreg[kLReg ? NC : 1];
#pragma unroll
    for (int i = 0; i < (kLReg ? NC : 1); ++i) lreg[i] = 0.f;
    if (!kLReg) {  // TMEM is undefined at allocation: clear this thread's row sums
      float z[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z[i] = 0.f;
#pragma unroll
      for (int c = 0; c < NC; c += 16) tmem_st16(tmem + lane_base + 3 * N + c0 + c, z);
      tmem_st_wait();
    }
    // E4M3: this key's scales, loaded one tile ahead of their use
    auto load_scales = [&](int n, float& ks, float& vs) {
      const long long jn = k_lo + (long long)n * kTcKeys + keyrow;
      const bool in = FP8 && n < n_tiles && jn < k_hi;
      ks = in ? p.k_scale[(long long)b * p.L + jn] : 0.f;
      vs = in ? p.v_scale[(long long)b * p.L + jn] : 0.f;
    };
    float ks_next = 0.f, vs_next = 0.f;
    if (FP8) load_scales(0, ks_next, vs_next);
    for (int n = 0; n < n_tiles; ++n) {
      const int bb = n & 1;
      const long long key0 = k_lo + (long long)n * kTcKeys;
      const long long j = key0 + keyrow;
      // this key's logit multiplier and P factor (per-token scales of an E4M3 cache)
      float sl = p.scale_log2, vsc = 1.f;
      if (FP8) {
        sl *= ks_next;
        vsc = vs_next;
        load_scales(n + 1, ks_next, vs_next);
      }
      failed |= !mbar_wait(&s_full[bb], (n >> 1) & 1);
      tc_fence_after();
      // a tile is "full" when every key is in range and causal for every query
      const bool full_tile = key0 + kTcKeys <= k_hi && key0 + kTcKeys - 1 <= p.qpos0 + t0;
      // key j (in range) is seen by the group's queries q >= j - qpos0 - t0.  This
      // thread's columns c0 .. c0+NC-1 are rows of queries c0/kH + (0 .. NQ-1):
      // vis[(c + i) / kH] is indexed at compile time (a per-query array with a
      // runtime index would sit in local memory)
      constexpr int NQ = (NC + kH - 1) / kH;
      bool vis[NQ];
#pragma unroll
      for (int k = 0; k < NQ; ++k) vis[k] = j < k_hi && (long long)(c0 / kH + k) >= j - p.qpos0 - t0;
      const uint32_t s_addr = tmem + lane_base + s_col(n) + c0;
      // kHold (NC <= 16): this key's logits of the warp's rows are loaded once and
      // kept for both sweeps; wider rows reload 16 columns at a time (registers)
      constexpr bool kHold = NC <= 16;
      float xs[kHold ? NC : 16];
      if (kHold) {
#pragma unroll
        for (int c = 0; c < NC; c += 16) tmem_ld16(s_addr + c, xs + (c % (kHold ? NC : 16)));
        tmem_ld_wait();
      }
      // p = 2^(x - m_ref), row sums, P^T (bf16, or f16 times the value scale for
      // an E4M3 cache) for the PV product; RETAIN: p replaces the logits in the
      // tile's TMEM block, with the tile's reference kept.  With `guard`, a logit
      // above its row's reference by more than 2^8 counts as 0 and is reported
      // (the tile is then redone after a rescale); undo: subtract the same
      // guarded values from the row sums again.
      uint8_t* pt = p_base + (n % NP) * SM::kPBytes;
      auto sweep = [&](bool guard, bool undo) {
        bool over_any = false;
#pragma unroll
        for (int c = 0; c < NC; c += 16) {
          float lv[16], pk[16];
          if (!kHold) tmem_ld16(s_addr + c, xs);
          if (kLReg) {
#pragma unroll
            for (int i = 0; i < 16; ++i) lv[i] = lreg[(c + i) % (kLReg ? NC : 1)];
          } else {
            tmem_ld16(tmem + lane_base + 3 * N + c0 + c, lv);
          }
          if (!kHold || !kLReg) tmem_ld_wait();
          const float* x = xs + (kHold ? c : 0);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int col = c0 + c + i;
            const bool ok = full_tile || vis[(c + i) / kH];
            const float mr = m_ref[col];
            const float xl = x[i] * sl;
            const bool over = guard && ok && xl > mr + kRescaleAbove;
            over_any |= over;
            const float pr = (ok && !over && mr != kNegInf) ? fast_exp2(xl - mr) : 0.f;
            pk[i] = pr;
            lv[i] = undo ? lv[i] - pr : lv[i] + pr;
          }
          if (!kPMN && !undo) {
            // P^T K-major: the two keys of a lane pair share each row's 4-byte
            // word -- the even lane writes rows c+2u, the odd lane rows c+2u+1
            const bool odd = (lane & 1) != 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float lo = FP8 ? pk[2 * u] * vsc : pk[2 * u];
              const float hi = FP8 ? pk[2 * u + 1] * vsc : pk[2 * u + 1];
              const float other = __shfl_xor_sync(0xffffffffu, odd ? lo : hi, 1);
              const uint32_t w = FP8 ? (odd ? pack_f16(other, hi) : pack_f16(lo, other))
                                     : (odd ? pack_bf16(other, hi) : pack_bf16(lo, other));
              const int r = c + 2 * u + (odd ? 1 : 0);
              *reinterpret_cast<uint32_t*>(pt + r * 128 + ((kchunk ^ (uint32_t)((c0 + r) & 7)) << 4) +
                                           kpair) = w;
            }
          }
          if (kPMN && !undo) {  // this key's 16 rows c0+c .. c0+c+15: two packed 16-byte chunks
            uint32_t w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
              w[u] = FP8 ? pack_f16(pk[2 * u] * vsc, pk[2 * u + 1] * vsc)
                         : pack_bf16(pk[2 * u], pk[2 * u + 1]);
            uint8_t* prow = pmn_row + (n % NP) * SM::kPBytes;
            const int ch = c >> 3;
            *reinterpret_cast<uint4*>(prow + ((ch ^ (keyrow & 7)) << 4)) =
                make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(prow + (((ch + 1) ^ (keyrow & 7)) << 4)) =
                make_uint4(w[4], w[5], w[6], w[7]);
          }
          if (kLReg) {
#pragma unroll
            for (int i = 0; i < 16; ++i) lreg[(c + i) % (kLReg ? NC : 1)] = lv[i];
          } else {
            tmem_st16(tmem + lane_base + 3 * N + c0 + c, lv);
          }
          if (RETAIN && !undo) tmem_st16(s_addr + c, pk);
        }
        return over_any;
      };
      // Wide rows (kOne: not held in registers) take one sweep with the current
      // references and redo the tile only when one must be raised (rare after
      // the first tiles); 16-column rows check first (sweep 1), then sweep.
      constexpr bool kOne = !kHold && !RETAIN;
      bool need = false;
      if (!kOne) {
        // sweep 1: does any logit exceed its row's reference by more than 2^8?
#pragma unroll
        for (int c = 0; c < NC; c += 16) {
          if (!kHold) {
            tmem_ld16(s_addr + c, xs);
            tmem_ld_wait();
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const bool ok = full_tile || vis[(c + i) / kH];
            need |= ok && xs[(kHold ? c : 0) + i] * sl > m_ref[c0 + c + i] + kRescaleAbove;
          }
        }
      }
      if (n >= NP) {  // the P^T buffer of this tile is free once PV(n - NP) is done
        failed |= !mbar_wait(&pv_done[n % NP], ((n - NP) / NP) & 1);
        tc_fence_after();
      }
      if (kOne) need = sweep(true, false);
      const bool any_need = softmax_any<kTcSoftmax>(need);
      if (softmax_any<kTcSoftmax>(failed)) break;
      if (any_need) {
        if (kOne) {  // the row sums lose this tile's guarded values again
          tmem_st_wait();
          sweep(true, true);
          tmem_st_wait();
        }
        // new reference: column max of this tile's logits (and the old reference)
#pragma unroll
        for (int c = 0; c < NC; c += 16) {
          if (!kHold) {
            tmem_ld16(s_addr + c, xs);
            tmem_ld_wait();
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const bool ok = full_tile || vis[(c + i) / kH];
            const float v = warp_max(ok ? xs[(kHold ? c : 0) + i] * sl : kNegInf);
            if (lane == 0) tmax[wq * N + c0 + c + i] = v;
          }
        }
        softmax_sync<kTcSoftmax>();
        if (st < N) {
          const float mo = m_ref[st];
          const float mn = fmaxf(fmaxf(mo, fmaxf(tmax[st], tmax[N + st])),
                                 fmaxf(tmax[2 * N + st], tmax[3 * N + st]));
          corr[st] = (mn == kNegInf) ? 1.f : fast_exp2(mo - mn);
          m_ref[st] = mn;
        }
        softmax_sync<kTcSoftmax>();
        if (n >= 1) {  // O^T is rescaled once PV(n - 1) is done
          failed |= !mbar_wait(&pv_done[(n - 1) % NP], ((n - 1) / NP) & 1);
          tc_fence_after();
        }
#pragma unroll
        for (int c = 0; c < NC; c += 16) {
          float v[16];
          if (kLReg) {
#pragma unroll
            for (int i = 0; i < 16; ++i) lreg[(c + i) % (kLReg ? NC : 1)] *= corr[c0 + c + i];
          } else {
            tmem_ld16(tmem + lane_base + 3 * N + c0 + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= corr[c0 + c + i];
            tmem_st16(tmem + lane_base + 3 * N + c0 + c, v);
          }
          if (n >= 1) {
            tmem_ld16(tmem + lane_base + kOCol + c0 + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= corr[c0 + c + i];
            tmem_st16(tmem + lane_base + kOCol + c0 + c, v);
          }
        }
        tmem_st_wait();  // the rescaled row sums are read back below
      }
      if (RETAIN && st < N)
        reinterpret_cast<float*>(smem + SM::kMhistOff)[n * N + st] = m_ref[st];
      if (!kOne || any_need) sweep(false, false);
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s_empty[bb]);
        mbar_arrive(&p_full[n % NP]);
      }
    }
    // ------------------------------------------------------- epilogue
    failed |= !mbar_wait(&pv_done[(n_tiles - 1) % NP], ((n_tiles - 1) / NP) & 1);
    tc_fence_after();
    if (!softmax_any<kTcSoftmax>(failed)) {
      float* lsum = tmax;  // [4 quarters][N]
#pragma unroll
      for (int c = 0; c < NC; c += 16) {
        float v[16];
        if (kLReg) {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = lreg[(c + i) % (kLReg ? NC : 1)];
        } else {
          tmem_ld16(tmem + lane_base + 3 * N + c0 + c, v);
          tmem_ld_wait();
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float s = warp_sum(v[i]);
          if (lane == 0) lsum[wq * N + c0 + c + i] = s;
        }
      }
#pragma unroll
      for (int c = 0; c < NC; c += 16) {
        float v[16];
        tmem_ld16(tmem + lane_base + kOCol + c0 + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) p.part_o[(part * N + c0 + c + i) * 128 + keyrow] = v[i];
      }
      softmax_sync<kTcSoftmax>();
      if (st < N) {
        const float lt = lsum[st] + lsum[N + st] + lsum[2 * N + st] + lsum[3 * N + st];
        p.part_ml[part * N + st] = make_float2(m_ref[st], lt);
      }
    }
    tc_fence_before();
  }
}

template <int N, int G, bool FP8>
__global__ void __launch_bounds__(tc_partial_threads(FP8), 1)
    attn_tc_partial_kernel(const __grid_constant__ CUtensorMap kmap,
                           const __grid_constant__ CUtensorMap vmap, const FullAttnParams p) {
  using SM = TcSmem<N, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kSlotOff);
  tc_partial_setup<N, FP8>(smem);
  if (threadIdx.x / 32 == 1) {
    tmem_alloc(tmem_slot, 4 * N);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  tc_partial_body<N, G, FP8>(kmap, vmap, p, smem, tmem);
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x / 32 == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 4 * N);
  }
}


// Arrival at a group-wide barrier of CTAs through a global counter (zeroed
// before the launch), then a bounded wait until `target` CTAs have arrived.
// Whole CTA.  The CTAs of a group must be co-resident (cooperative launch).
// Returns false in every thread of the CTA when the wait gave up (after
// limit_ns of %globaltimer, or 2^24 polls), having raised kStatusTimeout.
__device__ __forceinline__ bool group_arrive_wait(unsigned* ctr, unsigned target,
                                                  unsigned long long limit_ns) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    atomicAdd(ctr, 1u);
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 0;; ++it) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
      if (v >= target) break;
      if (it >= (1u << 24) || ((it & 15u) == 15u && globaltimer() - t0 > limit_ns)) {
        raise_status(kStatusTimeout);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// Fused decode pass: the partial pass of this CTA's (group, split), then --
// once every split of the group has its partials -- the score pass over the
// same split's keys (its K tiles are still in L2) while four warps merge this
// split's share of the group's output rows, then (fuse_select) the selection
// of the group's rows by all of the group's CTAs together, each keeping its
// split's candidate scores in shared memory (two more group barriers; see
// below).  Without fuse_select a separate selection kernel follows.
template <int N, int G, bool FP8, bool RETAIN>
__global__ void __launch_bounds__(tc_partial_threads(FP8), 1)
    attn_tc_fused_kernel(const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap, const FullAttnParams p) {
  constexpr uint32_t kTmemCols = RETAIN ? 512 : 4 * N;
  using SM = TcSmem<N, FP8>;
  static_assert(SM::kFusable, "score pass does not fit the tile ring");
  constexpr int kThreads = tc_partial_threads(FP8);
  constexpr int S2 = SM::kS2Stages;
  constexpr int kH = N / G;
  constexpr int W = kThreads / 32;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_res[2], s_tmp[32], s_prefix[4], s_need[4], s_base[2];
  static_assert(W <= 16, "per-warp counters");
  __shared__ int s_wg[4][16], s_we[4][16];
  uint8_t* smem = align1024(smem_raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kSlotOff);
  uint64_t* kv2_full = reinterpret_cast<uint64_t*>(smem + SM::kBar2Off);
  uint64_t* kv2_empty = kv2_full + S2;
  uint64_t* s2_full = kv2_empty + S2;  // [2]
  uint64_t* s2_empty = s2_full + 2;    // [2]
  uint64_t* k2_full = s2_empty + 2;    // [2], E4M3 only
  uint64_t* k2_free = k2_full + 2;     // [2]

  // phase k of this CTA reached: one global-timer stamp (tracing; off when null)
  // (written by thread `by` of the CTA, at a point that thread reaches only
  // once the phase is done: a timer read right after a block barrier may be
  // scheduled before it)
  auto stamp = [&](int k, int by = 0) {
    if (p.phase_stamps && threadIdx.x == by && (int)blockIdx.x < p.phase_ctas)
      p.phase_stamps[blockIdx.x * kPhases + k] = globaltimer();
  };
  stamp(0);
  pdl_launch_dependents();  // a following sparse layer may place its CTAs on idle SMs
  tc_partial_setup<N, FP8>(smem);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S2; ++s) {
      mbar_init(&kv2_full[s], 1);
      mbar_init(&kv2_empty[s], FP8 ? 2 * kTcConvert / 32 : 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s2_full[i], 1);
      mbar_init(&s2_empty[i], 4);
      mbar_init(&k2_full[i], 2 * kTcConvert / 32);
      mbar_init(&k2_free[i], 1);
    }
    fence_mbar_init();
  }
  if (threadIdx.x / 32 == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ------------------------------------------------------------ partials
  tc_partial_body<N, G, FP8, RETAIN>(kmap, vmap, p, smem, tmem);

  const int ns = p.n_splits;
  const int split = blockIdx.x % ns;
  const int grp = blockIdx.x / ns;
  const int b = grp / p.groups_per_seq;
  const int t0 = (grp % p.groups_per_seq) * G;
  const int t_last = min(p.T, t0 + G) - 1;
  const long long i_last = p.qpos0 + t_last;
  const long long k_lo = (long long)split * p.split_keys;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  unsigned* gsync = p.grp_sync + 8 * grp;
  const unsigned target = (unsigned)ns + p.barrier_extra;
  // a group barrier that gave up ends the CTA: nothing is in flight (the
  // partial pass has drained its TMA and MMA pipelines), so only the TMEM
  // columns are released
  auto give_up = [&]() {
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
  };
  stamp(1, 64);  // the first softmax thread has written its rows' partials
  tc_fence_before();
  if (!group_arrive_wait(gsync, target, p.wait_limit_ns)) {  // the group's partials are out
    give_up();
    return;
  }
  stamp(2);
  tc_fence_after();

  // --------------------------------------------------------- score pass
  const long long k2_hi = min(k_lo + (long long)p.split_keys, i_last - p.window + 1);
  const int n2 = k_lo < k2_hi ? (int)((k2_hi - k_lo + kTcKeys - 1) / kTcKeys) : 0;
  float2* ml_s = reinterpret_cast<float2*>(smem + SM::kS2MlOff);  // [N][ns]
  unsigned* hist_s = reinterpret_cast<unsigned*>(smem + SM::kS2HistOff);
  float* lse2_s = reinterpret_cast<float*>(smem + SM::kCorrOff);
  uint8_t* k16 = smem + SM::kK16Off;  // E4M3: two f16 K tiles
  // fuse_select: this split's candidate scores of row q at seg[q * split_keys + (j - k_lo)]
  float* seg = reinterpret_cast<float*>(smem + SM::kPOff);
  // RETAIN: the logits of every tile are still in TMEM: no loads, no MMA
  if (warp == 0) {
    if (lane == 0 && !RETAIN) {
      const uint64_t pol = policy_evict_first();
      for (int n = 0; n < n2; ++n) {
        const int s = n % S2;
        if (n >= S2 && !mbar_wait(&kv2_empty[s], ((n / S2) - 1) & 1)) break;
        uint8_t* st = smem + s * SM::kS2TileBytes;
        mbar_arrive_expect_tx(&kv2_full[s], SM::kS2TileBytes);
        const int row = (int)((long long)b * p.L + k_lo + (long long)n * kTcKeys);
        tma_load_2d(st, &kmap, &kv2_full[s], 0, row, pol);
        if (!FP8) tma_load_2d(st + 16384, &kmap, &kv2_full[s], 64, row, pol);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && !RETAIN) {
      const uint32_t q_addr = smem_u32(smem + SM::kQOff);
      for (int n = 0; n < n2; ++n) {
        const int s = n % S2, bb = n & 1;
        if (FP8) {
          if (!mbar_wait(&k2_full[bb], (n >> 1) & 1)) break;
        } else if (!mbar_wait(&kv2_full[s], (n / S2) & 1)) {
          break;
        }
        if (n >= 2 && !mbar_wait(&s2_empty[bb], ((n - 2) >> 1) & 1)) break;
        tc_fence_after();
        tc_issue_qk<N, FP8>(tmem + bb * N,
                            FP8 ? smem_u32(k16 + bb * kTcTileBytes)
                                : smem_u32(smem + s * SM::kS2TileBytes),
                            q_addr);
        tc_commit(&s2_full[bb]);
        tc_commit(FP8 ? &k2_free[bb] : &kv2_empty[s]);
      }
    }
  } else if (FP8 && warp >= 2 + kTcSoftmax / 32) {
    // E4M3 -> f16: every converter warp (both the partial pass's K and V ones)
    // converts its share of each K tile
    const int ct = threadIdx.x - (64 + kTcSoftmax);
    if (!RETAIN)
      for (int n = 0; n < n2; ++n) {
        const int s = n % S2, bb = n & 1;
        if (!mbar_wait(&kv2_full[s], (n / S2) & 1)) break;
        if (n >= 2 && !mbar_wait(&k2_free[bb], ((n - 2) >> 1) & 1)) break;
        fp8_rows_to_f16(smem + s * SM::kS2TileBytes, 0, kTcKeys, ct, 2 * kTcConvert,
                        k16 + bb * kTcTileBytes);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&kv2_empty[s]);
          mbar_arrive(&k2_full[bb]);
        }
      }
  } else {
    // warps 2-9: the group's (m, l) partials and lse (base 2) of its rows
    const int st = threadIdx.x - 64;
    const float2* ml_g = p.part_ml + (long long)grp * ns * N;
    // merge warps 6-9: the partial O of the first row this CTA merges (row
    // `split`, up to kPre splits) does not depend on lse -- load it now
    constexpr int kPre = FP8 ? 16 : 32;  // (E4M3: 128 registers per thread)
    float pre[kPre];
    if (warp >= 6 && split < N && t0 + split / kH < p.T) {
      const float* po = p.part_o + ((long long)grp * ns * N + split) * 128 + (threadIdx.x - 192);
#pragma unroll
      for (int k = 0; k < kPre; ++k) pre[k] = k < ns ? __ldcg(po + (long long)k * N * 128) : 0.f;
    }
    {
      constexpr int kLoadBatch = 4;   // independent L2 loads in flight per thread
      for (int u0 = st; u0 < N * ns; u0 += kLoadBatch * kTcSoftmax) {
        float2 v[kLoadBatch];
#pragma unroll
        for (int k = 0; k < kLoadBatch; ++k) {
          const int u = u0 + k * kTcSoftmax;
          v[k] = u < N * ns ? __ldcg(ml_g + u) : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kLoadBatch; ++k) {
          const int u = u0 + k * kTcSoftmax;
          if (u < N * ns) ml_s[(u % N) * ns + u / N] = v[k];
        }
      }
    }
    softmax_sync<kTcSoftmax>();
    {  // eight threads per row, each over every eighth split, then a shuffle combine
      static_assert(N * 8 == kTcSoftmax, "eight threads per row");
      const int r = st >> 3, sub = st & 7;
      float M = kNegInf;
      for (int sp = sub; sp < ns; sp += 8) M = fmaxf(M, ml_s[r * ns + sp].x);
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      float lt = 0.f;
      if (M != kNegInf)
        for (int sp = sub; sp < ns; sp += 8) {
          const float2 v = ml_s[r * ns + sp];
          lt += v.x == kNegInf ? 0.f : v.y * fast_exp2(v.x - M);
        }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) lt += __shfl_xor_sync(0xffffffffu, lt, o);
      if (sub == 0) lse2_s[r] = M + log2f(lt);
    }
    softmax_sync<kTcSoftmax>();
    // RETAIN: TMEM holds p = 2^(x - m_ref(tile)); f[tile][r] = 2^(m_ref(tile) - lse)
    // turns it into the softmax probability
    float* fct = reinterpret_cast<float*>(smem + SM::kMhistOff);
    if (RETAIN) {
      for (int u = st; u < n2 * N; u += kTcSoftmax) {
        const float mr = fct[u];
        fct[u] = mr == kNegInf ? 0.f : fast_exp2(mr - lse2_s[u % N]);
      }
      softmax_sync<kTcSoftmax>();
    }
    if (warp < 6) {
      // ---- score warps 2-5: one key (TMEM lane) each per tile
      const int sc = threadIdx.x - 64;
      for (int u = sc; u < G * kHistBins; u += 128) hist_s[u] = 0u;
      asm volatile("bar.sync 2, 128;" ::: "memory");
      const int wq = warp & 3;
      const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
      const int keyrow = wq * 32 + lane;
      auto load_ks = [&](int n) {
        const long long jn = k_lo + (long long)n * kTcKeys + keyrow;
        return (FP8 && !RETAIN && n < n2 && jn < k2_hi) ? p.k_scale[(long long)b * p.L + jn] : 0.f;
      };
      // tile n's candidate scores of this key: the selection's copies and histogram
      auto emit = [&](int n, const float* acc) {
        const long long j = k_lo + (long long)n * kTcKeys + keyrow;
#pragma unroll
        for (int q = 0; q < G; ++q) {
          const int t = t0 + q;
          const bool cand = t < p.T && j <= p.qpos0 + t - p.window;
          if (cand) {  // the fused selection reads the shared-memory copy only
            if (p.fuse_select) seg[q * p.split_keys + (int)(j - k_lo)] = acc[q];
            else p.score[((long long)b * p.T + t) * p.L + j] = acc[q];
          }
          hist_inc(hist_s + q * kHistBins, __float_as_uint(acc[q]) >> kHistShift, cand);
        }
      };
      if (RETAIN) {
        // two tiles' blocks per TMEM round trip; each query's 32/G-term dot
        // product in four independent partial sums
        auto dot = [&](int n, const float* x, float* acc) {
          const float4* f4 = reinterpret_cast<const float4*>(fct + n * N);
          float a4[G][4];
#pragma unroll
          for (int q = 0; q < G; ++q) a4[q][0] = a4[q][1] = a4[q][2] = a4[q][3] = 0.f;
#pragma unroll
          for (int i4 = 0; i4 < N / 4; ++i4) {
            const float4 f = f4[i4];
            const int q = 4 * i4 / kH;
            a4[q][0] = fmaf(x[4 * i4], f.x, a4[q][0]);
            a4[q][1] = fmaf(x[4 * i4 + 1], f.y, a4[q][1]);
            a4[q][2] = fmaf(x[4 * i4 + 2], f.z, a4[q][2]);
            a4[q][3] = fmaf(x[4 * i4 + 3], f.w, a4[q][3]);
          }
#pragma unroll
          for (int q = 0; q < G; ++q) acc[q] = (a4[q][0] + a4[q][1]) + (a4[q][2] + a4[q][3]);
        };
        for (int n = 0; n < n2; n += 2) {
          float x0[32], x1[32], acc[G];
          tmem_ld32(tmem + lane_base + N + n * N, x0);
          if (n + 1 < n2) tmem_ld32(tmem + lane_base + N + (n + 1) * N, x1);
          tmem_ld_wait();
          dot(n, x0, acc);
          emit(n, acc);
          if (n + 1 < n2) {
            dot(n + 1, x1, acc);
            emit(n + 1, acc);
          }
        }
        tc_fence_before();
      } else {
        float ks_next = load_ks(0);  // E4M3: one tile ahead of its use
        for (int n = 0; n < n2; ++n) {
          const int bb = n & 1;
          float sl = p.scale_log2;
          if (FP8) {
            sl *= ks_next;
            ks_next = load_ks(n + 1);
          }
          if (!mbar_wait(&s2_full[bb], (n >> 1) & 1)) break;
          tc_fence_after();
          float acc[G];
#pragma unroll
          for (int q = 0; q < G; ++q) acc[q] = 0.f;
#pragma unroll
          for (int c = 0; c < N / 32; ++c) {
            float x[32];
            tmem_ld32(tmem + lane_base + bb * N + 32 * c, x);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              acc[(32 * c + i) / kH] += fast_exp2(x[i] * sl - lse2_s[32 * c + i]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s2_empty[bb]);
          emit(n, acc);
        }
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
      for (int u = sc; u < G * kHistBins; u += 128) {
        const unsigned cnt = hist_s[u];
        const int t = t0 + u / kHistBins;
        if (cnt && t < p.T)
          atomicAdd(&p.hist[((long long)b * p.T + t) * kHistBins + (u % kHistBins)], cnt);
      }
      stamp(3, 64);  // the score warps' candidate scores and histogram counts are out
    } else {
      // ---- merge warps 6-9: output row r of the group is merged by the CTA of
      //      split r mod ns; thread d owns element d
      const int d = threadIdx.x - 192;
      for (int r = split; r < N; r += ns) {
        const int t = t0 + r / kH;
        if (t >= p.T) continue;
        const float l2 = lse2_s[r];
        const long long li = ((long long)b * p.T + t) * p.H + r % kH;
        if (d == 0) {
          p.lse[li] = l2 * 0.69314718055994531f;
          if (p.lse_out) p.lse_out[li] = l2 * 0.69314718055994531f;
        }
        const float* po = p.part_o + ((long long)grp * ns * N + r) * 128 + d;
        float acc = 0.f;
        int sp_first = 0;
        if (r == split) {  // the prefetched splits
#pragma unroll
          for (int k = 0; k < kPre; ++k) {
            if (k >= ns) break;
            const float2 v = ml_s[r * ns + k];
            const float f = (v.x == kNegInf) ? 0.f : fast_exp2(v.x - l2);
            acc += f * pre[k];
          }
          sp_first = kPre;
        }
        constexpr int kLoadBatch = 24;   // the splits' values of element d, loaded together
        for (int sp0 = sp_first; sp0 < ns; sp0 += kLoadBatch) {
          float x[kLoadBatch];
#pragma unroll
          for (int k = 0; k < kLoadBatch; ++k)
            x[k] = sp0 + k < ns ? __ldcg(po + (long long)(sp0 + k) * N * 128) : 0.f;
#pragma unroll
          for (int k = 0; k < kLoadBatch; ++k) {
            if (sp0 + k >= ns) break;
            const float2 v = ml_s[r * ns + sp0 + k];
            const float f = (v.x == kNegInf) ? 0.f : fast_exp2(v.x - l2);
            acc += f * x[k];
          }
        }
        p.o[li * 128 + d] = acc;
      }
    }
  }
  tc_fence_before();
  __syncthreads();

  // ------------------------------------------ selection (whole group)
  // The k-th largest score pattern tau, as in select_topk_kernel, in two group
  // barriers.  (1) Once the level-1 histogram (bits [30:20], built by the
  // score pass) is complete, every CTA finds the bin b1 holding the k-th
  // candidate, counts its split's candidates above b1 and writes the ones in
  // b1 to its slice of the row's list.  (2) Once every split has done so, every
  // CTA loads the row's whole b1 list (split order) and finds tau and the
  // number of ties to keep from two more digit levels (bits [19:9], [8:0]) in
  // shared memory; the list prefix before its own slice gives the survivors of
  // the lower splits, and it writes its own survivors in position order.  The
  // chain runs once per launch, after the streaming: the in-list digit searches
  // are one warp's (no block-wide scans), and every reduction one block barrier.
  if (p.fuse_select) {
    const unsigned* segu = reinterpret_cast<const unsigned*>(seg);
    unsigned* list_s = reinterpret_cast<unsigned*>(smem);                 // the row's b1 list
    unsigned* h = reinterpret_cast<unsigned*>(smem + SM::kSelWorkOff);    // 2048 counters
    int* off_s = reinterpret_cast<int*>(smem + SM::kSelWorkOff + 8192);   // [ns + 1] list offsets
    // the same digit counts of the list elements before this split's slice
    unsigned* hp2 = reinterpret_cast<unsigned*>(smem + SM::kSelWorkOff + 12288);  // 2048
    unsigned* hp3 = hp2 + 2048;                                                   // 512
    __shared__ int s_red[2][16];
    auto row_of = [&](int q) { return (long long)b * p.T + t0 + q; };
    auto nc_of = [&](int q) { return p.qpos0 + t0 + q - p.window + 1; };
    auto active = [&](int q) { return t0 + q < p.T && nc_of(q) > p.topk && p.topk > 0; };
    auto nseg_of = [&](int q) {
      return (int)max(0LL, min((long long)p.split_keys, nc_of(q) - k_lo));
    };
    auto list_g = [&](int q, int sp) {
      return p.sel_list + (row_of(q) * ns + sp) * (long long)p.split_keys;
    };
    // block totals of two counts (one block barrier; s_red is free again after
    // the caller's next barrier)
    auto block_sum2 = [&](int x, int y, int& xt, int& yt) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        x += __shfl_xor_sync(0xffffffffu, x, o);
        y += __shfl_xor_sync(0xffffffffu, y, o);
      }
      if (lane == 0) {
        s_red[0][warp] = x;
        s_red[1][warp] = y;
      }
      __syncthreads();
      xt = 0;
      yt = 0;
      for (int w = 0; w < W; ++w) {
        xt += s_red[0][w];
        yt += s_red[1][w];
      }
    };
    if (!group_arrive_wait(gsync + 1, target, p.wait_limit_ns)) {  // level-1 counts complete
      give_up();
      return;
    }
    stamp(4);
#pragma unroll 1
    for (int q = 0; q < G; ++q)
      if (active(q)) {
        sel_find_bin_global<kThreads, 2048>(p.hist + row_of(q) * kHistBins, p.topk, s_res, s_tmp);
        const unsigned b1 = (unsigned)s_res[0];
        if (threadIdx.x == 0) {
          s_prefix[q] = s_res[0];
          s_need[q] = s_res[1];
        }
        // this split's candidates above b1 and in b1, per warp-contiguous part
        const int n = nseg_of(q);
        const int wseg = (n + W - 1) / W;
        const int w0 = min(n, warp * wseg), w1 = min(n, w0 + wseg);
        int n_gt = 0, n_in = 0;
        for (int base = w0; base < w1; base += 32) {
          const int u = base + lane;
          const unsigned d = u < w1 ? (segu[q * p.split_keys + u] >> 20) : 0u;
          n_gt += __popc(__ballot_sync(0xffffffffu, u < w1 && d > b1));
          n_in += __popc(__ballot_sync(0xffffffffu, u < w1 && d == b1));
        }
        if (lane == 0) {
          s_wg[q][warp] = n_gt;
          s_we[q][warp] = n_in;
        }
        __syncthreads();
        int in_before = 0, gt_tot = 0, in_tot = 0;
        for (int w = 0; w < W; ++w) {
          if (w < warp) in_before += s_we[q][w];
          gt_tot += s_wg[q][w];
          in_tot += s_we[q][w];
        }
        if (threadIdx.x == 0) p.sel_cnt[row_of(q) * ns + split] = make_int2(gt_tot, in_tot);
        unsigned* lg = list_g(q, split);
        for (int base = w0; base < w1; base += 32) {
          const int u = base + lane;
          const unsigned v = u < w1 ? segu[q * p.split_keys + u] : 0u;
          const bool in = u < w1 && (v >> 20) == b1;
          const unsigned m = __ballot_sync(0xffffffffu, in);
          if (in) lg[in_before + __popc(m & ((1u << lane) - 1u))] = v;
          in_before += __popc(m);
        }
        __syncthreads();  // s_res / s_w* are reused by the next row
      }
    // every split's counts and b1 slice are out
    if (!group_arrive_wait(gsync + 2, target, p.wait_limit_ns)) {
      give_up();
      return;
    }
    stamp(5);
#pragma unroll 1
    for (int q = 0; q < G; ++q)
      if (active(q)) {
        // list offsets of the splits, and this split's survivors-above-b1 base
        if (ns <= 32) {  // one warp scans the splits' counts
          if (warp == 0) {
            int2 c = make_int2(0, 0);
            if (lane < ns) c = __ldcg(p.sel_cnt + row_of(q) * ns + lane);
            int ix = c.y, gx = c.x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int yi = __shfl_up_sync(0xffffffffu, ix, o);
              const int yg = __shfl_up_sync(0xffffffffu, gx, o);
              if (lane >= o) {
                ix += yi;
                gx += yg;
              }
            }
            if (lane < ns) off_s[lane] = ix - c.y;
            if (lane == ns - 1) off_s[ns] = ix;
            if (lane == split) {
              s_base[0] = gx - c.x;  // candidates above b1 in the lower splits
              s_base[1] = ix - c.y;  // list index of this split's slice
            }
          }
        } else {
          int2 c = make_int2(0, 0);
          if (threadIdx.x < ns) c = __ldcg(p.sel_cnt + row_of(q) * ns + threadIdx.x);
          int in_ex, gt_ex;
          const int m_all = sel_block_scan<kThreads>(c.y, in_ex, s_tmp);
          sel_block_scan<kThreads>(c.x, gt_ex, s_tmp);
          if (threadIdx.x < ns) off_s[threadIdx.x] = in_ex;
          if (threadIdx.x == ns) off_s[ns] = m_all;
          if (threadIdx.x == split) {
            s_base[0] = gt_ex;
            s_base[1] = in_ex;
          }
        }
        for (int e = threadIdx.x; e < 2048; e += kThreads) h[e] = hp2[e] = 0u;
        for (int e = threadIdx.x; e < 512; e += kThreads) hp3[e] = 0u;
        __syncthreads();
        const int m = off_s[ns];
        const bool in_smem = m <= SM::kSelCap;
        // element e of the row's list: slice sp with off_s[sp] <= e < off_s[sp + 1]
        auto list_at = [&](int e) {
          int lo = 0, hi = ns - 1;
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (off_s[mid] <= e) lo = mid;
            else hi = mid - 1;
          }
          return __ldcg(list_g(q, lo) + (e - off_s[lo]));
        };
        if (in_smem) {
          // the slices, one warp each at a time: all loads of a warp's slices
          // are independent (a single L2 round trip for a decode row)
          for (int sp = warp; sp < ns; sp += W) {
            const int o = off_s[sp], cnt = off_s[sp + 1] - o;
            const unsigned* src = list_g(q, sp);
            for (int e = lane; e < cnt; e += 32) list_s[o + e] = __ldcg(src + e);
          }
          __syncthreads();
        }
        auto val = [&](int e) { return in_smem ? list_s[e] : list_at(e); };
        // levels 2 and 3 -- bits [19:9], then [8:0], of the list's elements that
        // share the digits found so far -- as one loop over the same code (it
        // runs once per launch, so every distinct instruction is fetched cold)
        // The survivors of the lower splits' b1 slices (list elements e < own)
        // come from the same passes: hp2 / hp3 count their digits, and those
        // above each level's bin are above tau.
        const int own = s_base[1];
        unsigned tau = (unsigned)s_prefix[q];
        int need_tau = s_need[q];
        int a = 0;
#pragma unroll 1
        for (int lvl = 0; lvl < 2; ++lvl) {
          const int shift = lvl == 0 ? 9 : 0;
          const int kept = lvl == 0 ? 20 : 9;   // bits above the digit: those found so far
          const int nb = lvl == 0 ? 2048 : 512;
          unsigned* hp = lvl == 0 ? hp2 : hp3;
          if (lvl == 1) {
            for (int e = threadIdx.x; e < 512; e += kThreads) h[e] = 0u;
            __syncthreads();
          }
          for (int e = threadIdx.x; e < m; e += kThreads) {
            const unsigned v = val(e);
            const unsigned bin = (v >> shift) & (unsigned)(nb - 1);
            const bool in = (v >> kept) == tau;
            hist_inc(h, bin, in);
            hist_inc(hp, bin, in && e < own);
          }
          __syncthreads();
          if (warp == 0) {
            if (lvl == 0) sel_find_bin_warp<2048>(h, need_tau, s_res);
            else sel_find_bin_warp<512>(h, need_tau, s_res);
          }
          __syncthreads();
          for (int e = threadIdx.x; e < nb; e += kThreads) a += e > s_res[0] ? (int)hp[e] : 0;
          tau = (tau << (lvl == 0 ? 11 : 9)) | (unsigned)s_res[0];
          need_tau = s_res[1];
        }
        int a_tot, unused;
        block_sum2(a, 0, a_tot, unused);
        const int tie_tot = (int)hp3[tau & 511u];
        // this split's survivors, per warp-contiguous part: v > tau, v == tau
        const int n = nseg_of(q);
        const int wseg = (n + W - 1) / W;
        const int w0 = min(n, warp * wseg), w1 = min(n, w0 + wseg);
        int n_gt = 0, n_eq = 0;
        for (int base = w0; base < w1; base += 32) {
          const int u = base + lane;
          const unsigned v = u < w1 ? segu[q * p.split_keys + u] : 0u;
          n_gt += __popc(__ballot_sync(0xffffffffu, u < w1 && v > tau));
          n_eq += __popc(__ballot_sync(0xffffffffu, u < w1 && v == tau));
        }
        if (lane == 0) {
          s_wg[q][warp] = n_gt;
          s_we[q][warp] = n_eq;
        }
        __syncthreads();
        int gt_before = s_base[0] + a_tot, eq_before = tie_tot;
        for (int w = 0; w < warp; ++w) {
          gt_before += s_wg[q][w];
          eq_before += s_we[q][w];
        }
        int32_t* out = p.idx + row_of(q) * p.slots;
        int pos = gt_before + min(eq_before, need_tau);
        int eq_rank = eq_before;
        for (int base = w0; base < w1; base += 32) {
          const int u = base + lane;
          const unsigned v = u < w1 ? segu[q * p.split_keys + u] : 0u;
          const bool gt = u < w1 && v > tau;
          const bool eq = u < w1 && v == tau;
          const unsigned eqm = __ballot_sync(0xffffffffu, eq);
          const int my_eq_rank = eq_rank + __popc(eqm & ((1u << lane) - 1u));
          const bool sel = gt || (eq && my_eq_rank < need_tau);
          const unsigned selm = __ballot_sync(0xffffffffu, sel);
          if (sel) {
            const int o = pos + __popc(selm & ((1u << lane) - 1u));
            if (o < p.topk) out[o] = (int32_t)(k_lo + u);
          }
          pos += __popc(selm);
          eq_rank += __popc(eqm);
        }
        if (split == ns - 1 && warp == W - 1 && lane == 0 && pos != p.topk)
          raise_status(kStatusBadIndex);
        __syncthreads();  // shared state is rewritten for the next row
      }
    if (split == 0)  // window, padding and count; or every position when all are taken
      for (int q = 0; q < G && t0 + q < p.T; ++q) {
        const long long i = p.qpos0 + t0 + q;
        int32_t* out = p.idx + row_of(q) * p.slots;
        if (nc_of(q) <= p.topk) {
          for (int j = threadIdx.x; j < p.slots; j += kThreads) out[j] = j <= i ? (int32_t)j : -1;
          if (threadIdx.x == 0) p.n_sel[row_of(q)] = (int32_t)(i + 1);
        } else {
          const long long wstart = i - p.window + 1;
          for (int w = threadIdx.x; w < p.window; w += kThreads)
            out[p.topk + w] = (int32_t)(wstart + w);
          for (int j = p.topk + p.window + threadIdx.x; j < p.slots; j += kThreads) out[j] = -1;
          if (threadIdx.x == 0) p.n_sel[row_of(q)] = p.topk + p.window;
        }
      }
  }
  tc_fence_before();
  __syncthreads();
  stamp(6);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Score kernel: warps 0 (TMA), 1 (MMA), score warps 2-9 in two groups of four
// on alternating tiles (plus, for an E4M3 cache, converter warps 10-13 writing
// double-buffered f16 K tiles).
template <int N, int G, bool FP8>
__global__ void __launch_bounds__(tc_score_threads(FP8), 1)
    attn_tc_score_kernel(const __grid_constant__ CUtensorMap kmap, const FullAttnParams p) {
  using SM = TcSmem<N, FP8>;
  constexpr int S = SM::kSStages;
  constexpr int kH = N / G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  float2* ml_s = reinterpret_cast<float2*>(smem + SM::kSMlOff);  // [N][n_splits]
  unsigned* hist_s = reinterpret_cast<unsigned*>(smem + SM::kSHistOff);
  float* lse2_s = reinterpret_cast<float*>(smem + SM::kSLseOff);
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(smem + SM::kSBarOff);
  uint64_t* kv_empty = kv_full + S;
  uint64_t* s_full = kv_empty + S;  // [2]
  uint64_t* s_empty = s_full + 2;   // [2]
  uint64_t* q_ready = s_empty + 2;
  uint64_t* k16_full = q_ready + 1;  // [2], E4M3 only
  uint64_t* k16_free = k16_full + 2; // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kSSlotOff);

  const int split = blockIdx.x % p.score_splits;
  const int grp = blockIdx.x / p.score_splits;
  const int b = grp / p.groups_per_seq;
  const int t0 = (grp % p.groups_per_seq) * G;
  const int t_last = min(p.T, t0 + G) - 1;
  const long long i_last = p.qpos0 + t_last;
  const long long k_lo = (long long)split * p.score_keys;
  const long long k_hi = min(min(k_lo + p.score_keys, i_last - p.window + 1), p.L);
  const int n_tiles = (!p.no_score && k_lo < k_hi) ? (int)((k_hi - k_lo + kTcKeys - 1) / kTcKeys) : 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ns = p.n_splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], FP8 ? 4 : 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
      mbar_init(&k16_full[i], 4);
      mbar_init(&k16_free[i], 1);
    }
    mbar_init(q_ready, 8);
    fence_mbar_init();
  }
  if (warp == 1 && n_tiles > 0) {
    tmem_alloc(tmem_slot, 2 * N);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = n_tiles > 0 ? *tmem_slot : 0u;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      const uint64_t pol = policy_evict_first();
      for (int n = 0; n < n_tiles; ++n) {
        const int s = n % S;
        if (n >= S && !mbar_wait(&kv_empty[s], ((n / S) - 1) & 1)) break;
        uint8_t* st = smem + s * SM::kSStageBytes;
        mbar_arrive_expect_tx(&kv_full[s], SM::kSStageBytes);
        const int row = (int)((long long)b * p.L + k_lo + (long long)n * kTcKeys);
        tma_load_2d(st, &kmap, &kv_full[s], 0, row, pol);
        if (!FP8) tma_load_2d(st + 16384, &kmap, &kv_full[s], 64, row, pol);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n_tiles > 0 && mbar_wait(q_ready, 0)) {  // Q staged by the score warps
      const uint32_t q_addr = smem_u32(smem + SM::kSQOff);
      for (int n = 0; n < n_tiles; ++n) {
        const int s = n % S, bb = n & 1;
        if (FP8) {
          if (!mbar_wait(&k16_full[bb], (n >> 1) & 1)) break;
        } else if (!mbar_wait(&kv_full[s], (n / S) & 1)) {
          break;
        }
        if (n >= 2 && !mbar_wait(&s_empty[bb], ((n - 2) >> 1) & 1)) break;
        tc_fence_after();
        tc_issue_qk<N, FP8>(tmem + bb * N,
                            FP8 ? smem_u32(smem + SM::kSK16Off + bb * kTcTileBytes)
                                : smem_u32(smem + s * SM::kSStageBytes),
                            q_addr);
        tc_commit(&s_full[bb]);
        tc_commit(FP8 ? &k16_free[bb] : &kv_empty[s]);
      }
    }
  } else if (FP8 && warp >= 10) {
    // ---- E4M3 -> f16 converters: warp 10 + i converts key rows 32i .. 32i+31
    const int i = warp - 10;
    for (int n = 0; n < n_tiles; ++n) {
      const int s = n % S, bb = n & 1;
      if (!mbar_wait(&kv_full[s], (n / S) & 1)) break;
      if (n >= 2 && !mbar_wait(&k16_free[bb], ((n - 2) >> 1) & 1)) break;
      fp8_rows_to_f16(smem + s * SM::kSStageBytes, 32 * i, 32, lane, 32,
                      smem + SM::kSK16Off + bb * kTcTileBytes);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&kv_empty[s]);
        mbar_arrive(&k16_full[bb]);
      }
    }
  } else {
    // ---- score warps: stage Q (for the tensor cores), the group's (m, l)
    //      partials, clear the histograms; then lse (base 2) of the group's rows
    constexpr int kSc = 256;  // score threads
    const int st = threadIdx.x - 64;
    if (n_tiles > 0) {
      tc_stage_q<N, FP8>(p, b, t0, smem + SM::kSQOff, st, kSc);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    if (!p.lse_in) {
      const float2* ml_g = p.part_ml + (long long)grp * ns * N;
      for (int u = st; u < N * ns; u += kSc) {
        const int sp = u / N, r = u % N;
        ml_s[r * ns + sp] = ml_g[(long long)sp * N + r];
      }
    }
    for (int u = st; u < G * kHistBins; u += kSc) hist_s[u] = 0u;
    softmax_sync<kSc>();
    for (int r = st; r < N; r += kSc) {
      if (p.lse_in) {  // the normaliser over the whole context (context-parallel slice)
        const int t = t0 + r / kH;
        lse2_s[r] = t < p.T ? p.lse_in[((long long)b * p.T + t) * p.H + r % kH] * kLog2e : 0.f;
        continue;
      }
      float M = kNegInf;
      for (int sp = 0; sp < ns; ++sp) M = fmaxf(M, ml_s[r * ns + sp].x);
      float lt = 0.f;
      if (M != kNegInf)
        for (int sp = 0; sp < ns; ++sp) {
          const float2 v = ml_s[r * ns + sp];
          lt += v.x == kNegInf ? 0.f : v.y * fast_exp2(v.x - M);
        }
      lse2_s[r] = M + log2f(lt);
    }
    softmax_sync<kSc>();
    const int wq = warp & 3;
    const int half = (warp - 2) >> 2;  // this group's tiles: half, half + 2, ...
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const int keyrow = wq * 32 + lane;
    auto load_ks = [&](int n) {
      const long long jn = k_lo + (long long)n * kTcKeys + keyrow;
      return (FP8 && n < n_tiles && jn < k_hi) ? p.k_scale[(long long)b * p.L + jn] : 0.f;
    };
    float ks_next = load_ks(half);  // E4M3: one tile ahead of its use
    for (int n = half; n < n_tiles; n += 2) {
      const int bb = n & 1;
      const long long j = k_lo + (long long)n * kTcKeys + keyrow;
      float sl = p.scale_log2;
      if (FP8) {
        sl *= ks_next;
        ks_next = load_ks(n + 2);
      }
      if (!mbar_wait(&s_full[bb], (n >> 1) & 1)) break;
      tc_fence_after();
      float acc[G];
#pragma unroll
      for (int q = 0; q < G; ++q) acc[q] = 0.f;
#pragma unroll
      for (int c = 0; c < N / 32; ++c) {
        float x[32];
        tmem_ld32(tmem + lane_base + bb * N + 32 * c, x);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          acc[(32 * c + i) / kH] += fast_exp2(x[i] * sl - lse2_s[32 * c + i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[bb]);
#pragma unroll
      for (int q = 0; q < G; ++q) {
        const int t = t0 + q;
        // a candidate lies inside this split (and the cache: a context-parallel
        // slice may end before the query's candidates do)
        const bool cand = t < p.T && j < k_hi && j <= p.qpos0 + t - p.window;
        if (cand) p.score[((long long)b * p.T + t) * p.L + j] = acc[q];
        hist_inc(hist_s + q * kHistBins, __float_as_uint(acc[q]) >> kHistShift, cand);
      }
    }
    softmax_sync<kSc>();
    for (int u = st; u < G * kHistBins; u += kSc) {
      const unsigned cnt = hist_s[u];
      const int t = t0 + u / kHistBins;
      if (cnt && t < p.T) atomicAdd(&p.hist[((long long)b * p.T + t) * kHistBins + (u % kHistBins)], cnt);
    }
    // ---- O and lse of row r, merged by the CTA whose score-split index is r mod
    //      score_splits: each group takes every other such row, its thread d
    //      element d (not with a given normaliser: O and lse were produced by
    //      the slice's first pass)
    const int d = st & 127;
    for (int r = split + half * p.score_splits; r < N && !p.lse_in; r += 2 * p.score_splits) {
      const int t = t0 + r / kH;
      if (t >= p.T) continue;
      const float l2 = lse2_s[r];
      const long long li = ((long long)b * p.T + t) * p.H + r % kH;
      if (d == 0) {
        p.lse[li] = l2 * 0.69314718055994531f;
        if (p.lse_out) p.lse_out[li] = l2 * 0.69314718055994531f;
      }
      const float* po = p.part_o + ((long long)grp * ns * N + r) * 128 + d;
      float acc = 0.f;
#pragma unroll 8
      for (int sp = 0; sp < ns; ++sp) {
        const float2 v = ml_s[r * ns + sp];
        const float f = (v.x == kNegInf) ? 0.f : fast_exp2(v.x - l2);
        acc += f * po[(long long)sp * N * 128];
      }
      p.o[li * 128 + d] = acc;
    }
  }
  __syncthreads();
  if (warp == 1 && n_tiles > 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * N);
  }
}

}  // namespace hs2
