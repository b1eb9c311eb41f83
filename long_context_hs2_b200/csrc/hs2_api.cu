// libhs2: C ABI of the hybrid-block hot path (see include/hs2.h).
// One translation unit: every kernel header is included here.

#include <hs2.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "bridge_gemm.cuh"
#include "bridge_small.cuh"
#include "cp.cuh"
#include "full_attn.cuh"
#include "attn_tc.cuh"
#include "select.cuh"
#include "select_block.cuh"
#include "sparse_attn.cuh"

using namespace hs2;

namespace {

// ------------------------------------------------------------ TMA encode --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;  // resolved once; every thread resolves the same address
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D row-major tensor [rows][cols] of `elem`-byte elements, tile box
// {box_cols, box_rows}, 128-byte swizzle.
bool make_map_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, int elem,
                 uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const CUtensorMapDataType dt =
      elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)elem};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
bool aligned4(const void* p) { return ((uintptr_t)p & 3u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// ------------------------------------------- optional stage timing --
thread_local cudaEvent_t t_stage_begin = nullptr, t_stage_end = nullptr;

// ------------------------------------------------- fault injection --
constexpr unsigned long long kDefaultWaitLimitNs = 1000000000ull;
thread_local unsigned long long* t_phase_stamps = nullptr;
thread_local int t_phase_ctas = 0;
thread_local unsigned t_barrier_extra = 0;
thread_local unsigned long long t_wait_limit_ns = kDefaultWaitLimitNs;

// Records the caller's stage event (if any) on s; an external event node when
// s is being captured into a graph.
cudaError_t stage_mark(cudaStream_t s, bool begin) {
  cudaEvent_t ev = begin ? t_stage_begin : t_stage_end;
  if (!ev) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return cudaErrorUnknown;
  return cs == cudaStreamCaptureStatusActive
             ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
             : cudaEventRecord(ev, s);
}

// ------------------------------------------------ full-attention plan --
struct FullPlan {
  bool tc;       // tcgen05 path (D = 128)
  bool fused;    // one fused tcgen05 kernel (partials, score and selection) for N = 32
  int rows;      // query rows per group (N of the tcgen05 tiles, or 32)
  int tile;      // keys per pipeline tile
  int G, groups_per_seq, n_groups, n_splits, split_keys, score_splits, score_keys;
  size_t off_part_o, off_part_ml, off_lse, off_hist, off_score, off_sync, off_list, off_cnt,
      total;
};

bool check_attn_shape(int B, int T, int64_t L, int H, int D, hs2_kv_dtype dt) {
  if (B < 1 || T < 1 || L < T || L > INT32_MAX || (int64_t)B * L > INT32_MAX) return false;
  if (!(H == 8 || H == 16 || H == 32)) return false;
  if (!(D == 64 || D == 128)) return false;
  if (dt != HS2_KV_BF16 && dt != HS2_KV_FP8_E4M3) return false;
  return true;
}

// Host-side checks of hs2_full_attn_select's arguments, before any workspace
// or device state is looked at.
hs2_status check_full_args(const void* Q, const hs2_kv_cache* kv, int B, int T, int64_t L, int H,
                           int D, float scale, int topk, int window, hs2_kv_dtype dt,
                           const float* O, const float* lse, const int32_t* idx,
                           const int32_t* n_sel) {
  if (!Q || !kv || !kv->k || !kv->v || !O || !idx || !n_sel) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(kv->k) || !aligned16(kv->v) || !aligned16(O) ||
      !aligned4(idx) || !aligned4(n_sel) || (lse && !aligned4(lse)))
    return HS2_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || L < T || topk < 0 || window < 1 || !std::isfinite(scale))
    return HS2_ERR_INVALID_ARG;
  if (dt == HS2_KV_FP8_E4M3 && (!kv->k_scale || !kv->v_scale || !aligned4(kv->k_scale) ||
                                !aligned4(kv->v_scale)))
    return HS2_ERR_INVALID_ARG;
  if (!check_attn_shape(B, T, L, H, D, dt) || topk + window > 4096) return HS2_ERR_UNSUPPORTED;
  if (dt == HS2_KV_FP8_E4M3 && D != 128) return HS2_ERR_UNSUPPORTED;
  return HS2_OK;
}

bool make_full_plan(int B, int T, int64_t L, int H, int D, hs2_kv_dtype dt, FullPlan* pl,
                    bool allow_fused = true) {
  pl->tc = D == 128;
  pl->rows = pl->tc && H == 32 && T >= 4 ? 128 : 32;
  pl->fused = allow_fused && pl->tc && pl->rows == 32;
  pl->tile = pl->tc ? kTcKeys : kTile;
  pl->G = pl->rows / H;
  pl->groups_per_seq = (T + pl->G - 1) / pl->G;
  pl->n_groups = B * pl->groups_per_seq;
  const int64_t tiles = (L + pl->tile - 1) / pl->tile;
  // `target` CTAs over the groups, rounded down so that a one-wave grid stays one wave
  auto split = [&](int64_t target, int64_t max_splits, int* n_out, int* keys_out) {
    int64_t sp = target / pl->n_groups;
    sp = std::max<int64_t>(1, std::min<int64_t>(std::min<int64_t>(sp, tiles), max_splits));
    int64_t per = (L + sp - 1) / sp;
    per = (per + pl->tile - 1) / pl->tile * pl->tile;
    *n_out = (int)((L + per - 1) / per);
    *keys_out = (int)per;
  };
  // partials: about one wave of CTAs (each merged later); score pass: more
  // (the tcgen05 score kernel stages the group's (m, l) partials in 32 KB of
  //  shared memory: rows x splits x 8 bytes)
  split(sm_count(), pl->tc ? (32 << 10) / (8 * pl->rows) : tiles, &pl->n_splits,
        &pl->split_keys);
  split((pl->tc ? 1LL : 4LL) * sm_count(), tiles, &pl->score_splits, &pl->score_keys);
  const int R = pl->rows;
  size_t off = 0;
  pl->off_part_o = off;
  off = align_up(off + (size_t)pl->n_groups * pl->n_splits * R * D * 4, 256);
  pl->off_part_ml = off;
  off = align_up(off + (size_t)pl->n_groups * pl->n_splits * R * 8, 256);
  pl->off_lse = off;
  off = align_up(off + (size_t)B * T * H * 4, 256);
  pl->off_hist = off;
  off = align_up(off + (size_t)B * T * kHistBins * 4, 256);
  pl->off_score = off;
  off = align_up(off + (size_t)B * T * (size_t)L * 4, 256);
  pl->off_sync = pl->off_list = pl->off_cnt = off;
  if (pl->fused) {
    off = align_up(off + (size_t)pl->n_groups * 8 * 4, 256);
    pl->off_list = off;
    off = align_up(off + (size_t)B * T * pl->n_splits * pl->split_keys * 4, 256);
    pl->off_cnt = off;
    off = align_up(off + (size_t)B * T * pl->n_splits * 8, 256);
  }
  pl->total = off;
  return true;
}

// Launches `kernel` on stream s, as clusters of `cluster` CTAs along x when
// cluster > 1, and as a cooperative grid (all CTAs co-resident, or the launch
// fails) when coop.
template <typename... KArgs, typename... Args>
hs2_status launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     int cluster, bool coop, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[3];
  int na = 0;
  if (cluster > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)cluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (coop) {
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na].val.cooperative = 1;
    ++na;
  }
  if (pdl) {  // may start before the previous kernel ends; the kernel waits on it itself
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return HS2_ERR_CUDA;
  }
  return HS2_OK;
}

template <typename... KArgs, typename... Args>
hs2_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                  int cluster, Args&&... args) {
  return launch_ex(kernel, grid, block, smem, s, cluster, false, false,
                   std::forward<Args>(args)...);
}

template <typename K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
         cudaSuccess;
}

hs2_status run_select(const FullAttnParams& fp, SelectParams sp, cudaStream_t s) {
  // few queries: split each query's candidates over a cluster of up to 8 CTAs
  const long long rows = (long long)fp.B * fp.T;
  const int sms = sm_count();
  int cs = 1;
  while (cs < 8 && rows * cs * 2 <= sms) cs *= 2;
  sp.cs = cs;
  // the most candidates of any row (a context-parallel slice holds at most L)
  const long long nc_max =
      sp.cp ? std::max<long long>(1, std::min<long long>(fp.L, sp.qpos0 + fp.T - fp.window))
            : std::max<long long>(1, fp.L - fp.window + 1);
  const long long seg = ((nc_max + cs - 1) / cs + 3) / 4 * 4;
  const bool smem = seg <= kSelSmemMax;
  const int bytes = smem ? (int)std::max<long long>(16, seg * 4) : 0;
  auto k = smem ? select_topk_kernel<true> : select_topk_kernel<false>;
  if (!set_smem(k, std::max(bytes, 16))) return HS2_ERR_CUDA;
  return launch(k, dim3((unsigned)(rows * cs)), dim3(kSelThreads), (size_t)bytes, s, cs, sp);
}

template <int D, bool FP8>
hs2_status run_full(const CUtensorMap& km, const CUtensorMap& vm, const FullAttnParams& fp,
                    const FullPlan& pl, cudaStream_t s) {
  using SM = FullAttnSmem<D, FP8>;
  auto kp = attn_partial_kernel<D, FP8>;
  auto ks = fp.G == 1 ? attn_score_kernel<D, FP8, 1>
                      : (fp.G == 2 ? attn_score_kernel<D, FP8, 2> : attn_score_kernel<D, FP8, 4>);
  if (!set_smem(kp, SM::kBytes) || !set_smem(ks, SM::kScoreBytes)) return HS2_ERR_CUDA;
  if (stage_mark(s, true) != cudaSuccess) return HS2_ERR_CUDA;
  hs2_status st = launch(kp, dim3(pl.n_groups * pl.n_splits), dim3(160), SM::kBytes, s, 1, km,
                         vm, fp);
  if (st != HS2_OK) return st;
  if (stage_mark(s, false) != cudaSuccess) return HS2_ERR_CUDA;
  return launch(ks, dim3(pl.n_groups * pl.score_splits), dim3(160), SM::kScoreBytes, s, 1, km, fp);
}

template <int N, bool FP8>
hs2_status run_full_tc(const CUtensorMap& km, const CUtensorMap& vm, const FullAttnParams& fp,
                       const FullPlan& pl, cudaStream_t s) {
  using SM = TcSmem<N, FP8>;
  static_assert(SM::kBytes <= 232448 && SM::kSBytes <= 232448, "shared memory per CTA");
  auto kp = N == 128 ? attn_tc_partial_kernel<N, 4, FP8>
                     : (fp.G == 1 ? attn_tc_partial_kernel<N, 1, FP8>
                                  : (fp.G == 2 ? attn_tc_partial_kernel<N, 2, FP8>
                                               : attn_tc_partial_kernel<N, 4, FP8>));
  auto ks = N == 128 ? attn_tc_score_kernel<N, 4, FP8>
                     : (fp.G == 1 ? attn_tc_score_kernel<N, 1, FP8>
                                  : (fp.G == 2 ? attn_tc_score_kernel<N, 2, FP8>
                                               : attn_tc_score_kernel<N, 4, FP8>));
  if (!set_smem(kp, SM::kBytes) || !set_smem(ks, SM::kSBytes)) return HS2_ERR_CUDA;
  if (stage_mark(s, true) != cudaSuccess) return HS2_ERR_CUDA;
  const hs2_status st = launch(kp, dim3(pl.n_groups * pl.n_splits),
                               dim3(tc_partial_threads(FP8)), SM::kBytes, s, 1, km, vm, fp);
  if (st != HS2_OK) return st;
  if (stage_mark(s, false) != cudaSuccess) return HS2_ERR_CUDA;
  return launch(ks, dim3(pl.n_groups * pl.score_splits), dim3(tc_score_threads(FP8)), SM::kSBytes,
                s, 1, km, fp);
}

// The score kernel alone (a context-parallel slice's second pass: the
// normaliser comes from fp.lse_in).
template <int N, bool FP8>
hs2_status run_score_tc(const CUtensorMap& km, const FullAttnParams& fp, const FullPlan& pl,
                        cudaStream_t s) {
  using SM = TcSmem<N, FP8>;
  auto ks = N == 128 ? attn_tc_score_kernel<N, 4, FP8>
                     : (fp.G == 1 ? attn_tc_score_kernel<N, 1, FP8>
                                  : (fp.G == 2 ? attn_tc_score_kernel<N, 2, FP8>
                                               : attn_tc_score_kernel<N, 4, FP8>));
  if (!set_smem(ks, SM::kSBytes)) return HS2_ERR_CUDA;
  return launch(ks, dim3(pl.n_groups * pl.score_splits), dim3(tc_score_threads(FP8)), SM::kSBytes,
                s, 1, km, fp);
}

// The fused tcgen05 pass (N = 32): arrival counters cleared, then one
// cooperative launch (the CTAs of a group wait for one another); the
// selection runs inside it when a row's candidates fit its shared memory,
// else as the selection kernel after it.
template <bool FP8>
hs2_status run_fused_tc(const CUtensorMap& km, const CUtensorMap& vm, FullAttnParams fp,
                        const FullPlan& pl, const SelectParams& sp, bool token_select,
                        cudaStream_t s) {
  using SM = TcSmem<32, FP8>;
  static_assert(SM::kBytes <= 232448, "shared memory per CTA");
  // the selection is fused when a split's candidate scores of the group's
  // rows fit the P^T buffers (shared memory free after the partial pass);
  // without token_select the caller runs another selection on the scores
  fp.fuse_select = token_select && (long long)fp.G * fp.split_keys * 4 <= SM::kNP * SM::kPBytes &&
                   pl.n_splits <= 256;
  // the logits of every tile stay in TMEM for the score pass when a split has
  // at most kTcRetainTiles tiles
  const bool retain = (fp.split_keys + kTcKeys - 1) / kTcKeys <= kTcRetainTiles;
  auto kf = retain ? (fp.G == 1 ? attn_tc_fused_kernel<32, 1, FP8, true>
                                : (fp.G == 2 ? attn_tc_fused_kernel<32, 2, FP8, true>
                                             : attn_tc_fused_kernel<32, 4, FP8, true>))
                   : (fp.G == 1 ? attn_tc_fused_kernel<32, 1, FP8, false>
                                : (fp.G == 2 ? attn_tc_fused_kernel<32, 2, FP8, false>
                                             : attn_tc_fused_kernel<32, 4, FP8, false>));
  if (!set_smem(kf, SM::kBytes)) return HS2_ERR_CUDA;
  if (cudaMemsetAsync(fp.grp_sync, 0, (size_t)pl.n_groups * 8 * 4, s) != cudaSuccess) {
    cudaGetLastError();
    return HS2_ERR_CUDA;
  }
  if (stage_mark(s, true) != cudaSuccess) return HS2_ERR_CUDA;
  const hs2_status st = launch_ex(kf, dim3(pl.n_groups * pl.n_splits), dim3(tc_partial_threads(FP8)),
                                  SM::kBytes, s, 1, pl.n_splits > 1, false, km, vm, fp);
  if (st != HS2_OK) return st;
  if (stage_mark(s, false) != cudaSuccess) return HS2_ERR_CUDA;
  return (fp.fuse_select || !token_select) ? HS2_OK : run_select(fp, sp, s);
}

// Block-level selection from the score rows the attention pass wrote.
hs2_status run_select_blocks(const FullAttnParams& fp, int topk, int window, int block,
                             int32_t* idx, int32_t* n_sel, cudaStream_t s) {
  BlockSelectParams bp;
  bp.score = fp.score;
  bp.idx = idx;
  bp.n_sel = n_sel;
  bp.T = fp.T;
  bp.L = fp.L;
  bp.topk = topk;
  bp.window = window;
  bp.slots = topk + window;
  bp.block = block;
  bp.block_shift = (block & (block - 1)) == 0 ? __builtin_ctz((unsigned)block) : -1;
  bp.qpos0 = fp.qpos0;
  const long long nblk_max = std::max<long long>(1, (fp.L - window) / block + 1);
  const size_t bytes = (size_t)(nblk_max + topk / block) * 4;
  if (!set_smem(select_blocks_kernel, (int)bytes)) return HS2_ERR_CUDA;
  return launch(select_blocks_kernel, dim3((unsigned)((long long)fp.B * fp.T)), dim3(kBlkThreads),
                bytes, s, 1, bp);
}

// Shared memory of a sparse launch: the position array holds one CTA's share
// of the slots in whole tiles, plus n_sel.
template <int MT, int D, bool FP8>
size_t sparse_smem_bytes(int slots, int cs) {
  const int tiles_max = (sparse_share(slots, cs) + kSpTile - 1) / kSpTile;
  return (size_t)SparseSmem<MT, D, FP8>::kPosOff + (size_t)(tiles_max * kSpTile + 4) * 4 + 1024;
}

// p.cs is the power-of-two cluster size chosen by the caller.  When the
// slots of a query fill ceil(slots / tile) CTAs of one tile each and clusters
// of that size (up to 16, a non-portable size) are co-resident for every
// query at once, that size is used instead: each CTA then has a single tile.
template <int MT, int D, bool FP8>
hs2_status run_sparse(SparseParams p, cudaStream_t s) {
  using SM = SparseSmem<MT, D, FP8>;
  auto k = sparse_attn_kernel<MT, D, FP8>;
  if (!set_smem(k, SM::kBytes)) return HS2_ERR_CUDA;
  const long long queries = (long long)p.B * p.T;
  const int want = (p.slots + kSpTile - 1) / kSpTile;
  // co-resident clusters of `want` CTAs, per device and slot count (queried once)
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> resident;
  int dev = 0;
  cudaGetDevice(&dev);
  int n_res = -1;
  if (want > p.cs && want <= 16 && queries * want <= sm_count()) {
    std::lock_guard<std::mutex> lock(mu);
    auto it = resident.find({dev, p.slots});
    if (it != resident.end()) n_res = it->second;
  }
  if (n_res < 0 && want > p.cs && want <= 16 && queries * want <= sm_count()) {
    n_res = 0;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(queries * want));
      cfg.blockDim = dim3(kSpThreads);
      cfg.dynamicSmemBytes = sparse_smem_bytes<MT, D, FP8>(p.slots, want);
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = (unsigned)want;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int n_clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&n_clusters, k, &cfg) == cudaSuccess) n_res = n_clusters;
    }
    cudaGetLastError();
    std::lock_guard<std::mutex> lock(mu);
    resident[{dev, p.slots}] = n_res;
  }
  if (n_res >= queries) p.cs = want;
  const size_t bytes = sparse_smem_bytes<MT, D, FP8>(p.slots, p.cs);
  return launch_ex(k, dim3((unsigned)(queries * p.cs)), dim3(kSpThreads), bytes, s, p.cs, false,
                   true, p);
}

}  // namespace

extern "C" {

int hs2_version(void) { return 101; }

hs2_status hs2_set_fault_injection(unsigned extra_arrivals, unsigned long long wait_limit_ns) {
  t_barrier_extra = extra_arrivals;
  t_wait_limit_ns = wait_limit_ns ? wait_limit_ns : kDefaultWaitLimitNs;
  return HS2_OK;
}

static_assert(HS2_PHASES == hs2::kPhases, "phase stamps per CTA");

hs2_status hs2_set_phase_stamps(unsigned long long* stamps, int max_ctas) {
  if (stamps && (max_ctas < 1 || ((uintptr_t)stamps & 7u) != 0)) return HS2_ERR_INVALID_ARG;
  t_phase_stamps = stamps;
  t_phase_ctas = stamps ? max_ctas : 0;
  return HS2_OK;
}

hs2_status hs2_set_stage_events(void* begin_event, void* end_event) {
  if ((begin_event == nullptr) != (end_event == nullptr)) return HS2_ERR_INVALID_ARG;
  t_stage_begin = static_cast<cudaEvent_t>(begin_event);
  t_stage_end = static_cast<cudaEvent_t>(end_event);
  return HS2_OK;
}

const char* hs2_status_string(hs2_status st) {
  switch (st) {
    case HS2_OK: return "ok";
    case HS2_ERR_INVALID_ARG: return "invalid argument";
    case HS2_ERR_UNSUPPORTED: return "unsupported shape or type";
    case HS2_ERR_CUDA: return "CUDA error";
    case HS2_ERR_WORKSPACE: return "workspace missing or too small";
    case HS2_ERR_TIMEOUT: return "a kernel timed out waiting on a barrier";
    case HS2_ERR_DEVICE: return "a kernel met an out-of-range index";
  }
  return "unknown status";
}

hs2_status hs2_last_device_status(hs2_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return HS2_ERR_CUDA;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return HS2_ERR_CUDA;
  if (v && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return HS2_ERR_CUDA;
  if (v & kStatusTimeout) return HS2_ERR_TIMEOUT;
  if (v & kStatusBadIndex) return HS2_ERR_DEVICE;
  return HS2_OK;
}

size_t hs2_full_attn_select_workspace(int B, int T, int64_t L, int H, int D, int topk,
                                      int window, hs2_kv_dtype dt) {
  if (!check_attn_shape(B, T, L, H, D, dt) || topk < 0 || window < 1 || topk + window > 4096)
    return 0;
  FullPlan pl;
  make_full_plan(B, T, L, H, D, dt, &pl);
  return pl.total;
}

}  // extern "C"

namespace {

// Plan, tensor maps and kernel parameters of a full-attention call over a
// cache of L positions (allow_fused: the fused decode kernel may be planned).
hs2_status setup_full(const void* Q, const hs2_kv_cache* kv, int B, int T, int64_t L, int H, int D,
                      float scale, int topk, int window, hs2_kv_dtype dt, float* O, float* lse,
                      int32_t* idx, int32_t* n_sel, void* workspace, size_t workspace_bytes,
                      bool allow_fused, FullPlan& pl, CUtensorMap& km, CUtensorMap& vm,
                      FullAttnParams& fp, SelectParams& sp) {
  make_full_plan(B, T, L, H, D, dt, &pl, allow_fused);
  if (!workspace || workspace_bytes < pl.total || !aligned16(workspace)) return HS2_ERR_WORKSPACE;

  const bool fp8 = dt == HS2_KV_FP8_E4M3;
  const int elem = fp8 ? 1 : 2;
  const uint32_t box_cols = fp8 ? 128u : 64u;
  if (!make_map_2d(&km, kv->k, (uint64_t)B * L, D, elem, box_cols, pl.tile) ||
      !make_map_2d(&vm, kv->v, (uint64_t)B * L, D, elem, box_cols, pl.tile))
    return HS2_ERR_CUDA;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  fp.q = static_cast<const __nv_bfloat16*>(Q);
  fp.k_scale = fp8 ? kv->k_scale : nullptr;
  fp.v_scale = fp8 ? kv->v_scale : nullptr;
  fp.part_o = reinterpret_cast<float*>(ws + pl.off_part_o);
  fp.part_ml = reinterpret_cast<float2*>(ws + pl.off_part_ml);
  fp.lse = reinterpret_cast<float*>(ws + pl.off_lse);
  fp.lse_out = lse;
  fp.o = O;
  fp.score = reinterpret_cast<float*>(ws + pl.off_score);
  fp.hist = reinterpret_cast<unsigned*>(ws + pl.off_hist);
  fp.B = B;
  fp.T = T;
  fp.H = H;
  fp.D = D;
  fp.L = L;
  fp.G = pl.G;
  fp.groups_per_seq = pl.groups_per_seq;
  fp.n_splits = pl.n_splits;
  fp.split_keys = pl.split_keys;
  fp.score_splits = pl.score_splits;
  fp.score_keys = pl.score_keys;
  fp.window = window;
  fp.scale_log2 = scale * kLog2e;

  sp.score = fp.score;
  sp.hist = fp.hist;
  sp.idx = idx;
  sp.n_sel = n_sel;
  sp.T = T;
  sp.L = L;
  sp.topk = topk;
  sp.window = window;
  sp.slots = topk + window;
  sp.cs = 1;

  fp.grp_sync = reinterpret_cast<unsigned*>(ws + pl.off_sync);
  fp.sel_list = reinterpret_cast<unsigned*>(ws + pl.off_list);
  fp.sel_cnt = reinterpret_cast<int2*>(ws + pl.off_cnt);
  fp.idx = idx;
  fp.n_sel = n_sel;
  fp.topk = topk;
  fp.slots = topk + window;
  fp.fuse_select = 0;
  fp.phase_stamps = t_phase_stamps;
  fp.phase_ctas = t_phase_ctas;
  fp.wait_limit_ns = t_wait_limit_ns;
  fp.barrier_extra = t_barrier_extra;
  fp.qpos0 = L - T;
  fp.lse_in = nullptr;
  fp.no_score = 0;
  sp.qpos0 = L - T;
  sp.cp = 0;
  sp.key_off = 0;
  sp.cand_score = nullptr;
  return HS2_OK;
}

// The full-attention pass, then the token-level selection (sel_block == 0) or
// the block-level selection with blocks of sel_block positions.
hs2_status full_attn_select_impl(const void* Q, const hs2_kv_cache* kv, int B, int T, int64_t L,
                                 int H, int D, float scale, int topk, int window, int sel_block,
                                 hs2_kv_dtype dt, float* O, float* lse, int32_t* idx,
                                 int32_t* n_sel, void* workspace, size_t workspace_bytes,
                                 hs2_stream_t stream) {
  const hs2_status chk = check_full_args(Q, kv, B, T, L, H, D, scale, topk, window, dt, O, lse,
                                         idx, n_sel);
  if (chk != HS2_OK) return chk;
  FullPlan pl;
  CUtensorMap km, vm;
  FullAttnParams fp;
  SelectParams sp;
  const hs2_status su = setup_full(Q, kv, B, T, L, H, D, scale, topk, window, dt, O, lse, idx,
                                   n_sel, workspace, workspace_bytes, true, pl, km, vm, fp, sp);
  if (su != HS2_OK) return su;
  const bool fp8 = dt == HS2_KV_FP8_E4M3;

  cudaStream_t s = (cudaStream_t)stream;
  const bool token = sel_block == 0;
  hs2_status st;
  if (pl.fused) {
    st = fp8 ? run_fused_tc<true>(km, vm, fp, pl, sp, token, s)
             : run_fused_tc<false>(km, vm, fp, pl, sp, token, s);
    if (st != HS2_OK || token) return st;
  } else {
    if (pl.tc)
      st = fp8 ? (pl.rows == 128 ? run_full_tc<128, true>(km, vm, fp, pl, s)
                                 : run_full_tc<32, true>(km, vm, fp, pl, s))
               : (pl.rows == 128 ? run_full_tc<128, false>(km, vm, fp, pl, s)
                                 : run_full_tc<32, false>(km, vm, fp, pl, s));
    else  // head_dim 64 (bf16 only): the mma.sync kernels
      st = run_full<64, false>(km, vm, fp, pl, s);
    if (st != HS2_OK) return st;
    if (token) return run_select(fp, sp, s);
  }
  return run_select_blocks(fp, topk, window, sel_block, idx, n_sel, s);
}

}  // namespace

extern "C" {

hs2_status hs2_full_attn_select(const void* Q, const hs2_kv_cache* kv, int B, int T, int64_t L,
                                int H, int D, float scale, int topk, int window,
                                hs2_kv_dtype dt, float* O, float* lse, int32_t* idx,
                                int32_t* n_sel, void* workspace, size_t workspace_bytes,
                                hs2_stream_t stream) {
  return full_attn_select_impl(Q, kv, B, T, L, H, D, scale, topk, window, 0, dt, O, lse, idx,
                               n_sel, workspace, workspace_bytes, stream);
}

hs2_status hs2_full_attn_select_blocks(const void* Q, const hs2_kv_cache* kv, int B, int T,
                                       int64_t L, int H, int D, float scale, int topk,
                                       int window, int block, hs2_kv_dtype dt, float* O,
                                       float* lse, int32_t* idx, int32_t* n_sel,
                                       void* workspace, size_t workspace_bytes,
                                       hs2_stream_t stream) {
  if (block < 1 || topk < 0 || topk % block != 0) return HS2_ERR_INVALID_ARG;
  const hs2_status chk = check_full_args(Q, kv, B, T, L, H, D, scale, topk, window, dt, O, lse,
                                         idx, n_sel);
  if (chk != HS2_OK) return chk;
  if ((L - window) / block + 1 > kBlkMaxBlocks) return HS2_ERR_UNSUPPORTED;
  return full_attn_select_impl(Q, kv, B, T, L, H, D, scale, topk, window, block, dt, O, lse, idx,
                               n_sel, workspace, workspace_bytes, stream);
}

// ------------------------------------------------ context parallelism --
size_t hs2_cp_workspace(int B, int T, int64_t L_local, int H, int D, int topk, int window,
                        hs2_kv_dtype dt) {
  if (!check_attn_shape(B, 1, L_local, H, D, dt) || T < 1 || D != 128 || topk < 0 ||
      window < 1 || topk + window > 4096)
    return 0;
  FullPlan pl;
  make_full_plan(B, T, L_local, H, D, dt, &pl, false);
  return pl.total;
}

// Shared checks of the two per-slice calls; T may exceed L_local (a slice can
// be shorter than the chunk of queries).
static hs2_status check_cp_slice(const void* Q, const hs2_kv_cache* kv, int B, int T,
                                 int64_t L_local, int64_t q_pos_local, int H, int D, float scale,
                                 hs2_kv_dtype dt) {
  if (!Q || !kv || !kv->k || !kv->v || !aligned16(Q) || !aligned16(kv->k) || !aligned16(kv->v))
    return HS2_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || L_local < 1 || !std::isfinite(scale)) return HS2_ERR_INVALID_ARG;
  if (q_pos_local < -(int64_t)T || q_pos_local > ((int64_t)1 << 40)) return HS2_ERR_INVALID_ARG;
  if (dt == HS2_KV_FP8_E4M3 && (!kv->k_scale || !kv->v_scale || !aligned4(kv->k_scale) ||
                                !aligned4(kv->v_scale)))
    return HS2_ERR_INVALID_ARG;
  if (!check_attn_shape(B, 1, L_local, H, D, dt) || D != 128) return HS2_ERR_UNSUPPORTED;
  return HS2_OK;
}

hs2_status hs2_cp_attn_partial(const void* Q, const hs2_kv_cache* kv, int B, int T,
                               int64_t L_local, int64_t q_pos_local, int H, int D, float scale,
                               hs2_kv_dtype dt, float* O, float* lse, void* workspace,
                               size_t workspace_bytes, hs2_stream_t stream) {
  hs2_status st = check_cp_slice(Q, kv, B, T, L_local, q_pos_local, H, D, scale, dt);
  if (st != HS2_OK) return st;
  if (!O || !lse || !aligned16(O) || !aligned4(lse)) return HS2_ERR_INVALID_ARG;
  FullPlan pl;
  CUtensorMap km, vm;
  FullAttnParams fp;
  SelectParams sp;
  st = setup_full(Q, kv, B, T, L_local, H, D, scale, 0, 1, dt, O, lse, nullptr, nullptr,
                  workspace, workspace_bytes, false, pl, km, vm, fp, sp);
  if (st != HS2_OK) return st;
  fp.qpos0 = q_pos_local;
  fp.no_score = 1;
  const bool fp8 = dt == HS2_KV_FP8_E4M3;
  cudaStream_t s = (cudaStream_t)stream;
  return fp8 ? (pl.rows == 128 ? run_full_tc<128, true>(km, vm, fp, pl, s)
                               : run_full_tc<32, true>(km, vm, fp, pl, s))
             : (pl.rows == 128 ? run_full_tc<128, false>(km, vm, fp, pl, s)
                               : run_full_tc<32, false>(km, vm, fp, pl, s));
}

hs2_status hs2_cp_select_local(const void* Q, const hs2_kv_cache* kv, int B, int T,
                               int64_t L_local, int64_t q_pos_local, int64_t key_pos0, int H,
                               int D, float scale, int topk, int window, hs2_kv_dtype dt,
                               const float* lse, float* cand_score, int32_t* cand_idx,
                               void* workspace, size_t workspace_bytes, hs2_stream_t stream) {
  hs2_status st = check_cp_slice(Q, kv, B, T, L_local, q_pos_local, H, D, scale, dt);
  if (st != HS2_OK) return st;
  if (!lse || !cand_score || !cand_idx || !aligned4(lse) || !aligned4(cand_score) ||
      !aligned4(cand_idx) || topk < 1 || window < 1 || topk + window > 4096 || key_pos0 < 0 ||
      key_pos0 + L_local > INT32_MAX)
    return HS2_ERR_INVALID_ARG;
  FullPlan pl;
  CUtensorMap km, vm;
  FullAttnParams fp;
  SelectParams sp;
  st = setup_full(Q, kv, B, T, L_local, H, D, scale, topk, window, dt, nullptr, nullptr, cand_idx,
                  nullptr, workspace, workspace_bytes, false, pl, km, vm, fp, sp);
  if (st != HS2_OK) return st;
  fp.qpos0 = q_pos_local;
  fp.lse_in = lse;
  sp.qpos0 = q_pos_local;
  sp.cp = 1;
  sp.key_off = key_pos0;
  sp.cand_score = cand_score;
  sp.slots = topk;
  const bool fp8 = dt == HS2_KV_FP8_E4M3;
  cudaStream_t s = (cudaStream_t)stream;
  // the level-1 selection histograms are cleared by the partial pass, which
  // this call does not run
  if (cudaMemsetAsync(fp.hist, 0, (size_t)B * T * kHistBins * 4, s) != cudaSuccess) {
    cudaGetLastError();
    return HS2_ERR_CUDA;
  }
  st = fp8 ? (pl.rows == 128 ? run_score_tc<128, true>(km, fp, pl, s)
                             : run_score_tc<32, true>(km, fp, pl, s))
           : (pl.rows == 128 ? run_score_tc<128, false>(km, fp, pl, s)
                             : run_score_tc<32, false>(km, fp, pl, s));
  if (st != HS2_OK) return st;
  return run_select(fp, sp, s);
}

hs2_status hs2_cp_lse_combine(const float* lse_parts, int G, int64_t n, float* lse,
                              hs2_stream_t stream) {
  if (!lse_parts || !lse || G < 1 || n < 1) return HS2_ERR_INVALID_ARG;
  const int grid = (int)std::min<int64_t>((n + 255) / 256, 4 * sm_count());
  return launch(cp_lse_combine_kernel, dim3(grid), dim3(256), 0, (cudaStream_t)stream, 1,
                lse_parts, G, (long long)n, lse);
}

hs2_status hs2_cp_rescale(float* O_part, const float* lse_part, const float* lse, int64_t n,
                          int D, hs2_stream_t stream) {
  if (!O_part || !lse_part || !lse || n < 1 || D < 1) return HS2_ERR_INVALID_ARG;
  const int grid = (int)std::min<int64_t>((n * D + 255) / 256, 8 * sm_count());
  return launch(cp_rescale_kernel, dim3(grid), dim3(256), 0, (cudaStream_t)stream, 1, O_part,
                lse_part, lse, (long long)n, D);
}

hs2_status hs2_cp_merge_select(const float* cand_score, const int32_t* cand_idx, int G, int B,
                               int T, int64_t q_pos0, int topk, int window, int32_t* idx,
                               int32_t* n_sel, hs2_stream_t stream) {
  if (!cand_score || !cand_idx || !idx || !n_sel || G < 1 || B < 1 || T < 1 || topk < 1 ||
      window < 1 || topk + window > 4096 || q_pos0 < 0 || q_pos0 + T > INT32_MAX)
    return HS2_ERR_INVALID_ARG;
  if ((int64_t)G * topk * 4 > 200 * 1024) return HS2_ERR_UNSUPPORTED;
  CpMergeParams p;
  p.cand_score = cand_score;
  p.cand_idx = cand_idx;
  p.idx = idx;
  p.n_sel = n_sel;
  p.rows = (long long)B * T;
  p.G = G;
  p.T = T;
  p.topk = topk;
  p.window = window;
  p.qpos0 = q_pos0;
  const int bytes = G * topk * 4;
  if (!set_smem(cp_merge_select_kernel, bytes)) return HS2_ERR_CUDA;
  return launch(cp_merge_select_kernel, dim3((unsigned)p.rows), dim3(kCpThreads), (size_t)bytes,
                (cudaStream_t)stream, 1, p);
}

hs2_status hs2_sparse_attn(const void* Q, const hs2_kv_cache* kv, int B, int T, int64_t L, int H,
                           int D, float scale, const int32_t* idx, const int32_t* n_sel,
                           int slots, hs2_kv_dtype dt, float* O, hs2_stream_t stream) {
  if (!Q || !kv || !kv->k || !kv->v || !idx || !n_sel || !O) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(kv->k) || !aligned16(kv->v) || !aligned16(O) ||
      !aligned4(idx) || !aligned4(n_sel))
    return HS2_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || L < T || slots < 1 || !std::isfinite(scale)) return HS2_ERR_INVALID_ARG;
  if (dt == HS2_KV_FP8_E4M3 && (!kv->k_scale || !kv->v_scale || !aligned4(kv->k_scale) ||
                                !aligned4(kv->v_scale)))
    return HS2_ERR_INVALID_ARG;
  if (!check_attn_shape(B, T, L, H, D, dt) || slots > 4096) return HS2_ERR_UNSUPPORTED;
  if (dt == HS2_KV_FP8_E4M3 && D != 128) return HS2_ERR_UNSUPPORTED;

  SparseParams p;
  p.q = static_cast<const __nv_bfloat16*>(Q);
  p.k = static_cast<const uint8_t*>(kv->k);
  p.v = static_cast<const uint8_t*>(kv->v);
  p.k_scale = kv->k_scale;
  p.v_scale = kv->v_scale;
  p.idx = idx;
  p.n_sel = n_sel;
  p.o = O;
  p.B = B;
  p.T = T;
  p.H = H;
  p.D = D;
  p.slots = slots;
  p.L = L;
  p.scale_log2 = scale * kLog2e;
  const long long queries = (long long)B * T;
  const int sms = sm_count();
  int cs = 1;
  while (cs < 8 && queries * cs * 2 <= sms && cs * kSpTile < slots) cs *= 2;
  p.cs = cs;
  const bool fp8 = dt == HS2_KV_FP8_E4M3;
  cudaStream_t s = (cudaStream_t)stream;
  if (fp8) return H == 32 ? run_sparse<2, 128, true>(p, s) : run_sparse<1, 128, true>(p, s);
  if (D == 128) return H == 32 ? run_sparse<2, 128, false>(p, s) : run_sparse<1, 128, false>(p, s);
  return H == 32 ? run_sparse<2, 64, false>(p, s) : run_sparse<1, 64, false>(p, s);
}

}  // extern "C"

namespace {

void fill_bridge_params(BridgeParams* p, const hs2_kv_cache* caches, int n_layers, bool fp8,
                        int64_t T, int64_t row_offset, int hidden) {
  std::memset(p, 0, sizeof(*p));
  for (int l = 0; l < n_layers; ++l) {
    p->k[l] = caches[l].k;
    p->v[l] = caches[l].v;
    p->k_scale[l] = fp8 ? caches[l].k_scale : nullptr;
    p->v_scale[l] = fp8 ? caches[l].v_scale : nullptr;
  }
  p->T = T;
  p->row_offset = row_offset;
  p->hidden = hidden;
  p->n_layers = n_layers;
  p->fp8 = fp8 ? 1 : 0;
}

// The few-token path of hs2_bridge_kv (T <= kBsMaxT): one cluster of
// kBsCluster CTAs per 128-column segment, the hidden dimension split over the
// cluster (bridge_small.cuh).
hs2_status bridge_small(const void* X, int64_t T, int hidden, const void* Wt, int n_layers,
                        bool fp8, const hs2_kv_cache* caches, int64_t row_offset,
                        cudaStream_t s) {
  const int np = (int)((T + 15) / 16 * 16);
  CUtensorMap xm, wm;
  if (!make_map_2d(&xm, X, (uint64_t)T, (uint64_t)hidden, 2, kBrBK, (uint32_t)np) ||
      !make_map_2d(&wm, Wt, (uint64_t)n_layers * kBrBN, (uint64_t)hidden, 2, kBrBK, 128))
    return HS2_ERR_CUDA;
  BridgeParams p;
  fill_bridge_params(&p, caches, n_layers, fp8, T, row_offset, hidden);
  auto k = np == 16 ? bridge_small_kernel<16>
                    : np == 32 ? bridge_small_kernel<32>
                               : np == 48 ? bridge_small_kernel<48> : bridge_small_kernel<64>;
  const int bytes = np == 16 ? BsSmem<16>::kBytes
                             : np == 32 ? BsSmem<32>::kBytes
                                        : np == 48 ? BsSmem<48>::kBytes : BsSmem<64>::kBytes;
  if (!set_smem(k, bytes)) return HS2_ERR_CUDA;
  return launch(k, dim3((unsigned)(n_layers * 2 * kBsCluster)), dim3(kBsThreads), (size_t)bytes, s,
                kBsCluster, xm, wm, p);
}

}  // namespace

extern "C" hs2_status hs2_bridge_kv(const void* X, int64_t T, int hidden, const void* Wt,
                                    int n_layers, int D, hs2_kv_dtype out_dtype,
                                    const hs2_kv_cache* caches, int64_t cache_row_offset,
                                    hs2_stream_t stream) {
  if (!X || !Wt || !caches || T < 1 || hidden < 1 || n_layers < 1 || cache_row_offset < 0)
    return HS2_ERR_INVALID_ARG;
  if (out_dtype != HS2_KV_BF16 && out_dtype != HS2_KV_FP8_E4M3) return HS2_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Wt)) return HS2_ERR_INVALID_ARG;
  const bool fp8 = out_dtype == HS2_KV_FP8_E4M3;
  for (int l = 0; l < n_layers; ++l) {
    const hs2_kv_cache& c = caches[l];
    if (!c.k || !c.v || !aligned16(c.k) || !aligned16(c.v)) return HS2_ERR_INVALID_ARG;
    if (fp8 && (!c.k_scale || !c.v_scale || !aligned4(c.k_scale) || !aligned4(c.v_scale)))
      return HS2_ERR_INVALID_ARG;
  }
  if (D != 128 || hidden % kBrBK != 0 || n_layers > kBrMaxLayers || T > INT32_MAX - kBrBM)
    return HS2_ERR_UNSUPPORTED;
  if (T <= kBsMaxT) return bridge_small(X, T, hidden, Wt, n_layers, fp8, caches, cache_row_offset,
                                        (cudaStream_t)stream);
  CUtensorMap xm, wm;
  if (!make_map_2d(&xm, X, (uint64_t)T, (uint64_t)hidden, 2, kBrBK, kBrBM) ||
      !make_map_2d(&wm, Wt, (uint64_t)n_layers * kBrBN, (uint64_t)hidden, 2, kBrBK, kBrBN))
    return HS2_ERR_CUDA;
  BridgeParams p;
  fill_bridge_params(&p, caches, n_layers, fp8, T, cache_row_offset, hidden);
  if (!set_smem(bridge_gemm_kernel, kBrSmemBytes)) return HS2_ERR_CUDA;
  const long long tiles = (T + kBrBM - 1) / kBrBM * n_layers;
  const int grid = (int)std::min<long long>(tiles, sm_count());
  return launch(bridge_gemm_kernel, dim3(grid), dim3(kBrThreads), kBrSmemBytes,
                (cudaStream_t)stream, 1, xm, wm, p);
}

// ------------------------------------------------------------------------
// Allocation-free variant of hs2_full_attn_select: the workspace is a static
// device array compiled into the library (one per device, alive until the
// process exits), shared by every call.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[HS2_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device

// Device address of the scratch array on the current device.  Outside stream
// capture it is looked up on every call (a device reset reloads the module,
// and the array may then sit elsewhere); under capture the address of the last
// lookup on this device is used, since a lookup may load the module, which
// capture forbids.  (The host-side name of the array is only a stand-in: a
// kernel handed it would fault or read the wrong memory.)
hs2_status noalloc_scratch(cudaStream_t s, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HS2_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HS2_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    cudaGetLastError();
    return HS2_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cs == cudaStreamCaptureStatusNone || !g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return HS2_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HS2_OK;
}

}  // namespace

extern "C" hs2_status hs2_full_attn_select_noalloc(const void* Q, const hs2_kv_cache* kv, int B,
                                                   int T, int64_t L, int H, int D, float scale,
                                                   int topk, int window, hs2_kv_dtype dt,
                                                   float* O, float* lse, int32_t* idx,
                                                   int32_t* n_sel, hs2_stream_t stream) {
  // arguments first, exactly as hs2_full_attn_select checks them; then the size
  const hs2_status chk = check_full_args(Q, kv, B, T, L, H, D, scale, topk, window, dt, O, lse,
                                         idx, n_sel);
  if (chk != HS2_OK) return chk;
  const size_t need = hs2_full_attn_select_workspace(B, T, L, H, D, topk, window, dt);
  if (need == 0) return HS2_ERR_UNSUPPORTED;
  if (need > HS2_NOALLOC_SCRATCH_BYTES) return HS2_ERR_WORKSPACE;
  void* scratch = nullptr;
  const hs2_status st = noalloc_scratch((cudaStream_t)stream, &scratch);
  if (st != HS2_OK) return st;
  return hs2_full_attn_select(Q, kv, B, T, L, H, D, scale, topk, window, dt, O, lse, idx, n_sel,
                              scratch, (size_t)HS2_NOALLOC_SCRATCH_BYTES, stream);
}
