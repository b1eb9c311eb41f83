// Sparse-attention layer with KV Reuse: each query attends over its selected
// positions of the shared cache.
//
// One thread-block cluster of CS CTAs per query.  CTA r of the cluster takes
// the contiguous slot range [r*S, (r+1)*S), S = ceil(slots / CS), so every CTA
// of a full selection has the same work.  It loads its slots' positions, the
// query's n_sel and the query rows in one asynchronous round trip,
// range-checks the positions, and walks its range in 128-slot tiles: the K/V
// rows of a tile are gathered with 16-byte cp.async copies into 128B-swizzled
// shared-memory tiles (a two-stage ring) and each of the 8 warps runs the
// warp attention core over its 16-key group of the tile (a group with no
// valid key is neither gathered nor computed).  The CTA merges its warps;
// then each CTA pushes the slices of its merged partial to the CTAs that own
// them with distributed-shared-memory stores, and one cluster barrier later
// every CTA merges its slice of the query's H x D output from its own shared
// memory.  No global scratch is needed.
#pragma once

#include "attn_warp.cuh"

namespace hs2 {

constexpr int kSpWarps = 8;
constexpr int kSpThreads = kSpWarps * 32;
constexpr int kSpGroup = 16;                   // keys per warp per tile
constexpr int kSpTile = kSpWarps * kSpGroup;   // keys per tile

struct SparseParams {
  const __nv_bfloat16* q;  // [B][T][H][D]
  const uint8_t* k;        // [B][L][D] (bf16 or E4M3 bytes)
  const uint8_t* v;
  const float* k_scale;    // [B][L] or null
  const float* v_scale;
  const int32_t* idx;      // [B*T][slots]
  const int32_t* n_sel;    // [B*T]
  float* o;                // [B][T][H][D]
  int B, T, H, D, slots, cs;
  long long L;
  float scale_log2;
};

// Slots per CTA of a cluster of cs CTAs.
__host__ __device__ __forceinline__ int sparse_share(int slots, int cs) {
  return (slots + cs - 1) / cs;
}

template <int MT, int D, bool FP8>
struct SparseSmem {
  static constexpr int kRowsQ = MT * 16;
  static constexpr int kElem = FP8 ? 1 : 2;
  static constexpr int kTileBytes = kSpTile * D * kElem;
  // ring stages: a query with many tiles (one CTA per query) keeps kStages - 1
  // tiles of gathers in flight; E4M3 tiles are half the size, so three fit
  // beside the per-warp f16 staging
  static constexpr int kStages = FP8 ? 3 : 2;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStagingBytes = FP8 ? kSpWarps * 2 * kSpGroup * D * 2 : 0;
  static constexpr int kObufBytes = kSpWarps * kRowsQ * (D + 8) * 4;
  static constexpr int kRing = kStages * kStageBytes + kStagingBytes;
  static constexpr int kMain = kRing > kObufBytes ? kRing : kObufBytes;
  static constexpr int kQOff = kMain;
  static constexpr int kMlOff = kQOff + kRowsQ * D * 2;
  static constexpr int kClOff = kMlOff + kSpWarps * kRowsQ * 8;  // merge inputs
  // cs * ceil(H / cs) rows: at most H + cs - 1 for clusters of up to 16 CTAs
  static constexpr int kClRows = kRowsQ + 16;
  static constexpr int kClBytes = kClRows * 8 + kClRows * D * 4;
  static constexpr int kPosOff = kClOff + kClBytes;               // positions of the CTA's slots
  static constexpr int kMaxSlots = 4096;
  static constexpr int kBytes = kPosOff + (kMaxSlots + kSpTile + 4) * 4 + 1024;
  static_assert(kBytes <= 232448, "shared memory per CTA");
};

// 4-byte global->shared copy (the L1-allocating form; the .cg form moves 16
// bytes only); src_bytes == 0 writes zeros.
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}

// Gathers the K/V rows 0 .. rows-1 of one tile (positions pos[r], -1 =
// masked: zero-filled) into a ring stage.  All threads; one commit group.
template <int D, bool FP8>
__device__ __forceinline__ void sparse_gather_tile(const SparseParams& p, int b, const int* pos,
                                                   int rows, uint8_t* stage) {
  constexpr int kRowBytes = D * (FP8 ? 1 : 2);
  constexpr int kChunks = kRowBytes / 16;
  constexpr int kTileBytes = kSpTile * kRowBytes;
  const uint32_t dst0 = smem_u32(stage);
  const long long row0 = (long long)b * p.L;
  for (int u = threadIdx.x; u < rows * kChunks; u += kSpThreads) {
    const int r = u / kChunks, ch = u % kChunks;
    const int ps = pos[r];
    const long long src_off = (row0 + (ps < 0 ? 0 : ps)) * kRowBytes + ch * 16;
    uint32_t off;
    if (FP8)
      off = (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
    else
      off = sw128_offset(r, ch * 16, kSpTile);
    cp_async16(dst0 + off, p.k + src_off, ps < 0 ? 0 : 16);
    cp_async16(dst0 + kTileBytes + off, p.v + src_off, ps < 0 ? 0 : 16);
  }
  cp_async_commit();
}

template <int MT, int D, bool FP8>
__global__ void __launch_bounds__(kSpThreads) sparse_attn_kernel(const SparseParams p) {
  using SM = SparseSmem<MT, D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* qs = smem + SM::kQOff;
  float2* ml_s = reinterpret_cast<float2*>(smem + SM::kMlOff);
  // merge inputs: with a cluster, [source CTA][row of this CTA's slice] (m, l)
  // and [source CTA][element of the slice] O, written by the cluster's CTAs
  float2* cl_ml = reinterpret_cast<float2*>(smem + SM::kClOff);
  float* cl_o = reinterpret_cast<float*>(smem + SM::kClOff + SM::kClRows * 8);
  int* pos_all = reinterpret_cast<int*>(smem + SM::kPosOff);  // [tiles][kSpTile]

  const int cs = p.cs;
  pdl_launch_dependents();
  // first cluster phase: this CTA runs (its merge inputs may be written once
  // the phase completes, just before the merge)
  if (cs > 1) cluster_arrive_relaxed();
  const uint32_t rank = cs > 1 ? cluster_ctarank() : 0u;
  const long long qrow = blockIdx.x / cs;  // b*T + t
  const int b = (int)(qrow / p.T);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int32_t* sel = p.idx + qrow * p.slots;
  // this CTA's slot range [lo, hi) and the tiles it would take if all were used
  const int share = sparse_share(p.slots, cs);
  const int lo = (int)rank * share;
  const int hi = min(lo + share, p.slots);
  const int tiles_max = (share + kSpTile - 1) / kSpTile;
  int* nsel_s = pos_all + tiles_max * kSpTile;
  __shared__ int s_n_valid, s_redo;
  // The range's positions (slots past the range read as 0) and n_sel: valid
  // slots keep their position, the others -1 (out-of-range positions too,
  // raising kStatusBadIndex when `report`).  All threads; ends with a barrier.
  auto load_positions = [&](bool report) {
    if (threadIdx.x == 0) cp_async4(smem_u32(nsel_s), p.n_sel + qrow, 4);
    for (int u = threadIdx.x; u < tiles_max * kSpTile; u += kSpThreads) {
      const int slot = lo + u;
      const bool in = slot < hi;
      cp_async4(smem_u32(pos_all + u), in ? sel + slot : sel, in ? 4 : 0);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    const int nv = max(0, min(max(0, min(*nsel_s, p.slots)), hi) - lo);
    for (int u = threadIdx.x; u < tiles_max * kSpTile; u += kSpThreads) {
      int ps = pos_all[u];
      if (u >= nv) {
        ps = -1;
      } else if (ps < 0 || (long long)ps >= p.L) {
        if (report) raise_status(kStatusBadIndex);
        ps = -1;
      }
      pos_all[u] = ps;
    }
    if (threadIdx.x == 0) s_n_valid = nv;
    __syncthreads();
  };
  // rows of tile k that hold a valid slot's group: whole 16-key groups
  auto tile_rows = [&](int k, int nv) {
    const int v = min(kSpTile, nv - k * kSpTile);
    return (v + kSpGroup - 1) / kSpGroup * kSpGroup;
  };
  // prologue: fill kStages-1 ring slots (one commit group each)
  auto gather_prologue = [&](int nv) {
    const int mt = (nv + kSpTile - 1) / kSpTile;
#pragma unroll
    for (int s2 = 0; s2 < SM::kStages - 1; ++s2) {
      if (s2 < mt)
        sparse_gather_tile<D, FP8>(p, b, pos_all + s2 * kSpTile, tile_rows(s2, nv),
                                   smem + s2 * SM::kStageBytes);
      else
        cp_async_commit();
    }
  };
  // The positions and the first tiles' K/V rows are read before the wait on
  // the previous kernel: in a block of sparse layers the indices were final
  // before the previous layer began, and the gathers then overlap it.  After
  // the wait the positions are read again; if any differs (indices rewritten
  // by the previous kernel) the gathers are redone.
  load_positions(false);
  gather_prologue(s_n_valid);
  pdl_wait();  // indices, counts and queries come from earlier kernels
  {
    constexpr int kChunks = D * 2 / 16;
    const uint32_t q_s = smem_u32(qs);
    for (int u = threadIdx.x; u < SM::kRowsQ * kChunks; u += kSpThreads) {
      const int r = u / kChunks, ch = u % kChunks;
      const bool in = r < p.H;
      cp_async16(q_s + sw128_offset(r, ch * 16, SM::kRowsQ),
                 p.q + (qrow * p.H + (in ? r : 0)) * D + ch * 8, in ? 16 : 0);
    }
    cp_async_commit();
  }
  {  // validate the positions read before the wait
    const int nv0 = s_n_valid;
    if (threadIdx.x == 0) s_redo = 0;
    __syncthreads();
    const int nsel_now = __ldcg(p.n_sel + qrow);
    const int nv = max(0, min(max(0, min(nsel_now, p.slots)), hi) - lo);
    bool differs = nv != nv0;
    constexpr int kBatch = 8;  // independent loads in flight per thread
    for (int u0 = threadIdx.x; u0 < nv0; u0 += kBatch * kSpThreads) {
      int v[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int u = u0 + k * kSpThreads;
        v[k] = u < nv0 ? __ldcg(sel + lo + u) : 0;
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int u = u0 + k * kSpThreads;
        if (u < nv0) {
          const int ps = (v[k] < 0 || (long long)v[k] >= p.L) ? -1 : v[k];
          differs |= ps != pos_all[u];
        }
      }
    }
    if (differs) s_redo = 1;
    __syncthreads();
    if (s_redo) {  // (uniform) the gathers in flight land before the stages are refilled
      cp_async_wait<0>();
      __syncthreads();
      load_positions(true);
      gather_prologue(s_n_valid);
    } else {
      for (int u = threadIdx.x; u < nv0; u += kSpThreads)  // the status of bad positions
        if (pos_all[u] < 0) raise_status(kStatusBadIndex);
    }
  }
  cp_async_wait<0>();  // the query rows (and the prologue tiles, issued well before)
  __syncthreads();
  const int n_valid = s_n_valid;
  const int my_tiles = (n_valid + kSpTile - 1) / kSpTile;
  const float* ksc = FP8 ? p.k_scale + (long long)b * p.L : nullptr;
  const float* vsc = FP8 ? p.v_scale + (long long)b * p.L : nullptr;

  WarpAttn<MT, D> st;
  st.init();
  const uint32_t q_base = smem_u32(qs);
  uint8_t* stg_k = smem + SM::kStages * SM::kStageBytes + warp * 2 * kSpGroup * D * 2;
  uint8_t* stg_v = stg_k + kSpGroup * D * 2;

  for (int k = 0; k < my_tiles; ++k) {
    {  // refill the slot consumed in step k-1 (all threads passed the barrier ending it)
      const int kn = k + SM::kStages - 1;
      if (kn < my_tiles)
        sparse_gather_tile<D, FP8>(p, b, pos_all + kn * kSpTile, tile_rows(kn, n_valid),
                                   smem + (kn % SM::kStages) * SM::kStageBytes);
      else
        cp_async_commit();
    }
    cp_async_wait<SM::kStages - 1>();  // tile k has landed
    __syncthreads();
    // this warp's 16-key group: skipped when it holds no valid slot (its rows
    // were not gathered)
    if (warp * kSpGroup < tile_rows(k, n_valid)) {
      const int s = k % SM::kStages;
      uint8_t* stage = smem + s * SM::kStageBytes;
      const int* pos = pos_all + k * kSpTile;
      uint32_t kt, vt;
      int key0, rows;
      if (FP8) {
        warp_fp8_rows_to_bf16(stage, warp * kSpGroup, kSpGroup, stg_k, kSpGroup);
        warp_fp8_rows_to_bf16(stage + SM::kTileBytes, warp * kSpGroup, kSpGroup, stg_v, kSpGroup);
        __syncwarp();
        kt = smem_u32(stg_k);
        vt = smem_u32(stg_v);
        key0 = 0;
        rows = kSpGroup;
      } else {
        kt = smem_u32(stage);
        vt = smem_u32(stage + SM::kTileBytes);
        key0 = warp * kSpGroup;
        rows = kSpTile;
      }
      float x[MT][2][4];
      warp_qk<MT, D>(q_base, kt, key0, rows, x);
      float pvs[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int ps = pos[warp * kSpGroup + nt * 8 + 2 * c + j];
          const float ks = (FP8 && ps >= 0) ? ksc[ps] : 1.f;
          pvs[nt][j] = (FP8 && ps >= 0) ? vsc[ps] : 1.f;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              x[mt][nt][2 * h + j] =
                  ps >= 0 ? x[mt][nt][2 * h + j] * (p.scale_log2 * ks) : kNegInf;
        }
      warp_softmax_pv<MT, D>(st, x, vt, key0, rows, pvs);
    }
    __syncthreads();  // ring slot k % kStages is free again
  }
  cp_async_wait<0>();
  __syncthreads();

  // merge the warps: rescale each warp's O to the CTA's row maximum
  float lf[MT][2], f[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      lf[mt][h] = quad_sum(st.l[mt][h]);
      if (c == 0) ml_s[warp * SM::kRowsQ + mt * 16 + g + 8 * h] = make_float2(st.m[mt][h], lf[mt][h]);
    }
  __syncthreads();
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = mt * 16 + g + 8 * h;
      float M = kNegInf;
#pragma unroll
      for (int w = 0; w < kSpWarps; ++w) M = fmaxf(M, ml_s[w * SM::kRowsQ + r].x);
      f[mt][h] = (M == kNegInf) ? 0.f : fast_exp2(st.m[mt][h] - M);
    }
  float* obuf = reinterpret_cast<float*>(smem);
  warp_store_o<MT, D>(st, f, obuf + warp * SM::kRowsQ * (D + 8));
  // CTA `rank` of the cluster owns rows [rank*rpc, (rank+1)*rpc) of the H x D
  // output, rpc = ceil(H / cs): the last owner may own fewer rows, and CTAs past
  // it none (cs need not divide H)
  const int rpc = (p.H + cs - 1) / cs;
  const int chunk = rpc * D;
  const int own_rows = max(0, min(rpc, p.H - (int)rank * rpc));
  const uint32_t ml_addr = smem_u32(cl_ml), o_addr = smem_u32(cl_o);
  if (cs > 1) cluster_wait_acquire();  // first phase: every CTA of the cluster runs
  __syncthreads();
  // this CTA's (m, l) per row and its O summed over the warps, stored locally
  // (no cluster) or pushed to the slice's owner
  if (threadIdx.x < p.H) {
    const int r = threadIdx.x;
    float M = kNegInf;
    for (int w = 0; w < kSpWarps; ++w) M = fmaxf(M, ml_s[w * SM::kRowsQ + r].x);
    float lt = 0.f;
    if (M != kNegInf)
      for (int w = 0; w < kSpWarps; ++w) {
        const float2 v = ml_s[w * SM::kRowsQ + r];
        lt += v.y * fast_exp2(v.x - M);
      }
    if (cs == 1)
      cl_ml[r] = make_float2(M, lt);
    else
      st_dsmem_f32x2(mapa_shared(ml_addr + ((int)rank * rpc + r % rpc) * 8, (uint32_t)(r / rpc)),
                     make_float2(M, lt));
  }
  for (int u = 4 * threadIdx.x; u < p.H * D; u += 4 * kSpThreads) {
    const int r = u / D, d = u % D;
    float4 acc = *reinterpret_cast<const float4*>(obuf + r * (D + 8) + d);
#pragma unroll
    for (int w = 1; w < kSpWarps; ++w) {
      const float4 o = *reinterpret_cast<const float4*>(obuf + (w * SM::kRowsQ + r) * (D + 8) + d);
      acc.x += o.x;
      acc.y += o.y;
      acc.z += o.z;
      acc.w += o.w;
    }
    if (cs == 1)
      *reinterpret_cast<float4*>(cl_o + u) = acc;
    else
      st_dsmem_f32x4(mapa_shared(o_addr + ((int)rank * chunk + u % chunk) * 4, (uint32_t)(u / chunk)),
                     acc);
  }
  if (cs == 1) {
    __syncthreads();
    for (int u = 4 * threadIdx.x; u < p.H * D; u += 4 * kSpThreads) {
      const float2 v = cl_ml[u / D];
      const float inv = v.y > 0.f ? 1.f / v.y : 0.f;
      const float4 o = *reinterpret_cast<const float4*>(cl_o + u);
      *reinterpret_cast<float4*>(p.o + qrow * p.H * D + u) =
          make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
    }
    return;
  }
  // second phase: every CTA's pushes have landed; nothing reads another CTA's
  // shared memory after it, so each CTA may exit when its slice is written
  cluster_arrive_release();
  cluster_wait_acquire();
  for (int e = 4 * threadIdx.x; e < own_rows * D; e += 4 * kSpThreads) {
    const int rl = e / D;
    float M = kNegInf;
    for (int q = 0; q < cs; ++q) M = fmaxf(M, cl_ml[q * rpc + rl].x);
    float lt = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < cs; ++q) {
      const float2 ml = cl_ml[q * rpc + rl];
      const float f = (M == kNegInf || ml.x == kNegInf) ? 0.f : fast_exp2(ml.x - M);
      const float4 o = *reinterpret_cast<const float4*>(cl_o + q * chunk + e);
      lt += ml.y * f;
      acc.x += f * o.x;
      acc.y += f * o.y;
      acc.z += f * o.z;
      acc.w += f * o.w;
    }
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    *reinterpret_cast<float4*>(p.o + qrow * p.H * D + (long long)rank * chunk + e) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
}

}  // namespace hs2
