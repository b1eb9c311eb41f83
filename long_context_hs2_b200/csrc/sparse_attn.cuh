// Sparse-attention layer with KV Reuse: each query attends over its selected
// positions of the shared cache.
//
// One thread-block cluster of CS CTAs per query.  The query's selected slots
// are cut into 64-slot tiles dealt round-robin to the cluster's CTAs; each CTA
// gathers its tiles' K/V rows with 16-byte cp.async copies into 128B-swizzled
// shared-memory tiles (a multi-stage ring), runs the warp attention core
// (warps split every tile's keys 4 ways), merges its warps, and the cluster's
// rank 0 merges the CTAs' partials through distributed shared memory.  No
// global scratch is needed.
#pragma once

#include "attn_warp.cuh"

namespace hs2 {

constexpr int kSpTile = 64;
constexpr int kSpWarps = 4;

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

template <int MT, int D, bool FP8>
struct SparseSmem {
  static constexpr int kRowsQ = MT * 16;
  static constexpr int kElem = FP8 ? 1 : 2;
  static constexpr int kTileBytes = kSpTile * D * kElem;
  static constexpr int kStages = 3;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStagingBytes = FP8 ? kSpWarps * 2 * 16 * D * 2 : 0;
  static constexpr int kObufBytes = kSpWarps * kRowsQ * (D + 8) * 4;
  static constexpr int kRing = kStages * kStageBytes + kStagingBytes;
  static constexpr int kMain = kRing > kObufBytes ? kRing : kObufBytes;
  static constexpr int kQOff = kMain;
  static constexpr int kMlOff = kQOff + kRowsQ * D * 2;
  static constexpr int kClOff = kMlOff + kSpWarps * kRowsQ * 8;  // CTA result: ml[rows], o[rows][D]
  static constexpr int kClBytes = kRowsQ * 8 + kRowsQ * D * 4;
  static constexpr int kPosOff = kClOff + kClBytes;               // positions of the ring's tiles
  static constexpr int kBytes = kPosOff + kStages * kSpTile * 4 + 1024;
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Gathers the K/V rows of slots [slot0, slot0 + 64) into one ring stage and
// records their positions (-1 = masked).  All 128 threads; one commit group.
template <int D, bool FP8>
__device__ __forceinline__ void sparse_gather_tile(const SparseParams& p, int b,
                                                   const int32_t* sel, int n, int slot0,
                                                   uint8_t* stage, int* pos_s) {
  constexpr int kRowBytes = D * (FP8 ? 1 : 2);
  constexpr int kChunks = kRowBytes / 16;
  constexpr int kTileBytes = kSpTile * kRowBytes;
  for (int u = threadIdx.x; u < kSpTile; u += kSpWarps * 32) {
    const int slot = slot0 + u;
    int pos = -1;
    if (slot < n) {
      pos = sel[slot];
      if (pos < 0 || (long long)pos >= p.L) {
        raise_status(kStatusBadIndex);
        pos = -1;
      }
    }
    pos_s[u] = pos;
  }
  __syncthreads();
  const uint32_t dst0 = smem_u32(stage);
  for (int u = threadIdx.x; u < 2 * kSpTile * kChunks; u += kSpWarps * 32) {
    const int tsr = u / (kSpTile * kChunks);  // 0: K, 1: V
    const int rem = u % (kSpTile * kChunks);
    const int r = rem / kChunks, ch = rem % kChunks;
    const int pos = pos_s[r];
    const uint8_t* base = tsr ? p.v : p.k;
    const uint8_t* src = base + ((long long)b * p.L + (pos < 0 ? 0 : pos)) * kRowBytes + ch * 16;
    uint32_t off;
    if (FP8)
      off = (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
    else
      off = sw128_offset(r, ch * 16, kSpTile);
    cp_async16(dst0 + tsr * kTileBytes + off, src, pos < 0 ? 0 : 16);
  }
  cp_async_commit();
}

template <int MT, int D, bool FP8>
__global__ void __launch_bounds__(128) sparse_attn_kernel(const SparseParams p) {
  using SM = SparseSmem<MT, D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* qs = smem + SM::kQOff;
  float2* ml_s = reinterpret_cast<float2*>(smem + SM::kMlOff);
  float2* cl_ml = reinterpret_cast<float2*>(smem + SM::kClOff);
  float* cl_o = reinterpret_cast<float*>(smem + SM::kClOff + SM::kRowsQ * 8);
  int* pos_ring = reinterpret_cast<int*>(smem + SM::kPosOff);

  const int cs = p.cs;
  const uint32_t rank = cs > 1 ? cluster_ctarank() : 0u;
  const long long qrow = blockIdx.x / cs;  // b*T + t
  const int b = (int)(qrow / p.T);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  int n = p.n_sel[qrow];
  n = max(0, min(n, p.slots));
  const int32_t* sel = p.idx + qrow * p.slots;
  const int n_tiles_all = (n + kSpTile - 1) / kSpTile;
  const int my_tiles = n_tiles_all > (int)rank ? (n_tiles_all - (int)rank + cs - 1) / cs : 0;

  // query rows: head h = row (rows >= H are zero)
  {
    constexpr int kChunks = D * 2 / 16;
    for (int u = threadIdx.x; u < SM::kRowsQ * kChunks; u += 128) {
      const int r = u / kChunks, ch = u % kChunks;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < p.H) v = *reinterpret_cast<const uint4*>(p.q + (qrow * p.H + r) * D + ch * 8);
      *reinterpret_cast<uint4*>(qs + sw128_offset(r, ch * 16, SM::kRowsQ)) = v;
    }
  }
  const float* ksc = FP8 ? p.k_scale + (long long)b * p.L : nullptr;
  const float* vsc = FP8 ? p.v_scale + (long long)b * p.L : nullptr;

  // prologue: fill kStages-1 ring slots
#pragma unroll
  for (int s = 0; s < SM::kStages - 1; ++s) {
    if (s < my_tiles)
      sparse_gather_tile<D, FP8>(p, b, sel, n, ((int)rank + s * cs) * kSpTile,
                                 smem + s * SM::kStageBytes, pos_ring + s * kSpTile);
    else
      cp_async_commit();
  }

  WarpAttn<MT, D> st;
  st.init();
  const uint32_t q_base = smem_u32(qs);
  uint8_t* stg_k = smem + SM::kStages * SM::kStageBytes + warp * 2 * 16 * D * 2;
  uint8_t* stg_v = stg_k + 16 * D * 2;

  for (int k = 0; k < my_tiles; ++k) {
    cp_async_wait<SM::kStages - 2>();
    __syncthreads();
    const int s = k % SM::kStages;
    uint8_t* stage = smem + s * SM::kStageBytes;
    const int* pos = pos_ring + s * kSpTile;
    uint32_t kt, vt;
    int key0, rows;
    if (FP8) {
      warp_fp8_rows_to_bf16(stage, warp * 16, 16, stg_k, 16);
      warp_fp8_rows_to_bf16(stage + SM::kTileBytes, warp * 16, 16, stg_v, 16);
      __syncwarp();
      kt = smem_u32(stg_k);
      vt = smem_u32(stg_v);
      key0 = 0;
      rows = 16;
    } else {
      kt = smem_u32(stage);
      vt = smem_u32(stage + SM::kTileBytes);
      key0 = warp * 16;
      rows = kSpTile;
    }
    float x[MT][2][4];
    warp_qk<MT, D>(q_base, kt, key0, rows, x);
    float pvs[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int ps = pos[warp * 16 + nt * 8 + 2 * c + j];
        const float ks = (FP8 && ps >= 0) ? ksc[ps] : 1.f;
        pvs[nt][j] = (FP8 && ps >= 0) ? vsc[ps] : 1.f;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            x[mt][nt][2 * h + j] = ps >= 0 ? x[mt][nt][2 * h + j] * (p.scale_log2 * ks) : kNegInf;
      }
    warp_softmax_pv<MT, D>(st, x, vt, key0, rows, pvs);
    __syncthreads();  // ring slot s is free again
    const int kn = k + SM::kStages - 1;
    const int sn = kn % SM::kStages;
    if (kn < my_tiles)
      sparse_gather_tile<D, FP8>(p, b, sel, n, ((int)rank + kn * cs) * kSpTile,
                                 smem + sn * SM::kStageBytes, pos_ring + sn * kSpTile);
    else
      cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();

  // merge the warps into this CTA's (m, l, O) in cl_ml / cl_o
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
  __syncthreads();
  for (int u = threadIdx.x; u < SM::kRowsQ * D; u += 128) {
    const int r = u / D, d = u % D;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kSpWarps; ++w) acc += obuf[(w * SM::kRowsQ + r) * (D + 8) + d];
    cl_o[u] = acc;
  }
  if (threadIdx.x < SM::kRowsQ) {
    const int r = threadIdx.x;
    float M = kNegInf;
    for (int w = 0; w < kSpWarps; ++w) M = fmaxf(M, ml_s[w * SM::kRowsQ + r].x);
    float lt = 0.f;
    if (M != kNegInf)
      for (int w = 0; w < kSpWarps; ++w) {
        const float2 v = ml_s[w * SM::kRowsQ + r];
        lt += v.y * fast_exp2(v.x - M);
      }
    cl_ml[r] = make_float2(M, lt);
  }
  if (cs > 1) cluster_sync_all();
  else __syncthreads();

  if (rank == 0) {
    // merge the cluster's CTAs (rank 0 reads the others' results in place)
    const uint32_t ml_addr = smem_u32(cl_ml), o_addr = smem_u32(cl_o);
    for (int u = threadIdx.x; u < p.H * D; u += 128) {
      const int r = u / D;
      float M = kNegInf;
      for (int q = 0; q < cs; ++q) M = fmaxf(M, ld_dsmem_f32(mapa_shared(ml_addr + r * 8, q)));
      float lt = 0.f, acc = 0.f;
      if (M != kNegInf)
        for (int q = 0; q < cs; ++q) {
          const float m = ld_dsmem_f32(mapa_shared(ml_addr + r * 8, q));
          const float l = ld_dsmem_f32(mapa_shared(ml_addr + r * 8 + 4, q));
          const float fct = (m == kNegInf) ? 0.f : fast_exp2(m - M);
          lt += l * fct;
          acc += fct * ld_dsmem_f32(mapa_shared(o_addr + u * 4, q));
        }
      p.o[qrow * p.H * D + u] = lt > 0.f ? acc / lt : 0.f;
    }
  }
  if (cs > 1) cluster_sync_all();  // keep every CTA's shared memory alive until rank 0 is done
}

}  // namespace hs2
