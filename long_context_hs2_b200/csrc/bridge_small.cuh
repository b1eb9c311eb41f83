// KV Bridging for a few tokens at a time: the decode-time append of the bridged
// K/V rows (IT Home announcement, decode paragraph: the Cross-Decoder's layers
// take part in every generated token, so each new token's hidden state is
// bridged into every target layer's cache; cnyes.com article, section
// "預填充只走前半程").
//
// With T <= 64 tokens the projection Y = X * Wt^T is a matrix-vector product in
// all but name: every weight is read once and used T times, so the kernel is
// bound by reading Wt (n_layers * 256 rows x hidden bf16: 12.6 MB for 6 layers
// at hidden 4096), not by arithmetic.  The work is spread over the SMs by
// splitting both the output columns and the hidden dimension:
//   * one thread-block cluster of kBsCluster CTAs per 128-column segment (one
//     layer's K or V), CTA r of the cluster taking the r-th slice of the
//     hidden dimension (12 segments x 8 CTAs = 96 CTAs streaming weights);
//   * each CTA streams its 128 weight rows and the T token rows of X through a
//     TMA ring and accumulates the partial Y^T[128 columns][T] on the tensor
//     cores (tcgen05.mma kind::f16, M = 128 columns, N = T rounded up to 16,
//     fp32 accumulator in tensor memory);
//   * the cluster's partials are summed through distributed shared memory:
//     every CTA pushes its column values of token t to the CTA that owns t
//     (t mod kBsCluster), and the owner writes the finished rows -- bf16, or
//     E4M3 codes with the per-token scale max|y| / 448 -- at cache_row_offset.
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator and MMA issuer,
// warps 2-5 (128 threads: thread c owns output column c of the segment) read
// the accumulator, push, reduce and store.
#pragma once

#include "bridge_gemm.cuh"

namespace hs2 {

constexpr int kBsMaxT = 64;            // tokens per launch of this path
constexpr int kBsCluster = 8;          // CTAs per segment (slices of the hidden dimension)
constexpr int kBsStages = 8;           // ring stages: hidden 4096 = 8 slices of 64 per CTA, all in flight
constexpr int kBsWBytes = 128 * kBrBK * 2;       // 16 KB: 128 weight rows x 64 hidden
constexpr int kBsThreads = 192;

// Shared-memory plan for NP tokens (the MMA's N): ring stages of a weight slice
// and the token slice, the cluster reduction's receive buffer, barriers.
template <int NP>
struct BsSmem {
  static constexpr int kXBytes = NP * kBrBK * 2;              // NP token rows x 64 hidden
  static constexpr int kStageBytes = kBsWBytes + kXBytes;      // a multiple of 1024
  static constexpr int kTokPerOwner = (NP + kBsCluster - 1) / kBsCluster;
  static constexpr int kRedOff = kBsStages * kStageBytes;
  static constexpr int kRedBytes = kBsCluster * kTokPerOwner * 128 * 4;   // [src][token][column]
  static constexpr int kAmaxOff = kRedOff + kRedBytes;                    // float [4 warps]
  static constexpr int kBarOff = kAmaxOff + 64;
  static constexpr int kBytes = kBarOff + 256 + 1024;
};

// NP: tokens rounded up to a multiple of 16 (the MMA's N).  Grid: kBsCluster
// CTAs per segment along x, clusters of kBsCluster.
template <int NP>
__global__ void __launch_bounds__(kBsThreads, 1)
    bridge_small_kernel(const __grid_constant__ CUtensorMap xmap,
                        const __grid_constant__ CUtensorMap wmap, const BridgeParams p) {
  static_assert(NP % 16 == 0 && NP <= kBsMaxT, "N of the MMA");
  using SM = BsSmem<NP>;
  static_assert(SM::kBytes <= 232448, "shared memory per CTA");
  constexpr int kTokPerOwner = SM::kTokPerOwner;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint64_t* empty = full + kBsStages;
  uint64_t* done = empty + kBsStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  float* red = reinterpret_cast<float*>(smem + SM::kRedOff);
  float* wamax = reinterpret_cast<float*>(smem + SM::kAmaxOff);

  // first cluster phase: this CTA runs (its receive buffer may be written once
  // the phase completes)
  cluster_arrive_relaxed();
  const uint32_t rank = cluster_ctarank();
  const int seg = blockIdx.x / kBsCluster;      // layer * 2 + (0: K, 1: V)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb_total = p.hidden / kBrBK;
  const int kb_per = (kb_total + kBsCluster - 1) / kBsCluster;
  const int kb0 = min(kb_total, (int)rank * kb_per);
  const int n_kb = min(kb_total, kb0 + kb_per) - kb0;   // may be 0 for a small hidden

  if (threadIdx.x == 0) {
    for (int s = 0; s < kBsStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  float y[NP];
#pragma unroll
  for (int t = 0; t < NP; ++t) y[t] = 0.f;
  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&xmap);
      tma_prefetch_desc(&wmap);
      const uint64_t pol = policy_evict_normal();
      for (int i = 0; i < n_kb; ++i) {
        const int s = i % kBsStages;
        if (i >= kBsStages && !mbar_wait(&empty[s], ((i / kBsStages) - 1) & 1)) break;
        uint8_t* st = smem + s * SM::kStageBytes;
        mbar_arrive_expect_tx(&full[s], kBsWBytes + NP * kBrBK * 2);
        tma_load_2d(st, &wmap, &full[s], (kb0 + i) * kBrBK, seg * 128, pol);
        tma_load_2d(st + kBsWBytes, &xmap, &full[s], (kb0 + i) * kBrBK, 0, pol);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_kb > 0) {
      constexpr uint32_t idesc = tc_idesc_f16(128, NP, kTcBF16, false, false);
      bool ok = true;
      for (int i = 0; i < n_kb && ok; ++i) {
        const int s = i % kBsStages;
        if (!mbar_wait(&full[s], (i / kBsStages) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t w_addr = smem_u32(smem + s * SM::kStageBytes);
        const uint64_t adesc = sw128_kmajor_desc(w_addr);
        const uint64_t bdesc = sw128_kmajor_desc(w_addr + kBsWBytes);
#pragma unroll
        for (int k = 0; k < kBrBK / 16; ++k)  // +32 bytes along the hidden dimension per step
          tc_mma_f16(tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (i | k) != 0);
        tc_commit(&empty[s]);
      }
      if (ok) tc_commit(done);
    }
  } else {
    // ------------------------------- epilogue warps: this CTA's partial Y^T
    if (n_kb > 0 && mbar_wait(done, 0)) {
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
#pragma unroll
      for (int c = 0; c < NP; c += 16) tmem_ld16(taddr + c, y + c);
      tmem_ld_wait();
    }
  }
  cluster_wait_acquire();   // every CTA of the cluster runs
  const int col = (warp & 3) * 32 + lane;   // epilogue thread: output column of the segment
  if (warp >= 2) {
    const uint32_t red_addr = smem_u32(red);
#pragma unroll
    for (int t = 0; t < NP; ++t)
      if (t < p.T) {
        const uint32_t owner = (uint32_t)(t % kBsCluster);
        const int slot = ((int)rank * kTokPerOwner + t / kBsCluster) * 128 + col;
        st_dsmem_f32(mapa_shared(red_addr + slot * 4, owner), y[t]);
      }
  }
  cluster_arrive_release();
  cluster_wait_acquire();   // every push has landed
  if (warp >= 2) {
    const int layer = seg >> 1, kv = seg & 1;
    for (int tl = 0; tl < kTokPerOwner; ++tl) {
      const int t = tl * kBsCluster + (int)rank;
      if (t >= p.T) break;   // uniform across the epilogue warps
      float v = 0.f;
#pragma unroll
      for (int src = 0; src < kBsCluster; ++src)
        v += red[(src * kTokPerOwner + tl) * 128 + col];
      const long long row = p.row_offset + t;
      if (!p.fp8) {
        reinterpret_cast<__nv_bfloat16*>(kv ? p.v[layer] : p.k[layer])[row * 128 + col] =
            __float2bfloat16_rn(v);
      } else {
        float a = fabsf(v);
#pragma unroll
        for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (lane == 0) wamax[warp & 3] = a;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const float amax = fmaxf(fmaxf(wamax[0], wamax[1]), fmaxf(wamax[2], wamax[3]));
        asm volatile("bar.sync 1, 128;" ::: "memory");   // wamax is rewritten for the next token
        const float s = amax > 0.f ? amax / 448.f : 1.f;
        reinterpret_cast<__nv_fp8_storage_t*>(kv ? p.v[layer] : p.k[layer])[row * 128 + col] =
            __nv_cvt_float_to_fp8(__fdiv_rn(v, s), __NV_SATFINITE, __NV_E4M3);
        if (col == 0) (kv ? p.v_scale[layer] : p.k_scale[layer])[row] = s;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

}  // namespace hs2
