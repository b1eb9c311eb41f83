// Warp-level attention core: one warp owns MT*16 query rows and a 16-key
// slice of a key tile held in shared memory (bf16, 128B-swizzled layout of
// hs2_common.cuh).  It computes the logits with m16n8k16 tensor-core MMAs,
// keeps an online softmax (base-2 logits, per-row running max m and sum l)
// and accumulates O = P V, also on the tensor cores.
#pragma once

#include "hs2_common.cuh"

namespace hs2 {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kNegInf = -INFINITY;

// C-fragment ownership in m16n8k16: lane = 4*g + c holds rows g and g+8 of
// an m-tile and columns 2c, 2c+1 of an n-tile.
template <int MT, int D>
struct WarpAttn {
  float o[MT][D / 8][4];
  float m[MT][2];
  float l[MT][2];

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        m[mt][h] = kNegInf;
        l[mt][h] = 0.f;
      }
#pragma unroll
      for (int dn = 0; dn < D / 8; ++dn)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[mt][dn][e] = 0.f;
    }
  }
};

// S[mt][nt] (raw dot products) of the warp's rows against 16 keys starting at
// row `key0` of the key tile.  q_base/k_base are shared-memory addresses of
// the Q tile (rows_q rows per column half; the warp's rows start at q_row0)
// and of the key tile (rows_k rows per column half).
template <int MT, int D>
__device__ __forceinline__ void warp_qk(uint32_t q_base, uint32_t k_base, int key0, int rows_k,
                                        float s[MT][2][4], int q_row0 = 0, int rows_q = MT * 16) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[mt][nt][e] = 0.f;
  const int qrow = lane & 15;
  const int qcol = (lane >> 4) * 16;
  const int krow = key0 + (lane & 7) + ((lane >> 4) << 3);
  const int kcol = ((lane >> 3) & 1) * 16;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    uint32_t a[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
      ldsm_x4(q_base + sw128_offset(q_row0 + mt * 16 + qrow, ks * 32 + qcol, rows_q), a[mt][0],
              a[mt][1], a[mt][2], a[mt][3]);
    uint32_t b0, b1, b2, b3;
    ldsm_x4(k_base + sw128_offset(krow, ks * 32 + kcol, rows_k), b0, b1, b2, b3);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      mma_bf16_16816(s[mt][0], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
      mma_bf16_16816(s[mt][1], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b2, b3);
    }
  }
}

// Online-softmax update with base-2 logits x[mt][nt][e] (-inf = masked) and
// O += P V for the 16 keys at row key0 of the value tile, over the D value
// columns that start at byte column col0 of the tile.  pv_scale[nt][j] is the
// factor applied to p of key (nt*8 + 2c + j) before the PV product (the
// per-token E4M3 value scale; 1 for bf16).  l accumulates the unscaled p.
template <int MT, int D>
__device__ __forceinline__ void warp_softmax_pv(WarpAttn<MT, D>& st, float x[MT][2][4],
                                                uint32_t v_base, int key0, int rows_v,
                                                const float pv_scale[2][2], int col0 = 0) {
  const int lane = threadIdx.x & 31;
  uint32_t pa[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = fmaxf(fmaxf(x[mt][0][2 * h], x[mt][0][2 * h + 1]),
                       fmaxf(x[mt][1][2 * h], x[mt][1][2 * h + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(st.m[mt][h], mx);
      const float corr = (m_new == kNegInf) ? 1.f : fast_exp2(st.m[mt][h] - m_new);
      st.m[mt][h] = m_new;
      float rs = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float xv = x[mt][nt][2 * h + j];
          const float p = (xv == kNegInf) ? 0.f : fast_exp2(xv - m_new);
          rs += p;
          x[mt][nt][2 * h + j] = p * pv_scale[nt][j];
        }
      st.l[mt][h] = st.l[mt][h] * corr + rs;
#pragma unroll
      for (int dn = 0; dn < D / 8; ++dn) {
        st.o[mt][dn][2 * h] *= corr;
        st.o[mt][dn][2 * h + 1] *= corr;
      }
    }
    pa[mt][0] = pack_bf16(x[mt][0][0], x[mt][0][1]);
    pa[mt][1] = pack_bf16(x[mt][0][2], x[mt][0][3]);
    pa[mt][2] = pack_bf16(x[mt][1][0], x[mt][1][1]);
    pa[mt][3] = pack_bf16(x[mt][1][2], x[mt][1][3]);
  }
  const int vrow = key0 + (lane & 7) + (((lane >> 3) & 1) << 3);
  const int vcol = (lane >> 4) * 16;
#pragma unroll
  for (int dp = 0; dp < D / 16; ++dp) {
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(v_base + sw128_offset(vrow, col0 + dp * 32 + vcol, rows_v), b0, b1, b2, b3);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      mma_bf16_16816(st.o[mt][2 * dp], pa[mt][0], pa[mt][1], pa[mt][2], pa[mt][3], b0, b1);
      mma_bf16_16816(st.o[mt][2 * dp + 1], pa[mt][0], pa[mt][1], pa[mt][2], pa[mt][3], b2, b3);
    }
  }
}

// Converts `nkeys` rows (starting at row key0) of an E4M3 tile (128-byte
// swizzled rows of D = 128 codes) into the bf16 swizzled layout of a tile
// with rows_out rows per column half, as its rows dst_row0 .. dst_row0+nkeys-1.
// Whole warp.
__device__ __forceinline__ void warp_fp8_rows_to_bf16(const uint8_t* src, int key0, int nkeys,
                                                      uint8_t* dst, int rows_out,
                                                      int dst_row0 = 0) {
  const int lane = threadIdx.x & 31;
  for (int u = lane; u < nkeys * 8; u += 32) {
    const int r = u >> 3, ch = u & 7;  // 16 codes = columns 16ch .. 16ch+15
    const int sr = key0 + r;
    const uint4 raw =
        *reinterpret_cast<const uint4*>(src + sr * 128 + (((ch ^ (sr & 7))) << 4));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t outv[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      outv[2 * k] = e4m3x2_to_bf16x2((uint16_t)(w[k] & 0xFFFFu));
      outv[2 * k + 1] = e4m3x2_to_bf16x2((uint16_t)(w[k] >> 16));
    }
    // bf16 columns 16ch .. 16ch+7 and 16ch+8 .. 16ch+15 -> byte columns 32ch, 32ch+16
    *reinterpret_cast<uint4*>(dst + sw128_offset(dst_row0 + r, ch * 32, rows_out)) =
        make_uint4(outv[0], outv[1], outv[2], outv[3]);
    *reinterpret_cast<uint4*>(dst + sw128_offset(dst_row0 + r, ch * 32 + 16, rows_out)) =
        make_uint4(outv[4], outv[5], outv[6], outv[7]);
  }
}

// Writes the warp's un-normalised partial O (scaled by f[mt][h]) into a
// shared fp32 buffer obuf[row][D + 8].
template <int MT, int D>
__device__ __forceinline__ void warp_store_o(const WarpAttn<MT, D>& st, const float f[MT][2],
                                             float* obuf) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = mt * 16 + g + 8 * h;
#pragma unroll
      for (int dn = 0; dn < D / 8; ++dn) {
        float2 v = make_float2(st.o[mt][dn][2 * h] * f[mt][h], st.o[mt][dn][2 * h + 1] * f[mt][h]);
        *reinterpret_cast<float2*>(obuf + row * (D + 8) + dn * 8 + 2 * c) = v;
      }
    }
}

// Sum of the quad's partial row sums (lanes 4g .. 4g+3 share a row).
__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

}  // namespace hs2
