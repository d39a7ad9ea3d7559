// attn_core.cuh -- per-warp online-softmax attention over 64-key tiles held in
// shared memory (16 query rows per warp, bf16 operands, fp32 accumulation).
//
// Logits are kept in the log2 domain: x = (q . k) * (log2(e) / sqrt(d)), so that
// exp(s - m) == exp2(x - m2).  Row statistics m (running max) and l (running sum)
// are in that domain.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kKeyTile = 64;  // keys per tile

template <int D>
struct WarpAttn {
  static constexpr int kKSteps = D / 16;   // k16 steps over the head dimension
  static constexpr int kONTiles = D / 8;   // n8 tiles of the output
  static constexpr int kSNTiles = kKeyTile / 8;

  uint32_t qf[kKSteps][4];
  float o[kONTiles][4];
  float m[2], l[2];  // rows (lane/4) and (lane/4 + 8) of the warp's 16 rows

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i < kONTiles; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
  }

  // Q fragments of rows [row0, row0 + 16) of a swizzled [*, D] tile.
  __device__ __forceinline__ void load_q(uint32_t sQ, int row0, int lane) {
    const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int kk = 0; kk < kKSteps; ++kk) {
      const int row = row0 + ri + (mi & 1) * 8;
      const int chunk = kk * 2 + (mi >> 1);
      ldsm_x4(sQ + SwizzledTile<D>::offset(row, chunk), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }
  }

  // acc = Q K^T for the 64-key tile sK (swizzled [64, D]).
  __device__ __forceinline__ void scores(uint32_t sK, float (&acc)[kSNTiles][4], int lane) const {
#pragma unroll
    for (int j = 0; j < kSNTiles; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int jn = 0; jn < kSNTiles; jn += 2) {
#pragma unroll
      for (int kk = 0; kk < kKSteps; ++kk) {
        const int row = jn * 8 + ri + (mi >> 1) * 8;
        const int chunk = kk * 2 + (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + SwizzledTile<D>::offset(row, chunk), b0, b1, b2, b3);
        mma_16816(acc[jn], qf[kk], b0, b1);
        mma_16816(acc[jn + 1], qf[kk], b2, b3);
      }
    }
  }

  // Online-softmax update with the tile's logits.  key_ok(col) says whether key
  // column col of the tile takes part.  On return acc holds p = exp2(x - m_new)
  // and, when PAGE > 0, page_sum[pi][r] holds the sum of p over the PAGE columns
  // of page pi of the tile for row r (0: lane/4, 1: lane/4 + 8), full across
  // the quad.  m_out[r] receives m_new.
  template <int PAGE, class KeyOk>
  __device__ __forceinline__ void softmax_update(float (&acc)[kSNTiles][4], float sl2,
                                                 KeyOk key_ok, int lane,
                                                 float (*page_sum)[2], float (&m_out)[2]) {
    const int cq = 2 * (lane & 3);
    float mt[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < kSNTiles; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = j * 8 + cq + (e & 1);
        const float x = key_ok(col) ? acc[j][e] * sl2 : -INFINITY;
        acc[j][e] = x;
        mt[e >> 1] = fmaxf(mt[e >> 1], x);
      }
    }
    float alpha[2], mu[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mt[r] = fmaxf(mt[r], __shfl_xor_sync(0xffffffffu, mt[r], 1));
      mt[r] = fmaxf(mt[r], __shfl_xor_sync(0xffffffffu, mt[r], 2));
      const float mn = fmaxf(m[r], mt[r]);
      mu[r] = (mn == -INFINITY) ? 0.f : mn;  // a fully masked row keeps p = 0
      alpha[r] = fast_exp2(m[r] - mu[r]);
      m[r] = mn;
      m_out[r] = mn;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kSNTiles; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = fast_exp2(acc[j][e] - mu[e >> 1]);
        acc[j][e] = p;
        rs[e >> 1] += p;
      }
    }
    if constexpr (PAGE > 0) {
      constexpr int kPages = kKeyTile / PAGE;
      constexpr int kTilesPerPage = PAGE / 8;
#pragma unroll
      for (int pi = 0; pi < kPages; ++pi) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float v = 0.f;
#pragma unroll
          for (int j = pi * kTilesPerPage; j < (pi + 1) * kTilesPerPage; ++j)
            v += acc[j][2 * r] + acc[j][2 * r + 1];
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          page_sum[pi][r] = v;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 1);
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 2);
      l[r] = l[r] * alpha[r] + rs[r];
    }
#pragma unroll
    for (int i = 0; i < kONTiles; ++i) {
      o[i][0] *= alpha[0];
      o[i][1] *= alpha[0];
      o[i][2] *= alpha[1];
      o[i][3] *= alpha[1];
    }
  }

  // o += P V for the tile sV (swizzled [64, D]); p comes from softmax_update.
  __device__ __forceinline__ void pv(uint32_t sV, const float (&p)[kSNTiles][4], int lane) {
    const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int kk = 0; kk < kKeyTile / 16; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16x2(p[2 * kk][0], p[2 * kk][1]);
      a[1] = pack_bf16x2(p[2 * kk][2], p[2 * kk][3]);
      a[2] = pack_bf16x2(p[2 * kk + 1][0], p[2 * kk + 1][1]);
      a[3] = pack_bf16x2(p[2 * kk + 1][2], p[2 * kk + 1][3]);
#pragma unroll
      for (int dn = 0; dn < kONTiles; dn += 2) {
        const int row = kk * 16 + ri + (mi & 1) * 8;
        const int chunk = dn + (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + SwizzledTile<D>::offset(row, chunk), b0, b1, b2, b3);
        mma_16816(o[dn], a, b0, b1);
        mma_16816(o[dn + 1], a, b2, b3);
      }
    }
  }
};

}  // namespace dsa
