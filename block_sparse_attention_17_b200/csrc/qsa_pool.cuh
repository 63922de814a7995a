// Mean pooling of one B-row block of indexer keys (instagit MTPLX page, "Qwen
// Sparse Attention (QSA)": each block is represented by the mean of its keys).
// Every kernel that pools calls pool_block(), so the prefill pooling, the
// incremental decode finalisation and the cache rebuild write identical bits.
#pragma once

#include "qsa_common.cuh"

namespace qsa {

// Warp 0's last step of a pooling: the eight partial sums of lane l's dims
// (2l, 2l + 1) combined in a fixed tree, scaled by 1/B, turned by the indexer
// rotary embedding when rope_dim > 0, and stored (lanes with active set).
__device__ __forceinline__ void pool_finish(float2 (*part)[32], int lane, bool active, int B,
                                            float* dst, int rope_dim, float rope_theta, int pos) {
  float sx = 0.f, sy = 0.f;
  if (active) {
    float2 q[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) q[w] = part[w][lane];
    const float inv = 1.0f / (float)B;
    sx = (((q[0].x + q[1].x) + (q[2].x + q[3].x)) + ((q[4].x + q[5].x) + (q[6].x + q[7].x))) * inv;
    sy = (((q[0].y + q[1].y) + (q[2].y + q[3].y)) + ((q[4].y + q[5].y) + (q[6].y + q[7].y))) * inv;
  }
  if (rope_dim > 0) rope_lane_pair(sx, sy, lane, pos, rope_dim, rope_theta);
  if (active) *reinterpret_cast<float2*>(dst + 2 * lane) = make_float2(sx, sy);
}

template <typename T>
__device__ __forceinline__ float2 load_pair(const T* p);
template <>
__device__ __forceinline__ float2 load_pair<float>(const float* p) {
  return *reinterpret_cast<const float2*>(p);
}
template <>
__device__ __forceinline__ float2 load_pair<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// Pools rows[0 .. B) (di <= 64 dims each) into dst[0 .. di) with the whole CTA
// (nwarps warps, all threads call it). The order of the sums is fixed whatever
// nwarps is: eight partial sums, partial v over rows v, v + 8, v + 16, ... in
// ascending order (lane l owns dims 2l and 2l + 1), combined in the tree
// ((p0 + p1) + (p2 + p3)) + ((p4 + p5) + (p6 + p7)) and scaled by 1/B (B is a
// power of two). With rope_dim > 0 the mean is then turned at position `pos`
// (the block's first token) by rope_lane_pair. Rows r >= split come from
// new_rows[r - split] instead of rows[r] (a block completed by rows that are
// not in the cache yet); the sums are the same. part: 8 x 32 float2 of shared
// memory.
template <typename T>
__device__ __forceinline__ void pool_block(const T* __restrict__ rows, int B, int di,
                                           float* dst, float2 (*part)[32], int nwarps,
                                           int rope_dim = 0, float rope_theta = 0.f, int pos = 0,
                                           const T* __restrict__ new_rows = nullptr,
                                           int split = 1 << 30) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool active = 2 * lane < di;
  for (int v = warp; v < 8; v += nwarps) {
    float2 acc = make_float2(0.f, 0.f);
    if (active) {
      for (int i0 = v; i0 < B; i0 += 64) {   // eight rows' loads in flight, then their sums in order
        float2 x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          x[u] = i0 + 8 * u < B
                     ? load_pair<T>((i0 + 8 * u < split ? rows + (size_t)(i0 + 8 * u) * di
                                                        : new_rows + (size_t)(i0 + 8 * u - split) * di) +
                                    2 * lane)
                     : make_float2(0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (i0 + 8 * u < B) {
            acc.x += x[u].x;
            acc.y += x[u].y;
          }
      }
    }
    part[v][lane] = acc;
  }
  __syncthreads();
  if (warp == 0) pool_finish(part, lane, active, B, dst, rope_dim, rope_theta, pos);
}

}  // namespace qsa

namespace qsa {

// pool_block for a CTA of at least four warps and kDI = 32 or 64, in one round:
// half-warp v of warps 0-3 sums partial v (lane l' of it owns dims
// [kDI/16 * l', kDI/16 * (l' + 1))), with the same rows, order and final tree
// as pool_block, so both write identical bits.
template <typename T, int kDI>
__device__ __forceinline__ void pool_block_halves(const T* __restrict__ rows, int B, float* dst,
                                                  float2 (*part)[32], int rope_dim = 0,
                                                  float rope_theta = 0.f, int pos = 0) {
  static_assert(kDI == 32 || kDI == 64, "indexer dim");
  constexpr int kPer = kDI / 16;                  // dims per lane: 2 or 4
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < 4) {
    const int v = 2 * warp + (lane >> 4), l = lane & 15;
    float acc[kPer];
#pragma unroll
    for (int d = 0; d < kPer; ++d) acc[d] = 0.f;
    for (int i0 = v; i0 < B; i0 += 64) {   // eight rows in flight, then their sums in order
      float x[8][kPer];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int r = i0 + 8 * u;
#pragma unroll
        for (int d = 0; d < kPer; d += 2) {
          const float2 p = r < B ? load_pair<T>(rows + (size_t)r * kDI + kPer * l + d) : make_float2(0.f, 0.f);
          x[u][d] = p.x;
          x[u][d + 1] = p.y;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (i0 + 8 * u < B)
#pragma unroll
          for (int d = 0; d < kPer; ++d) acc[d] += x[u][d];
    }
#pragma unroll
    for (int d = 0; d < kPer; d += 2) part[v][(kPer * l + d) / 2] = make_float2(acc[d], acc[d + 1]);
  }
  __syncthreads();
  if (warp == 0) pool_finish(part, lane, 2 * lane < kDI, B, dst, rope_dim, rope_theta, pos);
}

}  // namespace qsa
