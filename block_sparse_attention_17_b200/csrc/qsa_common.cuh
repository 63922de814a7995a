// Shared device helpers for the QSA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qsa.h"

namespace qsa {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxTopK = 64;          // budget / block_size
constexpr int kMaxBlocksPerSeq = 4096;        // prefill
constexpr int kMaxDecodeBlocksPerSeq = 16384; // decode cache blocks (cap / B)

// Geometry (and the per-call debug counter) passed by value to every kernel.
struct Geom {
  int Hq, Hkv, G, D;
  int Hi, di;
  int B, k;
  float sm_scale_log2;   // softmax_scale * log2(e)
  float idx_scale;
  int gate_headwise;
  int rope_dim;         // indexer rotary embedding: dims rotated (0 = none)
  float rope_theta;
  unsigned long long* keys_visited;   // debug: (query, head, key) triples attended, or null
};

// Adds a warp's per-lane counts to the visited-keys counter (every lane calls it).
__device__ __forceinline__ void add_keys_visited(unsigned long long* ctr, unsigned v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0 && v) atomicAdd(ctr, (unsigned long long)v);
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Maps a score to an unsigned key whose integer order is the float order;
// -0 and +0 get the same key (a tie, broken by block index).
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The score a key came from (score_key's inverse; a -0 score comes back as +0).
__device__ __forceinline__ float key_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Programmatic dependent launch: a kernel launched with launch_dependent()
// may start while the kernel before it on the stream still runs; it calls
// grid_dependency_wait() before reading anything that kernel wrote. A kernel
// calls grid_dependents_launch() once the next kernel may start.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Indexer rotary embedding (llama.cpp PR #27739 page, QSA block-composition
// commit text: the indexer scores the roped query against pooled keys that
// take the same rope angles; instagit MTPLX page, "Multidimensional Rotary
// Embeddings (M-RoPE)": for text, the ordinary partial rotary embedding).
// Frequency f < rope_dim / 2 turns the pair (x[f], x[f + rope_dim / 2]) by the
// fp32 product of the position and fp32(theta^(-2f / rope_dim)); the power is
// taken in double precision so that its fp32 rounding is the correct one. The
// rotary helpers are kept out of line: the kernels that carry them run them
// only when rope_dim > 0, and their code stays out of the hot paths' fetch.
static __device__ __noinline__ float2 rope_cos_sin(int f, int pos, int rope_dim, float theta) {
  const float inv = (float)pow((double)theta, -2.0 * f / rope_dim);
  const float a = __fmul_rn((float)pos, inv);
  float s, c;
  sincosf(a, &s, &c);
  return make_float2(c, s);
}

// (lo, hi) -> (lo c - hi s, hi c + lo s), with the same roundings at every site.
__device__ __forceinline__ void rope_turn(float& lo, float& hi, float2 cs) {
  const float l = __fmaf_rn(lo, cs.x, -__fmul_rn(hi, cs.y));
  const float h = __fmaf_rn(hi, cs.x, __fmul_rn(lo, cs.y));
  lo = l;
  hi = h;
}

// Rotates nrows rows of shared memory in place: row r starts at base + r *
// stride and belongs to query r / per_q, whose position is pos0 + r / per_q.
// All threads of the CTA call it (tid, nthr); the caller synchronises around it.
static __device__ __noinline__ void rope_rows(float* base, int nrows, int per_q, int stride, int pos0,
                                          int rope_dim, float theta, int tid, int nthr) {
  const int hp = rope_dim >> 1;
  for (int e = tid; e < nrows * hp; e += nthr) {
    const int r = e / hp, f = e - r * hp;
    float* x = base + (size_t)r * stride;
    rope_turn(x[f], x[f + hp], rope_cos_sin(f, pos0 + r / per_q, rope_dim, theta));
  }
}

// One warp holds a row two dims per lane (lane l: dims 2l and 2l + 1, as x and
// y); turns its first rope_dim dims (rope_dim a multiple of 4) at `pos` with
// rope_turn's roundings. Every lane of the warp calls it.
static __device__ __noinline__ void rope_lane_pair(float& x, float& y, int lane, int pos, int rope_dim,
                                               float theta) {
  const int qo = rope_dim >> 2;                 // lanes holding the first half
  const bool in = lane < 2 * qo;
  const int src = !in ? lane : (lane < qo ? lane + qo : lane - qo);
  const float px = __shfl_sync(kFull, x, src), py = __shfl_sync(kFull, y, src);
  if (in) {
    const int f = 2 * (lane < qo ? lane : lane - qo);
    const float2 c0 = rope_cos_sin(f, pos, rope_dim, theta);
    const float2 c1 = rope_cos_sin(f + 1, pos, rope_dim, theta);
    if (lane < qo) {   // own dims are the pairs' first members
      x = __fmaf_rn(x, c0.x, -__fmul_rn(px, c0.y));
      y = __fmaf_rn(y, c1.x, -__fmul_rn(py, c1.y));
    } else {           // own dims are the second members
      x = __fmaf_rn(x, c0.x, __fmul_rn(px, c0.y));
      y = __fmaf_rn(y, c1.x, __fmul_rn(py, c1.y));
    }
  }
}

// 1 / (1 + e^-x) with the fast exponential and division (a few ulp; 0 for
// very negative x).
__device__ __forceinline__ float sigmoidf_(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

}  // namespace qsa
