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

// Geometry passed by value to every kernel.
struct Geom {
  int Hq, Hkv, G, D;
  int Hi, di;
  int B, k;
  float sm_scale_log2;   // softmax_scale * log2(e)
  float idx_scale;
  int gate_headwise;
};

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

// 1 / (1 + e^-x) with the fast exponential and division (a few ulp; 0 for
// very negative x).
__device__ __forceinline__ float sigmoidf_(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

}  // namespace qsa
