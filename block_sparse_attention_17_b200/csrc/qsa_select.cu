// Block pooling, indexer scoring and top-k selection (sm_100a).
//
// Pooling: kbar[j] = (1/B) sum_{i<B} ik[jB+i] for complete blocks (instagit MTPLX
// page, "Qwen Sparse Attention (QSA)": mean-pooled key blocks).
//
// Score: s[j] = c * sum_h w[h] * relu(iq[h] . kbar[j]) over complete visible
// blocks (llama.cpp PR #27739 page, QSA composition commit: per-head weights,
// n_head_scale 1, c = idx_dim^-0.5, window end kv_len / ratio).
//
// Top-k: the k = budget/B largest scores under (score desc, block index asc),
// written in ascending block order, followed by the tail block when the
// query's visible length is not a multiple of B (dev.to page, "Qwen Sparse
// Attention": the trailing incomplete block is always kept).
#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {

// ----------------------------------------------------------------- pooling
// One CTA of 256 threads pools one block: warp w sums rows w, w + 8, ... of
// the block (coalesced rows; lane l owns dims 2l and 2l + 1) in ascending
// order, then the 8 partial sums are combined in a fixed tree
// ((p0 + p1) + (p2 + p3)) + ((p4 + p5) + (p6 + p7)) and scaled by 1/B (B is a
// power of two). The prefill pooling, the incremental decode finalisation and
// the cache rebuild all call this one function, so they write identical bits.
constexpr int kPoolThreads = 256;

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

template <typename T>
__device__ __forceinline__ void pool_block_cta(const T* __restrict__ rows, int B, int di,
                                               float* __restrict__ dst) {
  __shared__ float2 part[8][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool active = 2 * lane < di;
  float2 acc = make_float2(0.f, 0.f);
  if (active) {
#pragma unroll 4
    for (int i = warp; i < B; i += 8) {
      const float2 x = load_pair<T>(rows + (size_t)i * di + 2 * lane);
      acc.x += x.x;
      acc.y += x.y;
    }
  }
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && active) {
    float2 q[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) q[w] = part[w][lane];
    const float inv = 1.0f / (float)B;
    const float sx = ((q[0].x + q[1].x) + (q[2].x + q[3].x)) + ((q[4].x + q[5].x) + (q[6].x + q[7].x));
    const float sy = ((q[0].y + q[1].y) + (q[2].y + q[3].y)) + ((q[4].y + q[5].y) + (q[6].y + q[7].y));
    *reinterpret_cast<float2*>(dst + 2 * lane) = make_float2(sx * inv, sy * inv);
  }
}

// Grid (blocks of the longest sequence, batch).
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
pool_prefill_kernel(const T* __restrict__ ik, const int* __restrict__ cu, int B, int di,
                    float* __restrict__ pooled, int max_nblk) {
  const int b = blockIdx.y, j = blockIdx.x;
  const int s0 = cu[b], L = cu[b + 1] - s0;
  if (j >= L / B) return;
  pool_block_cta(ik + ((size_t)s0 + (size_t)j * B) * di, B, di,
                 pooled + ((size_t)b * max_nblk + j) * di);
}

// mode 0: rebuild every complete block; mode 1: only the blocks completed by
// the last n_q appended rows. Grid (blocks in range, batch).
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
pool_cache_kernel(const T* __restrict__ ik_cache, const int* __restrict__ kv_len, int cap,
                  int n_q, int mode, int B, int di, float* __restrict__ pooled, int* dev_err) {
  const int b = blockIdx.y;
  const int kv = kv_len[b];
  if (kv < (mode ? n_q : 0) || kv > cap) {
    if (dev_err && threadIdx.x == 0 && blockIdx.x == 0) atomicExch(dev_err, 1);
    return;
  }
  const int jlo = mode ? (kv - n_q) / B : 0;
  const int j = jlo + blockIdx.x;
  if (j >= kv / B) return;
  pool_block_cta(ik_cache + ((size_t)b * cap + (size_t)j * B) * di, B, di,
                 pooled + ((size_t)b * (cap / B) + j) * di);
}

// ----------------------------------------------------------------- scoring
constexpr int kChunk = 64;   // pooled rows staged in shared memory at a time

// Score of pooled row `row` (kDI floats, padded stride) for one query whose
// indexer q (Hi x kDI, fp32) and weights sit in shared memory.
template <int kDI>
__device__ __forceinline__ float score_row(const float* __restrict__ krow,
                                           const float* __restrict__ iq_s,
                                           const float* __restrict__ iw_s, int Hi,
                                           float c) {
  float kv[kDI];
#pragma unroll
  for (int d = 0; d < kDI; ++d) kv[d] = krow[d];
  float s = 0.f;
  for (int h = 0; h < Hi; ++h) {
    const float4* qh = reinterpret_cast<const float4*>(iq_s + h * kDI);
    float dot = 0.f;
#pragma unroll
    for (int d4 = 0; d4 < kDI / 4; ++d4) {
      const float4 qv = qh[d4];
      dot = fmaf(qv.x, kv[4 * d4 + 0], dot);
      dot = fmaf(qv.y, kv[4 * d4 + 1], dot);
      dot = fmaf(qv.z, kv[4 * d4 + 2], dot);
      dot = fmaf(qv.w, kv[4 * d4 + 3], dot);
    }
    s = fmaf(iw_s[h], fmaxf(dot, 0.f), s);
  }
  return s * c;
}

// ----------------------------------------------------------------- top-k
__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Warp-cooperative selection of the k largest keys among keys[0..n) where a
// lower position wins a tie. Writes the chosen positions, ascending, to out[]
// and returns how many (min(k, n)). The k-th largest key is found by an
// MSB-first bit search on the 32-bit key; ties at that key are taken in
// ascending position order.
__device__ int warp_topk_positions(const uint32_t* keys, int n, int k, int* out, int lane) {
  if (n <= k) {
    for (int j = lane; j < n; j += 32) out[j] = j;
    __syncwarp();
    return n;
  }
  uint32_t tau = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = tau | (1u << bit);
    int c = 0;
    for (int j = lane; j < n; j += 32) c += keys[j] >= cand;
    c = __reduce_add_sync(kFull, c);
    if (c >= k) tau = cand;
  }
  int gt = 0;
  for (int j = lane; j < n; j += 32) gt += keys[j] > tau;
  gt = __reduce_add_sync(kFull, gt);
  const int need = k - gt;
  const unsigned lt = lanemask_lt();
  int m = 0, ties = 0;
  for (int base = 0; base < n; base += 32) {
    const int j = base + lane;
    const uint32_t key = j < n ? keys[j] : 0u;
    const bool tie = j < n && key == tau;
    const unsigned tb = __ballot_sync(kFull, tie);
    const bool pick = j < n && (key > tau || (tie && ties + __popc(tb & lt) < need));
    const unsigned pb = __ballot_sync(kFull, pick);
    if (pick) out[m + __popc(pb & lt)] = j;
    m += __popc(pb);
    ties += __popc(tb);
  }
  __syncwarp();
  return m;
}

// ------------------------------------------------- prefill: score + top-k
// Grid (ceil(max_seqlen / 8), batch); 8 warps, one query token per warp.
// Dynamic shared memory: kbar chunk [64][kDI+1], iq [8][Hi][kDI], iw [8][Hi],
// keys [8][nc_cap], positions [8][k].
template <typename T, int kDI>
__global__ void __launch_bounds__(256)
select_prefill_kernel(Geom g, const int* __restrict__ cu, int max_nblk, int words,
                      const T* __restrict__ iq, const float* __restrict__ iw,
                      const float* __restrict__ pooled, int nc_cap,
                      int* __restrict__ sel, int* __restrict__ nsel,
                      uint32_t* __restrict__ bitmask, float* __restrict__ scores,
                      int scores_ld) {
  extern __shared__ __align__(16) float smem[];
  constexpr int kStride = kDI + 1;
  float* kbar_s = smem;                               // kChunk * kStride
  float* iq_s = kbar_s + kChunk * kStride;            // 8 * Hi * kDI
  float* iw_s = iq_s + 8 * g.Hi * kDI;                // 8 * Hi
  uint32_t* keys_s = reinterpret_cast<uint32_t*>(iw_s + 8 * g.Hi);   // 8 * nc_cap
  int* pos_s = reinterpret_cast<int*>(keys_s + 8 * nc_cap);          // 8 * k

  const int b = blockIdx.y;
  const int s0 = cu[b], L = cu[b + 1] - s0;
  const int p0 = blockIdx.x * 8;
  if (p0 >= L) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = p0 + warp;
  const bool valid = p < L;
  const int n = p + 1;
  const int nc = valid ? n / g.B : 0;
  const size_t t = (size_t)s0 + p;

  float* my_iq = iq_s + warp * g.Hi * kDI;
  float* my_iw = iw_s + warp * g.Hi;
  for (int e = lane; e < g.Hi * kDI; e += 32)
    my_iq[e] = valid ? to_f32(iq[t * g.Hi * kDI + e]) : 0.f;
  for (int e = lane; e < g.Hi; e += 32) my_iw[e] = valid ? iw[t * g.Hi + e] : 0.f;

  uint32_t* my_keys = keys_s + warp * nc_cap;
  const int last = min(p0 + 8, L);          // one past the CTA's last valid position
  const int nc_cta = last / g.B;            // candidates of the CTA's last query
  const float* pooled_b = pooled + (size_t)b * max_nblk * kDI;

  for (int c0 = 0; c0 < nc_cta; c0 += kChunk) {
    const int rows = min(kChunk, nc_cta - c0);
    __syncthreads();
    for (int e = threadIdx.x; e < rows * kDI; e += blockDim.x) {
      const int r = e / kDI, d = e - r * kDI;
      kbar_s[r * kStride + d] = pooled_b[(size_t)(c0 + r) * kDI + d];
    }
    __syncthreads();
    for (int r = lane; r < rows; r += 32) {
      const int j = c0 + r;
      if (j < nc) {
        const float s = score_row<kDI>(kbar_s + r * kStride, my_iq, my_iw, g.Hi, g.idx_scale);
        my_keys[j] = score_key(s);
        if (scores) scores[t * scores_ld + j] = s;
      }
    }
  }
  __syncwarp();
  if (!valid) return;
  if (scores)
    for (int j = nc + lane; j < scores_ld; j += 32) scores[t * scores_ld + j] = -INFINITY;

  int* my_pos = pos_s + warp * g.k;
  const int m = warp_topk_positions(my_keys, nc, g.k, my_pos, lane);
  const int tail = n - nc * g.B;
  const int cnt = m + (tail > 0 ? 1 : 0);
  int* srow = sel + t * (g.k + 1);
  for (int e = lane; e < g.k + 1; e += 32) {
    int v = -1;
    if (e < m) v = my_pos[e];
    else if (e == m && tail > 0) v = nc;
    srow[e] = v;
  }
  if (lane == 0) nsel[t] = cnt;
  if (bitmask) {
    uint32_t* brow = bitmask + t * words;
    for (int w = lane; w < words; w += 32) brow[w] = 0u;
    __syncwarp();
    for (int e = lane; e < m; e += 32) atomicOr(&brow[my_pos[e] >> 5], 1u << (my_pos[e] & 31));
    if (lane == 0 && tail > 0) atomicOr(&brow[nc >> 5], 1u << (nc & 31));
  }
}

// -------------------------------------------------------- decode: scoring
// Grid (ceil(cap/B / 64), batch); 128 threads. Each CTA stages 64 pooled rows
// once and scores them for every new query of its sequence.
template <typename T, int kDI>
__global__ void __launch_bounds__(128)
decode_score_kernel(Geom g, int n_q, int cap, const int* __restrict__ kv_len,
                    const T* __restrict__ iq, const float* __restrict__ iw,
                    const float* __restrict__ pooled, float* __restrict__ scores) {
  extern __shared__ __align__(16) float smem[];
  constexpr int kStride = kDI + 1;
  float* kbar_s = smem;
  float* iq_s = kbar_s + kChunk * kStride;            // n_q * Hi * kDI
  float* iw_s = iq_s + n_q * g.Hi * kDI;              // n_q * Hi
  const int b = blockIdx.y;
  const int kv = kv_len[b];
  const int nblk_cap = cap / g.B;
  if (kv < n_q || kv > cap) return;
  const int nc_max = kv / g.B;                        // candidates of the last query
  const int c0 = blockIdx.x * kChunk;
  if (c0 >= nblk_cap) return;
  float* srow_b = scores + (size_t)b * n_q * nblk_cap;
  for (int e = threadIdx.x; e < n_q * g.Hi * kDI; e += blockDim.x)
    iq_s[e] = to_f32(iq[(size_t)b * n_q * g.Hi * kDI + e]);
  for (int e = threadIdx.x; e < n_q * g.Hi; e += blockDim.x)
    iw_s[e] = iw[(size_t)b * n_q * g.Hi + e];
  const int rows = max(0, min(kChunk, nc_max - c0));
  const float* src = pooled + ((size_t)b * nblk_cap + c0) * kDI;
  for (int e = threadIdx.x; e < rows * kDI; e += blockDim.x) {
    const int r = e / kDI, d = e - r * kDI;
    kbar_s[r * kStride + d] = src[(size_t)r * kDI + d];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n_q * kChunk; e += blockDim.x) {
    const int i = e / kChunk, r = e - i * kChunk;
    const int j = c0 + r;
    if (j >= nblk_cap) continue;
    const int n = kv - n_q + 1 + i;
    float s = -INFINITY;
    if (j < n / g.B)
      s = score_row<kDI>(kbar_s + r * kStride, iq_s + i * g.Hi * kDI, iw_s + i * g.Hi,
                         g.Hi, g.idx_scale);
    srow_b[(size_t)i * nblk_cap + j] = s;
  }
}

// --------------------------------------------------------- decode: top-k
// Grid (n_q, batch); 256 threads. Each warp takes the top-k of a contiguous
// slice of candidates (positions come out ascending, so concatenating the
// warps' picks keeps ascending block order); warp 0 then takes the top-k of
// the concatenation, where a lower position is a lower block index.
__global__ void __launch_bounds__(256)
decode_topk_kernel(Geom g, int n_q, int cap, const int* __restrict__ kv_len,
                   const float* __restrict__ scores, int* __restrict__ sel,
                   int* __restrict__ nsel, float* __restrict__ scores_out) {
  extern __shared__ __align__(16) uint32_t usmem[];
  const int nblk_cap = cap / g.B;
  uint32_t* keys = usmem;                                  // nblk_cap
  uint32_t* ckeys = keys + nblk_cap;                       // 8 * k
  int* cidx = reinterpret_cast<int*>(ckeys + 8 * g.k);     // 8 * k
  int* cpos = cidx + 8 * g.k;                              // 8 * k (per-warp scratch)
  __shared__ int cnt_w[8];
  const int i = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kv = kv_len[b];
  int* srow = sel + ((size_t)b * n_q + i) * (g.k + 1);
  if (kv < n_q || kv > cap) {
    for (int e = threadIdx.x; e < g.k + 1; e += blockDim.x) srow[e] = -1;
    if (threadIdx.x == 0) nsel[(size_t)b * n_q + i] = 0;
    return;
  }
  const int n = kv - n_q + 1 + i;
  const int nc = n / g.B;
  const float* s = scores + ((size_t)b * n_q + i) * nblk_cap;
  for (int j = threadIdx.x; j < nc; j += blockDim.x) keys[j] = score_key(s[j]);
  if (scores_out)
    for (int j = threadIdx.x; j < nblk_cap; j += blockDim.x)
      scores_out[((size_t)b * n_q + i) * nblk_cap + j] = j < nc ? s[j] : -INFINITY;
  __syncthreads();
  const int per = (nc + 7) / 8;
  const int lo = min(nc, warp * per), hi = min(nc, lo + per);
  int* wpos = cpos + warp * g.k;
  const int mw = warp_topk_positions(keys + lo, hi - lo, g.k, wpos, lane);
  if (lane == 0) cnt_w[warp] = mw;
  __syncthreads();
  int off = 0;
  for (int w = 0; w < warp; ++w) off += cnt_w[w];
  for (int e = lane; e < mw; e += 32) {
    ckeys[off + e] = keys[lo + wpos[e]];
    cidx[off + e] = lo + wpos[e];
  }
  __syncthreads();
  if (warp != 0) return;
  int total = 0;
  for (int w = 0; w < 8; ++w) total += cnt_w[w];
  int* fpos = cpos;   // reuse warp 0's slot (the first k entries)
  const int m = warp_topk_positions(ckeys, total, g.k, fpos, lane);
  const int tail = n - nc * g.B;
  for (int e = lane; e < g.k + 1; e += 32) {
    int v = -1;
    if (e < m) v = cidx[fpos[e]];
    else if (e == m && tail > 0) v = nc;
    srow[e] = v;
  }
  if (lane == 0) nsel[(size_t)b * n_q + i] = m + (tail > 0 ? 1 : 0);
}

// ------------------------------------------------------------ launchers
template <typename T>
static cudaError_t launch_pool_prefill_t(const void* ik, const int* cu, int batch, int max_seqlen,
                                         int B, int di, float* pooled, int max_nblk,
                                         cudaStream_t st) {
  const int nblk = max_seqlen / B;
  if (nblk == 0 || batch == 0) return cudaSuccess;
  pool_prefill_kernel<T><<<dim3(nblk, batch), kPoolThreads, 0, st>>>((const T*)ik, cu, B, di,
                                                                     pooled, max_nblk);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_pool_prefill(qsa_dtype dt, const void* ik, const int* cu, int batch,
                                int max_seqlen, int B, int di, float* pooled, int max_nblk,
                                cudaStream_t st) {
  return dt == QSA_BF16
             ? launch_pool_prefill_t<__nv_bfloat16>(ik, cu, batch, max_seqlen, B, di, pooled,
                                                    max_nblk, st)
             : launch_pool_prefill_t<float>(ik, cu, batch, max_seqlen, B, di, pooled, max_nblk, st);
}

cudaError_t launch_pool_cache(qsa_dtype dt, const void* ik_cache, const int* kv_len, int batch,
                              int cap, int n_q, int mode, int B, int di, float* pooled,
                              int* dev_err, cudaStream_t st) {
  const int span = mode ? (n_q + B - 1) / B + 1 : cap / B;
  if (batch == 0 || span == 0) return cudaSuccess;
  dim3 grid(span, batch);
  if (dt == QSA_BF16)
    pool_cache_kernel<__nv_bfloat16><<<grid, kPoolThreads, 0, st>>>(
        (const __nv_bfloat16*)ik_cache, kv_len, cap, n_q, mode, B, di, pooled, dev_err);
  else
    pool_cache_kernel<float><<<grid, kPoolThreads, 0, st>>>((const float*)ik_cache, kv_len, cap,
                                                            n_q, mode, B, di, pooled, dev_err);
  note_launch();
  return cudaGetLastError();
}

size_t select_prefill_smem(const Geom& g, int nc_cap) {
  return sizeof(float) * ((size_t)kChunk * (g.di + 1) + 8 * g.Hi * g.di + 8 * g.Hi) +
         sizeof(uint32_t) * 8 * (size_t)nc_cap + sizeof(int) * 8 * (size_t)g.k;
}

template <typename T, int kDI>
static cudaError_t launch_select_prefill_t(const Geom& g, const int* cu, int batch,
                                           int max_seqlen, int max_nblk, int words,
                                           const void* iq, const float* iw, const float* pooled,
                                           int* sel, int* nsel, uint32_t* bitmask,
                                           float* scores, int scores_ld, cudaStream_t st) {
  const int nc_cap = max(1, max_seqlen / g.B);
  const size_t smem = select_prefill_smem(g, nc_cap);
  auto kern = select_prefill_kernel<T, kDI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((max_seqlen + 7) / 8, batch);
  kern<<<grid, 256, smem, st>>>(g, cu, max_nblk, words, (const T*)iq, iw, pooled, nc_cap, sel,
                                nsel, bitmask, scores, scores_ld);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_select_prefill(qsa_dtype dt, const Geom& g, const int* cu, int batch,
                                  int max_seqlen, int max_nblk, int words, const void* iq,
                                  const float* iw, const float* pooled, int* sel, int* nsel,
                                  uint32_t* bitmask, float* scores, int scores_ld,
                                  cudaStream_t st) {
  if (batch == 0 || max_seqlen == 0) return cudaSuccess;
#define QSA_SEL(T, DI)                                                                      \
  return launch_select_prefill_t<T, DI>(g, cu, batch, max_seqlen, max_nblk, words, iq, iw,  \
                                        pooled, sel, nsel, bitmask, scores, scores_ld, st)
  if (dt == QSA_BF16) {
    if (g.di == 64) QSA_SEL(__nv_bfloat16, 64);
    QSA_SEL(__nv_bfloat16, 32);
  } else {
    if (g.di == 64) QSA_SEL(float, 64);
    QSA_SEL(float, 32);
  }
#undef QSA_SEL
}

template <typename T, int kDI>
static cudaError_t launch_decode_score_t(const Geom& g, int batch, int n_q, int cap,
                                         const int* kv_len, const void* iq, const float* iw,
                                         const float* pooled, float* scores, cudaStream_t st) {
  const int nblk_cap = cap / g.B;
  const size_t smem =
      sizeof(float) * ((size_t)kChunk * (kDI + 1) + (size_t)n_q * g.Hi * kDI + n_q * g.Hi);
  auto kern = decode_score_kernel<T, kDI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((nblk_cap + kChunk - 1) / kChunk, batch);
  kern<<<grid, 128, smem, st>>>(g, n_q, cap, kv_len, (const T*)iq, iw, pooled, scores);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_decode_select(qsa_dtype dt, const Geom& g, int batch, int n_q, int cap,
                                 const int* kv_len, const void* iq, const float* iw,
                                 const float* pooled, float* scores_ws, int* sel, int* nsel,
                                 float* scores_out, cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
  cudaError_t e;
#define QSA_DS(T, DI) \
  e = launch_decode_score_t<T, DI>(g, batch, n_q, cap, kv_len, iq, iw, pooled, scores_ws, st)
  if (dt == QSA_BF16) {
    if (g.di == 64) QSA_DS(__nv_bfloat16, 64); else QSA_DS(__nv_bfloat16, 32);
  } else {
    if (g.di == 64) QSA_DS(float, 64); else QSA_DS(float, 32);
  }
#undef QSA_DS
  if (e != cudaSuccess) return e;
  const int nblk_cap = cap / g.B;
  const size_t smem = sizeof(uint32_t) * ((size_t)nblk_cap + 3 * 8 * g.k);
  e = cudaFuncSetAttribute(decode_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  decode_topk_kernel<<<dim3(n_q, batch), 256, smem, st>>>(g, n_q, cap, kv_len, scores_ws, sel,
                                                          nsel, scores_out);
  note_launch();
  return cudaGetLastError();
}

}  // namespace qsa
