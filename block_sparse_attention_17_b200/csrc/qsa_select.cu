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
// ascending position order. Up to 256 keys are held in registers (8 per
// lane) for the whole search; longer lists are re-read from memory.
__device__ int warp_topk_positions(const uint32_t* keys, int n, int k, int* out, int lane) {
  if (n <= k) {
    for (int j = lane; j < n; j += 32) out[j] = j;
    __syncwarp();
    return n;
  }
  const unsigned lt = lanemask_lt();
  if (n <= 256) {
    uint32_t kr[8];
    bool ok[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = lane + 32 * i;
      ok[i] = j < n;
      kr[i] = ok[i] ? keys[j] : 0u;
    }
    uint32_t tau = 0;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      int c = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) c += (ok[i] && kr[i] >= cand) ? 1 : 0;
      c = __reduce_add_sync(kFull, c);
      if (c >= k) tau = cand;
    }
    int gt = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) gt += (ok[i] && kr[i] > tau) ? 1 : 0;
    gt = __reduce_add_sync(kFull, gt);
    const int need = k - gt;
    int m = 0, ties = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool tie = ok[i] && kr[i] == tau;
      const unsigned tb = __ballot_sync(kFull, tie);
      const bool pick = ok[i] && (kr[i] > tau || (tie && ties + __popc(tb & lt) < need));
      const unsigned pb = __ballot_sync(kFull, pick);
      if (pick) out[m + __popc(pb & lt)] = lane + 32 * i;
      m += __popc(pb);
      ties += __popc(tb);
    }
    __syncwarp();
    return m;
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

// ------------------------------------------------------- CTA top-k
// The k largest of keys[0..n) (shared memory) where a lower position wins a
// tie, chosen by a whole CTA of 256 threads with few dependent steps: four
// 8-bit radix passes find the k-th largest key tau (a shared histogram per
// pass, lanes with equal digits adding once), then each thread counts the
// keys > tau and == tau in its contiguous run of positions, one block scan
// turns the counts into output offsets, and the chosen positions are written
// in ascending order. Returns min(k, n).
constexpr int kTopkThreads = 256;

__device__ int cta_topk_radix(const uint32_t* keys, int n, int k, int* out) {
  __shared__ int hist[256];
  __shared__ int scan_s[2][kTopkThreads / 32];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_need;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (n <= k) {
    for (int j = tid; j < n; j += kTopkThreads) out[j] = j;
    __syncthreads();
    return n;
  }
  if (tid == 0) { s_prefix = 0u; s_mask = 0u; s_need = k; }
  for (int shift = 24; shift >= 0; shift -= 8) {
    hist[tid] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int base = 0; base < n; base += kTopkThreads) {
      const int j = base + tid;
      const uint32_t key = j < n ? keys[j] : 0u;
      const bool live = j < n && (key & mask) == prefix;
      const uint32_t digit = live ? (key >> shift) & 255u : 256u;
      const unsigned same = __match_any_sync(kFull, digit);
      if (live && (__ffs(same) - 1) == lane) atomicAdd(&hist[digit], __popc(same));
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255 - 8l down to 248 - 8l
      int cnt[8], local = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        cnt[e] = hist[255 - 8 * lane - e];
        local += cnt[e];
      }
      int incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
      }
      const int need = s_need;
      const int before = incl - local;
      if (before < need && incl >= need) {
        int run = before;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (run + cnt[e] >= need) {
            s_prefix = prefix | ((uint32_t)(255 - 8 * lane - e) << shift);
            s_mask = mask | (255u << shift);
            s_need = need - run;
            break;
          }
          run += cnt[e];
        }
      }
    }
    __syncthreads();
  }
  const uint32_t tau = s_prefix;
  const int need = s_need;   // keys equal to tau to take, lowest positions first
  // each thread owns the contiguous run [lo, hi)
  const int per = (n + kTopkThreads - 1) / kTopkThreads;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int n_gt = 0, n_eq = 0;
  for (int j = lo; j < hi; ++j) {
    const uint32_t key = keys[j];
    n_gt += key > tau;
    n_eq += key == tau;
  }
  // exclusive scans of the tie counts and of the greater counts
  int ie = n_eq, ig = n_gt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(kFull, ie, o), b = __shfl_up_sync(kFull, ig, o);
    if (lane >= o) { ie += a; ig += b; }
  }
  if (lane == 31) { scan_s[0][warp] = ie; scan_s[1][warp] = ig; }
  __syncthreads();
  int eq_before = ie - n_eq, gt_before = ig - n_gt;
  for (int w = 0; w < warp; ++w) { eq_before += scan_s[0][w]; gt_before += scan_s[1][w]; }
  // ties before this run that are taken, plus greater keys before this run
  int o_idx = gt_before + min(eq_before, need);
  int t_rank = eq_before;
  for (int j = lo; j < hi; ++j) {
    const uint32_t key = keys[j];
    if (key > tau) {
      out[o_idx++] = j;
    } else if (key == tau) {
      if (t_rank < need) out[o_idx++] = j;
      ++t_rank;
    }
  }
  __syncthreads();
  return k;
}

// ------------------------------------------------ decode: fused selection
// Grid (ceil(cap/B / 64), batch); 256 threads (8 warps). CTA c owns candidate blocks
// [64c, 64c + 64) of sequence b and
//  1. pools the blocks of its range that this step's tokens complete (the
//     incremental pooled-key cache) and writes them to the cache,
//  2. scores its blocks for every new query of the sequence (one thread per
//     (block, indexer head), summed over the heads by shuffles) and publishes
//     the score keys,
//  3. the last CTA of the sequence to finish (an atomic counter that the
//     caller zeroes before the launch) selects each query's top-k from all
//     of them (cta_topk_radix), then appends the tail block.
constexpr int kSelThreads = 256;
constexpr int kPart = 64;                 // candidate blocks per CTA

template <typename T, int kDI>
__global__ void __launch_bounds__(kSelThreads)
decode_select_kernel(Geom g, int n_q, int cap, const int* __restrict__ kv_len,
                     const T* __restrict__ iq, const T* __restrict__ ik_cache,
                     const float* __restrict__ iw, float* __restrict__ pooled,
                     float* __restrict__ scores_out, uint32_t* __restrict__ keys_ws,
                     int* __restrict__ counter, int* __restrict__ sel, int* __restrict__ nsel,
                     int* dev_err) {
  extern __shared__ __align__(16) float smem[];
  constexpr int kStride = kDI + 1;
  const int k = g.k;
  const int nblk_cap = cap / g.B;
  float* kbar_s = smem;                                       // kPart * kStride
  float* iq_s = kbar_s + kPart * kStride;                     // n_q * Hi * kDI
  float* iw_s = iq_s + n_q * g.Hi * kDI;                      // n_q * Hi
  uint32_t* keys_s = reinterpret_cast<uint32_t*>(iw_s + n_q * g.Hi);   // nblk_cap (merge)
  int* pos_s = reinterpret_cast<int*>(keys_s + nblk_cap);             // k
  __shared__ int last_s;

  const int c = blockIdx.x, b = blockIdx.y;
  const int kv = kv_len[b];
  const int kp1 = k + 1;
  if (kv < n_q || kv > cap) {
    if (c == 0) {
      for (int e = threadIdx.x; e < n_q * kp1; e += blockDim.x) sel[(size_t)b * n_q * kp1 + e] = -1;
      for (int e = threadIdx.x; e < n_q; e += blockDim.x) nsel[(size_t)b * n_q + e] = 0;
      if (dev_err && threadIdx.x == 0) atomicExch(dev_err, 1);
    }
    return;
  }
  const int nc_last = kv / g.B;                    // candidates of the last query
  const int nparts = max(1, (nc_last + kPart - 1) / kPart);
  if (c >= nparts) return;
  const int j0 = c * kPart;
  const int rows = max(0, min(kPart, nc_last - j0));

  // 1. blocks completed by this step's tokens (pool_block_cta needs the whole CTA)
  const int jnew_lo = max((kv - n_q) / g.B, j0), jnew_hi = min(nc_last, j0 + kPart);
  for (int j = jnew_lo; j < jnew_hi; ++j) {
    pool_block_cta(ik_cache + ((size_t)b * cap + (size_t)j * g.B) * kDI, g.B, kDI,
                   pooled + ((size_t)b * nblk_cap + j) * kDI);
    __syncthreads();
  }
  // 2. stage the range's pooled rows and the queries' indexer q / weights
  {   // every load of the stage is issued before the first store
    const float* src = pooled + ((size_t)b * nblk_cap + j0) * kDI;
    constexpr int kPerThr = kPart * (kDI / 4) / kSelThreads;   // float4 per thread
    float4 v[kPerThr];
#pragma unroll
    for (int u = 0; u < kPerThr; ++u) {
      const int e = u * kSelThreads + threadIdx.x;
      const int r = e / (kDI / 4), d4 = e - r * (kDI / 4);
      v[u] = r < rows ? *reinterpret_cast<const float4*>(src + (size_t)r * kDI + 4 * d4)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int nq_e = n_q * g.Hi * kDI;
    const T* iqb = iq + (size_t)b * nq_e;
    float qv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = u * kSelThreads + threadIdx.x;
      qv[u] = e < nq_e ? to_f32(iqb[e]) : 0.f;
    }
    const float wv = threadIdx.x < n_q * g.Hi ? iw[(size_t)b * n_q * g.Hi + threadIdx.x] : 0.f;
    for (int e = 4 * kSelThreads + threadIdx.x; e < nq_e; e += kSelThreads)
      iq_s[e] = to_f32(iqb[e]);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = u * kSelThreads + threadIdx.x;
      if (e < nq_e) iq_s[e] = qv[u];
    }
    if (threadIdx.x < n_q * g.Hi) iw_s[threadIdx.x] = wv;
#pragma unroll
    for (int u = 0; u < kPerThr; ++u) {
      const int e = u * kSelThreads + threadIdx.x;
      const int r = e / (kDI / 4), d4 = e - r * (kDI / 4);
      float* dst = kbar_s + r * kStride + 4 * d4;
      dst[0] = v[u].x; dst[1] = v[u].y; dst[2] = v[u].z; dst[3] = v[u].w;
    }
  }
  __syncthreads();
  // scores: one (query, block, head) triple per thread; heads are adjacent
  // lanes (Hi divides 32), so the weighted relu terms are summed by shuffles
  const int per_q = kPart * g.Hi;
  for (int base = 0; base < n_q * per_q; base += blockDim.x) {
    const int e = base + threadIdx.x;
    const int i = e / per_q, rem = e - i * per_q;
    const int r = rem / g.Hi, h = rem - r * g.Hi;
    float term = 0.f;
    const int j = j0 + r;
    const int nc_i = i < n_q ? (kv - n_q + 1 + i) / g.B : 0;
    const bool live = i < n_q && j < nc_i;
    if (live) {
      const float* krow = kbar_s + r * kStride;
      const float4* qh = reinterpret_cast<const float4*>(iq_s + (i * g.Hi + h) * kDI);
      float dot = 0.f;
#pragma unroll
      for (int d4 = 0; d4 < kDI / 4; ++d4) {
        const float4 qv = qh[d4];
        dot = fmaf(qv.x, krow[4 * d4 + 0], dot);
        dot = fmaf(qv.y, krow[4 * d4 + 1], dot);
        dot = fmaf(qv.z, krow[4 * d4 + 2], dot);
        dot = fmaf(qv.w, krow[4 * d4 + 3], dot);
      }
      term = iw_s[i * g.Hi + h] * fmaxf(dot, 0.f);
    }
    for (int o = 1; o < g.Hi; o <<= 1) term += __shfl_xor_sync(kFull, term, o);
    if (i < n_q && h == 0 && j < j0 + kPart && j < nblk_cap) {
      const float sc = live ? term * g.idx_scale : -INFINITY;
      if (live) keys_ws[((size_t)b * n_q + i) * nblk_cap + j] = score_key(sc);
      if (scores_out) scores_out[((size_t)b * n_q + i) * nblk_cap + j] = sc;
    }
  }
  // 3. the last range to finish selects
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last_s = atomicAdd(&counter[b], 1) == nparts - 1;
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  for (int i = 0; i < n_q; ++i) {
    const int n = kv - n_q + 1 + i;
    const int nc_i = n / g.B;
    {   // eight loads in flight per thread before any store
      const uint32_t* kq = keys_ws + ((size_t)b * n_q + i) * nblk_cap;
      for (int j0 = 0; j0 < nc_i; j0 += 8 * kSelThreads) {
        uint32_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + u * kSelThreads + threadIdx.x;
          v[u] = j < nc_i ? __ldcg(kq + j) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + u * kSelThreads + threadIdx.x;
          if (j < nc_i) keys_s[j] = v[u];
        }
      }
    }
    __syncthreads();
    const int m = cta_topk_radix(keys_s, nc_i, k, pos_s);
    const int tail = n - nc_i * g.B;
    int* srow = sel + ((size_t)b * n_q + i) * kp1;
    for (int e = threadIdx.x; e < kp1; e += blockDim.x) {
      int v = -1;
      if (e < m) v = pos_s[e];
      else if (e == m && tail > 0) v = nc_i;
      srow[e] = v;
    }
    if (threadIdx.x == 0) nsel[(size_t)b * n_q + i] = m + (tail > 0 ? 1 : 0);
    __syncthreads();
  }
  if (threadIdx.x == 0) counter[b] = 0;
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
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem);
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

size_t decode_select_smem(const Geom& g, int n_q, int cap) {
  return sizeof(float) * ((size_t)kPart * (g.di + 1) + (size_t)n_q * g.Hi * g.di + n_q * g.Hi) +
         sizeof(uint32_t) * (size_t)(cap / g.B) + sizeof(int) * (size_t)g.k;
}

int decode_select_parts(const Geom& g, int cap) { return (cap / g.B + kPart - 1) / kPart; }

template <typename T, int kDI>
static cudaError_t launch_decode_select_t(const Geom& g, int batch, int n_q, int cap,
                                          const int* kv_len, const void* iq, const void* ik_cache,
                                          const float* iw, float* pooled, float* scores_out,
                                          uint32_t* keys_ws, int* counter, int* sel, int* nsel,
                                          int* dev_err, cudaStream_t st) {
  const size_t smem = decode_select_smem(g, n_q, cap);
  auto kern = decode_select_kernel<T, kDI>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(decode_select_parts(g, cap), batch), kSelThreads, smem, st>>>(
      g, n_q, cap, kv_len, (const T*)iq, (const T*)ik_cache, iw, pooled, scores_out, keys_ws,
      counter, sel, nsel, dev_err);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_decode_select(qsa_dtype dt, const Geom& g, int batch, int n_q, int cap,
                                 const int* kv_len, const void* iq, const void* ik_cache,
                                 const float* iw, float* pooled, float* scores_out,
                                 uint32_t* keys_ws, int* counter, int* sel, int* nsel,
                                 int* dev_err, cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
#define QSA_DS(T, DI)                                                                       \
  return launch_decode_select_t<T, DI>(g, batch, n_q, cap, kv_len, iq, ik_cache, iw, pooled, \
                                       scores_out, keys_ws, counter, sel, nsel, dev_err, st)
  if (dt == QSA_BF16) {
    if (g.di == 64) QSA_DS(__nv_bfloat16, 64);
    QSA_DS(__nv_bfloat16, 32);
  } else {
    if (g.di == 64) QSA_DS(float, 64);
    QSA_DS(float, 32);
  }
#undef QSA_DS
}

}  // namespace qsa
