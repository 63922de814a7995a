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
#include <algorithm>

#include "qsa_common.cuh"
#include "qsa_kernels.h"
#include "qsa_pool.cuh"

namespace qsa {

// ----------------------------------------------------------------- pooling
// One CTA of 256 threads pools one block (pool_block: warp w sums rows w, w + 8,
// ... of the block in ascending order, then a fixed tree and the 1/B scale).
constexpr int kPoolThreads = 256;

template <typename T>
__device__ __forceinline__ void pool_block_cta(const T* __restrict__ rows, int B, int di,
                                               float* __restrict__ dst, int rope_dim,
                                               float rope_theta, int pos) {
  __shared__ float2 part[8][32];
  pool_block<T>(rows, B, di, dst, part, kPoolThreads / 32, rope_dim, rope_theta, pos);
}

// Grid (blocks of the longest sequence, batch).
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
pool_prefill_kernel(const T* __restrict__ ik, const int* __restrict__ cu, int B, int di,
                    float* __restrict__ pooled, int max_nblk, int rope_dim, float rope_theta) {
  grid_dependents_launch();   // the selection kernel may start its prologue
  const int b = blockIdx.y, j = blockIdx.x;
  const int s0 = cu[b], L = cu[b + 1] - s0;
  if (j >= L / B) return;
  pool_block_cta(ik + ((size_t)s0 + (size_t)j * B) * di, B, di,
                 pooled + ((size_t)b * max_nblk + j) * di, rope_dim, rope_theta, j * B);
}

// mode 0: rebuild every complete block; mode 1: only the blocks completed by
// the last n_q appended rows. Grid (blocks in range, batch).
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
pool_cache_kernel(const T* __restrict__ ik_cache, const int* __restrict__ kv_len, int cap,
                  int n_q, int mode, int B, int di, float* __restrict__ pooled, int* dev_err,
                  Pages pg, int rope_dim, float rope_theta, int block_lo) {
  const int b = blockIdx.y;
  // block_lo >= 0: a context-parallel shard starting at that block, kv_len
  // the full lengths (the shard holds the clamped remainder)
  const int kv = block_lo >= 0 ? min(max(kv_len[b] - block_lo * B, 0), cap) : kv_len[b];
  if (kv < (mode ? n_q : 0) || kv > cap) {
    if (dev_err && threadIdx.x == 0 && blockIdx.x == 0) atomicExch(dev_err, 1);
    return;
  }
  const int jlo = mode ? (kv - n_q) / B : 0;
  const int j = jlo + blockIdx.x;
  if (j >= kv / B) return;
  size_t row0 = ((size_t)b * cap + (size_t)j * B);
  if (pg.table) {
    const int page = pg.table[(size_t)b * (cap / B) + j];
    if (page < 0 || page >= pg.num_pages) {
      if (dev_err && threadIdx.x == 0) atomicExch(dev_err, 3);
      return;
    }
    row0 = (size_t)page * B;
  }
  pool_block_cta(ik_cache + row0 * di, B, di, pooled + ((size_t)b * (cap / B) + j) * di, rope_dim,
                 rope_theta, (j + max(block_lo, 0)) * B);
}

// --------------------------------------------- append (indexer front end)
// One CTA per sequence: writes the step's n_q new rows of K and V (optional)
// and of the indexer keys into the caches at rows kv - n_q .. kv - 1 (kv the
// post-append length), and in the same pass pools the blocks those rows
// complete (with the indexer rotary embedding), reading the block's earlier
// rows from the cache and its new rows from the inputs, in pool_block's order:
// the same bits as the cache rebuild. Paged caches (pg.table): token p of
// sequence b is row p % B of page table[b * (cap / B) + p / B].
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
append_kernel(Geom g, int n_q, int cap, const int* __restrict__ kv_len, const T* __restrict__ k_new,
              const T* __restrict__ v_new, const T* __restrict__ ik_new, T* __restrict__ k_cache,
              T* __restrict__ v_cache, T* __restrict__ ik_cache, float* __restrict__ pooled,
              int* dev_err, Pages pg) {
  constexpr int kVec = 16 / sizeof(T);
  const int b = blockIdx.x, tid = threadIdx.x;
  const int kv = kv_len[b];
  const int nblk_cap = cap / g.B;
  if (kv < n_q || kv > cap) {
    if (dev_err && tid == 0) atomicExch(dev_err, 1);
    return;
  }
  const int p0 = kv - n_q;
  // cache row of token p (-1: a page outside the pool, reported)
  auto row_of = [&](int p) -> long long {
    if (!pg.table) return (long long)b * cap + p;
    const int page = pg.table[(size_t)b * nblk_cap + p / g.B];
    if (page < 0 || page >= pg.num_pages) return -1;
    return (long long)page * g.B + p % g.B;
  };
  const int kvr = g.Hkv * g.D / kVec, ikr = g.di / kVec;   // 16-byte vectors per token row
  for (int e = tid; e < n_q * (ikr + (k_new ? 2 * kvr : 0)); e += blockDim.x) {
    const int per = ikr + (k_new ? 2 * kvr : 0);
    const int i = e / per, c = e - i * per;
    const long long r = row_of(p0 + i);
    if (r < 0) {
      if (dev_err) atomicExch(dev_err, 3);
      continue;
    }
    if (c < ikr) {
      reinterpret_cast<uint4*>(ik_cache + r * g.di)[c] =
          reinterpret_cast<const uint4*>(ik_new + ((size_t)b * n_q + i) * g.di)[c];
    } else if (c < ikr + kvr) {
      reinterpret_cast<uint4*>(k_cache + r * g.Hkv * g.D)[c - ikr] =
          reinterpret_cast<const uint4*>(k_new + ((size_t)b * n_q + i) * g.Hkv * g.D)[c - ikr];
    } else {
      reinterpret_cast<uint4*>(v_cache + r * g.Hkv * g.D)[c - ikr - kvr] =
          reinterpret_cast<const uint4*>(v_new + ((size_t)b * n_q + i) * g.Hkv * g.D)[c - ikr - kvr];
    }
  }
  // blocks completed by the new rows (n_q < B: the new rows of block j start
  // at split = p0 - j * B > 0)
  for (int j = p0 / g.B; j < kv / g.B; ++j) {
    const long long r0 = row_of(j * g.B);
    if (r0 < 0) continue;   // uniform across the CTA; reported above or by the decode step
    __shared__ float2 part[8][32];
    const int split = p0 - j * g.B;
    pool_block<T>(ik_cache + r0 * g.di, g.B, g.di, pooled + ((size_t)b * nblk_cap + j) * g.di, part,
                  kPoolThreads / 32, g.rope_dim, g.rope_theta, j * g.B,
                  ik_new + (size_t)b * n_q * g.di, split);
    __syncthreads();
  }
}

// ----------------------------------------------------------------- top-k
__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Warp-cooperative selection of the k largest keys among keys[0..n) where a
// lower position wins a tie. Writes the chosen positions, ascending, to out[]
// and their bitmap (bit j % 32 of word j / 32 for position j) to
// words[0..nw), and returns how many were chosen (min(k, n)).
//
// The selection threshold tau is found by an MSB-first bit search that keeps
// count(keys >= tau) >= k. It starts below the bits all keys share (those of
// the warp's max and min key agree above their highest differing bit) and
// stops as soon as a candidate threshold has exactly k keys at or above it;
// otherwise it ends on the k-th largest key, whose ties are then taken in
// ascending position order. Up to 32 * kR keys are held in registers; longer
// lists are re-read from shared memory.
template <int kR>
__device__ __forceinline__ uint32_t topk_threshold_regs(const uint32_t (&kr)[kR],
                                                        const bool (&ok)[kR], int k) {
  uint32_t hi = 0u, lo = 0xffffffffu;
#pragma unroll
  for (int i = 0; i < kR; ++i) {
    if (ok[i]) { hi = max(hi, kr[i]); lo = min(lo, kr[i]); }
  }
  hi = __reduce_max_sync(kFull, hi);
  lo = __reduce_min_sync(kFull, lo);
  if (hi == lo) return hi;
  const int top = 31 - __clz(hi ^ lo);                  // highest differing bit
  uint32_t tau = top == 31 ? 0u : (hi & ~((2u << top) - 1u));
#pragma unroll 1
  for (int bit = top; bit >= 0; --bit) {
    const uint32_t cand = tau | (1u << bit);
    int c = 0;
#pragma unroll
    for (int i = 0; i < kR; ++i) c += (ok[i] && kr[i] >= cand) ? 1 : 0;
    c = __reduce_add_sync(kFull, c);
    if (c >= k) tau = cand;
    if (c == k) break;
  }
  return tau;
}

template <int kR>
__device__ int warp_topk_regs(const uint32_t* keys, int n, int k, int* out, uint32_t* words,
                              int nw, int lane) {
  const unsigned lt = lanemask_lt();
  uint32_t kr[kR];
  bool ok[kR];
#pragma unroll
  for (int i = 0; i < kR; ++i) {
    const int j = lane + 32 * i;
    ok[i] = j < n;
    kr[i] = ok[i] ? keys[j] : 0u;
  }
  const uint32_t tau = topk_threshold_regs<kR>(kr, ok, k);
  int gt = 0;
#pragma unroll
  for (int i = 0; i < kR; ++i) gt += (ok[i] && kr[i] > tau) ? 1 : 0;
  const int need = k - __reduce_add_sync(kFull, gt);
  int m = 0, ties = 0;
  uint32_t mine = 0u;   // lane w keeps word w
#pragma unroll
  for (int i = 0; i < kR; ++i) {
    const bool tie = ok[i] && kr[i] == tau;
    const unsigned tb = __ballot_sync(kFull, tie);
    const bool pick = ok[i] && (kr[i] > tau || (tie && ties + __popc(tb & lt) < need));
    const unsigned pb = __ballot_sync(kFull, pick);
    if (pick) out[m + __popc(pb & lt)] = lane + 32 * i;
    if (lane == i) mine = pb;
    m += __popc(pb);
    ties += __popc(tb);
  }
  for (int w = lane; w < nw; w += 32) words[w] = w < kR ? mine : 0u;
  __syncwarp();
  return m;
}

__device__ int warp_topk(const uint32_t* keys, int n, int k, int* out, uint32_t* words, int nw,
                         int lane) {
  if (n <= k) {
    for (int j = lane; j < n; j += 32) out[j] = j;
    for (int w = lane; w < nw; w += 32) {
      const int lo = 32 * w;
      words[w] = lo >= n ? 0u : (n - lo >= 32 ? kFull : ((1u << (n - lo)) - 1u));
    }
    __syncwarp();
    return n;
  }
  if (n <= 128) return warp_topk_regs<4>(keys, n, k, out, words, nw, lane);
  if (n <= 256) return warp_topk_regs<8>(keys, n, k, out, words, nw, lane);
  const unsigned lt = lanemask_lt();
  uint32_t hi = 0u, lo = 0xffffffffu;
  for (int j = lane; j < n; j += 32) { hi = max(hi, keys[j]); lo = min(lo, keys[j]); }
  hi = __reduce_max_sync(kFull, hi);
  lo = __reduce_min_sync(kFull, lo);
  uint32_t tau = hi;
  if (hi != lo) {
    const int top = 31 - __clz(hi ^ lo);
    tau = top == 31 ? 0u : (hi & ~((2u << top) - 1u));
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      int c = 0;
      for (int j = lane; j < n; j += 32) c += keys[j] >= cand;
      c = __reduce_add_sync(kFull, c);
      if (c >= k) tau = cand;
      if (c == k) break;
    }
  }
  int gt = 0;
  for (int j = lane; j < n; j += 32) gt += keys[j] > tau;
  const int need = k - __reduce_add_sync(kFull, gt);
  int m = 0, ties = 0;
  for (int base = 0; base < n; base += 32) {
    const int j = base + lane;
    const uint32_t key = j < n ? keys[j] : 0u;
    const bool tie = j < n && key == tau;
    const unsigned tb = __ballot_sync(kFull, tie);
    const bool pick = j < n && (key > tau || (tie && ties + __popc(tb & lt) < need));
    const unsigned pb = __ballot_sync(kFull, pick);
    if (pick) out[m + __popc(pb & lt)] = j;
    if (lane == 0 && (base >> 5) < nw) words[base >> 5] = pb;
    m += __popc(pb);
    ties += __popc(tb);
  }
  for (int w = (n + 31) / 32 + lane; w < nw; w += 32) words[w] = 0u;
  __syncwarp();
  return m;
}

// ------------------------------------------------- prefill: score + top-k
// Work item = a group of kQc = 8 consecutive query tokens of one sequence.
// A CTA of 128 threads takes items from a counter in the workspace (zeroed
// before the launch), the groups with the most candidates first, so the SMs
// finish together. For an item it scores the group's queries against the
// pooled rows of the blocks its last query sees, 64 rows at a time staged in
// shared memory: thread (q, u) owns query q and rows u, u + 16, ... of the
// chunk and accumulates the dot products of four indexer heads at once; per
// head the dot runs over d in ascending order and the heads are folded in
// ascending order, s = c * sum_h w[h] * relu(dot_h). Then warp w selects the
// top-k of queries w and w + 4 from their score keys in shared memory.
// Dynamic shared memory: iq [kQc][Hi][kDI], iw [kQc][Hi], pooled chunk
// [64][kDI + 4], keys [kQc][nc_cap], positions [4][k].
constexpr int kChunk = 64;           // pooled rows staged in shared memory at a time
constexpr int kSelQc = 8;            // query tokens per work item
constexpr int kSelThreadsPrefill = 128;
constexpr int kSelCtasPerSm = 6;

template <typename T, int kDI>
__global__ void __launch_bounds__(kSelThreadsPrefill, 8)
select_prefill_kernel(Geom g, const int* __restrict__ cu, int batch, int n_groups,
                      int max_nblk, int words, const T* __restrict__ iq,
                      const float* __restrict__ iw, const float* __restrict__ pooled, int nc_cap,
                      int* __restrict__ sched, int* __restrict__ sel, int* __restrict__ nsel,
                      uint32_t* __restrict__ bitmask, float* __restrict__ scores,
                      int scores_ld) {
  constexpr int kQc = kSelQc;
  constexpr int kTpq = kSelThreadsPrefill / kQc;   // scoring threads per query (16)
  constexpr int kRpt = kChunk / kTpq;              // rows per thread per chunk (4)
  constexpr int kWarps = kSelThreadsPrefill / 32;
  constexpr int kStride = kDI + 4;                 // 16-byte rows, banks spread
  extern __shared__ __align__(16) float smem[];
  __shared__ int s_item;
  const int Hi = g.Hi;
  float* iq_s = smem;                                             // kQc * Hi * kDI
  float* iw_s = iq_s + kQc * Hi * kDI;                            // kQc * Hi (padded to 4)
  float* kb_s = iw_s + ((kQc * Hi + 3) & ~3);                     // kChunk * kStride
  uint32_t* keys_s = reinterpret_cast<uint32_t*>(kb_s + kChunk * kStride);   // kQc * nc_cap
  int* pos_s = reinterpret_cast<int*>(keys_s + kQc * nc_cap);     // kWarps * k

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q = tid / kTpq, u = tid % kTpq;
  const int n_items = n_groups * batch;
  grid_dependents_launch();   // the attention kernel may start its prologue
  for (;;) {
    if (tid == 0) s_item = atomicAdd(sched, 1);
    __syncthreads();
    const int item = s_item;
    if (item >= n_items) break;
    const int b = item % batch;
    const int p0 = (n_groups - 1 - item / batch) * kQc;
    const int s0 = cu[b], L = cu[b + 1] - s0;
    if (p0 < L) {
      const int nq = min(kQc, L - p0);
      const int nc_cta = (p0 + nq) / g.B;          // candidates of the group's last query

      // stage iq and iw of the group's queries (zeros past the sequence)
      {
        constexpr int kVec = 16 / sizeof(T);
        const int per_q = Hi * kDI;
        const T* src = iq + ((size_t)s0 + p0) * per_q;
        for (int e = tid * kVec; e < kQc * per_q; e += kSelThreadsPrefill * kVec) {
          const bool in = e < nq * per_q;
          const uint4 v = in ? *reinterpret_cast<const uint4*>(src + e) : make_uint4(0, 0, 0, 0);
          if constexpr (sizeof(T) == 2) {
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              iq_s[e + 2 * i] = __uint_as_float(w4[i] << 16);
              iq_s[e + 2 * i + 1] = __uint_as_float(w4[i] & 0xffff0000u);
            }
          } else {
            *reinterpret_cast<float4*>(iq_s + e) =
                make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                            __uint_as_float(v.w));
          }
        }
        for (int e = tid; e < kQc * Hi; e += kSelThreadsPrefill)
          iw_s[e] = e < nq * Hi ? iw[((size_t)s0 + p0) * Hi + e] : 0.f;
      }
      if (g.rope_dim) {   // query p0 + q turned at its position (read after the chunk barrier)
        __syncthreads();
        rope_rows(iq_s, nq * Hi, Hi, kDI, p0, g.rope_dim, g.rope_theta, tid, kSelThreadsPrefill);
      }

      grid_dependency_wait();   // pooled rows come from the pooling kernel
      const int nc_q = q < nq ? (p0 + q + 1) / g.B : 0;
      const size_t tq = (size_t)s0 + p0 + q;
      const float* pooled_b = pooled + (size_t)b * max_nblk * kDI;
      const float* myq = iq_s + q * Hi * kDI;
      const float* myw = iw_s + q * Hi;

      for (int c0 = 0; c0 < nc_cta; c0 += kChunk) {
        const int rows = min(kChunk, nc_cta - c0);
        const int nrpt = (rows + kTpq - 1) / kTpq;   // row slots in use (uniform)
        __syncthreads();
        {
          constexpr int kF4 = kChunk * kDI / 4 / kSelThreadsPrefill;   // float4 per thread
          float4 buf[kF4];
#pragma unroll
          for (int i = 0; i < kF4; ++i) {
            const int e = (tid + i * kSelThreadsPrefill) * 4;
            const int r = e / kDI;
            buf[i] = r < rows ? *reinterpret_cast<const float4*>(
                                    pooled_b + (size_t)(c0 + r) * kDI + (e - r * kDI))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int i = 0; i < kF4; ++i) {
            const int e = (tid + i * kSelThreadsPrefill) * 4;
            const int r = e / kDI;
            *reinterpret_cast<float4*>(kb_s + r * kStride + (e - r * kDI)) = buf[i];
          }
        }
        __syncthreads();
        float s[kRpt];
#pragma unroll
        for (int i = 0; i < kRpt; ++i) s[i] = 0.f;
        for (int hg = 0; hg < Hi; hg += 4) {
          float acc[kRpt][4];
#pragma unroll
          for (int i = 0; i < kRpt; ++i)
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) acc[i][hh] = 0.f;
#pragma unroll 1
          for (int d = 0; d < kDI; d += 4) {
            float4 qv[4];
#pragma unroll
            for (int hh = 0; hh < 4; ++hh)
              qv[hh] = hg + hh < Hi ? *reinterpret_cast<const float4*>(myq + (hg + hh) * kDI + d)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < kRpt; ++i) {
              if (i < nrpt) {
                const float4 kv =
                    *reinterpret_cast<const float4*>(kb_s + (u + i * kTpq) * kStride + d);
#pragma unroll
                for (int hh = 0; hh < 4; ++hh) {
                  float a = acc[i][hh];
                  a = fmaf(qv[hh].x, kv.x, a);
                  a = fmaf(qv[hh].y, kv.y, a);
                  a = fmaf(qv[hh].z, kv.z, a);
                  a = fmaf(qv[hh].w, kv.w, a);
                  acc[i][hh] = a;
                }
              }
            }
          }
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            if (hg + hh < Hi) {
              const float wh = myw[hg + hh];
#pragma unroll
              for (int i = 0; i < kRpt; ++i) s[i] = fmaf(wh, fmaxf(acc[i][hh], 0.f), s[i]);
            }
          }
        }
#pragma unroll
        for (int i = 0; i < kRpt; ++i) {
          const int j = c0 + u + i * kTpq;
          if (j < nc_q) {
            const float sc = s[i] * g.idx_scale;
            keys_s[q * nc_cap + j] = score_key(sc);
            if (scores) scores[tq * scores_ld + j] = sc;
          }
        }
      }
      if (scores && q < nq)
        for (int j = nc_q + u; j < scores_ld; j += kTpq) scores[tq * scores_ld + j] = -INFINITY;
      __syncthreads();

      int* my_pos = pos_s + warp * g.k;
      for (int qq = warp; qq < nq; qq += kWarps) {
        const int n = p0 + qq + 1;
        const int nc = n / g.B;
        const size_t t = (size_t)s0 + p0 + qq;
        uint32_t* brow = bitmask + t * words;
        const int m = warp_topk(keys_s + qq * nc_cap, nc, g.k, my_pos, brow, words, lane);
        const int tail = n - nc * g.B;
        int* srow = sel + t * (g.k + 1);
        for (int e = lane; e < g.k + 1; e += 32) {
          int v = -1;
          if (e < m) v = my_pos[e];
          else if (e == m && tail > 0) v = nc;
          srow[e] = v;
        }
        if (lane == 0) {
          nsel[t] = m + (tail > 0 ? 1 : 0);
          if (tail > 0 && words > 0) brow[nc >> 5] |= 1u << (nc & 31);   // after the word writes
        }
        __syncwarp();
      }
    }
    __syncthreads();   // every thread has read s_item and finished with shared memory
  }
}

// ------------------------------------------------------- CTA top-k
// The k largest of keys[0..n) (shared memory) where a lower position wins a
// tie, chosen by a whole CTA of 256 threads. The threshold tau comes from an
// MSB-first bit search that keeps count(keys >= tau) >= k: it starts below
// the bits all keys share (those of the CTA's max and min key agree above
// their highest differing bit), counts with one block reduction per bit, and
// stops as soon as a candidate has exactly k keys at or above it (else it
// ends on the k-th largest key). Then each thread counts the keys > tau and
// == tau in its contiguous run of positions, one block scan turns the counts
// into output offsets, and the chosen positions are written in ascending
// order, ties at tau lowest position first. Returns min(k, n).
constexpr int kTopkThreads = 256;

__device__ int cta_topk_bits(const uint32_t* keys, int n, int k, int* out) {
  constexpr int kW = kTopkThreads / 32;
  constexpr int kR = 8;                         // keys per thread kept in registers
  __shared__ uint32_t red_u[2][kW];
  __shared__ int red_c[2][kW];
  __shared__ int red_g[kW];
  __shared__ int scan_s[2][kW];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (n <= k) {
    for (int j = tid; j < n; j += kTopkThreads) out[j] = j;
    __syncthreads();
    return n;
  }
  const bool in_regs = n <= kR * kTopkThreads;
  uint32_t kr[kR];
#pragma unroll
  for (int u = 0; u < kR; ++u) {
    const int j = tid + u * kTopkThreads;
    kr[u] = (in_regs && j < n) ? keys[j] : 0u;
  }
  uint32_t hi = 0u, lo = 0xffffffffu;
  if (in_regs) {
#pragma unroll
    for (int u = 0; u < kR; ++u)
      if (tid + u * kTopkThreads < n) { hi = max(hi, kr[u]); lo = min(lo, kr[u]); }
  } else {
    for (int j = tid; j < n; j += kTopkThreads) { hi = max(hi, keys[j]); lo = min(lo, keys[j]); }
  }
  hi = __reduce_max_sync(kFull, hi);
  lo = __reduce_min_sync(kFull, lo);
  if (lane == 0) { red_u[0][warp] = hi; red_u[1][warp] = lo; }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kW; ++w) { hi = max(hi, red_u[0][w]); lo = min(lo, red_u[1][w]); }
  uint32_t tau = hi;
  if (hi != lo) {
    const int top = 31 - __clz(hi ^ lo);                  // highest differing bit
    tau = top == 31 ? 0u : (hi & ~((2u << top) - 1u));
    int slot = 0;
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      int c = 0;
      if (in_regs) {
#pragma unroll
        for (int u = 0; u < kR; ++u) c += (tid + u * kTopkThreads < n && kr[u] >= cand) ? 1 : 0;
      } else {
        for (int j = tid; j < n; j += kTopkThreads) c += keys[j] >= cand ? 1 : 0;
      }
      c = __reduce_add_sync(kFull, c);
      if (lane == 0) red_c[slot][warp] = c;
      __syncthreads();
      int tot = 0;
#pragma unroll
      for (int w = 0; w < kW; ++w) tot += red_c[slot][w];
      slot ^= 1;                                           // the next step writes the other slot
      if (tot >= k) tau = cand;
      if (tot == k) break;                                 // uniform: every thread read tot
    }
  }
  // keys > tau are all taken; of the keys == tau, the first `need` positions
  int gt = 0;
  if (in_regs) {
#pragma unroll
    for (int u = 0; u < kR; ++u) gt += (tid + u * kTopkThreads < n && kr[u] > tau) ? 1 : 0;
  } else {
    for (int j = tid; j < n; j += kTopkThreads) gt += keys[j] > tau ? 1 : 0;
  }
  gt = __reduce_add_sync(kFull, gt);
  if (lane == 0) red_g[warp] = gt;
  __syncthreads();
  int n_gt_all = 0;
#pragma unroll
  for (int w = 0; w < kW; ++w) n_gt_all += red_g[w];
  const int need = k - n_gt_all;   // keys equal to tau to take, lowest positions first
  // each thread owns the contiguous run [r_lo, r_hi)
  const int per = (n + kTopkThreads - 1) / kTopkThreads;
  const int r_lo = min(n, tid * per), r_hi = min(n, r_lo + per);
  int n_gt = 0, n_eq = 0;
  for (int j = r_lo; j < r_hi; ++j) {
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
  for (int j = r_lo; j < r_hi; ++j) {
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

// ------------------------------------------------ decode: selection kernel
// The decode step's selection as its own kernel: qsa_select_decode, and the
// two-launch decode where the one-launch decode kernel does not apply.
// Grid (ceil(cap/B / 64), batch); 256 threads (8 warps). CTA c owns candidate blocks
// [64c, 64c + 64) of sequence b and
//  1. pools the blocks of its range that this step's tokens complete (the
//     incremental pooled-key cache) and writes them to the cache,
//  2. scores its blocks for every new query of the sequence (one thread per
//     (block, indexer head), summed over the heads by shuffles) and publishes
//     the score keys,
//  3. the last CTA of the sequence to finish (an atomic counter that the
//     caller zeroes before the launch) selects each query's top-k from all
//     of them (cta_topk_bits), then appends the tail block.
constexpr int kSelThreads = 256;
constexpr int kPart = 64;                 // candidate blocks per CTA

template <typename T, int kDI>
__global__ void __launch_bounds__(kSelThreads)
decode_select_kernel(Geom g, int n_q, int cap, const int* __restrict__ kv_len,
                     const T* __restrict__ iq, const T* __restrict__ ik_cache,
                     const float* __restrict__ iw, float* __restrict__ pooled,
                     float* __restrict__ scores_out, uint32_t* __restrict__ keys_ws,
                     int* __restrict__ counter, int* __restrict__ sel, int* __restrict__ nsel,
                     int* dev_err, Pages pg, int* ready, CpShard cp) {
  grid_dependents_launch();   // the attention kernel may start its prologue
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
  // (context-parallel shard: lengths in the shard's rows; a query sees at most
  // the shard's cap rows and possibly none)
  const int kv = cp.on ? kv_len[b] - cp.row_off : kv_len[b];
  const int kp1 = k + 1;
  if (!cp.on && (kv < n_q || kv > cap)) {
    if (c == 0) {
      for (int e = threadIdx.x; e < n_q * kp1; e += blockDim.x) sel[(size_t)b * n_q * kp1 + e] = -1;
      for (int e = threadIdx.x; e < n_q; e += blockDim.x) nsel[(size_t)b * n_q + e] = 0;
      if (dev_err && threadIdx.x == 0) atomicExch(dev_err, 1);
    }
    return;
  }
  const int nc_last = min(max(kv, 0), cap) / g.B;   // candidates of the last query
  const int nparts = max(1, (nc_last + kPart - 1) / kPart);
  if (c >= nparts) return;
  const int j0 = c * kPart;
  const int rows = max(0, min(kPart, nc_last - j0));

  // 0. paged caches: every page id the attention may gather from this range
  //    (and the tail block, by the last range) must name a page of the pool
  if (pg.table) {
    const int nb_used = (kv + g.B - 1) / g.B;
    const int jend = c == nparts - 1 ? nb_used : min(nb_used, j0 + kPart);
    for (int j = j0 + (int)threadIdx.x; j < jend; j += blockDim.x) {
      const int page = pg.table[(size_t)b * nblk_cap + j];
      if ((page < 0 || page >= pg.num_pages) && dev_err) atomicExch(dev_err, 3);
    }
  }
  // 1. blocks completed by this step's tokens (pool_block_cta needs the whole CTA)
  const int jnew_lo = max(min(max(kv - n_q, 0), cap) / g.B, j0),
            jnew_hi = min(nc_last, j0 + kPart);
  for (int j = jnew_lo; j < jnew_hi; ++j) {
    size_t row0 = (size_t)b * cap + (size_t)j * g.B;
    if (pg.table) {
      const int page = pg.table[(size_t)b * nblk_cap + j];
      row0 = (page >= 0 && page < pg.num_pages) ? (size_t)page * g.B : SIZE_MAX;
    }
    if (row0 != SIZE_MAX)   // uniform across the CTA
      pool_block_cta(ik_cache + row0 * kDI, g.B, kDI, pooled + ((size_t)b * nblk_cap + j) * kDI,
                     g.rope_dim, g.rope_theta, (j + (cp.on ? cp.block_lo : 0)) * g.B);
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
  if (g.rope_dim) {   // query i turned at its position kv_len - n_q + i
    rope_rows(iq_s, n_q * g.Hi, g.Hi, kDI, kv_len[b] - n_q, g.rope_dim, g.rope_theta, threadIdx.x,
              blockDim.x);
    __syncthreads();
  }
  // scores: one (query, block, head) triple per thread; heads are adjacent
  // lanes (Hi divides 32), so the weighted relu terms are summed by shuffles
  const int per_q = kPart * g.Hi;
  for (int base = 0; base < n_q * per_q; base += blockDim.x) {
    const int e = base + threadIdx.x;
    const int i = e / per_q, rem = e - i * per_q;
    const int r = rem / g.Hi, h = rem - r * g.Hi;
    float term = 0.f;
    const int j = j0 + r;
    const int nc_i = i < n_q ? min(max(kv - n_q + 1 + i, 0), cap) / g.B : 0;
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
    const int n = min(max(kv - n_q + 1 + i, 0), cap);
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
    const int m = cta_topk_bits(keys_s, nc_i, k, pos_s);
    const int tail = n - nc_i * g.B;
    int* srow = sel + ((size_t)b * n_q + i) * kp1;
    for (int e = threadIdx.x; e < kp1; e += blockDim.x) {
      int v = -1;
      if (e < m) v = pos_s[e];
      else if (e == m && tail > 0) v = nc_i;
      srow[e] = v;
    }
    if (threadIdx.x == 0) nsel[(size_t)b * n_q + i] = m + (tail > 0 ? 1 : 0);
    if (cp.cand_score) {   // the shard's candidates: scores (keys decoded) and global ids
      for (int e = threadIdx.x; e < k; e += blockDim.x) {
        const size_t o = ((size_t)b * n_q + i) * k + e;
        cp.cand_score[o] = e < m ? key_score(keys_s[pos_s[e]]) : -INFINITY;
        cp.cand_id[o] = e < m ? pos_s[e] + cp.block_lo : -1;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) counter[b] = 0;
  if (ready) {   // this sequence's selections are written: release its attention CTAs
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
      asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(ready + b), "r"(1) : "memory");
  }
}

// ------------------------------------------------------------ launchers
template <typename T>
static cudaError_t launch_pool_prefill_t(const void* ik, const int* cu, int batch, int max_seqlen,
                                         const Geom& g, float* pooled, int max_nblk,
                                         cudaStream_t st) {
  const int nblk = max_seqlen / g.B;
  if (nblk == 0 || batch == 0) return cudaSuccess;
  pool_prefill_kernel<T><<<dim3(nblk, batch), kPoolThreads, 0, st>>>(
      (const T*)ik, cu, g.B, g.di, pooled, max_nblk, g.rope_dim, g.rope_theta);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_pool_prefill(qsa_dtype dt, const void* ik, const int* cu, int batch,
                                int max_seqlen, const Geom& g, float* pooled, int max_nblk,
                                cudaStream_t st) {
  return dt == QSA_BF16
             ? launch_pool_prefill_t<__nv_bfloat16>(ik, cu, batch, max_seqlen, g, pooled,
                                                    max_nblk, st)
             : launch_pool_prefill_t<float>(ik, cu, batch, max_seqlen, g, pooled, max_nblk, st);
}

cudaError_t launch_pool_cache(qsa_dtype dt, const void* ik_cache, const int* kv_len, int batch,
                              int cap, int n_q, int mode, const Geom& g, float* pooled,
                              int* dev_err, cudaStream_t st, Pages pg, int block_lo) {
  const int B = g.B, di = g.di;
  const int span = mode ? (n_q + B - 1) / B + 1 : cap / B;
  if (batch == 0 || span == 0) return cudaSuccess;
  dim3 grid(span, batch);
  if (dt == QSA_BF16)
    pool_cache_kernel<__nv_bfloat16><<<grid, kPoolThreads, 0, st>>>(
        (const __nv_bfloat16*)ik_cache, kv_len, cap, n_q, mode, B, di, pooled, dev_err, pg,
        g.rope_dim, g.rope_theta, block_lo);
  else
    pool_cache_kernel<float><<<grid, kPoolThreads, 0, st>>>((const float*)ik_cache, kv_len, cap,
                                                            n_q, mode, B, di, pooled, dev_err, pg,
                                                            g.rope_dim, g.rope_theta, block_lo);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_append(qsa_dtype dt, const Geom& g, int batch, int n_q, int cap,
                          const int* kv_len, const void* k_new, const void* v_new,
                          const void* ik_new, void* k_cache, void* v_cache, void* ik_cache,
                          float* pooled, int* dev_err, Pages pg, cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
  if (dt == QSA_BF16)
    append_kernel<__nv_bfloat16><<<batch, kPoolThreads, 0, st>>>(
        g, n_q, cap, kv_len, (const __nv_bfloat16*)k_new, (const __nv_bfloat16*)v_new,
        (const __nv_bfloat16*)ik_new, (__nv_bfloat16*)k_cache, (__nv_bfloat16*)v_cache,
        (__nv_bfloat16*)ik_cache, pooled, dev_err, pg);
  else
    append_kernel<float><<<batch, kPoolThreads, 0, st>>>(
        g, n_q, cap, kv_len, (const float*)k_new, (const float*)v_new, (const float*)ik_new,
        (float*)k_cache, (float*)v_cache, (float*)ik_cache, pooled, dev_err, pg);
  note_launch();
  return cudaGetLastError();
}

size_t select_prefill_smem(const Geom& g, int nc_cap) {
  return sizeof(float) * ((size_t)kSelQc * g.Hi * g.di +
                          (((size_t)kSelQc * g.Hi + 3) & ~(size_t)3) +
                          (size_t)kChunk * (g.di + 4)) +
         sizeof(uint32_t) * (size_t)kSelQc * nc_cap +
         sizeof(int) * (kSelThreadsPrefill / 32) * (size_t)g.k;
}

template <typename T, int kDI>
static cudaError_t launch_select_prefill_t(const Geom& g, const int* cu, int batch,
                                           int max_seqlen, int max_nblk, int words,
                                           const void* iq, const float* iw, const float* pooled,
                                           int* sched, int* sel, int* nsel, uint32_t* bitmask,
                                           float* scores, int scores_ld, cudaStream_t st) {
  const int nc_cap = max(1, max_seqlen / g.B);
  const size_t smem = select_prefill_smem(g, nc_cap);
  auto kern = select_prefill_kernel<T, kDI>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0, sms = 0;
  e = resident_ctas(reinterpret_cast<const void*>(kern), kSelThreadsPrefill, smem, &per_sm, &sms);
  if (e != cudaSuccess) return e;
  const int n_groups = (max_seqlen + kSelQc - 1) / kSelQc;
  const long long items = (long long)n_groups * batch;
  // fewer CTAs than items, so that the SMs that finish early take more items
  const int ctas = std::max(1, std::min(per_sm, kSelCtasPerSm) * sms);
  const int grid = (int)std::min<long long>(items, ctas);
  e = launch_dependent(kern, dim3(grid), dim3(kSelThreadsPrefill), smem, st, g, cu, batch,
                       n_groups, max_nblk, bitmask ? words : 0, (const T*)iq, iw, pooled, nc_cap,
                       sched, sel, nsel, bitmask, scores, scores_ld);
  note_launch();
  return e;
}

cudaError_t launch_select_prefill(qsa_dtype dt, const Geom& g, const int* cu, int batch,
                                  int max_seqlen, int max_nblk, int words, const void* iq,
                                  const float* iw, const float* pooled, int* sched, int* sel,
                                  int* nsel, uint32_t* bitmask, float* scores, int scores_ld,
                                  cudaStream_t st) {
  if (batch == 0 || max_seqlen == 0) return cudaSuccess;
#define QSA_SEL(T, DI)                                                                      \
  return launch_select_prefill_t<T, DI>(g, cu, batch, max_seqlen, max_nblk, words, iq, iw,  \
                                        pooled, sched, sel, nsel, bitmask, scores, scores_ld, st)
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
                                          int* dev_err, cudaStream_t st, Pages pg, int* ready,
                                          CpShard cp) {
  const size_t smem = decode_select_smem(g, n_q, cap);
  auto kern = decode_select_kernel<T, kDI>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(decode_select_parts(g, cap), batch), kSelThreads, smem, st>>>(
      g, n_q, cap, kv_len, (const T*)iq, (const T*)ik_cache, iw, pooled, scores_out, keys_ws,
      counter, sel, nsel, dev_err, pg, ready, cp);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_decode_select(qsa_dtype dt, const Geom& g, int batch, int n_q, int cap,
                                 const int* kv_len, const void* iq, const void* ik_cache,
                                 const float* iw, float* pooled, float* scores_out,
                                 uint32_t* keys_ws, int* counter, int* sel, int* nsel,
                                 int* dev_err, cudaStream_t st, Pages pg, int* ready,
                                 CpShard cp) {
  if (batch == 0) return cudaSuccess;
#define QSA_DS(T, DI)                                                                       \
  return launch_decode_select_t<T, DI>(g, batch, n_q, cap, kv_len, iq, ik_cache, iw, pooled, \
                                       scores_out, keys_ws, counter, sel, nsel, dev_err, st, pg, \
                                       ready, cp)
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
