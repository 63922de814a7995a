// Context-parallel QSA decode: the two steps between the processes' shards.
//
// A sequence too long for one GPU is split by blocks over the processes of a
// group; each process selects the top-k complete blocks of its own shard
// (decode_select_kernel in shard mode), the candidates of every process are
// all-gathered, and
//  1. cp_global_topk_kernel takes the top-k of the gathered candidates under
//     the selection's total order (score descending, block id ascending) and
//     appends the query's incomplete tail block. Every globally selected block
//     is in its own shard's top-k (fewer than k blocks of the whole cache beat
//     it, so fewer than k of its shard do), and the scores are computed by the
//     same arithmetic in every shard, so this is exactly the single-GPU
//     selection (the rule of the instagit MTPLX page, section "Qwen Sparse
//     Attention (QSA)", and of the llama.cpp PR #27739 page's QSA commit);
//  2. after each process has attended its share of the selection (gated fp32
//     partials with their log-sum-exp) and the partials are all-gathered,
//     cp_merge_kernel merges them: with M = max_r lse_r and
//     w_r = exp(lse_r - M) / sum_r exp(lse_r - M), out = sum_r w_r out_r and
//     lse = M + log sum_r exp(lse_r - M). The sigmoid gate on the output is
//     elementwise, so it commutes with this weighted sum.
#include <math.h>

#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {

namespace {

constexpr int kTopkThreads = 256;
constexpr int kMaxCand = 64 * 64;   // world * k candidates per query

// One CTA per (sequence, new query). A candidate is the 64-bit value
// (score key << 32) | ~id, larger = earlier in the order; the ids of one
// query are distinct, so the k-th largest value is unique and the selection
// is the values >= it. It is found by deciding its bits from the top, each
// step counting the values above the candidate prefix over the whole CTA.
__global__ void __launch_bounds__(kTopkThreads)
cp_global_topk_kernel(Geom g, int n_q, int world, const int* __restrict__ kv_len,
                      const float* __restrict__ cand_score, const int* __restrict__ cand_id,
                      int* __restrict__ sel, int* __restrict__ nsel, int batch) {
  __shared__ unsigned long long vals[kMaxCand];
  __shared__ int red[kTopkThreads / 32];
  __shared__ int chosen[kMaxTopK];
  __shared__ int n_chosen;
  const int bi = blockIdx.x, b = bi / n_q, i = bi - b * n_q;
  const int k = g.k, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = world * k;
  int valid = 0;
  for (int e = tid; e < n; e += kTopkThreads) {
    const int r = e / k, j = e - r * k;
    const size_t o = (((size_t)r * batch + b) * n_q + i) * k + j;
    const int id = cand_id[o];
    unsigned long long v = 0ull;   // padding: below every candidate
    if (id >= 0) {
      v = ((unsigned long long)score_key(cand_score[o]) << 32) | (0xffffffffu - (uint32_t)id);
      ++valid;
    }
    vals[e] = v;
  }
  valid = __reduce_add_sync(kFull, valid);
  if (lane == 0) red[warp] = valid;
  if (tid == 0) n_chosen = 0;
  __syncthreads();
  int total = 0;
  for (int w = 0; w < kTopkThreads / 32; ++w) total += red[w];
  const int m = min(k, total);   // candidates taken
  __syncthreads();
  unsigned long long tau = 0ull;   // the m-th largest value (0: take every valid one)
  if (m > 0 && m < total) {
    for (int bit = 63; bit >= 0; --bit) {
      const unsigned long long cand = tau | (1ull << bit);
      int c = 0;
      for (int e = tid; e < n; e += kTopkThreads) c += vals[e] >= cand ? 1 : 0;
      c = __reduce_add_sync(kFull, c);
      if (lane == 0) red[warp] = c;
      __syncthreads();
      int tot = 0;
      for (int w = 0; w < kTopkThreads / 32; ++w) tot += red[w];
      __syncthreads();
      if (tot >= m) tau = cand;
    }
  } else if (m > 0) {
    tau = 1ull;   // every valid candidate (valid values are nonzero: ~id > 0 for id < 2^32 - 1)
  }
  for (int e = tid; e < n; e += kTopkThreads) {
    const unsigned long long v = vals[e];
    if (m > 0 && v != 0ull && v >= tau) {
      const int slot = atomicAdd(&n_chosen, 1);
      if (slot < kMaxTopK) chosen[slot] = (int)(0xffffffffu - (uint32_t)(v & 0xffffffffull));
    }
  }
  __syncthreads();
  // ascending block ids (rank by counting; at most k <= 64 of them), then the tail
  const int kp1 = k + 1;
  int* srow = sel + ((size_t)b * n_q + i) * kp1;
  const int cnt = min(n_chosen, m);
  for (int e = tid; e < cnt; e += kTopkThreads) {
    const int id = chosen[e];
    int rank = 0;
    for (int f = 0; f < cnt; ++f) rank += chosen[f] < id ? 1 : 0;
    srow[rank] = id;
  }
  const int nv = kv_len[b] - n_q + 1 + i;   // tokens the query sees
  const int tail = nv > 0 ? nv % g.B : 0;
  for (int e = cnt + tid; e < kp1; e += kTopkThreads)
    srow[e] = (e == cnt && tail > 0) ? nv / g.B : -1;
  if (tid == 0) nsel[(size_t)b * n_q + i] = cnt + (tail > 0 ? 1 : 0);
}

// One thread per (row, 4 dims): rows = batch * n_q * Hq partial rows of D
// values, part_out [world, rows, D], part_lse [world, rows] (natural log).
template <typename T>
__global__ void cp_merge_kernel(int rows, int D, int world, const float* __restrict__ part_out,
                                const float* __restrict__ part_lse, T* __restrict__ out,
                                float* __restrict__ lse) {
  const int per_row = D / 4;
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)rows * per_row) return;
  const int r = (int)(e / per_row), d = (int)(e - (long long)r * per_row) * 4;
  float M = -INFINITY;
  for (int w = 0; w < world; ++w) M = fmaxf(M, part_lse[(size_t)w * rows + r]);
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -INFINITY) {
    for (int w = 0; w < world; ++w) {
      const float l = part_lse[(size_t)w * rows + r];
      if (l == -INFINITY) continue;
      const float wt = expf(l - M);
      const float4 v = *reinterpret_cast<const float4*>(part_out + ((size_t)w * rows + r) * D + d);
      L += wt;
      acc.x = fmaf(wt, v.x, acc.x);
      acc.y = fmaf(wt, v.y, acc.y);
      acc.z = fmaf(wt, v.z, acc.z);
      acc.w = fmaf(wt, v.w, acc.w);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  T* o = out + (size_t)r * D + d;
  o[0] = from_f32<T>(acc.x * inv);
  o[1] = from_f32<T>(acc.y * inv);
  o[2] = from_f32<T>(acc.z * inv);
  o[3] = from_f32<T>(acc.w * inv);
  if (lse && d == 0) lse[r] = L > 0.f ? M + logf(L) : -INFINITY;
}

}  // namespace

cudaError_t launch_cp_global_topk(const Geom& g, int batch, int n_q, int world,
                                  const int* kv_len, const float* cand_score,
                                  const int* cand_id, int* sel, int* nsel, cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
  if (world * g.k > kMaxCand || g.k > kMaxTopK) return cudaErrorInvalidValue;
  cp_global_topk_kernel<<<batch * n_q, kTopkThreads, 0, st>>>(g, n_q, world, kv_len, cand_score,
                                                             cand_id, sel, nsel, batch);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_cp_merge(qsa_dtype dt, int rows, int D, int world, const float* part_out,
                            const float* part_lse, void* out, float* lse, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const long long n = (long long)rows * (D / 4);
  const int threads = 256;
  const unsigned blocks = (unsigned)((n + threads - 1) / threads);
  if (dt == QSA_BF16)
    cp_merge_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(
        rows, D, world, part_out, part_lse, static_cast<__nv_bfloat16*>(out), lse);
  else
    cp_merge_kernel<float><<<blocks, threads, 0, st>>>(rows, D, world, part_out, part_lse,
                                                       static_cast<float*>(out), lse);
  note_launch();
  return cudaGetLastError();
}

}  // namespace qsa
