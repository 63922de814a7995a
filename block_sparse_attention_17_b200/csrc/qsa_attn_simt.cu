// Sparse gated GQA attention on CUDA cores (fp32 arithmetic).
//
// Prefill: one CTA per (query token, KV head). The selected tokens are
// gathered block by block from the selection list (ascending complete blocks,
// then the tail), so no dense mask over the causal prefix is ever built
// (ramgpt "Porting Qwen4 to llama.cpp", section "CUDA Optimization Should
// Follow State Correctness": gather selected K/V, online softmax, accumulate).
// This kernel is the fp32 path and the reference shape for the bf16
// tensor-core kernel.
//
// Decode: split-KV over the union of the n_q new queries' selected blocks.
// One CTA per (sequence, KV head, split) writes partial (m, l, O) for every
// query row of the group; qsa_combine merges the splits by log-sum-exp and
// applies the sigmoid gate on the output (llama.cpp PR #27739 page, QSA
// block-composition commit text).
#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace qsa {

constexpr int kChunkKeys = 128;   // keys per inner iteration == threads per CTA

// Loads 8 consecutive elements as fp32.
template <typename T> __device__ __forceinline__ void load8(const T* p, float* x);
template <> __device__ __forceinline__ void load8<float>(const float* p, float* x) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
template <> __device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Core of both kernels. R rows (query heads, or query rows of a decode group)
// attend the keys listed in pos_s[0..cnt) of one KV head. lg_s [R][128].
// Thread `tid` computes the logits of key tid for every row, then each warp
// updates the online softmax of rows w, w+4, ...; then thread tid accumulates
// output dim d = tid % D for rows r = tid / D + j * (128 / D).
template <typename T, int D, int kMaxOwn>
struct SimtAttn {
  float acc[kMaxOwn];
  unsigned visited;   // debug count: (row, key) pairs this thread's key slots let through

  __device__ void init() {
#pragma unroll
    for (int i = 0; i < kMaxOwn; ++i) acc[i] = 0.f;
    visited = 0;
  }

  // rowmask_s[r]: bit e of the chunk-entry visibility is handled by the caller
  // through `vis`, which returns whether row r may see key slot tid.
  template <typename Vis>
  __device__ void chunk(int R, const float* q_s, float* lg_s, float* m_s, float* l_s,
                        float* alpha_s, int* pos_s, int cnt, const T* kbase,
                        const T* vbase, size_t kv_row_stride, Vis vis) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // 1) logits. A key slot no row may see is never loaded (its pos becomes
    // -1), so unselected rows cannot leak into the result even through 0 * NaN.
    if (tid < cnt) {
      bool seen = false;
      for (int r = 0; r < R; ++r) {
        const bool v = vis(r, tid);
        seen |= v;
        visited += v ? 1u : 0u;
      }
      if (seen) {
        const T* krow = kbase + (size_t)pos_s[tid] * kv_row_stride;
        float dots[32];
#pragma unroll
        for (int r = 0; r < 32; ++r) dots[r] = 0.f;
#pragma unroll 2
        for (int d0 = 0; d0 < D; d0 += 8) {
          float kx[8];
          load8<T>(krow + d0, kx);
#pragma unroll
          for (int r = 0; r < 32; ++r) {
            if (r < R) {
              const float4 qa = *reinterpret_cast<const float4*>(q_s + r * D + d0);
              const float4 qb = *reinterpret_cast<const float4*>(q_s + r * D + d0 + 4);
              float s = dots[r];
              s = fmaf(qa.x, kx[0], s); s = fmaf(qa.y, kx[1], s);
              s = fmaf(qa.z, kx[2], s); s = fmaf(qa.w, kx[3], s);
              s = fmaf(qb.x, kx[4], s); s = fmaf(qb.y, kx[5], s);
              s = fmaf(qb.z, kx[6], s); s = fmaf(qb.w, kx[7], s);
              dots[r] = s;
            }
          }
        }
#pragma unroll
        for (int r = 0; r < 32; ++r)
          if (r < R) lg_s[r * kChunkKeys + tid] = vis(r, tid) ? dots[r] : -INFINITY;
      } else {
        for (int r = 0; r < R; ++r) lg_s[r * kChunkKeys + tid] = -INFINITY;
        pos_s[tid] = -1;
      }
    } else {
      for (int r = 0; r < R; ++r) lg_s[r * kChunkKeys + tid] = -INFINITY;
    }
    __syncthreads();
    // 2) online softmax per row (log2 domain; q_s is pre-scaled by scale*log2e)
    for (int r = warp; r < R; r += 4) {
      float x[4];
      float cm = -INFINITY;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[i] = lg_s[r * kChunkKeys + lane + 32 * i];
        cm = fmaxf(cm, x[i]);
      }
      cm = warp_max(cm);
      const float m_old = m_s[r];
      const float m_new = fmaxf(m_old, cm);
      const float ref = m_new == -INFINITY ? 0.f : m_new;
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float pexp = exp2f(x[i] - ref);
        lg_s[r * kChunkKeys + lane + 32 * i] = pexp;
        sum += pexp;
      }
      sum = warp_sum(sum);
      if (lane == 0) {
        const float a = exp2f(m_old - ref);
        alpha_s[r] = a;
        l_s[r] = l_s[r] * a + sum;
        m_s[r] = m_new;
      }
    }
    __syncthreads();
    // 3) P V
    constexpr int kRowsPerPass = kChunkKeys / D;
    const int d = tid % D, r0 = tid / D;
#pragma unroll
    for (int j = 0; j < kMaxOwn; ++j) {
      const int r = r0 + j * kRowsPerPass;
      if (r < R) acc[j] *= alpha_s[r];
    }
    for (int i = 0; i < cnt; ++i) {
      const int pos = pos_s[i];
      if (pos < 0) continue;
      const float vv = to_f32(vbase[(size_t)pos * kv_row_stride + d]);
#pragma unroll
      for (int j = 0; j < kMaxOwn; ++j) {
        const int r = r0 + j * kRowsPerPass;
        if (r < R) acc[j] = fmaf(lg_s[r * kChunkKeys + i], vv, acc[j]);
      }
    }
    __syncthreads();
  }
};

// ------------------------------------------------------------------ prefill
template <typename T, int D>
__global__ void __launch_bounds__(128)
attn_prefill_simt_kernel(Geom g, const int* __restrict__ cu, const T* __restrict__ q,
                         const T* __restrict__ k, const T* __restrict__ v,
                         const T* __restrict__ gate, const int* __restrict__ sel,
                         const int* __restrict__ nsel, T* __restrict__ out,
                         float* __restrict__ lse) {
  constexpr int kMaxOwn = 16 * D / kChunkKeys;   // G <= 16
  __shared__ __align__(16) float q_s[16 * D];
  __shared__ float lg_s[16 * kChunkKeys];
  __shared__ float m_s[16], l_s[16], alpha_s[16];
  __shared__ int pos_s[kChunkKeys];
  __shared__ int sel_s[kMaxTopK + 1];

  const int b = blockIdx.y, p = blockIdx.x, hk = blockIdx.z;
  const int s0 = cu[b], L = cu[b + 1] - s0;
  if (p >= L) return;
  const int G = g.G;
  const size_t t = (size_t)s0 + p;
  const int n = p + 1;
  const int tid = threadIdx.x;

  for (int e = tid; e < G * D; e += blockDim.x)
    q_s[e] = to_f32(q[(t * g.Hq + (size_t)hk * G) * D + e]) * g.sm_scale_log2;
  const int ns = nsel[t];
  for (int e = tid; e < ns; e += blockDim.x) sel_s[e] = sel[t * (g.k + 1) + e];
  if (tid < G) { m_s[tid] = -INFINITY; l_s[tid] = 0.f; }
  __syncthreads();

  const int nc = n / g.B;
  const int tail = n - nc * g.B;
  const int ntok = (ns - (tail > 0 ? 1 : 0)) * g.B + tail;
  const size_t kv_stride = (size_t)g.Hkv * D;
  const T* kbase = k + (size_t)s0 * kv_stride + (size_t)hk * D;
  const T* vbase = v + (size_t)s0 * kv_stride + (size_t)hk * D;

  SimtAttn<T, D, kMaxOwn> core;
  core.init();
  for (int base = 0; base < ntok; base += kChunkKeys) {
    const int cnt = min(kChunkKeys, ntok - base);
    if (tid < cnt) {
      const int i = base + tid;
      const int e = i / g.B;
      pos_s[tid] = sel_s[e] * g.B + (i - e * g.B);
    }
    __syncthreads();
    core.chunk(G, q_s, lg_s, m_s, l_s, alpha_s, pos_s, cnt, kbase, vbase, kv_stride,
               [](int, int) { return true; });
  }
  if (g.keys_visited) add_keys_visited(g.keys_visited, core.visited);

  constexpr int kRowsPerPass = kChunkKeys / D;
  const int d = tid % D, r0 = tid / D;
#pragma unroll
  for (int j = 0; j < kMaxOwn; ++j) {
    const int r = r0 + j * kRowsPerPass;
    if (r < G) {
      const int h = hk * G + r;
      const float l = l_s[r];
      const float o = l > 0.f ? core.acc[j] / l : 0.f;
      const float gl = g.gate_headwise ? to_f32(gate[t * g.Hq + h])
                                       : to_f32(gate[(t * g.Hq + h) * D + d]);
      out[(t * g.Hq + h) * D + d] = from_f32<T>(sigmoidf_(gl) * o);
      if (lse && d == 0)
        lse[t * g.Hq + h] = l > 0.f ? (m_s[r] + log2f(l)) * kLn2 : -INFINITY;
    }
  }
}

// ------------------------------------------------------------------- decode
// Union of the n_q selection lists of one sequence, ascending, deduplicated.
// Each entry also carries a bitmask of the queries that see it.
// Block ids are taken relative to `lo` (a context-parallel shard's first
// block; 0 otherwise) and those outside [0, nblk) are skipped.
__device__ int build_union(const int* sel_b, const int* nsel_b, int n_q, int kp1, int* u_blk,
                           int* u_qmask, int lo, int nblk) {
  // serial merge by thread 0: at most n_q * (k + 1) entries
  int cnt = 0;
  int idx[4] = {0, 0, 0, 0};
  while (true) {
    int best = 0x7fffffff;
    for (int i = 0; i < n_q; ++i)
      if (idx[i] < nsel_b[i]) best = min(best, sel_b[i * kp1 + idx[i]]);
    if (best == 0x7fffffff) break;
    int qm = 0;
    for (int i = 0; i < n_q; ++i)
      if (idx[i] < nsel_b[i] && sel_b[i * kp1 + idx[i]] == best) { qm |= 1 << i; ++idx[i]; }
    if (best - lo >= 0 && best - lo < nblk) {
      u_blk[cnt] = best - lo;
      u_qmask[cnt] = qm;
      ++cnt;
    }
  }
  return cnt;
}

template <typename T, int D>
__global__ void __launch_bounds__(128)
attn_decode_simt_kernel(Geom g, int n_q, int cap, int nsplit, int per_split,
                        const int* __restrict__ kv_len, const T* __restrict__ q,
                        const T* __restrict__ kc, const T* __restrict__ vc,
                        const int* __restrict__ sel, const int* __restrict__ nsel,
                        float* __restrict__ part_ml, float* __restrict__ part_o, CpShard cp) {
  constexpr int kMaxRows = 32;
  constexpr int kMaxOwn = kMaxRows * D / kChunkKeys;
  __shared__ __align__(16) float q_s[kMaxRows * D];
  __shared__ float lg_s[kMaxRows * kChunkKeys];
  __shared__ float m_s[kMaxRows], l_s[kMaxRows], alpha_s[kMaxRows];
  __shared__ int pos_s[kChunkKeys];
  __shared__ int u_blk[4 * (kMaxTopK + 1)], u_qm[4 * (kMaxTopK + 1)];
  __shared__ int u_cnt;

  const int split = blockIdx.x, b = blockIdx.y, hk = blockIdx.z;
  const int tid = threadIdx.x;
  const int G = g.G, R = n_q * G;
  const int kv = kv_len[b] - cp.row_off;   // (a shard's rows: may be past either end)
  const size_t part_row0 = (((size_t)b * g.Hkv + hk) * nsplit + split) * R;
  if (!cp.on && (kv < n_q || kv > cap)) {
    for (int r = tid; r < R; r += blockDim.x) {
      part_ml[2 * (part_row0 + r)] = -INFINITY;
      part_ml[2 * (part_row0 + r) + 1] = 0.f;
    }
    return;
  }
  // rows: r = i * G + gi  <->  query i, head hk * G + gi
  for (int e = tid; e < R * D; e += blockDim.x) {
    const int r = e / D, d = e - r * D;
    const int i = r / G, gi = r - i * G;
    q_s[e] = to_f32(q[(((size_t)b * n_q + i) * g.Hq + hk * G + gi) * D + d]) * g.sm_scale_log2;
  }
  if (tid == 0)
    u_cnt = build_union(sel + (size_t)b * n_q * (g.k + 1), nsel + (size_t)b * n_q, n_q,
                        g.k + 1, u_blk, u_qm, cp.block_lo, cap / g.B);
  if (tid < R) { m_s[tid] = -INFINITY; l_s[tid] = 0.f; }
  __syncthreads();

  const size_t kv_stride = (size_t)g.Hkv * D;
  const T* kbase = kc + (size_t)b * cap * kv_stride + (size_t)hk * D;
  const T* vbase = vc + (size_t)b * cap * kv_stride + (size_t)hk * D;
  SimtAttn<T, D, kMaxOwn> core;
  core.init();
  const int e0 = split * per_split, e1 = min(u_cnt, e0 + per_split);
  for (int e = e0; e < e1; ++e) {
    const int blk = u_blk[e];
    const int qm = u_qm[e];
    for (int c0 = 0; c0 < g.B; c0 += kChunkKeys) {
      const int cnt = min(kChunkKeys, g.B - c0);
      if (tid < cnt) pos_s[tid] = blk * g.B + c0 + tid;
      __syncthreads();
      const int first_new = kv - n_q;   // query i sees positions < first_new + 1 + i
      core.chunk(R, q_s, lg_s, m_s, l_s, alpha_s, pos_s, cnt, kbase, vbase, kv_stride,
                 [&](int r, int slot) {
                   const int i = r / G;
                   return ((qm >> i) & 1) && pos_s[slot] <= first_new + i;
                 });
    }
  }
  if (g.keys_visited) add_keys_visited(g.keys_visited, core.visited);
  constexpr int kRowsPerPass = kChunkKeys / D;
  const int d = tid % D, r0 = tid / D;
#pragma unroll
  for (int j = 0; j < kMaxOwn; ++j) {
    const int r = r0 + j * kRowsPerPass;
    if (r < R) part_o[(part_row0 + r) * D + d] = core.acc[j];
  }
  for (int r = tid; r < R; r += blockDim.x) {
    part_ml[2 * (part_row0 + r)] = m_s[r];
    part_ml[2 * (part_row0 + r) + 1] = l_s[r];
  }
}

// Merge the split partials (log2 domain) and apply the gate.
// Grid (n_q * Hq, batch); D threads.
template <typename T, int D>
__global__ void decode_combine_kernel(Geom g, int n_q, int cap, int nsplit,
                                      const int* __restrict__ kv_len,
                                      const float* __restrict__ part_ml,
                                      const float* __restrict__ part_o,
                                      const T* __restrict__ gate, T* __restrict__ out,
                                      float* __restrict__ lse, CpShard cp) {
  const int b = blockIdx.y;
  const int i = blockIdx.x / g.Hq, h = blockIdx.x - i * g.Hq;
  const int d = threadIdx.x;
  const int hk = h / g.G, gi = h - hk * g.G;
  const int R = n_q * g.G, r = i * g.G + gi;
  const int kv = kv_len[b];
  const size_t orow = ((size_t)b * n_q + i) * g.Hq + h;
  if (!cp.on && (kv < n_q || kv > cap)) {
    out[orow * D + d] = from_f32<T>(0.f);
    if (lse && d == 0) lse[orow] = -INFINITY;
    return;
  }
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) {
    const size_t pr = (((size_t)b * g.Hkv + hk) * nsplit + s) * R + r;
    M = fmaxf(M, part_ml[2 * pr]);
  }
  float Lsum = 0.f, o = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const size_t pr = (((size_t)b * g.Hkv + hk) * nsplit + s) * R + r;
      const float ms = part_ml[2 * pr];
      if (ms == -INFINITY) continue;
      const float w = exp2f(ms - M);
      Lsum = fmaf(part_ml[2 * pr + 1], w, Lsum);
      o = fmaf(part_o[pr * D + d], w, o);
    }
  }
  const float val = Lsum > 0.f ? o / Lsum : 0.f;
  const float gl = g.gate_headwise ? to_f32(gate[orow]) : to_f32(gate[orow * D + d]);
  if (cp.out_f32)
    cp.out_f32[orow * D + d] = sigmoidf_(gl) * val;
  else
    out[orow * D + d] = from_f32<T>(sigmoidf_(gl) * val);
  if (lse && d == 0) lse[orow] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
}

// ------------------------------------------------------------ launchers
cudaError_t launch_attn_prefill_simt(qsa_dtype dt, const Geom& g, const int* cu, int batch,
                                     int max_seqlen, const void* q, const void* k, const void* v,
                                     const void* gate, const int* sel, const int* nsel,
                                     void* out, float* lse, cudaStream_t st) {
  if (batch == 0 || max_seqlen == 0) return cudaSuccess;
  dim3 grid(max_seqlen, batch, g.Hkv);
#define QSA_AP(T, DD)                                                                     \
  attn_prefill_simt_kernel<T, DD><<<grid, 128, 0, st>>>(g, cu, (const T*)q, (const T*)k,  \
                                                        (const T*)v, (const T*)gate, sel, \
                                                        nsel, (T*)out, lse)
  if (dt == QSA_BF16) {
    if (g.D == 128) QSA_AP(__nv_bfloat16, 128); else QSA_AP(__nv_bfloat16, 64);
  } else {
    if (g.D == 128) QSA_AP(float, 128); else QSA_AP(float, 64);
  }
#undef QSA_AP
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_decode_combine(qsa_dtype dt, const Geom& g, int batch, int n_q, int cap,
                                  int nsplit, const int* kv_len, const float* part_ml,
                                  const float* part_o, const void* gate, void* out, float* lse,
                                  cudaStream_t st, CpShard cp) {
  if (batch == 0) return cudaSuccess;
  dim3 cgrid(n_q * g.Hq, batch);
#define QSA_CB(T, DD)                                                                     \
  decode_combine_kernel<T, DD><<<cgrid, DD, 0, st>>>(g, n_q, cap, nsplit, kv_len, part_ml,  \
                                                     part_o, (const T*)gate, (T*)out, lse, cp)
  if (dt == QSA_BF16) {
    if (g.D == 128) { QSA_CB(__nv_bfloat16, 128); } else { QSA_CB(__nv_bfloat16, 64); }
  } else {
    if (g.D == 128) { QSA_CB(float, 128); } else { QSA_CB(float, 64); }
  }
#undef QSA_CB
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_attn_decode_simt(qsa_dtype dt, const Geom& g, int batch, int n_q, int cap,
                                    int nsplit, int per_split, const int* kv_len, const void* q,
                                    const void* kc, const void* vc, const void* gate,
                                    const int* sel, const int* nsel, float* part_ml,
                                    float* part_o, void* out, float* lse, cudaStream_t st,
                                    CpShard cp) {
  if (batch == 0) return cudaSuccess;
  dim3 grid(nsplit, batch, g.Hkv);
  dim3 cgrid(n_q * g.Hq, batch);
#define QSA_AD(T, DD)                                                                       \
  attn_decode_simt_kernel<T, DD><<<grid, 128, 0, st>>>(g, n_q, cap, nsplit, per_split,      \
                                                       kv_len, (const T*)q, (const T*)kc,   \
                                                       (const T*)vc, sel, nsel, part_ml,    \
                                                       part_o, cp);                         \
  decode_combine_kernel<T, DD><<<cgrid, DD, 0, st>>>(g, n_q, cap, nsplit, kv_len, part_ml,  \
                                                     part_o, (const T*)gate, (T*)out, lse, cp)
  if (dt == QSA_BF16) {
    if (g.D == 128) { QSA_AD(__nv_bfloat16, 128); } else { QSA_AD(__nv_bfloat16, 64); }
  } else {
    if (g.D == 128) { QSA_AD(float, 128); } else { QSA_AD(float, 64); }
  }
#undef QSA_AD
  note_launch(2);
  return cudaGetLastError();
}

}  // namespace qsa
