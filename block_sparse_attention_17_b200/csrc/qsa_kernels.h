// Internal launcher declarations shared by the kernel files and the C ABI.
#pragma once

#include <utility>

#include <cuda_runtime.h>
#include <stdint.h>

#include "qsa.h"

namespace qsa {

struct Geom;

// Paged caches: block j of sequence b lives in page table[b * (cap / B) + j]
// of a pool of num_pages pages of B rows each. table == nullptr: contiguous
// [batch, cap] caches.
struct Pages {
  const int* table = nullptr;
  int num_pages = 0;
};

// Counts kernel launches made by the library (all host threads).
void note_launch(int n = 1);

// Raises a kernel's dynamic shared memory limit on the current device, once per
// (kernel, device, size) instead of on every launch.
cudaError_t set_max_dynamic_smem(const void* func, int bytes);

// CTAs of `func` (threads, dynamic shared memory) resident per SM, and the
// SM count of the current device (cached per function, device and shape).
cudaError_t resident_ctas(const void* func, int threads, size_t smem, int* per_sm, int* sms);

// fp8 (e4m3) K/V caches for the decode attention: one fp32 scale per
// (token, KV head) row, [batch, cap, Hkv]; rotated != 0 when the caches hold
// H k and H v for the orthonormal Walsh-Hadamard matrix H of order D.
struct Fp8Kv {
  bool on = false;
  const float* k_scale = nullptr;
  const float* v_scale = nullptr;
  int rotated = 0;
};

// Context-parallel decode: this process holds the rows [row_off, row_off +
// cap) of every sequence (blocks [block_lo, ...), row_off = block_lo * B);
// kv_len stays the sequences' full lengths. The selection kernel then scores
// the shard's complete visible blocks and writes each query's top-k of them
// as candidates (cand_score: the scores, cand_id: global block ids; -inf / -1
// padding); the attention kernel reads global block ids, attends those inside
// the shard, and writes fp32 gated partials (out_f32) with their lse.
struct CpShard {
  bool on = false;
  int row_off = 0;
  int block_lo = 0;
  float* cand_score = nullptr;
  int* cand_id = nullptr;
  float* out_f32 = nullptr;
};

// ready: [batch] flags the selection kernel sets (release) once a sequence's
// selections are written, zero before the launch; the decode attention kernel
// waits on its sequence's flag instead of on the whole selection grid.

// Launches `kernel` on `st` with programmatic stream serialization: it may
// start before the previous kernel on the stream finishes, and must call
// grid_dependency_wait() before reading that kernel's outputs.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Sets the message qsa_last_error() returns on this host thread.
void set_last_error(const char* msg);

cudaError_t launch_pool_prefill(qsa_dtype dt, const void* ik, const int* cu, int batch,
                                int max_seqlen, const Geom& g, float* pooled, int max_nblk,
                                cudaStream_t st);
cudaError_t launch_pool_cache(qsa_dtype dt, const void* ik_cache, const int* kv_len, int batch,
                              int cap, int n_q, int mode, const Geom& g, float* pooled,
                              int* dev_err, cudaStream_t st, Pages pg = Pages(),
                              int block_lo = -1);
// Appends the step's new K / V (optional: k_new == nullptr) and indexer-key
// rows and pools the blocks they complete (one launch).
cudaError_t launch_append(qsa_dtype dt, const Geom& g, int batch, int n_q, int cap,
                          const int* kv_len, const void* k_new, const void* v_new,
                          const void* ik_new, void* k_cache, void* v_cache, void* ik_cache,
                          float* pooled, int* dev_err, Pages pg, cudaStream_t st);
size_t select_prefill_smem(const Geom& g, int nc_cap);
// sched: one int the caller zeroed on the stream before the launch (the
// kernel's work counter).
cudaError_t launch_select_prefill(qsa_dtype dt, const Geom& g, const int* cu, int batch,
                                  int max_seqlen, int max_nblk, int words, const void* iq,
                                  const float* iw, const float* pooled, int* sched, int* sel,
                                  int* nsel, uint32_t* bitmask, float* scores, int scores_ld,
                                  cudaStream_t st);
int decode_select_parts(const Geom& g, int cap);
cudaError_t launch_decode_select(qsa_dtype dt, const Geom& g, int batch, int n_q, int cap,
                                 const int* kv_len, const void* iq, const void* ik_cache,
                                 const float* iw, float* pooled, float* scores_out,
                                 uint32_t* keys_ws, int* counter, int* sel, int* nsel,
                                 int* dev_err, cudaStream_t st, Pages pg = Pages(),
                                 int* ready = nullptr, CpShard cp = CpShard());
cudaError_t launch_attn_prefill_simt(qsa_dtype dt, const Geom& g, const int* cu, int batch,
                                     int max_seqlen, const void* q, const void* k, const void* v,
                                     const void* gate, const int* sel, const int* nsel,
                                     void* out, float* lse, cudaStream_t st);
cudaError_t launch_attn_decode_simt(qsa_dtype dt, const Geom& g, int batch, int n_q, int cap,
                                    int nsplit, int per_split, const int* kv_len, const void* q,
                                    const void* kc, const void* vc, const void* gate,
                                    const int* sel, const int* nsel, float* part_ml,
                                    float* part_o, void* out, float* lse, cudaStream_t st,
                                    CpShard cp = CpShard());

cudaError_t launch_decode_combine(qsa_dtype dt, const Geom& g, int batch, int n_q, int cap,
                                  int nsplit, const int* kv_len, const float* part_ml,
                                  const float* part_o, const void* gate, void* out, float* lse,
                                  cudaStream_t st, CpShard cp = CpShard());
bool attn_decode_mma_supported(const Geom& g, int n_q);
void decode_mma_split(const Geom& g, int batch, int n_q, int* nsplit, int* per_split);
cudaError_t launch_attn_decode_mma(const Geom& g, int batch, int n_q, int cap, int nsplit,
                                   int per_split, const int* kv_len, const void* q,
                                   const void* kc, const void* vc, const void* gate,
                                   const int* sel, const int* nsel, float* part_ml,
                                   float* part_o, int* counter, void* out, float* lse, int* err,
                                   cudaStream_t st, Pages pg = Pages(), const int* ready = nullptr,
                                   Fp8Kv f8 = Fp8Kv(), CpShard cp = CpShard());
bool attn_decode_fp8_supported(const Geom& g, int n_q);

// The selection of a decode step done inside the decode attention kernel (one
// launch per step): the indexer inputs, the pooled-key cache the kernel updates
// and reads, and the selection lists it writes ([batch, n_q, k + 1], [batch, n_q]).
struct DecodeSelIn {
  const void* iq = nullptr;
  const void* ik_cache = nullptr;
  const float* iw = nullptr;
  float* pooled = nullptr;
  int* sel = nullptr;
  int* nsel = nullptr;
};
// Whether launch_decode_fused can run this geometry (bf16, the tensor-map
// decode path, indexer dim 32 or 64, the selection's shared memory within the
// ring, a resident cluster of nsplit CTAs).
bool decode_fused_supported(const Geom& g, int n_q, int cap, int nsplit, bool fp8);
cudaError_t launch_decode_fused(const Geom& g, int batch, int n_q, int cap, int nsplit,
                                int per_split, const int* kv_len, const void* q, const void* kc,
                                const void* vc, const void* gate, const DecodeSelIn& si,
                                void* out, float* lse, int* err, cudaStream_t st,
                                Pages pg = Pages(), Fp8Kv f8 = Fp8Kv());
bool attn_prefill_tc_supported(const Geom& g);
// Context-parallel decode: the global top-k over every process's candidates
// ([world, batch, n_q, k] scores and global ids) plus each query's tail block
// (sel [batch, n_q, k + 1], nsel [batch, n_q], as qsa_decode writes them), and
// the log-sum-exp merge of the processes' gated fp32 partials.
cudaError_t launch_cp_global_topk(const Geom& g, int batch, int n_q, int world,
                                  const int* kv_len, const float* cand_score,
                                  const int* cand_id, int* sel, int* nsel, cudaStream_t st);
cudaError_t launch_cp_merge(qsa_dtype dt, int rows, int D, int world, const float* part_out,
                            const float* part_lse, void* out, float* lse, cudaStream_t st);
cudaError_t launch_attn_prefill_tc(const Geom& g, const int* cu, int batch, int total_tokens,
                                   int max_seqlen, int words, const uint32_t* bitmask,
                                   const void* q, const void* k, const void* v, const void* gate,
                                   void* out, float* lse, int* err, cudaStream_t st);

}  // namespace qsa
