/*
 * qsa.h -- C ABI of the B200 (sm_100a) Qwen Sparse Attention (QSA) library.
 *
 * QSA is gated grouped-query attention whose causal mask is intersected with a
 * per-query-token block selection (instagit "Native Backend Components for the
 * Qwen4-Generation Preview Family in MTPLX", section "Qwen Sparse Attention
 * (QSA)"; dev.to "Qwen4-Exp: How Per-Layer N-gram Embeddings and Sparse
 * Attention ...", section "Qwen Sparse Attention: Block-Level Selection ...").
 * For a query that sees n tokens of its sequence:
 *
 *   kbar[j]  = (1/B) * sum_{i<B} ik[j*B+i]                      complete blocks only
 *   s[j]     = c * sum_h w[h] * relu(iq[h] . kbar[j]),  j < floor(n/B)
 *   S        = top-(budget/B) blocks under (s desc, j asc)  U  tail [floor(n/B)*B, n)
 *   out[h]   = sigmoid(gate[h]) * softmax_{s in S}(scale * q[h] . k[s, h/G]) v[s, h/G]
 *
 * The indexer settings (per-head weights, no n_head scale, c = idx_dim^-0.5,
 * candidates = complete visible blocks) and the sigmoid gate on the output follow the
 * QSA block-composition commit text on the llama.cpp PR #27739 page.
 *
 * Conventions for every entry point
 * ---------------------------------
 * - Every pointer argument is a DEVICE pointer unless stated otherwise; the
 *   caller owns every buffer. The library never allocates device memory: the
 *   caller passes a workspace of at least the size the matching
 *   *_workspace_size() call returns (256-byte aligned).
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   All work is enqueued on it; no entry point synchronises the host, and no
 *   entry point reads device memory (lengths, offsets) on the host.
 * - Floating-point tensors are dense, row-major, in the config's dtype
 *   (QSA_F32 or QSA_BF16) except `iw` (always fp32) and the pooled caches
 *   (always fp32). Integer tensors are int32.
 * - Arguments are validated before any launch; a bad argument returns
 *   QSA_ERR_INVALID_ARG and a geometry outside the compiled kernels returns
 *   QSA_ERR_UNSUPPORTED, in both cases with nothing enqueued. A launch failure
 *   returns QSA_ERR_CUDA. qsa_last_error() gives a message for the calling
 *   host thread. No entry point throws, exits or traps.
 * - Supported on the GPU: head_dim in {64, 128}; block_size in {64, 128};
 *   budget a positive multiple of block_size with budget/block_size <= 64;
 *   num_q_heads % num_kv_heads == 0 with group size <= 16; idx_dim in {32, 64};
 *   idx_heads <= 16; at most 4096 blocks per sequence.
 */
#ifndef QSA_H_
#define QSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1,
  QSA_ERR_UNSUPPORTED = 2,
  QSA_ERR_WORKSPACE = 3,
  QSA_ERR_CUDA = 4
} qsa_status;

typedef enum { QSA_F32 = 0, QSA_BF16 = 1 } qsa_dtype;

/* QSA geometry. This metadata decides which memory attention may read, so it
 * is validated on every call (ramgpt "Porting Qwen4 to llama.cpp": QSA
 * metadata is part of the execution contract). */
typedef struct {
  int num_q_heads;     /* Hq */
  int num_kv_heads;    /* Hkv; query head h reads KV head h / (Hq/Hkv) */
  int head_dim;        /* D */
  int idx_heads;       /* Hi, indexer heads */
  int idx_dim;         /* di, indexer head dim (one indexer key row per token) */
  int block_size;      /* B, tokens per pooled block (the compression ratio) */
  int budget;          /* tokens; k = budget / B complete blocks are kept */
  float softmax_scale; /* attention logit scale; 0 => head_dim^-0.5 */
  float index_scale;   /* indexer score scale c; 0 => idx_dim^-0.5 */
  int gate_headwise;   /* 0: gate [.., Hq, D] elementwise; 1: gate [.., Hq] */
  qsa_dtype dtype;     /* dtype of q, k, v, iq, ik, gate, out */
  /* Indexer rotary embedding (llama.cpp PR #27739 page, QSA block-composition
   * commit text: the indexer scores the roped query against pooled keys that
   * take the same rope angles; instagit MTPLX page, "Multidimensional Rotary
   * Embeddings (M-RoPE)": for text it is the ordinary partial rotary
   * embedding). rope_dim = 0 turns it off. Otherwise the first rope_dim dims
   * (a multiple of 4, <= idx_dim) of every indexer query and pooled key are
   * turned in pairs (f, f + rope_dim/2) by the fp32 angle pos * fp32(rope_theta
   * ^ (-2f / rope_dim)): an indexer query at its own position (its token index
   * in the sequence), the pooled key of block j at position j * B. The caches
   * hold the raw indexer keys; the pooled-key cache and pooled_out hold the
   * turned means. Every call that pools or scores must be given the same two
   * values. */
  int rope_dim;
  float rope_theta;    /* > 0 when rope_dim > 0 */
} qsa_config;

/* Human-readable name of a status code (static storage). */
const char* qsa_status_string(qsa_status s);

/* Message describing the last failed call on this host thread ("" if none). */
const char* qsa_last_error(void);

/* Library ABI version: 100 * major + minor. */
int qsa_version(void);

/* Number of kernels the library has launched since it was loaded (all host
 * threads). Used to check that work really ran in the library's kernels. */
unsigned long long qsa_kernel_launch_count(void);

/* Profiling hook for the calling host thread: with count > 0, later calls of
 * qsa_prefill / qsa_decode on this thread record events[0] when their first
 * kernel is enqueued, events[1] before the attention kernel(s) and events[2]
 * after the last kernel, all on the call's stream. `events` are cudaEvent_t
 * handles created by the caller, passed as void*; count = 0 turns it off.
 * Returns QSA_ERR_INVALID_ARG for count outside [0, 4]. */
qsa_status qsa_set_stage_events(void* const* events, int count);

/* Debug counter of visited keys for the calling host thread (the keys_visited
 * count of the llama.cpp PR #27739 page's QSA commit text, 16400 sparse against
 * 24016 dense in its worked example). With counter != NULL (device memory, 8
 * bytes, owned and zeroed by the caller) the attention kernels of later
 * qsa_prefill / qsa_decode* / qsa_decode_attend / qsa_cp_attend calls on this
 * thread add to *counter the number of (query, head, key) triples they attend
 * over, counted where each kernel decides which keys a row sees: for a correct
 * sparse consumer that is sum over queries of Hq * (min(k, nc) * B + tail),
 * whatever extra work the kernel's tiles execute. NULL turns it off (the
 * default; the counting adds one register and one atomic per warp). The
 * pointer is baked into the launches: a CUDA graph captured while it is set
 * keeps adding to it on every replay. The counter must be memory of the GPU
 * the calls run on. */
void qsa_set_keys_visited(unsigned long long* counter);

/* ---------------------------------------------------------------- prefill --
 * Packed variable-length prefill. Sequence b owns tokens
 * [cu_seqlens[b], cu_seqlens[b+1]); query token t at position p of its
 * sequence sees n = p + 1 tokens (causal).
 *
 *   cu_seqlens  [batch+1] int32 (device), non-decreasing, cu_seqlens[0] = 0,
 *               cu_seqlens[batch] = total_tokens, every length <= max_seqlen.
 *   q           [total_tokens, Hq, D]      k, v [total_tokens, Hkv, D]
 *   iq          [total_tokens, Hi, di]     ik   [total_tokens, di]
 *   iw          [total_tokens, Hi] fp32    gate [total_tokens, Hq, D] (or [.., Hq])
 *   out         [total_tokens, Hq, D]      (written)
 *   lse         optional [total_tokens, Hq] fp32: natural-log sum-exp of the
 *               scaled logits over the selected tokens (written)
 *   sel         optional [total_tokens, k+1] int32: the selected complete
 *               blocks in ascending order, then the tail block id floor(n/B)
 *               when n % B != 0, then -1 padding (written)
 *   nsel        optional [total_tokens] int32: min(k, floor(n/B)) + (n%B != 0)
 *   pooled_out  optional [batch, ceil(max_seqlen/B), di] fp32: pooled keys of
 *               every complete block (rows past a sequence's last complete
 *               block are left untouched)
 * total_tokens and max_seqlen are host integers that must describe the
 * device cu_seqlens; a device length above max_seqlen is not detected.
 * The first 4 bytes of the workspace receive an int32 error word: 0 once the
 * call has run, non-zero if a kernel gave up on one of its bounded waits
 * (a pipeline that stopped making progress); the outputs are then invalid. */
size_t qsa_prefill_workspace_size(const qsa_config* cfg, int batch, int total_tokens,
                                  int max_seqlen);

qsa_status qsa_prefill(const qsa_config* cfg, int batch, int total_tokens, int max_seqlen,
                       const int32_t* cu_seqlens, const void* q, const void* k,
                       const void* v, const void* iq, const void* ik, const float* iw,
                       const void* gate, void* out, float* lse, int32_t* sel,
                       int32_t* nsel, float* pooled_out, void* workspace,
                       size_t workspace_bytes, void* stream);

/* Selection only, for packed prefill geometry (same arguments as qsa_prefill).
 * scores: optional [total_tokens, max_seqlen/B] fp32; entry j of query t is
 * the indexer score s[j] for j < floor(n/B) and -inf beyond. */
qsa_status qsa_select(const qsa_config* cfg, int batch, int total_tokens, int max_seqlen,
                      const int32_t* cu_seqlens, const void* iq, const void* ik,
                      const float* iw, int32_t* sel, int32_t* nsel, float* scores,
                      float* pooled_out, void* workspace, size_t workspace_bytes,
                      void* stream);

/* ----------------------------------------------------------------- decode --
 * One decode step for `batch` sequences, each with n_q new query tokens
 * (n_q = 1 plain decode, n_q = 2 MTP verification of one draft token).
 * The caller has already appended this step's K, V and indexer-key rows to
 * the caches; kv_len[b] counts the rows present after that append, and new
 * query i of sequence b sees n = kv_len[b] - n_q + 1 + i tokens.
 *
 *   kv_len        [batch] int32 (device), n_q <= kv_len[b] <= cap
 *   q             [batch, n_q, Hq, D]     gate [batch, n_q, Hq, D] (or [.., Hq])
 *   k_cache/v_cache [batch, cap, Hkv, D]  ik_cache [batch, cap, di]
 *   iq            [batch, n_q, Hi, di]    iw [batch, n_q, Hi] fp32
 *   pooled_cache  [batch, cap/B, di] fp32, in/out: rows of blocks completed
 *                 before this step must hold their pooled keys (qsa_prefill's
 *                 pooled_out or qsa_pool_build give them); this call writes the
 *                 rows of the blocks its n_q tokens complete.
 *   out           [batch, n_q, Hq, D] (written); lse/sel/nsel as for prefill,
 *                 with a leading [batch, n_q] instead of [total_tokens].
 *   dev_err       optional int32 (device): set to a non-zero code when a
 *                 kv_len entry is out of range; those sequences are skipped.
 * cap must be a multiple of B.
 * Execution: on bf16 geometries with head_dim 128, n_q * G <= 32 and a cache
 * whose selection keys fit the kernel's shared memory (about 12000 blocks per
 * sequence), the step is one kernel launch (each (sequence, KV head)
 * thread-block cluster selects, gathers and merges in on-chip memory);
 * otherwise a selection kernel and an attention kernel. Results are the same
 * either way. */
size_t qsa_decode_workspace_size(const qsa_config* cfg, int batch, int n_q, int cap);

qsa_status qsa_decode(const qsa_config* cfg, int batch, int n_q, int cap,
                      const int32_t* kv_len, const void* q, const void* k_cache,
                      const void* v_cache, const void* iq, const void* ik_cache,
                      const float* iw, const void* gate, float* pooled_cache, void* out,
                      float* lse, int32_t* sel, int32_t* nsel, int32_t* dev_err,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Decode attention over selections the caller provides: qsa_decode without
 * its selection step (no pooling, no scoring). Used by a context-parallel
 * decode, where each process attends its share of a global selection over its
 * shard of the cache.
 *   sel   [batch, n_q, k + 1] int32 (device): block ids of the caches for each
 *         new query, ascending; the first nsel[b, i] entries are used. Ids
 *         outside [0, cap / B) are ignored. A listed block is attended over the
 *         positions the query can see (keys below kv_len - n_q + 1 + i); the
 *         caller lists the query's incomplete block if it is to be attended.
 *   nsel  [batch, n_q] int32 (device).
 * Other arguments, the outputs and the workspace as qsa_decode; a query with
 * no listed block gets out = 0 and lse = -inf. */
qsa_status qsa_decode_attend(const qsa_config* cfg, int batch, int n_q, int cap,
                             const int32_t* kv_len, const void* q, const void* k_cache,
                             const void* v_cache, const void* gate, const int32_t* sel,
                             const int32_t* nsel, void* out, float* lse, int32_t* dev_err,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Selection only, for decode geometry (same arguments as qsa_decode; it also
 * finalises the pooled rows completed by this step). scores: optional
 * [batch, n_q, cap/B] fp32, -inf past a query's candidates. */
qsa_status qsa_select_decode(const qsa_config* cfg, int batch, int n_q, int cap,
                             const int32_t* kv_len, const void* iq, const void* ik_cache,
                             const float* iw, float* pooled_cache, int32_t* sel,
                             int32_t* nsel, float* scores, int32_t* dev_err,
                             void* workspace, size_t workspace_bytes, void* stream);

/* qsa_decode without a workspace argument. The pages describe nothing like
 * it; it exists for callers that cannot allocate device memory for scratch,
 * such as a host program whose own allocator owns all of the GPU's memory, or
 * a latency-critical loop that must never call cudaMalloc. The scratch comes
 * from a 4 MiB array the library declares statically in device memory: every
 * GPU that loads the library holds it until the process exits, and this call
 * allocates nothing. Arguments are those of qsa_decode minus the workspace.
 * - A geometry whose qsa_decode_workspace_size() exceeds 4 MiB returns
 *   QSA_ERR_WORKSPACE (qsa_last_error() says how much it needs).
 * - The first call on a device looks up the array's device address (once per
 *   device, with that device current), so make the first call on each device
 *   before any stream capture. The address is kept for the life of the
 *   process: after cudaDeviceReset() on a device, this entry point must not be
 *   called on that device again. Devices with ordinal 64 or more are refused
 *   (QSA_ERR_UNSUPPORTED).
 * - All calls on a device share the one array, which keeps the last call's
 *   contents (no part of it needs to start at zero): calls that overlap on the
 *   GPU, on different streams or host threads, race and corrupt each other. */
qsa_status qsa_decode_noalloc(const qsa_config* cfg, int batch, int n_q, int cap,
                              const int32_t* kv_len, const void* q, const void* k_cache,
                              const void* v_cache, const void* iq, const void* ik_cache,
                              const float* iw, const void* gate, float* pooled_cache,
                              void* out, float* lse, int32_t* sel, int32_t* nsel,
                              int32_t* dev_err, void* stream);

/* ----------------------------------------------- context-parallel decode --
 * A sequence whose KV cache does not fit one GPU is split by blocks over the
 * processes of a group, one per GPU (the pages describe no multi-GPU QSA; the
 * split follows the step's data dependencies). The process with shard
 * [block_lo, block_lo + cap / B) holds cache rows [block_lo * B, block_lo * B
 * + cap) of every sequence at local rows 0 .. cap - 1: k_shard, v_shard
 * [batch, cap, Hkv, D], ik_shard [batch, cap, di], pooled_shard
 * [batch, cap / B, di] (the shard's pooled keys, as qsa_cp_pool_build writes
 * them). kv_len [batch] are the sequences' FULL lengths after this
 * step's n_q tokens were appended (to the shard that holds those rows); a
 * shard may hold none, some or all of a sequence's visible rows. One step:
 *   1. qsa_cp_select on every process: pools the shard's blocks completed by
 *      this step, scores the shard's complete visible blocks, and writes each
 *      query's top-k of them as candidates;
 *   2. the caller all-gathers the candidates (cand_score, cand_id) of every
 *      process into [world, batch, n_q, k] arrays, ordered by process;
 *   3. qsa_cp_global_topk: the global selection, identical to qsa_decode's
 *      (every globally selected block is in its own shard's top-k);
 *   4. qsa_cp_attend on every process: gated attention over the selected
 *      blocks inside the shard, as fp32 partials with their log-sum-exp;
 *   5. the caller all-gathers the partials, and qsa_cp_merge merges them by
 *      log-sum-exp (the sigmoid gate commutes with the weighted sum).
 * The scores are computed by the same arithmetic as qsa_decode's, so the
 * selection is bit-identical to the single-GPU one.
 *
 * qsa_cp_select: iq [batch, n_q, Hi, di], iw [batch, n_q, Hi] fp32 as for
 *   qsa_decode; writes the pooled rows of the shard's blocks this step
 *   completes, and cand_score [batch, n_q, k] fp32 / cand_id [batch, n_q, k]
 *   int32 (global block ids; -inf / -1 in unused slots, k = budget / B). The
 *   workspace is qsa_decode_workspace_size(cfg, batch, n_q, cap)'s.
 *   dev_err (optional) is set if a kernel finds an inconsistent length. */
qsa_status qsa_cp_select(const qsa_config* cfg, int batch, int n_q, int cap, int block_lo,
                         const int32_t* kv_len, const void* iq, const void* ik_shard,
                         const float* iw, float* pooled_shard, float* cand_score,
                         int32_t* cand_id, int32_t* dev_err, void* workspace,
                         size_t workspace_bytes, void* stream);

/* qsa_cp_pool_build: (re)builds pooled_shard [batch, cap / B, di] from
 * ik_shard for every block of the shard that is complete under kv_len [batch]
 * (FULL lengths, as for qsa_cp_select: the shard holds min(max(kv_len -
 * block_lo * B, 0), cap) of a sequence's rows). The same bits as qsa_pool_build
 * of the whole cache, rows [block_lo, block_lo + cap / B); with the indexer
 * rotary embedding, block j of the shard turns at its global position
 * (block_lo + j) * B. Rows of blocks that are not complete are not written. */
qsa_status qsa_cp_pool_build(const qsa_config* cfg, int batch, int cap, int block_lo,
                             const int32_t* kv_len, const void* ik_shard, float* pooled_shard,
                             int32_t* dev_err, void* stream);

/* qsa_cp_global_topk: cand_score / cand_id [world, batch, n_q, k] gathered
 * from every process; writes sel [batch, n_q, k + 1] (global ids of the
 * selected complete blocks in ascending order, then the query's tail block
 * floor(n / B) when n % B != 0, then -1) and nsel [batch, n_q], exactly as
 * qsa_decode writes them. Supported: world * k <= 4096. */
qsa_status qsa_cp_global_topk(const qsa_config* cfg, int batch, int n_q, int world,
                              const int32_t* kv_len, const float* cand_score,
                              const int32_t* cand_id, int32_t* sel, int32_t* nsel,
                              void* stream);

/* qsa_cp_attend: attention of q [batch, n_q, Hq, D] over the blocks of the
 * global selection (sel / nsel from qsa_cp_global_topk) that lie in this
 * shard, each over the positions the query sees; part_out [batch, n_q, Hq, D]
 * fp32 receives the gated partial output and part_lse [batch, n_q, Hq] fp32
 * its natural-log sum-exp (-inf and 0 where the shard holds none of the
 * query's keys). Workspace as qsa_cp_select. Every geometry qsa_decode
 * supports; bf16 with head_dim 128 and n_q * (Hq / Hkv) <= 32 runs on the
 * tensor-map kernel, the rest on the CUDA-core kernels. */
qsa_status qsa_cp_attend(const qsa_config* cfg, int batch, int n_q, int cap, int block_lo,
                         const int32_t* kv_len, const void* q, const void* k_shard,
                         const void* v_shard, const void* gate, const int32_t* sel,
                         const int32_t* nsel, float* part_out, float* part_lse,
                         int32_t* dev_err, void* workspace, size_t workspace_bytes,
                         void* stream);

/* qsa_cp_merge: part_out [world, batch, n_q, Hq, D] fp32 and part_lse
 * [world, batch, n_q, Hq] gathered from every process; writes out
 * [batch, n_q, Hq, D] in the config's dtype and lse (optional) [batch, n_q,
 * Hq]. */
qsa_status qsa_cp_merge(const qsa_config* cfg, int batch, int n_q, int world,
                        const float* part_out, const float* part_lse, void* out, float* lse,
                        void* stream);

/* --------------------------------------------------------- paged decode --
 * qsa_decode over a paged KV cache (the llama.cpp PR #27739 page names paged
 * KV storage, next to continuous batching, among its speed levers; the QSA
 * block is the page).
 * A page holds the B consecutive rows of one block of one sequence:
 *   k_pages/v_pages [num_pages, B, Hkv, D]   ik_pages [num_pages, B, di]
 *   block_table     [batch, max_blocks] int32 (device): block j of sequence b
 *                   lives in page block_table[b * max_blocks + j]. Entries of
 *                   blocks past the sequence's last token are not read.
 * Everything else is as for qsa_decode with cap = max_blocks * B (pooled_cache
 * [batch, max_blocks, di]; the workspace size is
 * qsa_decode_workspace_size(cfg, batch, n_q, max_blocks * B)). The results
 * are bit-identical to qsa_decode on the same rows laid out contiguously.
 * A page id outside [0, num_pages) among a sequence's blocks sets *dev_err
 * to 3 (that sequence's outputs are then unspecified, and nothing outside the
 * pools is read). Supported: bf16, head_dim 128, n_q * (Hq / Hkv) <= 32;
 * otherwise QSA_ERR_UNSUPPORTED. */
qsa_status qsa_decode_paged(const qsa_config* cfg, int batch, int n_q, int max_blocks,
                            const int32_t* block_table, int num_pages, const int32_t* kv_len,
                            const void* q, const void* k_pages, const void* v_pages,
                            const void* iq, const void* ik_pages, const float* iw,
                            const void* gate, float* pooled_cache, void* out, float* lse,
                            int32_t* sel, int32_t* nsel, int32_t* dev_err, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------ fp8 decode --
 * qsa_decode over fp8 K/V caches (ramgpt "Porting Qwen4 to llama.cpp",
 * section "Quantized KV Is a Representation Contract": quantized K/V may be
 * stored in a Hadamard-rotated basis, and a fast attention path must honour
 * that storage contract).
 *   k_cache/v_cache [batch, cap, Hkv, D] uint8: e4m3 codes (OCP FP8 E4M3,
 *                   no infinities; code 0x7F/0xFF is NaN)
 *   k_scale/v_scale [batch, cap, Hkv] fp32: the row (token, KV head) stands
 *                   for scale * decode(code), elementwise over D
 *   rotated         0: the rows are k and v; non-zero: they are H k and H v
 *                   for the orthonormal Walsh-Hadamard matrix of order D
 *                   (Sylvester order, scaled by D^-1/2). The query is
 *                   rotated and the output rotated back inside the kernel, so
 *                   out is the attention over k and v either way.
 * q, gate, iq, ik_cache and the rest are as for qsa_decode (bf16; the indexer
 * path is unchanged); the workspace is qsa_decode_workspace_size's. K/V are
 * widened to fp16 times the scale before the MMAs; accumulation is fp32.
 * Supported: bf16 config, head_dim 128, Hkv <= 8, n_q * (Hq / Hkv) <= 16;
 * otherwise QSA_ERR_UNSUPPORTED. */
qsa_status qsa_decode_fp8(const qsa_config* cfg, int batch, int n_q, int cap,
                          const int32_t* kv_len, const void* q, const void* k_cache,
                          const float* k_scale, const void* v_cache, const float* v_scale,
                          int rotated, const void* iq, const void* ik_cache, const float* iw,
                          const void* gate, float* pooled_cache, void* out, float* lse,
                          int32_t* sel, int32_t* nsel, int32_t* dev_err, void* workspace,
                          size_t workspace_bytes, void* stream);

/* qsa_pool_build for a paged indexer-key cache (arguments as for
 * qsa_decode_paged); the rows it writes are bit-identical to qsa_pool_build's
 * on the same rows laid out contiguously. A bad page id sets *dev_err to 3
 * and leaves that block's pooled row untouched. */
qsa_status qsa_pool_build_paged(const qsa_config* cfg, int batch, int max_blocks,
                                const int32_t* block_table, int num_pages,
                                const int32_t* kv_len, const void* ik_pages,
                                float* pooled_cache, int32_t* dev_err, void* stream);

/* Indexer front end of a decode step (one launch): writes the step's n_q new
 * rows into the caches and, in the same pass, pools (and, with the indexer
 * rotary embedding, turns) every block those rows complete, the bits of
 * qsa_pool_build. Rows go to cache positions kv_len[b] - n_q + i (kv_len the
 * post-append lengths, device [batch]); the block's earlier rows are read from
 * the cache, its new rows from the inputs. Inputs: ik_new [batch, n_q, di];
 * k_new, v_new [batch, n_q, Hkv, D] (both NULL: only the indexer keys are
 * appended), all in cfg->dtype. Caches: block_table NULL: ik_cache
 * [batch, cap, di], k_cache / v_cache [batch, cap, Hkv, D], pooled_cache
 * [batch, cap / B, di] fp32; block_table [batch, cap / B] int32: paged caches
 * of num_pages pages of B rows ([num_pages, B, di], [num_pages, B, Hkv, D]).
 * A following qsa_decode (or its paged form) on the same lengths pools the same
 * blocks again to the same bits (the write-back is idempotent). Errors: a
 * length outside [n_q, cap] sets *dev_err to 1 and writes nothing for that
 * sequence; a bad page id sets it to 3 and skips that row or block. */
qsa_status qsa_append(const qsa_config* cfg, int batch, int n_q, int cap, const int32_t* kv_len,
                      const void* k_new, const void* v_new, const void* ik_new, void* k_cache,
                      void* v_cache, void* ik_cache, float* pooled_cache,
                      const int32_t* block_table, int num_pages, int32_t* dev_err, void* stream);

/* Rebuild the pooled-key cache of every complete block j < kv_len[b]/B from
 * the indexer-key cache (restore after a state reload). The rows it writes are
 * bit-identical to the ones the incremental decode path writes. */
qsa_status qsa_pool_build(const qsa_config* cfg, int batch, int cap, const int32_t* kv_len,
                          const void* ik_cache, float* pooled_cache, int32_t* dev_err,
                          void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H_ */
