// C ABI of the QSA library: argument validation, workspace carving and the
// launch sequence of each entry point. Nothing here reads device memory or
// synchronises the host; every kernel goes to the caller's stream.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "qsa_common.cuh"
#include "qsa_kernels.h"
#include <nvtx3/nvToolsExt.h>

// An NVTX range over one library call or one of its stages (shown by Nsight
// Systems and usable as an ncu filter; a no-op unless a tool is attached).
namespace {
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace
#define QSA_NVTX_CAT2(a, b) a##b
#define QSA_NVTX_CAT(a, b) QSA_NVTX_CAT2(a, b)
#define QSA_NVTX(name) NvtxRange QSA_NVTX_CAT(qsa_nvtx_range_, __LINE__)(name)

using namespace qsa;

namespace {
std::atomic<unsigned long long> g_launches{0};
}  // namespace

void qsa::note_launch(int n) { g_launches.fetch_add((unsigned long long)n); }

cudaError_t qsa::set_max_dynamic_smem(const void* func, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(func, dev);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[key] = bytes;
  return e;
}

cudaError_t qsa::resident_ctas(const void* func, int threads, size_t smem, int* per_sm,
                               int* sms) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int, size_t>, std::pair<int, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(func, dev, threads, smem);
  auto it = done.find(key);
  if (it != done.end()) {
    *per_sm = it->second.first;
    *sms = it->second.second;
    return cudaSuccess;
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, func, threads, smem);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  done[key] = std::make_pair(*per_sm, *sms);
  return cudaSuccess;
}

namespace {

// Optional profiling events (per host thread): recorded on the call's stream
// at stage boundaries, see qsa_set_stage_events().
thread_local cudaEvent_t g_stage_ev[4] = {nullptr, nullptr, nullptr, nullptr};
thread_local int g_stage_n = 0;

void stage_mark(int i, cudaStream_t st) {
  if (i < g_stage_n && g_stage_ev[i]) cudaEventRecord(g_stage_ev[i], st);
}

thread_local char g_err[512] = "";
thread_local unsigned long long* g_keys_visited = nullptr;   // see qsa_set_keys_visited()

qsa_status fail(qsa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

}  // namespace

void qsa::set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

namespace {

qsa_status cuda_fail(cudaError_t e, const char* where) {
  return fail(QSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr int kMaxDecodeQ = 4;
constexpr int kMaxDecodeRows = 32;
constexpr int kTargetCtas = 2 * 148;

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

qsa_status check_cfg(const qsa_config* c) {
  if (!c) return fail(QSA_ERR_INVALID_ARG, "cfg is NULL");
  if (c->num_q_heads <= 0 || c->num_kv_heads <= 0 || c->head_dim <= 0 || c->idx_heads <= 0 ||
      c->idx_dim <= 0 || c->block_size <= 0 || c->budget <= 0)
    return fail(QSA_ERR_INVALID_ARG, "geometry fields must be positive");
  if (c->num_q_heads % c->num_kv_heads)
    return fail(QSA_ERR_INVALID_ARG, "num_q_heads %% num_kv_heads != 0");
  if (c->budget % c->block_size)
    return fail(QSA_ERR_INVALID_ARG, "budget must be a multiple of block_size");
  if (c->dtype != QSA_F32 && c->dtype != QSA_BF16)
    return fail(QSA_ERR_INVALID_ARG, "unknown dtype %d", (int)c->dtype);
  if (c->softmax_scale < 0.f || c->index_scale < 0.f || !isfinite(c->softmax_scale) ||
      !isfinite(c->index_scale))
    return fail(QSA_ERR_INVALID_ARG, "scales must be finite and >= 0 (0 = default)");
  if (c->num_q_heads / c->num_kv_heads > 16)
    return fail(QSA_ERR_UNSUPPORTED, "group size Hq/Hkv > 16");
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(QSA_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", c->head_dim);
  if (c->block_size != 64 && c->block_size != 128)
    return fail(QSA_ERR_UNSUPPORTED, "block_size %d (supported: 64, 128)", c->block_size);
  if (c->budget / c->block_size > kMaxTopK)
    return fail(QSA_ERR_UNSUPPORTED, "budget/block_size > %d", kMaxTopK);
  if (c->idx_dim != 32 && c->idx_dim != 64)
    return fail(QSA_ERR_UNSUPPORTED, "idx_dim %d (supported: 32, 64)", c->idx_dim);
  if (c->idx_heads > 16) return fail(QSA_ERR_UNSUPPORTED, "idx_heads > 16");
  if (c->rope_dim < 0 || c->rope_dim > c->idx_dim || (c->rope_dim & 3))
    return fail(QSA_ERR_INVALID_ARG, "rope_dim %d (a multiple of 4 in [0, idx_dim])", c->rope_dim);
  if (c->rope_dim > 0 && !(c->rope_theta > 0.f && isfinite(c->rope_theta)))
    return fail(QSA_ERR_INVALID_ARG, "rope_theta must be finite and > 0 when rope_dim > 0");
  return QSA_OK;
}

Geom make_geom(const qsa_config* c) {
  Geom g;
  g.Hq = c->num_q_heads;
  g.Hkv = c->num_kv_heads;
  g.G = g.Hq / g.Hkv;
  g.D = c->head_dim;
  g.Hi = c->idx_heads;
  g.di = c->idx_dim;
  g.B = c->block_size;
  g.k = c->budget / c->block_size;
  const float sm = c->softmax_scale > 0.f ? c->softmax_scale : 1.0f / sqrtf((float)g.D);
  g.sm_scale_log2 = sm * kLog2e;
  g.idx_scale = c->index_scale > 0.f ? c->index_scale : 1.0f / sqrtf((float)g.di);
  g.gate_headwise = c->gate_headwise ? 1 : 0;
  g.rope_dim = c->rope_dim;
  g.rope_theta = c->rope_dim > 0 ? c->rope_theta : 0.f;
  g.keys_visited = g_keys_visited;
  return g;
}

// Bump allocator over the caller's workspace; every region is 256-byte aligned.
struct Carve {
  char* base;
  size_t off = 0;
  explicit Carve(void* b) : base((char*)b) {}
  template <typename T> T* take(size_t count) {
    off = (off + 255) & ~(size_t)255;
    T* p = base ? (T*)(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

struct PrefillWs {
  int* err;             // error word, then the selection kernel's work counter
  int* sched;
  float* pooled;
  int* sel;
  int* nsel;
  uint32_t* bitmask;
  size_t bytes;
};

PrefillWs carve_prefill(const Geom& g, void* ws, int batch, int T, int max_seqlen) {
  const int max_nblk = (max_seqlen + g.B - 1) / g.B;
  const int words = (max_nblk + 31) / 32;
  Carve c(ws);
  PrefillWs w;
  w.err = c.take<int>(2);
  w.sched = w.err + 1;
  w.pooled = c.take<float>((size_t)batch * max_nblk * g.di);
  w.sel = c.take<int>((size_t)T * (g.k + 1));
  w.nsel = c.take<int>((size_t)T);
  w.bitmask = c.take<uint32_t>((size_t)T * words);
  w.bytes = (c.off + 255) & ~(size_t)255;
  return w;
}

struct DecodeWs {
  int* err;
  int* counters;        // [batch] selection + [batch * Hkv] attention + [batch] ready
                        // flags, zeroed per call
  uint32_t* keys;       // [batch, n_q, cap / B] score keys
  int* sel;
  int* nsel;
  float* part_ml;
  float* part_o;
  int nsplit, per_split;
  size_t bytes;
};

bool decode_uses_mma(const qsa_config* cfg, const Geom& g, int n_q) {
  return cfg->dtype == QSA_BF16 && attn_decode_mma_supported(g, n_q);
}

DecodeWs carve_decode(const qsa_config* cfg, const Geom& g, void* ws, int batch, int n_q,
                      int cap) {
  DecodeWs w;
  if (decode_uses_mma(cfg, g, n_q)) {
    decode_mma_split(g, batch, n_q, &w.nsplit, &w.per_split);
  } else {
    const int max_union = n_q * (g.k + 1);
    const int pairs = std::max(1, batch * g.Hkv);
    int nsplit = std::min(max_union, std::max(1, (kTargetCtas + pairs - 1) / pairs));
    w.per_split = (max_union + nsplit - 1) / nsplit;
    w.nsplit = (max_union + w.per_split - 1) / w.per_split;
  }
  const int R = n_q * g.G;
  Carve c(ws);
  w.err = c.take<int>(1);
  w.counters = c.take<int>((size_t)batch * (2 + g.Hkv));
  w.keys = c.take<uint32_t>((size_t)batch * n_q * (cap / g.B));
  w.sel = c.take<int>((size_t)batch * n_q * (g.k + 1));
  w.nsel = c.take<int>((size_t)batch * n_q);
  w.part_ml = c.take<float>((size_t)batch * g.Hkv * w.nsplit * R * 2);
  w.part_o = c.take<float>((size_t)batch * g.Hkv * w.nsplit * R * g.D);
  w.bytes = (c.off + 255) & ~(size_t)255;
  return w;
}

qsa_status check_prefill_dims(const qsa_config* cfg, int batch, int T, int max_seqlen) {
  qsa_status s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if (batch < 0 || T < 0 || max_seqlen < 0)
    return fail(QSA_ERR_INVALID_ARG, "batch, total_tokens and max_seqlen must be >= 0");
  if (T > 0 && (batch == 0 || max_seqlen == 0))
    return fail(QSA_ERR_INVALID_ARG, "total_tokens > 0 needs batch > 0 and max_seqlen > 0");
  if ((long long)max_seqlen > (long long)T && batch == 1)
    return fail(QSA_ERR_INVALID_ARG, "max_seqlen > total_tokens for a single sequence");
  if ((max_seqlen + cfg->block_size - 1) / cfg->block_size > kMaxBlocksPerSeq)
    return fail(QSA_ERR_UNSUPPORTED, "more than %d blocks per sequence", kMaxBlocksPerSeq);
  return QSA_OK;
}

qsa_status check_decode_dims(const qsa_config* cfg, int batch, int n_q, int cap) {
  qsa_status s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if (batch < 0 || n_q <= 0 || cap <= 0)
    return fail(QSA_ERR_INVALID_ARG, "batch >= 0, n_q > 0 and cap > 0 are required");
  if (cap % cfg->block_size) return fail(QSA_ERR_INVALID_ARG, "cap must be a multiple of B");
  if (cap / cfg->block_size > kMaxDecodeBlocksPerSeq)
    return fail(QSA_ERR_UNSUPPORTED, "more than %d cache blocks", kMaxDecodeBlocksPerSeq);
  if ((long long)batch * cap > 2147483647LL)
    return fail(QSA_ERR_UNSUPPORTED, "batch * cap must fit in 31 bits");
  if (n_q > kMaxDecodeQ) return fail(QSA_ERR_UNSUPPORTED, "n_q > %d", kMaxDecodeQ);
  if (n_q * (cfg->num_q_heads / cfg->num_kv_heads) > kMaxDecodeRows)
    return fail(QSA_ERR_UNSUPPORTED, "n_q * group size > %d", kMaxDecodeRows);
  // the decode selection sums a block's indexer heads over adjacent lanes of a warp
  if (cfg->idx_heads & (cfg->idx_heads - 1))
    return fail(QSA_ERR_UNSUPPORTED, "decode: idx_heads must be a power of two");
  return QSA_OK;
}

#define QSA_REQUIRE(p, name)                                                  \
  do {                                                                        \
    if (!(p)) return fail(QSA_ERR_INVALID_ARG, "%s is NULL", name);           \
    if (!aligned16(p)) return fail(QSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
  } while (0)

#define QSA_CUDA(call, where)                          \
  do {                                                 \
    cudaError_t e_ = (call);                           \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

}  // namespace

extern "C" {

const char* qsa_status_string(qsa_status s) {
  switch (s) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARG: return "QSA_ERR_INVALID_ARG";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED";
    case QSA_ERR_WORKSPACE: return "QSA_ERR_WORKSPACE";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA";
  }
  return "QSA_ERR_UNKNOWN";
}

const char* qsa_last_error(void) { return g_err; }

int qsa_version(void) { return 101; }

unsigned long long qsa_kernel_launch_count(void) { return g_launches.load(); }

void qsa_set_keys_visited(unsigned long long* counter) { g_keys_visited = counter; }

qsa_status qsa_set_stage_events(void* const* events, int count) {
  if (count < 0 || count > 4 || (count > 0 && !events))
    return fail(QSA_ERR_INVALID_ARG, "count must be in [0, 4] with non-NULL events");
  for (int i = 0; i < 4; ++i) g_stage_ev[i] = i < count ? (cudaEvent_t)events[i] : nullptr;
  g_stage_n = count;
  return QSA_OK;
}

size_t qsa_prefill_workspace_size(const qsa_config* cfg, int batch, int total_tokens,
                                  int max_seqlen) {
  if (check_prefill_dims(cfg, batch, total_tokens, max_seqlen) != QSA_OK) return 0;
  return carve_prefill(make_geom(cfg), nullptr, batch, total_tokens, max_seqlen).bytes;
}

static qsa_status prefill_select_common(const qsa_config* cfg, const Geom& g, int batch,
                                        int T, int max_seqlen, const int32_t* cu,
                                        const void* iq, const void* ik, const float* iw,
                                        const PrefillWs& w, float* pooled, int32_t* sel,
                                        int32_t* nsel, float* scores, cudaStream_t st) {
  const int max_nblk = (max_seqlen + g.B - 1) / g.B;
  const int words = (max_nblk + 31) / 32;
  // the error word and the selection's work counter start at zero
  QSA_CUDA(cudaMemsetAsync(w.err, 0, 2 * sizeof(int), st), "clear error word");
  QSA_CUDA(launch_pool_prefill(cfg->dtype, ik, cu, batch, max_seqlen, g, pooled, max_nblk, st),
           "pool");
  QSA_CUDA(launch_select_prefill(cfg->dtype, g, cu, batch, max_seqlen, max_nblk, words, iq, iw,
                                 pooled, w.sched, sel, nsel, w.bitmask, scores,
                                 std::max(1, max_seqlen / g.B), st),
           "select");
  return QSA_OK;
}

qsa_status qsa_prefill(const qsa_config* cfg, int batch, int total_tokens, int max_seqlen,
                       const int32_t* cu_seqlens, const void* q, const void* k, const void* v,
                       const void* iq, const void* ik, const float* iw, const void* gate,
                       void* out, float* lse, int32_t* sel, int32_t* nsel, float* pooled_out,
                       void* workspace, size_t workspace_bytes, void* stream) {
  QSA_NVTX("qsa_prefill");
  g_err[0] = 0;
  qsa_status s = check_prefill_dims(cfg, batch, total_tokens, max_seqlen);
  if (s != QSA_OK) return s;
  if (total_tokens == 0) return QSA_OK;
  QSA_REQUIRE(cu_seqlens, "cu_seqlens");
  QSA_REQUIRE(q, "q"); QSA_REQUIRE(k, "k"); QSA_REQUIRE(v, "v");
  QSA_REQUIRE(iq, "iq"); QSA_REQUIRE(ik, "ik"); QSA_REQUIRE(iw, "iw");
  QSA_REQUIRE(gate, "gate"); QSA_REQUIRE(out, "out");
  if (lse) QSA_REQUIRE(lse, "lse");
  if (sel) QSA_REQUIRE(sel, "sel");
  if (nsel) QSA_REQUIRE(nsel, "nsel");
  if (pooled_out) QSA_REQUIRE(pooled_out, "pooled_out");
  const Geom g = make_geom(cfg);
  const PrefillWs need = carve_prefill(g, nullptr, batch, total_tokens, max_seqlen);
  if (!workspace || workspace_bytes < need.bytes || ((uintptr_t)workspace & 255u))
    return fail(QSA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", need.bytes);
  const PrefillWs w = carve_prefill(g, workspace, batch, total_tokens, max_seqlen);
  cudaStream_t st = (cudaStream_t)stream;
  float* pooled = pooled_out ? pooled_out : w.pooled;
  int* sel_p = sel ? sel : w.sel;
  int* nsel_p = nsel ? nsel : w.nsel;
  stage_mark(0, st);
  {
    QSA_NVTX("pool + select");
    s = prefill_select_common(cfg, g, batch, total_tokens, max_seqlen, cu_seqlens, iq, ik, iw, w,
                              pooled, sel_p, nsel_p, nullptr, st);
  }
  if (s != QSA_OK) return s;
  stage_mark(1, st);
  QSA_NVTX("attention");
  if (cfg->dtype == QSA_BF16 && attn_prefill_tc_supported(g)) {
    const int max_nblk = (max_seqlen + g.B - 1) / g.B;
    QSA_CUDA(launch_attn_prefill_tc(g, cu_seqlens, batch, total_tokens, max_seqlen,
                                    (max_nblk + 31) / 32, w.bitmask, q, k, v, gate, out, lse,
                                    w.err, st),
             "attention (tensor cores)");
  } else {
    QSA_CUDA(launch_attn_prefill_simt(cfg->dtype, g, cu_seqlens, batch, max_seqlen, q, k, v,
                                      gate, sel_p, nsel_p, out, lse, st),
             "attention");
  }
  stage_mark(2, st);
  return QSA_OK;
}

qsa_status qsa_select(const qsa_config* cfg, int batch, int total_tokens, int max_seqlen,
                      const int32_t* cu_seqlens, const void* iq, const void* ik, const float* iw,
                      int32_t* sel, int32_t* nsel, float* scores, float* pooled_out,
                      void* workspace, size_t workspace_bytes, void* stream) {
  QSA_NVTX("qsa_select");
  g_err[0] = 0;
  qsa_status s = check_prefill_dims(cfg, batch, total_tokens, max_seqlen);
  if (s != QSA_OK) return s;
  if (total_tokens == 0) return QSA_OK;
  QSA_REQUIRE(cu_seqlens, "cu_seqlens");
  QSA_REQUIRE(iq, "iq"); QSA_REQUIRE(ik, "ik"); QSA_REQUIRE(iw, "iw");
  QSA_REQUIRE(sel, "sel"); QSA_REQUIRE(nsel, "nsel");
  if (scores) QSA_REQUIRE(scores, "scores");
  if (pooled_out) QSA_REQUIRE(pooled_out, "pooled_out");
  const Geom g = make_geom(cfg);
  const PrefillWs need = carve_prefill(g, nullptr, batch, total_tokens, max_seqlen);
  if (!workspace || workspace_bytes < need.bytes || ((uintptr_t)workspace & 255u))
    return fail(QSA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", need.bytes);
  const PrefillWs w = carve_prefill(g, workspace, batch, total_tokens, max_seqlen);
  return prefill_select_common(cfg, g, batch, total_tokens, max_seqlen, cu_seqlens, iq, ik, iw,
                               w, pooled_out ? pooled_out : w.pooled, sel, nsel, scores,
                               (cudaStream_t)stream);
}

size_t qsa_decode_workspace_size(const qsa_config* cfg, int batch, int n_q, int cap) {
  if (check_decode_dims(cfg, batch, n_q, cap) != QSA_OK) return 0;
  return carve_decode(cfg, make_geom(cfg), nullptr, batch, n_q, cap).bytes;
}

static qsa_status decode_select_common(const qsa_config* cfg, const Geom& g, int batch, int n_q,
                                       int cap, const int32_t* kv_len, const void* iq,
                                       const void* ik_cache, const float* iw,
                                       float* pooled_cache, const DecodeWs& w, int32_t* sel,
                                       int32_t* nsel, float* scores, int32_t* dev_err,
                                       cudaStream_t st, Pages pg = Pages()) {
  QSA_CUDA(cudaMemsetAsync(w.counters, 0, sizeof(int) * (size_t)batch * (2 + g.Hkv), st),
           "clear counters");
  QSA_CUDA(launch_decode_select(cfg->dtype, g, batch, n_q, cap, kv_len, iq, ik_cache, iw,
                                pooled_cache, scores, w.keys, w.counters, sel, nsel, dev_err, st,
                                pg, w.counters + (size_t)batch * (1 + g.Hkv)),
           "decode select");
  return QSA_OK;
}

static qsa_status decode_impl(const qsa_config* cfg, int batch, int n_q, int cap, const int32_t* kv_len,
                      const void* q, const void* k_cache, const void* v_cache, const void* iq,
                      const void* ik_cache, const float* iw, const void* gate,
                      float* pooled_cache, void* out, float* lse, int32_t* sel, int32_t* nsel,
                      int32_t* dev_err, void* workspace, size_t workspace_bytes, void* stream,
                      Pages pg, Fp8Kv f8 = Fp8Kv()) {
  qsa_status s = check_decode_dims(cfg, batch, n_q, cap);
  if (s != QSA_OK) return s;
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(kv_len, "kv_len");
  QSA_REQUIRE(q, "q"); QSA_REQUIRE(k_cache, "k_cache"); QSA_REQUIRE(v_cache, "v_cache");
  QSA_REQUIRE(iq, "iq"); QSA_REQUIRE(ik_cache, "ik_cache"); QSA_REQUIRE(iw, "iw");
  QSA_REQUIRE(gate, "gate"); QSA_REQUIRE(pooled_cache, "pooled_cache"); QSA_REQUIRE(out, "out");
  if (lse) QSA_REQUIRE(lse, "lse");
  if (sel) QSA_REQUIRE(sel, "sel");
  if (nsel) QSA_REQUIRE(nsel, "nsel");
  const Geom g = make_geom(cfg);
  const DecodeWs need = carve_decode(cfg, g, nullptr, batch, n_q, cap);
  if (!workspace || workspace_bytes < need.bytes || ((uintptr_t)workspace & 255u))
    return fail(QSA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", need.bytes);
  const DecodeWs w = carve_decode(cfg, g, workspace, batch, n_q, cap);
  cudaStream_t st = (cudaStream_t)stream;
  int* sel_p = sel ? sel : w.sel;
  int* nsel_p = nsel ? nsel : w.nsel;
  stage_mark(0, st);
  // (every pointer was checked for 16-byte alignment above, as the fused
  // selection's vector loads need)
  if (decode_uses_mma(cfg, g, n_q) && decode_fused_supported(g, n_q, cap, w.nsplit, f8.on)) {
    // one launch: each (sequence, KV head) cluster pools, scores and selects,
    // then gathers K/V and merges its partials
    stage_mark(1, st);
    DecodeSelIn si;
    si.iq = iq;
    si.ik_cache = ik_cache;
    si.iw = iw;
    si.pooled = pooled_cache;
    si.sel = sel_p;
    si.nsel = nsel_p;
    QSA_CUDA(launch_decode_fused(g, batch, n_q, cap, w.nsplit, w.per_split, kv_len, q, k_cache,
                                 v_cache, gate, si, out, lse, dev_err ? dev_err : w.err, st, pg,
                                 f8),
             "decode");
    stage_mark(2, st);
    return QSA_OK;
  }
  s = decode_select_common(cfg, g, batch, n_q, cap, kv_len, iq, ik_cache, iw, pooled_cache, w,
                           sel_p, nsel_p, nullptr, dev_err, st, pg);
  if (s != QSA_OK) return s;
  stage_mark(1, st);
  if (decode_uses_mma(cfg, g, n_q)) {
    QSA_CUDA(launch_attn_decode_mma(g, batch, n_q, cap, w.nsplit, w.per_split, kv_len, q,
                                    k_cache, v_cache, gate, sel_p, nsel_p, w.part_ml, w.part_o,
                                    w.counters + batch, out, lse, dev_err ? dev_err : w.err, st,
                                    pg, w.counters + (size_t)batch * (1 + g.Hkv), f8),
             "decode attention");
  } else {
    QSA_CUDA(launch_attn_decode_simt(cfg->dtype, g, batch, n_q, cap, w.nsplit, w.per_split,
                                     kv_len, q, k_cache, v_cache, gate, sel_p, nsel_p, w.part_ml,
                                     w.part_o, out, lse, st),
             "decode attention");
  }
  stage_mark(2, st);
  return QSA_OK;
}

qsa_status qsa_decode(const qsa_config* cfg, int batch, int n_q, int cap, const int32_t* kv_len,
                      const void* q, const void* k_cache, const void* v_cache, const void* iq,
                      const void* ik_cache, const float* iw, const void* gate,
                      float* pooled_cache, void* out, float* lse, int32_t* sel, int32_t* nsel,
                      int32_t* dev_err, void* workspace, size_t workspace_bytes, void* stream) {
  QSA_NVTX("qsa_decode");
  g_err[0] = 0;
  return decode_impl(cfg, batch, n_q, cap, kv_len, q, k_cache, v_cache, iq, ik_cache, iw, gate,
                     pooled_cache, out, lse, sel, nsel, dev_err, workspace, workspace_bytes,
                     stream, Pages());
}

qsa_status qsa_decode_fp8(const qsa_config* cfg, int batch, int n_q, int cap,
                          const int32_t* kv_len, const void* q, const void* k_cache,
                          const float* k_scale, const void* v_cache, const float* v_scale,
                          int rotated, const void* iq, const void* ik_cache, const float* iw,
                          const void* gate, float* pooled_cache, void* out, float* lse,
                          int32_t* sel, int32_t* nsel, int32_t* dev_err, void* workspace,
                          size_t workspace_bytes, void* stream) {
  QSA_NVTX("qsa_decode_fp8");
  g_err[0] = 0;
  qsa_status s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  const Geom g = make_geom(cfg);
  if (cfg->dtype != QSA_BF16 || !attn_decode_fp8_supported(g, n_q))
    return fail(QSA_ERR_UNSUPPORTED,
                "fp8 decode needs bf16 activations, head_dim 128, Hkv <= 8 and n_q * group <= 16");
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(k_scale, "k_scale");
  QSA_REQUIRE(v_scale, "v_scale");
  Fp8Kv f8;
  f8.on = true;
  f8.k_scale = k_scale;
  f8.v_scale = v_scale;
  f8.rotated = rotated ? 1 : 0;
  return decode_impl(cfg, batch, n_q, cap, kv_len, q, k_cache, v_cache, iq, ik_cache, iw, gate,
                     pooled_cache, out, lse, sel, nsel, dev_err, workspace, workspace_bytes,
                     stream, Pages(), f8);
}

qsa_status qsa_decode_attend(const qsa_config* cfg, int batch, int n_q, int cap,
                             const int32_t* kv_len, const void* q, const void* k_cache,
                             const void* v_cache, const void* gate, const int32_t* sel,
                             const int32_t* nsel, void* out, float* lse, int32_t* dev_err,
                             void* workspace, size_t workspace_bytes, void* stream) {
  QSA_NVTX("qsa_decode_attend");
  g_err[0] = 0;
  qsa_status s = check_decode_dims(cfg, batch, n_q, cap);
  if (s != QSA_OK) return s;
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(kv_len, "kv_len");
  QSA_REQUIRE(q, "q"); QSA_REQUIRE(k_cache, "k_cache"); QSA_REQUIRE(v_cache, "v_cache");
  QSA_REQUIRE(gate, "gate"); QSA_REQUIRE(sel, "sel"); QSA_REQUIRE(nsel, "nsel");
  QSA_REQUIRE(out, "out");
  if (lse) QSA_REQUIRE(lse, "lse");
  const Geom g = make_geom(cfg);
  const DecodeWs need = carve_decode(cfg, g, nullptr, batch, n_q, cap);
  if (!workspace || workspace_bytes < need.bytes || ((uintptr_t)workspace & 255u))
    return fail(QSA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", need.bytes);
  const DecodeWs w = carve_decode(cfg, g, workspace, batch, n_q, cap);
  cudaStream_t st = (cudaStream_t)stream;
  QSA_CUDA(cudaMemsetAsync(w.counters, 0, sizeof(int) * (size_t)batch * (2 + g.Hkv), st),
           "clear counters");
  stage_mark(0, st);
  stage_mark(1, st);
  if (decode_uses_mma(cfg, g, n_q)) {
    QSA_CUDA(launch_attn_decode_mma(g, batch, n_q, cap, w.nsplit, w.per_split, kv_len, q,
                                    k_cache, v_cache, gate, sel, nsel, w.part_ml, w.part_o,
                                    w.counters + batch, out, lse, dev_err ? dev_err : w.err, st),
             "decode attention");
  } else {
    QSA_CUDA(launch_attn_decode_simt(cfg->dtype, g, batch, n_q, cap, w.nsplit, w.per_split,
                                     kv_len, q, k_cache, v_cache, gate, sel, nsel, w.part_ml,
                                     w.part_o, out, lse, st),
             "decode attention");
  }
  stage_mark(2, st);
  return QSA_OK;
}

// ------------------------------------------------------- context-parallel decode
static qsa_status check_shard(const qsa_config* cfg, int batch, int n_q, int cap, int block_lo) {
  qsa_status s = check_decode_dims(cfg, batch, n_q, cap);
  if (s != QSA_OK) return s;
  if (block_lo < 0) return fail(QSA_ERR_INVALID_ARG, "block_lo must be >= 0");
  if ((long long)block_lo * cfg->block_size + cap > 2147483647LL)
    return fail(QSA_ERR_UNSUPPORTED, "shard rows past 2^31");
  return QSA_OK;
}

qsa_status qsa_cp_pool_build(const qsa_config* cfg, int batch, int cap, int block_lo,
                             const int32_t* kv_len, const void* ik_shard, float* pooled_shard,
                             int32_t* dev_err, void* stream) {
  QSA_NVTX("qsa_cp_pool_build");
  g_err[0] = 0;
  qsa_status s = check_shard(cfg, batch, 1, cap, block_lo);
  if (s != QSA_OK) return s;
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(kv_len, "kv_len");
  QSA_REQUIRE(ik_shard, "ik_shard");
  QSA_REQUIRE(pooled_shard, "pooled_shard");
  QSA_CUDA(launch_pool_cache(cfg->dtype, ik_shard, kv_len, batch, cap, 0, 0, make_geom(cfg),
                             pooled_shard, dev_err, (cudaStream_t)stream, Pages(), block_lo),
           "shard pool build");
  return QSA_OK;
}

qsa_status qsa_cp_select(const qsa_config* cfg, int batch, int n_q, int cap, int block_lo,
                         const int32_t* kv_len, const void* iq, const void* ik_shard,
                         const float* iw, float* pooled_shard, float* cand_score,
                         int32_t* cand_id, int32_t* dev_err, void* workspace,
                         size_t workspace_bytes, void* stream) {
  QSA_NVTX("qsa_cp_select");
  g_err[0] = 0;
  qsa_status s = check_shard(cfg, batch, n_q, cap, block_lo);
  if (s != QSA_OK) return s;
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(kv_len, "kv_len");
  QSA_REQUIRE(iq, "iq"); QSA_REQUIRE(ik_shard, "ik_shard"); QSA_REQUIRE(iw, "iw");
  QSA_REQUIRE(pooled_shard, "pooled_shard");
  QSA_REQUIRE(cand_score, "cand_score"); QSA_REQUIRE(cand_id, "cand_id");
  const Geom g = make_geom(cfg);
  const DecodeWs need = carve_decode(cfg, g, nullptr, batch, n_q, cap);
  if (!workspace || workspace_bytes < need.bytes || ((uintptr_t)workspace & 255u))
    return fail(QSA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", need.bytes);
  const DecodeWs w = carve_decode(cfg, g, workspace, batch, n_q, cap);
  cudaStream_t st = (cudaStream_t)stream;
  CpShard cp;
  cp.on = true;
  cp.row_off = block_lo * cfg->block_size;
  cp.block_lo = block_lo;
  cp.cand_score = cand_score;
  cp.cand_id = cand_id;
  QSA_CUDA(cudaMemsetAsync(w.counters, 0, sizeof(int) * (size_t)batch * (2 + g.Hkv), st),
           "clear counters");
  QSA_CUDA(launch_decode_select(cfg->dtype, g, batch, n_q, cap, kv_len, iq, ik_shard, iw,
                                pooled_shard, nullptr, w.keys, w.counters, w.sel, w.nsel,
                                dev_err ? dev_err : w.err, st, Pages(), nullptr, cp),
           "shard select");
  return QSA_OK;
}

qsa_status qsa_cp_global_topk(const qsa_config* cfg, int batch, int n_q, int world,
                              const int32_t* kv_len, const float* cand_score,
                              const int32_t* cand_id, int32_t* sel, int32_t* nsel,
                              void* stream) {
  QSA_NVTX("qsa_cp_global_topk");
  g_err[0] = 0;
  qsa_status s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if (batch < 0 || n_q <= 0 || world <= 0)
    return fail(QSA_ERR_INVALID_ARG, "batch >= 0, n_q > 0 and world > 0 are required");
  if (n_q > kMaxDecodeQ) return fail(QSA_ERR_UNSUPPORTED, "n_q > %d", kMaxDecodeQ);
  if ((long long)world * (cfg->budget / cfg->block_size) > 4096)
    return fail(QSA_ERR_UNSUPPORTED, "world * budget / block_size > 4096");
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(kv_len, "kv_len");
  QSA_REQUIRE(cand_score, "cand_score"); QSA_REQUIRE(cand_id, "cand_id");
  QSA_REQUIRE(sel, "sel"); QSA_REQUIRE(nsel, "nsel");
  const Geom g = make_geom(cfg);
  QSA_CUDA(launch_cp_global_topk(g, batch, n_q, world, kv_len, cand_score, cand_id, sel, nsel,
                                 (cudaStream_t)stream),
           "global top-k");
  return QSA_OK;
}

qsa_status qsa_cp_attend(const qsa_config* cfg, int batch, int n_q, int cap, int block_lo,
                         const int32_t* kv_len, const void* q, const void* k_shard,
                         const void* v_shard, const void* gate, const int32_t* sel,
                         const int32_t* nsel, float* part_out, float* part_lse,
                         int32_t* dev_err, void* workspace, size_t workspace_bytes,
                         void* stream) {
  QSA_NVTX("qsa_cp_attend");
  g_err[0] = 0;
  qsa_status s = check_shard(cfg, batch, n_q, cap, block_lo);
  if (s != QSA_OK) return s;
  const Geom g = make_geom(cfg);
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(kv_len, "kv_len");
  QSA_REQUIRE(q, "q"); QSA_REQUIRE(k_shard, "k_shard"); QSA_REQUIRE(v_shard, "v_shard");
  QSA_REQUIRE(gate, "gate"); QSA_REQUIRE(sel, "sel"); QSA_REQUIRE(nsel, "nsel");
  QSA_REQUIRE(part_out, "part_out"); QSA_REQUIRE(part_lse, "part_lse");
  const DecodeWs need = carve_decode(cfg, g, nullptr, batch, n_q, cap);
  if (!workspace || workspace_bytes < need.bytes || ((uintptr_t)workspace & 255u))
    return fail(QSA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", need.bytes);
  const DecodeWs w = carve_decode(cfg, g, workspace, batch, n_q, cap);
  cudaStream_t st = (cudaStream_t)stream;
  CpShard cp;
  cp.on = true;
  cp.row_off = block_lo * cfg->block_size;
  cp.block_lo = block_lo;
  cp.out_f32 = part_out;
  QSA_CUDA(cudaMemsetAsync(w.counters, 0, sizeof(int) * (size_t)batch * (2 + g.Hkv), st),
           "clear counters");
  if (decode_uses_mma(cfg, g, n_q)) {
    QSA_CUDA(launch_attn_decode_mma(g, batch, n_q, cap, w.nsplit, w.per_split, kv_len, q,
                                    k_shard, v_shard, gate, sel, nsel, w.part_ml, w.part_o,
                                    w.counters + batch, nullptr, part_lse,
                                    dev_err ? dev_err : w.err, st, Pages(), nullptr, Fp8Kv(), cp),
             "shard attention");
  } else {
    QSA_CUDA(launch_attn_decode_simt(cfg->dtype, g, batch, n_q, cap, w.nsplit, w.per_split,
                                     kv_len, q, k_shard, v_shard, gate, sel, nsel, w.part_ml,
                                     w.part_o, nullptr, part_lse, st, cp),
             "shard attention");
  }
  return QSA_OK;
}

qsa_status qsa_cp_merge(const qsa_config* cfg, int batch, int n_q, int world,
                        const float* part_out, const float* part_lse, void* out, float* lse,
                        void* stream) {
  QSA_NVTX("qsa_cp_merge");
  g_err[0] = 0;
  qsa_status s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if (batch < 0 || n_q <= 0 || world <= 0)
    return fail(QSA_ERR_INVALID_ARG, "batch >= 0, n_q > 0 and world > 0 are required");
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(part_out, "part_out"); QSA_REQUIRE(part_lse, "part_lse"); QSA_REQUIRE(out, "out");
  if (lse) QSA_REQUIRE(lse, "lse");
  if ((long long)batch * n_q * cfg->num_q_heads > 2147483647LL)
    return fail(QSA_ERR_UNSUPPORTED, "too many rows");
  QSA_CUDA(launch_cp_merge(cfg->dtype, batch * n_q * cfg->num_q_heads, cfg->head_dim, world,
                           part_out, part_lse, out, lse, (cudaStream_t)stream),
           "merge");
  return QSA_OK;
}

static qsa_status check_pages(const qsa_config* cfg, int max_blocks, const int32_t* block_table,
                              int num_pages) {
  if (max_blocks <= 0 || num_pages <= 0)
    return fail(QSA_ERR_INVALID_ARG, "max_blocks and num_pages must be > 0");
  if ((long long)max_blocks * cfg->block_size > INT32_MAX ||
      (long long)num_pages * cfg->block_size > INT32_MAX)
    return fail(QSA_ERR_UNSUPPORTED, "more than 2^31 cache rows");
  QSA_REQUIRE(block_table, "block_table");
  return QSA_OK;
}

qsa_status qsa_append(const qsa_config* cfg, int batch, int n_q, int cap, const int32_t* kv_len,
                      const void* k_new, const void* v_new, const void* ik_new, void* k_cache,
                      void* v_cache, void* ik_cache, float* pooled_cache,
                      const int32_t* block_table, int num_pages, int32_t* dev_err, void* stream) {
  QSA_NVTX("qsa_append");
  g_err[0] = 0;
  qsa_status s = check_decode_dims(cfg, batch, n_q, cap);
  if (s != QSA_OK) return s;
  if (block_table && (s = check_pages(cfg, cap / cfg->block_size, block_table, num_pages)) != QSA_OK)
    return s;
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(kv_len, "kv_len");
  QSA_REQUIRE(ik_new, "ik_new"); QSA_REQUIRE(ik_cache, "ik_cache");
  QSA_REQUIRE(pooled_cache, "pooled_cache");
  if ((k_new == nullptr) != (v_new == nullptr) || (k_new == nullptr) != (k_cache == nullptr) ||
      (k_new == nullptr) != (v_cache == nullptr))
    return fail(QSA_ERR_INVALID_ARG, "k_new, v_new, k_cache and v_cache are given together or not at all");
  if (k_new) {
    QSA_REQUIRE(k_new, "k_new"); QSA_REQUIRE(v_new, "v_new");
    QSA_REQUIRE(k_cache, "k_cache"); QSA_REQUIRE(v_cache, "v_cache");
  }
  QSA_CUDA(launch_append(cfg->dtype, make_geom(cfg), batch, n_q, cap, kv_len, k_new, v_new, ik_new,
                         k_cache, v_cache, ik_cache, pooled_cache, dev_err,
                         block_table ? Pages{block_table, num_pages} : Pages(),
                         (cudaStream_t)stream),
           "append");
  return QSA_OK;
}

qsa_status qsa_decode_paged(const qsa_config* cfg, int batch, int n_q, int max_blocks,
                            const int32_t* block_table, int num_pages, const int32_t* kv_len,
                            const void* q, const void* k_pages, const void* v_pages,
                            const void* iq, const void* ik_pages, const float* iw,
                            const void* gate, float* pooled_cache, void* out, float* lse,
                            int32_t* sel, int32_t* nsel, int32_t* dev_err, void* workspace,
                            size_t workspace_bytes, void* stream) {
  QSA_NVTX("qsa_decode_paged");
  g_err[0] = 0;
  qsa_status s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if ((s = check_pages(cfg, max_blocks, block_table, num_pages)) != QSA_OK) return s;
  const Geom g = make_geom(cfg);
  if (!decode_uses_mma(cfg, g, n_q))
    return fail(QSA_ERR_UNSUPPORTED,
                "paged decode needs bf16, head_dim 128 and n_q * group size <= 32");
  return decode_impl(cfg, batch, n_q, max_blocks * cfg->block_size, kv_len, q, k_pages, v_pages,
                     iq, ik_pages, iw, gate, pooled_cache, out, lse, sel, nsel, dev_err,
                     workspace, workspace_bytes, stream, Pages{block_table, num_pages});
}

qsa_status qsa_select_decode(const qsa_config* cfg, int batch, int n_q, int cap,
                             const int32_t* kv_len, const void* iq, const void* ik_cache,
                             const float* iw, float* pooled_cache, int32_t* sel, int32_t* nsel,
                             float* scores, int32_t* dev_err, void* workspace,
                             size_t workspace_bytes, void* stream) {
  QSA_NVTX("qsa_select_decode");
  g_err[0] = 0;
  qsa_status s = check_decode_dims(cfg, batch, n_q, cap);
  if (s != QSA_OK) return s;
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(kv_len, "kv_len");
  QSA_REQUIRE(iq, "iq"); QSA_REQUIRE(ik_cache, "ik_cache"); QSA_REQUIRE(iw, "iw");
  QSA_REQUIRE(pooled_cache, "pooled_cache");
  QSA_REQUIRE(sel, "sel"); QSA_REQUIRE(nsel, "nsel");
  if (scores) QSA_REQUIRE(scores, "scores");
  const Geom g = make_geom(cfg);
  const DecodeWs need = carve_decode(cfg, g, nullptr, batch, n_q, cap);
  if (!workspace || workspace_bytes < need.bytes || ((uintptr_t)workspace & 255u))
    return fail(QSA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", need.bytes);
  const DecodeWs w = carve_decode(cfg, g, workspace, batch, n_q, cap);
  return decode_select_common(cfg, g, batch, n_q, cap, kv_len, iq, ik_cache, iw, pooled_cache,
                              w, sel, nsel, scores, dev_err, (cudaStream_t)stream);
}

qsa_status qsa_pool_build(const qsa_config* cfg, int batch, int cap, const int32_t* kv_len,
                          const void* ik_cache, float* pooled_cache, int32_t* dev_err,
                          void* stream) {
  QSA_NVTX("qsa_pool_build");
  g_err[0] = 0;
  qsa_status s = check_decode_dims(cfg, batch, 1, cap);
  if (s != QSA_OK) return s;
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(kv_len, "kv_len");
  QSA_REQUIRE(ik_cache, "ik_cache");
  QSA_REQUIRE(pooled_cache, "pooled_cache");
  QSA_CUDA(launch_pool_cache(cfg->dtype, ik_cache, kv_len, batch, cap, 0, 0, make_geom(cfg),
                             pooled_cache, dev_err, (cudaStream_t)stream),
           "pool build");
  return QSA_OK;
}

qsa_status qsa_pool_build_paged(const qsa_config* cfg, int batch, int max_blocks,
                                const int32_t* block_table, int num_pages,
                                const int32_t* kv_len, const void* ik_pages,
                                float* pooled_cache, int32_t* dev_err, void* stream) {
  QSA_NVTX("qsa_pool_build_paged");
  g_err[0] = 0;
  qsa_status s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if ((s = check_pages(cfg, max_blocks, block_table, num_pages)) != QSA_OK) return s;
  const int cap = max_blocks * cfg->block_size;
  if ((s = check_decode_dims(cfg, batch, 1, cap)) != QSA_OK) return s;
  if (batch == 0) return QSA_OK;
  QSA_REQUIRE(kv_len, "kv_len");
  QSA_REQUIRE(ik_pages, "ik_pages");
  QSA_REQUIRE(pooled_cache, "pooled_cache");
  QSA_CUDA(launch_pool_cache(cfg->dtype, ik_pages, kv_len, batch, cap, 0, 0, make_geom(cfg),
                             pooled_cache, dev_err, (cudaStream_t)stream,
                             Pages{block_table, num_pages}),
           "pool build");
  return QSA_OK;
}

}  // extern "C"
