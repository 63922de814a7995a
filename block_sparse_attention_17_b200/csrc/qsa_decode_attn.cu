// QSA decode step (sm_100a): selection, gather and attention in one kernel.
//
// One decode step reads, per (sequence, KV head), only the K/V rows of the
// union of the step's n_q queries' selections (selected complete blocks plus
// tail blocks): the gather consumer of the selection, never a mask over the
// whole cache (ramgpt "Porting Qwen4 to llama.cpp", section "CUDA Optimization
// Should Follow State Correctness"). The nsplit CTAs of one (sequence, KV head)
// form a thread-block cluster:
//  1. (kSelDI > 0) the cluster selects: each CTA pools the block this step
//     completes if it owns it, scores its range of candidate blocks and keeps
//     each query's top k of the range; after a cluster barrier every CTA
//     gathers these candidates from all CTAs through distributed shared memory
//     and takes the top k of them (select_in_cluster); with kSelDI == 0 the
//     selections come from the selection kernel, which releases a per-sequence
//     flag the CTAs wait on;
//  2. the union is cut into 64-key chunks; each CTA takes a contiguous range,
//     and a producer warp streams each chunk's K and V tiles with TMA through
//     a 3-stage ring (two CTAs per SM keep about 190 KB in flight per SM);
//  3. the per-chunk arithmetic is tiny (at most 32 query rows = n_q x group
//     heads, in one or two tiles of 16), so the four consumer warps use
//     warp-level MMAs (m16n8k16, fp32 accumulation): with one tile warp w
//     takes keys [16w, 16w + 16) of each chunk, with two tiles warps 2t, 2t + 1
//     take tile t's rows over keys [0, 32) and [32, 64); each warp keeps its
//     own online-softmax state (log2 domain), merged at the end into one
//     (m, l, O) partial per row;
//  4. the cluster merges the partials by log-sum-exp through distributed
//     shared memory (each CTA takes some rows) and applies the output's sigmoid
//     gate; where such a cluster cannot be resident (two-launch path only), the
//     partials go through global memory and the last CTA merges them.
// kFp8 reads e4m3 K/V codes with per-row scales instead of bf16 rows.
#include <map>
#include <mutex>
#include <tuple>

#include "qsa_common.cuh"
#include "qsa_kernels.h"
#include "qsa_pool.cuh"
#include "qsa_sm100.cuh"

namespace qsa {

using namespace sm100;

namespace {

constexpr int kD = 128;
constexpr int kChunk = 64;                      // keys per ring stage
constexpr int kStages = 3;
constexpr int kBoxBytes = kChunk * 128;         // 64 keys x 64 dims bf16 (one TMA box)
constexpr int kTileBytes = 2 * kBoxBytes;       // 64 keys x 128 dims
constexpr int kStageBytes = 2 * kTileBytes;     // K + V
constexpr int kConsumers = 4;
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kQStride = kD * 2 + 16;           // padded bf16 row of Q in shared memory
constexpr int kMaxUnion = 4 * (kMaxTopK + 1);
constexpr int kMaxClusterSplits = 16;           // CTAs of one cluster-merged (sequence, KV head)
constexpr int kSelRows = 160;                   // in-kernel selection: blocks per scoring pass

// fp8 caches: a stage holds the K and V rows as e4m3 bytes (one 128-byte box
// each) and the 64 rows' scales for every KV head (K, then V); each consumer
// warp widens its 16 keys into its own fp16 K and V tiles before its MMAs.
constexpr int kMaxHkvFp8 = 8;
constexpr int kF8BoxBytes = kChunk * kD;                      // 64 keys x 128 e4m3
constexpr int kF8ScaleBytes = kChunk * kMaxHkvFp8 * 4;       // 64 rows x Hkv fp32
constexpr int kF8StageBytes = 2 * kF8BoxBytes + 2 * kF8ScaleBytes;
constexpr int kWarpTileBytes = 16 * 128 * 2;                  // 16 keys x 128 fp16: two 2 KB boxes
constexpr int kF8ConvBytes = kConsumers * 2 * kWarpTileBytes; // [warp][K, V]
static_assert(kStages * kF8StageBytes + kF8ConvBytes >= kConsumers * 16 * kD * 4 + 512,
              "the fp8 layout must hold the partial-merge scratch");
static_assert(kStages * kF8StageBytes + kF8ConvBytes <= kStages * kStageBytes,
              "the fp8 layout fits in the bf16 ring's space");

constexpr int kOffStages = 0;
// Shared memory of a kernel that holds kRT tiles of 16 query rows (rows
// r = i * G + gi: new query i, head gi of the KV head). Dynamic shared memory:
// kOffBits + 4 * n_q * words + 1024 (alignment slack).
template <int kRT>
struct DecLayout {
  static constexpr int kRows = 16 * kRT;
  static constexpr int kOffQ = kOffStages + kStages * kStageBytes;
  static constexpr int kOffBar = kOffQ + kRows * kQStride;
  static constexpr int kOffMisc = kOffBar + 8 * 2 * kStages;
  static constexpr int kOffUnion = kOffMisc + 64;
  static constexpr int kOffGate = kOffUnion + 8 * kMaxUnion;   // cluster merge: [rows][128] gate
  static constexpr int kOffBits = kOffGate + kRows * kD * 2;   // [n_q][cap / B / 32] words
};

struct DecParams {
  Geom g;
  int n_q, cap, nsplit, per_split;   // per_split: chunks per CTA
  const int* kv_len;
  const __nv_bfloat16* q;
  const __nv_bfloat16* gate;
  const int* sel;
  const int* nsel;
  float* part_ml;
  float* part_o;
  int* counter;                      // [batch * Hkv], zero before the launch
  __nv_bfloat16* out;
  float* lse;
  int* err;
  const int* table;                  // paged caches: [batch, cap / B] page ids, else null
  const int* ready;                  // [batch] selection-written flags, else null
  const float* k_scale;              // fp8 caches: [batch, cap, Hkv] fp32 row scales
  const float* v_scale;
  int rotated;                       // fp8 caches hold H k and H v (Walsh-Hadamard, order D)
  int cluster;                       // the nsplit CTAs of a (sequence, KV head) form one
                                     // cluster and merge through distributed shared memory
  // selection inside the kernel (the cluster scores, pools and selects itself)
  const __nv_bfloat16* iq;           // [batch, n_q, Hi, di]
  const __nv_bfloat16* ik_cache;     // [batch * cap, di] (or pages)
  const float* iw;                   // [batch, n_q, Hi]
  float* pooled;                     // [batch, cap / B, di] pooled-key cache
  int num_pages;                     // paged caches: pages in the pool
  int* sel_w;                        // [batch, n_q, k + 1] selections out
  int* nsel_w;                       // [batch, n_q]
  int fo_cand, fo_gath, fo_kbar, fo_iq, fo_iw, fo_new, fo_hist;   // byte offsets in the ring's space
  // context-parallel shard (attention over given selections only): kv_len are
  // full lengths, the caches hold rows [row_off, row_off + cap), sel holds
  // global block ids; outputs are fp32 gated partials in out_f32
  int cp, row_off, block_lo;
  float* out_f32;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D = A (16x16 bf16, row) * B (16x8 bf16, col) + D, fp32
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void mma_f16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2h(float a, float b) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}
// two e4m3 codes (low byte first) -> fp16x2
__device__ __forceinline__ uint32_t e4m3x2(uint32_t two_bytes) {
  uint32_t h;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(h) : "r"(two_bytes));
  return h;
}
// two e4m3 codes (low byte first) -> fp16x2 times an fp16x2 scale
__device__ __forceinline__ uint32_t e4m3x2_scaled(uint32_t two_bytes, uint32_t scale2) {
  uint32_t h, r;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(h) : "r"(two_bytes));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(scale2));
  return r;
}

// Byte offset of (row, dim) in a warp's 16-row fp16 tile (two 128-byte-swizzled
// boxes of 64 dims, as tile_off); dim must be a multiple of 8.
__device__ __forceinline__ uint32_t tile16_off(int row, int dim) {
  const int box = dim >> 6;
  const int chunk = (dim & 63) >> 3;
  return box * 2048 + row * 128 + ((chunk ^ (row & 7)) << 4);
}

// In-place orthonormal Walsh-Hadamard transform of nrows rows of 128 floats
// (row stride 128) by nthr threads that synchronise with `sync` between the
// 7 butterfly stages; the result is scaled by 128^-1/2.
template <typename Sync>
__device__ __forceinline__ void fwht128_rows(float* rows, int nrows, int tid, int nthr, Sync sync) {
  for (int h = 1; h < kD; h <<= 1) {
    for (int e = tid; e < nrows * (kD / 2); e += nthr) {
      const int r = e / (kD / 2), p = e % (kD / 2);
      const int i = (p / h) * 2 * h + (p % h);
      float* row = rows + r * kD;
      const float a = row[i], c = row[i + h];
      row[i] = a + c;
      row[i + h] = a - c;
    }
    sync();
  }
  const float norm = 0.08838834764831845f;   // 128^-1/2
  for (int e = tid; e < nrows * kD; e += nthr) rows[e] *= norm;
  sync();
}

// Byte offset of (row, dim) in a 64-row K/V tile stored as two 128-byte-swizzled
// TMA boxes (dims 0..63, then 64..127); dim must be a multiple of 8.
__device__ __forceinline__ uint32_t tile_off(int row, int dim) {
  const int box = dim >> 6;
  const int chunk = (dim & 63) >> 3;
  return box * kBoxBytes + row * 128 + ((chunk ^ (row & 7)) << 4);
}

// ------------------------------------------------- selection in the cluster
__device__ __forceinline__ void cluster_arrive_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_all() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint4 ld_cluster_u32x4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ unsigned lane_mask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// One warp, keys[0 .. n) in shared memory: the threshold of the kk largest
// keys, a lower index winning among equal keys. Afterwards the chosen keys are
// those > tau plus the first `need` keys == tau in index order. tau is found
// by deciding its bits from the highest bit where the largest and the
// smallest key differ, each step counting the keys at or above the candidate
// over the warp; it stops early once exactly kk keys are at or above it. Up to
// 32 * kR keys are held in registers for the search (longer lists are re-read
// from shared memory at every step).
template <int kR>
__device__ __forceinline__ void warp_threshold(const uint32_t* keys, int n, int kk, uint32_t& tau,
                                               int& need) {
  const int lane = threadIdx.x & 31;
  if (kk <= 0) {
    tau = 0xffffffffu;   // above every score key: nothing is taken
    need = 0;
    return;
  }
  if (n <= kk) {
    tau = 0u;            // score keys are never 0: every key is taken
    need = 0;
    return;
  }
  const bool regs = n <= 32 * kR;   // uniform
  uint32_t kr[kR];
  uint32_t hi = 0u, lo = 0xffffffffu;
#pragma unroll
  for (int u = 0; u < kR; ++u) {
    const int j = lane + 32 * u;
    kr[u] = (regs && j < n) ? keys[j] : 0u;
    if (regs && j < n) {
      hi = max(hi, kr[u]);
      lo = min(lo, kr[u]);
    }
  }
  if (!regs)
    for (int j = lane; j < n; j += 32) {
      const uint32_t x = keys[j];
      hi = max(hi, x);
      lo = min(lo, x);
    }
  hi = __reduce_max_sync(kFull, hi);
  lo = __reduce_min_sync(kFull, lo);
  tau = hi;
  if (hi != lo) {
    const int top = 31 - __clz(hi ^ lo);
    tau = top == 31 ? 0u : (hi & ~((2u << top) - 1u));
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      int c = 0;
      if (regs) {
#pragma unroll
        for (int u = 0; u < kR; ++u) c += kr[u] >= cand ? 1 : 0;   // padding keys are 0
      } else {
        for (int j = lane; j < n; j += 32) c += keys[j] >= cand ? 1 : 0;
      }
      c = __reduce_add_sync(kFull, c);
      if (c >= kk) tau = cand;
      if (c == kk) break;
    }
  }
  int gt = 0;
  if (regs) {
#pragma unroll
    for (int u = 0; u < kR; ++u) gt += kr[u] > tau ? 1 : 0;
  } else {
    for (int j = lane; j < n; j += 32) gt += keys[j] > tau ? 1 : 0;
  }
  need = kk - __reduce_add_sync(kFull, gt);
}

// One warp: the kk largest of keys[0 .. n) (warp_threshold's rule), written in
// index order to out_key / out_pos (pos0 + index); slots kk .. kpad - 1 get a
// sentinel (key 0, below every score key).
__device__ __forceinline__ void warp_topk_compact(const uint32_t* keys, int n, int kk, int pos0,
                                                  uint32_t* out_key, int* out_pos, int kpad) {
  const int lane = threadIdx.x & 31;
  uint32_t tau;
  int need;
  warp_threshold<8>(keys, n, kk, tau, need);
  int base = 0;
  for (int j0 = 0; j0 < n && base < kk; j0 += 32) {   // uniform
    const int j = j0 + lane;
    const uint32_t x = j < n ? keys[j] : 0u;
    const bool eq = j < n && x == tau;
    const unsigned eb = __ballot_sync(kFull, eq);
    const bool t = (j < n && x > tau) || (eq && __popc(eb & lane_mask_lt()) < need);
    need -= __popc(eb);
    const unsigned tb = __ballot_sync(kFull, t);
    if (t) {
      const int sl = base + __popc(tb & lane_mask_lt());
      out_key[sl] = x;
      out_pos[sl] = pos0 + j;
    }
    base += __popc(tb);
  }
  for (int sl = kk + lane; sl < kpad; sl += 32) {
    out_key[sl] = 0u;
    out_pos[sl] = 0x7fffffff;
  }
}

// One warp: the kk largest of keys[0 .. n) (warp_threshold's rule); sets bit
// pos[j] % 32 of word pos[j] / 32 of bits for every chosen j.
__device__ __forceinline__ void warp_topk_bits(const uint32_t* keys, const int* pos, int n, int kk,
                                               uint32_t* bits) {
  const int lane = threadIdx.x & 31;
  uint32_t tau;
  int need;
  warp_threshold<16>(keys, n, kk, tau, need);
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t x = j < n ? keys[j] : 0u;
    const bool eq = j < n && x == tau;
    const unsigned eb = __ballot_sync(kFull, eq);
    const bool t = (j < n && x > tau) || (eq && __popc(eb & lane_mask_lt()) < need);
    need -= __popc(eb);
    if (t) atomicOr(&bits[pos[j] >> 5], 1u << (pos[j] & 31));
  }
}

// Sorted top-32 lists held one value per lane. A value packs a score key and
// a block position as (key << 32) | (0xffffffff - position): a larger value
// comes first in the selection's order (a larger key, or the same key at a
// lower position); 0 is padding, below every real value.
__device__ __forceinline__ unsigned long long cand_value(uint32_t key, int pos) {
  return ((unsigned long long)key << 32) | (0xffffffffu - (uint32_t)pos);
}
__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int m) {
  return __shfl_xor_sync(kFull, v, m);
}
// One warp: the 32 values (one per lane) sorted in descending order, lane =
// rank (a bitonic sorting network over the lanes).
__device__ __forceinline__ unsigned long long warp_sort32_desc(unsigned long long v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int sz = 2; sz <= 32; sz <<= 1)
#pragma unroll
    for (int j = sz >> 1; j > 0; j >>= 1) {
      const unsigned long long o = shfl_xor_u64(v, j);
      v = (((lane & j) == 0) == ((lane & sz) == 0 || sz == 32)) ? (v > o ? v : o) : (v < o ? v : o);
    }
  return v;
}
// One warp: the largest 32 of two descending lists (lane = rank), descending:
// max(a[i], b[31 - i]) is bitonic and holds them; one bitonic merge sorts it.
__device__ __forceinline__ unsigned long long warp_merge32_desc(unsigned long long a,
                                                                unsigned long long b) {
  const int lane = threadIdx.x & 31;
  const unsigned long long br = __shfl_sync(kFull, b, 31 - lane);
  unsigned long long v = a > br ? a : br;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const unsigned long long o = shfl_xor_u64(v, j);
    v = ((lane & j) == 0) ? (v > o ? v : o) : (v < o ? v : o);
  }
  return v;
}

// Chunk of candidate blocks one CTA of the cluster scores: a multiple of 4.
__host__ __device__ __forceinline__ int select_range(int nc_last, int nsplit) {
  const int per = ((nc_last > 1 ? nc_last : 1) + nsplit - 1) / nsplit;
  return (per + 3) & ~3;
}

// The selection step of one decode step, done by the cluster of one (sequence,
// KV head) before it gathers K and V (the indexer of the llama.cpp PR #27739
// page, QSA composition commit; the pooled keys of the instagit MTPLX page).
// CTA `split` owns candidate blocks [split * per, (split + 1) * per): it pools
// the blocks of its range that this step's tokens complete (writing them to the
// pooled-key cache once, from the KV head 0 cluster), scores its blocks for
// every query, s = c * sum_h w_h relu(q_h . kbar) (one thread per (query,
// block, head), the heads summed by shuffles; the same arithmetic as the
// selection kernel), and keeps the score keys in its shared memory; warp i
// takes query i's top k of the range as candidates. After a cluster barrier
// every CTA gathers all CTAs' candidates, selects each query's top k of them
// into the query's bitmap (warp_topk_bits) and adds the tail block; CTA
// (0, b, 0) also writes the selection lists. Ends with this CTA's arrival on
// the cluster barrier that the caller waits on before reusing the space.
//
// select_prefetch starts moving what select_in_cluster reads into L2 (bulk
// prefetches by one thread): the CTA's range of pooled rows, the indexer rows
// of the blocks this step completes, and the queries' indexer q.
template <int kDI>
__device__ __forceinline__ void select_prefetch(const DecParams& P, int kv, int split, int b) {
  const Geom& g = P.g;
  const int nblk_cap = P.cap / g.B, nc_last = kv / g.B;
  const int per = select_range(nc_last, P.nsplit);
  const int j0 = split * per, j1 = min(nc_last, j0 + per);
  if (j1 > j0)
    bulk_prefetch_l2(P.pooled + ((size_t)b * nblk_cap + j0) * kDI, (uint32_t)(j1 - j0) * kDI * 4u);
  const int jn_lo = max((kv - P.n_q) / g.B, j0), jn_hi = min(nc_last, j1);
  for (int j = jn_lo; j < jn_hi; ++j) {
    size_t r0 = (size_t)b * P.cap + (size_t)j * g.B;
    if (P.table) {
      const int page = P.table[(size_t)b * nblk_cap + j];
      if (page < 0 || page >= P.num_pages) continue;
      r0 = (size_t)page * g.B;
    }
    bulk_prefetch_l2(P.ik_cache + r0 * kDI, (uint32_t)g.B * kDI * 2u);
  }
  if (split == 0 || j1 > j0)
    bulk_prefetch_l2(P.iq + (size_t)b * P.n_q * g.Hi * kDI, (uint32_t)(P.n_q * g.Hi * kDI * 2));
}

template <int kDI>
__device__ __forceinline__ void select_in_cluster(const DecParams& P, uint8_t* smem, int kv, int split, int b,
                                  int hk, uint32_t* qbits, int words) {
  constexpr int kStride = kDI + 4;                 // 16-byte rows; 8 rows of a warp hit distinct banks
  constexpr int kQStrideI = kDI + 4;
  constexpr int kRows = kSelRows;                 // candidate blocks per scoring pass
  const Geom& g = P.g;
  const int n_q = P.n_q, Hi = g.Hi, k = g.k, kp1 = k + 1;
  const int tid = threadIdx.x, nthr = blockDim.x, warp = tid >> 5, lane = tid & 31;
  const int nblk_cap = P.cap / g.B;
  const int nc_last = kv / g.B;
  const int per = select_range(nc_last, P.nsplit);
  const int j0 = split * per, j1 = min(nc_last, j0 + per);
  uint8_t* ring = smem + kOffStages;
  uint32_t* keys_mine = reinterpret_cast<uint32_t*>(ring + 32);             // [n_q][per]
  const int kpad = (k + 3) & ~3;                                            // candidate slots per query
  uint32_t* cand_key = reinterpret_cast<uint32_t*>(ring + P.fo_cand);       // [n_q][kpad]
  int* cand_pos = reinterpret_cast<int*>(cand_key + n_q * kpad);            // [n_q][kpad]
  const int ng = P.nsplit * kpad;                                           // gathered per query
  uint32_t* gkey = reinterpret_cast<uint32_t*>(ring + P.fo_gath);           // [n_q][ng]
  int* gpos = reinterpret_cast<int*>(gkey + n_q * ng);                      // [n_q][ng]
  float* kbar_s = reinterpret_cast<float*>(ring + P.fo_kbar);               // [kRows][kStride]
  float* iq_s = reinterpret_cast<float*>(ring + P.fo_iq);                   // [n_q][Hi][kDI]
  float* iw_s = reinterpret_cast<float*>(ring + P.fo_iw);                   // [n_q][Hi]
  float* new_s = reinterpret_cast<float*>(ring + P.fo_new);                 // [2][kDI]
  int* hist = reinterpret_cast<int*>(ring + P.fo_hist);
  float2(*part)[32] = reinterpret_cast<float2(*)[32]>(hist + 280);           // [8][32]

  // paged caches: every page the step may gather must be in the pool
  if (P.table && hk == 0) {
    const int nb_used = (kv + g.B - 1) / g.B;
    for (int j = split + P.nsplit * tid; j < nb_used; j += P.nsplit * nthr) {
      const int page = P.table[(size_t)b * nblk_cap + j];
      if ((page < 0 || page >= P.num_pages) && P.err) atomicExch(P.err, 3);
    }
  }
  __syncthreads();   // the caller staged iq_s and iw_s
  if (g.rope_dim)     // query i turned at its position kv - n_q + i (read after the next barrier)
    rope_rows(iq_s, n_q * Hi, Hi, kQStrideI, kv - n_q, g.rope_dim, g.rope_theta, tid, nthr);
  // blocks completed by this step's tokens (at most two: n_q <= 4 < B)
  const int jn_lo = max((kv - n_q) / g.B, j0), jn_hi = min(nc_last, j1);
  for (int j = jn_lo; j < jn_hi; ++j) {
    size_t r0 = (size_t)b * P.cap + (size_t)j * g.B;
    bool ok = true;
    if (P.table) {
      const int page = P.table[(size_t)b * nblk_cap + j];
      ok = page >= 0 && page < P.num_pages;
      r0 = (size_t)page * g.B;
    }
    float* dst = new_s + (j - jn_lo) * kDI;
    if (ok) {   // uniform across the CTA
      pool_block_halves<__nv_bfloat16, kDI>(P.ik_cache + (ok ? r0 : 0) * kDI, g.B, dst, part,
                                            g.rope_dim, g.rope_theta, j * g.B);
    } else {    // a page outside the pool (reported): the cached row stands
      for (int d = tid; d < kDI; d += nthr) dst[d] = P.pooled[((size_t)b * nblk_cap + j) * kDI + d];
    }
    __syncthreads();
    if (hk == 0 && ok)
      for (int d = tid; d < kDI; d += nthr) P.pooled[((size_t)b * nblk_cap + j) * kDI + d] = dst[d];
  }
  // score the range, kRows blocks at a time
  for (int r0 = j0; r0 < j1; r0 += kRows) {
    const int rows = min(kRows, j1 - r0);
    {   // every load of the pass is issued before the first store
      constexpr int kLd = (kRows * (kDI / 4) + kThreads - 1) / kThreads;   // float4 per thread
      float4 v[kLd];
#pragma unroll
      for (int u = 0; u < kLd; ++u) {
        const int e = tid + u * kThreads;
        const int r = e / (kDI / 4), d4 = e - r * (kDI / 4);
        const int j = r0 + r;
        v[u] = r >= rows ? make_float4(0.f, 0.f, 0.f, 0.f)
               : (j >= jn_lo && j < jn_hi)
                   ? *reinterpret_cast<const float4*>(new_s + (j - jn_lo) * kDI + 4 * d4)
                   : __ldg(reinterpret_cast<const float4*>(P.pooled + ((size_t)b * nblk_cap + j) * kDI) + d4);
      }
#pragma unroll
      for (int u = 0; u < kLd; ++u) {
        const int e = tid + u * kThreads;
        const int r = e / (kDI / 4), d4 = e - r * (kDI / 4);
        if (r < rows) *reinterpret_cast<float4*>(kbar_s + r * kStride + 4 * d4) = v[u];
      }
    }
    __syncthreads();
    // For each query, thread t takes head t % Hi of blocks r = t / Hi + m * hpr,
    // m < 4 (hpr = nthr / Hi; nthr is a multiple of Hi, so a block's heads are
    // adjacent lanes of one warp): four blocks share each q load. Each dot
    // product is one fma chain over the dims in ascending order, as in the
    // selection kernel; the heads' terms are summed by shuffles. iq rows are
    // padded to kQStrideI floats so that the heads of a warp read distinct banks.
    const int hpr = nthr / Hi, h = tid % Hi, slot = tid / Hi;
    for (int i = 0; i < n_q; ++i) {
      const int lim = kv - n_q + 1 + i;   // block j is complete for query i iff (j + 1) B <= lim
      const float4* qv = reinterpret_cast<const float4*>(iq_s + (i * Hi + h) * kQStrideI);
      const float wq = iw_s[i * Hi + h];
      for (int rb = 0; rb < rows; rb += 4 * hpr) {   // uniform
        int rr[4];
        bool live[4];
        const float4* kr[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          rr[m] = rb + slot + m * hpr;
          live[m] = rr[m] < rows && (r0 + rr[m] + 1) * g.B <= lim;
          kr[m] = reinterpret_cast<const float4*>(kbar_s + (live[m] ? rr[m] : 0) * kStride);
        }
        float dt[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int d4 = 0; d4 < kDI / 4; ++d4) {
          const float4 qa = qv[d4];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const float4 ka = kr[m][d4];
            dt[m] = fmaf(qa.x, ka.x, dt[m]);
            dt[m] = fmaf(qa.y, ka.y, dt[m]);
            dt[m] = fmaf(qa.z, ka.z, dt[m]);
            dt[m] = fmaf(qa.w, ka.w, dt[m]);
          }
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float t = live[m] ? wq * fmaxf(dt[m], 0.f) : 0.f;
          for (int o = 1; o < Hi; o <<= 1) t += __shfl_xor_sync(kFull, t, o);
          if (h == 0 && live[m]) keys_mine[i * per + (r0 + rr[m] - j0)] = score_key(t * g.idx_scale);
        }
      }
    }
    __syncthreads();
  }
  // Top-k in two steps. Each CTA first takes the top k of its own range for
  // every query (warp i, query i): every block of the cluster's top k is among
  // them, since fewer than k blocks of the whole cache beat it, so fewer than k
  // of its range. After a cluster barrier each CTA gathers all CTAs'
  // candidates (CTA order is ascending block order, so a lower position still
  // wins a tie) and takes the top k of those for every query itself: no bitmap
  // has to cross the cluster afterwards.
  // With k <= 32 every list is a sorted top-32 held one value per lane: the
  // range's keys are sorted 32 at a time and merged into the running top 32,
  // and the candidate list is written in rank order.
  if (warp < n_q) {
    const int i = warp;
    const int cnt = max(0, min(j1, (kv - n_q + 1 + i) / g.B) - j0);   // query i's blocks here
    if (k <= 32) {
      const uint32_t* kq = keys_mine + i * per;
      unsigned long long top = 0ull;
      for (int r0 = 0; r0 < cnt; r0 += 32) {   // uniform
        const int r = r0 + lane;
        const unsigned long long v =
            warp_sort32_desc(r < cnt ? cand_value(kq[r], j0 + r) : 0ull);
        top = r0 == 0 ? v : warp_merge32_desc(top, v);
      }
      if (lane < kpad) {
        const bool real = lane < k && top != 0ull;
        cand_key[i * kpad + lane] = real ? (uint32_t)(top >> 32) : 0u;
        cand_pos[i * kpad + lane] = real ? (int)(0xffffffffu - (uint32_t)top) : 0x7fffffff;
      }
    } else {
      warp_topk_compact(keys_mine + i * per, cnt, min(k, cnt), j0, cand_key + i * kpad,
                        cand_pos + i * kpad, kpad);
    }
  }
  cluster_sync_all();   // every CTA's candidates are in place
  {   // 16-byte groups of four candidates (keys, then positions) from every CTA
    const int groups = n_q * P.nsplit * (kpad / 4);
    const uint32_t ck_s = smem_u32(cand_key), cp_s = smem_u32(cand_pos);
    for (int e = tid; e < groups; e += nthr) {
      const int i = e / (P.nsplit * (kpad / 4)), rem = e - i * (P.nsplit * (kpad / 4));
      const int c = rem / (kpad / 4), q4 = rem - c * (kpad / 4);
      const uint32_t off = 4u * (uint32_t)(i * kpad + 4 * q4);
      const uint4 kv4 = ld_cluster_u32x4(cluster_map(ck_s + off, c));
      const uint4 pv4 = ld_cluster_u32x4(cluster_map(cp_s + off, c));
      *reinterpret_cast<uint4*>(gkey + i * ng + c * kpad + 4 * q4) = kv4;
      *reinterpret_cast<uint4*>(gpos + i * ng + c * kpad + 4 * q4) = pv4;
    }
  }
  __syncthreads();
  if (warp < n_q) {
    const int i = warp;
    const int n = kv - n_q + 1 + i;
    const int nc_i = n / g.B;
    uint32_t* qb = qbits + i * words;
    if (k <= 32) {
      // every CTA's list is sorted: merge them pairwise into the top 32
      unsigned long long top = 0ull;
      for (int c = 0; c < P.nsplit; c += 2) {   // uniform
        const int a = i * ng + c * kpad + lane, bb = a + kpad;
        unsigned long long v = lane < kpad ? cand_value(gkey[a], gpos[a]) : 0ull;
        if (lane < kpad && gkey[a] == 0u) v = 0ull;
        if (c + 1 < P.nsplit) {
          unsigned long long w = lane < kpad ? cand_value(gkey[bb], gpos[bb]) : 0ull;
          if (lane < kpad && gkey[bb] == 0u) w = 0ull;
          v = warp_merge32_desc(v, w);
        }
        top = c == 0 ? v : warp_merge32_desc(top, v);
      }
      const int pos = (int)(0xffffffffu - (uint32_t)top);
      if (lane < min(k, nc_i) && top != 0ull) atomicOr(&qb[pos >> 5], 1u << (pos & 31));
    } else {
      warp_topk_bits(gkey + i * ng, gpos + i * ng, ng, min(k, nc_i), qb);
    }
    __syncwarp();
    if (lane == 0 && n - nc_i * g.B > 0) atomicOr(&qb[nc_i >> 5], 1u << (nc_i & 31));   // tail
  }
  __syncthreads();
  if (split == 0 && hk == 0 && warp < n_q) {   // the selection lists: ascending, tail last
    const int i = warp;
    const int nc_i = (kv - n_q + 1 + i) / g.B;
    const uint32_t* qb = qbits + i * words;
    int* srow = P.sel_w + ((size_t)b * n_q + i) * kp1;
    const int nw = min(words, (nc_i + 1 + 31) >> 5);
    int base = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int w = w0 + lane;
      uint32_t m = w < nw ? qb[w] : 0u;
      const int c = __popc(m);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
      }
      int off = base + incl - c;
      while (m) {
        const int bp = __ffs(m) - 1;
        m &= m - 1;
        if (off < kp1) srow[off] = w * 32 + bp;
        ++off;
      }
      base += __shfl_sync(kFull, incl, 31);
    }
    for (int e = base + lane; e < kp1; e += 32) srow[e] = -1;
    if (lane == 0) P.nsel_w[(size_t)b * n_q + i] = min(base, kp1);
  }
  cluster_arrive_all();   // this CTA has read the other CTAs' candidates
}

template <bool kFp8, int kSelDI, int kRT, bool kCount>
__global__ void __launch_bounds__(kThreads, kRT == 1 ? 2 : 1)
attn_decode_mma_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const DecParams P) {
  static_assert(kRT == 1 || (kRT == 2 && !kFp8), "fp8 caches: one 16-row tile");
  using L = DecLayout<kRT>;
  // Consumer warp w works on row tile w / kWPT and keys [kKW (w % kWPT), + kKW)
  // of every chunk: 16 keys with one row tile, 32 keys with two.
  constexpr int kWPT = kConsumers / kRT;   // consumer warps per row tile
  constexpr int kKW = kChunk / kWPT;       // keys per warp and chunk
  constexpr int kNT = kKW / 8;             // n-tiles of 8 keys (QK^T)
  constexpr int kKS = kKW / 16;            // k-steps of 16 keys (PV)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(smem);
  const Geom& g = P.g;
  const int split = blockIdx.x, b = blockIdx.y, hk = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = g.G, n_q = P.n_q, R = n_q * G;
  if constexpr (kSelDI > 0) grid_dependency_wait();   // every input may come from the previous kernel
  // Inputs that do not depend on the sequence's length are loaded together
  // with it, into registers: Q rows r = i * G + gi (query i, head hk * G + gi;
  // zero beyond R), the gate rows this CTA merges (cluster merge: rows split,
  // split + nsplit, ...), and for the in-kernel selection the queries' indexer
  // q and weights.
  constexpr int kQLd = (L::kRows * (kD / 8) + kThreads - 1) / kThreads;
  uint4 qreg[kQLd];
#pragma unroll
  for (int u = 0; u < kQLd; ++u) {
    const int e = threadIdx.x + u * kThreads, r = e / (kD / 8), c8 = e % (kD / 8);
    qreg[u] = make_uint4(0, 0, 0, 0);
    if (e < L::kRows * (kD / 8) && r < R)
      qreg[u] = *reinterpret_cast<const uint4*>(
          P.q + (((size_t)b * n_q + r / G) * g.Hq + hk * G + r % G) * kD + c8 * 8);
  }
  const int g_per_row = g.gate_headwise ? 1 : kD / 8;   // uint4 per gate row (or one value)
  const int g_rows = P.cluster && split < R ? (R - split + P.nsplit - 1) / P.nsplit : 0;
  constexpr int kGLd = (L::kRows * (kD / 8) + kThreads - 1) / kThreads;
  uint4 greg[kGLd];   // g_rows * g_per_row <= rows * 16
#pragma unroll
  for (int u = 0; u < kGLd; ++u) {
    const int e = threadIdx.x + u * kThreads;
    greg[u] = make_uint4(0, 0, 0, 0);
    if (e < g_rows * g_per_row) {
      const int lr = e / g_per_row, c8 = e - lr * g_per_row, r = split + lr * P.nsplit;
      const size_t orow = ((size_t)b * n_q + r / G) * g.Hq + hk * G + r % G;
      if (g.gate_headwise)
        greg[u].x = *reinterpret_cast<const unsigned short*>(P.gate + orow);
      else
        greg[u] = *reinterpret_cast<const uint4*>(P.gate + orow * kD + c8 * 8);
    }
  }
  uint4 iqreg[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
  float iwreg = 0.f;
  if constexpr (kSelDI > 0) {
    const int nq8 = n_q * g.Hi * kSelDI / 8;
    const uint4* iqb = reinterpret_cast<const uint4*>(P.iq + (size_t)b * nq8 * 8);
#pragma unroll
    for (int u = 0; u < 2; ++u)
      if (threadIdx.x + u * kThreads < nq8) iqreg[u] = iqb[threadIdx.x + u * kThreads];
    if (threadIdx.x < n_q * g.Hi) iwreg = P.iw[(size_t)b * n_q * g.Hi + threadIdx.x];
  }
  const int kv = P.kv_len[b] - P.row_off;   // (a shard's rows: may be past either end)
  const size_t row0 = (((size_t)b * g.Hkv + hk) * P.nsplit + split) * R;
  if (!P.cp && (kv < n_q || kv > P.cap)) {   // reported by the selection; outputs are zero
    if (split == 0 && hk == 0) {
      if constexpr (kSelDI > 0) {
        const int kp1 = g.k + 1;
        for (int e = threadIdx.x; e < n_q * kp1; e += blockDim.x) P.sel_w[(size_t)b * n_q * kp1 + e] = -1;
        for (int e = threadIdx.x; e < n_q; e += blockDim.x) P.nsel_w[(size_t)b * n_q + e] = 0;
      }
      if (P.err && threadIdx.x == 0) atomicExch(P.err, 1);
    }
    if (split == 0)
      for (int e = threadIdx.x; e < R * kD; e += blockDim.x) {
        const int r = e / kD, d = e - r * kD;
        const size_t orow = ((size_t)b * n_q + r / G) * g.Hq + hk * G + r % G;
        P.out[orow * kD + d] = __float2bfloat16_rn(0.f);
        if (P.lse && d == 0) P.lse[orow] = -INFINITY;
      }
    return;
  }
  if constexpr (kSelDI > 0)
    if (threadIdx.x == 0) select_prefetch<kSelDI>(P, kv, split, b);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  int* n_chunks_s = reinterpret_cast<int*>(smem + L::kOffMisc + 4);
  unsigned* visited_s = reinterpret_cast<unsigned*>(smem + L::kOffMisc + 8);   // debug, [kConsumers]
  int* u_blk = reinterpret_cast<int*>(smem + L::kOffUnion);
  int* u_qm = u_blk + kMaxUnion;
  const int cpb = g.B / kChunk;   // chunks per block

  // union of the n_q selections (selected blocks and tail blocks), ascending,
  // with a mask of the queries that selected each block: per-query bitmaps in
  // shared memory, then one ordered scan by warp 0
  const int words = (P.cap / g.B + 31) / 32;
  uint32_t* qbits = reinterpret_cast<uint32_t*>(smem + L::kOffBits);   // [n_q][words]
  for (int e = threadIdx.x; e < n_q * words; e += blockDim.x) qbits[e] = 0u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    *abort_flag = 0;
    if constexpr (kCount)
      for (int w = 0; w < kConsumers; ++w) visited_s[w] = 0u;
    fence_barrier_init();
    fence_proxy_async();
  }
  // Q to shared memory (before the selection exists)
  if constexpr (!kFp8) {
#pragma unroll
    for (int u = 0; u < kQLd; ++u) {
      const int e = threadIdx.x + u * kThreads, r = e / (kD / 8), c8 = e % (kD / 8);
      if (e < L::kRows * (kD / 8))
        *reinterpret_cast<uint4*>(smem + L::kOffQ + r * kQStride + c8 * 16) = qreg[u];
    }
  } else {
    // fp32 rows in the (still unused) fp16 tile area, rotated into the cache's
    // basis (q' = H q) when the cache holds H k, then stored as fp16
    float* qf = reinterpret_cast<float*>(smem + kOffStages + kStages * kF8StageBytes);
#pragma unroll
    for (int u = 0; u < kQLd; ++u) {
      const int e = threadIdx.x + u * kThreads;
      if (e < 16 * (kD / 8)) {
        const uint32_t w[4] = {qreg[u].x, qreg[u].y, qreg[u].z, qreg[u].w};
        float4* dst = reinterpret_cast<float4*>(qf + 8 * e);
        dst[0] = make_float4(__uint_as_float(w[0] << 16), __uint_as_float(w[0] & 0xffff0000u),
                             __uint_as_float(w[1] << 16), __uint_as_float(w[1] & 0xffff0000u));
        dst[1] = make_float4(__uint_as_float(w[2] << 16), __uint_as_float(w[2] & 0xffff0000u),
                             __uint_as_float(w[3] << 16), __uint_as_float(w[3] & 0xffff0000u));
      }
    }
    __syncthreads();
    if (P.rotated) fwht128_rows(qf, 16, (int)threadIdx.x, (int)blockDim.x, [] { __syncthreads(); });
    // Within each 16-dim block the MMA's k order is permuted (the same on the K
    // side, so the dot products are unchanged): fragment positions 2t, 2t + 1,
    // 2t + 8, 2t + 9 hold dims 4t .. 4t + 3, so that a thread's K fragment is
    // one 32-bit word of four e4m3 codes. Logical 8-group c8 holds dims
    // (c8 % 2) * 2 + 4m + {0, 1}, m < 4, of its block.
    for (int e = threadIdx.x; e < 16 * (kD / 8); e += blockDim.x) {
      const int r = e / (kD / 8), c8 = e % (kD / 8);
      const float* src = qf + r * kD + (c8 >> 1) * 16 + (c8 & 1) * 2;
      const uint4 v = make_uint4(pack2h(src[0], src[1]), pack2h(src[4], src[5]),
                                 pack2h(src[8], src[9]), pack2h(src[12], src[13]));
      *reinterpret_cast<uint4*>(smem + L::kOffQ + r * kQStride + c8 * 16) = v;
    }
  }
  // the gate rows this CTA merges (cluster merge), or the merging CTA's rows
  // into L2
  __nv_bfloat16* gate_s = reinterpret_cast<__nv_bfloat16*>(smem + L::kOffGate);
  if (P.cluster) {
#pragma unroll
    for (int u = 0; u < kGLd; ++u) {
      const int e = threadIdx.x + u * kThreads;
      if (e < g_rows * g_per_row) {
        const int lr = e / g_per_row, c8 = e - lr * g_per_row;
        if (g.gate_headwise)
          *reinterpret_cast<unsigned short*>(gate_s + lr * kD) = (unsigned short)greg[u].x;
        else
          *reinterpret_cast<uint4*>(gate_s + lr * kD + c8 * 8) = greg[u];
      }
    }
  } else if (split == 0 && !g.gate_headwise && threadIdx.x < R * (kD * 2 / 128)) {
    const int r = threadIdx.x / (kD * 2 / 128), part = threadIdx.x % (kD * 2 / 128);
    const size_t orow = ((size_t)b * n_q + r / G) * g.Hq + hk * G + r % G;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(P.gate + orow * kD + part * 64));
  }
  bool gave_up = false;
  if constexpr (kSelDI > 0) {
    __syncthreads();   // Q staging may have used the ring's space
    {   // the queries' indexer q (fp32, rows padded to di + 4 floats) and weights
      float* iq_s = reinterpret_cast<float*>(smem + kOffStages + P.fo_iq);
      const int nq8 = n_q * g.Hi * kSelDI / 8;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int e = threadIdx.x + u * kThreads;
        if (e < nq8) {
          const uint32_t w[4] = {iqreg[u].x, iqreg[u].y, iqreg[u].z, iqreg[u].w};
          float4* dst = reinterpret_cast<float4*>(iq_s + (8 * e / kSelDI) * (kSelDI + 4) + 8 * e % kSelDI);
          dst[0] = make_float4(__uint_as_float(w[0] << 16), __uint_as_float(w[0] & 0xffff0000u),
                               __uint_as_float(w[1] << 16), __uint_as_float(w[1] & 0xffff0000u));
          dst[1] = make_float4(__uint_as_float(w[2] << 16), __uint_as_float(w[2] & 0xffff0000u),
                               __uint_as_float(w[3] << 16), __uint_as_float(w[3] & 0xffff0000u));
        }
      }
      const uint4* iqb = reinterpret_cast<const uint4*>(P.iq + (size_t)b * nq8 * 8);
      for (int e = threadIdx.x + 2 * kThreads; e < nq8; e += kThreads) {   // beyond 2 per thread
        const uint4 v = iqb[e];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float4* dst = reinterpret_cast<float4*>(iq_s + (8 * e / kSelDI) * (kSelDI + 4) + 8 * e % kSelDI);
        dst[0] = make_float4(__uint_as_float(w[0] << 16), __uint_as_float(w[0] & 0xffff0000u),
                             __uint_as_float(w[1] << 16), __uint_as_float(w[1] & 0xffff0000u));
        dst[1] = make_float4(__uint_as_float(w[2] << 16), __uint_as_float(w[2] & 0xffff0000u),
                             __uint_as_float(w[3] << 16), __uint_as_float(w[3] & 0xffff0000u));
      }
      float* iw_s = reinterpret_cast<float*>(smem + kOffStages + P.fo_iw);
      if (threadIdx.x < n_q * g.Hi) iw_s[threadIdx.x] = iwreg;
    }
    select_in_cluster<kSelDI>(P, smem, kv, split, b, hk, qbits, words);
  } else {
    // the selections come from the selection kernel: wait for this sequence's
    // flag (bounded), or for the whole selection grid
    if (P.ready) {
      if (threadIdx.x == 0) {
        const long long t0 = clock64();
        while (true) {
          int v;
          asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(P.ready + b) : "memory");
          if (v != 0) break;
          if (clock64() - t0 > kWaitCycles) {
            *abort_flag = 1;
            break;
          }
          __nanosleep(128);
        }
      }
    } else {
      grid_dependency_wait();
    }
    __syncthreads();
    gave_up = *abort_flag != 0;
    if (gave_up && !P.cluster) {   // nothing issued yet: report and leave (no merge for this pair)
      if (threadIdx.x == 0 && P.err) atomicExch(P.err, 2);
      return;
    }
    // (a cluster CTA that gave up still takes part in the cluster's barriers, with
    // an empty partial)
    if (!gave_up) {
      const int kp1 = g.k + 1;
      const int nblk = P.cap / g.B;
      for (int e = threadIdx.x; e < n_q * kp1; e += blockDim.x) {
        const int i = e / kp1, j = e - i * kp1;
        if (j < P.nsel[(size_t)b * n_q + i]) {
          const int blk = P.sel[((size_t)b * n_q + i) * kp1 + j] - P.block_lo;
          if (blk >= 0 && blk < nblk) atomicOr(&qbits[i * words + (blk >> 5)], 1u << (blk & 31));
        }
      }
    }
    __syncthreads();
  }
  if (warp == 0) {
    int base = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int w = w0 + lane;
      uint32_t qw[4] = {0u, 0u, 0u, 0u}, bits = 0u;
      if (w < words)
        for (int i = 0; i < n_q; ++i) {
          qw[i] = qbits[i * words + w];
          bits |= qw[i];
        }
      const int c = __popc(bits);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
      }
      int off = base + incl - c;
      while (bits) {
        const int bp = __ffs(bits) - 1;
        bits &= bits - 1;
        int qm = 0;
        for (int i = 0; i < n_q; ++i) qm |= ((qw[i] >> bp) & 1u) << i;
        u_blk[off] = w * 32 + bp;
        u_qm[off] = qm;
        ++off;
      }
      base += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) *n_chunks_s = gave_up ? 0 : base * cpb;
  }
  __syncthreads();
  // (in-kernel selection: the other CTAs of the cluster have finished reading
  // this CTA's score keys, so the ring may be filled)
  if constexpr (kSelDI > 0) cluster_wait_all();
  const int n_chunks = *n_chunks_s;
  const int c0 = split * P.per_split;
  const int c1 = min(n_chunks, c0 + P.per_split);
  const int my_chunks = max(0, c1 - c0);
  const size_t krow_base = (size_t)b * P.cap;

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && my_chunks > 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int c = 0; c < my_chunks; ++c) {
        const int s = c % kStages;
        if (c >= kStages && !mbar_wait(&empty[s], ((c / kStages) - 1) & 1, abort_flag)) break;
        const int uc = c0 + c;
        const int blk = u_blk[uc / cpb], off = (uc % cpb) * kChunk;
        // the chunk's first cache row: in the sequence's slab, or in the block's
        // page (an out-of-range page id reads zeros; the selection kernel has
        // reported it)
        const int rowk = P.table ? P.table[(size_t)b * (P.cap / g.B) + blk] * g.B + off
                                 : (int)(krow_base + (size_t)blk * g.B + off);
        if constexpr (!kFp8) {
          const uint32_t st = sbase + kOffStages + s * kStageBytes;
          mbar_expect_tx(&full[s], kStageBytes);
          tma_load_3d(st, &tmK, 0, hk, rowk, &full[s]);
          tma_load_3d(st + kBoxBytes, &tmK, 64, hk, rowk, &full[s]);
          tma_load_3d(st + kTileBytes, &tmV, 0, hk, rowk, &full[s]);
          tma_load_3d(st + kTileBytes + kBoxBytes, &tmV, 64, hk, rowk, &full[s]);
        } else {
          // e4m3 rows (one 128-byte box each) and the chunk's row scales of all
          // KV heads (64 * Hkv contiguous floats: rowk is a multiple of 64)
          const uint32_t st = sbase + kOffStages + s * kF8StageBytes;
          const uint32_t sb = 64u * g.Hkv * 4u;
          mbar_expect_tx(&full[s], 2 * kF8BoxBytes + 2 * sb);
          tma_load_3d(st, &tmK, 0, hk, rowk, &full[s]);
          tma_load_3d(st + kF8BoxBytes, &tmV, 0, hk, rowk, &full[s]);
          bulk_load(st + 2 * kF8BoxBytes, P.k_scale + (size_t)rowk * g.Hkv, sb, &full[s]);
          bulk_load(st + 2 * kF8BoxBytes + kF8ScaleBytes, P.v_scale + (size_t)rowk * g.Hkv, sb,
                    &full[s]);
        }
        issued = c + 1;
      }
      for (int c = max(0, issued - kStages); c < issued; ++c)
        mbar_wait(&full[c % kStages], (c / kStages) & 1, abort_flag);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int gq = lane >> 2, tq = lane & 3;   // mma fragment row group / column pair
    const int tile = warp / kWPT;                // this warp's 16 query rows
    const int kw0 = (warp % kWPT) * kKW;         // and its keys of each chunk
    // Q as A fragments, all 8 k-slices of 16 dims
    uint32_t qa[8][4];
    {
      const int mi = lane >> 3, ri = lane & 7;
      const int row = tile * 16 + (mi & 1) * 8 + ri;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int col = kk * 16 + (mi >> 1) * 8;
        ldsm_x4(sbase + L::kOffQ + row * kQStride + col * 2, qa[kk][0], qa[kk][1], qa[kk][2],
                qa[kk][3]);
      }
    }
    // the two rows this thread holds: gq and gq + 8 of the tile
    int qrow[2], qpos[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int r = tile * 16 + gq + 8 * h2;
      qrow[h2] = r < R ? r / G : -1;                    // query index, -1 for padding
      qpos[h2] = r < R ? kv - n_q + qrow[h2] : -1;      // last visible position
    }
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    const float sc = g.sm_scale_log2;
    const int mi = lane >> 3, ri = lane & 7;
    for (int c = 0; c < my_chunks; ++c) {
      const int s = c % kStages;
      if (!mbar_wait(&full[s], (c / kStages) & 1, abort_flag)) break;
      const int uc = c0 + c;
      const int ub = uc / cpb;
      const int blk = u_blk[ub], qm = u_qm[ub];
      const int key0 = blk * g.B + (uc % cpb) * kChunk;
      // Keys no row of this CTA may see are not part of any selection (the
      // tail block's keys past the newest query): their V rows are zeroed so
      // that P = 0 cannot meet a non-finite V in the MMA.
      int lim_all = 0;
      for (int i = 0; i < n_q; ++i)
        if ((qm >> i) & 1) lim_all = max(lim_all, min(kChunk, max(0, kv - n_q + i + 1 - key0)));
      uint32_t kt = 0, vt;   // K and V tiles (64-key bf16 tiles; fp8: this warp's 16-key fp16 V tile)
      const uint32_t st8 = kOffStages + s * kF8StageBytes;   // fp8 stage: K codes, V codes, scales
      if constexpr (!kFp8) {
        kt = sbase + kOffStages + s * kStageBytes;
        vt = kt + kTileBytes;
      } else {
        // widen this warp's 16 V rows (rows 16w .. 16w + 15 of the chunk) from
        // e4m3 times the row scale to fp16; rows no query may see are zero. K is
        // read as e4m3 straight into the MMA fragments below (its row scales
        // multiply the scores).
        const uint32_t tiles = kOffStages + kStages * kF8StageBytes + warp * 2 * kWarpTileBytes;
        vt = sbase + tiles + kWarpTileBytes;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int u = lane + 32 * i;
          const int rr = u >> 3, ch = u & 7;   // row of the warp's 16, 16-dim chunk
          const int row = warp * 16 + rr;      // row in the chunk
          uint4 out0 = make_uint4(0, 0, 0, 0), out1 = make_uint4(0, 0, 0, 0);
          if (row < lim_all) {
            const uint4 in = *reinterpret_cast<const uint4*>(
                smem + st8 + kF8BoxBytes + row * 128 + ((ch ^ (row & 7)) << 4));
            const float scl = reinterpret_cast<const float*>(
                smem + st8 + 2 * kF8BoxBytes + kF8ScaleBytes)[row * g.Hkv + hk];
            const uint32_t s2 = pack2h(scl, scl);
            out0 = make_uint4(e4m3x2_scaled(in.x & 0xffffu, s2), e4m3x2_scaled(in.x >> 16, s2),
                              e4m3x2_scaled(in.y & 0xffffu, s2), e4m3x2_scaled(in.y >> 16, s2));
            out1 = make_uint4(e4m3x2_scaled(in.z & 0xffffu, s2), e4m3x2_scaled(in.z >> 16, s2),
                              e4m3x2_scaled(in.w & 0xffffu, s2), e4m3x2_scaled(in.w >> 16, s2));
          }
          uint8_t* dst = smem + tiles + kWarpTileBytes;
          *reinterpret_cast<uint4*>(dst + tile16_off(rr, 16 * ch)) = out0;
          *reinterpret_cast<uint4*>(dst + tile16_off(rr, 16 * ch + 8)) = out1;
        }
      }
      // visible keys of this chunk per held row: keys key0 + j with j < lim
      int lim[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
        lim[h2] = (qrow[h2] >= 0 && ((qm >> qrow[h2]) & 1))
                      ? max(0, min(kChunk, qpos[h2] + 1 - key0))
                      : 0;
      if (kCount && tq == 0)   // debug count of the visible (row, key) pairs of this
                               // warp's keys (a quad's threads share two rows)
        atomicAdd(reinterpret_cast<unsigned*>(smem + L::kOffMisc + 8) + warp, (unsigned)(min(kKW, max(0, lim[0] - kw0)) +
                                               min(kKW, max(0, lim[1] - kw0))));
      // S = Q K^T for the warp's keys [kw0, kw0 + kKW): kNT n-tiles of 8 keys
      float sfr[kNT][4];
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) sfr[nt][0] = sfr[nt][1] = sfr[nt][2] = sfr[nt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t b0, b1, b2, b3;
        if constexpr (!kFp8) {
#pragma unroll
          for (int n2 = 0; n2 < kNT / 2; ++n2) {
            const int key = kw0 + n2 * 16 + (mi >> 1) * 8 + ri;
            ldsm_x4(kt + tile_off(key, kk * 16 + (mi & 1) * 8), b0, b1, b2, b3);
            mma_bf16(sfr[2 * n2], qa[kk], b0, b1);
            mma_bf16(sfr[2 * n2 + 1], qa[kk], b2, b3);
          }
        } else {
          // B fragment of key row 16w + 8 nt + gq: the four e4m3 codes of dims
          // kk * 16 + 4 tq .. + 3 of the 128-byte-swizzled row (the permuted k
          // order of the Q staging), widened to two fp16x2
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const int row = warp * 16 + nt * 8 + gq;
            const uint32_t w4 = *reinterpret_cast<const uint32_t*>(
                smem + st8 + row * 128 + ((kk ^ (row & 7)) << 4) + 4 * tq);
            b0 = e4m3x2(w4 & 0xffffu);
            b1 = e4m3x2(w4 >> 16);
            mma_f16(sfr[nt], qa[kk], b0, b1);
          }
          (void)b2;
          (void)b3;
        }
      }
      // mask, scale, online softmax (per row across the quad's 4 threads); fp8:
      // the K row scales multiply the scores
      float ksc[2][2] = {{1.f, 1.f}, {1.f, 1.f}};
      if constexpr (kFp8) {
        const float* ks = reinterpret_cast<const float*>(smem + st8 + 2 * kF8BoxBytes);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int c = 0; c < 2; ++c) ksc[nt][c] = ks[(warp * 16 + nt * 8 + 2 * tq + c) * g.Hkv + hk];
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);   // K and its scales are read, V is widened
      }
      float x[kNT][4];
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h2 = e >> 1;
          const int j = kw0 + nt * 8 + 2 * tq + (e & 1);
          x[nt][e] = j < lim[h2] ? sfr[nt][e] * (kFp8 ? sc * ksc[nt & 1][e & 1] : sc) : -INFINITY;
        }
      float alpha[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        float mx = fmaxf(fmaxf(x[0][2 * h2], x[0][2 * h2 + 1]), fmaxf(x[1][2 * h2], x[1][2 * h2 + 1]));
#pragma unroll
        for (int nt = 2; nt < kNT; ++nt) mx = fmax3(mx, x[nt][2 * h2], x[nt][2 * h2 + 1]);
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        const float m_new = fmaxf(m[h2], mx);
        const float ref = m_new == -INFINITY ? 0.f : m_new;
        alpha[h2] = ex2_approx(m[h2] - ref);
        m[h2] = m_new;
        float rs = 0.f;
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
          for (int e = 2 * h2; e < 2 * h2 + 2; ++e) {
            x[nt][e] = ex2_approx(x[nt][e] - ref);
            rs += x[nt][e];
          }
        l[h2] = l[h2] * alpha[h2] + rs;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        o[i][0] *= alpha[0];
        o[i][1] *= alpha[0];
        o[i][2] *= alpha[1];
        o[i][3] *= alpha[1];
      }
      if (!kFp8 && lim_all < kw0 + kKW) {
        for (int e = lane; e < kKW * 16; e += 32) {   // kKW rows x 2 boxes x 8 chunks of 16 B
          const int row = kw0 + (e >> 4);
          const int box = (e >> 3) & 1, ch = e & 7;
          if (row >= lim_all)
            *reinterpret_cast<uint4*>(smem + (vt - sbase) + box * kBoxBytes + row * 128 + ch * 16) =
                make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }
      // P as A fragments of 16x16 (rows x keys) tiles, one per 16 keys
      uint32_t pa[kKS][4];
#pragma unroll
      for (int ks = 0; ks < kKS; ++ks) {
        if constexpr (!kFp8) {
          pa[ks][0] = pack2(x[2 * ks][0], x[2 * ks][1]);
          pa[ks][1] = pack2(x[2 * ks][2], x[2 * ks][3]);
          pa[ks][2] = pack2(x[2 * ks + 1][0], x[2 * ks + 1][1]);
          pa[ks][3] = pack2(x[2 * ks + 1][2], x[2 * ks + 1][3]);
        } else {
          pa[ks][0] = pack2h(x[2 * ks][0], x[2 * ks][1]);
          pa[ks][1] = pack2h(x[2 * ks][2], x[2 * ks][3]);
          pa[ks][2] = pack2h(x[2 * ks + 1][0], x[2 * ks + 1][1]);
          pa[ks][3] = pack2h(x[2 * ks + 1][2], x[2 * ks + 1][3]);
        }
      }
      // O += P V over the warp's keys, 16 n-tiles of 8 dims
#pragma unroll
      for (int ks = 0; ks < kKS; ++ks)
#pragma unroll
      for (int dn = 0; dn < 16; dn += 2) {
        uint32_t b0, b1, b2, b3;
        if constexpr (!kFp8) {
          const int key = kw0 + ks * 16 + (mi & 1) * 8 + ri;
          ldsm_x4_t(vt + tile_off(key, dn * 8 + (mi >> 1) * 8), b0, b1, b2, b3);
          mma_bf16(o[dn], pa[ks], b0, b1);
          mma_bf16(o[dn + 1], pa[ks], b2, b3);
        } else {
          const int key = (mi & 1) * 8 + ri;
          ldsm_x4_t(vt + tile16_off(key, dn * 8 + (mi >> 1) * 8), b0, b1, b2, b3);
          mma_f16(o[dn], pa[ks], b0, b1);
          mma_f16(o[dn + 1], pa[ks], b2, b3);
        }
      }
      __syncwarp();
      if (!kFp8 && lane == 0) mbar_arrive(&empty[s]);
    }
    // merge the states of the warps of each row tile through shared memory
    // (the ring is free): warp w's 16 rows are rows 16 (w / kWPT) + 0 .. 15
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      l[h2] += __shfl_xor_sync(kFull, l[h2], 1);
      l[h2] += __shfl_xor_sync(kFull, l[h2], 2);
    }
    named_bar_sync(1, 32 * kConsumers);   // every consumer is done with the ring
    float* so = reinterpret_cast<float*>(smem + kOffStages);   // [warp][16 rows][128]
    float* sm = so + kConsumers * 16 * kD;                     // [warp][16 rows][2]
#pragma unroll
    for (int dn = 0; dn < 16; ++dn) {
      const int d = dn * 8 + 2 * tq;
      *reinterpret_cast<float2*>(so + (warp * 16 + gq) * kD + d) = make_float2(o[dn][0], o[dn][1]);
      *reinterpret_cast<float2*>(so + (warp * 16 + gq + 8) * kD + d) =
          make_float2(o[dn][2], o[dn][3]);
    }
    if (tq == 0) {
      sm[(warp * 16 + gq) * 2] = m[0];
      sm[(warp * 16 + gq) * 2 + 1] = l[0];
      sm[(warp * 16 + gq + 8) * 2] = m[1];
      sm[(warp * 16 + gq + 8) * 2 + 1] = l[1];
    }
    named_bar_sync(1, 32 * kConsumers);
    if (kCount && threadIdx.x == 0)   // (every consumer warp's count is complete)
      atomicAdd(g.keys_visited, (unsigned long long)visited_s[0] + visited_s[1] + visited_s[2] +
                                    visited_s[3]);
    // thread t of the 128 consumers: rows t / 8 + 16 u (u < kRT), dims [16 (t % 8), + 16)
    const int t = threadIdx.x;
    const int d0 = (t & 7) * 16;
    // a rotated fp8 cache gives O' = H O: the merged rows are rotated back
    // (H is symmetric and orthonormal) before they leave as the partial
    // (cluster merge: every CTA's partial stays in its own shared memory, O in
    // urow and (m, l) in pml, for the cluster's CTAs to read)
    float* urow = sm + kConsumers * 16 * 2;                    // [rows][128]
    float* pml = urow + L::kRows * kD;                         // [rows][2]
    const bool unrotate = kFp8 && P.rotated;
    const bool local = unrotate || P.cluster;
#pragma unroll
    for (int u = 0; u < kRT; ++u) {
      const int rt = t >> 3, r = rt + 16 * u;   // row of tile u
      if (r < R) {
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < kWPT; ++ww) M = fmaxf(M, sm[((u * kWPT + ww) * 16 + rt) * 2]);
        float wsc[kWPT], Ls = 0.f;
#pragma unroll
        for (int ww = 0; ww < kWPT; ++ww) {
          const float mw = sm[((u * kWPT + ww) * 16 + rt) * 2];
          wsc[ww] = mw == -INFINITY ? 0.f : ex2_approx(mw - M);
          Ls += sm[((u * kWPT + ww) * 16 + rt) * 2 + 1] * wsc[ww];
        }
        float* dst = local ? urow + r * kD + d0 : P.part_o + (row0 + r) * kD + d0;
#pragma unroll
        for (int d = 0; d < 16; d += 4) {
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int ww = 0; ww < kWPT; ++ww) {
            const float4 v =
                *reinterpret_cast<const float4*>(so + ((u * kWPT + ww) * 16 + rt) * kD + d0 + d);
            acc.x += v.x * wsc[ww];
            acc.y += v.y * wsc[ww];
            acc.z += v.z * wsc[ww];
            acc.w += v.w * wsc[ww];
          }
          *reinterpret_cast<float4*>(dst + d) = acc;
        }
        if ((t & 7) == 0) {
          float* ml = P.cluster ? pml + 2 * r : P.part_ml + 2 * (row0 + r);
          ml[0] = M;
          ml[1] = Ls;
        }
      }
    }
    const int r = t >> 3;   // (fp8 caches: one row tile)
    if (unrotate) {
      named_bar_sync(1, 32 * kConsumers);
      fwht128_rows(urow, R, t, 32 * kConsumers, [] { named_bar_sync(1, 32 * kConsumers); });
      if (r < R && !P.cluster) {
        float* gdst = P.part_o + (row0 + r) * kD + d0;
#pragma unroll
        for (int d = 0; d < 16; d += 4)
          *reinterpret_cast<float4*>(gdst + d) = *reinterpret_cast<const float4*>(urow + r * kD + d0 + d);
      }
    }
  }
  if (P.cluster) {
    // The cluster's CTAs merge the partials by log-sum-exp straight from each
    // other's shared memory: CTA `split` takes rows split, split + nsplit, ...,
    // and each of its threads four dims of one row (all partials' loads in
    // flight at once), then applies the sigmoid gate on the output staged at the start.
    cluster_sync_all();
    const int ns = P.nsplit;
    const uint32_t pml_s = sbase + kOffStages + (uint32_t)(kConsumers * 16 * kD + kConsumers * 16 * 2 + L::kRows * kD) * 4u;
    const uint32_t po_s = sbase + kOffStages + (uint32_t)(kConsumers * 16 * kD + kConsumers * 16 * 2) * 4u;
    const int mr = split < R ? (R - split + ns - 1) / ns : 0;
    for (int e = threadIdx.x; e < mr * (kD / 4); e += blockDim.x) {
      const int lr = e / (kD / 4), f = e - lr * (kD / 4), r = split + lr * ns;
      float2 ml[kMaxClusterSplits];
#pragma unroll
      for (int j = 0; j < kMaxClusterSplits; ++j)
        if (j < ns) ml[j] = ld_cluster_f32x2(cluster_map(pml_s + 8u * r, j));
      float4 ov[kMaxClusterSplits];
#pragma unroll
      for (int j = 0; j < kMaxClusterSplits; ++j)
        if (j < ns) ov[j] = ld_cluster_f32x4(cluster_map(po_s + 4u * (r * kD + 4 * f), j));
      float M = -INFINITY;
#pragma unroll
      for (int j = 0; j < kMaxClusterSplits; ++j)
        if (j < ns) M = fmaxf(M, ml[j].x);
      float L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < kMaxClusterSplits; ++j)
        if (j < ns) {
          const float wj = ml[j].x == -INFINITY ? 0.f : ex2_approx(ml[j].x - M);
          L = fmaf(ml[j].y, wj, L);
          acc.x = fmaf(ov[j].x, wj, acc.x);
          acc.y = fmaf(ov[j].y, wj, acc.y);
          acc.z = fmaf(ov[j].z, wj, acc.z);
          acc.w = fmaf(ov[j].w, wj, acc.w);
        }
      const float inv = L > 0.f ? 1.f / L : 0.f;
      float gs[4];
      if (g.gate_headwise) {
        gs[0] = gs[1] = gs[2] = gs[3] = sigmoidf_(__bfloat162float(gate_s[lr * kD]));
      } else {
#pragma unroll
        for (int d = 0; d < 4; ++d) gs[d] = sigmoidf_(__bfloat162float(gate_s[lr * kD + 4 * f + d]));
      }
      const int i = r / G, gi = r % G;
      const size_t orow = ((size_t)b * n_q + i) * g.Hq + hk * G + gi;
      if (P.out_f32)
        *reinterpret_cast<float4*>(P.out_f32 + orow * kD + 4 * f) =
            make_float4(acc.x * inv * gs[0], acc.y * inv * gs[1], acc.z * inv * gs[2],
                        acc.w * inv * gs[3]);
      else
        *reinterpret_cast<uint2*>(P.out + orow * kD + 4 * f) =
            make_uint2(pack2(acc.x * inv * gs[0], acc.y * inv * gs[1]),
                       pack2(acc.z * inv * gs[2], acc.w * inv * gs[3]));
      if (P.lse && f == 0) P.lse[orow] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
    cluster_sync_relaxed();   // no CTA leaves while another may still read its partial
    if (threadIdx.x == 0 && *abort_flag && P.err) atomicExch(P.err, 2);
    return;
  }
  // the last CTA of this (sequence, KV head) merges the splits' partials by
  // log-sum-exp and applies the sigmoid gate on the output
  __threadfence();
  __syncthreads();
  __shared__ int last_s;
  if (threadIdx.x == 0) last_s = atomicAdd(&P.counter[(size_t)b * g.Hkv + hk], 1) == P.nsplit - 1;
  __syncthreads();
  if (last_s) {
    __threadfence();
    const size_t rowb = ((size_t)b * g.Hkv + hk) * P.nsplit * R;
    // per-row max over the splits, then each split's weight, in parallel
    float* wgt = reinterpret_cast<float*>(smem + kOffStages);   // [nsplit][R] (ring is free)
    float* rowM = wgt + P.nsplit * R;                            // [R]
    float* rowL = rowM + L::kRows;                               // [R]
    for (int e = threadIdx.x; e < P.nsplit * R; e += blockDim.x)
      wgt[e] = __ldcg(P.part_ml + 2 * (rowb + e));
    __syncthreads();
    if (threadIdx.x < R) {
      float M = -INFINITY;
      for (int sp = 0; sp < P.nsplit; ++sp) M = fmaxf(M, wgt[sp * R + threadIdx.x]);
      rowM[threadIdx.x] = M;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < P.nsplit * R; e += blockDim.x) {
      const float ms = wgt[e], M = rowM[e % R];
      wgt[e] = (ms == -INFINITY) ? 0.f : ex2_approx(ms - M);
    }
    __syncthreads();
    float* lw = rowL + L::kRows;                                  // [nsplit][R]
    for (int e = threadIdx.x; e < P.nsplit * R; e += blockDim.x)
      lw[e] = __ldcg(P.part_ml + 2 * (rowb + e) + 1) * wgt[e];
    __syncthreads();
    if (threadIdx.x < R) {
      float L = 0.f;
      for (int sp = 0; sp < P.nsplit; ++sp) L += lw[sp * R + threadIdx.x];
      rowL[threadIdx.x] = L;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < R * (kD / 16); e += blockDim.x) {
      const int r = e / (kD / 16), d0 = (e % (kD / 16)) * 16;
      float acc[16];
#pragma unroll
      for (int d = 0; d < 16; ++d) acc[d] = 0.f;
      // eight splits' loads in flight before they are used
      for (int sp0 = 0; sp0 < P.nsplit; sp0 += 8) {
        float4 v[8][4];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int sp = min(sp0 + u, P.nsplit - 1);
          const float4* src =
              reinterpret_cast<const float4*>(P.part_o + (rowb + sp * R + r) * kD + d0);
#pragma unroll
          for (int d = 0; d < 4; ++d) v[u][d] = __ldcg(src + d);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float wsp = sp0 + u < P.nsplit ? wgt[(sp0 + u) * R + r] : 0.f;
#pragma unroll
          for (int d = 0; d < 4; ++d) {
            acc[4 * d] = fmaf(v[u][d].x, wsp, acc[4 * d]);
            acc[4 * d + 1] = fmaf(v[u][d].y, wsp, acc[4 * d + 1]);
            acc[4 * d + 2] = fmaf(v[u][d].z, wsp, acc[4 * d + 2]);
            acc[4 * d + 3] = fmaf(v[u][d].w, wsp, acc[4 * d + 3]);
          }
        }
      }
      const float L = rowL[r], M = rowM[r];
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const int i = r / G, gi = r % G;
      const size_t orow = ((size_t)b * n_q + i) * g.Hq + hk * G + gi;
      float gsig[16];
      if (g.gate_headwise) {
        const float gs = sigmoidf_(__bfloat162float(P.gate[orow]));
#pragma unroll
        for (int d = 0; d < 16; ++d) gsig[d] = gs;
      } else {
        const uint4* gp = reinterpret_cast<const uint4*>(P.gate + orow * kD + d0);
        const uint4 g0 = gp[0], g1 = gp[1];
        const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int d = 0; d < 8; ++d) {
          gsig[2 * d] = sigmoidf_(__uint_as_float(gw[d] << 16));
          gsig[2 * d + 1] = sigmoidf_(__uint_as_float(gw[d] & 0xffff0000u));
        }
      }
      if (P.out_f32) {
        float4* dst = reinterpret_cast<float4*>(P.out_f32 + orow * kD + d0);
#pragma unroll
        for (int d = 0; d < 16; d += 4)
          dst[d / 4] = make_float4(acc[d] * inv * gsig[d], acc[d + 1] * inv * gsig[d + 1],
                                   acc[d + 2] * inv * gsig[d + 2], acc[d + 3] * inv * gsig[d + 3]);
      } else {
        uint32_t packed[8];
#pragma unroll
        for (int d = 0; d < 16; d += 2)
          packed[d / 2] = pack2(acc[d] * inv * gsig[d], acc[d + 1] * inv * gsig[d + 1]);
        uint4* dst = reinterpret_cast<uint4*>(P.out + orow * kD + d0);
        dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      }
      if (P.lse && d0 == 0) P.lse[orow] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
    if (threadIdx.x == 0) P.counter[(size_t)b * g.Hkv + hk] = 0;
  }
  if (threadIdx.x == 0 && *abort_flag && P.err) atomicExch(P.err, 2);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [batch * cap, Hkv, 128] bf16 cache viewed as 3-D with a (64 dims, 1 head, 64 rows) box.
bool make_cache_map(CUtensorMap* m, const void* ptr, int Hkv, long long rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)Hkv, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)Hkv * kD * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kChunk};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D uint8 map over [rows, Hkv, D] e4m3 codes with a (128, 1, 64) box: one
// 128-byte row per key.
bool make_cache_map_u8(CUtensorMap* m, const void* ptr, int Hkv, long long rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)Hkv, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)kD, (cuuint64_t)Hkv * kD};
  cuuint32_t box[3] = {(cuuint32_t)kD, 1, (cuuint32_t)kChunk};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Whether clusters of `size` CTAs of `kern` (with `smem` bytes of dynamic shared
// memory) can be resident at once; answers are cached per (kernel, size, smem).
bool cluster_fits(const void* kern, int size, int smem) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int>, bool> done;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(kern, size, smem);
  auto it = done.find(key);
  if (it != done.end()) return it->second;
  bool ok = size <= kMaxClusterSplits, refused = false;
  if (ok && size > 8) {
    ok = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    refused = !ok;
  }
  if (ok) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(size, 1, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = size;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t q = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    refused = q != cudaSuccess;
    ok = !refused && n >= 1;
  }
  if (refused) cudaGetLastError();   // a refused query leaves no error behind
  done[key] = ok;
  return ok;
}

}  // namespace

bool attn_decode_fp8_supported(const Geom& g, int n_q) {
  return attn_decode_mma_supported(g, n_q) && g.Hkv <= kMaxHkvFp8 && n_q * g.G <= 16;
}

namespace {
// Row tiles of 16 (query, head) rows the decode kernel holds: n_q * G rows.
int row_tiles(const Geom& g, int n_q) { return n_q * g.G > 16 ? 2 : 1; }
}  // namespace

bool attn_decode_mma_supported(const Geom& g, int n_q) {
  return g.D == kD && g.B % kChunk == 0 && n_q * g.G <= 32 && n_q <= 4;
}

// Chunks per CTA for the split-KV grid: about two CTAs per SM in one wave, and
// at most kMaxClusterSplits CTAs per (sequence, KV head) so that they can form
// one cluster.
void decode_mma_split(const Geom& g, int batch, int n_q, int* nsplit, int* per_split) {
  const int max_chunks = n_q * (g.k + 1) * (g.B / kChunk);
  const int pairs = batch * g.Hkv > 0 ? batch * g.Hkv : 1;
  // two CTAs per SM with one row tile, one with two (larger shared memory)
  int ns = ((row_tiles(g, n_q) == 1 ? 2 : 1) * 148) / pairs;
  if (ns < 1) ns = 1;
  if (ns > kMaxClusterSplits) ns = kMaxClusterSplits;
  if (ns > (max_chunks + 7) / 8) ns = (max_chunks + 7) / 8;   // at least 8 chunks per CTA
  *per_split = (max_chunks + ns - 1) / ns;
  *nsplit = (max_chunks + *per_split - 1) / *per_split;
}

namespace {

// The fused selection's shared-memory layout inside the ring's space (byte
// offsets; the CTA's own score keys first); false when it does not fit.
bool fused_layout(const Geom& g, int n_q, int cap, int nsplit, DecParams* p) {
  auto a16 = [](long long x) { return (x + 15) & ~15LL; };
  const int nblk_cap = cap / g.B;
  const long long per = select_range(nblk_cap, nsplit);
  const long long kpad = (g.k + 3) & ~3;
  long long off = a16(32 + 4LL * n_q * per);   // this CTA's keys
  p->fo_cand = (int)off;
  off += a16(8LL * n_q * kpad);                 // its candidates
  p->fo_gath = (int)off;
  off += a16(8LL * n_q * nsplit * kpad);        // every CTA's candidates
  p->fo_kbar = (int)off;
  off += a16(4LL * kSelRows * (g.di + 4));
  p->fo_iq = (int)off;
  off += a16(4LL * n_q * g.Hi * (g.di + 4));
  p->fo_iw = (int)off;
  off += a16(4LL * n_q * g.Hi);
  p->fo_new = (int)off;
  off += a16(4LL * 2 * g.di);
  p->fo_hist = (int)off;
  off += 4LL * 280 + 8LL * 8 * 32;
  return off <= (long long)kStages * kStageBytes;
}

// The kernel for (fp8, indexer dim, row tiles); kCount: the instantiation that
// adds to the visited-keys debug counter (the others carry no counting code).
template <bool kFp8, bool kCount>
const void* fused_kernel_c(int di, int rt) {
  if constexpr (kFp8) {
    return di == 64 ? reinterpret_cast<const void*>(attn_decode_mma_kernel<true, 64, 1, kCount>)
                    : reinterpret_cast<const void*>(attn_decode_mma_kernel<true, 32, 1, kCount>);
  } else {
    if (rt == 2)
      return di == 64 ? reinterpret_cast<const void*>(attn_decode_mma_kernel<false, 64, 2, kCount>)
                      : reinterpret_cast<const void*>(attn_decode_mma_kernel<false, 32, 2, kCount>);
    return di == 64 ? reinterpret_cast<const void*>(attn_decode_mma_kernel<false, 64, 1, kCount>)
                    : reinterpret_cast<const void*>(attn_decode_mma_kernel<false, 32, 1, kCount>);
  }
}
template <bool kFp8>
const void* fused_kernel(const Geom& g, int rt) {
  return g.keys_visited ? fused_kernel_c<kFp8, true>(g.di, rt) : fused_kernel_c<kFp8, false>(g.di, rt);
}
template <bool kCount>
const void* attend_kernel(bool fp8, int rt) {
  return fp8 ? reinterpret_cast<const void*>(attn_decode_mma_kernel<true, 0, 1, kCount>)
         : rt == 2 ? reinterpret_cast<const void*>(attn_decode_mma_kernel<false, 0, 2, kCount>)
                   : reinterpret_cast<const void*>(attn_decode_mma_kernel<false, 0, 1, kCount>);
}

int decode_smem(const Geom& g, int n_q, int cap) {
  const int words = (cap / g.B + 31) / 32;
  const int bits = row_tiles(g, n_q) == 1 ? DecLayout<1>::kOffBits : DecLayout<2>::kOffBits;
  return bits + 4 * n_q * words + 1024;
}

DecParams base_params(const Geom& g, int n_q, int cap, int nsplit, int per_split,
                      const int* kv_len, const void* q, const void* gate, void* out, float* lse,
                      int* err, Pages pg, Fp8Kv f8) {
  DecParams p = {};
  p.g = g;
  p.n_q = n_q;
  p.cap = cap;
  p.nsplit = nsplit;
  p.per_split = per_split;
  p.kv_len = kv_len;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.err = err;
  p.table = pg.table;
  p.num_pages = pg.num_pages;
  p.k_scale = f8.k_scale;
  p.v_scale = f8.v_scale;
  p.rotated = f8.rotated;
  return p;
}

bool make_maps(const Geom& g, int batch, int cap, const void* kc, const void* vc, Pages pg,
               bool fp8, CUtensorMap* mk, CUtensorMap* mv) {
  const long long rows = pg.table ? (long long)pg.num_pages * g.B : (long long)batch * cap;
  return fp8 ? make_cache_map_u8(mk, kc, g.Hkv, rows) && make_cache_map_u8(mv, vc, g.Hkv, rows)
             : make_cache_map(mk, kc, g.Hkv, rows) && make_cache_map(mv, vc, g.Hkv, rows);
}

cudaError_t launch_decode_kernel(const void* kern, dim3 grid, int smem, int cluster,
                                 cudaStream_t st, const CUtensorMap& mk, const CUtensorMap& mv,
                                 const DecParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster > 0 ? 2 : 1;
  void* args[3] = {const_cast<CUtensorMap*>(&mk), const_cast<CUtensorMap*>(&mv),
                   const_cast<DecParams*>(&p)};
  const cudaError_t e = cudaLaunchKernelExC(&cfg, kern, args);
  note_launch();
  return e;
}

}  // namespace

cudaError_t launch_attn_decode_mma(const Geom& g, int batch, int n_q, int cap, int nsplit,
                                   int per_split, const int* kv_len, const void* q,
                                   const void* kc, const void* vc, const void* gate,
                                   const int* sel, const int* nsel, float* part_ml,
                                   float* part_o, int* counter, void* out, float* lse, int* err,
                                   cudaStream_t st, Pages pg, const int* ready, Fp8Kv f8,
                                   CpShard cp) {
  if (batch == 0) return cudaSuccess;
  CUtensorMap mk, mv;
  if (!make_maps(g, batch, cap, kc, vc, pg, f8.on, &mk, &mv)) return cudaErrorInvalidValue;
  DecParams p = base_params(g, n_q, cap, nsplit, per_split, kv_len, q, gate, out, lse, err, pg, f8);
  p.cp = cp.on ? 1 : 0;
  p.row_off = cp.row_off;
  p.block_lo = cp.block_lo;
  p.out_f32 = cp.out_f32;
  p.sel = sel;
  p.nsel = nsel;
  p.part_ml = part_ml;
  p.part_o = part_o;
  p.counter = counter;
  p.ready = ready;
  const int smem = decode_smem(g, n_q, cap);
  const void* kern = g.keys_visited ? attend_kernel<true>(f8.on, row_tiles(g, n_q))
                                    : attend_kernel<false>(f8.on, row_tiles(g, n_q));
  cudaError_t e = set_max_dynamic_smem(kern, smem);
  if (e != cudaSuccess) return e;
  p.cluster = nsplit > 1 && cluster_fits(kern, nsplit, smem) ? 1 : 0;
  return launch_decode_kernel(kern, dim3(nsplit, batch, g.Hkv), smem, p.cluster ? nsplit : 0, st,
                              mk, mv, p);
}

bool decode_fused_supported(const Geom& g, int n_q, int cap, int nsplit, bool fp8) {
  if (!(fp8 ? attn_decode_fp8_supported(g, n_q) : attn_decode_mma_supported(g, n_q))) return false;
  if (g.di != 32 && g.di != 64) return false;
  if (g.Hi < 1 || g.Hi > 32 || (32 % g.Hi) != 0) return false;
  DecParams p = {};
  if (!fused_layout(g, n_q, cap, nsplit, &p)) return false;
  const void* kern = fp8 ? fused_kernel<true>(g, 1) : fused_kernel<false>(g, row_tiles(g, n_q));
  const int smem = decode_smem(g, n_q, cap);
  if (set_max_dynamic_smem(kern, smem) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return cluster_fits(kern, nsplit, smem);
}

cudaError_t launch_decode_fused(const Geom& g, int batch, int n_q, int cap, int nsplit,
                                int per_split, const int* kv_len, const void* q, const void* kc,
                                const void* vc, const void* gate, const DecodeSelIn& si,
                                void* out, float* lse, int* err, cudaStream_t st, Pages pg,
                                Fp8Kv f8) {
  if (batch == 0) return cudaSuccess;
  CUtensorMap mk, mv;
  if (!make_maps(g, batch, cap, kc, vc, pg, f8.on, &mk, &mv)) return cudaErrorInvalidValue;
  DecParams p = base_params(g, n_q, cap, nsplit, per_split, kv_len, q, gate, out, lse, err, pg, f8);
  if (!fused_layout(g, n_q, cap, nsplit, &p)) return cudaErrorInvalidValue;
  p.cluster = 1;
  p.iq = static_cast<const __nv_bfloat16*>(si.iq);
  p.ik_cache = static_cast<const __nv_bfloat16*>(si.ik_cache);
  p.iw = si.iw;
  p.pooled = si.pooled;
  p.sel_w = si.sel;
  p.nsel_w = si.nsel;
  const int smem = decode_smem(g, n_q, cap);
  const void* kern =
      f8.on ? fused_kernel<true>(g, 1) : fused_kernel<false>(g, row_tiles(g, n_q));
  const cudaError_t e = set_max_dynamic_smem(kern, smem);
  if (e != cudaSuccess) return e;
  return launch_decode_kernel(kern, dim3(nsplit, batch, g.Hkv), smem, nsplit, st, mk, mv, p);
}

}  // namespace qsa
