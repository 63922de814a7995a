// QSA decode attention, split-KV over the selected blocks (sm_100a).
//
// One decode step reads, per (sequence, KV head), only the K/V rows of the
// union of the step's n_q queries' selections (selected complete blocks plus
// tail blocks): the gather consumer of the selection, never a mask over the
// whole cache (ramgpt "Porting Qwen4 to llama.cpp", section "CUDA Optimization
// Should Follow State Correctness"). The step is bound by HBM bandwidth, so
// the kernel is built around streaming: the union is cut into 64-key chunks,
// each CTA takes a contiguous range of chunks of one (sequence, KV head), and
// a producer warp streams each chunk's K and V tiles with TMA through a
// 3-stage ring (two CTAs per SM keep about 190 KB in flight per SM).
//
// The arithmetic per chunk is tiny (at most 16 query rows = n_q x group
// heads), so the four consumer warps use warp-level bf16 MMAs (m16n8k16,
// fp32 accumulation): warp w takes keys [16w, 16w + 16) of each chunk and
// keeps its own online-softmax state (log2 domain); the four states are
// merged at the end and written as one (m, l, O) partial per row; the last
// CTA of each (sequence, KV head) merges the partials by log-sum-exp and
// applies the sigmoid output gate.
#include "qsa_common.cuh"
#include "qsa_kernels.h"
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
constexpr int kOffQ = kOffStages + kStages * kStageBytes;
constexpr int kOffBar = kOffQ + 16 * kQStride;
constexpr int kOffMisc = kOffBar + 8 * 2 * kStages;
constexpr int kOffUnion = kOffMisc + 64;
constexpr int kOffBits = kOffUnion + 8 * kMaxUnion;   // [n_q][cap / B / 32] words
// dynamic shared memory: kOffBits + 4 * n_q * words + 1024 (alignment slack)

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

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 2)
attn_decode_mma_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const DecParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(smem);
  const Geom& g = P.g;
  const int split = blockIdx.x, b = blockIdx.y, hk = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = g.G, n_q = P.n_q, R = n_q * G;
  const int kv = P.kv_len[b];
  const size_t row0 = (((size_t)b * g.Hkv + hk) * P.nsplit + split) * R;
  if (kv < n_q || kv > P.cap) {   // reported by the selection kernel; outputs are zero
    if (split == 0)
      for (int e = threadIdx.x; e < R * kD; e += blockDim.x) {
        const int r = e / kD, d = e - r * kD;
        const size_t orow = ((size_t)b * n_q + r / G) * g.Hq + hk * G + r % G;
        P.out[orow * kD + d] = __float2bfloat16_rn(0.f);
        if (P.lse && d == 0) P.lse[orow] = -INFINITY;
      }
    return;
  }
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc);
  int* n_chunks_s = reinterpret_cast<int*>(smem + kOffMisc + 4);
  int* u_blk = reinterpret_cast<int*>(smem + kOffUnion);
  int* u_qm = u_blk + kMaxUnion;
  const int cpb = g.B / kChunk;   // chunks per block

  // union of the n_q selections (selected blocks and tail blocks), ascending,
  // with a mask of the queries that selected each block: per-query bitmaps in
  // shared memory, then one ordered scan by warp 0
  const int words = (P.cap / g.B + 31) / 32;
  uint32_t* qbits = reinterpret_cast<uint32_t*>(smem + kOffBits);   // [n_q][words]
  for (int e = threadIdx.x; e < n_q * words; e += blockDim.x) qbits[e] = 0u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async();
  }
  // Q rows r = i * G + gi (query i, head hk * G + gi), zero beyond R: Q is an
  // input, so it is loaded before waiting for the selection kernel
  if constexpr (!kFp8) {
    for (int e = threadIdx.x; e < 16 * (kD / 8); e += blockDim.x) {
      const int r = e / (kD / 8), c8 = e % (kD / 8);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < R) {
        const int i = r / G, gi = r % G;
        v = *reinterpret_cast<const uint4*>(
            P.q + (((size_t)b * n_q + i) * g.Hq + hk * G + gi) * kD + c8 * 8);
      }
      *reinterpret_cast<uint4*>(smem + kOffQ + r * kQStride + c8 * 16) = v;
    }
  } else {
    // fp32 rows in the (still unused) fp16 tile area, rotated into the cache's
    // basis (q' = H q) when the cache holds H k, then stored as fp16
    float* qf = reinterpret_cast<float*>(smem + kOffStages + kStages * kF8StageBytes);
    for (int e = threadIdx.x; e < 16 * kD; e += blockDim.x) {
      const int r = e / kD, d = e - r * kD;
      float v = 0.f;
      if (r < R) {
        const int i = r / G, gi = r % G;
        v = __bfloat162float(P.q[(((size_t)b * n_q + i) * g.Hq + hk * G + gi) * kD + d]);
      }
      qf[e] = v;
    }
    __syncthreads();
    if (P.rotated) fwht128_rows(qf, 16, (int)threadIdx.x, (int)blockDim.x, [] { __syncthreads(); });
    for (int e = threadIdx.x; e < 16 * (kD / 8); e += blockDim.x) {
      const int r = e / (kD / 8), c8 = e % (kD / 8);
      const float* src = qf + r * kD + c8 * 8;
      const uint4 v = make_uint4(pack2h(src[0], src[1]), pack2h(src[2], src[3]),
                                 pack2h(src[4], src[5]), pack2h(src[6], src[7]));
      *reinterpret_cast<uint4*>(smem + kOffQ + r * kQStride + c8 * 16) = v;
    }
  }
  // the merging CTA's gate rows: fetch them into L2 now
  if (split == 0 && !g.gate_headwise && threadIdx.x < R * (kD * 2 / 128)) {
    const int r = threadIdx.x / (kD * 2 / 128), part = threadIdx.x % (kD * 2 / 128);
    const size_t orow = ((size_t)b * n_q + r / G) * g.Hq + hk * G + r % G;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(P.gate + orow * kD + part * 64));
  }
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
  if (*abort_flag) {   // nothing issued yet: report and leave (no merge for this pair)
    if (threadIdx.x == 0 && P.err) atomicExch(P.err, 2);
    return;
  }
  {
    const int kp1 = g.k + 1;
    const int nblk = P.cap / g.B;
    for (int e = threadIdx.x; e < n_q * kp1; e += blockDim.x) {
      const int i = e / kp1, j = e - i * kp1;
      if (j < P.nsel[(size_t)b * n_q + i]) {
        const int blk = P.sel[((size_t)b * n_q + i) * kp1 + j];
        if (blk >= 0 && blk < nblk) atomicOr(&qbits[i * words + (blk >> 5)], 1u << (blk & 31));
      }
    }
  }
  __syncthreads();
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
    if (lane == 0) *n_chunks_s = base * cpb;
  }
  __syncthreads();
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
    // Q as A fragments, all 8 k-slices of 16 dims
    uint32_t qa[8][4];
    {
      const int mi = lane >> 3, ri = lane & 7;
      const int row = (mi & 1) * 8 + ri;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int col = kk * 16 + (mi >> 1) * 8;
        ldsm_x4(sbase + kOffQ + row * kQStride + col * 2, qa[kk][0], qa[kk][1], qa[kk][2],
                qa[kk][3]);
      }
    }
    // the two rows this thread holds: gq and gq + 8
    int qrow[2], qpos[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int r = gq + 8 * h2;
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
      uint32_t kt, vt;   // this warp's K and V tiles (64-key bf16 tiles, or 16-key fp16 tiles)
      if constexpr (!kFp8) {
        kt = sbase + kOffStages + s * kStageBytes;
        vt = kt + kTileBytes;
      } else {
        // widen this warp's 16 keys (rows 16w .. 16w + 15 of the chunk) from
        // e4m3 times the row scale into fp16, then release the stage
        const uint32_t st8 = kOffStages + s * kF8StageBytes;
        const float* ks = reinterpret_cast<const float*>(smem + st8 + 2 * kF8BoxBytes);
        const float* vs = reinterpret_cast<const float*>(smem + st8 + 2 * kF8BoxBytes + kF8ScaleBytes);
        const uint32_t tiles = kOffStages + kStages * kF8StageBytes + warp * 2 * kWarpTileBytes;
        kt = sbase + tiles;
        vt = kt + kWarpTileBytes;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int u = lane + 32 * i;
          const int which = u >> 7, rr = (u >> 3) & 15, ch = u & 7;   // K/V, row, 16-dim chunk
          const int row = warp * 16 + rr;                               // row in the chunk
          uint4 out0 = make_uint4(0, 0, 0, 0), out1 = make_uint4(0, 0, 0, 0);
          if (!(which == 1 && row >= lim_all)) {
            const uint4 in = *reinterpret_cast<const uint4*>(
                smem + st8 + which * kF8BoxBytes + row * 128 + ((ch ^ (row & 7)) << 4));
            const float scl = (which ? vs : ks)[row * g.Hkv + hk];
            const uint32_t s2 = pack2h(scl, scl);
            out0 = make_uint4(e4m3x2_scaled(in.x & 0xffffu, s2), e4m3x2_scaled(in.x >> 16, s2),
                              e4m3x2_scaled(in.y & 0xffffu, s2), e4m3x2_scaled(in.y >> 16, s2));
            out1 = make_uint4(e4m3x2_scaled(in.z & 0xffffu, s2), e4m3x2_scaled(in.z >> 16, s2),
                              e4m3x2_scaled(in.w & 0xffffu, s2), e4m3x2_scaled(in.w >> 16, s2));
          }
          uint8_t* dst = smem + tiles + which * kWarpTileBytes;
          *reinterpret_cast<uint4*>(dst + tile16_off(rr, 16 * ch)) = out0;
          *reinterpret_cast<uint4*>(dst + tile16_off(rr, 16 * ch + 8)) = out1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      // visible keys of this chunk per held row: keys key0 + j with j < lim
      int lim[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
        lim[h2] = (qrow[h2] >= 0 && ((qm >> qrow[h2]) & 1))
                      ? max(0, min(kChunk, qpos[h2] + 1 - key0))
                      : 0;
      // S = Q K^T for keys [16w, 16w + 16): two n-tiles of 8 keys
      float sfr[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t b0, b1, b2, b3;
        if constexpr (!kFp8) {
          const int key = warp * 16 + (mi >> 1) * 8 + ri;
          ldsm_x4(kt + tile_off(key, kk * 16 + (mi & 1) * 8), b0, b1, b2, b3);
          mma_bf16(sfr[0], qa[kk], b0, b1);
          mma_bf16(sfr[1], qa[kk], b2, b3);
        } else {
          const int key = (mi >> 1) * 8 + ri;
          ldsm_x4(kt + tile16_off(key, kk * 16 + (mi & 1) * 8), b0, b1, b2, b3);
          mma_f16(sfr[0], qa[kk], b0, b1);
          mma_f16(sfr[1], qa[kk], b2, b3);
        }
      }
      // mask, scale, online softmax (per row across the quad's 4 threads)
      float x[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h2 = e >> 1;
          const int j = warp * 16 + nt * 8 + 2 * tq + (e & 1);
          x[nt][e] = j < lim[h2] ? sfr[nt][e] * sc : -INFINITY;
        }
      float alpha[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        float mx = fmaxf(fmaxf(x[0][2 * h2], x[0][2 * h2 + 1]), fmaxf(x[1][2 * h2], x[1][2 * h2 + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        const float m_new = fmaxf(m[h2], mx);
        const float ref = m_new == -INFINITY ? 0.f : m_new;
        alpha[h2] = ex2_approx(m[h2] - ref);
        m[h2] = m_new;
        float rs = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
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
      if (!kFp8 && lim_all < warp * 16 + 16) {
        for (int e = lane; e < 16 * 16; e += 32) {   // 16 rows x 2 boxes x 8 chunks of 16 B
          const int row = warp * 16 + (e >> 4);
          const int box = (e >> 3) & 1, ch = e & 7;
          if (row >= lim_all)
            *reinterpret_cast<uint4*>(smem + (vt - sbase) + box * kBoxBytes + row * 128 + ch * 16) =
                make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }
      // P as the A fragment of a 16x16 (rows x keys) tile
      uint32_t pa[4];
      if constexpr (!kFp8) {
        pa[0] = pack2(x[0][0], x[0][1]);
        pa[1] = pack2(x[0][2], x[0][3]);
        pa[2] = pack2(x[1][0], x[1][1]);
        pa[3] = pack2(x[1][2], x[1][3]);
      } else {
        pa[0] = pack2h(x[0][0], x[0][1]);
        pa[1] = pack2h(x[0][2], x[0][3]);
        pa[2] = pack2h(x[1][0], x[1][1]);
        pa[3] = pack2h(x[1][2], x[1][3]);
      }
      // O += P V over the warp's 16 keys, 16 n-tiles of 8 dims
#pragma unroll
      for (int dn = 0; dn < 16; dn += 2) {
        uint32_t b0, b1, b2, b3;
        if constexpr (!kFp8) {
          const int key = warp * 16 + (mi & 1) * 8 + ri;
          ldsm_x4_t(vt + tile_off(key, dn * 8 + (mi >> 1) * 8), b0, b1, b2, b3);
          mma_bf16(o[dn], pa, b0, b1);
          mma_bf16(o[dn + 1], pa, b2, b3);
        } else {
          const int key = (mi & 1) * 8 + ri;
          ldsm_x4_t(vt + tile16_off(key, dn * 8 + (mi >> 1) * 8), b0, b1, b2, b3);
          mma_f16(o[dn], pa, b0, b1);
          mma_f16(o[dn + 1], pa, b2, b3);
        }
      }
      __syncwarp();
      if (!kFp8 && lane == 0) mbar_arrive(&empty[s]);
    }
    // merge the four warps' states through shared memory (the ring is free)
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
    // thread t of the 128 consumers: row t / 8, dims [16 (t % 8), + 16)
    const int t = threadIdx.x;
    const int r = t >> 3, d0 = (t & 7) * 16;
    // a rotated fp8 cache gives O' = H O: the merged rows are rotated back
    // (H is symmetric and orthonormal) before they leave as the partial
    float* urow = sm + kConsumers * 16 * 2;                    // [16 rows][128]
    const bool unrotate = kFp8 && P.rotated;
    if (r < R) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, sm[(w * 16 + r) * 2]);
      float wsc[kConsumers], L = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) {
        const float mw = sm[(w * 16 + r) * 2];
        wsc[w] = mw == -INFINITY ? 0.f : ex2_approx(mw - M);
        L += sm[(w * 16 + r) * 2 + 1] * wsc[w];
      }
      float* dst = unrotate ? urow + r * kD + d0 : P.part_o + (row0 + r) * kD + d0;
#pragma unroll
      for (int d = 0; d < 16; d += 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) {
          const float4 v = *reinterpret_cast<const float4*>(so + (w * 16 + r) * kD + d0 + d);
          acc.x += v.x * wsc[w];
          acc.y += v.y * wsc[w];
          acc.z += v.z * wsc[w];
          acc.w += v.w * wsc[w];
        }
        *reinterpret_cast<float4*>(dst + d) = acc;
      }
      if ((t & 7) == 0) {
        P.part_ml[2 * (row0 + r)] = M;
        P.part_ml[2 * (row0 + r) + 1] = L;
      }
    }
    if (unrotate) {
      named_bar_sync(1, 32 * kConsumers);
      fwht128_rows(urow, R, t, 32 * kConsumers, [] { named_bar_sync(1, 32 * kConsumers); });
      if (r < R) {
        float* gdst = P.part_o + (row0 + r) * kD + d0;
#pragma unroll
        for (int d = 0; d < 16; d += 4)
          *reinterpret_cast<float4*>(gdst + d) = *reinterpret_cast<const float4*>(urow + r * kD + d0 + d);
      }
    }
  }
  // the last CTA of this (sequence, KV head) merges the splits' partials by
  // log-sum-exp and applies the sigmoid output gate
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
    float* rowL = rowM + 16;                                     // [R]
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
    float* lw = rowL + 16;                                        // [nsplit][R]
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
      uint32_t packed[8];
#pragma unroll
      for (int d = 0; d < 16; d += 2)
        packed[d / 2] = pack2(acc[d] * inv * gsig[d], acc[d + 1] * inv * gsig[d + 1]);
      uint4* dst = reinterpret_cast<uint4*>(P.out + orow * kD + d0);
      dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
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

}  // namespace

bool attn_decode_fp8_supported(const Geom& g, int n_q) {
  return attn_decode_mma_supported(g, n_q) && g.Hkv <= kMaxHkvFp8;
}

bool attn_decode_mma_supported(const Geom& g, int n_q) {
  return g.D == kD && g.B % kChunk == 0 && n_q * g.G <= 16 && n_q <= 4;
}

// Chunks per CTA for the split-KV grid: about two CTAs per SM in one wave.
void decode_mma_split(const Geom& g, int batch, int n_q, int* nsplit, int* per_split) {
  const int max_chunks = n_q * (g.k + 1) * (g.B / kChunk);
  const int pairs = batch * g.Hkv > 0 ? batch * g.Hkv : 1;
  int ns = (2 * 148) / pairs;
  if (ns < 1) ns = 1;
  if (ns > (max_chunks + 7) / 8) ns = (max_chunks + 7) / 8;   // at least 8 chunks per CTA
  *per_split = (max_chunks + ns - 1) / ns;
  *nsplit = (max_chunks + *per_split - 1) / *per_split;
}

cudaError_t launch_attn_decode_mma(const Geom& g, int batch, int n_q, int cap, int nsplit,
                                   int per_split, const int* kv_len, const void* q,
                                   const void* kc, const void* vc, const void* gate,
                                   const int* sel, const int* nsel, float* part_ml,
                                   float* part_o, int* counter, void* out, float* lse, int* err,
                                   cudaStream_t st, Pages pg, const int* ready, Fp8Kv f8) {
  if (batch == 0) return cudaSuccess;
  CUtensorMap mk, mv;
  const long long rows = pg.table ? (long long)pg.num_pages * g.B : (long long)batch * cap;
  const bool ok = f8.on ? make_cache_map_u8(&mk, kc, g.Hkv, rows) && make_cache_map_u8(&mv, vc, g.Hkv, rows)
                        : make_cache_map(&mk, kc, g.Hkv, rows) && make_cache_map(&mv, vc, g.Hkv, rows);
  if (!ok) return cudaErrorInvalidValue;
  DecParams p;
  p.g = g;
  p.n_q = n_q;
  p.cap = cap;
  p.nsplit = nsplit;
  p.per_split = per_split;
  p.kv_len = kv_len;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.counter = counter;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.sel = sel;
  p.nsel = nsel;
  p.part_ml = part_ml;
  p.part_o = part_o;
  p.err = err;
  p.table = pg.table;
  p.ready = ready;
  p.k_scale = f8.k_scale;
  p.v_scale = f8.v_scale;
  p.rotated = f8.rotated;
  const int words = (cap / g.B + 31) / 32;
  const int smem = kOffBits + 4 * n_q * words + 1024;
  auto kern = f8.on ? attn_decode_mma_kernel<true> : attn_decode_mma_kernel<false>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  e = launch_dependent(kern, dim3(nsplit, batch, g.Hkv), dim3(kThreads), smem, st, mk, mv, p);
  note_launch();
  return e;
}

}  // namespace qsa
