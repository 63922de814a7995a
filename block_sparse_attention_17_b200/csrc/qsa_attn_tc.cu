// QSA prefill attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA owns two tiles of 128 query rows each. A tile is Qt = 128 / G
// consecutive query tokens of one sequence times the G query heads that share
// one KV head (standard GQA, instagit MTPLX page "Qwen Sparse Attention
// (QSA)"). The CTA walks the UNION of the selected blocks of its 2 * Qt
// queries (selected complete blocks plus tail blocks), gathering each block's
// K and V rows with TMA, and masks per row the blocks that row's query did not
// select and the keys after the query inside its tail block. Rows never see a
// key outside their own selection, so the result is exactly QSA; the cost of
// sharing a tile is MMA work on masked entries.
//
// Warp roles (576 threads):
//   warp 0      TMA producer: Q of both tiles once, then K and V of each
//               128-key step (2 blocks of B = 64 or 1 block of B = 128) into
//               2-deep K and V rings.
//   warp 1      allocates TMEM; one thread issues the MMAs. Per step j and
//               tile t: O_t += P_t(j-1) V(j-1) (A = P from TMEM, V MN-major),
//               then S_t = Q_t K(j)^T (SS, K-major). The two tiles alternate,
//               so the tensor core works on one tile while the other tile's
//               softmax runs.
//   warps 2..9  softmax of tile 0, warps 10..17 softmax of tile 1: two
//               threads share each row (TMEM lane), one per 64-column half;
//               they mask, exchange the partial row max, keep the online
//               softmax in the log2 domain with lazy rescaling (O is rescaled
//               only when the running max grows by more than 2^8), write P as
//               bf16 over S, and in the epilogue apply 1/l and the sigmoid
//               gate (llama.cpp PR #27739 page, QSA block-composition commit text).
// Every wait is bounded; a timeout sets the workspace error word and the CTA
// unwinds (drains its TMA loads and MMAs, frees TMEM).
#include "qsa_common.cuh"
#include "qsa_kernels.h"
#include "qsa_sm100.cuh"

namespace qsa {

using namespace sm100;

namespace {

constexpr int kRows = 128;                  // M per tile
constexpr int kTiles = 2;                   // query tiles per CTA
constexpr int kKeys = 128;                  // N of QK^T, K of PV
constexpr int kHeadDim = 128;               // D
constexpr int kNK = 2, kNV = 2;             // K / V ring depth
constexpr int kChunkBytes = kRows * 128;    // 128 rows x 64 bf16
constexpr int kTileBytes = 2 * kChunkBytes; // 128 rows x 128 bf16
constexpr int kSoftmaxThreads = 256;          // per tile: 128 rows x 2 column halves
constexpr int kThreads = 64 + kTiles * kSoftmaxThreads;
constexpr uint32_t kTmemCols = 512;         // S0 S1 O0 O1, 128 columns each
constexpr float kRescaleThreshold = 8.0f;   // log2 domain
// Of every 8 probability pairs, this many are exponentiated on the FMA pipe
// (exp2_poly2) instead of MUFU, whose 16 results per clock and SM would
// otherwise bound the softmax.
constexpr int kPolyPairsOf8 = 1;

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTiles * kTileBytes;
constexpr int kOffV = kOffK + kNK * kTileBytes;
constexpr int kOffBar = kOffV + kNV * kTileBytes;
constexpr int kNumBars = 1 + 2 * kNK + 2 * kNV + 3 * kTiles + 1 + 4 * kTiles;
constexpr int kOffMisc = kOffBar + 8 * kNumBars;
constexpr int kOffBits = kOffMisc + 64;
constexpr int kMaxWords = kMaxBlocksPerSeq / 32;
constexpr int kOffList = kOffBits + 4 * kMaxWords;
constexpr int kOffXch = kOffList + 2 * kMaxBlocksPerSeq;   // [tile][slot][half][row] floats
constexpr int kSmemBytes = kOffXch + 4 * kTiles * 2 * 2 * kRows + 1024;   // + alignment slack

struct TcParams {
  Geom g;
  const int* cu;
  const uint32_t* bitmask;
  int words;
  int n_ctas;        // CTAs per (sequence, KV head) along the query axis
  int Qt;            // queries per tile
  int total_tokens;
  const __nv_bfloat16* gate;
  __nv_bfloat16* out;
  float* lse;
  int* err;
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int kB>
__global__ void __launch_bounds__(kThreads, 1)
attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const TcParams P) {
  constexpr int kNh = kKeys / kB;   // blocks per 128-key step
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y, hk = blockIdx.z;
  const int cta = P.n_ctas - 1 - static_cast<int>(blockIdx.x);   // longest first
  const int s0 = P.cu[b], L = P.cu[b + 1] - s0;
  const int q0 = cta * kTiles * P.Qt;
  if (q0 >= L) return;
  const int nq = min(kTiles * P.Qt, L - q0);   // valid queries of the CTA
  const int nt = nq > P.Qt ? 2 : 1;            // tiles with at least one valid query
  const Geom& g = P.g;
  const int G = g.G;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kNK;
  uint64_t* v_full = k_empty + kNK;
  uint64_t* v_empty = v_full + kNV;
  uint64_t* s_full = v_empty + kNV;     // [tile]
  uint64_t* p_full = s_full + kTiles;   // [tile]
  uint64_t* o_done = p_full + kTiles;   // [tile]
  uint64_t* mma_done = o_done + kTiles;
  uint64_t* xbar = mma_done + 1;        // [tile][lane quarter]: the row-max exchange of a warp pair
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  int* n_union_s = reinterpret_cast<int*>(smem + kOffMisc + 8);
  uint32_t* ubits = reinterpret_cast<uint32_t*>(smem + kOffBits);
  uint16_t* ulist = reinterpret_cast<uint16_t*>(smem + kOffList);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kNK; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < kNV; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], kSoftmaxThreads);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(mma_done, 1);
    for (int i = 0; i < 4 * kTiles; ++i) mbar_init(&xbar[i], 64);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async();
    // Q does not depend on the selections: start its load now
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    mbar_expect_tx(q_full, kTiles * kTileBytes);
    for (int t = 0; t < kTiles; ++t)
      for (int dc = 0; dc < 2; ++dc)
        tma_load_3d(smem_u32(smem + kOffQ + t * kTileBytes + dc * kChunkBytes), &tmQ, dc * 64,
                    hk * G, s0 + q0 + t * P.Qt, q_full);
  }
  // union of the CTA's selections (selected complete blocks + tail blocks):
  // one selection word per thread, OR-ed into shared memory
  for (int w = threadIdx.x; w < P.words; w += blockDim.x) ubits[w] = 0u;
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  grid_dependency_wait();   // the selection bitmaps come from the selection kernel
  __syncthreads();
  for (int e = threadIdx.x; e < nq * P.words; e += blockDim.x) {
    const uint32_t bits = P.bitmask[(size_t)(s0 + q0) * P.words + e];
    if (bits) atomicOr(&ubits[e % P.words], bits);
  }
  __syncthreads();
  if (warp == 0) {   // ascending list of the union's blocks
    int base = 0;
    for (int w0 = 0; w0 < P.words; w0 += 32) {
      const int w = w0 + lane;
      uint32_t bits = w < P.words ? ubits[w] : 0u;
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
        ulist[off++] = static_cast<uint16_t>(w * 32 + bp);
      }
      base += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) *n_union_s = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_union = *n_union_s;
  const int n_iter = (n_union + kNh - 1) / kNh;

  const uint32_t sQ = sbase + kOffQ;
  const uint32_t sK = sbase + kOffK;
  const uint32_t sV = sbase + kOffV;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      auto issue = [&](const CUtensorMap* tm, uint32_t dst, uint64_t* full, int j) {
        mbar_expect_tx(full, kTileBytes);
#pragma unroll
        for (int h = 0; h < kNh; ++h) {
          const int e = j * kNh + h;
          // a missing second block reads rows past the tensor: TMA fills zeros
          const int tok = e < n_union ? s0 + static_cast<int>(ulist[e]) * kB : P.total_tokens;
#pragma unroll
          for (int dc = 0; dc < 2; ++dc)
            tma_load_3d(dst + dc * kChunkBytes + h * kB * 128, tm, dc * 64, hk, tok, full);
        }
      };
      auto issue_k = [&](int j) -> bool {
        const int s = j % kNK;
        if (j >= kNK && !mbar_wait(&k_empty[s], ((j / kNK) - 1) & 1, abort_flag)) return false;
        issue(&tmK, sK + s * kTileBytes, &k_full[s], j);
        return true;
      };
      auto issue_v = [&](int j) -> bool {
        const int s = j % kNV;
        if (j >= kNV && !mbar_wait(&v_empty[s], ((j / kNV) - 1) & 1, abort_flag)) return false;
        issue(&tmV, sV + s * kTileBytes, &v_full[s], j);
        return true;
      };
      int nk = 0, nv = 0;   // loads issued
      if (n_iter > 0 && issue_k(0)) {
        nk = 1;
        for (int it = 0; it < n_iter; ++it) {
          if (it + 1 < n_iter) {
            if (!issue_k(it + 1)) break;
            nk = it + 2;
          }
          if (!issue_v(it)) break;
          nv = it + 1;
        }
      }
      // drain: no TMA write may still be in flight when the CTA exits
      mbar_wait(q_full, 0, abort_flag);
      for (int j = max(0, nk - kNK); j < nk; ++j)
        mbar_wait(&k_full[j % kNK], (j / kNK) & 1, abort_flag);
      for (int j = max(0, nv - kNV); j < nv; ++j)
        mbar_wait(&v_full[j % kNV], (j / kNV) & 1, abort_flag);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0 && n_iter > 0) {
      constexpr uint32_t idq = idesc_bf16_f32(kRows, kKeys, false, false);
      constexpr uint32_t idv = idesc_bf16_f32(kRows, kHeadDim, false, true);
      // O_t += P_t(j) V(j)
      auto pv = [&](int t, int j) -> bool {
        const int sv = j % kNV;
        if (!mbar_wait(&p_full[t], j & 1, abort_flag)) return false;
        if (t == 0 && !mbar_wait(&v_full[sv], (j / kNV) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vb = sV + sv * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          umma_ts(tmem + 256 + t * 128, tmem + t * 128 + (kk >> 2) * 64 + (kk & 3) * 8,
                  desc_sw128(vb + kk * 2048, kChunkBytes, 1024), idv,
                  (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&o_done[t]);
        if (t == nt - 1) umma_commit(&v_empty[sv]);
        return true;
      };
      // S_t = Q_t K(j)^T
      auto qk = [&](int t, int j) {
        const uint32_t kb = sK + (j % kNK) * kTileBytes;
        const uint32_t qb = sQ + t * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          umma_ss(tmem + t * 128, desc_sw128(qb + off, 16, 1024), desc_sw128(kb + off, 16, 1024),
                  idq, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[t]);
      };
      bool ok = mbar_wait(q_full, 0, abort_flag);
      for (int j = 0; ok && j < n_iter; ++j) {
        ok = mbar_wait(&k_full[j % kNK], (j / kNK) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        for (int t = 0; t < nt; ++t) {
          if (j > 0 && !(ok = pv(t, j - 1))) break;
          qk(t, j);
        }
        umma_commit(&k_empty[j % kNK]);
      }
      for (int t = 0; ok && t < nt; ++t) ok = pv(t, n_iter - 1);
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, abort_flag);
    }
  } else {
    // ------------------------------------------------------------ softmax
    // Tile t has 8 warps: each row (TMEM lane) is shared by two threads, one
    // per 64-column half of S; they exchange their partial row max through
    // shared memory, ordered by an mbarrier of the two warps (bounded waits).
    const int wt = warp - 2;
    const int t = wt >> 3;                    // tile
    const int hf = (wt >> 2) & 1;             // column half
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;        // row within the tile = TMEM lane
    const int qi = t * P.Qt + r / G, gg = r % G;
    const bool valid = qi < nq;
    const int pos = q0 + qi;
    const size_t tok = static_cast<size_t>(s0) + pos;
    const int h = hk * G + gg;
    const uint32_t* mrow = P.bitmask + (valid ? tok : 0) * P.words;
    // the epilogue's gate row: fetch it into L2 now
    if (valid && t < nt && !g.gate_headwise)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(P.gate + (tok * g.Hq + h) * kHeadDim + 64 * hf));
    const uint32_t tS = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + t * 128;
    const uint32_t tO = tS + 256;
    float* xch = reinterpret_cast<float*>(smem + kOffXch);
    auto xslot = [&](int slot, int half) { return xch + ((t * 2 + slot) * 2 + half) * kRows + r; };
    // exchange number e (step j, then n_iter for the final sums) uses data slot
    // e & 1 and phase e of the pair's mbarrier; the wait is bounded, so a warp
    // whose partner gave up does not block
    auto exchange = [&](int e, float x) -> bool {
      *xslot(e & 1, hf) = x;
      mbar_arrive(&xbar[t * 4 + quarter]);
      return __all_sync(kFull, mbar_wait_spin(&xbar[t * 4 + quarter], e & 1, abort_flag));
    };
    const float sc = g.sm_scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = t < nt;
    // the block under this thread's columns at step j, and its selection word
    // (fetched one step ahead of its use)
    auto fetch = [&](int j, uint32_t& w, int& blk) {
      const int e = kB == 64 ? j * 2 + hf : j;
      blk = e < n_union ? static_cast<int>(ulist[e]) : -1;
      w = (valid && blk >= 0) ? __ldg(mrow + (blk >> 5)) : 0u;
    };
    uint32_t wn = 0u;
    int bn = -1;
    unsigned visited = 0;   // debug count of the row's visible keys in these columns
    if (ok) fetch(0, wn, bn);
    for (int j = 0; ok && j < n_iter; ++j) {
      // visible keys among this thread's 64 columns: all of a selected
      // complete block, the keys up to the query in its tail block, or none
      int lim = 0;
      if (bn >= 0 && ((wn >> (bn & 31)) & 1u)) {
        const int col0 = bn * kB + (kB == 128 ? 64 * hf : 0);   // position of column 0
        lim = max(0, min(64, pos + 1 - col0));
      }
      visited += lim;
      if (j + 1 < n_iter) fetch(j + 1, wn, bn);
      const bool any_vis = __any_sync(kFull, lim > 0);
      const bool partial = __any_sync(kFull, lim > 0 && lim < 64);
      if (!__all_sync(kFull, mbar_wait(&s_full[t], j & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float pm = -INFINITY;
      if (any_vis) {   // (warp-uniform: the TMEM loads are warp-collective)
        // the thread's 64 S columns in two halves of 32 (register pressure)
        float cm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          tmem_ld32(tS + 64 * hf + 32 * half, v);
          tmem_wait_ld();
          if (partial) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (32 * half + i >= lim) v[i] = __float_as_uint(-INFINITY);
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            cm[(i >> 1) & 3] =
                fmax3(cm[(i >> 1) & 3], __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
        }
        pm = lim > 0 ? fmax3(cm[0], cm[1], fmaxf(cm[2], cm[3])) : -INFINITY;
      }
      if (!exchange(j, pm)) {
        ok = false;
        break;
      }
      const float mx = fmaxf(pm, *xslot(j & 1, hf ^ 1)) * sc;
      float m_tgt = m_used, alpha = 1.f;
      if (mx > m_used + kRescaleThreshold || (m_used == -INFINITY && mx != -INFINITY)) {
        m_tgt = mx;
        alpha = ex2_approx(m_used - mx);   // 0 when m_used is -inf
      }
      const float ref = m_tgt == -INFINITY ? 0.f : m_tgt;
      // P of this half is packed over the first 32 of its own 64 S columns,
      // so the two halves never touch each other's S
      float2 s2a = make_float2(0.f, 0.f), s2b = make_float2(0.f, 0.f);
      if (!any_vis) {
        uint32_t z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0u;
        tmem_st32(tS + 64 * hf, z);
      } else {
        // rows that do not see these columns subtract +inf: exp2(-inf) = 0
        const float nref = lim > 0 ? -ref : -INFINITY;
        const float2 sc2 = make_float2(sc, sc), nref2 = make_float2(nref, nref);
        // in two halves of 32 columns: half h's P pairs land in packed columns
        // 16 h .. 16 h + 15, whose S was read by half 0 already
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32], pk[16];
          tmem_ld32(tS + 64 * hf + 32 * half, v);
          tmem_wait_ld();
          if (partial) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (32 * half + i >= lim) v[i] = __float_as_uint(-INFINITY);
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 x = ffma2(make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])),
                                   sc2, nref2);
            const float2 pp = ((i >> 1) & 7) < kPolyPairsOf8
                                  ? exp2_poly2(x)
                                  : make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if ((i & 2) == 0) s2a = fadd2(s2a, pp); else s2b = fadd2(s2b, pp);
            pk[i >> 1] = pack_bf16(pp.x, pp.y);
          }
          tmem_st16(tS + 64 * hf + 16 * half, pk);
        }
      }
      l = l * alpha + ((s2a.x + s2a.y) + (s2b.x + s2b.y));
      if (j > 0 && __any_sync(kFull, alpha != 1.f)) {
        if (!__all_sync(kFull, mbar_wait(&o_done[t], (j - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 64 * hf + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + 64 * hf + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
      m_used = m_tgt;
    }
    if (g.keys_visited) add_keys_visited(g.keys_visited, visited);
    // ------------------------------------------------------------ epilogue
    // each thread writes its 64 output dims; l is the sum of both halves
    if (ok && n_iter > 0 &&
        __all_sync(kFull, mbar_wait(&o_done[t], (n_iter - 1) & 1, abort_flag))) {
      tc_fence_after();
      const bool have_l = exchange(n_iter, l);
      const float lt = have_l ? l + *xslot(n_iter & 1, hf ^ 1) : 0.f;
      const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
      __nv_bfloat16* orow = P.out + (tok * g.Hq + h) * kHeadDim;
      const __nv_bfloat16* grow =
          P.gate + (g.gate_headwise ? (tok * g.Hq + h) : (tok * g.Hq + h) * kHeadDim);
      const float gh = (valid && g.gate_headwise) ? sigmoidf_(__bfloat162float(grow[0])) : 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 64 * hf + c * 32, o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int v8 = 0; v8 < 4; ++v8) {
            const int d0 = 64 * hf + c * 32 + v8 * 8;
            float gv[8];
            if (g.gate_headwise) {
#pragma unroll
              for (int i = 0; i < 8; ++i) gv[i] = gh;
            } else {
              const uint4 gu = *reinterpret_cast<const uint4*>(grow + d0);
              const uint32_t gw[4] = {gu.x, gu.y, gu.z, gu.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                gv[2 * i] = sigmoidf_(__uint_as_float(gw[i] << 16));
                gv[2 * i + 1] = sigmoidf_(__uint_as_float(gw[i] & 0xffff0000u));
              }
            }
            uint4 ou;
            ou.x = pack_bf16(__uint_as_float(o[v8 * 8 + 0]) * inv_l * gv[0],
                             __uint_as_float(o[v8 * 8 + 1]) * inv_l * gv[1]);
            ou.y = pack_bf16(__uint_as_float(o[v8 * 8 + 2]) * inv_l * gv[2],
                             __uint_as_float(o[v8 * 8 + 3]) * inv_l * gv[3]);
            ou.z = pack_bf16(__uint_as_float(o[v8 * 8 + 4]) * inv_l * gv[4],
                             __uint_as_float(o[v8 * 8 + 5]) * inv_l * gv[5]);
            ou.w = pack_bf16(__uint_as_float(o[v8 * 8 + 6]) * inv_l * gv[6],
                             __uint_as_float(o[v8 * 8 + 7]) * inv_l * gv[7]);
            *reinterpret_cast<uint4*>(orow + d0) = ou;
          }
        }
      }
      if (valid && hf == 0 && P.lse)
        P.lse[tok * g.Hq + h] = lt > 0.f ? (m_used + log2f(lt)) * kLn2 : -INFINITY;
    }
  }
  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicExch(P.err, 1);
}

// ------------------------------------------------------------ host side
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

// 3-D bf16 map over a [rows, heads, D] tensor with a (64, box_h, box_rows) box.
bool make_map_3d(CUtensorMap* m, const void* ptr, int D, int heads, int rows, int box_h,
                 int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_h, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attn_prefill_tc_supported(const Geom& g) {
  return g.D == kHeadDim && (g.B == 64 || g.B == 128) && g.G >= 1 && (kRows % g.G) == 0;
}

cudaError_t launch_attn_prefill_tc(const Geom& g, const int* cu, int batch, int total_tokens,
                                   int max_seqlen, int words, const uint32_t* bitmask,
                                   const void* q, const void* k, const void* v, const void* gate,
                                   void* out, float* lse, int* err, cudaStream_t st) {
  if (batch == 0 || max_seqlen == 0 || total_tokens == 0) return cudaSuccess;
  const int Qt = kRows / g.G;
  CUtensorMap mq, mk, mv;
  if (!make_map_3d(&mq, q, kHeadDim, g.Hq, total_tokens, g.G, Qt) ||
      !make_map_3d(&mk, k, kHeadDim, g.Hkv, total_tokens, 1, g.B) ||
      !make_map_3d(&mv, v, kHeadDim, g.Hkv, total_tokens, 1, g.B))
    return cudaErrorInvalidValue;
  TcParams p;
  p.g = g;
  p.cu = cu;
  p.bitmask = bitmask;
  p.words = words;
  p.n_ctas = (max_seqlen + kTiles * Qt - 1) / (kTiles * Qt);
  p.Qt = Qt;
  p.total_tokens = total_tokens;
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.err = err;
  dim3 grid(p.n_ctas, batch, g.Hkv);
  cudaError_t e;
  auto kern = g.B == 64 ? attn_prefill_tc_kernel<64> : attn_prefill_tc_kernel<128>;
  e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), kSmemBytes);
  if (e != cudaSuccess) return e;
  e = launch_dependent(kern, grid, dim3(kThreads), kSmemBytes, st, mq, mk, mv, p);
  note_launch();
  return e;
}

}  // namespace qsa
