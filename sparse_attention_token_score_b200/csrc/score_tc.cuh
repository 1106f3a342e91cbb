// Lightning-indexer scoring on the 5th-generation tensor cores (tcgen05).
//
// Score (DeepSeek Sparse Attention lightning indexer; "MISA: Mixture of
// Indexer Sparse Attention for Long-Context LLM Inference", section "Problem
// statement"; signed head weights: "DoSA: Dots Sparse Attention", section 3):
//     I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:])
// FP8 inputs carry a per-token key scale and a per-(query, head) scale, and
// since ReLU(a*x) = a*ReLU(x) for a > 0 the kernel computes
//     I[t,s] = ks[s] * sum_h (w[t,h] * qs[t,h]) * ReLU(q8[t,h,:] . k8[s,:]).
//
// One persistent CTA per SM, warp-specialised:
//   producer warp(s) -> shared-memory ring of key tiles (TMA, or cp.async
//                       gathers of arbitrary key rows by four warps with
//                       asynchronous completion), plus the stationary query
//                       tile of the current query group (TMA; one or two
//                       buffers)
//   MMA warp         -> one thread issues tcgen05.mma into a ring of TMEM
//                       accumulators (as many as fit in 512 columns, <= 8)
//   8 epilogue warps -> tcgen05.ld, ReLU, head-weighted sum (head weights of
//                       the query group staged in shared memory), causal
//                       mask, fp32 store. The [T, H, L] head logits never
//                       leave TMEM.
//
// Orientation (score modes): keys on the MMA M dimension (128 TMEM lanes, one
// key per epilogue thread), QPT queries x H heads on N, so each thread reduces
// over heads inside its own registers. Router mode swaps the roles: QPT*H =
// 128 (query, head) rows on M, 256 pooled keys on N, and each thread reduces
// ReLU over the pooled keys (MISA page, section "Methodology", step 1).
//
// Work split: the (query group, key tile) pairs of the whole launch are
// flattened and every CTA takes one contiguous range, so causal imbalance
// between groups evens out; the query tile is reloaded only when the group
// changes. Router mode assigns whole groups round-robin (its per-row sums
// must not be split across CTAs).
#pragma once
#include "common.cuh"


namespace dsa {

#ifndef DSA_NACC_MAX
#define DSA_NACC_MAX 8
#endif


enum class ScoreMode : int { kTma = 0, kGather = 1, kRouter = 2 };

struct ScoreParams {
  int batch;            // independent sequences
  int T;                // queries per sequence
  int Lk;               // key rows per sequence (tokens, or pooled blocks)
  int L_tok;            // gather mode: tokens per sequence (rows of kg per sequence)
  long long q_offset;   // absolute position of query 0
  int pstride;          // key row s sits at position s * pstride (1 = tokens, B = blocks)
  const float* w;       // [batch*T, H] signed head weights
  const float* q_scale; // [batch*T, H] (FP8) or nullptr
  const float* k_scale; // [batch*Lk]   (FP8) or nullptr
  float* out;           // score: [batch*T, ldo]; router: 2 x [batch*T*H] partial sums
  long long ldo;
  const void* kg;           // gather mode: keys [batch*L_tok, D] (bf16 or e4m3)
  const int* cand;          // gather mode: [batch*T, n_slots] block / token ids, -1 = none
  int n_slots, blk, n_compact;  // compact position c -> cand[c / blk] * blk + c % blk
  int blk_tma;              // gather mode, blk % 128 == 0: a tile is one contiguous key run (TMA)
  unsigned* err;            // device error word
  // Optional compaction (score mode, ScoreCfg CMP): every visible score >=
  // cthr[row] is appended, with its key, to the row's candidate list
  // (cval / cidx [rows, ccap]). Each epilogue warp reserves slots CCHUNK at a
  // time (cres[row] counts reserved slots, requested one chunk ahead) and
  // fills the unused rest of its chunks with sentinels (-inf, -1) when it
  // leaves the group; creal[row] counts the real entries. Slots past ccap are
  // not written (cres then exceeds ccap). out may be null: no full scores.
  const float* cthr;
  float* cval;
  int* cidx;
  int* cres;
  int* creal;
  int ccap;
  // Optional work list (score mode): only the (query group, key tile) pairs
  // pairs[0 .. *pairs_n) are computed (groups counted over all sequences;
  // each group's tiles contiguous and ascending), split evenly over the CTAs.
  const int2* pairs;
  const int* pairs_n;

  // DoSA bound pass (ScoreCfg kEpiBound): the score computed is the bound's
  // augmented-head part; adding cbound[row] * knorm[key] gives the bound, and
  // a key tile becomes live for the refinement pass's query group
  // (live_qpt queries per group, live_gpb groups per sequence) when a visible
  // key of the tile has bound >= cthr[row]: live_out[group * live_ld + tile] = 1.
  const float* knorm;
  const float* cbound;
  uint8_t* live_out;
  long long live_ld;
  int live_qpt, live_gpb;
};

constexpr int CCHUNK = 64;  // candidate slots reserved per warp and query at a time

// Epilogue variants of the score mode: full scores (kEpiStore), candidate
// lists (kEpiCand), DoSA bounds -> live key tiles (kEpiBound).
enum : int { kEpiStore = 0, kEpiCand = 1, kEpiBound = 2 };

template <int ELEM_, int D_, int H_, int QPT_, ScoreMode MODE_, int NSTAGE_, int EPIW_ = 8, int NQBUF_ = 1,
          int EPI_ = kEpiStore, bool LIST_ = false, int CTAS_ = 1>
struct ScoreCfg {
  static constexpr int ELEM = ELEM_;  // bytes per element: 2 = bf16, 1 = e4m3
  static constexpr int D = D_, H = H_, QPT = QPT_, NSTAGE = NSTAGE_;
  static constexpr ScoreMode MODE = MODE_;
  static constexpr bool ROUTER = MODE_ == ScoreMode::kRouter;
  static constexpr bool GATHER = MODE_ == ScoreMode::kGather;
  // candidate compaction in the epilogue (ScoreParams::cres and friends) or
  // DoSA bounds (ScoreParams::knorm and friends)
  static constexpr bool CMP = EPI_ == kEpiCand;
  static constexpr bool BND = EPI_ == kEpiBound;
  static_assert(EPI_ == kEpiStore || (MODE_ == ScoreMode::kTma && QPT_ > 1),
                "epilogue variants: score mode, several queries per group");
  // work-list mode (ScoreParams::pairs): only listed (group, tile) pairs
  static constexpr bool LIST = LIST_;
  static_assert(!LIST || MODE_ == ScoreMode::kTma, "work lists: score mode");
  static constexpr int ROW_BYTES = D * ELEM;
  static_assert(ROW_BYTES == 128 || ROW_BYTES == 256, "rows must be 1 or 2 swizzle atoms wide");
  static constexpr int KBLK = ROW_BYTES / 128;          // 128-byte column blocks per row
  static constexpr int QROWS = QPT * H;                 // stationary query tile rows
  static constexpr int KROWS = ROUTER ? 256 : 128;      // streaming key tile rows
  static constexpr int MMA_N = ROUTER ? KROWS : QROWS;
  static_assert(ROUTER ? QROWS == 128 : (QROWS % 16 == 0 && QROWS >= 32 && QROWS <= 256),
                "bad tile shape");
  static_assert(!GATHER || (QPT == 1 && D == 128), "gather mode: one query per group, d = 128");
  // Gathers: the producer warps take tiles round robin. Stage s is refilled
  // for tile i only after the MMAs of tile i - NSTAGE are done, and the MMA
  // thread consumes tiles in order, so with NSTAGE >= NPROD a warp's wait on
  // a stage is never more than one phase behind and the arrivals of two
  // tiles never meet on one phase.
  static constexpr int NPROD = GATHER ? 4 : 1;          // producer warps
  static_assert(NSTAGE >= NPROD, "stages per producer warp");
  static constexpr int Q_BYTES = QROWS * ROW_BYTES;
  static constexpr int K_BYTES = KROWS * ROW_BYTES;
  static constexpr int NKSTEP = ROW_BYTES / 32;         // one MMA consumes 32 bytes of K
  // TMEM accumulators: as many MMA_N-column buffers as fit in the 512
  // columns (at most DSA_NACC_MAX). Narrow tiles (one query per group) carry
  // little MMA work each, so with two buffers the MMA -> epilogue -> MMA
  // round trip would set the pace; more buffers let the MMAs run ahead.
  // CTAs per SM: 1, or 2 for streams that want more loads in flight than one
  // CTA's shared memory holds (each then owns half of TMEM and of the SM's
  // registers, and its epilogue keeps one TMEM chunk in flight per warp)
  static constexpr int CTAS = CTAS_;
  static_assert(CTAS == 1 || (CTAS == 2 && !ROUTER), "CTAs per SM");
  static constexpr int NACC = ((512 / CTAS) / MMA_N < DSA_NACC_MAX) ? (512 / CTAS) / MMA_N : DSA_NACC_MAX;
  static_assert(NACC >= 2 && (NACC & (NACC - 1)) == 0, "accumulator buffers");
  static constexpr int TMEM_COLS = (NACC * MMA_N <= 32) ? 32 : (NACC * MMA_N <= 64) ? 64
                                 : (NACC * MMA_N <= 128) ? 128 : (NACC * MMA_N <= 256) ? 256 : 512;
  static constexpr int MMA_WARP = NPROD;
  static constexpr int EPI_WARP0 = NPROD + 1;
  // Epilogue warps: EPIW = 4 * NSETS; each set of 4 warps covers the 128
  // TMEM lanes. Sets take tiles round robin (router and one-query groups),
  // or split the queries of every tile between them.
  static constexpr int EPIW = EPIW_;
  static constexpr int NSETS = EPIW / 4;
  static constexpr bool SPLIT_TILES = ROUTER || QPT == 1;
  static_assert(EPIW == 8 || (EPIW == 16 && !ROUTER && (SPLIT_TILES || QPT % 4 == 0)), "epilogue warps");
  static constexpr int NTHREADS = (EPI_WARP0 + EPIW) * 32;
  static constexpr int TEMPTY_ARRIVALS = SPLIT_TILES ? 4 : EPIW;
  static constexpr uint32_t IDESC = umma_idesc(ELEM == 2 ? 1u : 0u, 128, MMA_N);
  // shared memory layout (offsets from a 1024-aligned base). NQBUF query-tile
  // buffers: with two, the next group's tile loads while the current group's
  // keys still stream (pays off where groups are short, e.g. token gathers).
  static constexpr int NQBUF = NQBUF_;
  static_assert(NQBUF == 1 || NQBUF == 2, "query buffers");
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = NQBUF * Q_BYTES;
  // FP8: the epilogue applies per-key dequant scales (loaded from global
  // memory by the thread that owns the key, ahead of the tile's MMAs; for
  // gathers, by the key's token). The router weights its pooled-key columns
  // by their scales instead.
  static constexpr bool KEY_SCALES = ELEM == 1 && !ROUTER;
  // the plain store epilogue (bf16, eight warps, one CTA per SM) has a loop of its own
  static constexpr bool PLAIN = EPI_ == kEpiStore && !LIST_ && ELEM == 2 && !ROUTER && !GATHER && EPIW == 8 &&
                                CTAS_ == 1 && !SPLIT_TILES;
  // the other bf16 store kernels (16 epilogue warps) likewise: 0.585 -> 0.561 ms
  // on the routed MISA pass; FP8 stays on the shared loop (1.41 against 1.46 ms
  // with its own on the FP8 DSA chunk)
  static constexpr bool PLAIN2 = EPI_ == kEpiStore && !LIST_ && ELEM == 2 && !ROUTER && !GATHER && !PLAIN;
  // per epilogue warp: the head weights (x query scales) of its columns for
  // the current query group, refilled when the group changes
  static constexpr int NCOL_THREAD = ROUTER ? 0 : (SPLIT_TILES ? QROWS : QROWS / NSETS);
  // DoSA bounds: (threshold, norm coefficient) of each query of the warp's
  // set, staged with the head weights
  static constexpr int NBND_THREAD = (EPI_ == 2) ? 2 * (QPT_ / NSETS) : 0;
  static constexpr int SMEM_COEF = SMEM_K + NSTAGE * K_BYTES;
  static constexpr int SMEM_BAR = SMEM_COEF + EPIW * (NCOL_THREAD + NBND_THREAD) * 4;
  static constexpr int NBAR = 2 * NSTAGE + 2 * NQBUF + 2 * NACC + 1;
  static constexpr int SMEM_USED = SMEM_BAR + NBAR * 8 + 16;
  // Pad to more than half an SM so two CTAs never share an SM's TMEM.
  static constexpr int SMEM_BYTES = CTAS == 2 ? SMEM_USED + 1024
                                   : ((SMEM_USED + 1024 < 120 * 1024) ? 120 * 1024 : SMEM_USED + 1024);
  static_assert(SMEM_BYTES <= (CTAS == 2 ? 112 * 1024 : 227 * 1024), "shared memory");
};

// Iterates this CTA's (group, tile) pairs. Every thread runs its own copy;
// all copies visit the same sequence.
template <class C>
struct TileSched {
  int gpb, G;
  int g, j, nt;
  int b, tg;        // sequence and query group within it (kept incrementally)
  long long left;   // tiles left (flat split)
  bool first, last, done;

  // key tiles of query group tg (the same for every sequence)
  __device__ __forceinline__ int ntile_tg(const ScoreParams& p, int tgi) const {
    if (C::GATHER) return (p.n_compact + C::KROWS - 1) / C::KROWS;
    const int t_last = min(p.T, (tgi + 1) * C::QPT) - 1;
    const long long pos = p.q_offset + t_last;
    long long nk;
    if (p.pstride == 1) nk = pos + 1;
    else if (pos < 0x7fffffffLL) nk = static_cast<unsigned>(pos) / static_cast<unsigned>(p.pstride) + 1;
    else nk = pos / p.pstride + 1;
    if (nk > p.Lk) nk = p.Lk;
    return static_cast<int>((nk + C::KROWS - 1) / C::KROWS);
  }
  __device__ __forceinline__ int ntile(const ScoreParams& p, int grp) const {
    return ntile_tg(p, grp % gpb);
  }

  // pair-list mode: position li of the list (left pairs to go, this included)
  int li;

  __device__ __forceinline__ void load_pair(const ScoreParams& p, bool at_start) {
    const int2 e = __ldg(p.pairs + li);
    g = e.x;
    j = e.y;
    b = g / gpb;
    tg = g - b * gpb;
    first = at_start || __ldg(&p.pairs[li - 1].x) != g;
    last = left == 1 || __ldg(&p.pairs[li + 1].x) != g;
  }

  // All 32 lanes of the warp call init together (warp-cooperative scans).
  __device__ __forceinline__ void init(const ScoreParams& p) {
    gpb = (p.T + C::QPT - 1) / C::QPT;
    G = p.batch * gpb;
    done = false;
    const int lane = threadIdx.x & 31;
    if constexpr (C::LIST) {
      const long long W = __ldg(p.pairs_n);
      const long long i0 = W * blockIdx.x / gridDim.x;
      left = W * (blockIdx.x + 1) / gridDim.x - i0;
      li = static_cast<int>(i0);
      if (left <= 0) { done = true; return; }
      load_pair(p, true);
      return;
    }
    if (C::ROUTER) {
      left = 0;
      g = blockIdx.x;
      while (g < G && (nt = ntile(p, g)) == 0) g += gridDim.x;
      if (g >= G) { done = true; return; }
      j = 0;
    } else {
      // total tiles: lane l sums groups l, l+32, ...
      long long W = 0;
      for (int q = lane; q < G; q += 32) W += ntile(p, q);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
      const long long b0 = W * blockIdx.x / gridDim.x;
      const long long b1 = W * (blockIdx.x + 1) / gridDim.x;
      left = b1 - b0;
      if (left <= 0) { done = true; return; }
      // first group whose tiles reach past b0: scan 32 groups at a time
      long long acc = 0;
      for (int base = 0;; base += 32) {
        const int q = base + lane;
        const long long nq = q < G ? ntile(p, q) : 0;
        long long inc = nq;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const long long y = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += y;
        }
        const long long tot = __shfl_sync(0xffffffffu, inc, 31);
        if (acc + tot > b0) {
          const uint32_t m = __ballot_sync(0xffffffffu, acc + inc > b0);
          const int src = __ffs(m) - 1;
          const long long inc_s = __shfl_sync(0xffffffffu, inc, src);
          const long long nq_s = __shfl_sync(0xffffffffu, nq, src);
          g = base + src;
          j = static_cast<int>(b0 - (acc + inc_s - nq_s));
          nt = static_cast<int>(nq_s);
          break;
        }
        acc += tot;
      }
    }
    b = g / gpb;
    tg = g - b * gpb;
    first = true;
    last = (j == nt - 1) || (!C::ROUTER && left == 1);
  }

  __device__ __forceinline__ void next(const ScoreParams& p) {
    if constexpr (C::LIST) {
      if (--left == 0) { done = true; return; }
      ++li;
      load_pair(p, false);
      return;
    }
    if (C::ROUTER) {
      if (++j == nt) {
        g += gridDim.x;
        while (g < G && (nt = ntile(p, g)) == 0) g += gridDim.x;
        if (g >= G) { done = true; return; }
        b = g / gpb;
        tg = g - b * gpb;
        j = 0;
        first = true;
      } else {
        first = false;
      }
      last = (j == nt - 1);
    } else {
      if (--left == 0) { done = true; return; }
      if (++j == nt) {
        do {
          ++g;
          if (++tg == gpb) { tg = 0; ++b; }
          nt = ntile_tg(p, tg);
        } while (nt == 0);
        j = 0;
        first = true;
      } else {
        first = false;
      }
      last = (j == nt - 1) || (left == 1);
    }
  }
};

// Token behind compact position c of gathered row r; -1 if there is none or it
// is not visible to the query (position q_pos).
__device__ __forceinline__ long long gathered_token(const ScoreParams& p, long long r, int c,
                                                    long long q_pos) {
  if (c >= p.n_compact) return -1;
  const int slot = c / p.blk;
  const int cb = __ldg(p.cand + r * p.n_slots + slot);
  if (cb < 0) return -1;
  const long long tok = static_cast<long long>(cb) * p.blk + (c - slot * p.blk);
  if (tok >= p.L_tok || tok > q_pos) return -1;
  return tok;
}

// Work list for the score kernel's pair-list mode: the (group, tile) pairs
// whose flag is set (flags[g * ld + j]), each group's tiles ascending and
// contiguous, j below the group's visible tile count (queries of a group are
// qpt consecutive ones; tiles of 128 keys). One warp per group; the group's
// run is placed with one atomic, so groups come in no particular order.
__global__ void pairs_build_kernel(const uint8_t* __restrict__ flags, long long ld, int groups, int gpb, int T,
                                   int qpt, long long q_offset, int L, int2* __restrict__ pairs,
                                   int* __restrict__ count) {
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (g >= groups) return;
  const int tg = g % gpb;
  const long long t_last = min(T, (tg + 1) * qpt) - 1;
  const long long nk = min(q_offset + t_last + 1, static_cast<long long>(L));
  const int nt = static_cast<int>((nk + 127) / 128);
  const uint8_t* f = flags + static_cast<long long>(g) * ld;
  int cnt = 0;
  for (int j0 = 0; j0 < nt; j0 += 32) {
    const int j = j0 + lane;
    cnt += __popc(__ballot_sync(0xffffffffu, j < nt && f[j] != 0));
  }
  if (cnt == 0) return;
  int base = 0;
  if (lane == 0) base = atomicAdd(count, cnt);
  base = __shfl_sync(0xffffffffu, base, 0);
  for (int j0 = 0; j0 < nt; j0 += 32) {
    const int j = j0 + lane;
    const bool on = j < nt && f[j] != 0;
    const uint32_t m = __ballot_sync(0xffffffffu, on);
    if (on) pairs[base + __popc(m & ((1u << lane) - 1u))] = make_int2(g, j);
    base += __popc(m);
  }
}

template <class C>
__global__ void __launch_bounds__(C::NTHREADS, C::CTAS)
score_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const ScoreParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base + C::SMEM_Q;
  const uint32_t s_k = s_base + C::SMEM_K;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  auto full = [&](int i) { return smem_u32(&bars[i]); };
  auto empty = [&](int i) { return smem_u32(&bars[C::NSTAGE + i]); };
  auto qfull = [&](int i) { return smem_u32(&bars[2 * C::NSTAGE + i]); };
  auto qempty = [&](int i) { return smem_u32(&bars[2 * C::NSTAGE + C::NQBUF + i]); };
  constexpr int TB = 2 * C::NSTAGE + 2 * C::NQBUF;
  auto tfull = [&](int b) { return smem_u32(&bars[TB + b]); };
  auto tempty = [&](int b) { return smem_u32(&bars[TB + C::NACC + b]); };
  const uint32_t mdone = smem_u32(&bars[TB + 2 * C::NACC]);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(full(i), (C::GATHER && !p.blk_tma) ? 32 : 1);
      mbar_init(empty(i), 1);  // a stage is free once its MMAs are done
    }
    for (int i = 0; i < C::NQBUF; ++i) {
      mbar_init(qfull(i), 1);
      mbar_init(qempty(i), 1);
    }
    for (int b = 0; b < C::NACC; ++b) {
      mbar_init(tfull(b), 1);
      mbar_init(tempty(b), C::TEMPTY_ARRIVALS);
    }
    mbar_init(mdone, 1);
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 32 * C::MMA_WARP + 1) {
    tma_prefetch_desc(&tm_q);
    if (!C::GATHER || p.blk_tma) tma_prefetch_desc(&tm_k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  TileSched<C> s;
  s.init(p);

  if (warp < C::NPROD) {
    // ------------------------------------------------------------ producer
    const int pw = warp;
    uint32_t it = 0, gq = 0;
    bool ok = true;
    for (; !s.done; s.next(p)) {
      const int b = s.b;
      const int tg = s.tg;
      // gathers: tiles round-robin over the producer warps (each owns its
      // stages); contiguous block tiles (TMA): warp 0 loads every tile
      const bool mine = C::GATHER ? (p.blk_tma ? pw == 0 : static_cast<int>(it % C::NPROD) == pw) : true;
      if (s.first) {
        // The query tile is always loaded by warp 0, group by group in order.
        if (pw == 0 && lane == 0) {
          const int qb = static_cast<int>(gq % C::NQBUF);
          if (!mbar_wait(qempty(qb), ((gq / C::NQBUF) & 1u) ^ 1u, p.err)) { ok = false; }
          else {
            mbar_arrive_expect_tx(qfull(qb), C::Q_BYTES);
            const int row0 = (b * p.T + tg * C::QPT) * C::H;
#pragma unroll
            for (int kb = 0; kb < C::KBLK; ++kb)
              tma_load_2d(s_q + qb * C::Q_BYTES + kb * C::QROWS * 128, &tm_q, qfull(qb),
                          kb * (128 / C::ELEM), row0);
          }
        }
        ++gq;
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      if (!mine) { ++it; continue; }
      const int stage = static_cast<int>(it % C::NSTAGE);
      const uint32_t ph = (it / C::NSTAGE) & 1u;
      if (C::GATHER && p.blk_tma) {
        // the tile's 128 compact positions are tokens cand[slot] * blk + [c0 % blk, +128)
        if (lane == 0) {
          if (!mbar_wait(empty(stage), ph ^ 1u, p.err)) { ok = false; }
          else {
            const long long r = static_cast<long long>(b) * p.T + tg;
            const int c0 = s.j * C::KROWS;
            const int slot = c0 / p.blk;
            const int cb = c0 < p.n_compact ? __ldg(p.cand + r * p.n_slots + slot) : -1;
            if (cb >= 0) {
              const long long tok0 = static_cast<long long>(cb) * p.blk + (c0 - slot * p.blk);
              mbar_arrive_expect_tx(full(stage), C::K_BYTES);
#pragma unroll
              for (int kb = 0; kb < C::KBLK; ++kb)
                tma_load_2d(s_k + stage * C::K_BYTES + kb * C::KROWS * 128, &tm_k, full(stage),
                            kb * (128 / C::ELEM), static_cast<int>(b * p.L_tok + tok0));
            } else {
              mbar_arrive(full(stage));  // no keys: the epilogue writes -inf for the whole tile
            }
          }
        }
      } else if (!C::GATHER) {
        if (lane == 0) {
          if (!mbar_wait(empty(stage), ph ^ 1u, p.err)) { ok = false; }
          else {
            const int krow0 = b * p.Lk + s.j * C::KROWS;
            mbar_arrive_expect_tx(full(stage), C::K_BYTES);
#pragma unroll
            for (int kb = 0; kb < C::KBLK; ++kb)
              tma_load_2d(s_k + stage * C::K_BYTES + kb * C::KROWS * 128, &tm_k, full(stage),
                          kb * (128 / C::ELEM), krow0);
          }
        }
      } else {
        // Gather 128 key rows (one per compact position) with 16-byte cp.async:
        // RCH lanes copy one row (16 for a 256-byte bf16 row, 8 for a
        // 128-byte FP8 row), chunk c of row r lands at its 128-byte-swizzle
        // slot (c ^ (r & 7)) of column block c / 8, so the tensor core sees the
        // same layout a TMA load would have written. Rows without a visible token
        // are zero-filled by the same instruction (nothing is read).
        // The tile's 128 token ids are resolved first (lane l owns rows l,
        // l+32, l+64, l+96: four independent loads), then handed to the
        // copying lanes with shuffles, so no copy waits on a dependent load.
        // Completion is asynchronous: every lane arrives on the stage's full
        // barrier (32 arrivals) once its copies have landed, and the warp
        // goes on to its next tile, so several tiles are in flight at once.
        const long long r = static_cast<long long>(b) * p.T + tg;
        const long long q_pos = p.q_offset + tg;
        long long toks[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) toks[u] = gathered_token(p, r, s.j * C::KROWS + 32 * u + lane, q_pos);
        if (!mbar_wait(empty(stage), ph ^ 1u, p.err)) ok = false;
        if (ok) {
          constexpr int RCH = C::ROW_BYTES / 16;  // lanes (16-byte chunks) per row
          constexpr int RPI = 32 / RCH;           // rows per warp instruction
          const int ch = lane % RCH;
          const uint32_t tile = s_k + stage * C::K_BYTES + (ch >> 3) * C::KROWS * 128;
          // per lane: the global address of its four rows and which of them exist
          const char* kseq = reinterpret_cast<const char*>(p.kg) +
                             static_cast<long long>(b) * p.L_tok * C::ROW_BYTES;
          unsigned long long ga[4];
          uint32_t vm[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            vm[u] = __ballot_sync(0xffffffffu, toks[u] >= 0);
            ga[u] = reinterpret_cast<unsigned long long>(kseq + (toks[u] >= 0 ? toks[u] : 0) * C::ROW_BYTES);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int i = 0; i < 32 / RPI; ++i) {
              const int rl = RPI * i + lane / RCH;  // row 32u + rl lives in lane rl
              const int row = 32 * u + rl;
              const unsigned long long a = __shfl_sync(0xffffffffu, ga[u], rl);
              const uint32_t dst = tile + row * 128 + (((ch & 7) ^ (rl & 7)) << 4);
              cp_async_16_zfill(dst, reinterpret_cast<const void*>(a + ch * 16),
                                ((vm[u] >> rl) & 1u) ? 16u : 0u);
            }
          }
          cp_async_mbar_arrive_noinc(full(stage));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      ++it;
    }
    // cp.async gathers still in flight land before the CTA can release its
    // shared memory (on the normal path the MMA warp has waited for them all)
    if (C::GATHER && !p.blk_tma) cp_async_wait_all();
    if (!ok && lane == 0) {
      // Error path: wait (bounded) for the TMA loads that may still be in
      // flight before the CTA releases its shared memory.
      if (pw == 0)
        for (uint32_t g = gq > C::NQBUF ? gq - C::NQBUF : 0; g < gq; ++g)
          mbar_drain(qfull(static_cast<int>(g % C::NQBUF)), (g / C::NQBUF) & 1u);
      if (!C::GATHER || p.blk_tma) {
        const uint32_t lo = it > C::NSTAGE ? it - C::NSTAGE : 0;
        for (uint32_t i = lo; i < it; ++i) mbar_drain(full(i % C::NSTAGE), (i / C::NSTAGE) & 1u);
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, gq = 0;
      bool ok = true;
      for (; !s.done; s.next(p)) {
        const int qb = static_cast<int>(gq % C::NQBUF);
        if (s.first && !mbar_wait(qfull(qb), (gq / C::NQBUF) & 1u, p.err)) { ok = false; break; }
        const int stage = static_cast<int>(it % C::NSTAGE);
        const uint32_t ph = (it / C::NSTAGE) & 1u;
        const int buf = static_cast<int>(it % C::NACC);
        const uint32_t tph = (it / C::NACC) & 1u;
        if (!mbar_wait(tempty(buf), tph ^ 1u, p.err)) { ok = false; break; }
        if (!mbar_wait(full(stage), ph, p.err)) { ok = false; break; }
        // cp.async gathers wrote the stage through the generic proxy: order
        // those writes before the tensor core's (async proxy) reads
        if (C::GATHER) fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * C::MMA_N);
        const uint32_t k_tile = s_k + stage * C::K_BYTES;
#pragma unroll
        for (int ks = 0; ks < C::NKSTEP; ++ks) {
          const int kb = (ks * 32) / 128;
          const int inner = (ks * 32) % 128;
          const uint64_t kdesc = umma_desc_sw128(k_tile + kb * C::KROWS * 128 + inner);
          const uint64_t qdesc = umma_desc_sw128(s_q + qb * C::Q_BYTES + kb * C::QROWS * 128 + inner);
          const uint64_t adesc = C::ROUTER ? qdesc : kdesc;
          const uint64_t bdesc = C::ROUTER ? kdesc : qdesc;
          if (C::ELEM == 2) mma_bf16(d_tmem, adesc, bdesc, C::IDESC, ks > 0 ? 1u : 0u);
          else mma_f8(d_tmem, adesc, bdesc, C::IDESC, ks > 0 ? 1u : 0u);
        }
        tc_commit(empty(stage));
        tc_commit(tfull(buf));
        if (s.last) { tc_commit(qempty(qb)); ++gq; }
        ++it;
      }
      if (!ok) {
        // Error path: let every MMA already issued finish before TMEM is freed.
        tc_commit(mdone);
        mbar_drain(mdone, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - C::EPI_WARP0;        // 0 .. EPIW-1
    const int quarter = warp & 3;              // TMEM lanes this warp may read
    const int set = e >> 2;                    // 0 .. NSETS-1
    const int row = quarter * 32 + lane;       // accumulator row = TMEM lane
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    float racc = 0.f;                          // router partial sum
    int coef_g = -1;                           // query group of the staged head weights
    uint32_t it = 0;
    if constexpr (C::PLAIN) {
      // Plain bf16 scores with eight epilogue warps (the dense 64-head tile):
      // the store path alone, without the variants' code below (with it in
      // the loop the same work compiled to code 3 % slower on the DSA chunk).
      for (; !s.done; s.next(p), ++it) {
        const int b = s.b;
        const int tg = s.tg;
        const int buf = static_cast<int>(it % C::NACC);
        if (!mbar_wait(tfull(buf), (it / C::NACC) & 1u, p.err)) break;
        tc_fence_after();
        const uint32_t taddr = lane_addr + static_cast<uint32_t>(buf * C::MMA_N);
        {
          constexpr int QH = C::QPT / C::NSETS;  // queries per thread
          constexpr int NC = QH * C::H;          // columns per thread
          constexpr int NCH = NC / 32;           // 32-column chunks
          constexpr int NP = C::H >= 32 ? 2 : 1;  // packed partial sums per query
          const int q0 = set * QH;               // first query (in group)
          const int key = s.j * C::KROWS + row;  // key row
          const long long rbase = static_cast<long long>(b) * p.T + tg * C::QPT + q0;
          // this warp's head weights for the group (queries past T reuse the
          // last query's weights; their outputs are never stored)
          static_assert(NC == C::NCOL_THREAD, "coefficient slot");
          float* cw = reinterpret_cast<float*>(smem + C::SMEM_COEF) + e * NC;
          if (s.g != coef_g) {
            for (int c = lane; c < NC; c += 32) {
              const int ql = c / C::H;
              const int h = c % C::H;
              const int tq = tg * C::QPT + q0 + ql;
              const long long ci = (rbase + ql - (tq < p.T ? 0 : tq - p.T + 1)) * C::H + h;
              cw[c] = __ldg(p.w + ci);
            }
            __syncwarp();
            coef_g = s.g;
          }
          float acc[QH][NP];
          unsigned long long acc2[QH][NP];
#pragma unroll
          for (int i = 0; i < QH; ++i)
#pragma unroll
            for (int j = 0; j < NP; ++j) acc2[i][j] = 0ull;
          // TMEM -> registers one 32-column chunk at a time: the next chunk's
          // load is issued before this chunk's arithmetic, and the buffer goes
          // back to the MMA warp as soon as the last chunk has landed, so the
          // next tile's MMAs overlap the remaining math.
          uint32_t vb[2][32];
          tmem_ld32_issue(taddr + q0 * C::H, vb[0]);
          tmem_ld_wait(vb[0]);
#pragma unroll
          for (int ph = 0; ph < NCH; ++ph) {
            if (ph + 1 < NCH) {
              tmem_ld32_issue(taddr + q0 * C::H + (ph + 1) * 32, vb[(ph + 1) & 1]);
            } else {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(tempty(buf));
            }
            const int cc = ph * 32;
            const uint32_t (&v)[32] = vb[ph & 1];
            float coef[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 c4 = *reinterpret_cast<const float4*>(cw + cc + i);
              coef[i] = c4.x; coef[i + 1] = c4.y; coef[i + 2] = c4.z; coef[i + 3] = c4.w;
            }
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const int ql = (cc + i) / C::H;
              const int pp = (i / 2) % NP;
              acc2[ql][pp] = ffma2(pack2(coef[i], coef[i + 1]),
                                   pack2(fmaxf(__uint_as_float(v[i]), 0.f),
                                         fmaxf(__uint_as_float(v[i + 1]), 0.f)),
                                   acc2[ql][pp]);
            }
            if (ph + 1 < NCH) tmem_ld_wait(vb[(ph + 1) & 1]);
          }
#pragma unroll
          for (int i = 0; i < QH; ++i)
#pragma unroll
            for (int j = 0; j < NP; ++j) {
              const float2 f = unpack2(acc2[i][j]);
              acc[i][j] = f.x + f.y;
            }
          float accq[QH];
#pragma unroll
          for (int i = 0; i < QH; ++i) {
            float a = acc[i][0];
            if (NP == 2) a = acc[i][0] + acc[i][1];
            accq[i] = a;
          }
          if (key < p.Lk) {
            // query q0+ql sees this key iff key * pstride <= q_offset + t0 + ql
            const int t0 = tg * C::QPT + q0;
            const long long e = static_cast<long long>(key) * p.pstride - (p.q_offset + t0);
            float* orow = p.out + rbase * p.ldo + key;
#pragma unroll
            for (int ql = 0; ql < QH; ++ql) {
              if (t0 + ql < p.T && e <= ql) orow[ql * p.ldo] = accq[ql];
            }
          }
        }
      }
    } else if constexpr (C::PLAIN2) {
      // The other bf16 store kernels (16 epilogue warps, or one query per
      // group) likewise without the variants' code.
      for (; !s.done; s.next(p), ++it) {
        const int b = s.b;
        const int tg = s.tg;
        const int buf = static_cast<int>(it % C::NACC);
        const bool mine = C::SPLIT_TILES ? (static_cast<int>(it % C::NSETS) == set) : true;
        if (mine) {
          constexpr int QH = C::SPLIT_TILES ? 1 : C::QPT / C::NSETS;  // queries per thread
          constexpr int NC = QH * C::H;                               // columns per thread
          constexpr int NCH = NC / 32;                                // 32-column chunks
          constexpr int NP = C::H >= 32 ? 2 : 1;                      // packed partial sums per query
          static_assert(NC == C::NCOL_THREAD && NC % 32 == 0 && NCH >= 1, "coefficient slot, chunks");
          const int q0 = C::SPLIT_TILES ? 0 : set * QH;               // first query (in group)
          const int key = s.j * C::KROWS + row;                       // key row
          const long long rbase = static_cast<long long>(b) * p.T + tg * C::QPT + q0;
          // FP8: this row's key dequant scale, loaded before the wait
          float ks = 1.f;
          if constexpr (C::KEY_SCALES) {
            if (key < p.Lk) ks = __ldg(p.k_scale + static_cast<long long>(b) * p.Lk + key);
          }
          if (!mbar_wait(tfull(buf), (it / C::NACC) & 1u, p.err)) break;
          tc_fence_after();
          const uint32_t taddr = lane_addr + static_cast<uint32_t>(buf * C::MMA_N);
          // this warp's head weights (x query scales) for the group
          float* cw = reinterpret_cast<float*>(smem + C::SMEM_COEF) + e * NC;
          if (s.g != coef_g) {
            for (int c = lane; c < NC; c += 32) {
              const int ql = c / C::H;
              const int h = c % C::H;
              const int tq = tg * C::QPT + q0 + ql;
              const long long ci = (rbase + ql - (tq < p.T ? 0 : tq - p.T + 1)) * C::H + h;
              float cv = __ldg(p.w + ci);
              if (C::ELEM == 1) cv *= __ldg(p.q_scale + ci);
              cw[c] = cv;
            }
            __syncwarp();
            coef_g = s.g;
          }
          unsigned long long acc2[QH][NP];
#pragma unroll
          for (int i = 0; i < QH; ++i)
#pragma unroll
            for (int j = 0; j < NP; ++j) acc2[i][j] = 0ull;
          if constexpr (C::EPIW == 16 || C::CTAS == 2) {
            // one 32-column chunk in flight per warp; the other warps of the
            // sub-partition hide its load latency
#pragma unroll
            for (int ph = 0; ph < NCH; ++ph) {
              uint32_t v[32];
              tmem_ld32_issue(taddr + q0 * C::H + ph * 32, v);
              tmem_ld_wait(v);
              if (ph == NCH - 1) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty(buf));
              }
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                const float4 c4 = *reinterpret_cast<const float4*>(cw + ph * 32 + i);
                const int ql = (ph * 32 + i) / C::H;
                acc2[ql][(i / 2) % NP] = ffma2(pack2(c4.x, c4.y),
                                               pack2(fmaxf(__uint_as_float(v[i]), 0.f),
                                                     fmaxf(__uint_as_float(v[i + 1]), 0.f)),
                                               acc2[ql][(i / 2) % NP]);
                acc2[ql][(i / 2 + 1) % NP] = ffma2(pack2(c4.z, c4.w),
                                                   pack2(fmaxf(__uint_as_float(v[i + 2]), 0.f),
                                                         fmaxf(__uint_as_float(v[i + 3]), 0.f)),
                                                   acc2[ql][(i / 2 + 1) % NP]);
              }
            }
          } else {
            // the next chunk's TMEM load issued before this chunk's arithmetic
            uint32_t vb[2][32];
            tmem_ld32_issue(taddr + q0 * C::H, vb[0]);
            tmem_ld_wait(vb[0]);
#pragma unroll
            for (int ph = 0; ph < NCH; ++ph) {
              if (ph + 1 < NCH) {
                tmem_ld32_issue(taddr + q0 * C::H + (ph + 1) * 32, vb[(ph + 1) & 1]);
              } else {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty(buf));
              }
              const int cc = ph * 32;
              const uint32_t (&v)[32] = vb[ph & 1];
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                const float4 c4 = *reinterpret_cast<const float4*>(cw + cc + i);
                const int ql = (cc + i) / C::H;
                acc2[ql][(i / 2) % NP] = ffma2(pack2(c4.x, c4.y),
                                               pack2(fmaxf(__uint_as_float(v[i]), 0.f),
                                                     fmaxf(__uint_as_float(v[i + 1]), 0.f)),
                                               acc2[ql][(i / 2) % NP]);
                acc2[ql][(i / 2 + 1) % NP] = ffma2(pack2(c4.z, c4.w),
                                                   pack2(fmaxf(__uint_as_float(v[i + 2]), 0.f),
                                                         fmaxf(__uint_as_float(v[i + 3]), 0.f)),
                                                   acc2[ql][(i / 2 + 1) % NP]);
              }
              if (ph + 1 < NCH) tmem_ld_wait(vb[(ph + 1) & 1]);
            }
          }
          float accq[QH];
#pragma unroll
          for (int i = 0; i < QH; ++i) {
            float a = 0.f;
#pragma unroll
            for (int j = 0; j < NP; ++j) {
              const float2 f = unpack2(acc2[i][j]);
              a += f.x + f.y;
            }
            accq[i] = a;
          }
          if (key < p.Lk) {
            // query q0+ql sees this key iff key * pstride <= q_offset + t0 + ql
            const int t0 = tg * C::QPT + q0;
            const long long e = static_cast<long long>(key) * p.pstride - (p.q_offset + t0);
            float* orow = p.out + rbase * p.ldo + key;
#pragma unroll
            for (int ql = 0; ql < QH; ++ql) {
              if (t0 + ql < p.T && e <= ql) orow[ql * p.ldo] = ks * accq[ql];
            }
          }
        }
      }
    } else {
    // candidate lists (CMP): lane ql keeps the reservation state of this
    // warp's query ql: current chunk (base, used), whether the next chunk has
    // been requested (and where it starts), and the real entries written
    constexpr int QHC = (C::ROUTER || C::GATHER || C::SPLIT_TILES) ? 1 : C::QPT / C::NSETS;
    int cbase = -1, cused = CCHUNK, chas = 0, cnext = 0, creal = 0;
    for (; !s.done; s.next(p)) {
      const int b = s.b;
      const int tg = s.tg;
      const int q0s = C::SPLIT_TILES ? 0 : set * QHC;            // this set's first query (in group)
      const long long rbase_s = static_cast<long long>(b) * p.T + tg * C::QPT + q0s;
      if constexpr (C::CMP) {
        // a new group (or this CTA's first tile): request the first chunk of
        // every query now, so it has landed by the first kept score
        if (s.first && lane < QHC && tg * C::QPT + q0s + lane < p.T) {
          cbase = -1;
          cused = CCHUNK;
          chas = 1;
          creal = 0;
          cnext = atomicAdd(p.cres + rbase_s + lane, CCHUNK);
        }
      }
      {
      const int buf = static_cast<int>(it % C::NACC);
      // split tiles: the two sets take alternate tiles (buffer b: set b & 1)
      const bool mine = C::SPLIT_TILES ? (static_cast<int>(it % C::NSETS) == set) : true;
      if (mine) {
        // gather mode: this row's token (and visibility), loaded before the
        // wait so that its latency hides behind the tile's MMAs
        long long gtok = -1;
        if constexpr (C::GATHER) {
          const int gkey = s.j * C::KROWS + row;
          if (gkey < p.n_compact)
            gtok = gathered_token(p, static_cast<long long>(b) * p.T + tg, gkey, p.q_offset + tg);
        }
        // FP8: this row's key dequant scale, likewise
        float ks = 1.f;
        if constexpr (C::KEY_SCALES && C::GATHER) {
          if (gtok >= 0) ks = __ldg(p.k_scale + static_cast<long long>(b) * p.L_tok + gtok);
        } else if constexpr (C::KEY_SCALES) {
          const int skey = s.j * C::KROWS + row;
          if (skey < p.Lk) ks = __ldg(p.k_scale + static_cast<long long>(b) * p.Lk + skey);
        }
        // DoSA: this row's key norm, likewise
        float kn = 0.f;
        if constexpr (C::BND) {
          const int nkey = s.j * C::KROWS + row;
          if (nkey < p.Lk) kn = __ldg(p.knorm + static_cast<long long>(b) * p.Lk + nkey);
        }
        // candidate thresholds of this thread's queries (compaction only)
        constexpr int QHT = QHC;
        float cthr[QHT];
#pragma unroll
        for (int ql = 0; ql < QHT; ++ql) cthr[ql] = INFINITY;
        if constexpr (C::CMP) {
          const int tq0 = tg * C::QPT + (C::SPLIT_TILES ? 0 : set * QHT);
#pragma unroll
          for (int ql = 0; ql < QHT; ++ql)
            if (tq0 + ql < p.T) cthr[ql] = __ldg(p.cthr + static_cast<long long>(b) * p.T + tq0 + ql);
        }
        if (!mbar_wait(tfull(buf), (it / C::NACC) & 1u, p.err)) break;
        tc_fence_after();
        const uint32_t taddr = lane_addr + static_cast<uint32_t>(buf * C::MMA_N);
        if constexpr (C::ROUTER) {
          // rows: (query, head) pairs; columns: pooled keys j*256 + c
          const int t = tg * C::QPT + row / C::H;
          const long long pos = p.q_offset + (t < p.T ? t : p.T - 1);
          long long mv = pos / p.pstride + 1;
          if (mv > p.Lk) mv = p.Lk;
          const long long m0 = static_cast<long long>(s.j) * C::KROWS;
          float part = 0.f;
#pragma unroll 1
          for (int cc = 0; cc < C::KROWS; cc += 32) {
            float v[32];
            tmem_ld32(taddr + cc, v);
            if constexpr (C::ELEM == 1) {
              // FP8 pooled keys: column m carries its dequant scale (>= 0, so
              // it moves out of the ReLU); lane i loads column cc + i's, 0 for
              // columns past the visible ones
              const long long mc = m0 + cc + lane;
              const float kl = mc < mv ? __ldg(p.k_scale + static_cast<long long>(b) * p.Lk + mc) : 0.f;
#pragma unroll
              for (int i = 0; i < 32; ++i) part = fmaf(__shfl_sync(0xffffffffu, kl, i), fmaxf(v[i], 0.f), part);
            } else if (m0 + cc + 32 <= mv) {
#pragma unroll
              for (int i = 0; i < 32; ++i) part += fmaxf(v[i], 0.f);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) part += (m0 + cc + i < mv) ? fmaxf(v[i], 0.f) : 0.f;
            }
          }
          racc += part;
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty(buf));
        } else {
          constexpr int QH = C::SPLIT_TILES ? 1 : C::QPT / C::NSETS;   // queries per thread
          static_assert(QH == QHT, "threshold slots");
          constexpr int NC = QH * C::H;                          // columns per thread
          constexpr int NCH = NC / 32;                           // 32-column chunks
          static_assert(NC % 32 == 0 && NCH >= 1, "each epilogue thread takes whole 32-column chunks");
          // independent partial sums per query (breaks the FMA dependency chain)
#if defined(DSA_NO_FFMA2)
          constexpr int NP = C::H >= 32 ? 4 : (C::H == 16 ? 2 : 1);
#else
          constexpr int NP = C::H >= 32 ? 2 : 1;   // packed pairs: 2 x 2 lanes
#endif
          const int q0 = C::SPLIT_TILES ? 0 : set * QH;          // first query (in group)
          const int key = s.j * C::KROWS + row;                  // key row / compact position
          const long long rbase = static_cast<long long>(b) * p.T + tg * C::QPT + q0;
          // head weights of this thread's columns are contiguous in w when every
          // query of the half-group exists
          // this warp's head weights for the group (queries past T reuse the
          // last query's weights; their outputs are never stored)
          static_assert(NC == C::NCOL_THREAD, "coefficient slot");
          float* cw = reinterpret_cast<float*>(smem + C::SMEM_COEF) + e * (NC + C::NBND_THREAD);
          if (s.g != coef_g) {
            for (int c = lane; c < NC; c += 32) {
              const int ql = c / C::H;
              const int h = c % C::H;
              const int tq = tg * C::QPT + q0 + ql;
              const long long ci = (rbase + ql - (tq < p.T ? 0 : tq - p.T + 1)) * C::H + h;
              float cv = __ldg(p.w + ci);
              if (C::ELEM == 1) cv *= __ldg(p.q_scale + ci);
              cw[c] = cv;
            }
            if constexpr (C::BND) {
              for (int ql = lane; ql < QH; ql += 32) {
                const bool in = tg * C::QPT + q0 + ql < p.T;
                cw[NC + 2 * ql] = in ? __ldg(p.cthr + rbase + ql) : INFINITY;
                cw[NC + 2 * ql + 1] = in ? __ldg(p.cbound + rbase + ql) : 0.f;
              }
            }
            __syncwarp();
            coef_g = s.g;
          }
          float acc[QH][NP];
#pragma unroll
          for (int i = 0; i < QH; ++i)
#pragma unroll
            for (int j = 0; j < NP; ++j) acc[i][j] = 0.f;
#if !defined(DSA_NO_FFMA2)
          unsigned long long acc2[QH][NP];
#pragma unroll
          for (int i = 0; i < QH; ++i)
#pragma unroll
            for (int j = 0; j < NP; ++j) acc2[i][j] = 0ull;
#endif
          if constexpr (C::EPIW == 16 || C::CTAS == 2) {
            // Sixteen epilogue warps (four per sub-partition, 96 registers a
            // thread): one 32-column chunk in flight per warp, the other
            // warps hide its load latency; head weights read four at a time.
#pragma unroll
            for (int ph = 0; ph < NCH; ++ph) {
              uint32_t v[32];
              tmem_ld32_issue(taddr + q0 * C::H + ph * 32, v);
              tmem_ld_wait(v);
              if (ph == NCH - 1) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty(buf));
              }
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                const float4 c4 = *reinterpret_cast<const float4*>(cw + ph * 32 + i);
                const int ql = (ph * 32 + i) / C::H;
#if defined(DSA_NO_FFMA2)
                acc[ql][i % NP] = fmaf(c4.x, fmaxf(__uint_as_float(v[i]), 0.f), acc[ql][i % NP]);
                acc[ql][(i + 1) % NP] = fmaf(c4.y, fmaxf(__uint_as_float(v[i + 1]), 0.f), acc[ql][(i + 1) % NP]);
                acc[ql][(i + 2) % NP] = fmaf(c4.z, fmaxf(__uint_as_float(v[i + 2]), 0.f), acc[ql][(i + 2) % NP]);
                acc[ql][(i + 3) % NP] = fmaf(c4.w, fmaxf(__uint_as_float(v[i + 3]), 0.f), acc[ql][(i + 3) % NP]);
#else
                acc2[ql][(i / 2) % NP] = ffma2(pack2(c4.x, c4.y),
                                               pack2(fmaxf(__uint_as_float(v[i]), 0.f),
                                                     fmaxf(__uint_as_float(v[i + 1]), 0.f)),
                                               acc2[ql][(i / 2) % NP]);
                acc2[ql][(i / 2 + 1) % NP] = ffma2(pack2(c4.z, c4.w),
                                                   pack2(fmaxf(__uint_as_float(v[i + 2]), 0.f),
                                                         fmaxf(__uint_as_float(v[i + 3]), 0.f)),
                                                   acc2[ql][(i / 2 + 1) % NP]);
#endif
              }
            }
          } else {
            // TMEM -> registers one 32-column chunk at a time: the next chunk's
            // load is issued before this chunk's arithmetic, and the buffer goes
            // back to the MMA warp as soon as the last chunk has landed, so the
            // next tile's MMAs overlap the remaining math.
            constexpr int PH = 1;  // chunks per phase (more would exceed the register budget)
            constexpr int NPHASE = NCH / PH;
            uint32_t vb[2][PH][32];
#pragma unroll
            for (int c = 0; c < PH; ++c) tmem_ld32_issue(taddr + q0 * C::H + c * 32, vb[0][c]);
#pragma unroll
            for (int c = 0; c < PH; ++c) tmem_ld_wait(vb[0][c]);
#pragma unroll
            for (int ph = 0; ph < NPHASE; ++ph) {
              if (ph + 1 < NPHASE) {
#pragma unroll
                for (int c = 0; c < PH; ++c)
                  tmem_ld32_issue(taddr + q0 * C::H + ((ph + 1) * PH + c) * 32, vb[(ph + 1) & 1][c]);
              } else {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty(buf));
              }
#pragma unroll
              for (int c = 0; c < PH; ++c) {
                const int cc = (ph * PH + c) * 32;
                const uint32_t (&v)[32] = vb[ph & 1][c];
                float coef[32];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                  const float4 c4 = *reinterpret_cast<const float4*>(cw + cc + i);
                  coef[i] = c4.x; coef[i + 1] = c4.y; coef[i + 2] = c4.z; coef[i + 3] = c4.w;
                }
#if defined(DSA_NO_FFMA2)
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  const int ql = (cc + i) / C::H;
                  const int pp = i % NP;
                  acc[ql][pp] = fmaf(coef[i], fmaxf(__uint_as_float(v[i]), 0.f), acc[ql][pp]);
                }
#else
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                  const int ql = (cc + i) / C::H;
                  const int pp = (i / 2) % NP;
                  acc2[ql][pp] = ffma2(pack2(coef[i], coef[i + 1]),
                                       pack2(fmaxf(__uint_as_float(v[i]), 0.f),
                                             fmaxf(__uint_as_float(v[i + 1]), 0.f)),
                                       acc2[ql][pp]);
                }
#endif
              }
              if (ph + 1 < NPHASE) {
#pragma unroll
                for (int c = 0; c < PH; ++c) tmem_ld_wait(vb[(ph + 1) & 1][c]);
              }
            }
          }
#if !defined(DSA_NO_FFMA2)
#pragma unroll
          for (int i = 0; i < QH; ++i)
#pragma unroll
            for (int j = 0; j < NP; ++j) {
              const float2 f = unpack2(acc2[i][j]);
              acc[i][j] = f.x + f.y;
            }
#endif
          float accq[QH];
#pragma unroll
          for (int i = 0; i < QH; ++i) {
            float a = acc[i][0];
            if (NP == 2) a = acc[i][0] + acc[i][1];
            if (NP == 4) a = (acc[i][0] + acc[i][1]) + (acc[i][2] + acc[i][3]);
            accq[i] = a;
          }
          if (C::GATHER) {
            const long long r = static_cast<long long>(b) * p.T + tg;
            if (key < p.n_compact) p.out[r * p.ldo + key] = gtok >= 0 ? ks * accq[0] : -INFINITY;
          } else {
            // query q0+ql sees this key iff key * pstride <= q_offset + t0 + ql
            const int t0 = tg * C::QPT + q0;
            const long long e = static_cast<long long>(key) * p.pstride - (p.q_offset + t0);
            if constexpr (C::BND) {
              // DoSA: bound >= threshold for some visible key of the warp ->
              // the tile is live for the query's refinement group
              uint32_t lmask = 0;  // bit ql: this key is live for query ql
#pragma unroll
              for (int ql = 0; ql < QH; ++ql) {
                const float2 tc = *reinterpret_cast<const float2*>(cw + NC + 2 * ql);  // (thr, c_t)
                const bool live = key < p.Lk && e <= ql && fmaf(tc.y, kn, accq[ql]) >= tc.x;
                lmask |= static_cast<uint32_t>(live) << ql;
              }
              // one flag per refinement group of live_qpt queries (t0 is a
              // multiple of QH, which is a multiple of live_qpt or covers a
              // part of one group)
              const int qg = p.live_qpt < QH ? p.live_qpt : QH;
              for (int g0 = 0; g0 < QH; g0 += qg) {
                const uint32_t gm = qg >= 32 ? 0xffffffffu : ((1u << qg) - 1u) << g0;
                if (__ballot_sync(0xffffffffu, (lmask & gm) != 0u) != 0u && lane == 0)
                  p.live_out[(static_cast<long long>(b) * p.live_gpb + (t0 + g0) / p.live_qpt) * p.live_ld + s.j] = 1;
              }
            } else if (key < p.Lk && (!C::CMP || p.out != nullptr)) {
              float* orow = p.out + rbase * p.ldo + key;
#pragma unroll
              for (int ql = 0; ql < QH; ++ql) {
                if (t0 + ql < p.T && e <= ql) orow[ql * p.ldo] = ks * accq[ql];
              }
            }
            if constexpr (C::CMP) {
              // candidate lists: the warp's kept scores of query ql fill
              // consecutive slots of its current chunk (lane ql holds the
              // chunk state, uniform across the warp after the shuffles); a
              // full chunk continues in the requested next one, and the chunk
              // after that is requested once half of the current one is used,
              // so the atomic's latency hides behind later tiles
              const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
              for (int ql = 0; ql < QH; ++ql) {
                const float sc = ks * accq[ql];
                const bool keep = key < p.Lk && t0 + ql < p.T && e <= ql && sc >= cthr[ql];
                const uint32_t msk = __ballot_sync(0xffffffffu, keep);
                if (msk == 0u) continue;
                const int n = __popc(msk);
                const int pre = __popc(msk & lt);
                const int used = __shfl_sync(0xffffffffu, cused, ql);
                const int base = __shfl_sync(0xffffffffu, cbase, ql);
                int slot;
                if (used + n <= CCHUNK) {
                  slot = base + used + pre;
                  if (lane == ql) cused = used + n;
                } else {
                  int nxt;
                  if (__shfl_sync(0xffffffffu, chas, ql)) {
                    nxt = __shfl_sync(0xffffffffu, cnext, ql);
                  } else {
                    int v = 0;
                    if (lane == ql) v = atomicAdd(p.cres + rbase + ql, CCHUNK);
                    nxt = __shfl_sync(0xffffffffu, v, ql);
                  }
                  const int room = CCHUNK - used;
                  slot = pre < room ? base + used + pre : nxt + (pre - room);
                  if (lane == ql) { cbase = nxt; cused = n - room; chas = 0; }
                }
                if (keep && slot < p.ccap) {
                  const long long o = (rbase + ql) * p.ccap + slot;
                  p.cval[o] = sc;
                  p.cidx[o] = key;
                }
                if (lane == ql) {
                  creal += n;
                  if (!chas && cused >= CCHUNK / 2) {
                    cnext = atomicAdd(p.cres + rbase + ql, CCHUNK);
                    chas = 1;
                  }
                }
              }
            }
          }
        }
      }
      ++it;
      }
      if constexpr (C::CMP) {
        if (s.last) {
          // leaving the group: sentinels over the unused slots of this warp's
          // chunks, then the real entries are counted
#pragma unroll 1
          for (int ql = 0; ql < QHC; ++ql) {
            if (tg * C::QPT + q0s + ql >= p.T) break;
            const long long orow = (rbase_s + ql) * p.ccap;
            const int base = __shfl_sync(0xffffffffu, cbase, ql);
            const int used = __shfl_sync(0xffffffffu, cused, ql);
            const int has = __shfl_sync(0xffffffffu, chas, ql);
            const int nxt = __shfl_sync(0xffffffffu, cnext, ql);
            if (base >= 0)
              for (int i = used + lane; i < CCHUNK; i += 32)
                if (base + i < p.ccap) { p.cval[orow + base + i] = -INFINITY; p.cidx[orow + base + i] = -1; }
            if (has)
              for (int i = lane; i < CCHUNK; i += 32)
                if (nxt + i < p.ccap) { p.cval[orow + nxt + i] = -INFINITY; p.cidx[orow + nxt + i] = -1; }
            if (lane == ql && creal > 0) atomicAdd(p.creal + rbase_s + ql, creal);
          }
          cbase = -1;
          cused = CCHUNK;
          chas = 0;
          creal = 0;
        }
      }
      if (C::ROUTER && s.last) {
        // End of a query group: each set writes its partial sums (possibly 0).
        const int t = tg * C::QPT + row / C::H;
        if (t < p.T) {
          const long long ix = (static_cast<long long>(b) * p.T + t) * C::H + (row % C::H);
          p.out[static_cast<long long>(set) * p.batch * p.T * C::H + ix] = racc;
        }
        racc = 0.f;
      }
    }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace dsa
