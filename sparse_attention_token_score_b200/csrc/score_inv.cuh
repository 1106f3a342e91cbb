// HISA token refinement, block-major ("HISA: Efficient Hierarchical Indexing
// for Fine-Grained Sparse Attention" review, section 3 and Figure 1: every
// query keeps its top-m blocks, then scores the tokens of those blocks with
// the full indexer,
//     I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:]),  s in a kept block, s <= p_t).
//
// The kept-block lists [rows, m] are inverted first (invert_* kernels below):
// for every block, the (row, slot) pairs of the queries that kept it. The
// scoring kernel then walks blocks, not queries: a 128-key tile of a block is
// loaded once into shared memory and stays there while the queries that chose
// the block stream through it, QC queries x H heads per MMA (N = QC * H = 128).
// A kept block is thus read once per block instead of once per query that
// kept it; the queries (H * d * 2 bytes each) are what streams.
//
// Work items, in order: (block g, key tile u of the block, chunk c of QC of
// its queries). Item counts per block are a prefix sum (ioff), so a CTA finds
// its first item by binary search and walks on from there; all items cost
// one MMA tile.
//
// One persistent CTA per SM, warp-specialised as the other score kernels:
// one TMA producer warp (key tile into one of two stationary buffers, query
// chunk into a ring stage), one MMA-issuing thread (D[key, query*H + h] in
// TMEM, NACC accumulators), two sets of four epilogue warps taking alternate
// items (tcgen05.ld, ReLU, head-weighted sum per query, causal / length mask,
// store into the query's compact row at slot * blk + u * 128 + key).
#pragma once
#include "common.cuh"

namespace dsa {

struct InvParams {
  int batch, T, L, M;       // sequences, queries per sequence, tokens per sequence, blocks per sequence
  int blk;                  // tokens per block (a multiple of 128)
  int m;                    // kept blocks per query (slots)
  long long q_offset;
  const float* w;           // [batch*T, H]
  float* out;               // [batch*T, ldo] compact rows: position slot * blk + i
  long long ldo;
  const int* cnt;           // [batch*M] queries that kept each block
  const int* qoff;          // [batch*M + 1] start of each block's list
  const int* ioff;          // [batch*M + 1] start of each block's items
  const int2* list;         // [total kept] (row, slot), grouped by block
  unsigned* err;
};

template <int H_, int NSTAGE_>
struct InvCfg {
  static constexpr int D = 128, H = H_, NSTAGE = NSTAGE_;
  static constexpr int ROW_BYTES = D * 2;                // bf16
  static constexpr int KBLK = ROW_BYTES / 128;           // 128-byte column blocks per row
  static constexpr int QC = 128 / H;                     // queries per item
  static constexpr int NROWS = QC * H;                   // streamed query rows per item (MMA N)
  static constexpr int KROWS = 128;                      // stationary key rows (MMA M)
  static_assert(NROWS == 128, "N = 128 columns per item");
  static constexpr int K_BYTES = KROWS * ROW_BYTES;      // one stationary key tile
  static constexpr int Q_BYTES = NROWS * ROW_BYTES;      // one query-chunk stage
  static constexpr int NKSTEP = ROW_BYTES / 32;
  static constexpr int NACC = 4;                         // 4 x 128 TMEM columns
  static constexpr int TMEM_COLS = 512;
  static constexpr int NKBUF = 2;                        // stationary key buffers
  static constexpr int MMA_WARP = 1;
  static constexpr int EPI_WARP0 = 2;
  static constexpr int EPIW = 8;
  static constexpr int NTHREADS = (EPI_WARP0 + EPIW) * 32;
  static constexpr uint32_t IDESC = umma_idesc(1u, 128, NROWS);
  static constexpr int SMEM_K = 0;
  static constexpr int SMEM_Q = NKBUF * K_BYTES;
  static constexpr int SMEM_COEF = SMEM_Q + NSTAGE * Q_BYTES;   // per epilogue warp: NROWS coefficients
  static constexpr int SMEM_BAR = SMEM_COEF + EPIW * NROWS * 4;
  static constexpr int NBAR = 2 * NSTAGE + 2 * NKBUF + 2 * NACC + 1;
  static constexpr int SMEM_BYTES = SMEM_BAR + NBAR * 8 + 16 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Walks this CTA's items; every thread runs its own copy, all copies visit
// the same sequence.
template <class C>
struct InvSched {
  long long i, i1;     // current item, end of this CTA's range
  int g;               // current block (global: b * M + j)
  int loc;             // item index inside the block
  int nq;              // queries of block g
  int nch;             // chunks of block g
  int u, ch;           // key tile inside the block, chunk
  bool first, last, done;

  __device__ __forceinline__ void load_block(const InvParams& p) {
    nq = __ldg(p.cnt + g);
    nch = (nq + C::QC - 1) / C::QC;
  }
  __device__ __forceinline__ void set_pos(const InvParams& p) {
    u = loc / nch;
    ch = loc - u * nch;
    // the key tile changes at the first chunk of every tile (and at this
    // CTA's first item); it is released after its last chunk (or this CTA's
    // last item)
    last = (ch == nch - 1) || (i + 1 == i1);
  }
  __device__ __forceinline__ void init(const InvParams& p, long long total) {
    const long long G = gridDim.x;
    i = total * blockIdx.x / G;
    i1 = total * (blockIdx.x + 1) / G;
    done = i >= i1;
    if (done) return;
    // block with ioff[g] <= i < ioff[g + 1] (ioff is non-decreasing)
    int lo = 0, hi = p.batch * p.M - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(p.ioff + mid) <= i) lo = mid;
      else hi = mid - 1;
    }
    g = lo;
    loc = static_cast<int>(i - __ldg(p.ioff + g));
    load_block(p);
    set_pos(p);
    first = true;
  }
  __device__ __forceinline__ void next(const InvParams& p) {
    if (++i >= i1) { done = true; return; }
    const int prev_u = u;
    ++loc;
    if (loc == (p.blk / 128) * nch) {
      do { ++g; } while (__ldg(p.ioff + g + 1) == __ldg(p.ioff + g));
      loc = 0;
      load_block(p);
      set_pos(p);
      first = true;
      return;
    }
    set_pos(p);
    first = (u != prev_u);
  }
};

template <class C>
__global__ void __launch_bounds__(C::NTHREADS, 1)
score_inv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const InvParams p, const long long* total_items) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_k = s_base + C::SMEM_K;
  const uint32_t s_q = s_base + C::SMEM_Q;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  auto full = [&](int i) { return smem_u32(&bars[i]); };                       // query stage loaded
  auto empty = [&](int i) { return smem_u32(&bars[C::NSTAGE + i]); };          // query stage consumed
  auto kfull = [&](int i) { return smem_u32(&bars[2 * C::NSTAGE + i]); };      // key tile loaded
  auto kempty = [&](int i) { return smem_u32(&bars[2 * C::NSTAGE + C::NKBUF + i]); };
  constexpr int TB = 2 * C::NSTAGE + 2 * C::NKBUF;
  auto tfull = [&](int b) { return smem_u32(&bars[TB + b]); };
  auto tempty = [&](int b) { return smem_u32(&bars[TB + C::NACC + b]); };
  const uint32_t mdone = smem_u32(&bars[TB + 2 * C::NACC]);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(full(i), 1);
      mbar_init(empty(i), 1);
    }
    for (int i = 0; i < C::NKBUF; ++i) {
      mbar_init(kfull(i), 1);
      mbar_init(kempty(i), 1);
    }
    for (int b = 0; b < C::NACC; ++b) {
      mbar_init(tfull(b), 1);
      mbar_init(tempty(b), 4);  // one arrival per warp of the set that owns the item
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
    tma_prefetch_desc(&tm_k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  InvSched<C> s;
  s.init(p, *total_items);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t it = 0, gk = 0;
    bool ok = true;
    if (lane == 0) {
      for (; !s.done; s.next(p), ++it) {
        const int b = s.g / p.M;
        const int j = s.g - b * p.M;
        if (s.first) {
          const int kb_ = static_cast<int>(gk % C::NKBUF);
          if (!mbar_wait(kempty(kb_), ((gk / C::NKBUF) & 1u) ^ 1u, p.err)) { ok = false; break; }
          mbar_arrive_expect_tx(kfull(kb_), C::K_BYTES);
          const int row0 = b * p.L + j * p.blk + s.u * 128;
#pragma unroll
          for (int cb = 0; cb < C::KBLK; ++cb)
            tma_load_2d(s_k + kb_ * C::K_BYTES + cb * C::KROWS * 128, &tm_k, kfull(kb_), cb * 64, row0);
          ++gk;
        }
        const int stage = static_cast<int>(it % C::NSTAGE);
        if (!mbar_wait(empty(stage), ((it / C::NSTAGE) & 1u) ^ 1u, p.err)) { ok = false; break; }
        const int q0 = __ldg(p.qoff + s.g) + s.ch * C::QC;
        const int nq = min(C::QC, s.nq - s.ch * C::QC);
        mbar_arrive_expect_tx(full(stage), static_cast<uint32_t>(nq * C::H * C::ROW_BYTES));
        for (int i = 0; i < nq; ++i) {
          const int r = __ldg(&p.list[q0 + i].x);
#pragma unroll
          for (int cb = 0; cb < C::KBLK; ++cb)
            tma_load_2d(s_q + stage * C::Q_BYTES + cb * C::NROWS * 128 + i * C::H * 128, &tm_q, full(stage),
                        cb * 64, r * C::H);
        }
      }
      if (!ok) {
        // error path: the loads already issued land before shared memory is released
        for (uint32_t g2 = gk > C::NKBUF ? gk - C::NKBUF : 0; g2 < gk; ++g2)
          mbar_drain(kfull(static_cast<int>(g2 % C::NKBUF)), (g2 / C::NKBUF) & 1u);
        const uint32_t lo = it > C::NSTAGE ? it - C::NSTAGE : 0;
        for (uint32_t i = lo; i < it; ++i) mbar_drain(full(i % C::NSTAGE), (i / C::NSTAGE) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, gk = 0;
      bool ok = true;
      for (; !s.done; s.next(p), ++it) {
        const int kb_ = static_cast<int>(gk % C::NKBUF);
        if (s.first && !mbar_wait(kfull(kb_), (gk / C::NKBUF) & 1u, p.err)) { ok = false; break; }
        const int stage = static_cast<int>(it % C::NSTAGE);
        const int buf = static_cast<int>(it % C::NACC);
        if (!mbar_wait(tempty(buf), ((it / C::NACC) & 1u) ^ 1u, p.err)) { ok = false; break; }
        if (!mbar_wait(full(stage), (it / C::NSTAGE) & 1u, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * C::NROWS);
#pragma unroll
        for (int ks = 0; ks < C::NKSTEP; ++ks) {
          const int cb = (ks * 32) / 128;
          const int inner = (ks * 32) % 128;
          const uint64_t adesc = umma_desc_sw128(s_k + kb_ * C::K_BYTES + cb * C::KROWS * 128 + inner);
          const uint64_t bdesc = umma_desc_sw128(s_q + stage * C::Q_BYTES + cb * C::NROWS * 128 + inner);
          mma_bf16(d_tmem, adesc, bdesc, C::IDESC, ks > 0 ? 1u : 0u);
        }
        tc_commit(empty(stage));
        tc_commit(tfull(buf));
        if (s.last) { tc_commit(kempty(kb_)); ++gk; }
      }
      if (!ok) {
        tc_commit(mdone);
        mbar_drain(mdone, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - C::EPI_WARP0;        // 0 .. 7
    const int quarter = warp & 3;              // TMEM lanes this warp may read
    const int set = e >> 2;                    // items alternate between the two sets
    const int row = quarter * 32 + lane;       // key of the tile = TMEM lane
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    float* cw = reinterpret_cast<float*>(smem + C::SMEM_COEF) + e * C::NROWS;
    uint32_t it = 0;
    for (; !s.done; s.next(p), ++it) {
      if (static_cast<int>(it & 1u) != set) continue;
      const int buf = static_cast<int>(it % C::NACC);
      const int b = s.g / p.M;
      const int j = s.g - b * p.M;
      const int q0 = __ldg(p.qoff + s.g) + s.ch * C::QC;
      const int nq = min(C::QC, s.nq - s.ch * C::QC);
      // this item's queries (row, slot) and their head weights, before the wait
      int2 ent[C::QC];
#pragma unroll
      for (int i = 0; i < C::QC; ++i) ent[i] = i < nq ? __ldg(p.list + q0 + i) : make_int2(-1, 0);
      {
        // lane l stages coefficients 4l .. 4l+3 (of query 4l / H; columns of
        // queries past nq take query 0's, their sums are never stored)
        const int c0 = 4 * lane;
        const int qi = c0 / C::H;
        const int2 eq = __ldg(p.list + q0 + (qi < nq ? qi : 0));
        const float4 wv = __ldg(reinterpret_cast<const float4*>(p.w + static_cast<long long>(eq.x) * C::H +
                                                                (c0 % C::H)));
        *reinterpret_cast<float4*>(cw + c0) = wv;
        __syncwarp();
      }
      const int tok = j * p.blk + s.u * 128 + row;  // token of this lane's key in its sequence
      if (!mbar_wait(tfull(buf), (it / C::NACC) & 1u, p.err)) break;
      tc_fence_after();
      const uint32_t taddr = lane_addr + static_cast<uint32_t>(buf * C::NROWS);
      unsigned long long acc2[C::QC][2];
#pragma unroll
      for (int i = 0; i < C::QC; ++i) { acc2[i][0] = 0ull; acc2[i][1] = 0ull; }
      constexpr int NCH = C::NROWS / 32;
      uint32_t vb[2][32];
      tmem_ld32_issue(taddr, vb[0]);
      tmem_ld_wait(vb[0]);
#pragma unroll
      for (int ph = 0; ph < NCH; ++ph) {
        if (ph + 1 < NCH) {
          tmem_ld32_issue(taddr + (ph + 1) * 32, vb[(ph + 1) & 1]);
        } else {
          // the accumulator is in registers: hand it back to the MMA thread
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty(buf));
        }
        const uint32_t (&v)[32] = vb[ph & 1];
        const int cc = ph * 32;
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int ql = (cc + i) / C::H;
          const int pp = (i / 2) & 1;
          const float2 cf = *reinterpret_cast<const float2*>(cw + cc + i);
          acc2[ql][pp] = ffma2(pack2(cf.x, cf.y),
                               pack2(fmaxf(__uint_as_float(v[i]), 0.f), fmaxf(__uint_as_float(v[i + 1]), 0.f)),
                               acc2[ql][pp]);
        }
        if (ph + 1 < NCH) tmem_ld_wait(vb[(ph + 1) & 1]);
      }
#pragma unroll
      for (int i = 0; i < C::QC; ++i) {
        if (i >= nq) continue;
        const float2 f0 = unpack2(acc2[i][0]);
        const float2 f1 = unpack2(acc2[i][1]);
        const float score = (f0.x + f0.y) + (f1.x + f1.y);
        const int r = ent[i].x;
        const long long pos = p.q_offset + (r % p.T);
        const bool vis = tok < p.L && tok <= pos;
        p.out[static_cast<long long>(r) * p.ldo + static_cast<long long>(ent[i].y) * p.blk + s.u * 128 + row] =
            vis ? score : -INFINITY;
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

// ------------------------------------------------------------------ inversion
// Kept blocks [rows, m] (block ids per sequence, -1 = empty slot) -> per
// block: count, list start, item start, and the (row, slot) list.

// Count the queries of every block; empty slots get -inf over their blk
// compact positions (no item writes them).
__global__ void invert_count_kernel(const int* __restrict__ blocks, long long rows, int m, int T, int M,
                                    int blk, int* __restrict__ cnt, float* __restrict__ out, long long ldo) {
  const long long n = rows * m;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = e / m;
    const int slot = static_cast<int>(e - r * m);
    const int jb = blocks[e];
    if (jb >= 0 && jb < M) {
      atomicAdd(cnt + (r / T) * M + jb, 1);
    } else {  // no block (or one past the sequence): no visible token
      float* o = out + r * ldo + static_cast<long long>(slot) * blk;
      for (int i = 0; i < blk; ++i) o[i] = -INFINITY;
    }
  }
}

// One CTA: exclusive prefix sums of the counts (list starts) and of the items
// per block (tiles x chunks); total items at ioff[nb]. Clears the cursors.
template <int NT>
__global__ void __launch_bounds__(NT) invert_scan_kernel(const int* __restrict__ cnt, int nb, int tiles,
                                                          int qc, int* __restrict__ qoff, int* __restrict__ ioff,
                                                          int* __restrict__ cursor, long long* __restrict__ total) {
  __shared__ int wsum[2][NT / 32];
  __shared__ int carry[2];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (threadIdx.x == 0) { carry[0] = 0; carry[1] = 0; }
  __syncthreads();
  for (int base = 0; base < nb; base += NT) {
    const int g = base + static_cast<int>(threadIdx.x);
    const int c = g < nb ? cnt[g] : 0;
    const int it = tiles * ((c + qc - 1) / qc);
    int a = c, bi = it;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, a, o);
      const int yb = __shfl_up_sync(0xffffffffu, bi, o);
      if (lane >= o) { a += ya; bi += yb; }
    }
    if (lane == 31) { wsum[0][wid] = a; wsum[1][wid] = bi; }
    __syncthreads();
    int pa = carry[0], pb = carry[1];
    for (int w2 = 0; w2 < wid; ++w2) { pa += wsum[0][w2]; pb += wsum[1][w2]; }
    if (g < nb) {
      qoff[g] = pa + a - c;
      ioff[g] = pb + bi - it;
      cursor[g] = 0;
    }
    __syncthreads();
    if (threadIdx.x == NT - 1) { carry[0] = pa + a; carry[1] = pb + bi; }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    qoff[nb] = carry[0];
    ioff[nb] = carry[1];
    *total = carry[1];
  }
}

// Scatter every kept (row, slot) into its block's list.
__global__ void invert_fill_kernel(const int* __restrict__ blocks, long long rows, int m, int T, int M,
                                   const int* __restrict__ qoff, int* __restrict__ cursor,
                                   int2* __restrict__ list) {
  const long long n = rows * m;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int jb = blocks[e];
    if (jb < 0 || jb >= M) continue;
    const long long r = e / m;
    const int g = static_cast<int>((r / T) * M + jb);
    const int at = atomicAdd(cursor + g, 1);
    list[qoff[g] + at] = make_int2(static_cast<int>(r), static_cast<int>(e - r * m));
  }
}

}  // namespace dsa
