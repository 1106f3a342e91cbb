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
// its queries), one record each (key tile, query rows, slots) built after the
// inversion; a CTA takes a contiguous range of items and every role reads
// their records 32 at a time; all items cost one MMA tile.
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
  const float* q_scale;     // [batch*T, H] (FP8) or nullptr
  const float* k_scale;     // [batch*L] (FP8) or nullptr
  float* out;               // [batch*T, ldo] compact rows: position slot * blk + i
  long long ldo;
  const int* it_tile;       // [items] key tile of item i: g * (blk / 128) + u (g = b * M + j)
  const int4* it_row;       // [items] the item's query rows (-1 past its queries)
  const int4* it_slot;      // [items] their slots in the compact rows
  unsigned* err;
};

template <int ELEM_, int H_, int NSTAGE_>
struct InvCfg {
  static constexpr int ELEM = ELEM_;                     // bytes per element: 2 = bf16, 1 = e4m3
  static constexpr int D = 128, H = H_, NSTAGE = NSTAGE_;
  static constexpr int ROW_BYTES = D * ELEM;
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
  static constexpr uint32_t IDESC = umma_idesc(ELEM == 2 ? 1u : 0u, 128, NROWS);
  static constexpr int SMEM_K = 0;
  static constexpr int SMEM_Q = NKBUF * K_BYTES;
  static constexpr int SMEM_COEF = SMEM_Q + NSTAGE * Q_BYTES;   // per epilogue warp: NROWS coefficients
  static constexpr int SMEM_BAR = SMEM_COEF + EPIW * NROWS * 4;
  static constexpr int NBAR = 2 * NSTAGE + 2 * NKBUF + 2 * NACC + 1;
  static constexpr int SMEM_BYTES = SMEM_BAR + NBAR * 8 + 16 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// A warp's walk over this CTA's items [i0, i1). Lane l holds the records of
// items bbase + l (current batch) and bbase + 32 + l (next batch), loaded 32
// at a time with coalesced loads, so per item only shuffles remain. All 32
// lanes call cur() and advance() together.
struct ItemWalk {
  long long i, i0, i1, bbase;
  int tile_c, tile_n;
  int4 row_c, row_n, slot_c, slot_n;
  int prev_tile;
  // the current item (uniform over the warp after cur())
  int tile;
  int4 rows, slots;
  bool first, last;

  __device__ __forceinline__ void load(const InvParams& p, long long base, int& t, int4& r, int4& sl,
                                       bool with_slots) {
    const long long idx = base + (threadIdx.x & 31);
    t = -1;
    r = make_int4(-1, -1, -1, -1);
    sl = make_int4(0, 0, 0, 0);
    if (idx < i1) {
      t = __ldg(p.it_tile + idx);
      r = __ldg(p.it_row + idx);
      if (with_slots) sl = __ldg(p.it_slot + idx);
    }
  }
  __device__ __forceinline__ void init(const InvParams& p, long long total, bool with_slots) {
    const long long G = gridDim.x;
    i0 = i = total * blockIdx.x / G;
    i1 = total * (blockIdx.x + 1) / G;
    bbase = i0;
    prev_tile = -1;
    load(p, bbase, tile_c, row_c, slot_c, with_slots);
    load(p, bbase + 32, tile_n, row_n, slot_n, with_slots);
  }
  __device__ __forceinline__ void cur() {
    const int l = static_cast<int>(i - bbase);
    tile = __shfl_sync(0xffffffffu, tile_c, l);
    rows.x = __shfl_sync(0xffffffffu, row_c.x, l);
    rows.y = __shfl_sync(0xffffffffu, row_c.y, l);
    rows.z = __shfl_sync(0xffffffffu, row_c.z, l);
    rows.w = __shfl_sync(0xffffffffu, row_c.w, l);
    slots.x = __shfl_sync(0xffffffffu, slot_c.x, l);
    slots.y = __shfl_sync(0xffffffffu, slot_c.y, l);
    slots.z = __shfl_sync(0xffffffffu, slot_c.z, l);
    slots.w = __shfl_sync(0xffffffffu, slot_c.w, l);
    const int nl = __shfl_sync(0xffffffffu, l + 1 < 32 ? tile_c : tile_n, (l + 1) & 31);
    first = i == i0 || prev_tile != tile;
    last = nl != tile;  // -1 past the range
  }
  // query rows of item i + ahead (1 <= ahead <= 32); -1s past the range
  __device__ __forceinline__ int4 peek_rows(int ahead) const {
    const int l2 = static_cast<int>(i - bbase) + ahead;
    const bool in_c = l2 < 32;
    int4 v;
    v.x = __shfl_sync(0xffffffffu, in_c ? row_c.x : row_n.x, l2 & 31);
    v.y = __shfl_sync(0xffffffffu, in_c ? row_c.y : row_n.y, l2 & 31);
    v.z = __shfl_sync(0xffffffffu, in_c ? row_c.z : row_n.z, l2 & 31);
    v.w = __shfl_sync(0xffffffffu, in_c ? row_c.w : row_n.w, l2 & 31);
    if (i + ahead >= i1) v = make_int4(-1, -1, -1, -1);
    return v;
  }
  __device__ __forceinline__ void advance(const InvParams& p, bool with_slots, int step = 1) {
    prev_tile = tile;
    i += step;
    while (i - bbase >= 32) {
      bbase += 32;
      tile_c = tile_n;
      row_c = row_n;
      slot_c = slot_n;
      load(p, bbase + 32, tile_n, row_n, slot_n, with_slots);
    }
  }
};

__device__ __forceinline__ int item_row(const int4& r, int i) {
  return i == 0 ? r.x : i == 1 ? r.y : i == 2 ? r.z : r.w;
}

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

  const long long total = *total_items;
  ItemWalk s;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    s.init(p, total, false);
    uint32_t it = 0, gk = 0;
    bool ok = true;
    for (; s.i < s.i1; s.advance(p, false), ++it) {
      s.cur();
      if (lane == 0) {
        if (s.first) {
          const int kb_ = static_cast<int>(gk % C::NKBUF);
          if (!mbar_wait(kempty(kb_), ((gk / C::NKBUF) & 1u) ^ 1u, p.err)) {
            ok = false;
          } else {
            const int U = p.blk / 128;
            const int g = s.tile / U;
            const int b = g / p.M;
            const int row0 = b * p.L + (g - b * p.M) * p.blk + (s.tile - g * U) * 128;
            mbar_arrive_expect_tx(kfull(kb_), C::K_BYTES);
#pragma unroll
            for (int cb = 0; cb < C::KBLK; ++cb)
              tma_load_2d(s_k + kb_ * C::K_BYTES + cb * C::KROWS * 128, &tm_k, kfull(kb_), cb * (128 / C::ELEM),
                          row0);
            ++gk;
          }
        }
        const int stage = static_cast<int>(it % C::NSTAGE);
        if (ok && !mbar_wait(empty(stage), ((it / C::NSTAGE) & 1u) ^ 1u, p.err)) ok = false;
        if (ok) {
          int nq = 0;
#pragma unroll
          for (int i = 0; i < C::QC; ++i) nq += item_row(s.rows, i) >= 0;
          mbar_arrive_expect_tx(full(stage), static_cast<uint32_t>(nq * C::H * C::ROW_BYTES));
#pragma unroll
          for (int i = 0; i < C::QC; ++i) {
            const int r = item_row(s.rows, i);
            if (r < 0) continue;
#pragma unroll
            for (int cb = 0; cb < C::KBLK; ++cb)
              tma_load_2d(s_q + stage * C::Q_BYTES + cb * C::NROWS * 128 + i * C::H * 128, &tm_q, full(stage),
                          cb * (128 / C::ELEM), r * C::H);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
    }
    if (!ok && lane == 0) {
      // error path: the loads already issued land before shared memory is released
      for (uint32_t g2 = gk > C::NKBUF ? gk - C::NKBUF : 0; g2 < gk; ++g2)
        mbar_drain(kfull(static_cast<int>(g2 % C::NKBUF)), (g2 / C::NKBUF) & 1u);
      const uint32_t lo = it > C::NSTAGE ? it - C::NSTAGE : 0;
      for (uint32_t i = lo; i < it; ++i) mbar_drain(full(i % C::NSTAGE), (i / C::NSTAGE) & 1u);
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    s.init(p, total, false);
    uint32_t it = 0, gk = 0;
    bool ok = true;
    for (; s.i < s.i1; s.advance(p, false), ++it) {
      s.cur();
      if (lane == 0) {
        const int kb_ = static_cast<int>(gk % C::NKBUF);
        const int stage = static_cast<int>(it % C::NSTAGE);
        const int buf = static_cast<int>(it % C::NACC);
        if (s.first && !mbar_wait(kfull(kb_), (gk / C::NKBUF) & 1u, p.err)) ok = false;
        if (ok && !mbar_wait(tempty(buf), ((it / C::NACC) & 1u) ^ 1u, p.err)) ok = false;
        if (ok && !mbar_wait(full(stage), (it / C::NSTAGE) & 1u, p.err)) ok = false;
        if (ok) {
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * C::NROWS);
#pragma unroll
          for (int ks = 0; ks < C::NKSTEP; ++ks) {
            const int cb = (ks * 32) / 128;
            const int inner = (ks * 32) % 128;
            const uint64_t adesc = umma_desc_sw128(s_k + kb_ * C::K_BYTES + cb * C::KROWS * 128 + inner);
            const uint64_t bdesc = umma_desc_sw128(s_q + stage * C::Q_BYTES + cb * C::NROWS * 128 + inner);
            if (C::ELEM == 2) mma_bf16(d_tmem, adesc, bdesc, C::IDESC, ks > 0 ? 1u : 0u);
            else mma_f8(d_tmem, adesc, bdesc, C::IDESC, ks > 0 ? 1u : 0u);
          }
          tc_commit(empty(stage));
          tc_commit(tfull(buf));
          if (s.last) { tc_commit(kempty(kb_)); ++gk; }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
    }
    if (!ok && lane == 0) {
      tc_commit(mdone);
      mbar_drain(mdone, 0);
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
    s.init(p, total, true);
    // lane l stages coefficients 4l .. 4l+3 of an item (of its query 4l / H;
    // columns of missing queries take the item's first query's, their sums
    // are never stored); the loads for the set's next item are issued while
    // the current item is processed
    const int c0 = 4 * lane;
    auto coef_load = [&](const int4& rows) {
      int r = item_row(rows, c0 / C::H);
      if (r < 0) r = rows.x;
      if (r < 0) return make_float4(0.f, 0.f, 0.f, 0.f);  // no such item
      const long long ci = static_cast<long long>(r) * C::H + (c0 % C::H);
      float4 wv = __ldg(reinterpret_cast<const float4*>(p.w + ci));
      if (C::ELEM == 1) {  // FP8: w * q_scale
        const float4 qs = __ldg(reinterpret_cast<const float4*>(p.q_scale + ci));
        wv.x *= qs.x; wv.y *= qs.y; wv.z *= qs.z; wv.w *= qs.w;
      }
      return wv;
    };
    // the two sets take alternate items: this set walks items i0 + set,
    // i0 + set + 2, ...
    if (set == 1) s.advance(p, true);
    float4 wnext = make_float4(0.f, 0.f, 0.f, 0.f);
    if (s.i < s.i1) {
      s.cur();
      wnext = coef_load(s.rows);
    }
    for (; s.i < s.i1; s.advance(p, true, 2)) {
      s.cur();
      const uint32_t it = static_cast<uint32_t>(s.i - s.i0);
      const int buf = static_cast<int>(it % C::NACC);
      const int U = p.blk / 128;
      const int g = s.tile / U;
      const int u = s.tile - g * U;
      const int j = g - (g / p.M) * p.M;
      *reinterpret_cast<float4*>(cw + c0) = wnext;
      __syncwarp();
      wnext = coef_load(s.peek_rows(2));
      const int tok = j * p.blk + u * 128 + row;  // token of this lane's key in its sequence
      float kscale = 1.f;  // FP8: this key's dequant scale
      if (C::ELEM == 1 && tok < p.L) kscale = __ldg(p.k_scale + static_cast<long long>(g / p.M) * p.L + tok);
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
        const int r = item_row(s.rows, i);
        if (r < 0) continue;
        const float2 f0 = unpack2(acc2[i][0]);
        const float2 f1 = unpack2(acc2[i][1]);
        const float score = ((f0.x + f0.y) + (f1.x + f1.y)) * kscale;
        const long long pos = p.q_offset + (r % p.T);
        const bool vis = tok < p.L && tok <= pos;
        p.out[static_cast<long long>(r) * p.ldo + static_cast<long long>(item_row(s.slots, i)) * p.blk + u * 128 +
              row] = vis ? score : -INFINITY;
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

// Exclusive prefix sums of the counts (list starts) and of the items per
// block (tiles x chunks); total items at ioff[nb]. Clears the cursors.
// CTA c scans blocks [4 NT c, 4 NT (c + 1)) (each thread 4 consecutive
// blocks, loads and stores coalesced); the sum of all blocks before its range
// it adds up itself (a coalesced read of at most nb counts), so the CTAs need
// no communication. The last CTA writes the totals.
template <int NT>
__global__ void __launch_bounds__(NT) invert_scan_kernel(const int* __restrict__ cnt, int nb, int tiles,
                                                          int qc, int* __restrict__ qoff, int* __restrict__ ioff,
                                                          int* __restrict__ cursor, long long* __restrict__ total) {
  __shared__ int wsum[2][NT / 32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int base = blockIdx.x * 4 * NT;
  // 1. sum of the blocks before this CTA's range
  int pa = 0, pb = 0;
  for (int g = static_cast<int>(threadIdx.x); g < base; g += NT) {
    const int c = cnt[g];
    pa += c;
    pb += tiles * ((c + qc - 1) / qc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    pa += __shfl_xor_sync(0xffffffffu, pa, o);
    pb += __shfl_xor_sync(0xffffffffu, pb, o);
  }
  if (lane == 0) { wsum[0][wid] = pa; wsum[1][wid] = pb; }
  __syncthreads();
  int carry_a = 0, carry_b = 0;
#pragma unroll 4
  for (int w = 0; w < NT / 32; ++w) { carry_a += wsum[0][w]; carry_b += wsum[1][w]; }
  __syncthreads();  // wsum is reused below
  // 2. this CTA's range: 4 consecutive blocks per thread
  const int g0 = base + 4 * static_cast<int>(threadIdx.x);
  int c[4], it[4];
  int sa = 0, sb = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    c[u] = g0 + u < nb ? cnt[g0 + u] : 0;
    it[u] = tiles * ((c[u] + qc - 1) / qc);
    sa += c[u];
    sb += it[u];
  }
  int a = sa, bi = sb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, a, o);
    const int yb = __shfl_up_sync(0xffffffffu, bi, o);
    if (lane >= o) { a += ya; bi += yb; }
  }
  if (lane == 31) { wsum[0][wid] = a; wsum[1][wid] = bi; }
  __syncthreads();
  if (wid == 0) {
    int wa = lane < NT / 32 ? wsum[0][lane] : 0;
    int wb = lane < NT / 32 ? wsum[1][lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, wa, o);
      const int yb = __shfl_up_sync(0xffffffffu, wb, o);
      if (lane >= o) { wa += ya; wb += yb; }
    }
    if (lane < NT / 32) { wsum[0][lane] = wa; wsum[1][lane] = wb; }
  }
  __syncthreads();
  int xa = carry_a + (wid > 0 ? wsum[0][wid - 1] : 0) + a - sa;   // exclusive start of this thread's 4
  int xb = carry_b + (wid > 0 ? wsum[1][wid - 1] : 0) + bi - sb;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    if (g0 + u < nb) {
      qoff[g0 + u] = xa;
      ioff[g0 + u] = xb;
      cursor[g0 + u] = 0;
    }
    xa += c[u];
    xb += it[u];
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) {
    const int ta = carry_a + wsum[0][NT / 32 - 1], tb = carry_b + wsum[1][NT / 32 - 1];
    qoff[nb] = ta;
    ioff[nb] = tb;
    *total = tb;
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

// Item records: one warp per block g; item loc of the block is (key tile
// u = loc / nch, chunk c = loc % nch) and holds queries c*QC .. c*QC+QC-1 of
// the block's list.
__global__ void invert_items_kernel(const int* __restrict__ cnt, const int* __restrict__ qoff,
                                    const int* __restrict__ ioff, const int2* __restrict__ list, int nb, int U,
                                    int qc, int* __restrict__ it_tile, int4* __restrict__ it_row,
                                    int4* __restrict__ it_slot) {
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (g >= nb) return;
  const int nq = cnt[g];
  const int nch = (nq + qc - 1) / qc;
  const int base = ioff[g];
  const int q0 = qoff[g];
  for (int loc = lane; loc < U * nch; loc += 32) {
    const int u = loc / nch;
    const int c = loc - u * nch;
    int rr[4] = {-1, -1, -1, -1}, ss[4] = {0, 0, 0, 0};
    for (int i = 0; i < qc && i < 4; ++i) {
      const int q = c * qc + i;
      if (q < nq) {
        const int2 e = list[q0 + q];
        rr[i] = e.x;
        ss[i] = e.y;
      }
    }
    it_tile[base + loc] = g * U + u;
    it_row[base + loc] = make_int4(rr[0], rr[1], rr[2], rr[3]);
    it_slot[base + loc] = make_int4(ss[0], ss[1], ss[2], ss[3]);
  }
}

}  // namespace dsa
