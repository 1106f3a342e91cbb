// Exact per-row top-k over fp32 scores (lightning-indexer token selection:
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// section "Problem statement"; "DoSA: Dots Sparse Attention", Top-K selection).
//
// Selection rule: the k largest scores of a row, ties broken toward the lower
// position; -inf marks an absent candidate; rows with fewer than k candidates
// return all of them. Output: selected positions in ascending order (mapped
// through an optional index map), padded with -1 (score -inf).
//
// Scores map to order-preserving 32-bit keys (-0 folded onto +0, absent -> 0)
// where integer order is needed; elsewhere scores are compared as floats
// (which already treat -0 and +0 as equal).
//
// Work split: a CTA (256 or 512 threads) owns one row at a time and several
// CTAs share an SM, so the barriers and latencies of one row overlap the work
// of others. Rows are read from global memory (the sampling read brings a row
// into L2, the band pass reads it from there). Per row:
//   1. every S-th score is sampled (S a power of two, at most 4096 samples);
//      a 2048-bin value histogram of the sample (bins evenly spaced between
//      the sample's min and max) brackets the k-th score in a band
//      [t_lo, t_hi] wide enough (4 standard deviations of the sample rank on
//      each side) that the k-th score lies inside with near certainty;
//   2. one pass over the row, 4 consecutive scores per lane: bitmap words of
//      "score > t_hi" and of "score in the band" (nibbles OR-ed over 8 lanes);
//   3. the band's entries go to one candidate list in position order (each
//      warp writes its segment's entries at its prefix offset);
//   4. an exact three-digit radix select (11 + 11 + 10 bits, digits on which
//      t_lo and t_hi agree skipped) over the candidates gives tau and how
//      many scores equal to tau to take; the selected candidates are OR-ed
//      into the "> t_hi" bitmap;
//   5. the bitmap is emitted in position order (per-lane popcounts, prefix
//      sums over lanes and warps); the positions are collected in shared
//      memory and written out with coalesced stores.
// If a check fails (unlucky sample, mass ties, a full candidate list, fewer
// present scores than k, rows longer than the bitmap), the row falls back to
// a full value histogram, an exact select over the k-th value's bin (or the
// whole row), a counting pass and an ordered write pass.
#pragma once
#include "common.cuh"

namespace dsa {

struct TopkParams {
  const float* scores;   // [rows, ld]
  long long ld;
  long long rows;
  int T;                 // row r belongs to query t = r % T
  long long q_offset;
  int pstride;           // > 0: row length = clamp((q_offset + t) / pstride + 1, 0, Lrow); 0: Lrow
  int Lrow;
  int k;
  int32_t* out_idx;      // [rows, k]
  float* out_score;      // [rows, k] or nullptr
  const int* cand;       // optional map: position j -> cand[r * n_slots + j / blk] * blk + j % blk
  int n_slots, blk;
  unsigned* err;         // device status word (unused: the kernel has no waits)
  // Optional candidate lists written by the score pass (every visible score
  // >= a per-row threshold): row r's entries (value, position) fill slots
  // [0, cres[r]) of cval / cidx[r * ccap + i], unused slots hold (-inf, -1);
  // creal[r] counts the real ones. When a row holds at least min(k, n) real
  // entries and cres[r] <= ccap, its top-k lies among them and the row's full
  // scores are not read.
  const float* cval;
  const int* cidx;
  const int* cres;
  const int* creal;
  int ccap;
};

constexpr int TK_BINS = 2048;        // histogram bins (11-bit digits, value bins)
constexpr int TK_SAMPLE = 4096;      // samples per row at most

// Shared-memory layout (32-bit words) of one CTA. BMW bitmap words: rows of
// up to 32 * BMW scores take the band path; CAP band candidates.
template <int BMW_, int CAP_, int UB_, int NT_, int MINC_>
struct TkCfg {
  static constexpr int BMW = BMW_;
  static constexpr int CAP = CAP_;
  static constexpr int UB = UB_;  // float4 loads in flight per lane in the band pass
  static constexpr int NT = NT_;  // threads per CTA (one row at a time)
  static constexpr int NW = NT / 32;
  static constexpr int MAX_ROW = 32 * BMW;
  static constexpr int W_HIST = 0;                                       // TK_BINS
  static constexpr int W_WS = W_HIST + TK_BINS;                          // 64 scratch
  static constexpr int W_VARS = W_WS + 64;                               // 64 row variables
  static constexpr int W_SAMP = W_VARS + 64;                             // sample, then band bitmap
  static constexpr int W_BMAP = W_SAMP + (TK_SAMPLE > BMW ? TK_SAMPLE : BMW);  // "> t_hi" bitmap
  static constexpr int W_KEY = W_BMAP + BMW;                             // CAP candidate keys
  static constexpr int W_POS = W_KEY + CAP;                              // CAP candidate positions
  static constexpr int WORDS = W_POS + CAP;
  static constexpr int BYTES = WORDS * 4;
  static constexpr int OUT_CAP = 2 * CAP;  // output positions staged in the key + position space
  static constexpr int MIN_CTAS = MINC_;  // CTAs per SM the register budget is sized for
  // Sample layout. Rows of up to 32768 scores: every S-th score, which
  // touches every 32-byte sector of the row, so the sampling read brings the
  // row into L2 for the band pass. Longer rows: runs of 32 consecutive
  // scores every 32 S (a few KB of the row), since the rows in flight of a
  // long-row launch do not fit in L2 and a row sampled into L2 would be
  // evicted before its band pass and read from HBM twice.
#ifndef DSA_TK_RUNS
#define DSA_TK_RUNS 1
#endif
  static constexpr bool RUN_SAMPLE = DSA_TK_RUNS && BMW_ > 1024;
  static_assert(MINC_ * (BYTES + 1024) <= 228 * 1024, "shared memory for MIN_CTAS CTAs per SM");
};
using TkShort = TkCfg<1024, 2048, 4, 256, 4>;  // rows up to 32768: 44.5 KB, 4 CTAs per SM
using TkLong = TkCfg<4096, 6144, 4, 512, 2>;   // rows up to 131072: 88.5 KB, 2 CTAs per SM
using TkWide = TkCfg<4096, 6144, 8, 512, 1>;   // as TkLong, one wider CTA per row for launches with few rows
using TkShortWide = TkCfg<1024, 2048, 8, 512, 1>;  // as TkShort, one wider CTA per row for launches with few rows

__device__ __forceinline__ uint32_t score_key(float x) {
  if (!(x > -INFINITY)) return 0u;  // -inf (absent) and NaN
  if (x == 0.f) x = 0.f;            // -0 -> +0
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ bool present(float x) { return x > -INFINITY; }  // false for -inf, NaN

// Value bin of a present score: TK_BINS evenly spaced bins over [lo, lo + TK_BINS/scale].
// For x in [lo, hi], (x - lo) * scale >= 0; adding 1.5 * 2^23 leaves round-to-nearest(v) in the low
// mantissa bits (a monotone map, no float-to-int conversion instruction).
// scale == 0 (all scores equal, or a span that overflows) puts everything in bin 0.
__device__ __forceinline__ int value_bin(float x, float lo, float scale) {
  const float v = (scale > 0.f ? (x - lo) * scale : 0.f) + 12582912.0f;
  const int b = __float_as_int(v) - 0x4B400000;
  return min(max(b, 0), TK_BINS - 1);  // scores outside [lo, hi] land in the end bins
}

// ---------------------------------------------------------------- block helpers
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}
__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exclusive prefix sum over the CTA's NT threads in thread order; `total`
// gets the sum. Uses ws[0 .. NT/32); ends with the CTA synchronised.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* ws, uint32_t& total) {
  constexpr int TK_NW = NT / 32;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const uint32_t inc = warp_incl_scan(v);
  if (lane == 31) ws[wid] = inc;
  __syncthreads();
  const uint32_t wv = lane < TK_NW ? ws[lane] : 0u;
  const uint32_t winc = warp_incl_scan(wv);
  const uint32_t before = __shfl_sync(0xffffffffu, winc - wv, wid);
  total = __shfl_sync(0xffffffffu, winc, TK_NW - 1);
  __syncthreads();
  return before + inc - v;
}

// Histogram of TK_BINS bins, 1-based rank `need` counted from the top: the
// bin holding that rank -> vars[0], the rank inside it -> vars[1] (vars[0]
// untouched when the histogram holds fewer than `need` entries).
template <int NT>
__device__ __forceinline__ void radix_pick(const uint32_t* hist, uint32_t need, uint32_t* ws,
                                           uint32_t* vars) {
  constexpr int BPT = TK_BINS / NT;
  const int u = NT - 1 - static_cast<int>(threadIdx.x);  // owner of bins [u*BPT, (u+1)*BPT)
  uint32_t c[BPT];
  uint32_t loc = 0;
#pragma unroll
  for (int i = 0; i < BPT; ++i) { c[i] = hist[u * BPT + i]; loc += c[i]; }
  uint32_t tot;
  uint32_t above = block_excl_scan<NT>(loc, ws, tot);  // entries in the bins of owners > u
#pragma unroll
  for (int i = BPT - 1; i >= 0; --i) {
    if (above < need && need <= above + c[i]) {
      vars[0] = static_cast<uint32_t>(u * BPT + i);
      vars[1] = need - above;
    }
    above += c[i];
  }
  __syncthreads();
}

// Exact radix select: the need-th largest of the keys (0 = absent, ignored)
// given by key_at(i), i in [0, n). Digits before d0 are known to equal the
// top bits of prefix0 for every key. Leaves vars[0] = tau and vars[1] = how
// many keys equal to tau rank within the top `need`.
template <int NT, class KeyAt>
__device__ void exact_select(const KeyAt& key_at, int n, uint32_t need, uint32_t* hist, uint32_t* ws,
                             uint32_t* vars, int d0 = 0, uint32_t prefix0 = 0) {
  uint32_t prefix = prefix0;
#pragma unroll 1
  for (int d = d0; d < 3; ++d) {
    const int sh = d == 0 ? 21 : (d == 1 ? 10 : 0);
    const uint32_t width = d == 2 ? 10u : 11u;
    const uint32_t hi_sh = sh + width;
    for (int i = threadIdx.x; i < TK_BINS; i += NT) hist[i] = 0;
    __syncthreads();
#pragma unroll 4
    for (int i = threadIdx.x; i < n; i += NT) {
      const uint32_t key = key_at(i);
      if (key != 0u && (hi_sh >= 32 || (key >> hi_sh) == prefix))
        atomicAdd(&hist[(key >> sh) & ((1u << width) - 1u)], 1u);
    }
    __syncthreads();
    radix_pick<NT>(hist, need, ws, vars);
    prefix = (prefix << width) | vars[0];
    need = vars[1];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    vars[0] = prefix;
    vars[1] = need;
  }
  __syncthreads();
}

// Entries i .. i+3 (i a multiple of 4) of a global row, -inf from `end` on;
// one vector load when all four exist and the row start is 16-byte aligned.
__device__ __forceinline__ float4 load4(const float* row, int i, int end, bool vec) {
  if (vec && i + 3 < end) return __ldcg(reinterpret_cast<const float4*>(row + i));
  float4 v = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
  if (i < end) v.x = __ldcg(row + i);
  if (i + 1 < end) v.y = __ldcg(row + i + 1);
  if (i + 2 < end) v.z = __ldcg(row + i + 2);
  if (i + 3 < end) v.w = __ldcg(row + i + 3);
  return v;
}

__device__ __forceinline__ int map_index(const TopkParams& p, long long r, int i) {
  if (!p.cand) return i;
  const int slot = i / p.blk;
  return __ldg(p.cand + r * p.n_slots + slot) * p.blk + (i - slot * p.blk);
}

// Write the positions set in the bitmap words [l0, l1) of each thread (the
// ranges ordered by thread) in ascending order: per-thread popcounts, a
// prefix over the CTA, then the positions (staged in shared memory when they
// fit, for coalesced stores) mapped through the index map; scores re-read
// from the row. keff positions in all.
template <class C>
__device__ void emit_bitmap(const TopkParams& p, uint32_t* sm, long long r, int l0, int l1, uint32_t keff,
                            const float* row) {
  uint32_t* ws = sm + C::W_WS;
  const uint32_t* bmap = sm + C::W_BMAP;
  uint32_t* obuf = sm + C::W_KEY;  // key + position space (no longer read)
  uint32_t cnt = 0;
  for (int wd = l0; wd < l1; ++wd) cnt += __popc(bmap[wd]);
  uint32_t tot;
  uint32_t out = block_excl_scan<C::NT>(cnt, ws, tot);  // threads in order = positions in order
  int32_t* oi = p.out_idx + r * p.k;
  float* os = p.out_score ? p.out_score + r * p.k : nullptr;
  const bool via_smem = keff <= static_cast<uint32_t>(C::OUT_CAP);
  for (int wd = l0; wd < l1; ++wd) {
    uint32_t bits = bmap[wd];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1u;
      const int i = wd * 32 + b;
      if (out < keff) {  // holds by construction; guards the row
        if (via_smem) {
          obuf[out] = static_cast<uint32_t>(i);
        } else {
          oi[out] = map_index(p, r, i);
          if (os) { const float x = __ldcg(row + i); os[out] = x == 0.f ? 0.f : x; }
        }
      }
      ++out;
    }
  }
  if (via_smem) {
    __syncthreads();
    for (int j = threadIdx.x; j < static_cast<int>(keff); j += C::NT) {
      const int i = static_cast<int>(obuf[j]);
      oi[j] = map_index(p, r, i);
      if (os) { const float x = __ldcg(row + i); os[j] = x == 0.f ? 0.f : x; }
    }
  }
}

// ---------------------------------------------------------------- band path
// Returns false (nothing written) when the row must take the fallback.
template <class C>
__device__ bool topk_row_band(const TopkParams& p, uint32_t* sm, long long r, int n, const float* row,
                              uint32_t& keff_out) {
  constexpr int TK_NT = C::NT, TK_NW = C::NW;
  uint32_t* hist = sm + C::W_HIST;
  uint32_t* ws = sm + C::W_WS;
  uint32_t* vars = sm + C::W_VARS;
  float* fsamp = reinterpret_cast<float*>(sm + C::W_SAMP);
  uint32_t* bbm = sm + C::W_SAMP;  // band bitmap, once the sample is consumed
  uint32_t* bmap = sm + C::W_BMAP;
  uint32_t* lkey = sm + C::W_KEY;
  uint32_t* lpos = sm + C::W_POS;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int k = p.k;

  // ---- 1. sample: present count, min / max, value histogram -> band
  int S = 4;
  while (static_cast<long long>(S) * TK_SAMPLE < n) S <<= 1;
  const int ns = (n + S - 1) / S;
  for (int i = tid; i < TK_BINS; i += TK_NT) hist[i] = 0;
  uint32_t nsv = 0;
  float vmin = INFINITY, vmax = -INFINITY;
  // eight samples per thread in flight: all loads first, then their uses
  for (int m0 = tid; m0 < ns; m0 += 8 * TK_NT) {
    float xs[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int m = m0 + u * TK_NT;
      const long long pos = C::RUN_SAMPLE ? static_cast<long long>(m >> 5) * (32 * S) + (m & 31)
                                          : static_cast<long long>(m) * S;
      xs[u] = (m < ns && pos < n) ? __ldcg(row + pos) : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int m = m0 + u * TK_NT;
      if (m < ns) fsamp[m] = xs[u];
      if (present(xs[u])) { ++nsv; vmin = fminf(vmin, xs[u]); vmax = fmaxf(vmax, xs[u]); }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    nsv += __shfl_xor_sync(0xffffffffu, nsv, o);
    vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  }
  float* fws = reinterpret_cast<float*>(ws);
  if (lane == 0) { ws[wid] = nsv; fws[16 + wid] = vmin; fws[32 + wid] = vmax; }
  __syncthreads();
  {
    const bool has = lane < TK_NW;
    uint32_t a = has ? ws[lane] : 0u;
    float mn = has ? fws[16 + lane] : INFINITY;
    float mx = has ? fws[32 + lane] : -INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    nsv = a; vmin = mn; vmax = mx;
  }
  const float span = vmax - vmin;
  const float scale = (span > 0.f && span < INFINITY) ? static_cast<float>(TK_BINS - 1) / span : 0.f;
  for (int m = tid; m < ns; m += TK_NT) {
    const float x = fsamp[m];
    if (present(x)) atomicAdd(&hist[value_bin(x, vmin, scale)], 1u);
  }
  if (tid == 0) { vars[12] = TK_BINS; vars[13] = 0; }
  __syncthreads();
  // expected rank of the k-th score inside the sample, +- 4 standard deviations
  const float nsvf = static_cast<float>(nsv);
  const float pr = fminf(1.f, static_cast<float>(k) / fmaxf(1.f, nsvf * static_cast<float>(S)));
  const float center = pr * nsvf;
  const float delta = 4.f * sqrtf(nsvf * pr * (1.f - pr)) + 4.f;
  const int r_hi = static_cast<int>(floorf(center - delta));
  const int r_lo = static_cast<int>(ceilf(center + delta));
  {
    constexpr int BPT = TK_BINS / TK_NT;
    const int u = TK_NT - 1 - tid;  // owner of bins [u*BPT, (u+1)*BPT)
    uint32_t c[BPT];
    uint32_t loc = 0;
#pragma unroll
    for (int q = 0; q < BPT; ++q) { c[q] = hist[u * BPT + q]; loc += c[q]; }
    uint32_t tot;
    long long above = block_excl_scan<TK_NT>(loc, ws, tot);
#pragma unroll
    for (int q = BPT - 1; q >= 0; --q) {
      if (r_hi >= 1 && above < r_hi && r_hi <= above + c[q]) vars[12] = u * BPT + q;
      if (r_lo <= static_cast<int>(tot) && above < r_lo && r_lo <= above + c[q]) vars[13] = u * BPT + q;
      above += c[q];
    }
    __syncthreads();
  }
  const int b_hi = static_cast<int>(vars[12]);
  const int b_lo = static_cast<int>(vars[13]);
  const float t_hi = (b_hi >= TK_BINS - 1 || scale == 0.f) ? INFINITY
                                                          : vmin + (static_cast<float>(b_hi) + 0.5f) / scale;
  const float t_lo = (b_lo <= 0 || scale == 0.f) ? -INFINITY
                                                 : vmin + (static_cast<float>(b_lo) - 0.5f) / scale;
  const float t_lo_p = t_lo > -INFINITY ? t_lo : -3.402823466e+38f;  // x >= t_lo_p: present and in band

  // ---- 2. band pass: "> t_hi" and band bitmap words, 4 scores per lane
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
  const int seg = ((n + TK_NW * 128 - 1) / (TK_NW * 128)) * 128;  // warp segments, multiples of 128
  const int s0 = min(n, wid * seg);
  const int s1 = min(n, s0 + seg);
  uint32_t c_above = 0;
  for (int base = s0; base < s1; base += 128 * C::UB) {
    float4 xv[C::UB];
#pragma unroll
    for (int j = 0; j < C::UB; ++j) xv[j] = load4(row, base + 128 * j + 4 * lane, s1, vec);
#pragma unroll
    for (int j = 0; j < C::UB; ++j) {
      const int i4 = base + 128 * j + 4 * lane;
      const float4 x = xv[j];
      const uint32_t nib = static_cast<uint32_t>(x.x > t_hi) | (static_cast<uint32_t>(x.y > t_hi) << 1) |
                           (static_cast<uint32_t>(x.z > t_hi) << 2) | (static_cast<uint32_t>(x.w > t_hi) << 3);
      const uint32_t bnib =
          (static_cast<uint32_t>(x.x >= t_lo_p) | (static_cast<uint32_t>(x.y >= t_lo_p) << 1) |
           (static_cast<uint32_t>(x.z >= t_lo_p) << 2) | (static_cast<uint32_t>(x.w >= t_lo_p) << 3)) &
          ~nib;
      c_above += __popc(nib);
      uint32_t word = nib << (4 * (lane & 7));
      uint32_t bword = bnib << (4 * (lane & 7));
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        word |= __shfl_xor_sync(0xffffffffu, word, o);
        bword |= __shfl_xor_sync(0xffffffffu, bword, o);
      }
      if ((lane & 7) == 0 && i4 < s1) { bmap[i4 >> 5] = word; bbm[i4 >> 5] = bword; }
    }
  }
  __syncwarp();
  // this warp's words and band count
  const int w0 = s0 >> 5;
  const int w1 = s1 > s0 ? (s1 + 31) >> 5 : w0;
  uint32_t c_band = 0;
  for (int wd = w0 + lane; wd < w1; wd += 32) c_band += __popc(bbm[wd]);
  c_above = warp_sum(c_above);
  c_band = warp_sum(c_band);
  if (lane == 0) { ws[wid] = c_above; ws[16 + wid] = c_band; }
  __syncthreads();
  uint32_t above_all, nc, band_before;
  {
    const uint32_t a = lane < TK_NW ? ws[lane] : 0u;
    const uint32_t bc = lane < TK_NW ? ws[16 + lane] : 0u;
    above_all = warp_sum(a);
    const uint32_t binc = warp_incl_scan(bc);
    nc = __shfl_sync(0xffffffffu, binc, TK_NW - 1);
    band_before = __shfl_sync(0xffffffffu, binc - bc, wid);
  }
  // with t_lo = -inf the present entries are exactly above + band
  const uint32_t keff =
      t_lo > -INFINITY ? static_cast<uint32_t>(k) : min(static_cast<uint32_t>(k), above_all + nc);
  const bool band_ok = nc <= static_cast<uint32_t>(C::CAP) && above_all < keff && keff <= above_all + nc;
  __syncthreads();
  if (!band_ok) return false;

  // ---- 3. band entries -> candidate list, in position order. A lane
  // takes a contiguous run of the warp's words; the scores of its entries are
  // re-read from L2 eight loads at a time.
  {
    const int per = (w1 - w0 + 31) / 32;
    const int l0 = min(w1, w0 + lane * per), l1 = min(w1, l0 + per);
    uint32_t cnt = 0;
    for (int wd = l0; wd < l1; ++wd) cnt += __popc(bbm[wd]);
    uint32_t slot = band_before + warp_incl_scan(cnt) - cnt;
    int wd = l0;
    uint32_t bits = wd < l1 ? bbm[wd] : 0u;
    while (true) {
      int pos[8];
      int m = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        while (!bits && wd + 1 < l1) bits = bbm[++wd];
        pos[u] = -1;
        if (bits) {
          pos[u] = wd * 32 + __ffs(bits) - 1;
          bits &= bits - 1u;
          ++m;
        }
      }
      if (m == 0) break;
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = pos[u] >= 0 ? __ldcg(row + pos[u]) : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (pos[u] >= 0) {
          lkey[slot] = score_key(v[u]);
          lpos[slot] = static_cast<uint32_t>(pos[u]);
          ++slot;
        }
      }
    }
  }
  __syncthreads();

  // ---- 4. exact select among the candidates. Every candidate lies in
  // [t_lo, t_hi]: digits on which both ends agree are skipped.
  int d0 = 0;
  uint32_t pre0 = 0;
  if (t_lo > -INFINITY && t_hi < INFINITY) {
    const uint32_t kl = score_key(t_lo), kh = score_key(t_hi);
    if ((kl >> 10) == (kh >> 10)) { d0 = 2; pre0 = kl >> 10; }
    else if ((kl >> 21) == (kh >> 21)) { d0 = 1; pre0 = kl >> 21; }
  }
  exact_select<TK_NT>([&](int i) { return lkey[i]; }, static_cast<int>(nc), keff - above_all, hist, ws, vars, d0,
               pre0);
  const uint32_t tau = vars[0];
  const uint32_t teq = vars[1];

  // selected candidates -> bitmap: keys above tau, and the first teq keys
  // equal to tau in position order (each thread takes a contiguous chunk)
  {
    const int chunk = (static_cast<int>(nc) + TK_NT - 1) / TK_NT;
    const int c0 = min(static_cast<int>(nc), tid * chunk), c1 = min(static_cast<int>(nc), c0 + chunk);
    uint32_t ceq = 0;
    for (int i = c0; i < c1; ++i) ceq += lkey[i] == tau;
    uint32_t tot;
    uint32_t rank = block_excl_scan<TK_NT>(ceq, ws, tot);
    for (int i = c0; i < c1; ++i) {
      const uint32_t key = lkey[i];
      bool take = key > tau;
      if (key == tau) { take = rank < teq; ++rank; }
      if (take) {
        const uint32_t pos = lpos[i];
        atomicOr(&bmap[pos >> 5], 1u << (pos & 31u));
      }
    }
  }
  __syncthreads();

  // ---- 5. emit the bitmap in position order
  const int per = (w1 - w0 + 31) / 32;  // words per lane (contiguous)
  const int l0 = min(w1, w0 + lane * per), l1 = min(w1, l0 + per);
  emit_bitmap<C>(p, sm, r, l0, l1, keff, row);
  keff_out = keff;
  return true;
}

// ---------------------------------------------------------------- candidate-list path
// The score pass appended every visible score >= the row's threshold to the
// row's candidate list, in no particular order. With at least min(k, n) of
// them (and none lost past the capacity) the row's k-th score is >= the
// threshold, so its top-k lies in the list: exact select of rank k over the
// candidates' score keys (unused slots hold -inf, key 0, and never count); if
// more scores equal the k-th than are taken, a second select over the
// inverted positions of those takes the lowest positions; the winners go into
// a position bitmap, emitted in order. Returns false (nothing written) when
// the row must use its full scores.
template <class C>
__device__ bool topk_row_compact(const TopkParams& p, uint32_t* sm, long long r, int n, const float* row,
                                 uint32_t& keff_out) {
  constexpr int TK_NT = C::NT;
  const int nc = __ldg(p.cres + r);
  const int keff_i = min(p.k, n);
  if (__ldg(p.creal + r) < keff_i || nc > p.ccap || n > C::MAX_ROW || n < 1) return false;
  uint32_t* hist = sm + C::W_HIST;
  uint32_t* ws = sm + C::W_WS;
  uint32_t* vars = sm + C::W_VARS;
  uint32_t* bmap = sm + C::W_BMAP;
  const int tid = threadIdx.x;
  const float* cv = p.cval + r * p.ccap;
  const int* ci = p.cidx + r * p.ccap;
  const uint32_t k = static_cast<uint32_t>(keff_i);
  exact_select<TK_NT>([&](int i) { return score_key(__ldcg(cv + i)); }, nc, k, hist, ws, vars);
  const uint32_t tau = vars[0];
  const uint32_t teq = vars[1];
  uint32_t neq = 0;
  for (int i = tid; i < nc; i += TK_NT) neq += score_key(__ldcg(cv + i)) == tau;
  uint32_t tot;
  block_excl_scan<TK_NT>(neq, ws, tot);
  const bool all_eq = tot == teq;
  uint32_t tau2 = 0;
  if (!all_eq) {
    exact_select<TK_NT>(
        [&](int i) { return score_key(__ldcg(cv + i)) == tau ? ~static_cast<uint32_t>(__ldcg(ci + i)) : 0u; },
        nc, teq, hist, ws, vars);
    tau2 = vars[0];
  }
  const int w1 = (n + 31) >> 5;
  for (int wd = tid; wd < w1; wd += TK_NT) bmap[wd] = 0u;
  __syncthreads();
  // The winners' scores go into the row's own buffer (library scratch that
  // the compacting score pass leaves unwritten), where the emit reads them.
  float* srow = const_cast<float*>(row);
  for (int i = tid; i < nc; i += TK_NT) {
    const float v = __ldcg(cv + i);
    const uint32_t key = score_key(v);
    const uint32_t pos = static_cast<uint32_t>(__ldcg(ci + i));
    const bool take = key > tau || (key == tau && (all_eq || ~pos >= tau2));
    if (take) {
      atomicOr(&bmap[pos >> 5], 1u << (pos & 31u));
      if (p.out_score) srow[pos] = v;
    }
  }
  __syncthreads();
  const int per = (w1 + TK_NT - 1) / TK_NT;
  const int l0 = min(w1, tid * per), l1 = min(w1, l0 + per);
  emit_bitmap<C>(p, sm, r, l0, l1, k, row);
  keff_out = k;
  return true;
}

// ---------------------------------------------------------------- fallback
// Any row: exact selection with a full value histogram, a counting pass and
// an ordered write pass.
template <class C>
__device__ void topk_row_fallback(const TopkParams& p, uint32_t* sm, long long r, int n, const float* row,
                                  uint32_t& keff_out) {
  constexpr int TK_NT = C::NT, TK_NW = C::NW;
  uint32_t* hist = sm + C::W_HIST;
  uint32_t* ws = sm + C::W_WS;
  uint32_t* vars = sm + C::W_VARS;
  uint32_t* ckey = sm + C::W_KEY;  // 2 * CAP words (keys and positions space)
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int k = p.k;

  uint32_t nv = 0;
  float vmin = INFINITY, vmax = -INFINITY;
  for (int i = tid; i < n; i += TK_NT) {
    const float x = __ldcg(row + i);
    if (present(x)) { ++nv; vmin = fminf(vmin, x); vmax = fmaxf(vmax, x); }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    nv += __shfl_xor_sync(0xffffffffu, nv, o);
    vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  }
  float* fws = reinterpret_cast<float*>(ws);
  if (lane == 0) { ws[wid] = nv; fws[16 + wid] = vmin; fws[32 + wid] = vmax; }
  __syncthreads();
  {
    const bool has = lane < TK_NW;
    uint32_t a = has ? ws[lane] : 0u;
    float mn = has ? fws[16 + lane] : INFINITY;
    float mx = has ? fws[32 + lane] : -INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    nv = a; vmin = mn; vmax = mx;
  }
  __syncthreads();
  const uint32_t keff = min(static_cast<uint32_t>(k), nv);
  float thr = -INFINITY;  // select score > thr, plus the first take_eq scores == thr
  uint32_t take_eq = 0;
  if (keff < nv) {
    const float span = vmax - vmin;
    const float scale = (span > 0.f && span < INFINITY) ? static_cast<float>(TK_BINS - 1) / span : 0.f;
    for (int i = tid; i < TK_BINS; i += TK_NT) hist[i] = 0;
    if (tid == 0) vars[10] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += TK_NT) {
      const float x = __ldcg(row + i);
      if (present(x)) atomicAdd(&hist[value_bin(x, vmin, scale)], 1u);
    }
    __syncthreads();
    radix_pick<TK_NT>(hist, keff, ws, vars);
    const int b = static_cast<int>(vars[0]);
    const uint32_t need = vars[1];
    const uint32_t cnt = hist[b];
    __syncthreads();
    if (cnt <= static_cast<uint32_t>(2 * C::CAP)) {
      for (int i = tid; i < n; i += TK_NT) {
        const float x = __ldcg(row + i);
        if (present(x) && value_bin(x, vmin, scale) == b) ckey[atomicAdd(&vars[10], 1u)] = score_key(x);
      }
      __syncthreads();
      exact_select<TK_NT>([&](int i) { return ckey[i]; }, static_cast<int>(cnt), need, hist, ws, vars);
    } else {
      exact_select<TK_NT>([&](int i) { return score_key(__ldcg(row + i)); }, n, keff, hist, ws, vars);
    }
    thr = key_score(vars[0]);
    take_eq = vars[1];
    __syncthreads();
  }
  // counting pass (per warp segment), prefix over the warps, ordered write
  const int seg = ((n + TK_NW * 128 - 1) / (TK_NW * 128)) * 128;
  const int s0 = min(n, wid * seg);
  const int s1 = min(n, s0 + seg);
  uint32_t cgt = 0, ceq = 0;
  for (int base = s0; base < s1; base += 128) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = base + 32 * j + lane;
      const float x = i < s1 ? __ldcg(row + i) : -INFINITY;
      cgt += x > thr;
      ceq += x == thr && present(x);
    }
  }
  cgt = warp_sum(cgt);
  ceq = warp_sum(ceq);
  if (lane == 0) { ws[wid] = cgt; ws[16 + wid] = ceq; }
  __syncthreads();
  uint32_t run_gt, run_eq;
  {
    const uint32_t g = lane < TK_NW ? ws[lane] : 0u;
    const uint32_t e = lane < TK_NW ? ws[16 + lane] : 0u;
    run_gt = __shfl_sync(0xffffffffu, warp_incl_scan(g) - g, wid);
    run_eq = __shfl_sync(0xffffffffu, warp_incl_scan(e) - e, wid);
  }
  __syncthreads();
  int32_t* oi = p.out_idx + r * p.k;
  float* os = p.out_score ? p.out_score + r * p.k : nullptr;
  for (int base = s0; base < s1; base += 128) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = base + 32 * j + lane;
      const float x = i < s1 ? __ldcg(row + i) : -INFINITY;
      const bool gt = x > thr;
      const bool eq = x == thr && present(x);
      const uint32_t mg = __ballot_sync(0xffffffffu, gt);
      const uint32_t me = __ballot_sync(0xffffffffu, eq);
      const uint32_t gb = run_gt + __popc(mg & lt_mask);
      const uint32_t eb = run_eq + __popc(me & lt_mask);
      if ((gt || (eq && eb < take_eq)) && gb + min(eb, take_eq) < static_cast<uint32_t>(k)) {
        const uint32_t pos = gb + min(eb, take_eq);
        oi[pos] = map_index(p, r, i);
        if (os) os[pos] = x == 0.f ? 0.f : x;
      }
      run_gt += __popc(mg);
      run_eq += __popc(me);
    }
  }
  keff_out = keff;
}

__device__ __forceinline__ int row_length(const TopkParams& p, long long r) {
  const int t = static_cast<int>(r % p.T);
  long long nl = p.Lrow;
  if (p.pstride > 0) {
    nl = (p.q_offset + t) / p.pstride + 1;
    if (nl > p.Lrow) nl = p.Lrow;
    if (nl < 0) nl = 0;
  }
  return static_cast<int>(nl);
}

template <class C>
__global__ void __launch_bounds__(C::NT, C::MIN_CTAS) topk_rows_kernel(const TopkParams p) {
  extern __shared__ uint32_t tk_smem[];
  for (long long r = blockIdx.x; r < p.rows; r += gridDim.x) {
    const int n = row_length(p, r);
    const float* row = p.scores + r * p.ld;
    uint32_t keff = 0;
    bool done = false;
    if (p.cres != nullptr) done = topk_row_compact<C>(p, tk_smem, r, n, row, keff);
    if (!done && n > p.k && n <= C::MAX_ROW) done = topk_row_band<C>(p, tk_smem, r, n, row, keff);
    if (!done) topk_row_fallback<C>(p, tk_smem, r, n, row, keff);
    int32_t* oi = p.out_idx + r * p.k;
    float* os = p.out_score ? p.out_score + r * p.k : nullptr;
    for (int j = static_cast<int>(keff) + threadIdx.x; j < p.k; j += C::NT) {
      oi[j] = -1;
      if (os) os[j] = -INFINITY;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- short rows
// Rows of at most NT * KPT scores (2048: 128 threads x 16 keys): one CTA per
// row (grid-stride over rows), KPT keys per
// thread in registers (position tid + NT j in slot j). The keff-th largest present key tau is found bit by bit from the top
// (tau = the largest t with at least keff keys >= t; only the bits below the
// common prefix of the row's smallest and largest present keys are searched,
// and the search stops once the keys >= the current prefix are exactly
// keff). Then the keys > tau and the lowest-positioned keys equal to tau are
// written in position order (per NT positions: warp ballots, the warps'
// counts through shared memory). Every step is a few instructions per thread
// and one CTA barrier; no histogram, no sample.
template <int NT, int KPT>
__global__ void __launch_bounds__(NT) topk_small_kernel(const TopkParams p) {
  constexpr int J = KPT, NW = NT / 32;
  constexpr int TK_SNT = NT;
  __shared__ uint32_t red[2][3][NW];          // double-buffered warp partials
  __shared__ uint32_t wcnt[2][NW];            // emit: selected / tau-equal keys per warp
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  int par = 0;                                // which red buffer the next reduction uses
  // sum (a), min (b) and max (c) over the CTA; one barrier
  auto reduce3 = [&](uint32_t& a, uint32_t& b2, uint32_t& c) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      b2 = min(b2, __shfl_xor_sync(0xffffffffu, b2, o));
      c = max(c, __shfl_xor_sync(0xffffffffu, c, o));
    }
    if (lane == 0) { red[par][0][wid] = a; red[par][1][wid] = b2; red[par][2][wid] = c; }
    __syncthreads();
    a = 0u; b2 = 0xffffffffu; c = 0u;
#pragma unroll
    for (int w = 0; w < NW; ++w) { a += red[par][0][w]; b2 = min(b2, red[par][1][w]); c = max(c, red[par][2][w]); }
    par ^= 1;
  };
  auto reduce_sum = [&](uint32_t a) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) red[par][0][wid] = a;
    __syncthreads();
    a = 0u;
#pragma unroll
    for (int w = 0; w < NW; ++w) a += red[par][0][w];
    par ^= 1;
    return a;
  };
  for (long long r = blockIdx.x; r < p.rows; r += gridDim.x) {
    const int n = row_length(p, r);
    const float* row = p.scores + r * p.ld;
    uint32_t key[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int pos = tid + TK_SNT * j;
      key[j] = pos < n ? __float_as_uint(__ldcg(row + pos)) : 0xff800000u;  // -inf past the row
    }
    uint32_t cnt = 0u, kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      key[j] = score_key(__uint_as_float(key[j]));
      if (key[j] != 0u) {
        ++cnt;
        kmin = min(kmin, key[j]);
        kmax = max(kmax, key[j]);
      }
    }
    reduce3(cnt, kmin, kmax);
    const uint32_t keff = min(static_cast<uint32_t>(p.k), cnt);
    uint32_t tau = kmin;  // keff == cnt, or every present key equal: tau = the smallest
    if (keff > 0u && keff < cnt && kmin != kmax) {
      // bits of tau above the highest bit where kmin and kmax differ are theirs
      const int hb = 31 - __clz(kmin ^ kmax);
      tau = kmax & ~((hb >= 31) ? 0xffffffffu : ((2u << hb) - 1u));
      // count(key >= tau) >= keff holds throughout; once it is exactly keff
      // the keys >= tau are the selection and the lower bits do not matter
      uint32_t clo = cnt;
      for (int b = hb; b >= 0 && clo != keff; --b) {
        const uint32_t t = tau | (1u << b);
        uint32_t c = 0u;
#pragma unroll
        for (int j = 0; j < J; ++j) c += key[j] >= t ? 1u : 0u;
        c = reduce_sum(c);
        if (c >= keff) { tau = t; clo = c; }
      }
    }
    // keys above tau, then as many tau-equal keys (lowest positions) as fit
    uint32_t above = 0u;
#pragma unroll
    for (int j = 0; j < J; ++j) above += (keff > 0u && key[j] > tau) ? 1u : 0u;
    above = reduce_sum(above);
    const uint32_t need = keff - above;
    int32_t* oi = p.out_idx + r * p.k;
    float* os = p.out_score ? p.out_score + r * p.k : nullptr;
    uint32_t eq_seen = 0u, out = 0u;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      // positions 128 j .. 128 j + 127: warp w holds 32 w .. 32 w + 31
      const bool gt = keff > 0u && key[j] > tau;
      const bool eq = keff > 0u && key[j] == tau && key[j] != 0u;
      const uint32_t em = __ballot_sync(0xffffffffu, eq);
      const uint32_t gm = __ballot_sync(0xffffffffu, gt);
      if (lane == 0) { wcnt[j & 1][wid] = __popc(em); red[par][0][wid] = __popc(gm); }
      __syncthreads();
      uint32_t eq_before = eq_seen, gt_before = 0u, eq_tot = 0u, gt_tot = 0u;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const uint32_t e = wcnt[j & 1][w], g = red[par][0][w];
        if (w < wid) { eq_before += e; gt_before += g; }
        eq_tot += e;
        gt_tot += g;
      }
      par ^= 1;
      // tau-equal keys taken before this warp's: min(need, eq_seen + earlier warps')
      const uint32_t eq_rank = eq_before + __popc(em & lt);
      const bool sel = gt || (eq && eq_rank < need);
      const uint32_t taken_before = min(need, eq_before);
      const uint32_t sm = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const uint32_t o = out + gt_before + taken_before - min(need, eq_seen) + __popc(sm & lt);
        oi[o] = map_index(p, r, tid + TK_SNT * j);
        if (os) os[o] = key_score(key[j]);
      }
      const uint32_t taken_all = min(need, eq_seen + eq_tot) - min(need, eq_seen);
      out += gt_tot + taken_all;
      eq_seen += eq_tot;
    }
    for (int j = static_cast<int>(keff) + tid; j < p.k; j += TK_SNT) {
      oi[j] = -1;
      if (os) os[j] = -INFINITY;
    }
    __syncthreads();  // the next row reuses the shared words
  }
}

// Rows whose candidate list cannot certify their top-k (fewer real entries
// than min(k, visible), or entries lost past the capacity) mark every key
// tile of their query group (qpt queries) for the fallback score pass.
__global__ void fused_check_kernel(const int* __restrict__ cres, const int* __restrict__ creal, long long rows,
                                   int T, long long q_offset, int L, int k, int cap, int qpt, int ntiles,
                                   uint8_t* __restrict__ fb) {
  const long long r = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (r >= rows) return;
  const int t = static_cast<int>(r % T);
  const long long V = min(q_offset + t + 1, static_cast<long long>(L));
  const int need = static_cast<int>(min(static_cast<long long>(k), V));
  if (cres[r] <= cap && creal[r] >= need) return;
  const long long g = (r / T) * ((T + qpt - 1) / qpt) + t / qpt;
  for (int j = 0; j < ntiles; ++j) fb[g * ntiles + j] = 1;
}

// ---------------------------------------------------------------- candidate thresholds
// Per row, from the scores of every S-th key (samp[r * lds + i] is the score
// of key i * S; the row has ns = min(p_t / S + 1, ns_max) of them): a
// threshold the row's k-th score is very likely to reach, the r_lo-th largest
// sample with r_lo = the sample rank expected for the k-th score + 4 standard
// deviations (binomial) + 4. -inf keeps every visible score (rows with no
// more than k visible keys, or too few samples). A wrong guess only costs
// time: rows whose lists come out short are selected from their full scores.
template <int NT>
__global__ void __launch_bounds__(NT) topk_threshold_kernel(const float* __restrict__ samp, long long rows,
                                                            long long lds, int T, long long q_offset, int S,
                                                            int ns_max, int L, int k, float* __restrict__ thr) {
  __shared__ uint32_t hist[TK_BINS];
  __shared__ uint32_t ws[64];
  __shared__ uint32_t vars[64];
  for (long long r = blockIdx.x; r < rows; r += gridDim.x) {
    const long long pos = q_offset + r % T;
    const long long V = min(pos + 1, static_cast<long long>(L));
    const int ns = static_cast<int>(min(pos / S + 1, static_cast<long long>(ns_max)));
    float t = -INFINITY;
    if (V > k) {
      const float pr = static_cast<float>(k) / static_cast<float>(V);
      const float mean = pr * ns;
      const float sd = sqrtf(static_cast<float>(ns) * pr * (1.f - pr));
      const int r_lo = static_cast<int>(ceilf(mean + 4.f * sd + 4.f));
      if (r_lo <= ns) {
        const float* row = samp + r * lds;
        exact_select<NT>([&](int i) { return score_key(__ldcg(row + i)); }, ns, static_cast<uint32_t>(r_lo), hist,
                         ws, vars);
        t = key_score(vars[0]);
      }
    }
    if (threadIdx.x == 0) thr[r] = t;
    __syncthreads();
  }
}

}  // namespace dsa
