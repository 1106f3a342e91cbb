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
// (which already treat -0 and +0 as equal). Per row:
//   1. stage the row in shared memory when it fits (one full-rate read),
//      and take every S-th score as a sample (S a power of two, at most 4096
//      samples; a longer row stays in global memory / L2 and only its sample
//      is read here);
//   2. a 2048-bin value histogram of the sample (bins evenly spaced between
//      the sample's min and max) brackets the k-th score in a band
//      [t_lo, t_hi] wide enough (4 standard deviations of the sample rank on
//      each side) that the k-th score lies inside with near certainty;
//   3. one pass over the row: each warp owns a contiguous segment; for every
//      32 consecutive positions the warp's ballot of "score > t_hi" is stored
//      as that word of a selection bitmap, and the band's scores go to the
//      warp's candidate list (key, position), in position order;
//   4. an exact three-digit radix select (11 + 11 + 10 bits) over the
//      candidates gives tau and how many scores equal to tau to take; the
//      selected candidates are OR-ed into the bitmap;
//   5. the bitmap is emitted in position order (per-warp popcounts, one
//      prefix sum over the warps, each lane writes its set bits).
// If a check fails (unlucky sample, mass ties, a full candidate list, fewer
// present scores than k), the row falls back to a full value histogram, an
// exact select over the k-th value's bin (or the whole row), a counting pass
// and an ordered write pass.
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
  unsigned* err;         // device status word (bounded waits)
};

constexpr int TK_THREADS = 1024;     // one row per CTA, one CTA per SM
constexpr int TK_CTAS_PER_SM = 1;
constexpr int TK_WARPS = TK_THREADS / 32;
static_assert(TK_WARPS == 32, "per-warp totals are reduced with one warp's shuffles");
constexpr int TK_BINS = 2048;
constexpr int TK_SMEM_ROW = 32768;   // rows up to this length are staged in shared memory
constexpr int TK_LIST = 128;         // band candidates per warp segment (staged rows)
// rows that are not staged keep their candidate lists in the unused stage area
constexpr int TK_LIST_LONG = TK_SMEM_ROW / (2 * (TK_THREADS / 32));
constexpr int TK_CAND_CAP = TK_WARPS * TK_LIST;
constexpr int TK_SAMPLE_MAX = 4096;  // sampled scores per row
constexpr int TK_BITMAP_WORDS = 4096;
// longer rows take the fallback path (their selection bitmap would not fit)
constexpr long long TK_MAX_BITMAP_ROW = 32LL * TK_BITMAP_WORDS;
constexpr int TK_SMEM_WORDS =
    TK_BINS + 128 + TK_SAMPLE_MAX + 2 * TK_CAND_CAP + TK_BITMAP_WORDS + TK_SMEM_ROW + 4;  // + barrier
constexpr int TK_SMEM_BYTES = TK_SMEM_WORDS * 4;
constexpr int TK_UNROLL = 8;         // float4 loads in flight per thread when staging a row

__device__ __forceinline__ uint32_t score_key(float x) {
  if (!(x > -INFINITY)) return 0u;  // -inf (absent) and NaN
  if (x == 0.f) x = 0.f;            // -0 -> +0
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Exclusive prefix sum over the 1024 threads in thread order; `total` gets the sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* ws, uint32_t& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) ws[wid] = x;
  __syncthreads();
  if (wid == 0) {
    const uint32_t s = lane < TK_THREADS / 32 ? ws[lane] : 0u;
    uint32_t inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    ws[lane] = inc - s;
    if (lane == 31) ws[32] = inc;
  }
  __syncthreads();
  const uint32_t r = ws[wid] + x - v;
  total = ws[32];
  __syncthreads();
  return r;
}

// Histogram of NB = 1024 * BPT bins, 1-based rank `need` counted from the top:
// find the bin holding that rank and the rank inside it -> vars[0], vars[1].
template <int BPT>
__device__ __forceinline__ void radix_pick(const uint32_t* hist, uint32_t need, uint32_t* ws,
                                           uint32_t* vars) {
  const int u = TK_THREADS - 1 - threadIdx.x;  // owner of bins [u*BPT, (u+1)*BPT)
  uint32_t loc = 0;
#pragma unroll
  for (int i = 0; i < BPT; ++i) loc += hist[u * BPT + i];
  uint32_t tot;
  uint32_t above = block_excl_scan(loc, ws, tot);  // count in the bins of owners > u
#pragma unroll
  for (int i = BPT - 1; i >= 0; --i) {
    const uint32_t c = hist[u * BPT + i];
    if (above < need && need <= above + c) {
      vars[0] = static_cast<uint32_t>(u * BPT + i);
      vars[1] = need - above;
    }
    above += c;
  }
  __syncthreads();
}

__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ float4 lds_f32x4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(a)
               : "memory");
  return v;
}
__device__ __forceinline__ void sts_f32x4(uint32_t a, float4 v) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

// Source of one row's scores: the shared-memory stage (explicit shared-window
// loads) or the global row, chosen at compile time so the passes carry no
// per-access branch.
template <bool STAGED>
struct RowSrc {
  uint32_t sbase;   // shared address of the staged row
  const float* g;   // global row
  __device__ __forceinline__ float get(int i) const {
    if constexpr (STAGED) return lds_f32(sbase + 4u * static_cast<uint32_t>(i));
    else return __ldcg(g + i);
  }
  // entries i .. i+3 (i a multiple of 4), -inf from `end` on; one vector
  // load when all four exist and the row start allows it (vec)
  __device__ __forceinline__ float4 get4(int i, int end, bool vec) const {
    if (i + 3 < end && (STAGED || vec)) {
      if constexpr (STAGED) return lds_f32x4(sbase + 4u * static_cast<uint32_t>(i));
      else return __ldcg(reinterpret_cast<const float4*>(g + i));
    }
    float4 v = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    if (i < end) v.x = get(i);
    if (i + 1 < end) v.y = get(i + 1);
    if (i + 2 < end) v.z = get(i + 2);
    if (i + 3 < end) v.w = get(i + 3);
    return v;
  }
};

__device__ __forceinline__ bool present(float x) { return x > -INFINITY; }  // false for -inf, NaN

// Exact radix select over keys (score_key) of a key buffer (cbuf != nullptr,
// n keys) or of positions [0, n) of a row; keys equal to 0 (absent) are
// ignored. Leaves vars[0] = tau, the need-th largest key, and vars[1] = how
// many keys equal to tau rank within the top `need`.
// lists != nullptr: cbuf holds one list per warp (stride `n`), warp w's first
// lists[w] entries are its keys, and each warp scans its own list.
template <class Src>
__device__ void exact_select(const uint32_t* cbuf, const Src& src, int n, uint32_t need,
                             uint32_t* hist, uint32_t* ws, uint32_t* vars, int d0 = 0,
                             uint32_t prefix0 = 0, const uint32_t* lists = nullptr) {
  // d0 > 0: every key shares its top bits with prefix0 (digits before d0 are known)
  uint32_t prefix = prefix0;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int lcount = lists ? static_cast<int>(min(lists[wid], static_cast<uint32_t>(n))) : 0;
#pragma unroll 1
  for (int d = d0; d < 3; ++d) {
    const int sh = d == 0 ? 21 : (d == 1 ? 10 : 0);
    const uint32_t width = d == 2 ? 10u : 11u;
    const uint32_t hi_sh = sh + width;
    for (int i = threadIdx.x; i < TK_BINS; i += TK_THREADS) hist[i] = 0;
    __syncthreads();
    if (lists) {
      for (int i = lane; i < lcount; i += 32) {
        const uint32_t key = cbuf[wid * n + i];
        if (key != 0u && (hi_sh >= 32 || (key >> hi_sh) == prefix))
          atomicAdd(&hist[(key >> sh) & ((1u << width) - 1u)], 1u);
      }
    } else {
#pragma unroll 4
      for (int i = threadIdx.x; i < n; i += TK_THREADS) {
        const uint32_t key = cbuf ? cbuf[i] : score_key(src.get(i));
        if (key != 0u && (hi_sh >= 32 || (key >> hi_sh) == prefix))
          atomicAdd(&hist[(key >> sh) & ((1u << width) - 1u)], 1u);
      }
    }
    __syncthreads();
    if (d < 2) radix_pick<2048 / TK_THREADS>(hist, need, ws, vars);
    else radix_pick<1024 / TK_THREADS>(hist, need, ws, vars);
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

// Value bin of a present score: TK_BINS evenly spaced bins over [lo, lo + TK_BINS/scale].
// For x in [lo, hi], (x - lo) * scale >= 0; adding 1.5 * 2^23 leaves round-to-nearest(v) in the low
// mantissa bits (a monotone map, no float-to-int conversion instruction).
// scale == 0 (all scores equal, or a span that overflows) puts everything in bin 0.
__device__ __forceinline__ int value_bin(float x, float lo, float scale) {
  const float v = (scale > 0.f ? (x - lo) * scale : 0.f) + 12582912.0f;
  const int b = __float_as_int(v) - 0x4B400000;
  return min(max(b, 0), TK_BINS - 1);  // scores outside [lo, hi] land in the end bins
}

// One row of the selection (see the file comment). STAGED: the row fits in
// shared memory and starts on a 16-byte boundary.
// The staged scores of the next row may already be on their way (prefetched
// by the previous row with a bulk copy on `sbar`); the row prefetches the
// CTA's next row (nxt, n_nxt) as soon as its own staged scores are no longer
// read. Returns whether it did.
template <bool STAGED>
__device__ __forceinline__ bool topk_row(const TopkParams& p, uint32_t* tk_smem, long long r, int n,
                                         const float* row, uint32_t sbar, uint32_t& sphase,
                                         bool prefetched, const float* nxt, int n_nxt) {
  uint32_t* hist = tk_smem;                      // TK_BINS
  uint32_t* ws = hist + TK_BINS;                 // 64
  uint32_t* vars = ws + 64;                      // 64
  uint32_t* samp = vars + 64;                    // TK_SAMPLE_MAX sampled scores (as floats)
  uint32_t* ckey = samp + TK_SAMPLE_MAX;         // TK_CAND_CAP keys (warp w: [w*TK_LIST, +TK_LIST))
  uint32_t* cpos = ckey + TK_CAND_CAP;           // TK_CAND_CAP positions
  uint32_t* bmap = cpos + TK_CAND_CAP;           // TK_BITMAP_WORDS selection bitmap
  float* stage = reinterpret_cast<float*>(bmap + TK_BITMAP_WORDS);  // TK_SMEM_ROW scores
  float* fvars = reinterpret_cast<float*>(vars + 32);
  float* fsamp = reinterpret_cast<float*>(samp);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const uint32_t s_stage = smem_u32(stage);
  const RowSrc<STAGED> src{s_stage, row};
  // per-warp band candidate lists (keys, positions)
  constexpr int LIST = STAGED ? TK_LIST : TK_LIST_LONG;
  uint32_t* lkey = STAGED ? ckey : reinterpret_cast<uint32_t*>(stage);
  uint32_t* lpos = STAGED ? cpos : reinterpret_cast<uint32_t*>(stage) + TK_WARPS * TK_LIST_LONG;
  const int k = p.k;
  // warp segments (multiples of 128 entries)
  const int seg = ((n + TK_WARPS * 128 - 1) / (TK_WARPS * 128)) * 128;
  const int s0 = min(n, wid * seg);
  const int s1 = min(n, s0 + seg);
  const bool fast = n > k && n <= TK_MAX_BITMAP_ROW;
  // sample stride: a power of two >= 4 so that samples sit at float4 starts
  int S = 4;
  while (static_cast<long long>(S) * TK_SAMPLE_MAX < n) S <<= 1;
  const int ns = (n + S - 1) / S;

  float thr = -INFINITY;  // select score > thr, plus the first take_eq scores == thr
  uint32_t take_eq = 0;
  uint32_t keff = 0;
  bool done = false;      // row written by the bitmap path

  bool issued_next = false;
  // Prefetch the next row into the stage (thread 0; the caller's __syncthreads
  // or this row's have retired every read of the stage).
  auto prefetch_next = [&]() {
    if constexpr (STAGED) {
      if (nxt != nullptr) {
        if (tid == 0) {
          fence_proxy_async_smem();
          const uint32_t bytes = static_cast<uint32_t>(n_nxt >> 2) * 16u;
          if (bytes) {
            mbar_arrive_expect_tx(sbar, bytes);
            bulk_load(s_stage, nxt, bytes, sbar);
          } else {
            mbar_arrive(sbar);
          }
        }
        issued_next = true;
      }
    }
  };

  // ---- 1. stage (or sample only)
  if constexpr (STAGED) {
    const int n4 = n >> 2;
    if (!prefetched && tid == 0) {
      fence_proxy_async_smem();  // earlier generic accesses of the stage before the copy
      const uint32_t bytes = static_cast<uint32_t>(n4) * 16u;
      if (bytes) {
        mbar_arrive_expect_tx(sbar, bytes);
        bulk_load(s_stage, row, bytes, sbar);
      } else {
        mbar_arrive(sbar);
      }
    }
    for (int i = 4 * n4 + tid; i < n; i += TK_THREADS) sts_f32(s_stage + 4u * static_cast<uint32_t>(i), __ldcg(row + i));
    // on a timeout (error recorded) the copy is still drained, bounded, so
    // that no copy is left in flight when the CTA moves on or exits
    if (!mbar_wait(sbar, sphase, p.err)) mbar_drain(sbar, sphase);
    sphase ^= 1u;
    __syncthreads();
    if (fast) {
      for (int m = tid; m < ns; m += TK_THREADS) fsamp[m] = src.get(m * S);
    }
  } else if (fast) {
#pragma unroll 8
    for (int m = tid; m < ns; m += TK_THREADS) fsamp[m] = __ldcg(row + static_cast<long long>(m) * S);
  }
  __syncthreads();

  if (fast) {
    // ---- 2. sample: present count, min / max, value histogram -> band
    uint32_t nsv = 0;
    float vmin = INFINITY, vmax = -INFINITY;
    for (int m = tid; m < ns; m += TK_THREADS) {
      const float x = fsamp[m];
      if (present(x)) { ++nsv; vmin = fminf(vmin, x); vmax = fmaxf(vmax, x); }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      nsv += __shfl_xor_sync(0xffffffffu, nsv, o);
      vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
      vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (lane == 0) { ws[wid] = nsv; fvars[wid] = vmin; reinterpret_cast<float*>(ws)[32 + wid] = vmax; }
    for (int i = tid; i < TK_BINS; i += TK_THREADS) hist[i] = 0;
    __syncthreads();
    if (wid == 0) {
      const bool has = lane < TK_WARPS;  // one partial per warp
      uint32_t a = has ? ws[lane] : 0u;
      float mn = has ? fvars[lane] : INFINITY;
      float mx = has ? reinterpret_cast<float*>(ws)[32 + lane] : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (lane == 0) {
        vars[8] = a;
        reinterpret_cast<float*>(vars)[16] = mn;
        reinterpret_cast<float*>(vars)[17] = mx;
      }
    }
    __syncthreads();
    const uint32_t nsvu = vars[8];
    const float lo = reinterpret_cast<float*>(vars)[16], hi = reinterpret_cast<float*>(vars)[17];
    const float span = hi - lo;
    const float scale = (span > 0.f && span < INFINITY) ? static_cast<float>(TK_BINS - 1) / span : 0.f;
    for (int m = tid; m < ns; m += TK_THREADS) {
      const float x = fsamp[m];
      if (present(x)) atomicAdd(&hist[value_bin(x, lo, scale)], 1u);
    }
    __syncthreads();
    // expected rank of the k-th score inside the sample
    const float nsvf = static_cast<float>(nsvu);
    const float pr = fminf(1.f, static_cast<float>(k) / fmaxf(1.f, nsvf * static_cast<float>(S)));
    const float center = pr * nsvf;
    const float delta = 4.f * sqrtf(nsvf * pr * (1.f - pr)) + 4.f;
    const int r_hi = static_cast<int>(floorf(center - delta));
    const int r_lo = static_cast<int>(ceilf(center + delta));
    {
      constexpr int BPT = TK_BINS / TK_THREADS;
      const int u = TK_THREADS - 1 - tid;  // owner of bins [u*BPT, (u+1)*BPT)
      uint32_t loc = 0;
#pragma unroll
      for (int q = 0; q < BPT; ++q) loc += hist[u * BPT + q];
      uint32_t tot;
      long long above = block_excl_scan(loc, ws, tot);
      if (tid == 0) { vars[12] = TK_BINS; vars[13] = 0; }
      __syncthreads();
#pragma unroll
      for (int q = BPT - 1; q >= 0; --q) {
        const long long c = hist[u * BPT + q];
        if (r_hi >= 1 && above < r_hi && r_hi <= above + c) vars[12] = u * BPT + q;
        if (r_lo <= static_cast<int>(tot) && above < r_lo && r_lo <= above + c) vars[13] = u * BPT + q;
        above += c;
      }
      __syncthreads();
    }
    const int b_hi = static_cast<int>(vars[12]);
    const int b_lo = static_cast<int>(vars[13]);
    const float t_hi = (b_hi >= TK_BINS - 1 || scale == 0.f) ? INFINITY
                                                            : lo + (static_cast<float>(b_hi) + 0.5f) / scale;
    const float t_lo = (b_lo <= 0 || scale == 0.f) ? -INFINITY
                                                   : lo + (static_cast<float>(b_lo) - 0.5f) / scale;
    __syncthreads();

    // ---- 3. band pass: bitmap words of "> t_hi" (bmap) and of the band
    // [t_lo, t_hi] (bbm, in the sample's space). A lane takes 4 consecutive
    // entries; a word (32 entries) is the OR of the nibbles of 8 lanes.
    // Present entries are not counted: with t_lo = -inf every present entry
    // is above or in the band, otherwise the band test below needs no count.
    const float t_lo_p = t_lo > -INFINITY ? t_lo : -3.402823466e+38f;  // x >= t_lo_p: present
    const bool vec = (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
    uint32_t* bbm = samp;
    uint32_t* my_key = lkey + wid * LIST;
    uint32_t* my_pos = lpos + wid * LIST;
    uint32_t c_above = 0;
    // rows read from global memory keep more loads in flight
    constexpr int UB = STAGED ? 2 : 4;
    for (int base = s0; base < s1; base += 128 * UB) {
      float4 xv[UB];
#pragma unroll
      for (int j = 0; j < UB; ++j) xv[j] = src.get4(base + 128 * j + 4 * lane, s1, vec);
#pragma unroll
      for (int j = 0; j < UB; ++j) {
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
    // this warp's band entries -> its list, in position order
    const int w0 = s0 >> 5;                              // this warp's words
    const int w1 = s1 > s0 ? (s1 + 31) >> 5 : w0;      // (none for an empty segment)
    uint32_t c_band = 0;
    for (int wb = w0; wb < w1; wb += 32) {
      const int wd = wb + lane;
      uint32_t bits = wd < w1 ? bbm[wd] : 0u;
      const uint32_t cnt = __popc(bits);
      uint32_t inc = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      uint32_t slot = c_band + inc - cnt;
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1u;
        if (slot < LIST) {
          const int i = wd * 32 + b;
          my_key[slot] = score_key(src.get(i));
          my_pos[slot] = static_cast<uint32_t>(i);
        }
        ++slot;
      }
      c_band += __shfl_sync(0xffffffffu, inc, 31);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c_above += __shfl_xor_sync(0xffffffffu, c_above, o);
    uint32_t* lcnt = vars + 32;                          // per-warp list lengths
    if (lane == 0) { ws[wid] = c_above; lcnt[wid] = c_band; }
    __syncthreads();
    uint32_t above_all = ws[lane], nc = lcnt[lane], cmax = lcnt[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      above_all += __shfl_xor_sync(0xffffffffu, above_all, o);
      nc += __shfl_xor_sync(0xffffffffu, nc, o);
      cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    }
    // with t_lo = -inf the present entries are exactly above + band
    keff = t_lo > -INFINITY ? static_cast<uint32_t>(k) : min(static_cast<uint32_t>(k), above_all + nc);
    const bool band_ok = cmax <= LIST && above_all < keff && keff <= above_all + nc;
    __syncthreads();
    if (band_ok) {
      // the staged scores are not read past this point: start the next row's copy
      prefetch_next();
      // ---- 4. exact select among the candidates. Every candidate lies in
      // [t_lo, t_hi]: digits on which both ends agree are skipped.
      int d0 = 0;
      uint32_t pre0 = 0;
      if (t_lo > -INFINITY && t_hi < INFINITY) {
        const uint32_t kl = score_key(t_lo), kh = score_key(t_hi);
        if ((kl >> 10) == (kh >> 10)) { d0 = 2; pre0 = kl >> 10; }
        else if ((kl >> 21) == (kh >> 21)) { d0 = 1; pre0 = kl >> 21; }
      }
      exact_select(lkey, src, LIST, keff - above_all, hist, ws, vars, d0, pre0, lcnt);
      const uint32_t tau = vars[0];
      const uint32_t teq = vars[1];
      // eq counts per warp list -> prefix (lists are in position order)
      const uint32_t cb = lcnt[wid];
      uint32_t ceq = 0;
      for (int sl = lane; sl < static_cast<int>(cb); sl += 32) ceq += my_key[sl] == tau;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ceq += __shfl_xor_sync(0xffffffffu, ceq, o);
      if (lane == 0) ws[wid] = ceq;
      __syncthreads();
      uint32_t eq_before;
      {
        const uint32_t e = ws[lane];                       // warps before this one
        uint32_t inc = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += y;
        }
        eq_before = __shfl_sync(0xffffffffu, inc - e, wid);
      }
      for (int base = 0; base < static_cast<int>(cb); base += 32) {
        const int sl = base + lane;
        const uint32_t key = sl < static_cast<int>(cb) ? my_key[sl] : 0u;
        const bool eq = key == tau && key != 0u;
        const uint32_t me = __ballot_sync(0xffffffffu, eq);
        const uint32_t rank = eq_before + __popc(me & lt_mask);
        if (key > tau || (eq && rank < teq)) {
          const uint32_t pos = my_pos[sl];
          atomicOr(&bmap[pos >> 5], 1u << (pos & 31u));
        }
        eq_before += __popc(me);
      }
      __syncthreads();
      // ---- 5. emit the bitmap in position order
      const int per = (w1 - w0 + 31) / 32;                 // words per lane (contiguous)
      const int l0 = min(w1, w0 + lane * per), l1 = min(w1, l0 + per);
      uint32_t cnt = 0;
      for (int wd = l0; wd < l1; ++wd) cnt += __popc(bmap[wd]);
      uint32_t inc = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      if (lane == 31) ws[32 + wid] = inc;
      __syncthreads();
      uint32_t wbase;
      {
        const uint32_t e = ws[32 + lane];
        uint32_t winc = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, winc, o);
          if (lane >= o) winc += y;
        }
        wbase = __shfl_sync(0xffffffffu, winc - e, wid);
      }
      uint32_t out = wbase + inc - cnt;
      int32_t* oi = p.out_idx + r * p.k;
      float* os = p.out_score ? p.out_score + r * p.k : nullptr;
      // positions are collected in shared memory (the candidate-list space,
      // no longer read) and written out below with coalesced stores
      uint32_t* obuf = ckey;
      const bool via_smem = k <= 2 * TK_CAND_CAP;
      for (int wd = l0; wd < l1; ++wd) {
        uint32_t bits = bmap[wd];
        while (bits) {
          const int b = __ffs(bits) - 1;
          bits &= bits - 1u;
          const int i = wd * 32 + b;
          if (out < static_cast<uint32_t>(k)) {  // holds by construction; guards the row
            if (via_smem) {
              obuf[out] = static_cast<uint32_t>(i);
            } else {
              int idx = i;
              if (p.cand) {
                const int slot = i / p.blk;
                idx = __ldg(p.cand + r * p.n_slots + slot) * p.blk + (i - slot * p.blk);
              }
              oi[out] = idx;
              if (os) { const float x = __ldcg(row + i); os[out] = x == 0.f ? 0.f : x; }
            }
          }
          ++out;
        }
      }
      if (via_smem) {
        __syncthreads();
        for (int j = tid; j < static_cast<int>(keff); j += TK_THREADS) {
          const int i = static_cast<int>(obuf[j]);
          int idx = i;
          if (p.cand) {
            const int slot = i / p.blk;
            idx = __ldg(p.cand + r * p.n_slots + slot) * p.blk + (i - slot * p.blk);
          }
          oi[j] = idx;
          if (os) { const float x = __ldcg(row + i); os[j] = x == 0.f ? 0.f : x; }
        }
      }
      done = true;
    }
    __syncthreads();
  }

  if (!done) {
    // ---- fallback: min / max and present count over the row, full value
    // histogram, exact select, counting pass, ordered write pass
    uint32_t nv = 0;
    float vmin = INFINITY, vmax = -INFINITY;
    for (int i = tid; i < n; i += TK_THREADS) {
      const float x = src.get(i);
      if (present(x)) { ++nv; vmin = fminf(vmin, x); vmax = fmaxf(vmax, x); }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      nv += __shfl_xor_sync(0xffffffffu, nv, o);
      vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
      vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (lane == 0) { ws[wid] = nv; fvars[wid] = vmin; reinterpret_cast<float*>(ws)[32 + wid] = vmax; }
    __syncthreads();
    if (wid == 0) {
      const bool has = lane < TK_WARPS;  // one partial per warp
      uint32_t a = has ? ws[lane] : 0u;
      float mn = has ? fvars[lane] : INFINITY;
      float mx = has ? reinterpret_cast<float*>(ws)[32 + lane] : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (lane == 0) {
        vars[8] = a;
        reinterpret_cast<float*>(vars)[16] = mn;
        reinterpret_cast<float*>(vars)[17] = mx;
      }
    }
    __syncthreads();
    const uint32_t nvalid = vars[8];
    const float lo = reinterpret_cast<float*>(vars)[16], hi = reinterpret_cast<float*>(vars)[17];
    keff = min(static_cast<uint32_t>(k), nvalid);
    __syncthreads();
    if (keff < nvalid) {
      const float span = hi - lo;
      const float scale = (span > 0.f && span < INFINITY) ? static_cast<float>(TK_BINS - 1) / span : 0.f;
      for (int i = tid; i < TK_BINS; i += TK_THREADS) hist[i] = 0;
      if (tid == 0) vars[10] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += TK_THREADS) {
        const float x = src.get(i);
        if (present(x)) atomicAdd(&hist[value_bin(x, lo, scale)], 1u);
      }
      __syncthreads();
      radix_pick<TK_BINS / TK_THREADS>(hist, keff, ws, vars);
      const int b = static_cast<int>(vars[0]);
      const uint32_t need = vars[1];
      const uint32_t cnt = hist[b];
      __syncthreads();
      if (cnt <= TK_CAND_CAP) {
        for (int i = tid; i < n; i += TK_THREADS) {
          const float x = src.get(i);
          if (present(x) && value_bin(x, lo, scale) == b) ckey[atomicAdd(&vars[10], 1u)] = score_key(x);
        }
        __syncthreads();
        exact_select(ckey, src, static_cast<int>(cnt), need, hist, ws, vars);
      } else {
        exact_select(nullptr, src, n, keff, hist, ws, vars);
      }
      thr = key_score(vars[0]);
      take_eq = vars[1];
      __syncthreads();
    }
    // counting pass (per warp segment), prefix over the warps, ordered write
    uint32_t cgt = 0, ceq = 0;
    for (int base = s0; base < s1; base += 128) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = base + 32 * j + lane;
        const float x = i < s1 ? src.get(i) : -INFINITY;
        cgt += x > thr;
        ceq += x == thr && present(x);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      cgt += __shfl_xor_sync(0xffffffffu, cgt, o);
      ceq += __shfl_xor_sync(0xffffffffu, ceq, o);
    }
    if (lane == 0) { ws[wid] = cgt; ws[32 + wid] = ceq; }
    __syncthreads();
    uint32_t run_gt = 0, run_eq = 0;
    for (int w = 0; w < wid; ++w) { run_gt += ws[w]; run_eq += ws[32 + w]; }
    __syncthreads();
    int32_t* oi = p.out_idx + r * p.k;
    float* os = p.out_score ? p.out_score + r * p.k : nullptr;
    for (int base = s0; base < s1; base += 128) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = base + 32 * j + lane;
        const float x = i < s1 ? src.get(i) : -INFINITY;
        const bool gt = x > thr;
        const bool eq = x == thr && present(x);
        const uint32_t mg = __ballot_sync(0xffffffffu, gt);
        const uint32_t me = __ballot_sync(0xffffffffu, eq);
        const uint32_t gb = run_gt + __popc(mg & lt_mask);
        const uint32_t eb = run_eq + __popc(me & lt_mask);
        if ((gt || (eq && eb < take_eq)) && gb + min(eb, take_eq) < static_cast<uint32_t>(k)) {
          const uint32_t pos = gb + min(eb, take_eq);
          int idx = i;
          if (p.cand) {
            const int slot = i / p.blk;
            idx = __ldg(p.cand + r * p.n_slots + slot) * p.blk + (i - slot * p.blk);
          }
          oi[pos] = idx;
          if (os) os[pos] = x == 0.f ? 0.f : x;
        }
        run_gt += __popc(mg);
        run_eq += __popc(me);
      }
    }
  }
  int32_t* oi = p.out_idx + r * p.k;
  float* os = p.out_score ? p.out_score + r * p.k : nullptr;
  for (int j = static_cast<int>(keff) + tid; j < k; j += TK_THREADS) {
    oi[j] = -1;
    if (os) os[j] = -INFINITY;
  }
  if (!issued_next) {
    __syncthreads();  // every read of the stage is done
    prefetch_next();
  }
  return issued_next;
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

__device__ __forceinline__ bool row_staged(const float* row, int n) {
  return n <= TK_SMEM_ROW && (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
}

__global__ void __launch_bounds__(TK_THREADS, TK_CTAS_PER_SM) topk_rows_kernel(const TopkParams p) {
  extern __shared__ uint32_t tk_smem[];
  const uint32_t sbar = smem_u32(tk_smem + TK_SMEM_WORDS - 2);  // stage copy barrier (8-byte aligned)
  if (threadIdx.x == 0) {
    mbar_init(sbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  uint32_t sphase = 0;
  bool prefetched = false;
  for (long long r = blockIdx.x; r < p.rows; r += gridDim.x) {
    const int n = row_length(p, r);
    const float* row = p.scores + r * p.ld;
    const long long rn = r + gridDim.x;
    const float* nrow = rn < p.rows ? p.scores + rn * p.ld : nullptr;
    const int nn = nrow ? row_length(p, rn) : 0;
    const float* nxt = (nrow && row_staged(nrow, nn)) ? nrow : nullptr;
    if (row_staged(row, n)) {
      prefetched = topk_row<true>(p, tk_smem, r, n, row, sbar, sphase, prefetched, nxt, nn);
    } else {
      topk_row<false>(p, tk_smem, r, n, row, sbar, sphase, false, nullptr, 0);
      prefetched = false;
    }
    __syncthreads();
  }
  // a prefetch is only issued for a row this CTA processes next: nothing is
  // left in flight here
}

}  // namespace dsa
