// Exact per-row top-k over fp32 scores (lightning-indexer token selection:
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// section "Problem statement"; "DoSA: Dots Sparse Attention", Top-K selection).
//
// Selection rule: the k largest scores of a row, ties broken toward the lower
// position; -inf marks an absent candidate; rows with fewer than k candidates
// return all of them. Output: selected positions in ascending order (mapped
// through an optional index map), padded with -1 (score -inf).
//
// Scores map to order-preserving 32-bit keys (-0 folded onto +0, absent -> 0).
// The k-th key tau and the number of keys equal to tau to take are found in
// two steps:
//   1. coarse: a 2048-bin histogram over *values* (bins evenly spaced between
//      the row's min and max, a monotone map, so contention stays low even
//      though the scores crowd a few exponents) locates the bin holding the
//      k-th value; the bin's elements are compacted into a small buffer;
//   2. exact: a three-digit radix select (11 + 11 + 10 bits) over that buffer.
// If the bin is too large for the buffer (mass ties), the exact radix select
// runs over the whole row instead. The write-out gives each warp a contiguous
// segment: count, one block-wide exclusive scan of the 32 warp counts, then
// ballot-ordered stores, so positions come out in ascending order.
// Rows up to TK_SMEM_ROW entries are staged once in shared memory; longer rows
// are re-read from global memory (L2) on each pass.
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
};

constexpr int TK_THREADS = 1024;
constexpr int TK_WARPS = TK_THREADS / 32;
constexpr int TK_BINS = 2048;
constexpr int TK_SMEM_ROW = 40960;   // rows up to this length are staged in shared memory
constexpr int TK_CAND_CAP = 8192;    // keys of the threshold bin
constexpr int TK_SMEM_WORDS = TK_BINS + 128 + TK_CAND_CAP + TK_SMEM_ROW + 4;
constexpr int TK_SMEM_BYTES = TK_SMEM_WORDS * 4;
constexpr int TK_UNROLL = 8;        // float4 loads in flight per thread in the row load

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
    const uint32_t s = ws[lane];
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

// Source of one row's scores: the shared-memory stage, or the global row.
struct RowSrc {
  const float* smem;  // staged scores (or nullptr)
  const float* g;     // global row
  __device__ __forceinline__ float get(int i) const { return smem ? smem[i] : __ldcg(g + i); }
  __device__ __forceinline__ float4 get4(int i4) const {
    return smem ? reinterpret_cast<const float4*>(smem)[i4]
                : __ldcg(reinterpret_cast<const float4*>(g) + i4);
  }
};

__device__ __forceinline__ bool present(float x) { return x > -INFINITY; }  // false for -inf, NaN

// Exact radix select over keys (score_key) of a key buffer (cbuf != nullptr,
// n keys) or of positions [0, n) of a row; keys equal to 0 (absent) are
// ignored. Leaves vars[0] = tau, the need-th largest key, and vars[1] = how
// many keys equal to tau rank within the top `need`.
__device__ void exact_select(const uint32_t* cbuf, const RowSrc& src, int n, uint32_t need,
                             uint32_t* hist, uint32_t* ws, uint32_t* vars) {
  uint32_t prefix = 0;
#pragma unroll 1
  for (int d = 0; d < 3; ++d) {
    const int sh = d == 0 ? 21 : (d == 1 ? 10 : 0);
    const uint32_t width = d == 2 ? 10u : 11u;
    const uint32_t hi_sh = sh + width;
    for (int i = threadIdx.x; i < TK_BINS; i += TK_THREADS) hist[i] = 0;
    __syncthreads();
#pragma unroll 4
    for (int i = threadIdx.x; i < n; i += TK_THREADS) {
      const uint32_t key = cbuf ? cbuf[i] : score_key(src.get(i));
      if (key != 0u && (hi_sh >= 32 || (key >> hi_sh) == prefix))
        atomicAdd(&hist[(key >> sh) & ((1u << width) - 1u)], 1u);
    }
    __syncthreads();
    if (d < 2) radix_pick<2>(hist, need, ws, vars);
    else radix_pick<1>(hist, need, ws, vars);
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
// (x - lo) * scale >= 0; adding 1.5 * 2^23 leaves round-to-nearest(v) in the low
// mantissa bits (a monotone map, no float-to-int conversion instruction).
// scale == 0 (all scores equal, or a span that overflows) puts everything in bin 0.
__device__ __forceinline__ int value_bin(float x, float lo, float scale) {
  const float v = (scale > 0.f ? (x - lo) * scale : 0.f) + 12582912.0f;
  const int b = __float_as_int(v) - 0x4B400000;
  return min(b, TK_BINS - 1);
}

__global__ void __launch_bounds__(TK_THREADS, 1) topk_rows_kernel(const TopkParams p) {
  extern __shared__ uint32_t tk_smem[];
  uint32_t* hist = tk_smem;                  // TK_BINS
  uint32_t* ws = hist + TK_BINS;             // 64
  uint32_t* vars = ws + 64;                  // 64
  uint32_t* cbuf = vars + 64;                // TK_CAND_CAP keys of the threshold bin
  float* stage = reinterpret_cast<float*>(cbuf + TK_CAND_CAP);  // TK_SMEM_ROW scores
  float* fvars = reinterpret_cast<float*>(vars + 32);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;

  for (long long r = blockIdx.x; r < p.rows; r += gridDim.x) {
    const int t = static_cast<int>(r % p.T);
    long long nl = p.Lrow;
    if (p.pstride > 0) {
      nl = (p.q_offset + t) / p.pstride + 1;
      if (nl > p.Lrow) nl = p.Lrow;
      if (nl < 0) nl = 0;
    }
    const int n = static_cast<int>(nl);
    const float* row = p.scores + r * p.ld;
    const bool vec = ((reinterpret_cast<uintptr_t>(row) & 15u) == 0);
    const bool staged = n <= TK_SMEM_ROW && vec;
    const RowSrc src{staged ? stage : nullptr, row};
    const int n4 = vec ? (n >> 2) : 0;     // float4 part [0, 4*n4), scalar tail [4*n4, n)
    const int k = p.k;

    // ---- pass 1: (stage) count present scores, min / max
    uint32_t nv = 0;
    float vmin = INFINITY, vmax = -INFINITY;
    for (int base = 0; base < n4; base += TK_THREADS * TK_UNROLL) {
      float4 x[TK_UNROLL];
#pragma unroll
      for (int u = 0; u < TK_UNROLL; ++u) {
        const int i = base + u * TK_THREADS + tid;
        x[u] = i < n4 ? __ldcg(reinterpret_cast<const float4*>(row) + i)
                      : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
#pragma unroll
      for (int u = 0; u < TK_UNROLL; ++u) {
        const int i = base + u * TK_THREADS + tid;
        if (staged && i < n4) reinterpret_cast<float4*>(stage)[i] = x[u];
        const float xs[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const bool pr = present(xs[j]);
          nv += pr;
          vmin = fminf(vmin, pr ? xs[j] : INFINITY);
          vmax = fmaxf(vmax, xs[j]);
        }
      }
    }
    for (int i = 4 * n4 + tid; i < n; i += TK_THREADS) {
      const float x = __ldcg(row + i);
      if (staged) stage[i] = x;
      const bool pr = present(x);
      nv += pr;
      vmin = fminf(vmin, pr ? x : INFINITY);
      vmax = fmaxf(vmax, x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      nv += __shfl_xor_sync(0xffffffffu, nv, o);
      vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
      vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (lane == 0) {
      ws[wid] = nv;
      fvars[wid] = vmin;
      reinterpret_cast<float*>(ws)[32 + wid] = vmax;
    }
    __syncthreads();
    if (wid == 0) {
      uint32_t a = ws[lane];
      float mn = fvars[lane], mx = reinterpret_cast<float*>(ws)[32 + lane];
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
    const uint32_t keff = min(static_cast<uint32_t>(k), nvalid);
    __syncthreads();

    // select score > thr, plus the first take_eq scores == thr (-0 == +0 as floats)
    float thr = -INFINITY;
    uint32_t take_eq = 0;
    if (keff < nvalid) {
      // ---- coarse: value-binned histogram
      const float span = hi - lo;
      const float scale = (span > 0.f && span < INFINITY) ? static_cast<float>(TK_BINS - 1) / span : 0.f;
      for (int i = tid; i < TK_BINS; i += TK_THREADS) hist[i] = 0;
      if (tid == 0) vars[10] = 0;
      __syncthreads();
#pragma unroll 2
      for (int i = tid; i < n4; i += TK_THREADS) {
        const float4 x = src.get4(i);
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (present(xs[j])) atomicAdd(&hist[value_bin(xs[j], lo, scale)], 1u);
      }
      for (int i = 4 * n4 + tid; i < n; i += TK_THREADS) {
        const float x = src.get(i);
        if (present(x)) atomicAdd(&hist[value_bin(x, lo, scale)], 1u);
      }
      __syncthreads();
      radix_pick<2>(hist, keff, ws, vars);
      const int b = static_cast<int>(vars[0]);
      const uint32_t need = vars[1];
      const uint32_t cnt = hist[b];
      __syncthreads();
      if (cnt <= TK_CAND_CAP) {
#pragma unroll 2
        for (int i = tid; i < n4; i += TK_THREADS) {
          const float4 x = src.get4(i);
          const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (present(xs[j]) && value_bin(xs[j], lo, scale) == b)
              cbuf[atomicAdd(&vars[10], 1u)] = score_key(xs[j]);
        }
        for (int i = 4 * n4 + tid; i < n; i += TK_THREADS) {
          const float x = src.get(i);
          if (present(x) && value_bin(x, lo, scale) == b) cbuf[atomicAdd(&vars[10], 1u)] = score_key(x);
        }
        __syncthreads();
        exact_select(cbuf, src, static_cast<int>(cnt), need, hist, ws, vars);
      } else {
        exact_select(nullptr, src, n, keff, hist, ws, vars);
      }
      thr = key_score(vars[0]);
      take_eq = vars[1];
      __syncthreads();
    }

    // ---- ordered write-out. Warp w owns the contiguous segment [s0, s1);
    // lane l of a 128-entry chunk owns entries 4l .. 4l+3 (one float4).
    const int seg = ((n + TK_WARPS * 128 - 1) / (TK_WARPS * 128)) * 128;
    const int s0 = min(n, wid * seg);
    const int s1 = min(n, s0 + seg);
    const bool v4 = vec;  // 16-byte aligned row: float4 chunks
    auto load4 = [&](int i, float (&x)[4]) {
      if (v4 && i + 3 < s1) {
        const float4 f = src.get4(i >> 2);
        x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) x[j] = (i + j < s1) ? src.get(i + j) : -INFINITY;
      }
    };
    uint32_t cgt = 0, ceq = 0;
#pragma unroll 2
    for (int base = s0; base < s1; base += 128) {
      float x[4];
      load4(base + 4 * lane, x);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        cgt += x[j] > thr;
        ceq += x[j] == thr && present(x[j]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      cgt += __shfl_xor_sync(0xffffffffu, cgt, o);
      ceq += __shfl_xor_sync(0xffffffffu, ceq, o);
    }
    if (lane == 0) { ws[wid] = cgt; ws[32 + wid] = ceq; }
    __syncthreads();
    if (wid == 0) {
      const uint32_t g = ws[lane], e = ws[32 + lane];
      uint32_t gi = g, ei = e;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, gi, o);
        const uint32_t z = __shfl_up_sync(0xffffffffu, ei, o);
        if (lane >= o) { gi += y; ei += z; }
      }
      ws[lane] = gi - g;
      ws[32 + lane] = ei - e;
    }
    __syncthreads();
    uint32_t run_gt = ws[wid], run_eq = ws[32 + wid];
    __syncthreads();
    int32_t* oi = p.out_idx + r * p.k;
    float* os = p.out_score ? p.out_score + r * p.k : nullptr;
    for (int base = s0; base < s1; base += 128) {
      const int i0 = base + 4 * lane;
      float x[4];
      load4(i0, x);
      uint32_t ng = 0, ne = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        ng += x[j] > thr;
        ne += x[j] == thr && present(x[j]);
      }
      // exclusive prefix over the lanes (entries of lower lanes come first)
      uint32_t pg = ng, pe = ne;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, pg, o);
        const uint32_t z = __shfl_up_sync(0xffffffffu, pe, o);
        if (lane >= o) { pg += y; pe += z; }
      }
      uint32_t gb = run_gt + pg - ng, eb = run_eq + pe - ne;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool gt = x[j] > thr;
        const bool eq = x[j] == thr && present(x[j]);
        if (gt || (eq && eb < take_eq)) {
          const uint32_t pos = gb + min(eb, take_eq);
          const int i = i0 + j;
          int idx = i;
          if (p.cand) {
            const int slot = i / p.blk;
            idx = __ldg(p.cand + r * p.n_slots + slot) * p.blk + (i - slot * p.blk);
          }
          oi[pos] = idx;
          if (os) os[pos] = x[j] == 0.f ? 0.f : x[j];
        }
        gb += gt;
        eb += eq;
      }
      run_gt += __shfl_sync(0xffffffffu, pg, 31);
      run_eq += __shfl_sync(0xffffffffu, pe, 31);
    }
    for (int j = static_cast<int>(keff) + tid; j < k; j += TK_THREADS) {
      oi[j] = -1;
      if (os) os[j] = -INFINITY;
    }
    __syncthreads();
  }
}

}  // namespace dsa
