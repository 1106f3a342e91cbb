// Exact per-row top-k over fp32 scores (lightning-indexer token selection:
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// section "Problem statement"; "DoSA: Dots Sparse Attention", Top-K selection).
//
// Selection rule: the k largest scores of a row, ties broken toward the lower
// position; -inf marks an absent candidate; rows with fewer than k candidates
// return all of them. Output: selected positions in ascending order (mapped
// through an optional index map), padded with -1 (score -inf).
//
// Method: scores map to order-preserving 32-bit keys (-0 folded onto +0,
// absent -> 0). A three-digit radix select (11 + 11 + 10 bits, shared-memory
// histograms with warp-aggregated atomics) finds the k-th key tau and how many
// keys equal to tau to take; a final ordered pass writes the keys above tau and
// the first keys equal to tau, in position order, through a block-wide scan.
// Rows up to TK_SMEM_ROW entries are staged once in shared memory; longer rows
// are streamed from global memory (L2) with a candidate cache for the third
// digit.
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
constexpr int TK_SMEM_ROW = 40960;   // rows up to this length are staged in shared memory
constexpr int TK_CAND_CAP = 20480;   // (key, position) pairs cached for long rows
constexpr int TK_SMEM_WORDS = 2048 + 64 + 16 + (TK_SMEM_ROW > 2 * TK_CAND_CAP ? TK_SMEM_ROW : 2 * TK_CAND_CAP);
constexpr int TK_SMEM_BYTES = TK_SMEM_WORDS * 4;

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

// Add one to hist[digit] for every lane with `has`, one atomic per distinct digit.
__device__ __forceinline__ void hist_add(uint32_t* hist, bool has, uint32_t digit) {
  const uint32_t m = __match_any_sync(0xffffffffu, has ? digit : 0xFFFFFFFFu);
  if (has && (threadIdx.x & 31) == static_cast<unsigned>(__ffs(m) - 1))
    atomicAdd(&hist[digit], static_cast<uint32_t>(__popc(m)));
}

// Given a histogram of NB bins (NB = 1024 * BPT) and a 1-based rank `need`
// counted from the largest digit, find the digit holding that rank and the
// rank inside it. Writes vars[0] = digit, vars[1] = new need.
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

__global__ void __launch_bounds__(TK_THREADS, 1) topk_rows_kernel(const TopkParams p) {
  extern __shared__ uint32_t tk_smem[];
  uint32_t* hist = tk_smem;          // 2048
  uint32_t* ws = hist + 2048;        // 64
  uint32_t* vars = ws + 64;          // 16
  uint32_t* cache = vars + 16;       // row keys, or (key, position) pairs
  const int tid = threadIdx.x;

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
    const bool staged = n <= TK_SMEM_ROW;
    const int k = p.k;

    // ---- digit 1 (bits 31..21) + count of present candidates
    for (int i = tid; i < 2048; i += TK_THREADS) hist[i] = 0;
    __syncthreads();
    uint32_t nv = 0;
    for (int base = 0; base < n; base += TK_THREADS) {
      const int i = base + tid;
      const uint32_t key = i < n ? score_key(__ldcg(row + i)) : 0u;
      if (staged && i < n) cache[i] = key;
      nv += key != 0u;
      hist_add(hist, key != 0u, key >> 21);
    }
    uint32_t nvalid;
    block_excl_scan(nv, ws, nvalid);
    const uint32_t keff = min(static_cast<uint32_t>(k), nvalid);

    uint32_t thr = 0, take_eq = 0;  // select key > thr, plus the first take_eq keys == thr
    if (keff < nvalid) {
      radix_pick<2>(hist, keff, ws, vars);
      const uint32_t d1 = vars[0];
      const uint32_t need1 = vars[1];
      const uint32_t cnt1 = hist[d1];
      const bool use_cache = !staged && cnt1 <= TK_CAND_CAP;
      __syncthreads();
      // ---- digit 2 (bits 20..10) among keys with digit 1 == d1
      for (int i = tid; i < 2048; i += TK_THREADS) hist[i] = 0;
      if (tid == 0) vars[2] = 0;
      __syncthreads();
      for (int base = 0; base < n; base += TK_THREADS) {
        const int i = base + tid;
        const uint32_t key = i < n ? (staged ? cache[i] : score_key(__ldcg(row + i))) : 0u;
        const bool in = key != 0u && (key >> 21) == d1;
        hist_add(hist, in, (key >> 10) & 0x7FFu);
        if (use_cache && in) {
          const uint32_t slot = atomicAdd(&vars[2], 1u);
          cache[2 * slot] = key;
          cache[2 * slot + 1] = static_cast<uint32_t>(i);
        }
      }
      __syncthreads();
      radix_pick<2>(hist, need1, ws, vars);
      const uint32_t d2 = vars[0];
      const uint32_t need2 = vars[1];
      const uint32_t ncache = vars[2];
      const uint32_t pre = (d1 << 11) | d2;
      __syncthreads();
      // ---- digit 3 (bits 9..0) among keys with digits 1-2 == pre
      for (int i = tid; i < 2048; i += TK_THREADS) hist[i] = 0;
      __syncthreads();
      if (use_cache) {
        for (int base = 0; base < static_cast<int>(ncache); base += TK_THREADS) {
          const int i = base + tid;
          const uint32_t key = i < static_cast<int>(ncache) ? cache[2 * i] : 0u;
          hist_add(hist, key != 0u && (key >> 10) == pre, key & 0x3FFu);
        }
      } else {
        for (int base = 0; base < n; base += TK_THREADS) {
          const int i = base + tid;
          const uint32_t key = i < n ? (staged ? cache[i] : score_key(__ldcg(row + i))) : 0u;
          hist_add(hist, key != 0u && (key >> 10) == pre, key & 0x3FFu);
        }
      }
      __syncthreads();
      radix_pick<1>(hist, need2, ws, vars);
      thr = (pre << 10) | vars[0];
      take_eq = vars[1];
      __syncthreads();
    }

    // ---- ordered write-out: keys > thr, then the first take_eq keys == thr
    int32_t* oi = p.out_idx + r * p.k;
    float* os = p.out_score ? p.out_score + r * p.k : nullptr;
    uint32_t run_gt = 0, run_eq = 0;
    for (int base = 0; base < n; base += TK_THREADS) {
      const int i = base + tid;
      const uint32_t key = i < n ? (staged ? cache[i] : score_key(__ldcg(row + i))) : 0u;
      const bool gt = key > thr;
      const bool eq = (key == thr) && key != 0u;
      uint32_t tot;
      const uint32_t ex = block_excl_scan((gt ? 0x10000u : 0u) | (eq ? 1u : 0u), ws, tot);
      const uint32_t eq_before = run_eq + (ex & 0xFFFFu);
      if (gt || (eq && eq_before < take_eq)) {
        const uint32_t pos = run_gt + (ex >> 16) + min(eq_before, take_eq);
        int idx = i;
        if (p.cand) {
          const int slot = i / p.blk;
          idx = __ldg(p.cand + r * p.n_slots + slot) * p.blk + (i - slot * p.blk);
        }
        oi[pos] = idx;
        if (os) os[pos] = key_score(key);
      }
      run_gt += tot >> 16;
      run_eq += tot & 0xFFFFu;
      if (run_gt + min(run_eq, take_eq) >= keff) break;
    }
    for (int j = static_cast<int>(keff) + tid; j < k; j += TK_THREADS) {
      oi[j] = -1;
      if (os) os[j] = -INFINITY;
    }
    __syncthreads();
  }
}

}  // namespace dsa
