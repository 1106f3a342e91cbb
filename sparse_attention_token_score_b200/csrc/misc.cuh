// Small kernels around the scoring and selection kernels: block mean-pooling of
// keys and the MISA head selection.
#pragma once
#include "common.cuh"

namespace dsa {

// Pooled keys ("MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
// Inference", section "Methodology", step 1: the prefix splits into
// M = ceil(L/B) blocks, each represented by its mean-pooled indexing key; the
// HISA review, section 3, uses the same pooled representatives):
//     kbar[b, m, :] = bf16( mean of k[b, mB : min((m+1)B, L), :] )
// The sum runs in fp64, which is exact for bf16 inputs at these block sizes,
// and is rounded to bf16 once (round to nearest even).
// Grid: batch * M blocks; threads over the d columns.
__global__ void meanpool_kernel(const __nv_bfloat16* __restrict__ k, int L, int d, int B, int M,
                                __nv_bfloat16* __restrict__ kbar) {
  const long long bm = blockIdx.x;
  const long long b = bm / M;
  const int m = static_cast<int>(bm % M);
  const int s0 = m * B;
  const int s1 = min(s0 + B, L);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    double acc = 0.0;
    for (int s = s0; s < s1; ++s) acc += static_cast<double>(__bfloat162float(k[(b * L + s) * d + c]));
    kbar[bm * d + c] = __double2bfloat16(acc / static_cast<double>(s1 - s0));
  }
}

// MISA routing (same page, "Methodology", step 1): per query, the head
// affinity a[h] = |w[h]| * (part0[h] + part1[h]) (the two partial ReLU sums
// over pooled keys from the router kernel); keep the top-hsel heads by
// (a descending, head ascending). Writes the kept heads in ascending order,
// their weights, and gathers their query rows into a compact [rows, hsel, d]
// tensor for the routed scoring pass. One warp per query row; H <= 64.
__global__ void select_heads_kernel(const float* __restrict__ part, long long rows, int H, int hsel,
                                    const float* __restrict__ w, const __nv_bfloat16* __restrict__ q,
                                    int d, int* __restrict__ heads, __nv_bfloat16* __restrict__ q_sel,
                                    float* __restrict__ w_sel) {
  const int lane = threadIdx.x & 31;
  const long long r = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const long long plane = rows * H;
  float a[2];
  int rank[2] = {0, 0};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int h = lane + 32 * i;
    a[i] = h < H ? fabsf(w[r * H + h]) * (part[r * H + h] + part[plane + r * H + h]) : -INFINITY;
  }
  for (int j = 0; j < H; ++j) {
    const float aj = __shfl_sync(0xffffffffu, a[j >> 5], j & 31);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int h = lane + 32 * i;
      if (aj > a[i] || (aj == a[i] && j < h)) ++rank[i];
    }
  }
  const bool sel0 = lane < H && rank[0] < hsel;
  const bool sel1 = lane + 32 < H && rank[1] < hsel;
  const uint32_t m0 = __ballot_sync(0xffffffffu, sel0);
  const uint32_t m1 = __ballot_sync(0xffffffffu, sel1);
  const uint32_t below = (1u << lane) - 1u;
  if (sel0) {
    const int pos = __popc(m0 & below);
    heads[r * hsel + pos] = lane;
    w_sel[r * hsel + pos] = w[r * H + lane];
  }
  if (sel1) {
    const int pos = __popc(m0) + __popc(m1 & below);
    heads[r * hsel + pos] = lane + 32;
    w_sel[r * hsel + pos] = w[r * H + lane + 32];
  }
  __syncwarp();
  // gather the kept query rows (16-byte chunks)
  const int chunks = d / 8;
  for (int i = lane; i < hsel * chunks; i += 32) {
    const int pos = i / chunks;
    const int c = i % chunks;
    const int h = heads[r * hsel + pos];
    const uint4 v = *reinterpret_cast<const uint4*>(q + (r * H + h) * d + c * 8);
    *reinterpret_cast<uint4*>(q_sel + (r * hsel + pos) * d + c * 8) = v;
  }
}

// Failure-path self-test: one warp waits on a barrier that nothing completes;
// the bounded wait gives up after its limit and records the timeout in *err.
__global__ void wait_timeout_kernel(unsigned* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, err);
  __syncwarp();
}

}  // namespace dsa
