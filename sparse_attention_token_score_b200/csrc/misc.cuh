// Small kernels around the scoring and selection kernels: block mean-pooling of
// keys and the MISA head selection.
#pragma once
#include "common.cuh"
#include <cuda_fp8.h>

namespace dsa {

// Pooled keys ("MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
// Inference", section "Methodology", step 1: the prefix splits into
// M = ceil(L/B) blocks, each represented by its mean-pooled indexing key; the
// HISA review, section 3, uses the same pooled representatives):
//     kbar[b, m, :] = bf16( mean of k[b, mB : min((m+1)B, L), :] )
// The sum runs in fp64, which is exact for bf16 inputs at these block sizes,
// and is rounded to bf16 once (round to nearest even). Every kernel below
// pools blocks m0 .. m0 + nm - 1 of every sequence (grid: batch * nm CTAs).
__global__ void meanpool_kernel(const __nv_bfloat16* __restrict__ k, int L, int d, int B, int M, int m0, int nm,
                                __nv_bfloat16* __restrict__ kbar) {
  const long long b = blockIdx.x / nm;
  const int m = m0 + static_cast<int>(blockIdx.x % nm);
  const long long bm = b * M + m;
  const int s0 = m * B;
  const int s1 = min(s0 + B, L);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    double acc = 0.0;
    for (int s = s0; s < s1; ++s) acc += static_cast<double>(__bfloat162float(k[(b * L + s) * d + c]));
    kbar[bm * d + c] = __double2bfloat16(acc / static_cast<double>(s1 - s0));
  }
}

// The same for bf16 rows of 16-byte multiples (d % 8 == 0, d <= 256): a CTA
// of 256 threads pools one block; each thread reads one 16-byte piece of
// token rows r, r + RPI, ... of the block and accumulates its 8 values in
// fp64; the per-thread partial sums are added per column through shared
// memory. The sums are exact, so the order does not change the result.
__global__ void __launch_bounds__(256) meanpool_vec_kernel(const __nv_bfloat16* __restrict__ k, int L, int d,
                                                           int B, int M, int m0, int nm,
                                                           __nv_bfloat16* __restrict__ kbar) {
  __shared__ double red[32 * 64];             // [rows in flight][d]: RPI * d = 2048
  const long long b = blockIdx.x / nm;
  const int m = m0 + static_cast<int>(blockIdx.x % nm);
  const long long bm = b * M + m;
  const int s0 = m * B;
  const int s1 = min(s0 + B, L);
  const int tpr = d / 8;                      // threads per row (16-byte pieces)
  const int rpi = 256 / tpr;                  // rows in flight
  const int t = threadIdx.x;
  const int r = t / tpr, c = t % tpr;
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
  if (r < rpi) {
    for (int s = s0 + r; s < s1; s += rpi) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(k + (b * L + s) * d) + c);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 8; ++e)
        acc[e] += static_cast<double>(__uint_as_float(((w4[e >> 1] >> (16 * (e & 1))) & 0xffffu) << 16));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[r * d + c * 8 + e] = acc[e];
  }
  __syncthreads();
  if (t < d) {
    const int nrow = min(rpi, s1 - s0);
    double sum = 0.0;
    for (int i = 0; i < nrow; ++i) sum += red[i * d + t];
    kbar[bm * d + t] = __double2bfloat16(sum / static_cast<double>(s1 - s0));
  }
}

// Pooled keys of an FP8 e4m3 key cache, kept in the cache's format: per
// block the fp64 mean of the dequantised keys (code value x per-token scale),
// a scale absmax/448 (absmax rounded to fp32, divided in fp32; 1 when the
// mean is zero) and codes e4m3(mean / scale), rounded to nearest even with
// saturation. 512 threads, d % 4 == 0, d <= 128, rows 4-byte aligned: thread
// (g, c) reads bytes 4c .. 4c + 3 of token rows g, g + G, ... of the block
// (G = 512 / (d / 4) row groups), eight rows and their scales loaded before
// any of them is used, so a block of up to 8 G tokens costs one round trip to
// memory; the G partial sums of a column are added in shared memory. The
// fp64 sums are exact here, so the order does not change the result.
__global__ void __launch_bounds__(512) meanpool_fp8_kernel(const uint8_t* __restrict__ k8,
                                                           const float* __restrict__ ks, int L, int d, int B,
                                                           int M, int m0, int nm, uint8_t* __restrict__ kbar8,
                                                           float* __restrict__ kbar_scale) {
  __shared__ double part[2048];  // [G][d]: G * d = 4 * 512
  __shared__ double red[16];
  const long long b = blockIdx.x / nm;
  const int m = m0 + static_cast<int>(blockIdx.x % nm);
  const long long bm = b * M + m;
  const int s0 = m * B;
  const int s1 = min(s0 + B, L);
  const int tpr = d / 4;  // threads per token row
  const int G = 512 / tpr;  // row groups
  const int g = threadIdx.x / tpr, c = threadIdx.x % tpr;
  if (g < G) {
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int sb = s0 + g; sb < s1; sb += 8 * G) {
      uint32_t v[8];
      float sc[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int s = sb + u * G;
        v[u] = s < s1 ? __ldg(reinterpret_cast<const uint32_t*>(k8 + (b * L + s) * d) + c) : 0u;
        sc[u] = s < s1 ? __ldg(ks + b * L + s) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          __nv_fp8_e4m3 x;
          x.__x = static_cast<__nv_fp8_storage_t>((v[u] >> (8 * e)) & 0xffu);
          acc[e] += static_cast<double>(static_cast<float>(x)) * static_cast<double>(sc[u]);
        }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) part[g * d + 4 * c + e] = acc[e];
  }
  __syncthreads();
  const int col = threadIdx.x;
  double mean = 0.0;
  if (col < d) {
    double sum = 0.0;
    for (int i = 0; i < G; ++i) sum += part[i * d + col];
    mean = sum / static_cast<double>(s1 - s0);
  }
  double a = col < d ? fabs(mean) : 0.0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmax(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((col & 31) == 0) red[col >> 5] = a;
  __syncthreads();
  double amax = 0.0;
  for (int w = 0; w < 16; ++w) amax = fmax(amax, red[w]);
  const float af = static_cast<float>(amax);
  const float scale = af > 0.f ? af / 448.f : 1.f;
  if (col < d)
    kbar8[bm * d + col] = static_cast<uint8_t>(
        __nv_cvt_double_to_fp8(mean / static_cast<double>(scale), __NV_SATFINITE, __NV_E4M3));
  if (col == 0) kbar_scale[bm] = scale;
}

// MISA routing (same page, "Methodology", step 1): per query, the head
// affinity a[h] = |w[h]| * (part0[h] + part1[h]) (the two partial ReLU sums
// over pooled keys from the router kernel); keep the top-hsel heads by
// (a descending, head ascending). Writes the kept heads in ascending order,
// their weights, and gathers their query rows into a compact [rows, hsel, d]
// tensor for the routed scoring pass. One warp per query row; H <= 64.
__global__ void select_heads_kernel(const float* __restrict__ part, long long rows, int H, int hsel,
                                    const float* __restrict__ w, const float* __restrict__ q_scale,
                                    const uint8_t* __restrict__ q, int row_bytes, int* __restrict__ heads,
                                    uint8_t* __restrict__ q_sel, float* __restrict__ w_sel,
                                    float* __restrict__ qs_sel) {
  // part: the router's two partial sums [2][rows, H]; q_scale (FP8 queries,
  // else null) scales the affinity like |w| and is gathered with the rows
  const int lane = threadIdx.x & 31;
  const long long r = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const long long plane = rows * H;
  float a[2];
  int rank[2] = {0, 0};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int h = lane + 32 * i;
    float s = 0.f;
    if (h < H) {
      s = fabsf(w[r * H + h]) * (part[r * H + h] + part[plane + r * H + h]);
      if (q_scale) s *= q_scale[r * H + h];
    }
    a[i] = h < H ? s : -INFINITY;
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
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool sel = i == 0 ? sel0 : sel1;
    if (!sel) continue;
    const int h = lane + 32 * i;
    const int pos = (i == 0 ? 0 : __popc(m0)) + __popc((i == 0 ? m0 : m1) & below);
    heads[r * hsel + pos] = h;
    w_sel[r * hsel + pos] = w[r * H + h];
    if (q_scale) qs_sel[r * hsel + pos] = q_scale[r * H + h];
  }
  __syncwarp();
  // gather the kept query rows (16-byte chunks)
  const int chunks = row_bytes / 16;
  for (int i = lane; i < hsel * chunks; i += 32) {
    const int pos = i / chunks;
    const int c = i % chunks;
    const int h = heads[r * hsel + pos];
    const uint4 v = *reinterpret_cast<const uint4*>(q + (r * H + h) * row_bytes + c * 16);
    *reinterpret_cast<uint4*>(q_sel + (r * hsel + pos) * row_bytes + c * 16) = v;
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
