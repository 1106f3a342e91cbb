// DoSA certified pruning, the per-query and per-key inputs of the bound pass
// ("DoSA: Dots Sparse Attention" review, section 3: screening dot products,
// bound evaluation; the certificate combines a threshold that the k-th score
// reaches, a non-negative projection of the positive-weight heads and an
// aggregate of the negative-weight heads).
//
// For query t with heads h (x_h = q_h . k_s), the screened set S_t (the
// n_screen heads with the largest |w_h| * ||q_h||), P_t = unscreened heads
// with w_h > 0, N_t = unscreened heads with w_h < 0:
//   I[t,s] <= sum_{h in S_t} w_h ReLU(x_h)
//             + 1/2 (k_s . v_P + A_P ||k_s||)            ReLU(x) = (x + |x|) / 2, |x_h| <= ||q_h|| ||k_s||
//             - ReLU(k_s . v_N)                          ReLU is subadditive
// with v_P = sum_P w_h q_h, A_P = sum_P w_h ||q_h||, v_N = sum_N |w_h| q_h.
// The bound pass evaluates it as an indexer score over augmented heads on the
// tensor cores: the screened heads with their weights, bf16(v_P) with +1/2,
// -bf16(v_P) with -1/2 (together 1/2 k.v_P), bf16(v_N) with -1, plus
// c_t * ||k_s|| in the epilogue, where c_t = A_P / 2 + the rounding of
// v_P, v_N to bf16 (||v - bf16(v)|| bounds the change of k.v per unit
// ||k||) + a relative slack of 1e-4 of sum_h |w_h| ||q_h|| + ||v_P|| + ||v_N||,
// which covers the fp32 accumulation of this bound and of the scores it is
// compared with.
#pragma once
#include "common.cuh"

namespace dsa {

constexpr double kDosaSlack = 1e-4;

// One warp per query row r: writes q_aug [rows, HA, D] bf16, w_aug [rows, HA]
// and cb[r] = c_t. HA = n_screen + 3 augmented heads (the rest zero). Lanes
// own D / 32 consecutive dimensions, so every head row is read with one
// coalesced load per lane.
template <int D>
__global__ void dosa_prep_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w, long long rows,
                                 int H, int n_screen, int HA, __nv_bfloat16* __restrict__ q_aug,
                                 float* __restrict__ w_aug, float* __restrict__ cb) {
  constexpr int DPL = D / 32;  // dimensions per lane (4 or 2)
  const int lane = threadIdx.x & 31;
  const long long r = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const __nv_bfloat16* qr = q + r * H * D;
  const float* wr = w + r * H;
  auto load = [&](int h, float (&v)[DPL]) {
    if constexpr (DPL == 4) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(qr + h * D) + lane);
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
      v[0] = __low2float(a); v[1] = __high2float(a); v[2] = __low2float(b); v[3] = __high2float(b);
    } else {
      const __nv_bfloat162 a = __ldg(reinterpret_cast<const __nv_bfloat162*>(qr + h * D) + lane);
      v[0] = __low2float(a); v[1] = __high2float(a);
    }
  };
  // ||q_h||: squares of bf16 values are exact in fp32; lane h % 32 keeps head h's
  double nrm[2] = {0.0, 0.0};
  for (int h = 0; h < H; ++h) {
    float v[DPL];
    load(h, v);
    float sq = 0.f;
#pragma unroll
    for (int c = 0; c < DPL; ++c) sq = fmaf(v[c], v[c], sq);
    double sd = sq;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sd += __shfl_xor_sync(0xffffffffu, sd, o);
    if (lane == (h & 31)) nrm[h >> 5] = sqrt(sd);
  }
  float g[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int h = lane + 32 * i;
    g[i] = h < H ? static_cast<float>(fabs(static_cast<double>(wr[h])) * nrm[i]) : -INFINITY;
  }
  // screened heads: rank by (g descending, h ascending)
  int rank[2] = {0, 0};
  for (int j = 0; j < H; ++j) {
    const float gj = __shfl_sync(0xffffffffu, g[j >> 5], j & 31);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int h = lane + 32 * i;
      if (gj > g[i] || (gj == g[i] && j < h)) ++rank[i];
    }
  }
  const bool scr0 = lane < H && rank[0] < n_screen;
  const bool scr1 = lane + 32 < H && rank[1] < n_screen;
  const uint32_t m0 = __ballot_sync(0xffffffffu, scr0);
  const uint32_t m1 = __ballot_sync(0xffffffffu, scr1);
  // aggregates (fp64): A_P, sum |w| ||q|| (slack scale)
  double ap = 0.0, wq = 0.0;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int h = lane + 32 * i;
    if (h < H) {
      const double wh = wr[h];
      wq += fabs(wh) * nrm[i];
      const bool scr = i == 0 ? scr0 : scr1;
      if (!scr && wh > 0.0) ap += wh * nrm[i];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ap += __shfl_xor_sync(0xffffffffu, ap, o);
    wq += __shfl_xor_sync(0xffffffffu, wq, o);
  }
  // v_P, v_N over this lane's dimensions (fp64)
  double vp[DPL], vn[DPL];
#pragma unroll
  for (int c = 0; c < DPL; ++c) { vp[c] = 0.0; vn[c] = 0.0; }
  for (int h = 0; h < H; ++h) {
    const bool scr = h < 32 ? ((m0 >> h) & 1u) : ((m1 >> (h - 32)) & 1u);
    const double wh = __ldg(wr + h);
    if (scr || wh == 0.0) continue;
    float v[DPL];
    load(h, v);
#pragma unroll
    for (int c = 0; c < DPL; ++c) {
      if (wh > 0.0) vp[c] = fma(wh, static_cast<double>(v[c]), vp[c]);
      else vn[c] = fma(-wh, static_cast<double>(v[c]), vn[c]);
    }
  }
  // bf16 roundings, their errors and the norms of v_P, v_N
  double ep = 0.0, en = 0.0, np2 = 0.0, nn2 = 0.0;
  __nv_bfloat16 bp[DPL], bn[DPL];
#pragma unroll
  for (int c = 0; c < DPL; ++c) {
    bp[c] = __double2bfloat16(vp[c]);
    bn[c] = __double2bfloat16(vn[c]);
    const double dp = vp[c] - static_cast<double>(__bfloat162float(bp[c]));
    const double dn = vn[c] - static_cast<double>(__bfloat162float(bn[c]));
    ep += dp * dp;
    en += dn * dn;
    np2 += vp[c] * vp[c];
    nn2 += vn[c] * vn[c];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ep += __shfl_xor_sync(0xffffffffu, ep, o);
    en += __shfl_xor_sync(0xffffffffu, en, o);
    np2 += __shfl_xor_sync(0xffffffffu, np2, o);
    nn2 += __shfl_xor_sync(0xffffffffu, nn2, o);
  }
  // augmented rows: screened heads (ascending), v_P, -v_P, v_N, zeros
  __nv_bfloat16* qa = q_aug + r * HA * D;
  const int ns = __popc(m0) + __popc(m1);
  uint32_t left0 = m0, left1 = m1;
  for (int a = 0; a < HA; ++a) {
    int src = -1;
    if (a < ns) {  // the a-th screened head: lowest remaining bit
      if (left0) { src = __ffs(left0) - 1; left0 &= left0 - 1u; }
      else { src = 32 + __ffs(left1) - 1; left1 &= left1 - 1u; }
    }
#pragma unroll
    for (int c = 0; c < DPL; ++c) {
      const int col = lane * DPL + c;
      __nv_bfloat16 v = __float2bfloat16(0.f);
      if (src >= 0) v = qr[src * D + col];
      else if (a == ns) v = bp[c];
      else if (a == ns + 1) v = __hneg(bp[c]);
      else if (a == ns + 2) v = bn[c];
      qa[a * D + col] = v;
    }
    if (lane == 0) {
      float wa = 0.f;
      if (src >= 0) wa = wr[src];
      else if (a == ns) wa = 0.5f;
      else if (a == ns + 1) wa = -0.5f;
      else if (a == ns + 2) wa = -1.f;
      w_aug[r * HA + a] = wa;
    }
  }
  if (lane == 0) {
    // the fp32 sums of squares above are within 1e-6 of their exact values,
    // far inside the 1e-4 slack
    const double c = 0.5 * ap + 0.5 * sqrt(ep) + sqrt(en) + kDosaSlack * (wq + sqrt(np2) + sqrt(nn2));
    cb[r] = static_cast<float>(c * (1.0 + 1e-6));  // rounded up into fp32
  }
}

// ||k_s|| of every key (fp64 sum of exact bf16 squares, rounded up into fp32).
template <int D>
__global__ void key_norm_kernel(const __nv_bfloat16* __restrict__ k, long long n, float* __restrict__ kn) {
  for (long long s = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; s < n;
       s += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4* row = reinterpret_cast<const uint4*>(k + s * D);
    double acc = 0.0;
#pragma unroll 4
    for (int i = 0; i < D / 8; ++i) {
      const uint4 u = __ldg(row + i);
      const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const double v = __bfloat162float(e[j]);
        acc += v * v;
      }
    }
    kn[s] = static_cast<float>(sqrt(acc) * (1.0 + 1e-6));
  }
}

}  // namespace dsa
