// C-ABI entry points of the lightning-indexer library (declared in
// include/dsa_indexer.h): host-side validation, workspace carving, TMA tensor
// map encoding and the launch chains of the dense, MISA and HISA paths.
#include "dsa_indexer.h"

#include <cudaTypedefs.h>

#include <climits>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "misc.cuh"
#include "score_tc.cuh"
#include "topk.cuh"

using namespace dsa;

namespace {

constexpr size_t kHdr = 256;
constexpr int kMaxDev = 64;

size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Carve {
  char* base;
  size_t off;
  template <class T>
  T* take(size_t count) {
    T* p = reinterpret_cast<T*>(base + off);
    off += al256(count * sizeof(T));
    return p;
  }
};

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D map over a row-major [rows, D] tensor, 128-byte swizzle, box of one
// 128-byte column block x box_rows rows. Out-of-range rows read as zero.
bool make_tmap(CUtensorMap* m, const void* base, bool fp8, int D, long long rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int elem = fp8 ? 1 : 2;
  cuuint64_t gdim[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t gstr[1] = {static_cast<cuuint64_t>(D) * elem};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<void*>(base), gdim, gstr, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Per-device caches below are filled on first use; concurrent first calls
// from several host threads may both fill an entry (idempotent), hence the
// relaxed atomics.
int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return -1;
  return dev;
}

int num_sms() {
  static std::atomic<int> cache[kMaxDev];
  const int dev = current_device();
  int n = dev >= 0 ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (n == 0) {
    int d = 0;
    cudaGetDevice(&d);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    if (n < 1) n = 1;
    if (dev >= 0) cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <class C>
dsa_status launch_score(const ScoreParams& p, const void* q, long long q_rows, const void* k,
                        long long k_rows, cudaStream_t st) {
  static std::atomic<bool> attr[kMaxDev];
  const int dev = current_device();
  if (dev < 0) return DSA_ERR_UNSUPPORTED;
  if (!attr[dev].load(std::memory_order_relaxed)) {
    if (cudaFuncSetAttribute(score_tc_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess)
      return DSA_ERR_CUDA;
    attr[dev].store(true, std::memory_order_relaxed);
  }
  CUtensorMap tq, tk;
  if (!make_tmap(&tq, q, C::ELEM == 1, C::D, q_rows, C::QROWS)) return DSA_ERR_CUDA;
  if (C::GATHER && !p.blk_tma) tk = tq;  // token gathers copy rows with cp.async (no key map)
  else if (!make_tmap(&tk, k, C::ELEM == 1, C::D, k_rows, C::KROWS)) return DSA_ERR_CUDA;
  int grid = num_sms();
  if (C::ROUTER) {
    const long long G = static_cast<long long>(p.batch) * ((p.T + C::QPT - 1) / C::QPT);
    if (G < grid) grid = static_cast<int>(G);
  }
  score_tc_kernel<C><<<grid, C::NTHREADS, C::SMEM_BYTES, st>>>(tq, tk, p);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Dense / routed / block scoring, bf16: N = 256 columns = (256 / H) queries x H heads.
dsa_status run_scores_bf16(int D, int H, const ScoreParams& p, const void* q, long long q_rows,
                           const void* k, long long k_rows, cudaStream_t st) {
#ifndef DSA_EPIW
#define DSA_EPIW 8
#endif
#define DSA_CASE(DD, HH)                                                                          \
  if (D == DD && H == HH)                                                                         \
    return launch_score<                                                                          \
        ScoreCfg<2, DD, HH, 256 / HH, ScoreMode::kTma, (DD == 128 ? 4 : 8), DSA_EPIW>>(          \
        p, q, q_rows, k, k_rows, st);
  DSA_CASE(64, 8) DSA_CASE(64, 16) DSA_CASE(64, 32) DSA_CASE(64, 64)
  DSA_CASE(128, 8) DSA_CASE(128, 16) DSA_CASE(128, 32) DSA_CASE(128, 64)
#undef DSA_CASE
  return DSA_ERR_UNSUPPORTED;
}

// FP8 decode scoring: one query per group, N = H.
#ifndef DSA_FP8_NSTAGE
#define DSA_FP8_NSTAGE 8
#endif
dsa_status run_scores_fp8(int D, int H, const ScoreParams& p, const void* q, long long q_rows,
                          const void* k, long long k_rows, cudaStream_t st) {
  if (D == 128 && H == 64)
    return launch_score<ScoreCfg<1, 128, 64, 1, ScoreMode::kTma, DSA_FP8_NSTAGE>>(p, q, q_rows, k, k_rows, st);
  if (D == 128 && H == 32)
    return launch_score<ScoreCfg<1, 128, 32, 1, ScoreMode::kTma, DSA_FP8_NSTAGE>>(p, q, q_rows, k, k_rows, st);
  return DSA_ERR_UNSUPPORTED;
}

// MISA router: M = 128 (query, head) rows, 256 pooled keys per tile.
dsa_status run_router(int D, int H, const ScoreParams& p, const void* q, long long q_rows,
                      const void* kbar, long long k_rows, cudaStream_t st) {
#define DSA_CASE(DD, HH)                                                                          \
  if (D == DD && H == HH)                                                                         \
    return launch_score<ScoreCfg<2, DD, HH, 128 / HH, ScoreMode::kRouter, (DD == 128 ? 2 : 4)>>( \
        p, q, q_rows, kbar, k_rows, st);
  DSA_CASE(64, 8) DSA_CASE(64, 16) DSA_CASE(64, 32) DSA_CASE(64, 64)
  DSA_CASE(128, 8) DSA_CASE(128, 16) DSA_CASE(128, 32) DSA_CASE(128, 64)
#undef DSA_CASE
  return DSA_ERR_UNSUPPORTED;
}

// Gathered re-scoring (MISA-dagger candidates, HISA surviving blocks).
// When blk is a multiple of 128, every 128-row tile is one contiguous key
// run and is fetched with TMA; otherwise rows are gathered with cp.async.
#ifndef DSA_GATHER_NS
#define DSA_GATHER_NS 5
#endif
#ifndef DSA_GATHER_NQ
#define DSA_GATHER_NQ 2
#endif
dsa_status run_gather(int D, int H, ScoreParams p, const void* q, long long q_rows,
                      cudaStream_t st) {
  p.blk_tma = (p.blk % 128 == 0) ? 1 : 0;
  const long long k_rows = static_cast<long long>(p.batch) * p.L_tok;
  if (D == 128 && H == 64)
    return launch_score<ScoreCfg<2, 128, 64, 1, ScoreMode::kGather, DSA_GATHER_NS, 8, DSA_GATHER_NQ>>(
        p, q, q_rows, p.kg, k_rows, st);
  if (D == 128 && H == 32)
    return launch_score<ScoreCfg<2, 128, 32, 1, ScoreMode::kGather, 6>>(p, q, q_rows, p.kg, k_rows, st);
  return DSA_ERR_UNSUPPORTED;
}

// ws: the call's workspace; its first word is the device status the
// kernel's bounded waits report to.
template <class C>
dsa_status launch_topk_cfg(const TopkParams& tp, cudaStream_t st) {
  static std::atomic<int> ctas[kMaxDev];
  const int dev = current_device();
  if (dev < 0) return DSA_ERR_UNSUPPORTED;
  int occ = ctas[dev].load(std::memory_order_relaxed);
  if (occ == 0) {
    if (cudaFuncSetAttribute(topk_rows_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, topk_rows_kernel<C>, C::NT, C::BYTES) !=
            cudaSuccess ||
        occ < 1)
      return DSA_ERR_CUDA;
    ctas[dev].store(occ, std::memory_order_relaxed);
  }
  long long grid = static_cast<long long>(num_sms()) * occ;
  if (tp.rows < grid) grid = tp.rows;
  topk_rows_kernel<C><<<static_cast<int>(grid), C::NT, C::BYTES, st>>>(tp);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ws: the call's workspace (its first word is the device status word).
// Rows up to 32768 scores use the short-row layout (4 CTAs of 256 threads per
// SM); longer rows use 2 CTAs of 512 threads per SM when there are enough rows
// to fill the GPU, else one 512-thread CTA (with more loads in flight) per row.
dsa_status launch_topk(void* ws, TopkParams tp, cudaStream_t st) {
  tp.err = static_cast<unsigned*>(ws);
  if (tp.Lrow <= TkShort::MAX_ROW) return launch_topk_cfg<TkShort>(tp, st);
  if (tp.rows >= static_cast<long long>(num_sms()) * TkLong::MIN_CTAS) return launch_topk_cfg<TkLong>(tp, st);
  return launch_topk_cfg<TkWide>(tp, st);
}

bool h_supported_bf16(int H) { return H == 8 || H == 16 || H == 32 || H == 64; }

dsa_status validate(const dsa_indexer_args* a, bool bf16_only) {
  if (!a || !a->q || !a->k || !a->w) return DSA_ERR_ARG;
  if (a->batch < 1 || a->T < 1 || a->L < 1 || a->H < 1 || a->d < 1 || a->q_offset < 0)
    return DSA_ERR_ARG;
  if (a->qk_dtype != DSA_BF16 && a->qk_dtype != DSA_FP8_E4M3) return DSA_ERR_ARG;
  if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->w, 16)) return DSA_ERR_ARG;
  const bool fp8 = a->qk_dtype == DSA_FP8_E4M3;
  if (fp8) {
    if (!a->q_scale || !a->k_scale) return DSA_ERR_ARG;
    if (!aligned(a->q_scale, 16) || !aligned(a->k_scale, 16)) return DSA_ERR_ARG;
  }
  if (a->q_offset > (1LL << 40)) return DSA_ERR_ARG;
  if (static_cast<long long>(a->batch) * a->T * a->H > INT_MAX ||
      static_cast<long long>(a->batch) * a->L > INT_MAX)
    return DSA_ERR_UNSUPPORTED;
  if (a->d != 64 && a->d != 128) return DSA_ERR_UNSUPPORTED;
  if (fp8) {
    if (bf16_only) return DSA_ERR_UNSUPPORTED;
    if (a->d != 128 || (a->H != 32 && a->H != 64)) return DSA_ERR_UNSUPPORTED;
  } else if (!h_supported_bf16(a->H)) {
    return DSA_ERR_UNSUPPORTED;
  }
  return DSA_OK;
}

dsa_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return DSA_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return DSA_ERR_ARG;
  if (ws_bytes < need) return DSA_ERR_WORKSPACE;
  return DSA_OK;
}

ScoreParams base_params(const dsa_indexer_args* a, unsigned* err) {
  ScoreParams p{};
  p.batch = a->batch;
  p.T = a->T;
  p.Lk = a->L;
  p.L_tok = a->L;
  p.q_offset = a->q_offset;
  p.pstride = 1;
  p.w = a->w;
  p.q_scale = a->q_scale;
  p.k_scale = a->k_scale;
  p.blk = 1;
  p.err = err;
  return p;
}

TopkParams topk_params(const float* scores, long long rows, long long ld, int T, long long q_offset,
                       int pstride, int row_len, int k, int32_t* oi, float* os, const int* cand,
                       int n_slots, int blk) {
  TopkParams t{};
  t.scores = scores;
  t.ld = ld;
  t.rows = rows;
  t.T = T;
  t.q_offset = q_offset;
  t.pstride = pstride;
  t.Lrow = row_len;
  t.k = k;
  t.out_idx = oi;
  t.out_score = os;
  t.cand = cand;
  t.n_slots = n_slots;
  t.blk = blk;
  t.err = nullptr;
  return t;
}

#define DSA_TRY(x)                  \
  do {                              \
    const dsa_status s_ = (x);      \
    if (s_ != DSA_OK) return s_;    \
  } while (0)

dsa_status clear_status(void* ws, cudaStream_t st) {
  return cudaMemsetAsync(ws, 0, 4, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

long long blocks_of(long long L, int block) { return (L + block - 1) / block; }

}  // namespace

extern "C" {

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case DSA_ERR_WORKSPACE: return "workspace too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

dsa_status dsa_device_status(void* workspace, void* stream) {
  if (!workspace) return DSA_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, workspace, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemset(workspace, 0, 4) != cudaSuccess) return DSA_ERR_CUDA;
  return word ? DSA_ERR_TIMEOUT : DSA_OK;
}

dsa_status dsa_selftest_wait_timeout(void* workspace, size_t ws_bytes, void* stream) {
  DSA_TRY(check_ws(workspace, ws_bytes, kHdr));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(workspace, st));
  wait_timeout_kernel<<<1, 32, 0, st>>>(static_cast<unsigned*>(workspace));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

size_t indexer_workspace_size(const dsa_indexer_args* a, int topk) {
  (void)topk;
  if (!a || a->batch < 1 || a->T < 1 || a->L < 1) return 0;
  return kHdr + al256(static_cast<size_t>(a->batch) * a->T * a->L * sizeof(float));
}

dsa_status indexer_scores(const dsa_indexer_args* a, float* out, long long ld, void* ws,
                          size_t ws_bytes, void* stream) {
  DSA_TRY(validate(a, false));
  if (!out || ld < a->L || !aligned(out, 4)) return DSA_ERR_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, kHdr));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  ScoreParams p = base_params(a, static_cast<unsigned*>(ws));
  p.out = out;
  p.ldo = ld;
  const long long q_rows = static_cast<long long>(a->batch) * a->T * a->H;
  const long long k_rows = static_cast<long long>(a->batch) * a->L;
  if (a->qk_dtype == DSA_FP8_E4M3) return run_scores_fp8(a->d, a->H, p, a->q, q_rows, a->k, k_rows, st);
  return run_scores_bf16(a->d, a->H, p, a->q, q_rows, a->k, k_rows, st);
}

dsa_status indexer_score_gathered(const dsa_indexer_args* a, const int32_t* cand, int n_slots,
                                  int blk, float* out, long long ld, void* ws, size_t ws_bytes,
                                  void* stream) {
  DSA_TRY(validate(a, true));
  if (!cand || !out || n_slots < 1 || blk < 1 || !aligned(cand, 4) || !aligned(out, 4))
    return DSA_ERR_ARG;
  if (static_cast<long long>(n_slots) * blk > INT_MAX / 2) return DSA_ERR_UNSUPPORTED;
  if (ld < static_cast<long long>(n_slots) * blk) return DSA_ERR_ARG;
  if (a->d != 128 || (a->H != 32 && a->H != 64)) return DSA_ERR_UNSUPPORTED;
  DSA_TRY(check_ws(ws, ws_bytes, kHdr));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  ScoreParams pg = base_params(a, static_cast<unsigned*>(ws));
  pg.out = out;
  pg.ldo = ld;
  pg.kg = static_cast<const __nv_bfloat16*>(a->k);
  pg.cand = cand;
  pg.n_slots = n_slots;
  pg.blk = blk;
  pg.n_compact = n_slots * blk;
  return run_gather(a->d, a->H, pg, a->q, static_cast<long long>(a->batch) * a->T * a->H, st);
}

dsa_status indexer_topk_rows(const float* scores, long long rows, long long ld, int T,
                             long long q_offset, int pstride, int row_len, int topk,
                             const int32_t* cand, int n_slots, int blk, int32_t* out_idx,
                             float* out_score, void* ws, size_t ws_bytes, void* stream) {
  if (!scores || !out_idx || rows < 1 || T < 1 || row_len < 0 || ld < row_len || topk < 1 ||
      pstride < 0 || q_offset < 0 || topk > (1 << 24))
    return DSA_ERR_ARG;
  if (cand && (n_slots < 1 || blk < 1 || static_cast<long long>(n_slots) * blk < row_len))
    return DSA_ERR_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, kHdr));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  return launch_topk(ws, topk_params(scores, rows, ld, T, q_offset, pstride, row_len, topk, out_idx,
                                 out_score, cand, cand ? n_slots : 0, cand ? blk : 1),
                     st);
}

dsa_status indexer_score_topk(const dsa_indexer_args* a, int topk, int32_t* out_idx,
                              float* out_score, void* ws, size_t ws_bytes, void* stream) {
  DSA_TRY(validate(a, false));
  if (!out_idx || topk < 1 || topk > (1 << 24)) return DSA_ERR_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, indexer_workspace_size(a, topk)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  Carve c{static_cast<char*>(ws), kHdr};
  float* scores = c.take<float>(static_cast<size_t>(a->batch) * a->T * a->L);
  ScoreParams p = base_params(a, static_cast<unsigned*>(ws));
  p.out = scores;
  p.ldo = a->L;
  const long long q_rows = static_cast<long long>(a->batch) * a->T * a->H;
  const long long k_rows = static_cast<long long>(a->batch) * a->L;
  if (a->qk_dtype == DSA_FP8_E4M3)
    DSA_TRY(run_scores_fp8(a->d, a->H, p, a->q, q_rows, a->k, k_rows, st));
  else
    DSA_TRY(run_scores_bf16(a->d, a->H, p, a->q, q_rows, a->k, k_rows, st));
  return launch_topk(ws, topk_params(scores, static_cast<long long>(a->batch) * a->T, a->L, a->T,
                                 a->q_offset, 1, a->L, topk, out_idx, out_score, nullptr, 0, 1),
                     st);
}

dsa_status dsa_meanpool_keys(const void* k, int batch, int L, int d, int block, void* kbar,
                             void* stream) {
  if (!k || !kbar || batch < 1 || L < 1 || d < 1 || d > 1024 || block < 1) return DSA_ERR_ARG;
  const long long M = blocks_of(L, block);
  if (static_cast<long long>(batch) * M > INT_MAX) return DSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  meanpool_kernel<<<static_cast<int>(batch * M), d < 128 ? d : 128, 0, st>>>(
      static_cast<const __nv_bfloat16*>(k), L, d, block, static_cast<int>(M),
      static_cast<__nv_bfloat16*>(kbar));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

size_t misa_workspace_size(const dsa_indexer_args* a, int block, int h, int topk, int kprime) {
  (void)topk;
  if (!a || a->batch < 1 || a->T < 1 || a->L < 1 || a->H < 1 || a->d < 1 || block < 1 || h < 1)
    return 0;
  const size_t BT = static_cast<size_t>(a->batch) * a->T;
  const size_t M = static_cast<size_t>(blocks_of(a->L, block));
  size_t n = kHdr;
  n += al256(a->batch * M * a->d * 2);            // pooled keys
  n += al256(2 * BT * a->H * sizeof(float));      // router partial sums
  n += al256(BT * h * a->d * 2);                  // gathered queries of the kept heads
  n += al256(BT * h * sizeof(float));             // their weights
  n += al256(BT * h * sizeof(int32_t));           // kept heads
  n += al256(BT * a->L * sizeof(float));          // routed scores
  if (kprime > 0) {
    n += al256(BT * kprime * sizeof(int32_t));    // candidates
    n += al256(BT * kprime * sizeof(float));      // full-H candidate scores
  }
  return n;
}

dsa_status misa_route_score_topk(const dsa_indexer_args* a, int block, int h, int topk, int kprime,
                                 int32_t* out_idx, float* out_score, int32_t* out_heads,
                                 int32_t* out_cand, void* ws, size_t ws_bytes, void* stream) {
  DSA_TRY(validate(a, true));
  if (!out_idx || block < 1 || h < 1 || h > a->H || topk < 1 || topk > (1 << 24) || kprime < 0 ||
      kprime > (1 << 24))
    return DSA_ERR_ARG;
  if (!h_supported_bf16(h) || a->H > 64) return DSA_ERR_UNSUPPORTED;
  if (kprime > 0 && (a->d != 128 || (a->H != 32 && a->H != 64))) return DSA_ERR_UNSUPPORTED;
  DSA_TRY(check_ws(ws, ws_bytes, misa_workspace_size(a, block, h, topk, kprime)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  unsigned* err = static_cast<unsigned*>(ws);
  const long long BT = static_cast<long long>(a->batch) * a->T;
  const long long M = blocks_of(a->L, block);
  if (static_cast<long long>(a->batch) * M > INT_MAX) return DSA_ERR_UNSUPPORTED;

  Carve c{static_cast<char*>(ws), kHdr};
  __nv_bfloat16* kbar = c.take<__nv_bfloat16>(static_cast<size_t>(a->batch) * M * a->d);
  float* part = c.take<float>(2 * static_cast<size_t>(BT) * a->H);
  __nv_bfloat16* q_sel = c.take<__nv_bfloat16>(static_cast<size_t>(BT) * h * a->d);
  float* w_sel = c.take<float>(static_cast<size_t>(BT) * h);
  int32_t* heads_ws = c.take<int32_t>(static_cast<size_t>(BT) * h);
  float* routed = c.take<float>(static_cast<size_t>(BT) * a->L);
  int32_t* heads = out_heads ? out_heads : heads_ws;

  // 1. pooled keys
  DSA_TRY(dsa_meanpool_keys(a->k, a->batch, a->L, a->d, block, kbar, stream));
  // 2. router affinities (partial ReLU sums over visible pooled keys)
  ScoreParams pr = base_params(a, err);
  pr.Lk = static_cast<int>(M);
  pr.pstride = block;
  pr.out = part;
  DSA_TRY(run_router(a->d, a->H, pr, a->q, BT * a->H, kbar, a->batch * M, st));
  // 3. top-h heads per query; gather their query rows and weights
  select_heads_kernel<<<static_cast<int>((BT + 7) / 8), 256, 0, st>>>(
      part, BT, a->H, h, a->w, static_cast<const __nv_bfloat16*>(a->q), a->d, heads, q_sel, w_sel);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  // 4. routed token scores with the kept heads only
  ScoreParams ps = base_params(a, err);
  ps.w = w_sel;
  ps.out = routed;
  ps.ldo = a->L;
  DSA_TRY(run_scores_bf16(a->d, h, ps, q_sel, BT * h, a->k, static_cast<long long>(a->batch) * a->L, st));
  if (kprime == 0) {
    return launch_topk(ws, topk_params(routed, BT, a->L, a->T, a->q_offset, 1, a->L, topk, out_idx,
                                   out_score, nullptr, 0, 1),
                       st);
  }
  // 5. MISA-dagger: top-k' candidates, full-H re-score, top-k
  int32_t* cand_ws = c.take<int32_t>(static_cast<size_t>(BT) * kprime);
  float* compact = c.take<float>(static_cast<size_t>(BT) * kprime);
  int32_t* cand = out_cand ? out_cand : cand_ws;
  DSA_TRY(launch_topk(ws, topk_params(routed, BT, a->L, a->T, a->q_offset, 1, a->L, kprime, cand,
                                  nullptr, nullptr, 0, 1),
                      st));
  ScoreParams pg = base_params(a, err);
  pg.out = compact;
  pg.ldo = kprime;
  pg.kg = static_cast<const __nv_bfloat16*>(a->k);
  pg.cand = cand;
  pg.n_slots = kprime;
  pg.blk = 1;
  pg.n_compact = kprime;
  DSA_TRY(run_gather(a->d, a->H, pg, a->q, BT * a->H, st));
  return launch_topk(ws, topk_params(compact, BT, kprime, a->T, a->q_offset, 0, kprime, topk, out_idx,
                                 out_score, cand, kprime, 1),
                     st);
}

size_t hisa_workspace_size(const dsa_indexer_args* a, int block, int m, int topk) {
  (void)topk;
  if (!a || a->batch < 1 || a->T < 1 || a->L < 1 || a->d < 1 || block < 1 || m < 1) return 0;
  const size_t BT = static_cast<size_t>(a->batch) * a->T;
  const size_t M = static_cast<size_t>(blocks_of(a->L, block));
  size_t n = kHdr;
  n += al256(a->batch * M * a->d * 2);                        // pooled keys
  n += al256(BT * M * sizeof(float));                         // block scores
  n += al256(BT * m * sizeof(int32_t));                       // kept blocks
  n += al256(BT * static_cast<size_t>(m) * block * sizeof(float));  // token scores of kept blocks
  return n;
}

dsa_status hisa_block_filter_topk(const dsa_indexer_args* a, int block, int m, int topk,
                                  int32_t* out_idx, float* out_score, int32_t* out_blocks,
                                  void* ws, size_t ws_bytes, void* stream) {
  DSA_TRY(validate(a, true));
  if (!out_idx || block < 1 || m < 1 || topk < 1 || topk > (1 << 24)) return DSA_ERR_ARG;
  if (static_cast<long long>(m) * block > INT_MAX / 2) return DSA_ERR_UNSUPPORTED;
  if (a->d != 128 || (a->H != 32 && a->H != 64)) return DSA_ERR_UNSUPPORTED;
  DSA_TRY(check_ws(ws, ws_bytes, hisa_workspace_size(a, block, m, topk)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  unsigned* err = static_cast<unsigned*>(ws);
  const long long BT = static_cast<long long>(a->batch) * a->T;
  const long long M = blocks_of(a->L, block);
  if (static_cast<long long>(a->batch) * M > INT_MAX) return DSA_ERR_UNSUPPORTED;
  const int ncomp = m * block;

  Carve c{static_cast<char*>(ws), kHdr};
  __nv_bfloat16* kbar = c.take<__nv_bfloat16>(static_cast<size_t>(a->batch) * M * a->d);
  float* bscore = c.take<float>(static_cast<size_t>(BT) * M);
  int32_t* blocks_ws = c.take<int32_t>(static_cast<size_t>(BT) * m);
  float* compact = c.take<float>(static_cast<size_t>(BT) * ncomp);
  int32_t* blocks = out_blocks ? out_blocks : blocks_ws;

  // 1. pooled keys
  DSA_TRY(dsa_meanpool_keys(a->k, a->batch, a->L, a->d, block, kbar, stream));
  // 2. block scores on the pooled keys (block m visible iff m * block <= p_t)
  ScoreParams pb = base_params(a, err);
  pb.Lk = static_cast<int>(M);
  pb.pstride = block;
  pb.out = bscore;
  pb.ldo = M;
  DSA_TRY(run_scores_bf16(a->d, a->H, pb, a->q, BT * a->H, kbar, a->batch * M, st));
  // 3. top-m blocks
  DSA_TRY(launch_topk(ws, topk_params(bscore, BT, M, a->T, a->q_offset, block, static_cast<int>(M), m,
                                  blocks, nullptr, nullptr, 0, 1),
                      st));
  // 4. token scores inside the kept blocks (compact rows of m * block)
  ScoreParams pg = base_params(a, err);
  pg.out = compact;
  pg.ldo = ncomp;
  pg.kg = static_cast<const __nv_bfloat16*>(a->k);
  pg.cand = blocks;
  pg.n_slots = m;
  pg.blk = block;
  pg.n_compact = ncomp;
  DSA_TRY(run_gather(a->d, a->H, pg, a->q, BT * a->H, st));
  // 5. top-k tokens
  return launch_topk(ws, topk_params(compact, BT, ncomp, a->T, a->q_offset, 0, ncomp, topk, out_idx,
                                 out_score, blocks, m, block),
                     st);
}

}  // extern "C"

// ------------------------------------------------------------------ no-allocation variant
// Dense score + top-k for callers that cannot allocate device memory. The
// scores scratch lives in a file-scope __device__ array that every device
// loading this library reserves until exit. Host code must not pass
// `g_noalloc_scratch` itself to a kernel: on the host that name is only a
// stand-in for the device symbol. The device address is looked up once per
// device with cudaGetSymbolAddress (the first call on a device, with that
// device current) and cached.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDev] = {nullptr};

dsa_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDev) return DSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return DSA_OK;
}

}  // namespace

extern "C" dsa_status indexer_score_topk_noalloc(const dsa_indexer_args* a, int topk,
                                                 int32_t* out_idx, float* out_score,
                                                 void* stream) {
  DSA_TRY(validate(a, false));
  if (!out_idx || topk < 1 || topk > (1 << 24)) return DSA_ERR_ARG;
  if (indexer_workspace_size(a, topk) > kNoAllocScratchBytes) return DSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  DSA_TRY(noalloc_scratch(&scratch));
  // Same launches as indexer_score_topk; its status word (first 4 bytes of
  // the scratch) is cleared on the stream before the kernels run.
  return indexer_score_topk(a, topk, out_idx, out_score, scratch, kNoAllocScratchBytes, stream);
}
