// C-ABI entry points of the lightning-indexer library (declared in
// include/dsa_indexer.h): host-side validation, workspace carving, TMA tensor
// map encoding and the launch chains of the dense, MISA and HISA paths.
#include "dsa_indexer.h"

#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "dosa.cuh"
#include "misc.cuh"
#include "score_inv.cuh"
#include "score_tc.cuh"
#include "topk.cuh"

using namespace dsa;

namespace {

constexpr size_t kHdr = 256;
constexpr int kMaxDev = 64;

size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
long long blocks_of(long long L, int block) { return (L + block - 1) / block; }

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
// `stride` is the distance between rows in elements (D for a dense tensor;
// S * D views every S-th row).
bool make_tmap(CUtensorMap* m, const void* base, bool fp8, int D, long long rows, int box_rows,
               long long stride = 0) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int elem = fp8 ? 1 : 2;
  cuuint64_t gdim[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t gstr[1] = {static_cast<cuuint64_t>(stride > 0 ? stride : D) * elem};
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

// ------------------------------------------------------------ launch profiling (dsa_profile_*)
// While enabled, every kernel launch of the library is bracketed by a pair of
// CUDA events recorded on the launching stream and filed under a name: the
// current stage of the chain (if any) and the kernel's label.
namespace prof {
std::atomic<bool> on{false};
std::mutex mu;
struct Rec {
  std::string name;
  cudaEvent_t a, b;
};
std::vector<Rec> recs;
thread_local std::string stage;  // nested stages joined by '/'

struct Stage {  // names the launches made while it lives ("routed", "sample pass", ...)
  size_t prev;
  explicit Stage(const char* s) : prev(stage.size()) { set(s); }
  // replaces this stage's name (the steps of one chain, one after another)
  void set(const char* s) {
    stage.resize(prev);
    if (!stage.empty()) stage += '/';
    stage += s;
  }
  ~Stage() { stage.resize(prev); }
};

struct Launch {  // construct right before a launch, destroy right after it
  cudaStream_t st;
  cudaEvent_t a = nullptr, b = nullptr;
  std::string name;
  Launch(cudaStream_t s, const char* label) : st(s) {
    if (!on.load(std::memory_order_relaxed)) return;
    name = stage.empty() ? std::string(label) : stage + ": " + label;
    if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) { a = b = nullptr; return; }
    cudaEventRecord(a, st);
  }
  ~Launch() {
    if (!a) return;
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> lock(mu);
    recs.push_back({name, a, b});
  }
};
}  // namespace prof

template <class C>
dsa_status launch_score(const ScoreParams& p, const void* q, long long q_rows, const void* k,
                        long long k_rows, cudaStream_t st, long long k_stride = 0) {
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
  else if (!make_tmap(&tk, k, C::ELEM == 1, C::D, k_rows, C::KROWS, k_stride)) return DSA_ERR_CUDA;
  int grid = num_sms() * C::CTAS;
  if (C::ROUTER) {
    const long long G = static_cast<long long>(p.batch) * ((p.T + C::QPT - 1) / C::QPT);
    if (G < grid) grid = static_cast<int>(G);
  }
  prof::Launch pl(st, C::ROUTER ? "score_tc router" : C::GATHER ? "score_tc gathered"
                     : C::CMP ? "score_tc + candidate lists" : C::BND ? "score_tc bounds"
                     : (C::ELEM == 1 ? "score_tc fp8" : "score_tc"));
  score_tc_kernel<C><<<grid, C::NTHREADS, C::SMEM_BYTES, st>>>(tq, tk, p);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Dense / routed / block scoring, bf16: N = 256 columns = (256 / H) queries x H heads.
// epi: kEpiStore (full scores), kEpiCand (candidate lists: p.cthr ...
// p.ccap), kEpiBound (DoSA live tiles: p.knorm ... p.live_gpb; H = 8 or 16
// augmented heads); k_stride: key rows every k_stride elements; p.pairs set:
// only the listed (group, tile) pairs (work-list instantiations).
dsa_status run_scores_bf16(int D, int H, const ScoreParams& p, const void* q, long long q_rows,
                           const void* k, long long k_rows, cudaStream_t st, int epi = kEpiStore,
                           long long k_stride = 0) {
// Epilogue warps: 8 for 64 heads (4 queries per tile); 16 for fewer heads,
// where a thread of an 8-warp epilogue holds 8 to 16 queries' partial sums
// and spills (the 8-head MISA routed pass: 0.59 against 0.70-0.81 ms).
#ifndef DSA_EPIW64
#define DSA_EPIW64 8
#endif
  const bool list = p.pairs != nullptr;
#define DSA_CFG(DD, HH, EE, LL) \
  ScoreCfg<2, DD, HH, 256 / HH, ScoreMode::kTma, (DD == 128 ? 4 : 8), (HH == 64 ? DSA_EPIW64 : 16), 1, EE, LL>
#define DSA_LAUNCH(DD, HH, EE, LL) return launch_score<DSA_CFG(DD, HH, EE, LL)>(p, q, q_rows, k, k_rows, st, k_stride);
#define DSA_CASE(DD, HH)                                            \
  if (D == DD && H == HH) {                                         \
    if (epi == kEpiCand) {                                          \
      if (list && HH >= 16) { DSA_LAUNCH(DD, HH, kEpiCand, true) }  \
      if (!list) { DSA_LAUNCH(DD, HH, kEpiCand, false) }            \
      return DSA_ERR_UNSUPPORTED;                                   \
    }                                                               \
    if (list) { DSA_LAUNCH(DD, HH, kEpiStore, true) }               \
    DSA_LAUNCH(DD, HH, kEpiStore, false)                            \
  }
#define DSA_CASE_B(DD, HH) \
  if (D == DD && H == HH && epi == kEpiBound && !list) { DSA_LAUNCH(DD, HH, kEpiBound, false) }
  DSA_CASE_B(64, 8) DSA_CASE_B(64, 16) DSA_CASE_B(128, 8) DSA_CASE_B(128, 16)
  if (epi == kEpiBound) return DSA_ERR_UNSUPPORTED;
  DSA_CASE(64, 8) DSA_CASE(64, 16) DSA_CASE(64, 32) DSA_CASE(64, 64)
  DSA_CASE(128, 8) DSA_CASE(128, 16) DSA_CASE(128, 32) DSA_CASE(128, 64)
#undef DSA_CASE
#undef DSA_CASE_B
#undef DSA_LAUNCH
#undef DSA_CFG
  return DSA_ERR_UNSUPPORTED;
}

// FP8 scoring (kind::f8f6f4). Decode (one query per sequence): one query per
// group, N = H. Prefill (T > 1): 256 / H queries per group, N = 256, as the
// bf16 path, with sixteen epilogue warps (the FP8 MMAs take half the time of
// bf16 ones, so the epilogue arithmetic sets the pace: 1.40 against 1.44 ms
// with eight on the FP8 DSA chunk).
#ifndef DSA_FP8_NSTAGE
#define DSA_FP8_NSTAGE 8
#endif
#ifndef DSA_FP8_EPIW
#define DSA_FP8_EPIW 16
#endif
#ifndef DSA_FP8_DEC_EPIW
#define DSA_FP8_DEC_EPIW 8
#endif
// Decode (one query per sequence, a pure key stream): two CTAs per SM with 5
// stages each, so 10 key tiles per SM are in flight instead of 8: 0.249 ->
// 0.200 ms on the 64 x 131072 decode batch (0.68 -> 0.85 of HBM).
#ifndef DSA_FP8_DEC_NSTAGE
#define DSA_FP8_DEC_NSTAGE 5
#endif
#ifndef DSA_FP8_DEC_CTAS
#define DSA_FP8_DEC_CTAS 2
#endif
dsa_status run_scores_fp8(int D, int H, const ScoreParams& p, const void* q, long long q_rows,
                          const void* k, long long k_rows, cudaStream_t st) {
  const bool prefill = p.T > 1;
  // 8 or 16 heads (MISA's routed pass): each of the two epilogue warp sets
  // takes at least 32 columns, so a group has 64 / H queries even in decode,
  // where only the first of them exists
  if (D == 128 && H == 16)
    return prefill ? launch_score<ScoreCfg<1, 128, 16, 16, ScoreMode::kTma, DSA_FP8_NSTAGE, 16>>(p, q, q_rows, k, k_rows, st)
                   : launch_score<ScoreCfg<1, 128, 16, 4, ScoreMode::kTma, DSA_FP8_DEC_NSTAGE, 8, 1, kEpiStore, false,
                                           DSA_FP8_DEC_CTAS>>(p, q, q_rows, k, k_rows, st);
  if (D == 128 && H == 8)
    return prefill ? launch_score<ScoreCfg<1, 128, 8, 32, ScoreMode::kTma, DSA_FP8_NSTAGE, 16>>(p, q, q_rows, k, k_rows, st)
                   : launch_score<ScoreCfg<1, 128, 8, 8, ScoreMode::kTma, DSA_FP8_DEC_NSTAGE, 8, 1, kEpiStore, false,
                                           DSA_FP8_DEC_CTAS>>(p, q, q_rows, k, k_rows, st);
  if (D == 128 && H == 64)
    return prefill ? launch_score<ScoreCfg<1, 128, 64, 4, ScoreMode::kTma, DSA_FP8_NSTAGE, DSA_FP8_EPIW>>(p, q, q_rows, k, k_rows, st)
                   : launch_score<ScoreCfg<1, 128, 64, 1, ScoreMode::kTma, DSA_FP8_DEC_NSTAGE, DSA_FP8_DEC_EPIW, 1,
                                           kEpiStore, false, DSA_FP8_DEC_CTAS>>(p, q, q_rows, k, k_rows, st);
  if (D == 128 && H == 32)
    return prefill ? launch_score<ScoreCfg<1, 128, 32, 8, ScoreMode::kTma, DSA_FP8_NSTAGE, DSA_FP8_EPIW>>(p, q, q_rows, k, k_rows, st)
                   : launch_score<ScoreCfg<1, 128, 32, 1, ScoreMode::kTma, DSA_FP8_DEC_NSTAGE, DSA_FP8_DEC_EPIW, 1,
                                           kEpiStore, false, DSA_FP8_DEC_CTAS>>(p, q, q_rows, k, k_rows, st);
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

// MISA router on an FP8 cache: e4m3 queries against e4m3 pooled keys,
// p.k_scale = the pooled keys' scales (the router weights its columns by
// them; the query scales are applied with |w| when the heads are chosen).
dsa_status run_router_fp8(int D, int H, const ScoreParams& p, const void* q, long long q_rows,
                          const void* kbar, long long k_rows, cudaStream_t st) {
  if (D == 128 && H == 64)
    return launch_score<ScoreCfg<1, 128, 64, 2, ScoreMode::kRouter, 4>>(p, q, q_rows, kbar, k_rows, st);
  if (D == 128 && H == 32)
    return launch_score<ScoreCfg<1, 128, 32, 4, ScoreMode::kRouter, 4>>(p, q, q_rows, kbar, k_rows, st);
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
// FP8 gathers (decode MISA-dagger candidates, decode HISA kept blocks): two
// CTAs per SM with 5 stages each (decode HISA token stage: 0.089 -> 0.080 ms
// with the kept blocks streaming by TMA; 0.125 ms block major).
#ifndef DSA_GATHER8_NS
#define DSA_GATHER8_NS 5
#endif
#ifndef DSA_GATHER8_CTAS
#define DSA_GATHER8_CTAS 2
#endif
dsa_status run_gather(int D, int H, ScoreParams p, const void* q, long long q_rows,
                      cudaStream_t st, bool fp8 = false) {
  p.blk_tma = (p.blk % 128 == 0) ? 1 : 0;
  const long long k_rows = static_cast<long long>(p.batch) * p.L_tok;
  if (fp8) {  // e4m3 rows of 128 bytes, per-token key scales (p.k_scale)
    if (D == 128 && H == 64)
      return launch_score<ScoreCfg<1, 128, 64, 1, ScoreMode::kGather, DSA_GATHER8_NS, 8, DSA_GATHER_NQ, kEpiStore,
                                   false, DSA_GATHER8_CTAS>>(p, q, q_rows, p.kg, k_rows, st);
    if (D == 128 && H == 32)
      return launch_score<ScoreCfg<1, 128, 32, 1, ScoreMode::kGather, DSA_GATHER8_NS, 8, DSA_GATHER_NQ, kEpiStore,
                                   false, DSA_GATHER8_CTAS>>(p, q, q_rows, p.kg, k_rows, st);
    return DSA_ERR_UNSUPPORTED;
  }
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
  prof::Launch pl(st, tp.cres ? "topk_rows (candidate lists)" : "topk_rows");
  topk_rows_kernel<C><<<static_cast<int>(grid), C::NT, C::BYTES, st>>>(tp);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ws: the call's workspace (its first word is the device status word).
// Rows up to 32768 scores use the short-row layout (4 CTAs of 256 threads per
// SM, or one 512-thread CTA per row when there are fewer rows than SMs);
// longer rows use 2 CTAs of 512 threads per SM when there are enough rows to
// fill the GPU, else one 512-thread CTA (with more loads in flight) per row.
// (One CTA per SM for long rows, so fewer rows in flight stay in L2 between
// the sampling read and the band pass, measured slower: 0.72 vs 0.59 ms on
// the MISA-dagger k' selection.)
dsa_status launch_topk(void* ws, TopkParams tp, cudaStream_t st) {
  tp.err = static_cast<unsigned*>(ws);
  if (tp.Lrow <= 2048 && tp.cres == nullptr) {
    // short rows: one 128-thread CTA per row (16 keys per thread in
    // registers), up to 16 CTAs per SM. (The same design with 512 threads for
    // rows of 8192 and 16384 took 0.22 / 0.26 ms against 0.084 / 0.063 ms for
    // the sampled-band CTAs on the MISA-dagger and HISA rows.)
    const long long cap = static_cast<long long>(num_sms()) * 16;
    prof::Launch pl(st, "topk_rows");
    topk_small_kernel<128, 16><<<static_cast<int>(tp.rows < cap ? tp.rows : cap), 128, 0, st>>>(tp);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
  }
  if (tp.Lrow <= TkShort::MAX_ROW) {
    // fewer rows than SMs (decode): one 512-thread CTA per row with more
    // loads in flight (64 rows of 16384: 0.019 against 0.023 ms)
    if (tp.rows < num_sms()) return launch_topk_cfg<TkShortWide>(tp, st);
    return launch_topk_cfg<TkShort>(tp, st);
  }
  if (tp.rows >= static_cast<long long>(num_sms()) * TkLong::MIN_CTAS) return launch_topk_cfg<TkLong>(tp, st);
  return launch_topk_cfg<TkWide>(tp, st);
}

// ------------------------------------------------------------ block-major HISA refinement
// Workspace of the inverted kept-block lists (after the caller's own parts):
// counts, cursors, list starts, item starts, the item total and the list.
struct InvWs {
  int* cnt;
  int* cursor;
  int* qoff;
  int* ioff;
  long long* total;
  int2* list;
  int* it_tile;
  int4* it_row;
  int4* it_slot;
};

// Items: at most tiles-per-block x (kept pairs / queries per item + blocks).
long long inv_max_items(long long rows, int m, long long nb, int blk, int H) {
  return static_cast<long long>(blk / 128) * (rows * m / (128 / H) + nb + 1);
}

size_t inv_ws_bytes(long long rows, int m, long long nb, int blk, int H) {
  const size_t items = static_cast<size_t>(inv_max_items(rows, m, nb, blk, H));
  return 4 * al256(static_cast<size_t>(nb + 1) * sizeof(int)) + al256(sizeof(long long)) +
         al256(static_cast<size_t>(rows) * m * sizeof(int2)) + al256(items * sizeof(int)) +
         2 * al256(items * sizeof(int4));
}

InvWs inv_carve(Carve& c, long long rows, int m, long long nb, int blk, int H) {
  InvWs w;
  const size_t items = static_cast<size_t>(inv_max_items(rows, m, nb, blk, H));
  w.cnt = c.take<int>(nb + 1);
  w.cursor = c.take<int>(nb + 1);
  w.qoff = c.take<int>(nb + 1);
  w.ioff = c.take<int>(nb + 1);
  w.total = c.take<long long>(1);
  w.list = c.take<int2>(static_cast<size_t>(rows) * m);
  w.it_tile = c.take<int>(items);
  w.it_row = c.take<int4>(items);
  w.it_slot = c.take<int4>(items);
  return w;
}

// The block-major kernel takes kept blocks whose size is a multiple of 128
// (whole key tiles), bf16, d = 128, H in {32, 64}.
bool inv_supported(const dsa_indexer_args* a, int blk) {
  return blk % 128 == 0 && a->d == 128 && (a->H == 32 || a->H == 64);
}

template <class C>
dsa_status launch_inv(const InvParams& p, const void* q, long long q_rows, const void* k, long long k_rows,
                      const long long* total, cudaStream_t st) {
  static std::atomic<bool> attr[kMaxDev];
  const int dev = current_device();
  if (dev < 0) return DSA_ERR_UNSUPPORTED;
  if (!attr[dev].load(std::memory_order_relaxed)) {
    if (cudaFuncSetAttribute(score_inv_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess)
      return DSA_ERR_CUDA;
    attr[dev].store(true, std::memory_order_relaxed);
  }
  CUtensorMap tq, tk;
  if (!make_tmap(&tq, q, C::ELEM == 1, C::D, q_rows, C::H)) return DSA_ERR_CUDA;     // one query per box
  if (!make_tmap(&tk, k, C::ELEM == 1, C::D, k_rows, C::KROWS)) return DSA_ERR_CUDA;
  prof::Launch pl(st, "score_inv (block-major)");
  score_inv_kernel<C><<<num_sms(), C::NTHREADS, C::SMEM_BYTES, st>>>(tq, tk, p, total);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

#ifndef DSA_INV_NSTAGE
#define DSA_INV_NSTAGE 4
#endif
// Invert the kept blocks [rows, m] and score every kept (query, block) pair:
// out[r * ldo + slot * blk + i] = I[t, blocks[r, slot] * blk + i], -inf where
// that token is not visible, past L, or the slot is empty.
dsa_status run_refine_inverted(const dsa_indexer_args* a, const int32_t* blocks, int m, int blk, float* out,
                               long long ldo, const InvWs& w, unsigned* err, cudaStream_t st) {
  const long long rows = static_cast<long long>(a->batch) * a->T;
  const long long M = blocks_of(a->L, blk);
  const long long nb = a->batch * M;
  if (cudaMemsetAsync(w.cnt, 0, static_cast<size_t>(nb) * sizeof(int), st) != cudaSuccess) return DSA_ERR_CUDA;
  const long long n = rows * m;
  const int grid = static_cast<int>(std::min<long long>((n + 255) / 256, 8LL * num_sms()));
  {
    prof::Launch pl(st, "invert_count");
    invert_count_kernel<<<grid, 256, 0, st>>>(blocks, rows, m, a->T, static_cast<int>(M), blk, w.cnt, out, ldo);
  }
  {
    prof::Launch pl(st, "invert_scan");
    invert_scan_kernel<1024><<<static_cast<int>((nb + 4095) / 4096), 1024, 0, st>>>(
        w.cnt, static_cast<int>(nb), blk / 128, 128 / a->H, w.qoff, w.ioff, w.cursor, w.total);
  }
  {
    prof::Launch pl(st, "invert_fill");
    invert_fill_kernel<<<grid, 256, 0, st>>>(blocks, rows, m, a->T, static_cast<int>(M), w.qoff, w.cursor, w.list);
  }
  {
    prof::Launch pl(st, "invert_items");
    invert_items_kernel<<<static_cast<int>((nb + 7) / 8), 256, 0, st>>>(w.cnt, w.qoff, w.ioff, w.list,
                                                                       static_cast<int>(nb), blk / 128, 128 / a->H,
                                                                       w.it_tile, w.it_row, w.it_slot);
  }
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  InvParams p{};
  p.batch = a->batch;
  p.T = a->T;
  p.L = a->L;
  p.M = static_cast<int>(M);
  p.blk = blk;
  p.m = m;
  p.q_offset = a->q_offset;
  p.w = a->w;
  p.q_scale = a->q_scale;
  p.k_scale = a->k_scale;
  p.out = out;
  p.ldo = ldo;
  p.it_tile = w.it_tile;
  p.it_row = w.it_row;
  p.it_slot = w.it_slot;
  p.err = err;
  const long long q_rows = rows * a->H;
  const long long k_rows = static_cast<long long>(a->batch) * a->L;
  if (a->qk_dtype == DSA_FP8_E4M3) {
    if (a->H == 32) return launch_inv<InvCfg<1, 32, 8>>(p, a->q, q_rows, a->k, k_rows, w.total, st);
    return launch_inv<InvCfg<1, 64, 8>>(p, a->q, q_rows, a->k, k_rows, w.total, st);
  }
  if (a->H == 32) return launch_inv<InvCfg<2, 32, DSA_INV_NSTAGE>>(p, a->q, q_rows, a->k, k_rows, w.total, st);
  return launch_inv<InvCfg<2, 64, DSA_INV_NSTAGE>>(p, a->q, q_rows, a->k, k_rows, w.total, st);
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

// ------------------------------------------------------------ fused score -> candidate lists -> top-k
// LiteTopK's idea ("DoSA: Dots Sparse Attention" review: scoring fused with
// filtering to cut memory traffic), kept exact: a first pass scores every S-th
// key; from that sample each row gets a threshold its k-th score is very
// likely to reach; the full pass then appends every visible score >= the
// threshold to the row's candidate list, and the top-k selects from the lists.
// A row whose list holds fewer than k (or more than its capacity) is selected
// from its full scores, which the full pass still writes.
struct FusedPlan {
  bool on;
  int S;       // sample stride (keys)
  int ns_max;  // samples per full row (L / S)
  int cap;     // candidate list capacity per row
  int qpt;     // queries per group of the score kernel (256 / heads)
  int ntiles;  // key tiles per full row
};

FusedPlan fused_plan(int L, int topk, bool bf16, int heads) {
  FusedPlan f{false, 0, 0, 0, 0, 0};
  if (!bf16 || L < 4096 || static_cast<long long>(topk) * 8 > L || heads < 1 || 256 % heads != 0) return f;
  int S = 16;
  while (L / S > 4096) S <<= 1;  // 2048 .. 4096 samples per full row
  if (L % S != 0) return f;
  f.on = true;
  f.S = S;
  f.ns_max = L / S;
  // twice the expected list length at the longest rows (k plus the
  // threshold's margin: 4 standard deviations + 4 samples, each sample
  // standing for S keys), plus the unused tails of the reserved chunks (two
  // chunks per warp, four warps per query, a few CTAs per query group)
  const double c = 2.0 * (topk + 4.0 * std::sqrt(static_cast<double>(topk) * S) + 4.0 * S) + 32.0 * CCHUNK;
  f.cap = static_cast<int>((static_cast<long long>(std::ceil(c)) + 255) / 256 * 256);
  f.qpt = 256 / heads;
  f.ntiles = (L + 127) / 128;
  return f;
}

long long fused_groups(long long batch, int T, const FusedPlan& f) { return batch * ((T + f.qpt - 1) / f.qpt); }
// Pair lists of the score kernel's work-list mode: flags [groups, ntiles],
// the list and its length.
size_t pairs_ws_bytes(long long groups, int ntiles) {
  return al256(static_cast<size_t>(groups) * ntiles) + al256(static_cast<size_t>(groups) * ntiles * sizeof(int2)) +
         al256(sizeof(int));
}

size_t fused_ws_bytes(long long batch, int T, const FusedPlan& f) {
  if (!f.on) return 0;
  const size_t rows = static_cast<size_t>(batch) * T;
  return al256(rows * f.ns_max * sizeof(float)) + 3 * al256(rows * 4) + 2 * al256(rows * f.cap * 4) +
         pairs_ws_bytes(fused_groups(batch, T, f), f.ntiles);
}

struct PairWs {
  uint8_t* flags;  // [groups, ntiles]
  int2* list;      // [groups * ntiles]
  int* n;
};

PairWs pairs_carve(Carve& c, long long groups, int ntiles) {
  PairWs w;
  w.flags = c.take<uint8_t>(static_cast<size_t>(groups) * ntiles);
  w.list = c.take<int2>(static_cast<size_t>(groups) * ntiles);
  w.n = c.take<int>(1);
  return w;
}

struct FusedWs {
  float* samp;
  float* thr;
  int* cres;
  int* creal;
  float* cval;
  int* cidx;
  PairWs fb;  // the fallback pass's tiles
};

FusedWs fused_carve(Carve& c, long long batch, int T, const FusedPlan& f) {
  const long long rows = batch * T;
  FusedWs w;
  w.samp = c.take<float>(static_cast<size_t>(rows) * f.ns_max);
  w.thr = c.take<float>(rows);
  w.cres = c.take<int>(rows);
  w.creal = c.take<int>(rows);
  c.take<int>(rows);  // spare (keeps the two counters apart)
  w.cval = c.take<float>(static_cast<size_t>(rows) * f.cap);
  w.cidx = c.take<int>(static_cast<size_t>(rows) * f.cap);
  w.fb = pairs_carve(c, fused_groups(batch, T, f), f.ntiles);
  return w;
}

// Clear a pair workspace (stream-ordered).
dsa_status pairs_clear(const PairWs& w, long long groups, int ntiles, cudaStream_t st) {
  if (cudaMemsetAsync(w.flags, 0, static_cast<size_t>(groups) * ntiles, st) != cudaSuccess ||
      cudaMemsetAsync(w.n, 0, sizeof(int), st) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

// flags -> work list (pairs_build_kernel).
dsa_status pairs_build(const PairWs& w, long long groups, int ntiles, int T, int qpt, long long q_offset, int L,
                       cudaStream_t st) {
  prof::Launch pl(st, "work list");
  const int gpb = (T + qpt - 1) / qpt;
  pairs_build_kernel<<<static_cast<int>((groups + 7) / 8), 256, 0, st>>>(w.flags, ntiles, static_cast<int>(groups), gpb,
                                                                         T, qpt, q_offset, L, w.list, w.n);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Scores of every visible key with the Hh heads of q ([rows * Hh, D] bf16;
// weights in base.w) and the top-k of every row through candidate lists;
// scores [rows, L] receives full scores only for rows whose list fails the
// check (and the winners' scores). base: batch, T, q_offset, w, err set.
// DoSA pruning between the thresholds and the candidate pass: the bound pass
// marks the key tiles each query group must score (live), the candidate pass
// skips the others.
struct Prune {
  const void* q_aug;  // [rows, ha, D] bf16 augmented heads
  const float* w_aug; // [rows, ha]
  const float* cb;    // [rows] norm coefficient c_t
  const float* kn;    // [batch * L] key norms
  int ha;             // augmented heads (8 or 16)
  PairWs live;        // tiles the bound pass keeps
};

dsa_status fused_score_topk(int D, int Hh, const ScoreParams& base, const void* q, const void* k, int L,
                            int topk, int32_t* out_idx, float* out_score, float* scores, const FusedPlan& f,
                            const FusedWs& w, void* ws, cudaStream_t st, const Prune* prune = nullptr) {
  const long long rows = static_cast<long long>(base.batch) * base.T;
  const long long groups = fused_groups(base.batch, base.T, f);
  if (cudaMemsetAsync(w.cres, 0, 2 * al256(static_cast<size_t>(rows) * 4), st) != cudaSuccess) return DSA_ERR_CUDA;
  DSA_TRY(pairs_clear(w.fb, groups, f.ntiles, st));
  if (prune) DSA_TRY(pairs_clear(prune->live, groups, f.ntiles, st));
  // 1. sample pass: keys 0, S, 2S, ... (a strided view of the key rows)
  {
    prof::Stage sample_stage("sample pass");
    ScoreParams ps = base;
    ps.Lk = f.ns_max;
    ps.pstride = f.S;
    ps.out = w.samp;
    ps.ldo = f.ns_max;
    DSA_TRY(run_scores_bf16(D, Hh, ps, q, rows * Hh, k, static_cast<long long>(base.batch) * f.ns_max, st, kEpiStore,
                            static_cast<long long>(f.S) * D));
  }
  // 2. thresholds
  const int tgrid = static_cast<int>(std::min<long long>(rows, 8LL * num_sms()));
  {
    prof::Launch pl(st, "thresholds");
    topk_threshold_kernel<256><<<tgrid, 256, 0, st>>>(w.samp, rows, f.ns_max, base.T, base.q_offset, f.S, f.ns_max,
                                                       L, topk, w.thr);
  }
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  // 2b. DoSA: bounds over the augmented heads -> live key tiles
  if (prune) {
    prof::Stage bound_stage("bounds");
    ScoreParams pb = base;
    pb.Lk = L;
    pb.pstride = 1;
    pb.out = nullptr;
    pb.w = prune->w_aug;
    pb.cthr = w.thr;
    pb.cbound = prune->cb;
    pb.knorm = prune->kn;
    pb.live_out = prune->live.flags;
    pb.live_ld = f.ntiles;
    pb.live_qpt = f.qpt;
    pb.live_gpb = (base.T + f.qpt - 1) / f.qpt;
    DSA_TRY(run_scores_bf16(D, prune->ha, pb, prune->q_aug, rows * prune->ha, k, static_cast<long long>(base.batch) * L,
                            st, kEpiBound));
    DSA_TRY(pairs_build(prune->live, groups, f.ntiles, base.T, f.qpt, base.q_offset, L, st));
  }
  // 3. candidate lists (no full scores)
  ScoreParams pm = base;
  if (prune) {
    pm.pairs = prune->live.list;
    pm.pairs_n = prune->live.n;
  }
  pm.Lk = L;
  pm.pstride = 1;
  pm.out = nullptr;
  pm.cthr = w.thr;
  pm.cval = w.cval;
  pm.cidx = w.cidx;
  pm.cres = w.cres;
  pm.creal = w.creal;
  pm.ccap = f.cap;
  DSA_TRY(run_scores_bf16(D, Hh, pm, q, rows * Hh, k, static_cast<long long>(base.batch) * L, st, kEpiCand));
  // 4. rows whose list is short (or overflowed): full scores of their groups
  {
    prof::Launch pl(st, "list check");
    fused_check_kernel<<<static_cast<int>((rows + 255) / 256), 256, 0, st>>>(
        w.cres, w.creal, rows, base.T, base.q_offset, L, topk, f.cap, f.qpt, f.ntiles, w.fb.flags);
  }
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  DSA_TRY(pairs_build(w.fb, groups, f.ntiles, base.T, f.qpt, base.q_offset, L, st));
  {
    prof::Stage fb_stage("fallback");
    ScoreParams pf = base;
    pf.Lk = L;
    pf.pstride = 1;
    pf.out = scores;
    pf.ldo = L;
    pf.pairs = w.fb.list;
    pf.pairs_n = w.fb.n;
    DSA_TRY(run_scores_bf16(D, Hh, pf, q, rows * Hh, k, static_cast<long long>(base.batch) * L, st));
  }
  // 5. top-k from the lists (from the full scores where a list failed)
  TopkParams tp = topk_params(scores, rows, L, base.T, base.q_offset, 1, L, topk, out_idx, out_score, nullptr, 0, 1);
  tp.cval = w.cval;
  tp.cidx = w.cidx;
  tp.cres = w.cres;
  tp.creal = w.creal;
  tp.ccap = f.cap;
  return launch_topk(ws, tp, st);
}

dsa_status clear_status(void* ws, cudaStream_t st) {
  return cudaMemsetAsync(ws, 0, 4, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}


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
  DSA_TRY(validate(a, false));
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
  pg.kg = a->k;
  pg.cand = cand;
  pg.n_slots = n_slots;
  pg.blk = blk;
  pg.n_compact = n_slots * blk;
  return run_gather(a->d, a->H, pg, a->q, static_cast<long long>(a->batch) * a->T * a->H, st,
                    a->qk_dtype == DSA_FP8_E4M3);
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

// The dense score + top-k: full scores, then the row top-k.
dsa_status indexer_score_topk(const dsa_indexer_args* a, int topk, int32_t* out_idx, float* out_score, void* ws,
                              size_t ws_bytes, void* stream) {
  DSA_TRY(validate(a, false));
  if (!out_idx || topk < 1 || topk > (1 << 24)) return DSA_ERR_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, indexer_workspace_size(a, topk)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  Carve c{static_cast<char*>(ws), kHdr};
  const size_t rows = static_cast<size_t>(a->batch) * a->T;
  float* scores = c.take<float>(rows * a->L);
  ScoreParams p = base_params(a, static_cast<unsigned*>(ws));
  p.out = scores;
  p.ldo = a->L;
  const long long q_rows = static_cast<long long>(a->batch) * a->T * a->H;
  const long long k_rows = static_cast<long long>(a->batch) * a->L;
  if (a->qk_dtype == DSA_FP8_E4M3)
    DSA_TRY(run_scores_fp8(a->d, a->H, p, a->q, q_rows, a->k, k_rows, st));
  else
    DSA_TRY(run_scores_bf16(a->d, a->H, p, a->q, q_rows, a->k, k_rows, st));
  return launch_topk(ws, topk_params(scores, static_cast<long long>(rows), a->L, a->T, a->q_offset, 1, a->L, topk,
                                 out_idx, out_score, nullptr, 0, 1),
                     st);
}

// The dense selection through candidate lists (fused_score_topk).
size_t indexer_lists_workspace_size(const dsa_indexer_args* a, int topk) {
  if (!a || a->batch < 1 || a->T < 1 || a->L < 1) return 0;
  const FusedPlan f = fused_plan(a->L, topk, a->qk_dtype == DSA_BF16, a->H);
  if (!f.on) return 0;
  return kHdr + al256(static_cast<size_t>(a->batch) * a->T * a->L * sizeof(float)) +
         fused_ws_bytes(a->batch, a->T, f);
}

dsa_status indexer_score_topk_lists(const dsa_indexer_args* a, int topk, int32_t* out_idx, float* out_score,
                                    void* ws, size_t ws_bytes, void* stream) {
  DSA_TRY(validate(a, true));
  if (!out_idx || topk < 1 || topk > (1 << 24)) return DSA_ERR_ARG;
  const FusedPlan f = fused_plan(a->L, topk, true, a->H);
  if (!f.on) return DSA_ERR_UNSUPPORTED;
  DSA_TRY(check_ws(ws, ws_bytes, indexer_lists_workspace_size(a, topk)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  Carve c{static_cast<char*>(ws), kHdr};
  float* scores = c.take<float>(static_cast<size_t>(a->batch) * a->T * a->L);
  const FusedWs w = fused_carve(c, a->batch, a->T, f);
  const ScoreParams p = base_params(a, static_cast<unsigned*>(ws));
  return fused_score_topk(a->d, a->H, p, a->q, a->k, a->L, topk, out_idx, out_score, scores, f, w, ws, st);
}

// bf16 pooling of blocks [m0, m0 + nm) of every sequence.
dsa_status launch_meanpool_bf16(const void* k, int batch, int L, int d, int block, long long M, long long m0,
                                long long nm, void* kbar, cudaStream_t st) {
  if (static_cast<long long>(batch) * nm > INT_MAX) return DSA_ERR_UNSUPPORTED;
  if (nm < 1) return DSA_OK;
  prof::Launch pl(st, "meanpool");
  const int grid = static_cast<int>(batch * nm);
  if (d % 8 == 0 && d <= 256 && aligned(k, 16))
    meanpool_vec_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(k), L, d, block,
                                              static_cast<int>(M), static_cast<int>(m0), static_cast<int>(nm),
                                              static_cast<__nv_bfloat16*>(kbar));
  else
    meanpool_kernel<<<grid, d < 128 ? d : 128, 0, st>>>(static_cast<const __nv_bfloat16*>(k), L, d, block,
                                                        static_cast<int>(M), static_cast<int>(m0),
                                                        static_cast<int>(nm), static_cast<__nv_bfloat16*>(kbar));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status dsa_meanpool_keys(const void* k, int batch, int L, int d, int block, void* kbar,
                             void* stream) {
  if (!k || !kbar || batch < 1 || L < 1 || d < 1 || d > 1024 || block < 1) return DSA_ERR_ARG;
  const long long M = blocks_of(L, block);
  return launch_meanpool_bf16(k, batch, L, d, block, M, 0, M, kbar, static_cast<cudaStream_t>(stream));
}

// Pooled keys of MISA and HISA: bf16 [batch*M, d], or on an FP8 cache e4m3
// codes [batch*M, d] plus fp32 scales [batch*M] (the cache's format).
struct Pooled {
  __nv_bfloat16* kbar;  // bf16
  uint8_t* kbar8;       // FP8 codes
  float* scale;         // FP8 scales
};

size_t pooled_bytes(const dsa_indexer_args* a, long long M) {
  const size_t n = static_cast<size_t>(a->batch) * M;
  return al256(n * a->d * 2) + al256(n * sizeof(float));
}

Pooled pooled_carve(Carve& c, const dsa_indexer_args* a, long long M) {
  const size_t n = static_cast<size_t>(a->batch) * M;
  Pooled pk{};
  if (a->qk_dtype == DSA_FP8_E4M3) {
    pk.kbar8 = c.take<uint8_t>(n * a->d);
    pk.scale = c.take<float>(n);
    c.off += al256(n * a->d * 2) - al256(n * a->d);  // keep the bf16 layout's size
  } else {
    pk.kbar = c.take<__nv_bfloat16>(n * a->d);
    pk.scale = c.take<float>(n);
  }
  return pk;
}

// Pools blocks [m0, m1) of every sequence into pk.
dsa_status run_meanpool(const dsa_indexer_args* a, int block, long long M, const Pooled& pk, cudaStream_t st,
                        long long m0 = 0, long long m1 = -1) {
  if (m1 < 0 || m1 > M) m1 = M;
  if (m0 < 0) m0 = 0;
  const long long nm = m1 - m0;
  if (a->qk_dtype != DSA_FP8_E4M3)
    return launch_meanpool_bf16(a->k, a->batch, a->L, a->d, block, M, m0, nm, pk.kbar, st);
  if (nm < 1) return DSA_OK;
  if (static_cast<long long>(a->batch) * nm > INT_MAX) return DSA_ERR_UNSUPPORTED;
  prof::Launch pl(st, "meanpool fp8");
  // FP8 caches: d % 4 == 0 and d <= 128, rows 16-byte aligned (checked by validate)
  meanpool_fp8_kernel<<<static_cast<int>(a->batch * nm), 512, 0, st>>>(
      static_cast<const uint8_t*>(a->k), a->k_scale, a->L, a->d, block, static_cast<int>(M), static_cast<int>(m0),
      static_cast<int>(nm), pk.kbar8, pk.scale);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Caller-kept pooled keys (the *_pooled entry points): checked and wrapped.
dsa_status given_pooled(const dsa_indexer_args* a, const void* kbar, const float* kbar_scale, Pooled& pk) {
  if (!kbar || !aligned(kbar, 16)) return DSA_ERR_ARG;
  pk = Pooled{};
  if (a->qk_dtype == DSA_FP8_E4M3) {
    if (!kbar_scale || !aligned(kbar_scale, 4)) return DSA_ERR_ARG;
    pk.kbar8 = const_cast<uint8_t*>(static_cast<const uint8_t*>(kbar));
    pk.scale = const_cast<float*>(kbar_scale);
  } else {
    pk.kbar = const_cast<__nv_bfloat16*>(static_cast<const __nv_bfloat16*>(kbar));
  }
  return DSA_OK;
}

dsa_status dsa_pool_keys(const dsa_indexer_args* a, int block, int m0, int m1, void* kbar, float* kbar_scale,
                         void* stream) {
  DSA_TRY(validate(a, false));
  if (block < 1 || m0 < 0 || m1 < m0) return DSA_ERR_ARG;
  Pooled pk{};
  DSA_TRY(given_pooled(a, kbar, kbar_scale, pk));
  const long long M = blocks_of(a->L, block);
  return run_meanpool(a, block, M, pk, static_cast<cudaStream_t>(stream), m0, m1 < M ? m1 : M);
}

size_t misa_workspace_size(const dsa_indexer_args* a, int block, int h, int topk, int kprime) {
  (void)topk;
  if (!a || a->batch < 1 || a->T < 1 || a->L < 1 || a->H < 1 || a->d < 1 || block < 1 || h < 1)
    return 0;
  const size_t BT = static_cast<size_t>(a->batch) * a->T;
  const size_t M = static_cast<size_t>(blocks_of(a->L, block));
  size_t n = kHdr;
  n += pooled_bytes(a, static_cast<long long>(M));  // pooled keys
  n += al256(2 * BT * a->H * sizeof(float));      // router partial sums
  n += al256(BT * h * a->d * 2);                  // gathered queries of the kept heads
  n += al256(BT * h * sizeof(float));             // their weights
  n += al256(BT * h * sizeof(float));             // their query scales (FP8)
  n += al256(BT * h * sizeof(int32_t));           // kept heads
  n += al256(BT * a->L * sizeof(float));          // routed scores
  if (kprime > 0) {
    n += al256(BT * kprime * sizeof(int32_t));    // candidates
    n += al256(BT * kprime * sizeof(float));      // full-H candidate scores
  }
  return n;
}

// given: caller-kept pooled keys (nullptr: pooled here, into the workspace)
dsa_status misa_run(const dsa_indexer_args* a, int block, int h, int topk, int kprime, const Pooled* given,
                    int32_t* out_idx, float* out_score, int32_t* out_heads, int32_t* out_cand, void* ws,
                    size_t ws_bytes, void* stream) {
  if (!out_idx || block < 1 || h < 1 || h > a->H || topk < 1 || topk > (1 << 24) || kprime < 0 ||
      kprime > (1 << 24))
    return DSA_ERR_ARG;
  if (!h_supported_bf16(h) || a->H > 64) return DSA_ERR_UNSUPPORTED;
  const bool fp8 = a->qk_dtype == DSA_FP8_E4M3;
  if (kprime > 0 && (a->d != 128 || (a->H != 32 && a->H != 64))) return DSA_ERR_UNSUPPORTED;
  DSA_TRY(check_ws(ws, ws_bytes, misa_workspace_size(a, block, h, topk, kprime)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  unsigned* err = static_cast<unsigned*>(ws);
  const long long BT = static_cast<long long>(a->batch) * a->T;
  const long long M = blocks_of(a->L, block);
  if (static_cast<long long>(a->batch) * M > INT_MAX) return DSA_ERR_UNSUPPORTED;

  Carve c{static_cast<char*>(ws), kHdr};
  const Pooled pk_ws = pooled_carve(c, a, M);
  const Pooled& pk = given ? *given : pk_ws;
  float* part = c.take<float>(2 * static_cast<size_t>(BT) * a->H);
  uint8_t* q_sel = c.take<uint8_t>(static_cast<size_t>(BT) * h * a->d * 2);
  float* w_sel = c.take<float>(static_cast<size_t>(BT) * h);
  float* qs_sel = c.take<float>(static_cast<size_t>(BT) * h);
  int32_t* heads_ws = c.take<int32_t>(static_cast<size_t>(BT) * h);
  float* routed = c.take<float>(static_cast<size_t>(BT) * a->L);
  int32_t* heads = out_heads ? out_heads : heads_ws;

  // 1. pooled keys (FP8 cache: in the cache's format), unless the caller keeps them
  if (!given) DSA_TRY(run_meanpool(a, block, M, pk, st));
  // 2. router affinities (partial ReLU sums over visible pooled keys)
  prof::Stage misa_stage("router");
  ScoreParams pr = base_params(a, err);
  pr.Lk = static_cast<int>(M);
  pr.pstride = block;
  pr.out = part;
  if (fp8) {
    pr.k_scale = pk.scale;
    DSA_TRY(run_router_fp8(a->d, a->H, pr, a->q, BT * a->H, pk.kbar8, a->batch * M, st));
  } else {
    DSA_TRY(run_router(a->d, a->H, pr, a->q, BT * a->H, pk.kbar, a->batch * M, st));
  }
  // 3. top-h heads per query; gather their query rows, weights (and query scales)
  {
    prof::Launch pl(st, "select_heads");
    select_heads_kernel<<<static_cast<int>((BT + 7) / 8), 256, 0, st>>>(
        part, BT, a->H, h, a->w, fp8 ? a->q_scale : nullptr, static_cast<const uint8_t*>(a->q),
        a->d * (fp8 ? 1 : 2), heads, q_sel, w_sel, qs_sel);
  }
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  // 4. routed token scores with the kept heads only, and their top-k (or
  // top-k' candidates)
  misa_stage.set("routed");
  ScoreParams ps = base_params(a, err);
  ps.w = w_sel;
  ps.q_scale = fp8 ? qs_sel : nullptr;
  ps.out = routed;
  ps.ldo = a->L;
  const long long k_rows = static_cast<long long>(a->batch) * a->L;
  int32_t* cand = nullptr;
  float* compact = nullptr;
  if (kprime > 0) {
    int32_t* cand_ws = c.take<int32_t>(static_cast<size_t>(BT) * kprime);
    compact = c.take<float>(static_cast<size_t>(BT) * kprime);
    cand = out_cand ? out_cand : cand_ws;
  }
  const int ksel = kprime > 0 ? kprime : topk;
  int32_t* sel = kprime > 0 ? cand : out_idx;
  float* sel_score = kprime > 0 ? nullptr : out_score;
  // (The candidate-list selection of indexer_score_topk_lists was measured
  // here too: 2.78 against 2.19 ms for the whole MISA-dagger step, so the
  // routed rows are written in full and selected by the row top-k.)
  if (fp8) DSA_TRY(run_scores_fp8(a->d, h, ps, q_sel, BT * h, a->k, k_rows, st));
  else DSA_TRY(run_scores_bf16(a->d, h, ps, q_sel, BT * h, a->k, k_rows, st));
  DSA_TRY(launch_topk(ws, topk_params(routed, BT, a->L, a->T, a->q_offset, 1, a->L, ksel, sel, sel_score, nullptr,
                                      0, 1),
                      st));
  if (kprime == 0) return DSA_OK;
  // 5. MISA-dagger: full-H re-score of the k' candidates, top-k
  misa_stage.set("re-score");
  ScoreParams pg = base_params(a, err);
  pg.out = compact;
  pg.ldo = kprime;
  pg.kg = a->k;
  pg.cand = cand;
  pg.n_slots = kprime;
  pg.blk = 1;
  pg.n_compact = kprime;
  DSA_TRY(run_gather(a->d, a->H, pg, a->q, BT * a->H, st, fp8));
  return launch_topk(ws, topk_params(compact, BT, kprime, a->T, a->q_offset, 0, kprime, topk, out_idx,
                                 out_score, cand, kprime, 1),
                     st);
}

dsa_status misa_route_score_topk(const dsa_indexer_args* a, int block, int h, int topk, int kprime,
                                 int32_t* out_idx, float* out_score, int32_t* out_heads,
                                 int32_t* out_cand, void* ws, size_t ws_bytes, void* stream) {
  DSA_TRY(validate(a, false));
  return misa_run(a, block, h, topk, kprime, nullptr, out_idx, out_score, out_heads, out_cand, ws, ws_bytes,
                  stream);
}

dsa_status misa_route_score_topk_pooled(const dsa_indexer_args* a, int block, int h, int topk, int kprime,
                                        const void* kbar, const float* kbar_scale, int32_t* out_idx,
                                        float* out_score, int32_t* out_heads, int32_t* out_cand, void* ws,
                                        size_t ws_bytes, void* stream) {
  DSA_TRY(validate(a, false));
  Pooled pk{};
  DSA_TRY(given_pooled(a, kbar, kbar_scale, pk));
  return misa_run(a, block, h, topk, kprime, &pk, out_idx, out_score, out_heads, out_cand, ws, ws_bytes, stream);
}

size_t hisa_workspace_size(const dsa_indexer_args* a, int block, int m, int topk) {
  (void)topk;
  if (!a || a->batch < 1 || a->T < 1 || a->L < 1 || a->d < 1 || block < 1 || m < 1) return 0;
  const size_t BT = static_cast<size_t>(a->batch) * a->T;
  const size_t M = static_cast<size_t>(blocks_of(a->L, block));
  size_t n = kHdr;
  n += pooled_bytes(a, static_cast<long long>(M));            // pooled keys (FP8: codes + scales)
  n += al256(BT * M * sizeof(float));                         // block scores
  n += al256(BT * m * sizeof(int32_t));                       // kept blocks
  n += al256(BT * static_cast<size_t>(m) * block * sizeof(float));  // token scores of kept blocks
  if (inv_supported(a, block))
    n += inv_ws_bytes(static_cast<long long>(BT), m, a->batch * static_cast<long long>(M), block, a->H);
  return n;
}

size_t hisa_refine_workspace_size(const dsa_indexer_args* a, int m, int blk) {
  if (!a || a->batch < 1 || a->T < 1 || a->L < 1 || m < 1 || blk < 1) return 0;
  return kHdr + inv_ws_bytes(static_cast<long long>(a->batch) * a->T, m, a->batch * blocks_of(a->L, blk), blk,
                             a->H > 0 ? a->H : 1);
}

dsa_status hisa_refine_scores(const dsa_indexer_args* a, const int32_t* blocks, int m, int blk, float* out,
                              long long ld, void* ws, size_t ws_bytes, void* stream) {
  DSA_TRY(validate(a, false));
  if (!blocks || !out || m < 1 || blk < 1 || !aligned(blocks, 4) || !aligned(out, 4)) return DSA_ERR_ARG;
  if (static_cast<long long>(m) * blk > INT_MAX / 2) return DSA_ERR_UNSUPPORTED;
  if (ld < static_cast<long long>(m) * blk) return DSA_ERR_ARG;
  if (!inv_supported(a, blk)) return DSA_ERR_UNSUPPORTED;
  if (a->batch * blocks_of(a->L, blk) > INT_MAX / 2) return DSA_ERR_UNSUPPORTED;
  DSA_TRY(check_ws(ws, ws_bytes, hisa_refine_workspace_size(a, m, blk)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  Carve c{static_cast<char*>(ws), kHdr};
  const long long rows = static_cast<long long>(a->batch) * a->T;
  const InvWs w = inv_carve(c, rows, m, a->batch * blocks_of(a->L, blk), blk, a->H);
  return run_refine_inverted(a, blocks, m, blk, out, ld, w, static_cast<unsigned*>(ws), st);
}

dsa_status hisa_run(const dsa_indexer_args* a, int block, int m, int topk, const Pooled* given,
                    int32_t* out_idx, float* out_score, int32_t* out_blocks, void* ws, size_t ws_bytes,
                    void* stream) {
  if (!out_idx || block < 1 || m < 1 || topk < 1 || topk > (1 << 24)) return DSA_ERR_ARG;
  if (static_cast<long long>(m) * block > INT_MAX / 2) return DSA_ERR_UNSUPPORTED;
  if (a->d != 128 || (a->H != 32 && a->H != 64)) return DSA_ERR_UNSUPPORTED;
  const bool fp8 = a->qk_dtype == DSA_FP8_E4M3;
  if (fp8 && block % 128 != 0) return DSA_ERR_UNSUPPORTED;  // FP8 refinement: whole key tiles only
  DSA_TRY(check_ws(ws, ws_bytes, hisa_workspace_size(a, block, m, topk)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  unsigned* err = static_cast<unsigned*>(ws);
  const long long BT = static_cast<long long>(a->batch) * a->T;
  const long long M = blocks_of(a->L, block);
  if (static_cast<long long>(a->batch) * M > INT_MAX) return DSA_ERR_UNSUPPORTED;
  const int ncomp = m * block;

  Carve c{static_cast<char*>(ws), kHdr};
  const Pooled pk_ws = pooled_carve(c, a, M);
  const Pooled& pk = given ? *given : pk_ws;
  float* bscore = c.take<float>(static_cast<size_t>(BT) * M);
  int32_t* blocks_ws = c.take<int32_t>(static_cast<size_t>(BT) * m);
  float* compact = c.take<float>(static_cast<size_t>(BT) * ncomp);
  int32_t* blocks = out_blocks ? out_blocks : blocks_ws;

  // 1. pooled keys (FP8 cache: e4m3 codes + per-block scales), unless the caller keeps them
  if (!given) DSA_TRY(run_meanpool(a, block, M, pk, st));
  // 2. block scores on the pooled keys (block m visible iff m * block <= p_t)
  prof::Stage hisa_stage("blocks");
  ScoreParams pb = base_params(a, err);
  pb.Lk = static_cast<int>(M);
  pb.pstride = block;
  pb.out = bscore;
  pb.ldo = M;
  if (fp8) {
    pb.k_scale = pk.scale;
    DSA_TRY(run_scores_fp8(a->d, a->H, pb, a->q, BT * a->H, pk.kbar8, a->batch * M, st));
  } else {
    DSA_TRY(run_scores_bf16(a->d, a->H, pb, a->q, BT * a->H, pk.kbar, a->batch * M, st));
  }
  // 3. top-m blocks
  DSA_TRY(launch_topk(ws, topk_params(bscore, BT, M, a->T, a->q_offset, block, static_cast<int>(M), m,
                                  blocks, nullptr, nullptr, 0, 1),
                      st));
  hisa_stage.set("tokens");
  // 4. token scores inside the kept blocks (compact rows of m * block):
  // block-major over the inverted kept-block lists when blocks are whole key
  // tiles and a sequence has several queries to share them; with one query
  // per sequence (decode) nothing is shared, so its query stays stationary
  // and its kept blocks stream through whole-tile TMA loads (the gather
  // path); blocks that are not whole tiles are gathered row by row
#ifndef DSA_HISA_DECODE_GATHER
#define DSA_HISA_DECODE_GATHER 1
#endif
  if (inv_supported(a, block) && !(DSA_HISA_DECODE_GATHER && a->T == 1)) {
    const InvWs w = inv_carve(c, BT, m, a->batch * M, block, a->H);
    DSA_TRY(run_refine_inverted(a, blocks, m, block, compact, ncomp, w, err, st));
    return launch_topk(ws, topk_params(compact, BT, ncomp, a->T, a->q_offset, 0, ncomp, topk, out_idx,
                                   out_score, blocks, m, block),
                       st);
  }
  ScoreParams pg = base_params(a, err);
  pg.out = compact;
  pg.ldo = ncomp;
  pg.kg = a->k;
  pg.cand = blocks;
  pg.n_slots = m;
  pg.blk = block;
  pg.n_compact = ncomp;
  DSA_TRY(run_gather(a->d, a->H, pg, a->q, BT * a->H, st, fp8));
  // 5. top-k tokens
  return launch_topk(ws, topk_params(compact, BT, ncomp, a->T, a->q_offset, 0, ncomp, topk, out_idx,
                                 out_score, blocks, m, block),
                     st);
}

dsa_status hisa_block_filter_topk(const dsa_indexer_args* a, int block, int m, int topk,
                                  int32_t* out_idx, float* out_score, int32_t* out_blocks,
                                  void* ws, size_t ws_bytes, void* stream) {
  DSA_TRY(validate(a, false));
  return hisa_run(a, block, m, topk, nullptr, out_idx, out_score, out_blocks, ws, ws_bytes, stream);
}

dsa_status hisa_block_filter_topk_pooled(const dsa_indexer_args* a, int block, int m, int topk, const void* kbar,
                                         const float* kbar_scale, int32_t* out_idx, float* out_score,
                                         int32_t* out_blocks, void* ws, size_t ws_bytes, void* stream) {
  DSA_TRY(validate(a, false));
  Pooled pk{};
  DSA_TRY(given_pooled(a, kbar, kbar_scale, pk));
  return hisa_run(a, block, m, topk, &pk, out_idx, out_score, out_blocks, ws, ws_bytes, stream);
}

// ------------------------------------------------------------ DoSA
static int dosa_aug_heads(int n_screen) { return n_screen + 3 <= 8 ? 8 : 16; }

static dsa_status dosa_check(const dsa_indexer_args* a, int topk, int n_screen, FusedPlan* f) {
  DSA_TRY(validate(a, true));
  if (topk < 1 || topk > (1 << 24) || n_screen < 0) return DSA_ERR_ARG;
  if (n_screen + 3 > 16 || n_screen >= a->H || (a->H != 16 && a->H != 32 && a->H != 64)) return DSA_ERR_UNSUPPORTED;
  *f = fused_plan(a->L, topk, true, a->H);
  if (!f->on) return DSA_ERR_UNSUPPORTED;  // rows too short for sampled thresholds
  return DSA_OK;
}

static size_t dosa_extra_bytes(const dsa_indexer_args* a, int n_screen, const FusedPlan& f) {
  const size_t rows = static_cast<size_t>(a->batch) * a->T;
  const int ha = dosa_aug_heads(n_screen);
  return al256(rows * ha * a->d * 2) + al256(rows * ha * 4) + al256(rows * 4) +
         al256(static_cast<size_t>(a->batch) * a->L * 4) + pairs_ws_bytes(fused_groups(a->batch, a->T, f), f.ntiles);
}

size_t dosa_workspace_size(const dsa_indexer_args* a, int topk, int n_screen) {
  if (!a || a->batch < 1 || a->T < 1 || a->L < 1 || n_screen < 0) return 0;
  FusedPlan f;
  if (dosa_check(a, topk, n_screen, &f) == DSA_ERR_UNSUPPORTED || !f.on) return 0;
  const size_t rows = static_cast<size_t>(a->batch) * a->T;
  return kHdr + al256(rows * a->L * sizeof(float)) + fused_ws_bytes(a->batch, a->T, f) +
         dosa_extra_bytes(a, n_screen, f);
}

dsa_status dosa_score_topk(const dsa_indexer_args* a, int topk, int n_screen, int32_t* out_idx, float* out_score,
                           uint8_t* out_live, void* ws, size_t ws_bytes, void* stream) {
  FusedPlan f;
  DSA_TRY(dosa_check(a, topk, n_screen, &f));
  if (!out_idx) return DSA_ERR_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, dosa_workspace_size(a, topk, n_screen)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DSA_TRY(clear_status(ws, st));
  const long long rows = static_cast<long long>(a->batch) * a->T;
  const int ha = dosa_aug_heads(n_screen);
  Carve c{static_cast<char*>(ws), kHdr};
  float* scores = c.take<float>(static_cast<size_t>(rows) * a->L);
  const FusedWs w = fused_carve(c, a->batch, a->T, f);
  Prune pr;
  __nv_bfloat16* q_aug = c.take<__nv_bfloat16>(static_cast<size_t>(rows) * ha * a->d);
  float* w_aug = c.take<float>(static_cast<size_t>(rows) * ha);
  float* cb = c.take<float>(rows);
  float* kn = c.take<float>(static_cast<size_t>(a->batch) * a->L);
  pr.live = pairs_carve(c, fused_groups(a->batch, a->T, f), f.ntiles);
  pr.q_aug = q_aug;
  pr.w_aug = w_aug;
  pr.cb = cb;
  pr.kn = kn;
  pr.ha = ha;
  const size_t live_bytes = static_cast<size_t>(fused_groups(a->batch, a->T, f)) * f.ntiles;
  {
    prof::Stage prep_stage("bounds");
    {
      prof::Launch pl(st, "dosa_prep");
      const int grid = static_cast<int>((rows + 7) / 8);
      if (a->d == 128)
        dosa_prep_kernel<128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(a->q), a->w, rows, a->H,
                                                    n_screen, ha, q_aug, w_aug, cb);
      else
        dosa_prep_kernel<64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(a->q), a->w, rows, a->H,
                                                   n_screen, ha, q_aug, w_aug, cb);
    }
    {
      prof::Launch pl(st, "key_norm");
      const long long nk = static_cast<long long>(a->batch) * a->L;
      const int grid = static_cast<int>(std::min<long long>((nk + 255) / 256, 8LL * num_sms()));
      if (a->d == 128)
        key_norm_kernel<128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(a->k), nk, kn);
      else
        key_norm_kernel<64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(a->k), nk, kn);
    }
    if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  }
  ScoreParams p = base_params(a, static_cast<unsigned*>(ws));
  DSA_TRY(fused_score_topk(a->d, a->H, p, a->q, a->k, a->L, topk, out_idx, out_score, scores, f, w, ws, st, &pr));
  if (out_live && cudaMemcpyAsync(out_live, pr.live.flags, live_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

// ------------------------------------------------------------ launch profiling
dsa_status dsa_profile_begin(void) {
  std::lock_guard<std::mutex> lock(prof::mu);
  for (auto& r : prof::recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  prof::recs.clear();
  prof::on.store(true);
  return DSA_OK;
}

int dsa_profile_end(char* names, size_t names_bytes, float* ms, int max_entries) {
  prof::on.store(false);
  std::lock_guard<std::mutex> lock(prof::mu);
  int n = 0;
  size_t used = 0;
  bool failed = false;
  for (auto& r : prof::recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) failed = true;
    if (n < max_entries && ms && names && used + r.name.size() + 1 <= names_bytes) {
      ms[n] = t;
      std::memcpy(names + used, r.name.c_str(), r.name.size() + 1);
      used += r.name.size() + 1;
      ++n;
    }
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  prof::recs.clear();
  return failed ? -1 : n;
}

// ------------------------------------------------------------ IndexCache
// Layers marked 'F' run their own indexer; layers marked 'S' reuse the top-k
// indices of the nearest preceding 'F' layer ("IndexCache: Accelerating Sparse
// Attention via Cross-Layer Index Reuse", section 2). Every F layer is
// validated before the first launch; S layers only need batch and T (their
// output shape), which must match their F layer's.
static dsa_status indexcache_check(const dsa_indexer_args* layers, int n_layers, const char* pattern,
                                   int topk, int32_t* const* out_idx, float* const* out_score) {
  if (!layers || !pattern || !out_idx || n_layers < 1 || topk < 1 || topk > (1 << 24)) return DSA_ERR_ARG;
  if (pattern[0] != 'F') return DSA_ERR_ARG;
  int f = 0;
  for (int l = 0; l < n_layers; ++l) {
    if (!out_idx[l]) return DSA_ERR_ARG;
    if (pattern[l] == 'F') {
      DSA_TRY(validate(&layers[l], false));
      f = l;
    } else if (pattern[l] == 'S') {
      if (layers[l].batch != layers[f].batch || layers[l].T != layers[f].T) return DSA_ERR_ARG;
      if (out_score && out_score[l] && !out_score[f]) return DSA_ERR_ARG;  // no scores to reuse
    } else {
      return DSA_ERR_ARG;  // includes a pattern shorter than n_layers
    }
  }
  return DSA_OK;
}

size_t indexcache_workspace_size(const dsa_indexer_args* layers, int n_layers, const char* pattern,
                                 int topk) {
  if (!layers || !pattern || n_layers < 1) return 0;
  size_t n = 0;
  for (int l = 0; l < n_layers; ++l) {
    if (pattern[l] != 'F' && pattern[l] != 'S') return 0;
    if (pattern[l] == 'F') {
      const size_t m = indexer_workspace_size(&layers[l], topk);
      if (m == 0) return 0;
      if (m > n) n = m;
    }
  }
  return n;
}

dsa_status indexcache_score_topk(const dsa_indexer_args* layers, int n_layers, const char* pattern,
                                 int topk, int32_t* const* out_idx, float* const* out_score, void* ws,
                                 size_t ws_bytes, void* stream) {
  DSA_TRY(indexcache_check(layers, n_layers, pattern, topk, out_idx, out_score));
  DSA_TRY(check_ws(ws, ws_bytes, indexcache_workspace_size(layers, n_layers, pattern, topk)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int f = 0;
  for (int l = 0; l < n_layers; ++l) {
    float* os = out_score ? out_score[l] : nullptr;
    if (pattern[l] == 'F') {
      f = l;
      DSA_TRY(indexer_score_topk(&layers[l], topk, out_idx[l], os, ws, ws_bytes, stream));
      continue;
    }
    // S: the cached indices of layer f (no copy when the caller aliases the buffers)
    const size_t n = static_cast<size_t>(layers[l].batch) * layers[l].T * topk;
    if (out_idx[l] != out_idx[f] &&
        cudaMemcpyAsync(out_idx[l], out_idx[f], n * sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return DSA_ERR_CUDA;
    const float* fs = out_score ? out_score[f] : nullptr;
    if (os && os != fs) {
      if (cudaMemcpyAsync(os, fs, n * sizeof(float), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return DSA_ERR_CUDA;
    }
  }
  return DSA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ no-allocation variant
// Dense score + top-k for callers that cannot allocate device memory. The
// scores scratch lives in a file-scope __device__ array that every device
// loading this library reserves until exit. Host code must not pass
// `g_noalloc_scratch` itself to a kernel: on the host that name is only a
// stand-in for the device symbol. Its device address is looked up with
// cudaGetSymbolAddress on every call, with the caller's device current, so a
// new primary context (after cudaDeviceReset, say), where the module may sit
// at another address, never sees a stale pointer. The lookup is a host-side
// table read once the module is loaded; the first call on a device loads it.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

dsa_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDev) return DSA_ERR_UNSUPPORTED;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
  *out = p;
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

// The status word of the static scratch: a bounded wait that gave up inside an
// indexer_score_topk_noalloc call on this device is reported here, as
// dsa_device_status reports it for a caller workspace.
extern "C" dsa_status dsa_noalloc_status(void* stream) {
  void* scratch = nullptr;
  DSA_TRY(noalloc_scratch(&scratch));
  return dsa_device_status(scratch, stream);
}
