// C ABI of the verify-step library: host-side argument checks, workspace
// layout, TMA descriptor creation, kernel launches and launch instrumentation.
// Declarations and the contract of every entry point: include/moe_verify.h.

#include <cudaTypedefs.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include "moe_verify.h"
#include "mv_device.cuh"
#include "mv_internal.h"

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};
std::atomic<int64_t> g_timeout_ns{2000000000LL};
constexpr int64_t kDefaultTimeoutNs = 2000000000LL;

mv_status fail(mv_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

mv_status cuda_fail(cudaError_t e, const char* what) {
  return fail(MV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int num_sms() {
  static std::mutex mu;
  static std::unordered_map<int, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  cache[dev] = n;
  return n;
}

// ---------------------------------------------------------------------------
// launch instrumentation
// ---------------------------------------------------------------------------
enum Kind {
  KIND_ROUTER = 0,
  KIND_PERMUTE,
  KIND_GEMM_MOE,
  KIND_COMBINE,
  KIND_COMBINE_ROUTE,
  KIND_LM_GEMM,
  KIND_LM_FINALIZE,
  KIND_ACCEPT,
  KIND_DRAFT_GEMM,
  KIND_DRAFT_LM,
  KIND_DRAFT_STEP,
  KIND_RMSNORM,
  KIND_ATTENTION,
  KIND_COUNT
};
const char* kKindNames[KIND_COUNT] = {"router_topk",       "expert_permute",     "grouped_moe_gemm",
                                      "combine_unpermute", "combine_route",      "lm_head_gemm_argmax",
                                      "lm_argmax_finalize", "greedy_accept",     "draft_block_gemm",
                                      "draft_lm_head_argmax", "draft_step", "rmsnorm", "decode_attention"};

struct ProfRec {
  int kind;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
std::atomic<bool> g_prof_on{false};
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Set while verify_graph_create records a step: launches then go into the
// graph instead of running, so they are neither timed nor counted here (a
// replay counts its kernels when it is launched).
thread_local bool t_recording = false;

template <class F>
cudaError_t run_kernel(int kind, cudaStream_t s, F&& launch) {
  cudaEvent_t a = nullptr, b = nullptr;
  const bool prof = !t_recording && g_prof_on.load(std::memory_order_relaxed);
  if (prof) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    a = take_event();
    b = take_event();
    cudaEventRecord(a, s);
  }
  cudaError_t e = launch();
  if (prof) {
    cudaEventRecord(b, s);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_recs.push_back({kind, a, b});
  }
  if (e == cudaSuccess && !t_recording) g_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}

// ---------------------------------------------------------------------------
// TMA descriptors: 2D bf16 [rows][cols] row-major, box = 64 columns x box_rows,
// 128-byte swizzle, zero fill out of bounds.  Cached by (address, shape, box).
// ---------------------------------------------------------------------------
struct TmKey {
  const void* ptr;
  uint64_t rows, cols;
  uint32_t box_rows;
  uint32_t rank;  // 2: [rows][cols] tiles; 3: [k-block][rows][64] view, two k-blocks per box
  bool operator==(const TmKey& o) const {
    return ptr == o.ptr && rows == o.rows && cols == o.cols && box_rows == o.box_rows && rank == o.rank;
  }
};
struct TmHash {
  size_t operator()(const TmKey& k) const {
    size_t h = reinterpret_cast<size_t>(k.ptr);
    h ^= (k.rows * 0x9E3779B97F4A7C15ull) + (h << 6) + (h >> 2);
    h ^= (k.cols * 0xC2B2AE3D27D4EB4Full) + (h << 6) + (h >> 2);
    h ^= k.box_rows + (h << 6) + (h >> 2);
    h ^= k.rank + (h << 6) + (h >> 2);
    return h;
  }
};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

std::mutex g_tm_mu;
std::unordered_map<TmKey, CUtensorMap, TmHash> g_tm_cache;

mv_status tmap_rank(CUtensorMap* out, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
                    uint32_t rank) {
  TmKey key{ptr, rows, cols, box_rows, rank};
  {
    std::lock_guard<std::mutex> lk(g_tm_mu);
    auto it = g_tm_cache.find(key);
    if (it != g_tm_cache.end()) {
      *out = it->second;
      return MV_OK;
    }
  }
  auto fn = encode_fn();
  if (!fn) return fail(MV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  CUtensorMap m;
  std::memset(&m, 0, sizeof(m));
  CUresult r;
  if (rank == 3) {
    // element (x, y, z) = row y, column 64 z + x: each box is two consecutive
    // 64-wide k-blocks of box_rows rows, stored k-block after k-block
    const cuuint64_t dims[3] = {64, rows, cols / 64};
    const cuuint64_t strides[2] = {cols * 2, 128};
    const cuuint32_t box[3] = {64, box_rows, 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  if (r != CUDA_SUCCESS)
    return fail(MV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for [%llu x %llu] box %u", static_cast<int>(r),
                static_cast<unsigned long long>(rows), static_cast<unsigned long long>(cols), box_rows);
  std::lock_guard<std::mutex> lk(g_tm_mu);
  if (g_tm_cache.size() > 8192) g_tm_cache.clear();
  g_tm_cache[key] = m;
  *out = m;
  return MV_OK;
}

mv_status tmap(CUtensorMap* out, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return tmap_rank(out, ptr, rows, cols, box_rows, 2);
}

// The weights-on-M GEMM tiles (GEMM_MOE_DECODE) read every operand through 3D
// maps, two k-blocks per box.
mv_status tmap3(CUtensorMap* out, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return tmap_rank(out, ptr, rows, cols, box_rows, 3);
}

// ---------------------------------------------------------------------------
// argument checks
// ---------------------------------------------------------------------------
#define MV_TRY(expr)                     \
  do {                                   \
    mv_status _st = (expr);              \
    if (_st != MV_OK) return _st;        \
  } while (0)

mv_status check_ptr(const void* p, const char* name, bool nullable = false) {
  if (!p) return nullable ? MV_OK : fail(MV_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(MV_ERR_MISALIGNED, "%s is not 16-byte aligned", name);
  return MV_OK;
}

mv_status check_shape(const mv_moe_shape* s) {
  if (!s) return fail(MV_ERR_INVALID_ARG, "shape is NULL");
  if (s->H <= 0 || s->E <= 0 || s->I <= 0 || s->I_shared < 0 || s->k <= 0)
    return fail(MV_ERR_INVALID_ARG, "shape has a non-positive size (H=%d E=%d I=%d I_shared=%d k=%d)",
                s->H, s->E, s->I, s->I_shared, s->k);
  if (s->k > s->E) return fail(MV_ERR_INVALID_ARG, "k=%d exceeds E=%d", s->k, s->E);
  if (s->H % 64 || s->I % 64 || s->I_shared % 64)
    return fail(MV_ERR_UNSUPPORTED_SHAPE, "H, I and I_shared must be multiples of 64 (H=%d I=%d I_shared=%d)",
                s->H, s->I, s->I_shared);
  if (s->E > 256 || s->k > 8)
    return fail(MV_ERR_UNSUPPORTED_SHAPE, "E must be <= 256 and k <= 8 (E=%d k=%d)", s->E, s->k);
  if (s->H > 16384 || s->I > 65536 || s->I_shared > 65536)
    return fail(MV_ERR_UNSUPPORTED_SHAPE, "H or I too large");
  return MV_OK;
}

mv_status check_rows(int64_t T, const mv_moe_shape* s) {
  if (T < 0) return fail(MV_ERR_INVALID_ARG, "T=%lld is negative", static_cast<long long>(T));
  const int64_t wide = std::max<int64_t>(std::max<int64_t>(s->H, s->I), s->I_shared);
  if (T * s->k * wide >= (int64_t(1) << 31) || T > (int64_t(1) << 24))
    return fail(MV_ERR_UNSUPPORTED_SHAPE, "T=%lld rows is too large for this shape", static_cast<long long>(T));
  return MV_OK;
}

mv_status check_weights(const mv_moe_weights* w, const mv_moe_shape* s) {
  if (!w) return fail(MV_ERR_INVALID_ARG, "weights is NULL");
  MV_TRY(check_ptr(w->w_router, "w_router"));
  MV_TRY(check_ptr(w->router_bias, "router_bias", true));
  MV_TRY(check_ptr(w->w_gate, "w_gate"));
  MV_TRY(check_ptr(w->w_up, "w_up"));
  MV_TRY(check_ptr(w->w_down, "w_down"));
  if (s->I_shared > 0) {
    MV_TRY(check_ptr(w->ws_gate, "ws_gate"));
    MV_TRY(check_ptr(w->ws_up, "ws_up"));
    MV_TRY(check_ptr(w->ws_down, "ws_down"));
  }
  MV_TRY(check_ptr(w->norm_gain, "norm_gain", true));
  return MV_OK;
}

// ---------------------------------------------------------------------------
// workspace layouts (every region 1024-byte aligned relative to the base)
// ---------------------------------------------------------------------------
constexpr size_t kHeader = 1024;  // sticky error word + reserved
constexpr size_t kSchedBytes = mv::kSchedInts * sizeof(int);  // scheduling state of one GEMM launch

struct Carve {
  char* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = align_up(off + count * sizeof(T), 1024);
    return p;
  }
};

struct FfnWs {
  int32_t *counts, *offsets, *perm, *inv, *sort;
  int32_t* inv_alt;  // slab layout: the other layer's inverse map (layers alternate)
  int32_t* ent;      // slab layout: the routing entry (r * k + j) of each slab row
  uint16_t *x_perm, *a_perm, *a_sh;
  float *y_perm, *y_sh;
  int64_t n_pos;     // rows of x_perm / a_perm / y_perm
};

// Decode-sized verify steps group the routed rows by expert inside the
// routing kernel (combine_route) instead of a permute launch: expert e owns
// rows [e*T, (e+1)*T) of x_perm and a_perm (a row selects an expert at most
// once, so T rows always suffice) and its row count is an atomic counter in
// the layer's scheduling block; the down projection stores its outputs in
// y_perm by routing entry (row * k + slot, through the `ent` map the routing
// kernel writes), so the combine reads them without a gather map.  Larger
// batches keep the compact stable permutation.
bool use_slabs(int64_t T, const mv_moe_shape& s) {
  return T * s.k <= 16LL * s.E && mv::combine_route_supported(static_cast<int>(T), s.H, s.E);
}
constexpr int kSlabCountOff = 768;  // per-expert slab counters within a layer's scheduling block
static_assert(1 + mv::kMaxGroups <= kSlabCountOff && kSlabCountOff + 256 <= mv::kSchedInts, "scheduling block");

FfnWs carve_ffn(Carve& c, int64_t T, const mv_moe_shape& s, bool slabs = false) {
  FfnWs w;
  const size_t n = static_cast<size_t>(T) * s.k;
  const size_t rows = slabs ? static_cast<size_t>(T) * s.E : n;
  w.n_pos = static_cast<int64_t>(rows);
  w.counts = c.take<int32_t>(s.E);
  w.offsets = c.take<int32_t>(s.E + 1);
  w.perm = c.take<int32_t>(n);
  w.inv = c.take<int32_t>(n);
  w.inv_alt = slabs ? c.take<int32_t>(n) : nullptr;
  w.ent = slabs ? c.take<int32_t>(rows) : nullptr;
  w.sort = c.take<int32_t>(mv::permute_uses_sort(static_cast<int>(T), s.k) ? mv::sort_scratch_ints(static_cast<int>(T), s.E, s.k) : 1);
  w.x_perm = c.take<uint16_t>(rows * s.H);
  w.a_perm = c.take<uint16_t>(rows * s.I);
  w.a_sh = c.take<uint16_t>(static_cast<size_t>(T) * s.I_shared);
  w.y_perm = c.take<float>(rows * s.H);
  w.y_sh = c.take<float>(static_cast<size_t>(T) * s.H);
  return w;
}

constexpr int kMaxLayers = 64;  // decoder layers one verify_step call may run

int lm_parts(int V) { return (V + 255) / 256 * 4; }  // (256-row vocabulary tile, lane quarter)
int lm_parts_alloc(int V) { return (V + 127) / 128 * 4; }  // any split into 256- and 128-row tiles
#ifndef MV_LM_PAIR_MIN_ROWS
#define MV_LM_PAIR_MIN_ROWS 256
#endif
constexpr int kLmPairMinRows = MV_LM_PAIR_MIN_ROWS;  // LM heads of this many rows or more run on CTA pairs

uint64_t timeout_ns() {
  const int64_t t = g_timeout_ns.load();
  return static_cast<uint64_t>(t > 0 ? t : kDefaultTimeoutNs);
}

int gemm_grid(int64_t units) {
  const int sms = num_sms();
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units, sms)));
}

// ---------------------------------------------------------------------------
// the path
// ---------------------------------------------------------------------------
// The weights the grouped MoE GEMM of a layer streams first, in claim order
// (shared gate/up, then the routed gate/up of experts 0, 1, ...), up to
// `budget` bytes: what a kernel running before it can pull into L2 while HBM
// is otherwise idle.  A batch of T rows with T * k <= E touches only a few
// experts, unknown before its routing, so there the shared expert (gate, up
// and down) is all that is prefetched.
mv::L2Prefetch moe_first_wave(const mv_moe_shape& s, const mv_moe_weights& w, uint64_t budget, int64_t T = 0) {
  mv::L2Prefetch pf{};
  const uint64_t sh = static_cast<uint64_t>(s.I_shared) * s.H * 2;
  if (T > 0 && T * s.k <= s.E) {  // few rows: the shared expert only (which routed experts is unknown)
    if (s.I_shared > 0 && budget >= 3 * sh) {
      pf.ptr[0] = w.ws_gate;
      pf.bytes[0] = sh;
      pf.ptr[1] = w.ws_up;
      pf.bytes[1] = sh;
      pf.ptr[2] = w.ws_down;
      pf.bytes[2] = sh;
      pf.n = 3;
    }
    return pf;
  }
  if (s.I_shared > 0 && budget >= 2 * sh) {
    pf.ptr[pf.n] = w.ws_gate;
    pf.bytes[pf.n++] = sh;
    pf.ptr[pf.n] = w.ws_up;
    pf.bytes[pf.n++] = sh;
    budget -= 2 * sh;
  }
  const uint64_t per_expert = static_cast<uint64_t>(s.I) * s.H * 2;
  const uint64_t ne = std::min<uint64_t>(s.E, budget / (2 * per_expert));
  if (ne > 0) {
    pf.ptr[pf.n] = w.w_gate;
    pf.bytes[pf.n++] = ne * per_expert;
    pf.ptr[pf.n] = w.w_up;
    pf.bytes[pf.n++] = ne * per_expert;
  }
  return pf;
}

// The first vocabulary rows of the LM head, up to `budget` bytes.
mv::L2Prefetch lm_first_wave(const uint16_t* w_lm, int V, int H, uint64_t budget) {
  mv::L2Prefetch pf{};
  pf.ptr[0] = w_lm;
  pf.bytes[0] = std::min<uint64_t>(static_cast<uint64_t>(V) * H * 2, budget) & ~uint64_t(15);
  pf.n = 1;
  return pf;
}

#ifndef MV_PREFETCH_BUDGET_MB
#define MV_PREFETCH_BUDGET_MB 24  // measured best of 0 / 8 / 16 / 20 / 24 / 32 / 40 / 48 / 64 / 96 MB on the concurrency-32 step
#endif
constexpr uint64_t kPrefetchBudget = static_cast<uint64_t>(MV_PREFETCH_BUDGET_MB) << 20;

// The fused grouped GEMM of one MoE layer: gate/up (SwiGLU epilogue) and down
// projection (fp32 rows) of the shared expert and the routed experts in one
// persistent launch; a down unit waits for its expert's gate/up units.
mv_status moe_gemm_impl(const uint16_t* x, int T, const mv_moe_shape& s, const mv_moe_weights& w,
                        const FfnWs& ws, int* err, int* sched, cudaStream_t st,
                        const int32_t* slab_counts = nullptr) {
  const int H = s.H, E = s.E, I = s.I, Ish = s.I_shared, k = s.k;
  const int n = T * k;
  const bool decode = static_cast<int64_t>(n) <= 16LL * E;  // routed groups average <= 16 rows
  const int BN = decode ? 32 : 128;
  mv::GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.err = err;
  p.sched = sched;
  p.timeout_ns = timeout_ns();
  int ns = 0;
  int64_t units = 0;
  int sh1 = -1, rt1 = -1;
  auto base = [](mv::GemmSet& S, int mode, int epi) {
    S.mode = mode;
    S.epi = epi;
    S.m_tile = 128;
    S.dep_set = -1;
  };
  const bool tokm = !decode;  // large groups: tokens on the MMA's M side
  // Large groups run on CTA pairs (cta_group::2) when pairs can be resident:
  // 256-token units, every operand through 3D maps with 128-row boxes.
  const int pair_clusters = tokm ? mv::gemm_pair_max_clusters() : 0;
  const bool pair = pair_clusters > 0;
  const int bbox = decode ? mv::kDecodeBBox : mv::kPrefillBBox;
  auto map = [decode, pair](CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box) {
    if (pair) return mv::kPairKB == 2 ? tmap3(m, ptr, rows, cols, 128) : tmap(m, ptr, rows, cols, 128);
    return decode ? tmap3(m, ptr, rows, cols, box) : tmap(m, ptr, rows, cols, box);
  };
  if (Ish > 0) {  // shared expert, gate/up
    mv::GemmSet& S = p.set[ns];
    base(S, tokm ? mv::MODE_TGATEUP : mv::MODE_GATEUP, tokm ? mv::EPI_SWIGLU_ROWS : mv::EPI_SWIGLU);
    MV_TRY(map(&S.a0, w.ws_gate, Ish, H, 128));
    MV_TRY(map(&S.a1, w.ws_up, Ish, H, 128));
    MV_TRY(map(&S.b, x, T, H, bbox));
    S.out = ws.a_sh;
    S.ld_out = Ish;
    S.K = H;
    S.M = Ish;
    S.groups = 1;
    S.static_rows = T;
    S.signal = 1;
    units += int64_t((Ish + 127) / 128) * ((T + BN - 1) / BN);
    sh1 = ns++;
  }
  {  // routed experts, gate/up
    mv::GemmSet& S = p.set[ns];
    base(S, tokm ? mv::MODE_TGATEUP : mv::MODE_GATEUP, tokm ? mv::EPI_SWIGLU_ROWS : mv::EPI_SWIGLU);
    MV_TRY(map(&S.a0, w.w_gate, static_cast<uint64_t>(E) * I, H, 128));
    MV_TRY(map(&S.a1, w.w_up, static_cast<uint64_t>(E) * I, H, 128));
    MV_TRY(map(&S.b, ws.x_perm, ws.n_pos, H, bbox));
    S.out = ws.a_perm;
    S.ld_out = I;
    S.K = H;
    S.M = I;
    S.groups = E;
    S.counts = slab_counts ? slab_counts : ws.counts;
    S.offsets = slab_counts ? nullptr : ws.offsets;
    S.slab_rows = slab_counts ? T : 0;
    S.a_group_stride = I;
    S.signal = 1;
    units += int64_t((I + 127) / 128) * (std::min(E, n) + (n + BN - 1) / BN);
    rt1 = ns++;
  }
  // Decode tiles put the weights on the MMA's M side; the down projection
  // pairs two k-blocks per stage (MODE_KPAIR).  Prefill tiles put 128 tokens
  // on M and 256 weight rows on N (gate|up, or two halves of W_down).  Either
  // way every stage carries 32 KB of weights.
  const int down_mode = decode ? mv::MODE_KPAIR : (tokm ? mv::MODE_TPAIR : mv::MODE_MPAIR);
  const int down_epi = tokm ? mv::EPI_STORE_ROWS : mv::EPI_STORE_F32;
  const int down_tile = decode ? 128 : 256;
  if (Ish > 0) {  // shared expert, down
    mv::GemmSet& S = p.set[ns++];
    base(S, down_mode, down_epi);
    S.m_tile = down_tile;
    MV_TRY(map(&S.a0, w.ws_down, H, Ish, decode ? 128 : 256));  // MODE_TPAIR: one 256-row box
    MV_TRY(map(&S.b, ws.a_sh, T, Ish, bbox));
    S.a1 = S.a0;
    S.out = ws.y_sh;
    S.ld_out = H;
    S.K = Ish;
    S.M = H;
    S.groups = 1;
    S.static_rows = T;
    S.dep_set = sh1;
    units += int64_t((H + 127) / 128) * ((T + BN - 1) / BN);
  }
  {  // routed experts, down
    mv::GemmSet& S = p.set[ns++];
    base(S, down_mode, down_epi);
    S.m_tile = down_tile;
    MV_TRY(map(&S.a0, w.w_down, static_cast<uint64_t>(E) * H, I, decode ? 128 : 256));
    MV_TRY(map(&S.b, ws.a_perm, ws.n_pos, I, bbox));
    S.a1 = S.a0;
    S.out = ws.y_perm;
    // slab layout: rows are stored by routing entry, so the combine needs no gather map
    S.row_map = slab_counts ? ws.ent : nullptr;
    S.ld_out = H;
    S.K = I;
    S.M = H;
    S.groups = E;
    S.counts = slab_counts ? slab_counts : ws.counts;
    S.offsets = slab_counts ? nullptr : ws.offsets;
    S.slab_rows = slab_counts ? T : 0;
    S.a_group_stride = H;
    S.dep_set = rt1;
    units += int64_t((H + 127) / 128) * (std::min(E, n) + (n + BN - 1) / BN);
  }
  p.nsets = ns;
  // With few rows (a few experts' units for the whole GPU) the down units'
  // weights go out while their gate/up groups finish: 570 -> 560 us per
  // 12-layer batch-1 step.  At 128 rows it measured 4 us a step slower.
  const int config = !decode ? mv::GEMM_MOE_PREFILL : (n <= E ? mv::GEMM_MOE_DECODE_FEW : mv::GEMM_MOE_DECODE);
  cudaError_t e = run_kernel(KIND_GEMM_MOE, st, [&] {
    if (pair) return mv::launch_gemm_pair(p, pair_clusters, st);
    return mv::launch_gemm(config, p, gemm_grid(units), st);
  });
  return e == cudaSuccess ? MV_OK : cuda_fail(e, "grouped_moe_gemm launch");
}

// Grouping, fused GEMM and (unless do_combine is false: the caller fuses the
// combine into the next layer's routing) the combine of one MoE layer.
mv_status ffn_forward_impl(const uint16_t* x, int T, const mv_moe_shape& s, const mv_moe_weights& w,
                           const int32_t* idx, const float* tw, const uint16_t* res, uint16_t* out,
                           const FfnWs& ws, int* err, int* sched, cudaStream_t st, bool do_combine = true,
                           const mv::L2Prefetch& combine_pf = mv::L2Prefetch{},
                           const int32_t* slab_counts = nullptr, const int32_t* slab_inv = nullptr) {
  // With slab_counts the routing kernel has already grouped the rows (slab
  // layout; slab_inv is its inverse map) and no permute launch is needed.
  cudaError_t e = cudaSuccess;
  if (!slab_counts) {
    e = run_kernel(KIND_PERMUTE, st, [&] {
      if (mv::permute_uses_sort(T, s.k))
        return mv::launch_permute_sorted(idx, T, s.E, s.k, ws.counts, ws.offsets, ws.perm, ws.inv, x, s.H, ws.x_perm,
                                         ws.sort, st);
      return mv::launch_permute(idx, T, s.E, s.k, ws.counts, ws.offsets, ws.perm, ws.inv, x, s.H, ws.x_perm, st);
    });
    if (e != cudaSuccess) return cuda_fail(e, "expert_permute launch");
  }
  MV_TRY(moe_gemm_impl(x, T, s, w, ws, err, sched, st, slab_counts));
  if (!do_combine) return MV_OK;
  const int32_t* inv = slab_counts ? slab_inv : ws.inv;
  e = run_kernel(KIND_COMBINE, st, [&] {
    return mv::launch_combine(ws.y_perm, s.I_shared > 0 ? ws.y_sh : nullptr, inv, tw, res, out, T, s.H, s.k,
                              static_cast<int>(ws.n_pos), err, combine_pf, st, slab_counts != nullptr);
  });
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  return MV_OK;
}

// Routing of T rows: the streaming combine+route kernel in route-only mode for
// decode-sized batches, the shared-memory-staged router up to 1024 rows (both
// give bit-identical logits and choices), the tensor cores beyond (fp32 logits
// summed in another order: choices can differ only at near-tied logits).
mv_status route_impl(const uint16_t* x, int T, const mv_moe_shape& s, const uint16_t* wr, const float* bias,
                     int32_t* idx, float* tw, int* err, cudaStream_t st,
                     const mv::L2Prefetch& pf = mv::L2Prefetch{}) {
  if (T > 1024 && s.E <= 128) {
    // Large batches: the router is a [T x H] . [H x E] contraction on the tensor
    // cores, 128 tokens x E experts per unit; each epilogue thread holds one
    // token's logits and does the top-k and renormalised softmax in registers.
    // Static unit schedule, so no workspace is needed.
    mv::GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.err = err;
    p.sched = nullptr;
    p.timeout_ns = timeout_ns();
    mv::GemmSet& S = p.set[0];
    S.mode = mv::MODE_TROUTE;
    S.epi = mv::EPI_TOPK;
    S.m_tile = 128;
    S.dep_set = -1;
    MV_TRY(tmap(&S.a0, wr, s.E, s.H, 128));
    MV_TRY(tmap(&S.b, x, T, s.H, mv::kPrefillBBox));
    S.a1 = S.a0;
    S.out = idx;
    S.out2 = tw;
    S.bias = bias;
    S.topk = s.k;
    S.K = s.H;
    S.M = s.E;
    S.groups = 1;
    S.static_rows = T;
    p.nsets = 1;
    const int64_t units = (T + 127) / 128;
    cudaError_t e = run_kernel(KIND_ROUTER, st, [&] {
      return mv::launch_gemm(mv::GEMM_MOE_PREFILL, p, gemm_grid(units), st);
    });
    return e == cudaSuccess ? MV_OK : cuda_fail(e, "router_topk (tensor-core) launch");
  }
  cudaError_t e = run_kernel(KIND_ROUTER, st, [&] {
    if (mv::combine_route_supported(T, s.H, s.E)) {
      mv::CombineRouteArgs a{};
      a.x = x;
      a.T = T;
      a.H = s.H;
      a.E = s.E;
      a.k = s.k;
      a.wr = wr;
      a.bias = bias;
      a.idx = idx;
      a.w = tw;
      a.err = err;
      a.timeout_ns = timeout_ns();
      a.pf = pf;
      return mv::launch_combine_route(a, st);
    }
    return mv::launch_router(x, T, s.H, s.E, s.k, wr, bias, idx, tw, err, timeout_ns(), st);
  });
  return e == cudaSuccess ? MV_OK : cuda_fail(e, "router_topk launch");
}

// LM head + fused argmax.  Units are 256-row vocabulary tiles (two 128-row
// halves sharing each token k-block).  With `balance`, whole waves of the
// persistent grid take 256-row units and the rows left over are cut into
// 128-row units, so the last wave is half as long; keys then need up to
// lm_parts_alloc(V) slots per token.  Returns the key slots used per token
// (the row stride of `parts` is `ld`).
mv_status lm_gemm_impl(const uint16_t* h, int T, int H, const uint16_t* w_lm, int V, uint64_t* parts, int ld,
                       int* err, int* sched, cudaStream_t st, bool balance, int* nparts_used,
                       int kind = KIND_LM_GEMM) {
  mv::GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.err = err;
  p.sched = sched;
  p.timeout_ns = timeout_ns();
  // From 256 rows the contraction is tensor-bound (each vocabulary tile is
  // reused by several token tiles) and runs on CTA pairs: 256 tokens x 256
  // vocabulary rows per unit, each SM loading half of both, so a k-block
  // costs an SM 32 KB of shared-memory fill instead of 48 KB.
  const int pair_clusters = T >= kLmPairMinRows ? mv::gemm_pair_max_clusters() : 0;
  if (pair_clusters > 0) {
    mv::GemmSet& S = p.set[0];
    S.mode = mv::MODE_TLM;
    S.epi = mv::EPI_ARGMAX_ROWS;
    S.m_tile = 256;
    S.dep_set = -1;
    const auto pmap = [](CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols) {
      return mv::kPairKB == 2 ? tmap3(m, ptr, rows, cols, 128) : tmap(m, ptr, rows, cols, 128);
    };
    MV_TRY(pmap(&S.a0, w_lm, V, H));
    MV_TRY(pmap(&S.b, h, T, H));
    S.a1 = S.a0;
    S.out = parts;
    S.ld_out = ld;
    S.K = H;
    S.M = V;
    S.groups = 1;
    S.static_rows = T;
    p.nsets = 1;
    const int used = (V + 255) / 256;  // one key per token and 256-row vocabulary tile
    if (used > ld) return fail(MV_ERR_INTERNAL, "LM key slots %d exceed the row stride %d", used, ld);
    *nparts_used = used;
    const int64_t units = int64_t(used) * ((T + 255) / 256);
    const int clusters = static_cast<int>(std::min<int64_t>(pair_clusters, units));
    cudaError_t e = run_kernel(kind, st, [&] { return mv::launch_gemm_pair(p, clusters, st); });
    if (e != cudaSuccess) return cuda_fail(e, "lm_head_gemm_argmax launch");
    return MV_OK;
  }
  const int nt = (T + 127) / 128;
  const bool wide = T >= 128;  // whole 128-row token tiles: one TMA box per stage
  const int bbox = wide ? mv::kLmWideBBox : mv::kLmBBox;
  const int n256 = (V + 255) / 256;
  const int sms = num_sms();
  int V0 = V;  // rows served by 256-row units
  if (balance && n256 * nt > sms && (n256 * nt) % sms != 0) {
    const int full_units = ((n256 * nt) / sms) * sms;
    V0 = std::min(V, (full_units / nt) * 256);
  }
  auto set_up = [&](mv::GemmSet& S, const uint16_t* a_base, int rows, int row_base, int part_base, bool pair) {
    S.mode = pair ? mv::MODE_MPAIR : mv::MODE_SINGLE;
    S.epi = mv::EPI_ARGMAX;
    S.m_tile = pair ? 256 : 128;
    S.dep_set = -1;
    S.key_row_base = row_base;
    S.key_part_base = part_base;
    S.out = parts;
    S.ld_out = ld;
    S.K = H;
    S.M = rows;
    S.groups = 1;
    S.static_rows = T;
    return MV_OK;
  };
  int ns = 0;
  int used = 0;
  int64_t units = 0;
  if (V0 > 0) {
    mv::GemmSet& S = p.set[ns++];
    MV_TRY(tmap(&S.a0, w_lm, V0, H, 256));  // MODE_MPAIR: both 128-row halves in one box
    MV_TRY(tmap(&S.b, h, T, H, bbox));
    S.a1 = S.a0;
    set_up(S, w_lm, V0, 0, 0, true);
    used = (V0 + 255) / 256 * 4;
    units += int64_t((V0 + 255) / 256) * nt;
  }
  if (V0 < V) {
    mv::GemmSet& S = p.set[ns++];
    const uint16_t* tail = w_lm + static_cast<size_t>(V0) * H;
    MV_TRY(tmap(&S.a0, tail, V - V0, H, 128));
    MV_TRY(tmap(&S.b, h, T, H, bbox));
    S.a1 = S.a0;
    set_up(S, tail, V - V0, V0, used, false);
    used += (V - V0 + 127) / 128 * 4;
    units += int64_t((V - V0 + 127) / 128) * nt;
  }
  p.nsets = ns;
  if (used > ld) return fail(MV_ERR_INTERNAL, "LM key slots %d exceed the row stride %d", used, ld);
  *nparts_used = used;
  cudaError_t e = run_kernel(kind, st, [&] { return mv::launch_gemm(wide ? mv::GEMM_LM_WIDE : mv::GEMM_LM, p, gemm_grid(units), st); });
  if (e != cudaSuccess) return cuda_fail(e, "lm_head_gemm_argmax launch");
  return MV_OK;
}

// ---------------------------------------------------------------------------
// decoder self-attention over the key/value cache
// ---------------------------------------------------------------------------
constexpr int kAttnHeadDim = 128;
constexpr int kAttnMaxHeads = 256;

// Positions per split of one (sequence, head): a fixed 1,024, so the split
// boundaries (and with them the fp32 summation order of every row) depend on
// nothing but the position: a sequence gives the same bits whatever B, K or
// max_ctx the call has (batch invariance).  At 128 rows and 4,096 cached
// positions that is 5 splits per pair, 1,600 CTAs: several waves of the GPU
// (512-position splits measured 7 % slower: twice the per-CTA set-up and
// merge for the same bytes).
constexpr int kAttnSplit = 1024;
struct AttnPlan {
  int split_len, n_split, nq;
};
AttnPlan attn_plan(int64_t B, int K, int n_heads, int max_ctx) {
  (void)B;
  (void)n_heads;
  AttnPlan pl{};
  pl.nq = mv::attention_nq(K);
  const int64_t n_keys = static_cast<int64_t>(max_ctx) + K + 1;
  pl.split_len = kAttnSplit;
  pl.n_split = static_cast<int>((n_keys + kAttnSplit - 1) / kAttnSplit);
  return pl;
}

struct AttnWs {
  int* counters;
  float* part_ml;
  float* part_o;
};
AttnWs carve_attn(Carve& c, int64_t B, int n_heads, const AttnPlan& pl) {
  AttnWs w;
  const size_t pairs = static_cast<size_t>(B) * n_heads;
  w.counters = c.take<int>(pairs);
  w.part_ml = c.take<float>(pairs * pl.n_split * pl.nq * 2);
  w.part_o = c.take<float>(pairs * pl.n_split * pl.nq * kAttnHeadDim);
  return w;
}

}  // namespace

// ===========================================================================
// exported entry points
// ===========================================================================
extern "C" {

const char* mv_last_error(void) { return g_last_error.c_str(); }

const char* mv_version(void) { return "moe_verify 0.1.0 sm_100a"; }

uint64_t mv_launch_count(void) { return g_launches.load(); }

void mv_set_wait_timeout_ns(int64_t ns) { g_timeout_ns.store(ns > 0 ? ns : kDefaultTimeoutNs); }

void mv_profile_enable(int32_t on) { g_prof_on.store(on != 0); }

const char* mv_kernel_name(int32_t kind) {
  return (kind >= 0 && kind < KIND_COUNT) ? kKindNames[kind] : nullptr;
}

int32_t mv_profile_collect(int64_t* launches, double* total_ms, int32_t n_kinds) {
  std::vector<ProfRec> recs;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    recs.swap(g_prof_recs);
  }
  const int n = std::min<int>(n_kinds, KIND_COUNT);
  for (int i = 0; i < n; ++i) {
    if (launches) launches[i] = 0;
    if (total_ms) total_ms[i] = 0.0;
  }
  for (auto& r : recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess &&
        r.kind < n) {
      if (launches) launches[r.kind] += 1;
      if (total_ms) total_ms[r.kind] += ms;
    }
  }
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : recs) {
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  return n;
}

mv_status moe_router_topk(const uint16_t* x, int32_t T, const mv_moe_shape* shape, const uint16_t* w_router,
                          const float* router_bias, int32_t* topk_idx, float* topk_w, mv_stream_t stream) {
  MV_TRY(check_shape(shape));
  MV_TRY(check_rows(T, shape));
  MV_TRY(check_ptr(x, "x"));
  MV_TRY(check_ptr(w_router, "w_router"));
  MV_TRY(check_ptr(router_bias, "router_bias", true));
  MV_TRY(check_ptr(topk_idx, "topk_idx"));
  MV_TRY(check_ptr(topk_w, "topk_w"));
  if (T == 0) return MV_OK;
  return route_impl(x, T, *shape, w_router, router_bias, topk_idx, topk_w, nullptr,
                    reinterpret_cast<cudaStream_t>(stream));
}

mv_status moe_expert_permute(const int32_t* topk_idx, int32_t T, int32_t E, int32_t k, int32_t* counts,
                             int32_t* offsets, int32_t* perm, int32_t* inv, mv_stream_t stream) {
  if (T < 0 || E <= 0 || E > 256 || k <= 0 || k > 8 || k > E)
    return fail(MV_ERR_INVALID_ARG, "bad sizes T=%d E=%d k=%d", T, E, k);
  MV_TRY(check_ptr(topk_idx, "topk_idx", T == 0));
  MV_TRY(check_ptr(counts, "counts"));
  MV_TRY(check_ptr(offsets, "offsets"));
  MV_TRY(check_ptr(perm, "perm", T == 0));
  MV_TRY(check_ptr(inv, "inv", T == 0));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // H = 0: no rows are gathered
  cudaError_t e = run_kernel(KIND_PERMUTE, st, [&] {
    return mv::launch_permute(topk_idx, T, E, k, counts, offsets, perm, inv, nullptr, 0, nullptr, st);
  });
  return e == cudaSuccess ? MV_OK : cuda_fail(e, "expert_permute launch");
}

mv_status moe_rmsnorm(const uint16_t* x, int32_t T, int32_t H, const uint16_t* gain, uint16_t* out,
                      mv_stream_t stream) {
  if (T < 0 || H <= 0) return fail(MV_ERR_INVALID_ARG, "bad sizes T=%d H=%d", T, H);
  if (H % 8) return fail(MV_ERR_UNSUPPORTED_SHAPE, "H=%d must be a multiple of 8", H);
  MV_TRY(check_ptr(x, "x", T == 0));
  MV_TRY(check_ptr(gain, "gain"));
  MV_TRY(check_ptr(out, "out", T == 0));
  if (T > 0 && out == x) return fail(MV_ERR_INVALID_ARG, "out may not alias x");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = run_kernel(KIND_RMSNORM, st, [&] { return mv::launch_rmsnorm(x, T, H, gain, out, st); });
  return e == cudaSuccess ? MV_OK : cuda_fail(e, "rmsnorm launch");
}

size_t moe_ffn_workspace_size(int32_t T, const mv_moe_shape* shape) {
  if (!shape || T < 0) return 0;
  Carve c{nullptr};
  c.take<char>(kSchedBytes);
  carve_ffn(c, T, *shape);
  return kHeader + c.off + 1024;
}

mv_status moe_ffn_forward(const uint16_t* x, int32_t T, const mv_moe_shape* shape, const mv_moe_weights* weights,
                          const int32_t* topk_idx, const float* topk_w, const uint16_t* residual, uint16_t* out,
                          void* ws, size_t ws_bytes, mv_stream_t stream) {
  MV_TRY(check_shape(shape));
  MV_TRY(check_rows(T, shape));
  MV_TRY(check_weights(weights, shape));
  MV_TRY(check_ptr(x, "x"));
  MV_TRY(check_ptr(topk_idx, "topk_idx"));
  MV_TRY(check_ptr(topk_w, "topk_w"));
  MV_TRY(check_ptr(residual, "residual", true));
  MV_TRY(check_ptr(out, "out"));
  MV_TRY(check_ptr(ws, "workspace"));
  if (out == x) return fail(MV_ERR_INVALID_ARG, "out may not alias x");
  const size_t need = moe_ffn_workspace_size(T, shape);
  if (ws_bytes < need)
    return fail(MV_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, %zu needed", ws_bytes, need);
  if (T == 0) return MV_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Carve c{static_cast<char*>(ws) + kHeader};
  int* sched = c.take<int>(mv::kSchedInts);
  FfnWs fw = carve_ffn(c, T, *shape);
  cudaError_t e = cudaMemsetAsync(sched, 0, kSchedBytes, st);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the scheduling state");
  return ffn_forward_impl(x, T, *shape, *weights, topk_idx, topk_w, residual, out, fw, static_cast<int*>(ws), sched,
                          st);
}

size_t lm_head_workspace_size(int32_t T, int32_t V) {
  if (T < 0 || V <= 0) return 0;
  return kHeader + kSchedBytes + align_up(static_cast<size_t>(lm_parts_alloc(V)) * T * 8, 1024) + 1024;
}

mv_status lm_head_argmax(const uint16_t* h, int32_t T, int32_t H, const uint16_t* w_lm, int32_t V, int32_t* argmax,
                         void* ws, size_t ws_bytes, mv_stream_t stream) {
  if (T < 0 || H <= 0 || V <= 0) return fail(MV_ERR_INVALID_ARG, "bad sizes T=%d H=%d V=%d", T, H, V);
  if (H % 64 || V % 8 || H > 16384 || T > (1 << 24))
    return fail(MV_ERR_UNSUPPORTED_SHAPE, "H must be a multiple of 64 and V of 8 (H=%d V=%d)", H, V);
  MV_TRY(check_ptr(h, "h"));
  MV_TRY(check_ptr(w_lm, "w_lm"));
  MV_TRY(check_ptr(argmax, "argmax"));
  MV_TRY(check_ptr(ws, "workspace"));
  const size_t need = lm_head_workspace_size(T, V);
  if (ws_bytes < need)
    return fail(MV_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, %zu needed", ws_bytes, need);
  if (T == 0) return MV_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* sched = reinterpret_cast<int*>(static_cast<char*>(ws) + kHeader);
  uint64_t* parts = reinterpret_cast<uint64_t*>(static_cast<char*>(ws) + kHeader + kSchedBytes);
  cudaError_t e0 = cudaMemsetAsync(sched, 0, kSchedBytes, st);
  if (e0 != cudaSuccess) return cuda_fail(e0, "clearing the scheduling state");
  int used = 0;
  MV_TRY(lm_gemm_impl(h, T, H, w_lm, V, parts, lm_parts_alloc(V), static_cast<int*>(ws), sched, st, true, &used));
  cudaError_t e = run_kernel(KIND_LM_FINALIZE, st, [&] {
    return mv::launch_lm_finalize(parts, used, lm_parts_alloc(V), T, argmax, st);
  });
  return e == cudaSuccess ? MV_OK : cuda_fail(e, "lm_argmax_finalize launch");
}

mv_status greedy_accept(const int32_t* argmax, const int32_t* drafts, int32_t B, int32_t K, int32_t* accepted,
                        int32_t* next_token, int32_t* emitted, mv_stream_t stream) {
  if (B < 0 || K < 0 || K > 32) return fail(MV_ERR_INVALID_ARG, "bad sizes B=%d K=%d (K <= 32)", B, K);
  MV_TRY(check_ptr(argmax, "argmax", B == 0));
  MV_TRY(check_ptr(drafts, "drafts", K == 0 || B == 0));
  MV_TRY(check_ptr(accepted, "accepted", B == 0));
  MV_TRY(check_ptr(next_token, "next_token", B == 0));
  MV_TRY(check_ptr(emitted, "emitted", true));
  if (B == 0) return MV_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = run_kernel(KIND_ACCEPT, st, [&] {
    return mv::launch_accept(argmax, K > 0 ? drafts : nullptr, B, K, accepted, next_token, emitted, st);
  });
  return e == cudaSuccess ? MV_OK : cuda_fail(e, "greedy_accept launch");
}

size_t verify_step_workspace_size(int32_t B, int32_t K, const mv_moe_shape* shape, int32_t V) {
  if (!shape || B < 0 || K < 0 || V <= 0) return 0;
  const int64_t T = int64_t(B) * (K + 1);
  Carve c{nullptr};
  c.take<uint16_t>(static_cast<size_t>(T) * shape->H);
  c.take<uint16_t>(static_cast<size_t>(T) * shape->H);
  c.take<int32_t>(static_cast<size_t>(T) * shape->k * 2);
  c.take<float>(static_cast<size_t>(T) * shape->k * 2);
  c.take<uint64_t>(static_cast<size_t>(lm_parts_alloc(V)) * T);
  c.take<char>(kSchedBytes * (kMaxLayers + 1));
  carve_ffn(c, T, *shape, use_slabs(T, *shape));
  c.take<uint16_t>(static_cast<size_t>(T) * shape->H);  // normalised rows (pre-RMSNorm layers)
  return kHeader + c.off + 1024;
}

// The verify step; *h_final (when given) receives the device address of the
// last layer's hidden rows (inside the workspace, or `hidden` with no layers).
// The host-side argument checks of verify_step (shared with the graph
// executor, which must reject bad arguments before touching the GPU).
static mv_status verify_step_check(const uint16_t* hidden, const int32_t* drafts, int32_t B, int32_t K,
                                   const mv_moe_shape* shape, const mv_moe_weights* layers, int32_t n_layers,
                                   const uint16_t* w_lm, int32_t V, int32_t* accepted, int32_t* next_token,
                                   int32_t* emitted, int32_t* argmax, void* ws, size_t ws_bytes) {
  MV_TRY(check_shape(shape));
  if (B < 0 || K < 0 || K > 32 || n_layers < 0 || n_layers > kMaxLayers || V <= 0)
    return fail(MV_ERR_INVALID_ARG, "bad sizes B=%d K=%d (K <= 32) n_layers=%d (<= %d) V=%d", B, K, n_layers,
                kMaxLayers, V);
  if (V % 8) return fail(MV_ERR_UNSUPPORTED_SHAPE, "V=%d must be a multiple of 8", V);
  const int64_t T = int64_t(B) * (K + 1);
  MV_TRY(check_rows(T, shape));
  if (n_layers > 0 && !layers) return fail(MV_ERR_INVALID_ARG, "layers is NULL");
  for (int l = 0; l < n_layers; ++l) MV_TRY(check_weights(&layers[l], shape));
  MV_TRY(check_ptr(hidden, "hidden", B == 0));
  MV_TRY(check_ptr(drafts, "drafts", K == 0 || B == 0));
  MV_TRY(check_ptr(w_lm, "w_lm"));
  MV_TRY(check_ptr(accepted, "accepted", B == 0));
  MV_TRY(check_ptr(next_token, "next_token", B == 0));
  MV_TRY(check_ptr(emitted, "emitted", true));
  MV_TRY(check_ptr(argmax, "argmax", true));
  MV_TRY(check_ptr(ws, "workspace"));
  const size_t need = verify_step_workspace_size(B, K, shape, V);
  if (ws_bytes < need)
    return fail(MV_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, %zu needed", ws_bytes, need);
  return MV_OK;
}

static mv_status verify_step_impl(const uint16_t* hidden, const int32_t* drafts, int32_t B, int32_t K,
                                  const mv_moe_shape* shape, const mv_moe_weights* layers, int32_t n_layers,
                                  const uint16_t* w_lm, int32_t V, int32_t* accepted, int32_t* next_token,
                                  int32_t* emitted, int32_t* argmax, void* ws, size_t ws_bytes, mv_stream_t stream,
                                  const uint16_t** h_final) {
  MV_TRY(verify_step_check(hidden, drafts, B, K, shape, layers, n_layers, w_lm, V, accepted, next_token, emitted,
                           argmax, ws, ws_bytes));
  const int64_t T = int64_t(B) * (K + 1);
  if (B == 0) return MV_OK;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* err = static_cast<int*>(ws);
  Carve c{static_cast<char*>(ws) + kHeader};
  uint16_t* hbuf[2] = {c.take<uint16_t>(static_cast<size_t>(T) * shape->H),
                       c.take<uint16_t>(static_cast<size_t>(T) * shape->H)};
  const size_t tk = static_cast<size_t>(T) * shape->k;
  int32_t* idx_buf = c.take<int32_t>(tk * 2);
  float* tw_buf = c.take<float>(tk * 2);
  uint64_t* parts = c.take<uint64_t>(static_cast<size_t>(lm_parts_alloc(V)) * T);
  int* sched = c.take<int>(static_cast<size_t>(mv::kSchedInts) * (kMaxLayers + 1));
  const bool slabs = use_slabs(T, *shape);
  FfnWs fw = carve_ffn(c, T, *shape, slabs);
  uint16_t* xn_buf = c.take<uint16_t>(static_cast<size_t>(T) * shape->H);  // RMSNorm(h) * g of the current layer
  cudaError_t e0 = cudaMemsetAsync(sched, 0, kSchedBytes * (n_layers + 1), st);
  if (e0 != cudaSuccess) return cuda_fail(e0, "clearing the scheduling state");
  auto slab_counts = [&](int l) -> int32_t* {
    return slabs ? sched + static_cast<size_t>(l) * mv::kSchedInts + kSlabCountOff : nullptr;
  };
  auto slab_inv = [&](int l) -> int32_t* { return slabs ? ((l & 1) ? fw.inv_alt : fw.inv) : nullptr; };

  // Layer l's combine runs fused with layer l+1's routing (combine_route) when
  // the batch is decode-sized; otherwise as its own kernel before the router.
  // Decode-sized batches also group the routed rows by expert in that kernel
  // (slab layout) instead of a permute launch.
  // A layer with a norm gain (the pre-RMSNorm variant) routes and runs its
  // experts on xn_buf = bf16(RMSNorm(h) * g), written by the routing kernel
  // (or by the RMSNorm kernel when the routing is not fused), and keeps the
  // residual h.
  const bool fused = mv::combine_route_supported(static_cast<int>(T), shape->H, shape->E);
  const uint16_t* h = hidden;
  auto rmsnorm = [&](const uint16_t* src, const uint16_t* g) -> mv_status {
    cudaError_t e = run_kernel(KIND_RMSNORM, st, [&] {
      return mv::launch_rmsnorm(src, static_cast<int>(T), shape->H, g, xn_buf, st);
    });
    return e == cudaSuccess ? MV_OK : cuda_fail(e, "rmsnorm launch");
  };
  if (n_layers > 0 && fused) {
    cudaError_t e = run_kernel(KIND_ROUTER, st, [&] {
      mv::CombineRouteArgs a{};
      a.x = h;
      a.T = static_cast<int>(T);
      a.H = shape->H;
      a.E = shape->E;
      a.k = shape->k;
      a.wr = layers[0].w_router;
      a.bias = layers[0].router_bias;
      a.idx = idx_buf;
      a.w = tw_buf;
      a.err = err;
      a.timeout_ns = timeout_ns();
      a.pf = moe_first_wave(*shape, layers[0], kPrefetchBudget, T);
      a.slab_counts = slab_counts(0);
      a.inv_out = slab_inv(0);
      a.ent_out = fw.ent;
      a.x_slab = fw.x_perm;
      a.slab_rows = static_cast<int>(T);
      a.norm_gain = layers[0].norm_gain;
      a.xn_out = xn_buf;
      return mv::launch_combine_route(a, st);
    });
    if (e != cudaSuccess) return cuda_fail(e, "router_topk launch");
  } else if (n_layers > 0) {
    if (layers[0].norm_gain) MV_TRY(rmsnorm(h, layers[0].norm_gain));
    MV_TRY(route_impl(layers[0].norm_gain ? xn_buf : h, static_cast<int>(T), *shape, layers[0].w_router,
                      layers[0].router_bias, idx_buf, tw_buf, err, st,
                      moe_first_wave(*shape, layers[0], kPrefetchBudget)));
  }
  for (int l = 0; l < n_layers; ++l) {
    const mv_moe_weights& w = layers[l];
    int32_t* idx = idx_buf + (l & 1) * tk;
    float* tw = tw_buf + (l & 1) * tk;
    uint16_t* next = hbuf[l & 1];
    const bool last = (l + 1 == n_layers);
    const uint16_t* x_in = w.norm_gain ? xn_buf : h;
    MV_TRY(ffn_forward_impl(x_in, static_cast<int>(T), *shape, w, idx, tw, h, next, fw, err,
                            sched + static_cast<size_t>(l) * mv::kSchedInts, st, last || !fused,
                            last ? lm_first_wave(w_lm, V, shape->H, kPrefetchBudget) : mv::L2Prefetch{},
                            slab_counts(l), slab_inv(l)));
    if (!last) {
      int32_t* idx_n = idx_buf + ((l + 1) & 1) * tk;
      float* tw_n = tw_buf + ((l + 1) & 1) * tk;
      const mv_moe_weights& wn = layers[l + 1];
      if (fused) {
        cudaError_t e = run_kernel(KIND_COMBINE_ROUTE, st, [&] {
          mv::CombineRouteArgs a{};
          a.x = h;
          a.y_perm = fw.y_perm;
          a.y_sh = shape->I_shared > 0 ? fw.y_sh : nullptr;
          a.inv = slabs ? slab_inv(l) : fw.inv;
          a.n_pos = static_cast<int>(fw.n_pos);
          a.w_prev = tw;
          a.k_prev = shape->k;
          a.out = next;
          a.T = static_cast<int>(T);
          a.H = shape->H;
          a.E = shape->E;
          a.k = shape->k;
          a.wr = wn.w_router;
          a.bias = wn.router_bias;
          a.idx = idx_n;
          a.w = tw_n;
          a.err = err;
          a.timeout_ns = timeout_ns();
          a.pf = moe_first_wave(*shape, wn, kPrefetchBudget, T);
          a.slab_counts = slab_counts(l + 1);
          a.inv_out = slab_inv(l + 1);
          a.ent_out = fw.ent;
          a.y_by_entry = slabs ? 1 : 0;
          a.x_slab = fw.x_perm;
          a.slab_rows = static_cast<int>(T);
          a.norm_gain = wn.norm_gain;
          a.xn_out = xn_buf;
          return mv::launch_combine_route(a, st);
        });
        if (e != cudaSuccess) return cuda_fail(e, "combine_route launch");
      } else {
        if (wn.norm_gain) MV_TRY(rmsnorm(next, wn.norm_gain));
        MV_TRY(route_impl(wn.norm_gain ? xn_buf : next, static_cast<int>(T), *shape, wn.w_router, wn.router_bias,
                          idx_n, tw_n, err, st));
      }
    }
    h = next;
  }
  if (h_final) *h_final = h;
  int used = 0;
  MV_TRY(lm_gemm_impl(h, static_cast<int>(T), shape->H, w_lm, V, parts, lm_parts_alloc(V), err,
                      sched + static_cast<size_t>(n_layers) * mv::kSchedInts, st, true, &used));
  cudaError_t e = run_kernel(KIND_ACCEPT, st, [&] {
    return mv::launch_accept_from_keys(parts, used, lm_parts_alloc(V), K > 0 ? drafts : nullptr, B, K, accepted,
                                       next_token, emitted, argmax, st);
  });
  return e == cudaSuccess ? MV_OK : cuda_fail(e, "greedy_accept launch");
}

mv_status verify_step(const uint16_t* hidden, const int32_t* drafts, int32_t B, int32_t K, const mv_moe_shape* shape,
                      const mv_moe_weights* layers, int32_t n_layers, const uint16_t* w_lm, int32_t V,
                      int32_t* accepted, int32_t* next_token, int32_t* emitted, int32_t* argmax, void* ws,
                      size_t ws_bytes, mv_stream_t stream) {
  return verify_step_impl(hidden, drafts, B, K, shape, layers, n_layers, w_lm, V, accepted, next_token, emitted,
                          argmax, ws, ws_bytes, stream, nullptr);
}

// ---------------------------------------------------------------------------
// FastMTP draft block
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

constexpr float kDraftRmsEps = 1e-6f;

struct DraftWs {
  int* sched;       // 2 GEMM launches per step
  uint16_t* u;      // [B][2H] block input
  uint16_t* z;      // [B][H] projection
  uint16_t* a;      // [B][I_d] SwiGLU activation
  uint16_t* h[2];   // step outputs (ping-pong) when the caller keeps none
  uint64_t* keys;   // [B][lm_parts_alloc(V)] LM argmax keys
};

DraftWs carve_draft(Carve& c, int64_t B, int K, int H, int Id, int V) {
  DraftWs w;
  w.sched = c.take<int>(static_cast<size_t>(mv::kSchedInts) * 2 * std::max(K, 1));
  w.u = c.take<uint16_t>(static_cast<size_t>(B) * 2 * H);
  w.z = c.take<uint16_t>(static_cast<size_t>(B) * H);
  w.a = c.take<uint16_t>(static_cast<size_t>(B) * Id);
  w.h[0] = c.take<uint16_t>(static_cast<size_t>(B) * H);
  w.h[1] = c.take<uint16_t>(static_cast<size_t>(B) * H);
  w.keys = c.take<uint64_t>(static_cast<size_t>(lm_parts_alloc(V)) * B);
  return w;
}

mv_status check_draft(const mv_draft_weights* d, int H) {
  if (!d) return fail(MV_ERR_INVALID_ARG, "draft weights are NULL");
  if (d->I_d <= 0 || d->I_d % 64) return fail(MV_ERR_UNSUPPORTED_SHAPE, "I_d=%d must be a positive multiple of 64", d->I_d);
  if (H % 64) return fail(MV_ERR_UNSUPPORTED_SHAPE, "H=%d must be a multiple of 64", H);
  MV_TRY(check_ptr(d->w_emb, "draft.w_emb"));
  MV_TRY(check_ptr(d->g_hidden, "draft.g_hidden"));
  MV_TRY(check_ptr(d->g_embed, "draft.g_embed"));
  MV_TRY(check_ptr(d->w_proj, "draft.w_proj"));
  MV_TRY(check_ptr(d->w_gate, "draft.w_gate"));
  MV_TRY(check_ptr(d->w_up, "draft.w_up"));
  MV_TRY(check_ptr(d->w_down, "draft.w_down"));
  return MV_OK;
}

// One launch of the draft block's dense part for B rows, three dependent sets
// of swap-AB tiles: z = bf16(u . W_proj^T); a = bf16(silu(z Wg^T) * (z Wu^T));
// h' = bf16(z + a . Wd^T).  Each later set waits for the earlier one through
// the launch's completion counters.
mv_status draft_gemm_impl(const uint16_t* u, int B, int H, const mv_draft_weights& d, uint16_t* z, uint16_t* a,
                          uint16_t* hout, int* err, int* sched, cudaStream_t st) {
  mv::GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.err = err;
  p.sched = sched;
  p.timeout_ns = timeout_ns();
  const int Id = d.I_d, BN = 32, bbox = mv::kDecodeBBox;
  const int64_t ntile = (B + BN - 1) / BN;
  mv::GemmSet& P = p.set[0];
  P.mode = mv::MODE_KPAIR;
  P.epi = mv::EPI_STORE_BF16;
  P.m_tile = 128;
  P.dep_set = -1;
  MV_TRY(tmap3(&P.a0, d.w_proj, H, 2 * static_cast<uint64_t>(H), 128));
  P.a1 = P.a0;
  MV_TRY(tmap3(&P.b, u, B, 2 * static_cast<uint64_t>(H), bbox));
  P.out = z;
  P.ld_out = H;
  P.K = 2 * H;
  P.M = H;
  P.groups = 1;
  P.static_rows = B;
  P.signal = 1;
  mv::GemmSet& G = p.set[1];
  G.mode = mv::MODE_GATEUP;
  G.epi = mv::EPI_SWIGLU;
  G.m_tile = 128;
  G.dep_set = 0;
  MV_TRY(tmap3(&G.a0, d.w_gate, Id, H, 128));
  MV_TRY(tmap3(&G.a1, d.w_up, Id, H, 128));
  MV_TRY(tmap3(&G.b, z, B, H, bbox));
  G.out = a;
  G.ld_out = Id;
  G.K = H;
  G.M = Id;
  G.groups = 1;
  G.static_rows = B;
  G.signal = 1;
  mv::GemmSet& D = p.set[2];
  D.mode = mv::MODE_KPAIR;
  D.epi = mv::EPI_STORE_BF16;
  D.m_tile = 128;
  D.dep_set = 1;
  MV_TRY(tmap3(&D.a0, d.w_down, H, Id, 128));
  D.a1 = D.a0;
  MV_TRY(tmap3(&D.b, a, B, Id, bbox));
  D.out = hout;
  D.res = z;
  D.ld_out = H;
  D.K = Id;
  D.M = H;
  D.groups = 1;
  D.static_rows = B;
  p.nsets = 3;
  const int64_t units = ntile * ((H + 127) / 128 * 2 + (Id + 127) / 128);
  cudaError_t e = run_kernel(KIND_DRAFT_GEMM, st, [&] {
    return mv::launch_gemm(mv::GEMM_MOE_DECODE, p, gemm_grid(units), st);
  });
  return e == cudaSuccess ? MV_OK : cuda_fail(e, "draft_block_gemm launch");
}

// K recursive draft-block steps from h (row b*row_stride + acc[b] of h_src)
// and t0; drafts[b][j-1] is step j's greedy choice.
mv_status draft_impl(const uint16_t* h_src, int row_stride, const int32_t* acc, const int32_t* t0, int B, int K,
                     int H, const mv_draft_weights& d, const uint16_t* w_lm, int V, int32_t* drafts,
                     uint16_t* h_steps, const DraftWs& w, int* err, cudaStream_t st) {
  if (B == 0 || K == 0) return MV_OK;
  cudaError_t e = cudaMemsetAsync(w.sched, 0, kSchedBytes * 2 * K, st);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the draft scheduling state");
  mv::MtpStepArgs a{};
  a.t0 = t0;
  a.drafts = drafts;
  a.K = K;
  a.w_emb = d.w_emb;
  a.V = V;
  a.g_h = d.g_hidden;
  a.g_e = d.g_embed;
  a.H = H;
  a.eps = kDraftRmsEps;
  a.err = err;
  a.B = B;
  a.j = 0;
  a.h_src = h_src;
  a.row_stride = row_stride;
  a.acc = acc;
  a.u = w.u;
  e = run_kernel(KIND_DRAFT_STEP, st, [&] { return mv::launch_mtp_step(a, st); });
  if (e != cudaSuccess) return cuda_fail(e, "draft_step launch");
  const int ld = lm_parts_alloc(V);
  for (int j = 1; j <= K; ++j) {
    uint16_t* hout = h_steps ? h_steps + static_cast<size_t>(j - 1) * B * H : w.h[(j - 1) & 1];
    int* sched = w.sched + static_cast<size_t>(2 * (j - 1)) * mv::kSchedInts;
    MV_TRY(draft_gemm_impl(w.u, B, H, d, w.z, w.a, hout, err, sched, st));
    int used = 0;
    MV_TRY(lm_gemm_impl(hout, B, H, w_lm, V, w.keys, ld, err, sched + mv::kSchedInts, st, true, &used,
                        KIND_DRAFT_LM));
    a.keys = w.keys;
    a.nparts = used;
    a.ld = ld;
    a.j = j;
    a.h_src = hout;
    a.row_stride = 1;
    a.acc = nullptr;
    a.u = (j < K) ? w.u : nullptr;
    e = run_kernel(KIND_DRAFT_STEP, st, [&] { return mv::launch_mtp_step(a, st); });
    if (e != cudaSuccess) return cuda_fail(e, "draft_step launch");
  }
  return MV_OK;
}

}  // namespace

extern "C" {

size_t fastmtp_draft_workspace_size(int32_t B, int32_t K, int32_t H, int32_t I_d, int32_t V) {
  if (B < 0 || K < 0 || H <= 0 || I_d <= 0 || V <= 0) return 0;
  Carve c{nullptr};
  carve_draft(c, B, K, H, I_d, V);
  return kHeader + c.off + 1024;
}

mv_status fastmtp_draft(const uint16_t* h0, const int32_t* t0, int32_t B, int32_t K, int32_t H,
                        const mv_draft_weights* draft, const uint16_t* w_lm, int32_t V, int32_t* drafts,
                        uint16_t* h_steps, void* ws, size_t ws_bytes, mv_stream_t stream) {
  if (B < 0 || K < 0 || K > 32 || H <= 0 || V <= 0)
    return fail(MV_ERR_INVALID_ARG, "bad sizes B=%d K=%d (K <= 32) H=%d V=%d", B, K, H, V);
  MV_TRY(check_draft(draft, H));
  if (V % 8) return fail(MV_ERR_UNSUPPORTED_SHAPE, "V=%d must be a multiple of 8", V);
  const bool none = (B == 0 || K == 0);
  MV_TRY(check_ptr(h0, "h0", none));
  MV_TRY(check_ptr(t0, "t0", none));
  MV_TRY(check_ptr(w_lm, "w_lm"));
  MV_TRY(check_ptr(drafts, "drafts", none));
  MV_TRY(check_ptr(h_steps, "h_steps", true));
  MV_TRY(check_ptr(ws, "workspace"));
  const size_t need = fastmtp_draft_workspace_size(B, K, H, draft->I_d, V);
  if (ws_bytes < need) return fail(MV_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, %zu needed", ws_bytes, need);
  if (none) return MV_OK;
  Carve c{static_cast<char*>(ws) + kHeader};
  const DraftWs w = carve_draft(c, B, K, H, draft->I_d, V);
  return draft_impl(h0, 1, nullptr, t0, B, K, H, *draft, w_lm, V, drafts, h_steps, w, static_cast<int*>(ws),
                    reinterpret_cast<cudaStream_t>(stream));
}

size_t speculative_step_workspace_size(int32_t B, int32_t K, const mv_moe_shape* shape, int32_t I_d, int32_t V) {
  if (!shape) return 0;
  const size_t v = verify_step_workspace_size(B, K, shape, V);
  const size_t d = fastmtp_draft_workspace_size(B, K, shape->H, I_d, V);
  if (!v || !d) return 0;
  return align_up(v, 1024) + d;
}

mv_status speculative_step(const uint16_t* hidden, const int32_t* drafts, int32_t B, int32_t K,
                           const mv_moe_shape* shape, const mv_moe_weights* layers, int32_t n_layers,
                           const uint16_t* w_lm, int32_t V, const mv_draft_weights* draft, int32_t* accepted,
                           int32_t* next_token, int32_t* emitted, int32_t* argmax, int32_t* next_drafts, void* ws,
                           size_t ws_bytes, mv_stream_t stream) {
  MV_TRY(check_shape(shape));
  MV_TRY(check_draft(draft, shape->H));
  MV_TRY(check_ptr(next_drafts, "next_drafts", K == 0 || B == 0));
  if (next_drafts && drafts && next_drafts == drafts) return fail(MV_ERR_INVALID_ARG, "next_drafts may not alias drafts");
  const size_t need = speculative_step_workspace_size(B, K, shape, draft->I_d, V);
  if (!need) return fail(MV_ERR_INVALID_ARG, "bad sizes B=%d K=%d V=%d", B, K, V);
  MV_TRY(check_ptr(ws, "workspace"));
  if (ws_bytes < need) return fail(MV_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, %zu needed", ws_bytes, need);
  const size_t vbytes = align_up(verify_step_workspace_size(B, K, shape, V), 1024);
  const uint16_t* h_last = nullptr;
  MV_TRY(verify_step_impl(hidden, drafts, B, K, shape, layers, n_layers, w_lm, V, accepted, next_token, emitted,
                          argmax, ws, vbytes, stream, &h_last));
  if (B == 0 || K == 0) return MV_OK;
  Carve c{static_cast<char*>(ws) + vbytes + kHeader};
  const DraftWs w = carve_draft(c, B, K, shape->H, draft->I_d, V);
  return draft_impl(h_last, K + 1, accepted, next_token, B, K, shape->H, *draft, w_lm, V, next_drafts, nullptr, w,
                    static_cast<int*>(ws), reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

struct mv_verify_graph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  int32_t kernels = 0;
};

namespace {

void free_graph(mv_verify_graph* g) {
  if (!g) return;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  delete g;
}

}  // namespace

extern "C" {

mv_status verify_graph_create(const uint16_t* hidden, const int32_t* drafts, int32_t B, int32_t K,
                              const mv_moe_shape* shape, const mv_moe_weights* layers, int32_t n_layers,
                              const uint16_t* w_lm, int32_t V, int32_t* accepted, int32_t* next_token,
                              int32_t* emitted, int32_t* argmax, void* ws, size_t ws_bytes,
                              mv_verify_graph** graph) {
  if (!graph) return fail(MV_ERR_INVALID_ARG, "graph out-parameter is NULL");
  *graph = nullptr;
  if (g_prof_on.load()) return fail(MV_ERR_INVALID_ARG, "profiling is on: its events cannot be recorded into a graph");
  MV_TRY(verify_step_check(hidden, drafts, B, K, shape, layers, n_layers, w_lm, V, accepted, next_token, emitted,
                           argmax, ws, ws_bytes));
  cudaStream_t cs = nullptr;
  cudaError_t e = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking);
  if (e != cudaSuccess) return cuda_fail(e, "creating the recording stream");
  // Relaxed mode: the one-time host set-up a first call may do (kernel
  // attributes, tensor-map encoding) is not a stream operation and stays
  // legal while this thread records.
  e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed);
  if (e != cudaSuccess) {
    cudaStreamDestroy(cs);
    return cuda_fail(e, "beginning the graph recording");
  }
  t_recording = true;
  const mv_status st = verify_step(hidden, drafts, B, K, shape, layers, n_layers, w_lm, V, accepted, next_token,
                                   emitted, argmax, ws, ws_bytes, reinterpret_cast<mv_stream_t>(cs));
  t_recording = false;
  const std::string step_msg = g_last_error;
  mv_verify_graph* g = new mv_verify_graph();
  e = cudaStreamEndCapture(cs, &g->graph);
  cudaStreamDestroy(cs);
  if (st != MV_OK) {
    free_graph(g);
    g_last_error = step_msg;
    return st;
  }
  if (e != cudaSuccess) {
    free_graph(g);
    return cuda_fail(e, "ending the graph recording");
  }
  size_t n = 0;
  e = cudaGraphGetNodes(g->graph, nullptr, &n);
  std::vector<cudaGraphNode_t> nodes(n);
  if (e == cudaSuccess && n) e = cudaGraphGetNodes(g->graph, nodes.data(), &n);
  if (e != cudaSuccess) {
    free_graph(g);
    return cuda_fail(e, "listing the graph's nodes");
  }
  for (cudaGraphNode_t node : nodes) {
    cudaGraphNodeType t{};
    if (cudaGraphNodeGetType(node, &t) == cudaSuccess && t == cudaGraphNodeTypeKernel) ++g->kernels;
  }
  e = cudaGraphInstantiateWithFlags(&g->exec, g->graph, 0);
  if (e != cudaSuccess) {
    g->exec = nullptr;
    free_graph(g);
    return cuda_fail(e, "instantiating the graph");
  }
  *graph = g;
  return MV_OK;
}

mv_status verify_graph_launch(mv_verify_graph* graph, mv_stream_t stream) {
  if (!graph || !graph->exec) return fail(MV_ERR_INVALID_ARG, "graph is NULL");
  cudaError_t e = cudaGraphLaunch(graph->exec, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "graph launch");
  g_launches.fetch_add(static_cast<uint64_t>(graph->kernels), std::memory_order_relaxed);
  return MV_OK;
}

int32_t verify_graph_kernels(const mv_verify_graph* graph) { return graph ? graph->kernels : -1; }

mv_status verify_graph_destroy(mv_verify_graph* graph) {
  free_graph(graph);
  return MV_OK;
}

size_t decode_attention_workspace_size(int32_t B, int32_t K, int32_t n_heads, int32_t max_ctx) {
  if (B < 0 || K < 0 || n_heads <= 0 || max_ctx < 0 || mv::attention_nq(K) == 0) return 0;
  Carve c{nullptr};
  c.off = kHeader;
  carve_attn(c, B, n_heads, attn_plan(B, K, n_heads, max_ctx));
  return c.off;
}

mv_status decode_attention(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                           const int32_t* ctx_len, int32_t B, int32_t K, int32_t n_heads, int32_t head_dim,
                           int32_t L_max, int32_t max_ctx, uint16_t* out, void* ws, size_t ws_bytes,
                           mv_stream_t stream) {
  if (B < 0 || K < 0 || n_heads <= 0 || L_max <= 0 || max_ctx < 0)
    return fail(MV_ERR_INVALID_ARG, "bad sizes B=%d K=%d n_heads=%d L_max=%d max_ctx=%d", B, K, n_heads, L_max,
                max_ctx);
  if (head_dim != kAttnHeadDim) return fail(MV_ERR_UNSUPPORTED_SHAPE, "head_dim=%d (only 128)", head_dim);
  if (mv::attention_nq(K) == 0) return fail(MV_ERR_UNSUPPORTED_SHAPE, "K=%d (at most 7 drafts)", K);
  if (n_heads > kAttnMaxHeads) return fail(MV_ERR_UNSUPPORTED_SHAPE, "n_heads=%d (at most %d)", n_heads, kAttnMaxHeads);
  if (static_cast<int64_t>(max_ctx) + K + 1 > L_max)
    return fail(MV_ERR_INVALID_ARG, "max_ctx + K + 1 = %lld exceeds the cache length L_max=%d",
                static_cast<long long>(max_ctx) + K + 1, L_max);
  if (static_cast<int64_t>(B) * n_heads * L_max >= (1LL << 31))
    return fail(MV_ERR_UNSUPPORTED_SHAPE, "B * n_heads * L_max must stay below 2^31 cache rows");
  MV_TRY(check_ptr(q, "q", B == 0));
  MV_TRY(check_ptr(k_cache, "k_cache"));
  MV_TRY(check_ptr(v_cache, "v_cache"));
  MV_TRY(check_ptr(ctx_len, "ctx_len", B == 0));
  MV_TRY(check_ptr(out, "out", B == 0));
  MV_TRY(check_ptr(ws, "workspace"));
  const size_t need = decode_attention_workspace_size(B, K, n_heads, max_ctx);
  if (ws_bytes < need) return fail(MV_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, %zu needed", ws_bytes, need);
  if (B == 0) return MV_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const AttnPlan pl = attn_plan(B, K, n_heads, max_ctx);
  Carve c{static_cast<char*>(ws) + kHeader};
  const AttnWs aw = carve_attn(c, B, n_heads, pl);
  mv::AttnParams p;
  std::memset(&p, 0, sizeof(p));
  const uint64_t rows = static_cast<uint64_t>(B) * n_heads * L_max;
  MV_TRY(tmap3(&p.k_map, k_cache, rows, kAttnHeadDim, 64));
  MV_TRY(tmap3(&p.v_map, v_cache, rows, kAttnHeadDim, 64));
  p.q = q;
  p.ctx_len = ctx_len;
  p.out = out;
  p.part_o = aw.part_o;
  p.part_ml = aw.part_ml;
  p.counters = aw.counters;
  p.err = static_cast<int*>(ws);
  p.K = K;
  p.n_heads = n_heads;
  p.L_max = L_max;
  p.max_ctx = max_ctx;
  p.split_len = pl.split_len;
  p.n_split = pl.n_split;
  p.scale = 1.0f / sqrtf(static_cast<float>(kAttnHeadDim));
  p.timeout_ns = timeout_ns();
  cudaError_t e = cudaMemsetAsync(aw.counters, 0, static_cast<size_t>(B) * n_heads * sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the attention split counters");
  e = run_kernel(KIND_ATTENTION, st, [&] { return mv::launch_decode_attention(p, B, st); });
  return e == cudaSuccess ? MV_OK : cuda_fail(e, "decode_attention launch");
}

mv_status mv_workspace_init(void* ws, size_t ws_bytes, mv_stream_t stream) {
  MV_TRY(check_ptr(ws, "workspace"));
  if (ws_bytes < kHeader) return fail(MV_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes is below the header", ws_bytes);
  cudaError_t e = cudaMemsetAsync(ws, 0, kHeader, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MV_OK : cuda_fail(e, "clearing the workspace header");
}

mv_status mv_sync_status(void* ws, mv_stream_t stream) {
  MV_TRY(check_ptr(ws, "workspace"));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int word = 0;
  e = cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (word != 0) {
    e = cudaMemset(ws, 0, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    if (word & mv::kErrTimeout) return fail(MV_ERR_TIMEOUT, "a device-side wait ran out (error word 0x%x)", word);
    return fail(MV_ERR_INTERNAL, "a device-side check failed (error word 0x%x)", word);
  }
  return MV_OK;
}

}  // extern "C"

// ===========================================================================
// lm_head_argmax_noalloc: the LM-head greedy choice for callers that must not
// allocate device memory.  Its scratch (error word, work-claim counter and the
// per-token partial argmax keys) is one file-scope device array instead of a
// caller workspace.
// ===========================================================================
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB, held by every GPU that loads the library
constexpr size_t kNoAllocErrBytes = 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoAllocAddr {
  void* ptr = nullptr;
  unsigned long long ctx_id = 0;  // the CUDA context the address belongs to
};
NoAllocAddr g_noalloc_addr[kNoAllocMaxDevices];

// Unique id of the calling thread's current CUDA context (driver entry points
// through the runtime, which the library links statically); 0 if unknown.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array on the current device.  The array's name
// is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, with the device current, once per device and context:
// the first call on a device does it (this may load the library's device
// code), later calls reuse it, and a call after the device's context was
// destroyed and re-created (cudaDeviceReset) looks it up again.
mv_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(MV_ERR_UNSUPPORTED_SHAPE, "device %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoAllocAddr& a = g_noalloc_addr[dev];
  const unsigned long long id = current_context_id();
  if (!a.ptr || id == 0 || id != a.ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress of the no-alloc scratch");
    a.ptr = p;
    a.ctx_id = current_context_id();  // the lookup made the device's primary context current
  }
  *out = a.ptr;
  return MV_OK;
}

// Reduces each token's partial keys to its argmax; writes -1 for every token
// if a bounded device-side wait of the GEMM ran out (the callers of this path
// have no workspace through which to read the error word).
__global__ void __launch_bounds__(128) noalloc_finalize_kernel(const uint64_t* __restrict__ keys, int nparts,
                                                               int ld, int T, int32_t* __restrict__ argmax,
                                                               const int* __restrict__ err) {
  __shared__ uint64_t red[4];
  mv::pdl_trigger();
  mv::pdl_wait();
  const int t = blockIdx.x;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const uint64_t* row = keys + static_cast<size_t>(t) * ld;  // the first nparts keys of the row are written
  uint64_t best = 0;
  for (int p = threadIdx.x; p < nparts; p += 128) {
    const uint64_t v = row[p];
    best = v > best ? v : best;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t v = __shfl_xor_sync(0xffffffffu, best, o);
    best = v > best ? v : best;
  }
  if (lane == 0) red[wid] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t b = red[0];
    for (int i = 1; i < 4; ++i) b = red[i] > b ? red[i] : b;
    argmax[t] = (*err != 0) ? -1 : static_cast<int32_t>(mv::argmax_key_index(b));
  }
}

}  // namespace

extern "C" MV_API mv_status lm_head_argmax_noalloc(const uint16_t* h, int32_t T, int32_t H, const uint16_t* w_lm,
                                                   int32_t V, int32_t* argmax, mv_stream_t stream) {
  if (T < 0 || H <= 0 || V <= 0) return fail(MV_ERR_INVALID_ARG, "bad sizes T=%d H=%d V=%d", T, H, V);
  if (H % 64 || V % 8 || H > 16384)
    return fail(MV_ERR_UNSUPPORTED_SHAPE, "H must be a multiple of 64 and V of 8 (H=%d V=%d)", H, V);
  MV_TRY(check_ptr(h, "h"));
  MV_TRY(check_ptr(w_lm, "w_lm"));
  MV_TRY(check_ptr(argmax, "argmax"));
  const size_t keys_bytes = static_cast<size_t>(lm_parts(V)) * static_cast<size_t>(T) * 8;
  const size_t need = kNoAllocErrBytes + kSchedBytes + keys_bytes;
  if (need > kNoAllocScratchBytes)
    return fail(MV_ERR_UNSUPPORTED_SHAPE,
                "T=%d rows x V=%d needs %zu bytes of scratch; the built-in no-alloc scratch holds %zu "
                "(use lm_head_argmax with a workspace)",
                T, V, need, kNoAllocScratchBytes);
  if (T == 0) return MV_OK;
  void* base = nullptr;
  MV_TRY(noalloc_scratch(&base));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* err = static_cast<int*>(base);
  int* sched = reinterpret_cast<int*>(static_cast<char*>(base) + kNoAllocErrBytes);
  uint64_t* parts = reinterpret_cast<uint64_t*>(static_cast<char*>(base) + kNoAllocErrBytes + kSchedBytes);
  cudaError_t e = cudaMemsetAsync(base, 0, kNoAllocErrBytes + kSchedBytes, st);  // error word and claim counter
  if (e != cudaSuccess) return cuda_fail(e, "clearing the no-alloc scratch");
  int used = 0;
  MV_TRY(lm_gemm_impl(h, T, H, w_lm, V, parts, lm_parts(V), err, sched, st, false, &used));
  e = run_kernel(KIND_LM_FINALIZE, st, [&] {
    return mv::launch_pdl(noalloc_finalize_kernel, dim3(T), dim3(128), 0, st, static_cast<const uint64_t*>(parts),
                          used, lm_parts(V), static_cast<int>(T), argmax, static_cast<const int*>(err));
  });
  return e == cudaSuccess ? MV_OK : cuda_fail(e, "no-alloc argmax finalize launch");
}
