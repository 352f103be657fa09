// CUDA-core kernels of the verify step: router top-k, grouping by expert,
// weighted combine, LM-head argmax finalisation and greedy acceptance.
// Methods follow the jina-ocr-v1 model card (jina.ai/models/jina-ocr-v1):
// architecture paragraph (64 routed + 2 shared experts, top-6 routing,
// 129,280-token vocabulary), decoding-speed paragraph and introduction
// (K drafts verified greedily, lossless).

#include "mv_device.cuh"
#include "mv_internal.h"

namespace mv {

namespace {

constexpr int kPermuteStage = 8192;  // routing entries the grouping kernel stages in shared memory

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint64_t pack2f(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 unpack2f(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return make_float2(lo, hi);
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// The fp32 pair of one bf16x2 word: (element 2i, element 2i+1).
__device__ __forceinline__ uint64_t bf16x2_pair(uint32_t w) {
  return pack2f(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// acc += x . w over 8 bf16 elements as two fp32 partial sums, element 2i
// into the low half and 2i+1 into the high half (one packed FMA per pair).
__device__ __forceinline__ uint64_t dot8_pairs(const uint4& x, const uint4& w, uint64_t acc) {
  acc = ffma2(bf16x2_pair(x.x), bf16x2_pair(w.x), acc);
  acc = ffma2(bf16x2_pair(x.y), bf16x2_pair(w.y), acc);
  acc = ffma2(bf16x2_pair(x.z), bf16x2_pair(w.z), acc);
  return ffma2(bf16x2_pair(x.w), bf16x2_pair(w.w), acc);
}

// This CTA's share of the L2 prefetch ranges: the concatenated ranges are cut
// into gridDim.x equal slices (16-byte multiples), issued as 64 KB bulk
// prefetches by one thread.  Fire and forget: nothing waits for them.
__device__ __forceinline__ void prefetch_share(const L2Prefetch& pf) {
  if (threadIdx.x != 0 || pf.n <= 0) return;
  uint64_t total = 0;
  for (int i = 0; i < pf.n; ++i) total += pf.bytes[i];
  const uint64_t per = ((total + gridDim.x - 1) / gridDim.x + 15) & ~uint64_t(15);
  uint64_t lo = per * blockIdx.x, hi = lo + per;
  if (hi > total) hi = total;
  uint64_t base = 0;
  for (int i = 0; i < pf.n && lo < hi; ++i) {
    const uint64_t r0 = base, r1 = base + pf.bytes[i];
    base = r1;
    if (hi <= r0 || lo >= r1) continue;
    uint64_t a = (lo > r0 ? lo : r0) - r0, b = (hi < r1 ? hi : r1) - r0;
    const uint8_t* p = static_cast<const uint8_t*>(pf.ptr[i]);
    while (a < b) {
      const uint32_t sz = static_cast<uint32_t>(((b - a) < 65536 ? (b - a) : 65536) & ~uint64_t(15));
      if (sz == 0) break;
      prefetch_l2_bulk(p + a, sz);
      a += sz;
    }
  }
}

// Order key of a logit: larger logits give larger keys, -0 and +0 the same
// key, and NaN the smallest key of all (below -inf), so that a NaN is only
// ever selected when a row has fewer than k numbers.
__device__ __forceinline__ uint32_t logit_key(float v) {
  uint32_t u = __float_as_uint(v);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;  // NaN
  if ((u << 1) == 0u) u = 0u;                       // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k of `nrows` rows of E logits (shared memory, row r at ls + r * E) by
// the whole block; every thread must call it, as it synchronises the block.
// Selection by rank: the rank of an element is the number of elements of its
// row that come before it in the order "larger logit first, equal logits ->
// lower expert id first" (NaN last), and the element of rank j < k takes
// slot j, so the slots are in descending logit order.  Eight consecutive
// threads share one element, each comparing it with an eighth of the row,
// and add their counts with shuffles (topk_rank_block, ending with a block
// barrier).  Then a warp writes each row's slots (topk_weights_rows): ids,
// and the renormalised softmax weights exp(l_j - l_0) / sum_{i<k}
// exp(l_i - l_0), the sum taken in slot order.  slot_s holds 8 entries per
// row (k <= 8) and keeps the selected ids for the caller.  topk_rows_block
// does both with every warp of the block.
__device__ void topk_rank_block(const float* ls, int E, int k, int nrows, int32_t* slot_s) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int chunk = (E + 7) >> 3;
  const int items = nrows * E * 8;
  for (int base = 0; base < items; base += blockDim.x) {  // uniform trip count: shuffles see full warps
    const int it = base + tid;
    const int q = it >> 3, sub = it & 7;
    int cnt = 0, e = 0;
    const float* lr = ls;
    if (it < items) {
      const int r = q / E;
      e = q - r * E;
      lr = ls + r * E;
      const uint32_t ke = logit_key(lr[e]);
      const int i1 = min(E, (sub + 1) * chunk);
#pragma unroll 8
      for (int i = sub * chunk; i < i1; ++i) {
        const uint32_t ki = logit_key(lr[i]);
        cnt += (ki > ke || (ki == ke && i < e)) ? 1 : 0;
      }
    }
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 1);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 2);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, 4);
    if (it < items && sub == 0 && cnt < k) slot_s[(q / E) * 8 + cnt] = e;
  }
  __syncthreads();
}

// The slots' renormalised softmax weights, after topk_rank_block: warp
// w0 + i handles rows i, i + nw, ... (lane j computes slot j's exponential;
// the sum adds them in slot order); whole warps call it.
__device__ void topk_weights_rows(const float* ls, int E, int k, int nrows, const int32_t* slot_s,
                                  int32_t* __restrict__ idx_out, float* __restrict__ w_out, int w0, int nw) {
  const int lane = threadIdx.x & 31;
  const int wi = (static_cast<int>(threadIdx.x) >> 5) - w0;
  if (wi < 0 || wi >= nw) return;  // warp-uniform
  for (int r = wi; r < nrows; r += nw) {  // whole warps: the shuffles see every lane
    const float* lr = ls + r * E;
    const int32_t* sl = slot_s + r * 8;
    const int e = lane < k ? sl[lane] : 0;
    const float mx = lr[sl[0]];
    const float ex = lane < k ? expf(lr[e] - mx) : 0.f;
    float s = 0.f;
#pragma unroll 8
    for (int j = 0; j < k; ++j) s += __shfl_sync(0xffffffffu, ex, j);
    if (lane < k) {
      idx_out[r * k + lane] = e;
      w_out[r * k + lane] = ex / s;
    }
  }
}

__device__ void topk_rows_block(const float* ls, int E, int k, int nrows, int32_t* slot_s,
                                int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
  topk_rank_block(ls, E, k, nrows, slot_s);
  topk_weights_rows(ls, E, k, nrows, slot_s, idx_out, w_out, 0, static_cast<int>(blockDim.x >> 5));
}

}  // namespace

// ---------------------------------------------------------------------------
// Router: logits = x . W_r^T (+ bias) in fp32, top-k on the logits (ties to
// the lower expert id, slots in descending order), weights =
// exp(l_j - l_max) / sum_selected exp(l - l_max), which equals the softmax
// over all E restricted to the kept experts and renormalised.
// Every CUDA-core router takes the dot products in the same order: lane L
// of a warp sums its 16-byte vectors L, L+32, ... as two fp32 partial sums
// (even and odd elements, one packed f32x2 FMA per element pair), adds the
// two, and the warp adds the lanes by an xor-shuffle tree.
// A CTA of 8 warps owns R rows: the rows sit in shared memory, warp w computes
// experts w, w+8, ... for all R rows (each router weight row is read once per
// CTA, 16-byte loads), then the block selects the top-k of its rows by rank.
// ---------------------------------------------------------------------------
template <int R>
__global__ void __launch_bounds__(256) router_topk_kernel(const uint16_t* __restrict__ x, int T,
                                                          int H, int E, int k,
                                                          const uint16_t* __restrict__ wr,
                                                          const float* __restrict__ bias,
                                                          int32_t* __restrict__ idx,
                                                          float* __restrict__ wout) {
  extern __shared__ __align__(128) uint8_t sm[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(sm);                        // [R][H]
  float* ls = reinterpret_cast<float*>(sm + static_cast<size_t>(R) * H * 2);  // [R][E]
  __shared__ int32_t slot_s[R * 8];
  pdl_trigger();
  pdl_wait();
  const int row0 = blockIdx.x * R;
  const int nrows = min(R, T - row0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hv = H / 8;  // 16-byte vectors per row

  for (int i = tid; i < R * hv; i += blockDim.x) {
    const int r = i / hv, c = i % hv;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < nrows) v = reinterpret_cast<const uint4*>(x + static_cast<size_t>(row0 + r) * H)[c];
    reinterpret_cast<uint4*>(xs + static_cast<size_t>(r) * H)[c] = v;
  }
  __syncthreads();

  for (int e = warp; e < E; e += 8) {
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    const uint4* we = reinterpret_cast<const uint4*>(wr + static_cast<size_t>(e) * H);
    uint64_t acc2[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc2[r] = 0ull;
    for (int c = lane; c < hv; c += 32) {
      const uint4 wv = __ldg(we + c);
#pragma unroll
      for (int r = 0; r < R; ++r) acc2[r] = dot8_pairs(reinterpret_cast<const uint4*>(xs + static_cast<size_t>(r) * H)[c], wv, acc2[r]);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float2 pr = unpack2f(acc2[r]);
      acc[r] = pr.x + pr.y;
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float v = acc[r];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) ls[r * E + e] = bias ? v + bias[e] : v;
    }
  }
  __syncthreads();

  topk_rows_block(ls, E, k, nrows, slot_s, idx + static_cast<size_t>(row0) * k, wout + static_cast<size_t>(row0) * k);
}

// Router with the whole router weight matrix staged in shared memory
// (E*H bf16, 160 KB at the model shape) by bulk asynchronous copies (16 KB
// each, one mbarrier), so a CTA pulls it with a handful of large requests;
// each CTA then loops over blocks of R rows.  Same arithmetic and selection as
// router_topk_kernel.  The wait for the copies is bounded: if it ever ran out
// the rows get expert id -1 (which the grouping and combine kernels report)
// and the sticky error bit is set when an error word is given.
template <int R>
__global__ void __launch_bounds__(256, 1) router_smem_kernel(const uint16_t* __restrict__ x, int T, int H, int E,
                                                             int k, const uint16_t* __restrict__ wr,
                                                             const float* __restrict__ bias,
                                                             int32_t* __restrict__ idx, float* __restrict__ wout,
                                                             int* err, uint64_t timeout_ns) {
  extern __shared__ __align__(128) uint8_t sm[];
  uint16_t* wsm = reinterpret_cast<uint16_t*>(sm);                            // [E][H]
  uint16_t* xs = wsm + static_cast<size_t>(E) * H;                           // [R][H]
  float* ls = reinterpret_cast<float*>(xs + static_cast<size_t>(R) * H);      // [R][E]
  __shared__ __align__(8) uint64_t bar;
  __shared__ int ok_s;
  __shared__ int32_t slot_s[R * 8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hv = H / 8;
  const uint32_t total = static_cast<uint32_t>(E) * H * 2;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(&bar, total);
    constexpr uint32_t kChunk = 16384;
    for (uint32_t off = 0; off < total; off += kChunk) {
      const uint32_t sz = min(kChunk, total - off);
      asm volatile(
          "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              smem_u32(sm + off)),
          "l"(reinterpret_cast<const uint8_t*>(wr) + off), "r"(sz), "r"(smem_u32(&bar))
          : "memory");
    }
  }
  pdl_trigger();
  pdl_wait();  // the rows to route come from the previous kernel
  const int nblocks = (T + R - 1) / R;
  bool first = true;
  for (int rb = blockIdx.x; rb < nblocks; rb += gridDim.x) {
    const int row0 = rb * R;
    const int nrows = min(R, T - row0);
    for (int i = tid; i < R * hv; i += blockDim.x) {
      const int r = i / hv, c = i % hv;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < nrows) v = reinterpret_cast<const uint4*>(x + static_cast<size_t>(row0 + r) * H)[c];
      reinterpret_cast<uint4*>(xs + static_cast<size_t>(r) * H)[c] = v;
    }
    if (first) {
      if (tid == 0) {
        int dummy = 0;
        ok_s = mbar_wait(&bar, 0, &dummy, err, globaltimer_ns() + timeout_ns) ? 1 : 0;
        // Whatever the outcome, the copies must land before this CTA may exit.
        if (!ok_s) mbar_wait(&bar, 0, &dummy, nullptr, globaltimer_ns() + kDrainNs);
      }
      first = false;
    }
    __syncthreads();
    if (!ok_s) {  // the weights never arrived: report instead of computing on garbage
      if (warp < nrows && lane < k) {
        idx[static_cast<size_t>(row0 + warp) * k + lane] = -1;
        wout[static_cast<size_t>(row0 + warp) * k + lane] = 0.f;
      }
      continue;
    }
    for (int e = warp; e < E; e += 8) {
      float acc[R];
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = 0.f;
      const uint4* we = reinterpret_cast<const uint4*>(wsm + static_cast<size_t>(e) * H);
      uint64_t acc2[R];
#pragma unroll
      for (int r = 0; r < R; ++r) acc2[r] = 0ull;
      for (int c = lane; c < hv; c += 32) {
        const uint4 wv = we[c];
#pragma unroll
        for (int r = 0; r < R; ++r)
          acc2[r] = dot8_pairs(reinterpret_cast<const uint4*>(xs + static_cast<size_t>(r) * H)[c], wv, acc2[r]);
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float2 pr = unpack2f(acc2[r]);
        acc[r] = pr.x + pr.y;
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float v = acc[r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) ls[r * E + e] = bias ? v + bias[e] : v;
      }
    }
    __syncthreads();
    topk_rows_block(ls, E, k, nrows, slot_s, idx + static_cast<size_t>(row0) * k,
                    wout + static_cast<size_t>(row0) * k);
    __syncthreads();
  }
}

template <int R>
static void launch_router_r(const uint16_t* x, int T, int H, int E, int k, const uint16_t* wr,
                            const float* bias, int32_t* idx, float* w, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(R) * H * 2 + static_cast<size_t>(R) * E * 4;
  launch_pdl(router_topk_kernel<R>, dim3((T + R - 1) / R), dim3(256), smem, s, x, T, H, E, k, wr, bias, idx, w);
}

template <int R>
static cudaError_t launch_router_smem(const uint16_t* x, int T, int H, int E, int k, const uint16_t* wr,
                                      const float* bias, int32_t* idx, float* w, int* err, uint64_t timeout_ns,
                                      cudaStream_t s, size_t smem) {
  static thread_local int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(router_smem_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         220 * 1024);
    if (e != cudaSuccess) return e;
    configured_dev = dev;
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int nblocks = (T + R - 1) / R;
  return launch_pdl(router_smem_kernel<R>, dim3(min(nblocks, sms)), dim3(256), smem, s, x, T, H, E, k, wr, bias, idx, w,
                    err, timeout_ns);
}

// Rows per block: 4 for decode-sized batches (more CTAs share the work), 8 for
// large ones.  The router weights go to shared memory when they fit (E*H*2 up
// to ~200 KB); otherwise the global-load kernel streams them.
cudaError_t launch_router(const uint16_t* x, int T, int H, int E, int k, const uint16_t* wr,
                          const float* bias, int32_t* idx, float* w, int* err, uint64_t timeout_ns,
                          cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const int R = (T <= 256) ? 2 : (T <= 1024) ? 4 : 8;
  const size_t smem_v2 = static_cast<size_t>(E) * H * 2 + static_cast<size_t>(R) * H * 2 + static_cast<size_t>(R) * E * 4;
  if (smem_v2 <= 200 * 1024) {
    if (R == 2) return launch_router_smem<2>(x, T, H, E, k, wr, bias, idx, w, err, timeout_ns, s, smem_v2);
    if (R == 4) return launch_router_smem<4>(x, T, H, E, k, wr, bias, idx, w, err, timeout_ns, s, smem_v2);
    return launch_router_smem<8>(x, T, H, E, k, wr, bias, idx, w, err, timeout_ns, s, smem_v2);
  }
  auto fits = [&](int r) { return static_cast<size_t>(r) * H * 2 + static_cast<size_t>(r) * E * 4 <= 48 * 1024; };
  int r = R;
  while (r > 1 && !fits(r)) r >>= 1;
  switch (r) {
    case 8: launch_router_r<8>(x, T, H, E, k, wr, bias, idx, w, s); break;
    case 4: launch_router_r<4>(x, T, H, E, k, wr, bias, idx, w, s); break;
    case 2: launch_router_r<2>(x, T, H, E, k, wr, bias, idx, w, s); break;
    default: launch_router_r<1>(x, T, H, E, k, wr, bias, idx, w, s); break;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Combine + route (decode-sized batches).  One CTA owns R token rows:
//  (1) with expert outputs given: h[r] = bf16(res[r] + sum_j w_j * y_j + y_sh)
//      for its rows (the combine of the layer that just ran; products and sums
//      rounded separately, in slot order, shared last), written to `out` and
//      kept in shared memory; without them, the rows of `x` are loaded as is;
//  (2) the router of the next layer on those rows: logits h[r] . W_r[e]
//      (+ bias) in fp32, warp w owning experts w, w+16, ... (NV 16-byte
//      vectors per lane per expert row).  With STAGE the whole router matrix
//      is copied into shared memory by bulk copies issued at the CTA's start,
//      before it waits for its predecessor (the weights depend on nothing),
//      so the copy overlaps that wait and the combine; otherwise the router
//      rows stream from L2 four experts at a time;
//  (3) top-k with renormalised softmax weights (topk_rows_block);
//  (4) with slab_counts: the grouping by expert of the next layer, done here
//      instead of by a separate permute launch.  Each routed entry claims the
//      next free row of its expert's slab (an atomic counter per expert) and
//      the CTA copies its rows there from shared memory.  A claim past the
//      slab's capacity (only possible for rows whose logits are all -inf or
//      NaN) is undone, reported as an internal error and its entry skipped.
// ---------------------------------------------------------------------------
template <int R, int NV, bool STAGE>
__global__ void __launch_bounds__(512) combine_route_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ y_perm, const float* __restrict__ y_sh,
    const int32_t* __restrict__ inv, const float* __restrict__ w_prev, int k_prev, int n_pos,
    uint16_t* __restrict__ out, int T, int H, int E, int k, const uint16_t* __restrict__ wr,
    const float* __restrict__ bias, int32_t* __restrict__ idx, float* __restrict__ wout, int* err,
    const L2Prefetch pf, int32_t* __restrict__ slab_counts, int32_t* __restrict__ inv_out,
    uint16_t* __restrict__ x_slab, int slab_rows, const uint16_t* __restrict__ norm_gain,
    uint16_t* __restrict__ xn_out, uint64_t timeout_ns, int32_t* __restrict__ ent_out, int y_by_entry) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ int32_t sel_s[R * 8];  // the experts each row selected, by slot
  __shared__ int32_t pos_s[R * 8];  // their slab rows (-1: skipped)
  __shared__ float nred[R][16];     // RMSNorm partial sums, one per warp
  __shared__ __align__(8) uint64_t wbar;  // STAGE: the router matrix has landed
  __shared__ int wok_s;
  const uint32_t wbytes = STAGE ? static_cast<uint32_t>(E) * H * 2 : 0u;
  const uint16_t* wsm = reinterpret_cast<const uint16_t*>(sm);           // STAGE: [E][H]
  uint16_t* hs = reinterpret_cast<uint16_t*>(sm + wbytes);                // [R][H]
  float* ls = reinterpret_cast<float*>(hs + static_cast<size_t>(R) * H);  // [R][E]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hv = H / 8;
  const int row0 = blockIdx.x * R;
  const int nrows = min(R, T - row0);
  pdl_trigger();
  if (STAGE) {
    if (row0 < T && tid == 0) {
      mbar_init(&wbar, 1);
      fence_barrier_init();
      mbar_arrive_expect_tx(&wbar, wbytes);
      constexpr uint32_t kChunk = 32768;
      for (uint32_t off = 0; off < wbytes; off += kChunk) {
        const uint32_t sz = min(kChunk, wbytes - off);
        asm volatile(
            "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                smem_u32(sm + off)),
            "l"(reinterpret_cast<const uint8_t*>(wr) + off), "r"(sz), "r"(smem_u32(&wbar))
            : "memory");
      }
    }
  } else if (blockIdx.x == 0 && tid == 0) {
    prefetch_l2_bulk(wr, static_cast<uint32_t>(E) * H * 2);  // weights: no dependency
  }
  prefetch_share(pf);  // the next GEMM's first weights, while HBM is otherwise idle
  if (row0 >= T) return;  // a prefetch-only CTA (uniform across the CTA)
  pdl_wait();  // expert outputs / rows come from the previous kernel

  // (1) rows of h into shared memory
  for (int i = tid; i < R * hv; i += blockDim.x) {
    const int r = i / hv, c = i % hv;
    uint4 o = make_uint4(0, 0, 0, 0);
    if (r < nrows) {
      const size_t row = static_cast<size_t>(row0 + r);
      if (y_perm) {
        int pos[8];
        float wj[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          pos[j] = (j < k_prev) ? inv[row * k_prev + j] : -1;
          wj[j] = (j < k_prev) ? w_prev[row * k_prev + j] : 0.f;
        }
        float4 ya[8], yb[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          // by entry, the row address needs no routing data: the loads issue with those of inv
          const bool ok = y_by_entry ? (j < k_prev) : (pos[j] >= 0 && pos[j] < n_pos);
          const size_t yrow = y_by_entry ? row * k_prev + j : static_cast<size_t>(pos[j]);
          if (ok) {
            const float4* yp = reinterpret_cast<const float4*>(y_perm + yrow * H) + 2 * c;
            ya[j] = yp[0];
            yb[j] = yp[1];
          } else {
            ya[j] = yb[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        float4 sa = make_float4(0.f, 0.f, 0.f, 0.f), sb = sa;
        if (y_sh) {
          const float4* ys = reinterpret_cast<const float4*>(y_sh + row * H) + 2 * c;
          sa = ys[0];
          sb = ys[1];
        }
        const uint4 rv = reinterpret_cast<const uint4*>(x + row * H)[c];
        float m[8];
#pragma unroll
        for (int i2 = 0; i2 < 8; ++i2) m[i2] = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < k_prev) {
            if (pos[j] < 0 || pos[j] >= n_pos) {
              if (err && c == 0) atomicOr(err, kErrInternal);
              continue;
            }
            const float yv[8] = {ya[j].x, ya[j].y, ya[j].z, ya[j].w, yb[j].x, yb[j].y, yb[j].z, yb[j].w};
#pragma unroll
            for (int i2 = 0; i2 < 8; ++i2) m[i2] = __fadd_rn(m[i2], __fmul_rn(wj[j], yv[i2]));
          }
        }
        if (y_sh) {
          const float yv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
#pragma unroll
          for (int i2 = 0; i2 < 8; ++i2) m[i2] = __fadd_rn(m[i2], yv[i2]);
        }
        float rf[8];
        bf16x8_to_f32(rv, rf);
        uint32_t ow[4];
#pragma unroll
        for (int i2 = 0; i2 < 4; ++i2)
          ow[i2] = static_cast<uint32_t>(f32_to_bf16_bits(__fadd_rn(rf[2 * i2], m[2 * i2]))) |
                   (static_cast<uint32_t>(f32_to_bf16_bits(__fadd_rn(rf[2 * i2 + 1], m[2 * i2 + 1]))) << 16);
        o = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        reinterpret_cast<uint4*>(out + row * H)[c] = o;
      } else {
        o = reinterpret_cast<const uint4*>(x + row * H)[c];
      }
    }
    reinterpret_cast<uint4*>(hs + static_cast<size_t>(r) * H)[c] = o;
  }
  __syncthreads();

  // (1b) pre-RMSNorm variant: the router and the experts take
  //      x = bf16((h * s) * g), s = 1 / sqrt(sum(h^2) / H + eps); the rows are
  //      normalised in shared memory and written to xn_out (the shared
  //      expert's input); the combined rows written above stay the residual.
  if (norm_gain) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float ss = 0.f;
      for (int c = tid; c < hv; c += blockDim.x) {
        float f[8];
        bf16x8_to_f32(reinterpret_cast<const uint4*>(hs + static_cast<size_t>(r) * H)[c], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = __fadd_rn(ss, __fmul_rn(f[i], f[i]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
      if (lane == 0) nred[r][warp] = ss;
    }
    __syncthreads();
    for (int i = tid; i < R * hv; i += blockDim.x) {
      const int r = i / hv, c = i % hv;
      if (r >= nrows) continue;
      float tot = 0.f;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot = __fadd_rn(tot, nred[r][w]);
      const float sc = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, static_cast<float>(H)), kRmsNormEps)));
      float f[8], g[8];
      bf16x8_to_f32(reinterpret_cast<const uint4*>(hs + static_cast<size_t>(r) * H)[c], f);
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(norm_gain) + c), g);
      uint32_t ow[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        ow[q] = static_cast<uint32_t>(f32_to_bf16_bits(__fmul_rn(__fmul_rn(f[2 * q], sc), g[2 * q]))) |
                (static_cast<uint32_t>(f32_to_bf16_bits(__fmul_rn(__fmul_rn(f[2 * q + 1], sc), g[2 * q + 1]))) << 16);
      const uint4 o = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      reinterpret_cast<uint4*>(hs + static_cast<size_t>(r) * H)[c] = o;
      reinterpret_cast<uint4*>(xn_out + static_cast<size_t>(row0 + r) * H)[c] = o;
    }
    __syncthreads();
  }

  if (STAGE) {  // bounded wait for the router matrix; on a timeout the rows are reported, not routed
    if (tid == 0) {
      int dummy = 0;
      wok_s = mbar_wait(&wbar, 0, &dummy, err, globaltimer_ns() + timeout_ns) ? 1 : 0;
      // whatever the outcome, the copies must land before this CTA may exit
      if (!wok_s) mbar_wait(&wbar, 0, &dummy, nullptr, globaltimer_ns() + kDrainNs);
    }
    __syncthreads();
    if (!wok_s) {
      if (tid < nrows * k) {
        const size_t i = static_cast<size_t>(row0) * k + tid;
        idx[i] = -1;
        wout[i] = 0.f;
        if (slab_counts) inv_out[i] = -1;
      }
      return;
    }
  }

  // (2) router logits: warp w owns experts w, w+16, w+32, w+48 (one batch of
  //     loads for E <= 64); each x vector is converted once and reused, and
  //     the products go through packed f32x2 FMAs (even and odd partial sums).
  constexpr int EB = 4;
  const int nwarps = blockDim.x >> 5;
  for (int e0 = warp; e0 < E; e0 += nwarps * EB) {
    uint4 wv[EB][NV];
#pragma unroll
    for (int b = 0; b < EB; ++b) {
      const int e = e0 + nwarps * b;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const int c = lane + 32 * v;
        if (STAGE)
          wv[b][v] = (e < E && c < hv) ? reinterpret_cast<const uint4*>(wsm + static_cast<size_t>(e) * H)[c]
                                       : make_uint4(0, 0, 0, 0);
        else
          wv[b][v] = (e < E && c < hv) ? __ldg(reinterpret_cast<const uint4*>(wr + static_cast<size_t>(e) * H) + c)
                                       : make_uint4(0, 0, 0, 0);
      }
    }
    float acc[EB][R];
#pragma unroll
    for (int b = 0; b < EB; ++b)
#pragma unroll
      for (int r = 0; r < R; ++r) acc[b][r] = 0.f;
    uint64_t acc2[EB][R];
#pragma unroll
    for (int b = 0; b < EB; ++b)
#pragma unroll
      for (int r = 0; r < R; ++r) acc2[b][r] = 0ull;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int c = lane + 32 * v;
      if (c < hv) {
        uint64_t xp[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint4 xv = reinterpret_cast<const uint4*>(hs + static_cast<size_t>(r) * H)[c];
          const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) xp[r][i] = bf16x2_pair(xw[i]);
        }
#pragma unroll
        for (int b = 0; b < EB; ++b) {
          const uint32_t ww[4] = {wv[b][v].x, wv[b][v].y, wv[b][v].z, wv[b][v].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint64_t wp = bf16x2_pair(ww[i]);
#pragma unroll
            for (int r = 0; r < R; ++r) acc2[b][r] = ffma2(xp[r][i], wp, acc2[b][r]);
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < EB; ++b)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float2 pr = unpack2f(acc2[b][r]);
        acc[b][r] = pr.x + pr.y;
      }
#pragma unroll
    for (int b = 0; b < EB; ++b) {
      const int e = e0 + nwarps * b;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float v = acc[b][r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && e < E) ls[r * E + e] = bias ? v + bias[e] : v;
      }
    }
  }
  __syncthreads();

  // (3) top-k: the ranks by the whole block, then the weights by warps
  //     0..R-1 while the last warp claims the slab rows (4)
  topk_rank_block(ls, E, k, nrows, sel_s);
  topk_weights_rows(ls, E, k, nrows, sel_s, idx + static_cast<size_t>(row0) * k, wout + static_cast<size_t>(row0) * k,
                    0, R);
  if (!slab_counts) return;  // uniform across the CTA

  // (4) slab placement of the routed rows
  const int ct = tid - (static_cast<int>(blockDim.x) - 32);  // lane of the last warp
  if (ct >= 0 && ct < nrows * k) {
    const int r = ct / k, j = ct % k;
    const int e = sel_s[r * 8 + j];
    int p = -1;
    if (e >= 0 && e < E) {
      const int c = atomicAdd(&slab_counts[e], 1);
      if (c < slab_rows) {
        p = e * slab_rows + c;
      } else {
        atomicSub(&slab_counts[e], 1);
      }
    }
    if (p < 0 && err) atomicOr(err, kErrInternal);
    pos_s[r * 8 + j] = p;
    inv_out[static_cast<size_t>(row0 + r) * k + j] = p;
    if (ent_out && p >= 0) ent_out[p] = (row0 + r) * k + j;
  }
  __syncthreads();
  for (int i = tid; i < nrows * k * hv; i += blockDim.x) {
    const int q = i / hv, c = i % hv;
    const int r = q / k, j = q % k;
    const int p = pos_s[r * 8 + j];
    if (p >= 0)
      reinterpret_cast<uint4*>(x_slab + static_cast<size_t>(p) * H)[c] =
          reinterpret_cast<const uint4*>(hs + static_cast<size_t>(r) * H)[c];
  }
}

// Shared memory of one combine-route CTA: the rows and their logits, plus
// the router matrix when it is staged.
static size_t combine_route_smem(int R, int H, int E, bool stage) {
  return (stage ? static_cast<size_t>(E) * H * 2 : 0) + static_cast<size_t>(R) * H * 2 +
         static_cast<size_t>(R) * E * 4;
}

template <int R, int NV, bool STAGE>
static cudaError_t launch_combine_route_rvs(const CombineRouteArgs& a, cudaStream_t s) {
  const size_t smem = combine_route_smem(R, a.H, a.E, STAGE);
  if (STAGE) {
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
      cudaError_t e = cudaFuncSetAttribute(combine_route_kernel<R, NV, STAGE>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
      if (e != cudaSuccess) return e;
      configured_dev = dev;
    }
  }
  const int rows_ctas = (a.T + R - 1) / R;
  const int grid = rows_ctas > prefetch_ctas(a.pf) ? rows_ctas : prefetch_ctas(a.pf);  // extra CTAs only prefetch
  return launch_pdl(combine_route_kernel<R, NV, STAGE>, dim3(grid), dim3(512), smem, s, a.x, a.y_perm, a.y_sh,
                    a.inv, a.w_prev, a.k_prev, a.n_pos > 0 ? a.n_pos : a.T * a.k_prev, a.out, a.T, a.H, a.E, a.k,
                    a.wr, a.bias, a.idx, a.w, a.err, a.pf, a.slab_counts, a.inv_out, a.x_slab, a.slab_rows,
                    a.norm_gain, a.xn_out, a.timeout_ns > 0 ? a.timeout_ns : kDrainNs, a.ent_out,
                    a.y_by_entry ? 1 : 0);
}

// The router matrix is staged when it fits beside the rows (E * H * 2 bytes,
// 160 KB at the model shape) and its address suits the bulk copy.
template <int R, int NV>
static cudaError_t launch_combine_route_rv(const CombineRouteArgs& a, cudaStream_t s) {
  const bool stage = combine_route_smem(R, a.H, a.E, true) <= 200 * 1024 &&
                     (reinterpret_cast<uintptr_t>(a.wr) & 15) == 0;
  return stage ? launch_combine_route_rvs<R, NV, true>(a, s) : launch_combine_route_rvs<R, NV, false>(a, s);
}

// Larger batches route with the shared-memory-staged router instead (each of
// its persistent CTAs reads the router weights once).
bool combine_route_supported(int T, int H, int E) {
  return T <= 1024 && H <= 2048 && E <= 256 && (2 * H * 2 + 2 * E * 4) <= 48 * 1024;
}

cudaError_t launch_combine_route(const CombineRouteArgs& a, cudaStream_t s) {
  if (a.T <= 0) return cudaSuccess;
  if (!combine_route_supported(a.T, a.H, a.E)) return cudaErrorInvalidValue;
  const int nv = (a.H / 8 + 31) / 32;
  // one row per CTA while that keeps the router-row traffic from L2 modest
  const int R = a.T <= 512 ? 1 : 2;
#define MV_CR(RR)                                              \
  switch (nv) {                                                \
    case 1: return launch_combine_route_rv<RR, 1>(a, s);       \
    case 2: return launch_combine_route_rv<RR, 2>(a, s);       \
    case 3: return launch_combine_route_rv<RR, 3>(a, s);       \
    case 4: return launch_combine_route_rv<RR, 4>(a, s);       \
    case 5: return launch_combine_route_rv<RR, 5>(a, s);       \
    case 6: return launch_combine_route_rv<RR, 6>(a, s);       \
    case 7: return launch_combine_route_rv<RR, 7>(a, s);       \
    default: return launch_combine_route_rv<RR, 8>(a, s);      \
  }
  if (R == 1) { MV_CR(1) }
  MV_CR(2)
#undef MV_CR
}

// ---------------------------------------------------------------------------
// Grouping by expert.  One CTA per expert e:
//   counts[e]  = #entries routed to e, offsets[e] = #entries routed below e,
//   perm[offsets[e] + p] = the p-th entry (row order) routed to e,
//   inv[entry] = its position in perm,
//   x_perm[position] = x[row of entry]  (the gathered GEMM input).
// Entries are i = r*k + j; a row never selects the same expert twice, so row
// order within an expert is (row, slot) order.  Exact and deterministic.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) permute_kernel(const int32_t* __restrict__ idx, int T, int E,
                                                      int k, int32_t* __restrict__ counts,
                                                      int32_t* __restrict__ offsets,
                                                      int32_t* __restrict__ perm,
                                                      int32_t* __restrict__ inv,
                                                      const uint16_t* __restrict__ x, int H,
                                                      uint16_t* __restrict__ x_perm) {
  extern __shared__ int32_t idx_s[];  // the routing staged once (when it fits), else read from global
  const int e = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = T * k;
  const bool staged = n <= kPermuteStage;
  __shared__ int red_eq[8], red_lt[8], wsum[8];
  __shared__ int base_s, running_s;
  __shared__ int plist[kPermuteStage / 4];  // this expert's entries (when staged)

  pdl_trigger();
  pdl_wait();
  if (staged)
    for (int i = tid; i < n; i += blockDim.x) idx_s[i] = idx[i];
  __syncthreads();
  const int32_t* src = staged ? idx_s : idx;

  int c_eq = 0, c_lt = 0;
  for (int i = tid; i < n; i += blockDim.x) {
    const int v = src[i];
    c_eq += (v == e);
    c_lt += (v >= 0 && v < e);
    if (e == 0 && (v < 0 || v >= E)) inv[i] = -1;  // out-of-range id: routed nowhere
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c_eq += __shfl_xor_sync(0xffffffffu, c_eq, o);
    c_lt += __shfl_xor_sync(0xffffffffu, c_lt, o);
  }
  if (lane == 0) {
    red_eq[warp] = c_eq;
    red_lt[warp] = c_lt;
  }
  __syncthreads();
  if (tid == 0) {
    int a = 0, b = 0;
    for (int w = 0; w < 8; ++w) {
      a += red_eq[w];
      b += red_lt[w];
    }
    counts[e] = a;
    offsets[e] = b;
    if (e == E - 1) offsets[E] = a + b;
    base_s = b;
    running_s = 0;
  }
  __syncthreads();
  const int base = base_s;
  const bool local_list = staged && (n / 4 >= 1);

  for (int r0 = 0; r0 < T; r0 += blockDim.x) {
    const int r = r0 + tid;
    int slot = -1;
    if (r < T)
      for (int j = 0; j < k; ++j)
        if (src[static_cast<size_t>(r) * k + j] == e) slot = j;
    const unsigned bal = __ballot_sync(0xffffffffu, slot >= 0);
    const int before = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int wpre = 0, tot = 0;
    for (int w = 0; w < 8; ++w) {
      if (w < warp) wpre += wsum[w];
      tot += wsum[w];
    }
    if (slot >= 0) {
      const int p = running_s + wpre + before;
      const int ent = r * k + slot;
      perm[base + p] = ent;
      inv[ent] = base + p;
      if (local_list && p < kPermuteStage / 4) plist[p] = ent;
    }
    __syncthreads();
    if (tid == 0) running_s += tot;
    __syncthreads();
  }

  // gather the routed rows (each warp copies whole rows with 16-byte vectors)
  const int cnt = running_s;
  const int hv = H / 8;
  for (int p = warp; p < cnt; p += 8) {
    const int ent = (local_list && p < kPermuteStage / 4) ? plist[p] : perm[base + p];
    const uint4* srcr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(ent / k) * H);
    uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(base + p) * H);
    for (int c0 = 0; c0 < hv; c0 += 32 * 8) {  // all loads of up to 8 vectors per lane before the stores
      uint4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = c0 + lane + 32 * i;
        if (c < hv) v[i] = srcr[c];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = c0 + lane + 32 * i;
        if (c < hv) dst[c] = v[i];
      }
    }
  }
}

cudaError_t launch_permute(const int32_t* idx, int T, int E, int k, int32_t* counts,
                           int32_t* offsets, int32_t* perm, int32_t* inv, const uint16_t* x,
                           int H, uint16_t* x_perm, cudaStream_t s) {
  const size_t smem = (static_cast<size_t>(T) * k <= kPermuteStage) ? static_cast<size_t>(T) * k * 4 : 0;
  return launch_pdl(permute_kernel, dim3(E), dim3(256), smem, s, idx, T, E, k, counts, offsets, perm, inv, x, H, x_perm);
}

// ---------------------------------------------------------------------------
// Grouping by expert for large batches: a stable counting sort of the T*k
// routing entries by expert, in three kernels.
//  rank:  one CTA per chunk of kSortChunkRows rows walks its entries in id
//         order, 256 at a time: ranks within a warp from __match_any_sync,
//         across warps and waves from per-expert running counts; writes each
//         entry's rank within (chunk, expert) and the chunk's per-expert counts.
//  scan:  per expert, exclusive prefix over chunks; counts, offsets.
//  place: position = offsets[e] + chunk base + rank; writes perm / inv and
//         copies the row into the grouped input (one warp per entry, all SMs).
// The result is the same permutation as permute_kernel's.
// ---------------------------------------------------------------------------
constexpr int kSortChunkRows = 256;

__global__ void __launch_bounds__(256) sort_rank_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                                                        int32_t* __restrict__ rank, int32_t* __restrict__ chunk_counts) {
  extern __shared__ int32_t sh[];
  int32_t* cnt = sh;           // [E] running counts of this chunk
  int32_t* wcnt = sh + E;      // [8][E] per-warp counts of the current wave
  pdl_trigger();
  pdl_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int ent0 = c * kSortChunkRows * k;
  const int ent1 = min(T, (c + 1) * kSortChunkRows) * k;
  for (int i = tid; i < E; i += 256) cnt[i] = 0;
  for (int e0 = ent0; e0 < ent1; e0 += 256) {
    for (int i = tid; i < 8 * E; i += 256) wcnt[i] = 0;
    __syncthreads();
    const int ent = e0 + tid;
    int e = (ent < ent1) ? idx[ent] : -1;
    if (e >= E) e = -1;
    const unsigned mask = __match_any_sync(0xffffffffu, e);
    const int rw = __popc(mask & ((1u << lane) - 1u));
    if (e >= 0 && rw == 0) wcnt[warp * E + e] = __popc(mask);
    __syncthreads();
    for (int ex = tid; ex < E; ex += 256) {  // prefix over warps, carried across waves
      int run = cnt[ex];
      for (int w = 0; w < 8; ++w) {
        const int t = wcnt[w * E + ex];
        wcnt[w * E + ex] = run;
        run += t;
      }
      cnt[ex] = run;
    }
    __syncthreads();
    if (e >= 0) rank[ent] = wcnt[warp * E + e] + rw;
    __syncthreads();
  }
  for (int i = tid; i < E; i += 256) chunk_counts[static_cast<size_t>(c) * E + i] = cnt[i];
}

__global__ void __launch_bounds__(256) sort_scan_kernel(int32_t* __restrict__ chunk_counts, int nchunks, int E,
                                                        int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
  __shared__ int32_t tot[256];
  pdl_trigger();
  pdl_wait();
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    for (int c = 0; c < nchunks; ++c) {  // in place: chunk counts become chunk bases
      const int v = chunk_counts[static_cast<size_t>(c) * E + e];
      chunk_counts[static_cast<size_t>(c) * E + e] = run;
      run += v;
    }
    counts[e] = run;
  }
  tot[e] = (e < E) ? run : 0;
  __syncthreads();
  if (e == 0) {
    int acc = 0;
    for (int i = 0; i < E; ++i) {
      offsets[i] = acc;
      acc += tot[i];
    }
    offsets[E] = acc;
  }
}

__global__ void __launch_bounds__(256) sort_place_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                                                         const int32_t* __restrict__ rank,
                                                         const int32_t* __restrict__ chunk_base,
                                                         const int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                         const uint16_t* __restrict__ x, int H,
                                                         uint16_t* __restrict__ x_perm) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  const int hv = H / 8;
  for (int ent = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); ent < T * k; ent += nwarps) {
    const int e = idx[ent];
    if (e < 0 || e >= E) {
      if (lane == 0) inv[ent] = -1;  // out-of-range id: routed nowhere
      continue;
    }
    const int row = ent / k;
    const int pos = offsets[e] + chunk_base[static_cast<size_t>(row / kSortChunkRows) * E + e] + rank[ent];
    if (lane == 0) {
      perm[pos] = ent;
      inv[ent] = pos;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(row) * H);
    uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(pos) * H);
    for (int c0 = 0; c0 < hv; c0 += 32 * 8) {
      uint4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = c0 + lane + 32 * i;
        if (c < hv) v[i] = src[c];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = c0 + lane + 32 * i;
        if (c < hv) dst[c] = v[i];
      }
    }
  }
}

size_t sort_scratch_ints(int T, int E, int k) {
  const int nchunks = (T + kSortChunkRows - 1) / kSortChunkRows;
  return static_cast<size_t>(T) * k + static_cast<size_t>(nchunks) * E;
}

bool permute_uses_sort(int T, int k) { return static_cast<int64_t>(T) * k > kPermuteStage; }

cudaError_t launch_permute_sorted(const int32_t* idx, int T, int E, int k, int32_t* counts, int32_t* offsets,
                                  int32_t* perm, int32_t* inv, const uint16_t* x, int H, uint16_t* x_perm,
                                  int32_t* scratch, cudaStream_t s) {
  const int nchunks = (T + kSortChunkRows - 1) / kSortChunkRows;
  int32_t* rank = scratch;
  int32_t* chunk = scratch + static_cast<size_t>(T) * k;
  cudaError_t e = launch_pdl(sort_rank_kernel, dim3(nchunks), dim3(256), static_cast<size_t>(9 * E) * 4, s, idx, T, E,
                             k, rank, chunk);
  if (e != cudaSuccess) return e;
  e = launch_pdl(sort_scan_kernel, dim3(1), dim3(256), 0, s, chunk, nchunks, E, counts, offsets);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return launch_pdl(sort_place_kernel, dim3(sms * 4), dim3(256), 0, s, idx, T, E, k,
                    static_cast<const int32_t*>(rank), static_cast<const int32_t*>(chunk),
                    static_cast<const int32_t*>(offsets), perm, inv, x, H, x_perm);
}

// ---------------------------------------------------------------------------
// Combine: out[r] = bf16(res[r] + (sum_j w[r][j] * y[pos(r, j)] + y_sh[r])), the
// products and sums singly rounded (no fused multiply-add), in slot order with
// the shared expert last.  A warp task is one 256-element slice of a row:
// lanes 0..k-1 load the row's routing and broadcast it, then lane l combines
// the 8 consecutive features of chunk 32 * slice + l; all the loads of a chunk
// (k expert rows, the shared row, the residual) issue together.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y_perm,
                                                      const float* __restrict__ y_sh,
                                                      const int32_t* __restrict__ inv,
                                                      const float* __restrict__ w,
                                                      const uint16_t* res, uint16_t* out, int T,
                                                      int H, int k, int n_pos, int* err, const L2Prefetch pf,
                                                      int by_entry) {
  pdl_trigger();
  prefetch_share(pf);
  pdl_wait();
  const int hv = H / 8;
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  // A warp task is one 32-chunk slice (256 elements) of one row, so that a
  // decode batch of a hundred rows still spreads over every launched warp.
  const int nslice = (hv + 31) / 32;
  const long long ntask = static_cast<long long>(T) * nslice;
  for (long long q = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; q < ntask; q += nwarps) {  // uniform per warp
    const int r = static_cast<int>(q / nslice);
    const int slice = static_cast<int>(q - static_cast<long long>(r) * nslice);
    const int pl = (lane < k) ? inv[static_cast<size_t>(r) * k + lane] : -1;
    const float wl = (lane < k) ? w[static_cast<size_t>(r) * k + lane] : 0.f;
    int pos[8];
    float wj[8];
    bool okj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      pos[j] = __shfl_sync(0xffffffffu, pl, j);
      wj[j] = __shfl_sync(0xffffffffu, wl, j);
      okj[j] = (j < k) && pos[j] >= 0 && pos[j] < n_pos;
    }
    bool bad = false;
#pragma unroll
    for (int j = 0; j < 8; ++j) bad |= (j < k) && !okj[j];
    if (lane == 0 && slice == 0 && err && bad) atomicOr(err, kErrInternal);  // an entry routed to no valid expert
    const int c = slice * 32 + lane;
    if (c < hv) {
      float4 ya[8], yb[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // by entry, the row address needs no routing data
        const bool ld = by_entry ? (j < k) : okj[j];
        const size_t yrow = by_entry ? static_cast<size_t>(r) * k + j : static_cast<size_t>(pos[j]);
        if (ld) {
          const float4* yp = reinterpret_cast<const float4*>(y_perm + yrow * H) + 2 * c;
          ya[j] = yp[0];
          yb[j] = yp[1];
        } else {
          ya[j] = yb[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float4 sa = make_float4(0.f, 0.f, 0.f, 0.f), sb = sa;
      if (y_sh) {
        const float4* ys = reinterpret_cast<const float4*>(y_sh + static_cast<size_t>(r) * H) + 2 * c;
        sa = ys[0];
        sb = ys[1];
      }
      uint4 rv = make_uint4(0, 0, 0, 0);
      if (res) rv = reinterpret_cast<const uint4*>(res + static_cast<size_t>(r) * H)[c];
      float m[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (!okj[j]) continue;
        const float yv[8] = {ya[j].x, ya[j].y, ya[j].z, ya[j].w, yb[j].x, yb[j].y, yb[j].z, yb[j].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = __fadd_rn(m[i], __fmul_rn(wj[j], yv[i]));
      }
      if (y_sh) {
        const float yv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = __fadd_rn(m[i], yv[i]);
      }
      if (res) {
        float rf[8];
        bf16x8_to_f32(rv, rf);
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = __fadd_rn(rf[i], m[i]);
      }
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[i] = static_cast<uint32_t>(f32_to_bf16_bits(m[2 * i])) |
               (static_cast<uint32_t>(f32_to_bf16_bits(m[2 * i + 1])) << 16);
      reinterpret_cast<uint4*>(out + static_cast<size_t>(r) * H)[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

cudaError_t launch_combine(const float* y_perm, const float* y_sh, const int32_t* inv,
                           const float* w, const uint16_t* res, uint16_t* out, int T, int H,
                           int k, int n_pos, int* err, const L2Prefetch& pf, cudaStream_t s, bool y_by_entry) {
  if (T <= 0) return cudaSuccess;
  const long long tasks = static_cast<long long>(T) * ((H / 8 + 31) / 32);  // (row, 256-element slice)
  const long long blocks = (tasks + 7) / 8;  // 8 tasks (warps) per CTA
  int grid = static_cast<int>(blocks < 148LL * 8 ? blocks : 148LL * 8);
  if (grid < prefetch_ctas(pf)) grid = prefetch_ctas(pf);  // the grid-stride loop leaves the extra CTAs idle
  return launch_pdl(combine_kernel, dim3(grid), dim3(256), 0, s, y_perm, y_sh, inv, w, res, out, T, H, k, n_pos, err,
                    pf, y_by_entry ? 1 : 0);
}

// ---------------------------------------------------------------------------
// LM-head argmax finalisation: the GEMM epilogue leaves, per token, packed
// (order-preserving logit, inverted index) keys, token-major ([T][nparts]):
// one per (256-row vocabulary tile, lane quarter) of the single-CTA tiles, or
// one per 256-row tile on CTA pairs; the largest key is the argmax with ties
// to the lower index.  `nthr` threads (a multiple of 32) reduce one token's
// keys with coalesced, unrolled loads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t umax64(uint64_t a, uint64_t b) { return a > b ? a : b; }

__device__ __forceinline__ uint64_t row_max_key(const uint64_t* row, int nparts, int t0, int nthr,
                                                uint64_t* red, int lane, int wid) {
  // sixteen independent loads in flight per thread: 256 threads cover the
  // 2,264 keys of a 129,280-row vocabulary in one round trip
  constexpr int kInFlight = 16;
  uint64_t b[kInFlight];
#pragma unroll
  for (int i = 0; i < kInFlight; ++i) b[i] = 0;
  for (int p0 = t0; p0 < nparts; p0 += kInFlight * nthr) {
#pragma unroll
    for (int i = 0; i < kInFlight; ++i) {
      const int p = p0 + i * nthr;
      if (p < nparts) b[i] = umax64(b[i], row[p]);
    }
  }
#pragma unroll
  for (int w = kInFlight / 2; w > 0; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) b[i] = umax64(b[i], b[i + w]);
  uint64_t best = b[0];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = umax64(best, __shfl_xor_sync(0xffffffffu, best, o));
  if (lane == 0) red[wid] = best;
  return best;
}

__global__ void __launch_bounds__(128) lm_finalize_kernel(const uint64_t* __restrict__ keys, int nparts,
                                                          int ld, int T, int32_t* __restrict__ argmax) {
  __shared__ uint64_t red[4];
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  row_max_key(keys + static_cast<size_t>(t) * ld, nparts, threadIdx.x, 128, red, lane, wid);
  __syncthreads();
  if (threadIdx.x == 0)
    argmax[t] = static_cast<int32_t>(argmax_key_index(umax64(umax64(red[0], red[1]), umax64(red[2], red[3]))));
}

cudaError_t launch_lm_finalize(const uint64_t* keys, int nparts, int ld, int T, int32_t* argmax,
                               cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  return launch_pdl(lm_finalize_kernel, dim3(T), dim3(128), 0, s, keys, nparts, ld, T, argmax);
}

// ---------------------------------------------------------------------------
// RMSNorm of T rows (the pre-RMSNorm layer variant): one CTA of 256 threads
// per row, out = bf16((x * s) * g), s = 1 / sqrt(sum(x^2) / H + eps), with the
// products and sums singly rounded.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) rmsnorm_kernel(const uint16_t* __restrict__ x, int H,
                                                      const uint16_t* __restrict__ gain, uint16_t* __restrict__ out) {
  __shared__ float red[8];
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(r) * H);
  const int hv = H / 8;
  float ss = 0.f;
  for (int c = tid; c < hv; c += 256) {
    float f[8];
    bf16x8_to_f32(xr[c], f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = __fadd_rn(ss, __fmul_rn(f[i], f[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
  if (lane == 0) red[wid] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot = __fadd_rn(tot, red[w]);
  const float sc = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, static_cast<float>(H)), kRmsNormEps)));
  uint4* orow = reinterpret_cast<uint4*>(out + static_cast<size_t>(r) * H);
  for (int c = tid; c < hv; c += 256) {
    float f[8], g[8];
    bf16x8_to_f32(xr[c], f);
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(gain) + c), g);
    uint32_t ow[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      ow[q] = static_cast<uint32_t>(f32_to_bf16_bits(__fmul_rn(__fmul_rn(f[2 * q], sc), g[2 * q]))) |
              (static_cast<uint32_t>(f32_to_bf16_bits(__fmul_rn(__fmul_rn(f[2 * q + 1], sc), g[2 * q + 1]))) << 16);
    orow[c] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  }
}

cudaError_t launch_rmsnorm(const uint16_t* x, int T, int H, const uint16_t* gain, uint16_t* out, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  return launch_pdl(rmsnorm_kernel, dim3(T), dim3(256), 0, s, x, H, gain, out);
}

// ---------------------------------------------------------------------------
// FastMTP draft block: the per-sequence step between its GEMMs (jina-ocr-v1
// model card, decoding-speed paragraph: one dense draft block applied
// recursively).  One CTA of 256 threads per sequence b:
//  (1) the token t: with keys, the previous step's draft = the greedy choice
//      of the LM head (largest packed key of row b), written to
//      drafts[b][j-1]; without, t0[b] (the verifier's next token);
//  (2) with u, the block's next input row
//        u[b] = [ bf16((h * r_h) * g_h) ; bf16((e * r_e) * g_e) ],  e = w_emb[t],
//        r = 1 / sqrt(sum(x^2) / H + eps)  (products and sums rounded singly),
//      h = row b*row_stride + (acc ? acc[b] : 0) of h_src.
// A token outside [0, V) (a failed LM step, or a bad t0) is reported as an
// internal error, written as -1, and embeds row 0.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float block_sum_256(float v, float* red8, int lane, int wid) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) red8[wid] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) s = __fadd_rn(s, red8[w]);
  return s;
}

__global__ void __launch_bounds__(256) mtp_step_kernel(
    const uint64_t* __restrict__ keys, int nparts, int ld, const int32_t* __restrict__ t0,
    int32_t* __restrict__ drafts, int K, int j, const uint16_t* __restrict__ h_src, int row_stride,
    const int32_t* __restrict__ acc, const uint16_t* __restrict__ w_emb, int V, const uint16_t* __restrict__ g_h,
    const uint16_t* __restrict__ g_e, int H, float eps, uint16_t* __restrict__ u, int* err) {
  __shared__ uint64_t red[8];
  __shared__ float red_h[8], red_e[8];
  __shared__ int t_s;
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (keys) {
    row_max_key(keys + static_cast<size_t>(b) * ld, nparts, tid, 256, red, lane, wid);
    __syncthreads();
    if (tid == 0) {
      uint64_t best = red[0];
      for (int w = 1; w < 8; ++w) best = umax64(best, red[w]);
      int t = static_cast<int>(argmax_key_index(best));
      if (t < 0 || t >= V) {
        t = -1;
        if (err) atomicOr(err, kErrInternal);
      }
      drafts[static_cast<size_t>(b) * K + (j - 1)] = t;
      t_s = t;
    }
  } else if (tid == 0) {
    int t = t0[b];
    if (t < 0 || t >= V) {
      t = -1;
      if (err) atomicOr(err, kErrInternal);
    }
    t_s = t;
  }
  __syncthreads();
  if (!u) return;  // uniform: the last step only writes its draft
  const int t = t_s < 0 ? 0 : t_s;
  int a = acc ? acc[b] : 0;
  a = a < 0 ? 0 : (a >= row_stride ? row_stride - 1 : a);
  const uint4* hrow = reinterpret_cast<const uint4*>(h_src + (static_cast<size_t>(b) * row_stride + a) * H);
  const uint4* erow = reinterpret_cast<const uint4*>(w_emb + static_cast<size_t>(t) * H);
  const int hv = H / 8;
  float sh = 0.f, se = 0.f;
  for (int c = tid; c < hv; c += 256) {
    float fh[8], fe[8];
    bf16x8_to_f32(hrow[c], fh);
    bf16x8_to_f32(__ldg(erow + c), fe);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sh = __fadd_rn(sh, __fmul_rn(fh[i], fh[i]));
      se = __fadd_rn(se, __fmul_rn(fe[i], fe[i]));
    }
  }
  sh = block_sum_256(sh, red_h, lane, wid);
  se = block_sum_256(se, red_e, lane, wid);
  const float rh = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(sh, static_cast<float>(H)), eps)));
  const float re = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(se, static_cast<float>(H)), eps)));
  uint4* urow = reinterpret_cast<uint4*>(u + static_cast<size_t>(b) * 2 * H);
  const uint4* gh = reinterpret_cast<const uint4*>(g_h);
  const uint4* ge = reinterpret_cast<const uint4*>(g_e);
  for (int c = tid; c < hv; c += 256) {
    float fh[8], fe[8], gfh[8], gfe[8];
    bf16x8_to_f32(hrow[c], fh);
    bf16x8_to_f32(__ldg(erow + c), fe);
    bf16x8_to_f32(__ldg(gh + c), gfh);
    bf16x8_to_f32(__ldg(ge + c), gfe);
    uint32_t oh[4], oe[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      oh[i] = static_cast<uint32_t>(f32_to_bf16_bits(__fmul_rn(__fmul_rn(fh[2 * i], rh), gfh[2 * i]))) |
              (static_cast<uint32_t>(f32_to_bf16_bits(__fmul_rn(__fmul_rn(fh[2 * i + 1], rh), gfh[2 * i + 1]))) << 16);
      oe[i] = static_cast<uint32_t>(f32_to_bf16_bits(__fmul_rn(__fmul_rn(fe[2 * i], re), gfe[2 * i]))) |
              (static_cast<uint32_t>(f32_to_bf16_bits(__fmul_rn(__fmul_rn(fe[2 * i + 1], re), gfe[2 * i + 1]))) << 16);
    }
    urow[c] = make_uint4(oh[0], oh[1], oh[2], oh[3]);
    urow[hv + c] = make_uint4(oe[0], oe[1], oe[2], oe[3]);
  }
}

cudaError_t launch_mtp_step(const MtpStepArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  return launch_pdl(mtp_step_kernel, dim3(a.B), dim3(256), 0, s, a.keys, a.nparts, a.ld, a.t0, a.drafts, a.K, a.j,
                    a.h_src, a.row_stride, a.acc, a.w_emb, a.V, a.g_h, a.g_e, a.H, a.eps, a.u, a.err);
}

// ---------------------------------------------------------------------------
// Greedy acceptance (one thread per sequence).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void accept_one(const int32_t* g, const int32_t* d, int K, int b,
                                           int32_t* accepted, int32_t* next_token,
                                           int32_t* emitted) {
  int a = 0;
  while (a < K && d[a] == g[a]) ++a;
  accepted[b] = a;
  next_token[b] = g[a];
  if (emitted)
    for (int j = 0; j <= K; ++j) emitted[static_cast<size_t>(b) * (K + 1) + j] = (j <= a) ? g[j] : -1;
}

__global__ void accept_kernel(const int32_t* __restrict__ argmax, const int32_t* __restrict__ drafts,
                              int B, int K, int32_t* accepted, int32_t* next_token,
                              int32_t* emitted) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  accept_one(argmax + static_cast<size_t>(b) * (K + 1),
             drafts ? drafts + static_cast<size_t>(b) * K : nullptr, K, b, accepted, next_token,
             emitted);
}

cudaError_t launch_accept(const int32_t* argmax, const int32_t* drafts, int B, int K,
                          int32_t* accepted, int32_t* next_token, int32_t* emitted,
                          cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  return launch_pdl(accept_kernel, dim3((B + 127) / 128), dim3(128), 0, s, argmax, drafts, B, K, accepted, next_token,
                    emitted);
}

// Fused LM finalisation + acceptance: one CTA per sequence; 4 warps reduce
// each of its K+1 rows (up to 8 rows at a time), then one thread accepts.
__global__ void __launch_bounds__(1024) accept_from_keys_kernel(
    const uint64_t* __restrict__ keys, int nparts, int ld, const int32_t* __restrict__ drafts, int B, int K,
    int32_t* accepted, int32_t* next_token, int32_t* emitted, int32_t* argmax_out) {
  constexpr int kRowThreads = 256;
  __shared__ int32_t g[64];
  __shared__ uint64_t red[32];
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int rows_at_once = blockDim.x / kRowThreads;
  const int sub = threadIdx.x / kRowThreads;  // which row of the group this thread serves
  const int t_in = threadIdx.x % kRowThreads;
  constexpr int kWarpsPerRow = kRowThreads / 32;
  for (int j0 = 0; j0 <= K; j0 += rows_at_once) {
    const int j = j0 + sub;
    if (j <= K) {
      const int t = b * (K + 1) + j;
      row_max_key(keys + static_cast<size_t>(t) * ld, nparts, t_in, kRowThreads, red, lane, wid);
    }
    __syncthreads();
    if (t_in == 0 && j <= K) {
      uint64_t best = 0;
      for (int i = 0; i < kWarpsPerRow; ++i) best = umax64(best, red[sub * kWarpsPerRow + i]);
      g[j] = static_cast<int32_t>(argmax_key_index(best));
      if (argmax_out) argmax_out[b * (K + 1) + j] = g[j];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0)
    accept_one(g, drafts ? drafts + static_cast<size_t>(b) * K : nullptr, K, b, accepted,
               next_token, emitted);
}

cudaError_t launch_accept_from_keys(const uint64_t* keys, int nparts, int ld, const int32_t* drafts,
                                    int B, int K, int32_t* accepted, int32_t* next_token,
                                    int32_t* emitted, int32_t* argmax, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  const int rows_at_once = min(4, K + 1);
  return launch_pdl(accept_from_keys_kernel, dim3(B), dim3(256 * rows_at_once), 0, s, keys, nparts, ld, drafts, B,
                    K, accepted, next_token, emitted, argmax);
}

}  // namespace mv
