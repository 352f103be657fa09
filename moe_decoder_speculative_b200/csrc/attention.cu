// Decoder self-attention of the verify rows over the key/value cache (sm_100a).
//
// The jina-ocr-v1 model card (architecture paragraph) gives the decoder's
// attention only its 32,768-position limit; the reading this kernel follows
// is causal multi-head attention with as many key/value heads as query heads
// (head dim 128) over a per-sequence cache that already holds the rotated keys
// and the values of every earlier position and of this step's K+1 rows:
// query row j of sequence b (position ctx_len[b] + j) sees positions
// 0..ctx_len[b]+j, scores s = (q . k) / sqrt(128), o = softmax(s) . v.
//
// A decode step has K+1 queries per (sequence, head) against thousands of
// cached positions: 4 flops per byte of cache, far below the tensor cores'
// ridge, so this is a streaming kernel on the CUDA cores, bound by HBM.
// Layout and work split:
//   * cache [B][heads][L_max][128] bf16 (head-major), so a tile of 64
//     positions of one (sequence, head) is 16 KB of contiguous rows; one TMA
//     load of a [k-half][row][64] view brings a K or V tile into shared
//     memory with the 128-byte swizzle (bank-conflict-free row reads);
//   * CTA (split, head, sequence) streams its split of the positions through
//     a ring of STAGES tiles with an online softmax in fp32;
//   * QK on the tensor core: the tile's K rows are the A operand of an
//     M = 128 MMA, the queries (padded to 16 rows) the B operand, the scores
//     land in TMEM and warps 0-1 read them (one position per thread); PV on
//     the CUDA cores: a thread owns 4 dims of the output for a quarter of the
//     positions; partial outputs are summed in a fixed order;
//   * splits of one (sequence, head) are merged by the last CTA to finish
//     (an atomic count per pair), in split order: deterministic.
// Every wait is bounded; a CTA that gives up drains its copies, sets the
// sticky timeout bit and leaves its (sequence, head) unwritten.  No TMA
// multicast is used.

#include "mv_device.cuh"
#include "mv_internal.h"

namespace mv {

namespace {

constexpr int kHd = 128;          // head dim
constexpr int kTile = 64;         // cache positions per tile
constexpr int kTileBytes = kTile * kHd * 2;  // 16 KB per K or V tile
constexpr int kAttnThreads = 128;
constexpr int kQRows = 16;        // the queries padded to the MMA's N (16)

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// bf16 element `col` (0..127) of row `row` of a swizzled [half][64 rows][64]
// tile: 16-byte chunk index XOR (row % 8) within each 128-byte row.
__device__ __forceinline__ const uint8_t* tile_chunk(const uint8_t* tile, int row, int half, int chunk) {
  return tile + half * (kTile * 128) + row * 128 + ((chunk ^ (row & 7)) << 4);
}

}  // namespace

template <int NQ, int STAGES>
__global__ void __launch_bounds__(kAttnThreads) decode_attention_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // the queries as the MMA's B operand: bf16 [2 k-blocks][16 rows][64], 128-byte swizzle
  uint8_t* q_mma = smem + STAGES * 2 * kTileBytes;
  float* p_s = reinterpret_cast<float*>(q_mma + 2 * kQRows * 128);  // [kTile][NQ]
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t s_bar;  // the tile's scores are in TMEM
  __shared__ __align__(8) uint64_t done_bar;  // every MMA of this CTA has completed (before TMEM is freed)
  __shared__ float red_s[4][NQ];
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  __shared__ int last_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nq = p.K + 1;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;

  pdl_trigger();
  pdl_wait();  // the queries and the appended cache rows may come from the previous kernel

  const int ctx = p.ctx_len[b];
  if (ctx < 0 || ctx > p.max_ctx || ctx + nq > p.L_max) {  // uniform across the CTA
    if (split == 0 && tid == 0) atomicOr(p.err, kErrInternal);
    return;
  }
  const int n_keys = ctx + nq;  // positions 0 .. ctx + K
  const int n_split_b = (n_keys + p.split_len - 1) / p.split_len;
  if (split >= n_split_b) return;  // this sequence is shorter than the longest one
  const int k0 = split * p.split_len;
  const int k1 = min(n_keys, k0 + p.split_len);
  const int ntiles = (k1 - k0 + kTile - 1) / kTile;
  const int64_t row0 = (static_cast<int64_t>(b) * p.n_heads + h) * p.L_max + k0;

  if (tid == 0) {
    abort_s = 0;
    for (int i = 0; i < STAGES; ++i) mbar_init(&full_bar[i], 1);
    mbar_init(&s_bar, 1);
    mbar_init(&done_bar, 1);
    fence_barrier_init();
    tma_prefetch_desc(&p.k_map);
    tma_prefetch_desc(&p.v_map);
  }
  if (warp == 0) {  // 32 TMEM columns: the 16 score columns of one tile
    tmem_alloc(&tmem_s, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int t) {  // tile t of this split into stage t % STAGES
    const int st = t % STAGES;
    uint8_t* dst = smem + st * 2 * kTileBytes;
    mbar_arrive_expect_tx(&full_bar[st], 2 * kTileBytes);
    const int y = static_cast<int>(row0 + static_cast<int64_t>(t) * kTile);
    tma_load_3d(dst, &p.k_map, 0, y, 0, &full_bar[st], pol);
    tma_load_3d(dst + kTileBytes, &p.v_map, 0, y, 0, &full_bar[st], pol);
  };
  int issued = 0;
  if (tid == 0)
    for (; issued < STAGES && issued < ntiles; ++issued) issue(issued);

  // queries of this (sequence, head) into the swizzled B tile: row j = query
  // j (rows past K+1 zero), 16-byte chunk c of k-block kb at
  // kb * 2 KB + j * 128 + ((c ^ (j % 8)) * 16)
  for (int i = tid; i < kQRows * 16; i += kAttnThreads) {
    const int j = i >> 4, c = i & 15;  // 16 chunks of 8 dims per row
    uint4 v = make_uint4(0, 0, 0, 0);
    if (j < nq)
      v = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(b) * nq + j) * (p.n_heads * kHd) + h * kHd + c * 8);
    const int kb = c >> 3, cc = c & 7;
    *reinterpret_cast<uint4*>(q_mma + kb * (kQRows * 128) + j * 128 + ((cc ^ (j & 7)) << 4)) = v;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the MMA reads the queries through the async proxy
  __syncthreads();

  const int g = tid & 31, kg = tid >> 5;  // PV: dims [4g, 4g+4), positions kg, kg+4, ...
  const float scale = p.scale;
  // QK on the tensor core: S[128 x 16] = K_tile[128 x 128] . Q[16 x 128]^T with
  // the tile's 64 positions in rows 0-63 (rows 64-127 read the next 8 KB of
  // the stage and are ignored), fp32 in TMEM lanes = positions.
  const uint32_t idesc = idesc_bf16_f32(128, kQRows);
  float m[NQ], l_part[NQ], o[4][NQ];
#pragma unroll
  for (int j = 0; j < NQ; ++j) {
    m[j] = -__int_as_float(0x7f800000);
    l_part[j] = 0.f;
#pragma unroll
    for (int d = 0; d < 4; ++d) o[d][j] = 0.f;
  }

  bool ok = true;
  for (int t = 0; t < ntiles; ++t) {
    const int st = t % STAGES;
    const uint8_t* kt = smem + st * 2 * kTileBytes;
    const uint8_t* vt = kt + kTileBytes;
    if (!mbar_wait(&full_bar[st], static_cast<uint32_t>((t / STAGES) & 1), &abort_s, p.err, deadline)) ok = false;
    tc_fence_before();
    __syncthreads();
    if (abort_s) break;  // uniform after the barrier
    const int tk0 = k0 + t * kTile;
    const int nk = min(kTile, k1 - tk0);  // valid positions in this tile
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ka = smem_u32(kt), qb = smem_u32(q_mma);
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_bf16(tmem, smem_desc_k128(ka + kb * (kTile * 128) + kk * 32),
                      smem_desc_k128(qb + kb * (kQRows * 128) + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
      tc_commit(&s_bar);
    }

    // ---- scores: s_j = (q_j . k) * scale, -inf where position > ctx + j ----
    const int key = tid;  // warps 0-1: position `key` of the tile (TMEM lane)
    float s[NQ];
    if (warp < 2) {
      if (!mbar_wait(&s_bar, static_cast<uint32_t>(t & 1), &abort_s, p.err, deadline)) ok = false;
      tc_fence_after();
      uint32_t r[kQRows];
      tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16), r);
      tmem_ld_wait();
      const int pos = tk0 + key;
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        const bool vis = key < nk && j < nq && pos <= ctx + j;
        s[j] = vis ? __uint_as_float(r[j]) * scale : -__int_as_float(0x7f800000);
        float v = s[j];
#pragma unroll
        for (int o2 = 1; o2 < 32; o2 <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o2));
        if (lane == 0) red_s[warp][j] = v;
      }
    }
    tc_fence_before();
    __syncthreads();
    if (abort_s) break;
    float alpha[NQ];
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      const float tm = fmaxf(red_s[0][j], red_s[1][j]);
      const float mn = fmaxf(m[j], tm);
      const bool none = (mn == -__int_as_float(0x7f800000));  // nothing visible yet for this query
      alpha[j] = none ? 1.f : expf(m[j] - mn);
      if (warp < 2) {
        const float pj = (none || s[j] == -__int_as_float(0x7f800000)) ? 0.f : expf(s[j] - mn);
        l_part[j] = l_part[j] * alpha[j] + pj;
        p_s[key * NQ + j] = pj;
      }
      m[j] = mn;
    }
    __syncthreads();

    // ---- o += p . v over this tile's valid positions ----
#pragma unroll
    for (int d = 0; d < 4; ++d)
#pragma unroll
      for (int j = 0; j < NQ; ++j) o[d][j] *= alpha[j];
  const int vhalf = g >> 4, vchunk = (g & 15) >> 1, vsub = (g & 1) * 8;
    for (int kk = kg; kk < nk; kk += 4) {
      const uint2 vv = *reinterpret_cast<const uint2*>(tile_chunk(vt, kk, vhalf, vchunk) + vsub);
      const float vf[4] = {__uint_as_float(vv.x << 16), __uint_as_float(vv.x & 0xFFFF0000u),
                           __uint_as_float(vv.y << 16), __uint_as_float(vv.y & 0xFFFF0000u)};
      float pk[NQ];
      if constexpr (NQ >= 4) {
#pragma unroll
        for (int j = 0; j < NQ; j += 4) {
          const float4 p4 = *reinterpret_cast<const float4*>(p_s + kk * NQ + j);
          pk[j] = p4.x;
          pk[j + 1] = p4.y;
          pk[j + 2] = p4.z;
          pk[j + 3] = p4.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < NQ; ++j) pk[j] = p_s[kk * NQ + j];
      }
#pragma unroll
      for (int d = 0; d < 4; ++d)
#pragma unroll
        for (int j = 0; j < NQ; ++j) o[d][j] = fmaf(pk[j], vf[d], o[d][j]);
    }
    __syncthreads();  // every thread is done with this stage and with p_s
    if (tid == 0 && issued < ntiles) {
      fence_proxy_async_smem();  // order the reads of this stage before the copy that refills it
      issue(issued);
      ++issued;
    }
  }

  // No MMA is issued after the loop: wait for the last ones, then free TMEM.
  if (tid == 0) {
    tc_commit(&done_bar);
    int dummy = 0;
    mbar_wait(&done_bar, 0, &dummy, p.err, globaltimer_ns() + kDrainNs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 32);

  if (!ok || abort_s) {
    // Drain: every issued copy must land before the CTA exits.
    if (tid == 0) {
      const uint64_t dl = globaltimer_ns() + kDrainNs;
      int dummy = 0;
      for (int t = max(0, issued - STAGES); t < issued; ++t)
        mbar_wait(&full_bar[t % STAGES], static_cast<uint32_t>((t / STAGES) & 1), &dummy, p.err, dl);
    }
    __syncthreads();
    return;
  }

  // ---- reduce l over positions and o over the four position groups (fixed order) ----
  float* o_red = reinterpret_cast<float*>(smem);  // [4][NQ][128]; the ring is idle now
#pragma unroll
  for (int j = 0; j < NQ; ++j) {
    float v = l_part[j];
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o2);
    l_part[j] = v;
  }
  __syncthreads();
  if (lane == 0)
#pragma unroll
    for (int j = 0; j < NQ; ++j) red_s[warp][j] = l_part[j];
#pragma unroll
  for (int d = 0; d < 4; ++d)
#pragma unroll
    for (int j = 0; j < NQ; ++j) o_red[(kg * NQ + j) * kHd + 4 * g + d] = o[d][j];
  __syncthreads();
  const int dim = tid;  // one output dim per thread
  float lsum[NQ], osum[NQ];
#pragma unroll
  for (int j = 0; j < NQ; ++j) {
    lsum[j] = ((red_s[0][j] + red_s[1][j]) + red_s[2][j]) + red_s[3][j];
    osum[j] = ((o_red[(0 * NQ + j) * kHd + dim] + o_red[(1 * NQ + j) * kHd + dim]) + o_red[(2 * NQ + j) * kHd + dim]) +
              o_red[(3 * NQ + j) * kHd + dim];
  }
  const size_t ld_out = static_cast<size_t>(p.n_heads) * kHd;
  if (n_split_b == 1) {
#pragma unroll
    for (int j = 0; j < NQ; ++j)
      if (j < nq) p.out[(static_cast<size_t>(b) * nq + j) * ld_out + h * kHd + dim] = f32_to_bf16_bits(osum[j] / lsum[j]);
    return;
  }
  // several splits: write this split's (m, l, o), the last CTA of the pair merges them
  const size_t pair = static_cast<size_t>(b) * p.n_heads + h;
  float* po = p.part_o + (pair * p.n_split + split) * NQ * kHd;
  float* pml = p.part_ml + (pair * p.n_split + split) * NQ * 2;
#pragma unroll
  for (int j = 0; j < NQ; ++j) po[j * kHd + dim] = osum[j];
#pragma unroll
  for (int j = 0; j < NQ; ++j)
    if (tid == j) {  // (a loop, not m[tid]: register arrays take constant indices)
      pml[2 * j] = m[j];
      pml[2 * j + 1] = lsum[j];
    }
  __threadfence();
  __syncthreads();
  if (tid == 0) last_s = (atomicAdd(p.counters + pair, 1) == n_split_b - 1) ? 1 : 0;
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  const float* po0 = p.part_o + pair * p.n_split * NQ * kHd;
  const float* pml0 = p.part_ml + pair * p.n_split * NQ * 2;
#pragma unroll
  for (int j = 0; j < NQ; ++j) {
    if (j >= nq) continue;
    float M = -__int_as_float(0x7f800000);
    for (int sp = 0; sp < n_split_b; ++sp) M = fmaxf(M, __ldcg(pml0 + (sp * NQ + j) * 2));
    float L = 0.f, O = 0.f;
    for (int sp = 0; sp < n_split_b; ++sp) {
      const float ms = __ldcg(pml0 + (sp * NQ + j) * 2);
      const float w = (ms == -__int_as_float(0x7f800000)) ? 0.f : expf(ms - M);
      L = fmaf(w, __ldcg(pml0 + (sp * NQ + j) * 2 + 1), L);
      O = fmaf(w, __ldcg(po0 + (sp * NQ + j) * kHd + dim), O);
    }
    p.out[(static_cast<size_t>(b) * nq + j) * ld_out + h * kHd + dim] = f32_to_bf16_bits(O / L);
  }
  if (tid == 0) p.counters[pair] = 0;  // ready for the next call on this workspace
}

// Dynamic shared memory of one CTA: the tile ring, the queries, the weights.
static size_t attention_smem(int nq_t, int stages) {
  return static_cast<size_t>(stages) * 2 * kTileBytes + static_cast<size_t>(2) * kQRows * 128 +
         static_cast<size_t>(kTile) * nq_t * 4 + 1024;
}

template <int NQ, int STAGES>
static cudaError_t launch_attention_t(const AttnParams& p, int B, cudaStream_t s) {
  auto kern = decode_attention_kernel<NQ, STAGES>;
  const size_t smem = attention_smem(NQ, STAGES);
  static thread_local int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_dev = dev;
  }
  return launch_pdl(kern, dim3(p.n_split, p.n_heads, B), dim3(kAttnThreads), smem, s, p);
}

int attention_nq(int K) {
  const int nq = K + 1;
  return nq <= 1 ? 1 : nq <= 2 ? 2 : nq <= 4 ? 4 : nq <= 8 ? 8 : 0;
}

cudaError_t launch_decode_attention(const AttnParams& p, int B, cudaStream_t s) {
  constexpr int kStages = 2;
  switch (attention_nq(p.K)) {
    case 1: return launch_attention_t<1, kStages>(p, B, s);
    case 2: return launch_attention_t<2, kStages>(p, B, s);
    case 4: return launch_attention_t<4, kStages>(p, B, s);
    case 8: return launch_attention_t<8, kStages>(p, B, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace mv
