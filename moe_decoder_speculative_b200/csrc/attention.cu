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
// ridge, so this is a streaming kernel bound by HBM; the MMAs only keep the
// per-tile instruction count (and so the latency chain) short.
// Layout and work split:
//   * cache [B][heads][L_max][128] bf16 (head-major), so a tile of 64
//     positions of one (sequence, head) is 16 KB of contiguous rows; one TMA
//     load of a [k-half][row][64] view brings a K or V tile into shared
//     memory with the 128-byte swizzle (bank-conflict-free row reads);
//   * CTA (split, head, sequence) streams its split of the positions through
//     a ring of STAGES tiles with an online softmax in fp32;
//   * QK on the tensor core: the tile's K rows are the A operand of an
//     M = 128 MMA, the queries (padded to 16 rows) the B operand, the scores
//     land in TMEM and warps 0-1 read them (one position per thread);
//   * PV on the tensor cores too, as warp-level MMAs (mma.sync m16n8k16, fp32
//     accumulators in registers): V^T tiles straight from the swizzled stage
//     (ldmatrix.trans), the softmax weights as two bf16 parts (high and the
//     rounding remainder, summing to the fp32 weight within 2^-18 of it), so
//     the products keep fp32 accuracy; warp w owns output dims [32w, 32w+32);
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
constexpr int kPRow = kTile + 8;  // bf16 elements per row of the softmax-weight buffers
constexpr int kQRows = 16;        // the queries padded to the MMA's N (16)

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace

template <int NQ, int STAGES>
__global__ void __launch_bounds__(kAttnThreads) decode_attention_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // the queries as the MMA's B operand: bf16 [2 k-blocks][16 rows][64], 128-byte swizzle
  uint8_t* q_mma = smem + STAGES * 2 * kTileBytes;
  // the tile's softmax weights as bf16 high and low parts, [8 queries][64
  // positions] each, rows kPRow elements apart (16 bytes of padding: the PV
  // fragment loads of the 8 queries then hit 8 different bank groups)
  uint16_t* p_hi = reinterpret_cast<uint16_t*>(q_mma + 2 * kQRows * 128);
  uint16_t* p_lo = p_hi + 8 * kPRow;
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

  // PV on the tensor cores (mma.sync m16n8k16, fp32 accumulators): warp w
  // owns output dims [32w, 32w + 32) as two 16-dim tiles; thread (gq, tq) of
  // a tile holds dims gq, gq + 8 for queries 2 tq, 2 tq + 1.
  const int gq = lane >> 2, tq = lane & 3;
  const float scale = p.scale;
  // QK on the tensor core: S[128 x 16] = K_tile[128 x 128] . Q[16 x 128]^T with
  // the tile's 64 positions in rows 0-63 (rows 64-127 read the next 8 KB of
  // the stage and are ignored), fp32 in TMEM lanes = positions.
  const uint32_t idesc = idesc_bf16_f32(128, kQRows);
  float m[NQ], l_part[NQ], o[2][4];
#pragma unroll
  for (int j = 0; j < NQ; ++j) {
    m[j] = -__int_as_float(0x7f800000);
    l_part[j] = 0.f;
  }
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int q = 0; q < 4; ++q) o[t][q] = 0.f;

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
        // bf16 high and low parts: p_hi + p_lo = pj to 2^-18 of it
        const uint16_t hi = f32_to_bf16_bits(pj);
        p_hi[j * kPRow + key] = hi;
        p_lo[j * kPRow + key] = f32_to_bf16_bits(pj - bf16_bits_to_f32(hi));
      }
      m[j] = mn;
    }
    if (nk < kTile) {  // the rows past the split (never visible) may hold anything: zero them for the MMAs
      uint8_t* vz = const_cast<uint8_t*>(vt);
      for (int i = tid; i < (kTile - nk) * 16; i += kAttnThreads) {
        const int r = nk + (i >> 4), c = i & 15;  // row r, 16-byte chunk c of the two 64-dim halves
        *reinterpret_cast<uint4*>(vz + (c >> 3) * (kTile * 128) + r * 128 + (c & 7) * 16) = make_uint4(0, 0, 0, 0);
      }
    }
    __syncthreads();

    // ---- o = o * alpha + P V^T on the tensor cores ----
    {
      float a_lo = 1.f, a_hi = 1.f;  // alpha of queries 2 tq, 2 tq + 1
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        if (j == 2 * tq) a_lo = alpha[j];
        if (j == 2 * tq + 1) a_hi = alpha[j];
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        o[t][0] *= a_lo;
        o[t][1] *= a_hi;
        o[t][2] *= a_lo;
        o[t][3] *= a_hi;
      }
      const uint32_t vbase = smem_u32(vt);
      const int li = lane >> 3;  // the 8 x 8 matrix this lane addresses: dims + 8 (li & 1), positions + 8 (li >> 1)
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks) {
        uint32_t bh0 = 0, bh1 = 0, bl0 = 0, bl1 = 0;  // P^T: positions 16 ks + 2 tq (+1) and +8, query gq
        if (gq < NQ) {
          const int pp = gq * kPRow + 16 * ks + 2 * tq;
          bh0 = *reinterpret_cast<const uint32_t*>(p_hi + pp);
          bh1 = *reinterpret_cast<const uint32_t*>(p_hi + pp + 8);
          bl0 = *reinterpret_cast<const uint32_t*>(p_lo + pp);
          bl1 = *reinterpret_cast<const uint32_t*>(p_lo + pp + 8);
        }
        const int pos = 16 * ks + 8 * (li >> 1) + (lane & 7);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int dim = warp * 32 + t * 16 + 8 * (li & 1);
          const uint32_t addr = vbase + static_cast<uint32_t>((dim >> 6) * (kTile * 128) + pos * 128) +
                                static_cast<uint32_t>((((dim & 63) >> 3) ^ (pos & 7)) << 4);
          uint32_t a0, a1, a2, a3;  // V^T: dims x positions
          asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                       : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                       : "r"(addr));
          asm volatile(
              "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
              "{%0, %1, %2, %3};"
              : "+f"(o[t][0]), "+f"(o[t][1]), "+f"(o[t][2]), "+f"(o[t][3])
              : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(bh0), "r"(bh1));
          asm volatile(
              "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
              "{%0, %1, %2, %3};"
              : "+f"(o[t][0]), "+f"(o[t][1]), "+f"(o[t][2]), "+f"(o[t][3])
              : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(bl0), "r"(bl1));
        }
      }
    }
    __syncthreads();  // every thread is done with this stage and with the weights
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

  // ---- l over positions (fixed order); each thread's outputs are already whole ----
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
  __syncthreads();
  float lsum[NQ];
#pragma unroll
  for (int j = 0; j < NQ; ++j) lsum[j] = ((red_s[0][j] + red_s[1][j]) + red_s[2][j]) + red_s[3][j];
  const size_t ld_out = static_cast<size_t>(p.n_heads) * kHd;
  if (n_split_b == 1) {
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int dim = warp * 32 + t * 16 + gq + (q >= 2 ? 8 : 0), j = 2 * tq + (q & 1);
        if (j < nq) {
          const float lj = ((red_s[0][j] + red_s[1][j]) + red_s[2][j]) + red_s[3][j];
          p.out[(static_cast<size_t>(b) * nq + j) * ld_out + h * kHd + dim] = f32_to_bf16_bits(o[t][q] / lj);
        }
      }
    return;
  }
  // several splits: write this split's (m, l, o), the last CTA of the pair merges them
  const size_t pair = static_cast<size_t>(b) * p.n_heads + h;
  float* po = p.part_o + (pair * p.n_split + split) * NQ * kHd;
  float* pml = p.part_ml + (pair * p.n_split + split) * NQ * 2;
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int dim = warp * 32 + t * 16 + gq + (q >= 2 ? 8 : 0), j = 2 * tq + (q & 1);
      if (j < NQ) po[j * kHd + dim] = o[t][q];
    }
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
  const int dim = tid;  // the merge: one output dim per thread
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

// Dynamic shared memory of one CTA: the tile ring, the queries, the weights (bf16 high and low parts).
static size_t attention_smem(int nq_t, int stages) {
  (void)nq_t;
  return static_cast<size_t>(stages) * 2 * kTileBytes + static_cast<size_t>(2) * kQRows * 128 +
         static_cast<size_t>(2) * 8 * kPRow * 2 + 1024;
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
