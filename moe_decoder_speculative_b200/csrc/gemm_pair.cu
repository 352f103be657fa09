// Grouped tensor-core GEMM on CTA pairs (tcgen05 cta_group::2) for the large
// token groups of a prefill-sized MoE layer (8 pages x 1,156 visual tokens:
// about 870 rows per routed expert; jina-ocr-v1 model card, architecture
// paragraph: 64 routed + 2 shared SwiGLU experts), and for the LM head of 256
// or more rows (129,280-token vocabulary, same paragraph), where each
// vocabulary tile serves several token tiles and the tensor core bounds it.
//
// Why pairs.  With one CTA per tile (128 tokens x 256 weight rows) every
// 64-wide k-block writes 48 KB into shared memory and the MMAs read the same
// 48 KB back: at 128 bytes per clock of shared-memory bandwidth that is more
// time than the tensor core needs for the k-block (a 128x256x16 MMA took ~230
// clocks against 128).  A cluster of two CTAs multiplies a 256-token x
// 256-weight-row tile: each CTA loads its own 128 token rows and HALF of the
// weight rows, and one MMA stream (issued by the even CTA) reads both CTAs'
// shared memory.  Per SM that is 32 KB per k-block instead of 48, which the
// shared-memory port can feed at the tensor core's rate.
//
// Roles (6 warps, both CTAs unless noted):
//   warp 0      TMA producer: own token rows + own half of the weights, two
//               64-wide k-blocks per stage through 3D tensor maps; the
//               transaction bytes of BOTH CTAs complete the even CTA's full
//               barrier (cta_group::2 loads), no multicast
//   warp 1      TMEM allocation (cta_group::2, both CTAs); MMA issue (even
//               CTA only): M = 256 (128 rows per CTA), N = 256 (128 per CTA)
//   warps 2..5  epilogue on this CTA's 128 token rows x 256 columns (gate|up
//               -> SwiGLU, or two halves of W_down -> fp32 rows, or 256 LM-head
//               rows -> one argmax key per token)
// Units (group, M tile, 256-token tile) are assigned statically: cluster c
// takes c, c + clusters, c + 2 clusters, ...  A down unit waits (bounded
// acquire-poll) until every epilogue warp of both CTAs of every unit of its
// expert's gate/up group has signalled; units only wait on earlier units and
// every cluster is resident (the grid is sized to the resident count), so the
// waits always end.  Every wait is bounded; a CTA that gives up drains its
// copies and MMAs, and both CTAs meet at the final cluster barrier before
// TMEM is freed and either exits.

#include "mv_device.cuh"
#include "mv_internal.h"

namespace mv {

namespace {

constexpr int kPairThreads = 192;
constexpr int kHalfTile = 128 * 128;           // 128 rows x 64 bf16 (one k-block)
constexpr int kKB = kPairKB;                   // k-blocks per stage
constexpr int kPairStageBytes = 2 * kKB * kHalfTile;  // A: kKB k-blocks x 128 rows, B: the same
constexpr int kPairStages = 6 / kKB;           // 192 KB of stages
constexpr int kPairTok = 256;                  // token rows per unit (128 per CTA)
constexpr int kAccCols = 256;                  // one accumulator: 256 columns; two of them
constexpr int kPairTBufBytes = 4 * 32 * 33 * 4;  // fp32 32 x 33 transpose buffer per epilogue warp

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// 2D tiled TMA load into this CTA's shared memory whose completion counts on
// the barrier at `bar_cluster` (the even CTA's), for a CTA-pair MMA.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* m, int32_t x, int32_t y,
                                                 uint32_t bar_cluster, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(bar_cluster), "l"(policy)
      : "memory");
}

// 3D tiled TMA load into this CTA's shared memory whose completion counts on
// the barrier at `bar_cluster` (the even CTA's), for a CTA-pair MMA.
__device__ __forceinline__ void tma_load_3d_pair(void* smem_dst, const CUtensorMap* m, int32_t x, int32_t y,
                                                 int32_t z, uint32_t bar_cluster, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z), "r"(bar_cluster), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on this CTA's barrier when every tcgen05 operation issued so
// far by this thread (CTA-pair MMAs included) has completed.
__device__ __forceinline__ void tc_commit_pair_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Arrive (once) on the barrier at this offset in both CTAs of the pair when
// every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit_pair_both(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

struct PairUnit {
  int set, g, gi, m0, nvalid, b_row0;
};

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    gemm_pair_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kPairStages];
  __shared__ __align__(8) uint64_t empty_bar[kPairStages];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t mma_done_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int g_begin[kMaxGroups + 1];
  __shared__ int g_rows[kMaxGroups];
  __shared__ int g_row0[kMaxGroups];
  __shared__ short g_nt[kMaxGroups];
  __shared__ unsigned char g_set[kMaxGroups];
  __shared__ short g_gi[kMaxGroups];
  __shared__ int set_base[5];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int cluster = static_cast<int>(blockIdx.x) >> 1;
  const int nclusters = static_cast<int>(gridDim.x) >> 1;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;

  pdl_trigger();
  if (tid == 0) {
    abort_s = 0;
    for (int i = 0; i < kPairStages; ++i) {
      mbar_init(&full_bar[i], 1);   // the even CTA's producer arms it; both CTAs' loads complete it
      mbar_init(&empty_bar[i], 1);  // the MMA commit, multicast to both CTAs
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);   // the MMA commit, multicast
      mbar_init(&tempty_bar[i], 8);  // 4 epilogue warps of each CTA (even CTA's barrier)
    }
    mbar_init(&mma_done_bar, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < p.nsets; ++s) {
      tma_prefetch_desc(&p.set[s].a0);
      tma_prefetch_desc(&p.set[s].a1);
      tma_prefetch_desc(&p.set[s].b);
    }
  }
  if (warp == 1) tmem_alloc_pair(&tmem_base_s, 2 * kAccCols);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers and TMEM exist before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  if (warp == 1) tmem_relinquish_pair();

  pdl_wait();  // the group sizes and the token rows come from the previous kernels

  // ---- group table (every CTA builds the same one) ------------------------
  if (tid == 0) {
    int b = 0;
    for (int s = 0; s < p.nsets; ++s) {
      set_base[s] = b;
      b += p.set[s].groups;
    }
    set_base[p.nsets] = b;
  }
  __syncthreads();
  const int ng = set_base[p.nsets];
  for (int g = tid; g < ng; g += kPairThreads) {
    int s = 0;
    while (g >= set_base[s + 1]) ++s;
    const int gi = g - set_base[s];
    const GemmSet& S = p.set[s];
    int rows = S.counts ? __ldcg(S.counts + gi) : S.static_rows;
    if (S.slab_rows > 0 && rows > S.slab_rows) rows = S.slab_rows;  // a slab never holds more
    g_rows[g] = rows;
    g_row0[g] = S.offsets ? __ldcg(S.offsets + gi) : gi * S.slab_rows;
    g_set[g] = static_cast<unsigned char>(s);
    g_gi[g] = static_cast<short>(gi);
    const int mt = (S.M + S.m_tile - 1) / S.m_tile;
    const int nt = rows > 0 ? (rows + kPairTok - 1) / kPairTok : 0;
    g_nt[g] = static_cast<short>(nt);
    g_begin[g + 1] = mt * nt;
  }
  if (tid == 0) g_begin[0] = 0;
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < ng; base += 32) {
      const int g = base + lane;
      int v = (g < ng) ? g_begin[g + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
      }
      if (g < ng) g_begin[g + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  __syncthreads();
  const int total_units = g_begin[ng];
  auto decode = [&](int u) -> PairUnit {
    int lo = 0, hi = ng;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (g_begin[mid] <= u) lo = mid; else hi = mid;
    }
    const int local = u - g_begin[lo];
    const int nt = g_nt[lo];
    PairUnit ui;
    ui.g = lo;
    ui.set = g_set[lo];
    ui.gi = g_gi[lo];
    ui.m0 = (local / nt) * p.set[ui.set].m_tile;
    const int n0 = (local % nt) * kPairTok;
    ui.nvalid = min(kPairTok, g_rows[lo] - n0);
    ui.b_row0 = g_row0[lo] + n0;
    return ui;
  };
  const int my_units = total_units > cluster ? (total_units - cluster + nclusters - 1) / nclusters : 0;
  auto unit_stages = [&](const GemmSet& S) { return (S.K / 64 + kKB - 1) / kKB; };

  if (warp == 0) {
    // ========================= TMA producer ==================================
    if (lane == 0) {
      // Weights stream once per token tile: kept in L2 (evict-last) when
      // three or more token tiles of the group read the same weight tile, so
      // the later readers hit; streamed through (evict-first) otherwise.
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      const uint32_t full0 = map_to_rank(&full_bar[0], 0);  // the even CTA's barriers
      int stage = 0;
      uint32_t phase = 0;
      int fills[kPairStages] = {};
      bool ok = true;
      for (int it = 0; it < my_units && ok; ++it) {
        const PairUnit ui = decode(cluster + it * nclusters);
        const GemmSet& S = p.set[ui.set];
        if (S.dep_set >= 0) {  // a down unit: its expert's gate/up group must be complete
          const int gd = set_base[S.dep_set] + ui.gi;
          const int target = 8 * (g_begin[gd + 1] - g_begin[gd]);
          while (ld_acquire(p.sched + 1 + gd) < target) {
            __nanosleep(64);
            if (*static_cast<volatile int*>(&abort_s) || globaltimer_ns() > deadline) {
              if (!abort_s) {
                abort_s = 1;
                atomicOr(p.err, kErrTimeout);
              }
              ok = false;
              break;
            }
          }
          if (!ok) break;
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        const int nstage = unit_stages(S);
        const uint64_t pol_w = g_nt[ui.g] >= 3 ? pol_x : pol_stream;
        const bool gu = (S.mode == MODE_TGATEUP);
        // this CTA's weight rows: gate (even) / up (odd) of the 128-feature
        // tile, or the even / odd 128-row half of a 256-row W_down tile
        const CUtensorMap* wmap = (gu && !leader) ? &S.a1 : &S.a0;
        const int w_row = ui.gi * S.a_group_stride + ui.m0 + (gu ? 0 : 128 * static_cast<int>(rank));
        const int t_row = ui.b_row0 + 128 * static_cast<int>(rank);
        for (int ks = 0; ks < nstage; ++ks) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_s, p.err, deadline)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * kPairStageBytes;
          // both CTAs' A and B boxes (a box past the last k-block is zero-filled and still counts)
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2u * kPairStageBytes);
          if (kKB == 2) {  // one 3D box brings two k-blocks
            tma_load_3d_pair(st, &S.b, 0, t_row, 2 * ks, full0 + stage * 8, pol_x);
            tma_load_3d_pair(st + kKB * kHalfTile, wmap, 0, w_row, 2 * ks, full0 + stage * 8, pol_w);
          } else {
            tma_load_2d_pair(st, &S.b, ks * 64, t_row, full0 + stage * 8, pol_x);
            tma_load_2d_pair(st + kKB * kHalfTile, wmap, ks * 64, w_row, full0 + stage * 8, pol_w);
          }
          fills[stage]++;
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: the even CTA waits until every armed stage has landed (its
      // barriers count both CTAs' bytes); the final cluster barrier keeps the
      // odd CTA alive until then.
      if (leader) {
        const uint64_t dl = globaltimer_ns() + kDrainNs;
        for (int i = 0; i < kPairStages; ++i)
          if (fills[i] > 0) {
            int dummy = 0;
            mbar_wait(&full_bar[i], static_cast<uint32_t>((fills[i] - 1) & 1), &dummy, p.err, dl);
          }
      }
    }
  } else if (warp == 1) {
    // ========================= MMA issuer (even CTA) ========================
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      // M = 256 (128 rows per CTA), N = 256 (128 weight rows per CTA)
      const uint32_t idesc = idesc_bf16_f32(256, 256);
      for (int it = 0; it < my_units && ok; ++it) {
        const PairUnit ui = decode(cluster + it * nclusters);
        const GemmSet& S = p.set[ui.set];
        const int slot = it & 1;
        if (!mbar_wait(&tempty_bar[slot], ((it >> 1) & 1) ^ 1u, &abort_s, p.err, deadline)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(slot * kAccCols);
        const int kblocks = S.K / 64;
        const int nstage = unit_stages(S);
        for (int ks = 0; ks < nstage; ++ks) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_s, p.err, deadline)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + stage * kPairStageBytes);
#pragma unroll
          for (int h = 0; h < kKB; ++h) {
            if (h > 0 && kKB * ks + h >= kblocks) break;
            const uint32_t a = st + h * kHalfTile;            // token rows, k-block h
            const uint32_t b = st + (kKB + h) * kHalfTile;    // weight rows, k-block h
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma_pair(d0, smem_desc_k128(a + kk * 32), smem_desc_k128(b + kk * 32), idesc,
                          (ks | h | kk) != 0 ? 1u : 0u);
          }
          tc_commit_pair_both(&empty_bar[stage]);
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_both(&tfull_bar[slot]);
      }
      tc_commit_pair_local(&mma_done_bar);
      int dummy = 0;
      mbar_wait(&mma_done_bar, 0, &dummy, p.err, globaltimer_ns() + kDrainNs);
    }
  } else {
    // ========================= epilogue (warps 2..5, both CTAs) ==============
    const int wq = warp & 3;
    float* tbuf = reinterpret_cast<float*>(smem + kPairStages * kPairStageBytes);
    const uint32_t tempty0 = map_to_rank(&tempty_bar[0], 0);
    for (int it = 0; it < my_units; ++it) {
      const PairUnit ui = decode(cluster + it * nclusters);
      const GemmSet& S = p.set[ui.set];
      const int slot = it & 1;
      if (!mbar_wait(&tfull_bar[slot], (it >> 1) & 1, &abort_s, p.err, deadline)) break;
      tc_fence_after();
      const int row = wq * 32 + lane;  // this CTA's token row of the unit
      const int nvalid = ui.nvalid - 128 * static_cast<int>(rank);
      const bool tvalid = row < nvalid;
      const size_t orow = static_cast<size_t>(ui.b_row0 + 128 * static_cast<int>(rank) + row) * S.ld_out;
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + static_cast<uint32_t>(slot * kAccCols);
      if (S.epi == EPI_SWIGLU_ROWS) {
        uint16_t* out = static_cast<uint16_t*>(S.out);
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t g[32], v[32];
          tmem_ld32(tl + c0, g);
          tmem_ld32(tl + 128 + c0, v);
          tmem_ld_wait();
          if (tvalid && ui.m0 + c0 < S.M) {
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float a2[2];
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const float gf = __uint_as_float(g[2 * j + q]);
                const float uf = __uint_as_float(v[2 * j + q]);
                // silu(g) * u = g u / (1 + e^-g) with the fast exponential and
                // division (a few ulp of fp32, far below the bf16 rounding of a);
                // the IEEE forms made this epilogue the kernel's bottleneck
                a2[q] = __fdividef(gf * uf, 1.0f + __expf(-gf));
              }
              packed[j] = static_cast<uint32_t>(f32_to_bf16_bits(a2[0])) |
                          (static_cast<uint32_t>(f32_to_bf16_bits(a2[1])) << 16);
            }
            uint4* dst = reinterpret_cast<uint4*>(out + orow + ui.m0 + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
          }
        }
      } else if (S.epi == EPI_STORE_ROWS) {
        // fp32 rows, written line by line: the warp's 32 rows x 32 columns
        // pass through a padded buffer (row writes and column reads both
        // bank-conflict-free), then each store instruction writes one row's
        // 32 columns, a whole 128-byte line, instead of 16 bytes of 32 rows.
        float* out = static_cast<float*>(S.out);
        float* tb = tbuf + wq * (32 * 33);
        const int row_base = ui.b_row0 + 128 * static_cast<int>(rank) + wq * 32;
        const int rows_here = min(32, nvalid - wq * 32);  // valid rows of this warp (may be <= 0)
        for (int c0 = 0; c0 < 256; c0 += 32) {
          uint32_t d[32];
          tmem_ld32(tl + c0, d);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) tb[lane * 33 + j] = __uint_as_float(d[j]);
          __syncwarp();
          const int col = ui.m0 + c0 + lane;
          if (col < S.M)
            for (int r = 0; r < rows_here; ++r)
              out[static_cast<size_t>(row_base + r) * S.ld_out + col] = tb[r * 33 + lane];
          __syncwarp();
        }
      } else if (S.epi == EPI_ARGMAX_ROWS) {
        // LM head: this thread's token row holds the logits of vocabulary rows
        // m0 .. m0 + 255 (this CTA's 128 and the other CTA's 128).  Per group
        // of 32 rows: the first row's logit, then any strictly larger one (so
        // the lowest index among equal maxima), packed with its index into a
        // key (larger logit first, then lower index); rows past the vocabulary
        // count as -inf.  The largest of the 8 keys is the unit's; tokens
        // reduce their keys over all units afterwards.
        uint64_t best_key = 0;
        for (int c0 = 0; c0 < 256; c0 += 32) {
          uint32_t d[32];
          tmem_ld32(tl + c0, d);
          tmem_ld_wait();
          const int v0 = ui.m0 + c0;
          float best = v0 < S.M ? __uint_as_float(d[0]) : -__int_as_float(0x7f800000);
          int bi = 0;
#pragma unroll
          for (int j = 1; j < 32; ++j) {
            const float x = (v0 + j < S.M) ? __uint_as_float(d[j]) : -__int_as_float(0x7f800000);
            if (x > best) {
              best = x;
              bi = j;
            }
          }
          const uint64_t key = argmax_key(best, static_cast<uint32_t>(S.key_row_base + v0 + bi));
          best_key = key > best_key ? key : best_key;
        }
        if (tvalid) static_cast<uint64_t*>(S.out)[orow + S.key_part_base + ui.m0 / 256] = best_key;
      } else if (lane == 0) {
        atomicOr(p.err, kErrInternal);  // a set this kernel is not built for
      }
      // hand the accumulator slot back to the even CTA's MMA issuer
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty0 + slot * 8);
      if (S.signal && p.sched) {  // release this warp's stores to the units that depend on the group
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          atomicAdd(p.sched + 1 + ui.g, 1);
        }
      }
      __syncwarp();
    }
  }

  // ---- teardown: both CTAs meet before TMEM is freed or either exits -------
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 2 * kAccCols);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// The stage ring, the epilogue warps' 32 x 33 transpose buffers, alignment.
static size_t pair_smem() { return static_cast<size_t>(kPairStages) * kPairStageBytes + kPairTBufBytes + 1024; }

static cudaError_t pair_configure(int dev) {
  static thread_local int configured_dev = -1;
  if (configured_dev == dev) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(pair_smem()));
  if (e != cudaSuccess) return e;
  configured_dev = dev;
  return cudaSuccess;
}

int gemm_pair_max_clusters() {
  static thread_local int cached_dev = -1, cached = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cached_dev == dev) return cached;
  if (pair_configure(dev) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = pair_smem();
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cached_dev = dev;
  cached = n;
  return n;
}

cudaError_t launch_gemm_pair(const GemmParams& p, int clusters, cudaStream_t stream) {
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t e = pair_configure(dev);
  if (e != cudaSuccess) return e;
  return launch_pdl(gemm_pair_kernel, dim3(2 * clusters), dim3(kPairThreads), pair_smem(), stream, p);
}

}  // namespace mv
