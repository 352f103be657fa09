// Grouped tensor-core GEMM engine for sm_100a (tcgen05 + TMEM + TMA).
//
// One launch computes, for every group g of up to four operand sets,
//     D_g[m][n] = sum_k A_g[m][k] * B_g[n][k]          (bf16 x bf16 -> fp32)
// where A_g is a weight matrix (rows = output features, K-major) and B_g the
// token rows routed to that group (K-major).  Weights sit on the MMA's M side
// (128-row tiles) and tokens on its N side ("swap-AB"), so the few tokens per
// expert of a decode step still fill whole weight tiles; each tile's N extent
// is the group's real row count rounded up to 16.
//
// The contractions of the verify step (jina-ocr-v1 model card, architecture
// paragraph: MoE decoder with 64 routed + 2 shared SwiGLU experts and a
// 129,280-token LM head) map onto operand modes and epilogues:
//   gate/up   MODE_GATEUP: A0 = gate rows, A1 = up rows of the same tile, one
//             B k-block; epilogue EPI_SWIGLU writes a = bf16(silu(g) * u)
//   down      MODE_KPAIR: A0/A1 = two consecutive k-blocks of the same rows,
//             B0/B1 the matching token k-blocks; epilogue EPI_STORE_F32
//   LM head   MODE_MPAIR: A0/A1 = two 128-row vocabulary tiles sharing one B
//             k-block; epilogue EPI_ARGMAX reduces each token column to a
//             packed (logit, lowest index) key per 32 vocabulary rows -- the
//             logits never reach memory
// Every stage therefore moves 32 KB of weights.  For large groups (prefill)
// the same tiles are multiplied tokens-on-M: 128 token rows x 256 weight rows
// (MODE_TGATEUP: gate|up side by side; MODE_TPAIR: two halves of W_down) into
// one 256-column accumulator, which halves the shared-memory operand traffic
// per MMA; its epilogues (EPI_SWIGLU_ROWS, EPI_STORE_ROWS) write whole row
// segments with 16-byte stores.
//
// Scheduling: persistent CTAs (at most one per SM) claim work units (group,
// M tile, N tile) from a global atomic counter in list order -- sets in order,
// largest units first -- and hand them to the MMA and epilogue warps through a
// shared-memory ring.  A set may depend on an earlier one (the down projection
// of expert e on the gate/up of expert e): its units wait, with a bounded
// acquire-poll, until the epilogue warps of every unit of that group have
// released their stores (with few rows, the unit's first stages take their
// weights before that wait).  Claims are in list order and only running CTAs
// claim, so every unit waited on is already held by a running CTA: no
// deadlock whatever the residency.
//
// Warp roles (6 warps):
//   warp 0      TMA producer (one thread) and work claimer
//   warp 1      TMEM allocator and MMA issuer (one thread), 128xNx16 MMAs
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns per warp
// Accumulators are double-buffered in TMEM.  Every wait is bounded (see
// mv_device.cuh); on timeout the CTA drains its copies, frees TMEM and exits
// with the sticky error bit set.  No TMA multicast is used.

#include "mv_device.cuh"
#include "mv_internal.h"

namespace mv {

namespace {

constexpr int kThreads = 192;
constexpr int kATileBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kRing = 4;                // claimed units in flight inside a CTA

struct UnitInfo {
  int set, g, gi, m0, nvalid, b_row0;
};


__device__ __forceinline__ int upper_pow2_cols(int c) {
  int n = 32;
  while (n < c) n <<= 1;
  return n;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

}  // namespace

// DEPW: a unit that must wait for the group it reads from issues its first
// stages' weights before that wait (they do not depend on it).
template <int BN, int STAGES, int NB, bool LM, int BBOX, bool DEPW>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmParams p) {
  constexpr int kBBox = BBOX;  // B rows per TMA box (the B tensor maps are built with this box height)
  static_assert(BBOX % 8 == 0 && BBOX <= BN, "BBOX");
  constexpr int B_TILE_BYTES = BN * 128;
  // Weights-on-M tiles (BN = 32) take two k-blocks per stage through 3D tensor
  // maps: one TMA instruction brings both k-blocks of a 128-row weight tile
  // (or of the token rows).  A TMA instruction costs about 0.25 us of the SM's
  // copy engine whatever its size, which bounds one SM's stream when only a
  // few SMs have work (batch 1, the draft block).  Stage layout: A0 [kb0][kb1],
  // A1 (the up weights) [kb0][kb1], B [kb0][kb1].
  constexpr bool kKB2 = !LM && BN == 32;
  static_assert(!kKB2 || NB == 2, "two B slots per stage");
  constexpr int STAGE_BYTES = (kKB2 ? 4 : 2) * kATileBytes + NB * B_TILE_BYTES;
  constexpr int ACC_COLS = 2 * BN;  // two accumulators (D0, D1) per slot
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 128, "BN");
  static_assert(2 * ACC_COLS <= 512, "TMEM");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t ufull_bar[kRing];
  __shared__ __align__(8) uint64_t uempty_bar[kRing];
  __shared__ __align__(8) uint64_t mma_done_bar;
  __shared__ int unit_ring[kRing];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int g_begin[kMaxGroups + 1];  // first unit of each group
  __shared__ int g_rows[kMaxGroups];
  __shared__ int g_row0[kMaxGroups];
  __shared__ short g_nt[kMaxGroups];
  __shared__ unsigned char g_set[kMaxGroups];
  __shared__ short g_gi[kMaxGroups];
  __shared__ int set_base[5];

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;
  // Each tile configuration compiles only the epilogues it is launched with
  // (a smaller kernel keeps its hot loops in the instruction cache): the
  // weights-on-M tiles (BN = 32) the SwiGLU / fp32 / bf16 stores,
  // the tokens-on-M tiles (BN = 128) the row stores and the router top-k, the
  // LM head the argmax.
  constexpr bool kSwapAB = !LM && BN == 32;
  constexpr bool kTokM = !LM && BN == 128;

  pdl_trigger();
  // ---- set-up that needs nothing from the previous kernel ----------------
  // Barriers, TMEM (one CTA per SM by shared memory, so two GEMM launches
  // never hold TMEM on one SM) and descriptors.
  if (tid == 0) {
    abort_s = 0;
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 4);
    }
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&ufull_bar[i], 1);
      mbar_init(&uempty_bar[i], 5);  // the MMA thread + 4 epilogue warps
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
  const int tmem_cols = upper_pow2_cols(2 * ACC_COLS);
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;

  // TMA issue of one stage of a unit: the weights (A) part with the stage's
  // full byte count, and/or the token-row (B) part.
  const uint64_t pol_w = policy_evict_first();
  const uint64_t pol_x = policy_evict_last();
  auto issue_stage = [&](const GemmSet& S, const UnitInfo& ui, int ks, int stg, bool wts, bool toks) {
    uint8_t* st = smem + stg * STAGE_BYTES;
    uint8_t* b0 = st + 2 * kATileBytes;
    const int a_row0 = ui.gi * S.a_group_stride + ui.m0;
    const int nchunk = (ui.nvalid + kBBox - 1) / kBBox;
    const uint32_t b_bytes = nchunk * kBBox * 128;
    const int kblocks = S.K / 64;
    if (kKB2) {
      const int kb0 = 2 * ks;
      const bool gu = (S.mode == MODE_GATEUP);
      if (wts) {
        mbar_arrive_expect_tx(&full_bar[stg], (gu ? 4u : 2u) * kATileBytes + 2u * B_TILE_BYTES);
        tma_load_3d(st, &S.a0, 0, a_row0, kb0, &full_bar[stg], pol_w);
        if (gu) tma_load_3d(st + 2 * kATileBytes, &S.a1, 0, a_row0, kb0, &full_bar[stg], pol_w);
      }
      if (toks) tma_load_3d(st + 4 * kATileBytes, &S.b, 0, ui.b_row0, kb0, &full_bar[stg], pol_x);
      (void)nchunk;
      (void)b_bytes;
    } else if (S.mode == MODE_KPAIR) {
      const int kb0 = 2 * ks;
      const bool two = kb0 + 1 < kblocks;
      uint8_t* b1 = b0 + (NB > 1 ? B_TILE_BYTES : 0);
      if (wts) {
        mbar_arrive_expect_tx(&full_bar[stg], (two ? 2u : 1u) * (kATileBytes + b_bytes));
        tma_load_2d(st, &S.a0, kb0 * 64, a_row0, &full_bar[stg], pol_w);
        if (two) tma_load_2d(st + kATileBytes, &S.a0, (kb0 + 1) * 64, a_row0, &full_bar[stg], pol_w);
      }
      if (toks) {
        for (int c = 0; c < nchunk; ++c)
          tma_load_2d(b0 + c * kBBox * 128, &S.b, kb0 * 64, ui.b_row0 + c * kBBox, &full_bar[stg], pol_x);
        if (two)
          for (int c = 0; c < nchunk; ++c)
            tma_load_2d(b1 + c * kBBox * 128, &S.b, (kb0 + 1) * 64, ui.b_row0 + c * kBBox, &full_bar[stg], pol_x);
      }
    } else {
      const bool two = (S.mode != MODE_SINGLE && S.mode != MODE_TROUTE);
      const int kx = ks * 64;
      if (wts) {
        mbar_arrive_expect_tx(&full_bar[stg], (two ? 2u : 1u) * kATileBytes + b_bytes);
        tma_load_2d(st, &S.a0, kx, a_row0, &full_bar[stg], pol_w);
        // MODE_MPAIR / MODE_TPAIR: the a0 tensor map of those sets has a
        // 256-row box, so the one load above fills both 128-row halves (each
        // TMA instruction costs a fixed ~0.25 us of the SM's copy engine, so
        // one 32 KB box streams ~1.8x faster than two of 16 KB).
        if (S.mode == MODE_GATEUP || S.mode == MODE_TGATEUP)
          tma_load_2d(st + kATileBytes, &S.a1, kx, a_row0, &full_bar[stg], pol_w);
      }
      if (toks)
        for (int c = 0; c < nchunk; ++c)
          tma_load_2d(b0 + c * kBBox * 128, &S.b, kx, ui.b_row0 + c * kBBox, &full_bar[stg], pol_x);
    }
  };
  auto unit_stages = [](const GemmSet& S) {
    const int kblocks = S.K / 64;
    return (kKB2 || S.mode == MODE_KPAIR) ? (kblocks + 1) / 2 : kblocks;
  };

  // The first set, when its rows are static and it depends on nothing, gives
  // CTA b its first unit b (the others are claimed in order after them), so
  // the weights of that unit can stream before the previous kernel ends: its
  // first stages are issued here, weights only; the token rows follow the wait.
  const GemmSet& S0 = p.set[0];
  const bool first_static = !S0.counts && !S0.offsets && S0.groups == 1 && S0.dep_set < 0 && S0.static_rows > 0;
  const int nt0 = first_static ? (S0.static_rows + BN - 1) / BN : 0;
  const int units0 = first_static ? (S0.M + S0.m_tile - 1) / S0.m_tile * nt0 : 0;
  const int nstatic = min(units0, static_cast<int>(gridDim.x));
  const bool early = static_cast<int>(blockIdx.x) < nstatic;
  UnitInfo ui0{};
  if (early) {
    const int u0 = static_cast<int>(blockIdx.x);
    const int n0 = (u0 % nt0) * BN;
    ui0.g = 0;
    ui0.set = 0;
    ui0.gi = 0;
    ui0.m0 = (u0 / nt0) * S0.m_tile;
    ui0.nvalid = min(BN, S0.static_rows - n0);
    ui0.b_row0 = n0;
  }
  int stage = 0;  // producer state (warp 0, lane 0)
  uint32_t phase = 0;
  int fills[STAGES];
#pragma unroll
  for (int i = 0; i < STAGES; ++i) fills[i] = 0;
  const int npre = early ? min(STAGES, unit_stages(S0)) : 0;
  if (warp == 0 && lane == 0) {
    for (int ks = 0; ks < npre; ++ks) {  // fresh barriers: no empty-slot wait
      issue_stage(S0, ui0, ks, ks, true, false);
      fills[ks]++;
    }
  }
  // A decode CTA without an early unit takes its first dynamic claim before
  // the wait (the counter was zeroed before the step's first kernel), so the
  // claim's round trip overlaps the wait instead of following the group table.
  int pre_claim = -1;
  if (kSwapAB && warp == 0 && lane == 0 && !early && p.sched) pre_claim = atomicAdd(p.sched, 1);
  if (tid == 0) {  // set offsets of the group table: kernel parameters only
    int b = 0;
    for (int s = 0; s < p.nsets; ++s) {
      set_base[s] = b;
      b += p.set[s].groups;
    }
    set_base[p.nsets] = b;
  }
  __syncthreads();

  pdl_wait();  // the group sizes and the B operands come from the previous kernels

  // ---- group table (every CTA builds the same one) -----------------------
  const int ng = set_base[p.nsets];
  for (int g = tid; g < ng; g += kThreads) {
    int s = 0;
    while (g >= set_base[s + 1]) ++s;
    const int gi = g - set_base[s];
    const GemmSet& S = p.set[s];
    int rows = S.counts ? S.counts[gi] : S.static_rows;
    if (S.slab_rows > 0 && rows > S.slab_rows) rows = S.slab_rows;  // a slab never holds more
    g_rows[g] = rows;
    g_row0[g] = S.offsets ? S.offsets[gi] : gi * S.slab_rows;
    g_set[g] = static_cast<unsigned char>(s);
    g_gi[g] = static_cast<short>(gi);
    const int mt = (S.M + S.m_tile - 1) / S.m_tile;
    const int nt = rows > 0 ? (rows + BN - 1) / BN : 0;
    g_nt[g] = static_cast<short>(nt);
    g_begin[g + 1] = mt * nt;  // unit count, scanned below
  }
  if (tid == 0) g_begin[0] = 0;
  __syncthreads();
  if (warp == 0) {  // inclusive scan of unit counts, 32 groups at a time
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

  auto decode = [&](int u) -> UnitInfo {
    int lo = 0, hi = ng;  // g with g_begin[g] <= u < g_begin[g+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (g_begin[mid] <= u) lo = mid; else hi = mid;
    }
    const int local = u - g_begin[lo];
    const int nt = g_nt[lo];
    UnitInfo ui;
    ui.g = lo;
    ui.set = g_set[lo];
    ui.gi = g_gi[lo];
    ui.m0 = (local / nt) * p.set[ui.set].m_tile;
    const int n0 = (local % nt) * BN;
    ui.nvalid = min(BN, g_rows[lo] - n0);
    ui.b_row0 = g_row0[lo] + n0;
    return ui;
  };
  auto group_units = [&](int g) { return g_begin[g + 1] - g_begin[g]; };

  if (total_units == 0) {
    // nothing to do (uniform across the CTA); no copy was issued early, since
    // an early unit implies a non-empty first set
  } else if (warp == 0) {
    // ======================= claimer + TMA producer ========================
    if (lane == 0) {
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int q = it % kRing;
        if (!mbar_wait(&uempty_bar[q], ((it / kRing) & 1) ^ 1u, &abort_s, p.err, deadline)) break;
        int u;
        if (it == 0 && early)
          u = static_cast<int>(blockIdx.x);
        else if (it == 0 && pre_claim >= 0)
          u = nstatic + pre_claim;
        else
          u = p.sched ? nstatic + atomicAdd(p.sched, 1) : static_cast<int>(blockIdx.x) + it * static_cast<int>(gridDim.x);
        if (u >= total_units) u = -1;
        unit_ring[q] = u;
        mbar_arrive(&ufull_bar[q]);
        if (u < 0) break;
        const UnitInfo ui = decode(u);
        const GemmSet& S = p.set[ui.set];
        const int nstage = unit_stages(S);
        int pre_u = 0;  // DEPW: stages of this unit whose weights went out before its dependency wait
        if (S.dep_set >= 0) {  // wait until the group this unit reads from is complete
          const int gd = set_base[S.dep_set] + ui.gi;
          const int target = 4 * group_units(gd);
          const int* flag = p.sched + 1 + gd;
          if constexpr (DEPW) {
            const int stage_u = stage;
            if (ld_acquire_gpu(flag) < target) {
              // HBM keeps streaming this unit's weights while the group finishes.
              for (const int want = min(STAGES, nstage); pre_u < want; ++pre_u) {
                if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_s, p.err, deadline)) {
                  ok = false;
                  break;
                }
                issue_stage(S, ui, pre_u, stage, true, false);
                fills[stage]++;
                if (++stage == STAGES) {
                  stage = 0;
                  phase ^= 1u;
                }
              }
              while (ok && ld_acquire_gpu(flag) < target) {
                __nanosleep(64);
                if (*static_cast<volatile int*>(&abort_s) || globaltimer_ns() > deadline) {
                  if (!abort_s) {
                    abort_s = 1;
                    atomicOr(p.err, kErrTimeout);
                  }
                  ok = false;
                }
              }
            }
            fence_proxy_async_global();
            // The token rows of those stages (also after an abort, so that every
            // armed barrier completes and the drain below ends).
            for (int ks = 0; ks < pre_u; ++ks) issue_stage(S, ui, ks, (stage_u + ks) % STAGES, false, true);
            if (!ok) break;
          } else {
            while (ld_acquire_gpu(flag) < target) {
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
            fence_proxy_async_global();
          }
        }
        for (int ks = pre_u; ks < nstage; ++ks) {
          const bool pre = (it == 0 && ks < npre);  // weights already issued before the wait
          if (!pre && !mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_s, p.err, deadline)) {
            ok = false;
            break;
          }
          issue_stage(S, ui, ks, stage, !pre, true);
          if (!pre) fills[stage]++;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: every issued copy must have landed before the CTA may exit.
      const uint64_t drain_deadline = globaltimer_ns() + kDrainNs;
      for (int i = 0; i < STAGES; ++i)
        if (fills[i] > 0) {
          int dummy = 0;
          mbar_wait(&full_bar[i], static_cast<uint32_t>((fills[i] - 1) & 1), &dummy, p.err, drain_deadline);
        }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer ====================================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int it = 0;; ++it) {
        const int q = it % kRing;
        if (!mbar_wait(&ufull_bar[q], (it / kRing) & 1, &abort_s, p.err, deadline)) break;
        const int u = unit_ring[q];
        mbar_arrive(&uempty_bar[q]);
        if (u < 0) break;
        const UnitInfo ui = decode(u);
        const GemmSet& S = p.set[ui.set];
        const int slot = it & 1;
        if (!mbar_wait(&tempty_bar[slot], ((it >> 1) & 1) ^ 1u, &abort_s, p.err, deadline)) break;
        tc_fence_after();
        const bool tok_m = (S.mode == MODE_TGATEUP || S.mode == MODE_TPAIR || S.mode == MODE_TROUTE);
        const uint32_t n_mma = static_cast<uint32_t>((ui.nvalid + 15) & ~15);
        const uint32_t n_tok = (S.mode == MODE_TROUTE) ? static_cast<uint32_t>((S.M + 15) & ~15) : 256u;
        const uint32_t idesc = tok_m ? idesc_bf16_f32(128, n_tok) : idesc_bf16_f32(128, n_mma);
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(slot * ACC_COLS);
        const int kblocks = S.K / 64;
        const int nstage = unit_stages(S);
        bool ok = true;
        for (int ks = 0; ks < nstage; ++ks) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_s, p.err, deadline)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t a1 = st + kATileBytes;
          const uint32_t b0 = st + 2 * kATileBytes;
          if (kKB2) {
            // two k-blocks: D0 += A0[h] B[h] (and D1 += A1[h] B[h] for gate/up)
            const bool gu = (S.mode == MODE_GATEUP);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (h == 1 && 2 * ks + 1 >= kblocks) break;
              const uint32_t ah = st + h * kATileBytes;
              const uint32_t uh = st + (2 + h) * kATileBytes;
              const uint32_t bh = st + 4 * kATileBytes + h * B_TILE_BYTES;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc_mma_bf16(d0, smem_desc_k128(ah + kk * 32), smem_desc_k128(bh + kk * 32), idesc,
                            (ks | h | kk) != 0 ? 1u : 0u);
              if (gu) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  tc_mma_bf16(d0 + BN, smem_desc_k128(uh + kk * 32), smem_desc_k128(bh + kk * 32), idesc,
                              (ks | h | kk) != 0 ? 1u : 0u);
              }
            }
          } else if (tok_m) {
            // A = the token rows (B slot), B = the 256 weight rows of slots 0-1
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma_bf16(d0, smem_desc_k128(b0 + kk * 32), smem_desc_k128(st + kk * 32), idesc,
                          (ks | kk) != 0 ? 1u : 0u);
          } else if (S.mode == MODE_KPAIR) {
            const uint32_t b1 = b0 + (NB > 1 ? B_TILE_BYTES : 0);
            const bool two = 2 * ks + 1 < kblocks;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma_bf16(d0, smem_desc_k128(st + kk * 32), smem_desc_k128(b0 + kk * 32), idesc,
                          (ks | kk) != 0 ? 1u : 0u);
            if (two) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc_mma_bf16(d0, smem_desc_k128(a1 + kk * 32), smem_desc_k128(b1 + kk * 32), idesc, 1u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma_bf16(d0, smem_desc_k128(st + kk * 32), smem_desc_k128(b0 + kk * 32), idesc,
                          (ks | kk) != 0 ? 1u : 0u);
            if (S.mode != MODE_SINGLE) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc_mma_bf16(d0 + BN, smem_desc_k128(a1 + kk * 32), smem_desc_k128(b0 + kk * 32), idesc,
                            (ks | kk) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&empty_bar[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tfull_bar[slot]);
      }
      // Every MMA issued must be complete before TMEM is released.
      tc_commit(&mma_done_bar);
      int dummy = 0;
      mbar_wait(&mma_done_bar, 0, &dummy, p.err, globaltimer_ns() + kDrainNs);
    }
  } else {
    // ======================= epilogue (warps 2..5) =========================
    const int wq = warp & 3;  // TMEM lane quarter this warp may read
    float* tbuf = LM ? reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES) + wq * (32 * 33) : nullptr;
    for (int it = 0;; ++it) {
      const int q = it % kRing;
      if (!mbar_wait(&ufull_bar[q], (it / kRing) & 1, &abort_s, p.err, deadline)) break;
      const int u = unit_ring[q];
      __syncwarp();
      if (lane == 0) mbar_arrive(&uempty_bar[q]);
      if (u < 0) break;
      const UnitInfo ui = decode(u);
      const GemmSet& S = p.set[ui.set];
      const int slot = it & 1;
      if (!mbar_wait(&tfull_bar[slot], (it >> 1) & 1, &abort_s, p.err, deadline)) break;
      tc_fence_after();
      const int row = wq * 32 + lane;  // row of the 128-row tile held by this thread
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + static_cast<uint32_t>(slot * ACC_COLS);
      const int n_mma = (ui.nvalid + 15) & ~15;
      // The accumulator slot goes back to the MMA warp as soon as this warp
      // has read its last TMEM columns of the unit, before the stores: slow
      // stores then delay only this warp, not the next unit's MMAs.
      bool released = false;
      auto release_tmem = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty_bar[slot]);
        released = true;
      };
      if (kTokM && S.epi == EPI_TOPK) {
        // tokens on M: this thread holds all router logits of token `row`;
        // top-k on the logits, slots in descending order, weights
        // exp(l_j - l_0) / sum over the kept experts in slot order.  The order
        // is the one every router of this library uses: a larger logit first,
        // equal logits (-0 equal to +0) by the lower id, a NaN after every
        // number (-inf included), so a row with fewer than k numbers still
        // keeps k distinct experts.  Each logit becomes one 64-bit key (its
        // order key above the inverted expert id), so all keys differ and an
        // empty slot (key 0) sorts below every expert.  The TMEM loads are
        // warp-collective, so every lane issues them; only the selection and
        // the stores depend on the row being valid.
        const bool tvalid = row < ui.nvalid;
        constexpr int kMaxK = 8;
        // Two independent sorted lists (even and odd experts of each chunk of
        // 32), so consecutive insertions do not wait on each other, merged at
        // the end.  An insertion keeps a list sorted, larger key first.
        uint64_t ka[kMaxK], kb[kMaxK];
        float va[kMaxK], vb[kMaxK];
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
          ka[j] = kb[j] = 0;
          va[j] = vb[j] = 0.f;
        }
        auto insert = [](uint64_t (&sk)[kMaxK], float (&sv)[kMaxK], uint64_t ck, float v) {
          if (ck > sk[kMaxK - 1]) {
#pragma unroll
            for (int q = 0; q < kMaxK; ++q) {  // carry the smaller of (slot, candidate) down the list
              const bool gt = ck > sk[q];
              const uint64_t tk = gt ? sk[q] : ck;
              const float tv = gt ? sv[q] : v;
              sk[q] = gt ? ck : sk[q];
              sv[q] = gt ? v : sv[q];
              ck = tk;
              v = tv;
            }
          }
        };
        // Four logits per TMEM load in a rolled loop: a fully unrolled pass
        // over 32 logits (each with its insertion network) did not fit the
        // instruction cache and stalled on instruction fetch.
#pragma unroll 1
        for (int c0 = 0; c0 < S.M; c0 += 4) {
          uint32_t d[4];
          tmem_ld4(tl + c0, d);
          tmem_ld_wait();
          if (tvalid) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int e = c0 + j;
              if (e >= S.M) continue;
              float v = __uint_as_float(d[j]);
              if (S.bias) v += S.bias[e];
              uint32_t u = __float_as_uint(v);
              uint32_t okey;
              if ((u & 0x7fffffffu) > 0x7f800000u) {
                okey = 0u;  // NaN: below every number
              } else {
                if ((u << 1) == 0u) u = 0u;  // -0 -> +0
                okey = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
              }
              const uint64_t ck = (static_cast<uint64_t>(okey) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - e);
              if (j & 1)
                insert(kb, vb, ck, v);
              else
                insert(ka, va, ck, v);
            }
          }
        }
        // merge: the k largest of the two lists are max(ka[i], kb[7 - i])
        // (a bitonic sequence), sorted by a bitonic network of 3 x 4 steps
        uint64_t sk[kMaxK];
        float sv[kMaxK];
#pragma unroll
        for (int i = 0; i < kMaxK; ++i) {
          const bool ga = ka[i] > kb[kMaxK - 1 - i];
          sk[i] = ga ? ka[i] : kb[kMaxK - 1 - i];
          sv[i] = ga ? va[i] : vb[kMaxK - 1 - i];
        }
#pragma unroll
        for (int step = kMaxK / 2; step > 0; step >>= 1)
#pragma unroll
          for (int i = 0; i < kMaxK; ++i)
            if ((i & step) == 0) {
              const int jx = i + step;
              if (sk[jx] > sk[i]) {  // larger key first
                const uint64_t tk = sk[i];
                const float tv = sv[i];
                sk[i] = sk[jx];
                sv[i] = sv[jx];
                sk[jx] = tk;
                sv[jx] = tv;
              }
            }
        if (tvalid) {
          float ex[kMaxK];
          float s = 0.f;
#pragma unroll
          for (int j = 0; j < kMaxK; ++j) {
            ex[j] = (j < S.topk) ? expf(sv[j] - sv[0]) : 0.f;
            if (j < S.topk) s += ex[j];
          }
          int32_t* oi = static_cast<int32_t*>(S.out) + static_cast<size_t>(ui.b_row0 + row) * S.topk;
          float* ow = static_cast<float*>(S.out2) + static_cast<size_t>(ui.b_row0 + row) * S.topk;
#pragma unroll
          for (int j = 0; j < kMaxK; ++j)
            if (j < S.topk) {
              oi[j] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(sk[j] & 0xFFFFFFFFull));
              ow[j] = ex[j] / s;
            }
        }
      } else if (kTokM && (S.epi == EPI_SWIGLU_ROWS || S.epi == EPI_STORE_ROWS)) {
        // tokens on M: this thread holds token row `row` of the tile, the
        // columns are 256 weight outputs (gate|up, or two halves of W_down)
        const bool tvalid = row < ui.nvalid;
        const size_t orow = static_cast<size_t>(ui.b_row0 + row) * S.ld_out;
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
                  a2[q] = (gf / (1.0f + expf(-gf))) * uf;
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
        } else {
          float* out = static_cast<float*>(S.out);
          for (int c0 = 0; c0 < 256; c0 += 32) {
            uint32_t d[32];
            tmem_ld32(tl + c0, d);
            tmem_ld_wait();
            if (tvalid && ui.m0 + c0 < S.M) {
              float4* dst = reinterpret_cast<float4*>(out + orow + ui.m0 + c0);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(__uint_as_float(d[4 * q]), __uint_as_float(d[4 * q + 1]),
                                     __uint_as_float(d[4 * q + 2]), __uint_as_float(d[4 * q + 3]));
            }
          }
        }
      } else if (kSwapAB && S.epi == EPI_SWIGLU) {
        const int m = ui.m0 + row;
        const bool mvalid = m < S.M;
        uint16_t* out = static_cast<uint16_t*>(S.out);
        for (int c0 = 0; c0 < n_mma; c0 += 32) {
          uint32_t g[32], v[32];
          tmem_ld32(tl + c0, g);
          tmem_ld32(tl + BN + c0, v);
          tmem_ld_wait();
          if (c0 + 32 >= n_mma) release_tmem();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int n = c0 + j;
            if (mvalid && n < ui.nvalid) {
              const float gf = __uint_as_float(g[j]);
              const float uf = __uint_as_float(v[j]);
              const float s = gf / (1.0f + expf(-gf));
              out[static_cast<size_t>(ui.b_row0 + n) * S.ld_out + m] = f32_to_bf16_bits(s * uf);
            }
          }
        }
      } else if (kSwapAB && S.epi == EPI_STORE_F32) {
        float* out = static_cast<float*>(S.out);
        const int halves = (S.mode == MODE_MPAIR) ? 2 : 1;
        for (int h = 0; h < halves; ++h) {
          const int m = ui.m0 + h * 128 + row;
          const bool mvalid = m < S.M;
          for (int c0 = 0; c0 < n_mma; c0 += 32) {
            // output rows of these 32 B rows: lane j holds row j's (row_map, or b itself)
            const int bj = ui.b_row0 + c0 + lane;
            const int orow = (S.row_map && c0 + lane < ui.nvalid) ? __ldg(S.row_map + bj) : bj;
            uint32_t d[32];
            tmem_ld32(tl + h * BN + c0, d);
            tmem_ld_wait();
            if (h + 1 == halves && c0 + 32 >= n_mma) release_tmem();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int n = c0 + j;
              const int o = __shfl_sync(0xffffffffu, orow, j);
              if (mvalid && n < ui.nvalid) out[static_cast<size_t>(o) * S.ld_out + m] = __uint_as_float(d[j]);
            }
          }
        }
      } else if (kSwapAB && S.epi == EPI_STORE_BF16) {
        // out[n][m] = bf16(res[n][m] + acc) (res nullable).  res was written
        // by an earlier set of this launch (a dependency): read it from L2.
        uint16_t* out = static_cast<uint16_t*>(S.out);
        const int m = ui.m0 + row;
        const bool mvalid = m < S.M;
        for (int c0 = 0; c0 < n_mma; c0 += 32) {
          uint32_t d[32];
          tmem_ld32(tl + c0, d);
          tmem_ld_wait();
          if (c0 + 32 >= n_mma) release_tmem();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int n = c0 + j;
            if (mvalid && n < ui.nvalid) {
              const size_t o = static_cast<size_t>(ui.b_row0 + n) * S.ld_out + m;
              float v = __uint_as_float(d[j]);
              if (S.res) v = __fadd_rn(bf16_bits_to_f32(__ldcg(S.res + o)), v);
              out[o] = f32_to_bf16_bits(v);
            }
          }
        }
      } else if (LM) {  // EPI_ARGMAX over the tile's 128 (MODE_SINGLE) or 256 (MODE_MPAIR) vocabulary rows
        const int halves = (S.mode == MODE_MPAIR) ? 2 : 1;
        uint64_t* out = static_cast<uint64_t*>(S.out);
        for (int c0 = 0; c0 < n_mma; c0 += 32) {
          uint64_t best_key = 0;
          for (int h = 0; h < halves; ++h) {
            const int m = ui.m0 + h * 128 + row;
            const bool mvalid = m < S.M;
            uint32_t d[32];
            tmem_ld32(tl + h * BN + c0, d);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              tbuf[lane * 33 + j] = mvalid ? __uint_as_float(d[j]) : -__int_as_float(0x7f800000);
            __syncwarp();
            // lane j scans column c0 + j over this warp's 32 rows of this half
            float best = tbuf[lane];
            int bi = 0;
#pragma unroll 8
            for (int i = 1; i < 32; ++i) {
              const float x = tbuf[i * 33 + lane];
              if (x > best) {
                best = x;
                bi = i;
              }
            }
            __syncwarp();
            const uint64_t key =
                argmax_key(best, static_cast<uint32_t>(S.key_row_base + ui.m0 + h * 128 + wq * 32 + bi));
            best_key = key > best_key ? key : best_key;
          }
          const int n = c0 + lane;
          if (n < ui.nvalid) {
            const int part = S.key_part_base + (ui.m0 / S.m_tile) * 4 + wq;  // (M tile, lane quarter), token-major
            out[static_cast<size_t>(ui.b_row0 + n) * S.ld_out + part] = best_key;
          }
        }
      } else if (lane == 0) {
        atomicOr(p.err, kErrInternal);  // a set this tile configuration is not compiled for
      }
      if (!released) tc_fence_before();
      if (S.signal && p.sched) {  // release this warp's stores to the units that depend on the group
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          atomicAdd(p.sched + 1 + ui.g, 1);
        }
      }
      __syncwarp();
      if (!released && lane == 0) mbar_arrive(&tempty_bar[slot]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
}

// ---------------------------------------------------------------------------
// host-side launch
// ---------------------------------------------------------------------------
template <int BN, int STAGES, int NB, bool LM, int BBOX, bool DEPW = false>
static cudaError_t launch_gemm_impl(const GemmParams& p, int grid, cudaStream_t stream) {
  constexpr int STAGE_BYTES = ((!LM && BN == 32) ? 4 : 2) * kATileBytes + NB * BN * 128;  // as in the kernel
  constexpr int EXTRA = LM ? 4 * 32 * 33 * 4 : 0;  // argmax epilogue transpose buffers
  constexpr int SMEM = STAGES * STAGE_BYTES + EXTRA + 1024;
  // the kernel's static shared memory is 9,216 bytes (ptxas); the opt-in limit is 227 KB
  static_assert(SMEM + 9216 <= 227 * 1024, "shared memory (dynamic + static)");
  auto kern = gemm_tc_kernel<BN, STAGES, NB, LM, BBOX, DEPW>;
  static thread_local int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    configured_dev = dev;
  }
  return launch_pdl(kern, dim3(grid), dim3(kThreads), SMEM, stream, p);
}

// Tile configurations:
//   GEMM_MOE_DECODE   BN = 32, two k-blocks per stage (3D boxes), 3 stages of 72 KB
//   GEMM_MOE_DECODE_FEW  the same, the down units' weights issued before their dependency wait
//   GEMM_MOE_PREFILL  BN = 128, one B slot, 4 stages of 48 KB (tokens-on-M modes)
//   GEMM_LM           BN = 128, one B slot, 4 stages of 48 KB (MODE_MPAIR), 16-row token boxes
//   GEMM_LM_WIDE      the same with 128-row token boxes, for 128 or more tokens
cudaError_t launch_gemm(int config, const GemmParams& p, int grid, cudaStream_t stream) {
  switch (config) {
    case GEMM_MOE_DECODE: return launch_gemm_impl<32, 3, 2, false, kDecodeBBox>(p, grid, stream);
    case GEMM_MOE_DECODE_FEW: return launch_gemm_impl<32, 3, 2, false, kDecodeBBox, true>(p, grid, stream);
    case GEMM_MOE_PREFILL: return launch_gemm_impl<128, 4, 1, false, kPrefillBBox>(p, grid, stream);
    case GEMM_LM: return launch_gemm_impl<128, 4, 1, true, kLmBBox>(p, grid, stream);
    case GEMM_LM_WIDE: return launch_gemm_impl<128, 4, 1, true, kLmWideBBox>(p, grid, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace mv
