// Grouped tensor-core GEMM engine for sm_100a (tcgen05 + TMEM + TMA).
//
// One launch computes, for every group g of one or two operand sets,
//     D_g[m][n] = sum_k A_g[m][k] * B_g[n][k]          (bf16 x bf16 -> fp32)
// where A_g is a weight matrix (rows = output features, K-major) and B_g the
// token rows routed to that group (K-major).  Weights sit on the MMA's M side
// (128 rows per tile) and tokens on its N side ("swap-AB"), so the few tokens
// per expert of a decode step still fill whole 128-row weight tiles; the N
// extent of each tile is the group's real row count rounded up to 16.
//
// Used for the three contractions of the verify step (jina-ocr-v1 model card,
// architecture paragraph: MoE decoder with routed + shared experts and a
// 129,280-token LM head):
//   EPI_SWIGLU    gate and up projections together (two A operands into two
//                 accumulators), epilogue a = bf16(silu(g) * u)
//   EPI_STORE_F32 down projection, epilogue stores fp32 rows
//   EPI_ARGMAX    LM head, epilogue reduces each token column to a packed
//                 (logit, lowest index) key per 32 vocabulary rows; the logits
//                 never reach memory
//
// Structure: persistent CTAs (at most one per SM), 6 warps.
//   warp 0      TMA producer (one thread): A tiles [128 x 64] and B tiles
//               [16-row chunks x 64], 128-byte swizzle, STAGES-deep ring
//   warp 1      TMEM allocator and MMA issuer (one thread), 128xNx16 MMAs
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns per warp
// Accumulators are double-buffered in TMEM so the epilogue of one tile
// overlaps the main loop of the next.  Work units (group, 128-row M tile,
// BN-column N tile) are enumerated on the device from the per-group row
// counts, shared-expert units first, N fastest so that the units reading the
// same weight tile run side by side.  Every wait is bounded (see mv_device.cuh).
// No TMA multicast is used.

#include "mv_device.cuh"
#include "mv_internal.h"

namespace mv {

namespace {

constexpr int kThreads = 192;
constexpr int kMaxGroups = 264;
constexpr int kATileBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kBBox = 16;               // B rows per TMA box

template <int EPI>
struct EpiTraits;
template <>
struct EpiTraits<EPI_SWIGLU> {
  static constexpr int NA = 2;
};
template <>
struct EpiTraits<EPI_STORE_F32> {
  static constexpr int NA = 1;
};
template <>
struct EpiTraits<EPI_ARGMAX> {
  static constexpr int NA = 1;
};

struct UnitInfo {
  int set, gi, m0, n0, nvalid, b_row0;
};

__device__ __forceinline__ int upper_pow2_cols(int c) {
  int n = 32;
  while (n < c) n <<= 1;
  return n;
}

}  // namespace

template <int EPI, int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmParams p) {
  constexpr int NA = EpiTraits<EPI>::NA;
  constexpr int B_TILE_BYTES = BN * 128;
  constexpr int STAGE_BYTES = NA * kATileBytes + B_TILE_BYTES;
  constexpr int ACC_COLS = NA * BN;            // TMEM columns of one accumulator set
  constexpr int ACC_SLOTS = (2 * ACC_COLS <= 512) ? 2 : 1;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
  static_assert(ACC_COLS <= 512, "TMEM");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t mma_done_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int g_begin[kMaxGroups + 1];  // first unit of each group
  __shared__ int g_rows[kMaxGroups];
  __shared__ int g_row0[kMaxGroups];
  __shared__ int g_nt[kMaxGroups];
  __shared__ short g_set[kMaxGroups];
  __shared__ short g_gi[kMaxGroups];
  __shared__ int n_groups_s;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint64_t deadline = globaltimer_ns() + p.timeout_ns;

  // ---- group table ---------------------------------------------------------
  int ng = 0;
  for (int s = 0; s < p.nsets; ++s) ng += p.set[s].groups;
  if (tid == 0) n_groups_s = ng;
  for (int g = tid; g < ng; g += kThreads) {
    int s = 0, gi = g;
    while (gi >= p.set[s].groups) {
      gi -= p.set[s].groups;
      ++s;
    }
    const GemmSet& S = p.set[s];
    int rows = S.counts ? S.counts[gi] : S.static_rows;
    int row0 = S.offsets ? S.offsets[gi] : 0;
    g_rows[g] = rows;
    g_row0[g] = row0;
    g_set[g] = static_cast<short>(s);
    g_gi[g] = static_cast<short>(gi);
    const int mt = (S.M + 127) / 128;
    const int nt = rows > 0 ? (rows + BN - 1) / BN : 0;
    g_nt[g] = nt;
    g_begin[g + 1] = mt * nt;  // unit count, scanned below
  }
  if (tid == 0) {
    g_begin[0] = 0;
    abort_s = 0;
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 4);
    }
    mbar_init(&mma_done_bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {  // inclusive scan of unit counts, 32 groups at a time
    int carry = 0;
    for (int base = 0; base < ng; base += 32) {
      int g = base + lane;
      int v = (g < ng) ? g_begin[g + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
      }
      if (g < ng) g_begin[g + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  __syncthreads();
  const int total_units = g_begin[ng];
  if (static_cast<int>(blockIdx.x) >= total_units) return;  // uniform across the CTA

  auto decode = [&](int u) -> UnitInfo {
    int lo = 0, hi = ng;  // find g with g_begin[g] <= u < g_begin[g+1]
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (g_begin[mid] <= u) lo = mid; else hi = mid;
    }
    const int g = lo;
    const int local = u - g_begin[g];
    const int nt = g_nt[g];
    UnitInfo ui;
    ui.set = g_set[g];
    ui.gi = g_gi[g];
    ui.m0 = (local / nt) * 128;
    ui.n0 = (local % nt) * BN;
    ui.nvalid = min(BN, g_rows[g] - ui.n0);
    ui.b_row0 = g_row0[g] + ui.n0;
    return ui;
  };

  const int tmem_cols = upper_pow2_cols(ACC_SLOTS * ACC_COLS);
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, tmem_cols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < p.nsets; ++s) {
      tma_prefetch_desc(&p.set[s].a0);
      if (NA == 2) tma_prefetch_desc(&p.set[s].a1);
      tma_prefetch_desc(&p.set[s].b);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;

  if (warp == 0) {
    // ======================= TMA producer ==================================
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int fills[STAGES];
#pragma unroll
      for (int i = 0; i < STAGES; ++i) fills[i] = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const UnitInfo ui = decode(u);
        const GemmSet& S = p.set[ui.set];
        const int a_row0 = ui.gi * S.a_group_stride + ui.m0;
        const int nchunk = (ui.nvalid + kBBox - 1) / kBBox;
        const uint32_t bytes = NA * kATileBytes + nchunk * kBBox * 128;
        const int kblocks = S.K / 64;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_s, p.err, deadline)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&full_bar[stage], bytes);
          tma_load_2d(st, &S.a0, kb * 64, a_row0, &full_bar[stage], pol_w);
          if (NA == 2) tma_load_2d(st + kATileBytes, &S.a1, kb * 64, a_row0, &full_bar[stage], pol_w);
          uint8_t* bt = st + NA * kATileBytes;
          for (int c = 0; c < nchunk; ++c)
            tma_load_2d(bt + c * kBBox * 128, &S.b, kb * 64, ui.b_row0 + c * kBBox, &full_bar[stage],
                        pol_x);
          fills[stage]++;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: every issued copy must have landed before the CTA may exit.
      const uint64_t drain_deadline = globaltimer_ns() + p.timeout_ns;
      for (int i = 0; i < STAGES; ++i)
        if (fills[i] > 0) {
          int dummy = 0;
          mbar_wait(&full_bar[i], static_cast<uint32_t>((fills[i] - 1) & 1), &dummy, p.err,
                    drain_deadline);
        }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer ====================================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++it) {
        const UnitInfo ui = decode(u);
        const GemmSet& S = p.set[ui.set];
        const int slot = (ACC_SLOTS == 2) ? (it & 1) : 0;
        const uint32_t aphase = static_cast<uint32_t>((ACC_SLOTS == 2 ? (it >> 1) : it) & 1);
        if (!mbar_wait(&tempty_bar[slot], aphase ^ 1u, &abort_s, p.err, deadline)) break;
        tc_fence_after();
        const uint32_t n_mma = static_cast<uint32_t>((ui.nvalid + 15) & ~15);
        const uint32_t idesc = idesc_bf16_f32(128, n_mma);
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(slot * ACC_COLS);
        const int kblocks = S.K / 64;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_s, p.err, deadline)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t bt = st + NA * kATileBytes;
#pragma unroll
          for (int a = 0; a < NA; ++a) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t adesc = smem_desc_k128(st + a * kATileBytes + kk * 32);
              const uint64_t bdesc = smem_desc_k128(bt + kk * 32);
              tc_mma_bf16(d0 + a * BN, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
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
      mbar_wait(&mma_done_bar, 0, &dummy, p.err, globaltimer_ns() + p.timeout_ns);
    }
  } else {
    // ======================= epilogue (warps 2..5) =========================
    const int wq = warp & 3;  // TMEM lane quarter this warp may read
    float* tbuf = nullptr;
    if (EPI == EPI_ARGMAX)
      tbuf = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES) + wq * (32 * 33);
    int it = 0;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++it) {
      const UnitInfo ui = decode(u);
      const GemmSet& S = p.set[ui.set];
      const int slot = (ACC_SLOTS == 2) ? (it & 1) : 0;
      const uint32_t aphase = static_cast<uint32_t>((ACC_SLOTS == 2 ? (it >> 1) : it) & 1);
      if (!mbar_wait(&tfull_bar[slot], aphase, &abort_s, p.err, deadline)) break;
      tc_fence_after();
      const int row = wq * 32 + lane;  // row of the 128-row tile held by this thread
      const int m = ui.m0 + row;
      const bool mvalid = m < S.M;
      const uint32_t tl = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) +
                          static_cast<uint32_t>(slot * ACC_COLS);
      const int n_mma = (ui.nvalid + 15) & ~15;
      for (int c0 = 0; c0 < n_mma; c0 += 32) {
        if (EPI == EPI_SWIGLU) {
          uint32_t g[32], v[32];
          tmem_ld32(tl + c0, g);
          tmem_ld32(tl + BN + c0, v);
          tmem_ld_wait();
          uint16_t* out = static_cast<uint16_t*>(S.out);
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
        } else if (EPI == EPI_STORE_F32) {
          uint32_t d[32];
          tmem_ld32(tl + c0, d);
          tmem_ld_wait();
          float* out = static_cast<float*>(S.out);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int n = c0 + j;
            if (mvalid && n < ui.nvalid)
              out[static_cast<size_t>(ui.b_row0 + n) * S.ld_out + m] = __uint_as_float(d[j]);
          }
        } else {  // EPI_ARGMAX
          uint32_t d[32];
          tmem_ld32(tl + c0, d);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            tbuf[lane * 33 + j] = mvalid ? __uint_as_float(d[j]) : -__int_as_float(0x7f800000);
          __syncwarp();
          // lane j now scans column c0 + j over this warp's 32 rows
          float best = tbuf[lane];
          int bi = 0;
#pragma unroll 8
          for (int i = 1; i < 32; ++i) {
            const float v = tbuf[i * 33 + lane];
            if (v > best) {
              best = v;
              bi = i;
            }
          }
          __syncwarp();
          const int n = c0 + lane;
          if (n < ui.nvalid) {
            uint64_t* out = static_cast<uint64_t*>(S.out);
            const int part = (ui.m0 / 128) * 4 + wq;  // (M tile, lane quarter); keys are token-major
            out[static_cast<size_t>(ui.b_row0 + n) * S.ld_out + part] =
                argmax_key(best, static_cast<uint32_t>(ui.m0 + wq * 32 + bi));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[slot]);
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
template <int EPI, int BN, int STAGES>
static cudaError_t launch_gemm_impl(const GemmParams& p, int grid, cudaStream_t stream) {
  constexpr int NA = EpiTraits<EPI>::NA;
  constexpr int STAGE_BYTES = NA * kATileBytes + BN * 128;
  constexpr int EXTRA = (EPI == EPI_ARGMAX) ? 4 * 32 * 33 * 4 : 0;
  constexpr int SMEM = STAGES * STAGE_BYTES + EXTRA + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory");
  auto kern = gemm_tc_kernel<EPI, BN, STAGES>;
  static thread_local int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    configured_dev = dev;
  }
  kern<<<grid, kThreads, SMEM, stream>>>(p);
  return cudaGetLastError();
}

// Tile configurations.  bn = 32 is the decode configuration (a few tokens per
// expert): the B tile shrinks to 4 KB per stage so 6 (gate/up) or 10 (down)
// stages keep 192 / 160 KB of weights in flight per SM.  bn = 128 serves
// larger groups and the LM head.
cudaError_t launch_gemm(int epi, int bn, const GemmParams& p, int grid, cudaStream_t stream) {
  if (epi == EPI_SWIGLU && bn == 32) return launch_gemm_impl<EPI_SWIGLU, 32, 6>(p, grid, stream);
  if (epi == EPI_SWIGLU && bn == 128) return launch_gemm_impl<EPI_SWIGLU, 128, 4>(p, grid, stream);
  if (epi == EPI_STORE_F32 && bn == 32) return launch_gemm_impl<EPI_STORE_F32, 32, 10>(p, grid, stream);
  if (epi == EPI_STORE_F32 && bn == 128) return launch_gemm_impl<EPI_STORE_F32, 128, 6>(p, grid, stream);
  if (epi == EPI_ARGMAX && bn == 128) return launch_gemm_impl<EPI_ARGMAX, 128, 6>(p, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace mv
