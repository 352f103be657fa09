// Internal host/device declarations shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

#include "gemm_params.h"

namespace mv {

// Launch `kernel` on `stream` with programmatic stream serialization, so it may
// begin (up to its pdl_wait()) while the previous kernel on the stream drains.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

cudaError_t launch_gemm(int config, const GemmParams& p, int grid, cudaStream_t stream);
// CTA-pair (cta_group::2) form of the tokens-on-M modes (MODE_TGATEUP with
// EPI_SWIGLU_ROWS, MODE_TPAIR with EPI_STORE_ROWS) for prefill-sized groups:
// 256-token units, 3D tensor maps with 128-row boxes for every operand.
// gemm_pair_max_clusters(): pairs that can be resident at once (0: unavailable).
int gemm_pair_max_clusters();
cudaError_t launch_gemm_pair(const GemmParams& p, int clusters, cudaStream_t stream);

// Up to four device ranges a kernel prefetches into L2 before it waits for its
// predecessor (the first weights the next GEMM will stream), split evenly over
// the kernel's CTAs.
struct L2Prefetch {
  const void* ptr[4];
  uint64_t bytes[4];
  int n;
};

// CTAs a kernel needs so that no CTA issues more than 256 KB of the prefetch:
// one SM issues bulk prefetches at roughly 200 GB/s, so a kernel with few
// rows (one CTA per row at batch 1) launches extra CTAs that only prefetch.
inline int prefetch_ctas(const L2Prefetch& pf) {
  uint64_t total = 0;
  for (int i = 0; i < pf.n; ++i) total += pf.bytes[i];
  const uint64_t n = (total + (256u << 10) - 1) >> 18;
  return static_cast<int>(n < 148 ? n : 148);
}

// Small CUDA-core kernels (kernels_small.cu).
struct CombineRouteArgs {
  const uint16_t* x;        // residual rows (combine) or the rows to route (route only)
  const float* y_perm;      // expert outputs by grouped position, or nullptr: route only
  const float* y_sh;        // shared-expert outputs or nullptr
  const int32_t* inv;       // position of entry r*k_prev+j in y_perm
  const float* w_prev;      // routing weights of the layer being combined
  int k_prev;
  uint16_t* out;            // combined rows (when y_perm is given)
  int T, H, E, k;
  const uint16_t* wr;       // router weights of the layer to route
  const float* bias;
  int32_t* idx;
  float* w;
  int* err;
  L2Prefetch pf;
  int n_pos;                // entries of y_perm (positions valid in inv); 0: T * k_prev
  // Grouping by expert fused into the routing (slab layout), or nullptr: each
  // routed entry (row r, slot j -> expert e) takes the next free row of expert
  // e's slab of slab_rows rows: p = e * slab_rows + atomicAdd(&slab_counts[e], 1),
  // x_slab[p] = the routed row, inv_out[r * k + j] = p.  slab_counts must be
  // zero at launch.  Rows land in a slab in any order; every consumer reads
  // them through slab_counts and inv_out, and no result depends on the order.
  int32_t* slab_counts;
  int32_t* inv_out;
  uint16_t* x_slab;
  int slab_rows;
  int32_t* ent_out;         // with slab_counts, or nullptr: ent_out[p] = r * k + j (the entry of slab row p)
  // y_perm holds the combined layer's expert outputs by entry (row r * k_prev
  // + j) instead of by grouped position; inv then only tells valid entries.
  int y_by_entry;
  // Pre-RMSNorm variant, or nullptr: the rows are routed (and placed) as
  // bf16(RMSNorm(row) * norm_gain), also written to xn_out [T][H].
  const uint16_t* norm_gain;
  uint16_t* xn_out;
  // Bound on the wait for the staged router matrix (0: the drain bound).
  uint64_t timeout_ns;
};
constexpr float kRmsNormEps = 1e-6f;
cudaError_t launch_rmsnorm(const uint16_t* x, int T, int H, const uint16_t* gain, uint16_t* out, cudaStream_t s);
bool combine_route_supported(int T, int H, int E);
cudaError_t launch_combine_route(const CombineRouteArgs& a, cudaStream_t s);
cudaError_t launch_router(const uint16_t* x, int T, int H, int E, int k, const uint16_t* wr,
                          const float* bias, int32_t* idx, float* w, int* err, uint64_t timeout_ns,
                          cudaStream_t s);
cudaError_t launch_permute(const int32_t* idx, int T, int E, int k, int32_t* counts,
                           int32_t* offsets, int32_t* perm, int32_t* inv, const uint16_t* x,
                           int H, uint16_t* x_perm, cudaStream_t s);
bool permute_uses_sort(int T, int k);
size_t sort_scratch_ints(int T, int E, int k);
cudaError_t launch_permute_sorted(const int32_t* idx, int T, int E, int k, int32_t* counts, int32_t* offsets,
                                  int32_t* perm, int32_t* inv, const uint16_t* x, int H, uint16_t* x_perm,
                                  int32_t* scratch, cudaStream_t s);
// n_pos: the number of y_perm rows (positions in inv are checked against it).
// y_by_entry: y_perm rows are entries r * k + j (inv only marks valid ones).
cudaError_t launch_combine(const float* y_perm, const float* y_sh, const int32_t* inv,
                           const float* w, const uint16_t* res, uint16_t* out, int T, int H,
                           int k, int n_pos, int* err, const L2Prefetch& pf, cudaStream_t s,
                           bool y_by_entry = false);
// The FastMTP draft block's per-sequence step (kernels_small.cu, mtp_step_kernel).
struct MtpStepArgs {
  const uint64_t* keys;   // previous step's LM keys [B][ld] (nparts used), or nullptr: take t0
  int nparts, ld;
  const int32_t* t0;      // [B] first tokens (when keys is nullptr)
  int32_t* drafts;        // [B][K]; step j writes column j-1
  int K, j;
  const uint16_t* h_src;  // previous hidden states, row b*row_stride + (acc ? acc[b] : 0)
  int row_stride;
  const int32_t* acc;
  const uint16_t* w_emb;  // [V][H]
  int V;
  const uint16_t *g_h, *g_e;
  int H;
  float eps;
  uint16_t* u;            // [B][2H] next input rows, or nullptr (last step)
  int* err;
  int B;
};
cudaError_t launch_mtp_step(const MtpStepArgs& a, cudaStream_t s);
cudaError_t launch_lm_finalize(const uint64_t* keys, int nparts, int ld, int T, int32_t* argmax,
                               cudaStream_t s);
cudaError_t launch_accept(const int32_t* argmax, const int32_t* drafts, int B, int K,
                          int32_t* accepted, int32_t* next_token, int32_t* emitted,
                          cudaStream_t s);
cudaError_t launch_accept_from_keys(const uint64_t* keys, int nparts, int ld, const int32_t* drafts,
                                    int B, int K, int32_t* accepted, int32_t* next_token,
                                    int32_t* emitted, int32_t* argmax, cudaStream_t s);

// Decoder self-attention of the verify rows over the key/value cache
// (attention.cu).  Head dim 128; cache [B][n_heads][L_max][128] bf16 read
// through 3D tensor maps ([k-half][row][64] view, 64-row boxes).
struct AttnParams {
  CUtensorMap k_map;
  CUtensorMap v_map;
  const uint16_t* q;        // [B*(K+1)][n_heads*128] bf16
  const int32_t* ctx_len;   // [B]
  uint16_t* out;            // [B*(K+1)][n_heads*128] bf16
  float* part_o;            // [B*n_heads][n_split][NQ][128]
  float* part_ml;           // [B*n_heads][n_split][NQ][2]: running max, sum of weights
  int* counters;            // [B*n_heads], zero at launch
  int* err;
  int K, n_heads, L_max, max_ctx;
  int split_len;            // positions per split, a multiple of 64
  int n_split;              // grid.x: splits of the longest sequence
  float scale;              // 1 / sqrt(128)
  uint64_t timeout_ns;
};
int attention_nq(int K);  // query rows per (sequence, head) the kernel is compiled for: 1, 2, 4, 8 (0: K too large)
cudaError_t launch_decode_attention(const AttnParams& p, int B, cudaStream_t s);

}  // namespace mv
