/*
 * moe_verify.h - C ABI of the B200 (sm_100a) greedy MoE speculative-verify step.
 *
 * The step verifies K draft tokens per sequence for the mixture-of-experts
 * decoder of jina-ocr-v1.  Shapes and the method come from the jina-ocr-v1
 * model card (jina.ai/models/jina-ocr-v1):
 *   - architecture paragraph: 12 decoder layers, hidden 1280, 64 routed
 *     experts plus 2 shared under top-6 routing, 129,280-token vocabulary;
 *   - decoding-speed paragraph and introduction: K drafts (K=3) are checked
 *     greedily, so the output equals plain autoregressive decoding, and up to
 *     K+1 tokens are committed per verifier pass;
 *   - usage paragraph: turning speculation off (K = 0) leaves the text as is.
 * and from the tldrocket write-up "Jina AI Releases jina-ocr-v1 ...",
 * speculative paragraph: the decoder keeps only the drafts that match its
 * own choice.
 *
 * Conventions for every call below
 *   Memory      All tensor pointers are DEVICE pointers owned by the caller.
 *               bf16 tensors are passed as uint16_t bit patterns.  The
 *               library never allocates device memory on these paths; the
 *               scratch space it needs is the caller's workspace, sized by the
 *               matching *_workspace_size() call.
 *   Layout      Row-major, densely packed, in the shapes given per argument.
 *               Token rows of a verify step are sequence-major:
 *               row r = b*(K+1) + j, j = 0 the current token, j = 1..K draft j.
 *   Alignment   Every pointer must be 16-byte aligned (MV_ERR_MISALIGNED).
 *               H, I and I_shared must be multiples of 64 and V a multiple
 *               of 8 (MV_ERR_UNSUPPORTED_SHAPE).  Limits: E <= 256,
 *               1 <= k <= min(E, 8).
 *   Streams     Every call is asynchronous on the given stream (NULL = the
 *               legacy default stream).  Argument checks happen on the host
 *               before anything is launched; a call that returns an error
 *               launched nothing.  A launch failure returns MV_ERR_CUDA.
 *   Device      Waits inside the library's kernels are bounded; a wait that
 *   errors      runs out records MV_ERR_TIMEOUT in a sticky error word that
 *               lives in the workspace.  mv_sync_status() reads and clears it.
 *   Errors      mv_last_error() gives a message for the last non-OK status
 *               returned on the calling thread.  No C++ exception crosses
 *               this interface.
 *   Determinism Every result is a deterministic function of the inputs: no
 *               floating-point atomics, and the same row gives the same bits
 *               whatever other rows share its batch, among batches of one
 *               size class: decode-sized batches (T*k <= 16*E routed entries,
 *               T <= 1024) run one set of tile forms, larger ones another
 *               (tokens on the MMA's M side, CTA pairs, the tensor-core
 *               router), whose fp32 sums differ in the last bits.  The LM
 *               head has its own two classes: below 256 rows and from 256
 *               rows (CTA pairs).
 */
#ifndef MOE_VERIFY_H
#define MOE_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MV_API __attribute__((visibility("default")))
#else
#define MV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* mv_stream_t;

typedef enum {
  MV_OK = 0,
  MV_ERR_INVALID_ARG = 1,         /* null pointer, negative size, bad k/E/K */
  MV_ERR_UNSUPPORTED_SHAPE = 2,   /* H/I/I_shared not multiples of 64, V not of 8, limits */
  MV_ERR_MISALIGNED = 3,          /* a pointer is not 16-byte aligned */
  MV_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes below the *_workspace_size() value */
  MV_ERR_CUDA = 5,                /* a CUDA runtime call or launch failed */
  MV_ERR_TIMEOUT = 6,             /* a bounded device-side wait ran out */
  MV_ERR_INTERNAL = 7             /* a device-side consistency check failed */
} mv_status;

/* Shape of one MoE layer.  I_shared = 0 means no shared expert.  The model
 * card's two shared experts are passed as one always-on SwiGLU of
 * I_shared = 2*I whose gate/up rows and down columns are the two concatenated;
 * that is exactly the sum of the two experts' outputs. */
typedef struct {
  int32_t H;        /* hidden size (1280) */
  int32_t E;        /* routed experts (64) */
  int32_t I;        /* routed expert intermediate size (896) */
  int32_t I_shared; /* shared intermediate size (1792), or 0 */
  int32_t k;        /* experts kept per token (6) */
} mv_moe_shape;

/* Device pointers to one layer's weights (bf16 bits unless noted). */
typedef struct {
  const uint16_t* w_router;  /* [E][H] */
  const float* router_bias;  /* [E] fp32 added to the router logits, or NULL */
  const uint16_t* w_gate;    /* [E][I][H] */
  const uint16_t* w_up;      /* [E][I][H] */
  const uint16_t* w_down;    /* [E][H][I] */
  const uint16_t* ws_gate;   /* [I_shared][H]  (NULL when I_shared == 0) */
  const uint16_t* ws_up;     /* [I_shared][H] */
  const uint16_t* ws_down;   /* [H][I_shared] */
  /* [H] gain of the pre-RMSNorm variant of the layer, or NULL (plain layer).
   * With it, verify_step and speculative_step route and run the experts on
   * x = bf16(RMSNorm(h) * norm_gain) and keep the residual h:
   * h' = bf16(h + MoE(x)).  The pages name no norm (the model card's
   * architecture paragraph gives only the decoder's shape); this is the
   * DeepSeek-style decoder block without its attention.  moe_ffn_forward
   * ignores it: compose moe_rmsnorm, moe_router_topk and moe_ffn_forward
   * (x = the normalised rows, residual = h) instead. */
  const uint16_t* norm_gain;
} mv_moe_weights;

/* ---------------------------------------------------------------------------
 * moe_router_topk - router of one MoE layer (model card, architecture
 * paragraph: each token is routed to 6 of the 64 routed experts).
 * For every row r: logits l[e] = x[r] . w_router[e] (+ router_bias[e]) in
 * fp32; the k largest logits are kept (equal logits: lower expert id first),
 * slot j holding the j-th largest; topk_w[r][j] = softmax over all E logits
 * restricted to the kept experts and renormalised to sum 1.
 *   x          [T][H] bf16           topk_idx  [T][k] int32 (out)
 *   w_router   [E][H] bf16           topk_w    [T][k] fp32  (out)
 *   router_bias [E] fp32 or NULL
 * T = 0 is legal and launches nothing.
 * ------------------------------------------------------------------------- */
MV_API mv_status moe_router_topk(const uint16_t* x, int32_t T, const mv_moe_shape* shape,
                          const uint16_t* w_router, const float* router_bias,
                          int32_t* topk_idx, float* topk_w, mv_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_expert_permute - group the (row, slot) routing entries by expert (model
 * card, architecture paragraph: each token goes to 6 of 64 routed experts, so
 * an expert's FFN runs on the rows routed to it, gathered together).
 * Entry id i = r*k + j.  counts[e] = number of entries routed to e;
 * offsets[e] = sum of counts[e'] for e' < e, offsets[E] = T*k; perm lists the
 * entry ids grouped by expert, ascending within each expert; inv[i] is the
 * position of entry i in perm.  Integer, exact, deterministic.
 *   topk_idx [T][k] int32 in [0, E)   counts [E], offsets [E+1],
 *                                      perm [T*k], inv [T*k]  int32 (out)
 * ------------------------------------------------------------------------- */
MV_API mv_status moe_expert_permute(const int32_t* topk_idx, int32_t T, int32_t E, int32_t k,
                             int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                             mv_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_rmsnorm - out[r] = bf16((x[r] * s_r) * gain), s_r = 1 / sqrt(sum_h
 * x[r][h]^2 / H + 1e-6) in fp32 (products and sums singly rounded), for the
 * pre-RMSNorm layer variant (see mv_moe_weights.norm_gain).
 *   x, out [T][H] bf16 (may not alias), gain [H] bf16.  H a multiple of 8.
 * ------------------------------------------------------------------------- */
MV_API mv_status moe_rmsnorm(const uint16_t* x, int32_t T, int32_t H, const uint16_t* gain, uint16_t* out,
                             mv_stream_t stream);

/* Bytes of workspace moe_ffn_forward needs for T rows. */
MV_API size_t moe_ffn_workspace_size(int32_t T, const mv_moe_shape* shape);

/* ---------------------------------------------------------------------------
 * moe_ffn_forward - one MoE FFN layer given its routing (model card,
 * architecture paragraph: 64 routed experts plus 2 always-on shared experts,
 * each row's output mixing its 6 routed experts; model card, mixture-of-
 * experts paragraph: about 570M of the 3.4B parameters are active per token).
 * For every row r: m[r] = sum_j topk_w[r][j] * SwiGLU_{topk_idx[r][j]}(x[r])
 *                        + SwiGLU_shared(x[r]),
 * SwiGLU_e(x) = W_down[e] . bf16(silu(W_gate[e] . x) * (W_up[e] . x)),
 * products in bf16 x bf16 -> fp32, the activation rounded to bf16 once.
 * out[r] = bf16(residual[r] + m[r]), or bf16(m[r]) when residual is NULL.
 *   x, residual, out [T][H] bf16 (out may not alias x; it may alias residual)
 *   topk_idx [T][k] int32, topk_w [T][k] fp32 (e.g. from moe_router_topk)
 *   ws / ws_bytes: caller-owned device workspace, >= moe_ffn_workspace_size().
 * Grouping by expert, the grouped tensor-core GEMMs and the combine all run
 * on the stream; nothing returns to the host.
 * ------------------------------------------------------------------------- */
MV_API mv_status moe_ffn_forward(const uint16_t* x, int32_t T, const mv_moe_shape* shape,
                          const mv_moe_weights* weights, const int32_t* topk_idx,
                          const float* topk_w, const uint16_t* residual, uint16_t* out,
                          void* ws, size_t ws_bytes, mv_stream_t stream);

/* Bytes of workspace lm_head_argmax needs for T rows and a V-token vocabulary. */
MV_API size_t lm_head_workspace_size(int32_t T, int32_t V);

/* ---------------------------------------------------------------------------
 * lm_head_argmax - the verifier's own greedy choice per row (model card,
 * architecture paragraph: 129,280-token vocabulary; write-up, speculative
 * paragraph: drafts are kept only where they match the decoder's choice).
 * argmax[r] = argmax_v  h[r] . w_lm[v]  (fp32 logits; equal logits: the lower
 * v wins; -0 and +0 are equal).  The logits are never written to memory.
 *   h [T][H] bf16, w_lm [V][H] bf16, argmax [T] int32 (out)
 * ------------------------------------------------------------------------- */
MV_API mv_status lm_head_argmax(const uint16_t* h, int32_t T, int32_t H, const uint16_t* w_lm,
                         int32_t V, int32_t* argmax, void* ws, size_t ws_bytes,
                         mv_stream_t stream);

/* ---------------------------------------------------------------------------
 * greedy_accept - greedy acceptance of K drafts per sequence (model card,
 * introduction and decoding-speed paragraph; write-up, speculative paragraph).
 * With g = argmax[b*(K+1) .. b*(K+1)+K] and d = drafts[b][0..K-1]:
 *   accepted[b]   = largest a <= K with d[i] == g[i] for every i < a
 *   next_token[b] = g[a]
 *   emitted[b][j] = g[j] for j <= a, -1 for j > a  (emitted may be NULL)
 * so accepted[b] + 1 tokens are committed.  K = 0 is plain greedy decoding.
 * Draft ids outside [0, V) are legal and never match.
 *   argmax [B][K+1], drafts [B][K] (NULL allowed when K = 0), outputs int32.
 * ------------------------------------------------------------------------- */
MV_API mv_status greedy_accept(const int32_t* argmax, const int32_t* drafts, int32_t B, int32_t K,
                        int32_t* accepted, int32_t* next_token, int32_t* emitted,
                        mv_stream_t stream);

/* ---------------------------------------------------------------------------
 * lm_head_argmax_noalloc - lm_head_argmax for callers that must not allocate
 * device memory (the pages have no counterpart; this is an interface
 * convenience).  Some callers cannot call cudaMalloc: code embedded in a host
 * framework that owns every device allocation, or latency-critical threads
 * that may not take the allocator's locks and implicit synchronisation.  They
 * pass inputs and outputs only; the scratch (partial argmax keys, a work
 * counter and an error word) is a 4 MiB array built into the library, which
 * every GPU that loads the library holds until the process exits.
 *   Same arguments and result as lm_head_argmax, without ws / ws_bytes.
 *   Limit: ceil(V/256)*4*T*8 + 4352 bytes must fit in 4 MiB (T <= 259 rows
 *   at V = 129,280); larger sizes return MV_ERR_UNSUPPORTED_SHAPE and launch
 *   nothing.
 *   The first call on a device looks up the array's device address (this
 *   may load the library's device code); make that first call before any
 *   stream capture.  Later calls reuse the address while the device keeps
 *   the same CUDA context; after cudaDeviceReset the next call looks it up
 *   again.  Every call on a device shares the one array and clears
 *   its counter and error word on the stream, so calls that overlap on the
 *   GPU (other streams, other threads) race: serialise them.  If a bounded
 *   device-side wait ever runs out, every argmax of that call is -1.
 * ------------------------------------------------------------------------- */
MV_API mv_status lm_head_argmax_noalloc(const uint16_t* h, int32_t T, int32_t H, const uint16_t* w_lm,
                                        int32_t V, int32_t* argmax, mv_stream_t stream);

/* Bytes of workspace verify_step needs. */
MV_API size_t verify_step_workspace_size(int32_t B, int32_t K, const mv_moe_shape* shape, int32_t V);

/* ---------------------------------------------------------------------------
 * verify_step - the whole greedy speculative-verify step, fused into one
 * stream of launches with no host synchronisation:
 *   h_0 = hidden;  for l < n_layers:  route h_l (moe_router_topk with
 *   layers[l]), h_{l+1} = bf16(h_l + MoE_l(h_l)) (moe_ffn_forward with the
 *   residual);  g = lm_head_argmax(h_L);  greedy_accept(g, drafts).
 * The residual add between layers is a reading of the pages (they name no
 * norms or residuals); n_layers = 12 is the model card's decoder depth.
 *   hidden  [B*(K+1)][H] bf16, not modified     drafts [B][K] int32
 *   layers  HOST array of n_layers weight sets (device pointers inside)
 *   w_lm    [V][H] bf16
 *   accepted, next_token [B]; emitted [B][K+1] (nullable); argmax [B*(K+1)]
 *   (nullable: the verifier's choice for every row) - all int32 outputs.
 * ------------------------------------------------------------------------- */
MV_API mv_status verify_step(const uint16_t* hidden, const int32_t* drafts, int32_t B, int32_t K,
                      const mv_moe_shape* shape, const mv_moe_weights* layers,
                      int32_t n_layers, const uint16_t* w_lm, int32_t V, int32_t* accepted,
                      int32_t* next_token, int32_t* emitted, int32_t* argmax, void* ws,
                      size_t ws_bytes, mv_stream_t stream);

/* ---------------------------------------------------------------------------
 * FastMTP draft block (jina-ocr-v1 model card, decoding-speed paragraph, and
 * the tldrocket write-up's speculative paragraph: the drafts come from one
 * dense draft block applied recursively for K steps, not K separate heads).
 * The pages give the block no shape; this library's reading is:
 *   u_j  = [ RMSNorm(h_{j-1}) * g_hidden ; RMSNorm(w_emb[t_{j-1}]) * g_embed ]
 *   z_j  = bf16(u_j . w_proj^T)                      w_proj [H][2H]
 *   h_j  = bf16(z_j + SwiGLU(z_j))                   dense, intermediate I_d
 *   t_j  = argmax_v h_j . w_lm[v]  (the verifier's LM head; ties to lower v)
 * for j = 1..K, from h_0 = the verifier's last hidden state and t_0 = the
 * verifier's next token; drafts = t_1..t_K.  RMSNorm(x) = x / sqrt(mean(x^2)
 * + 1e-6) in fp32; u, z and the SwiGLU activation are rounded to bf16 (they
 * feed bf16 MMAs).
 * All weights are bf16 device pointers, row-major, 16-byte aligned:
 *   w_emb [V][H], g_hidden [H], g_embed [H], w_proj [H][2H],
 *   w_gate [I_d][H], w_up [I_d][H], w_down [H][I_d];  I_d a multiple of 64.
 * ------------------------------------------------------------------------- */
typedef struct {
  const uint16_t* w_emb;
  const uint16_t* g_hidden;
  const uint16_t* g_embed;
  const uint16_t* w_proj;
  const uint16_t* w_gate;
  const uint16_t* w_up;
  const uint16_t* w_down;
  int32_t I_d;
} mv_draft_weights;

/* Bytes of workspace fastmtp_draft needs. */
MV_API size_t fastmtp_draft_workspace_size(int32_t B, int32_t K, int32_t H, int32_t I_d, int32_t V);

/* fastmtp_draft - K recursive draft-block steps for B sequences.
 *   h0 [B][H] bf16 (the verifier's last hidden state of each sequence),
 *   t0 [B] int32 (its next token, in [0, V); another value is reported as
 *   MV_ERR_INTERNAL by mv_sync_status and drafts from embedding row 0),
 *   w_lm [V][H] bf16 (the verifier's LM head), drafts [B][K] int32 output,
 *   h_steps [K][B][H] bf16 output of every step (nullable).
 * Asynchronous on `stream`; device-side errors land in the workspace's sticky
 * word (mv_sync_status).  K = 0 or B = 0 launches nothing. */
MV_API mv_status fastmtp_draft(const uint16_t* h0, const int32_t* t0, int32_t B, int32_t K, int32_t H,
                               const mv_draft_weights* draft, const uint16_t* w_lm, int32_t V,
                               int32_t* drafts, uint16_t* h_steps, void* ws, size_t ws_bytes,
                               mv_stream_t stream);

/* Bytes of workspace speculative_step needs. */
MV_API size_t speculative_step_workspace_size(int32_t B, int32_t K, const mv_moe_shape* shape, int32_t I_d,
                                              int32_t V);

/* speculative_step - one iteration of the draft-and-verify loop on the GPU:
 * verify_step (same arguments and outputs), then fastmtp_draft from the
 * verifier's final hidden state at each sequence's last kept row
 * (row b*(K+1) + accepted[b] of h_L) and its next token, writing the K
 * drafts the next iteration verifies to next_drafts [B][K] (may not alias
 * drafts).  One stream of launches, no host synchronisation. */
MV_API mv_status speculative_step(const uint16_t* hidden, const int32_t* drafts, int32_t B, int32_t K,
                                  const mv_moe_shape* shape, const mv_moe_weights* layers, int32_t n_layers,
                                  const uint16_t* w_lm, int32_t V, const mv_draft_weights* draft,
                                  int32_t* accepted, int32_t* next_token, int32_t* emitted, int32_t* argmax,
                                  int32_t* next_drafts, void* ws, size_t ws_bytes, mv_stream_t stream);

/* ---------------------------------------------------------------------------
 * verify_graph_* - verify_step recorded once into a CUDA graph and replayed.
 * The model card's decoding-speed paragraph reports that replaying the
 * decoder as CUDA graphs changes which draft count K is fastest at batch 1,
 * because a batch-1 step is bound by launch latency more than by bytes.
 *
 * verify_graph_create takes exactly verify_step's arguments (same meaning,
 * layout and checks; the stream is replaced by the handle out-parameter) and
 * records the step on a private stream without running it.  Every pointer,
 * size, the weights and the device-wait bound in force
 * (mv_set_wait_timeout_ns) are fixed in the graph: before each replay the
 * caller writes the step's inputs into the SAME hidden and drafts buffers, and
 * reads the outputs from the same output buffers after it.
 * verify_graph_launch replays the step on `stream` (asynchronous, like
 * verify_step); replays on one workspace must not overlap in time, so launch
 * them on one stream or order them with events.  Device-side errors land in
 * the workspace's sticky word as with verify_step (read by mv_sync_status).
 * verify_graph_kernels gives the number of kernels one replay launches
 * (mv_launch_count advances by it per replay); verify_graph_destroy frees the
 * graph (NULL is allowed).  The handle is owned by the caller and belongs to
 * the device that was current at creation.  Creation fails with
 * MV_ERR_INVALID_ARG while mv_profile_enable is on (its per-launch events
 * cannot be recorded into a graph) and with MV_ERR_CUDA if the CUDA runtime
 * refuses to record or instantiate the graph.
 * ------------------------------------------------------------------------- */
typedef struct mv_verify_graph mv_verify_graph;

MV_API mv_status verify_graph_create(const uint16_t* hidden, const int32_t* drafts, int32_t B, int32_t K,
                                     const mv_moe_shape* shape, const mv_moe_weights* layers,
                                     int32_t n_layers, const uint16_t* w_lm, int32_t V, int32_t* accepted,
                                     int32_t* next_token, int32_t* emitted, int32_t* argmax, void* ws,
                                     size_t ws_bytes, mv_verify_graph** graph);
MV_API mv_status verify_graph_launch(mv_verify_graph* graph, mv_stream_t stream);
MV_API int32_t verify_graph_kernels(const mv_verify_graph* graph);
MV_API mv_status verify_graph_destroy(mv_verify_graph* graph);

/* ---------------------------------------------------------------------------
 * decode_attention - the decoder's self-attention on the verify rows, over a
 * key/value cache.  The jina-ocr-v1 model card (architecture paragraph) gives
 * the decoder's attention only a 32,768-position limit; the reading this call
 * follows is causal multi-head attention with as many key/value heads as query
 * heads (Q, K, V, O each H x H, which keeps the card's ~570M active
 * parameters per token) and head dim 128 (10 heads at H = 1280), keys
 * rotated before they enter the cache.
 * Sequence b holds ctx_len[b] earlier positions; this step's K+1 rows sit at
 * positions ctx_len[b] + j (their keys and values already written into the
 * cache).  For query row r = b*(K+1) + j and head h:
 *   s_p = (q[r][h] . k_cache[b][h][p]) / sqrt(128)   for p = 0..ctx_len[b]+j
 *   out[r][h] = sum_p softmax(s)_p * v_cache[b][h][p]
 * in fp32 (products of bf16 values, online softmax), rounded to bf16 once.
 *   q, out   [B*(K+1)][n_heads*128] bf16 (heads concatenated per row)
 *   k_cache, v_cache [B][n_heads][L_max][128] bf16 (head-major, each
 *            sequence's positions contiguous per head); positions past
 *            ctx_len[b]+K are never read into a result
 *   ctx_len  [B] int32, DEVICE memory; every value must satisfy
 *            0 <= ctx_len[b] <= max_ctx and ctx_len[b] + K + 1 <= L_max.  A
 *            value outside that range is not read past: the sequence's rows
 *            are left unwritten and mv_sync_status reports MV_ERR_INTERNAL.
 *   max_ctx  host-side bound on ctx_len (sizes the work split and workspace)
 * head_dim must be 128 and K <= 7 (MV_ERR_UNSUPPORTED_SHAPE otherwise).
 * The workspace holds the split results; calls on one workspace must not
 * overlap in time.
 * ------------------------------------------------------------------------- */
MV_API size_t decode_attention_workspace_size(int32_t B, int32_t K, int32_t n_heads, int32_t max_ctx);
MV_API mv_status decode_attention(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                                  const int32_t* ctx_len, int32_t B, int32_t K, int32_t n_heads, int32_t head_dim,
                                  int32_t L_max, int32_t max_ctx, uint16_t* out, void* ws, size_t ws_bytes,
                                  mv_stream_t stream);

/* Clears the workspace's header (its sticky error word) on the stream.  Call
 * once on a freshly allocated workspace before its first use (a workspace
 * allocated zero-filled needs no call). */
MV_API mv_status mv_workspace_init(void* ws, size_t ws_bytes, mv_stream_t stream);

/* Synchronises the stream, then reads and clears the sticky device error
 * word kept in a workspace used by moe_ffn_forward, lm_head_argmax or
 * verify_step.  Returns MV_OK, MV_ERR_TIMEOUT, MV_ERR_INTERNAL or MV_ERR_CUDA. */
MV_API mv_status mv_sync_status(void* ws, mv_stream_t stream);

/* Message for the last non-OK status returned on the calling thread. */
MV_API const char* mv_last_error(void);

/* Library version string. */
MV_API const char* mv_version(void);

/* ---------------------------------------------------------------------------
 * Instrumentation (off the hot path unless enabled).
 * mv_launch_count: kernels this library has launched in the process.
 * mv_profile_enable(1) brackets every subsequent kernel launch with CUDA
 * events on its stream; mv_profile_collect synchronises those events and
 * writes, per kernel kind (see mv_kernel_name), the number of launches and
 * the summed device milliseconds, then clears the record.  n_kinds is the
 * array length; returns the number of kinds written.
 * ------------------------------------------------------------------------- */
MV_API uint64_t mv_launch_count(void);
MV_API void mv_profile_enable(int32_t on);
MV_API int32_t mv_profile_collect(int64_t* launches, double* total_ms, int32_t n_kinds);
MV_API const char* mv_kernel_name(int32_t kind);

/* Test hook: the bound, in nanoseconds, on every device-side wait of later
 * launches (default 2e9).  Values <= 0 restore the default. */
MV_API void mv_set_wait_timeout_ns(int64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* MOE_VERIFY_H */
