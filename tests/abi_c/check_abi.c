/* A plain C11 caller of the verify-step library, built against
 * include/moe_verify.h and linked to the shared library.  It needs no GPU:
 * it checks that the header is valid C, that the structs have the layout the
 * library reads, that the host-side size queries answer, and that bad
 * arguments are rejected on the host before anything is launched.
 * Exit status 0 = every check passed. */
#include <stddef.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "moe_verify.h"

static int failures = 0;

#define CHECK(cond, what)                                        \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "FAIL %s (line %d)\n", what, __LINE__);    \
      ++failures;                                                \
    }                                                            \
  } while (0)

/* A 16-byte aligned address that is never dereferenced on the host. */
#define FAKE ((const void*)(uintptr_t)(1u << 20))

int main(void) {
  /* struct layouts the library relies on */
  CHECK(sizeof(mv_moe_shape) == 5 * sizeof(int32_t), "mv_moe_shape size");
  CHECK(sizeof(mv_moe_weights) == 9 * sizeof(void*), "mv_moe_weights size");
  CHECK(offsetof(mv_moe_weights, norm_gain) == 8 * sizeof(void*), "norm_gain offset");
  CHECK(offsetof(mv_draft_weights, I_d) == 7 * sizeof(void*), "mv_draft_weights I_d offset");

  const char* v = mv_version();
  CHECK(v && strstr(v, "sm_100a") != NULL, "version names the architecture");

  mv_moe_shape s = {1280, 64, 896, 1792, 6};
  const size_t ws_verify = verify_step_workspace_size(32, 3, &s, 129280);
  const size_t ws_ffn = moe_ffn_workspace_size(128, &s);
  const size_t ws_lm = lm_head_workspace_size(128, 129280);
  const size_t ws_draft = fastmtp_draft_workspace_size(32, 3, 1280, 1792, 129280);
  const size_t ws_spec = speculative_step_workspace_size(32, 3, &s, 1792, 129280);
  CHECK(ws_verify > ws_ffn && ws_ffn > 0 && ws_lm > 0 && ws_draft > 0, "workspace sizes");
  CHECK(ws_spec >= ws_verify + ws_draft, "speculative_step workspace covers both parts");
  CHECK(verify_step_workspace_size(-1, 3, &s, 129280) == 0, "negative B has no workspace");

  /* host-side argument checks: nothing is launched, no GPU is touched */
  mv_moe_weights w;
  memset(&w, 0, sizeof(w));
  w.w_router = FAKE;
  w.w_gate = FAKE;
  w.w_up = FAKE;
  w.w_down = FAKE;
  w.ws_gate = FAKE;
  w.ws_up = FAKE;
  w.ws_down = FAKE;
  int32_t* out = (int32_t*)FAKE;
  mv_status st = verify_step(NULL, (const int32_t*)FAKE, 32, 3, &s, &w, 1, (const uint16_t*)FAKE, 129280, out,
                             out, NULL, NULL, (void*)FAKE, ws_verify, NULL);
  CHECK(st == MV_ERR_INVALID_ARG, "NULL hidden");
  CHECK(strlen(mv_last_error()) > 0, "an error message");
  st = verify_step((const uint16_t*)((uintptr_t)FAKE + 2), (const int32_t*)FAKE, 32, 3, &s, &w, 1,
                   (const uint16_t*)FAKE, 129280, out, out, NULL, NULL, (void*)FAKE, ws_verify, NULL);
  CHECK(st == MV_ERR_MISALIGNED, "misaligned hidden");
  st = verify_step((const uint16_t*)FAKE, (const int32_t*)FAKE, 32, 3, &s, &w, 1, (const uint16_t*)FAKE, 129283,
                   out, out, NULL, NULL, (void*)FAKE, ws_verify, NULL);
  CHECK(st == MV_ERR_UNSUPPORTED_SHAPE, "V not a multiple of 8");
  st = verify_step((const uint16_t*)FAKE, (const int32_t*)FAKE, 32, 3, &s, &w, 1, (const uint16_t*)FAKE, 129280,
                   out, out, NULL, NULL, (void*)FAKE, ws_verify - 1, NULL);
  CHECK(st == MV_ERR_WORKSPACE_TOO_SMALL, "workspace one byte short");
  w.norm_gain = (const uint16_t*)((uintptr_t)FAKE + 8);
  st = verify_step((const uint16_t*)FAKE, (const int32_t*)FAKE, 32, 3, &s, &w, 1, (const uint16_t*)FAKE, 129280,
                   out, out, NULL, NULL, (void*)FAKE, ws_verify, NULL);
  CHECK(st == MV_ERR_MISALIGNED, "misaligned norm gain");
  w.norm_gain = NULL;
  mv_moe_shape bad = {1280, 64, 900, 1792, 6};
  st = moe_router_topk((const uint16_t*)FAKE, 4, &bad, (const uint16_t*)FAKE, NULL, out, (float*)FAKE, NULL);
  CHECK(st == MV_ERR_UNSUPPORTED_SHAPE, "I not a multiple of 64");
  st = greedy_accept((const int32_t*)FAKE, NULL, 4, 3, out, out, NULL, NULL);
  CHECK(st == MV_ERR_INVALID_ARG, "K > 0 needs drafts");
  mv_draft_weights d;
  memset(&d, 0, sizeof(d));
  d.I_d = 1792;
  st = fastmtp_draft((const uint16_t*)FAKE, (const int32_t*)FAKE, 32, 3, 1280, &d, (const uint16_t*)FAKE, 129280,
                     out, NULL, (void*)FAKE, ws_draft, NULL);
  CHECK(st == MV_ERR_INVALID_ARG, "draft weights missing");
  mv_verify_graph* g = (mv_verify_graph*)FAKE;
  st = verify_graph_create(NULL, NULL, 32, 3, &s, &w, 1, (const uint16_t*)FAKE, 129280, out, out, NULL, NULL,
                           (void*)FAKE, ws_verify, &g);
  CHECK(st == MV_ERR_INVALID_ARG && g == NULL, "graph creation checks like verify_step");
  CHECK(verify_graph_kernels(NULL) == -1, "no graph, no kernels");
  CHECK(verify_graph_destroy(NULL) == MV_OK, "destroying NULL is allowed");

  if (failures == 0) printf("C ABI checks passed\n");
  return failures == 0 ? 0 : 1;
}
