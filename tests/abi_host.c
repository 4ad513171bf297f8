/* A plain C99 caller of libmta.so that needs no GPU: it includes only
 * include/mta.h, links the library, and checks the host-side half of the ABI
 * (version, status strings, workspace queries, argument checks that return
 * before anything is enqueued).  tests/test_abi.py compiles it with gcc
 * -std=c99 -pedantic -Werror and runs it. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "mta.h"

static int fails = 0;

#define EXPECT(cond)                                          \
  do {                                                        \
    if (!(cond)) {                                            \
      printf("FAIL line %d: %s\n", __LINE__, #cond);          \
      ++fails;                                                \
    }                                                         \
  } while (0)

/* Distinct, 256-byte aligned addresses 1 GiB apart (so that no two tensors of
 * these shapes overlap) that the library never dereferences on the host: every
 * call below returns before any CUDA call. */
static void *fake(uintptr_t i) { return (void *)(((uintptr_t)1 << 36) + (i << 30)); }

static mta_cfg recipe(void) {
  mta_cfg c;
  memset(&c, 0, sizeof c);
  c.B = 4; c.H = 16; c.L = 2048; c.d = 128;
  c.c_q = 6; c.c_k = 11; c.c_h = 2;
  c.kq_place = MTA_PRE; c.head_place = MTA_POST; c.kq_post = 0;
  c.dtype = MTA_BF16; c.path = 0; c.scale = 0.f;
  return c;
}

int main(void) {
  mta_cfg c = recipe(), bad;
  const float *th = (const float *)fake(4), *w = (const float *)fake(5);
  size_t ws;
  mta_gn gn;

  EXPECT(mta_abi_version() == MTA_ABI_VERSION);
  EXPECT(strcmp(mta_status_string(MTA_OK), "ok") == 0);
  EXPECT(mta_status_string(MTA_ERR_TIMEOUT) != NULL);

  /* workspace queries: the contraction kernel's operands make the attention
   * workspace at least c_q*B*H*L*d fp16 convolved keys */
  ws = mta_attn_workspace_bytes(&c);
  EXPECT(ws >= (size_t)6 * 4 * 16 * 2048 * 128 * 2);
  EXPECT(mta_layer_workspace_bytes(&c) > ws);
  /* the backward: the status word and its tensor-core strips (one query block of
   * every head, several 128-row strips spanning the keys) */
  EXPECT(mta_attn_bwd_workspace_bytes(&c) > (size_t)256 + (size_t)4 * 16 * 128 * 2048 * 4);

  /* kernel choice on the host: the contraction kernel once its operands fit */
  EXPECT(mta_attn_kernel(&c) == -MTA_ERR_WORKSPACE);
  c.workspace_bytes = ws;
  EXPECT(mta_attn_kernel(&c) == 3);
  c.workspace_bytes = 256;
  EXPECT(mta_attn_kernel(&c) == 2);
  c = recipe();

  /* invalid configurations: no workspace size, MTA_ERR_INVALID from the call */
  bad = c; bad.c_k = 4;
  EXPECT(mta_attn_workspace_bytes(&bad) == 0);
  EXPECT(mta_attn_fwd(fake(1), fake(2), fake(3), th, w, &bad, fake(6)) == MTA_ERR_INVALID);
  bad = c; bad.L = 0;
  EXPECT(mta_attn_fwd(fake(1), fake(2), fake(3), th, w, &bad, fake(6)) == MTA_ERR_INVALID);
  bad = c; bad.H = 15;
  EXPECT(mta_attn_fwd(fake(1), fake(2), fake(3), th, w, &bad, fake(6)) == MTA_ERR_INVALID);
  EXPECT(mta_attn_fwd(fake(1), fake(2), fake(3), th, w, NULL, fake(6)) == MTA_ERR_INVALID);

  /* a null tensor, then a valid call without its workspace */
  EXPECT(mta_attn_fwd(NULL, fake(2), fake(3), th, w, &c, fake(6)) == MTA_ERR_INVALID);
  EXPECT(mta_attn_fwd(fake(1), fake(2), fake(3), th, w, &c, NULL) == MTA_ERR_INVALID);
  EXPECT(mta_attn_fwd(fake(1), fake(2), fake(3), th, w, &c, fake(6)) == MTA_ERR_WORKSPACE);
  c.workspace = fake(7);
  c.workspace_bytes = 64;
  EXPECT(mta_attn_fwd(fake(1), fake(2), fake(3), th, w, &c, fake(6)) == MTA_ERR_WORKSPACE);
  c = recipe();

  /* the layer and the backward pass check their arguments the same way */
  memset(&gn, 0, sizeof gn);
  gn.gamma = (const float *)fake(8);
  gn.beta = (const float *)fake(9);
  gn.depth_scale = -1.f;
  gn.layer = 12;
  EXPECT(mta_layer_fwd(fake(1), fake(2), th, w, NULL, fake(3), &c, fake(6)) == MTA_ERR_INVALID);
  EXPECT(mta_layer_fwd(fake(1), fake(2), th, w, &gn, fake(3), &c, fake(6)) == MTA_ERR_WORKSPACE);
  bad = c; bad.dtype = MTA_F32;
  EXPECT(mta_layer_fwd(fake(1), fake(2), th, w, &gn, fake(3), &bad, fake(6)) == MTA_ERR_UNSUPPORTED);
  EXPECT(mta_attn_bwd(fake(1), fake(2), fake(3), th, w, fake(10), &c, NULL, (float *)fake(12),
                      (float *)fake(13), NULL, NULL) == MTA_ERR_INVALID);
  bad = c; bad.path = 2;  /* no direct tensor-core backward */
  EXPECT(mta_attn_bwd(fake(1), fake(2), fake(3), th, w, fake(10), &bad, (float *)fake(11),
                      (float *)fake(12), (float *)fake(13), NULL, NULL) == MTA_ERR_UNSUPPORTED);
  bad = c; bad.path = 3;  /* the tensor-core backward: its strips do not fit the workspace */
  EXPECT(mta_attn_bwd(fake(1), fake(2), fake(3), th, w, fake(10), &bad, (float *)fake(11),
                      (float *)fake(12), (float *)fake(13), NULL, NULL) == MTA_ERR_WORKSPACE);
  EXPECT(mta_gemm_bf16_nt(fake(1), fake(2), fake(3), 128, 256, 60, NULL) == MTA_ERR_INVALID);

  /* an output that overlaps an input is refused before anything is enqueued */
  c.workspace = fake(7);
  c.workspace_bytes = ws;
  EXPECT(mta_attn_fwd(fake(1), fake(2), fake(3), th, w, &c, fake(3)) == MTA_ERR_INVALID);
  EXPECT(mta_attn_fwd(fake(1), fake(2), fake(3), th, w, &c, (char *)fake(1) + 4096) == MTA_ERR_INVALID);
  c = recipe();
  EXPECT(mta_sync_status(NULL) == MTA_ERR_INVALID);

  if (fails) return 1;
  printf("ok\n");
  return 0;
}
