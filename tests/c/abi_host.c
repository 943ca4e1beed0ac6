/* abi_host.c -- the C ABI from plain C, host-side paths only (no GPU needed): version and
 * status strings, workspace sizes, and argument checks that return before any launch.
 * Exit status 0 when every check holds; otherwise the number of failed checks. */
#include <stdio.h>
#include <string.h>

#include "diffattn.h"

static int failures = 0;

static void expect(int got, int want, const char* what) {
  if (got != want) {
    fprintf(stderr, "FAIL %s: got %d, want %d\n", what, got, want);
    ++failures;
  }
}

static diffattn_prefill_params v2_prefill(void) {
  diffattn_prefill_params p;
  memset(&p, 0, sizeof(p));
  p.variant = DIFFATTN_V2;
  p.dtype = DIFFATTN_BF16;
  p.batch = 1;
  p.seqlen = 256;
  p.n_q_heads = 16;
  p.n_kv_heads = 2;
  p.head_dim = 128;
  p.causal = 1;
  p.norm_eps = 1e-5f;
  p.q_strides[0] = 256 * 16 * 128; p.q_strides[1] = 16 * 128; p.q_strides[2] = 128;
  p.k_strides[0] = 256 * 2 * 128;  p.k_strides[1] = 2 * 128;  p.k_strides[2] = 128;
  p.v_strides[0] = 256 * 2 * 128;  p.v_strides[1] = 2 * 128;  p.v_strides[2] = 128;
  p.o_strides[0] = 256 * 8 * 128;  p.o_strides[1] = 8 * 128;  p.o_strides[2] = 128;
  return p;
}

int main(void) {
  expect(diffattn_version(), 100, "version");
  expect(strlen(diffattn_status_string(DIFFATTN_OK)) > 0, 1, "status string");
  expect(strlen(diffattn_status_string(-99)) > 0, 1, "status string of an unknown code");

  /* stand-in device addresses: validation fails before anything dereferences them */
  void* const A = (void*)(size_t)(1u << 20);
  void* const Bp = (void*)(size_t)((1u << 20) + 4096);

  diffattn_prefill_params p = v2_prefill();
  expect(diffattn_fwd_prefill(NULL, A, A, A, (const float*)A, NULL, Bp, NULL, NULL),
         DIFFATTN_ERR_INVALID_ARG, "prefill: no parameters");
  expect(diffattn_fwd_prefill(&p, A, Bp, Bp, (const float*)A, NULL, A, NULL, NULL),
         DIFFATTN_ERR_INVALID_ARG, "prefill: out aliases q");
  p.head_dim = 96;
  expect(diffattn_fwd_prefill(&p, A, A, A, (const float*)A, NULL, Bp, NULL, NULL),
         DIFFATTN_ERR_UNSUPPORTED, "prefill: bf16 V2 with d = 96");
  p = v2_prefill();
  p.kv_seqlen = 100;
  expect(diffattn_fwd_prefill(&p, A, A, A, (const float*)A, NULL, Bp, NULL, NULL),
         DIFFATTN_ERR_INVALID_ARG, "prefill: fewer keys than queries");
  p = v2_prefill();
  p.batch = 0;
  expect(diffattn_fwd_prefill(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL), DIFFATTN_OK,
         "prefill: empty batch launches nothing");

  size_t bytes = 0;
  p = v2_prefill();
  expect(diffattn_bwd_workspace_size(&p, &bytes), DIFFATTN_OK, "backward workspace");
  expect(bytes > 0, 1, "backward workspace is not empty");

  diffattn_decode_params d;
  memset(&d, 0, sizeof(d));
  d.variant = DIFFATTN_V2;
  d.dtype = DIFFATTN_BF16;
  d.batch = 4;
  d.max_kv_len = 1000;
  d.n_q_heads = 64;
  d.n_kv_heads = 8;
  d.head_dim = 128;
  d.num_splits = 3;
  d.q_strides[0] = 64 * 128; d.q_strides[1] = 128;
  d.kv_strides[0] = 1000 * 8 * 128; d.kv_strides[1] = 8 * 128; d.kv_strides[2] = 128;
  d.o_strides[0] = 32 * 128; d.o_strides[1] = 128;
  expect(diffattn_decode_workspace_size(&d, &bytes), DIFFATTN_OK, "decode workspace");
  expect(diffattn_fwd_decode(&d, A, A, A, NULL, (const float*)A, Bp, NULL, 0, NULL, NULL),
         DIFFATTN_ERR_WORKSPACE, "decode: no workspace");

  diffattn_paged_kv pk;
  memset(&pk, 0, sizeof(pk));
  pk.page_size = 12; /* not a power of two */
  pk.num_pages = 64;
  pk.max_pages_per_seq = 100;
  expect(diffattn_fwd_decode_paged(&d, &pk, A, A, A, (const int32_t*)A, NULL, (const float*)A, NULL,
                                   0, 1e-5f, Bp, A, bytes, NULL, NULL),
         DIFFATTN_ERR_INVALID_ARG, "paged decode: page size");

  expect(diffattn_lambda(NULL, NULL, NULL, NULL, 4, 64, 1, NULL, NULL, NULL),
         DIFFATTN_ERR_INVALID_ARG, "lambda: null vectors");
  expect(diffattn_selftest_timeout(NULL, 100, NULL), DIFFATTN_ERR_INVALID_ARG, "selftest: no status");

  if (failures == 0) printf("abi_host: all checks hold\n");
  return failures;
}
