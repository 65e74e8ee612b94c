/* A plain C99 caller of libmsa: the boundary needs no C++, Python or torch.
 * Host-only: it sizes workspaces and checks that argument errors come back as
 * status codes before any device work (no GPU is needed).  Built and run by
 * tests/test_abi_host.py. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "msa.h"

static int failures = 0;

static void expect(int cond, const char* what) {
  if (!cond) {
    printf("FAIL: %s\n", what);
    ++failures;
  }
}

int main(void) {
  /* the 128K prefill workload: 64 query heads over 8 KV groups, d = 128,
   * index dim 64, 16 blocks of 128 tokens */
  msa_shape s;
  memset(&s, 0, sizeof s);
  s.batch = 1;
  s.seq_q = 131072;
  s.seq_kv = 131072;
  s.q_offset = 0;
  s.n_q_heads = 64;
  s.n_kv_heads = 8;
  s.head_dim = 128;
  s.index_dim = 64;
  s.block = 128;
  s.topk = 16;

  size_t bytes = 0;
  expect(msa_workspace_size(&s, MSA_OP_INDEX_SCORES, &bytes) == MSA_OK && bytes == 0,
         "index scores need no workspace");
  /* partial outputs alone: T * G * k entries x r heads x d bf16 = 32 GiB */
  expect(msa_workspace_size(&s, MSA_OP_SPARSE_PREFILL, &bytes) == MSA_OK &&
             bytes > (size_t)32 << 30,
         "prefill workspace holds the partial outputs");
  size_t fwd = 0;
  expect(msa_workspace_size(&s, MSA_OP_FORWARD, &fwd) == MSA_OK && fwd > bytes,
         "forward adds pooled scores and the selection");
  expect(msa_workspace_size(&s, MSA_OP_SPARSE_DECODE, &bytes) == MSA_ERR_INVALID_SHAPE,
         "decode needs T == 1");
  expect(msa_workspace_size(&s, MSA_OP_FORWARD, NULL) == MSA_ERR_NULL_PTR, "NULL size pointer");

  msa_shape d = s;
  d.batch = 32;
  d.seq_q = 1;
  d.q_offset = d.seq_kv - 1;
  expect(msa_workspace_size(&d, MSA_OP_SPARSE_DECODE, &bytes) == MSA_OK && bytes > 0,
         "decode workspace");

  msa_shape bad = s;
  bad.block = 64;
  expect(msa_workspace_size(&bad, MSA_OP_FORWARD, &bytes) == MSA_ERR_UNSUPPORTED,
         "block 64 is unsupported");
  bad = s;
  bad.n_q_heads = 60;
  expect(msa_workspace_size(&bad, MSA_OP_FORWARD, &bytes) == MSA_ERR_INVALID_SHAPE,
         "H not a multiple of G");

  /* pointer checks run before the device is touched: these addresses are
   * never dereferenced */
  const uint16_t* p16 = (const uint16_t*)(uintptr_t)(1u << 20);
  uint16_t* o16 = (uint16_t*)(uintptr_t)(1u << 20);
  const uint16_t* odd = (const uint16_t*)(uintptr_t)((1u << 20) + 8);
  void* ws = (void*)(uintptr_t)(1u << 20);
  expect(msa_forward(&s, NULL, p16, p16, p16, p16, o16, NULL, NULL, ws, fwd, NULL) ==
             MSA_ERR_NULL_PTR,
         "NULL q");
  expect(msa_forward(&s, odd, p16, p16, p16, p16, o16, NULL, NULL, ws, fwd, NULL) ==
             MSA_ERR_MISALIGNED,
         "q not 16-byte aligned");
  expect(msa_forward(&s, p16, p16, p16, p16, p16, o16, NULL, NULL, ws, 16, NULL) ==
             MSA_ERR_WORKSPACE_TOO_SMALL,
         "workspace too small");
  expect(msa_forward_decode_paged(&d, 0, NULL, NULL, p16, p16, p16, p16, p16, o16, NULL, NULL,
                                  ws, fwd, NULL) == MSA_ERR_INVALID_SHAPE,
         "paged decode with an empty pool");

  for (int c = MSA_OK; c <= MSA_ERR_DEVICE_TIMEOUT; ++c)
    expect(msa_status_string((msa_status)c) != NULL, "status string");

  if (failures == 0) printf("ok\n");
  return failures == 0 ? 0 : 1;
}
