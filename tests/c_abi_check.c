/* A plain C99 caller of the DSA library's C ABI (include/dsa.h), built and run on the CPU
 * by tests/test_c_abi_cpu.py: the header compiles as C, the library links from C, and the
 * host-side entry points behave as declared. No call here reaches a kernel launch: each
 * one fails its argument checks first, or only computes a size. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "dsa.h"

static int failures = 0;

static void expect(int cond, const char* what) {
  if (!cond) {
    printf("FAIL %s\n", what);
    ++failures;
  }
}

int main(void) {
  int32_t seq_lens_dummy = 0, table_dummy = 0;
  void* fake = (void*)(uintptr_t)0x100000; /* never dereferenced */
  dsa_paging pg;
  memset(&pg, 0, sizeof pg);
  pg.B = 2;
  pg.n_q = 1;
  pg.seq_lens = &seq_lens_dummy;
  pg.q_pos = NULL;
  pg.block_table = &table_dummy;
  pg.max_pages_per_seq = 4;
  pg.page_size = 64;
  pg.num_pages = 8;

  /* status strings exist for every code */
  for (int s = DSA_OK; s <= DSA_ERR_TIMEOUT; ++s) {
    const char* msg = dsa_status_string((dsa_status)s);
    expect(msg != NULL && msg[0] != '\0', "status string");
  }

  /* workspace sizes: 256-byte multiples, 0 for invalid requests */
  size_t idx = dsa_workspace_size(&pg, 256, 0, DSA_OP_INDEXER);
  size_t topk = dsa_workspace_size(&pg, 256, 16, DSA_OP_TOPK);
  size_t layer = dsa_workspace_size(&pg, 0, 16, DSA_OP_LAYER);
  size_t local = dsa_workspace_size(&pg, 256, 16, DSA_OP_SHARD_LOCAL);
  size_t select = dsa_workspace_size(&pg, 0, 16, DSA_OP_SHARD_SELECT);
  expect(idx >= 256 && idx % 256 == 0, "indexer workspace");
  expect(topk >= 256 && topk % 256 == 0, "top-k workspace");
  expect(layer > topk, "layer workspace holds the scores and index lists");
  expect(local >= 256 + 2 * 16 * 4, "shard-local workspace holds the local selection");
  expect(select >= 256, "shard-select workspace");
  expect(dsa_workspace_size(&pg, 0, 0, DSA_OP_LAYER) == 0, "invalid top_k");
  expect(dsa_workspace_size(NULL, 0, 16, DSA_OP_LAYER) == 0, "no paging");
  expect(dsa_workspace_size(&pg, 0, 16, 99) == 0, "unknown op");

  /* argument errors return before any launch */
  expect(dsa_indexer_scores(NULL, fake, DSA_FP8_E4M3, fake, fake, fake, DSA_FP8_E4M3, fake, fake, 256, fake, idx,
                            NULL) == DSA_ERR_INVALID_ARG, "indexer without paging");
  expect(dsa_topk_pagemap(&pg, fake, 256, 0, fake, fake, fake, topk, NULL) == DSA_ERR_INVALID_ARG,
         "top-k with top_k 0");
  expect(dsa_pagemap(&pg, NULL, 16, fake, fake, topk, NULL) == DSA_ERR_INVALID_ARG, "page map without input");
  expect(mla_sparse_decode(0, fake, fake, DSA_FP8_E4M3, fake, 1024, fake, 16, 0.1f, fake, DSA_BF16, NULL, fake,
                           1 << 20, NULL) == DSA_ERR_INVALID_ARG, "MLA with no queries");
  expect(dsa_shard_local_topk(&pg, fake, 256, 16, NULL, fake, fake, fake, local, NULL) == DSA_ERR_INVALID_ARG,
         "shard-local without offsets");
  expect(dsa_shard_select(&pg, 2, 2, fake, fake, 16, fake, fake, NULL, fake, select, NULL) == DSA_ERR_INVALID_ARG,
         "shard-select with rank out of range");
  expect(dsa_shard_merge(1, 2, fake, fake, fake, DSA_FP8_E4M3, NULL, NULL) == DSA_ERR_INVALID_ARG,
         "shard-merge to an fp8 output");
  expect(dsa_topk_pagemap(&pg, fake, 256, 16, fake, fake, fake, topk - 1, NULL) == DSA_ERR_WORKSPACE,
         "top-k with a short workspace");

  printf("%s %d\n", failures == 0 ? "OK" : "FAILED", failures);
  return failures == 0 ? 0 : 1;
}
