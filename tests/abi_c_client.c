/* A plain C99 caller of libmla.so: include/mla.h compiled as C, the library linked as any C library.
 * Only host-side calls are made (handle, workspace arithmetic, argument validation, status strings),
 * so it runs without a GPU. Exit status 0 and "ok" on success; otherwise the number of the failed
 * check. Built and run by tests/test_abi_host.py. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "mla.h"

#define CHECK(n, cond)                              \
  do {                                              \
    if (!(cond)) {                                  \
      fprintf(stderr, "check %d failed\n", (n));    \
      return (n);                                   \
    }                                               \
  } while (0)

int main(void) {
  /* the DeepSeek-V3 layer: d, n_h, d_h, d_c, d_c', d_h^R, RoPE base */
  const mla_dims_t v3 = {7168, 128, 128, 512, 1536, 64, 10000.0};
  mla_handle_t *h = NULL;
  CHECK(1, mla_create(&v3, MLA_BF16, 0, &h) == MLA_OK && h != NULL);

  /* workspace arithmetic: the decode of 16 sequences, one query token each */
  size_t n = 0, off = 0;
  CHECK(2, mla_workspace_size(h, MLA_OP_DECODE, 16, 1, 0, &n) == MLA_OK && n > 0);
  CHECK(3, mla_workspace_offset(h, MLA_OP_DECODE, 16, 1, 0, MLA_BUF_OLAT, &off) == MLA_OK && off < n);
  CHECK(4, mla_workspace_offset(h, MLA_OP_DECODE, 16, 1, 0, MLA_BUF_KC, &off) == MLA_ERR_INVALID_ARG);
  CHECK(5, mla_workspace_size(h, MLA_OP_DECODE, 16, 3, 0, &n) == MLA_ERR_INVALID_ARG);

  /* host validation returns before any CUDA call: a null query, a misaligned cache, no weights */
  const uintptr_t a = 0x10000;   /* an aligned address that is never dereferenced */
  const int64_t *cu = (const int64_t *)a;
  CHECK(6, mla_decode(h, NULL, 16, 1, cu, (const void *)a, 65536, (void *)a, (void *)a, n, NULL) ==
               MLA_ERR_INVALID_ARG);
  CHECK(7, mla_decode(h, (const void *)a, 16, 1, cu, (const void *)(a + 2), 65536, (void *)a, (void *)a, n, NULL) ==
               MLA_ERR_ALIGNMENT);
  CHECK(8, mla_decode(h, (const void *)a, 16, 1, cu, (const void *)a, 65536, (void *)a, (void *)a, n, NULL) ==
               MLA_ERR_NO_WEIGHTS);

  /* the FP8 cache format: set, the prefill refuses it, the append's workspace grows by its staged rows */
  size_t ws16 = 0, ws8 = 0;
  CHECK(9, mla_workspace_size(h, MLA_OP_CACHE_APPEND, 0, 1, 700, &ws16) == MLA_OK);
  CHECK(10, mla_set_cache_format(h, MLA_CACHE_FP8) == MLA_OK);
  CHECK(11, mla_workspace_size(h, MLA_OP_CACHE_APPEND, 0, 1, 700, &ws8) == MLA_OK);
  CHECK(12, ws8 >= ws16 + (size_t)700 * 576 * 2);
  CHECK(13, mla_prefill(h, (const void *)a, 1, cu, 64, 64, (void *)a, 64, (void *)a, (void *)a, 1u << 30, NULL) ==
                MLA_ERR_UNSUPPORTED);
  CHECK(14, mla_set_cache_format(h, (mla_cache_format_t)2) == MLA_ERR_INVALID_ARG);
  CHECK(15, mla_set_cache_format(h, MLA_CACHE_BF16) == MLA_OK);

  /* routing and status strings */
  CHECK(16, mla_uses_tensor_cores(h, MLA_OP_DECODE) == 1);
  CHECK(17, strncmp(mla_status_string(MLA_ERR_ALIGNMENT), "MLA_ERR_ALIGNMENT", 17) == 0);
  mla_destroy(h);

  /* BF16 exists at the DeepSeek-V3 head layout only; FP32 runs the generic kernels at any size */
  const mla_dims_t tiny = {256, 4, 32, 64, 96, 16, 10000.0};
  h = NULL;
  CHECK(18, mla_create(&tiny, MLA_BF16, 0, &h) == MLA_ERR_UNSUPPORTED);
  CHECK(19, mla_create(&tiny, MLA_FP32, 0, &h) == MLA_OK && h != NULL);
  CHECK(20, mla_uses_tensor_cores(h, MLA_OP_DECODE) == 0);
  CHECK(21, mla_set_cache_format(h, MLA_CACHE_FP8) == MLA_ERR_UNSUPPORTED);
  mla_destroy(h);
  printf("ok\n");
  return 0;
}
