/* Compiled (not run) by tests/test_abi.py: bha.h must be plain C99, self-contained, and
 * declare every entry point with the argument types used here. */
#include "bha.h"

typedef int (*featuremap_fn)(const bha_dims*, const void*, int32_t, const void*, void*, int32_t,
                             void*);
typedef int (*featuremap_checked_fn)(const bha_dims*, const void*, int32_t, const void*, void*,
                                     int32_t, int32_t*, void*);
typedef int (*hybrid_fn)(const bha_dims*, const int32_t*, const int32_t*, const void*, const void*,
                         const void*, const float*, const float*, const void*, const float*, void*,
                         int32_t*, void*);
typedef int (*hybrid_commit_fn)(const bha_dims*, const int32_t*, const int32_t*, const void*,
                                const void*, const void*, float*, float*, const void*,
                                const float*, void*, int32_t*, void*);
typedef int (*commit_fn)(const bha_dims*, const int32_t*, const int32_t*, const void*, const void*,
                         const void*, float*, float*, int32_t*, void*);
typedef int (*teacher_fn)(const bha_dims*, const int32_t*, const int32_t*, const void*, const void*,
                          const void*, int64_t, void*, void*, size_t, int32_t*, void*);
typedef int (*teacher_noalloc_fn)(const bha_dims*, const int32_t*, const int32_t*, const void*,
                                  const void*, const void*, int64_t, void*, int32_t*, void*);

int c_header_check(void) {
  featuremap_fn f0 = bha_featuremap;
  hybrid_fn f1 = bha_hybrid_attn;
  commit_fn f2 = bha_commit_block;
  teacher_fn f3 = bha_full_prefix_attn;
  teacher_noalloc_fn f4 = bha_full_prefix_attn_noalloc;
  size_t (*f5)(const bha_dims*, int64_t) = bha_full_prefix_workspace_bytes;
  const char* (*f6)(int) = bha_status_string;
  int (*f7)(const bha_dims*, int32_t) = bha_kernel_variant;
  int (*f8)(void) = bha_version;
  int (*f9)(int64_t, int32_t*, void*) = bha_selftest_bounded_wait;
  hybrid_commit_fn f10 = bha_hybrid_attn_commit;
  featuremap_checked_fn f11 = bha_featuremap_checked;
  bha_dims d = {1, 4, 1, 128, 256, 32, 32, 1, BHA_BF16};
  (void)d;
  return (f0 != 0) + (f1 != 0) + (f2 != 0) + (f3 != 0) + (f4 != 0) + (f5 != 0) + (f6 != 0) +
         (f7 != 0) + (f8 != 0) + (f9 != 0) + (f10 != 0) + (f11 != 0) + (BHA_NOALLOC_SCRATCH_BYTES > 0) + (BHA_OK == 0) +
         (BHA_ERR_TIMEOUT < 0) + (BHA_F32 == 1);
}
