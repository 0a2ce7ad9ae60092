/* A plain C99 consumer of the library's C ABI: it includes include/hstu.h,
 * links against libhstu.so, takes the address of every declared entry point
 * (so the link must resolve each one) and calls the ones that need no GPU.
 * Built and run by tests/test_abi.py. */
#include <stdio.h>
#include <string.h>

#include "hstu.h"

typedef void (*any_fn)(void);

int main(void) {
  const any_fn entry_points[] = {
      (any_fn)hstu_create, (any_fn)hstu_destroy, (any_fn)hstu_layer_forward,
      (any_fn)hstu_stack_forward, (any_fn)hstu_status_string, (any_fn)hstu_get_device_error,
      (any_fn)hstu_time_bucket_thresholds, (any_fn)hstu_set_kernel_timing,
      (any_fn)hstu_get_kernel_timing, (any_fn)hstu_attention_noalloc,
      (any_fn)hstu_cache_create, (any_fn)hstu_cache_destroy, (any_fn)hstu_cache_prefill,
      (any_fn)hstu_cache_score, (any_fn)hstu_stochastic_length_scratch_bytes,
      (any_fn)hstu_stochastic_length, (any_fn)hstu_copy_intermediate,
      (any_fn)hstu_debug_attention_buckets, (any_fn)hstu_debug_umma_tile,
      (any_fn)hstu_attention_backward, (any_fn)hstu_layer_backward,
      (any_fn)hstu_attention_forward, (any_fn)hstu_set_wait_limit};
  size_t i, n = sizeof(entry_points) / sizeof(entry_points[0]);
  for (i = 0; i < n; ++i)
    if (entry_points[i] == NULL) return 2;
  printf("entry_points %u\n", (unsigned)n);

  {
    int64_t thr[128];
    if (hstu_time_bucket_thresholds(0.301, 128, thr) != HSTU_OK) return 3;
    printf("thresholds %lld %lld %lld %lld\n", (long long)thr[0], (long long)thr[1],
           (long long)thr[3], (long long)thr[40]);
  }
  printf("status %s\n", hstu_status_string(HSTU_ERR_WORKSPACE));
  {
    hstu_config cfg;
    hstu_handle* h = NULL;
    memset(&cfg, 0, sizeof cfg);
    cfg.d_model = 256;
    cfg.num_heads = 3;            /* 256 != 3 * 85: rejected before any CUDA call */
    cfg.head_dim = 85;
    printf("create %d %s\n", (int)hstu_create(&cfg, 0, &h), h == NULL ? "null" : "set");
  }
  printf("sl_scratch %lu\n", (unsigned long)hstu_stochastic_length_scratch_bytes(1000, 10));
  return 0;
}
