/* A plain C99 consumer of include/gemm_f16.h, compiled and run by
 * tests/test_c_abi.py on a machine without a GPU: every entry point is
 * referenced (so the program only links if the library exports them all with
 * C linkage), and the host-only ones are called and print their results. */
#include <stdint.h>
#include <stdio.h>

#include "gemm_f16.h"

typedef void (*any_fn)(void);

int main(void) {
  const any_fn entry_points[] = {
      (any_fn)gemm_relu_f16,         (any_fn)gemm_f16,
      (any_fn)gemm_f16_ex,           (any_fn)gemm_bias_act_f16,
      (any_fn)gemm_f16_general,      (any_fn)gemm_f16_config,
      (any_fn)gemm_config_smem_bytes, (any_fn)gemm_config_list,
      (any_fn)gemm_auto_config,      (any_fn)gemm_select_path,
      (any_fn)gemm_status_string,    (any_fn)gemm_get_device_status,
      (any_fn)gemm_selftest_wait_timeout, (any_fn)gemm_relu_f16_noalloc,
      (any_fn)gemm_f16_host,         (any_fn)gemm_relu_f16_host,
      (any_fn)gemm_host_plan_for,    (any_fn)gemm_f16_host_planned,
      (any_fn)gemm_host_release,     (any_fn)gemm_activation_f32,
      (any_fn)gemm_read_probe,       (any_fn)gemm_abi_version,
      (any_fn)gemm_release};
  const int n_entry = (int)(sizeof(entry_points) / sizeof(entry_points[0]));
  int i, missing = 0;
  for (i = 0; i < n_entry; ++i) missing += entry_points[i] == NULL;
  printf("entry_points %d missing %d\n", n_entry, missing);
  printf("abi %d\n", gemm_abi_version());
  printf("path_cube %d path_decode %d\n", gemm_select_path(8192, 8192, 8192),
         gemm_select_path(32, 28672, 8192));
  {
    gemm_host_plan p;
    const int rc = gemm_host_plan_for(8192, 8192, 8192, &p);
    printf("plan rc %d split %d panels %d extent %lld\n", rc, (int)p.split, (int)p.panels,
           (long long)p.panel_extent);
  }
  {
    gemm_config c = {GEMM_PATH_TILE_PAIR_TALL, 256, 4, 0, 0};
    printf("smem %d configs %d\n", gemm_config_smem_bytes(&c), gemm_config_list(NULL, 0));
  }
  /* argument errors come back before any device work */
  printf("bad_size %d empty %d\n",
         gemm_relu_f16(NULL, NULL, NULL, -1, 4, 4, 8, 8, 8, (gemm_stream_t)0),
         gemm_relu_f16(NULL, NULL, NULL, 0, 4, 4, 8, 8, 8, (gemm_stream_t)0));
  printf("status %s\n", gemm_status_string(GEMM_ERR_ALIGNMENT));
  return 0;
}
