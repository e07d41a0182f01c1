/* A plain C11 caller of the library, built by tests/test_c_consumer.py.
 *
 * It includes moe_b200.h as C, links libmoe_b200.so with no C++ and no torch,
 * and exercises the calls that need no GPU: configuration checks, the size and
 * layout queries, status strings, and argument validation that returns before
 * any CUDA call.  It prints one "key value..." line per result for the test
 * to compare against the Python binding. */
#include <stdint.h>
#include <stdio.h>

#include "moe_b200.h"

static void print_layout(const char* name, const moe_config* cfg) {
  moe_weights_layout lay;
  moe_status st = moe_get_weights_layout(cfg, &lay);
  printf("%s %d %lld %lld %lld %lld %lld %lld\n", name, (int)st, (long long)lay.w13_codes, (long long)lay.w13_sf,
         (long long)lay.w2_codes, (long long)lay.w2_sf, (long long)lay.scales, (long long)lay.total_bytes);
}

int main(void) {
  const moe_config nv = {384, 8, 4096, 2560, MOE_NVFP4};
  const moe_config mx = {384, 8, 4096, 2560, MOE_MXFP8};
  const moe_config bad_k = {384, 9, 4096, 2560, MOE_NVFP4};
  const moe_config small = {8, 2, 256, 128, MOE_NVFP4};
  int64_t T;

  printf("check %d %d %d\n", (int)moe_check_config(&nv), (int)moe_check_config(&mx), (int)moe_check_config(&bad_k));
  print_layout("layout_nvfp4", &nv);
  print_layout("layout_mxfp8", &mx);
  for (T = 0; T <= 8192; T = T ? T * 8 : 1) {
    printf("rows %lld %lld %lld\n", (long long)T, (long long)moe_max_rows(&nv, T),
           (long long)moe_route_workspace_bytes(&nv, T));
  }
  printf("codes %lld %lld %lld %lld\n", (long long)moe_codes_bytes(&nv, 128, 4096),
         (long long)moe_codes_bytes(&mx, 128, 4096), (long long)moe_sf_bytes(&nv, 128, 4096),
         (long long)moe_sf_bytes(&mx, 256, 2560));
  printf("sf_offset %lld %lld\n", (long long)moe_sf_offset(130, 5, 256), (long long)moe_sf_offset(31, 3, 4));
  printf("status_string %s\n", moe_status_string(MOE_ERR_WORKSPACE));

  /* argument validation: no pointer is dereferenced and no CUDA call is made */
  printf("null_logits %d\n", (int)moe_route_topk(&small, 4, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL));
  printf("bad_config %d\n", (int)moe_unpermute_combine(&bad_k, 4, NULL, NULL, NULL, NULL, NULL));
  printf("empty_permute %d\n", (int)moe_permute(&small, 0, NULL, NULL, NULL, NULL, NULL, NULL));
  return 0;
}
