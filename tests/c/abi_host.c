/* A C99 caller of libspark_attn.so: the header compiles as C, the library links, and the host-side
 * entry points (layer schedule, cache and workspace sizes, argument checks) answer without a GPU.
 * Prints one line per fact for the Python test to compare. */
#include <stdio.h>
#include "spark_attn.h"

int main(void) {
  int layer;
  for (layer = 0; layer < 36; ++layer) {
    spark_layer_cfg c;
    if (spark_layer_cfg_for_layer(layer, &c) != SPARK_OK) return 1;
    printf("layer %d kind %d rot %d theta %.1f window %d heads %d %d dim %d\n", layer, c.kind, c.rot_dim, c.theta,
           c.window, c.n_q, c.n_kv, c.head_dim);
  }
  {
    spark_layer_cfg bad;
    printf("layer 36 status %d\n", spark_layer_cfg_for_layer(36, &bad));
  }
  {
    spark_layer_cfg full, sliding;
    spark_layer_cfg_for_kind(SPARK_FULL, &full);
    spark_layer_cfg_for_kind(SPARK_SLIDING, &sliding);
    printf("kv bytes full 1 token %lld\n", spark_kv_cache_bytes(&full, 1, 1));
    printf("kv bytes q8 full 1 token %lld\n", spark_kv_cache_q8_bytes(&full, 1, 1));
    printf("stack bytes 1 sequence 131072 %lld\n", spark_stack_kv_bytes(1, 131072));
    printf("prefill q8 workspace sliding B=2 %zu\n", spark_prefill_q8_workspace_bytes(2, 512, &sliding));
    printf("prefill q8 workspace sliding cap 600 %zu\n", spark_prefill_q8_workspace_bytes(1, 600, &sliding));
    /* an argument error is returned before any device call, with its message */
    printf("prefill unknown flags status %d\n",
           spark_attn_prefill((void*)16, (void*)16, (void*)16, (void*)16, (void*)16, 0, 0, 0, 1, 128, 0, 0, 0, 0,
                              (const int*)16, &full, 0x80u, 0));
    printf("last error set %d\n", spark_last_error() != 0 && spark_last_error()[0] != 0);
  }
  return 0;
}
