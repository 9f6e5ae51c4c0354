/* A plain C99 caller of the library: includes include/moe.h alone (no CUDA or torch header),
 * links against libmoe_b200.so, takes the address of every entry point and makes the host-only
 * calls, which need no GPU: the workspace size of the DeepSeek-V3-shaped layer and the rejection
 * of a bad configuration. Prints "ok <workspace bytes>" or what failed. */
#include <stdio.h>
#include <string.h>

#include "moe.h"

typedef void (*any_fn)(void);

int main(void) {
  const any_fn entry[] = {
      (any_fn)moe_workspace_size, (any_fn)moe_route,          (any_fn)moe_permute,
      (any_fn)moe_expert_ffn,     (any_fn)moe_combine,        (any_fn)moe_layer_forward,
      (any_fn)moe_quantize_fp8,   (any_fn)moe_route_hash,     (any_fn)moe_bias_update,
      (any_fn)moe_route_static_scratch, (any_fn)moe_ep_workspace_size, (any_fn)moe_ep_layer_forward,
      (any_fn)moe_ep_export_handle, (any_fn)moe_ep_open_handle, (any_fn)moe_ep_close_handle,
      (any_fn)moe_sync_status,    (any_fn)moe_status_string};
  size_t i;
  for (i = 0; i < sizeof entry / sizeof entry[0]; ++i) {
    if (!entry[i]) {
      printf("entry point %u unresolved\n", (unsigned)i);
      return 1;
    }
  }
  moe_config c;
  memset(&c, 0, sizeof c);
  c.d_model = 7168;
  c.n_routed = 256;
  c.n_shared = 1;
  c.top_k = 8;
  c.n_group = 8;
  c.topk_group = 4;
  c.moe_intermediate_size = 2048;
  c.score_fn = MOE_SCORE_SIGMOID;
  c.renormalize = 1;
  c.routed_scaling_factor = 2.5f;
  c.cap_policy = MOE_CAP_NONE;
  c.dtype = MOE_BF16;
  size_t bytes = 0;
  moe_status st = moe_workspace_size(&c, 16384, &bytes);
  if (st != MOE_OK || bytes == 0) {
    printf("workspace size: %s\n", moe_status_string(st));
    return 1;
  }
  c.top_k = 0;
  size_t ignored = 0;
  if (moe_workspace_size(&c, 16384, &ignored) != MOE_ERR_INVALID_ARG) {
    printf("top_k = 0 accepted\n");
    return 1;
  }
  if (strcmp(moe_status_string(MOE_OK), moe_status_string(MOE_ERR_TIMEOUT)) == 0) {
    printf("status strings not distinct\n");
    return 1;
  }
  printf("ok %llu\n", (unsigned long long)bytes);
  return 0;
}
