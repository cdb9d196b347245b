/* Plain C99 client of the library: includes moe.h, links libmoe_b200.so and
 * calls the host-side entry points.  Built and run by tests/test_abi_host.py
 * on a machine without a GPU, where every call that would launch work must
 * refuse (MOE_ERR_CUDA), never fall back to the CPU. */
#include <stdint.h>
#include <stdio.h>

#include "moe.h"

int main(void) {
  moe_shape s = {64, 256, 8, 2, 512, 0};
  size_t ws_bytes = moe_workspace_size(&s);
  int64_t load[8] = {9, 1, 1, 1, 1, 1, 1, 1};
  int32_t p2l[10], off[9], phys[10];
  int plan = moe_eplb_plan(load, 8, 2, 2, p2l, off, phys);
  /* fake, aligned device addresses: never dereferenced without a device */
  void* a = (void*)(uintptr_t)(1u << 20);
  int fwd = moe_forward((const moe_bf16*)a, (const float*)a, NULL, (const moe_bf16*)a,
                        (const moe_bf16*)a, &s, (moe_bf16*)a, NULL, NULL, NULL, a, NULL);
  int bad = moe_forward(NULL, NULL, NULL, NULL, NULL, &s, NULL, NULL, NULL, NULL, a, NULL);
  printf("version=%d ws=%zu plan=%d p2l0=%d forward=%d bad=%d err=%s\n", moe_version(),
         ws_bytes, plan, (int)p2l[0], fwd, bad, moe_error_string(fwd));
  return 0;
}
