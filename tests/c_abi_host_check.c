/* Compiled as C (not C++) against include/littlebit.h and linked with the
 * library by tests/test_capi_cpu.py: the boundary is a plain C ABI.  Runs the
 * host-side entry points only (no device work), printing their results. */
#include <stdio.h>

#include "littlebit.h"

int main(void) {
  lb_layer L = {0};
  L.d_in = 100; /* not a multiple of 256: rejected before any device work */
  L.d_out = 128;
  L.s = 4;
  printf("eff_bits %.9f\n", littlebit_eff_bits(4096, 4096, 86, 1));
  printf("packed_bytes %zu\n", littlebit_packed_bytes(LB_ROLE_V, 86, 4096));
  printf("forward %d\n", (int)littlebit_linear_forward(&L, (const void*)16, (void*)16, 1, LB_F16, NULL));
  printf("status %s\n", littlebit_status_string(LB_ERR_SHAPE));
  /* host-buffer stack call: NULL host buffers are refused before device work */
  printf("host %d\n", (int)littlebit_linear_forward_many_host(&L, 1, NULL, NULL, 1, LB_F16, 4, NULL));
  return 0;
}
