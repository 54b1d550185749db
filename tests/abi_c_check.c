/* Compiled and run by test_abi_cpu.py: the public header is valid C99 and the library links and answers
 * from plain C, with no GPU (only the host-side entry points are called). */
#include <stdio.h>
#include <string.h>

#include "eta.h"

int main(void) {
  long long items = 0, whole = 0;
  int ctas = 0;
  /* B1 H32 N4096 d64 non-causal on 148 SMs: 512 items, the last 68 split */
  if (eta_prefill_plan(0, 32, 4096, 64, 0, 148, &items, &whole, &ctas) != ETA_OK) return 1;
  if (items != 512 || whole != 444 || ctas != 148) return 2;
  if (eta_prefill_plan(0, 32, 4096, 80, 0, 148, NULL, NULL, NULL) != ETA_ERR_HEAD_DIM) return 3;
  if (attn_decode_workspace_size(1, 1, 100, 96) != 0) return 4;
  if (strlen(eta_strerror(ETA_ERR_SHAPE)) == 0) return 5;
  if (attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1, 128, 64, 0.125f, 0, ETA_OUT_BF16, NULL) != ETA_ERR_NULL) return 6;
  printf("ok\n");
  return 0;
}
