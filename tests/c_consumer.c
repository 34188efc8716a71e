/* A C99 consumer of include/moe_b200.h, built and run by test_c_consumer.py:
 * the header compiles as C, the library links from C, and the calls below
 * need no GPU (version, status strings, host-side size queries and argument
 * checks).  It prints the argument structs' sizes and field offsets, which
 * the test compares with the Python binding's ctypes mirrors. */
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include "moe_b200.h"

int main(void) {
  size_t P = 0, NB = 0, ws = 0, ffn_ws = 0, fwd_ws = 0;
  moe_ffn_args fa;
  moe_forward_args wa;

  if (moe_version() != MOE_ABI_VERSION) return 1;
  if (strcmp(moe_status_string(MOE_ERR_WORKSPACE), "MOE_ERR_WORKSPACE") != 0) return 2;
  if (moe_align_sort_sizes(16384, 8, 256, 64, &P, &NB, &ws) != MOE_OK) return 3;
  /* argument errors come back synchronously, with nothing launched */
  if (moe_align_sort_sizes(4, 2, 0, 16, &P, &NB, &ws) != MOE_ERR_INVALID_ARG) return 4;
  if (moe_align_sort_sizes(16384, 8, 256, 64, &P, &NB, &ws) != MOE_OK) return 5;

  memset(&fa, 0, sizeof fa);
  fa.T = 2048; fa.H = 7168; fa.I = 2048; fa.E = 256; fa.k = 8; fa.block_size = 64;
  fa.wdtype = MOE_BF16;
  if (moe_ffn_workspace(&fa, &ffn_ws) != MOE_OK) return 6;

  memset(&wa, 0, sizeof wa);
  wa.T = 2048; wa.H = 7168; wa.I = 2048; wa.E = 256; wa.k = 8; wa.block_size = 64;
  wa.wdtype = MOE_BF16; wa.out_dtype = MOE_BF16;
  if (moe_forward_workspace(&wa, &fwd_ws) != MOE_OK) return 7;

  printf("align %zu %zu %zu\n", P, NB, ws);
  printf("ffn_ws %zu\n", ffn_ws);
  printf("forward_ws %zu\n", fwd_ws);
  printf("sizeof moe_ffn_args %zu\n", sizeof(moe_ffn_args));
  printf("sizeof moe_forward_args %zu\n", sizeof(moe_forward_args));
  printf("sizeof moe_backward_args %zu\n", sizeof(moe_backward_args));
  printf("offset moe_ffn_args w2_mx_scale %zu\n", offsetof(moe_ffn_args, w2_mx_scale));
  printf("offset moe_ffn_args tile_tokens %zu\n", offsetof(moe_ffn_args, tile_tokens));
  printf("offset moe_forward_args stage_events %zu\n", offsetof(moe_forward_args, stage_events));
  printf("offset moe_forward_args w2_mx_scale %zu\n", offsetof(moe_forward_args, w2_mx_scale));
  printf("offset moe_backward_args dw2 %zu\n", offsetof(moe_backward_args, dw2));
  return 0;
}
