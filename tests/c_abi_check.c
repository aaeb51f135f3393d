/* Plain C99 use of the libttcd C ABI.  Compiled against include/ttcd.h alone
 * and linked to libttcd.so by tests/test_c_abi.py; it makes only host-side
 * calls (size queries, offsets, status strings, argument validation), so it
 * runs without a GPU.  Prints one "key value" line per result. */
#include <stdio.h>
#include <string.h>

#include "ttcd.h"

int main(void) {
  ttcd_block_params p;
  memset(&p, 0, sizeof p);
  p.B = 1;
  p.T = 65536;
  p.d_model = 1024;
  p.n_q_heads = 16;
  p.n_kv_heads = 8;
  p.head_dim = 128;
  p.d_ff = 3072;
  p.w_S = 512;
  p.w_T = 8192;
  p.chunk = 1024;
  p.conv_k = 4;
  p.rms_eps = 1e-6f;
  p.l2_eps = 1e-6f;
  p.rope_theta = 1e4f;
  p.softmax_scale = 0.0f;
  p.dtype = TTCD_BF16;

  printf("version %s\n", ttcd_version());
  printf("block_ws %zu\n", ttcd_block_forward_workspace_size(&p));
  printf("mlp_ws %zu\n", ttcd_fastweight_mlp_workspace_size(&p));
  printf("decode_state %zu\n", ttcd_decode_state_size(&p));
  printf("decode_ws %zu\n", ttcd_decode_workspace_size(&p));
  printf("noalloc_capacity %zu\n", ttcd_fastweight_mlp_noalloc_capacity());

  size_t off = 0;
  ttcd_status s = ttcd_block_workspace_offset(&p, "Wall", &off);
  printf("offset_Wall %d %zu\n", (int)s, off);
  s = ttcd_block_workspace_offset(&p, "no such name", &off);
  printf("offset_unknown %d\n", (int)s);

  ttcd_block_params bad = p;
  bad.w_S = bad.w_T + 1;
  printf("bad_windows_ws %zu\n", ttcd_block_forward_workspace_size(&bad));

  /* every pointer null: rejected on the host before any device work */
  s = ttcd_block_forward(NULL, NULL, NULL, &p, NULL, NULL, NULL, 0, NULL);
  printf("null_block %d %s\n", (int)s, ttcd_status_string(s));
  printf("status_timeout %s\n", ttcd_status_string(TTCD_ERR_TIMEOUT));
  return 0;
}
