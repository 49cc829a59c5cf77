/* Builds the plan of a Wan2.1-1.3B-shaped 4-chunk round through the C ABI
 * from plain C11 (no CUDA headers, no device: num_ctas is given) and writes
 * the blob to the file named on the command line.  Exit status 0 on success. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "wf.h"

int main(int argc, char** argv) {
  if (argc != 2) return 2;
  wf_round_desc d;
  memset(&d, 0, sizeof(d));
  d.num_heads = 12;
  d.head_dim = 128;
  d.frame_h = 30;
  d.frame_w = 52;
  d.frames_per_chunk = 3;
  d.cache_chunks = 7;
  d.inround_chunks = 4;
  d.pool_slots = 0;
  d.n0 = 16;
  d.noise_t[0] = 250;
  d.noise_t[1] = 500;
  d.noise_t[2] = 750;
  d.noise_t[3] = 1000;
  d.rope_theta = 10000.0;
  d.dtype = WF_BF16;
  d.num_ctas = 148;
  const size_t n = wf_plan_bytes(&d);
  if (n == 0) return 3;
  /* the plan wants 16-byte alignment */
  void* buf = aligned_alloc(256, (n + 255) / 256 * 256);
  if (!buf) return 4;
  const wf_status s = wf_plan_round(&d, buf, n, NULL, 0, NULL);
  if (s != WF_OK) {
    fprintf(stderr, "%s\n", wf_status_string(s));
    return 5;
  }
  /* an invalid description is rejected with a status, not a crash */
  d.inround_chunks = WF_MAX_INROUND + 1;
  if (wf_plan_bytes(&d) != 0 || wf_plan_round(&d, buf, n, NULL, 0, NULL) != WF_ERR_INVALID_ARG) return 6;
  FILE* f = fopen(argv[1], "wb");
  if (!f || fwrite(buf, 1, n, f) != n) return 7;
  fclose(f);
  free(buf);
  return 0;
}
