/* A plain C99 client of libtq: include/tq.h compiled as C, the library
 * linked and called with host-only entry points (no GPU is touched):
 * codebook construction, its tables, the workspace sizes, and one call that
 * the argument checks reject.  Prints one "key value" line per result for
 * the test that builds and runs it. */
#include <stdio.h>
#include <string.h>

#include "tq.h"

int main(void) {
  tq_params p;
  memset(&p, 0, sizeof p);
  p.head_dim = 128;
  p.k_bits = 3;
  p.v_bits = 4;
  p.qjl = 1;
  p.seed = 42;
  p.codebook = TQ_CODEBOOK_GAUSSIAN;

  tq_codebook* cb = NULL;
  tq_layout lay;
  tq_status st = tq_codebook_init(&p, &cb, &lay);
  printf("init %d\n", (int)st);
  if (st != TQ_OK) return 1;
  printf("layout %zu %zu %zu %zu\n", lay.k_code_bytes, lay.v_code_bytes, lay.k_sign_bytes,
         lay.norm_halves);

  float kc[8], kb[7], vc[16], vb[15];
  int8_t s1[128], s2[128];
  st = tq_codebook_tables(cb, kc, kb, vc, vb, s1, s2);
  printf("tables %d\n", (int)st);
  printf("k_centroids");
  for (int i = 0; i < 8; ++i) printf(" %.9g", kc[i]);
  printf("\nsigns1");
  for (int i = 0; i < 16; ++i) printf(" %d", (int)s1[i]);
  printf("\n");

  printf("decode_ws %zu\n", tq_decode_workspace_bytes(cb, 32, 32, 8, 65536));
  printf("lut_ws %zu\n", tq_lut_matmul_workspace_bytes(cb, 16384, 8192, 16));

  st = tq_decode_attention(cb, NULL, NULL, TQ_BF16, 32, 0.0f, 64, NULL, NULL, 0, NULL);
  printf("rejected %d %s\n", (int)st, tq_last_error());

  tq_free(cb);
  return 0;
}
