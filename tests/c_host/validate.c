/* A plain C11 host of the library: includes the header, links libmla.so and makes only
 * calls that are validated on the host before any device work, so it runs without a GPU.
 * Prints one line per check; the test that builds it compares the lines. */
#include <stdio.h>
#include <string.h>

#include "mla.h"

static mla_shape chunk_shape(void) {
  mla_shape s;
  memset(&s, 0, sizeof s);
  s.batch = 1; s.n_heads = 32; s.d_nope = 128; s.d_latent = 512; s.d_rope = 64;
  s.rope_pairs[0] = 8; s.rope_pairs[1] = 12; s.rope_pairs[2] = 12;
  s.rope_theta = 10000.0; s.grid_h = 30; s.grid_w = 52; s.ring_slots = 6240;
  s.dtype = MLA_BF16;
  return s;
}

int main(void) {
  static _Alignas(16) char fake[64];                   /* never dereferenced */
  mla_shape s = chunk_shape();
  printf("status %s\n", mla_status_string(MLA_ERR_RANGE));
  printf("materialised_ws %zu\n", mla_attend_materialised_workspace_size(&s));
  /* a query past the key window is refused before launch */
  printf("attend_range %s\n",
         mla_status_string(mla_attend(&s, fake, 1560, 3 * 1560 + 1, fake, 0, 6240, 0.07f, fake,
                                      NULL, NULL, 0, NULL)));
  /* an odd RoPE width is an argument error */
  mla_shape bad = s;
  bad.d_rope = 63;
  printf("shape_arg %s\n",
         mla_status_string(mla_cache_write(&bad, fake, 4096, 1560, 0, fake, fake, fake, NULL,
                                           NULL)));
  /* empty calls succeed without touching the device */
  printf("empty_up_v %s\n", mla_status_string(mla_up_v(&s, fake, 0, fake, fake, NULL)));
  printf("empty_shift %s\n", mla_status_string(mla_cache_shift_frames(&s, fake, 0, 0, 1, NULL)));
  /* the low-bit ring: a 3-bit code width is refused, an empty range succeeds */
  float* fs = (float*)(void*)fake;
  printf("quant_bits %s\n",
         mla_status_string(mla_cache_quantise(&s, fake, 0, 6240, 3, 4, fake, fake, fs, fs,
                                              NULL)));
  printf("empty_dequant %s\n",
         mla_status_string(mla_cache_dequantise(&s, fake, fake, fs, fs, 2, 4, 0, 0, fake,
                                                NULL)));
  /* the no-workspace attention: checked like mla_attend, an empty call succeeds */
  printf("fixed_range %s\n",
         mla_status_string(mla_attend_fixed_scratch(&s, fake, 1560, 3 * 1560 + 1, fake, 0,
                                                    6240, 0.07f, fake, NULL, NULL)));
  printf("fixed_align %s\n",
         mla_status_string(mla_attend_fixed_scratch(&s, fake + 8, 1560, 3 * 1560, fake, 0,
                                                    6240, 0.07f, fake, NULL, NULL)));
  printf("fixed_empty %s\n",
         mla_status_string(mla_attend_fixed_scratch(&s, fake, 0, 0, fake, 0, 6240, 0.07f, fake,
                                                    NULL, NULL)));
  return 0;
}
