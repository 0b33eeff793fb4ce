/* Plain C99 caller of libkvq (no GPU needed): the header compiles as C, the library links
 * from C, and the host-only entry points answer: chunk sizes, status strings, and an
 * argument error returned before anything is enqueued.  Exit status 0 on success. */
#include <stdio.h>
#include <string.h>

#include "kvq.h"

int main(void) {
  static const size_t want[6] = {4096, 2304, 1280, 768, 384, 2176}; /* one chunk, D = 128 */
  kvq_cache c;
  int t;
  for (t = 0; t < 6; ++t)
    if (kvq_chunk_bytes(t, 128) != want[t]) return 1;
  if (kvq_chunk_bytes(6, 128) != 0 || kvq_chunk_bytes(0, 96) != 0) return 2;
  if (strcmp(kvq_status_string(KVQ_OK), "ok") != 0) return 3;
  memset(&c, 0, sizeof c);
  c.B = 1; c.Hq = 8; c.Hkv = 2; c.D = 96; c.page_size = 16; c.max_pages = 4; c.dtype = KVQ_DT_F16;
  if (kvq_page_scores(&c, NULL, NULL, NULL) != KVQ_ERR_UNSUPPORTED) return 4; /* D = 96 */
  c.D = 64;
  if (kvq_page_scores(&c, NULL, NULL, NULL) != KVQ_ERR_INVALID_ARG) return 5;  /* null buffers */
  printf("c abi ok\n");
  return 0;
}
