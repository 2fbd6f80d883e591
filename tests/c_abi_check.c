/* A plain C consumer of libcce: includes only include/cce.h, links the
 * shared library and checks its host-side contract (no GPU needed): version,
 * error strings, workspace sizes, and argument rejection before any device
 * work.  Exit status 0 on success; the failing check is printed otherwise. */
#include <stdio.h>
#include <string.h>

#include "cce.h"

#define CHECK(c)                                              \
  do {                                                        \
    if (!(c)) {                                               \
      fprintf(stderr, "check failed: %s (line %d)\n", #c, __LINE__); \
      return 1;                                               \
    }                                                         \
  } while (0)

int main(void) {
  static char dummy[64] __attribute__((aligned(256)));
  void* p = dummy;
  float* f = (float*)dummy;
  int32_t* st = (int32_t*)dummy;
  const int32_t* y = (const int32_t*)dummy;

  CHECK(cce_version() >= 10000);
  for (int c = CCE_OK; c <= CCE_EDEVICE; ++c) CHECK(cce_strerror(c) && strlen(cce_strerror(c)) > 0);

  CHECK(cce_fwd_workspace_size(4096, 2048, 128256, 0) > 0);
  CHECK(cce_fwd_workspace_size(4096, 2050, 128256, 0) == 0); /* D % 8 != 0 */
  CHECK(cce_bwd_workspace_size(4096, 2048, 128256, 0, 0) > 0);
  CHECK(cce_bwd_workspace_size(4096, 2048, 128256, 0, CCE_FULL_DE) > 0);
  {
    /* the size classes add up, and the logits class stays below N V 2 / 8 */
    size_t rows = 0, vocab = 0, logits = 0;
    CHECK(cce_bwd_workspace_parts(4096, 2048, 128256, 0, CCE_FULL_DE, &rows, &vocab, &logits) ==
          CCE_OK);
    CHECK(rows + vocab + logits == cce_bwd_workspace_size(4096, 2048, 128256, 0, CCE_FULL_DE));
    CHECK(logits < (size_t)4096 * 128256 * 2 / 8);
    CHECK(cce_bwd_workspace_parts(4096, 2048, 128256, 0, 0, NULL, &vocab, &logits) == CCE_EINVAL);
  }
  CHECK(cce_vocab_sort_workspace_size(4096, 128256, 0) > 0);
  CHECK(cce_kl_fwd_workspace_size(4096, 2048, 128256) > 0);

  /* NULL required pointers and bad shapes are rejected on the host */
  CHECK(cce_fwd(NULL, p, y, 4, 8, 10, -100, NULL, 0, f, f, NULL, p, 1u << 30, st, NULL) ==
        CCE_EINVAL);
  CHECK(cce_fwd(p, p, y, 4, 12, 10, -100, NULL, 0, f, f, NULL, p, 1u << 30, st, NULL) ==
        CCE_EINVAL);
  CHECK(cce_bwd(p, p, y, f, f, 4, 8, 10, -100, NULL, 0, 0.f, NULL, NULL, 64u, p, p, NULL, NULL, 0,
                p, 1u << 30, st, NULL) == CCE_EINVAL); /* unknown flag */
  CHECK(cce_kl_bwd(p, p, p, p, NULL, f, f, f, 4, 8, 10, 0.f, CCE_FULL_DE, p, p, NULL, NULL, 0, p,
                   1u << 30, st, NULL) == CCE_EINVAL);
  /* the vocabulary-parallel combine and the wait diagnostic check their arguments */
  CHECK(cce_vocab_combine(f, 0, y, 4, 10, -100, NULL, 0, f, f, NULL) == CCE_EINVAL);
  CHECK(cce_vocab_combine(NULL, 0, y, 0, 10, -100, NULL, 0, f, f, NULL) == CCE_EINVAL);
  CHECK(cce_debug_stall(0, st, NULL) == CCE_EINVAL);
  CHECK(cce_debug_stall_pair(0, st, NULL) == CCE_EINVAL);
  CHECK(cce_debug_stall_pair(1000, NULL, NULL) == CCE_EINVAL);
  /* an empty batch is a no-op */
  CHECK(cce_fwd(p, p, y, 0, 8, 10, -100, NULL, 0, f, f, NULL, p, 1u << 30, st, NULL) == CCE_OK);

  /* a composite head: two segments with a gap, each with its own E */
  cce_segment segs[2];
  memset(segs, 0, sizeof(segs));
  segs[0].vocab_begin = 0;
  segs[0].vocab_end = 6;
  segs[0].E = p;
  segs[1].vocab_begin = 4; /* overlaps segment 0: rejected */
  segs[1].vocab_end = 10;
  segs[1].E = p;
  CHECK(cce_fwd(p, NULL, y, 4, 8, 10, -100, segs, 2, f, f, NULL, p, 1u << 30, st, NULL) ==
        CCE_EINVAL);
  printf("c abi ok\n");
  return 0;
}
