/* A plain C consumer of include/lvsa.h, compiled and run by tests/test_c_abi_consumer.py.
 * It prints the frame lists of the tiny case (T=8, C=4, W=2) for steps 0..2 in the format of
 * tests/golden/worked_example_T8_C4_W2.txt, then the status of calls the library must refuse
 * before touching any device memory. */
#include <stdint.h>
#include <stdio.h>

#include "lvsa.h"

int main(void) {
  int32_t lists[8 * 4];
  int L = 0;
  for (long long s = 0; s < 3; ++s) {
    lvsa_status st = lvsa_build_frame_lists(8, 4, 2, s, lists, 8 * 4, &L);
    if (st != LVSA_OK || L != 4) {
      printf("build failed: %s\n", lvsa_status_string(st));
      return 1;
    }
    for (int t = 0; t < 8; ++t) {
      printf("%lld %d :", s, t);
      for (int i = 0; i < L; ++i) printf(" %d", (int)lists[t * L + i]);
      printf("\n");
    }
  }
  int32_t anchors[2];
  int G = 0;
  const lvsa_status sa = lvsa_build_anchors(8, 4, 2, 1, anchors, 2, &G);
  printf("anchors %s G=%d %d %d\n", lvsa_status_string(sa), G, (int)anchors[0], (int)anchors[1]);
  /* refused before any CUDA call */
  /* fake, 16-byte aligned, non-overlapping addresses: validation fails before any is used */
  const uintptr_t A = (uintptr_t)1 << 24, M = (uintptr_t)1 << 20;
  printf("null q: %s\n", lvsa_status_string(lvsa_attention(NULL, (void*)(A + M), (void*)(A + 2 * M),
                                                           (const int32_t*)(A + 3 * M), 4, 8, 64, 2, 64, 1, 0.0f,
                                                           (void*)(A + 4 * M), NULL)));
  printf("d=96: %s\n", lvsa_status_string(lvsa_attention((void*)A, (void*)(A + M), (void*)(A + 2 * M),
                                                         (const int32_t*)(A + 3 * M), 4, 8, 64, 2, 96, 1, 0.0f,
                                                         (void*)(A + 4 * M), NULL)));
  printf("small buffer: %s\n", lvsa_status_string(lvsa_build_frame_lists(8, 4, 2, 0, lists, 4, &L)));
  printf("version %d\n", lvsa_version());
  return 0;
}
