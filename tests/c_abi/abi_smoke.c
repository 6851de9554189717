/* A plain C caller of libwaveprune.so: only the header and the shared
 * library, no Python and no GPU (the calls used here touch no device).
 * Prints the group cutoffs and the tile-class counts of one schedule so the
 * test can compare them with the Python binding. */
#include <stdio.h>
#include <stdint.h>
#include "waveprune.h"

int main(void) {
  int32_t chan[64], grp[8];
  int st = wp_cutoffs(128, 1e6, NULL, 1.0, 2.0, WP_ROPE_HALF_SPLIT, chan, grp);
  if (st != WP_OK) {
    printf("wp_cutoffs: %s\n", wp_status_str(st));
    return 1;
  }
  for (int g = 0; g < 8; ++g) printf("%d%c", grp[g], g == 7 ? '\n' : ' ');
  int64_t counts[3 * 8];
  st = wp_schedule(4096, 128, 128, grp, 8, NULL, counts);
  if (st != WP_OK) {
    printf("wp_schedule: %s\n", wp_status_str(st));
    return 1;
  }
  for (int i = 0; i < 3 * 8; ++i) printf("%lld%c", (long long)counts[i], i == 23 ? '\n' : ' ');
  /* argument errors come back as status codes */
  printf("%d %s\n", wp_cutoffs(100, 1e6, NULL, 1.0, 2.0, WP_ROPE_HALF_SPLIT, chan, grp),
         wp_status_str(WP_ERR_ARG));
  return 0;
}
