/* Plain C99 user of the C ABI: the host-only entry points, no GPU needed.
 * Prints the library version, the K-pass sizes and the loss-row count of a
 * two-conversation batch, one value per line. */
#include <stdint.h>
#include <stdio.h>

#include "opr.h"

int main(void) {
  /* two conversations: turns (2,3,2), (1,2,1) and (4,2,3) */
  const int32_t turn_lens[] = {2, 3, 2, 1, 2, 1, 4, 2, 3};
  const int32_t conv_turn_ptr[] = {0, 2, 3};
  int64_t n_out_turns = -1, n_out_convs = -1;
  printf("%s\n", opr_version());
  if (opr_kpass_sizes(conv_turn_ptr, 2, 2, &n_out_turns, &n_out_convs) != OPR_OK) return 1;
  printf("%lld\n%lld\n", (long long)n_out_turns, (long long)n_out_convs);
  printf("%lld\n", (long long)opr_loss_row_count(turn_lens, 3));
  printf("%d\n", (int)(opr_kpass_sizes(conv_turn_ptr, 2, 0, &n_out_turns, &n_out_convs) == OPR_INVALID_ARG));
  return 0;
}
