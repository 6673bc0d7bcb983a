/* Plain C99 user of the C ABI: the host-only entry points, no GPU needed.
 * Prints the library version, the K-pass sizes (turns, passes, tokens, longest
 * sequence, original tokens) and the loss-row count of a two-conversation
 * batch in one sequence, the refusal of a K of 0, and whether the test hook of
 * opr_testing.h places the row counts first in the layout workspace, one
 * value per line. */
#include <stdint.h>
#include <stdio.h>

#include "opr.h"
#include "opr_testing.h"

int main(void) {
  /* two conversations: turns (2,3,2), (1,2,1) and (4,2,3) */
  const int32_t turn_lens[] = {2, 3, 2, 1, 2, 1, 4, 2, 3};
  const int32_t conv_turn_ptr[] = {0, 2, 3};
  const int32_t seq_conv_ptr[] = {0, 2};
  int64_t n_out_turns = -1, n_out_convs = -1, total = -1, max_seqlen = -1, orig = -1;
  printf("%s\n", opr_version());
  if (opr_kpass_sizes(turn_lens, conv_turn_ptr, seq_conv_ptr, 1, 2, 3, 2, &n_out_turns, &n_out_convs, &total,
                      &max_seqlen, &orig) != OPR_OK)
    return 1;
  printf("%lld\n%lld\n%lld\n%lld\n%lld\n", (long long)n_out_turns, (long long)n_out_convs, (long long)total,
         (long long)max_seqlen, (long long)orig);
  printf("%lld\n", (long long)opr_loss_row_count(turn_lens, 3));
  printf("%d\n", (int)(opr_kpass_sizes(turn_lens, conv_turn_ptr, seq_conv_ptr, 1, 2, 3, 0, &n_out_turns,
                                        &n_out_convs, &total, &max_seqlen, &orig) == OPR_INVALID_ARG));
  {
    uint64_t off[4] = {0, 0, 0, 0};
    const int st = opr_testing_layout_tables(1, 2, 3, total, max_seqlen, off);
    printf("%d\n", (int)(st == OPR_OK && off[0] < off[1] && off[1] < off[2] && off[2] < off[3]));
  }
  return 0;
}
