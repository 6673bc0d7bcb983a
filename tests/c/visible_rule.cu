// Host build of the visibility rule the attention kernels and the layout use
// (opr_internal.cuh: visible), for a CPU test against the oracle's mask.  Reads
// lines "qg qconv qmeta kg kconv kmeta" from stdin and prints 0 or 1 per line.
#include <cstdio>

#include "../../block_sparse_masked_segment_b200/csrc/opr_internal.cuh"

int main() {
  int qg, qc, qm, kg, kc, km;
  while (std::scanf("%d %d %d %d %d %d", &qg, &qc, &qm, &kg, &kc, &km) == 6)
    std::printf("%d\n", opr::visible(qg, qc, qm, kg, kc, km) ? 1 : 0);
  return 0;
}
