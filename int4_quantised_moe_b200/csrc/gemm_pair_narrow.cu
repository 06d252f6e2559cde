// Narrow configuration of the CTA-pair GEMM (gemm_pair.cu) for layers with
// few rows per expert: token tiles of at most kTileRowsNarrow rows, eight A
// tiles in shared memory, hand-off groups of four stages.
#define R4_PAIR_NARROW 1
#include "gemm_pair.cu"
