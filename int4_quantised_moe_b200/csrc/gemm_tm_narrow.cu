// Narrow configuration of the tensor-memory GEMM (gemm_tm.cu) for layers with
// few rows per expert: token tiles of at most kTileRowsNarrow rows, eight A
// stages in tensor memory, hand-off groups of four stages. Built for the
// forward modes of either base format.
#define R4_TM_NARROW 1
#include "gemm_tm.cu"
