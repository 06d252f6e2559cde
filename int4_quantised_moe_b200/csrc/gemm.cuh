#pragma once
#include "common.cuh"

namespace r4 {

// The four dequant-fused grouped GEMMs of the layer. Weight rows (output
// features) sit on the UMMA M side and up to 256 permuted tokens of one expert
// on the N side: D[m, n] = sum_k A[m, k] * B[n, k]. Two kernels implement
// them (both take the same parameters):
//   gemm.cu       one CTA per SM, 256 weight rows per work item as two
//                 M = 128 MMAs sharing every B tile (gate/up, down, gate/up^T)
//   gemm_pair.cu  CTA pairs on SM pairs (tcgen05 cta_group::2), 256 weight
//                 rows per item as one M = 256 pair MMA; each SM's TMEM holds
//                 only 128 rows, so 256-token accumulators double-buffer and
//                 a heavy epilogue overlaps the next item (down^T)
enum GemmMode : int {
  kModeGateUp = 0,   // fwd  G/U = X W_{g,u}^T (+ LoRA), SwiGLU epilogue      A: K-major decode of W_g/W_u rows
  kModeDown = 1,     // fwd  y = h W_d^T (+ LoRA), route-weight epilogue       A: K-major decode of W_d rows
  kModeDownT = 2,    // bwd  dh = dY W_d (+ LoRA), SwiGLU' + dRoute epilogue   A: MN-major decode of W_d (transpose-free)
  kModeGateUpT = 3,  // bwd  dx = dG W_g + dU W_u (+ LoRA)                     A: MN-major decode of W_g/W_u
};

constexpr int kBlockK = 64;        // reduction elements per pipeline stage
constexpr int kTmAccCols = 192;    // gemm_tm.cu: columns of one TMEM accumulator = max token-tile rows
constexpr int kLoraPad = 64;       // width of the LoRA side matrices (>= 2 * rank)

struct GemmParams {
  const int4* tok_tiles;     // {expert, first permuted row, rows, 0}
  const WsHeader* hdr;       // n_tok_tiles
  uint32_t* status;
  int n_rowblk;              // output feature blocks (work items) per token tile
  int feat;                  // output features of the mode (the last block may hold only 128)
  int n_main;                // main reduction stages (K / 64)
  int need_saved;            // backward: run only when a saved forward is pending
  // frozen base scales of projection 0 and 1 (bf16)
  const uint16_t* s0;
  const uint16_t* s1;
  const uint8_t* e0;         // MXFP4 base (gemm_tm.cu): UE8M0 scale bytes of projection 0 and 1
  const uint8_t* e1;
  int64_t s_expert;          // scale elements per expert
  int s_row;                 // scales per stored row
  int stored_rows;           // stored rows per expert of one projection
  // LoRA operand of the extra reduction stage (bf16 LoRA tensors)
  const uint16_t* lx0;
  const uint16_t* lx1;
  int64_t lx_expert;         // elements per expert
  int lx_ld;                 // row length of the LoRA tensor
  int rank;
  int rpad;                  // rank rounded up to 16 (width of one rank block in the side matrices)
  // epilogue
  const float* w_perm;
  float* out_a;              // GU: G; DOWN: Yw; GU_T: dx
  float* out_b;              // GU: U
  uint16_t* out_h;           // GU: h (fp16); DOWN_T: dG|dU (fp16)
  const float* in_g;         // DOWN_T: saved G
  const float* in_u;         // DOWN_T: saved U
  float* droute_part;        // DOWN_T: [rows, n_parts] route-gradient partial sums
  int n_parts;               // DOWN_T: partials per row (one per CTA and feature block)
  int ld_out;                // row length of out_a / out_b / out_h / in_*
  int inter;
  float limit;
  unsigned long long wait_ns;  // bound on any pipeline wait (gemm_tm.cu)
};

struct GemmMaps {
  CUtensorMap q0;     // packed projection 0: 3D uint8 {stored K bytes, stored rows, E}
  CUtensorMap q1;     // packed projection 1
  CUtensorMap b[4];   // B main: 2D fp16 {K, rows}, 128B swizzle, boxes {64, 16 << i}
  CUtensorMap bx[4];  // B LoRA: 2D fp16 {64, rows}, 128B swizzle, boxes {64, 16 << i}
};

// One CTA per SM; `grid` CTAs (at most one per SM).
cudaError_t launch_gemm(int mode, const GemmParams& p, const GemmMaps& maps, int grid, cudaStream_t stream);
// CTA pairs (down^T only); `clusters` pairs (at most the number resident at once).
cudaError_t launch_gemm_pair(int mode, const GemmParams& p, const GemmMaps& maps, int clusters, cudaStream_t stream);
// CTA pairs of the pair kernel's mode resident at once on this device (0 on error).
int gemm_pair_max_clusters(int mode);
// CTA pairs with the decoded weights in tensor memory (gemm_tm.cu), every
// mode; fmt: RAWINT4_FORMAT_RAWINT4 (bf16 scales s0/s1) or
// RAWINT4_FORMAT_MXFP4 (E2M1 codes, UE8M0 scale bytes e0/e1).
cudaError_t launch_gemm_tm(int mode, int fmt, const GemmParams& p, const GemmMaps& maps, int clusters,
                           cudaStream_t stream);
int gemm_tm_max_clusters(int mode, int fmt);

}  // namespace r4
