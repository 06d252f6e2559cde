#pragma once
#include "common.cuh"

namespace r4 {

// Tensor-core kernel for the rank-r LoRA products (both operands by TMA, FP16
// in, FP32 accumulate, N = 64 columns, M = 128 rows).
//
// kSkRows: side matrices of the permuted rows, per expert e
//   out0[p, seg*sw + j] = scale * sum_k L[p, lcol[seg] + k] * R_seg[e][j][k]
//   out1[p, ...]        = w_perm[p] * out0[p, ...]               (optional)
//   (tokens on M, rank on N; R_seg are the FP16 LoRA tensors laid out
//   [E, sw, K] so that both operands are K-major; sw is a multiple of 16,
//   at most 64.) Within a segment, column j is kept when j % rpad < rank (the
//   rest are the zero rows that pad each rank block to rpad =
//   roundup16(rank)). The side matrices are kLoraPad columns wide; columns
//   past the segments are written as zeros up to 64 (all kLoraPad when the
//   segments reach past 64).
// kSkGrads: the six LoRA gradients, per (job, expert, 128-feature block)
//   D[p, j] = sum over the expert's rows of L[row, lcol + p] * S[row, scol + j]
//   (features on M, 64 rank columns on N, reduction over the expert's rows;
//   both operands MN-major) stored with the authoritative window of the
//   contract test: buf = (accumulate ? buf : 0) + grad_scale * D. A rank up
//   to 32 lets one job carry the gate and up rank blocks (the splits below);
//   a larger rank gives every output buffer a job of its own (kSplitNone,
//   ranks from D columns [0, rank)).
enum SkMode : int { kSkRows = 0, kSkGrads = 1 };

constexpr int kSkThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kSkStages = 3;
constexpr int kSkCtasPerSm = 2;   // resident skinny CTAs per SM (grid = kSkCtasPerSm x SMs)

// How a gradient job maps D columns/rows to the output buffers.
enum SkSplit : int {
  kSplitNone = 0,     // j < rank -> out_lo
  kSplitFeature = 1,  // feature p < P/2: out_lo[p] with D[j]; p >= P/2: out_hi[p - P/2] with D[rpad + j]
                      // (P/2 a multiple of 32: decided per warp of 32 features)
  kSplitRank = 2,     // D[j] -> out_lo[.., j], D[rpad + j] -> out_hi[.., j]
};

struct SkJob {
  int P;           // features of L used by the job (M extent)
  int lcol;        // first column of L
  int amap;        // tensor map of L (SkMaps::a)
  int bmap;        // tensor map of S (SkMaps::b)
  int scol;        // first column of S
  int nfb;         // 128-feature blocks: ceil(P / 128)
  int split;       // SkSplit
  int transposed;  // 0: out[e][p][j] ([E, Pout, r]); 1: out[e][j][p] ([E, r, Pout])
  int pout;        // features per expert of the output buffers
  uint16_t* out_lo;
  uint16_t* out_hi;
};

struct SkParams {
  const int4* tok_tiles;
  const WsHeader* hdr;
  uint32_t* status;
  int need_saved;
  int rank;
  // rows
  int nseg;
  int seg_lcol[2];
  int nk;          // K stages per segment
  int sw;          // output columns (and R rows) per segment, multiple of 16, <= 64
  int rpad;        // rank rounded up to 16: width of one rank block
  float scale;
  uint16_t* out0;
  uint16_t* out1;
  const float* w_perm;
  // grads
  const int32_t* offsets;
  int experts;
  int njobs;
  SkJob job[6];
  int accumulate;
  float grad_scale;
};

struct SkMaps {
  CUtensorMap a[4];  // rows: [0] L (box {64, 128}); grads: the L tensors of the jobs (box {64, 64})
  CUtensorMap b[4];  // rows: R of each segment (3D, box {64, sw, 1}); grads: the S tensors of the jobs (box {64, 64})
};

cudaError_t launch_skinny(int mode, const SkParams& p, const SkMaps& m, int grid, cudaStream_t stream);

// FP16 copies of the LoRA tensors in the K-major layouts the row products
// read; every rank block is padded with zero rows to rpad = roundup16(r).
//   gu16  [E, 2 rpad, H]: rows [0, r) = A_g, [rpad, rpad + r) = A_u   (fwd: xa)
//   ad16  [E, rpad, I] = A_d                                       (fwd: ha)
//   bdt16 [E, rpad, H] = B_d^T, bgt16 / but16 [E, rpad, I] = B_g^T / B_u^T  (bwd: gd, gb)
struct LoraCvt {
  const uint16_t* src0;  // bf16 source ([E, r, cols], or [E, cols, r] when transposed)
  const uint16_t* src1;  // second stacked source (nsrc = 2)
  uint16_t* dst;
  int rank;
  int rpad;
  int cols;              // K of the product
  int transpose;         // 1: src is [E, cols, r] and is transposed
  int nsrc;              // 1 or 2
};
cudaError_t launch_lora_convert(const LoraCvt* jobs, int njobs, int experts, cudaStream_t stream);

}  // namespace r4
