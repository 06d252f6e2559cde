#pragma once
#include "common.cuh"

namespace r4 {

// dst[p, :] = fp16(src[perm[p] / top_k, :]) for p < hdr->routed (bf16 src [Q, H]).
// need_saved: the kernel does nothing unless the header holds a pending saved forward (backward use).
cudaError_t launch_gather_rows(const uint16_t* src_bf16, const int32_t* perm, int top_k, const WsHeader* hdr,
                               uint16_t* dst_f16, int H, int max_rows, uint32_t* status, int need_saved,
                               cudaStream_t stream);

// out[t, :] = bf16(sum_s src[inv[t*k+s], :]) in slot order, t < hdr->qlen (fp32 src [R, H]).
cudaError_t launch_combine_rows(const float* src, const int32_t* inv, int top_k, const WsHeader* hdr,
                                uint16_t* out_bf16, int H, int max_tokens, int need_saved, cudaStream_t stream);

// grad_route[t, s] = sum_b part[inv[f], b] (0 for dropped slots), f = t*k+s < hdr->qlen*k.
cudaError_t launch_combine_route(const float* part, int nparts, const int32_t* inv, int top_k, const WsHeader* hdr,
                                 float* grad_route, int max_tokens, cudaStream_t stream);

// Rank-r side matrices of the LoRA products, per permuted row p of expert e:
//   out0[p, half*rank + j] = scale * sum_k L[p, colL[half] + k] * R_half(e, j, k)
//   out1[p, ...]           = w_perm[p] * out0[p, ...]            (optional)
// R style 0: R[e][j][k] (LoRA A, [E, r, K]); style 1: R[e][k][j] (LoRA B, [E, K, r]).
// Columns from halves*rank to 63 are written as 0. Rows past hdr->routed up to
// the next multiple of 16 are written as 0.
struct LoraRowsArgs {
  const uint16_t* L;  // fp16 [rows, ldL]
  int ldL;
  int colL[2];
  int K;
  const uint16_t* R[2];  // bf16
  int64_t r_expert;
  int r_style;
  int rank;
  int halves;
  float scale;
  uint16_t* out0;  // fp16 [rows, 64]
  uint16_t* out1;  // fp16 [rows, 64] or null
  const float* w_perm;
};
cudaError_t launch_lora_rows(const LoraRowsArgs& a, const int4* tok_tiles, const WsHeader* hdr, int max_tiles,
                             int need_saved, cudaStream_t stream);

// One LoRA gradient: G[e](p, j) = sum over rows of expert e of L[row, colL + p] * S[row, colS + j],
// stored with the authoritative window: buf = (accumulate ? buf : 0) + grad_scale * G,
// bf16 round-to-nearest-even; experts without rows keep/zero their block.
struct GradJob {
  const uint16_t* L;  // fp16 [rows, ldL]
  int ldL;
  int colL;
  int P;
  const uint16_t* S;  // fp16 [rows, 64]
  int colS;
  uint16_t* out;      // bf16, [E, P, r] (transposed = 0) or [E, r, P] (transposed = 1)
  int transposed;
};
struct GradJobs {
  GradJob j[6];
};
// Only runs when the header holds a pending saved forward.
cudaError_t launch_lora_grads(const GradJobs& jobs, int njobs, int pmax, const int32_t* offsets, int experts, int rank,
                              int accumulate, float grad_scale, const WsHeader* hdr, cudaStream_t stream);

// Workspace header bookkeeping.
cudaError_t launch_header_begin_fwd(WsHeader* hdr, int save, cudaStream_t stream);
cudaError_t launch_header_check_bwd(WsHeader* hdr, cudaStream_t stream);
cudaError_t launch_header_end_bwd(WsHeader* hdr, cudaStream_t stream);

// Zero `count` fp16/bf16 elements (generic 16-bit fill) and fp32 fill.
cudaError_t launch_fill_u16(uint16_t* p, int64_t count, uint16_t value, cudaStream_t stream);

// Bit-exact decode check export.
cudaError_t launch_decode(const uint8_t* q, const uint16_t* s, int64_t n, int64_t k, float* out_f32, uint16_t* out_f16,
                          cudaStream_t stream);

}  // namespace r4
