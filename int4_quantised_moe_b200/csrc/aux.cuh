#pragma once
#include "common.cuh"

namespace r4 {

// dst[inv[t * top_k + s], :] = fp16(src[t, :]) for t < hdr->qlen and every s with
// inv[t * top_k + s] >= 0 (bf16 src [Q, H]): each permuted row receives its token's row.
// need_saved: the kernel does nothing unless the header holds a pending saved forward (backward use).
// scale_dy: grad_out; values are multiplied by 2^s (dy_scale_exponent of hdr->dy_amax) and s is
// recorded in hdr->dy_exp.
cudaError_t launch_gather_rows(const uint16_t* src_bf16, const int32_t* inv, int top_k, WsHeader* hdr,
                               uint16_t* dst_f16, int H, int max_tokens, uint32_t* status, int need_saved, int scale_dy,
                               cudaStream_t stream);

// hdr->dy_amax = max(hdr->dy_amax, largest |v| of the first hdr->qlen rows of bf16 src [*, H]);
// runs only with a pending saved forward (backward use).
cudaError_t launch_absmax_rows(const uint16_t* src_bf16, WsHeader* hdr, int H, int max_tokens, cudaStream_t stream);

// out[t, :] = bf16(sum_s src[inv[t*k+s], :]) in slot order, t < hdr->qlen (fp32 src [R, H]);
// unscale_dy: the sum is multiplied by 2^-hdr->dy_exp before rounding.
cudaError_t launch_combine_rows(const float* src, const int32_t* inv, int top_k, const WsHeader* hdr,
                                uint16_t* out_bf16, int H, int max_tokens, int need_saved, int unscale_dy,
                                cudaStream_t stream);

// grad_route[t, s] = 2^-hdr->dy_exp sum_b part[inv[f], b] (0 for dropped slots), f = t*k+s < hdr->qlen*k.
// Expert-parallel row moves (see the C-ABI declarations).
cudaError_t launch_dispatch_rows(const uint16_t* src, const int32_t* perm, int32_t n, int top_k, int width,
                                 uint16_t* dst, cudaStream_t stream);
cudaError_t launch_combine_slots(const uint16_t* src, const int32_t* inv, int32_t qlen, int top_k, int width,
                                 uint16_t* out, cudaStream_t stream);
cudaError_t launch_gather_slots(const float* src, const int32_t* inv, int32_t n_slots, float* out, cudaStream_t stream);

cudaError_t launch_combine_route(const float* part, int nparts, const int32_t* inv, int top_k, const WsHeader* hdr,
                                 float* grad_route, int max_tokens, cudaStream_t stream);

// Workspace header bookkeeping.
cudaError_t launch_header_begin_fwd(WsHeader* hdr, int save, cudaStream_t stream);
cudaError_t launch_header_check_bwd(WsHeader* hdr, cudaStream_t stream);
cudaError_t launch_header_end_bwd(WsHeader* hdr, cudaStream_t stream);

// Zero `count` fp16/bf16 elements (generic 16-bit fill) and fp32 fill.
cudaError_t launch_fill_u16(uint16_t* p, int64_t count, uint16_t value, cudaStream_t stream);

// Bit-exact decode check exports (RAWINT4 with bf16 scales; MXFP4 with UE8M0 scale bytes).
cudaError_t launch_decode_mxfp4(const uint8_t* q, const uint8_t* s, int64_t n, int64_t k, float* out_f32,
                                uint16_t* out_f16, cudaStream_t stream);
cudaError_t launch_decode(const uint8_t* q, const uint16_t* s, int64_t n, int64_t k, float* out_f32, uint16_t* out_f16,
                          cudaStream_t stream);

}  // namespace r4
