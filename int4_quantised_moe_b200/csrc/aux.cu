// Memory-bound helpers of the layer: row gather into expert order (with the
// bf16 -> fp16 operand conversion), the fixed-order top-k combines, header
// bookkeeping and the decode check export.
#include "aux.cuh"

namespace r4 {

namespace {

__device__ __forceinline__ bool bwd_enabled(const WsHeader* hdr) { return hdr->saved == 1u; }

// ------------------------------------------------------------------ gather
// One warp per token: each 16-byte piece of the token's row is loaded and
// converted once and stored to every permuted row the token was routed to
// (inv[t * top_k + s], -1 for an entry that routes nowhere), so the source
// matrix is read once instead of once per routed copy.
// scale_dy (grad_out): every value is multiplied by 2^s first, s from the
// largest magnitude found by absmax_rows_kernel (exact: a power of two).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ inv,
                                                          int top_k, WsHeader* hdr, uint4* __restrict__ dst,
                                                          int vecs_per_row, uint32_t* status, int need_saved,
                                                          int scale_dy) {
  if (need_saved && !bwd_enabled(hdr)) return;
  const int64_t tokens = hdr->qlen;
  float sc = 1.0f;
  if (scale_dy) {
    const int e = dy_scale_exponent(hdr->dy_amax);
    sc = ldexpf(1.0f, e);
    if (blockIdx.x == 0 && threadIdx.x == 0) hdr->dy_exp = e;
  }
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  bool overflow = false;
  for (int64_t t = warp0; t < tokens; t += nwarps) {
    const uint4* s = src + t * vecs_per_row;
    const int32_t* slots = inv + t * top_k;
#pragma unroll 2
    for (int c = lane; c < vecs_per_row; c += 32) {
      const uint4 v = __ldg(s + c);
      const uint32_t in[4] = {v.x, v.y, v.z, v.w};
      uint32_t out[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = sc * __uint_as_float(in[j] << 16);
        const float hi = sc * __uint_as_float(in[j] & 0xFFFF0000u);
        __half2 h = __floats2half2_rn(lo, hi);
        // each half on its own: a finite value that became inf (an inf or NaN
        // input is not an overflow of the conversion)
        overflow |= (__hisinf(__low2half(h)) != 0 && isfinite(lo)) || (__hisinf(__high2half(h)) != 0 && isfinite(hi));
        out[j] = *reinterpret_cast<uint32_t*>(&h);
      }
      const uint4 o = make_uint4(out[0], out[1], out[2], out[3]);
      for (int k = 0; k < top_k; ++k) {
        const int32_t row = __ldg(slots + k);
        if (row >= 0) dst[(int64_t)row * vecs_per_row + c] = o;
      }
    }
  }
  if (overflow) raise_status(status, RAWINT4_DEV_FP16_OVERFLOW);
}

// Largest |v| over the first hdr->qlen rows of a bf16 [rows, 8 * vecs] matrix,
// as bf16 magnitude bits, folded into hdr->dy_amax (reset by the backward's
// header check). Magnitude bits of finite values order like the values.
__global__ void __launch_bounds__(256) absmax_rows_kernel(const uint4* __restrict__ src, int vecs_per_row, WsHeader* hdr) {
  if (!bwd_enabled(hdr)) return;
  const int64_t total = (int64_t)hdr->qlen * vecs_per_row;
  uint32_t m = 0u;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(src + i);
    m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
  }
  m = max(m & 0xFFFFu, m >> 16);
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0 && m != 0u) atomicMax(&hdr->dy_amax, m);
}

// ----------------------------------------------------------------- combine
// unscale_dy: the rows carry grad_out's power-of-two scale; multiply by 2^-s.
__global__ void combine_rows_kernel(const float4* __restrict__ src, const int32_t* __restrict__ inv, int top_k,
                                    const WsHeader* hdr, uint2* __restrict__ out, int vecs_per_row, int need_saved,
                                    int unscale_dy) {
  if (need_saved && !bwd_enabled(hdr)) return;
  const int64_t total = (int64_t)hdr->qlen * vecs_per_row;
  const float sc = unscale_dy ? ldexpf(1.0f, -hdr->dy_exp) : 1.0f;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = idx / vecs_per_row;
    const int c = (int)(idx - t * vecs_per_row);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < top_k; ++s) {
      const int32_t p = inv[t * top_k + s];
      if (p >= 0) {
        const float4 v = src[(int64_t)p * vecs_per_row + c];
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
    }
    const uint32_t lo = (uint32_t)bf16_bits_rn(sc * acc.x) | ((uint32_t)bf16_bits_rn(sc * acc.y) << 16);
    const uint32_t hi = (uint32_t)bf16_bits_rn(sc * acc.z) | ((uint32_t)bf16_bits_rn(sc * acc.w) << 16);
    out[idx] = make_uint2(lo, hi);
  }
}

__global__ void combine_route_kernel(const float* __restrict__ part, int nparts, const int32_t* __restrict__ inv,
                                     int top_k, const WsHeader* hdr, float* __restrict__ grad_route) {
  if (!bwd_enabled(hdr)) return;
  const int64_t total = (int64_t)hdr->qlen * top_k;
  const float sc = ldexpf(1.0f, -hdr->dy_exp);  // the partials carry grad_out's scale
  for (int64_t f = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; f < total; f += (int64_t)gridDim.x * blockDim.x) {
    const int32_t p = inv[f];
    float acc = 0.f;
    if (p >= 0)
      for (int b = 0; b < nparts; ++b) acc += part[(int64_t)p * nparts + b];
    grad_route[f] = sc * acc;
  }
}

// ---------------------------------------------------------------- header
__global__ void header_begin_fwd_kernel(WsHeader* hdr, int save) {
  hdr->magic = kWsMagic;
  hdr->saved = save ? 1u : 0u;
}
__global__ void header_check_bwd_kernel(WsHeader* hdr) {
  hdr->dy_amax = 0u;
  hdr->dy_exp = 0;
  if (hdr->magic != kWsMagic || hdr->saved != 1u) {
    hdr->saved = 0u;
    atomicOr(&hdr->status, (uint32_t)RAWINT4_DEV_NO_SAVED_FORWARD);
  }
}
__global__ void header_end_bwd_kernel(WsHeader* hdr) { hdr->saved = 0u; }

__global__ void fill_u16_kernel(uint16_t* p, int64_t count, uint16_t value) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = value;
}

// ---------------------------------------------------------------- decode
__global__ void decode_kernel(const uint8_t* __restrict__ q, const uint16_t* __restrict__ s, int64_t n, int64_t k,
                              float* __restrict__ out_f32, uint16_t* __restrict__ out_f16) {
  const int64_t groups = n * (k / 32);
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = g / (k / 32);
    const int64_t grp = g - row * (k / 32);
    const uint8_t* src = q + row * (k / 2) + grp * 16;
    const uint16_t sb = s[row * (k / 32) + grp];
    uint4 qv;
    uint8_t* qb = reinterpret_cast<uint8_t*>(&qv);
#pragma unroll
    for (int i = 0; i < 16; ++i) qb[i] = src[i];
    const int64_t o = row * k + grp * 32;
    if (out_f16) {
      uint32_t w[16];
      decode_group32(qv, bf16_scale_to_h2(sb), w);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        out_f16[o + 2 * i] = (uint16_t)(w[i] & 0xFFFFu);
        out_f16[o + 2 * i + 1] = (uint16_t)(w[i] >> 16);
      }
    }
    if (out_f32) {
#pragma unroll
      for (int i = 0; i < 32; ++i) out_f32[o + i] = decode_one_f32(qb[i >> 1], i & 1, sb);
    }
  }
}

// MXFP4 check: out_f16 from the GEMM producers' routine; out_f32 from the
// format's definition, value table times 2^(e - 127), written separately.
__constant__ float kE2M1[16] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f,
                                -0.0f, -0.5f, -1.0f, -1.5f, -2.0f, -3.0f, -4.0f, -6.0f};

__global__ void decode_mxfp4_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ s, int64_t n, int64_t k,
                                    float* __restrict__ out_f32, uint16_t* __restrict__ out_f16) {
  const int64_t groups = n * (k / 32);
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = g / (k / 32);
    const int64_t grp = g - row * (k / 32);
    const uint8_t* src = q + row * (k / 2) + grp * 16;
    const uint32_t e = s[row * (k / 32) + grp];
    uint4 qv;
    uint8_t* qb = reinterpret_cast<uint8_t*>(&qv);
#pragma unroll
    for (int i = 0; i < 16; ++i) qb[i] = src[i];
    const int64_t o = row * k + grp * 32;
    if (out_f16) {
      const uint32_t hb = ue8m0_to_h(e);
      uint32_t w[16];
      decode_group32_mxfp4(qv, __halves2half2(*reinterpret_cast<const __half*>(&hb), *reinterpret_cast<const __half*>(&hb)), w);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        out_f16[o + 2 * i] = (uint16_t)(w[i] & 0xFFFFu);
        out_f16[o + 2 * i + 1] = (uint16_t)(w[i] >> 16);
      }
    }
    if (out_f32) {
      const float sc = e == 0 ? 0.0f : (e == 255 ? INFINITY : ldexpf(1.0f, (int)e - 127));
#pragma unroll
      for (int i = 0; i < 32; ++i) out_f32[o + i] = kE2M1[(qb[i >> 1] >> (4 * (i & 1))) & 15] * sc;
    }
  }
}

// ---------------------------------------------- expert-parallel row moves
// dst[p, :] = src[perm[p] / top_k, :] for p < n (bf16 rows of `vecs` 16-byte
// vectors; every perm[p] in the range is a valid slot).
__global__ void __launch_bounds__(256) dispatch_rows_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ perm,
                                                            int32_t n, int top_k, int vecs, uint4* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t p = warp0; p < n; p += nwarps) {
    const uint4* s = src + (int64_t)(perm[p] / top_k) * vecs;
    uint4* d = dst + p * vecs;
#pragma unroll 4
    for (int c = lane; c < vecs; c += 32) d[c] = __ldg(s + c);
  }
}

// out[t, :] = bf16(sum over s of src[inv[t * top_k + s], :]) in slot order,
// fp32 sums, slots with inv < 0 skipped (8 bf16 per thread and step).
__global__ void combine_slots_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ inv, int32_t qlen,
                                     int top_k, int vecs, uint4* __restrict__ out) {
  const int64_t total = (int64_t)qlen * vecs;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = idx / vecs;
    const int c = (int)(idx - t * vecs);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < top_k; ++s) {
      const int32_t p = inv[t * top_k + s];
      if (p >= 0) {
        const uint4 v = __ldg(src + (int64_t)p * vecs + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[2 * j] += __uint_as_float(w[j] << 16);
          acc[2 * j + 1] += __uint_as_float(w[j] & 0xFFFF0000u);
        }
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      o[j] = (uint32_t)bf16_bits_rn(acc[2 * j]) | ((uint32_t)bf16_bits_rn(acc[2 * j + 1]) << 16);
    out[idx] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// out[f] = inv[f] >= 0 ? src[inv[f]] : 0 for f < n_slots.
__global__ void gather_slots_kernel(const float* __restrict__ src, const int32_t* __restrict__ inv, int32_t n_slots,
                                    float* __restrict__ out) {
  for (int64_t f = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; f < n_slots; f += (int64_t)gridDim.x * blockDim.x) {
    const int32_t p = inv[f];
    out[f] = p >= 0 ? src[p] : 0.f;
  }
}

int grid_for(int64_t work, int threads) {
  int64_t g = (work + threads - 1) / threads;
  if (g > 148 * 16) g = 148 * 16;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

cudaError_t launch_gather_rows(const uint16_t* src_bf16, const int32_t* inv, int top_k, WsHeader* hdr,
                               uint16_t* dst_f16, int H, int max_tokens, uint32_t* status, int need_saved, int scale_dy,
                               cudaStream_t stream) {
  const int vecs = H / 8;
  gather_rows_kernel<<<grid_for((int64_t)max_tokens * 32, 256), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(src_bf16), inv, top_k, hdr, reinterpret_cast<uint4*>(dst_f16), vecs, status,
      need_saved, scale_dy);
  return cudaGetLastError();
}

cudaError_t launch_absmax_rows(const uint16_t* src_bf16, WsHeader* hdr, int H, int max_tokens, cudaStream_t stream) {
  const int vecs = H / 8;
  absmax_rows_kernel<<<grid_for((int64_t)max_tokens * vecs, 256), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(src_bf16), vecs, hdr);
  return cudaGetLastError();
}

cudaError_t launch_combine_rows(const float* src, const int32_t* inv, int top_k, const WsHeader* hdr, uint16_t* out_bf16,
                                int H, int max_tokens, int need_saved, int unscale_dy, cudaStream_t stream) {
  const int vecs = H / 4;
  combine_rows_kernel<<<grid_for((int64_t)max_tokens * vecs, 256), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(src), inv, top_k, hdr, reinterpret_cast<uint2*>(out_bf16), vecs, need_saved,
      unscale_dy);
  return cudaGetLastError();
}

cudaError_t launch_combine_route(const float* part, int nparts, const int32_t* inv, int top_k, const WsHeader* hdr,
                                 float* grad_route, int max_tokens, cudaStream_t stream) {
  combine_route_kernel<<<grid_for((int64_t)max_tokens * top_k, 256), 256, 0, stream>>>(part, nparts, inv, top_k, hdr,
                                                                                       grad_route);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_rows(const uint16_t* src, const int32_t* perm, int32_t n, int top_k, int width,
                                 uint16_t* dst, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  dispatch_rows_kernel<<<grid_for((int64_t)n * 32, 256), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(src), perm, n, top_k, width / 8, reinterpret_cast<uint4*>(dst));
  return cudaGetLastError();
}

cudaError_t launch_combine_slots(const uint16_t* src, const int32_t* inv, int32_t qlen, int top_k, int width,
                                 uint16_t* out, cudaStream_t stream) {
  if (qlen <= 0) return cudaSuccess;
  combine_slots_kernel<<<grid_for((int64_t)qlen * (width / 8), 256), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(src), inv, qlen, top_k, width / 8, reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

cudaError_t launch_gather_slots(const float* src, const int32_t* inv, int32_t n_slots, float* out, cudaStream_t stream) {
  if (n_slots <= 0) return cudaSuccess;
  gather_slots_kernel<<<grid_for(n_slots, 256), 256, 0, stream>>>(src, inv, n_slots, out);
  return cudaGetLastError();
}

cudaError_t launch_header_begin_fwd(WsHeader* hdr, int save, cudaStream_t stream) {
  header_begin_fwd_kernel<<<1, 1, 0, stream>>>(hdr, save);
  return cudaGetLastError();
}
cudaError_t launch_header_check_bwd(WsHeader* hdr, cudaStream_t stream) {
  header_check_bwd_kernel<<<1, 1, 0, stream>>>(hdr);
  return cudaGetLastError();
}
cudaError_t launch_header_end_bwd(WsHeader* hdr, cudaStream_t stream) {
  header_end_bwd_kernel<<<1, 1, 0, stream>>>(hdr);
  return cudaGetLastError();
}

cudaError_t launch_fill_u16(uint16_t* p, int64_t count, uint16_t value, cudaStream_t stream) {
  if (count <= 0) return cudaSuccess;
  fill_u16_kernel<<<grid_for(count, 256), 256, 0, stream>>>(p, count, value);
  return cudaGetLastError();
}

cudaError_t launch_decode_mxfp4(const uint8_t* q, const uint8_t* s, int64_t n, int64_t k, float* out_f32,
                                uint16_t* out_f16, cudaStream_t stream) {
  if (n <= 0 || k <= 0) return cudaSuccess;
  decode_mxfp4_kernel<<<grid_for(n * (k / 32), 128), 128, 0, stream>>>(q, s, n, k, out_f32, out_f16);
  return cudaGetLastError();
}

cudaError_t launch_decode(const uint8_t* q, const uint16_t* s, int64_t n, int64_t k, float* out_f32, uint16_t* out_f16,
                          cudaStream_t stream) {
  if (n <= 0 || k <= 0) return cudaSuccess;
  decode_kernel<<<grid_for(n * (k / 32), 128), 128, 0, stream>>>(q, s, n, k, out_f32, out_f16);
  return cudaGetLastError();
}

}  // namespace r4
