// Token -> expert permutation (histogram, exclusive prefix sum, stable
// scatter) and the token-tile list the grouped GEMMs consume.
//
// The permutation is the stable counting sort of the flat slot index
// f = t * top_k + s by expert id: the gathered-by-expert order that the
// explicit MoE loop of the adjacent ScatterMoE test (test_gemma4_moe.py,
// flatten_sort_count) names, restated for this layer. Rows of one expert
// keep ascending f, so the result is unique and checked bit-exactly.
#include "route.cuh"

namespace r4 {

// Block b counts the experts of slots [b*kRouteChunk, (b+1)*kRouteChunk).
__global__ void __launch_bounds__(kRouteChunk) route_count_kernel(const int64_t* __restrict__ ids, int32_t routed_slots,
                                                                  int32_t experts, int32_t* __restrict__ block_hist,
                                                                  uint32_t* status) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < experts; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int32_t f = blockIdx.x * kRouteChunk + threadIdx.x;
  if (f < routed_slots) {
    const int64_t e = ids[f];
    if (e >= 0 && e < experts) {
      atomicAdd(&hist[e], 1);
    } else {
      raise_status(status, RAWINT4_DEV_BAD_EXPERT_ID);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < experts; e += blockDim.x) block_hist[(size_t)blockIdx.x * experts + e] = hist[e];
}

// Single block: per-expert totals, exclusive prefix over experts (offsets),
// per-(block, expert) scatter bases, and the token-tile list.
__global__ void __launch_bounds__(1024) route_scan_kernel(int32_t* __restrict__ block_hist, int32_t nblocks, int32_t experts,
                                                          int32_t* __restrict__ offsets, int4* __restrict__ tok_tiles,
                                                          WsHeader* hdr, int32_t qlen, int32_t tile_rows) {
  extern __shared__ int32_t sm[];
  int32_t* total = sm;                 // [experts]
  int32_t* ntile = sm + experts;       // [experts]
  int32_t* scratch = sm + 2 * experts; // [1024]
  const int tid = threadIdx.x;
  for (int e = tid; e < experts; e += blockDim.x) {
    int32_t run = 0;
    for (int b = 0; b < nblocks; ++b) {
      const int32_t c = block_hist[(size_t)b * experts + e];
      block_hist[(size_t)b * experts + e] = run;  // exclusive within the expert
      run += c;
    }
    total[e] = run;
    int32_t nt = 0;
    if (run > 0) {
      const int32_t per = (run + tile_rows - 1) / tile_rows;
      int32_t sz = (run + per - 1) / per;
      sz = (sz + 15) / 16 * 16;
      nt = (run + sz - 1) / sz;
    }
    ntile[e] = nt;
  }
  __syncthreads();
  // Two exclusive scans over experts (counts -> offsets, tiles -> tile bases)
  // with a sequential pass per thread over a contiguous slice.
  const int per_t = (experts + blockDim.x - 1) / blockDim.x;
  const int e0 = tid * per_t;
  const int e1 = min(experts, e0 + per_t);
  int32_t s_cnt = 0, s_til = 0;
  for (int e = e0; e < e1; ++e) {
    s_cnt += total[e];
    s_til += ntile[e];
  }
  // block scan of (s_cnt, s_til) packed as two passes through `scratch`
  for (int pass = 0; pass < 2; ++pass) {
    int32_t v = pass == 0 ? s_cnt : s_til;
    scratch[tid] = v;
    __syncthreads();
    for (int off = 1; off < (int)blockDim.x; off <<= 1) {
      const int32_t add = tid >= off ? scratch[tid - off] : 0;
      __syncthreads();
      scratch[tid] += add;
      __syncthreads();
    }
    const int32_t excl = scratch[tid] - v;
    __syncthreads();
    if (pass == 0) {
      int32_t run = excl;
      for (int e = e0; e < e1; ++e) {
        offsets[e] = run;
        run += total[e];
      }
      if (tid == blockDim.x - 1) {
        offsets[experts] = scratch[tid];
        hdr->routed = scratch[tid];
      }
    } else {
      int32_t tb = excl;
      for (int e = e0; e < e1; ++e) {
        const int32_t run = total[e];
        if (run > 0) {
          const int32_t per = (run + tile_rows - 1) / tile_rows;
          int32_t sz = (run + per - 1) / per;
          sz = (sz + 15) / 16 * 16;
          for (int i = 0; i < ntile[e]; ++i) {
            const int32_t r0 = i * sz;
            tok_tiles[tb + i] = make_int4(e, offsets[e] + r0, min(sz, run - r0), 0);
          }
        }
        tb += ntile[e];
      }
      if (tid == blockDim.x - 1) {
        hdr->n_tok_tiles = scratch[tid];
        hdr->qlen = qlen;
      }
    }
    __syncthreads();
  }
  // turn per-(block, expert) exclusive counts into global scatter bases
  for (int e = tid; e < experts; e += blockDim.x) {
    const int32_t base = offsets[e];
    for (int b = 0; b < nblocks; ++b) block_hist[(size_t)b * experts + e] += base;
  }
}

// Stable scatter: slot f goes to base[block][e] + (number of earlier slots
// of the same expert in this block). Warps are walked in order so that the
// rank inside the block ascends with f.
__global__ void __launch_bounds__(kRouteChunk) route_scatter_kernel(const int64_t* __restrict__ ids,
                                                                    const float* __restrict__ rw, int32_t routed_slots,
                                                                    int32_t experts, const int32_t* __restrict__ block_base,
                                                                    int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                                    float* __restrict__ w_perm) {
  extern __shared__ int32_t cursor[];  // [experts]
  for (int e = threadIdx.x; e < experts; e += blockDim.x)
    cursor[e] = block_base[(size_t)blockIdx.x * experts + e];
  __syncthreads();
  const int32_t f = blockIdx.x * kRouteChunk + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  int64_t e64 = -1;
  if (f < routed_slots) e64 = ids[f];
  const bool valid = (f < routed_slots) && e64 >= 0 && e64 < experts;
  const int key = valid ? (int)e64 : -1 - (f >= routed_slots ? 1 : 0);
  const uint32_t peers = __match_any_sync(0xffffffffu, key);
  const uint32_t lt = (1u << lane) - 1u;
  const int rank = __popc(peers & lt);
  const bool leader = (peers & lt) == 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
    if (warp == w && valid) {
      const int32_t pos = cursor[key] + rank;
      perm[pos] = f;
      inv[f] = pos;
      if (w_perm) w_perm[pos] = rw[f];
    }
    __syncwarp();
    if (warp == w && valid && leader) cursor[key] += __popc(peers);
    __syncthreads();
  }
  if (f < routed_slots && !valid) inv[f] = -1;
}

__global__ void fill_i32_kernel(int32_t* p, int32_t from, int32_t to, int32_t value) {
  for (int32_t i = from + blockIdx.x * blockDim.x + threadIdx.x; i < to; i += gridDim.x * blockDim.x) p[i] = value;
}

__global__ void tail_fill_kernel(int32_t* perm, const int32_t* offsets, int32_t experts, int32_t total) {
  const int32_t start = offsets[experts];
  for (int32_t i = start + blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) perm[i] = -1;
}

size_t route_scratch_bytes(int32_t routed_slots, int32_t experts) {
  const int32_t nblocks = (routed_slots + kRouteChunk - 1) / kRouteChunk;
  return (size_t)(nblocks > 0 ? nblocks : 1) * experts * sizeof(int32_t);
}

cudaError_t launch_route(const int64_t* ids, const float* rw, int32_t qlen, int32_t top_k, int32_t experts,
                         int32_t* offsets, int32_t* perm, int32_t* inv, float* w_perm, int4* tok_tiles,
                         int32_t* block_hist, WsHeader* hdr, cudaStream_t stream, int32_t tile_rows) {
  const int32_t slots = qlen * top_k;
  const int32_t nblocks = (slots + kRouteChunk - 1) / kRouteChunk;
  uint32_t* status = hdr ? &hdr->status : nullptr;
  if (nblocks > 0) {
    route_count_kernel<<<nblocks, kRouteChunk, experts * sizeof(int32_t), stream>>>(ids, slots, experts, block_hist,
                                                                                   status);
  }
  const size_t scan_smem = (2 * (size_t)experts + 1024) * sizeof(int32_t);
  route_scan_kernel<<<1, 1024, scan_smem, stream>>>(block_hist, nblocks, experts, offsets, tok_tiles, hdr, qlen,
                                                     tile_rows);
  if (nblocks > 0) {
    route_scatter_kernel<<<nblocks, kRouteChunk, experts * sizeof(int32_t), stream>>>(ids, rw, slots, experts,
                                                                                     block_hist, perm, inv, w_perm);
  }
  return cudaGetLastError();
}

}  // namespace r4
