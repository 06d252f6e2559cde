// Top-k softmax router: selection (the layer's expert_ids and route weights)
// and the hand-off of the layer's route gradient back into the router's
// expert scores, as the adjacent MoE system's router computes them
// (test_gemma4_moe.py, Gemma4TextRouter.forward): p = softmax(scores) over
// all experts, the top-k of p, the k renormalised to sum 1, times the
// per-expert scale.
//
// Backward, with r the renormalised weights, c the per-expert scale of each
// selected expert and g the layer's dRoute: h = g c, and the score gradient
// is r_s (h_s - sum_s' r_s' h_s') on the k selected experts and 0 on the
// others (the softmax's normalisation over all experts cancels in r); the
// per-expert scale gradient is the sum of g r over the slots routed to it.
#include "router.cuh"

namespace r4 {
namespace {

constexpr int kRouterWarps = 4;  // tokens per block (one warp each)

__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
    if (v2 > v || (v2 == v && i2 < i)) {
      v = v2;
      i = i2;
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// One warp per token: the probabilities in shared memory, then k rounds of
// arg-max (ties to the lower expert index), each removing its winner.
__global__ void __launch_bounds__(32 * kRouterWarps) router_topk_kernel(const float* __restrict__ scores, int Q, int E,
                                                                        int k, const float* __restrict__ escale,
                                                                        int64_t* __restrict__ ids,
                                                                        float* __restrict__ weights) {
  extern __shared__ float sp[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouterWarps + warp;
  if (t >= Q) return;
  float* p = sp + (size_t)warp * E;
  const float* z = scores + (int64_t)t * E;
  float m = -INFINITY;
  for (int e = lane; e < E; e += 32) m = fmaxf(m, z[e]);
  m = warp_max(m);
  float s = 0.f;
  for (int e = lane; e < E; e += 32) {
    const float v = __expf(z[e] - m);
    p[e] = v;
    s += v;
  }
  s = warp_sum(s);
  const float inv = 1.0f / s;
  __syncwarp();
  float my_p = 0.f;  // lane j < k keeps the j-th selected probability
  int my_i = 0;
  for (int j = 0; j < k; ++j) {
    float v = -1.0f;
    int idx = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      const float pe = p[e];
      if (pe > v || (pe == v && e < idx)) {
        v = pe;
        idx = e;
      }
    }
    warp_argmax(v, idx);
    if (lane == j) {
      my_p = v * inv;
      my_i = idx;
    }
    if (lane == (idx & 31)) p[idx] = -2.0f;  // remove the winner (probabilities are >= 0)
    __syncwarp();
  }
  const float tot = warp_sum(lane < k ? my_p : 0.f);
  if (lane < k) {
    const float c = escale ? escale[my_i] : 1.0f;
    ids[(int64_t)t * k + lane] = my_i;
    weights[(int64_t)t * k + lane] = my_p / tot * c;
  }
}

__global__ void __launch_bounds__(32 * kRouterWarps) router_bwd_kernel(const float* __restrict__ scores, int Q, int E, int k,
                                                                       const int64_t* __restrict__ ids,
                                                                       const float* __restrict__ grad_route,
                                                                       const float* __restrict__ escale,
                                                                       float* __restrict__ grad_scores) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouterWarps + warp;
  if (t >= Q) return;
  float* dz = grad_scores + (int64_t)t * E;
  for (int e = lane; e < E; e += 32) dz[e] = 0.f;
  __syncwarp();
  // the k selected entries: r = softmax over their scores
  int id = 0;
  float z = -INFINITY, g = 0.f, c = 1.f;
  if (lane < k) {
    id = (int)ids[(int64_t)t * k + lane];
    z = scores[(int64_t)t * E + id];
    g = grad_route[(int64_t)t * k + lane];
    c = escale ? escale[id] : 1.0f;
  }
  const float m = warp_max(z);
  const float ez = lane < k ? __expf(z - m) : 0.f;
  const float r = ez / warp_sum(ez);
  const float h = g * c;
  const float hbar = warp_sum(lane < k ? h * r : 0.f);
  if (lane < k) dz[id] = r * (h - hbar);
}

// Per-expert scale gradient, one thread per expert, slots in a fixed order
// (deterministic): sum of g r over the slots routed to the expert.
__global__ void router_scale_grad_kernel(const float* __restrict__ scores, int Q, int E, int k,
                                         const int64_t* __restrict__ ids, const float* __restrict__ grad_route,
                                         float* __restrict__ grad_scale) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  float acc = 0.f;
  for (int t = 0; t < Q; ++t) {
    const int64_t* it = ids + (int64_t)t * k;
    int hit = -1;
    for (int s = 0; s < k; ++s)
      if (it[s] == e) hit = s;
    if (hit < 0) continue;
    // r of this slot: softmax over the token's selected scores
    float m = -INFINITY;
    for (int s = 0; s < k; ++s) m = fmaxf(m, scores[(int64_t)t * E + it[s]]);
    float sum = 0.f, mine = 0.f;
    for (int s = 0; s < k; ++s) {
      const float v = __expf(scores[(int64_t)t * E + it[s]] - m);
      sum += v;
      if (it[s] == e) mine += v * grad_route[(int64_t)t * k + s];
    }
    acc += mine / sum;
  }
  grad_scale[e] = acc;
}

}  // namespace

cudaError_t launch_router_topk(const float* scores, int Q, int E, int k, const float* escale, int64_t* ids,
                               float* weights, cudaStream_t stream) {
  if (Q <= 0) return cudaSuccess;
  const size_t smem = (size_t)kRouterWarps * E * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(router_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
  }
  router_topk_kernel<<<(Q + kRouterWarps - 1) / kRouterWarps, 32 * kRouterWarps, smem, stream>>>(scores, Q, E, k, escale,
                                                                                                  ids, weights);
  return cudaGetLastError();
}

cudaError_t launch_router_bwd(const float* scores, int Q, int E, int k, const int64_t* ids, const float* grad_route,
                              const float* escale, float* grad_scores, float* grad_scale, cudaStream_t stream) {
  if (Q > 0) {
    router_bwd_kernel<<<(Q + kRouterWarps - 1) / kRouterWarps, 32 * kRouterWarps, 0, stream>>>(
        scores, Q, E, k, ids, grad_route, escale, grad_scores);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  if (grad_scale) {
    router_scale_grad_kernel<<<(E + 127) / 128, 128, 0, stream>>>(scores, Q, E, k, ids, grad_route, grad_scale);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace r4
