#pragma once
#include "common.cuh"

namespace r4 {

// scores fp32 [Q, E] -> ids int64 [Q, k], weights fp32 [Q, k] (renormalised top-k softmax
// probabilities times escale[id], escale may be null = 1); 1 <= k <= min(E, 32), E <= 4096.
cudaError_t launch_router_topk(const float* scores, int Q, int E, int k, const float* escale, int64_t* ids,
                               float* weights, cudaStream_t stream);

// grad_scores fp32 [Q, E] (overwritten) and grad_scale fp32 [E] (overwritten, may be null)
// from grad_route fp32 [Q, k] = dL/dweights of the selection ids.
cudaError_t launch_router_bwd(const float* scores, int Q, int E, int k, const int64_t* ids, const float* grad_route,
                              const float* escale, float* grad_scores, float* grad_scale, cudaStream_t stream);

}  // namespace r4
