// Per-launch timing hook (see prof.cuh) and its two C entry points.
#include <mutex>
#include <vector>

#include "../../include/rawint4_moe.h"
#include "prof.cuh"

namespace r4 {
namespace {
struct Rec {
  const char* name;
  cudaEvent_t a, b;
};
std::mutex g_mu;
bool g_on = false;
bool g_open = false;
std::vector<cudaEvent_t> g_pool;
std::vector<Rec> g_recs;
}  // namespace

void prof_mark_begin(const char* name, cudaStream_t stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on || g_open || 2 * (g_recs.size() + 1) > g_pool.size()) return;
  Rec r{name, g_pool[2 * g_recs.size()], g_pool[2 * g_recs.size() + 1]};
  if (cudaEventRecord(r.a, stream) != cudaSuccess) return;
  g_recs.push_back(r);
  g_open = true;
}

void prof_mark_end(cudaStream_t stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on || !g_open) return;
  cudaEventRecord(g_recs.back().b, stream);
  g_open = false;
}

}  // namespace r4

using namespace r4;

extern "C" {

RAWINT4_API int rawint4_moe_profile_begin(int max_launches) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_on || max_launches <= 0 || max_launches > (1 << 16)) return RAWINT4_INVALID_ARGUMENT;
  g_pool.resize(2 * (size_t)max_launches);
  for (auto& e : g_pool)
    if (cudaEventCreate(&e) != cudaSuccess) return RAWINT4_CUDA_ERROR;
  g_recs.clear();
  g_open = false;
  g_on = true;
  return RAWINT4_OK;
}

RAWINT4_API int rawint4_moe_profile_end(int max_out, int* n_out, const char** names, float* ms) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on || !n_out) return RAWINT4_INVALID_ARGUMENT;
  g_on = false;
  int rc = RAWINT4_OK;
  int n = 0;
  for (const Rec& r : g_recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
      rc = RAWINT4_CUDA_ERROR;
      break;
    }
    if (n < max_out) {
      if (names) names[n] = r.name;
      if (ms) ms[n] = t;
    }
    ++n;
  }
  *n_out = n;
  for (auto& e : g_pool) cudaEventDestroy(e);
  g_pool.clear();
  g_recs.clear();
  return rc;
}

}  // extern "C"
