// Token -> expert permutation that needs no caller-provided scratch.
//
// rawint4_moe_permute needs a device scratch buffer (a header, the token-tile
// list and one per-block expert histogram). Some callers cannot call
// cudaMalloc to provide it: code that runs while another component (for
// example a framework's caching allocator) owns all device memory, or code
// that must not risk the device-wide synchronisation a cudaMalloc can cause
// in the middle of a stream of asynchronous work. This entry point keeps that
// scratch in a fixed-size array in the library's own device memory instead.
#include <mutex>

#include "route.cuh"

namespace r4 {
namespace {

// Scratch of the static variant. Every GPU that loads the library holds this
// array until the process exits; all calls share it.
constexpr size_t kStaticScratchBytes = size_t(1) << 20;  // 1 MiB
__device__ __align__(256) uint8_t g_permute_scratch[kStaticScratchBytes];

constexpr size_t kAlignS = 256;
inline size_t align_s(size_t v) { return (v + kAlignS - 1) / kAlignS * kAlignS; }

// Device address of g_permute_scratch, looked up once per device. In host
// code the array's name is only a host-side stand-in, never a device address.
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RAWINT4_CUDA_ERROR;
  if (dev < 0 || dev >= kMaxDevices) return RAWINT4_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p) {
      cudaGetLastError();  // leave no sticky error for the next library call to report
      return RAWINT4_CUDA_ERROR;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return RAWINT4_OK;
}

}  // namespace
}  // namespace r4

using namespace r4;

extern "C" {

RAWINT4_API size_t rawint4_moe_permute_static_max_bytes(void) { return kStaticScratchBytes; }

RAWINT4_API int rawint4_moe_permute_static(const int64_t* ids, int32_t qlen, int32_t top_k, int32_t experts,
                                           int32_t* offsets, int32_t* perm, int32_t* inv, void* stream_) {
  if (qlen < 0 || top_k < 1 || experts < 1 || experts > 4096 || (int64_t)qlen * top_k > (1 << 24))
    return RAWINT4_INVALID_ARGUMENT;
  if (!offsets || (qlen > 0 && (!ids || !perm || !inv))) return RAWINT4_INVALID_ARGUMENT;
  const int32_t slots = qlen * top_k;
  const size_t hdr_bytes = align_s(sizeof(WsHeader));
  const size_t tile_bytes = align_s((size_t)max_tok_tiles(slots, experts) * 16);
  const size_t need = hdr_bytes + tile_bytes + route_scratch_bytes(slots, experts);
  if (need > kStaticScratchBytes) return RAWINT4_STATIC_SCRATCH_TOO_SMALL;

  int sms = 0;
  int rc = check_device(&sms);  // a device without sm_100 code is UNSUPPORTED, not a CUDA error
  if (rc != RAWINT4_OK) return rc;
  void* base = nullptr;
  rc = scratch_address(&base);
  if (rc != RAWINT4_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream_);
  uint8_t* b = static_cast<uint8_t*>(base);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(b);
  int4* tiles = reinterpret_cast<int4*>(b + hdr_bytes);
  int32_t* hist = reinterpret_cast<int32_t*>(b + hdr_bytes + tile_bytes);
  // the previous call left its header behind: start from zero
  if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st) != cudaSuccess) return RAWINT4_CUDA_ERROR;
  if (launch_route(ids, nullptr, qlen, top_k, experts, offsets, perm, inv, nullptr, tiles, hist, hdr, st) !=
      cudaSuccess)
    return RAWINT4_CUDA_ERROR;
  if (slots > 0) {
    tail_fill_kernel<<<(slots + 255) / 256, 256, 0, st>>>(perm, offsets, experts, slots);
    if (cudaGetLastError() != cudaSuccess) return RAWINT4_CUDA_ERROR;
  }
  return RAWINT4_OK;
}

}  // extern "C"
