#pragma once
#include "common.cuh"

namespace r4 {

// The four dequant-fused grouped GEMMs of the layer. Weight rows (output
// features) sit on the UMMA M side and up to kTileRows permuted tokens of one
// expert on the N side: D[m, n] = sum_k A[m, k] * B[n, k]. Both kernels run on
// CTA pairs (tcgen05 cta_group::2, M = 256 per pair MMA, each SM's TMEM
// holding its 128 rows x N, so two accumulators double-buffer and the
// epilogue of an item overlaps the next item's mainloop); they take the same
// parameters and differ in where the decoded weights go:
//   gemm_tm.cu    into tensor memory (UMMA A operand read from TMEM): the
//                 forward GEMMs (K-major decode) of either base format; its
//                 transpose-free modes are a second path for testing
//   gemm_pair.cu  into shared memory (UMMA A operand from a descriptor): the
//                 transpose-free backward GEMMs of either base format, whose
//                 MN-major tiles need no transposition there
// Each is also built in a narrow tile configuration (gemm_tm_narrow.cu,
// gemm_pair_narrow.cu) for layers with few rows per expert.
enum GemmMode : int {
  kModeGateUp = 0,   // fwd  G/U = X W_{g,u}^T (+ LoRA), SwiGLU epilogue      A: K-major decode of W_g/W_u rows
  kModeDown = 1,     // fwd  y = h W_d^T (+ LoRA), route-weight epilogue       A: K-major decode of W_d rows
  kModeDownT = 2,    // bwd  dh = dY W_d (+ LoRA), SwiGLU' + dRoute epilogue   A: MN-major decode of W_d (transpose-free)
  kModeGateUpT = 3,  // bwd  dx = dG W_g + dU W_u (+ LoRA)                     A: MN-major decode of W_g/W_u
};

constexpr int kBlockK = 64;        // reduction elements per pipeline stage
constexpr int kTmAccCols = 192;    // gemm_tm.cu: columns of one TMEM accumulator = max token-tile rows

// ------------------------------------------------ shared by the pair kernels
constexpr uint64_t kDrainNs = 20000000ull;  // bound on the drains of an aborted call (20 ms)

// UMMA N of a token tile: rounded up to 32 so each CTA's half is a whole
// number of 16-row boxes.
__device__ __forceinline__ int pair_n(int rows) { return max(32, (rows + 31) & ~31); }

// ------------------------------------------------------------ bounded waits
// Sets this CTA's abort flag and the peer's (distributed shared memory), so
// that every role of the pair leaves at its next wait.
__device__ __forceinline__ void abort_pair(volatile int* abort_flag) {
  *abort_flag = 1;
  const uint32_t peer = cluster_addr((const void*)abort_flag, cluster_ctarank() ^ 1u);
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1u) : "memory");
}

// A bound below kPollBelowNs is polled with the non-blocking test (a
// try_wait may suspend until the phase completes, outlasting a short bound).
constexpr uint64_t kPollBelowNs = 1000000ull;

__device__ __forceinline__ bool wait_lim(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* status,
                                         uint64_t limit_ns) {
  const bool poll = limit_ns < kPollBelowNs;
  if (poll ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (poll ? mbar_test_wait(bar, parity) : mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > limit_ns) {
      raise_status(status, RAWINT4_DEV_TIMEOUT);
      abort_pair(abort_flag);
      return false;
    }
  }
}
// The UMMA issuer's wait: never suspends (a suspended issuer resumes late and
// the tensor pipe drains meanwhile) but naps 32 ns between polls, which
// leaves the issue slots of its scheduler to the decoder warps that share it;
// the bound is checked every 256 polls.
__device__ __forceinline__ bool wait_issuer(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* status,
                                            uint64_t limit_ns) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t n = 1;; ++n) {
    __nanosleep(32);
    if (mbar_test_wait(bar, parity)) return true;
    if ((n & 255u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) {
        raise_status(status, RAWINT4_DEV_TIMEOUT);
        abort_pair(abort_flag);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* status,
                                          uint64_t limit_ns) {
  const bool ok = wait_lim(bar, parity, abort_flag, status, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// Waits (bounded) for the fills of the last `n` (at most `stages`) stages a
// producer issued into `full`: a call that aborts must not leave with copies
// still landing in its shared memory.
__device__ __forceinline__ void drain_ring(uint64_t* full, Ring r, int issued, int stages) {
  const int n = issued < stages ? issued : stages;
  const uint64_t t0 = globaltimer();
  for (int j = 0; j < n; ++j) {
    // step back to the previous issue
    if (r.stage == 0) {
      r.stage = stages - 1;
      r.phase ^= 1u;
    } else {
      --r.stage;
    }
    while (!mbar_try_wait(&full[r.stage], r.phase)) {
      if (globaltimer() - t0 > kDrainNs) return;
    }
  }
}
// Copies whose completion is counted on the leader's barrier cannot be
// observed by the peer: it waits a grace period that any issued copy ends in.
__device__ __forceinline__ void grace_wait() {
  const uint64_t t0 = globaltimer();
  while (globaltimer() - t0 < 200000ull) __nanosleep(1000);
}

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
  const uint8_t* e0;         // MXFP4 base: UE8M0 scale bytes of projection 0 and 1
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
  unsigned long long wait_ns;  // bound on any pipeline wait
};

struct GemmMaps {
  CUtensorMap q0;     // packed projection 0: 3D uint8 {stored K bytes, stored rows, E}
  CUtensorMap q1;     // packed projection 1
  CUtensorMap b[4];   // B main: 2D fp16 {K, rows}, 128B swizzle, boxes {64, 16 << i}
  CUtensorMap bx[4];  // B LoRA: 2D fp16 {64, rows}, 128B swizzle, boxes {64, 16 << i}
};

// CTA pairs with the decoded weights in shared memory (gemm_pair.cu), the
// transpose-free modes down^T and gate/up^T of a RAWINT4 or an MXFP4 base
// (fmt); `clusters` pairs (at most the number resident at once).
cudaError_t launch_gemm_pair(int mode, int fmt, const GemmParams& p, const GemmMaps& maps, int clusters,
                             cudaStream_t stream);
// CTA pairs of the pair kernel's mode resident at once on this device (0 on error).
int gemm_pair_max_clusters(int mode, int fmt);
// CTA pairs with the decoded weights in tensor memory (gemm_tm.cu), every
// mode; fmt: RAWINT4_FORMAT_RAWINT4 (bf16 scales s0/s1) or
// RAWINT4_FORMAT_MXFP4 (E2M1 codes, UE8M0 scale bytes e0/e1).
cudaError_t launch_gemm_tm(int mode, int fmt, const GemmParams& p, const GemmMaps& maps, int clusters,
                           cudaStream_t stream);
int gemm_tm_max_clusters(int mode, int fmt);
// The narrow configurations (token tiles of at most kTileRowsNarrow rows,
// hand-off groups of four stages): gemm_tm_narrow.cu for the RAWINT4 forward
// modes, gemm_pair_narrow.cu for the transpose-free backward modes.
cudaError_t launch_gemm_tm_narrow(int mode, int fmt, const GemmParams& p, const GemmMaps& maps, int clusters,
                                  cudaStream_t stream);
int gemm_tm_max_clusters_narrow(int mode, int fmt);
cudaError_t launch_gemm_pair_narrow(int mode, int fmt, const GemmParams& p, const GemmMaps& maps, int clusters,
                                    cudaStream_t stream);
int gemm_pair_max_clusters_narrow(int mode, int fmt);

}  // namespace r4
