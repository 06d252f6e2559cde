// Shared device helpers for the sm_100a RAWINT4 MoE-LoRA kernels:
// inline-PTX wrappers for mbarriers, TMA (cp.async.bulk.tensor), tcgen05
// (TMEM alloc, UMMA issue/commit, TMEM loads), bounded waits, and the
// RAWINT4 -> FP16 decode used by every GEMM producer and by the decode
// check export.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/rawint4_moe.h"

namespace r4 {

// Host: whether a one-time per-device setting (a kernel's shared-memory
// opt-in) was applied on the current device; the caller sets the bit after
// applying it. Per device, so a process that drives several GPUs applies it
// on each.
inline bool device_flag_test(std::atomic<unsigned long long>& mask, int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  *dev_out = dev;
  return dev < 64 && (mask.load() & (1ull << dev)) != 0;
}
inline void device_flag_set(std::atomic<unsigned long long>& mask, int dev) {
  if (dev < 64) mask.fetch_or(1ull << dev);
}

// Host: the current device is an sm_100 part (RAWINT4_UNSUPPORTED otherwise,
// RAWINT4_CUDA_ERROR when a query fails); *sms receives its SM count.
int check_device(int* sms);

// ------------------------------------------------------------------ status
// Workspace header shared by all kernels of one layer call. Lives at the
// start of the caller's workspace.
struct WsHeader {
  uint32_t magic;        // RAWINT4_WS_MAGIC once a forward ran
  uint32_t saved;        // 1: a saved forward context is pending
  int32_t qlen;          // tokens of the saved / last forward
  int32_t routed;        // valid permuted rows (ids in [0, E))
  uint32_t status;       // OR of RAWINT4_DEV_* bits
  int32_t n_tok_tiles;   // entries of the token-tile list
  uint32_t dy_amax;      // backward: largest |grad_out| element, as its bf16 magnitude bits
  int32_t dy_exp;        // backward: grad_out enters the fp16 operands scaled by 2^dy_exp
  int32_t pad[8];
};
static_assert(sizeof(WsHeader) == 64, "workspace header layout");

// Exponent s of the power-of-two scale applied to grad_out before it is
// converted to fp16 operands: the largest magnitude times 2^s lies in [1, 2),
// so every element keeps fp16's full relative precision unless it is more
// than 2^14 times smaller than the largest one, and nothing overflows. The
// backward is linear in grad_out (the clamp masks depend only on the saved
// forward), so every output is exact after multiplying by 2^-s in fp32. An
// all-zero or non-finite grad_out takes s = 0.
__device__ __forceinline__ int dy_scale_exponent(uint32_t amax_bits16) {
  if (amax_bits16 == 0u || amax_bits16 >= 0x7F80u) return 0;
  int e = 0;
  frexpf(__uint_as_float(amax_bits16 << 16), &e);  // |max| = f 2^e, f in [0.5, 1)
  return min(120, max(-120, 1 - e));
}
constexpr uint32_t kWsMagic = 0x52344d45u;  // "R4ME"
// Width (fp16 columns) of the rank-side matrices of the LoRA products: the gate
// and up rank blocks, each padded to a multiple of 16 (rank <= 64).
constexpr int kLoraPad = 128;

constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s bound on any spin

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void raise_status(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

// ------------------------------------------------------------- smem / misc
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;  // (a & b) | c
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ANDs a predicate over the participating threads:
// every participant gets the same result.
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.b32 p, %1, 0;\n bar.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of phase `parity` (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that may suspend the thread (instead of spinning) for up to
// `hint_ns` while the phase is incomplete; it returns as soon as the phase
// completes, so waiting warps leave the issue slots to working warps.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait on phase `parity`. Returns false (and raises the abort flag and
// the device timeout bit) when the bound expires or another role aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      raise_status(status, RAWINT4_DEV_TIMEOUT);
      return false;
    }
  }
}

// Warp-wide bounded wait: every lane polls, the result is made uniform.
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// Position in a ring of pipeline stages: stage index and its phase parity.
struct Ring {
  int stage = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance(int n) {
    if (++stage == n) {
      stage = 0;
      phase ^= 1u;
    }
  }
};

// --------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t c0,
                                            int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t c0,
                                            int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// ----------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, FP16 inputs, FP32 accumulator.
__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when all previously issued MMAs of this thread finish.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Instruction descriptor, kind::f16: FP16 A/B, FP32 D, M = 128 (or 256 for
// a CTA-pair MMA).
__host__ __device__ constexpr uint32_t make_idesc_f16(uint32_t n, bool a_mn_major, bool b_mn_major,
                                                      uint32_t m = 128) {
  return (1u << 4)                          // D format: F32
         | (0u << 7) | (0u << 10)           // A, B format: F16
         | ((a_mn_major ? 1u : 0u) << 15)   // A major
         | ((b_mn_major ? 1u : 0u) << 16)   // B major
         | ((n >> 3) << 17)                 // N / 8
         | ((m >> 4) << 24);                // M / 16
}

// Shared-memory matrix descriptor with 128-byte swizzling.
// lbo/sbo in bytes (multiples of 16); the atom base must be 1024-byte aligned.
__device__ __forceinline__ uint64_t make_sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// 32 lanes x 32 consecutive 32-bit columns of TMEM into registers.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Registers into 32 lanes x 16 consecutive 32-bit columns of TMEM (thread i
// of the warp writes lane base + i); tmem_wait_st waits for this thread's
// stores to complete.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns of TMEM into registers.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------- cp.async with mbarrier
// Small asynchronous global->shared copies whose completion is counted on an
// mbarrier: the issuing thread never waits for them (unlike ordinary loads,
// which a later release-arrive of the same thread would have to wait for).
// `src_bytes` 0 fills the destination with zeros without reading.
__device__ __forceinline__ void cp_async_4(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_8(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(src_bytes)
               : "memory");
}
// Arrive on `bar` once all cp.async of this thread issued so far have landed
// (the barrier's expected count includes these arrivals).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ------------------------------------------------------ CTA pairs (2 SMs)
// A cluster of two CTAs on one SM pair: rank 0 (the leader) issues the
// pair-wide MMAs; every other wrapper runs in both CTAs.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// All threads of both CTAs (each warp converged).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The shared::cluster address of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Arrive on an mbarrier given by its shared::cluster address (either CTA),
// with the default (CTA-scope release) semantics: the operand data the
// arrival announces lives in the arriving CTA's own shared memory and is
// made visible to that SM's tensor-core (async) proxy by a proxy fence
// before the arrival. A cluster-scope release here costs a full memory
// barrier per arrival (about 0.7 us measured) and is not needed for that.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// try_wait for phases completed by the peer CTA or by pair-wide tensor-core
// commits (default acquire semantics, as for local phases).
__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             uint32_t* status) {
  if (mbar_try_wait_cl(bar, parity, 0u)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_cl(bar, parity, 1000000u)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      raise_status(status, RAWINT4_DEV_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ bool wait_all_cl(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                            uint32_t* status) {
  const bool ok = mbar_wait_cl(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}
// Tiled TMA load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (shared::cluster address). Each CTA
// loads only its own tile, from this GPU's memory, into its own shared memory.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int32_t c0,
                                                 int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Pair-wide D[tmem] (+)= A * B^T: M = 256 (rows 0-127 from the leader's A
// tile, 128-255 from the peer's at the same offset), N columns of B split
// between the two CTAs (first half in the leader), FP16 in, FP32 accumulate;
// each CTA's TMEM receives its own 128 rows. Issued by one leader thread.
__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Pair-wide D[tmem] (+)= A[tmem] * B^T: as umma_f16_pair, but the A operand
// (128 rows x 16 fp16 per CTA, K-major, two elements per 32-bit column) is
// read from each CTA's tensor memory at the same address instead of shared
// memory.
__device__ __forceinline__ void umma_f16_pair_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` (same offset) in every CTA of `cta_mask` when all MMAs
// this thread issued so far have finished.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// ------------------------------------------------------------------ decode
// bf16 bit pattern -> fp16 pair holding the same value twice (exact for
// magnitudes in the fp16 normal range).
__device__ __forceinline__ __half2 bf16_scale_to_h2(uint16_t bits) {
  const float f = __uint_as_float(static_cast<uint32_t>(bits) << 16);
  return __float2half2_rn(f);
}

// Decode 16 packed bytes (32 RAWINT4 codes, low nibble first) that share one
// group scale into 16 fp16x2 words, element order preserved: word j holds
// values 2j (low half) and 2j+1 (high half).
//
// Per byte b: replicate it, keep the low nibble in bits 0-3 of the low half
// and the high nibble in bits 4-7 of the high half, and OR in the exponent
// of 1024.0 (fp16 0x6400, whose ulp is 1). That yields exactly 1024 + lo and
// 1024 + 16*hi; one fused multiply-add by (1, 1/16) plus (-1032, -72) gives
// lo - 8 and hi - 8 exactly, and one multiply by the scale gives the weight
// (exact: at most 11 significant bits).
__device__ __forceinline__ void decode_group32(const uint4 q, const __half2 s2, uint32_t (&out)[16]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  const __half2 mul = __halves2half2(__float2half_rn(1.0f), __float2half_rn(0.0625f));
  const __half2 add = __halves2half2(__float2half_rn(-1032.0f), __float2half_rn(-72.0f));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t rep = __byte_perm(w[i], 0u, 0x1111u * j);
      const uint32_t v = lop3_and_or(rep, 0x00F0000Fu, 0x64006400u);
      __half2 h = __hfma2(*reinterpret_cast<const __half2*>(&v), mul, add);
      h = __hmul2(h, s2);
      out[i * 4 + j] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
}

// ------------------------------------------------------------------ MXFP4
// UE8M0 scale byte e -> fp16 bits of its value 2^(e - 127) (the pages' bit-cast
// of e into a bf16 exponent). fp16 holds it exactly for e in [103, 142]
// (normal for e >= 113, subnormal below); e == 0 -> 0, a larger e -> inf, a
// smaller nonzero e -> 0 (outside the supported range).
__device__ __forceinline__ uint32_t ue8m0_to_h(uint32_t e) {
  if (e >= 113u && e <= 142u) return (e - 112u) << 10;
  if (e >= 103u && e < 113u) return 1u << (e - 103u);
  return e > 142u ? 0x7C00u : 0u;
}

// Two E2M1 codes (bits 0-3: first value, 4-7: second) -> fp16 pair, by the
// hardware conversion (exact: every E2M1 value is an fp16 number).
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte_lo8) {
  uint32_t d;
  asm("{\n .reg .b8 t;\n cvt.u8.u32 t, %1;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}" : "=r"(d) : "r"(byte_lo8));
  return d;
}

// Decode 16 packed bytes (32 E2M1 codes, low nibble first) that share one
// group scale (fp16 pair `s2`) into 16 fp16x2 words, element order preserved.
// Exact whenever the product is an fp16 number (scale bytes in [104, 140]).
__device__ __forceinline__ void decode_group32_mxfp4(const uint4 q, const __half2 s2, uint32_t (&out)[16]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t v = e2m1x2_to_h2(w[i] >> (8 * j));
      __half2 h = __hmul2(*reinterpret_cast<const __half2*>(&v), s2);
      out[i * 4 + j] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
}

// Plain fp32 decode of one code (for the check export's fp32 output).
__device__ __forceinline__ float decode_one_f32(uint8_t byte, int hi, uint16_t scale_bits) {
  const int code = hi ? (byte >> 4) : (byte & 15);
  return static_cast<float>(code - 8) * __uint_as_float(static_cast<uint32_t>(scale_bits) << 16);
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}
__device__ __forceinline__ float bf16_bits_to_float(uint16_t bits) {
  return __uint_as_float(static_cast<uint32_t>(bits) << 16);
}
__device__ __forceinline__ uint16_t f16_bits_rn(float f) {
  __half h = __float2half_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}
__device__ __forceinline__ float f16_bits_to_float(uint16_t bits) {
  __half h = *reinterpret_cast<__half*>(&bits);
  return __half2float(h);
}

// SiLU pieces with the exponent argument clamped so that exp never
// overflows (the tails give sigma = 0 or 1 without NaN).
__device__ __forceinline__ float sigmoid_clamped(float z) {
  const float e = __expf(fminf(-z, 88.0f));
  return 1.0f / (1.0f + e);
}

}  // namespace r4
