// Dequant-fused grouped GEMMs of the routed RAWINT4 MoE-LoRA layer on
// sm_100a tensor cores: CTA pairs (tcgen05 cta_group::2), TMEM accumulators,
// TMA-fed operands. The library runs the transpose-free backward modes here,
// for a RAWINT4 or an MXFP4 base.
//
// Clusters of two CTAs on an SM pair walk (token tile, feature block) work
// items. A token tile is up to kTileRows permuted rows of one expert; a feature
// block is 256 weight rows (gate/up: the same 128 features of gate and up),
// 128 of them decoded in each CTA. The pair-wide MMA (M = 256) reads both
// CTAs' A tiles and both halves of the token tile (each CTA loads its half),
// so every activation byte fetched from L2 feeds 256 weight rows, and each
// CTA's TMEM holds only its 128 rows x N: two accumulators of up to 256
// columns fit, and the epilogue of an item always overlaps the next item's
// mainloop. Warp roles, in each CTA:
//   warp 0      TMA producer of this CTA's packed int4 tiles (ring of kStagesP
//               stages, filled and released in slots of kGroup stages)
//   warp 3      loader of the group scales (cp.async beside each packed
//               stage; its completion is counted on the packed slot's
//               barrier, so a decoder waits once per group for both)
//   warp 2      TMA producer of this CTA's half of the token tile (ring of kStagesB)
//   warps 8-15  decoders: int4 -> fp16 into the UMMA A layout (ring of kStagesA)
//   warp 1      leader CTA: pair-wide UMMA issuer; both CTAs: TMEM allocation
//   warps 4-7   epilogue: this CTA's TMEM rows -> fused math -> global
// The leader's barriers gather both CTAs' readiness (remote arrivals of the
// peer's decoders and epilogue, the peer's TMA bytes counted on the leader's
// barrier); the MMA's commits arrive on both CTAs' barriers.
//
// Hand-off granularity: every synchronisation point in the UMMA issuer's
// stream costs the tensor pipe a few hundred idle cycles, so the issuer waits
// once per group of kGroup stages, on one barrier that means "A and B of the
// whole group are ready": both CTAs' decoders arrive on it after storing the
// group's A tiles, the leader's first decoder warp only once the group's B
// tiles have landed. The decoders decode a group into registers before they
// wait for its A tiles to be free, so only the shared-memory stores sit on
// the chain from the MMA's release of an A tile to its next fill.
//
// The LoRA side product of each projection runs as one extra 64-wide
// reduction stage in the same accumulators: its A operand is the LoRA tensor
// of the expert (loaded into registers at the start of the item and stored
// by the decoders), its B operand the precomputed c-scaled rank-r side matrix.
//
// The backward modes read the packed base along its stored output dimension
// (transpose-free dX, rawint4_sft_reference.py transpose_free_rawint4_dx):
// the decoders write the same packed bytes into an MN-major A tile, so no
// transposed or dense copy of any base weight ever exists.
//
// Two configurations are built from this file: the wide one (this
// translation unit: token tiles of up to kTileRows rows, hand-off groups of
// two stages) and the narrow one (gemm_pair_narrow.cu, R4_PAIR_NARROW = 1:
// tiles of at most kTileRowsNarrow rows, whose small activation tiles leave
// shared memory for eight A tiles in groups of four stages).
#include "gemm.cuh"
#include "route.cuh"

#ifndef R4_PAIR_NARROW
#define R4_PAIR_NARROW 0
#endif
#if R4_PAIR_NARROW
#define R4_PAIR_NS pairk_narrow
#define R4_PAIR_LAUNCH launch_gemm_pair_narrow
#define R4_PAIR_MAXCL gemm_pair_max_clusters_narrow
#else
#define R4_PAIR_NS pairk
#define R4_PAIR_LAUNCH launch_gemm_pair
#define R4_PAIR_MAXCL gemm_pair_max_clusters
#endif

namespace r4 {

namespace R4_PAIR_NS {

constexpr int kRowsM = 128;        // weight rows per CTA (256 per CTA pair)
constexpr int kStagesA = R4_PAIR_NARROW ? 8 : 4;  // decoded FP16 A tiles (16 KB each): two groups
constexpr int kGroup = R4_PAIR_NARROW ? 4 : 2;    // stages per hand-off (issuer wait, decoder arrival)
constexpr int kAGroups = kStagesA / kGroup;
constexpr int kStagesB = 6;        // TMA-loaded B tiles (this CTA's half of up to kTileRows tokens)
constexpr int kStagesP = R4_PAIR_NARROW ? 12 : 16;  // TMA-loaded packed int4 tiles (4 KB each)
constexpr int kStagesS = kStagesP;  // group scales of one stage (512 B each), one per packed stage
// Packed stages and their scales are filled and released in slots of kGroup
// consecutive stages (a hand-off group): one barrier per slot.
constexpr int kSlotsP = kStagesP / kGroup;
constexpr int kThreads = 512;      // 16 warps
constexpr int kEpiWarp0 = 4;       // warps 4..7: epilogue
constexpr int kDecWarp0 = 8;       // warps 8..15: decoders
constexpr int kDecThreads = 256;

constexpr int kABytes = kRowsM * kBlockK * 2;  // 16 KB
constexpr int kTileMax = R4_PAIR_NARROW ? kTileRowsNarrow : kTileRows;  // rows of a token tile
constexpr int kBBytes = (kTileMax / 2) * kBlockK * 2;  // this CTA's half of <= kTileMax tokens (12 KB wide)
constexpr int kPBytes = kRowsM * kBlockK / 2;  // 4 KB
constexpr int kSBytes = 512;                   // 256 bf16 group scales of one stage
constexpr int kOffA = 0;
constexpr int kOffB = kOffA + kStagesA * kABytes;
constexpr int kOffP = kOffB + kStagesB * kBBytes;
constexpr int kOffS = kOffP + kStagesP * kPBytes;
constexpr int kOffBar = kOffS + kStagesS * kSBytes;
constexpr int kNumBars = 2 * kSlotsP + 2 * kAGroups + 2 * kStagesB + 4 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kOffEpi = (kOffMisc + 16 + 127) / 128 * 128;
constexpr int kEpiFloats = 4 * 32 * 33 + 4 * 32;  // DOWN_T route partials; gate/up exchange uses the first 2 * 32 * 33
constexpr int kSmemBytes = kOffEpi + kEpiFloats * 4 + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");
constexpr uint16_t kPairMask = 3;

template <int MODE>
constexpr bool kAMnMajor = (MODE == kModeDownT || MODE == kModeGateUpT);

// 16-wide MMA steps of the LoRA stage: one rank block (padded to rpad) per
// projection, two for the gate/up pair.
template <int MODE>
__device__ __forceinline__ int kext_steps(int rpad) {
  const int kext = (MODE == kModeGateUp || MODE == kModeGateUpT) ? 2 * rpad : rpad;
  return kext / 16;
}

// First output feature of CTA `cta`'s 128 rows of block rb (gate/up: 64
// features, rows 0-63 gate and 64-127 up).
template <int MODE>
__device__ __forceinline__ int cta_f0(int rb, int cta) {
  return MODE == kModeGateUp ? rb * 128 + 64 * cta : rb * 256 + 128 * cta;
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a
// 128B-swizzled block whose rows are 128 bytes and whose 8-row atoms are
// 1024 bytes apart.
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4));
}

// Decoder thread dt decodes one group of 32 weights per stage.
// K-major: weight row dt >> 1, reduction half dt & 1.
// MN-major: stored (reduction) row mn_kr of the 32 features [32 mn_qq, +32);
// each group of 8 consecutive lanes takes 8 consecutive rows of the same
// features, so its 16-byte stores (and its reads of the swizzled packed tile)
// hit 8 distinct bank groups.
__device__ __forceinline__ int mn_kr(int dt) { return 8 * (dt >> 5) + (dt & 7); }
__device__ __forceinline__ int mn_qq(int dt) { return (dt >> 3) & 3; }

// Offset of output chunk j (0..3, 8 fp16 each) of decoder thread dt in the A tile.
template <int MODE>
__device__ __forceinline__ uint32_t a_chunk_off(int dt, int j) {
  if constexpr (!kAMnMajor<MODE>) {
    return sw128_off(dt >> 1, 4 * (dt & 1) + j);
  } else {
    const int qq = mn_qq(dt);
    return (uint32_t)((qq >> 1) * 8192) + sw128_off(mn_kr(dt), 4 * (qq & 1) + j);
  }
}

// This thread's 16 packed bytes in the stage's packed tile. K-major tiles hold
// row r at r * 32; MN-major tiles (64 stored rows x 64 bytes) are loaded with
// 64-byte swizzling (16-byte chunk c of row r at chunk c ^ ((r >> 1) & 3)).
template <int MODE>
__device__ __forceinline__ uint4 packed_group(const uint8_t* P, int dt) {
  if constexpr (!kAMnMajor<MODE>) {
    return *reinterpret_cast<const uint4*>(P + (dt >> 1) * 32 + (dt & 1) * 16);
  } else {
    const int kr = mn_kr(dt);
    return *reinterpret_cast<const uint4*>(P + kr * 64 + 16 * (mn_qq(dt) ^ ((kr >> 1) & 3)));
  }
}

// Scale slot of one stage (written by the loader warp). K-major: [128 rows][2]
// (the two groups of the stage's 64 reduction elements of each weight row).
// MN-major: [64 stored rows][4] (the 4 groups of 32 of this CTA's 128
// features). Decoder thread dt reads its group's scale.
template <int MODE>
__device__ __forceinline__ uint32_t scale_off(int dt) {
  if constexpr (!kAMnMajor<MODE>) {
    return (uint32_t)(dt * 2);  // row (dt >> 1) * 4 bytes + half (dt & 1) * 2
  } else {
    return (uint32_t)(mn_kr(dt) * 8 + mn_qq(dt) * 2);
  }
}

// Loader lane `ln` issues the cp.async copies of stage s's scales into slot
// `S` (zero-filled past the mode's features).
template <int MODE, int FMT>
__device__ __forceinline__ void load_stage_scales(const GemmParams& p, int e, int fc, int s, int ln, uint8_t* S) {
  if constexpr (!kAMnMajor<MODE>) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int row = ln + 32 * t;
      const uint16_t* sp = p.s0;
      int f;
      if constexpr (MODE == kModeGateUp) {
        sp = row < 64 ? p.s0 : p.s1;
        f = fc + (row & 63);
      } else {
        f = fc + row;
      }
      const bool ok = f < p.feat;
      const uint16_t* src = ok ? sp + (int64_t)e * p.s_expert + (int64_t)f * p.s_row + 2 * s : p.s0;
      cp_async_4(S + row * 4, src, ok ? 4u : 0u);
    }
  } else if constexpr (FMT == RAWINT4_FORMAT_MXFP4) {
    // [64 stored rows][4] UE8M0 bytes: the 4 groups of this CTA's 128
    // features (H and I are multiples of 128, so a row's 4 bytes are 4-byte
    // aligned and all inside the features)
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int kr = ln + 32 * t;
      int row = s * kBlockK + kr;
      const uint8_t* sp = p.e0;
      if (MODE == kModeGateUpT && row >= p.stored_rows) {
        row -= p.stored_rows;
        sp = p.e1;
      }
      const bool ok = fc < p.feat;
      const uint8_t* src = sp + (int64_t)e * p.s_expert + (int64_t)row * p.s_row + fc / 32;
      cp_async_4(S + kr * 4, ok ? src : p.e0, ok ? 4u : 0u);
    }
  } else {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int kr = ln + 32 * t;
      int row = s * kBlockK + kr;
      const uint16_t* sp = p.s0;
      if (MODE == kModeGateUpT && row >= p.stored_rows) {
        row -= p.stored_rows;
        sp = p.s1;
      }
      // groups past the features are zero (features come in multiples of 64)
      const uint16_t* src = sp + (int64_t)e * p.s_expert + (int64_t)row * p.s_row + fc / 32;
      const bool ok0 = fc < p.feat, ok1 = fc + 64 < p.feat;
      cp_async_4(S + kr * 8, ok0 ? src : p.s0, ok0 ? 4u : 0u);
      cp_async_4(S + kr * 8 + 4, ok1 ? src + 2 : p.s0, ok1 ? 4u : 0u);
    }
  }
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// This thread's 32 values of the A tile of the LoRA reduction stage that
// starts at column k0, as 16 fp16 pairs in decode order (see a_chunk_off).
// The first stage's values are loaded at the start of a work item, long
// before the stage is stored, which takes the latency of these loads off the
// critical path.
template <int MODE>
__device__ __forceinline__ void lora_values(const GemmParams& p, int e, int fc, int dt, int k0, uint32_t (&w)[16]) {
  const int r = p.rank;
  if constexpr (!kAMnMajor<MODE>) {
    // A[m, j], j in [32 half, 32 half + 32): LoRA B rows (rank contiguous)
    const int m = dt >> 1, half = dt & 1;
    const uint16_t* src = nullptr;
    int jlo = 0;  // first reduction column holding this row's values
    if constexpr (MODE == kModeGateUp) {
      const bool up = m >= 64;
      src = (up ? p.lx1 : p.lx0) + (int64_t)e * p.lx_expert + (int64_t)(fc + (m & 63)) * p.lx_ld;
      jlo = up ? p.rpad : 0;
    } else {
      if (fc + m < p.feat) src = p.lx0 + (int64_t)e * p.lx_expert + (int64_t)(fc + m) * p.lx_ld;
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float v[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int jj = k0 + 32 * half + 2 * t + u - jlo;
        v[u] = (src != nullptr && jj >= 0 && jj < r) ? bf16_bits_to_float(__ldg(src + jj)) : 0.0f;
      }
      w[t] = pack_h2(v[0], v[1]);
    }
  } else {
    // A[m, kr], m in [32 qq, 32 qq + 32): LoRA A rows (feature contiguous)
    const int kr = k0 + mn_kr(dt), f = fc + 32 * mn_qq(dt);
    const uint16_t* src = nullptr;
    if (f < p.feat) {
      if (kr < r)
        src = p.lx0 + (int64_t)e * p.lx_expert + (int64_t)kr * p.lx_ld + f;
      else if (MODE == kModeGateUpT && kr >= p.rpad && kr < p.rpad + r)
        src = p.lx1 + (int64_t)e * p.lx_expert + (int64_t)(kr - p.rpad) * p.lx_ld + f;
    }
    if (src != nullptr) {
      const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 b = __ldg(s4 + c);
        const uint32_t in[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int t = 0; t < 4; ++t)
          w[4 * c + t] = pack_h2(__uint_as_float(in[t] << 16), __uint_as_float(in[t] & 0xFFFF0000u));
      }
    } else {
#pragma unroll
      for (int t = 0; t < 16; ++t) w[t] = 0u;
    }
  }
}

template <int MODE, int FMT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ GemmMaps maps) {
  static_assert(FMT == RAWINT4_FORMAT_RAWINT4 || kAMnMajor<MODE>, "an MXFP4 base runs the transpose-free modes only");
  const CUtensorMap& tq0 = maps.q0;
  const CUtensorMap& tq1 = maps.q1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + kOffA;
  uint8_t* sB = smem + kOffB;
  uint8_t* sP = smem + kOffP;
  uint8_t* sS = smem + kOffS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* p_full = bars;                   // local [kSlotsP]: this CTA's packed slot and its scales landed
  uint64_t* p_empty = p_full + kSlotsP;      // local [kSlotsP]: this CTA's decoders read them
  uint64_t* a_full = p_empty + kSlotsP;      // leader [kAGroups]: the group's A (both CTAs) and B are ready
  uint64_t* a_empty = a_full + kAGroups;     // both [kAGroups]: the pair MMA finished reading the group's A
  uint64_t* b_full = a_empty + kAGroups;     // leader: both CTAs' B halves landed
  uint64_t* b_empty = b_full + kStagesB;     // both: the pair MMA finished reading B
  uint64_t* acc_full = b_empty + kStagesB;   // both [2]: accumulator complete
  uint64_t* acc_empty = acc_full + 2;        // leader [2]: both epilogues drained it
  uint64_t* mma_drain = acc_empty + 2;       // leader: all issued MMAs finished (abort path)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  float* epi = reinterpret_cast<float*>(smem + kOffEpi);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = (int)cluster_ctarank();
  const uint64_t lim = p.wait_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlotsP; ++i) {
      mbar_init(&p_full[i], 1 + 32);  // the TMA producer's arrival (with its bytes) + the scale loader's lanes
      mbar_init(&p_empty[i], kDecThreads / 32);
    }
    for (int i = 0; i < kAGroups; ++i) {
      mbar_init(&a_full[i], 2 * kDecThreads / 32);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < kStagesB; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 2 * 4);
    }
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tq0);
    tma_prefetch_desc(&tq1);
    for (int i = 0; i < 4; ++i) {
      tma_prefetch_desc(&maps.b[i]);
      tma_prefetch_desc(&maps.bx[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // every barrier of both CTAs initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int n_rowblk = p.n_rowblk;
  const int n_tiles = (p.need_saved && p.hdr->saved != 1u) ? 0 : p.hdr->n_tok_tiles * n_rowblk;
  const int n_main = p.n_main;
  // LoRA side product: 64-wide reduction stages over the rank blocks (two
  // for the gate/up pair with a rank above 32)
  const int n_lora = (kext_steps<MODE>(p.rpad) + kBlockK / 16 - 1) / (kBlockK / 16);
  const int tile0 = (int)cluster_id_x();
  const int tile_step = (int)cluster_count_x();
  uint32_t* status = p.status;

  if (warp == 0) {
    // ------------------------------------------------ packed weight producer
    Ring ring;
    int issued = 0;
    for (int tile = tile0; tile < n_tiles; tile += tile_step) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int fc = cta_f0<MODE>(tile % n_rowblk, cta);
      const int e = tt.x;
      for (int s0 = 0; s0 < n_main; s0 += kGroup) {
        const int nsub = min(kGroup, n_main - s0);
        if (!wait_warp(&p_empty[ring.stage], ring.phase ^ 1u, abort_flag, status, lim)) goto drain_p;
        if (lane == 0) {
          uint64_t* bar = &p_full[ring.stage];
          // every box is counted in full, also where it reaches past the
          // tensor (zero-filled rows of a half block)
          mbar_expect_tx(bar, nsub * kPBytes);
          for (int u = 0; u < nsub; ++u) {
          const int s = s0 + u;
          uint8_t* dst = sP + (ring.stage * kGroup + u) * kPBytes;
          if constexpr (MODE == kModeGateUp) {
            tma_load_3d(dst, &tq0, bar, s * (kBlockK / 2), fc, e);
            tma_load_3d(dst + kPBytes / 2, &tq1, bar, s * (kBlockK / 2), fc, e);
          } else if constexpr (MODE == kModeDown) {
            tma_load_3d(dst, &tq0, bar, s * (kBlockK / 2), fc, e);
          } else if constexpr (MODE == kModeDownT) {
            tma_load_3d(dst, &tq0, bar, fc / 2, s * kBlockK, e);
          } else {
            const int k0 = s * kBlockK;
            if (k0 < p.stored_rows)
              tma_load_3d(dst, &tq0, bar, fc / 2, k0, e);
            else
              tma_load_3d(dst, &tq1, bar, fc / 2, k0 - p.stored_rows, e);
          }
          }
        }
        __syncwarp();
        ring.advance(kSlotsP);
        ++issued;
      }
    }
    goto done;
  drain_p:
    if (lane == 0) drain_ring(p_full, ring, issued, kSlotsP);
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------- scale loader
    Ring ring;
    for (int tile = tile0; tile < n_tiles; tile += tile_step) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int fc = cta_f0<MODE>(tile % n_rowblk, cta);
      for (int s0 = 0; s0 < n_main; s0 += kGroup) {
        const int nsub = min(kGroup, n_main - s0);
        if (!wait_warp(&p_empty[ring.stage], ring.phase ^ 1u, abort_flag, status, lim)) goto drain_s;
        for (int u = 0; u < nsub; ++u)
          load_stage_scales<MODE, FMT>(p, tt.x, fc, s0 + u, lane, sS + (ring.stage * kGroup + u) * kSBytes);
        cp_async_arrive_noinc(&p_full[ring.stage]);
        ring.advance(kSlotsP);
      }
    }
  drain_s:
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == 2) {
    // ------------------------------------------------------ B tile producer
    Ring ring;
    int issued = 0;
    for (int tile = tile0; tile < n_tiles; tile += tile_step) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int nb = pair_n(tt.z) / 2;  // this CTA's token rows (multiple of 16)
      const int row0 = tt.y + cta * nb;
      for (int s = 0; s < n_main + n_lora; ++s) {
        if (!wait_warp(&b_empty[ring.stage], ring.phase ^ 1u, abort_flag, status, lim)) goto drain_b;
        if (lane == 0) {
          uint8_t* dst = sB + ring.stage * kBBytes;
          const uint32_t bar = cluster_addr(&b_full[ring.stage], 0);
          if (cta == 0) mbar_expect_tx(&b_full[ring.stage], 2 * nb * 128);
          int row = 0;
          for (int lvl = 3; lvl >= 0; --lvl) {
            const int h = 16 << lvl;
            while (nb - row >= h) {
              if (s < n_main)
                tma_load_2d_pair(dst + row * 128, &maps.b[lvl], bar, s * kBlockK, row0 + row);
              else
                tma_load_2d_pair(dst + row * 128, &maps.bx[lvl], bar, kBlockK * (s - n_main), row0 + row);
              row += h;
            }
          }
        }
        __syncwarp();
        ring.advance(kStagesB);
        ++issued;
      }
    }
    goto done;
  drain_b:
    if (lane == 0) {
      if (cta == 0) drain_ring(b_full, ring, issued, kStagesB);
      grace_wait();
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------- pair UMMA issuer (leader)
    // One thread runs the whole issue loop: per group of stages it waits once
    // (A and B of the group ready), issues the group's UMMAs, frees each B
    // tile and then the group's A tiles by commits.
    if (cta == 0) {
      if (lane == 0) {
        Ring rg, rbr;
        int it = 0;
        bool aborted = false;
        const int ksteps_x = kext_steps<MODE>(p.rpad);
        // descriptors of A tile 0 and B tile 0; a tile adds its bytes, a
        // 16-wide reduction step 32 bytes (K-major) or 2048 bytes (MN-major
        // A: 16 rows of two 8 KB halves), all in 16-byte units
        const uint64_t adesc0 = kAMnMajor<MODE> ? make_sdesc_sw128(smem_u32(sA), 8192, 1024)
                                                : make_sdesc_sw128(smem_u32(sA), 16, 1024);
        const uint64_t bdesc0 = make_sdesc_sw128(smem_u32(sB), 16, 1024);
        constexpr uint64_t kAStep = kAMnMajor<MODE> ? 2048 / 16 : 32 / 16;
        for (int tile = tile0; tile < n_tiles; tile += tile_step, ++it) {
          const int4 tt = p.tok_tiles[tile / n_rowblk];
          const uint32_t idesc = make_idesc_f16((uint32_t)pair_n(tt.z), kAMnMajor<MODE>, false, 256);
          const int ab = it & 1;
          if (!wait_issuer(&acc_empty[ab], ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag, status, lim)) {
            aborted = true;
            goto mma_out;
          }
          tc_fence_after();
          {
            const uint32_t d_tmem = tmem + (uint32_t)(ab * 256);
            uint32_t acc = 0u;  // the item's first UMMA overwrites the accumulator
            // main stages in groups of kGroup, then the LoRA stages as a group
            for (int s = 0; s <= n_main; s += kGroup) {
              const bool lora = s == n_main;
              const int nb = lora ? n_lora : min(kGroup, n_main - s);
              if (!wait_issuer(&a_full[rg.stage], rg.phase, abort_flag, status, lim)) {
                aborted = true;
                goto mma_out;
              }
              tc_fence_after();
              for (int b = 0; b < nb; ++b) {
                const uint64_t ad = adesc0 + (uint64_t)(((kGroup * rg.stage + b) * kABytes) >> 4);
                const uint64_t bd = bdesc0 + (uint64_t)((rbr.stage * kBBytes) >> 4);
                if (!lora) {
#pragma unroll
                  for (int kk = 0; kk < kBlockK / 16; ++kk) {
                    umma_f16_pair(d_tmem, ad + kAStep * kk, bd + (uint64_t)(2 * kk), idesc, acc);
                    acc = 1u;
                  }
                } else {
                  const int ks = min(kBlockK / 16, ksteps_x - (kBlockK / 16) * b);
                  for (int kk = 0; kk < ks; ++kk) {
                    umma_f16_pair(d_tmem, ad + kAStep * kk, bd + (uint64_t)(2 * kk), idesc, acc);
                    acc = 1u;
                  }
                }
                umma_commit_pair(&b_empty[rbr.stage], kPairMask);
                rbr.advance(kStagesB);
              }
              umma_commit_pair(&a_empty[rg.stage], kPairMask);
              rg.advance(kAGroups);
              if (lora) break;
              if (s + kGroup > n_main) s = n_main - kGroup;  // an odd last main stage was its own group
            }
          }
          umma_commit_pair(&acc_full[ab], kPairMask);
        }
      mma_out:
        if (aborted) {
          // every MMA this thread issued has finished before the pair leaves
          umma_commit_pair(mma_drain, 1);
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(mma_drain, 0u)) {
            if (globaltimer() - t0 > kDrainNs) break;
          }
        }
      }
      __syncwarp();
    }
  } else if (warp >= kEpiWarp0 && warp < kDecWarp0) {
    // --------------------------------------------------------------- epilogue
    const int q = warp & 3;       // TMEM lane quarter this warp may access
    const int m = 32 * q + lane;  // accumulator row of this thread
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    int it = 0;
    for (int tile = tile0; tile < n_tiles; tile += tile_step, ++it) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int rb = tile % n_rowblk;
      const int fc = cta_f0<MODE>(rb, cta);
      const bool live = MODE == kModeGateUp || fc < p.feat;  // a half block has no rows in the peer
      const int n_rows = tt.z;
      const int p0 = tt.y;
      const int ab = it & 1;
      if constexpr (MODE == kModeDownT) {
        // the item's saved G/U rows (this warp's 32 features, 128 bytes a
        // row) are brought into L2 while its accumulator is computed
        if (live && fc + 32 * q < p.feat) {
          for (int n = lane; n < n_rows; n += 32) {
            const int64_t o = (int64_t)(p0 + n) * p.ld_out + fc + 32 * q;
            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.in_g + o));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.in_u + o));
          }
        }
      }
      // the four epilogue warps leave together or not at all: a warp that
      // went on alone would wait forever at the exchange barriers
      const bool ok = wait_warp(&acc_full[ab], (uint32_t)(it >> 1) & 1u, abort_flag, status, lim);
      if (!named_bar_and(3, 128, ok)) goto done;
      tc_fence_after();
      const uint32_t d_tmem = tmem + lane_base + (uint32_t)(ab * 256);
      for (int c0 = 0; c0 < n_rows; c0 += 32) {
        uint32_t v[32];
        if constexpr (MODE == kModeGateUp) {
          // rows 0-63: gate features fc + m; rows 64-127: up features fc + m - 64
          tmem_ld32(d_tmem + (uint32_t)c0, v);
          float* xch = epi + (q & 1) * 32 * 33;
          if (q >= 2) {
#pragma unroll
            for (int c = 0; c < 32; ++c) xch[lane * 33 + c] = __uint_as_float(v[c]);
          }
          named_bar_sync(1 + (q & 1), 64);
          if (q < 2) {
            const int i = fc + m;
            const float L = p.limit;
            bool overflow = false;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int n = c0 + c;
              if (n < n_rows) {
                const int64_t o = (int64_t)(p0 + n) * p.ld_out + i;
                const float g = __uint_as_float(v[c]);
                const float u = xch[lane * 33 + c];
                const float gc = L > 0.f ? fminf(g, L) : g;
                const float uc = L > 0.f ? fminf(fmaxf(u, -L), L) : u;
                const float h = gc * sigmoid_clamped(gc) * uc;
                const __half hh = __float2half_rn(h);
                overflow |= __hisinf(hh) != 0;
                p.out_a[o] = g;
                p.out_b[o] = u;
                p.out_h[o] = *reinterpret_cast<const uint16_t*>(&hh);
              }
            }
            if (overflow) raise_status(status, RAWINT4_DEV_FP16_OVERFLOW);
          }
          named_bar_sync(1 + (q & 1), 64);
        } else if constexpr (MODE == kModeDown || MODE == kModeGateUpT) {
          if (live) {
            tmem_ld32(d_tmem + (uint32_t)c0, v);
            float wl = 1.0f;
            if constexpr (MODE == kModeDown) wl = __ldg(p.w_perm + p0 + min(c0 + lane, n_rows - 1));
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int n = c0 + c;
              const float w = __shfl_sync(0xffffffffu, wl, c);
              if (n < n_rows && fc + m < p.feat) {
                float a = __uint_as_float(v[c]);
                if constexpr (MODE == kModeDown) a *= w;
                p.out_a[(int64_t)(p0 + n) * p.ld_out + fc + m] = a;
              }
            }
          }
        } else {  // kModeDownT
          // accumulators of 32 tokens, then the saved G/U of 16 tokens at a
          // time, loaded together ahead of their use (these loads are the
          // epilogue's latency: 16 in flight per thread took down^T from
          // 3.68 to 3.41 ms at the largest layer, against 4)
          const float L = p.limit;
          float* red = epi + q * 32 * 33;
          float* red2 = epi + 4 * 32 * 33;
          bool overflow = false;
          if (live) {
            tmem_ld32(d_tmem + (uint32_t)c0, v);
            const float wl = __ldg(p.w_perm + p0 + min(c0 + lane, n_rows - 1));
            const int i = fc + m;
            const bool row_live = i < p.feat;  // a partial last block
#pragma unroll
            for (int cb = 0; cb < 32; cb += 16) {
              float gq[16], uq[16];
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const int64_t row = p0 + min(c0 + cb + c, n_rows - 1);
                gq[c] = row_live ? __ldg(p.in_g + row * p.ld_out + i) : 0.f;
                uq[c] = row_live ? __ldg(p.in_u + row * p.ld_out + i) : 0.f;
              }
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const int n = c0 + cb + c;
                const float w = __shfl_sync(0xffffffffu, wl, cb + c);
                float pr = 0.f;
                if (n < n_rows && row_live) {
                  const int64_t row = p0 + n;
                  const float acc_v = __uint_as_float(v[cb + c]);
                  const float g = gq[c];
                  const float u = uq[c];
                  const float gc = L > 0.f ? fminf(g, L) : g;
                  const float uc = L > 0.f ? fminf(fmaxf(u, -L), L) : u;
                  const bool pass_g = !(L > 0.f) || g <= L;
                  const bool pass_u = !(L > 0.f) || (u >= -L && u <= L);
                  const float sg = sigmoid_clamped(gc);
                  const float silu = gc * sg;
                  const float dsilu = sg * (1.0f + gc * (1.0f - sg));
                  const float dh = w * acc_v;
                  const float dg = pass_g ? dh * uc * dsilu : 0.f;
                  const float du = pass_u ? dh * silu : 0.f;
                  const __half hg = __float2half_rn(dg);
                  const __half hu = __float2half_rn(du);
                  overflow |= (__hisinf(hg) | __hisinf(hu)) != 0;
                  p.out_h[row * (2 * p.inter) + i] = *reinterpret_cast<const uint16_t*>(&hg);
                  p.out_h[row * (2 * p.inter) + p.inter + i] = *reinterpret_cast<const uint16_t*>(&hu);
                  pr = acc_v * silu * uc;
                }
                red[lane * 33 + cb + c] = pr;
              }
            }
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) red[lane * 33 + c] = 0.f;
          }
          if (overflow) raise_status(status, RAWINT4_DEV_FP16_OVERFLOW);
          __syncwarp();
          float colsum = 0.f;
#pragma unroll 8
          for (int r2 = 0; r2 < 32; ++r2) colsum += red[r2 * 33 + lane];
          red2[q * 32 + lane] = colsum;
          named_bar_sync(3, 128);
          if (q == 0) {
            const int n = c0 + lane;
            if (n < n_rows) {
              const float sum = red2[lane] + red2[32 + lane] + red2[64 + lane] + red2[96 + lane];
              p.droute_part[(int64_t)(p0 + n) * p.n_parts + 2 * rb + cta] = sum;
            }
          }
          named_bar_sync(3, 128);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_addr(&acc_empty[ab], 0));
    }
  } else if (warp >= kDecWarp0) {
    // --------------------------------------------------------------- decoders
    const int dt = threadIdx.x - kDecWarp0 * 32;
    // the leader's first decoder warp also waits for each group's B tiles
    const bool b_watch = cta == 0 && warp == kDecWarp0;
    Ring rg, rp, rbd;
    // this thread's scale in a stage's scale slot (MXFP4: one byte per group)
    const uint32_t s_off = FMT == RAWINT4_FORMAT_MXFP4 ? (uint32_t)(mn_kr(dt) * 4 + mn_qq(dt)) : scale_off<MODE>(dt);
    for (int tile = tile0; tile < n_tiles; tile += tile_step) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int fc = cta_f0<MODE>(tile % n_rowblk, cta);
      const int e = tt.x;
      uint32_t lora_w[16];
      lora_values<MODE>(p, e, fc, dt, 0, lora_w);
      for (int s = 0; s < n_main; s += kGroup) {
        const int nb = min(kGroup, n_main - s);
        // decode the group into registers (needs only its packed and scale
        // stages), then wait for its A tiles to be free and store
        if (!wait_warp(&p_full[rp.stage], rp.phase, abort_flag, status, lim)) goto done;
        // two stages at a time (decoded words of more would not stay in
        // registers); the group's A tiles are waited for once
        for (int h = 0; h < nb; h += 2) {
          uint32_t w[2][16];
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            if (h + b < nb) {
              const int st = rp.stage * kGroup + h + b;
              const uint4 q4 = packed_group<MODE>(sP + st * kPBytes, dt);
              if constexpr (FMT == RAWINT4_FORMAT_MXFP4) {
                const uint32_t hb = ue8m0_to_h(sS[st * kSBytes + s_off]);
                const uint32_t h2 = hb | (hb << 16);
                decode_group32_mxfp4(q4, *reinterpret_cast<const __half2*>(&h2), w[b]);
              } else {
                const uint16_t sc = *reinterpret_cast<const uint16_t*>(sS + st * kSBytes + s_off);
                decode_group32(q4, bf16_scale_to_h2(sc), w[b]);
              }
            }
          }
          if (h + 2 >= nb) {
            // The packed slot and its scales are released once every lane has
            // used the values it loaded from them: the empty asm makes the
            // decoded words (which depend on every loaded byte and on the
            // scale) inputs, so the loads have returned before the release. A
            // release right after the loads were issued could let the refill
            // of the slot land under loads still in flight.
#pragma unroll
            for (int b = 0; b < 2; ++b)
              if (h + b < nb) asm volatile("" ::"r"(w[b][0]), "r"(w[b][15]) : "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_empty[rp.stage]);
            rp.advance(kSlotsP);
          }
          if (h == 0)
            if (!wait_warp(&a_empty[rg.stage], rg.phase ^ 1u, abort_flag, status, lim)) goto done;
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            if (h + b < nb) {
              uint8_t* A = sA + (kGroup * rg.stage + h + b) * kABytes;
#pragma unroll
              for (int j = 0; j < 4; ++j)
                *reinterpret_cast<uint4*>(A + a_chunk_off<MODE>(dt, j)) =
                    make_uint4(w[b][4 * j], w[b][4 * j + 1], w[b][4 * j + 2], w[b][4 * j + 3]);
            }
          }
        }
        fence_proxy_async_smem();
        if (b_watch) {
          for (int b = 0; b < nb; ++b) {
            if (!wait_warp(&b_full[rbd.stage], rbd.phase, abort_flag, status, lim)) goto done;
            rbd.advance(kStagesB);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cluster_addr(&a_full[rg.stage], 0));
        rg.advance(kAGroups);
      }
      // the LoRA reduction stages, a group of their own (the second one, for a
      // rank above 32, loaded here)
      {
        uint32_t lora_w1[16];
        if (n_lora > 1) lora_values<MODE>(p, e, fc, dt, kBlockK, lora_w1);
        if (!wait_warp(&a_empty[rg.stage], rg.phase ^ 1u, abort_flag, status, lim)) goto done;
        uint8_t* A = sA + (kGroup * rg.stage) * kABytes;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(A + a_chunk_off<MODE>(dt, j)) =
              make_uint4(lora_w[4 * j], lora_w[4 * j + 1], lora_w[4 * j + 2], lora_w[4 * j + 3]);
        if (n_lora > 1) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(A + kABytes + a_chunk_off<MODE>(dt, j)) =
                make_uint4(lora_w1[4 * j], lora_w1[4 * j + 1], lora_w1[4 * j + 2], lora_w1[4 * j + 3]);
        }
        fence_proxy_async_smem();
        if (b_watch) {
          for (int b = 0; b < n_lora; ++b) {
            if (!wait_warp(&b_full[rbd.stage], rbd.phase, abort_flag, status, lim)) goto done;
            rbd.advance(kStagesB);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cluster_addr(&a_full[rg.stage], 0));
        rg.advance(kAGroups);
      }
    }
  }

done:
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no MMA, commit or remote arrival of either CTA is still pending
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

template <int MODE, int FMT>
bool set_smem_attr() {
  static std::atomic<unsigned long long> done{0};
  int dev = 0;
  if (!device_flag_test(done, &dev)) {
    if (cudaFuncSetAttribute(gemm_pair_kernel<MODE, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
      return false;
    device_flag_set(done, dev);
  }
  return true;
}

template <int MODE, int FMT>
cudaError_t launch_mode(const GemmParams& p, const GemmMaps& m, int clusters, cudaStream_t stream) {
  if (!set_smem_attr<MODE, FMT>()) return cudaErrorInvalidValue;
  gemm_pair_kernel<MODE, FMT><<<2 * clusters, kThreads, kSmemBytes, stream>>>(p, m);
  return cudaGetLastError();
}

template <int MODE, int FMT>
int max_clusters_mode() {
  if (!set_smem_attr<MODE, FMT>()) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<MODE, FMT>, &cfg) != cudaSuccess) return 0;
  return n;
}

}  // namespace R4_PAIR_NS

// The library runs the two transpose-free backward GEMMs (MN-major decoded
// A tiles in shared memory) on this kernel; the kernel itself is written for
// every mode.
cudaError_t R4_PAIR_LAUNCH(int mode, int fmt, const GemmParams& p, const GemmMaps& maps, int clusters,
                           cudaStream_t stream) {
  constexpr int R = RAWINT4_FORMAT_RAWINT4;
  if (fmt == R) {
    if (mode == kModeDownT) return R4_PAIR_NS::launch_mode<kModeDownT, R>(p, maps, clusters, stream);
    if (mode == kModeGateUpT) return R4_PAIR_NS::launch_mode<kModeGateUpT, R>(p, maps, clusters, stream);
  }
  constexpr int X = RAWINT4_FORMAT_MXFP4;
  if (fmt == X) {
    if (mode == kModeDownT) return R4_PAIR_NS::launch_mode<kModeDownT, X>(p, maps, clusters, stream);
    if (mode == kModeGateUpT) return R4_PAIR_NS::launch_mode<kModeGateUpT, X>(p, maps, clusters, stream);
  }
  return cudaErrorInvalidValue;
}

int R4_PAIR_MAXCL(int mode, int fmt) {
  constexpr int R = RAWINT4_FORMAT_RAWINT4;
  if (fmt == R) {
    if (mode == kModeDownT) return R4_PAIR_NS::max_clusters_mode<kModeDownT, R>();
    if (mode == kModeGateUpT) return R4_PAIR_NS::max_clusters_mode<kModeGateUpT, R>();
  }
  constexpr int X = RAWINT4_FORMAT_MXFP4;
  if (fmt == X) {
    if (mode == kModeDownT) return R4_PAIR_NS::max_clusters_mode<kModeDownT, X>();
    if (mode == kModeGateUpT) return R4_PAIR_NS::max_clusters_mode<kModeGateUpT, X>();
  }
  return 0;
}

}  // namespace r4
