// Dequant-fused grouped GEMMs of the routed RAWINT4 MoE-LoRA layer on
// sm_100a tensor cores with the decoded weight operand in tensor memory.
//
// Clusters of two CTAs on an SM pair walk (token tile, feature block) work
// items, as the CTA-pair kernel of gemm_pair.cu does: 256 weight rows per item
// (128 per CTA), one pair-wide M = 256 UMMA per 16-wide reduction step, each
// CTA loading its half of the token tile. The difference is where the decoded
// weights go: the decoder warps store them with tcgen05.st into a ring of A
// stages in each CTA's tensor memory, and the UMMA reads A from there
// (tcgen05.mma [d], [a-tmem], b-desc). Shared memory then holds only the TMA
// rings of packed weights, group scales and activation tiles, which can be
// made several times deeper than with decoded tiles in shared memory, and the
// tensor cores read only the activation tiles from it.
//
// Tensor memory of each CTA (512 columns x 128 lanes):
//   [0, 2 kAccCols)                 two accumulators of up to kAccCols token columns
//   [2 kAccCols, + 32 kAStages)     A stages: 128 weight rows x 64 reduction fp16
// so a token tile has at most kAccCols rows (the tile list is cut to that).
//
// Hand-off granularity: every synchronisation point in the UMMA issuer's
// stream (a barrier wait, also one delegated to another warp) leaves the
// tensor pipe idle for a few hundred cycles, so the issuer waits once per
// group of kGroup stages (4 kGroup UMMAs) on one barrier that means "A and B
// of the whole group are ready": the decoders arrive on it after storing the
// group's A stages, and the leader's first decoder warp arrives only once the
// group's B stages have landed. The A stages form kAStages / kGroup groups.
//
// Warp roles, in each CTA:
//   warp 0      TMA producer of this CTA's packed int4 tiles (ring of kStagesP)
//   warp 1      leader CTA: pair-wide UMMA issuer; both CTAs: TMEM allocation
//   warp 2      TMA producer of this CTA's half of the token tile (ring of kStagesB)
//   warp 3      loader of the group scales (cp.async into the scale slot of
//               each packed slot; its completion is counted on the packed
//               slot's barrier, so a decoder waits once per slot for both)
//   warps 4-7   epilogue: this CTA's TMEM rows -> fused math -> global
//   warps 8-15  decoders: int4 -> fp16 -> tensor memory (two warps per lane quarter)
//
// K-major modes (gate/up and down forward): decoder warp (q, g) owns TMEM
// lanes 32q..32q+31 (weight rows) and the 32-wide reduction group g of each
// 64-wide stage; a thread decodes the 16 packed bytes of its row and group
// and stores the 32 fp16 values as 16 columns of its lane.
//
// MN-major modes (the transpose-free backward, rawint4_sft_reference.py
// transpose_free_rawint4_dx: down^T and gate/up^T): the packed base is read
// along its stored output dimension, so one stored row holds one reduction
// index for many weight rows. Decoder warp (q, g) loads the 32 stored rows of
// group g (lane i: row i, the 16 bytes of the warp's 32 weight rows), turns
// that 32 x 32 nibble block around across the warp with five shuffle and
// byte-permute steps (lane m then holds the 32 reduction values of weight row
// m), decodes with the per-row group scales and stores to its TMEM lane as in
// the K-major modes. No transposed or dense copy of a base weight is made.
//
// The LoRA side product of each projection runs as one extra 64-wide
// reduction stage in the same accumulators: its A operand is the LoRA tensor
// of the expert (loaded into registers at the start of the item and stored by
// the decoders), its B operand the precomputed c-scaled rank-r side matrix.
//
// Two configurations are built from this file. The wide one (this
// translation unit) holds token tiles of up to kTmAccCols rows with groups of
// two stages; the narrow one (gemm_tm_narrow.cu, R4_TM_NARROW = 1), for
// layers with few rows per expert, holds tiles of at most kTileRowsNarrow
// rows, so tensor memory has room for eight A stages and the hand-off groups
// are four stages long (half the synchronisations per weight byte); it runs
// the forward modes of either base format.
#include "gemm.cuh"
#include "route.cuh"

#ifndef R4_TM_NARROW
#define R4_TM_NARROW 0
#endif
#if R4_TM_NARROW
#define R4_TM_NS tmk_narrow
#define R4_TM_LAUNCH launch_gemm_tm_narrow
#define R4_TM_MAXCL gemm_tm_max_clusters_narrow
#else
#define R4_TM_NS tmk
#define R4_TM_LAUNCH launch_gemm_tm
#define R4_TM_MAXCL gemm_tm_max_clusters
#endif

namespace r4 {

namespace R4_TM_NS {

constexpr int kAccCols = R4_TM_NARROW ? kTileRowsNarrow : kTmAccCols;  // columns of one accumulator
constexpr int kAStages = R4_TM_NARROW ? 8 : 4;    // A stages in tensor memory (32 columns each)
constexpr uint32_t kACol0 = 2 * kAccCols;         // first A column
static_assert(kACol0 + 32 * kAStages <= 512, "tensor memory columns");
constexpr int kStagesB = 10;                      // TMA-loaded B half tiles
// Packed weights and their scales arrive in slots of several reduction
// stages: a TMA box row is one memory request, and a K-major row of one stage
// is only 32 bytes, so a slot holds kPSub stages of each row (a 128-byte box
// row). K-major: 4 stages per slot (16 KB, 4 slots); MN-major: 2 stages (two
// 64-row boxes of 64-byte rows, 8 KB, 8 slots).
template <int MODE>
constexpr int kPSub = (MODE == kModeDownT || MODE == kModeGateUpT) ? 2 : 4;
constexpr int kPSlotBytes = 16384;                // largest packed slot
constexpr int kPRing = 65536;                     // bytes of the packed ring
template <int MODE>
constexpr int kStagesP = kPRing / (kPSub<MODE> * 4096);  // packed slots
constexpr int kMaxStagesP = 16;
constexpr int kSSlotBytes = 2048;                 // largest scale slot
constexpr int kStagesS = 8;                       // scale slots: one per packed slot (at most 8 packed slots)
static_assert(kStagesS >= kPRing / (2 * 4096), "a scale slot for every packed slot");
constexpr int kThreads = 512;                     // 16 warps
constexpr int kEpiWarp0 = 4;                      // warps 4..7: epilogue
constexpr int kDecWarp0 = 8;                      // warps 8..15: decoders
constexpr int kDecWarps = 8;
constexpr int kGroup = R4_TM_NARROW ? 4 : 2;      // stages per hand-off (issuer wait, decoder arrival)
constexpr int kAGroups = kAStages / kGroup;       // groups of A stages in tensor memory
static_assert(kAGroups >= 2, "the MMA consumes one group while the next is decoded");

constexpr int kBBytes = (kAccCols / 2) * kBlockK * 2;    // this CTA's half of <= kAccCols tokens
template <int MODE>
constexpr int kPBytes = kPSub<MODE> * 4096;              // one packed slot (4 KB per stage)
template <int MODE>
constexpr int kSBytes = kPSub<MODE> * 512;               // one scale slot (256 bf16 per stage)
constexpr int kOffB = 0;
constexpr int kOffP = kOffB + kStagesB * kBBytes;
constexpr int kOffS = kOffP + kPRing;
constexpr int kOffBar = kOffS + kStagesS * kSSlotBytes;
constexpr int kNumBars = 2 * kMaxStagesP + 2 * kAStages + 2 * kStagesB + 2 * kStagesS + 4 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kOffEpi = (kOffMisc + 16 + 127) / 128 * 128;
constexpr int kEpiFloats = 4 * 32 * 33 + 4 * 32;  // down^T dRoute partials; gate/up exchange uses 2 * 32 * 33
constexpr int kTabBytes = 8 * 64 * 2;             // MN-major: 16-pair scale tables, two per decoder warp
constexpr int kOffScaleTab = kOffEpi + kEpiFloats * 4;
constexpr int kSmemBytes = kOffScaleTab + kTabBytes + 1024;  // + alignment slack
static_assert(kBBytes % 1024 == 0 && kPRing % kPSlotBytes == 0, "1024-byte aligned stages");
static_assert(kSmemBytes <= 232448, "shared memory budget");
constexpr uint16_t kPairMask = 3;

template <int MODE>
constexpr bool kAMnMajor = (MODE == kModeDownT || MODE == kModeGateUpT);

template <int MODE>
__device__ __forceinline__ int kext_steps(int rpad) {
  const int kext = (MODE == kModeGateUp || MODE == kModeGateUpT) ? 2 * rpad : rpad;
  return kext / 16;
}

// First output feature of CTA `cta`'s 128 rows of block rb (gate/up: 64
// features, TMEM lanes 0-63 gate and 64-127 up).
template <int MODE>
__device__ __forceinline__ int cta_f0(int rb, int cta) {
  return MODE == kModeGateUp ? rb * 128 + 64 * cta : rb * 256 + 128 * cta;
}

// First packed slot of work item (tile, feature block rb): the items of
// one token tile start their reduction at evenly spread stages (and wrap
// around), so the CTA pairs that work on the same token tile at the same time
// read different activation rows from L2 instead of the same ones in step.
__device__ __forceinline__ int k_rotation(int rb, int n_rowblk, int n_slots) {
#ifdef R4_NO_KROT
  return 0;
#else
  return (int)(((int64_t)rb * n_slots) / n_rowblk);
#endif
}
__device__ __forceinline__ int rotated(int s, int rot, int n_main) {
  const int k = s + rot;
  return k >= n_main ? k - n_main : k;
}

// ----------------------------------------------------------- K-major decode
// K-major scale slot j: [128 rows][8] bf16, the groups 8j..8j+7 of each
// weight row (its two groups of each of the slot's 4 stages); entries past the
// features or the reduction are zero.
template <int MODE, int FMT>
__device__ __forceinline__ void load_slot_scales(const GemmParams& p, int e, int fc, int j, int n_main, int ln,
                                                 uint8_t* S) {
  if constexpr (FMT == RAWINT4_FORMAT_MXFP4) {
    // UE8M0 bytes: [128 rows][8], 4 bytes (two stages) per copy; rows are
    // 4-byte aligned (K % 128 == 0)
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int row = ln + 32 * t;
      const uint8_t* ep = p.e0;
      int f;
      if constexpr (MODE == kModeGateUp) {
        ep = row < 64 ? p.e0 : p.e1;
        f = fc + (row & 63);
      } else {
        f = fc + row;
      }
      const bool ok = f < p.feat;
      const uint8_t* src = ep + (int64_t)e * p.s_expert + (int64_t)f * p.s_row + 8 * j;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const bool v = ok && 4 * j + 2 * h < n_main;
        cp_async_4(S + row * 8 + 4 * h, v ? src + 4 * h : p.e0, v ? 4u : 0u);
      }
    }
  } else {
  const bool full = 4 * j + 4 <= n_main && (p.s_row & 7) == 0;  // 16-byte aligned whole slot
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
    const uint16_t* src = sp + (int64_t)e * p.s_expert + (int64_t)f * p.s_row + 8 * j;
    if (full) {
      cp_async_16(S + row * 16, ok ? src : p.s0, ok ? 16u : 0u);
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool v = ok && 4 * j + u < n_main;
        cp_async_4(S + row * 16 + 4 * u, v ? src + 2 * u : p.s0, v ? 4u : 0u);
      }
    }
  }
  }
}

template <int MODE, int FMT>
__device__ __forceinline__ void load_slot_scales_mn(const GemmParams& p, int e, int fc, int j, int n_main, int ln,
                                                    uint8_t* S) {
  if constexpr (FMT == RAWINT4_FORMAT_MXFP4) {
    // UE8M0 bytes: [128 stored rows][4] (this CTA's 4 groups; features and
    // stored rows are multiples of 128 for MXFP4, so a group is all in or out)
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int kr = ln + 32 * t;
      if (2 * j + (kr >> 6) >= n_main) continue;
      int row = 2 * j * kBlockK + kr;
      const uint8_t* ep = p.e0;
      if (MODE == kModeGateUpT && row >= p.stored_rows) {
        row -= p.stored_rows;
        ep = p.e1;
      }
      const bool ok = fc < p.feat;
      cp_async_4(S + kr * 4, ok ? ep + (int64_t)e * p.s_expert + (int64_t)row * p.s_row + fc / 32 : p.e0, ok ? 4u : 0u);
    }
  } else {
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int kr = ln + 32 * t;
    if (2 * j + (kr >> 6) >= n_main) continue;
    int row = 2 * j * kBlockK + kr;
    const uint16_t* sp = p.s0;
    if (MODE == kModeGateUpT && row >= p.stored_rows) {
      row -= p.stored_rows;
      sp = p.s1;
    }
    // groups past the features are zero (a zero scale decodes every code to
    // 0); features come in multiples of 64, so the two 4-byte halves suffice
    const uint16_t* src = sp + (int64_t)e * p.s_expert + (int64_t)row * p.s_row + fc / 32;
    const bool ok0 = fc < p.feat, ok1 = fc + 64 < p.feat;
    cp_async_4(S + kr * 8, ok0 ? src : p.s0, ok0 ? 4u : 0u);
    cp_async_4(S + kr * 8 + 4, ok1 ? src + 2 : p.s0, ok1 ? 4u : 0u);
  }
  }
}

// 32 x 32 transpose of 4-bit values across a warp. On entry lane i holds row
// i (nibble c at bits 4 (c % 8) of w[c / 8]); on exit lane i holds column i
// in the same layout. Step d (16, 8, 4, 2, 1) swaps, between lanes l and
// l ^ d, the entries whose column bit d differs from the lane's bit d.
__device__ __forceinline__ void transpose_nibbles(uint32_t (&w)[4], int lane) {
  constexpr uint32_t kFull = 0xffffffffu;
  {
    const bool b = lane & 16;
    const uint32_t y0 = __shfl_xor_sync(kFull, b ? w[0] : w[2], 16);
    const uint32_t y1 = __shfl_xor_sync(kFull, b ? w[1] : w[3], 16);
    if (b) {
      w[0] = y0;
      w[1] = y1;
    } else {
      w[2] = y0;
      w[3] = y1;
    }
  }
  {
    const bool b = lane & 8;
    const uint32_t y0 = __shfl_xor_sync(kFull, b ? w[0] : w[1], 8);
    const uint32_t y1 = __shfl_xor_sync(kFull, b ? w[2] : w[3], 8);
    if (b) {
      w[0] = y0;
      w[2] = y1;
    } else {
      w[1] = y0;
      w[3] = y1;
    }
  }
  {  // half words
    const bool b = lane & 4;
    const uint32_t ps = b ? 0x5410u : 0x7632u;
    const uint32_t y0 = __shfl_xor_sync(kFull, __byte_perm(w[0], w[1], ps), 4);
    const uint32_t y1 = __shfl_xor_sync(kFull, __byte_perm(w[2], w[3], ps), 4);
    const uint32_t u0 = b ? 0x3254u : 0x5410u, u1 = b ? 0x3276u : 0x7610u;
    w[0] = __byte_perm(w[0], y0, u0);
    w[1] = __byte_perm(w[1], y0, u1);
    w[2] = __byte_perm(w[2], y1, u0);
    w[3] = __byte_perm(w[3], y1, u1);
  }
  {  // bytes
    const bool b = lane & 2;
    const uint32_t ps = b ? 0x6420u : 0x7531u;
    const uint32_t y0 = __shfl_xor_sync(kFull, __byte_perm(w[0], w[1], ps), 2);
    const uint32_t y1 = __shfl_xor_sync(kFull, __byte_perm(w[2], w[3], ps), 2);
    const uint32_t u0 = b ? 0x3514u : 0x5240u, u1 = b ? 0x3716u : 0x7260u;
    w[0] = __byte_perm(w[0], y0, u0);
    w[1] = __byte_perm(w[1], y0, u1);
    w[2] = __byte_perm(w[2], y1, u0);
    w[3] = __byte_perm(w[3], y1, u1);
  }
  {  // nibbles
    constexpr uint32_t kLo = 0x0F0F0F0Fu, kHi = 0xF0F0F0F0u;
    const bool b = lane & 1;
    const uint32_t x0 = b ? ((w[0] & kLo) | ((w[1] << 4) & kHi)) : (((w[0] >> 4) & kLo) | (w[1] & kHi));
    const uint32_t x1 = b ? ((w[2] & kLo) | ((w[3] << 4) & kHi)) : (((w[2] >> 4) & kLo) | (w[3] & kHi));
    const uint32_t y0 = __shfl_xor_sync(kFull, x0, 1);
    const uint32_t y1 = __shfl_xor_sync(kFull, x1, 1);
    if (b) {
      w[0] = (y0 & kLo) | (w[0] & kHi);
      w[1] = ((y0 >> 4) & kLo) | (w[1] & kHi);
      w[2] = (y1 & kLo) | (w[2] & kHi);
      w[3] = ((y1 >> 4) & kLo) | (w[3] & kHi);
    } else {
      w[0] = (w[0] & kLo) | ((y0 << 4) & kHi);
      w[1] = (w[1] & kLo) | (y0 & kHi);
      w[2] = (w[2] & kLo) | ((y1 << 4) & kHi);
      w[3] = (w[3] & kLo) | (y1 & kHi);
    }
  }
}

// 32 codes (byte j of w: values 2j low nibble, 2j + 1 high nibble) with one
// scale per pair of values (sc[j] = fp16 pair of the scales of values 2j and
// 2j + 1) into 16 fp16x2 words, as decode_group32 does with one scale.
__device__ __forceinline__ void decode_pairs32(const uint32_t (&w)[4], const uint32_t (&sc)[16], uint32_t (&out)[16]) {
  const __half2 mul = __halves2half2(__float2half_rn(1.0f), __float2half_rn(0.0625f));
  const __half2 add = __halves2half2(__float2half_rn(-1032.0f), __float2half_rn(-72.0f));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t rep = __byte_perm(w[i], 0u, 0x1111u * j);
      const uint32_t v = lop3_and_or(rep, 0x00F0000Fu, 0x64006400u);
      __half2 h = __hfma2(*reinterpret_cast<const __half2*>(&v), mul, add);
      h = __hmul2(h, *reinterpret_cast<const __half2*>(&sc[i * 4 + j]));
      out[i * 4 + j] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
}

// As decode_pairs32 for E2M1 codes (hardware conversion of each byte).
__device__ __forceinline__ void decode_pairs32_mxfp4(const uint32_t (&w)[4], const uint32_t (&sc)[16],
                                                     uint32_t (&out)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t v = e2m1x2_to_h2(w[i] >> (8 * j));
      __half2 h = __hmul2(*reinterpret_cast<const __half2*>(&v), *reinterpret_cast<const __half2*>(&sc[i * 4 + j]));
      out[i * 4 + j] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Row m, reduction group g of the LoRA stage that starts at column k0
// (columns [k0 + 32 g, k0 + 32 g + 32)) as 16 fp16 pairs: the LoRA B row of
// the weight row (rank contiguous), placed at the rank block of its
// projection.
template <int MODE>
__device__ __forceinline__ void lora_values(const GemmParams& p, int e, int fc, int m, int g, int k0,
                                            uint32_t (&w)[16]) {
  const int r = p.rank;
  const uint16_t* src = nullptr;
  int jlo = 0;
  if constexpr (MODE == kModeGateUp) {
    const bool up = m >= 64;
    const int f = fc + (m & 63);
    if (f < p.feat) src = (up ? p.lx1 : p.lx0) + (int64_t)e * p.lx_expert + (int64_t)f * p.lx_ld;
    jlo = up ? p.rpad : 0;
  } else {
    if (fc + m < p.feat) src = p.lx0 + (int64_t)e * p.lx_expert + (int64_t)(fc + m) * p.lx_ld;
  }
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    float v[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int jj = k0 + 32 * g + 2 * t + u - jlo;
      v[u] = (src != nullptr && jj >= 0 && jj < r) ? bf16_bits_to_float(__ldg(src + jj)) : 0.0f;
    }
    w[t] = pack_h2(v[0], v[1]);
  }
}

// MN-major: weight row m (feature fc + m), reduction group g of the LoRA
// stage that starts at column k0: the LoRA A column of the feature (rank rows
// [k0 + 32 g, k0 + 32 g + 32); gate/up^T stacks gate ranks at [0, r) and up
// ranks at [rpad, rpad + r)), as 16 fp16 pairs.
template <int MODE>
__device__ __forceinline__ void lora_values_mn(const GemmParams& p, int e, int fc, int m, int g, int k0,
                                               uint32_t (&w)[16]) {
  const int r = p.rank;
  const int f = fc + m;
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    float v[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int kr = k0 + 32 * g + 2 * t + u;
      const uint16_t* src = nullptr;
      if (f < p.feat) {
        if (kr < r)
          src = p.lx0 + (int64_t)e * p.lx_expert + (int64_t)kr * p.lx_ld + f;
        else if (MODE == kModeGateUpT && kr >= p.rpad && kr < p.rpad + r)
          src = p.lx1 + (int64_t)e * p.lx_expert + (int64_t)(kr - p.rpad) * p.lx_ld + f;
      }
      v[u] = src ? bf16_bits_to_float(__ldg(src)) : 0.0f;
    }
    w[t] = pack_h2(v[0], v[1]);
  }
}

template <int MODE, int FMT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_tm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ GemmMaps maps) {
  static_assert(kPSub<MODE> % kGroup == 0, "a hand-off group lies within one packed slot");
  const CUtensorMap& tq0 = maps.q0;
  const CUtensorMap& tq1 = maps.q1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem + kOffB;
  uint8_t* sP = smem + kOffP;
  uint8_t* sS = smem + kOffS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* p_full = bars;                   // local: this CTA's packed slot and its scales landed
  uint64_t* p_empty = p_full + kMaxStagesP;  // local: this CTA's decoders read them
  uint64_t* a_full = p_empty + kMaxStagesP;  // leader [kAGroups]: the group's A (both CTAs) and B are ready
  uint64_t* a_empty = a_full + kAStages;     // both [kAGroups]: the pair MMA finished reading the group's A
  uint64_t* b_full = a_empty + kAStages;     // leader: both CTAs' B halves landed
  uint64_t* b_empty = b_full + kStagesB;     // both: the pair MMA finished reading B
  uint64_t* s_full = b_empty + kStagesB;     // local: a stage's scales landed
  uint64_t* s_empty = s_full + kStagesS;     // local: this CTA's decoders read them
  uint64_t* acc_full = s_empty + kStagesS;   // both [2]: accumulator complete
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
    for (int i = 0; i < kStagesP<MODE>; ++i) {
      mbar_init(&p_full[i], 1 + 32);  // the TMA producer's arrival (with its bytes) + the scale loader's lanes
      mbar_init(&p_empty[i], kDecWarps);
    }
    for (int i = 0; i < kAGroups; ++i) {
      mbar_init(&a_full[i], 2 * kDecWarps);
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
  constexpr int PS = kPSub<MODE>;                   // reduction stages per packed slot
  const int n_slots = (n_main + PS - 1) / PS;
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
      const int rot = k_rotation(tile % n_rowblk, n_rowblk, n_slots);
      for (int j0 = 0; j0 < n_slots; ++j0) {
        const int j = rotated(j0, rot, n_slots);
        if (!wait_warp(&p_empty[ring.stage], ring.phase ^ 1u, abort_flag, status, lim)) goto drain_p;
        if (lane == 0) {
          uint64_t* bar = &p_full[ring.stage];
          uint8_t* dst = sP + ring.stage * kPBytes<MODE>;
          // every box is counted in full, also where it reaches past the
          // tensor (zero-filled rows or reduction columns of a partial slot)
          mbar_expect_tx(bar, kPBytes<MODE>);
          if constexpr (MODE == kModeGateUp) {
            // 64 rows x 128 bytes (4 stages) of gate, then of up
            tma_load_3d(dst, &tq0, bar, j * 128, fc, e);
            tma_load_3d(dst + kPBytes<MODE> / 2, &tq1, bar, j * 128, fc, e);
          } else if constexpr (MODE == kModeDown) {
            tma_load_3d(dst, &tq0, bar, j * 128, fc, e);
            tma_load_3d(dst + kPBytes<MODE> / 2, &tq0, bar, j * 128, fc + 64, e);
          } else {
            // two boxes of 64 stored rows x 64 bytes (this CTA's 128 weight
            // rows), one per stage: a stage never straddles gate and up
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int k0 = (2 * j + u) * kBlockK;
              if (MODE == kModeDownT || k0 < p.stored_rows)
                tma_load_3d(dst + 4096 * u, &tq0, bar, fc / 2, k0, e);
              else
                tma_load_3d(dst + 4096 * u, &tq1, bar, fc / 2, k0 - p.stored_rows, e);
            }
          }
        }
        __syncwarp();
        ring.advance(kStagesP<MODE>);
        ++issued;
      }
    }
    goto done;
  drain_p:
    if (lane == 0) drain_ring(p_full, ring, issued, kStagesP<MODE>);
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------- scale loader
    Ring ring;
    for (int tile = tile0; tile < n_tiles; tile += tile_step) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int fc = cta_f0<MODE>(tile % n_rowblk, cta);
      const int rot = k_rotation(tile % n_rowblk, n_rowblk, n_slots);
      for (int j0 = 0; j0 < n_slots; ++j0) {
        const int j = rotated(j0, rot, n_slots);
        if (!wait_warp(&p_empty[ring.stage], ring.phase ^ 1u, abort_flag, status, lim)) goto drain_s;
        if constexpr (kAMnMajor<MODE>)
          load_slot_scales_mn<MODE, FMT>(p, tt.x, fc, j, n_main, lane, sS + ring.stage * kSSlotBytes);
        else
          load_slot_scales<MODE, FMT>(p, tt.x, fc, j, n_main, lane, sS + ring.stage * kSSlotBytes);
        cp_async_arrive_noinc(&p_full[ring.stage]);
        ring.advance(kStagesP<MODE>);
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
      const int rot = k_rotation(tile % n_rowblk, n_rowblk, n_slots);
      // the item's stage order: slot-rotated main stages, then the LoRA stages
      for (int j0 = 0; j0 <= n_slots; ++j0) {
        const int j = j0 < n_slots ? rotated(j0, rot, n_slots) : 0;
        const int nsub = j0 < n_slots ? min(PS, n_main - PS * j) : n_lora;
        for (int u = 0; u < nsub; ++u) {
        const int s = j0 < n_slots ? PS * j + u : n_main + u;
        if (!wait_warp(&b_empty[ring.stage], ring.phase ^ 1u, abort_flag, status, lim)) goto drain_b;
        if (lane == 0) {
          uint8_t* dst = sB + ring.stage * kBBytes;
          const uint32_t bar = cluster_addr(&b_full[ring.stage], 0);
          if (cta == 0) mbar_expect_tx(&b_full[ring.stage], 2 * nb * 128);
          int row = 0;
          for (int lvl = 2; lvl >= 0; --lvl) {
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
    // stage and then the group's A stages by commits.
    if (cta == 0) {
      if (lane == 0) {
        Ring rg, rbr;
        int it = 0;
        bool aborted = false;
        const int ksteps_x = kext_steps<MODE>(p.rpad);
        // shared-memory descriptor of B stage 0; stage s adds s kBBytes, a
        // 16-wide reduction step adds 32 bytes (both in 16-byte units)
        const uint64_t bdesc0 = make_sdesc_sw128(smem_u32(sB), 16, 1024);
        const uint32_t a_col0 = tmem + kACol0;
        for (int tile = tile0; tile < n_tiles; tile += tile_step, ++it) {
          const int4 tt = p.tok_tiles[tile / n_rowblk];
          const uint32_t idesc = make_idesc_f16((uint32_t)pair_n(tt.z), false, false, 256);
          const int ab = it & 1;
          const int rot = k_rotation(tile % n_rowblk, n_rowblk, n_slots);
          if (!wait_issuer(&acc_empty[ab], ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag, status, lim)) {
            aborted = true;
            goto mma_out;
          }
          tc_fence_after();
          {
            const uint32_t d_tmem = tmem + (uint32_t)(ab * kAccCols);
            uint32_t acc = 0u;  // the item's first UMMA overwrites the accumulator
            // the item's stages: slot-rotated main stages in groups within each
            // slot, then the LoRA stage as a group of its own
            for (int j0 = 0; j0 <= n_slots; ++j0) {
              const bool lora = j0 == n_slots;
              const int nsub = lora ? n_lora : min(PS, n_main - PS * rotated(j0, rot, n_slots));
              for (int u = 0; u < nsub; u += kGroup) {
                const int nb = min(kGroup, nsub - u);
                if (!wait_issuer(&a_full[rg.stage], rg.phase, abort_flag, status, lim)) {
                  aborted = true;
                  goto mma_out;
                }
                tc_fence_after();
                for (int b = 0; b < nb; ++b) {
                  const uint32_t a_tm = a_col0 + (uint32_t)(32 * (kGroup * rg.stage + b));
                  const uint64_t bd = bdesc0 + (uint64_t)((rbr.stage * kBBytes) >> 4);
                  if (!lora) {
#pragma unroll
                    for (int kk = 0; kk < kBlockK / 16; ++kk) {
                      umma_f16_pair_ts(d_tmem, a_tm + (uint32_t)(8 * kk), bd + (uint64_t)(2 * kk), idesc, acc);
                      acc = 1u;
                    }
                  } else {
                    const int ks = min(kBlockK / 16, ksteps_x - (kBlockK / 16) * (u + b));
                    for (int kk = 0; kk < ks; ++kk) {
                      umma_f16_pair_ts(d_tmem, a_tm + (uint32_t)(8 * kk), bd + (uint64_t)(2 * kk), idesc, acc);
                      acc = 1u;
                    }
                  }
                  umma_commit_pair(&b_empty[rbr.stage], kPairMask);
                  rbr.advance(kStagesB);
                }
                umma_commit_pair(&a_empty[rg.stage], kPairMask);
                rg.advance(kAGroups);
              }
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
      const int n_rows = tt.z;
      const int p0 = tt.y;
      const int ab = it & 1;
      // the four epilogue warps leave together or not at all: a warp that
      // went on alone would wait forever at the gate/up exchange barrier
      const bool ok = wait_warp(&acc_full[ab], (uint32_t)(it >> 1) & 1u, abort_flag, status, lim);
      if (!named_bar_and(3, 128, ok)) goto done;
      tc_fence_after();
      const uint32_t d_tmem = tmem + lane_base + (uint32_t)(ab * kAccCols);
      for (int c0 = 0; c0 < n_rows; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(d_tmem + (uint32_t)c0, v);
        if constexpr (MODE == kModeGateUp) {
          // lanes 0-63: gate features fc + m; lanes 64-127: up features fc + m - 64
          float* xch = epi + (q & 1) * 32 * 33;
          if (q >= 2) {
#pragma unroll
            for (int c = 0; c < 32; ++c) xch[lane * 33 + c] = __uint_as_float(v[c]);
          }
          named_bar_sync(1 + (q & 1), 64);
          const int i = fc + m;
          if (q < 2 && i < p.feat) {
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
          // down: Yw = w y; gate/up^T: dx rows as they are
          const int f = fc + m;
          float wl = 1.0f;
          if constexpr (MODE == kModeDown) wl = __ldg(p.w_perm + p0 + min(c0 + lane, n_rows - 1));
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int n = c0 + c;
            const float w = __shfl_sync(0xffffffffu, wl, c);
            if (n < n_rows && f < p.feat) p.out_a[(int64_t)(p0 + n) * p.ld_out + f] = w * __uint_as_float(v[c]);
          }
        } else {  // kModeDownT
          // dh = w acc; SwiGLU' with the clamp masks decided on the saved fp32
          // G and U; dRoute partial = sum over this CTA's features of acc h
          // (h from the saved G, U), reduced over the 128 rows through shared
          // memory. The saved G/U of 4 tokens are loaded together ahead of use.
          const float L = p.limit;
          float* red = epi + q * 32 * 33;
          float* red2 = epi + 4 * 32 * 33;
          bool overflow = false;
          const int i = fc + m;
          const bool live = i < p.feat;
          const float wl = __ldg(p.w_perm + p0 + min(c0 + lane, n_rows - 1));
#pragma unroll
          for (int cb = 0; cb < 32; cb += 4) {
            float gq[4], uq[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int64_t row = p0 + min(c0 + cb + c, n_rows - 1);
              gq[c] = live ? __ldg(p.in_g + row * p.ld_out + i) : 0.f;
              uq[c] = live ? __ldg(p.in_u + row * p.ld_out + i) : 0.f;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int n = c0 + cb + c;
              const float w = __shfl_sync(0xffffffffu, wl, cb + c);
              float pr = 0.f;
              if (live && n < n_rows) {
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
    const int q = warp & 3;
    const int g = (warp - kDecWarp0) >> 2;  // reduction group of each stage
    const int m = 32 * q + lane;            // weight row (TMEM lane)
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    // Packed slot layout. K-major: row m holds the 4 stages' 128 bytes with
    // 128-byte swizzling (16-byte chunk c of row m at chunk c ^ (m & 7)); the
    // thread reads chunk 2u + g of sub-stage u, and every 8 lanes hit all bank
    // groups. MN-major: stage u's 64 stored rows of 64 bytes with 64-byte
    // swizzling (chunk q of stored row r at q ^ ((r >> 1) & 3)); lane i reads
    // stored row 32 g + i, the chunk of the warp's 32 weight rows.
    auto p_off = [&](int u) -> uint32_t {
      if constexpr (kAMnMajor<MODE>) {
        const int kr = 32 * g + lane;
        return (uint32_t)(4096 * u + kr * 64 + 16 * (q ^ ((kr >> 1) & 3)));
      } else {
        return (uint32_t)(m * 128 + 16 * ((2 * u + g) ^ (m & 7)));
      }
    };
    // scale of this thread's group: K-major [128 rows][8] (2 per stage),
    // MN-major [128 stored rows][4 groups]
    auto s_off = [&](int u) -> uint32_t {
      if constexpr (FMT == RAWINT4_FORMAT_MXFP4) {  // scale bytes
        if constexpr (kAMnMajor<MODE>)
          return (uint32_t)((64 * u + 32 * g + lane) * 4 + q);
        else
          return (uint32_t)(m * 8 + 2 * u + g);
      } else if constexpr (kAMnMajor<MODE>) {
        return (uint32_t)((64 * u + 32 * g + lane) * 8 + 2 * q);
      } else {
        return (uint32_t)(m * 16 + (2 * u + g) * 2);
      }
    };
    uint32_t* tab = reinterpret_cast<uint32_t*>(smem + kOffScaleTab) + 32 * (warp - kDecWarp0);
    Ring rg, rp, rs, rbd;
    // the leader's first decoder warp also waits for each group's B stages
    const bool b_watch = cta == 0 && warp == kDecWarp0;
    // Decodes sub-stage u of packed slot rp / scale slot rs into w; table `tb`
    // holds the MN-major scale pairs.
    auto decode_stage = [&](const Ring& rs_, const Ring& rp_, int u, uint32_t* tb, uint32_t (&w)[16]) {
      const uint8_t* sptr = sS + rs_.stage * kSSlotBytes + s_off(u);
      // fp16 bits of this thread's group scale
      uint32_t hb;
      if constexpr (FMT == RAWINT4_FORMAT_MXFP4) {
        hb = ue8m0_to_h(*sptr);
      } else {
        const __half hs = __float2half_rn(bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(sptr)));
        hb = (uint32_t)(*reinterpret_cast<const uint16_t*>(&hs));
      }
      const uint4 q4 = *reinterpret_cast<const uint4*>(sP + rp_.stage * kPBytes<MODE> + p_off(u));
      if constexpr (kAMnMajor<MODE>) {
        // every stored row has its own scale: pair them up (lane 2t holds
        // the scales of values 2t and 2t + 1) through a per-warp table
        const uint32_t nb = __shfl_down_sync(0xffffffffu, hb, 1);
        if ((lane & 1) == 0) tb[lane >> 1] = hb | (nb << 16);
        __syncwarp();
        uint32_t sp2[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 t4 = *reinterpret_cast<const uint4*>(tb + 4 * j);
          sp2[4 * j] = t4.x;
          sp2[4 * j + 1] = t4.y;
          sp2[4 * j + 2] = t4.z;
          sp2[4 * j + 3] = t4.w;
        }
        uint32_t nib[4] = {q4.x, q4.y, q4.z, q4.w};
        transpose_nibbles(nib, lane);
        if constexpr (FMT == RAWINT4_FORMAT_MXFP4)
          decode_pairs32_mxfp4(nib, sp2, w);
        else
          decode_pairs32(nib, sp2, w);
      } else {
        const uint32_t h2 = hb | (hb << 16);
        if constexpr (FMT == RAWINT4_FORMAT_MXFP4)
          decode_group32_mxfp4(q4, *reinterpret_cast<const __half2*>(&h2), w);
        else
          decode_group32(q4, *reinterpret_cast<const __half2*>(&h2), w);
      }
    };
    for (int tile = tile0; tile < n_tiles; tile += tile_step) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int fc = cta_f0<MODE>(tile % n_rowblk, cta);
      const int e = tt.x;
      const int rot = k_rotation(tile % n_rowblk, n_rowblk, n_slots);
      uint32_t lora_w[16];
      if constexpr (kAMnMajor<MODE>)
        lora_values_mn<MODE>(p, e, fc, m, g, 0, lora_w);
      else
        lora_values<MODE>(p, e, fc, m, g, 0, lora_w);
      for (int j0 = 0; j0 < n_slots; ++j0) {
        const int j = rotated(j0, rot, n_slots);
        const int nsub = min(PS, n_main - PS * j);
        if (!wait_warp(&p_full[rp.stage], rp.phase, abort_flag, status, lim)) goto done;
        // the slot's stages a group at a time: decoded into registers first
        // (that needs only the packed and scale slots), then one wait for the
        // group's A stages, the tensor-memory stores, one store completion,
        // fence and arrival: only the stores sit on the chain from the MMA's
        // release of the A stages to their next fill
        for (int u = 0; u < nsub; u += kGroup) {
          const int nb = min(kGroup, nsub - u);
          // two stages at a time (decoded words of more would not stay in
          // registers); the group's A stages are waited for once
          for (int h = 0; h < nb; h += 2) {
            uint32_t w[2][16];
#pragma unroll
            for (int b = 0; b < 2; ++b)
              if (h + b < nb) decode_stage(rs, rp, u + h + b, tab + 16 * b, w[b]);
            if (h + 2 >= nb && u + kGroup >= nsub) {
              // the slot's last stages decoded: release the packed and scale
              // slot once every lane has used the values it loaded (the empty
              // asm makes the decoded words, which depend on every loaded byte
              // and scale, inputs, so the loads have returned)
#pragma unroll
              for (int b = 0; b < 2; ++b)
                if (h + b < nb) asm volatile("" ::"r"(w[b][0]), "r"(w[b][15]) : "memory");
              __syncwarp();
              if (lane == 0) mbar_arrive(&p_empty[rp.stage]);
            }
            if (h == 0)
              if (!wait_warp(&a_empty[rg.stage], rg.phase ^ 1u, abort_flag, status, lim)) goto done;
#pragma unroll
            for (int b = 0; b < 2; ++b)
              if (h + b < nb)
                tmem_st16(tmem + lane_base + kACol0 + (uint32_t)(32 * (kGroup * rg.stage + h + b) + 16 * g), w[b]);
          }
          tmem_wait_st();
          tc_fence_before();
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
        rp.advance(kStagesP<MODE>);
        rs.advance(kStagesP<MODE>);
      }
      // the LoRA stages, a group of their own (the second one, for a rank
      // above 32, loaded here)
      uint32_t lora_w1[16];
      if (n_lora > 1) {
        if constexpr (kAMnMajor<MODE>)
          lora_values_mn<MODE>(p, e, fc, m, g, kBlockK, lora_w1);
        else
          lora_values<MODE>(p, e, fc, m, g, kBlockK, lora_w1);
      }
      if (!wait_warp(&a_empty[rg.stage], rg.phase ^ 1u, abort_flag, status, lim)) goto done;
      tmem_st16(tmem + lane_base + kACol0 + (uint32_t)(32 * kGroup * rg.stage + 16 * g), lora_w);
      if (n_lora > 1) tmem_st16(tmem + lane_base + kACol0 + (uint32_t)(32 * kGroup * rg.stage + 32 + 16 * g), lora_w1);
      tmem_wait_st();
      tc_fence_before();
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
    if (cudaFuncSetAttribute(gemm_tm_kernel<MODE, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
        cudaSuccess)
      return false;
    device_flag_set(done, dev);
  }
  return true;
}

template <int MODE, int FMT>
cudaError_t launch_mode(const GemmParams& p, const GemmMaps& m, int clusters, cudaStream_t stream) {
  if (!set_smem_attr<MODE, FMT>()) return cudaErrorInvalidValue;
  gemm_tm_kernel<MODE, FMT><<<2 * clusters, kThreads, kSmemBytes, stream>>>(p, m);
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
  if (cudaOccupancyMaxActiveClusters(&n, gemm_tm_kernel<MODE, FMT>, &cfg) != cudaSuccess) return 0;
  return n;
}

}  // namespace R4_TM_NS

cudaError_t R4_TM_LAUNCH(int mode, int fmt, const GemmParams& p, const GemmMaps& maps, int clusters,
                           cudaStream_t stream) {
  [[maybe_unused]] constexpr int R = RAWINT4_FORMAT_RAWINT4, X = RAWINT4_FORMAT_MXFP4;
  switch (mode * 2 + (fmt == X ? 1 : 0)) {
    case kModeGateUp * 2: return R4_TM_NS::launch_mode<kModeGateUp, R>(p, maps, clusters, stream);
    case kModeDown * 2: return R4_TM_NS::launch_mode<kModeDown, R>(p, maps, clusters, stream);
    case kModeGateUp * 2 + 1: return R4_TM_NS::launch_mode<kModeGateUp, X>(p, maps, clusters, stream);
    case kModeDown * 2 + 1: return R4_TM_NS::launch_mode<kModeDown, X>(p, maps, clusters, stream);
#if !R4_TM_NARROW  // the narrow configuration serves the forward modes only
    case kModeDownT * 2: return R4_TM_NS::launch_mode<kModeDownT, R>(p, maps, clusters, stream);
    case kModeDownT * 2 + 1: return R4_TM_NS::launch_mode<kModeDownT, X>(p, maps, clusters, stream);
    case kModeGateUpT * 2: return R4_TM_NS::launch_mode<kModeGateUpT, R>(p, maps, clusters, stream);
    case kModeGateUpT * 2 + 1: return R4_TM_NS::launch_mode<kModeGateUpT, X>(p, maps, clusters, stream);
#endif
    default: return cudaErrorInvalidValue;
  }
}

int R4_TM_MAXCL(int mode, int fmt) {
  [[maybe_unused]] constexpr int R = RAWINT4_FORMAT_RAWINT4, X = RAWINT4_FORMAT_MXFP4;
  switch (mode * 2 + (fmt == X ? 1 : 0)) {
    case kModeGateUp * 2: return R4_TM_NS::max_clusters_mode<kModeGateUp, R>();
    case kModeDown * 2: return R4_TM_NS::max_clusters_mode<kModeDown, R>();
    case kModeGateUp * 2 + 1: return R4_TM_NS::max_clusters_mode<kModeGateUp, X>();
    case kModeDown * 2 + 1: return R4_TM_NS::max_clusters_mode<kModeDown, X>();
#if !R4_TM_NARROW  // the narrow configuration serves the forward modes only
    case kModeDownT * 2: return R4_TM_NS::max_clusters_mode<kModeDownT, R>();
    case kModeDownT * 2 + 1: return R4_TM_NS::max_clusters_mode<kModeDownT, X>();
    case kModeGateUpT * 2: return R4_TM_NS::max_clusters_mode<kModeGateUpT, R>();
    case kModeGateUpT * 2 + 1: return R4_TM_NS::max_clusters_mode<kModeGateUpT, X>();
#endif
    default: return 0;
  }
}

}  // namespace r4
