// Dequant-fused grouped GEMMs of the routed RAWINT4 MoE-LoRA layer on
// sm_100a tensor cores (tcgen05, TMEM accumulators, TMA-fed operands), one
// CTA per SM: gate/up (forward), down (forward) and gate/up^T (backward dX).
// The down^T GEMM runs on CTA pairs (gemm_pair.cu).
//
// One persistent CTA per SM walks (token tile, feature block) work items. A
// token tile is up to 256 permuted rows of one expert; a feature block is 256
// weight rows (gate/up: the same 128 features of gate and of up). Each
// K-stage issues two M=128 UMMAs (weight rows 0-127 and 128-255) on the same
// B tile, so every activation tile read from L2 feeds 256 weight rows.
// Warp roles:
//   warp 0      TMA producer of packed int4 weight tiles   (ring of kStagesP)
//   warp 3      loader of the group scales (cp.async, ring of kStagesS)
//   warp 2      TMA producer of B tiles (activations)      (ring of kStagesB)
//   warps 8-15  decoders: int4 -> fp16 into the UMMA A layout (ring of kStagesA)
//   warp 1      UMMA issuer (one elected lane) and TMEM owner
//   warps 4-7   epilogue: TMEM -> registers -> fused math -> global
// TMEM (512 columns) holds two halves of 256 columns. A tile of at most 128
// tokens keeps both of its accumulators in one half, so consecutive narrow
// items alternate halves and the epilogue of one overlaps the MMAs of the
// next; a wider tile takes both halves.
//
// The LoRA side product of each projection runs as one extra 64-wide
// reduction stage in the same accumulators: its A operand is the LoRA tensor
// of the expert (loaded into registers at the start of the item and stored
// by the decoders), its B operand the precomputed c-scaled rank-r side matrix.
//
// The gate/up^T mode reads the packed base along its stored output dimension
// (transpose-free dX, rawint4_sft_reference.py transpose_free_rawint4_dx):
// the decoders write the same packed bytes into an MN-major A tile, so no
// transposed or dense copy of any base weight ever exists.
#include "gemm.cuh"

namespace r4 {

namespace {

constexpr int kRowsM = 256;        // weight rows per work item (two UMMAs of M = 128)
constexpr int kStagesA = 2;        // decoded FP16 A tiles (32 KB each)
constexpr int kStagesB = 3;        // TMA-loaded B tiles (32 KB each)
constexpr int kStagesP = 4;        // TMA-loaded packed int4 tiles (8 KB each)
constexpr int kStagesS = 8;        // group scales of one stage (1 KB each)
constexpr int kThreads = 512;      // 16 warps
constexpr int kEpiWarp0 = 4;       // warps 4..7: epilogue
constexpr int kDecWarp0 = 8;       // warps 8..15: decoders
constexpr int kDecThreads = 256;

constexpr int kABytes = kRowsM * kBlockK * 2;  // 32 KB
constexpr int kAHalf = kABytes / 2;            // weight rows 128-255 start here (both layouts)
constexpr int kBBytes = 256 * kBlockK * 2;     // 32 KB
constexpr int kPBytes = kRowsM * kBlockK / 2;  // 8 KB
constexpr int kOffA = 0;
constexpr int kOffB = kOffA + kStagesA * kABytes;
constexpr int kOffP = kOffB + kStagesB * kBBytes;
constexpr int kSBytes = 1024;
constexpr int kOffS = kOffP + kStagesP * kPBytes;
constexpr int kOffBar = kOffS + kStagesS * kSBytes;
constexpr int kNumBars = 2 * kStagesP + 2 * kStagesA + 2 * kStagesB + 2 * kStagesS + 4;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

template <int MODE>
constexpr bool kAMnMajor = (MODE == kModeDownT || MODE == kModeGateUpT);

// 16-wide MMA steps of the LoRA stage: one rank block (padded to rpad) per
// projection, two for the gate/up pair.
template <int MODE>
__device__ __forceinline__ int kext_steps(int rpad) {
  const int kext = (MODE == kModeGateUp || MODE == kModeGateUpT) ? 2 * rpad : rpad;
  return kext / 16;
}

// First output feature of block rb.
template <int MODE>
__device__ __forceinline__ int block_f0(int rb) {
  return MODE == kModeGateUp ? rb * 128 : rb * 256;
}

// Whether block rb has its second 128-row half (always, for gate/up).
template <int MODE>
__device__ __forceinline__ bool block_two(const GemmParams& p, int rb) {
  return MODE == kModeGateUp || block_f0<MODE>(rb) + 128 < p.feat;
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a
// 128B-swizzled block whose rows are 128 bytes and whose 8-row atoms are
// 1024 bytes apart.
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4));
}

// MN-major decode: thread dt owns K row kr of the 64 features [64 qq, +64),
// which form one 8 KB MN block of the A tile. Each group of 8 consecutive
// lanes takes 8 consecutive K rows of one block, so its 16-byte stores (and
// its reads of the swizzled packed tile) hit 8 distinct bank groups.
__device__ __forceinline__ int mn_kr(int dt) { return 8 * (dt >> 5) + (dt & 7); }
__device__ __forceinline__ int mn_qq(int dt) { return (dt >> 3) & 3; }

// Offset of output chunk c (0..7, 8 fp16 each) of decoder thread dt in the A
// tile. K-major: thread dt owns weight row dt (all 64 K of the stage).
template <int MODE>
__device__ __forceinline__ uint32_t a_chunk_off(int dt, int c) {
  if constexpr (!kAMnMajor<MODE>) {
    return sw128_off(dt, c);
  } else {
    return (uint32_t)(mn_qq(dt) * 8192) + sw128_off(mn_kr(dt), c);
  }
}

// The 32 packed bytes decoder thread dt decodes at one stage: two groups of
// 32 weights (q0 first). K-major tiles hold row dt at dt * 32, and the two
// halves are read in an order that spreads each 8-lane group over all bank
// groups. MN-major tiles are loaded with 128-byte swizzling.
template <int MODE>
__device__ __forceinline__ void packed_pair(const uint8_t* P, int dt, uint4& q0, uint4& q1) {
  if constexpr (!kAMnMajor<MODE>) {
    const int sw = (dt >> 2) & 1;
    const uint4 a = *reinterpret_cast<const uint4*>(P + dt * 32 + sw * 16);
    const uint4 b = *reinterpret_cast<const uint4*>(P + dt * 32 + (sw ^ 1) * 16);
    q0 = sw ? b : a;
    q1 = sw ? a : b;
  } else {
    const int kr = mn_kr(dt), qq = mn_qq(dt);
    q0 = *reinterpret_cast<const uint4*>(P + sw128_off(kr, 2 * qq));
    q1 = *reinterpret_cast<const uint4*>(P + sw128_off(kr, 2 * qq + 1));
  }
}

// The two group scales decoder thread dt needs at K-stage s, as bf16 bits
// (first group low, second high); 0 past the mode's features.
template <int MODE>
__device__ __forceinline__ uint32_t load_scales(const GemmParams& p, int e, int rb, int s, int dt) {
  const int f0 = block_f0<MODE>(rb);
  const uint16_t* sp = p.s0;
  int64_t idx;
  if constexpr (MODE == kModeGateUp) {
    sp = dt < 128 ? p.s0 : p.s1;
    idx = (int64_t)(f0 + (dt & 127)) * p.s_row + 2 * s;
  } else if constexpr (MODE == kModeDown) {
    if (f0 + dt >= p.feat) return 0u;
    idx = (int64_t)(f0 + dt) * p.s_row + 2 * s;
  } else {
    const int kr = mn_kr(dt), qq = mn_qq(dt);
    if (f0 + 64 * qq >= p.feat) return 0u;
    int row = s * kBlockK + kr;
    if (MODE == kModeGateUpT && row >= p.stored_rows) {
      row -= p.stored_rows;
      sp = p.s1;
    }
    idx = (int64_t)row * p.s_row + (f0 + 64 * qq) / 32;
  }
  sp += (int64_t)e * p.s_expert + idx;
  return (uint32_t)__ldg(sp) | ((uint32_t)__ldg(sp + 1) << 16);
}

template <int MODE>
__device__ __forceinline__ uint32_t scale_off(int dt) {
  if constexpr (!kAMnMajor<MODE>) return (uint32_t)(dt * 4);
  else return (uint32_t)(mn_kr(dt) * 16 + mn_qq(dt) * 4);
}
template <int MODE>
__device__ __forceinline__ void load_stage_scales(const GemmParams& p, int e, int rb, int s, int ln, uint8_t* S) {
  const int f0 = block_f0<MODE>(rb);
  if constexpr (!kAMnMajor<MODE>) {
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int r = ln + 32 * t;
      const uint16_t* sp = p.s0;
      int f;
      if constexpr (MODE == kModeGateUp) {
        sp = r < 128 ? p.s0 : p.s1;
        f = f0 + (r & 127);
      } else {
        f = f0 + r;
      }
      const bool ok = f < p.feat;
      const uint16_t* src = ok ? sp + (int64_t)e * p.s_expert + (int64_t)f * p.s_row + 2 * s : p.s0;
      cp_async_4(S + r * 4, src, ok ? 4u : 0u);
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
      const uint16_t* src = sp + (int64_t)e * p.s_expert + (int64_t)row * p.s_row + f0 / 32;
      const bool ok0 = f0 < p.feat, ok1 = f0 + 128 < p.feat;
      cp_async_8(S + kr * 16, ok0 ? src : p.s0, ok0 ? 8u : 0u);
      cp_async_8(S + kr * 16 + 8, ok1 ? src + 4 : p.s0, ok1 ? 8u : 0u);
    }
  }
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// This thread's 64 values of the A tile of the LoRA reduction stage, as 32
// fp16 pairs in decode order (chunk c = words 4c..4c+3, see a_chunk_off).
// Loaded at the start of a work item, long before the stage is stored: a
// decoder warp that stored operand data right after long-latency global loads
// at the tail of a work item produced corrupted rows in earlier builds, and
// the early load also takes that latency off the critical path.
template <int MODE>
__device__ __forceinline__ void lora_values(const GemmParams& p, int e, int rb, int dt, uint32_t (&w)[32]) {
  const int r = p.rank;
  const int f0 = block_f0<MODE>(rb);
  if constexpr (!kAMnMajor<MODE>) {
    // A[m, j], j in [0, 64): LoRA B rows (rank contiguous)
    const uint16_t* src = nullptr;
    int jlo = 0;  // first reduction column holding this row's values
    if constexpr (MODE == kModeGateUp) {
      // rows past the features (a partial last block) read nothing
      if (f0 + (dt & 127) < p.feat)
        src = (dt < 128 ? p.lx0 : p.lx1) + (int64_t)e * p.lx_expert + (int64_t)(f0 + (dt & 127)) * p.lx_ld;
      jlo = dt < 128 ? 0 : p.rpad;
    } else {
      if (f0 + dt < p.feat) src = p.lx0 + (int64_t)e * p.lx_expert + (int64_t)(f0 + dt) * p.lx_ld;
    }
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      float v[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int jj = 2 * t + u - jlo;
        v[u] = (src != nullptr && jj >= 0 && jj < r) ? bf16_bits_to_float(__ldg(src + jj)) : 0.0f;
      }
      w[t] = pack_h2(v[0], v[1]);
    }
  } else {
    // A[m, kr], m in [64 qq, 64 qq + 64): LoRA A rows (feature contiguous)
    const int kr = mn_kr(dt), qq = mn_qq(dt);
    const uint16_t* src = nullptr;
    if (f0 + 64 * qq < p.feat) {
      if (kr < r)
        src = p.lx0 + (int64_t)e * p.lx_expert + (int64_t)kr * p.lx_ld + f0 + 64 * qq;
      else if (MODE == kModeGateUpT && kr >= p.rpad && kr < p.rpad + r)
        src = p.lx1 + (int64_t)e * p.lx_expert + (int64_t)(kr - p.rpad) * p.lx_ld + f0 + 64 * qq;
    }
    if (src != nullptr) {
      const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 b = __ldg(s4 + c);
        const uint32_t in[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int t = 0; t < 4; ++t)
          w[4 * c + t] = pack_h2(__uint_as_float(in[t] << 16), __uint_as_float(in[t] & 0xFFFF0000u));
      }
    } else {
#pragma unroll
      for (int t = 0; t < 32; ++t) w[t] = 0u;
    }
  }
}

// Which TMEM half (or both) an item's accumulators occupy. The MMA issuer and
// the epilogue step identical copies through the same item sequence.
struct AccTrack {
  uint32_t uses[2] = {0u, 0u};  // completed items per half (phase parity source)
  int next = 0;                 // half the next narrow item takes
  __device__ __forceinline__ void retire(bool wide) {
    if (wide) {
      ++uses[0];
      ++uses[1];
      next = 0;
    } else {
      ++uses[next];
      next ^= 1;
    }
  }
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ GemmMaps maps) {
  static_assert(MODE != kModeDownT, "down^T runs on the CTA-pair kernel (gemm_pair.cu)");
  const CUtensorMap& tq0 = maps.q0;
  const CUtensorMap& tq1 = maps.q1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + kOffA;
  uint8_t* sB = smem + kOffB;
  uint8_t* sP = smem + kOffP;
  uint8_t* sS = smem + kOffS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* p_full = bars;
  uint64_t* p_empty = p_full + kStagesP;
  uint64_t* a_full = p_empty + kStagesP;
  uint64_t* a_empty = a_full + kStagesA;
  uint64_t* b_full = a_empty + kStagesA;
  uint64_t* b_empty = b_full + kStagesB;
  uint64_t* s_full = b_empty + kStagesB;
  uint64_t* s_empty = s_full + kStagesS;
  uint64_t* acc_full = s_empty + kStagesS;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagesP; ++i) {
      mbar_init(&p_full[i], 1);
      mbar_init(&p_empty[i], kDecThreads / 32);
    }
    for (int i = 0; i < kStagesA; ++i) {
      mbar_init(&a_full[i], kDecThreads / 32);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < kStagesB; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < kStagesS; ++i) {
      mbar_init(&s_full[i], 32);
      mbar_init(&s_empty[i], kDecThreads / 32);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
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
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int n_rowblk = p.n_rowblk;
  const int n_tiles = (p.need_saved && p.hdr->saved != 1u) ? 0 : p.hdr->n_tok_tiles * n_rowblk;
  const int n_main = p.n_main;
  uint32_t* status = p.status;

  if (warp == 0) {
    // ------------------------------------------------ packed weight producer
    Ring ring;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int f0 = block_f0<MODE>(tile % n_rowblk);
      const int e = tt.x;
      for (int s = 0; s < n_main; ++s) {
        if (!wait_all(&p_empty[ring.stage], ring.phase ^ 1u, abort_flag, status)) goto done;
        if (lane == 0) {
          uint64_t* bar = &p_full[ring.stage];
          uint8_t* dst = sP + ring.stage * kPBytes;
          // every box is counted in full, also where it reaches past the
          // tensor (zero-filled rows of a half block)
          mbar_expect_tx(bar, kPBytes);
          if constexpr (MODE == kModeGateUp) {
            tma_load_3d(dst, &tq0, bar, s * (kBlockK / 2), f0, e);
            tma_load_3d(dst + kPBytes / 2, &tq1, bar, s * (kBlockK / 2), f0, e);
          } else if constexpr (MODE == kModeDown) {
            tma_load_3d(dst, &tq0, bar, s * (kBlockK / 2), f0, e);
          } else if constexpr (MODE == kModeDownT) {
            tma_load_3d(dst, &tq0, bar, f0 / 2, s * kBlockK, e);
          } else {
            const int k0 = s * kBlockK;
            if (k0 < p.stored_rows)
              tma_load_3d(dst, &tq0, bar, f0 / 2, k0, e);
            else
              tma_load_3d(dst, &tq1, bar, f0 / 2, k0 - p.stored_rows, e);
          }
        }
        __syncwarp();
        ring.advance(kStagesP);
      }
    }
  } else if (warp == 3) {
    Ring ring;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int rb = tile % n_rowblk;
      for (int s = 0; s < n_main; ++s) {
        if (!wait_all(&s_empty[ring.stage], ring.phase ^ 1u, abort_flag, status)) goto done;
        load_stage_scales<MODE>(p, tt.x, rb, s, lane, sS + ring.stage * kSBytes);
        cp_async_arrive_noinc(&s_full[ring.stage]);
        ring.advance(kStagesS);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------ B tile producer
    Ring ring;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int nbox = (tt.z + 15) >> 4;
      for (int s = 0; s <= n_main; ++s) {
        if (!wait_all(&b_empty[ring.stage], ring.phase ^ 1u, abort_flag, status)) goto done;
        if (lane == 0) {
          uint64_t* bar = &b_full[ring.stage];
          uint8_t* dst = sB + ring.stage * kBBytes;
          mbar_expect_tx(bar, nbox * 2048);
          // the tile's rows in at most a few boxes of 128/64/32/16 rows
          int row = 0;
          for (int lvl = 3; lvl >= 0; --lvl) {
            const int h = 16 << lvl;
            while (16 * nbox - row >= h) {
              if (s < n_main)
                tma_load_2d(dst + row * 128, &maps.b[lvl], bar, s * kBlockK, tt.y + row);
              else
                tma_load_2d(dst + row * 128, &maps.bx[lvl], bar, 0, tt.y + row);
              row += h;
            }
          }
        }
        __syncwarp();
        ring.advance(kStagesB);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    Ring ra, rbr;
    AccTrack acc;
    const int ksteps_x = kext_steps<MODE>(p.rpad);
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const bool two = block_two<MODE>(p, tile % n_rowblk);
      const int n_mma = (tt.z + 15) & ~15;
      const bool wide = n_mma > 128;
      const uint32_t idesc = make_idesc_f16((uint32_t)n_mma, kAMnMajor<MODE>, false);
      uint32_t d0;
      if (wide) {
        if (!wait_all(&acc_empty[0], (acc.uses[0] & 1u) ^ 1u, abort_flag, status)) goto done;
        if (!wait_all(&acc_empty[1], (acc.uses[1] & 1u) ^ 1u, abort_flag, status)) goto done;
        d0 = tmem;
      } else {
        if (!wait_all(&acc_empty[acc.next], (acc.uses[acc.next] & 1u) ^ 1u, abort_flag, status)) goto done;
        d0 = tmem + (uint32_t)(acc.next * 256);
      }
      const uint32_t d1 = d0 + (wide ? 256u : 128u);
      tc_fence_after();
      for (int s = 0; s <= n_main; ++s) {
        if (!wait_all(&a_full[ra.stage], ra.phase, abort_flag, status)) goto done;
        if (!wait_all(&b_full[rbr.stage], rbr.phase, abort_flag, status)) goto done;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_base = smem_u32(sA + ra.stage * kABytes);
          const uint32_t b_base = smem_u32(sB + rbr.stage * kBBytes);
          const int ksteps = (s < n_main) ? (kBlockK / 16) : ksteps_x;
          for (int kk = 0; kk < ksteps; ++kk) {
            const uint32_t a_off = kAMnMajor<MODE> ? (uint32_t)kk * 2048u : (uint32_t)kk * 32u;
            const uint32_t lbo = kAMnMajor<MODE> ? 8192u : 16u;
            const uint64_t a0 = make_sdesc_sw128(a_base + a_off, lbo, 1024);
            const uint64_t a1 = make_sdesc_sw128(a_base + kAHalf + a_off, lbo, 1024);
            const uint64_t bdesc = make_sdesc_sw128(b_base + kk * 32, 16, 1024);
            const uint32_t accum = (s > 0 || kk > 0) ? 1u : 0u;
            umma_f16_ss(d0, a0, bdesc, idesc, accum);
            if (two) umma_f16_ss(d1, a1, bdesc, idesc, accum);
          }
          umma_commit(&a_empty[ra.stage]);
          umma_commit(&b_empty[rbr.stage]);
        }
        __syncwarp();
        ra.advance(kStagesA);
        rbr.advance(kStagesB);
      }
      if (lane == 0) {
        if (wide) {
          umma_commit(&acc_full[0]);
          umma_commit(&acc_full[1]);
        } else {
          umma_commit(&acc_full[acc.next]);
        }
      }
      __syncwarp();
      acc.retire(wide);
    }
  } else if (warp >= kEpiWarp0 && warp < kDecWarp0) {
    // --------------------------------------------------------------- epilogue
    const int q = warp & 3;       // TMEM lane quarter this warp may access
    const int m = 32 * q + lane;  // accumulator row of this thread in each MMA
    AccTrack acc;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int rb = tile % n_rowblk;
      const bool two = block_two<MODE>(p, rb);
      const int f0 = block_f0<MODE>(rb);
      const int n_rows = tt.z;
      const int p0 = tt.y;
      const int n_mma = (n_rows + 15) & ~15;
      const bool wide = n_mma > 128;
      uint32_t d0;
      if (wide) {
        if (!wait_all(&acc_full[0], acc.uses[0] & 1u, abort_flag, status)) goto done;
        if (!wait_all(&acc_full[1], acc.uses[1] & 1u, abort_flag, status)) goto done;
        d0 = tmem;
      } else {
        if (!wait_all(&acc_full[acc.next], acc.uses[acc.next] & 1u, abort_flag, status)) goto done;
        d0 = tmem + (uint32_t)(acc.next * 256);
      }
      const uint32_t d1 = d0 + (wide ? 256u : 128u);
      tc_fence_after();
      const uint32_t lane_base = (uint32_t)(32 * q) << 16;
      for (int c0 = 0; c0 < n_mma; c0 += 32) {
        uint32_t v0[32], v1[32];
        {
          tmem_ld32(d0 + lane_base + (uint32_t)c0, v0);
          if (two) {
            tmem_ld32(d1 + lane_base + (uint32_t)c0, v1);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) v1[c] = 0u;
          }
        }
        if constexpr (MODE == kModeGateUp) {
          // row m of the first MMA is gate feature f0 + m, of the second up feature f0 + m
          const int i = f0 + m;
          const float L = p.limit;
          bool overflow = false;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int n = c0 + c;
            if (n < n_rows && i < p.feat) {
              const int64_t o = (int64_t)(p0 + n) * p.ld_out + i;
              const float g = __uint_as_float(v0[c]);
              const float u = __uint_as_float(v1[c]);
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
        } else if constexpr (MODE == kModeDown || MODE == kModeGateUpT) {
          float wl = 1.0f;
          if constexpr (MODE == kModeDown) wl = __ldg(p.w_perm + p0 + min(c0 + lane, n_rows - 1));
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int n = c0 + c;
            const float w = __shfl_sync(0xffffffffu, wl, c);
            if (n < n_rows) {
              const int64_t row = p0 + n;
              float a = __uint_as_float(v0[c]);
              float b = __uint_as_float(v1[c]);
              if constexpr (MODE == kModeDown) {
                a *= w;
                b *= w;
              }
              if (f0 + m < p.feat) p.out_a[row * p.ld_out + f0 + m] = a;  // a partial last block
              if (two && f0 + 128 + m < p.feat) p.out_a[row * p.ld_out + f0 + 128 + m] = b;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (wide) {
          mbar_arrive(&acc_empty[0]);
          mbar_arrive(&acc_empty[1]);
        } else {
          mbar_arrive(&acc_empty[acc.next]);
        }
      }
      acc.retire(wide);
    }
  } else if (warp >= kDecWarp0) {
    // --------------------------------------------------------------- decoders
    const int dt = threadIdx.x - kDecWarp0 * 32;
    Ring ra, rp, rs;
    const uint32_t s_off = scale_off<MODE>(dt);
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int rb = tile % n_rowblk;
      const int e = tt.x;
      uint32_t lora_w[32];
      lora_values<MODE>(p, e, rb, dt, lora_w);
      for (int s = 0; s <= n_main; ++s) {
        if (!wait_all(&a_empty[ra.stage], ra.phase ^ 1u, abort_flag, status)) goto done;
        uint8_t* A = sA + ra.stage * kABytes;
        int p_release = -1;  // packed stage to hand back once its bytes are consumed
        int s_release = -1;
        if (s < n_main) {
          if (!wait_all(&s_full[rs.stage], rs.phase, abort_flag, status)) goto done;
          const uint32_t sc = *reinterpret_cast<const uint32_t*>(sS + rs.stage * kSBytes + s_off);
          s_release = rs.stage;
          rs.advance(kStagesS);
          if (!wait_all(&p_full[rp.stage], rp.phase, abort_flag, status)) goto done;
          uint4 q0, q1;
          packed_pair<MODE>(sP + rp.stage * kPBytes, dt, q0, q1);
          p_release = rp.stage;
          rp.advance(kStagesP);
          uint32_t w0[16], w1[16];
          decode_group32(q0, bf16_scale_to_h2((uint16_t)(sc & 0xFFFFu)), w0);
          decode_group32(q1, bf16_scale_to_h2((uint16_t)(sc >> 16)), w1);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            *reinterpret_cast<uint4*>(A + a_chunk_off<MODE>(dt, c)) =
                make_uint4(w0[4 * c], w0[4 * c + 1], w0[4 * c + 2], w0[4 * c + 3]);
            *reinterpret_cast<uint4*>(A + a_chunk_off<MODE>(dt, 4 + c)) =
                make_uint4(w1[4 * c], w1[4 * c + 1], w1[4 * c + 2], w1[4 * c + 3]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(A + a_chunk_off<MODE>(dt, c)) =
                make_uint4(lora_w[4 * c], lora_w[4 * c + 1], lora_w[4 * c + 2], lora_w[4 * c + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // The packed stage is released only here, after the decoded values
          // that consume its bytes were stored: an arrive issued right after
          // the shared loads can overtake them, and the refill of the stage
          // then lands under loads still in flight.
          if (p_release >= 0) mbar_arrive(&p_empty[p_release]);
          if (s_release >= 0) mbar_arrive(&s_empty[s_release]);
          mbar_arrive(&a_full[ra.stage]);
        }
        ra.advance(kStagesA);
      }
    }
  }

done:
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int MODE>
cudaError_t launch_mode(const GemmParams& p, const GemmMaps& m, int grid, cudaStream_t stream) {
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  if (!device_flag_test(attr_set, &dev)) {
    cudaError_t err = cudaFuncSetAttribute(gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    device_flag_set(attr_set, dev);
  }
  gemm_kernel<MODE><<<grid, kThreads, kSmemBytes, stream>>>(p, m);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(int mode, const GemmParams& p, const GemmMaps& maps, int grid, cudaStream_t stream) {
  switch (mode) {
    case kModeGateUp: return launch_mode<kModeGateUp>(p, maps, grid, stream);
    case kModeDown: return launch_mode<kModeDown>(p, maps, grid, stream);
    case kModeGateUpT: return launch_mode<kModeGateUpT>(p, maps, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace r4
