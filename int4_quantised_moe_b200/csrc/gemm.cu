// Dequant-fused grouped GEMMs of the routed RAWINT4 MoE-LoRA layer on
// sm_100a tensor cores (tcgen05, TMEM accumulators, TMA-fed operands).
//
// One persistent CTA per SM walks (token tile, output row block) work items.
// A token tile is up to 256 permuted rows of one expert; a row block is 128
// output features (64 gate + 64 up features in the gate/up mode). Warp roles:
//   warp 0      TMA producer of packed int4 weight tiles   (ring of kStagesP)
//   warp 2      TMA producer of B tiles (activations)      (ring of kStagesB)
//   warps 8-15  decoders: int4 -> fp16 into the UMMA A layout (ring of kStagesA)
//   warp 1      UMMA issuer (one elected lane) and TMEM owner
//   warps 4-7   epilogue: TMEM -> registers -> fused math -> global
// The LoRA side product of each projection runs as one extra 64-wide
// reduction stage in the same accumulator: its A operand is the LoRA tensor
// of the expert (copied/converted by the decoders), its B operand the
// precomputed c-scaled rank-r side matrix of the tokens.
//
// The backward modes read the packed base along its stored output dimension
// (transpose-free dX, rawint4_sft_reference.py transpose_free_rawint4_dx):
// the decoders write the same packed bytes into an MN-major A tile, so no
// transposed or dense copy of any base weight ever exists.
#include "gemm.cuh"

namespace r4 {

namespace {

constexpr int kABytes = kRowsM * kBlockK * 2;  // 16 KB
constexpr int kBBytes = 256 * kBlockK * 2;     // 32 KB
constexpr int kPBytes = kRowsM * kBlockK / 2;  // 4 KB
constexpr int kOffA = 0;
constexpr int kOffB = kOffA + kStagesA * kABytes;
constexpr int kOffP = kOffB + kStagesB * kBBytes;
constexpr int kOffBar = kOffP + kStagesP * kPBytes;
constexpr int kNumBars = 2 * kStagesP + 2 * kStagesA + 2 * kStagesB + 4;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kOffEpi = (kOffMisc + 16 + 127) / 128 * 128;
constexpr int kEpiFloats = 4 * 32 * 33 + 4 * 32;
constexpr int kSmemBytes = kOffEpi + kEpiFloats * 4 + 1024;  // + alignment slack
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

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a
// 128B-swizzled block whose rows are 128 bytes and whose 8-row atoms are
// 1024 bytes apart.
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int MODE>
__device__ __forceinline__ uint32_t a_chunk_off(int dt, int j) {
  if constexpr (!kAMnMajor<MODE>) {
    const int m = dt >> 1, half = dt & 1;
    return sw128_off(m, 4 * half + j);
  } else {
    const int kr = dt >> 2, qq = dt & 3;
    return (uint32_t)((qq >> 1) * 8192) + sw128_off(kr, 4 * (qq & 1) + j);
  }
}

template <int MODE>
__device__ __forceinline__ uint16_t load_scale(const GemmParams& p, int e, int rb, int s, int dt) {
  if constexpr (MODE == kModeGateUp) {
    const int m = dt >> 1, half = dt & 1;
    const uint16_t* sp = (m < 64) ? p.s0 : p.s1;
    const int row = rb * 64 + (m & 63);
    return __ldg(sp + (int64_t)e * p.s_expert + (int64_t)row * p.s_row + 2 * s + half);
  } else if constexpr (MODE == kModeDown) {
    const int m = dt >> 1, half = dt & 1;
    const int row = rb * 128 + m;
    return __ldg(p.s0 + (int64_t)e * p.s_expert + (int64_t)row * p.s_row + 2 * s + half);
  } else if constexpr (MODE == kModeDownT) {
    const int kr = dt >> 2, qq = dt & 3;
    const int row = s * kBlockK + kr;
    return __ldg(p.s0 + (int64_t)e * p.s_expert + (int64_t)row * p.s_row + rb * 4 + qq);
  } else {
    const int kr = dt >> 2, qq = dt & 3;
    int row = s * kBlockK + kr;
    const uint16_t* sp = p.s0;
    if (row >= p.stored_rows) {
      row -= p.stored_rows;
      sp = p.s1;
    }
    return __ldg(sp + (int64_t)e * p.s_expert + (int64_t)row * p.s_row + rb * 4 + qq);
  }
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// This thread's 32 values of the A tile of the LoRA reduction stage, as 16
// fp16 pairs in the same order the decode produces (see a_chunk_off).
// Loaded at the start of a work item, long before the stage is stored: a
// decoder warp that stores operand data right after long-latency global loads
// at the tail of a work item produced corrupted rows in earlier builds, and
// the early load also takes that latency off the critical path.
template <int MODE>
__device__ __forceinline__ void lora_values(const GemmParams& p, int e, int rb, int dt, uint32_t (&w)[16]) {
  const int r = p.rank;
  if constexpr (!kAMnMajor<MODE>) {
    // A[m, j] with j in [32*half, 32*half + 32): LoRA B rows (K-major, rank contiguous)
    const int m = dt >> 1, half = dt & 1;
    const uint16_t* src;
    int jlo;  // first reduction column that holds this row's values
    if constexpr (MODE == kModeGateUp) {
      const bool up = m >= 64;
      src = (up ? p.lx1 : p.lx0) + (int64_t)e * p.lx_expert + (int64_t)(rb * 64 + (m & 63)) * p.lx_ld;
      jlo = up ? p.rpad : 0;
    } else {
      src = p.lx0 + (int64_t)e * p.lx_expert + (int64_t)(rb * 128 + m) * p.lx_ld;
      jlo = 0;
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float v[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int jj = 32 * half + 2 * t + u - jlo;
        v[u] = (jj >= 0 && jj < r) ? bf16_bits_to_float(__ldg(src + jj)) : 0.0f;
      }
      w[t] = pack_h2(v[0], v[1]);
    }
  } else {
    // A[m, kr] with m in [32*qq, 32*qq + 32): LoRA A rows (MN-major, feature contiguous)
    const int kr = dt >> 2, qq = dt & 3;
    const uint16_t* src = nullptr;
    if (kr < r)
      src = p.lx0 + (int64_t)e * p.lx_expert + (int64_t)kr * p.lx_ld + rb * 128 + 32 * qq;
    else if (MODE == kModeGateUpT && kr >= p.rpad && kr < p.rpad + r)
      src = p.lx1 + (int64_t)e * p.lx_expert + (int64_t)(kr - p.rpad) * p.lx_ld + rb * 128 + 32 * qq;
    if (src) {
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

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ GemmMaps maps) {
  const CUtensorMap& tq0 = maps.q0;
  const CUtensorMap& tq1 = maps.q1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + kOffA;
  uint8_t* sB = smem + kOffB;
  uint8_t* sP = smem + kOffP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* p_full = bars;
  uint64_t* p_empty = p_full + kStagesP;
  uint64_t* a_full = p_empty + kStagesP;
  uint64_t* a_empty = a_full + kStagesA;
  uint64_t* b_full = a_empty + kStagesA;
  uint64_t* b_empty = b_full + kStagesB;
  uint64_t* acc_full = b_empty + kStagesB;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  float* epi = reinterpret_cast<float*>(smem + kOffEpi);

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
      const int rb = tile % n_rowblk;
      const int e = tt.x;
      for (int s = 0; s < n_main; ++s) {
        if (!wait_all(&p_empty[ring.stage], ring.phase ^ 1u, abort_flag, status)) goto done;
        if (lane == 0) {
          uint64_t* bar = &p_full[ring.stage];
          uint8_t* dst = sP + ring.stage * kPBytes;
          mbar_expect_tx(bar, kPBytes);
          if constexpr (MODE == kModeGateUp) {
            tma_load_3d(dst, &tq0, bar, s * (kBlockK / 2), rb * 64, e);
            tma_load_3d(dst + kPBytes / 2, &tq1, bar, s * (kBlockK / 2), rb * 64, e);
          } else if constexpr (MODE == kModeDown) {
            tma_load_3d(dst, &tq0, bar, s * (kBlockK / 2), rb * 128, e);
          } else if constexpr (MODE == kModeDownT) {
            tma_load_3d(dst, &tq0, bar, rb * 64, s * kBlockK, e);
          } else {
            const int k0 = s * kBlockK;
            if (k0 < p.stored_rows)
              tma_load_3d(dst, &tq0, bar, rb * 64, k0, e);
            else
              tma_load_3d(dst, &tq1, bar, rb * 64, k0 - p.stored_rows, e);
          }
        }
        __syncwarp();
        ring.advance(kStagesP);
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
    int it = 0;
    const int ksteps_x = kext_steps<MODE>(p.rpad);
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int n_mma = (tt.z + 15) & ~15;
      const uint32_t idesc = make_idesc_f16((uint32_t)n_mma, kAMnMajor<MODE>, false);
      const int ab = it & 1;
      const uint32_t acc_ph = (uint32_t)(it >> 1) & 1u;
      if (!wait_all(&acc_empty[ab], acc_ph ^ 1u, abort_flag, status)) goto done;
      tc_fence_after();
      const uint32_t d_tmem = tmem + (uint32_t)(ab * 256);
      for (int s = 0; s <= n_main; ++s) {
        if (!wait_all(&a_full[ra.stage], ra.phase, abort_flag, status)) goto done;
        if (!wait_all(&b_full[rbr.stage], rbr.phase, abort_flag, status)) goto done;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_base = smem_u32(sA + ra.stage * kABytes);
          const uint32_t b_base = smem_u32(sB + rbr.stage * kBBytes);
          const int ksteps = (s < n_main) ? (kBlockK / 16) : ksteps_x;
          for (int kk = 0; kk < ksteps; ++kk) {
            uint64_t adesc;
            if constexpr (kAMnMajor<MODE>)
              adesc = make_sdesc_sw128(a_base + kk * 2048, 8192, 1024);
            else
              adesc = make_sdesc_sw128(a_base + kk * 32, 16, 1024);
            const uint64_t bdesc = make_sdesc_sw128(b_base + kk * 32, 16, 1024);
            umma_f16_ss(d_tmem, adesc, bdesc, idesc, (s > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&a_empty[ra.stage]);
          umma_commit(&b_empty[rbr.stage]);
        }
        __syncwarp();
        ra.advance(kStagesA);
        rbr.advance(kStagesB);
      }
      if (lane == 0) umma_commit(&acc_full[ab]);
      __syncwarp();
    }
  } else if (warp >= kEpiWarp0 && warp < kDecWarp0) {
    // --------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int rb = tile % n_rowblk;
      const int n_rows = tt.z;
      const int p0 = tt.y;
      const int n_mma = (n_rows + 15) & ~15;
      const int ab = it & 1;
      const uint32_t acc_ph = (uint32_t)(it >> 1) & 1u;
      if (!wait_all(&acc_full[ab], acc_ph, abort_flag, status)) goto done;
      tc_fence_after();
      for (int c0 = 0; c0 < n_mma; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(ab * 256 + c0), v);
        if constexpr (MODE == kModeGateUp) {
          float* xch = epi + (q & 1) * 32 * 33;
          if (q >= 2) {
#pragma unroll
            for (int c = 0; c < 32; ++c) xch[lane * 33 + c] = __uint_as_float(v[c]);
          }
          named_bar_sync(1 + (q & 1), 64);
          if (q < 2) {
            const int i = rb * 64 + 32 * q + lane;
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
          const int m = rb * 128 + 32 * q + lane;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int n = c0 + c;
            if (n < n_rows) {
              const int64_t row = p0 + n;
              float val = __uint_as_float(v[c]);
              if constexpr (MODE == kModeDown) val *= __ldg(p.w_perm + row);
              p.out_a[row * p.ld_out + m] = val;
            }
          }
        } else {  // kModeDownT
          const int i = rb * 128 + 32 * q + lane;
          const float L = p.limit;
          float* red = epi + q * 32 * 33;
          float* red2 = epi + 4 * 32 * 33;
          bool overflow = false;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int n = c0 + c;
            float prod = 0.f;
            if (n < n_rows) {
              const int64_t row = p0 + n;
              const float acc = __uint_as_float(v[c]);
              const float w = __ldg(p.w_perm + row);
              const float g = p.in_g[row * p.ld_out + i];
              const float u = p.in_u[row * p.ld_out + i];
              const float gc = L > 0.f ? fminf(g, L) : g;
              const float uc = L > 0.f ? fminf(fmaxf(u, -L), L) : u;
              const bool pass_g = !(L > 0.f) || g <= L;
              const bool pass_u = !(L > 0.f) || (u >= -L && u <= L);
              const float sg = sigmoid_clamped(gc);
              const float silu = gc * sg;
              const float dsilu = sg * (1.0f + gc * (1.0f - sg));
              const float dh = w * acc;
              const float dg = pass_g ? dh * uc * dsilu : 0.f;
              const float du = pass_u ? dh * silu : 0.f;
              const __half hg = __float2half_rn(dg);
              const __half hu = __float2half_rn(du);
              overflow |= (__hisinf(hg) | __hisinf(hu)) != 0;
              p.out_h[row * (2 * p.inter) + i] = *reinterpret_cast<const uint16_t*>(&hg);
              p.out_h[row * (2 * p.inter) + p.inter + i] = *reinterpret_cast<const uint16_t*>(&hu);
              prod = acc * silu * uc;
            }
            red[lane * 33 + c] = prod;
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
              p.droute_part[(int64_t)(p0 + n) * n_rowblk + rb] = sum;
            }
          }
          named_bar_sync(3, 128);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  } else if (warp >= kDecWarp0) {
    // --------------------------------------------------------------- decoders
    const int dt = threadIdx.x - kDecWarp0 * 32;
    Ring ra, rp;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      const int4 tt = p.tok_tiles[tile / n_rowblk];
      const int rb = tile % n_rowblk;
      const int e = tt.x;
      uint32_t lora_w[16];
      lora_values<MODE>(p, e, rb, dt, lora_w);
      // group scales of the next four stages, loaded well before their use
      uint16_t sq0 = n_main > 0 ? load_scale<MODE>(p, e, rb, 0, dt) : 0;
      uint16_t sq1 = n_main > 1 ? load_scale<MODE>(p, e, rb, 1, dt) : 0;
      uint16_t sq2 = n_main > 2 ? load_scale<MODE>(p, e, rb, 2, dt) : 0;
      uint16_t sq3 = n_main > 3 ? load_scale<MODE>(p, e, rb, 3, dt) : 0;
      for (int s = 0; s <= n_main; ++s) {
        if (!wait_all(&a_empty[ra.stage], ra.phase ^ 1u, abort_flag, status)) goto done;
        uint8_t* A = sA + ra.stage * kABytes;
        if (s < n_main) {
          const uint16_t scale = sq0;
          sq0 = sq1;
          sq1 = sq2;
          sq2 = sq3;
          sq3 = (s + 4 < n_main) ? load_scale<MODE>(p, e, rb, s + 4, dt) : 0;
          if (!wait_all(&p_full[rp.stage], rp.phase, abort_flag, status)) goto done;
          const uint4 qv = *reinterpret_cast<const uint4*>(sP + rp.stage * kPBytes + dt * 16);
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_empty[rp.stage]);
          rp.advance(kStagesP);
          uint32_t w[16];
          decode_group32(qv, bf16_scale_to_h2(scale), w);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(A + a_chunk_off<MODE>(dt, j)) =
                make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(A + a_chunk_off<MODE>(dt, j)) =
                make_uint4(lora_w[4 * j], lora_w[4 * j + 1], lora_w[4 * j + 2], lora_w[4 * j + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[ra.stage]);
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
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t err = cudaFuncSetAttribute(gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    attr_set = true;
  }
  gemm_kernel<MODE><<<grid, kThreads, kSmemBytes, stream>>>(p, m);
  return cudaGetLastError();
}

}  // namespace

size_t gemm_smem_bytes() { return kSmemBytes; }

cudaError_t launch_gemm(int mode, const GemmParams& p, const GemmMaps& maps, int grid, cudaStream_t stream) {
  switch (mode) {
    case kModeGateUp: return launch_mode<kModeGateUp>(p, maps, grid, stream);
    case kModeDown: return launch_mode<kModeDown>(p, maps, grid, stream);
    case kModeDownT: return launch_mode<kModeDownT>(p, maps, grid, stream);
    case kModeGateUpT: return launch_mode<kModeGateUpT>(p, maps, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace r4
