// Rank-r LoRA products on the tensor cores (see skinny.cuh).
//
// Two persistent CTAs per SM (about 105 KB of shared memory and 256 TMEM
// columns each): the UMMAs of these products are small (M = 128, N = 64), so
// one issuer leaves the tensor pipe mostly idle and a second CTA's stream
// fills it. In each CTA warp 0 issues TMA loads of both operands into a ring
// of stages, warp 1 issues the UMMAs into a double-buffered TMEM
// accumulator, warps 2-5 run the epilogue. No thread ever writes an operand
// tile except to clear the rows past an expert's last row in the gradient
// mode (constant stores, fenced for the async proxy before the MMA reads).
#include "skinny.cuh"

namespace r4 {
namespace {

constexpr int kSkA = 128 * 64 * 2;  // A tile: 128 rows x 64 fp16
constexpr int kSkB = 64 * 64 * 2;   // B tile: 64 rows x 64 fp16
constexpr int kSkStage = kSkA + kSkB;
// Shared memory of each mode: the ring of stages, the barriers, and (Grads
// only) the gradient staging of the transposed outputs:
// [2 outputs][32 rank][128 features] fp32. Rows mode spends the staging's
// room on a fourth stage.
template <int MODE>
constexpr int kSkStagesOf = MODE == kSkRows ? kSkStages + 1 : kSkStages;
template <int MODE>
constexpr int kSkOffBar = kSkStagesOf<MODE> * kSkStage;
template <int MODE>
constexpr int kSkNumBars = 2 * kSkStagesOf<MODE> + 4;
template <int MODE>
constexpr int kSkOffMisc = kSkOffBar<MODE> + kSkNumBars<MODE> * 8;
template <int MODE>
constexpr int kSkOffStage = (kSkOffMisc<MODE> + 16 + 15) / 16 * 16;
constexpr int kSkStageFloats = 2 * 32 * 128;
template <int MODE>
constexpr int kSkSmem = kSkOffStage<MODE> + (MODE == kSkGrads ? kSkStageFloats * 4 : 0) + 1024;
static_assert(2 * (kSkSmem<kSkRows> + 1024) <= 233472 && 2 * (kSkSmem<kSkGrads> + 1024) <= 233472,
              "two CTAs per SM (228 KB per SM, 1 KB reserved per CTA)");
constexpr uint32_t kSkTmemCols = 256;

struct GradItem {
  int job, e, fb;
};

__device__ __forceinline__ GradItem grad_item(const SkParams& p, int item) {
  GradItem g{0, 0, 0};
  int base = 0;
  for (int j = 0; j < p.njobs; ++j) {
    const int n = p.experts * p.job[j].nfb;
    if (item < base + n) {
      const int rem = item - base;
      g.job = j;
      g.e = rem / p.job[j].nfb;
      g.fb = rem - g.e * p.job[j].nfb;
      return g;
    }
    base += n;
  }
  return g;
}

__device__ __forceinline__ int total_items(const SkParams& p, int mode) {
  if (mode == kSkRows) return p.hdr->n_tok_tiles * 2;
  int n = 0;
  for (int j = 0; j < p.njobs; ++j) n += p.experts * p.job[j].nfb;
  return n;
}

// Zero rows [r0, r1) of a 64-row MN-major 128B-swizzled block (rows are 128 B).
__device__ __forceinline__ void zero_rows(uint8_t* blk, int r0, int r1, int lane) {
  const int n16 = (r1 - r0) * 8;
  for (int i = lane; i < n16; i += 32) {
    const int row = r0 + (i >> 3);
    *reinterpret_cast<uint4*>(blk + (row >> 3) * 1024 + (row & 7) * 128 + ((i & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Authoritative-window store of one gradient element.
__device__ __forceinline__ void grad_store(uint16_t* out, int64_t o, float v, int accumulate) {
  if (accumulate) v += bf16_bits_to_float(out[o]);
  out[o] = bf16_bits_rn(v);
}

__device__ __forceinline__ uint32_t grad_pair(uint32_t old, float a, float b, int accumulate) {
  if (accumulate) {
    a += __uint_as_float(old << 16);
    b += __uint_as_float(old & 0xFFFF0000u);
  }
  return (uint32_t)bf16_bits_rn(a) | ((uint32_t)bf16_bits_rn(b) << 16);
}

// Ranks [jlo, jlo + n) (n <= 32) of feature pp of expert e in one output
// buffer whose rank extent is `ld`: buf = (accumulate ? buf : 0) + gs * D[j],
// D read from the accumulator columns in `v` (all zero when `zero`).
// [E, pout, ld] rows are contiguous and go out as 16-byte vectors when n, ld
// and jlo are multiples of 8 and the buffer is 16-byte aligned; [E, ld, pout]
// columns are written one element per rank index, contiguous across the
// warp's lanes.
__device__ __forceinline__ void grad_row(uint16_t* buf, const SkJob& jb, int ld, int jlo, int n, int e, int pp,
                                         const uint32_t (&v)[32], float gs, int accumulate, bool zero) {
  if (zero) accumulate = 0;
  if (!jb.transposed) {
    uint16_t* dst = buf + ((int64_t)e * jb.pout + pp) * ld + jlo;
    if (((n | ld | jlo) & 7) == 0 && (reinterpret_cast<uintptr_t>(buf) & 15u) == 0) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (8 * c < n) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 8 * c);
          const uint4 old = accumulate ? *d4 : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
          uint32_t nw[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float a = zero ? 0.f : gs * __uint_as_float(v[8 * c + 2 * t]);
            const float b = zero ? 0.f : gs * __uint_as_float(v[8 * c + 2 * t + 1]);
            nw[t] = grad_pair(ow[t], a, b, accumulate);
          }
          *d4 = make_uint4(nw[0], nw[1], nw[2], nw[3]);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < n) grad_store(dst, j, zero ? 0.f : gs * __uint_as_float(v[j]), accumulate);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < n)
        grad_store(buf, ((int64_t)e * ld + jlo + j) * jb.pout + pp, zero ? 0.f : gs * __uint_as_float(v[j]),
                   accumulate);
  }
}

// One part of the [E, ld, pout] outputs of a 128-feature block: ranks
// [jlo, jlo + n) (n <= 32) of buffer `buf`, from `v`.
struct GradPart {
  uint16_t* buf;
  int jlo, n;
};

// The transposed outputs of one 128-feature block, in up to two parts (the
// two buffers of the rank split, or the two rank halves of a rank above 32):
// the four epilogue warps write their features' gradients into shared
// memory, then store whole 256-byte rows (8 features per thread and step)
// with the authoritative-window rule (accumulate: add the old value, round
// once). All 128 epilogue threads take part (named barrier 1).
__device__ __forceinline__ void grad_block_transposed(const SkJob& jb, int ld, int e, int p0, GradPart q0, GradPart q1,
                                                      int nparts, const uint32_t (&v0)[32], const uint32_t (&v1)[32],
                                                      float gs, int accumulate, bool zero, float* st, int c, int tid) {
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if (j < q0.n) st[j * 128 + c] = zero ? 0.f : gs * __uint_as_float(v0[j]);
    if (nparts > 1 && j < q1.n) st[4096 + j * 128 + c] = zero ? 0.f : gs * __uint_as_float(v1[j]);
  }
  named_bar_sync(1, 128);
  const int n_all = q0.n * 16 + (nparts > 1 ? q1.n * 16 : 0);
  for (int idx = tid; idx < n_all; idx += 128) {
    const int o = idx < q0.n * 16 ? 0 : 1;
    const int rem = o ? idx - q0.n * 16 : idx;
    const int j = rem >> 4, v8 = rem & 15;
    const float* src = st + o * 4096 + j * 128 + 8 * v8;
    if (p0 + 8 * v8 >= jb.pout) continue;  // past the last feature (a partial last block)
    const GradPart& q = o ? q1 : q0;
    uint4* dst = reinterpret_cast<uint4*>(q.buf + ((int64_t)e * ld + q.jlo + j) * jb.pout + p0 + 8 * v8);
    const uint4 old = accumulate ? *dst : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
    uint32_t nw[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) nw[t] = grad_pair(ow[t], src[2 * t], src[2 * t + 1], accumulate);
    *dst = make_uint4(nw[0], nw[1], nw[2], nw[3]);
  }
  named_bar_sync(1, 128);
}

template <int MODE>
__global__ void __launch_bounds__(kSkThreads, 1)
    skinny_kernel(const __grid_constant__ SkParams p, const __grid_constant__ SkMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kStages = kSkStagesOf<MODE>;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSkOffBar<MODE>);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kSkOffMisc<MODE>);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSkOffMisc<MODE> + 4);
  float* gstage = reinterpret_cast<float*>(smem + kSkOffStage<MODE>);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kSkTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  uint32_t* status = p.status;
  const bool enabled = !(p.need_saved && p.hdr->saved != 1u);
  const int n_items = enabled ? total_items(p, MODE) : 0;

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    Ring ring;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      if constexpr (MODE == kSkRows) {
        const int4 tt = p.tok_tiles[item >> 1];
        const int mb = item & 1;
        if (mb * 128 >= tt.z) continue;
        const int p0 = tt.y + mb * 128;
        const int bb = p.sw * 128;  // R box: sw rows of 64 fp16
        for (int s = 0; s < p.nseg; ++s) {
          for (int k = 0; k < p.nk; ++k) {
            if (!wait_all(&empty[ring.stage], ring.phase ^ 1u, abort_flag, status)) goto done;
            if (lane == 0) {
              uint8_t* st = smem + ring.stage * kSkStage;
              mbar_expect_tx(&full[ring.stage], kSkA + bb);
              tma_load_2d(st, &maps.a[0], &full[ring.stage], p.seg_lcol[s] + 64 * k, p0);
              tma_load_3d(st + kSkA, &maps.b[s], &full[ring.stage], 64 * k, 0, tt.x);
            }
            __syncwarp();
            ring.advance(kStages);
          }
        }
      } else {
        const GradItem g = grad_item(p, item);
        const SkJob& jb = p.job[g.job];
        // every gradient is linear in grad_out, whose fp16 copy carries the scale 2^dy_exp
        const float gsc = ldexpf(p.grad_scale, -p.hdr->dy_exp);
        const int row0 = p.offsets[g.e], row1 = p.offsets[g.e + 1];
        const int nk = (row1 - row0 + 63) / 64;
        for (int k = 0; k < nk; ++k) {
          if (!wait_all(&empty[ring.stage], ring.phase ^ 1u, abort_flag, status)) goto done;
          if (lane == 0) {
            uint8_t* st = smem + ring.stage * kSkStage;
            mbar_expect_tx(&full[ring.stage], kSkA + kSkB);
            const int x = jb.lcol + 128 * g.fb;
            tma_load_2d(st, &maps.a[jb.amap], &full[ring.stage], x, row0 + 64 * k);
            tma_load_2d(st + kSkA / 2, &maps.a[jb.amap], &full[ring.stage], x + 64, row0 + 64 * k);
            tma_load_2d(st + kSkA, &maps.b[jb.bmap], &full[ring.stage], jb.scol, row0 + 64 * k);
          }
          __syncwarp();
          ring.advance(kStages);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    Ring ring;
    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      int nk, nseg, row0 = 0, rows = 0;
      if constexpr (MODE == kSkRows) {
        const int4 tt = p.tok_tiles[item >> 1];
        if ((item & 1) * 128 >= tt.z) continue;
        nk = p.nk;
        nseg = p.nseg;
      } else {
        const GradItem g = grad_item(p, item);
        row0 = p.offsets[g.e];
        rows = p.offsets[g.e + 1] - row0;
        nk = (rows + 63) / 64;
        nseg = 1;
        if (nk == 0) continue;
      }
      const int ab = it & 1;
      if (!wait_all(&acc_empty[ab], ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag, status)) goto done;
      tc_fence_after();
      for (int s = 0; s < nseg; ++s) {
        const uint32_t d_tmem = tmem + (uint32_t)(ab * 128 + s * 64);
        for (int k = 0; k < nk; ++k) {
          if (!wait_all(&full[ring.stage], ring.phase, abort_flag, status)) goto done;
          uint8_t* st = smem + ring.stage * kSkStage;
          int ksteps = 4;
          if constexpr (MODE == kSkGrads) {
            const int rem = rows - 64 * k;
            if (rem < 64) {
              // rows past the expert's last row belong to other experts: clear
              // them in both operands up to the next 16-row MMA step
              ksteps = (rem + 15) / 16;
              const int r1 = ksteps * 16;
              zero_rows(st, rem, r1, lane);
              zero_rows(st + kSkA / 2, rem, r1, lane);
              zero_rows(st + kSkA, rem, r1, lane);
              fence_proxy_async_smem();
              __syncwarp();
            }
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t a_base = smem_u32(st);
            const uint32_t b_base = smem_u32(st + kSkA);
            for (int kk = 0; kk < ksteps; ++kk) {
              uint64_t ad, bd;
              uint32_t idesc;
              if constexpr (MODE == kSkRows) {
                ad = make_sdesc_sw128(a_base + kk * 32, 16, 1024);
                bd = make_sdesc_sw128(b_base + kk * 32, 16, 1024);
                idesc = make_idesc_f16(64, false, false);
              } else {
                ad = make_sdesc_sw128(a_base + kk * 2048, 8192, 1024);
                bd = make_sdesc_sw128(b_base + kk * 2048, 8192, 1024);
                idesc = make_idesc_f16(64, true, true);
              }
              umma_f16_ss(d_tmem, ad, bd, idesc, (k > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&empty[ring.stage]);
          }
          __syncwarp();
          ring.advance(kStages);
        }
      }
      if (lane == 0) umma_commit(&acc_full[ab]);
      __syncwarp();
      ++it;
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int q = warp & 3;
    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      if constexpr (MODE == kSkRows) {
        const int4 tt = p.tok_tiles[item >> 1];
        const int mb = item & 1;
        if (mb * 128 >= tt.z) continue;
        const int nrows = min(128, tt.z - mb * 128);
        const int ab = it & 1;
        if (!wait_all(&acc_full[ab], (uint32_t)(it >> 1) & 1u, abort_flag, status)) goto done;
        tc_fence_after();
        const int m = 32 * q + lane;
        const int64_t row = tt.y + mb * 128 + m;
        const float w = (p.out1 && m < nrows) ? __ldg(p.w_perm + row) : 0.f;
        // output column c = s * sw + j  <-  accumulator column s * 64 + j,
        // kept when j lies inside a rank block (j % rpad < rank)
        const int ncols = p.nseg * p.sw > 64 ? kLoraPad : 64;
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          const int s = c0 / p.sw;
          const int j0 = c0 - s * p.sw;
          uint32_t v[16];
          const bool live = s < p.nseg;
          if (live) tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(ab * 128 + s * 64 + j0), v);
          if (m < nrows) {
            uint32_t o0[8], o1[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              const bool ka = live && ((j0 + 2 * t) % p.rpad) < p.rank;
              const bool kb = live && ((j0 + 2 * t + 1) % p.rpad) < p.rank;
              const float a = ka ? p.scale * __uint_as_float(v[2 * t]) : 0.f;
              const float b = kb ? p.scale * __uint_as_float(v[2 * t + 1]) : 0.f;
              __half2 h = __floats2half2_rn(a, b);
              o0[t] = *reinterpret_cast<uint32_t*>(&h);
              __half2 hw = __floats2half2_rn(w * a, w * b);
              o1[t] = *reinterpret_cast<uint32_t*>(&hw);
            }
            uint4* d0 = reinterpret_cast<uint4*>(p.out0 + row * kLoraPad + c0);
            d0[0] = make_uint4(o0[0], o0[1], o0[2], o0[3]);
            d0[1] = make_uint4(o0[4], o0[5], o0[6], o0[7]);
            if (p.out1) {
              uint4* d1 = reinterpret_cast<uint4*>(p.out1 + row * kLoraPad + c0);
              d1[0] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
              d1[1] = make_uint4(o1[4], o1[5], o1[6], o1[7]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        ++it;
      } else {
        const GradItem g = grad_item(p, item);
        const SkJob& jb = p.job[g.job];
        // every gradient is linear in grad_out, whose fp16 copy carries the scale 2^dy_exp
        const float gsc = ldexpf(p.grad_scale, -p.hdr->dy_exp);
        const int rows = p.offsets[g.e + 1] - p.offsets[g.e];
        const int pf = 128 * g.fb + 32 * q + lane;  // feature of this lane
        // outputs of this item: the low rank block -> out_lo, except the
        // second feature half of a feature split (high block -> out_hi); the
        // rank split writes both blocks
        uint16_t* out0 = jb.out_lo;
        uint32_t col0 = 0;
        int pbase = 0;
        // the split point P/2 (= I) is a multiple of 32, so each warp's 32
        // features lie on one side of it (a block may straddle it)
        if (jb.split == kSplitFeature && 128 * g.fb + 32 * q >= jb.P / 2) {
          out0 = jb.out_hi;
          col0 = (uint32_t)p.rpad;
          pbase = jb.P / 2;
        }
        const bool both = jb.split == kSplitRank;
        const bool wide = !both && p.rank > 32;  // one buffer, ranks from D columns [0, rank)
        // the parts this lane writes: (buffer, first rank, ranks) from v0 and v1
        GradPart q0{out0, 0, min(p.rank, 32)}, q1{nullptr, 0, 0};
        int nparts = 1;
        if (both) {
          q1 = GradPart{jb.out_hi, 0, p.rank};
          nparts = 2;
        } else if (wide) {
          q1 = GradPart{out0, 32, p.rank - 32};
          nparts = 2;
        }
        const bool live = pf < jb.P;
        uint32_t v0[32], v1[32];
        if (rows == 0) {
          // no rows of this expert in the call: cleared, or kept when accumulating
          if (p.accumulate) continue;
#pragma unroll
          for (int j = 0; j < 32; ++j) v0[j] = v1[j] = 0u;
          if (jb.transposed) {
            grad_block_transposed(jb, p.rank, g.e, 128 * g.fb - pbase, q0, q1, nparts, v0, v1, 0.f, 0, true, gstage,
                                  32 * q + lane, threadIdx.x - 64);
          } else if (live) {
            grad_row(q0.buf, jb, p.rank, q0.jlo, q0.n, g.e, pf - pbase, v0, 0.f, 0, true);
            if (nparts > 1) grad_row(q1.buf, jb, p.rank, q1.jlo, q1.n, g.e, pf - pbase, v1, 0.f, 0, true);
          }
          continue;
        }
        const int ab = it & 1;
        if (!wait_all(&acc_full[ab], (uint32_t)(it >> 1) & 1u, abort_flag, status)) goto done;
        tc_fence_after();
        const uint32_t t0 = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(ab * 128);
        tmem_ld32(t0 + col0, v0);
        if (both) tmem_ld32(t0 + (uint32_t)p.rpad, v1);
        if (wide) tmem_ld32(t0 + 32u, v1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        ++it;
        if (jb.transposed) {
          grad_block_transposed(jb, p.rank, g.e, 128 * g.fb - pbase, q0, q1, nparts, v0, v1, gsc, p.accumulate,
                                false, gstage, 32 * q + lane, threadIdx.x - 64);
        } else if (live) {
          grad_row(q0.buf, jb, p.rank, q0.jlo, q0.n, g.e, pf - pbase, v0, gsc, p.accumulate, false);
          if (nparts > 1) grad_row(q1.buf, jb, p.rank, q1.jlo, q1.n, g.e, pf - pbase, v1, gsc, p.accumulate, false);
        }
      }
    }
  }

done:
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kSkTmemCols);
}

template <int MODE>
cudaError_t launch_sk(const SkParams& p, const SkMaps& m, int grid, cudaStream_t stream) {
  static std::atomic<unsigned long long> attr{0};
  int dev = 0;
  if (!device_flag_test(attr, &dev)) {
    cudaError_t e = cudaFuncSetAttribute(skinny_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSkSmem<MODE>);
    if (e != cudaSuccess) return e;
    // the largest shared-memory carveout, so that two CTAs fit on an SM
    e = cudaFuncSetAttribute(skinny_kernel<MODE>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    device_flag_set(attr, dev);
  }
  skinny_kernel<MODE><<<grid, kSkThreads, kSkSmem<MODE>, stream>>>(p, m);
  return cudaGetLastError();
}

// ---------------------------------------------------------- LoRA to FP16
__device__ __forceinline__ uint32_t bf16x2_to_h2(uint32_t v) {
  __half2 h = __floats2half2_rn(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
  return *reinterpret_cast<uint32_t*>(&h);
}

// One job per blockIdx.y. Copies: one warp per output row, 8 elements per
// lane and vector (16-byte loads and stores; K is a multiple of 64).
// Transposes with a rank that is a multiple of 8: two adjacent columns per
// thread (below). Other ranks: tiles of 64 columns of one expert; the tile's
// 64 source rows of r elements are one contiguous, 16-byte aligned run of
// 128 r bytes, loaded as 16-byte vectors, turned around in shared memory and
// stored as rows of 64 fp16.
__global__ void __launch_bounds__(256) lora_convert_kernel(LoraCvt j0, LoraCvt j1, LoraCvt j2, int experts) {
  const LoraCvt jb = blockIdx.y == 0 ? j0 : (blockIdx.y == 1 ? j1 : j2);
  if (!jb.dst) return;
  const int r = jb.rank, rp = jb.rpad, cols = jb.cols;
  if (!jb.transpose) {
    // one warp per output row: the row's expert and rank are found once, and
    // its vectors go four per lane and pass, loads ahead of stores
    const int rows_out = rp * jb.nsrc;
    const int vpr = cols / 8;
    const int rows_total = experts * rows_out;
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    uint4* dst = reinterpret_cast<uint4*>(jb.dst);
    for (int rg = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; rg < rows_total; rg += nwarps) {
      const int e = rg / rows_out;
      const int row = rg - e * rows_out;
      const int blk = row / rp, j = row - blk * rp;
      uint4* d = dst + (int64_t)rg * vpr;
      if (j >= r) {
        for (int v = lane; v < vpr; v += 32) d[v] = make_uint4(0u, 0u, 0u, 0u);
        continue;
      }
      const uint4* src = reinterpret_cast<const uint4*>((blk == 0 ? jb.src0 : jb.src1) + ((int64_t)e * r + j) * cols);
      for (int v0 = lane; v0 < vpr; v0 += 128) {
        uint4 in[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (v0 + 32 * q < vpr) in[q] = __ldg(src + v0 + 32 * q);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (v0 + 32 * q < vpr)
            d[v0 + 32 * q] = make_uint4(bf16x2_to_h2(in[q].x), bf16x2_to_h2(in[q].y), bf16x2_to_h2(in[q].z),
                                        bf16x2_to_h2(in[q].w));
      }
    }
  } else if (r % 8 == 0) {
    // transposes of a rank that fills 16-byte vectors: thread -> two adjacent
    // columns c, c + 1 of one expert, whose 2 r source values are one
    // contiguous, 16-byte aligned run; for each rank j the warp stores 64
    // adjacent fp16 (128 bytes) of output row j
    const int64_t pairs = (int64_t)experts * (cols / 2);
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    const int rv = r / 8;  // 16-byte vectors per source row
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < pairs; t += step) {
      const int e = (int)(t / (cols / 2));
      const int c = 2 * (int)(t - (int64_t)e * (cols / 2));
      const uint4* src = reinterpret_cast<const uint4*>(jb.src0 + ((int64_t)e * cols + c) * r);  // [2][r]
      uint16_t* d = jb.dst + (int64_t)e * rp * cols + c;
      for (int j0 = 0; j0 < r; j0 += 8) {
        const uint4 a = __ldg(src + j0 / 8);       // column c, ranks j0..j0+7
        const uint4 b = __ldg(src + rv + j0 / 8);  // column c + 1
        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float fa = __uint_as_float(((wa[u >> 1] >> (16 * (u & 1))) & 0xFFFFu) << 16);
          const float fb = __uint_as_float(((wb[u >> 1] >> (16 * (u & 1))) & 0xFFFFu) << 16);
          const uint32_t h = (uint32_t)f16_bits_rn(fa) | ((uint32_t)f16_bits_rn(fb) << 16);
          *reinterpret_cast<uint32_t*>(d + (int64_t)(j0 + u) * cols) = h;
        }
      }
      for (int j = r; j < rp; ++j) *reinterpret_cast<uint32_t*>(d + (int64_t)j * cols) = 0u;
    }
  } else {
    __shared__ float tile[64][65];  // 64 source rows x up to 64 ranks (+1: no bank conflicts)
    const int tiles_per_e = cols / 64;
    for (int t = blockIdx.x; t < experts * tiles_per_e; t += gridDim.x) {
      const int e = t / tiles_per_e;
      const int c0 = (t - e * tiles_per_e) * 64;
      const uint4* src = reinterpret_cast<const uint4*>(jb.src0 + ((int64_t)e * cols + c0) * r);  // [64][r], contiguous
      for (int v = threadIdx.x; v < 8 * r; v += blockDim.x) {
        const uint4 in = __ldg(src + v);
        const uint32_t w[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int flat = 8 * v + u;
          const int c = flat / r, j = flat - c * r;
          const uint32_t bits = (w[u >> 1] >> (16 * (u & 1))) & 0xFFFFu;
          tile[c][j] = __uint_as_float(bits << 16);
        }
      }
      __syncthreads();
      for (int o = threadIdx.x; o < rp * 8; o += blockDim.x) {
        const int j = o >> 3, v = o & 7;
        uint32_t h[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float a = j < r ? tile[8 * v + 2 * u][j] : 0.f;
          const float b = j < r ? tile[8 * v + 2 * u + 1][j] : 0.f;
          h[u] = (uint32_t)f16_bits_rn(a) | ((uint32_t)f16_bits_rn(b) << 16);
        }
        *reinterpret_cast<uint4*>(jb.dst + ((int64_t)e * rp + j) * cols + c0 + 8 * v) = make_uint4(h[0], h[1], h[2], h[3]);
      }
      __syncthreads();
    }
  }
}

}  // namespace

cudaError_t launch_skinny(int mode, const SkParams& p, const SkMaps& m, int grid, cudaStream_t stream) {
  return mode == kSkRows ? launch_sk<kSkRows>(p, m, grid, stream) : launch_sk<kSkGrads>(p, m, grid, stream);
}

cudaError_t launch_lora_convert(const LoraCvt* jobs, int njobs, int experts, cudaStream_t stream) {
  LoraCvt z{};
  LoraCvt j[3] = {njobs > 0 ? jobs[0] : z, njobs > 1 ? jobs[1] : z, njobs > 2 ? jobs[2] : z};
  if (njobs <= 0) return cudaSuccess;
  dim3 grid(148 * 8, njobs > 3 ? 3 : njobs, 1);
  lora_convert_kernel<<<grid, 256, 0, stream>>>(j[0], j[1], j[2], experts);
  return cudaGetLastError();
}

}  // namespace r4
