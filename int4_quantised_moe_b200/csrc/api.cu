// C ABI of the routed RAWINT4 MoE-LoRA layer: argument checks, workspace
// carve-up, TMA descriptors and the launch sequences of forward and backward.
// Entry points mirror forward_sft / backward of the contract test
// (test_rawint4_sft_numerical.py, _forward and _backward).
#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>

#include "aux.cuh"
#include "gemm.cuh"
#include "prof.cuh"
#include "route.cuh"
#include "router.cuh"
#include "skinny.cuh"

namespace r4 {
namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Device buffers of one layer call, carved out of the caller's workspace.
struct Layout {
  size_t hdr, offsets, perm, inv, w_perm, tiles, hist;
  size_t xp, xa, g, u, h, ha, hw, y, gp, gd, gdw, dgu, gb, dpart;
  size_t gu16, ad16, bdt16, bgt16, but16;  // FP16 LoRA copies for the row products
  int rpad;
  size_t total;
  int64_t rows;  // padded permuted-row capacity
  int max_tiles;
};

Layout make_layout(const rawint4_moe_cfg& c) {
  Layout L{};
  const int64_t R = (int64_t)c.max_tokens * c.top_k;
  // capacity rounded to whole 256-row tiles plus one spare tile: TMA boxes of
  // the last token tile and zero-padded LoRA side rows stay inside the buffers
  L.rows = (R + kTileRows - 1) / kTileRows * kTileRows + kTileRows;
  L.max_tiles = max_tok_tiles((int32_t)R, c.experts, kTileRowsNarrow);  // either tile configuration
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  const int64_t H = c.hidden, I = c.inter, E = c.experts, rows = L.rows;
  L.hdr = take(sizeof(WsHeader));
  L.offsets = take((E + 1) * 4);
  L.perm = take(rows * 4);
  L.inv = take(rows * 4);
  L.w_perm = take(rows * 4);
  L.tiles = take((size_t)L.max_tiles * 16);
  L.hist = take(route_scratch_bytes((int32_t)R, c.experts));
  L.xp = take(rows * H * 2);
  L.xa = take(rows * kLoraPad * 2);
  L.g = take(rows * I * 4);
  L.u = take(rows * I * 4);
  L.h = take(rows * I * 2);
  L.ha = take(rows * kLoraPad * 2);
  L.hw = take(rows * kLoraPad * 2);
  L.y = take(rows * H * 4);
  L.gp = take(rows * H * 2);
  L.gd = take(rows * kLoraPad * 2);
  L.gdw = take(rows * kLoraPad * 2);
  L.dgu = take(rows * 2 * I * 2);
  L.gb = take(rows * kLoraPad * 2);
  L.dpart = take(rows * 2 * ((I + 255) / 256) * 4);
  L.rpad = (c.rank + 15) / 16 * 16;
  const int64_t rp = L.rpad;
  L.gu16 = take(E * 2 * rp * H * 2);
  L.ad16 = take(E * rp * I * 2);
  L.bdt16 = take(E * rp * H * 2);
  L.bgt16 = take(E * rp * I * 2);
  L.but16 = take(E * rp * I * 2);
  L.total = off;
  return L;
}

bool cfg_ok(const rawint4_moe_cfg* c) {
  if (!c) return false;
  if (c->experts < 1 || c->experts > 4096) return false;
  if (c->top_k < 1 || c->top_k > c->experts) return false;
  if (c->hidden < 64 || c->hidden % 64 != 0) return false;
  if (c->inter < 64 || c->inter % 64 != 0) return false;
  if (c->rank < 1 || c->rank > 64) return false;
  if (!std::isfinite(c->alpha)) return false;
  if (!std::isfinite(c->swiglu_limit) || c->swiglu_limit < 0.f) return false;
  if (c->max_tokens < 1) return false;
  if (c->weight_format != RAWINT4_FORMAT_RAWINT4 && c->weight_format != RAWINT4_FORMAT_MXFP4) return false;
  if (c->weight_format == RAWINT4_FORMAT_MXFP4 && (c->hidden % 128 != 0 || c->inter % 128 != 0)) return false;
  if ((int64_t)c->max_tokens * c->top_k > (1 << 24)) return false;
  return true;
}

// Base and LoRA tensors are read by TMA and by 16-byte vector loads: their
// starting addresses must be 16-byte aligned.
bool a16(const void* p) { return p && reinterpret_cast<uintptr_t>(p) % 16 == 0; }
bool base_ok(const rawint4_moe_base* b) {
  return b && a16(b->gate_q) && a16(b->up_q) && a16(b->down_q) && a16(b->gate_s) && a16(b->up_s) && a16(b->down_s);
}
bool lora_ok(const rawint4_moe_lora* l) {
  return l && a16(l->gate_a) && a16(l->gate_b) && a16(l->up_a) && a16(l->up_b) && a16(l->down_a) && a16(l->down_b);
}
bool grads_ok(const rawint4_moe_lora_grads* g) {
  return g && a16(g->gate_a) && a16(g->gate_b) && a16(g->up_a) && a16(g->up_b) && a16(g->down_a) && a16(g->down_b);
}

}  // namespace

// --------------------------------------------------------------- device
namespace {
std::mutex g_mu;
int g_checked_device = -1;
int g_sm_count = 0;
}  // namespace

int check_device(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RAWINT4_CUDA_ERROR;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_checked_device != dev) {
    int major = 0, minor = 0, count = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return RAWINT4_CUDA_ERROR;
    if (major != 10 || minor != 0) return RAWINT4_UNSUPPORTED;
    g_checked_device = dev;
    g_sm_count = count;
  }
  *sms = g_sm_count;
  return RAWINT4_OK;
}

namespace {

// ------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// packed projection [E, rows, kbytes] uint8; box {box_x bytes, box_y rows, 1};
// the 128- and 64-byte-wide boxes of the transposed modes are loaded with the
// matching swizzle (conflict-free reads by the decoders)
bool map_packed(CUtensorMap* m, const uint8_t* base, int64_t E, int64_t rows, int64_t kbytes, int box_x, int box_y,
                bool swizzle32 = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kbytes, (cuuint64_t)rows, (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)kbytes, (cuuint64_t)(kbytes * rows)};
  cuuint32_t box[3] = {(cuuint32_t)box_x, (cuuint32_t)box_y, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = box_x == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : box_x == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : swizzle32   ? CU_TENSOR_MAP_SWIZZLE_32B
                                              : CU_TENSOR_MAP_SWIZZLE_NONE;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp16 row-major [rows, cols]; box {64, box_rows}, 128-byte swizzle (UMMA
// K-major operand rows, or MN-major atoms when rows are the reduction)
bool map_act(CUtensorMap* m, const uint16_t* base, int64_t rows, int64_t cols, int box_rows = 16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// the four row-box variants {64, 16/32/64/128} of one fp16 activation matrix
bool map_act_boxes(CUtensorMap* m, const uint16_t* base, int64_t rows, int64_t cols) {
  for (int i = 0; i < 4; ++i)
    if (!map_act(&m[i], base, rows, cols, 16 << i)) return false;
  return true;
}

// fp16 per-expert matrices [E, rows, cols]; box {64, rows, 1}, 128-byte swizzle
// fp16 [E, expert_rows, cols]: `rows` rows of every expert (from `base`), box
// {64, rows, 1}, 128-byte swizzle (expert_rows = rows unless a block of rows
// of a taller per-expert matrix is mapped)
bool map_expert_rows(CUtensorMap* m, const uint16_t* base, int64_t E, int64_t rows, int64_t cols,
                     int64_t expert_rows = 0) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (expert_rows <= 0) expert_rows = rows;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)(cols * 2), (cuuint64_t)(cols * expert_rows * 2)};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<uint16_t*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

int common_checks(const rawint4_moe_cfg* cfg, const rawint4_moe_base* base, const rawint4_moe_lora* lora,
                  void* workspace, size_t ws_bytes, Layout* L) {
  // lora may be NULL (base-only forward); the entry points check where that is allowed
  if (!cfg_ok(cfg) || !base_ok(base) || (lora && !lora_ok(lora)) || !workspace) return RAWINT4_INVALID_ARGUMENT;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign != 0) return RAWINT4_INVALID_ARGUMENT;
  *L = make_layout(*cfg);
  if (ws_bytes < L->total) return RAWINT4_INVALID_ARGUMENT;
  return RAWINT4_OK;
}

int grid_for_tiles(int sms, int max_tiles, int rowblk) {
  const int64_t t = (int64_t)max_tiles * rowblk;
  return (int)(t < sms ? (t > 0 ? t : 1) : sms);
}

// CTA pairs for a pair-kernel launch: all that fit at once, or fewer for a small
// problem (work items = token tiles x feature blocks).
int gemm_clusters(int mode, int fmt, bool narrow, int sms, int max_tiles, int rowblk) {
  static std::atomic<int> cached[64][2][2][4];  // per device, configuration, format and mode; 0 = not queried yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  int fit = cached[dev][narrow][fmt][mode].load();
  if (fit <= 0) {
    const int n = narrow ? gemm_pair_max_clusters_narrow(mode, fmt) : gemm_pair_max_clusters(mode, fmt);
    fit = n > 0 ? n : (sms / 2 > 0 ? sms / 2 : 1);  // occupancy query unavailable: one pair per SM pair
    cached[dev][narrow][fmt][mode].store(fit);
  }
  const int64_t items = (int64_t)max_tiles * rowblk;
  return (int)(items < fit ? (items > 0 ? items : 1) : fit);
}

// CTA pairs for a launch of the tensor-memory GEMM (gemm_tm.cu).
int tm_clusters(int mode, int fmt, bool narrow, int sms, int max_tiles, int rowblk) {
  static std::atomic<int> cached[64][2][2][4];  // per device, configuration, format and mode; 0 = not queried yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  int fit = cached[dev][narrow][fmt][mode].load();
  if (fit <= 0) {
    const int n = narrow ? gemm_tm_max_clusters_narrow(mode, fmt) : gemm_tm_max_clusters(mode, fmt);
    fit = n > 0 ? n : (sms / 2 > 0 ? sms / 2 : 1);
    cached[dev][narrow][fmt][mode].store(fit);
  }
  const int64_t items = (int64_t)max_tiles * rowblk;
  return (int)(items < fit ? (items > 0 ? items : 1) : fit);
}

// Token-tile configuration of a call: narrow (tiles of at most
// kTileRowsNarrow rows, the GEMMs' narrow configurations) when the workspace
// averages at most kTileRowsNarrow / 2 routed rows per expert (max_tokens x
// top_k / experts), wide otherwise. The choice depends on the configuration
// only, so a backward always matches its forward. The environment may force
// it (RAWINT4_TILES=narrow or wide) for testing.
bool narrow_tiles(const rawint4_moe_cfg& c) {
  const char* e = getenv("RAWINT4_TILES");
  if (e && strcmp(e, "narrow") == 0) return true;
  if (e && strcmp(e, "wide") == 0) return false;
  return 2LL * c.max_tokens * c.top_k <= (long long)kTileRowsNarrow * c.experts;
}

// Which kernel runs the transpose-free backward GEMMs (down^T, gate/up^T):
// the shared-memory operand pair kernel (gemm_pair.cu: MN-major decoded
// tiles, no transposition), or the tensor-memory pair kernel (gemm_tm.cu)
// when the environment selects it (RAWINT4_GEMM=tm). The forward GEMMs
// always run on the tensor-memory kernel.
bool use_tm_gemm(int) {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("RAWINT4_GEMM");
    v = (e && strcmp(e, "tm") == 0) ? 1 : 0;
  }
  return v == 1;
}

// Bound on any pipeline wait of the GEMM kernels (test export can shorten it).
std::atomic<unsigned long long> g_wait_ns{4000000000ull};

#define R4_TRY(x)                                \
  do {                                           \
    if ((x) != cudaSuccess) return RAWINT4_CUDA_ERROR; \
  } while (0)

}  // namespace
}  // namespace r4

using namespace r4;

extern "C" {

int rawint4_moe_lora_workspace_size(const rawint4_moe_cfg* cfg, size_t* bytes) {
  if (!cfg_ok(cfg) || !bytes) return RAWINT4_INVALID_ARGUMENT;
  *bytes = make_layout(*cfg).total;
  return RAWINT4_OK;
}

const char* rawint4_moe_lora_strerror(int code) {
  switch (code) {
    case RAWINT4_OK: return "ok";
    case RAWINT4_INVALID_ARGUMENT: return "invalid argument (null pointer, unsupported size or workspace too small)";
    case RAWINT4_FROZEN_BASE: return "frozen base: base-weight gradients are never formed; pass NULL base gradient buffers";
    case RAWINT4_NO_SAVED_FORWARD: return "backward without a pending saved forward on this workspace";
    case RAWINT4_CUDA_ERROR: return "a CUDA runtime or driver call failed";
    case RAWINT4_BAD_EXPERT_ID: return "an expert id outside [0, experts) was routed; that slot contributed nothing";
    case RAWINT4_DEVICE_TIMEOUT: return "a device pipeline wait exceeded its bound; results are invalid";
    case RAWINT4_FP16_OVERFLOW: return "an activation exceeded the fp16 operand range; results are invalid";
    case RAWINT4_UNSUPPORTED: return "unsupported device (needs sm_100) or configuration";
    case RAWINT4_STATIC_SCRATCH_TOO_SMALL:
      return "problem too large for the fixed scratch of rawint4_moe_permute_static; use rawint4_moe_permute";
    default: return "unknown status code";
  }
}

int rawint4_moe_lora_fwd(const rawint4_moe_cfg* cfg, const rawint4_moe_base* base, const rawint4_moe_lora* lora,
                         int32_t qlen, const int64_t* expert_ids, const float* route_weights, const uint16_t* x,
                         uint16_t* out, int save_for_backward, void* workspace, size_t ws_bytes, void* stream_) {
  Layout L;
  int rc = common_checks(cfg, base, lora, workspace, ws_bytes, &L);
  if (rc != RAWINT4_OK) return rc;
  if (qlen < 0 || qlen > cfg->max_tokens) return RAWINT4_INVALID_ARGUMENT;
  if (qlen > 0 && (!expert_ids || !route_weights || !x || !out)) return RAWINT4_INVALID_ARGUMENT;
  // Without LoRA the call is a frozen-base inference forward: it saves no
  // context, so there is nothing a backward could consume.
  const bool has_lora = lora != nullptr;
  if (!has_lora && save_for_backward) return RAWINT4_INVALID_ARGUMENT;
  int sms = 0;
  rc = check_device(&sms);
  if (rc != RAWINT4_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream_);
  const rawint4_moe_cfg& c = *cfg;
  const int H = c.hidden, I = c.inter, E = c.experts, k = c.top_k, r = c.rank, rp = L.rpad;
  const float scaling = c.alpha / (float)r;
  void* ws = workspace;
  WsHeader* hdr = at<WsHeader>(ws, L.hdr);
  const bool nar = narrow_tiles(c);  // token-tile configuration of this layer

  {
    R4_PROF("header_fwd", st);
    R4_TRY(launch_header_begin_fwd(hdr, save_for_backward, st));
  }
  {
    R4_PROF("route", st);
    R4_TRY(launch_route(expert_ids, route_weights, qlen, k, E, at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.perm),
                        at<int32_t>(ws, L.inv), at<float>(ws, L.w_perm), at<int4>(ws, L.tiles),
                        at<int32_t>(ws, L.hist), hdr, st, nar ? kTileRowsNarrow : kTileRows));
  }
  if (qlen == 0) return RAWINT4_OK;
  const int maxR = qlen * k;
  const int max_tiles = max_tok_tiles(maxR, E, nar ? kTileRowsNarrow : kTileRows);
  {
    R4_PROF("gather_x", st);
    R4_TRY(launch_gather_rows(x, at<int32_t>(ws, L.inv), k, hdr, at<uint16_t>(ws, L.xp), H, qlen, &hdr->status, 0, 0,
                              st));
  }
  if (has_lora) {
    R4_PROF("lora_convert", st);
    LoraCvt cv[2] = {{lora->gate_a, lora->up_a, at<uint16_t>(ws, L.gu16), r, rp, H, 0, 2},
                     {lora->down_a, nullptr, at<uint16_t>(ws, L.ad16), r, rp, I, 0, 1}};
    R4_TRY(launch_lora_convert(cv, 2, E, st));
  }
  // Base-only forward: the GEMMs' rank stage multiplies zero side rows by a
  // zero B operand (every row of it read from the first elements of the
  // zeroed xa buffer), which adds exact zeros to the accumulators.
  const uint16_t* zero_rows = at<uint16_t>(ws, L.xa);

  SkParams sp{};
  sp.tok_tiles = at<int4>(ws, L.tiles);
  sp.hdr = hdr;
  sp.status = &hdr->status;
  sp.need_saved = 0;
  sp.rank = r;
  sp.rpad = rp;
  sp.scale = scaling;
  sp.w_perm = at<float>(ws, L.w_perm);
  SkMaps sm;
  const int rows_grid = grid_for_tiles(kSkCtasPerSm * sms, 2 * max_tiles, 1);

  // xa = c * X_perm [A_g; A_u]^T: gate in columns [0, r), up in [rp, rp + r);
  // both rank blocks in one 64-wide segment up to rank 32, one segment each
  // above (the same X_perm columns, the gate and up halves of gu16)
  if (!map_act(&sm.a[0], at<uint16_t>(ws, L.xp), L.rows, H, 128)) return RAWINT4_CUDA_ERROR;
  if (2 * rp <= 64) {
    if (!map_expert_rows(&sm.b[0], at<uint16_t>(ws, L.gu16), E, 2 * rp, H)) return RAWINT4_CUDA_ERROR;
    sp.nseg = 1;
    sp.sw = 2 * rp;
  } else {
    if (!map_expert_rows(&sm.b[0], at<uint16_t>(ws, L.gu16), E, rp, H, 2 * rp) ||
        !map_expert_rows(&sm.b[1], at<uint16_t>(ws, L.gu16) + (int64_t)rp * H, E, rp, H, 2 * rp))
      return RAWINT4_CUDA_ERROR;
    sp.nseg = 2;
    sp.seg_lcol[1] = 0;
    sp.sw = rp;
  }
  sp.seg_lcol[0] = 0;
  sp.nk = H / 64;
  sp.out0 = at<uint16_t>(ws, L.xa);
  sp.out1 = nullptr;
  if (has_lora) {
    R4_PROF("lora_xa", st);
    R4_TRY(launch_skinny(kSkRows, sp, sm, rows_grid, st));
  } else {
    R4_PROF("zero_xa", st);
    R4_TRY(launch_fill_u16(at<uint16_t>(ws, L.xa), L.rows * kLoraPad, 0, st));
  }

  GemmMaps mp;
  GemmParams gp{};
  gp.tok_tiles = at<int4>(ws, L.tiles);
  gp.hdr = hdr;
  gp.status = &hdr->status;
  gp.need_saved = 0;
  gp.rank = r;
  gp.rpad = rp;
  gp.w_perm = at<float>(ws, L.w_perm);
  gp.inter = I;
  gp.limit = c.swiglu_limit;

  // gate/up: G, U (fp32, saved) and h = silu(G') U' (fp16)
  const int fmt = c.weight_format;
  // tensor-memory kernel: boxes of 64 rows x 128 bytes (4 reduction stages)
  if (!map_packed(&mp.q0, base->gate_q, E, I, H / 2, 128, 64) ||
      !map_packed(&mp.q1, base->up_q, E, I, H / 2, 128, 64) ||
      !map_act_boxes(mp.b, at<uint16_t>(ws, L.xp), L.rows, H) || !map_act_boxes(mp.bx, at<uint16_t>(ws, L.xa), L.rows, kLoraPad))
    return RAWINT4_CUDA_ERROR;
  gp.wait_ns = g_wait_ns.load();
  gp.n_rowblk = (I + 127) / 128;
  gp.feat = I;
  gp.n_main = H / kBlockK;
  gp.s0 = static_cast<const uint16_t*>(base->gate_s);
  gp.s1 = static_cast<const uint16_t*>(base->up_s);
  gp.e0 = static_cast<const uint8_t*>(base->gate_s);
  gp.e1 = static_cast<const uint8_t*>(base->up_s);
  gp.s_expert = (int64_t)I * (H / 32);
  gp.s_row = H / 32;
  gp.stored_rows = I;
  gp.lx0 = has_lora ? lora->gate_b : zero_rows;
  gp.lx1 = has_lora ? lora->up_b : zero_rows;
  gp.lx_expert = has_lora ? (int64_t)I * r : 0;
  gp.lx_ld = has_lora ? r : 0;
  gp.out_a = at<float>(ws, L.g);
  gp.out_b = at<float>(ws, L.u);
  gp.out_h = at<uint16_t>(ws, L.h);
  gp.ld_out = I;
  {
    R4_PROF("gemm_gate_up", st);
    const int ncl = tm_clusters(kModeGateUp, fmt, nar, sms, max_tiles, gp.n_rowblk);
    R4_TRY(nar ? launch_gemm_tm_narrow(kModeGateUp, fmt, gp, mp, ncl, st) : launch_gemm_tm(kModeGateUp, fmt, gp, mp, ncl, st));
  }

  // ha = c * h A_d^T and hw = w * ha
  if (has_lora) {
    if (!map_act(&sm.a[0], at<uint16_t>(ws, L.h), L.rows, I, 128) ||
        !map_expert_rows(&sm.b[0], at<uint16_t>(ws, L.ad16), E, rp, I))
      return RAWINT4_CUDA_ERROR;
    sp.nk = I / 64;
    sp.sw = rp;
    sp.out0 = at<uint16_t>(ws, L.ha);
    sp.out1 = at<uint16_t>(ws, L.hw);
    R4_PROF("lora_ha", st);
    R4_TRY(launch_skinny(kSkRows, sp, sm, rows_grid, st));
  } else {
    R4_PROF("zero_ha", st);
    R4_TRY(launch_fill_u16(at<uint16_t>(ws, L.ha), L.rows * kLoraPad, 0, st));
  }

  // down: Yw = w * (h W_d^T + ha B_d^T)
  if (!map_packed(&mp.q0, base->down_q, E, H, I / 2, 128, 64) || !map_packed(&mp.q1, base->down_q, E, H, I / 2, 128, 64) ||
      !map_act_boxes(mp.b, at<uint16_t>(ws, L.h), L.rows, I) || !map_act_boxes(mp.bx, at<uint16_t>(ws, L.ha), L.rows, kLoraPad))
    return RAWINT4_CUDA_ERROR;
  gp.n_rowblk = (H + 255) / 256;
  gp.feat = H;
  gp.n_main = I / kBlockK;
  gp.s0 = gp.s1 = static_cast<const uint16_t*>(base->down_s);
  gp.e0 = gp.e1 = static_cast<const uint8_t*>(base->down_s);
  gp.s_expert = (int64_t)H * (I / 32);
  gp.s_row = I / 32;
  gp.stored_rows = H;
  gp.lx0 = gp.lx1 = has_lora ? lora->down_b : zero_rows;
  gp.lx_expert = has_lora ? (int64_t)H * r : 0;
  gp.lx_ld = has_lora ? r : 0;
  gp.out_a = at<float>(ws, L.y);
  gp.out_b = nullptr;
  gp.out_h = nullptr;
  gp.ld_out = H;
  {
    R4_PROF("gemm_down", st);
    const int ncl = tm_clusters(kModeDown, fmt, nar, sms, max_tiles, gp.n_rowblk);
    R4_TRY(nar ? launch_gemm_tm_narrow(kModeDown, fmt, gp, mp, ncl, st) : launch_gemm_tm(kModeDown, fmt, gp, mp, ncl, st));
  }
  {
    R4_PROF("combine_out", st);
    R4_TRY(launch_combine_rows(at<float>(ws, L.y), at<int32_t>(ws, L.inv), k, hdr, out, H, qlen, 0, 0, st));
  }
  return RAWINT4_OK;
}

int rawint4_moe_lora_bwd(const rawint4_moe_cfg* cfg, const rawint4_moe_base* base, const rawint4_moe_lora* lora,
                         const uint16_t* grad_out, uint16_t* grad_in, float* grad_route,
                         const rawint4_moe_lora_grads* grads, const void* base_grad_gate, const void* base_grad_up,
                         const void* base_grad_down, int accumulate, float grad_scale, void* workspace, size_t ws_bytes,
                         void* stream_) {
  // The base is frozen: refuse any base-gradient buffer before touching anything.
  if (base_grad_gate || base_grad_up || base_grad_down) return RAWINT4_FROZEN_BASE;
  if (!lora) return RAWINT4_INVALID_ARGUMENT;  // the backward trains the LoRA adapters
  Layout L;
  int rc = common_checks(cfg, base, lora, workspace, ws_bytes, &L);
  if (rc != RAWINT4_OK) return rc;
  if (!grad_out || !grad_in || !grads_ok(grads) || !std::isfinite(grad_scale)) return RAWINT4_INVALID_ARGUMENT;
  int sms = 0;
  rc = check_device(&sms);
  if (rc != RAWINT4_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream_);
  const rawint4_moe_cfg& c = *cfg;
  const int H = c.hidden, I = c.inter, E = c.experts, k = c.top_k, r = c.rank, rp = L.rpad;
  const float scaling = c.alpha / (float)r;
  void* ws = workspace;
  WsHeader* hdr = at<WsHeader>(ws, L.hdr);
  const int maxQ = c.max_tokens;
  const int maxR = maxQ * k;
  const bool nar = narrow_tiles(c);  // the forward's tile configuration
  const int max_tiles = max_tok_tiles(maxR, E, nar ? kTileRowsNarrow : kTileRows);

  {
    R4_PROF("header_bwd", st);
    R4_TRY(launch_header_check_bwd(hdr, st));
  }
  // grad_out enters the fp16 operands scaled by an exact power of two chosen
  // from its largest magnitude; the combines and the gradient epilogue undo it
  {
    R4_PROF("absmax_dy", st);
    R4_TRY(launch_absmax_rows(grad_out, hdr, H, maxQ, st));
  }
  {
    R4_PROF("gather_dy", st);
    R4_TRY(launch_gather_rows(grad_out, at<int32_t>(ws, L.inv), k, hdr, at<uint16_t>(ws, L.gp), H, maxQ,
                              &hdr->status, 1, 1, st));
  }
  {
    R4_PROF("lora_convert", st);
    LoraCvt cv[3] = {{lora->down_b, nullptr, at<uint16_t>(ws, L.bdt16), r, rp, H, 1, 1},
                     {lora->gate_b, nullptr, at<uint16_t>(ws, L.bgt16), r, rp, I, 1, 1},
                     {lora->up_b, nullptr, at<uint16_t>(ws, L.but16), r, rp, I, 1, 1}};
    R4_TRY(launch_lora_convert(cv, 3, E, st));
  }

  SkParams sp{};
  sp.tok_tiles = at<int4>(ws, L.tiles);
  sp.hdr = hdr;
  sp.status = &hdr->status;
  sp.need_saved = 1;
  sp.rank = r;
  sp.rpad = rp;
  sp.scale = scaling;
  sp.w_perm = at<float>(ws, L.w_perm);
  SkMaps sm;
  const int rows_grid = grid_for_tiles(kSkCtasPerSm * sms, 2 * max_tiles, 1);

  // gd = c * g B_d and gdw = w * gd
  if (!map_act(&sm.a[0], at<uint16_t>(ws, L.gp), L.rows, H, 128) ||
      !map_expert_rows(&sm.b[0], at<uint16_t>(ws, L.bdt16), E, rp, H))
    return RAWINT4_CUDA_ERROR;
  sp.nseg = 1;
  sp.seg_lcol[0] = 0;
  sp.nk = H / 64;
  sp.sw = rp;
  sp.out0 = at<uint16_t>(ws, L.gd);
  sp.out1 = at<uint16_t>(ws, L.gdw);
  {
    R4_PROF("lora_gd", st);
    R4_TRY(launch_skinny(kSkRows, sp, sm, rows_grid, st));
  }

  GemmMaps mp;
  GemmParams gp{};
  gp.tok_tiles = at<int4>(ws, L.tiles);
  gp.hdr = hdr;
  gp.status = &hdr->status;
  gp.need_saved = 1;
  gp.rank = r;
  gp.rpad = rp;
  gp.w_perm = at<float>(ws, L.w_perm);
  gp.inter = I;
  gp.limit = c.swiglu_limit;
  gp.wait_ns = g_wait_ns.load();

  // down, transpose-free: dh = w (g W_d + gd A_d); SwiGLU' -> dG | dU; dRoute partials
  const int fmt = c.weight_format;
  const bool tm = use_tm_gemm(fmt);
  if (!map_packed(&mp.q0, base->down_q, E, H, I / 2, 64, 64) || !map_packed(&mp.q1, base->down_q, E, H, I / 2, 64, 64) ||
      !map_act_boxes(mp.b, at<uint16_t>(ws, L.gp), L.rows, H) || !map_act_boxes(mp.bx, at<uint16_t>(ws, L.gd), L.rows, kLoraPad))
    return RAWINT4_CUDA_ERROR;
  gp.n_rowblk = (I + 255) / 256;
  gp.feat = I;
  gp.n_main = H / kBlockK;
  gp.s0 = gp.s1 = static_cast<const uint16_t*>(base->down_s);
  gp.e0 = gp.e1 = static_cast<const uint8_t*>(base->down_s);
  gp.s_expert = (int64_t)H * (I / 32);
  gp.s_row = I / 32;
  gp.stored_rows = H;
  gp.lx0 = gp.lx1 = lora->down_a;
  gp.lx_expert = (int64_t)r * I;
  gp.lx_ld = I;
  gp.out_a = nullptr;
  gp.out_b = nullptr;
  gp.out_h = at<uint16_t>(ws, L.dgu);
  gp.in_g = at<float>(ws, L.g);
  gp.in_u = at<float>(ws, L.u);
  gp.droute_part = at<float>(ws, L.dpart);
  gp.n_parts = 2 * gp.n_rowblk;
  gp.ld_out = I;
  {
    R4_PROF("gemm_down_t", st);
    if (tm)
      R4_TRY(launch_gemm_tm(kModeDownT, fmt, gp, mp, tm_clusters(kModeDownT, fmt, false, sms, max_tiles, gp.n_rowblk), st));
    else {
      const int ncl = gemm_clusters(kModeDownT, fmt, nar, sms, max_tiles, gp.n_rowblk);
      R4_TRY(nar ? launch_gemm_pair_narrow(kModeDownT, fmt, gp, mp, ncl, st) : launch_gemm_pair(kModeDownT, fmt, gp, mp, ncl, st));
    }
  }

  // gb = c * [dG B_g, dU B_u]: gate in columns [0, r), up in [rp, rp + r)
  if (!map_act(&sm.a[0], at<uint16_t>(ws, L.dgu), L.rows, 2 * I, 128) ||
      !map_expert_rows(&sm.b[0], at<uint16_t>(ws, L.bgt16), E, rp, I) ||
      !map_expert_rows(&sm.b[1], at<uint16_t>(ws, L.but16), E, rp, I))
    return RAWINT4_CUDA_ERROR;
  sp.nseg = 2;
  sp.seg_lcol[0] = 0;
  sp.seg_lcol[1] = I;
  sp.nk = I / 64;
  sp.sw = rp;
  sp.out0 = at<uint16_t>(ws, L.gb);
  sp.out1 = nullptr;
  {
    R4_PROF("lora_gb", st);
    R4_TRY(launch_skinny(kSkRows, sp, sm, rows_grid, st));
  }

  // gate/up, transpose-free: dx = dG W_g + dU W_u + gb [A_g; A_u]
  if (!map_packed(&mp.q0, base->gate_q, E, I, H / 2, 64, 64) || !map_packed(&mp.q1, base->up_q, E, I, H / 2, 64, 64) ||
      !map_act_boxes(mp.b, at<uint16_t>(ws, L.dgu), L.rows, 2 * I) || !map_act_boxes(mp.bx, at<uint16_t>(ws, L.gb), L.rows, kLoraPad))
    return RAWINT4_CUDA_ERROR;
  gp.n_rowblk = (H + 255) / 256;
  gp.feat = H;
  gp.n_main = 2 * I / kBlockK;
  gp.s0 = static_cast<const uint16_t*>(base->gate_s);
  gp.s1 = static_cast<const uint16_t*>(base->up_s);
  gp.e0 = static_cast<const uint8_t*>(base->gate_s);
  gp.e1 = static_cast<const uint8_t*>(base->up_s);
  gp.s_expert = (int64_t)I * (H / 32);
  gp.s_row = H / 32;
  gp.stored_rows = I;
  gp.lx0 = lora->gate_a;
  gp.lx1 = lora->up_a;
  gp.lx_expert = (int64_t)r * H;
  gp.lx_ld = H;
  gp.out_a = at<float>(ws, L.y);
  gp.out_h = nullptr;
  gp.in_g = gp.in_u = nullptr;
  gp.droute_part = nullptr;
  gp.ld_out = H;
  {
    R4_PROF("gemm_gate_up_t", st);
    if (tm)
      R4_TRY(launch_gemm_tm(kModeGateUpT, fmt, gp, mp, tm_clusters(kModeGateUpT, fmt, false, sms, max_tiles, gp.n_rowblk), st));
    else {
      const int ncl = gemm_clusters(kModeGateUpT, fmt, nar, sms, max_tiles, gp.n_rowblk);
      R4_TRY(nar ? launch_gemm_pair_narrow(kModeGateUpT, fmt, gp, mp, ncl, st) : launch_gemm_pair(kModeGateUpT, fmt, gp, mp, ncl, st));
    }
  }
  {
    R4_PROF("combine_dx", st);
    R4_TRY(launch_combine_rows(at<float>(ws, L.y), at<int32_t>(ws, L.inv), k, hdr, grad_in, H, maxQ, 1, 1, st));
  }
  if (grad_route) {
    R4_PROF("combine_route", st);
    R4_TRY(launch_combine_route(at<float>(ws, L.dpart), 2 * ((I + 255) / 256), at<int32_t>(ws, L.inv), k, hdr, grad_route, maxQ,
                                st));
  }

  // the six LoRA gradients with the authoritative window
  {
    SkParams gq{};
    gq.hdr = hdr;
    gq.status = &hdr->status;
    gq.need_saved = 1;
    gq.rank = r;
    gq.rpad = rp;
    gq.offsets = at<int32_t>(ws, L.offsets);
    gq.experts = E;
    gq.accumulate = accumulate;
    gq.grad_scale = grad_scale;
    // features, first L column, L map, S map, first S column, feature
    // blocks, split, transposed, output features, outputs. Maps: L = gp, h,
    // dgu, xp; S = hw, gdw, xa, gb (each S holds the rank blocks at [0, r)
    // and, for the gate/up pairs, [rp, rp + r)).
    auto nfb = [](int P) { return (P + 127) / 128; };  // a partial last block is masked
    gq.job[0] = SkJob{H, 0, 0, 0, 0, nfb(H), kSplitNone, 0, H, grads->down_b, nullptr};
    gq.job[1] = SkJob{I, 0, 1, 1, 0, nfb(I), kSplitNone, 1, I, grads->down_a, nullptr};
    if (2 * rp <= 64) {
      // both rank blocks inside the 64 D columns of one job
      gq.njobs = 4;
      gq.job[2] = SkJob{2 * I, 0, 2, 2, 0, nfb(2 * I), kSplitFeature, 0, I, grads->gate_b, grads->up_b};
      gq.job[3] = SkJob{H, 0, 3, 3, 0, nfb(H), kSplitRank, 1, H, grads->gate_a, grads->up_a};
    } else {
      // a job per gate/up buffer, each reading its rank block of S
      gq.njobs = 6;
      gq.job[2] = SkJob{I, 0, 2, 2, 0, nfb(I), kSplitNone, 0, I, grads->gate_b, nullptr};
      gq.job[3] = SkJob{I, I, 2, 2, rp, nfb(I), kSplitNone, 0, I, grads->up_b, nullptr};
      gq.job[4] = SkJob{H, 0, 3, 3, 0, nfb(H), kSplitNone, 1, H, grads->gate_a, nullptr};
      gq.job[5] = SkJob{H, 0, 3, 3, rp, nfb(H), kSplitNone, 1, H, grads->up_a, nullptr};
    }
    SkMaps gm;
    if (!map_act(&gm.a[0], at<uint16_t>(ws, L.gp), L.rows, H, 64) ||
        !map_act(&gm.b[0], at<uint16_t>(ws, L.hw), L.rows, kLoraPad, 64) ||
        !map_act(&gm.a[1], at<uint16_t>(ws, L.h), L.rows, I, 64) ||
        !map_act(&gm.b[1], at<uint16_t>(ws, L.gdw), L.rows, kLoraPad, 64) ||
        !map_act(&gm.a[2], at<uint16_t>(ws, L.dgu), L.rows, 2 * I, 64) ||
        !map_act(&gm.b[2], at<uint16_t>(ws, L.xa), L.rows, kLoraPad, 64) ||
        !map_act(&gm.a[3], at<uint16_t>(ws, L.xp), L.rows, H, 64) ||
        !map_act(&gm.b[3], at<uint16_t>(ws, L.gb), L.rows, kLoraPad, 64))
      return RAWINT4_CUDA_ERROR;
    int items = 0;
    for (int j = 0; j < gq.njobs; ++j) items += E * gq.job[j].nfb;
    R4_PROF("lora_grads", st);
    R4_TRY(launch_skinny(kSkGrads, gq, gm, grid_for_tiles(kSkCtasPerSm * sms, items, 1), st));
  }
  {
    R4_PROF("header_end", st);
    R4_TRY(launch_header_end_bwd(hdr, st));
  }
  return RAWINT4_OK;
}

static bool router_args_ok(const float* scores, int32_t qlen, int32_t experts, int32_t top_k) {
  return qlen >= 0 && experts >= 1 && experts <= 4096 && top_k >= 1 && top_k <= 32 && top_k <= experts &&
         (qlen == 0 || scores != nullptr);
}

int rawint4_moe_router_topk(const float* scores, int32_t qlen, int32_t experts, int32_t top_k, const float* escale,
                            int64_t* ids, float* weights, void* stream_) {
  if (!router_args_ok(scores, qlen, experts, top_k) || (qlen > 0 && (!ids || !weights))) return RAWINT4_INVALID_ARGUMENT;
  int sms = 0;
  int rc = check_device(&sms);
  if (rc != RAWINT4_OK) return rc;
  R4_PROF("router_topk", static_cast<cudaStream_t>(stream_));
  R4_TRY(launch_router_topk(scores, qlen, experts, top_k, escale, ids, weights, static_cast<cudaStream_t>(stream_)));
  return RAWINT4_OK;
}

int rawint4_moe_router_bwd(const float* scores, int32_t qlen, int32_t experts, int32_t top_k, const int64_t* ids,
                           const float* grad_route, const float* escale, float* grad_scores, float* grad_escale,
                           void* stream_) {
  if (!router_args_ok(scores, qlen, experts, top_k) || (qlen > 0 && (!ids || !grad_route || !grad_scores)))
    return RAWINT4_INVALID_ARGUMENT;
  int sms = 0;
  int rc = check_device(&sms);
  if (rc != RAWINT4_OK) return rc;
  R4_PROF("router_bwd", static_cast<cudaStream_t>(stream_));
  R4_TRY(launch_router_bwd(scores, qlen, experts, top_k, ids, grad_route, escale, grad_scores, grad_escale,
                           static_cast<cudaStream_t>(stream_)));
  return RAWINT4_OK;
}

int rawint4_moe_lora_saved_preacts(const rawint4_moe_cfg* cfg, const void* workspace, size_t ws_bytes, int32_t* perm,
                                   float* g, float* u, int32_t* routed, void* stream_) {
  if (!cfg_ok(cfg) || !workspace || !perm || !g || !u || !routed) return RAWINT4_INVALID_ARGUMENT;
  const Layout L = make_layout(*cfg);
  if (ws_bytes < L.total) return RAWINT4_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream_);
  void* ws = const_cast<void*>(workspace);
  WsHeader h{};
  if (cudaStreamSynchronize(st) != cudaSuccess) return RAWINT4_CUDA_ERROR;
  if (cudaMemcpy(&h, at<WsHeader>(ws, L.hdr), sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return RAWINT4_CUDA_ERROR;
  if (h.magic != kWsMagic || h.saved != 1u) return RAWINT4_NO_SAVED_FORWARD;
  const size_t rows = (size_t)cfg->max_tokens * cfg->top_k;
  const size_t row_bytes = (size_t)cfg->inter * sizeof(float);
  if (cudaMemcpyAsync(perm, at<int32_t>(ws, L.perm), rows * sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(g, at<float>(ws, L.g), rows * row_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(u, at<float>(ws, L.u), rows * row_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return RAWINT4_CUDA_ERROR;
  *routed = h.routed;
  return RAWINT4_OK;
}

int rawint4_moe_set_wait_limit_ns(uint64_t ns) {
  g_wait_ns.store(ns == 0 ? 4000000000ull : (unsigned long long)ns);
  return RAWINT4_OK;
}

int rawint4_moe_lora_status(void* workspace, void* stream_, uint32_t* device_status) {
  if (!workspace || !device_status) return RAWINT4_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream_);
  WsHeader* hdr = static_cast<WsHeader*>(workspace);
  uint32_t v = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return RAWINT4_CUDA_ERROR;
  if (cudaMemcpy(&v, &hdr->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return RAWINT4_CUDA_ERROR;
  if (cudaMemset(&hdr->status, 0, sizeof(v)) != cudaSuccess) return RAWINT4_CUDA_ERROR;
  *device_status = v;
  return RAWINT4_OK;
}

int rawint4_decode(const uint8_t* q, const uint16_t* s, int64_t n, int64_t k, float* out_f32, uint16_t* out_f16,
                   void* stream_) {
  if (!q || !s || n < 0 || k < 0 || k % 32 != 0 || (!out_f32 && !out_f16)) return RAWINT4_INVALID_ARGUMENT;
  int sms = 0;
  int rc = check_device(&sms);
  if (rc != RAWINT4_OK) return rc;
  if (launch_decode(q, s, n, k, out_f32, out_f16, static_cast<cudaStream_t>(stream_)) != cudaSuccess)
    return RAWINT4_CUDA_ERROR;
  return RAWINT4_OK;
}

int rawint4_mxfp4_decode(const uint8_t* q, const uint8_t* s, int64_t n, int64_t k, float* out_f32, uint16_t* out_f16,
                         void* stream_) {
  if (!q || !s || n < 0 || k < 0 || k % 32 != 0 || (!out_f32 && !out_f16)) return RAWINT4_INVALID_ARGUMENT;
  int sms = 0;
  int rc = check_device(&sms);
  if (rc != RAWINT4_OK) return rc;
  if (launch_decode_mxfp4(q, s, n, k, out_f32, out_f16, static_cast<cudaStream_t>(stream_)) != cudaSuccess)
    return RAWINT4_CUDA_ERROR;
  return RAWINT4_OK;
}

int rawint4_moe_permute_workspace_size(int32_t qlen, int32_t top_k, int32_t experts, size_t* bytes) {
  if (!bytes || qlen < 0 || top_k < 1 || experts < 1 || experts > 4096 || (int64_t)qlen * top_k > (1 << 24))
    return RAWINT4_INVALID_ARGUMENT;
  const int32_t slots = qlen * top_k;
  *bytes = align_up(sizeof(WsHeader), kAlign) + align_up((size_t)max_tok_tiles(slots, experts) * 16, kAlign) +
           route_scratch_bytes(slots, experts);
  return RAWINT4_OK;
}

int rawint4_moe_permute(const int64_t* ids, int32_t qlen, int32_t top_k, int32_t experts, int32_t* offsets,
                        int32_t* perm, int32_t* inv, void* workspace, size_t ws_bytes, void* stream_) {
  size_t need = 0;
  if (rawint4_moe_permute_workspace_size(qlen, top_k, experts, &need) != RAWINT4_OK) return RAWINT4_INVALID_ARGUMENT;
  if (!offsets || !workspace || ws_bytes < need || reinterpret_cast<uintptr_t>(workspace) % kAlign) return RAWINT4_INVALID_ARGUMENT;
  if (qlen > 0 && (!ids || !perm || !inv)) return RAWINT4_INVALID_ARGUMENT;
  int sms = 0;
  int rc = check_device(&sms);
  if (rc != RAWINT4_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream_);
  const int32_t slots = qlen * top_k;
  WsHeader* hdr = static_cast<WsHeader*>(workspace);
  int4* tiles = at<int4>(workspace, align_up(sizeof(WsHeader), kAlign));
  int32_t* hist = at<int32_t>(workspace, align_up(sizeof(WsHeader), kAlign) +
                                             align_up((size_t)max_tok_tiles(slots, experts) * 16, kAlign));
  if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st) != cudaSuccess) return RAWINT4_CUDA_ERROR;
  {
    R4_PROF("route", st);
    R4_TRY(launch_route(ids, nullptr, qlen, top_k, experts, offsets, perm, inv, nullptr, tiles, hist, hdr, st));
  }
  if (slots > 0) {
    tail_fill_kernel<<<(slots + 255) / 256, 256, 0, st>>>(perm, offsets, experts, slots);
    R4_TRY(cudaGetLastError());
  }
  return RAWINT4_OK;
}

int rawint4_moe_dispatch_rows(const uint16_t* src, const int32_t* perm, int32_t n, int32_t top_k, int32_t width,
                              uint16_t* dst, void* stream) {
  if (n < 0 || top_k < 1 || width < 8 || width % 8 != 0 || (n > 0 && (!src || !perm || !dst)))
    return RAWINT4_INVALID_ARGUMENT;
  if (n == 0) return RAWINT4_OK;
  int sms = 0;
  const int rc = check_device(&sms);
  if (rc != RAWINT4_OK) return rc;
  return launch_dispatch_rows(src, perm, n, top_k, width, dst, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? RAWINT4_OK
             : RAWINT4_CUDA_ERROR;
}

int rawint4_moe_combine_slots(const uint16_t* src, const int32_t* inv, int32_t qlen, int32_t top_k, int32_t width,
                              uint16_t* out, void* stream) {
  if (qlen < 0 || top_k < 1 || width < 8 || width % 8 != 0 || (qlen > 0 && (!inv || !out)))
    return RAWINT4_INVALID_ARGUMENT;
  if (qlen == 0) return RAWINT4_OK;
  int sms = 0;
  const int rc = check_device(&sms);
  if (rc != RAWINT4_OK) return rc;
  return launch_combine_slots(src, inv, qlen, top_k, width, out, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? RAWINT4_OK
             : RAWINT4_CUDA_ERROR;
}

int rawint4_moe_gather_slots(const float* src, const int32_t* inv, int32_t n_slots, float* out, void* stream) {
  if (n_slots < 0 || (n_slots > 0 && (!inv || !out))) return RAWINT4_INVALID_ARGUMENT;
  if (n_slots == 0) return RAWINT4_OK;
  int sms = 0;
  const int rc = check_device(&sms);
  if (rc != RAWINT4_OK) return rc;
  return launch_gather_slots(src, inv, n_slots, out, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? RAWINT4_OK
             : RAWINT4_CUDA_ERROR;
}

}  // extern "C"
