// Host side of the C ABI declared in include/moe.h: argument checks, workspace layout, TMA
// descriptors and the launch sequence of the MoE-layer forward on the caller's stream.
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <initializer_list>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "gemm_splitk.cuh"
#include "gemm_swap_pair.cuh"
#include "gemm_tc.cuh"
#include "kernels_simt.cuh"

namespace moe {
namespace {

// ------------------------------------------------------------------ small helpers

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool all_aligned(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (!aligned16(p)) return false;
  return true;
}
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int cdiv(long a, long b) { return static_cast<int>((a + b - 1) / b); }

// k-split latent projections (decode-sized batches): at most this many splits, for at most this
// many rows.
constexpr int kMaxDenseSplits = 8;
constexpr int kMaxSplitRows = 64;

struct DeviceInfo {
  int sms = 0;
};

DeviceInfo& device_info() {
  static std::mutex mu;
  static DeviceInfo info[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  DeviceInfo& d = info[dev & 63];
  if (d.sms <= 0 &&
      cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    d.sms = 0;  // callers report MOE_ERR_CUDA rather than launch an empty grid
  return d;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 row-major [rows, cols] tensor, boxes of 64 columns x box_rows rows, 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

std::atomic<unsigned long long> g_launches{0};  // kernels this library has launched

// Status of the kernel launch(es) just issued; counts `n` launches.
moe_status_t last_launch(int n = 1) {
  g_launches.fetch_add(static_cast<unsigned long long>(n), std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Every kernel is launched with programmatic stream serialization: it may begin while the kernel
// before it on the stream finishes, and waits (pdl_wait) for that kernel's results before it reads
// anything an earlier kernel writes.  Errors surface through last_launch().
template <typename... KArgs, typename... Args>
void launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// The same launch in thread-block clusters of `cluster` CTAs along x.
template <typename... KArgs, typename... Args>
void launch_k_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, int cluster,
                      cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------------------ GEMM launcher

// Tuning knob: MOE_TAIL_M64=0 in the environment runs a group's last chunk of at most 64 rows as
// an M = 128 tile (padding rows multiplied) instead of M = 64 MMAs.
bool tail_m64_enabled() {
  const char* v = getenv("MOE_TAIL_M64");
  return !(v && v[0] == '0');
}

template <bool kSwap, int BN, int kEpi, int kStages>
moe_status_t launch_gemm(const void* X, long x_rows, const void* W, long w_rows,
                         const GemmParams& p, long max_tiles, cudaStream_t st) {
  using S = GemmShape<kSwap, BN, kEpi>;
  constexpr int smem = gemm_smem_bytes<kSwap, BN, kEpi, kStages>();
  static_assert(smem <= 232448, "shared memory budget");
  auto kern = gemm_tc_kernel<kSwap, BN, kEpi, kStages>;
  static std::once_flag once;  // the attribute is per function; set it once per process
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (attr_err != cudaSuccess) return MOE_ERR_CUDA;
  CUtensorMap tx, tw;
  // X is [x_rows, K], or [x_rows, x_k_period] when its k coordinate wraps (W then has K columns)
  const uint64_t x_cols = static_cast<uint64_t>(p.x_k_period > 0 ? p.x_k_period : p.K);
  if (!make_tmap(&tx, X, static_cast<uint64_t>(x_rows), x_cols, S::kXBoxRows))
    return MOE_ERR_CUDA;
  if (!make_tmap(&tw, W, static_cast<uint64_t>(w_rows), static_cast<uint64_t>(p.K), S::kWBoxRows))
    return MOE_ERR_CUDA;
  // Output map for the staged epilogue stores (boxes of 32 rows x 64 columns); where the output
  // cannot be described (unaligned base or row stride) the epilogue stores directly.
  GemmParams q = p;
  q.tail_m64 = (!kSwap && tail_m64_enabled()) ? 1 : 0;
  CUtensorMap to = tx;
  q.out_tma = stages_output<kSwap, kEpi>() &&
              make_tmap(&to, p.out, static_cast<uint64_t>(x_rows), static_cast<uint64_t>(p.Nout), 32);
  if (max_tiles <= 0) return MOE_OK;
  long grid = device_info().sms;
  if (grid <= 0) return MOE_ERR_CUDA;  // the SM count could not be read
  if (max_tiles < grid) grid = max_tiles;
  launch_k(kern, static_cast<unsigned>(grid), kGemmThreads, smem, st, tx, tw, to, q);
  return last_launch();
}

// CTA-pair variant: grid of whole clusters of 2.
template <int BN, int kEpi, int kStages>
moe_status_t launch_gemm_pair(const void* X, long x_rows, const void* W, long w_rows,
                              const GemmParams& p, long max_tiles, cudaStream_t st) {
  constexpr int smem = gemm_pair_smem_bytes<BN, kEpi, kStages>();
  static_assert(smem <= 232448, "shared memory budget");
  auto kern = gemm_tc_pair_kernel<BN, kEpi, kStages>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (attr_err != cudaSuccess) return MOE_ERR_CUDA;
  CUtensorMap tx, tw;
  if (p.x_k_period > 0) return MOE_ERR_UNSUPPORTED;  // the pair kernel has no wrapping X
  if (!make_tmap(&tx, X, static_cast<uint64_t>(x_rows), static_cast<uint64_t>(p.K), 128))
    return MOE_ERR_CUDA;
  if (!make_tmap(&tw, W, static_cast<uint64_t>(w_rows), static_cast<uint64_t>(p.K), BN / 2))
    return MOE_ERR_CUDA;
  GemmParams q = p;
  q.tail_m64 = 0;  // the pair kernel's tiles are 256 rows
  CUtensorMap to = tx;
  q.out_tma = make_tmap(&to, p.out, static_cast<uint64_t>(x_rows), static_cast<uint64_t>(p.Nout), 32);
  if (max_tiles <= 0) return MOE_OK;
  long pairs = device_info().sms / 2;
  if (pairs <= 0) return MOE_ERR_CUDA;  // the SM count could not be read
  if (max_tiles < pairs) pairs = max_tiles;
  launch_k(kern, static_cast<unsigned>(2 * pairs), kGemmThreads, smem, st, tx, tw, to, q);
  return last_launch();
}

// Swapped CTA-pair variant (prefill-sized expert groups): grid of whole clusters of 2.
template <int kEpi, int kStages>
moe_status_t launch_gemm_swap_pair(const void* X, long x_rows, const void* W, long w_rows,
                                   const GemmParams& p, long max_tiles, cudaStream_t st) {
  using S = SwapPairShape<kEpi>;
  constexpr int smem = gemm_swap_pair_smem_bytes<kEpi, kStages>();
  static_assert(smem <= 232448, "shared memory budget");
  auto kern = gemm_swap_pair_kernel<kEpi, kStages>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (attr_err != cudaSuccess) return MOE_ERR_CUDA;
  if (p.x_k_period > 0 || !p.seg) return MOE_ERR_UNSUPPORTED;
  CUtensorMap tx, tw;
  if (!make_tmap(&tx, X, static_cast<uint64_t>(x_rows), static_cast<uint64_t>(p.K), 128))
    return MOE_ERR_CUDA;
  if (!make_tmap(&tw, W, static_cast<uint64_t>(w_rows), static_cast<uint64_t>(p.K), S::kWBoxRows))
    return MOE_ERR_CUDA;
  if (max_tiles <= 0) return MOE_OK;
  long pairs = device_info().sms / 2;
  if (pairs <= 0) return MOE_ERR_CUDA;  // the SM count could not be read
  if (max_tiles < pairs) pairs = max_tiles;
  launch_k(kern, static_cast<unsigned>(2 * pairs), kGemmThreads, smem, st, tx, tw, p);
  return last_launch();
}

// Upper bound of the tile count of a grouped GEMM (each group adds at most one partial chunk).
long tile_bound(long rows, int G, int ch, int ft) { return (static_cast<long>(cdiv(rows, ch)) + G) * ft; }

enum class Orient { kNormal, kSwap, kPair, kSwapPair };

// Output-feature tile choice of the normal orientation: the widest of 256/128/64 dividing Nout
// (for SwiGLU the tile holds gate and up halves, so the output width per tile is BN/2).
int pick_bn_normal(int nout, bool dual) {
  const int div = dual ? 2 : 1;
  for (int bn : {256, 128, 64})
    if (!(dual && bn < 128) && nout % (bn / div) == 0) return bn;
  return 0;
}

// Grouped expert GEMM (or dense projection when seg == nullptr).
moe_status_t run_gemm(int epi, Orient o, int bn, const void* X, long x_rows, const void* W,
                      long w_rows, const GemmParams& p, cudaStream_t st) {
  const bool dual = epi == EPI_SWIGLU;
  if (o == Orient::kSwap) {
    const int ft = p.Nout / 128;
    const long mt = tile_bound(x_rows, p.G, bn, ft);
#define SW(BN_, E_, ST_) \
  if (bn == BN_ && epi == E_) return launch_gemm<true, BN_, E_, ST_>(X, x_rows, W, w_rows, p, mt, st);
    SW(16, EPI_SWIGLU, 6) SW(32, EPI_SWIGLU, 6) SW(64, EPI_SWIGLU, 5)
    SW(16, EPI_STORE, 10) SW(32, EPI_STORE, 9) SW(64, EPI_STORE, 8)
    SW(16, EPI_RELU, 10) SW(32, EPI_RELU, 9) SW(64, EPI_RELU, 8)
    SW(16, EPI_RESGATE, 10) SW(32, EPI_RESGATE, 9) SW(64, EPI_RESGATE, 8)
#undef SW
    return MOE_ERR_UNSUPPORTED;
  }
  if (o == Orient::kSwapPair) {
    const int fo = dual ? SwapPairShape<EPI_SWIGLU>::kFO : SwapPairShape<EPI_STORE>::kFO;
    if (p.Nout % fo) return MOE_ERR_UNSUPPORTED;
    const long pt = tile_bound(x_rows, p.G, 256, p.Nout / fo);
    if (epi == EPI_SWIGLU) return launch_gemm_swap_pair<EPI_SWIGLU, 4>(X, x_rows, W, w_rows, p, pt, st);
    if (epi == EPI_STORE) return launch_gemm_swap_pair<EPI_STORE, 4>(X, x_rows, W, w_rows, p, pt, st);
    if (epi == EPI_RELU) return launch_gemm_swap_pair<EPI_RELU, 4>(X, x_rows, W, w_rows, p, pt, st);
    return MOE_ERR_UNSUPPORTED;
  }
  const int fo = dual ? bn / 2 : bn;
  if (o == Orient::kPair) {
    const long pt = tile_bound(x_rows, p.G, 256, cdiv(p.Nout, fo));
#define PR(BN_, E_, ST_) \
  if (bn == BN_ && epi == E_) return launch_gemm_pair<BN_, E_, ST_>(X, x_rows, W, w_rows, p, pt, st);
    PR(256, EPI_SWIGLU, 6) PR(256, EPI_STORE, 6) PR(256, EPI_RELU, 6) PR(256, EPI_RESGATE, 6)
#undef PR
    return MOE_ERR_UNSUPPORTED;
  }
  const long mt = tile_bound(x_rows, p.G, 128, cdiv(p.Nout, fo));
#define NM(BN_, E_, ST_) \
  if (bn == BN_ && epi == E_) return launch_gemm<false, BN_, E_, ST_>(X, x_rows, W, w_rows, p, mt, st);
  NM(256, EPI_SWIGLU, 4) NM(128, EPI_SWIGLU, 6)
  NM(256, EPI_STORE, 4) NM(128, EPI_STORE, 6) NM(64, EPI_STORE, 8)
  NM(256, EPI_RELU, 4) NM(128, EPI_RELU, 6) NM(64, EPI_RELU, 8)
  NM(256, EPI_RESGATE, 4) NM(128, EPI_RESGATE, 6) NM(64, EPI_RESGATE, 8)
  NM(256, EPI_ROUTER, 4) NM(128, EPI_ROUTER, 6) NM(64, EPI_ROUTER, 8) NM(32, EPI_ROUTER, 8)
#undef NM
  return MOE_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ configuration checks

int expert_in(const moe_config_t& c) { return c.d_latent > 0 ? c.d_latent : c.d_model; }
int gu_rows(const moe_config_t& c) { return c.expert_act == MOE_ACT_SWIGLU ? 2 * c.d_ff : c.d_ff; }

moe_status_t check_cfg(const moe_config_t* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d_model <= 0 || c->d_latent < 0 || c->d_ff <= 0 || c->n_experts <= 0 ||
      c->top_k <= 0)
    return MOE_ERR_INVALID_ARG;
  if (c->top_k > c->n_experts) return MOE_ERR_INVALID_ARG;
  if (c->n_experts > kMaxExperts || c->top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (c->expert_act != MOE_ACT_RELU && c->expert_act != MOE_ACT_SWIGLU) return MOE_ERR_UNSUPPORTED;
  if (c->resid_mode < MOE_RESID_NONE || c->resid_mode > MOE_RESID_LITERAL) return MOE_ERR_UNSUPPORTED;
  if (c->gate_mode != MOE_GATE_SOFTMAX && c->gate_mode != MOE_GATE_SIGMOID) return MOE_ERR_UNSUPPORTED;
  if (c->router_f32 != 0 && c->router_f32 != 1) return MOE_ERR_INVALID_ARG;
  if (c->gate_mode == MOE_GATE_SIGMOID && !(c->logit_mult == c->logit_mult)) return MOE_ERR_INVALID_ARG;
  if ((c->input_norm != 0 && c->input_norm != 1) || (c->post_norm != 0 && c->post_norm != 1))
    return MOE_ERR_INVALID_ARG;
  if ((c->input_norm || c->post_norm) && !(c->eps_block >= 0.0f)) return MOE_ERR_INVALID_ARG;
  if ((c->input_norm || c->post_norm) && c->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (c->post_norm && c->d_latent == 0) return MOE_ERR_UNSUPPORTED;
  if (c->input_norm && c->d_model > 8192) return MOE_ERR_UNSUPPORTED;  // row kernels
  if (c->post_norm && c->d_model > 8192) return MOE_ERR_UNSUPPORTED;
  if (!(c->eps >= 0.0f) || !(c->tau > 0.0f) || !(c->resid_floor >= 0.0f)) return MOE_ERR_INVALID_ARG;
  if (static_cast<long>(c->T) * c->top_k > 0x7fffffffL / 2) return MOE_ERR_UNSUPPORTED;
  if (c->dtype == MOE_BF16) {
    if (c->d_model % 64 || c->d_latent % 64 || c->d_ff % 64) return MOE_ERR_UNSUPPORTED;
    if (expert_in(*c) > 8192) return MOE_ERR_UNSUPPORTED;  // row kernels hold a row in registers
    if (c->d_latent == 0 && c->resid_mode != MOE_RESID_NONE) return MOE_ERR_UNSUPPORTED;
    if (c->pre_norm && c->d_latent == 0) return MOE_ERR_UNSUPPORTED;
  } else {
    if (c->d_latent != 0 || c->pre_norm || c->resid_mode != MOE_RESID_NONE) return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

size_t dsize(const moe_config_t& c) { return c.dtype == MOE_BF16 ? 2 : 4; }
int nchunks(const moe_config_t& c) { return cdiv(c.T, kPermChunk); }

struct Workspace {
  size_t idx, w, logits, z_raw, offsets, perm, inv, counts, x_perm, act, y, u_norm, b, ss, total;
};

int sumsq_parts(const moe_config_t& c);
constexpr int kMaxFusedSsParts = 32;  // moe_layer_forward passes row partials up to this many

Workspace layout(const moe_config_t& c) {
  Workspace L{};
  const size_t TK = static_cast<size_t>(c.T) * c.top_k, E = expert_in(c), ds = dsize(c);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  L.idx = take(TK * 4);
  L.w = take(TK * 4);
  L.logits = take(static_cast<size_t>(c.T) * c.n_experts * 4);
  L.z_raw = take(c.d_latent > 0 ? static_cast<size_t>(c.T) * c.d_latent * ds : 0);
  L.offsets = take((c.n_experts + 1) * 4);
  L.perm = take(TK * 4);
  L.inv = take(TK * 4);
  L.counts = take(static_cast<size_t>(nchunks(c)) * c.n_experts * 4);
  L.x_perm = take(TK * E * ds);
  L.act = take(TK * c.d_ff * ds);
  L.y = take(c.d_latent > 0 ? static_cast<size_t>(c.T) * E * ds : 0);
  L.u_norm = take(c.input_norm ? static_cast<size_t>(c.T) * c.d_model * ds : 0);
  L.b = take(c.post_norm ? static_cast<size_t>(c.T) * c.d_model * ds : 0);
  L.ss = take(c.expert_norm && c.dtype == MOE_BF16 ? TK * sumsq_parts(c) * 4 : 0);
  L.total = o;
  return L;
}

template <typename T>
T* at(void* base, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(base) + off); }

// CTA-pair 256-row tiles (same values as the 1-SM tiles).  For expert groups they are off by
// default: groups are ragged, a group's last 256-row tile is mostly padding, and under the power
// cap those steps measured slower than the 1-SM 128 x 256 tiles.  Dense projections over at least
// kDensePairMinRows rows have no such tails, and there the pair tiles read a third fewer operand
// bytes per MMA from L2: at prefill latent down took 0.89-0.92 against 0.96-0.98 ms and latent up
// 0.91-0.94 against 1.02-1.04 ms, with the same bits.  Tuning knob: MOE_GEMM_PAIR=1 in the
// environment also puts large expert groups and dense projections from 256 rows on the pair
// tiles; MOE_GEMM_PAIR=0 puts nothing on them.
constexpr long kDensePairMinRows = 2048;
int pair_tiles_knob() {  // 1: on everywhere, 0: off everywhere, -1: default
  const char* v = getenv("MOE_GEMM_PAIR");
  if (v && v[0] == '1') return 1;
  if (v && v[0] == '0') return 0;
  return -1;
}
bool pair_tiles_enabled() { return pair_tiles_knob() == 1; }

// Grouped-GEMM orientation for the experts from the mean rows per expert.
int expert_in_width(const moe_config_t& c) { return c.d_latent > 0 ? c.d_latent : c.d_model; }

// Expert tilings for groups too large for the swapped 1-SM tiles (more than 48 rows per expert on
// average).  The 1-SM tiles put 128 token rows on the MMA's M side, so a group's last chunk pays for
// up to 127 padding rows; the swapped CTA-pair tiles put the tokens on N, cut to 16 rows.  Measured
// inside the layer:
//   - at 512 rows per expert (the prefill batch) both GEMMs take about as long either way; the
//     pair tiles do more work per clock but spend more energy per launch under the 1 kW cap;
//   - at about 128 rows per expert with 1 MB experts (the Shazeer batch, d 512, hidden 1024: the
//     128-row chunks do 1.48x the MMA work) the down GEMM is faster on the pair tiles (0.076
//     against 0.088 ms), while the first GEMM, whose reduction is only 512 deep, is slower (0.094
//     against 0.081 ms);
//   - at 64 and 128 rows per expert with the Muse experts (reductions 4096 deep) the pair tiles
//     are slower for both GEMMs (down 1.69 against 1.41 ms and 1.84 against 1.70 ms): there the
//     weight stream, not the MMA work, sets the pace.
// So by default the down GEMM takes the pair tiles from 49 to 256 mean rows per expert when its
// reduction is at most 1024 deep.  Tuning knob: MOE_EXPERT_TILES=swap_pair (both GEMMs on the pair
// tiles for every group above 48 rows) or MOE_EXPERT_TILES=normal (neither).  The values are the
// same up to the fp32 summation inside the tensor core.
enum class TilePref { kDefault, kSwapPair, kNormal };
TilePref expert_tile_pref() {
  const char* v = getenv("MOE_EXPERT_TILES");
  if (v && v[0] == 's') return TilePref::kSwapPair;
  if (v && v[0] == 'n') return TilePref::kNormal;
  return TilePref::kDefault;
}

constexpr double kSwapMaxMeanRows = 48.0;      // swapped 1-SM tiles up to this mean
constexpr double kDownPairMaxMeanRows = 256.0; // down GEMM on the pair tiles up to this mean
constexpr int kDownPairMaxK = 1024;            // ... and up to this reduction depth

// `down` selects the rule of the second expert GEMM (a -> o), `dual` the SwiGLU pairing of the first.
void pick_expert_orient(const moe_config_t& c, int nout, bool dual, bool down, Orient* o, int* bn) {
  const double mean_rows = static_cast<double>(c.T) * c.top_k / c.n_experts;
  const TilePref pref = expert_tile_pref();
  const int fo = dual ? SwapPairShape<EPI_SWIGLU>::kFO : SwapPairShape<EPI_STORE>::kFO;
  const bool pair_ok = !pair_tiles_enabled() && nout % fo == 0;
  if (nout % 128 == 0 && mean_rows <= kSwapMaxMeanRows) {
    *o = Orient::kSwap;
    *bn = mean_rows <= 12.0 ? 16 : (mean_rows <= 24.0 ? 32 : 64);
  } else if (pair_ok && (pref == TilePref::kSwapPair ||
                         (pref == TilePref::kDefault && down && c.d_ff <= kDownPairMaxK &&
                          mean_rows <= kDownPairMaxMeanRows))) {
    // tokens on the MMA's N side, cut to 16 rows, on CTA pairs
    *o = Orient::kSwapPair;
    *bn = 256;
  } else {
    *bn = pick_bn_normal(nout, dual);
    // 256-row CTA-pair tiles once groups are large enough to fill them
    *o = (pair_tiles_enabled() && *bn == 256 && mean_rows >= 192.0) ? Orient::kPair
                                                                     : Orient::kNormal;
  }
}

// Partial sums of squares per expert-output row that the expert down GEMM writes (row_sumsq):
// one per 256/128/64-column feature tile in the normal (and CTA-pair) orientation, one per CTA's
// 128 features in the swapped CTA-pair orientation, one per 32-feature warp slice of each
// 128-feature tile in the swapped orientation.
int sumsq_parts(const moe_config_t& c) {
  Orient o;
  int bn;
  pick_expert_orient(c, expert_in_width(c), false, true, &o, &bn);
  if (bn <= 0) return 1;
  if (o == Orient::kSwapPair) return expert_in_width(c) / 128;  // one per CTA's 128 features
  return o == Orient::kSwap ? expert_in_width(c) / 128 * 4 : expert_in_width(c) / bn;
}

// Dense projections: CTA-pair tiles for a 256-wide feature tile over at least kDensePairMinRows
// rows (from 256 rows with MOE_GEMM_PAIR=1).
Orient dense_orient(int rows, int bn) {
  if (bn != 256) return Orient::kNormal;
  const int knob = pair_tiles_knob();
  if (knob == 1) return rows >= 256 ? Orient::kPair : Orient::kNormal;
  return (knob == -1 && rows >= kDensePairMinRows) ? Orient::kPair : Orient::kNormal;
}

// Dense projection (latent down / up) over `rows` activation rows into `nout` features.  Up to
// 256 rows the weight stream decides the time, and the normal orientation would spread it over
// only Nout/256 tiles per 128-row chunk (16 CTAs for the 4096-wide latent at T=64).  The swapped
// orientation puts 128 weight rows on the MMA's M side and the activation rows on N: Nout/128
// tiles per chunk of BN rows.  BN is the widest of 64/32/16 that still gives two thirds of the
// SMs a tile (narrower chunks re-read each weight tile from L2, not from HBM).
void pick_dense(int rows, int nout, Orient* o, int* bn) {
  if (rows <= 256 && nout % 128 == 0) {
    *o = Orient::kSwap;
    const long ft = nout / 128;
    int b = 64;
    while (b > 16 && (b / 2 >= rows || cdiv(rows, b) * ft * 3 < 2L * device_info().sms)) b /= 2;
    *bn = b;
    return;
  }
  *bn = pick_bn_normal(nout, false);
  *o = dense_orient(rows, *bn);
}

// Dense projections over at most 64 rows split their reduction: with S k-ranges the swapped tiles
// number Nout/128 * S, each streaming 1/S of a weight tile, and the S CTAs of a feature tile (one
// thread-block cluster) add their fp32 partial tiles in split order in distributed shared memory
// before the epilogue.  S is the largest power of two up to kMaxDenseSplits whose tiles still fit
// on the SMs at once and divides the k-blocks.
int dense_k_splits(int rows, int nout, int K) {
  if (rows > kMaxSplitRows || nout % 128 != 0) return 1;
  const long ft = nout / 128;
  const int kb = K / 64;
  int sp = 1;
  while (sp < kMaxDenseSplits && ft * sp * 2 <= device_info().sms && kb % (sp * 2) == 0) sp *= 2;
  return sp;
}

// Dense projection of at most kMaxSplitRows rows with its reduction split over clusters of
// `splits` CTAs, which add their partial tiles in distributed shared memory.
template <int kEpi>
moe_status_t launch_gemm_splitk(const void* X, long x_rows, const void* W, long w_rows,
                                const GemmParams& p, int splits, cudaStream_t st) {
  constexpr int smem = gemm_splitk_smem_bytes();
  static_assert(smem <= 232448, "shared memory budget");
  auto kern = gemm_splitk_cluster_kernel<kEpi>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (attr_err != cudaSuccess) return MOE_ERR_CUDA;
  if (x_rows > kSplitBN || splits < 2 || splits > kSplitMaxCluster || p.Nout % 128 ||
      (p.K / 64) % splits)
    return MOE_ERR_UNSUPPORTED;
  CUtensorMap tx, tw;
  if (!make_tmap(&tx, X, static_cast<uint64_t>(x_rows), static_cast<uint64_t>(p.K), kSplitBN))
    return MOE_ERR_CUDA;
  if (!make_tmap(&tw, W, static_cast<uint64_t>(w_rows), static_cast<uint64_t>(p.K), 128))
    return MOE_ERR_CUDA;
  launch_k_cluster(kern, static_cast<unsigned>(p.Nout / 128 * splits), kGemmThreads, smem, splits,
                   st, tx, tw, p);
  return last_launch();
}

// ------------------------------------------------------------------ steps

// Tokens up to which the router runs as a many-CTA logits kernel + a top-k kernel (a single
// GEMM tile would leave most SMs idle while it streams the router weights).
constexpr int kSmallRouterMaxT = 256;

// Schedule of a dense projection (one group of x_rows rows against Nw weight rows): when the
// activations outnumber the weight rows, feature tiles run fastest so each activation chunk is
// read from HBM once while the weights stay in L2.  (Every tile reduces over k in the same
// order, so a token's result does not depend on where it sits in the batch.)
void dense_schedule(GemmParams& p, long x_rows) {
  p.tile_order = x_rows > p.Nw ? TILE_FEATURE_FASTEST : TILE_CHUNK_FASTEST;
}

moe_status_t do_route(const moe_config_t& c, const void* u, const void* w_router,
                      const float* bias, const float* sel_bias, float* logits, int32_t* idx,
                      float* w, cudaStream_t st, float* logits_scratch = nullptr) {
  if (c.T == 0) return MOE_OK;
  const bool sig = c.gate_mode == MOE_GATE_SIGMOID;
  const float mult = sig ? c.logit_mult : 1.0f;
  if (c.dtype == MOE_F32) {
    const int warps = 4;
    launch_k(router_f32_kernel, cdiv(c.T, warps), 32 * warps, 0, st,
        static_cast<const float*>(u), static_cast<const float*>(w_router), bias, c.T, c.d_model,
        c.n_experts, c.top_k, c.routed_scale, c.gate_mode, mult, sel_bias, logits, idx, w);
    return last_launch();
  }
  const int wk = c.router_f32 ? 3 * c.d_model : c.d_model;  // router weight row length
  float* lbuf = logits ? logits : logits_scratch;
  const size_t small_smem = static_cast<size_t>(kRouterTok) * c.d_model * 2;
  if (c.T <= kSmallRouterMaxT && lbuf && small_smem <= 200 * 1024) {
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [] {
      attr = cudaFuncSetAttribute(router_logits_small_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    });
    if (attr != cudaSuccess) return MOE_ERR_CUDA;
    dim3 grid(cdiv(c.n_experts, kRouterExp), cdiv(c.T, kRouterTok));
    launch_k(router_logits_small_kernel, grid, kRouterThreads, small_smem, st,
        static_cast<const uint16_t*>(u), static_cast<const uint16_t*>(w_router), bias, c.T,
        c.d_model, c.n_experts, wk, mult, lbuf);
    launch_k(topk_rows_kernel, cdiv(c.T, 8), 256, 0, st, lbuf, c.T, c.n_experts, c.top_k,
                                                    c.routed_scale, c.gate_mode, sel_bias, idx, w);
    return last_launch(2);
  }
  // With a logits buffer (the caller's, or the layer's workspace) the GEMM only stores the
  // pre-activation logits and a warp per token selects the top-k; without one, the GEMM's
  // epilogue selects from the accumulators itself (k passes over each row).  Selecting in the
  // epilogue with a buffer present was measured slower, with these k passes (0.089 against 0.033
  // ms of route for the Shazeer batch) and with a single pass keeping the best k in registers
  // (0.124 against 0.040 ms; 0.27 against 0.16 ms at prefill: the insertion into the k-list runs
  // predicated for every column in each thread), while the warp-per-token kernel spreads the
  // selection over every SM.
  const bool split = lbuf != nullptr;
  GemmParams p{};
  p.G = 1;
  p.M = c.T;
  p.K = wk;
  p.x_k_period = c.router_f32 ? c.d_model : 0;
  p.Nw = c.n_experts;
  p.Nout = c.n_experts;
  p.logits = split ? lbuf : nullptr;
  p.router_select = split ? 0 : 1;
  p.topk_idx = idx;
  p.topk_w = w;
  p.bias = bias;
  p.top_k = c.top_k;
  p.routed_scale = c.routed_scale;
  p.gate_mode = c.gate_mode;
  p.logit_mult = mult;
  p.sel_bias = sel_bias;
  dense_schedule(p, c.T);
  int bn = c.n_experts <= 32 ? 32 : c.n_experts <= 64 ? 64 : c.n_experts <= 128 ? 128 : 256;
  // When only storing logits, a batch with few row tiles splits the experts over narrower
  // tiles, so that more of the SMs take part (the selection that follows sees whole rows).
  if (split) {
    const long chunks = cdiv(c.T, 128);
    while (bn > 32 && chunks * cdiv(c.n_experts, bn) * 2 <= device_info().sms) bn /= 2;
  }
  moe_status_t s = run_gemm(EPI_ROUTER, Orient::kNormal, bn, u, c.T, w_router, c.n_experts, p, st);
  if (s != MOE_OK || !split) return s;
  launch_k(topk_rows_kernel, cdiv(c.T, 8), 256, 0, st, lbuf, c.T, c.n_experts, c.top_k, c.routed_scale,
                                                  c.gate_mode, sel_bias, idx, w);
  return last_launch();
}

moe_status_t do_dispatch_rows(const moe_config_t& c, const int32_t* inv, const void* x,
                              const float* gamma_pre, void* x_perm, cudaStream_t st);

moe_status_t do_permute(const moe_config_t& c, const int32_t* idx, int32_t* offsets,
                        int32_t* perm, int32_t* inv, const void* x, const float* gamma_pre,
                        void* x_perm, int32_t* counts, cudaStream_t st) {
  const int n = c.n_experts, k = c.top_k, nc = nchunks(c);
  if (c.T == 0) {
    cudaMemsetAsync(offsets, 0, (n + 1) * sizeof(int32_t), st);
    return last_launch(0);
  }
  if (c.dtype == MOE_BF16 && static_cast<long>(c.T) * k <= kSmallDispatchSlots) {
    // small batch: indices, offsets and (with x) the row scatter in one launch
    const int E = c.d_latent > 0 ? c.d_latent : c.d_model;
    const int nvec = E / 8;
    const int threads = nvec >= 256 ? 256 : std::max(32, ((nvec + 31) / 32) * 32);
    const int vec = cdiv(nvec, threads);
    const uint16_t* xs = static_cast<const uint16_t*>(x);
    uint16_t* xp = static_cast<uint16_t*>(x_perm);
#define SD(V) launch_k(dispatch_small_bf16_kernel<V>, c.T, threads, 0, st, idx, c.T, k, n, xs, E, \
      gamma_pre, c.eps, offsets, perm, inv, xp)
    switch (vec) {
      case 1: SD(1); break;
      case 2: SD(2); break;
      case 3:
      case 4: SD(4); break;
      default: return MOE_ERR_UNSUPPORTED;
    }
#undef SD
    return last_launch();
  }
  launch_k(perm_count_kernel, nc, 256, 0, st, idx, c.T, k, n, counts);
  launch_k(perm_scan_kernel, 1, kMaxExperts, 0, st, counts, nc, n, offsets);
  launch_k(perm_rank_kernel, nc, 32, 0, st, idx, c.T, k, n, counts, offsets, perm, inv);
  moe_status_t s = last_launch(3);
  if (s != MOE_OK || !x) return s;
  return do_dispatch_rows(c, inv, x, gamma_pre, x_perm, st);
}

moe_status_t do_dispatch_rows(const moe_config_t& c, const int32_t* inv, const void* x,
                              const float* gamma_pre, void* x_perm, cudaStream_t st) {
  const int k = c.top_k;
  const int E = c.d_latent > 0 ? c.d_latent : c.d_model;
  if (c.dtype == MOE_F32) {
    launch_k(scatter_rows_f32_kernel<float>, c.T, 128, 0, st, static_cast<const float*>(x), E, k, inv,
                                                        static_cast<float*>(x_perm));
    return last_launch();
  }
  const int nvec = E / 8;
  const int threads = nvec >= 256 ? 256 : ((nvec + 31) / 32) * 32;
  const int vec = cdiv(nvec, threads);
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  uint16_t* xp = static_cast<uint16_t*>(x_perm);
  switch (vec) {
    case 1: launch_k(scatter_rows_bf16_kernel<1>, c.T, threads, 0, st, xs, E, k, inv, gamma_pre, c.eps, xp); break;
    case 2: launch_k(scatter_rows_bf16_kernel<2>, c.T, threads, 0, st, xs, E, k, inv, gamma_pre, c.eps, xp); break;
    case 3:
    case 4: launch_k(scatter_rows_bf16_kernel<4>, c.T, threads, 0, st, xs, E, k, inv, gamma_pre, c.eps, xp); break;
    default: return MOE_ERR_UNSUPPORTED;
  }
  return last_launch();
}

// ------------------------------------------------------------------ stage timing

struct Profiler {
  std::vector<cudaEvent_t> ev;  // max_calls x (MOE_PROFILE_STAGES + 1)
  int max_calls = 0, calls = 0;
  bool active = false;
};

Profiler& prof() {
  static Profiler p;
  return p;
}

constexpr int kMarks = MOE_PROFILE_STAGES + 1;

// Stage names of the forward, for the NVTX ranges a profiler's timeline shows around each stage's
// launches (a range per stage, from this mark to the next).
constexpr const char* kStageNames[MOE_PROFILE_STAGES] = {
    "moe.route", "moe.latent_down", "moe.dispatch", "moe.expert_gate_up", "moe.expert_down",
    "moe.combine", "moe.latent_up"};

void prof_mark(cudaStream_t st, int i) {
  Profiler& p = prof();
  if (p.active && p.calls < p.max_calls) cudaEventRecord(p.ev[p.calls * kMarks + i], st);
  if (i > 0) nvtxRangePop();
  if (i < MOE_PROFILE_STAGES) nvtxRangePushA(kStageNames[i]);
}

void prof_next_call() {
  Profiler& p = prof();
  if (p.active && p.calls < p.max_calls) ++p.calls;
}

constexpr size_t kL2KeepBytes = 80u << 20;  // expert activations kept in L2, at most

moe_status_t do_experts(const moe_config_t& c, const void* x_perm, const int32_t* offsets,
                        const void* w_gu, const void* w_down, const float* gamma_e,
                        void* out_perm, void* act, cudaStream_t st, bool mark = false,
                        float* row_ss = nullptr) {
  const long TK = static_cast<long>(c.T) * c.top_k;
  if (TK == 0) return MOE_OK;
  const int E = expert_in(c), H = c.d_ff, n = c.n_experts;
  if (c.dtype == MOE_F32) {
    const size_t smem = static_cast<size_t>(E + H) * sizeof(float);
    if (smem > 48 * 1024) return MOE_ERR_UNSUPPORTED;
    launch_k(expert_ffn_f32_kernel, static_cast<unsigned>(TK), 128, smem, st,
        static_cast<const float*>(x_perm), offsets, n, E, H, c.expert_act,
        static_cast<const float*>(w_gu), static_cast<const float*>(w_down),
        c.expert_norm ? gamma_e : nullptr, static_cast<float*>(out_perm));
    return last_launch();
  }
  const bool swiglu = c.expert_act == MOE_ACT_SWIGLU;
  // When the expert activation fits in L2 next to the weights in flight, the GEMMs stream their
  // weights as evict-first lines and keep their outputs (the activation the down GEMM reads, the
  // rows the combine reads) as evict-last lines, so the activation does not go out to DRAM and
  // back.
  const int hints = static_cast<size_t>(TK) * H * 2 <= kL2KeepBytes ? 1 : 0;
  // first GEMM: x_perm [TK, E] x W_gu[e]^T -> act [TK, H]
  GemmParams p1{};
  p1.l2_hints = hints;
  p1.seg = offsets;
  p1.G = n;
  p1.K = E;
  p1.Nw = gu_rows(c);
  p1.Nout = H;
  p1.out = act;
  Orient o1;
  int bn1;
  pick_expert_orient(c, H, swiglu, false, &o1, &bn1);
  if (bn1 == 0) return MOE_ERR_UNSUPPORTED;
  moe_status_t s = run_gemm(swiglu ? EPI_SWIGLU : EPI_RELU, o1, bn1, x_perm, TK, w_gu,
                            static_cast<long>(n) * p1.Nw, p1, st);
  if (s != MOE_OK) return s;
  if (mark) prof_mark(st, 4);
  // second GEMM: act [TK, H] x W_down[e]^T -> out [TK, E] (scaled by 1 + gamma for I_gamma)
  GemmParams p2{};
  p2.l2_hints = hints;
  p2.seg = offsets;
  p2.G = n;
  p2.K = H;
  p2.Nw = E;
  p2.Nout = E;
  p2.out = out_perm;
  p2.gamma = c.expert_norm ? gamma_e : nullptr;
  p2.row_ss = c.expert_norm ? row_ss : nullptr;
  p2.ss_parts = sumsq_parts(c);
  Orient o2;
  int bn2;
  pick_expert_orient(c, E, false, true, &o2, &bn2);
  if (bn2 == 0) return MOE_ERR_UNSUPPORTED;
  return run_gemm(EPI_STORE, o2, bn2, act, TK, w_down, static_cast<long>(n) * E, p2, st);
}

constexpr int kBulkCombineMinT = 1024;        // tokens from which the bulk-copy combine runs
constexpr int kBulkCombineSmem = 220 * 1024;   // its shared-memory ring, at most
constexpr int kBulkCombineMinBytes = 32 * 1024; // expert-row bytes of a token, at least

moe_status_t do_combine(const moe_config_t& c, const void* s, const int32_t* inv,
                        const float* w, void* y, cudaStream_t st, const float* row_ss = nullptr) {
  if (c.T == 0) return MOE_OK;
  const int E = expert_in(c);
  if (c.dtype == MOE_F32) {
    launch_k(combine_f32_kernel, c.T, 128, 0, st, static_cast<const float*>(s), E, c.top_k, inv, w,
                                            c.expert_norm, c.eps, static_cast<float*>(y));
    return last_launch();
  }
  const int nvec = E / 8;
  const int threads = nvec >= kCombineMaxThreads ? kCombineMaxThreads : ((nvec + 31) / 32) * 32;
  const int vec = cdiv(nvec, threads);
  const uint16_t* sp = static_cast<const uint16_t*>(s);
  uint16_t* yp = static_cast<uint16_t*>(y);
  // Prefill-sized batches of wide rows: one persistent CTA per SM with the expert rows (and their
  // partial sums of squares) brought in by bulk copies, when the row partials are given or no norm
  // is taken and at least two tokens' rows fit in shared memory.  (Narrow rows keep the per-token
  // kernel: there a token's copies are too small to amortise the ring's per-token handshakes.)
  const int parts_b = row_ss && c.expert_norm ? sumsq_parts(c) : 0;
  if (c.T >= kBulkCombineMinT && static_cast<long>(c.top_k) * E * 2 >= kBulkCombineMinBytes &&
      (parts_b * 4) % 16 == 0 && (!c.expert_norm || row_ss)) {
    const BulkCombineStage B = bulk_combine_stage(E, c.top_k, parts_b);
    const int nst = std::min(8, (kBulkCombineSmem - 128 - 16 * 8) / B.bytes);
    if (nst >= 2) {
      const size_t smem = 128 + static_cast<size_t>(nst) * B.bytes + 16 * static_cast<size_t>(nst);
      static std::once_flag once;
      static cudaError_t attr = cudaSuccess;
      std::call_once(once, [] {
        attr = cudaFuncSetAttribute(combine_bf16_bulk_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kBulkCombineSmem);
      });
      if (attr != cudaSuccess) return MOE_ERR_CUDA;
      const int grid = std::min(c.T, std::max(device_info().sms, 1));
      launch_k(combine_bf16_bulk_kernel, grid, kBulkCombineConsumers + 32, smem, st,
          sp, E, c.top_k, inv, w, row_ss, parts_b, c.expert_norm, c.eps, yp, c.T, nst);
      return last_launch();
    }
  }
  if (row_ss && c.expert_norm) {
    const int parts = sumsq_parts(c);
    switch (vec) {
      case 1: launch_k(combine_bf16_ss_kernel<1>, c.T, threads, 0, st, sp, E, c.top_k, inv, w, row_ss, parts, c.eps, yp); break;
      case 2: launch_k(combine_bf16_ss_kernel<2>, c.T, threads, 0, st, sp, E, c.top_k, inv, w, row_ss, parts, c.eps, yp); break;
      default: return MOE_ERR_UNSUPPORTED;  // E <= 8192: at most 2 vectors per thread
    }
    return last_launch();
  }
  switch (vec) {
    case 1: launch_k(combine_bf16_kernel<1>, c.T, threads, 0, st, sp, E, c.top_k, inv, w, c.expert_norm, c.eps, yp); break;
    case 2: launch_k(combine_bf16_kernel<2>, c.T, threads, 0, st, sp, E, c.top_k, inv, w, c.expert_norm, c.eps, yp); break;
    default: return MOE_ERR_UNSUPPORTED;  // E <= 8192: at most 2 vectors per thread
  }
  return last_launch();
}

moe_status_t do_latent_down(const moe_config_t& c, const void* u, const void* p_down, void* z,
                            cudaStream_t st) {
  if (c.T == 0) return MOE_OK;
  GemmParams p{};
  p.G = 1;
  p.M = c.T;
  p.K = c.d_model;
  p.Nw = c.d_latent;
  p.Nout = c.d_latent;
  p.out = z;
  dense_schedule(p, c.T);
  const int splits = dense_k_splits(c.T, c.d_latent, c.d_model);
  if (splits > 1) return launch_gemm_splitk<EPI_STORE>(u, c.T, p_down, c.d_latent, p, splits, st);
  Orient o;
  int bn;
  pick_dense(c.T, c.d_latent, &o, &bn);
  if (bn == 0) return MOE_ERR_UNSUPPORTED;
  return run_gemm(EPI_STORE, o, bn, u, c.T, p_down, c.d_latent, p, st);
}

moe_status_t do_latent_up(const moe_config_t& c, const void* y, const void* p_up, const void* r,
                          const float* g, void* out, cudaStream_t st) {
  if (c.T == 0) return MOE_OK;
  GemmParams p{};
  p.G = 1;
  p.M = c.T;
  p.K = c.d_latent;
  p.Nw = c.d_model;
  p.Nout = c.d_model;
  p.out = out;
  p.resid = static_cast<const uint16_t*>(r);
  p.gparam = g;
  p.tau = c.tau;
  p.floor_ = c.resid_floor;
  p.resid_mode = c.resid_mode;
  dense_schedule(p, c.T);
  const int splits = dense_k_splits(c.T, c.d_model, c.d_latent);
  if (splits > 1) return launch_gemm_splitk<EPI_RESGATE>(y, c.T, p_up, c.d_model, p, splits, st);
  Orient o;
  int bn;
  pick_dense(c.T, c.d_model, &o, &bn);
  if (bn == 0) return MOE_ERR_UNSUPPORTED;
  return run_gemm(EPI_RESGATE, o, bn, y, c.T, p_up, c.d_model, p, st);
}

// Workspace of moe_noisy_gate: clean and noise logits, scratch routing of the two logit passes,
// per-warp partial sums.
struct GateWorkspace {
  size_t l, m, idx, w, pi, pl, total;
  int nparts;
};
GateWorkspace gate_layout(const moe_config_t& c) {
  GateWorkspace L{};
  const size_t Tn = static_cast<size_t>(c.T) * c.n_experts, Tk = static_cast<size_t>(c.T) * c.top_k;
  const int warps = cdiv(c.T, kGateTokensPerWarp);
  L.nparts = cdiv(warps, 4) * 4;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  L.l = take(Tn * 4);
  L.m = take(Tn * 4);
  L.idx = take(Tk * 4);
  L.w = take(Tk * 4);
  L.pi = take(static_cast<size_t>(L.nparts) * c.n_experts * 4);
  L.pl = take(static_cast<size_t>(L.nparts) * c.n_experts * 4);
  L.total = o;
  return L;
}

// Launch shape of the one-CTA-per-row kernels for a row of D bf16 values.
bool row_launch(int D, int* threads, int* vec) {
  const int nvec = D / 8;
  *threads = nvec >= 256 ? 256 : ((nvec + 31) / 32) * 32;
  *vec = cdiv(nvec, *threads);
  if (*vec == 3) *vec = 4;
  return *vec <= 4;
}

moe_status_t do_input_norm(const moe_config_t& c, const void* r, const float* gamma_in, void* u,
                           cudaStream_t st) {
  if (c.T == 0) return MOE_OK;
  int threads, vec;
  if (!row_launch(c.d_model, &threads, &vec)) return MOE_ERR_UNSUPPORTED;
  const uint16_t* x = static_cast<const uint16_t*>(r);
  uint16_t* o = static_cast<uint16_t*>(u);
  switch (vec) {
    case 1: launch_k(rownorm_centered_bf16_kernel<1>, c.T, threads, 0, st, x, c.d_model, gamma_in, c.eps_block, o); break;
    case 2: launch_k(rownorm_centered_bf16_kernel<2>, c.T, threads, 0, st, x, c.d_model, gamma_in, c.eps_block, o); break;
    default: launch_k(rownorm_centered_bf16_kernel<4>, c.T, threads, 0, st, x, c.d_model, gamma_in, c.eps_block, o); break;
  }
  return last_launch();
}

moe_status_t do_resid_update(const moe_config_t& c, const void* b, const void* r,
                             const float* gamma_post, const float* g, void* out, cudaStream_t st) {
  if (c.T == 0) return MOE_OK;
  int threads, vec;
  if (!row_launch(c.d_model, &threads, &vec)) return MOE_ERR_UNSUPPORTED;
  const uint16_t* bp = static_cast<const uint16_t*>(b);
  const uint16_t* rp = static_cast<const uint16_t*>(r);
  uint16_t* o = static_cast<uint16_t*>(out);
#define RU(V) launch_k(resid_update_bf16_kernel<V>, c.T, threads, 0, st, bp, rp, c.d_model, gamma_post, \
      c.eps_block, g, c.resid_mode, c.tau, c.resid_floor, o)
  switch (vec) {
    case 1: RU(1); break;
    case 2: RU(2); break;
    default: RU(4); break;
  }
#undef RU
  return last_launch();
}

// Host-side checks of a whole-layer forward (nothing is launched when they fail).  T == 0 passes.
moe_status_t check_forward(const moe_config_t* cfg, const moe_weights_t* w, const void* u,
                           const void* r, const void* out, const float* logits_out,
                           const int32_t* topk_idx_out, const float* topk_w_out,
                           const void* workspace, size_t workspace_bytes) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  const moe_config_t& c = *cfg;
  if (!w) return MOE_ERR_INVALID_ARG;
  if (c.T == 0) return MOE_OK;
  const bool latent = c.d_latent > 0;
  if ((!u && !c.input_norm) || !out || !w->w_router || !w->w_gu || !w->w_down)
    return MOE_ERR_INVALID_ARG;
  if (c.input_norm && (!r || !w->gamma_in)) return MOE_ERR_INVALID_ARG;
  if (c.post_norm && !w->gamma_post) return MOE_ERR_INVALID_ARG;
  if (latent && (!w->p_down || !w->p_up)) return MOE_ERR_INVALID_ARG;
  if (c.pre_norm && !w->gamma_pre) return MOE_ERR_INVALID_ARG;
  if (c.expert_norm && !w->gamma_expert) return MOE_ERR_INVALID_ARG;
  if (c.resid_mode != MOE_RESID_NONE && (!r || !w->resid_g)) return MOE_ERR_INVALID_ARG;
  if (!all_aligned({u, r, static_cast<const void*>(out), static_cast<const void*>(logits_out),
                        static_cast<const void*>(topk_idx_out), static_cast<const void*>(topk_w_out),
                        workspace, w->w_router, w->p_down, w->p_up, w->w_gu, w->w_down,
                        static_cast<const void*>(w->gamma_pre),
                        static_cast<const void*>(w->gamma_expert),
                        static_cast<const void*>(w->resid_g), static_cast<const void*>(w->logit_bias),
                        static_cast<const void*>(w->correction_bias),
                        static_cast<const void*>(w->gamma_in),
                        static_cast<const void*>(w->gamma_post)})) return MOE_ERR_ALIGNMENT;
  const Workspace L = layout(c);
  if (!workspace || workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// Copy streams and events of moe_layer_forward_host, created on first use on each device.
struct HostPipe {
  bool ok = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t in_ready[2] = {}, in_free[2] = {}, out_free[2] = {};
};

HostPipe* host_pipe() {
  static std::mutex mu;
  static HostPipe pipes[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  HostPipe& h = pipes[dev];
  if (!h.ok) {
    bool good = cudaStreamCreateWithFlags(&h.h2d, cudaStreamNonBlocking) == cudaSuccess &&
                cudaStreamCreateWithFlags(&h.d2h, cudaStreamNonBlocking) == cudaSuccess;
    cudaEvent_t* evs[] = {&h.start,       &h.done,       &h.in_ready[0], &h.in_ready[1],
                          &h.in_free[0],  &h.in_free[1], &h.out_free[0], &h.out_free[1]};
    for (cudaEvent_t* e : evs)
      good = good && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    if (!good) return nullptr;
    h.ok = true;
  }
  return &h;
}

// Bytes of one staging buffer (T x d_model elements, rounded up to 256 bytes).
size_t staging_slot_bytes(const moe_config_t& c) {
  const size_t b = static_cast<size_t>(c.T) * c.d_model * (c.dtype == MOE_F32 ? 4 : 2);
  return (b + 255) / 256 * 256;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape or mode not supported";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT: pointer not 16-byte aligned";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA call failed";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a bounded wait inside a kernel ran out";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK: device-side index check failed";
  }
  return "unknown moe_status_t";
}

moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* bytes) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = layout(*cfg).total;
  return MOE_OK;
}

moe_status_t moe_route(const moe_config_t* cfg, const void* u, const void* w_router,
                       const float* logit_bias, const float* correction_bias, float* logits_out,
                       int32_t* topk_idx, float* topk_w, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (cfg->T > 0 && (!u || !w_router || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
  if (!all_aligned({u, w_router, static_cast<const void*>(logit_bias),
                    static_cast<const void*>(correction_bias), static_cast<const void*>(logits_out),
                    static_cast<const void*>(topk_idx), static_cast<const void*>(topk_w)}))
    return MOE_ERR_ALIGNMENT;
  return do_route(*cfg, u, w_router, logit_bias, correction_bias, logits_out, topk_idx, topk_w,
                  static_cast<cudaStream_t>(stream));
}

moe_status_t moe_router_split_weights(const float* w, int32_t n, int32_t d, void* w_split,
                                      void* stream) {
  if (!w || !w_split || n <= 0 || d <= 0) return MOE_ERR_INVALID_ARG;
  if (d % 64) return MOE_ERR_UNSUPPORTED;
  if (!all_aligned({static_cast<const void*>(w), static_cast<const void*>(w_split)}))
    return MOE_ERR_ALIGNMENT;
  const size_t count = static_cast<size_t>(n) * d;
  const unsigned blocks = static_cast<unsigned>(std::min<size_t>((count + 255) / 256, static_cast<size_t>(std::max(device_info().sms, 1)) * 16));
  launch_k(router_split_kernel, blocks, 256, 0, static_cast<cudaStream_t>(stream),
      w, count, d, static_cast<uint16_t*>(w_split));
  return last_launch();
}

moe_status_t moe_permute(const moe_config_t* cfg, const int32_t* topk_idx,
                         int32_t* expert_offsets, int32_t* perm_token, int32_t* inv_perm,
                         const void* x, const float* gamma_pre, void* x_perm, void* workspace,
                         size_t workspace_bytes, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (!expert_offsets || (cfg->T > 0 && (!topk_idx || !perm_token || !inv_perm)))
    return MOE_ERR_INVALID_ARG;
  if (x && !x_perm) return MOE_ERR_INVALID_ARG;
  if (gamma_pre && (cfg->dtype != MOE_BF16 || cfg->d_latent == 0)) return MOE_ERR_UNSUPPORTED;
  if (!all_aligned({static_cast<const void*>(topk_idx), static_cast<const void*>(expert_offsets),
                        static_cast<const void*>(perm_token), static_cast<const void*>(inv_perm), x,
                        static_cast<const void*>(gamma_pre), x_perm, workspace})) return MOE_ERR_ALIGNMENT;
  const size_t need = static_cast<size_t>(nchunks(*cfg)) * cfg->n_experts * 4;
  if (cfg->T > 0 && (!workspace || workspace_bytes < need)) return MOE_ERR_WORKSPACE;
  return do_permute(*cfg, topk_idx, expert_offsets, perm_token, inv_perm, x, gamma_pre, x_perm,
                    static_cast<int32_t*>(workspace), static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ------------------------------------------------------------------ allocation-free dispatch
//
// Scratch of moe_permute_static: the per-chunk expert histograms of the dispatch permutation
// (ceil(T/128) x n int32), held in a file-scope device array instead of a caller workspace.  Every
// device that loads the library holds these 256 KB until the process exits.  Host code must not
// pass the symbol itself to a kernel (on the host it names a host-side stand-in); its device
// address is taken once per device with cudaGetSymbolAddress and passed as a plain pointer.
static __device__ __align__(256) int32_t g_permute_scratch[MOE_PERMUTE_STATIC_MAX_COUNTS];

namespace {

// Device address of g_permute_scratch on the current device, looked up on the first call on
// that device (nullptr if the lookup fails).
int32_t* permute_scratch_ptr() {
  static std::mutex mu;
  static int32_t* ptr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
    ptr[dev] = static_cast<int32_t*>(p);
  }
  return ptr[dev];
}

}  // namespace

extern "C" {

moe_status_t moe_permute_static(const moe_config_t* cfg, const int32_t* topk_idx,
                                int32_t* expert_offsets, int32_t* perm_token, int32_t* inv_perm,
                                const void* x, const float* gamma_pre, void* x_perm, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (!expert_offsets || (cfg->T > 0 && (!topk_idx || !perm_token || !inv_perm)))
    return MOE_ERR_INVALID_ARG;
  if (x && !x_perm) return MOE_ERR_INVALID_ARG;
  if (gamma_pre && (cfg->dtype != MOE_BF16 || cfg->d_latent == 0)) return MOE_ERR_UNSUPPORTED;
  if (!all_aligned({static_cast<const void*>(topk_idx), static_cast<const void*>(expert_offsets),
                    static_cast<const void*>(perm_token), static_cast<const void*>(inv_perm), x,
                    static_cast<const void*>(gamma_pre), x_perm}))
    return MOE_ERR_ALIGNMENT;
  const long need = static_cast<long>(nchunks(*cfg)) * cfg->n_experts;
  if (need > MOE_PERMUTE_STATIC_MAX_COUNTS) return MOE_ERR_WORKSPACE;
  int32_t* scratch = permute_scratch_ptr();
  if (!scratch) return MOE_ERR_CUDA;
  // The count kernel overwrites every histogram entry this call uses, so no clearing is needed.
  return do_permute(*cfg, topk_idx, expert_offsets, perm_token, inv_perm, x, gamma_pre, x_perm,
                    scratch, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_dispatch_rows(const moe_config_t* cfg, const int32_t* inv_perm, const void* x,
                               const float* gamma_pre, void* x_perm, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (cfg->T > 0 && (!inv_perm || !x || !x_perm)) return MOE_ERR_INVALID_ARG;
  if (gamma_pre && (cfg->dtype != MOE_BF16 || cfg->d_latent == 0)) return MOE_ERR_UNSUPPORTED;
  if (!all_aligned({static_cast<const void*>(inv_perm), x, static_cast<const void*>(gamma_pre),
                    x_perm}))
    return MOE_ERR_ALIGNMENT;
  if (cfg->T == 0) return MOE_OK;
  return do_dispatch_rows(*cfg, inv_perm, x, gamma_pre, x_perm, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_row_sumsq_parts(const moe_config_t* cfg, int32_t* parts) {
  if (!parts) return MOE_ERR_INVALID_ARG;
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  *parts = sumsq_parts(*cfg);
  return MOE_OK;
}

moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* x_perm,
                            const int32_t* expert_offsets, const void* w_gu, const void* w_down,
                            const float* gamma_expert, void* out_perm, float* row_sumsq,
                            void* workspace, size_t workspace_bytes, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  const size_t TK = static_cast<size_t>(cfg->T) * cfg->top_k;
  if (TK > 0 && (!x_perm || !expert_offsets || !w_gu || !w_down || !out_perm))
    return MOE_ERR_INVALID_ARG;
  if (cfg->expert_norm && TK > 0 && !gamma_expert) return MOE_ERR_INVALID_ARG;
  if (!all_aligned({x_perm, static_cast<const void*>(expert_offsets), w_gu, w_down,
                        static_cast<const void*>(gamma_expert), out_perm,
                        static_cast<const void*>(row_sumsq), workspace})) return MOE_ERR_ALIGNMENT;
  const size_t need = TK * cfg->d_ff * dsize(*cfg);
  if (cfg->dtype == MOE_BF16 && TK > 0 && (!workspace || workspace_bytes < need))
    return MOE_ERR_WORKSPACE;
  return do_experts(*cfg, x_perm, expert_offsets, w_gu, w_down, gamma_expert, out_perm, workspace,
                    static_cast<cudaStream_t>(stream), false,
                    cfg->dtype == MOE_BF16 ? row_sumsq : nullptr);
}

moe_status_t moe_combine(const moe_config_t* cfg, const void* out_perm, const float* row_sumsq,
                         const int32_t* inv_perm, const float* topk_w, void* y, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (cfg->T > 0 && (!out_perm || !inv_perm || !topk_w || !y)) return MOE_ERR_INVALID_ARG;
  if (!all_aligned({out_perm, static_cast<const void*>(row_sumsq),
                    static_cast<const void*>(inv_perm), static_cast<const void*>(topk_w),
                    static_cast<const void*>(y)})) return MOE_ERR_ALIGNMENT;
  return do_combine(*cfg, out_perm, inv_perm, topk_w, y, static_cast<cudaStream_t>(stream),
                    cfg->dtype == MOE_BF16 ? row_sumsq : nullptr);
}

moe_status_t moe_latent_down(const moe_config_t* cfg, const void* u, const void* p_down,
                             void* z_raw, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (cfg->d_latent == 0 || cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (cfg->T > 0 && (!u || !p_down || !z_raw)) return MOE_ERR_INVALID_ARG;
  if (!all_aligned({u, p_down, static_cast<const void*>(z_raw)})) return MOE_ERR_ALIGNMENT;
  return do_latent_down(*cfg, u, p_down, z_raw, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_latent_up(const moe_config_t* cfg, const void* y, const void* p_up,
                           const void* r, const float* resid_g, void* out, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (cfg->d_latent == 0 || cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (cfg->T > 0 && (!y || !p_up || !out)) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && cfg->resid_mode != MOE_RESID_NONE && (!r || !resid_g)) return MOE_ERR_INVALID_ARG;
  if (!all_aligned({y, p_up, r, static_cast<const void*>(resid_g), static_cast<const void*>(out)})) return MOE_ERR_ALIGNMENT;
  return do_latent_up(*cfg, y, p_up, r, resid_g, out, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// Copies of the intermediates a caller asked for (moe_layer_forward_taps), each queued right
// after the stage that produces it.
struct Taps {
  const moe_layer_taps_t* t = nullptr;
  moe_status_t inv(const moe_config_t& c, const int32_t* inv, cudaStream_t st) const {
    if (!t || !t->inv_perm) return MOE_OK;
    const size_t bytes = static_cast<size_t>(c.T) * c.top_k * sizeof(int32_t);
    return cudaMemcpyAsync(t->inv_perm, inv, bytes, cudaMemcpyDeviceToDevice, st) == cudaSuccess
               ? MOE_OK : MOE_ERR_CUDA;
  }
  // z[t] = x_perm[inv[t*k]]: every slot of a token carries the same dispatched row
  moe_status_t z(const moe_config_t& c, const void* x_perm, const int32_t* inv,
                 cudaStream_t st) const {
    if (!t || !t->z) return MOE_OK;
    const long rb = static_cast<long>(expert_in(c)) * static_cast<long>(dsize(c));
    const int row_vec = static_cast<int>(rb / 16);
    const int threads = row_vec >= 256 ? 256 : ((row_vec + 31) / 32) * 32;
    const long grid = std::min<long>(c.T, static_cast<long>(std::max(device_info().sms, 1)) * 16);
    launch_k(gather_rows_kernel, static_cast<unsigned>(grid), threads, 0, st,
        static_cast<const uint4*>(x_perm), static_cast<long>(c.T) * c.top_k, inv,
        static_cast<long>(c.T), c.top_k, row_vec, static_cast<uint4*>(t->z));
    return last_launch();
  }
  moe_status_t copy(void* dst, const void* src, size_t rows, const moe_config_t& c,
                    cudaStream_t st) const {
    if (!dst) return MOE_OK;
    const size_t bytes = rows * static_cast<size_t>(expert_in(c)) * dsize(c);
    return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st) == cudaSuccess
               ? MOE_OK : MOE_ERR_CUDA;
  }
};

moe_status_t layer_forward_impl(const moe_config_t* cfg, const moe_weights_t* w, const void* u,
                                const void* r, void* out, float* logits_out,
                                int32_t* topk_idx_out, float* topk_w_out, const Taps& taps,
                                void* workspace, size_t workspace_bytes, void* stream) {
  moe_status_t s = check_forward(cfg, w, u, r, out, logits_out, topk_idx_out, topk_w_out,
                                 workspace, workspace_bytes);
  if (s != MOE_OK) return s;
  const moe_config_t& c = *cfg;
  if (c.T == 0) return MOE_OK;
  const bool latent = c.d_latent > 0;
  const Workspace L = layout(c);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* idx = topk_idx_out ? topk_idx_out : at<int32_t>(workspace, L.idx);
  float* wt = topk_w_out ? topk_w_out : at<float>(workspace, L.w);
  int32_t* offsets = at<int32_t>(workspace, L.offsets);
  int32_t* perm = at<int32_t>(workspace, L.perm);
  int32_t* inv = at<int32_t>(workspace, L.inv);
  void* x_perm = at<void>(workspace, L.x_perm);
  void* act = at<void>(workspace, L.act);

  prof_mark(st, 0);
  if (c.input_norm) {  // the branch input is the residual stream's norm (counted in stage 0)
    void* un = at<void>(workspace, L.u_norm);
    if ((s = do_input_norm(c, r, w->gamma_in, un, st)) != MOE_OK) return s;
    u = un;
  }
  if ((s = do_route(c, u, w->w_router, w->logit_bias, w->correction_bias, logits_out, idx, wt, st,
                    at<float>(workspace, L.logits))) != MOE_OK)
    return s;
  prof_mark(st, 1);
  const void* xin = u;
  if (latent) {
    void* z = at<void>(workspace, L.z_raw);
    if ((s = do_latent_down(c, u, w->p_down, z, st)) != MOE_OK) return s;
    xin = z;
  }
  prof_mark(st, 2);
  if ((s = do_permute(c, idx, offsets, perm, inv, xin, c.pre_norm ? w->gamma_pre : nullptr, x_perm,
                      at<int32_t>(workspace, L.counts), st)) != MOE_OK)
    return s;
  if ((s = taps.inv(c, inv, st)) != MOE_OK || (s = taps.z(c, x_perm, inv, st)) != MOE_OK) return s;
  prof_mark(st, 3);
  // The expert output overwrites the dispatched input rows (no longer needed after GEMM 1).
  // The down GEMM leaves each row's partial sums of squares for the combine's I_gamma norms when
  // its tiles are the normal orientation (a few per row); the swapped orientation's many per-warp
  // partials would cost the combine more than its own reduction.
  float* row_ss = c.expert_norm && c.dtype == MOE_BF16 && sumsq_parts(c) <= kMaxFusedSsParts
                      ? at<float>(workspace, L.ss) : nullptr;
  if ((s = do_experts(c, x_perm, offsets, w->w_gu, w->w_down, w->gamma_expert, x_perm, act, st,
                      true, row_ss)) != MOE_OK)
    return s;
  if (c.dtype == MOE_F32) prof_mark(st, 4);  // one fused kernel: all time in stage 3
  if (taps.t && (s = taps.copy(taps.t->s, x_perm, static_cast<size_t>(c.T) * c.top_k, c, st)) != MOE_OK)
    return s;
  prof_mark(st, 5);
  void* y = latent ? at<void>(workspace, L.y) : out;
  if ((s = do_combine(c, x_perm, inv, wt, y, st, row_ss)) != MOE_OK) return s;
  if (taps.t && (s = taps.copy(taps.t->y, y, static_cast<size_t>(c.T), c, st)) != MOE_OK) return s;
  prof_mark(st, 6);
  if (latent && !c.post_norm &&
      (s = do_latent_up(c, y, w->p_up, r, w->resid_g, out, st)) != MOE_OK)
    return s;
  if (c.post_norm) {  // b to the workspace, then output norm + residual gate per row
    moe_config_t plain = c;
    plain.resid_mode = MOE_RESID_NONE;
    void* b = at<void>(workspace, L.b);
    if ((s = do_latent_up(plain, y, w->p_up, nullptr, nullptr, b, st)) != MOE_OK) return s;
    if ((s = do_resid_update(c, b, r, w->gamma_post, w->resid_g, out, st)) != MOE_OK) return s;
  }
  prof_mark(st, 7);
  prof_next_call();
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status_t moe_layer_forward(const moe_config_t* cfg, const moe_weights_t* w, const void* u,
                               const void* r, void* out, float* logits_out,
                               int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                               size_t workspace_bytes, void* stream) {
  return layer_forward_impl(cfg, w, u, r, out, logits_out, topk_idx_out, topk_w_out, Taps{},
                            workspace, workspace_bytes, stream);
}

moe_status_t moe_layer_forward_taps(const moe_config_t* cfg, const moe_weights_t* w,
                                    const void* u, const void* r, void* out, float* logits_out,
                                    int32_t* topk_idx_out, float* topk_w_out,
                                    const moe_layer_taps_t* taps, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (taps && !all_aligned({taps->z, taps->s, taps->y, static_cast<const void*>(taps->inv_perm)}))
    return MOE_ERR_ALIGNMENT;
  Taps tp;
  tp.t = taps;
  return layer_forward_impl(cfg, w, u, r, out, logits_out, topk_idx_out, topk_w_out, tp,
                            workspace, workspace_bytes, stream);
}

moe_status_t moe_residual_update(const moe_config_t* cfg, const void* b, const void* r,
                                 const float* gamma_post, const float* resid_g, void* out,
                                 void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (cfg->dtype != MOE_BF16 || cfg->d_model > 8192) return MOE_ERR_UNSUPPORTED;
  if (cfg->T > 0 && (!b || !out)) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && cfg->resid_mode != MOE_RESID_NONE && (!r || !resid_g)) return MOE_ERR_INVALID_ARG;
  if (!all_aligned({b, r, static_cast<const void*>(gamma_post), static_cast<const void*>(resid_g),
                    static_cast<const void*>(out)}))
    return MOE_ERR_ALIGNMENT;
  return do_resid_update(*cfg, b, r, gamma_post, resid_g, out, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_noisy_gate_workspace_size(const moe_config_t* cfg, size_t* bytes) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = gate_layout(*cfg).total;
  return MOE_OK;
}

moe_status_t moe_noisy_gate(const moe_config_t* cfg, const void* u, const void* w_router,
                            const void* w_noise, const float* noise_eps, float* noisy_logits_out,
                            int32_t* topk_idx, float* topk_w, float* load_prob_out,
                            float* importance, float* load, float* cv2, void* workspace,
                            size_t workspace_bytes, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  const moe_config_t& c = *cfg;
  if (c.top_k >= c.n_experts) return MOE_ERR_UNSUPPORTED;  // kth_excluding needs k < n
  if (c.T == 0) return MOE_ERR_INVALID_ARG;                 // statistics of an empty batch
  if (!u || !w_router || !w_noise || !noise_eps || !topk_idx || !topk_w || !importance || !load ||
      !cv2)
    return MOE_ERR_INVALID_ARG;
  if (!all_aligned({u, w_router, w_noise, static_cast<const void*>(noise_eps),
                    static_cast<const void*>(noisy_logits_out), static_cast<const void*>(topk_idx),
                    static_cast<const void*>(topk_w), static_cast<const void*>(load_prob_out),
                    static_cast<const void*>(importance), static_cast<const void*>(load),
                    static_cast<const void*>(cv2), workspace}))
    return MOE_ERR_ALIGNMENT;
  const GateWorkspace L = gate_layout(c);
  if (!workspace || workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the two logit passes are plain logits (softmax-gate router, no bias)
  moe_config_t plain = c;
  plain.gate_mode = MOE_GATE_SOFTMAX;
  float* lb = at<float>(workspace, L.l);
  float* mb = at<float>(workspace, L.m);
  int32_t* si = at<int32_t>(workspace, L.idx);
  float* sw = at<float>(workspace, L.w);
  if ((s = do_route(plain, u, w_router, nullptr, nullptr, lb, si, sw, st)) != MOE_OK) return s;
  if ((s = do_route(plain, u, w_noise, nullptr, nullptr, mb, si, sw, st)) != MOE_OK) return s;
  float* pi = at<float>(workspace, L.pi);
  float* pl = at<float>(workspace, L.pl);
  launch_k(noisy_gate_kernel, L.nparts / 4, 128, 0, st, lb, mb, noise_eps, c.T, c.n_experts, c.top_k,
                                                  noisy_logits_out, topk_idx, topk_w,
                                                  load_prob_out, pi, pl);
  launch_k(gate_stats_reduce_kernel, 1, kMaxExperts, 0, st, pi, pl, L.nparts, c.n_experts, importance,
                                                      load, cv2);
  return last_launch(2);
}

unsigned long long moe_launch_count(void) { return g_launches.load(); }

moe_status_t moe_selftest_wait_timeout(long long budget_clocks, int32_t* gave_up, void* stream) {
  if (!gave_up || budget_clocks <= 0 || budget_clocks > kWaitBudgetClocks) return MOE_ERR_INVALID_ARG;
  if (!aligned16(gave_up)) return MOE_ERR_ALIGNMENT;
  launch_k(wait_timeout_selftest_kernel, 1, 32, 0, static_cast<cudaStream_t>(stream), budget_clocks,
                                                                                gave_up);
  return last_launch();
}

moe_status_t moe_profile_begin(int32_t max_calls) {
  if (max_calls <= 0 || max_calls > 100000) return MOE_ERR_INVALID_ARG;
  Profiler& p = prof();
  if (p.active) return MOE_ERR_INVALID_ARG;
  p.ev.assign(static_cast<size_t>(max_calls) * kMarks, nullptr);
  for (auto& e : p.ev)
    if (cudaEventCreate(&e) != cudaSuccess) {
      for (auto& f : p.ev)
        if (f) cudaEventDestroy(f);
      p.ev.clear();
      return MOE_ERR_CUDA;
    }
  p.max_calls = max_calls;
  p.calls = 0;
  p.active = true;
  return MOE_OK;
}

moe_status_t moe_profile_end(float* stage_ms, int32_t* calls) {
  Profiler& p = prof();
  if (!p.active || !stage_ms) return MOE_ERR_INVALID_ARG;
  moe_status_t s = MOE_OK;
  for (int i = 0; i < MOE_PROFILE_STAGES; ++i) stage_ms[i] = 0.0f;
  if (p.calls > 0 && cudaEventSynchronize(p.ev[(p.calls - 1) * kMarks + MOE_PROFILE_STAGES]) !=
                         cudaSuccess)
    s = MOE_ERR_CUDA;
  for (int c = 0; c < p.calls && s == MOE_OK; ++c)
    for (int i = 0; i < MOE_PROFILE_STAGES; ++i) {
      float ms = 0.0f;
      if (cudaEventElapsedTime(&ms, p.ev[c * kMarks + i], p.ev[c * kMarks + i + 1]) != cudaSuccess) {
        s = MOE_ERR_CUDA;
        break;
      }
      stage_ms[i] += ms;
    }
  if (calls) *calls = p.calls;
  for (auto& e : p.ev) cudaEventDestroy(e);
  p.ev.clear();
  p.active = false;
  p.calls = p.max_calls = 0;
  return s;
}

moe_status_t moe_host_staging_size(const moe_config_t* cfg, size_t* bytes) {
  if (!bytes) return MOE_ERR_INVALID_ARG;
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  *bytes = 4 * staging_slot_bytes(*cfg);
  return MOE_OK;
}

moe_status_t moe_layer_forward_host(const moe_config_t* cfg, const moe_weights_t* w,
                                    int32_t n_batches, const void* const* u_host,
                                    void* const* out_host, void* staging, size_t staging_bytes,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (n_batches < 0 || (n_batches > 0 && (!u_host || !out_host))) return MOE_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n_batches; ++i)
    if (!u_host[i] || !out_host[i]) return MOE_ERR_INVALID_ARG;
  const moe_config_t& c = *cfg;
  const size_t slot = staging_slot_bytes(c);
  if (!staging || staging_bytes < 4 * slot) return MOE_ERR_WORKSPACE;
  if (!all_aligned({staging})) return MOE_ERR_ALIGNMENT;
  uint8_t* base = static_cast<uint8_t*>(staging);
  void* in[2] = {base, base + slot};
  void* outb[2] = {base + 2 * slot, base + 3 * slot};
  if ((s = check_forward(cfg, w, in[0], in[0], outb[0], nullptr, nullptr, nullptr, workspace,
                         workspace_bytes)) != MOE_OK)
    return s;
  if (n_batches == 0 || c.T == 0) return MOE_OK;
  HostPipe* hp = host_pipe();
  if (!hp) return MOE_ERR_CUDA;
  const size_t bytes = static_cast<size_t>(c.T) * c.d_model * (c.dtype == MOE_F32 ? 4 : 2);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The copy streams start after what is already queued on the caller's stream.
  cudaEventRecord(hp->start, st);
  cudaStreamWaitEvent(hp->h2d, hp->start, 0);
  cudaStreamWaitEvent(hp->d2h, hp->start, 0);
  for (int32_t i = 0; i < n_batches && s == MOE_OK; ++i) {
    const int b = i & 1;
    // input slot b is free once batch i-2's kernels are done with it
    if (i >= 2) cudaStreamWaitEvent(hp->h2d, hp->in_free[b], 0);
    cudaMemcpyAsync(in[b], u_host[i], bytes, cudaMemcpyHostToDevice, hp->h2d);
    cudaEventRecord(hp->in_ready[b], hp->h2d);
    cudaStreamWaitEvent(st, hp->in_ready[b], 0);
    // output slot b is free once batch i-2's output copy has read it
    if (i >= 2) cudaStreamWaitEvent(st, hp->out_free[b], 0);
    s = moe_layer_forward(cfg, w, in[b], in[b], outb[b], nullptr, nullptr, nullptr, workspace,
                          workspace_bytes, stream);
    cudaEventRecord(hp->in_free[b], st);  // batch i's kernels are done: input read, output ready
    cudaStreamWaitEvent(hp->d2h, hp->in_free[b], 0);
    if (s == MOE_OK)
      cudaMemcpyAsync(out_host[i], outb[b], bytes, cudaMemcpyDeviceToHost, hp->d2h);
    cudaEventRecord(hp->out_free[b], hp->d2h);
  }
  // The caller's stream reaches the end of every copy this call queued.
  cudaEventRecord(hp->done, hp->d2h);
  cudaStreamWaitEvent(st, hp->done, 0);
  if (s != MOE_OK) return s;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_gather_rows(const void* src, int64_t src_rows, const int32_t* rows,
                             int64_t n_rows, int64_t row_bytes, void* dst, void* stream) {
  if (n_rows < 0 || src_rows < 0 || row_bytes < 0) return MOE_ERR_INVALID_ARG;
  if (row_bytes == 0 || row_bytes % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (n_rows == 0) return MOE_OK;
  if (!src || !rows || !dst) return MOE_ERR_INVALID_ARG;
  if (!all_aligned({src, static_cast<const void*>(rows), dst})) return MOE_ERR_ALIGNMENT;
  const int row_vec = static_cast<int>(row_bytes / 16);
  const int threads = row_vec >= 256 ? 256 : ((row_vec + 31) / 32) * 32;
  const long grid = std::min<long>(n_rows, static_cast<long>(std::max(device_info().sms, 1)) * 16);
  launch_k(gather_rows_kernel, static_cast<unsigned>(grid), threads, 0, static_cast<cudaStream_t>(stream),
      static_cast<const uint4*>(src), static_cast<long>(src_rows), rows, static_cast<long>(n_rows),
      1, row_vec, static_cast<uint4*>(dst));
  return last_launch();
}

moe_status_t moe_get_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  return static_cast<moe_status_t>(v);
}

}  // extern "C"
