// Grouped GEMM on the 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM, operands
// staged by TMA with the 128-byte swizzle), persistent and warp-specialised, with the MoE
// layer's epilogues fused in.
//
//   out[r, c] = epi( sum_k X[r, k] * W[g*Nw + c', k] )      for r in group g's row segment
//
// X is the activation matrix (rows grouped by expert, or one group for a dense projection) and
// W the stacked weights of all groups, both K-major bf16.  Two orientations:
//   normal : tcgen05 M = 128 rows of X, N = BN rows of W    (prefill-sized groups)
//   swap   : tcgen05 M = 128 rows of W, N = BN rows of X    (decode: a few tokens per expert;
//            the weights fill the 128-wide M side and the tokens the narrow N side)
// Tiles are ordered (group, feature tile, row chunk) with the row chunk fastest, so the CTAs
// working at one time share weight tiles through L2 and each weight tile leaves HBM about once.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM allocator + MMA issuer,
// warps 2..5 = epilogue (TMEM -> registers -> fused math -> global).  The accumulator is double
// buffered in TMEM so the epilogue of one tile overlaps the MMAs of the next.
#pragma once

#include "common.cuh"

namespace moe {

enum EpiKind : int {
  EPI_STORE = 0,    // dtype(acc), optionally dtype(dtype(acc) * (1 + gamma[col]))
  EPI_RELU = 1,     // dtype(max(acc, 0))
  EPI_SWIGLU = 2,   // dtype(SiLU(gate) * up), gate/up W rows paired (rows c and Nw/2 + c)
  EPI_RESGATE = 3,  // residual update of the latent up-projection
  EPI_ROUTER = 4,   // top-k selection and renormalised weights over the row's logits
};

enum TileOrder : int { TILE_CHUNK_FASTEST = 0, TILE_FEATURE_FASTEST = 1 };

struct GemmParams {
  const int* seg;   // [G+1] row offsets of the groups in X, or nullptr: one group of M rows
  int G;            // groups
  int M;            // rows of X when seg == nullptr
  int K;            // reduction length, multiple of 64
  int Nw;           // W rows per group
  int Nout;         // output columns (= row stride of out)
  void* out;        // [rows, Nout]: bf16 bits
  const float* gamma;        // EPI_STORE: optional gain (1 + gamma[col])
  const uint16_t* resid;     // EPI_RESGATE: residual r [rows, Nout]
  const float* gparam;       // EPI_RESGATE: g [Nout]
  float tau, floor_;
  int resid_mode;            // MOE_RESID_*
  float* logits;             // EPI_ROUTER: [rows, Nout] fp32 or nullptr
  int32_t* topk_idx;         // EPI_ROUTER: [rows, top_k]
  float* topk_w;             // EPI_ROUTER: [rows, top_k]
  const float* bias;         // EPI_ROUTER: [Nout] or nullptr
  int top_k;
  float routed_scale;
  int gate_mode;             // EPI_ROUTER: MOE_GATE_SOFTMAX | MOE_GATE_SIGMOID
  float logit_mult;          // EPI_ROUTER (sigmoid): output_multiplier
  const float* sel_bias;     // EPI_ROUTER (sigmoid): selection-only correction bias [Nout]
  int x_k_period;            // > 0: X's k coordinate wraps every x_k_period columns (W's K is
                             // a multiple: the fp32 router weights' hi/mid/lo bf16 parts)
  int router_select;         // EPI_ROUTER: 1 = select the top-k in the epilogue (logits, if
                             // stored, are the payloads); 0 = only store the pre-activation
                             // logits (output_multiplier * acc + bias) for a separate selection
  int tile_order;            // TILE_CHUNK_FASTEST | TILE_FEATURE_FASTEST
  float* row_ss;             // EPI_STORE (optional): [rows, ss_parts] partial sums of squares of
  int ss_parts;              // the stored bf16 values, one per row and column block
  int out_tma;               // bf16 epilogues of the normal orientation: 1 = the output tensor
                             // map is valid and whole-warp row blocks leave by TMA stores
  int l2_hints;              // 1: weight tiles are loaded as the first lines L2 evicts (each is
                             // read by the tiles running at the same time, then not again), and
                             // the staged output stores are kept in L2 ahead of other lines (the
                             // next GEMM reads them); for layers whose activations fit in L2
  int tail_m64;              // 1: normal-orientation tiles of at most 64 rows run M = 64 MMAs
};

// Shared memory that stages the bf16 output of the normal-orientation epilogues: one 4 KB
// buffer (32 rows x 128 bytes) per epilogue warp.
constexpr int kStageOutBytes = 4 * 4096;

template <bool kSwap, int BN, int kEpi>
struct GemmShape {
  static constexpr bool kDual = (kEpi == EPI_SWIGLU);
  static constexpr int kBK = 64;                                  // 128 bytes of bf16
  static constexpr int kABytes = 128 * 128 * ((kSwap && kDual) ? 2 : 1);
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kFO = kSwap ? 128 : (kDual ? BN / 2 : BN);  // output features per tile
  static constexpr int kCH = kSwap ? BN : 128;                     // X rows per tile
  static constexpr int kAccCols = (kSwap && kDual) ? 2 * BN : BN;  // fp32 TMEM columns
  static constexpr int kTmemCols = (2 * kAccCols <= 32)    ? 32
                                   : (2 * kAccCols <= 64)  ? 64
                                   : (2 * kAccCols <= 128) ? 128
                                   : (2 * kAccCols <= 256) ? 256
                                                           : 512;
  static constexpr int kXBoxRows = kSwap ? BN : 128;
  static constexpr int kWBoxRows = kSwap ? 128 : (kDual ? BN / 2 : BN);
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, BN);
  static constexpr uint32_t kIdesc64 = idesc_bf16_f32(64, BN);  // a group's last chunk of <= 64 rows
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "tcgen05 M=128 needs N % 16 == 0");
  static_assert(2 * kAccCols <= 512, "two accumulators must fit in TMEM");
};

constexpr int kMaxGroups = 256;
constexpr int kGemmThreads = 192;
constexpr int kSmemMisc = 8192;  // barriers, TMEM slot, group tables, residual-gate coefficients

// Barrier 1 among the 128 epilogue threads only (barrier 0 is __syncthreads).
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Barrier 1 with an AND over the 128 epilogue threads: every thread gets the same answer, so a
// bounded wait that ran out in one thread makes all of them leave together (none is left
// waiting at a later barrier for threads that already left).
__device__ __forceinline__ bool epilogue_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// Whether a kernel instance stages its output for TMA stores (bf16 epilogues, normal orientation).
template <bool kSwap, int kEpi>
__host__ __device__ constexpr bool stages_output() {
  return !kSwap && kEpi != EPI_ROUTER;
}

template <bool kSwap, int BN, int kEpi, int kStages>
constexpr int gemm_smem_bytes() {
  return kStages * GemmShape<kSwap, BN, kEpi>::kStageBytes +
         (stages_output<kSwap, kEpi>() ? kStageOutBytes : 0) + 1024 + kSmemMisc;
}

// Where one epilogue warp's output goes.  A warp whose 32 rows all lie inside the tile stages
// each 32 x 64 chunk in its shared-memory buffer (128-byte rows, 16-byte units XOR-swizzled by
// the row: the layout a SWIZZLE_128B tensor map reads, and free of bank conflicts) and stores it
// with one TMA box store; a warp holding rows past the tile's end (the next group's rows follow
// in the same matrix) stores its valid rows directly, 16 bytes at a time.
struct EpiOut {
  const CUtensorMap* tm;  // output tensor map, or nullptr: direct stores only
  uint8_t* buf;           // this warp's 4 KB staging buffer (1024-byte aligned)
  bool whole;             // all 32 rows of this warp lie inside the tile
  bool keep;              // store with the L2 evict-last policy
};

// Emits one 64-column chunk (8 x 16 bytes per row) of this thread's row at output column x of
// row block y (the warp's first row); `dst` is the row's address at column x.
__device__ __forceinline__ void emit_chunk(const EpiOut& eo, const uint4 (&ch)[8], uint16_t* dst,
                                           bool valid, int x, int y, int lane) {
  if (eo.tm != nullptr && eo.whole) {
    if (lane == 0) bulk_wait_read_all();  // the buffer's previous store has read it
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<uint4*>(eo.buf + lane * 128 + ((j ^ (lane & 7)) << 4)) = ch[j];
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (eo.keep) tma_store_2d_hint(eo.tm, eo.buf, x, y, l2_policy_evict_last());
      else tma_store_2d(eo.tm, eo.buf, x, y);
      bulk_commit();
    }
  } else if (valid) {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int j = 0; j < 8; ++j) d[j] = ch[j];
  }
}

__device__ __forceinline__ void pack8(const float* v, uint4& lo, uint4& hi) {
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  lo = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  hi = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

struct TileCoord {
  int g, ft, chunk, row0, nrows;
};

// Tile t's group, feature tile and row chunk.  Within a group the tiles run in one of two orders:
//   TILE_CHUNK_FASTEST   : (feature tile, row chunk), row chunk fastest.  The CTAs working at one
//                          time share each weight tile; a group's activation rows are re-read per
//                          feature tile, from L2 when the group's rows are few (expert GEMMs).
//   TILE_FEATURE_FASTEST : (row chunk, feature tile).  The CTAs working at one time share each
//                          activation chunk, so a large activation matrix leaves HBM once and the
//                          (smaller) weight matrix is the operand re-read from L2 (dense
//                          projections over many tokens).
__device__ __forceinline__ TileCoord decode_tile(int t, const int* s_seg, const int* s_pref,
                                                 int G, int FT, int CH, int order) {
  int lo = 0, hi = G;
  while (lo < hi) {  // last g with s_pref[g] <= t
    int mid = (lo + hi + 1) >> 1;
    if (s_pref[mid] <= t) lo = mid; else hi = mid - 1;
  }
  TileCoord c;
  c.g = lo;
  const int chunks = (s_pref[lo + 1] - s_pref[lo]) / FT;
  const int local = t - s_pref[lo];
  if (order == TILE_FEATURE_FASTEST) {
    c.chunk = local / FT;
    c.ft = local - c.chunk * FT;
  } else {
    c.ft = local / chunks;
    c.chunk = local - c.ft * chunks;
  }
  c.row0 = s_seg[lo] + c.chunk * CH;
  int rem = s_seg[lo + 1] - c.row0;
  c.nrows = rem < CH ? rem : CH;
  return c;
}

// Router epilogue: selection key and payload of logit accumulator value `acc` at column `col`.
// Softmax gate: the logit l = acc (+ bias) is both.  Muse sigmoid gate: the score
// s = sigmoid(output_multiplier * acc (+ bias)) is the payload (what the weights are made of and
// what logits_out returns in this mode) and s + correction bias (one fp32 addition, selection
// only) the key.
__device__ __forceinline__ float router_pre(const GemmParams& p, float acc, int col) {
  const int c = col < p.Nout ? col : 0;
  const float m = p.gate_mode == MOE_GATE_SIGMOID ? acc * p.logit_mult : acc;
  return m + (p.bias ? p.bias[c] : 0.0f);
}
__device__ __forceinline__ void router_key(const GemmParams& p, float acc, int col, float& key,
                                           float& pay) {
  const int c = col < p.Nout ? col : 0;
  const float l = router_pre(p, acc, col);
  if (p.gate_mode == MOE_GATE_SIGMOID) {
    pay = 1.0f / (1.0f + expf(-l));
    key = pay + (p.sel_bias ? p.sel_bias[c] : 0.0f);
  } else {
    pay = l;
    key = l;
  }
}

// Epilogue of the normal orientation: this thread owns row row0 + rpw*q + lane of the tile (valid
// if lane < rpw and below nrows) and the tile's BN accumulator columns (output features f0 ...).
// An M = 128 tile holds row r in TMEM lane r (rpw = 32); an M = 64 tile holds rows 16q .. 16q+15
// in lanes 32q .. 32q+15 (rpw = 16).
template <int BN, int kEpi>
__device__ __forceinline__ void epilogue_rows(const GemmParams& p, int row0, int nrows, int f0,
                                              uint32_t tbase, int q, int lane, float* s_coef,
                                              const EpiOut& eo, int rpw = 32) {
    const int rl = q * rpw + lane;
    const bool valid = lane < rpw && rl < nrows;
    const size_t row = static_cast<size_t>(row0 + rl);
    const int yblk = row0 + q * 32;  // first row of this warp's row block
    if constexpr (kEpi == EPI_ROUTER) {
      // Logits out (when asked for): one pass over the row's accumulator columns.  A tile holds
      // experts [f0, f0 + BN): all of them when it selects (router_select), else possibly a part.
      if (p.logits) {
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float v[16];
          tmem_ld16(tbase + c0, v);
          const int g0 = f0 + c0;  // expert of accumulator column c0
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (p.router_select) {
              float key;
              router_key(p, v[i], g0 + i, key, v[i]);
            } else {
              v[i] = router_pre(p, v[i], g0 + i);
            }
          }
          if (valid) {
            float* dst = p.logits + row * p.Nout + g0;
            if (g0 + 16 <= p.Nout && (p.Nout & 3) == 0) {
#pragma unroll
              for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (g0 + i < p.Nout) dst[i] = v[i];
            }
          }
        }
      }
      // Top-k by k selection passes over the row (re-read from TMEM each pass): pass j takes the
      // best entry in the order (key descending, column ascending) among those ranked after the
      // previous pick.  That is the order of a stable descending sort, so ties keep the lower
      // column first; the state is a few scalars per pass, all in registers.
      if (!p.router_select) return;
      float pick_pay[8];
      int pick_col[8];
      float prev_key = INFINITY;
      int prev_col = -1;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        pick_pay[j] = 0.0f;
        pick_col[j] = -1;
        if (j >= p.top_k) continue;
        float bk = -INFINITY, bp = 0.0f;
        int bc = 0x7fffffff;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float v[16];
          tmem_ld16(tbase + c0, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int col = c0 + i;
            float key, pay;
            router_key(p, v[i], col, key, pay);
            const bool after = key < prev_key || (key == prev_key && col > prev_col);
            const bool better = key > bk || (key == bk && col < bc);
            if (col < p.Nout && after && better) { bk = key; bc = col; bp = pay; }
          }
        }
        pick_pay[j] = bp;
        pick_col[j] = bc;
        prev_key = bk;
        prev_col = bc;
      }
      if (valid) {
        // weights: softmax over the kept logits (= softmax over all, renormalised), or the
        // sigmoid gate's scores / (their sum + 1e-15); times routed_scale
        const bool sig = p.gate_mode == MOE_GATE_SIGMOID;
        float e[8], sum = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          e[j] = 0.0f;
          if (j < p.top_k) e[j] = sig ? pick_pay[j] : __expf(pick_pay[j] - pick_pay[0]);
          sum += e[j];
        }
        const float scale = sig ? p.routed_scale / (sum + 1e-15f) : p.routed_scale / sum;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < p.top_k) {
            p.topk_idx[row * p.top_k + j] = pick_col[j];
            p.topk_w[row * p.top_k + j] = e[j] * scale;
          }
        }
      }
    } else if constexpr (kEpi == EPI_SWIGLU) {
      // accumulator columns [0, BN/2) are the gate projection, [BN/2, BN) the up projection
      uint16_t* out = static_cast<uint16_t*>(p.out) + row * p.Nout + f0;
      for (int c0 = 0; c0 < BN / 2; c0 += 64) {
        uint4 ch[8];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          float gv[16], uv[16];
          tmem_ld16(tbase + c0 + 16 * qq, gv);
          tmem_ld16(tbase + BN / 2 + c0 + 16 * qq, uv);
#pragma unroll
          for (int i = 0; i < 16; ++i) gv[i] = silu(gv[i]) * uv[i];
          pack8(gv, ch[2 * qq], ch[2 * qq + 1]);
        }
        emit_chunk(eo, ch, out + c0, valid, f0 + c0, yblk, lane);
      }
    } else if constexpr (kEpi == EPI_RESGATE) {
      // Per-column coefficients of this tile, computed once by the 128 epilogue threads:
      // out = alpha * r + beta * b  (MUSE gate: beta = sigmoid(g/tau), alpha =
      // sqrt(max(sigmoid(-g/tau)(1+beta), floor)); literal: alpha = 1, beta = g; none: 0, 1).
      epilogue_bar();  // the previous tile's readers are done with s_coef
      for (int cc = static_cast<int>(threadIdx.x) - 64; cc < BN; cc += 128) {
        const float g = p.gparam ? p.gparam[f0 + cc] : 0.0f;
        float a = 0.0f, b = 1.0f;
        if (p.resid_mode == MOE_RESID_MUSE_GATE) {
          b = sigmoidf_(g / p.tau);
          a = sqrtf(fmaxf(sigmoidf_(-g / p.tau) * (1.0f + b), p.floor_));
        } else if (p.resid_mode == MOE_RESID_LITERAL) {
          a = 1.0f;
          b = g;
        }
        s_coef[cc] = a;
        s_coef[BN + cc] = b;
      }
      epilogue_bar();
      const bool has_r = p.resid_mode != MOE_RESID_NONE;
      uint16_t* out = static_cast<uint16_t*>(p.out) + row * p.Nout + f0;
      const uint16_t* hrow = has_r ? p.resid + row * p.Nout + f0 : nullptr;
      for (int c0 = 0; c0 < BN; c0 += 64) {
        uint4 hv[8];  // 64 residual values, loaded together so their latency overlaps
#pragma unroll
        for (int i = 0; i < 8; ++i)
          hv[i] = (valid && has_r) ? reinterpret_cast<const uint4*>(hrow + c0)[i]
                                   : make_uint4(0, 0, 0, 0);
        uint4 ch[8];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          float v[16];
          tmem_ld16(tbase + c0 + 16 * qq, v);
          const uint16_t* hs = reinterpret_cast<const uint16_t*>(&hv[2 * qq]);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int col = c0 + 16 * qq + i;
            v[i] = s_coef[col] * bf16_to_f32(hs[i]) + s_coef[BN + col] * round_bf16(v[i]);
          }
          pack8(v, ch[2 * qq], ch[2 * qq + 1]);
        }
        emit_chunk(eo, ch, out + c0, valid, f0 + c0, yblk, lane);
      }
    } else {
      uint16_t* out = static_cast<uint16_t*>(p.out) + row * p.Nout + f0;
      float ss = 0.0f;  // EPI_STORE with row_ss: this row's sum of squares over the tile's columns
      for (int c0 = 0; c0 < BN; c0 += 64) {
        uint4 ch[8];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          float v[16];
          tmem_ld16(tbase + c0 + 16 * qq, v);
          if constexpr (kEpi == EPI_RELU) {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = fmaxf(v[i], 0.0f);
          } else if constexpr (kEpi == EPI_STORE) {
            if (p.gamma) {  // 16 gains as four 16-byte loads (the column offset is a multiple of 16)
              const float4* g4 = reinterpret_cast<const float4*>(p.gamma + f0 + c0 + 16 * qq);
#pragma unroll
              for (int i4 = 0; i4 < 4; ++i4) {
                const float4 g = __ldg(g4 + i4);
                v[4 * i4 + 0] = round_bf16(v[4 * i4 + 0]) * (1.0f + g.x);
                v[4 * i4 + 1] = round_bf16(v[4 * i4 + 1]) * (1.0f + g.y);
                v[4 * i4 + 2] = round_bf16(v[4 * i4 + 2]) * (1.0f + g.z);
                v[4 * i4 + 3] = round_bf16(v[4 * i4 + 3]) * (1.0f + g.w);
              }
            }
            if (p.row_ss) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float b = round_bf16(v[i]);
                ss = fmaf(b, b, ss);
              }
            }
          }
          pack8(v, ch[2 * qq], ch[2 * qq + 1]);
        }
        emit_chunk(eo, ch, out + c0, valid, f0 + c0, yblk, lane);
      }
      if constexpr (kEpi == EPI_STORE) {
        if (p.row_ss && valid) p.row_ss[row * p.ss_parts + f0 / BN] = ss;
      }
    }
}

template <bool kSwap, int BN, int kEpi, int kStages>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                   const __grid_constant__ CUtensorMap tmO, const GemmParams p) {
  using S = GemmShape<kSwap, BN, kEpi>;
  constexpr bool kStageOut = stages_output<kSwap, kEpi>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint8_t* stage_out = tiles + kStages * S::kStageBytes;  // 1024-byte aligned (stage multiple)
  uint64_t* full =
      reinterpret_cast<uint64_t*>(stage_out + (kStageOut ? kStageOutBytes : 0));
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* s_seg = reinterpret_cast<int*>(tmem_slot + 4);
  int* s_pref = s_seg + (kMaxGroups + 4);
  float* s_coef = reinterpret_cast<float*>(s_pref + (kMaxGroups + 4));  // [2][BN] alpha, beta

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;
  const int FT = (p.Nout + S::kFO - 1) / S::kFO;  // the router's last tile may be partial
  const int KB = p.K / S::kBK;

  // Setup that reads nothing an earlier kernel writes (barriers, TMEM, the tensor-map prefetch)
  // runs before the dependency wait and overlaps the previous kernel's tail.
  if (threadIdx.x == 32) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 128); }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, S::kTmemCols);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  pdl_wait();
  pdl_launch_dependents();  // one CTA per SM, all resident: the next kernel may launch

  // ---- group segments and the per-group tile prefix (warp 0)
  if (warp == 0) {
    const int per = (G + 31) / 32;
    int local = 0;
    for (int j = 0; j < per; ++j) {
      int g = lane * per + j;
      if (g < G) {
        int a = p.seg ? p.seg[g] : 0, b = p.seg ? p.seg[g + 1] : p.M;
        if (b < a) { latch_status(MOE_ERR_DEVICE_CHECK); b = a; }
        s_seg[g] = a;
        if (g == G - 1) s_seg[G] = b;
        local += ((b - a + S::kCH - 1) / S::kCH) * FT;
      }
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - local;
    for (int j = 0; j < per; ++j) {
      int g = lane * per + j;
      if (g < G) {
        int a = p.seg ? p.seg[g] : 0, b = p.seg ? p.seg[g + 1] : p.M;
        if (b < a) b = a;
        s_pref[g] = run;
        run += ((b - a + S::kCH - 1) / S::kCH) * FT;
      }
    }
    if (lane == 31) s_pref[G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_pref[G];

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    uint32_t stage = 0, phase = 0;
    uint32_t last_parity[kStages];
    bool issued[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) { issued[s] = false; last_parity[s] = 0; }
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      TileCoord c = decode_tile(t, s_seg, s_pref, G, FT, S::kCH, p.tile_order);
      const int wrow = c.g * p.Nw + c.ft * S::kFO;
      for (int kb = 0; kb < KB; ++kb) {
        // weight-stream-bound layers (l2_hints): L2 fetches the weight k-block one ring ahead, so
        // more DRAM requests are in flight than the shared-memory ring holds
        if (!kSwap && p.l2_hints && kb + kStages < KB) {
          const int kp = (kb + kStages) * S::kBK;
          tma_prefetch_2d(&tmW, kp, wrow);
          if (S::kDual) tma_prefetch_2d(&tmW, kp, wrow + p.Nw / 2);
        }
        if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
        uint8_t* sa = tiles + stage * S::kStageBytes;
        uint8_t* sb = sa + S::kABytes;
        mbar_arrive_expect_tx(&full[stage], S::kStageBytes);
        const int kx = kb * S::kBK;
        const int kxx = p.x_k_period > 0 ? kx % p.x_k_period : kx;  // X's k coordinate
        if (!kSwap) {
          tma_load_2d(&tmX, &full[stage], sa, kxx, c.row0);
          if (p.l2_hints) {
            const uint64_t pol = l2_policy_evict_first();
            tma_load_2d_hint(&tmW, &full[stage], sb, kx, wrow, pol);
            if (S::kDual)
              tma_load_2d_hint(&tmW, &full[stage], sb + (BN / 2) * 128, kx, wrow + p.Nw / 2, pol);
          } else {
            tma_load_2d(&tmW, &full[stage], sb, kx, wrow);
            if (S::kDual) tma_load_2d(&tmW, &full[stage], sb + (BN / 2) * 128, kx, wrow + p.Nw / 2);
          }
        } else {
          tma_load_2d(&tmW, &full[stage], sa, kx, wrow);
          if (S::kDual) tma_load_2d(&tmW, &full[stage], sa + 128 * 128, kx, wrow + p.Nw / 2);
          tma_load_2d(&tmX, &full[stage], sb, kxx, c.row0);
        }
        issued[stage] = true;
        last_parity[stage] = phase;
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
    }
    // No copy may still be landing in shared memory when the CTA exits.
    for (int s = 0; s < kStages; ++s)
      if (issued[s]) mbar_wait(&full[s], last_parity[s]);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      uint32_t idesc = S::kIdesc;
      if (!kSwap && p.tail_m64) {
        const TileCoord c = decode_tile(t, s_seg, s_pref, G, FT, S::kCH, p.tile_order);
        if (c.nrows <= 64) idesc = S::kIdesc64;
      }
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1)) break;
      tc_fence_after();
      const uint32_t d = tmem_base + acc * S::kAccCols;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(tiles + stage * S::kStageBytes);
        const uint32_t b_addr = a_addr + S::kABytes;
#pragma unroll
        for (int k = 0; k < S::kBK / 16; ++k) {
          const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
          const uint64_t bdesc = smem_desc_k128(b_addr + 32 * k);
          tc_mma_bf16(d, smem_desc_k128(a_addr + 32 * k), bdesc, idesc, accum);
          if (kSwap && S::kDual)
            tc_mma_bf16(d + BN, smem_desc_k128(a_addr + 128 * 128 + 32 * k), bdesc, S::kIdesc,
                        accum);
        }
        tc_commit(&empty[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      tc_commit(&tfull[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    // Every MMA of this CTA has finished before TMEM is released.
    tc_commit(done);
    mbar_wait(done, 0);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint32_t acc = 0, acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      TileCoord c = decode_tile(t, s_seg, s_pref, G, FT, S::kCH, p.tile_order);
      if (!epilogue_all(mbar_wait(&tfull[acc], acc_phase))) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * S::kAccCols;
      const int f0 = c.ft * S::kFO;
      if constexpr (!kSwap) {
        const int rpw = (p.tail_m64 && c.nrows <= 64) ? 16 : 32;  // rows per warp (M = 64 / 128)
        const EpiOut eo{(kStageOut && p.out_tma) ? &tmO : nullptr, stage_out + q * 4096,
                        rpw == 32 && c.nrows >= q * 32 + 32, p.l2_hints != 0};
        epilogue_rows<BN, kEpi>(p, c.row0, c.nrows, f0, tbase, q, lane, s_coef, eo, rpw);
      } else {
        // swap orientation: this thread owns output feature f for the BN rows of the chunk
        const int f = f0 + q * 32 + lane;
        float coefA = 1.0f, coefB = 0.0f, gsc = 1.0f;
        if constexpr (kEpi == EPI_STORE) gsc = p.gamma ? (1.0f + p.gamma[f]) : 1.0f;
        if constexpr (kEpi == EPI_RESGATE) {
          const float g = p.gparam ? p.gparam[f] : 0.0f;
          if (p.resid_mode == MOE_RESID_MUSE_GATE) {
            coefB = sigmoidf_(g / p.tau);
            coefA = sqrtf(fmaxf(sigmoidf_(-g / p.tau) * (1.0f + coefB), p.floor_));
          } else if (p.resid_mode == MOE_RESID_LITERAL) {
            coefA = 1.0f;
            coefB = g;
          }
        }
        uint16_t* out = static_cast<uint16_t*>(p.out);
        for (int j0 = 0; j0 < BN; j0 += 16) {
          float v[16];
          tmem_ld16(tbase + j0, v);
          if constexpr (kEpi == EPI_SWIGLU) {
            float uv[16];
            tmem_ld16(tbase + BN + j0, uv);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = silu(v[i]) * uv[i];
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int j = j0 + i;
            if (j < c.nrows) {
              const size_t row = static_cast<size_t>(c.row0 + j);
              float x = v[i];
              if constexpr (kEpi == EPI_RELU) x = fmaxf(x, 0.0f);
              if constexpr (kEpi == EPI_STORE) {
                if (p.gamma) x = round_bf16(x) * gsc;
                if (p.row_ss) {  // sum of squares over this warp's 32 features (fixed tree order)
                  const float b = round_bf16(x);
                  float sq = b * b;
#pragma unroll
                  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
                  if (lane == 0) p.row_ss[row * p.ss_parts + (f0 / 128) * 4 + q] = sq;
                }
              }
              if constexpr (kEpi == EPI_RESGATE) {
                const float b = round_bf16(x);
                if (p.resid_mode == MOE_RESID_NONE) x = b;
                else x = coefA * bf16_to_f32(p.resid[row * p.Nout + f]) + coefB * b;
              }
              out[row * p.Nout + f] = f32_to_bf16(x);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    // The staged stores have completed before the CTA (and its shared memory) goes away.
    if (kStageOut && lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

// ==================================================================== CTA-pair variant
//
// Normal orientation with a 256 x BN tile computed by the two CTAs of a cluster:
// tcgen05.mma.cta_group::2 (M = 256) issued by the leader, each CTA holding 128 rows of X and
// BN/2 rows of W in its own shared memory, each CTA's TMEM holding the accumulator of its 128
// rows.  Per SM this halves the W bytes staged and read per MMA, which is what bounds the 1-SM
// 128 x 256 tile (its TMA fill plus operand reads exceed the shared-memory bandwidth).
//   - Both CTAs load their halves with cta_group::2 TMA (no multicast); the bytes complete on
//     the leader's full barrier, whose expected count the leader sets for both halves.
//   - The leader's MMA commits arrive on both CTAs' empty / tmem-full barriers (multicast commit).
//   - Each CTA's epilogue drains its own TMEM lanes; one thread per CTA then arrives on the
//     leader's tmem-empty barrier (count 2).
//   - For SwiGLU the leader loads the 128 gate rows and the peer the 128 up rows, so accumulator
//     columns [0, 128) are the gate and [128, 256) the up projection, as in the 1-SM tile.

template <int BN, int kEpi>
struct PairShape {
  static constexpr bool kDual = (kEpi == EPI_SWIGLU);
  static constexpr int kBK = 64;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytes = (BN / 2) * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kFO = kDual ? BN / 2 : BN;
  static constexpr int kCH = 256;
  static constexpr int kTmemCols = 2 * BN <= 256 ? 256 : 512;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(256, BN);
  static_assert(BN == 128 || BN == 256, "pair tile width");
};

template <int BN, int kEpi, int kStages>
constexpr int gemm_pair_smem_bytes() {
  return kStages * PairShape<BN, kEpi>::kStageBytes + kStageOutBytes + 1024 + kSmemMisc;
}

template <int BN, int kEpi, int kStages>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ CUtensorMap tmO, const GemmParams p) {
  using S = PairShape<BN, kEpi>;
  static_assert(kEpi != EPI_ROUTER, "the pair kernel has bf16 epilogues only");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint8_t* stage_out = tiles + kStages * S::kStageBytes;  // 1024-byte aligned (stage multiple)
  uint64_t* full = reinterpret_cast<uint64_t*>(stage_out + kStageOutBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* s_seg = reinterpret_cast<int*>(tmem_slot + 4);
  int* s_pref = s_seg + (kMaxGroups + 4);
  float* s_coef = reinterpret_cast<float*>(s_pref + (kMaxGroups + 4));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int G = p.G;
  const int FT = p.Nout / S::kFO;
  const int KB = p.K / S::kBK;

  // Setup that reads nothing an earlier kernel writes (barriers, TMEM, the tensor-map prefetch)
  // runs before the dependency wait and overlaps the previous kernel's tail.
  if (threadIdx.x == 32) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 2); }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, S::kTmemCols);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  pdl_wait();
  pdl_launch_dependents();  // one CTA per SM, all resident: the next kernel may launch

  if (warp == 0) {  // group segments and tile prefix, as in the 1-SM kernel (256-row chunks)
    const int per = (G + 31) / 32;
    int local = 0;
    for (int j = 0; j < per; ++j) {
      int g = lane * per + j;
      if (g < G) {
        int a = p.seg ? p.seg[g] : 0, b = p.seg ? p.seg[g + 1] : p.M;
        if (b < a) { latch_status(MOE_ERR_DEVICE_CHECK); b = a; }
        s_seg[g] = a;
        if (g == G - 1) s_seg[G] = b;
        local += ((b - a + S::kCH - 1) / S::kCH) * FT;
      }
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - local;
    for (int j = 0; j < per; ++j) {
      int g = lane * per + j;
      if (g < G) {
        int a = p.seg ? p.seg[g] : 0, b = p.seg ? p.seg[g + 1] : p.M;
        if (b < a) b = a;
        s_pref[g] = run;
        run += ((b - a + S::kCH - 1) / S::kCH) * FT;
      }
    }
    if (lane == 31) s_pref[G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before any remote arrive or TMA completion
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_pref[G];

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    uint32_t stage = 0, phase = 0;
    uint32_t last_parity[kStages];
    bool issued[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) { issued[s] = false; last_parity[s] = 0; }
    bool ok = true;
    for (int t = pair; t < total && ok; t += npairs) {
      TileCoord c = decode_tile(t, s_seg, s_pref, G, FT, S::kCH, p.tile_order);
      const int xrow = c.row0 + 128 * static_cast<int>(rank);
      const int wrow = S::kDual ? c.g * p.Nw + (leader ? 0 : p.Nw / 2) + c.ft * (BN / 2)
                                : c.g * p.Nw + c.ft * BN + static_cast<int>(rank) * (BN / 2);
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
        uint8_t* sa = tiles + stage * S::kStageBytes;
        uint8_t* sb = sa + S::kABytes;
        if (leader) mbar_arrive_expect_tx(&full[stage], 2 * S::kStageBytes);
        const uint32_t fb = cluster_addr(&full[stage], 0);
        const int kx = kb * S::kBK;
        tma_load_2d_pair(&tmX, fb, sa, kx, xrow);
        tma_load_2d_pair(&tmW, fb, sb, kx, wrow);
        issued[stage] = true;
        last_parity[stage] = phase;
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
    }
    // The leader's full barriers count both CTAs' bytes: no copy is still landing afterwards.
    if (leader)
      for (int s = 0; s < kStages; ++s)
        if (issued[s]) mbar_wait(&full[s], last_parity[s]);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (leader) {
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(tiles + stage * S::kStageBytes);
          const uint32_t b_addr = a_addr + S::kABytes;
#pragma unroll
          for (int k = 0; k < S::kBK / 16; ++k)
            tc_mma_bf16_pair(d, smem_desc_k128(a_addr + 32 * k), smem_desc_k128(b_addr + 32 * k),
                             S::kIdesc, (kb | k) != 0);
          tc_commit_pair(&empty[stage], 0x3);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit_pair(&tfull[acc], 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      tc_commit_pair(done, 0x3);  // both CTAs learn that every pair MMA has finished
    }
    mbar_wait(done, 0);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    uint32_t acc = 0, acc_phase = 0;
    const uint32_t tempty_leader = cluster_addr(&tempty[0], 0);
    for (int t = pair; t < total; t += npairs) {
      TileCoord c = decode_tile(t, s_seg, s_pref, G, FT, S::kCH, p.tile_order);
      const int row0 = c.row0 + 128 * static_cast<int>(rank);
      const int nrows = max(0, min(128, c.nrows - 128 * static_cast<int>(rank)));
      if (!epilogue_all(mbar_wait(&tfull[acc], acc_phase))) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
      const EpiOut eo{p.out_tma ? &tmO : nullptr, stage_out + q * 4096, nrows >= q * 32 + 32,
                      p.l2_hints != 0};
      epilogue_rows<BN, kEpi>(p, row0, nrows, c.ft * S::kFO, tbase, q, lane, s_coef, eo);
      tc_fence_before();
      epilogue_bar();  // all 128 epilogue threads have finished reading this accumulator
      if (threadIdx.x == 64) {
        if (leader) mbar_arrive(&tempty[acc]);
        else mbar_arrive_cluster(tempty_leader + acc * static_cast<uint32_t>(sizeof(uint64_t)));
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (lane == 0) bulk_wait_all();  // staged stores complete before the CTA leaves
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the pair's MMAs may still use its memory
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, S::kTmemCols);
  }
}

}  // namespace moe
