// Grouped expert GEMM for prefill-sized groups on CTA pairs, weights on the MMA's M side:
//
//   out[r, f] = epi( sum_k X[r, k] * W[g*Nw + f', k] )   for rows r of group g
//
// One tile is 256 weight rows (M, 128 in each CTA of the pair) by up to 256 rows of X (N, the
// tile's token rows split in halves between the two CTAs), issued as
// tcgen05.mma.cta_group::2 by the pair leader.  Putting the tokens on N lets a tile end where its
// group ends, to 16 rows: a group's m rows are cut into ceil(m/256) chunks of equal size (rounded
// up to 16), so at most 15 padding rows per chunk are multiplied, against up to 127 for 128-row
// activation tiles.  Per SM the pair reads half the operand bytes of a 1-SM 128x256 tile from
// shared memory per MMA (each CTA stages 128 weight rows and half of the token rows).
//
//   - SwiGLU: each CTA's 128 weight rows are 64 gate rows and the same 64 features' up rows, so
//     its accumulator holds the gate in TMEM lanes 0-63 and the up projection in lanes 64-127.
//     The epilogue warps of lane quarters q and q^2 hold gate and up of the same 32 features and
//     trade alternate 16-token blocks through shared memory.
//   - STORE (expert down, optional gain (1 + gamma) and per-row partial sums of squares over the
//     CTA's 128 features) and RELU.
//   - Each thread owns one output feature; a warp writes 32 consecutive features (64 bytes) of a
//     token row per store, so a tile's last, partial 16-token block stores only its valid rows.
//   - Loads: TMA without multicast, both CTAs' bytes counted on the leader's full barrier; the
//     leader's commits arrive on both CTAs' barriers; each CTA's epilogue drains its own TMEM.
//   - Every mbarrier wait is bounded; on a timeout the roles stop issuing and wind down as in
//     the other GEMM kernels.
#pragma once

#include "gemm_tc.cuh"

namespace moe {

template <int kEpi>
struct SwapPairShape {
  static constexpr bool kDual = (kEpi == EPI_SWIGLU);
  static constexpr int kBK = 64;                      // 128 bytes of bf16
  static constexpr int kABytes = 128 * 128;           // 128 weight rows per CTA
  static constexpr int kBBytes = 128 * 128;           // up to 128 token rows per CTA
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kFO = kDual ? 128 : 256;       // output features per pair tile
  static constexpr int kMaxN = 256;                   // token rows per pair tile
  static constexpr int kTmemCols = 512;               // two accumulators of kMaxN columns
  static constexpr int kWBoxRows = kDual ? 64 : 128;  // weight rows per TMA box
  static constexpr int kXchgBytes = kDual ? 4 * 16 * 32 * 4 : 0;  // SwiGLU exchange buffers
  static constexpr int kSsBytes = 4 * kMaxN * 4;                  // per-warp row partials
};

template <int kEpi, int kStages>
constexpr int gemm_swap_pair_smem_bytes() {
  using S = SwapPairShape<kEpi>;
  return kStages * S::kStageBytes + S::kXchgBytes + S::kSsBytes + 1024 + kSmemMisc;
}

// Tile t of the swapped pair schedule: group g, feature tile ft, token rows [row0, row0 + nrows)
// and the MMA width n (nrows rounded up to 16).  A group of m rows has ceil(m/256) chunks of cs =
// roundup16(ceil(m / chunks)) rows (the last may be shorter; (chunks - 1) * cs < m, so none is
// empty); its tiles run (feature tile, chunk) with the chunk fastest.
struct SwapTile {
  int g, ft, row0, nrows, n;
};

__device__ __forceinline__ int swap_chunks(int m) { return (m + 255) >> 8; }

__device__ __forceinline__ SwapTile decode_swap_tile(int t, const int* s_seg, const int* s_pref,
                                                     int G) {
  int lo = 0, hi = G;
  while (lo < hi) {  // last g with s_pref[g] <= t
    int mid = (lo + hi + 1) >> 1;
    if (s_pref[mid] <= t) lo = mid; else hi = mid - 1;
  }
  SwapTile c;
  c.g = lo;
  const int m = s_seg[lo + 1] - s_seg[lo];
  const int nch = swap_chunks(m);
  const int cs = (((m + nch - 1) / nch) + 15) & ~15;
  const int local = t - s_pref[lo];
  c.ft = local / nch;
  const int chunk = local - c.ft * nch;
  c.row0 = s_seg[lo] + chunk * cs;
  const int rem = s_seg[lo + 1] - c.row0;
  c.nrows = rem < cs ? rem : cs;
  c.n = (c.nrows + 15) & ~15;
  return c;
}

// Sums v[0..15] of every lane over the 32 lanes of the warp, for each of the 16 indices, with 16
// shuffles (a butterfly that halves the values each lane keeps).  Returns the sum of index
// swap_ss_index(lane); lanes l and l ^ 1 return the same index.  The order of the additions
// depends only on the lane positions, so it is the same for every tile.
template <int W, int kBit>
__device__ __forceinline__ void halve_sum(float (&v)[16], int lane) {
  // keep W values: the upper half when this lane's kBit is set, else the lower half
  const bool upper = (lane & kBit) != 0;
#pragma unroll
  for (int i = 0; i < W; ++i) {
    const float send = upper ? v[i] : v[i + W];
    const float keep = upper ? v[i + W] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, kBit);
  }
}
__device__ __forceinline__ float warp_transpose_sum16(float (&v)[16], int lane) {
  halve_sum<8, 16>(v, lane);
  halve_sum<4, 8>(v, lane);
  halve_sum<2, 4>(v, lane);
  halve_sum<1, 2>(v, lane);
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}
__device__ __forceinline__ int swap_ss_index(int lane) {
  return ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
}

// Named barrier of the two epilogue warps of lane quarters q and q ^ 2 (ids 2 and 3).
__device__ __forceinline__ void xchg_bar(int q) {
  asm volatile("bar.sync %0, 64;" ::"r"(2 + (q & 1)) : "memory");
}

// 16 consecutive token columns [c0, c0 + 16) of this thread's TMEM lane.
__device__ __forceinline__ void swap_ld16(uint32_t tbase, int c0, float* v) { tmem_ld16(tbase + c0, v); }

template <int kEpi, int kStages>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_swap_pair_kernel(const __grid_constant__ CUtensorMap tmX,
                          const __grid_constant__ CUtensorMap tmW, const GemmParams p) {
  using S = SwapPairShape<kEpi>;
  static_assert(kEpi == EPI_SWIGLU || kEpi == EPI_STORE || kEpi == EPI_RELU,
                "the swapped pair kernel has the expert epilogues");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  float* xchg = reinterpret_cast<float*>(tiles + kStages * S::kStageBytes);  // [4][16][32]
  float* ssbuf = reinterpret_cast<float*>(tiles + kStages * S::kStageBytes + S::kXchgBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(tiles + kStages * S::kStageBytes + S::kXchgBytes +
                                               S::kSsBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* s_seg = reinterpret_cast<int*>(tmem_slot + 4);
  int* s_pref = s_seg + (kMaxGroups + 4);

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
  pdl_launch_dependents();  // every CTA is resident: the next kernel may launch

  if (warp == 0) {  // group segments and the per-group tile prefix
    const int per = (G + 31) / 32;
    int local = 0;
    for (int j = 0; j < per; ++j) {
      int g = lane * per + j;
      if (g < G) {
        int a = p.seg ? p.seg[g] : 0, b = p.seg ? p.seg[g + 1] : p.M;
        if (b < a) { latch_status(MOE_ERR_DEVICE_CHECK); b = a; }
        s_seg[g] = a;
        if (g == G - 1) s_seg[G] = b;
        local += swap_chunks(b - a) * FT;
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
        run += swap_chunks(b - a) * FT;
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
      const SwapTile c = decode_swap_tile(t, s_seg, s_pref, G);
      // this CTA's weight rows and its half of the tile's token rows
      const int wrow = S::kDual ? c.g * p.Nw + c.ft * 128 + 64 * static_cast<int>(rank)
                                : c.g * p.Nw + c.ft * 256 + 128 * static_cast<int>(rank);
      const int xrow = c.row0 + static_cast<int>(rank) * (c.n >> 1);
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
        uint8_t* sa = tiles + stage * S::kStageBytes;
        uint8_t* sb = sa + S::kABytes;
        if (leader) mbar_arrive_expect_tx(&full[stage], 2 * S::kStageBytes);
        const uint32_t fb = cluster_addr(&full[stage], 0);
        const int kx = kb * S::kBK;
        tma_load_2d_pair(&tmW, fb, sa, kx, wrow);
        if (S::kDual) tma_load_2d_pair(&tmW, fb, sa + 64 * 128, kx, wrow + p.Nw / 2);
        tma_load_2d_pair(&tmX, fb, sb, kx, xrow);
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
        const SwapTile c = decode_swap_tile(t, s_seg, s_pref, G);
        const uint32_t idesc = idesc_bf16_f32(256, c.n);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * S::kMaxN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(tiles + stage * S::kStageBytes);
          const uint32_t b_addr = a_addr + S::kABytes;
#pragma unroll
          for (int k = 0; k < S::kBK / 16; ++k)
            tc_mma_bf16_pair(d, smem_desc_k128(a_addr + 32 * k), smem_desc_k128(b_addr + 32 * k),
                             idesc, (kb | k) != 0);
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
    const int q = warp & 3;  // TMEM lane quarter of this warp
    uint32_t acc = 0, acc_phase = 0;
    const uint32_t tempty_leader = cluster_addr(&tempty[0], 0);
    uint16_t* out = static_cast<uint16_t*>(p.out);
    for (int t = pair; t < total; t += npairs) {
      const SwapTile c = decode_swap_tile(t, s_seg, s_pref, G);
      if (!epilogue_all(mbar_wait(&tfull[acc], acc_phase))) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * S::kMaxN;
      const int nblk = c.n >> 4;  // 16-token blocks of the tile
      if constexpr (S::kDual) {
        // lanes 0-63 gate, 64-127 up, of features f .. f + 63; quarter q and q ^ 2 pair up
        const bool gate = q < 2;
        const int f = c.ft * 128 + 64 * static_cast<int>(rank) + (q & 1) * 32 + lane;
        float* mine = xchg + q * (16 * 32);
        const float* theirs = xchg + (q ^ 2) * (16 * 32);
        for (int b0 = 0; b0 < nblk; b0 += 2) {
          // block b0 is produced by the gate warp, block b0 + 1 (if any) by the up warp; each
          // hands the other the block it does not produce
          const bool has2 = b0 + 1 < nblk;
          float own[16], other[16];
          const int own_blk = gate ? b0 : b0 + 1;
          const int give_blk = gate ? b0 + 1 : b0;
          if (gate || has2) swap_ld16(tbase, own_blk * 16, own);
          if (!gate || has2) {
            swap_ld16(tbase, give_blk * 16, other);
#pragma unroll
            for (int i = 0; i < 16; ++i) mine[i * 32 + lane] = other[i];
          }
          xchg_bar(q);
          if (gate || has2) {
            const int tok0 = own_blk * 16;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float pv = theirs[i * 32 + lane];  // the partner's half of the pair
              const float gv = gate ? own[i] : pv;
              const float uv = gate ? pv : own[i];
              const int tok = tok0 + i;
              if (tok < c.nrows)
                out[static_cast<size_t>(c.row0 + tok) * p.Nout + f] = f32_to_bf16(silu(gv) * uv);
            }
          }
          xchg_bar(q);  // both warps are done with the exchange buffers of this block pair
        }
      } else {
        const int f = c.ft * 256 + 128 * static_cast<int>(rank) + q * 32 + lane;
        const float gsc = (kEpi == EPI_STORE && p.gamma) ? 1.0f + p.gamma[f] : 1.0f;
        // (ssbuf is free: every reader of the previous tile's partials passed the barrier that
        // ends that tile)
        const bool want_ss = kEpi == EPI_STORE && p.row_ss != nullptr;
        for (int b = 0; b < nblk; ++b) {
          float v[16];
          swap_ld16(tbase, b * 16, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if constexpr (kEpi == EPI_RELU) v[i] = fmaxf(v[i], 0.0f);
            if constexpr (kEpi == EPI_STORE) {
              if (p.gamma) v[i] = round_bf16(v[i]) * gsc;
            }
            const int tok = b * 16 + i;
            if (tok < c.nrows) out[static_cast<size_t>(c.row0 + tok) * p.Nout + f] = f32_to_bf16(v[i]);
          }
          if (want_ss) {
            float sq[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float r = round_bf16(v[i]);
              sq[i] = r * r;
            }
            const float tot = warp_transpose_sum16(sq, lane);
            if ((lane & 1) == 0) ssbuf[q * S::kMaxN + b * 16 + swap_ss_index(lane)] = tot;
          }
        }
        if (want_ss) {
          epilogue_bar();  // the four warps' partials of every token are in ssbuf
          const int part = c.ft * 2 + static_cast<int>(rank);  // this CTA's 128 features
          for (int tok = static_cast<int>(threadIdx.x) - 64; tok < c.nrows; tok += 128) {
            const float s = ((ssbuf[tok] + ssbuf[S::kMaxN + tok]) + ssbuf[2 * S::kMaxN + tok]) +
                            ssbuf[3 * S::kMaxN + tok];
            p.row_ss[static_cast<size_t>(c.row0 + tok) * p.ss_parts + part] = s;
          }
        }
      }
      tc_fence_before();
      epilogue_bar();  // all 128 epilogue threads have finished reading this accumulator
      if (threadIdx.x == 64) {
        if (leader) mbar_arrive(&tempty[acc]);
        else mbar_arrive_cluster(tempty_leader + acc * static_cast<uint32_t>(sizeof(uint64_t)));
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
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
