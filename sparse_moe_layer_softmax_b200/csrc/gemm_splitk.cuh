// Dense projection of a few rows (at most 64: a decode batch) with its reduction split over the
// CTAs of a thread-block cluster: the latent down-projection z_raw = u P_down^T and the latent
// up-projection with the residual gate, out = alpha * r + beta * dtype(y P_up^T) ("Muse Spark
// Open: Norm-Preserving Gates Are Not a Norm Guarantee", sections "Latent experts" and
// "Residual gates").
//
// At this size the weight stream is the whole cost (67 MB per projection), and the 128-row weight
// tiles of a 4096- or 8192-wide output number only 32 or 64, fewer than the SMs.  So each
// 128-feature tile is shared by the S CTAs of one cluster, CTA s streaming k-blocks
// [s K/S, (s+1) K/S) into its own TMEM accumulator (swapped orientation: 128 weight rows on the
// MMA's M side, the batch's rows on N).  The CTAs then add their fp32 partial tiles through
// distributed shared memory, in the fixed order s = 0, 1, ..., S-1, each finishing 128/S of the
// features: no partial sums go out to HBM and no second kernel runs.
//   - TMA loads without multicast; every mbarrier wait is bounded; the cluster barriers are
//     reached by every thread of every CTA, also after a wait ran out.
//   - The partial tile [rows][128] fp32 reuses the operand ring once the MMAs have finished.
#pragma once

#include "gemm_tc.cuh"

namespace moe {

constexpr int kSplitBN = 64;      // rows of the batch on the MMA's N side (all of them)
constexpr int kSplitStages = 8;
constexpr int kSplitMaxCluster = 8;
using SplitShape = GemmShape<true, kSplitBN, EPI_STORE>;

constexpr int gemm_splitk_smem_bytes() {
  return kSplitStages * SplitShape::kStageBytes + 1024 + 256;
}
static_assert(kSplitBN * 128 * 4 <= kSplitStages * SplitShape::kStageBytes,
              "the partial tile fits in the operand ring");

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t caddr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(caddr)
               : "memory");
  return v;
}

// Reduce + epilogue of one CTA of a cluster of NS: CTA `rank` finishes features
// [rank * 128/NS, (rank + 1) * 128/NS) of feature tile `ft` for every row, in vectors of 8
// features.  Thread (group g, row lane r) of the 128 epilogue threads takes features g*8 .. g*8+7
// of that part and rows r, r + nr, ... (8/NS rows); all of its loads (the NS partial tiles through
// distributed shared memory, the residual rows) are issued before the first sum, and the partials
// are added in the order s = 0, 1, ..., NS-1.
template <int kEpi, int NS>
__device__ __forceinline__ void splitk_reduce(const GemmParams& p, const float* part, uint32_t rank,
                                              int ft) {
  constexpr int kFs = 128 / NS, kGroups = kFs / 8, kNr = 128 / kGroups, kRows = kSplitBN / kNr;
  static_assert(kRows * kNr == kSplitBN && kGroups * 8 == kFs, "reduce layout");
  const int et = static_cast<int>(threadIdx.x) - 64;
  const int g = et % kGroups, r0 = et / kGroups;
  const int fl = static_cast<int>(rank) * kFs + g * 8;  // first feature within the tile
  const int col = ft * 128 + fl;
  float4 cur[NS][kRows][2];
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const uint32_t base = cluster_addr(part, static_cast<uint32_t>(s));
#pragma unroll
    for (int q = 0; q < kRows; ++q) {
      const int row = r0 + q * kNr;
      if (row < p.M) {
        const uint32_t off = base + static_cast<uint32_t>((row * 128 + fl) * 4);
        cur[s][q][0] = ld_cluster_f32x4(off);
        cur[s][q][1] = ld_cluster_f32x4(off + 16);
      }
    }
  }
  const bool has_r = kEpi == EPI_RESGATE && p.resid_mode != MOE_RESID_NONE;
  uint4 rv[kRows];
#pragma unroll
  for (int q = 0; q < kRows; ++q) {
    const int row = r0 + q * kNr;
    rv[q] = make_uint4(0, 0, 0, 0);
    if (row < p.M && has_r)
      rv[q] = __ldg(reinterpret_cast<const uint4*>(p.resid + static_cast<size_t>(row) * p.Nout + col));
  }
  float a[8], b[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    a[j] = 0.0f;
    b[j] = 1.0f;
    if constexpr (kEpi == EPI_RESGATE) {
      const float gg = p.gparam ? p.gparam[col + j] : 0.0f;
      if (p.resid_mode == MOE_RESID_MUSE_GATE) {
        b[j] = sigmoidf_(gg / p.tau);
        a[j] = sqrtf(fmaxf(sigmoidf_(-gg / p.tau) * (1.0f + b[j]), p.floor_));
      } else if (p.resid_mode == MOE_RESID_LITERAL) {
        a[j] = 1.0f;
        b[j] = gg;
      }
    }
  }
  uint16_t* out = static_cast<uint16_t*>(p.out);
#pragma unroll
  for (int q = 0; q < kRows; ++q) {
    const int row = r0 + q * kNr;
    if (row >= p.M) continue;
    float v[8] = {cur[0][q][0].x, cur[0][q][0].y, cur[0][q][0].z, cur[0][q][0].w,
                  cur[0][q][1].x, cur[0][q][1].y, cur[0][q][1].z, cur[0][q][1].w};
#pragma unroll
    for (int s = 1; s < NS; ++s) {
      v[0] += cur[s][q][0].x; v[1] += cur[s][q][0].y; v[2] += cur[s][q][0].z; v[3] += cur[s][q][0].w;
      v[4] += cur[s][q][1].x; v[5] += cur[s][q][1].y; v[6] += cur[s][q][1].z; v[7] += cur[s][q][1].w;
    }
    const uint16_t* rh = reinterpret_cast<const uint16_t*>(&rv[q]);
    uint4 o;
    uint16_t* oh = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float x = v[j];
      if constexpr (kEpi == EPI_RESGATE)
        x = __fmaf_rn(a[j], bf16_to_f32(rh[j]), __fmul_rn(b[j], round_bf16(x)));
      oh[j] = f32_to_bf16(x);
    }
    *reinterpret_cast<uint4*>(out + static_cast<size_t>(row) * p.Nout + col) = o;
  }
}

// kEpi: EPI_STORE (out = dtype(sum)) or EPI_RESGATE (out = dtype(alpha r + beta dtype(sum))).
// Grid: (Nout / 128) * S CTAs in clusters of S (2 <= S <= 8, S divides K / 64); rows p.M <= kSplitBN.
template <int kEpi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_splitk_cluster_kernel(const __grid_constant__ CUtensorMap tmX,
                               const __grid_constant__ CUtensorMap tmW, const GemmParams p) {
  static_assert(kEpi == EPI_STORE || kEpi == EPI_RESGATE, "dense projection epilogues");
  using S = SplitShape;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  float* part = reinterpret_cast<float*>(tiles);  // after the MMAs: [kSplitBN rows][128 features]
  uint64_t* full = reinterpret_cast<uint64_t*>(tiles + kSplitStages * S::kStageBytes);
  uint64_t* empty = full + kSplitStages;
  uint64_t* tfull = empty + kSplitStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int ns = static_cast<int>(cluster_nctarank());
  const int ft = static_cast<int>(blockIdx.x) / ns;
  const int kbs = p.K / S::kBK / ns;
  const int kb0 = static_cast<int>(rank) * kbs;

  // Setup that reads nothing an earlier kernel writes runs before the dependency wait.
  if (threadIdx.x == 32) {
    for (int s = 0; s < kSplitStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(tfull, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kSplitBN);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  pdl_wait();
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    uint32_t stage = 0, phase = 0;
    uint32_t last_parity[kSplitStages];
    bool issued[kSplitStages];
#pragma unroll
    for (int s = 0; s < kSplitStages; ++s) { issued[s] = false; last_parity[s] = 0; }
    for (int kb = kb0; kb < kb0 + kbs; ++kb) {
      if (!mbar_wait(&empty[stage], phase ^ 1)) break;
      uint8_t* sa = tiles + stage * S::kStageBytes;
      mbar_arrive_expect_tx(&full[stage], S::kStageBytes);
      tma_load_2d(&tmW, &full[stage], sa, kb * S::kBK, ft * 128);
      tma_load_2d(&tmX, &full[stage], sa + S::kABytes, kb * S::kBK, 0);
      issued[stage] = true;
      last_parity[stage] = phase;
      if (++stage == kSplitStages) { stage = 0; phase ^= 1; }
    }
    // No copy may still be landing in the ring once the partial tile is written there.
    for (int s = 0; s < kSplitStages; ++s)
      if (issued[s]) mbar_wait(&full[s], last_parity[s]);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t stage = 0, phase = 0;
    for (int kb = kb0; kb < kb0 + kbs; ++kb) {
      if (!mbar_wait(&full[stage], phase)) break;
      tc_fence_after();
      const uint32_t a_addr = smem_u32(tiles + stage * S::kStageBytes);
      const uint32_t b_addr = a_addr + S::kABytes;
#pragma unroll
      for (int k = 0; k < S::kBK / 16; ++k)
        tc_mma_bf16(tmem_base, smem_desc_k128(a_addr + 32 * k), smem_desc_k128(b_addr + 32 * k),
                    S::kIdesc, (kb > kb0 || k > 0) ? 1u : 0u);
      tc_commit(&empty[stage]);
      if (++stage == kSplitStages) { stage = 0; phase ^= 1; }
    }
    // Arrives when every MMA issued above has finished (and with them every operand load the
    // producer issued, each of which an MMA waited for), so the ring may be overwritten; the
    // issuer waits for it too, so no MMA is in flight when TMEM is released.
    tc_commit(tfull);
    mbar_wait(tfull, 0);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ partial tile to shared memory
    const int q = warp & 3;  // TMEM lane quarter: features 32q .. 32q + 31
    mbar_wait(tfull, 0);
    tc_fence_after();
    const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const int f = q * 32 + lane;
#pragma unroll 1
    for (int j0 = 0; j0 < kSplitBN; j0 += 16) {
      float v[16];
      tmem_ld16(tb + j0, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) part[(j0 + i) * 128 + f] = v[i];
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // every CTA's partial tile is complete and visible to the cluster

  if (warp >= 2) {
    // ------------------------------------------------------------ reduce + epilogue
    switch (ns) {
      case 2: splitk_reduce<kEpi, 2>(p, part, rank, ft); break;
      case 4: splitk_reduce<kEpi, 4>(p, part, rank, ft); break;
      default: splitk_reduce<kEpi, 8>(p, part, rank, ft); break;
    }
  }
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while a peer may still read its partial tile
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kSplitBN);
  }
}

}  // namespace moe
