// Grouped GEMM on CTA pairs: tcgen05.mma.cta_group::2 with M = 256 per pair.
//
// Same problem and epilogues as grouped_gemm.cuh (gate/up + clipped SwiGLU,
// down + routing weight + un-permutation), but each MMA spans the two CTAs of a
// cluster: every CTA stages its own 128 rows of A and half of the N = 240 rows
// of B, so a CTA's shared memory carries 31 KB per 64-wide K step instead of
// 46 KB for the same MMA work.  For gate/up the halves are the two projections:
// the leader CTA holds the gate tile and its peer the up tile, so TMEM columns
// [0, 120) are g and [120, 240) are u for both CTAs' rows.  For down the halves
// are output columns [n0, n0+120) and [n0+120, n0+240).
//
// Roles (192 threads per CTA, both CTAs):
//   warp 0     TMA producer: loads this CTA's A and B halves; completion bytes
//              are counted on the leader's `full` barrier, which only the
//              leader arms (with both CTAs' bytes).
//   warp 1     TMEM (512 columns, pair allocation); in the leader, one thread
//              issues the pair MMAs and multicasts each commit to both CTAs
//              (`empty` stage release, `tfull` accumulator ready).
//   warps 2-5  epilogue on this CTA's 128 accumulator rows; one lane per warp
//              then arrives on the leader's `tempty` (8 arrivals per tile).
// Tiles: (expert, 256-row block, output-column block), numbered as in the
// single-CTA kernel, walked by clusters with a grid stride.
// All waits are bounded; a cluster barrier closes the kernel so neither CTA
// leaves while its peer may still signal its barriers.
#pragma once

#include "grouped_gemm.cuh"

namespace moe {

constexpr int kPairBM = 256;        // rows per pair tile (MMA M)
constexpr int kPairBand = 8;        // pair row blocks per band in the tile order

template <int TNH>
struct PairLayout {
  static constexpr int A_BYTES = 128 * kRowBytes;
  static constexpr int B_BYTES = TNH * kRowBytes;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static_assert(TNH % 8 == 0 && (2 * TNH) % 16 == 0 && 2 * TNH <= 256, "pair MMA N = 2 * TNH");
  static constexpr int EXTRA = 1024 + 4096;
  static constexpr int smem_bytes(int stages) { return stages * STAGE_BYTES + EXTRA; }
};

__device__ __forceinline__ TileInfo decode_pair_tile(int i, const int* tile_off, const int* goff, int G, int NT,
                                                     int TNO) {
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_off[mid] * NT <= i) lo = mid; else hi = mid;
  }
  const int MT = tile_off[lo + 1] - tile_off[lo];
  const int local = i - tile_off[lo] * NT;
  const int band = local / (kPairBand * NT);
  const int rem = local - band * kPairBand * NT;
  const int rows = min(kPairBand, MT - band * kPairBand);
  const int nt = rem / rows;
  const int mt = band * kPairBand + (rem - nt * rows);
  TileInfo t;
  t.g = lo;
  t.m0 = goff[lo] + mt * kPairBM;
  t.m_end = goff[lo + 1];
  t.n0 = nt * TNO;
  return t;
}

// EPI: EPI_SWIGLU (B halves = gate | up, TNO = TNH output columns per tile) or
//      EPI_BIAS / EPI_BIAS_WSCATTER (B halves = two column blocks, TNO = 2 * TNH).
template <int TNH, int EPI, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                             const __grid_constant__ CUtensorMap tmB1, const GemmArgs args) {
  pdl_enter();
  using T = __nv_bfloat16;
  using LY = PairLayout<TNH>;
  constexpr int BK = kRowBytes / 2;
  constexpr int KSTEPS = kRowBytes / 32;
  constexpr int TNO = (EPI == EPI_SWIGLU) ? TNH : 2 * TNH;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * LY::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* never_flag = abort_flag + 1;
  int* tile_off = never_flag + 2;
  int* goff = tile_off + (kMaxGroups + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();          // 0 = leader (issues the MMAs)
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int G = args.num_groups;
  const int NT = (args.n_out + TNO - 1) / TNO;
  const int KB = (args.k_dim + BK - 1) / BK;
  // down over h kept as two bf16 halves: K blocks [0, KB) read hi, [KB, 2 KB) lo (same weights)
  const bool hsplit = EPI != EPI_SWIGLU && args.h_halves == 2;
  const int KBT = hsplit ? 2 * KB : KB;
  const uint64_t lim = args.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&tfull[0], 1);
    mbar_init(&tfull[1], 1);
    mbar_init(&tempty[0], 8);
    mbar_init(&tempty[1], 8);
    mbar_init(drain, 1);
    *abort_flag = 0;
    *never_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    int bad = 0;
    for (int g = lane; g <= G; g += 32) {
      int v = args.group_off[g];
      if (v < 0 || v > args.m_total) { bad = 1; v = min(max(v, 0), args.m_total); }
      goff[g] = v;
    }
    __syncwarp();
    int running = 0;
    if (lane == 0) tile_off[0] = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int cnt = 0;
      if (g < G) {
        const int rows = goff[g + 1] - goff[g];
        if (rows < 0) bad = 1;
        cnt = rows > 0 ? (rows + kPairBM - 1) / kPairBM : 0;
      }
      int incl = cnt;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += o;
      }
      if (g < G) tile_off[g + 1] = running + incl;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0 && rank == 0) flag_error(DEVERR_BOUNDS);
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB0);
      tma_prefetch_desc(&tmB1);
    }
  } else if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // barriers of both CTAs initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_off[G] * NT;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      const void* tmb = (EPI == EPI_SWIGLU && rank == 1) ? static_cast<const void*>(&tmB1)
                                                          : static_cast<const void*>(&tmB0);
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int i = cluster; ok && i < total; i += nclusters) {
        const TileInfo ti = decode_pair_tile(i, tile_off, goff, G, NT, TNO);
        const int a_row = ti.m0 + static_cast<int>(rank) * 128;
        const int b_row = (EPI == EPI_SWIGLU) ? ti.n0 : ti.n0 + static_cast<int>(rank) * TNH;
        for (int kb = 0; kb < KBT; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * LY::STAGE_BYTES);
          uint8_t* sa = smem + s * LY::STAGE_BYTES;
          uint8_t* sb = sa + LY::A_BYTES;
          const uint32_t fb = full_leader + static_cast<uint32_t>(s) * 8u;
          const int half = hsplit ? kb / KB : 0;
          const int kbl = kb - half * KB;
          if (hsplit) tma_load_3d_pair(sa, &tmA, fb, kbl * BK, half, a_row);
          else tma_load_2d_pair(sa, &tmA, fb, kb * BK, a_row);
          tma_load_3d_pair(sb, tmb, fb, kbl * BK, b_row, ti.g);
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(DEVERR_TIMEOUT);
        // the peer's barrier cannot be polled from here: give loads in flight time to land
        for (int q = 0; q < 2000; ++q) __nanosleep(1000);
      }
      if (rank == 0) {
        for (int q = 0; q < STAGES; ++q)
          if ((issued >> q) & 1u)
            if (!mbar_wait(&full[q], (issued_par >> q) & 1u, never_flag, kDrainLimitNs)) flag_error(DEVERR_TIMEOUT);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (rank == 0 && lane == 0) {
      const uint32_t idesc = make_idesc(kPairBM, 2 * TNH, 1u);
      int s = 0, it = 0;
      uint32_t ph = 0;
      bool ok = true;
      bool issued_any = false;
      for (int i = cluster; ok && i < total; i += nclusters, ++it) {
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait_cluster(&tempty[acc], aph ^ 1u, abort_flag, lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccStride);
        for (int kb = 0; kb < KBT; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * LY::STAGE_BYTES);
          const uint32_t b_addr = a_addr + LY::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk)
            tc_mma_pair(d_tmem, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), idesc,
                        (kb | kk) != 0 ? 1u : 0u);
          issued_any = true;
          tc_commit_pair_mc(&empty[s], 0x3);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_mc(&tfull[acc], 0x3);
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(DEVERR_TIMEOUT);
      }
      if (issued_any) {
        tc_commit_pair(drain);
        if (!mbar_wait(drain, 0, never_flag, kDrainLimitNs)) flag_error(DEVERR_TIMEOUT);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int r_in_tile = static_cast<int>(rank) * 128 + quarter * 32 + lane;
    const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);
    int it = 0;
    bool ok = true;
    for (int i = cluster; i < total; i += nclusters, ++it) {
      const TileInfo ti = decode_pair_tile(i, tile_off, goff, G, NT, TNO);
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, abort_flag, lim));
      if (!got) { ok = false; break; }
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kAccStride);
      const int row = ti.m0 + r_in_tile;
      const bool rvalid = row < ti.m_end;
      if constexpr (EPI == EPI_SWIGLU) epi_swiglu<T, TNH>(tbase, row, rvalid, ti, args);
      else if constexpr (EPI == EPI_BIAS) epi_bias<T, 2 * TNH, false>(tbase, row, rvalid, ti, args);
      else epi_bias<T, 2 * TNH, true>(tbase, row, rvalid, ti, args);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + static_cast<uint32_t>(acc) * 8u);
    }
    if (!ok) {
      *abort_flag = 1;
      flag_error(DEVERR_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // no CTA leaves while its peer may still signal it or read its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace moe
