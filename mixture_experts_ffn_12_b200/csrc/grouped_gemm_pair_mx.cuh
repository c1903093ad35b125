// CTA-pair grouped GEMM with MXFP4 expert weights dequantised inside the mainloop.
//
// Same tiles, roles and epilogues as grouped_gemm_pair.cuh, plus four converter
// warps per CTA.  Per stage each CTA receives, by TMA, its 128 rows of A (bf16,
// 128-byte swizzle) and its 120 rows of packed E2M1 weights (32 bytes = 64 codes
// per row); the converters turn the packed rows into the bf16 swizzled tile the
// MMA reads, each value being the E2M1 code times the row's E8M0 block scale
// 2^(s-127) for its 32-element block along K (OCP MX encoding: code bit 3 sign,
// bits 2..1 exponent with bias 1, bit 0 mantissa; element 2i in the low nibble of
// byte i).  Every decoded value is a bf16 number, so the MMA sees exactly the
// dequantised weights.  The leader's MMA waits for both CTAs' A bytes (`full`) and
// both CTAs' converted halves (`conv`, 8 warp arrivals).
//
// Scale bytes (90 per row for K = 2880) are read from global memory by the
// converters, one k-block ahead, since rows that are not a multiple of 16 bytes
// cannot be described to TMA.
#pragma once

#include "grouped_gemm_pair.cuh"

namespace moe {

constexpr int kMxThreads = 320;     // 6 warps as in the bf16 kernels + 4 converter warps
constexpr int kMxConvThreads = 128;

template <int TNH>
struct PairMxLayout {
  static constexpr int A_BYTES = 128 * kRowBytes;            // bf16 activations
  static constexpr int B_BYTES = TNH * kRowBytes;            // dequantised bf16 weights
  static constexpr int P_BYTES = (TNH * 32 + 1023) / 1024 * 1024;   // packed E2M1 rows (32 B each)
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + P_BYTES;
  static constexpr int EXTRA = 1024 + 4096;
  static constexpr int smem_bytes(int stages) { return stages * STAGE_BYTES + EXTRA; }
};

// 8 E2M1 codes (one 32-bit word, element i in nibble i) times a bf16 scale -> 8 bf16 in a uint4.
__device__ __forceinline__ uint4 mxfp4_decode8(uint32_t w, __nv_bfloat162 scale2) {
  // bf16 bit patterns of the 8 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}: high and low bytes,
  // looked up with byte permutes (selector = the 3-bit magnitude of each code)
  constexpr uint32_t HI_A = 0x3F3F3F00u, HI_B = 0x40404040u;   // high bytes for m = 0..3 | 4..7
  constexpr uint32_t LO_A = 0xC0800000u, LO_B = 0xC0804000u;   // low bytes  for m = 0..3 | 4..7
  const uint32_t mag = w & 0x77777777u;
  const uint32_t hi0 = __byte_perm(HI_A, HI_B, mag & 0xFFFFu);
  const uint32_t lo0 = __byte_perm(LO_A, LO_B, mag & 0xFFFFu);
  const uint32_t hi1 = __byte_perm(HI_A, HI_B, mag >> 16);
  const uint32_t lo1 = __byte_perm(LO_A, LO_B, mag >> 16);
  uint32_t v[4];
  v[0] = __byte_perm(lo0, hi0, 0x5140u);   // elements 0, 1
  v[1] = __byte_perm(lo0, hi0, 0x7362u);   // elements 2, 3
  v[2] = __byte_perm(lo1, hi1, 0x5140u);   // elements 4, 5
  v[3] = __byte_perm(lo1, hi1, 0x7362u);   // elements 6, 7
  // sign of element i = bit 4i+3 of w -> bit 15 (even element) or 31 (odd element) of its word
  v[0] |= ((w << 12) & 0x00008000u) | ((w << 24) & 0x80000000u);
  v[1] |= ((w << 4) & 0x00008000u) | ((w << 16) & 0x80000000u);
  v[2] |= ((w >> 4) & 0x00008000u) | ((w << 8) & 0x80000000u);
  v[3] |= ((w >> 12) & 0x00008000u) | (w & 0x80000000u);
  uint4 out;
  uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&v[i]);
    x = __hmul2(x, scale2);   // exact: 3 significant bits times a power of two
    o[i] = *reinterpret_cast<uint32_t*>(&x);
  }
  return out;
}

// E8M0 byte -> 2^(s - 127) as bf16 (s = 0 is the subnormal 2^-127; 255 is not a number in MX).
__device__ __forceinline__ __nv_bfloat162 e8m0_to_bf16x2(uint32_t s) {
  const uint16_t bits = s == 0 ? uint16_t(0x0040) : (s == 255 ? uint16_t(0x7FC0) : uint16_t(s << 7));
  __nv_bfloat16 h = __ushort_as_bfloat16(bits);
  return __halves2bfloat162(h, h);
}

template <int TNH, int EPI, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMxThreads, 1)
    grouped_gemm_pair_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmP0,
                                const __grid_constant__ CUtensorMap tmP1, const GemmArgs args) {
  using T = __nv_bfloat16;
  using LY = PairMxLayout<TNH>;
  constexpr int BK = kRowBytes / 2;        // 64 K elements per stage
  constexpr int KSTEPS = kRowBytes / 32;
  constexpr int TNO = (EPI == EPI_SWIGLU) ? TNH : 2 * TNH;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * LY::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* pk = empty + STAGES;           // packed rows landed (local)
  uint64_t* conv = pk + STAGES;            // both CTAs' halves converted (leader, 8 arrivals)
  uint64_t* tfull = conv + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* never_flag = abort_flag + 1;
  int* tile_off = never_flag + 2;
  int* goff = tile_off + (kMaxGroups + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int G = args.num_groups;
  const int NT = (args.n_out + TNO - 1) / TNO;
  const int KB = (args.k_dim + BK - 1) / BK;
  const int KS = args.k_dim / 32;          // scale bytes per weight row
  const uint64_t lim = args.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&pk[s], 1);
      mbar_init(&conv[s], 8);
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
      tma_prefetch_desc(&tmP0);
      tma_prefetch_desc(&tmP1);
    }
  } else if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_off[G] * NT;
  // this CTA's half of B: gate (leader) / up (peer) rows for SwiGLU, else two column blocks
  const void* tmp = (EPI == EPI_SWIGLU && rank == 1) ? static_cast<const void*>(&tmP1)
                                                      : static_cast<const void*>(&tmP0);
  const uint8_t* scales = (EPI == EPI_SWIGLU && rank == 1) ? args.scale1 : args.scale0;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int i = cluster; ok && i < total; i += nclusters) {
        const TileInfo ti = decode_pair_tile(i, tile_off, goff, G, NT, TNO);
        const int a_row = ti.m0 + static_cast<int>(rank) * 128;
        const int b_row = (EPI == EPI_SWIGLU) ? ti.n0 : ti.n0 + static_cast<int>(rank) * TNH;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * LY::A_BYTES);
          uint8_t* sa = smem + s * LY::STAGE_BYTES;
          uint8_t* sp = sa + LY::A_BYTES + LY::B_BYTES;
          tma_load_2d_pair(sa, &tmA, full_leader + static_cast<uint32_t>(s) * 8u, kb * BK, a_row);
          mbar_arrive_expect_tx(&pk[s], TNH * 32);
          tma_load_3d(sp, tmp, &pk[s], kb * 32, b_row, ti.g);
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(DEVERR_TIMEOUT);
        for (int q = 0; q < 2000; ++q) __nanosleep(1000);
      }
      // packed loads signal this CTA's own barriers: wait for every one issued
      for (int q = 0; q < STAGES; ++q)
        if ((issued >> q) & 1u) {
          if (!mbar_wait(&pk[q], (issued_par >> q) & 1u, never_flag, kDrainLimitNs)) flag_error(DEVERR_TIMEOUT);
          if (rank == 0 && !mbar_wait(&full[q], (issued_par >> q) & 1u, never_flag, kDrainLimitNs))
            flag_error(DEVERR_TIMEOUT);
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
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag, lim)) { ok = false; break; }
          if (!mbar_wait(&conv[s], ph, abort_flag, lim)) { ok = false; break; }
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
  } else if (warp < 6) {
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
  } else {
    // ------------------------------------------------------------ converters (both CTAs)
    const int ct = threadIdx.x - 6 * 32;                 // 0..127
    const uint32_t conv_leader = mapa_shared(smem_u32(conv), 0);
    const int c = ct & 7;                                // 16-byte chunk within a row (8 codes)
    const int r0 = ct >> 3;                              // rows r0, r0 + 16, ...
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int i = cluster; ok && i < total; i += nclusters) {
      const TileInfo ti = decode_pair_tile(i, tile_off, goff, G, NT, TNO);
      const int b_row = (EPI == EPI_SWIGLU) ? ti.n0 : ti.n0 + static_cast<int>(rank) * TNH;
      // this thread's scale bytes for one k-block: rows r0 + 16 j, block kb * 2 + c / 4
      const uint8_t* srow = scales + (static_cast<size_t>(ti.g) * args.n_out + b_row) * KS + (c >> 2);
      uint8_t sc_next[(TNH + 15) / 16];
#pragma unroll
      for (int j = 0; j < (TNH + 15) / 16; ++j) {
        const int r = r0 + 16 * j;
        sc_next[j] = (r < TNH && b_row + r < args.n_out) ? srow[static_cast<size_t>(r) * KS] : uint8_t(127);
      }
      for (int kb = 0; kb < KB; ++kb) {
        uint8_t sc[(TNH + 15) / 16];
#pragma unroll
        for (int j = 0; j < (TNH + 15) / 16; ++j) sc[j] = sc_next[j];
        if (!__all_sync(0xffffffffu, mbar_wait(&pk[s], ph, abort_flag, lim))) { ok = false; break; }
        const uint8_t* sp = smem + s * LY::STAGE_BYTES + LY::A_BYTES + LY::B_BYTES;
        uint8_t* sb = smem + s * LY::STAGE_BYTES + LY::A_BYTES;
#pragma unroll
        for (int j = 0; j < (TNH + 15) / 16; ++j) {
          const int r = r0 + 16 * j;
          if (r < TNH) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(sp + r * 32 + c * 4);
            const uint4 v = mxfp4_decode8(w, e8m0_to_bf16x2(sc[j]));
            *reinterpret_cast<uint4*>(sb + r * kRowBytes + ((c ^ (r & 7)) << 4)) = v;
          }
        }
        fence_proxy_async_smem();     // generic-proxy stores -> visible to the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(conv_leader + static_cast<uint32_t>(s) * 8u);
        // next k-block's scales: issued after the fence so that it never waits for them
        if (kb + 1 < KB) {
#pragma unroll
          for (int j = 0; j < (TNH + 15) / 16; ++j) {
            const int r = r0 + 16 * j;
            sc_next[j] = (r < TNH && b_row + r < args.n_out) ? srow[static_cast<size_t>(r) * KS + (kb + 1) * 2]
                                                             : uint8_t(127);
          }
        }
        if (++s == STAGES) { s = 0; ph ^= 1u; }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      flag_error(DEVERR_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace moe
