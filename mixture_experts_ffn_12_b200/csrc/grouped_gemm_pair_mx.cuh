// CTA-pair grouped GEMM with MXFP4 expert weights dequantised inside the mainloop.
//
// Same tiles, MMA and epilogues as grouped_gemm_pair.cuh; the weight half each
// CTA feeds the MMA is decoded from MXFP4 in shared memory by converter warps.
// MX encoding (OCP MX): E2M1 codes (bit 3 sign, bits 2..1 exponent with bias 1,
// bit 0 mantissa; element 2i in the low nibble of byte i) times the E8M0 scale
// 2^(s-127) of their 32-element block along K.  Every decoded value is a bf16
// number, so the MMA sees exactly the dequantised weights.
//
// The packed weights travel on a ring of their own, decoupled from the MMA
// stages: a packed slot holds one 64-wide K step of this CTA's 120 weight rows
// (32 bytes each) and their 240 scale bytes, both loaded by TMA, and the ring is
// 16 slots deep, so packed data is resident long before the MMA needs it.  The
// converters wait for a packed slot and for the MMA stage's weight tile to be
// free, decode into it, fence the generic-proxy stores for the tensor core and
// arrive on the leader's `conv` barrier (one arrival per converter warp of the pair); the
// leader's MMA waits for `full` (both CTAs' activation rows, TMA) and `conv`.
// Scales are read from a copy relaid as [E][K/64][N][2] (moe_abi's workspace,
// written by mx_scale_relayout_kernel each call), because rows of K/32 bytes are
// not a multiple of 16 bytes and cannot be described to TMA as they are stored.
//
// Roles (608 threads per CTA):
//   warp 0      activation producer (TMA, both CTAs, bytes counted on the leader)
//   warp 1      TMEM; the leader's lane 0 issues the pair MMAs
//   warps 2-5   epilogue (this CTA's 128 accumulator rows)
//   warp 6      packed-weight producer (TMA into the packed ring, this CTA)
//   warps 7-18  converters, in three groups of four warps: group g decodes the K steps
//               j with j % 3 == g (every row of the step), so three steps are decoded
//               at once and a step's decode latency is hidden behind the other two
#pragma once

#include "grouped_gemm_pair.cuh"

namespace moe {

constexpr int kMxConvWarp0 = 7;     // first converter warp
constexpr int kMxConvGroups = 3;    // K steps decoded concurrently
constexpr int kMxGroupWarps = 4;    // warps per group (one per SM sub-partition)
constexpr int kMxThreads = (kMxConvWarp0 + kMxConvGroups * kMxGroupWarps) * 32;
constexpr int kMxPackSlots = 16;    // depth of the packed-weight ring

template <int TNH>
struct PairMxLayout {
  static constexpr int A_BYTES = 128 * kRowBytes;            // bf16 activations
  static constexpr int B_BYTES = TNH * kRowBytes;            // dequantised bf16 weights
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int P_BYTES = TNH * 32;                   // packed E2M1 rows of one K step
  static constexpr int S_BYTES = TNH * 2;                    // their two scale bytes per row
  static constexpr int SLOT_BYTES = (P_BYTES + S_BYTES + 255) / 256 * 256;
  static constexpr int EXTRA = 1024 + 4096;
  static constexpr int smem_bytes(int stages) { return stages * STAGE_BYTES + kMxPackSlots * SLOT_BYTES + EXTRA; }
  static_assert(STAGE_BYTES % 1024 == 0, "stages stay 1024-byte aligned for the 128-byte swizzle");
  static_assert(P_BYTES % 16 == 0 && S_BYTES % 16 == 0, "TMA destinations are 16-byte aligned");
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

// Scales [E][N][K/32] -> [E][ceil(K/64)][N][2]: the two scale bytes of K step kb for
// row n sit at ((g * KB + kb) * N + n) * 2; a missing second block (K % 64 == 32)
// gets 127 (its codes are zero).  gridDim.y selects one of up to three matrices.
struct MxScaleJob {
  const uint8_t* src[3];
  uint8_t* dst[3];
  int rows[3];     // N of each matrix
  int kdim[3];     // K of each matrix
  int groups;
};

__global__ void __launch_bounds__(256) mx_scale_relayout_kernel(MxScaleJob job) {
  pdl_enter();
  const int m = blockIdx.y;
  const int N = m == 0 ? job.rows[0] : m == 1 ? job.rows[1] : job.rows[2];
  const int K = m == 0 ? job.kdim[0] : m == 1 ? job.kdim[1] : job.kdim[2];
  const uint8_t* src = m == 0 ? job.src[0] : m == 1 ? job.src[1] : job.src[2];
  uint16_t* dst = reinterpret_cast<uint16_t*>(m == 0 ? job.dst[0] : m == 1 ? job.dst[1] : job.dst[2]);
  const int KS = K / 32, KB = (K + 63) / 64;
  // 32-bit index arithmetic: the config check keeps groups * KB * N (and twice it) below 2^31
  const int total = job.groups * KB * N;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int gk = i / N;
    const int n = i - gk * N;
    const int g = gk / KB;
    const int kb = gk - g * KB;
    const uint8_t* row = src + (static_cast<size_t>(g) * N + n) * KS;
    const uint32_t lo = row[2 * kb];
    const uint32_t hi = 2 * kb + 1 < KS ? row[2 * kb + 1] : 127u;
    dst[i] = static_cast<uint16_t>(lo | (hi << 8));
  }
}

// tmA: activations [R, K] (128-row boxes).  tmP0 / tmP1: packed weights [E][N][K/2]
// (TNH-row boxes of 32 bytes); tmS0 / tmS1: relaid scales [E][KB][2N] (boxes of
// 2*TNH bytes).  For SwiGLU index 0 is the gate (leader) and 1 the up projection
// (peer); otherwise both are the down weights and the CTAs take two column blocks.
template <int TNH, int EPI, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMxThreads, 1)
    grouped_gemm_pair_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmP0,
                                const __grid_constant__ CUtensorMap tmP1, const __grid_constant__ CUtensorMap tmS0,
                                const __grid_constant__ CUtensorMap tmS1, const GemmArgs args) {
  pdl_enter();
  using T = __nv_bfloat16;
  using LY = PairMxLayout<TNH>;
  constexpr int BK = kRowBytes / 2;        // 64 K elements per step
  constexpr int KSTEPS = kRowBytes / 32;
  constexpr int TNO = (EPI == EPI_SWIGLU) ? TNH : 2 * TNH;
  constexpr int PS = kMxPackSlots;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* pring = smem + STAGES * LY::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(pring + PS * LY::SLOT_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* conv = empty + STAGES;         // both CTAs' weight halves decoded (leader, one group of each CTA)
  uint64_t* pfull = conv + STAGES;         // packed slot landed (local, TMA)
  uint64_t* pempty = pfull + PS;           // packed slot read by the local group that decoded it
  uint64_t* tfull = pempty + PS;
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
  const uint64_t lim = args.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&conv[s], 2 * kMxGroupWarps);
    }
    for (int p = 0; p < PS; ++p) {
      mbar_init(&pfull[p], 1);
      mbar_init(&pempty[p], kMxGroupWarps);
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
      tma_prefetch_desc(&tmS0);
      tma_prefetch_desc(&tmS1);
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
  // this CTA's weight half: gate (leader) / up (peer) rows for SwiGLU, else two column blocks
  const bool second = EPI == EPI_SWIGLU && rank == 1;
  const void* tmp = second ? static_cast<const void*>(&tmP1) : static_cast<const void*>(&tmP0);
  const void* tms = second ? static_cast<const void*>(&tmS1) : static_cast<const void*>(&tmS0);

  if (warp == 0) {
    // ------------------------------------------------------------ activation producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int i = cluster; ok && i < total; i += nclusters) {
        const TileInfo ti = decode_pair_tile(i, tile_off, goff, G, NT, TNO);
        const int a_row = ti.m0 + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * LY::A_BYTES);
          tma_load_2d_pair(smem + s * LY::STAGE_BYTES, &tmA, full_leader + static_cast<uint32_t>(s) * 8u, kb * BK,
                           a_row);
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
  } else if (warp == 6) {
    // ------------------------------------------------------------ packed-weight producer (both CTAs)
    if (lane == 0) {
      int p = 0;
      uint32_t pph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int i = cluster; ok && i < total; i += nclusters) {
        const TileInfo ti = decode_pair_tile(i, tile_off, goff, G, NT, TNO);
        const int b_row = (EPI == EPI_SWIGLU) ? ti.n0 : ti.n0 + static_cast<int>(rank) * TNH;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&pempty[p], pph ^ 1u, abort_flag, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&pfull[p], LY::P_BYTES + LY::S_BYTES);
          uint8_t* slot = pring + p * LY::SLOT_BYTES;
          tma_load_3d(slot, tmp, &pfull[p], kb * 32, b_row, ti.g);
          tma_load_3d(slot + LY::P_BYTES, tms, &pfull[p], 2 * b_row, kb, ti.g);
          issued |= 1u << p;
          issued_par = (issued_par & ~(1u << p)) | (pph << p);
          if (++p == PS) { p = 0; pph ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(DEVERR_TIMEOUT);
      }
      // these loads signal this CTA's own barriers: wait for every one issued
      for (int q = 0; q < PS; ++q)
        if ((issued >> q) & 1u)
          if (!mbar_wait(&pfull[q], (issued_par >> q) & 1u, never_flag, kDrainLimitNs)) flag_error(DEVERR_TIMEOUT);
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
          if (!mbar_wait_cluster(&conv[s], ph, abort_flag, lim)) { ok = false; break; }
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
    const int cw = warp - kMxConvWarp0;                  // 0 .. groups * group warps - 1
    const int grp = cw / kMxGroupWarps;
    const int ct = (cw % kMxGroupWarps) * 32 + lane;     // 0..127 within the group
    const uint32_t conv_leader = mapa_shared(smem_u32(conv), 0);
    // this cluster's K steps, numbered across its tiles like the producers walk them
    const int my_tiles = cluster < total ? (total - cluster + nclusters - 1) / nclusters : 0;
    const int steps = my_tiles * KB;
    bool ok = true;
    for (int j = grp; ok && j < steps; j += kMxConvGroups) {
      const int s = j % STAGES, p = j % PS;
      const uint32_t ph = static_cast<uint32_t>(j / STAGES) & 1u, pph = static_cast<uint32_t>(j / PS) & 1u;
      // packed slot landed, and the MMA is done with this stage's weight tile
      if (!__all_sync(0xffffffffu, mbar_wait(&pfull[p], pph, abort_flag, lim))) { ok = false; break; }
      if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim))) { ok = false; break; }
      const uint8_t* sp = pring + p * LY::SLOT_BYTES;
      const uint8_t* ss = sp + LY::P_BYTES;
      uint8_t* sb = smem + s * LY::STAGE_BYTES + LY::A_BYTES;
      // a task is half a packed row: 16 bytes = 32 codes = one scale block, i.e.
      // four 16-byte chunks (8 bf16 each) of the swizzled bf16 row
#pragma unroll
      for (int q = 0; q < (2 * TNH + 127) / 128; ++q) {
        const int tk = ct + 128 * q;
        if (tk < 2 * TNH) {
          const int r = tk >> 1, h = tk & 1, x = r & 7;
          const uint4 w4 = *reinterpret_cast<const uint4*>(sp + r * 32 + h * 16);
          const __nv_bfloat162 sc = e8m0_to_bf16x2(ss[r * 2 + h]);
          uint8_t* row = sb + r * kRowBytes;
          *reinterpret_cast<uint4*>(row + (((4 * h + 0) ^ x) << 4)) = mxfp4_decode8(w4.x, sc);
          *reinterpret_cast<uint4*>(row + (((4 * h + 1) ^ x) << 4)) = mxfp4_decode8(w4.y, sc);
          *reinterpret_cast<uint4*>(row + (((4 * h + 2) ^ x) << 4)) = mxfp4_decode8(w4.z, sc);
          *reinterpret_cast<uint4*>(row + (((4 * h + 3) ^ x) << 4)) = mxfp4_decode8(w4.w, sc);
        }
      }
      fence_proxy_async_smem();     // generic-proxy stores -> visible to the tensor core
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_cluster(conv_leader + static_cast<uint32_t>(s) * 8u);
        mbar_arrive(&pempty[p]);
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
