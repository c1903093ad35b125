// Expert GEMMs for few tokens per expert (decode): weights as the M operand.
//
// With a handful of routed rows per expert the layer is a stream of expert
// weights from HBM.  Here the MMA's M = 128 rows are weight rows and its
// N = NTOK columns are the expert's tokens (C^T = W X^T), so one tcgen05.mma
// per 16-wide K step costs 128 x NTOK x 16 and the tensor cores never hold the
// stream back; shared memory holds a deep ring of 16 KB weight tiles.
//   gate/up: a work unit is 64 output features f0..f0+63 of one expert; its
//            weight tile stacks the 64 gate rows (TMEM lanes 0..63) over the 64
//            up rows (lanes 64..127).  The up warps pass their values through
//            shared memory to the gate warps, which apply the clipped SwiGLU
//            ("Ollama Imagegen GPT OSS", Description) and store h.
//   down:    a work unit is 128 output features d0..d0+127 of one expert;
//            epilogue = bias (+ routing weight and un-permutation, fp32).
// Units are (expert, feature block, token chunk of NTOK), experts without rows
// produce no units; each CTA walks the unit list with a grid stride.  Roles and
// bounded waits as in grouped_gemm.cuh.
#pragma once

#include "grouped_gemm.cuh"

namespace moe {

constexpr int kDecKBS = 1;           // 64-wide K blocks per stage
constexpr int kDecStages = 10;       // one CTA per SM
constexpr int kDecStagesDual = 5;    // two CTAs per SM
constexpr int kDecTmemCols = 64;   // two accumulators of NTOK = 32 columns

// A stage holds KBS consecutive 64-wide K blocks: [KBS weight tiles][KBS token tiles].
template <int NTOK, int KBS = 1>
struct DecLayout {
  static constexpr int W_BYTES = 128 * kRowBytes;     // 16 KB of weight rows per K block
  static constexpr int X_BYTES = NTOK * kRowBytes;
  static constexpr int STAGE_BYTES = KBS * (W_BYTES + X_BYTES);
  static constexpr int UP_BYTES = 64 * NTOK * 4;      // up values handed to the gate warps
  static constexpr int EXTRA = 1024 + 2560;   // alignment slack; barriers, unit and group offsets (2.3 KB)
  static constexpr int smem_bytes(int stages) { return stages * STAGE_BYTES + UP_BYTES + EXTRA; }
  static_assert(NTOK % 16 == 0 && NTOK <= 256, "MMA N");
  static_assert(KBS > 1 || 2 * (STAGE_BYTES * kDecStagesDual + UP_BYTES + EXTRA + 1024) <= 233472,
                "two CTAs per SM (plus 1 KB reserved each) fit the 228 KB of shared memory");
};

struct UnitInfo {
  int g, m0, m_end, f0;
};

// unit u -> (expert, token chunk, feature block); chunks of one feature block are
// consecutive so CTAs running side by side reuse the same weight tile from L2.
__device__ __forceinline__ UnitInfo decode_unit(int u, const int* unit_off, const int* goff, int G, int FB, int FBW,
                                                int NTOK) {
  int lo = 0, hi = G;                       // unit_off[lo] <= u < unit_off[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (unit_off[mid] <= u) lo = mid; else hi = mid;
  }
  const int nch = (unit_off[lo + 1] - unit_off[lo]) / FB;
  const int local = u - unit_off[lo];
  const int fb = local / nch;
  const int ch = local - fb * nch;
  UnitInfo t;
  t.g = lo;
  t.m0 = goff[lo] + ch * NTOK;
  t.m_end = goff[lo + 1];
  t.f0 = fb * FBW;
  return t;
}

// Zeroes n floats (the weighted rows a K-split decode launch adds into).
__global__ void __launch_bounds__(256) zero_f32_kernel(float* __restrict__ p, int64_t n) {
  pdl_enter();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = 0.0f;
}

// EPI_SWIGLU: tmW0 = W_gate, tmW1 = W_up (boxes of 64 rows); EPI_BIAS / EPI_BIAS_WSCATTER: tmW0 = W_down (128 rows).
template <int EPI, int NTOK, int STAGES, int KBS = 1>
__global__ void __launch_bounds__(kGemmThreads, 1)
    decode_gemm_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmW1,
                       const __grid_constant__ CUtensorMap tmX, const GemmArgs args) {
  pdl_enter();
  using T = __nv_bfloat16;
  using LY = DecLayout<NTOK, KBS>;
  constexpr int BK = kRowBytes / 2;
  constexpr int KSTEPS = kRowBytes / 32;
  constexpr bool kGateUp = EPI == EPI_SWIGLU;
  constexpr int FBW = kGateUp ? 64 : 128;   // output features per unit

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* up_stage = reinterpret_cast<float*>(smem + STAGES * LY::STAGE_BYTES);      // [64][NTOK]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * LY::STAGE_BYTES + LY::UP_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* upfull = drain + 1;    // up rows written to up_stage (64 arrivals)
  uint64_t* upempty = upfull + 1;  // gate rows done reading it (64 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(upempty + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* never_flag = abort_flag + 1;
  int* unit_off = never_flag + 2;
  int* goff = unit_off + (kMaxGroups + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = args.num_groups;
  const int FB = (args.n_out + FBW - 1) / FBW;
  const int KB = (args.k_dim + BK - 1) / BK;
  // down over h kept as two bf16 halves: K blocks [0, KB) read hi, [KB, 2 KB) lo (same weights)
  const bool hsplit = !kGateUp && args.h_halves == 2;
  const int KBT = hsplit ? 2 * KB : KB;
  const int KSTEP_STAGES = (KBT + KBS - 1) / KBS;     // stages per unit (blocks past K read zeros)
  const uint64_t lim = args.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&tfull[0], 1);
    mbar_init(&tfull[1], 1);
    mbar_init(&tempty[0], 128);
    mbar_init(&tempty[1], 128);
    mbar_init(drain, 1);
    mbar_init(upfull, 64);
    mbar_init(upempty, 64);
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
    if (lane == 0) unit_off[0] = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int cnt = 0;
      if (g < G) {
        const int rows = goff[g + 1] - goff[g];
        if (rows < 0) bad = 1;
        cnt = rows > 0 ? FB * ((rows + NTOK - 1) / NTOK) : 0;
      }
      int incl = cnt;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += o;
      }
      if (g < G) unit_off[g + 1] = running + incl;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) flag_error(DEVERR_BOUNDS);
    if (lane == 0) {
      tma_prefetch_desc(&tmW0);
      if (kGateUp) tma_prefetch_desc(&tmW1);
      tma_prefetch_desc(&tmX);
    }
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, kDecTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // EPI_BIAS_WSCATTER may split K in S ranges (units S times as many, split
  // fastest); each range adds its weighted partial into the zeroed fp32 rows
  const int S = (EPI == EPI_BIAS_WSCATTER && args.k_splits > 1) ? args.k_splits : 1;
  const int total = unit_off[G] * S;
  const int per_split = (KSTEP_STAGES + S - 1) / S;

  auto unit = [&](int u) { return decode_unit(u / S, unit_off, goff, G, FB, FBW, NTOK); };
  auto stage_range = [&](int u, int& b, int& e) {
    b = (u % S) * per_split;
    e = min(KSTEP_STAGES, b + per_split);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t tx_bytes = LY::STAGE_BYTES;
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
        const UnitInfo ui = unit(u);
        int ks0, ks1;
        stage_range(u, ks0, ks1);
        for (int ks = ks0; ks < ks1; ++ks) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], tx_bytes);
#pragma unroll
          for (int b = 0; b < KBS; ++b) {
            const int kb = ks * KBS + b;
            uint8_t* sw = smem + s * LY::STAGE_BYTES + b * LY::W_BYTES;
            uint8_t* sx = smem + s * LY::STAGE_BYTES + KBS * LY::W_BYTES + b * LY::X_BYTES;
            if (kGateUp) {
              tma_load_3d(sw, &tmW0, &full[s], kb * BK, ui.f0, ui.g);
              tma_load_3d(sw + 64 * kRowBytes, &tmW1, &full[s], kb * BK, ui.f0, ui.g);
              tma_load_2d(sx, &tmX, &full[s], kb * BK, ui.m0);
            } else if (hsplit) {
              // blocks past 2 KB fall outside both the halves and the weights: zeros
              const int half = kb / KB;
              const int kbl = kb - half * KB;
              tma_load_3d(sw, &tmW0, &full[s], kbl * BK, ui.f0, ui.g);
              tma_load_3d(sx, &tmX, &full[s], kbl * BK, half, ui.m0);
            } else {
              tma_load_3d(sw, &tmW0, &full[s], kb * BK, ui.f0, ui.g);
              tma_load_2d(sx, &tmX, &full[s], kb * BK, ui.m0);
            }
          }
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(DEVERR_TIMEOUT);
      }
      for (int q = 0; q < STAGES; ++q)
        if ((issued >> q) & 1u)
          if (!mbar_wait(&full[q], (issued_par >> q) & 1u, never_flag, kDrainLimitNs)) flag_error(DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc(128, NTOK, 1u);
      int s = 0, it = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < total; u += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * NTOK);
        int ks0, ks1;
        stage_range(u, ks0, ks1);
        for (int ks = ks0; ks < ks1; ++ks) {
          if (!mbar_wait(&full[s], ph, abort_flag, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t stage_addr = smem_u32(smem + s * LY::STAGE_BYTES);
#pragma unroll
          for (int b = 0; b < KBS; ++b) {
            const uint32_t w_addr = stage_addr + b * LY::W_BYTES;
            const uint32_t x_addr = stage_addr + KBS * LY::W_BYTES + b * LY::X_BYTES;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk)
              tc_mma<false>(d_tmem, sw128_kmajor_desc(w_addr + kk * 32), sw128_kmajor_desc(x_addr + kk * 32), idesc,
                            (ks != ks0 || b != 0 || kk != 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(DEVERR_TIMEOUT);
      }
      tc_commit(drain);
      if (!mbar_wait(drain, 0, never_flag, kDrainLimitNs)) flag_error(DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;          // TMEM lanes quarter*32 .. +31 = weight rows
    const int wrow = quarter * 32 + lane;
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++it) {
      const UnitInfo ui = unit(u);
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, abort_flag, lim));
      if (!got) { ok = false; break; }
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * NTOK);
      float v[NTOK];
#pragma unroll
      for (int c = 0; c < NTOK; c += 8) {
        float t8[8];
        tmem_ld8(tbase + c, t8);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[c + j] = t8[j];
      }
      tmem_ld_wait();
      tc_fence_before();
      const int ntok = min(NTOK, ui.m_end - ui.m0);
      if constexpr (kGateUp) {
        // rows 64..127 (quarters 2, 3) are up: hand them to the gate rows through shared memory
        const uint32_t xph = it & 1;
        if (quarter >= 2) {
          if (!__all_sync(0xffffffffu, mbar_wait(upempty, xph ^ 1u, abort_flag, lim))) { ok = false; break; }
#pragma unroll
          for (int c = 0; c < NTOK; ++c) up_stage[(wrow - 64) * NTOK + c] = v[c];
          mbar_arrive(upfull);
        } else {
          if (!__all_sync(0xffffffffu, mbar_wait(upfull, xph, abort_flag, lim))) { ok = false; break; }
          const int f = ui.f0 + wrow;
          if (f < args.n_out) {
            const float bg = to_f32<T>(static_cast<const T*>(args.bias0)[static_cast<size_t>(ui.g) * args.n_out + f]);
            const float bu = to_f32<T>(static_cast<const T*>(args.bias1)[static_cast<size_t>(ui.g) * args.n_out + f]);
            T* out = static_cast<T*>(args.out);
            for (int c = 0; c < ntok; ++c) {
              const float gc = fminf(fmaxf(v[c] + bg, args.gate_lo), args.limit);
              const float uc = fminf(fmaxf(up_stage[wrow * NTOK + c] + bu, -args.limit), args.limit);
              const float h = __fdividef(gc * uc, 1.0f + __expf(-args.alpha * gc));
              const T hi = __float2bfloat16_rn(h);
              out[static_cast<size_t>(ui.m0 + c) * args.ldo + f] = hi;
              if (args.h_halves == 2)
                out[static_cast<size_t>(ui.m0 + c) * args.ldo + args.n_out + f] =
                    __float2bfloat16_rn(h - __bfloat162float(hi));
            }
          }
          mbar_arrive(upempty);
        }
      } else {
        const int d = ui.f0 + wrow;
        if (d < args.n_out) {
          const float b = to_f32<T>(static_cast<const T*>(args.bias0)[static_cast<size_t>(ui.g) * args.n_out + d]);
          for (int c = 0; c < ntok; ++c) {
            const int row = ui.m0 + c;
            if constexpr (EPI == EPI_BIAS_WSCATTER) {
              const int slot = args.slot_of_row[row];
              if (slot < 0 || slot >= args.m_total) {
                flag_error(DEVERR_BOUNDS);
                continue;
              }
              float* dst = static_cast<float*>(args.out) + static_cast<size_t>(slot) * args.ldo + d;
              if (S == 1) {
                *dst = args.topk_w[slot] * (v[c] + b);
              } else {
                // the K ranges add into zeroed memory; the first carries the bias.  With
                // two ranges the sum is the same whichever lands first (0 + x + y = x + y)
                atomicAdd(dst, args.topk_w[slot] * (v[c] + (u % S == 0 ? b : 0.0f)));
              }
            } else {
              static_cast<T*>(args.out)[static_cast<size_t>(row) * args.ldo + d] = __float2bfloat16_rn(v[c] + b);
            }
          }
        }
      }
      mbar_arrive(&tempty[acc]);
    }
    if (!ok) {
      *abort_flag = 1;
      flag_error(DEVERR_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kDecTmemCols);
  }
}

}  // namespace moe
