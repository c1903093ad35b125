// Grouped expert GEMMs on CTA pairs with the weights as the MMA's M operand.
//
// C^T = W X^T per expert: tcgen05.mma.cta_group::2 with M = 256 weight rows
// (128 in each CTA of the pair) and N = the expert's tokens, up to 256 per tile
// (each CTA stages half of them).  Putting the tokens in N means a ragged expert
// segment only rounds up to 16 columns, where 128- or 256-row token tiles pad a
// whole tile; the weight side pads only at the end of F or D.  Per 64-wide K step
// each CTA's shared memory takes 16 KB of weights and up to 16 KB of tokens by TMA
// and the tensor core reads the same back, about what the CTA-pair kernel with
// weights in N moves.
//
//   gate/up  a unit covers 128 output features f0..f0+127 of one expert: the
//            leader holds f0..f0+63, its peer f0+64..f0+127.  A CTA's 128 weight
//            rows are four groups of [16 gate rows | 16 up rows] for the same 16
//            features, so TMEM lane quarter q holds gate (lanes 0..15) and up
//            (lanes 16..31) of 16 features and the clipped SwiGLU ("Ollama Imagegen
//            GPT OSS", Description) pairs them with one shuffle; h is stored
//            [token, f] in bf16.
//   down     a unit covers 256 output features d0..d0+255 (128 per CTA);
//            epilogue = bias, then either bf16 rows or (routing weight,
//            un-permutation) fp32 rows in slot order.
//
// Roles (192 threads per CTA, both CTAs), bounded waits and the closing cluster
// barrier are those of grouped_gemm_pair.cuh: warp 0 loads this CTA's weight rows
// and token half into its own stage, counting the bytes on the leader's `full`
// barrier; the leader's warp 1 issues the MMAs and multicasts each commit; warps
// 2-5 drain this CTA's 128 accumulator lanes.
// Units: (expert, weight block, token tile), weight-block major inside an
// expert, so clusters running side by side share a weight block through L2.
#pragma once

#include "grouped_gemm_pair.cuh"

namespace moe {

constexpr int kWmTok = 256;          // tokens per tile (MMA N, at most)
constexpr int kWmStages = 6;

struct WmLayout {
  static constexpr int W_BYTES = 128 * kRowBytes;    // this CTA's 128 weight rows
  static constexpr int X_BYTES = 128 * kRowBytes;    // this CTA's token half (<= 128 rows)
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
  static constexpr int EXTRA = 1024 + 4096;
  static constexpr int smem_bytes(int stages) { return stages * STAGE_BYTES + EXTRA; }
};

struct WmUnit {
  int g;       // expert
  int m0;      // first token row of the tile (in the permuted order)
  int m_end;   // end of the expert's rows
  int n;       // MMA N: tokens of the tile rounded up to 16, at least 32
  int w0;      // first output feature of the pair
};

// unit u -> (expert, weight block, token tile); unit_off[g] = units before expert g.
__device__ __forceinline__ WmUnit decode_wm_unit(int u, const int* unit_off, const int* goff, int G, int WB,
                                                 int WPAIR) {
  int lo = 0, hi = G;                        // unit_off[lo] <= u < unit_off[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (unit_off[mid] <= u) lo = mid; else hi = mid;
  }
  const int nt = (unit_off[lo + 1] - unit_off[lo]) / WB;
  const int local = u - unit_off[lo];
  const int wb = local / nt;
  const int tt = local - wb * nt;
  WmUnit w;
  w.g = lo;
  w.m0 = goff[lo] + tt * kWmTok;
  w.m_end = goff[lo + 1];
  w.n = max(32, (min(kWmTok, w.m_end - w.m0) + 15) & ~15);
  w.w0 = wb * WPAIR;
  return w;
}

// Epilogue of one warp: TMEM lane quarter q (this CTA's weight rows 32q..32q+31).
template <int EPI>
__device__ __forceinline__ void wm_epilogue(uint32_t tbase, const WmUnit& un, int q, int lane, uint32_t rank,
                                            const GemmArgs& a) {
  using T = __nv_bfloat16;
  const int valid = un.m_end - un.m0;        // columns < valid are real tokens
  if constexpr (EPI == EPI_SWIGLU) {
    const bool is_up = lane >= 16;
    const int f = un.w0 + 64 * static_cast<int>(rank) + 16 * q + (lane & 15);
    const bool fvalid = f < a.n_out;
    float bg = 0.0f, bu = 0.0f;
    if (fvalid) {
      bg = to_f32<T>(static_cast<const T*>(a.bias0)[static_cast<size_t>(un.g) * a.n_out + f]);
      bu = to_f32<T>(static_cast<const T*>(a.bias1)[static_cast<size_t>(un.g) * a.n_out + f]);
    }
    const float L = a.limit, alpha = a.alpha;
    T* out = static_cast<T*>(a.out) + f;
#pragma unroll 1
    for (int c = 0; c < un.n; c += 8) {
      float v[8];
      tmem_ld8(tbase + c, v);
      tmem_ld_wait();
      // gate lanes finish tokens c..c+3, up lanes tokens c+4..c+7
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float r = __shfl_xor_sync(0xffffffffu, is_up ? v[i] : v[4 + i], 16);
        const float gv = is_up ? r : v[i];
        const float uv = is_up ? v[4 + i] : r;
        const int col = c + (is_up ? 4 + i : i);
        if (fvalid && col < valid) {
          const float gc = fminf(fmaxf(gv + bg, a.gate_lo), L);
          const float uc = fminf(fmaxf(uv + bu, -L), L);
          const float h = __fdividef(gc * uc, 1.0f + __expf(-alpha * gc));
          out[static_cast<size_t>(un.m0 + col) * a.ldo] = __float2bfloat16_rn(h);
        }
      }
    }
  } else {
    const int d = un.w0 + 128 * static_cast<int>(rank) + 32 * q + lane;
    const bool dvalid = d < a.n_out;
    const float b =
        dvalid ? to_f32<T>(static_cast<const T*>(a.bias0)[static_cast<size_t>(un.g) * a.n_out + d]) : 0.0f;
    // slot and routing weight of tokens 32t + lane, handed out by shuffles below
    int my_slot[kWmTok / 32];
    float my_w[kWmTok / 32];
#pragma unroll
    for (int t = 0; t < kWmTok / 32; ++t) {
      my_slot[t] = -1;
      my_w[t] = 0.0f;
      if constexpr (EPI == EPI_BIAS_WSCATTER) {
        const int col = 32 * t + lane;
        if (col < valid) {
          const int slot = a.slot_of_row[un.m0 + col];
          if (slot < 0 || slot >= a.m_total) {
            flag_error(DEVERR_BOUNDS);
          } else {
            my_slot[t] = slot;
            my_w[t] = a.topk_w[slot];
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kWmTok / 32; ++t) {
      if (32 * t >= un.n) break;
#pragma unroll 1
      for (int c8 = 0; c8 < 32; c8 += 8) {
        const int c = 32 * t + c8;
        if (c >= un.n) break;
        float v[8];
        tmem_ld8(tbase + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if constexpr (EPI == EPI_BIAS_WSCATTER) {
            // the weighted, un-permuted rows are staged in fp32 (one rounding, at the layer output)
            const int slot = __shfl_sync(0xffffffffu, my_slot[t], c8 + j);
            const float w = __shfl_sync(0xffffffffu, my_w[t], c8 + j);
            if (slot >= 0 && dvalid) static_cast<float*>(a.out)[static_cast<size_t>(slot) * a.ldo + d] = w * (v[j] + b);
          } else {
            const int col = c + j;
            if (col < valid && dvalid)
              static_cast<T*>(a.out)[static_cast<size_t>(un.m0 + col) * a.ldo + d] = __float2bfloat16_rn(v[j] + b);
          }
        }
      }
    }
  }
}

// EPI_SWIGLU: tmW0 = W_gate, tmW1 = W_up (16-row boxes);
// EPI_BIAS / EPI_BIAS_WSCATTER: tmW0 = tmW1 = W_down (128-row boxes).
// tmX: tokens with 128-row boxes; tmX16: the same tokens with 16-row boxes (partial tiles).
template <int EPI, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_wm_pair_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmW1,
                                const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmX16,
                                const GemmArgs args) {
  pdl_enter();
  using LY = WmLayout;
  constexpr int BK = kRowBytes / 2;
  constexpr int KSTEPS = kRowBytes / 32;
  constexpr bool kGateUp = EPI == EPI_SWIGLU;
  constexpr int WPAIR = kGateUp ? 128 : 256;    // output features per unit

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
  int* unit_off = never_flag + 2;
  int* goff = unit_off + (kMaxGroups + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();          // 0 = leader (issues the MMAs)
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int G = args.num_groups;
  const int WB = (args.n_out + WPAIR - 1) / WPAIR;
  const int KB = (args.k_dim + BK - 1) / BK;
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
    if (lane == 0) unit_off[0] = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int cnt = 0;
      if (g < G) {
        const int rows = goff[g + 1] - goff[g];
        if (rows < 0) bad = 1;
        cnt = rows > 0 ? WB * ((rows + kWmTok - 1) / kWmTok) : 0;
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
    if (__any_sync(0xffffffffu, bad) && lane == 0 && rank == 0) flag_error(DEVERR_BOUNDS);
    if (lane == 0) {
      tma_prefetch_desc(&tmW0);
      tma_prefetch_desc(&tmW1);
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmX16);
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
  const int total = unit_off[G];

  auto unit = [&](int u) { return decode_wm_unit(u, unit_off, goff, G, WB, WPAIR); };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int u = cluster; ok && u < total; u += nclusters) {
        const WmUnit un = unit(u);
        const int half = un.n >> 1;                           // token rows per CTA (multiple of 8)
        const int x_row = un.m0 + static_cast<int>(rank) * half;
        const int nx16 = half == 128 ? 0 : (half + 15) >> 4;  // 16-row boxes for a partial tile
        const uint32_t x_bytes = half == 128 ? 128u * kRowBytes : static_cast<uint32_t>(nx16) * 16u * kRowBytes;
        const int wrow = un.w0 + static_cast<int>(rank) * (WPAIR / 2);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * (LY::W_BYTES + x_bytes));
          uint8_t* sw = smem + s * LY::STAGE_BYTES;
          uint8_t* sx = sw + LY::W_BYTES;
          const uint32_t fb = full_leader + static_cast<uint32_t>(s) * 8u;
          if (kGateUp) {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              tma_load_3d_pair(sw + (32 * b) * kRowBytes, &tmW0, fb, kb * BK, wrow + 16 * b, un.g);
              tma_load_3d_pair(sw + (32 * b + 16) * kRowBytes, &tmW1, fb, kb * BK, wrow + 16 * b, un.g);
            }
          } else {
            tma_load_3d_pair(sw, &tmW0, fb, kb * BK, wrow, un.g);
          }
          if (nx16 == 0) {
            tma_load_2d_pair(sx, &tmX, fb, kb * BK, x_row);
          } else {
            for (int j = 0; j < nx16; ++j) tma_load_2d_pair(sx + j * 16 * kRowBytes, &tmX16, fb, kb * BK, x_row + 16 * j);
          }
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
      int s = 0, it = 0;
      uint32_t ph = 0;
      bool ok = true;
      bool issued_any = false;
      for (int u = cluster; ok && u < total; u += nclusters, ++it) {
        const WmUnit un = unit(u);
        const uint32_t idesc = make_idesc(kPairBM, un.n, 1u);
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait_cluster(&tempty[acc], aph ^ 1u, abort_flag, lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccStride);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t w_addr = smem_u32(smem + s * LY::STAGE_BYTES);
          const uint32_t x_addr = w_addr + LY::W_BYTES;
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk)
            tc_mma_pair(d_tmem, sw128_kmajor_desc(w_addr + kk * 32), sw128_kmajor_desc(x_addr + kk * 32), idesc,
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
    const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);
    int it = 0;
    bool ok = true;
    for (int u = cluster; u < total; u += nclusters, ++it) {
      const WmUnit un = unit(u);
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, abort_flag, lim));
      if (!got) { ok = false; break; }
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kAccStride);
      wm_epilogue<EPI>(tbase, un, quarter, lane, rank, args);
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
