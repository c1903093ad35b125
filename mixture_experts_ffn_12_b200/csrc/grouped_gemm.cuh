// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA, with the MoE layer's epilogues fused in.
//
// Problem: for every group g (an expert) with rows [off[g], off[g+1]) of A,
//     C[r, n] = sum_k A[r, k] * B_g[n, k]          (A and B_g both K-major)
// followed by one of the epilogues
//   EPI_SWIGLU        two B operands (gate, up) share one MMA: the tile's gate
//                     columns sit in TMEM columns [0, TN), its up columns in
//                     [TN, 2 TN).  h = clip(g,0,L) * sigmoid(a clip(g,0,L)) * clip(u,-L,L)
//                     with the per-expert biases added first (GPT-OSS clipped
//                     SwiGLU: "Ollama Imagegen GPT OSS", Description).
//   EPI_BIAS          y_perm[r, n] = C + b[g, n]   (expert down projection, wo + bias).
//   EPI_BIAS_WSCATTER ys[s, n] = w[s] * (C + b[g, n]) (fp32) with s = slot_of_row[r]:
//                     the routing weight and the un-permutation of the combine
//                     ("Ollama glm4_moe_lite.go", MoE.Forward / SwitchMLP.Forward)
//                     done in the down projection's epilogue.
//   EPI_TOPK          router: logits = C + b[n]; the k largest per row (ties -> lower
//                     expert index) and the softmax over them.
//   EPI_PARTIAL       router, K split: the tile's column block index selects one of
//                     k_splits K ranges; the fp32 partial logits go to `partial`.
//
// Kernel organisation (one CTA per SM, 192 threads):
//   warp 0      TMA producer: A tile [128 x 128 B] and B tile(s) [TN x 128 B] per
//               stage, 128-byte swizzle, STAGES-deep ring of mbarriers.
//   warp 1      TMEM owner (512 columns = 2 accumulator buffers of 256) and MMA
//               issuer: 4 x tcgen05.mma per stage (K = 32 bytes each), commits
//               release the stage and, at the end of a tile, hand the
//               accumulator to the epilogue.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator rows this warp may
//               access (TMEM lane quarter = warp % 4), fused math, global stores.
// Tiles (group, 128-row block, TN-column block) are numbered group by group and,
// inside a group, in bands of GM row blocks with the row block fastest, so the
// CTAs that run at the same time share weight tiles and A rows in L2.  Every
// CTA walks the same numbering with a grid stride; no host sync is needed since
// the per-group tile counts are derived on the device from `off`.
//
// Every wait is bounded (mbar_wait); on a timeout the CTA raises an abort flag,
// records DEVERR_TIMEOUT, lets its in-flight TMA loads and MMAs land, frees TMEM
// and exits.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace moe {

enum EpiKind : int { EPI_SWIGLU = 0, EPI_BIAS = 1, EPI_BIAS_WSCATTER = 2, EPI_TOPK = 3, EPI_PARTIAL = 4 };

struct GemmArgs {
  const int32_t* group_off;    // [G+1] row offsets of the groups in A; nullptr = one group of m_total rows
  int num_groups;              // G
  int m_total;                 // rows of A (and of row-indexed outputs)
  int n_out;                   // output columns per B operand
  int k_dim;                   // reduction length (elements)
  int mma_n;                   // MMA N (EPI_TOPK only; otherwise TN * NB)
  const void* bias0;           // [G, n_out] (router: [n_out])
  const void* bias1;           // [G, n_out] (EPI_SWIGLU: up bias)
  float limit, alpha;          // EPI_SWIGLU
  float gate_lo;               // EPI_SWIGLU: lower clip of the gate (0; -inf with limit = inf, alpha = 1: SiLU(g) * u)
  void* out;                   // output rows
  int ldo;                     // elements between output rows
  const int32_t* slot_of_row;  // EPI_BIAS_WSCATTER
  const float* topk_w;         // EPI_BIAS_WSCATTER
  int32_t* topk_ids;           // EPI_TOPK [m_total, topk_k]
  float* topk_wout;            // EPI_TOPK [m_total, topk_k]
  int topk_k;
  unsigned long long wait_limit_ns;
  const uint8_t* scale0;       // MXFP4: E8M0 scales of B0 / B1, [G, n_out, k_dim / 32]
  const uint8_t* scale1;
  int k_splits;                // EPI_PARTIAL: K ranges; column block index = K range
  float* partial;              // EPI_PARTIAL: [k_splits, n_out, m_total] fp32
  const int32_t* gather_slots; // non-null (EPI_SWIGLU, bf16): A row r is row gather_slots[r] / gather_k of
  int gather_k;                //   the tensor map's matrix (x), loaded four rows at a time with TMA
  int gather_rows;             //   gather4; rows of that matrix (clamp for rows past a group's end)
  int h_halves;                // 2: h is kept as two bf16 halves per row, [R, 2, F] (h = hi + lo):
                               // EPI_SWIGLU writes hi = bf16(h) and lo = bf16(h - hi); the down
                               // GEMM reads h through a 3-D tensor map {F, 2, R} and sums over
                               // both halves against the same weights (K = 2F).  0 or 1: one bf16 h.
};

constexpr int kBM = 128;           // rows per tile (MMA M)
constexpr int kRowBytes = 128;     // bytes of K per smem row = swizzle span
constexpr int kGroupBand = 16;     // row blocks per band in the tile order
constexpr int kAccStride = 256;    // TMEM columns between the two accumulator buffers
constexpr int kTmemCols = 512;
constexpr int kGemmThreads = 192;
constexpr int kMaxGroups = 256;
// Limit of the end-of-kernel drain waits (TMA loads and MMAs already in flight
// always complete; this bound only guards against a broken barrier).
constexpr uint64_t kDrainLimitNs = 2000000000ull;

template <int TN, int NB>
struct GemmLayout {
  static constexpr int A_BYTES = kBM * kRowBytes;
  static constexpr int B_BYTES = TN * NB * kRowBytes;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static_assert((TN * NB) % 16 == 0 && TN * NB <= 256, "MMA N must be a multiple of 16, at most 256");
  static_assert(TN % 8 == 0, "second B operand must start on a 1024-byte swizzle atom");
  static constexpr int EXTRA = 1024 /*align*/ + 4096 /*barriers, tables*/;
  static constexpr int smem_bytes(int stages) { return stages * STAGE_BYTES + EXTRA; }
};

struct TileInfo {
  int g, m0, m_end, n0;
};

__device__ __forceinline__ TileInfo decode_tile(int i, const int* tile_off, const int* goff, int G, int NT, int TN) {
  int lo = 0, hi = G;                       // tile_off[lo] * NT <= i < tile_off[hi] * NT
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_off[mid] * NT <= i) lo = mid; else hi = mid;
  }
  const int MT = tile_off[lo + 1] - tile_off[lo];
  const int local = i - tile_off[lo] * NT;
  const int band = local / (kGroupBand * NT);
  const int rem = local - band * kGroupBand * NT;
  const int rows = min(kGroupBand, MT - band * kGroupBand);
  const int nt = rem / rows;
  const int mt = band * kGroupBand + (rem - nt * rows);
  TileInfo t;
  t.g = lo;
  t.m0 = goff[lo] + mt * kBM;
  t.m_end = goff[lo + 1];
  t.n0 = nt * TN;
  return t;
}

// ---------------------------------------------------------------------------
// epilogues: one thread = one accumulator row (TMEM lane)
// ---------------------------------------------------------------------------
template <typename T, int TN>
__device__ __forceinline__ void epi_swiglu(uint32_t tbase, int row, bool rvalid, const TileInfo& ti,
                                           const GemmArgs& a) {
  const T* bg = static_cast<const T*>(a.bias0) + static_cast<size_t>(ti.g) * a.n_out + ti.n0;
  const T* bu = static_cast<const T*>(a.bias1) + static_cast<size_t>(ti.g) * a.n_out + ti.n0;
  T* out = static_cast<T*>(a.out) + static_cast<size_t>(row) * a.ldo + ti.n0;
  const float L = a.limit, alpha = a.alpha;
#pragma unroll 1
  for (int c = 0; c < TN; c += 8) {
    float g[8], u[8];
    tmem_ld8(tbase + c, g);
    tmem_ld8(tbase + TN + c, u);
    tmem_ld_wait();
    if (rvalid && ti.n0 + c < a.n_out) {
      float b0[8], b1[8], h[8];
      load8<T>(bg + c, b0);
      load8<T>(bu + c, b1);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float gc = fminf(fmaxf(g[j] + b0[j], a.gate_lo), L);
        const float uc = fminf(fmaxf(u[j] + b1[j], -L), L);
        h[j] = __fdividef(gc * uc, 1.0f + __expf(-alpha * gc));
      }
      store8<T>(out + c, h);
      if constexpr (!std::is_same<T, float>::value) {
        if (a.h_halves == 2) {
          // the part of h that its bf16 rounding dropped, itself in bf16 (h - hi is exact in fp32)
          float lo[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) lo[j] = h[j] - __bfloat162float(__float2bfloat16_rn(h[j]));
          store8<T>(out + a.n_out + c, lo);
        }
      }
    }
  }
}

template <typename T, int TN, bool kScatter>
__device__ __forceinline__ void epi_bias(uint32_t tbase, int row, bool rvalid, const TileInfo& ti,
                                         const GemmArgs& a) {
  const T* bd = static_cast<const T*>(a.bias0) + static_cast<size_t>(ti.g) * a.n_out + ti.n0;
  float wv = 1.0f;
  size_t orow = static_cast<size_t>(row);
  if (kScatter && rvalid) {
    const int s = a.slot_of_row[row];
    if (s < 0 || s >= a.m_total) {
      flag_error(DEVERR_BOUNDS);
      rvalid = false;
    } else {
      orow = static_cast<size_t>(s);
      wv = a.topk_w[s];
    }
  }
  // the weighted, un-permuted rows are staged in fp32 (one rounding, at the layer output)
  using OutT = typename std::conditional<kScatter, float, T>::type;
  OutT* out = static_cast<OutT*>(a.out) + orow * a.ldo + ti.n0;
#pragma unroll 1
  for (int c = 0; c < TN; c += 8) {
    float v[8];
    tmem_ld8(tbase + c, v);
    tmem_ld_wait();
    if (rvalid && ti.n0 + c < a.n_out) {
      float b[8];
      load8<T>(bd + c, b);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = kScatter ? wv * (v[j] + b[j]) : v[j] + b[j];
      store8<OutT>(out + c, v);
    }
  }
}

template <typename T>
__device__ __forceinline__ void epi_topk(uint32_t tbase, int row, bool rvalid, const GemmArgs& a) {
  // running top-8, sorted descending; strict '>' keeps the lower expert index first on ties
  float tv[8];
  int tix[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) { tv[j] = -INFINITY; tix[j] = -1; }
  const T* br = static_cast<const T*>(a.bias0);
  const int E = a.n_out;
#pragma unroll 1
  for (int c = 0; c < a.mma_n; c += 8) {
    float v[8];
    tmem_ld8(tbase + c, v);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = c + j;
      if (e < E) {
        float cv = v[j] + to_f32<T>(br[e]);
        int ci = e;
        if (cv > tv[7]) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const bool gt = cv > tv[q];
            const float t = tv[q];
            const int tq = tix[q];
            tv[q] = gt ? cv : t;
            tix[q] = gt ? ci : tq;
            cv = gt ? t : cv;
            ci = gt ? tq : ci;
          }
        }
      }
    }
  }
  if (!rvalid) return;
  const int k = a.topk_k;
  float z = 0.0f, ex[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    ex[j] = (j < k) ? expf(tv[j] - tv[0]) : 0.0f;
    z += ex[j];
  }
  const float inv = 1.0f / z;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
      a.topk_ids[static_cast<size_t>(row) * k + j] = tix[j];
      a.topk_wout[static_cast<size_t>(row) * k + j] = ex[j] * inv;
    }
  }
}

// Partial logits go to partial[split][e][row] (expert-major), so for each column
// the 32 rows of a warp store 128 contiguous bytes.
__device__ __forceinline__ void epi_partial(uint32_t tbase, int row, bool rvalid, const TileInfo& ti,
                                            const GemmArgs& a, int split) {
  float* out = a.partial + static_cast<size_t>(split) * a.n_out * a.m_total + row;
#pragma unroll 1
  for (int c = 0; c < a.mma_n; c += 8) {
    float v[8];
    tmem_ld8(tbase + c, v);
    tmem_ld_wait();
    if (rvalid) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (c + j < a.n_out) out[static_cast<size_t>(c + j) * a.m_total] = v[j];
    }
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <typename T, int TN, int NB, int EPI, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, const GemmArgs args) {
  pdl_enter();
  constexpr bool kTF32 = std::is_same<T, float>::value;
  using LY = GemmLayout<TN, NB>;
  constexpr int BK = kRowBytes / static_cast<int>(sizeof(T));   // K elements per stage
  constexpr int KSTEPS = kRowBytes / 32;                         // MMAs per stage (32 bytes of K each)

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
  int* tile_off = never_flag + 2;              // [G+1]
  int* goff = tile_off + (kMaxGroups + 2);     // [G+1]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool single = args.group_off == nullptr;
  const int G = single ? 1 : args.num_groups;
  const int NT = (EPI == EPI_PARTIAL) ? args.k_splits : (args.n_out + TN - 1) / TN;
  const int KB = (args.k_dim + BK - 1) / BK;
  const int KBS = (EPI == EPI_PARTIAL) ? (KB + args.k_splits - 1) / args.k_splits : KB;   // k-blocks per range
  // down projection over h kept as two bf16 halves: K blocks [0, KB) read hi, [KB, 2 KB) lo,
  // both against the weights' K blocks [0, KB)
  const bool hsplit = (EPI == EPI_BIAS || EPI == EPI_BIAS_WSCATTER) && args.h_halves == 2;
  const int KBT = hsplit ? 2 * KB : KB;
  const uint64_t lim = args.wait_limit_ns;
  // k-block range of a tile: all of K, or (EPI_PARTIAL) the range of its column block index
  auto kb_range = [&](const TileInfo& ti, int& b, int& e) {
    if (EPI == EPI_PARTIAL) {
      const int split = ti.n0 / TN;
      b = split * KBS;
      e = min(KB, b + KBS);
    } else {
      b = 0;
      e = KBT;
    }
  };

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
    *abort_flag = 0;
    *never_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    // group offsets (clamped into [0, m_total]) and the prefix of 128-row blocks per group
    int bad = 0;
    for (int g = lane; g <= G; g += 32) {
      int v = single ? (g == 0 ? 0 : args.m_total) : args.group_off[g];
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
        cnt = rows > 0 ? (rows + kBM - 1) / kBM : 0;
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
    if (__any_sync(0xffffffffu, bad) && lane == 0) flag_error(DEVERR_BOUNDS);
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB0);
      if (NB == 2) tma_prefetch_desc(&tmB1);
    }
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_off[G] * NT;

  if (warp == 0 && EPI == EPI_SWIGLU && !kTF32 && args.gather_slots != nullptr) {
    // ------------------------------------------------------------ TMA producer, A rows gathered
    // Lane j loads A rows 4j .. 4j + 3 of every stage with one gather4 from x (the row of
    // each permuted row's token); lane 0 waits for the slot, arms the barrier and loads B.
    const uint32_t tx_bytes = LY::A_BYTES + static_cast<uint32_t>(TN * NB) * kRowBytes;
    int s = 0;
    uint32_t ph = 0, issued = 0, issued_par = 0;
    bool ok = true;
    for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
      const TileInfo ti = decode_tile(i, tile_off, goff, G, NT, TN);
      int src[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int row = ti.m0 + 4 * lane + q;
        int t = 0;
        if (row < ti.m_end) {
          t = __ldg(args.gather_slots + row) / args.gather_k;
          if (t < 0 || t >= args.gather_rows) { flag_error(DEVERR_BOUNDS); t = 0; }
        }
        src[q] = t;   // rows past the group read row 0; their outputs are never written
      }
      for (int kb = 0; kb < KB; ++kb) {
        bool got = true;
        if (lane == 0) {
          got = mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim);
          if (got) mbar_arrive_expect_tx(&full[s], tx_bytes);
        }
        if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) { ok = false; break; }
        uint8_t* sa = smem + s * LY::STAGE_BYTES;
        tma_gather4_2d(sa + 4 * lane * kRowBytes, &tmA, &full[s], kb * BK, src[0], src[1], src[2], src[3]);
        if (lane == 0) {
          uint8_t* sb = sa + LY::A_BYTES;
          tma_load_3d(sb, &tmB0, &full[s], kb * BK, ti.n0, ti.g);
          if (NB == 2) tma_load_3d(sb + TN * kRowBytes, &tmB1, &full[s], kb * BK, ti.n0, ti.g);
        }
        issued |= 1u << s;
        issued_par = (issued_par & ~(1u << s)) | (ph << s);
        if (++s == STAGES) { s = 0; ph ^= 1u; }
      }
    }
    if (lane == 0) {
      if (!ok) {
        *abort_flag = 1;
        flag_error(DEVERR_TIMEOUT);
      }
      for (int q = 0; q < STAGES; ++q)
        if ((issued >> q) & 1u)
          if (!mbar_wait(&full[q], (issued_par >> q) & 1u, never_flag, kDrainLimitNs)) flag_error(DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int mma_n = (EPI == EPI_TOPK || EPI == EPI_PARTIAL) ? args.mma_n : TN * NB;
      const uint32_t tx_bytes = LY::A_BYTES + static_cast<uint32_t>(mma_n) * kRowBytes;
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
        const TileInfo ti = decode_tile(i, tile_off, goff, G, NT, TN);
        int kb0, kb1;
        kb_range(ti, kb0, kb1);
        const int b_row = (EPI == EPI_PARTIAL) ? 0 : ti.n0;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], tx_bytes);
          uint8_t* sa = smem + s * LY::STAGE_BYTES;
          uint8_t* sb = sa + LY::A_BYTES;
          const int half = hsplit ? kb / KB : 0;
          const int kbl = kb - half * KB;
          // the weight boxes first: they come more often from HBM or the other die than the
          // activation rows, which neighbouring tiles reuse from L2
          tma_load_3d(sb, &tmB0, &full[s], kbl * BK, b_row, ti.g);
          if (NB == 2) tma_load_3d(sb + TN * kRowBytes, &tmB1, &full[s], kb * BK, ti.n0, ti.g);
          if (hsplit) tma_load_3d(sa, &tmA, &full[s], kbl * BK, half, ti.m0);
          else tma_load_2d(sa, &tmA, &full[s], kb * BK, ti.m0);
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(DEVERR_TIMEOUT);
      }
      // every issued load must have landed before this CTA may exit
      for (int q = 0; q < STAGES; ++q)
        if ((issued >> q) & 1u)
          if (!mbar_wait(&full[q], (issued_par >> q) & 1u, never_flag, kDrainLimitNs)) flag_error(DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const int mma_n = (EPI == EPI_TOPK || EPI == EPI_PARTIAL) ? args.mma_n : TN * NB;
      const uint32_t idesc = make_idesc(kBM, mma_n, kTF32 ? 2u : 1u);
      int s = 0, it = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = blockIdx.x; ok && i < total; i += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        int kb0, kb1;
        kb_range(decode_tile(i, tile_off, goff, G, NT, TN), kb0, kb1);
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccStride);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * LY::STAGE_BYTES);
          const uint32_t b_addr = a_addr + LY::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk)
            tc_mma<kTF32>(d_tmem, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), idesc,
                          (kb != kb0 || kk != 0) ? 1u : 0u);
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
      tc_commit(drain);   // arrives once every MMA issued above has retired
      if (!mbar_wait(drain, 0, never_flag, kDrainLimitNs)) flag_error(DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int r_in_tile = quarter * 32 + lane;
    int it = 0;
    bool ok = true;
    for (int i = blockIdx.x; i < total; i += gridDim.x, ++it) {
      const TileInfo ti = decode_tile(i, tile_off, goff, G, NT, TN);
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      // warp-uniform decision: the tcgen05.ld below is a whole-warp instruction
      const bool got = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, abort_flag, lim));
      if (!got) { ok = false; break; }
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kAccStride);
      const int row = ti.m0 + r_in_tile;
      const bool rvalid = row < ti.m_end;
      if constexpr (EPI == EPI_SWIGLU) epi_swiglu<T, TN>(tbase, row, rvalid, ti, args);
      else if constexpr (EPI == EPI_BIAS) epi_bias<T, TN, false>(tbase, row, rvalid, ti, args);
      else if constexpr (EPI == EPI_BIAS_WSCATTER) epi_bias<T, TN, true>(tbase, row, rvalid, ti, args);
      else if constexpr (EPI == EPI_PARTIAL) epi_partial(tbase, row, rvalid, ti, args, ti.n0 / TN);
      else epi_topk<T>(tbase, row, rvalid, args);
      tc_fence_before();
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
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace moe
