// Expert GEMMs of the MXFP4 layer on the block-scaled tensor cores, with the
// activations in MXFP8 (the layer's block-scaled numerics variant).
//
// The expert weights stay in the caller's MXFP4 form (E2M1 codes, one E8M0 scale
// per 32 elements along K: "GPT-OSS 20B GGUF with MoE CPU Offloading", Model
// Specifications; group size 32 for the 4-bit and MXFP8 formats: "Ollama
// glm4_moe_lite.go", quantizationParams).  The activations -- x_perm for gate/up,
// h for down -- are quantized to MXFP8 (E4M3 elements, one E8M0 scale per 32
// elements along K; the scale 2^X is the smallest power of two with the block's
// largest magnitude <= 448 * 2^X, so nothing saturates; elements round to nearest,
// ties to even).  One tcgen05.mma.kind::mxf8f6f4.block_scale then multiplies
// E4M3 by E2M1 with both operands' block scales applied by the tensor core, so
// no weight is ever decoded in software.
//
// Operands in shared memory (128-byte swizzle, K-major, 128 K elements a stage):
//   A  E4M3 rows by TMA (uint8 tensor map), 128 rows x 128 B.
//   B  the f8f6f4 MMA reads 4-bit operands with each 16 codes (8 B) in 16 B of
//      shared memory, the upper 8 B unused.  Whole 128-code K blocks come by TMA
//      with its 4-bit unpacking type (16U4_ALIGN16B), which writes exactly that
//      layout into the 128-byte-swizzled tile; the unpacking type wants the rows
//      described in whole 128-code blocks, so a last partial block (K = 2880 =
//      22.5 x 128) and weights the type cannot describe (K / 2 not a multiple of
//      32 bytes, or a base not 32-byte aligned) arrive packed (64 B per 128 codes)
//      by a plain byte TMA in a staging area, and four converter warps widen every
//      8 B to 16 B (zeros above) into the tile -- byte moves only, any K that is a
//      multiple of 32.
//   SF the E8M0 scales, loaded by a warp of their own with 32-bit loads (four
//      K blocks = one stage per load) from row-major copies padded to SFS bytes
//      a row, stored into the 512-byte chunks tcgen05.cp copies to TMEM: byte
//      16 (r % 32) + 4 (r / 32) + j holds row r's scale of the stage's block j,
//      so TMEM lane r % 32 (replicated to all four lane quarters by .warpx4),
//      column r / 32, byte j holds it -- the layout the block-scaled MMA reads
//      with scale-factor id j.
//
// Roles (one CTA per SM, 448 threads): warp 0 TMA producer; warp 1 TMEM owner
// and MMA issuer (tcgen05.cp of the stage's scales, then four MMAs of K = 32);
// warps 2..5 epilogue; warps 7..10 converters; warps 6, 11, 12, 13 scale loaders
// (a stage's scales are one round trip of 32-bit loads, longer than its MMAs: four
// loaders keep four round trips in flight).  Loader j owns the ring slots s with
// s % 4 == j and feeds every use of them in order, so each of its parity waits is
// for the release of a use it fed itself (a loader that took uses of a slot in turn
// with other loaders could wait two phases ahead, where a parity wait passes at
// once).  Bounded waits throughout, as in grouped_gemm.cuh.
//
// Epilogues:
//   EPI_SWIGLU        NB = 2 (gate | up), TN = 96 features a tile (three 32-wide
//                     blocks): the clipped SwiGLU, then h quantized to MXFP8 --
//                     E4M3 codes into hq [R, F] and scales into sfh [R, SFS(F)].
//   EPI_BIAS_WSCATTER NB = 1, TN = 240: ys[slot] = w[slot] * (C + b_d), fp32 rows
//                     in slot order (the routing weight and un-permutation).
#pragma once

#include "grouped_gemm.cuh"

namespace moe {

constexpr int kMx8Threads = 448;
constexpr int kMx8ConvWarps = 4;
constexpr int kMx8SfWarps = 4;
constexpr int kMx8BK = 128;                 // K elements per stage (= 128 B of E4M3)
constexpr int kMx8TNGateUp = 96;            // features per gate/up tile (F = 2880 = 30 x 96)
constexpr int kMx8TNDown = 240;             // outputs per down tile (D = 2880 = 12 x 240)
constexpr int kMx8StagesGateUp = 4;
constexpr int kMx8StagesDown = 3;

// bytes of scale per activation / weight row: four per 128-wide K block, rounded up to 16
__host__ __device__ constexpr int mx8_sf_stride(int K) { return ((4 * ((K + 127) / 128)) + 15) / 16 * 16; }

template <int TN, int NB>
struct Mx8Layout {
  static constexpr int N = TN * NB;                       // MMA N
  static constexpr int A_BYTES = kBM * kMx8BK;            // 16 KB of E4M3
  static constexpr int B_BYTES = N * kMx8BK;              // widened E2M1, 128 B a row
  static constexpr int P_BYTES = N * kMx8BK / 2;          // packed E2M1 as the TMA delivers it
  static constexpr int SF_CHUNKS_B = (N + 127) / 128;
  static constexpr int SF_BYTES = 512 * (1 + SF_CHUNKS_B);
  static constexpr int STAGE_BYTES = (A_BYTES + B_BYTES + P_BYTES + SF_BYTES + 1023) / 1024 * 1024;
  static constexpr int EXTRA = 1024 + 4096;
  static constexpr int smem_bytes(int stages) { return stages * STAGE_BYTES + EXTRA; }
  // TMEM: accumulators at columns 0 and 256, then the scales of A (4 columns) and B
  static constexpr int SFA_COL = 256 + (N + 3) / 4 * 4;
  static constexpr int SFB_COL = SFA_COL + 4;
  static_assert(N % 16 == 0 && N <= 256, "MMA N");
  static_assert(SFB_COL + 4 * SF_CHUNKS_B <= kTmemCols, "scales fit beside the accumulators");
  static_assert((TN * kMx8BK) % 1024 == 0, "the up operand starts on a swizzle atom");
  static_assert((N * 8) % (32 * kMx8ConvWarps) == 0, "16-byte chunks split evenly over the converters");
};

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------
// Instruction descriptor of kind::mxf8f6f4.block_scale: A E4M3 (0), B E2M1 (5),
// E8M0 scales, K-major operands, fp32 accumulator; the scale-factor ids pick the
// byte of each TMEM scale column the instruction uses.
__host__ __device__ constexpr uint32_t make_idesc_mx8(int M, int N, uint32_t a_sf_id, uint32_t b_sf_id) {
  return (b_sf_id << 4) | (0u << 7) | (5u << 10) | ((static_cast<uint32_t>(N) >> 3) << 17) | (1u << 23) |
         ((static_cast<uint32_t>(M) >> 4) << 24) | (a_sf_id << 29);
}

__device__ __forceinline__ void tc_mma_mx8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// 32 rows x 16 B of shared memory to TMEM lanes 0..31 (and copies in lanes 32..127),
// four consecutive 32-bit columns from `taddr`.
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory descriptor of a 32 x 16 B scale chunk: no swizzle, 8-row core
// matrices of 128 B one after another (both byte offsets 128).
__device__ __forceinline__ uint64_t sf_chunk_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(128 >> 4) << 16;
  d |= static_cast<uint64_t>(128 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// The block scale exponent: the smallest X with amax <= 448 * 2^X (448 = 1.75 * 2^8),
// read off amax's exponent and mantissa bits; -127 for zero and for amax < 2^-126.
__device__ __forceinline__ int mx8_exponent(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int ef = static_cast<int>((b >> 23) & 0xFFu);
  if (ef == 0) return -127;
  const int X = (ef - 127) - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return max(-127, min(127, X));
}

// 2^e for an integer e in [-127, 127], exactly.
__device__ __forceinline__ float exp2_int(int e) {
  return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// Two floats to E4M3, round to nearest even (satfinite), `lo` in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Quantizes 32 values (one block) to MXFP8: 32 E4M3 bytes in q[8] (little-endian
// words) and the E8M0 scale byte.
__device__ __forceinline__ uint32_t mx8_quantize32(const float (&v)[32], uint32_t (&q)[8]) {
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
  const int X = mx8_exponent(amax);
  const float inv = exp2_int(-X);
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const uint32_t p0 = e4m3x2(v[4 * w] * inv, v[4 * w + 1] * inv);
    const uint32_t p1 = e4m3x2(v[4 * w + 2] * inv, v[4 * w + 3] * inv);
    q[w] = p0 | (p1 << 16);
  }
  return static_cast<uint32_t>(X + 127);
}

// ---------------------------------------------------------------------------
// activations to MXFP8: x [T, K] bf16 -> xq [T, K] E4M3, sf [T, SFS] E8M0
// (scales of K/32 blocks, then 127 = 2^0 up to SFS so that padded K blocks scale
// finite zeros).  One warp a row, a lane a 32-element block.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) mx8_quant_rows_kernel(const __nv_bfloat16* __restrict__ x, int T, int K,
                                                             int SFS, uint8_t* __restrict__ xq,
                                                             uint8_t* __restrict__ sf) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int nb = K / 32;
  for (int t = gw; t < T; t += nw) {
    const __nv_bfloat16* row = x + static_cast<size_t>(t) * K;
    for (int b = lane; b < nb; b += 32) {
      float v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float f[8];
        load8<__nv_bfloat16>(row + 32 * b + 8 * c, f);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[8 * c + j] = f[j];
      }
      uint32_t q[8];
      const uint32_t s = mx8_quantize32(v, q);
      uint4* dst = reinterpret_cast<uint4*>(xq + static_cast<size_t>(t) * K + 32 * b);
      dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
      dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
      sf[static_cast<size_t>(t) * SFS + b] = static_cast<uint8_t>(s);
    }
    for (int b = nb + lane; b < SFS; b += 32) sf[static_cast<size_t>(t) * SFS + b] = 127;
  }
}

// Weight scales [G, N, K/32] -> [G, N, SFS] (127 past K/32), for up to three matrices.
struct Mx8SfJob {
  const uint8_t* src[3];
  uint8_t* dst[3];
  int rows[3];     // G * N
  int nblk[3];     // K / 32
  int sfs[3];      // SFS(K)
};
// One thread per 16-byte chunk of an output row (the rows are tens of bytes; 32-bit indices).
__global__ void __launch_bounds__(256) mx8_weight_sf_kernel(Mx8SfJob job) {
  pdl_enter();
  const int m = blockIdx.y;
  const int rows = m == 0 ? job.rows[0] : m == 1 ? job.rows[1] : job.rows[2];
  const int nblk = m == 0 ? job.nblk[0] : m == 1 ? job.nblk[1] : job.nblk[2];
  const int sfs = m == 0 ? job.sfs[0] : m == 1 ? job.sfs[1] : job.sfs[2];
  const uint8_t* src = m == 0 ? job.src[0] : m == 1 ? job.src[1] : job.src[2];
  uint8_t* dst = m == 0 ? job.dst[0] : m == 1 ? job.dst[1] : job.dst[2];
  const int cpr = sfs / 16;
  const int total = rows * cpr;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int r = i / cpr;
    const int c = i - r * cpr;
    const uint8_t* s = src + static_cast<size_t>(r) * nblk;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t v = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int j = 16 * c + 4 * q + b;
        v |= (j < nblk ? static_cast<uint32_t>(s[j]) : 127u) << (8 * b);
      }
      w[q] = v;
    }
    *reinterpret_cast<uint4*>(dst + static_cast<size_t>(r) * sfs + 16 * c) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ---------------------------------------------------------------------------
// arguments of the block-scaled GEMM
// ---------------------------------------------------------------------------
struct Mx8Args {
  const int32_t* group_off;   // [G+1]
  int num_groups;
  int m_total;                // rows of A
  int n_out;                  // weight rows per operand (F for gate/up, D for down)
  int k_dim;                  // K
  const uint8_t* sfa;         // [m_total, sfs_a] activation scales
  int sfs_a;
  const uint8_t* sfw0;        // [G, n_out, sfs_a] weight scales of B0 (and B1)
  const uint8_t* sfw1;
  const void* bias0;          // bf16 [G, n_out]
  const void* bias1;
  float limit, alpha, gate_lo;
  uint8_t* hq;                // EPI_SWIGLU: [m_total, n_out] E4M3
  uint8_t* sfh;               // EPI_SWIGLU: [m_total, sfs_h]
  int sfs_h;
  float* out;                 // EPI_BIAS_WSCATTER: [m_total, n_out] fp32, slot order
  const int32_t* slot_of_row;
  const float* topk_w;
  unsigned long long wait_limit_ns;
  int kb_unpacked;            // K blocks [0, kb_unpacked) come through the unpacking maps
};

// ---------------------------------------------------------------------------
// epilogues (one thread = one accumulator row)
// ---------------------------------------------------------------------------
// gate/up: TMEM columns [gate 0..TN-1 | up TN..2TN-1].
template <int TN>
__device__ __forceinline__ void mx8_epi_swiglu(uint32_t tbase, int row, bool rvalid, const TileInfo& ti,
                                               const Mx8Args& a) {
  const int F = a.n_out;
  using T = __nv_bfloat16;
  const T* bg = static_cast<const T*>(a.bias0) + static_cast<size_t>(ti.g) * F;
  const T* bu = static_cast<const T*>(a.bias1) + static_cast<size_t>(ti.g) * F;
#pragma unroll 1
  for (int b = 0; b < TN / 32; ++b) {
    const int f0 = ti.n0 + 32 * b;
    float g[32], u[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      tmem_ld8(tbase + 32 * b + 8 * c, *reinterpret_cast<float(*)[8]>(g + 8 * c));
      tmem_ld8(tbase + TN + 32 * b + 8 * c, *reinterpret_cast<float(*)[8]>(u + 8 * c));
    }
    tmem_ld_wait();
    if (!rvalid || f0 >= F) continue;
    float h[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float b0[8], b1[8];
      load8<T>(bg + f0 + 8 * c, b0);
      load8<T>(bu + f0 + 8 * c, b1);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float gc = fminf(fmaxf(g[8 * c + j] + b0[j], a.gate_lo), a.limit);
        const float uc = fminf(fmaxf(u[8 * c + j] + b1[j], -a.limit), a.limit);
        h[8 * c + j] = __fdividef(gc * uc, 1.0f + __expf(-a.alpha * gc));
      }
    }
    uint32_t q[8];
    const uint32_t s = mx8_quantize32(h, q);
    uint4* dst = reinterpret_cast<uint4*>(a.hq + static_cast<size_t>(row) * F + f0);
    dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
    dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
    a.sfh[static_cast<size_t>(row) * a.sfs_h + f0 / 32] = static_cast<uint8_t>(s);
  }
  // scales of the padded K blocks of the down projection: 2^0 (finite, multiplying zeros)
  if (rvalid && ti.n0 == 0)
    for (int c = F / 32; c < a.sfs_h; ++c) a.sfh[static_cast<size_t>(row) * a.sfs_h + c] = 127;
}

// down: TMEM columns 0..TN-1 = outputs n0..n0+TN-1; fp32 rows in slot order.
template <int TN>
__device__ __forceinline__ void mx8_epi_wscatter(uint32_t tbase, int row, bool rvalid, const TileInfo& ti,
                                                 const Mx8Args& a) {
  const int D = a.n_out;
  using T = __nv_bfloat16;
  float wv = 0.0f;
  size_t orow = 0;
  if (rvalid) {
    const int s = a.slot_of_row[row];
    if (s < 0 || s >= a.m_total) {
      flag_error(DEVERR_BOUNDS);
      rvalid = false;
    } else {
      orow = static_cast<size_t>(s);
      wv = a.topk_w[s];
    }
  }
  const T* bd = static_cast<const T*>(a.bias0) + static_cast<size_t>(ti.g) * D;
#pragma unroll 1
  for (int c = 0; c < TN; c += 8) {
    float v[8];
    tmem_ld8(tbase + c, v);
    tmem_ld_wait();
    const int d0 = ti.n0 + c;
    if (!rvalid || d0 >= D) continue;
    float b[8];
    load8<T>(bd + d0, b);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = wv * (v[j] + b[j]);
    store8<float>(a.out + orow * D + d0, v);
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
// tmA: E4M3 activations [m_total, K]; tmB0 / tmB1: packed E2M1 weights [G, n_out, K/2] bytes,
// boxes of 64 B (128 codes) x TN rows; tmU0 / tmU1: the same weights through the 4-bit
// unpacking type, boxes of 128 codes x TN rows (used for K blocks below kb_unpacked).
template <int EPI, int TN, int NB, int STAGES>
__global__ void __launch_bounds__(kMx8Threads, 1)
    grouped_gemm_mx8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                            const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmU0,
                            const __grid_constant__ CUtensorMap tmU1, const Mx8Args args) {
  pdl_enter();
  using LY = Mx8Layout<TN, NB>;
  constexpr int N = LY::N;
  constexpr int KSTEPS = kMx8BK / 32;     // MMAs per stage (K = 32 each)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * LY::STAGE_BYTES);
  uint64_t* conv = full + STAGES;              // widened B tile and scales in place
  uint64_t* empty = conv + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* never_flag = abort_flag + 1;
  int* tile_off = never_flag + 2;              // [G+1]
  int* goff = tile_off + (kMaxGroups + 2);     // [G+1]
  // a stage: [A | B widened | B packed | scales]
  auto stage_a = [&](int s) { return smem + s * LY::STAGE_BYTES; };
  auto stage_b = [&](int s) { return smem + s * LY::STAGE_BYTES + LY::A_BYTES; };
  auto stage_p = [&](int s) { return smem + s * LY::STAGE_BYTES + LY::A_BYTES + LY::B_BYTES; };
  auto stage_sf = [&](int s) { return smem + s * LY::STAGE_BYTES + LY::A_BYTES + LY::B_BYTES + LY::P_BYTES; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = args.num_groups;
  const int NT = (args.n_out + TN - 1) / TN;
  const int KB = (args.k_dim + kMx8BK - 1) / kMx8BK;
  const uint64_t lim = args.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&conv[s], kMx8ConvWarps + 1);   // the converter warps and the scale loader
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
      if (args.kb_unpacked > 0) {
        tma_prefetch_desc(&tmU0);
        if (NB == 2) tma_prefetch_desc(&tmU1);
      }
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // an unpacked box counts the packed bytes it reads, as a packed box does
      const uint32_t tx_bytes = LY::A_BYTES + LY::P_BYTES;
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
        const TileInfo ti = decode_tile(i, tile_off, goff, G, NT, TN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], tx_bytes);
          tma_load_2d(stage_a(s), &tmA, &full[s], kb * kMx8BK, ti.m0);
          if (kb < args.kb_unpacked) {
            tma_load_3d(stage_b(s), &tmU0, &full[s], kb * kMx8BK, ti.n0, ti.g);
            if (NB == 2) tma_load_3d(stage_b(s) + TN * kMx8BK, &tmU1, &full[s], kb * kMx8BK, ti.n0, ti.g);
          } else {
            tma_load_3d(stage_p(s), &tmB0, &full[s], kb * (kMx8BK / 2), ti.n0, ti.g);
            if (NB == 2) tma_load_3d(stage_p(s) + TN * (kMx8BK / 2), &tmB1, &full[s], kb * (kMx8BK / 2), ti.n0, ti.g);
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
  } else if (warp >= 7 && warp <= 10) {
    // ------------------------------------------------------------ converters: packed -> widened B
    // 16-byte chunk q of the tile (row q / 8, chunk q % 8) takes the 8 packed bytes of its 16 codes
    // and zeros; chunk c of row r sits at r * 128 + ((c ^ (r % 8)) * 16) under the 128-byte swizzle
    const int ct = threadIdx.x - 7 * 32;
    constexpr int PER = N * 8 / (32 * kMx8ConvWarps);
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag, lim))) { ok = false; break; }
        if (kb >= args.kb_unpacked) {   // an unpacked stage is already in place
          const uint8_t* src = stage_p(s);
          uint8_t* dst = stage_b(s);
          uint2 v[PER];
#pragma unroll
          for (int j = 0; j < PER; ++j) {
            const int q = ct + j * 32 * kMx8ConvWarps;
            v[j] = *reinterpret_cast<const uint2*>(src + 8 * q);
          }
#pragma unroll
          for (int j = 0; j < PER; ++j) {
            const int q = ct + j * 32 * kMx8ConvWarps;
            const int r = q >> 3, c = q & 7;
            *reinterpret_cast<uint4*>(dst + r * 128 + ((c ^ (r & 7)) << 4)) = make_uint4(v[j].x, v[j].y, 0u, 0u);
          }
          fence_proxy_async_smem();   // the widened tile is read by the tensor core (async proxy)
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&conv[s]);
        if (++s == STAGES) { s = 0; ph ^= 1u; }
      }
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      flag_error(DEVERR_TIMEOUT);
    }
  } else if (warp == 6 || warp > 10) {
    // ------------------------------------------------------------ scale loaders (slot s: loader s % 4)
    // Step n of this CTA is K block n % KB of its (n / KB)-th tile.  A loader issues the
    // global loads of its next step before it waits for the current step's slot, so the
    // load round trip overlaps the wait.
    const int me = warp == 6 ? 0 : warp - 10;
    const uint32_t one = 0x7F7F7F7Fu;   // four scales of 2^0
    const int my_tiles = static_cast<int>(blockIdx.x) < total
                             ? (total - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                                   static_cast<int>(gridDim.x)
                             : 0;
    const int steps = my_tiles * KB;
    auto owned_from = [&](int n) {      // first step >= n whose slot this loader owns
      while (n < steps && (n % STAGES) % kMx8SfWarps != me) ++n;
      return n;
    };
    constexpr int NB4 = 4 * LY::SF_CHUNKS_B;
    auto load = [&](int n, uint32_t (&va)[4], uint32_t (&vb)[NB4]) {
      const TileInfo ti = decode_tile(static_cast<int>(blockIdx.x) + (n / KB) * static_cast<int>(gridDim.x),
                                      tile_off, goff, G, NT, TN);
      const int kb = n % KB;
#pragma unroll
      for (int j = 0; j < 4; ++j) {            // A rows lane + 32 j
        const int r = ti.m0 + lane + 32 * j;
        va[j] = r < args.m_total
                    ? *reinterpret_cast<const uint32_t*>(args.sfa + static_cast<size_t>(r) * args.sfs_a + 4 * kb)
                    : one;
      }
#pragma unroll
      for (int j = 0; j < NB4; ++j) {          // B positions lane + 32 j
        const int c = lane + 32 * j;
        uint32_t v = one;
        if (c < N) {
          const int op = c / TN;
          const int nrow = ti.n0 + (c - op * TN);
          if (nrow < args.n_out) {
            const uint8_t* src = op == 0 ? args.sfw0 : args.sfw1;
            v = *reinterpret_cast<const uint32_t*>(
                src + (static_cast<size_t>(ti.g) * args.n_out + nrow) * args.sfs_a + 4 * kb);
          }
        }
        vb[j] = v;
      }
    };
    bool ok = true;
    uint32_t va[4], vb[NB4], na[4], nb[NB4];
    int n = owned_from(0);
    if (n < steps) load(n, va, vb);
    while (ok && n < steps) {
      const int next = owned_from(n + 1);
      if (next < steps) load(next, na, nb);
      const int s = n % STAGES;
      const uint32_t ph = static_cast<uint32_t>(n / STAGES) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim))) { ok = false; break; }
      uint8_t* sf = stage_sf(s);
      *reinterpret_cast<uint4*>(sf + 16 * lane) = make_uint4(va[0], va[1], va[2], va[3]);
#pragma unroll
      for (int ch = 0; ch < LY::SF_CHUNKS_B; ++ch)
        *reinterpret_cast<uint4*>(sf + 512 * (1 + ch) + 16 * lane) =
            make_uint4(vb[4 * ch], vb[4 * ch + 1], vb[4 * ch + 2], vb[4 * ch + 3]);
      fence_proxy_async_smem();   // the stores above are read by tcgen05.cp (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(&conv[s]);
#pragma unroll
      for (int j = 0; j < 4; ++j) va[j] = na[j];
#pragma unroll
      for (int j = 0; j < NB4; ++j) vb[j] = nb[j];
      n = next;
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      flag_error(DEVERR_TIMEOUT);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t sfa_t = tmem_base + static_cast<uint32_t>(LY::SFA_COL);
      const uint32_t sfb_t = tmem_base + static_cast<uint32_t>(LY::SFB_COL);
      int s = 0, it = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = blockIdx.x; ok && i < total; i += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccStride);
        for (int kb = 0; kb < KB; ++kb) {
          // the converters waited for the TMA (A, packed B) before arriving here
          if (!mbar_wait(&conv[s], ph, abort_flag, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stage_a(s));
          const uint32_t b_addr = smem_u32(stage_b(s));
          const uint32_t sf_addr = smem_u32(stage_sf(s));
          // the stage's scales into TMEM; tcgen05 operations of this thread run in order,
          // so the previous stage's MMAs have read the old scales before these land
          tc_cp_sf(sfa_t, sf_chunk_desc(sf_addr));
#pragma unroll
          for (int ch = 0; ch < LY::SF_CHUNKS_B; ++ch)
            tc_cp_sf(sfb_t + 4 * ch, sf_chunk_desc(sf_addr + 512 * (1 + ch)));
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk) {
            const uint32_t sel = static_cast<uint32_t>(kk) << 30;   // scale byte kk of each TMEM column
            tc_mma_mx8(d_tmem, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32),
                       make_idesc_mx8(kBM, N, kk, kk), sfa_t | sel, sfb_t | sel, (kb | kk) != 0 ? 1u : 0u);
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
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;
    const int r_in_tile = quarter * 32 + lane;
    int it = 0;
    bool ok = true;
    for (int i = blockIdx.x; i < total; i += gridDim.x, ++it) {
      const TileInfo ti = decode_tile(i, tile_off, goff, G, NT, TN);
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, abort_flag, lim));
      if (!got) { ok = false; break; }
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kAccStride);
      const int row = ti.m0 + r_in_tile;
      const bool rvalid = row < ti.m_end;
      if constexpr (EPI == EPI_SWIGLU) mx8_epi_swiglu<TN>(tbase, row, rvalid, ti, args);
      else mx8_epi_wscatter<TN>(tbase, row, rvalid, ti, args);
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
