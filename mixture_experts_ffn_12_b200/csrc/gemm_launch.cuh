#pragma once
// Host side of the tcgen05 grouped GEMMs: TMA tensor maps and launches.
//
//   router (bf16, many tokens)  A = x [T, D],        B = Wr [1, E, D],   EPI_TOPK
//   gate/up                     A = x_perm [R, D],   B = W_g, W_u [E, F, D], EPI_SWIGLU
//   down                        A = h [R, F],        B = W_d [E, D, F],  EPI_BIAS / EPI_BIAS_WSCATTER
//
// fp32 layers use the fp32-FMA grouped GEMM of simt_gemm.cuh instead.
// Every operand is K-major; tensor maps cut [rows x 128 B] boxes with the
// 128-byte swizzle, out-of-range rows and columns read as zero (ragged expert
// segments, the last column block of F or D, a partial last K block).
#include <mutex>

#include "grouped_gemm.cuh"
#include "decode_gemm.cuh"
#include "decode_layer.cuh"
#include "grouped_gemm_pair.cuh"
#include "grouped_gemm_pair_mx.cuh"
#include "grouped_gemm_mx8.cuh"
#include "grouped_gemm_wm_pair.cuh"
#include "internal.h"
#include "simt_gemm.cuh"

namespace moe {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// K-major matrix: [rows, K] (groups == 0) or [groups, rows, K]; box = box_rows x 128 bytes.
static cudaError_t make_tmap(CUtensorMap* m, const void* ptr, bool f32, uint64_t K, uint64_t rows, uint64_t groups,
                             uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const uint64_t elem = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {K, rows, groups ? groups : 1};
  const cuuint64_t strides[2] = {K * elem, K * elem * rows};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kRowBytes / elem), box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        groups ? 3 : 2, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// h kept as two bf16 halves per row, [rows][2][K]: dims {K, 2, rows}; a box is box_rows rows
// of one half x 128 bytes, laid out in shared memory exactly as a [box_rows x 128 B] box of a
// plain [rows, K] map (the middle dimension's box is 1).
static cudaError_t make_tmap_halves(CUtensorMap* m, const void* ptr, uint64_t K, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {K, 2, rows};
  const cuuint64_t strides[2] = {K * 2, K * 2 * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kRowBytes / 2), 1, box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Packed MXFP4 rows: [groups, rows, K/2] bytes, boxes of box_rows x 32 bytes (64 codes), no swizzle.
static cudaError_t make_tmap_packed(CUtensorMap* m, const void* ptr, uint64_t K, uint64_t rows, uint64_t groups,
                                   uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {K / 2, rows, groups};
  const cuuint64_t strides[2] = {K / 2, (K / 2) * rows};
  const cuuint32_t box[3] = {32, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Relaid MXFP4 scales: [groups][KB][2 * rows] bytes, boxes of box_bytes x 1 x 1, no swizzle.
static cudaError_t make_tmap_scales(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t KB, uint64_t groups,
                                   uint32_t box_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {2 * rows, KB, groups};
  const cuuint64_t strides[2] = {2 * rows, 2 * rows * KB};
  const cuuint32_t box[3] = {box_bytes, 1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <typename T, int TN, int NB, int EPI, int STAGES>
static cudaError_t launch(const Launch& L, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                          const GemmArgs& args, int64_t max_tiles) {
  if (max_tiles <= 0) return cudaSuccess;
  auto kern = grouped_gemm_kernel<T, TN, NB, EPI, STAGES>;
  constexpr int smem = GemmLayout<TN, NB>::smem_bytes(STAGES);
  static_assert(smem <= 232448, "shared memory budget");
  int dev = 0;
  cudaGetDevice(&dev);
  static std::mutex mu;
  static uint64_t configured = 0;   // one bit per device
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev >= 64 || !((configured >> dev) & 1u)) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      if (dev < 64) configured |= uint64_t(1) << dev;
    }
  }
  const int grid = static_cast<int>(std::min<int64_t>(max_tiles, L.num_sms));
  pdl_launch(kern, dim3(grid), dim3(kGemmThreads), smem, L.stream, a, b0, b1, args);
  count_launch();
  return cudaGetLastError();
}

// CTA-pair kernels (cluster of 2; grid = 2 x clusters).
template <int TNH, int EPI, int STAGES>
static cudaError_t launch_pair(const Launch& L, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                               const GemmArgs& args, int64_t max_tiles) {
  if (max_tiles <= 0) return cudaSuccess;
  auto kern = grouped_gemm_pair_kernel<TNH, EPI, STAGES>;
  constexpr int smem = PairLayout<TNH>::smem_bytes(STAGES);
  static_assert(smem <= 232448, "shared memory budget");
  int dev = 0;
  cudaGetDevice(&dev);
  static std::mutex mu;
  static uint64_t configured = 0;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev >= 64 || !((configured >> dev) & 1u)) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      if (dev < 64) configured |= uint64_t(1) << dev;
    }
  }
  const int clusters = static_cast<int>(std::min<int64_t>(max_tiles, L.num_sms / 2));
  pdl_launch(kern, dim3(2 * clusters), dim3(kGemmThreads), smem, L.stream, a, b0, b1, args);
  count_launch();
  return cudaGetLastError();
}

template <int TNH, int EPI, int STAGES>
static cudaError_t launch_pair_mx(const Launch& L, const CUtensorMap& a, const CUtensorMap& p0, const CUtensorMap& p1,
                                  const CUtensorMap& s0, const CUtensorMap& s1, const GemmArgs& args,
                                  int64_t max_tiles) {
  if (max_tiles <= 0) return cudaSuccess;
  auto kern = grouped_gemm_pair_mx_kernel<TNH, EPI, STAGES>;
  constexpr int smem = PairMxLayout<TNH>::smem_bytes(STAGES);
  static_assert(smem <= 232448, "shared memory budget");
  int dev = 0;
  cudaGetDevice(&dev);
  static std::mutex mu;
  static uint64_t configured = 0;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev >= 64 || !((configured >> dev) & 1u)) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      if (dev < 64) configured |= uint64_t(1) << dev;
    }
  }
  const int clusters = static_cast<int>(std::min<int64_t>(max_tiles, L.num_sms / 2));
  pdl_launch(kern, dim3(2 * clusters), dim3(kMxThreads), smem, L.stream, a, p0, p1, s0, s1, args);
  count_launch();
  return cudaGetLastError();
}

// CTA pairs with the weights in M (cluster of 2; grid = 2 x clusters).
template <int EPI>
static cudaError_t launch_wm_pair(const Launch& L, const CUtensorMap& w0, const CUtensorMap& w1, const CUtensorMap& x,
                                  const CUtensorMap& x16, const GemmArgs& args, int64_t max_units) {
  if (max_units <= 0) return cudaSuccess;
  auto kern = grouped_gemm_wm_pair_kernel<EPI, kWmStages>;
  constexpr int smem = WmLayout::smem_bytes(kWmStages);
  static_assert(smem <= 232448, "shared memory budget");
  int dev = 0;
  cudaGetDevice(&dev);
  static std::mutex mu;
  static uint64_t configured = 0;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev >= 64 || !((configured >> dev) & 1u)) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      if (dev < 64) configured |= uint64_t(1) << dev;
    }
  }
  const int clusters = static_cast<int>(std::min<int64_t>(max_units, L.num_sms / 2));
  pdl_launch(kern, dim3(2 * clusters), dim3(kGemmThreads), smem, L.stream, w0, w1, x, x16, args);
  count_launch();
  return cudaGetLastError();
}

// Expert-GEMM variant (moe_set_expert_gemm_variant): 0 = by size, 1 = single-CTA
// tiles, 2 = CTA-pair tiles, 3 = weight-stationary decode kernel, 4 = CTA pairs
// with the weights in M, 5 = the two-kernel decode layer wherever it applies,
// 6 = by size, except that the layer's gate/up rows are gathered from x (TMA gather4),
// 7 = by size, and the MXFP4 x MXFP8 GEMMs widen every E2M1 stage in their converter warps.
inline std::atomic<int> g_gemm_variant{0};

enum GemmKind { GK_SINGLE = 1, GK_PAIR = 2, GK_DECODE = 3, GK_WM_PAIR = 4 };

// By default: the decode kernel while experts average at most 16 rows (the
// layer is a weight stream); otherwise single-CTA 128-row tiles for gate/up and
// CTA pairs for down (measured fastest for each on the GPT-OSS shapes).
static GemmKind gemm_kind(int64_t R, int E, bool down = false) {
  const int v = g_gemm_variant.load();
  if (v >= 1 && v <= 4) return static_cast<GemmKind>(v);
  if (R <= int64_t(16) * E) return GK_DECODE;
  return down ? GK_PAIR : GK_SINGLE;
}
static bool use_pair(int64_t R, int E, bool down = false) { return gemm_kind(R, E, down) == GK_PAIR; }

constexpr int kDecTok = 32;

template <int EPI, int STAGES>
static cudaError_t launch_decode_st(const Launch& L, const CUtensorMap& w0, const CUtensorMap& w1,
                                    const CUtensorMap& x, const GemmArgs& args, int grid) {
  auto kern = decode_gemm_kernel<EPI, kDecTok, STAGES, kDecKBS>;
  constexpr int smem = DecLayout<kDecTok, kDecKBS>::smem_bytes(STAGES);
  static_assert(smem <= 232448, "shared memory budget");
  int dev = 0;
  cudaGetDevice(&dev);
  static std::mutex mu;
  static uint64_t configured = 0;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev >= 64 || !((configured >> dev) & 1u)) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      if (dev < 64) configured |= uint64_t(1) << dev;
    }
  }
  pdl_launch(kern, dim3(grid), dim3(kGemmThreads), smem, L.stream, w0, w1, x, args);
  count_launch();
  return cudaGetLastError();
}

// Up to one unit per SM: one CTA per SM with the deep ring.  More units than SMs:
// two CTAs per SM with half the ring each, so every unit of a short list (T = 1
// gate/up: 4 experts x 45 feature blocks = 180 units) streams at once instead of
// a second partial wave.
template <int EPI>
static cudaError_t launch_decode(const Launch& L, const CUtensorMap& w0, const CUtensorMap& w1, const CUtensorMap& x,
                                 const GemmArgs& args, int64_t max_units) {
  if (max_units <= 0) return cudaSuccess;
  if (max_units <= L.num_sms)
    return launch_decode_st<EPI, kDecStages>(L, w0, w1, x, args, static_cast<int>(max_units));
  const int grid = static_cast<int>(std::min<int64_t>(max_units, int64_t(2) * L.num_sms));
  return launch_decode_st<EPI, kDecStagesDual>(L, w0, w1, x, args, grid);
}

static GemmArgs base_args(const Launch& L) {
  GemmArgs a{};
  a.wait_limit_ns = L.wait_limit_ns;
  a.alpha = 1.702f;
  return a;
}

static int64_t max_row_blocks(int64_t R, int G) { return (R + kBM - 1) / kBM + G; }

constexpr int kStages = 4;
constexpr int kPairStages = 6;
constexpr int kTNHalf = 120;     // pair tiles: each CTA holds 120 B rows (N = 240)
constexpr int kTNGateUp = 128;   // 2 x 128 = 256 MMA columns (F = 2880: 23 column blocks, the last half used)
constexpr int kTNDown = 240;     // D = 2880 = 12 x 240

cudaError_t router_tc(const Launch& L, int64_t T, int D, int E, int k, const void* x, const void* w_router,
                      const void* b_router, int32_t* ids, float* w) {
  const int mma_n = (E + 15) / 16 * 16;
  CUtensorMap ta, tb;
  cudaError_t e;
  if ((e = make_tmap(&ta, x, false, D, T, 0, kBM)) != cudaSuccess) return e;
  if ((e = make_tmap(&tb, w_router, false, D, E, 1, mma_n)) != cudaSuccess) return e;
  GemmArgs a = base_args(L);
  a.group_off = nullptr;
  a.num_groups = 1;
  a.m_total = static_cast<int>(T);
  a.n_out = E;
  a.k_dim = D;
  a.mma_n = mma_n;
  a.bias0 = b_router;
  a.topk_ids = ids;
  a.topk_wout = w;
  a.topk_k = k;
  // one CTA per 128 tokens: few CTAs stream x, so the ring is as deep as shared memory allows
  const int64_t tiles = (T + kBM - 1) / kBM;
  if (mma_n <= 64) return launch<__nv_bfloat16, 64, 1, EPI_TOPK, 9>(L, ta, tb, tb, a, tiles);
  if (mma_n <= 128) return launch<__nv_bfloat16, 128, 1, EPI_TOPK, 6>(L, ta, tb, tb, a, tiles);
  return launch<__nv_bfloat16, 256, 1, EPI_TOPK, kStages>(L, ta, tb, tb, a, tiles);
}

// Router with K split over `splits` ranges: tile (m, s) writes fp32 partial logits of
// tokens m*128.. over K range s to partial[s][E][T] (expert-major); the top-k kernel sums them.
cudaError_t router_tc_partial(const Launch& L, int64_t T, int D, int E, int splits, const void* x,
                              const void* w_router, float* partial) {
  const int mma_n = (E + 15) / 16 * 16;
  CUtensorMap ta, tb;
  cudaError_t e;
  if ((e = make_tmap(&ta, x, false, D, T, 0, kBM)) != cudaSuccess) return e;
  if ((e = make_tmap(&tb, w_router, false, D, E, 1, mma_n)) != cudaSuccess) return e;
  GemmArgs a = base_args(L);
  a.group_off = nullptr;
  a.num_groups = 1;
  a.m_total = static_cast<int>(T);
  a.n_out = E;
  a.k_dim = D;
  a.mma_n = mma_n;
  a.k_splits = splits;
  a.partial = partial;
  const int64_t tiles = (T + kBM - 1) / kBM * splits;
  if (mma_n <= 64) return launch<__nv_bfloat16, 64, 1, EPI_PARTIAL, 9>(L, ta, tb, tb, a, tiles);
  if (mma_n <= 128) return launch<__nv_bfloat16, 128, 1, EPI_PARTIAL, 6>(L, ta, tb, tb, a, tiles);
  return launch<__nv_bfloat16, 256, 1, EPI_PARTIAL, kStages>(L, ta, tb, tb, a, tiles);
}

constexpr int kMxStages = 5;

size_t mx_scale_bytes(int rows, int K, int E) {
  return static_cast<size_t>(E) * ((K + 63) / 64) * rows * 2;
}

cudaError_t mx_scale_relayout(const Launch& L, int D, int F, int E, const ExpertWeights& w, uint8_t* s_gate,
                              uint8_t* s_up, uint8_t* s_down) {
  MxScaleJob job{};
  job.src[0] = w.s_gate; job.dst[0] = s_gate; job.rows[0] = F; job.kdim[0] = D;
  job.src[1] = w.s_up;   job.dst[1] = s_up;   job.rows[1] = F; job.kdim[1] = D;
  job.src[2] = w.s_down; job.dst[2] = s_down; job.rows[2] = D; job.kdim[2] = F;
  job.groups = E;
  const int64_t most = std::max(mx_scale_bytes(F, D, E), mx_scale_bytes(D, F, E)) / 2;
  const dim3 grid(static_cast<unsigned>(std::min<int64_t>((most + 255) / 256, int64_t(8) * L.num_sms)), 3);
  pdl_launch(mx_scale_relayout_kernel, dim3(grid), dim3(256), 0, L.stream, job);
  count_launch();
  return cudaGetLastError();
}

cudaError_t expert_gateup_mxfp4(const Launch& L, int64_t R, int D, int F, int E, const void* x_perm,
                                const int32_t* expert_off, const ExpertWeights& w, const uint8_t* s_gate2,
                                const uint8_t* s_up2, float limit, float alpha, void* h) {
  if (R == 0) return cudaSuccess;
  CUtensorMap ta, pg, pu, sg, su;
  cudaError_t e;
  const int KB = (D + 63) / 64;
  if ((e = make_tmap(&ta, x_perm, false, D, R, 0, kBM)) != cudaSuccess) return e;
  if ((e = make_tmap_packed(&pg, w.w_gate, D, F, E, kTNHalf)) != cudaSuccess) return e;
  if ((e = make_tmap_packed(&pu, w.w_up, D, F, E, kTNHalf)) != cudaSuccess) return e;
  if ((e = make_tmap_scales(&sg, s_gate2, F, KB, E, 2 * kTNHalf)) != cudaSuccess) return e;
  if ((e = make_tmap_scales(&su, s_up2, F, KB, E, 2 * kTNHalf)) != cudaSuccess) return e;
  GemmArgs a = base_args(L);
  a.group_off = expert_off;
  a.num_groups = E;
  a.m_total = static_cast<int>(R);
  a.n_out = F;
  a.k_dim = D;
  a.bias0 = w.b_gate;
  a.bias1 = w.b_up;
  a.limit = limit;
  a.alpha = alpha;
  a.out = h;
  a.ldo = F;
  const int64_t ptiles = ((R + kPairBM - 1) / kPairBM + E) * ((F + kTNHalf - 1) / kTNHalf);
  return launch_pair_mx<kTNHalf, EPI_SWIGLU, kMxStages>(L, ta, pg, pu, sg, su, a, ptiles);
}

cudaError_t expert_down_mxfp4(const Launch& L, int64_t R, int D, int F, int E, const void* h,
                              const int32_t* expert_off, const ExpertWeights& w, const uint8_t* s_down2,
                              const int32_t* slot_of_row, const float* topk_w, void* out) {
  if (R == 0) return cudaSuccess;
  CUtensorMap ta, pd, sd;
  cudaError_t e;
  const int KB = (F + 63) / 64;
  if ((e = make_tmap(&ta, h, false, F, R, 0, kBM)) != cudaSuccess) return e;
  if ((e = make_tmap_packed(&pd, w.w_down, F, D, E, kTNHalf)) != cudaSuccess) return e;
  if ((e = make_tmap_scales(&sd, s_down2, D, KB, E, 2 * kTNHalf)) != cudaSuccess) return e;
  GemmArgs a = base_args(L);
  a.group_off = expert_off;
  a.num_groups = E;
  a.m_total = static_cast<int>(R);
  a.n_out = D;
  a.k_dim = F;
  a.bias0 = w.b_down;
  a.out = out;
  a.ldo = D;
  a.slot_of_row = slot_of_row;
  a.topk_w = topk_w;
  const int64_t ptiles = ((R + kPairBM - 1) / kPairBM + E) * ((D + 2 * kTNHalf - 1) / (2 * kTNHalf));
  if (slot_of_row != nullptr)
    return launch_pair_mx<kTNHalf, EPI_BIAS_WSCATTER, kMxStages>(L, ta, pd, pd, sd, sd, a, ptiles);
  return launch_pair_mx<kTNHalf, EPI_BIAS, kMxStages>(L, ta, pd, pd, sd, sd, a, ptiles);
}

// Whether the single-CTA gate/up kernel takes its A rows from x by TMA gather4 (so the
// layer needs no x_perm): only with expert-GEMM variant 6.  Correct (bit-identical to the
// x_perm form) but slower: a 128-row A tile takes 32 gather4 loads per 64-wide K block,
// and on the GPT-OSS-20B prefill layer gate/up ran 1.38-1.41 ms against 0.50 ms.
bool gateup_gathers(bool bf16, int64_t R, int E) {
  return bf16 && g_gemm_variant.load() == 6 && gemm_kind(R, E) == GK_SINGLE;
}

cudaError_t expert_gateup(const Launch& L, bool bf16, int64_t R, int D, int F, int E, const void* x_perm,
                          const int32_t* expert_off, const ExpertWeights& w, float limit, float alpha, void* h,
                          float gate_lo, int h_halves, const GateupGather* gather) {
  if (R == 0) return cudaSuccess;
  if (gather != nullptr && !gateup_gathers(bf16, R, E)) return cudaErrorInvalidValue;
  if (h_halves == 2 && (!bf16 || gemm_kind(R, E) == GK_WM_PAIR)) return cudaErrorNotSupported;
  if (!bf16) {
    GemmArgs a = base_args(L);
    a.group_off = expert_off;
    a.num_groups = E;
    a.m_total = static_cast<int>(R);
    a.n_out = F;
    a.k_dim = D;
    a.bias0 = w.b_gate;
    a.bias1 = w.b_up;
    a.limit = limit;
    a.alpha = alpha;
    a.gate_lo = gate_lo;
    a.out = h;
    a.ldo = F;
    const dim3 grid((F + kSimtBN - 1) / kSimtBN, static_cast<unsigned>((R + kSimtBM - 1) / kSimtBM + E));
    pdl_launch(simt_grouped_gemm_f32<EPI_SWIGLU>, dim3(grid), dim3(256), 0, L.stream, 
        static_cast<const float*>(x_perm), static_cast<const float*>(w.w_gate), static_cast<const float*>(w.w_up), a);
    count_launch();
    return cudaGetLastError();
  }
  CUtensorMap ta, tg, tu;
  cudaError_t e;
  // gathering: A is x [T, D] with one-row boxes, read four rows per gather4
  if (gather != nullptr) e = make_tmap(&ta, gather->x, false, D, gather->T, 0, 1);
  else e = make_tmap(&ta, x_perm, !bf16, D, R, 0, kBM);
  if (e != cudaSuccess) return e;
  if ((e = make_tmap(&tg, w.w_gate, !bf16, D, F, E, kTNGateUp)) != cudaSuccess) return e;
  if ((e = make_tmap(&tu, w.w_up, !bf16, D, F, E, kTNGateUp)) != cudaSuccess) return e;
  GemmArgs a = base_args(L);
  if (gather != nullptr) {
    a.gather_slots = gather->slot_of_row;
    a.gather_k = gather->k;
    a.gather_rows = static_cast<int>(gather->T);
  }
  a.group_off = expert_off;
  a.num_groups = E;
  a.m_total = static_cast<int>(R);
  a.n_out = F;
  a.k_dim = D;
  a.bias0 = w.b_gate;
  a.bias1 = w.b_up;
  a.limit = limit;
  a.alpha = alpha;
  a.gate_lo = gate_lo;
  a.out = h;
  a.ldo = h_halves == 2 ? 2 * F : F;
  a.h_halves = h_halves;
  if (gemm_kind(R, E) == GK_DECODE) {
    CUtensorMap wg, wu, tx;
    if ((e = make_tmap(&wg, w.w_gate, false, D, F, E, 64)) != cudaSuccess) return e;
    if ((e = make_tmap(&wu, w.w_up, false, D, F, E, 64)) != cudaSuccess) return e;
    if ((e = make_tmap(&tx, x_perm, false, D, R, 0, kDecTok)) != cudaSuccess) return e;
    const int64_t units = (std::min<int64_t>(E, R) + R / kDecTok) * ((F + 63) / 64);
    return launch_decode<EPI_SWIGLU>(L, wg, wu, tx, a, units);
  }
  if (gemm_kind(R, E) == GK_WM_PAIR) {
    CUtensorMap wg, wu, tx16;
    if ((e = make_tmap(&wg, w.w_gate, false, D, F, E, 16)) != cudaSuccess) return e;
    if ((e = make_tmap(&wu, w.w_up, false, D, F, E, 16)) != cudaSuccess) return e;
    if ((e = make_tmap(&tx16, x_perm, false, D, R, 0, 16)) != cudaSuccess) return e;
    const int64_t units = ((R + kWmTok - 1) / kWmTok + E) * ((F + 127) / 128);
    return launch_wm_pair<EPI_SWIGLU>(L, wg, wu, ta, tx16, a, units);
  }
  if (use_pair(R, E)) {
    // the pair kernel's weight halves are kTNHalf rows: boxes of that height
    CUtensorMap pg, pu;
    if ((e = make_tmap(&pg, w.w_gate, false, D, F, E, kTNHalf)) != cudaSuccess) return e;
    if ((e = make_tmap(&pu, w.w_up, false, D, F, E, kTNHalf)) != cudaSuccess) return e;
    const int64_t ptiles = ((R + kPairBM - 1) / kPairBM + E) * ((F + kTNHalf - 1) / kTNHalf);
    return launch_pair<kTNHalf, EPI_SWIGLU, kPairStages>(L, ta, pg, pu, a, ptiles);
  }
  const int64_t tiles = max_row_blocks(R, E) * ((F + kTNGateUp - 1) / kTNGateUp);
  return launch<__nv_bfloat16, kTNGateUp, 2, EPI_SWIGLU, kStages>(L, ta, tg, tu, a, tiles);
}

cudaError_t expert_down(const Launch& L, bool bf16, int64_t R, int D, int F, int E, const void* h,
                        const int32_t* expert_off, const ExpertWeights& w, const int32_t* slot_of_row,
                        const float* topk_w, void* out, int h_halves) {
  if (R == 0) return cudaSuccess;
  const bool hsplit = h_halves == 2;
  if (hsplit && (!bf16 || gemm_kind(R, E, true) == GK_WM_PAIR)) return cudaErrorNotSupported;
  if (!bf16) {
    GemmArgs a = base_args(L);
    a.group_off = expert_off;
    a.num_groups = E;
    a.m_total = static_cast<int>(R);
    a.n_out = D;
    a.k_dim = F;
    a.bias0 = w.b_down;
    a.out = out;
    a.ldo = D;
    a.slot_of_row = slot_of_row;
    a.topk_w = topk_w;
    const dim3 grid((D + kSimtBN - 1) / kSimtBN, static_cast<unsigned>((R + kSimtBM - 1) / kSimtBM + E));
    if (slot_of_row != nullptr)
      pdl_launch(simt_grouped_gemm_f32<EPI_BIAS_WSCATTER>, dim3(grid), dim3(256), 0, L.stream, 
          static_cast<const float*>(h), static_cast<const float*>(w.w_down), nullptr, a);
    else
      pdl_launch(simt_grouped_gemm_f32<EPI_BIAS>, dim3(grid), dim3(256), 0, L.stream, static_cast<const float*>(h),
                                                                  static_cast<const float*>(w.w_down), nullptr, a);
    count_launch();
    return cudaGetLastError();
  }
  CUtensorMap ta, tb;
  cudaError_t e;
  if (hsplit) e = make_tmap_halves(&ta, h, F, R, kBM);
  else e = make_tmap(&ta, h, !bf16, F, R, 0, kBM);
  if (e != cudaSuccess) return e;
  GemmArgs a = base_args(L);
  a.group_off = expert_off;
  a.num_groups = E;
  a.m_total = static_cast<int>(R);
  a.n_out = D;
  a.k_dim = F;
  a.bias0 = w.b_down;
  a.out = out;
  a.ldo = D;
  a.slot_of_row = slot_of_row;
  a.topk_w = topk_w;
  a.h_halves = h_halves;
  if (gemm_kind(R, E, true) == GK_DECODE) {
    CUtensorMap wd, th;
    if ((e = make_tmap(&wd, w.w_down, false, F, D, E, 128)) != cudaSuccess) return e;
    if (hsplit) e = make_tmap_halves(&th, h, F, R, kDecTok);
    else e = make_tmap(&th, h, false, F, R, 0, kDecTok);
    if (e != cudaSuccess) return e;
    const int64_t units = (std::min<int64_t>(E, R) + R / kDecTok) * ((D + 127) / 128);
    if (slot_of_row != nullptr) {
      // the split needs a K stage (kDecKBS 64-wide K blocks) in each half: with a single
      // stage the second half would be empty and add an accumulator that no MMA wrote
      constexpr int kStageK = 64 * kDecKBS;
      if (units <= L.num_sms && (F + kStageK - 1) / kStageK >= 2) {
        // fewer units than SMs (T = 1: 4 experts x 23 feature blocks): split K in two,
        // each half adding its weighted partial into the zeroed fp32 rows
        const int64_t n = R * static_cast<int64_t>(D);
        pdl_launch(zero_f32_kernel, dim3(static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 4 * L.num_sms))),
                   dim3(256), 0, L.stream, static_cast<float*>(out), n);
        count_launch();
        a.k_splits = 2;
        return launch_decode<EPI_BIAS_WSCATTER>(L, wd, wd, th, a, 2 * units);
      }
      return launch_decode<EPI_BIAS_WSCATTER>(L, wd, wd, th, a, units);
    }
    return launch_decode<EPI_BIAS>(L, wd, wd, th, a, units);
  }
  if (gemm_kind(R, E, true) == GK_WM_PAIR) {
    CUtensorMap wd, th16;
    if ((e = make_tmap(&wd, w.w_down, false, F, D, E, 128)) != cudaSuccess) return e;
    if ((e = make_tmap(&th16, h, false, F, R, 0, 16)) != cudaSuccess) return e;
    const int64_t units = ((R + kWmTok - 1) / kWmTok + E) * ((D + 255) / 256);
    if (slot_of_row != nullptr) return launch_wm_pair<EPI_BIAS_WSCATTER>(L, wd, wd, ta, th16, a, units);
    return launch_wm_pair<EPI_BIAS>(L, wd, wd, ta, th16, a, units);
  }
  const bool pair = use_pair(R, E, true);
  if ((e = make_tmap(&tb, w.w_down, !bf16, F, D, E, pair ? kTNHalf : kTNDown)) != cudaSuccess) return e;
  if (pair) {
    const int64_t ptiles = ((R + kPairBM - 1) / kPairBM + E) * ((D + 2 * kTNHalf - 1) / (2 * kTNHalf));
    if (slot_of_row != nullptr)
      return launch_pair<kTNHalf, EPI_BIAS_WSCATTER, kPairStages>(L, ta, tb, tb, a, ptiles);
    return launch_pair<kTNHalf, EPI_BIAS, kPairStages>(L, ta, tb, tb, a, ptiles);
  }
  const int64_t tiles = max_row_blocks(R, E) * ((D + kTNDown - 1) / kTNDown);
  if (slot_of_row != nullptr)
    return launch<__nv_bfloat16, kTNDown, 1, EPI_BIAS_WSCATTER, kStages>(L, ta, tb, tb, a, tiles);
  return launch<__nv_bfloat16, kTNDown, 1, EPI_BIAS, kStages>(L, ta, tb, tb, a, tiles);
}


// ---------------------------------------------------------------------------
// MXFP4 weights with MXFP8 activations on the block-scaled tensor cores
// ---------------------------------------------------------------------------
// E4M3 rows [rows, K] bytes; boxes of 128 rows x 128 B, 128-byte swizzle.
static cudaError_t make_tmap_e4m3(CUtensorMap* m, const void* ptr, uint64_t K, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kMx8BK), static_cast<cuuint32_t>(kBM)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Packed E2M1 weights [G, N, K/2] bytes as they are; boxes of 64 B (128 codes) x box_rows,
// no swizzle (the converter warps widen them into the swizzled tile).
static cudaError_t make_tmap_e2m1(CUtensorMap* m, const void* ptr, uint64_t K, uint64_t N, uint64_t G,
                                  uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {K / 2, N, G};
  const cuuint64_t strides[2] = {K / 2, (K / 2) * N};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kMx8BK / 2), box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The same weights through TMA's 4-bit unpacking type: each 16 codes land in 16 bytes of
// shared memory (the upper 8 unused), 128-byte swizzle -- the tile the f8f6f4 MMA reads.
// The type describes rows in whole 128-code blocks: dims {K rounded down to 128, N, G};
// boxes of 128 codes x box_rows.  Its strides and base need 32-byte alignment.
// (Expert-GEMM variant 7 turns the unpacking off: every stage is widened by the converters.)
static bool e2m1_unpack_ok(const void* ptr, uint64_t K) {
  return g_gemm_variant.load() != 7 && K >= 128 && (K / 2) % 32 == 0 && (reinterpret_cast<uintptr_t>(ptr) & 31u) == 0;
}
static cudaError_t make_tmap_e2m1_unpack(CUtensorMap* m, const void* ptr, uint64_t K, uint64_t N, uint64_t G,
                                         uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {K / kMx8BK * kMx8BK, N, G};
  const cuuint64_t strides[2] = {K / 2, (K / 2) * N};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kMx8BK), box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int EPI, int TN, int NB, int STAGES>
static cudaError_t launch_mx8(const Launch& L, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                              const CUtensorMap& u0, const CUtensorMap& u1, const Mx8Args& args, int64_t max_tiles) {
  if (max_tiles <= 0) return cudaSuccess;
  auto kern = grouped_gemm_mx8_kernel<EPI, TN, NB, STAGES>;
  constexpr int smem = Mx8Layout<TN, NB>::smem_bytes(STAGES);
  static_assert(smem <= 232448, "shared memory budget");
  int dev = 0;
  cudaGetDevice(&dev);
  static std::mutex mu;
  static uint64_t configured = 0;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev >= 64 || !((configured >> dev) & 1u)) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      if (dev < 64) configured |= uint64_t(1) << dev;
    }
  }
  const int grid = static_cast<int>(std::min<int64_t>(max_tiles, L.num_sms));
  pdl_launch(kern, dim3(grid), dim3(kMx8Threads), smem, L.stream, a, b0, b1, u0, u1, args);
  count_launch();
  return cudaGetLastError();
}

int mx8_sf_bytes_per_row(int K) { return mx8_sf_stride(K); }

cudaError_t mx8_quant_rows(const Launch& L, int64_t T, int K, const void* x, uint8_t* xq, uint8_t* sf) {
  if (T == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<int64_t>((T + 7) / 8, int64_t(L.num_sms) * 8));
  pdl_launch(mx8_quant_rows_kernel, dim3(blocks), dim3(256), 0, L.stream, static_cast<const __nv_bfloat16*>(x),
             static_cast<int>(T), K, mx8_sf_stride(K), xq, sf);
  count_launch();
  return cudaGetLastError();
}

cudaError_t mx8_weight_scales(const Launch& L, int D, int F, int E, const ExpertWeights& w, uint8_t* sf_gate,
                              uint8_t* sf_up, uint8_t* sf_down) {
  Mx8SfJob job{};
  job.src[0] = w.s_gate; job.dst[0] = sf_gate; job.rows[0] = E * F; job.nblk[0] = D / 32; job.sfs[0] = mx8_sf_stride(D);
  job.src[1] = w.s_up;   job.dst[1] = sf_up;   job.rows[1] = E * F; job.nblk[1] = D / 32; job.sfs[1] = mx8_sf_stride(D);
  job.src[2] = w.s_down; job.dst[2] = sf_down; job.rows[2] = E * D; job.nblk[2] = F / 32; job.sfs[2] = mx8_sf_stride(F);
  const int64_t most = std::max(int64_t(E) * F * job.sfs[0], int64_t(E) * D * job.sfs[2]) / 16;   // chunks
  const dim3 grid(static_cast<unsigned>(std::min<int64_t>((most + 255) / 256, int64_t(8) * L.num_sms)), 3);
  pdl_launch(mx8_weight_sf_kernel, grid, dim3(256), 0, L.stream, job);
  count_launch();
  return cudaGetLastError();
}

cudaError_t expert_gateup_mx8(const Launch& L, int64_t R, int D, int F, int E, const uint8_t* xq,
                              const uint8_t* sfx, const int32_t* expert_off, const ExpertWeights& w,
                              const uint8_t* sf_gate, const uint8_t* sf_up, float limit, float alpha, uint8_t* hq,
                              uint8_t* sfh) {
  if (R == 0) return cudaSuccess;
  CUtensorMap ta, tg, tu;
  cudaError_t e;
  if ((e = make_tmap_e4m3(&ta, xq, D, R)) != cudaSuccess) return e;
  if ((e = make_tmap_e2m1(&tg, w.w_gate, D, F, E, kMx8TNGateUp)) != cudaSuccess) return e;
  if ((e = make_tmap_e2m1(&tu, w.w_up, D, F, E, kMx8TNGateUp)) != cudaSuccess) return e;
  Mx8Args a{};
  a.group_off = expert_off;
  a.num_groups = E;
  a.m_total = static_cast<int>(R);
  a.n_out = F;
  a.k_dim = D;
  a.sfa = sfx;
  a.sfs_a = mx8_sf_stride(D);
  a.sfw0 = sf_gate;
  a.sfw1 = sf_up;
  a.bias0 = w.b_gate;
  a.bias1 = w.b_up;
  a.limit = limit;
  a.alpha = alpha;
  a.gate_lo = 0.0f;
  a.hq = hq;
  a.sfh = sfh;
  a.sfs_h = mx8_sf_stride(F);
  a.wait_limit_ns = L.wait_limit_ns;
  CUtensorMap ug = tg, uu = tu;
  if (e2m1_unpack_ok(w.w_gate, D) && e2m1_unpack_ok(w.w_up, D)) {
    if ((e = make_tmap_e2m1_unpack(&ug, w.w_gate, D, F, E, kMx8TNGateUp)) != cudaSuccess) return e;
    if ((e = make_tmap_e2m1_unpack(&uu, w.w_up, D, F, E, kMx8TNGateUp)) != cudaSuccess) return e;
    a.kb_unpacked = D / kMx8BK;
  }
  const int64_t tiles = max_row_blocks(R, E) * ((F + kMx8TNGateUp - 1) / kMx8TNGateUp);
  return launch_mx8<EPI_SWIGLU, kMx8TNGateUp, 2, kMx8StagesGateUp>(L, ta, tg, tu, ug, uu, a, tiles);
}

cudaError_t expert_down_mx8(const Launch& L, int64_t R, int D, int F, int E, const uint8_t* hq, const uint8_t* sfh,
                            const int32_t* expert_off, const ExpertWeights& w, const uint8_t* sf_down,
                            const int32_t* slot_of_row, const float* topk_w, float* ys) {
  if (R == 0) return cudaSuccess;
  CUtensorMap ta, td;
  cudaError_t e;
  if ((e = make_tmap_e4m3(&ta, hq, F, R)) != cudaSuccess) return e;
  if ((e = make_tmap_e2m1(&td, w.w_down, F, D, E, kMx8TNDown)) != cudaSuccess) return e;
  Mx8Args a{};
  a.group_off = expert_off;
  a.num_groups = E;
  a.m_total = static_cast<int>(R);
  a.n_out = D;
  a.k_dim = F;
  a.sfa = sfh;
  a.sfs_a = mx8_sf_stride(F);
  a.sfw0 = sf_down;
  a.sfw1 = sf_down;
  a.bias0 = w.b_down;
  a.out = ys;
  a.slot_of_row = slot_of_row;
  a.topk_w = topk_w;
  a.wait_limit_ns = L.wait_limit_ns;
  CUtensorMap ud = td;
  if (e2m1_unpack_ok(w.w_down, F)) {
    if ((e = make_tmap_e2m1_unpack(&ud, w.w_down, F, D, E, kMx8TNDown)) != cudaSuccess) return e;
    a.kb_unpacked = F / kMx8BK;
  }
  const int64_t tiles = max_row_blocks(R, E) * ((D + kMx8TNDown - 1) / kMx8TNDown);
  return launch_mx8<EPI_BIAS_WSCATTER, kMx8TNDown, 1, kMx8StagesDown>(L, ta, td, td, ud, ud, a, tiles);
}

// x_perm-style row gather of byte rows (row_bytes a multiple of 16): dst[r] = src[slot_of_row[r] / k].
cudaError_t gather_rows(const Launch& L, const void* src, const int32_t* slot_of_row, int64_t R, int k, int64_t T,
                        int row_bytes, void* dst) {
  if (R == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<int64_t>((R + 7) / 8, int64_t(L.num_sms) * 8));
  pdl_launch(permute_gather_kernel, dim3(blocks), dim3(256), 0, L.stream, static_cast<const uint4*>(src), slot_of_row,
             static_cast<int>(R), k, static_cast<int>(T), row_bytes / 16, static_cast<uint4*>(dst));
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// the decode layer (decode_layer.cuh): router logits, then one persistent kernel
// ---------------------------------------------------------------------------
// Shapes it serves: bf16, at most kDlMaxRows routed rows and experts averaging at
// most 16 of them (the weight-streaming regime), E <= 256 and k <= 8 (the warp top-k).
bool decode_layer_shape(bool bf16, int64_t T, int k, int E, int D, int F) {
  const int64_t R = T * k;
  return bf16 && R >= 1 && R <= kDlMaxRows && R <= int64_t(16) * E && E <= kDlMaxExperts && k <= 8 &&
         D % 8 == 0 && F % 8 == 0 && D / 8 <= kRouterMaxChunks;
}

size_t decode_layer_counter_words(int64_t T, int k, int E, int D, int F) {
  return static_cast<size_t>(dl_counters(T, k, E, D, F).total);
}

size_t decode_layer_part_bytes() { return kDlPartFloats * sizeof(float); }

// Variant 5 takes it for every shape it serves.  By size (variant 0) it is taken from two
// tokens up to one routed row per expert on average: measured on the GPT-OSS-20B layer
// (graph replay, 4 rotated weight copies) it beats the separate kernels at T = 2, 4, 8
// (93 / 138 / 188 us against 100 / 159 / 201 us), ties at T = 16 and loses at T = 1 and
// T >= 12, where its fixed hand-off latencies (dispatch, the gate/up -> down wait, the last
// partial sums and the combine) weigh more than its balanced weight stream gains.
bool decode_layer_selected(bool bf16, int64_t T, int k, int E, int D, int F) {
  const int v = g_gemm_variant.load();
  if (v == 5) return decode_layer_shape(bf16, T, k, E, D, F);
  return v == 0 && T >= 2 && T * k <= E && decode_layer_shape(bf16, T, k, E, D, F);
}

cudaError_t decode_layer(const Launch& L, int64_t T, int D, int F, int E, int k, const void* x, const void* w_router,
                         const void* b_router, const ExpertWeights& w, float limit, float alpha, float gate_lo,
                         int h_halves, bool out_f32, void* y, int32_t* ids_out, float* w_out, float* logits, int* cnt,
                         float* part, void* h, float* ys) {
  if (T == 0) return cudaSuccess;
  CUtensorMap wg, wu, wd;
  cudaError_t e;
  if ((e = make_tmap(&wg, w.w_gate, false, D, F, E, 64)) != cudaSuccess) return e;
  if ((e = make_tmap(&wu, w.w_up, false, D, F, E, 64)) != cudaSuccess) return e;
  if ((e = make_tmap(&wd, w.w_down, false, F, D, E, 64)) != cudaSuccess) return e;
  const DlCounters dc = dl_counters(T, k, E, D, F);
  const int rblocks = static_cast<int>(T) * ((E + 7) / 8);
  const int rgrid = std::max(1, std::min(rblocks, 4 * L.num_sms));
  pdl_launch(decode_router_kernel, dim3(rgrid), dim3(256), 0, L.stream, static_cast<const __nv_bfloat16*>(x),
             static_cast<const __nv_bfloat16*>(w_router), static_cast<const __nv_bfloat16*>(b_router),
             static_cast<int>(T), D, E, logits, cnt, dc.total);
  count_launch();
  DecLayerArgs a{};
  a.logits = logits;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.h = static_cast<__nv_bfloat16*>(h);
  a.ys = ys;
  a.y = y;
  a.ids_out = ids_out;
  a.w_out = w_out;
  a.b_gate = static_cast<const __nv_bfloat16*>(w.b_gate);
  a.b_up = static_cast<const __nv_bfloat16*>(w.b_up);
  a.b_down = static_cast<const __nv_bfloat16*>(w.b_down);
  a.part = part;
  a.cnt = cnt;
  a.off_done = dc.off_done;
  a.off_gu = dc.off_gu;
  a.off_dn = dc.off_dn;
  a.off_cb = dc.off_cb;
  a.T = static_cast<int>(T);
  a.k = k;
  a.E = E;
  a.D = D;
  a.F = F;
  a.h_halves = h_halves;
  a.out_f32 = out_f32 ? 1 : 0;
  a.limit = limit;
  a.alpha = alpha;
  a.gate_lo = gate_lo;
  a.wait_limit_ns = L.wait_limit_ns;
  constexpr int smem = DlLayout::smem_bytes;
  int dev = 0;
  cudaGetDevice(&dev);
  static std::mutex mu;
  static uint64_t configured = 0;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev >= 64 || !((configured >> dev) & 1u)) {
      e = cudaFuncSetAttribute(decode_layer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      if (dev < 64) configured |= uint64_t(1) << dev;
    }
  }
  const int grid = std::min(L.num_sms, kDlMaxCtas);
  pdl_launch(decode_layer_kernel, dim3(grid), dim3(kDlThreads), smem, L.stream, wg, wu, wd, a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe
