#pragma once
// The GLM4-MoE-Lite variant of the layer ("Ollama glm4_moe_lite.go": MoEGate.Forward,
// SwitchMLP.Forward, SharedExperts.Forward, MoE.Forward), built from the GPT-OSS
// layer's kernels plus the few below.
//   router:  logits from the tensor-core K-split router (bf16, T >= 256) or from
//            glm_logits_simt_kernel (exact fp32 FMA), then glm_topk_kernel:
//            scores = sigmoid(logits); the experts are chosen by scores +
//            e_score_correction_bias (equal values: lower expert index first); the
//            weights are the chosen experts' uncorrected scores, divided by their sum
//            when k > 1 and norm_topk_prob is set, times routed_scaling_factor.
//   experts: the clipped-SwiGLU expert GEMMs with the gate floor at -inf, no upper
//            clip and alpha = 1, which is SiLU(g) * u, on zero biases (the page's
//            experts have none).
//   shared:  the same GEMMs with one expert that holds all T rows.
//   combine: the k weighted slots of a token plus its shared-expert row.
#include "router_permute_combine.cuh"

namespace moe {

// Router logits of one token per block, one K range: partial[e * Tn + t].
template <typename T>
__global__ void __launch_bounds__(kRouterWarps * 32)
    glm_logits_simt_kernel(const T* __restrict__ x, const T* __restrict__ wr, int D, int E, int Tn,
                           float* __restrict__ partial) {
  pdl_enter();
  __shared__ uint4 xs[kRouterMaxChunks];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * D);
  const int nchunk = D * static_cast<int>(sizeof(T)) / 16;
  const bool staged = nchunk <= kRouterMaxChunks;        // else the row is read from global memory
  if (staged)
    for (int c = threadIdx.x; c < nchunk; c += blockDim.x) xs[c] = xr[c];
  __syncthreads();
  for (int e = warp; e < E; e += kRouterWarps) {
    const float l = dot_row16<T>(staged ? xs : xr, wr + static_cast<size_t>(e) * D, D, lane);
    if (lane == 0) partial[static_cast<size_t>(e) * Tn + t] = l;
  }
}

// Sigmoid scores, choice by corrected score, normalised and scaled weights; one
// thread per token.  partial is [SPLITS][E][Tn] (expert-major, so each expert's
// loads are coalesced across the block's tokens).  The running list keeps the 8
// best (corrected score, score, expert) in order; experts arrive in increasing
// index and only a strictly larger value displaces, so equal values keep the lower
// index first.
template <typename T, int SPLITS>
__global__ void __launch_bounds__(256) glm_topk_kernel(const float* __restrict__ partial, const T* __restrict__ corr,
                                                       int Tn, int E, int k, int norm, float scale,
                                                       int32_t* __restrict__ ids, float* __restrict__ wout) {
  pdl_enter();
  __shared__ float cb[256];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cb[e] = corr != nullptr ? to_f32<T>(corr[e]) : 0.0f;
  __syncthreads();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= Tn) return;
  const size_t plane = static_cast<size_t>(E) * Tn;
  float tv[8], ts[8];
  int tix[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    tv[j] = -INFINITY;
    ts[j] = 0.0f;
    tix[j] = 0x7fffffff;
  }
#pragma unroll 1
  for (int e = 0; e < E; ++e) {
    float l = __ldcg(partial + static_cast<size_t>(e) * Tn + t);
#pragma unroll
    for (int sp = 1; sp < SPLITS; ++sp) l += __ldcg(partial + sp * plane + static_cast<size_t>(e) * Tn + t);
    float cs = 1.0f / (1.0f + expf(-l));
    float cv = cs + cb[e];
    int ci = e;
    if (cv > tv[7]) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const bool gt = cv > tv[q];
        const float tq = tv[q], sq = ts[q];
        const int iq = tix[q];
        tv[q] = gt ? cv : tq;
        ts[q] = gt ? cs : sq;
        tix[q] = gt ? ci : iq;
        cv = gt ? tq : cv;
        cs = gt ? sq : cs;
        ci = gt ? iq : ci;
      }
    }
  }
  float sum = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < k) sum += ts[j];
  const float f = (k > 1 && norm) ? scale / sum : scale;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < k) {
      ids[static_cast<size_t>(t) * k + j] = tix[j];
      wout[static_cast<size_t>(t) * k + j] = ts[j] * f;
    }
}

// The shared expert's one group: rows [0, T).
__global__ void glm_shared_off_kernel(int32_t* __restrict__ off, int32_t* __restrict__ ident,
                                      float* __restrict__ ones, int Tn) {
  pdl_enter();
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    off[0] = 0;
    off[1] = Tn;
  }
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < Tn; i += gridDim.x * blockDim.x) {
    ident[i] = i;
    ones[i] = 1.0f;
  }
}

// y[t] = sum_j ys[t*k + j] (fp32, slot order) + y_shared[t] (fp32; may be null), stored as T.
template <typename T>
__global__ void combine_slots_shared_kernel(const float* __restrict__ ys, const float* __restrict__ y_shared, int Tn,
                                            int k, int D, T* __restrict__ y) {
  pdl_enter();
  const int nv = D / 8;
  const int64_t total = static_cast<int64_t>(Tn) * nv;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / nv);
    const int c = static_cast<int>(i - static_cast<int64_t>(t) * nv) * 8;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k; ++j) {
      float v[8];
      load8<float>(ys + (static_cast<size_t>(t) * k + j) * D + c, v);
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] += v[q];
    }
    if (y_shared != nullptr) {
      float v[8];
      load8<float>(y_shared + static_cast<size_t>(t) * D + c, v);
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] += v[q];
    }
    store8<T>(y + static_cast<size_t>(t) * D + c, acc);
  }
}

// Router + choice + weights of the variant.  partial: router_partial_bytes(T, E) of scratch.
cudaError_t glm_router(const Launch& L, bool bf16, int64_t T, int D, int E, int k, const void* x,
                       const void* w_router, const void* corr, bool norm, float scale, int32_t* ids, float* w,
                       float* partial) {
  if (T == 0) return cudaSuccess;
  const int Ti = static_cast<int>(T);
  const dim3 tgrid(static_cast<unsigned>((Ti + 255) / 256));
  const int kblocks = (D + 63) / 64, per_split = (kblocks + kRouterSplits - 1) / kRouterSplits;
  if (bf16 && T >= 256 && (kRouterSplits - 1) * per_split < kblocks) {
    cudaError_t e = router_tc_partial(L, T, D, E, kRouterSplits, x, w_router, partial);
    if (e != cudaSuccess) return e;
    pdl_launch(glm_topk_kernel<__nv_bfloat16, kRouterSplits>, tgrid, dim3(256), 0, L.stream, partial,
               static_cast<const __nv_bfloat16*>(corr), Ti, E, k, norm ? 1 : 0, scale, ids, w);
    count_launch();
    return cudaGetLastError();
  }
  if (bf16) {
    pdl_launch(glm_logits_simt_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(Ti)), dim3(kRouterWarps * 32), 0,
               L.stream, static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w_router), D, E, Ti,
               partial);
    pdl_launch(glm_topk_kernel<__nv_bfloat16, 1>, tgrid, dim3(256), 0, L.stream, partial,
               static_cast<const __nv_bfloat16*>(corr), Ti, E, k, norm ? 1 : 0, scale, ids, w);
  } else {
    pdl_launch(glm_logits_simt_kernel<float>, dim3(static_cast<unsigned>(Ti)), dim3(kRouterWarps * 32), 0,
               L.stream, static_cast<const float*>(x), static_cast<const float*>(w_router), D, E, Ti, partial);
    pdl_launch(glm_topk_kernel<float, 1>, tgrid, dim3(256), 0, L.stream, partial, static_cast<const float*>(corr),
               Ti, E, k, norm ? 1 : 0, scale, ids, w);
  }
  count_launch(2);
  return cudaGetLastError();
}

// The shared expert as one group of T rows: offsets [0, T), and an identity slot map with
// unit weights so that its down projection writes fp32 rows through the scatter epilogue.
cudaError_t glm_shared_off(const Launch& L, int64_t T, int32_t* off, int32_t* ident, float* ones) {
  const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((T + 255) / 256, int64_t(L.num_sms))));
  pdl_launch(glm_shared_off_kernel, dim3(blocks), dim3(256), 0, L.stream, off, ident, ones, static_cast<int>(T));
  count_launch();
  return cudaGetLastError();
}

cudaError_t combine_slots_shared(const Launch& L, bool out_bf16, int64_t T, int D, int k, const void* ys,
                                 const void* y_shared, void* y) {
  if (T == 0) return cudaSuccess;
  const int64_t items = T * (D / 8);
  const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((items + 255) / 256, int64_t(L.num_sms) * 16)));
  if (out_bf16)
    pdl_launch(combine_slots_shared_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, L.stream,
               static_cast<const float*>(ys), static_cast<const float*>(y_shared), static_cast<int>(T), k, D,
               static_cast<__nv_bfloat16*>(y));
  else
    pdl_launch(combine_slots_shared_kernel<float>, dim3(blocks), dim3(256), 0, L.stream,
               static_cast<const float*>(ys), static_cast<const float*>(y_shared), static_cast<int>(T), k, D,
               static_cast<float*>(y));
  count_launch();
  return cudaGetLastError();
}
}  // namespace moe
