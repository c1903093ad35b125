// Grouped expert GEMMs for fp32 layers, in plain fp32 FMA (CUDA cores).
//
// fp32 layers are computed "fp32 throughout": the tensor cores' TF32 path
// truncates operands to 10 mantissa bits, which on the tiny fp32 layer left
// a max error of 3e-2 of the output RMS (above the 2e-2 bound), so these layers
// run here instead.  Same problem and epilogues as grouped_gemm.cuh: for each
// expert segment [off[g], off[g+1]) of A, C = A B_g^T, then SwiGLU (two B
// operands) or bias (+ routing weight and un-permutation).
#pragma once

#include "grouped_gemm.cuh"

namespace moe {

constexpr int kSimtBM = 64, kSimtBN = 64, kSimtBK = 16;

template <int EPI>
__global__ void __launch_bounds__(256)
    simt_grouped_gemm_f32(const float* __restrict__ A, const float* __restrict__ B0, const float* __restrict__ B1,
                          const GemmArgs args) {
  pdl_enter();
  constexpr bool kTwo = EPI == EPI_SWIGLU;
  __shared__ float sa[kSimtBK][kSimtBM + 4];
  __shared__ float sb0[kSimtBK][kSimtBN + 4];
  __shared__ float sb1[kTwo ? kSimtBK : 1][kTwo ? kSimtBN + 4 : 1];
  __shared__ int goff[kMaxGroups + 2];
  __shared__ int toff[kMaxGroups + 2];

  const int G = args.num_groups, N = args.n_out, K = args.k_dim;
  // per-group 64-row block prefix (serial: G <= 256 and these layers are small)
  for (int g = threadIdx.x; g <= G; g += blockDim.x) {
    int v = args.group_off[g];
    v = min(max(v, 0), args.m_total);
    goff[g] = v;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    toff[0] = 0;
    for (int g = 0; g < G; ++g) toff[g + 1] = toff[g] + max(0, (goff[g + 1] - goff[g] + kSimtBM - 1) / kSimtBM);
  }
  __syncthreads();
  const int mt = blockIdx.y;
  if (mt >= toff[G]) return;
  int g = 0;
  while (toff[g + 1] <= mt) ++g;
  const int m0 = goff[g] + (mt - toff[g]) * kSimtBM;
  const int m_end = goff[g + 1];
  const int n0 = blockIdx.x * kSimtBN;
  const float* Bg0 = B0 + static_cast<size_t>(g) * N * K;
  const float* Bg1 = kTwo ? B1 + static_cast<size_t>(g) * N * K : nullptr;

  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16 threads, 4 x 4 outputs each
  float acc0[4][4] = {}, acc1[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kSimtBK) {
    for (int i = threadIdx.x; i < kSimtBM * kSimtBK; i += 256) {
      const int r = i / kSimtBK, kk = i % kSimtBK;
      const int row = m0 + r, col = k0 + kk;
      sa[kk][r] = (row < m_end && col < K) ? A[static_cast<size_t>(row) * K + col] : 0.0f;
      const int n = n0 + r;
      sb0[kk][r] = (n < N && col < K) ? Bg0[static_cast<size_t>(n) * K + col] : 0.0f;
      if constexpr (kTwo) sb1[kk][r] = (n < N && col < K) ? Bg1[static_cast<size_t>(n) * K + col] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSimtBK; ++kk) {
      float a[4], b0[4], b1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sa[kk][ty * 4 + i];
        b0[i] = sb0[kk][tx * 4 + i];
        if constexpr (kTwo) b1[i] = sb1[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
          if constexpr (kTwo) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }
  const float* bias0 = static_cast<const float*>(args.bias0) + static_cast<size_t>(g) * N;
  const float* bias1 = kTwo ? static_cast<const float*>(args.bias1) + static_cast<size_t>(g) * N : nullptr;
  float* out = static_cast<float*>(args.out);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = m0 + ty * 4 + i;
    if (row >= m_end) continue;
    size_t orow = static_cast<size_t>(row);
    float wv = 1.0f;
    if constexpr (EPI == EPI_BIAS_WSCATTER) {
      const int s = args.slot_of_row[row];
      if (s < 0 || s >= args.m_total) {
        flag_error(DEVERR_BOUNDS);
        continue;
      }
      orow = static_cast<size_t>(s);
      wv = args.topk_w[s];
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v;
      if constexpr (EPI == EPI_SWIGLU) {
        const float gc = fminf(fmaxf(acc0[i][j] + bias0[n], args.gate_lo), args.limit);
        const float uc = fminf(fmaxf(acc1[i][j] + bias1[n], -args.limit), args.limit);
        v = gc * uc / (1.0f + expf(-args.alpha * gc));
      } else if constexpr (EPI == EPI_BIAS_WSCATTER) {
        v = wv * (acc0[i][j] + bias0[n]);
      } else {
        v = acc0[i][j] + bias0[n];
      }
      out[orow * args.ldo + n] = v;
    }
  }
}

}  // namespace moe
