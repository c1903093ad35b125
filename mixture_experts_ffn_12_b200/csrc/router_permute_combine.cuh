#pragma once
// Router (SIMT path), dispatch (histogram -> scan -> stable scatter -> row gather),
// and combine kernels of the GPT-OSS MoE layer.
//
// Router: l[t,e] = x[t] . Wr[e] + br[e] (MaxText GPT-OSS weight map, "MoE Router":
// router kernel + router bias); the k largest logits per token, ties to the lower
// expert index, and the softmax over the selected k.  This SIMT kernel computes
// in exact fp32 FMA (no TF32), so fp32 layers route exactly as their definition;
// bf16 layers with many tokens use the tensor-core router instead.
//
// Dispatch: the permutation is the stable sort of the (token, slot) pairs by
// expert id ("Ollama glm4_moe_lite.go", SwitchMLP.Forward: argsort of the
// flattened ids, rows gathered from order / k).  It is built without a sort and
// without order-dependent atomics: per 256-token chunk, every warp builds one
// 32-bit lane mask per expert (atomicOr is commutative, so the result is
// deterministic); popcounts give the per-chunk histogram; one scan over
// (expert, chunk) gives every chunk's base row; a token's row is its base plus the
// popcount of the lanes before it in its warp and of the warps before it.
//
// Combine: y[t] = sum_j w[t,j] * Y[row(t,j)] in fixed j order
// ("Ollama glm4_moe_lite.go", MoE.Forward: score-weighted sum over the k experts).
#include "common.cuh"
#include "internal.h"

namespace moe {


// ---------------------------------------------------------------------------
// router, SIMT: one block (16 warps) per token
// ---------------------------------------------------------------------------
constexpr int kRouterWarps = 32;   // one block per token: a warp per expert for E <= 32
constexpr int kRouterSplits = 4;   // K ranges of the tensor-core router inside the fused layer
constexpr int kRouterMaxChunks = 1024;   // x row staged in shared memory: D * elem <= 16 KB
constexpr int kTopkExpertsPerThread = 8; // router top-k after the K split: experts scanned per thread

// Dot product of a row of x (staged in shared memory, or in global memory) with a weight row in global
// memory; lanes stride over 16-byte chunks.  The weight loads of a batch are all
// issued before any is used, so a row costs ceil(chunks / (32 * kDotBatch)) memory
// round trips instead of one per chunk a lane handles.
constexpr int kDotBatch = 6;

template <typename T>
__device__ __forceinline__ float dot_row16(const uint4* xs, const T* b, int D, int lane) {
  constexpr int EPC = 16 / sizeof(T);
  const int nchunk = D / EPC;
  const uint4* pb = reinterpret_cast<const uint4*>(b);
  float acc = 0.0f;
  for (int c0 = lane; c0 < nchunk; c0 += 32 * kDotBatch) {
    uint4 wv[kDotBatch];
#pragma unroll
    for (int u = 0; u < kDotBatch; ++u) {
      const int c = c0 + 32 * u;
      wv[u] = c < nchunk ? pb[c] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kDotBatch; ++u) {
      const int c = c0 + 32 * u;
      if (c < nchunk) {
        const uint4 ua = xs[c];
        if constexpr (sizeof(T) == 4) {
          const float* fa = reinterpret_cast<const float*>(&ua);
          const float* fb = reinterpret_cast<const float*>(&wv[u]);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc = fmaf(fa[i], fb[i], acc);
        } else {
          const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&ua);
          const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&wv[u]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 fa = __bfloat1622float2(ha[i]);
            const float2 fb = __bfloat1622float2(hb[i]);
            acc = fmaf(fa.x, fb.x, acc);
            acc = fmaf(fa.y, fb.y, acc);
          }
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// Top-k of the logits one warp holds (lane i holds experts i, i+32, ...; -inf past E)
// and the softmax over the selected ones; lane 0 writes ids[0..k) in descending logit
// order (ties -> lower expert index) and their weights w[0..k).  Clobbers v.
__device__ __forceinline__ void warp_topk_softmax(float (&v)[8], int lane, int E, int k, int32_t* ids, float* w) {
  float sel_v[8];
  int sel_e[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    sel_v[j] = -INFINITY;
    sel_e[j] = -1;
    if (j < k) {
      // lane-local best: larger value, then lower expert index
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < E && (v[i] > bv || (v[i] == bv && e < be))) { bv = v[i]; be = e; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
      }
      sel_v[j] = bv;
      sel_e[j] = be;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (lane + 32 * i == be) v[i] = -INFINITY;
    }
  }
  if (lane == 0) {
    float z = 0.0f, ex[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      ex[j] = j < k ? expf(sel_v[j] - sel_v[0]) : 0.0f;
      z += ex[j];
    }
    const float inv = 1.0f / z;
    for (int j = 0; j < k; ++j) {
      ids[j] = sel_e[j];
      w[j] = ex[j] * inv;
    }
  }
}

// Top-k + softmax of one token by one thread: a running top-8 over the logits in expert
// order, where a value displaces only a smaller one (so equal logits keep the lower expert
// first), then the softmax over the k kept, in warp_topk_softmax's arithmetic (the same
// ids and weights).  lg: the token's E logits (16-byte aligned when E % 4 == 0).
__device__ __forceinline__ void thread_topk_softmax(const float* lg, int E, int k, int32_t* ids, float* w) {
  float tv[8];
  int ti[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    tv[j] = -INFINITY;
    ti[j] = 0x7fffffff;
  }
  for (int e0 = 0; e0 < E; e0 += 32) {
    float v32[32];
    if ((E & 3) == 0) {
#pragma unroll
      for (int u = 0; u < 32; u += 4) {
        float4 f4 = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (e0 + u < E) f4 = __ldcg(reinterpret_cast<const float4*>(lg + e0 + u));
        v32[u] = f4.x;
        v32[u + 1] = f4.y;
        v32[u + 2] = f4.z;
        v32[u + 3] = f4.w;
      }
    } else {
#pragma unroll
      for (int u = 0; u < 32; ++u) v32[u] = e0 + u < E ? __ldcg(lg + e0 + u) : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      float cv = v32[u];
      int ci = e0 + u;
      if (ci >= E || !(cv > tv[7])) continue;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const bool gt = cv > tv[q];
        const float tq = tv[q];
        const int iq = ti[q];
        tv[q] = gt ? cv : tq;
        ti[q] = gt ? ci : iq;
        cv = gt ? tq : cv;
        ci = gt ? iq : ci;
      }
    }
  }
  float z = 0.0f, ex[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    ex[j] = j < k ? expf(tv[j] - tv[0]) : 0.0f;
    z += ex[j];
  }
  const float inv = 1.0f / z;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < k) {
      ids[j] = ti[j];
      w[j] = ex[j] * inv;
    }
}

// Fused-layer router tail: sum of the K-range partial logits (partial[split][e][t])
// + router bias, top-k and the softmax over the k selected.  P threads per token
// (P = power of two >= E / 8), each scanning up to 8 experts: thread (part, t)
// with t fastest in the block, so each expert's loads are coalesced across tokens.
// Each thread keeps a running top-k of its experts in index order (strict '>'
// keeps the lower index first on ties); part 0 merges the P lists through shared
// memory, taking lower parts first on ties, which keeps the global order.
template <typename T, int SPLITS, int P>
__global__ void __launch_bounds__(256) router_topk_partials_kernel(const float* __restrict__ partial,
                                                                   const T* __restrict__ br, int Tn, int E, int k,
                                                                   int32_t* __restrict__ ids,
                                                                   float* __restrict__ wout) {
  pdl_enter();
  constexpr int TPB = 256 / P;                       // tokens per block
  __shared__ float bias[256];
  __shared__ float lv[P][8][TPB];
  __shared__ int li[P][8][TPB];
  for (int e = threadIdx.x; e < E; e += blockDim.x) bias[e] = to_f32<T>(br[e]);
  __syncthreads();
  const int part = threadIdx.x / TPB, tl = threadIdx.x % TPB;
  const int t = blockIdx.x * TPB + tl;
  const bool tv_ok = t < Tn;
  float tv[8];
  int tix[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) { tv[j] = -INFINITY; tix[j] = 0x7fffffff; }
  const size_t plane = static_cast<size_t>(E) * Tn;
  const int e_begin = part * kTopkExpertsPerThread, e_end = min(E, e_begin + kTopkExpertsPerThread);
  if (tv_ok) {
#pragma unroll 1
    for (int e0 = e_begin; e0 < e_end; e0 += 8) {
      float p[8][SPLITS];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int sp = 0; sp < SPLITS; ++sp)
          p[i][sp] = e0 + i < e_end ? __ldcg(partial + sp * plane + static_cast<size_t>(e0 + i) * Tn + t) : 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i;
        if (e >= e_end) break;
        float cv = p[i][0];
#pragma unroll
        for (int sp = 1; sp < SPLITS; ++sp) cv += p[i][sp];
        cv += bias[e];
        int ci = e;
        if (cv > tv[7]) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const bool gt = cv > tv[q];
            const float tq = tv[q];
            const int iq = tix[q];
            tv[q] = gt ? cv : tq;
            tix[q] = gt ? ci : iq;
            cv = gt ? tq : cv;
            ci = gt ? iq : ci;
          }
        }
      }
    }
  }
  if constexpr (P > 1) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      lv[part][j][tl] = tv[j];
      li[part][j][tl] = tix[j];
    }
    __syncthreads();
    if (part != 0) return;
    // merge parts 1..P-1 into part 0's list; a candidate displaces only on '>', and
    // parts come in increasing expert order, so ties keep the lower index first
#pragma unroll 1
    for (int q2 = 1; q2 < P; ++q2) {
#pragma unroll
      for (int j2 = 0; j2 < 8; ++j2) {
        float cv = lv[q2][j2][tl];
        int ci = li[q2][j2][tl];
        if (cv > tv[7]) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const bool gt = cv > tv[q];
            const float tq = tv[q];
            const int iq = tix[q];
            tv[q] = gt ? cv : tq;
            tix[q] = gt ? ci : iq;
            cv = gt ? tq : cv;
            ci = gt ? iq : ci;
          }
        }
      }
    }
  }
  if (!tv_ok) return;
  float z = 0.0f, ex[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    ex[j] = j < k ? expf(tv[j] - tv[0]) : 0.0f;
    z += ex[j];
  }
  const float inv = 1.0f / z;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < k) {
      ids[static_cast<size_t>(t) * k + j] = tix[j];
      wout[static_cast<size_t>(t) * k + j] = ex[j] * inv;
    }
}

template <typename T>
__global__ void __launch_bounds__(kRouterWarps * 32)
    router_simt_kernel(const T* __restrict__ x, const T* __restrict__ wr, const T* __restrict__ br, int D, int E,
                       int k, int32_t* __restrict__ ids, float* __restrict__ wout) {
  pdl_enter();
  __shared__ float logits[256];
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
    if (lane == 0) logits[e] = l + to_f32<T>(br[e]);
  }
  __syncthreads();
  if (warp != 0) return;
  // each lane holds experts lane, lane+32, ... (E <= 256 -> 8 values)
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? logits[e] : -INFINITY;
  }
  warp_topk_softmax(v, lane, E, k, ids + static_cast<size_t>(t) * k, wout + static_cast<size_t>(t) * k);
}

cudaError_t router_tc(const Launch& L, int64_t T, int D, int E, int k, const void* x, const void* w_router,
                      const void* b_router, int32_t* ids, float* w);   // gemm_launch.cuh
cudaError_t router_tc_partial(const Launch& L, int64_t T, int D, int E, int splits, const void* x,
                              const void* w_router, float* partial);    // gemm_launch.cuh

size_t router_partial_bytes(int64_t T, int E) { return static_cast<size_t>(kRouterSplits) * T * E * 4; }

cudaError_t router_topk(const Launch& L, bool bf16, int64_t T, int D, int E, int k, const void* x,
                        const void* w_router, const void* b_router, int32_t* ids, float* w, float* partial) {
  if (T == 0) return cudaSuccess;
  // every K range must hold at least one 64-element k-block
  const int kblocks = (D + 63) / 64, per_split = (kblocks + kRouterSplits - 1) / kRouterSplits;
  if (bf16 && T >= 256 && partial != nullptr && (kRouterSplits - 1) * per_split < kblocks) {
    // K split over kRouterSplits ranges so that more CTAs stream x, then sum + top-k
    cudaError_t e = router_tc_partial(L, T, D, E, kRouterSplits, x, w_router, partial);
    if (e != cudaSuccess) return e;
    const __nv_bfloat16* br = static_cast<const __nv_bfloat16*>(b_router);
    const int Ti = static_cast<int>(T);
    const int parts = (E + kTopkExpertsPerThread - 1) / kTopkExpertsPerThread;
    if (parts <= 1)
      pdl_launch(router_topk_partials_kernel<__nv_bfloat16, kRouterSplits, 1>, dim3((Ti + 255) / 256), dim3(256), 0,
                 L.stream, partial, br, Ti, E, k, ids, w);
    else if (parts <= 2)
      pdl_launch(router_topk_partials_kernel<__nv_bfloat16, kRouterSplits, 2>, dim3((Ti + 127) / 128), dim3(256), 0,
                 L.stream, partial, br, Ti, E, k, ids, w);
    else if (parts <= 4)
      pdl_launch(router_topk_partials_kernel<__nv_bfloat16, kRouterSplits, 4>, dim3((Ti + 63) / 64), dim3(256), 0,
                 L.stream, partial, br, Ti, E, k, ids, w);
    else if (parts <= 8)
      pdl_launch(router_topk_partials_kernel<__nv_bfloat16, kRouterSplits, 8>, dim3((Ti + 31) / 32), dim3(256), 0,
                 L.stream, partial, br, Ti, E, k, ids, w);
    else if (parts <= 16)
      pdl_launch(router_topk_partials_kernel<__nv_bfloat16, kRouterSplits, 16>, dim3((Ti + 15) / 16), dim3(256), 0,
                 L.stream, partial, br, Ti, E, k, ids, w);
    else
      pdl_launch(router_topk_partials_kernel<__nv_bfloat16, kRouterSplits, 32>, dim3((Ti + 7) / 8), dim3(256), 0,
                 L.stream, partial, br, Ti, E, k, ids, w);
    count_launch();
    return cudaGetLastError();
  }
  if (bf16 && T >= 256) return router_tc(L, T, D, E, k, x, w_router, b_router, ids, w);
  const dim3 grid(static_cast<unsigned>(T));
  if (bf16)
    pdl_launch(router_simt_kernel<__nv_bfloat16>, dim3(grid), dim3(kRouterWarps * 32), 0, L.stream, 
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w_router),
        static_cast<const __nv_bfloat16*>(b_router), D, E, k, ids, w);
  else
    pdl_launch(router_simt_kernel<float>, dim3(grid), dim3(kRouterWarps * 32), 0, L.stream, 
        static_cast<const float*>(x), static_cast<const float*>(w_router), static_cast<const float*>(b_router), D,
        E, k, ids, w);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// dispatch
// ---------------------------------------------------------------------------
constexpr int kChunk = 256;   // tokens per chunk = 8 warps x 32 lanes
constexpr int kChunkWarps = kChunk / 32;

size_t permute_scratch_words(int64_t T, int E) {
  const int64_t nchunks = (T + kChunk - 1) / kChunk;
  return static_cast<size_t>(2 * nchunks * E);
}

// Build the per-warp expert lane masks of one chunk.  Returns false (and flags the
// device error word) if an id is out of range or repeated within a token.
__device__ __forceinline__ void build_masks(uint32_t (*mask)[256], const int32_t* __restrict__ ids, int T, int k,
                                            int E) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kChunkWarps * 256; i += blockDim.x) (&mask[0][0])[i] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kChunk + threadIdx.x;
  if (t < T) {
    int prev[8];
    for (int j = 0; j < k; ++j) {
      const int e = ids[static_cast<size_t>(t) * k + j];
      bool bad = e < 0 || e >= E;
      for (int q = 0; q < j && q < 8; ++q) bad |= (prev[q] == e);
      if (j < 8) prev[j] = e;
      if (bad) {
        flag_error(DEVERR_BOUNDS);
        continue;
      }
      atomicOr(&mask[warp][e], 1u << lane);
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kChunk) permute_count_kernel(const int32_t* __restrict__ ids, int T, int k, int E,
                                                               int nchunks, int32_t* __restrict__ chunk_cnt) {
  pdl_enter();
  __shared__ uint32_t mask[kChunkWarps][256];
  build_masks(mask, ids, T, k, E);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kChunkWarps; ++w) c += __popc(mask[w][e]);
    chunk_cnt[static_cast<size_t>(e) * nchunks + blockIdx.x] = c;
  }
}

// Exclusive scan over the expert-major (expert, chunk) counts; one block.
__global__ void __launch_bounds__(1024) permute_scan_kernel(const int32_t* __restrict__ cnt, int n, int E, int nchunks,
                                                            int32_t* __restrict__ base, int32_t* __restrict__ expert_off) {
  pdl_enter();
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int b = min(n, tid * per), e = min(n, b + per);
  int local = 0;
  for (int i = b; i < e; ++i) local += cnt[i];
  int incl = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int v = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, v, d);
      if (lane >= d) v += o;
    }
    if (lane < nw) warp_tot[lane] = v;   // inclusive
  }
  __syncthreads();
  int run = incl - local + (warp > 0 ? warp_tot[warp - 1] : 0);
  for (int i = b; i < e; ++i) {
    base[i] = run;
    run += cnt[i];
  }
  __syncthreads();
  for (int q = tid; q < E; q += blockDim.x) expert_off[q] = base[static_cast<size_t>(q) * nchunks];
  if (tid == blockDim.x - 1) expert_off[E] = warp_tot[(blockDim.x >> 5) - 1];
}

// Chunk c's first row per expert is base[e * nchunks + c] (from permute_scan_kernel), or,
// with base == nullptr (few counts: E * nchunks <= kScatterScanMax), this CTA works it out
// from the chunk counts itself -- the same exclusive scan over the expert-major (expert,
// chunk) order -- and CTA 0 writes expert_off; one kernel boundary fewer in the dispatch.
constexpr int kScatterScanMax = 4096;

__global__ void __launch_bounds__(kChunk) permute_scatter_kernel(const int32_t* __restrict__ ids, int T, int k, int E,
                                                                 int nchunks, const int32_t* __restrict__ base,
                                                                 const int32_t* __restrict__ chunk_cnt,
                                                                 int32_t* __restrict__ expert_off,
                                                                 int32_t* __restrict__ row_of_slot,
                                                                 int32_t* __restrict__ slot_of_row) {
  pdl_enter();
  __shared__ uint32_t mask[kChunkWarps][256];
  __shared__ int base_s[256];
  __shared__ int warp_tot[kChunkWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (base == nullptr) {
    // thread e (< E <= 256): expert e's rows in all chunks and in the chunks before this one
    int tot = 0, pre = 0;
    if (static_cast<int>(threadIdx.x) < E) {
      const int32_t* ce = chunk_cnt + static_cast<size_t>(threadIdx.x) * nchunks;
      for (int c = 0; c < nchunks; ++c) {
        const int v = ce[c];
        tot += v;
        pre += c < static_cast<int>(blockIdx.x) ? v : 0;
      }
    }
    int incl = tot;   // exclusive scan of the totals over the experts
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += o;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    const int ex = before + incl - tot;
    if (static_cast<int>(threadIdx.x) < E) {
      base_s[threadIdx.x] = ex + pre;
      if (blockIdx.x == 0) {
        expert_off[threadIdx.x] = ex;
        if (static_cast<int>(threadIdx.x) == E - 1) expert_off[E] = ex + tot;
      }
    }
    __syncthreads();
  }
  build_masks(mask, ids, T, k, E);
  const int t = blockIdx.x * kChunk + threadIdx.x;
  if (t >= T) return;
  const uint32_t lt = (1u << lane) - 1u;
  const int R = T * k;
  for (int j = 0; j < k; ++j) {
    const int e = ids[static_cast<size_t>(t) * k + j];
    if (e < 0 || e >= E) continue;
    int r = (base != nullptr ? base[static_cast<size_t>(e) * nchunks + blockIdx.x] : base_s[e]) +
            __popc(mask[warp][e] & lt);
    for (int w = 0; w < warp; ++w) r += __popc(mask[w][e]);
    if (r < 0 || r >= R) {
      flag_error(DEVERR_BOUNDS);
      continue;
    }
    row_of_slot[static_cast<size_t>(t) * k + j] = r;
    slot_of_row[r] = t * k + j;
  }
}

// x_perm[r] = x[slot_of_row[r] / k], one warp per row, 16-byte vectors.
__global__ void permute_gather_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ slot_of_row, int R,
                                      int k, int T, int vec_per_row, uint4* __restrict__ x_perm) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int r = gw; r < R; r += nw) {
    const int s = slot_of_row[r];
    const int t = s / k;
    if (s < 0 || t >= T) {
      if (lane == 0) flag_error(DEVERR_BOUNDS);
      continue;
    }
    const uint4* src = x + static_cast<size_t>(t) * vec_per_row;
    uint4* dst = x_perm + static_cast<size_t>(r) * vec_per_row;
    // batches of kGatherBatch independent loads per lane before the stores
    constexpr int kGatherBatch = 12;
    for (int v0 = lane; v0 < vec_per_row; v0 += 32 * kGatherBatch) {
      uint4 buf[kGatherBatch];
#pragma unroll
      for (int u = 0; u < kGatherBatch; ++u) {
        const int v = v0 + 32 * u;
        if (v < vec_per_row) buf[u] = src[v];
      }
#pragma unroll
      for (int u = 0; u < kGatherBatch; ++u) {
        const int v = v0 + 32 * u;
        if (v < vec_per_row) dst[v] = buf[u];
      }
    }
  }
}

// The whole dispatch of at most one chunk (T <= 256) in one CTA: lane masks, the
// per-expert scan, ranks, both index maps, and the row copies (decode sizes).
constexpr int kSmallMaxRows = kChunk * 8;   // T <= 256 tokens, k <= 8
constexpr int kSmallCopyRows = 32;          // above this many rows the copy runs on many CTAs
__global__ void __launch_bounds__(kChunk) permute_small_kernel(const int32_t* __restrict__ ids, int T, int k, int E,
                                                               const uint4* __restrict__ x, int vec_per_row,
                                                               int32_t* __restrict__ expert_off,
                                                               int32_t* __restrict__ row_of_slot,
                                                               int32_t* __restrict__ slot_of_row,
                                                               uint4* __restrict__ x_perm) {
  pdl_enter();
  __shared__ uint32_t mask[kChunkWarps][256];
  __shared__ int base[257];
  __shared__ int sor[kSmallMaxRows];
  build_masks(mask, ids, T, k, E);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    // exclusive scan of the per-expert counts, 8 experts per lane
    int c[8], tot = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      int v = 0;
      if (e < E) {
#pragma unroll
        for (int w = 0; w < kChunkWarps; ++w) v += __popc(mask[w][e]);
      }
      c[i] = v;
      tot += v;
    }
    int incl = tot;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += o;
    }
    int run = incl - tot;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      if (e < E) base[e] = run;
      run += c[i];
    }
    if (lane == 31) base[E] = incl;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += blockDim.x) expert_off[e] = base[e];
  const int R = T * k;
  const int t = threadIdx.x;
  if (t < T) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = ids[t * k + j];
      if (e < 0 || e >= E) continue;
      int r = base[e] + __popc(mask[warp][e] & lt);
      for (int w = 0; w < warp; ++w) r += __popc(mask[w][e]);
      if (r < 0 || r >= R) {
        flag_error(DEVERR_BOUNDS);
        continue;
      }
      row_of_slot[t * k + j] = r;
      slot_of_row[r] = t * k + j;
      sor[r] = t * k + j;
    }
  }
  __syncthreads();
  if (x == nullptr) return;
  // (row, chunk) pairs spread over the block; each thread issues kCopyBatch loads before storing
  constexpr int kCopyBatch = 16;
  const int n = R * vec_per_row;
  for (int i0 = threadIdx.x; i0 < n; i0 += kChunk * kCopyBatch) {
    uint4 v[kCopyBatch];
#pragma unroll
    for (int u = 0; u < kCopyBatch; ++u) {
      const int i = i0 + u * kChunk;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (i < n) {
        const int r = i / vec_per_row;
        const int src = sor[r] / k;
        if (src >= 0 && src < T) v[u] = x[static_cast<size_t>(src) * vec_per_row + (i - r * vec_per_row)];
      }
    }
#pragma unroll
    for (int u = 0; u < kCopyBatch; ++u) {
      const int i = i0 + u * kChunk;
      if (i < n) x_perm[i] = v[u];
    }
  }
}

cudaError_t permute(const Launch& L, bool bf16, int64_t T, int D, int E, int k, const int32_t* ids, const void* x,
                    int32_t* expert_off, int32_t* row_of_slot, int32_t* slot_of_row, void* x_perm,
                    int32_t* scratch) {
  if (T == 0) {
    return cudaMemsetAsync(expert_off, 0, sizeof(int32_t) * (E + 1), L.stream);
  }
  const int nchunks = static_cast<int>((T + kChunk - 1) / kChunk);
  if (nchunks == 1) {
    // one CTA builds the maps; it also copies the rows when there are few of them
    const bool rows = x != nullptr && x_perm != nullptr;
    const bool copy_here = rows && T * k <= kSmallCopyRows;
    pdl_launch(permute_small_kernel, dim3(1), dim3(kChunk), 0, L.stream, ids, static_cast<int>(T), k, E,
                                                     copy_here ? static_cast<const uint4*>(x) : nullptr,
                                                     D * (bf16 ? 2 : 4) / 16, expert_off, row_of_slot, slot_of_row,
                                                     copy_here ? static_cast<uint4*>(x_perm) : nullptr);
    count_launch();
    if (!rows || copy_here) return cudaGetLastError();
  } else {
    int32_t* cnt = scratch;
    int32_t* base = scratch + static_cast<size_t>(nchunks) * E;
    pdl_launch(permute_count_kernel, dim3(nchunks), dim3(kChunk), 0, L.stream, ids, static_cast<int>(T), k, E, nchunks, cnt);
    const bool scan_here = static_cast<int64_t>(E) * nchunks <= kScatterScanMax;
    if (!scan_here) {
      pdl_launch(permute_scan_kernel, dim3(1), dim3(1024), 0, L.stream, cnt, nchunks * E, E, nchunks, base, expert_off);
      count_launch();
    }
    pdl_launch(permute_scatter_kernel, dim3(nchunks), dim3(kChunk), 0, L.stream, ids, static_cast<int>(T), k, E, nchunks,
               scan_here ? static_cast<const int32_t*>(nullptr) : static_cast<const int32_t*>(base),
               static_cast<const int32_t*>(cnt), expert_off, row_of_slot, slot_of_row);
    count_launch(2);
  }
  if (x != nullptr && x_perm != nullptr) {
    const int R = static_cast<int>(T * k);
    const int vpr = D * (bf16 ? 2 : 4) / 16;
    const int warps_needed = R;
    const int blocks = static_cast<int>(std::min<int64_t>((warps_needed + 7) / 8, int64_t(L.num_sms) * 8));
    pdl_launch(permute_gather_kernel, dim3(blocks), dim3(256), 0, L.stream, static_cast<const uint4*>(x), slot_of_row, R, k,
                                                       static_cast<int>(T), vpr, static_cast<uint4*>(x_perm));
    count_launch();
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// combine
// ---------------------------------------------------------------------------
template <typename T, typename TO>
__global__ void combine_gather_kernel(const T* __restrict__ y_perm, const int32_t* __restrict__ row_of_slot,
                                      const float* __restrict__ w, int Tn, int k, int D, TO* __restrict__ y) {
  pdl_enter();
  const int nv = D / 8;
  const int64_t total = static_cast<int64_t>(Tn) * nv;
  const int R = Tn * k;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / nv);
    const int c = static_cast<int>(i - static_cast<int64_t>(t) * nv) * 8;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k; ++j) {
      const int r = row_of_slot[static_cast<size_t>(t) * k + j];
      if (r < 0 || r >= R) {
        flag_error(DEVERR_BOUNDS);
        continue;
      }
      const float wt = w[static_cast<size_t>(t) * k + j];
      float v[8];
      load8<T>(y_perm + static_cast<size_t>(r) * D + c, v);
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = fmaf(wt, v[q], acc[q]);
    }
    store8<TO>(y + static_cast<size_t>(t) * D + c, acc);
  }
}

template <typename T>
__global__ void combine_slots_kernel(const float* __restrict__ ys, int Tn, int k, int D, T* __restrict__ y) {
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
    store8<T>(y + static_cast<size_t>(t) * D + c, acc);
  }
}

static int elementwise_blocks(const Launch& L, int64_t items) {
  const int64_t want = (items + 255) / 256;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, int64_t(L.num_sms) * 16)));
}

cudaError_t combine_gather(const Launch& L, bool bf16, bool out_f32, int64_t T, int D, int k, const void* y_perm,
                           const int32_t* row_of_slot, const float* w, void* y) {
  if (T == 0) return cudaSuccess;
  const int blocks = elementwise_blocks(L, T * (D / 8));
  const int Ti = static_cast<int>(T);
  if (bf16 && !out_f32)
    pdl_launch(combine_gather_kernel<__nv_bfloat16, __nv_bfloat16>, dim3(blocks), dim3(256), 0, L.stream,
               static_cast<const __nv_bfloat16*>(y_perm), row_of_slot, w, Ti, k, D, static_cast<__nv_bfloat16*>(y));
  else if (bf16)
    pdl_launch(combine_gather_kernel<__nv_bfloat16, float>, dim3(blocks), dim3(256), 0, L.stream,
               static_cast<const __nv_bfloat16*>(y_perm), row_of_slot, w, Ti, k, D, static_cast<float*>(y));
  else
    pdl_launch(combine_gather_kernel<float, float>, dim3(blocks), dim3(256), 0, L.stream,
               static_cast<const float*>(y_perm), row_of_slot, w, Ti, k, D, static_cast<float*>(y));
  count_launch();
  return cudaGetLastError();
}

// y in bf16 (out_bf16) or fp32; the fp32 sums are the same either way
cudaError_t combine_slots(const Launch& L, bool out_bf16, int64_t T, int D, int k, const void* ys, void* y) {
  if (T == 0) return cudaSuccess;
  const int blocks = elementwise_blocks(L, T * (D / 8));
  if (out_bf16)
    pdl_launch(combine_slots_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, L.stream,
               static_cast<const float*>(ys), static_cast<int>(T), k, D, static_cast<__nv_bfloat16*>(y));
  else
    pdl_launch(combine_slots_kernel<float>, dim3(blocks), dim3(256), 0, L.stream, static_cast<const float*>(ys),
               static_cast<int>(T), k, D, static_cast<float*>(y));
  count_launch();
  return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(int* bits) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  *bits = v;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
}

}  // namespace moe
