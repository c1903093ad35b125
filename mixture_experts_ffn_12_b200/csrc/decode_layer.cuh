// The MoE layer for a few tokens (decode) in two kernels: the router logits, then
// one persistent kernel for everything after them.
//
// With a handful of tokens the layer is a stream of the touched experts' weights
// (GPT-OSS-20B at T = 1: 4 experts x 3 x 2880 x 2880 bf16 = 199 MB).  As separate
// kernels (router, dispatch, gate/up, down, combine) the GPU idles between launches
// and each GEMM's short unit list runs in uneven waves.  Here one CTA per SM does:
//   0  top-k and softmax of the router logits (the router kernels' own arithmetic)
//      and the stable permutation by expert, built in shared memory by every CTA
//      from the logits, so no CTA waits for another to know the work;
//   A  gate/up + clipped SwiGLU ("Ollama Imagegen GPT OSS", Description) -> h;
//   B  down + bias + routing weight -> the fp32 row of each (token, slot);
//   C  the k-way combine of a token's rows ("Ollama glm4_moe_lite.go",
//      MoE.Forward), by the CTA that completes the last of them.
// A and B are split "stream-K": each phase's (unit, 64-wide K block) steps are cut
// into equal contiguous ranges, one per CTA, so every SM streams the same number
// of weight bytes whatever the unit count.  A unit cut between CTAs leaves fp32
// partial accumulators in global memory; the CTA whose piece completes the unit's
// count adds the pieces in CTA order (the same order whichever finishes last, so
// results are reproducible) and runs the epilogue.
// A stage's weight tile comes by TMA; its token rows (x rows of the unit's tokens in
// A, h rows in B) are copied by a gather warp with cp.async, so the dispatch needs
// no x_perm copy in global memory.  A down tile of expert e needs all of e's h: the
// gather warp waits (bounded) for the count of e's finished gate/up units, while the
// weight tiles of the next few stages are already on their way.
//
// Units and MMA shapes are those of decode_gemm.cuh: the weights are the MMA's
// M = 128 rows (gate/up: 64 gate rows over the same features' 64 up rows; down:
// 128 output features), up to kDlTok of an expert's rows are its N.
#pragma once

#include "decode_gemm.cuh"
#include "router_permute_combine.cuh"

namespace moe {

constexpr int kDlTok = 32;           // an expert's rows per unit (MMA N)
constexpr int kDlStages = 10;        // ring depth (one CTA per SM)
constexpr int kDlMaxRows = 512;      // T * k at most
constexpr int kDlMaxExperts = 256;
constexpr int kDlMaxCtas = 160;      // grid = min(SMs, this); sizes the partial buffers
constexpr int kDlThreads = 224;     // producer, MMA, 4 epilogue warps, gather warp
constexpr int kDlWarps = kDlThreads / 32;
constexpr int kDlGatherLag = 6;    // stages between a token copy's issue and the wait for it
// weight tiles issued ahead of the token copies: a deeper burst while the gather warp waits
// for h queues the hand-off's own small messages (counters, partial sums) behind it
constexpr int kDlHoldAhead = 2;

struct DlLayout {
  static constexpr int W_BYTES = 128 * kRowBytes;      // 16 KB of weight rows per K block
  static constexpr int X_BYTES = kDlTok * kRowBytes;   // 4 KB of token rows (x or h)
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;
  static constexpr int RING = kDlStages * STAGE_BYTES;
  static constexpr int UP_LD = kDlTok + 1;             // row stride of the up values (no bank conflicts)
  static constexpr int UP = 64 * UP_LD * 4;            // up values handed to the gate rows
  // slot_of_row, routing weights; expert row offsets and unit offsets of both phases;
  // combine flags; the epilogue warps' votes
  static constexpr int MAPS = ((2 * kDlMaxRows + 3 * (kDlMaxExperts + 1) + kDlTok + 8) * 4 + 15) / 16 * 16;
  // phase-0 scratch at the start of the ring (free until the first TMA load): expert id
  // per slot, rows per expert, per 32-slot chunk the rows of each expert before it
  static constexpr int SCRATCH = (kDlMaxRows + kDlMaxExperts) * 4 + (kDlMaxRows / 32) * kDlMaxExperts * 2;
  static_assert(SCRATCH <= RING, "phase-0 scratch fits the ring");
  static constexpr int BARS = (3 * kDlStages + 5) * 8 + 32;   // + 6 ints of flags
  static constexpr int smem_bytes = 1024 + RING + UP + MAPS + BARS;
  static_assert(smem_bytes <= 232448, "shared memory budget");
  static_assert((RING + UP + MAPS) % 16 == 0, "the mbarriers that follow the maps are 8-byte aligned");
};

// fp32 partial accumulators: [phase][CTA][first or last unit of the CTA's range][column][row]
constexpr size_t kDlPartFloats = size_t(2) * kDlMaxCtas * 2 * kDlTok * 128;

struct DecLayerArgs {
  const float* logits;            // [T, E] router logits incl. bias
  const __nv_bfloat16* x;         // [T, D]
  __nv_bfloat16* h;               // [R, h_halves * F]
  float* ys;                      // [R, D] weighted down rows, in slot order
  void* y;                        // [T, D] bf16 or fp32
  int32_t* ids_out;               // [T, k] or null
  float* w_out;                   // [T, k] or null
  const __nv_bfloat16* b_gate;    // [E, F]
  const __nv_bfloat16* b_up;      // [E, F]
  const __nv_bfloat16* b_down;    // [E, D]
  float* part;                    // kDlPartFloats
  int* cnt;                       // counters, zero at entry (the router kernel clears them)
  int off_done, off_gu, off_dn, off_cb;
  int T, k, E, D, F;
  int h_halves, out_f32;
  float limit, alpha, gate_lo;
  uint64_t wait_limit_ns;
};

// counters: [0] unused; [off_done + e] finished gate/up
// units of expert e; [off_gu + u], [off_dn + u] finished pieces of a split unit;
// [off_cb + t * DB + db] finished down units of token t's column block db
struct DlCounters {
  int off_done, off_gu, off_dn, off_cb, total;
};
inline DlCounters dl_counters(int64_t T, int k, int E, int D, int F) {
  const int64_t R = T * k;
  const int64_t chunks = std::min<int64_t>(E, R) + R / kDlTok;   // >= sum over experts of ceil(rows / kDlTok)
  DlCounters c{};
  c.off_done = 1;
  c.off_gu = c.off_done + E;
  c.off_dn = c.off_gu + static_cast<int>(chunks * ((F + 63) / 64));
  c.off_cb = c.off_dn + static_cast<int>(chunks * ((D + 127) / 128));
  c.total = c.off_cb + static_cast<int>(T * ((D + 127) / 128));
  return c;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_relaxed_gpu(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ void red_release_gpu_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int atom_acq_rel_gpu_add(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
// orders this thread's generic-proxy global accesses with async-proxy (TMA) ones
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// 16-byte global -> shared copy; src_bytes 0 writes zeros and reads nothing
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// the four epilogue warps
__device__ __forceinline__ void dl_epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// stream-K: CTA c of C owns steps [N c / C, N (c + 1) / C); step i belongs to the
// largest c whose range starts at or before it
__device__ __forceinline__ int64_t sk_begin(int64_t N, int C, int c) { return N * c / C; }
__device__ __forceinline__ int sk_owner(int64_t N, int C, int64_t i) { return static_cast<int>(((i + 1) * C - 1) / N); }

// Router logits of the decode layer: l[t, e] = x[t] . Wr[e] + br[e], with x[t] staged in
// shared memory and a warp per expert, as in the SIMT router (same arithmetic, so the same
// routing); a CTA per (token, 8 experts).  The grid also clears the decode layer's counters.
__global__ void __launch_bounds__(256) decode_router_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const __nv_bfloat16* __restrict__ wr,
                                                            const __nv_bfloat16* __restrict__ br, int T, int D, int E,
                                                            float* __restrict__ logits, int* __restrict__ cnt,
                                                            int ncnt) {
  pdl_enter();
  __shared__ uint4 xs[kRouterMaxChunks];
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < ncnt; i += gridDim.x * blockDim.x) cnt[i] = 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int EB = (E + 7) / 8;
  const int nchunk = D / 8;
  for (int blk = blockIdx.x; blk < T * EB; blk += gridDim.x) {
    const int t = blk / EB, e = (blk - t * EB) * 8 + warp;
    __syncthreads();
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * D);
    for (int c = threadIdx.x; c < nchunk; c += blockDim.x) xs[c] = xr[c];
    __syncthreads();
    if (e < E) {
      const float l = dot_row16<__nv_bfloat16>(xs, wr + static_cast<size_t>(e) * D, D, lane);
      if (lane == 0) logits[static_cast<size_t>(t) * E + e] = l + __bfloat162float(br[e]);
    }
  }
}

// tmWg / tmWu: W_gate / W_up [E, F, D] (64-row boxes); tmWd: W_down [E, D, F] (64-row boxes,
// two per stage).
__global__ void __launch_bounds__(kDlThreads, 1)
    decode_layer_kernel(const __grid_constant__ CUtensorMap tmWg, const __grid_constant__ CUtensorMap tmWu,
                        const __grid_constant__ CUtensorMap tmWd, const DecLayerArgs a) {
  // let the next kernel be scheduled; the wait for the previous one (the router) comes after
  // the setup below, which reads nothing that kernel writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  using LY = DlLayout;
  constexpr int KSTEPS = kRowBytes / 32;     // 16-wide MMA K steps per stage

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* up_s = reinterpret_cast<float*>(smem + LY::RING);                          // [64][UP_LD]
  int* sor_s = reinterpret_cast<int*>(smem + LY::RING + LY::UP);                     // [kDlMaxRows] per row
  float* w_s = reinterpret_cast<float*>(sor_s + kDlMaxRows);                         // [kDlMaxRows] per slot
  int* off_s = reinterpret_cast<int*>(w_s + kDlMaxRows);                             // [E + 1] rows
  int* uoa_s = off_s + (kDlMaxExperts + 1);                                          // [E + 1] gate/up units
  int* uob_s = uoa_s + (kDlMaxExperts + 1);                                          // [E + 1] down units
  int* last_s = uob_s + (kDlMaxExperts + 1);                                         // [kDlTok]
  int* vote_s = last_s + kDlTok;                                                     // [2][4]
  int* ids_s = reinterpret_cast<int*>(smem);                                         // scratch [kDlMaxRows]
  int* cnt_s = ids_s + kDlMaxRows;                                                   // scratch [kDlMaxExperts]
  uint16_t* chk_s = reinterpret_cast<uint16_t*>(cnt_s + kDlMaxExperts);              // scratch [R / 32][kDlMaxExperts]
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + LY::RING + LY::UP + LY::MAPS);   // weight tile landed
  uint64_t* xfull = wfull + kDlStages;                                               // token rows landed (32 lanes)
  uint64_t* empty = xfull + kDlStages;
  uint64_t* tfull = empty + kDlStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* never_flag = abort_flag + 1;
  int* flag_s = never_flag + 1;
  volatile int* gprog = never_flag + 2;   // stages whose token copies the gather warp has issued
  volatile int* gwait = never_flag + 3;   // the gather warp is waiting for an expert's h

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int T = a.T, k = a.k, E = a.E, D = a.D, F = a.F;
  const int R = T * k;
  const int C = gridDim.x;
  const int cta = blockIdx.x;
  const uint64_t lim = a.wait_limit_ns;
  const unsigned lt = (1u << lane) - 1u;
  if (threadIdx.x == 0) { *gprog = 0; *gwait = 0; }

  // ---------------------------------------------------------------- phase 0
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDlStages; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&xfull[s], 32);
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
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kDecTmemCols);
    tmem_relinquish();
  } else if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmWg);
    tma_prefetch_desc(&tmWu);
    tma_prefetch_desc(&tmWd);
  } else if (warp == kDlWarps - 1) {
    // the x rows are read by this warp's copies: bring their translations and lines in
    const size_t xbytes = static_cast<size_t>(T) * D * 2;
    for (size_t o = static_cast<size_t>(lane) * 4096; o < xbytes; o += 32 * 4096)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(a.x) + o));
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");   // the router's logits and cleared counters
  const int nch = (R + 31) / 32;
  for (int i = threadIdx.x; i < E; i += blockDim.x) cnt_s[i] = 0;
  for (int i = threadIdx.x; i < nch * E; i += blockDim.x) chk_s[(i / E) * kDlMaxExperts + i % E] = 0;
  // top-k and softmax in the arithmetic of the router kernels (the k largest logits, equal
  // logits in expert order, softmax over the k).  Few tokens: a warp per token (each lane
  // holds experts lane, lane + 32, ...); more: a thread per token keeping a running top-8 over
  // the logits in expert order, where a value displaces only a smaller one.
  if (T <= 2 * kDlWarps) {
    for (int t = warp; t < T; t += kDlWarps) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? __ldcg(a.logits + static_cast<size_t>(t) * E + e) : -INFINITY;
      }
      warp_topk_softmax(v, lane, E, k, ids_s + t * k, w_s + t * k);
    }
  } else {
    for (int t = threadIdx.x; t < T; t += blockDim.x)
      thread_topk_softmax(a.logits + static_cast<size_t>(t) * E, E, k, ids_s + t * k, w_s + t * k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (cta == 0) {
    for (int s = threadIdx.x; s < R; s += blockDim.x) {
      if (a.ids_out != nullptr) a.ids_out[s] = ids_s[s];
      if (a.w_out != nullptr) a.w_out[s] = w_s[s];
    }
  }
  // the stable permutation by expert: rows per expert, and per 32-slot chunk the rows of
  // each expert in it (lanes with equal ids counted once, by their leader)
  int bad = 0;
  for (int s = threadIdx.x; s < R; s += blockDim.x) {
    const int e = ids_s[s];
    if (e >= 0 && e < E) atomicAdd(&cnt_s[e], 1);
    else bad = 1;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0 && cta == 0) flag_error(DEVERR_BOUNDS);
  for (int c = warp; c < nch; c += kDlWarps) {
    const int s = c * 32 + lane;
    int e = s < R ? ids_s[s] : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned m = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(m) - 1) chk_s[c * kDlMaxExperts + e] = static_cast<uint16_t>(__popc(m));
  }
  __syncthreads();
  const int FBA = (F + 63) / 64, FBB = (D + 127) / 128;   // feature blocks of a gate/up and a down unit
  if (warp == 0) {
    // exclusive scans over experts (8 consecutive experts per lane): rows, gate/up units, down units
    int c[8], ua[8], ub[8], tc = 0, ta = 0, tb = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      c[i] = e < E ? cnt_s[e] : 0;
      const int ch = (c[i] + kDlTok - 1) / kDlTok;
      ua[i] = ch * FBA;
      ub[i] = ch * FBB;
      tc += c[i];
      ta += ua[i];
      tb += ub[i];
    }
    int ic = tc, ia = ta, ib = tb;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int oc = __shfl_up_sync(0xffffffffu, ic, d);
      const int oa = __shfl_up_sync(0xffffffffu, ia, d);
      const int ob = __shfl_up_sync(0xffffffffu, ib, d);
      if (lane >= d) { ic += oc; ia += oa; ib += ob; }
    }
    int rc = ic - tc, ra = ia - ta, rb = ib - tb;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      if (e < E) { off_s[e] = rc; uoa_s[e] = ra; uob_s[e] = rb; }
      rc += c[i];
      ra += ua[i];
      rb += ub[i];
    }
    if (lane == 31) { off_s[E] = ic; uoa_s[E] = ia; uob_s[E] = ib; }
  } else {
    // per expert: rows of the chunks before each chunk (exclusive prefix over chunks)
    for (int e = threadIdx.x - 32; e < E; e += blockDim.x - 32) {
      int run = 0;
      for (int c = 0; c < nch; ++c) {
        const int v = chk_s[c * kDlMaxExperts + e];
        chk_s[c * kDlMaxExperts + e] = static_cast<uint16_t>(run);
        run += v;
      }
    }
  }
  __syncthreads();
  for (int c = warp; c < nch; c += kDlWarps) {
    const int s = c * 32 + lane;
    int e = s < R ? ids_s[s] : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned m = __match_any_sync(0xffffffffu, e);
    if (e >= 0) sor_s[off_s[e] + chk_s[c * kDlMaxExperts + e] + __popc(m & lt)] = s;
  }
  fence_proxy_async_smem();   // the scratch above is ring memory that TMA and cp.async write next
  __syncthreads();
  // ---------------------------------------------------------------- phases A and B
  const int KSA = (D + 63) / 64;
  const int KB = (F + 63) / 64;
  const bool hsplit = a.h_halves == 2;
  const int KSB = hsplit ? 2 * KB : KB;
  const int64_t NA = static_cast<int64_t>(uoa_s[E]) * KSA;
  const int64_t NB = static_cast<int64_t>(uob_s[E]) * KSB;
  const int64_t a0 = sk_begin(NA, C, cta), a1 = sk_begin(NA, C, cta + 1);
  const int64_t b0 = sk_begin(NB, C, cta), b1 = sk_begin(NB, C, cta + 1);
  const int ldh = hsplit ? 2 * F : F;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (weights)
    if (lane == 0) {
      uint32_t issued = 0, issued_par = 0;
      bool ok = true;
      int q = 0, s = 0;
      uint32_t ph = 0;
      for (int phase = 0; ok && phase < 2; ++phase) {
        const int64_t i0 = phase == 0 ? a0 : b0, i1 = phase == 0 ? a1 : b1;
        const int KS = phase == 0 ? KSA : KSB;
        for (int64_t i = i0; ok && i < i1;) {
          const int u = static_cast<int>(i / KS);
          const int64_t ub = static_cast<int64_t>(u) * KS;
          const int kb_end = static_cast<int>((ub + KS < i1 ? ub + KS : i1) - ub);
          const UnitInfo ui = phase == 0 ? decode_unit(u, uoa_s, off_s, E, FBA, 64, kDlTok)
                                         : decode_unit(u, uob_s, off_s, E, FBB, 128, kDlTok);
          for (int kb = static_cast<int>(i - ub); kb < kb_end; ++kb, ++q) {
            // while the gather warp waits for h, at most kDlHoldAhead stages ahead of its copies
            if (*gwait && q - *gprog >= kDlHoldAhead) {
              const uint64_t tw = global_timer_ns();
              while (*gwait && q - *gprog >= kDlHoldAhead) {
                if (*abort_flag != 0 || lim <= 1 || global_timer_ns() - tw > lim) { ok = false; break; }
                __nanosleep(64);
              }
              if (!ok) break;
            }
            if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) { ok = false; break; }
            mbar_arrive_expect_tx(&wfull[s], LY::W_BYTES);
            uint8_t* sw = smem + s * LY::STAGE_BYTES;
            if (phase == 0) {
              tma_load_3d(sw, &tmWg, &wfull[s], kb * 64, ui.f0, ui.g);
              tma_load_3d(sw + 64 * kRowBytes, &tmWu, &wfull[s], kb * 64, ui.f0, ui.g);
            } else {
              // h_split: blocks [KB, 2 KB) read the lo halves with the same weights
              const int kbl = kb >= KB ? kb - KB : kb;
              tma_load_3d(sw, &tmWd, &wfull[s], kbl * 64, ui.f0, ui.g);
              tma_load_3d(sw + 64 * kRowBytes, &tmWd, &wfull[s], kbl * 64, ui.f0 + 64, ui.g);
            }
            issued |= 1u << s;
            issued_par = (issued_par & ~(1u << s)) | (ph << s);
            if (++s == kDlStages) { s = 0; ph ^= 1u; }
          }
          i = ub + kb_end;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(DEVERR_TIMEOUT);
      }
      for (int st = 0; st < kDlStages; ++st)
        if ((issued >> st) & 1u)
          if (!mbar_wait(&wfull[st], (issued_par >> st) & 1u, never_flag, kDrainLimitNs)) flag_error(DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == kDlWarps - 1) {
    // ------------------------------------------------------------ gather warp (token rows)
    // Lane j copies row j of the stage's 32-row token tile: the x row of the unit's j-th
    // token (A) or h row (B), one 128-byte K block = 8 x 16 B into the 128-byte-swizzled
    // slot; columns past D (or F) read as zeros; rows past the unit's tokens are left as
    // they are (they only feed MMA columns no epilogue reads).  The copies of a stage are
    // waited for kDlGatherLag stages later, then fenced for the tensor core and announced.
    int s = 0, q = 0, arrived = 0;
    uint32_t ph = 0;
    int ready_e = -1;
    bool ok = true;
    auto announce = [&](int upto) {   // stages [arrived, upto): copies complete
      for (; arrived < upto; ++arrived) mbar_arrive(&xfull[arrived % kDlStages]);
    };
    for (int phase = 0; ok && phase < 2; ++phase) {
      const int64_t i0 = phase == 0 ? a0 : b0, i1 = phase == 0 ? a1 : b1;
      const int KS = phase == 0 ? KSA : KSB;
      for (int64_t i = i0; ok && i < i1;) {
        const int u = static_cast<int>(i / KS);
        const int64_t ub = static_cast<int64_t>(u) * KS;
        const int kb_end = static_cast<int>((ub + KS < i1 ? ub + KS : i1) - ub);
        const UnitInfo ui = phase == 0 ? decode_unit(u, uoa_s, off_s, E, FBA, 64, kDlTok)
                                       : decode_unit(u, uob_s, off_s, E, FBB, 128, kDlTok);
        const int ntok = min(kDlTok, ui.m_end - ui.m0);
        if (phase == 1 && ui.g != ready_e) {
          // expert g's h: every gate/up unit of g finished.  Announce what is copied first
          // (the MMA may need it for the gate/up units this wait depends on).
          cp_async_wait<0>();
          fence_proxy_async_smem();
          announce(q);
          const int need = uoa_s[ui.g + 1] - uoa_s[ui.g];
          bool got = true;
          if (lane == 0 && ld_relaxed_gpu(a.cnt + a.off_done + ui.g) < need) {
            *gwait = 1;
            const uint64_t tw = global_timer_ns();
            while (ld_relaxed_gpu(a.cnt + a.off_done + ui.g) < need) {
              if (*abort_flag != 0 || lim <= 1 || global_timer_ns() - tw > lim) { got = false; break; }
              __nanosleep(256);
            }
            *gwait = 0;
          }
          if (lane == 0) fence_acq_rel_gpu();
          if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) { ok = false; break; }
          ready_e = ui.g;
        }
        // the source row of lane j, advanced by one K block per stage
        const __nv_bfloat16* src = nullptr;
        if (lane < ntok) {
          const int r = ui.m0 + lane;
          src = phase == 0 ? a.x + static_cast<size_t>(sor_s[r] / k) * D : a.h + static_cast<size_t>(r) * ldh;
        }
        for (int kb = static_cast<int>(i - ub); kb < kb_end; ++kb, ++q) {
          if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim))) { ok = false; break; }
          if (lane < ntok) {
            const int half = phase == 1 && kb >= KB ? 1 : 0;
            const int col0 = (kb - half * KB) * 64;            // first column of the K block
            const int ncol = phase == 0 ? D : F;
            const __nv_bfloat16* row = src + half * F;
            uint8_t* dst = smem + s * LY::STAGE_BYTES + LY::W_BYTES + lane * kRowBytes;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const bool in = col0 + c * 8 < ncol;
              cp_async16(dst + ((c ^ (lane & 7)) << 4), in ? row + col0 + c * 8 : row, in ? 16u : 0u);
            }
          }
          cp_async_commit();
          if (lane == 0) *gprog = q + 1;
          // the stage kDlGatherLag - 1 before this one is complete: fence it and announce it
          cp_async_wait<kDlGatherLag - 1>();
          fence_proxy_async_smem();
          announce(q + 1 - (kDlGatherLag - 1));
          if (++s == kDlStages) { s = 0; ph ^= 1u; }
        }
        i = ub + kb_end;
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    if (ok) announce(q);
    if (!ok) {
      *abort_flag = 1;
      flag_error(DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc(128, kDlTok, 1u);
      int s = 0, it = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int phase = 0; ok && phase < 2; ++phase) {
        const int64_t i0 = phase == 0 ? a0 : b0, i1 = phase == 0 ? a1 : b1;
        const int KS = phase == 0 ? KSA : KSB;
        for (int64_t i = i0; ok && i < i1; ++it) {
          const int64_t ue = (i / KS + 1) * KS;
          const int n = static_cast<int>((ue < i1 ? ue : i1) - i);
          const int acc = it & 1;
          const uint32_t aph = (it >> 1) & 1;
          if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_flag, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kDlTok);
          for (int j = 0; j < n; ++j) {
            if (!mbar_wait(&wfull[s], ph, abort_flag, lim) || !mbar_wait(&xfull[s], ph, abort_flag, lim)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t w_addr = smem_u32(smem + s * LY::STAGE_BYTES);
            const uint32_t x_addr = w_addr + LY::W_BYTES;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk)
              tc_mma<false>(d_tmem, sw128_kmajor_desc(w_addr + kk * 32), sw128_kmajor_desc(x_addr + kk * 32), idesc,
                            (j != 0 || kk != 0) ? 1u : 0u);
            tc_commit(&empty[s]);
            if (++s == kDlStages) { s = 0; ph ^= 1u; }
          }
          if (!ok) break;
          tc_commit(&tfull[acc]);
          i += n;
        }
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
    // Cross-CTA hand-offs follow one pattern: this CTA's stores, a barrier of the four
    // warps, then one thread's release (or acquire-release) atomic; a reader acquires with
    // its atomic or load, and the barrier after it orders the other threads' reads.
    const int quarter = warp & 3;          // TMEM lanes quarter*32 .. +31 = weight rows
    const int wrow = quarter * 32 + lane;
    const int et = threadIdx.x - 64;       // 0..127 over the four epilogue warps
    int it = 0;
    bool ok = true;
    for (int phase = 0; ok && phase < 2; ++phase) {
      const int64_t i0 = phase == 0 ? a0 : b0, i1 = phase == 0 ? a1 : b1;
      const int KS = phase == 0 ? KSA : KSB;
      const int64_t N = phase == 0 ? NA : NB;
      const int first_u = static_cast<int>(i0 / KS);
      for (int64_t i = i0; i < i1; ++it) {
        const int u = static_cast<int>(i / KS);
        const int64_t ub = static_cast<int64_t>(u) * KS, ue = ub + KS;
        const int64_t pe = ue < i1 ? ue : i1;
        const bool whole = i == ub && pe == ue;
        i = pe;
        const UnitInfo ui = phase == 0 ? decode_unit(u, uoa_s, off_s, E, FBA, 64, kDlTok)
                                       : decode_unit(u, uob_s, off_s, E, FBB, 128, kDlTok);
        const int ntok = min(kDlTok, ui.m_end - ui.m0);
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        // the four warps agree before going on: they meet at named barriers below, which do not time out
        const bool got = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, abort_flag, lim));
        int* vote = vote_s + 4 * (it & 1);
        if (lane == 0) vote[quarter] = got ? 1 : 0;
        dl_epi_bar();
        if (!(vote[0] && vote[1] && vote[2] && vote[3])) { ok = false; break; }
        tc_fence_after();
        const uint32_t tbase =
            tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kDlTok);
        float v[kDlTok];
#pragma unroll
        for (int c = 0; c < kDlTok; c += 8) {
          float t8[8];
          tmem_ld8(tbase + c, t8);
#pragma unroll
          for (int j = 0; j < 8; ++j) v[c + j] = t8[j];
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        if (!whole) {
          // this CTA's piece of a split unit: publish it; the piece that completes the unit sums them all
          const int slot = u == first_u ? 0 : 1;
          float* mine = a.part + ((static_cast<size_t>(phase) * kDlMaxCtas + cta) * 2 + slot) * (kDlTok * 128);
#pragma unroll
          for (int c = 0; c < kDlTok; ++c)
            if (c < ntok) __stcg(mine + c * 128 + wrow, v[c]);
          const int cf = sk_owner(N, C, ub), cl = sk_owner(N, C, ue - 1);
          dl_epi_bar();
          if (et == 0) {
            int pieces = 0;
            for (int cc = cf; cc <= cl; ++cc) pieces += sk_begin(N, C, cc) < sk_begin(N, C, cc + 1) ? 1 : 0;
            const int old = atom_acq_rel_gpu_add(a.cnt + (phase == 0 ? a.off_gu : a.off_dn) + u, 1);
            *flag_s = old == pieces - 1;
          }
          dl_epi_bar();
          if (!*flag_s) continue;
          float sum[kDlTok];
#pragma unroll
          for (int c = 0; c < kDlTok; ++c) sum[c] = 0.0f;
          for (int cc = cf; cc <= cl; ++cc) {
            const int64_t cb = sk_begin(N, C, cc);
            if (cb == sk_begin(N, C, cc + 1)) continue;   // an empty range holds no piece
            if (cc == cta) {
#pragma unroll
              for (int c = 0; c < kDlTok; ++c) sum[c] += v[c];
            } else {
              const int sl = u == static_cast<int>(cb / KS) ? 0 : 1;
              const float* q = a.part + ((static_cast<size_t>(phase) * kDlMaxCtas + cc) * 2 + sl) * (kDlTok * 128);
#pragma unroll
              for (int c = 0; c < kDlTok; ++c)
                if (c < ntok) sum[c] += __ldcg(q + c * 128 + wrow);
            }
          }
#pragma unroll
          for (int c = 0; c < kDlTok; ++c) v[c] = sum[c];
        }
        if (phase == 0) {
          // gate rows (0..63) take the up values of the same features from rows 64..127
          if (wrow >= 64) {
#pragma unroll
            for (int c = 0; c < kDlTok; ++c) up_s[(wrow - 64) * LY::UP_LD + c] = v[c];
          }
          dl_epi_bar();
          if (wrow < 64) {
            const int f = ui.f0 + wrow;
            if (f < F) {
              const float bg = __bfloat162float(a.b_gate[static_cast<size_t>(ui.g) * F + f]);
              const float bu = __bfloat162float(a.b_up[static_cast<size_t>(ui.g) * F + f]);
#pragma unroll
              for (int c = 0; c < kDlTok; ++c) {
                if (c >= ntok) break;
                const float gc = fminf(fmaxf(v[c] + bg, a.gate_lo), a.limit);
                const float uc = fminf(fmaxf(up_s[wrow * LY::UP_LD + c] + bu, -a.limit), a.limit);
                const float hv = __fdividef(gc * uc, 1.0f + __expf(-a.alpha * gc));
                const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
                __nv_bfloat16* dst = a.h + static_cast<size_t>(ui.m0 + c) * ldh + f;
                dst[0] = hi;
                if (hsplit) dst[F] = __float2bfloat16_rn(hv - __bfloat162float(hi));
              }
            }
          }
          dl_epi_bar();
          if (et == 0) red_release_gpu_add(a.cnt + a.off_done + ui.g, 1);
        } else {
          // bias + routing weight -> the slot's fp32 row; then the token's combine if this completes it
          const int d = ui.f0 + wrow;
          if (d < D) {
            const float b = __bfloat162float(a.b_down[static_cast<size_t>(ui.g) * D + d]);
#pragma unroll
            for (int c = 0; c < kDlTok; ++c) {
              if (c >= ntok) break;
              const int slot = sor_s[ui.m0 + c];
              __stcg(a.ys + static_cast<size_t>(slot) * D + d, w_s[slot] * (v[c] + b));
            }
          }
          dl_epi_bar();
          const int db = ui.f0 / 128, DB = (D + 127) / 128;
          if (et < ntok) {
            const int t = sor_s[ui.m0 + et] / k;
            const int old = atom_acq_rel_gpu_add(a.cnt + a.off_cb + t * DB + db, 1);
            last_s[et] = old == k - 1 ? t : -1;
          }
          dl_epi_bar();
          const int dd = ui.f0 + et;
          for (int c = 0; c < ntok; ++c) {
            const int t = last_s[c];
            if (t < 0 || dd >= D) continue;
            float sv = 0.0f;
            for (int j = 0; j < k; ++j) sv += __ldcg(a.ys + (static_cast<size_t>(t) * k + j) * D + dd);
            if (a.out_f32) static_cast<float*>(a.y)[static_cast<size_t>(t) * D + dd] = sv;
            else static_cast<__nv_bfloat16*>(a.y)[static_cast<size_t>(t) * D + dd] = __float2bfloat16_rn(sv);
          }
        }
      }
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
