/*
 * moe.h -- C ABI of libmoe: the GPT-OSS Mixture-of-Experts FFN layer on B200 (sm_100a).
 *
 * The layer (per token t, with D = hidden_size, E = num_local_experts,
 * k = num_experts_per_tok, F = intermediate_size, L = swiglu_limit):
 *   l[t,e]  = x[t] . Wr[e] + br[e]                      router kernel + bias
 *             (MaxText GPT-OSS weight map, "MoE Router")
 *   S_t     = the k largest l[t,.], descending, ties -> lower expert index
 *   w[t,j]  = softmax over {l[t,e] : e in S_t}
 *   for e in S_t:
 *     g = x[t] Wg[e]^T + bg[e],  u = x[t] Wu[e]^T + bu[e]   (wi_0 / wi_1 with biases,
 *                                                         MaxText "MOE EXPERTS")
 *     h = clip(g,0,L) * sigmoid(alpha clip(g,0,L)) * clip(u,-L,L), alpha = 1.702
 *         ("Ollama Imagegen GPT OSS", Description: the clipped SwiGLU)
 *     o_e = h Wd[e]^T + bd[e]                            (wo with bias)
 *   y[t]    = sum_j w[t,j] o_{S_t[j]}                    ("Ollama glm4_moe_lite.go", MoE.Forward)
 * The config mirrors the GPT-OSS Config struct (hidden_size, num_local_experts,
 * num_experts_per_tok, swiglu_limit; "Ollama Imagegen GPT OSS", Signature).
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *    16-byte aligned.  The library never allocates or frees device memory and
 *    never synchronises the host on these calls; work is enqueued on `stream`
 *    (a cudaStream_t, NULL = the legacy default stream) of the current device.
 *  - Weights are stored K-major ("[N, K]", the reduction dim contiguous):
 *      w_router [E, D]; w_gate, w_up [E, F, D]; w_down [E, D, F];
 *      b_router [E]; b_gate, b_up [E, F]; b_down [E, D].
 *    Activations, router and dense expert weights, biases and outputs use
 *    `dtype` (fp32 or bf16).  Routing weights are always fp32, ids int32.
 *  - MXFP4 expert weights (wfmt = MOE_W_MXFP4, dtype must be bf16): packed
 *    E2M1 codes [.., N, K/2] uint8 (element 2i = low nibble of byte i, code bit 3
 *    = sign, bits 2..1 = exponent with bias 1, bit 0 = mantissa) and E8M0 scale
 *    bytes [.., N, K/32] (scale 2^(s-127) for 32 consecutive elements along K),
 *    per the OCP Microscaling formats; the pages name the format "MXFP4"
 *    ("GPT-OSS 20B GGUF with MoE CPU Offloading", Model Specifications).
 *  - Kernels are launched with programmatic dependent launch: each of the
 *    library's kernels lets the next kernel on the stream be scheduled early and
 *    itself waits (griddepcontrol.wait) for the preceding kernel's completion and
 *    memory before touching any buffer, so stream order is kept for callers'
 *    kernels and copies before and after a call.
 *  - Arguments are validated before any launch; a rejected call launches
 *    nothing and returns MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED /
 *    MOE_ERR_WORKSPACE.  T = 0 is a successful no-op (expert_off is zeroed
 *    where it is an output).  Launch failures return MOE_ERR_CUDA.
 *  - Faults found on the device (an out-of-range id or row index read from a
 *    caller buffer, a bounded wait that gave up) never trap: the kernels skip
 *    the access or end early and set a per-device error word, which
 *    moe_last_device_error() reads after a synchronisation.  Results of such a
 *    call are unspecified.
 *  - Supported sizes: 1 <= k <= min(E, 8), 1 <= E <= 256, D and F multiples of
 *    16 (of 32 for MXFP4), T >= 0 with T*k < 2^31; swiglu_limit finite and > 0.
 *  - NaN/Inf inputs: unspecified.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 2

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or config field */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but not supported (e.g. MXFP4 with fp32 activations) */
  MOE_ERR_WORKSPACE = 3,    /* workspace pointer null or smaller than the size function says */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  MOE_ERR_TIMEOUT = 5,      /* moe_last_device_error: a kernel's bounded wait gave up */
  MOE_ERR_DEVICE_BOUNDS = 6 /* moe_last_device_error: an index read on the device was out of range */
} moe_status_t;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;
/* MOE_W_MXFP4_A8: the MXFP4 weights of MOE_W_MXFP4, multiplied on the
 * block-scaled tensor cores (tcgen05.mma kind::mxf8f6f4) with the activations of
 * both expert projections (x_perm and h) quantized to MXFP8: E4M3 elements, one
 * E8M0 scale per 32 elements along K, the scale 2^X the smallest power of two
 * with the block's largest magnitude <= 448 * 2^X (no element saturates),
 * elements rounded to nearest, ties to even.  A numerics variant of the layer
 * (the pages name MXFP8 and its group size 32, "Ollama glm4_moe_lite.go",
 * quantizationParams); its results differ from MOE_W_MXFP4 by that
 * quantization.  Same weight layout and sizes as MOE_W_MXFP4;
 * moe_layer_forward only (moe_expert_ffn returns MOE_ERR_UNSUPPORTED). */
typedef enum { MOE_W_DENSE = 0, MOE_W_MXFP4 = 1, MOE_W_MXFP4_A8 = 2 } moe_wfmt_t;

/* Field names follow the GPT-OSS Config (hidden_size, num_local_experts,
 * num_experts_per_tok, swiglu_limit); intermediate_size is F. */
typedef struct {
  int32_t hidden_size;         /* D */
  int32_t intermediate_size;   /* F */
  int32_t num_local_experts;   /* E */
  int32_t num_experts_per_tok; /* k */
  float swiglu_limit;          /* L, e.g. 7.0 */
  float swiglu_alpha;          /* 1.702 for GPT-OSS */
  int32_t dtype;               /* moe_dtype_t */
  int32_t wfmt;                /* moe_wfmt_t */
  int32_t y_f32;               /* 0: the layer output y is stored in dtype; 1: y is stored in fp32,
                                  i.e. the fp32 sums before their rounding to dtype (for a bf16
                                  layer the dtype output is exactly the round-to-nearest-even
                                  of this fp32 output).  Applies to moe_layer_forward,
                                  moe_combine and moe_glm_layer_forward. */
  int32_t h_split;             /* 0: the SwiGLU output h is kept in dtype between the two expert
                                  GEMMs.  1 (bf16 layers with dense weights): h is kept as two
                                  bf16 halves, hi = bf16(h) and lo = bf16(h - hi), and the down
                                  projection sums over both against the same weights (twice its
                                  tensor-core work), so h carries about 16 significant bits
                                  instead of 8.  No effect on fp32 layers; MOE_ERR_UNSUPPORTED
                                  with MXFP4 weights or with expert-GEMM variant 4. */
} moe_config_t;

/* Expert parameters (device pointers).  Dense: w_* in dtype, s_* NULL.
 * MXFP4: w_* packed E2M1 uint8, s_* E8M0 uint8.  Biases always in dtype. */
typedef struct {
  const void* w_gate;     /* [E, F, D]   (MXFP4: [E, F, D/2]) */
  const void* w_up;       /* [E, F, D]   (MXFP4: [E, F, D/2]) */
  const void* w_down;     /* [E, D, F]   (MXFP4: [E, D, F/2]) */
  const uint8_t* s_gate;  /* MXFP4: [E, F, D/32] */
  const uint8_t* s_up;    /* MXFP4: [E, F, D/32] */
  const uint8_t* s_down;  /* MXFP4: [E, D, F/32] */
  const void* b_gate;     /* [E, F] */
  const void* b_up;       /* [E, F] */
  const void* b_down;     /* [E, D] */
} moe_expert_weights_t;

/* ABI version of the loaded library (MOE_ABI_VERSION). */
MOE_API int32_t moe_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
MOE_API const char* moe_status_string(moe_status_t status);

/* Checks a config without touching the GPU: MOE_OK or the reason it is rejected. */
MOE_API moe_status_t moe_config_check(const moe_config_t* cfg);

/* Bytes of workspace moe_permute needs for T tokens (its histogram and scan
 * scratch).  0 when T == 0; (size_t)-1 if cfg is invalid. */
MOE_API size_t moe_permute_workspace_size(const moe_config_t* cfg, int64_t T);

/* Bytes of workspace moe_expert_ffn needs: 0 for dense weights; for MXFP4 the
 * E8M0 scales of the three projections relaid for TMA (per matrix with N rows
 * and reduction length K: E * ceil(K/64) * N * 2 bytes, each region rounded up
 * to 256 bytes), rewritten from the caller's scales on every call.  Independent
 * of T.  (size_t)-1 if cfg is invalid. */
MOE_API size_t moe_expert_ffn_workspace_size(const moe_config_t* cfg, int64_t T);

/* Bytes of workspace moe_layer_forward needs for T tokens: routing ids and
 * weights, dispatch maps, permuted activations x_perm [T*k, D], the SwiGLU
 * output h [T*k, F] ([T*k, 2, F] with h_split), the weighted expert outputs [T*k, D] in fp32 (sharing
 * x_perm's space), plus what the sub-steps need.  (size_t)-1 if cfg is invalid. */
MOE_API size_t moe_workspace_size(const moe_config_t* cfg, int64_t T);

/* Router + top-k + softmax (steps l, S_t, w above).
 *   x [T, D], w_router [E, D], b_router [E] in dtype
 *   -> topk_ids [T, k] int32 (descending logit, ties -> lower index),
 *      topk_w   [T, k] fp32 (softmax over the k selected logits).
 * The logits are accumulated in fp32 (bf16 products are exact in fp32; fp32
 * inputs use fp32 FMA, never TF32). */
MOE_API moe_status_t moe_router_topk(const moe_config_t* cfg, int64_t T, const void* x, const void* w_router,
                             const void* b_router, int32_t* topk_ids, float* topk_w, void* stream);

/* Dispatch: the stable sort of the T*k (token, slot) pairs by expert id
 * ("Ollama glm4_moe_lite.go", SwitchMLP.Forward: argsort of the flattened ids).
 *   topk_ids [T, k] int32 (distinct per token, each in [0, E)),
 *   x [T, D] dtype (may be NULL together with x_perm: index maps only)
 *   -> expert_off  [E+1] int32: rows of expert e are [expert_off[e], expert_off[e+1]),
 *      row_of_slot [T*k] int32: permuted row of pair (t, j) at index t*k+j,
 *      slot_of_row [T*k] int32: t*k+j of the pair held by each permuted row,
 *      x_perm [T*k, D] dtype:   x_perm[r] = x[slot_of_row[r] / k].
 * Rows of one expert are in increasing token order.  Deterministic.
 * ws: moe_permute_workspace_size(cfg, T) bytes of device scratch. */
MOE_API moe_status_t moe_permute(const moe_config_t* cfg, int64_t T, const int32_t* topk_ids, const void* x,
                         int32_t* expert_off, int32_t* row_of_slot, int32_t* slot_of_row, void* x_perm, void* ws,
                         size_t ws_bytes, void* stream);

/* moe_permute without a workspace argument and without any allocation.
 * The pages have no counterpart: this entry point exists for callers that are
 * not allowed to allocate device memory -- a plugin or custom operator inside a
 * host framework or inference server whose allocator owns the whole GPU, or a
 * service whose device-memory budget is fixed at start-up -- and so cannot call
 * cudaMalloc for moe_permute's scratch or keep a workspace between calls.
 * Same arguments, results and errors as moe_permute, except:
 *  - the histogram/scan scratch is a fixed array inside the library (256 KiB,
 *    one per GPU that loads the library, held until the process exits), so
 *    num_local_experts * ceil(T / 256) must be at most 32768 (e.g. T <= 65536
 *    with E = 128); larger sizes return MOE_ERR_UNSUPPORTED and launch nothing;
 *  - each call finds that array's device address in the current CUDA context
 *    (cudaGetSymbolAddress, a runtime call that allocates nothing); the first
 *    call in a context does the lookup and caches it for that context (keyed by
 *    its unique context id, so a context of the caller's own or the one made
 *    after cudaDeviceReset gets a fresh lookup); make that first call before
 *    any stream capture;
 *  - every call on a device shares the array and it keeps the last call's
 *    contents (each call writes every word it reads, so nothing needs clearing),
 *    hence calls that may overlap on the GPU (other streams, other threads) race
 *    and must be serialised by the caller.
 * It calls no cudaMalloc, cudaFree or other allocating routine. */
MOE_API moe_status_t moe_permute_noalloc(const moe_config_t* cfg, int64_t T, const int32_t* topk_ids, const void* x,
                                         int32_t* expert_off, int32_t* row_of_slot, int32_t* slot_of_row,
                                         void* x_perm, void* stream);

/* Per-expert FFN over the permuted rows (R = T*k):
 *   x_perm [R, D], expert_off [E+1] (as produced by moe_permute; read on the device)
 *   -> h [R, F]: clipped SwiGLU of the gate/up projections (+ biases); with
 *      cfg->h_split, h is [R, 2, F]: row r holds bf16(h[r]) then the bf16 rounding
 *      of h[r] - bf16(h[r]),
 *      y_perm [R, D]: h Wd[e]^T + bd[e] for the expert e that owns each row.
 * Computed on the tcgen05 tensor cores with fp32 accumulation from bf16
 * operands (MXFP4 weights are decoded to bf16 in shared memory inside the GEMM
 * mainloop; fp32 layers run in fp32 FMA).  ws: moe_expert_ffn_workspace_size
 * bytes, 16-byte aligned (may be NULL when that is 0); MOE_ERR_WORKSPACE if it
 * is missing or too small. */
MOE_API moe_status_t moe_expert_ffn(const moe_config_t* cfg, int64_t T, const void* x_perm, const int32_t* expert_off,
                            const moe_expert_weights_t* weights, void* h, void* y_perm, void* ws, size_t ws_bytes,
                            void* stream);

/* Weighted combine: y[t] = sum_{j<k} topk_w[t,j] * y_perm[row_of_slot[t,j]],
 * summed in fp32 in fixed j order.  y_perm [T*k, D] in dtype; y [T, D] in dtype,
 * or in fp32 when cfg->y_f32 is set. */
MOE_API moe_status_t moe_combine(const moe_config_t* cfg, int64_t T, const void* y_perm, const int32_t* row_of_slot,
                         const float* topk_w, void* y, void* stream);

/* The whole layer: router/top-k -> dispatch -> gate/up + SwiGLU -> down with
 * the routing weight and the un-permutation fused into its epilogue -> sum
 * over k.  x [T, D] in dtype; y [T, D] in dtype, or in fp32 when cfg->y_f32
 * is set (the k weighted expert outputs are summed in fp32 either way; a dtype
 * output is that sum rounded once).  topk_ids_out [T, k] and topk_w_out
 * [T, k] are optional (NULL: kept in the workspace).  ws: moe_workspace_size
 * bytes. */
MOE_API moe_status_t moe_layer_forward(const moe_config_t* cfg, int64_t T, const void* x, const void* w_router,
                               const void* b_router, const moe_expert_weights_t* weights, void* y,
                               int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes, void* stream);

/* MXFP8 quantization of activation rows, the one MOE_W_MXFP4_A8 applies to x_perm
 * and h (the pages give MXFP8 and its group size 32, "Ollama glm4_moe_lite.go",
 * quantizationParams; the scale rule and rounding are this library's reading):
 *   x [rows, K] bf16 (K a multiple of 32)
 *   -> xq [rows, K] uint8 E4M3 codes (sign bit 7, exponent bits 6..3 bias 7,
 *        mantissa bits 2..0), xq[r, j] = RNE(x[r, j] / 2^X) for j in block b,
 *      sf [rows, moe_mxfp8_scale_stride(K)] uint8: sf[r, b] = X + 127 for the
 *        K/32 blocks b, X the smallest integer with max |x| of the block <=
 *        448 * 2^X (-127 for an all-zero block), then 127 up to the stride.
 * Device pointers, 16-byte aligned.  rows = 0 is a no-op. */
MOE_API int32_t moe_mxfp8_scale_stride(int32_t K);
MOE_API moe_status_t moe_quantize_mxfp8(int64_t rows, int32_t K, const void* x, uint8_t* xq, uint8_t* sf,
                                        void* stream);

/* Reads and clears the current device's error word (synchronises the device).
 * MOE_OK if no kernel flagged anything since the last call, MOE_ERR_TIMEOUT if a
 * bounded wait gave up, MOE_ERR_DEVICE_BOUNDS if an index read on the device was
 * out of range, MOE_ERR_CUDA if the read itself failed. */
MOE_API moe_status_t moe_last_device_error(void);

/* Profiling aid: CUDA events recorded around the stages of moe_layer_forward
 * (and the gate/up and down stages of moe_expert_ffn).  starts[i] and
 * stops[i] (cudaEvent_t handles, may be NULL) are recorded on the call's
 * stream right before and right after stage i: 0 router + top-k, 1 dispatch,
 * 2 gate/up GEMM + SwiGLU, 3 down GEMM (+ weighting and un-permutation),
 * 4 combine.  n <= 5 entries are copied; they apply to every later call in
 * this process until the next call of this function (n = 0 clears). */
MOE_API void moe_set_stage_events(void* const* starts, void* const* stops, int32_t n);

/* Tuning knob for the bf16 expert GEMMs of every later call in this process:
 * 0 = choose by size (default: the weight-stationary decode kernel while the
 * experts average at most 16 routed rows; otherwise single-CTA 128-row tiles for
 * gate/up and CTA-pair tiles for down),
 * 1 = single-CTA tiles, 2 = CTA-pair tiles (256 rows), 3 = decode kernel,
 * 4 = CTA pairs with the expert weights as the MMA's M operand (tokens in N),
 * 5 = moe_layer_forward as the two-kernel decode layer (router logits, then one
 * persistent kernel for top-k, dispatch, both projections and the combine)
 * wherever it applies: dense bf16 weights, T*k <= 512 routed rows averaging at
 * most 16 per expert, E <= 256, k <= 8, hidden_size <= 8192; by size (0) it is
 * taken for 2 <= T with T*k <= E; 6 = as 0 (but never the decode layer), except
 * that moe_layer_forward's single-CTA gate/up kernel gathers its rows from x with
 * TMA gather4 instead of
 * reading a dispatched copy (x_perm), which is then not written (same results bit
 * for bit; slower); 7 = as 6 without the gather, and the MOE_W_MXFP4_A8 GEMMs
 * widen every stage of E2M1 weights in their converter warps instead of loading
 * whole 128-code K blocks through TMA's 4-bit unpacking type (same results bit for
 * bit).  Results are the same up to fp32 accumulation order (the
 * decode layer's are reproducible call to call).  MOE_ERR_INVALID_ARG for other
 * values. */
MOE_API moe_status_t moe_set_expert_gemm_variant(int32_t variant);

/* Number of kernels this library has launched in this process so far. */
MOE_API uint64_t moe_launch_count(void);

/* Time limit, in nanoseconds, of every bounded wait inside the kernels
 * launched afterwards by this process (default 1e9 = 1 s; 0 restores the
 * default).  A debugging aid: a tiny limit makes waits give up early, which
 * moe_last_device_error then reports. */
MOE_API void moe_set_wait_limit_ns(uint64_t ns);

/* ------------------------------------------------------------------------ *
 * The GLM4-MoE-Lite variant of the layer ("Ollama glm4_moe_lite.go":
 * MoEGate.Forward, SwitchMLP.Forward, SharedExperts.Forward, MoE.Forward):
 *   l[t,e]  = x[t] . Wr[e]                               gate linear, no bias
 *   s[t,e]  = sigmoid(l[t,e])
 *   S_t     = the k largest s[t,e] + c[e] (c = e_score_correction_bias, zero
 *             when absent), listed by descending value, ties -> lower index
 *   w[t,j]  = s[t,S_t[j]] / (sum_i s[t,S_t[i]] if k > 1 and norm_topk_prob,
 *             else 1), times routed_scaling_factor
 *   o_e     = (SiLU(x[t] Wg[e]^T) * (x[t] Wu[e]^T)) Wd[e]^T   (no biases, no clip)
 *   y[t]    = sum_j w[t,j] o_{S_t[j]} + shared(x[t]),
 *             shared(x) = (SiLU(x Wsg^T) * (x Wsu^T)) Wsd^T (n_shared_experts > 0)
 * It takes the same moe_config_t (swiglu_limit and swiglu_alpha are not used;
 * wfmt must be MOE_W_DENSE, else MOE_ERR_UNSUPPORTED) and the same expert
 * weight struct, whose bias and scale pointers are ignored.  Ties among the
 * chosen experts and their order are this library's reading; the page leaves
 * them to Argpartition.
 * ------------------------------------------------------------------------ */
typedef struct {
  int32_t norm_topk_prob;               /* nonzero: weights divided by their sum when k > 1 */
  float routed_scaling_factor;          /* every routing weight is multiplied by it (finite) */
  const void* e_score_correction_bias;  /* [E] in dtype, added to the scores for the choice only; NULL = none */
  const void* ws_gate;                  /* shared expert [Fs, D] in dtype (ignored when Fs = 0) */
  const void* ws_up;                    /* shared expert [Fs, D] */
  const void* ws_down;                  /* shared expert [D, Fs] */
  int32_t shared_intermediate_size;     /* Fs: 0 (no shared expert) or a multiple of 16, <= 2^20 */
} moe_glm_params_t;

/* Bytes of workspace moe_glm_router_topk needs for T tokens (the router's fp32
 * logits).  (size_t)-1 if cfg is invalid. */
MOE_API size_t moe_glm_router_workspace_size(const moe_config_t* cfg, int64_t T);

/* Bytes of workspace moe_glm_layer_forward needs for T tokens: as for
 * moe_layer_forward, plus zero biases for the expert GEMMs and, with a shared
 * expert, its offsets, identity slot map and unit weights [T], SiLU output
 * [T, Fs] in dtype and fp32 output rows [T, D].
 * (size_t)-1 if cfg or p is invalid. */
MOE_API size_t moe_glm_workspace_size(const moe_config_t* cfg, const moe_glm_params_t* p, int64_t T);

/* The variant's router: x [T, D], w_router [E, D] in dtype -> topk_ids [T, k]
 * int32, topk_w [T, k] fp32, as defined above.  ws: moe_glm_router_workspace_size
 * bytes. */
MOE_API moe_status_t moe_glm_router_topk(const moe_config_t* cfg, const moe_glm_params_t* p, int64_t T,
                                         const void* x, const void* w_router, int32_t* topk_ids, float* topk_w,
                                         void* ws, size_t ws_bytes, void* stream);

/* The whole variant layer: router, dispatch (the same permutation as
 * moe_permute), SiLU experts, weighted combine plus the shared expert.
 * x [T, D] in dtype; y [T, D] in dtype (fp32 when cfg->y_f32 is set); the
 * routed and shared expert outputs are summed in fp32 and rounded once.
 * weights->w_gate, w_up [E, F, D], w_down [E, D, F] in dtype.  topk_ids_out / topk_w_out optional as in moe_layer_forward.
 * ws: moe_glm_workspace_size bytes. */
MOE_API moe_status_t moe_glm_layer_forward(const moe_config_t* cfg, const moe_glm_params_t* p, int64_t T,
                                           const void* x, const void* w_router, const moe_expert_weights_t* weights,
                                           void* y, int32_t* topk_ids_out, float* topk_w_out, void* ws,
                                           size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
