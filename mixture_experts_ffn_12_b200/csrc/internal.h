// Host-side internal interface between the C ABI (moe_abi.cu) and the kernel
// launchers.  Not installed; the public interface is include/moe.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace moe {

// Kernels this library has launched in this process (moe_launch_count).
inline std::atomic<uint64_t> g_launches{0};
inline void count_launch(uint64_t n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

struct Launch {
  cudaStream_t stream;
  int num_sms;
  unsigned long long wait_limit_ns;
};

// Router + top-k + softmax.  ids/w are [T, k].  `partial` (router_partial_bytes of
// scratch, may be null) lets large bf16 batches split K across more CTAs.
cudaError_t router_topk(const Launch& L, bool bf16, int64_t T, int D, int E, int k, const void* x,
                        const void* w_router, const void* b_router, int32_t* ids, float* w,
                        float* partial = nullptr);
size_t router_partial_bytes(int64_t T, int E);

// Scratch (int32 words) the permute needs for T tokens and E experts.
size_t permute_scratch_words(int64_t T, int E);

// Dispatch: expert_off [E+1], row_of_slot [T*k], slot_of_row [T*k], x_perm [T*k, D].
// x / x_perm may be null (index maps only).
cudaError_t permute(const Launch& L, bool bf16, int64_t T, int D, int E, int k, const int32_t* ids,
                    const void* x, int32_t* expert_off, int32_t* row_of_slot, int32_t* slot_of_row,
                    void* x_perm, int32_t* scratch);

struct ExpertWeights {
  const void *w_gate, *w_up, *w_down;        // dense [E,F,D],[E,F,D],[E,D,F]; MXFP4: packed [..,K/2]
  const uint8_t *s_gate, *s_up, *s_down;     // MXFP4 scales [..,K/32]
  const void *b_gate, *b_up, *b_down;        // [E,F],[E,F],[E,D]
};

// h[R, F] = swiglu(x_perm W_g^T + b_g, x_perm W_u^T + b_u), per expert segment.
// gate_lo is the gate's lower clip: 0 for the clipped SwiGLU; -inf with limit = inf and
// alpha = 1 gives SiLU(g) * u.  h_halves = 2 (bf16 only): h is [R, 2, F], the bf16 rounding
// of h and the bf16 rounding of what that dropped (cudaErrorNotSupported for the fp32
// kernels and the weights-in-M pair kernel).
// gather (the layer only): A row r is x[slot_of_row[r] / k] (x [T, D] bf16), read by TMA
// gather4 instead of from x_perm, which is then not read (may be null); only where
// gateup_gathers() holds.
struct GateupGather {
  const void* x;
  const int32_t* slot_of_row;
  int k;
  int64_t T;
};
bool gateup_gathers(bool bf16, int64_t R, int E);
cudaError_t expert_gateup(const Launch& L, bool bf16, int64_t R, int D, int F, int E, const void* x_perm,
                          const int32_t* expert_off, const ExpertWeights& w, float limit, float alpha, void* h,
                          float gate_lo = 0.0f, int h_halves = 1, const GateupGather* gather = nullptr);

// Down projection.  If slot_of_row == nullptr: out[r] = h[r] W_d^T + b_d (permuted order, dtype);
// else out[slot_of_row[r]] = topk_w[slot] * (h[r] W_d^T + b_d) (slot order, fp32).
// h_halves = 2: h is [R, 2, F] as written by expert_gateup, and both halves are summed.
cudaError_t expert_down(const Launch& L, bool bf16, int64_t R, int D, int F, int E, const void* h,
                        const int32_t* expert_off, const ExpertWeights& w, const int32_t* slot_of_row,
                        const float* topk_w, void* out, int h_halves = 1);

// y[t] = sum_j w[t,j] * y_perm[row_of_slot[t,j]]   (y_perm in dtype; y in dtype, or fp32 if out_f32)
cudaError_t combine_gather(const Launch& L, bool bf16, bool out_f32, int64_t T, int D, int k, const void* y_perm,
                           const int32_t* row_of_slot, const float* w, void* y);
// y[t] = sum_j ys[t*k + j]   (ys fp32; y bf16 if out_bf16, else fp32)
cudaError_t combine_slots(const Launch& L, bool out_bf16, int64_t T, int D, int k, const void* ys, void* y);

// MXFP4 weights with MXFP8 activations on the block-scaled tensor cores.
// Scale rows of K-long activation or weight rows: mx8_sf_bytes_per_row(K) bytes
// (one E8M0 byte per 32 elements, then 127 = 2^0 for the padded K blocks).
int mx8_sf_bytes_per_row(int K);
// x [T, K] bf16 -> xq [T, K] E4M3 and sf [T, mx8_sf_bytes_per_row(K)].
cudaError_t mx8_quant_rows(const Launch& L, int64_t T, int K, const void* x, uint8_t* xq, uint8_t* sf);
// The caller's weight scales [E, N, K/32] as padded rows [E, N, mx8_sf_bytes_per_row(K)].
cudaError_t mx8_weight_scales(const Launch& L, int D, int F, int E, const ExpertWeights& w, uint8_t* sf_gate,
                              uint8_t* sf_up, uint8_t* sf_down);
// gate/up + clipped SwiGLU: xq/sfx MXFP8 x_perm -> hq [R, F] E4M3 + sfh scale rows.
cudaError_t expert_gateup_mx8(const Launch& L, int64_t R, int D, int F, int E, const uint8_t* xq,
                              const uint8_t* sfx, const int32_t* expert_off, const ExpertWeights& w,
                              const uint8_t* sf_gate, const uint8_t* sf_up, float limit, float alpha, uint8_t* hq,
                              uint8_t* sfh);
// down: ys[slot_of_row[r]] = topk_w[slot] * (hq[r] W_d^T + b_d), fp32.
cudaError_t expert_down_mx8(const Launch& L, int64_t R, int D, int F, int E, const uint8_t* hq, const uint8_t* sfh,
                            const int32_t* expert_off, const ExpertWeights& w, const uint8_t* sf_down,
                            const int32_t* slot_of_row, const float* topk_w, float* ys);
// dst[r] = src[slot_of_row[r] / k] for byte rows of row_bytes (a multiple of 16).
cudaError_t gather_rows(const Launch& L, const void* src, const int32_t* slot_of_row, int64_t R, int k, int64_t T,
                        int row_bytes, void* dst);

// The same two projections with MXFP4 expert weights, dequantised inside the GEMM mainloop.
// The kernels read the E8M0 scales from a copy relaid as [E][ceil(K/64)][N][2]
// (mx_scale_bytes each), written by mx_scale_relayout on the same stream.
size_t mx_scale_bytes(int rows, int K, int E);
cudaError_t mx_scale_relayout(const Launch& L, int D, int F, int E, const ExpertWeights& w, uint8_t* s_gate,
                              uint8_t* s_up, uint8_t* s_down);
cudaError_t expert_gateup_mxfp4(const Launch& L, int64_t R, int D, int F, int E, const void* x_perm,
                                const int32_t* expert_off, const ExpertWeights& w, const uint8_t* s_gate2,
                                const uint8_t* s_up2, float limit, float alpha, void* h);
cudaError_t expert_down_mxfp4(const Launch& L, int64_t R, int D, int F, int E, const void* h,
                              const int32_t* expert_off, const ExpertWeights& w, const uint8_t* s_down2,
                              const int32_t* slot_of_row, const float* topk_w, void* out);

// The whole layer for a few tokens (bf16; decode_layer_shape): router logits into
// `logits` [T, E], then one persistent kernel for top-k, dispatch, both projections and
// the combine.  Scratch: cnt (decode_layer_counter_words ints), part
// (decode_layer_part_bytes), h [R, h_halves * F], ys [R, D] fp32.  x and the rows of h are
// read with 16-byte copies (x 16-byte aligned).  ids_out / w_out [T, k] may be null.
bool decode_layer_shape(bool bf16, int64_t T, int k, int E, int D, int F);
bool decode_layer_selected(bool bf16, int64_t T, int k, int E, int D, int F);
size_t decode_layer_counter_words(int64_t T, int k, int E, int D, int F);
size_t decode_layer_part_bytes();
cudaError_t decode_layer(const Launch& L, int64_t T, int D, int F, int E, int k, const void* x, const void* w_router,
                         const void* b_router, const ExpertWeights& w, float limit, float alpha, float gate_lo,
                         int h_halves, bool out_f32, void* y, int32_t* ids_out, float* w_out, float* logits, int* cnt,
                         float* part, void* h, float* ys);

cudaError_t read_and_clear_device_error(int* bits);

}  // namespace moe
