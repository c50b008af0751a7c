// Internal launchers of libmoe (host side).  The public C ABI is include/moe.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#ifndef MOE_USE_PDL
#define MOE_USE_PDL 1
#endif

namespace moe {

int num_sms();  // SM count of the current device (cached per device)

// Launch with programmatic stream serialisation (see griddep_wait in common.cuh).  pdl = false
// gives an ordinary launch; it is used when the previous operation on the stream is not a kernel
// (a memset), so that ordering never depends on how programmatic serialisation treats it.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_if(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (pdl && MOE_USE_PDL) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  return launch_pdl_if(true, kernel, grid, block, smem, s, std::forward<Args>(args)...);
}
  // SM count of the current device (cached per device)

cudaError_t launch_route(const float* logits, int T, int E, int k, int renorm, int32_t* topk_idx,
                         float* topk_w, int32_t* routed, cudaStream_t s);

// Dispatch workspace layout (bytes from the 256-byte-aligned base):
//   [0, 4)    status word (kStatus* bits)
//   [256, ..) per-chunk expert histogram [n_chunks][E] int32, chunks of dispatch_chunk_tokens(k)
int dispatch_chunk_tokens(int k);     // 16 * floor(128 / k), at least 16: ~2048 slots per chunk
size_t dispatch_workspace_bytes(int T, int E, int k);

cudaError_t launch_dispatch(const void* x, int T, int H, const int32_t* topk_idx, int k, int E,
                            int R, int capacity, int fp8, void* send, float* send_scales,
                            int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_offsets,
                            int32_t* slot_row, int32_t* row_token, void* ws, cudaStream_t s);

// The same two kernels with the scratch pieces given separately (status word, histogram table).
cudaError_t launch_dispatch_parts(const void* x, int T, int H, const int32_t* topk_idx, int k,
                                  int E, int R, int capacity, int fp8, void* send,
                                  float* send_scales, int32_t* expert_counts,
                                  int32_t* expert_offsets, int32_t* rank_offsets,
                                  int32_t* slot_row, int32_t* row_token, int* status,
                                  int32_t* hist, cudaStream_t s);

cudaError_t launch_combine(const void* expert_out, int max_rows, const int32_t* slot_row,
                           const float* topk_w, int T, int k, int H, void* y, int* status,
                           cudaStream_t s);

// FFN workspace layout: [0,4) status, [256, ..) h [max_rows, F] bf16, then for the FP8 payload the
// dequantised rows [max_rows, H] bf16, then the GEMM-1 completion counters.
// w8: room for the FFN input rows' e4m3 codes [max_rows, H] and scales [max_rows] as well.
size_t ffn_workspace_bytes(int max_rows, int H, int F, int fp8, int E, int w8 = 0);

// wlist == nullptr: the weights are contiguous [E, F, H] / [E, H, F] arrays; otherwise the
// per-expert descriptors written by ffn_weight_list_init (and w_gate / w_up / w_down are unused).
// w_gate_scale / w_up_scale non-null: w_gate / w_up are e4m3 codes [E, F, H] with one fp32 scale
// per row [E, F] (FP8 first projection); wlist must then be nullptr.
cudaError_t launch_expert_ffn(const void* send, const float* send_scales, int fp8,
                              const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                              const void* w_gate, const void* w_up, const void* w_down,
                              const void* wlist, const float* w_gate_scale,
                              const float* w_up_scale, void* expert_out, void* ws, cudaStream_t s);

// Rows of bf16 [rows, K] -> e4m3 codes [rows, K] + one fp32 scale per row (amax / 448).
cudaError_t launch_quantize_rows_fp8(const void* x, int rows, int K, void* codes, float* scales,
                                     cudaStream_t s);

// Per-expert weight descriptors: four 128-byte TMA descriptors per expert.
size_t ffn_weight_list_bytes(int E);
cudaError_t ffn_weight_list_init(const void* const* w_gate, const void* const* w_up,
                                 const void* const* w_down, int E, int H, int F, void* list,
                                 cudaStream_t s);

// The backward's two halves: the combine backward (d_eo, routing-weight and logit gradients, the
// unit weights of the final combine when `ones` is given) and the experts' GEMMs (workspace:
// status | h, dg, du).
cudaError_t launch_combine_backward(const void* dy, int T, int H, int k, int E,
                                   const float* logits, int renormalize, const int32_t* topk_idx,
                                   const float* topk_w, const int32_t* slot_row, int max_rows,
                                   const void* expert_out, void* d_eo, float* d_topk_w,
                                   float* d_logits, float* ones, cudaStream_t s);
size_t expert_backward_workspace_bytes(int max_rows, int F);
cudaError_t launch_expert_backward(const void* ffn_input, const void* d_eo,
                                   const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                                   const void* w_gate, const void* w_up, const void* w_down,
                                   void* dx_rows, float* d_w_gate, float* d_w_up, float* d_w_down,
                                   int* status, void* h, void* dg, void* du, cudaStream_t s);
// Backward of the layer (workspace: status | d_eo | h, dg, du | dx_rows | unit weights).
size_t backward_workspace_bytes(int max_rows, int T, int k, int H, int F);
cudaError_t launch_backward(const void* dy, int T, int H, int k, int E, int F, const float* logits,
                            int renormalize, const int32_t* topk_idx, const float* topk_w,
                            const int32_t* slot_row, const int32_t* expert_offsets, int max_rows,
                            const void* ffn_input, const void* expert_out, const void* w_gate,
                            const void* w_up, const void* w_down, void* dx, float* d_logits,
                            float* d_topk_w, float* d_w_gate, float* d_w_up, float* d_w_down,
                            void* ws, cudaStream_t s);

// Rows between this rank's expert-major buffer and every source's packed buffer (peer pointers).
cudaError_t launch_ep_exchange(const int32_t* all_counts, int R, int E, int rank, int push,
                               const unsigned long long* peer_rows,
                               const unsigned long long* peer_aux, int peer_cap, void* local_rows,
                               void* local_aux, int local_cap, size_t row_bytes, size_t aux_bytes,
                               int32_t* local_offsets, int* status, cudaStream_t s);

// Segmented row copy between the layouts on the two sides of an expert-parallel all-to-all.
cudaError_t launch_ep_regroup(const int32_t* counts, int A, int B, int src_order, int src_stride,
                              int src_rows, int dst_order, int dst_stride, int dst_rows,
                              const void* src, void* dst, size_t row_bytes, const void* src_aux,
                              void* dst_aux, size_t aux_row_bytes, int32_t* dst_offsets,
                              int* status, cudaStream_t s);

}  // namespace moe
