// C ABI of libmoe (include/moe.h): argument validation, workspace checks and launches.
// Every check here runs on the host before anything is enqueued; device-side findings go to the
// workspace status word and are reported by moe_sync_status.
#include <math.h>
#include <stdint.h>

#include "../../include/moe.h"
#include "common.cuh"
#include "launch.h"

namespace moe {

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace moe

namespace {

constexpr int kMaxE = 1024;
constexpr int kMaxK = 32;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status_t from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  cudaGetLastError();  // clear a sticky launch error so the next call starts clean
  return MOE_ERR_CUDA;
}

}  // namespace

extern "C" {

int moe_abi_version(void) { return 1; }

const char* moe_status_string(moe_status_t st) {
  switch (st) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_INVALID_TOPK: return "MOE_ERR_INVALID_TOPK: routing index out of range";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape not supported";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA launch or runtime error";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace too small or misaligned";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a bounded device wait ran out";
    case MOE_ERR_INVALID_COUNTS: return "MOE_ERR_INVALID_COUNTS: row counts do not fit the buffers";
  }
  return "unknown moe_status_t";
}

int moe_capacity(double cf, int T, int k, int E) {
  if (T < 0 || k < 1 || E < 1) return -1;
  if (!(cf > 0.0)) return 0;
  const double c = ceil(cf * (static_cast<double>(T) * k) / E);
  if (c > 2147483647.0) return 2147483647;
  return static_cast<int>(c);
}

moe_status_t moe_route(const float* logits, int T, int E, int k, int renormalize,
                       int32_t* topk_idx, float* topk_w, int32_t* expert_routed,
                       moe_stream_t stream) {
  if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > E || k > kMaxK) return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * E > INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (logits == nullptr || topk_idx == nullptr || topk_w == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(logits, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) ||
      !aligned(expert_routed, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_route(logits, T, E, k, renormalize ? 1 : 0, topk_idx, topk_w,
                                     expert_routed, reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_dispatch_workspace_size(int T, int E, int k) {
  if (T < 0 || E < 1 || k < 1) return 0;
  return moe::dispatch_workspace_bytes(T, E, k);
}

moe_status_t moe_dispatch(const void* x, int T, int H, const int32_t* topk_idx, int k, int E,
                          int R, int capacity, moe_payload_t payload, void* send,
                          float* send_scales, int32_t* expert_counts, int32_t* expert_offsets,
                          int32_t* rank_offsets, int32_t* slot_row, int32_t* row_token, void* ws,
                          size_t ws_bytes, moe_stream_t stream) {
  if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > E || k > kMaxK || R < 1 || E % R != 0 ||
      capacity < 0 || H < 8)
    return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * k >= INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (payload != MOE_PAYLOAD_BF16 && payload != MOE_PAYLOAD_FP8_E4M3_B128)
    return MOE_ERR_INVALID_ARG;
  if (H % 8 != 0) return MOE_ERR_UNSUPPORTED;
  const bool fp8 = payload == MOE_PAYLOAD_FP8_E4M3_B128;
  if (fp8 && H % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (expert_counts == nullptr || expert_offsets == nullptr || rank_offsets == nullptr ||
      ws == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && (x == nullptr || topk_idx == nullptr || send == nullptr || slot_row == nullptr ||
                row_token == nullptr || (fp8 && send_scales == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(send, 16) || !aligned(send_scales, 4) || !aligned(topk_idx, 4))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256) || ws_bytes < moe::dispatch_workspace_bytes(T, E, k)) return MOE_ERR_WORKSPACE;
  return from_cuda(moe::launch_dispatch(x, T, H, topk_idx, k, E, R, capacity, fp8 ? 1 : 0, send,
                                        send_scales, expert_counts, expert_offsets, rank_offsets,
                                        slot_row, row_token, ws,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_ffn_workspace_size(int max_rows, int E, int H, int F, moe_payload_t payload) {
  if (max_rows < 0 || E < 1 || H < 1 || F < 1) return 0;
  return moe::ffn_workspace_bytes(max_rows, H, F, payload == MOE_PAYLOAD_FP8_E4M3_B128, E);
}

moe_status_t moe_expert_ffn(const void* send, const float* send_scales, moe_payload_t payload,
                            const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                            const void* w_gate, const void* w_up, const void* w_down,
                            void* expert_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (max_rows < 0 || E < 1 || E > kMaxE || H < 1 || F < 1) return MOE_ERR_INVALID_ARG;
  if (payload != MOE_PAYLOAD_BF16 && payload != MOE_PAYLOAD_FP8_E4M3_B128)
    return MOE_ERR_INVALID_ARG;
  const bool fp8 = payload == MOE_PAYLOAD_FP8_E4M3_B128;
  if (H % 64 != 0 || F % 64 != 0 || (fp8 && H % 128 != 0)) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(E) * F > INT32_MAX || static_cast<long long>(E) * H > INT32_MAX)
    return MOE_ERR_UNSUPPORTED;
  if (expert_offsets == nullptr || w_gate == nullptr || w_up == nullptr || w_down == nullptr ||
      ws == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (max_rows > 0 && (send == nullptr || expert_out == nullptr || (fp8 && send_scales == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(send, 16) || !aligned(w_gate, 16) || !aligned(w_up, 16) || !aligned(w_down, 16) ||
      !aligned(expert_out, 16) || !aligned(expert_offsets, 4) || !aligned(send_scales, 4))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256) || ws_bytes < moe::ffn_workspace_bytes(max_rows, H, F, fp8 ? 1 : 0, E))
    return MOE_ERR_WORKSPACE;
  return from_cuda(moe::launch_expert_ffn(send, send_scales, fp8 ? 1 : 0, expert_offsets, max_rows,
                                          E, H, F, w_gate, w_up, w_down, nullptr, nullptr, nullptr,
                                          expert_out, ws, reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_ffn_weight_list_bytes(int E) {
  if (E < 1 || E > kMaxE) return 0;
  return moe::ffn_weight_list_bytes(E);
}

moe_status_t moe_ffn_weight_list_init(const void* const* w_gate, const void* const* w_up,
                                      const void* const* w_down, int E, int H, int F, void* list,
                                      moe_stream_t stream) {
  if (E < 1 || E > kMaxE || H < 1 || F < 1) return MOE_ERR_INVALID_ARG;
  if (H % 64 != 0 || F % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (w_gate == nullptr || w_up == nullptr || w_down == nullptr || list == nullptr ||
      !aligned(list, 64))
    return MOE_ERR_INVALID_ARG;
  for (int e = 0; e < E; ++e)
    if (w_gate[e] == nullptr || w_up[e] == nullptr || w_down[e] == nullptr ||
        !aligned(w_gate[e], 16) || !aligned(w_up[e], 16) || !aligned(w_down[e], 16))
      return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::ffn_weight_list_init(w_gate, w_up, w_down, E, H, F, list,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_ffn_list(const void* send, const float* send_scales, moe_payload_t payload,
                                 const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                                 const void* list, void* expert_out, void* ws, size_t ws_bytes,
                                 moe_stream_t stream) {
  if (max_rows < 0 || E < 1 || E > kMaxE || H < 1 || F < 1) return MOE_ERR_INVALID_ARG;
  if (payload != MOE_PAYLOAD_BF16 && payload != MOE_PAYLOAD_FP8_E4M3_B128)
    return MOE_ERR_INVALID_ARG;
  const bool fp8 = payload == MOE_PAYLOAD_FP8_E4M3_B128;
  if (H % 64 != 0 || F % 64 != 0 || (fp8 && H % 128 != 0)) return MOE_ERR_UNSUPPORTED;
  if (expert_offsets == nullptr || list == nullptr || ws == nullptr || !aligned(list, 64))
    return MOE_ERR_INVALID_ARG;
  if (max_rows > 0 && (send == nullptr || expert_out == nullptr || (fp8 && send_scales == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(send, 16) || !aligned(expert_out, 16) || !aligned(expert_offsets, 4) ||
      !aligned(send_scales, 4))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256) || ws_bytes < moe::ffn_workspace_bytes(max_rows, H, F, fp8 ? 1 : 0, E))
    return MOE_ERR_WORKSPACE;
  return from_cuda(moe::launch_expert_ffn(send, send_scales, fp8 ? 1 : 0, expert_offsets, max_rows,
                                          E, H, F, nullptr, nullptr, nullptr, list, nullptr,
                                          nullptr, expert_out, ws,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_quantize_rows_fp8(const void* x, int rows, int K, void* codes, float* scales,
                                   moe_stream_t stream) {
  if (rows < 0 || K < 8) return MOE_ERR_INVALID_ARG;
  if (K % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (rows > 0 && (x == nullptr || codes == nullptr || scales == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 4)) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_quantize_rows_fp8(x, rows, K, codes, scales,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_ffn_w8_workspace_size(int max_rows, int E, int H, int F, moe_payload_t payload) {
  if (max_rows < 0 || E < 1 || H < 1 || F < 1) return 0;
  return moe::ffn_workspace_bytes(max_rows, H, F, payload == MOE_PAYLOAD_FP8_E4M3_B128, E, 1);
}

moe_status_t moe_expert_ffn_w8(const void* send, const float* send_scales, moe_payload_t payload,
                               const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                               const void* w_gate_q, const float* w_gate_scale,
                               const void* w_up_q, const float* w_up_scale, const void* w_down,
                               void* expert_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (max_rows < 0 || E < 1 || E > kMaxE || H < 1 || F < 1) return MOE_ERR_INVALID_ARG;
  if (payload != MOE_PAYLOAD_BF16 && payload != MOE_PAYLOAD_FP8_E4M3_B128)
    return MOE_ERR_INVALID_ARG;
  const bool fp8 = payload == MOE_PAYLOAD_FP8_E4M3_B128;
  if (H % 64 != 0 || F % 64 != 0 || (fp8 && H % 128 != 0)) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(E) * F > INT32_MAX || static_cast<long long>(E) * H > INT32_MAX)
    return MOE_ERR_UNSUPPORTED;
  if (expert_offsets == nullptr || w_gate_q == nullptr || w_gate_scale == nullptr ||
      w_up_q == nullptr || w_up_scale == nullptr || w_down == nullptr || ws == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (max_rows > 0 && (send == nullptr || expert_out == nullptr || (fp8 && send_scales == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(send, 16) || !aligned(w_gate_q, 16) || !aligned(w_up_q, 16) ||
      !aligned(w_down, 16) || !aligned(expert_out, 16) || !aligned(expert_offsets, 4) ||
      !aligned(send_scales, 4) || !aligned(w_gate_scale, 8) || !aligned(w_up_scale, 8))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256) || ws_bytes < moe::ffn_workspace_bytes(max_rows, H, F, fp8 ? 1 : 0, E, 1))
    return MOE_ERR_WORKSPACE;
  return from_cuda(moe::launch_expert_ffn(send, send_scales, fp8 ? 1 : 0, expert_offsets, max_rows,
                                          E, H, F, w_gate_q, w_up_q, w_down, nullptr, w_gate_scale,
                                          w_up_scale, expert_out, ws,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_regroup(const int32_t* counts, int A, int B, int src_order, int src_stride,
                            int src_rows, int dst_order, int dst_stride, int dst_rows,
                            const void* src, void* dst, size_t row_bytes, const void* src_aux,
                            void* dst_aux, size_t aux_row_bytes, int32_t* dst_offsets,
                            int32_t* status, moe_stream_t stream) {
  if (A < 1 || B < 1 || static_cast<long long>(A) * B > moe::kMaxRegroupSegments)
    return MOE_ERR_INVALID_ARG;
  if ((src_order != 0 && src_order != 1) || (dst_order != 0 && dst_order != 1))
    return MOE_ERR_INVALID_ARG;
  if (src_stride < 0 || dst_stride < 0 || src_rows < 0 || dst_rows < 0) return MOE_ERR_INVALID_ARG;
  if (counts == nullptr || !aligned(counts, 4) || !aligned(status, 4) || !aligned(dst_offsets, 4))
    return MOE_ERR_INVALID_ARG;
  if (row_bytes == 0 || row_bytes % 4 != 0 || src == nullptr || dst == nullptr ||
      !aligned(src, 4) || !aligned(dst, 4) || src == dst)
    return MOE_ERR_INVALID_ARG;
  if (aux_row_bytes != 0 && (aux_row_bytes % 4 != 0 || src_aux == nullptr || dst_aux == nullptr ||
                             !aligned(src_aux, 4) || !aligned(dst_aux, 4) || src_aux == dst_aux))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_ep_regroup(
      counts, A, B, src_order, src_stride, src_rows, dst_order, dst_stride, dst_rows, src, dst,
      row_bytes, aux_row_bytes ? src_aux : nullptr, aux_row_bytes ? dst_aux : nullptr,
      aux_row_bytes, dst_offsets, reinterpret_cast<int*>(status),
      reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_exchange(const int32_t* all_counts, int R, int E, int rank, int direction,
                             const uint64_t* peer_rows, const uint64_t* peer_aux,
                             int peer_rows_cap, void* local_rows, void* local_aux,
                             int local_rows_cap, size_t row_bytes, size_t aux_row_bytes,
                             int32_t* local_offsets, int32_t* status, moe_stream_t stream) {
  if (R < 1 || R > moe::kMaxEpRanks || E < R || E % R != 0 || E > moe::kMaxRegroupSegments)
    return MOE_ERR_INVALID_ARG;
  if (rank < 0 || rank >= R || (direction != MOE_EP_PULL && direction != MOE_EP_PUSH))
    return MOE_ERR_INVALID_ARG;
  if (peer_rows_cap < 0 || local_rows_cap < 0) return MOE_ERR_INVALID_ARG;
  if (all_counts == nullptr || peer_rows == nullptr || local_rows == nullptr ||
      !aligned(all_counts, 4) || !aligned(peer_rows, 8) || !aligned(local_rows, 4) ||
      !aligned(status, 4) || !aligned(local_offsets, 4))
    return MOE_ERR_INVALID_ARG;
  if (row_bytes == 0 || row_bytes % 4 != 0) return MOE_ERR_INVALID_ARG;
  if (aux_row_bytes != 0 && (aux_row_bytes % 4 != 0 || peer_aux == nullptr ||
                             local_aux == nullptr || !aligned(peer_aux, 8) ||
                             !aligned(local_aux, 4)))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_ep_exchange(
      all_counts, R, E, rank, direction == MOE_EP_PUSH ? 1 : 0,
      reinterpret_cast<const unsigned long long*>(peer_rows),
      reinterpret_cast<const unsigned long long*>(peer_aux), peer_rows_cap, local_rows,
      aux_row_bytes ? local_aux : nullptr, local_rows_cap, row_bytes, aux_row_bytes, local_offsets,
      reinterpret_cast<int*>(status), reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_backward_workspace_size(int max_rows, int T, int k, int H, int F) {
  if (max_rows < 0 || T < 0 || k < 1 || H < 1 || F < 1) return 0;
  return moe::backward_workspace_bytes(max_rows, T, k, H, F);
}

moe_status_t moe_backward(const void* dy, int T, int H, int k, int E, int F, const float* logits,
                          int renormalize, const int32_t* topk_idx, const float* topk_w,
                          const int32_t* slot_row, const int32_t* expert_offsets, int max_rows,
                          const void* ffn_input, const void* expert_out, const void* w_gate,
                          const void* w_up, const void* w_down, void* dx, float* d_logits,
                          float* d_topk_w, float* d_w_gate, float* d_w_up, float* d_w_down,
                          void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (T < 0 || k < 1 || k > 32 || E < 1 || E > 1024 || k > E || max_rows < 0 || H < 8 || F < 1)
    return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * k > max_rows) return MOE_ERR_INVALID_ARG;
  if (H % 64 != 0 || F % 64 != 0) return MOE_ERR_UNSUPPORTED;
  const void* need[] = {expert_offsets, w_gate, w_up, w_down, d_w_gate, d_w_up, d_w_down, ws};
  for (const void* q : need)
    if (q == nullptr) return MOE_ERR_INVALID_ARG;
  // the per-token arrays are empty (possibly NULL) for an empty batch
  if (T > 0 && (dy == nullptr || dx == nullptr || ffn_input == nullptr || expert_out == nullptr ||
                topk_idx == nullptr || topk_w == nullptr || slot_row == nullptr ||
                d_logits == nullptr || d_topk_w == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!renormalize && T > 0 && logits == nullptr) return MOE_ERR_INVALID_ARG;
  const void* a16[] = {dy, dx, ffn_input, expert_out, w_gate, w_up, w_down, d_w_gate, d_w_up,
                       d_w_down};
  for (const void* q : a16)
    if (!aligned(q, 16)) return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < moe::backward_workspace_bytes(max_rows, T, k, H, F)) return MOE_ERR_WORKSPACE;
  return from_cuda(moe::launch_backward(dy, T, H, k, E, F, logits, renormalize, topk_idx, topk_w,
                                        slot_row, expert_offsets, max_rows, ffn_input, expert_out,
                                        w_gate, w_up, w_down, dx, d_logits, d_topk_w, d_w_gate,
                                        d_w_up, d_w_down, ws,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_combine_backward(const void* dy, int T, int H, int k, int E, const float* logits,
                                  int renormalize, const int32_t* topk_idx, const float* topk_w,
                                  const int32_t* slot_row, int max_rows, const void* expert_out,
                                  void* d_eo, float* d_topk_w, float* d_logits,
                                  moe_stream_t stream) {
  if (T < 0 || k < 1 || k > 32 || E < 1 || E > 1024 || k > E || max_rows < 0 || H < 8)
    return MOE_ERR_INVALID_ARG;
  if (H % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (T > 0 && (dy == nullptr || topk_idx == nullptr || topk_w == nullptr || slot_row == nullptr ||
                expert_out == nullptr || d_eo == nullptr || d_topk_w == nullptr ||
                d_logits == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!renormalize && T > 0 && logits == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(dy, 16) || !aligned(expert_out, 16) || !aligned(d_eo, 16)) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_combine_backward(
      dy, T, H, k, E, logits, renormalize, topk_idx, topk_w, slot_row, max_rows, expert_out, d_eo,
      d_topk_w, d_logits, nullptr, reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_expert_backward_workspace_size(int max_rows, int F) {
  if (max_rows < 0 || F < 1) return 0;
  return moe::expert_backward_workspace_bytes(max_rows, F);
}

moe_status_t moe_expert_backward(const void* ffn_input, const void* d_eo,
                                 const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                                 const void* w_gate, const void* w_up, const void* w_down,
                                 void* dx_rows, float* d_w_gate, float* d_w_up, float* d_w_down,
                                 void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (E < 1 || E > 1024 || max_rows < 0 || H < 64 || F < 64) return MOE_ERR_INVALID_ARG;
  if (H % 64 != 0 || F % 64 != 0) return MOE_ERR_UNSUPPORTED;
  const void* need[] = {expert_offsets, w_gate, w_up, w_down, d_w_gate, d_w_up, d_w_down, ws};
  for (const void* q : need)
    if (q == nullptr) return MOE_ERR_INVALID_ARG;
  if (max_rows > 0 && (ffn_input == nullptr || d_eo == nullptr || dx_rows == nullptr))
    return MOE_ERR_INVALID_ARG;
  const void* a16[] = {ffn_input, d_eo, dx_rows, w_gate, w_up, w_down, d_w_gate, d_w_up, d_w_down};
  for (const void* q : a16)
    if (!aligned(q, 16)) return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < moe::expert_backward_workspace_bytes(max_rows, F)) return MOE_ERR_WORKSPACE;
  auto up = [](size_t b) { return (b + 255) / 256 * 256; };
  const size_t r = static_cast<size_t>(max_rows > 0 ? max_rows : 1);
  uint8_t* w = static_cast<uint8_t*>(ws);
  void* h = w + 256;
  void* dg = w + 256 + up(r * F * 2);
  void* du = w + 256 + 2 * up(r * F * 2);
  return from_cuda(moe::launch_expert_backward(
      ffn_input, d_eo, expert_offsets, max_rows, E, H, F, w_gate, w_up, w_down, dx_rows, d_w_gate,
      d_w_up, d_w_down, reinterpret_cast<int*>(w), h, dg, du,
      reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_combine(const void* expert_out, int max_rows, const int32_t* slot_row,
                         const float* topk_w, int T, int k, int H, void* y, int32_t* status,
                         moe_stream_t stream) {
  if (T < 0 || k < 1 || k > kMaxK || H < 8 || max_rows < 0) return MOE_ERR_INVALID_ARG;
  if (H % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (T > 0 && (slot_row == nullptr || topk_w == nullptr || y == nullptr ||
                (max_rows > 0 && expert_out == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(expert_out, 16) || !aligned(y, 16) || !aligned(slot_row, 4) ||
      !aligned(topk_w, 4) || !aligned(status, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_combine(expert_out, max_rows, slot_row, topk_w, T, k, H, y,
                                       reinterpret_cast<int*>(status),
                                       reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_sync_status(void* ws, moe_stream_t stream) {
  if (ws == nullptr || !aligned(ws, 4)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return from_cuda(cudaErrorUnknown);
  int word = 0;
  if (cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return from_cuda(cudaErrorUnknown);
  if (word != 0 && cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return from_cuda(cudaErrorUnknown);
  if (word & moe::kStatusInvalidTopk) return MOE_ERR_INVALID_TOPK;
  if (word & moe::kStatusTimeout) return MOE_ERR_TIMEOUT;
  if (word & moe::kStatusBadCounts) return MOE_ERR_INVALID_COUNTS;
  return MOE_OK;
}

}  // extern "C"
