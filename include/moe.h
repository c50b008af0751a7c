/*
 * moe.h - C ABI of libmoe.so: the MoE expert-parallel token shuffle on one B200 (sm_100a).
 *
 * The path has four stream-ordered calls, each a set of hand-written CUDA kernels:
 *
 *   moe_route       fused fp32 softmax + top-k router with a per-expert histogram
 *   moe_dispatch    per-expert counts, offsets and stable positions, then the packed
 *                   expert-major (= rank-major) send buffer, bf16 or FP8 e4m3 + fp32 block scales,
 *                   with optional capacity dropping in token order
 *   moe_expert_ffn  grouped SwiGLU expert FFN on the packed rows (tcgen05 / TMEM / TMA)
 *   moe_combine     weighted gather back into token order, fp32 accumulate in fixed slot order
 *
 * Expert-parallel ranks are emulated as partitions of one HBM pool: rank r owns experts
 * [r*E/R, (r+1)*E/R), so the expert-major send buffer is rank-major too and rank r's slice is
 * rows rank_offsets[r] .. rank_offsets[r+1].
 *
 * Conventions for every call:
 *  - Ownership: every pointer is caller-owned memory.  Unless stated otherwise it is DEVICE memory
 *    of the current CUDA device.  The library allocates nothing and frees nothing; scratch memory is
 *    the caller's workspace (sizes from the *_workspace_size queries).  This follows the
 *    group/handle split with caller-registered allocation of the NCCL EP page ("NCCL EP架构解析",
 *    sections 1 and 3.1).
 *  - Layout: row-major, contiguous.  Pointers to arrays read or written with 16-byte vectors
 *    (x, send, expert_out, y, weights) must be 16-byte aligned.
 *  - Synchrony: every call only enqueues work on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and returns.  No call synchronises with the host; the number of kept rows stays on the
 *    device (expert_offsets[E]).
 *  - Errors: the return value reports host-side argument validation (checked before anything is
 *    launched) and launch failures.  Errors found on the device (an expert id out of range, a
 *    pipeline wait that ran out) are recorded in a status word at the start of the workspace and
 *    reported by moe_sync_status.  Error names follow the NCCL EP page's error table (section 5.1:
 *    INVALID_TOPK for an out-of-range routing index, CUDA_ERROR for a failed launch).
 *  - Workspaces must be zero-filled once after allocation (cudaMemset); the calls keep them in a
 *    reusable state afterwards.  Calls that share one workspace must not overlap on the GPU.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* == cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer, k > E, E % R != 0 ... */
  MOE_ERR_INVALID_TOPK = 2, /* a routing index outside [0, E) (found on the device)               */
  MOE_ERR_UNSUPPORTED = 3,  /* valid but not implemented here (e.g. H % 64 != 0)                  */
  MOE_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed                               */
  MOE_ERR_WORKSPACE = 5,    /* workspace too small or not 256-byte aligned                        */
  MOE_ERR_TIMEOUT = 6,      /* a bounded device-side wait ran out; the kernel stopped early       */
  MOE_ERR_INVALID_COUNTS = 7 /* row counts (found on the device) do not fit the buffers they describe */
} moe_status_t;

typedef enum {
  MOE_PAYLOAD_BF16 = 0,         /* send rows are the token's bf16 bytes                             */
  MOE_PAYLOAD_FP8_E4M3_B128 = 1 /* send rows are e4m3 codes + one fp32 scale per 128 elements       */
} moe_payload_t;

/* Version of this interface (incremented on any incompatible change). */
int moe_abi_version(void);

/* Static, NUL-terminated description of a status code. */
const char* moe_status_string(moe_status_t status);

/*
 * Per-expert capacity C = ceil(cf * T * k / E), computed in double; cf <= 0 returns 0 (no limit).
 * Mean expert load is T*k/E ("大模型MoE稀疏激活原理与硬件适配实战", section 2.3: (B*S*K)/E with
 * the example 32*2048*2/128 = 1024).  Host function; returns -1 for T < 0, k < 1 or E < 1.
 */
int moe_capacity(double cf, int T, int k, int E);

/*
 * Router: per token, the k largest fp32 logits (ties -> lower expert id; NaN ranks below -inf),
 * in descending order, and their routing weights; the selection and the weights are fp32 ("大模型
 * MoE稀疏激活原理与硬件适配实战", section 3.2, fine ranking; section 5.3, scenario 3: router in FP32;
 * section 4.1: one token's experts are distinct).
 *   logits        fp32 [T, E]       router logits (any bias already added)
 *   renormalize   1: weights = softmax over the k selected logits (they sum to 1)
 *                 0: weights = the selected entries of the softmax over all E logits
 *   topk_idx      int32 [T, k]      out: expert ids, best first
 *   topk_w        fp32  [T, k]      out: routing weights, same order
 *   expert_routed int32 [E] or NULL out: number of tokens routed to each expert (overwritten)
 * Limits: 1 <= k <= E <= 1024, k <= 32, T >= 0 (T == 0 launches nothing but clears expert_routed).
 * Non-finite logits: the weights are the softmax's limits (NaN counts as -inf; +inf entries share
 * the mass; an all -inf denominator shares it equally).
 */
moe_status_t moe_route(const float* logits, int T, int E, int k, int renormalize,
                       int32_t* topk_idx, float* topk_w, int32_t* expert_routed,
                       moe_stream_t stream);

/* Bytes of scratch moe_dispatch needs for T tokens, E experts, k slots per token: a status word and
 * one expert histogram per chunk of 16 * floor(128 / k) tokens.  The caller allocates it (the NCCL
 * EP page, sections 1 and 3.1: the caller registers the memory a group or handle works in); returns
 * 0 for T < 0, E < 1 or k < 1. */
size_t moe_dispatch_workspace_size(int T, int E, int k);

/*
 * Dispatch: pack every kept (token, slot) into one contiguous expert-major send buffer (the
 * ThunderEP page, section 2.1, redundancy 1: all tokens bound for one destination in one buffer;
 * NCCL EP page, section 2.2: packed [sum T x H] high-throughput layout; section 2.1: expert-major
 * layout, FP8 payload with a scale tensor).
 *
 * Within an expert, rows are in ascending token order.  With capacity C > 0, a slot whose position
 * among its expert's slots (in token order) is >= C is dropped: slot_row = -1, no row is written.
 *   x              bf16 [T, H]              token activations
 *   topk_idx       int32 [T, k]             expert ids (each in [0, E))
 *   capacity       0 = keep every slot, else C (see moe_capacity)
 *   payload        MOE_PAYLOAD_BF16 or MOE_PAYLOAD_FP8_E4M3_B128 (needs H % 128 == 0)
 *   send           [T*k, H] bf16 or e4m3    out: rows 0 .. expert_offsets[E]-1 are written
 *   send_scales    fp32 [T*k, H/128]        out (FP8 only, else may be NULL): per-block scales,
 *                                           scale = amax/448 (1 if amax == 0), code =
 *                                           e4m3_rn_satfinite(x / scale), fp32 IEEE division
 *   expert_counts  int32 [E]                out: kept rows per expert
 *   expert_offsets int32 [E+1]              out: exclusive scan of expert_counts
 *   rank_offsets   int32 [R+1]              out: rank_offsets[r] = expert_offsets[r*E/R]
 *   slot_row       int32 [T, k]             out: packed row of each slot, -1 if dropped
 *   row_token      int32 [T*k]              out: token of each packed row (first S entries)
 *   ws, ws_bytes   device scratch >= moe_dispatch_workspace_size(T, E, k), 256-byte aligned,
 *                  zero-filled once after allocation
 * Limits: T*k < 2^31, 1 <= k <= E <= 1024, R >= 1, E % R == 0, H % 8 == 0, H >= 8.
 * An expert id outside [0, E) is not written anywhere: its slot gets slot_row = -1 and the status
 * word records MOE_ERR_INVALID_TOPK (reported by moe_sync_status).
 */
moe_status_t moe_dispatch(const void* x, int T, int H, const int32_t* topk_idx, int k, int E,
                          int R, int capacity, moe_payload_t payload, void* send,
                          float* send_scales, int32_t* expert_counts, int32_t* expert_offsets,
                          int32_t* rank_offsets, int32_t* slot_row, int32_t* row_token, void* ws,
                          size_t ws_bytes, moe_stream_t stream);

/*
 * moe_dispatch_noalloc: moe_dispatch for callers that cannot allocate.  The pages have no
 * counterpart; this is a convenience of this library.
 *
 * Some callers cannot hand the library a workspace: programs that route every device allocation
 * through their own pool and forbid others, plug-ins inside such programs, and latency-critical
 * code that must not call cudaMalloc (it can synchronise the whole device).  This entry point takes
 * the same inputs and outputs as moe_dispatch, without ws / ws_bytes, and calls no cudaMalloc,
 * cudaFree or allocating library routine.  Its scratch is a static device array of
 * MOE_DISPATCH_NOALLOC_SCRATCH_BYTES (1 MiB) inside the library, which every GPU that loads the
 * library holds until the process exits.
 *   status  optional (may be NULL) device int32 owned by the caller, zeroed by the caller: device
 *           findings are OR-ed into it (1 = expert id out of range); moe_sync_status(status, s)
 *           reads and clears it like a workspace status word.
 * Limits: those of moe_dispatch, plus 256 + ceil(T / C) * E * 4 <= 1 MiB, where C = 16 * floor(128 / k)
 * tokens (at least 16) is the counting chunk (e.g. T <= 261120 at E = 1024, k = 2; T <= 65280 at
 * E = 1024, k = 8); larger shapes return MOE_ERR_WORKSPACE without launching.
 * Every call looks up the array's device address in the current context (cudaGetSymbolAddress, no
 * allocation); the first call in a context may load the library's module there, so make that first
 * call before any stream capture.  All calls share the one
 * array: calls that overlap on the GPU (different streams, or the same array from several host
 * threads without ordering) race and give wrong results; order them on one stream.
 */
#define MOE_DISPATCH_NOALLOC_SCRATCH_BYTES (1u << 20)
moe_status_t moe_dispatch_noalloc(const void* x, int T, int H, const int32_t* topk_idx, int k,
                                  int E, int R, int capacity, moe_payload_t payload, void* send,
                                  float* send_scales, int32_t* expert_counts,
                                  int32_t* expert_offsets, int32_t* rank_offsets,
                                  int32_t* slot_row, int32_t* row_token, int32_t* status,
                                  moe_stream_t stream);

/* Bytes of scratch moe_expert_ffn needs: a status word, the bf16 intermediate h [max_rows, F], for
 * the FP8 payload the dequantised bf16 input rows [max_rows, H], and the int32 counters of the
 * tile pipeline (two per 128-row block plus two for each of the two run-time tile schedulers).  Caller-allocated
 * as for moe_dispatch_workspace_size (NCCL EP page, sections 1 and 3.1); `payload` is needed
 * because only the FP8 payload has the dequantised rows.  Returns 0 for invalid sizes. */
size_t moe_ffn_workspace_size(int max_rows, int E, int H, int F, moe_payload_t payload);

/*
 * Grouped SwiGLU expert FFN on the packed rows ("细粒度专家并行方案对比：MegaMoE与传统方案",
 * section 核心差异分析 1: two linear layers and SwiGLU per expert; "DWDP: 在NVL72上的高性能分布式权重
 * 数据并行", run_moe: fused w3_w1 first projection with SwiGLU, then w2).  For expert e and every
 * packed row x in [expert_offsets[e], expert_offsets[e+1]):
 *     h = bf16( silu(x . W_gate[e]^T) * (x . W_up[e]^T) ),  silu(g) = g * sigmoid(g)
 *     expert_out = bf16( h . W_down[e]^T )
 * with bf16 operands on the tensor cores and fp32 accumulation.  For the FP8 payload the input
 * row is first dequantised: x = bf16(fp32(q) * scale).  Experts with two or more 128-row blocks
 * run as 256-row tiles on pairs of SMs (2-CTA clusters), the others as 128-row tiles on one SM;
 * every output element is computed by one tile in a fixed k order, so results are reproducible.
 *   send           [max_rows, H] bf16 or e4m3 (rows past expert_offsets[E] are ignored)
 *   send_scales    fp32 [max_rows, H/128] (FP8 only, else NULL)
 *   expert_offsets int32 [E+1] device array (read on the device; no host sync)
 *   w_gate, w_up   bf16 [E, F, H], one contiguous block per expert
 *   w_down         bf16 [E, H, F]
 *   expert_out     bf16 [max_rows, H]       out: rows 0 .. expert_offsets[E]-1
 *   ws, ws_bytes   device scratch >= moe_ffn_workspace_size(...), 256-byte aligned, zero-filled once
 * Limits: H % 64 == 0, F % 64 == 0 (else MOE_ERR_UNSUPPORTED), E <= 1024,
 * expert_offsets[E] <= max_rows (rows beyond max_rows are not computed).
 * The workspace also holds per-row-block completion counters and the tile-claim counters of the
 * kernel's run-time tile scheduler, which every successful call leaves at zero; after a call that
 * reported MOE_ERR_TIMEOUT, zero-fill the workspace again before reuse.
 */
moe_status_t moe_expert_ffn(const void* send, const float* send_scales, moe_payload_t payload,
                            const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                            const void* w_gate, const void* w_up, const void* w_down,
                            void* expert_out, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Per-expert weight lists: experts whose weights live at separate addresses (each its own
 * allocation, e.g. local experts next to experts prefetched from elsewhere), consumed by the grouped
 * FFN without first copying them into one [E, ...] block ("DWDP: 在NVL72上的高性能分布式权重数据
 * 并行", sections 消除D2D时延开销 and 关键优化实施: the grouped GEMM takes a TensorList and picks
 * each expert's buffer inside the kernel, instead of merging split weights device to device).
 *
 * moe_ffn_weight_list_bytes: bytes of the device buffer moe_ffn_weight_list_init fills (four
 * 128-byte TMA descriptors per expert); 0 for E outside [1, 1024].
 *
 * moe_ffn_weight_list_init: set-up call, once per set of weight addresses.
 *   w_gate, w_up   HOST arrays of E device pointers, each bf16 [F, H] (16-byte aligned)
 *   w_down         HOST array of E device pointers, each bf16 [H, F]
 *   list           device buffer >= moe_ffn_weight_list_bytes(E), 64-byte aligned (caller-owned)
 * Enqueues a host-to-device copy on `stream` from pageable memory (the call returns once the host
 * data has been taken; it is not meant for stream capture).  The weights must stay at these
 * addresses while the list is used.  Limits: H % 64 == 0, F % 64 == 0, E <= 1024.
 *
 * moe_expert_ffn_list: moe_expert_ffn with the weights given by a list instead of three [E, ...]
 * arrays; same arguments otherwise, and the same results bit for bit (same tiles, same k order).
 */
size_t moe_ffn_weight_list_bytes(int E);
moe_status_t moe_ffn_weight_list_init(const void* const* w_gate, const void* const* w_up,
                                      const void* const* w_down, int E, int H, int F, void* list,
                                      moe_stream_t stream);
moe_status_t moe_expert_ffn_list(const void* send, const float* send_scales, moe_payload_t payload,
                                 const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                                 const void* list, void* expert_out, void* ws, size_t ws_bytes,
                                 moe_stream_t stream);

/*
 * FP8 expert weights for the first projection (W8A8), with the down projection kept in bf16.  The
 * DWDP page's expert weights are low-precision values with scales ("DWDP: 在NVL72上的高性能分布式
 * 权重数据并行", 关键优化实施: NvFp4WeightView's w3_w1 weights and their scale tensors); here the
 * gate and up weights are e4m3 with one fp32 scale per output row, and each FFN input row is
 * quantised on its own the same way, so g = sx * sw * sum(qx * qw) exactly factorises and the
 * tensor cores run tcgen05.mma kind::f8f6f4 on the codes.
 *
 * moe_quantize_rows_fp8: rows of bf16 x [rows, K] -> e4m3 codes [rows, K] and fp32 scales [rows]:
 *   scale = amax / 448 of the row (1 when amax == 0), code = e4m3 round-to-nearest-even, saturating,
 *   of the fp32 IEEE quotient x / scale (the rule of the FP8 payload, with the whole row as the
 *   block).  Set-up call for the weights (w_gate and w_up as [E*F, H]).  Limits: K % 16 == 0;
 *   x and codes 16-byte aligned.
 *
 * moe_ffn_w8_workspace_size / moe_expert_ffn_w8: moe_expert_ffn with
 *   w_gate_q, w_up_q      e4m3 codes [E, F, H] (16-byte aligned)
 *   w_gate_scale,
 *   w_up_scale            fp32 [E, F] (8-byte aligned): the rows' scales
 *   w_down                bf16 [E, H, F] as for moe_expert_ffn
 * and a workspace of moe_ffn_w8_workspace_size (it also holds the input rows' codes and scales).
 * For expert e and each packed row x (for the FP8 payload, its dequantised bf16 values):
 *   (qx, sx) = per-row FP8 of x;  g[f] = sx * sg[e,f] * sum_h qx[h] qg[e,f,h], u likewise (fp32
 *   accumulate);  h = bf16(silu(g) * u);  expert_out = bf16(h . W_down[e]^T).
 * Limits as for moe_expert_ffn.
 */
moe_status_t moe_quantize_rows_fp8(const void* x, int rows, int K, void* codes, float* scales,
                                   moe_stream_t stream);
size_t moe_ffn_w8_workspace_size(int max_rows, int E, int H, int F, moe_payload_t payload);
moe_status_t moe_expert_ffn_w8(const void* send, const float* send_scales, moe_payload_t payload,
                               const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                               const void* w_gate_q, const float* w_gate_scale,
                               const void* w_up_q, const float* w_up_scale, const void* w_down,
                               void* expert_out, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Combine: y[t] = bf16( sum_{j=0..k-1, slot_row[t,j] >= 0} topk_w[t,j] * expert_out[slot_row[t,j]] )
 * accumulated in fp32 in slot order j = 0, 1, ... with each product and sum rounded to fp32
 * separately (the NCCL EP page, section 2.1: the combine loops over the top-k slots and adds each
 * expert output times the token's routing weight).  A token whose slots were all dropped gives 0.
 *   expert_out bf16 [max_rows, H]; slot_row int32 [T, k]; topk_w fp32 [T, k]; y bf16 [T, H] (out)
 *   status     optional (may be NULL) device int32 status word (e.g. the first word of a dispatch
 *              or FFN workspace) for device-side findings, reported by moe_sync_status(status,
 *              stream); the current combine kernel has no device-side waits and never sets it
 * Rows outside [0, max_rows) are treated as dropped.  Limits: H % 8 == 0.
 */
moe_status_t moe_combine(const void* expert_out, int max_rows, const int32_t* slot_row,
                         const float* topk_w, int T, int k, int H, void* y, int32_t* status,
                         moe_stream_t stream);

/*
 * moe_backward: gradients of the layer for an output gradient dy, reusing the forward's routing and
 * plan (the NCCL EP page, section 3.2: the training step's backward dispatches the output gradient
 * through the forward's handle to the experts, runs them backward, and combines the gradients).
 *   1. combine backward, per kept slot (t, j) -> row: d_eo[row] = bf16(fp32(topk_w[t,j] * dy[t]))
 *      and d_topk_w[t,j] = <dy[t], expert_out[row]> (0 for a dropped slot);
 *   2. expert backward (tcgen05 GEMMs): g = x Wg^T, u = x Wu^T recomputed, dh = d_eo Wd,
 *      dg = bf16(dh u s (1 + g (1 - s))), du = bf16(dh g s) with s = sigmoid(g),
 *      dx_rows = bf16(dg Wg + du Wu), d_w_down = d_eo^T h, d_w_gate = dg^T x, d_w_up = du^T x
 *      (fp32 accumulation; h = bf16(g s u) as in the forward);
 *   3. dx[t] = bf16(sum over kept slots of dx_rows[slot_row[t,j]]), fp32 in slot order;
 *   4. d_logits [T,E]: with renormalize, for a selected expert i: w_i (d_w_i - sum_j w_j d_w_j), 0
 *      elsewhere; without, the full-E softmax backward p_e (d_e - sum p d) (logits needed).
 * Inputs from the forward: topk_idx, topk_w, slot_row, expert_offsets (moe_route / moe_dispatch;
 * a slot whose expert id lies outside [0, E), which moe_dispatch reports as MOE_ERR_INVALID_TOPK,
 * adds nothing to d_logits, a slot_row outside [0, max_rows) marks a dropped slot, and
 * expert_offsets are clamped to [0, max_rows]),
 * ffn_input = the FFN's input rows bf16 [max_rows, H] (the send buffer for the bf16 payload; the
 * dequantised rows of the FFN workspace for the FP8 payload), expert_out bf16 [max_rows, H]; the
 * weights as for moe_expert_ffn.  Outputs (device, caller-owned): dx bf16 [T,H], d_logits fp32
 * [T,E], d_topk_w fp32 [T,k], d_w_gate / d_w_up fp32 [E,F,H], d_w_down fp32 [E,H,F] (every element
 * written, zeros for experts without rows).  ws: moe_backward_workspace_size bytes, 256-byte
 * aligned; it holds [status | d_eo bf16 [max_rows,H] | h, dg, du bf16 [max_rows,F] | dx_rows bf16
 * [max_rows,H] | unit weights fp32 [T,k]], each part 256-byte aligned.
 * Limits: H % 64 == 0, F % 64 == 0 (MOE_ERR_UNSUPPORTED), k <= 32, E <= 1024, T*k <= max_rows.
 */
size_t moe_backward_workspace_size(int max_rows, int T, int k, int H, int F);
moe_status_t moe_backward(const void* dy, int T, int H, int k, int E, int F, const float* logits,
                          int renormalize, const int32_t* topk_idx, const float* topk_w,
                          const int32_t* slot_row, const int32_t* expert_offsets, int max_rows,
                          const void* ffn_input, const void* expert_out, const void* w_gate,
                          const void* w_up, const void* w_down, void* dx, float* d_logits,
                          float* d_topk_w, float* d_w_gate, float* d_w_up, float* d_w_down,
                          void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The two halves of moe_backward, for callers that move rows between them (expert parallelism):
 *   moe_combine_backward: step 1 of moe_backward on this rank's tokens: d_eo [max_rows, H] bf16 in
 *     the dispatch's row layout (rows of kept slots written), d_topk_w fp32 [T,k], d_logits fp32
 *     [T,E].  expert_out holds the expert outputs of this rank's slots in the same row layout.
 *   moe_expert_backward: step 2 on expert-major rows: ffn_input and d_eo bf16 [max_rows, H] laid
 *     out by expert_offsets [E+1] (the experts' rows in the order their forward used), dx_rows
 *     bf16 [max_rows, H] out, and the fp32 weight gradients of these E experts.  ws:
 *     moe_expert_backward_workspace_size(max_rows, F) bytes, 256-byte aligned, holding
 *     [status | h, dg, du bf16 [max_rows, F]]; device findings (a bounded wait that ran out) are
 *     read with moe_sync_status(ws).
 * moe_backward is exactly moe_combine_backward, moe_expert_backward and a moe_combine of dx_rows
 * with unit weights.  Limits as for moe_backward.
 */
moe_status_t moe_combine_backward(const void* dy, int T, int H, int k, int E, const float* logits,
                                  int renormalize, const int32_t* topk_idx, const float* topk_w,
                                  const int32_t* slot_row, int max_rows, const void* expert_out,
                                  void* d_eo, float* d_topk_w, float* d_logits,
                                  moe_stream_t stream);
size_t moe_expert_backward_workspace_size(int max_rows, int F);
moe_status_t moe_expert_backward(const void* ffn_input, const void* d_eo,
                                 const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                                 const void* w_gate, const void* w_up, const void* w_down,
                                 void* dx_rows, float* d_w_gate, float* d_w_up, float* d_w_down,
                                 void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_ep_regroup: the row moves on both sides of an expert-parallel all-to-all, as one segmented
 * copy.
 *
 * With expert parallelism over R ranks, rank r owns experts [r*E_loc, (r+1)*E_loc), E_loc = E/R.
 * A rank's moe_dispatch with that R leaves its send buffer destination-major (rank_offsets are the
 * send displacements) and, inside each destination's block, expert-major; expert_counts viewed as
 * [R, E_loc] counts the rows of every (destination, expert) segment.  After the exchange, the
 * receiver holds R source blocks, source s's block holding recv_counts[s][e] rows of each local
 * expert e in turn (the NCCL EP page, section 2.2: packed per-destination buffers in the
 * high-throughput mode, one [E x M x H] block per peer in the low-latency mode; the ThunderEP page,
 * section 2.1: one contiguous block per destination).  The grouped FFN wants those rows
 * expert-major, and the return trip wants them back in source-major order.
 *
 * counts [A, B] int32 (device, row-major) names A*B segments; segment (a, b) holds counts[a][b]
 * rows of row_bytes bytes.  Each side lays the segments out in one of two orders:
 *   order 0 (a-major): segment (a, b) follows (a, b-1); block a starts at row a*stride, or, with
 *                      stride 0, right after block a-1 (packed);
 *   order 1 (b-major): segment (a, b) follows (a-1, b); block b starts at row b*stride, or packed.
 * Row q of segment (a, b) moves from its src position to its dst position; rows of neither side
 * outside the segments are left untouched.  An optional second payload (src_aux / dst_aux,
 * aux_row_bytes per row, e.g. the FP8 block scales) moves with the same row map.
 *   receive side:  A = R sources, B = E_loc, src order 0 (stride 0, or the padded block rows),
 *                  dst order 1 packed, dst_offsets [E_loc + 1] gets the expert offsets for the FFN;
 *   return trip:   the same counts with src and dst swapped;
 *   low-latency padding of the send buffer: A = R destinations, B = E_loc, src order 0 packed,
 *                  dst order 0 with stride M (and back).
 * src_rows / dst_rows are the row capacities of the two buffers; a position outside them, a
 * negative count, or a block longer than its stride is not copied, and records
 * MOE_ERR_INVALID_COUNTS in *status (a word read by moe_sync_status, may be NULL): the counts come
 * from other ranks, so the device checks them.  dst_offsets (may be NULL) gets the packed b-major
 * start of every b and the total at [B].
 * Limits: A*B <= 4096; row_bytes and aux_row_bytes multiples of 4 (16-byte vectors when rows and
 * pointers allow); src != dst.  Asynchronous on `stream`.
 */
moe_status_t moe_ep_regroup(const int32_t* counts, int A, int B, int src_order, int src_stride,
                            int src_rows, int dst_order, int dst_stride, int dst_rows,
                            const void* src, void* dst, size_t row_bytes, const void* src_aux,
                            void* dst_aux, size_t aux_row_bytes, int32_t* dst_offsets,
                            int32_t* status, moe_stream_t stream);

/*
 * moe_ep_exchange: the expert-parallel exchange over peer memory, fused with the regrouping: one
 * kernel moves every row between this rank's expert-major buffer and the other ranks' packed
 * buffers, reading (pull) or writing (push) the other GPUs' memory directly over NVLink (the NCCL
 * EP page, section 1: kernels that load and store peer memory over NVLink in place of staged
 * copies; section 2.1: the dispatch writes each token into the expert owner's receive buffer and
 * the combine reads the outputs back).
 *
 * Rank `rank` of R owns experts [rank*E_loc, (rank+1)*E_loc), E_loc = E / R.  all_counts [R, E]
 * int32 (device, this rank's copy, e.g. from an all-gather) holds every rank's expert_counts from
 * its moe_dispatch; source s's packed expert-major buffer then holds the rows for this rank's
 * expert e from row  sum_{e' < rank*E_loc + e} all_counts[s][e']  on.  peer_rows [R] (device, 64-bit
 * addresses) holds the base of every rank's packed buffer as this GPU sees it (its own buffer for
 * s = rank, peer mappings for the others); peer_aux [R] likewise for the second payload (the FP8
 * block scales; NULL when aux_row_bytes is 0).
 *   MOE_EP_PULL: rows move from the sources' buffers into local_rows, expert-major over this rank's
 *                experts and, within an expert, source-major (packed); local_offsets [E_loc + 1]
 *                (may be NULL) gets the expert offsets for moe_expert_ffn;
 *   MOE_EP_PUSH: the reverse (local_rows expert-major into every source's buffer at the same
 *                positions), e.g. the FFN outputs into each source's combine input.  The kernel
 *                ends with a system-scope fence, so its stores are visible to the other GPUs once
 *                it has completed.
 * The caller orders the exchange against the other ranks: the sources' buffers must be complete
 * before a pull (e.g. a stream-ordered collective after every rank's dispatch) and the pushes of
 * every rank must be complete before a source reads its buffer.  peer_rows_cap / local_rows_cap are
 * the row capacities of every peer buffer and of local_rows; a negative count, or a block or total
 * that does not fit them, copies nothing and records MOE_ERR_INVALID_COUNTS in *status (may be
 * NULL).  Rows move with 16-byte vectors when sizes and addresses allow, else 4-byte words.
 * Limits: R <= 1024, E <= 4096, E % R == 0, row_bytes and aux_row_bytes multiples of 4.
 */
#define MOE_EP_PULL 0
#define MOE_EP_PUSH 1
moe_status_t moe_ep_exchange(const int32_t* all_counts, int R, int E, int rank, int direction,
                             const uint64_t* peer_rows, const uint64_t* peer_aux,
                             int peer_rows_cap, void* local_rows, void* local_aux,
                             int local_rows_cap, size_t row_bytes, size_t aux_row_bytes,
                             int32_t* local_offsets, int32_t* status, moe_stream_t stream);

/*
 * Synchronise `stream`, read the device status word at the start of a dispatch or FFN workspace
 * (or any status word given to moe_combine / moe_dispatch_noalloc), clear it, and report it:
 * MOE_OK, MOE_ERR_INVALID_TOPK, MOE_ERR_TIMEOUT or MOE_ERR_INVALID_COUNTS (MOE_ERR_CUDA if the
 * stream itself failed).
 * This is how device-side findings reach the host as the error codes of the NCCL EP page's table
 * ("NCCL EP架构解析", section 5.1: INVALID_TOPK for a routing index out of range, CUDA_ERROR for a
 * failed kernel).  It is the only call of the library that waits for the GPU.
 */
moe_status_t moe_sync_status(void* ws, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
