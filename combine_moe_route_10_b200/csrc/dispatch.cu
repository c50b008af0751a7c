// Dispatch: deterministic expert-major packing of every kept (token, slot) into one send buffer.
//
// Sender-side merge of everything bound for one destination into one contiguous buffer is the
// ThunderEP page's section 2.1 (redundancy 1); the packed [sum T x H] layout is the NCCL EP page's
// section 2.2 (high-throughput mode), expert-major for the expert compute (its section 2.1), with
// the FP8 payload and its scale tensor from the same section.  Each emulated rank owns a contiguous
// expert range, so the buffer is rank-major too and a rank's slice is given by rank_offsets (the
// ThunderEP page's section 2.2: each rank keeps only its own slice of the routing table).
//
// Two kernels, no host synchronisation, no order-dependent atomics in any result.  Slots are cut
// into chunks of C tokens (about 2048 slots per chunk).
//   1. count: one CTA per chunk writes the chunk's expert histogram hist[chunk][E].
//   2. rank_permute: one CTA per `tile` tokens.  Before waiting for the count kernel (inputs only):
//      L2 prefetch of its token rows, the per-expert count of the chunk's slots before its first
//      token, and the warp-synchronous (__match_any) ranking of its own slots, giving each slot its
//      position relative to the chunk start.  After the wait: from hist, every CTA derives its
//      chunk's base position per expert and the expert totals, applies the capacity, scans the kept
//      counts into expert offsets (CTA 0 also writes counts / offsets / rank offsets), turns
//      positions into rows (position >= capacity: dropped, -1), writes slot_row / row_token, and
//      copies the rows (bf16) or quantises them per 128-element block to e4m3 with an fp32 scale
//      (FP8), one warp (or a segment of a row per warp) per token.
#include <cuda_fp8.h>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Add 1 to hist[e] for a valid expert id (shared-memory atomics: counts are order-independent).
__device__ __forceinline__ void hist_add(int* hist, int e, bool ok) {
  if (ok) atomicAdd(&hist[e], 1);
}

// Exclusive scan of n <= 4*kThreads ints in shared memory; returns the total.  All threads call.
__device__ int block_exclusive_scan(int* data, int n, int* warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int v[4];
  int local = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = tid * 4 + i;
    v[i] = idx < n ? data[idx] : 0;
    local += v[i];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int w = 0; w < kWarps; ++w) {
      const int t = warp_tot[w];
      warp_tot[w] = run;
      run += t;
    }
    warp_tot[kWarps] = run;
  }
  __syncthreads();
  int run = warp_tot[warp] + incl - local;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = tid * 4 + i;
    if (idx < n) data[idx] = run;
    run += v[i];
  }
  const int total = warp_tot[kWarps];
  __syncthreads();
  return total;
}

// bf16 payload of one token: the warp reads the row once (UNROLL 16-byte vectors in flight per
// lane) and writes it to each kept row.
template <int UNROLL>
__device__ __forceinline__ void copy_token_bf16(const uint4* __restrict__ src, int nvec, int vbeg,
                                                int vend, int my_row, uint4* __restrict__ send) {
  const int lane = threadIdx.x & 31;
  const unsigned keep = __ballot_sync(0xFFFFFFFFu, my_row >= 0);
  for (int v0 = vbeg; v0 < vend; v0 += 32 * UNROLL) {
    uint4 buf[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < vend) buf[u] = ld_nc_v4(src + v);
    }
    for (unsigned m = keep; m != 0; m &= m - 1) {
      const int row = __shfl_sync(0xFFFFFFFFu, my_row, __ffs(m) - 1);
      uint4* dst = send + static_cast<size_t>(row) * nvec;
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < vend) st_cs_v4(dst + v, buf[u]);  // streaming: evict-first in L2
      }
    }
  }
}

// FP8 payload of one token: each half-warp quantises one 128-element block per step.
// scale = amax / 448 (1 when amax == 0); code = e4m3 round-to-nearest-even, saturating, of the fp32
// IEEE quotient x / scale.
template <int UNROLL>
__device__ __forceinline__ void quant_token_fp8(const uint4* __restrict__ src, int H, int bbeg,
                                                int nblk, int my_row, uint8_t* __restrict__ send,
                                                float* __restrict__ send_scales) {
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4, hl = lane & 15;
  const int nblk_row = H / 128;
  const unsigned keep = __ballot_sync(0xFFFFFFFFu, my_row >= 0);
  for (int b0 = bbeg; b0 < nblk; b0 += 2 * UNROLL) {
    uint4 raw[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int b = b0 + 2 * u + half;
      if (b < nblk) raw[u] = ld_nc_v4(src + b * 16 + hl);
    }
    uint2 q[UNROLL];
    float scale[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int b = b0 + 2 * u + half;
      float f[8];
      const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16_lo(w[i]);
        f[2 * i + 1] = bf16_hi(w[i]);
      }
      float amax = 0.0f;
      if (b < nblk) {
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      const float sc = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
      scale[u] = sc;
      uint32_t packed[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 pr = make_float2(__fdiv_rn(f[2 * i], sc), __fdiv_rn(f[2 * i + 1], sc));
        packed[i] = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3));
      }
      q[u] = make_uint2(packed[0] | (packed[1] << 16), packed[2] | (packed[3] << 16));
    }
    for (unsigned m = keep; m != 0; m &= m - 1) {
      const int row = __shfl_sync(0xFFFFFFFFu, my_row, __ffs(m) - 1);
      uint8_t* dst = send + static_cast<size_t>(row) * H;
      float* dsc = send_scales + static_cast<size_t>(row) * nblk_row;
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int b = b0 + 2 * u + half;
        if (b < nblk) {
          *reinterpret_cast<uint2*>(dst + b * 128 + hl * 8) = q[u];
          if (hl == 0) dsc[b] = scale[u];
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads)
    count_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int E, int chunk_tokens,
                 int* status, int32_t* __restrict__ hist) {
  extern __shared__ int s_hist[];
  const int tid = threadIdx.x;
  const int c = blockIdx.x;
  for (int e = tid; e < E; e += kThreads) s_hist[e] = 0;
  griddep_wait();
  // rank_permute may start now: its pre-wait phase reads only the dispatch inputs, which are
  // complete once every CTA of this grid has passed the wait above
  griddep_launch_dependents();
  __syncthreads();
  const long long s0 = static_cast<long long>(c) * chunk_tokens * k;
  const long long s1 = static_cast<long long>(min(T, (c + 1) * chunk_tokens)) * k;
  bool bad = false;
  for (long long s = s0 + tid; s < s1; s += kThreads) {
    const int e = __ldg(topk_idx + s);
    const bool ok = static_cast<unsigned>(e) < static_cast<unsigned>(E);
    hist_add(s_hist, e, ok);
    bad |= !ok;
  }
  if (__syncthreads_or(bad) && tid == 0) record_status(status, kStatusInvalidTopk);
  for (int e = tid; e < E; e += kThreads) hist[static_cast<size_t>(c) * E + e] = s_hist[e];
}

template <bool FP8, int UNROLL>
__global__ void __launch_bounds__(kThreads)
    rank_permute_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int E, int R, int cap,
                        int chunk_tokens, int n_chunks, const int32_t* __restrict__ hist,
                        int32_t* __restrict__ expert_counts, int32_t* __restrict__ expert_offsets,
                        int32_t* __restrict__ rank_offsets, int32_t* __restrict__ slot_row,
                        int32_t* __restrict__ row_token, const uint4* __restrict__ x, int H,
                        int tile, void* __restrict__ send, float* __restrict__ send_scales) {
  extern __shared__ int s_mem[];
  int* cnt = s_mem;               // [E] relative positions, then chunk base + relative count
  int* s_off = cnt + E;           // [max(E, 4*kThreads)] kept counts, scanned into offsets
  int* s_rel = s_off + max(E, 4 * kThreads);  // [tile*k] relative position (or -1) per slot
  int* s_exp = s_rel + tile * k;  // [tile*k] expert per slot
  __shared__ int s_warp_tot[kWarps + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * tile;
  const int t1 = min(T, t0 + tile);
  const int c = t0 / chunk_tokens;

  // ---- before the wait: inputs only ---------------------------------------------------------------
  if (tid < t1 - t0) {
    const char* row = reinterpret_cast<const char*>(x) + static_cast<size_t>(t0 + tid) * H * 2;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(row), "r"(H * 2) : "memory");
  }
  for (int e = tid; e < E; e += kThreads) cnt[e] = 0;
  __syncthreads();
  const long long p1 = static_cast<long long>(t0) * k;
  for (long long s = static_cast<long long>(c) * chunk_tokens * k + tid; s < p1; s += kThreads) {
    const int e = __ldg(topk_idx + s);
    hist_add(cnt, e, static_cast<unsigned>(e) < static_cast<unsigned>(E));
  }
  __syncthreads();
  if (warp == 0) {
    const unsigned lt_mask = (1u << lane) - 1u;
    const long long q1 = static_cast<long long>(t1) * k;
    for (long long base = p1; base < q1; base += 32) {
      const long long s = base + lane;
      const bool valid = s < q1;
      const int e = valid ? __ldg(topk_idx + s) : -1;
      const bool ok = valid && static_cast<unsigned>(e) < static_cast<unsigned>(E);
      const int key = ok ? e : E + lane;  // unique key for lanes without a slot
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
      int rel = -1;
      if (ok) rel = cnt[e] + __popc(peers & lt_mask);
      __syncwarp();
      if (ok && lane == __ffs(peers) - 1) cnt[e] += __popc(peers);
      __syncwarp();
      if (valid) {
        s_rel[s - p1] = rel;
        s_exp[s - p1] = ok ? e : -1;
      }
    }
  }

  // ---- after the wait: the histogram is complete ---------------------------------------------------
  griddep_wait();
  griddep_launch_dependents();
  __syncthreads();
  for (int e = tid; e < E; e += kThreads) {
    int before = 0, total = 0;
#pragma unroll 8
    for (int cc = 0; cc < n_chunks; ++cc) {
      const int v = __ldcg(hist + static_cast<size_t>(cc) * E + e);
      total += v;
      before += cc < c ? v : 0;
    }
    cnt[e] = before;                                // positions of expert e before this chunk
    s_off[e] = cap > 0 ? min(total, cap) : total;   // kept rows of expert e
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = tid; e < E; e += kThreads) expert_counts[e] = s_off[e];
  const int total_kept = block_exclusive_scan(s_off, E, s_warp_tot);
  if (blockIdx.x == 0) {
    for (int e = tid; e < E; e += kThreads) expert_offsets[e] = s_off[e];
    if (tid == 0) expert_offsets[E] = total_kept;
    const int per_rank = E / R;
    for (int r = tid; r <= R; r += kThreads)
      rank_offsets[r] = (r == R) ? total_kept : s_off[r * per_rank];
  }
  const int n_slots = (t1 - t0) * k;
  for (int i = tid; i < n_slots; i += kThreads) {
    const int e = s_exp[i];
    int row = -1;
    if (e >= 0) {
      const int pos = cnt[e] + s_rel[i];
      if (cap == 0 || pos < cap) {
        row = s_off[e] + pos;
        row_token[row] = t0 + i / k;
      }
    }
    slot_row[p1 + i] = row;
    s_rel[i] = row;
  }
  __syncthreads();

  // warps per token: 1 when tile >= 8, else 8/tile warps split the row into segments
  const int wpt = tile >= kWarps ? 1 : kWarps / tile;
  const int seg = warp % wpt;
  const int units = FP8 ? H / 128 : H / 8;                 // 128-element blocks or 16-B vectors
  const int per = ((units + wpt - 1) / wpt + (FP8 ? 1 : 31)) / (FP8 ? 2 : 32) * (FP8 ? 2 : 32);
  const int ubeg = min(units, seg * per), uend = min(units, ubeg + per);
  for (int t = t0 + warp / wpt; t < t1; t += kWarps / wpt) {
    const int my_row = lane < k ? s_rel[(t - t0) * k + lane] : -1;
    if (FP8)
      quant_token_fp8<UNROLL>(x + static_cast<size_t>(t) * (H / 8), H, ubeg, uend, my_row,
                              static_cast<uint8_t*>(send), send_scales);
    else
      copy_token_bf16<UNROLL>(x + static_cast<size_t>(t) * (H / 8), H / 8, ubeg, uend, my_row,
                              static_cast<uint4*>(send));
  }
}

}  // namespace

int dispatch_chunk_tokens(int k) {
  const int c = 16 * (128 / k);
  return c < 16 ? 16 : c;
}

size_t dispatch_workspace_bytes(int T, int E, int k) {
  const size_t ct = static_cast<size_t>(dispatch_chunk_tokens(k));
  const size_t n_chunks = (static_cast<size_t>(T) + ct - 1) / ct;
  const size_t tab = (n_chunks > 0 ? n_chunks : 1) * static_cast<size_t>(E) * sizeof(int32_t);
  return 256 + (tab + 255) / 256 * 256;
}

cudaError_t launch_dispatch(const void* x, int T, int H, const int32_t* topk_idx, int k, int E,
                            int R, int capacity, int fp8, void* send, float* send_scales,
                            int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_offsets,
                            int32_t* slot_row, int32_t* row_token, void* ws, cudaStream_t s) {
  char* base = static_cast<char*>(ws);
  return launch_dispatch_parts(x, T, H, topk_idx, k, E, R, capacity, fp8, send, send_scales,
                               expert_counts, expert_offsets, rank_offsets, slot_row, row_token,
                               reinterpret_cast<int*>(base), reinterpret_cast<int32_t*>(base + 256),
                               s);
}

cudaError_t launch_dispatch_parts(const void* x, int T, int H, const int32_t* topk_idx, int k,
                                  int E, int R, int capacity, int fp8, void* send,
                                  float* send_scales, int32_t* expert_counts,
                                  int32_t* expert_offsets, int32_t* rank_offsets,
                                  int32_t* slot_row, int32_t* row_token, int* status,
                                  int32_t* hist, cudaStream_t s) {
  if (T == 0) {
    // nothing routed: zero counts and offsets
    cudaError_t e1 = cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * E, s);
    if (e1 != cudaSuccess) return e1;
    e1 = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), s);
    if (e1 != cudaSuccess) return e1;
    return cudaMemsetAsync(rank_offsets, 0, sizeof(int32_t) * (R + 1), s);
  }
  const int chunk_tokens = dispatch_chunk_tokens(k);
  const int n_chunks = (T + chunk_tokens - 1) / chunk_tokens;
  cudaError_t err = launch_pdl(count_kernel, dim3(n_chunks), dim3(kThreads), sizeof(int) * E, s,
                               topk_idx, T, k, E, chunk_tokens, status, hist);
  if (err != cudaSuccess) return err;
  // tokens per rank+permute CTA: about four CTAs per SM, at most 16
  int tile = 1;
  while (tile < kDispatchTileMax && (T + 2 * tile - 1) / (2 * tile) >= 4 * num_sms()) tile *= 2;
  const int tiles = (T + tile - 1) / tile;
  const int scan_n = E > 4 * kThreads ? E : 4 * kThreads;
  const size_t smem = sizeof(int) * (E + scan_n + 2 * tile * k);
  const uint4* xv = static_cast<const uint4*>(x);
  auto kern = fp8 ? rank_permute_kernel<true, 2> : rank_permute_kernel<false, 8>;
  err = launch_pdl(kern, dim3(tiles), dim3(kThreads), smem, s, topk_idx, T, k, E, R, capacity,
                   chunk_tokens, n_chunks, static_cast<const int32_t*>(hist), expert_counts,
                   expert_offsets, rank_offsets, slot_row, row_token, xv, H, tile, send,
                   send_scales);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace moe
