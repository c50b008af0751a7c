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
// into chunks of C tokens (C * k <= 2048 slots).
//   1. count: one CTA per chunk writes the chunk's expert histogram hist[chunk][E].
//   2. rank_permute: CTA b of G owns the tokens [T*b/G, T*(b+1)/G) (any length; a range may cross
//      chunk boundaries).  Before waiting for the count kernel (inputs only): L2 prefetch of the
//      rows its warps copy first, the per-expert count of the slots between the start of its first
//      token's chunk and its first token, and the warp-synchronous (__match_any) ranking of its
//      own slots in slot order, which continues that count.  After the wait: from hist, the slots
//      of every expert in the chunks before, the expert totals, the capacity and the scanned
//      expert offsets (CTA 0 also writes counts / offsets / rank offsets); then each slot's row
//      (position >= capacity: dropped, -1), slot_row / row_token, and the copy of the rows (bf16)
//      or their per-128-element e4m3 quantisation with an fp32 scale (FP8).  The CTA's token x
//      copy-unit space is split evenly over its warps, and each warp keeps an L2 prefetch one
//      token ahead of its copy.
#include <cuda_fp8.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// Tokens per chunk are 16 * floor(128 / k), so a chunk holds at most kChunkSlotsMax slots.
constexpr int kChunkSlotsMax = 2048;
constexpr int kPerThread = kChunkSlotsMax / kThreads;
// Launch shape of rank_permute (measured on B200): one wave of kCtasPerSm CTAs per SM while that
// leaves at most kPersistMax tokens per CTA, else CTAs of kTokensPerCta tokens (many short CTAs
// pace the L2 prefetch of large inputs better than long-lived ones); never fewer CTAs than
// min(T, kCtasPerSm * SMs).
constexpr int kCtasPerSm = 3;
constexpr int kPersistMaxBf16 = 12, kPersistMaxFp8 = 1;
constexpr int kTokensPerCta = 8;
constexpr int kPrefetchDepth = 1;  // tokens of a warp's share prefetched ahead of its copy
constexpr int kUnrollBf16 = 8, kUnrollFp8 = 2;  // 16-byte loads in flight per lane per step

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
  // a chunk holds at most kChunkSlotsMax slots: every load is issued before the first atomic
  int ev[kPerThread];
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const long long s = s0 + tid + i * kThreads;
    ev[i] = s < s1 ? __ldg(topk_idx + s) : 0;
  }
  bool bad = false;
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    if (s0 + tid + i * kThreads < s1) {
      const bool ok = static_cast<unsigned>(ev[i]) < static_cast<unsigned>(E);
      hist_add(s_hist, ev[i], ok);
      bad |= !ok;
    }
  }
  if (__syncthreads_or(bad) && tid == 0) record_status(status, kStatusInvalidTopk);
  for (int e = tid; e < E; e += kThreads) hist[static_cast<size_t>(c) * E + e] = s_hist[e];
}

// Warp 0 ranks slots [q0, q1) in slot order: s_rel[i] = running count of the slot's expert before
// it (cnt[e] on entry counts the earlier slots), s_exp[i] = its expert or -1; cnt is advanced.
__device__ __forceinline__ void rank_slots(const int32_t* __restrict__ topk_idx, long long q0,
                                           long long q1, int E, int* cnt, int* s_rel,
                                           int* s_exp) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  int e_next = q0 + lane < q1 ? __ldg(topk_idx + q0 + lane) : -1;
  for (long long base = q0; base < q1; base += 32) {
    const long long s = base + lane;
    const bool valid = s < q1;
    const int e = e_next;
    e_next = s + 32 < q1 ? __ldg(topk_idx + s + 32) : -1;  // next round's load in flight
    const bool ok = valid && static_cast<unsigned>(e) < static_cast<unsigned>(E);
    const int key = ok ? e : E + lane;  // unique key for lanes without a slot
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
    int rel = -1;
    if (ok) rel = cnt[e] + __popc(peers & lt_mask);
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) cnt[e] += __popc(peers);
    __syncwarp();
    if (valid) {
      s_rel[s - q0] = rel;
      s_exp[s - q0] = ok ? e : -1;
    }
  }
}

// The contiguous share [ubeg, uend) of n_units copy units taken by `warp`, in multiples of gran.
__device__ __forceinline__ void warp_share(int n_units, int gran, int warp, int& ubeg, int& uend) {
  const int per = ((n_units + kWarps - 1) / kWarps + gran - 1) / gran * gran;
  ubeg = min(n_units, warp * per);
  uend = min(n_units, ubeg + per);
}

// L2 prefetch of the part of token (ub / upr + j) that lies in the unit range [ub, ue) of the token
// range starting at token tb (nothing when that part is empty).
template <int kUnitElems>
__device__ __forceinline__ void prefetch_share_token(const uint4* x, int tb, int H, int upr, int ub,
                                                     int ue, int j) {
  if (ub >= ue) return;
  const int tt = ub / upr + j;
  const int a = max(ub, tt * upr), b = min(ue, (tt + 1) * upr);
  if (a >= b) return;
  const char* p = reinterpret_cast<const char*>(x) +
                  (static_cast<size_t>(tb + tt) * H + static_cast<size_t>(a - tt * upr) * kUnitElems) * 2;
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"((b - a) * kUnitElems * 2)
               : "memory");
}

// Rank + permute.  CTA b of G owns the tokens [T*b/G, T*(b+1)/G), at most ceil(T/G) of them (the
// launcher sizes the per-slot shared arrays for that).  A copy unit is a 16-byte vector (bf16) or a
// 128-element block (FP8); the CTA's token x unit space is split evenly over the warps, so a warp
// may finish one token and start the next.
template <bool FP8, int UNROLL>
__global__ void __launch_bounds__(kThreads)
    rank_permute_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int E, int R, int cap,
                        int chunk_tokens, int n_chunks, const int32_t* __restrict__ hist,
                        int32_t* __restrict__ expert_counts, int32_t* __restrict__ expert_offsets,
                        int32_t* __restrict__ rank_offsets, int32_t* __restrict__ slot_row,
                        int32_t* __restrict__ row_token, const uint4* __restrict__ x, int H,
                        void* __restrict__ send, float* __restrict__ send_scales, int max_slots) {
  extern __shared__ int s_mem[];
  int* cnt = s_mem;                            // [E] slots of expert e from the chunk start on
  int* s_base = cnt + E;                       // [E] slots of expert e in earlier chunks
  int* s_off = s_base + E;                     // [max(E, 4*kThreads)] kept counts -> offsets
  int* s_rel = s_off + max(E, 4 * kThreads);   // [ceil(T/G)*k] relative position, then row
  int* s_exp = s_rel + max_slots;              // [ceil(T/G)*k] expert per slot (or -1)
  __shared__ int s_warp_tot[kWarps + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = static_cast<int>(static_cast<long long>(T) * blockIdx.x / gridDim.x);
  const int t1 = static_cast<int>(static_cast<long long>(T) * (blockIdx.x + 1) / gridDim.x);
  const int c = t0 / chunk_tokens;
  constexpr int kUnitElems = FP8 ? 128 : 8;
  constexpr int kGran = FP8 ? 2 : 32;  // units one warp step covers per lane group
  const int upr = H / kUnitElems;      // copy units per row

  // ---- before the wait: inputs only ---------------------------------------------------------------
  {
    // L2 prefetch of the first kPrefetchDepth tokens of each warp's share
    int ub, ue;
    warp_share((t1 - t0) * upr, kGran, warp, ub, ue);
    if (lane < kPrefetchDepth) prefetch_share_token<kUnitElems>(x, t0, H, upr, ub, ue, lane);
  }
  for (int e = tid; e < E; e += kThreads) cnt[e] = 0;
  __syncthreads();
  {
    // slots of the chunk before t0 (at most kChunkSlotsMax): loads first, then the atomics
    const long long pc0 = static_cast<long long>(c) * chunk_tokens * k;
    const long long p1 = static_cast<long long>(t0) * k;
    int ev[kPerThread];
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      const long long s = pc0 + tid + i * kThreads;
      ev[i] = s < p1 ? __ldg(topk_idx + s) : -1;
    }
#pragma unroll
    for (int i = 0; i < kPerThread; ++i)
      hist_add(cnt, ev[i], static_cast<unsigned>(ev[i]) < static_cast<unsigned>(E));
  }
  __syncthreads();
  if (warp == 0)
    rank_slots(topk_idx, static_cast<long long>(t0) * k, static_cast<long long>(t1) * k, E, cnt,
               s_rel, s_exp);

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
    s_base[e] = before;
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

  const long long q0 = static_cast<long long>(t0) * k;
  const int n_slots = (t1 - t0) * k;
  for (int i = tid; i < n_slots; i += kThreads) {
    const int e = s_exp[i];
    int row = -1;
    if (e >= 0) {
      const int pos = s_base[e] + s_rel[i];
      if (cap == 0 || pos < cap) {
        row = s_off[e] + pos;
        row_token[row] = t0 + i / k;
      }
    }
    slot_row[q0 + i] = row;
    s_rel[i] = row;
  }
  __syncthreads();
  int ub, ue;
  warp_share((t1 - t0) * upr, kGran, warp, ub, ue);
  for (int u = ub; u < ue;) {
    const int tt = u / upr, a = u - tt * upr, b = min(upr, a + (ue - u));
    const int t = t0 + tt;
    // keep the prefetch kPrefetchDepth tokens of the share ahead of the copy
    if (lane == 0)
      prefetch_share_token<kUnitElems>(x, t0, H, upr, ub, ue, tt - ub / upr + kPrefetchDepth);
    const int my_row = lane < k ? s_rel[tt * k + lane] : -1;
    if (FP8)
      quant_token_fp8<UNROLL>(x + static_cast<size_t>(t) * (H / 8), H, a, b, my_row,
                              static_cast<uint8_t*>(send), send_scales);
    else
      copy_token_bf16<UNROLL>(x + static_cast<size_t>(t) * (H / 8), H / 8, a, b, my_row,
                              static_cast<uint4*>(send));
    u += b - a;
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
  const long long resident = static_cast<long long>(kCtasPerSm) * num_sms();
  long long grid_ll = T < resident ? T : resident;
  if (T > grid_ll * (fp8 ? kPersistMaxFp8 : kPersistMaxBf16))
    grid_ll = std::max(grid_ll, (static_cast<long long>(T) + kTokensPerCta - 1) / kTokensPerCta);
  const int grid = static_cast<int>(grid_ll);
  const int max_slots = static_cast<int>((T + grid_ll - 1) / grid_ll) * k;  // <= 12 * 32
  const int scan_n = E > 4 * kThreads ? E : 4 * kThreads;
  const size_t smem = sizeof(int) * (2 * E + scan_n + 2 * static_cast<size_t>(max_slots));
  const uint4* xv = static_cast<const uint4*>(x);
  auto kern = fp8 ? rank_permute_kernel<true, kUnrollFp8> : rank_permute_kernel<false, kUnrollBf16>;
  err = launch_pdl(kern, dim3(grid), dim3(kThreads), smem, s, topk_idx, T, k, E, R, capacity,
                   chunk_tokens, n_chunks, static_cast<const int32_t*>(hist), expert_counts,
                   expert_offsets, rank_offsets, slot_row, row_token, xv, H, send, send_scales,
                   max_slots);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace moe
