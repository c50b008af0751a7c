// Dispatch: deterministic expert-major packing of every kept (token, slot) into one send buffer.
//
// Sender-side merge of everything bound for one destination into one contiguous buffer is the
// ThunderEP page's section 2.1 (redundancy 1); the packed [sum T x H] layout is the NCCL EP page's
// section 2.2 (high-throughput mode), expert-major for the expert compute (its section 2.1), with
// the FP8 payload and its scale tensor from the same section.  Each emulated rank owns a contiguous
// expert range, so the buffer is rank-major too and a rank's slice is given by rank_offsets (the
// ThunderEP page's section 2.2: each rank keeps only its own slice of the routing table).
//
// Three kernels, no host synchronisation, no order-dependent atomics in any result:
//   1. count_scan: one CTA per 256-token chunk builds the chunk's expert histogram; the last CTA to
//      arrive turns the [chunk][expert] table into per-chunk base positions and writes the kept
//      counts (capacity applied), the expert offsets and the rank offsets.
//   2. rank: one CTA per chunk gives every slot its position inside its expert, in token order
//      (per-warp histograms, then warp-synchronous __match_any ranking), and writes slot_row and
//      row_token; slots at positions >= capacity are dropped (-1).
//   3. permute: one warp per token reads the row once with 16-byte loads and writes it to each of
//      its kept rows (bf16), or quantises it per 128-element block to e4m3 with an fp32 scale and
//      writes codes and scales to each kept row (FP8).
#include <cuda_fp8.h>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

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

__global__ void __launch_bounds__(kThreads)
    count_scan_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int E, int R, int cap,
                      int* status, unsigned* arrivals, int32_t* chunk_tab,
                      int32_t* __restrict__ expert_counts, int32_t* __restrict__ expert_offsets,
                      int32_t* __restrict__ rank_offsets) {
  extern __shared__ int s_hist[];  // E (+ padding to 4*kThreads for the scan)
  __shared__ int s_warp_tot[kWarps + 1];
  __shared__ bool s_last;
  const int tid = threadIdx.x;
  const int c = blockIdx.x;
  for (int e = tid; e < E; e += kThreads) s_hist[e] = 0;
  __syncthreads();
  const long long s0 = static_cast<long long>(c) * kDispatchChunk * k;
  const long long s1 = static_cast<long long>(min(T, (c + 1) * kDispatchChunk)) * k;
  bool bad = false;
  for (long long s = s0 + tid; s < s1; s += kThreads) {
    const int e = __ldg(topk_idx + s);
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E))
      atomicAdd(&s_hist[e], 1);
    else
      bad = true;
  }
  if (__syncthreads_or(bad) && tid == 0) record_status(status, kStatusInvalidTopk);
  for (int e = tid; e < E; e += kThreads) chunk_tab[static_cast<size_t>(c) * E + e] = s_hist[e];
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(arrivals, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // Last CTA: per-chunk base positions (exclusive over chunks, in place) and expert totals.
  const int n_chunks = gridDim.x;
  for (int e = tid; e < E; e += kThreads) {
    int run = 0;
    for (int cc = 0; cc < n_chunks; ++cc) {
      int32_t* p = chunk_tab + static_cast<size_t>(cc) * E + e;
      const int v = __ldcg(p);
      *p = run;
      run += v;
    }
    const int kept = cap > 0 ? min(run, cap) : run;
    expert_counts[e] = kept;
    s_hist[e] = kept;
  }
  __syncthreads();
  const int total = block_exclusive_scan(s_hist, E, s_warp_tot);
  for (int e = tid; e < E; e += kThreads) expert_offsets[e] = s_hist[e];
  if (tid == 0) expert_offsets[E] = total;
  const int per_rank = E / R;
  for (int r = tid; r <= R; r += kThreads) rank_offsets[r] = (r == R) ? total : s_hist[r * per_rank];
  if (tid == 0) *arrivals = 0u;  // every CTA has arrived: ready for the next call
}

__global__ void __launch_bounds__(kThreads)
    rank_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int E, int cap,
                const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ expert_offsets,
                int32_t* __restrict__ slot_row, int32_t* __restrict__ row_token) {
  extern __shared__ int s_whist[];  // [kWarps][E]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x;
  const long long s0 = static_cast<long long>(c) * kDispatchChunk * k;
  const long long s1 = static_cast<long long>(min(T, (c + 1) * kDispatchChunk)) * k;
  // each warp owns a contiguous, 32-aligned sub-range of the chunk's slots
  const long long n = s1 - s0;
  const long long per_warp = ((n + kWarps - 1) / kWarps + 31) / 32 * 32;
  const long long w0 = s0 + warp * per_warp;
  const long long w1 = min(s1, w0 + per_warp);
  int* my_hist = s_whist + warp * E;

  for (int i = tid; i < kWarps * E; i += kThreads) s_whist[i] = 0;
  __syncthreads();
  for (long long s = w0 + lane; s < w1; s += 32) {
    const int e = __ldg(topk_idx + s);
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicAdd(&my_hist[e], 1);
  }
  __syncthreads();
  for (int e = tid; e < E; e += kThreads) {
    int run = __ldg(chunk_base + static_cast<size_t>(c) * E + e);
    for (int w = 0; w < kWarps; ++w) {
      const int v = s_whist[w * E + e];
      s_whist[w * E + e] = run;
      run += v;
    }
  }
  __syncthreads();

  const unsigned lt_mask = (1u << lane) - 1u;
  for (long long base = w0; base < w1; base += 32) {
    const long long s = base + lane;
    const bool valid = s < w1;
    const int e = valid ? __ldg(topk_idx + s) : -1;
    const bool ok = valid && static_cast<unsigned>(e) < static_cast<unsigned>(E);
    const int key = ok ? e : E + lane;  // unique key for lanes without a slot
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
    int pos = 0;
    if (ok) pos = my_hist[e] + __popc(peers & lt_mask);
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) my_hist[e] += __popc(peers);
    __syncwarp();
    if (valid) {
      int row = -1;
      if (ok && (cap == 0 || pos < cap)) {
        row = __ldg(expert_offsets + e) + pos;
        row_token[row] = static_cast<int32_t>(s / k);
      }
      slot_row[s] = row;
    }
  }
}

// bf16 payload: one warp per token, UNROLL 16-byte vectors in flight per lane.
template <int UNROLL>
__global__ void __launch_bounds__(kThreads)
    permute_bf16_kernel(const uint4* __restrict__ x, int T, int nvec, int k,
                        const int32_t* __restrict__ slot_row, uint4* __restrict__ send) {
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kWarps;
  for (int t = blockIdx.x * kWarps + (threadIdx.x >> 5); t < T; t += nwarps) {
    const int my_row = lane < k ? __ldg(slot_row + static_cast<size_t>(t) * k + lane) : -1;
    const unsigned keep = __ballot_sync(0xFFFFFFFFu, my_row >= 0);
    const uint4* src = x + static_cast<size_t>(t) * nvec;
    for (int v0 = 0; v0 < nvec; v0 += 32 * UNROLL) {
      uint4 buf[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < nvec) buf[u] = ld_nc_v4(src + v);
      }
      for (unsigned m = keep; m != 0; m &= m - 1) {
        const int j = __ffs(m) - 1;
        const int row = __shfl_sync(0xFFFFFFFFu, my_row, j);
        uint4* dst = send + static_cast<size_t>(row) * nvec;
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          const int v = v0 + u * 32 + lane;
          if (v < nvec) st_v4(dst + v, buf[u]);
        }
      }
    }
  }
}

// FP8 payload: one warp per token, each half-warp quantises one 128-element block per step.
// scale = amax / 448 (1 when amax == 0), code = e4m3 round-to-nearest-even, saturating, of the fp32
// IEEE quotient x / scale.
template <int UNROLL>
__global__ void __launch_bounds__(kThreads)
    permute_fp8_kernel(const uint4* __restrict__ x, int T, int H, int k,
                       const int32_t* __restrict__ slot_row, uint8_t* __restrict__ send,
                       float* __restrict__ send_scales) {
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4, hl = lane & 15;
  const int nblk = H / 128;
  const int nvec = H / 8;
  const int nwarps = gridDim.x * kWarps;
  for (int t = blockIdx.x * kWarps + (threadIdx.x >> 5); t < T; t += nwarps) {
    const int my_row = lane < k ? __ldg(slot_row + static_cast<size_t>(t) * k + lane) : -1;
    const unsigned keep = __ballot_sync(0xFFFFFFFFu, my_row >= 0);
    const uint4* src = x + static_cast<size_t>(t) * nvec;
    for (int b0 = 0; b0 < nblk; b0 += 2 * UNROLL) {
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
        const float s = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
        scale[u] = s;
        uint32_t packed[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 pr = make_float2(__fdiv_rn(f[2 * i], s), __fdiv_rn(f[2 * i + 1], s));
          packed[i] = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3));
        }
        q[u] = make_uint2(packed[0] | (packed[1] << 16), packed[2] | (packed[3] << 16));
      }
      for (unsigned m = keep; m != 0; m &= m - 1) {
        const int j = __ffs(m) - 1;
        const int row = __shfl_sync(0xFFFFFFFFu, my_row, j);
        uint8_t* dst = send + static_cast<size_t>(row) * H;
        float* dsc = send_scales + static_cast<size_t>(row) * nblk;
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
}

int permute_grid(int T) {
  int blocks = (T + kWarps - 1) / kWarps;
  const int cap = num_sms() * 8;
  return blocks < cap ? blocks : cap;
}

}  // namespace

size_t dispatch_workspace_bytes(int T, int E) {
  const size_t n_chunks = (static_cast<size_t>(T) + kDispatchChunk - 1) / kDispatchChunk;
  const size_t tab = (n_chunks > 0 ? n_chunks : 1) * static_cast<size_t>(E) * sizeof(int32_t);
  return 256 + (tab + 255) / 256 * 256;
}

cudaError_t launch_dispatch(const void* x, int T, int H, const int32_t* topk_idx, int k, int E,
                            int R, int capacity, int fp8, void* send, float* send_scales,
                            int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_offsets,
                            int32_t* slot_row, int32_t* row_token, void* ws, cudaStream_t s) {
  char* base = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(base);
  unsigned* arrivals = reinterpret_cast<unsigned*>(base + 4);
  int32_t* chunk_tab = reinterpret_cast<int32_t*>(base + 256);
  if (T == 0) {
    // nothing routed: zero counts and offsets
    cudaError_t e1 = cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * E, s);
    if (e1 != cudaSuccess) return e1;
    e1 = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), s);
    if (e1 != cudaSuccess) return e1;
    return cudaMemsetAsync(rank_offsets, 0, sizeof(int32_t) * (R + 1), s);
  }
  const int n_chunks = (T + kDispatchChunk - 1) / kDispatchChunk;
  const int scan_n = E > 4 * kThreads ? E : 4 * kThreads;
  count_scan_kernel<<<n_chunks, kThreads, sizeof(int) * scan_n, s>>>(
      topk_idx, T, k, E, R, capacity, status, arrivals, chunk_tab, expert_counts, expert_offsets,
      rank_offsets);
  const size_t rank_smem = sizeof(int) * kWarps * E;
  if (rank_smem > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(rank_smem));
    if (err != cudaSuccess) return err;
  }
  rank_kernel<<<n_chunks, kThreads, rank_smem, s>>>(topk_idx, T, k, E, capacity, chunk_tab,
                                                    expert_offsets, slot_row, row_token);
  const int grid = permute_grid(T);
  if (fp8) {
    permute_fp8_kernel<2><<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(x), T, H, k,
                                                    slot_row, static_cast<uint8_t*>(send),
                                                    send_scales);
  } else {
    permute_bf16_kernel<8><<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(x), T, H / 8, k,
                                                     slot_row, static_cast<uint4*>(send));
  }
  return cudaGetLastError();
}

cudaError_t launch_dispatch_parts(const void* x, int T, int H, const int32_t* topk_idx, int k,
                                  int E, int R, int capacity, int fp8, void* send,
                                  float* send_scales, int32_t* expert_counts,
                                  int32_t* expert_offsets, int32_t* rank_offsets,
                                  int32_t* slot_row, int32_t* row_token, int* status,
                                  unsigned* arrivals, int32_t* chunk_tab, cudaStream_t s) {
  if (T == 0) {
    cudaError_t e1 = cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * E, s);
    if (e1 != cudaSuccess) return e1;
    e1 = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), s);
    if (e1 != cudaSuccess) return e1;
    return cudaMemsetAsync(rank_offsets, 0, sizeof(int32_t) * (R + 1), s);
  }
  const int n_chunks = (T + kDispatchChunk - 1) / kDispatchChunk;
  const int scan_n = E > 4 * kThreads ? E : 4 * kThreads;
  count_scan_kernel<<<n_chunks, kThreads, sizeof(int) * scan_n, s>>>(
      topk_idx, T, k, E, R, capacity, status, arrivals, chunk_tab, expert_counts, expert_offsets,
      rank_offsets);
  const size_t rank_smem = sizeof(int) * kWarps * E;
  rank_kernel<<<n_chunks, kThreads, rank_smem, s>>>(topk_idx, T, k, E, capacity, chunk_tab,
                                                    expert_offsets, slot_row, row_token);
  const int grid = permute_grid(T);
  if (fp8) {
    permute_fp8_kernel<2><<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(x), T, H, k,
                                                    slot_row, static_cast<uint8_t*>(send),
                                                    send_scales);
  } else {
    permute_bf16_kernel<8><<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(x), T, H / 8, k,
                                                     slot_row, static_cast<uint4*>(send));
  }
  return cudaGetLastError();
}

}  // namespace moe
