// Router: fused fp32 top-k + softmax weights + per-expert histogram, one warp per token.
//
// Selection follows the fine-ranking stage of "大模型MoE稀疏激活原理与硬件适配实战" (section 3.2:
// sort the router logits, keep the best k), in FP32 as its section 5.3 (scenario 3) requires; the
// k experts of a token are distinct (section 4.1).  Ordering: logit descending, ties to the lower
// expert id, NaN below every number.  Each lane holds E/32 logits as 64-bit keys
// (order-preserving image of the float, then the complemented expert id), and k rounds of a warp
// arg-max pick the experts best-first.
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

__device__ __forceinline__ unsigned long long route_key(float x, int e) {
  if (x == 0.0f) x = 0.0f;  // -0 and +0 compare equal: tie broken by id, not by sign
  uint32_t b = __float_as_uint(x);
  uint32_t ord;
  if (x != x) {
    ord = 0u;  // NaN: below -inf (whose image is 0x007FFFFF)
  } else {
    ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  }
  return (static_cast<unsigned long long>(ord) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(e));
}

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int m) {
  uint32_t lo = static_cast<uint32_t>(v), hi = static_cast<uint32_t>(v >> 32);
  lo = __shfl_xor_sync(0xFFFFFFFFu, lo, m);
  hi = __shfl_xor_sync(0xFFFFFFFFu, hi, m);
  return (static_cast<unsigned long long>(hi) << 32) | lo;
}

template <int VPL>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int T, int E,
                                                    int k, int renorm, int32_t* __restrict__ topk_idx,
                                                    float* __restrict__ topk_w,
                                                    int32_t* __restrict__ routed) {
  extern __shared__ int s_hist[];
  for (int i = threadIdx.x; i < E; i += blockDim.x) s_hist[i] = 0;
  griddep_wait();
  griddep_launch_dependents();
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int nwarps = gridDim.x * wpb;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += nwarps) {
    const float* row = logits + static_cast<size_t>(t) * E;
    float v[VPL];
    unsigned long long key[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      const float x = (e < E) ? __ldg(row + e) : 0.0f;
      v[i] = (x != x) ? -INFINITY : x;  // NaN weighs like -inf
      key[i] = (e < E) ? route_key(x, e) : 0ull;
    }

    int my_e = 0;
    float my_v = -INFINITY;
    for (int j = 0; j < k; ++j) {
      unsigned long long best = 0ull;
#pragma unroll
      for (int i = 0; i < VPL; ++i) best = key[i] > best ? key[i] : best;
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) {
        const unsigned long long o = shfl_xor_u64(best, m);
        best = o > best ? o : best;
      }
      const int e_sel = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(best));
      const int owner = e_sel & 31, slot = e_sel >> 5;
      float val = -INFINITY;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        if (lane == owner && i == slot) {
          val = v[i];
          key[i] = 0ull;  // removed: below every live key (NaN keys keep their id bits)
        }
      }
      val = __shfl_sync(0xFFFFFFFFu, val, owner);
      if (lane == j) {
        my_e = e_sel;
        my_v = val;
      }
    }

    const bool mine = lane < k;
    const float m = __shfl_sync(0xFFFFFFFFu, my_v, 0);  // the best selected value = row maximum
    float w;
    if (renorm) {
      const int n_inf = __popc(__ballot_sync(0xFFFFFFFFu, mine && my_v == INFINITY));
      if (n_inf > 0) {
        w = (my_v == INFINITY) ? 1.0f / static_cast<float>(n_inf) : 0.0f;
      } else if (m == -INFINITY) {
        w = 1.0f / static_cast<float>(k);
      } else {
        const float ex = mine ? expf(my_v - m) : 0.0f;
        float s = 0.0f;
        for (int j = 0; j < k; ++j) s += __shfl_sync(0xFFFFFFFFu, ex, j);  // fixed order
        w = ex / s;
      }
    } else {
      int n_inf = 0;
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        n_inf += __popc(__ballot_sync(0xFFFFFFFFu, (lane + 32 * i < E) && v[i] == INFINITY));
      if (n_inf > 0) {
        w = (my_v == INFINITY) ? 1.0f / static_cast<float>(n_inf) : 0.0f;
      } else if (m == -INFINITY) {
        w = 1.0f / static_cast<float>(E);
      } else {
        float part = 0.0f;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
          if (lane + 32 * i < E) part += expf(v[i] - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, o);
        w = expf(my_v - m) / part;
      }
    }
    if (mine) {
      topk_idx[static_cast<size_t>(t) * k + lane] = my_e;
      topk_w[static_cast<size_t>(t) * k + lane] = w;
      atomicAdd(&s_hist[my_e], 1);
    }
  }
  __syncthreads();
  if (routed != nullptr) {
    for (int i = threadIdx.x; i < E; i += blockDim.x)
      if (s_hist[i]) atomicAdd(&routed[i], s_hist[i]);
  }
}

}  // namespace

cudaError_t launch_route(const float* logits, int T, int E, int k, int renorm, int32_t* topk_idx,
                         float* topk_w, int32_t* routed, cudaStream_t s) {
  if (routed != nullptr) {
    cudaError_t err = cudaMemsetAsync(routed, 0, sizeof(int32_t) * E, s);
    if (err != cudaSuccess) return err;
  }
  if (T == 0) return cudaSuccess;
  constexpr int kThreads = 256;
  const int wpb = kThreads / 32;
  int blocks = (T + wpb - 1) / wpb;
  const int max_blocks = num_sms() * 8;
  if (blocks > max_blocks) blocks = max_blocks;
  const size_t smem = sizeof(int) * E;
  const bool pdl = routed == nullptr;  // after the histogram memset: ordinary launch
#define MOE_ROUTE_CASE(VPL)                                                                 \
  err = launch_pdl_if(pdl, route_kernel<VPL>, dim3(blocks), dim3(kThreads), smem, s, logits, T, \
                      E, k, renorm, topk_idx, topk_w, routed);                                 \
  break;
  cudaError_t err = cudaSuccess;
  switch ((E + 31) / 32) {
    case 1: MOE_ROUTE_CASE(1)
    case 2: MOE_ROUTE_CASE(2)
    case 3:
    case 4: MOE_ROUTE_CASE(4)
    case 5: case 6: case 7:
    case 8: MOE_ROUTE_CASE(8)
    case 9: case 10: case 11: case 12: case 13: case 14: case 15:
    case 16: MOE_ROUTE_CASE(16)
    default: MOE_ROUTE_CASE(32)
  }
  if (err != cudaSuccess) return err;
#undef MOE_ROUTE_CASE
  return cudaGetLastError();
}

}  // namespace moe
