// Combine: weighted gather of each token's expert outputs back into token order.
//
// The NCCL EP page's low-latency combine (section 2.1) loops over the token's top-k slots and adds
// each expert output times the token's routing weight.  Here: one warp per token, 16-byte gathers
// of the k packed rows, fp32 accumulation in the fixed slot order j = 0, 1, ... with every product
// and every sum rounded separately (no fused multiply-add, so the result does not depend on
// contraction choices), one bf16 rounding at the end.  Dropped slots (row -1) contribute nothing.
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// Three CTAs (24 warps) per SM: the k <= 2 variants otherwise take 84 registers, which the
// per-warp register granularity turns into two CTAs per SM (measured: train combine 26.6 -> 24.5 us).
constexpr int kMinCtasPerSm = 3;

__device__ __forceinline__ void accumulate(float acc[8], float w, uint4 v) {
  const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(w, bf16_lo(words[i])));
    acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(w, bf16_hi(words[i])));
  }
}

// KS rows are gathered together per step (loads issued before any accumulation); UNROLL vectors
// per lane per row.
template <int KS, int UNROLL, bool SPLIT>
__global__ void __launch_bounds__(kThreads, kMinCtasPerSm)
    combine_kernel(const uint4* __restrict__ expert_out, int max_rows,
                   const int32_t* __restrict__ slot_row, const float* __restrict__ topk_w, int T,
                   int k, int nvec, int wpt, uint4* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int gwarp = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * kWarps;
  // wpt warps per token (wpt divides nvec), each takes nseg consecutive vectors of the row
  const int nseg = SPLIT ? nvec / wpt : nvec;
  const int vofs = SPLIT ? (gwarp % wpt) * nseg : 0;
  griddep_wait();
  griddep_launch_dependents();
  for (int t = SPLIT ? gwarp / wpt : gwarp; t < T; t += SPLIT ? nwarps / wpt : nwarps) {
    int my_row = -1;
    float my_w = 0.0f;
    if (lane < k) {
      my_row = __ldg(slot_row + static_cast<size_t>(t) * k + lane);
      my_w = __ldg(topk_w + static_cast<size_t>(t) * k + lane);
      if (my_row >= max_rows) my_row = -1;
    }
    const unsigned live = __ballot_sync(0xFFFFFFFFu, my_row >= 0);
    uint4* dst = y + static_cast<size_t>(t) * nvec + vofs;
    for (int v0 = 0; v0 < nseg; v0 += 32 * UNROLL) {
      float acc[UNROLL][8];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
      // slots in ascending j, KS rows loaded before they are accumulated
      for (unsigned m = live; m != 0;) {
        int rows[KS];
        float ws[KS];
        int n = 0;
#pragma unroll
        for (int q = 0; q < KS; ++q) {
          rows[q] = -1;
          ws[q] = 0.0f;
          if (m != 0) {
            const int j = __ffs(m) - 1;
            m &= m - 1;
            rows[q] = j;
            n = q + 1;
          }
        }
        uint4 vals[KS][UNROLL];
#pragma unroll
        for (int q = 0; q < KS; ++q) {
          if (q < n) {
            const int j = rows[q];
            const int row = __shfl_sync(0xFFFFFFFFu, my_row, j);
            ws[q] = __shfl_sync(0xFFFFFFFFu, my_w, j);
            const uint4* src = expert_out + static_cast<size_t>(row) * nvec + vofs;
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
              const int v = v0 + u * 32 + lane;
              if (v < nseg) vals[q][u] = ld_nc_v4(src + v);
            }
          }
        }
#pragma unroll
        for (int q = 0; q < KS; ++q) {
          if (q < n) {
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
              const int v = v0 + u * 32 + lane;
              if (v < nseg) accumulate(acc[u], ws[q], vals[q][u]);
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < nseg) {
          uint4 o;
          o.x = pack_bf16x2(acc[u][0], acc[u][1]);
          o.y = pack_bf16x2(acc[u][2], acc[u][3]);
          o.z = pack_bf16x2(acc[u][4], acc[u][5]);
          o.w = pack_bf16x2(acc[u][6], acc[u][7]);
          st_v4(dst + v, o);
        }
      }
    }
  }
}


}  // namespace

cudaError_t launch_combine(const void* expert_out, int max_rows, const int32_t* slot_row,
                           const float* topk_w, int T, int k, int H, void* y, int* status,
                           cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  (void)status;  // the combine has no device-side waits, so it never records a status bit
  // warps per token: split rows so that about 64 warps per SM have work (small T)
  const int nvec = H / 8;
  int wpt = 1;
  while (wpt < 8 && static_cast<long long>(T) * wpt < 64LL * num_sms() && nvec % (2 * wpt) == 0 &&
         nvec / (2 * wpt) >= 32)
    wpt *= 2;
  const long long warps = static_cast<long long>(T) * wpt;
  int blocks = static_cast<int>((warps + kWarps - 1) / kWarps);
  const int cap = num_sms() * 8;
  if (blocks > cap) blocks = cap;  // grid-stride; cap is a multiple of 8, so of wpt
  const uint4* eo = static_cast<const uint4*>(expert_out);
  uint4* yo = static_cast<uint4*>(y);
  // rows gathered together sized to k: enough loads in flight, few registers (high occupancy)
  using Kern = void (*)(const uint4*, int, const int32_t*, const float*, int, int, int, int, uint4*);
  Kern kern;
  if (wpt > 1)
    kern = k <= 2 ? combine_kernel<2, 4, true>
                  : (k <= 4 ? combine_kernel<4, 2, true> : combine_kernel<8, 1, true>);
  else
    kern = k <= 2 ? combine_kernel<2, 4, false>
                  : (k <= 4 ? combine_kernel<4, 2, false> : combine_kernel<8, 1, false>);
  const cudaError_t err = launch_pdl(kern, dim3(blocks), dim3(kThreads), 0, s, eo, max_rows,
                                     slot_row, topk_w, T, k, nvec, wpt, yo);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace moe
