// Expert parallelism across GPUs: the row regrouping on both sides of the all-to-all.
//
// Each rank dispatches its own tokens with R = the number of ranks, so its send buffer is
// destination-rank-major and, inside a destination's block, expert-major over that rank's experts
// (the ThunderEP page's section 2.1, redundancy 1: all rows for one destination in one contiguous
// block; the NCCL EP page's section 2.2: packed per-destination buffers in the high-throughput mode).
// After the exchange, rank r holds R source blocks, and source s's block holds counts[s][e] rows of
// each local expert e in turn.  The grouped FFN wants the rows expert-major; the return trip wants
// them back in source-major order.  Both moves, and the padding of the low-latency mode (every
// (source, destination) block at a fixed stride, the NCCL EP page's [E x M x H] layout), are one
// segmented copy: a [A, B] count matrix names the segments, each side of the copy lays them out
// a-major or b-major, packed or at a fixed stride per block, and every row moves once.
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / kWarp;
constexpr int kItems = kMaxRegroupSegments / kThreads;  // scan items per thread

// Exclusive scan of n <= kMaxRegroupSegments counts: item i reads counts[read(i)] and its exclusive
// prefix goes to out[slot(i)] (out[n] = total); items past n read as 0.  All threads of the CTA take
// part.  The sums are taken in 64 bits: a negative count, a count above `limit`, or a total above
// `limit` sets `bad` (the stored starts are then meaningless and must not be used).
template <typename Read, typename Slot>
__device__ void block_scan(const int32_t* __restrict__ counts, int n, Read read, Slot slot,
                           long long limit, int* out, long long* warp_tot, bool& bad) {
  long long v[kItems];
  long long run = 0;
#pragma unroll
  for (int i = 0; i < kItems; ++i) {
    const int j = threadIdx.x * kItems + i;
    long long c = j < n ? __ldg(counts + read(j)) : 0;
    if (c < 0 || c > limit) { bad = true; c = 0; }
    v[i] = run;
    run += c;
  }
  const int lane = threadIdx.x % kWarp, warp = threadIdx.x / kWarp;
  long long incl = run;
#pragma unroll
  for (int d = 1; d < kWarp; d <<= 1) {
    const long long o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == kWarp - 1) warp_tot[warp] = incl;
  __syncthreads();
  long long base = 0;
  for (int w = 0; w < warp; ++w) base += warp_tot[w];
  base += incl - run;
#pragma unroll
  for (int i = 0; i < kItems; ++i) {
    const int j = threadIdx.x * kItems + i;
    if (j < n) out[slot(j)] = static_cast<int>(base + v[i]);
  }
  if (threadIdx.x == kThreads - 1) {
    if (base + run > limit) bad = true;
    out[n] = static_cast<int>(base + run);
  }
  __syncthreads();
}

struct Side {
  int order;   // 0: a-major, 1: b-major
  int stride;  // rows per major block, 0 = packed
  int rows;    // row capacity of the buffer
};

// Row position of row q of segment (a, b) on one side.  am / bm: packed a-major / b-major starts of
// every segment (index a*B + b), with the totals at [A*B].
__device__ __forceinline__ long long position(const Side& sd, int a, int b, int q, int B, int A,
                                              const int* am, const int* bm) {
  const int seg = a * B + b;
  if (sd.order == 0) {
    const long long base = sd.stride > 0 ? static_cast<long long>(a) * sd.stride : am[a * B];
    return base + (am[seg] - am[a * B]) + q;
  }
  const long long base = sd.stride > 0 ? static_cast<long long>(b) * sd.stride : bm[b];
  return base + (bm[seg] - bm[b]) + q;
}

template <typename V>
__device__ __forceinline__ void copy_row(const unsigned char* __restrict__ src,
                                         unsigned char* __restrict__ dst, size_t bytes, int lane) {
  const V* s = reinterpret_cast<const V*>(src);
  V* d = reinterpret_cast<V*>(dst);
  const int n = static_cast<int>(bytes / sizeof(V));
  constexpr int kU = 4;  // vectors in flight per lane (2 KB per warp for 16-byte vectors)
  int i = lane;
  for (; i + (kU - 1) * kWarp < n; i += kU * kWarp) {
    V t[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) t[u] = __ldcs(s + i + u * kWarp);
#pragma unroll
    for (int u = 0; u < kU; ++u) __stcs(d + i + u * kWarp, t[u]);
  }
  for (; i < n; i += kWarp) __stcs(d + i, __ldcs(s + i));
}

__host__ __device__ __forceinline__ bool vec16_ok(const void* a, const void* b, size_t bytes) {
  return bytes % 16 == 0 && reinterpret_cast<uintptr_t>(a) % 16 == 0 &&
         reinterpret_cast<uintptr_t>(b) % 16 == 0;
}

struct Payload {
  const unsigned char* src;
  unsigned char* dst;
  size_t bytes;  // per row; 0 = absent
  int vec16;     // rows and base addresses allow 16-byte vectors (else 4-byte words)
};

// Up to kCtasPerSm CTAs per SM (64 registers a thread): the copies are latency-bound per warp, so
// the grid keeps as many warps in flight as the registers allow.
constexpr int kCtasPerSm = 4;

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    ep_regroup_kernel(const int32_t* __restrict__ counts, int A, int B, Side src_side,
                      Side dst_side, Payload p0, Payload p1, int32_t* __restrict__ dst_offsets,
                      int* status) {
  __shared__ int am[kMaxRegroupSegments + 1];  // packed a-major segment starts
  // packed b-major segment starts, indexed a*B + b; bm[b] (segment (0, b)) starts block b
  __shared__ int bm[kMaxRegroupSegments + 1];
  __shared__ long long warp_tot[kWarps];
  __shared__ int s_bad;
  griddep_wait();
  griddep_launch_dependents();
  const int n = A * B;
  if (threadIdx.x == 0) s_bad = 0;
  bool bad = false;
  // no segment and no total can exceed the smaller buffer
  const long long limit = src_side.rows < dst_side.rows ? src_side.rows : dst_side.rows;
  const auto same = [](int j) { return j; };
  block_scan(counts, n, same, same, limit, am, warp_tot, bad);
  // b-major order visits (a, b) as j = b*A + a
  const auto transposed = [A, B](int j) { return (j % A) * B + j / A; };
  block_scan(counts, n, transposed, transposed, limit, bm, warp_tot, bad);
  if (bad) s_bad = 1;
  __syncthreads();
  if (s_bad) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(status, kStatusBadCounts);
    return;
  }
  // strided layouts: a block's rows must fit its stride
  for (int i = threadIdx.x; i < (src_side.order ? B : A); i += kThreads) {
    if (src_side.stride <= 0) break;
    const int used = src_side.order ? bm[i + 1 < B ? i + 1 : n] - bm[i]
                                    : am[(i + 1) * B] - am[i * B];
    if (used > src_side.stride) s_bad = 1;
  }
  for (int i = threadIdx.x; i < (dst_side.order ? B : A); i += kThreads) {
    if (dst_side.stride <= 0) break;
    const int used = dst_side.order ? bm[i + 1 < B ? i + 1 : n] - bm[i]
                                    : am[(i + 1) * B] - am[i * B];
    if (used > dst_side.stride) s_bad = 1;
  }
  __syncthreads();
  const int total = am[n];
  if (s_bad) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(status, kStatusBadCounts);
    return;
  }
  if (dst_offsets != nullptr && blockIdx.x == 0) {
    for (int b = threadIdx.x; b <= B; b += kThreads) dst_offsets[b] = b < B ? bm[b] : total;
  }
  const int lane = threadIdx.x % kWarp;
  bool oob = false;
  for (int r = blockIdx.x * kWarps + threadIdx.x / kWarp; r < total; r += gridDim.x * kWarps) {
    // the segment holding packed a-major row r: the last start <= r
    int lo = 0, hi = n - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (am[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int a = lo / B, b = lo % B, q = r - am[lo];
    const long long ps = position(src_side, a, b, q, B, A, am, bm);
    const long long pd = position(dst_side, a, b, q, B, A, am, bm);
    if (ps < 0 || ps >= src_side.rows || pd < 0 || pd >= dst_side.rows) {
      oob = true;
      continue;
    }
    if (p0.vec16) copy_row<uint4>(p0.src + ps * p0.bytes, p0.dst + pd * p0.bytes, p0.bytes, lane);
    else copy_row<uint32_t>(p0.src + ps * p0.bytes, p0.dst + pd * p0.bytes, p0.bytes, lane);
    if (p1.bytes != 0) {
      if (p1.vec16) copy_row<uint4>(p1.src + ps * p1.bytes, p1.dst + pd * p1.bytes, p1.bytes, lane);
      else copy_row<uint32_t>(p1.src + ps * p1.bytes, p1.dst + pd * p1.bytes, p1.bytes, lane);
    }
  }
  if (oob && lane == 0) record_status(status, kStatusBadCounts);
}

// ---- the exchange over peer memory -------------------------------------------------------------
//
// Rank `rank` of R owns experts [rank*E_loc, (rank+1)*E_loc).  all_counts [R, E] holds every rank's
// expert_counts (the dispatch's kept rows per expert), so source s's rows for this rank's expert e
// sit in s's packed expert-major buffer from row  sum_{e' < rank*E_loc + e} all_counts[s][e']  on.
// Pull: every such row is read from the source's buffer (a peer pointer) and written expert-major
// into this rank's buffer (b-major over (s, e), packed), with the local expert offsets.  Push: the
// reverse, from this rank's expert-major buffer into every source's buffer at the same positions.

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    ep_exchange_kernel(const int32_t* __restrict__ all_counts, int R, int E, int rank, int E_loc,
                       int push, const unsigned long long* __restrict__ peer_rows,
                       const unsigned long long* __restrict__ peer_aux, int peer_cap,
                       unsigned char* __restrict__ local_rows, unsigned char* __restrict__ local_aux,
                       int local_cap, size_t row_bytes, size_t aux_bytes,
                       int32_t* __restrict__ local_offsets, int* status) {
  __shared__ int am[kMaxRegroupSegments + 1];  // packed (s, e) starts, s-major
  __shared__ int bm[kMaxRegroupSegments + 1];  // packed (s, e) starts, e-major; bm[e] starts expert e
  __shared__ long long block0[kMaxEpRanks];      // first row of this rank's block in source s
  __shared__ long long warp_tot[kWarps];
  __shared__ int s_bad;
  griddep_wait();
  griddep_launch_dependents();
  const int n = R * E_loc;
  const int e0 = rank * E_loc;
  if (threadIdx.x == 0) s_bad = 0;
  bool bad = false;
  // the rows received from all sources fill this rank's buffer; each source's block is checked
  // against the peer capacity below
  const long long limit = local_cap;
  const auto read_s_major = [E, E_loc, e0](int j) { return (j / E_loc) * E + e0 + j % E_loc; };
  const auto same = [](int j) { return j; };
  block_scan(all_counts, n, read_s_major, same, limit, am, warp_tot, bad);
  // e-major order visits (s, e) as j = e*R + s
  const auto read_e_major = [R, E, e0](int j) { return (j % R) * E + e0 + j / R; };
  const auto slot_e_major = [R, E_loc](int j) { return (j % R) * E_loc + j / R; };
  block_scan(all_counts, n, read_e_major, slot_e_major, limit, bm, warp_tot, bad);
  // block starts: one warp per source sums the counts of the experts before this rank's
  const int lane = threadIdx.x % kWarp, warp = threadIdx.x / kWarp;
  for (int src = warp; src < R; src += kWarps) {
    long long sum = 0;
    for (int e = lane; e < e0; e += kWarp) {
      const long long c = __ldg(all_counts + static_cast<long long>(src) * E + e);
      if (c < 0) bad = true;
      sum += c;
    }
#pragma unroll
    for (int d = kWarp / 2; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
    if (lane == 0) block0[src] = sum;
  }
  if (bad) s_bad = 1;
  __syncthreads();
  // this rank's block of every source must lie inside the source's buffer
  for (int src = threadIdx.x; src < R; src += kThreads) {
    const long long len = am[(src + 1) * E_loc] - am[src * E_loc];
    if (block0[src] + len > peer_cap) s_bad = 1;
  }
  __syncthreads();
  const int total = am[n];
  if (s_bad) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(status, kStatusBadCounts);
    return;
  }
  if (local_offsets != nullptr && blockIdx.x == 0) {
    for (int e = threadIdx.x; e <= E_loc; e += kThreads) local_offsets[e] = e < E_loc ? bm[e] : total;
  }
  for (int r = blockIdx.x * kWarps + warp; r < total; r += gridDim.x * kWarps) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (am[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int src = lo / E_loc, q = r - am[lo];
    const long long pp = block0[src] + (am[lo] - am[src * E_loc]) + q;  // row in the peer's buffer
    const long long pl = static_cast<long long>(bm[lo]) + q;             // row in this rank's
    unsigned char* peer = reinterpret_cast<unsigned char*>(peer_rows[src]);
    const unsigned char* from = push ? local_rows + pl * row_bytes : peer + pp * row_bytes;
    unsigned char* to = push ? peer + pp * row_bytes : local_rows + pl * row_bytes;
    if (vec16_ok(from, to, row_bytes)) copy_row<uint4>(from, to, row_bytes, lane);
    else copy_row<uint32_t>(from, to, row_bytes, lane);
    if (aux_bytes != 0) {
      unsigned char* pa = reinterpret_cast<unsigned char*>(peer_aux[src]);
      const unsigned char* af = push ? local_aux + pl * aux_bytes : pa + pp * aux_bytes;
      unsigned char* at = push ? pa + pp * aux_bytes : local_aux + pl * aux_bytes;
      if (vec16_ok(af, at, aux_bytes)) copy_row<uint4>(af, at, aux_bytes, lane);
      else copy_row<uint32_t>(af, at, aux_bytes, lane);
    }
  }
  // stores into other GPUs' memory: make them visible system-wide before this grid completes
  if (push) __threadfence_system();
}



}  // namespace

cudaError_t launch_ep_exchange(const int32_t* all_counts, int R, int E, int rank, int push,
                               const unsigned long long* peer_rows,
                               const unsigned long long* peer_aux, int peer_cap, void* local_rows,
                               void* local_aux, int local_cap, size_t row_bytes, size_t aux_bytes,
                               int32_t* local_offsets, int* status, cudaStream_t s) {
  const int E_loc = E / R;
  long long blocks = (static_cast<long long>(local_cap) + kWarps - 1) / kWarps;
  if (blocks > kCtasPerSm * static_cast<long long>(num_sms())) blocks = kCtasPerSm * static_cast<long long>(num_sms());
  if (blocks < 1) blocks = 1;
  const cudaError_t err = launch_pdl(
      ep_exchange_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0, s, all_counts, R,
      E, rank, E_loc, push, peer_rows, aux_bytes ? peer_aux : nullptr, peer_cap,
      static_cast<unsigned char*>(local_rows), static_cast<unsigned char*>(local_aux), local_cap,
      row_bytes, aux_bytes, local_offsets, status);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

cudaError_t launch_ep_regroup(const int32_t* counts, int A, int B, int src_order, int src_stride,
                              int src_rows, int dst_order, int dst_stride, int dst_rows,
                              const void* src, void* dst, size_t row_bytes, const void* src_aux,
                              void* dst_aux, size_t aux_row_bytes, int32_t* dst_offsets,
                              int* status, cudaStream_t s) {
  const Side ss{src_order, src_stride, src_rows};
  const Side ds{dst_order, dst_stride, dst_rows};
  const Payload p0{static_cast<const unsigned char*>(src), static_cast<unsigned char*>(dst),
                   row_bytes, vec16_ok(src, dst, row_bytes) ? 1 : 0};
  const Payload p1{static_cast<const unsigned char*>(src_aux), static_cast<unsigned char*>(dst_aux),
                   aux_row_bytes, vec16_ok(src_aux, dst_aux, aux_row_bytes) ? 1 : 0};
  // rows moved are at most the smaller capacity; one warp per row, a few waves at most
  const long long rows = src_rows < dst_rows ? src_rows : dst_rows;
  long long blocks = (rows + kWarps - 1) / kWarps;
  if (blocks > kCtasPerSm * static_cast<long long>(num_sms())) blocks = kCtasPerSm * static_cast<long long>(num_sms());
  if (blocks < 1) blocks = 1;
  const cudaError_t err =
      launch_pdl(ep_regroup_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0, s,
                 counts, A, B, ss, ds, p0, p1, dst_offsets, status);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace moe
