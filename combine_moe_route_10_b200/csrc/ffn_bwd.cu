// Backward of the MoE layer: the gradient goes back through the forward's plan (the training step
// of the NCCL EP page, section 3.2: the backward reuses the forward's routing handle, dispatches the
// output gradient to the experts, runs the experts backward and combines the gradients).
//
//   1. combine_bwd_kernel (warp per token): d_eo[row] = bf16(w[t,j] * dy[t]) for every kept slot,
//      the routing-weight gradient d_w[t,j] = <dy[t], eo[row]>, and from it the router's logit
//      gradient (softmax backward over the selected k, or over all E without renormalisation).
//   2. bwd_gemm_kernel<kRecompute> (tcgen05, M = 256 rows over a CTA pair, 128 h columns, k = 32
//      per stage with the 64-byte swizzle): recomputes g = x Wg^T and u = x Wu^T (one N = 256 MMA:
//      CTA 0 stages the gate rows, CTA 1 the up rows) and computes dh = d_eo Wd (N = 128, Wd read
//      MN-major) in the same K loop over H, then the SwiGLU backward in the epilogue: h, dg, du
//      (bf16).
//   3. bwd_gemm_kernel<kInputGrad> (M = 256, N = 256): dx_rows = dg Wg + du Wu, one K loop over
//      2F, the weights read MN-major.
//   4. bwd_gemm_kernel<kWeightGrad> (M = 256, N = 256, K = the expert's rows): dWd = d_eo^T h,
//      dWg = dg^T x, dWu = du^T x in fp32, both operands MN-major; the rows past the expert's end in
//      the last K block are zeroed in shared memory before the MMA reads them; TMA stores.
//   5. the forward combine with unit weights: dx[t] = bf16(sum of dx_rows of its kept slots).
//   (moe_combine_backward is step 1 alone, moe_expert_backward steps 2-4.)
//
// The GEMM kernels are persistent 2-CTA clusters (tcgen05.mma.cta_group::2, one CTA per SM, a
// static tile order shared by both CTAs), warp-specialised like the forward's pair kernel: warp 0
// = TMA producer (CTA 1's copies complete on CTA 0's barriers), warp 1 = TMEM allocation and, in
// CTA 0, the MMA thread of the pair, warps 2..5 = epilogue of the CTA's 128 rows; two accumulators
// (one for the recompute) so that an epilogue overlaps the next tile's MMAs.  Every wait is bounded
// (kStatusTimeout); no TMA multicast.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int kBM = 128;         // rows of a tile held by one CTA of the pair (one TMEM lane each)
constexpr int kPairM = 256;      // rows (or output rows) of a pair tile
constexpr int kBK = 64;
constexpr int kUK = 16;
constexpr int kBwdThreads = 192;
constexpr int kTmemColsBwd = 512;
constexpr int kAccStride = 256;  // TMEM columns between the two accumulators
constexpr int kNF1 = 128;        // h columns per recompute tile
constexpr int kBK1 = 32;         // recompute: k per stage (64-byte rows, 64-byte swizzle)
constexpr int kNOut = 256;       // output columns per input-gradient / weight-gradient tile

enum Mode { kRecompute = 1, kInputGrad = 2, kWeightGrad = 3 };

// Per CTA of a pair: its own 128 rows of A and half of B.
template <int MODE>
struct Cfg {
  // recompute: x, d_eo (128 rows x 32 k, 8 KB each), the gate (CTA 0) or up (CTA 1) block of
  // 128 rows x 32 k (8 KB), 64 f columns of Wd^T x 32 k (4 KB): 28 KB.  Others: A 16 KB + half of
  // B 16 KB.
  static constexpr int kStageBytes = MODE == kRecompute ? 3 * 8192 + 4096 : 16384 + 16384;
  static constexpr int kStages = MODE == kRecompute ? 7 : 6;
  // the recompute's accumulators (g | u 256 columns, dh 128) fill one TMEM set; the others
  // alternate between two so that an epilogue overlaps the next tile's MMAs
  static constexpr int kAccBufs = MODE == kRecompute ? 1 : 2;
};

// ---- PTX wrappers -----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Shared::cluster address of the same shared-memory offset in CTA `rank` of the pair.
__device__ __forceinline__ uint32_t mapa(uint32_t local, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(local), "r"(rank));
  return out;
}
__device__ __forceinline__ void pair_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Count `bytes` of transactions done on the other CTA's mbarrier (a signal without an arrival).
constexpr uint32_t kTailToken = 16;
__device__ __forceinline__ void complete_tx_remote(uint32_t cluster_addr, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.relaxed.cluster.shared::cluster.b64 [%0], %1;" ::"r"(
                   cluster_addr),
               "r"(bytes)
               : "memory");
}
// Arrive on the other CTA's mbarrier, releasing this thread's prior writes at cluster scope.
__device__ __forceinline__ void arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ bool try_wait_cl(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// CTA 0's copy into its own shared memory, completing on its own barrier.
__device__ __forceinline__ void tma2d(uint32_t dst, const CUtensorMap* tm, uint32_t bar, int x,
                                      int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// CTA 1's copy into its own shared memory, completing its bytes on CTA 0's barrier `bar_cta0`
// (a shared::cluster address); a plain, not multicast, load.
__device__ __forceinline__ void tma2d_to_leader(uint32_t dst, const CUtensorMap* tm,
                                                uint32_t bar_cta0, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar_cta0)
      : "memory");
}
__device__ __forceinline__ void fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on the mbarrier at this offset in BOTH CTAs when the MMAs issued so far complete.
__device__ __forceinline__ void commit_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}
__device__ __forceinline__ void commit_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                    uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory descriptors (version 1).  K-major, 128-byte swizzle (layout type 2): rows of 128
// bytes hold 64 k values, 8-row groups 1024 bytes apart (stride byte offset; the leading byte offset
// is unused).  K-major, 64-byte swizzle (layout type 4): rows of 64 bytes hold 32 k values, 8-row
// groups 512 bytes apart.  MN-major, 128-byte swizzle: rows of 128 bytes hold 64 m (or n) values
// of one k, 8-k groups 1024 bytes apart (stride byte offset), and the next 64 m values lie `lbo`
// bytes further (the next TMA box: leading byte offset).
__device__ __forceinline__ uint64_t desc_k(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}
__device__ __forceinline__ uint64_t desc_k64(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(512 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(4) << 61);
}
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr, uint32_t lbo) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) |
         (static_cast<uint64_t>(lbo >> 4) << 16) | (static_cast<uint64_t>(1024 >> 4) << 32) |
         (static_cast<uint64_t>(1) << 46) | (static_cast<uint64_t>(2) << 61);
}
// kind::f16 instruction descriptor: fp32 D, bf16 A and B, a_mn / b_mn = MN-major operands.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Bounded wait on a barrier phase (arrivals may come from either CTA of the pair).  False if this
// CTA aborts or the limit runs out (which records kStatusTimeout and raises the abort).
__device__ __forceinline__ bool cwait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                      int* status) {
  if (try_wait_cl(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (true) {
    if (try_wait_cl(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      record_status(status, kStatusTimeout);
      return false;
    }
  }
}
// The same wait regardless of the abort flag (a CTA draining its own copies / MMAs).
__device__ __forceinline__ void cdrain(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = global_timer_ns();
  while (!try_wait_cl(bar, parity) && global_timer_ns() - t0 <= kWaitLimitNs) {
  }
}

struct BwdArgs {
  const int32_t* expert_offsets;  // [E + 1], packed rows of every expert
  int E, H, F, max_rows;
  void* out0;  // recompute: h; input grad: dx_rows; weight grad: dWd
  void* out1;  // recompute: dg;                       weight grad: dWg
  void* out2;  // recompute: du;                       weight grad: dWu
  int* status;
};

// Rows [off, off + rows) of expert e, its offsets clamped to [0, max_rows] as in the forward, so
// that offsets past the row buffers (a caller's mistake) make no tile read or write outside them.
__device__ __forceinline__ int expert_span(const BwdArgs& a, int e, int& rows) {
  const int lo = min(max(__ldg(a.expert_offsets + e), 0), a.max_rows);
  const int hi = min(max(__ldg(a.expert_offsets + e + 1), 0), a.max_rows);
  rows = max(hi - lo, 0);
  return lo;
}

// Pair tiles of every item (prefix in shared memory) and the decoding of a tile index.
struct Tile {
  int e, p, mb, nb;  // expert, sub-problem (weight grad), 256-row block, column block
};
template <int MODE>
__device__ __forceinline__ int tiles_of(const BwdArgs& a, int rows, int p) {
  if (MODE == kRecompute) return ((rows + kPairM - 1) / kPairM) * ((a.F + kNF1 - 1) / kNF1);
  if (MODE == kInputGrad) return ((rows + kPairM - 1) / kPairM) * ((a.H + kNOut - 1) / kNOut);
  // weight gradients: p = 0 dWd [H, F]; p = 1, 2 dWg, dWu [F, H]
  const int M = p == 0 ? a.H : a.F, N = p == 0 ? a.F : a.H;
  return ((M + kPairM - 1) / kPairM) * ((N + kNOut - 1) / kNOut);
}

// Weight gradients: every (sub-problem, expert) item has the same tile count, so a tile's item is a
// division (no table).
__device__ __forceinline__ int wgrad_tiles_per_item(const BwdArgs& a) {
  return ((a.H + kPairM - 1) / kPairM) * ((a.F + kNOut - 1) / kNOut);
}

template <int MODE>
__device__ __forceinline__ Tile decode(const BwdArgs& a, const int* start, int tile) {
  if (MODE == kWeightGrad) {
    // items p*E + e in order; dWd [H, F] and dWg, dWu [F, H] have the same 256 x 256 tile count
    const int per = wgrad_tiles_per_item(a);
    const int item = tile / per, local = tile - item * per;
    Tile t;
    t.p = item / a.E;
    t.e = item % a.E;
    // both operands (the expert's rows) stay in L2 across the output blocks
    const int ncol = ((t.p == 0 ? a.F : a.H) + kNOut - 1) / kNOut;
    t.mb = local / ncol;
    t.nb = local % ncol;
    return t;
  }
  // start[i] = first tile of expert i
  const int n_items = a.E;
  int lo = 0, hi = n_items - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  Tile t;
  t.p = 0;
  t.e = lo;
  const int local = tile - start[lo];
  {
    // row blocks fastest: the tiles running at the same time share one weight slice, which then
    // crosses HBM once per expert instead of once per row block
    int rows;
    expert_span(a, t.e, rows);
    const int nrow = (rows + kPairM - 1) / kPairM;
    t.mb = local % nrow;
    t.nb = local / nrow;
  }
  return t;
}

template <int MODE>
__device__ __forceinline__ int k_blocks(const BwdArgs& a, int rows) {
  if (MODE == kRecompute) return a.H / kBK1;
  if (MODE == kInputGrad) return 2 * (a.F / kBK);
  return (rows + kBK - 1) / kBK;
}

// Operand maps of a mode (unused ones are zero); the weight-gradient mode also gets the three
// output maps (fp32 [E][M][N], 32 x 32 boxes with the 128-byte swizzle) for its TMA stores.
struct BwdMaps {
  CUtensorMap m[6];
  CUtensorMap out[3];
};
constexpr int kStageOutBytes = 32 * 32 * 4;  // one epilogue warp's 32 x 32 fp32 block

__device__ __forceinline__ void tma_store3d(const CUtensorMap* tm, uint32_t src, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(tm)),
      "r"(src), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The shared-memory source of every store issued so far has been read (_1: all but the latest).
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// One 2-CTA cluster per pair of SMs; both CTAs walk the same tile sequence.  CTA 0 (the leader)
// owns the full and accumulator-empty barriers that count both CTAs, and its MMA thread issues
// every MMA of the pair; each CTA's epilogue reads its own TMEM (its 128 rows).
template <int MODE>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_gemm_kernel(const __grid_constant__ BwdMaps maps, const BwdArgs args) {
  constexpr int kStages = Cfg<MODE>::kStages;
  constexpr int kStageBytes = Cfg<MODE>::kStageBytes;
  constexpr int kBufs = Cfg<MODE>::kAccBufs;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned stages, then the store staging, barriers and the tile prefix table
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr int kOutBytes = MODE == kWeightGrad ? 8 * kStageOutBytes : 0;
  uint8_t* out_stage = base + kStages * kStageBytes;  // 1024-aligned: [4 warps][2][32 x 32 fp32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(out_stage + kOutBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* fix_bar = acc_empty + 2;
  uint64_t* drain_bar = fix_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* start = reinterpret_cast<int*>(tmem_slot + 4);  // [items + 1]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();
  const int E = args.E;
  const int n_items = MODE == kWeightGrad ? 3 * E : E;
  const int cid = static_cast<int>(blockIdx.x) >> 1, ncl = static_cast<int>(gridDim.x) >> 1;

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_addr(&full[i]), 1);   // CTA 0's copy: its arrival + both CTAs' bytes
      mbar_init(smem_addr(&empty[i]), 1);  // each CTA's own: the multicast commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&acc_full[i]), 1);   // each CTA's own: the multicast commit
      mbar_init(smem_addr(&acc_empty[i]), 8);  // CTA 0's copy: four epilogue warps of each CTA
    }
    mbar_init(smem_addr(fix_bar), 1);
    mbar_init(smem_addr(drain_bar), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  } else if (warp == 1) {
    // the same warp of both CTAs allocates, as cta_group::2 requires
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kTmemColsBwd)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  griddep_wait();
  griddep_launch_dependents();
  if (MODE == kWeightGrad) {
    if (threadIdx.x == 0) start[0] = 3 * E * wgrad_tiles_per_item(args);  // the tile count
  } else if (warp == 2 && lane == 0) {
    int run = 0;
    for (int i = 0; i < n_items; ++i) {
      start[i] = run;
      int rows;
      expert_span(args, i % E, rows);
      run += tiles_of<MODE>(args, rows, i / E);
    }
    start[n_items] = run;
  }
  fence_before();
  __syncthreads();
  pair_sync();  // both CTAs' barriers are initialised before any remote arrive or copy
  fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = MODE == kWeightGrad ? start[0] : start[n_items];
  const uint32_t stage0 = smem_addr(base);

  if (warp == 0) {
    // ---- TMA producer (lane 0 issues; the whole warp zeroes a ragged K tail) ----------------------
    int stage = 0;
    uint32_t phase = 0, fix_phase = 0;
    uint32_t issued_mask = 0, issued_parity = 0;
    bool stop = false;
    for (int tile = cid; tile < total && !stop; tile += ncl) {
      const Tile t = decode<MODE>(args, start, tile);
      int rows;
      const int off = expert_span(args, t.e, rows);
      const int nkb = k_blocks<MODE>(args, rows);
      const int half = static_cast<int>(rank) * kBM;  // this CTA's rows / columns of the tile
      for (int kb = 0; kb < nkb; ++kb) {
        int ok = 1;
        if (lane == 0) ok = cwait(smem_addr(&empty[stage]), phase ^ 1u, abort_flag, args.status);
        if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
          stop = true;
          break;
        }
        const uint32_t a = stage0 + stage * kStageBytes;
        const uint32_t fb = smem_addr(&full[stage]);  // CTA 0's copy counts both CTAs
        const uint32_t fb0 = mapa(fb, 0);
        // CTA 0 arrives once and announces the pair's bytes; CTA 1's copies complete on CTA 0's
        // barrier
        auto load = [&](const CUtensorMap* tm, uint32_t dst, int x, int y) {
          if (rank == 0) tma2d(dst, tm, fb, x, y);
          else tma2d_to_leader(dst, tm, fb0, x, y);
        };
        bool tail = false;
        int valid = kBK;
        if (MODE == kWeightGrad) {
          valid = min(kBK, rows - kb * kBK);
          tail = valid < kBK;
        }
        if (!tail) {
          if (lane == 0) {
            if (rank == 0) mbar_arrive_expect_tx(fb, 2 * kStageBytes);
            if (MODE == kRecompute) {
              // x and d_eo: this CTA's 128 rows x 32 k; B: the gate (CTA 0) or up (CTA 1) block of
              // 128 rows x 32 k, then 64 of the tile's 128 f columns of Wd^T.  Rows past the
              // expert's F only reach accumulator columns the epilogue does not store.
              const int kx = kb * kBK1, row0 = off + t.mb * kPairM + half, f0 = t.nb * kNF1;
              load(&maps.m[0], a, kx, row0);
              load(&maps.m[1], a + 8192, kx, row0);
              load(&maps.m[rank == 0 ? 2 : 3], a + 16384, kx, t.e * args.F + f0);
              load(&maps.m[4], a + 24576, f0 + static_cast<int>(rank) * 64, t.e * args.H + kx);
            } else if (MODE == kInputGrad) {
              const int nf = args.F / kBK;
              const bool up = kb >= nf;
              const int kx = (up ? kb - nf : kb) * kBK, row0 = off + t.mb * kPairM + half;
              const int n0 = t.nb * kNOut + half;
              load(&maps.m[up ? 1 : 0], a, kx, row0);  // dg or du rows (K-major)
              // Wg or Wu: this CTA's 128 of the tile's 256 h columns, 64 f each (MN-major)
              load(&maps.m[up ? 3 : 2], a + 16384, n0, t.e * args.F + kx);
              load(&maps.m[up ? 3 : 2], a + 24576, n0 + 64, t.e * args.F + kx);
            } else {
              const CUtensorMap* ma = &maps.m[t.p == 0 ? 0 : (t.p == 1 ? 1 : 2)];  // d_eo, dg, du
              const CUtensorMap* mb = &maps.m[t.p == 0 ? 3 : 4];                   // h, x
              const int y = off + kb * kBK, m0 = t.mb * kPairM + half, n0 = t.nb * kNOut + half;
              load(ma, a, m0, y);
              load(ma, a + 8192, m0 + 64, y);
              load(mb, a + 16384, n0, y);
              load(mb, a + 24576, n0 + 64, y);
            }
          }
        } else {
          // the expert's last rows: this CTA's copies complete on its own barrier, the rows past
          // the end are zeroed in all four boxes; then CTA 0 arrives on its full barrier expecting
          // a 16-byte token from CTA 1, which CTA 1 completes (after a cluster-scope fence) once
          // its own rows are zeroed
          const uint32_t xb = smem_addr(fix_bar);
          if (lane == 0) {
            const CUtensorMap* ma = &maps.m[t.p == 0 ? 0 : (t.p == 1 ? 1 : 2)];
            const CUtensorMap* mb = &maps.m[t.p == 0 ? 3 : 4];
            const int y = off + kb * kBK, m0 = t.mb * kPairM + half, n0 = t.nb * kNOut + half;
            mbar_arrive_expect_tx(xb, kStageBytes);
            tma2d(a, ma, xb, m0, y);
            tma2d(a + 8192, ma, xb, m0 + 64, y);
            tma2d(a + 16384, mb, xb, n0, y);
            tma2d(a + 24576, mb, xb, n0 + 64, y);
          }
          // every lane waits, so that its stores below follow the copy's writes
          const int got = cwait(xb, fix_phase, abort_flag, args.status) ? 1 : 0;
          fix_phase ^= 1u;
          if (__all_sync(0xFFFFFFFFu, got) == 0) {
            stop = true;
            break;
          }
          uint4* sm = reinterpret_cast<uint4*>(base + stage * kStageBytes);
          const int per_box = (kBK - valid) * 8;  // 16-byte chunks in the rows to clear
          for (int i = lane; i < 4 * per_box; i += 32) {
            const int box = i / per_box, c = i % per_box;
            sm[box * 512 + valid * 8 + c] = make_uint4(0u, 0u, 0u, 0u);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            if (rank == 0) {
              mbar_arrive_expect_tx(fb, kTailToken);
            } else {
              asm volatile("fence.acq_rel.cluster;" ::: "memory");
              complete_tx_remote(fb0, kTailToken);
            }
          }
        }
        issued_mask |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (*abort_flag && lane == 0 && rank == 0) {
      // CTA 0's barriers count both CTAs' bytes: wait for the latest phase of each stage
      for (int st = 0; st < kStages; ++st)
        if (issued_mask & (1u << st)) cdrain(smem_addr(&full[st]), (issued_parity >> st) & 1u);
    }
  } else if (warp == 1) {
    // ---- MMA thread (CTA 0 only): M = 256 over the pair ---------------------------------------------
    if (rank == 0 && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool issued_any = false;
      int it = 0;
      for (int tile = cid; tile < total; tile += ncl, ++it) {
        const Tile t = decode<MODE>(args, start, tile);
        int rows;
        expert_span(args, t.e, rows);
        const int nkb = k_blocks<MODE>(args, rows);
        const int acc = kBufs == 2 ? (it & 1) : 0;
        const uint32_t acc_par = kBufs == 2 ? ((it >> 1) & 1) : (it & 1);
        if (!cwait(smem_addr(&acc_empty[acc]), acc_par ^ 1u, abort_flag, args.status)) break;
        fence_after();
        const uint32_t d = tmem_base + acc * kAccStride;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!cwait(smem_addr(&full[stage]), phase, abort_flag, args.status)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t a = stage0 + stage * kStageBytes;
#pragma unroll
          for (int kk = 0; kk < (MODE == kRecompute ? kBK1 : kBK) / kUK; ++kk) {
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            if (MODE == kRecompute) {
              // g | u: N = 256 (CTA 0's gate rows -> columns 0..127, CTA 1's up rows -> 128..255);
              // dh: N = 128 (64 f columns of Wd^T in each CTA) in columns 256..383
              constexpr uint32_t iGU = idesc_bf16(kPairM, 2 * kNF1, 0, 0);
              constexpr uint32_t iMN = idesc_bf16(kPairM, kNF1, 0, 1);
              mma(d, desc_k64(a + kk * 32), desc_k64(a + 16384 + kk * 32), iGU, accum);
              mma(d + 256, desc_k64(a + 8192 + kk * 32), desc_mn(a + 24576 + kk * 2048, 4096),
                  iMN, accum);
            } else if (MODE == kInputGrad) {
              constexpr uint32_t iMN = idesc_bf16(kPairM, kNOut, 0, 1);
              mma(d, desc_k(a + kk * 32), desc_mn(a + 16384 + kk * 2048, 8192), iMN, accum);
            } else {
              constexpr uint32_t iMM = idesc_bf16(kPairM, kNOut, 1, 1);
              mma(d, desc_mn(a + kk * 2048, 8192), desc_mn(a + 16384 + kk * 2048, 8192), iMM,
                  accum);
            }
          }
          issued_any = true;
          commit_both(smem_addr(&empty[stage]));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        // a tile without K blocks (an expert with no rows) has nothing to wait for: the epilogues
        // write zeros; the commit still orders it after the previous tile's MMAs
        commit_both(smem_addr(&acc_full[acc]));
      }
      if (issued_any) {
        commit_local(smem_addr(drain_bar));
        cdrain(smem_addr(drain_bar), 0);
      }
    }
  } else {
    // ---- epilogue: warp (w & 3) owns TMEM lanes (= this CTA's rows) [32 (w & 3), +32) -------------
    const int quarter = warp & 3;
    const int r = static_cast<int>(rank) * kBM + quarter * 32 + lane;  // row of the pair tile
    const uint32_t acc_empty0 = mapa(smem_addr(&acc_empty[0]), 0);
    const uint32_t acc_empty1 = mapa(smem_addr(&acc_empty[1]), 0);
    // weight gradients: the stores of consecutive blocks, across tiles too, alternate between
    // this warp's two staging blocks
    int chunk = 0;
    int it = 0;
    for (int tile = cid; tile < total; tile += ncl, ++it) {
      const Tile t = decode<MODE>(args, start, tile);
      int rows;
      const int off = expert_span(args, t.e, rows);
      const int acc = kBufs == 2 ? (it & 1) : 0;
      const uint32_t acc_par = kBufs == 2 ? ((it >> 1) & 1) : (it & 1);
      int ok = 1;
      if (lane == 0) ok = cwait(smem_addr(&acc_full[acc]), acc_par, abort_flag, args.status);
      if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) break;
      fence_after();
      const uint32_t tb = tmem_base + acc * kAccStride + (static_cast<uint32_t>(quarter * 32) << 16);
      if (MODE == kRecompute) {
        const bool valid = t.mb * kPairM + r < rows;
        const size_t row = static_cast<size_t>(off + t.mb * kPairM + r);
        __nv_bfloat16* h_out = static_cast<__nv_bfloat16*>(args.out0);
        __nv_bfloat16* dg_out = static_cast<__nv_bfloat16*>(args.out1);
        __nv_bfloat16* du_out = static_cast<__nv_bfloat16*>(args.out2);
#pragma unroll 1
        for (int c = 0; c < kNF1; c += 32) {
          if (t.nb * kNF1 + c >= args.F) break;  // uniform over the warp
          uint32_t g[32], u[32], dh[32];
          ld32(tb + c, g);
          ld32(tb + kNF1 + c, u);
          ld32(tb + 2 * kNF1 + c, dh);
          ld_wait();
          uint32_t ph[16], pg[16], pu[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float hv[2], dgv[2], duv[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const float gv = __uint_as_float(g[2 * i + q]), uv = __uint_as_float(u[2 * i + q]);
              const float dv = __uint_as_float(dh[2 * i + q]);
              const float sg = 1.0f / (1.0f + expf(-gv));
              const float silu = gv * sg;
              hv[q] = silu * uv;
              dgv[q] = dv * uv * sg * (1.0f + gv * (1.0f - sg));
              duv[q] = dv * silu;
            }
            ph[i] = pack_bf16x2(hv[0], hv[1]);
            pg[i] = pack_bf16x2(dgv[0], dgv[1]);
            pu[i] = pack_bf16x2(duv[0], duv[1]);
          }
          if (valid) {
            const size_t col = static_cast<size_t>(t.nb * kNF1 + c);
            uint4* hp = reinterpret_cast<uint4*>(h_out + row * args.F + col);
            uint4* gp = reinterpret_cast<uint4*>(dg_out + row * args.F + col);
            uint4* up = reinterpret_cast<uint4*>(du_out + row * args.F + col);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              hp[v] = make_uint4(ph[4 * v], ph[4 * v + 1], ph[4 * v + 2], ph[4 * v + 3]);
              gp[v] = make_uint4(pg[4 * v], pg[4 * v + 1], pg[4 * v + 2], pg[4 * v + 3]);
              up[v] = make_uint4(pu[4 * v], pu[4 * v + 1], pu[4 * v + 2], pu[4 * v + 3]);
            }
          }
        }
      } else if (MODE == kInputGrad) {
        const bool valid = t.mb * kPairM + r < rows;
        const size_t row = static_cast<size_t>(off + t.mb * kPairM + r);
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out0);
#pragma unroll 1
        for (int c = 0; c < kNOut; c += 32) {
          const int col = t.nb * kNOut + c;
          if (col >= args.H) break;  // uniform over the warp
          uint32_t v[32];
          ld32(tb + c, v);
          ld_wait();
          if (valid) {
            uint4* p = reinterpret_cast<uint4*>(out + row * args.H + col);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              p[q] = make_uint4(
                  pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                  pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                  pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                  pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
          }
        }
      } else {
        // each 32 x 32 block: TMEM -> registers (lane = row) -> this warp's staging block in the
        // 128-byte swizzled layout -> one TMA store (rows past M and columns past N are clipped)
        const int N = t.p == 0 ? args.F : args.H;
        const CUtensorMap* om = &maps.out[t.p];
        const bool any_k = rows > 0;  // uniform over the warp
        uint8_t* stg = out_stage + 2 * quarter * kStageOutBytes;  // this warp's two blocks
        const uint32_t stg_addr = smem_addr(stg);
        if (!any_k) {
          // an expert without rows: one zero block, stored to every 32-column block of this
          // warp's rows without waiting in between (the source does not change)
          const int zb = chunk & 1;
          if (lane == 0) bulk_wait_read();
          __syncwarp();
          uint4* row_p = reinterpret_cast<uint4*>(stg + zb * kStageOutBytes + lane * 128);
#pragma unroll
          for (int q = 0; q < 8; ++q) row_p[q] = make_uint4(0u, 0u, 0u, 0u);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            for (int c = 0; c < kNOut && t.nb * kNOut + c < N; c += 32)
              tma_store3d(om, stg_addr + zb * kStageOutBytes, t.nb * kNOut + c,
                          t.mb * kPairM + static_cast<int>(rank) * kBM + quarter * 32, t.e);
            bulk_commit();
          }
          ++chunk;
        }
#pragma unroll 1
        for (int c = 0; any_k && c < kNOut; c += 32) {
          const int col = t.nb * kNOut + c;
          if (col >= N) break;
          uint32_t v[32];
          ld32(tb + c, v);
          ld_wait();
          // alternate staging blocks: the store issued two blocks ago (same block) has read it,
          // the previous block's store may still be reading the other one
          const int b = chunk & 1;
          if (lane == 0) bulk_wait_read_1();
          __syncwarp();
          uint4* row_p = reinterpret_cast<uint4*>(stg + b * kStageOutBytes + lane * 128);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            row_p[q ^ (lane & 7)] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            tma_store3d(om, stg_addr + b * kStageOutBytes, col,
                        t.mb * kPairM + static_cast<int>(rank) * kBM + quarter * 32, t.e);
            bulk_commit();
          }
          ++chunk;
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) {
        const uint32_t ae = acc == 0 ? acc_empty0 : acc_empty1;
        if (rank == 0) mbar_arrive(smem_addr(&acc_empty[acc]));
        else arrive_remote(ae);
      }
    }
  }

  if (MODE == kWeightGrad && warp >= 2 && lane == 0) bulk_wait_all();
  fence_before();
  __syncthreads();
  pair_sync();  // no MMA of the pair is in flight when either CTA frees its TMEM
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemColsBwd)
                 : "memory");
  }
}

// ---- combine backward and the router's gradient (warp per token) ---------------------------------
// d_eo[row] = bf16(fp32(w * dy)) for every kept slot; d_w[t,j] = <dy[t], eo[row]> (0 for a dropped
// slot); d_logits[t, :] from d_w (softmax backward); ones[t,j] = 1 when given (the unit weights of the final
// combine of the input gradients).
__global__ void __launch_bounds__(256)
    combine_bwd_kernel(const uint4* __restrict__ dy, const uint4* __restrict__ eo, int max_rows,
                       const int32_t* __restrict__ slot_row, const float* __restrict__ topk_w,
                       const int32_t* __restrict__ topk_idx, const float* __restrict__ logits,
                       int renormalize, int T, int k, int E, int H, uint4* __restrict__ d_eo,
                       float* __restrict__ d_w, float* __restrict__ d_logits,
                       float* __restrict__ ones) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int nv = H / 8;
  for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < T; t += gridDim.x * 8) {
    // slot j's routing data and, after its pass over H, its d_w live in lane j
    const int my_row = lane < k ? __ldg(slot_row + t * k + lane) : -1;
    const float my_w = lane < k ? __ldg(topk_w + t * k + lane) : 0.0f;
    int my_e = lane < k ? __ldg(topk_idx + t * k + lane) : -1;
    // an expert id outside [0, E) (rejected by the forward's dispatch) gives no d_logits entry
    if (static_cast<unsigned>(my_e) >= static_cast<unsigned>(E)) my_e = -1;
    float my_dw = 0.0f;
    const uint4* dy_row = dy + static_cast<size_t>(t) * nv;
    for (int j = 0; j < k; ++j) {
      const int row = __shfl_sync(0xFFFFFFFFu, my_row, j);
      if (row < 0 || row >= max_rows) continue;  // uniform over the warp
      const float w = __shfl_sync(0xFFFFFFFFu, my_w, j);
      const uint4* eo_row = eo + static_cast<size_t>(row) * nv;
      uint4* de_row = d_eo + static_cast<size_t>(row) * nv;
      float acc = 0.0f;
      for (int v = lane; v < nv; v += 32) {
        const uint4 g = ld_nc_v4(dy_row + v);  // the token's row: from L1 / L2 after the first slot
        const uint4 o = ld_nc_v4(eo_row + v);
        const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, ow[4] = {o.x, o.y, o.z, o.w};
        uint32_t pk[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float g0 = bf16_lo(gw[q]), g1 = bf16_hi(gw[q]);
          acc = fmaf(g0, bf16_lo(ow[q]), acc);
          acc = fmaf(g1, bf16_hi(ow[q]), acc);
          pk[q] = pack_bf16x2(__fmul_rn(w, g0), __fmul_rn(w, g1));
        }
        st_cs_v4(de_row + v, make_uint4(pk[0], pk[1], pk[2], pk[3]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
      if (lane == j) my_dw = acc;
    }
    if (lane < k) {
      d_w[t * k + lane] = my_dw;
      if (ones != nullptr) ones[t * k + lane] = 1.0f;
    }
    float* dl = d_logits + static_cast<size_t>(t) * E;
    if (renormalize) {
      // d_logits[e_j] = w_j (d_w_j - sum_i w_i d_w_i); the other experts get 0
      float c = my_w * my_dw;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
      for (int e = lane; e < E; e += 32) dl[e] = 0.0f;
      __syncwarp();
      if (my_e >= 0) dl[my_e] = my_w * (my_dw - c);
    } else {
      // p = softmax over all E logits; d_e = d_w of the slot that selected e, else 0
      const float* lg = logits + static_cast<size_t>(t) * E;
      float mx = -INFINITY;
      for (int e = lane; e < E; e += 32) mx = fmaxf(mx, __ldg(lg + e));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
      float sum = 0.0f;
      for (int e = lane; e < E; e += 32) sum += expf(__ldg(lg + e) - mx);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
      // sum_e p_e d_e over the selected experts only (d is 0 elsewhere)
      float pd = my_e >= 0 ? expf(__ldg(lg + my_e) - mx) / sum * my_dw : 0.0f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) pd += __shfl_xor_sync(0xFFFFFFFFu, pd, o);
      for (int e = lane; e < E; e += 32) dl[e] = -(expf(__ldg(lg + e) - mx) / sum) * pd;
      __syncwarp();
      if (my_e >= 0) {
        const float p = expf(__ldg(lg + my_e) - mx) / sum;
        dl[my_e] = p * (my_dw - pd);
      }
    }
  }
}

// ---- host ---------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// bf16 [rows, cols] (cols contiguous), boxes of box_cols (64: 128-byte swizzle; 32: 64-byte
// swizzle) x box_rows, out-of-range elements read as zero.
bool tmap_bf16(CUtensorMap* tm, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
               uint32_t box_cols = 64) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw =
      box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
size_t bwd_smem() {
  // stages, store staging, barriers, and the tile table (E + 1 entries; none for the weights)
  return 1024 + static_cast<size_t>(Cfg<MODE>::kStages) * Cfg<MODE>::kStageBytes +
         (MODE == kWeightGrad ? 8 * kStageOutBytes : 0) + 256 +
         (MODE == kWeightGrad ? 16 : 4 * (1024 + 1));
}

// fp32 [E][M][N] (N contiguous) written in 32 x 32 boxes from a 128-byte-swizzled staging block;
// elements outside [E][M][N] are not written.
bool tmap_f32_out(CUtensorMap* tm, void* ptr, uint64_t E, uint64_t M, uint64_t N) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {N, M, E};
  cuuint64_t strides[2] = {N * 4, M * N * 4};
  cuuint32_t box[3] = {32u, 32u, 1u};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_bwd_gemm(const BwdMaps& maps, const BwdArgs& a, cudaStream_t s) {
  const size_t smem = bwd_smem<MODE>();
  static int grid_of[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kBwdThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  if (grid_of[dev] == 0) {
    cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // as many pairs as can be resident at once (one CTA per SM)
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    cfg.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, bwd_gemm_kernel<MODE>, &cfg);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorLaunchOutOfResources;
    grid_of[dev] = 2 * min(clusters, num_sms() / 2);
  }
  cfg.gridDim = dim3(grid_of[dev]);
  cfg.numAttrs = MOE_USE_PDL ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, bwd_gemm_kernel<MODE>, maps, a);
}

}  // namespace

size_t backward_workspace_bytes(int max_rows, int T, int k, int H, int F) {
  const size_t r = static_cast<size_t>(max_rows > 0 ? max_rows : 1);
  const size_t tk = static_cast<size_t>(T > 0 ? T : 1) * static_cast<size_t>(k > 0 ? k : 1);
  auto up = [](size_t b) { return (b + 255) / 256 * 256; };
  // status | d_eo [r,H] | h, dg, du [r,F] | dx_rows [r,H] | ones [T,k]
  return 256 + up(r * H * 2) + 3 * up(r * F * 2) + up(r * H * 2) + up(tk * 4);
}

cudaError_t launch_combine_backward(const void* dy, int T, int H, int k, int E,
                                   const float* logits, int renormalize, const int32_t* topk_idx,
                                   const float* topk_w, const int32_t* slot_row, int max_rows,
                                   const void* expert_out, void* d_eo, float* d_topk_w,
                                   float* d_logits, float* ones, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  int blocks = (T + 7) / 8;
  if (blocks > 8 * num_sms()) blocks = 8 * num_sms();
  return launch_pdl(combine_bwd_kernel, dim3(blocks), dim3(256), 0, s,
                    static_cast<const uint4*>(dy), static_cast<const uint4*>(expert_out),
                    max_rows, slot_row, topk_w, topk_idx, logits, renormalize, T, k, E, H,
                    static_cast<uint4*>(d_eo), d_topk_w, d_logits, ones);
}

size_t expert_backward_workspace_bytes(int max_rows, int F) {
  const size_t r = static_cast<size_t>(max_rows > 0 ? max_rows : 1);
  return 256 + 3 * ((r * F * 2 + 255) / 256 * 256);  // status | h, dg, du [r, F]
}

cudaError_t launch_expert_backward(const void* ffn_input, const void* d_eo,
                                   const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                                   const void* w_gate, const void* w_up, const void* w_down,
                                   void* dx_rows, float* d_w_gate, float* d_w_up, float* d_w_down,
                                   int* status, void* h, void* dg, void* du, cudaStream_t s) {
  if (max_rows == 0) {
    // no rows at all: every expert's gradients are zero
    const size_t n = static_cast<size_t>(E) * H * F * sizeof(float);
    cudaError_t e = cudaMemsetAsync(d_w_gate, 0, n, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_w_up, 0, n, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_w_down, 0, n, s);
    return e;
  }
  BwdArgs a{expert_offsets, E, H, F, max_rows, nullptr, nullptr, nullptr, status};
  BwdMaps m1{}, m2{}, m3{};
  const uint64_t mr = static_cast<uint64_t>(max_rows);
  if (!tmap_bf16(&m1.m[0], ffn_input, mr, H, 128, 32) ||
      !tmap_bf16(&m1.m[1], d_eo, mr, H, 128, 32) ||
      !tmap_bf16(&m1.m[2], w_gate, static_cast<uint64_t>(E) * F, H, 128, 32) ||
      !tmap_bf16(&m1.m[3], w_up, static_cast<uint64_t>(E) * F, H, 128, 32) ||
      !tmap_bf16(&m1.m[4], w_down, static_cast<uint64_t>(E) * H, F, 32))
    return cudaErrorInvalidValue;
  if (!tmap_bf16(&m2.m[0], dg, mr, F, 128) || !tmap_bf16(&m2.m[1], du, mr, F, 128) ||
      !tmap_bf16(&m2.m[2], w_gate, static_cast<uint64_t>(E) * F, H, 64) ||
      !tmap_bf16(&m2.m[3], w_up, static_cast<uint64_t>(E) * F, H, 64))
    return cudaErrorInvalidValue;
  if (!tmap_bf16(&m3.m[0], d_eo, mr, H, 64) || !tmap_bf16(&m3.m[1], dg, mr, F, 64) ||
      !tmap_bf16(&m3.m[2], du, mr, F, 64) || !tmap_bf16(&m3.m[3], h, mr, F, 64) ||
      !tmap_bf16(&m3.m[4], ffn_input, mr, H, 64) ||
      !tmap_f32_out(&m3.out[0], d_w_down, E, H, F) || !tmap_f32_out(&m3.out[1], d_w_gate, E, F, H) ||
      !tmap_f32_out(&m3.out[2], d_w_up, E, F, H))
    return cudaErrorInvalidValue;
  a.out0 = h;
  a.out1 = dg;
  a.out2 = du;
  cudaError_t e = launch_bwd_gemm<kRecompute>(m1, a, s);
  if (e != cudaSuccess) return e;
  a.out0 = dx_rows;
  a.out1 = a.out2 = nullptr;
  e = launch_bwd_gemm<kInputGrad>(m2, a, s);
  if (e != cudaSuccess) return e;
  a.out0 = d_w_down;
  a.out1 = d_w_gate;
  a.out2 = d_w_up;
  e = launch_bwd_gemm<kWeightGrad>(m3, a, s);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_backward(const void* dy, int T, int H, int k, int E, int F, const float* logits,
                            int renormalize, const int32_t* topk_idx, const float* topk_w,
                            const int32_t* slot_row, const int32_t* expert_offsets, int max_rows,
                            const void* ffn_input, const void* expert_out, const void* w_gate,
                            const void* w_up, const void* w_down, void* dx, float* d_logits,
                            float* d_topk_w, float* d_w_gate, float* d_w_up, float* d_w_down,
                            void* ws, cudaStream_t s) {
  auto up = [](size_t b) { return (b + 255) / 256 * 256; };
  const size_t r = static_cast<size_t>(max_rows > 0 ? max_rows : 1);
  uint8_t* w = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(w);
  uint8_t* p = w + 256;
  void* d_eo = p;     p += up(r * H * 2);
  void* h = p;        p += up(r * F * 2);
  void* dg = p;       p += up(r * F * 2);
  void* du = p;       p += up(r * F * 2);
  void* dx_rows = p;  p += up(r * H * 2);
  float* ones = reinterpret_cast<float*>(p);
  if (T == 0) {
    return launch_expert_backward(ffn_input, d_eo, expert_offsets, 0, E, H, F, w_gate, w_up,
                                  w_down, dx_rows, d_w_gate, d_w_up, d_w_down, status, h, dg, du,
                                  s);
  }
  cudaError_t e = launch_combine_backward(dy, T, H, k, E, logits, renormalize, topk_idx, topk_w,
                                          slot_row, max_rows, expert_out, d_eo, d_topk_w,
                                          d_logits, ones, s);
  if (e != cudaSuccess) return e;
  e = launch_expert_backward(ffn_input, d_eo, expert_offsets, max_rows, E, H, F, w_gate, w_up,
                             w_down, dx_rows, d_w_gate, d_w_up, d_w_down, status, h, dg, du, s);
  if (e != cudaSuccess) return e;
  e = launch_combine(dx_rows, max_rows, slot_row, ones, T, k, H, dx, nullptr, s);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
