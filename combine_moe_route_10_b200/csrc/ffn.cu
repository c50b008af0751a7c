// Grouped SwiGLU expert FFN on the packed send buffer: tcgen05 tensor cores, TMEM accumulators,
// TMA-fed shared-memory pipelines.
//
// Per expert e and each of its packed rows x (expert-major layout of the NCCL EP page, section
// 2.1; two linear layers with SwiGLU per expert as in "细粒度专家并行方案对比：MegaMoE与传统方案",
// section 核心差异分析 1; fused w3_w1 projection with the SwiGLU epilogue, then w2, as in the
// run_moe passage of "DWDP: 在NVL72上的高性能分布式权重数据并行"):
//     h = bf16( silu(x W_gate[e]^T) * (x W_up[e]^T) ),   expert_out = bf16( h W_down[e]^T ).
//
// Two persistent kernels split the experts by size, each running all GEMM-1 tiles of its experts
// and then all their GEMM-2 tiles (a GEMM-2 tile waits on per-row-block completion counters of
// the GEMM-1 tiles), with tiles claimed at run time from a global counter:
//
// * ffn_pair_kernel: experts with more than 64 rows.  A 2-CTA cluster computes a tile of
//   (expert, pair of row blocks, column block) as one 256 x 256 product with
//   tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): CTA v holds its row block of A and rows
//   [128v, 128v + 128) of the 256 weight rows of B, so each SM stages half of the weight tile per
//   k-step, a stage is 32 KB and six are in flight; CTA v's TMEM receives its 128 rows x 256
//   columns.  GEMM-1 puts the gate rows in CTA 0's half of B and the up rows in CTA 1's.  CTA 1's
//   TMA loads complete their bytes on CTA 0's barriers, CTA 0's single MMA thread issues for both
//   and its commits arrive on both CTAs' barriers (multicast commit, not multicast loads).
// * ffn_single_kernel: experts with at most 64 rows (a tile is bound by streaming the expert's
//   weights, not by the MMA).  One CTA per tile: tcgen05.mma.cta_group::1 (M = 128, N = 256),
//   40 KB stages (an A box of 16, 32 or 64 rows + the whole weight tile), five in flight.
//
// Roles (192 threads): warp 0 = TMA producer (CTA 0 of a pair also claims tiles and passes the ids
// to both CTAs through shared-memory queues); warp 1 = TMEM allocation and the MMA thread;
// warps 2..5 = epilogue of the CTA's 128 rows: tcgen05.ld of the accumulator, then SwiGLU (GEMM-1:
// gate columns 0..127 and up columns 128..255 of one accumulator) or a bf16 cast (GEMM-2), masked
// row / column stores.  Two 256-column accumulators let the epilogue of one tile overlap the MMAs
// of the next.  Every mbarrier and counter wait is bounded; on a timeout a CTA records
// kStatusTimeout (and stops its peer), drains what it issued, and both CTAs of a pair meet at the
// final cluster barrier before TMEM is freed.  No TMA multicast anywhere.  The tile schedules are
// derived on the device from expert_offsets, so nothing is synchronised with the host.
// For the FP8 payload a separate pass (dequant_fp8_kernel) first writes the bf16 input rows.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

#include <string.h>

#include <vector>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int BM = 128;          // rows per CTA tile (one TMEM lane per row)
constexpr int BK = 64;           // k per stage: 64 bf16 = one 128-byte swizzle atom row
constexpr int UMMA_K = 16;       // k per tcgen05.mma for kind::f16
constexpr int kAccCols = 256;    // fp32 TMEM columns per accumulator
constexpr int kTmemCols = 512;   // two accumulators
constexpr int kThreads = 192;
constexpr int kATileBytes = BM * BK * 2;   // 16 KB: 128 rows of A
constexpr int kBHalfBytes = 128 * BK * 2;  // 16 KB: 128 weight rows
// Experts with at most this many rows run in the single-block kernel, the others in the pair kernel.
constexpr int kSingleMaxRows = 64;
// Pair kernel: six 32-KB stages (A rows + half of B).  Single kernel: five 40-KB stages (an A box of
// at most 64 rows + all 256 rows of B).
constexpr int kStagesPair = 6;
constexpr int kStagesSingle = 5;
constexpr int kASingleBytes = kSingleMaxRows * BK * 2;  // 8 KB
constexpr int kTileQ = 4;
// Consumers of a pair kernel's queue slot, all arriving on CTA 0's q_empty: CTA 0's MMA thread and
// four epilogue warps, CTA 1's producer and four epilogue warps.
constexpr int kPairQueueConsumers = 10;
constexpr int kSingleQueueConsumers = 5;  // the MMA thread and four epilogue warps

// ---- PTX wrappers ------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tm, uint32_t bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// CTA 1's copy into its own shared memory, completing its bytes on CTA 0's barrier `bar_cta0`
// (a shared::cluster address); a plain (not multicast) load.
__device__ __forceinline__ void tma_load_2d_to_leader(uint32_t dst, const CUtensorMap* tm,
                                                      uint32_t bar_cta0, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar_cta0)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
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
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// cta_group::1 (single kernel)
__device__ __forceinline__ void tc_commit1(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_mma1(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// kind::f8f6f4 (e4m3 x e4m3 -> fp32), the first projection with FP8 weights
__device__ __forceinline__ void tc_mma1_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_mma2_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// cta_group::2 (pair kernel)
// Arrive once on the mbarrier at this shared-memory offset in BOTH CTAs of the pair when the MMAs
// issued so far have completed.
__device__ __forceinline__ void tc_commit2_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}
// Arrive on this CTA's own mbarrier when the MMAs issued so far have completed.
__device__ __forceinline__ void tc_commit2_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_mma2(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ---- cluster helpers ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Shared::cluster address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(local), "r"(rank));
  return out;
}
__device__ __forceinline__ void st_cluster_s32(uint32_t cluster_addr, int v) {
  asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
// Arrive on an mbarrier of the other CTA, releasing this thread's prior writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cl(uint32_t bar, uint32_t parity) {
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
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Abort state of a CTA: its own flag and, in the pair kernel, the peer's flag, so that a timeout
// in either CTA ends the waits of both.
struct Abort {
  volatile int* local;
  uint32_t peer;  // shared::cluster address of the peer's flag (pair kernel only)
  bool has_peer;
  int* status;
  __device__ __forceinline__ void raise_timeout() const {
    *local = 1;
    if (has_peer) st_cluster_s32(peer, 1);
    record_status(status, kStatusTimeout);
  }
};

// Bounded wait on an mbarrier phase (arrivals may come from either CTA of a pair).  False if this
// CTA is aborting or the limit ran out (which raises the abort).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Abort& ab) {
  if (mbar_try_wait_cl(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if (*ab.local) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      ab.raise_timeout();
      return false;
    }
  }
}
// The same wait that ignores the abort flag (used to drain a CTA's own copies and MMAs).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait_cl(bar, parity)) return;
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait_cl(bar, parity) && global_timer_ns() - t0 <= kWaitLimitNs) {
  }
}

// Shared-memory matrix descriptor of a K-major bf16 tile stored with the 128-byte swizzle:
// rows of 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), descriptor version 1,
// layout type 2 (SWIZZLE_128B).  The leading byte offset is unused for swizzled K-major tiles.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;                // leading byte offset (16 B, unused)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;        // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                // SWIZZLE_128B
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator, bf16 A and B, both K-major.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N) {
  return (1u << 4)                                    // D format: f32
         | (1u << 7)                                  // A format: bf16
         | (1u << 10)                                 // B format: bf16
         | (static_cast<uint32_t>(N >> 3) << 17)      // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);     // M / 16
}

// Instruction descriptor of tcgen05.mma kind::f8f6f4: fp32 accumulator, e4m3 A and B (format code
// 0 for both), both K-major.
__host__ __device__ constexpr uint32_t make_idesc_e4m3(int M, int N) {
  return (1u << 4)                                    // D format: f32
         | (static_cast<uint32_t>(N >> 3) << 17)      // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);     // M / 16
}

__device__ __forceinline__ int owner_of(const int* start, int E, int idx) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {  // largest expert whose first unit is <= idx (it owns the tile)
    const int mid = (lo + hi + 1) >> 1;
    if (start[mid] <= idx) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
  return g / (1.0f + expf(-g)) * u;
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait until *p >= target (acquire).  False if the CTA aborts or the limit runs out.
__device__ __forceinline__ bool wait_counter(const int* p, int target, const Abort& ab) {
  if (ld_acquire(p) >= target) return true;
  const unsigned long long t0 = global_timer_ns();
  while (true) {
    __nanosleep(64);
    if (ld_acquire(p) >= target) return true;
    if (*ab.local) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      ab.raise_timeout();
      return false;
    }
  }
}

// Tensor maps of the A operand (input rows, h) with row boxes of 16, 32 and 64: a row block with
// few rows loads only the rows it has (the stale rows above them in shared memory feed only
// accumulator rows the epilogue does not store).
struct SmallBoxMaps {
  CUtensorMap m[3];
};
__host__ __device__ constexpr int small_box_rows(int i) { return 16 << i; }
__device__ __forceinline__ int small_box_index(int rows) {
  return rows <= 16 ? 0 : (rows <= 32 ? 1 : (rows <= 64 ? 2 : 3));
}
// Bytes of the A box that covers `rows` rows (0 when there are none).
__device__ __forceinline__ uint32_t a_box_bytes(int rows) {
  if (rows <= 0) return 0u;
  const int bi = small_box_index(rows);
  return bi < 3 ? static_cast<uint32_t>(small_box_rows(bi) * BK * 2) : kATileBytes;
}

// ---- tile schedule -------------------------------------------------------------------------------
//
// The tiles of a kernel are numbered [all GEMM-1 tiles][all GEMM-2 tiles] over the experts of its
// class; inside a phase expert by expert, column block by column block, with the units (row
// blocks, or pairs of row blocks) fastest, so tiles running together share a weight column block
// through L2.  A GEMM-2 tile reads the rows of h that the GEMM-1 tiles of its row block write, so
// its producer first waits (bounded) until the block's completion counter reaches 4 * n1 (four
// epilogue warps per GEMM-1 tile, n1 column blocks).  GEMM-1 tiles never wait, and every GEMM-1
// tile is claimed before any GEMM-2 tile, by a CTA that finishes it without waiting, so the waits
// of running CTAs always end; they are bounded anyway.  Writers: st.global of h, fence.proxy.async
// (generic -> async proxy), release increment.  Readers: acquire load of the counter,
// fence.proxy.async, then the TMA loads of h.
struct FfnArgs {
  const int32_t* expert_offsets;  // [E+1], device
  int E, max_rows, H, F;
  __nv_bfloat16* h;               // [max_rows, F] workspace
  __nv_bfloat16* out;             // [max_rows, H]
  int* status;
  int* done;                      // [row blocks] GEMM-1 completion counters, zero on entry
  int* used;                      // [row blocks] GEMM-2 tiles that passed the wait, zero on entry
  int* sched;                     // [2] this kernel's next tile to claim, CTAs that finished
  // Per-expert weight descriptors (moe_ffn_weight_list_init): 4 per expert (gate, up, down with
  // 128-row and 256-row boxes), rows local to the expert; nullptr: the grid-constant maps of the
  // contiguous [E, ...] weights, rows global.
  const CUtensorMap* wlist;
  // FP8 first projection (all three non-null) or bf16 (all null): the A and gate / up maps then
  // hold e4m3 codes, x_scale [max_rows] the input rows' scales, g_scale / u_scale [E*F] the
  // weight rows' scales.
  const float* x_scale;
  const float* g_scale;
  const float* u_scale;
};

// Elements of the K dimension one 128-byte swizzled smem row holds: 64 bf16 or 128 e4m3.
__device__ __forceinline__ int k_per_stage(const FfnArgs& a, int phase) {
  return (phase == 1 && a.x_scale != nullptr) ? 128 : BK;
}

// The descriptor of the weight tile a tile loads, and its first row.  `which`: 0 gate, 1 up,
// 2 down (128-row box), 3 down (256-row box); `local_row` is the row inside expert e's matrix.
__device__ __forceinline__ const CUtensorMap* weight_map(const FfnArgs& args, const CUtensorMap* tm,
                                                         int e, int which, int local_row,
                                                         int rows_per_expert, int& row) {
  if (args.wlist == nullptr) {
    row = e * rows_per_expert + local_row;
    return tm;
  }
  const CUtensorMap* m = args.wlist + 4 * e + which;
  // the descriptors were written to global memory by a copy before this launch
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(
                   reinterpret_cast<uint64_t>(m))
               : "memory");
  row = local_row;
  return m;
}

struct Tables {
  int* off;     // [E+1] row offsets (clamped to [0, max_rows])
  int* mt;      // [E]   row blocks per expert
  int* units;   // [E]   units of this kernel's class per expert (0 for the other class)
  int* ms_rb;   // [E+1] first global row block of each expert (over all experts)
  int* ms_u;    // [E+1] first unit of each expert among this kernel's units
  int* stats;   // [2]   experts of the single-block kernel, pairs of row blocks of the others
};
__host__ __device__ constexpr int table_ints(int E) { return 5 * E + 5; }

__device__ __forceinline__ Tables carve_tables(int* p, int E) {
  Tables t;
  t.off = p;
  t.mt = t.off + (E + 1);
  t.units = t.mt + E;
  t.ms_rb = t.units + E;
  t.ms_u = t.ms_rb + (E + 1);
  t.stats = t.ms_u + (E + 1);
  return t;
}

// One warp builds the tables from expert_offsets (warp scans).  PAIRS: the units are pairs of row
// blocks of the experts with more than kSingleMaxRows rows; otherwise the single row block of each
// of the others.
template <bool PAIRS>
__device__ __forceinline__ void build_tables(const Tables& tb, const FfnArgs& args, int lane) {
  const int E = args.E;
  int carry_r = 0, carry_u = 0, n_single = 0, n_pairs = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    int lo = 0, hi = 0;
    if (e < E) {
      // L2 loads: the pair kernel may start before the kernel ahead of it has finished
      lo = min(max(__ldcg(args.expert_offsets + e), 0), args.max_rows);
      hi = min(max(__ldcg(args.expert_offsets + e + 1), 0), args.max_rows);
    }
    const int mt = (max(hi - lo, 0) + BM - 1) / BM;
    const bool paired = hi - lo > kSingleMaxRows;
    const int u = PAIRS ? (paired ? (mt + 1) / 2 : 0) : (paired ? 0 : mt);
    n_single += __popc(__ballot_sync(0xFFFFFFFFu, !paired && mt == 1));
    n_pairs += paired ? (mt + 1) / 2 : 0;
    int ir = mt, iu = u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yr = __shfl_up_sync(0xFFFFFFFFu, ir, o);
      const int yu = __shfl_up_sync(0xFFFFFFFFu, iu, o);
      if (lane >= o) {
        ir += yr;
        iu += yu;
      }
    }
    if (e < E) {
      tb.off[e] = lo;
      tb.mt[e] = mt;
      tb.units[e] = u;
      tb.ms_rb[e] = carry_r + ir - mt;
      tb.ms_u[e] = carry_u + iu - u;
    }
    carry_r += __shfl_sync(0xFFFFFFFFu, ir, 31);
    carry_u += __shfl_sync(0xFFFFFFFFu, iu, 31);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n_pairs += __shfl_xor_sync(0xFFFFFFFFu, n_pairs, o);
  if (lane == 0) {
    tb.ms_rb[E] = carry_r;
    tb.ms_u[E] = carry_u;
    tb.off[E] = min(max(__ldcg(args.expert_offsets + E), 0), args.max_rows);
    tb.stats[0] = n_single;
    tb.stats[1] = n_pairs;
  }
}

// CTAs of the single-block kernel that work while the pair kernel runs beside it on the other
// SMs: the grid's share of the two kinds of work, each at a per-SM rate.  A single-block expert
// streams its 3 H F bf16 weights (85 GB/s per SM) and a pair of row blocks does 6 * 256 * H * F
// flops (9 TFLOP/s per SM on the 2-CTA tiles), so the ratio does not depend on H and F.  The scale
// factor 1.5 was the best of 1.0 / 1.5 / 2.0 / 2.5 / 3.0 on B200 for a routing with 100 single-block
// experts beside 29 larger ones (FFN 3.61-3.64 ms against 3.69-3.77 at 1.0; the two kinds slow each
// other down when they run together).  Rounded to whole clusters of two, at least one cluster
// when there is such work.
#ifndef MOE_SINGLE_SHARE_SCALE
#define MOE_SINGLE_SHARE_SCALE 1.5f
#endif
__device__ __forceinline__ int single_kernel_ctas(const Tables& tb, int grid) {
  const int n_single = tb.stats[0], n_pairs = tb.stats[1];
  if (n_single == 0) return 0;
  if (n_pairs == 0) return grid;
  const float t_single = static_cast<float>(n_single) * 6.0f / 85e9f;
  const float t_pairs = static_cast<float>(n_pairs) * 1536.0f / 9e12f;
  const float share = MOE_SINGLE_SHARE_SCALE * t_single / (t_single + t_pairs);
  int g = 2 * static_cast<int>(0.5f * share * static_cast<float>(grid) + 0.5f);
  return max(2, min(grid, g));
}

struct FTile {
  int phase;  // 1: GEMM-1 (SwiGLU), 2: GEMM-2 (down)
  int e, unit, n_blk;
};

__device__ __forceinline__ FTile fdecode(const Tables& tb, int E, int n1, int n2, int tile) {
  FTile t;
  const int U = tb.ms_u[E];
  int nt, idx;
  if (tile < U * n1) {
    t.phase = 1;
    nt = n1;
    idx = tile;
  } else {
    t.phase = 2;
    nt = n2;
    idx = tile - U * n1;
  }
  t.e = owner_of(tb.ms_u, E, idx / nt);
  const int local = idx - nt * tb.ms_u[t.e];
  const int u = tb.units[t.e];
  t.n_blk = local / u;
  t.unit = local - t.n_blk * u;
  return t;
}

// GEMM-2 producer side of row block m_blk of expert e: wait for its rows of h, then the last of the
// n2 GEMM-2 tiles of the block to get here returns both counters to zero, so the workspace is
// ready for the next call without a memset.
__device__ __forceinline__ bool gemm2_acquire(const FfnArgs& args, const Tables& tb, int e,
                                              int m_blk, int n1, int n2, const Abort& ab) {
  const int rb = tb.ms_rb[e] + m_blk;
  if (!wait_counter(args.done + rb, 4 * n1, ab)) return false;
  asm volatile("fence.proxy.async.global;" ::: "memory");
  if (atomicAdd(args.used + rb, 1) == n2 - 1) {
    atomicExch(args.done + rb, 0);
    atomicExch(args.used + rb, 0);
  }
  return true;
}

// Epilogue of one accumulator for this warp's 32 rows (r_local) of row block m_blk of expert e.
__device__ __forceinline__ void epilogue_tile(const FfnArgs& args, const Tables& tb, int phase,
                                              int e, int m_blk, int n_blk, uint32_t t_row,
                                              int r_local, int lane) {
  const int row = tb.off[e] + m_blk * BM + r_local;
  const bool row_ok = row < tb.off[e + 1];
  if (phase == 1) {
    __nv_bfloat16* out_row = args.h + static_cast<size_t>(row) * args.F;
    const bool w8 = args.x_scale != nullptr;
    const float sx = (w8 && row_ok) ? args.x_scale[row] : 1.0f;
#pragma unroll 1
    for (int c = 0; c < 128; c += 32) {
      uint32_t g[32], u[32];
      tmem_ld32(t_row + c, g);
      tmem_ld32(t_row + 128 + c, u);
      tmem_wait_ld();
      const int col = n_blk * 128 + c;
      if (row_ok && col < args.F) {
        // FP8 first projection: g = sx * sw * sum(qx qw), the row's scale times each weight row's
        // scale (columns past F read as 0; they are not stored).  F % 64 == 0, so a 32-column chunk
        // is either wholly inside F or wholly outside.
        const float2* sg2 = w8 ? reinterpret_cast<const float2*>(args.g_scale + static_cast<size_t>(e) * args.F + col) : nullptr;
        const float2* su2 = w8 ? reinterpret_cast<const float2*>(args.u_scale + static_cast<size_t>(e) * args.F + col) : nullptr;
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
          float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
          if (w8) {
            const float2 a = __ldg(sg2 + i), b = __ldg(su2 + i);
            g0 *= sx * a.x;
            g1 *= sx * a.y;
            u0 *= sx * b.x;
            u1 *= sx * b.y;
          }
          packed[i] = pack_bf16x2(silu_mul(g0, u0), silu_mul(g1, u1));
        }
        uint4* dst = reinterpret_cast<uint4*>(out_row + col);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
      }
    }
    if (m_blk < tb.mt[e]) {
      // publish: this warp's rows of h for (e, block, n) are written
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __threadfence();
      __syncwarp();
      if (lane == 0) red_release_add(args.done + tb.ms_rb[e] + m_blk, 1);
    }
  } else {
    __nv_bfloat16* out_row = args.out + static_cast<size_t>(row) * args.H;
#pragma unroll 1
    for (int c = 0; c < 256; c += 32) {
      uint32_t v[32];
      tmem_ld32(t_row + c, v);
      tmem_wait_ld();
      const int col = n_blk * 256 + c;
      if (row_ok && col < args.H) {
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
        uint4* dst = reinterpret_cast<uint4*>(out_row + col);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
      }
    }
  }
}

// Shared-memory layout common to both kernels: the stage ring, the mbarriers, the tile queue and
// the tables.
struct Ring {
  uint8_t* tiles;
  uint64_t *full, *empty, *acc_full, *acc_empty, *drain, *q_full, *q_empty;
  int* tile_q;  // [kTileQ] claimed tile ids (-1: no more tiles)
  uint32_t* tmem_base;
  int* abort_flag;
  Tables tb;
};

__device__ __forceinline__ Ring carve(uint8_t* raw, int E, int stages, int stage_bytes) {
  Ring s;
  const uint32_t a = smem_addr(raw);
  uint8_t* p = raw + ((1024u - (a & 1023u)) & 1023u);
  s.tiles = p;
  p += static_cast<size_t>(stages) * stage_bytes;
  s.full = reinterpret_cast<uint64_t*>(p);
  s.empty = s.full + stages;
  s.acc_full = s.empty + stages;
  s.acc_empty = s.acc_full + 2;
  s.drain = s.acc_empty + 2;
  s.q_full = s.drain + 1;
  s.q_empty = s.q_full + kTileQ;
  s.tmem_base = reinterpret_cast<uint32_t*>(s.q_empty + kTileQ);
  s.abort_flag = reinterpret_cast<int*>(s.tmem_base + 1);
  s.tile_q = s.abort_flag + 2;
  s.tb = carve_tables(s.tile_q + kTileQ, E);
  return s;
}

size_t ring_smem_bytes(int E, int stages, int stage_bytes) {
  return 1024 + static_cast<size_t>(stages) * stage_bytes +
         8 * (2 * static_cast<size_t>(stages) + 5 + 2 * kTileQ) + 16 +
         sizeof(int) * (static_cast<size_t>(table_ints(E)) + 2 + kTileQ);
}

__device__ __forceinline__ void init_ring(const Ring& s, int stages, int acc_empty_count,
                                          int q_consumers) {
  for (int i = 0; i < stages; ++i) {
    mbar_init(smem_addr(&s.full[i]), 1);
    mbar_init(smem_addr(&s.empty[i]), 1);
  }
  for (int i = 0; i < 2; ++i) {
    mbar_init(smem_addr(&s.acc_full[i]), 1);
    mbar_init(smem_addr(&s.acc_empty[i]), acc_empty_count);
  }
  mbar_init(smem_addr(s.drain), 1);
  for (int i = 0; i < kTileQ; ++i) {
    mbar_init(smem_addr(&s.q_full[i]), 1);
    mbar_init(smem_addr(&s.q_empty[i]), q_consumers);
  }
  *s.abort_flag = 0;
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Next tile id from this CTA's queue (bounded).  remote_empty: the slot's q_empty is CTA 0's.
__device__ __forceinline__ bool take_tile(const Ring& s, int& qi, uint32_t& qph, bool remote_empty,
                                          const Abort& ab, int& tile) {
  if (!wait_bar(smem_addr(&s.q_full[qi]), qph, ab)) return false;
  tile = s.tile_q[qi];
  const uint32_t qe = smem_addr(&s.q_empty[qi]);
  if (remote_empty)
    mbar_arrive_cluster(peer_addr(qe, 0));
  else
    mbar_arrive(qe);
  if (++qi == kTileQ) {
    qi = 0;
    qph ^= 1u;
  }
  return true;
}

// The epilogue warps' queue step: lane 0 takes the tile, every lane advances its slot index.
__device__ __forceinline__ bool warp_take_tile(const Ring& s, int& qi, uint32_t& qph,
                                               bool remote_empty, const Abort& ab, int lane,
                                               int& tile) {
  bool okq = true;
  tile = -1;
  if (lane == 0) {
    okq = take_tile(s, qi, qph, remote_empty, ab, tile);
  } else if (++qi == kTileQ) {
    qi = 0;
    qph ^= 1u;
  }
  okq = __shfl_sync(0xFFFFFFFFu, okq ? 1 : 0, 0) != 0;
  tile = __shfl_sync(0xFFFFFFFFu, tile, 0);
  return okq;
}

// Prefetch of the descriptors in kernel parameter space (the weight maps only when they are used).
__device__ __forceinline__ void prefetch_maps(const CUtensorMap* a, const CUtensorMap* b,
                                              const CUtensorMap* c, const CUtensorMap* d,
                                              const CUtensorMap* e, const SmallBoxMaps& xs,
                                              const SmallBoxMaps& hs, bool weights) {
  const CUtensorMap* all[5] = {a, d, b, c, e};  // x, h, then the three weight maps
  for (int i = 0; i < (weights ? 5 : 2); ++i)
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(all[i])) : "memory");
  for (int i = 0; i < 3; ++i) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xs.m[i])) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&hs.m[i])) : "memory");
  }
}

// Every claim of this CTA is done: the last CTA of the grid to get here returns this kernel's
// claim counters to zero.
__device__ __forceinline__ void release_schedule(int* sched) {
  __threadfence();
  if (atomicAdd(sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
    atomicExch(sched, 0);
    atomicExch(sched + 1, 0);
  }
}

// ================================================================================================
// Pair kernel: experts with more than kSingleMaxRows rows; 2-CTA clusters, cta_group::2.
// ================================================================================================
__global__ void __launch_bounds__(kThreads, 1)
    ffn_pair_kernel(const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ SmallBoxMaps tm_xs,
                    const __grid_constant__ CUtensorMap tm_g,
                    const __grid_constant__ CUtensorMap tm_u,
                    const __grid_constant__ CUtensorMap tm_h,
                    const __grid_constant__ SmallBoxMaps tm_hs,
                    const __grid_constant__ CUtensorMap tm_d128, const FfnArgs args) {
  constexpr int kStages = kStagesPair;
  constexpr int kStageBytes = kATileBytes + kBHalfBytes;
  extern __shared__ uint8_t smem_raw[];
  const int E = args.E;
  const Ring s = carve(smem_raw, E, kStages, kStageBytes);
  const Tables& tb = s.tb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // CTA 0 claims the tiles and issues the MMAs
  const int n1 = (args.F + 127) / 128;   // GEMM-1 column blocks (128 h columns each)
  const int n2 = (args.H + 255) / 256;   // GEMM-2 column blocks (256 output columns each)
  const int ks1 = k_per_stage(args, 1);  // K elements per GEMM-1 stage: 64 bf16 or 128 e4m3
  const int kb1 = (args.H + ks1 - 1) / ks1, kb2 = (args.F + BK - 1) / BK;
  const bool w8 = args.x_scale != nullptr;
  const Abort ab{s.abort_flag, peer_addr(smem_addr(s.abort_flag), rank ^ 1u), true, args.status};

  if (warp == 0) {
    if (lane == 0) {
      init_ring(s, kStages, 8, kPairQueueConsumers);  // acc_empty: four epilogue warps per CTA
      prefetch_maps(&tm_x, &tm_g, &tm_u, &tm_h, &tm_d128, tm_xs, tm_hs, args.wlist == nullptr);
    }
  } else if (warp == 1) {
    // the same warp of both CTAs allocates, as cta_group::2 requires
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(s.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  } else if (warp == 2) {
    build_tables<true>(tb, args, lane);
  }
  // No wait for the single-block kernel launched ahead: its experts are disjoint from these, and
  // this grid can only start once every CTA of that kernel has passed its own wait for the
  // dispatch, so the packed rows and offsets are complete (they are read through L2).  The wait at
  // the end makes this grid's completion imply that kernel's too.
  griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_base;
  const int U = tb.ms_u[E];
  const int total_tiles = U * (n1 + n2);
  const uint32_t tiles_base = smem_addr(s.tiles);
  volatile int* abort_flag = s.abort_flag;

  if (warp == 0) {
    // ---- TMA producer of this CTA's A rows and B half ------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      int qi = 0;
      uint32_t qph = 0;
      while (!*abort_flag) {
        int tile;
        if (rank == 0) {
          tile = atomicAdd(args.sched, 1);
          if (tile >= total_tiles) tile = -1;
          // hand the id to the consumers of both CTAs
          if (!wait_bar(smem_addr(&s.q_empty[qi]), qph ^ 1u, ab)) break;
          s.tile_q[qi] = tile;
          st_cluster_s32(peer_addr(smem_addr(&s.tile_q[qi]), 1), tile);
          mbar_arrive(smem_addr(&s.q_full[qi]));
          mbar_arrive_cluster(peer_addr(smem_addr(&s.q_full[qi]), 1));
          if (++qi == kTileQ) {
            qi = 0;
            qph ^= 1u;
          }
        } else {
          if (!take_tile(s, qi, qph, true, ab, tile)) break;
        }
        if (tile < 0) break;
        const FTile t = fdecode(tb, E, n1, n2, tile);
        const int m_blk = 2 * t.unit + static_cast<int>(rank);  // this CTA's row block
        const int row_a = tb.off[t.e] + m_blk * BM;
        const int rows = m_blk < tb.mt[t.e] ? min(BM, tb.off[t.e + 1] - row_a) : 0;
        const int bi = small_box_index(rows);
        // CTA 0's barrier counts both CTAs' bytes of each stage
        const int row_a1 = tb.off[t.e] + (2 * t.unit + 1) * BM;
        const int rows1 = 2 * t.unit + 1 < tb.mt[t.e] ? min(BM, tb.off[t.e + 1] - row_a1) : 0;
        const int row_a0 = tb.off[t.e] + 2 * t.unit * BM;
        const int rows0 = min(BM, tb.off[t.e + 1] - row_a0);
        const uint32_t stage_tx = a_box_bytes(rows0) + a_box_bytes(rows1) + 2 * kBHalfBytes;
        int nkb;
        const CUtensorMap *ma, *mb;
        int row_b;
        if (t.phase == 1) {
          nkb = kb1;
          ma = bi < 3 ? &tm_xs.m[bi] : &tm_x;
          // gate rows -> accumulator columns 0..127, up rows -> 128..255
          mb = weight_map(args, rank == 0 ? &tm_g : &tm_u, t.e, static_cast<int>(rank),
                          t.n_blk * 128, args.F, row_b);
        } else {
          if (rows > 0 && !gemm2_acquire(args, tb, t.e, m_blk, n1, n2, ab)) break;
          nkb = kb2;
          ma = bi < 3 ? &tm_hs.m[bi] : &tm_h;
          mb = weight_map(args, &tm_d128, t.e, 2, t.n_blk * 256 + static_cast<int>(rank) * 128,
                          args.H, row_b);
        }
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_bar(smem_addr(&s.empty[stage]), phase ^ 1u, ab)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = tiles_base + stage * kStageBytes;
          const uint32_t b_dst = a_dst + kATileBytes;
          const uint32_t fb = smem_addr(&s.full[stage]);
          const int kx = kb * (t.phase == 1 ? ks1 : BK);
          if (rank == 0) {
            mbar_arrive_expect_tx(fb, stage_tx);
            if (rows > 0) tma_load_2d(a_dst, ma, fb, kx, row_a);
            tma_load_2d(b_dst, mb, fb, kx, row_b);
          } else {
            const uint32_t fb0 = peer_addr(fb, 0);
            if (rows > 0) tma_load_2d_to_leader(a_dst, ma, fb0, kx, row_a);
            tma_load_2d_to_leader(b_dst, mb, fb0, kx, row_b);
          }
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        if (rank == 0) {
          // CTA 0's barriers count both CTAs' bytes: wait for the latest phase of each stage
          for (int st = 0; st < kStages; ++st)
            if (issued_mask & (1u << st)) drain_wait(smem_addr(&s.full[st]), (issued_parity >> st) & 1u);
        } else if (issued_mask != 0) {
          // CTA 1's copies complete on CTA 0's barriers: give them time to land (a copy takes
          // microseconds) before this CTA may leave
          const unsigned long long t0 = global_timer_ns();
          while (global_timer_ns() - t0 < 100000ull) __nanosleep(1000);
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer (CTA 0): M = 256 over the pair, N = 256 ------------------------------------
    if (rank == 0 && lane == 0) {
      const uint32_t idesc16 = make_idesc(2 * BM, 256), idesc8 = make_idesc_e4m3(2 * BM, 256);
      int stage = 0;
      uint32_t phase = 0;
      bool issued_any = false;
      int qi = 0;
      uint32_t qph = 0;
      for (int it = 0;; ++it) {
        int tile;
        if (!take_tile(s, qi, qph, false, ab, tile)) break;
        if (tile < 0) break;
        const bool g1 = tile < U * n1;
        const int nkb = g1 ? kb1 : kb2;
        const bool f8 = g1 && w8;  // e4m3 operands: K = 32 per MMA, the same 32 bytes of a row
        const int acc = it & 1;
        const uint32_t acc_parity = (it >> 1) & 1;
        if (!wait_bar(smem_addr(&s.acc_empty[acc]), acc_parity ^ 1u, ab)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_bar(smem_addr(&s.full[stage]), phase, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = tiles_base + stage * kStageBytes;
          const uint32_t b_addr = a_addr + kATileBytes;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            const uint64_t ad = sw128_desc(a_addr + kk * 32), bd = sw128_desc(b_addr + kk * 32);
            if (f8)
              tc_mma2_f8(d_tmem, ad, bd, idesc8, (kb | kk) != 0 ? 1u : 0u);
            else
              tc_mma2(d_tmem, ad, bd, idesc16, (kb | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          tc_commit2_both(smem_addr(&s.empty[stage]));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit2_both(smem_addr(&s.acc_full[acc]));
      }
      if (issued_any) {
        tc_commit2_local(smem_addr(s.drain));
        drain_wait(smem_addr(s.drain), 0);
      }
    }
  } else {
    // ---- epilogue of this CTA's 128 rows ---------------------------------------------------------
    const int quarter = warp & 3;
    const int r_local = quarter * 32 + lane;
    const uint32_t acc_empty0 = smem_addr(&s.acc_empty[0]);
    int qi = 0;
    uint32_t qph = 0;
    for (int it = 0;; ++it) {
      int tile;
      if (!warp_take_tile(s, qi, qph, rank != 0, ab, lane, tile) || tile < 0) break;
      const FTile t = fdecode(tb, E, n1, n2, tile);
      const int acc = it & 1;
      const uint32_t acc_parity = (it >> 1) & 1;
      bool ok = true;
      if (lane == 0) ok = wait_bar(smem_addr(&s.acc_full[acc]), acc_parity, ab);
      if (!__shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + acc * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16);
      epilogue_tile(args, tb, t.phase, t.e, 2 * t.unit + static_cast<int>(rank), t.n_blk, t_row,
                    r_local, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        const uint32_t ae = acc_empty0 + acc * 8;
        if (rank == 0)
          mbar_arrive(ae);
        else
          mbar_arrive_cluster(peer_addr(ae, 0));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) release_schedule(args.sched);
  // neither CTA leaves (or frees TMEM) while the other may still touch its shared memory or TMEM
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
  }
  griddep_wait();  // the single-block kernel ahead has completed too
}

// ================================================================================================
// Single kernel: experts with one row block; one CTA per tile, cta_group::1.
// ================================================================================================
__global__ void __launch_bounds__(kThreads, 1)
    ffn_single_kernel(const __grid_constant__ CUtensorMap tm_x,
                      const __grid_constant__ SmallBoxMaps tm_xs,
                      const __grid_constant__ CUtensorMap tm_g,
                      const __grid_constant__ CUtensorMap tm_u,
                      const __grid_constant__ CUtensorMap tm_h,
                      const __grid_constant__ SmallBoxMaps tm_hs,
                      const __grid_constant__ CUtensorMap tm_d256, const FfnArgs args) {
  constexpr int kStages = kStagesSingle;
  constexpr int kBTileBytes = 2 * kBHalfBytes;  // all 256 weight rows
  constexpr int kStageBytes = kASingleBytes + kBTileBytes;
  // The MMA reads 128 A rows: rows 64..127 come from the B tile behind the A box and feed only
  // accumulator rows that are never stored (the expert has at most 64 rows).
  extern __shared__ uint8_t smem_raw[];
  const int E = args.E;
  const Ring s = carve(smem_raw, E, kStages, kStageBytes);
  const Tables& tb = s.tb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n1 = (args.F + 127) / 128;
  const int n2 = (args.H + 255) / 256;
  const int ks1 = k_per_stage(args, 1);  // K elements per GEMM-1 stage: 64 bf16 or 128 e4m3
  const int kb1 = (args.H + ks1 - 1) / ks1, kb2 = (args.F + BK - 1) / BK;
  const bool w8 = args.x_scale != nullptr;
  const Abort ab{s.abort_flag, 0u, false, args.status};

  if (warp == 0) {
    if (lane == 0) {
      init_ring(s, kStages, 4, kSingleQueueConsumers);
      prefetch_maps(&tm_x, &tm_g, &tm_u, &tm_h, &tm_d256, tm_xs, tm_hs, args.wlist == nullptr);
    }
  } else if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(s.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  } else if (warp == 2) {
    griddep_wait();
    build_tables<false>(tb, args, lane);
  }
  griddep_wait();
  // the pair kernel launched behind this one may start as soon as every CTA gets here
  griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_base;
  const int U = tb.ms_u[E];
  const int total_tiles = U * (n1 + n2);
  const uint32_t tiles_base = smem_addr(s.tiles);
  volatile int* abort_flag = s.abort_flag;
  // This grid is launched as 2-CTA clusters, one CTA per SM; only the first single_kernel_ctas()
  // CTAs work, the others leave at once so that the pair kernel gets their SMs (whole pairs).
  const bool working = static_cast<int>(blockIdx.x) < single_kernel_ctas(tb, gridDim.x);

  if (!working) {
    // nothing to do: fall through to the common exit
  } else if (warp == 0) {
    // ---- TMA producer ----------------------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      int qi = 0;
      uint32_t qph = 0;
      while (!*abort_flag) {
        int tile = atomicAdd(args.sched, 1);
        if (tile >= total_tiles) tile = -1;
        // hand the id to the MMA thread and the epilogue warps
        if (!wait_bar(smem_addr(&s.q_empty[qi]), qph ^ 1u, ab)) break;
        s.tile_q[qi] = tile;
        mbar_arrive(smem_addr(&s.q_full[qi]));
        if (++qi == kTileQ) {
          qi = 0;
          qph ^= 1u;
        }
        if (tile < 0) break;
        const FTile t = fdecode(tb, E, n1, n2, tile);
        const int m_blk = t.unit;
        const int row_a = tb.off[t.e] + m_blk * BM;
        const int rows = min(kSingleMaxRows, tb.off[t.e + 1] - row_a);
        const int bi = small_box_index(rows);  // 16, 32 or 64 rows
        const uint32_t stage_tx = a_box_bytes(rows) + kBTileBytes;
        int nkb;
        const CUtensorMap *ma, *mb0, *mb1 = nullptr;
        int row_b;
        if (t.phase == 1) {
          nkb = kb1;
          ma = &tm_xs.m[bi];
          mb0 = weight_map(args, &tm_g, t.e, 0, t.n_blk * 128, args.F, row_b);
          mb1 = weight_map(args, &tm_u, t.e, 1, t.n_blk * 128, args.F, row_b);
        } else {
          if (!gemm2_acquire(args, tb, t.e, m_blk, n1, n2, ab)) break;
          nkb = kb2;
          ma = &tm_hs.m[bi];
          mb0 = weight_map(args, &tm_d256, t.e, 3, t.n_blk * 256, args.H, row_b);
        }
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_bar(smem_addr(&s.empty[stage]), phase ^ 1u, ab)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = tiles_base + stage * kStageBytes;
          const uint32_t b_dst = a_dst + kASingleBytes;
          const uint32_t fb = smem_addr(&s.full[stage]);
          const int kx = kb * (t.phase == 1 ? ks1 : BK);
          mbar_arrive_expect_tx(fb, stage_tx);
          tma_load_2d(a_dst, ma, fb, kx, row_a);
          if (t.phase == 1) {
            // gate rows -> B rows 0..127 (accumulator columns 0..127), up rows -> 128..255
            tma_load_2d(b_dst, mb0, fb, kx, row_b);
            tma_load_2d(b_dst + kBHalfBytes, mb1, fb, kx, row_b);
          } else {
            tma_load_2d(b_dst, mb0, fb, kx, row_b);
          }
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        for (int st = 0; st < kStages; ++st)
          if (issued_mask & (1u << st)) drain_wait(smem_addr(&s.full[st]), (issued_parity >> st) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer (M = 128, N = 256) ---------------------------------------------------------
    if (lane == 0) {
      const uint32_t idesc16 = make_idesc(BM, 256), idesc8 = make_idesc_e4m3(BM, 256);
      int stage = 0;
      uint32_t phase = 0;
      bool issued_any = false;
      int qi = 0;
      uint32_t qph = 0;
      for (int it = 0;; ++it) {
        int tile;
        if (!take_tile(s, qi, qph, false, ab, tile)) break;
        if (tile < 0) break;
        const bool g1 = tile < U * n1;
        const int nkb = g1 ? kb1 : kb2;
        const bool f8 = g1 && w8;  // e4m3 operands: K = 32 per MMA, the same 32 bytes of a row
        const int acc = it & 1;
        const uint32_t acc_parity = (it >> 1) & 1;
        if (!wait_bar(smem_addr(&s.acc_empty[acc]), acc_parity ^ 1u, ab)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_bar(smem_addr(&s.full[stage]), phase, ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = tiles_base + stage * kStageBytes;
          const uint32_t b_addr = a_addr + kASingleBytes;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            const uint64_t ad = sw128_desc(a_addr + kk * 32), bd = sw128_desc(b_addr + kk * 32);
            if (f8)
              tc_mma1_f8(d_tmem, ad, bd, idesc8, (kb | kk) != 0 ? 1u : 0u);
            else
              tc_mma1(d_tmem, ad, bd, idesc16, (kb | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          tc_commit1(smem_addr(&s.empty[stage]));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit1(smem_addr(&s.acc_full[acc]));
      }
      if (issued_any) {
        tc_commit1(smem_addr(s.drain));
        drain_wait(smem_addr(s.drain), 0);
      }
    }
  } else {
    // ---- epilogue --------------------------------------------------------------------------------
    const int quarter = warp & 3;
    const int r_local = quarter * 32 + lane;
    int qi = 0;
    uint32_t qph = 0;
    for (int it = 0;; ++it) {
      int tile;
      if (!warp_take_tile(s, qi, qph, false, ab, lane, tile) || tile < 0) break;
      const FTile t = fdecode(tb, E, n1, n2, tile);
      const int acc = it & 1;
      const uint32_t acc_parity = (it >> 1) & 1;
      bool ok = true;
      if (lane == 0) ok = wait_bar(smem_addr(&s.acc_full[acc]), acc_parity, ab);
      if (!__shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + acc * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16);
      epilogue_tile(args, tb, t.phase, t.e, t.unit, t.n_blk, t_row, r_local, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&s.acc_empty[acc]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) release_schedule(args.sched);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// FP8 payload -> bf16 FFN input rows: x = bf16(fp32(code) * scale), rows [0, expert_offsets[E]).
__global__ void __launch_bounds__(256)
    dequant_fp8_kernel(const uint8_t* __restrict__ q, const float* __restrict__ scales,
                       const int32_t* __restrict__ total_rows, int max_rows, int H,
                       uint4* __restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const int S = min(__ldg(total_rows), max_rows);
  const int per_row = H / 16;  // 16 codes per thread step
  const long long n = static_cast<long long>(S) * per_row;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / per_row;
    const int c16 = static_cast<int>(i - row * per_row);
    const uint4 codes = ld_nc_v4(q + i * 16);
    const float sc = __ldg(scales + row * (H / 128) + (c16 * 16) / 128);
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>(w[j] >> (16 * h));
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);  // exact
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        o[2 * j + h] = pack_bf16x2(__fmul_rn(f.x, sc), __fmul_rn(f.y, sc));
      }
    }
    out[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    out[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// FP8 rows with one scale per row (FP8 weights, and the FFN's own input rows for the FP8 first
// projection): one warp per row.  scale = amax / 448 (1 when amax == 0); code = e4m3
// round-to-nearest-even, saturating, of the fp32 IEEE quotient value / scale.  Rows [0, n) with
// n = min(*n_rows_dev, n_rows) when n_rows_dev is given, else n_rows.
__global__ void __launch_bounds__(256)
    quant_rows_fp8_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ n_rows_dev,
                          int n_rows, int K, uint8_t* __restrict__ codes,
                          float* __restrict__ scales) {
  griddep_wait();
  griddep_launch_dependents();
  const int rows = n_rows_dev != nullptr ? min(__ldg(n_rows_dev), n_rows) : n_rows;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int nv = K / 8;  // 16-byte vectors of 8 bf16 per row
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < rows; r += gridDim.x * wpb) {
    const uint4* row = src + static_cast<size_t>(r) * nv;
    float amax = 0.0f;
    for (int v = lane; v < nv; v += 32) {
      const uint4 w = ld_nc_v4(row + v);
      const uint32_t q[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(q[i])), fabsf(bf16_hi(q[i]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const float sc = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
    uint2* out = reinterpret_cast<uint2*>(codes + static_cast<size_t>(r) * K);
    for (int v = lane; v < nv; v += 32) {
      const uint4 w = ld_nc_v4(row + v);
      const uint32_t q[4] = {w.x, w.y, w.z, w.w};
      uint32_t packed[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 pr = make_float2(__fdiv_rn(bf16_lo(q[i]), sc), __fdiv_rn(bf16_hi(q[i]), sc));
        packed[i] = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3));
      }
      out[v] = make_uint2(packed[0] | (packed[1] << 16), packed[2] | (packed[3] << 16));
    }
    if (lane == 0) scales[r] = sc;
  }
}

// ---- host side -----------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2-D bf16 tensor [rows, cols] (cols contiguous) read in boxes of box_rows x 64 with the
// 128-byte swizzle; out-of-range elements read as zero.
bool make_tmap(CUtensorMap* tm, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D tensor of bytes (e4m3 codes) [rows, cols] read in boxes of box_rows x 128 with the 128-byte
// swizzle: the same shared-memory rows as a box_rows x 64 bf16 box.
bool make_tmap_u8(CUtensorMap* tm, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t launch_quant_rows(const void* src, const int32_t* n_rows_dev, int n_rows, int K,
                              void* codes, float* scales, cudaStream_t s) {
  if (n_rows == 0) return cudaSuccess;
  long long blocks = (static_cast<long long>(n_rows) + 7) / 8;
  const long long cap = static_cast<long long>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  return launch_pdl(quant_rows_fp8_kernel, dim3(static_cast<int>(blocks)), dim3(256), 0, s,
                    static_cast<const uint4*>(src), n_rows_dev, n_rows, K,
                    static_cast<uint8_t*>(codes), scales);
}

}  // namespace

cudaError_t launch_quantize_rows_fp8(const void* x, int rows, int K, void* codes, float* scales,
                                     cudaStream_t s) {
  const cudaError_t err = launch_quant_rows(x, nullptr, rows, K, codes, scales, s);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

// Persistent grid of 2-CTA clusters of `kernel`: as many clusters as can be resident at once (one
// CTA per SM), looked up once per device, kernel and shared-memory size.
using FfnKernel = void (*)(CUtensorMap, SmallBoxMaps, CUtensorMap, CUtensorMap, CUtensorMap,
                           SmallBoxMaps, CUtensorMap, FfnArgs);
static cudaError_t cluster_grid(FfnKernel kernel, const cudaLaunchConfig_t& cfg_in, int* grid) {
  struct Entry {
    int dev;
    FfnKernel kernel;
    size_t smem;
    int grid;
  };
  static Entry cache[16];
  static int n_cache = 0;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  for (int i = 0; i < n_cache; ++i)
    if (cache[i].dev == dev && cache[i].kernel == kernel &&
        cache[i].smem == cfg_in.dynamicSmemBytes) {
      *grid = cache[i].grid;
      return cudaSuccess;
    }
  cudaLaunchConfig_t cfg = cfg_in;
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  int clusters = 0;
  err = cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg);
  if (err != cudaSuccess) return err;
  if (clusters < 1) return cudaErrorInvalidConfiguration;
  *grid = 2 * (clusters < num_sms() / 2 ? clusters : num_sms() / 2);
  if (n_cache < 16) cache[n_cache++] = Entry{dev, kernel, cfg_in.dynamicSmemBytes, *grid};
  return cudaSuccess;
}

// Workspace: [0,4) status | [256, ..) h bf16 [max_rows, F] | (FP8) dequantised rows bf16
// [max_rows, H] | GEMM-1 completion counters and GEMM-2 arrival counters, int32
// [2][max_rows/128 + E + 1] | the claim and finished-CTA counters of the pair and of the single
// kernel, int32 [4].
static size_t round256(size_t b) { return (b + 255) / 256 * 256; }
static size_t ffn_counter_count(int max_rows, int E) {
  return static_cast<size_t>(max_rows) / BM + static_cast<size_t>(E) + 1;
}

// W8 (FP8 first projection): after the dequantised rows, the input rows' e4m3 codes [max_rows, H]
// and their scales fp32 [max_rows].
static size_t ffn_w8_bytes(int max_rows, int H) {
  return round256(static_cast<size_t>(max_rows) * H) + round256(static_cast<size_t>(max_rows) * 4);
}

size_t ffn_workspace_bytes(int max_rows, int H, int F, int fp8, int E, int w8) {
  const size_t h_bytes = round256(static_cast<size_t>(max_rows) * F * 2);
  const size_t x_bytes = fp8 ? round256(static_cast<size_t>(max_rows) * H * 2) : 0;
  const size_t q_bytes = w8 ? ffn_w8_bytes(max_rows, H) : 0;
  return 256 + h_bytes + x_bytes + q_bytes +
         round256((2 * ffn_counter_count(max_rows, E) + 4) * sizeof(int));
}

size_t ffn_weight_list_bytes(int E) { return static_cast<size_t>(E) * 4 * sizeof(CUtensorMap); }

cudaError_t ffn_weight_list_init(const void* const* w_gate, const void* const* w_up,
                                 const void* const* w_down, int E, int H, int F, void* list,
                                 cudaStream_t s) {
  std::vector<CUtensorMap> maps(static_cast<size_t>(E) * 4);
  for (int e = 0; e < E; ++e) {
    CUtensorMap* m = maps.data() + 4 * static_cast<size_t>(e);
    if (!make_tmap(m + 0, w_gate[e], F, H, 128) || !make_tmap(m + 1, w_up[e], F, H, 128) ||
        !make_tmap(m + 2, w_down[e], H, F, 128) || !make_tmap(m + 3, w_down[e], H, F, 256))
      return cudaErrorInvalidValue;
  }
  // from pageable memory: the call returns once the host array has been taken
  return cudaMemcpyAsync(list, maps.data(), ffn_weight_list_bytes(E), cudaMemcpyHostToDevice, s);
}

cudaError_t launch_expert_ffn(const void* send, const float* send_scales, int fp8,
                              const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                              const void* w_gate, const void* w_up, const void* w_down,
                              const void* wlist, const float* w_gate_scale,
                              const float* w_up_scale, void* expert_out, void* ws,
                              cudaStream_t s) {
  if (max_rows == 0) return cudaSuccess;
  const bool w8 = w_gate_scale != nullptr;
  char* base = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(base);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(base + 256);
  size_t off = 256 + round256(static_cast<size_t>(max_rows) * F * 2);
  uint4* xdq = nullptr;
  if (fp8) {
    xdq = reinterpret_cast<uint4*>(base + off);
    off += round256(static_cast<size_t>(max_rows) * H * 2);
  }
  uint8_t* xq = nullptr;
  float* xs = nullptr;
  if (w8) {
    xq = reinterpret_cast<uint8_t*>(base + off);
    xs = reinterpret_cast<float*>(base + off + round256(static_cast<size_t>(max_rows) * H));
    off += ffn_w8_bytes(max_rows, H);
  }
  int* done = reinterpret_cast<int*>(base + off);
  int* used = done + ffn_counter_count(max_rows, E);
  int* sched = used + ffn_counter_count(max_rows, E);  // [0..1] pair kernel, [2..3] single kernel
  // all counters are zero on entry (zero-filled workspace, reset by the previous call)
  cudaError_t err = cudaSuccess;
  const void* a_src = send;
  if (fp8) {
    const long long work = static_cast<long long>(max_rows) * (H / 16);
    long long blocks = (work + 255) / 256;
    const long long cap = static_cast<long long>(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    err = launch_pdl(dequant_fp8_kernel, dim3(static_cast<int>(blocks)), dim3(256), 0, s,
                     static_cast<const uint8_t*>(send), send_scales, expert_offsets + E, max_rows,
                     H, xdq);
    if (err != cudaSuccess) return err;
    a_src = xdq;
  }
  if (w8) {
    // the FFN input rows, each quantised on its own: e4m3 codes and one scale per row
    err = launch_quant_rows(a_src, expert_offsets + E, max_rows, H, xq, xs, s);
    if (err != cudaSuccess) return err;
  }
  CUtensorMap tm_x, tm_g, tm_u, tm_h, tm_d128, tm_d256;
  SmallBoxMaps tm_xs, tm_hs;
  for (int i = 0; i < 3; ++i)
    if (!(w8 ? make_tmap_u8(&tm_xs.m[i], xq, max_rows, H, small_box_rows(i))
             : make_tmap(&tm_xs.m[i], a_src, max_rows, H, small_box_rows(i))) ||
        !make_tmap(&tm_hs.m[i], h, max_rows, F, small_box_rows(i)))
      return cudaErrorInvalidValue;
  if (!(w8 ? make_tmap_u8(&tm_x, xq, max_rows, H, BM) : make_tmap(&tm_x, a_src, max_rows, H, BM)) ||
      !make_tmap(&tm_h, h, max_rows, F, BM))
    return cudaErrorInvalidValue;
  if (w8) {
    // e4m3 gate / up codes [E * F, H]; the down projection stays bf16
    if (!make_tmap_u8(&tm_g, w_gate, static_cast<uint64_t>(E) * F, H, 128) ||
        !make_tmap_u8(&tm_u, w_up, static_cast<uint64_t>(E) * F, H, 128) ||
        !make_tmap(&tm_d128, w_down, static_cast<uint64_t>(E) * H, F, 128) ||
        !make_tmap(&tm_d256, w_down, static_cast<uint64_t>(E) * H, F, 256))
      return cudaErrorInvalidValue;
  } else if (wlist != nullptr) {
    // the kernels take each expert's descriptors from the list; these are never read
    memset(&tm_g, 0, sizeof(CUtensorMap));
    memset(&tm_u, 0, sizeof(CUtensorMap));
    memset(&tm_d128, 0, sizeof(CUtensorMap));
    memset(&tm_d256, 0, sizeof(CUtensorMap));
  } else if (!make_tmap(&tm_g, w_gate, static_cast<uint64_t>(E) * F, H, 128) ||
             !make_tmap(&tm_u, w_up, static_cast<uint64_t>(E) * F, H, 128) ||
             !make_tmap(&tm_d128, w_down, static_cast<uint64_t>(E) * H, F, 128) ||
             !make_tmap(&tm_d256, w_down, static_cast<uint64_t>(E) * H, F, 256)) {
    return cudaErrorInvalidValue;
  }
  const CUtensorMap* wl = static_cast<const CUtensorMap*>(wlist);

  // Both kernels are persistent grids of 2-CTA clusters, one CTA per SM.  The single-block kernel
  // goes first: its CTAs beyond its share of the work leave at once, and the pair kernel, launched
  // programmatically behind it, starts on those SMs without waiting for it (it waits at its end).
  const FfnArgs fa_single{expert_offsets, E, max_rows, H, F, h,
                          static_cast<__nv_bfloat16*>(expert_out), status, done, used, sched + 2,
                          wl, xs, w_gate_scale, w_up_scale};
  const FfnArgs fa_pair{expert_offsets, E, max_rows, H, F, h,
                        static_cast<__nv_bfloat16*>(expert_out), status, done, used, sched, wl,
                        xs, w_gate_scale, w_up_scale};
  const size_t smem_single = ring_smem_bytes(E, kStagesSingle, kASingleBytes + 2 * kBHalfBytes);
  const size_t smem_pair = ring_smem_bytes(E, kStagesPair, kATileBytes + kBHalfBytes);
  err = cudaFuncSetAttribute(ffn_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_single));
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(ffn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_pair));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  int grid_single = 0, grid_pair = 0;
  cfg.numAttrs = 1;
  cfg.dynamicSmemBytes = smem_single;
  err = cluster_grid(ffn_single_kernel, cfg, &grid_single);
  if (err != cudaSuccess) return err;
  cfg.dynamicSmemBytes = smem_pair;
  err = cluster_grid(ffn_pair_kernel, cfg, &grid_pair);
  if (err != cudaSuccess) return err;
  cfg.numAttrs = MOE_USE_PDL ? 2 : 1;
  cfg.gridDim = dim3(grid_single);
  cfg.dynamicSmemBytes = smem_single;
  err = cudaLaunchKernelEx(&cfg, ffn_single_kernel, tm_x, tm_xs, tm_g, tm_u, tm_h, tm_hs, tm_d256,
                           fa_single);
  if (err != cudaSuccess) return err;
  cfg.gridDim = dim3(grid_pair);
  cfg.dynamicSmemBytes = smem_pair;
  err = cudaLaunchKernelEx(&cfg, ffn_pair_kernel, tm_x, tm_xs, tm_g, tm_u, tm_h, tm_hs, tm_d128,
                           fa_pair);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace moe
