// Grouped SwiGLU expert FFN on the packed send buffer: tcgen05 tensor cores, TMEM accumulators,
// TMA-fed shared-memory pipeline.
//
// Per expert e and each of its packed rows x (expert-major layout of the NCCL EP page, section
// 2.1; two linear layers with SwiGLU per expert as in "细粒度专家并行方案对比：MegaMoE与传统方案",
// section 核心差异分析 1; fused w3_w1 projection with the SwiGLU epilogue, then w2, as in the
// run_moe passage of "DWDP: 在NVL72上的高性能分布式权重数据并行"):
//     h = bf16( silu(x W_gate[e]^T) * (x W_up[e]^T) ),   expert_out = bf16( h W_down[e]^T ).
//
// One persistent launch (one CTA per SM, 192 threads) runs the GEMM-1 tiles and then the GEMM-2
// tiles (the latter wait on per-row-block completion counters of the former); each CTA claims its
// next tile at run time from a global counter:
//   warp 0      TMA producer: claims tiles, passes their ids to the other roles through a small
//               shared-memory queue, and loads an A tile (128 rows x 64 k; 16/32/64 rows for a
//               small row block) + B tile (256 rows x 64 k) per stage, 128-byte swizzle, 4-stage
//               mbarrier ring;
//   warp 1      TMEM allocator and MMA issuer: one thread issues tcgen05.mma (M=128, N=256,
//               K=16, bf16 -> fp32) into one of two 256-column TMEM accumulators, and
//               tcgen05.commit frees smem stages / publishes finished accumulators;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (one TMEM lane quarter per warp), then
//               SwiGLU (GEMM-1: gate columns 0..127 and up columns 128..255 of one accumulator)
//               or a plain bf16 cast (GEMM-2), masked row/column stores.
// The tile schedule (expert, row block, column block) is derived on the device from
// expert_offsets, so nothing is synchronised with the host.  Row blocks of an expert are the
// fastest-varying index, so CTAs running together share weight column blocks through L2.
// Every mbarrier and counter wait is bounded; on a timeout the CTA records MOE status bit
// kStatusTimeout, drains its own outstanding TMA loads and MMAs, frees TMEM and returns.
// For the FP8 payload a separate pass (dequant_fp8_kernel) first writes the bf16 input rows.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int BM = 128;          // rows per tile (UMMA M, one TMEM lane per row)
constexpr int BK = 64;           // k per stage: 64 bf16 = one 128-byte swizzle atom row
constexpr int UMMA_K = 16;       // k per tcgen05.mma for kind::f16
constexpr int kStages = 4;
constexpr int kAccCols = 256;    // fp32 TMEM columns per accumulator
constexpr int kTmemCols = 512;   // two accumulators
constexpr int kThreads = 192;
constexpr int kATileBytes = BM * BK * 2;   // 16 KB
constexpr int kBTileBytes = 256 * BK * 2;  // 32 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes;

// Experts with at least this many 128-row blocks are "hot" (their weight blocks are reused from L2
// by several row blocks, so their tiles are tensor-bound); their tiles are interleaved evenly with
// the other experts' tiles, which stream weights from HBM, so both kinds run at the same time.
// 0 disables the interleave (plain expert order).
#ifndef MOE_FFN_HOT_MTILES
#define MOE_FFN_HOT_MTILES 2
#endif
constexpr int kGemm2NTile = 256;  // output columns per GEMM-2 tile (128 measured slower)
// Tiles are claimed at run time from a global counter by the producer; a kTileQ-deep shared-memory
// queue passes the ids to the MMA thread and the epilogue warps.
constexpr int kTileQ = 4;


// ---- PTX wrappers ------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tm, uint32_t bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
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

__device__ __forceinline__ int owner_of(const int* start, int E, int idx) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {  // largest expert whose first tile is <= idx (it owns the tile)
    const int mid = (lo + hi + 1) >> 1;
    if (start[mid] <= idx) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
  return g / (1.0f + expf(-g)) * u;
}

// ---- fused FFN: GEMM-1 (gate|up + SwiGLU) and GEMM-2 (down) tiles in one persistent launch -------
//
// Tiles are numbered [all GEMM-1 tiles][all GEMM-2 tiles]; CTAs claim them in increasing order
// from an atomic counter.
// A GEMM-2 tile (expert e, row block m) reads the rows of h that the GEMM-1 tiles of (e, m) write,
// so its producer first waits (bounded) until the completion counter of (e, m) reaches 4 * n1 (four
// epilogue warps per GEMM-1 tile, n1 column blocks).  GEMM-1 tiles never wait, and every GEMM-1
// tile is claimed before any GEMM-2 tile, by a CTA that finishes it without waiting, so with all
// CTAs resident (one per SM) the waits always end; they are bounded anyway.  Writers: st.global of h, fence.proxy.async (generic -> async proxy), release increment.
// Readers: acquire load of the counter, fence.proxy.async, then the TMA loads of h.
struct FfnArgs {
  const int32_t* expert_offsets;  // [E+1], device
  int E, max_rows, H, F;
  __nv_bfloat16* h;               // [max_rows, F] workspace
  __nv_bfloat16* out;             // [max_rows, H]
  int* status;
  int* done;                      // [row blocks] GEMM-1 completion counters, zero on entry
  int* used;                      // [row blocks] GEMM-2 tiles that passed the wait, zero on entry
  int* sched;                     // [2] next tile to claim, CTAs that finished; zero on entry
};

struct FSmem {
  uint8_t* tiles;
  uint64_t *full, *empty, *acc_full, *acc_empty, *drain, *q_full, *q_empty;
  int* tile_q;   // [kTileQ] claimed tile ids (-1: no more tiles)
  uint32_t* tmem_base;
  int* abort_flag;
  int* off;      // [E+1] row offsets (clamped to max_rows)
  int* mt;       // [E]   row blocks per expert
  int* ms_all;   // [E+1] first global row block of each expert
  int* ms_cold;  // [E+1] first row block of each non-hot expert among non-hot row blocks
  int* ms_hot;   // [E+1] same among hot row blocks
  int* totals;   // [2] non-hot, hot row blocks
};

__device__ __forceinline__ FSmem fcarve(uint8_t* raw, int E) {
  FSmem s;
  const uint32_t a = smem_addr(raw);
  uint8_t* p = raw + ((1024u - (a & 1023u)) & 1023u);
  s.tiles = p;
  p += kStages * kStageBytes;
  s.full = reinterpret_cast<uint64_t*>(p);
  s.empty = s.full + kStages;
  s.acc_full = s.empty + kStages;
  s.acc_empty = s.acc_full + 2;
  s.drain = s.acc_empty + 2;
  s.q_full = s.drain + 1;
  s.q_empty = s.q_full + kTileQ;
  s.tmem_base = reinterpret_cast<uint32_t*>(s.q_empty + kTileQ);
  s.abort_flag = reinterpret_cast<int*>(s.tmem_base + 1);
  s.tile_q = s.abort_flag + 2;
  s.off = s.tile_q + kTileQ;
  s.mt = s.off + (E + 1);
  s.ms_all = s.mt + E;
  s.ms_cold = s.ms_all + (E + 1);
  s.ms_hot = s.ms_cold + (E + 1);
  s.totals = s.ms_hot + (E + 1);
  return s;
}

size_t fused_smem_bytes(int E) {
  return 1024 + static_cast<size_t>(kStages) * kStageBytes + 8 * (2 * kStages + 5 + 2 * kTileQ) +
         16 + sizeof(int) * (5 * static_cast<size_t>(E) + 8 + kTileQ);
}

struct FTile {
  int phase;  // 1: GEMM-1 (SwiGLU), 2: GEMM-2 (down)
  int e, m_blk, n_blk, mg;
};

// Tile -> phase, expert, row block, column block (row blocks fastest inside an expert); hot and
// non-hot experts' tiles are spread evenly over each phase as in the two-launch kernel.
__device__ __forceinline__ FTile fdecode(const FSmem& s, int E, int n1, int n2, int tile) {
  FTile t;
  const int MC = s.totals[0], MH = s.totals[1];
  const int N1 = (MC + MH) * n1;
  int nt, idx;
  if (tile < N1) {
    t.phase = 1;
    nt = n1;
    idx = tile;
  } else {
    t.phase = 2;
    nt = n2;
    idx = tile - N1;
  }
  const int* ms = s.ms_cold;
  if (MH > 0) {
    if (MC == 0) {
      ms = s.ms_hot;
    } else {
      const long long Nt = static_cast<long long>(MC + MH) * nt;
      const long long hn = static_cast<long long>(MH) * nt;
      const long long h0 = static_cast<long long>(idx) * hn / Nt;
      const long long h1 = static_cast<long long>(idx + 1) * hn / Nt;
      if (h1 > h0) {
        ms = s.ms_hot;
        idx = static_cast<int>(h0);
      } else {
        idx -= static_cast<int>(h0);
      }
    }
  }
  t.e = owner_of(ms, E, idx / nt);
  const int local = idx - nt * ms[t.e];
  const int mt = s.mt[t.e];
  t.n_blk = local / mt;
  t.m_blk = local - t.n_blk * mt;
  t.mg = s.ms_all[t.e] + t.m_blk;
  return t;
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
__device__ __forceinline__ bool wait_counter(const int* p, int target, volatile int* abort_flag,
                                             int* status) {
  if (ld_acquire(p) >= target) return true;
  const unsigned long long t0 = global_timer_ns();
  while (true) {
    __nanosleep(64);
    if (ld_acquire(p) >= target) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      record_status(status, kStatusTimeout);
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

__global__ void __launch_bounds__(kThreads, 1)
    fused_ffn_kernel(const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ SmallBoxMaps tm_xs,
                     const __grid_constant__ CUtensorMap tm_g,
                     const __grid_constant__ CUtensorMap tm_u,
                     const __grid_constant__ CUtensorMap tm_h,
                     const __grid_constant__ SmallBoxMaps tm_hs,
                     const __grid_constant__ CUtensorMap tm_d, const FfnArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const int E = args.E;
  FSmem s = fcarve(smem_raw, E);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n1 = (args.F + 127) / 128;       // GEMM-1 column blocks (128 h columns each)
  const int n2 = (args.H + 255) / 256;       // GEMM-2 column blocks (256 output columns each)
  const int kb1 = (args.H + BK - 1) / BK, kb2 = (args.F + BK - 1) / BK;
  volatile int* abort_flag = s.abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < kStages; ++i) {
        mbar_init(smem_addr(&s.full[i]), 1);
        mbar_init(smem_addr(&s.empty[i]), 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(smem_addr(&s.acc_full[i]), 1);
        mbar_init(smem_addr(&s.acc_empty[i]), 4);
      }
      mbar_init(smem_addr(s.drain), 1);
      for (int i = 0; i < kTileQ; ++i) {
        mbar_init(smem_addr(&s.q_full[i]), 1);
        mbar_init(smem_addr(&s.q_empty[i]), 5);  // the MMA thread and the four epilogue warps
      }
      *s.abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_x)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_g)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_u)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_h)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_d)) : "memory");
      for (int i = 0; i < 3; ++i) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_xs.m[i]))
                     : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_hs.m[i]))
                     : "memory");
      }
    }
  } else if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(s.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  } else if (warp == 2) {
    griddep_wait();
    int carry_a = 0, carry_c = 0, carry_h = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      int lo = 0, hi = 0;
      if (e < E) {
        lo = min(__ldg(args.expert_offsets + e), args.max_rows);
        hi = min(__ldg(args.expert_offsets + e + 1), args.max_rows);
      }
      const int mt = (max(hi - lo, 0) + BM - 1) / BM;
      const bool hot = MOE_FFN_HOT_MTILES > 0 && mt >= MOE_FFN_HOT_MTILES;
      const int mc = hot ? 0 : mt, mh = hot ? mt : 0;
      int ia = mt, ic = mc, ih = mh;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xFFFFFFFFu, ia, o);
        const int yc = __shfl_up_sync(0xFFFFFFFFu, ic, o);
        const int yh = __shfl_up_sync(0xFFFFFFFFu, ih, o);
        if (lane >= o) {
          ia += ya;
          ic += yc;
          ih += yh;
        }
      }
      if (e < E) {
        s.off[e] = lo;
        s.mt[e] = mt;
        s.ms_all[e] = carry_a + ia - mt;
        s.ms_cold[e] = carry_c + ic - mc;
        s.ms_hot[e] = carry_h + ih - mh;
      }
      carry_a += __shfl_sync(0xFFFFFFFFu, ia, 31);
      carry_c += __shfl_sync(0xFFFFFFFFu, ic, 31);
      carry_h += __shfl_sync(0xFFFFFFFFu, ih, 31);
    }
    if (lane == 0) {
      s.ms_all[E] = carry_a;
      s.ms_cold[E] = carry_c;
      s.ms_hot[E] = carry_h;
      s.totals[0] = carry_c;
      s.totals[1] = carry_h;
      s.off[E] = min(__ldg(args.expert_offsets + E), args.max_rows);
    }
  }
  griddep_wait();
  griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_base;
  const int total_tiles = (s.totals[0] + s.totals[1]) * (n1 + n2);
  const uint32_t tiles_base = smem_addr(s.tiles);

  if (warp == 0) {
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
        if (!wait_phase(smem_addr(&s.q_empty[qi]), qph ^ 1u, abort_flag, args.status)) break;
        s.tile_q[qi] = tile;
        mbar_arrive(smem_addr(&s.q_full[qi]));
        if (++qi == kTileQ) {
          qi = 0;
          qph ^= 1u;
        }
        if (tile < 0) break;
        const FTile t = fdecode(s, E, n1, n2, tile);
        const int row_a = s.off[t.e] + t.m_blk * BM;
        // rows of this block: the A box shrinks to 16 / 32 / 64 rows when that covers them
        const int bi = small_box_index(min(BM, s.off[t.e + 1] - row_a));
        const uint32_t stage_tx = (bi < 3 ? small_box_rows(bi) * BK * 2 : kATileBytes) + kBTileBytes;
        int nkb;
        const CUtensorMap *ma, *mb;
        int row_b;
        if (t.phase == 1) {
          nkb = kb1;
          ma = bi < 3 ? &tm_xs.m[bi] : &tm_x;
          mb = &tm_g;
          row_b = t.e * args.F + t.n_blk * 128;
        } else {
          // the rows of h this tile reads are complete once all GEMM-1 tiles of (e, m) are
          if (!wait_counter(args.done + t.mg, 4 * n1, abort_flag, args.status)) break;
          asm volatile("fence.proxy.async.global;" ::: "memory");
          // the last of the n2 GEMM-2 tiles of (e, m) to get here returns both counters to zero,
          // so the workspace is ready for the next call without a memset
          if (atomicAdd(args.used + t.mg, 1) == n2 - 1) {
            atomicExch(args.done + t.mg, 0);
            atomicExch(args.used + t.mg, 0);
          }
          nkb = kb2;
          ma = bi < 3 ? &tm_hs.m[bi] : &tm_h;
          mb = &tm_d;
          row_b = t.e * args.H + t.n_blk * 256;
        }
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_phase(smem_addr(&s.empty[stage]), phase ^ 1u, abort_flag, args.status)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = tiles_base + stage * kStageBytes;
          const uint32_t b_dst = a_dst + kATileBytes;
          const uint32_t fb = smem_addr(&s.full[stage]);
          mbar_arrive_expect_tx(fb, stage_tx);
          tma_load_2d(a_dst, ma, fb, kb * BK, row_a);
          tma_load_2d(b_dst, mb, fb, kb * BK, row_b);
          if (t.phase == 1) tma_load_2d(b_dst + kBTileBytes / 2, &tm_u, fb, kb * BK, row_b);
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
        volatile int no_abort = 0;
        for (int st = 0; st < kStages; ++st)
          if (issued_mask & (1u << st))
            wait_phase(smem_addr(&s.full[st]), (issued_parity >> st) & 1u, &no_abort,
                       args.status);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer (M=128, N=256 for both phases) -------------------------------------------------
    if (lane == 0) {
      const uint32_t idesc = make_idesc(BM, 256);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool issued_any = false;
      int qi = 0;
      uint32_t qph = 0;
      for (;; ++it) {
        if (!wait_phase(smem_addr(&s.q_full[qi]), qph, abort_flag, args.status)) break;
        const int tile = s.tile_q[qi];
        mbar_arrive(smem_addr(&s.q_empty[qi]));
        if (++qi == kTileQ) {
          qi = 0;
          qph ^= 1u;
        }
        if (tile < 0) break;
        const int nkb = tile < (s.totals[0] + s.totals[1]) * n1 ? kb1 : kb2;
        const int acc = it & 1;
        const uint32_t acc_parity = (it >> 1) & 1;
        if (!wait_phase(smem_addr(&s.acc_empty[acc]), acc_parity ^ 1u, abort_flag, args.status))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_phase(smem_addr(&s.full[stage]), phase, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = tiles_base + stage * kStageBytes;
          const uint32_t b_addr = a_addr + kATileBytes;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            tc_mma(d_tmem, sw128_desc(a_addr + kk * UMMA_K * 2),
                   sw128_desc(b_addr + kk * UMMA_K * 2), idesc, (kb | kk) != 0 ? 1u : 0u);
          issued_any = true;
          tc_commit(smem_addr(&s.empty[stage]));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(smem_addr(&s.acc_full[acc]));
      }
      if (issued_any) {
        tc_commit(smem_addr(s.drain));
        volatile int no_abort = 0;
        wait_phase(smem_addr(s.drain), 0, &no_abort, args.status);
      }
    }
  } else {
    // ---- epilogue ----------------------------------------------------------------------------------
    const int quarter = warp & 3;
    const int r_local = quarter * 32 + lane;
    int it = 0;
    int qi = 0;
    uint32_t qph = 0;
    for (;; ++it) {
      int tile = -1;
      bool okq = true;
      if (lane == 0) {
        okq = wait_phase(smem_addr(&s.q_full[qi]), qph, abort_flag, args.status);
        if (okq) {
          tile = s.tile_q[qi];
          mbar_arrive(smem_addr(&s.q_empty[qi]));
        }
      }
      if (++qi == kTileQ) {
        qi = 0;
        qph ^= 1u;
      }
      okq = __shfl_sync(0xFFFFFFFFu, okq ? 1 : 0, 0) != 0;
      tile = __shfl_sync(0xFFFFFFFFu, tile, 0);
      if (!okq || tile < 0) break;
      const FTile t = fdecode(s, E, n1, n2, tile);
      const int acc = it & 1;
      const uint32_t acc_parity = (it >> 1) & 1;
      bool ok = true;
      if (lane == 0) ok = wait_phase(smem_addr(&s.acc_full[acc]), acc_parity, abort_flag, args.status);
      if (!__shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0)) break;
      tc_fence_after();
      const int row = s.off[t.e] + t.m_blk * BM + r_local;
      const bool row_ok = row < s.off[t.e + 1];
      const uint32_t t_row = tmem_base + acc * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16);
      if (t.phase == 1) {
        __nv_bfloat16* out_row = args.h + static_cast<size_t>(row) * args.F;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(t_row + c, g);
          tmem_ld32(t_row + 128 + c, u);
          tmem_wait_ld();
          const int col = t.n_blk * 128 + c;
          if (row_ok && col < args.F) {
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i]));
              const float h1 = silu_mul(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1]));
              packed[i] = pack_bf16x2(h0, h1);
            }
            uint4* dst = reinterpret_cast<uint4*>(out_row + col);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
          }
        }
        // publish: this warp's rows of h for (e, m, n) are written
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_add(args.done + t.mg, 1);
      } else {
        __nv_bfloat16* out_row = args.out + static_cast<size_t>(row) * args.H;
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
          uint32_t v[32];
          tmem_ld32(t_row + c, v);
          tmem_wait_ld();
          const int col = t.n_blk * 256 + c;
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&s.acc_empty[acc]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    // every claim of this CTA is done: the last CTA to get here returns the counters to zero
    __threadfence();
    if (atomicAdd(args.sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      atomicExch(args.sched, 0);
      atomicExch(args.sched + 1, 0);
    }
  }
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

}  // namespace

// Workspace: [0,4) status | [256, ..) h bf16 [max_rows, F] | (FP8) dequantised rows bf16
// [max_rows, H] | GEMM-1 completion counters and GEMM-2 arrival counters, int32
// [2][max_rows/128 + E + 1] | tile-claim counter and finished-CTA counter, int32 [2].
static size_t round256(size_t b) { return (b + 255) / 256 * 256; }
static size_t ffn_counter_count(int max_rows, int E) {
  return static_cast<size_t>(max_rows) / BM + static_cast<size_t>(E) + 1;
}

size_t ffn_workspace_bytes(int max_rows, int H, int F, int fp8, int E) {
  const size_t h_bytes = round256(static_cast<size_t>(max_rows) * F * 2);
  const size_t x_bytes = fp8 ? round256(static_cast<size_t>(max_rows) * H * 2) : 0;
  return 256 + h_bytes + x_bytes + round256((2 * ffn_counter_count(max_rows, E) + 2) * sizeof(int));
}

cudaError_t launch_expert_ffn(const void* send, const float* send_scales, int fp8,
                              const int32_t* expert_offsets, int max_rows, int E, int H, int F,
                              const void* w_gate, const void* w_up, const void* w_down,
                              void* expert_out, void* ws, cudaStream_t s) {
  if (max_rows == 0) return cudaSuccess;
  char* base = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(base);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(base + 256);
  size_t off = 256 + round256(static_cast<size_t>(max_rows) * F * 2);
  uint4* xdq = nullptr;
  if (fp8) {
    xdq = reinterpret_cast<uint4*>(base + off);
    off += round256(static_cast<size_t>(max_rows) * H * 2);
  }
  int* done = reinterpret_cast<int*>(base + off);
  int* used = done + ffn_counter_count(max_rows, E);
  int* sched = used + ffn_counter_count(max_rows, E);
  // all counters are zero on entry (zero-filled workspace, reset by the previous call)
  cudaError_t err = cudaSuccess;
  bool pdl_next = true;
  const void* a_src = send;
  if (fp8) {
    const long long work = static_cast<long long>(max_rows) * (H / 16);
    long long blocks = (work + 255) / 256;
    const long long cap = static_cast<long long>(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    err = launch_pdl_if(pdl_next, dequant_fp8_kernel, dim3(static_cast<int>(blocks)), dim3(256), 0,
                        s, static_cast<const uint8_t*>(send), send_scales, expert_offsets + E,
                        max_rows, H, xdq);
    if (err != cudaSuccess) return err;
    a_src = xdq;
    pdl_next = true;
  }
  CUtensorMap tm_x, tm_g, tm_u, tm_h, tm_d;
  SmallBoxMaps tm_xs, tm_hs;
  for (int i = 0; i < 3; ++i)
    if (!make_tmap(&tm_xs.m[i], a_src, max_rows, H, small_box_rows(i)) ||
        !make_tmap(&tm_hs.m[i], h, max_rows, F, small_box_rows(i)))
      return cudaErrorInvalidValue;
  if (!make_tmap(&tm_x, a_src, max_rows, H, BM) ||
      !make_tmap(&tm_g, w_gate, static_cast<uint64_t>(E) * F, H, 128) ||
      !make_tmap(&tm_u, w_up, static_cast<uint64_t>(E) * F, H, 128) ||
      !make_tmap(&tm_h, h, max_rows, F, BM) ||
      !make_tmap(&tm_d, w_down, static_cast<uint64_t>(E) * H, F, kGemm2NTile))
    return cudaErrorInvalidValue;
  FfnArgs fa{expert_offsets, E, max_rows, H, F, h, static_cast<__nv_bfloat16*>(expert_out), status,
             done, used, sched};
  const size_t smem = fused_smem_bytes(E);
  err = cudaFuncSetAttribute(fused_ffn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  err = launch_pdl_if(pdl_next, fused_ffn_kernel, dim3(num_sms()), dim3(kThreads), smem, s, tm_x,
                      tm_xs, tm_g, tm_u, tm_h, tm_hs, tm_d, fa);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace moe
