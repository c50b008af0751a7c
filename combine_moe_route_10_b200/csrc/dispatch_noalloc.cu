// moe_dispatch_noalloc: the dispatch with its scratch memory in a static device array, for callers
// that cannot allocate.
//
// moe_dispatch asks the caller for a workspace.  Some callers cannot provide one: host programs
// that own every byte of device memory through their own pool and forbid extra allocations,
// plug-ins embedded in such programs, and latency-critical paths where cudaMalloc (which can
// synchronise the device) is not acceptable.  This entry point needs only the inputs and outputs.
//
// The scratch (the per-chunk expert histogram) lives in g_dispatch_scratch,
// a file-scope __device__ array of kNoallocScratchBytes.  Every GPU that loads the library keeps it
// until the process exits.  Host code must not pass the array's name to a kernel (on the host it is
// only a stand-in symbol): every call looks up the array's device address in the context that is
// current at that moment (cudaGetSymbolAddress, a host-side lookup that allocates nothing), so the
// address is never one left over from another context of the same device (a driver-API context of
// the caller's, or the primary context before a cudaDeviceReset).  The first call in a context may
// load the library's module there, which is why it should come before any stream capture.
#include "../../include/moe.h"
#include "common.cuh"
#include "launch.h"

namespace {

constexpr size_t kNoallocScratchBytes = MOE_DISPATCH_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_dispatch_scratch[kNoallocScratchBytes];

// Device address of g_dispatch_scratch in the current context (looked up on every call).
cudaError_t scratch_for_current_context(unsigned char** out) {
  void* p = nullptr;
  const cudaError_t err = cudaGetSymbolAddress(&p, g_dispatch_scratch);
  if (err != cudaSuccess) return err;
  *out = static_cast<unsigned char*>(p);
  return cudaSuccess;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" moe_status_t moe_dispatch_noalloc(const void* x, int T, int H, const int32_t* topk_idx,
                                             int k, int E, int R, int capacity,
                                             moe_payload_t payload, void* send, float* send_scales,
                                             int32_t* expert_counts, int32_t* expert_offsets,
                                             int32_t* rank_offsets, int32_t* slot_row,
                                             int32_t* row_token, int32_t* status,
                                             moe_stream_t stream) {
  if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 32 || R < 1 || E % R != 0 ||
      capacity < 0 || H < 8)
    return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * k >= INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (payload != MOE_PAYLOAD_BF16 && payload != MOE_PAYLOAD_FP8_E4M3_B128)
    return MOE_ERR_INVALID_ARG;
  if (H % 8 != 0) return MOE_ERR_UNSUPPORTED;
  const bool fp8 = payload == MOE_PAYLOAD_FP8_E4M3_B128;
  if (fp8 && H % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (expert_counts == nullptr || expert_offsets == nullptr || rank_offsets == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && (x == nullptr || topk_idx == nullptr || send == nullptr || slot_row == nullptr ||
                row_token == nullptr || (fp8 && send_scales == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(send, 16) || !aligned(send_scales, 4) ||
      !aligned(topk_idx, 4) || !aligned(status, 4))
    return MOE_ERR_INVALID_ARG;
  // the static scratch has a fixed size: reject shapes whose chunk table does not fit
  if (moe::dispatch_workspace_bytes(T, E, k) > kNoallocScratchBytes) return MOE_ERR_WORKSPACE;

  unsigned char* scratch = nullptr;
  if (scratch_for_current_context(&scratch) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents.  Nothing in it has to start at zero: the
  // histogram table is fully written by the count kernel before it is read, and the status word
  // is the caller's.
  int32_t* hist = reinterpret_cast<int32_t*>(scratch + 256);
  const cudaError_t err = moe::launch_dispatch_parts(
      x, T, H, topk_idx, k, E, R, capacity, fp8 ? 1 : 0, send, send_scales, expert_counts,
      expert_offsets, rank_offsets, slot_row, row_token, reinterpret_cast<int*>(status), hist, s);
  if (err != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
