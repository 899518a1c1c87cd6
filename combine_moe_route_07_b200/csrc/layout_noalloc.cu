// layout_noalloc.cu -- moe_layout for callers that cannot allocate device
// memory.
//
// Some callers have no way to hand the library a workspace: plugin or
// custom-op hosts that pass a kernel only its inputs and outputs, serving
// runtimes whose memory pool owns every byte of the device, and code on a
// latency-critical path where cudaMalloc (which may synchronise the device)
// is not allowed.  This entry point runs the same count and place kernels as
// moe_layout, with their scratch (error word, the layout's counters and its
// two tile tables) in a file-scope device array instead of a caller workspace.
//
// The array is kMoeNoallocScratchBytes bytes; every GPU that loads the library
// holds it until the process exits.  Every call looks up the array's device
// address on the current device (cudaGetSymbolAddress), so no address outlives
// the context it came from (after cudaDeviceReset the library's module is
// loaded again and its array has a new, zero-filled copy).  The first call that
// sees an address on a device clears the array there; make that first call
// before any stream capture.  Every call leaves the array ready for the next
// one (the layout kernels clear the counters they used); a call whose launch
// fails clears the whole array again.  Calls share the array, so calls that
// overlap on the GPU (different streams, or different host threads, without
// ordering) race and give wrong results.  The kernels' error word lives in the
// array too; nothing reads it and nothing clears it (see the header).
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "moe_route07.h"

namespace {

constexpr size_t kHeader = sizeof(moe::WsHeader);
constexpr size_t kMoeNoallocScratchBytes = kHeader + MOE_NOALLOC_TABLE_BYTES;

static __device__ __align__(256) unsigned char g_layout_scratch[kMoeNoallocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_cleared[kMaxDevices] = {nullptr};  // address last cleared on each device
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, looked up on
// every call; the first call that sees an address on a device zero-fills the
// array (cudaMemsetAsync on `stream`).
moe_status_t scratch_for_current_device(cudaStream_t stream, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || p == nullptr)
    return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_cleared[dev] != p) {
    if (cudaMemsetAsync(p, 0, kMoeNoallocScratchBytes, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_cleared[dev] = p;
  }
  *out = p;
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_layout_noalloc(const moe_shape_t* shape, const int32_t* ids,
                                           int32_t* counts, int32_t* expert_off,
                                           int32_t* rank_off, int32_t* rank_counts,
                                           int32_t* dst_pos, int32_t* src_idx,
                                           moe_stream_t stream) {
  // Shape checks: the same limits as moe_layout, plus the static table size.
  const int64_t rows = moe_layout_rows(shape);
  if (rows < 0 || (shape->flags & MOE_F_SRC_LAYOUT) != 0u) return MOE_ERR_INVALID_ARG;
  const size_t need = moe_workspace_bytes(shape);
  if (need == 0) return MOE_ERR_INVALID_ARG;
  if (need > kMoeNoallocScratchBytes) return MOE_ERR_UNSUPPORTED;
  if (counts == nullptr || expert_off == nullptr || rank_off == nullptr ||
      rank_counts == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (shape->tokens > 0 && (ids == nullptr || dst_pos == nullptr)) return MOE_ERR_INVALID_ARG;
  if (rows > 0 && src_idx == nullptr) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {ids, counts, expert_off, rank_off, rank_counts, dst_pos, src_idx};
  for (const void* p : ptrs)
    if ((reinterpret_cast<uintptr_t>(p) & 3u) != 0u) return MOE_ERR_INVALID_ARG;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  moe_status_t st = scratch_for_current_device(s, &scratch);
  if (st != MOE_OK) return st;

  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  moe::LaunchEnv env;
  env.stream = s;
  env.num_sms = sms;
  moe::WsHeader* hdr = static_cast<moe::WsHeader*>(scratch);
  uint32_t* tables = reinterpret_cast<uint32_t*>(static_cast<char*>(scratch) + kHeader);
  const size_t half_words = (MOE_NOALLOC_TABLE_BYTES / 8) / 4 * 4;
  const cudaError_t err = moe::launch_layout(
      env, ids, shape->tokens, shape->experts, shape->k, shape->ranks, shape->capacity,
      shape->align, rows, tables, half_words, hdr, counts, expert_off, rank_off, rank_counts,
      dst_pos, src_idx, true);
  if (err != cudaSuccess) {
    (void)cudaMemsetAsync(scratch, 0, kMoeNoallocScratchBytes, s);  // back to a clean array
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
