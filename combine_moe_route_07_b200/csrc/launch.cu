// launch.cu -- host-side launch helpers shared by the kernel files.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "kernels.h"

namespace moe {

namespace {

struct OccEntry {
  int dev;
  const void* kernel;
  int threads;
  size_t smem;
  int blocks;
};

struct SmemEntry {
  int dev;
  const void* kernel;
  size_t smem;  // the kernel's dynamic shared-memory limit as last raised
};

std::mutex g_occ_mu;
std::vector<OccEntry> g_occ;
std::vector<SmemEntry> g_smem;

// Raise (never lower) the kernel's dynamic shared-memory limit to `smem`.
cudaError_t raise_smem_limit(int dev, const void* kernel, size_t smem) {
  for (SmemEntry& e : g_smem)
    if (e.dev == dev && e.kernel == kernel) {
      if (e.smem >= smem) return cudaSuccess;
      const cudaError_t err =
          cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err == cudaSuccess) e.smem = smem;
      return err;
    }
  const cudaError_t err =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err == cudaSuccess) g_smem.push_back(SmemEntry{dev, kernel, smem});
  return err;
}

}  // namespace

cudaError_t blocks_per_sm(const void* kernel, int threads, size_t smem, int* out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(g_occ_mu);
  // any dynamic shared memory: the default limit is 48 KiB less the static
  // shared memory, which a 48 KiB request already exceeds
  if (smem > 0) {
    err = raise_smem_limit(dev, kernel, smem);
    if (err != cudaSuccess) return err;
  }
  for (const OccEntry& e : g_occ)
    if (e.dev == dev && e.kernel == kernel && e.threads == threads && e.smem == smem) {
      *out = e.blocks;
      return cudaSuccess;
    }
  int n = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem);
  if (err != cudaSuccess) return err;
  if (n < 1) n = 1;
  g_occ.push_back(OccEntry{dev, kernel, threads, smem, n});
  *out = n;
  return cudaSuccess;
}

}  // namespace moe
