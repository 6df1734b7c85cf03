// Small transfers of a decode step (the query and the new position's K/V rows in, the output
// out) done by one kernel instead of the copy engine. Either side may be mapped pinned host
// memory: the kernel's loads (or stores) then cross the host link directly. A copy-engine
// transfer of a few KB inside a CUDA graph costs several microseconds of scheduling between
// engines; the kernel costs one round trip over the link plus a launch.
#include "common.cuh"

namespace commvq {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyMaxBlocks = 148;

// 16-byte pieces, grid-strided; the bytes past the last whole piece by block 0's first threads.
__global__ void __launch_bounds__(kCopyThreads) copy_kernel(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                                            int64_t n16, uint8_t* __restrict__ dst_tail,
                                                            const uint8_t* __restrict__ src_tail, int tail) {
  // launched as a programmatic dependent: the launch overlaps the kernel before, and the wait
  // gives it that kernel's writes (ordinary stream order) before any load or store; the kernel
  // after it may then start its own set-up
  pdl_wait();
  pdl_trigger();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kCopyThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kCopyThreads + threadIdx.x; i < n16; i += stride)
    dst[i] = src[i];
  if (blockIdx.x == 0 && threadIdx.x < tail) dst_tail[threadIdx.x] = src_tail[threadIdx.x];
}

}  // namespace
}  // namespace commvq

using namespace commvq;

extern "C" commvq_status commvq_copy_async(void* dst, const void* src, size_t bytes, void* stream) {
  const NvtxRange nvtx_range("commvq_copy_async");
  if (bytes == 0) return COMMVQ_OK;
  if (!dst || !src) return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(dst, 16) || !aligned(src, 16)) return COMMVQ_ERR_INVALID_ARG;
  const char* d = static_cast<const char*>(dst);
  const char* s = static_cast<const char*>(src);
  if (d < s + bytes && s < d + bytes) return COMMVQ_ERR_INVALID_ARG;   // overlapping ranges
  const int64_t n16 = static_cast<int64_t>(bytes / 16);
  const int tail = static_cast<int>(bytes % 16);
  int64_t blocks = (n16 + kCopyThreads - 1) / kCopyThreads;
  if (blocks < 1) blocks = 1;
  if (blocks > kCopyMaxBlocks) blocks = kCopyMaxBlocks;
  if (launch_dependent(copy_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kCopyThreads), 0,
                       static_cast<cudaStream_t>(stream), static_cast<uint4*>(dst), static_cast<const uint4*>(src),
                       n16, static_cast<uint8_t*>(dst) + n16 * 16, static_cast<const uint8_t*>(src) + n16 * 16,
                       tail) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  return launch_status();
}
