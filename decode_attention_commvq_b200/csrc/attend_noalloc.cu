// Decode attention without a caller-provided workspace.
//
// Some callers cannot allocate device memory: a plugin or extension running inside a host
// framework that owns the device allocator and forbids direct cudaMalloc, or a
// latency-critical serving loop where a cudaMalloc (which can synchronise the device) is not
// acceptable and no memory pool is at hand. For them this file keeps the attention scratch
// (the split partials, the fp16 codebook images and the score buffer) in one file-scope
// device array of a fixed size, and forwards to commvq_attend_decode with that array as the
// workspace.
//
// Cost of the choice: every GPU that loads the library holds the array until the process
// exits, and all calls on a device share it.
#include <mutex>

#include "common.cuh"

namespace commvq {
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(32) << 20;   // 32 MiB per device

// The scratch itself. In host code this name is only a stand-in for the symbol; the device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_attend_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_attend_scratch on the current device, looked up once per device.
commvq_status scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return COMMVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attend_scratch) != cudaSuccess || !p) return COMMVQ_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return COMMVQ_OK;
}

}  // namespace
}  // namespace commvq

using namespace commvq;

extern "C" commvq_status commvq_attend_decode_noalloc(
    const commvq_config* cfg, const void* q, commvq_dtype q_dtype, const void* k_codes,
    const void* v_codes, const int64_t* seq_offsets, int32_t B, int64_t max_T,
    const float* k_codebook, const float* v_codebook, float* out, float* lse,
    const commvq_attend_options* options, void* stream) {
  const NvtxRange nvtx_range("commvq_attend_decode_noalloc");
  // Prepared state would have to survive in the shared array from an earlier call, which any
  // other call on the device (another layer's codebooks, another rope base) may have
  // overwritten since: this entry point always rebuilds it.
  if (options && (options->flags & COMMVQ_ATTEND_PREPARED)) return COMMVQ_ERR_INVALID_ARG;
  if (B == 0)   // nothing to run: let the regular call validate the rest and return
    return commvq_attend_decode(cfg, q, q_dtype, k_codes, v_codes, seq_offsets, B, max_T, k_codebook,
                                v_codebook, out, lse, nullptr, 0, options, stream);
  const size_t need = commvq_attend_workspace_bytes(cfg, B, max_T, options);
  if (need == 0)   // invalid or unsupported arguments: the regular call reports which
    return commvq_attend_decode(cfg, q, q_dtype, k_codes, v_codes, seq_offsets, B, max_T, k_codebook,
                                v_codebook, out, lse, nullptr, 0, options, stream);
  if (need > kNoAllocScratchBytes) return COMMVQ_ERR_WORKSPACE;   // larger than the fixed scratch
  void* scratch = nullptr;
  const commvq_status rc = scratch_address(&scratch);
  if (rc != COMMVQ_OK) return rc;
  // Without COMMVQ_ATTEND_PREPARED the regular call clears the scratch's error words and writes
  // everything else it reads from the scratch earlier in the same call, so a previous call's
  // leftovers do not matter.
  return commvq_attend_decode(cfg, q, q_dtype, k_codes, v_codes, seq_offsets, B, max_T, k_codebook,
                              v_codebook, out, lse, scratch, kNoAllocScratchBytes, options, stream);
}
