// Host entry point of decode attention, the split-T combine kernel, and the library's
// status/utility calls.
#include <math.h>
#include <mutex>

#include "attend.cuh"

namespace commvq {

DeviceInfo current_device_info() {
  static std::mutex mu;
  static DeviceInfo cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DeviceInfo{};
  std::lock_guard<std::mutex> lock(mu);
  DeviceInfo& di = cache[dev];
  if (di.device != dev) {
    int sms = 0, smem = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return DeviceInfo{};
    di.sms = sms;
    di.smem_optin = static_cast<size_t>(smem);
    di.device = dev;
  }
  return di;
}

namespace {

constexpr size_t kHeaderBytes = 256;   // device error word + padding

// Split-T merge (flash-decoding style log-sum-exp combine of the per-split partials):
// out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s, lse = (M + log2 L) ln 2.
__global__ void __launch_bounds__(kD) combine_kernel(AttendArgs a, int S) {
  const int bh = blockIdx.x;
  const int dim = threadIdx.x;
  const Partial* p = a.partials + static_cast<int64_t>(bh) * S;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, p[s].m);
  float L = 0.0f, acc = 0.0f;
  if (M != -INFINITY) {
    for (int s = 0; s < S; ++s) {
      const float w = exp2f(p[s].m - M);
      L = fmaf(w, p[s].l, L);
      acc = fmaf(w, p[s].o[dim], acc);
    }
  }
  a.out[static_cast<int64_t>(bh) * kD + dim] = L > 0.0f ? acc / L : 0.0f;
  if (a.lse && dim == 0)
    a.lse[bh] = L > 0.0f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

int choose_splits(int B, int q_heads, int64_t max_T, const commvq_attend_options* opt) {
  if (opt && opt->splits > 0) return opt->splits;
  const DeviceInfo di = current_device_info();
  const int sms = di.sms > 0 ? di.sms : 148;
  const int64_t units = static_cast<int64_t>(B) * q_heads;
  int64_t S = units >= sms ? 1 : sms / units;
  const int64_t by_len = (max_T + 511) / 512;
  if (S > by_len) S = by_len;
  if (S < 1) S = 1;
  if (S > 4096) S = 4096;
  return static_cast<int>(S);
}

// Shape checks shared by the workspace query and the call. Returns OK, INVALID or UNSUPPORTED.
commvq_status check_config(const commvq_config* cfg) {
  if (!cfg) return COMMVQ_ERR_INVALID_ARG;
  const int d = cfg->d, g = cfg->g, R = cfg->R, Nc = cfg->n_codes;
  if (d <= 0 || g <= 0 || d % g || g % 2 || R < 1 || Nc < 1 || Nc > 65536 || cfg->q_heads < 1 ||
      cfg->kv_heads < 1 || cfg->q_heads % cfg->kv_heads || !(cfg->rope_base > 0.0) ||
      !isfinite(cfg->rope_base))
    return COMMVQ_ERR_INVALID_ARG;
  if (cfg->code_bytes != (Nc <= 256 ? 1 : 2)) return COMMVQ_ERR_INVALID_ARG;
  if (d != kD || g != kG || Nc > 256 || R > 4) return COMMVQ_ERR_UNSUPPORTED;
  if (cfg->q_heads > 65535) return COMMVQ_ERR_UNSUPPORTED;
  return COMMVQ_OK;
}

}  // namespace
}  // namespace commvq

using namespace commvq;

extern "C" size_t commvq_attend_workspace_bytes(const commvq_config* cfg, int32_t B, int64_t max_T,
                                                const commvq_attend_options* options) {
  if (check_config(cfg) != COMMVQ_OK || B < 0 || max_T < 0) return 0;
  const int S = choose_splits(B > 0 ? B : 1, cfg->q_heads, max_T, options);
  return kHeaderBytes + static_cast<size_t>(B) * cfg->q_heads * S * sizeof(Partial);
}

extern "C" commvq_status commvq_attend_decode(const commvq_config* cfg, const void* q,
                                              commvq_dtype q_dtype, const void* k_codes,
                                              const void* v_codes, const int64_t* seq_offsets,
                                              int32_t B, int64_t max_T, const float* k_codebook,
                                              const float* v_codebook, float* out, float* lse,
                                              void* workspace, size_t workspace_bytes,
                                              const commvq_attend_options* options, void* stream) {
  const commvq_status cs = check_config(cfg);
  if (cs != COMMVQ_OK) return cs;
  if (B < 0 || max_T < 0) return COMMVQ_ERR_INVALID_ARG;
  if (q_dtype != COMMVQ_F32 && q_dtype != COMMVQ_F16 && q_dtype != COMMVQ_BF16)
    return COMMVQ_ERR_INVALID_ARG;
  const int algo = options ? options->algo : COMMVQ_ATTN_AUTO;
  if (options && (options->splits < 0 || options->splits > 65535)) return COMMVQ_ERR_INVALID_ARG;
  if (algo != COMMVQ_ATTN_AUTO && algo != COMMVQ_ATTN_TABLE && algo != COMMVQ_ATTN_DECODE_MMA)
    return COMMVQ_ERR_INVALID_ARG;
  if (B == 0) return COMMVQ_OK;
  if (B > 65535) return COMMVQ_ERR_UNSUPPORTED;
  if (!q || !k_codes || !v_codes || !seq_offsets || !k_codebook || !v_codebook || !out || !workspace)
    return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_codes, 16) || !aligned(v_codes, 16) || !aligned(k_codebook, 16) ||
      !aligned(v_codebook, 16) || !aligned(out, 16) || !aligned(lse, 4) || !aligned(seq_offsets, 8) ||
      !aligned(workspace, 256))
    return COMMVQ_ERR_INVALID_ARG;
  const size_t need = commvq_attend_workspace_bytes(cfg, B, max_T, options);
  if (need == 0 || workspace_bytes < need) return COMMVQ_ERR_WORKSPACE;

  const DeviceInfo di = current_device_info();
  if (di.device < 0) return COMMVQ_ERR_CUDA;
  if (algo == COMMVQ_ATTN_DECODE_MMA) return COMMVQ_ERR_UNSUPPORTED;
  if (table_smem_bytes(cfg->R, cfg->n_codes) > di.smem_optin) return COMMVQ_ERR_UNSUPPORTED;

  const int S = choose_splits(B, cfg->q_heads, max_T, options);
  AttendArgs a;
  a.k_codes = static_cast<const uint8_t*>(k_codes);
  a.v_codes = static_cast<const uint8_t*>(v_codes);
  a.seq_offsets = seq_offsets;
  a.k_codebook = k_codebook;
  a.v_codebook = v_codebook;
  a.out = out;
  a.lse = lse;
  a.error_word = static_cast<int*>(workspace);
  a.partials = reinterpret_cast<Partial*>(static_cast<unsigned char*>(workspace) + kHeaderBytes);
  a.max_T = max_T;
  a.rope_base = cfg->rope_base;
  a.B = B;
  a.q_heads = cfg->q_heads;
  a.kv_heads = cfg->kv_heads;
  a.R = cfg->R;
  a.n_codes = cfg->n_codes;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(a.error_word, 0, sizeof(int), st) != cudaSuccess) return COMMVQ_ERR_CUDA;
  // External records so the events keep their timestamps inside a captured CUDA graph too.
  if (options && options->main_start &&
      cudaEventRecordWithFlags(static_cast<cudaEvent_t>(options->main_start), st,
                               cudaEventRecordExternal) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  commvq_status rc = launch_attend_table(a, q, q_dtype, S, st);
  if (rc != COMMVQ_OK) return rc;
  if (options && options->main_stop &&
      cudaEventRecordWithFlags(static_cast<cudaEvent_t>(options->main_stop), st,
                               cudaEventRecordExternal) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  return launch_combine(a, S, st);
}

namespace commvq {
commvq_status launch_combine(const AttendArgs& a, int S, cudaStream_t st) {
  combine_kernel<<<a.B * a.q_heads, kD, 0, st>>>(a, S);
  return launch_status();
}
}  // namespace commvq

extern "C" commvq_status commvq_workspace_error(const void* workspace, int32_t* device_error,
                                                void* stream) {
  if (!workspace || !device_error) return COMMVQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return COMMVQ_ERR_CUDA;
  *device_error = v;
  return v ? COMMVQ_ERR_DEVICE_CHECK : COMMVQ_OK;
}

extern "C" const char* commvq_status_string(commvq_status s) {
  switch (s) {
    case COMMVQ_OK: return "ok";
    case COMMVQ_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size or shape)";
    case COMMVQ_ERR_UNSUPPORTED: return "shape or type not supported by this build";
    case COMMVQ_ERR_CUDA: return "CUDA runtime error";
    case COMMVQ_ERR_WORKSPACE: return "workspace missing or too small";
    case COMMVQ_ERR_DEVICE_CHECK: return "device recorded a data error (code out of range)";
    default: return "unknown status";
  }
}

extern "C" int32_t commvq_abi_version(void) { return 1; }
