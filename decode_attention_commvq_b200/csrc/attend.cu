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
// Grid: (sequence x head, 4 quarters of the 128 output dims), 256 threads = 32 groups of 8
// lanes. Lane gl of group grp owns float4 gl of the quarter's 32 dims and the splits grp,
// grp + 32, ...; it issues the loads of (m, l, its float4 of o) for 8 splits at a time before
// any arithmetic, folds them in with a running maximum, and the 32 groups are merged in parallel
// in a fixed order (shuffles, then the 8 warps' sums), so one call's result does not depend on
// timing.
constexpr int kCombineThreads = 256;
constexpr int kCombineQuarters = 4;
constexpr int kCombineGroups = kCombineThreads / 8;
constexpr int kCombinePer = 8;   // splits per lane per pass
constexpr int kMaxSplits = 4096;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(AttendArgs a, int S) {
  __shared__ float4 acc_s[kCombineGroups][8];
  __shared__ float ml_s[kCombineGroups][2];
  pdl_trigger();   // the next decode step's scores kernel may copy its codebook image meanwhile
  pdl_wait();      // launched as a dependent of the kernel that writes the partials
  const int bh = blockIdx.x, quarter = blockIdx.y;
  const int tid = threadIdx.x, grp = tid >> 3, gl = tid & 7;
  if (bh == 0 && quarter == 0 && tid == 0 && a.error_word) publish_error(a.error_word);   // the call's last kernel
  const Partial* p = a.partials + static_cast<int64_t>(bh) * S;
  const int dim4 = quarter * 8 + gl;   // float4 index within o[128]

  float M = -INFINITY, L = 0.0f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = grp; s0 < S; s0 += kCombineGroups * kCombinePer) {
    float m[kCombinePer], l[kCombinePer];
    float4 o[kCombinePer];
#pragma unroll
    for (int k = 0; k < kCombinePer; ++k) {
      const int s = s0 + k * kCombineGroups;
      if (s < S) {
        const float2 ml = *reinterpret_cast<const float2*>(&p[s].m);
        m[k] = ml.x;
        l[k] = ml.y;
        o[k] = reinterpret_cast<const float4*>(p[s].o)[dim4];
      } else {
        m[k] = -INFINITY;
        l[k] = 0.0f;
        o[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float mx = M;
#pragma unroll
    for (int k = 0; k < kCombinePer; ++k) mx = fmaxf(mx, m[k]);
    if (mx == -INFINITY) continue;   // only empty splits so far
    const float sc = exp2f(M - mx);
    acc.x *= sc;
    acc.y *= sc;
    acc.z *= sc;
    acc.w *= sc;
    L *= sc;
#pragma unroll
    for (int k = 0; k < kCombinePer; ++k) {
      const float w = exp2f(m[k] - mx);
      acc.x = fmaf(w, o[k].x, acc.x);
      acc.y = fmaf(w, o[k].y, acc.y);
      acc.z = fmaf(w, o[k].z, acc.z);
      acc.w = fmaf(w, o[k].w, acc.w);
      L = fmaf(w, l[k], L);
    }
    M = mx;
  }
  acc_s[grp][gl] = acc;
  if (gl == 0) {
    ml_s[grp][0] = M;
    ml_s[grp][1] = L;
  }
  __syncthreads();
  // Merge of the 32 groups in parallel, in a fixed order: thread (grp, gl) weights float4 gl of
  // group grp by 2^(M_grp - Mg); lanes with equal gl add the warp's four groups (xor 8, then 16),
  // and 8 threads add the 8 warps' sums in warp order.
  static_assert(kCombineGroups == 32 && kCombineThreads == 256, "one max per lane, 8 warps");
  __shared__ float4 wsum[kCombineThreads / 32][8];
  __shared__ float lsum_w[kCombineThreads / 32];
  const int lane = tid & 31, wid = tid >> 5;
  float Mg = ml_s[lane][0];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) Mg = fmaxf(Mg, __shfl_xor_sync(0xffffffffu, Mg, o));
  const float w = Mg == -INFINITY ? 0.0f : exp2f(ml_s[grp][0] - Mg);
  float4 v = acc_s[grp][gl];
  v = make_float4(w * v.x, w * v.y, w * v.z, w * v.w);
  float lv = gl == 0 ? w * ml_s[grp][1] : 0.0f;
#pragma unroll
  for (int o = 8; o < 32; o <<= 1) {
    v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
    v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
    v.z += __shfl_xor_sync(0xffffffffu, v.z, o);
    v.w += __shfl_xor_sync(0xffffffffu, v.w, o);
    lv += __shfl_xor_sync(0xffffffffu, lv, o);
  }
  if (lane < 8) wsum[wid][lane] = v;
  if (lane == 0) lsum_w[wid] = lv;
  __syncthreads();
  if (tid < 8) {
    float4 t = wsum[0][tid];
    float Lt = lsum_w[0];
#pragma unroll
    for (int w2 = 1; w2 < kCombineThreads / 32; ++w2) {
      const float4 u = wsum[w2][tid];
      t.x += u.x;
      t.y += u.y;
      t.z += u.z;
      t.w += u.w;
      Lt += lsum_w[w2];
    }
    const float inv = Lt > 0.0f ? 1.0f / Lt : 0.0f;
    reinterpret_cast<float4*>(a.out + static_cast<int64_t>(bh) * kD)[quarter * 8 + tid] =
        make_float4(t.x * inv, t.y * inv, t.z * inv, t.w * inv);
    if (a.lse && quarter == 0 && tid == 0)
      a.lse[bh] = Lt > 0.0f ? (Mg + log2f(Lt)) * 0.6931471805599453f : -INFINITY;
  }
}

// Whether an algorithm takes the shape (the table's shared-memory fit is checked at the call).
bool algo_supported(const commvq_config* cfg, int algo) {
  const bool g8 = cfg->g == kG && cfg->n_codes <= 256;
  switch (algo) {
    case COMMVQ_ATTN_DECODE_MMA: return g8 && mma_supported(cfg->R, cfg->q_heads, cfg->kv_heads, cfg->n_codes);
    case COMMVQ_ATTN_TABLE: return g8 && cfg->R <= 4;
    case COMMVQ_ATTN_GENERIC: return generic_supported(cfg);
    default: return false;
  }
}

// Algorithm actually run for a request: AUTO takes decode-and-rotate, else the table form,
// else the generic form, whichever first supports the shape (-1: none).
int resolve_algo(const commvq_config* cfg, const commvq_attend_options* opt) {
  const int algo = opt ? opt->algo : COMMVQ_ATTN_AUTO;
  if (algo != COMMVQ_ATTN_AUTO) return algo;
  for (int a : {COMMVQ_ATTN_DECODE_MMA, COMMVQ_ATTN_TABLE, COMMVQ_ATTN_GENERIC})
    if (algo_supported(cfg, a)) return a;
  return -1;
}

// Split-T partitions per sequence. Table form: one CTA per (sequence, query head, split);
// decode-and-rotate form: one CTA per (sequence, split) covering every head. Both aim at
// one wave of CTAs on the SMs.
int choose_splits(int algo, int B, int q_heads, int64_t max_T, const commvq_attend_options* opt) {
  if (opt && opt->splits > 0) return opt->splits;
  const DeviceInfo di = current_device_info();
  const int sms = di.sms > 0 ? di.sms : 148;
  int64_t S;
  if (algo == COMMVQ_ATTN_DECODE_MMA) {
    S = B >= sms ? 1 : sms / B;
    const int64_t by_len = (max_T + 15) / 16;
    if (S > by_len) S = by_len;
  } else if (algo == COMMVQ_ATTN_GENERIC) {   // latency bound: several CTAs per SM
    S = 4 * sms / B;
    const int64_t by_len = (max_T + 63) / 64;
    if (S > by_len) S = by_len;
  } else {
    const int64_t units = static_cast<int64_t>(B) * q_heads;
    S = units >= sms ? 1 : sms / units;
    const int64_t by_len = (max_T + 511) / 512;
    if (S > by_len) S = by_len;
  }
  if (S < 1) S = 1;
  if (S > kMaxSplits) S = kMaxSplits;
  return static_cast<int>(S);
}

// Partial slots per (sequence, head): the generic form writes one per warp of a KV head.
int partial_slots(const commvq_config* cfg, int algo, int S) {
  return algo == COMMVQ_ATTN_GENERIC ? S * generic_warps_per_kv(cfg->kv_heads) : S;
}

struct WorkspaceLayout {
  size_t partials_off, kimg_off, vimg_off, phase_off, scores_off, tables_off, total;
};
// theta, rows, advance: attend_mma.cu's tables (128 offset rows); the fast kernels' (64 rows) fit
constexpr size_t kPhaseBytes = 64 * sizeof(double) + 128 * 64 * 8 + 64 * 8;

void set_phase_tables(AttendArgs& a, unsigned char* base, bool fast) {
  a.theta = reinterpret_cast<const double*>(base);
  a.rowph = reinterpret_cast<const float4*>(base + 64 * sizeof(double));
  a.advph = a.rowph + (fast ? 64 * 64 / 2 : 128 * 32);   // float4 units: 64 x 64 (cos, sin) or 128 x 32
}

bool use_fast(const commvq_config* cfg) {
  return fast_supported(cfg->g, cfg->R, cfg->q_heads, cfg->kv_heads, cfg->n_codes);
}

// The prepared state (codebook images, RoPE tables) depends only on cfg and the codebooks, so
// it sits at fixed offsets right after the header: a workspace prepared once stays valid for
// any B, max_T and split count that fit in it. Per-call buffers (partials, scores) follow.
// fast: the fast kernels' image size (128 KB each); otherwise attend_mma.cu's (512 Nc' bytes).
WorkspaceLayout workspace_layout(const commvq_config* cfg, int algo, int B, int64_t max_T, int S, bool fast) {
  WorkspaceLayout L{};
  size_t end = kHeaderBytes;
  if (algo == COMMVQ_ATTN_DECODE_MMA) {
    const size_t img = fast ? static_cast<size_t>(131072) : static_cast<size_t>(512) * cfg->n_codes;
    L.kimg_off = end;
    L.vimg_off = round_up(L.kimg_off + img, 256);
    L.phase_off = round_up(L.vimg_off + img, 256);
    end = round_up(L.phase_off + kPhaseBytes, 256);
  }
  L.partials_off = end;
  end = L.partials_off + static_cast<size_t>(B) * cfg->q_heads * partial_slots(cfg, algo, S) * sizeof(Partial);
  if (algo == COMMVQ_ATTN_GENERIC) {
    L.tables_off = round_up(end, 256);
    end = L.tables_off + generic_tables_bytes(max_T);
  }
  if (algo == COMMVQ_ATTN_DECODE_MMA) {
    L.scores_off = round_up(end, 256);
    end = L.scores_off + static_cast<size_t>(B) * ((max_T + 15) / 16 * 16) * cfg->q_heads * sizeof(float);
  }
  L.total = round_up(end, 256);
  return L;
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
  if (d != kD || (g != 8 && g != 16 && g != 32 && g != 64) || R > 32) return COMMVQ_ERR_UNSUPPORTED;
  if (cfg->q_heads > 65535) return COMMVQ_ERR_UNSUPPORTED;
  return COMMVQ_OK;
}

}  // namespace
}  // namespace commvq

using namespace commvq;

extern "C" size_t commvq_attend_workspace_bytes(const commvq_config* cfg, int32_t B, int64_t max_T,
                                                const commvq_attend_options* options) {
  if (check_config(cfg) != COMMVQ_OK || B < 0 || max_T < 0) return 0;
  if (options && (options->splits < 0 || options->splits > kMaxSplits || options->algo < 0 || options->algo > 3))
    return 0;
  const int algo = resolve_algo(cfg, options);
  if (!algo_supported(cfg, algo)) return 0;
  const int S = choose_splits(algo, B > 0 ? B : 1, cfg->q_heads, max_T, options);
  return workspace_layout(cfg, algo, B, max_T, S, algo == COMMVQ_ATTN_DECODE_MMA && use_fast(cfg)).total;
}

extern "C" commvq_status commvq_attend_decode(const commvq_config* cfg, const void* q,
                                              commvq_dtype q_dtype, const void* k_codes,
                                              const void* v_codes, const int64_t* seq_offsets,
                                              int32_t B, int64_t max_T, const float* k_codebook,
                                              const float* v_codebook, float* out, float* lse,
                                              void* workspace, size_t workspace_bytes,
                                              const commvq_attend_options* options, void* stream) {
  const NvtxRange nvtx_range("commvq_attend_decode");
  const commvq_status cs = check_config(cfg);
  if (cs != COMMVQ_OK) return cs;
  if (B < 0 || max_T < 0) return COMMVQ_ERR_INVALID_ARG;
  if (q_dtype != COMMVQ_F32 && q_dtype != COMMVQ_F16 && q_dtype != COMMVQ_BF16)
    return COMMVQ_ERR_INVALID_ARG;
  const int algo = options ? options->algo : COMMVQ_ATTN_AUTO;
  if (options && (options->splits < 0 || options->splits > kMaxSplits)) return COMMVQ_ERR_INVALID_ARG;
  if (algo < COMMVQ_ATTN_AUTO || algo > COMMVQ_ATTN_GENERIC) return COMMVQ_ERR_INVALID_ARG;
  if (B == 0) return COMMVQ_OK;
  if (B > 65535) return COMMVQ_ERR_UNSUPPORTED;
  if (!q || !k_codes || !v_codes || !seq_offsets || !k_codebook || !v_codebook || !out || !workspace)
    return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_codes, 16) || !aligned(v_codes, 16) || !aligned(k_codebook, 16) ||
      !aligned(v_codebook, 16) || !aligned(out, 16) || !aligned(lse, 4) || !aligned(seq_offsets, 8) ||
      !aligned(workspace, 256))
    return COMMVQ_ERR_INVALID_ARG;
  const int run = resolve_algo(cfg, options);
  if (!algo_supported(cfg, run)) return COMMVQ_ERR_UNSUPPORTED;
  const size_t need = commvq_attend_workspace_bytes(cfg, B, max_T, options);
  if (need == 0 || workspace_bytes < need) return COMMVQ_ERR_WORKSPACE;

  const DeviceInfo di = current_device_info();
  if (di.device < 0) return COMMVQ_ERR_CUDA;
  const bool fast = run == COMMVQ_ATTN_DECODE_MMA && use_fast(cfg);
  if (fast) {
    if (fast_smem_bytes(cfg->R, cfg->kv_heads, cfg->q_heads) > di.smem_optin) return COMMVQ_ERR_UNSUPPORTED;
  } else if (run == COMMVQ_ATTN_DECODE_MMA) {
    if (mma_scores_smem_bytes(cfg->R, cfg->kv_heads, cfg->n_codes) > di.smem_optin ||
        mma_values_smem_bytes(cfg->R, cfg->kv_heads, cfg->q_heads, cfg->n_codes) > di.smem_optin)
      return COMMVQ_ERR_UNSUPPORTED;
  } else if (run == COMMVQ_ATTN_TABLE && table_smem_bytes(cfg->R, cfg->n_codes) > di.smem_optin) {
    return COMMVQ_ERR_UNSUPPORTED;
  }

  const int S = choose_splits(run, B, cfg->q_heads, max_T, options);
  const WorkspaceLayout L = workspace_layout(cfg, run, B, max_T, S, fast);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  AttendArgs a{};
  a.k_codes = static_cast<const uint8_t*>(k_codes);
  a.v_codes = static_cast<const uint8_t*>(v_codes);
  a.seq_offsets = seq_offsets;
  a.k_codebook = k_codebook;
  a.v_codebook = v_codebook;
  a.out = out;
  a.lse = lse;
  a.error_word = static_cast<int*>(workspace);
  a.partials = reinterpret_cast<Partial*>(ws + L.partials_off);
  if (run == COMMVQ_ATTN_DECODE_MMA) {
    a.k_img = reinterpret_cast<const uint4*>(ws + L.kimg_off);
    a.v_img = reinterpret_cast<const uint4*>(ws + L.vimg_off);
    a.scores = reinterpret_cast<float*>(ws + L.scores_off);
    set_phase_tables(a, ws + L.phase_off, fast);
  }
  a.main_start = options ? options->main_start : nullptr;
  a.main_stop = options ? options->main_stop : nullptr;
  a.max_T = max_T;
  a.rope_base = cfg->rope_base;
  a.B = B;
  a.q_heads = cfg->q_heads;
  a.kv_heads = cfg->kv_heads;
  a.R = cfg->R;
  a.n_codes = cfg->n_codes;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool prepared = options && (options->flags & COMMVQ_ATTEND_PREPARED);
  commvq_status rc;
  if (fast) {
    if (!prepared) {
      rc = launch_fast_prep(a, st);   // also clears the error words
      if (rc != COMMVQ_OK) return rc;
    }   // else: the previous call's merge left the running error word clear
    // the attention kernel copies the prepared state before its dependency wait: launch it as a
    // programmatic dependent only when the kernel before it is not the one writing that state
    rc = launch_attend_fast(a, q, q_dtype, S, st, prepared);
  } else if (run == COMMVQ_ATTN_DECODE_MMA) {
    if (!prepared) {
      rc = launch_attend_prep(a, st);   // also clears the error words
      if (rc != COMMVQ_OK) return rc;
    }   // else: the previous call's merge left the running error word clear
    rc = launch_attend_mma(a, q, q_dtype, S, st);
  } else if (run == COMMVQ_ATTN_GENERIC) {
    rc = launch_attend_generic(a, cfg, q, q_dtype, S, ws + L.tables_off, st);   // clears the error word
  } else {
    if (cudaMemsetAsync(a.error_word, 0, 2 * sizeof(int), st) != cudaSuccess) return COMMVQ_ERR_CUDA;
    // Timing events around the main kernel (external event nodes when the stream is captured).
    if (a.main_start && record_event(a.main_start, st) != cudaSuccess)
      return COMMVQ_ERR_CUDA;
    rc = launch_attend_table(a, q, q_dtype, S, st);
    if (rc == COMMVQ_OK && a.main_stop &&
        record_event(a.main_stop, st) !=
            cudaSuccess)
      return COMMVQ_ERR_CUDA;
  }
  if (rc != COMMVQ_OK) return rc;
  return launch_combine(a, partial_slots(cfg, run, S), st, fast && static_cast<int64_t>(S) * B >= di.sms);
}

extern "C" commvq_status commvq_attend_prepare(const commvq_config* cfg, int32_t B, int64_t max_T,
                                               const float* k_codebook, const float* v_codebook,
                                               void* workspace, size_t workspace_bytes,
                                               const commvq_attend_options* options, void* stream) {
  const NvtxRange nvtx_range("commvq_attend_prepare");
  const commvq_status cs = check_config(cfg);
  if (cs != COMMVQ_OK) return cs;
  if (B < 0 || max_T < 0) return COMMVQ_ERR_INVALID_ARG;
  const int algo = options ? options->algo : COMMVQ_ATTN_AUTO;
  if (options && (options->splits < 0 || options->splits > kMaxSplits)) return COMMVQ_ERR_INVALID_ARG;
  if (algo < COMMVQ_ATTN_AUTO || algo > COMMVQ_ATTN_GENERIC) return COMMVQ_ERR_INVALID_ARG;
  if (B == 0) return COMMVQ_OK;
  if (B > 65535) return COMMVQ_ERR_UNSUPPORTED;
  if (!k_codebook || !v_codebook || !workspace) return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(k_codebook, 16) || !aligned(v_codebook, 16) || !aligned(workspace, 256))
    return COMMVQ_ERR_INVALID_ARG;
  const int run = resolve_algo(cfg, options);
  if (!algo_supported(cfg, run)) return COMMVQ_ERR_UNSUPPORTED;
  const size_t need = commvq_attend_workspace_bytes(cfg, B, max_T, options);
  if (need == 0 || workspace_bytes < need) return COMMVQ_ERR_WORKSPACE;
  const DeviceInfo di = current_device_info();
  if (di.device < 0) return COMMVQ_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if (run != COMMVQ_ATTN_DECODE_MMA)
    return cudaMemsetAsync(workspace, 0, 2 * sizeof(int), st) == cudaSuccess ? COMMVQ_OK : COMMVQ_ERR_CUDA;
  const int S = choose_splits(run, B, cfg->q_heads, max_T, options);
  const bool fast = use_fast(cfg);
  const WorkspaceLayout L = workspace_layout(cfg, run, B, max_T, S, fast);
  AttendArgs a{};
  a.k_codebook = k_codebook;
  a.v_codebook = v_codebook;
  a.error_word = static_cast<int*>(workspace);
  a.k_img = reinterpret_cast<const uint4*>(ws + L.kimg_off);
  a.v_img = reinterpret_cast<const uint4*>(ws + L.vimg_off);
  set_phase_tables(a, ws + L.phase_off, fast);
  a.max_T = max_T;
  a.rope_base = cfg->rope_base;
  a.B = B;
  a.q_heads = cfg->q_heads;
  a.kv_heads = cfg->kv_heads;
  a.R = cfg->R;
  a.n_codes = cfg->n_codes;
  return fast ? launch_fast_prep(a, st) : launch_attend_prep(a, st);
}

namespace commvq {
int mma_splits(int B, int q_heads, int64_t max_T) {
  commvq_attend_options o{COMMVQ_ATTN_DECODE_MMA, 0, nullptr, nullptr, 0};
  return choose_splits(COMMVQ_ATTN_DECODE_MMA, B, q_heads, max_T, &o);
}

int attend_mma_setup(const commvq_config* cfg, int B, int64_t max_T, unsigned char* ws,
                     const int64_t* seq_offsets, const void* k_codes, const float* k_codebook, AttendArgs& a) {
  commvq_attend_options o{COMMVQ_ATTN_DECODE_MMA, 0, nullptr, nullptr, 0};
  const int S = choose_splits(COMMVQ_ATTN_DECODE_MMA, B, cfg->q_heads, max_T, &o);
  const WorkspaceLayout L = workspace_layout(cfg, COMMVQ_ATTN_DECODE_MMA, B, max_T, S, false);
  a.k_codes = static_cast<const uint8_t*>(k_codes);
  a.v_codes = static_cast<const uint8_t*>(k_codes);
  a.seq_offsets = seq_offsets;
  a.k_codebook = k_codebook;
  a.v_codebook = k_codebook;
  a.error_word = reinterpret_cast<int*>(ws);
  a.partials = reinterpret_cast<Partial*>(ws + L.partials_off);
  a.k_img = reinterpret_cast<const uint4*>(ws + L.kimg_off);
  a.v_img = reinterpret_cast<const uint4*>(ws + L.vimg_off);
  a.scores = reinterpret_cast<float*>(ws + L.scores_off);
  set_phase_tables(a, ws + L.phase_off, false);
  a.max_T = max_T;
  a.rope_base = cfg->rope_base;
  a.B = B;
  a.q_heads = cfg->q_heads;
  a.kv_heads = cfg->kv_heads;
  a.R = cfg->R;
  a.n_codes = cfg->n_codes;
  return S;
}
}  // namespace commvq

namespace commvq {
// one_per_sm: the kernel before has one CTA on every SM and lets this grid launch early. Its CTAs
// then take SMs as that kernel's CTAs leave; left alone, the scheduler stacks them on the first
// SMs to free up (at a 32K context: 128 CTAs on 46 SMs, three on most), where they share those
// SMs' load paths for every split's partials (spread out, that merge ran 0.9 us faster). A dynamic shared-memory request of over half an SM's capacity (unused by the kernel)
// leaves room for one merge CTA per SM, so they spread out. When the kernel before leaves SMs
// idle, the CTAs go there at once and stacking them costs less than waiting for SMs.
commvq_status launch_combine(const AttendArgs& a, int S, cudaStream_t st, bool one_per_sm) {
  size_t dyn = 0;
  if (one_per_sm) {
    const DeviceInfo di = current_device_info();
    if (di.device < 0) return COMMVQ_ERR_CUDA;
    dyn = di.smem_optin / 2 + 4096;
    if (cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn)) !=
        cudaSuccess)
      return COMMVQ_ERR_CUDA;
  }
  if (launch_dependent(combine_kernel, dim3(a.B * a.q_heads, kCombineQuarters), dim3(kCombineThreads), dyn, st, a,
                       S) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  return launch_status();
}
}  // namespace commvq

extern "C" commvq_status commvq_workspace_error(const void* workspace, int32_t* device_error,
                                                void* stream) {
  const NvtxRange nvtx_range("commvq_workspace_error");
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
    case COMMVQ_ERR_DEVICE_CHECK: return "device recorded a data error (code or sequence length out of range)";
    default: return "unknown status";
  }
}

extern "C" int32_t commvq_abi_version(void) { return 2; }
