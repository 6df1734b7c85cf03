// Residual nearest-codeword encoder (CommVQ abstract: additive quantization of every K/V
// vector; machine review "What carries the argument": g scalars share one index, R
// residual rounds).
//
// The work is a dense distance scan bound by the fp32 pipe: per row and group, R * Nc'
// candidate entries of g scalars, one subtract and one fused multiply-add each. HBM traffic
// is tiny in comparison (2g B of fp16 input and R code bytes per row and group).
//
// Grid: x = blocks of kThreads rows (2 kThreads for g = 8), y = group j. The block stages a
// tile of its group's sub-codebook in shared memory; every thread reads the same entry at the
// same time (a broadcast), so the scan issues g/4 shared loads per entry for 1 (g = 8: 2)
// rows of arithmetic. For g = 8 the tile holds entries in pairs and the scan runs on sm_100's
// packed fp32x2 instructions, two entries per instruction with each lane the scalar rule. g = 8 is the library's attention layout; 16, 32 and 64 cover the
// pages' own setting (g = 64, Nc' = 64, R = 21 or 11).
#include "common.cuh"

namespace commvq {
namespace {

constexpr int kTileFloats = 8192;   // codebook floats staged per pass (32 KB)

// One tensor's encode: rows, codebook, codes out, residual out (nullable). A launch covers one
// or two of them (blockIdx.z), e.g. a decode step's new key row and value row together.
template <typename XT>
struct EncodeJob {
  const XT* x;
  const float* cb;
  void* codes;
  float* residual_out;
};
template <typename XT>
struct EncodeJobs {
  EncodeJob<XT> job[2];
};

// Rows per thread: g = 8 takes two (independent distance chains for the packed scan, and one
// shared-memory read of an entry pair serves both; four rows need ~160 registers and run slower),
// larger groups one.
template <int GG>
constexpr int kEncodeRows = GG == 8 ? 2 : 1;

// GG: scalars per group (8, 16, 32 or 64). Each thread encodes kRows rows of one group.
template <typename XT, bool kTrack, int GG>
__global__ void __launch_bounds__(kThreads)
encode_kernel(EncodeJobs<XT> jobs, int64_t n_rows, int d, int R, int n_codes, int code_bytes,
              unsigned long long* __restrict__ near_ties) {
  const XT* __restrict__ x = jobs.job[blockIdx.z].x;
  const float* __restrict__ cb = jobs.job[blockIdx.z].cb;
  void* __restrict__ codes = jobs.job[blockIdx.z].codes;
  float* __restrict__ residual_out = jobs.job[blockIdx.z].residual_out;
  constexpr int kRows = kEncodeRows<GG>;
  constexpr int kTile = kTileFloats / GG;   // entries per pass
  __shared__ float4 tile[kTileFloats / 4];
  const int G = d / GG;
  const int j = blockIdx.y;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * (kThreads * kRows) + threadIdx.x;

  float res[kRows][GG];
  bool valid[kRows];
#pragma unroll
  for (int i = 0; i < kRows; ++i) {
    const int64_t n = row0 + static_cast<int64_t>(i) * kThreads;
    valid[i] = n < n_rows;
#pragma unroll
    for (int q = 0; q < GG / kG; ++q) {
      float v[kG];
      if (valid[i]) {
        load_row8(x + n * d + j * GG + q * kG, v);
      } else {
#pragma unroll
        for (int k = 0; k < kG; ++k) v[k] = 0.0f;
      }
#pragma unroll
      for (int k = 0; k < kG; ++k) res[i][q * kG + k] = v[k];
    }
  }

  unsigned ties = 0;
  for (int r = 0; r < R; ++r) {
    const float* sub = cb + (static_cast<int64_t>(r) * G + j) * n_codes * GG;
    Nearest best[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) nearest_init(best[i]);

    if constexpr (GG == kG) {
      // packed scan: two entries per fp32x2 instruction, each lane the scalar rule
      f32x2 res2[kRows][kG];
#pragma unroll
      for (int i = 0; i < kRows; ++i)
#pragma unroll
        for (int k = 0; k < kG; ++k) res2[i][k] = pack2(res[i][k], res[i][k]);
      for (int c0 = 0; c0 < n_codes; c0 += kTile) {
        const int n = min(kTile, n_codes - c0);
        __syncthreads();
        stage_pairs8(tile, sub + static_cast<int64_t>(c0) * GG, n);
        __syncthreads();
        const int pairs = n >> 1;
#pragma unroll 2
        for (int p = 0; p < pairs; ++p) {
#pragma unroll
          for (int i = 0; i < kRows; ++i) {
            float d0, d1;
            unpack2(pair_dist8(res2[i], tile + 4 * p), d0, d1);
            nearest_take<kTrack>(best[i], d0, c0 + 2 * p);
            nearest_take<kTrack>(best[i], d1, c0 + 2 * p + 1);
          }
        }
        if (n & 1) {
#pragma unroll
          for (int i = 0; i < kRows; ++i) {
            float d0, d1;
            unpack2(pair_dist8(res2[i], tile + 4 * pairs), d0, d1);
            nearest_take<kTrack>(best[i], d0, c0 + n - 1);
          }
        }
      }
    } else {
      for (int c0 = 0; c0 < n_codes; c0 += kTile) {
        const int n = min(kTile, n_codes - c0);
        __syncthreads();
        for (int e = threadIdx.x; e < n * (GG / 4); e += kThreads)
          tile[e] = __ldg(reinterpret_cast<const float4*>(sub + static_cast<int64_t>(c0) * GG) + e);
        __syncthreads();
#pragma unroll 2
        for (int c = 0; c < n; ++c) {
#pragma unroll
          for (int i = 0; i < kRows; ++i) nearest_step_g<GG, kTrack>(best[i], res[i], tile + c * (GG / 4), c0 + c);
        }
      }
    }

#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const int64_t n = row0 + static_cast<int64_t>(i) * kThreads;
      if (!valid[i]) continue;
      if (kTrack) ties += near_tie(best[i], n_codes) ? 1u : 0u;
      store_code(codes, (n * R + r) * G + j, best[i].idx, code_bytes);
#pragma unroll
      for (int q = 0; q < GG / kG; ++q) {
        float w[kG];
        load_row8(sub + static_cast<int64_t>(best[i].idx) * GG + q * kG, w);
#pragma unroll
        for (int k = 0; k < kG; ++k) res[i][q * kG + k] = __fsub_rn(res[i][q * kG + k], w[k]);
      }
    }
  }

  if (residual_out) {
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const int64_t n = row0 + static_cast<int64_t>(i) * kThreads;
      if (!valid[i]) continue;
      float4* dst = reinterpret_cast<float4*>(residual_out + n * d + j * GG);
#pragma unroll
      for (int q = 0; q < GG / 4; ++q)
        dst[q] = make_float4(res[i][4 * q], res[i][4 * q + 1], res[i][4 * q + 2], res[i][4 * q + 3]);
    }
  }

  if (kTrack) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ties += __shfl_xor_sync(0xffffffffu, ties, o);
    if ((threadIdx.x & 31) == 0 && ties) atomicAdd(near_ties, static_cast<unsigned long long>(ties));
  }
}

// Few rows (a decode step's new position): kWarpsPerUnit warps per (row, group), so that each lane
// scans only a few entries and a round costs one round trip of entry loads. Warp p of a unit takes
// entries p*32 + lane, p*32 + lane + 128, ... in increasing order with the same fp32 distance rule
// (entries read through L1/L2); each warp merges (best, index, second best) over its lanes by
// shuffles, and the unit's warps then merge their four results through shared memory. The merge
// is exact in any order (the smallest distance wins, ties go to the lowest entry, the second best
// is the second smallest distance overall): what the in-order scan of encode_kernel produces, so
// codes and near-tie counts are the same.
constexpr int kWarpsPerUnit = 4;
constexpr int kWarpUnitsPerBlock = 2;   // 8 warps per block

__device__ __forceinline__ void nearest_merge(Nearest& n, float ob, int oi, float os) {
  const float hi = fmaxf(n.best, ob);
  if (ob < n.best || (ob == n.best && oi < n.idx)) {
    n.best = ob;
    n.idx = oi;
  }
  n.second = fminf(hi, fminf(n.second, os));
}

template <typename XT, bool kTrack, int GG>
__global__ void __launch_bounds__(32 * kWarpsPerUnit * kWarpUnitsPerBlock)
encode_warp_kernel(EncodeJobs<XT> jobs, int64_t n_rows, int d, int R, int n_codes, int code_bytes,
                   unsigned long long* __restrict__ near_ties) {
  // launched as a programmatic dependent: the launch overlaps the kernel before, and the wait
  // gives it that kernel's writes (the rows, a step's input copy) before anything is read or
  // written. Then a following dependent (a decode step's attention) may start its own set-up; it
  // waits for this grid before it reads the codes.
  pdl_wait();
  pdl_trigger();
  __shared__ float m_best[kWarpUnitsPerBlock][kWarpsPerUnit];
  __shared__ float m_second[kWarpUnitsPerBlock][kWarpsPerUnit];
  __shared__ int m_idx[kWarpUnitsPerBlock][kWarpsPerUnit];
  const XT* __restrict__ x = jobs.job[blockIdx.z].x;
  const float* __restrict__ cb = jobs.job[blockIdx.z].cb;
  void* __restrict__ codes = jobs.job[blockIdx.z].codes;
  float* __restrict__ residual_out = jobs.job[blockIdx.z].residual_out;
  const int G = d / GG;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ul = warp / kWarpsPerUnit, part = warp % kWarpsPerUnit;
  const int64_t unit = static_cast<int64_t>(blockIdx.x) * kWarpUnitsPerBlock + ul;
  const bool valid = unit < n_rows * G;   // every warp stays for the block barriers
  const int64_t n = valid ? unit / G : 0;
  const int j = valid ? static_cast<int>(unit - n * G) : 0;
  const bool leader = valid && part == 0 && lane == 0;
  float res[GG];
#pragma unroll
  for (int q = 0; q < GG / kG; ++q) {
    float v[kG];
    if (valid) {
      load_row8(x + n * d + j * GG + q * kG, v);
    } else {
#pragma unroll
      for (int k = 0; k < kG; ++k) v[k] = 0.0f;
    }
#pragma unroll
    for (int k = 0; k < kG; ++k) res[q * kG + k] = v[k];
  }
  unsigned ties = 0;
  for (int r = 0; r < R; ++r) {
    const float* sub = cb + (static_cast<int64_t>(r) * G + j) * n_codes * GG;
    Nearest best;
    nearest_init(best);
    if (valid)
      for (int c = part * 32 + lane; c < n_codes; c += 32 * kWarpsPerUnit)
        nearest_step_g<GG, kTrack>(best, res, reinterpret_cast<const float4*>(sub + static_cast<int64_t>(c) * GG), c);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best.best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, best.idx, o);
      const float os = __shfl_xor_sync(0xffffffffu, best.second, o);
      nearest_merge(best, ob, oi, os);
    }
    if (lane == 0) {
      m_best[ul][part] = best.best;
      m_second[ul][part] = best.second;
      m_idx[ul][part] = best.idx;
    }
    __syncthreads();
    Nearest u;
    u.best = m_best[ul][0];
    u.second = m_second[ul][0];
    u.idx = m_idx[ul][0];
#pragma unroll
    for (int p = 1; p < kWarpsPerUnit; ++p) nearest_merge(u, m_best[ul][p], m_idx[ul][p], m_second[ul][p]);
    __syncthreads();   // the slots are written again in the next round
    if (leader) {
      if (kTrack) ties += near_tie(u, n_codes) ? 1u : 0u;
      store_code(codes, (n * R + r) * G + j, u.idx, code_bytes);
    }
    if (valid) {
#pragma unroll
      for (int q = 0; q < GG / kG; ++q) {
        float w[kG];
        load_row8(sub + static_cast<int64_t>(u.idx) * GG + q * kG, w);
#pragma unroll
        for (int k = 0; k < kG; ++k) res[q * kG + k] = __fsub_rn(res[q * kG + k], w[k]);
      }
    }
  }
  if (residual_out && leader) {
    float4* dst = reinterpret_cast<float4*>(residual_out + n * d + j * GG);
#pragma unroll
    for (int q = 0; q < GG / 4; ++q) dst[q] = make_float4(res[4 * q], res[4 * q + 1], res[4 * q + 2], res[4 * q + 3]);
  }
  if (kTrack && leader && ties) atomicAdd(near_ties, static_cast<unsigned long long>(ties));
}

// Row counts up to this many (row, group) units take the warp-per-unit kernel.
constexpr int64_t kWarpEncodeMaxUnits = 4096;

template <typename XT, int GG>
void launch_encode_g(const EncodeJobs<XT>& jobs, int n_jobs, int64_t n_rows, int d, int R, int n_codes,
                     int code_bytes, unsigned long long* near_ties, cudaStream_t s) {
  const int64_t units = n_rows * (d / GG);
  if (units <= kWarpEncodeMaxUnits) {
    const unsigned blocks = static_cast<unsigned>((units + kWarpUnitsPerBlock - 1) / kWarpUnitsPerBlock);
    const dim3 grid(blocks, 1, n_jobs);
    const dim3 block(32 * kWarpsPerUnit * kWarpUnitsPerBlock);
    if (near_ties)
      (void)launch_dependent(encode_warp_kernel<XT, true, GG>, grid, block, 0, s, jobs, n_rows, d, R, n_codes,
                             code_bytes, near_ties);
    else
      (void)launch_dependent(encode_warp_kernel<XT, false, GG>, grid, block, 0, s, jobs, n_rows, d, R, n_codes,
                             code_bytes, static_cast<unsigned long long*>(nullptr));
    return;
  }
  const int64_t per_block = kThreads * kEncodeRows<GG>;
  dim3 grid(static_cast<unsigned>((n_rows + per_block - 1) / per_block), d / GG, n_jobs);
  if (near_ties)
    encode_kernel<XT, true, GG><<<grid, kThreads, 0, s>>>(jobs, n_rows, d, R, n_codes, code_bytes, near_ties);
  else
    encode_kernel<XT, false, GG><<<grid, kThreads, 0, s>>>(jobs, n_rows, d, R, n_codes, code_bytes, nullptr);
}

template <typename XT>
void launch_encode(const EncodeJobs<XT>& jobs, int n_jobs, int64_t n_rows, int d, int g, int R, int n_codes,
                   int code_bytes, unsigned long long* near_ties, cudaStream_t s) {
  switch (g) {
    case 8: launch_encode_g<XT, 8>(jobs, n_jobs, n_rows, d, R, n_codes, code_bytes, near_ties, s); break;
    case 16: launch_encode_g<XT, 16>(jobs, n_jobs, n_rows, d, R, n_codes, code_bytes, near_ties, s); break;
    case 32: launch_encode_g<XT, 32>(jobs, n_jobs, n_rows, d, R, n_codes, code_bytes, near_ties, s); break;
    default: launch_encode_g<XT, 64>(jobs, n_jobs, n_rows, d, R, n_codes, code_bytes, near_ties, s); break;
  }
}

// Host checks shared by the one- and two-tensor calls: OK, INVALID_ARG or UNSUPPORTED.
commvq_status check_encode(const commvq_config* cfg, commvq_dtype x_dtype, int64_t n_tokens) {
  if (!cfg) return COMMVQ_ERR_INVALID_ARG;
  const int d = cfg->d, g = cfg->g, R = cfg->R, Nc = cfg->n_codes, H = cfg->kv_heads;
  if (d <= 0 || g <= 0 || d % g || g % 2 || R < 1 || Nc < 1 || H < 1 || n_tokens < 0)
    return COMMVQ_ERR_INVALID_ARG;
  if (cfg->code_bytes != (Nc <= 256 ? 1 : 2)) return COMMVQ_ERR_INVALID_ARG;
  if (Nc > 65536) return COMMVQ_ERR_INVALID_ARG;
  if ((g != 8 && g != 16 && g != 32 && g != 64) || R > 32) return COMMVQ_ERR_UNSUPPORTED;
  if (x_dtype != COMMVQ_F32 && x_dtype != COMMVQ_F16) return COMMVQ_ERR_UNSUPPORTED;
  const int64_t n_rows = n_tokens * H;
  if (n_tokens > 0 && (n_rows / H != n_tokens || (n_rows + kThreads) / kThreads > INT32_MAX))
    return COMMVQ_ERR_INVALID_ARG;
  return COMMVQ_OK;
}

commvq_status run_encode(const commvq_config* cfg, commvq_dtype x_dtype, int64_t n_tokens, const void* const* x,
                         const float* const* cb, void* const* codes, float* const* residual, int n_jobs,
                         unsigned long long* near_ties, cudaStream_t s) {
  const int64_t n_rows = n_tokens * cfg->kv_heads;
  if (x_dtype == COMMVQ_F32) {
    EncodeJobs<float> jobs{};
    for (int k = 0; k < n_jobs; ++k) jobs.job[k] = {static_cast<const float*>(x[k]), cb[k], codes[k], residual[k]};
    launch_encode(jobs, n_jobs, n_rows, cfg->d, cfg->g, cfg->R, cfg->n_codes, cfg->code_bytes, near_ties, s);
  } else {
    EncodeJobs<__half> jobs{};
    for (int k = 0; k < n_jobs; ++k) jobs.job[k] = {static_cast<const __half*>(x[k]), cb[k], codes[k], residual[k]};
    launch_encode(jobs, n_jobs, n_rows, cfg->d, cfg->g, cfg->R, cfg->n_codes, cfg->code_bytes, near_ties, s);
  }
  return launch_status();
}

}  // namespace
}  // namespace commvq

using namespace commvq;

extern "C" commvq_status commvq_encode(const commvq_config* cfg, const void* x, commvq_dtype x_dtype,
                                       int64_t n_tokens, const float* codebook, void* codes,
                                       unsigned long long* near_ties, float* residual_out,
                                       void* stream) {
  const NvtxRange nvtx_range("commvq_encode");
  const commvq_status cs = check_encode(cfg, x_dtype, n_tokens);
  if (cs != COMMVQ_OK) return cs;
  if (n_tokens == 0) return COMMVQ_OK;
  if (!x || !codebook || !codes) return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codebook, 16) || !aligned(near_ties, 8) || !aligned(residual_out, 16))
    return COMMVQ_ERR_INVALID_ARG;
  const void* xs[1] = {x};
  const float* cbs[1] = {codebook};
  void* cs1[1] = {codes};
  float* rs[1] = {residual_out};
  return run_encode(cfg, x_dtype, n_tokens, xs, cbs, cs1, rs, 1, near_ties, static_cast<cudaStream_t>(stream));
}

extern "C" commvq_status commvq_encode_kv(const commvq_config* cfg, const void* k_x, const void* v_x,
                                          commvq_dtype x_dtype, int64_t n_tokens, const float* k_codebook,
                                          const float* v_codebook, void* k_codes, void* v_codes,
                                          unsigned long long* near_ties, void* stream) {
  const NvtxRange nvtx_range("commvq_encode_kv");
  const commvq_status cs = check_encode(cfg, x_dtype, n_tokens);
  if (cs != COMMVQ_OK) return cs;
  if (n_tokens == 0) return COMMVQ_OK;
  if (!k_x || !v_x || !k_codebook || !v_codebook || !k_codes || !v_codes) return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(k_x, 16) || !aligned(v_x, 16) || !aligned(k_codebook, 16) || !aligned(v_codebook, 16) ||
      !aligned(near_ties, 8))
    return COMMVQ_ERR_INVALID_ARG;
  const void* xs[2] = {k_x, v_x};
  const float* cbs[2] = {k_codebook, v_codebook};
  void* cs2[2] = {k_codes, v_codes};
  float* rs[2] = {nullptr, nullptr};
  return run_encode(cfg, x_dtype, n_tokens, xs, cbs, cs2, rs, 2, near_ties, static_cast<cudaStream_t>(stream));
}
