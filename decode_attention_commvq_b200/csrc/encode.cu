// Residual nearest-codeword encoder (CommVQ abstract: additive quantization of every K/V
// vector; machine review "What carries the argument": g scalars share one index, R
// residual rounds).
//
// The work is a dense distance scan bound by the fp32 pipe: per row and group, R * Nc'
// candidate entries of 8 scalars, one subtract and one fused multiply-add each. HBM traffic
// is tiny in comparison (16 B of fp16 input and R code bytes per row and group).
//
// Grid: x = blocks of kThreads * kRowsPerThread rows, y = group j. The block stages a tile
// of its group's sub-codebook in shared memory; every thread reads the same entry at the
// same time (a broadcast), so the scan issues 2 shared loads per entry for kRowsPerThread
// rows of arithmetic.
#include "common.cuh"

namespace commvq {
namespace {

constexpr int kRowsPerThread = 2;
constexpr int kTile = 1024;   // codebook entries staged per pass (32 KB)

template <typename XT, bool kTrack>
__global__ void __launch_bounds__(kThreads)
encode_kernel(const XT* __restrict__ x, int64_t n_rows, int d, int R, int n_codes,
              const float* __restrict__ cb, void* __restrict__ codes, int code_bytes,
              unsigned long long* __restrict__ near_ties, float* __restrict__ residual_out) {
  __shared__ float4 tile[kTile * 2];
  const int G = d / kG;
  const int j = blockIdx.y;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * (kThreads * kRowsPerThread) + threadIdx.x;

  float res[kRowsPerThread][kG];
  bool valid[kRowsPerThread];
#pragma unroll
  for (int i = 0; i < kRowsPerThread; ++i) {
    const int64_t n = row0 + static_cast<int64_t>(i) * kThreads;
    valid[i] = n < n_rows;
    if (valid[i]) {
      load_row8(x + n * d + j * kG, res[i]);
    } else {
#pragma unroll
      for (int k = 0; k < kG; ++k) res[i][k] = 0.0f;
    }
  }

  unsigned ties = 0;
  for (int r = 0; r < R; ++r) {
    const float* sub = cb + (static_cast<int64_t>(r) * G + j) * n_codes * kG;
    Nearest best[kRowsPerThread];
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) nearest_init(best[i]);

    for (int c0 = 0; c0 < n_codes; c0 += kTile) {
      const int n = min(kTile, n_codes - c0);
      __syncthreads();
      for (int e = threadIdx.x; e < 2 * n; e += kThreads)
        tile[e] = __ldg(reinterpret_cast<const float4*>(sub + static_cast<int64_t>(c0) * kG) + e);
      __syncthreads();
#pragma unroll 4
      for (int c = 0; c < n; ++c) {
        const float4 lo = tile[2 * c];
        const float4 hi = tile[2 * c + 1];
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) nearest_step<kTrack>(best[i], res[i], lo, hi, c0 + c);
      }
    }

#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
      const int64_t n = row0 + static_cast<int64_t>(i) * kThreads;
      if (!valid[i]) continue;
      if (kTrack) ties += near_tie(best[i], n_codes) ? 1u : 0u;
      store_code(codes, (n * R + r) * G + j, best[i].idx, code_bytes);
      float w[kG];
      load_row8(sub + static_cast<int64_t>(best[i].idx) * kG, w);
#pragma unroll
      for (int k = 0; k < kG; ++k) res[i][k] = __fsub_rn(res[i][k], w[k]);
    }
  }

  if (residual_out) {
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
      const int64_t n = row0 + static_cast<int64_t>(i) * kThreads;
      if (!valid[i]) continue;
      float4* dst = reinterpret_cast<float4*>(residual_out + n * d + j * kG);
      dst[0] = make_float4(res[i][0], res[i][1], res[i][2], res[i][3]);
      dst[1] = make_float4(res[i][4], res[i][5], res[i][6], res[i][7]);
    }
  }

  if (kTrack) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ties += __shfl_xor_sync(0xffffffffu, ties, o);
    if ((threadIdx.x & 31) == 0 && ties) atomicAdd(near_ties, static_cast<unsigned long long>(ties));
  }
}

template <typename XT>
void launch_encode(const XT* x, int64_t n_rows, int d, int R, int n_codes, const float* cb,
                   void* codes, int code_bytes, unsigned long long* near_ties, float* residual_out,
                   cudaStream_t s) {
  const int64_t per_block = kThreads * kRowsPerThread;
  dim3 grid(static_cast<unsigned>((n_rows + per_block - 1) / per_block), d / kG);
  if (near_ties)
    encode_kernel<XT, true><<<grid, kThreads, 0, s>>>(x, n_rows, d, R, n_codes, cb, codes,
                                                      code_bytes, near_ties, residual_out);
  else
    encode_kernel<XT, false><<<grid, kThreads, 0, s>>>(x, n_rows, d, R, n_codes, cb, codes,
                                                       code_bytes, nullptr, residual_out);
}

}  // namespace
}  // namespace commvq

using namespace commvq;

extern "C" commvq_status commvq_encode(const commvq_config* cfg, const void* x, commvq_dtype x_dtype,
                                       int64_t n_tokens, const float* codebook, void* codes,
                                       unsigned long long* near_ties, float* residual_out,
                                       void* stream) {
  if (!cfg) return COMMVQ_ERR_INVALID_ARG;
  const int d = cfg->d, g = cfg->g, R = cfg->R, Nc = cfg->n_codes, H = cfg->kv_heads;
  if (d <= 0 || g <= 0 || d % g || g % 2 || R < 1 || Nc < 1 || H < 1 || n_tokens < 0)
    return COMMVQ_ERR_INVALID_ARG;
  if (cfg->code_bytes != (Nc <= 256 ? 1 : 2)) return COMMVQ_ERR_INVALID_ARG;
  if (Nc > 65536) return COMMVQ_ERR_INVALID_ARG;
  if (g != kG || R > 16) return COMMVQ_ERR_UNSUPPORTED;
  if (x_dtype != COMMVQ_F32 && x_dtype != COMMVQ_F16) return COMMVQ_ERR_UNSUPPORTED;
  if (n_tokens == 0) return COMMVQ_OK;
  if (!x || !codebook || !codes) return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codebook, 16) || !aligned(near_ties, 8) || !aligned(residual_out, 16))
    return COMMVQ_ERR_INVALID_ARG;
  const int64_t n_rows = n_tokens * H;
  if (n_rows / H != n_tokens || (n_rows + kThreads * kRowsPerThread) / (kThreads * kRowsPerThread) > INT32_MAX)
    return COMMVQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (x_dtype == COMMVQ_F32)
    launch_encode(static_cast<const float*>(x), n_rows, d, R, Nc, codebook, codes, cfg->code_bytes,
                  near_ties, residual_out, s);
  else
    launch_encode(static_cast<const __half*>(x), n_rows, d, R, Nc, codebook, codes, cfg->code_bytes,
                  near_ties, residual_out, s);
  return launch_status();
}
