// One EM step of a residual round's codebook (review: codebook fit by EM, Algorithm 1 /
// Eq. 20 -- hard assignment, closed-form centroid update).
//
// Kernel 1 (grid: row chunks x groups): assigns every row of the chunk to its nearest
// entry with the encoder's exact fp32 rule, then sums the assigned sub-vectors per entry
// in fp64. Each entry's sum is taken by one thread over the chunk's rows in row order, so
// the partial is independent of scheduling. Kernel 2 (grid: entries) adds the chunk
// partials in chunk order and writes (float)(sum / count), keeping entries that no row
// chose; it also reduces the SSE partials in a fixed order. The whole step is therefore
// deterministic run to run.
#include "common.cuh"

namespace commvq {
namespace {

constexpr int kRowsPerThread = 2;
constexpr int kSub = kThreads * kRowsPerThread;   // rows assigned per pass
constexpr int kChunkRows = 512;                   // rows per CTA (4096 rows fill 128 CTAs)
constexpr int kTile = 1024;                       // codebook entries staged per pass
constexpr int kMaxCodes = 4096;

struct EmLayout {
  int64_t chunks;
  size_t sums_off, counts_off, sse_off, total;
};

EmLayout em_layout(int64_t N, int G, int Nc) {
  EmLayout L;
  L.chunks = (N + kChunkRows - 1) / kChunkRows;
  L.sums_off = 0;
  L.counts_off = round_up(L.sums_off + sizeof(double) * L.chunks * G * Nc * kG, 256);
  L.sse_off = round_up(L.counts_off + sizeof(int32_t) * L.chunks * G * Nc, 256);
  L.total = round_up(L.sse_off + sizeof(double) * L.chunks * G, 256);
  return L;
}

__global__ void __launch_bounds__(kThreads)
em_assign_kernel(const float* __restrict__ rows, int64_t N, int d, int Nc,
                 const float* __restrict__ cb, void* __restrict__ codes_out, int code_bytes,
                 double* __restrict__ psum, int32_t* __restrict__ pcnt, double* __restrict__ psse) {
  __shared__ float4 tile[kTile * 2];
  __shared__ uint16_t code_s[kChunkRows];
  __shared__ float dist_s[kChunkRows];
  __shared__ double red[kThreads];
  const int G = d / kG;
  const int j = blockIdx.y;
  const int64_t chunk = blockIdx.x;
  const int64_t base = chunk * kChunkRows;
  const int rows_here = static_cast<int>(min(static_cast<int64_t>(kChunkRows), N - base));
  const float* sub_cb = cb + static_cast<int64_t>(j) * Nc * kG;

  for (int s0 = 0; s0 < rows_here; s0 += kSub) {
    float res[kRowsPerThread][kG];
    Nearest best[kRowsPerThread];
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
      const int li = s0 + threadIdx.x + i * kThreads;
      nearest_init(best[i]);
      if (li < rows_here) {
        load_row8(rows + (base + li) * d + j * kG, res[i]);
      } else {
#pragma unroll
        for (int k = 0; k < kG; ++k) res[i][k] = 0.0f;
      }
    }
    for (int c0 = 0; c0 < Nc; c0 += kTile) {
      const int n = min(kTile, Nc - c0);
      __syncthreads();
      for (int e = threadIdx.x; e < 2 * n; e += kThreads)
        tile[e] = __ldg(reinterpret_cast<const float4*>(sub_cb + static_cast<int64_t>(c0) * kG) + e);
      __syncthreads();
#pragma unroll 4
      for (int c = 0; c < n; ++c) {
        const float4 lo = tile[2 * c];
        const float4 hi = tile[2 * c + 1];
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) nearest_step<false>(best[i], res[i], lo, hi, c0 + c);
      }
    }
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
      const int li = s0 + threadIdx.x + i * kThreads;
      if (li < rows_here) {
        code_s[li] = static_cast<uint16_t>(best[i].idx);
        dist_s[li] = best[i].best;
        if (codes_out) store_code(codes_out, (base + li) * G + j, best[i].idx, code_bytes);
      }
    }
  }
  __syncthreads();

  // SSE of the chunk: thread t sums rows t, t + 256, ... in order, then a fixed tree.
  double sse = 0.0;
  for (int li = threadIdx.x; li < rows_here; li += kThreads) sse += static_cast<double>(dist_s[li]);
  red[threadIdx.x] = sse;
  __syncthreads();
  for (int w = kThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) psse[chunk * G + j] = red[0];

  // Per-entry sums of the assigned sub-vectors, in row order.
  for (int c = threadIdx.x; c < Nc; c += kThreads) {
    double acc[kG];
#pragma unroll
    for (int k = 0; k < kG; ++k) acc[k] = 0.0;
    int cnt = 0;
    for (int li = 0; li < rows_here; ++li) {
      if (code_s[li] != c) continue;
      float v[kG];
      load_row8(rows + (base + li) * d + j * kG, v);
#pragma unroll
      for (int k = 0; k < kG; ++k) acc[k] += static_cast<double>(v[k]);
      ++cnt;
    }
    const int64_t at = (chunk * G + j) * Nc + c;
#pragma unroll
    for (int k = 0; k < kG; ++k) psum[at * kG + k] = acc[k];
    pcnt[at] = cnt;
  }
}

__global__ void __launch_bounds__(kThreads)
em_update_kernel(int64_t chunks, int G, int Nc, float* __restrict__ cb, const double* __restrict__ psum,
                 const int32_t* __restrict__ pcnt, const double* __restrict__ psse,
                 double* __restrict__ sse_out) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;   // j * Nc + c
  if (e < static_cast<int64_t>(G) * Nc) {
    double acc[kG];
#pragma unroll
    for (int k = 0; k < kG; ++k) acc[k] = 0.0;
    int64_t cnt = 0;
    for (int64_t ch = 0; ch < chunks; ++ch) {
      const int64_t at = ch * G * Nc + e;
      const int32_t m = pcnt[at];
      if (m == 0) continue;
      cnt += m;
#pragma unroll
      for (int k = 0; k < kG; ++k) acc[k] += psum[at * kG + k];
    }
    if (cnt > 0) {
#pragma unroll
      for (int k = 0; k < kG; ++k) cb[e * kG + k] = __double2float_rn(acc[k] / static_cast<double>(cnt));
    }
  }
  if (sse_out && blockIdx.x == 0 && threadIdx.x == 0) {
    double s = 0.0;
    for (int64_t i = 0; i < chunks * G; ++i) s += psse[i];
    *sse_out = s;
  }
}

}  // namespace
}  // namespace commvq

using namespace commvq;

static commvq_status em_check(const commvq_config* cfg, int64_t N) {
  if (!cfg) return COMMVQ_ERR_INVALID_ARG;
  const int d = cfg->d, g = cfg->g, Nc = cfg->n_codes;
  if (d <= 0 || g <= 0 || d % g || g % 2 || Nc < 1 || Nc > 65536 || N < 1) return COMMVQ_ERR_INVALID_ARG;
  if (cfg->code_bytes != (Nc <= 256 ? 1 : 2)) return COMMVQ_ERR_INVALID_ARG;
  if (g != kG || Nc > kMaxCodes) return COMMVQ_ERR_UNSUPPORTED;
  if ((N + kChunkRows - 1) / kChunkRows > INT32_MAX) return COMMVQ_ERR_UNSUPPORTED;
  return COMMVQ_OK;
}

extern "C" size_t commvq_em_workspace_bytes(const commvq_config* cfg, int64_t N) {
  if (em_check(cfg, N) != COMMVQ_OK) return 0;
  return em_layout(N, cfg->d / kG, cfg->n_codes).total;
}

extern "C" commvq_status commvq_em_step(const commvq_config* cfg, const float* rows, int64_t N,
                                        float* codebook_round, void* codes_out, double* sse_out,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  const commvq_status cs = em_check(cfg, N);
  if (cs != COMMVQ_OK) return cs;
  if (!rows || !codebook_round || !workspace) return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(rows, 16) || !aligned(codebook_round, 16) || !aligned(sse_out, 8) ||
      !aligned(workspace, 256) || !aligned(codes_out, cfg->code_bytes))
    return COMMVQ_ERR_INVALID_ARG;
  const int G = cfg->d / kG, Nc = cfg->n_codes;
  const EmLayout L = em_layout(N, G, Nc);
  if (workspace_bytes < L.total) return COMMVQ_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  double* psum = reinterpret_cast<double*>(ws + L.sums_off);
  int32_t* pcnt = reinterpret_cast<int32_t*>(ws + L.counts_off);
  double* psse = reinterpret_cast<double*>(ws + L.sse_off);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 g1(static_cast<unsigned>(L.chunks), G);
  em_assign_kernel<<<g1, kThreads, 0, st>>>(rows, N, cfg->d, Nc, codebook_round, codes_out,
                                            cfg->code_bytes, psum, pcnt, psse);
  commvq_status rc = launch_status();
  if (rc != COMMVQ_OK) return rc;
  const unsigned g2 = static_cast<unsigned>((static_cast<int64_t>(G) * Nc + kThreads - 1) / kThreads);
  em_update_kernel<<<g2, kThreads, 0, st>>>(L.chunks, G, Nc, codebook_round, psum, pcnt, psse, sse_out);
  return launch_status();
}
