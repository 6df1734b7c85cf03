// One EM step of a residual round's codebook (review: codebook fit by EM, Algorithm 1 /
// Eq. 20 -- hard assignment, closed-form centroid update). The hard step takes g = 8, 16, 32
// or 64 scalars per group (g = 64 is the pages' own setting); the soft step takes g = 8.
//
// Kernel 1 (grid: row chunks x groups; 512-row chunks, 256 when that leaves fewer than two CTAs
// per SM, e.g. a 4096-row fit): assigns every row of the chunk to its nearest
// entry with the encoder's exact fp32 rule, then sums the assigned sub-vectors per entry
// in fp64. Each entry's sum is taken by one thread over the chunk's rows in row order, so
// the partial is independent of scheduling. Kernel 2 (grid: entries) adds the chunk
// partials in chunk order and writes (float)(sum / count), keeping entries that no row
// chose; it also reduces the SSE partials in a fixed order. The whole step is therefore
// deterministic run to run.
#include <math.h>

#include "common.cuh"

namespace commvq {
namespace {

constexpr int kChunkRows = 512;                   // rows per CTA of the hard step, at most
constexpr int64_t kFillCtas = 2 * 148;            // CTAs below which chunks halve (two per B200 SM)
constexpr int kTile = 1024;                       // codebook entries staged per pass (g = 8)
constexpr int kTileFloats = kTile * kG;           // 32 KB of entries per pass, any g
constexpr int kMaxCodes = 4096;

constexpr int kSoftChunkRows = 256;               // rows per CTA of the soft step

// Workspace regions, sized for the larger chunk count of the two steps: per (chunk, group,
// entry) fp64 sums of g scalars, then 8 bytes (int32 counts of the hard step or fp64 weight
// sums of the soft step), then per (chunk, group) fp64 SSE partials.
struct EmLayout {
  int chunk_rows;         // hard-step rows per chunk: 512, or 256 when 512 would leave SMs idle
  int64_t chunks;        // hard-step chunks
  int64_t soft_chunks;   // soft-step chunks
  size_t sums_off, counts_off, sse_off, total;
};

EmLayout em_layout(int64_t N, int G, int Nc, int g) {
  EmLayout L;
  L.chunk_rows = ((N + kChunkRows - 1) / kChunkRows) * G >= kFillCtas ? kChunkRows : kChunkRows / 2;
  L.chunks = (N + L.chunk_rows - 1) / L.chunk_rows;
  L.soft_chunks = (N + kSoftChunkRows - 1) / kSoftChunkRows;
  const int64_t cap = L.soft_chunks > L.chunks ? L.soft_chunks : L.chunks;
  L.sums_off = 0;
  L.counts_off = round_up(L.sums_off + sizeof(double) * cap * G * Nc * g, 256);
  L.sse_off = round_up(L.counts_off + sizeof(double) * cap * G * Nc, 256);
  L.total = round_up(L.sse_off + sizeof(double) * cap * G, 256);
  return L;
}

// GG: scalars per group (8, 16, 32 or 64); kRowsT rows per thread and pass (2 for GG = 8 with
// 512-row chunks, else 1, so that a 256-row chunk keeps every thread busy).
template <int GG, int kRowsT>
__global__ void __launch_bounds__(kThreads)
em_assign_kernel(const float* __restrict__ rows, int64_t N, int d, int Nc,
                 const float* __restrict__ cb, void* __restrict__ codes_out, int code_bytes,
                 double* __restrict__ psum, int32_t* __restrict__ pcnt, double* __restrict__ psse,
                 int chunk_rows) {
  constexpr int kRows = kRowsT;
  constexpr int kSub = kThreads * kRows;          // rows assigned per pass
  constexpr int kTileE = kTileFloats / GG;        // entries staged per pass
  __shared__ float4 tile[kTileFloats / 4];
  __shared__ __align__(16) uint16_t code_s[kChunkRows];
  __shared__ float dist_s[kChunkRows];
  __shared__ double red[kThreads];
  const int G = d / GG;
  const int j = blockIdx.y;
  const int64_t chunk = blockIdx.x;
  const int64_t base = chunk * chunk_rows;
  const int rows_here = static_cast<int>(min(static_cast<int64_t>(chunk_rows), N - base));
  const float* sub_cb = cb + static_cast<int64_t>(j) * Nc * GG;

  for (int s0 = 0; s0 < rows_here; s0 += kSub) {
    float res[kRows][GG];
    Nearest best[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const int li = s0 + threadIdx.x + i * kThreads;
      nearest_init(best[i]);
#pragma unroll
      for (int q = 0; q < GG / kG; ++q) {
        float v[kG];
        if (li < rows_here) {
          load_row8(rows + (base + li) * d + j * GG + q * kG, v);
        } else {
#pragma unroll
          for (int k = 0; k < kG; ++k) v[k] = 0.0f;
        }
#pragma unroll
        for (int k = 0; k < kG; ++k) res[i][q * kG + k] = v[k];
      }
    }
    if constexpr (GG == kG) {
      // packed scan (the encoder's): two entries per fp32x2 instruction, each lane the scalar rule
      f32x2 res2[kRows][kG];
#pragma unroll
      for (int i = 0; i < kRows; ++i)
#pragma unroll
        for (int k = 0; k < kG; ++k) res2[i][k] = pack2(res[i][k], res[i][k]);
      for (int c0 = 0; c0 < Nc; c0 += kTileE) {
        const int n = min(kTileE, Nc - c0);
        __syncthreads();
        stage_pairs8(tile, sub_cb + static_cast<int64_t>(c0) * GG, n);
        __syncthreads();
        const int pairs = n >> 1;
#pragma unroll 2
        for (int p = 0; p < pairs; ++p) {
#pragma unroll
          for (int i = 0; i < kRows; ++i) {
            float d0, d1;
            unpack2(pair_dist8(res2[i], tile + 4 * p), d0, d1);
            nearest_take<false>(best[i], d0, c0 + 2 * p);
            nearest_take<false>(best[i], d1, c0 + 2 * p + 1);
          }
        }
        if (n & 1) {
#pragma unroll
          for (int i = 0; i < kRows; ++i) {
            float d0, d1;
            unpack2(pair_dist8(res2[i], tile + 4 * pairs), d0, d1);
            nearest_take<false>(best[i], d0, c0 + n - 1);
          }
        }
      }
    } else {
      for (int c0 = 0; c0 < Nc; c0 += kTileE) {
        const int n = min(kTileE, Nc - c0);
        __syncthreads();
        for (int e = threadIdx.x; e < n * (GG / 4); e += kThreads)
          tile[e] = __ldg(reinterpret_cast<const float4*>(sub_cb + static_cast<int64_t>(c0) * GG) + e);
        __syncthreads();
#pragma unroll 2
        for (int c = 0; c < n; ++c) {
#pragma unroll
          for (int i = 0; i < kRows; ++i) nearest_step_g<GG, false>(best[i], res[i], tile + c * (GG / 4), c0 + c);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
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

  // Per-entry sums of the assigned sub-vectors, in row order, 8 scalars at a time.
  for (int c = threadIdx.x; c < Nc; c += kThreads) {
    const int64_t at = (chunk * G + j) * Nc + c;
    int cnt = 0;
#pragma unroll 1
    for (int q = 0; q < GG / kG; ++q) {
      double acc[kG];
#pragma unroll
      for (int k = 0; k < kG; ++k) acc[k] = 0.0;
      cnt = 0;
      // the chunk's codes eight at a time (one 16-byte shared load), matches taken in row order
      for (int l0 = 0; l0 < rows_here; l0 += 8) {
        const uint4 w8 = *reinterpret_cast<const uint4*>(code_s + l0);
        const uint32_t w[4] = {w8.x, w8.y, w8.z, w8.w};
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) {
          const int li = l0 + k8;
          const uint32_t code = (w[k8 >> 1] >> (16 * (k8 & 1))) & 0xFFFFu;
          if (li >= rows_here || code != static_cast<uint32_t>(c)) continue;
          float v[kG];
          load_row8(rows + (base + li) * d + j * GG + q * kG, v);
#pragma unroll
          for (int k = 0; k < kG; ++k) acc[k] += static_cast<double>(v[k]);
          ++cnt;
        }
      }
#pragma unroll
      for (int k = 0; k < kG; ++k) psum[at * GG + q * kG + k] = acc[k];
    }
    pcnt[at] = cnt;
  }
}

template <int GG>
__global__ void __launch_bounds__(kThreads)
em_update_kernel(int64_t chunks, int G, int Nc, float* __restrict__ cb, const double* __restrict__ psum,
                 const int32_t* __restrict__ pcnt, const double* __restrict__ psse,
                 double* __restrict__ sse_out) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;   // j * Nc + c
  if (e < static_cast<int64_t>(G) * Nc) {
#pragma unroll 1
    for (int q = 0; q < GG / kG; ++q) {
      double acc[kG];
#pragma unroll
      for (int k = 0; k < kG; ++k) acc[k] = 0.0;
      int64_t cnt = 0;
      // four chunks' counts and sums loaded before any is used (the loads do not wait on one
      // another), then added in chunk order, skipping chunks where no row chose the entry
      for (int64_t ch0 = 0; ch0 < chunks; ch0 += 4) {
        int32_t m[4];
        double v[4][kG];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          m[u] = 0;
          if (ch0 + u < chunks) {
            const int64_t at = (ch0 + u) * G * Nc + e;
            m[u] = pcnt[at];
#pragma unroll
            for (int k = 0; k < kG; ++k) v[u][k] = psum[at * GG + q * kG + k];
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (m[u] == 0) continue;
          cnt += m[u];
#pragma unroll
          for (int k = 0; k < kG; ++k) acc[k] += v[u][k];
        }
      }
      if (cnt > 0) {
#pragma unroll
        for (int k = 0; k < kG; ++k)
          cb[e * GG + q * kG + k] = __double2float_rn(acc[k] / static_cast<double>(cnt));
      }
    }
  }
  if (sse_out && blockIdx.x == 0 && threadIdx.x == 0) {
    double s = 0.0;
    for (int64_t i = 0; i < chunks * G; ++i) s += psse[i];
    *sse_out = s;
  }
}

// Soft assignment (one step at temperature tau): responsibilities w = exp(-(d - d_min)/tau)/Z
// over a group's entries, with the encoder's exact fp32 distances. Phase 1 (row threads)
// streams the codebook once per row keeping the running minimum and the partition sum
// (rescaled when the minimum drops); phase 2 (entry threads) recomputes the same distances
// against the chunk's rows, staged in shared memory, and accumulates w x and w in fp64 in row
// order. Distances, minima and weights are fp32; sums are fp64.
__global__ void __launch_bounds__(kThreads)
em_soft_assign_kernel(const float* __restrict__ rows, int64_t N, int d, int Nc,
                      const float* __restrict__ cb, float tau, double* __restrict__ psum,
                      double* __restrict__ pw, double* __restrict__ psse) {
  __shared__ float4 tile[kTile * 2];
  __shared__ float4 xs[kSoftChunkRows * 2];
  __shared__ float dmin_s[kSoftChunkRows];
  __shared__ float zinv_s[kSoftChunkRows];
  __shared__ double red[kThreads];
  const int G = d / kG;
  const int j = blockIdx.y;
  const int64_t chunk = blockIdx.x;
  const int64_t base = chunk * kSoftChunkRows;
  const int rows_here = static_cast<int>(min(static_cast<int64_t>(kSoftChunkRows), N - base));
  const float* sub_cb = cb + static_cast<int64_t>(j) * Nc * kG;
  const float inv_tau = 1.0f / tau;

  // phase 1: one row per thread
  const int li = threadIdx.x;
  float x[kG];
  const bool valid = li < rows_here;
  if (valid) {
    load_row8(rows + (base + li) * d + j * kG, x);
    xs[2 * li] = make_float4(x[0], x[1], x[2], x[3]);
    xs[2 * li + 1] = make_float4(x[4], x[5], x[6], x[7]);
  } else {
#pragma unroll
    for (int k = 0; k < kG; ++k) x[k] = 0.0f;
  }
  float m = __int_as_float(0x7f800000), Z = 0.0f;
  for (int c0 = 0; c0 < Nc; c0 += kTile) {
    const int n = min(kTile, Nc - c0);
    __syncthreads();
    for (int e = threadIdx.x; e < 2 * n; e += kThreads)
      tile[e] = __ldg(reinterpret_cast<const float4*>(sub_cb + static_cast<int64_t>(c0) * kG) + e);
    __syncthreads();
    for (int c = 0; c < n; ++c) {
      const float4 lo = tile[2 * c], hi = tile[2 * c + 1];
      Nearest nb;
      nearest_init(nb);
      nearest_step<false>(nb, x, lo, hi, 0);
      const float dist = nb.best;
      if (dist < m) {
        Z = Z * expf((dist - m) * inv_tau) + 1.0f;
        m = dist;
      } else {
        Z += expf((m - dist) * inv_tau);
      }
    }
  }
  if (valid) {
    dmin_s[li] = m;
    zinv_s[li] = 1.0f / Z;
  }
  red[threadIdx.x] = valid ? static_cast<double>(m) : 0.0;
  __syncthreads();
  for (int w = kThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) psse[chunk * G + j] = red[0];

  // phase 2: one entry per thread, rows in order
  for (int c = threadIdx.x; c < Nc; c += kThreads) {
    float e_c[kG];
    load_row8(sub_cb + static_cast<int64_t>(c) * kG, e_c);
    const float4 lo = make_float4(e_c[0], e_c[1], e_c[2], e_c[3]);
    const float4 hi = make_float4(e_c[4], e_c[5], e_c[6], e_c[7]);
    double acc[kG];
#pragma unroll
    for (int k = 0; k < kG; ++k) acc[k] = 0.0;
    double wsum = 0.0;
    for (int r = 0; r < rows_here; ++r) {
      const float4 a = xs[2 * r], b = xs[2 * r + 1];
      const float xr[kG] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      Nearest nb;
      nearest_init(nb);
      nearest_step<false>(nb, xr, lo, hi, 0);
      const float w = expf((dmin_s[r] - nb.best) * inv_tau) * zinv_s[r];
      if (w == 0.0f) continue;
      const double wd = static_cast<double>(w);
      wsum += wd;
#pragma unroll
      for (int k = 0; k < kG; ++k) acc[k] = fma(wd, static_cast<double>(xr[k]), acc[k]);
    }
    const int64_t at = (chunk * G + j) * Nc + c;
#pragma unroll
    for (int k = 0; k < kG; ++k) psum[at * kG + k] = acc[k];
    pw[at] = wsum;
  }
}

__global__ void __launch_bounds__(kThreads)
em_soft_update_kernel(int64_t chunks, int G, int Nc, float* __restrict__ cb, const double* __restrict__ psum,
                      const double* __restrict__ pw, const double* __restrict__ psse,
                      double* __restrict__ sse_out) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;   // j * Nc + c
  if (e < static_cast<int64_t>(G) * Nc) {
    double acc[kG];
#pragma unroll
    for (int k = 0; k < kG; ++k) acc[k] = 0.0;
    double wsum = 0.0;
    for (int64_t ch = 0; ch < chunks; ++ch) {
      const int64_t at = ch * G * Nc + e;
      wsum += pw[at];
#pragma unroll
      for (int k = 0; k < kG; ++k) acc[k] += psum[at * kG + k];
    }
    if (wsum > 0.0) {
#pragma unroll
      for (int k = 0; k < kG; ++k) cb[e * kG + k] = __double2float_rn(acc[k] / wsum);
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
  if ((g != 8 && g != 16 && g != 32 && g != 64) || Nc > kMaxCodes) return COMMVQ_ERR_UNSUPPORTED;
  if ((N + kSoftChunkRows - 1) / kSoftChunkRows > INT32_MAX) return COMMVQ_ERR_UNSUPPORTED;
  return COMMVQ_OK;
}

extern "C" size_t commvq_em_workspace_bytes(const commvq_config* cfg, int64_t N) {
  if (em_check(cfg, N) != COMMVQ_OK) return 0;
  return em_layout(N, cfg->d / cfg->g, cfg->n_codes, cfg->g).total;
}

namespace {
template <int GG>
commvq_status launch_em_hard(const commvq_config* cfg, const float* rows, int64_t N, float* cb,
                             void* codes_out, double* sse_out, const EmLayout& L, unsigned char* ws,
                             cudaStream_t st) {
  const int G = cfg->d / GG, Nc = cfg->n_codes;
  double* psum = reinterpret_cast<double*>(ws + L.sums_off);
  int32_t* pcnt = reinterpret_cast<int32_t*>(ws + L.counts_off);
  double* psse = reinterpret_cast<double*>(ws + L.sse_off);
  const dim3 grid(static_cast<unsigned>(L.chunks), G);
  if (GG == kG && L.chunk_rows == kChunkRows)
    em_assign_kernel<GG, 2><<<grid, kThreads, 0, st>>>(rows, N, cfg->d, Nc, cb, codes_out, cfg->code_bytes, psum,
                                                        pcnt, psse, L.chunk_rows);
  else
    em_assign_kernel<GG, 1><<<grid, kThreads, 0, st>>>(rows, N, cfg->d, Nc, cb, codes_out, cfg->code_bytes, psum,
                                                        pcnt, psse, L.chunk_rows);
  const commvq_status rc = launch_status();
  if (rc != COMMVQ_OK) return rc;
  const unsigned g2 = static_cast<unsigned>((static_cast<int64_t>(G) * Nc + kThreads - 1) / kThreads);
  em_update_kernel<GG><<<g2, kThreads, 0, st>>>(L.chunks, G, Nc, cb, psum, pcnt, psse, sse_out);
  return launch_status();
}
}  // namespace

extern "C" commvq_status commvq_em_step(const commvq_config* cfg, const float* rows, int64_t N,
                                        float* codebook_round, void* codes_out, double* sse_out,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("commvq_em_step");
  const commvq_status cs = em_check(cfg, N);
  if (cs != COMMVQ_OK) return cs;
  if (!rows || !codebook_round || !workspace) return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(rows, 16) || !aligned(codebook_round, 16) || !aligned(sse_out, 8) ||
      !aligned(workspace, 256) || !aligned(codes_out, cfg->code_bytes))
    return COMMVQ_ERR_INVALID_ARG;
  const EmLayout L = em_layout(N, cfg->d / cfg->g, cfg->n_codes, cfg->g);
  if (workspace_bytes < L.total) return COMMVQ_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (cfg->g) {
    case 8: return launch_em_hard<8>(cfg, rows, N, codebook_round, codes_out, sse_out, L, ws, st);
    case 16: return launch_em_hard<16>(cfg, rows, N, codebook_round, codes_out, sse_out, L, ws, st);
    case 32: return launch_em_hard<32>(cfg, rows, N, codebook_round, codes_out, sse_out, L, ws, st);
    default: return launch_em_hard<64>(cfg, rows, N, codebook_round, codes_out, sse_out, L, ws, st);
  }
}

extern "C" commvq_status commvq_em_step_soft(const commvq_config* cfg, const float* rows, int64_t N,
                                             float* codebook_round, float tau, double* sse_out,
                                             void* workspace, size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("commvq_em_step_soft");
  const commvq_status cs = em_check(cfg, N);
  if (cs != COMMVQ_OK) return cs;
  if (!(tau > 0.0f) || !isfinite(tau)) return COMMVQ_ERR_INVALID_ARG;
  if (cfg->g != kG) return COMMVQ_ERR_UNSUPPORTED;
  if (!rows || !codebook_round || !workspace) return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(rows, 16) || !aligned(codebook_round, 16) || !aligned(sse_out, 8) || !aligned(workspace, 256))
    return COMMVQ_ERR_INVALID_ARG;
  const int G = cfg->d / kG, Nc = cfg->n_codes;
  const EmLayout L = em_layout(N, G, Nc, kG);
  if (workspace_bytes < L.total) return COMMVQ_ERR_WORKSPACE;
  const int64_t chunks = L.soft_chunks;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  double* psum = reinterpret_cast<double*>(ws + L.sums_off);
  double* pw = reinterpret_cast<double*>(ws + L.counts_off);
  double* psse = reinterpret_cast<double*>(ws + L.sse_off);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  em_soft_assign_kernel<<<dim3(static_cast<unsigned>(chunks), G), kThreads, 0, st>>>(
      rows, N, cfg->d, Nc, codebook_round, tau, psum, pw, psse);
  commvq_status rc = launch_status();
  if (rc != COMMVQ_OK) return rc;
  const unsigned g2 = static_cast<unsigned>((static_cast<int64_t>(G) * Nc + kThreads - 1) / kThreads);
  em_soft_update_kernel<<<g2, kThreads, 0, st>>>(chunks, G, Nc, codebook_round, psum, pw, psse, sse_out);
  return launch_status();
}
