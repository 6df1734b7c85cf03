// Decode attention on the codes for any group size the encoder takes (g = 8, 16, 32, 64),
// up to 32 residual rounds and up to 65536 entries: the pages' own setting (g = 64, Nc' = 64,
// R = 21 or 11; review, "Assumptions & free parameters") as well as the library's g = 8 layout.
//
// It computes exactly what commvq_attend_decode defines, in fp32 throughout. One warp takes one
// (position, KV head) at a time; lane l owns dims 4l..4l+3 (RoPE pairs 2l, 2l+1), which lie in
// group 4l / g at offset 4l % g. A decoded row is the fp32 sum over rounds of the selected
// entries, read straight from the fp32 codebooks through L1/L2: with 21 rounds of 64-scalar
// entries the codebooks (2 x 688 KB) do not fit in shared memory. Keys are rotated in fp32
// with phasors from fp64 angles (per-chunk x per-offset tables). Scores are warp-reduced dot
// products; an online softmax per query head accumulates p v in fp32. Every warp writes a
// partial (m, l, o) per head for the split-T combine.
//
// This is bound by L2 and latency, not HBM: at R = 21 a (position, KV head) reads ~21 KB of
// codebook entries against 42 code bytes. The decode-and-rotate kernels are the fast form for
// g = 8, R <= 2.
#include <math.h>

#include "attend.cuh"

namespace commvq {
namespace {

constexpr int kGenThreads = 256;   // 8 warps
constexpr int kGenWarps = 8;
constexpr int kGenChunk = 128;     // positions per coarse phasor
constexpr int kGenMaxG = 16;       // query heads per KV head

// blockIdx.y = 0: per-offset phasors e^{i o theta_p}, o < 128; 1: per-chunk phasors
// e^{i 128 h theta_p}, both from fp64 angles, in the packed layout of put_phasor.
__global__ void generic_prep_kernel(float4* rowph, float4* coarse, int n_hi, double rope_base, int* error_word) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e == 0 && blockIdx.y == 0) error_word[0] = error_word[1] = 0;
  const int p = e % (kD / 2), row = e / (kD / 2);
  const double th = pow(rope_base, -2.0 * p / kD);
  double sn, cs;
  if (blockIdx.y == 0) {
    if (row >= kGenChunk) return;
    sincos(static_cast<double>(row) * th, &sn, &cs);
    put_phasor(rowph + row * (kD / 4), p, cs, sn);
  } else {
    if (row >= n_hi) return;
    sincos(static_cast<double>(row) * kGenChunk * th, &sn, &cs);
    put_phasor(coarse + static_cast<int64_t>(row) * (kD / 4), p, cs, sn);
  }
}

struct GenericArgs {
  const void* k_codes;
  const void* v_codes;
  const int64_t* seq_offsets;
  const float* k_codebook;
  const float* v_codebook;
  const float4* rowph;
  const float4* coarse;
  Partial* partials;
  int* error_word;
  int64_t max_T;
  int q_heads, kv_heads, g, R, n_codes, code_bytes;
};

__device__ __forceinline__ int load_code(const void* codes, int64_t at, int code_bytes) {
  return code_bytes == 1 ? static_cast<int>(static_cast<const uint8_t*>(codes)[at])
                         : static_cast<int>(static_cast<const uint16_t*>(codes)[at]);
}

// The fp32 sum over rounds of the lane's 4 dims of record rec (round order 0..R-1).
__device__ __forceinline__ float4 decode4(const GenericArgs& a, const void* codes, const float* cb,
                                          int64_t rec, int j, int off, int G, int& err) {
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r = 0; r < a.R; ++r) {
    int c = load_code(codes, (rec * a.R + r) * G + j, a.code_bytes);
    if (c >= a.n_codes) {
      c = a.n_codes - 1;
      err = 1;
    }
    const float4 v = __ldg(reinterpret_cast<const float4*>(
        cb + ((static_cast<int64_t>(r) * G + j) * a.n_codes + c) * a.g + off));
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  return acc;
}

template <typename QT>
__device__ __forceinline__ float qget(const QT* q, int i);
template <>
__device__ __forceinline__ float qget<float>(const float* q, int i) { return q[i]; }
template <>
__device__ __forceinline__ float qget<__half>(const __half* q, int i) { return __half2float(q[i]); }
template <>
__device__ __forceinline__ float qget<__nv_bfloat16>(const __nv_bfloat16* q, int i) {
  return __bfloat162float(q[i]);
}

// MAXG: a bound on the query heads per KV head (4 or 16); the per-head state is sized by it.
template <typename QT, int MAXG>
__global__ void __launch_bounds__(kGenThreads) attend_generic_kernel(GenericArgs a, const QT* __restrict__ q) {
  const int KV = a.kv_heads, Gq = a.q_heads / KV, G = kD / a.g;
  const int wpk = kGenWarps / KV;   // warps per KV head (KV divides 8)
  const int s = blockIdx.x, b = blockIdx.y, S = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kv = warp / wpk, sub = warp % wpk;
  const int j = (4 * lane) / a.g, off = (4 * lane) % a.g;

  int64_t row0;
  const int64_t Tb = sequence_rows(a.seq_offsets, b, a.max_T, running_error(a.error_word), row0);
  int64_t per = (Tb + S - 1) / S;
  const int64_t t_begin = min(Tb, static_cast<int64_t>(s) * per);
  const int64_t t_end = min(Tb, t_begin + per);

  float qv[MAXG][4];
#pragma unroll
  for (int h = 0; h < MAXG; ++h) {
    if (h < Gq) {
      const QT* qh = q + (static_cast<int64_t>(b) * a.q_heads + kv * Gq + h) * kD + 4 * lane;
      qv[h][0] = qget(qh, 0);
      qv[h][1] = qget(qh, 1);
      qv[h][2] = qget(qh, 2);
      qv[h][3] = qget(qh, 3);
    } else {
      qv[h][0] = qv[h][1] = qv[h][2] = qv[h][3] = 0.0f;
    }
  }
  const float scale = 1.4426950408889634f / sqrtf(static_cast<float>(kD));   // exp2 domain
  float O[MAXG][4], m[MAXG], l[MAXG];
#pragma unroll
  for (int h = 0; h < MAXG; ++h) {
    O[h][0] = O[h][1] = O[h][2] = O[h][3] = 0.0f;
    m[h] = -INFINITY;
    l[h] = 0.0f;
  }
  int err = 0;
  for (int64_t t = t_begin + sub; t < t_end; t += wpk) {
    const int64_t rec = (row0 + t) * KV + kv;
    float4 k = decode4(a, a.k_codes, a.k_codebook, rec, j, off, G, err);
    // rotate pairs 2 lane, 2 lane + 1 to position t
    f32x2 pc, ps, hc, hs;
    load_phasor(__ldg(a.rowph + (t % kGenChunk) * (kD / 4) + lane), pc, ps);
    load_phasor(__ldg(a.coarse + (t / kGenChunk) * (kD / 4) + lane), hc, hs);
    cmul2(pc, ps, hc, hs);
    float c0, c1, s0, s1;
    unpack2(pc, c0, c1);
    unpack2(ps, s0, s1);
    const float kx0 = k.x * c0 - k.y * s0, ky0 = k.x * s0 + k.y * c0;
    const float kx1 = k.z * c1 - k.w * s1, ky1 = k.z * s1 + k.w * c1;
    const float4 v = decode4(a, a.v_codes, a.v_codebook, rec, j, off, G, err);
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
      if (h >= Gq) break;
      float part = qv[h][0] * kx0 + qv[h][1] * ky0 + qv[h][2] * kx1 + qv[h][3] * ky1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      const float sc = part * scale;
      const float mn = fmaxf(m[h], sc);
      const float al = exp2f(m[h] - mn), p = exp2f(sc - mn);
      m[h] = mn;
      l[h] = l[h] * al + p;
      O[h][0] = O[h][0] * al + p * v.x;
      O[h][1] = O[h][1] * al + p * v.y;
      O[h][2] = O[h][2] * al + p * v.z;
      O[h][3] = O[h][3] * al + p * v.w;
    }
  }
  const int SE = S * wpk;
#pragma unroll
  for (int h = 0; h < MAXG; ++h) {
    if (h >= Gq) break;
    Partial* p = a.partials + (static_cast<int64_t>(b) * a.q_heads + kv * Gq + h) * SE + s * wpk + sub;
    reinterpret_cast<float4*>(p->o)[lane] = make_float4(O[h][0], O[h][1], O[h][2], O[h][3]);
    if (lane == 0) {
      p->m = m[h];
      p->l = l[h];
    }
  }
  err = __syncthreads_or(err);
  if (err && threadIdx.x == 0) atomicOr(running_error(a.error_word), kErrCodeRange);
}

}  // namespace

bool generic_supported(const commvq_config* cfg) {
  const int KV = cfg->kv_heads, g = cfg->g;
  return cfg->d == kD && (g == 8 || g == 16 || g == 32 || g == 64) && cfg->R >= 1 && cfg->R <= 32 &&
         (KV == 1 || KV == 2 || KV == 4 || KV == 8) && cfg->q_heads / KV <= kGenMaxG;
}

int generic_warps_per_kv(int kv_heads) { return kGenWarps / kv_heads; }

size_t generic_tables_bytes(int64_t max_T) {
  const int64_t n_hi = (max_T + kGenChunk - 1) / kGenChunk;
  return static_cast<size_t>(kGenChunk + (n_hi > 0 ? n_hi : 1)) * (kD / 4) * sizeof(float4);
}

commvq_status launch_attend_generic(const AttendArgs& a, const commvq_config* cfg, const void* q,
                                    commvq_dtype qt, int S, void* tables, cudaStream_t st) {
  GenericArgs g{};
  g.k_codes = a.k_codes;
  g.v_codes = a.v_codes;
  g.seq_offsets = a.seq_offsets;
  g.k_codebook = a.k_codebook;
  g.v_codebook = a.v_codebook;
  float4* rowph = static_cast<float4*>(tables);
  float4* coarse = rowph + kGenChunk * (kD / 4);
  g.rowph = rowph;
  g.coarse = coarse;
  g.partials = a.partials;
  g.error_word = a.error_word;
  g.max_T = a.max_T;
  g.q_heads = cfg->q_heads;
  g.kv_heads = cfg->kv_heads;
  g.g = cfg->g;
  g.R = cfg->R;
  g.n_codes = cfg->n_codes;
  g.code_bytes = cfg->code_bytes;
  const int n_hi = static_cast<int>((a.max_T + kGenChunk - 1) / kGenChunk);
  const int items = (kGenChunk > n_hi ? kGenChunk : n_hi) * (kD / 2);
  generic_prep_kernel<<<dim3((items + 255) / 256, 2), 256, 0, st>>>(rowph, coarse, n_hi, cfg->rope_base,
                                                                  a.error_word);
  if (launch_status() != COMMVQ_OK) return COMMVQ_ERR_CUDA;
  if (a.main_start && record_event(a.main_start, st) != cudaSuccess) return COMMVQ_ERR_CUDA;
  const dim3 grid(S, a.B);
  const bool small = cfg->q_heads / cfg->kv_heads <= 4;
#define COMMVQ_GENERIC(QTYPE)                                                                        \
  if (small)                                                                                         \
    attend_generic_kernel<QTYPE, 4><<<grid, kGenThreads, 0, st>>>(g, static_cast<const QTYPE*>(q));   \
  else                                                                                               \
    attend_generic_kernel<QTYPE, kGenMaxG><<<grid, kGenThreads, 0, st>>>(g, static_cast<const QTYPE*>(q));
  if (qt == COMMVQ_F32) {
    COMMVQ_GENERIC(float)
  } else if (qt == COMMVQ_F16) {
    COMMVQ_GENERIC(__half)
  } else {
    COMMVQ_GENERIC(__nv_bfloat16)
  }
#undef COMMVQ_GENERIC
  if (launch_status() != COMMVQ_OK) return COMMVQ_ERR_CUDA;
  if (a.main_stop && record_event(a.main_stop, st) != cudaSuccess) return COMMVQ_ERR_CUDA;
  return COMMVQ_OK;
}

}  // namespace commvq
