// Decode attention on CommVQ codes, table form: one CTA per (sequence b, query head h,
// split s of the sequence's positions).
//
//  1. Query x codebook table (review, "What carries the argument": the query-dependent and
//     codebook-dependent factors are formed once and reused for all cached positions).
//     For pair p = 4j + i of group j and entry c of round r with stored pair (a, b):
//        tab[r][j][c][i] = conj(q_p) (a + ib) = (q0 a + q1 b) + i (q0 b - q1 a),
//     with q pre-scaled by log2(e)/sqrt(d) so scores come out in the exp2 domain. The table
//     lives in shared memory as fp16 (4 complex = 16 B per (r, j, c)), laid out
//     [r][j/8][c][j%8] so that the 8 lanes of one shared-memory phase, which hold groups
//     j = 0..7 (or 8..15) of one token, always hit 8 different 16-byte bank groups.
//  2. Scores: lane j of a half-warp owns group j of one token; it gathers R table entries,
//     sums them, and rotates by e^{i t theta_p} (the RoPE rotation moved past the codebook
//     by commutation, Property 1). A 4-step shuffle sums the 16 groups.
//  3. Online softmax over chunks of kChunk positions: chunk scores go to shared memory, the
//     running max is updated once per chunk, and the value histograms are rescaled when it
//     grows.
//  4. Values (review, "If this is right": softmax weights multiply the value codes before
//     the codebook multiply): H[r][c][j] += p_t for c = vcode[t][r][j] (shared atomics).
//  5. End of split: o[8j + k] = sum_r sum_c H[r][c][j] vcb[r][j][c][k]; the unnormalised o,
//     the running max m and the sum l go to the workspace. A second kernel merges splits.
#include <math.h>

#include "attend.cuh"

namespace commvq {
namespace {

constexpr int kChunk = 256;  // positions per online-softmax step (8 warps x 32)

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename QT>
__device__ __forceinline__ float load_q(const QT* q, int i);
template <>
__device__ __forceinline__ float load_q<float>(const float* q, int i) { return q[i]; }
template <>
__device__ __forceinline__ float load_q<__half>(const __half* q, int i) { return __half2float(q[i]); }
template <>
__device__ __forceinline__ float load_q<__nv_bfloat16>(const __nv_bfloat16* q, int i) {
  return __bfloat162float(q[i]);
}

template <int R, bool kCheck, typename QT>
__global__ void __launch_bounds__(kThreads, 1)
attend_table_kernel(AttendArgs a, const QT* __restrict__ q) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int Nc = a.n_codes;
  uint4* tab = reinterpret_cast<uint4*>(smem);                                   // R*2*Nc*8
  float* hist = reinterpret_cast<float*>(tab + static_cast<size_t>(R) * 2 * Nc * 8);  // R*Nc*16
  float* sc = hist + static_cast<size_t>(R) * Nc * kGroups;                      // kChunk
  float* qs = sc + kChunk;                                                       // kD
  float* red = qs + kD;                                                          // 2 * 8
  uint8_t* kbuf = reinterpret_cast<uint8_t*>(red + 16);        // [2][kChunk][R][16] key codes
  uint8_t* vbuf = kbuf + 2 * kChunk * R * kGroups;             // [2][kChunk][R][16] value codes

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int S = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kvh = h / (a.q_heads / a.kv_heads);
  int64_t row0;
  const int64_t Tb = sequence_rows(a.seq_offsets, b, a.max_T, running_error(a.error_word), row0);
  const int64_t per = (Tb + S - 1) / S;
  const int64_t t_begin = min(Tb, static_cast<int64_t>(s) * per);
  const int64_t t_end = min(Tb, t_begin + per);
  Partial* part = a.partials + (static_cast<int64_t>(b) * a.q_heads + h) * S + s;

  if (t_begin >= t_end) {  // empty split: neutral partial
    if (tid < kD) part->o[tid] = 0.0f;
    if (tid == 0) {
      part->m = -INFINITY;
      part->l = 0.0f;
    }
    return;
  }

  // ---- 1. scaled query and table --------------------------------------------------------
  const float qscale = 1.4426950408889634f / sqrtf(static_cast<float>(kD));
  const QT* qh = q + (static_cast<int64_t>(b) * a.q_heads + h) * kD;
  if (tid < kD) qs[tid] = load_q(qh, tid) * qscale;
  for (int e = tid; e < R * Nc * kGroups; e += kThreads) hist[e] = 0.0f;
  __syncthreads();
  for (int e = tid; e < R * kGroups * Nc; e += kThreads) {
    const int c = e % Nc;
    const int rj = e / Nc;            // r * 16 + j
    const int j = rj % kGroups, r = rj / kGroups;
    float w[kG];
    load_row8(a.k_codebook + static_cast<int64_t>(e) * kG, w);   // [r][j][c][8] is e*8
    uint4 packed;
    __half2* hp = reinterpret_cast<__half2*>(&packed);
#pragma unroll
    for (int i = 0; i < kPairs; ++i) {
      const float q0 = qs[j * kG + 2 * i], q1 = qs[j * kG + 2 * i + 1];
      const float x = w[2 * i], y = w[2 * i + 1];
      const float u = fmaf(q0, x, q1 * y);
      const float v = fmaf(q0, y, -q1 * x);
      hp[i] = __floats2half2_rn(u, v);
    }
    tab[((static_cast<size_t>(r) * 2 + (j >> 3)) * Nc + c) * 8 + (j & 7)] = packed;
  }

  // ---- per-lane constants: group j, token slot, RoPE frequencies of the lane's 4 pairs ----
  const int j = lane & 15, slot = lane >> 4;
  double theta[kPairs];
#pragma unroll
  for (int i = 0; i < kPairs; ++i)
    theta[i] = pow(a.rope_base, -2.0 * static_cast<double>(j * kPairs + i) / kD);
  const int64_t code_row = static_cast<int64_t>(a.kv_heads) * R * kGroups;  // bytes per position
  const uint8_t* kc = a.k_codes + row0 * code_row + static_cast<int64_t>(kvh) * R * kGroups;
  const uint8_t* vc = a.v_codes + row0 * code_row + static_cast<int64_t>(kvh) * R * kGroups;
  int err = 0;

  // Prefetch of one chunk's key and value codes (R 16-byte pieces per position and tensor).
  auto issue = [&](int64_t c0, int stage) {
    const int n = static_cast<int>(min(static_cast<int64_t>(kChunk), t_end - c0));
    const int pieces = n * R;
    for (int p = tid; p < 2 * pieces; p += kThreads) {
      const int tensor = p >= pieces;
      const int qp = p - tensor * pieces;
      const int t = qp / R, r = qp - (qp / R) * R;
      const uint8_t* src = (tensor ? vc : kc) + (c0 + t) * code_row + r * kGroups;
      uint8_t* dst = (tensor ? vbuf : kbuf) + ((stage * kChunk + t) * R + r) * kGroups;
      cp_async16(dst, src);
    }
    cp_async_commit();
  };

  float m_run = -INFINITY;   // running max (exp2 domain)
  float l_run = 0.0f;        // this thread's share of the running sum
  issue(t_begin, 0);
  int stage = 0;

  for (int64_t c0 = t_begin; c0 < t_end; c0 += kChunk, stage ^= 1) {
    const int n = static_cast<int>(min(static_cast<int64_t>(kChunk), t_end - c0));
    if (c0 + kChunk < t_end)
      issue(c0 + kChunk, stage ^ 1);
    else
      cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint8_t* kchunk = kbuf + stage * kChunk * R * kGroups;
    const uint8_t* vchunk = vbuf + stage * kChunk * R * kGroups;

    // ---- 2. scores of this chunk ----------------------------------------------------------
#pragma unroll 2
    for (int step = 0; step < 16; ++step) {
      const int tl = warp * 32 + step * 2 + slot;
      float part_s = 0.0f;
      if (tl < n) {
        const int64_t t = c0 + tl;
        const uint8_t* cp = kchunk + tl * R * kGroups + j;
        float U[kPairs] = {0.f, 0.f, 0.f, 0.f}, W[kPairs] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < R; ++r) {
          int code = cp[r * kGroups];
          if (kCheck && code >= Nc) {
            err = 1;
            code = Nc - 1;
          }
          const uint4 e = tab[((static_cast<size_t>(r) * 2 + (j >> 3)) * Nc + code) * 8 + (j & 7)];
          const __half2* hp = reinterpret_cast<const __half2*>(&e);
#pragma unroll
          for (int i = 0; i < kPairs; ++i) {
            const float2 f = __half22float2(hp[i]);
            U[i] += f.x;
            W[i] += f.y;
          }
        }
#pragma unroll
        for (int i = 0; i < kPairs; ++i) {
          const double ang = static_cast<double>(t) * theta[i];
          const double k = rint(ang * 0.15915494309189535);
          const float red_ang = static_cast<float>(fma(-k, 6.283185307179586, ang));
          float sn, cs;
          __sincosf(red_ang, &sn, &cs);
          part_s = fmaf(U[i], cs, part_s);
          part_s = fmaf(-W[i], sn, part_s);
        }
      }
      part_s += __shfl_xor_sync(0xffffffffu, part_s, 8);
      part_s += __shfl_xor_sync(0xffffffffu, part_s, 4);
      part_s += __shfl_xor_sync(0xffffffffu, part_s, 2);
      part_s += __shfl_xor_sync(0xffffffffu, part_s, 1);
      if (j == 0 && tl < n) sc[tl] = part_s;
    }
    __syncthreads();

    // ---- 3. online softmax: chunk max, rescale ----------------------------------------------
    float v = tid < n ? sc[tid] : -INFINITY;
    v = warp_max(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float cmax = red[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) cmax = fmaxf(cmax, red[w]);
    const float m_new = fmaxf(m_run, cmax);
    if (m_new > m_run) {
      const float alpha = exp2f(m_run - m_new);   // 0 on the first chunk
      l_run *= alpha;
      if (m_run != -INFINITY)
        for (int e = tid; e < R * Nc * kGroups; e += kThreads) hist[e] *= alpha;
      m_run = m_new;
    }
    if (tid < n) {
      const float p = exp2f(sc[tid] - m_run);
      sc[tid] = p;
      l_run += p;
    }
    __syncthreads();

    // ---- 4. value histograms ----------------------------------------------------------------
#pragma unroll 2
    for (int step = 0; step < 16; ++step) {
      const int tl = warp * 32 + step * 2 + slot;
      if (tl < n) {
        const float p = sc[tl];
        const uint8_t* cp = vchunk + tl * R * kGroups + j;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          int code = cp[r * kGroups];
          if (kCheck && code >= Nc) {
            err = 1;
            code = Nc - 1;
          }
          atomicAdd(&hist[(r * Nc + code) * kGroups + j], p);
        }
      }
    }
    __syncthreads();
  }

  // ---- 5. histogram x value-codebook contraction, partial result -----------------------------
  float l = warp_sum(l_run);
  if (lane == 0) red[8 + warp] = l;
  const int dim = tid & (kD - 1), half = tid >> 7;
  const int gj = dim >> 3, k = dim & 7;
  float acc = 0.0f;
  for (int idx = half; idx < R * Nc; idx += 2) {
    const int r = idx / Nc, c = idx - r * Nc;
    const float hv = hist[idx * kGroups + gj];
    acc = fmaf(hv, __ldg(a.v_codebook + ((static_cast<int64_t>(r) * kGroups + gj) * Nc + c) * kG + k), acc);
  }
  __syncthreads();
  if (half == 1) sc[dim] = acc;
  __syncthreads();
  if (half == 0) part->o[dim] = acc + sc[dim];
  if (tid == 0) {
    float lt = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) lt += red[8 + w];
    part->m = m_run;
    part->l = lt;
  }
  if (kCheck) {
    err = __syncthreads_or(err);
    if (err && tid == 0) atomicOr(running_error(a.error_word), kErrCodeRange);
  }
}

template <int R, bool kCheck>
commvq_status launch_table_r(const AttendArgs& a, const void* q, commvq_dtype qt, int splits,
                             size_t smem, cudaStream_t st) {
  dim3 grid(splits, a.q_heads, a.B);
  switch (qt) {
    case COMMVQ_F32: {
      auto k = attend_table_kernel<R, kCheck, float>;
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return COMMVQ_ERR_CUDA;
      k<<<grid, kThreads, smem, st>>>(a, static_cast<const float*>(q));
      break;
    }
    case COMMVQ_F16: {
      auto k = attend_table_kernel<R, kCheck, __half>;
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return COMMVQ_ERR_CUDA;
      k<<<grid, kThreads, smem, st>>>(a, static_cast<const __half*>(q));
      break;
    }
    case COMMVQ_BF16: {
      auto k = attend_table_kernel<R, kCheck, __nv_bfloat16>;
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return COMMVQ_ERR_CUDA;
      k<<<grid, kThreads, smem, st>>>(a, static_cast<const __nv_bfloat16*>(q));
      break;
    }
    default:
      return COMMVQ_ERR_UNSUPPORTED;
  }
  return launch_status();
}

template <int R>
commvq_status launch_table_c(const AttendArgs& a, const void* q, commvq_dtype qt, int splits,
                             size_t smem, cudaStream_t st) {
  if (a.n_codes < 256) return launch_table_r<R, true>(a, q, qt, splits, smem, st);
  return launch_table_r<R, false>(a, q, qt, splits, smem, st);
}

}  // namespace

size_t table_smem_bytes(int R, int n_codes) {
  return static_cast<size_t>(R) * n_codes * (2 * 8 * 16 + kGroups * 4) +
         (kChunk + kD + 16) * sizeof(float) + static_cast<size_t>(4) * kChunk * R * kGroups;
}

commvq_status launch_attend_table(const AttendArgs& a, const void* q, commvq_dtype qt, int splits,
                                  cudaStream_t st) {
  const size_t smem = table_smem_bytes(a.R, a.n_codes);
  switch (a.R) {
    case 1: return launch_table_c<1>(a, q, qt, splits, smem, st);
    case 2: return launch_table_c<2>(a, q, qt, splits, smem, st);
    case 3: return launch_table_c<3>(a, q, qt, splits, smem, st);
    case 4: return launch_table_c<4>(a, q, qt, splits, smem, st);
    default: return COMMVQ_ERR_UNSUPPORTED;
  }
}

}  // namespace commvq
