// The comparator behind the CommVQ review's latency claim ("What carries the argument" and
// Table 5: decode latency against a naive implementation of the same quantization). It
// decompresses every cached key and value from its codes into dense 16-bit rows, with each key
// rotated by RoPE at its position, then runs ordinary dense flash-decoding over those rows.
// Both steps are library calls of their own, so the fused path can be timed against them on
// the same inputs.
//
// commvq_decompress: persistent CTAs, one side (keys or values) each. The side's codebook is
//   an fp16 image in shared memory. Work items are 128-position chunks of one sequence. A
//   thread decodes one (position, KV head, group) at a time: it sums the R gathered entries,
//   rotates key pairs in fp32 and writes 8 outputs (16 bytes), so a warp writes 512
//   contiguous bytes. Key phasors are the product of a per-chunk phasor e^{i 128 h theta} and
//   a per-offset phasor e^{i o theta}; both come from fp64 angles.
// commvq_dense_decode: flash-decoding with mma.sync. A CTA takes one split of one sequence
//   and streams K and V stages (64 KB each, three in flight) into shared memory with 16-byte
//   asynchronous copies. Rows are XOR-swizzled so ldmatrix reads are conflict-free. Each warp
//   owns one KV head and 16 positions per stage: S = Q K^T with the group's query heads as
//   the mma rows, an online softmax, then O += P V with P taken straight from the S
//   accumulators. Every warp writes its own partial (m, l, o), and the split-T combine of the
//   fused path merges them.
#include <math.h>

#include <algorithm>

#include "attend.cuh"

namespace commvq {
namespace {

constexpr size_t kHeader = 256;   // device error word + padding
constexpr int kDecThreads = 512;
constexpr int kChunk = 128;       // positions per decompress work item

struct DecompArgs {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const int64_t* seq_offsets;
  const float* k_codebook;
  const float* v_codebook;
  void* k_out;
  void* v_out;
  uint4* k_img;
  uint4* v_img;
  float4* rowph;    // [kChunk offsets][32] packed phasors e^{i o theta}
  float4* coarse;   // [n_hi][32] packed phasors e^{i 128 h theta}
  int* error_word;
  int64_t max_T;
  double rope_base;
  int B;
  int kv_heads;
  int R;
  int n_codes;
  int n_hi;
};

// fp16 image slot of entry (round r, group j, code c): eight consecutive groups of one round
// fall in eight different 16-byte bank groups, and a half-warp reads groups 0..15.
__device__ __forceinline__ int dslot(int r, int j, int c, int Nc) {
  return ((r * 2 + (j >> 3)) * Nc + c) * 8 + ((j + 4 * r) & 7);
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// blockIdx.y = 0 / 1: key / value image; 2: offset phasors; 3: chunk phasors.
__global__ void decompress_prep_kernel(DecompArgs a) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e == 0 && blockIdx.y == 0) *a.error_word = 0;
  if (blockIdx.y <= 1) {
    const int Nc = a.n_codes;
    if (e >= a.R * kGroups * Nc) return;
    const int c = e % Nc, rj = e / Nc, j = rj % kGroups, r = rj / kGroups;
    const float* cb = blockIdx.y ? a.v_codebook : a.k_codebook;
    float w[kG];
    load_row8(cb + (static_cast<int64_t>(r * kGroups + j) * Nc + c) * kG, w);
    uint4 o;
    o.x = h2u(__floats2half2_rn(w[0], w[1]));
    o.y = h2u(__floats2half2_rn(w[2], w[3]));
    o.z = h2u(__floats2half2_rn(w[4], w[5]));
    o.w = h2u(__floats2half2_rn(w[6], w[7]));
    (blockIdx.y ? a.v_img : a.k_img)[dslot(r, j, c, Nc)] = o;
    return;
  }
  const int p = e % (kD / 2), row = e / (kD / 2);
  const double th = pow(a.rope_base, -2.0 * p / kD);
  double sn, cs;
  if (blockIdx.y == 2) {
    if (row >= kChunk) return;
    sincos(static_cast<double>(row) * th, &sn, &cs);
    put_phasor(a.rowph + row * (kD / 4), p, cs, sn);
  } else {
    if (row >= a.n_hi) return;
    sincos(static_cast<double>(row) * kChunk * th, &sn, &cs);
    put_phasor(a.coarse + static_cast<int64_t>(row) * (kD / 4), p, cs, sn);
  }
}

template <typename OT>
__device__ __forceinline__ uint32_t pack_out(float x, float y);
template <>
__device__ __forceinline__ uint32_t pack_out<__half>(float x, float y) {
  return h2u(__floats2half2_rn(x, y));
}
template <>
__device__ __forceinline__ uint32_t pack_out<__nv_bfloat16>(float x, float y) {
  __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Rotate stored pairs (a0, b0), (a1, b1) (half2 words w0, w1) by packed phasors (c, s) in fp32
// and pack the results (x0, y0), (x1, y1) to the output type.
template <typename OT>
__device__ __forceinline__ void rotate_out(uint32_t w0, uint32_t w1, f32x2 c, f32x2 s, uint32_t& o0,
                                           uint32_t& o1) {
  const float2 f0 = __half22float2(u2h(w0));
  const float2 f1 = __half22float2(u2h(w1));
  const f32x2 av = pack2(f0.x, f1.x), bv = pack2(f0.y, f1.y);
  const f32x2 x = sub2(mul2(av, c), mul2(bv, s));
  const f32x2 y = fma2(av, s, mul2(bv, c));
  float x0, x1, y0, y1;
  unpack2(x, x0, x1);
  unpack2(y, y0, y1);
  o0 = pack_out<OT>(x0, y0);
  o1 = pack_out<OT>(x1, y1);
}

template <typename OT>
__device__ __forceinline__ uint32_t convert_out(uint32_t w) {
  const float2 f = __half22float2(u2h(w));
  return pack_out<OT>(f.x, f.y);
}
template <>
__device__ __forceinline__ uint32_t convert_out<__half>(uint32_t w) {
  return w;
}

// Chunk codes (128 positions x KV heads x R x 16 bytes, contiguous in HBM) into shared memory.
template <int R>
__device__ __forceinline__ void issue_chunk(uint8_t* dst, const uint8_t* codes, int64_t rec0, int rows, int KV) {
  const int pieces = rows * KV * R;
  const uint8_t* src = codes + rec0 * (R * kGroups);
  for (int p = threadIdx.x; p < pieces; p += kDecThreads) cp_async16(dst + p * 16, src + p * 16);
}

// One CTA per SM; it decodes its share of the chunks for the keys, then for the values. Thread
// t keeps KV head (t/16) % KV and group j = t % 16 throughout, and takes every
// (kDecThreads / (16 KV))-th row of a chunk, so its key phasors advance by a fixed step.
template <int R, int KV, typename OT>
__global__ void __launch_bounds__(kDecThreads, 1) decompress_kernel(DecompArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int kRowStep = kDecThreads / (kGroups * KV);     // rows between a thread's items
  constexpr int kChunkBytes = kChunk * KV * R * kGroups;
  const int Nc = a.n_codes;
  uint4* img = reinterpret_cast<uint4*>(smem);
  uint8_t* cbuf = smem + R * kGroups * Nc * 16;               // [2][kChunkBytes]
  const bool check = Nc < 256;
  const int tid = threadIdx.x, j = tid & (kGroups - 1), rk0 = tid >> 4;   // record index within a row step
  const int o0 = rk0 / KV;                                    // first row of the thread
  int err = 0;
  const int64_t n_items = static_cast<int64_t>(a.B) * a.n_hi;

  // step phasor e^{i kRowStep theta} of the thread's pairs 4j..4j+3 (two packed entries)
  f32x2 sc[2], ss[2];
  load_phasor(a.rowph[kRowStep * (kD / 4) + 2 * j], sc[0], ss[0]);
  load_phasor(a.rowph[kRowStep * (kD / 4) + 2 * j + 1], sc[1], ss[1]);

  auto chunk_of = [&](int64_t w, int64_t& rec0, int& rows, int& h) {
    const int b = static_cast<int>(w / a.n_hi);
    h = static_cast<int>(w % a.n_hi);
    int64_t row0;
    const int64_t Tb = sequence_rows(a.seq_offsets, b, a.max_T, a.error_word, row0);
    const int64_t t0 = static_cast<int64_t>(h) * kChunk;
    rows = t0 >= Tb ? 0 : static_cast<int>(min(static_cast<int64_t>(kChunk), Tb - t0));
    rec0 = (row0 + t0) * KV;
  };

  for (int side = 0; side < 2; ++side) {
    const uint8_t* codes = side ? a.v_codes : a.k_codes;
    uint4* out = static_cast<uint4*>(side ? a.v_out : a.k_out);
    const uint4* src = side ? a.v_img : a.k_img;
    __syncthreads();   // the previous side is done with the image and the code buffers
    for (int p = tid; p < R * kGroups * Nc; p += kDecThreads) cp_async16(img + p, src + p);
    int64_t w = blockIdx.x;
    int64_t rec0 = 0;
    int rows = 0, h = 0, buf = 0;
    if (w < n_items) {
      chunk_of(w, rec0, rows, h);
      issue_chunk<R>(cbuf, codes, rec0, rows, KV);
    }
    cp_async_commit();
    for (; w < n_items; w += gridDim.x, buf ^= 1) {
      int64_t nrec0 = 0;
      int nrows = 0, nh = 0;
      if (w + gridDim.x < n_items) {
        chunk_of(w + gridDim.x, nrec0, nrows, nh);
        issue_chunk<R>(cbuf + (buf ^ 1) * kChunkBytes, codes, nrec0, nrows, KV);
      }
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      const uint8_t* cb = cbuf + buf * kChunkBytes;
      f32x2 pc[2], ps[2];   // phasors of the thread's pairs at its current row
      if (side == 0) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          f32x2 hc, hs;
          load_phasor(a.coarse[static_cast<int64_t>(h) * (kD / 4) + 2 * j + q], hc, hs);
          load_phasor(a.rowph[o0 * (kD / 4) + 2 * j + q], pc[q], ps[q]);
          cmul2(pc[q], ps[q], hc, hs);
        }
      }
      for (int o = o0; o < rows; o += kRowStep) {
        const int rk = o * KV + (rk0 % KV);
        const uint8_t* cr = cb + rk * (R * kGroups) + j;
        int c0 = cr[0];
        if (check && c0 >= Nc) { c0 = Nc - 1; err = 1; }
        uint4 e = img[dslot(0, j, c0, Nc)];
        if (R == 2) {
          int c1 = cr[kGroups];
          if (check && c1 >= Nc) { c1 = Nc - 1; err = 1; }
          const uint4 f = img[dslot(1, j, c1, Nc)];
          e.x = h2u(__hadd2(u2h(e.x), u2h(f.x)));
          e.y = h2u(__hadd2(u2h(e.y), u2h(f.y)));
          e.z = h2u(__hadd2(u2h(e.z), u2h(f.z)));
          e.w = h2u(__hadd2(u2h(e.w), u2h(f.w)));
        }
        uint4 v;
        if (side == 0) {
          rotate_out<OT>(e.x, e.y, pc[0], ps[0], v.x, v.y);
          rotate_out<OT>(e.z, e.w, pc[1], ps[1], v.z, v.w);
          cmul2(pc[0], ps[0], sc[0], ss[0]);
          cmul2(pc[1], ps[1], sc[1], ss[1]);
        } else {
          v.x = convert_out<OT>(e.x);
          v.y = convert_out<OT>(e.y);
          v.z = convert_out<OT>(e.z);
          v.w = convert_out<OT>(e.w);
        }
        out[(rec0 + rk) * kGroups + j] = v;
      }
      __syncthreads();   // this buffer is refilled two chunks on
      rec0 = nrec0;
      rows = nrows;
      h = nh;
    }
    cp_async_wait<0>();
  }
  if (check) {
    err = __syncthreads_or(err);
    if (err && tid == 0) atomicOr(a.error_word, kErrCodeRange);
  }
}

// ---------------------------------------------------------------------------------------
// Dense flash-decoding.
constexpr int kDenseThreads = 256;   // 8 warps
constexpr int kDenseWarps = 8;
constexpr int kDenseStages = 3;
constexpr int kDenseStageBytes = 65536;   // (16 * 8 / KV) positions x KV heads x (K + V) 256 B rows

struct DenseArgs {
  const void* k;
  const void* v;
  const int64_t* seq_offsets;
  Partial* partials;
  int* error_word;
  int64_t max_T;
  int B;
  int q_heads;
  int kv_heads;
};

// 16-byte asynchronous copy that writes zeros instead when !valid (src-size 0).
__device__ __forceinline__ void cp_async16_zfill(void* smem_dst, const void* gmem_src, bool valid) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem_src), "r"(n) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

template <typename T>
__device__ __forceinline__ void mma_kv(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1);
template <>
__device__ __forceinline__ void mma_kv<__half>(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <>
__device__ __forceinline__ void mma_kv<__nv_bfloat16>(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                                      uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <typename QT>
__device__ __forceinline__ float qload(const QT* q, int i);
template <>
__device__ __forceinline__ float qload<float>(const float* q, int i) { return q[i]; }
template <>
__device__ __forceinline__ float qload<__half>(const __half* q, int i) { return __half2float(q[i]); }
template <>
__device__ __forceinline__ float qload<__nv_bfloat16>(const __nv_bfloat16* q, int i) {
  return __bfloat162float(q[i]);
}

// Byte offset of 16-byte chunk c (8 dims) of the row of stage position pos and KV head kv;
// the chunk index is XOR-swizzled by the position's low 3 bits.
__device__ __forceinline__ uint32_t dense_slot(int pos, int kv, int c, int KV) {
  return static_cast<uint32_t>(((pos * KV + kv) * 16 + (c ^ (pos & 7))) * 16);
}

template <int KV, typename T, typename QT>
__global__ void __launch_bounds__(kDenseThreads, 1) dense_decode_kernel(DenseArgs a, const QT* __restrict__ q) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int kWpk = kDenseWarps / KV;      // warps per KV head
  constexpr int kSP = 16 * kWpk;              // positions per stage
  constexpr int kSideBytes = kSP * KV * 256;  // K (or V) bytes per stage
  static_assert(2 * kSideBytes == kDenseStageBytes, "stage size");
  const int G = a.q_heads / KV;
  const int s = blockIdx.x, b = blockIdx.y, S = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, i = lane & 3;
  const int kv = warp / kWpk, sub = warp % kWpk;

  int64_t row0;
  const int64_t Tb = sequence_rows(a.seq_offsets, b, a.max_T, running_error(a.error_word), row0);
  int64_t per = (Tb + S - 1) / S;
  per = (per + 15) / 16 * 16;
  const int64_t t_begin = min(Tb, static_cast<int64_t>(s) * per);
  const int64_t t_end = min(Tb, t_begin + per);

  const unsigned char* kg = static_cast<const unsigned char*>(a.k) + row0 * KV * 256;
  const unsigned char* vg = static_cast<const unsigned char*>(a.v) + row0 * KV * 256;
  auto issue = [&](int buf, int64_t t) {
    unsigned char* dst = smem + buf * kDenseStageBytes;
    for (int c = tid; c < kSP * KV * 16; c += kDenseThreads) {
      const int pos = c / (KV * 16), kvc = (c / 16) % KV, ch = c & 15;
      const bool ok = t + pos < t_end;
      const int64_t off = ok ? (t * KV * 256 + static_cast<int64_t>(c) * 16) : 0;
      const uint32_t d = dense_slot(pos, kvc, ch, KV);
      cp_async16_zfill(dst + d, kg + off, ok);
      cp_async16_zfill(dst + kSideBytes + d, vg + off, ok);
    }
  };

  // Query fragments (mma A, rows = the group's heads, k = dims), in the K/V element type.
  uint32_t qa[8][4];
  {
    const int h0 = kv * G + g, h1 = kv * G + g + 8;
    const QT* q0 = q + (static_cast<int64_t>(b) * a.q_heads + h0) * kD;
    const QT* q1 = q + (static_cast<int64_t>(b) * a.q_heads + h1) * kD;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int d0 = 16 * kk + 2 * i;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (g < G) {
        v[0] = qload(q0, d0); v[1] = qload(q0, d0 + 1);
        v[4] = qload(q0, d0 + 8); v[5] = qload(q0, d0 + 9);
      }
      if (g + 8 < G) {
        v[2] = qload(q1, d0); v[3] = qload(q1, d0 + 1);
        v[6] = qload(q1, d0 + 8); v[7] = qload(q1, d0 + 9);
      }
      qa[kk][0] = pack_out<T>(v[0], v[1]);
      qa[kk][1] = pack_out<T>(v[2], v[3]);
      qa[kk][2] = pack_out<T>(v[4], v[5]);
      qa[kk][3] = pack_out<T>(v[6], v[7]);
    }
  }

  const float scale = 1.4426950408889634f / sqrtf(static_cast<float>(kD));   // exp2 domain
  float O[16][4];
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) O[dt][0] = O[dt][1] = O[dt][2] = O[dt][3] = 0.0f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;   // rows g, g+8

  if (t_begin < t_end) {
    issue(0, t_begin);
    cp_async_commit();
    issue(1, t_begin + kSP);
    cp_async_commit();
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    int it = 0;
    for (int64_t t = t_begin; t < t_end; t += kSP, ++it) {
      if (t + 2 * kSP < t_end) issue((it + 2) % kDenseStages, t + 2 * kSP);
      cp_async_commit();
      cp_async_wait<2>();
      __syncthreads();
      const int64_t tt0 = t + sub * 16;
      const int nvalid = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(16), t_end - tt0)));
      if (nvalid > 0) {
        const uint32_t kb = sbase + (it % kDenseStages) * kDenseStageBytes;
        const uint32_t vb = kb + kSideBytes;
        const int p0 = sub * 16;
        // S^T tile: rows = heads, cols = 16 positions (two n-tiles of 8)
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
          const int lp = p0 + (lane & 7) + ((lane >> 4) << 3);
          const int lc = (lane >> 3) & 1;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            uint32_t r[4];
            ldsm_x4(kb + dense_slot(lp, kv, 2 * kk + lc, KV), r);
            mma_kv<T>(acc[0], qa[kk], r[0], r[1]);
            mma_kv<T>(acc[1], qa[kk], r[2], r[3]);
          }
        }
        float sc[2][4];
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int pos = nt * 8 + 2 * i + (c & 1);
            sc[nt][c] = pos < nvalid ? acc[nt][c] * scale : -INFINITY;
            if (c < 2) mx0 = fmaxf(mx0, sc[nt][c]); else mx1 = fmaxf(mx1, sc[nt][c]);
          }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        // every tile has a valid position, so the new maxima are finite
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
        const float al0 = exp2f(m0 - n0), al1 = exp2f(m1 - n1);
        m0 = n0;
        m1 = n1;
        float pr[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int c = 0; c < 4; ++c) pr[nt][c] = exp2f(sc[nt][c] - (c < 2 ? n0 : n1));
        l0 = l0 * al0 + (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
        l1 = l1 * al1 + (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]);
#pragma unroll
        for (int dt = 0; dt < 16; ++dt) {
          O[dt][0] *= al0;
          O[dt][1] *= al0;
          O[dt][2] *= al1;
          O[dt][3] *= al1;
        }
        // P as the A operand (rows = heads, k = the 16 positions)
        const uint32_t pa[4] = {pack_out<T>(pr[0][0], pr[0][1]), pack_out<T>(pr[0][2], pr[0][3]),
                                pack_out<T>(pr[1][0], pr[1][1]), pack_out<T>(pr[1][2], pr[1][3])};
        {
          const int lp = p0 + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int lc = lane >> 4;
#pragma unroll
          for (int dt = 0; dt < 16; dt += 2) {
            uint32_t r[4];
            ldsm_x4_trans(vb + dense_slot(lp, kv, dt + lc, KV), r);
            mma_kv<T>(O[dt], pa, r[0], r[1]);
            mma_kv<T>(O[dt + 1], pa, r[2], r[3]);
          }
        }
      }
      __syncthreads();
    }
    cp_async_wait<0>();
  }

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const int SE = S * kWpk;   // partial slots per (sequence, head)
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int row = g + 8 * rr;
    if (row >= G) continue;
    Partial* p = a.partials + (static_cast<int64_t>(b) * a.q_heads + kv * G + row) * SE + s * kWpk + sub;
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      p->o[dt * 8 + 2 * i] = O[dt][2 * rr];
      p->o[dt * 8 + 2 * i + 1] = O[dt][2 * rr + 1];
    }
    if (i == 0) {
      p->m = rr ? m1 : m0;
      p->l = rr ? l1 : l0;
    }
  }
}

int dense_splits(int B, int64_t max_T, const commvq_attend_options* opt) {
  if (opt && opt->splits > 0) return opt->splits;
  const DeviceInfo di = current_device_info();
  const int sms = di.sms > 0 ? di.sms : 148;
  int64_t S = B >= sms ? 1 : sms / B;
  const int64_t by_len = (max_T + 63) / 64;
  if (S > by_len) S = by_len;
  if (S < 1) S = 1;
  if (S > 512) S = 512;
  return static_cast<int>(S);
}

bool dense_shape_ok(const commvq_config* cfg) {
  if (!cfg || cfg->d != kD || cfg->q_heads < 1 || cfg->kv_heads < 1 || cfg->q_heads % cfg->kv_heads) return false;
  const int KV = cfg->kv_heads;
  return (KV == 1 || KV == 2 || KV == 4 || KV == 8) && cfg->q_heads / KV <= 16;
}

template <int KV, typename T>
commvq_status launch_dense_t(const DenseArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st) {
  const dim3 grid(S, a.B);
  const int smem = kDenseStages * kDenseStageBytes;
#define COMMVQ_DENSE(QTYPE)                                                                      \
  {                                                                                              \
    auto k = dense_decode_kernel<KV, T, QTYPE>;                                                  \
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) \
      return COMMVQ_ERR_CUDA;                                                                    \
    k<<<grid, kDenseThreads, smem, st>>>(a, static_cast<const QTYPE*>(q));                       \
  }
  if (qt == COMMVQ_F32) COMMVQ_DENSE(float)
  else if (qt == COMMVQ_F16) COMMVQ_DENSE(__half)
  else COMMVQ_DENSE(__nv_bfloat16)
#undef COMMVQ_DENSE
  return launch_status();
}

template <typename T>
commvq_status launch_dense_kv(const DenseArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st) {
  switch (a.kv_heads) {
    case 1: return launch_dense_t<1, T>(a, q, qt, S, st);
    case 2: return launch_dense_t<2, T>(a, q, qt, S, st);
    case 4: return launch_dense_t<4, T>(a, q, qt, S, st);
    case 8: return launch_dense_t<8, T>(a, q, qt, S, st);
    default: return COMMVQ_ERR_UNSUPPORTED;
  }
}

struct DecompLayout {
  size_t kimg_off, vimg_off, rowph_off, coarse_off, total;
};
DecompLayout decomp_layout(const commvq_config* cfg, int64_t max_T) {
  DecompLayout L{};
  const size_t img = static_cast<size_t>(cfg->R) * kGroups * cfg->n_codes * 16;
  const int64_t n_hi = (max_T + kChunk - 1) / kChunk;
  L.kimg_off = kHeader;
  L.vimg_off = round_up(L.kimg_off + img, 256);
  L.rowph_off = round_up(L.vimg_off + img, 256);
  L.coarse_off = round_up(L.rowph_off + static_cast<size_t>(kChunk) * (kD / 4) * sizeof(float4), 256);
  L.total = round_up(L.coarse_off + static_cast<size_t>(n_hi > 0 ? n_hi : 1) * (kD / 4) * sizeof(float4), 256);
  return L;
}

commvq_status decomp_check(const commvq_config* cfg) {
  if (!cfg) return COMMVQ_ERR_INVALID_ARG;
  const int Nc = cfg->n_codes;
  if (cfg->d <= 0 || cfg->g <= 0 || cfg->d % cfg->g || cfg->g % 2 || cfg->R < 1 || Nc < 1 || Nc > 65536 ||
      cfg->q_heads < 1 || cfg->kv_heads < 1 || cfg->q_heads % cfg->kv_heads || !(cfg->rope_base > 0.0) ||
      !isfinite(cfg->rope_base))
    return COMMVQ_ERR_INVALID_ARG;
  if (cfg->code_bytes != (Nc <= 256 ? 1 : 2)) return COMMVQ_ERR_INVALID_ARG;
  const int KV = cfg->kv_heads;
  if (cfg->d != kD || cfg->g != kG || Nc > 256 || cfg->R > 2 || (KV != 1 && KV != 2 && KV != 4 && KV != 8))
    return COMMVQ_ERR_UNSUPPORTED;
  return COMMVQ_OK;
}

}  // namespace
}  // namespace commvq

using namespace commvq;

extern "C" size_t commvq_decompress_workspace_bytes(const commvq_config* cfg, int64_t max_T) {
  if (decomp_check(cfg) != COMMVQ_OK || max_T < 0 || max_T > (int64_t(1) << 31)) return 0;
  return decomp_layout(cfg, max_T).total;
}

extern "C" commvq_status commvq_decompress(const commvq_config* cfg, const void* k_codes, const void* v_codes,
                                           const int64_t* seq_offsets, int32_t B, int64_t max_T,
                                           const float* k_codebook, const float* v_codebook,
                                           commvq_dtype out_dtype, void* k_out, void* v_out, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("commvq_decompress");
  const commvq_status cs = decomp_check(cfg);
  if (cs != COMMVQ_OK) return cs;
  if (B < 0 || max_T < 0) return COMMVQ_ERR_INVALID_ARG;
  if (out_dtype != COMMVQ_F16 && out_dtype != COMMVQ_BF16) return COMMVQ_ERR_INVALID_ARG;
  if (B == 0) return COMMVQ_OK;
  if (!k_codes || !v_codes || !seq_offsets || !k_codebook || !v_codebook || !k_out || !v_out || !workspace)
    return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(k_codebook, 16) || !aligned(v_codebook, 16) || !aligned(k_out, 16) || !aligned(v_out, 16) ||
      !aligned(seq_offsets, 8) || !aligned(workspace, 256))
    return COMMVQ_ERR_INVALID_ARG;
  const size_t need = commvq_decompress_workspace_bytes(cfg, max_T);
  if (need == 0 || workspace_bytes < need) return COMMVQ_ERR_WORKSPACE;
  const DeviceInfo di = current_device_info();
  if (di.device < 0) return COMMVQ_ERR_CUDA;
  const size_t smem = static_cast<size_t>(cfg->R) * kGroups * cfg->n_codes * 16 +
                      static_cast<size_t>(2) * kChunk * cfg->kv_heads * cfg->R * kGroups;
  if (smem > di.smem_optin) return COMMVQ_ERR_UNSUPPORTED;

  const DecompLayout L = decomp_layout(cfg, max_T);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  DecompArgs a{};
  a.k_codes = static_cast<const uint8_t*>(k_codes);
  a.v_codes = static_cast<const uint8_t*>(v_codes);
  a.seq_offsets = seq_offsets;
  a.k_codebook = k_codebook;
  a.v_codebook = v_codebook;
  a.k_out = k_out;
  a.v_out = v_out;
  a.k_img = reinterpret_cast<uint4*>(ws + L.kimg_off);
  a.v_img = reinterpret_cast<uint4*>(ws + L.vimg_off);
  a.rowph = reinterpret_cast<float4*>(ws + L.rowph_off);
  a.coarse = reinterpret_cast<float4*>(ws + L.coarse_off);
  a.error_word = static_cast<int*>(workspace);
  a.max_T = max_T;
  a.rope_base = cfg->rope_base;
  a.B = B;
  a.kv_heads = cfg->kv_heads;
  a.R = cfg->R;
  a.n_codes = cfg->n_codes;
  a.n_hi = static_cast<int>((max_T + kChunk - 1) / kChunk);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (max_T == 0) return cudaMemsetAsync(a.error_word, 0, sizeof(int), st) == cudaSuccess ? COMMVQ_OK : COMMVQ_ERR_CUDA;

  const int prep_items = std::max(cfg->R * kGroups * cfg->n_codes, std::max(kChunk, a.n_hi) * (kD / 2));
  decompress_prep_kernel<<<dim3((prep_items + 255) / 256, 4), 256, 0, st>>>(a);
  if (launch_status() != COMMVQ_OK) return COMMVQ_ERR_CUDA;
  const int64_t items = static_cast<int64_t>(B) * a.n_hi;
  const int grid_x = static_cast<int>(std::min<int64_t>(items, di.sms > 0 ? di.sms : 148));
#define COMMVQ_DECOMP(RR, KVV, OT)                                                                 \
  {                                                                                                \
    auto k = decompress_kernel<RR, KVV, OT>;                                                       \
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) \
      return COMMVQ_ERR_CUDA;                                                                      \
    k<<<grid_x, kDecThreads, smem, st>>>(a);                                                       \
  }
#define COMMVQ_DECOMP_KV(RR, OT)                            \
  switch (cfg->kv_heads) {                                  \
    case 1: COMMVQ_DECOMP(RR, 1, OT) break;                 \
    case 2: COMMVQ_DECOMP(RR, 2, OT) break;                 \
    case 4: COMMVQ_DECOMP(RR, 4, OT) break;                 \
    default: COMMVQ_DECOMP(RR, 8, OT) break;                \
  }
  if (cfg->R == 1) {
    if (out_dtype == COMMVQ_F16) { COMMVQ_DECOMP_KV(1, __half) } else { COMMVQ_DECOMP_KV(1, __nv_bfloat16) }
  } else {
    if (out_dtype == COMMVQ_F16) { COMMVQ_DECOMP_KV(2, __half) } else { COMMVQ_DECOMP_KV(2, __nv_bfloat16) }
  }
#undef COMMVQ_DECOMP_KV
#undef COMMVQ_DECOMP
  return launch_status();
}

extern "C" size_t commvq_dense_decode_workspace_bytes(const commvq_config* cfg, int32_t B, int64_t max_T,
                                                      const commvq_attend_options* options) {
  if (!dense_shape_ok(cfg) || B < 0 || max_T < 0) return 0;
  if (options && (options->splits < 0 || options->splits > 512)) return 0;
  const int S = dense_splits(B > 0 ? B : 1, max_T, options);
  const int kWpk = kDenseWarps / cfg->kv_heads;
  return round_up(kHeader + static_cast<size_t>(B) * cfg->q_heads * S * kWpk * sizeof(Partial), 256);
}

extern "C" commvq_status commvq_dense_decode(const commvq_config* cfg, const void* q, commvq_dtype q_dtype,
                                             const void* k, const void* v, commvq_dtype kv_dtype,
                                             const int64_t* seq_offsets, int32_t B, int64_t max_T, float* out,
                                             float* lse, void* workspace, size_t workspace_bytes,
                                             const commvq_attend_options* options, void* stream) {
  const NvtxRange nvtx_range("commvq_dense_decode");
  if (!cfg) return COMMVQ_ERR_INVALID_ARG;
  if (cfg->q_heads < 1 || cfg->kv_heads < 1 || cfg->q_heads % cfg->kv_heads || cfg->d <= 0)
    return COMMVQ_ERR_INVALID_ARG;
  if (!dense_shape_ok(cfg)) return COMMVQ_ERR_UNSUPPORTED;
  if (B < 0 || max_T < 0) return COMMVQ_ERR_INVALID_ARG;
  if (q_dtype != COMMVQ_F32 && q_dtype != COMMVQ_F16 && q_dtype != COMMVQ_BF16) return COMMVQ_ERR_INVALID_ARG;
  if (kv_dtype != COMMVQ_F16 && kv_dtype != COMMVQ_BF16) return COMMVQ_ERR_INVALID_ARG;
  if (options && (options->splits < 0 || options->splits > 512)) return COMMVQ_ERR_INVALID_ARG;
  if (B == 0) return COMMVQ_OK;
  if (B > 65535) return COMMVQ_ERR_UNSUPPORTED;
  if (!q || !k || !v || !seq_offsets || !out || !workspace) return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
      !aligned(seq_offsets, 8) || !aligned(workspace, 256))
    return COMMVQ_ERR_INVALID_ARG;
  const size_t need = commvq_dense_decode_workspace_bytes(cfg, B, max_T, options);
  if (need == 0 || workspace_bytes < need) return COMMVQ_ERR_WORKSPACE;
  const DeviceInfo di = current_device_info();
  if (di.device < 0) return COMMVQ_ERR_CUDA;
  if (static_cast<size_t>(kDenseStages) * kDenseStageBytes > di.smem_optin) return COMMVQ_ERR_UNSUPPORTED;

  const int S = dense_splits(B, max_T, options);
  const int kWpk = kDenseWarps / cfg->kv_heads;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  DenseArgs d{};
  d.k = k;
  d.v = v;
  d.seq_offsets = seq_offsets;
  d.partials = reinterpret_cast<Partial*>(ws + kHeader);
  d.error_word = static_cast<int*>(workspace);
  d.max_T = max_T;
  d.B = B;
  d.q_heads = cfg->q_heads;
  d.kv_heads = cfg->kv_heads;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* start = options ? options->main_start : nullptr;
  void* stop = options ? options->main_stop : nullptr;
  if (cudaMemsetAsync(d.error_word, 0, 2 * sizeof(int), st) != cudaSuccess) return COMMVQ_ERR_CUDA;
  if (start && record_event(start, st) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  const commvq_status rc = kv_dtype == COMMVQ_F16 ? launch_dense_kv<__half>(d, q, q_dtype, S, st)
                                                  : launch_dense_kv<__nv_bfloat16>(d, q, q_dtype, S, st);
  if (rc != COMMVQ_OK) return rc;
  if (stop && record_event(stop, st) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  AttendArgs c{};
  c.out = out;
  c.lse = lse;
  c.partials = d.partials;
  c.error_word = d.error_word;
  c.B = B;
  c.q_heads = cfg->q_heads;
  return launch_combine(c, S * kWpk, st);
}
