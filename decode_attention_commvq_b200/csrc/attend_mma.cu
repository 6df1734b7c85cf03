// Decode attention on CommVQ codes, decode-and-rotate form with tensor-core dot products.
//
// The same attention as the table form, reorganised for B200's throughput balance. The
// table form gathers a per-query-head table entry for every (position, query head, round,
// group); here each (position, KV head) is decoded once for all query heads of its GQA
// group (the sum over rounds commutes with the query product: sum_r conj(q) c_r =
// conj(q) sum_r c_r), rotated once by e^{i t theta_p} (RoPE, moved onto the decoded key by
// the commuting-block property of the review's "What carries the argument"), and the dot
// products with the query heads run on the tensor cores (mma.sync m16n8k16, fp16 in, fp32
// accumulate). Values are decoded per (position, KV head) the same way and the softmax
// weights multiply them on the tensor cores (the value codebook multiply after the
// softmax weights, as in "If this is right").
//
// The fp16 key and value codebooks of a 2-round, 256-entry layer take 128 KB each, which
// do not fit one SM's shared memory together, so the step runs as two kernels over the
// same position splits:
//   scores : K codebook image in shared memory; for every 16-position tile and KV head,
//            gather + round sum + rotate straight into mma A fragments; S = K~ Q^T; scaled
//            scores (exp2 domain) go to an L2-resident buffer, per-split maxima to the
//            partials.
//   values : V codebook image in shared memory; p = exp2(s - m_split) straight into mma B
//            fragments; decoded values straight into A fragments; O^T += V^T P^T.
// The split-T merge kernel of the table form then combines the partials.
//
// Shared-memory gathers bound both kernels (16 bytes of codebook per code byte). The
// codebook image is laid out so that every 8-lane phase of a 128-bit gather touches 8
// different 16-byte bank groups: entry (v, j, c) -- v a "virtual round" -- sits in slot
// ((v*2 + j/8)*Nc' + c)*8 + ((j + 4v) % 8). With two rounds v is the round and lanes of
// odd and even rows load the rounds in opposite order; with one round the image holds the
// round twice (v = copy) and odd rows read the second copy.
#include <math.h>

#include "attend.cuh"

namespace commvq {
namespace {

constexpr int kMmaThreads = 512;           // 16 warps per CTA, one CTA per SM
constexpr int kMmaWarps = kMmaThreads / 32;
constexpr int kTiles = 8;                  // mma row blocks per pipeline stage
constexpr int kTileT = 16;                 // positions per mma row block
constexpr int kStageT = kTiles * kTileT;   // positions per pipeline stage

// Barrier for a subset of the CTA's warps (ids 1..15; id 0 is __syncthreads).
__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}
constexpr int kRefresh = 16;               // phasor recurrence steps between exact refreshes

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

__device__ __forceinline__ uint4 hadd2x4(uint4 a, uint4 b) {
  uint4 r;
  r.x = h2_as_u32(__hadd2(u32_as_h2(a.x), u32_as_h2(b.x)));
  r.y = h2_as_u32(__hadd2(u32_as_h2(a.y), u32_as_h2(b.y)));
  r.z = h2_as_u32(__hadd2(u32_as_h2(a.z), u32_as_h2(b.z)));
  r.w = h2_as_u32(__hadd2(u32_as_h2(a.w), u32_as_h2(b.w)));
  return r;
}

__device__ __forceinline__ uint32_t word(const uint4& v, int k) {
  return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
}

// Rotate the stored pair (a, b) (one half2) by the phasor (cos, sin) in fp32; fp16 result.
__device__ __forceinline__ uint32_t rotate_pair(uint32_t ab, float2 ph) {
  const float2 f = __half22float2(u32_as_h2(ab));
  const float x = fmaf(f.x, ph.x, -f.y * ph.y);
  const float y = fmaf(f.x, ph.y, f.y * ph.x);
  return h2_as_u32(__floats2half2_rn(x, y));
}

template <typename QT>
__device__ __forceinline__ float qval(const QT* q, int i);
template <>
__device__ __forceinline__ float qval<float>(const float* q, int i) { return q[i]; }
template <>
__device__ __forceinline__ float qval<__half>(const __half* q, int i) { return __half2float(q[i]); }
template <>
__device__ __forceinline__ float qval<__nv_bfloat16>(const __nv_bfloat16* q, int i) {
  return __bfloat162float(q[i]);
}

// Position range of split s of sequence b: tile-aligned pieces of ceil(T_b / S).
__device__ __forceinline__ void split_range(const AttendArgs& a, int b, int s, int S, int64_t& row0,
                                            int64_t& t_begin, int64_t& t_end) {
  row0 = a.seq_offsets[b];
  int64_t Tb = a.seq_offsets[b + 1] - row0;
  Tb = Tb < 0 ? 0 : (Tb > a.max_T ? a.max_T : Tb);
  int64_t per = (Tb + S - 1) / S;
  per = (per + kTileT - 1) / kTileT * kTileT;
  t_begin = min(Tb, static_cast<int64_t>(s) * per);
  t_end = min(Tb, t_begin + per);
}

// Copy one stage (kStageT positions x KV heads x R x 16 code bytes, contiguous in HBM) into
// shared memory with 16-byte asynchronous copies. Positions past t_end are not copied. The
// 16-byte pieces of a position's record are XOR-swizzled by the position's low 3 bits (when
// a record has at least 8 pieces) so that reads of the same piece of neighbouring positions
// fall in different bank groups.
template <int R, int KV>
struct StageLayout {
  static constexpr int kPieces = KV * R;                 // 16-byte pieces per position
  static constexpr int kSwz = kPieces >= 8 ? 7 : 0;
  static constexpr int kBytes = kStageT * kPieces * 16;
  __device__ static __forceinline__ int offset(int row, int piece) {
    return (row * kPieces + (piece ^ (row & kSwz))) * 16;
  }
};

template <int R, int KV>
__device__ __forceinline__ void issue_stage(uint8_t* dst, const uint8_t* codes, int64_t row0,
                                            int64_t t0, int64_t t_end) {
  using SL = StageLayout<R, KV>;
  const int n = static_cast<int>(min(static_cast<int64_t>(kStageT), t_end - t0));
  const int pieces = n * SL::kPieces;
  const uint8_t* src = codes + (row0 + t0) * (SL::kPieces * 16);
  for (int p = threadIdx.x; p < pieces; p += blockDim.x) {
    const int row = p / SL::kPieces, piece = p - row * SL::kPieces;
    cp_async16(dst + SL::offset(row, piece), src + p * 16);
  }
}

// Scores are stored tile-blocked: for sequence b, 16-position tile tau, KV head kv, head
// column col < G and values-kernel lane quad i, four floats for positions 2i, 2i+1, 2i+8,
// 2i+9 -- the exact B-fragment order of the values kernel.
__device__ __forceinline__ int64_t score_index(int64_t b, int64_t tau, int kv, int col, int i, int k,
                                               int64_t n_tiles, int KV, int G) {
  return ((((b * n_tiles + tau) * KV + kv) * G + col) * 4 + i) * 4 + k;
}

__device__ __forceinline__ int clamp_code(int c, int Nc, int& err) {
  if (c >= Nc) {
    err = 1;
    return Nc - 1;
  }
  return c;
}

// ---------------------------------------------------------------------------------------
// Per-call preparation. blockIdx.y = 0 / 1: key / value codebook image, fp32 [R][16][Nc'][8]
// -> fp16 slots (see the file comment). blockIdx.y = 2: RoPE tables, all from fp64:
//   theta[p] = base^(-2p/d), row[delta][p] = e^{i delta theta_p} for the 128 rows of a stage,
//   adv[p] = e^{i 128 theta_p} (one stage further).
constexpr int kPhaseRows = kStageT;

// blockIdx.y = 3: query fragments of every (sequence, KV head) in the scores kernel's mma
// k-order (see attend_scores_kernel); blockIdx.y = 4: base phasor e^{i t_begin theta_p} of
// every (sequence, split), from an fp64 angle.
template <typename QT>
__device__ __forceinline__ void prep_qfrag(const AttendArgs& a, const QT* q, int e) {
  const int KV = a.kv_heads, G = a.q_heads / KV;
  if (e >= a.B * KV * 256) return;
  const int b = e / (KV * 256), r = e % (KV * 256);
  const int kv = r >> 8, st = (r >> 5) & 7, ln = r & 31;
  const int gg = ln >> 2, ii = ln & 3;
  uint2 v = make_uint2(0u, 0u);
  if (gg < G) {
    const QT* qh = q + (static_cast<int64_t>(b) * a.q_heads + kv * G + gg) * kD;
    const int d0 = 8 * (4 * (st >> 1) + ii) + 4 * (st & 1);
    v.x = h2_as_u32(__floats2half2_rn(qval(qh, d0), qval(qh, d0 + 1)));
    v.y = h2_as_u32(__floats2half2_rn(qval(qh, d0 + 2), qval(qh, d0 + 3)));
  }
  const_cast<uint2*>(a.qfrag)[e] = v;
}

__global__ void prep_kernel(AttendArgs a, int R, const void* __restrict__ q, int q_dtype, int S) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int Nc = a.n_codes;
  if (e == 0 && blockIdx.y == 0) *a.error_word = 0;   // this call's device error word starts clear
  if (blockIdx.y == 3) {
    if (q_dtype == COMMVQ_F32) prep_qfrag(a, static_cast<const float*>(q), e);
    else if (q_dtype == COMMVQ_F16) prep_qfrag(a, static_cast<const __half*>(q), e);
    else prep_qfrag(a, static_cast<const __nv_bfloat16*>(q), e);
    return;
  }
  if (blockIdx.y == 4) {
    if (e >= a.B * S * (kD / 2)) return;
    const int p = e % (kD / 2), bs = e / (kD / 2), s = bs % S, b = bs / S;
    int64_t row0, t_begin, t_end;
    split_range(a, b, s, S, row0, t_begin, t_end);
    double sn, cs;
    sincos(static_cast<double>(t_begin) * pow(a.rope_base, -2.0 * p / kD), &sn, &cs);
    const_cast<float2*>(a.basetab)[e] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
    return;
  }
  const double rope_base = a.rope_base;
  double* theta = const_cast<double*>(a.theta);
  float2* rowph = const_cast<float2*>(a.rowph);
  float2* advph = const_cast<float2*>(a.advph);
  const float* kcb = a.k_codebook;
  const float* vcb = a.v_codebook;
  uint4* kimg = const_cast<uint4*>(a.k_img);
  uint4* vimg = const_cast<uint4*>(a.v_img);
  if (blockIdx.y == 2) {
    if (e >= kPhaseRows * (kD / 2)) return;
    const int delta = e / (kD / 2), p = e % (kD / 2);
    const double th = pow(rope_base, -2.0 * p / kD);
    double sn, cs;
    sincos(static_cast<double>(delta) * th, &sn, &cs);
    rowph[e] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
    if (delta == 0) {
      theta[p] = th;
      sincos(static_cast<double>(kStageT) * th, &sn, &cs);
      advph[p] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
    }
    return;
  }
  if (e >= 2 * kGroups * Nc) return;   // (v, j, c)
  const float* cb = blockIdx.y ? vcb : kcb;
  uint4* img = blockIdx.y ? vimg : kimg;
  const int c = e % Nc, vj = e / Nc, j = vj % kGroups, v = vj / kGroups;
  const int r = (R == 2) ? v : 0;
  float w[kG];
  load_row8(cb + ((static_cast<int64_t>(r) * kGroups + j) * Nc + c) * kG, w);
  uint4 o;
  o.x = h2_as_u32(__floats2half2_rn(w[0], w[1]));
  o.y = h2_as_u32(__floats2half2_rn(w[2], w[3]));
  o.z = h2_as_u32(__floats2half2_rn(w[4], w[5]));
  o.w = h2_as_u32(__floats2half2_rn(w[6], w[7]));
  img[((v * 2 + (j >> 3)) * Nc + c) * 8 + ((j + 4 * v) & 7)] = o;
}

__device__ __forceinline__ int slot(int v, int j, int c, int Nc) {
  return ((v * 2 + (j >> 3)) * Nc + c) * 8 + ((j + 4 * v) & 7);
}

// Shared-memory loads at a byte offset from the start of the dynamic shared array.
__device__ __forceinline__ uint4 lds128(const unsigned char* smem, uint32_t off) {
  return *reinterpret_cast<const uint4*>(smem + off);
}
__device__ __forceinline__ uint2 lds64(const unsigned char* smem, uint32_t off) {
  return *reinterpret_cast<const uint2*>(smem + off);
}
__device__ __forceinline__ uint32_t lds32(const unsigned char* smem, uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(smem + off);
}
// Byte b of w, zero-extended (one PRMT); sel = byte_sel(b).
__device__ __forceinline__ uint32_t byte_sel(int b) { return 0x4440u | static_cast<uint32_t>(b); }
__device__ __forceinline__ uint32_t take_byte(uint32_t w, uint32_t sel) { return __byte_perm(w, 0u, sel); }

// ---------------------------------------------------------------------------------------
// Scores. A 16-position tile is shared by a pair of warps (tile = warp / 2, half = warp % 2).
// Thread (g = lane/4, i = lane%4) owns rows g and g+8 of the tile and, through the k-order of
// the mma, 8 RoPE pairs: k-step 2u+h covers pairs 2h and 2h+1 of group 4u+i, and half h of
// the pair takes u = 2h and 2h+1 (groups i, 4+i or 8+i, 12+i). One 16-byte gather fills two
// k-steps of a row. Each half accumulates a partial S over its 64 dimensions; the halves add
// them through a small double-buffered exchange in shared memory, ordered by a named barrier
// per warp pair. The query fragments use the same k-order. Splitting the pairs halves the
// phasor registers, which lets 16 warps share an SM.
// NC: the entry count when it is 256 (compile-time; every uint8 code is valid), else 0
// (run-time count, codes checked against it).
template <int R, int KV, int NC, typename QT>
__global__ void __launch_bounds__(kMmaThreads, 1)
attend_scores_kernel(AttendArgs a, const QT* __restrict__ q) {
  constexpr bool kCheck = NC != 256;
  extern __shared__ __align__(16) unsigned char smem[];
  const int Nc = NC ? NC : a.n_codes;
  const int G = a.q_heads / KV;
  uint4* cbk = reinterpret_cast<uint4*>(smem);                       // 32 * Nc slots
  uint2* qf = reinterpret_cast<uint2*>(cbk + 32 * Nc);               // [KV][8][32]
  float2* base = reinterpret_cast<float2*>(qf + KV * 8 * 32);       // [64] e^{i t0 theta_p}
  float* red = reinterpret_cast<float*>(base + 64);                  // [8 tiles][KV*8]
  float4* xch = reinterpret_cast<float4*>(red + kTiles * KV * 8);    // [8 tiles][2][32]
  uint8_t* stage_buf = reinterpret_cast<uint8_t*>(xch + kTiles * 2 * 32);   // [2][kStageT][KV][R][16]
  using SL = StageLayout<R, KV>;
  constexpr int kStageBytes = SL::kBytes;

  const int s = blockIdx.x, b = blockIdx.y, S = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = warp >> 1, half = warp & 1;
  const int g = lane >> 2, i = lane & 3, par = g & 1;
  int64_t row0, t_begin, t_end;
  split_range(a, b, s, S, row0, t_begin, t_end);
  Partial* part = a.partials + static_cast<int64_t>(b) * a.q_heads * S + s;   // + h * S

  if (t_begin >= t_end) {
    for (int h = tid; h < a.q_heads; h += kMmaThreads) part[static_cast<int64_t>(h) * S].m = -INFINITY;
    return;
  }

  // Set-up is all asynchronous copies of what the prep kernel made: codebook image, query
  // fragments of this sequence, base phasors of this split; then the first code stage.
  for (int p = tid; p < 32 * Nc; p += kMmaThreads) cp_async16(cbk + p, a.k_img + p);
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.qfrag + static_cast<int64_t>(b) * KV * 256);
    for (int p = tid; p < KV * 256 / 2; p += kMmaThreads) cp_async16(reinterpret_cast<uint4*>(qf) + p, src + p);
    const uint4* bsrc = reinterpret_cast<const uint4*>(a.basetab + (static_cast<int64_t>(b) * S + s) * (kD / 2));
    if (tid < kD / 4) cp_async16(reinterpret_cast<uint4*>(base) + tid, bsrc + tid);
  }
  cp_async_commit();
  issue_stage<R, KV>(stage_buf, a.k_codes, row0, t_begin, t_end);
  cp_async_commit();
  (void)q;

  // Phasors of the thread's 8 pairs (k = 4 ul + m -> pair 4(4(2 half + ul) + i) + m) at its two
  // rows, and the per-iteration advance e^{i kStageT theta}. A refresh rebuilds them exactly
  // from the stage's base phasor (fp64 angle, in shared memory) times the prep row table.
  auto pair_of = [&](int k) { return 4 * (4 * (2 * half + (k >> 2)) + i) + (k & 3); };
  float2 ph[2][8], adv[8];
  auto load_rows = [&]() {
#pragma unroll
    for (int k = 0; k < 8; ++k)
#pragma unroll
      for (int rho = 0; rho < 2; ++rho) ph[rho][k] = a.rowph[(tile * kTileT + g + 8 * rho) * (kD / 2) + pair_of(k)];
  };
  auto times_base = [&]() {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 bp = base[pair_of(k)];
#pragma unroll
      for (int rho = 0; rho < 2; ++rho) {
        const float2 rp = ph[rho][k];
        ph[rho][k] = make_float2(fmaf(bp.x, rp.x, -bp.y * rp.y), fmaf(bp.x, rp.y, bp.y * rp.x));
      }
    }
  };
  load_rows();   // global loads in flight while the asynchronous copies land
#pragma unroll
  for (int k = 0; k < 8; ++k) adv[k] = a.advph[pair_of(k)];

  for (int e = tid; e < kTiles * KV * 8; e += kMmaThreads) red[e] = -INFINITY;
  const int64_t n_tiles = (a.max_T + kTileT - 1) / kTileT;
  const float scale = 1.4426950408889634f / sqrtf(static_cast<float>(kD));
  int err = 0;
  int stage = 0, it = 0;
  // Byte offsets of the thread's gathers: entry c of group 4u+i lives at g?[u - 2 half] + 128 c,
  // gF in the v = par half of the image (first round / copy), gS in the other.
  const uint32_t sel_i = byte_sel(i);
  uint32_t gF[2], gS[2];
#pragma unroll
  for (int ul = 0; ul < 2; ++ul) {
    const int j = 4 * (2 * half + ul) + i;
    gF[ul] = static_cast<uint32_t>(slot(par, j, 0, Nc)) * 16;
    gS[ul] = static_cast<uint32_t>(slot(par ^ 1, j, 0, Nc)) * 16;
  }

  for (int64_t t0 = t_begin; t0 < t_end; t0 += kStageT, stage ^= 1, ++it) {
    if (t0 + kStageT < t_end)
      issue_stage<R, KV>(stage_buf + (stage ^ 1) * kStageBytes, a.k_codes, row0, t0 + kStageT, t_end);
    cp_async_commit();
    if (it > 0 && it % kRefresh == 0 && tid < kD / 2) {   // later refresh: fp64 angle
      double sn, cs;
      sincos(static_cast<double>(t0) * a.theta[tid], &sn, &cs);
      base[tid] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
    }
    cp_async_wait<1>();
    __syncthreads();

    const int64_t tt0 = t0 + tile * kTileT;        // this warp pair's tile
    if (it % kRefresh == 0) {
      if (it > 0) load_rows();
      times_base();
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k)
#pragma unroll
        for (int rho = 0; rho < 2; ++rho) {
          const float2 p = ph[rho][k], d = adv[k];
          ph[rho][k] = make_float2(fmaf(p.x, d.x, -p.y * d.y), fmaf(p.x, d.y, p.y * d.x));
        }
    }
    if (tt0 < t_end) {   // uniform over the warp pair
      const uint32_t sb = static_cast<uint32_t>(stage_buf - smem) + stage * kStageBytes;
      const int rem = static_cast<int>(min(static_cast<int64_t>(kTileT), t_end - tt0));  // valid rows
      const bool valid0 = g < rem, valid1 = g + 8 < rem;
#pragma unroll 1
      for (int kv = 0; kv < KV; ++kv) {
        // code words 2 half, 2 half + 1 (groups 8 half .. 8 half + 7) of each row; with two
        // rounds, round `par` first (it pairs with the v = par half of the image)
        uint2 cw[2][R];
#pragma unroll
        for (int rho = 0; rho < 2; ++rho) {
          const bool valid = rho ? valid1 : valid0;
          const int row = tile * kTileT + g + 8 * rho;
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const int piece = kv * R + (R == 2 ? (r ^ par) : r);
            const uint32_t off = sb + SL::offset(row, piece) + 8 * half;
            cw[rho][r] = valid ? lds64(smem, off) : make_uint2(0u, 0u);
          }
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ul = 0; ul < 2; ++ul) {
          const int u = 2 * half + ul;
          uint32_t A[2][4];
#pragma unroll
          for (int rho = 0; rho < 2; ++rho) {
            uint4 e;
            int c0 = static_cast<int>(take_byte(ul ? cw[rho][0].y : cw[rho][0].x, sel_i));
            if (kCheck) c0 = clamp_code(c0, Nc, err);
            if (R == 2) {
              int c1 = static_cast<int>(take_byte(ul ? cw[rho][R - 1].y : cw[rho][R - 1].x, sel_i));
              if (kCheck) c1 = clamp_code(c1, Nc, err);
              e = hadd2x4(lds128(smem, gF[ul] + (c0 << 7)), lds128(smem, gS[ul] + (c1 << 7)));
            } else {
              e = lds128(smem, gF[ul] + (c0 << 7));
            }
            A[0][rho] = rotate_pair(e.x, ph[rho][4 * ul + 0]);
            A[0][2 + rho] = rotate_pair(e.y, ph[rho][4 * ul + 1]);
            A[1][rho] = rotate_pair(e.z, ph[rho][4 * ul + 2]);
            A[1][2 + rho] = rotate_pair(e.w, ph[rho][4 * ul + 3]);
          }
          const uint2 b0 = qf[(kv * 8 + 2 * u) * 32 + lane];
          const uint2 b1 = qf[(kv * 8 + 2 * u + 1) * 32 + lane];
          mma16816(acc, A[0][0], A[0][1], A[0][2], A[0][3], b0.x, b0.y);
          mma16816(acc, A[1][0], A[1][1], A[1][2], A[1][3], b1.x, b1.y);
        }
        // Add the two halves' partial S. For even kv half 1 hands its partial to half 0, for
        // odd kv the reverse, so the finishing work (stores, maxima) alternates between the
        // two warps. The buffer alternates with kv, so the handing half can run one kv ahead.
        const int finisher = kv & 1;
        float4* xs = xch + (tile * 2 + (kv & 1)) * 32 + lane;
        if (half != finisher) *xs = make_float4(acc[0], acc[1], acc[2], acc[3]);
        named_barrier_sync(1 + tile, 64);
        if (half != finisher) continue;
        {
          const float4 o = *xs;
          acc[0] += o.x;
          acc[1] += o.y;
          acc[2] += o.z;
          acc[3] += o.w;
        }
        // acc: rows g (c0, c1) and g+8 (c2, c3); columns 2i, 2i+1 = query heads kv*G + col.
        const int64_t tau = tt0 / kTileT;
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col = 2 * i + c;
          if (col >= G) continue;
          const float v0 = acc[c] * scale, v1 = acc[2 + c] * scale;
          float* sp = a.scores + score_index(b, tau, kv, col, g >> 1, g & 1, n_tiles, KV, G);
          if (valid0) sp[0] = v0;
          if (valid1) sp[2] = v1;
          const float mv = fmaxf(valid0 ? v0 : -INFINITY, valid1 ? v1 : -INFINITY);
          if (c == 0) m0 = mv; else m1 = mv;
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
          m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
        }
        if (g == 0) {
          float* rw = red + tile * KV * 8 + kv * 8 + 2 * i;
          rw[0] = fmaxf(rw[0], m0);
          rw[1] = fmaxf(rw[1], m1);
        }
      }
    }
    __syncthreads();
  }

  // split maxima: each tile's warp pair kept a row of maxima (entries of even kv heads written
  // by half 0, odd by half 1); take the max over tiles
  for (int e = tid; e < KV * 8; e += kMmaThreads) {
    const int kv = e >> 3, col = e & 7;
    if (col >= G) continue;
    float v = -INFINITY;
#pragma unroll
    for (int w = 0; w < kTiles; ++w) v = fmaxf(v, red[w * KV * 8 + e]);
    part[static_cast<int64_t>(kv * G + col) * S].m = v;
  }
  if (kCheck) {
    err = __syncthreads_or(err);
    if (err && tid == 0) atomicOr(a.error_word, kErrCodeRange);
  }
}

// ---------------------------------------------------------------------------------------
// Values. O^T (128 dims x 8 columns) += V^T (dims x 16 positions) P^T (positions x heads).
// Thread (g, i) owns value dims 16g..16g+15 (groups 2g, 2g+1; mma row g of m-tile m is dim
// 16g+m, row g+8 is dim 16g+8+m) and positions 2i, 2i+1, 2i+8, 2i+9 of each tile, which are
// exactly the positions of its P^T fragment, so probabilities go from the score buffer into
// registers with no exchange. Warps are spread over KV heads (16/KV warps per head, each
// taking every (16/KV)-th tile of a stage); the A fragments are built one position pair at a
// time to stay within the 128 registers that 16 warps per SM allow.
template <int R, int KV, int NC>
__global__ void __launch_bounds__(kMmaThreads, 1)
attend_values_kernel(AttendArgs a) {
  constexpr bool kCheck = NC != 256;
  extern __shared__ __align__(16) unsigned char smem[];
  const int Nc = NC ? NC : a.n_codes;
  const int G = a.q_heads / KV;
  constexpr int kWpk = kMmaWarps / KV;               // warps per KV head
  using SL = StageLayout<R, KV>;
  uint4* cbv = reinterpret_cast<uint4*>(smem);
  uint8_t* stage_buf = reinterpret_cast<uint8_t*>(cbv + 32 * Nc);
  constexpr int kStageBytes = SL::kBytes;
  const int score_stage_bytes = kTiles * a.q_heads * 16 * 4;   // 8 tiles x Hq x 16 floats
  uint8_t* score_buf = stage_buf + 2 * kStageBytes;
  float* xred = reinterpret_cast<float*>(stage_buf);  // reused after the loop: [warps][32][33]

  const int s = blockIdx.x, b = blockIdx.y, S = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, i = lane & 3;
  const int kv = warp / kWpk, sub = warp % kWpk;
  int64_t row0, t_begin, t_end;
  split_range(a, b, s, S, row0, t_begin, t_end);
  Partial* part = a.partials + static_cast<int64_t>(b) * a.q_heads * S + s;

  if (t_begin >= t_end) {
    for (int e = tid; e < a.q_heads * (kD + 1); e += kMmaThreads) {
      const int h = e / (kD + 1), d = e % (kD + 1);
      if (d < kD)
        part[static_cast<int64_t>(h) * S].o[d] = 0.0f;
      else
        part[static_cast<int64_t>(h) * S].l = 0.0f;
    }
    return;
  }

  const int64_t n_tiles = (a.max_T + kTileT - 1) / kTileT;
  // the stage's tile-blocked scores: whole tiles, contiguous, 16-byte pieces
  auto issue_scores = [&](uint8_t* dst, int64_t t0) {
    const int64_t tau0 = t0 / kTileT;
    const int64_t tau1 = (min(t_end, t0 + kStageT) + kTileT - 1) / kTileT;
    const int pieces = static_cast<int>((tau1 - tau0) * a.q_heads * 4);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(
        a.scores + score_index(b, tau0, 0, 0, 0, 0, n_tiles, KV, G));
    for (int p = tid; p < pieces; p += kMmaThreads) cp_async16(dst + p * 16, src + p * 16);
  };
  for (int p = tid; p < 32 * Nc; p += kMmaThreads) cp_async16(cbv + p, a.v_img + p);
  cp_async_commit();
  issue_stage<R, KV>(stage_buf, a.v_codes, row0, t_begin, t_end);
  issue_scores(score_buf, t_begin);
  cp_async_commit();

  const float m_h = (g < G) ? part[static_cast<int64_t>(kv * G + g) * S].m : 0.0f;
  float O[8][4];
#pragma unroll
  for (int m = 0; m < 8; ++m) O[m][0] = O[m][1] = O[m][2] = O[m][3] = 0.0f;
  float lsum = 0.0f;
  int err = 0;
  const int odd = i & 1, vsel = (i >> 1) & 1;
  int stage = 0;
  // Per-thread constants. Lane i reads group jA = 2g + (i & 1) before jB = 2g + 1 - (i & 1)
  // and image half vsel = (i >> 1) before the other, so each 8-lane phase of a gather hits 8
  // bank groups; odd lanes swap the sums back. gA[x], gB[x]: byte offset of entry 0 of jA/jB
  // in the x-th half read; cw_off[k][x]: offset of the code word (groups 2g, 2g+1) of
  // position tau[k] in a tile, for the round read x-th.
  const int jA = 2 * g + odd, jB = 2 * g + (odd ^ 1);
  const uint32_t selA = byte_sel(jA & 3), selB = byte_sel(jB & 3);
  uint32_t gA[R], gB[R], cw_off[4][R];
#pragma unroll
  for (int x = 0; x < R; ++x) {
    gA[x] = static_cast<uint32_t>(slot(vsel ^ x, jA, 0, Nc)) * 16;
    gB[x] = static_cast<uint32_t>(slot(vsel ^ x, jB, 0, Nc)) * 16;
  }
  {
    const int tau4[4] = {2 * i, 2 * i + 1, 2 * i + 8, 2 * i + 9};
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int x = 0; x < R; ++x) {
        const int r = (R == 2) ? (vsel ^ x) : 0;
        cw_off[k][x] = static_cast<uint32_t>(SL::offset(tau4[k], kv * R + r) + 4 * (g >> 1));
      }
  }

  for (int64_t t0 = t_begin; t0 < t_end; t0 += kStageT, stage ^= 1) {
    if (t0 + kStageT < t_end) {
      issue_stage<R, KV>(stage_buf + (stage ^ 1) * kStageBytes, a.v_codes, row0, t0 + kStageT, t_end);
      issue_scores(score_buf + (stage ^ 1) * score_stage_bytes, t0 + kStageT);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sb = static_cast<uint32_t>(stage_buf - smem) + stage * kStageBytes;
    const float* ssc = reinterpret_cast<const float*>(score_buf + stage * score_stage_bytes);

    for (int tile = sub; tile < kTiles; tile += kWpk) {
      const int64_t tt0 = t0 + tile * kTileT;
      if (tt0 >= t_end) break;
      const int rem = static_cast<int>(min(static_cast<int64_t>(kTileT), t_end - tt0));  // valid positions
      // probabilities of this thread's 4 positions for head column g
      const int tau[4] = {2 * i, 2 * i + 1, 2 * i + 8, 2 * i + 9};
      float p[4] = {0.f, 0.f, 0.f, 0.f};
      if (g < G) {
        const float4 sv = *reinterpret_cast<const float4*>(ssc + (((tile * KV + kv) * G + g) * 4 + i) * 4);
        const float sk[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (tau[k] < rem) p[k] = exp2f(sk[k] - m_h);
          lsum += p[k];
        }
      }
      const uint32_t b0 = h2_as_u32(__floats2half2_rn(p[0], p[1]));
      const uint32_t b1 = h2_as_u32(__floats2half2_rn(p[2], p[3]));

      // A fragments of the 8 m-tiles: row g = dim 16g+m (group 2g, element m), row g+8 = dim
      // 16g+8+m (group 2g+1, element m); register 2*pr (+1) holds positions of pair pr
      // ((2i, 2i+1) or (2i+8, 2i+9)) for row g (g+8).
      const uint32_t sbt = sb + tile * kTileT * SL::kPieces * 16;
      uint32_t A[8][4];
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        uint4 E0[2], E1[2];   // decoded groups 2g and 2g+1 of the pair's two positions
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          const int k = 2 * pr + k2;
          const bool valid = tau[k] < rem;
          // the code word of groups 2g, 2g+1; with two rounds, round vsel first
          const uint32_t w0 = valid ? lds32(smem, sbt + cw_off[k][0]) : 0u;
          int cA0 = static_cast<int>(take_byte(w0, selA)), cB0 = static_cast<int>(take_byte(w0, selB));
          if (kCheck) {
            cA0 = clamp_code(cA0, Nc, err);
            cB0 = clamp_code(cB0, Nc, err);
          }
          uint4 SA = lds128(smem, gA[0] + (cA0 << 7));
          uint4 SB = lds128(smem, gB[0] + (cB0 << 7));
          if (R == 2) {
            const uint32_t w1 = valid ? lds32(smem, sbt + cw_off[k][R - 1]) : 0u;
            int cA1 = static_cast<int>(take_byte(w1, selA)), cB1 = static_cast<int>(take_byte(w1, selB));
            if (kCheck) {
              cA1 = clamp_code(cA1, Nc, err);
              cB1 = clamp_code(cB1, Nc, err);
            }
            SA = hadd2x4(SA, lds128(smem, gA[R - 1] + (cA1 << 7)));
            SB = hadd2x4(SB, lds128(smem, gB[R - 1] + (cB1 << 7)));
          }
          E0[k2] = odd ? SB : SA;
          E1[k2] = odd ? SA : SB;
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const unsigned sel = (m & 1) ? 0x7632u : 0x5410u;
          A[m][2 * pr] = __byte_perm(word(E0[0], m >> 1), word(E0[1], m >> 1), sel);
          A[m][2 * pr + 1] = __byte_perm(word(E1[0], m >> 1), word(E1[1], m >> 1), sel);
        }
      }
#pragma unroll
      for (int m = 0; m < 8; ++m) mma16816(O[m], A[m][0], A[m][1], A[m][2], A[m][3], b0, b1);
    }
    __syncthreads();
  }

  // l: sum over the quad (lanes with equal g hold the same head column)
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);

  // Warps of one KV head add their accumulators (fixed order) through shared memory.
  if (kWpk > 1) {
    cp_async_wait<0>();
    float* mine = xred + (warp * 32 + lane) * 33;
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int c = 0; c < 4; ++c) mine[m * 4 + c] = O[m][c];
    mine[32] = lsum;
    __syncthreads();
    if (sub == 0) {
      for (int w = 1; w < kWpk; ++w) {
        const float* other = xred + ((warp + w) * 32 + lane) * 33;
#pragma unroll
        for (int m = 0; m < 8; ++m)
#pragma unroll
          for (int c = 0; c < 4; ++c) O[m][c] += other[m * 4 + c];
        lsum += other[32];
      }
    }
  }
  if (sub == 0) {
    // C fragment of m-tile m: (row g, cols 2i, 2i+1) = dim 16g+m; (row g+8, ...) = dim 16g+8+m.
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int col = 2 * i + c;
      if (col >= G) continue;
      Partial* ph = part + static_cast<int64_t>(kv * G + col) * S;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        ph->o[16 * g + m] = O[m][c];
        ph->o[16 * g + 8 + m] = O[m][2 + c];
      }
    }
    // l of head column g lives in every lane of quad g
    if (i == 0 && g < G) part[static_cast<int64_t>(kv * G + g) * S].l = lsum;
  }
  if (kCheck) {
    err = __syncthreads_or(err);
    if (err && tid == 0) atomicOr(a.error_word, kErrCodeRange);
  }
}

template <int R, int KV, int NC>
commvq_status launch_mma_rk(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st) {
  const size_t smem_s = mma_scores_smem_bytes(R, KV, a.n_codes);
  const size_t smem_v = mma_values_smem_bytes(R, KV, a.q_heads, a.n_codes);
  dim3 grid(S, a.B);
  {
    const int n = 2 * kGroups * a.n_codes;
    int bx = max((n + kThreads - 1) / kThreads, (kPhaseRows * (kD / 2) + kThreads - 1) / kThreads);
    bx = max(bx, (a.B * a.kv_heads * 256 + kThreads - 1) / kThreads);
    bx = max(bx, (a.B * S * (kD / 2) + kThreads - 1) / kThreads);
    prep_kernel<<<dim3(bx, 5), kThreads, 0, st>>>(a, R, q, static_cast<int>(qt), S);
  }
  if (a.main_start &&
      cudaEventRecordWithFlags(static_cast<cudaEvent_t>(a.main_start), st, cudaEventRecordExternal) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
#define COMMVQ_LAUNCH_SCORES(T)                                                                      \
  {                                                                                                \
    auto k = attend_scores_kernel<R, KV, NC, T>;                                               \
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s) != cudaSuccess) \
      return COMMVQ_ERR_CUDA;                                                                      \
    k<<<grid, kMmaThreads, smem_s, st>>>(a, static_cast<const T*>(q));                             \
  }
  switch (qt) {
    case COMMVQ_F32: COMMVQ_LAUNCH_SCORES(float) break;
    case COMMVQ_F16: COMMVQ_LAUNCH_SCORES(__half) break;
    case COMMVQ_BF16: COMMVQ_LAUNCH_SCORES(__nv_bfloat16) break;
    default: return COMMVQ_ERR_UNSUPPORTED;
  }
#undef COMMVQ_LAUNCH_SCORES
  {
    auto k = attend_values_kernel<R, KV, NC>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_v) != cudaSuccess)
      return COMMVQ_ERR_CUDA;
    k<<<grid, kMmaThreads, smem_v, st>>>(a);
  }
  if (a.main_stop &&
      cudaEventRecordWithFlags(static_cast<cudaEvent_t>(a.main_stop), st, cudaEventRecordExternal) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  return launch_status();
}

template <int R, int KV>
commvq_status launch_mma_r(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st) {
  if (a.n_codes == 256) return launch_mma_rk<R, KV, 256>(a, q, qt, S, st);
  return launch_mma_rk<R, KV, 0>(a, q, qt, S, st);
}

template <int R>
commvq_status launch_mma_kv(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st) {
  switch (a.kv_heads) {
    case 1: return launch_mma_r<R, 1>(a, q, qt, S, st);
    case 2: return launch_mma_r<R, 2>(a, q, qt, S, st);
    case 4: return launch_mma_r<R, 4>(a, q, qt, S, st);
    case 8: return launch_mma_r<R, 8>(a, q, qt, S, st);
    default: return COMMVQ_ERR_UNSUPPORTED;
  }
}

}  // namespace

size_t mma_scores_smem_bytes(int R, int KV, int n_codes) {
  return static_cast<size_t>(512) * n_codes + static_cast<size_t>(KV) * 8 * 32 * 8 + 64 * sizeof(float2) +
         static_cast<size_t>(kTiles) * KV * 8 * 4 + static_cast<size_t>(kTiles) * 2 * 32 * 16 +
         static_cast<size_t>(2) * kStageT * KV * R * kGroups;
}

size_t mma_values_smem_bytes(int R, int KV, int q_heads, int n_codes) {
  // code stages and score stages; after the loop the same bytes hold the per-warp partial
  // sums when several warps share a KV head
  size_t stages = static_cast<size_t>(2) * kStageT * KV * R * kGroups +
                  static_cast<size_t>(2) * kTiles * q_heads * 16 * 4;
  const size_t xred = static_cast<size_t>(kMmaWarps) * 32 * 33 * 4;
  if (KV < kMmaWarps && stages < xred) stages = xred;
  return static_cast<size_t>(512) * n_codes + stages;
}

bool mma_supported(int R, int q_heads, int kv_heads, int n_codes) {
  if (R < 1 || R > 2 || n_codes > 256) return false;
  if (kv_heads != 1 && kv_heads != 2 && kv_heads != 4 && kv_heads != 8) return false;
  if (q_heads % kv_heads || q_heads / kv_heads > 8) return false;
  return true;
}

commvq_status launch_attend_mma(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st) {
  if (a.R == 1) return launch_mma_kv<1>(a, q, qt, S, st);
  if (a.R == 2) return launch_mma_kv<2>(a, q, qt, S, st);
  return COMMVQ_ERR_UNSUPPORTED;
}

}  // namespace commvq
