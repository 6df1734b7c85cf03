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

// f32(h) - x for an fp16 value h, in one instruction (sm_100 mixed-precision subtract); exact
// when h is x rounded to fp16.
__device__ __forceinline__ float sub_h_f(__half h, float x) {
  float d;
  asm("sub.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(__half_as_ushort(h)), "f"(x));
  return d;
}

// Rotate two stored pairs (a0, b0), (a1, b1) (half2 words w0, w1) by their phasors, packed as
// c = (cos 0, cos 1), s = (sin 0, sin 1), in fp32: x = a cos - b sin, y = a sin + b cos.
// Each rotated pair leaves as two fp16 pairs: hi = (x, y) rounded (h0, h1) and the negated
// rounding error nlo = hi - (x, y) rounded (n0, n1), so hi - nlo carries x and y to about
// 2^-22 relative and a product with an fp16 query loses nothing to the fp16 operand type.
// f32(low or high fp16 half of w) + x in one instruction (sm_100 mixed precision); the sum of two
// fp16 entries is exact in fp32.
__device__ __forceinline__ float addh_lo(uint32_t w, float x) {
  float d;
  asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %1;\n add.rn.f32.f16 %0, l, %2;\n}" : "=f"(d) : "r"(w), "f"(x));
  return d;
}
__device__ __forceinline__ float addh_hi(uint32_t w, float x) {
  float d;
  asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %1;\n add.rn.f32.f16 %0, h, %2;\n}" : "=f"(d) : "r"(w), "f"(x));
  return d;
}

// kSum: the stored pairs are the sum of w0/w1 (first round) and v0/v1 (second round), formed in fp32.
template <bool kSum>
__device__ __forceinline__ void rotate_two(uint32_t w0, uint32_t w1, uint32_t v0, uint32_t v1, f32x2 c, f32x2 s,
                                           uint32_t& h0, uint32_t& h1, uint32_t& n0, uint32_t& n1) {
  float2 f0 = __half22float2(u32_as_h2(w0));
  float2 f1 = __half22float2(u32_as_h2(w1));
  if (kSum) {
    f0 = make_float2(addh_lo(v0, f0.x), addh_hi(v0, f0.y));
    f1 = make_float2(addh_lo(v1, f1.x), addh_hi(v1, f1.y));
  }
  float c0, c1, s0, s1;
  unpack2(c, c0, c1);
  unpack2(s, s0, s1);
  const float x0 = fmaf(f0.x, c0, -f0.y * s0), y0 = fmaf(f0.x, s0, f0.y * c0);
  const float x1 = fmaf(f1.x, c1, -f1.y * s1), y1 = fmaf(f1.x, s1, f1.y * c1);
  const __half2 p0 = __floats2half2_rn(x0, y0), p1 = __floats2half2_rn(x1, y1);
  h0 = h2_as_u32(p0);
  h1 = h2_as_u32(p1);
  n0 = h2_as_u32(__floats2half2_rn(sub_h_f(__low2half(p0), x0), sub_h_f(__high2half(p0), y0)));
  n1 = h2_as_u32(__floats2half2_rn(sub_h_f(__low2half(p1), x1), sub_h_f(__high2half(p1), y1)));
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
  const int64_t Tb = sequence_rows(a.seq_offsets, b, a.max_T, running_error(a.error_word), row0);
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
// Preparation (once per codebook pair; see commvq_attend_prepare). blockIdx.y = 0 / 1: key /
// value codebook image, fp32 [R][16][Nc'][8] -> fp16 slots (see the file comment).
// blockIdx.y = 2: RoPE tables, all from fp64: theta[p] = base^(-2p/d),
// row[delta][p] = e^{i delta theta_p} for the 128 rows of a stage, adv[p] = e^{i 128 theta_p}
// (one stage further).
constexpr int kPhaseRows = kStageT;

__global__ void prep_kernel(AttendArgs a, int R) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int Nc = a.n_codes;
  if (e == 0 && blockIdx.y == 0) a.error_word[0] = a.error_word[1] = 0;   // both error words start clear
  const double rope_base = a.rope_base;
  double* theta = const_cast<double*>(a.theta);
  float4* rowph = const_cast<float4*>(a.rowph);
  float4* advph = const_cast<float4*>(a.advph);
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
    put_phasor(rowph + delta * (kD / 4), p, cs, sn);
    if (delta == 0) {
      theta[p] = th;
      sincos(static_cast<double>(kStageT) * th, &sn, &cs);
      put_phasor(advph, p, cs, sn);
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
__device__ __forceinline__ uint32_t lds32(const unsigned char* smem, uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(smem + off);
}
// Byte b of w, zero-extended (one PRMT); sel = byte_sel(b).
__device__ __forceinline__ uint32_t byte_sel(int b) { return 0x4440u | static_cast<uint32_t>(b); }
__device__ __forceinline__ uint32_t take_byte(uint32_t w, uint32_t sel) { return __byte_perm(w, 0u, sel); }

// ---------------------------------------------------------------------------------------
// Scores. Warp w takes the 8 positions 8w .. 8w+7 of each 128-position stage, over all 128
// dimensions, for every KV head in turn; there is no exchange between warps. Thread
// (g = lane/4, i = lane%4) owns position row g; the mma rows 8..15 are zero (the tensor pipe
// has room to spare). Through the k-order of the mma the thread owns 16 RoPE pairs: k-step
// 2u+h covers pairs 2h and 2h+1 of group 4u+i (u = 0..3), so one 16-byte gather of group 4u+i
// fills k-steps 2u and 2u+1 of the row. The query fragments use the same k-order.
// NC: the entry count when it is 256 (compile-time; every uint8 code is valid), else 0
// (run-time count, codes checked against it).
template <int R, int KV, int NC, typename QT>
__global__ void __launch_bounds__(kMmaThreads, 1)
attend_scores_kernel(AttendArgs a, const QT* __restrict__ q) {
  constexpr bool kCheck = NC != 256;
  constexpr int kRows = 8;                                           // positions per warp and stage
  static_assert(kMmaWarps * kRows == kStageT, "stage split");
  extern __shared__ __align__(16) unsigned char smem[];
  const int Nc = NC ? NC : a.n_codes;
  const int G = a.q_heads / KV;
  uint4* cbk = reinterpret_cast<uint4*>(smem);                       // 32 * Nc slots
  uint2* qf = reinterpret_cast<uint2*>(cbk + 32 * Nc);               // [KV][8][32]
  float4* base = reinterpret_cast<float4*>(qf + KV * 8 * 32);       // [32] e^{i t0 theta_p}, packed
  float4* advs = base + 32;                                          // [32] e^{i kStageT theta_p}, packed
  float* red = reinterpret_cast<float*>(advs + 32);                  // [16 warps][KV*8]
  float4* base_all = reinterpret_cast<float4*>(red + kMmaWarps * KV * 8);   // [16 warps][32] refreshes
  uint8_t* stage_all = reinterpret_cast<uint8_t*>(base_all + kMmaWarps * 32);   // [16 warps][2][8 rows][KV R][16]
  using SL = StageLayout<R, KV>;
  // One warp's rows of one stage, each padded to at least 8 pieces of 16 bytes so that a
  // 3-bit XOR swizzle has room (see kRowSwz).
  constexpr int kRowPieces = SL::kPieces > 8 ? SL::kPieces : 8;
  constexpr int kWarpStage = kRows * kRowPieces * 16;

  const int s = blockIdx.x, b = blockIdx.y, S = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, i = lane & 3, par = g & 1;
  int64_t row0, t_begin, t_end;
  split_range(a, b, s, S, row0, t_begin, t_end);
  Partial* part = a.partials + static_cast<int64_t>(b) * a.q_heads * S + s;   // + h * S

  // The prepared codebook image and advance phasors are not written by the kernel this one may
  // be a programmatic dependent of (the previous decode step's combine): copy them first, then
  // wait for that kernel before touching anything else.
  if (t_begin < t_end) {
    for (int p = tid; p < 32 * Nc; p += kMmaThreads) cp_async16(cbk + p, a.k_img + p);
    if (tid < kD / 4) cp_async16(reinterpret_cast<uint4*>(advs) + tid, reinterpret_cast<const uint4*>(a.advph) + tid);
  }
  cp_async_commit();
  pdl_wait();
  if (t_begin >= t_end) {
    for (int h = tid; h < a.q_heads; h += kMmaThreads) part[static_cast<int64_t>(h) * S].m = -INFINITY;
    return;
  }

  pdl_trigger();   // the values kernel may take SMs as this grid's CTAs finish
  // Each warp streams its own rows: the 8 rows 8w..8w+7 of every 128-position stage, into a
  // private double buffer (XOR-swizzled pieces, as StageLayout), with no CTA barrier in the loop.
  // Piece p of warp row r sits at slot p ^ (r & kRowSwz). With two rounds a row reads piece
  // kv R + (r' ^ parity), the round order already flipped by the row's parity, so only bits 1-2
  // of the row enter the XOR; with one round all three do. Either way the 8 rows of a load fall
  // in 8 different 16-byte bank groups.
  constexpr int kRowSwz = R == 2 ? 6 : 7;
  uint8_t* wstage = stage_all + warp * 2 * kWarpStage;
  auto issue_rows = [&](int buf, int64_t t0) {
    const int64_t r0 = t0 + warp * kRows;
    const int n = static_cast<int>(min(static_cast<int64_t>(kRows), t_end - r0));
    const uint8_t* src = a.k_codes + (row0 + r0) * (SL::kPieces * 16);
    for (int p = lane; p < n * SL::kPieces; p += 32) {
      const int row = p / SL::kPieces, piece = p - row * SL::kPieces;
      cp_async16(wstage + buf * kWarpStage + (row * kRowPieces + (piece ^ (row & kRowSwz))) * 16, src + p * 16);
    }
  };
  // Set-up: the warp's first rows (the image is on its way); meanwhile the query fragments and
  // the split's base phasor are formed.
  if (t_begin + warp * kRows < t_end) issue_rows(0, t_begin);
  cp_async_commit();
  // Query fragments of this sequence in the mma k-order: entry (kv, k-step st, lane) holds, for
  // head column lane/4, the dims of pairs 2(st&1) and 2(st&1)+1 of group 4(st>>1) + lane%4, fp16.
  for (int e = tid; e < KV * 256; e += kMmaThreads) {
    const int kv = e >> 8, st = (e >> 5) & 7, ln = e & 31, gg = ln >> 2, ii = ln & 3;
    uint2 v = make_uint2(0u, 0u);
    if (gg < G) {
      const QT* qh = q + (static_cast<int64_t>(b) * a.q_heads + kv * G + gg) * kD;
      const int d0 = 8 * (4 * (st >> 1) + ii) + 4 * (st & 1);
      v.x = h2_as_u32(__floats2half2_rn(qval(qh, d0), qval(qh, d0 + 1)));
      v.y = h2_as_u32(__floats2half2_rn(qval(qh, d0 + 2), qval(qh, d0 + 3)));
    }
    qf[e] = v;
  }
  if (tid >= kD / 2 && tid < kD) {   // base phasor e^{i t_begin theta_p}, fp64 angle
    double sn, cs;
    sincos(static_cast<double>(t_begin) * a.theta[tid - kD / 2], &sn, &cs);
    put_phasor(base, tid - kD / 2, cs, sn);
  }

  // Phasors of the thread's 16 pairs at its row, packed two pairs per register pair: entry
  // qq = 2u + h holds pairs 2h, 2h+1 of group 4u+i, i.e. packed table entry 2(4u+i) + h. A
  // refresh rebuilds them exactly from the stage's base phasor (fp64 angle, in shared memory;
  // the split's first, then the warp's own) times the prep row table; in between they advance
  // by e^{i kStageT theta} per stage.
  auto quad_of = [&](int qq) { return 2 * (4 * (qq >> 1) + i) + (qq & 1); };
  f32x2 pc[8], ps[8];
  const int srow = warp * kRows + g;                                 // row within the stage
  auto load_rows = [&]() {
#pragma unroll
    for (int qq = 0; qq < 8; ++qq) load_phasor(a.rowph[srow * (kD / 4) + quad_of(qq)], pc[qq], ps[qq]);
  };
  load_rows();   // global loads in flight while the asynchronous copies land

  for (int e = tid; e < kMmaWarps * KV * 8; e += kMmaThreads) red[e] = -INFINITY;
  const int64_t n_tiles = (a.max_T + kTileT - 1) / kTileT;
  const float scale = 1.4426950408889634f / sqrtf(static_cast<float>(kD));
  int err = 0;
  int stage = 0, it = 0;
  // Byte offsets of the thread's gathers: entry c of group 4u+i lives at gF[u] + 128 c in the
  // v = par half of the image (first round / copy) and gS[u] + 128 c in the other half.
  const uint32_t sel_i = byte_sel(i);
  uint32_t gF[4], gS[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    gF[u] = static_cast<uint32_t>(slot(par, 4 * u + i, 0, Nc)) * 16;
    gS[u] = static_cast<uint32_t>(slot(par ^ 1, 4 * u + i, 0, Nc)) * 16;
  }
  // The row's record: piece kv R + r sits at 16 ((kv R + r) ^ swz), swz = g & kRowSwz.
  const int swz = g & kRowSwz;
  const uint32_t cw_lane = static_cast<uint32_t>(g * kRowPieces * 16);
  // score buffer slot of this row: 16-position tile, values-kernel quad g/2, k = (g&1) + 2 (w&1)
  const int sc_k = (g & 1) + 2 * (warp & 1);
  float* red_w = red + warp * KV * 8;

  auto times_base = [&](const float4* bt) {
#pragma unroll
    for (int qq = 0; qq < 8; ++qq) {
      f32x2 bc, bs;
      load_phasor(bt[quad_of(qq)], bc, bs);
      cmul2(pc[qq], ps[qq], bc, bs);
    }
  };
  cp_async_wait<1>();   // the image (every thread's share) is in; the warp's rows may still land
  __syncthreads();
  times_base(base);
  float4* base_w = base_all + warp * 32;

  for (int64_t t0 = t_begin; t0 + warp * kRows < t_end; t0 += kStageT, stage ^= 1, ++it) {
    if (t0 + kStageT + warp * kRows < t_end) issue_rows(stage ^ 1, t0 + kStageT);
    cp_async_commit();
    if (it > 0) {
      if (it % kRefresh == 0) {   // the warp's own refresh: fp64 angles of all 64 pairs
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          double sn, cs;
          sincos(static_cast<double>(t0) * a.theta[lane + 32 * h], &sn, &cs);
          put_phasor(base_w, lane + 32 * h, cs, sn);
        }
        __syncwarp();
        load_rows();
        times_base(base_w);
      } else {
#pragma unroll
        for (int qq = 0; qq < 8; ++qq) {
          f32x2 dc, ds;
          load_phasor(advs[quad_of(qq)], dc, ds);
          cmul2(pc[qq], ps[qq], dc, ds);
        }
      }
    }
    cp_async_wait<1>();
    __syncwarp();
    const int64_t pos = t0 + warp * kRows + g;
    {
      const bool valid = pos < t_end;
      const uint32_t cwb = static_cast<uint32_t>(wstage - smem) + stage * kWarpStage + cw_lane;
      const int64_t tau = pos / kTileT;
#pragma unroll 1
      for (int kv = 0; kv < KV; ++kv) {
        // the row's code pieces of this KV head, round `par` first (it pairs with the v = par
        // image half). With 256 entries every byte is a valid code, so rows past the end read
        // stale codes whose scores are neither stored nor counted; with fewer entries they read 0.
        uint4 cw[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int rr = (R == 2) ? (r ^ par) : r;
          const uint32_t off = cwb + static_cast<uint32_t>(((kv * R + rr) ^ swz) * 16);
          cw[r] = (kCheck && !valid) ? make_uint4(0u, 0u, 0u, 0u) : lds128(smem, off);
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};    // q . hi
        float accn[4] = {0.f, 0.f, 0.f, 0.f};   // q . nlo
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 e, e2 = make_uint4(0u, 0u, 0u, 0u);
          int c0 = static_cast<int>(take_byte(word(cw[0], u), sel_i));
          if (kCheck) c0 = clamp_code(c0, Nc, err);
          e = lds128(smem, gF[u] + (c0 << 7));
          if (R == 2) {   // the second round's entry, added in fp32 (an fp16 sum would round the key)
            int c1 = static_cast<int>(take_byte(word(cw[R - 1], u), sel_i));
            if (kCheck) c1 = clamp_code(c1, Nc, err);
            e2 = lds128(smem, gS[u] + (c1 << 7));
          }
          uint32_t h0, h2, n0, n2, h0b, h2b, n0b, n2b;
          rotate_two<R == 2>(e.x, e.y, e2.x, e2.y, pc[2 * u], ps[2 * u], h0, h2, n0, n2);
          rotate_two<R == 2>(e.z, e.w, e2.z, e2.w, pc[2 * u + 1], ps[2 * u + 1], h0b, h2b, n0b, n2b);
          const uint2 b0 = qf[(kv * 8 + 2 * u) * 32 + lane];
          const uint2 b1 = qf[(kv * 8 + 2 * u + 1) * 32 + lane];
          mma16816(acc, h0, 0u, h2, 0u, b0.x, b0.y);
          mma16816(accn, n0, 0u, n2, 0u, b0.x, b0.y);
          mma16816(acc, h0b, 0u, h2b, 0u, b1.x, b1.y);
          mma16816(accn, n0b, 0u, n2b, 0u, b1.x, b1.y);
        }
        acc[0] -= accn[0];
        acc[1] -= accn[1];
        // acc[0], acc[1]: row g, columns 2i, 2i+1 = query heads kv*G + col (rows 8..15 are zero)
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col = 2 * i + c;
          if (col >= G) continue;
          const float v = acc[c] * scale;
          if (valid) a.scores[score_index(b, tau, kv, col, g >> 1, sc_k, n_tiles, KV, G)] = v;
          if (c == 0) m0 = valid ? v : -INFINITY; else m1 = valid ? v : -INFINITY;
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
          m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
        }
        if (g == 0) {
          float* rw = red_w + kv * 8 + 2 * i;
          rw[0] = fmaxf(rw[0], m0);
          rw[1] = fmaxf(rw[1], m1);
        }
      }
    }
    __syncwarp();   // the buffer just read is refilled by the next iteration's copies
  }
  cp_async_wait<0>();
  __syncthreads();

  // split maxima: each warp kept a row of maxima; take the max over warps
  for (int e = tid; e < KV * 8; e += kMmaThreads) {
    const int kv = e >> 3, col = e & 7;
    if (col >= G) continue;
    float v = -INFINITY;
#pragma unroll
    for (int w = 0; w < kMmaWarps; ++w) v = fmaxf(v, red[w * KV * 8 + e]);
    part[static_cast<int64_t>(kv * G + col) * S].m = v;
  }
  if (kCheck) {
    err = __syncthreads_or(err);
    if (err && tid == 0) atomicOr(running_error(a.error_word), kErrCodeRange);
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
  pdl_trigger();   // the combine may be scheduled as SMs free up; it waits for this grid
  // The prologue reads only prepared state and codes; the scores kernel may still be running.
  for (int p = tid; p < 32 * Nc; p += kMmaThreads) cp_async16(cbv + p, a.v_img + p);
  cp_async_commit();
  issue_stage<R, KV>(stage_buf, a.v_codes, row0, t_begin, t_end);
  pdl_wait();      // the scores kernel's maxima and score buffer are complete from here on
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
          // the code word of groups 2g, 2g+1; with two rounds, round vsel first. (With 256
          // entries every byte is a valid code: positions past the end read stale codes and
          // weigh them by p = 0; with fewer entries they read code 0.)
          const uint32_t w0 = (kCheck && !valid) ? 0u : lds32(smem, sbt + cw_off[k][0]);
          int cA0 = static_cast<int>(take_byte(w0, selA)), cB0 = static_cast<int>(take_byte(w0, selB));
          if (kCheck) {
            cA0 = clamp_code(cA0, Nc, err);
            cB0 = clamp_code(cB0, Nc, err);
          }
          uint4 SA = lds128(smem, gA[0] + (cA0 << 7));
          uint4 SB = lds128(smem, gB[0] + (cB0 << 7));
          if (R == 2) {
            const uint32_t w1 = (kCheck && !valid) ? 0u : lds32(smem, sbt + cw_off[k][R - 1]);
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
    if (err && tid == 0) atomicOr(running_error(a.error_word), kErrCodeRange);
  }
}

template <int R, int KV, int NC>
commvq_status launch_mma_rk(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st,
                            bool with_values) {
  const size_t smem_s = mma_scores_smem_bytes(R, KV, a.n_codes);
  const size_t smem_v = mma_values_smem_bytes(R, KV, a.q_heads, a.n_codes);
  dim3 grid(S, a.B);
  if (a.main_start &&
      record_event(a.main_start, st) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
#define COMMVQ_LAUNCH_SCORES(T)                                                                      \
  {                                                                                                \
    auto k = attend_scores_kernel<R, KV, NC, T>;                                               \
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s) != cudaSuccess) \
      return COMMVQ_ERR_CUDA;                                                                      \
    if (launch_dependent(k, grid, dim3(kMmaThreads), smem_s, st, a, static_cast<const T*>(q)) != cudaSuccess) \
      return COMMVQ_ERR_CUDA;                                                                      \
  }
  switch (qt) {
    case COMMVQ_F32: COMMVQ_LAUNCH_SCORES(float) break;
    case COMMVQ_F16: COMMVQ_LAUNCH_SCORES(__half) break;
    case COMMVQ_BF16: COMMVQ_LAUNCH_SCORES(__nv_bfloat16) break;
    default: return COMMVQ_ERR_UNSUPPORTED;
  }
#undef COMMVQ_LAUNCH_SCORES
  if (!with_values) return launch_status();
  {
    auto k = attend_values_kernel<R, KV, NC>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_v) != cudaSuccess)
      return COMMVQ_ERR_CUDA;
    if (launch_dependent(k, grid, dim3(kMmaThreads), smem_v, st, a) != cudaSuccess) return COMMVQ_ERR_CUDA;
  }
  if (a.main_stop &&
      record_event(a.main_stop, st) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  return launch_status();
}

template <int R, int KV>
commvq_status launch_mma_r(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st,
                           bool with_values) {
  if (a.n_codes == 256) return launch_mma_rk<R, KV, 256>(a, q, qt, S, st, with_values);
  return launch_mma_rk<R, KV, 0>(a, q, qt, S, st, with_values);
}

template <int R>
commvq_status launch_mma_kv(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st,
                            bool with_values) {
  switch (a.kv_heads) {
    case 1: return launch_mma_r<R, 1>(a, q, qt, S, st, with_values);
    case 2: return launch_mma_r<R, 2>(a, q, qt, S, st, with_values);
    case 4: return launch_mma_r<R, 4>(a, q, qt, S, st, with_values);
    case 8: return launch_mma_r<R, 8>(a, q, qt, S, st, with_values);
    default: return COMMVQ_ERR_UNSUPPORTED;
  }
}

}  // namespace

size_t mma_scores_smem_bytes(int R, int KV, int n_codes) {
  const size_t row_pieces = KV * R > 8 ? static_cast<size_t>(KV * R) : 8;
  return static_cast<size_t>(512) * n_codes + static_cast<size_t>(KV) * 8 * 32 * 8 + 2 * 32 * sizeof(float4) +
         static_cast<size_t>(kMmaWarps) * KV * 8 * 4 + static_cast<size_t>(kMmaWarps) * 32 * sizeof(float4) +
         static_cast<size_t>(2) * kStageT * row_pieces * 16;
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

commvq_status launch_attend_prep(const AttendArgs& a, cudaStream_t st) {
  if (a.R != 1 && a.R != 2) return COMMVQ_ERR_UNSUPPORTED;
  const int n = 2 * kGroups * a.n_codes;
  const int bx = max((n + kThreads - 1) / kThreads, (kPhaseRows * (kD / 2) + kThreads - 1) / kThreads);
  prep_kernel<<<dim3(bx, 3), kThreads, 0, st>>>(a, a.R);
  return launch_status();
}

commvq_status launch_attend_mma(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st) {
  if (a.R == 1) return launch_mma_kv<1>(a, q, qt, S, st, true);
  if (a.R == 2) return launch_mma_kv<2>(a, q, qt, S, st, true);
  return COMMVQ_ERR_UNSUPPORTED;
}

commvq_status launch_attend_scores(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st) {
  if (a.R == 1) return launch_mma_kv<1>(a, q, qt, S, st, false);
  if (a.R == 2) return launch_mma_kv<2>(a, q, qt, S, st, false);
  return COMMVQ_ERR_UNSUPPORTED;
}

}  // namespace commvq
