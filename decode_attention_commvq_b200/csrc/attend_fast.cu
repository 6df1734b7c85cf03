// Decode attention on CommVQ codes, decode-and-rotate form: the fast kernel for layers with 2, 4
// or 8 KV heads (up to 8 query heads each), R <= 2 rounds and Nc' <= 256 entries.
//
// The attention is the one of attend_mma.cu (and of the table form): each (position, KV head)
// key is decoded once for its GQA group (exact fp32 sum over rounds of fp16 codebook entries),
// rotated by e^{i t theta_p} in fp32 -- the rotation moved onto the decoded key by the
// commuting-block property of the review's "What carries the argument" (Property 1 / Eq. 7-8) --
// and multiplied with the query heads on the tensor cores as one fp16 operand. (With the rounds
// summed exactly, one fp16 rounding of the rotated key keeps the worst head of every parity
// workload at <= 4.2e-3 against the 5e-3 bound; the two-term operand of attend_mma.cu cost a
// fifth of this kernel's instructions.) Values are decoded the same way and the softmax weights
// multiply them on the tensor cores ("If this is right": weights meet the value codes before
// the codebook multiply).
//
// What differs from attend_mma.cu is the work split, chosen to spend fewer instructions per
// (position, KV head):
//   keys   : a thread owns two positions (rows g and g + 8 of a 16-row mma tile) and 8 RoPE pairs
//            (two groups of one half of the head dimension), so every mma row is used; the
//            rotation runs in packed fp32x2; a gather's shared-memory address is one byte permute
//            of the code word; the two halves of the head dimension are done by two warps whose
//            partial scores meet in shared memory.
//   values : a thread owns 16 value dims (two groups) and four positions of a 16-position tile;
//            the round sum is one fp16x2 add per word, the transpose into mma fragments one byte
//            permute per register.
// One 512-thread CTA per SM runs both phases over its split of positions: the keys phase with the
// key codebook image (128 KB, fp16) in shared memory, then the values phase with the value image
// loaded over it, each streaming stages of code records with 16-byte asynchronous copies.
//
// Codebook image layout (per codebook, 128 KB): half h = j / 8 of the 16 groups at h * 64 KB;
// entry (v, j, c) -- v the round, or for one round a copy index -- at byte
//   (j / 8) * 65536 + c * 256 + (v * 8 + ((j % 8 + 4 v) % 8)) * 16,
// so the byte offset of an entry is (code << 8) | (slot << 4) | (half << 16): one PRMT of the code
// word with a per-thread constant. The slot's 16-byte bank group is (j % 8 + 4 v) % 8: the eight
// lanes of each quarter-warp gather eight different (round, group) slots, whatever the codes.
#include <math.h>

#include <type_traits>

#include "attend.cuh"

namespace commvq {
namespace {

constexpr int kFThreads = 512;
constexpr int kFWarps = kFThreads / 32;
constexpr int kFTile = 16;                  // positions per mma tile
constexpr int kFStageTiles = 4;
constexpr int kFStage = kFTile * kFStageTiles;   // positions per stage
constexpr int kFImgHalf = 65536;
constexpr int kFImg = 2 * kFImgHalf;
constexpr int kFRefresh = 16;               // stages between exact phasor refreshes
constexpr int kFPhaseRows = kFStage;        // rows of the offset phasor table
constexpr uint32_t kImgWaitPolls = 1u << 20;   // bound on the image copies' mbarrier wait

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

__device__ __forceinline__ uint4 hadd4(uint4 a, uint4 b) {
  uint4 r;
  r.x = h2u(__hadd2(u2h(a.x), u2h(b.x)));
  r.y = h2u(__hadd2(u2h(a.y), u2h(b.y)));
  r.z = h2u(__hadd2(u2h(a.z), u2h(b.z)));
  r.w = h2u(__hadd2(u2h(a.w), u2h(b.w)));
  return r;
}

// f32(low or high fp16 half of w) + x, one instruction (sm_100 mixed precision): with x the other
// round's entry widened to fp32, the sum of two fp16 entries is exact.
__device__ __forceinline__ float add_lo(uint32_t w, float x) {
  float d;
  asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %1;\n add.rn.f32.f16 %0, l, %2;\n}" : "=f"(d) : "r"(w), "f"(x));
  return d;
}
__device__ __forceinline__ float add_hi(uint32_t w, float x) {
  float d;
  asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %1;\n add.rn.f32.f16 %0, h, %2;\n}" : "=f"(d) : "r"(w), "f"(x));
  return d;
}

// 2^x for x <= 0 (a softmax weight relative to a maximum), the hardware approximation (relative
// error ~2^-22, far below the fp16 rounding the weight then takes).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int k) {
  return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
}

// Shared-memory loads at a byte offset from the dynamic shared array.
__device__ __forceinline__ uint4 ld16(const unsigned char* base, uint32_t off) {
  return *reinterpret_cast<const uint4*>(base + off);
}
__device__ __forceinline__ uint2 ld8(const unsigned char* base, uint32_t off) {
  return *reinterpret_cast<const uint2*>(base + off);
}
__device__ __forceinline__ uint32_t ld4(const unsigned char* base, uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(base + off);
}

// Image slot byte (within a code's 256-byte row) of round / copy v and group j.
__host__ __device__ __forceinline__ uint32_t img_slot(int v, int j) {
  return static_cast<uint32_t>((v * 8 + (((j & 7) + 4 * v) & 7)) * 16);
}
// Constant word of an entry address: byte 0 = slot, bytes 2-3 = image half.
__device__ __forceinline__ uint32_t img_const(int v, int j) {
  return img_slot(v, j) | (static_cast<uint32_t>(j >> 3) << 16);
}
// PRMT selector that puts byte b of the code word in bits 8..15 and keeps bytes 0, 2, 3 of the
// constant: (half << 16) | (code << 8) | slot.
__device__ __forceinline__ uint32_t img_sel(int b) { return 0x7604u | (static_cast<uint32_t>(b) << 4); }
__device__ __forceinline__ uint32_t img_addr(uint32_t code_word, uint32_t cst, uint32_t sel) {
  return __byte_perm(code_word, cst, sel);
}
// The same address with the code checked against Nc' (clamped, and recorded in err).
__device__ __forceinline__ uint32_t img_addr_checked(uint32_t code_word, int b, uint32_t cst, int Nc, int& err) {
  uint32_t c = (code_word >> (8 * b)) & 0xFFu;
  if (c >= static_cast<uint32_t>(Nc)) {
    err = 1;
    c = static_cast<uint32_t>(Nc - 1);
  }
  return cst | (c << 8);
}

// Two fp32 values to fp16x2 (low half = lo), rounded to nearest, finite values saturating at
// +-65504 (a query component outside the fp16 range cannot become inf).
__device__ __forceinline__ uint32_t pack_f16_sat(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
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

// Positions of split s of sequence b: tile-aligned pieces of ceil(T_b / S).
__device__ __forceinline__ void fast_split(const AttendArgs& a, int b, int s, int S, int64_t& row0, int64_t& t_begin,
                                           int64_t& t_end) {
  const int64_t Tb = sequence_rows(a.seq_offsets, b, a.max_T, running_error(a.error_word), row0);
  int64_t per = (Tb + S - 1) / S;
  per = (per + kFTile - 1) / kFTile * kFTile;
  t_begin = min(Tb, static_cast<int64_t>(s) * per);
  t_end = min(Tb, t_begin + per);
}

// The rows t0 .. t0 + 15 (those before t_end) of one 16-position row tile, copied by that tile's
// 128 threads (lt: the thread's index among them) into the tile's place of a stage.
template <int kRec>
__device__ __forceinline__ void fast_issue_tile(unsigned char* dst, const uint8_t* codes, int64_t row0, int64_t t0,
                                                int64_t t_end, int lt) {
  constexpr int kPieces = kRec / 16;
  const int n = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(kFTile), t_end - t0)));
  const uint8_t* src = codes + (row0 + t0) * kRec;
  for (int p = lt; p < n * kPieces; p += 4 * 32) {
    const int row = p / kPieces, piece = p - row * kPieces;
    cp_async16(dst + row * (kRec + 16) + piece * 16, src + p * 16);
  }
}

// ---------------------------------------------------------------------------------------------
// Preparation, once per codebook pair: blockIdx.y = 0 / 1 key / value image (layout above) from
// the fp32 codebooks; blockIdx.y = 2 the RoPE tables from fp64 angles: theta[p] = base^(-2p/d),
// rows[delta][p] = e^{i delta theta_p} (delta < 64), adv[p] = e^{i 64 theta_p}. It also clears the
// two error words.
__global__ void fast_prep_kernel(AttendArgs a, int R) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e == 0 && blockIdx.y == 0) a.error_word[0] = a.error_word[1] = 0;
  if (blockIdx.y == 2) {
    if (e >= kFPhaseRows * (kD / 2)) return;
    const int delta = e / (kD / 2), p = e % (kD / 2);
    const double th = pow(a.rope_base, -2.0 * p / kD);
    double sn, cs;
    sincos(static_cast<double>(delta) * th, &sn, &cs);
    float2* rows = reinterpret_cast<float2*>(const_cast<float4*>(a.rowph));
    rows[delta * (kD / 2) + p] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
    if (delta == 0) {
      const_cast<double*>(a.theta)[p] = th;
      sincos(static_cast<double>(kFStage) * th, &sn, &cs);
      reinterpret_cast<float2*>(const_cast<float4*>(a.advph))[p] =
          make_float2(static_cast<float>(cs), static_cast<float>(sn));
    }
    return;
  }
  const int Nc = a.n_codes;
  if (e >= 2 * kGroups * Nc) return;   // (v, j, c)
  const int c = e % Nc, vj = e / Nc, j = vj % kGroups, v = vj / kGroups;
  const int r = (R == 2) ? v : 0;
  const float* cb = blockIdx.y ? a.v_codebook : a.k_codebook;
  unsigned char* img = reinterpret_cast<unsigned char*>(const_cast<uint4*>(blockIdx.y ? a.v_img : a.k_img));
  float w[kG];
  load_row8(cb + ((static_cast<int64_t>(r) * kGroups + j) * Nc + c) * kG, w);
  uint4 o;
  o.x = h2u(__floats2half2_rn(w[0], w[1]));
  o.y = h2u(__floats2half2_rn(w[2], w[3]));
  o.z = h2u(__floats2half2_rn(w[4], w[5]));
  o.w = h2u(__floats2half2_rn(w[6], w[7]));
  *reinterpret_cast<uint4*>(img + (j >> 3) * kFImgHalf + c * 256 + img_slot(v, j)) = o;
}

// ---------------------------------------------------------------------------------------------
// The codebook image (the Nc' used rows of each 64 KB half) into shared memory by two bulk copies
// of the tensor memory accelerator, completing on `bar` (issued by thread 0). Then every thread
// waits for the phase of `parity`; a wait that runs out sets the wait bit of the error word and
// waits once more (bounded), so that no copy is left in flight when the CTA goes on.
__device__ __forceinline__ void image_copy_issue(unsigned char* smem, const uint4* img, int Nc, uint64_t* bar) {
  if (threadIdx.x == 0) {
    const uint32_t half = static_cast<uint32_t>(Nc) * 256u;
    mbar_arrive_expect_tx(bar, 2 * half);
    bulk_copy_g2s(smem, img, half, bar);
    bulk_copy_g2s(smem + kFImgHalf, reinterpret_cast<const unsigned char*>(img) + kFImgHalf, half, bar);
  }
}
__device__ __forceinline__ void image_copy_wait(const AttendArgs& a, uint64_t* bar, uint32_t parity) {
  if (!mbar_wait_bounded(bar, parity, kImgWaitPolls)) {
    atomicOr(running_error(a.error_word), kErrWaitLimit);
    mbar_wait_bounded(bar, parity, kImgWaitPolls);
  }
}

// ---------------------------------------------------------------------------------------------
// Keys. Warp w: row tile rt = w / 4 of each 64-position stage, half hf = (w / 2) % 2 of the head
// dimension (groups 8 hf .. 8 hf + 7), KV heads kg + 2m (kg = w % 2, m < KV / 2). Thread (g, i):
// rows g and g + 8 of the tile; local groups i and i + 4 of its half. mma k-step u (0..3) covers
// group i + 4 (u / 2), pairs A = 2 (u % 2) and B = A + 1 of that group: k-columns 2i, 2i + 1 hold
// the rotated x of pairs A, B and 2i + 8, 2i + 9 their y, the query fragments the same dims.
// A thread's phasors are packed per (row, k-step) as (pair A, pair B). The warp of half 0
// finalises the first half of its KV heads, the warp of half 1 the rest: it adds the partner's
// partial scores (shared memory, in the order half 0 + half 1), scales them to the exp2 domain,
// stores them in the score buffer and keeps their maxima.
template <int R, int KV, typename QT, bool kCheck>
__device__ __forceinline__ void keys_phase(const AttendArgs& a, const QT* __restrict__ q, unsigned char* smem,
                                           int64_t row0, int64_t t_begin, int64_t t_end, float* msplit,
                                           uint64_t* ibar) {
  constexpr int MK = KV / 2;                  // KV heads per warp
  constexpr int kFin = MK > 1 ? MK / 2 : 1;   // KV heads each warp of a pair finalises (KV = 2: half 0 only)
  constexpr int kRec = KV * R * 16;
  constexpr int kRowStride = kRec + 16;
  constexpr int kStageBytes = kFStage * kRowStride;
  unsigned char* stages = smem + kFImg;                                          // [2][64 rows][kRowStride]
  uint2* qf = reinterpret_cast<uint2*>(stages + 2 * kStageBytes);                 // [KV][2 hf][4 u][32 lanes]
  // partial scores of the non-finalising warps, [4 rt][KV][16][8]: written and read between the
  // barrier at the top of a stage and the next one, so one buffer serves every stage
  float* xbuf = reinterpret_cast<float*>(qf + KV * 2 * 4 * 32);
  float4* advt = reinterpret_cast<float4*>(xbuf + kFStageTiles * KV * 16 * 8);   // [2 hf][4 i][4 u]
  float2* basep = reinterpret_cast<float2*>(advt + 32);                          // [16 warps][32]
  float* mred = reinterpret_cast<float*>(basep + kFWarps * 32);                  // [4 rt][KV][8]

  const int Nc = kCheck ? a.n_codes : 256;
  const int G = a.q_heads / KV;
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, i = lane & 3;
  const int rt = warp >> 2, hf = (warp >> 1) & 1, kg = warp & 1;

  // Prepared state (codebook image, advance phasors) and the queries are not written by the
  // kernel this one may follow as a programmatic dependent: copy and form them before the wait.
  if (tid == 0) {
    mbar_init(ibar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  image_copy_issue(smem, a.k_img, Nc, ibar);   // rows of codes >= Nc' are never read
  // query fragments: entry (kv, hf2, u, ln) = (x of pair A, x of pair B), (y of A, y of B) of head
  // column ln / 4 (zero past G) in the key operand type
  for (int e = tid; e < KV * 2 * 4 * 32; e += kFThreads) {
    const int ln = e & 31, u = (e >> 5) & 3, hf2 = (e >> 7) & 1, kv = e >> 8;
    const int col = ln >> 2, ii = ln & 3;
    uint2 v = make_uint2(0u, 0u);
    if (col < G) {
      const QT* qh = q + (static_cast<int64_t>(b) * a.q_heads + kv * G + col) * kD;
      const int pA = 4 * (8 * hf2 + ii + 4 * (u >> 1)) + 2 * (u & 1), pB = pA + 1;
      v.x = pack_f16_sat(qget(qh, 2 * pA), qget(qh, 2 * pB));
      v.y = pack_f16_sat(qget(qh, 2 * pA + 1), qget(qh, 2 * pB + 1));
    }
    qf[e] = v;
  }
  if (tid < 32) {   // advance phasors: (cos A, cos B, sin A, sin B) of e^{i 64 theta} per (hf, i, u)
    const int hf2 = tid >> 4, ii = (tid >> 2) & 3, u = tid & 3;
    const int pA = 4 * (8 * hf2 + ii + 4 * (u >> 1)) + 2 * (u & 1);
    const float2* adv = reinterpret_cast<const float2*>(a.advph);
    const float2 cA = adv[pA], cB = adv[pA + 1];
    advt[tid] = make_float4(cA.x, cB.x, cA.y, cB.y);
  }
  pdl_wait();
  pdl_trigger();   // the merge kernel may be scheduled; it waits for this grid

  // each row tile's four warps copy and wait for their own rows (a named barrier per tile)
  fast_issue_tile<kRec>(stages + kFTile * rt * kRowStride, a.k_codes, row0, t_begin + kFTile * rt, t_end, tid & 127);
  cp_async_commit();

  // Per-thread constants. Rows of the thread in a stage, code-word offsets (round order by row
  // parity: round g % 2 first, so the two rows of a quarter-warp read different rounds), entry
  // address constants per (group i or i + 4, first or second round), phasor tables.
  const int v1 = (R == 2) ? (g & 1) : (g & 1);      // R == 1: the image copy g % 2
  const uint32_t rowoff0 = static_cast<uint32_t>((kFTile * rt + g) * kRowStride);
  const uint32_t rowoff1 = rowoff0 + 8 * kRowStride;
  const uint32_t cwoff1 = static_cast<uint32_t>(((kg * R) + ((R == 2) ? v1 : 0)) * 16 + hf * 8);
  const uint32_t cwoff2 = static_cast<uint32_t>(((kg * R) + ((R == 2) ? (v1 ^ 1) : 0)) * 16 + hf * 8);
  uint32_t kc[2][2];   // [group i / i + 4][first / second round]
#pragma unroll
  for (int gs = 0; gs < 2; ++gs) {
    kc[gs][0] = img_const(v1, 8 * hf + i + 4 * gs);
    kc[gs][1] = img_const(v1 ^ 1, 8 * hf + i + 4 * gs);
  }
  const uint32_t sel = img_sel(i);

  // phasors of the thread's two rows and four k-steps, from an exact base: e^{i t0 theta_p} (fp64
  // angle, per warp in shared memory) times e^{i delta theta_p} (prep table, fp64 angles)
  f32x2 C[2][4], Sn[2][4];
  float2* base_w = basep + warp * 32;
  auto refresh = [&](int64_t t0) {
    {
      const int p = 32 * hf + lane;   // the warp's 32 pairs
      double sn, cs;
      sincos(static_cast<double>(t0) * a.theta[p], &sn, &cs);
      base_w[lane] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
    }
    __syncwarp();
    const float2* rows = reinterpret_cast<const float2*>(a.rowph);
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int delta = kFTile * rt + g + 8 * rr;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int pA = 4 * (8 * hf + i + 4 * (u >> 1)) + 2 * (u & 1);
        float cc[2], ss[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const float2 bp = base_w[pA + k - 32 * hf];
          const float2 rp = rows[delta * (kD / 2) + pA + k];
          cc[k] = bp.x * rp.x - bp.y * rp.y;
          ss[k] = bp.x * rp.y + bp.y * rp.x;
        }
        C[rr][u] = pack2(cc[0], cc[1]);
        Sn[rr][u] = pack2(ss[0], ss[1]);
      }
    }
    __syncwarp();
  };
  refresh(t_begin);
  image_copy_wait(a, ibar, 0);

  const float scale = 1.4426950408889634f / sqrtf(static_cast<float>(kD));
  const int64_t n_tiles = (a.max_T + kFTile - 1) / kFTile;
  // Score buffer of sequence b: [tile][Hq][16 slots] floats; tile position g sits in slot
  // 4 (g / 2) + g % 2, position g + 8 two slots later. A thread finalises head columns 2i, 2i + 1
  // (those below G) of rows g, g + 8: per finalised KV head f its slots start at fo[f].
  const int tile_floats = a.q_heads * kFTile;
  float* const sc_seq = a.scores + static_cast<int64_t>(b) * n_tiles * tile_floats;
  const bool col0 = 2 * i < G, col1 = 2 * i + 1 < G;
  float mrun[kFin][2];
#pragma unroll
  for (int f = 0; f < kFin; ++f) mrun[f][0] = mrun[f][1] = -INFINITY;
  int err = 0;
  const int fin0 = hf * kFin;            // first m this warp finalises (MK == 2 kFin, or KV = 2)
  const bool fins = (MK > 1) || hf == 0;  // KV = 2: only half 0 finalises
  int fo[kFin];
#pragma unroll
  for (int f = 0; f < kFin; ++f) fo[f] = ((kg + 2 * (fin0 + f)) * G + 2 * i) * kFTile + (g >> 1) * 4 + (g & 1);

  // One stage; kFull: all its positions lie before t_end, so no row needs a check.
  auto stage_body = [&](auto full_tag, int64_t t0, int stage) {
    constexpr bool kFull = decltype(full_tag)::value;
    const int64_t tile_t0 = t0 + kFTile * rt;
    const int rows_valid =
        kFull ? kFTile : static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(kFTile), t_end - tile_t0)));
    const bool tile_live = kFull || rows_valid > 0;
    const bool valid0 = kFull || g < rows_valid, valid1 = kFull || g + 8 < rows_valid;
    const unsigned char* sb = stages + stage * kStageBytes;
    float* xb = xbuf + (rt * KV) * 16 * 8;
    float fin[kFin][4];
    if (tile_live) {
#pragma unroll
      for (int m = 0; m < MK; ++m) {
        const int kv = kg + 2 * m;
        const uint32_t mo = static_cast<uint32_t>(2 * m * R * 16);
        // code words: rows g, g + 8; first / second round; groups i (low word) and i + 4 (high word)
        uint2 cw[2][2];
        cw[0][0] = ld8(sb, rowoff0 + cwoff1 + mo);
        cw[1][0] = ld8(sb, rowoff1 + cwoff1 + mo);
        if (R == 2) {
          cw[0][1] = ld8(sb, rowoff0 + cwoff2 + mo);
          cw[1][1] = ld8(sb, rowoff1 + cwoff2 + mo);
        }
        if (kCheck && !kFull) {   // rows past the end may hold stale bytes: read them as code 0
          if (!valid0) { cw[0][0] = make_uint2(0u, 0u); cw[0][1] = make_uint2(0u, 0u); }
          if (!valid1) { cw[1][0] = make_uint2(0u, 0u); cw[1][1] = make_uint2(0u, 0u); }
        }
        const uint2* qk = qf + ((kv * 2 + hf) * 4) * 32 + lane;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int gs = 0; gs < 2; ++gs) {
          uint4 e[2], e2[2];   // rows g, g + 8: group i + 4 gs, first and second round's entries
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const uint32_t w1 = gs ? cw[rr][0].y : cw[rr][0].x;
            const uint32_t a1 = kCheck ? img_addr_checked(w1, i, kc[gs][0], Nc, err) : img_addr(w1, kc[gs][0], sel);
            e[rr] = ld16(smem, a1);
            if (R == 2) {
              const uint32_t w2 = gs ? cw[rr][1].y : cw[rr][1].x;
              const uint32_t a2 = kCheck ? img_addr_checked(w2, i, kc[gs][1], Nc, err) : img_addr(w2, kc[gs][1], sel);
              e2[rr] = ld16(smem, a2);
            }
          }
#pragma unroll
          for (int hp = 0; hp < 2; ++hp) {
            const int u = 2 * gs + hp;
            uint32_t hx[2], hy[2];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              float2 fA = __half22float2(u2h(word_of(e[rr], 2 * hp)));
              float2 fB = __half22float2(u2h(word_of(e[rr], 2 * hp + 1)));
              if (R == 2) {   // the rounds' sum in fp32 (exact): an fp16 sum would round the key
                const uint32_t vA = word_of(e2[rr], 2 * hp), vB = word_of(e2[rr], 2 * hp + 1);
                fA = make_float2(add_lo(vA, fA.x), add_hi(vA, fA.y));
                fB = make_float2(add_lo(vB, fB.x), add_hi(vB, fB.y));
              }
              const f32x2 X = pack2(fA.x, fB.x), Y = pack2(fA.y, fB.y);
              const f32x2 Xr = sub2(mul2(X, C[rr][u]), mul2(Y, Sn[rr][u]));
              const f32x2 Yr = fma2(X, Sn[rr][u], mul2(Y, C[rr][u]));
              float xA, xB, yA, yB;
              unpack2(Xr, xA, xB);
              unpack2(Yr, yA, yB);
              hx[rr] = h2u(__floats2half2_rn(xA, xB));
              hy[rr] = h2u(__floats2half2_rn(yA, yB));
            }
            const uint2 qb = qk[u * 32];
            mma_f16(acc, hx[0], hx[1], hy[0], hy[1], qb.x, qb.y);
          }
        }
        // acc: (row g, col 2i), (row g, col 2i + 1), (row g + 8, col 2i), (row g + 8, col 2i + 1);
        // the first kFin KV heads are finalised by the half-0 warp, the rest by the half-1 warp
        // (compile-time slots: no local memory)
        const bool mine = fins && ((m < kFin) == (hf == 0));
        if (mine) {
#pragma unroll
          for (int k = 0; k < 4; ++k) fin[m < kFin ? m : m - kFin][k] = acc[k];
        } else {
          float* xr = xb + kv * 16 * 8;
          *reinterpret_cast<float2*>(xr + g * 8 + 2 * i) = make_float2(acc[0], acc[1]);
          *reinterpret_cast<float2*>(xr + (g + 8) * 8 + 2 * i) = make_float2(acc[2], acc[3]);
        }
      }
    }
    // the two warps of a (tile, KV group) pair meet: named barrier 1 + (rt * 2 + kg)
    asm volatile("bar.sync %0, 64;\n" ::"r"(1 + rt * 2 + kg) : "memory");
    if (tile_live && fins) {
      float* dst = sc_seq + (tile_t0 >> 4) * tile_floats;
#pragma unroll
      for (int f = 0; f < kFin; ++f) {
        const int kv = kg + 2 * (fin0 + f);
        const float* xr = xb + kv * 16 * 8;
        const float2 p0 = *reinterpret_cast<const float2*>(xr + g * 8 + 2 * i);
        const float2 p1 = *reinterpret_cast<const float2*>(xr + (g + 8) * 8 + 2 * i);
        // half 0 + half 1, the same sum in either warp
        const float s00 = (hf == 0 ? fin[f][0] + p0.x : p0.x + fin[f][0]) * scale;
        const float s01 = (hf == 0 ? fin[f][1] + p0.y : p0.y + fin[f][1]) * scale;
        const float s10 = (hf == 0 ? fin[f][2] + p1.x : p1.x + fin[f][2]) * scale;
        const float s11 = (hf == 0 ? fin[f][3] + p1.y : p1.y + fin[f][3]) * scale;
        float* d = dst + fo[f];   // column 2i at d, column 2i + 1 one slot row later
        // maxima over every column (past G: zero scores, never read back)
        if (valid0) {
          if (col0) d[0] = s00;
          if (col1) d[kFTile] = s01;
          mrun[f][0] = fmaxf(mrun[f][0], s00);
          mrun[f][1] = fmaxf(mrun[f][1], s01);
        }
        if (valid1) {
          if (col0) d[2] = s10;
          if (col1) d[kFTile + 2] = s11;
          mrun[f][0] = fmaxf(mrun[f][0], s10);
          mrun[f][1] = fmaxf(mrun[f][1], s11);
        }
      }
    }
  };

  __syncthreads();   // the query fragments and phasor tables of the prologue are in place
  int stage = 0, it = 0;
  for (int64_t t0 = t_begin; t0 < t_end; t0 += kFStage, stage ^= 1, ++it) {
    cp_async_wait<0>();
    // this stage's rows of the row tile are in shared memory, and the tile's four warps are done
    // with its previous buffer (named barrier 9 + rt, 128 threads; the warps of other tiles run on)
    asm volatile("bar.sync %0, 128;\n" ::"r"(9 + rt) : "memory");
    if (t0 + kFStage < t_end)
      fast_issue_tile<kRec>(stages + (stage ^ 1) * kStageBytes + kFTile * rt * kRowStride, a.k_codes, row0,
                            t0 + kFStage + kFTile * rt, t_end, tid & 127);
    cp_async_commit();
    if (it > 0) {
      if (it % kFRefresh == 0) {
        refresh(t0);
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 d = advt[(hf * 4 + i) * 4 + u];
          const f32x2 dc = pack2(d.x, d.y), ds = pack2(d.z, d.w);
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) cmul2(C[rr][u], Sn[rr][u], dc, ds);
        }
      }
    }
    if (t0 + kFStage <= t_end)
      stage_body(std::true_type{}, t0, stage);
    else
      stage_body(std::false_type{}, t0, stage);
  }
  cp_async_wait<0>();

  // split maxima: over the 8 rows of a warp (lanes with equal i), then over the 4 row tiles
#pragma unroll
  for (int f = 0; f < kFin; ++f)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float m = mrun[f][c];
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
      mrun[f][c] = m;
    }
  if (fins && g == 0) {
#pragma unroll
    for (int f = 0; f < kFin; ++f) {
      const int kv = kg + 2 * (fin0 + f);
      mred[(rt * KV + kv) * 8 + 2 * i] = mrun[f][0];
      mred[(rt * KV + kv) * 8 + 2 * i + 1] = mrun[f][1];
    }
  }
  __syncthreads();
  // every warp is done with the key image: the value image's bulk copies start now, under the
  // rest of this phase and the values phase's set-up (the proxy fence orders the image reads
  // before the copies' writes)
  if (tid == 0) fence_async_smem();
  image_copy_issue(smem, a.v_img, Nc, ibar);
  // [KV][8] (columns past G: the max of their zero scores)
  for (int e = tid; e < KV * 8; e += kFThreads) {
    float m = -INFINITY;
#pragma unroll
    for (int r2 = 0; r2 < kFStageTiles; ++r2) m = fmaxf(m, mred[r2 * KV * 8 + e]);
    msplit[e] = m;
  }
  if (kCheck) {
    err = __syncthreads_or(err);
    if (err && tid == 0) atomicOr(running_error(a.error_word), kErrCodeRange);
  }
}

// ---------------------------------------------------------------------------------------------
// Values. O^T (128 dims x 8 head columns) += V^T (dims x 16 positions) P^T (positions x heads) per
// 16-position tile on mma.sync m16n8k16. Warps per KV head WPK = 16 / KV; warp (kv, sub) takes
// tiles sub, sub + WPK, ... of each stage. Thread (g, i) owns dims of groups 2g, 2g + 1 (m-tile m,
// row g = dim 16 g + m, row g + 8 = dim 16 g + 8 + m) and tile positions 2i, 2i + 1, 2i + 8,
// 2i + 9 (its P^T fragment). Gather n (0..3) of a position reads group 2g + ((i ^ n) & 1) of round
// ((i >> 1) ^ (n >> 1)) & 1, so the lanes of a quarter-warp read eight different (round, group)
// slots; lanes with odd i swap the two group sums back.
template <int R, int KV, bool kCheck>
__device__ __forceinline__ void values_phase(const AttendArgs& a, unsigned char* smem, int64_t row0, int64_t t_begin,
                                             int64_t t_end, Partial* part, const float* msplit, uint64_t* ibar) {
  constexpr int WPK = kFWarps / KV;
  constexpr int kTiles = WPK > kFStageTiles ? WPK : kFStageTiles;
  constexpr int kStageT = kFTile * kTiles;
  constexpr int kRec = KV * R * 16;
  constexpr int kRowStride = kRec + 16;
  constexpr int kStageBytes = kStageT * kRowStride;
  unsigned char* stages = smem + kFImg;                       // [2][kStageT][kRowStride]
  unsigned char* sstage = stages + 2 * kStageBytes;            // [2][kTiles][Hq][16] floats

  const int Nc = kCheck ? a.n_codes : 256;
  const int G = a.q_heads / KV;
  const int b = blockIdx.y, S = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, i = lane & 3;
  const int kv = warp / WPK, sub = warp % WPK;
  const int64_t n_tiles = (a.max_T + kFTile - 1) / kFTile;
  const int tile_floats = a.q_heads * kFTile;                  // one tile of the score buffer
  const int score_stage_bytes = kTiles * tile_floats * 4;
  // the value image's bulk copies were issued at the end of the keys phase
  // The warps with the same sub (one per KV head) share their tiles' rows and score tiles: they
  // copy and wait for those alone (named barrier 1 + sub), so the WPK groups run independently.
  constexpr int kGroupThreads = KV * 32;
  const int lt = kv * 32 + lane;   // the thread's index in its group
  auto issue_group = [&](unsigned char* cdst, unsigned char* sdst, int64_t t0) {
    constexpr int kPieces = kRec / 16;
#pragma unroll
    for (int ti = 0; ti < kTiles / WPK; ++ti) {
      const int tile = sub + ti * WPK;
      const int64_t tt0 = t0 + tile * kFTile;
      const int n = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(kFTile), t_end - tt0)));
      const uint8_t* src = a.v_codes + (row0 + tt0) * kRec;
      unsigned char* d = cdst + tile * kFTile * kRowStride;
      for (int q = lt; q < n * kPieces; q += kGroupThreads) {
        const int row = q / kPieces, piece = q - row * kPieces;
        cp_async16(d + row * kRowStride + piece * 16, src + q * 16);
      }
      if (n > 0) {   // the tile's scores, written by this CTA's keys phase before the barrier
        const float* ss = a.scores + (static_cast<int64_t>(b) * n_tiles + tt0 / kFTile) * tile_floats;
        unsigned char* sd = sdst + tile * tile_floats * 4;
        for (int q = lt; q < tile_floats / 4; q += kGroupThreads) cp_async16_ca(sd + q * 16, ss + 4 * q);
      }
    }
  };
  issue_group(stages, sstage, t_begin);
  cp_async_commit();

  // head column g of this warp's KV head; a column past G reads column G - 1 (finite weights in an
  // mma column that is never written out)
  const int gc = min(g, G - 1);
  const float m_h = msplit[kv * 8 + gc];
  const int sc_off = (kv * G + gc) * kFTile + 4 * i;   // the thread's 4 slots in a score tile
  float O[8][4];
#pragma unroll
  for (int m = 0; m < 8; ++m) O[m][0] = O[m][1] = O[m][2] = O[m][3] = 0.0f;
  float lsum = 0.0f;
  int err = 0;
  const int odd = i & 1;
  // gather n's address constant and code-byte selector; code-word offsets of the first / second
  // round read by this lane (round (i >> 1) & 1 first) for the tile positions 2i, 2i+1, 2i+8, 2i+9
  uint32_t vc[4];
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    const int j = 2 * g + ((i ^ n) & 1);
    const int v = (R == 2) ? (((i >> 1) ^ (n >> 1)) & 1) : ((i >> 1) & 1);
    vc[n] = img_const(v, j);
  }
  const uint32_t vs0 = img_sel((2 * g + (i & 1)) & 3), vs1 = img_sel((2 * g + ((i ^ 1) & 1)) & 3);
  const int rfirst = (R == 2) ? ((i >> 1) & 1) : 0;
  // code-word offsets of tile position 2i (the others at + 1, 8, 9 rows)
  const uint32_t cwo0 = static_cast<uint32_t>(2 * i * kRowStride + (kv * R + rfirst) * 16 + (g >> 1) * 4);
  const uint32_t cwo1 = static_cast<uint32_t>(2 * i * kRowStride + (kv * R + (rfirst ^ 1)) * 16 + (g >> 1) * 4);
  constexpr int kTauOff[4] = {0, 1, 8, 9};

  // One 16-position tile; kFull: all 16 positions lie before t_end (rem is then 16).
  auto tile_body = [&](auto full_tag, int tile, const unsigned char* sb, const float* ssc, int rem) {
    constexpr bool kFull = decltype(full_tag)::value;
    const float4 sv = *reinterpret_cast<const float4*>(ssc + tile * tile_floats + sc_off);
    float p[4] = {ex2(sv.x - m_h), ex2(sv.y - m_h), ex2(sv.z - m_h), ex2(sv.w - m_h)};
    if (!kFull) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (2 * i + kTauOff[k] >= rem) p[k] = 0.0f;   // past the end: stale slots
    }
    lsum += (p[0] + p[1]) + (p[2] + p[3]);
    const uint32_t b0 = h2u(__floats2half2_rn(p[0], p[1]));
    const uint32_t b1 = h2u(__floats2half2_rn(p[2], p[3]));
    const uint32_t tb = static_cast<uint32_t>(tile * kFTile * kRowStride);
    uint4 E[4][2];   // [position k][group 2g, 2g + 1]
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t w0 = ld4(sb, tb + cwo0 + kTauOff[k] * kRowStride);
      uint32_t w1 = (R == 2) ? ld4(sb, tb + cwo1 + kTauOff[k] * kRowStride) : 0u;
      if (kCheck && !kFull && 2 * i + kTauOff[k] >= rem) w0 = w1 = 0u;   // stale bytes read as code 0
      uint4 sA, sB;
      // gathers n = 0, 1 use the first round's word, n = 2, 3 the second's
      const uint32_t a0 = kCheck ? img_addr_checked(w0, (2 * g + (i & 1)) & 3, vc[0], Nc, err) : img_addr(w0, vc[0], vs0);
      const uint32_t a1 = kCheck ? img_addr_checked(w0, (2 * g + ((i ^ 1) & 1)) & 3, vc[1], Nc, err) : img_addr(w0, vc[1], vs1);
      sA = ld16(smem, a0);
      sB = ld16(smem, a1);
      if (R == 2) {
        const uint32_t a2 = kCheck ? img_addr_checked(w1, (2 * g + (i & 1)) & 3, vc[2], Nc, err) : img_addr(w1, vc[2], vs0);
        const uint32_t a3 = kCheck ? img_addr_checked(w1, (2 * g + ((i ^ 1) & 1)) & 3, vc[3], Nc, err) : img_addr(w1, vc[3], vs1);
        sA = hadd4(sA, ld16(smem, a2));
        sB = hadd4(sB, ld16(smem, a3));
      }
      E[k][0] = odd ? sB : sA;
      E[k][1] = odd ? sA : sB;
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const uint32_t sl = (m & 1) ? 0x7632u : 0x5410u;
      const uint32_t A0 = __byte_perm(word_of(E[0][0], m >> 1), word_of(E[1][0], m >> 1), sl);
      const uint32_t A1 = __byte_perm(word_of(E[0][1], m >> 1), word_of(E[1][1], m >> 1), sl);
      const uint32_t A2 = __byte_perm(word_of(E[2][0], m >> 1), word_of(E[3][0], m >> 1), sl);
      const uint32_t A3 = __byte_perm(word_of(E[2][1], m >> 1), word_of(E[3][1], m >> 1), sl);
      mma_f16(O[m], A0, A1, A2, A3, b0, b1);
    }
  };

  image_copy_wait(a, ibar, 1);
  int stage = 0;
  for (int64_t t0 = t_begin; t0 < t_end; t0 += kStageT, stage ^= 1) {
    cp_async_wait<0>();
    // the group's codes and scores of this stage are in; its warps are done with the other buffers
    asm volatile("bar.sync %0, %1;\n" ::"r"(1 + sub), "r"(kGroupThreads) : "memory");
    if (t0 + kStageT < t_end)
      issue_group(stages + (stage ^ 1) * kStageBytes, sstage + (stage ^ 1) * score_stage_bytes, t0 + kStageT);
    cp_async_commit();
    const unsigned char* sb = stages + stage * kStageBytes;
    const float* ssc = reinterpret_cast<const float*>(sstage + stage * score_stage_bytes);
    if (t0 + kStageT <= t_end) {
#pragma unroll
      for (int ti = 0; ti < kTiles / WPK; ++ti) tile_body(std::true_type{}, sub + ti * WPK, sb, ssc, kFTile);
    } else {
#pragma unroll
      for (int ti = 0; ti < kTiles / WPK; ++ti) {
        const int tile = sub + ti * WPK;
        const int64_t tt0 = t0 + tile * kFTile;
        if (tt0 >= t_end) break;
        tile_body(std::false_type{}, tile, sb, ssc, static_cast<int>(min(static_cast<int64_t>(kFTile), t_end - tt0)));
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();   // every warp is done with the image: its space holds the warps' sums below

  // l: sum over the quad (lanes with equal g hold the same head column)
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
  // Each warp's O^T (8 head columns x 128 dims) goes to shared memory, [warp][col][dim'] with
  // dim' = dim + 4 (dim / 16) and a column stride of 164 floats (16-byte stores of a quarter-warp
  // hit distinct banks); then the warps of a KV head are added in a fixed order and the split's
  // partials are written with coalesced 16-byte stores.
  constexpr int kColStride = 164, kWarpStride = 8 * kColStride;
  float* obuf = reinterpret_cast<float*>(smem);
  float* lbuf = obuf + kFWarps * kWarpStride;   // [warp][8]
  {
    float* mine = obuf + warp * kWarpStride + 20 * g;
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int h8 = 0; h8 < 2; ++h8)
#pragma unroll
        for (int q4 = 0; q4 < 2; ++q4)
          *reinterpret_cast<float4*>(mine + (2 * i + c) * kColStride + 8 * h8 + 4 * q4) =
              make_float4(O[4 * q4][2 * h8 + c], O[4 * q4 + 1][2 * h8 + c], O[4 * q4 + 2][2 * h8 + c],
                          O[4 * q4 + 3][2 * h8 + c]);
    if (i == 0) lbuf[warp * 8 + g] = lsum;
  }
  __syncthreads();
  for (int e = tid; e < a.q_heads * (kD / 4); e += kFThreads) {
    const int h = e >> 5, d4 = e & 31;   // head kv * G + col, dims 4 d4 .. 4 d4 + 3
    const int hk = h / G, col = h - hk * G;
    const float* src = obuf + (hk * WPK) * kWarpStride + col * kColStride + 20 * (d4 >> 2) + 4 * (d4 & 3);
    float4 acc = *reinterpret_cast<const float4*>(src);
#pragma unroll
    for (int w = 1; w < WPK; ++w) {
      const float4 o = *reinterpret_cast<const float4*>(src + w * kWarpStride);
      acc.x += o.x;
      acc.y += o.y;
      acc.z += o.z;
      acc.w += o.w;
    }
    reinterpret_cast<float4*>(part[static_cast<int64_t>(h) * S].o)[d4] = acc;
  }
  for (int h = tid; h < a.q_heads; h += kFThreads) {
    const int hk = h / G, col = h - hk * G;
    float l = lbuf[(hk * WPK) * 8 + col];
#pragma unroll
    for (int w = 1; w < WPK; ++w) l += lbuf[(hk * WPK + w) * 8 + col];
    *reinterpret_cast<float2*>(&part[static_cast<int64_t>(h) * S].m) = make_float2(msplit[hk * 8 + col], l);
  }
  if (kCheck) {
    err = __syncthreads_or(err);
    if (err && tid == 0) atomicOr(running_error(a.error_word), kErrCodeRange);
  }
}

// One CTA per (split, sequence): the keys phase (scores of the split into the L2-resident score
// buffer, the split's maxima), then, in the same shared memory, the values phase with the split's
// own maxima -- no grid-wide dependency between the two. msplit_off: byte offset of the split
// maxima in shared memory (past both phases' buffers).
template <int R, int KV, typename QT, bool kCheck>
__global__ void __launch_bounds__(kFThreads, 1) fast_attend_kernel(AttendArgs a, const QT* __restrict__ q,
                                                                    int msplit_off) {
  extern __shared__ __align__(1024) unsigned char smem[];
  float* msplit = reinterpret_cast<float*>(smem + msplit_off);            // [KV][8]
  uint64_t* ibar = reinterpret_cast<uint64_t*>(smem + msplit_off + 64 * sizeof(float));   // image copies
  const int s = blockIdx.x, b = blockIdx.y, S = gridDim.x;
  int64_t row0, t_begin, t_end;
  fast_split(a, b, s, S, row0, t_begin, t_end);
  Partial* part = a.partials + static_cast<int64_t>(b) * a.q_heads * S + s;
  if (t_begin >= t_end) {   // an empty split: m = -inf, o = 0, l = 0
    pdl_wait();
    pdl_trigger();
    for (int e = threadIdx.x; e < a.q_heads * (kD + 2); e += kFThreads) {
      const int h = e / (kD + 2), d = e % (kD + 2);
      Partial* ph = part + static_cast<int64_t>(h) * S;
      if (d < kD)
        ph->o[d] = 0.0f;
      else if (d == kD)
        ph->l = 0.0f;
      else
        ph->m = -INFINITY;
    }
    return;
  }
  keys_phase<R, KV, QT, kCheck>(a, q, smem, row0, t_begin, t_end, msplit, ibar);
  // the score buffer rows written above are read back by this CTA's own (L1) copies: the
  // barrier makes them visible
  __syncthreads();
  values_phase<R, KV, kCheck>(a, smem, row0, t_begin, t_end, part, msplit, ibar);
}

template <int R, int KV, bool kCheck>
commvq_status launch_fast_rkc(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st,
                              bool dependent) {
  const size_t smem = fast_smem_bytes(R, KV, a.q_heads);
  const size_t smem_main = smem - 64 * sizeof(float) - 16;   // split maxima and mbarrier past both phases' buffers
  dim3 grid(S, a.B);
  if (a.main_start && record_event(a.main_start, st) != cudaSuccess) return COMMVQ_ERR_CUDA;
#define COMMVQ_FAST(QT)                                                                               \
  {                                                                                                   \
    auto k = fast_attend_kernel<R, KV, QT, kCheck>;                                                   \
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)   \
      return COMMVQ_ERR_CUDA;                                                                         \
    const QT* qq = static_cast<const QT*>(q);                                                         \
    const int off = static_cast<int>(smem_main);                                                      \
    if (dependent) {                                                                                  \
      if (launch_dependent(k, grid, dim3(kFThreads), smem, st, a, qq, off) != cudaSuccess) return COMMVQ_ERR_CUDA; \
    } else {                                                                                          \
      k<<<grid, kFThreads, smem, st>>>(a, qq, off);                                                   \
    }                                                                                                 \
  }
  switch (qt) {
    case COMMVQ_F32: COMMVQ_FAST(float) break;
    case COMMVQ_F16: COMMVQ_FAST(__half) break;
    case COMMVQ_BF16: COMMVQ_FAST(__nv_bfloat16) break;
    default: return COMMVQ_ERR_UNSUPPORTED;
  }
#undef COMMVQ_FAST
  if (a.main_stop && record_event(a.main_stop, st) != cudaSuccess) return COMMVQ_ERR_CUDA;
  return launch_status();
}

template <int R, int KV>
commvq_status launch_fast_rk(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st,
                             bool dependent) {
  if (a.n_codes == 256) return launch_fast_rkc<R, KV, false>(a, q, qt, S, st, dependent);
  return launch_fast_rkc<R, KV, true>(a, q, qt, S, st, dependent);
}

template <int R>
commvq_status launch_fast_r(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st,
                            bool dependent) {
  switch (a.kv_heads) {
    case 2: return launch_fast_rk<R, 2>(a, q, qt, S, st, dependent);
    case 4: return launch_fast_rk<R, 4>(a, q, qt, S, st, dependent);
    case 8: return launch_fast_rk<R, 8>(a, q, qt, S, st, dependent);
    default: return COMMVQ_ERR_UNSUPPORTED;
  }
}

}  // namespace

size_t fast_keys_smem_bytes(int R, int KV) {
  const size_t row = static_cast<size_t>(KV) * R * 16 + 16;
  return kFImg + 2 * kFStage * row + static_cast<size_t>(KV) * 2 * 4 * 32 * 8 +
         static_cast<size_t>(kFStageTiles) * KV * 16 * 8 * 4 + 32 * 16 + kFWarps * 32 * 8 +
         static_cast<size_t>(kFStageTiles) * KV * 8 * 4;
}

size_t fast_values_smem_bytes(int R, int KV, int q_heads) {
  const int wpk = kFWarps / KV;
  const int tiles = wpk > kFStageTiles ? wpk : kFStageTiles;
  const size_t row = static_cast<size_t>(KV) * R * 16 + 16;
  const size_t stages = static_cast<size_t>(2) * kFTile * tiles * row;
  // the warps' sums after the loop (16 x 8 x 164 floats + 16 x 8) reuse the image's space
  static_assert(kFWarps * 8 * 164 * 4 + kFWarps * 8 * 4 <= kFImg, "epilogue buffer exceeds the image");
  return kFImg + stages + static_cast<size_t>(2) * tiles * q_heads * kFTile * 4;
}

size_t fast_smem_bytes(int R, int KV, int q_heads) {
  const size_t k = fast_keys_smem_bytes(R, KV), v = fast_values_smem_bytes(R, KV, q_heads);
  return (k > v ? k : v) + 64 * sizeof(float) + 16;
}

bool fast_supported(int g, int R, int q_heads, int kv_heads, int n_codes) {
  if (g != kG || R < 1 || R > 2 || n_codes < 1 || n_codes > 256) return false;
  if (kv_heads != 2 && kv_heads != 4 && kv_heads != 8) return false;
  return q_heads % kv_heads == 0 && q_heads / kv_heads <= 8;
}

commvq_status launch_fast_prep(const AttendArgs& a, cudaStream_t st) {
  const int n = 2 * kGroups * a.n_codes;
  const int bx = max((n + kThreads - 1) / kThreads, (kFPhaseRows * (kD / 2) + kThreads - 1) / kThreads);
  fast_prep_kernel<<<dim3(bx, 3), kThreads, 0, st>>>(a, a.R);
  return launch_status();
}

commvq_status launch_attend_fast(const AttendArgs& a, const void* q, commvq_dtype qt, int S, cudaStream_t st,
                                 bool dependent) {
  if (a.R == 1) return launch_fast_r<1>(a, q, qt, S, st, dependent);
  if (a.R == 2) return launch_fast_r<2>(a, q, qt, S, st, dependent);
  return COMMVQ_ERR_UNSUPPORTED;
}

}  // namespace commvq
