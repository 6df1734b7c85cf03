// Decode attention with the paper's binary value code (CommVQ review, "Assumptions & free
// parameters": a value codebook of Nc rows over the whole KV dimension, Nc / d bits per scalar;
// Nc = 1024 for 1 bit and 2048 for 2 bits at d = 1024). Position t stores bits s_t in {0,1}^Nc
// and its value row, all KV heads together, is v_t = s_t^T C with C [Nc, kv_heads * 128]. Keys
// keep CommVQ's additive RoPE-commutative code and its scores kernel.
//
// Because v_t is linear in s_t, the softmax weights can be folded into the bits first:
//   out_h = (sum_t p_{h,t} s_t) C[:, slice of h's KV head] / sum_t p_{h,t}.
// After the scores kernel, four kernels:
// * weights (grid: value splits x parts x sequences): p = 2^(score - m_v) once per value split, as
//   24-bit fixed point in three 8-bit digits laid out as an MMA operand. A value split is a run
//   of whole splits of the scores kernel, so m_v is the maximum of their maxima and p <= 1.
// * accumulate (grid: value splits x 256-bit slices x sequences): the per-split sums
//   H_v^T[n, h] = sum_t s_t[n] p_{h,t} with tcgen05 kind::i8 MMAs and exact int32 sums: A = the
//   bits of 128 codebook rows (M) for 32 positions (K) as bytes 0 / 1 in tensor memory, B = one
//   digit plane of the weights of all 32 query-head columns (N) in shared memory, D in tensor
//   memory.
// * merge and contract (grid: KV heads x 64-row chunks of C): the splits' H merged with
//   log-sum-exp weights and contracted with the chunk of C.
// * finalize (grid: sequences x query heads): the chunks summed in order and divided by the
//   softmax sum.
#include <math.h>

#include "attend.cuh"

namespace commvq {
namespace {

constexpr int kBvThreads = 512;   // 16 warps
constexpr int kBvBitsPerCta = 256;                              // two M = 128 halves
constexpr int kBvSliceBytes = kBvBitsPerCta / 8;                // 32
constexpr int kBvMaxHeads = 32;
constexpr int kBvTile = 16;       // positions per MMA K step (one tile of the scores buffer)
constexpr int kBvMaxSplits = 64;
constexpr int kBvCRows = 64;                       // rows of C per merge-and-contract CTA
constexpr int kBvMaxG = 8;

struct BinvArgs {
  const float* scores;        // the scores kernel's exp2-domain scores, tile-blocked
  const Partial* partials;    // the scores kernel's per-split maxima (m)
  const int64_t* seq_offsets;
  const uint8_t* bits;        // [total_T, Nc / 8]
  const float* C;             // [Nc, KV * 128]
  unsigned char* wts;         // [B][n_tiles] 1.5 KB blocks: weight digits, the MMA's B layout
  float* mvec;                // [B][Sv][Hq] value-split maxima m_v
  float* lpart;               // [B][Sv][P][Hq] partial sums of the weights
  float* hpart;               // [B][Sv][Hq][Nc]
  float* opart;               // [B][Hq][Nc / kBvCRows][128]
  float2* ml;                 // [B][Hq] (M, L)
  float* out;
  float* lse;
  int* error_word;
  int64_t max_T, n_tiles;
  int B, Hq, KV, Nc, S, K, Sv, P;   // S scores splits, K of them per value split, Sv value splits,
                                    // P weight-kernel parts per value split
};

// C chunk, split weights, merged H, the second half's contraction, split maxima and sums
constexpr size_t kBvMcSmem =
    (kBvCRows * kD + kBvMaxG * kBvMaxSplits + kBvMaxG * kBvCRows + kBvMaxG * kD + 2 * kBvMaxG * kBvMaxSplits) * 4;

// Value split v of sequence b: scores splits vK .. vK + K - 1 (the same tile-aligned pieces of
// ceil(T_b / S) positions).
__device__ __forceinline__ void bv_split(const BinvArgs& a, int b, int v, int64_t& row0, int64_t& t_begin,
                                         int64_t& t_end) {
  const int64_t Tb = sequence_rows(a.seq_offsets, b, a.max_T, running_error(a.error_word), row0);
  int64_t per = (Tb + a.S - 1) / a.S;
  per = (per + kBvTile - 1) / kBvTile * kBvTile;
  t_begin = min(Tb, static_cast<int64_t>(v) * a.K * per);
  t_end = min(Tb, t_begin + a.K * per);
}

__device__ __forceinline__ void cp_async16_z(void* smem_dst, const void* gmem_src, bool valid) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem_src), "r"(valid ? 16 : 0)
               : "memory");
}


// ---------------------------------------------------------------------------------------
// tcgen05 pieces (PTX ISA 8.6, sm_100a): TMEM allocation, loads and stores, the f16 MMA with its
// A operand in TMEM and B in shared memory, completion through an mbarrier.

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}
// D[128 x N] (+)= A[128 x 32] (TMEM, unsigned 8-bit) * B[32 x N] (shared memory descriptor,
// unsigned 8-bit), int32 D.
__device__ __forceinline__ void umma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}

// Instruction descriptor, kind::i8: D int32 (bits 4-5 = 2), A and B unsigned 8-bit (formats 0),
// both K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kBvIdesc = (2u << 4) | ((32u >> 3) << 17) | ((128u >> 4) << 24);
// Shared-memory descriptor of a K-major, unswizzled operand: 8-row x 16-byte core matrices,
// LBO = byte step between the two 16-byte K halves, SBO = byte step between 8-row groups,
// version 1 at bits 46-47.
__device__ __forceinline__ uint64_t smem_desc_k(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Weights as 24-bit fixed point q = round(p (2^24 - 1)) in three 8-bit digits (most significant
// first): the MMA sums s_t[n] x digit exactly in int32 (at most 2^8 x positions per split), and
// H = (D0 2^16 + D1 2^8 + D2) / (2^24 - 1) carries each weight to 2^-25 absolute, as good as
// fp16 down to 2^-14 and better below.
constexpr float kBvQScale = 16777215.0f;
constexpr int kBvDigits = 3;
constexpr int kBvWTile = kBvDigits * 512;   // weight bytes per 16-position tile
constexpr int kBvCols = 512;       // TMEM columns: D (2 halves x 3 digits x 32), A (2 buffers x 2 halves x 32)
constexpr int kBvColA = 2 * kBvDigits * 32;
constexpr int kBvCk = 128;         // positions per chunk (4 MMA K steps of 32)
constexpr int kBvStep = 32;
constexpr int kBvRing = 6;         // chunk stages in shared memory
constexpr int kBvDist = 3;         // chunks in flight ahead of the one being expanded
constexpr uint32_t kBvWaitPolls = 1u << 20;
constexpr int kBvPlane = kBvCk * 16;                                      // one 16-byte half of every slice
constexpr int kBvStageBytes = 2 * kBvPlane + (kBvCk / kBvTile) * kBvWTile;   // bits + 8 weight tiles
constexpr size_t kBvTcSmem = static_cast<size_t>(kBvRing) * kBvStageBytes + kBvRing * 8 + 16;

// Weights once per value split: p = 2^(score - m_v), its three digits in 1.5 KB blocks per
// 16-position tile laid out as the MMA's B operand (digit d, head h, position k of the tile at
// d 512 + (h / 8) 128 + (h % 8) 16 + k; heads >= Hq and positions past the sequence are 0), the
// split's maxima, and fp32 partial sums of p per part. Grid: value splits x parts x sequences;
// thread (h, j) takes positions 2j, 2j + 1 of each tile of its part.
__global__ void __launch_bounds__(256) binv_weights_kernel(BinvArgs a) {
  __shared__ float mrow[kBvMaxHeads];
  const int v = blockIdx.x, part = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, h = tid >> 3, j = tid & 7;
  int64_t row0, t_begin, t_end;
  bv_split(a, b, v, row0, t_begin, t_end);
  const int64_t n_tl = (t_end - t_begin + kBvTile - 1) / kBvTile;
  const int64_t per = (n_tl + a.P - 1) / a.P;
  const int64_t tl0 = min(n_tl, part * per), tl1 = min(n_tl, tl0 + per);
  pdl_wait();
  {   // the split's maximum per head: the maxima of its K scores splits (8 lanes per head)
    float m = -INFINITY;
    if (h < a.Hq) {
      const Partial* ph = a.partials + (static_cast<int64_t>(b) * a.Hq + h) * a.S;
      for (int s = v * a.K + j; s < min(a.S, (v + 1) * a.K); s += 8) m = fmaxf(m, ph[s].m);
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (j == 0) mrow[h] = m;
  }
  __syncthreads();
  const float m = mrow[h];
  // the scores buffer holds position tau of a tile at ((tau % 8) / 2) 4 + tau % 2 + 2 (tau / 8):
  // positions 2j and 2j + 1 are neighbours
  const int slot0 = (j & 3) * 4 + 2 * (j >> 2);
  const uint32_t woff = static_cast<uint32_t>((h >> 3) * 128 + (h & 7) * 16 + 2 * j);
  float lsum = 0.0f;
  const float* sbase = a.scores + (static_cast<int64_t>(b) * a.n_tiles + t_begin / kBvTile) * a.Hq * kBvTile +
                       h * kBvTile + slot0;
  unsigned char* wbase = a.wts + (static_cast<int64_t>(b) * a.n_tiles + t_begin / kBvTile) * kBvWTile + woff;
  for (int64_t tl = tl0; tl < tl1; tl += 4) {   // four tiles' loads in flight
    float2 f[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      f[u] = (h < a.Hq && tl + u < tl1)
                 ? *reinterpret_cast<const float2*>(sbase + (tl + u) * a.Hq * kBvTile)
                 : make_float2(0.0f, 0.0f);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (tl + u >= tl1) break;
      const int64_t t0 = t_begin + (tl + u) * kBvTile;
      const bool hv = h < a.Hq;
      const float p0 = (hv && t0 + 2 * j < t_end) ? exp2f(f[u].x - m) : 0.0f;
      const float p1 = (hv && t0 + 2 * j + 1 < t_end) ? exp2f(f[u].y - m) : 0.0f;
      lsum += p0 + p1;
      const uint32_t q0 = __float2uint_rn(p0 * kBvQScale), q1 = __float2uint_rn(p1 * kBvQScale);
      unsigned char* w = wbase + (tl + u) * kBvWTile;
#pragma unroll
      for (int d = 0; d < kBvDigits; ++d) {
        const int sh = 8 * (kBvDigits - 1 - d);
        *reinterpret_cast<uint16_t*>(w + d * 512) =
            static_cast<uint16_t>(((q0 >> sh) & 0xFFu) | (((q1 >> sh) & 0xFFu) << 8));
      }
    }
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  if (j == 0 && h < a.Hq) {
    a.lpart[((static_cast<int64_t>(b) * a.Sv + v) * a.P + part) * a.Hq + h] = lsum;
    if (part == 0) a.mvec[(static_cast<int64_t>(b) * a.Sv + v) * a.Hq + h] = m;
  }
}

// 32 x 32 bit transpose across a warp: lane p holds w with bit l = row l at position p; returns,
// in lane l, the word whose bit p = row l at position p. Five butterfly exchanges; at block size
// jj a lane keeps its own half of every 2jj-bit block and takes the partner's other half, moved
// by a rotation (left by jj in the lower lane, right by jj in the upper).
struct BitTranspose {
  uint32_t keep[5], rot[5];
  __device__ __forceinline__ explicit BitTranspose(int lane) {
    const uint32_t masks[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      const int jj = 16 >> k;
      keep[k] = (lane & jj) ? ~masks[k] : masks[k];
      rot[k] = (lane & jj) ? 32u - jj : static_cast<uint32_t>(jj);
    }
  }
  __device__ __forceinline__ uint32_t operator()(uint32_t x) const {
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      const uint32_t t = __shfl_xor_sync(0xffffffffu, x, 16 >> k);
      const uint32_t u = __funnelshift_l(t, t, rot[k]);
      x = (x & keep[k]) | (u & ~keep[k]);
    }
    return x;
  }
};

// H_v^T[n, h] = sum_t s_t[n] q_{h,t} for the CTA's 256 codebook rows (two M = 128 halves) and 32
// head columns on tcgen05 (kind::i8, exact int32 sums). Per 128-position chunk: cp.async brings
// the bits and the weight tiles into a ring stage; each warp turns two 32-position x 32-row bit
// blocks (its TMEM lane quarter) into bytes 0 / 1 through a warp bit transpose and a nibble
// spread, and stores them into TMEM (A). 24 MMAs per chunk (4 steps x 2 halves x 3 digits),
// spread over four issuing warps, take their B operand (a digit plane) from the stage; each
// issuing warp commits its MMAs to the stage's mbarrier. The wait for chunk c - 2 before chunk
// c's stores frees both the A buffer and the stage that chunk c + 3 is copied into. One CTA
// barrier per chunk.
__global__ void __launch_bounds__(kBvThreads, 1) binv_accumulate_kernel(BinvArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* ring = smem;                                                     // [kBvRing][stage]
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + kBvRing * kBvStageBytes);   // [kBvRing]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(mbar + kBvRing);

  const int v = blockIdx.x, slice = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t row0, t_begin, t_end;
  bv_split(a, b, v, row0, t_begin, t_end);
  const int len = static_cast<int>(t_end - t_begin);   // at most max_T / S * K positions
  const int n_c = (len + kBvCk - 1) / kBvCk;
  const int64_t rowb = a.Nc / 8;
  const uint8_t* bsrc = a.bits + (row0 + t_begin) * rowb + slice * kBvSliceBytes;   // the split's first row
  const unsigned char* wsrc = a.wts + (static_cast<int64_t>(b) * a.n_tiles + t_begin / kBvTile) * kBvWTile;

  if (warp == 0) {   // all of TMEM: one CTA per SM
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tslot)),
                 "r"(kBvCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {   // a chunk's four issuing warps each commit once
    for (int s = 0; s < kBvRing; ++s) mbar_init(&mbar[s], 4);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  pdl_wait();   // the weight tiles are complete from here on

  // Each thread copies two 16-byte pieces of every chunk: threads 0-255 one piece of bits
  // (position tid / 2, half tid % 2) and weight piece tid + 256, threads 256-511 weight pieces
  // tid - 256 and tid + 256 (a chunk holds 256 bit pieces and 768 weight pieces of 16 bytes).
  constexpr int kTilePieces = kBvWTile / 16;   // 96 per weight tile
  const bool bits_piece = tid < 256;
  const int w0 = bits_piece ? -1 : tid - 256, w1 = tid + 256;
  const int p_lim0 = bits_piece ? tid >> 1 : (w0 / kTilePieces) * kBvTile;   // position that must exist
  const int p_lim1 = (w1 / kTilePieces) * kBvTile;
  const uint8_t* src0 = bits_piece ? bsrc + (tid >> 1) * rowb + 16 * (tid & 1) : wsrc + 16 * w0;
  const unsigned char* src1 = wsrc + 16 * w1;
  const int64_t step0 = bits_piece ? kBvCk * rowb : (kBvCk / kBvTile) * kBvWTile;   // per chunk
  constexpr int64_t step1 = (kBvCk / kBvTile) * kBvWTile;
  const int doff0 = bits_piece ? (tid & 1) * kBvPlane + (tid >> 1) * 16 : 2 * kBvPlane + 16 * w0;
  const int doff1 = 2 * kBvPlane + 16 * w1;
  auto issue = [&](int c, int st) {   // chunk c into stage st (pieces past the split zero-filled)
    unsigned char* dst = ring + st * kBvStageBytes;
    const int pos = c * kBvCk;
    const bool ok0 = pos + p_lim0 < len, ok1 = pos + p_lim1 < len;
    cp_async16_z(dst + doff0, ok0 ? src0 + c * step0 : a.wts, ok0);
    cp_async16_z(dst + doff1, ok1 ? src1 + c * step1 : a.wts, ok1);
  };
#pragma unroll
  for (int s = 0; s < kBvDist; ++s) {
    if (s < n_c) issue(s, s);
    cp_async_commit();
  }
  tc_fence_before();
  __syncthreads();   // TMEM address
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const int quarter = warp & 3;
  const uint32_t tq = tbase + (static_cast<uint32_t>(32 * quarter) << 16);
  if (warp < 4) {   // zero the accumulators: every MMA then adds, in whatever order they run
    uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
    for (int c8 = 0; c8 < kBvColA / 8; ++c8) tmem_st8(tq + c8 * 8, z);
    tc_wait_st();
  }
  cp_async_wait<kBvDist - 1>();   // chunk 0 (this thread's pieces)
  fence_async_smem();
  tc_fence_before();
  __syncthreads();   // mbarriers, zeroed accumulators, chunk 0
  tc_fence_after();
  const BitTranspose transpose(lane);
  // this warp's two 32 x 32 bit blocks: rows hb 128 + 32 quarter + lane, positions 32 step + 0..31
  const int grp = warp >> 2;
  uint32_t lds_off[2], col_off[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int idx = grp * 2 + u, hb = idx >> 2, step = idx & 3;
    lds_off[u] = static_cast<uint32_t>(hb * kBvPlane + (kBvStep * step + lane) * 16 + 4 * quarter);
    col_off[u] = static_cast<uint32_t>(kBvColA + hb * 32 + step * 8);
  }
  // MMA issue, spread over the four warps 0, 4, 8, 12: warp 4g takes group g's units (half g / 2,
  // steps 2 (g % 2) and 2 (g % 2) + 1) for all three digits. Descriptors of stage 0; a stage,
  // step or digit moves only the start-address field (addresses stay below 2^18 bytes).
  const int ghb = grp >> 1, gs0 = 2 * (grp & 1);
  const uint64_t desc0 = smem_desc_k(smem_u32(ring + 2 * kBvPlane), kBvWTile, 128);
  bool ok = true;
  // ring positions: chunk c in stage st, chunk c - 2 in stage stw with mbarrier phase parity pw
  // (starting from chunk -2: stage kBvRing - 2, parity 1), chunk c + kBvDist in stage sti
  int st = 0, stw = kBvRing - 2, sti = kBvDist;
  uint32_t pw = 1;
  int last_issued = -1;   // the last chunk whose MMAs were issued and committed (uniform)
  for (int c = 0; c < n_c; ++c) {
    const uint32_t bbc = static_cast<uint32_t>(c & 1) * 64;
    const unsigned char* sg = ring + st * kBvStageBytes;
    if (c >= 2) {   // chunk c - 2's MMAs are done: its A buffer, and chunk c - 3's stage, are free
      ok = mbar_wait_bounded(&mbar[stw], pw, kBvWaitPolls) && ok;
      tc_fence_after();
    }
    if (c + kBvDist < n_c) issue(c + kBvDist, sti);   // into chunk c - 3's stage
    cp_async_commit();
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t x = transpose(*reinterpret_cast<const uint32_t*>(sg + lds_off[u]));
      uint32_t col[8];   // byte k of column g: position 4g + k
#pragma unroll
      for (int g = 0; g < 8; ++g) col[g] = (((x >> (4 * g)) & 0xFu) * 0x00204081u) & 0x01010101u;
      tmem_st8(tq + col_off[u] + bbc, col);
    }
    tc_wait_st();
    cp_async_wait<kBvDist - 1>();   // chunk c + 1 (this thread's pieces)
    fence_async_smem();              // cp.async writes -> the tensor cores' reads of the weights
    tc_fence_before();
    ok = __syncthreads_and(ok) != 0;   // A of chunk c stored, chunk c + 1 landed, every wait succeeded
    if (!ok) break;                    // (uniform) a wait gave up: issue nothing more
    if ((warp & 3) == 0 && lane == 0) {
      tc_fence_after();
      const uint64_t dst = desc0 + static_cast<uint64_t>((st * kBvStageBytes) >> 4);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int step = gs0 + k;
#pragma unroll
        for (int d = 0; d < kBvDigits; ++d)   // two consecutive tiles make the step's K = 32: LBO = one tile
          umma_i8_ts(tbase + (ghb * kBvDigits + d) * 32, tbase + kBvColA + bbc + ghb * 32 + step * 8,
                     dst + static_cast<uint64_t>(((2 * step) * kBvWTile + d * 512) >> 4), kBvIdesc, 1u);
      }
      umma_commit(&mbar[st]);
    }
    last_issued = c;
    st = st + 1 == kBvRing ? 0 : st + 1;
    sti = sti + 1 == kBvRing ? 0 : sti + 1;
    if (++stw == kBvRing) {
      stw = 0;
      pw ^= 1u;
    }
  }
  cp_async_wait<0>();
  // The last commit covers every MMA issued before it. It is waited for on the normal path and
  // after a give-up alike (again bounded), so that TMEM is not read or freed while MMAs of this
  // CTA may still write it. Its mbarrier phase is unambiguous: every earlier use of that stage
  // (chunk last_issued - kBvRing) was waited for before chunk last_issued was issued.
  if (last_issued >= 0) {
    const bool done = mbar_wait_bounded(&mbar[last_issued % kBvRing],
                                        static_cast<uint32_t>((last_issued / kBvRing) & 1), kBvWaitPolls);
    ok = ok && done;
  }
  tc_fence_after();
  ok = __syncthreads_and(ok) != 0;
  if (!ok && tid == 0) atomicOr(running_error(a.error_word), kErrWaitLimit);

  if (warp < 8) {   // warps 0-3: rows 0-127 (half 0), warps 4-7: rows 128-255
    const int hb = warp >> 2;
    const bool have = n_c > 0 && ok;   // uniform
    float hsum[32];
#pragma unroll
    for (int h = 0; h < 32; ++h) hsum[h] = 0.0f;
    if (have) {
#pragma unroll
      for (int d = 0; d < kBvDigits; ++d) {
        uint32_t r[32];
        tmem_ld32(tq + (hb * kBvDigits + d) * 32, r);
        tc_wait_ld();
        const float wd = d == 0 ? 65536.0f : (d == 1 ? 256.0f : 1.0f);
#pragma unroll
        for (int h = 0; h < 32; ++h) hsum[h] = fmaf(static_cast<float>(r[h]), wd, hsum[h]);
      }
    }
    const int64_t base = (static_cast<int64_t>(b) * a.Sv + v) * a.Hq;
    float* dst = a.hpart + base * a.Nc + slice * kBvBitsPerCta + hb * 128 + 32 * quarter + lane;
#pragma unroll
    for (int h = 0; h < kBvMaxHeads; ++h)
      if (h < a.Hq) dst[static_cast<int64_t>(h) * a.Nc] = hsum[h] * (1.0f / kBvQScale);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(kBvCols) : "memory");
  }
}

// One (sequence, KV head, 128-row chunk of C): merge the G heads' split sums over the chunk,
//   H[h, n] = sum_v 2^(m_v - M) H_v[h, n],  M = max_v m_v,
// and contract: opart[h, chunk, :] = sum_{n in chunk} H[h, n] C[n, kv 128 : kv 128 + 128].
// The chunk's rows of C are copied into shared memory before the wait on the previous kernel.
// The chunk-0 CTA also stores (M, L = sum_v 2^(m_v - M) l_v).
__global__ void __launch_bounds__(256) binv_merge_contract_kernel(BinvArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  float* cs = reinterpret_cast<float*>(smem);                 // [kBvCRows][128]
  float* wts = cs + kBvCRows * kD;                            // [kBvMaxG][kBvMaxSplits]
  float* hc = wts + kBvMaxG * kBvMaxSplits;                   // [kBvMaxG][kBvCRows]
  float* half_out = hc + kBvMaxG * kBvCRows;                  // [kBvMaxG][128]
  float* msplit = half_out + kBvMaxG * kD;                    // [kBvMaxG][kBvMaxSplits]
  float* lsplit = msplit + kBvMaxG * kBvMaxSplits;            // [kBvMaxG][kBvMaxSplits]
  const int bkv = blockIdx.x, chunk = blockIdx.y;
  const int b = bkv / a.KV, kv = bkv % a.KV, G = a.Hq / a.KV;
  const int tid = threadIdx.x;
  const int n0 = chunk * kBvCRows;
  const int64_t ld = static_cast<int64_t>(a.KV) * kD;
  {
    const float* src = a.C + n0 * ld + kv * kD;
    for (int e = tid; e < kBvCRows * (kD / 4); e += 256) {
      const int r = e / (kD / 4), c4 = e % (kD / 4);
      cp_async16(cs + r * kD + 4 * c4, src + r * ld + 4 * c4);
    }
    cp_async_commit();
  }
  pdl_wait();
  for (int e = tid; e < G * a.Sv; e += 256) {   // each (head, split): its maximum and weight sum
    const int h = e / a.Sv, s = e % a.Sv;
    const int64_t bs = static_cast<int64_t>(b) * a.Sv + s;
    const float* lp = a.lpart + bs * a.P * a.Hq + kv * G + h;
    float l = 0.0f;
#pragma unroll 16
    for (int q = 0; q < a.P; ++q) l += lp[static_cast<int64_t>(q) * a.Hq];
    msplit[h * kBvMaxSplits + s] = a.mvec[bs * a.Hq + kv * G + h];
    lsplit[h * kBvMaxSplits + s] = l;
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (int s = 0; s < a.Sv; ++s) M = fmaxf(M, msplit[tid * kBvMaxSplits + s]);
    float L = 0.0f;
    for (int s = 0; s < a.Sv; ++s) {
      const float w = M == -INFINITY ? 0.0f : exp2f(msplit[tid * kBvMaxSplits + s] - M);
      wts[tid * kBvMaxSplits + s] = w;
      L = fmaf(w, lsplit[tid * kBvMaxSplits + s], L);
    }
    if (chunk == 0) a.ml[static_cast<int64_t>(b) * a.Hq + kv * G + tid] = make_float2(M, L);
  }
  __syncthreads();
  // merged H of the chunk: element (h, n), n fastest (coalesced); sixteen split sums in flight
  for (int e = tid; e < G * kBvCRows; e += 256) {
    const int h = e / kBvCRows, n = e % kBvCRows;
    const float* src = a.hpart + (static_cast<int64_t>(b) * a.Sv * a.Hq + kv * G + h) * a.Nc + n0 + n;
    const int64_t step = static_cast<int64_t>(a.Hq) * a.Nc;
    const float* w = wts + h * kBvMaxSplits;
    float acc = 0.0f;
    for (int s0 = 0; s0 < a.Sv; s0 += 16) {
      float x[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) x[u] = s0 + u < a.Sv ? src[(s0 + u) * step] : 0.0f;
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (s0 + u < a.Sv) acc = fmaf(w[s0 + u], x[u], acc);
    }
    hc[h * kBvCRows + n] = acc;
  }
  cp_async_wait<0>();
  __syncthreads();
  // contraction: thread (d, half) sums 64 rows of the chunk for every head
  const int d = tid & (kD - 1), hf = tid >> 7;
  float acc[kBvMaxG];
#pragma unroll
  for (int h = 0; h < kBvMaxG; ++h) acc[h] = 0.0f;
#pragma unroll 8
  for (int n = hf * (kBvCRows / 2); n < (hf + 1) * (kBvCRows / 2); ++n) {
    const float c = cs[n * kD + d];
#pragma unroll
    for (int h = 0; h < kBvMaxG; ++h)
      if (h < G) acc[h] = fmaf(hc[h * kBvCRows + n], c, acc[h]);
  }
  if (hf == 1) {
#pragma unroll
    for (int h = 0; h < kBvMaxG; ++h)
      if (h < G) half_out[h * kD + d] = acc[h];
  }
  __syncthreads();
  if (hf == 0) {
    const int nch = a.Nc / kBvCRows;
#pragma unroll
    for (int h = 0; h < kBvMaxG; ++h)
      if (h < G)
        a.opart[((static_cast<int64_t>(b) * a.Hq + kv * G + h) * nch + chunk) * kD + d] = acc[h] + half_out[h * kD + d];
  }
}

// out[b, h, :] = sum over chunks / L; lse = (M + log2 L) ln 2 (-inf and a zero row when empty).
__global__ void __launch_bounds__(kD) binv_finalize_kernel(BinvArgs a) {
  const int bh = blockIdx.x, d = threadIdx.x;
  pdl_trigger();   // the next decode step's scores kernel may copy its codebook image meanwhile
  pdl_wait();
  if (bh == 0 && d == 0) publish_error(a.error_word);   // every kernel of the call has finished
  const int nch = a.Nc / kBvCRows;
  const float* src = a.opart + static_cast<int64_t>(bh) * nch * kD + d;
  float s = 0.0f;
  for (int c = 0; c < nch; ++c) s += src[c * kD];
  const float2 ml = a.ml[bh];
  a.out[static_cast<int64_t>(bh) * kD + d] = ml.y > 0.0f ? s / ml.y : 0.0f;
  if (a.lse && d == 0) a.lse[bh] = ml.y > 0.0f ? (ml.x + log2f(ml.y)) * 0.6931471805599453f : -INFINITY;
}

// Scores splits per value split (K) and the value split count (Sv): the smallest K with
// ceil(S / K) x slices x B CTAs within one wave of the SMs, at most kBvMaxSplits splits.
void bv_geometry(int B, int Nc, int S, int& K, int& Sv) {
  const DeviceInfo di = current_device_info();
  const int sms = di.sms > 0 ? di.sms : 148;
  const int slices = Nc / kBvBitsPerCta;
  K = 1;
  while (K < S && ((S + K - 1) / K > kBvMaxSplits ||
                   static_cast<int64_t>((S + K - 1) / K) * slices * B > sms))
    ++K;
  Sv = (S + K - 1) / K;
}

// Parts per value split in the weights kernel: about four CTAs per SM in all.
int bv_parts(int B, int Sv) {
  const DeviceInfo di = current_device_info();
  const int sms = di.sms > 0 ? di.sms : 148;
  int P = 4 * sms / (B * Sv);
  return P < 1 ? 1 : (P > 32 ? 32 : P);
}

struct BvLayout {
  size_t attend_bytes, wts_off, mvec_off, lpart_off, hpart_off, opart_off, ml_off, total;
  int S, K, Sv, P;
};

BvLayout bv_layout(const commvq_config* cfg, int Nc, int B, int64_t max_T, const commvq_attend_options* o) {
  BvLayout L{};
  L.attend_bytes = commvq_attend_workspace_bytes(cfg, B, max_T, o);
  L.S = mma_splits(B > 0 ? B : 1, cfg->q_heads, max_T);
  bv_geometry(B > 0 ? B : 1, Nc, L.S, L.K, L.Sv);
  L.P = bv_parts(B > 0 ? B : 1, L.Sv);
  const size_t n_tiles = static_cast<size_t>((max_T + kBvTile - 1) / kBvTile);
  L.wts_off = round_up(L.attend_bytes, 1024);
  L.mvec_off = round_up(L.wts_off + static_cast<size_t>(B) * n_tiles * kBvWTile, 256);
  L.lpart_off = round_up(L.mvec_off + static_cast<size_t>(B) * L.Sv * cfg->q_heads * sizeof(float), 256);
  L.hpart_off = round_up(L.lpart_off + static_cast<size_t>(B) * L.Sv * L.P * cfg->q_heads * sizeof(float), 256);
  L.opart_off = round_up(L.hpart_off + static_cast<size_t>(B) * L.Sv * cfg->q_heads * Nc * sizeof(float), 256);
  L.ml_off = round_up(L.opart_off + static_cast<size_t>(B) * cfg->q_heads * (Nc / kBvCRows) * kD * sizeof(float), 256);
  L.total = round_up(L.ml_off + static_cast<size_t>(B) * cfg->q_heads * sizeof(float2), 256);
  return L;
}

bool bv_shape_ok(const commvq_config* cfg, int Nc) {
  return Nc >= 1024 && Nc % 1024 == 0 && Nc <= 8192 && cfg->q_heads <= kBvMaxHeads && cfg->g == kG &&
         mma_supported(cfg->R, cfg->q_heads, cfg->kv_heads, cfg->n_codes);
}

}  // namespace
}  // namespace commvq

using namespace commvq;

extern "C" size_t commvq_attend_binv_workspace_bytes(const commvq_config* cfg, int32_t n_bits, int32_t B,
                                                     int64_t max_T) {
  if (!cfg || B < 0 || max_T < 0 || !bv_shape_ok(cfg, n_bits)) return 0;
  commvq_attend_options o{COMMVQ_ATTN_DECODE_MMA, 0, nullptr, nullptr, 0};
  const BvLayout L = bv_layout(cfg, n_bits, B, max_T, &o);
  return L.attend_bytes == 0 ? 0 : L.total;
}

extern "C" commvq_status commvq_attend_decode_binv(const commvq_config* cfg, const void* q, commvq_dtype q_dtype,
                                                   const void* k_codes, const uint8_t* v_bits, int32_t n_bits,
                                                   const int64_t* seq_offsets, int32_t B, int64_t max_T,
                                                   const float* k_codebook, const float* v_codebook, float* out,
                                                   float* lse, void* workspace, size_t workspace_bytes,
                                                   int32_t flags, void* stream) {
  const NvtxRange nvtx_range("commvq_attend_decode_binv");
  if (!cfg) return COMMVQ_ERR_INVALID_ARG;
  if (B < 0 || max_T < 0 || n_bits <= 0) return COMMVQ_ERR_INVALID_ARG;
  if (q_dtype != COMMVQ_F32 && q_dtype != COMMVQ_F16 && q_dtype != COMMVQ_BF16) return COMMVQ_ERR_INVALID_ARG;
  if (!bv_shape_ok(cfg, n_bits)) return COMMVQ_ERR_UNSUPPORTED;
  if (B == 0) return COMMVQ_OK;
  if (B > 65535) return COMMVQ_ERR_UNSUPPORTED;
  if (!q || !k_codes || !v_bits || !seq_offsets || !k_codebook || !v_codebook || !out || !workspace)
    return COMMVQ_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_codes, 16) || !aligned(v_bits, 16) || !aligned(k_codebook, 16) ||
      !aligned(v_codebook, 16) || !aligned(out, 16) || !aligned(lse, 4) || !aligned(seq_offsets, 8) ||
      !aligned(workspace, 256))
    return COMMVQ_ERR_INVALID_ARG;
  const size_t need = commvq_attend_binv_workspace_bytes(cfg, n_bits, B, max_T);
  if (need == 0 || workspace_bytes < need) return COMMVQ_ERR_WORKSPACE;
  const DeviceInfo di = current_device_info();
  if (di.device < 0) return COMMVQ_ERR_CUDA;
  if (mma_scores_smem_bytes(cfg->R, cfg->kv_heads, cfg->n_codes) > di.smem_optin) return COMMVQ_ERR_UNSUPPORTED;

  commvq_attend_options o{COMMVQ_ATTN_DECODE_MMA, 0, nullptr, nullptr, 0};
  const BvLayout L = bv_layout(cfg, n_bits, B, max_T, &o);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  AttendArgs a{};
  // the key side's state in the first part of the workspace (the value image is built from the
  // key codebook and not used)
  const int S = attend_mma_setup(cfg, B, max_T, ws, seq_offsets, k_codes, k_codebook, a);
  if (S != L.S) return COMMVQ_ERR_INVALID_ARG;   // the layout and the scores kernel agree on the splits
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  commvq_status rc = COMMVQ_OK;
  if (!(flags & COMMVQ_ATTEND_PREPARED)) {
    rc = launch_attend_prep(a, st);   // also clears the error words
    if (rc != COMMVQ_OK) return rc;
  }   // else: the previous call's last kernel left the running error word clear
  rc = launch_attend_scores(a, q, q_dtype, S, st);
  if (rc != COMMVQ_OK) return rc;

  BinvArgs v{};
  v.scores = a.scores;
  v.partials = a.partials;
  v.error_word = a.error_word;
  v.seq_offsets = seq_offsets;
  v.bits = v_bits;
  v.C = v_codebook;
  v.hpart = reinterpret_cast<float*>(ws + L.hpart_off);
  v.wts = ws + L.wts_off;
  v.mvec = reinterpret_cast<float*>(ws + L.mvec_off);
  v.lpart = reinterpret_cast<float*>(ws + L.lpart_off);
  v.opart = reinterpret_cast<float*>(ws + L.opart_off);
  v.ml = reinterpret_cast<float2*>(ws + L.ml_off);
  v.out = out;
  v.lse = lse;
  v.max_T = max_T;
  v.n_tiles = (max_T + 15) / 16;
  v.B = B;
  v.Hq = cfg->q_heads;
  v.KV = cfg->kv_heads;
  v.Nc = n_bits;
  v.S = L.S;
  v.K = L.K;
  v.Sv = L.Sv;
  v.P = L.P;
  if (cudaFuncSetAttribute(binv_accumulate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kBvTcSmem)) != cudaSuccess ||
      cudaFuncSetAttribute(binv_merge_contract_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kBvMcSmem)) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  if (launch_dependent(binv_weights_kernel, dim3(L.Sv, L.P, B), dim3(256), 0, st, v) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  if (launch_dependent(binv_accumulate_kernel, dim3(L.Sv, n_bits / kBvBitsPerCta, B), dim3(kBvThreads), kBvTcSmem,
                       st, v) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  if (launch_dependent(binv_merge_contract_kernel, dim3(B * cfg->kv_heads, n_bits / kBvCRows), dim3(256), kBvMcSmem,
                       st, v) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  if (launch_dependent(binv_finalize_kernel, dim3(B * cfg->q_heads), dim3(kD), 0, st, v) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  return launch_status();
}
