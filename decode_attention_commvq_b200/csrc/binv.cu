// Decode attention with the paper's binary value code (CommVQ review, "Assumptions & free
// parameters": a value codebook of Nc rows over the whole KV dimension, Nc / d bits per scalar;
// Nc = 1024 for 1 bit and 2048 for 2 bits at d = 1024). Position t stores bits s_t in {0,1}^Nc
// and its value row, all KV heads together, is v_t = s_t^T C with C [Nc, kv_heads * 128]. Keys
// keep CommVQ's additive RoPE-commutative code and its scores kernel.
//
// Because v_t is linear in s_t, the softmax weights can be folded into the bits first:
//   out_h = (sum_t p_{h,t} s_t) C[:, slice of h's KV head] / sum_t p_{h,t}.
// Kernel 1 (grid: position splits x 256-bit slices x sequences) forms the per-split sums
// H_v[h, n] = sum_t 2^(score - m_v) s_t[n] with tcgen05 MMAs, as H_v^T = S^T P^T: A = the bits of
// 128 codebook rows (M) for 16 positions (K), expanded to fp16 0 / 1 and stored into tensor memory;
// B = the weights of all 32 query-head columns (N) in shared memory; D accumulates in tensor
// memory. A split is a run of whole splits of the scores kernel, so its maximum m_v is the maximum
// of their maxima and every weight is at most 1. Kernel 2 (grid: KV heads x 128-row chunks of C)
// merges the splits' H with log-sum-exp weights and contracts its chunk with C; kernel 3 sums the
// chunks and divides by the softmax sum.
#include <math.h>

#include "attend.cuh"

namespace commvq {
namespace {

constexpr int kBvThreads = 512;   // 16 warps
constexpr int kBvPosGroups = 4;   // 16-position MMA steps per chunk
constexpr int kBvBitsPerCta = 256;                              // two M = 128 halves
constexpr int kBvSliceBytes = kBvBitsPerCta / 8;                // 32
constexpr int kBvMaxHeads = 32;
constexpr int kBvTile = 16;       // positions per MMA K step (one tile of the scores buffer)
constexpr int kBvChunk = kBvPosGroups * kBvTile;   // positions per pipeline step
constexpr int kBvStages = 4;
constexpr int kBvMaxSplits = 64;
constexpr int kBvCRows = 128;                      // rows of C per merge-and-contract CTA
constexpr int kBvMaxG = 8;

struct BinvArgs {
  const float* scores;        // the scores kernel's exp2-domain scores, tile-blocked
  const Partial* partials;    // the scores kernel's per-split maxima (m)
  const int64_t* seq_offsets;
  const uint8_t* bits;        // [total_T, Nc / 8]
  const float* C;             // [Nc, KV * 128]
  float* hpart;               // [B][Sv][Hq][Nc]
  float2* mlpart;             // [B][Sv][Hq] (m, l)
  float* opart;               // [B][Hq][Nc / kBvCRows][128]
  float2* ml;                 // [B][Hq] (M, L)
  float* out;
  float* lse;
  int* error_word;
  int64_t max_T, n_tiles;
  int B, Hq, KV, Nc, S, K, Sv;   // S scores splits, K of them per value split, Sv value splits
};

constexpr size_t kBvMcSmem = (kBvCRows * kD + kBvMaxG * kBvMaxSplits + 2 * kBvMaxG * kBvCRows) * 4;

// Value split v of sequence b: scores splits vK .. vK + K - 1 (the same tile-aligned pieces of
// ceil(T_b / S) positions).
__device__ __forceinline__ void bv_split(const BinvArgs& a, int b, int v, int64_t& row0, int64_t& t_begin,
                                         int64_t& t_end) {
  row0 = a.seq_offsets[b];
  int64_t Tb = a.seq_offsets[b + 1] - row0;
  Tb = Tb < 0 ? 0 : (Tb > a.max_T ? a.max_T : Tb);
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

// Position tau of a 16-position tile sits at this offset of the head's 16 scores (the scores
// kernel's fragment order).
__device__ __forceinline__ int tile_slot(int tau) { return ((tau & 7) >> 1) * 4 + (tau & 1) + 2 * (tau >> 3); }

// ---------------------------------------------------------------------------------------
// tcgen05 pieces (PTX ISA 8.6, sm_100a): TMEM allocation, loads and stores, the f16 MMA with its
// A operand in TMEM and B in shared memory, completion through an mbarrier.

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `parity` to complete, giving up after `limit` polls (each poll may
// itself block for a while). Returns false when it gave up.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t limit) {
  for (uint32_t n = 0; n < limit; ++n)
    if (mbar_test(bar, parity)) return true;
  return false;
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

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
// D[128 x N] (+)= A[128 x 16] (TMEM, fp16) * B[16 x N] (shared memory descriptor, fp16), fp32 D.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B fp16 (formats 0), both
// K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kBvIdesc = (1u << 4) | ((32u >> 3) << 17) | ((128u >> 4) << 24);
// Shared-memory descriptor of a K-major, unswizzled operand: 8-row x 16-byte core matrices,
// LBO = byte step between the two 8-element K halves, SBO = byte step between 8-row groups,
// version 1 at bits 46-47.
__device__ __forceinline__ uint64_t smem_desc_k(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

constexpr int kBvCols = 256;       // TMEM columns: D (2 x 32), A (2 buffers x 2 halves x 32)
constexpr int kBvColA = 64;
constexpr uint32_t kBvWaitPolls = 1u << 20;
// B operand of one buffer: 4 k-steps x [32 heads x 16 positions] fp16, K-major core matrices:
// (head h, position k of the step) at ks 1024 + (h / 8) 256 + (k / 8) 128 + (h % 8) 16 + (k % 8) 2.
constexpr int kBvBBytes = kBvPosGroups * kBvMaxHeads * kBvTile * 2;
constexpr size_t kBvTcSmem = 2 * kBvBBytes + kBvStages * (kBvChunk * kBvSliceBytes + kBvPosGroups * kBvMaxHeads * kBvTile * 4) +
                             kBvMaxHeads * 4 + 2 * 8 + 16;

// H_v^T[n, h] = sum_t s_t[n] 2^(score_{h,t} - m_v) for the CTA's 256 codebook rows (two M = 128
// halves) and all 32 head columns, on tcgen05: per 64-position chunk, 16 warps expand the bits to
// fp16 0 / 1 straight into TMEM (A, one 32-lane quarter and one 16-position step per store), all
// threads write the weights into shared memory (B), and one thread issues 8 MMAs (2 halves x 4
// steps) and commits them to the buffer's mbarrier. Two A/B buffers: chunk c + 1 is built while
// chunk c's MMAs run.
__global__ void __launch_bounds__(kBvThreads, 1) binv_accumulate_kernel(BinvArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* bbuf = smem;                                                  // [2][kBvBBytes]
  unsigned char* stg = smem + 2 * kBvBBytes;                                   // [stages][bits | scores]
  constexpr int kStgBits = kBvChunk * kBvSliceBytes;                           // 2048
  constexpr int kStgBytes = kStgBits + kBvPosGroups * kBvMaxHeads * kBvTile * 4;
  float* mrow = reinterpret_cast<float*>(stg + kBvStages * kStgBytes);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(mrow + kBvMaxHeads);            // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(mbar + 2);

  const int v = blockIdx.x, slice = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t row0, t_begin, t_end;
  bv_split(a, b, v, row0, t_begin, t_end);
  const int64_t n_c = (t_end - t_begin + kBvChunk - 1) / kBvChunk;
  const uint8_t* bsrc = a.bits + row0 * (a.Nc / 8) + slice * kBvSliceBytes;
  const float* ssrc = a.scores + (static_cast<int64_t>(b) * a.n_tiles + t_begin / kBvTile) * a.Hq * kBvTile;

  if (warp == 0) {   // TMEM for the accumulators and the A buffers (one CTA per SM)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tslot)),
                 "r"(kBvCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(&mbar[0], 1);
    mbar_init(&mbar[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  pdl_wait();   // the scores kernel's buffer and maxima are complete from here on

  {   // the split's maximum per head: the maxima of its K scores splits (16 lanes per head)
    const int h = tid >> 4, l = tid & 15;
    float m = -INFINITY;
    if (h < a.Hq) {
      const Partial* ph = a.partials + (static_cast<int64_t>(b) * a.Hq + h) * a.S;
      for (int s = v * a.K + l; s < min(a.S, (v + 1) * a.K); s += 16) m = fmaxf(m, ph[s].m);
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (l == 0) mrow[h] = m;
  }
  const int n_copies = kStgBits / 16 + kBvPosGroups * a.Hq * kBvTile / 4;
  auto issue = [&](int st, int64_t c) {   // chunk c into stage st (pieces past the split zero-filled)
    const int64_t t0 = t_begin + c * kBvChunk;
    unsigned char* dst = stg + st * kStgBytes;
    for (int e = tid; e < n_copies; e += kBvThreads) {
      if (e < kStgBits / 16) {
        const int p = e >> 1, h16 = e & 1;
        const bool ok = t0 + p < t_end;
        cp_async16_z(dst + p * kBvSliceBytes + 16 * h16, ok ? bsrc + (t0 + p) * (a.Nc / 8) + 16 * h16 : a.bits, ok);
      } else {
        const int j = e - kStgBits / 16;
        const int q = j / (a.Hq * kBvTile / 4);
        const bool ok = t0 + q * kBvTile < t_end;
        cp_async16_z(dst + kStgBits + 16 * j, ok ? ssrc + c * kBvPosGroups * a.Hq * kBvTile + 4 * j : a.scores, ok);
      }
    }
  };
#pragma unroll
  for (int s = 0; s < kBvStages - 1; ++s) {
    if (s < n_c) issue(s, s);
    cp_async_commit();
  }
  tc_fence_before();
  __syncthreads();   // TMEM address, mbarriers, mrow
  tc_fence_after();
  const uint32_t tbase = *tslot;

  const int ph = tid >> 4, pt = tid & 15;   // weight builder: head, position column of each step
  const int pslot = tile_slot(pt);
  const float m_h = mrow[ph];
  const uint32_t boff = static_cast<uint32_t>((ph >> 3) * 256 + (pt >> 3) * 128 + (ph & 7) * 16 + (pt & 7) * 2);
  // bit expansion: this warp's TMEM lane quarter and its two (half, step) units
  const int quarter = warp & 3;
  float lacc = 0.0f;
  bool ok = true;
  for (int64_t c = 0; c < n_c; ++c) {
    const int st = static_cast<int>(c % kBvStages), bb = static_cast<int>(c & 1);
    cp_async_wait<kBvStages - 2>();
    __syncthreads();   // chunk c landed; chunk c - 1's stage reads are done
    {
      const int64_t cn = c + kBvStages - 1;
      if (cn < n_c) issue(static_cast<int>(cn % kBvStages), cn);
      cp_async_commit();
    }
    if (c >= 2) {   // the MMAs of chunk c - 2 read buffer bb
      ok = mbar_wait_bounded(&mbar[bb], static_cast<uint32_t>(((c >> 1) - 1) & 1), kBvWaitPolls) && ok;
      tc_fence_after();
    }
    const unsigned char* sg = stg + st * kStgBytes;
    const float* sc = reinterpret_cast<const float*>(sg + kStgBits);
    // weights 2^(score - m), fp16, into B; fp32 row sums
#pragma unroll
    for (int q = 0; q < kBvPosGroups; ++q) {
      const int64_t t = t_begin + c * kBvChunk + q * kBvTile + pt;
      const bool valid = ph < a.Hq && t < t_end;
      const float p = valid ? exp2f(sc[(q * a.Hq + ph) * kBvTile + pslot] - m_h) : 0.0f;
      lacc += p;
      *reinterpret_cast<__half*>(bbuf + bb * kBvBBytes + q * 1024 + boff) = __float2half_rn(p);
    }
    fence_async_smem();   // generic-proxy writes of B, read by the tensor cores
    // bits -> fp16 0 / 1 in TMEM: lane `lane` of quarter `quarter` is codebook row
    // hb 128 + 32 quarter + lane; column j of a step holds positions 2j (low half) and 2j + 1
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int unit = (warp >> 2) * 2 + u, hb = unit >> 2, ks = unit & 3;
      const unsigned char* rows = sg + (ks * kBvTile) * kBvSliceBytes + hb * 16 + 4 * quarter;
      uint32_t col[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(rows + (2 * j) * kBvSliceBytes);
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(rows + (2 * j + 1) * kBvSliceBytes);
        col[j] = (((w0 >> lane) & 1u) | (((w1 >> lane) & 1u) << 16)) * 0x3C00u;
      }
      tmem_st8(tbase + (static_cast<uint32_t>(32 * quarter) << 16) + kBvColA + (bb * 2 + hb) * 32 + ks * 8, col);
    }
    tc_wait_st();
    tc_fence_before();
    ok = __syncthreads_and(ok) != 0;   // B and A of chunk c are complete; every wait succeeded
    if (!ok) break;                    // (uniform) a wait gave up: issue nothing more
    if (tid == 0) {
      tc_fence_after();
      const uint32_t bsa = smem_u32(bbuf + bb * kBvBBytes);
#pragma unroll
      for (int ks = 0; ks < kBvPosGroups; ++ks) {
        const uint64_t bd = smem_desc_k(bsa + ks * 1024, 128, 256);
#pragma unroll
        for (int hb = 0; hb < 2; ++hb)
          umma_f16_ts(tbase + hb * 32, tbase + kBvColA + (bb * 2 + hb) * 32 + ks * 8, bd, kBvIdesc,
                      (c > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit(&mbar[bb]);
    }
  }
  cp_async_wait<0>();
  // the last commit covers every MMA issued before it
  if (n_c > 0 && ok) {
    const int64_t cl = n_c - 1;
    ok = mbar_wait_bounded(&mbar[cl & 1], static_cast<uint32_t>((cl >> 1) & 1), kBvWaitPolls);
  }
  tc_fence_after();
  ok = __syncthreads_and(ok) != 0;
  if (!ok && tid == 0) atomicOr(a.error_word, kErrWaitLimit);

#pragma unroll
  for (int o = 1; o < 16; o <<= 1) lacc += __shfl_xor_sync(0xffffffffu, lacc, o);
  const int64_t base = (static_cast<int64_t>(b) * a.Sv + v) * a.Hq;
  if (slice == 0 && pt == 0 && ph < a.Hq) a.mlpart[base + ph] = make_float2(m_h, lacc);
  if (warp < 8) {   // warps 0-3: rows 0-127 (D of half 0), warps 4-7: rows 128-255
    const int hb = warp >> 2;
    const bool have = n_c > 0 && ok;   // uniform
    uint32_t r[32];
    if (have) {
      tmem_ld32(tbase + (static_cast<uint32_t>(32 * quarter) << 16) + hb * 32, r);
      tc_wait_ld();
    }
    float* dst = a.hpart + base * a.Nc + slice * kBvBitsPerCta + hb * 128 + 32 * quarter + lane;
#pragma unroll
    for (int h = 0; h < kBvMaxHeads; ++h)
      if (h < a.Hq) dst[static_cast<int64_t>(h) * a.Nc] = have ? __uint_as_float(r[h]) : 0.0f;
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
  const float2* mlb = a.mlpart + static_cast<int64_t>(b) * a.Sv * a.Hq + kv * G;
  if (tid < G) {
    float M = -INFINITY;
    for (int s = 0; s < a.Sv; ++s) M = fmaxf(M, mlb[static_cast<int64_t>(s) * a.Hq + tid].x);
    float L = 0.0f;
    for (int s = 0; s < a.Sv; ++s) {
      const float2 m_l = mlb[static_cast<int64_t>(s) * a.Hq + tid];
      const float w = M == -INFINITY ? 0.0f : exp2f(m_l.x - M);
      wts[tid * kBvMaxSplits + s] = w;
      L = fmaf(w, m_l.y, L);
    }
    if (chunk == 0) a.ml[static_cast<int64_t>(b) * a.Hq + kv * G + tid] = make_float2(M, L);
  }
  __syncthreads();
  // merged H of the chunk: element (h, n), n fastest (coalesced); four independent partial sums
  for (int e = tid; e < G * kBvCRows; e += 256) {
    const int h = e / kBvCRows, n = e % kBvCRows;
    const float* src = a.hpart + (static_cast<int64_t>(b) * a.Sv * a.Hq + kv * G + h) * a.Nc + n0 + n;
    const int64_t step = static_cast<int64_t>(a.Hq) * a.Nc;
    const float* w = wts + h * kBvMaxSplits;
    float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
    int s = 0;
    for (; s + 4 <= a.Sv; s += 4) {
      s0 = fmaf(w[s], src[s * step], s0);
      s1 = fmaf(w[s + 1], src[(s + 1) * step], s1);
      s2 = fmaf(w[s + 2], src[(s + 2) * step], s2);
      s3 = fmaf(w[s + 3], src[(s + 3) * step], s3);
    }
    for (; s < a.Sv; ++s) s0 = fmaf(w[s], src[s * step], s0);
    hc[h * kBvCRows + n] = (s0 + s1) + (s2 + s3);
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
  pdl_wait();
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

struct BvLayout {
  size_t attend_bytes, hpart_off, mlpart_off, opart_off, ml_off, total;
  int S, K, Sv;
};

BvLayout bv_layout(const commvq_config* cfg, int Nc, int B, int64_t max_T, const commvq_attend_options* o) {
  BvLayout L{};
  L.attend_bytes = commvq_attend_workspace_bytes(cfg, B, max_T, o);
  L.S = mma_splits(B > 0 ? B : 1, cfg->q_heads, max_T);
  bv_geometry(B > 0 ? B : 1, Nc, L.S, L.K, L.Sv);
  L.hpart_off = round_up(L.attend_bytes, 256);
  L.mlpart_off = round_up(L.hpart_off + static_cast<size_t>(B) * L.Sv * cfg->q_heads * Nc * sizeof(float), 256);
  L.opart_off = round_up(L.mlpart_off + static_cast<size_t>(B) * L.Sv * cfg->q_heads * sizeof(float2), 256);
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
    rc = launch_attend_prep(a, st);   // also clears the error word
    if (rc != COMMVQ_OK) return rc;
  } else if (cfg->n_codes < 256 && cudaMemsetAsync(a.error_word, 0, sizeof(int), st) != cudaSuccess) {
    return COMMVQ_ERR_CUDA;
  }
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
  v.mlpart = reinterpret_cast<float2*>(ws + L.mlpart_off);
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
  if (cudaFuncSetAttribute(binv_accumulate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kBvTcSmem)) != cudaSuccess ||
      cudaFuncSetAttribute(binv_merge_contract_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kBvMcSmem)) != cudaSuccess)
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
