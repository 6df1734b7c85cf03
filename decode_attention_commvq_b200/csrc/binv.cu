// Decode attention with the paper's binary value code (CommVQ review, "Assumptions & free
// parameters": a value codebook of Nc rows over the whole KV dimension, Nc / d bits per scalar;
// Nc = 1024 for 1 bit and 2048 for 2 bits at d = 1024). Position t stores bits s_t in {0,1}^Nc
// and its value row, all KV heads together, is v_t = s_t^T C with C [Nc, kv_heads * 128]. Keys
// keep CommVQ's additive RoPE-commutative code and its scores kernel.
//
// Because v_t is linear in s_t, the softmax weights can be folded into the bits first:
//   out_h = (sum_t p_{h,t} s_t) C[:, slice of h's KV head] / sum_t p_{h,t}.
// Kernel 1 (grid: position splits x 256-bit slices x sequences) forms the per-split sums
// H_v[h, n] = sum_t 2^(score - m_v) s_t[n] on the tensor cores: A = the weights of all query heads
// (rows) for 16 positions (k), B = the 16 positions' bits for 8 codebook rows (n), expanded to
// fp16 0 / 1 in registers. A split is a run of whole splits of the scores kernel, so its maximum
// m_v is the maximum of their maxima and every weight is at most 1. Kernel 2 (grid: KV heads x
// 128-row chunks of C) merges the splits' H with log-sum-exp weights and contracts its chunk with
// C; kernel 3 sums the chunks and divides by the softmax sum.
#include <math.h>

#include "attend.cuh"

namespace commvq {
namespace {

constexpr int kBvThreads = 512;   // 16 warps: 4 bit groups x 4 position groups
constexpr int kBvBitGroups = 4;
constexpr int kBvPosGroups = 4;
constexpr int kBvBitsPerWarp = 64;
constexpr int kBvBitsPerCta = kBvBitGroups * kBvBitsPerWarp;   // 256
constexpr int kBvSliceBytes = kBvBitsPerCta / 8;                // 32
constexpr int kBvRowBytes = 48;   // padded: the 4 rows a warp reads at once hit distinct banks
constexpr int kBvMaxHeads = 32;
constexpr int kBvTile = 16;       // positions per mma k-step (one tile of the scores buffer)
constexpr int kBvChunk = kBvPosGroups * kBvTile;   // positions per pipeline step
constexpr int kBvStages = 4;
constexpr int kPStride = kBvChunk + 8;             // halves per weight row (144 B: conflict-free ldmatrix)
constexpr int kBvMaxSplits = 64;
constexpr int kHRed = kBvBitsPerWarp + 8;          // floats per head row of the reduction buffer
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
  int64_t max_T, n_tiles;
  int B, Hq, KV, Nc, S, K, Sv;   // S scores splits, K of them per value split, Sv value splits
};

struct BvStage {
  uint8_t bits[kBvChunk][kBvRowBytes];
  float sc[kBvPosGroups * kBvMaxHeads * kBvTile];   // 4 tiles' score blocks, head h of tile q at 16 (q Hq + h)
};
static_assert(sizeof(BvStage) % 16 == 0, "stage alignment");
constexpr size_t kBvLoopSmem = kBvStages * sizeof(BvStage) + kBvMaxHeads * kPStride * 2 + kBvMaxHeads * 4;
constexpr size_t kBvRedSmem = (kBvPosGroups - 1) * kBvBitGroups * kBvMaxHeads * kHRed * 4;
constexpr size_t kBvAccSmem = kBvLoopSmem > kBvRedSmem ? kBvLoopSmem : kBvRedSmem;
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

__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// fp16 pair (bit lo, bit hi) as 1.0 / 0.0 (0x3C00 is fp16 1.0)
__device__ __forceinline__ uint32_t bits_to_h2(uint32_t lo, uint32_t hi) { return lo * 0x3C00u + hi * 0x3C000000u; }

// Position tau of a 16-position tile sits at this offset of the head's 16 scores (the scores
// kernel's fragment order).
__device__ __forceinline__ int tile_slot(int tau) { return ((tau & 7) >> 1) * 4 + (tau & 1) + 2 * (tau >> 3); }

__global__ void __launch_bounds__(kBvThreads, 1) binv_accumulate_kernel(BinvArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  BvStage* stage = reinterpret_cast<BvStage*>(smem);
  __half(*ptile)[kPStride] = reinterpret_cast<__half(*)[kPStride]>(smem + kBvStages * sizeof(BvStage));
  float* mrow = reinterpret_cast<float*>(smem + kBvStages * sizeof(BvStage) + kBvMaxHeads * kPStride * 2);
  float* hred = reinterpret_cast<float*>(smem);   // after the loop: [pos group - 1][bit group][head][kHRed]
  const int v = blockIdx.x, slice = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bg = warp & (kBvBitGroups - 1), pg = warp / kBvBitGroups;
  const int g = lane >> 2, i = lane & 3;
  int64_t row0, t_begin, t_end;
  bv_split(a, b, v, row0, t_begin, t_end);
  const int64_t n_c = (t_end - t_begin + kBvChunk - 1) / kBvChunk;
  const uint8_t* bsrc = a.bits + row0 * (a.Nc / 8) + slice * kBvSliceBytes;
  const float* ssrc = a.scores + (static_cast<int64_t>(b) * a.n_tiles + t_begin / kBvTile) * a.Hq * kBvTile;
  pdl_wait();   // the scores kernel's buffer and maxima are complete from here on

  // the split's maximum per head: the maxima of its K scores splits (16 lanes per head)
  {
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

  // chunk c of the split into stage st: 64 positions' 32-byte bit slices, then the 4 tiles'
  // score blocks (tiles past the split's end are zero-filled, never read as weights)
  const int n_copies = 2 * kBvChunk + kBvPosGroups * a.Hq * kBvTile / 4;
  auto issue = [&](int st, int64_t c) {
    const int64_t t0 = t_begin + c * kBvChunk;
    for (int e = tid; e < n_copies; e += kBvThreads) {
      if (e < 2 * kBvChunk) {
        const int p = e >> 1, h16 = e & 1;
        const bool ok = t0 + p < t_end;
        cp_async16_z(&stage[st].bits[p][16 * h16], ok ? bsrc + (t0 + p) * (a.Nc / 8) + 16 * h16 : a.bits, ok);
      } else {
        const int j = e - 2 * kBvChunk;                  // 16-byte piece of the 4 score blocks
        const int q = j / (a.Hq * kBvTile / 4);
        const bool ok = t0 + q * kBvTile < t_end;
        cp_async16_z(&stage[st].sc[4 * j], ok ? ssrc + c * kBvPosGroups * a.Hq * kBvTile + 4 * j : a.scores, ok);
      }
    }
  };
#pragma unroll
  for (int s = 0; s < kBvStages - 1; ++s) {
    if (s < n_c) issue(s, s);
    cp_async_commit();
  }
  __syncthreads();   // mrow

  float H[2][8][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) H[mt][nt][0] = H[mt][nt][1] = H[mt][nt][2] = H[mt][nt][3] = 0.0f;
  const int ph = tid >> 4, pt = tid & 15;   // weight builder: head row, position column of each tile
  const int pslot = tile_slot(pt);
  const float m_h = mrow[ph];
  const bool two_mt = a.Hq > 16;
  float lacc = 0.0f;
  // ldmatrix row addresses of the weight tile: matrix (lane >> 3) is rows 0-7 / 8-15 of k 0-7,
  // then rows 0-7 / 8-15 of k 8-15; this warp's k columns are those of its position group
  const int lrow = (lane & 7) + (((lane >> 3) & 1) << 3), lcol = pg * kBvTile + ((lane >> 4) << 3);
  const int brow = pg * kBvTile + 2 * i;
  for (int64_t c = 0; c < n_c; ++c) {
    const int st = static_cast<int>(c % kBvStages);
    cp_async_wait<kBvStages - 2>();   // chunk c has landed (this thread's pieces)
    __syncthreads();                  // ... everyone's; and chunk c - 1 is done with its stage and the weights
    {
      const int64_t cn = c + kBvStages - 1;
      if (cn < n_c) issue(static_cast<int>(cn % kBvStages), cn);
      cp_async_commit();
    }
    // weights 2^(score - m), fp16, and their fp32 row sums
#pragma unroll
    for (int q = 0; q < kBvPosGroups; ++q) {
      const int64_t t = t_begin + c * kBvChunk + q * kBvTile + pt;
      const bool valid = ph < a.Hq && t < t_end;
      const float p = valid ? exp2f(stage[st].sc[(q * a.Hq + ph) * kBvTile + pslot] - m_h) : 0.0f;
      lacc += p;
      ptile[ph][q * kBvTile + pt] = __float2half_rn(p);
    }
    __syncthreads();
    uint32_t A[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const unsigned addr = static_cast<unsigned>(__cvta_generic_to_shared(&ptile[mt * 16 + lrow][lcol]));
      asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                   : "=r"(A[mt][0]), "=r"(A[mt][1]), "=r"(A[mt][2]), "=r"(A[mt][3])
                   : "r"(addr));
    }
    // the warp's 64 codebook rows: bytes 8 bg .. 8 bg + 7 of its tile's positions' slices
    const uint2 w0 = *reinterpret_cast<const uint2*>(&stage[st].bits[brow][8 * bg]);
    const uint2 w1 = *reinterpret_cast<const uint2*>(&stage[st].bits[brow + 1][8 * bg]);
    const uint2 w2 = *reinterpret_cast<const uint2*>(&stage[st].bits[brow + 8][8 * bg]);
    const uint2 w3 = *reinterpret_cast<const uint2*>(&stage[st].bits[brow + 9][8 * bg]);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int sh = (nt & 3) * 8 + g;   // bit nt * 8 + g of the 64-bit slice
      const uint32_t x0 = nt < 4 ? w0.x : w0.y, x1 = nt < 4 ? w1.x : w1.y;
      const uint32_t x2 = nt < 4 ? w2.x : w2.y, x3 = nt < 4 ? w3.x : w3.y;
      const uint32_t b0 = bits_to_h2((x0 >> sh) & 1u, (x1 >> sh) & 1u);
      const uint32_t b1 = bits_to_h2((x2 >> sh) & 1u, (x3 >> sh) & 1u);
      mma_f16(H[0][nt], A[0], b0, b1);
      if (two_mt) mma_f16(H[1][nt], A[1], b0, b1);
    }
  }
  cp_async_wait<0>();
  __syncthreads();   // the stages are free: the reduction buffer overlays them

  // row sums: the 16 builders of a head are 16 consecutive lanes
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) lacc += __shfl_xor_sync(0xffffffffu, lacc, o);
  const int64_t base = (static_cast<int64_t>(b) * a.Sv + v) * a.Hq;
  if (slice == 0 && pt == 0 && ph < a.Hq) a.mlpart[base + ph] = make_float2(m_h, lacc);
  // the four position groups' sums: groups 1-3 through shared memory into group 0
  if (pg > 0) {
    float* dst = hred + ((pg - 1) * kBvBitGroups + bg) * kBvMaxHeads * kHRed;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
          *reinterpret_cast<float2*>(dst + (mt * 16 + g + 8 * rr) * kHRed + nt * 8 + 2 * i) =
              make_float2(H[mt][nt][2 * rr], H[mt][nt][2 * rr + 1]);
  }
  __syncthreads();
  if (pg == 0) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int h = mt * 16 + g + 8 * rr;
        if (h >= a.Hq) continue;
        float* dst = a.hpart + (base + h) * a.Nc + slice * kBvBitsPerCta + bg * kBvBitsPerWarp;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          float2 sum = make_float2(H[mt][nt][2 * rr], H[mt][nt][2 * rr + 1]);
#pragma unroll
          for (int q = 0; q < kBvPosGroups - 1; ++q) {
            const float2 o = *reinterpret_cast<const float2*>(
                hred + ((q * kBvBitGroups + bg) * kBvMaxHeads + h) * kHRed + nt * 8 + 2 * i);
            sum.x += o.x;
            sum.y += o.y;
          }
          *reinterpret_cast<float2*>(dst + nt * 8 + 2 * i) = sum;
        }
      }
  }
}

// One (sequence, KV head, 128-row chunk of C): merge the G heads' split sums over the chunk,
//   H[h, n] = sum_v 2^(m_v - M) H_v[h, n],  M = max_v m_v,
// and contract: opart[h, chunk, :] = sum_{n in chunk} H[h, n] C[n, kv 128 : kv 128 + 128].
// The chunk's rows of C are copied into shared memory before the wait on the previous kernel.
// The chunk-0 CTA also stores (M, L = sum_v 2^(m_v - M) l_v).
__global__ void __launch_bounds__(256) binv_merge_contract_kernel(BinvArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
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
                           static_cast<int>(kBvAccSmem)) != cudaSuccess ||
      cudaFuncSetAttribute(binv_merge_contract_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kBvMcSmem)) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  if (launch_dependent(binv_accumulate_kernel, dim3(L.Sv, n_bits / kBvBitsPerCta, B), dim3(kBvThreads), kBvAccSmem,
                       st, v) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  if (launch_dependent(binv_merge_contract_kernel, dim3(B * cfg->kv_heads, n_bits / kBvCRows), dim3(256), kBvMcSmem,
                       st, v) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  if (launch_dependent(binv_finalize_kernel, dim3(B * cfg->q_heads), dim3(kD), 0, st, v) != cudaSuccess)
    return COMMVQ_ERR_CUDA;
  return launch_status();
}
