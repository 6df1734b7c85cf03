// Shared host/device helpers of the CommVQ B200 library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include "commvq.h"

namespace commvq {

constexpr int kThreads = 256;
constexpr int kG = 8;          // scalars per shared index
constexpr int kD = 128;        // head dimension of the attention kernels
constexpr int kGroups = kD / kG;
constexpr int kPairs = kG / 2; // RoPE pairs per group

// Device error word bits (first 4 bytes of an attention workspace).
constexpr int kErrCodeRange = 1;
constexpr int kErrWaitLimit = 2;   // a bounded wait on asynchronous tensor-core work gave up
constexpr int kErrLength = 4;      // a sequence length outside [0, max_T] (taken as clamped)

// An attention call's kernels OR their error bits into the running word (int 1 of the
// workspace); the call's last kernel publishes it as the error word (int 0) and clears the
// running word for the next call. Both kernels run in stream order, so the publication never
// races with a setter.
__device__ __forceinline__ int* running_error(int* error_word) { return error_word + 1; }
__device__ __forceinline__ void publish_error(int* error_word) {
  error_word[0] = error_word[1];
  error_word[1] = 0;
}

// Rows of sequence b: seq_offsets[b] .. seq_offsets[b+1]-1, at most max_T of them. A length
// outside [0, max_T] is clamped, and thread 0 of the calling CTA ORs kErrLength into *err_bits
// (nullable: no report).
__device__ __forceinline__ int64_t sequence_rows(const int64_t* seq_offsets, int b, int64_t max_T,
                                                 int* err_bits, int64_t& row0) {
  row0 = seq_offsets[b];
  const int64_t Tb = seq_offsets[b + 1] - row0;
  if (Tb < 0 || Tb > max_T) {
    if (threadIdx.x == 0 && err_bits) atomicOr(err_bits, kErrLength);
    return Tb < 0 ? 0 : max_T;
  }
  return Tb;
}

// An NVTX range around a C-ABI call, named after it (visible in Nsight timelines; with no
// profiler attached the header-only NVTX calls return at once).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline commvq_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? COMMVQ_OK : COMMVQ_ERR_CUDA;
}

// Cached per-device attributes (the only state the library keeps).
struct DeviceInfo {
  int device = -1;
  int sms = 0;
  size_t smem_optin = 0;
};
DeviceInfo current_device_info();

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Programmatic dependent launch: a kernel launched with launch_dependent may be scheduled as
// soon as every CTA of the kernel before it has signalled pdl_trigger() (or exited), and must
// call pdl_wait() before it touches anything that kernel writes. Without the launch attribute
// pdl_wait() returns at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" :::); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Record a caller's timing event on `st`. Inside a stream capture the record becomes an
// external event node, so the event keeps real timestamps when the graph is replayed; outside
// a capture it is an ordinary record.
inline cudaError_t record_event(void* ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  const cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  return cs == cudaStreamCaptureStatusActive
             ? cudaEventRecordWithFlags(static_cast<cudaEvent_t>(ev), st, cudaEventRecordExternal)
             : cudaEventRecord(static_cast<cudaEvent_t>(ev), st);
}

// ---------------------------------------------------------------------------------------
// Nearest entry of a sub-codebook, the encoder's distance rule. Exactly the fp32 operations
// the definition names, so codes are reproducible bit for bit:
//   e_k = res_k - c_k (round to nearest), dist = fma(e_k, e_k, dist), k = 0..7 in order,
//   strictly smaller distance replaces the winner (ties -> lowest index).
struct Nearest {
  float best;
  float second;
  int idx;
};

__device__ __forceinline__ void nearest_init(Nearest& n) {
  n.best = __int_as_float(0x7f800000);
  n.second = __int_as_float(0x7f800000);
  n.idx = 0;
}

template <bool kTrack>
__device__ __forceinline__ void nearest_step(Nearest& n, const float (&res)[kG], const float4 lo,
                                             const float4 hi, int c) {
  float dist = 0.0f;
  float e;
  e = __fsub_rn(res[0], lo.x); dist = __fmaf_rn(e, e, dist);
  e = __fsub_rn(res[1], lo.y); dist = __fmaf_rn(e, e, dist);
  e = __fsub_rn(res[2], lo.z); dist = __fmaf_rn(e, e, dist);
  e = __fsub_rn(res[3], lo.w); dist = __fmaf_rn(e, e, dist);
  e = __fsub_rn(res[4], hi.x); dist = __fmaf_rn(e, e, dist);
  e = __fsub_rn(res[5], hi.y); dist = __fmaf_rn(e, e, dist);
  e = __fsub_rn(res[6], hi.z); dist = __fmaf_rn(e, e, dist);
  e = __fsub_rn(res[7], hi.w); dist = __fmaf_rn(e, e, dist);
  if (dist < n.best) {
    if (kTrack) n.second = n.best;
    n.best = dist;
    n.idx = c;
  } else if (kTrack && dist < n.second) {
    n.second = dist;
  }
}

// Nearest entry for GG-scalar groups: the same fp32 rule as nearest_step (subtract, then a fused
// multiply-add, k = 0..GG-1 in order; strictly smaller wins), entry read from shared memory.
template <int GG, bool kTrack>
__device__ __forceinline__ void nearest_step_g(Nearest& n, const float (&res)[GG], const float4* e, int c) {
  float dist = 0.0f;
#pragma unroll
  for (int q = 0; q < GG / 4; ++q) {
    const float4 v = e[q];
    float t;
    t = __fsub_rn(res[4 * q + 0], v.x); dist = __fmaf_rn(t, t, dist);
    t = __fsub_rn(res[4 * q + 1], v.y); dist = __fmaf_rn(t, t, dist);
    t = __fsub_rn(res[4 * q + 2], v.z); dist = __fmaf_rn(t, t, dist);
    t = __fsub_rn(res[4 * q + 3], v.w); dist = __fmaf_rn(t, t, dist);
  }
  if (dist < n.best) {
    if (kTrack) n.second = n.best;
    n.best = dist;
    n.idx = c;
  } else if (kTrack && dist < n.second) {
    n.second = dist;
  }
}

// Near tie: at least two entries and (d2 - d1) <= 1e-5 * d2, in fp32.
__device__ __forceinline__ bool near_tie(const Nearest& n, int n_codes) {
  if (n_codes < 2) return false;
  const float gap = __fsub_rn(n.second, n.best);
  const float lim = __fmul_rn(1e-5f, n.second);
  return gap <= lim;
}

__device__ __forceinline__ void load_row8(const float* p, float (&v)[kG]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load_row8(const __half* p, float (&v)[kG]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ void store_code(void* codes, int64_t at, int code, int code_bytes) {
  if (code_bytes == 1)
    static_cast<uint8_t*>(codes)[at] = static_cast<uint8_t>(code);
  else
    static_cast<uint16_t*>(codes)[at] = static_cast<uint16_t>(code);
}

// Ampere-style asynchronous 16-byte global -> shared copies (bypass L1), used to prefetch
// code chunks one step ahead of the compute that consumes them.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem_src) : "memory");
}
// The same copy through L1 (.ca): used for data this CTA wrote to global memory before a
// barrier, which the barrier makes visible to the CTA's own reads.
__device__ __forceinline__ void cp_async16_ca(void* smem_dst, const void* gmem_src) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// mbarriers (shared memory, CTA scope) and 1-D bulk copies of the tensor memory accelerator.
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
// One arrival on `bar` that also expects `bytes` of asynchronous transfers on its phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory"); }
// Global -> this CTA's shared memory, `bytes` (a multiple of 16, both addresses 16-byte aligned)
// counted against `bar`'s transaction count; the destination is this CTA's own shared memory.
__device__ __forceinline__ void bulk_copy_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   smem_u32(smem_dst)),
               "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Two fp32 values in one 64-bit register pair, for the packed fp32x2 arithmetic of sm_100
// (one instruction works on both lanes; each lane rounds as its scalar counterpart would).
using f32x2 = unsigned long long;
__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(f32x2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// Complex product of packed phasors: (c, s) <- (c, s) * (cc, ss), two pairs at a time.
__device__ __forceinline__ void cmul2(f32x2& c, f32x2& s, f32x2 cc, f32x2 ss) {
  const f32x2 nc = sub2(mul2(c, cc), mul2(s, ss));
  s = fma2(c, ss, mul2(s, cc));
  c = nc;
}
// The phasors of RoPE pairs (p, p+1) from a packed row entry (cos p, cos p+1, sin p, sin p+1).
__device__ __forceinline__ void load_phasor(float4 v, f32x2& c, f32x2& s) {
  c = pack2(v.x, v.y);
  s = pack2(v.z, v.w);
}

// Nearest-entry update with a distance already computed by the encoder's fp32 rule (the
// comparison half of nearest_step). A distance is a sum of squares from +0, so it is >= +0 (or
// NaN for non-finite input); on such values the fp32 order is the unsigned order of the bit
// patterns, with NaN above +inf (never taken, as in the fp32 comparison). The comparisons run
// as integer instructions, leaving the fp32 pipe to the distance arithmetic.
template <bool kTrack>
__device__ __forceinline__ void nearest_take(Nearest& n, float dist, int c) {
  const uint32_t d = __float_as_uint(dist);
  if (d < __float_as_uint(n.best)) {
    if (kTrack) n.second = n.best;
    n.best = dist;
    n.idx = c;
  } else if (kTrack && d < __float_as_uint(n.second)) {
    n.second = dist;
  }
}

// g = 8 sub-codebook tile for the packed scan: entries 2p and 2p + 1 side by side, so that one
// packed fp32x2 instruction takes the same step of both distances. Pair p occupies float4s
// 4p .. 4p + 3; float4 kk holds (e_2p[2kk], e_2p+1[2kk], e_2p[2kk+1], e_2p+1[2kk+1]). An odd last
// entry is paired with itself (its second lane is never compared). src: n entries of 8 floats.
__device__ __forceinline__ void stage_pairs8(float4* tile, const float* src, int n) {
  const int pairs = (n + 1) >> 1;
  for (int e = threadIdx.x; e < pairs * 4; e += blockDim.x) {
    const int p = e >> 2, kk = e & 3;
    const int c1 = min(2 * p + 1, n - 1);
    const float2 lo = __ldg(reinterpret_cast<const float2*>(src + static_cast<int64_t>(2 * p) * kG) + kk);
    const float2 hi = __ldg(reinterpret_cast<const float2*>(src + static_cast<int64_t>(c1) * kG) + kk);
    tile[e] = make_float4(lo.x, hi.x, lo.y, hi.y);
  }
}

// Distances of one row to entries 2p and 2p + 1 of a pair tile; res2[k] holds the row's residual
// k in both lanes. Each lane follows the encoder's fp32 rule exactly (k = 0..7 in order: subtract,
// then a fused multiply-add onto the running sum from +0), so the distances -- and the codes they
// decide -- are bit-identical to the scalar scan.
__device__ __forceinline__ f32x2 pair_dist8(const f32x2 (&res2)[kG], const float4* pair) {
  f32x2 acc = 0ull;   // +0.0f in both lanes
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const float4 v = pair[kk];
    f32x2 t = sub2(res2[2 * kk], pack2(v.x, v.y));
    acc = fma2(t, t, acc);
    t = sub2(res2[2 * kk + 1], pack2(v.z, v.w));
    acc = fma2(t, t, acc);
  }
  return acc;
}

// Phasor e^{i phi} of RoPE pair p into a packed row: float4 p/2 holds (cos p, cos p+1, sin p,
// sin p+1) for even p, the operand order of the packed rotation.
__device__ __forceinline__ void put_phasor(float4* row, int p, double cs, double sn) {
  float* f = reinterpret_cast<float*>(row + (p >> 1));
  f[p & 1] = static_cast<float>(cs);
  f[2 + (p & 1)] = static_cast<float>(sn);
}

}  // namespace commvq
