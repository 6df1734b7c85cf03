/*
 * commvq.h -- C ABI of the CommVQ decode-attention library for B200 (sm_100a).
 *
 * CommVQ (CommVQ: Commutative Vector Quantization for KV Cache Compression) stores the
 * key/value cache as additive vector-quantization codes: g consecutive scalars share one
 * index, R residual rounds each pick one entry of an Nc'-entry sub-codebook, and a row is
 * decoded as the sum of its selected entries (abstract: decoding is a matrix multiply;
 * machine review, "What carries the argument": index sharing, R rounds,
 * R*log2(Nc')/g bits per scalar). The key codebook's 2x2 blocks [[x, y], [-y, x]] commute
 * with the RoPE rotation, so attention scores can be formed from a per-query
 * query x codebook table and rotated afterwards ("What carries the argument",
 * Property 1 / Eq. 7-8). Values are decoded after the softmax weights have been folded
 * into the codes ("If this is right": weights multiply value codes before the codebook
 * multiply).
 *
 * Conventions shared by every call
 *  - g = 8 (4 RoPE pairs per index, d/g = 16 groups) is the layout of the fast attention
 *    kernels; g = 16, 32 and 64 (the pages' own g) are taken by the encoder, the hard EM
 *    step and the GENERIC attention algorithm. Attention needs d = 128.
 *  - RoPE pair p is channels (2p, 2p+1), theta_p = rope_base^(-2p/d); the key of row t of
 *    a sequence sits at position t; queries arrive already rotated; scores are scaled
 *    by 1/sqrt(d); there is no mask.
 *  - A stored key pair (a, b) is the reconstructed 2-vector (its commuting block is
 *    [[a, -b], [b, a]]).
 *  - Codes: [T, kv_heads, R, d/g], one code per element, uint8 when Nc' <= 256
 *    (code_bytes = 1) else uint16 (code_bytes = 2), little-endian.
 *  - Codebooks: [R, d/g, Nc', g] float32, shared by all KV heads and sequences.
 *  - Query head h reads KV head h / (q_heads / kv_heads).
 *
 * Ownership and memory: the caller owns every buffer. All tensor pointers are device
 * pointers (CUDA global memory) unless stated; the config struct is host memory. The
 * library allocates nothing, keeps no state besides cached device attributes, and never
 * synchronises a stream except where a call says so. Calls are asynchronous on `stream`
 * (a cudaStream_t; NULL = legacy default stream).
 *
 * Errors: arguments are validated on the host before any launch; a failed check returns
 * a status and launches nothing. A launch failure returns COMMVQ_ERR_CUDA. Data errors
 * found on the device (a code >= Nc', a sequence length outside [0, max_T]) never trap:
 * the kernel clamps the value, records the error in the workspace's error word and carries
 * on; read it with commvq_workspace_error().
 */
#ifndef COMMVQ_H_
#define COMMVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  COMMVQ_OK = 0,
  COMMVQ_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size or shape */
  COMMVQ_ERR_UNSUPPORTED = 2,   /* valid CommVQ shape this build does not implement */
  COMMVQ_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  COMMVQ_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
  COMMVQ_ERR_DEVICE_CHECK = 5   /* the device recorded a data error (code or length out of range) */
} commvq_status;

typedef enum { COMMVQ_F32 = 0, COMMVQ_F16 = 1, COMMVQ_BF16 = 2 } commvq_dtype;

/* Attention algorithms (both compute the same attention; see commvq_attend_decode). */
typedef enum {
  COMMVQ_ATTN_AUTO = 0,       /* the library's fastest for the shape */
  COMMVQ_ATTN_TABLE = 1,      /* per-query table + value histograms, one CTA per (b, q head, split) */
  COMMVQ_ATTN_DECODE_MMA = 2, /* decode each (token, KV head) once, rotate, tensor-core QK and PV */
  COMMVQ_ATTN_GENERIC = 3     /* any g in {8, 16, 32, 64}, R <= 32, Nc' <= 65536: fp32 decode from
                                 the fp32 codebooks, one warp per (token, KV head) */
} commvq_attn_algo;

typedef struct {
  int32_t d;          /* head dimension */
  int32_t g;          /* scalars per shared index */
  int32_t R;          /* residual rounds */
  int32_t n_codes;    /* Nc', entries per sub-codebook */
  int32_t q_heads;    /* query heads (attention only) */
  int32_t kv_heads;   /* KV heads */
  double rope_base;   /* RoPE base (attention only) */
  int32_t code_bytes; /* 1 if n_codes <= 256 else 2 */
} commvq_config;

/* commvq_attend_options.flags */
enum {
  /* The workspace already holds this configuration's and these codebooks' prepared state,
     written by commvq_attend_prepare (or by an earlier commvq_attend_decode without the
     flag) with the same cfg and algo; the call skips rewriting it. The prepared state sits at
     fixed offsets at the start of the workspace, so B, max_T and splits may differ between the
     preparing call and later ones (the workspace must be large enough for each call). */
  COMMVQ_ATTEND_PREPARED = 1
};

typedef struct {
  int32_t algo;        /* commvq_attn_algo */
  int32_t splits;      /* split-T partitions per sequence; 0 = chosen by the library */
  void* main_start;    /* nullable cudaEvent_t, recorded on `stream` right before the main
                          attention kernel (instrumentation; no effect on the result) */
  void* main_stop;     /* nullable cudaEvent_t, recorded right after it, before the merge */
  int32_t flags;       /* COMMVQ_ATTEND_* bits; 0 = none */
} commvq_attend_options;

/* Residual nearest-codeword encoder (abstract: additive quantization; "What carries the
 * argument": g scalars per index, R residual rounds; Figure 1: every K/V vector is
 * encoded on its own).
 * For each row n of x and group j, with res = x[n, j*g:(j+1)*g] in fp32 and r = 0..R-1:
 *   dist(c) = fused sum over k = 0..g-1 in order of e_k^2, e_k = res_k - cb[r,j,c,k]
 *             (fp32 subtract, then fmaf(e, e, dist) starting from 0),
 *   code = first c with the strictly smallest dist (ties -> lowest index),
 *   res  = res - cb[r, j, code, :] (fp32).
 * x        [n_tokens, kv_heads, d] in x_dtype (COMMVQ_F32 or COMMVQ_F16), pre-RoPE keys or
 *          values, 16-byte aligned, contiguous.
 * codebook [R, d/g, Nc', g] float32, 16-byte aligned.
 * codes    [n_tokens, kv_heads, R, d/g] out, code_bytes per element.
 * near_ties nullable device counter; if given, the number of (row, round, group)
 *          decisions whose two smallest distances d1 <= d2 satisfy d2 - d1 <= 1e-5 * d2
 *          (fp32, Nc' >= 2) is ADDED to it.
 * residual_out nullable [n_tokens, kv_heads, d] float32, 16-byte aligned: the residual
 *          after the last round (what a further round, or the next round of a codebook
 *          fit, would encode).
 * Supports g in {8, 16, 32, 64}, d % g == 0, 1 <= Nc' <= 65536, 1 <= R <= 32. n_tokens = 0 is
 * a no-op. A small encode (up to 4096 rows x groups) runs as described under commvq_encode_kv:
 * a programmatic dependent launch that waits for the kernel before it first (stream order). */
commvq_status commvq_encode(const commvq_config* cfg, const void* x, commvq_dtype x_dtype,
                            int64_t n_tokens, const float* codebook, void* codes,
                            unsigned long long* near_ties, float* residual_out, void* stream);

/* commvq_encode of a key tensor and a value tensor of the same shape in one launch (the abstract:
 * the encoder turns every fresh K and V vector into codes): a decode step's new positions, whose
 * two small encodes would otherwise be two launches. Each tensor is encoded exactly as
 * commvq_encode encodes it (same codes, bit for bit) against its own codebook.
 * k_x, v_x          [n_tokens, kv_heads, d] in x_dtype (F32 or F16), 16-byte aligned.
 * k_codebook, v_codebook  [R, d/g, Nc', g] float32, 16-byte aligned.
 * k_codes, v_codes  [n_tokens, kv_heads, R, d/g] out, code_bytes per element.
 * near_ties         nullable device counter; both tensors' near-tie decisions are ADDED to it.
 * A small encode (up to 4096 rows x groups, e.g. a decode step's new position) is launched as a
 * programmatic dependent of the kernel before it on the stream, so that its launch overlaps that
 * kernel, and waits for that kernel's completion before it reads or writes anything: ordinary
 * stream order. Only then may a following programmatic dependent (the attention of a decode step
 * with COMMVQ_ATTEND_PREPARED) start its set-up; that kernel reads the codes only after the
 * encode has finished. Limits and errors as commvq_encode. */
commvq_status commvq_encode_kv(const commvq_config* cfg, const void* k_x, const void* v_x,
                               commvq_dtype x_dtype, int64_t n_tokens, const float* k_codebook,
                               const float* v_codebook, void* k_codes, void* v_codes,
                               unsigned long long* near_ties, void* stream);

/* Bytes of device workspace commvq_attend_decode needs for B sequences whose longest
 * has max_T cached rows (options may be NULL = defaults). Returns 0 for invalid input. */
size_t commvq_attend_workspace_bytes(const commvq_config* cfg, int32_t B, int64_t max_T,
                                     const commvq_attend_options* options);

/* Decode-step attention computed on the codes (no decompressed cache is formed in HBM).
 * For sequence b (rows seq_offsets[b] .. seq_offsets[b+1]-1, positions 0..T_b-1) and
 * query head h reading KV head kvh = h / (q_heads / kv_heads):
 *   k^_t = sum_r kcb[r, j, kcode[t,kvh,r,j], :] per group j, k~_t = RoPE_t(k^_t),
 *   s_t = q[b,h] . k~_t / sqrt(d), p = softmax(s),
 *   out[b,h] = sum_t p_t v^_t, v^_t = sum_r vcb[r, j, vcode[t,kvh,r,j], :],
 *   lse[b,h] = log(sum_t exp(s_t)) (natural log); an empty sequence gives out = 0 and
 *   lse = -inf.
 * The rotation is applied per position to query x codebook products (key side) and the
 * softmax weights are accumulated per code before the value codebook multiply, as the
 * review describes. Precision: fp32 accumulation. Codebook entries are held in fp16 (relative
 * error <= 2^-11 each). The table algorithm keeps its per-query table in fp16. The
 * decode-and-rotate algorithm sums a key's rounds exactly in fp32 and rotates it in fp32; with
 * 2, 4 or 8 KV heads it feeds the rotated key and the query to the tensor cores as fp16 (query
 * components saturate at +-65504), otherwise as two fp16 terms (value and rounding error).
 * Softmax weights and value entries (their rounds summed in fp16) enter the second product in
 * fp16. On the parity workloads this keeps every head within 4.2e-3 of the exact attention.
 * q           [B, q_heads, d] in q_dtype (F32, F16 or BF16), 16-byte aligned.
 * k_codes, v_codes  [total_T, kv_heads, R, d/g], code_bytes per element (uint16 above 256
 *             entries, GENERIC only), 16-byte aligned; total_T = seq_offsets[B].
 * seq_offsets [B+1] int64 device array, non-decreasing, seq_offsets[0] = 0, every
 *             0 <= T_b <= max_T. A length outside that range is clamped to it (a longer
 *             sequence is truncated to max_T rows, a negative one read as empty) and bit 2
 *             of the device error word is set.
 * k_codebook, v_codebook [R, d/g, Nc', g] float32, 16-byte aligned.
 * out         [B, q_heads, d] float32 out, 16-byte aligned.
 * lse         [B, q_heads] float32 out, nullable.
 * workspace   device buffer of at least commvq_attend_workspace_bytes(...) bytes,
 *             256-byte aligned; its first 64 bytes hold the device error word (int 0) and
 *             the running word the call's kernels set bits in (int 1); the call's last
 *             kernel copies the running word to the error word and clears it. Calls that
 *             share a workspace must be ordered on one stream. A call that returned an error
 *             status leaves the workspace's prepared state unspecified: prepare it again.
 * options     nullable (defaults: AUTO algorithm, library-chosen splits, no flags). With
 *             COMMVQ_ATTEND_PREPARED the workspace's prepared state (see commvq_attend_prepare)
 *             is used as it stands; otherwise the call writes it first. A prepared
 *             decode-and-rotate call launches its attention kernel as a programmatic dependent
 *             of the kernel before it on the stream, and that kernel reads q (and the prepared
 *             state) before it waits: q must not be written by the immediately preceding
 *             kernel on the stream (an event record or a copy in between, or a call without
 *             the flag, orders it fully).
 * Shapes: d = 128, q_heads % kv_heads == 0, B >= 0 (B = 0 is a no-op), and per algorithm
 *   DECODE_MMA  g = 8, R <= 2, Nc' <= 256, kv_heads in {1, 2, 4, 8}, q_heads / kv_heads <= 8;
 *   TABLE       g = 8, R <= 4, Nc' <= 256;
 *   GENERIC     g in {8, 16, 32, 64}, R <= 32, Nc' <= 65536, kv_heads in {1, 2, 4, 8},
 *               q_heads / kv_heads <= 16 (the pages' g = 64, Nc' = 64, R = 21 / 11 setting).
 * AUTO takes the first of DECODE_MMA, TABLE, GENERIC that accepts the shape; an explicit algo
 * that does not accept it returns COMMVQ_ERR_UNSUPPORTED. */
commvq_status commvq_attend_decode(const commvq_config* cfg, const void* q, commvq_dtype q_dtype,
                                   const void* k_codes, const void* v_codes,
                                   const int64_t* seq_offsets, int32_t B, int64_t max_T,
                                   const float* k_codebook, const float* v_codebook,
                                   float* out, float* lse, void* workspace,
                                   size_t workspace_bytes, const commvq_attend_options* options,
                                   void* stream);

/* Write the state of commvq_attend_decode that depends only on cfg and the codebooks into
 * the workspace: for the decode-and-rotate algorithm, the fp16 codebook images and the RoPE
 * phasor tables; it also clears the device error words. Later commvq_attend_decode calls with
 * the same cfg, algo, codebooks and workspace pass COMMVQ_ATTEND_PREPARED in options->flags and
 * skip this work (it is the same for every decode step of a layer, whatever the step's B and
 * max_T). The prepared state stays valid until the workspace or the codebooks change. With the
 * table algorithm there is no such state and the call only clears the error words.
 * Arguments and errors as in commvq_attend_decode. */
commvq_status commvq_attend_prepare(const commvq_config* cfg, int32_t B, int64_t max_T,
                                    const float* k_codebook, const float* v_codebook,
                                    void* workspace, size_t workspace_bytes,
                                    const commvq_attend_options* options, void* stream);

/* commvq_attend_decode for callers that cannot allocate device memory -- for example a
 * plugin inside a host framework that owns the device allocator, or a latency-critical loop
 * where a cudaMalloc (which may synchronise the device) is not allowed. This call has no
 * counterpart in the paper; it is a packaging variant of commvq_attend_decode.
 * Arguments and results are those of commvq_attend_decode without workspace/workspace_bytes:
 * the workspace is a fixed 32 MiB device array inside the library (every GPU that loads the
 * library holds it until the process exits). No cudaMalloc, cudaFree or other allocating
 * routine is called.
 * - Limit: a request whose commvq_attend_workspace_bytes exceeds 32 MiB returns
 *   COMMVQ_ERR_WORKSPACE without launching. (The 2-bit 32K layer needs ~7 MiB; the 1-bit
 *   128K layer and a batch of 16 sequences of up to 8192 positions need ~19-20 MiB.)
 * - Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before any
 *   stream capture.
 * - Sharing: all calls on a device use the same array and it keeps the last call's
 *   contents. Each call rewrites everything it reads, so results do not depend on earlier
 *   calls, but calls that overlap on the GPU (different streams without ordering) race.
 * - COMMVQ_ATTEND_PREPARED in options->flags is rejected with COMMVQ_ERR_INVALID_ARG: the
 *   prepared state would live in the shared array, where any other call on the device may
 *   have replaced it, so every call rebuilds it (one small kernel).
 * - Device data checks: codes >= Nc' are still clamped, but the error word lives in the
 *   internal array and is not reported by this entry point. */
commvq_status commvq_attend_decode_noalloc(const commvq_config* cfg, const void* q,
                                           commvq_dtype q_dtype, const void* k_codes,
                                           const void* v_codes, const int64_t* seq_offsets,
                                           int32_t B, int64_t max_T, const float* k_codebook,
                                           const float* v_codebook, float* out, float* lse,
                                           const commvq_attend_options* options, void* stream);

/* Bytes of device workspace commvq_em_step and commvq_em_step_soft need for N rows. 0 for
 * invalid input. */
size_t commvq_em_workspace_bytes(const commvq_config* cfg, int64_t N);

/* One EM step for one residual round's codebook (review: codebook fit by EM, Algorithm 1
 * and Eq. 20 -- hard assignment, closed-form centroid update; "no convergence guarantee
 * beyond local").
 *   assignment: the encoder's rule (one round) of every row's groups against the input
 *               codebook_round;
 *   update:     entry (j, c) = (float)(S / m), S the fp64 sum of the m fp32 sub-vectors
 *               assigned to it; an entry with m = 0 keeps its value.
 * Every stored pair already has the commuting-block form, so the key codebook needs no
 * projection after the mean.
 * rows           [N, d] float32 residual rows of this round, 16-byte aligned.
 * codebook_round [d/g, Nc', g] float32, read and overwritten in place.
 * codes_out      [N, d/g] nullable, code_bytes per element: assignments against the input
 *                codebook.
 * sse_out        nullable device double: sum over (row, group) of the assignment distance,
 *                accumulated in fp64.
 * workspace      >= commvq_em_workspace_bytes(cfg, N) bytes, 256-byte aligned.
 * The result does not depend on launch order (fixed-order fp64 reductions). Supports
 * g in {8, 16, 32, 64}, d % g == 0, 1 <= Nc' <= 4096, N >= 1. cfg->R is ignored. */
commvq_status commvq_em_step(const commvq_config* cfg, const float* rows, int64_t N,
                             float* codebook_round, void* codes_out, double* sse_out,
                             void* workspace, size_t workspace_bytes, void* stream);

/* One soft-assignment EM step at temperature tau (review, "Assumptions & free parameters":
 * the paper stabilises its EM with soft assignment and annealing; lowering tau from call to
 * call is the annealing). For each (row n, group j), with the encoder's fp32 distances d_c
 * against the input codebook and d_min = min_c d_c:
 *   w_c = exp(-(d_c - d_min) / tau) / sum_c' exp(-(d_c' - d_min) / tau)        (fp32),
 *   entry (j, c) = (float)(sum_n w_c x_n / sum_n w_c) with fp64 sums; an entry whose weight
 *   sum is 0 keeps its value.
 * sse_out: sum over (row, group) of d_min (the hard distortion against the input codebook).
 * tau must be finite and > 0 (COMMVQ_ERR_INVALID_ARG otherwise); as tau -> 0 the step tends
 * to commvq_em_step. Arguments, workspace (commvq_em_workspace_bytes covers both steps) and
 * limits are those of commvq_em_step, except that this step takes g = 8 only. Deterministic
 * run to run. */
commvq_status commvq_em_step_soft(const commvq_config* cfg, const float* rows, int64_t N,
                                  float* codebook_round, float tau, double* sse_out,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* ---- Binary value code -------------------------------------------------------------------
 * The paper's value encoding (review, "Assumptions & free parameters"): one bit vector
 * s_t in {0,1}^n_bits per position over the whole KV dimension (kv_heads * 128 scalars), decoded
 * as v_t = sum_n s_{t,n} C[n, :]; n_bits / (kv_heads * 128) bits per scalar (1024 -> 1 bit,
 * 2048 -> 2 bits at 8 KV heads). Keys keep the additive RoPE-commutative code of cfg.
 */

/* Bytes of device workspace commvq_attend_decode_binv needs. 0 for invalid or unsupported
 * input. */
size_t commvq_attend_binv_workspace_bytes(const commvq_config* cfg, int32_t n_bits, int32_t B, int64_t max_T);

/* Decode attention with CommVQ keys and binary values:
 *   s_t (keys) as in commvq_attend_decode, p = softmax(s),
 *   out[b,h] = sum_t p_t (s_t^T C)[kvh * 128 : kvh * 128 + 128], kvh = h / (q_heads / kv_heads),
 *   lse as in commvq_attend_decode.
 * The softmax weights are folded into the bits first, H_h = sum_t p_t s_t on the tensor cores
 * (int8 MMAs: bits as bytes 0 / 1, each weight as 24-bit fixed point in three 8-bit digits,
 * exact int32 sums; a weight carries 2^-25 absolute error), then H_h is contracted with C in fp32.
 * v_bits      [total_T, n_bits / 8] uint8, bit n of position t = byte n/8, bit n%8 (least
 *             significant first), 16-byte aligned.
 * v_codebook  C [n_bits, kv_heads * 128] float32.
 * Other arguments as commvq_attend_decode (q, k_codes, seq_offsets, B, max_T, k_codebook, out,
 * lse, workspace of commvq_attend_binv_workspace_bytes bytes).
 * Supports the DECODE_MMA key shapes (g = 8, R <= 2, Nc' <= 256, kv_heads in {1, 2, 4, 8}),
 * q_heads <= 32, n_bits a multiple of 1024 up to 8192.
 * flags: COMMVQ_ATTEND_PREPARED when this workspace already holds the key side's codebook images
 * and RoPE tables from an earlier call with the same cfg, B, max_T and k_codebook (the first call
 * on a workspace passes 0). Codes out of range are clamped and reported as by
 * commvq_attend_decode (commvq_workspace_error on this workspace). */
commvq_status commvq_attend_decode_binv(const commvq_config* cfg, const void* q, commvq_dtype q_dtype,
                                        const void* k_codes, const uint8_t* v_bits, int32_t n_bits,
                                        const int64_t* seq_offsets, int32_t B, int64_t max_T,
                                        const float* k_codebook, const float* v_codebook, float* out,
                                        float* lse, void* workspace, size_t workspace_bytes, int32_t flags,
                                        void* stream);

/* ---- Decompress-then-attend comparator ----------------------------------------------------
 * The review compares CommVQ's decode latency with a "naive implementation of the same
 * quantization" ("What carries the argument", Table 5: 6x-9.6x lower latency). These two calls
 * are that implementation: commvq_decompress writes the whole cache out as dense 16-bit rows,
 * keys already rotated, and commvq_dense_decode runs ordinary flash-decoding over them. Together
 * they compute what commvq_attend_decode computes, with the cache decompressed in HBM.
 */

/* Bytes of device workspace commvq_decompress needs (its fp16 codebook images and phasor
 * tables). 0 for invalid or unsupported input. */
size_t commvq_decompress_workspace_bytes(const commvq_config* cfg, int64_t max_T);

/* Decode every cached position and write it densely:
 *   k_out[t, kvh, :] = RoPE_pos(sum_r kcb[r, j, kcode[t,kvh,r,j], :] per group j),
 *   v_out[t, kvh, :] = sum_r vcb[r, j, vcode[t,kvh,r,j], :],
 * where pos = t - seq_offsets[b] is the row's position in its sequence b (RoPE as in
 * commvq_attend_decode: pair p = channels (2p, 2p+1), theta_p = rope_base^(-2p/d)).
 * k_codes, v_codes  [total_T, kv_heads, R, d/g] uint8, total_T = seq_offsets[B].
 * seq_offsets       [B+1] int64 device array as in commvq_attend_decode; rows past
 *                   max_T positions of a sequence are not written (and set bit 2 of the
 *                   error word, as a negative length does).
 * out_dtype         COMMVQ_BF16 or COMMVQ_F16.
 * k_out, v_out      [total_T, kv_heads, d] of out_dtype, 16-byte aligned.
 * workspace         >= commvq_decompress_workspace_bytes(cfg, max_T) bytes, 256-byte aligned;
 *                   its first 4 bytes are the device error word (bit 0: a code >= Nc' was
 *                   seen and clamped; bit 2: a sequence length outside [0, max_T]), cleared
 *                   by this call.
 * Precision: entries are held in fp16 and summed in fp16; keys are rotated in fp32 with
 * phasors from fp64 angles; one final rounding to out_dtype.
 * Supports d = 128, g = 8, R <= 2, Nc' <= 256. */
commvq_status commvq_decompress(const commvq_config* cfg, const void* k_codes, const void* v_codes,
                                const int64_t* seq_offsets, int32_t B, int64_t max_T,
                                const float* k_codebook, const float* v_codebook,
                                commvq_dtype out_dtype, void* k_out, void* v_out, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Bytes of device workspace commvq_dense_decode needs (per-split partials). 0 for invalid or
 * unsupported input. options: only `splits` is read (0 = library choice, at most 512). */
size_t commvq_dense_decode_workspace_bytes(const commvq_config* cfg, int32_t B, int64_t max_T,
                                           const commvq_attend_options* options);

/* Dense decode attention over rows that already carry their rotation:
 *   s_t = q[b,h] . k[t, h / (q_heads / kv_heads)] / sqrt(d), out[b,h] = softmax(s) . v,
 *   lse[b,h] = log sum_t exp(s_t) (natural log); an empty sequence gives 0 and -inf.
 * q       [B, q_heads, d] in q_dtype (F32, F16 or BF16), converted to kv_dtype for the
 *         tensor-core products.
 * k, v    [total_T, kv_heads, d] in kv_dtype (F16 or BF16), 16-byte aligned.
 * seq_offsets, B, max_T, out, lse: as in commvq_attend_decode.
 * workspace >= commvq_dense_decode_workspace_bytes(...) bytes, 256-byte aligned; its first 4
 *         bytes are the device error word (bit 2: a sequence length outside [0, max_T], clamped),
 *         written by this call (read it with commvq_workspace_error).
 * options nullable: splits (0 = library choice) and the main_start / main_stop events, recorded
 *         around the attention kernel (before the split combine).
 * Precision: fp32 accumulation; softmax weights are rounded to kv_dtype for the second product.
 * Supports d = 128, kv_heads in {1, 2, 4, 8}, q_heads / kv_heads <= 16. */
commvq_status commvq_dense_decode(const commvq_config* cfg, const void* q, commvq_dtype q_dtype,
                                  const void* k, const void* v, commvq_dtype kv_dtype,
                                  const int64_t* seq_offsets, int32_t B, int64_t max_T, float* out,
                                  float* lse, void* workspace, size_t workspace_bytes,
                                  const commvq_attend_options* options, void* stream);

/* The device error word in an attention workspace: synchronises `stream`, copies the word
 * to the host and writes it to *device_error (0 = none; bit 0 = a code >= Nc' was seen
 * and clamped; bit 1 = a bounded wait for the tensor cores' asynchronous work gave up, the
 * output of that call is not valid; bit 2 = a sequence length outside [0, max_T] was
 * clamped). Returns COMMVQ_ERR_DEVICE_CHECK when the word is non-zero. */
commvq_status commvq_workspace_error(const void* workspace, int32_t* device_error, void* stream);

/* Copies `bytes` bytes from src to dst with one kernel on `stream` (asynchronous, like
 * cudaMemcpyAsync). Either pointer may be device memory or mapped pinned host memory (memory
 * from cudaHostAlloc / cudaMallocHost, whose host address the device can use under unified
 * addressing): the kernel's loads or stores then cross the host link. Meant for the few-KB
 * per-step transfers of a decode loop (the query and the new position's K/V rows in, the output
 * out), where a copy-engine transfer inside a CUDA graph costs more in scheduling than the bytes.
 * Both pointers 16-byte aligned, ranges not overlapping (else COMMVQ_ERR_INVALID_ARG); bytes = 0
 * is a no-op. The caller owns both buffers. The kernel is launched as a programmatic dependent of
 * the kernel before it on the stream (its launch overlaps that kernel) and waits for that
 * kernel's completion before its first load or store, so it is ordered like any stream operation;
 * a following programmatic dependent may start its set-up once every block has passed that wait.
 * Not part of the method: plumbing for the end-to-end step of a decode loop. */
commvq_status commvq_copy_async(void* dst, const void* src, size_t bytes, void* stream);

/* Static description of a status code. */
const char* commvq_status_string(commvq_status status);

/* ABI version of this library (incremented on any signature change). */
int32_t commvq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* COMMVQ_H_ */
