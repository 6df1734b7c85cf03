// Internal interface between the attention entry point and its kernels.
#pragma once

#include "common.cuh"

namespace commvq {

// One split's result for one (sequence, query head): o is unnormalised (sum of
// exp2(s - m) v), m the split's max score and l the sum of exp2(s - m), both in the
// exp2 domain (scores pre-multiplied by log2 e).
struct __align__(16) Partial {
  float o[kD];
  float m;
  float l;
  float pad[2];
};

struct AttendArgs {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const int64_t* seq_offsets;
  const float* k_codebook;
  const float* v_codebook;
  float* out;
  float* lse;
  Partial* partials;
  int* error_word;
  float* scores;          // decode-and-rotate form: tile-blocked exp2-domain scores
  const uint4* k_img;     // decode-and-rotate form: fp16 codebook images (see attend_mma.cu)
  const uint4* v_img;
  // decode-and-rotate form: RoPE tables written by its prep kernel. Phasor rows hold, per
  // pair of RoPE pairs (p, p+1) with p even, one float4 (cos p, cos p+1, sin p, sin p+1).
  const double* theta;
  const float4* rowph;    // [128 offsets][32]
  const float4* advph;    // [32]
  void* main_start;       // optional cudaEvent_t pair around the main kernel(s)
  void* main_stop;
  int64_t max_T;
  double rope_base;
  int B;
  int q_heads;
  int kv_heads;
  int R;
  int n_codes;
};

size_t table_smem_bytes(int R, int n_codes);
size_t mma_scores_smem_bytes(int R, int KV, int n_codes);
size_t mma_values_smem_bytes(int R, int KV, int q_heads, int n_codes);
bool mma_supported(int R, int q_heads, int kv_heads, int n_codes);
commvq_status launch_attend_prep(const AttendArgs& a, cudaStream_t st);
commvq_status launch_attend_mma(const AttendArgs& a, const void* q, commvq_dtype qt, int splits,
                                cudaStream_t st);
// Position splits of the decode-and-rotate scores kernel for this batch (the count
// attend_mma_setup returns).
int mma_splits(int B, int q_heads, int64_t max_T);
// AttendArgs for the decode-and-rotate key side in an attention workspace laid out for
// (cfg, B, max_T) with the DECODE_MMA algorithm; returns the split count.
int attend_mma_setup(const commvq_config* cfg, int B, int64_t max_T, unsigned char* ws,
                     const int64_t* seq_offsets, const void* k_codes, const float* k_codebook, AttendArgs& a);
// The scores kernel alone (maxima in the partials' m, exp2-domain scores in a.scores).
commvq_status launch_attend_scores(const AttendArgs& a, const void* q, commvq_dtype qt, int splits,
                                   cudaStream_t st);
// The score buffer's slot of (sequence b, position t, KV head kv, head column col).
__host__ __device__ inline int64_t score_slot(int64_t b, int64_t t, int kv, int col, int64_t n_tiles, int KV, int G) {
  const int tau = static_cast<int>(t % 16);
  return ((((b * n_tiles + t / 16) * KV + kv) * G + col) * 4 + ((tau & 7) >> 1)) * 4 + (tau & 1) + 2 * (tau >> 3);
}
commvq_status launch_attend_table(const AttendArgs& a, const void* q, commvq_dtype qt, int splits,
                                  cudaStream_t st);
commvq_status launch_combine(const AttendArgs& a, int splits, cudaStream_t st, bool one_per_sm = false);
// The fast decode-and-rotate kernels (attend_fast.cu): KV heads in {2, 4, 8}, up to 8 query heads
// per KV head, R <= 2, Nc' <= 256, g = 8. Their prepared state is 128 KB per codebook image, RoPE
// tables theta [64] fp64, offset rows [64][64] (cos, sin) and the 64-position advance [64].
bool fast_supported(int g, int R, int q_heads, int kv_heads, int n_codes);
size_t fast_keys_smem_bytes(int R, int KV);
size_t fast_values_smem_bytes(int R, int KV, int q_heads);
size_t fast_smem_bytes(int R, int KV, int q_heads);   // the fused kernel's dynamic shared memory
commvq_status launch_fast_prep(const AttendArgs& a, cudaStream_t st);
// dependent: launch the attention kernel as a programmatic dependent of the previous kernel (only when
// that kernel does not write the prepared state).
commvq_status launch_attend_fast(const AttendArgs& a, const void* q, commvq_dtype qt, int splits, cudaStream_t st,
                                 bool dependent);
bool generic_supported(const commvq_config* cfg);
int generic_warps_per_kv(int kv_heads);
size_t generic_tables_bytes(int64_t max_T);
commvq_status launch_attend_generic(const AttendArgs& a, const commvq_config* cfg, const void* q,
                                    commvq_dtype qt, int S, void* tables, cudaStream_t st);

}  // namespace commvq
