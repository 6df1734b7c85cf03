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
  int64_t max_T;
  double rope_base;
  int B;
  int q_heads;
  int kv_heads;
  int R;
  int n_codes;
};

size_t table_smem_bytes(int R, int n_codes);
commvq_status launch_attend_table(const AttendArgs& a, const void* q, commvq_dtype qt, int splits,
                                  cudaStream_t st);
commvq_status launch_combine(const AttendArgs& a, int splits, cudaStream_t st);

}  // namespace commvq
