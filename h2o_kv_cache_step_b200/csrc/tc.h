// tc.h -- tensor-core (tcgen05 / TMEM / TMA) kernels of the bf16 H2O step.
#pragma once

#include <cuda.h>

#include "kernels.h"

namespace h2o {

// True when the device is sm_100 and the head dimension has a tensor-core path.
bool tc_supported(int device, int d);
// Workspace floats the weight-sum partials need for chunks of up to tmax tokens.
size_t tc_partial_elems(int B, int Hq, int Hkv, int C, int tmax);
// Row stride of the -log2(LSE) table the weight sums read (rows per KV group, padded).
int tc_rows_pad(int Hq, int Hkv, int tmax);
// Number of weight-sum partials (row parts) a chunk of T tokens produces.
int tc_partial_count(int Hq, int Hkv, int T);
// Names of the tensor-core kernels one step launches (returns the count).
int tc_kernel_plan(int B, int Hq, int Hkv, int d, int C, int T, int n, int num_sms, const char** names,
                   int max_names);
// Floats of the workspace a step's split SDPA needs (0 when it does not split).
size_t tc_sdpa_part_elems(int B, int Hq, int Hkv, int d, int T, int n, int num_sms);
// Evaluates the polynomial exp2 (degrees 3 and 4) and ex2.approx on x[0..n).
cudaError_t tc_exp2_selftest(const float* x, float* y3, float* y4, float* ym, int n, cudaStream_t s);
// Chunk SDPA: O and per-row LSE.
cudaError_t tc_sdpa(const StepArgs& a);
// Per-key weight sums added to the scores (writes cand_score / cand_pos).
cudaError_t tc_wsum(const StepArgs& a);
// 2-D TMA map over a [rows, d] bf16 matrix: boxes of box_rows rows x 64
// columns, 128-byte swizzle (the UMMA K-major / MN-major operand layouts).
bool tc_make_map(CUtensorMap* m, const void* base, uint64_t rows, int d, int box_rows);
// Backward of the chunk SDPA on the tensor cores (bf16 inputs; fp32 gradients).
cudaError_t tc_backward(const BwdArgs& a);

}  // namespace h2o
