// ssm_seqpar_internal.h -- parameters of the sequence-split helpers shared by
// the C entry points (ssm_api.cu) and the kernels (ssm_seqpar.cu). Not part
// of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssm {

struct SeqParParams {
  int batch, seqlen, dim, dstate;
  int softplus;
  int rank;                // compose: chunks 0..rank-1 precede this one
  const void* delta;       // delta_sum: (batch, seqlen, dim) io
  const float* bias;       // (dim) or null
  float* dsum;             // delta_sum output: (batch, dim)
  const float* A;          // compose: (dim, dstate)
  const float* h0;         // compose: (batch, dim, dstate) or null
  const float* hend_all;   // compose: (ranks, batch, dim, dstate)
  const float* dsum_all;   // compose: (ranks, batch, dim)
  float* h_in;             // compose output: (batch, dim, dstate)
};

cudaError_t launch_delta_sum(const SeqParParams& p, bool bf16, cudaStream_t stream);
cudaError_t launch_compose(const SeqParParams& p, cudaStream_t stream);

}  // namespace ssm
