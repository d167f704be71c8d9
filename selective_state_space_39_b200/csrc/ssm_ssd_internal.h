// ssm_ssd_internal.h -- parameters of the multi-head SSD scan shared by the C
// entry point (ssm_api.cu) and the kernel (ssm_ssd.cu). Not part of the
// public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

// Steps per chunk and head width of the tensor-core SSD kernel.
constexpr int kSsdChunk = 32;
constexpr int kSsdHeadDim = 64;

struct SsdParams {
  int batch, nheads, dstate;
  int64_t seqlen;
  int softplus;
  const uint16_t* x;   // (batch, seqlen, nheads, headdim) bf16
  const uint16_t* dt;  // (batch, seqlen, nheads) bf16
  const uint16_t* B;   // (batch, seqlen, dstate) bf16
  const uint16_t* C;   // (batch, seqlen, dstate) bf16
  const float* A;      // (nheads)
  const float* D;      // (nheads) or null
  const float* dt_bias;  // (nheads) or null
  const float* h0;     // (batch, nheads, headdim, dstate) or null
  uint16_t* y;         // (batch, seqlen, nheads, headdim) bf16
  float* h_last;       // (batch, nheads, headdim, dstate) or null
};

bool ssd_dstate_supported(int dstate);
cudaError_t launch_ssd_fwd(const SsdParams& p, cudaStream_t stream);

}  // namespace ssm
