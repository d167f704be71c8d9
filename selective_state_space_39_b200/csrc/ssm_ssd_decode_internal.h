// ssm_ssd_decode_internal.h -- parameters of the multi-head SSD decode step
// shared by the C entry point (ssm_api.cu) and the kernel
// (ssm_ssd_decode.cu). Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

struct SsdDecodeParams {
  int batch, nheads, headdim, dstate, softplus;
  float* state;          // (batch, nheads, headdim, dstate), updated in place
  const void* x;         // (batch, nheads, headdim) io
  const void* dt;        // (batch, nheads) io
  const void* B;         // (batch, dstate) io
  const void* C;         // (batch, dstate) io
  const float* A;        // (nheads)
  const float* D;        // (nheads) or null
  const float* dt_bias;  // (nheads) or null
  void* y;               // (batch, nheads, headdim) io
};

// dstate values of the decode kernel (one warp per state row, dstate/32
// states per lane).
bool ssd_decode_dstate_supported(int dstate);
cudaError_t launch_ssd_decode(const SsdDecodeParams& p, bool bf16, cudaStream_t stream);

}  // namespace ssm
