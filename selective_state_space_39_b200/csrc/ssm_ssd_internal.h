// ssm_ssd_internal.h -- parameters of the multi-head SSD scan shared by the C
// entry point (ssm_api.cu) and the kernel (ssm_ssd.cu). Not part of the
// public ABI.
#pragma once

#include <cuda.h>
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
  uint64_t wait_limit_ns;  // bound on every wait of the tensor-core kernel
  int test_stall;          // test hook: its first CTA waits for 16 bytes that never arrive
};

// TMA maps of the tensor-core kernel (128-byte swizzle): x as (headdim, nheads,
// seqlen, batch) with a 64 x 1 x 128 x 1 box; B and C as (dstate, seqlen,
// batch) with a 64 x 128 x 1 box.
struct alignas(64) SsdTcMaps {
  CUtensorMap x, B, C, y;  // y: the same geometry as x
};

bool ssd_dstate_supported(int dstate);
cudaError_t launch_ssd_fwd(const SsdParams& p, cudaStream_t stream);
// The tensor-core (tcgen05) kernel: dstate 64 or 128, an even head count.
bool ssd_tc_supported(int dstate, int nheads);
cudaError_t launch_ssd_tc(const SsdParams& p, const SsdTcMaps& maps, cudaStream_t stream);
// Synchronise `stream`; *out = 1 (and the flag cleared) if a CTA of the
// tensor-core kernel gave up a wait since the last call, else 0.
cudaError_t ssd_tc_status(cudaStream_t stream, int* out);

}  // namespace ssm
