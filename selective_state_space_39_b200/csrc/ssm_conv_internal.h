// ssm_conv_internal.h -- parameters of the causal depthwise conv1d + SiLU
// shared by the C entry points (ssm_api.cu) and the kernels (ssm_conv1d.cu).
// Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssm {

// Steps per CTA chunk along the sequence (measured best on the 8 x 2048 x
// 1536 bf16 layer among 32 .. 256): forward 32, backward 256.
constexpr int kConvChunkFwd = 32;
constexpr int kConvChunkBwd = 256;

struct ConvParams {
  int batch, seqlen, dim, width, chunk;
  int silu;
  int w_vec;          // w is 16-byte aligned (width-4 taps load as one vector)
  const void* x;      // (batch, seqlen, dim) io
  const float* w;     // (dim, width)
  const float* bias;  // (dim) or null
  void* out;          // forward output (batch, seqlen, dim) io
  const void* dout;   // backward: upstream gradient (batch, seqlen, dim) io
  void* dx;           // backward: (batch, seqlen, dim) io
  float* dw;          // backward: (dim, width) or null
  float* dbias;       // backward: (dim) or null
  float* ws_dw;       // backward workspace: [batch * chunks][dim][width]
  float* ws_db;       // backward workspace: [batch * chunks][dim]
};

bool conv_width_supported(int width);
// Decode step: p.out is the rolling state (batch, dim, width-1) io, p.x the
// new input (batch, dim), p.dx the output (batch, dim).
cudaError_t launch_conv_update(const ConvParams& p, bool bf16, cudaStream_t stream);
// vec: 8-byte vector path (dim a multiple of 4 for bf16 / 2 for fp32, 8-byte
// aligned tensors); otherwise one element per thread.
cudaError_t launch_conv(const ConvParams& p, bool bf16, bool vec, bool backward,
                        cudaStream_t stream);

}  // namespace ssm
