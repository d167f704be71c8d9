// ssm_bwd_internal.h -- parameters of the backward pass shared by the C
// entry point (ssm_api.cu) and its kernels (ssm_scan_bwd.cu). Not part of
// the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssm {

// Steps per backward tile (the depth of the register history of states) and
// channels per CTA (one channel per thread).
constexpr int kBwdTileSteps = 4;
constexpr int kBwdThreads = 128;

// How one backward call is split: `nseg` segments of `seg_steps` steps (a
// multiple of kBwdTileSteps) along the sequence, `dblocks` CTAs along dim.
struct BwdPlan {
  int nseg, seg_steps, dblocks, ntiles;  // ntiles: tiles of the whole sequence
  size_t off_ck, off_qk, off_hloc, off_mloc, off_hin, off_muin, off_qseg, off_dbc, off_dA,
      off_dD, off_dbias, bytes;
};

struct BwdParams {
  int batch, seqlen, dim;
  int nseg, seg_steps, dblocks, ntiles;
  int softplus;
  int scal_pairs;  // bf16: per-step tensors may be copied two channels per 4-byte copy
  // forward inputs
  const void* x;
  const void* delta;
  const void* z;
  const void* B;
  const void* C;
  const float* A;
  const float* D;
  const float* bias;
  const float* h0;
  // upstream gradients
  const void* dy;
  const float* dh_last;
  // gradients
  void* dx;
  void* ddelta;
  void* dz;
  float* dA;
  float* dB;
  float* dC;
  float* dD;
  float* dbias;
  float* dh0;
  // workspace
  float* ws_ck;     // [batch][ntiles][N][dim]  state at each tile start, from the segment start at 0
  float* ws_qk;     // [batch][ntiles][dim]     sum of the decay exponent scale from the segment start
  float* ws_hloc;   // [batch][nseg][N][dim]    segment end state from a zero start
  float* ws_mloc;   // [batch][nseg][N][dim]    segment's outgoing adjoint from a zero end
  float* ws_hin;    // [batch][nseg][N][dim]    true state entering each segment
  float* ws_muin;   // [batch][nseg][N][dim]    true adjoint entering each segment from the right
  float* ws_qseg;   // [batch][nseg][dim]       the segment's summed exponent scale
  float* ws_dbc;    // [batch][dblocks][seqlen][2N] per-CTA partial dB (n < N) and dC
  float* ws_dA;     // [batch][nseg][N][dim]    per-segment partial dA
  float* ws_dD;     // [batch][nseg][dim]
  float* ws_dbias;  // [batch][nseg][dim]
};

bool scan_bwd_dstate_supported(int dstate);
cudaError_t launch_scan_bwd(const BwdParams& p, int dstate, bool bf16, cudaStream_t stream);

}  // namespace ssm
