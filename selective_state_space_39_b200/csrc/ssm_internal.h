// ssm_internal.h -- parameters shared by the C entry points (ssm_api.cu) and
// the kernel launchers (ssm_scan_kernels.cu). Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssm {

// Launch shape of the scan: threads per CTA and sequence steps per tile.
#ifndef SSM_TILE_STEPS
#define SSM_TILE_STEPS 16
#endif
#ifndef SSM_STAGES
#define SSM_STAGES 2
#endif
#ifndef SSM_CTA_THREADS
#define SSM_CTA_THREADS 128
#endif
constexpr int kScanThreads = SSM_CTA_THREADS;  // threads per CTA with 1 or 2 channels per thread
// Threads per CTA of the scan for a given number of channels per thread
// (4 channels per thread use half as many threads).
constexpr int scan_threads(int cpt) { return cpt == 4 ? kScanThreads / 2 : kScanThreads; }
constexpr int kScanTileSteps = SSM_TILE_STEPS;
constexpr int kScanStages = SSM_STAGES;
// Segment counts up to which the main pass composes the segment carries in
// its prologue (above it a separate kernel does, between the two passes).
constexpr int kScanPrologueCompose = 9;
// Per-CTA status codes written to the workspace status area.
constexpr int kCtaOk = 0;
constexpr int kCtaTimeout = 1;
// Default bound on any wait inside a kernel (nanoseconds).
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;

// How one call of the scan is split: the sequence is cut into `nseg`
// segments of `seg_steps` steps (a multiple of kScanTileSteps); segment
// carries live in the caller's workspace.
struct ScanPlan {
  int channels_per_thread;  // 2 for dstate <= 16, 1 above
  int dtile;                // channels per CTA
  int dtiles;               // CTAs along dim
  int nseg;                 // sequence segments
  int seg_steps;            // steps per segment
  int ctas_agg;             // CTAs of the carry pass (0 when nseg == 1)
  int ctas_main;            // CTAs of the main pass
  size_t off_status, off_state, off_sum, off_h0, bytes;
};

struct ScanParams {
  int batch, seqlen, dim;
  int nseg, seg_steps;
  int softplus;
  const void* x;
  const void* delta;
  const void* z;
  const void* B;
  const void* C;
  const float* A;
  const float* D;
  const float* bias;
  const float* h0;  // caller's h0 (read only when nseg == 1)
  void* y;
  float* h_last;
  float* ws_state;  // [batch][nseg-1][N][dim]
  float* ws_sum;    // [batch][nseg-1][dim]
  float* ws_h0;     // [batch][dim][N] copy of h0 taken by the carry pass
  int* status;      // one int per CTA: carry-pass CTAs first, then main pass
  uint64_t wait_limit_ns;
  int test_stall;   // test hook: CTA 0 of the main pass waits for 16 bytes that never arrive
};

struct alignas(64) ScanMaps {
  CUtensorMap x, delta, z, B, C;
};

struct DecodeParams {
  int batch, dim;
  int softplus;
  float* state;
  const void* x;
  const void* delta;
  const void* z;
  const void* B;
  const void* C;
  const float* A;
  const float* D;
  const float* bias;
  void* y;
};

// Kernel launchers (ssm_scan_kernels.cu). Return a cudaError_t.
// zoh: the exact zero-order-hold input term instead of Delta B.
cudaError_t launch_scan(const ScanPlan& plan, const ScanParams& p, const ScanMaps* maps,
                        bool use_tma, int dstate, bool bf16, bool zoh, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams& p, int dstate, bool bf16, bool zoh,
                          cudaStream_t stream);
bool scan_dstate_supported(int dstate);
// Resident CTAs per SM of the main-pass kernel on the current device (0 if
// the query fails).
int scan_ctas_per_sm(int dstate, bool bf16);

}  // namespace ssm
