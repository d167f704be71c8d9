// ssm_scan_kernels.cu -- sm_100a kernels of the selective state-space scan.
//
// What is computed (page "Mamba 논문 리뷰: Selective State Space Models로
// Transformer를 넘어서", youngju.dev; §2.2 discretised recurrence, §3.1
// softplus step, §3.3 selective_scan, §3.4 D skip and SiLU(z) gate):
//   Delta_t = softplus(delta_t + bias),  a_n(t) = exp(Delta_t A_n)
//   h_n(t)  = a_n(t) h_n(t-1) + Delta_t x_t B_n(t)
//   y_t     = (sum_n C_n(t) h_n(t) + D x_t) * SiLU(z_t)
//
// Design (B200): the path is bound by FP32 arithmetic, not by memory, at
// dstate = 16 (about 60 FP32 operations per 8 bytes moved), so the kernels
// are built to minimise FP32 pipe work per element:
//
//  * Each thread owns CPT (2) channels and their whole state in registers;
//    state pairs are updated with packed FP32x2 FMAs.
//  * Structured A (A[d,n] = (n+1) A[d,0], which Mamba's A = -exp(log(
//    arange(1, N+1))) init gives) is detected per channel from A itself;
//    then a_n = r^(n+1) with r = exp(Delta A_0): one exp and a multiply
//    chain instead of N exps. Other A falls back to one exp per state.
//  * Scaled recurrence. The state is kept as g_n = h_n / s_t with s_t the
//    step's input multiplier Delta_t x_t, so that
//        g_n(t) = (a_n(t) s_{t-1}/s_t) g_n(t-1) + B_n(t),   y_t = s_t sum_n C_n g_n
//    costs one multiply (the chain of alpha_n = s_{t-1}/s_t r^(n+1)) and two
//    FMAs per state, instead of two multiplies and two FMAs. A step whose
//    Delta_t x_t is below 2^-64 in magnitude (a zero input, a zero step)
//    keeps the previous scale and weights B by the exact Delta_t x_t / s_t in
//    a slow path: every step follows the recurrence exactly.
//  * The per-step scalar chain (softplus, exp, reciprocal, the gate) of a
//    thread's two channels goes through packed FP32x2 instructions.
//  * B and C (shared by all channels of a step) are widened to fp32 once per
//    CTA in shared memory and read as broadcasts.
//  * x, delta, z, B, C tiles of 16 steps are staged in shared memory by TMA
//    (cp.async.bulk.tensor, no multicast) through a 2-stage mbarrier
//    pipeline; every wait is bounded by a time limit.
//  * The sequence is split into segments so the whole GPU is busy: a carry
//    pass computes each segment's end state from a zero start (and the sum
//    of Delta, which gives the segment's decay exp(A_n sum Delta)), and the
//    affine carries are composed ((a1,b1) then (a2,b2) -> (a1 a2, a2 b1 +
//    b2), the associative scan of the state update) into every segment's
//    true start state (by the main pass's prologue for a few segments, by a
//    small kernel between the passes for many), from which the main pass
//    runs its segment exactly.
//
// bf16 io uses MUFU approximations (ex2/lg2/rcp/tanh.approx); fp32 io uses
// the accurate expf / log1pf / IEEE division.
#include <stdlib.h>

#include <algorithm>
#include <mutex>
#include <set>
#include <type_traits>
#include <utility>

#include "ssm_device.cuh"
#include "ssm_internal.h"

// Steps unrolled together inside a full tile, and the minimum resident CTAs
// per SM requested from the register allocator.
#ifndef SSM_TILE_UNROLL
#define SSM_TILE_UNROLL 4
#endif
// Packed FP32x2 instructions for the per-step scalar chain of a thread's
// channel pairs (1) or scalar instructions (0).
#ifndef SSM_PACK_SCALARS
#define SSM_PACK_SCALARS 1
#endif
// Channels per thread at dstate 16.
#ifndef SSM_CPT16
#define SSM_CPT16 2
#endif
#ifndef SSM_MIN_CTAS
#define SSM_MIN_CTAS 3
#endif
// The exact-ZOH variant keeps more per-state values live: fewer CTAs.
#ifndef SSM_MIN_CTAS_ZOH
#define SSM_MIN_CTAS_ZOH 2
#endif

namespace ssm {

namespace {

constexpr int kTileUnroll = SSM_TILE_UNROLL;
// Up to this many segments the main pass composes the carries in its
// prologue (a few dependent loads per CTA); above it scan_compose_kernel
// composes them once, between the passes.
constexpr int kPrologueCompose = kScanPrologueCompose;

constexpr int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Shared-memory layout of one pipeline stage. The carry pass (kAgg) stages
// x, delta and B; the main pass also z and C.
template <typename IOT, int N, int CPT, int NT, int T, bool kAgg>
struct ScanLayout {
  static constexpr int DT = NT * CPT;
  static constexpr int kTileBytes = T * DT * (int)sizeof(IOT);
  static constexpr int kBCBytes = T * N * (int)sizeof(IOT);
  static constexpr int kOffX = 0;
  static constexpr int kOffD = kTileBytes;
  static constexpr int kOffZ = 2 * kTileBytes;  // main pass only
  static constexpr int kOffB = (kAgg ? 2 : 3) * kTileBytes;
  static constexpr int kOffC = kOffB + round_up(kBCBytes, 128);  // main pass only
  static constexpr int kStageBytes = kOffB + (kAgg ? 1 : 2) * round_up(kBCBytes, 128);
  // fp32 copies of B (pre-scaled) and C for the tile: [2 buffers][1 or 2][T][N]
  static constexpr int kBCF32Bytes = 2 * (kAgg ? 1 : 2) * T * N * 4;
};

template <typename IOT, int N, int CPT, int NT, int T, int STAGES, bool kAgg>
constexpr int scan_smem_bytes() {
  using L = ScanLayout<IOT, N, CPT, NT, T, kAgg>;
  return STAGES * L::kStageBytes + L::kBCF32Bytes + 8 * STAGES;
}

// ------------------------------------------------ packed per-channel math --
// The scalar chain of a step works on the CPT channels of a thread together:
// pairs of channels go through one packed FP32x2 instruction.
template <int CPT>
__device__ __forceinline__ void vmul(float (&d)[CPT], const float (&a)[CPT],
                                     const float (&b)[CPT]) {
  if constexpr (!SSM_PACK_SCALARS) {
#pragma unroll
    for (int c = 0; c < CPT; ++c) d[c] = a[c] * b[c];
    return;
  }
#pragma unroll
  for (int c = 0; c + 1 < CPT; c += 2) {
    const float2 r = mul2(make_float2(a[c], a[c + 1]), make_float2(b[c], b[c + 1]));
    d[c] = r.x;
    d[c + 1] = r.y;
  }
  if constexpr (CPT & 1) d[CPT - 1] = a[CPT - 1] * b[CPT - 1];
}
template <int CPT>
__device__ __forceinline__ void vfma(float (&d)[CPT], const float (&a)[CPT], float b,
                                     const float (&c_)[CPT]) {
  if constexpr (!SSM_PACK_SCALARS) {
#pragma unroll
    for (int c = 0; c < CPT; ++c) d[c] = fmaf(a[c], b, c_[c]);
    return;
  }
#pragma unroll
  for (int c = 0; c + 1 < CPT; c += 2) {
    const float2 r = fma2(make_float2(a[c], a[c + 1]), make_float2(b, b),
                          make_float2(c_[c], c_[c + 1]));
    d[c] = r.x;
    d[c + 1] = r.y;
  }
  if constexpr (CPT & 1) d[CPT - 1] = fmaf(a[CPT - 1], b, c_[CPT - 1]);
}
template <int CPT>
__device__ __forceinline__ void vadd(float (&d)[CPT], const float (&a)[CPT], float b) {
  if constexpr (!SSM_PACK_SCALARS) {
#pragma unroll
    for (int c = 0; c < CPT; ++c) d[c] = a[c] + b;
    return;
  }
#pragma unroll
  for (int c = 0; c + 1 < CPT; c += 2) {
    const float2 r = add2(make_float2(a[c], a[c + 1]), make_float2(b, b));
    d[c] = r.x;
    d[c + 1] = r.y;
  }
  if constexpr (CPT & 1) d[CPT - 1] = a[CPT - 1] + b;
}

// Per-channel constants of a thread's CPT channels.
template <int CPT>
struct Chan {
  float A0[CPT];    // A[d,0] (natural units)
  float iA0[CPT];   // 1 / A[d,0] (exact zero-order hold, structured A)
  float bias[CPT];  // fast path: bias * log2(e); precise path: bias
  float Dd[CPT];    // skip weight (0 without D)
  bool valid[CPT];  // d < dim
};

// Per-step quantities of a thread's channels. They do not depend on the
// state, so they are computed one step ahead of the state update.
template <int CPT>
struct StepSc {
  float s[CPT];            // the state scale s_t
  float u[CPT];            // the step's input multiplier u_t (Delta x; ZOH: x / A_0, or x)
  float a0[CPT], a1[CPT];  // structured A: alpha of states 0 and 1 (rho r, rho r^2)
  float rr[CPT];           // r^2, the step of the alpha chain over state pairs
  float rho[CPT];          // s_{t-1} / s_t
  float q[CPT];            // Delta (precise) or Delta log2(e) (fast)
  float m0[CPT], m1[CPT];  // ZOH, structured A: exp(Delta A_n) - 1 for states 0 and 1
  float e2[CPT];           // ZOH, structured A: the step of that chain over state pairs
  bool floored;            // |u_t| < 2^-64 for one of the channels (exact slow path)
};

// Step size, decay base and state scale of a step for the thread's channels.
//
// Scaled state. The state is kept as g_n = h_n / s_t, so that with
// alpha_n = exp(Delta_t A_n) s_{t-1} / s_t
//     g_n(t) = alpha_n g_n(t-1) + (u_t / s_t) B_n(t),   y_t = s_t sum_n C_n g_n
// where u_t multiplies the input term (Delta_t x_t for the Delta B form). With
// s_t = u_t the input weight u_t / s_t is 1 and the update is one FMA per
// state. A step whose |u_t| is below 2^-64 (a zero input, a zero step) keeps
// s_t = s_{t-1} instead (rho = 1 exactly) and takes the slow path, which
// multiplies B by the exact weight u_t / s_t (zero for a zero input): every
// step follows the recurrence exactly, without any floor.
//
// Input term (kZoh = false, the deltaB of the selective_scan listing):
// Delta x B_n, u = Delta x (fast: times log2 e, matched by B pre-scaled by
// ln 2). Exact zero-order hold (kZoh, §2.2 B-bar): x B_n (exp(Delta A_n) -
// 1) / A_n. With structured A (kS) that is u B_n / (n+1) m_n with u = x / A_0
// and m_n = r^(n+1) - 1 (B pre-scaled by 1/(n+1)); m_n is built without
// cancellation from m_0 = expm1(Delta A_0): m_(n+2) = m_n r^2 + m_0 (1 + r),
// every term of one sign. Generic A under ZOH uses u = x and forms each
// state's factor itself.
template <bool kFast, bool kZoh, bool kS, bool kSlow, int CPT>
__device__ __forceinline__ void step_scalars(const float (&xv)[CPT], const float (&dv)[CPT],
                                             const Chan<CPT>& ch, int softplus, float sp_off,
                                             const float (&s_prev)[CPT], StepSc<CPT>& o) {
  float q[CPT], r[CPT];
  if constexpr (kFast) {
    // softplus in log2 units: max(v, log2(1 + 2^min(v, cut))); the max
    // picks v above the cut (and below it the softplus, which exceeds v).
    // sp_off = -inf turns the softplus off (q = v).
    float v[CPT], e[CPT];
    vfma(v, dv, kLog2e, ch.bias);
#pragma unroll
    for (int c = 0; c < CPT; ++c) e[c] = ex2_approx(fminf(v[c], kSoftplusCut * kLog2e));
    vadd(e, e, 1.f);
#pragma unroll
    for (int c = 0; c < CPT; ++c) e[c] = lg2_approx(e[c]);
    vadd(e, e, sp_off);
#pragma unroll
    for (int c = 0; c < CPT; ++c) q[c] = fmaxf(v[c], e[c]);
    float qa[CPT];
    vmul(qa, q, ch.A0);
#pragma unroll
    for (int c = 0; c < CPT; ++c) r[c] = ex2_approx(qa[c]);  // exp(Delta A0)
  } else {
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const float v = dv[c] + ch.bias[c];
      q[c] = softplus ? (v > kSoftplusCut ? v : log1pf(expf(v))) : v;
      // correctly rounded exp(Delta A_0): over a long run of steps without
      // input the state is this factor's product, so its rounding must not
      // lean one way (fp32 io only)
      r[c] = (float)exp((double)q[c] * (double)ch.A0[c]);
    }
  }
  float u[CPT];
  if constexpr (!kZoh) {
    vmul(u, q, xv);
  } else if constexpr (kS) {
    vmul(u, xv, ch.iA0);
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const float em1 = kFast ? r[c] - 1.f : expm1f(q[c] * ch.A0[c]);  // exp(Delta A_0) - 1
      o.m0[c] = em1;
      o.m1[c] = fmaf(em1, r[c], em1);
      o.e2[c] = em1 * (1.f + r[c]);
    }
  } else {
#pragma unroll
    for (int c = 0; c < CPT; ++c) u[c] = xv[c];
  }
  // The fast pass takes s_t = u_t and only notes whether a step was floored
  // (the CTA then runs its segment again in the slow pass); the slow pass
  // keeps s_{t-1} on a floored step (rho = 1 exactly).
  bool fl = false;
  float rs[CPT];
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const bool t = ch.valid[c] && fabsf(u[c]) < kScaleFloor;
    fl = fl || t;
    if constexpr (kSlow) o.s[c] = t ? s_prev[c] : u[c];
    else o.s[c] = u[c];
    if constexpr (kFast) rs[c] = rcp_approx(o.s[c]);
  }
  if constexpr (kFast) {
    vmul(o.rho, s_prev, rs);
    if constexpr (kSlow) {
#pragma unroll
      for (int c = 0; c < CPT; ++c)
        if (ch.valid[c] && fabsf(u[c]) < kScaleFloor) o.rho[c] = 1.f;
    }
  } else {
#pragma unroll
    for (int c = 0; c < CPT; ++c) o.rho[c] = s_prev[c] / o.s[c];  // 1 on a floored step
  }
  vmul(o.a0, o.rho, r);
  vmul(o.a1, o.a0, r);
  vmul(o.rr, r, r);
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    o.u[c] = u[c];
    o.q[c] = q[c];
  }
  o.floored = fl;
}

// -------------------------------------------------------------------------
// The scan kernel. kAgg = carry pass (segments 0..nseg-2: end state and
// sum of Delta, no output); !kAgg = main pass (all segments, y and h_last).
// Grid: (dtiles, segments, batch). Block: NT threads, CPT channels each.
template <typename IOT, int N, int CPT, int NT, int T, int STAGES, bool kAgg, bool kTma,
          bool kZoh>
__global__ void __launch_bounds__(NT, kZoh ? SSM_MIN_CTAS_ZOH : SSM_MIN_CTAS)
    scan_kernel(const ScanParams p,
                                                  const __grid_constant__ ScanMaps maps) {
  using IO = Io<IOT>;
  using L = ScanLayout<IOT, N, CPT, NT, T, kAgg>;
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  constexpr int DT = L::DT;
  constexpr int NP = N / 2;
  constexpr int kBCBufs = kAgg ? 1 : 2;
  static_assert(N % 2 == 0, "dstate must be even");

  extern __shared__ __align__(128) unsigned char smem[];
  float* bcf = reinterpret_cast<float*>(smem + STAGES * L::kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * L::kStageBytes + L::kBCF32Bytes);

  const int tid = threadIdx.x;
  const int dtile = blockIdx.x, seg = blockIdx.y, b = blockIdx.z;
  const int dim = p.dim, L_ = p.seqlen;
  const int d_local = tid * CPT;
  const int d_first = dtile * DT + d_local;
  const bool has_z = !kAgg && p.z != nullptr;
  const int softplus = p.softplus;
  const float sp_off = softplus ? 0.f : -INFINITY;
  const int t_begin = seg * p.seg_steps;
  const int t_end = min(t_begin + p.seg_steps, L_);
  const int ntiles = t_end > t_begin ? (t_end - t_begin + T - 1) / T : 0;

  const uint32_t stage_tx = (uint32_t)((kAgg ? 2 : (has_z ? 3 : 2)) * L::kTileBytes +
                                       kBCBufs * L::kBCBytes);

  // Test hook (ssm_scan_fwd with SSM_SCAN_TEST_STALL=1): the first CTA of the
  // main pass expects 16 bytes more than its first tile brings, so its
  // bounded wait runs out and it reports a timeout.
  const bool stall_here = !kAgg && p.test_stall && dtile == 0 && seg == 0 && b == 0;
  auto issue_tile = [&](int it) {
    unsigned char* st = smem + (it % STAGES) * L::kStageBytes;
    uint64_t* bar = &full[it % STAGES];
    const int t0 = t_begin + it * T;
    mbar_arrive_expect_tx(bar, stage_tx + ((stall_here && it == 0) ? 16u : 0u));
    tma_load_3d(st + L::kOffX, &maps.x, bar, dtile * DT, t0, b);
    tma_load_3d(st + L::kOffD, &maps.delta, bar, dtile * DT, t0, b);
    if (has_z) tma_load_3d(st + L::kOffZ, &maps.z, bar, dtile * DT, t0, b);
    tma_load_3d(st + L::kOffB, &maps.B, bar, 0, t0, b);
    if (!kAgg) tma_load_3d(st + L::kOffC, &maps.C, bar, 0, t0, b);
  };

  int issued = 0;  // tiles whose loads were issued in this pass (thread 0 only)
  bool aborted = false;
  // Completed phases of each stage's barrier (every thread keeps the count;
  // a second pass over the segment continues from it).
  int uses[STAGES];
#pragma unroll
  for (int s = 0; s < STAGES; ++s) uses[s] = 0;
  if (tid == 0) {
    if constexpr (kTma) {
      prefetch_tensormap(&maps.x);
      prefetch_tensormap(&maps.delta);
      prefetch_tensormap(&maps.B);
      if (!kAgg) prefetch_tensormap(&maps.C);
      if (has_z) prefetch_tensormap(&maps.z);
      for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
      fence_mbar_init();
    }
  }
  __syncthreads();
  auto issue_prologue = [&]() {
    if constexpr (kTma) {
      issued = 0;
      if (tid == 0)
        for (; issued < STAGES - 1 && issued < ntiles; ++issued) issue_tile(issued);
    }
  };
  issue_prologue();

  // ---- per-channel constants and structure of A ------------------------
  Chan<CPT> ch;
  bool structured = true;
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const int d = d_first + c;
    ch.valid[c] = d < dim;
    if (ch.valid[c]) {
      const float* Ar = p.A + (size_t)d * N;
      ch.A0[c] = Ar[0];
#pragma unroll
      for (int n = 1; n < N; ++n) structured = structured && (Ar[n] == (float)(n + 1) * Ar[0]);
      // the ZOH chain divides by A_0: A = 0 takes the per-state path
      if constexpr (kZoh) structured = structured && Ar[0] != 0.f;
      const float bias = p.bias ? p.bias[d] : 0.f;
      ch.bias[c] = kFast ? bias * kLog2e : bias;
      ch.Dd[c] = p.D ? p.D[d] : 0.f;
    } else {
      ch.A0[c] = -1.f;
      ch.bias[c] = 0.f;
      ch.Dd[c] = 0.f;
    }
    ch.iA0[c] = 1.f / ch.A0[c];
  }
  // One code path per CTA: the multiply-chain path when every channel of the
  // CTA has structured A, one exp per state otherwise.
  const bool cta_structured = __syncthreads_and(structured) != 0;

  // ---- initial state ----------------------------------------------------
  float2 g[CPT][NP];  // scaled state g = h / s_prev
  float s_prev[CPT];
  float qsum[CPT];
  // The segment's start state (h0, zero, or the composed carries); called
  // again when the segment is run a second time in the slow pass.
  auto load_start = [&]() {
    const int nagg = p.nseg - 1;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      s_prev[c] = 1.f;
      qsum[c] = 0.f;
#pragma unroll
      for (int k = 0; k < NP; ++k) g[c][k] = make_float2(0.f, 0.f);
      if (!ch.valid[c]) continue;
      const int d = d_first + c;
      if constexpr (kAgg) {
        // Segment 0 starts from h0 and keeps a copy of it for the main pass
        // (so that h_last may alias h0); later segments start from zero.
        if (seg == 0 && p.h0) {
          const float2* src = reinterpret_cast<const float2*>(p.h0 + ((size_t)b * dim + d) * N);
          float2* cpy = reinterpret_cast<float2*>(p.ws_h0 + ((size_t)b * dim + d) * N);
#pragma unroll
          for (int k = 0; k < NP; ++k) {
            g[c][k] = src[k];
            cpy[k] = g[c][k];
          }
        }
      } else {
        const float* h0 = p.nseg > 1 ? (p.h0 ? p.ws_h0 : nullptr) : p.h0;
        if (seg > 0 && p.nseg > kPrologueCompose) {
          // The state entering this segment, composed from the carries by
          // scan_compose_kernel (segment 1: segment 0's end state itself).
          const float* st = p.ws_state + ((size_t)b * nagg + (seg - 1)) * N * dim + d;
#pragma unroll
          for (int k = 0; k < NP; ++k)
            g[c][k] = make_float2(__ldcg(st + (size_t)(2 * k) * dim),
                                  __ldcg(st + (size_t)(2 * k + 1) * dim));
        } else if (seg > 0) {
          // Few segments: compose here. Segment 0's end state (it includes
          // h0), then the carries h <- exp(A_n S_j) h + e_j of segments
          // 1 .. seg-1, the next carry's loads issued before the current one
          // is applied.
          const float* st0 = p.ws_state + ((size_t)b * nagg) * N * dim + d;
#pragma unroll
          for (int k = 0; k < NP; ++k)
            g[c][k] = make_float2(__ldcg(st0 + (size_t)(2 * k) * dim),
                                  __ldcg(st0 + (size_t)(2 * k + 1) * dim));
          float bj[N], sd = 0.f;
          auto load_carry = [&](int j) {
            sd = __ldcg(p.ws_sum + ((size_t)b * nagg + j) * dim + d);
            const float* stj = p.ws_state + ((size_t)b * nagg + j) * N * dim + d;
#pragma unroll
            for (int n = 0; n < N; ++n) bj[n] = __ldcg(stj + (size_t)n * dim);
          };
          if (seg > 1) load_carry(1);
          for (int j = 1; j < seg; ++j) {
            float cur[N];
            const float sdc = sd;
#pragma unroll
            for (int n = 0; n < N; ++n) cur[n] = bj[n];
            if (j + 1 < seg) load_carry(j + 1);
            if (cta_structured) {
              // exp(A_n S) = e^(n+1) with e = exp(A_0 S)
              const float e = expf(ch.A0[c] * sdc);
              float en = e;
#pragma unroll
              for (int k = 0; k < NP; ++k) {
                const float e0 = en, e1 = en * e;
                en = e1 * e;
                g[c][k].x = fmaf(e0, g[c][k].x, cur[2 * k]);
                g[c][k].y = fmaf(e1, g[c][k].y, cur[2 * k + 1]);
              }
            } else {
#pragma unroll
              for (int k = 0; k < NP; ++k) {
                const float2 An = *reinterpret_cast<const float2*>(p.A + (size_t)d * N + 2 * k);
                g[c][k].x = fmaf(expf(An.x * sdc), g[c][k].x, cur[2 * k]);
                g[c][k].y = fmaf(expf(An.y * sdc), g[c][k].y, cur[2 * k + 1]);
              }
            }
          }
        } else if (h0) {
          const float2* src = reinterpret_cast<const float2*>(h0 + ((size_t)b * dim + d) * N);
#pragma unroll
          for (int k = 0; k < NP; ++k) g[c][k] = src[k];
        }
      }
    }
  };
  // The main pass may start while the carry pass finishes (programmatic
  // dependent launch): everything above reads only inputs; the carries and
  // the h0 copy are read after this wait.
  if constexpr (!kAgg) griddep_wait();
  load_start();

  // ---- per-step pieces ----------------------------------------------------
  // vector stores of the thread's CPT outputs: all valid and rows aligned
  const bool vec_store = CPT >= 2 && (p.dim % CPT) == 0 && ch.valid[CPT - 1];
  struct StepIn {
    float x[CPT], d[CPT], z[CPT];
  };
  // x, delta, z of smem row `row` for this thread's channels
  auto load_in = [&](const unsigned char* st, int row) {
    StepIn in;
    const IOT* sx = reinterpret_cast<const IOT*>(st + L::kOffX) + d_local + row * DT;
    const IOT* sdl = reinterpret_cast<const IOT*>(st + L::kOffD) + d_local + row * DT;
    const IOT* sz = reinterpret_cast<const IOT*>(st + L::kOffZ) + d_local + row * DT;
    if constexpr (CPT == 2) {
      const float2 x2 = IO::load2(sx), d2 = IO::load2(sdl);
      in.x[0] = x2.x; in.x[1] = x2.y; in.d[0] = d2.x; in.d[1] = d2.y;
      if (!kAgg && has_z) {
        const float2 z2 = IO::load2(sz);
        in.z[0] = z2.x; in.z[1] = z2.y;
      } else {
        in.z[0] = in.z[1] = 0.f;
      }
    } else if constexpr (CPT == 4) {
      const float4 x4 = IO::load4(sx), d4 = IO::load4(sdl);
      in.x[0] = x4.x; in.x[1] = x4.y; in.x[2] = x4.z; in.x[3] = x4.w;
      in.d[0] = d4.x; in.d[1] = d4.y; in.d[2] = d4.z; in.d[3] = d4.w;
      if (!kAgg && has_z) {
        const float4 z4 = IO::load4(sz);
        in.z[0] = z4.x; in.z[1] = z4.y; in.z[2] = z4.z; in.z[3] = z4.w;
      } else {
        in.z[0] = in.z[1] = in.z[2] = in.z[3] = 0.f;
      }
    } else {
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        in.x[c] = IO::load(sx + c);
        in.d[c] = IO::load(sdl + c);
        in.z[c] = (!kAgg && has_z) ? IO::load(sz + c) : 0.f;
      }
    }
    return in;
  };

  // Rows of A for the one-exp-per-state path, held in registers (loaded by
  // run_tiles for that path only).
  float2 Areg[CPT][NP];

  // State update (and readout) of one step, given its precomputed scalars.
  // kSlow: some channel's input multiplier is below the floor this step; B is
  // then weighted by u_t / s_t (exactly 1 for the other channels).
  auto state_step = [&](auto kStructTag, auto kSlowTag, const StepIn& in, const StepSc<CPT>& sc,
                        const float* Bt, const float* Ct, int t_abs) {
    constexpr bool kS = decltype(kStructTag)::value;
    constexpr bool kSlow = decltype(kSlowTag)::value;
    const float2* B2 = reinterpret_cast<const float2*>(Bt);
    const float2* C2 = reinterpret_cast<const float2*>(Ct);
    (void)C2;
    float2 acc[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      acc[c] = make_float2(0.f, 0.f);
      float2 w2 = make_float2(1.f, 1.f);
      if constexpr (kSlow) {
        // input weight u_t / s_t: exactly 1 unless the step is floored
        const bool f = ch.valid[c] && fabsf(sc.u[c]) < kScaleFloor;
        const float w = !f ? 1.f : kFast ? sc.u[c] * rcp_approx(sc.s[c]) : sc.u[c] / sc.s[c];
        w2 = make_float2(w, w);
      }
      if constexpr (kS) {
        // alpha_n = rho r^(n+1), two states at a time: (a0, a1) * (r^2)^k
        float2 a = make_float2(sc.a0[c], sc.a1[c]);
        const float2 rr = make_float2(sc.rr[c], sc.rr[c]);
        if constexpr (kZoh) {
          // input B_n / (n+1) m_n, m pairs stepped by m <- m r^2 + m_0 (1 + r)
          float2 m = make_float2(sc.m0[c], sc.m1[c]);
          const float2 e2 = make_float2(sc.e2[c], sc.e2[c]);
          if constexpr (kSlow) m = mul2(m, w2);
#pragma unroll
          for (int k = 0; k < NP; ++k) {
            g[c][k] = fma2(a, g[c][k], mul2(B2[k], m));
            if (k + 1 < NP) {
              a = mul2(a, rr);
              m = fma2(m, rr, kSlow ? mul2(e2, w2) : e2);
            }
            if constexpr (!kAgg) acc[c] = fma2(C2[k], g[c][k], acc[c]);
          }
        } else {
#pragma unroll
          for (int k = 0; k < NP; ++k) {
            g[c][k] = fma2(a, g[c][k], kSlow ? mul2(B2[k], w2) : B2[k]);
            if (k + 1 < NP) a = mul2(a, rr);
            if constexpr (!kAgg) acc[c] = fma2(C2[k], g[c][k], acc[c]);
          }
        }
      } else {
        const float rho = sc.rho[c], q = sc.q[c];
#pragma unroll
        for (int k = 0; k < NP; ++k) {
          float2 a;
          const float A_lo = Areg[c][k].x, A_hi = Areg[c][k].y;
          const float e_lo = kFast ? ex2_approx(q * A_lo) : expf(q * A_lo);
          const float e_hi = kFast ? ex2_approx(q * A_hi) : expf(q * A_hi);
          a = make_float2(rho * e_lo, rho * e_hi);
          float2 in2;
          if constexpr (kZoh) {
            // input B_n (exp(Delta A_n) - 1) / A_n (Delta where A_n = 0), u = x
            const float dt = kFast ? q * kLn2 : q;
            auto coef = [&](float An, float e) {
              if (An == 0.f) return dt;
              return kFast ? (e - 1.f) * rcp_approx(An) : expm1f(dt * An) / An;
            };
            in2 = make_float2(B2[k].x * coef(A_lo, e_lo), B2[k].y * coef(A_hi, e_hi));
          } else {
            in2 = B2[k];
          }
          if constexpr (kSlow) in2 = mul2(in2, w2);
          g[c][k] = fma2(a, g[c][k], in2);
          if constexpr (!kAgg) acc[c] = fma2(C2[k], g[c][k], acc[c]);
        }
      }
    }
    if constexpr (!kAgg) {
      // y = (s sum_n C_n g_n + D x) SiLU(z), the channels in packed pairs
      float ysum[CPT], dx[CPT], yv[CPT];
#pragma unroll
      for (int c = 0; c < CPT; ++c) ysum[c] = acc[c].x + acc[c].y;
      vmul(dx, ch.Dd, in.x);
#pragma unroll
      for (int c = 0; c + 1 < CPT; c += 2) {
        const float2 r = fma2(make_float2(sc.s[c], sc.s[c + 1]), make_float2(ysum[c], ysum[c + 1]),
                              make_float2(dx[c], dx[c + 1]));
        yv[c] = r.x;
        yv[c + 1] = r.y;
      }
      if constexpr (CPT & 1) yv[CPT - 1] = fmaf(sc.s[CPT - 1], ysum[CPT - 1], dx[CPT - 1]);
      if (has_z) {
        if constexpr (kFast) {
          // z sigmoid(z) = hz + hz tanh(hz), hz = z / 2
          float hz[CPT], th[CPT];
#pragma unroll
          for (int c = 0; c < CPT; ++c) hz[c] = 0.5f * in.z[c];
#pragma unroll
          for (int c = 0; c < CPT; ++c) th[c] = tanh_approx(hz[c]);
#pragma unroll
          for (int c = 0; c + 1 < CPT; c += 2) {
            const float2 sg = fma2(make_float2(hz[c], hz[c + 1]), make_float2(th[c], th[c + 1]),
                                   make_float2(hz[c], hz[c + 1]));
            const float2 r = mul2(make_float2(yv[c], yv[c + 1]), sg);
            yv[c] = r.x;
            yv[c + 1] = r.y;
          }
          if constexpr (CPT & 1) yv[CPT - 1] *= fmaf(hz[CPT - 1], th[CPT - 1], hz[CPT - 1]);
        } else {
#pragma unroll
          for (int c = 0; c < CPT; ++c) yv[c] *= in.z[c] / (1.f + expf(-in.z[c]));
        }
      }
      IOT* yrow = reinterpret_cast<IOT*>(p.y) + ((size_t)b * L_ + t_abs) * dim + d_first;
      if (!p.y) {
        // state only (y not wanted)
      } else if (vec_store) {
        if constexpr (CPT == 4)
          IO::store4(yrow, yv[0], yv[1], yv[2], yv[3]);
        else
          IO::store2(yrow, yv[0], yv[CPT - 1]);
      } else {
#pragma unroll
        for (int c = 0; c < CPT; ++c)
          if (ch.valid[c]) IO::store(yrow + c, yv[c]);
      }
    }
  };

  // ---- tile loop ----------------------------------------------------------
  // One pass over the segment's tiles. The fast pass (kSlowTag false) stops
  // with kPassFloored at the first tile boundary after a floored step; the
  // slow pass handles those steps exactly. kPassTimeout: a wait ran out.
  constexpr int kPassDone = 0, kPassFloored = 1, kPassTimeout = 2;
  auto run_tiles = [&](auto kStructTag, auto kSlowTag) -> int {
    constexpr bool kS = decltype(kStructTag)::value;
    constexpr bool kSlow = decltype(kSlowTag)::value;
    if constexpr (!kS) {
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const float2* Ar =
            reinterpret_cast<const float2*>(p.A + (size_t)(ch.valid[c] ? d_first + c : 0) * N);
#pragma unroll
        for (int k = 0; k < NP; ++k) Areg[c][k] = __ldg(Ar + k);
      }
    }
    bool floored = false;  // this thread saw a floored step (fast pass)
    for (int it = 0; it < ntiles; ++it) {
      const int buf = it & 1;
      unsigned char* st;
      if constexpr (kTma) {
        const int stage = it % STAGES;
        st = smem + stage * L::kStageBytes;
        const bool ok = mbar_wait_bounded(&full[stage], (uint32_t)(uses[stage] & 1),
                                          p.wait_limit_ns);
        if (__syncthreads_or(!ok)) {
          // Let the loads already issued land (bounded) before the CTA's
          // shared memory is released.
          if (tid == 0)
            for (int j = it; j < issued; ++j)
              (void)mbar_wait_bounded(&full[j % STAGES], (uint32_t)(uses[j % STAGES] & 1),
                                      1000000ull);
          return kPassTimeout;
        }
        ++uses[stage];
      } else {
        st = smem;
        __syncthreads();  // every thread is done with the previous tile
        const int t0 = t_begin + it * T;
        const IOT* gx = reinterpret_cast<const IOT*>(p.x);
        const IOT* gd = reinterpret_cast<const IOT*>(p.delta);
        const IOT* gz = reinterpret_cast<const IOT*>(p.z);
        IOT* sx = reinterpret_cast<IOT*>(st + L::kOffX);
        IOT* sd = reinterpret_cast<IOT*>(st + L::kOffD);
        IOT* sz = reinterpret_cast<IOT*>(st + L::kOffZ);
        for (int i = tid; i < T * DT; i += NT) {
          const int tt = t0 + i / DT, dd = dtile * DT + i % DT;
          const bool in = tt < L_ && dd < dim;
          const size_t gi = ((size_t)b * L_ + tt) * dim + dd;
          sx[i] = in ? gx[gi] : IOT(0);
          sd[i] = in ? gd[gi] : IOT(0);
          if (has_z) sz[i] = in ? gz[gi] : IOT(0);
        }
        const IOT* gb = reinterpret_cast<const IOT*>(p.B);
        const IOT* gc = reinterpret_cast<const IOT*>(p.C);
        IOT* sb = reinterpret_cast<IOT*>(st + L::kOffB);
        IOT* sc = reinterpret_cast<IOT*>(st + L::kOffC);
        for (int i = tid; i < T * N; i += NT) {
          const int tt = t0 + i / N;
          const size_t gi = ((size_t)b * L_ + tt) * N + i % N;
          sb[i] = tt < L_ ? gb[gi] : IOT(0);
          if (!kAgg) sc[i] = tt < L_ ? gc[gi] : IOT(0);
        }
        __syncthreads();
      }

      // widen B (times ln2 on the fast path) and C to fp32
      {
        const IOT* sb = reinterpret_cast<const IOT*>(st + L::kOffB);
        const IOT* sc = reinterpret_cast<const IOT*>(st + L::kOffC);
        float* fb = bcf + (buf * kBCBufs + 0) * T * N;
        float* fc = bcf + (buf * kBCBufs + (kBCBufs - 1)) * T * N;
        for (int i = tid; i < T * N; i += NT) {
          // Delta B (fast: ln 2, see step_scalars); ZOH: 1/(n+1) (structured) or 1
          float bscale;
          if constexpr (kZoh) bscale = cta_structured ? 1.f / (float)(i % N + 1) : 1.f;
          else bscale = kFast ? kLn2 : 1.f;
          fb[i] = IO::load(sb + i) * bscale;
          if (!kAgg) fc[i] = IO::load(sc + i);
        }
      }
      // The barrier also tells every thread whether a step of the previous
      // tile was floored; the fast pass then stops here (with two stages no
      // copy is in flight at this point: the next tile is issued below).
      if (__syncthreads_or(floored)) {
        if constexpr (kTma) {
          // tiles it+1 .. (issued so far) - 1 are in flight (none with two
          // stages): every thread waits for them, keeping the phase counts
          const int iss = min(ntiles, STAGES - 1 + it);
          for (int j = it + 1; j < iss; ++j) {
            (void)mbar_wait_bounded(&full[j % STAGES], (uint32_t)(uses[j % STAGES] & 1),
                                    p.wait_limit_ns);
            ++uses[j % STAGES];
          }
        }
        return kPassFloored;
      }
      if constexpr (kTma) {
        // The stage consumed by the previous tile is free: refill it.
        if (tid == 0 && issued < ntiles) issue_tile(issued++);
      }

      const float* fb = bcf + (buf * kBCBufs + 0) * T * N;
      const float* fc = bcf + (buf * kBCBufs + (kBCBufs - 1)) * T * N;
      const int t0 = t_begin + it * T;
      const int steps = min(T, t_end - t0);
      // Software pipeline: the scalar chain of step row+1 (which does not
      // depend on the state) is computed in the same iteration as the state
      // update of step row, so the two interleave. Full tiles are unrolled
      // (all shared-memory offsets become constants); the look-ahead at the
      // last row re-reads that row and its result is discarded.
      auto step_loop = [&](auto kFullTag, int nsteps) {
        constexpr bool kFull = decltype(kFullTag)::value;
        const int nst = kFull ? T : nsteps;
        StepIn in_next = load_in(st, 0);
        StepSc<CPT> sc_next;
        step_scalars<kFast, kZoh, kS, kSlow>(in_next.x, in_next.d, ch, softplus, sp_off, s_prev,
                                             sc_next);
#pragma unroll(kFull ? kTileUnroll : 1)
        for (int row = 0; row < nst; ++row) {
          const StepIn in = in_next;
          const StepSc<CPT> sc = sc_next;
          if constexpr (kAgg) {
#pragma unroll
            for (int c = 0; c < CPT; ++c) qsum[c] += sc.q[c];
          }
          if constexpr (!kSlow) floored = floored || sc.floored;
          in_next = load_in(st, min(row + 1, nst - 1));
          step_scalars<kFast, kZoh, kS, kSlow>(in_next.x, in_next.d, ch, softplus, sp_off, sc.s,
                                               sc_next);
          state_step(kStructTag, kSlowTag, in, sc, fb + row * N, fc + row * N, t0 + row);
#pragma unroll
          for (int c = 0; c < CPT; ++c) s_prev[c] = sc.s[c];  // scale of the last step
        }
      };
      if (steps == T)
        step_loop(std::true_type{}, T);
      else
        step_loop(std::false_type{}, steps);
    }
    // floored steps in the last tile
    if (__syncthreads_or(floored)) return kPassFloored;
    return kPassDone;
  };
  // Fast pass; a segment with a floored step (a zero input or step, rare
  // outside padding) is run again from its start in the slow pass, which
  // overwrites the fast pass's outputs.
  int pass;
  if (cta_structured)
    pass = run_tiles(std::true_type{}, std::false_type{});
  else
    pass = run_tiles(std::false_type{}, std::false_type{});
  if (pass == kPassFloored) {
    load_start();
    issue_prologue();
    if (cta_structured)
      pass = run_tiles(std::true_type{}, std::true_type{});
    else
      pass = run_tiles(std::false_type{}, std::true_type{});
  }
  aborted = pass == kPassTimeout;

  // ---- outputs of the segment ------------------------------------------
  if (!aborted) {
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      if (!ch.valid[c]) continue;
      const int d = d_first + c;
      if constexpr (kAgg) {
        const int nagg = p.nseg - 1;
        p.ws_sum[((size_t)b * nagg + seg) * dim + d] = kFast ? qsum[c] * kLn2 : qsum[c];
        float* dst = p.ws_state + ((size_t)b * nagg + seg) * N * dim + d;
#pragma unroll
        for (int k = 0; k < NP; ++k) {
          dst[(size_t)(2 * k) * dim] = s_prev[c] * g[c][k].x;
          dst[(size_t)(2 * k + 1) * dim] = s_prev[c] * g[c][k].y;
        }
      } else if (p.h_last && seg == p.nseg - 1) {
        float2* dst = reinterpret_cast<float2*>(p.h_last + ((size_t)b * dim + d) * N);
        const float2 sp = make_float2(s_prev[c], s_prev[c]);
#pragma unroll
        for (int k = 0; k < NP; ++k) dst[k] = mul2(sp, g[c][k]);
      }
    }
  }
  if (tid == 0 && p.status) {
    const int ctas_agg = kAgg ? 0 : (p.nseg > 1 ? p.batch * (p.nseg - 1) * (int)gridDim.x : 0);
    const int id = ctas_agg + (b * (int)gridDim.y + seg) * (int)gridDim.x + dtile;
    p.status[id] = aborted ? kCtaTimeout : kCtaOk;
  }
  if constexpr (kAgg) {
    // This CTA's carries are written: the main pass may proceed past its
    // wait once every CTA of this grid has done the same.
    __syncthreads();
    griddep_launch_dependents();
  }
}

// -------------------------------------------------------------------------
// Carry composition between the two passes. Segment j (< nseg-1) acts on the
// state as h -> exp(A_n S_j) h + e_j (S_j its sum of Delta, e_j its end state
// from zero; segment 0's e_0 already includes h0). The state entering segment
// j+1 is P_j = exp(A_n S_j) P_{j-1} + e_j, P_0 = e_0: one thread per
// (batch, state, channel) runs that chain over the segments, in place
// (e_j is replaced by P_j), with the loads of 8 segments issued ahead.
__global__ void __launch_bounds__(256) scan_compose_kernel(const ScanParams p, int dstate) {
  const int nagg = p.nseg - 1;
  const size_t per_b = (size_t)dstate * p.dim;
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  griddep_wait();  // the carry pass has finished and its writes are visible
  if (i < (size_t)p.batch * per_b) {
    const int b = (int)(i / per_b);
    const size_t nd = i % per_b;  // n * dim + d
    const int n = (int)(nd / p.dim), d = (int)(nd % p.dim);
    const float An = p.A[(size_t)d * dstate + n];
    float* st = p.ws_state + (size_t)b * nagg * per_b + nd;
    const float* sum = p.ws_sum + (size_t)b * nagg * p.dim + d;
    float P = __ldcg(st);
    constexpr int kAhead = 8;
    for (int j0 = 1; j0 < nagg; j0 += kAhead) {
      float e[kAhead], sd[kAhead];
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        if (j0 + u < nagg) {
          e[u] = __ldcg(st + (size_t)(j0 + u) * per_b);
          sd[u] = __ldcg(sum + (size_t)(j0 + u) * p.dim);
        }
      }
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        if (j0 + u < nagg) {
          P = fmaf(expf(An * sd[u]), P, e[u]);
          st[(size_t)(j0 + u) * per_b] = P;
        }
      }
    }
  }
  __syncthreads();
  griddep_launch_dependents();
}

// -------------------------------------------------------------------------
// Decode: one step of the recurrence per (batch, channel). LPC lanes share a
// channel, SPT states each (one float4 of the state per lane, so a warp reads
// and writes contiguous runs of the (batch, dim, dstate) state); y is reduced
// across the LPC lanes by shuffles. Every load of a thread is issued before
// any arithmetic, so each thread makes a single round trip to memory: the
// kernel is otherwise bound by the latency of its waves, not by bandwidth.
// States per thread of the one-shot decode kernel (8: two groups of four,
// where N allows) and batch rows per thread (the row of A is loaded once for
// them: with the state it is most of a thread's bytes in flight).
#ifndef SSM_DEC_SPT8
#define SSM_DEC_SPT8 1
#endif
#ifndef SSM_DEC_RB
#define SSM_DEC_RB 2
#endif
template <int N>
struct DecShape {
  static constexpr int SPT = (SSM_DEC_SPT8 && N >= 8) ? 8 : (N % 4 == 0 ? 4 : 2);
  static constexpr int GS = SPT >= 4 ? 4 : SPT;  // states per partial sum of y
  static constexpr int NG = SPT / GS;            // partial sums per thread and row
  static constexpr int LPC = N / SPT;            // lanes per channel
  static constexpr int RB = SSM_DEC_RB;          // batch rows per thread
  static_assert(LPC <= 32 && (LPC & (LPC - 1)) == 0, "lanes per channel must divide a warp");
};

template <typename IOT, int N, bool kZoh>
__global__ void __launch_bounds__(256) decode_kernel(const DecodeParams p) {
  using IO = Io<IOT>;
  using S = DecShape<N>;
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  constexpr int SPT = S::SPT, GS = S::GS, NG = S::NG, LPC = S::LPC, RB = S::RB;
  // grid: x covers one batch row's channels (LPC lanes each), y groups of RB
  // batch rows; no division by the run-time dim
  const int tl = blockIdx.x * blockDim.x + threadIdx.x;
  const int lane_in = tl % LPC;
  const bool valid = tl / LPC < p.dim;
  const int d = valid ? tl / LPC : p.dim - 1;
  const int b0 = blockIdx.y * RB;

  // ---- all loads first ----
  const float* Ar = p.A + (size_t)d * N + lane_in * SPT;
  float a[SPT], h[RB][SPT], bb[RB][SPT], cv[RB][SPT], xv[RB], draw[RB], zz[RB];
  if constexpr (SPT % 4 == 0) {
#pragma unroll
    for (int v = 0; v < SPT; v += 4) {
      const float4 a4 = __ldg(reinterpret_cast<const float4*>(Ar + v));
      a[v] = a4.x; a[v + 1] = a4.y; a[v + 2] = a4.z; a[v + 3] = a4.w;
    }
  } else {
    const float2 a2 = __ldg(reinterpret_cast<const float2*>(Ar));
    a[0] = a2.x; a[1] = a2.y;
  }
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    const int b = min(b0 + r, p.batch - 1);  // rows past the end load row batch-1
    const size_t cc = (size_t)b * p.dim + d;
    const float* hp = p.state + cc * N + lane_in * SPT;
    const IOT* Bp = reinterpret_cast<const IOT*>(p.B) + (size_t)b * N + lane_in * SPT;
    const IOT* Cp = reinterpret_cast<const IOT*>(p.C) + (size_t)b * N + lane_in * SPT;
    if constexpr (SPT % 4 == 0) {
#pragma unroll
      for (int v = 0; v < SPT; v += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(hp + v);
        h[r][v] = t4.x; h[r][v + 1] = t4.y; h[r][v + 2] = t4.z; h[r][v + 3] = t4.w;
        const float4 b4 = IO::load4(Bp + v), c4 = IO::load4(Cp + v);
        bb[r][v] = b4.x; bb[r][v + 1] = b4.y; bb[r][v + 2] = b4.z; bb[r][v + 3] = b4.w;
        cv[r][v] = c4.x; cv[r][v + 1] = c4.y; cv[r][v + 2] = c4.z; cv[r][v + 3] = c4.w;
      }
    } else {
      const float2 t2 = *reinterpret_cast<const float2*>(hp);
      h[r][0] = t2.x; h[r][1] = t2.y;
      const float2 b2 = IO::load2(Bp), c2 = IO::load2(Cp);
      bb[r][0] = b2.x; bb[r][1] = b2.y; cv[r][0] = c2.x; cv[r][1] = c2.y;
    }
    xv[r] = IO::load(reinterpret_cast<const IOT*>(p.x) + cc);
    draw[r] = IO::load(reinterpret_cast<const IOT*>(p.delta) + cc);
    zz[r] = p.z ? IO::load(reinterpret_cast<const IOT*>(p.z) + cc) : 0.f;
  }
  const float bias = p.bias ? p.bias[d] : 0.f;
  const float Dd = p.D ? p.D[d] : 0.f;

  // ---- arithmetic, row by row ----
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    const float v = draw[r] + bias;
    float dt;
    if (!p.softplus) {
      dt = v;
    } else if constexpr (kFast) {
      dt = v > kSoftplusCut ? v : kLn2 * lg2_approx(1.f + ex2_approx(v * kLog2e));
    } else {
      dt = v > kSoftplusCut ? v : log1pf(expf(v));
    }
    const float dx = dt * xv[r];
    const float dtl = kFast ? dt * kLog2e : dt;
    float part[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < GS; ++j) {
        const int k = g * GS + j;
        const float e = kFast ? ex2_approx(dtl * a[k]) : expf(dtl * a[k]);
        if constexpr (kZoh) {
          // exact ZOH input: x B_n (exp(Delta A_n) - 1) / A_n (Delta where A_n = 0)
          const float coef = a[k] == 0.f ? dt
                             : kFast     ? (e - 1.f) * rcp_approx(a[k])
                                         : expm1f(dt * a[k]) / a[k];
          h[r][k] = fmaf(e, h[r][k], xv[r] * coef * bb[r][k]);
        } else {
          h[r][k] = fmaf(e, h[r][k], dx * bb[r][k]);
        }
        acc = fmaf(cv[r][k], h[r][k], acc);
      }
      part[g] = acc;
    }
    // y: the partial sums of the channel's N / GS groups of GS states combined
    // by the same pairing as an xor tree over one group per lane (group g with
    // g ^ off, off = N / (2 GS) .. 1), so every kernel sums in the same order
#pragma unroll
    for (int off = N / GS / 2; off >= NG && off >= 1; off >>= 1)
#pragma unroll
      for (int g = 0; g < NG; ++g) part[g] += __shfl_xor_sync(0xffffffffu, part[g], off / NG);
    float acc = part[0];
    if constexpr (NG == 2) acc = part[0] + part[1];
    const int b = b0 + r;
    if (!valid || b >= p.batch) continue;
    const size_t cc = (size_t)b * p.dim + d;
    float* hp = p.state + cc * N + lane_in * SPT;
#pragma unroll
    for (int v = 0; v < SPT; v += (SPT % 4 == 0 ? 4 : 2)) {
      if constexpr (SPT % 4 == 0)
        *reinterpret_cast<float4*>(hp + v) =
            make_float4(h[r][v], h[r][v + 1], h[r][v + 2], h[r][v + 3]);
      else
        *reinterpret_cast<float2*>(hp + v) = make_float2(h[r][v], h[r][v + 1]);
    }
    if (lane_in == 0) {
      float yy = fmaf(Dd, xv[r], acc);
      if (p.z) {
        if constexpr (kFast) {
          const float hz = 0.5f * zz[r];
          yy *= fmaf(hz, tanh_approx(hz), hz);
        } else {
          yy *= zz[r] / (1.f + expf(-zz[r]));
        }
      }
      IO::store(reinterpret_cast<IOT*>(p.y) + cc, yy);
    }
  }
}

// -------------------------------------------------------------------------
// Decode, pipelined (SSM_DECODE_PIPELINED=1): the same step as decode_kernel for the common aligned
// shapes, but a CTA walks tiles of kDecTB batch rows x (1024 / N) channels
// (16 KB of state) and brings the next tile's state, A rows and inputs into
// shared memory by cp.async while it computes the current one. The state is
// a pure stream (read and written once per call); a thread of the one-shot
// kernel waits one memory round trip for its 16 bytes, whereas here every
// CTA keeps a whole tile in flight. Grid: at most the resident CTAs, each
// taking every gridDim.x-th tile.
constexpr int kDecTB = 4;  // batch rows per tile

template <typename IOT, int N>
struct Dec2Layout {
  static constexpr int TD = 1024 / N;  // channels per tile
  static constexpr int kState = kDecTB * TD * N;  // floats
  static constexpr int kA = TD * N;               // floats
  static constexpr int kIo = kDecTB * TD;         // x, delta, z elements each
  static constexpr int kBC = kDecTB * N;          // B, C elements each
  // stage: state | A | D | bias | x | delta | z | B | C
  static constexpr int kOffA = kState * 4;
  static constexpr int kOffD = kOffA + kA * 4;
  static constexpr int kOffBias = kOffD + TD * 4;
  static constexpr int kOffX = kOffBias + TD * 4;
  static constexpr int kOffDl = kOffX + kIo * (int)sizeof(IOT);
  static constexpr int kOffZ = kOffDl + kIo * (int)sizeof(IOT);
  static constexpr int kOffB = kOffZ + kIo * (int)sizeof(IOT);
  static constexpr int kOffC = kOffB + kBC * (int)sizeof(IOT);
  static constexpr int kStage = round_up(kOffC + kBC * (int)sizeof(IOT), 128);
  static constexpr int kBytes = 2 * kStage;
  static_assert((kIo * (int)sizeof(IOT)) % 16 == 0 && (kBC * (int)sizeof(IOT)) % 16 == 0,
                "16-byte pieces");
};

template <typename IOT, int N, bool kZoh>
__global__ void __launch_bounds__(256) decode2_kernel(const DecodeParams p, int tiles_d,
                                                      int ntiles) {
  using IO = Io<IOT>;
  using Ly = Dec2Layout<IOT, N>;
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  constexpr int TD = Ly::TD, LPC = N / 4;
  constexpr int ES = (int)sizeof(IOT);
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x;
  const bool has_z = p.z != nullptr, has_d = p.D != nullptr, has_bias = p.bias != nullptr;

  // every 16-byte piece of one tile, spread over the CTA's threads
  auto issue = [&](int tile, int stage) {
    unsigned char* st = smem + stage * Ly::kStage;
    const int b0 = (tile / tiles_d) * kDecTB, d0 = (tile % tiles_d) * TD;
    constexpr int kRowState = TD * N * 4 / 16;  // pieces per batch row of the state tile
    for (int i = tid; i < kDecTB * kRowState; i += 256) {
      const int r = i / kRowState, q = i % kRowState;
      cp_async_16(st + (r * kRowState + q) * 16,
                  reinterpret_cast<const unsigned char*>(p.state + ((size_t)(b0 + r) * p.dim + d0) * N) + q * 16);
    }
    for (int i = tid; i < TD * N / 4; i += 256)
      cp_async_16(st + Ly::kOffA + i * 16, reinterpret_cast<const unsigned char*>(p.A + (size_t)d0 * N) + i * 16);
    if (tid < TD / 4) {
      if (has_d) cp_async_16(st + Ly::kOffD + tid * 16, p.D + d0 + 4 * tid);
      if (has_bias) cp_async_16(st + Ly::kOffBias + tid * 16, p.bias + d0 + 4 * tid);
    }
    constexpr int kRowIo = TD * ES / 16;
    for (int i = tid; i < kDecTB * kRowIo; i += 256) {
      const int r = i / kRowIo, q = i % kRowIo;
      const size_t off = ((size_t)(b0 + r) * p.dim + d0) * ES + q * 16;
      cp_async_16(st + Ly::kOffX + i * 16, reinterpret_cast<const unsigned char*>(p.x) + off);
      cp_async_16(st + Ly::kOffDl + i * 16, reinterpret_cast<const unsigned char*>(p.delta) + off);
      if (has_z) cp_async_16(st + Ly::kOffZ + i * 16, reinterpret_cast<const unsigned char*>(p.z) + off);
    }
    constexpr int kBCPieces = kDecTB * N * ES / 16;
    if (tid < kBCPieces) {
      const size_t off = (size_t)b0 * N * ES + tid * 16;
      cp_async_16(st + Ly::kOffB + tid * 16, reinterpret_cast<const unsigned char*>(p.B) + off);
      cp_async_16(st + Ly::kOffC + tid * 16, reinterpret_cast<const unsigned char*>(p.C) + off);
    }
  };

  int tile = blockIdx.x, stage = 0;
  if (tile < ntiles) issue(tile, 0);
  cp_async_commit_group();
  for (; tile < ntiles; tile += gridDim.x, stage ^= 1) {
    const int next = tile + gridDim.x;
    if (next < ntiles) issue(next, stage ^ 1);
    cp_async_commit_group();
    cp_async_wait_group<1>();  // this tile's pieces (every thread's) have landed
    __syncthreads();
    const unsigned char* st = smem + stage * Ly::kStage;
    const float* sS = reinterpret_cast<const float*>(st);
    const float* sA = reinterpret_cast<const float*>(st + Ly::kOffA);
    const float* sD = reinterpret_cast<const float*>(st + Ly::kOffD);
    const float* sBias = reinterpret_cast<const float*>(st + Ly::kOffBias);
    const IOT* sx = reinterpret_cast<const IOT*>(st + Ly::kOffX);
    const IOT* sdl = reinterpret_cast<const IOT*>(st + Ly::kOffDl);
    const IOT* sz = reinterpret_cast<const IOT*>(st + Ly::kOffZ);
    const IOT* sB = reinterpret_cast<const IOT*>(st + Ly::kOffB);
    const IOT* sC = reinterpret_cast<const IOT*>(st + Ly::kOffC);
    const int b0 = (tile / tiles_d) * kDecTB, d0 = (tile % tiles_d) * TD;
    // items (pair, lane): LPC consecutive threads share a (row, channel) pair
#pragma unroll
    for (int it = 0; it < kDecTB * TD * LPC / 256; ++it) {
      const int item = it * 256 + tid;
      const int pair = item / LPC, lane_in = item % LPC;
      const int r = pair / TD, dl = pair % TD;
      const float4 h4 = *reinterpret_cast<const float4*>(sS + pair * N + lane_in * 4);
      const float4 a4 = *reinterpret_cast<const float4*>(sA + dl * N + lane_in * 4);
      const float4 bb = IO::load4(sB + r * N + lane_in * 4);
      const float4 cc = IO::load4(sC + r * N + lane_in * 4);
      float h[4] = {h4.x, h4.y, h4.z, h4.w}, a[4] = {a4.x, a4.y, a4.z, a4.w};
      const float bv[4] = {bb.x, bb.y, bb.z, bb.w}, cv[4] = {cc.x, cc.y, cc.z, cc.w};
      const float xv = IO::load(sx + pair), draw = IO::load(sdl + pair);
      const float v = draw + (has_bias ? sBias[dl] : 0.f);
      float dt;
      if (!p.softplus) {
        dt = v;
      } else if constexpr (kFast) {
        dt = v > kSoftplusCut ? v : kLn2 * lg2_approx(1.f + ex2_approx(v * kLog2e));
      } else {
        dt = v > kSoftplusCut ? v : log1pf(expf(v));
      }
      const float dx = dt * xv;
      const float dtl = kFast ? dt * kLog2e : dt;
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float e = kFast ? ex2_approx(dtl * a[k]) : expf(dtl * a[k]);
        if constexpr (kZoh) {
          const float coef = a[k] == 0.f ? dt
                             : kFast     ? (e - 1.f) * rcp_approx(a[k])
                                         : expm1f(dt * a[k]) / a[k];
          h[k] = fmaf(e, h[k], xv * coef * bv[k]);
        } else {
          h[k] = fmaf(e, h[k], dx * bv[k]);
        }
        acc = fmaf(cv[k], h[k], acc);
      }
#pragma unroll
      for (int off = LPC / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      float* hp = p.state + ((size_t)(b0 + r) * p.dim + d0 + dl) * N + lane_in * 4;
      *reinterpret_cast<float4*>(hp) = make_float4(h[0], h[1], h[2], h[3]);
      if (lane_in == 0) {
        float yy = fmaf(has_d ? sD[dl] : 0.f, xv, acc);
        if (has_z) {
          const float zz = IO::load(sz + pair);
          if constexpr (kFast) {
            const float hz = 0.5f * zz;
            yy *= fmaf(hz, tanh_approx(hz), hz);
          } else {
            yy *= zz / (1.f + expf(-zz));
          }
        }
        IO::store(reinterpret_cast<IOT*>(p.y) + (size_t)(b0 + r) * p.dim + d0 + dl, yy);
      }
    }
    __syncthreads();  // the stage is refilled by the next iteration's issue
  }
  cp_async_wait_group<0>();
}

// -------------------------------------------------------------------------
// cudaFuncSetAttribute once per (kernel, device).
cudaError_t ensure_smem_attr(const void* kernel, int smem) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kernel, dev})) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) done.insert({kernel, dev});
  return e;
}

// SSM_DECODE_PIPELINED=1 in the environment runs the pipelined kernel where
// the shape allows; by default every decode step takes the one-shot kernel,
// which measured faster (it is issue-bound, and the pipelined kernel adds the
// staging's instructions and barriers).
bool decode2_enabled() {
  const char* v = getenv("SSM_DECODE_PIPELINED");
  return v && v[0] == '1';
}

template <typename IOT, int N, int CPT, bool kZoh>
cudaError_t launch_scan_t(const ScanPlan& plan, const ScanParams& p, const ScanMaps* maps,
                          bool use_tma, cudaStream_t stream) {
  constexpr int NT = scan_threads(CPT), T = kScanTileSteps, S = kScanStages;
  static const ScanMaps none{};
  const ScanMaps& m = maps ? *maps : none;
  const dim3 block(NT);
  cudaError_t err = cudaSuccess;
  // `dependent`: launch with programmatic stream serialisation, so the grid
  // may begin while the previous kernel on the stream finishes.
  auto run = [&](auto kernel, int smem, dim3 grid, bool dependent = false) -> cudaError_t {
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kernel), smem);
    if (e != cudaSuccess) return e;
    if (!dependent) {
      kernel<<<grid, block, smem, stream>>>(p, m);
      return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p, m);
  };
  // composition of the carries (with three or more segments), between the
  // passes; a programmatic dependent launch like the main pass
  auto compose = [&]() -> cudaError_t {
    if (plan.nseg <= kPrologueCompose) return cudaSuccess;
    const size_t n = (size_t)p.batch * N * p.dim;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((n + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, scan_compose_kernel, p, N);
  };
  if (use_tma) {
    constexpr int smem_agg = scan_smem_bytes<IOT, N, CPT, NT, T, S, true>();
    constexpr int smem = scan_smem_bytes<IOT, N, CPT, NT, T, S, false>();
    if (plan.nseg > 1) {
      err = run(scan_kernel<IOT, N, CPT, NT, T, S, true, true, kZoh>, smem_agg,
                dim3(plan.dtiles, plan.nseg - 1, p.batch));
      if (err != cudaSuccess) return err;
      err = compose();
      if (err != cudaSuccess) return err;
    }
    return run(scan_kernel<IOT, N, CPT, NT, T, S, false, true, kZoh>, smem,
               dim3(plan.dtiles, plan.nseg, p.batch), plan.nseg > 1);
  }
  constexpr int smem_agg = scan_smem_bytes<IOT, N, CPT, NT, T, 1, true>();
  constexpr int smem = scan_smem_bytes<IOT, N, CPT, NT, T, 1, false>();
  if (plan.nseg > 1) {
    err = run(scan_kernel<IOT, N, CPT, NT, T, 1, true, false, kZoh>, smem_agg,
              dim3(plan.dtiles, plan.nseg - 1, p.batch));
    if (err != cudaSuccess) return err;
    err = compose();
    if (err != cudaSuccess) return err;
  }
  return run(scan_kernel<IOT, N, CPT, NT, T, 1, false, false, kZoh>, smem,
             dim3(plan.dtiles, plan.nseg, p.batch), plan.nseg > 1);
}

template <typename IOT, int N, int CPT>
int ctas_per_sm_t() {
  constexpr int NT = scan_threads(CPT), T = kScanTileSteps, S = kScanStages;
  int n = 0;
  auto kernel = scan_kernel<IOT, N, CPT, NT, T, S, false, true, false>;
  constexpr int smem = scan_smem_bytes<IOT, N, CPT, NT, T, S, false>();
  if (ensure_smem_attr(reinterpret_cast<const void*>(kernel), smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, NT, smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <typename IOT>
int ctas_per_sm_io(int dstate) {
  switch (dstate) {
    case 2: return ctas_per_sm_t<IOT, 2, 2>();
    case 4: return ctas_per_sm_t<IOT, 4, 2>();
    case 8: return ctas_per_sm_t<IOT, 8, 2>();
    case 16: return ctas_per_sm_t<IOT, 16, SSM_CPT16>();
    case 32: return ctas_per_sm_t<IOT, 32, 1>();
    case 64: return ctas_per_sm_t<IOT, 64, 1>();
    default: return 0;
  }
}

template <typename IOT, bool kZoh>
cudaError_t launch_scan_io(const ScanPlan& plan, const ScanParams& p, const ScanMaps* maps,
                           bool use_tma, int dstate, cudaStream_t stream) {
  switch (dstate) {
    case 2: return launch_scan_t<IOT, 2, 2, kZoh>(plan, p, maps, use_tma, stream);
    case 4: return launch_scan_t<IOT, 4, 2, kZoh>(plan, p, maps, use_tma, stream);
    case 8: return launch_scan_t<IOT, 8, 2, kZoh>(plan, p, maps, use_tma, stream);
    case 16: return launch_scan_t<IOT, 16, SSM_CPT16, kZoh>(plan, p, maps, use_tma, stream);
    case 32: return launch_scan_t<IOT, 32, 1, kZoh>(plan, p, maps, use_tma, stream);
    case 64: return launch_scan_t<IOT, 64, 1, kZoh>(plan, p, maps, use_tma, stream);
    default: return cudaErrorInvalidValue;
  }
}

// The pipelined decode for shapes whose tiles are whole and whose rows are
// 16-byte aligned; nullptr when the shape needs the one-shot kernel.
template <typename IOT, int N, bool kZoh>
cudaError_t launch_decode2(const DecodeParams& p, cudaStream_t stream, bool* used) {
  using Ly = Dec2Layout<IOT, N>;
  *used = false;
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  if (p.batch % kDecTB != 0 || p.dim % Ly::TD != 0) return cudaSuccess;
  if (!al(p.state) || !al(p.A) || !al(p.x) || !al(p.delta) || !al(p.B) || !al(p.C) ||
      (p.z && !al(p.z)) || (p.D && !al(p.D)) || (p.bias && !al(p.bias)))
    return cudaSuccess;
  auto kernel = decode2_kernel<IOT, N, kZoh>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kernel), Ly::kBytes);
  if (e != cudaSuccess) return e;
  static int slots_cache[64] = {};
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int slots = (dev >= 0 && dev < 64) ? slots_cache[dev] : 0;
  if (slots <= 0) {
    int per_sm = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, Ly::kBytes);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    slots = std::max(1, per_sm * sms);
    if (dev >= 0 && dev < 64) slots_cache[dev] = slots;
  }
  const int tiles_d = p.dim / Ly::TD;
  const long long ntiles = (long long)(p.batch / kDecTB) * tiles_d;
  if (ntiles <= 0 || ntiles > (1ll << 30)) return cudaSuccess;
  // equal tile counts per CTA: ceil(tiles / slots) tiles each
  const long long per = (ntiles + slots - 1) / slots;
  const unsigned grid = (unsigned)((ntiles + per - 1) / per);
  kernel<<<grid, 256, Ly::kBytes, stream>>>(p, tiles_d, (int)ntiles);
  *used = true;
  return cudaGetLastError();
}

template <typename IOT, bool kZoh>
cudaError_t launch_decode_io(const DecodeParams& p, int dstate, cudaStream_t stream) {
  if (decode2_enabled()) {
    bool used = false;
    cudaError_t e = cudaSuccess;
    switch (dstate) {
      case 16: e = launch_decode2<IOT, 16, kZoh>(p, stream, &used); break;
      case 32: e = launch_decode2<IOT, 32, kZoh>(p, stream, &used); break;
      case 64: e = launch_decode2<IOT, 64, kZoh>(p, stream, &used); break;
      default: break;
    }
    if (e != cudaSuccess || used) return e;
  }
  auto go = [&](auto kernel, int lpc) -> cudaError_t {
    constexpr int RB = SSM_DEC_RB;
    const dim3 grid((unsigned)(((size_t)p.dim * lpc + 255) / 256),
                    (unsigned)((p.batch + RB - 1) / RB));
    kernel<<<grid, 256, 0, stream>>>(p);
    return cudaGetLastError();
  };
  switch (dstate) {
    case 2: return go(decode_kernel<IOT, 2, kZoh>, DecShape<2>::LPC);
    case 4: return go(decode_kernel<IOT, 4, kZoh>, DecShape<4>::LPC);
    case 8: return go(decode_kernel<IOT, 8, kZoh>, DecShape<8>::LPC);
    case 16: return go(decode_kernel<IOT, 16, kZoh>, DecShape<16>::LPC);
    case 32: return go(decode_kernel<IOT, 32, kZoh>, DecShape<32>::LPC);
    case 64: return go(decode_kernel<IOT, 64, kZoh>, DecShape<64>::LPC);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool scan_dstate_supported(int dstate) {
  return dstate == 2 || dstate == 4 || dstate == 8 || dstate == 16 || dstate == 32 ||
         dstate == 64;
}

int scan_channels_per_thread(int dstate) { return dstate < 16 ? 2 : dstate == 16 ? SSM_CPT16 : 1; }

int scan_ctas_per_sm(int dstate, bool bf16) {
  return bf16 ? ctas_per_sm_io<uint16_t>(dstate) : ctas_per_sm_io<float>(dstate);
}

cudaError_t launch_scan(const ScanPlan& plan, const ScanParams& p, const ScanMaps* maps,
                        bool use_tma, int dstate, bool bf16, bool zoh, cudaStream_t stream) {
  if (zoh)
    return bf16 ? launch_scan_io<uint16_t, true>(plan, p, maps, use_tma, dstate, stream)
                : launch_scan_io<float, true>(plan, p, maps, use_tma, dstate, stream);
  return bf16 ? launch_scan_io<uint16_t, false>(plan, p, maps, use_tma, dstate, stream)
              : launch_scan_io<float, false>(plan, p, maps, use_tma, dstate, stream);
}

cudaError_t launch_decode(const DecodeParams& p, int dstate, bool bf16, bool zoh,
                          cudaStream_t stream) {
  if (zoh)
    return bf16 ? launch_decode_io<uint16_t, true>(p, dstate, stream)
                : launch_decode_io<float, true>(p, dstate, stream);
  return bf16 ? launch_decode_io<uint16_t, false>(p, dstate, stream)
              : launch_decode_io<float, false>(p, dstate, stream);
}

}  // namespace ssm
