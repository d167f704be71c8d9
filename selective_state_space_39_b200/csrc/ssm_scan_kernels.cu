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
//  * Scaled recurrence. With s_t ~ Delta_t x_t (never zero, see below) the
//    state is kept as g_n = h_n / s_t, so that
//        g_n(t) = (a_n(t) s_{t-1}/s_t) g_n(t-1) + B_n(t),   y_t = s_t sum_n C_n g_n
//    costs one multiply (the chain of alpha_n = s_{t-1}/s_t r^(n+1)) and two
//    FMAs per state, instead of two multiplies and two FMAs. s_t is Delta_t x_t
//    plus copysign(2^-64); the computed state therefore follows the exact
//    recurrence with Delta_t x_t replaced by s_t, |s_t - Delta_t x_t| <= 2^-64.
//  * B and C (shared by all channels of a step) are widened to fp32 once per
//    CTA in shared memory and read as broadcasts.
//  * x, delta, z, B, C tiles of 16 steps are staged in shared memory by TMA
//    (cp.async.bulk.tensor, no multicast) through a 2-stage mbarrier
//    pipeline; every wait is bounded by a time limit.
//  * The sequence is split into segments so the whole GPU is busy: a carry
//    pass computes each segment's end state from a zero start (and the sum
//    of Delta, which gives the segment's decay exp(A_n sum Delta)), and the
//    main pass composes those affine carries ((a1,b1) then (a2,b2) ->
//    (a1 a2, a2 b1 + b2), the associative scan of the state update) in its
//    prologue before running its own segment exactly from the true start.
//
// bf16 io uses MUFU approximations (ex2/lg2/rcp/tanh.approx); fp32 io uses
// the accurate expf / log1pf / IEEE division.
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
// Depth-3 decay tree and split readout accumulator (1) or linear chains (0).
#ifndef SSM_SHORT_CHAINS
#define SSM_SHORT_CHAINS 0
#endif
// Channels per thread at dstate 16.
#ifndef SSM_CPT16
#define SSM_CPT16 2
#endif
#ifndef SSM_MIN_CTAS
#define SSM_MIN_CTAS 1
#endif

namespace ssm {

namespace {

constexpr int kTileUnroll = SSM_TILE_UNROLL;

constexpr int round_up(int v, int m) { return (v + m - 1) / m * m; }

template <typename IOT, int N, int CPT, int NT, int T>
struct ScanLayout {
  static constexpr int DT = NT * CPT;
  static constexpr int kTileBytes = T * DT * (int)sizeof(IOT);
  static constexpr int kBCBytes = T * N * (int)sizeof(IOT);
  static constexpr int kOffX = 0;
  static constexpr int kOffD = kTileBytes;
  static constexpr int kOffZ = 2 * kTileBytes;
  static constexpr int kOffB = 3 * kTileBytes;
  static constexpr int kOffC = kOffB + round_up(kBCBytes, 128);
  static constexpr int kStageBytes = kOffC + round_up(kBCBytes, 128);
  // fp32 copies of B (pre-scaled) and C for the tile: [2 buffers][2][T][N]
  static constexpr int kBCF32Bytes = 2 * 2 * T * N * 4;
};

template <typename IOT, int N, int CPT, int NT, int T, int STAGES>
constexpr int scan_smem_bytes() {
  using L = ScanLayout<IOT, N, CPT, NT, T>;
  return STAGES * L::kStageBytes + L::kBCF32Bytes + 8 * STAGES;
}

// Per-channel constants.
struct Chan {
  float A0;     // A[d,0] (natural units)
  float bias;   // fast path: bias * log2(e); precise path: bias
  float Dd;     // skip weight
  bool valid;   // d < dim
};

// Per-step, per-channel quantities computed ahead of the state update.
struct StepScalars {
  float a0, a1;  // alpha for states 0 and 1: rho r, rho r^2 (structured A)
  float rr;      // r^2, the step of the alpha chain over state pairs
  float rho;     // s_{t-1} / s_t (generic A)
  float q;       // Delta (precise) or Delta log2(e) (fast)
  float s;       // the state scale s_t ~ Delta x (ZOH: x / A_0, or x)
  float m0, m1;  // ZOH, structured A: exp(Delta A_n) - 1 for states 0 and 1
  float e2;      // ZOH, structured A: the step of that chain over state pairs
};

// Step size, decay base and state scale for one channel and step.
//
// Input term (kZoh = false, the simplified deltaB of the selective_scan
// listing): Delta x B_n, with s = Delta x (fast: times log2 e, matched by B
// pre-scaled by ln 2). Exact zero-order hold (kZoh, §2.2 B-bar):
// x B_n (exp(Delta A_n) - 1) / A_n. With structured A (kS) that is
// s B_n / (n+1) m_n with s = x / A_0 and m_n = r^(n+1) - 1 (B
// pre-scaled by 1/(n+1)); m_n is built without cancellation from
// m_0 = expm1(Delta A_0): m_(n+2) = m_n r^2 + m_0 (1 + r), every term of one
// sign. Generic A under ZOH uses s = x and forms each state's factor itself.
template <bool kFast, bool kZoh = false, bool kS = true>
__device__ __forceinline__ StepScalars step_scalars(float xv, float dv, const Chan& ch,
                                                    int softplus, float& s_prev) {
  StepScalars o;
  float q, r;
  if constexpr (kFast) {
    const float v = fmaf(dv, kLog2e, ch.bias);
    q = softplus ? (v > kSoftplusCut * kLog2e ? v : lg2_approx(1.f + ex2_approx(v))) : v;
    r = ex2_approx(q * ch.A0);  // exp(Delta A0)
  } else {
    const float v = dv + ch.bias;
    q = softplus ? (v > kSoftplusCut ? v : log1pf(expf(v))) : v;
    r = expf(q * ch.A0);
  }
  float s;
  if constexpr (!kZoh) {
    s = q * xv;
  } else if constexpr (kS) {
    s = kFast ? xv * rcp_approx(ch.A0) : xv / ch.A0;
    const float em1 = kFast ? r - 1.f : expm1f(q * ch.A0);  // exp(Delta A_0) - 1
    o.m0 = em1;
    o.m1 = fmaf(em1, r, em1);
    o.e2 = em1 * (1.f + r);
  } else {
    s = xv;
  }
  s = s + copysignf(kScaleFloor, s);  // kept away from zero
  const float rho = kFast ? s_prev * rcp_approx(s) : s_prev / s;
  s_prev = s;
  o.q = q;
  o.s = s;
  o.rho = rho;
  o.a0 = rho * r;
  o.a1 = o.a0 * r;
  o.rr = r * r;
  return o;
}

// -------------------------------------------------------------------------
// The scan kernel. kAgg = carry pass (segments 0..nseg-2: end state and
// sum of Delta, no output); !kAgg = main pass (all segments, y and h_last).
// Grid: (dtiles, segments, batch). Block: NT threads, CPT channels each.
template <typename IOT, int N, int CPT, int NT, int T, int STAGES, bool kAgg, bool kTma,
          bool kZoh>
__global__ void __launch_bounds__(NT, SSM_MIN_CTAS) scan_kernel(const ScanParams p,
                                                  const __grid_constant__ ScanMaps maps) {
  using IO = Io<IOT>;
  using L = ScanLayout<IOT, N, CPT, NT, T>;
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  constexpr int DT = L::DT;
  constexpr int NP = N / 2;
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
  const int t_begin = seg * p.seg_steps;
  const int t_end = min(t_begin + p.seg_steps, L_);
  const int ntiles = t_end > t_begin ? (t_end - t_begin + T - 1) / T : 0;

  const uint32_t stage_tx = (uint32_t)((kAgg ? 2 : (has_z ? 3 : 2)) * L::kTileBytes +
                                       (kAgg ? 1 : 2) * L::kBCBytes);

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

  int issued = 0;  // tiles whose loads were issued (thread 0 only)
  bool aborted = false;
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
  if constexpr (kTma) {
    if (tid == 0)
      for (; issued < STAGES - 1 && issued < ntiles; ++issued) issue_tile(issued);
  }

  // ---- per-channel constants and structure of A ------------------------
  Chan ch[CPT];
  bool structured = true;
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const int d = d_first + c;
    ch[c].valid = d < dim;
    if (ch[c].valid) {
      const float* Ar = p.A + (size_t)d * N;
      ch[c].A0 = Ar[0];
#pragma unroll
      for (int n = 1; n < N; ++n) structured = structured && (Ar[n] == (float)(n + 1) * Ar[0]);
      // the ZOH chain divides by A_0: A = 0 takes the per-state path
      if constexpr (kZoh) structured = structured && Ar[0] != 0.f;
      const float bias = p.bias ? p.bias[d] : 0.f;
      ch[c].bias = kFast ? bias * kLog2e : bias;
      ch[c].Dd = p.D ? p.D[d] : 0.f;
    } else {
      ch[c].A0 = -1.f;
      ch[c].bias = 0.f;
      ch[c].Dd = 0.f;
    }
  }
  // One code path per CTA: the multiply-chain path when every channel of the
  // CTA has structured A, one exp per state otherwise.
  const bool cta_structured = __syncthreads_and(structured) != 0;

  // ---- initial state ----------------------------------------------------
  float2 g[CPT][NP];  // scaled state g = h / s_prev
  float s_prev[CPT];
  float qsum[CPT];
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    s_prev[c] = 1.f;
    qsum[c] = 0.f;
#pragma unroll
    for (int k = 0; k < NP; ++k) g[c][k] = make_float2(0.f, 0.f);
  }
  // The main pass may start while the carry pass finishes (programmatic
  // dependent launch): everything above reads only inputs; the carries and
  // the h0 copy are read after this wait.
  if constexpr (!kAgg) griddep_wait();
  {
    const int nagg = p.nseg - 1;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      if (!ch[c].valid) continue;
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
        if (seg > 0) {
          // Inclusive end state of segment 0, then compose the carries
          // (decay exp(A_n sum Delta), end state) of segments 1..seg-1.
          const float* st0 = p.ws_state + ((size_t)b * nagg) * N * dim + d;
#pragma unroll
          for (int k = 0; k < NP; ++k)
            g[c][k] = make_float2(__ldcg(st0 + (size_t)(2 * k) * dim),
                                  __ldcg(st0 + (size_t)(2 * k + 1) * dim));
          const float* Ar = p.A + (size_t)d * N;
          for (int j = 1; j < seg; ++j) {
            const float sd = __ldcg(p.ws_sum + ((size_t)b * nagg + j) * dim + d);
            const float* stj = p.ws_state + ((size_t)b * nagg + j) * N * dim + d;
            float bj[N];
#pragma unroll
            for (int n = 0; n < N; ++n) bj[n] = __ldcg(stj + (size_t)n * dim);
            if (cta_structured) {
              const float e = expf(ch[c].A0 * sd);
              float en = e;
#pragma unroll
              for (int k = 0; k < NP; ++k) {
                const float e0 = en, e1 = en * e;
                en = e1 * e;
                g[c][k].x = fmaf(e0, g[c][k].x, bj[2 * k]);
                g[c][k].y = fmaf(e1, g[c][k].y, bj[2 * k + 1]);
              }
            } else {
#pragma unroll
              for (int k = 0; k < NP; ++k) {
                g[c][k].x = fmaf(expf(Ar[2 * k] * sd), g[c][k].x, bj[2 * k]);
                g[c][k].y = fmaf(expf(Ar[2 * k + 1] * sd), g[c][k].y, bj[2 * k + 1]);
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
  }

  // ---- per-step pieces ----------------------------------------------------
  // vector stores of the thread's CPT outputs: all valid and rows aligned
  const bool vec_store = CPT >= 2 && (p.dim % CPT) == 0 && ch[CPT - 1].valid;
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
      }
    } else if constexpr (CPT == 4) {
      const float4 x4 = IO::load4(sx), d4 = IO::load4(sdl);
      in.x[0] = x4.x; in.x[1] = x4.y; in.x[2] = x4.z; in.x[3] = x4.w;
      in.d[0] = d4.x; in.d[1] = d4.y; in.d[2] = d4.z; in.d[3] = d4.w;
      if (!kAgg && has_z) {
        const float4 z4 = IO::load4(sz);
        in.z[0] = z4.x; in.z[1] = z4.y; in.z[2] = z4.z; in.z[3] = z4.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        in.x[c] = IO::load(sx + c);
        in.d[c] = IO::load(sdl + c);
        if (!kAgg && has_z) in.z[c] = IO::load(sz + c);
      }
    }
    return in;
  };

  // Rows of A for the one-exp-per-state path, held in registers (loaded by
  // run_tiles for that path only).
  float2 Areg[CPT][NP];

  // State update (and readout) of one step, given its precomputed scalars.
  auto state_step = [&](auto kStructTag, const StepIn& in, const StepScalars* sc, const float* Bt,
                        const float* Ct, int t_abs) {
    constexpr bool kS = decltype(kStructTag)::value;
    float2 acc[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[c] = make_float2(0.f, 0.f);
    if constexpr (kS) {
      const float2* B2 = reinterpret_cast<const float2*>(Bt);
      const float2* C2 = reinterpret_cast<const float2*>(Ct);
      (void)C2;
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
#if SSM_SHORT_CHAINS
        // alpha pairs P_k = (a0, a1) (r^2)^k by a depth-3 tree, and two
        // readout accumulators, to shorten the dependency chains.
        float2 P[NP];
        const float2 rr1 = make_float2(sc[c].rr, sc[c].rr);
        P[0] = make_float2(sc[c].a0, sc[c].a1);
        if constexpr (NP > 1) P[1] = mul2(P[0], rr1);
        if constexpr (NP > 2) {
          const float2 rr2 = mul2(rr1, rr1);
          P[2] = mul2(P[0], rr2);
          if constexpr (NP > 3) P[3] = mul2(P[1], rr2);
          if constexpr (NP > 4) {
            const float2 rr4 = mul2(rr2, rr2);
#pragma unroll
            for (int k = 4; k < 8 && k < NP; ++k) P[k] = mul2(P[k - 4], rr4);
            if constexpr (NP > 8) {
              const float2 rr8 = mul2(rr4, rr4);
#pragma unroll
              for (int k = 8; k < NP; ++k) P[k] = mul2(P[k - 8], rr8);
            }
          }
        }
        float2 acc1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < NP; ++k) {
          g[c][k] = fma2(P[k], g[c][k], B2[k]);
          if constexpr (!kAgg) {
            if (k & 1)
              acc1 = fma2(C2[k], g[c][k], acc1);
            else
              acc[c] = fma2(C2[k], g[c][k], acc[c]);
          }
        }
        if constexpr (!kAgg) acc[c] = make_float2(acc[c].x + acc1.x, acc[c].y + acc1.y);
#else
        // alpha_n = rho r^(n+1), two states at a time: (a0, a1) * (r^2)^k
        float2 a = make_float2(sc[c].a0, sc[c].a1);
        const float2 rr = make_float2(sc[c].rr, sc[c].rr);
        if constexpr (kZoh) {
          // input B_n / (n+1) m_n, m pairs stepped by m <- m r^2 + m_0 (1 + r)
          float2 m = make_float2(sc[c].m0, sc[c].m1);
          const float2 e2 = make_float2(sc[c].e2, sc[c].e2);
#pragma unroll
          for (int k = 0; k < NP; ++k) {
            g[c][k] = fma2(a, g[c][k], mul2(B2[k], m));
            if (k + 1 < NP) {
              a = mul2(a, rr);
              m = fma2(m, rr, e2);
            }
            if constexpr (!kAgg) acc[c] = fma2(C2[k], g[c][k], acc[c]);
          }
        } else {
#pragma unroll
          for (int k = 0; k < NP; ++k) {
            g[c][k] = fma2(a, g[c][k], B2[k]);
            if (k + 1 < NP) a = mul2(a, rr);
            if constexpr (!kAgg) acc[c] = fma2(C2[k], g[c][k], acc[c]);
          }
        }
#endif
      }
    } else {
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const float2* B2 = reinterpret_cast<const float2*>(Bt);
        const float2* C2 = reinterpret_cast<const float2*>(Ct);
        (void)C2;
        const float rho = sc[c].rho, q = sc[c].q;
#pragma unroll
        for (int k = 0; k < NP; ++k) {
          float2 a;
          const float A_lo = Areg[c][k].x, A_hi = Areg[c][k].y;
          const float e_lo = kFast ? ex2_approx(q * A_lo) : expf(q * A_lo);
          const float e_hi = kFast ? ex2_approx(q * A_hi) : expf(q * A_hi);
          a = make_float2(rho * e_lo, rho * e_hi);
          if constexpr (kZoh) {
            // input B_n (exp(Delta A_n) - 1) / A_n (Delta where A_n = 0), s = x
            const float dt = kFast ? q * kLn2 : q;
            auto coef = [&](float An, float e) {
              if (An == 0.f) return dt;
              return kFast ? (e - 1.f) * rcp_approx(An) : expm1f(dt * An) / An;
            };
            const float2 in2 = make_float2(B2[k].x * coef(A_lo, e_lo), B2[k].y * coef(A_hi, e_hi));
            g[c][k] = fma2(a, g[c][k], in2);
          } else {
            g[c][k] = fma2(a, g[c][k], B2[k]);
          }
          if constexpr (!kAgg) acc[c] = fma2(C2[k], g[c][k], acc[c]);
        }
      }
    }
    if constexpr (!kAgg) {
      float yv[CPT];
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        float yy = fmaf(sc[c].s, acc[c].x + acc[c].y, ch[c].Dd * in.x[c]);
        if (has_z) {
          if constexpr (kFast) {
            const float hz = 0.5f * in.z[c];
            yy *= fmaf(hz, tanh_approx(hz), hz);  // z * sigmoid(z)
          } else {
            yy *= in.z[c] / (1.f + expf(-in.z[c]));
          }
        }
        yv[c] = yy;
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
          if (ch[c].valid) IO::store(yrow + c, yv[c]);
      }
    }
  };

  // ---- tile loop ----------------------------------------------------------
  auto run_tiles = [&](auto kStructTag) {
    if constexpr (!decltype(kStructTag)::value) {
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const float2* Ar =
            reinterpret_cast<const float2*>(p.A + (size_t)(ch[c].valid ? d_first + c : 0) * N);
#pragma unroll
        for (int k = 0; k < NP; ++k) Areg[c][k] = __ldg(Ar + k);
      }
    }
    for (int it = 0; it < ntiles; ++it) {
      const int buf = it & 1;
      unsigned char* st;
      if constexpr (kTma) {
        st = smem + (it % STAGES) * L::kStageBytes;
        const bool ok = mbar_wait_bounded(&full[it % STAGES], (uint32_t)((it / STAGES) & 1),
                                          p.wait_limit_ns);
        if (__syncthreads_or(!ok)) {
          aborted = true;  // uniform across the CTA
          // Let the loads already issued land (bounded) before the CTA's
          // shared memory is released.
          if (tid == 0)
            for (int j = it; j < issued; ++j)
              (void)mbar_wait_bounded(&full[j % STAGES], (uint32_t)((j / STAGES) & 1), 1000000ull);
          return;
        }
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
        float* fb = bcf + (buf * 2 + 0) * T * N;
        float* fc = bcf + (buf * 2 + 1) * T * N;
        for (int i = tid; i < T * N; i += NT) {
          // Delta B (fast: ln 2, see step_scalars); ZOH: 1/(n+1) (structured) or 1
          float bscale;
          if constexpr (kZoh) bscale = cta_structured ? 1.f / (float)(i % N + 1) : 1.f;
          else bscale = kFast ? kLn2 : 1.f;
          fb[i] = IO::load(sb + i) * bscale;
          if (!kAgg) fc[i] = IO::load(sc + i);
        }
      }
      __syncthreads();
      if constexpr (kTma) {
        // The stage consumed by the previous tile is free: refill it.
        if (tid == 0 && issued < ntiles) issue_tile(issued++);
      }

      const float* fb = bcf + (buf * 2 + 0) * T * N;
      const float* fc = bcf + (buf * 2 + 1) * T * N;
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
        StepScalars sc_next[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c)
          sc_next[c] = step_scalars<kFast, kZoh, decltype(kStructTag)::value>(
              in_next.x[c], in_next.d[c], ch[c], softplus, s_prev[c]);
        float s_last[CPT];
#pragma unroll(kFull ? kTileUnroll : 1)
        for (int row = 0; row < nst; ++row) {
          const StepIn in = in_next;
          StepScalars sc[CPT];
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            sc[c] = sc_next[c];
            s_last[c] = sc[c].s;
            if constexpr (kAgg) qsum[c] += sc[c].q;
          }
          in_next = load_in(st, min(row + 1, nst - 1));
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            float sp = sc[c].s;
            sc_next[c] = step_scalars<kFast, kZoh, decltype(kStructTag)::value>(
                in_next.x[c], in_next.d[c], ch[c], softplus, sp);
          }
          state_step(kStructTag, in, sc, fb + row * N, fc + row * N, t0 + row);
        }
#pragma unroll
        for (int c = 0; c < CPT; ++c) s_prev[c] = s_last[c];  // scale of the last step
      };
      if (steps == T)
        step_loop(std::true_type{}, T);
      else
        step_loop(std::false_type{}, steps);
    }
  };
  if (cta_structured)
    run_tiles(std::true_type{});
  else
    run_tiles(std::false_type{});

  // ---- outputs of the segment ------------------------------------------
  if (!aborted) {
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      if (!ch[c].valid) continue;
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
// Decode: one step of the recurrence per (batch, channel). LPC lanes share a
// channel, SPT states each (one float4 of the state per lane, so a warp reads
// and writes contiguous runs of the (batch, dim, dstate) state); y is reduced
// across the LPC lanes by shuffles. Every load of a thread is issued before
// any arithmetic, so each thread makes a single round trip to memory: the
// kernel is otherwise bound by the latency of its waves, not by bandwidth.
template <typename IOT, int N, bool kZoh>
__global__ void __launch_bounds__(256) decode_kernel(const DecodeParams p) {
  using IO = Io<IOT>;
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  constexpr int SPT = (N % 4 == 0) ? 4 : 2;
  constexpr int LPC = N / SPT;
  static_assert(LPC <= 32 && (LPC & (LPC - 1)) == 0, "lanes per channel must divide a warp");
  const size_t gtid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t chan = gtid / LPC;  // b * dim + d
  const int lane_in = (int)(gtid % LPC);
  const size_t nchan = (size_t)p.batch * p.dim;
  const bool valid = chan < nchan;
  const size_t cc = valid ? chan : 0;
  const int b = (int)(cc / p.dim), d = (int)(cc % p.dim);

  // ---- all loads first ----
  float* hp = p.state + cc * N + lane_in * SPT;
  const float* Ar = p.A + (size_t)d * N + lane_in * SPT;
  const IOT* Bp = reinterpret_cast<const IOT*>(p.B) + (size_t)b * N + lane_in * SPT;
  const IOT* Cp = reinterpret_cast<const IOT*>(p.C) + (size_t)b * N + lane_in * SPT;
  float h[SPT], a[SPT], bb[SPT], cv[SPT];
  if constexpr (SPT == 4) {
    const float4 t4 = *reinterpret_cast<const float4*>(hp);
    h[0] = t4.x; h[1] = t4.y; h[2] = t4.z; h[3] = t4.w;
    const float4 a4 = __ldg(reinterpret_cast<const float4*>(Ar));
    a[0] = a4.x; a[1] = a4.y; a[2] = a4.z; a[3] = a4.w;
    const float4 b4 = IO::load4(Bp), c4 = IO::load4(Cp);
    bb[0] = b4.x; bb[1] = b4.y; bb[2] = b4.z; bb[3] = b4.w;
    cv[0] = c4.x; cv[1] = c4.y; cv[2] = c4.z; cv[3] = c4.w;
  } else {
    const float2 t2 = *reinterpret_cast<const float2*>(hp);
    h[0] = t2.x; h[1] = t2.y;
    const float2 a2 = __ldg(reinterpret_cast<const float2*>(Ar));
    a[0] = a2.x; a[1] = a2.y;
    const float2 b2 = IO::load2(Bp), c2 = IO::load2(Cp);
    bb[0] = b2.x; bb[1] = b2.y; cv[0] = c2.x; cv[1] = c2.y;
  }
  const float xv = IO::load(reinterpret_cast<const IOT*>(p.x) + cc);
  const float draw = IO::load(reinterpret_cast<const IOT*>(p.delta) + cc);
  const float bias = p.bias ? p.bias[d] : 0.f;
  const float Dd = p.D ? p.D[d] : 0.f;
  const float zz = p.z ? IO::load(reinterpret_cast<const IOT*>(p.z) + cc) : 0.f;

  // ---- arithmetic ----
  const float v = draw + bias;
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
  for (int k = 0; k < SPT; ++k) {
    const float e = kFast ? ex2_approx(dtl * a[k]) : expf(dtl * a[k]);
    if constexpr (kZoh) {
      // exact ZOH input: x B_n (exp(Delta A_n) - 1) / A_n (Delta where A_n = 0)
      const float coef = a[k] == 0.f ? dt
                         : kFast     ? (e - 1.f) * rcp_approx(a[k])
                                     : expm1f(dt * a[k]) / a[k];
      h[k] = fmaf(e, h[k], xv * coef * bb[k]);
    } else {
      h[k] = fmaf(e, h[k], dx * bb[k]);
    }
    acc = fmaf(cv[k], h[k], acc);
  }
#pragma unroll
  for (int off = LPC / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (!valid) return;
  if constexpr (SPT == 4) {
    *reinterpret_cast<float4*>(hp) = make_float4(h[0], h[1], h[2], h[3]);
  } else {
    *reinterpret_cast<float2*>(hp) = make_float2(h[0], h[1]);
  }
  if (lane_in == 0) {
    float yy = fmaf(Dd, xv, acc);
    if (p.z) {
      if constexpr (kFast) {
        const float hz = 0.5f * zz;
        yy *= fmaf(hz, tanh_approx(hz), hz);
      } else {
        yy *= zz / (1.f + expf(-zz));
      }
    }
    IO::store(reinterpret_cast<IOT*>(p.y) + cc, yy);
  }
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
  if (use_tma) {
    constexpr int smem = scan_smem_bytes<IOT, N, CPT, NT, T, S>();
    if (plan.nseg > 1) {
      err = run(scan_kernel<IOT, N, CPT, NT, T, S, true, true, kZoh>, smem,
                dim3(plan.dtiles, plan.nseg - 1, p.batch));
      if (err != cudaSuccess) return err;
    }
    return run(scan_kernel<IOT, N, CPT, NT, T, S, false, true, kZoh>, smem,
               dim3(plan.dtiles, plan.nseg, p.batch), plan.nseg > 1);
  }
  constexpr int smem = scan_smem_bytes<IOT, N, CPT, NT, T, 1>();
  if (plan.nseg > 1) {
    err = run(scan_kernel<IOT, N, CPT, NT, T, 1, true, false, kZoh>, smem,
              dim3(plan.dtiles, plan.nseg - 1, p.batch));
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
  constexpr int smem = scan_smem_bytes<IOT, N, CPT, NT, T, S>();
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

template <typename IOT, bool kZoh>
cudaError_t launch_decode_io(const DecodeParams& p, int dstate, cudaStream_t stream) {
  const size_t chans = (size_t)p.batch * p.dim;
  auto go = [&](auto kernel, int lpc) -> cudaError_t {
    const size_t threads = chans * lpc;
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    kernel<<<blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
  };
  switch (dstate) {
    case 2: return go(decode_kernel<IOT, 2, kZoh>, 1);
    case 4: return go(decode_kernel<IOT, 4, kZoh>, 1);
    case 8: return go(decode_kernel<IOT, 8, kZoh>, 2);
    case 16: return go(decode_kernel<IOT, 16, kZoh>, 4);
    case 32: return go(decode_kernel<IOT, 32, kZoh>, 8);
    case 64: return go(decode_kernel<IOT, 64, kZoh>, 16);
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
