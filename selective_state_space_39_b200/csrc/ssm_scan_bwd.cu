// ssm_scan_bwd.cu -- sm_100a kernels of the selective scan's backward pass.
//
// The gradient of the scan (page "Mamba 논문 리뷰: Selective State Space
// Models로 Transformer를 넘어서", youngju.dev, §3.3 Hardware-Aware algorithm:
// training keeps no per-step state in HBM and recomputes it) for the loss
// sum dy*y + sum dh_last*h_last. Per channel, with a_n(t) = exp(Delta_t A_n),
// g_t = dy_t SiLU(z_t) and the adjoint lam_n(t) = dLoss/dh_n(t):
//
//   lam_n(t)  = C_n(t) g_t + a_n(t+1) lam_n(t+1)     (lam(L) a(L) := dh_last)
//   dx_t      = D g_t + Delta_t sum_n lam_n B_n
//   dDelta_t  = x_t sum_n lam_n B_n + sum_n lam_n A_n a_n h_n(t-1)
//   ddelta_t  = dDelta_t sigmoid(v_t)   (softplus'; 1 above the cut or without it)
//   dz_t      = dy_t s_t SiLU'(z_t),   s_t = sum_n C_n h_n(t) + D x_t
//   dA_n     += lam_n Delta_t a_n h_n(t-1),  dB_n(t) += lam_n Delta_t x_t,
//   dC_n(t)  += g_t h_n(t),  dD += g_t x_t,  dbias += ddelta_t,  dh0 = a(0) lam(0)
//
// Design (B200). Like the forward, the work is FP32-issue bound; memory is
// used to avoid recomputation where it is cheaper than arithmetic:
//
//  * Five launches, none of which waits on another CTA:
//    1. carry: per (segment, channel block, batch row) one forward sweep from
//       a zero state, storing the state at every 4-step tile start (and the
//       summed decay exponent there) and the segment's end state; the same
//       sweep accumulates the segment's outgoing adjoint from a zero end,
//       a(t0) lam(t0) = sum_t [prod_{t0<=u<=t} a(u)] C(t) g(t), forwards.
//    2. compose: per (b, n, d) the exact chaining of those affine carries
//       across segments, giving the true entering state and adjoint of every
//       segment (the associative scan of (a, b) maps, done sequentially over
//       the few segments).
//    3. main: per segment, tiles of 4 steps in reverse order. A tile's true
//       entry state is its checkpoint plus exp(A_n Q) times the segment's
//       entering state; the tile's 4 steps are recomputed into a register
//       history, then the adjoint runs backwards through them.
//    4. reduce (two launches): dB and dC (sums over channels) from per-CTA
//       partials, dA, dD, dbias (sums over batch rows and segments) from
//       per-segment partials, in a fixed order, so results do not depend on
//       scheduling.
//  * One channel per thread with its whole state in registers; the sums over
//    n are in-thread. The sums over channels (dB, dC) go through shared
//    memory: every thread writes its 2N values per step, then each thread
//    sums one (step, value) row of 128 channels with vector loads.
//  * Structured A (A[d,n] = (n+1) A[d,0], as the forward detects it) takes one
//    exp per step and a multiply chain for the decays; other A one exp per
//    state.
//
// bf16 io uses MUFU approximations (ex2/lg2/rcp/tanh.approx); fp32 io uses
// expf / log1pf and IEEE division.
#include <algorithm>
#include <type_traits>

#include "ssm_bwd_internal.h"
#include "ssm_device.cuh"

namespace ssm {

namespace {

// 4-byte asynchronous copy global -> shared (cp.async); `src_bytes` < 4 copies that many
// bytes and zero-fills the rest (0: nothing is read, `src` is not touched).
__device__ __forceinline__ void cp_async4(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Wait until at most `Pending` of this thread's committed groups are in flight.
template <int Pending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(Pending) : "memory");
}

// Packed FP32x2 add (see fma2 / mul2).
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
#if SSM_PACKED_FP32
  return __fadd2_rn(a, b);
#else
  return make_float2(a.x + b.x, a.y + b.y);
#endif
}

constexpr int kBT = kBwdTileSteps;
constexpr int kNT = kBwdThreads;
// Channel-sum buffer: one row per (step, dB or dC, state pair) holding the
// pair's two values for each of the CTA's channels, interleaved; rows are
// padded so that row starts fall on different bank groups.
constexpr int kRowF = 2 * kNT + 4;

// Shared memory of the two sequential kernels. Per-step scalars (NTEN io
// tensors x kBT steps x 128 channels) and the fp32 B / C rows of a tile are
// double-buffered: the copies of the next tile are in flight while the
// current one is computed.
template <typename IOT, int N>
struct MainSmem {
  static constexpr int kTen = 4;  // x, delta, dy, z
  static constexpr int kRedBytes = kBT * N * kRowF * 4;
  static constexpr int kHinBytes = N * kNT * 4;
  static constexpr int kCkBytes = 2 * (N + 1) * kNT * 4;  // state checkpoint + its Q
  static constexpr int kBCBytes = 2 * kBT * 2 * N * 4;
  static constexpr int kScalBytes = 2 * kTen * kBT * kNT * (int)sizeof(IOT);
  static constexpr int kOffRed = 0;
  static constexpr int kOffHin = kOffRed + kRedBytes;
  static constexpr int kOffCk = kOffHin + kHinBytes;
  static constexpr int kOffBC = kOffCk + kCkBytes;
  static constexpr int kOffScal = kOffBC + kBCBytes;
  static constexpr int kBytes = kOffScal + kScalBytes;
};

template <typename IOT, int N>
struct CarrySmem {
  static constexpr int kTen = 4;  // x, delta, dy, z
  static constexpr int kBCBytes = 2 * kBT * 2 * N * 4;
  static constexpr int kScalBytes = 2 * kTen * kBT * kNT * (int)sizeof(IOT);
  static constexpr int kOffBC = 0;
  static constexpr int kOffScal = kBCBytes;
  static constexpr int kBytes = kOffScal + kScalBytes;
};

// exp of an exponent already in the path's units (log2 units when kFast).
template <bool kFast>
__device__ __forceinline__ float exp_u(float e) {
  if constexpr (kFast) return ex2_approx(e);
  else return expf(e);
}

// Step size and the derivative of the softplus at v = delta + bias.
// dt: Delta (natural units); q: the decay exponent scale (Delta, or Delta
// log2(e) when kFast); sp: dDelta/dv.
template <bool kFast>
__device__ __forceinline__ void step_size(float v, int softplus, float& dt, float& q, float& sp) {
  if (!softplus) {
    dt = v;
    sp = 1.f;
  } else if (v > kSoftplusCut) {
    dt = v;
    sp = 1.f;
  } else if constexpr (kFast) {
    const float e = ex2_approx(v * kLog2e);
    dt = kLn2 * lg2_approx(1.f + e);
    sp = e * rcp_approx(1.f + e);
  } else {
    dt = log1pf(expf(v));
    sp = 1.f / (1.f + expf(-v));
  }
  q = kFast ? dt * kLog2e : dt;
}

// sigmoid(z)
template <bool kFast>
__device__ __forceinline__ float sigmoid_f(float z) {
  if constexpr (kFast) {
    return fmaf(0.5f, tanh_approx(0.5f * z), 0.5f);
  } else {
    return 1.f / (1.f + expf(-z));
  }
}

// Decays a_n = exp(Delta A_n) of one step as pairs (a_2k, a_2k+1):
// structured A by a multiply chain from r = exp(Delta A_0), else one exp per
// state (Ap: the row of A as pairs, in registers).
template <int N, bool kFast, bool kStruct>
__device__ __forceinline__ void decays2(float q, float A0, const float2 (&Ap)[N / 2],
                                        float2 (&a)[N / 2]) {
  if constexpr (kStruct) {
    const float r = exp_u<kFast>(q * A0);
    const float r2 = r * r;
    a[0] = make_float2(r, r2);
    const float2 rr = make_float2(r2, r2);
#pragma unroll
    for (int k = 1; k < N / 2; ++k) a[k] = mul2(a[k - 1], rr);
  } else {
#pragma unroll
    for (int k = 0; k < N / 2; ++k)
      a[k] = make_float2(exp_u<kFast>(q * Ap[k].x), exp_u<kFast>(q * Ap[k].y));
  }
}

// Structured-A test over the CTA (A[d,n] == (n+1) A[d,0] for all its channels).
template <int N>
__device__ __forceinline__ bool cta_structured(const float* Arow, float& A0) {
  A0 = Arow[0];
  bool st = true;
#pragma unroll
  for (int n = 1; n < N; ++n) st = st && (Arow[n] == (float)(n + 1) * A0);
  return __syncthreads_and(st) != 0;
}

// src[ten] for a run-time `ten`, by selects (no local-memory array).
template <typename IOT, int NTEN>
__device__ __forceinline__ const IOT* pick(const IOT* const (&src)[NTEN], int ten) {
  const IOT* s = src[0];
#pragma unroll
  for (int i = 1; i < NTEN; ++i) s = ten == i ? src[i] : s;
  return s;
}

// Issue the asynchronous copies of the per-step scalars of one tile: NTEN io
// tensors (nullptr entries are skipped) x kBT steps x the CTA's 128 channels
// into dst[NTEN][kBT][kNT], spread over the CTA's NTHR threads. Steps at or
// past `nt` and channels past dim are zero-filled. bf16 moves pairs of
// channels per 4-byte copy when `pairs` (even dim, 4-byte aligned tensors);
// otherwise each element is loaded synchronously.
template <typename IOT, int NTEN, int NTHR>
__device__ __forceinline__ void issue_scalars(IOT* dst, const IOT* const (&src)[NTEN],
                                              const BwdParams& p, int b, int tau, int nt,
                                              int d0, bool pairs) {
  const int tid = threadIdx.x;
  const int L = p.seqlen, dim = p.dim;
  constexpr int kRows = NTEN * kBT;
  if (sizeof(IOT) == 4 || pairs) {
    constexpr int EPC = 4 / (int)sizeof(IOT);  // elements per 4-byte copy
    constexpr int CPR = kNT / EPC;             // copies per row
    static_assert((kRows * CPR) % NTHR == 0, "copies must spread evenly over the CTA");
#pragma unroll
    for (int it = 0; it < kRows * CPR / NTHR; ++it) {
      const int c = it * NTHR + tid;
      const int r = c / CPR, q = c % CPR;
      const int ten = r / kBT, j = r % kBT;
      const IOT* sp = pick<IOT, NTEN>(src, ten);
      if (!sp) continue;
      const int d = d0 + EPC * q;
      const uint32_t bytes =
          (j < nt && d < dim) ? (uint32_t)(min(EPC, dim - d) * (int)sizeof(IOT)) : 0u;
      const IOT* g = bytes ? sp + ((size_t)b * L + tau + j) * dim + d : sp;
      cp_async4(dst + r * kNT + EPC * q, g, bytes);
    }
  } else {
    for (int c = tid; c < kRows * kNT; c += NTHR) {
      const int r = c / kNT, q = c % kNT;
      const int ten = r / kBT, j = r % kBT;
      const IOT* sp = pick<IOT, NTEN>(src, ten);
      if (!sp) continue;
      const int d = d0 + q;
      dst[c] = (j < nt && d < dim) ? sp[((size_t)b * L + tau + j) * dim + d] : IOT(0);
    }
  }
}

// One element of a tile's B / C rows (threads < kBT * ncols), as fp32.
template <typename IOT, int N>
__device__ __forceinline__ float bc_element(const BwdParams& p, const IOT* B, const IOT* C, int b,
                                            int tau, int nt, int ncols) {
  using IO = Io<IOT>;
  const int tid = threadIdx.x;
  if (tid >= kBT * ncols) return 0.f;
  const int j = tid / ncols, v = tid % ncols;
  if (j >= nt) return 0.f;
  const IOT* src = (v < N ? B : C) + ((size_t)b * p.seqlen + tau + j) * N + (v % N);
  return IO::load(src);
}

// Per-step quantities of one channel, from the staged scalars.
struct StepIn {
  float x, dt, q, sp, dy, z, g;
};

template <typename IOT, bool kFast>
__device__ __forceinline__ StepIn step_in(const IOT* sScal, int j, int tid, float bias,
                                          int softplus, bool has_z) {
  using IO = Io<IOT>;
  StepIn s;
  s.x = IO::load(sScal + (0 * kBT + j) * kNT + tid);
  step_size<kFast>(IO::load(sScal + (1 * kBT + j) * kNT + tid) + bias, softplus, s.dt, s.q, s.sp);
  s.dy = IO::load(sScal + (2 * kBT + j) * kNT + tid);
  if (has_z) {
    s.z = IO::load(sScal + (3 * kBT + j) * kNT + tid);
    s.g = s.dy * s.z * sigmoid_f<kFast>(s.z);
  } else {
    s.z = 0.f;
    s.g = s.dy;
  }
  return s;
}

// ---------------------------------------------------------------------------
// 1. carry: checkpoints, local segment end states and outgoing adjoints.
template <typename IOT, int N, bool kStruct>
__device__ __forceinline__ void carry_body(const BwdParams& p, unsigned char* smem,
                                           const float* Arow, float A0, int b, int seg, int dblk,
                                           int dc, bool valid) {
  using SM = CarrySmem<IOT, N>;
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  constexpr int NP = N / 2, V = 2 * N;
  float* sBC = reinterpret_cast<float*>(smem + SM::kOffBC);  // [2][kBT][V]
  IOT* sScal = reinterpret_cast<IOT*>(smem + SM::kOffScal);  // [2][4][kBT][kNT]
  constexpr int kBuf = SM::kTen * kBT * kNT;
  const int tid = threadIdx.x;
  const int L = p.seqlen, dim = p.dim, d0 = dblk * kNT;
  const int t0 = seg * p.seg_steps;
  const int t1 = min(L, t0 + p.seg_steps);
  const int ntile = (t1 - t0 + kBT - 1) / kBT;
  const bool pairs = p.scal_pairs != 0, has_z = p.z != nullptr;
  const IOT* Bg = reinterpret_cast<const IOT*>(p.B);
  const IOT* Cg = reinterpret_cast<const IOT*>(p.C);
  const float bias = p.bias ? p.bias[dc] : 0.f;
  const IOT* const src[4] = {reinterpret_cast<const IOT*>(p.x),
                             reinterpret_cast<const IOT*>(p.delta),
                             reinterpret_cast<const IOT*>(p.dy),
                             reinterpret_cast<const IOT*>(p.z)};

  // One forward sweep from a zero state over the segment:
  //   h     the state (checkpointed at every tile start),
  //   P_n   prod_{u <= t} a_n(u) from the segment start,
  //   m_n   sum_t P_n(t) C_n(t) g_t: the segment's outgoing adjoint from a
  //         zero end, a(t0) lam(t0), accumulated forwards.
  float2 Ap[NP];  // row of A as pairs (the one-exp-per-state path reads it)
#pragma unroll
  for (int k = 0; k < NP; ++k)
    Ap[k] = kStruct ? make_float2(0.f, 0.f) : __ldg(reinterpret_cast<const float2*>(Arow) + k);
  float2 h[NP], P[NP], m[NP];
#pragma unroll
  for (int k = 0; k < NP; ++k) {
    h[k] = make_float2(0.f, 0.f);
    P[k] = make_float2(1.f, 1.f);
    m[k] = make_float2(0.f, 0.f);
  }
  float Q = 0.f;
  float bcr = bc_element<IOT, N>(p, Bg, Cg, b, t0, min(kBT, t1 - t0), V);
  issue_scalars<IOT, 4, kNT>(sScal, src, p, b, t0, min(kBT, t1 - t0), d0, pairs);
  cp_async_commit();
  for (int k = 0; k < ntile; ++k) {
    const int tau = t0 + k * kBT;
    const int nt = min(kBT, t1 - tau);
    const int buf = k & 1;
    if (tid < kBT * V) sBC[buf * kBT * V + tid] = bcr;
    if (k + 1 < ntile) {
      const int tn = tau + kBT, ntn = min(kBT, t1 - tn);
      bcr = bc_element<IOT, N>(p, Bg, Cg, b, tn, ntn, V);
      issue_scalars<IOT, 4, kNT>(sScal + (buf ^ 1) * kBuf, src, p, b, tn, ntn, d0, pairs);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (valid) {
      const int gt = tau / kBT;
      float* ck = p.ws_ck + ((size_t)b * p.ntiles + gt) * N * dim + dc;
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        ck[(size_t)(2 * q) * dim] = h[q].x;
        ck[(size_t)(2 * q + 1) * dim] = h[q].y;
      }
      p.ws_qk[((size_t)b * p.ntiles + gt) * dim + dc] = Q;
    }
    const IOT* sS = sScal + buf * kBuf;
    const float2* sBC2 = reinterpret_cast<const float2*>(sBC + buf * kBT * V);
#pragma unroll
    for (int j = 0; j < kBT; ++j) {
      if (j < nt) {
        const StepIn s = step_in<IOT, kFast>(sS, j, tid, bias, p.softplus, has_z);
        float2 a[NP];
        decays2<N, kFast, kStruct>(s.q, A0, Ap, a);
        const float2 dtx = make_float2(s.dt * s.x, s.dt * s.x);
        const float2 g2 = make_float2(s.g, s.g);
#pragma unroll
        for (int q = 0; q < NP; ++q) {
          h[q] = fma2(a[q], h[q], mul2(dtx, sBC2[j * N + q]));
          P[q] = mul2(P[q], a[q]);
          m[q] = fma2(P[q], mul2(sBC2[j * N + NP + q], g2), m[q]);
        }
        Q += s.q;
      }
    }
    __syncthreads();  // buffer `buf` is refilled next
  }
  cp_async_wait<0>();
  if (valid) {
    const size_t sb = (size_t)b * p.nseg + seg;
    p.ws_qseg[sb * dim + dc] = Q;
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      if (seg < p.nseg - 1) {
        p.ws_hloc[(sb * N + 2 * q) * dim + dc] = h[q].x;
        p.ws_hloc[(sb * N + 2 * q + 1) * dim + dc] = h[q].y;
      }
      if (seg > 0) {
        p.ws_mloc[(sb * N + 2 * q) * dim + dc] = m[q].x;
        p.ws_mloc[(sb * N + 2 * q + 1) * dim + dc] = m[q].y;
      }
    }
  }
}

template <typename IOT, int N>
__global__ void __launch_bounds__(kNT) bwd_carry_kernel(const BwdParams p) {
  extern __shared__ float4 smem4[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(smem4);
  const int dblk = blockIdx.x, seg = blockIdx.y, b = blockIdx.z;
  const int d = dblk * kNT + threadIdx.x;
  const bool valid = d < p.dim;
  const int dc = valid ? d : p.dim - 1;
  const float* Arow = p.A + (size_t)dc * N;
  float A0;
  if (cta_structured<N>(Arow, A0)) carry_body<IOT, N, true>(p, smem, Arow, A0, b, seg, dblk, dc, valid);
  else carry_body<IOT, N, false>(p, smem, Arow, A0, b, seg, dblk, dc, valid);
}

// ---------------------------------------------------------------------------
// 2. compose: true entering state and adjoint of every segment.
template <bool kFast>
__global__ void __launch_bounds__(256) bwd_compose_kernel(const BwdParams p, int N) {
  const size_t total = (size_t)p.batch * N * p.dim;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int d = (int)(i % p.dim);
    const int n = (int)((i / p.dim) % N);
    const int b = (int)(i / ((size_t)p.dim * N));
    const float An = p.A[(size_t)d * N + n];
    // the loads of 8 segments are issued before their 8 dependent steps
    constexpr int G = 8;
    float h = p.h0 ? p.h0[((size_t)b * p.dim + d) * N + n] : 0.f;
    for (int s0 = 0; s0 < p.nseg; s0 += G) {
      float qv[G], lc[G];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const int s = s0 + j;
        const size_t sb = (size_t)b * p.nseg + s;
        const bool step = s < p.nseg - 1;  // the last segment's carry is not needed
        qv[j] = step ? p.ws_qseg[sb * p.dim + d] : 0.f;
        lc[j] = step ? p.ws_hloc[(sb * N + n) * p.dim + d] : 0.f;
      }
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const int s = s0 + j;
        if (s >= p.nseg) break;
        const size_t sb = (size_t)b * p.nseg + s;
        p.ws_hin[(sb * N + n) * p.dim + d] = h;
        if (s < p.nseg - 1) h = fmaf(exp_u<kFast>(qv[j] * An), h, lc[j]);
      }
    }
    float mu = p.dh_last ? p.dh_last[((size_t)b * p.dim + d) * N + n] : 0.f;
    for (int s0 = p.nseg - 1; s0 >= 0; s0 -= G) {
      float qv[G], lc[G];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const int s = s0 - j;
        const size_t sb = (size_t)b * p.nseg + (s > 0 ? s : 0);
        const bool step = s > 0;  // the first segment's carry is not needed
        qv[j] = step ? p.ws_qseg[sb * p.dim + d] : 0.f;
        lc[j] = step ? p.ws_mloc[(sb * N + n) * p.dim + d] : 0.f;
      }
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const int s = s0 - j;
        if (s < 0) break;
        const size_t sb = (size_t)b * p.nseg + s;
        p.ws_muin[(sb * N + n) * p.dim + d] = mu;
        if (s > 0) mu = fmaf(exp_u<kFast>(qv[j] * An), mu, lc[j]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// 3. main: tiles of 4 steps in reverse, recomputed into registers.
// Threads per channel of the main kernel (each holds N / TPC states), the
// resulting CTA size, and the threads that share one row of the channel sum.
// One thread per channel measured fastest at N = 16: two threads per channel
// halve the registers and double the resident warps, but duplicate the
// per-channel scalar work and add three shuffles per step.
#ifndef SSM_BWD_TPC
#define SSM_BWD_TPC 1
#endif
template <int N>
struct MainShape {
  static constexpr int TPC = (N >= 4) ? SSM_BWD_TPC : 1;
  static constexpr int NTHR = kNT * TPC;
  static constexpr int NQ = N / 2 / TPC;  // state pairs per thread
  static constexpr int kRows = kBT * N;   // rows of the channel-sum buffer
  static constexpr int RT0 = NTHR / kRows;
  static constexpr int RT = RT0 >= 4 ? 4 : (RT0 >= 2 ? 2 : 1);  // threads per row
  static constexpr int kMinBlocks = TPC == 2 ? 2 : (N <= 4 ? 4 : 2);
};

template <typename IOT, int N>
__device__ __forceinline__ void issue_main_tile(const BwdParams& p, unsigned char* smem, int buf,
                                                int b, int tau, int nt, int dblk, int dc, int h,
                                                bool valid, float& bcr) {
  using SM = MainSmem<IOT, N>;
  using S = MainShape<N>;
  const int c = threadIdx.x / S::TPC;  // channel within the CTA
  const int dim = p.dim;
  IOT* sScal = reinterpret_cast<IOT*>(smem + SM::kOffScal) + buf * SM::kTen * kBT * kNT;
  const IOT* const src[4] = {reinterpret_cast<const IOT*>(p.x),
                             reinterpret_cast<const IOT*>(p.delta),
                             reinterpret_cast<const IOT*>(p.dy),
                             reinterpret_cast<const IOT*>(p.z)};
  issue_scalars<IOT, 4, S::NTHR>(sScal, src, p, b, tau, nt, dblk * kNT, p.scal_pairs != 0);
  // checkpoint of the tile start (this thread's states) and its summed exponent
  float* sCk = reinterpret_cast<float*>(smem + SM::kOffCk) + buf * (N + 1) * kNT;
  const int gt = tau / kBT;
  const float* ck = p.ws_ck + ((size_t)b * p.ntiles + gt) * N * dim + dc;
  constexpr int NS = N / S::TPC;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    const int n = h * NS + i;
    cp_async4(sCk + n * kNT + c, ck + (size_t)n * dim, valid ? 4u : 0u);
  }
  if (h == 0)
    cp_async4(sCk + N * kNT + c, p.ws_qk + ((size_t)b * p.ntiles + gt) * dim + dc, valid ? 4u : 0u);
  bcr = bc_element<IOT, N>(p, reinterpret_cast<const IOT*>(p.B), reinterpret_cast<const IOT*>(p.C),
                           b, tau, nt, 2 * N);
}

// Decays of this thread's state pairs q0 .. q0+NQ-1: (r^(2q+1), r^(2q+2)),
// or one exp per state for generic A (Ap: this thread's pairs of A).
template <int N, bool kFast, bool kStruct>
__device__ __forceinline__ void decays_own(float qs, float A0,
                                           const float2 (&Ap)[MainShape<N>::NQ], int q0,
                                           float2 (&a)[MainShape<N>::NQ]) {
  constexpr int NQ = MainShape<N>::NQ;
  if constexpr (kStruct) {
    const float r = exp_u<kFast>(qs * A0);
    const float r2 = r * r;
    float base = 1.f;
    if constexpr (MainShape<N>::TPC == 2) {
      // r^(2 q0) for q0 in {0, NQ}: 2 NQ = N / 2 is a power of two
      float rp = r2;
#pragma unroll
      for (int m = 2; m < 2 * NQ; m *= 2) rp *= rp;
      base = q0 ? rp : 1.f;
    }
    a[0] = make_float2(r * base, r2 * base);
    const float2 rr = make_float2(r2, r2);
#pragma unroll
    for (int i = 1; i < NQ; ++i) a[i] = mul2(a[i - 1], rr);
  } else {
#pragma unroll
    for (int i = 0; i < NQ; ++i)
      a[i] = make_float2(exp_u<kFast>(qs * Ap[i].x), exp_u<kFast>(qs * Ap[i].y));
    (void)q0;
  }
}

template <typename IOT, int N, bool kStruct>
__device__ __forceinline__ void main_body(const BwdParams& p, unsigned char* smem,
                                          const float* Arow, float A0, int b, int seg, int dblk,
                                          int dc, bool valid) {
  using IO = Io<IOT>;
  using SM = MainSmem<IOT, N>;
  using S = MainShape<N>;
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  constexpr int NP = N / 2, NQ = S::NQ, TPC = S::TPC;
  constexpr int V = 2 * N;  // channel-summed values per step: dB_n, dC_n
  float* sRed = reinterpret_cast<float*>(smem + SM::kOffRed);   // [kBT][2][NP][kRowF]
  float* sHin = reinterpret_cast<float*>(smem + SM::kOffHin);   // [N][kNT]
  const float* sCkAll = reinterpret_cast<const float*>(smem + SM::kOffCk);
  float* sBCAll = reinterpret_cast<float*>(smem + SM::kOffBC);  // [2][kBT][V]
  const IOT* sScalAll = reinterpret_cast<const IOT*>(smem + SM::kOffScal);
  const int tid = threadIdx.x;
  const int c = tid / TPC, h = tid % TPC;  // channel within the CTA, half of the state
  const int q0 = h * NQ;                   // first state pair of this thread
  const int L = p.seqlen, dim = p.dim;
  const int t0 = seg * p.seg_steps;
  const int t1 = min(L, t0 + p.seg_steps);
  const int ntile = (t1 - t0 + kBT - 1) / kBT;
  const bool has_z = p.z != nullptr;
  IOT* dxg = reinterpret_cast<IOT*>(p.dx);
  IOT* ddg = reinterpret_cast<IOT*>(p.ddelta);
  IOT* dzg = reinterpret_cast<IOT*>(p.dz);
  const float bias = p.bias ? p.bias[dc] : 0.f;
  const float Dd = p.D ? p.D[dc] : 0.f;

  const size_t sb = (size_t)b * p.nseg + seg;
  float2 mu[NQ], dA[NQ], coef[NQ];
#pragma unroll
  for (int i = 0; i < NQ; ++i) {
    const int n = 2 * (q0 + i);
    sHin[n * kNT + c] = p.ws_hin[(sb * N + n) * dim + dc];
    sHin[(n + 1) * kNT + c] = p.ws_hin[(sb * N + n + 1) * dim + dc];
    // channels past dim carry a zero adjoint, so they add nothing to dB
    mu[i] = valid ? make_float2(p.ws_muin[(sb * N + n) * dim + dc],
                                p.ws_muin[(sb * N + n + 1) * dim + dc])
                  : make_float2(0.f, 0.f);
    dA[i] = make_float2(0.f, 0.f);
    // A_n for the dDelta sum: (n + 1) when structured (times A_0 after the sum)
    coef[i] = kStruct ? make_float2((float)(n + 1), (float)(n + 2))
                      : make_float2(__ldg(Arow + n), __ldg(Arow + n + 1));
  }
  float dD_acc = 0.f, dbias_acc = 0.f;

  float bcr;
  {
    const int tau = t0 + (ntile - 1) * kBT;
    issue_main_tile<IOT, N>(p, smem, 0, b, tau, t1 - tau, dblk, dc, h, valid, bcr);
    cp_async_commit();
  }
  for (int k = ntile - 1, it = 0; k >= 0; --k, ++it) {
    const int tau = t0 + k * kBT;
    const int nt = min(kBT, t1 - tau);
    const int buf = it & 1;
    if (tid < kBT * V) sBCAll[buf * kBT * V + tid] = bcr;
    if (k > 0)
      issue_main_tile<IOT, N>(p, smem, buf ^ 1, b, tau - kBT, kBT, dblk, dc, h, valid, bcr);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();  // tile k staged by every thread; sRed free

    const IOT* sScal = sScalAll + buf * SM::kTen * kBT * kNT;
    const float* sCk = sCkAll + buf * (N + 1) * kNT;
    // row j: (B_j pairs)[NP], (C_j pairs)[NP]
    const float2* sBC2 = reinterpret_cast<const float2*>(sBCAll + buf * kBT * V);
    // the tile's true entry state: checkpoint + exp(A_n Q) h_in
    float2 he[NQ];
    {
      float2 P[NQ];
      decays_own<N, kFast, kStruct>(sCk[N * kNT + c], A0, coef, q0, P);
#pragma unroll
      for (int i = 0; i < NQ; ++i) {
        const int n = 2 * (q0 + i);
        he[i] = fma2(P[i], make_float2(sHin[n * kNT + c], sHin[(n + 1) * kNT + c]),
                     make_float2(sCk[n * kNT + c], sCk[(n + 1) * kNT + c]));
      }
    }
    // recompute the tile's states
    float2 hist[kBT][NQ];
#pragma unroll
    for (int j = 0; j < kBT; ++j) {
      const StepIn s = step_in<IOT, kFast>(sScal, j, c, bias, p.softplus, has_z);
      float2 a[NQ];
      decays_own<N, kFast, kStruct>(s.q, A0, coef, q0, a);
      const float2 dtx = make_float2(s.dt * s.x, s.dt * s.x);
#pragma unroll
      for (int i = 0; i < NQ; ++i)
        hist[j][i] = fma2(a[i], j == 0 ? he[i] : hist[j - 1][i], mul2(dtx, sBC2[j * N + q0 + i]));
    }
    // adjoint, backwards through the tile
#pragma unroll
    for (int j = kBT - 1; j >= 0; --j) {
      if (j < nt) {
        const StepIn s = step_in<IOT, kFast>(sScal, j, c, bias, p.softplus, has_z);
        float2 a[NQ];
        decays_own<N, kFast, kStruct>(s.q, A0, coef, q0, a);
        const float2 g2 = make_float2(s.g, s.g);
        const float2 dt2 = make_float2(s.dt, s.dt);
        const float2 dtx2 = make_float2(s.dt * s.x, s.dt * s.x);
        float2 S1 = make_float2(0.f, 0.f), S2 = S1, ys = S1;
        float2* rowB = reinterpret_cast<float2*>(sRed + (size_t)((j * 2 + 0) * NP + q0) * kRowF) + c;
        float2* rowC = reinterpret_cast<float2*>(sRed + (size_t)((j * 2 + 1) * NP + q0) * kRowF) + c;
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
          const float2 B2 = sBC2[j * N + q0 + i], C2 = sBC2[j * N + NP + q0 + i];
          const float2 prev = j == 0 ? he[i] : hist[j - 1][i];
          const float2 lam = fma2(C2, g2, mu[i]);
          S1 = fma2(lam, B2, S1);
          const float2 qv = mul2(lam, mul2(a[i], prev));
          S2 = fma2(qv, coef[i], S2);
          dA[i] = fma2(qv, dt2, dA[i]);
          ys = fma2(C2, hist[j][i], ys);
          rowB[i * (kRowF / 2)] = mul2(lam, dtx2);
          rowC[i * (kRowF / 2)] = mul2(g2, hist[j][i]);
          mu[i] = mul2(a[i], lam);
        }
        float s1 = S1.x + S1.y, s2 = S2.x + S2.y, yss = ys.x + ys.y;
        if constexpr (TPC == 2) {
          s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
          s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
          yss += __shfl_xor_sync(0xffffffffu, yss, 1);
        }
        if constexpr (kStruct) s2 *= A0;
        const float dxv = fmaf(Dd, s.g, s.dt * s1);
        const float ddv = fmaf(s.x, s1, s2) * s.sp;
        dD_acc = fmaf(s.g, s.x, dD_acc);
        dbias_acc += ddv;
        if (valid) {
          const size_t gi = ((size_t)b * L + tau + j) * dim + dc;
          if (h == 0) {
            IO::store(dxg + gi, dxv);
            IO::store(ddg + gi, ddv);
          }
          if (has_z && h == TPC - 1) {
            const float sg = sigmoid_f<kFast>(s.z);
            const float ssum = fmaf(Dd, s.x, yss);
            IO::store(dzg + gi, s.dy * ssum * sg * fmaf(s.z, 1.f - sg, 1.f));
          }
        }
      }
    }
    __syncthreads();  // every channel's values are in sRed
    // sum over the CTA's channels: RT threads per row (a share of the channels each)
    {
      constexpr int kRows = S::kRows, RT = S::RT;
      constexpr int F4 = kNT / 2 / RT;  // float4 (two channels, one pair) per thread
      const int r = tid / RT, qr = tid % RT;
      float2 sum = make_float2(0.f, 0.f);
      if (r < kRows) {
        const float4* row = reinterpret_cast<const float4*>(sRed + (size_t)r * kRowF) + qr * F4;
        float2 a0 = make_float2(0.f, 0.f), a1 = a0;
#pragma unroll 8
        for (int m = 0; m < F4; ++m) {
          // rotated start: the RT threads of neighbouring rows hit different banks
          const float4 w = row[(m + (8 / RT) * qr) & (F4 - 1)];
          a0 = add2(a0, make_float2(w.x, w.y));
          a1 = add2(a1, make_float2(w.z, w.w));
        }
        sum = add2(a0, a1);
      }
#pragma unroll
      for (int o = 1; o < RT; o *= 2) {
        sum.x += __shfl_xor_sync(0xffffffffu, sum.x, o);
        sum.y += __shfl_xor_sync(0xffffffffu, sum.y, o);
      }
      if (r < kRows && qr == 0) {
        const int j = r / N, rem = r % N, kind = rem / NP, q = rem % NP;
        if (j < nt)
          *reinterpret_cast<float2*>(
              p.ws_dbc + (((size_t)b * p.dblocks + dblk) * L + tau + j) * V + kind * N + 2 * q) = sum;
      }
    }
  }
  cp_async_wait<0>();
  if (valid) {
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
      const int n = 2 * (q0 + i);
      if (seg == 0 && p.dh0) {
        p.dh0[((size_t)b * dim + dc) * N + n] = mu[i].x;
        p.dh0[((size_t)b * dim + dc) * N + n + 1] = mu[i].y;
      }
      p.ws_dA[(sb * N + n) * dim + dc] = dA[i].x;
      p.ws_dA[(sb * N + n + 1) * dim + dc] = dA[i].y;
    }
    if (h == 0) {
      p.ws_dD[sb * dim + dc] = dD_acc;
      p.ws_dbias[sb * dim + dc] = dbias_acc;
    }
  }
}

template <typename IOT, int N>
__global__ void __launch_bounds__(MainShape<N>::NTHR, MainShape<N>::kMinBlocks)
    bwd_main_kernel(const BwdParams p) {
  extern __shared__ float4 smem4[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(smem4);
  const int dblk = blockIdx.x, seg = blockIdx.y, b = blockIdx.z;
  const int d = dblk * kNT + (int)threadIdx.x / MainShape<N>::TPC;
  const bool valid = d < p.dim;
  const int dc = valid ? d : p.dim - 1;
  const float* Arow = p.A + (size_t)dc * N;
  float A0;
  if (cta_structured<N>(Arow, A0)) main_body<IOT, N, true>(p, smem, Arow, A0, b, seg, dblk, dc, valid);
  else main_body<IOT, N, false>(p, smem, Arow, A0, b, seg, dblk, dc, valid);
}

// ---------------------------------------------------------------------------
// 4. reduce, two launches in a fixed order of summation (results do not
// depend on scheduling). dB, dC: per (b, t, v) the sum over channel blocks,
// one batch row per grid row (V = 2N a compile-time power of two: no
// division by a run-time size).
template <int N>
__global__ void __launch_bounds__(256) bwd_reduce_bc_kernel(const BwdParams p) {
  constexpr int V = 2 * N;
  const int b = blockIdx.y;
  const size_t per_row = (size_t)p.seqlen * V;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < per_row;
       i += (size_t)gridDim.x * blockDim.x) {
    const int v = (int)(i % V);
    const size_t t = i / V;
    float acc = 0.f;
    for (int k = 0; k < p.dblocks; ++k)
      acc += p.ws_dbc[(((size_t)b * p.dblocks + k) * p.seqlen + t) * V + v];
    const size_t bt = (size_t)b * p.seqlen + t;
    if (v < N) p.dB[bt * N + v] = acc;
    else p.dC[bt * N + (v - N)] = acc;
  }
}

// dA, dD, dbias: sums over the (batch, segment) partials. A CTA takes 32
// consecutive channels (lanes: coalesced reads) and one state n (grid row n;
// row N: dD and dbias); its 8 warps each sum every 8th partial, and the 8
// slices are added in a fixed order (results do not depend on scheduling).
template <int N>
__global__ void __launch_bounds__(256) bwd_reduce_par_kernel(const BwdParams p) {
  __shared__ float part[2][8][33];
  const int lane = threadIdx.x & 31, slice = threadIdx.x >> 5;
  const int d = blockIdx.x * 32 + lane;
  const int n = blockIdx.y;
  const bool valid = d < p.dim;
  const size_t bs = (size_t)p.batch * p.nseg;
  float a1 = 0.f, a2 = 0.f;
  if (valid) {
    if (n < N) {
      const float* src = p.ws_dA + (size_t)n * p.dim + d;  // [s][N][dim]
      const size_t stride = (size_t)N * p.dim;
#pragma unroll 4
      for (size_t s = slice; s < bs; s += 8) a1 += src[s * stride];
    } else {
#pragma unroll 4
      for (size_t s = slice; s < bs; s += 8) {
        a1 += p.ws_dD[s * p.dim + d];
        a2 += p.ws_dbias[s * p.dim + d];
      }
    }
  }
  part[0][slice][lane] = a1;
  part[1][slice][lane] = a2;
  __syncthreads();
  if (slice == 0 && valid) {
    float r1 = 0.f, r2 = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      r1 += part[0][k][lane];
      r2 += part[1][k][lane];
    }
    if (n < N) {
      p.dA[(size_t)d * N + n] = r1;
    } else {
      if (p.dD) p.dD[d] = r1;
      if (p.dbias) p.dbias[d] = r2;
    }
  }
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

int grid_for(size_t work, int threads) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  const size_t want = (work + threads - 1) / threads;
  return (int)std::max<size_t>(1, std::min<size_t>(want, (size_t)sms * 8));
}

template <typename IOT, int N>
cudaError_t launch_bwd_t(const BwdParams& p, cudaStream_t stream) {
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  const dim3 grid(p.dblocks, p.nseg, p.batch);
  const int carry_bytes = CarrySmem<IOT, N>::kBytes;
  const int main_bytes = MainSmem<IOT, N>::kBytes;
  cudaError_t e = set_smem(bwd_carry_kernel<IOT, N>, carry_bytes);
  if (e != cudaSuccess) return e;
  e = set_smem(bwd_main_kernel<IOT, N>, main_bytes);
  if (e != cudaSuccess) return e;
  bwd_carry_kernel<IOT, N><<<grid, kNT, carry_bytes, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_compose_kernel<kFast><<<grid_for((size_t)p.batch * N * p.dim, 256), 256, 0, stream>>>(p, N);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_main_kernel<IOT, N><<<grid, MainShape<N>::NTHR, main_bytes, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    const size_t per_row = (size_t)p.seqlen * 2 * N;
    const int gx = std::max(1, std::min(grid_for(per_row, 256), 1 + 1184 / std::max(1, p.batch)));
    bwd_reduce_bc_kernel<N><<<dim3((unsigned)gx, (unsigned)p.batch), 256, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  bwd_reduce_par_kernel<N><<<dim3((unsigned)((p.dim + 31) / 32), (unsigned)(N + 1)), 256, 0,
                               stream>>>(p);
  return cudaGetLastError();
}

template <typename IOT>
cudaError_t launch_bwd_io(const BwdParams& p, int dstate, cudaStream_t stream) {
  switch (dstate) {
    case 2: return launch_bwd_t<IOT, 2>(p, stream);
    case 4: return launch_bwd_t<IOT, 4>(p, stream);
    case 8: return launch_bwd_t<IOT, 8>(p, stream);
    case 16: return launch_bwd_t<IOT, 16>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool scan_bwd_dstate_supported(int dstate) {
  return dstate == 2 || dstate == 4 || dstate == 8 || dstate == 16;
}

cudaError_t launch_scan_bwd(const BwdParams& p, int dstate, bool bf16, cudaStream_t stream) {
  return bf16 ? launch_bwd_io<uint16_t>(p, dstate, stream) : launch_bwd_io<float>(p, dstate, stream);
}

}  // namespace ssm
