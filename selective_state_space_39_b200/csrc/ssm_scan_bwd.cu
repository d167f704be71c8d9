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
//  * Four launches, none of which waits on another CTA:
//    1. carry: per (segment, channel block, batch row) the forward from a
//       zero state, storing the state at every 4-step tile start (and the
//       summed decay exponent there), the segment's end state, and the
//       segment's outgoing adjoint from a zero end (the reverse recurrence).
//    2. compose: per (b, n, d) the exact chaining of those affine carries
//       across segments, giving the true entering state and adjoint of every
//       segment (the associative scan of (a, b) maps, done sequentially over
//       the few segments).
//    3. main: per segment, tiles of 4 steps in reverse order. A tile's true
//       entry state is its checkpoint plus exp(A_n Q) times the segment's
//       entering state; the tile's 4 steps are recomputed into a register
//       history, then the adjoint runs backwards through them.
//    4. reduce: dB and dC (sums over channels) from per-CTA partials, dA, dD,
//       dbias (sums over batch rows and segments) from per-segment partials,
//       in a fixed order, so results do not depend on scheduling.
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

#include "ssm_device.cuh"
#include "ssm_internal.h"

namespace ssm {

namespace {

constexpr int kBT = kBwdTileSteps;
constexpr int kNT = kBwdThreads;
// Row stride (floats) of the channel-sum buffer: 16-byte aligned rows whose
// starts fall on different bank groups.
constexpr int kRedStride = kNT + 4;

// Shared memory of the two sequential kernels. Per-step scalars (NTEN io
// tensors x kBT steps x 128 channels) and the fp32 B / C rows of a tile are
// double-buffered: the copies of the next tile are in flight while the
// current one is computed.
template <typename IOT, int N>
struct MainSmem {
  static constexpr int kTen = 4;  // x, delta, dy, z
  static constexpr int kRedBytes = kBT * 2 * N * kRedStride * 4;
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
  static constexpr int kTen = 3;  // x, delta (forward); delta, dy, z (adjoint)
  static constexpr int kBCBytes = 2 * kBT * N * 4;
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

// Decays a_n = exp(Delta A_n) for one step: structured A by a multiply chain
// from r = exp(Delta A_0), else one exp per state (A row read through L1).
template <int N, bool kFast, bool kStruct>
__device__ __forceinline__ void decays(float q, float A0, const float* Arow, float (&a)[N]) {
  if constexpr (kStruct) {
    const float r = exp_u<kFast>(q * A0);
    a[0] = r;
    if constexpr (N > 1) {
      const float r2 = r * r;
      a[1] = r2;
#pragma unroll
      for (int n = 2; n < N; ++n) a[n] = a[n - 2] * r2;
    }
  } else {
#pragma unroll
    for (int n = 0; n < N; ++n) a[n] = exp_u<kFast>(q * __ldg(Arow + n));
  }
}

// A_n for the dDelta sum: (n+1) when structured (times A_0 after the sum).
template <int N, bool kStruct>
__device__ __forceinline__ float a_coef(int n, const float* Arow) {
  if constexpr (kStruct) return (float)(n + 1);
  else return __ldg(Arow + n);
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

// Issue the asynchronous copies of the per-step scalars of one tile: NTEN io
// tensors (nullptr entries are skipped) x kBT steps x the CTA's 128 channels
// into dst[NTEN][kBT][kNT]. Steps at or past `nt` and channels past dim are
// zero-filled. bf16 moves pairs of channels per 4-byte copy when `pairs`
// (even dim, 4-byte aligned tensors); otherwise each thread loads its own
// elements synchronously.
// src[ten] for a run-time `ten`, by selects (no local-memory array).
template <typename IOT, int NTEN>
__device__ __forceinline__ const IOT* pick(const IOT* const (&src)[NTEN], int ten) {
  const IOT* s = src[0];
#pragma unroll
  for (int i = 1; i < NTEN; ++i) s = ten == i ? src[i] : s;
  return s;
}

template <typename IOT, int NTEN>
__device__ __forceinline__ void issue_scalars(IOT* dst, const IOT* const (&src)[NTEN],
                                              const BwdParams& p, int b, int tau, int nt,
                                              int d0, bool pairs) {
  const int tid = threadIdx.x;
  const int L = p.seqlen, dim = p.dim;
  if constexpr (sizeof(IOT) == 4) {
    const int d = d0 + tid;
#pragma unroll
    for (int r = 0; r < NTEN * kBT; ++r) {
      const int ten = r / kBT, j = r % kBT;
      if (!src[ten]) continue;
      const bool ok = j < nt && d < dim;
      const IOT* g = ok ? src[ten] + ((size_t)b * L + tau + j) * dim + d : src[ten];
      cp_async4(dst + r * kNT + tid, g, ok ? 4u : 0u);
    }
  } else if (pairs) {
#pragma unroll
    for (int r2 = 0; r2 < NTEN * kBT / 2; ++r2) {
      const int c = r2 * kNT + tid;  // chunk: row c / 64, channel pair c % 64
      const int r = c / (kNT / 2), q = c % (kNT / 2);
      const int ten = r / kBT, j = r % kBT;
      const IOT* sp = pick<IOT, NTEN>(src, ten);
      if (!sp) continue;
      const int d = d0 + 2 * q;
      const uint32_t bytes = (j < nt && d < dim) ? (uint32_t)min(2, dim - d) * 2u : 0u;
      const IOT* g = bytes ? sp + ((size_t)b * L + tau + j) * dim + d : sp;
      cp_async4(dst + r * kNT + 2 * q, g, bytes);
    }
  } else {
    const int d = d0 + tid;
#pragma unroll
    for (int r = 0; r < NTEN * kBT; ++r) {
      const int ten = r / kBT, j = r % kBT;
      if (!src[ten]) continue;
      const bool ok = j < nt && d < dim;
      dst[r * kNT + tid] = ok ? src[ten][((size_t)b * L + tau + j) * dim + d] : IOT(0);
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

// ---------------------------------------------------------------------------
// 1. carry: checkpoints, local segment end states and outgoing adjoints.
template <typename IOT, int N, bool kStruct>
__device__ __forceinline__ void carry_body(const BwdParams& p, unsigned char* smem,
                                           const float* Arow, float A0, int b, int seg, int dblk,
                                           int dc, bool valid) {
  using IO = Io<IOT>;
  using SM = CarrySmem<IOT, N>;
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  float* sBC = reinterpret_cast<float*>(smem + SM::kOffBC);                   // [2][kBT][N]
  IOT* sScal = reinterpret_cast<IOT*>(smem + SM::kOffScal);                   // [2][3][kBT][kNT]
  constexpr int kBuf = SM::kTen * kBT * kNT;
  const int tid = threadIdx.x;
  const int L = p.seqlen, dim = p.dim, d0 = dblk * kNT;
  const int t0 = seg * p.seg_steps;
  const int t1 = min(L, t0 + p.seg_steps);
  const int ntile = (t1 - t0 + kBT - 1) / kBT;
  const bool pairs = p.scal_pairs != 0;
  const IOT* Bg = reinterpret_cast<const IOT*>(p.B);
  const IOT* Cg = reinterpret_cast<const IOT*>(p.C);
  const float bias = p.bias ? p.bias[dc] : 0.f;

  // ---- forward from a zero state, checkpoint at every tile start ----
  const IOT* const fsrc[3] = {reinterpret_cast<const IOT*>(p.x),
                              reinterpret_cast<const IOT*>(p.delta), nullptr};
  float h[N];
#pragma unroll
  for (int n = 0; n < N; ++n) h[n] = 0.f;
  float Q = 0.f;
  float bcr = bc_element<IOT, N>(p, Bg, Bg, b, t0, min(kBT, t1 - t0), N);
  issue_scalars<IOT, 3>(sScal, fsrc, p, b, t0, min(kBT, t1 - t0), d0, pairs);
  cp_async_commit();
  for (int k = 0; k < ntile; ++k) {
    const int tau = t0 + k * kBT;
    const int nt = min(kBT, t1 - tau);
    const int buf = k & 1;
    if (tid < kBT * N) sBC[buf * kBT * N + tid] = bcr;
    if (k + 1 < ntile) {
      const int tn = tau + kBT, ntn = min(kBT, t1 - tn);
      bcr = bc_element<IOT, N>(p, Bg, Bg, b, tn, ntn, N);
      issue_scalars<IOT, 3>(sScal + (buf ^ 1) * kBuf, fsrc, p, b, tn, ntn, d0, pairs);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (valid) {
      const int gt = tau / kBT;
      float* ck = p.ws_ck + ((size_t)b * p.ntiles + gt) * N * dim + dc;
#pragma unroll
      for (int n = 0; n < N; ++n) ck[(size_t)n * dim] = h[n];
      p.ws_qk[((size_t)b * p.ntiles + gt) * dim + dc] = Q;
    }
    const IOT* sx = sScal + buf * kBuf;
    const IOT* sd = sx + kBT * kNT;
    const float* sB = sBC + buf * kBT * N;
#pragma unroll
    for (int j = 0; j < kBT; ++j) {
      if (j < nt) {
        const float xv = IO::load(sx + j * kNT + tid);
        float dt, q, sp;
        step_size<kFast>(IO::load(sd + j * kNT + tid) + bias, p.softplus, dt, q, sp);
        float a[N];
        decays<N, kFast, kStruct>(q, A0, Arow, a);
        const float dtx = dt * xv;
#pragma unroll
        for (int n = 0; n < N; ++n) h[n] = fmaf(a[n], h[n], dtx * sB[j * N + n]);
        Q += q;
      }
    }
    __syncthreads();  // buffer `buf` is refilled next
  }
  cp_async_wait<0>();
  if (valid) {
    const size_t sb = (size_t)b * p.nseg + seg;
    p.ws_qseg[sb * dim + dc] = Q;
    if (seg < p.nseg - 1) {
#pragma unroll
      for (int n = 0; n < N; ++n) p.ws_hloc[(sb * N + n) * dim + dc] = h[n];
    }
  }
  if (seg == 0) return;  // uniform over the CTA

  // ---- the segment's outgoing adjoint from a zero end: mu <- a (C g + mu) ----
  const IOT* const bsrc[3] = {reinterpret_cast<const IOT*>(p.delta),
                              reinterpret_cast<const IOT*>(p.dy),
                              reinterpret_cast<const IOT*>(p.z)};
  const bool has_z = p.z != nullptr;
  float mu[N];
#pragma unroll
  for (int n = 0; n < N; ++n) mu[n] = 0.f;
  {
    const int tau = t0 + (ntile - 1) * kBT;
    bcr = bc_element<IOT, N>(p, Cg, Cg, b, tau, t1 - tau, N);
    issue_scalars<IOT, 3>(sScal, bsrc, p, b, tau, t1 - tau, d0, pairs);
    cp_async_commit();
  }
  for (int k = ntile - 1, it = 0; k >= 0; --k, ++it) {
    const int tau = t0 + k * kBT;
    const int nt = min(kBT, t1 - tau);
    const int buf = it & 1;
    if (tid < kBT * N) sBC[buf * kBT * N + tid] = bcr;
    if (k > 0) {
      const int tn = tau - kBT;
      bcr = bc_element<IOT, N>(p, Cg, Cg, b, tn, kBT, N);
      issue_scalars<IOT, 3>(sScal + (buf ^ 1) * kBuf, bsrc, p, b, tn, kBT, d0, pairs);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const IOT* sd = sScal + buf * kBuf;
    const IOT* sdy = sd + kBT * kNT;
    const IOT* sz = sdy + kBT * kNT;
    const float* sC = sBC + buf * kBT * N;
#pragma unroll
    for (int j = kBT - 1; j >= 0; --j) {
      if (j < nt) {
        float dt, q, sp;
        step_size<kFast>(IO::load(sd + j * kNT + tid) + bias, p.softplus, dt, q, sp);
        float g = IO::load(sdy + j * kNT + tid);
        if (has_z) {
          const float zv = IO::load(sz + j * kNT + tid);
          g *= zv * sigmoid_f<kFast>(zv);
        }
        float a[N];
        decays<N, kFast, kStruct>(q, A0, Arow, a);
#pragma unroll
        for (int n = 0; n < N; ++n) mu[n] = a[n] * fmaf(sC[j * N + n], g, mu[n]);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  if (valid) {
    const size_t sb = (size_t)b * p.nseg + seg;
#pragma unroll
    for (int n = 0; n < N; ++n) p.ws_mloc[(sb * N + n) * dim + dc] = mu[n];
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
    float h = p.h0 ? p.h0[((size_t)b * p.dim + d) * N + n] : 0.f;
    for (int s = 0; s < p.nseg; ++s) {
      const size_t sb = (size_t)b * p.nseg + s;
      const size_t at = (sb * N + n) * p.dim + d;
      p.ws_hin[at] = h;
      if (s < p.nseg - 1) h = fmaf(exp_u<kFast>(p.ws_qseg[sb * p.dim + d] * An), h, p.ws_hloc[at]);
    }
    float mu = p.dh_last ? p.dh_last[((size_t)b * p.dim + d) * N + n] : 0.f;
    for (int s = p.nseg - 1; s >= 0; --s) {
      const size_t sb = (size_t)b * p.nseg + s;
      const size_t at = (sb * N + n) * p.dim + d;
      p.ws_muin[at] = mu;
      if (s > 0) mu = fmaf(exp_u<kFast>(p.ws_qseg[sb * p.dim + d] * An), mu, p.ws_mloc[at]);
    }
  }
}

// ---------------------------------------------------------------------------
// 3. main: tiles of 4 steps in reverse, recomputed into registers.
struct StepIn {
  float x, dt, q, sp, dy, z, g, dtx;
};

template <typename IOT, int N>
__device__ __forceinline__ void issue_main_tile(const BwdParams& p, unsigned char* smem, int buf,
                                                int b, int tau, int nt, int dblk, int dc,
                                                bool valid, float& bcr) {
  using SM = MainSmem<IOT, N>;
  const int tid = threadIdx.x;
  const int dim = p.dim;
  IOT* sScal = reinterpret_cast<IOT*>(smem + SM::kOffScal) + buf * SM::kTen * kBT * kNT;
  const IOT* const src[4] = {reinterpret_cast<const IOT*>(p.x),
                             reinterpret_cast<const IOT*>(p.delta),
                             reinterpret_cast<const IOT*>(p.dy),
                             reinterpret_cast<const IOT*>(p.z)};
  issue_scalars<IOT, 4>(sScal, src, p, b, tau, nt, dblk * kNT, p.scal_pairs != 0);
  // checkpoint of the tile start and its summed exponent
  float* sCk = reinterpret_cast<float*>(smem + SM::kOffCk) + buf * (N + 1) * kNT;
  const int gt = tau / kBT;
  const float* ck = p.ws_ck + ((size_t)b * p.ntiles + gt) * N * dim + dc;
#pragma unroll
  for (int n = 0; n < N; ++n) cp_async4(sCk + n * kNT + tid, ck + (size_t)n * dim, valid ? 4u : 0u);
  cp_async4(sCk + N * kNT + tid, p.ws_qk + ((size_t)b * p.ntiles + gt) * dim + dc, valid ? 4u : 0u);
  bcr = bc_element<IOT, N>(p, reinterpret_cast<const IOT*>(p.B), reinterpret_cast<const IOT*>(p.C),
                           b, tau, nt, 2 * N);
}

template <typename IOT, int N, bool kStruct>
__device__ __forceinline__ void main_body(const BwdParams& p, unsigned char* smem,
                                          const float* Arow, float A0, int b, int seg, int dblk,
                                          int dc, bool valid) {
  using IO = Io<IOT>;
  using SM = MainSmem<IOT, N>;
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  constexpr int V = 2 * N;  // channel-summed values per step: dB_n, dC_n
  float* sRed = reinterpret_cast<float*>(smem + SM::kOffRed);   // [kBT][V][kRedStride]
  float* sHin = reinterpret_cast<float*>(smem + SM::kOffHin);   // [N][kNT]
  const float* sCkAll = reinterpret_cast<const float*>(smem + SM::kOffCk);
  float* sBCAll = reinterpret_cast<float*>(smem + SM::kOffBC);  // [2][kBT][V]
  const IOT* sScalAll = reinterpret_cast<const IOT*>(smem + SM::kOffScal);
  const int tid = threadIdx.x;
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
  float mu[N], dA[N];
#pragma unroll
  for (int n = 0; n < N; ++n) {
    sHin[n * kNT + tid] = p.ws_hin[(sb * N + n) * dim + dc];
    // channels past dim carry a zero adjoint, so they add nothing to dB
    mu[n] = valid ? p.ws_muin[(sb * N + n) * dim + dc] : 0.f;
    dA[n] = 0.f;
  }
  float dD_acc = 0.f, dbias_acc = 0.f;

  float bcr;
  {
    const int tau = t0 + (ntile - 1) * kBT;
    issue_main_tile<IOT, N>(p, smem, 0, b, tau, t1 - tau, dblk, dc, valid, bcr);
    cp_async_commit();
  }
  for (int k = ntile - 1, it = 0; k >= 0; --k, ++it) {
    const int tau = t0 + k * kBT;
    const int nt = min(kBT, t1 - tau);
    const int buf = it & 1;
    if (tid < kBT * V) sBCAll[buf * kBT * V + tid] = bcr;
    if (k > 0) issue_main_tile<IOT, N>(p, smem, buf ^ 1, b, tau - kBT, kBT, dblk, dc, valid, bcr);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();  // tile k staged by every thread; sRed free

    const IOT* sScal = sScalAll + buf * SM::kTen * kBT * kNT;
    const float* sCk = sCkAll + buf * (N + 1) * kNT;
    const float* sB = sBCAll + buf * kBT * V;  // row j: B_j[0..N), C_j[0..N)
    // per-step scalars
    StepIn st[kBT];
#pragma unroll
    for (int j = 0; j < kBT; ++j) {
      const float xv = IO::load(sScal + (0 * kBT + j) * kNT + tid);
      step_size<kFast>(IO::load(sScal + (1 * kBT + j) * kNT + tid) + bias, p.softplus, st[j].dt,
                       st[j].q, st[j].sp);
      st[j].x = xv;
      st[j].dtx = st[j].dt * xv;
      const float dyv = IO::load(sScal + (2 * kBT + j) * kNT + tid);
      st[j].dy = dyv;
      if (has_z) {
        const float zv = IO::load(sScal + (3 * kBT + j) * kNT + tid);
        st[j].z = zv;
        st[j].g = dyv * zv * sigmoid_f<kFast>(zv);
      } else {
        st[j].z = 0.f;
        st[j].g = dyv;
      }
    }
    // the tile's true entry state: checkpoint + exp(A_n Q) h_in
    float he[N];
    {
      float P[N];
      decays<N, kFast, kStruct>(sCk[N * kNT + tid], A0, Arow, P);
#pragma unroll
      for (int n = 0; n < N; ++n) he[n] = fmaf(P[n], sHin[n * kNT + tid], sCk[n * kNT + tid]);
    }
    // recompute the tile's states
    float hist[kBT][N];
#pragma unroll
    for (int j = 0; j < kBT; ++j) {
      float a[N];
      decays<N, kFast, kStruct>(st[j].q, A0, Arow, a);
#pragma unroll
      for (int n = 0; n < N; ++n) {
        const float prev = j == 0 ? he[n] : hist[j - 1][n];
        hist[j][n] = fmaf(a[n], prev, st[j].dtx * sB[j * V + n]);
      }
    }
    // adjoint, backwards through the tile
#pragma unroll
    for (int j = kBT - 1; j >= 0; --j) {
      if (j < nt) {
        const StepIn& s = st[j];
        float a[N];
        decays<N, kFast, kStruct>(s.q, A0, Arow, a);
        float S1 = 0.f, S2 = 0.f, ys = 0.f;
        float* red = sRed + (size_t)j * V * kRedStride + tid;
#pragma unroll
        for (int n = 0; n < N; ++n) {
          const float Bn = sB[j * V + n], Cn = sB[j * V + N + n];
          const float prev = j == 0 ? he[n] : hist[j - 1][n];
          const float lam = fmaf(Cn, s.g, mu[n]);
          S1 = fmaf(lam, Bn, S1);
          const float qv = lam * (a[n] * prev);
          S2 = fmaf(qv, a_coef<N, kStruct>(n, Arow), S2);
          dA[n] = fmaf(qv, s.dt, dA[n]);
          ys = fmaf(Cn, hist[j][n], ys);
          red[n * kRedStride] = lam * s.dtx;
          red[(N + n) * kRedStride] = s.g * hist[j][n];
          mu[n] = a[n] * lam;
        }
        if constexpr (kStruct) S2 *= A0;
        const float dxv = fmaf(Dd, s.g, s.dt * S1);
        const float ddv = fmaf(s.x, S1, S2) * s.sp;
        dD_acc = fmaf(s.g, s.x, dD_acc);
        dbias_acc += ddv;
        if (valid) {
          const size_t i = ((size_t)b * L + tau + j) * dim + dc;
          IO::store(dxg + i, dxv);
          IO::store(ddg + i, ddv);
          if (has_z) {
            const float sg = sigmoid_f<kFast>(s.z);
            const float ssum = fmaf(Dd, s.x, ys);
            IO::store(dzg + i, s.dy * ssum * sg * fmaf(s.z, 1.f - sg, 1.f));
          }
        }
      }
    }
    __syncthreads();  // every channel's values are in sRed
    // sum over the CTA's channels: thread -> (step j, value v)
    if (tid < kBT * V) {
      const int j = tid / V, v = tid % V;
      if (j < nt) {
        const float4* row = reinterpret_cast<const float4*>(sRed + (size_t)(j * V + v) * kRedStride);
        float4 acc = row[0];
#pragma unroll 8
        for (int c = 1; c < kNT / 4; ++c) {
          const float4 w = row[c];
          acc.x += w.x;
          acc.y += w.y;
          acc.z += w.z;
          acc.w += w.w;
        }
        p.ws_dbc[(((size_t)b * p.dblocks + dblk) * L + tau + j) * V + v] =
            (acc.x + acc.y) + (acc.z + acc.w);
      }
    }
  }
  cp_async_wait<0>();
  if (valid) {
    if (seg == 0 && p.dh0) {
#pragma unroll
      for (int n = 0; n < N; ++n) p.dh0[((size_t)b * dim + dc) * N + n] = mu[n];
    }
#pragma unroll
    for (int n = 0; n < N; ++n) p.ws_dA[(sb * N + n) * dim + dc] = dA[n];
    p.ws_dD[sb * dim + dc] = dD_acc;
    p.ws_dbias[sb * dim + dc] = dbias_acc;
  }
}

template <typename IOT, int N>
__global__ void __launch_bounds__(kNT, 2) bwd_main_kernel(const BwdParams p) {
  extern __shared__ float4 smem4[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(smem4);
  const int dblk = blockIdx.x, seg = blockIdx.y, b = blockIdx.z;
  const int d = dblk * kNT + threadIdx.x;
  const bool valid = d < p.dim;
  const int dc = valid ? d : p.dim - 1;
  const float* Arow = p.A + (size_t)dc * N;
  float A0;
  if (cta_structured<N>(Arow, A0)) main_body<IOT, N, true>(p, smem, Arow, A0, b, seg, dblk, dc, valid);
  else main_body<IOT, N, false>(p, smem, Arow, A0, b, seg, dblk, dc, valid);
}

// ---------------------------------------------------------------------------
// 4. reduce: dB, dC over channel blocks; dA, dD, dbias over (batch, segment).
__global__ void __launch_bounds__(256) bwd_reduce_kernel(const BwdParams p, int N) {
  const int V = 2 * N;
  const size_t n_bc = (size_t)p.batch * p.seqlen * V;
  const size_t n_a = (size_t)p.dim * N;
  const size_t total = n_bc + n_a + (size_t)p.dim;
  const size_t bs = (size_t)p.batch * p.nseg;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    if (i < n_bc) {
      const int v = (int)(i % V);
      const size_t bt = i / V;  // b * L + t
      const int t = (int)(bt % p.seqlen);
      const int b = (int)(bt / p.seqlen);
      float acc = 0.f;
      for (int k = 0; k < p.dblocks; ++k)
        acc += p.ws_dbc[(((size_t)b * p.dblocks + k) * p.seqlen + t) * V + v];
      if (v < N) p.dB[bt * N + v] = acc;
      else p.dC[bt * N + (v - N)] = acc;
    } else if (i < n_bc + n_a) {
      const size_t j = i - n_bc;  // d * N + n
      const int n = (int)(j % N);
      const int d = (int)(j / N);
      float acc = 0.f;
      for (size_t s = 0; s < bs; ++s) acc += p.ws_dA[(s * N + n) * p.dim + d];
      p.dA[j] = acc;
    } else {
      const int d = (int)(i - n_bc - n_a);
      float a1 = 0.f, a2 = 0.f;
      for (size_t s = 0; s < bs; ++s) {
        a1 += p.ws_dD[s * p.dim + d];
        a2 += p.ws_dbias[s * p.dim + d];
      }
      if (p.dD) p.dD[d] = a1;
      if (p.dbias) p.dbias[d] = a2;
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
  bwd_main_kernel<IOT, N><<<grid, kNT, main_bytes, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t red = (size_t)p.batch * p.seqlen * 2 * N + (size_t)p.dim * N + p.dim;
  bwd_reduce_kernel<<<grid_for(red, 256), 256, 0, stream>>>(p, N);
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
