// ssm_ssd_decode.cu -- sm_100a kernel of one decode step of the multi-head SSD.
//
// Page "Mamba 논문 리뷰: Selective State Space Models로 Transformer를 넘어서"
// (youngju.dev), §4.1: the recurrent side of the duality (the state update
// that gives O(1) work per generated token). Per batch b, head h, row p of the
// head's state (fp32, carried between calls):
//   Delta = softplus(dt[b,h] + dt_bias[h]),  a = exp(Delta A[h])
//   S[n]  = a S[n] + Delta B[b,n] x[b,h,p],  y[b,h,p] = sum_n C[b,n] S[n] + D[h] x[b,h,p]
// A warp takes kRows state rows (N fp32 each = N/32 per lane, vector loads and
// stores), y reduced by shuffles. Bound by the state's read and write.
#include "ssm_device.cuh"
#include "ssm_ssd_decode_internal.h"

namespace ssm {

namespace {

template <typename IOT, int K>
struct VecLoad;  // K consecutive values as floats
template <typename IOT>
struct VecLoad<IOT, 1> {
  __device__ static void run(const IOT* p, float* v) { v[0] = Io<IOT>::load(p); }
};
template <typename IOT>
struct VecLoad<IOT, 2> {
  __device__ static void run(const IOT* p, float* v) {
    const float2 u = Io<IOT>::load2(p);
    v[0] = u.x; v[1] = u.y;
  }
};
template <typename IOT>
struct VecLoad<IOT, 4> {
  __device__ static void run(const IOT* p, float* v) {
    const float4 u = Io<IOT>::load4(p);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
};
template <typename IOT>
struct VecLoad<IOT, 8> {
  __device__ static void run(const IOT* p, float* v) {
    VecLoad<IOT, 4>::run(p, v);
    VecLoad<IOT, 4>::run(p + 4, v + 4);
  }
};

template <int K>
__device__ __forceinline__ void store_state(float* p, const float* v) {
  if constexpr (K == 1) {
    p[0] = v[0];
  } else if constexpr (K == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  } else {
#pragma unroll
    for (int i = 0; i < K; i += 4)
      *reinterpret_cast<float4*>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
  }
}

#ifndef SSM_SSD_DECODE_ROWS
#define SSM_SSD_DECODE_ROWS 1
#endif
// State rows per warp: all their loads are issued before any arithmetic, so a
// warp keeps kRows x 512 B (N = 128) of state reads in flight. Measured on the
// 64 x 64-head, d_state 128 layer: 1 and 2 rows tie (67.7 us), 4 rows are
// slower (77.6 us).
constexpr int kRows = SSM_SSD_DECODE_ROWS;

template <typename IOT, int N>
__global__ void __launch_bounds__(256) ssd_decode_kernel(const SsdDecodeParams p) {
  using IO = Io<IOT>;
  constexpr int SPT = N / 32;
  // bf16 io takes the MUFU approximations (as the other kernels), fp32 io expf / log1pf
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  // row indices fit 32 bits (the entry point admits at most 2^26 rows): the
  // (b, h) of a row comes from 32-bit divisions, far cheaper than 64-bit ones
  const uint32_t warp_id = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t P = (uint32_t)p.headdim, H = (uint32_t)p.nheads;
  const uint32_t rows = (uint32_t)p.batch * H * P;
  const uint32_t row0 = warp_id * kRows;
  if (row0 >= rows) return;  // warp-uniform

  // ---- every load of every row first (rows past the end repeat the last one)
  float s[kRows][SPT], bb[kRows][SPT], cv[kRows][SPT], xv[kRows], raw[kRows], bias[kRows],
      Ah[kRows], Dh[kRows];
  uint32_t rr[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    rr[r] = row0 + r < rows ? row0 + r : rows - 1;
    const uint32_t bh = rr[r] / P;
    const int h = (int)(bh % H);
    const size_t b = bh / H;
    VecLoad<float, SPT>::run(p.state + (size_t)rr[r] * N + lane * SPT, s[r]);
    VecLoad<IOT, SPT>::run(static_cast<const IOT*>(p.B) + b * N + lane * SPT, bb[r]);
    VecLoad<IOT, SPT>::run(static_cast<const IOT*>(p.C) + b * N + lane * SPT, cv[r]);
    xv[r] = IO::load(static_cast<const IOT*>(p.x) + rr[r]);
    raw[r] = IO::load(static_cast<const IOT*>(p.dt) + bh);
    bias[r] = p.dt_bias ? p.dt_bias[h] : 0.f;
    Ah[r] = p.A[h];
    Dh[r] = p.D ? p.D[h] : 0.f;
  }

  // ---- the step, row by row
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const float v = raw[r] + bias[r];
    float d = v;
    if (p.softplus && v <= kSoftplusCut)
      d = kFast ? kLn2 * lg2_approx(1.f + ex2_approx(v * kLog2e)) : log1pf(expf(v));
    const float a = kFast ? ex2_approx(d * Ah[r] * kLog2e) : expf(d * Ah[r]);
    const float dx = d * xv[r];
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < SPT; ++i) {
      s[r][i] = fmaf(a, s[r][i], dx * bb[r][i]);
      acc = fmaf(cv[r][i], s[r][i], acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (row0 + r < rows) {
      store_state<SPT>(p.state + (size_t)rr[r] * N + lane * SPT, s[r]);
      if (lane == 0) IO::store(static_cast<IOT*>(p.y) + rr[r], fmaf(Dh[r], xv[r], acc));
    }
  }
}

template <typename IOT>
cudaError_t launch_io(const SsdDecodeParams& p, cudaStream_t stream) {
  const size_t rows = (size_t)p.batch * p.nheads * p.headdim;
  const size_t threads = (rows + kRows - 1) / kRows * 32;
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  switch (p.dstate) {
    case 32: ssd_decode_kernel<IOT, 32><<<blocks, 256, 0, stream>>>(p); break;
    case 64: ssd_decode_kernel<IOT, 64><<<blocks, 256, 0, stream>>>(p); break;
    case 128: ssd_decode_kernel<IOT, 128><<<blocks, 256, 0, stream>>>(p); break;
    case 256: ssd_decode_kernel<IOT, 256><<<blocks, 256, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

bool ssd_decode_dstate_supported(int dstate) {
  return dstate == 32 || dstate == 64 || dstate == 128 || dstate == 256;
}

cudaError_t launch_ssd_decode(const SsdDecodeParams& p, bool bf16, cudaStream_t stream) {
  return bf16 ? launch_io<uint16_t>(p, stream) : launch_io<float>(p, stream);
}

}  // namespace ssm
