// ssm_ssd_decode.cu -- sm_100a kernel of one decode step of the multi-head SSD.
//
// Page "Mamba 논문 리뷰: Selective State Space Models로 Transformer를 넘어서"
// (youngju.dev), §4.1: the recurrent side of the duality (the state update
// that gives O(1) work per generated token). Per batch b, head h, row p of the
// head's state (fp32, carried between calls):
//   Delta = softplus(dt[b,h] + dt_bias[h]),  a = exp(Delta A[h])
//   S[n]  = a S[n] + Delta B[b,n] x[b,h,p],  y[b,h,p] = sum_n C[b,n] S[n] + D[h] x[b,h,p]
// One warp per state row (N fp32 = N/32 per lane, one vector load and store
// each), y reduced by shuffles. Bound by the state's read and write.
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

template <typename IOT, int N>
__global__ void __launch_bounds__(256) ssd_decode_kernel(const SsdDecodeParams p) {
  using IO = Io<IOT>;
  constexpr int SPT = N / 32;
  const size_t row = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // (b H + h) P + p
  const int lane = threadIdx.x & 31;
  if (row >= (size_t)p.batch * p.nheads * p.headdim) return;  // warp-uniform
  const size_t bh = row / p.headdim;
  const int h = (int)(bh % p.nheads);
  const size_t b = bh / p.nheads;

  // ---- every load first
  float* sp = p.state + row * N + lane * SPT;
  float s[SPT], bb[SPT], cv[SPT];
  VecLoad<float, SPT>::run(sp, s);
  VecLoad<IOT, SPT>::run(static_cast<const IOT*>(p.B) + b * N + lane * SPT, bb);
  VecLoad<IOT, SPT>::run(static_cast<const IOT*>(p.C) + b * N + lane * SPT, cv);
  const float xv = IO::load(static_cast<const IOT*>(p.x) + row);
  const float raw = IO::load(static_cast<const IOT*>(p.dt) + bh);
  const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
  const float Ah = p.A[h];
  const float Dh = p.D ? p.D[h] : 0.f;

  // ---- the step
  const float v = raw + bias;
  const float d = p.softplus ? (v > kSoftplusCut ? v : log1pf(expf(v))) : v;
  const float a = expf(d * Ah);
  const float dx = d * xv;
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < SPT; ++i) {
    s[i] = fmaf(a, s[i], dx * bb[i]);
    acc = fmaf(cv[i], s[i], acc);
  }
  store_state<SPT>(sp, s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) IO::store(static_cast<IOT*>(p.y) + row, fmaf(Dh, xv, acc));
}

template <typename IOT>
cudaError_t launch_io(const SsdDecodeParams& p, cudaStream_t stream) {
  const size_t threads = (size_t)p.batch * p.nheads * p.headdim * 32;
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
