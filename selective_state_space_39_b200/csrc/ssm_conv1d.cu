// ssm_conv1d.cu -- sm_100a kernels of the Mamba block's causal depthwise
// convolution with SiLU, and its backward.
//
// What is computed (page "Mamba 논문 리뷰: Selective State Space Models로
// Transformer를 넘어서", youngju.dev, §3.4 Mamba Block: nn.Conv1d(d_inner,
// d_inner, d_conv, padding=d_conv-1, groups=d_inner) cut to the first L
// outputs, then SiLU), per batch row b, step t, channel d, taps k < W:
//
//   u[b,t,d]   = bias[d] + sum_k w[d,k] x[b, t-(W-1)+k, d]   (zero before t = 0)
//   out[b,t,d] = SiLU(u)  (or u)
//
// and for the loss sum dout * out:
//
//   du[t] = dout[t] SiLU'(u[t]),  dx[s] = sum_k w[d,k] du[s+(W-1)-k],
//   dw[d,k] = sum_(b,t) du[t] x[t-(W-1)+k],  dbias[d] = sum_(b,t) du[t].
//
// Design (B200): both directions are HBM-bound elementwise streams (a few
// FLOPs per element), so the kernels are built for bandwidth: each thread owns
// VEC adjacent channels (vector loads and stores: 4 bf16 or 2 fp32 channels in
// 8 bytes; 2 bf16 in 4 bytes in the bf16 backward) and a chunk of T steps, keeps the W-1 previous rows in registers (a sliding
// window: every input element is read once, plus a W-1 row halo per chunk),
// and issues the loads of several steps before using them. Warps cover
// contiguous channel runs of a row, so every access is coalesced. The weight
// gradients are summed per (batch row, chunk) and reduced by a second kernel
// in a fixed order (deterministic results).
#include <string.h>

#include <algorithm>
#include <type_traits>

#include "ssm_conv_internal.h"
#include "ssm_device.cuh"

namespace ssm {

namespace {

constexpr int kMaxThreads = 192;  // CTA size cap: two or more CTAs per SM
constexpr int kUnroll = 8;     // forward: steps whose loads are in flight together
constexpr int kUnrollBwd = 4;  // backward: the same (two tensors per step)
#ifndef SSM_CONV_BWD_VEC_BF16
#define SSM_CONV_BWD_VEC_BF16 2
#endif
// bf16 channels per thread in the backward (4: 8-byte vectors, 2: 4-byte).
// Two measured faster on the 8 x 2048 x 1536 layer (74.7 vs 78.8 us): 64
// registers instead of 149, five CTAs per SM instead of two.
constexpr int kConvBwdVecBf16 = SSM_CONV_BWD_VEC_BF16;

template <bool kFast>
__device__ __forceinline__ float sigmoid_c(float u) {
  if constexpr (kFast) return fmaf(0.5f, tanh_approx(0.5f * u), 0.5f);
  else return 1.f / (1.f + expf(-u));
}

// VEC io elements <-> fp32.
template <typename IOT, int VEC>
struct Vec;

template <>
struct Vec<uint16_t, 4> {
  using Raw = uint2;
  __device__ static __forceinline__ void unpack(const Raw& r, float (&f)[4]) {
    f[0] = bf16_lo(r.x); f[1] = bf16_hi(r.x); f[2] = bf16_lo(r.y); f[3] = bf16_hi(r.y);
  }
  __device__ static __forceinline__ Raw pack(const float (&f)[4]) {
    return make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
  }
};

template <>
struct Vec<uint16_t, 2> {
  using Raw = uint32_t;
  __device__ static __forceinline__ void unpack(const Raw& r, float (&f)[2]) {
    f[0] = bf16_lo(r); f[1] = bf16_hi(r);
  }
  __device__ static __forceinline__ Raw pack(const float (&f)[2]) { return pack_bf16x2(f[0], f[1]); }
};

template <>
struct Vec<float, 2> {
  using Raw = float2;
  __device__ static __forceinline__ void unpack(const Raw& r, float (&f)[2]) {
    f[0] = r.x; f[1] = r.y;
  }
  __device__ static __forceinline__ Raw pack(const float (&f)[2]) { return make_float2(f[0], f[1]); }
};

template <typename IOT>
struct Vec<IOT, 1> {
  using Raw = IOT;
  __device__ static __forceinline__ void unpack(const Raw& r, float (&f)[1]) {
    f[0] = Io<IOT>::load(&r);
  }
  __device__ static __forceinline__ Raw pack(const float (&f)[1]) {
    Raw r;
    Io<IOT>::store(&r, f[0]);
    return r;
  }
};

// Row t of this thread's channels as stored (all-zero bits outside [0, L)),
// kept packed until used so that several rows can be in flight.
template <typename IOT, int VEC>
__device__ __forceinline__ typename Vec<IOT, VEC>::Raw load_raw(const IOT* base, int t, int L,
                                                                int dim, int d0, size_t row0) {
  using Raw = typename Vec<IOT, VEC>::Raw;
  if (t < 0 || t >= L) {
    Raw z;
    memset(&z, 0, sizeof z);
    return z;
  }
  return *reinterpret_cast<const Raw*>(base + (row0 + (size_t)t) * dim + d0);
}

template <typename IOT, int VEC>
__device__ __forceinline__ void load_row(const IOT* base, int t, int L, int dim, int d0,
                                         size_t row0, float (&f)[VEC]) {
  Vec<IOT, VEC>::unpack(load_raw<IOT, VEC>(base, t, L, dim, d0, row0), f);
}

template <typename IOT, int VEC>
__device__ __forceinline__ void store_row(IOT* base, int t, int L, int dim, int d0, size_t row0,
                                          const float (&f)[VEC]) {
  using V = Vec<IOT, VEC>;
  if (t >= L || d0 >= dim) return;
  *reinterpret_cast<typename V::Raw*>(base + (row0 + (size_t)t) * dim + d0) = V::pack(f);
}

// Taps and bias of this thread's VEC channels (one 16-byte load per channel
// when W == 4; the caller checks that w is 16-byte aligned).
template <int VEC, int W>
__device__ __forceinline__ void load_taps(const ConvParams& p, int d0, float (&w)[VEC][W],
                                          float (&bias)[VEC]) {
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    if constexpr (W == 4) {
      if (p.w_vec) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(p.w) + (d0 + i));
        w[i][0] = t.x; w[i][1] = t.y; w[i][2] = t.z; w[i][3] = t.w;
      } else {
#pragma unroll
        for (int k = 0; k < W; ++k) w[i][k] = __ldg(p.w + (size_t)(d0 + i) * W + k);
      }
    } else {
#pragma unroll
      for (int k = 0; k < W; ++k) w[i][k] = __ldg(p.w + (size_t)(d0 + i) * W + k);
    }
    bias[i] = p.bias ? __ldg(p.bias + d0 + i) : 0.f;
  }
}

// ---------------------------------------------------------------------------
// forward
template <typename IOT, int VEC, int W>
__global__ void __launch_bounds__(kMaxThreads) conv_fwd_kernel(const ConvParams p) {
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  const int d0 = (blockIdx.x * blockDim.x + threadIdx.x) * VEC;
  const int t0 = blockIdx.y * p.chunk;
  const int b = blockIdx.z;
  const int L = p.seqlen, dim = p.dim;
  if (d0 >= dim) return;
  const IOT* x = reinterpret_cast<const IOT*>(p.x);
  IOT* out = reinterpret_cast<IOT*>(p.out);
  const size_t row0 = (size_t)b * L;
  float w[VEC][W], bias[VEC];
  load_taps<VEC, W>(p, d0, w, bias);
  // sliding window: win[k] = x row t-(W-1)+k for k < W-1
  float win[W - 1][VEC];
#pragma unroll
  for (int k = 0; k < W - 1; ++k) load_row<IOT, VEC>(x, t0 - (W - 1) + k, L, dim, d0, row0, win[k]);
  const int t1 = min(L, t0 + p.chunk);
  // rows of the next group are loaded before the current group is computed
  typename Vec<IOT, VEC>::Raw nxt[kUnroll];
#pragma unroll
  for (int j = 0; j < kUnroll; ++j) nxt[j] = load_raw<IOT, VEC>(x, t0 + j, t1, dim, d0, row0);
  for (int tb = t0; tb < t1; tb += kUnroll) {
    typename Vec<IOT, VEC>::Raw raw[kUnroll];
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      raw[j] = nxt[j];
      nxt[j] = load_raw<IOT, VEC>(x, tb + kUnroll + j, t1, dim, d0, row0);
    }
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      float cur[1][VEC];
      Vec<IOT, VEC>::unpack(raw[j], cur[0]);
      float o[VEC];
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        float u = bias[i];
#pragma unroll
        for (int k = 0; k < W - 1; ++k) u = fmaf(w[i][k], win[k][i], u);
        u = fmaf(w[i][W - 1], cur[0][i], u);
        o[i] = p.silu ? u * sigmoid_c<kFast>(u) : u;
      }
      store_row<IOT, VEC>(out, tb + j, t1, dim, d0, row0, o);
#pragma unroll
      for (int k = 0; k < W - 2; ++k)
#pragma unroll
        for (int i = 0; i < VEC; ++i) win[k][i] = win[k + 1][i];
#pragma unroll
      for (int i = 0; i < VEC; ++i) win[W - 2][i] = cur[0][i];
    }
  }
}

// ---------------------------------------------------------------------------
// backward: dx for the chunk's steps, per-(row, chunk) partial dw and dbias.
template <typename IOT, int VEC, int W>
__global__ void __launch_bounds__(kMaxThreads) conv_bwd_kernel(const ConvParams p) {
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  const int d0 = (blockIdx.x * blockDim.x + threadIdx.x) * VEC;
  const int chunk = blockIdx.y;
  const int t0 = chunk * p.chunk;
  const int b = blockIdx.z;
  const int L = p.seqlen, dim = p.dim;
  if (d0 >= dim) return;
  const IOT* x = reinterpret_cast<const IOT*>(p.x);
  const IOT* dout = reinterpret_cast<const IOT*>(p.dout);
  IOT* dx = reinterpret_cast<IOT*>(p.dx);
  const size_t row0 = (size_t)b * L;
  float w[VEC][W], bias[VEC], dw[VEC][W], db[VEC];
  load_taps<VEC, W>(p, d0, w, bias);
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
#pragma unroll
    for (int k = 0; k < W; ++k) dw[i][k] = 0.f;
    db[i] = 0.f;
  }
  const int t1 = min(L, t0 + p.chunk);
  // x window (the W-1 rows before t) and du window (du of the W-1 rows
  // after s = t-(W-1), i.e. du[t-(W-1)+1 .. t-1] once t has been reached)
  float xwin[W - 1][VEC], duwin[W - 1][VEC];
#pragma unroll
  for (int k = 0; k < W - 1; ++k) {
    load_row<IOT, VEC>(x, t0 - (W - 1) + k, L, dim, d0, row0, xwin[k]);
#pragma unroll
    for (int i = 0; i < VEC; ++i) duwin[k][i] = 0.f;
  }
  // t runs over [t0, t1 + W - 1): du[t] for the chunk and the W-1 rows after
  // it (needed by dx of the chunk's last rows); dx[s] for s = t - (W-1) >= t0.
  const int tend = t1 + (W - 1);
  const int tlim = min(L, tend);
  // rows of the next group are loaded before the current group is computed
  typename Vec<IOT, VEC>::Raw xn[kUnrollBwd], gn[kUnrollBwd];
#pragma unroll
  for (int j = 0; j < kUnrollBwd; ++j) {
    xn[j] = load_raw<IOT, VEC>(x, t0 + j, tlim, dim, d0, row0);
    gn[j] = load_raw<IOT, VEC>(dout, t0 + j, tlim, dim, d0, row0);
  }
  for (int tb = t0; tb < tend; tb += kUnrollBwd) {
    typename Vec<IOT, VEC>::Raw xr[kUnrollBwd], gr[kUnrollBwd];
#pragma unroll
    for (int j = 0; j < kUnrollBwd; ++j) {
      xr[j] = xn[j];
      gr[j] = gn[j];
      xn[j] = load_raw<IOT, VEC>(x, tb + kUnrollBwd + j, tlim, dim, d0, row0);
      gn[j] = load_raw<IOT, VEC>(dout, tb + kUnrollBwd + j, tlim, dim, d0, row0);
    }
#pragma unroll
    for (int j = 0; j < kUnrollBwd; ++j) {
      const int t = tb + j;
      if (t >= tend) break;
      float xcj[VEC], gcj[VEC];
      Vec<IOT, VEC>::unpack(xr[j], xcj);
      Vec<IOT, VEC>::unpack(gr[j], gcj);
      float du[VEC];
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        float u = bias[i];
#pragma unroll
        for (int k = 0; k < W - 1; ++k) u = fmaf(w[i][k], xwin[k][i], u);
        u = fmaf(w[i][W - 1], xcj[i], u);
        float g = gcj[i];  // zero for t >= L
        if (p.silu) {
          const float sg = sigmoid_c<kFast>(u);
          g *= sg * fmaf(u, 1.f - sg, 1.f);
        }
        du[i] = g;
      }
      if (t < t1) {  // this chunk's steps: weight gradients
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
#pragma unroll
          for (int k = 0; k < W - 1; ++k) dw[i][k] = fmaf(du[i], xwin[k][i], dw[i][k]);
          dw[i][W - 1] = fmaf(du[i], xcj[i], dw[i][W - 1]);
          db[i] += du[i];
        }
      }
      const int s = t - (W - 1);
      if (s >= t0 && s < t1) {
        // dx[s] = sum_k w_k du[s + (W-1) - k]: du[t] is tap 0, duwin[W-2-k'] ...
        float o[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
          float a = w[i][0] * du[i];
#pragma unroll
          for (int k = 1; k < W; ++k) a = fmaf(w[i][k], duwin[W - 1 - k][i], a);
          o[i] = a;
        }
        store_row<IOT, VEC>(dx, s, t1, dim, d0, row0, o);
      }
#pragma unroll
      for (int k = 0; k < W - 2; ++k)
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
          xwin[k][i] = xwin[k + 1][i];
          duwin[k][i] = duwin[k + 1][i];
        }
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        xwin[W - 2][i] = xcj[i];
        duwin[W - 2][i] = du[i];
      }
    }
  }
  // partial sums of this (batch row, chunk)
  const size_t part = (size_t)b * gridDim.y + chunk;
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    if (d0 + i >= dim) break;
#pragma unroll
    for (int k = 0; k < W; ++k) p.ws_dw[(part * dim + d0 + i) * W + k] = dw[i][k];
    p.ws_db[part * dim + d0 + i] = db[i];
  }
}

// dw, dbias: sums of the partials over (batch row, chunk), in order.
__global__ void __launch_bounds__(256) conv_reduce_kernel(const ConvParams p, int W, int parts) {
  const int n = p.dim * (W + 1);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    float acc = 0.f;
    if (i < p.dim * W) {
      for (int q = 0; q < parts; ++q) acc += p.ws_dw[(size_t)q * p.dim * W + i];
      if (p.dw) p.dw[i] = acc;
    } else {
      const int d = i - p.dim * W;
      for (int q = 0; q < parts; ++q) acc += p.ws_db[(size_t)q * p.dim + d];
      if (p.dbias) p.dbias[d] = acc;
    }
  }
}

// One decode step per (b, d): out = SiLU(bias + sum_k w_k state_k + w_(W-1) x),
// then the rolling state (the last W-1 inputs, oldest first, in the io type)
// drops its oldest entry and appends x.
template <typename IOT, int W>
__global__ void __launch_bounds__(256) conv_update_kernel(const ConvParams p) {
  using IO = Io<IOT>;
  constexpr bool kFast = std::is_same<IOT, uint16_t>::value;
  // grid: x over the channels, y over the batch rows (no division per thread)
  const int d = blockIdx.x * blockDim.x + threadIdx.x;
  if (d >= p.dim) return;
  const size_t i = (size_t)blockIdx.y * p.dim + d;
  IOT* st = reinterpret_cast<IOT*>(p.out) + i * (W - 1);  // the state (in/out)
  float sv[W - 1];
#pragma unroll
  for (int k = 0; k < W - 1; ++k) sv[k] = IO::load(st + k);
  const float xv = IO::load(reinterpret_cast<const IOT*>(p.x) + i);
  float u = p.bias ? __ldg(p.bias + d) : 0.f;
#pragma unroll
  for (int k = 0; k < W - 1; ++k) u = fmaf(__ldg(p.w + (size_t)d * W + k), sv[k], u);
  u = fmaf(__ldg(p.w + (size_t)d * W + W - 1), xv, u);
  IO::store(reinterpret_cast<IOT*>(p.dx) + i, p.silu ? u * sigmoid_c<kFast>(u) : u);
#pragma unroll
  for (int k = 0; k + 1 < W - 1; ++k) IO::store(st + k, sv[k + 1]);
  IO::store(st + (W - 2), xv);
}

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  return sms;
}

// Threads per CTA along the channels (never above kMaxThreads, the launch
// bound the kernels are compiled for): a whole row when it fits, so that a
// CTA streams one contiguous block of rows; otherwise the largest multiple of
// 32 up to kMaxThreads that divides the row, else kMaxThreads.
int conv_block(int threads_per_row) {
  const int whole = (threads_per_row + 31) / 32 * 32;
  if (whole <= kMaxThreads) return whole;
  for (int nt = kMaxThreads; nt >= 64; nt -= 32)
    if (threads_per_row % nt == 0) return nt;
  return kMaxThreads;
}

template <typename IOT, int VEC, int W>
cudaError_t launch_t(const ConvParams& p, bool backward, cudaStream_t stream) {
  const int per_row = (p.dim + VEC - 1) / VEC;
  const int nt = conv_block(per_row);
  const dim3 grid((unsigned)((per_row + nt - 1) / nt),
                  (unsigned)((p.seqlen + p.chunk - 1) / p.chunk), (unsigned)p.batch);
  if (!backward) {
    conv_fwd_kernel<IOT, VEC, W><<<grid, nt, 0, stream>>>(p);
    return cudaGetLastError();
  }
  conv_bwd_kernel<IOT, VEC, W><<<grid, nt, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n = p.dim * (W + 1);
  const int blocks = std::max(1, std::min((n + 255) / 256, sm_count() * 4));
  conv_reduce_kernel<<<blocks, 256, 0, stream>>>(p, W, (int)(grid.y * grid.z));
  return cudaGetLastError();
}

template <typename IOT, int VEC>
cudaError_t launch_w(const ConvParams& p, bool backward, cudaStream_t stream) {
  switch (p.width) {
    case 2: return launch_t<IOT, VEC, 2>(p, backward, stream);
    case 3: return launch_t<IOT, VEC, 3>(p, backward, stream);
    case 4: return launch_t<IOT, VEC, 4>(p, backward, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename IOT>
cudaError_t launch_update_io(const ConvParams& p, cudaStream_t stream) {
  const dim3 blocks((unsigned)((p.dim + 255) / 256), (unsigned)p.batch);
  switch (p.width) {
    case 2: conv_update_kernel<IOT, 2><<<blocks, 256, 0, stream>>>(p); break;
    case 3: conv_update_kernel<IOT, 3><<<blocks, 256, 0, stream>>>(p); break;
    case 4: conv_update_kernel<IOT, 4><<<blocks, 256, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_conv_update(const ConvParams& p, bool bf16, cudaStream_t stream) {
  return bf16 ? launch_update_io<uint16_t>(p, stream) : launch_update_io<float>(p, stream);
}

bool conv_width_supported(int width) { return width >= 2 && width <= 4; }

cudaError_t launch_conv(const ConvParams& p, bool bf16, bool vec, bool backward,
                        cudaStream_t stream) {
  // Vector paths: 8-byte vectors (4 bf16 or 2 fp32 channels per thread), and
  // for the bf16 backward 4-byte vectors (2 channels), whose 64 registers let
  // five CTAs share an SM
  if (bf16) {
    if (!vec) return launch_w<uint16_t, 1>(p, backward, stream);
    return backward ? launch_w<uint16_t, kConvBwdVecBf16>(p, true, stream)
                    : launch_w<uint16_t, 4>(p, false, stream);
  }
  return vec ? launch_w<float, 2>(p, backward, stream) : launch_w<float, 1>(p, backward, stream);
}

}  // namespace ssm
