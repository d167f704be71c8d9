// ssm_seqpar.cu -- sm_100a kernels for splitting one sequence across ranks.
//
// The scan's recurrence h <- exp(Delta A_n) h + u (page "Mamba 논문 리뷰",
// §2.2; §3.3 selective_scan) is an affine map per step, and affine maps
// compose associatively (page "맘바(Mamba)와 상태공간모델(SSM) 쉽게
// 이해하기", allinfo.ai.kr: the parallel associative scan). A contiguous
// chunk of steps therefore acts on the state as h -> P h + e with
// P_n = exp(A_n sum_t Delta_t) and e = the chunk's end state from a zero
// start. A rank holding chunk r needs only the (P, e) of chunks 0..r-1 to
// know its true entering state; these kernels compute the sum of Delta of a
// chunk and compose gathered carries.
#include <algorithm>

#include "ssm_device.cuh"
#include "ssm_seqpar_internal.h"

namespace ssm {

namespace {

// sum_t Delta_t per (b, d): Delta = softplus(delta + bias) (or delta + bias).
// One thread per (b, d), coalesced over d; fp64-free, fp32 sequential sum.
template <typename IOT>
__global__ void __launch_bounds__(256) delta_sum_kernel(const SeqParParams p) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)p.batch * p.dim) return;
  const int d = (int)(i % p.dim);
  const size_t b = i / p.dim;
  const IOT* dl = reinterpret_cast<const IOT*>(p.delta) + b * (size_t)p.seqlen * p.dim + d;
  const float bias = p.bias ? p.bias[d] : 0.f;
  float acc = 0.f;
  for (int t = 0; t < p.seqlen; ++t) {
    const float v = Io<IOT>::load(dl + (size_t)t * p.dim) + bias;
    float dt;
    if (!p.softplus || v > kSoftplusCut) {
      dt = v;
    } else if constexpr (sizeof(IOT) == 2) {
      dt = kLn2 * lg2_approx(1.f + ex2_approx(v * kLog2e));
    } else {
      dt = log1pf(expf(v));
    }
    acc += dt;
  }
  p.dsum[i] = acc;
}

// h_in[b,d,n] = compose over chunks 0..rank-1 of (exp(A_n S_r), e_r) applied
// to h0 (or 0): h <- exp(A_n S_r) h + e_r in chunk order.
__global__ void __launch_bounds__(256) compose_kernel(const SeqParParams p) {
  const size_t total = (size_t)p.batch * p.dim * p.dstate;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int n = (int)(i % p.dstate);
    const size_t bd = i / p.dstate;  // b * dim + d
    const int d = (int)(bd % p.dim);
    const float An = p.A[(size_t)d * p.dstate + n];
    float h = p.h0 ? p.h0[i] : 0.f;
    for (int r = 0; r < p.rank; ++r) {
      const size_t off = (size_t)r * total;
      h = fmaf(expf(An * p.dsum_all[(size_t)r * p.batch * p.dim + bd]), h, p.hend_all[off + i]);
    }
    p.h_in[i] = h;
  }
}

}  // namespace

cudaError_t launch_delta_sum(const SeqParParams& p, bool bf16, cudaStream_t stream) {
  const size_t n = (size_t)p.batch * p.dim;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (bf16) delta_sum_kernel<uint16_t><<<blocks, 256, 0, stream>>>(p);
  else delta_sum_kernel<float><<<blocks, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_compose(const SeqParParams& p, cudaStream_t stream) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  const size_t n = (size_t)p.batch * p.dim * p.dstate;
  const unsigned blocks = (unsigned)std::max<size_t>(1, std::min<size_t>((n + 255) / 256, (size_t)sms * 8));
  compose_kernel<<<blocks, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace ssm
