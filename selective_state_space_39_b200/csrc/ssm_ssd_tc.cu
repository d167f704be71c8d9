// ssm_ssd_tc.cu -- the multi-head SSD scan (Mamba-2) on the fifth-generation
// tensor cores (tcgen05), with the head state in tensor memory.
//
// Page "Mamba 논문 리뷰: Selective State Space Models로 Transformer를 넘어서"
// (youngju.dev), §4.1 State Space Duality and §4.2. Head h (width P = 64) has
// one scalar A[h] and one step Delta_t = softplus(dt[b,t,h] + dt_bias[h]); B_t
// and C_t (N wide) are shared by the heads; a_t = exp(Delta_t A[h]). Over a
// chunk of Q = 128 steps, with cum_t = sum_{r<=t} Delta_r A[h] inside the
// chunk and H the N x P state entering it (§4.1's semi-separable matrix,
// split into its diagonal block and the part carried by the state):
//
//   S       = C B^T                                     (shared by the heads)
//   G[t][s] = S[t][s] e^{cum_t - cum_s} Delta_s  (s <= t, else 0)
//   y_t     = sum_s G[t][s] x_s + e^{cum_t} C_t H + D x_t
//   H      <- e^{cum_end} H + sum_s w_s x_s B_s^T,   w_s = e^{cum_end - cum_s} Delta_s
//
// Design (B200). One CTA (128 threads, one per TMEM lane) per batch row and
// pair of heads walks the chunks in order. Every product is one tcgen05 MMA
// of M = 128 (bf16 operands from shared memory, fp32 accumulators in TMEM):
// S (t x s, K = N), the readout C H^T (t x (2 heads x p), K = N), the
// state update (2 heads x p) x n with K = s, and G X per head (t x p, K = s).
// The state (2 x 64 rows, N columns) never leaves TMEM: each chunk one pass
// of the threads reads it, keeps a bf16 copy in shared memory for the
// readout, and writes it back scaled by e^{cum_end} before the update MMA
// accumulates onto it. x, B and C chunks arrive by TMA with the 128-byte
// swizzle the MMA descriptors describe (no multicast); the next chunk's B, C
// and x are loaded as soon as the current chunk's MMAs have released their
// buffers (two x buffers alternate between the raw x and the w-scaled x).
// Steps past the sequence end read zeros and take Delta = 0, so they change
// nothing. Every wait is bounded; a wait that runs out stops the CTA (after
// its copies and MMAs in flight land, bounded too), frees its TMEM and sets
// the status word that ssm_ssd_scan_status reports.
#include <stdlib.h>

#include <mutex>
#include <set>
#include <utility>

#include "ssm_device.cuh"
#include "ssm_ssd_internal.h"
#include "ssm_tc.cuh"

namespace ssm {

// Set to 1 by a CTA of the tensor-core SSD kernel whose bounded wait ran out.
__device__ int g_ssd_status = 0;

namespace {

constexpr int kTQ = 128;        // steps per chunk
constexpr int kTP = 64;         // head width
constexpr int kTHeads = 2;      // heads per CTA
constexpr int kTThreads = 128;  // one thread per TMEM lane
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColH = 0, kColS = 128, kColYd = 256, kColYo = 384;

constexpr int round_up(int v, int m) { return (v + m - 1) / m * m; }

template <int N>
struct TcLayout {
  static constexpr int kNB = N / 64;                     // 64-wide blocks of the state
  static constexpr int kBlk = kTQ * 128;                 // one [128 rows][64] bf16 tile
  static constexpr int kXBuf = kTHeads * kBlk;           // [head][t][64 p]
  static constexpr int kBC = kNB * kBlk;                 // [n block][t][64 n]
  static constexpr int kG = 2 * kBlk;                    // [s block][t][64 s]
  static constexpr int kHb = kNB * kBlk;                 // [n block][2 x 64 rows hp][64 n]
  static constexpr int kOffX0 = 0;
  static constexpr int kOffX1 = kXBuf;
  static constexpr int kOffB = 2 * kXBuf;
  static constexpr int kOffC = kOffB + kBC;
  static constexpr int kOffG = kOffC + kBC;
  static constexpr int kOffHb = kOffG + kG;
  static constexpr int kOffSteps = kOffHb + kHb;
  // per head: Delta[Q], cum[Q], w[Q], E[Q]; warp sums [2][4]; decay [2]
  static constexpr int kStepFloats = kTHeads * 4 * kTQ + kTHeads * 4 + kTHeads + 2;
  static constexpr int kOffBar = round_up(kOffSteps + kStepFloats * 4, 8);
  static constexpr int kNumBars = 6;  // B/C, x (two buffers), S, first MMAs, second MMAs
  static constexpr int kOffSlot = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffSlot + 16 + 1024;  // + room to align the base to 1024
  static_assert(N == 64 || N == 128, "state width 64 or 128");
};

// Wait for phase `parity` of `bar`, every thread of the CTA; false everywhere
// if any thread's wait ran out.
__device__ __forceinline__ bool cta_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const bool ok = mbar_wait_bounded(bar, parity, limit_ns);
  return __syncthreads_and(ok) != 0;
}

// Eight fp32 values scaled and packed as eight bf16 (one 16-byte chunk).
__device__ __forceinline__ uint4 pack8(const float* v) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
}

template <int N>
__global__ void __launch_bounds__(kTThreads, 1)
    ssd_tc_kernel(const SsdParams p, const __grid_constant__ SsdTcMaps maps) {
  using Ly = TcLayout<N>;
  constexpr int kNB = Ly::kNB;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h0 = blockIdx.x * kTHeads, b = blockIdx.y;
  const int H = p.nheads;
  const int64_t L = p.seqlen;
  const int nchunks = (int)((L + kTQ - 1) / kTQ);

  float* f_delta = reinterpret_cast<float*>(sm + Ly::kOffSteps);  // [2][Q]
  float* f_cum = f_delta + kTHeads * kTQ;                          // [2][Q]
  float* f_w = f_cum + kTHeads * kTQ;                              // [2][Q]
  float* f_e = f_w + kTHeads * kTQ;                                // [2][Q]
  float* f_wsum = f_e + kTHeads * kTQ;                             // [2][4]
  float* f_decay = f_wsum + kTHeads * 4;                           // [2]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Ly::kOffBar);
  uint64_t* bar_bc = bars + 0;
  uint64_t* bar_x = bars + 1;  // [2]
  uint64_t* bar_s = bars + 3;
  uint64_t* bar_m1 = bars + 4;
  uint64_t* bar_m2 = bars + 5;
  (void)bar_m2;
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + Ly::kOffSlot);
  unsigned char* const xbuf0 = sm + Ly::kOffX0;
  unsigned char* const xbuf1 = sm + Ly::kOffX1;
  unsigned char* sB = sm + Ly::kOffB;
  unsigned char* sC = sm + Ly::kOffC;
  unsigned char* sG = sm + Ly::kOffG;
  unsigned char* sHb = sm + Ly::kOffHb;

  float Ah[kTHeads], bias[kTHeads], Dh[kTHeads];
#pragma unroll
  for (int i = 0; i < kTHeads; ++i) {
    Ah[i] = p.A[h0 + i];
    bias[i] = p.dt_bias ? p.dt_bias[h0 + i] : 0.f;
    Dh[i] = p.D ? p.D[h0 + i] : 0.f;
  }

  if (tid == 0) {
    for (int i = 0; i < Ly::kNumBars; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    prefetch_tensormap(&maps.x);
    prefetch_tensormap(&maps.B);
    prefetch_tensormap(&maps.C);
  }
  if (warp == 0) tc::tmem_alloc(slot, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tm = *slot;
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
  const uint32_t tH = tm + lane_base + kColH, tS = tm + lane_base + kColS;
  const uint32_t tYd = tm + lane_base + kColYd, tYo = tm + lane_base + kColYo;

  // ---- initial state: thread = TMEM lane = state row (head h0 + tid / 64, p)
  {
    const float* src = p.h0 ? p.h0 + (((size_t)b * H + h0 + tid / kTP) * kTP + tid % kTP) * N
                            : nullptr;
#pragma unroll
    for (int c0 = 0; c0 < N; c0 += 32) {
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const float4 q = src ? *reinterpret_cast<const float4*>(src + c0 + j)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        v[j] = q.x; v[j + 1] = q.y; v[j + 2] = q.z; v[j + 3] = q.w;
      }
      tc::st32(tH + c0, v);
    }
    tc::wait_st();
  }

  // TMA issue (thread 0): B and C of chunk c; x of chunk c into buffer i.
  const bool stall = p.test_stall && blockIdx.x == 0 && blockIdx.y == 0;
  auto issue_bc = [&](int c) {
    mbar_arrive_expect_tx(bar_bc, (uint32_t)(2 * kNB * Ly::kBlk));
#pragma unroll
    for (int nb = 0; nb < kNB; ++nb) {
      tma_load_3d(sB + nb * Ly::kBlk, &maps.B, bar_bc, nb * 64, c * kTQ, b);
      tma_load_3d(sC + nb * Ly::kBlk, &maps.C, bar_bc, nb * 64, c * kTQ, b);
    }
  };
  auto issue_x = [&](int c, int i) {
    uint64_t* bar = i ? &bar_x[1] : &bar_x[0];
    unsigned char* dst = i ? xbuf1 : xbuf0;
    mbar_arrive_expect_tx(bar, (uint32_t)(kTHeads * Ly::kBlk) + ((stall && c == 0) ? 16u : 0u));
#pragma unroll
    for (int hh = 0; hh < kTHeads; ++hh)
      tc::tma_load_4d(dst + hh * Ly::kBlk, &maps.x, bar, 0, h0 + hh, c * kTQ, b);
  };
  // Each barrier completes once per chunk (an x buffer every other chunk), in
  // order, so the phase to wait for follows from the chunk index; on the
  // error path thread 0 waits (bounded) for the completions still owed.
  // armed_*: phases armed so far by thread 0 (B/C, x0, x1, S, MMA1, MMA2).
  int armed_bc = 0, armed_x0 = 0, armed_x1 = 0, armed_s = 0, armed_m1 = 0, armed_m2 = 0;
  // phases waited (every thread)
  int waited_bc = 0, waited_x0 = 0, waited_x1 = 0, waited_s = 0, waited_m1 = 0, waited_m2 = 0;
  if (tid == 0 && nchunks > 0) {
    issue_bc(0);
    issue_x(0, 0);
    armed_bc = 1;
    armed_x0 = 1;
  }
  // raw dt of this thread's step in chunk c, both heads (one 4-byte load:
  // h0 and H are even)
  auto load_dt = [&](int c, float (&r)[kTHeads]) {
    const int64_t t = (int64_t)c * kTQ + tid;
    const uint32_t w = t < L ? *reinterpret_cast<const uint32_t*>(p.dt + ((size_t)b * L + t) * H + h0)
                             : 0u;
    r[0] = bf16_lo(w);
    r[1] = bf16_hi(w);
  };
  float dt_next[kTHeads];
  if (nchunks > 0) load_dt(0, dt_next);

  bool ok = true;
  int c = 0;
  for (; c < nchunks; ++c) {
    const int xi = c & 1;
    const int64_t t0 = (int64_t)c * kTQ;
    // ---- 1. steps of the chunk: Delta, the in-chunk cumulative sum of
    //      Delta A (block scan over the 128 threads), the weights w
    float dtr[kTHeads];
#pragma unroll
    for (int hh = 0; hh < kTHeads; ++hh) dtr[hh] = dt_next[hh];
    if (c + 1 < nchunks) load_dt(c + 1, dt_next);
    float dl[kTHeads], cum[kTHeads];
#pragma unroll
    for (int hh = 0; hh < kTHeads; ++hh) {
      float d = 0.f;
      if (t0 + tid < L) {
        const float v = dtr[hh] + bias[hh];
        d = p.softplus ? (v > kSoftplusCut ? v : log1pf(expf(v))) : v;
      }
      dl[hh] = d;
      float a = d * Ah[hh];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, a, o);
        if (lane >= o) a += u;
      }
      cum[hh] = a;
      if (lane == 31) f_wsum[hh * 4 + warp] = a;
    }
    __syncthreads();
#pragma unroll
    for (int hh = 0; hh < kTHeads; ++hh) {
      float off = 0.f;
      for (int w = 0; w < warp; ++w) off += f_wsum[hh * 4 + w];
      cum[hh] += off;
      f_delta[hh * kTQ + tid] = dl[hh];
      f_cum[hh * kTQ + tid] = cum[hh];
    }
    __syncthreads();
#pragma unroll
    for (int hh = 0; hh < kTHeads; ++hh) {
      const float cend = f_cum[hh * kTQ + kTQ - 1];
      f_w[hh * kTQ + tid] = expf(cend - cum[hh]) * dl[hh];
      // factor of column s of G below the diagonal 32 x 32 blocks (<= Delta_s)
      f_e[hh * kTQ + tid] = expf(f_cum[hh * kTQ + (tid | 31)] - cum[hh]) * dl[hh];
      if (tid == 0) f_decay[hh] = expf(cend);
    }
    // ---- 2. S = C B^T once this chunk's B and C have landed
    ok = cta_wait(bar_bc, (uint32_t)(c & 1), p.wait_limit_ns);
    if (!ok) break;
    ++waited_bc;
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, 128, 0, 0);
#pragma unroll
      for (int ks = 0; ks < N / 16; ++ks) {
        const uint32_t o = (ks / 4) * Ly::kBlk + (ks % 4) * 32;
        tc::mma_bf16(tm + kColS, tc::sdesc(smem_u32(sC) + o, 16, 1024),
                     tc::sdesc(smem_u32(sB) + o, 16, 1024), id, ks > 0);
      }
      tc::commit(bar_s);
      ++armed_s;
    }
    // ---- 3. this chunk's x: w-scaled copy into the other buffer (row s =
    //      thread); the state: bf16 copy for the readout, then scaled by
    //      e^{cum_end} in place for the update (row hp = thread)
    ok = cta_wait(xi ? &bar_x[1] : &bar_x[0], (uint32_t)((c >> 1) & 1), p.wait_limit_ns);
    if (!ok) break;
    if (xi) ++waited_x1; else ++waited_x0;
    unsigned char* const xcur = xi ? xbuf1 : xbuf0;  // x of this chunk
    unsigned char* const xoth = xi ? xbuf0 : xbuf1;  // its w-scaled copy
    {
      const unsigned char* src = xcur;
      unsigned char* dst = xoth;
#pragma unroll
      for (int hh = 0; hh < kTHeads; ++hh) {
        const float w = f_w[hh * kTQ + tid];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t o = hh * Ly::kBlk + tid * 128 + ((j + tid) & 7) * 16;
          const uint4 q = *reinterpret_cast<const uint4*>(src + o);
          const float v[8] = {bf16_lo(q.x) * w, bf16_hi(q.x) * w, bf16_lo(q.y) * w,
                              bf16_hi(q.y) * w, bf16_lo(q.z) * w, bf16_hi(q.z) * w,
                              bf16_lo(q.w) * w, bf16_hi(q.w) * w};
          *reinterpret_cast<uint4*>(dst + o) = pack8(v);
        }
      }
      const float decay = f_decay[tid / kTP];
#pragma unroll
      for (int c0 = 0; c0 < N; c0 += 64) {
        float v[32], u[32];
        tc::ld32(tH + c0, v);
        tc::ld32(tH + c0 + 32, u);
        tc::wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          *reinterpret_cast<uint4*>(sHb + (c0 / 64) * Ly::kBlk + tc::sw128(tid, j)) = pack8(v + j);
          *reinterpret_cast<uint4*>(sHb + (c0 / 64) * Ly::kBlk + tc::sw128(tid, 32 + j)) =
              pack8(u + j);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          v[j] *= decay;
          u[j] *= decay;
        }
        tc::st32(tH + c0, v);
        tc::st32(tH + c0 + 32, u);
      }
      tc::wait_st();
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    // ---- 4. G of head 0 from S (row t = thread)
    ok = cta_wait(bar_s, (uint32_t)(c & 1), p.wait_limit_ns);
    if (!ok) break;
    ++waited_s;
    tc::fence_after_sync();
    // G row t (= thread) of head hh from S, in 32-column blocks j: below the
    // diagonal block (32 j + 31 < t's block) e^{cum_t - cum_s} Delta_s =
    // F_j E_s with F_j = e^{cum_t - cum_{32 j + 31}} (both factors <= 1, one
    // exp per block); the diagonal block takes one exp per entry; above it G
    // is zero.
    auto make_g = [&](int hh) {
      const float ct = f_cum[hh * kTQ + tid];
      const int tb = tid >> 5;  // this row's diagonal block
#pragma unroll
      for (int c0 = 0; c0 < kTQ; c0 += 64) {
        float v[2][32];
        tc::ld32(tS + c0, v[0]);
        tc::ld32(tS + c0 + 32, v[1]);
        tc::wait_ld();
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          const int j = (c0 >> 5) + hb;  // column block
          const int s0 = 32 * j;
          float g[32];
          if (j < tb) {
            const float F = expf(ct - f_cum[hh * kTQ + s0 + 31]);
#pragma unroll
            for (int e = 0; e < 32; ++e) g[e] = v[hb][e] * F * f_e[hh * kTQ + s0 + e];
          } else if (j == tb) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int sidx = s0 + e;
              g[e] = sidx <= tid ? v[hb][e] * ex2_approx((ct - f_cum[hh * kTQ + sidx]) * kLog2e) *
                                       f_delta[hh * kTQ + sidx]
                                 : 0.f;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) g[e] = 0.f;
          }
#pragma unroll
          for (int e = 0; e < 32; e += 8)
            *reinterpret_cast<uint4*>(sG + (s0 / 64) * Ly::kBlk + tc::sw128(tid, (s0 + e) % 64)) =
                pack8(g + e);
        }
      }
    };
    make_g(0);
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    // ---- 5. the readout C H^T, the state update, G X of head 0
    if (tid == 0) {
      tc::fence_after_sync();
      {  // Yo (t x 2P) = C (t x N) . Hb^T, both K-major over n
        constexpr uint32_t id = tc::idesc_bf16(128, 128, 0, 0);
#pragma unroll
        for (int ks = 0; ks < N / 16; ++ks) {
          const uint32_t o = (ks / 4) * Ly::kBlk + (ks % 4) * 32;
          tc::mma_bf16(tm + kColYo, tc::sdesc(smem_u32(sC) + o, 16, 1024),
                       tc::sdesc(smem_u32(sHb) + o, 16, 1024), id, ks > 0);
        }
      }
      {  // H (2P x N) += Xt^T (2P x s) . B (s x N), both MN-major over s
        constexpr uint32_t id = tc::idesc_bf16(128, N, 1, 1);
#pragma unroll
        for (int ks = 0; ks < kTQ / 16; ++ks) {
          const uint32_t o = ks * 2048;
          tc::mma_bf16(tm + kColH, tc::sdesc(smem_u32(xoth) + o, Ly::kBlk, 1024),
                       tc::sdesc(smem_u32(sB) + o, Ly::kBlk, 1024), id, 1u);
        }
      }
      {  // Yd[:, head 0] (t x P) = G (t x s, K-major) . x_0 (s x P, MN-major)
        constexpr uint32_t id = tc::idesc_bf16(128, kTP, 0, 1);
#pragma unroll
        for (int ks = 0; ks < kTQ / 16; ++ks) {
          const uint32_t oa = (ks / 4) * Ly::kBlk + (ks % 4) * 32;
          tc::mma_bf16(tm + kColYd, tc::sdesc(smem_u32(sG) + oa, 16, 1024),
                       tc::sdesc(smem_u32(xcur) + ks * 2048, Ly::kBlk, 1024), id, ks > 0);
        }
      }
      tc::commit(bar_m1);
      ++armed_m1;
    }
    // ---- 6. the buffers of B, C and the scaled x are free: next chunk's
    //      loads; G of head 1 (G's buffer is free too), then its G X
    ok = cta_wait(bar_m1, (uint32_t)(c & 1), p.wait_limit_ns);
    if (!ok) break;
    ++waited_m1;
    tc::fence_after_sync();
    if (tid == 0 && c + 1 < nchunks) {
      issue_bc(c + 1);
      issue_x(c + 1, xi ^ 1);
      ++armed_bc;
      if (xi) ++armed_x0; else ++armed_x1;
    }
    make_g(1);
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, kTP, 0, 1);
#pragma unroll
      for (int ks = 0; ks < kTQ / 16; ++ks) {
        const uint32_t oa = (ks / 4) * Ly::kBlk + (ks % 4) * 32;
        tc::mma_bf16(tm + kColYd + kTP, tc::sdesc(smem_u32(sG) + oa, 16, 1024),
                     tc::sdesc(smem_u32(xcur) + Ly::kBlk + ks * 2048, Ly::kBlk, 1024), id,
                     ks > 0);
      }
      tc::commit(bar_m2);
      ++armed_m2;
    }
    // ---- 7. y_t = Yd + e^{cum_t} Yo + D x_t (row t = thread)
    ok = cta_wait(bar_m2, (uint32_t)(c & 1), p.wait_limit_ns);
    if (!ok) break;
    ++waited_m2;
    tc::fence_after_sync();
    {
      const int64_t t = t0 + tid;
#pragma unroll
      for (int hh = 0; hh < kTHeads; ++hh) {
        const float ec = expf(f_cum[hh * kTQ + tid]);
        uint16_t* yrow = p.y + (((size_t)b * L + (t < L ? t : 0)) * H + h0 + hh) * kTP;
#pragma unroll
        for (int c0 = 0; c0 < kTP; c0 += 32) {
          float yd[32], yo[32];
          tc::ld32(tYd + hh * kTP + c0, yd);
          tc::ld32(tYo + hh * kTP + c0, yo);
          tc::wait_ld();
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            const int pc = c0 + j;
            const uint4 q = *reinterpret_cast<const uint4*>(xcur + hh * Ly::kBlk +
                                                            tc::sw128(tid, pc));
            const float xv[8] = {bf16_lo(q.x), bf16_hi(q.x), bf16_lo(q.y), bf16_hi(q.y),
                                 bf16_lo(q.z), bf16_hi(q.z), bf16_lo(q.w), bf16_hi(q.w)};
            float o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = fmaf(Dh[hh], xv[e], fmaf(ec, yo[j + e], yd[j + e]));
            if (t < L) *reinterpret_cast<uint4*>(yrow + pc) = pack8(o);
          }
        }
      }
    }
    tc::fence_before_sync();
    __syncthreads();
  }

  if (ok) {
    if (p.h_last) {
      tc::fence_after_sync();
      float* dst = p.h_last + (((size_t)b * H + h0 + tid / kTP) * kTP + tid % kTP) * N;
#pragma unroll
      for (int c0 = 0; c0 < N; c0 += 32) {
        float v[32];
        tc::ld32(tH + c0, v);
        tc::wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(dst + c0 + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      }
    }
  } else if (tid == 0) {
    // A wait ran out: let this CTA's own copies and MMAs in flight land
    // (bounded) before its shared and tensor memory are released.
    auto drain = [&](uint64_t* bar, int done, int armed) {
      for (int k = done; k < armed; ++k) (void)mbar_wait_bounded(bar, (uint32_t)(k & 1), 1000000ull);
    };
    drain(bar_bc, waited_bc, armed_bc);
    drain(&bar_x[0], waited_x0, armed_x0);
    drain(&bar_x[1], waited_x1, armed_x1);
    drain(bar_s, waited_s, armed_s);
    drain(bar_m1, waited_m1, armed_m1);
    drain(bar_m2, waited_m2, armed_m2);
    atomicExch(&g_ssd_status, 1);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tm, kTmemCols);
}

cudaError_t set_smem_tc(const void* kernel, int smem) {
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

template <int N>
cudaError_t launch_tc_n(const SsdParams& p, const SsdTcMaps& maps, cudaStream_t stream) {
  constexpr int smem = TcLayout<N>::kBytes;
  cudaError_t e = set_smem_tc(reinterpret_cast<const void*>(ssd_tc_kernel<N>), smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)(p.nheads / kTHeads), (unsigned)p.batch);
  ssd_tc_kernel<N><<<grid, kTThreads, smem, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace

bool ssd_tc_supported(int dstate, int nheads) {
  return (dstate == 64 || dstate == 128) && nheads % kTHeads == 0;
}

cudaError_t launch_ssd_tc(const SsdParams& p, const SsdTcMaps& maps, cudaStream_t stream) {
  switch (p.dstate) {
    case 64: return launch_tc_n<64>(p, maps, stream);
    case 128: return launch_tc_n<128>(p, maps, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t ssd_tc_status(cudaStream_t stream, int* out) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_ssd_status, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_ssd_status, &zero, sizeof(int));
    if (e != cudaSuccess) return e;
  }
  *out = v;
  return cudaSuccess;
}

}  // namespace ssm
