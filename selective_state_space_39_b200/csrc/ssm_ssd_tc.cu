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
// Design (B200). One CTA per batch row and pair of heads walks the chunks in
// order. Warp roles: one warp issues every TMA copy and MMA, one computes the
// step quantities (Delta, cum, w, E, e^{cum_end}) up to three chunks ahead,
// sixteen compute warps do the rest (warps w, w + 4, w + 8, w + 12 share TMEM
// lanes 32 (w % 4) .. and take a quarter of each row's columns, or a head and
// half its columns, each). They meet at mbarriers: the readout and the state
// update run while the compute warps form G, G X of the first head while they
// form the second head's G, the next chunk's S while they write this chunk's
// outputs. Every product is a tcgen05 MMA of M = 128 with fp32 accumulators
// in TMEM:
//   S = C B^T (t x s, K = N; both operands from shared memory),
//   the readout C H^T (t x (2 heads x p), K = N; H as a bf16 copy in shared
//   memory),
//   the state update (2 heads x p) x n, K = s (w-scaled x and B from shared
//   memory, accumulating onto the state in TMEM),
//   G X per head (t x p, K = s; G from TMEM, where it is written over S).
// The state (2 x 64 rows, N columns) never leaves TMEM: each chunk the
// threads read it, keep the bf16 copy for the readout and write it back
// scaled by e^{cum_end} before the update MMA accumulates onto it. x, B and
// C arrive by TMA with the 128-byte swizzle the MMA descriptors describe (no
// multicast): x a chunk ahead into two buffers, B and C once the readout and
// the update have released them. y is written over the chunk's x in shared
// memory and stored by TMA. Steps past the sequence end read zeros and take
// Delta = 0, so they change nothing. Every wait is bounded; a wait that runs
// out stops the CTA (after its copies and MMAs in flight land, bounded too),
// frees its TMEM and sets the flag that ssm_ssd_scan_status reports.
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
constexpr int kTWork = 512;     // sixteen compute warps, four per TMEM lane quadrant
// and two warps: one issues the copies and MMAs, one computes the step quantities
constexpr int kTThreads = kTWork + 64;
constexpr uint32_t kTmemCols = 512;
// TMEM columns: the state, S (then G of both heads, bf16 pairs), G X, C H^T
constexpr uint32_t kColH = 0, kColS = 128, kColYd = 256, kColYo = 384;

constexpr int round_up(int v, int m) { return (v + m - 1) / m * m; }

template <int N>
struct TcLayout {
  static constexpr int kNB = N / 64;               // 64-wide blocks of the state
  static constexpr int kBlk = kTQ * 128;           // one [128 rows][64] bf16 tile
  static constexpr int kXBuf = kTHeads * kBlk;     // [head][t][64 p]
  static constexpr int kBC = kNB * kBlk;           // [n block][t][64 n]
  static constexpr int kHb = kNB * kBlk;           // [n block][2 x 64 rows hp][64 n]
  // two buffers of raw x (a chunk's y is staged over its x), the w-scaled x
  static constexpr int kOffX0 = 0;
  static constexpr int kOffX1 = kXBuf;
  static constexpr int kOffXs = 2 * kXBuf;
  static constexpr int kOffB = 3 * kXBuf;
  static constexpr int kOffC = kOffB + kBC;
  static constexpr int kOffHb = kOffC + kBC;
  static constexpr int kOffSteps = kOffHb + kHb;
  // step quantities, per head Delta[Q], cum[Q], w[Q], E[Q]
  static constexpr int kStepBuf = kTHeads * 4 * kTQ;
  // three buffers (chunk % 3), then e^{cum_end} per buffer and head, a flag
  static constexpr int kStepFloats = 3 * kStepBuf + 3 * kTHeads + 2;
  static constexpr int kOffBar = round_up(kOffSteps + kStepFloats * 4, 8);
  // B/C, x (two buffers), S, readout + update, G X, operands, x buffer free,
  // scaled x and state written, step buffer written (3), step buffer read (3),
  // the second head's G written
  static constexpr int kNumBars = 16;
  static constexpr int kOffSlot = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffSlot + 16 + 1024;  // + room to align the base to 1024
  static_assert(N == 64 || N == 128, "state width 64 or 128");
  static_assert(kBytes <= 227 * 1024, "shared memory of one CTA");
};

// Eight fp32 values packed as eight bf16 (one 16-byte chunk).
__device__ __forceinline__ uint4 pack8(const float* v) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
}

// D (TMEM) = A B (+ D): A (M x 16, bf16 pairs) from TMEM, B from a
// shared-memory descriptor; one K = 16 step, issued by one thread.
__device__ __forceinline__ void mma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Named barrier of the compute warps (id 1, 256 threads) with an AND vote:
// every compute thread gets the same answer, so all leave a loop together.
__device__ __forceinline__ bool work_vote(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred q, p;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "barrier.cta.red.and.pred p, 1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kTWork)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void work_sync() {
  asm volatile("barrier.cta.sync 1, %0;" ::"n"(kTWork) : "memory");
}
// Non-blocking test of phase `parity` of `bar`.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return r != 0;
}
// A value the compiler cannot treat as loop-invariant: the issuing warp
// derives its descriptors from it each chunk instead of keeping dozens live.
__device__ __forceinline__ uint32_t opaque(uint32_t v) {
  asm volatile("mov.b32 %0, %0;" : "+r"(v));
  return v;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
template <int N>
__global__ void __launch_bounds__(kTThreads, 1)
    ssd_tc_kernel(const SsdParams p, const __grid_constant__ SsdTcMaps maps) {
  using Ly = TcLayout<N>;
  constexpr int kNB = Ly::kNB;
  constexpr int kQN = N / 4;  // state columns per compute warp of a lane quadrant
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool issuer = warp == kTWork / 32;       // warp 16 issues copies and MMAs
  const bool stepper = warp == kTWork / 32 + 1;  // warp 17 computes step quantities
  // a compute warp's TMEM lane quadrant and its quarter of the quadrant's work
  const int quad = warp & 3, grp = (warp >> 2) & 3;
  const int row = 32 * quad + lane;  // a compute thread's TMEM lane: a step t or a state row
  const int h0 = blockIdx.x * kTHeads, b = blockIdx.y;
  const int H = p.nheads;
  const int64_t L = p.seqlen;
  const int nchunks = (int)((L + kTQ - 1) / kTQ);

  float* steps = reinterpret_cast<float*>(sm + Ly::kOffSteps);
  float* f_decay = steps + 3 * Ly::kStepBuf;  // [buffer][head]
  // step arrays of buffer i, each [head][Q]: Delta, cum (in units of log2,
  // i.e. log2 e times the sum of Delta A), w, E
  auto sdelta = [&](int i) { return steps + i * Ly::kStepBuf; };
  auto scum = [&](int i) { return steps + i * Ly::kStepBuf + kTHeads * kTQ; };
  auto sw = [&](int i) { return steps + i * Ly::kStepBuf + 2 * kTHeads * kTQ; };
  auto se = [&](int i) { return steps + i * Ly::kStepBuf + 3 * kTHeads * kTQ; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Ly::kOffBar);
  uint64_t* bar_bc = bars + 0;     // B and C of a chunk landed (TMA)
  uint64_t* bar_x0 = bars + 1;     // x landed in buffer 0 / 1 (TMA)
  uint64_t* bar_x1 = bars + 2;
  uint64_t* bar_s = bars + 3;      // S = C B^T done (MMA commit)
  uint64_t* bar_h = bars + 4;      // readout C H^T and state update done (MMA commit)
  uint64_t* bar_m = bars + 5;      // G X done: every product of the chunk (MMA commit)
  uint64_t* bar_work = bars + 6;   // G of the first head is written (256 arrivals)
  uint64_t* bar_xfree = bars + 7;  // a chunk's y has left its x buffer (bulk store read)
  uint64_t* bar_xs = bars + 8;     // the scaled x and the prepared state are written (256)
  uint64_t* bar_sready = bars + 9;  // [3] step buffer written (32 arrivals)
  uint64_t* bar_sfree = bars + 12;  // [3] step buffer read for the last time
  uint64_t* bar_work1 = bars + 15;  // G of the second head is written (256 arrivals)
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + Ly::kOffSlot);
  unsigned char* const xbuf0 = sm + Ly::kOffX0;
  unsigned char* const xbuf1 = sm + Ly::kOffX1;
  unsigned char* const sXs = sm + Ly::kOffXs;
  unsigned char* sB = sm + Ly::kOffB;
  unsigned char* sC = sm + Ly::kOffC;
  unsigned char* sHb = sm + Ly::kOffHb;
  int* f_fail = reinterpret_cast<int*>(f_decay + 3 * kTHeads);

  if (tid == 0) {
    for (int i = 0; i < Ly::kNumBars; ++i)
      mbar_init(&bars[i], (i == 6 || i == 8 || i == 15) ? kTWork : (i >= 9 && i < 12) ? 32 : 1);
    *f_fail = 0;
    fence_mbar_init();
    prefetch_tensormap(&maps.x);
    prefetch_tensormap(&maps.B);
    prefetch_tensormap(&maps.C);
    prefetch_tensormap(&maps.y);
  }
  if (warp == 0) tc::tmem_alloc(slot, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tm = *slot;
  const bool stall = p.test_stall && blockIdx.x == 0 && blockIdx.y == 0;

  if (issuer) {
    // ------------------------------------------------------ issuing warp --
    if (lane == 0 && nchunks > 0) {
      auto issue_bc = [&](int c) {
        mbar_arrive_expect_tx(bar_bc, (uint32_t)(2 * kNB * Ly::kBlk));
#pragma unroll
        for (int nb = 0; nb < kNB; ++nb) {
          tma_load_3d(sB + nb * Ly::kBlk, &maps.B, bar_bc, nb * 64, c * kTQ, b);
          tma_load_3d(sC + nb * Ly::kBlk, &maps.C, bar_bc, nb * 64, c * kTQ, b);
        }
      };
      auto issue_x = [&](int c, int i) {
        uint64_t* bar = i ? bar_x1 : bar_x0;
        unsigned char* dst = i ? xbuf1 : xbuf0;
        mbar_arrive_expect_tx(bar,
                              (uint32_t)(kTHeads * Ly::kBlk) + ((stall && c == 0) ? 16u : 0u));
#pragma unroll
        for (int hh = 0; hh < kTHeads; ++hh)
          tc::tma_load_4d(dst + hh * Ly::kBlk, &maps.x, bar, 0, h0 + hh, c * kTQ, b);
      };
      // last phase armed per barrier (-1: none): on the error path each is
      // waited for (bounded); earlier phases complete first
      int last_bc = 0, last_x0 = 0, last_x1 = -1, last_s = -1, last_h = -1, last_m = -1;
      issue_bc(0);
      issue_x(0, 0);
      bool ok = true;
      for (int c = 0; c < nchunks; ++c) {
        const int xi = c & 1;
        const uint32_t uB = opaque(smem_u32(sB)), uC = opaque(smem_u32(sC));
        const uint32_t uHb = opaque(smem_u32(sHb)), uXs = opaque(smem_u32(sXs));
        const uint32_t uxcur = opaque(smem_u32(xi ? xbuf1 : xbuf0));
        const uint32_t tmo = opaque(tm);
        // S = C B^T once this chunk's B and C have landed and the previous
        // chunk's G X no longer reads the S columns
        ok = mbar_wait_bounded(bar_bc, (uint32_t)(c & 1), p.wait_limit_ns);
        if (ok && c > 0) ok = mbar_wait_bounded(bar_m, (uint32_t)((c - 1) & 1), p.wait_limit_ns);
        if (!ok) break;
        tc::fence_after_sync();
        {
          constexpr uint32_t id = tc::idesc_bf16(128, 128, 0, 0);
#pragma unroll
          for (int ks = 0; ks < N / 16; ++ks) {
            const uint32_t o = (ks / 4) * Ly::kBlk + (ks % 4) * 32;
            tc::mma_bf16(tmo + kColS, tc::sdesc(uC + o, 16, 1024), tc::sdesc(uB + o, 16, 1024), id,
                         ks > 0);
          }
          tc::commit(bar_s);
          last_s = c;
        }
        // the next chunk's x, into the buffer the previous chunk's y has left
        if (c + 1 < nchunks) {
          if (c > 0) {
            ok = mbar_wait_bounded(bar_xfree, (uint32_t)((c - 1) & 1), p.wait_limit_ns);
            if (!ok) break;
          }
          issue_x(c + 1, xi ^ 1);
          if (xi) last_x0 = c + 1; else last_x1 = c + 1;
        }
        // the compute warps have written the scaled x, the bf16 copy of the
        // state and the scaled state
        ok = mbar_wait_bounded(bar_xs, (uint32_t)(c & 1), p.wait_limit_ns);
        if (!ok) break;
        tc::fence_after_sync();
        {  // Yo (t x 2P) = C (t x N) . Hb^T, both K-major over n
          constexpr uint32_t id = tc::idesc_bf16(128, 128, 0, 0);
#pragma unroll
          for (int ks = 0; ks < N / 16; ++ks) {
            const uint32_t o = (ks / 4) * Ly::kBlk + (ks % 4) * 32;
            tc::mma_bf16(tmo + kColYo, tc::sdesc(uC + o, 16, 1024), tc::sdesc(uHb + o, 16, 1024),
                         id, ks > 0);
          }
        }
        {  // H (2P x N) += Xs^T (2P x s) . B (s x N), both MN-major over s
          constexpr uint32_t id = tc::idesc_bf16(128, N, 1, 1);
#pragma unroll
          for (int ks = 0; ks < kTQ / 16; ++ks) {
            const uint32_t o = ks * 2048;
            tc::mma_bf16(tmo + kColH, tc::sdesc(uXs + o, Ly::kBlk, 1024),
                         tc::sdesc(uB + o, Ly::kBlk, 1024), id, 1u);
          }
        }
        tc::commit(bar_h);
        last_h = c;
        // ... and G (over S), head by head: Yd[:, head hh] (t x P) =
        // G_hh (TMEM, t x s) . x_hh (s x P, MN-major). B and C of the next
        // chunk go out once the readout and the state update are done.
        bool bc_out = c + 1 >= nchunks;
#pragma unroll
        for (int hh = 0; hh < kTHeads; ++hh) {
          ok = mbar_wait_bounded(hh ? bar_work1 : bar_work, (uint32_t)(c & 1), p.wait_limit_ns);
          if (!ok) break;
          tc::fence_after_sync();
          constexpr uint32_t id = tc::idesc_bf16(128, kTP, 0, 1);
#pragma unroll
          for (int ks = 0; ks < kTQ / 16; ++ks)
            mma_bf16_tmem_a(tmo + kColYd + kTP * hh,
                            tmo + kColS + 32 * (ks / 2) + 16 * hh + 8 * (ks % 2),
                            tc::sdesc(uxcur + hh * Ly::kBlk + ks * 2048, Ly::kBlk, 1024), id,
                            ks > 0);
          if (hh == 0 && !bc_out && mbar_test_wait(bar_h, (uint32_t)(c & 1))) {
            issue_bc(c + 1);
            last_bc = c + 1;
            bc_out = true;
          }
        }
        if (!ok) break;
        tc::commit(bar_m);
        last_m = c;
        if (!bc_out) {
          ok = mbar_wait_bounded(bar_h, (uint32_t)(c & 1), p.wait_limit_ns);
          if (!ok) break;
          issue_bc(c + 1);
          last_bc = c + 1;
        }
      }
      if (!ok) {
        // let this CTA's own copies and MMAs in flight land (bounded) before
        // its shared and tensor memory are released
        auto drain = [&](uint64_t* bar, int k) {
          if (k >= 0) (void)mbar_wait_bounded(bar, (uint32_t)(k & 1), 1000000ull);
        };
        drain(bar_bc, last_bc);
        drain(bar_x0, last_x0 >= 0 ? last_x0 / 2 : -1);
        drain(bar_x1, last_x1 >= 0 ? last_x1 / 2 : -1);
        drain(bar_s, last_s);
        drain(bar_h, last_h);
        // MMAs issued after the last commit (a chunk's first G X) complete
        // with one more phase of bar_m
        tc::commit(bar_m);
        drain(bar_m, last_m + 1);
        *f_fail = 1;
      }
    }
    __syncwarp();
  } else if (stepper) {
    // ------------------------------------------------------- steps warp --
    // Step quantities of chunk k into buffer k % 3, up to three chunks ahead
    // of the compute warps; lane = the four steps t = 4 lane + u of both
    // heads: Delta, cum (the in-chunk inclusive sum of Delta A, in log2
    // units), w_s = e^{cum_end - cum_s} Delta_s, E_s = e^{cum_{end of s's
    // 32-step block} - cum_s} Delta_s, and e^{cum_end} per head.
    float A2[kTHeads], bias[kTHeads];
#pragma unroll
    for (int hh = 0; hh < kTHeads; ++hh) {
      A2[hh] = p.A[h0 + hh] * kLog2e;
      bias[hh] = p.dt_bias ? p.dt_bias[h0 + hh] : 0.f;
    }
    bool ok = true;
    for (int k = 0; k < nchunks; ++k) {
      const int i = k % 3;
      const int64_t tb = (int64_t)k * kTQ + 4 * lane;
      uint32_t raw[4];  // dt of heads h0, h0 + 1 (4-byte aligned pairs)
#pragma unroll
      for (int u = 0; u < 4; ++u)
        raw[u] = tb + u < L ? *reinterpret_cast<const uint32_t*>(
                                  p.dt + ((size_t)b * L + tb + u) * H + h0)
                            : 0u;
      // the buffer's previous chunk has been read for the last time
      if (k >= 3) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar_sfree[i], (uint32_t)(((k - 3) / 3) & 1),
                                                        p.wait_limit_ns));
        if (!ok) break;
      }
#pragma unroll
      for (int hh = 0; hh < kTHeads; ++hh) {
        float d[4], a[4];
        float run = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float v = (hh ? bf16_hi(raw[u]) : bf16_lo(raw[u])) + bias[hh];
          // softplus(v) = ln 2 log2(1 + 2^(v log2 e)); v above the cut
          const float dv =
              tb + u >= L ? 0.f
              : p.softplus
                  ? (v > kSoftplusCut ? v : kLn2 * lg2_approx(1.f + ex2_approx(v * kLog2e)))
                  : v;
          d[u] = dv;
          run = fmaf(dv, A2[hh], run);
          a[u] = run;
        }
        float incl = run;  // scan of the lanes' sums
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float q = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += q;
        }
        const float excl = incl - run;
#pragma unroll
        for (int u = 0; u < 4; ++u) a[u] += excl;
        const float cend = __shfl_sync(0xffffffffu, a[3], 31);
        const float cblk = __shfl_sync(0xffffffffu, a[3], lane | 7);  // t = 32 (t / 32) + 31
        float w[4], e[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          w[u] = ex2_approx(cend - a[u]) * d[u];
          e[u] = ex2_approx(cblk - a[u]) * d[u];
        }
        const int o = hh * kTQ + 4 * lane;
        *reinterpret_cast<float4*>(sdelta(i) + o) = make_float4(d[0], d[1], d[2], d[3]);
        *reinterpret_cast<float4*>(scum(i) + o) = make_float4(a[0], a[1], a[2], a[3]);
        *reinterpret_cast<float4*>(sw(i) + o) = make_float4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<float4*>(se(i) + o) = make_float4(e[0], e[1], e[2], e[3]);
        if (lane == 0) f_decay[i * kTHeads + hh] = ex2_approx(cend);
      }
      mbar_arrive(&bar_sready[i]);
    }
    if (!ok && lane == 0) *f_fail = 1;
  } else {
    // ----------------------------------------------------- compute warps --
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    const uint32_t tH = tm + lane_base + kColH, tS = tm + lane_base + kColS;
    const uint32_t tYd = tm + lane_base + kColYd, tYo = tm + lane_base + kColYo;
    // the scaled copy of x: thread = (half of a row's 16-byte chunks, head, step)
    const int s_t = tid & 127, s_hh = (tid >> 7) & 1, s_ch = tid >> 8;
    // the epilogue: thread = (head, half of the head's 64 columns, step)
    const int e_hh = grp >> 1, e_ph = grp & 1;
    // the skip D x_t enters through G's diagonal: (G + diag(D)) X
    const float D0 = p.D ? p.D[h0] : 0.f, D1 = p.D ? p.D[h0 + 1] : 0.f;
    // this warp's N / 4 columns of the state (TMEM lane = state row)
    auto ldq = [&](uint32_t a, float (&v)[kQN]) {
      if constexpr (kQN == 32) tc::ld32(a, v);
      else tc::ld16(a, v);
    };
    auto stq = [&](uint32_t a, const float (&v)[kQN]) {
      if constexpr (kQN == 32) {
        tc::st32(a, v);
      } else {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(v[i]);
        tc::st16(a, r);
      }
    };
    const int q0 = grp * kQN;  // first state column of this warp

    // initial state: TMEM lane = state row (head h0 + row / 64, p)
    {
      const float* src = p.h0 ? p.h0 + (((size_t)b * H + h0 + row / kTP) * kTP + row % kTP) * N
                              : nullptr;
      float v[kQN];
#pragma unroll
      for (int j = 0; j < kQN; j += 4) {
        const float4 q = src ? *reinterpret_cast<const float4*>(src + q0 + j)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        v[j] = q.x; v[j + 1] = q.y; v[j + 2] = q.z; v[j + 3] = q.w;
      }
      stq(tH + q0, v);
      tc::wait_st();
    }

    // The state entering a chunk (thread = state row, N / 4 columns): a bf16
    // copy for the readout, then scaled by e^{cum_end} in TMEM so that the
    // update MMA accumulates onto it.
    auto prep_state = [&](int i) {
      const float decay = f_decay[i * kTHeads + row / kTP];
      float v[kQN];
      ldq(tH + q0, v);
      tc::wait_ld();
#pragma unroll
      for (int j = 0; j < kQN; j += 8) {
        const int col = q0 + j;
        *reinterpret_cast<uint4*>(sHb + (col / 64) * Ly::kBlk + tc::sw128(row, col % 64)) =
            pack8(v + j);
      }
#pragma unroll
      for (int j = 0; j < kQN; j += 2) {
        const float2 q2 = mul2(make_float2(v[j], v[j + 1]), make_float2(decay, decay));
        v[j] = q2.x;
        v[j + 1] = q2.y;
      }
      stq(tH + q0, v);
      tc::wait_st();
    };
    bool ok = true;
    if (nchunks > 0) {
      ok = work_vote(mbar_wait_bounded(&bar_sready[0], 0u, p.wait_limit_ns));
      if (ok) prep_state(0);
    }
    for (int c = 0; c < nchunks && ok; ++c) {
      const int xi = c & 1, sb = c % 3;
      const int64_t t0 = (int64_t)c * kTQ;
      unsigned char* const xcur = xi ? xbuf1 : xbuf0;  // x of this chunk, then its y
      // ---- the w-scaled copy of x (thread = (head, step, half the chunks))
      ok = work_vote(mbar_wait_bounded(xi ? bar_x1 : bar_x0, (uint32_t)((c >> 1) & 1),
                                       p.wait_limit_ns));
      if (!ok) break;
      {
        const float w = sw(sb)[s_hh * kTQ + s_t];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          // a rotated chunk order keeps a warp's 16-byte accesses on distinct banks
          const int j = 4 * s_ch + jj;
          const uint32_t o = s_hh * Ly::kBlk + s_t * 128 + ((j + s_t) & 7) * 16;
          const uint4 q = *reinterpret_cast<const uint4*>(xcur + o);
          const float2 w2 = make_float2(w, w);
          const float2 a0 = mul2(make_float2(bf16_lo(q.x), bf16_hi(q.x)), w2);
          const float2 a1 = mul2(make_float2(bf16_lo(q.y), bf16_hi(q.y)), w2);
          const float2 a2 = mul2(make_float2(bf16_lo(q.z), bf16_hi(q.z)), w2);
          const float2 a3 = mul2(make_float2(bf16_lo(q.w), bf16_hi(q.w)), w2);
          *reinterpret_cast<uint4*>(sXs + o) =
              make_uint4(pack_bf16x2(a0.x, a0.y), pack_bf16x2(a1.x, a1.y), pack_bf16x2(a2.x, a2.y),
                         pack_bf16x2(a3.x, a3.y));
        }
      }
      // the scaled x (and the state prepared in the previous iteration) are
      // ready for the readout and update MMAs
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(bar_xs);
      // the previous chunk's y store has read its buffer: the issuing warp
      // may load the next x there
      if (c > 0 && tid == 0) {
        tc::bulk_wait_read_all();
        mbar_arrive(bar_xfree);
      }
      // ---- G of both heads from S (thread = step t, the 32 steps s of block
      //      j = this warp's quarter), written as bf16 pairs over the S columns
      //      the thread read: G_hh(t, s) at column kColS + 32 (s / 32) + 16 hh
      //      + (s % 32) / 2, so no other warp's columns are touched. Blocks
      //      below the diagonal: e^{cum_t - cum_s} Delta_s = F_j E_s with F_j =
      //      e^{cum_t - cum_{32 j + 31}} (both factors <= 1, one exp per block);
      //      the diagonal block one exp per entry; above it zero.
      ok = work_vote(mbar_wait_bounded(bar_s, (uint32_t)(c & 1), p.wait_limit_ns));
      if (!ok) break;
      tc::fence_after_sync();
      {
        float v[32];
        tc::ld32(tS + 32 * grp, v);
        tc::wait_ld();
        const int t = row, tb = t >> 5, j = grp, s0 = 32 * j;
#pragma unroll
        for (int hh = 0; hh < kTHeads; ++hh) {
          const float* cum = scum(sb) + hh * kTQ;
          const float* del = sdelta(sb) + hh * kTQ;
          const float* E = se(sb) + hh * kTQ;
          const float ct = cum[t];
          uint32_t gp[16];
          if (j < tb) {
            const float F = ex2_approx(ct - cum[s0 + 31]);
            const float2 F2 = make_float2(F, F);
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 E4 = *reinterpret_cast<const float4*>(E + s0 + e);
              const float2 g0 =
                  mul2(mul2(make_float2(v[e], v[e + 1]), F2), make_float2(E4.x, E4.y));
              const float2 g1 =
                  mul2(mul2(make_float2(v[e + 2], v[e + 3]), F2), make_float2(E4.z, E4.w));
              gp[e / 2] = pack_bf16x2(g0.x, g0.y);
              gp[e / 2 + 1] = pack_bf16x2(g1.x, g1.y);
            }
          } else if (j == tb) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 c4 = *reinterpret_cast<const float4*>(cum + s0 + e);
              const float4 d4 = *reinterpret_cast<const float4*>(del + s0 + e);
              const float ex0 = ex2_approx(ct - c4.x), ex1 = ex2_approx(ct - c4.y);
              const float ex2v = ex2_approx(ct - c4.z), ex3 = ex2_approx(ct - c4.w);
              float2 g0 = mul2(mul2(make_float2(v[e], v[e + 1]), make_float2(ex0, ex1)),
                               make_float2(d4.x, d4.y));
              float2 g1 = mul2(mul2(make_float2(v[e + 2], v[e + 3]), make_float2(ex2v, ex3)),
                               make_float2(d4.z, d4.w));
              const int sb0 = s0 + e;  // steps s > t are above the diagonal
              if (sb0 > t) g0.x = 0.f;
              if (sb0 + 1 > t) g0.y = 0.f;
              if (sb0 + 2 > t) g1.x = 0.f;
              if (sb0 + 3 > t) g1.y = 0.f;
              const float Dh = hh ? D1 : D0;  // the diagonal entry s = t takes D
              if (sb0 == t) g0.x += Dh;
              if (sb0 + 1 == t) g0.y += Dh;
              if (sb0 + 2 == t) g1.x += Dh;
              if (sb0 + 3 == t) g1.y += Dh;
              gp[e / 2] = pack_bf16x2(g0.x, g0.y);
              gp[e / 2 + 1] = pack_bf16x2(g1.x, g1.y);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) gp[e] = 0u;
          }
          tc::st16(tS + 32 * j + 16 * hh, gp);
          // this head's G is written: its G X may start
          tc::wait_st();
          tc::fence_before_sync();
          mbar_arrive(hh ? bar_work1 : bar_work);
        }
      }
      // ---- the state entering the next chunk, once this chunk's readout and
      //      update are in and the next chunk's step quantities are written
      {
        bool w = mbar_wait_bounded(bar_h, (uint32_t)(c & 1), p.wait_limit_ns);
        if (w && c + 1 < nchunks)
          w = mbar_wait_bounded(&bar_sready[(c + 1) % 3], (uint32_t)(((c + 1) / 3) & 1),
                                p.wait_limit_ns);
        ok = work_vote(w);
      }
      if (!ok) break;
      tc::fence_after_sync();
      if (c + 1 < nchunks) prep_state((c + 1) % 3);
      // ---- y_t = Yd + e^{cum_t} Yo (thread = (head, 32 of its columns, step t);
      //      D x_t is in Yd), written over x_t in shared memory, then stored by TMA
      ok = work_vote(mbar_wait_bounded(bar_m, (uint32_t)(c & 1), p.wait_limit_ns));
      if (!ok) break;
      tc::fence_after_sync();
      {
        const int t = row, hh = e_hh;
        const float ec = ex2_approx(scum(sb)[hh * kTQ + t]);
        unsigned char* const xrow = xcur + hh * Ly::kBlk;
        {
          const int c0 = 32 * e_ph;
          float yd[32], yo[32];
          tc::ld32(tYd + hh * kTP + c0, yd);
          tc::ld32(tYo + hh * kTP + c0, yo);
          tc::wait_ld();
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4* const px = reinterpret_cast<uint4*>(xrow + tc::sw128(t, c0 + j));
            float o[8];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const float2 r = fma2(make_float2(ec, ec), make_float2(yo[j + e], yo[j + e + 1]),
                                    make_float2(yd[j + e], yd[j + e + 1]));
              o[e] = r.x;
              o[e + 1] = r.y;
            }
            *px = pack8(o);
          }
        }
      }
      tc::fence_proxy_async_smem();
      work_sync();
      if (tid == 0) {  // rows past the sequence end are not written
#pragma unroll
        for (int hh = 0; hh < kTHeads; ++hh)
          tc::tma_store_4d(&maps.y, xcur + hh * Ly::kBlk, 0, h0 + hh, (int)t0, b);
        tc::bulk_commit();
        mbar_arrive(&bar_sfree[sb]);  // the chunk's step buffer is free
      }
    }
    if (tid == 0) tc::bulk_wait_all();
    if (ok && p.h_last) {
      tc::fence_after_sync();
      float* dst = p.h_last + (((size_t)b * H + h0 + row / kTP) * kTP + row % kTP) * N + q0;
      float v[kQN];
      ldq(tH + q0, v);
      tc::wait_ld();
#pragma unroll
      for (int j = 0; j < kQN; j += 4)
        *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    }
    if (!ok && tid == 0) *f_fail = 1;
  }
  tc::fence_before_sync();
  __syncthreads();
  if (tid == 0 && *f_fail) atomicExch(&g_ssd_status, 1);
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
