// ssm_ssd.cu -- sm_100a kernel of the multi-head SSD scan (Mamba-2).
//
// Page "Mamba 논문 리뷰: Selective State Space Models로 Transformer를 넘어서"
// (youngju.dev), §4.1 State Space Duality and §4.2 (multi-head, larger
// state). A head h of width P = 64 has one scalar A[h] and one step
// Delta_t = softplus(dt[b,t,h] + dt_bias[h]) per token; B_t and C_t (N wide)
// are shared by the heads. With a_t = exp(Delta_t A[h]) the head's output is
// the semi-separable matrix of §4.1 acting on its inputs,
//   y_t = sum_{s<=t} (C_t . B_s) [prod_{s<r<=t} a_r] Delta_s x_s + D[h] x_t,
// which the kernel evaluates chunk by chunk (Q = 32 steps), walking the
// chunks of one (batch, head) in order and carrying the N x P state H in fp32
// registers. With cum_t = sum_{r<=t} Delta_r A[h] inside the chunk:
//   G[t][s] = (C_t . B_s) e^{cum_t - cum_s} Delta_s   (s <= t, else 0)
//   Y       = G X + diag(e^{cum}) C H + D X
//   H      <- e^{cum_end} H + (w X)^T B,   w_s = e^{cum_end - cum_s} Delta_s
// The four products (C B^T, G X, C H, (w X)^T B) are bf16 tensor-core MMAs
// (mma.sync m16n8k16, fp32 accumulation) fed from shared memory by ldmatrix,
// except that C H reads the state from the accumulators it lives in; x, B and
// C chunks arrive by cp.async two chunks ahead (zero-filled past the end of
// the sequence, where Delta is taken as 0 so that the padded steps change
// nothing).
#include <mutex>
#include <set>
#include <utility>

#include "ssm_device.cuh"
#include "ssm_ssd_internal.h"

namespace ssm {

namespace {

constexpr int kQ = kSsdChunk;    // steps per chunk
constexpr int kP = kSsdHeadDim;  // head width
constexpr int kThreads = 256;    // 8 warps
constexpr int kPadX = kP + 8;    // shared row of an x chunk (elements; 16-byte skew)
constexpr int kPadG = kQ + 8;    // shared row of G

static_assert(kQ == 32, "the in-chunk cumulative sum is one warp's scan");
// The warp that computes the steps (Delta, cumulative sums, weights): warp 2
// holds an S tile above the diagonal (row tile 0, columns 16..23) and so has
// no S product to take.
constexpr int kStepWarp = 2;

template <int N>
struct SsdLayout {
  static constexpr int kPadN = N + 8;
  static constexpr int kStages = 3;               // x, B, C chunk buffers
  static constexpr int x_elems = kQ * kPadX;      // one buffer
  static constexpr int bc_elems = kQ * kPadN;     // one buffer of B (or C)
  static constexpr int g_elems = kQ * kPadG;      // one buffer of G (two)
  static constexpr int bf16_bytes = 2 * (kStages * (x_elems + 2 * bc_elems) + 2 * g_elems);
  static constexpr int step_floats = 4 * kQ + 4;  // Delta, cum, e^cum, w, e^cum_end
  // the C H halves the two warps of a state-row pair hand each other: per
  // pair and direction, one row tile of 16 x 16 fp32 (8 floats per lane)
  static constexpr int part_floats = 4 * 2 * 32 * 8;
  static constexpr int bytes = bf16_bytes + 4 * kStages * step_floats + 4 * part_floats;
  static_assert(bf16_bytes % 16 == 0, "float arrays start 16-byte aligned");
};

// ------------------------------------------------------------ PTX wrappers --
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// d += a (16x16, row) * b (16x8, col), bf16 operands, fp32 accumulators.
// Registers only (not volatile): independent MMAs may be interleaved.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// 16-byte asynchronous copy; with valid == false nothing is read and the
// destination is zero-filled.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}
// Named barrier of the two warps that share state rows (ids 1..4, one per
// pair; id 0 is __syncthreads), 64 threads: both warps write their hand-over
// to shared memory, pass the barrier (which makes the writes visible to the
// partner), then read the partner's. Both pass it once per chunk,
// unconditionally. Immediate ids: the kernel reserves five barriers.
__device__ __forceinline__ void named_sync(int pair) {
  switch (pair) {
    case 0: asm volatile("bar.sync 1, 64;" ::: "memory"); break;
    case 1: asm volatile("bar.sync 2, 64;" ::: "memory"); break;
    case 2: asm volatile("bar.sync 3, 64;" ::: "memory"); break;
    default: asm volatile("bar.sync 4, 64;" ::: "memory"); break;
  }
}
// Both halves of a bf16 pair times their own weight, repacked.
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t v, float lo, float hi) {
  return pack_bf16x2(bf16_lo(v) * lo, bf16_hi(v) * hi);
}

// Per-chunk step quantities (one of three rotating buffers).
struct StepBuf {
  float* dt;    // Delta_s
  float* cum;   // cum_t
  float* ecum;  // e^{cum_t}
  float* w;     // e^{cum_end - cum_s} Delta_s
  float* decay; // [0] = e^{cum_end}
};

// S = C B^T on warp (rt, cq)'s 16 x 8 tile, then G = S e^{cum_t - cum_s}
// Delta_s (s <= t, else 0) as bf16 into Gd.
template <int N>
__device__ __forceinline__ void chunk_g(const uint16_t* Bb, const uint16_t* Cb, uint16_t* Gd,
                                        const StepBuf& st, int rt, int cq, int lane) {
  constexpr int kPadN = N + 8;
  const int g = lane >> 2, tig = lane & 3;
  float sacc[4] = {0.f, 0.f, 0.f, 0.f}, sodd[4] = {0.f, 0.f, 0.f, 0.f};
  if (8 * cq <= 16 * rt + 15) {  // the tile holds entries with s <= t
#pragma unroll
    for (int k0 = 0; k0 < N; k0 += 32) {
      uint32_t b0, b1, b2, b3, a0, a1, a2, a3, c0, c1, c2, c3;
      ldsm_x4(smem_u32(Bb + (8 * cq + (lane & 7)) * kPadN + k0 + (lane >> 3) * 8), b0, b1, b2,
              b3);
      ldsm_x4(smem_u32(Cb + (16 * rt + (lane & 15)) * kPadN + k0 + (lane >> 4) * 8), a0, a1, a2,
              a3);
      ldsm_x4(smem_u32(Cb + (16 * rt + (lane & 15)) * kPadN + k0 + 16 + (lane >> 4) * 8), c0, c1,
              c2, c3);
      mma_bf16(sacc, a0, a1, a2, a3, b0, b1);  // two chains: even and odd k-steps
      mma_bf16(sodd, c0, c1, c2, c3, b2, b3);
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) sacc[e] += sodd[e];
  const int ta = 16 * rt + g, tb = ta + 8, s0 = 8 * cq + 2 * tig;
  const float cuma = st.cum[ta], cumb = st.cum[tb];
  const float cs0 = st.cum[s0], cs1 = st.cum[s0 + 1];
  const float d0 = st.dt[s0], d1 = st.dt[s0 + 1];
  const float g0 = s0 <= ta ? sacc[0] * __expf(cuma - cs0) * d0 : 0.f;
  const float g1 = s0 + 1 <= ta ? sacc[1] * __expf(cuma - cs1) * d1 : 0.f;
  const float g2 = s0 <= tb ? sacc[2] * __expf(cumb - cs0) * d0 : 0.f;
  const float g3 = s0 + 1 <= tb ? sacc[3] * __expf(cumb - cs1) * d1 : 0.f;
  *reinterpret_cast<uint32_t*>(Gd + ta * kPadG + s0) = pack_bf16x2(g0, g1);
  *reinterpret_cast<uint32_t*>(Gd + tb * kPadG + s0) = pack_bf16x2(g2, g3);
}

// One CTA per (head, batch row); 8 warps. Warp w owns the S / G tile rows
// 16*(w/4).., columns 8*(w%4)..; and the state tile rows p in 16*(w%4)..,
// state columns (w/4)*N/2... The readout C H is taken from the state
// accumulators themselves: each warp forms it over its half of the states for
// its 16 rows p and all 32 steps; the two warps of a pair exchange halves
// through shared memory (a named barrier per pair) and each finishes Y for
// one row tile of those rows.
//
// Software pipeline, one CTA barrier per chunk: iteration c computes G of
// chunk c+1, Y and the state update of chunk c, the step quantities of chunk
// c+2 (warp kStepWarp), and has the x/B/C copy of chunk c+2 in flight. x, B,
// C and the step quantities rotate through three buffers; G through two.
template <int N>
__global__ void __launch_bounds__(kThreads, (N <= 128) ? 2 : 1) ssd_fwd_kernel(const SsdParams p) {
  using Lay = SsdLayout<N>;
  constexpr int kPadN = Lay::kPadN;
  constexpr int kS = Lay::kStages;
  constexpr int kNW = N / 2;   // state columns per warp
  constexpr int kNT = kNW / 8; // n8 tiles per warp
  static_assert(kNT % 2 == 0, "state tiles come in pairs from one ldmatrix.x4");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint16_t* Xs = reinterpret_cast<uint16_t*>(smem_raw);
  uint16_t* Bs = Xs + kS * Lay::x_elems;
  uint16_t* Cs = Bs + kS * Lay::bc_elems;
  uint16_t* Gs = Cs + kS * Lay::bc_elems;
  float* fbase = reinterpret_cast<float*>(smem_raw + Lay::bf16_bytes);
  float4* part = reinterpret_cast<float4*>(fbase + kS * Lay::step_floats);
  auto step_buf = [&](int i) {
    float* f = fbase + i * Lay::step_floats;
    return StepBuf{f, f + kQ, f + 2 * kQ, f + 3 * kQ, f + 4 * kQ};
  };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int h = blockIdx.x, b = blockIdx.y;
  const int H = p.nheads;
  const int64_t L = p.seqlen;
  const float Ah = p.A[h];
  const float bias = p.dt_bias ? p.dt_bias[h] : 0.f;
  const float Dh = p.D ? p.D[h] : 0.f;
  const int nchunks = (int)((L + kQ - 1) / kQ);
  const size_t row_x = (size_t)H * kP;  // elements between steps of x and y
  const uint16_t* xg = p.x + ((size_t)b * L * H + h) * kP;
  const uint16_t* Bg = p.B + (size_t)b * L * N;
  const uint16_t* Cg = p.C + (size_t)b * L * N;
  const uint16_t* dtg = p.dt + (size_t)b * L * H + h;
  uint16_t* yg = p.y + ((size_t)b * L * H + h) * kP;
  const int rt = warp >> 2;  // row tile of S, G, Y
  const int cq = warp & 3;   // column quarter of S, G, Y

  // ---- state tile in registers: hacc[j] = rows p0, p0 + 8; columns n_j, n_j + 1
  const int pt = warp & 3, ng = warp >> 2;
  const int p0 = 16 * pt + g;
  float hacc[kNT][4];
#pragma unroll
  for (int j = 0; j < kNT; ++j) {
    const int n = ng * kNW + 8 * j + 2 * tig;
    if (p.h0) {
      const float* src = p.h0 + (((size_t)b * H + h) * kP + p0) * N + n;
      const float2 u = *reinterpret_cast<const float2*>(src);
      const float2 v = *reinterpret_cast<const float2*>(src + 8 * N);
      hacc[j][0] = u.x; hacc[j][1] = u.y; hacc[j][2] = v.x; hacc[j][3] = v.y;
    } else {
      hacc[j][0] = hacc[j][1] = hacc[j][2] = hacc[j][3] = 0.f;
    }
  }


  // ---- chunk loader (x: kQ rows of 128 B; B, C: kQ rows of 2N B)
  auto load_chunk = [&](int c) {
    const int buf = c % kS;
    const int64_t t0 = (int64_t)c * kQ;
    constexpr int kXPieces = kQ * kP / 8;
    constexpr int kBPieces = kQ * N / 8;
#pragma unroll
    for (int i = tid; i < kXPieces; i += kThreads) {
      const int r = i / (kP / 8), q = i % (kP / 8);
      const bool ok = t0 + r < L;
      const uint16_t* src = ok ? xg + (size_t)(t0 + r) * row_x + q * 8 : xg;
      cp_async16(smem_u32(Xs + buf * Lay::x_elems + r * kPadX + q * 8), src, ok);
    }
#pragma unroll
    for (int i = tid; i < kBPieces; i += kThreads) {
      const int r = i / (N / 8), q = i % (N / 8);
      const bool ok = t0 + r < L;
      const size_t off = ok ? (size_t)(t0 + r) * N + q * 8 : 0;
      cp_async16(smem_u32(Bs + buf * Lay::bc_elems + r * kPadN + q * 8), Bg + off, ok);
      cp_async16(smem_u32(Cs + buf * Lay::bc_elems + r * kPadN + q * 8), Cg + off, ok);
    }
  };
  // raw step of chunk c (lane = step in the chunk), 0 past the end
  auto load_dt = [&](int c) {
    const int64_t t = (int64_t)c * kQ + lane;
    return t < L ? bf16_to_f32(dtg[(size_t)t * H]) : 0.f;
  };
  // kStepWarp: Delta, its in-chunk cumulative sum and the weights of chunk c
  auto chunk_steps = [&](int c, float raw) {
    const StepBuf st = step_buf(c % kS);
    float d = 0.f;
    if ((int64_t)c * kQ + lane < L) {
      const float v = raw + bias;
      d = p.softplus ? (v > kSoftplusCut ? v : log1pf(__expf(v))) : v;
    }
    float cum = d * Ah;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, cum, o);
      if (lane >= o) cum += u;
    }
    const float cend = __shfl_sync(0xffffffffu, cum, 31);
    st.dt[lane] = d;
    st.cum[lane] = cum;
    st.ecum[lane] = __expf(cum);
    st.w[lane] = __expf(cend - cum) * d;
    if (lane == 0) st.decay[0] = __expf(cend);
  };

  if (nchunks > 0) {
    // ---- prologue: chunks 0 and 1 in shared memory, their steps, G of chunk 0
    load_chunk(0);
    if (nchunks > 1) load_chunk(1);
    cp_async_commit();
    float dt_raw = 0.f;  // kStepWarp: raw steps two chunks ahead
    if (warp == kStepWarp) {
      chunk_steps(0, load_dt(0));
      if (nchunks > 1) chunk_steps(1, load_dt(1));
      dt_raw = load_dt(2);
    }
    cp_async_wait_all();
    __syncthreads();
    chunk_g<N>(Bs, Cs, Gs, step_buf(0), rt, cq, lane);
    __syncthreads();

    for (int c = 0; c < nchunks; ++c) {
      const int buf = c % kS;
      const int64_t t0 = (int64_t)c * kQ;
      if (c + 2 < nchunks) load_chunk(c + 2);
      cp_async_commit();
      if (warp == kStepWarp && c + 2 < nchunks) {
        chunk_steps(c + 2, dt_raw);
        dt_raw = load_dt(c + 3);
      }
      // ---- G of the next chunk
      if (c + 1 < nchunks) {
        const int nb = (c + 1) % kS;
        chunk_g<N>(Bs + nb * Lay::bc_elems, Cs + nb * Lay::bc_elems,
                   Gs + ((c + 1) & 1) * Lay::g_elems, step_buf(nb), rt, cq, lane);
      }
      const StepBuf st = step_buf(buf);
      const uint16_t* Xb = Xs + buf * Lay::x_elems;
      const uint16_t* Bb = Bs + buf * Lay::bc_elems;
      const uint16_t* Cb = Cs + buf * Lay::bc_elems;
      const uint16_t* Gb = Gs + (c & 1) * Lay::g_elems;

      // ---- C H for rows t (both row tiles) x this warp's 16 state rows p, over
      // its half of the states: the fp32 state accumulators, packed to bf16,
      // are the B operand as they stand (rows p, state pairs 2 tig, 2 tig + 1).
      float yc[2][2][4];
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int e = 0; e < 4; ++e) yc[r][q][e] = 0.f;
#pragma unroll
      for (int i = 0; i < kNT / 2; ++i) {
        const uint32_t b00 = pack_bf16x2(hacc[2 * i][0], hacc[2 * i][1]);
        const uint32_t b01 = pack_bf16x2(hacc[2 * i + 1][0], hacc[2 * i + 1][1]);
        const uint32_t b10 = pack_bf16x2(hacc[2 * i][2], hacc[2 * i][3]);
        const uint32_t b11 = pack_bf16x2(hacc[2 * i + 1][2], hacc[2 * i + 1][3]);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(smem_u32(Cb + (16 * r + (lane & 15)) * kPadN + ng * kNW + 16 * i +
                           (lane >> 4) * 8),
                  a0, a1, a2, a3);
          mma_bf16(yc[r][0], a0, a1, a2, a3, b00, b01);
          mma_bf16(yc[r][1], a0, a1, a2, a3, b10, b11);
        }
      }
      // Each warp of a pair finishes one row tile of Y (ng = 0: steps 0..15,
      // ng = 1: steps 16..31) and hands its half-state sum for the other
      // tile to its partner.
#pragma unroll
      for (int q = 0; q < 2; ++q) {  // static indices: yc stays in registers
        const float4 v0 = make_float4(yc[0][q][0], yc[0][q][1], yc[0][q][2], yc[0][q][3]);
        const float4 v1 = make_float4(yc[1][q][0], yc[1][q][1], yc[1][q][2], yc[1][q][3]);
        part[((pt * 2 + ng) * 2 + q) * 32 + lane] = ng ? v0 : v1;  // the partner's tile
      }

      // ---- H <- e^{cum_end} H + (w X)^T B on rows 16 pt.. (p), columns ng N/2.. (n)
      {
        const float decay = st.decay[0];
#pragma unroll
        for (int j = 0; j < kNT; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) hacc[j][e] *= decay;
#pragma unroll
        for (int k0 = 0; k0 < kQ; k0 += 16) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(smem_u32(Xb + (k0 + (lane & 7) + (lane >> 4) * 8) * kPadX + 16 * pt +
                             ((lane >> 3) & 1) * 8),
                    a0, a1, a2, a3);
          const int s = k0 + 2 * tig;
          const float w0 = st.w[s], w1 = st.w[s + 1], w8 = st.w[s + 8], w9 = st.w[s + 9];
          a0 = scale_bf16x2(a0, w0, w1);
          a1 = scale_bf16x2(a1, w0, w1);
          a2 = scale_bf16x2(a2, w8, w9);
          a3 = scale_bf16x2(a3, w8, w9);
#pragma unroll
          for (int j = 0; j < kNT; j += 2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(smem_u32(Bb + (k0 + (lane & 7) + ((lane >> 3) & 1) * 8) * kPadN +
                               ng * kNW + 8 * j + (lane >> 4) * 8),
                      b0, b1, b2, b3);
            mma_bf16(hacc[j], a0, a1, a2, a3, b0, b1);
            mma_bf16(hacc[j + 1], a0, a1, a2, a3, b2, b3);
          }
        }
      }

      // ---- Y = G X + diag(e^cum) C H + D x on row tile r = ng, columns 16 pt..
      {
        const int r = ng;
        float y1[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int k0 = 0; k0 < kQ; k0 += 16) {
          if (k0 <= 16 * r) {
            uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
            ldsm_x4(smem_u32(Gb + (16 * r + (lane & 15)) * kPadG + k0 + (lane >> 4) * 8), a0,
                    a1, a2, a3);
            ldsm_x4_t(smem_u32(Xb + (k0 + (lane & 7) + ((lane >> 3) & 1) * 8) * kPadX +
                               16 * pt + (lane >> 4) * 8),
                      b0, b1, b2, b3);
            mma_bf16(y1[0], a0, a1, a2, a3, b0, b1);
            mma_bf16(y1[1], a0, a1, a2, a3, b2, b3);
          }
        }
        named_sync(pt);  // both warps of the pair have written their hand-over
        float ysum[2][4];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float4 o = part[((pt * 2 + (1 - ng)) * 2 + q) * 32 + lane];
          ysum[q][0] = (ng ? yc[1][q][0] : yc[0][q][0]) + o.x;
          ysum[q][1] = (ng ? yc[1][q][1] : yc[0][q][1]) + o.y;
          ysum[q][2] = (ng ? yc[1][q][2] : yc[0][q][2]) + o.z;
          ysum[q][3] = (ng ? yc[1][q][3] : yc[0][q][3]) + o.w;
        }
        const int ta = 16 * r + g, tb = ta + 8;
        const float ea = st.ecum[ta], eb = st.ecum[tb];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int pc = 16 * pt + 8 * q + 2 * tig;
          const uint32_t xa = *reinterpret_cast<const uint32_t*>(Xb + ta * kPadX + pc);
          const uint32_t xb = *reinterpret_cast<const uint32_t*>(Xb + tb * kPadX + pc);
          if (t0 + ta < L)
            *reinterpret_cast<uint32_t*>(yg + (size_t)(t0 + ta) * row_x + pc) =
                pack_bf16x2(fmaf(Dh, bf16_lo(xa), fmaf(ea, ysum[q][0], y1[q][0])),
                            fmaf(Dh, bf16_hi(xa), fmaf(ea, ysum[q][1], y1[q][1])));
          if (t0 + tb < L)
            *reinterpret_cast<uint32_t*>(yg + (size_t)(t0 + tb) * row_x + pc) =
                pack_bf16x2(fmaf(Dh, bf16_lo(xb), fmaf(eb, ysum[q][2], y1[q][2])),
                            fmaf(Dh, bf16_hi(xb), fmaf(eb, ysum[q][3], y1[q][3])));
        }
      }
      cp_async_wait_all();
      __syncthreads();
    }
  }

  if (p.h_last) {
#pragma unroll
    for (int j = 0; j < kNT; ++j) {
      const int n = ng * kNW + 8 * j + 2 * tig;
      float* dst = p.h_last + (((size_t)b * H + h) * kP + p0) * N + n;
      *reinterpret_cast<float2*>(dst) = make_float2(hacc[j][0], hacc[j][1]);
      *reinterpret_cast<float2*>(dst + 8 * N) = make_float2(hacc[j][2], hacc[j][3]);
    }
  }
}

cudaError_t set_smem_once(const void* kernel, int smem) {
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
cudaError_t launch_n(const SsdParams& p, cudaStream_t stream) {
  constexpr int smem = SsdLayout<N>::bytes;
  cudaError_t e = set_smem_once(reinterpret_cast<const void*>(ssd_fwd_kernel<N>), smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)p.nheads, (unsigned)p.batch);
  ssd_fwd_kernel<N><<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

bool ssd_dstate_supported(int dstate) { return dstate == 64 || dstate == 128 || dstate == 256; }

cudaError_t launch_ssd_fwd(const SsdParams& p, cudaStream_t stream) {
  switch (p.dstate) {
    case 64: return launch_n<64>(p, stream);
    case 128: return launch_n<128>(p, stream);
    case 256: return launch_n<256>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ssm
