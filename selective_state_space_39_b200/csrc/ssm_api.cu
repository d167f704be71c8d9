// ssm_api.cu -- the extern "C" entry points declared in include/ssm_scan.h:
// argument validation (on the host, before anything is enqueued), the
// sequence-segment plan, TMA tensor-map encoding and kernel launch.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <initializer_list>
#include <mutex>

#include "../../include/ssm_scan.h"
#include "ssm_bwd_internal.h"
#include "ssm_conv_internal.h"
#include "ssm_seqpar_internal.h"
#include "ssm_ssd_decode_internal.h"
#include "ssm_ssd_internal.h"
#include "ssm_internal.h"

namespace ssm {

int scan_channels_per_thread(int dstate);

namespace {

constexpr int kVersion = 10000;  // 1.0.0

// Detail of the last failure on this host thread (ssm_last_error_detail).
thread_local char g_detail[256] = "";

struct Dims {
  int64_t batch, seqlen, dim, dstate;
  int io;
};

size_t io_bytes(int io) { return io == SSM_DTYPE_BF16 ? 2 : 4; }
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Tensors past 2^40 elements are rejected: no GPU holds one, and every byte
// count and index computed for an accepted call then stays far from 64-bit
// overflow. The product is taken in double, which cannot overflow here.
constexpr double kMaxElements = 1099511627776.0;
bool too_large(std::initializer_list<int64_t> dims) {
  double n = 1.0;
  for (int64_t d : dims) n *= (double)d;
  return n > kMaxElements;
}

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

int dims_status(const Dims& d) {
  if (d.io != SSM_DTYPE_F32 && d.io != SSM_DTYPE_BF16) return SSM_ERR_UNSUPPORTED;
  if (d.batch < 0 || d.seqlen < 0 || d.dim < 0) return SSM_ERR_INVALID_ARG;
  if (d.dstate <= 0) return SSM_ERR_INVALID_ARG;
  if (!scan_dstate_supported((int)std::min<int64_t>(d.dstate, 1 << 20))) return SSM_ERR_UNSUPPORTED;
  // grid and index limits of this library
  if (d.batch > 65535 || d.dim > (1 << 24) || d.seqlen > (1 << 30)) return SSM_ERR_UNSUPPORTED;
  if (too_large({d.batch, d.seqlen, d.dim}) || too_large({d.batch, d.seqlen, d.dstate}) ||
      too_large({d.batch, d.dim, d.dstate}))
    return SSM_ERR_UNSUPPORTED;
  return SSM_OK;
}

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0) {
    cudaGetLastError();  // clear: no device is not an error for planning
    return 148;          // B200
  }
  return sms;
}

long env_long(const char* name, long dflt) {
  const char* v = getenv(name);
  if (!v || !*v) return dflt;
  char* end = nullptr;
  const long r = strtol(v, &end, 10);
  return (end && *end == '\0') ? r : dflt;
}

// Split of the sequence into segments: enough CTAs for about
// `ctas_per_sm` resident CTAs on every SM, in whole tiles.
ScanPlan make_plan(const Dims& d) {
  ScanPlan pl{};
  const int T = kScanTileSteps;
  pl.channels_per_thread = scan_channels_per_thread((int)d.dstate);
  pl.dtile = scan_threads(pl.channels_per_thread) * pl.channels_per_thread;
  pl.dtiles = (int)std::max<int64_t>(1, (d.dim + pl.dtile - 1) / pl.dtile);
  const int64_t tiles = std::max<int64_t>(1, (d.seqlen + T - 1) / T);
  const int64_t cols = std::max<int64_t>(1, d.batch * pl.dtiles);
  long per_sm = env_long("SSM_SCAN_CTAS_PER_SM", 0);
  if (per_sm <= 0) per_sm = std::max(1, scan_ctas_per_sm((int)d.dstate, d.io == SSM_DTYPE_BF16));
  int64_t nseg = std::max<int64_t>(1, (int64_t)device_sms() * per_sm / cols);
  const long forced = env_long("SSM_SCAN_SEGMENTS", 0);
  if (forced > 0) nseg = forced;
  nseg = std::min<int64_t>(std::min<int64_t>(nseg, tiles), 65535);
  const int64_t tiles_per_seg = (tiles + nseg - 1) / nseg;
  pl.seg_steps = (int)(tiles_per_seg * T);
  pl.nseg = (int)((tiles + tiles_per_seg - 1) / tiles_per_seg);
  pl.ctas_agg = pl.nseg > 1 ? (int)(d.batch * (pl.nseg - 1) * pl.dtiles) : 0;
  pl.ctas_main = (int)(d.batch * pl.nseg * pl.dtiles);
  size_t off = 0;
  pl.off_status = off;
  off = align_up(off + sizeof(int) * (size_t)(pl.ctas_agg + pl.ctas_main), 256);
  const size_t nagg = (size_t)(pl.nseg - 1);
  pl.off_state = off;
  off = align_up(off + sizeof(float) * (size_t)d.batch * nagg * d.dstate * d.dim, 256);
  pl.off_sum = off;
  off = align_up(off + sizeof(float) * (size_t)d.batch * nagg * d.dim, 256);
  pl.off_h0 = off;
  if (pl.nseg > 1) off = align_up(off + sizeof(float) * (size_t)d.batch * d.dim * d.dstate, 256);
  pl.bytes = off;
  return pl;
}

// Split of the backward pass: enough (segment, channel block, batch row) CTAs
// for about 16 resident carry-pass CTAs per SM, segments of at least 8 tiles
// of 4 steps; the workspace layout follows BwdParams.
int bwd_dims_status(const Dims& d) {
  if (d.io != SSM_DTYPE_F32 && d.io != SSM_DTYPE_BF16) return SSM_ERR_UNSUPPORTED;
  if (d.batch < 0 || d.seqlen < 0 || d.dim < 0 || d.dstate <= 0) return SSM_ERR_INVALID_ARG;
  if (!scan_bwd_dstate_supported((int)std::min<int64_t>(d.dstate, 1 << 20)))
    return SSM_ERR_UNSUPPORTED;
  if (d.batch > 65535 || d.dim > (1 << 24) || d.seqlen > (1 << 30)) return SSM_ERR_UNSUPPORTED;
  if (too_large({d.batch, d.seqlen, d.dim}) || too_large({d.batch, d.seqlen, d.dstate}) ||
      too_large({d.batch, d.dim, d.dstate}))
    return SSM_ERR_UNSUPPORTED;
  return SSM_OK;
}

BwdPlan make_bwd_plan(const Dims& d) {
  BwdPlan pl{};
  const int T = kBwdTileSteps;
  pl.dblocks = (int)std::max<int64_t>(1, (d.dim + kBwdThreads - 1) / kBwdThreads);
  const int64_t tiles = std::max<int64_t>(1, (d.seqlen + T - 1) / T);
  pl.ntiles = (int)tiles;
  const int64_t cols = std::max<int64_t>(1, d.batch * pl.dblocks);
  int64_t nseg = std::max<int64_t>(1, ((int64_t)device_sms() * 16 + cols - 1) / cols);
  nseg = std::min<int64_t>(nseg, std::max<int64_t>(1, tiles / 8));
  const long forced = env_long("SSM_SCAN_BWD_SEGMENTS", 0);
  if (forced > 0) nseg = forced;
  nseg = std::min<int64_t>(std::min<int64_t>(nseg, tiles), 65535);
  const int64_t tiles_per_seg = (tiles + nseg - 1) / nseg;
  pl.seg_steps = (int)(tiles_per_seg * T);
  pl.nseg = (int)((tiles + tiles_per_seg - 1) / tiles_per_seg);
  const size_t B = (size_t)d.batch, N = (size_t)d.dstate, Dm = (size_t)d.dim;
  const size_t S = (size_t)pl.nseg, L = (size_t)std::max<int64_t>(d.seqlen, 0);
  size_t off = 0;
  auto take = [&](size_t floats) {
    const size_t at = off;
    off = align_up(off + sizeof(float) * floats, 256);
    return at;
  };
  pl.off_ck = take(B * tiles * N * Dm);
  pl.off_qk = take(B * tiles * Dm);
  pl.off_hloc = take(B * S * N * Dm);
  pl.off_mloc = take(B * S * N * Dm);
  pl.off_hin = take(B * S * N * Dm);
  pl.off_muin = take(B * S * N * Dm);
  pl.off_qseg = take(B * S * Dm);
  pl.off_dbc = take(B * pl.dblocks * L * 2 * N);
  pl.off_dA = take(B * S * N * Dm);
  pl.off_dD = take(B * S * Dm);
  pl.off_dbias = take(B * S * Dm);
  pl.bytes = off;
  return pl;
}

// --- TMA tensor maps --------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 3-D map over a (batch, rows, cols) row-major tensor with a box of
// (1, box_rows, box_cols); out-of-range elements read as zero.
bool encode_3d(CUtensorMap* map, const void* base, int io, int64_t batch, int64_t rows,
               int64_t cols, int box_rows, int box_cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const size_t es = io_bytes(io);
  const cuuint64_t gdim[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batch};
  const cuuint64_t gstride[2] = {(cuuint64_t)(cols * es), (cuuint64_t)(rows * cols * es)};
  const cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  const CUtensorMapDataType dt =
      io == SSM_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const CUresult r = fn(map, dt, 3, const_cast<void*>(base), gdim, gstride, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    snprintf(g_detail, sizeof g_detail,
             "cuTensorMapEncodeTiled failed (CUresult %d) for dims (%lld, %lld, %lld) box (%d, %d)",
             (int)r, (long long)cols, (long long)rows, (long long)batch, box_cols, box_rows);
  return r == CUDA_SUCCESS;
}

// Tiled map of a bf16 tensor with the 128-byte swizzle (rank dims, innermost
// first; strides in bytes of dims 1..rank-1); box rows of 64 elements.
bool encode_sw128_bf16(CUtensorMap* map, const void* base, int rank, const cuuint64_t* gdim,
                       const cuuint64_t* gstride, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint32_t estride[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                        const_cast<void*>(base), gdim, gstride, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    snprintf(g_detail, sizeof g_detail, "cuTensorMapEncodeTiled (128-byte swizzle) failed: %d",
             (int)r);
  return r == CUDA_SUCCESS;
}

// TMA needs 16-byte aligned bases and 16-byte multiples for row strides.
bool tma_eligible(const Dims& d, const void* x, const void* delta, const void* z, const void* B,
                  const void* C) {
  if (env_long("SSM_SCAN_DISABLE_TMA", 0) != 0) return false;
  const size_t es = io_bytes(d.io);
  if ((d.dim * es) % 16 != 0 || (d.dstate * es) % 16 != 0) return false;
  if (!aligned(x, 16) || !aligned(delta, 16) || !aligned(B, 16) || !aligned(C, 16)) return false;
  if (z && !aligned(z, 16)) return false;
  if (d.seqlen <= 0 || d.dim <= 0 || d.batch <= 0) return false;
  return encode_fn() != nullptr;
}

int fail(int code, const char* what, cudaError_t e = cudaSuccess) {
  if (e != cudaSuccess)
    snprintf(g_detail, sizeof g_detail, "%s: %s (%s)", what, cudaGetErrorString(e),
             cudaGetErrorName(e));
  else
    snprintf(g_detail, sizeof g_detail, "%s", what);
  return code;
}

int cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return SSM_OK;
  return fail(SSM_ERR_CUDA, what, e);
}

}  // namespace
}  // namespace ssm

using namespace ssm;

extern "C" {

int ssm_scan_version(void) { return kVersion; }

const char* ssm_last_error_detail(void) { return g_detail; }

const char* ssm_status_string(int status) {
  switch (status) {
    case SSM_OK: return "ok";
    case SSM_ERR_INVALID_ARG: return "invalid argument";
    case SSM_ERR_UNSUPPORTED: return "unsupported size or dtype";
    case SSM_ERR_WORKSPACE: return "workspace missing or too small";
    case SSM_ERR_CUDA: return "CUDA error";
    case SSM_ERR_TIMEOUT: return "a kernel wait timed out";
    default: return "unknown status";
  }
}

int ssm_scan_plan(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int io_dtype,
                  ssm_scan_plan_t* out) {
  const Dims d{batch, seqlen, dim, dstate, io_dtype};
  const int st = dims_status(d);
  if (st != SSM_OK) return st;
  if (!out) return SSM_ERR_INVALID_ARG;
  const ScanPlan pl = make_plan(d);
  out->segments = pl.nseg;
  out->segment_steps = pl.seg_steps;
  out->channel_tiles = pl.dtiles;
  out->channels_per_cta = pl.dtile;
  out->ctas_carry = pl.ctas_agg;
  out->ctas_main = pl.ctas_main;
  out->kernels = (batch > 0 && dim > 0) ? (pl.nseg > kScanPrologueCompose ? 3 : pl.nseg > 1 ? 2 : 1) : 0;
  out->workspace_bytes = (int64_t)pl.bytes;
  return SSM_OK;
}

size_t ssm_scan_workspace_bytes(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                                int io_dtype) {
  const Dims d{batch, seqlen, dim, dstate, io_dtype};
  if (dims_status(d) != SSM_OK) return 0;
  return make_plan(d).bytes;
}

static int scan_fwd_impl(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                         int io_dtype, const void* x, const void* delta, const float* A,
                         const void* B, const void* C, const float* D, const void* z,
                         const float* delta_bias, int softplus, const float* h0, void* y,
                         float* h_last, void* workspace, size_t workspace_bytes, void* stream,
                         bool zoh);

int ssm_scan_fwd(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int io_dtype,
                 const void* x, const void* delta, const float* A, const void* B,
                 const void* C, const float* D, const void* z, const float* delta_bias,
                 int softplus, const float* h0, void* y, float* h_last, void* workspace,
                 size_t workspace_bytes, void* stream) {
  return scan_fwd_impl(batch, seqlen, dim, dstate, io_dtype, x, delta, A, B, C, D, z, delta_bias,
                       softplus, h0, y, h_last, workspace, workspace_bytes, stream, false);
}

int ssm_scan_fwd_zoh(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int io_dtype,
                     const void* x, const void* delta, const float* A, const void* B,
                     const void* C, const float* D, const void* z, const float* delta_bias,
                     int softplus, const float* h0, void* y, float* h_last, void* workspace,
                     size_t workspace_bytes, void* stream) {
  return scan_fwd_impl(batch, seqlen, dim, dstate, io_dtype, x, delta, A, B, C, D, z, delta_bias,
                       softplus, h0, y, h_last, workspace, workspace_bytes, stream, true);
}

static int scan_fwd_impl(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                         int io_dtype, const void* x, const void* delta, const float* A,
                         const void* B, const void* C, const float* D, const void* z,
                         const float* delta_bias, int softplus, const float* h0, void* y,
                         float* h_last, void* workspace, size_t workspace_bytes, void* stream,
                         bool zoh) {
  const Dims d{batch, seqlen, dim, dstate, io_dtype};
  int st = dims_status(d);
  if (st != SSM_OK) return st;
  if (batch == 0 || dim == 0) return SSM_OK;
  const size_t es = io_bytes(io_dtype);
  const size_t n_bld = (size_t)batch * seqlen * dim, n_bln = (size_t)batch * seqlen * dstate;
  // required pointers and element alignment
  if (!A) return SSM_ERR_INVALID_ARG;
  // y may be NULL when h_last is wanted alone (the state after the sequence)
  if (seqlen > 0 && (!x || !delta || !B || !C || (!y && !h_last))) return SSM_ERR_INVALID_ARG;
  const void* io_ptrs[] = {x, delta, B, C, z, y};
  for (const void* p : io_ptrs)
    if (p && !aligned(p, es)) return SSM_ERR_INVALID_ARG;
  const void* f32_ptrs[] = {A, D, delta_bias};
  for (const void* p : f32_ptrs)
    if (p && !aligned(p, 4)) return SSM_ERR_INVALID_ARG;
  if ((h0 && !aligned(h0, 8)) || (h_last && !aligned(h_last, 8))) return SSM_ERR_INVALID_ARG;
  if (!aligned(A, 8)) return SSM_ERR_INVALID_ARG;  // rows of A are read as pairs
  // y must not overlap an input
  const size_t by = n_bld * es;
  if (overlap(y, by, x, n_bld * es) || overlap(y, by, delta, n_bld * es) ||
      overlap(y, by, z, n_bld * es) || overlap(y, by, B, n_bln * es) ||
      overlap(y, by, C, n_bln * es))
    return SSM_ERR_INVALID_ARG;
  const ScanPlan pl = make_plan(d);
  if (pl.bytes > 0 && (!workspace || workspace_bytes < pl.bytes || !aligned(workspace, 16)))
    return SSM_ERR_WORKSPACE;

  ScanParams p{};
  p.batch = (int)batch;
  p.seqlen = (int)seqlen;
  p.dim = (int)dim;
  p.nseg = pl.nseg;
  p.seg_steps = pl.seg_steps;
  p.softplus = softplus ? 1 : 0;
  p.x = x; p.delta = delta; p.z = z; p.B = B; p.C = C;
  p.A = A; p.D = D; p.bias = delta_bias; p.h0 = h0;
  p.y = y; p.h_last = h_last;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.status = reinterpret_cast<int*>(ws + pl.off_status);
  p.ws_state = reinterpret_cast<float*>(ws + pl.off_state);
  p.ws_sum = reinterpret_cast<float*>(ws + pl.off_sum);
  p.ws_h0 = reinterpret_cast<float*>(ws + pl.off_h0);
  p.wait_limit_ns = (uint64_t)std::max(1L, env_long("SSM_SCAN_WAIT_LIMIT_NS",
                                                    (long)kDefaultWaitLimitNs));
  p.test_stall = env_long("SSM_SCAN_TEST_STALL", 0) != 0 ? 1 : 0;

  const bool use_tma = tma_eligible(d, x, delta, z, B, C);
  ScanMaps maps;
  memset(&maps, 0, sizeof maps);
  if (use_tma) {
    const int T = kScanTileSteps, DT = pl.dtile;
    bool ok = encode_3d(&maps.x, x, io_dtype, batch, seqlen, dim, T, DT) &&
              encode_3d(&maps.delta, delta, io_dtype, batch, seqlen, dim, T, DT) &&
              encode_3d(&maps.B, B, io_dtype, batch, seqlen, dstate, T, (int)dstate) &&
              encode_3d(&maps.C, C, io_dtype, batch, seqlen, dstate, T, (int)dstate);
    if (ok && z) ok = encode_3d(&maps.z, z, io_dtype, batch, seqlen, dim, T, DT);
    if (!ok) return SSM_ERR_CUDA;
  }
  st = cuda_status(launch_scan(pl, p, use_tma ? &maps : nullptr, use_tma, (int)dstate,
                               io_dtype == SSM_DTYPE_BF16, zoh, static_cast<cudaStream_t>(stream)),
                   use_tma ? "scan launch (TMA path)" : "scan launch (plain-load path)");
  return st;
}

int ssm_scan_status(const void* workspace, size_t workspace_bytes, int64_t batch,
                    int64_t seqlen, int64_t dim, int64_t dstate, int io_dtype, void* stream) {
  const Dims d{batch, seqlen, dim, dstate, io_dtype};
  int st = dims_status(d);
  if (st != SSM_OK) return st;
  if (batch == 0 || dim == 0) return SSM_OK;
  const ScanPlan pl = make_plan(d);
  if (!workspace || workspace_bytes < pl.bytes) return SSM_ERR_WORKSPACE;
  const int n = pl.ctas_agg + pl.ctas_main;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SSM_ERR_CUDA, "ssm_scan_status: stream synchronize", e);
  int buf[1024];
  const unsigned char* ws = static_cast<const unsigned char*>(workspace) + pl.off_status;
  for (int i = 0; i < n; i += 1024) {
    const int m = std::min(1024, n - i);
    e = cudaMemcpy(buf, ws + sizeof(int) * (size_t)i, sizeof(int) * (size_t)m,
                   cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(SSM_ERR_CUDA, "ssm_scan_status: read status", e);
    for (int k = 0; k < m; ++k)
      if (buf[k] != kCtaOk) return fail(SSM_ERR_TIMEOUT, "a CTA's bounded wait timed out");
  }
  return SSM_OK;
}

static int state_update_impl(int64_t batch, int64_t dim, int64_t dstate, int io_dtype,
                             float* state, const void* x, const void* delta, const float* A,
                             const void* B, const void* C, const float* D, const void* z,
                             const float* delta_bias, int softplus, void* y, void* stream,
                             bool zoh);

int ssm_state_update(int64_t batch, int64_t dim, int64_t dstate, int io_dtype, float* state,
                     const void* x, const void* delta, const float* A, const void* B,
                     const void* C, const float* D, const void* z, const float* delta_bias,
                     int softplus, void* y, void* stream) {
  return state_update_impl(batch, dim, dstate, io_dtype, state, x, delta, A, B, C, D, z,
                           delta_bias, softplus, y, stream, false);
}

int ssm_state_update_zoh(int64_t batch, int64_t dim, int64_t dstate, int io_dtype, float* state,
                         const void* x, const void* delta, const float* A, const void* B,
                         const void* C, const float* D, const void* z, const float* delta_bias,
                         int softplus, void* y, void* stream) {
  return state_update_impl(batch, dim, dstate, io_dtype, state, x, delta, A, B, C, D, z,
                           delta_bias, softplus, y, stream, true);
}

static int state_update_impl(int64_t batch, int64_t dim, int64_t dstate, int io_dtype,
                             float* state, const void* x, const void* delta, const float* A,
                             const void* B, const void* C, const float* D, const void* z,
                             const float* delta_bias, int softplus, void* y, void* stream,
                             bool zoh) {
  const Dims d{batch, 1, dim, dstate, io_dtype};
  int st = dims_status(d);
  if (st != SSM_OK) return st;
  if (batch == 0 || dim == 0) return SSM_OK;
  if (!state || !x || !delta || !A || !B || !C || !y) return SSM_ERR_INVALID_ARG;
  const size_t es = io_bytes(io_dtype);
  const void* io_ptrs[] = {x, delta, B, C, z, y};
  for (const void* p : io_ptrs)
    if (p && !aligned(p, es)) return SSM_ERR_INVALID_ARG;
  const void* f32_ptrs[] = {A, D, delta_bias};
  for (const void* p : f32_ptrs)
    if (p && !aligned(p, 4)) return SSM_ERR_INVALID_ARG;
  if (!aligned(state, dstate % 4 == 0 ? 16 : 8)) return SSM_ERR_INVALID_ARG;
  // the kernel reads B, C in pairs of elements and rows of A as vectors
  const size_t bc_align = (dstate % 4 == 0 ? 4 : 2) * es;
  if (!aligned(B, bc_align) || !aligned(C, bc_align)) return SSM_ERR_INVALID_ARG;
  if (!aligned(A, dstate % 4 == 0 ? 16 : 8)) return SSM_ERR_INVALID_ARG;
  const size_t nbd = (size_t)batch * dim, nbn = (size_t)batch * dstate;
  const size_t by = nbd * es;
  if (overlap(y, by, x, nbd * es) || overlap(y, by, delta, nbd * es) ||
      overlap(y, by, z, nbd * es) || overlap(y, by, B, nbn * es) || overlap(y, by, C, nbn * es) ||
      overlap(y, by, state, nbd * dstate * sizeof(float)))
    return SSM_ERR_INVALID_ARG;
  DecodeParams p{};
  p.batch = (int)batch;
  p.dim = (int)dim;
  p.softplus = softplus ? 1 : 0;
  p.state = state;
  p.x = x; p.delta = delta; p.z = z; p.B = B; p.C = C;
  p.A = A; p.D = D; p.bias = delta_bias; p.y = y;
  return cuda_status(launch_decode(p, (int)dstate, io_dtype == SSM_DTYPE_BF16, zoh,
                                   static_cast<cudaStream_t>(stream)),
                     "decode launch");
}

size_t ssm_scan_bwd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                                    int io_dtype) {
  const Dims d{batch, seqlen, dim, dstate, io_dtype};
  if (bwd_dims_status(d) != SSM_OK) return 0;
  if (batch == 0 || dim == 0 || seqlen == 0) return 0;
  return make_bwd_plan(d).bytes;
}

int ssm_scan_bwd(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int io_dtype,
                 const void* x, const void* delta, const float* A, const void* B,
                 const void* C, const float* D, const void* z, const float* delta_bias,
                 int softplus, const float* h0, const void* dy, const float* dh_last,
                 void* dx, void* ddelta, float* dA, float* dB, float* dC, float* dD, void* dz,
                 float* ddelta_bias, float* dh0, void* workspace, size_t workspace_bytes,
                 void* stream) {
  const Dims d{batch, seqlen, dim, dstate, io_dtype};
  int st = bwd_dims_status(d);
  if (st != SSM_OK) return st;
  if (batch == 0 || dim == 0) return SSM_OK;
  if (!A || !dA || (!z) != (!dz)) return SSM_ERR_INVALID_ARG;
  if (seqlen > 0 && (!x || !delta || !B || !C || !dy || !dx || !ddelta || !dB || !dC))
    return SSM_ERR_INVALID_ARG;
  const size_t es = io_bytes(io_dtype);
  const void* io_ptrs[] = {x, delta, B, C, z, dy, dx, ddelta, dz};
  for (const void* p : io_ptrs)
    if (p && !aligned(p, es)) return SSM_ERR_INVALID_ARG;
  const void* f32_ptrs[] = {A, D, delta_bias, h0, dh_last, dA, dB, dC, dD, ddelta_bias, dh0};
  for (const void* p : f32_ptrs)
    if (p && !aligned(p, 4)) return SSM_ERR_INVALID_ARG;
  if (!aligned(A, 8)) return SSM_ERR_INVALID_ARG;  // rows of A are read as pairs
  // no output may overlap an input or another output
  const size_t n_bld = (size_t)batch * seqlen * dim, n_bln = (size_t)batch * seqlen * dstate;
  const size_t n_bdn = (size_t)batch * dim * dstate, n_dn = (size_t)dim * dstate;
  struct Span {
    const void* p;
    size_t bytes;
  };
  const Span ins[] = {{x, n_bld * es},      {delta, n_bld * es}, {z, n_bld * es},
                      {dy, n_bld * es},     {B, n_bln * es},     {C, n_bln * es},
                      {A, n_dn * 4},        {D, (size_t)dim * 4}, {delta_bias, (size_t)dim * 4},
                      {h0, n_bdn * 4},      {dh_last, n_bdn * 4}};
  const Span outs[] = {{dx, n_bld * es},  {ddelta, n_bld * es}, {dz, n_bld * es},
                       {dA, n_dn * 4},    {dB, n_bln * 4},      {dC, n_bln * 4},
                       {dD, (size_t)dim * 4}, {ddelta_bias, (size_t)dim * 4}, {dh0, n_bdn * 4}};
  for (size_t i = 0; i < sizeof outs / sizeof outs[0]; ++i) {
    for (const Span& in : ins)
      if (overlap(outs[i].p, outs[i].bytes, in.p, in.bytes))
        return fail(SSM_ERR_INVALID_ARG, "ssm_scan_bwd: an output overlaps an input");
    for (size_t j = i + 1; j < sizeof outs / sizeof outs[0]; ++j)
      if (overlap(outs[i].p, outs[i].bytes, outs[j].p, outs[j].bytes))
        return fail(SSM_ERR_INVALID_ARG, "ssm_scan_bwd: two outputs overlap");
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (seqlen == 0) {
    // no steps: h_last = h0, so dh0 = dh_last; every other gradient is zero
    cudaError_t e = cudaMemsetAsync(dA, 0, n_dn * 4, s);
    if (e == cudaSuccess && dD) e = cudaMemsetAsync(dD, 0, (size_t)dim * 4, s);
    if (e == cudaSuccess && ddelta_bias) e = cudaMemsetAsync(ddelta_bias, 0, (size_t)dim * 4, s);
    if (e == cudaSuccess && dh0)
      e = dh_last ? cudaMemcpyAsync(dh0, dh_last, n_bdn * 4, cudaMemcpyDeviceToDevice, s)
                  : cudaMemsetAsync(dh0, 0, n_bdn * 4, s);
    return cuda_status(e, "ssm_scan_bwd: empty sequence");
  }
  const BwdPlan pl = make_bwd_plan(d);
  if (!workspace || workspace_bytes < pl.bytes || !aligned(workspace, 16))
    return fail(SSM_ERR_WORKSPACE, "ssm_scan_bwd: workspace missing, too small or unaligned");

  BwdParams p{};
  p.batch = (int)batch;
  p.seqlen = (int)seqlen;
  p.dim = (int)dim;
  p.nseg = pl.nseg;
  p.seg_steps = pl.seg_steps;
  p.dblocks = pl.dblocks;
  p.ntiles = pl.ntiles;
  p.softplus = softplus ? 1 : 0;
  p.scal_pairs = (io_dtype == SSM_DTYPE_BF16 && dim % 2 == 0 && aligned(x, 4) &&
                  aligned(delta, 4) && aligned(dy, 4) && (!z || aligned(z, 4)))
                     ? 1
                     : 0;
  p.x = x; p.delta = delta; p.z = z; p.B = B; p.C = C;
  p.A = A; p.D = D; p.bias = delta_bias; p.h0 = h0;
  p.dy = dy; p.dh_last = dh_last;
  p.dx = dx; p.ddelta = ddelta; p.dz = dz;
  p.dA = dA; p.dB = dB; p.dC = dC; p.dD = dD; p.dbias = ddelta_bias; p.dh0 = dh0;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.ws_ck = reinterpret_cast<float*>(ws + pl.off_ck);
  p.ws_qk = reinterpret_cast<float*>(ws + pl.off_qk);
  p.ws_hloc = reinterpret_cast<float*>(ws + pl.off_hloc);
  p.ws_mloc = reinterpret_cast<float*>(ws + pl.off_mloc);
  p.ws_hin = reinterpret_cast<float*>(ws + pl.off_hin);
  p.ws_muin = reinterpret_cast<float*>(ws + pl.off_muin);
  p.ws_qseg = reinterpret_cast<float*>(ws + pl.off_qseg);
  p.ws_dbc = reinterpret_cast<float*>(ws + pl.off_dbc);
  p.ws_dA = reinterpret_cast<float*>(ws + pl.off_dA);
  p.ws_dD = reinterpret_cast<float*>(ws + pl.off_dD);
  p.ws_dbias = reinterpret_cast<float*>(ws + pl.off_dbias);
  return cuda_status(launch_scan_bwd(p, (int)dstate, io_dtype == SSM_DTYPE_BF16, s),
                     "backward launch");
}

// ---- causal depthwise conv1d + SiLU --------------------------------------

static int conv_check(int64_t batch, int64_t seqlen, int64_t dim, int64_t width, int io_dtype) {
  if (io_dtype != SSM_DTYPE_F32 && io_dtype != SSM_DTYPE_BF16) return SSM_ERR_UNSUPPORTED;
  if (batch < 0 || seqlen < 0 || dim < 0 || width < 1) return SSM_ERR_INVALID_ARG;
  if (!conv_width_supported((int)std::min<int64_t>(width, 1 << 20))) return SSM_ERR_UNSUPPORTED;
  if (batch > 65535 || dim > (1 << 24) || seqlen > (1 << 30)) return SSM_ERR_UNSUPPORTED;
  if (too_large({batch, seqlen, dim})) return SSM_ERR_UNSUPPORTED;
  return SSM_OK;
}

static bool conv_vec(int64_t dim, int io_dtype, std::initializer_list<const void*> ptrs) {
  const int64_t vec = io_dtype == SSM_DTYPE_BF16 ? 4 : 2;
  if (dim % vec != 0) return false;
  for (const void* p : ptrs)
    if (p && !aligned(p, 8)) return false;
  return true;
}

// Steps per CTA along the sequence (SSM_CONV_CHUNK overrides, 8 .. 4096).
static int conv_chunk(bool backward) {
  return (int)std::max(8L, std::min(4096L, env_long("SSM_CONV_CHUNK",
                                                    backward ? kConvChunkBwd : kConvChunkFwd)));
}

static ConvParams conv_params(int64_t batch, int64_t seqlen, int64_t dim, int64_t width,
                              int silu, bool backward) {
  ConvParams p{};
  p.batch = (int)batch;
  p.seqlen = (int)seqlen;
  p.dim = (int)dim;
  p.width = (int)width;
  p.chunk = conv_chunk(backward);
  p.silu = silu ? 1 : 0;
  p.w_vec = 0;
  return p;
}

int ssm_conv1d_silu_fwd(int64_t batch, int64_t seqlen, int64_t dim, int64_t width, int io_dtype,
                        const void* x, const float* w, const float* bias, int silu, void* out,
                        void* stream) {
  int st = conv_check(batch, seqlen, dim, width, io_dtype);
  if (st != SSM_OK) return st;
  if (batch == 0 || dim == 0 || seqlen == 0) return SSM_OK;
  if (!x || !w || !out) return SSM_ERR_INVALID_ARG;
  const size_t es = io_bytes(io_dtype), n = (size_t)batch * seqlen * dim;
  if (!aligned(x, es) || !aligned(out, es) || !aligned(w, 4) || (bias && !aligned(bias, 4)))
    return SSM_ERR_INVALID_ARG;
  if (overlap(out, n * es, x, n * es) || overlap(out, n * es, w, (size_t)dim * width * 4) ||
      overlap(out, n * es, bias, (size_t)dim * 4))
    return fail(SSM_ERR_INVALID_ARG, "ssm_conv1d_silu_fwd: out overlaps an input");
  ConvParams p = conv_params(batch, seqlen, dim, width, silu, false);
  p.x = x; p.w = w; p.bias = bias; p.out = out;
  p.w_vec = aligned(w, 16) ? 1 : 0;
  return cuda_status(launch_conv(p, io_dtype == SSM_DTYPE_BF16, conv_vec(dim, io_dtype, {x, out}),
                                 false, static_cast<cudaStream_t>(stream)),
                     "conv1d forward launch");
}

int ssm_conv1d_silu_update(int64_t batch, int64_t dim, int64_t width, int io_dtype,
                           void* conv_state, const void* x, const float* w, const float* bias,
                           int silu, void* out, void* stream) {
  int st = conv_check(batch, 1, dim, width, io_dtype);
  if (st != SSM_OK) return st;
  if (batch == 0 || dim == 0) return SSM_OK;
  if (!conv_state || !x || !w || !out) return SSM_ERR_INVALID_ARG;
  const size_t es = io_bytes(io_dtype), n = (size_t)batch * dim;
  if (!aligned(conv_state, es) || !aligned(x, es) || !aligned(out, es) || !aligned(w, 4) ||
      (bias && !aligned(bias, 4)))
    return SSM_ERR_INVALID_ARG;
  const size_t bs = n * (size_t)(width - 1) * es;
  if (overlap(out, n * es, conv_state, bs) || overlap(out, n * es, x, n * es) ||
      overlap(conv_state, bs, x, n * es) || overlap(out, n * es, w, (size_t)dim * width * 4) ||
      overlap(conv_state, bs, w, (size_t)dim * width * 4))
    return fail(SSM_ERR_INVALID_ARG, "ssm_conv1d_silu_update: buffers overlap");
  ConvParams p = conv_params(batch, 1, dim, width, silu, false);
  p.x = x; p.w = w; p.bias = bias; p.out = conv_state; p.dx = out;
  return cuda_status(launch_conv_update(p, io_dtype == SSM_DTYPE_BF16,
                                        static_cast<cudaStream_t>(stream)),
                     "conv1d update launch");
}

int ssm_ssd_scan_fwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                     int64_t dstate, int io_dtype, const void* x, const void* dt, const float* A,
                     const void* B, const void* C, const float* D, const float* dt_bias,
                     int softplus, const float* h0, void* y, float* h_last, void* stream) {
  if (io_dtype != SSM_DTYPE_F32 && io_dtype != SSM_DTYPE_BF16) return SSM_ERR_INVALID_ARG;
  if (batch < 0 || seqlen < 0 || nheads < 0 || headdim <= 0 || dstate <= 0)
    return SSM_ERR_INVALID_ARG;
  if (io_dtype != SSM_DTYPE_BF16 || headdim != kSsdHeadDim ||
      !ssd_dstate_supported((int)std::min<int64_t>(dstate, 1 << 20)))
    return fail(SSM_ERR_UNSUPPORTED, "ssm_ssd_scan_fwd: bf16 io, headdim 64 and dstate 64, "
                                     "128 or 256 only");
  if (batch > 65535 || nheads > (1 << 20) || seqlen > (1 << 30)) return SSM_ERR_UNSUPPORTED;
  if (too_large({batch, seqlen, nheads, headdim}) || too_large({batch, seqlen, dstate}) ||
      too_large({batch, nheads, headdim, dstate}))
    return SSM_ERR_UNSUPPORTED;
  if (batch == 0 || nheads == 0) return SSM_OK;
  if (!A) return SSM_ERR_INVALID_ARG;
  if (seqlen > 0 && (!x || !dt || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16) ||
      !aligned(dt, 2) || !aligned(A, 4) || (D && !aligned(D, 4)) ||
      (dt_bias && !aligned(dt_bias, 4)) || (h0 && !aligned(h0, 8)) ||
      (h_last && !aligned(h_last, 8)))
    return fail(SSM_ERR_INVALID_ARG, "ssm_ssd_scan_fwd: misaligned pointer");
  const size_t nx = (size_t)batch * seqlen * nheads * headdim * 2;
  const size_t nbc = (size_t)batch * seqlen * dstate * 2;
  const size_t ndt = (size_t)batch * seqlen * nheads * 2;
  const size_t nh = (size_t)batch * nheads * headdim * dstate * 4;
  if (overlap(y, nx, x, nx) || overlap(y, nx, dt, ndt) || overlap(y, nx, B, nbc) ||
      overlap(y, nx, C, nbc) || overlap(y, nx, h_last, nh) || overlap(h_last, nh, x, nx) ||
      overlap(h_last, nh, B, nbc) || overlap(h_last, nh, C, nbc) ||
      (h_last != h0 && overlap(h_last, nh, h0, nh)))
    return fail(SSM_ERR_INVALID_ARG, "ssm_ssd_scan_fwd: buffers overlap");
  SsdParams p{};
  p.batch = (int)batch;
  p.nheads = (int)nheads;
  p.dstate = (int)dstate;
  p.seqlen = seqlen;
  p.softplus = softplus ? 1 : 0;
  p.x = static_cast<const uint16_t*>(x);
  p.dt = static_cast<const uint16_t*>(dt);
  p.B = static_cast<const uint16_t*>(B);
  p.C = static_cast<const uint16_t*>(C);
  p.A = A;
  p.D = D;
  p.dt_bias = dt_bias;
  p.h0 = h0;
  p.y = static_cast<uint16_t*>(y);
  p.h_last = h_last;
  p.wait_limit_ns = (uint64_t)std::max(1L, env_long("SSM_SCAN_WAIT_LIMIT_NS",
                                                    (long)kDefaultWaitLimitNs));
  p.test_stall = env_long("SSM_SSD_TEST_STALL", 0) != 0 ? 1 : 0;
  // The tcgen05 kernel: dstate 64 or 128, an even head count, 16-byte aligned
  // state buffers, 4-byte aligned dt; SSM_SSD_LEGACY=1 keeps the mma.sync kernel.
  const bool tc = seqlen > 0 && ssd_tc_supported((int)dstate, (int)nheads) &&
                  env_long("SSM_SSD_LEGACY", 0) == 0 && aligned(dt, 4) && (!h0 || aligned(h0, 16)) &&
                  (!h_last || aligned(h_last, 16)) && encode_fn() != nullptr;
  if (tc) {
    SsdTcMaps maps;
    memset(&maps, 0, sizeof maps);
    const cuuint64_t xd[4] = {(cuuint64_t)headdim, (cuuint64_t)nheads, (cuuint64_t)seqlen,
                              (cuuint64_t)batch};
    const cuuint64_t xs[3] = {(cuuint64_t)(headdim * 2), (cuuint64_t)(nheads * headdim * 2),
                              (cuuint64_t)(seqlen * nheads * headdim * 2)};
    const cuuint32_t xb[4] = {64, 1, 128, 1};
    const cuuint64_t bd[3] = {(cuuint64_t)dstate, (cuuint64_t)seqlen, (cuuint64_t)batch};
    const cuuint64_t bs[2] = {(cuuint64_t)(dstate * 2), (cuuint64_t)(seqlen * dstate * 2)};
    const cuuint32_t bb[3] = {64, 128, 1};
    if (!encode_sw128_bf16(&maps.x, x, 4, xd, xs, xb) ||
        !encode_sw128_bf16(&maps.B, B, 3, bd, bs, bb) ||
        !encode_sw128_bf16(&maps.C, C, 3, bd, bs, bb) ||
        !encode_sw128_bf16(&maps.y, y, 4, xd, xs, xb))
      return SSM_ERR_CUDA;
    return cuda_status(launch_ssd_tc(p, maps, static_cast<cudaStream_t>(stream)),
                       "ssd scan launch (tcgen05)");
  }
  return cuda_status(launch_ssd_fwd(p, static_cast<cudaStream_t>(stream)), "ssd scan launch");
}

int ssm_ssd_scan_status(void* stream) {
  int v = 0;
  const cudaError_t e = ssd_tc_status(static_cast<cudaStream_t>(stream), &v);
  if (e != cudaSuccess) return fail(SSM_ERR_CUDA, "ssm_ssd_scan_status", e);
  return v ? fail(SSM_ERR_TIMEOUT, "a CTA of the SSD scan gave up a bounded wait") : SSM_OK;
}

int ssm_ssd_state_update(int64_t batch, int64_t nheads, int64_t headdim, int64_t dstate,
                         int io_dtype, float* state, const void* x, const void* dt,
                         const float* A, const void* B, const void* C, const float* D,
                         const float* dt_bias, int softplus, void* y, void* stream) {
  if (io_dtype != SSM_DTYPE_F32 && io_dtype != SSM_DTYPE_BF16) return SSM_ERR_INVALID_ARG;
  if (batch < 0 || nheads < 0 || headdim < 0 || dstate <= 0) return SSM_ERR_INVALID_ARG;
  if (!ssd_decode_dstate_supported((int)std::min<int64_t>(dstate, 1 << 20)))
    return fail(SSM_ERR_UNSUPPORTED, "ssm_ssd_state_update: dstate 32, 64, 128 or 256 only");
  if (batch > (1 << 24) || nheads > (1 << 20) || headdim > (1 << 20) ||
      too_large({batch, nheads, headdim, (int64_t)1 << 14}))  // at most 2^26 state rows
    return SSM_ERR_UNSUPPORTED;
  if (batch == 0 || nheads == 0 || headdim == 0) return SSM_OK;
  if (!state || !x || !dt || !A || !B || !C || !y) return SSM_ERR_INVALID_ARG;
  const size_t es = io_bytes(io_dtype);
  if (!aligned(state, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(x, es) ||
      !aligned(dt, es) || !aligned(y, es) || !aligned(A, 4) || (D && !aligned(D, 4)) ||
      (dt_bias && !aligned(dt_bias, 4)))
    return fail(SSM_ERR_INVALID_ARG, "ssm_ssd_state_update: misaligned pointer");
  const size_t rows = (size_t)batch * nheads * headdim;
  const size_t ns = rows * dstate * 4, nx = rows * es, ndt = (size_t)batch * nheads * es,
               nbc = (size_t)batch * dstate * es;
  if (overlap(y, nx, state, ns) || overlap(y, nx, x, nx) || overlap(y, nx, dt, ndt) ||
      overlap(y, nx, B, nbc) || overlap(y, nx, C, nbc) || overlap(state, ns, x, nx) ||
      overlap(state, ns, dt, ndt) || overlap(state, ns, B, nbc) || overlap(state, ns, C, nbc) ||
      overlap(state, ns, A, (size_t)nheads * 4))
    return fail(SSM_ERR_INVALID_ARG, "ssm_ssd_state_update: buffers overlap");
  SsdDecodeParams p{};
  p.batch = (int)batch;
  p.nheads = (int)nheads;
  p.headdim = (int)headdim;
  p.dstate = (int)dstate;
  p.softplus = softplus ? 1 : 0;
  p.state = state;
  p.x = x;
  p.dt = dt;
  p.B = B;
  p.C = C;
  p.A = A;
  p.D = D;
  p.dt_bias = dt_bias;
  p.y = y;
  return cuda_status(launch_ssd_decode(p, io_dtype == SSM_DTYPE_BF16,
                                       static_cast<cudaStream_t>(stream)),
                     "ssd decode launch");
}

size_t ssm_conv1d_silu_bwd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t dim,
                                           int64_t width, int io_dtype) {
  if (conv_check(batch, seqlen, dim, width, io_dtype) != SSM_OK) return 0;
  const int64_t ch = conv_chunk(true);
  const size_t chunks = (size_t)((seqlen + ch - 1) / ch);
  return align_up(sizeof(float) * (size_t)batch * chunks * dim * width, 256) +
         sizeof(float) * (size_t)batch * chunks * dim;
}

int ssm_conv1d_silu_bwd(int64_t batch, int64_t seqlen, int64_t dim, int64_t width, int io_dtype,
                        const void* x, const float* w, const float* bias, int silu,
                        const void* dout, void* dx, float* dw, float* dbias, void* workspace,
                        size_t workspace_bytes, void* stream) {
  int st = conv_check(batch, seqlen, dim, width, io_dtype);
  if (st != SSM_OK) return st;
  if (batch == 0 || dim == 0) return SSM_OK;
  if (!w) return SSM_ERR_INVALID_ARG;
  if (seqlen > 0 && (!x || !dout || !dx)) return SSM_ERR_INVALID_ARG;
  const size_t es = io_bytes(io_dtype), n = (size_t)batch * seqlen * dim;
  const void* io_ptrs[] = {x, dout, dx};
  for (const void* q : io_ptrs)
    if (q && !aligned(q, es)) return SSM_ERR_INVALID_ARG;
  const void* f_ptrs[] = {w, bias, dw, dbias};
  for (const void* q : f_ptrs)
    if (q && !aligned(q, 4)) return SSM_ERR_INVALID_ARG;
  const size_t bw = (size_t)dim * width * 4, bd = (size_t)dim * 4;
  if (overlap(dx, n * es, x, n * es) || overlap(dx, n * es, dout, n * es) ||
      overlap(dx, n * es, w, bw) || overlap(dx, n * es, bias, bd) || overlap(dw, bw, w, bw) ||
      overlap(dw, bw, bias, bd) || overlap(dbias, bd, w, bw) || overlap(dbias, bd, bias, bd) ||
      overlap(dw, bw, dx, n * es) || overlap(dbias, bd, dx, n * es) || overlap(dw, bw, dbias, bd) ||
      overlap(dw, bw, x, n * es) || overlap(dw, bw, dout, n * es) ||
      overlap(dbias, bd, x, n * es) || overlap(dbias, bd, dout, n * es))
    return fail(SSM_ERR_INVALID_ARG, "ssm_conv1d_silu_bwd: an output overlaps an input");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (seqlen == 0) {
    cudaError_t e = dw ? cudaMemsetAsync(dw, 0, bw, s) : cudaSuccess;
    if (e == cudaSuccess && dbias) e = cudaMemsetAsync(dbias, 0, bd, s);
    return cuda_status(e, "ssm_conv1d_silu_bwd: empty sequence");
  }
  const size_t need = ssm_conv1d_silu_bwd_workspace_bytes(batch, seqlen, dim, width, io_dtype);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 16))
    return fail(SSM_ERR_WORKSPACE, "ssm_conv1d_silu_bwd: workspace missing, too small or unaligned");
  ConvParams p = conv_params(batch, seqlen, dim, width, silu, true);
  p.x = x; p.w = w; p.bias = bias; p.dout = dout; p.dx = dx; p.dw = dw; p.dbias = dbias;
  p.w_vec = aligned(w, 16) ? 1 : 0;
  const size_t chunks = (size_t)((seqlen + p.chunk - 1) / p.chunk);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.ws_dw = reinterpret_cast<float*>(ws);
  p.ws_db = reinterpret_cast<float*>(
      ws + align_up(sizeof(float) * (size_t)batch * chunks * dim * width, 256));
  return cuda_status(launch_conv(p, io_dtype == SSM_DTYPE_BF16,
                                 conv_vec(dim, io_dtype, {x, dout, dx}), true, s),
                     "conv1d backward launch");
}

// ---- one sequence split across ranks ----------------------------------------

int ssm_delta_sum(int64_t batch, int64_t seqlen, int64_t dim, int io_dtype, const void* delta,
                  const float* delta_bias, int softplus, float* dsum, void* stream) {
  if (io_dtype != SSM_DTYPE_F32 && io_dtype != SSM_DTYPE_BF16) return SSM_ERR_UNSUPPORTED;
  if (batch < 0 || seqlen < 0 || dim < 0) return SSM_ERR_INVALID_ARG;
  if (too_large({batch, seqlen, dim})) return SSM_ERR_UNSUPPORTED;
  if (batch == 0 || dim == 0) return SSM_OK;
  if (!dsum || (seqlen > 0 && !delta)) return SSM_ERR_INVALID_ARG;
  const size_t es = io_bytes(io_dtype);
  if ((delta && !aligned(delta, es)) || !aligned(dsum, 4) || (delta_bias && !aligned(delta_bias, 4)))
    return SSM_ERR_INVALID_ARG;
  if (overlap(dsum, (size_t)batch * dim * 4, delta, (size_t)batch * seqlen * dim * es))
    return SSM_ERR_INVALID_ARG;
  SeqParParams p{};
  p.batch = (int)batch;
  p.seqlen = (int)seqlen;
  p.dim = (int)dim;
  p.softplus = softplus ? 1 : 0;
  p.delta = delta;
  p.bias = delta_bias;
  p.dsum = dsum;
  return cuda_status(launch_delta_sum(p, io_dtype == SSM_DTYPE_BF16,
                                      static_cast<cudaStream_t>(stream)),
                     "delta-sum launch");
}

int ssm_compose_carries(int64_t rank, int64_t batch, int64_t dim, int64_t dstate, const float* A,
                        const float* h0, const float* hend_all, const float* dsum_all,
                        float* h_in, void* stream) {
  if (rank < 0 || batch < 0 || dim < 0 || dstate <= 0) return SSM_ERR_INVALID_ARG;
  if (too_large({rank + 1, batch, dim, dstate})) return SSM_ERR_UNSUPPORTED;
  if (batch == 0 || dim == 0) return SSM_OK;
  if (!A || !h_in || (rank > 0 && (!hend_all || !dsum_all))) return SSM_ERR_INVALID_ARG;
  const void* f[] = {A, h0, hend_all, dsum_all, h_in};
  for (const void* q : f)
    if (q && !aligned(q, 4)) return SSM_ERR_INVALID_ARG;
  const size_t state = (size_t)batch * dim * dstate * 4;
  if (overlap(h_in, state, hend_all, (size_t)rank * state) ||
      overlap(h_in, state, dsum_all, (size_t)rank * batch * dim * 4) ||
      overlap(h_in, state, A, (size_t)dim * dstate * 4))
    return SSM_ERR_INVALID_ARG;
  SeqParParams p{};
  p.batch = (int)batch;
  p.dim = (int)dim;
  p.dstate = (int)dstate;
  p.rank = (int)rank;
  p.A = A;
  p.h0 = h0;
  p.hend_all = hend_all;
  p.dsum_all = dsum_all;
  p.h_in = h_in;
  return cuda_status(launch_compose(p, static_cast<cudaStream_t>(stream)), "compose launch");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Entry point for callers that cannot allocate device memory.
//
// Some callers have no way to call cudaMalloc around this library: code that
// runs inside a memory pool or arena it does not own, real-time or embedded
// callers that must not allocate after start-up, and plugins whose host
// framework hands them only the input and output tensors. For them,
// ssm_scan_fwd_noalloc takes its scratch (the per-CTA status words and the
// sequence-segment carries that ssm_scan_fwd keeps in the caller's
// workspace) from one array the library reserves in device memory for
// every GPU that loads it, and calls ssm_scan_fwd with that array as the
// workspace. It allocates nothing.
namespace {

constexpr size_t kNoallocScratchBytes = size_t(16) << 20;  // 16 MiB per GPU
constexpr int kNoallocMaxDevices = 64;

// The reserved scratch. In host code this name is only a stand-in for the
// symbol, not a device address: the address must be looked up with
// cudaGetSymbolAddress on each device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mu;
// Address of the scratch per device, with the context it was looked up in:
// a context that was torn down and created again (cudaDeviceReset) loads the
// module again, and the address is then looked up again.
struct NoallocEntry {
  CUcontext ctx;
  void* ptr;
};
NoallocEntry g_noalloc[kNoallocMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

// Device address of the scratch on the current device, looked up (with the
// device current) the first time this device's context is seen.
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SSM_ERR_CUDA, "ssm_scan_fwd_noalloc: cudaGetDevice", e);
  if (dev < 0 || dev >= kNoallocMaxDevices)
    return fail(SSM_ERR_UNSUPPORTED, "ssm_scan_fwd_noalloc: device index above 63");
  CtxGetCurrentFn ctx_fn = ctx_get_current_fn();
  if (!ctx_fn) return fail(SSM_ERR_CUDA, "ssm_scan_fwd_noalloc: cuCtxGetCurrent unavailable");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  CUcontext ctx = nullptr;
  if (ctx_fn(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  if (!ctx || g_noalloc[dev].ctx != ctx || !g_noalloc[dev].ptr) {
    void* p = nullptr;
    // also makes the device's primary context current when none was
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(SSM_ERR_CUDA, "ssm_scan_fwd_noalloc: cudaGetSymbolAddress of the scratch", e);
    if (ctx_fn(&ctx) != CUDA_SUCCESS || !ctx)
      return fail(SSM_ERR_CUDA, "ssm_scan_fwd_noalloc: no current context");
    g_noalloc[dev].ctx = ctx;
    g_noalloc[dev].ptr = p;
  }
  *out = g_noalloc[dev].ptr;
  return SSM_OK;
}

// Scratch bytes a problem needs, or an error code when it is invalid or does
// not fit the reserved array.
int noalloc_need(const Dims& d, size_t* need) {
  const int st = dims_status(d);
  if (st != SSM_OK) return st;
  *need = make_plan(d).bytes;
  if (*need > kNoallocScratchBytes) {
    snprintf(g_detail, sizeof g_detail,
             "ssm_scan_fwd_noalloc: this problem needs %zu bytes of scratch but the built-in "
             "scratch holds %zu; call ssm_scan_fwd with a workspace instead",
             *need, kNoallocScratchBytes);
    return SSM_ERR_WORKSPACE;
  }
  return SSM_OK;
}

}  // namespace

extern "C" int ssm_scan_fwd_noalloc(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                                    int io_dtype, const void* x, const void* delta,
                                    const float* A, const void* B, const void* C,
                                    const float* D, const void* z, const float* delta_bias,
                                    int softplus, const float* h0, void* y, float* h_last,
                                    void* stream) {
  const Dims d{batch, seqlen, dim, dstate, io_dtype};
  const int st = dims_status(d);
  if (st != SSM_OK) return st;
  if (batch == 0 || dim == 0) return SSM_OK;
  size_t need = 0;
  int rc = noalloc_need(d, &need);
  if (rc != SSM_OK) return rc;
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != SSM_OK) return rc;
  return ssm_scan_fwd(batch, seqlen, dim, dstate, io_dtype, x, delta, A, B, C, D, z, delta_bias,
                      softplus, h0, y, h_last, scratch, kNoallocScratchBytes, stream);
}

// The per-CTA status words of a no-alloc call live in the reserved scratch,
// which its callers cannot name: this reads them there (as ssm_scan_status
// does from a caller's workspace).
extern "C" int ssm_scan_status_noalloc(int64_t batch, int64_t seqlen, int64_t dim,
                                       int64_t dstate, int io_dtype, void* stream) {
  const Dims d{batch, seqlen, dim, dstate, io_dtype};
  const int st = dims_status(d);
  if (st != SSM_OK) return st;
  if (batch == 0 || dim == 0) return SSM_OK;
  size_t need = 0;
  int rc = noalloc_need(d, &need);
  if (rc != SSM_OK) return rc;
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != SSM_OK) return rc;
  return ssm_scan_status(scratch, kNoallocScratchBytes, batch, seqlen, dim, dstate, io_dtype,
                         stream);
}
