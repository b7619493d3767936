// C ABI of libbitlinear.so: argument checks, workspace layout and the
// choice of contraction engine.  Declarations and the contract of each
// entry point are in include/bitlinear.h.
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "../../include/bitlinear.h"
#include "kernels.h"

using namespace bitlinear;

namespace {

constexpr int64_t kMaxMN = int64_t(1) << 23;
constexpr int64_t kMaxK = int64_t(1) << 19;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// Forward workspace: [status | s_x | rowsum | xq | (host staging: x | y)]
struct FwdLayout {
  size_t off_sx, off_rs, off_xq, end_dev, off_xh, off_yh, end_host;
};

FwdLayout fwd_layout(int64_t M, int64_t N, int64_t K) {
  FwdLayout L;
  L.off_sx = 256;
  L.off_rs = align_up(L.off_sx + 4 * size_t(M), 256);
  L.off_xq = align_up(L.off_rs + 4 * size_t(M), 1024);
  L.end_dev = align_up(L.off_xq + size_t(M) * size_t(K), 256);
  L.off_xh = L.end_dev;
  L.off_yh = align_up(L.off_xh + 2 * size_t(M) * size_t(K), 256);
  L.end_host = align_up(L.off_yh + 2 * size_t(M) * size_t(N), 256);
  return L;
}

struct DevInfo {
  int checked = 0;  // 0 unknown, 1 ok, -1 not sm_100
  int sms = 148;
};
DevInfo g_dev[64];

int check_device(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BITLINEAR_ERR_CUDA;
  if (dev < 0 || dev >= 64) return BITLINEAR_ERR_DEVICE;
  DevInfo& d = g_dev[dev];
  if (d.checked == 0) {
    int major = 0, minor = 0, n = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    d.sms = n;
    d.checked = (major == 10 && minor == 0) ? 1 : -1;
  }
  if (sms) *sms = d.sms;
  return d.checked == 1 ? BITLINEAR_OK : BITLINEAR_ERR_DEVICE;
}

}  // namespace

// The current device is a B200 (sm_100): BITLINEAR_OK, BITLINEAR_ERR_DEVICE
// or BITLINEAR_ERR_CUDA.  Used by entry points defined in other files.
int bitlinear::current_device_status() { return check_device(nullptr); }

// Forced-timeout test hook (bitlinear_test_force_timeout): while it is on,
// every launch gets the short main-loop wait limit and one wait on a barrier
// that nothing signals.
static std::atomic<int> g_force_timeout{0};
uint64_t bitlinear::launch_wait_ns() { return g_force_timeout.load() ? kTestWaitLimitNs : kWaitLimitNs; }
int bitlinear::launch_stall() { return g_force_timeout.load() ? 1 : 0; }

namespace {

int check_shape(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || M > kMaxMN || N < 1 || N > kMaxMN || K < 64 || K > kMaxK || (K % 64) != 0)
    return BITLINEAR_ERR_SHAPE;
  return BITLINEAR_OK;
}

int status_of(cudaError_t e) { return e == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA; }

// Shared body of the forward entry points; x is a device pointer.
//
// Decode (M <= 16) is one kernel that quantises x itself.  Prefill is the
// act-quant kernel followed by the tcgen05 GEMM, launched as its
// programmatic dependent so that its launch and weight loads overlap the
// act-quant kernel.  The first kernel is an ordinary stream launch -- every
// earlier write to the packed weights is complete before they are read --
// unless BITLINEAR_WEIGHTS_RESIDENT is set, which lets the forward start
// streaming weights while the previous kernel on the stream finishes.
static_assert(BITLINEAR_MAX_GROUPS == kMaxGroups, "header and kernels agree on the group limit");

struct Groups {
  int n;
  int end[kMaxGroups];
};

Groups single_group(int64_t N) {
  Groups g{};
  g.n = 1;
  g.end[0] = int(N);
  return g;
}

int forward_impl_g(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                   const float* w_scale, const uint16_t* bias, uint16_t* y, int8_t* xq_out, float* sx_out,
                   int32_t* acc_out, float* y32_out, int engine, unsigned flags, void* ws, size_t ws_bytes,
                   cudaStream_t stream, const Groups& grp) {
  (void)ws_bytes;
  int sms = 148;
  int st = check_device(&sms);
  if (st != BITLINEAR_OK) return st;
  const FwdLayout L = fwd_layout(M, N, K);
  char* base = static_cast<char*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  const bool resident = (flags & BITLINEAR_WEIGHTS_RESIDENT) != 0;
  const bool faithful = (flags & BITLINEAR_BF16_FAITHFUL) != 0;
  const bool decode = engine == 1 || (engine == 0 && M <= 16);
  cudaError_t e;
  float* s_x = reinterpret_cast<float*>(base + L.off_sx);
  int32_t* rowsum = reinterpret_cast<int32_t*>(base + L.off_rs);
  int8_t* xq = reinterpret_cast<int8_t*>(base + L.off_xq);
  if (decode) {
    // Above 8 tokens, and at 8 tokens when K spans more than two 4096-k
    // rounds, the activations are quantised once by the act-quant kernel and
    // the GEMV reads int8 x: every CTA of the GEMV needs all of x, and
    // quantising it 148 times over (re-reading bf16 x per round) costs more
    // than the extra launch.  At 2-4 tokens and K = 28672 the act-quant
    // kernel (one CTA per token) took longer than the re-reads.
    const bool pre = M > 8 || (M == 8 && K > 8192);
    if (pre) {
      e = launch_act_quant(x, int(M), int(K), xq, s_x, rowsum, status, resident, stream, faithful);
      if (e != cudaSuccess) return BITLINEAR_ERR_CUDA;
    }
    DecodeArgs d;
    d.x = pre ? nullptr : x;
    d.xq = pre ? xq : nullptr;
    d.s_x = pre ? s_x : nullptr;
    d.rowsum = pre ? rowsum : nullptr;
    d.packed = packed_w;
    d.w_scale = w_scale;
    d.bias = bias;
    d.y = y;
    d.xq_out = xq_out;
    d.sx_out = sx_out;
    d.acc_out = acc_out;
    d.y32_out = y32_out;
    d.status = status;
    d.M = int(M);
    d.N = int(N);
    d.K = int(K);
    d.weights_early = resident ? 1 : 0;
    d.faithful = faithful ? 1 : 0;
    d.ngroups = grp.n;
    for (int g = 0; g < kMaxGroups; ++g) d.group_end[g] = grp.end[g];
    d.wait_ns = launch_wait_ns();
    d.stall = launch_stall();
    if (pre) {
      d.xq_out = nullptr;                          // copied from the workspace below
      d.sx_out = nullptr;
    }
    e = launch_decode(d, sms, stream);
    if (e == cudaSuccess && pre && xq_out)
      e = cudaMemcpyAsync(xq_out, xq, size_t(M) * size_t(K), cudaMemcpyDeviceToDevice, stream);
    if (e == cudaSuccess && pre && sx_out) e = cudaMemcpyAsync(sx_out, s_x, 4 * size_t(M), cudaMemcpyDeviceToDevice, stream);
    return status_of(e);
  }
  e = launch_act_quant(x, int(M), int(K), xq, s_x, rowsum, status, resident, stream, faithful);
  if (e != cudaSuccess) return BITLINEAR_ERR_CUDA;
  ForwardArgs a;
  a.xq = xq;
  a.s_x = s_x;
  a.rowsum = rowsum;
  a.packed = packed_w;
  a.w_scale = w_scale;
  a.bias = bias;
  a.y = y;
  a.acc_out = acc_out;
  a.y32_out = y32_out;
  a.status = status;
  a.M = int(M);
  a.N = int(N);
  a.K = int(K);
  a.pdl = true;
  a.faithful = faithful;
  a.ngroups = grp.n;
  for (int g = 0; g < kMaxGroups; ++g) a.group_end[g] = grp.end[g];
  a.wait_ns = launch_wait_ns();
  a.stall = launch_stall();
  e = launch_gemm_prefill(a, sms, stream);
  if (e != cudaSuccess) return BITLINEAR_ERR_CUDA;
  if (xq_out) e = cudaMemcpyAsync(xq_out, xq, size_t(M) * size_t(K), cudaMemcpyDeviceToDevice, stream);
  if (e == cudaSuccess && sx_out) e = cudaMemcpyAsync(sx_out, s_x, 4 * size_t(M), cudaMemcpyDeviceToDevice, stream);
  return status_of(e);
}

int forward_impl(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                 const float* w_scale, const uint16_t* bias, uint16_t* y, int8_t* xq_out, float* sx_out,
                 int32_t* acc_out, float* y32_out, int engine, unsigned flags, void* ws, size_t ws_bytes,
                 cudaStream_t stream) {
  return forward_impl_g(x, M, K, packed_w, N, w_scale, bias, y, xq_out, sx_out, acc_out, y32_out, engine, flags, ws,
                        ws_bytes, stream, single_group(N));
}

int check_forward_args(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                       const float* w_scale, const uint16_t* bias, uint16_t* y, void* ws, size_t ws_bytes,
                       size_t need, bool host) {
  int st = check_shape(M, N, K);
  if (st != BITLINEAR_OK) return st;
  if (!x || !packed_w || !w_scale || !y) return BITLINEAR_ERR_NULL;
  if ((!host && (misaligned(x) || misaligned(y))) || misaligned(packed_w) || misaligned(w_scale) ||
      misaligned(bias))
    return BITLINEAR_ERR_ALIGN;
  if (!ws || ws_bytes < need) return BITLINEAR_ERR_WORKSPACE;
  if (misaligned(ws)) return BITLINEAR_ERR_ALIGN;
  return BITLINEAR_OK;
}

}  // namespace

extern "C" {

const char* bitlinear_status_string(int status) {
  switch (status) {
    case BITLINEAR_OK: return "BITLINEAR_OK";
    case BITLINEAR_ERR_NULL: return "BITLINEAR_ERR_NULL: a required pointer is NULL";
    case BITLINEAR_ERR_SHAPE: return "BITLINEAR_ERR_SHAPE: bad M, N or K (K must be a positive multiple of 64)";
    case BITLINEAR_ERR_ALIGN: return "BITLINEAR_ERR_ALIGN: a device pointer is not 16-byte aligned";
    case BITLINEAR_ERR_WORKSPACE: return "BITLINEAR_ERR_WORKSPACE: workspace missing or too small";
    case BITLINEAR_ERR_CUDA: return "BITLINEAR_ERR_CUDA: a CUDA call or kernel launch failed";
    case BITLINEAR_ERR_TIMEOUT: return "BITLINEAR_ERR_TIMEOUT: a device-side wait gave up";
    case BITLINEAR_ERR_DEVICE: return "BITLINEAR_ERR_DEVICE: the current GPU is not sm_100 (B200)";
    default: return "BITLINEAR: unknown status";
  }
}

int bitlinear_version(void) { return (1 << 16) | 0; }

size_t bitlinear_packed_bytes(int64_t N, int64_t K) {
  if (N < 1 || K < 64 || (K % 64) != 0) return 0;
  return size_t(N) * size_t(K) / 4;
}

size_t bitlinear_pack_workspace_bytes(int64_t N, int64_t K) {
  (void)N;
  (void)K;
  return kPackWsBytes;
}

size_t bitlinear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (check_shape(M, N, K) != BITLINEAR_OK) return 0;
  return fwd_layout(M, N, K).end_dev;
}

size_t bitlinear_host_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (check_shape(M, N, K) != BITLINEAR_OK) return 0;
  return fwd_layout(M, N, K).end_host;
}

int bitlinear_pack_weights(const float* w, int64_t N, int64_t K, uint8_t* packed, float* w_scale,
                           float* w_mean, void* ws, size_t ws_bytes, void* stream) {
  if (N < 1 || K < 64 || (K % 64) != 0 || N > kMaxMN || K > kMaxK || N * K >= (int64_t(1) << 39))
    return BITLINEAR_ERR_SHAPE;
  if (!w || !packed || !w_scale) return BITLINEAR_ERR_NULL;
  if (misaligned(w) || misaligned(packed) || misaligned(w_scale) || misaligned(w_mean))
    return BITLINEAR_ERR_ALIGN;
  if (!ws || ws_bytes < kPackWsBytes) return BITLINEAR_ERR_WORKSPACE;
  if (misaligned(ws)) return BITLINEAR_ERR_ALIGN;
  int st = check_device(nullptr);
  if (st != BITLINEAR_OK) return st;
  return status_of(launch_pack(w, N, K, packed, w_scale, w_mean, pack_workspace(ws),
                               static_cast<cudaStream_t>(stream)));
}

int bitlinear_quant_act(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* x_scale,
                        int32_t* xq_rowsum, void* stream) {
  if (M < 0 || M > kMaxMN || K < 64 || K > kMaxK || (K % 64) != 0) return BITLINEAR_ERR_SHAPE;
  if (M == 0) return BITLINEAR_OK;
  if (!x || !xq || !x_scale) return BITLINEAR_ERR_NULL;
  if (misaligned(x) || misaligned(xq) || misaligned(x_scale) || misaligned(xq_rowsum))
    return BITLINEAR_ERR_ALIGN;
  int st = check_device(nullptr);
  if (st != BITLINEAR_OK) return st;
  return status_of(launch_act_quant(x, int(M), int(K), xq, x_scale, xq_rowsum, nullptr, false,
                                    static_cast<cudaStream_t>(stream)));
}

int bitlinear_forward(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                      const float* w_scale, const uint16_t* bias, uint16_t* y, void* ws, size_t ws_bytes,
                      void* stream) {
  int st = check_forward_args(x, M, K, packed_w, N, w_scale, bias, y, ws, ws_bytes,
                              bitlinear_workspace_bytes(M, N, K), false);
  if (st != BITLINEAR_OK) return st;
  if (M == 0) return BITLINEAR_OK;
  return forward_impl(x, M, K, packed_w, N, w_scale, bias, y, nullptr, nullptr, nullptr, nullptr, 0, 0u, ws,
                      ws_bytes, static_cast<cudaStream_t>(stream));
}

int bitlinear_forward_ex(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                         const float* w_scale, const uint16_t* bias, uint16_t* y, unsigned flags, void* ws,
                         size_t ws_bytes, void* stream) {
  if (flags & ~static_cast<unsigned>(BITLINEAR_WEIGHTS_RESIDENT | BITLINEAR_BF16_FAITHFUL)) return BITLINEAR_ERR_SHAPE;
  int st = check_forward_args(x, M, K, packed_w, N, w_scale, bias, y, ws, ws_bytes,
                              bitlinear_workspace_bytes(M, N, K), false);
  if (st != BITLINEAR_OK) return st;
  if (M == 0) return BITLINEAR_OK;
  return forward_impl(x, M, K, packed_w, N, w_scale, bias, y, nullptr, nullptr, nullptr, nullptr, 0, flags, ws,
                      ws_bytes, static_cast<cudaStream_t>(stream));
}

int bitlinear_forward_grouped(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w,
                              const int64_t* group_rows, int groups, const float* w_scales, const uint16_t* bias,
                              uint16_t* y, unsigned flags, void* ws, size_t ws_bytes, void* stream) {
  if (flags & ~static_cast<unsigned>(BITLINEAR_WEIGHTS_RESIDENT | BITLINEAR_BF16_FAITHFUL)) return BITLINEAR_ERR_SHAPE;
  if (!group_rows) return BITLINEAR_ERR_NULL;
  if (groups < 1 || groups > BITLINEAR_MAX_GROUPS) return BITLINEAR_ERR_SHAPE;
  Groups grp{};
  grp.n = groups;
  int64_t N = 0;
  for (int g = 0; g < groups; ++g) {
    if (group_rows[g] < 1) return BITLINEAR_ERR_SHAPE;
    N += group_rows[g];
    if (N > kMaxMN) return BITLINEAR_ERR_SHAPE;
    grp.end[g] = int(N);
  }
  int st = check_forward_args(x, M, K, packed_w, N, w_scales, bias, y, ws, ws_bytes,
                              bitlinear_workspace_bytes(M, N, K), false);
  if (st != BITLINEAR_OK) return st;
  if (M == 0) return BITLINEAR_OK;
  return forward_impl_g(x, M, K, packed_w, N, w_scales, bias, y, nullptr, nullptr, nullptr, nullptr, 0, flags, ws,
                        ws_bytes, static_cast<cudaStream_t>(stream), grp);
}

int bitlinear_forward_q8(const int8_t* xq, const float* x_scale, const int32_t* xq_rowsum, int64_t M,
                         int64_t K, const uint8_t* packed_w, int64_t N, const float* w_scale,
                         const uint16_t* bias, uint16_t* y, void* ws, size_t ws_bytes, void* stream) {
  int st = check_shape(M, N, K);
  if (st != BITLINEAR_OK) return st;
  if (!xq || !x_scale || !xq_rowsum || !packed_w || !w_scale || !y) return BITLINEAR_ERR_NULL;
  if (misaligned(xq) || misaligned(x_scale) || misaligned(xq_rowsum) || misaligned(packed_w) ||
      misaligned(w_scale) || misaligned(bias) || misaligned(y))
    return BITLINEAR_ERR_ALIGN;
  if (!ws || ws_bytes < 256) return BITLINEAR_ERR_WORKSPACE;
  if (misaligned(ws)) return BITLINEAR_ERR_ALIGN;
  if (M == 0) return BITLINEAR_OK;
  int sms = 148;
  st = check_device(&sms);
  if (st != BITLINEAR_OK) return st;
  ForwardArgs a;
  a.xq = xq;
  a.s_x = x_scale;
  a.rowsum = xq_rowsum;
  a.packed = packed_w;
  a.w_scale = w_scale;
  a.bias = bias;
  a.y = y;
  a.acc_out = nullptr;
  a.y32_out = nullptr;
  a.status = static_cast<uint32_t*>(ws);
  a.M = int(M);
  a.N = int(N);
  a.K = int(K);
  a.pdl = false;
  a.faithful = false;
  a.ngroups = 1;
  a.group_end[0] = int(N);
  a.wait_ns = launch_wait_ns();
  a.stall = launch_stall();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M > 16) return status_of(launch_gemm_prefill(a, sms, s));
  // the previous operation on the stream is unknown: read the weights only
  // after the dependency wait
  DecodeArgs d;
  d.x = nullptr;
  d.xq = xq;
  d.s_x = x_scale;
  d.rowsum = xq_rowsum;
  d.packed = packed_w;
  d.w_scale = w_scale;
  d.bias = bias;
  d.y = y;
  d.xq_out = nullptr;
  d.sx_out = nullptr;
  d.acc_out = nullptr;
  d.y32_out = nullptr;
  d.status = a.status;
  d.M = int(M);
  d.N = int(N);
  d.K = int(K);
  d.weights_early = 0;
  d.faithful = 0;
  d.ngroups = 1;
  d.group_end[0] = int(N);
  d.wait_ns = a.wait_ns;
  d.stall = a.stall;
  return status_of(launch_decode(d, sms, s));
}

int bitlinear_dequant_weights(const uint8_t* packed_w, int64_t N, int64_t K, const float* w_scale,
                              uint16_t* w_bf16, void* stream) {
  int st = check_shape(1, N, K);
  if (st != BITLINEAR_OK) return st;
  if (!packed_w || !w_scale || !w_bf16) return BITLINEAR_ERR_NULL;
  if (misaligned(packed_w) || misaligned(w_scale) || misaligned(w_bf16)) return BITLINEAR_ERR_ALIGN;
  int sms = 148;
  st = check_device(&sms);
  if (st != BITLINEAR_OK) return st;
  return status_of(launch_dequant(packed_w, N, K, w_scale, w_bf16, sms, static_cast<cudaStream_t>(stream)));
}

int bitlinear_forward_debug(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                            const float* w_scale, const uint16_t* bias, uint16_t* y, int8_t* xq,
                            float* x_scale, int32_t* acc, float* y32, int engine, void* ws,
                            size_t ws_bytes, void* stream) {
  int st = check_forward_args(x, M, K, packed_w, N, w_scale, bias, y, ws, ws_bytes,
                              bitlinear_workspace_bytes(M, N, K), false);
  if (st != BITLINEAR_OK) return st;
  if (engine < 0 || engine > 2 || (engine == 1 && M > 16)) return BITLINEAR_ERR_SHAPE;
  if (misaligned(xq) || misaligned(x_scale) || misaligned(acc) || misaligned(y32)) return BITLINEAR_ERR_ALIGN;
  if (M == 0) return BITLINEAR_OK;
  return forward_impl(x, M, K, packed_w, N, w_scale, bias, y, xq, x_scale, acc, y32, engine, 0u, ws, ws_bytes,
                      static_cast<cudaStream_t>(stream));
}

int bitlinear_forward_debug_ex(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                               const float* w_scale, const uint16_t* bias, uint16_t* y, int8_t* xq,
                               float* x_scale, int32_t* acc, float* y32, int engine, unsigned flags, void* ws,
                               size_t ws_bytes, void* stream) {
  if (flags & ~static_cast<unsigned>(BITLINEAR_BF16_FAITHFUL)) return BITLINEAR_ERR_SHAPE;
  int st = check_forward_args(x, M, K, packed_w, N, w_scale, bias, y, ws, ws_bytes,
                              bitlinear_workspace_bytes(M, N, K), false);
  if (st != BITLINEAR_OK) return st;
  if (engine < 0 || engine > 2 || (engine == 1 && M > 16)) return BITLINEAR_ERR_SHAPE;
  if (misaligned(xq) || misaligned(x_scale) || misaligned(acc) || misaligned(y32)) return BITLINEAR_ERR_ALIGN;
  if (M == 0) return BITLINEAR_OK;
  return forward_impl(x, M, K, packed_w, N, w_scale, bias, y, xq, x_scale, acc, y32, engine, flags, ws, ws_bytes,
                      static_cast<cudaStream_t>(stream));
}

namespace {
int forward_host_impl(const uint16_t* x_host, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                      const float* w_scale, const uint16_t* bias, uint16_t* y_host, unsigned flags, void* ws,
                      size_t ws_bytes, cudaStream_t s, bool sync) {
  int st = check_forward_args(x_host, M, K, packed_w, N, w_scale, bias, y_host, ws, ws_bytes,
                              bitlinear_host_workspace_bytes(M, N, K), true);
  if (st != BITLINEAR_OK) return st;
  if (M == 0) return BITLINEAR_OK;
  const FwdLayout L = fwd_layout(M, N, K);
  char* base = static_cast<char*>(ws);
  uint16_t* xd = reinterpret_cast<uint16_t*>(base + L.off_xh);
  uint16_t* yd = reinterpret_cast<uint16_t*>(base + L.off_yh);
  if (cudaMemcpyAsync(xd, x_host, 2 * size_t(M) * size_t(K), cudaMemcpyHostToDevice, s) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  st = forward_impl(xd, M, K, packed_w, N, w_scale, bias, yd, nullptr, nullptr, nullptr, nullptr, 0, flags, ws,
                    ws_bytes, s);
  if (st != BITLINEAR_OK) return st;
  if (cudaMemcpyAsync(y_host, yd, 2 * size_t(M) * size_t(N), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  return sync ? status_of(cudaStreamSynchronize(s)) : BITLINEAR_OK;
}
}  // namespace

int bitlinear_forward_host(const uint16_t* x_host, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                           const float* w_scale, const uint16_t* bias, uint16_t* y_host, void* ws,
                           size_t ws_bytes, void* stream) {
  return forward_host_impl(x_host, M, K, packed_w, N, w_scale, bias, y_host, 0u, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream), true);
}

int bitlinear_forward_host_async(const uint16_t* x_host, int64_t M, int64_t K, const uint8_t* packed_w, int64_t N,
                                 const float* w_scale, const uint16_t* bias, uint16_t* y_host, unsigned flags,
                                 void* ws, size_t ws_bytes, void* stream) {
  if (flags & ~static_cast<unsigned>(BITLINEAR_WEIGHTS_RESIDENT | BITLINEAR_BF16_FAITHFUL)) return BITLINEAR_ERR_SHAPE;
  return forward_host_impl(x_host, M, K, packed_w, N, w_scale, bias, y_host, flags, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream), false);
}

// ---- tensor-parallel K-split pieces -----------------------------------------

static_assert(BITLINEAR_ABSMEAN_BINS == kAbsmeanBins, "header and kernels agree on the bin count");
static_assert(BITLINEAR_MAX_PARTS == kMaxParts, "header and kernels agree on the partial-sum limit");

int bitlinear_absmean_bins(const float* w, int64_t N, int64_t K, uint64_t* bins, void* stream) {
  if (N < 1 || K < 64 || (K % 64) != 0 || N > kMaxMN || K > kMaxK || N * K >= (int64_t(1) << 39))
    return BITLINEAR_ERR_SHAPE;
  if (!w || !bins) return BITLINEAR_ERR_NULL;
  if (misaligned(w) || misaligned(bins)) return BITLINEAR_ERR_ALIGN;
  int st = check_device(nullptr);
  if (st != BITLINEAR_OK) return st;
  return status_of(launch_absmean_bins(w, N, K, bins, static_cast<cudaStream_t>(stream)));
}

int bitlinear_pack_weights_from_bins(const float* w, int64_t N, int64_t K, const uint64_t* bins, int64_t n_total,
                                     uint8_t* packed, float* w_scale, float* w_mean, void* ws, size_t ws_bytes,
                                     void* stream) {
  if (N < 1 || K < 64 || (K % 64) != 0 || N > kMaxMN || K > kMaxK || N * K >= (int64_t(1) << 39))
    return BITLINEAR_ERR_SHAPE;
  if (n_total < N * K || n_total >= (int64_t(1) << 39)) return BITLINEAR_ERR_SHAPE;
  if (!w || !bins || !packed || !w_scale) return BITLINEAR_ERR_NULL;
  if (misaligned(w) || misaligned(bins) || misaligned(packed) || misaligned(w_scale) || misaligned(w_mean))
    return BITLINEAR_ERR_ALIGN;
  if (!ws || ws_bytes < kPackWsBytes) return BITLINEAR_ERR_WORKSPACE;
  if (misaligned(ws)) return BITLINEAR_ERR_ALIGN;
  int st = check_device(nullptr);
  if (st != BITLINEAR_OK) return st;
  return status_of(launch_pack_from_bins(w, N, K, bins, n_total, packed, w_scale, w_mean, pack_workspace(ws),
                                         static_cast<cudaStream_t>(stream)));
}

int bitlinear_act_absmax(const uint16_t* x, int64_t M, int64_t K, float* absmax, void* stream) {
  if (M < 0 || M > kMaxMN || K < 64 || K > kMaxK || (K % 64) != 0) return BITLINEAR_ERR_SHAPE;
  if (M == 0) return BITLINEAR_OK;
  if (!x || !absmax) return BITLINEAR_ERR_NULL;
  if (misaligned(x) || misaligned(absmax)) return BITLINEAR_ERR_ALIGN;
  int st = check_device(nullptr);
  if (st != BITLINEAR_OK) return st;
  return status_of(launch_act_absmax(x, int(M), int(K), absmax, static_cast<cudaStream_t>(stream)));
}

int bitlinear_forward_partial(const uint16_t* x, int64_t M, int64_t K, const float* absmax, const uint8_t* packed_w,
                              int64_t N, int32_t* acc, unsigned flags, void* ws, size_t ws_bytes, void* stream) {
  if (flags & ~static_cast<unsigned>(BITLINEAR_BF16_FAITHFUL)) return BITLINEAR_ERR_SHAPE;
  int st = check_shape(M, N, K);
  if (st != BITLINEAR_OK) return st;
  if (!x || !absmax || !packed_w || !acc) return BITLINEAR_ERR_NULL;
  if (misaligned(x) || misaligned(absmax) || misaligned(packed_w) || misaligned(acc)) return BITLINEAR_ERR_ALIGN;
  if (!ws || ws_bytes < bitlinear_workspace_bytes(M, N, K)) return BITLINEAR_ERR_WORKSPACE;
  if (misaligned(ws)) return BITLINEAR_ERR_ALIGN;
  if (M == 0) return BITLINEAR_OK;
  int sms = 148;
  st = check_device(&sms);
  if (st != BITLINEAR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const FwdLayout L = fwd_layout(M, N, K);
  char* base = static_cast<char*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  float* s_x = reinterpret_cast<float*>(base + L.off_sx);
  int32_t* rowsum = reinterpret_cast<int32_t*>(base + L.off_rs);
  int8_t* xq = reinterpret_cast<int8_t*>(base + L.off_xq);
  // this shard's x, quantised with the scale of the whole row
  const bool faithful = (flags & BITLINEAR_BF16_FAITHFUL) != 0;
  if (launch_act_quant(x, int(M), int(K), xq, s_x, rowsum, status, false, s, faithful, absmax) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  // the contraction alone: exact int32 partial sums, no bf16 output
  if (M > 16) {
    ForwardArgs a;
    a.xq = xq;
    a.s_x = s_x;
    a.rowsum = rowsum;
    a.packed = packed_w;
    a.w_scale = s_x;              // any finite scale: the quotient is not stored
    a.bias = nullptr;
    a.y = nullptr;
    a.acc_out = acc;
    a.y32_out = nullptr;
    a.status = status;
    a.M = int(M);
    a.N = int(N);
    a.K = int(K);
    a.pdl = true;
    a.faithful = false;
    a.ngroups = 1;
    a.group_end[0] = int(N);
    a.wait_ns = launch_wait_ns();
    a.stall = launch_stall();
    return status_of(launch_gemm_prefill(a, sms, s));
  }
  DecodeArgs d;
  d.x = nullptr;
  d.xq = xq;
  d.s_x = s_x;
  d.rowsum = rowsum;
  d.packed = packed_w;
  d.w_scale = s_x;
  d.bias = nullptr;
  d.y = nullptr;
  d.xq_out = nullptr;
  d.sx_out = nullptr;
  d.acc_out = acc;
  d.y32_out = nullptr;
  d.status = status;
  d.M = int(M);
  d.N = int(N);
  d.K = int(K);
  d.weights_early = 0;
  d.faithful = 0;
  d.ngroups = 1;
  d.group_end[0] = int(N);
  d.wait_ns = launch_wait_ns();
  d.stall = launch_stall();
  return status_of(launch_decode(d, sms, s));
}

int bitlinear_epilogue_sum(const int32_t* const* partials, int nparts, int64_t M, int64_t N, const float* absmax,
                           const float* w_scale, const uint16_t* bias, uint16_t* y, int32_t* acc_out,
                           unsigned flags, void* stream) {
  if (flags & ~static_cast<unsigned>(BITLINEAR_BF16_FAITHFUL)) return BITLINEAR_ERR_SHAPE;
  if (M < 0 || M > kMaxMN || N < 1 || N > kMaxMN) return BITLINEAR_ERR_SHAPE;
  if (nparts < 1 || nparts > BITLINEAR_MAX_PARTS) return BITLINEAR_ERR_SHAPE;
  if (!partials) return BITLINEAR_ERR_NULL;
  if (M == 0) return BITLINEAR_OK;
  EpilogueArgs a{};
  for (int r = 0; r < nparts; ++r) {
    if (!partials[r]) return BITLINEAR_ERR_NULL;
    if (misaligned(partials[r])) return BITLINEAR_ERR_ALIGN;
    a.part[r] = partials[r];
  }
  if (!absmax || !w_scale || !y) return BITLINEAR_ERR_NULL;
  if (misaligned(absmax) || misaligned(w_scale) || misaligned(bias) || misaligned(y) || misaligned(acc_out))
    return BITLINEAR_ERR_ALIGN;
  int sms = 148;
  int st = check_device(&sms);
  if (st != BITLINEAR_OK) return st;
  a.nparts = nparts;
  a.absmax = absmax;
  a.w_scale = w_scale;
  a.bias = bias;
  a.y = y;
  a.acc_out = acc_out;
  a.M = M;
  a.N = N;
  a.faithful = (flags & BITLINEAR_BF16_FAITHFUL) ? 1 : 0;
  return status_of(launch_epilogue(a, sms, static_cast<cudaStream_t>(stream)));
}

int bitlinear_measure_i8_peak(int iters, int* grid, void* ws, size_t ws_bytes, void* stream) {
  if (iters < 1 || iters > (1 << 24)) return BITLINEAR_ERR_SHAPE;
  if (!grid) return BITLINEAR_ERR_NULL;
  if (!ws || ws_bytes < 256) return BITLINEAR_ERR_WORKSPACE;
  if (misaligned(ws)) return BITLINEAR_ERR_ALIGN;
  int sms = 148;
  int st = check_device(&sms);
  if (st != BITLINEAR_OK) return st;
  *grid = sms;
  if (cudaMemsetAsync(ws, 0, 4, static_cast<cudaStream_t>(stream)) != cudaSuccess) return BITLINEAR_ERR_CUDA;
  return status_of(launch_tc_i8_peak(iters, sms, static_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream)));
}

int bitlinear_test_force_timeout(int on) {
  return g_force_timeout.exchange(on ? 1 : 0);
}

int bitlinear_check_status(const void* ws, size_t ws_bytes, void* stream) {
  if (!ws) return BITLINEAR_ERR_NULL;
  if (ws_bytes < 4) return BITLINEAR_ERR_WORKSPACE;
  uint32_t word = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&word, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return BITLINEAR_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BITLINEAR_ERR_CUDA;
  if (word != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpyAsync(const_cast<void*>(ws), &zero, 4, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return BITLINEAR_ERR_CUDA;
  }
  return (word & kStatusTimeout) ? BITLINEAR_ERR_TIMEOUT : BITLINEAR_OK;
}

}  // extern "C"
