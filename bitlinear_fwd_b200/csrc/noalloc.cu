// bitlinear_forward_noalloc: the forward for callers that cannot allocate
// device memory.
//
// Some callers cannot call cudaMalloc: code that runs inside a CUDA-graph
// capture of someone else's stream, plugins of inference servers that hand
// out no allocator, or real-time paths that must never allocate (an
// allocation can synchronise the device or fail under memory pressure).
// They pass only inputs and outputs; the workspace the forward needs (the
// status word, s_x, row sums and int8 activations) lives instead in one
// fixed array of device memory that this file declares.  Every GPU that
// loads the library holds that array until the process exits.
//
// The array's name is a host-side stand-in in host code, not a device
// address, so its device address is looked up once per device (with that
// device current) and cached.  All calls share the array and it keeps the
// last call's contents: calls that overlap on the GPU (different streams,
// or host threads racing) corrupt each other's scratch.  Nothing in it has
// to start at zero: each forward writes every scratch byte it reads, and
// its first kernel resets the status word.
#include <mutex>

#include "../../include/bitlinear.h"
#include "kernels.h"

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[BITLINEAR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on
// the first call for that device).  Returns a bitlinear status.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BITLINEAR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BITLINEAR_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return BITLINEAR_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return BITLINEAR_OK;
}

}  // namespace

extern "C" int bitlinear_forward_noalloc(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed_w,
                                         int64_t N, const float* w_scale, const uint16_t* bias, uint16_t* y,
                                         void* stream) {
  const size_t need = bitlinear_workspace_bytes(M, N, K);
  if (need == 0) return BITLINEAR_ERR_SHAPE;
  if (need > BITLINEAR_NOALLOC_SCRATCH_BYTES) return BITLINEAR_ERR_WORKSPACE;   // beyond the fixed scratch
  // the device check comes first: on a GPU the library has no code for, the
  // symbol lookup below would fail with a less telling error
  int st = bitlinear::current_device_status();
  if (st != BITLINEAR_OK) return st;
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != BITLINEAR_OK) return st;
  return bitlinear_forward(x, M, K, packed_w, N, w_scale, bias, y, scratch, BITLINEAR_NOALLOC_SCRATCH_BYTES,
                           stream);
}

// The status word lives at the start of the scratch array, as in any
// workspace; this reads and clears it for the current device.
extern "C" int bitlinear_noalloc_check_status(void* stream) {
  int st = bitlinear::current_device_status();
  if (st != BITLINEAR_OK) return st;
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != BITLINEAR_OK) return st;
  return bitlinear_check_status(scratch, BITLINEAR_NOALLOC_SCRATCH_BYTES, stream);
}
