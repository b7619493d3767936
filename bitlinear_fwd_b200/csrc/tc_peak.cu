// Measurement utility (not part of the BitLinear forward): the dense int8
// tensor-core rate of this GPU, the denominator the prefill GEMM is judged
// against.  One CTA per SM; one thread issues back-to-back
// tcgen05.mma.cta_group::1.kind::i8 of M = 128, N = 256, K = 32 (the largest
// single-CTA shape) from shared-memory operands into a tensor-memory
// accumulator, then waits for them with a bounded wait.  The operands are
// zeros: the tensor core's rate does not depend on the values.  The caller
// times the launch with CUDA events: int8 ops = 2 * 128 * 256 * 32 * 4 *
// iters * grid.
#include "kernels.h"

namespace bitlinear {

namespace {

constexpr int kRows = 128, kCols = 256;           // MMA M (A rows) and N (B rows)
constexpr uint32_t kABytes = kRows * 128;         // 128-byte K-major rows (128 k)
constexpr uint32_t kBBytes = kCols * 128;
constexpr uint32_t kSmem = kABytes + kBBytes + 1024 + 64;

__global__ void __launch_bounds__(128, 1) tc_i8_peak_kernel(int iters, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* done = reinterpret_cast<uint64_t*>(smem + kABytes + kBBytes);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  for (uint32_t i = threadIdx.x; i < (kABytes + kBBytes) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();                        // the zeros are visible to the tensor core
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(tslot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tslot;
  bool drained = true;
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = umma_idesc_i8(kRows, kCols, true, true);
    const uint32_t a_addr = smem_u32(smem), b_addr = smem_u32(smem + kABytes);
    for (int it = 0; it < iters; ++it)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
        umma_i8(tmem_d, umma_desc_sw128(a_addr + 32 * jj), umma_desc_sw128(b_addr + 32 * jj), idesc,
                (it | jj) != 0);
    umma_commit(done);
    drained = mbar_wait(done, 0, kWaitLimitNs);
    if (!drained) report_status(status, kStatusTimeout);
  }
  drained = __syncthreads_and(drained);
  // tensor memory is freed only once every MMA has completed
  if (threadIdx.x < 32 && drained) {
    tc_fence_after();
    tmem_dealloc(tmem_d, kCols);
  }
}

}  // namespace

cudaError_t launch_tc_i8_peak(int iters, int num_sms, uint32_t* status, cudaStream_t stream) {
  static unsigned long long attr_done = 0;
  cudaError_t e = set_smem_attr_once(tc_i8_peak_kernel, static_cast<int>(kSmem), &attr_done);
  if (e != cudaSuccess) return e;
  tc_i8_peak_kernel<<<num_sms, 128, kSmem, stream>>>(iters, status);
  return cudaGetLastError();
}

}  // namespace bitlinear
