// The epilogue of BitLinear.forward (Falcon-Edge blog, section "Falcon-Edge,
// a series of universal models": post_quant_process and the bias add) on
// int32 accumulators that arrive as partial sums -- one per K-shard of a
// tensor-parallel split.  The partial sums are added in int32 (exact: the
// total is the full contraction, |acc| <= 127 K), then
//   s_x = 127 / max(a, 1e-5)   from the token's absmax a over the whole K,
//   y32 = float(acc) / (s_x * s_w) (+ bias),   y = bf16_rne(y32),
// the same float32 operations as the fused epilogues of both engines (and
// the bf16-module rounding of every step in the bf16-faithful mode).
//
// The partial-sum pointers may point into other GPUs' memory (peer access):
// the kernel only loads them, with plain loads, so the reduction over the
// shards happens in this kernel's reads.  The caller makes sure every
// partial sum is complete before the launch.
//
// Memory bound: 4 B per element per partial sum read, 2 B written.  One
// element per thread per step of a grid-stride loop, consecutive threads on
// consecutive columns, so every load and store is coalesced.
#include "kernels.h"

namespace bitlinear {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) epilogue_kernel(const EpilogueArgs a) {
  pdl_wait_primary();
  const int64_t total = a.M * a.N;
  const float s_w = a.faithful ? bf16_round(*a.w_scale) : *a.w_scale;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < total; i += stride) {
    const int64_t m = i / a.N, n = i - m * a.N;
    int acc = 0;
#pragma unroll 1
    for (int r = 0; r < a.nparts; ++r) acc += a.part[r][i];
    const float am = a.absmax[m];
    float y32;
    if (!a.faithful) {
      const float s_x = __fdiv_rn(127.0f, fmaxf(am, 1e-5f));
      y32 = __fdiv_rn(static_cast<float>(acc), __fmul_rn(s_x, s_w));
      if (a.bias) y32 = __fadd_rn(y32, bf16_bits_to_f32(a.bias[n]));
    } else {
      const float s_x = bf16_round(__fmul_rn(bf16_round(__fdiv_rn(1.0f, fmaxf(am, bf16_round(1e-5f)))), 127.0f));
      y32 = bf16_round(__fdiv_rn(bf16_round(static_cast<float>(acc)), bf16_round(__fmul_rn(s_w, s_x))));
      if (a.bias) y32 = bf16_round(__fadd_rn(y32, bf16_bits_to_f32(a.bias[n])));
    }
    a.y[i] = f32_to_bf16_bits(y32);
    if (a.acc_out) a.acc_out[i] = acc;
  }
}

}  // namespace

cudaError_t launch_epilogue(const EpilogueArgs& a, int num_sms, cudaStream_t stream) {
  if (a.M <= 0) return cudaSuccess;
  const int64_t total = a.M * a.N;
  int64_t blocks = (total + kThreads - 1) / kThreads;
  const int64_t cap = 8LL * num_sms;
  blocks = blocks < cap ? blocks : cap;
  epilogue_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace bitlinear
