// bf16 export of packed ternary weights: the state-dict loop of the
// Falcon-Edge blog (section "Falcon-Edge, a series of universal models":
// param_value = u / param_scale, stored as bfloat16), so that a plain bf16
// linear layer can load the weights.  u / s_w is rounded to float32 once and
// then to bfloat16; for u in {-1, 0, 1} that is -v, +0, v with
// v = bf16(RN(1 / s_w)).  A zero exports as +0 (the packed codes do not keep
// the sign of a zero that round() produced).
//
// Memory-bound: 0.25 B read and 2 B written per weight.  One thread turns a
// packed word (16 weights, k = 16g + 4i + j at bits 8j + 2i) into 32 output
// bytes, written as two 16-byte stores; a packed row of K/16 words becomes the
// K bf16 values of the same row, so word w maps to output bytes [32w, 32w+32).
// Each output word (two bf16 values, k and k + 1 = bytes j and j + 1 of
// field i) is one byte permutation of the eight bytes {bf16(+v), 0, 0,
// bf16(-v), 0, 0}: a code c selects bytes 4 - 2c and 5 - 2c (2 -> +v, 1 -> 0,
// 0 -> -v), so the selector of a pair of codes (c0, c1) is 0x5454 - (c0 +
// 256 c1) 0x22, and (word >> 2i) & 0x03030303 holds c0 + 256 c1 for both
// pairs of field i.  Four instructions per output word instead of a compare
// and select per value (the loop was issue-bound).  A word holding the
// invalid code 3 exports unspecified values.
#include "kernels.h"

namespace bitlinear {

namespace {

__global__ void __launch_bounds__(256) dequant_kernel(const uint32_t* __restrict__ packed, size_t words,
                                                      const float* __restrict__ w_scale, uint4* __restrict__ out) {
  // bytes 0-1: bf16(+v), 2-3: zero; bytes 4-5: bf16(-v), 6-7: zero
  const uint32_t pos = f32_to_bf16_bits(__fdiv_rn(1.0f, *w_scale));
  const uint32_t neg = pos ^ 0x8000u;
  for (size_t idx = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; idx < words;
       idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint32_t wd = __ldg(packed + idx);
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {                  // output words 2i (k = 4i, 4i+1) and 2i + 1 (k = 4i+2, 4i+3)
      const uint32_t u = (wd >> (2 * i)) & 0x03030303u;
      o[2 * i] = __byte_perm(pos, neg, 0x5454u - u * 0x22u);           // the selector uses the low 16 bits
      o[2 * i + 1] = __byte_perm(pos, neg, 0x5454u - (u >> 16) * 0x22u);
    }
    out[2 * idx] = make_uint4(o[0], o[1], o[2], o[3]);
    out[2 * idx + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace

cudaError_t launch_dequant(const uint8_t* packed, int64_t N, int64_t K, const float* w_scale, uint16_t* w_bf16,
                           int num_sms, cudaStream_t stream) {
  const size_t words = static_cast<size_t>(N) * static_cast<size_t>(K / 16);
  if (words == 0) return cudaSuccess;
  const size_t want = (words + 255) / 256;
  const unsigned grid = static_cast<unsigned>(want < static_cast<size_t>(num_sms) * 8 ? want : static_cast<size_t>(num_sms) * 8);
  dequant_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint32_t*>(packed), words, w_scale,
                                           reinterpret_cast<uint4*>(w_bf16));
  return cudaGetLastError();
}

}  // namespace bitlinear
