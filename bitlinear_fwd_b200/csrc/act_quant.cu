// Per-token activation quantisation (activation_norm_quant of the
// Falcon-Edge blog, section "Falcon-Edge, a series of universal models"):
//   s_x = 127 / max(max_k |x|, 1e-5),  q = clamp(round_half_even(x * s_x), -128, 127)
// in float32, plus the row sum of q that the contraction engines use.  In
// the bf16-faithful mode every step is rounded as a bf16 module rounds it.
//
// One CTA per row.  The row is read once with 16-byte loads and kept in
// registers between the absmax pass and the quantisation pass (rows of up
// to 32768 elements; longer rows are read twice).  The absmax runs on the
// bf16 bit patterns: for finite values |x| orders like its bits & 0x7FFF.
#include "kernels.h"

namespace bitlinear {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t absmax_pair(uint32_t acc, uint32_t w) {
  return __vmaxu2(acc, w & 0x7FFF7FFFu);
}

__device__ __forceinline__ uint32_t reduce_max_u32(uint32_t v, uint32_t* red) {
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t t = threadIdx.x < (kThreads / 32) ? red[threadIdx.x] : 0u;
    for (int o = 16; o > 0; o >>= 1) t = max(t, __shfl_xor_sync(0xffffffffu, t, o));
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  const uint32_t r = red[0];
  __syncthreads();
  return r;
}

__device__ __forceinline__ int reduce_add_i32(int v, int* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int t = 0;
  if (threadIdx.x == 0)
    for (int i = 0; i < kThreads / 32; ++i) t += red[i];
  return t;  // valid in thread 0
}

// Four bf16 values (two words) -> four int8 q = round_half_even(x * s), packed.
// p = x * s is rounded to float32 first; adding 1.5 * 2^23 then rounds p to an
// integer with ties to even (the sum lies in [2^23, 2^24), where the float
// spacing is 1, and the constant is even), and the low byte of the sum's bits
// is q as a two's-complement byte.  In float32 |p| <= 127 because s was formed
// from the row's absmax (or, for a K-shard, the whole row's), so the
// [-128, 127] clamp never acts there; the bf16-faithful path rounds p to bf16
// and clamps explicitly (bf16(x * scale) can reach 128).
constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23

__device__ __forceinline__ uint32_t quant4(uint32_t w01, uint32_t w23, float s, bool faithful) {
  float p[4] = {__fmul_rn(__uint_as_float(w01 << 16), s), __fmul_rn(__uint_as_float(w01 & 0xFFFF0000u), s),
                __fmul_rn(__uint_as_float(w23 << 16), s), __fmul_rn(__uint_as_float(w23 & 0xFFFF0000u), s)};
  if (faithful) {
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = fminf(fmaxf(bf16_round(p[e]), -128.0f), 127.0f);
  }
  const uint32_t b0 = __float_as_uint(__fadd_rn(p[0], kRoundMagic));
  const uint32_t b1 = __float_as_uint(__fadd_rn(p[1], kRoundMagic));
  const uint32_t b2 = __float_as_uint(__fadd_rn(p[2], kRoundMagic));
  const uint32_t b3 = __float_as_uint(__fadd_rn(p[3], kRoundMagic));
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// Quantises 16 bf16 values (two 16-byte vectors) into one 16-byte vector of
// int8 and adds their sum to `sum`.
__device__ __forceinline__ uint4 quant16(uint4 lo, uint4 hi, float s, int& sum, bool faithful) {
  uint4 q;
  q.x = quant4(lo.x, lo.y, s, faithful);
  q.y = quant4(lo.z, lo.w, s, faithful);
  q.z = quant4(hi.x, hi.y, s, faithful);
  q.w = quant4(hi.z, hi.w, s, faithful);
  sum = __dp4a(static_cast<int>(q.x), 0x01010101, sum);
  sum = __dp4a(static_cast<int>(q.y), 0x01010101, sum);
  sum = __dp4a(static_cast<int>(q.z), 0x01010101, sum);
  sum = __dp4a(static_cast<int>(q.w), 0x01010101, sum);
  return q;
}

template <int CPT>  // 16-element chunks cached per thread; 0 = read the row twice
__global__ void __launch_bounds__(kThreads) act_quant_kernel(const uint16_t* __restrict__ x, int K,
                                                             int8_t* __restrict__ xq,
                                                             float* __restrict__ s_x,
                                                             int32_t* __restrict__ rowsum,
                                                             uint32_t* status_clear, bool faithful,
                                                             const float* __restrict__ absmax_in) {
  pdl_launch_dependents();
  pdl_wait_primary();
  if (status_clear && blockIdx.x == 0 && threadIdx.x == 0) *status_clear = 0u;
  __shared__ uint32_t red[kThreads / 32];

  const int row = blockIdx.x;
  const int chunks = K >> 4;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(row) * K);
  uint4* qr = reinterpret_cast<uint4*>(xq + static_cast<size_t>(row) * K);

  uint4 cache[CPT > 0 ? 2 * CPT : 1];
  uint32_t amax = 0;
  if constexpr (CPT > 0) {
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = threadIdx.x + i * kThreads;
      if (c < chunks) {
        cache[2 * i] = __ldg(xr + 2 * c);
        cache[2 * i + 1] = __ldg(xr + 2 * c + 1);
      } else {
        cache[2 * i] = make_uint4(0, 0, 0, 0);
        cache[2 * i + 1] = make_uint4(0, 0, 0, 0);
      }
      amax = absmax_pair(amax, cache[2 * i].x);
      amax = absmax_pair(amax, cache[2 * i].y);
      amax = absmax_pair(amax, cache[2 * i].z);
      amax = absmax_pair(amax, cache[2 * i].w);
      amax = absmax_pair(amax, cache[2 * i + 1].x);
      amax = absmax_pair(amax, cache[2 * i + 1].y);
      amax = absmax_pair(amax, cache[2 * i + 1].z);
      amax = absmax_pair(amax, cache[2 * i + 1].w);
    }
  } else {
    for (int c = threadIdx.x; c < chunks; c += kThreads) {
      const uint4 a = __ldg(xr + 2 * c), b = __ldg(xr + 2 * c + 1);
      amax = absmax_pair(amax, a.x); amax = absmax_pair(amax, a.y);
      amax = absmax_pair(amax, a.z); amax = absmax_pair(amax, a.w);
      amax = absmax_pair(amax, b.x); amax = absmax_pair(amax, b.y);
      amax = absmax_pair(amax, b.z); amax = absmax_pair(amax, b.w);
    }
  }
  amax = max(amax & 0xFFFFu, amax >> 16);
  amax = reduce_max_u32(amax, red);

  // a K-shard takes the absmax of the whole row, all-reduced over the shards
  const float a = absmax_in ? absmax_in[row] : bf16_bits_to_f32(amax);
  // float32: 127 / max(a, 1e-5).  bf16 module: PyTorch evaluates 127.0 / t as
  // t.reciprocal() * 127, each rounded to bf16.
  const float s = faithful ? bf16_round(__fmul_rn(bf16_round(__fdiv_rn(1.0f, fmaxf(a, bf16_round(1e-5f)))), 127.0f))
                           : __fdiv_rn(127.0f, fmaxf(a, 1e-5f));

  int sum = 0;
  if constexpr (CPT > 0) {
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = threadIdx.x + i * kThreads;
      if (c < chunks) qr[c] = quant16(cache[2 * i], cache[2 * i + 1], s, sum, faithful);
    }
  } else {
    for (int c = threadIdx.x; c < chunks; c += kThreads)
      qr[c] = quant16(__ldg(xr + 2 * c), __ldg(xr + 2 * c + 1), s, sum, faithful);
  }
  sum = reduce_add_i32(sum, reinterpret_cast<int*>(red));
  if (threadIdx.x == 0) {
    s_x[row] = s;
    if (rowsum) rowsum[row] = sum;
  }
}

// Per-token absmax over this x (one K-shard of the row), as float32: the
// partial reduction of activation_norm_quant that an all-reduce MAX completes.
__global__ void __launch_bounds__(kThreads) act_absmax_kernel(const uint16_t* __restrict__ x, int K,
                                                              float* __restrict__ absmax) {
  pdl_wait_primary();
  __shared__ uint32_t red[kThreads / 32];
  const int row = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(row) * K);
  uint32_t amax = 0;
  for (int c = threadIdx.x; c < (K >> 3); c += kThreads) {
    const uint4 a = __ldg(xr + c);
    amax = absmax_pair(amax, a.x); amax = absmax_pair(amax, a.y);
    amax = absmax_pair(amax, a.z); amax = absmax_pair(amax, a.w);
  }
  amax = max(amax & 0xFFFFu, amax >> 16);
  amax = reduce_max_u32(amax, red);
  if (threadIdx.x == 0) absmax[row] = bf16_bits_to_f32(amax);
}

}  // namespace

cudaError_t launch_act_absmax(const uint16_t* x, int M, int K, float* absmax, cudaStream_t stream) {
  if (M <= 0) return cudaSuccess;
  act_absmax_kernel<<<M, kThreads, 0, stream>>>(x, K, absmax);
  return cudaGetLastError();
}

template <int CPT>
cudaError_t launch_cpt(const uint16_t* x, int M, int K, int8_t* xq, float* s_x, int32_t* rowsum,
                       uint32_t* status_clear, bool pdl, cudaStream_t stream, bool faithful, const float* absmax_in) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, act_quant_kernel<CPT>, x, K, xq, s_x, rowsum, status_clear, faithful, absmax_in);
}

cudaError_t launch_act_quant(const uint16_t* x, int M, int K, int8_t* xq, float* s_x,
                             int32_t* rowsum, uint32_t* status_clear, bool pdl, cudaStream_t stream,
                             bool faithful, const float* absmax_in) {
  if (M <= 0) return cudaSuccess;
  const int chunks = K / 16;
  const float* am = absmax_in;
  if (chunks <= kThreads) return launch_cpt<1>(x, M, K, xq, s_x, rowsum, status_clear, pdl, stream, faithful, am);
  if (chunks <= 2 * kThreads) return launch_cpt<2>(x, M, K, xq, s_x, rowsum, status_clear, pdl, stream, faithful, am);
  if (chunks <= 4 * kThreads) return launch_cpt<4>(x, M, K, xq, s_x, rowsum, status_clear, pdl, stream, faithful, am);
  if (chunks <= 8 * kThreads) return launch_cpt<8>(x, M, K, xq, s_x, rowsum, status_clear, pdl, stream, faithful, am);
  return launch_cpt<0>(x, M, K, xq, s_x, rowsum, status_clear, pdl, stream, faithful, am);
}

}  // namespace bitlinear
