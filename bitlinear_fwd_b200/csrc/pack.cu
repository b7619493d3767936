// Weight ternarisation and 2-bit packing (_weight_quant of the Falcon-Edge
// blog, section "Falcon-Edge, a series of universal models"):
//   s_w = 1 / max(mean |w|, 1e-5) over the whole tensor,
//   u   = clamp(round_half_even(w * s_w), -1, 1),  stored as code u + 1.
//
// Three kernels:
//   absmean_bins      exact sum of |w|: every float32 |w| is m * 2^(max(e,1)-150)
//                     (m its 24-bit significand, e its biased exponent), so
//                     the significands are summed per exponent in 64-bit
//                     integers -- exact and independent of order.  A warp
//                     first adds the significands of lanes that share an
//                     exponent (redux.sync), then one lane adds the group's
//                     sum into a shared-memory bin; CTAs flush their bins
//                     to global memory with 64-bit atomics.
//   absmean_finalize  one thread turns the 256 bins into the exact sum
//                     (a 352-bit integer in 16-bit limbs), divides it by
//                     N*K by long division, rounds the quotient once to
//                     float32 (ties to even), and forms s_w.
//   ternarise_pack    16 weights -> one 32-bit word in the library layout
//                     (k = 16g + 4i + j at bits 8j + 2i of word g).
#include "kernels.h"

namespace bitlinear {

namespace {

constexpr int kThreads = 256;
constexpr unsigned kFull = 0xffffffffu;

// Adds |w| (given as its bits, sign cleared) of every valid lane to the bins.
__device__ __forceinline__ void bin_add_warp(uint32_t abits, bool valid, unsigned long long* sbins) {
  const uint32_t e = abits >> 23;
  const uint32_t m = (abits & 0x7FFFFFu) | (e ? 0x800000u : 0u);
  const bool live = valid && m != 0u;
  const int key = live ? static_cast<int>(e) : -1;
  unsigned todo = __ballot_sync(kFull, live);
  const int lane = threadIdx.x & 31;
  while (todo) {
    const int leader = __ffs(todo) - 1;
    const int ke = __shfl_sync(kFull, key, leader);
    const bool mine = (key == ke);
    const unsigned grp = __ballot_sync(kFull, mine);
    const unsigned s = __reduce_add_sync(kFull, mine ? m : 0u);   // < 32 * 2^24
    if (lane == leader) atomicAdd(&sbins[ke], static_cast<unsigned long long>(s));
    todo &= ~grp;
  }
}

__global__ void __launch_bounds__(kThreads) absmean_bins_kernel(const float4* __restrict__ w4,
                                                                int64_t n4,
                                                                unsigned long long* gbins) {
  __shared__ unsigned long long sbins[256];
  sbins[threadIdx.x] = 0ull;
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  // warp-uniform trip count so that every lane joins the warp collectives
  const int64_t warp_base = static_cast<int64_t>(blockIdx.x) * kThreads + (threadIdx.x & ~31);
  for (int64_t base = warp_base; base < n4; base += stride) {
    const int64_t i = base + (threadIdx.x & 31);
    const bool valid = i < n4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (valid) v = __ldg(w4 + i);
    bin_add_warp(__float_as_uint(v.x) & 0x7FFFFFFFu, valid, sbins);
    bin_add_warp(__float_as_uint(v.y) & 0x7FFFFFFFu, valid, sbins);
    bin_add_warp(__float_as_uint(v.z) & 0x7FFFFFFFu, valid, sbins);
    bin_add_warp(__float_as_uint(v.w) & 0x7FFFFFFFu, valid, sbins);
  }
  __syncthreads();
  const unsigned long long b = sbins[threadIdx.x];
  if (b) atomicAdd(&gbins[threadIdx.x], b);
}

constexpr int kLimbs = 24;  // 16-bit limbs: 384 bits > 53 + 253 + margin

__device__ __forceinline__ uint32_t window16(const uint32_t* limb, int pos) {
  // bits [pos, pos + 16) of the limb array (pos >= 0)
  const int li = pos >> 4, off = pos & 15;
  uint32_t lo = li < kLimbs ? limb[li] : 0u;
  uint32_t hi = (li + 1) < kLimbs ? limb[li + 1] : 0u;
  return ((lo >> off) | (hi << (16 - off))) & 0xFFFFu;
}

__global__ void absmean_finalize_kernel(const unsigned long long* __restrict__ bins, uint64_t n,
                                        float* w_scale, float* mean_ws, float* mean_out) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  // S = sum_e bins[e] * 2^(max(e,1) - 1), in 16-bit limbs (units of 2^-149)
  uint64_t accl[kLimbs];
  for (int i = 0; i < kLimbs; ++i) accl[i] = 0;
  for (int e = 0; e < 256; ++e) {
    const uint64_t v = bins[e];
    if (!v) continue;
    const int s = (e > 1 ? e : 1) - 1;
    const int li = s >> 4, off = s & 15;
    for (int p = 0; p < 4; ++p) {  // v < 2^53: four 16-bit pieces
      const uint64_t piece = ((v >> (16 * p)) & 0xFFFFull) << off;   // < 2^31
      accl[li + p] += piece & 0xFFFFull;
      accl[li + p + 1] += piece >> 16;
    }
  }
  uint32_t limb[kLimbs];
  uint64_t carry = 0;
  for (int i = 0; i < kLimbs; ++i) {
    const uint64_t t = accl[i] + carry;
    limb[i] = static_cast<uint32_t>(t & 0xFFFFull);
    carry = t >> 16;
  }
  int top = kLimbs - 1;
  while (top >= 0 && limb[top] == 0) --top;
  float mean = 0.0f;
  if (top >= 0) {
    const int Ls = 16 * top + (32 - __clz(limb[top]));     // bit length of S
    const int Ln = 64 - __clzll(static_cast<long long>(n));  // bit length of n
    const int sh = 26 - Ls + Ln;        // quotient S * 2^sh / n lies in [2^25, 2^27)
    const int a = sh < 0 ? -sh : 0;     // right shift of S
    // sticky: bits of S below position a
    bool sticky = false;
    for (int i = 0; i < kLimbs && 16 * i < a; ++i) {
      const int nb = a - 16 * i;
      const uint32_t mask = nb >= 16 ? 0xFFFFu : ((1u << nb) - 1u);
      if (limb[i] & mask) sticky = true;
    }
    // long division of T = S >> a by n, most significant limb first
    const int tl = (Ls - a + 15) >> 4;  // limbs of T
    uint64_t rem = 0, Q = 0;
    for (int i = tl - 1; i >= 0; --i) {
      rem = (rem << 16) | window16(limb, a + 16 * i);   // rem < n < 2^40
      Q = (Q << 16) | (rem / n);
      rem %= n;
    }
    for (int i = 0; i < (sh > 0 ? sh : 0); ++i) {   // append sh zero bits
      rem <<= 1;
      Q <<= 1;
      if (rem >= n) { rem -= n; Q |= 1; }
    }
    sticky = sticky || rem != 0;
    // mean = (Q + frac) * 2^(-sh - 149); keep 24 significant bits
    const int b = 64 - __clzll(static_cast<long long>(Q));
    int d = b - 24;
    int E = -sh - 149 + d;             // weight of the last kept bit
    if (E < -149) { d += -149 - E; E = -149; }
    uint64_t q = 0;
    if (d < 60) {
      const uint64_t r = Q & ((1ull << d) - 1ull);
      const uint64_t half = 1ull << (d - 1);
      q = Q >> d;
      if (r > half || (r == half && (sticky || (q & 1ull)))) ++q;
    }
    if (q == (1ull << 24)) { q >>= 1; ++E; }
    uint32_t bits;
    if (q >= (1ull << 23)) bits = (static_cast<uint32_t>(E + 150) << 23) | static_cast<uint32_t>(q & 0x7FFFFFull);
    else bits = static_cast<uint32_t>(q);        // gradual underflow (E == -149)
    mean = __uint_as_float(bits);
  }
  const float s = __fdiv_rn(1.0f, fmaxf(mean, 1e-5f));
  *w_scale = s;
  *mean_ws = mean;
  if (mean_out) *mean_out = mean;
}

__device__ __forceinline__ uint32_t ternary_code(float w, float s) {
  const float r = rintf(__fmul_rn(w, s));
  return static_cast<uint32_t>(static_cast<int>(fminf(fmaxf(r, -1.0f), 1.0f)) + 1);
}

__global__ void __launch_bounds__(kThreads) ternarise_pack_kernel(const float4* __restrict__ w4,
                                                                  int64_t nwords,
                                                                  const float* __restrict__ w_scale,
                                                                  uint32_t* __restrict__ words) {
  const float s = *w_scale;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; g < nwords; g += stride) {
    uint32_t word = 0;
#pragma unroll
    for (int v = 0; v < 4; ++v) {          // elements 4v .. 4v+3: i = v, j = 0..3
      const float4 f = __ldg(w4 + 4 * g + v);
      word |= ternary_code(f.x, s) << (2 * v);
      word |= ternary_code(f.y, s) << (8 + 2 * v);
      word |= ternary_code(f.z, s) << (16 + 2 * v);
      word |= ternary_code(f.w, s) << (24 + 2 * v);
    }
    words[g] = word;
  }
}

}  // namespace

PackWorkspace pack_workspace(void* ws) {
  char* base = static_cast<char*>(ws);
  PackWorkspace p;
  p.status = reinterpret_cast<uint32_t*>(base);
  p.mean = reinterpret_cast<float*>(base + 16);
  p.bins = reinterpret_cast<uint64_t*>(base + 256);
  return p;
}

cudaError_t launch_pack(const float* w, int64_t N, int64_t K, uint8_t* packed, float* w_scale,
                        float* w_mean, const PackWorkspace& pws, cudaStream_t stream) {
  cudaError_t err = cudaMemsetAsync(pws.status, 0, 256 + 256 * sizeof(uint64_t), stream);
  if (err != cudaSuccess) return err;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t n = N * K;
  const int64_t n4 = n / 4;
  int64_t blocks = (n4 + kThreads - 1) / kThreads;
  blocks = blocks < 8LL * sms ? blocks : 8LL * sms;
  absmean_bins_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      reinterpret_cast<const float4*>(w), n4, reinterpret_cast<unsigned long long*>(pws.bins));
  absmean_finalize_kernel<<<1, 32, 0, stream>>>(reinterpret_cast<const unsigned long long*>(pws.bins),
                                                static_cast<uint64_t>(n), w_scale, pws.mean, w_mean);
  const int64_t nwords = n / 16;
  int64_t pblocks = (nwords + kThreads - 1) / kThreads;
  pblocks = pblocks < 16LL * sms ? pblocks : 16LL * sms;
  ternarise_pack_kernel<<<static_cast<unsigned>(pblocks), kThreads, 0, stream>>>(
      reinterpret_cast<const float4*>(w), nwords, w_scale, reinterpret_cast<uint32_t*>(packed));
  return cudaGetLastError();
}

}  // namespace bitlinear
