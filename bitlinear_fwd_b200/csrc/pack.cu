// Weight ternarisation and 2-bit packing (_weight_quant of the Falcon-Edge
// blog, section "Falcon-Edge, a series of universal models"):
//   s_w = 1 / max(mean |w|, 1e-5) over the whole tensor,
//   u   = clamp(round_half_even(w * s_w), -1, 1),  stored as code u + 1.
//
// Three kernels:
//   absmean_bins      exact sum of |w|: every float32 |w| is m * 2^(max(e,1)-150)
//                     (m its 24-bit significand, e its biased exponent).  Each
//                     warp picks an anchor exponent B from its first loads
//                     (B = max(e0 - 36, 1), e0 the largest exponent there); a
//                     weight with max(e,1) in [B, B + 39] adds m << (max(e,1) - B)
//                     (< 2^63) to its thread's 128-bit integer sum -- exact, and
//                     independent of order.  At the end each thread's sum is cut
//                     into 24-bit chunks; chunk j, summed over the warp, goes to
//                     exponent bin B + 24j.  The rare weight outside the window
//                     goes to its own exponent's bin directly: the warp adds the
//                     significands of lanes that share an exponent (redux.sync)
//                     and one lane adds the group's sum.  Bins live in shared
//                     memory, then are flushed to global memory with 64-bit
//                     atomics.  Bin e holds a sum of significands of weight
//                     2^(max(e,1) - 150); 320 bins cover the chunks' exponents.
//   absmean_finalize  one warp turns the bins into the exact sum S (a 416-bit
//                     integer in 16-bit limbs), one thread divides S by N*K by
//                     long division, rounds the quotient once to float32 (ties
//                     to even), and forms s_w.
//   ternarise_pack    16 weights -> one 32-bit word in the library layout
//                     (k = 16g + 4i + j at bits 8j + 2i of word g).
#include "kernels.h"

namespace bitlinear {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;                 // float4 loads in flight per thread
constexpr unsigned kFull = 0xffffffffu;
constexpr int kAnchorBelow = 36;           // B = e0 - 36: the window reaches 2^-36 below the first loads' max
constexpr int kWindow = 39;                // shifts 0..39 keep m << d below 2^63

// Adds |w| (given as its bits, sign cleared) of every live lane to its
// exponent's bin.
__device__ __forceinline__ void bin_add_warp(uint32_t abits, bool live_in, unsigned long long* sbins) {
  const uint32_t e = abits >> 23;
  const uint32_t m = (abits & 0x7FFFFFu) | (e ? 0x800000u : 0u);
  const bool live = live_in && m != 0u;
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

// The window sum of one weight: adds m << (max(e,1) - B) to (hi:lo) when the
// shift is in [0, kWindow]; returns true when the weight is nonzero and
// outside the window.
__device__ __forceinline__ bool window_add(uint32_t bits, int B, uint64_t& lo, uint64_t& hi) {
  const uint32_t ab = bits & 0x7FFFFFFFu;
  const uint32_t e = ab >> 23;
  const uint32_t m = (ab & 0x7FFFFFu) | (e ? 0x800000u : 0u);
  const int d = static_cast<int>(e > 1u ? e : 1u) - B;
  const bool in = static_cast<unsigned>(d) <= static_cast<unsigned>(kWindow);
  const uint64_t v = in ? (static_cast<uint64_t>(m) << (d & 63)) : 0ull;
  asm("add.cc.u64 %0, %0, %2;\n\taddc.u64 %1, %1, 0;" : "+l"(lo), "+l"(hi) : "l"(v));
  return !in && m != 0u;
}

__global__ void __launch_bounds__(kThreads) absmean_bins_kernel(const float4* __restrict__ w4,
                                                                int64_t n4,
                                                                unsigned long long* gbins) {
  __shared__ unsigned long long sbins[kAbsmeanBins];
  for (int i = threadIdx.x; i < kAbsmeanBins; i += kThreads) sbins[i] = 0ull;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  // warp-uniform trip counts, so that every lane joins the warp collectives
  const int64_t warp_base = static_cast<int64_t>(blockIdx.x) * kThreads + (threadIdx.x & ~31);

  // anchor: the largest exponent among the warp's first loads
  uint32_t e0 = 0;
  if (warp_base + lane < n4) {
    const float4 f = __ldg(w4 + warp_base + lane);
    e0 = max(max(__float_as_uint(f.x) & 0x7FFFFFFFu, __float_as_uint(f.y) & 0x7FFFFFFFu),
             max(__float_as_uint(f.z) & 0x7FFFFFFFu, __float_as_uint(f.w) & 0x7FFFFFFFu)) >> 23;
  }
  e0 = __reduce_max_sync(kFull, e0);
  const int B = max(static_cast<int>(e0) - kAnchorBelow, 1);

  // one 128-bit sum per unrolled load: four independent carry chains
  uint64_t lo[kUnroll], hi[kUnroll];
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) lo[u] = hi[u] = 0;
  for (int64_t base = warp_base; base < n4; base += stride * kUnroll) {
    float4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + lane + u * stride;
      v[u] = i < n4 ? __ldg(w4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    bool out = false;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      out |= window_add(__float_as_uint(v[u].x), B, lo[u], hi[u]);
      out |= window_add(__float_as_uint(v[u].y), B, lo[u], hi[u]);
      out |= window_add(__float_as_uint(v[u].z), B, lo[u], hi[u]);
      out |= window_add(__float_as_uint(v[u].w), B, lo[u], hi[u]);
    }
    if (__any_sync(kFull, out)) {
      // rare: weights outside the window go to their own exponent's bin
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const uint32_t c[4] = {__float_as_uint(v[u].x), __float_as_uint(v[u].y), __float_as_uint(v[u].z),
                               __float_as_uint(v[u].w)};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t ab = c[q] & 0x7FFFFFFFu;
          const int d = static_cast<int>(max(ab >> 23, 1u)) - B;
          bin_add_warp(ab, static_cast<unsigned>(d) > static_cast<unsigned>(kWindow), sbins);
        }
      }
    }
  }
  // the thread's sum is below 2^96 (fewer than 2^33 terms below 2^63): four
  // 24-bit chunks, chunk j of weight 2^(B + 24j - 150)
  uint64_t lo_t = lo[0], hi_t = hi[0];
#pragma unroll
  for (int u = 1; u < kUnroll; ++u)
    asm("add.cc.u64 %0, %0, %2;\n\taddc.u64 %1, %1, %3;" : "+l"(lo_t), "+l"(hi_t) : "l"(lo[u]), "l"(hi[u]));
  const uint64_t lo_s = lo_t, hi_s = hi_t;
  const uint32_t ch[4] = {static_cast<uint32_t>(lo_s & 0xFFFFFFull), static_cast<uint32_t>((lo_s >> 24) & 0xFFFFFFull),
                          static_cast<uint32_t>(((lo_s >> 48) | (hi_s << 16)) & 0xFFFFFFull),
                          static_cast<uint32_t>((hi_s >> 8) & 0xFFFFFFull)};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t s = __reduce_add_sync(kFull, ch[j]);   // < 32 * 2^24
    if (lane == 0 && s) atomicAdd(&sbins[B + 24 * j], static_cast<unsigned long long>(s));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kAbsmeanBins; i += kThreads) {
    const unsigned long long b = sbins[i];
    if (b) atomicAdd(&gbins[i], b);
  }
}

constexpr int kLimbs = 26;  // 16-bit limbs: 416 bits > 319 + 64 + carries

__device__ __forceinline__ uint32_t window16(const uint32_t* limb, int pos) {
  // bits [pos, pos + 16) of the limb array (pos >= 0)
  const int li = pos >> 4, off = pos & 15;
  uint32_t lo = li < kLimbs ? limb[li] : 0u;
  uint32_t hi = (li + 1) < kLimbs ? limb[li + 1] : 0u;
  return ((lo >> off) | (hi << (16 - off))) & 0xFFFFu;
}

// (rem * 2^16 + w) / n and its remainder, for rem < n < 2^39 and w < 2^16:
// a double-precision estimate of the quotient (< 2^16), corrected exactly in
// integers.
__device__ __forceinline__ uint64_t divstep(uint64_t& rem, uint32_t w, uint64_t n) {
  const uint64_t num = (rem << 16) | w;                 // < 2^55
  uint64_t q = static_cast<uint64_t>(__ddiv_rn(static_cast<double>(num), static_cast<double>(n)));
  int64_t r = static_cast<int64_t>(num) - static_cast<int64_t>(q * n);
  while (r < 0) { --q; r += static_cast<int64_t>(n); }
  while (r >= static_cast<int64_t>(n)) { ++q; r -= static_cast<int64_t>(n); }
  rem = static_cast<uint64_t>(r);
  return q;
}

__global__ void __launch_bounds__(32) absmean_finalize_kernel(const unsigned long long* __restrict__ bins,
                                                              uint64_t n, float* w_scale, float* mean_ws,
                                                              float* mean_out) {
  // S = sum_e bins[e] * 2^(max(e,1) - 1), in 16-bit limbs (units of 2^-149):
  // the lanes spread the bins' 16-bit pieces over shared 64-bit limb sums
  __shared__ unsigned long long accl[kLimbs + 1];
  const int lane = threadIdx.x;
  for (int i = lane; i <= kLimbs; i += 32) accl[i] = 0ull;
  __syncwarp();
  for (int e = lane; e < kAbsmeanBins; e += 32) {
    const uint64_t v = bins[e];
    if (!v) continue;
    const int s = (e > 1 ? e : 1) - 1;
    const int li = s >> 4, off = s & 15;
    for (int p = 0; p < 4; ++p) {  // v < 2^64: four 16-bit pieces
      const uint64_t piece = ((v >> (16 * p)) & 0xFFFFull) << off;   // < 2^31
      if (piece & 0xFFFFull) atomicAdd(&accl[li + p], piece & 0xFFFFull);
      if (piece >> 16) atomicAdd(&accl[li + p + 1], piece >> 16);
    }
  }
  __syncwarp();
  if (lane != 0) return;
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
    for (int i = tl - 1; i >= 0; --i) Q = (Q << 16) | divstep(rem, window16(limb, a + 16 * i), n);
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

namespace {

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

cudaError_t launch_bins_kernel(const float* w, int64_t n, uint64_t* bins, cudaStream_t stream) {
  const int64_t n4 = n / 4;
  int64_t blocks = (n4 + kThreads * kUnroll - 1) / (kThreads * kUnroll);
  const int64_t cap = 8LL * sm_count();
  blocks = blocks < cap ? blocks : cap;
  if (blocks < 1) blocks = 1;
  absmean_bins_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      reinterpret_cast<const float4*>(w), n4, reinterpret_cast<unsigned long long*>(bins));
  return cudaGetLastError();
}

cudaError_t launch_finalize_and_pack(const float* w, int64_t n, const uint64_t* bins, int64_t n_total,
                                     uint8_t* packed, float* w_scale, float* w_mean, float* mean_ws,
                                     cudaStream_t stream) {
  absmean_finalize_kernel<<<1, 32, 0, stream>>>(reinterpret_cast<const unsigned long long*>(bins),
                                                static_cast<uint64_t>(n_total), w_scale, mean_ws, w_mean);
  const int64_t nwords = n / 16;
  int64_t pblocks = (nwords + kThreads - 1) / kThreads;
  const int64_t cap = 16LL * sm_count();
  pblocks = pblocks < cap ? pblocks : cap;
  ternarise_pack_kernel<<<static_cast<unsigned>(pblocks), kThreads, 0, stream>>>(
      reinterpret_cast<const float4*>(w), nwords, w_scale, reinterpret_cast<uint32_t*>(packed));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pack(const float* w, int64_t N, int64_t K, uint8_t* packed, float* w_scale,
                        float* w_mean, const PackWorkspace& pws, cudaStream_t stream) {
  cudaError_t err = cudaMemsetAsync(pws.status, 0, 256 + kAbsmeanBins * sizeof(uint64_t), stream);
  if (err != cudaSuccess) return err;
  const int64_t n = N * K;
  err = launch_bins_kernel(w, n, pws.bins, stream);
  if (err != cudaSuccess) return err;
  return launch_finalize_and_pack(w, n, pws.bins, n, packed, w_scale, w_mean, pws.mean, stream);
}

cudaError_t launch_absmean_bins(const float* w, int64_t N, int64_t K, uint64_t* bins, cudaStream_t stream) {
  cudaError_t err = cudaMemsetAsync(bins, 0, kAbsmeanBins * sizeof(uint64_t), stream);
  if (err != cudaSuccess) return err;
  return launch_bins_kernel(w, N * K, bins, stream);
}

cudaError_t launch_pack_from_bins(const float* w, int64_t N, int64_t K, const uint64_t* bins, int64_t n_total,
                                  uint8_t* packed, float* w_scale, float* w_mean, const PackWorkspace& pws,
                                  cudaStream_t stream) {
  cudaError_t err = cudaMemsetAsync(pws.status, 0, 256, stream);
  if (err != cudaSuccess) return err;
  return launch_finalize_and_pack(w, N * K, bins, n_total, packed, w_scale, w_mean, pws.mean, stream);
}

}  // namespace bitlinear
