// Decode engine (M <= 16 tokens): the whole BitLinear forward of the
// Falcon-Edge blog (section "Falcon-Edge, a series of universal models":
// activation_norm_quant, F.linear on the unpacked ternary weights,
// post_quant_process and the bias add) in one kernel that streams the 2-bit
// packed weights once.
//
// Work split: a CTA owns 128 weight rows (8 warps x 16 rows) and a K-slice
// of whole "boxes" (512 k = 128 packed bytes per row); the C CTAs of a
// thread-block cluster (C in {1,2,4,8}, along K) own the slices of the same
// 128 rows.
//   1. At launch one thread issues TMA loads of the CTA's weight boxes
//      (128 rows x 128 bytes, 128-byte swizzle) into a shared-memory ring.
//      With resident weights this happens before the wait for the previous
//      kernel on the stream, so the stream overlaps that kernel's tail.
//   2. Activation quantisation of the CTA's slice of x: the per-token absmax
//      of the slice is exchanged across the cluster through distributed
//      shared memory, so every CTA derives the whole-row
//      s_x = 127 / max(absmax, 1e-5) (float32) and the same int8 values; the
//      int8 slice goes to shared memory (padded, swizzled for conflict-free
//      fragment loads) with its row sums.  TMA copies are asynchronous, so
//      the cluster barrier's release fence does not wait for the weight
//      stream.  Pre-quantised int8 input is copied in instead.
//   3. Warp w walks the boxes: per 256-k unit each thread takes one 16-byte
//      vector of two weight rows and the x words of the same k, and issues
//      mma.sync m16n8k32 (weights as A, u8; tokens as B, s8; a second
//      8-token tile for M > 8).  The codes c = u + 1 enter unshifted:
//      A_i = word & (0x03030303 << 2i) holds 4^i * c per byte lane, so field i
//      accumulates 4^i * sum(c q) in its own int32 accumulator; the fields
//      are combined with exact arithmetic shifts, and the slice's sum of q
//      is subtracted (sum(c q) - sum(q) = sum(u q)).
//   4. The cluster sums the slices' partial sums through distributed shared
//      memory; CTA r of the cluster finishes rows r*128/C ..:
//      y = acc / (s_x s_w) (+ bias) -> bf16.
// Rows beyond N and k beyond K are zero-filled by TMA (code 0) and x is
// zero-padded, so they add nothing.
//
// Fragment layout.  MMA row g of a warp's 16-row group is shared-memory row
// pi(g) = (g >> 1) | ((g & 1) << 2) (and pi(g) + 8), so that the two rows a
// quarter-warp reads differ in bit 2 and the 128-byte swizzle puts their
// chunks in disjoint bank groups.  Inside a unit thread (g, t) covers
// k = 64t .. 64t + 63: register a0 of field i / pair p holds
// k = 64t + 32p + 4i + {0..3}, a2 the same + 16; the B registers are the x
// words at byte offsets 64t + 32p + 4i and 64t + 32p + 16 + 4i.
#include <cooperative_groups.h>

#include "kernels.h"

namespace cg = cooperative_groups;

namespace bitlinear {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kRowsPerCta = 16 * kWarps;              // 128
constexpr int kBoxK = 512;                            // k per TMA box
constexpr int kBoxBytes = kRowsPerCta * kBoxK / 4;    // 16 KB
constexpr int kMaxRing = 4;                           // boxes in flight per CTA
constexpr int kSmemBudget = 110 * 1024;               // keeps two CTAs per SM
constexpr uint32_t kCodeMask = 0x03030303u;

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16-byte chunk position in a token row of the x slice: within every 16
// chunks, chunks 8..15 swap pairs (p ^ 2), so the four quad lanes t of a
// fragment load hit four different bank groups.
__device__ __forceinline__ int xs_chunk(int ch) { return ch ^ (((ch >> 3) & 1) << 1); }

__device__ __forceinline__ int mma_row_to_smem(int g) { return (g >> 1) | ((g & 1) << 2); }

// largest |x| of 16 bf16 values, as bf16 bits (finite values order like bits & 0x7FFF)
__device__ __forceinline__ uint32_t absmax16_bits(uint4 lo, uint4 hi) {
  uint32_t m = 0;
  m = __vmaxu2(m, lo.x & 0x7FFF7FFFu); m = __vmaxu2(m, lo.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, lo.z & 0x7FFF7FFFu); m = __vmaxu2(m, lo.w & 0x7FFF7FFFu);
  m = __vmaxu2(m, hi.x & 0x7FFF7FFFu); m = __vmaxu2(m, hi.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, hi.z & 0x7FFF7FFFu); m = __vmaxu2(m, hi.w & 0x7FFF7FFFu);
  return max(m & 0xFFFFu, m >> 16);
}

// q = clamp(round_half_even(x * s), -128, 127) for 16 bf16 values; adds sum(q)
__device__ __forceinline__ uint4 quant16(uint4 lo, uint4 hi, float s, int& sum) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  uint32_t out[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    uint32_t packed = 0;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int e = 4 * b + h;
      const uint32_t bits = (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu);
      int q = __float2int_rn(__fmul_rn(bf16_bits_to_f32(bits), s));
      q = min(127, max(-128, q));
      sum += q;
      packed |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * h);
    }
    out[b] = packed;
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

__device__ __forceinline__ int bytesum16(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  int s = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    s += static_cast<int8_t>(w[i] & 0xFF) + static_cast<int8_t>((w[i] >> 8) & 0xFF) +
         static_cast<int8_t>((w[i] >> 16) & 0xFF) + static_cast<int8_t>(w[i] >> 24);
  return s;
}

__device__ __forceinline__ uint32_t mapa_u32(uint32_t local_smem_addr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_smem_addr), "r"(rank));
  return r;
}
// 32-bit / 64-bit store into a peer CTA's shared memory that completes
// bytes on the peer's mbarrier.
__device__ __forceinline__ void st_async_u32(uint32_t raddr, uint32_t v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(raddr), "r"(v),
               "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t raddr, uint32_t v0, uint32_t v1, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(raddr),
               "r"(v0), "r"(v1), "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

constexpr int kChunkRegs = 4;   // 16-element x chunks a lane keeps in registers

struct SmemTail {
  uint64_t bar[kMaxRing];      // weight boxes
  uint64_t bar_amax;           // slice maxima from the peers
  uint64_t bar_red;            // partial sums from the peers
  uint32_t amax[8][16];        // [source rank][token] slice absmax (bf16 bits)
  uint32_t red_max[16];        // this slice's absmax per token, then the row's
  int red[8 * 16 * 16];        // [source rank][row_local][token] partials for this CTA's rows
  int rsum[16];                // this slice's sum of q per token
  float sx[16];                // s_x per token
  uint16_t bias[kRowsPerCta];  // bias of this CTA's output rows
};

size_t smem_bytes(int ntok, int ring, int boxes_per_cta) {
  return 1024 + static_cast<size_t>(ring) * kBoxBytes + static_cast<size_t>(ntok) * (boxes_per_cta * kBoxK + 16) +
         sizeof(SmemTail);
}

template <int NT, int C>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tm_w, const DecodeArgs a) {
  constexpr int NTOK = NT * 8;
  constexpr int R = kRowsPerCta / C;                  // output rows finished by this CTA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int ring = a.ring;
  const int S = a.xs_stride;                          // bytes per token row of the x slice
  uint8_t* rbuf = base;                               // ring of weight boxes, 1024-aligned
  int8_t* xs = reinterpret_cast<int8_t*>(base + ring * kBoxBytes);
  SmemTail& sm = *reinterpret_cast<SmemTail*>(base + ring * kBoxBytes + NTOK * S);

  pdl_launch_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int crank = blockIdx.x, rb = blockIdx.y;
  const int K = a.K, N = a.N, M = a.M;
  const int nbox_total = (K + kBoxK - 1) / kBoxK;
  const int b_begin = crank * a.boxes_per_cta;
  const int nb = max(0, min(nbox_total, b_begin + a.boxes_per_cta) - b_begin);
  const int npairs = (M + 1) >> 1;                    // token pairs exchanged per row

  if (threadIdx.x == 0) {
    for (int s = 0; s < ring; ++s) mbar_init(&sm.bar[s], 1);
    mbar_init(&sm.bar_amax, 1);
    mbar_init(&sm.bar_red, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_w);
    if (C > 1) {
      mbar_arrive_expect_tx(&sm.bar_amax, a.x ? static_cast<uint32_t>((C - 1) * M * 4) : 0u);
      mbar_arrive_expect_tx(&sm.bar_red, static_cast<uint32_t>((C - 1) * R * npairs * 8));
    }
  }
  if (threadIdx.x < 16) {
    sm.red_max[threadIdx.x] = 0u;
    sm.rsum[threadIdx.x] = 0;
  }
  __syncthreads();
  if (C > 1) cluster_arrive_relaxed();                // peers may push once their barriers exist

  int issued = 0;                                     // meaningful in thread 0 only
  auto issue = [&](int b) {
    const int s = b % ring;
    mbar_arrive_expect_tx(&sm.bar[s], kBoxBytes);
    tma_load_2d(rbuf + s * kBoxBytes, &tm_w, &sm.bar[s], (b_begin + b) * (kBoxK / 4), rb * kRowsPerCta);
    issued = b + 1;
  };
  float s_w = 0.0f;
  if (a.weights_early) {
    if (threadIdx.x == 0)
      for (int b = 0; b < min(nb, ring); ++b) issue(b);
    s_w = *a.w_scale;
  }
  // every peer's barriers exist from here on; the wait overlaps the
  // dependency wait below instead of the activation phase
  if (C > 1) cluster_wait();
  pdl_wait_primary();
  if (a.status && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *a.status = 0u;
  if (!a.weights_early) {
    if (threadIdx.x == 0)
      for (int b = 0; b < min(nb, ring); ++b) issue(b);
    s_w = *a.w_scale;
  }
  if (threadIdx.x < R) {
    const int n = rb * kRowsPerCta + crank * R + threadIdx.x;
    sm.bias[threadIdx.x] = (a.bias && n < N) ? a.bias[n] : static_cast<uint16_t>(0);
  }

  // ---------------- x slice -> int8 in shared memory ----------------
  // Items are (token m, 16-element chunk ch) with it = m * chunks + ch; the
  // chunk count is a multiple of 32, so the 32 items a warp holds at a time
  // belong to one token and reduce with one warp-wide max / sum.
  const int chunks = a.boxes_per_cta * (kBoxK / 16);  // 16-element chunks per token row of the slice
  const int k_begin = b_begin * kBoxK;
  const bool write_xq = rb == 0 && a.xq_out != nullptr;
  if (a.x) {
    const int items = M * chunks;
    uint4 xr[kChunkRegs][2];
#pragma unroll
    for (int j = 0; j < kChunkRegs; ++j) {
      const int it = threadIdx.x + kThreads * j;
      const int m = it / chunks, ch = it - m * chunks;
      const int k0 = k_begin + 16 * ch;
      uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
      if (it < items && k0 < K) {
        const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(m) * K + k0);
        lo = __ldg(src);
        hi = __ldg(src + 1);
      }
      xr[j][0] = lo;
      xr[j][1] = hi;
    }
    // slice absmax per token: registers, then the rest of the slice
    for (int j = 0; j * kThreads < items; ++j) {
      const int it = threadIdx.x + kThreads * j;       // warp-uniform token
      const int m = min(it, items - 1) / chunks;
      uint32_t mx = 0;
      if (it < items) {
        if (j < kChunkRegs) {
#pragma unroll
          for (int jj = 0; jj < kChunkRegs; ++jj)
            if (jj == j) mx = absmax16_bits(xr[jj][0], xr[jj][1]);
        } else {
          const int ch = it - m * chunks, k0 = k_begin + 16 * ch;
          if (k0 < K) {
            const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(m) * K + k0);
            mx = absmax16_bits(__ldg(src), __ldg(src + 1));
          }
        }
      }
      mx = __reduce_max_sync(0xffffffffu, mx);
      if (lane == 0 && it < items) atomicMax(&sm.red_max[m], mx);
    }
    __syncthreads();
    if (C > 1) {
      if (threadIdx.x < M * C) {                      // thread (m, r) sends token m's maximum to rank r
        const int m = threadIdx.x / C, r = threadIdx.x - m * C;
        const uint32_t v = sm.red_max[m];
        if (r == crank) sm.amax[crank][m] = v;
        else st_async_u32(mapa_u32(smem_u32(&sm.amax[crank][m]), r), v, mapa_u32(smem_u32(&sm.bar_amax), r));
      }
      if (!mbar_wait(&sm.bar_amax, 0, kWaitLimitNs)) report_status(a.status, kStatusTimeout);
      __syncthreads();
      if (threadIdx.x < M) {
        uint32_t mx = 0;
#pragma unroll
        for (int r = 0; r < C; ++r) mx = max(mx, sm.amax[r][threadIdx.x]);
        sm.red_max[threadIdx.x] = mx;
      }
    }
    __syncthreads();
    if (threadIdx.x < M) {
      const float sxv = __fdiv_rn(127.0f, fmaxf(bf16_bits_to_f32(sm.red_max[threadIdx.x]), 1e-5f));
      sm.sx[threadIdx.x] = sxv;
      if (write_xq && crank == 0 && a.sx_out) a.sx_out[threadIdx.x] = sxv;
    }
    __syncthreads();
    for (int j = 0; j * kThreads < items; ++j) {
      const int it = threadIdx.x + kThreads * j;
      const int m = min(it, items - 1) / chunks, ch = it - m * chunks;
      const int k0 = k_begin + 16 * ch;
      int sum = 0;
      if (it < items) {
        uint4 q = make_uint4(0, 0, 0, 0);
        if (k0 < K) {
          uint4 lo, hi;
          if (j < kChunkRegs) {
#pragma unroll
            for (int jj = 0; jj < kChunkRegs; ++jj)
              if (jj == j) { lo = xr[jj][0]; hi = xr[jj][1]; }
          } else {
            const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(m) * K + k0);
            lo = __ldg(src);
            hi = __ldg(src + 1);
          }
          q = quant16(lo, hi, sm.sx[m], sum);
          if (write_xq) *reinterpret_cast<uint4*>(a.xq_out + static_cast<size_t>(m) * K + k0) = q;
        }
        *reinterpret_cast<uint4*>(xs + m * S + 16 * xs_chunk(ch)) = q;
      }
      sum = __reduce_add_sync(0xffffffffu, sum);
      if (lane == 0 && it < items) atomicAdd(&sm.rsum[m], sum);
    }
  } else {
    // pre-quantised input: copy the int8 slice, sum it per token
    const int items = M * chunks;
    for (int j = 0; j * kThreads < items; ++j) {
      const int it = threadIdx.x + kThreads * j;
      const int m = min(it, items - 1) / chunks, ch = it - m * chunks;
      const int k0 = k_begin + 16 * ch;
      int sum = 0;
      if (it < items) {
        uint4 q = make_uint4(0, 0, 0, 0);
        if (k0 < K) {
          q = __ldg(reinterpret_cast<const uint4*>(a.xq + static_cast<size_t>(m) * K + k0));
          sum = bytesum16(q);
        }
        *reinterpret_cast<uint4*>(xs + m * S + 16 * xs_chunk(ch)) = q;
      }
      sum = __reduce_add_sync(0xffffffffu, sum);
      if (lane == 0 && it < items) atomicAdd(&sm.rsum[m], sum);
    }
    if (threadIdx.x < M) sm.sx[threadIdx.x] = a.s_x[threadIdx.x];
  }
  // padding token rows M .. NTOK-1 read as zeros
  for (int it = threadIdx.x; it < (NTOK - M) * chunks; it += kThreads) {
    const int m = M + it / chunks, ch = it % chunks;
    *reinterpret_cast<uint4*>(xs + m * S + 16 * xs_chunk(ch)) = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();

  // ---------------- contraction over the slice ----------------
  int acc[4][NT][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[i][nt][r] = 0;

  const int r0 = warp * 16 + mma_row_to_smem(g);     // shared-memory rows r0 and r0 + 8
  bool ok = true;
  for (int b = 0; b < nb; ++b) {
    const int s = b % ring;
    if (ok) ok = mbar_wait(&sm.bar[s], (b / ring) & 1, kWaitLimitNs);
    if (ok) {
      const uint8_t* box = rbuf + s * kBoxBytes;
#pragma unroll
      for (int v = 0; v < 2; ++v) {                   // two 256-k units per box
        const int cw = 4 * v + t;                     // 16-byte chunk of the 128-byte row
        const uint4 wa = *reinterpret_cast<const uint4*>(box + r0 * 128 + ((cw ^ (r0 & 7)) << 4));
        const uint4 wb = *reinterpret_cast<const uint4*>(box + (r0 + 8) * 128 + ((cw ^ ((r0 + 8) & 7)) << 4));
        const uint32_t w0[4] = {wa.x, wa.y, wa.z, wa.w};
        const uint32_t w1[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
          // x words 8pr .. 8pr + 7 of the thread's 64-byte span (chunks 2pr, 2pr + 1)
          uint32_t xw[NT][8];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int8_t* xrow = xs + (nt * 8 + g) * S;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const uint4 xv =
                  *reinterpret_cast<const uint4*>(xrow + 16 * xs_chunk(32 * b + 16 * v + 4 * t + 2 * pr + c));
              xw[nt][4 * c + 0] = xv.x; xw[nt][4 * c + 1] = xv.y;
              xw[nt][4 * c + 2] = xv.z; xw[nt][4 * c + 3] = xv.w;
            }
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t mask = kCodeMask << (2 * i);
            const uint32_t a0 = w0[2 * pr] & mask, a1 = w1[2 * pr] & mask;
            const uint32_t a2 = w0[2 * pr + 1] & mask, a3 = w1[2 * pr + 1] & mask;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_u8s8(acc[i][nt], a0, a1, a2, a3, xw[nt][i], xw[nt][4 + i]);
          }
        }
      }
    }
    if (b + ring < nb) {               // refill the slot once every warp is done with it
      __syncthreads();
      if (threadIdx.x == 0 && ok) issue(b + ring);
    }
  }
  if (threadIdx.x == 0) {
    // drain: every box issued into the ring has landed before the CTA exits
    for (int s = 0; s < ring && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / ring) * ring;
      if (!mbar_wait(&sm.bar[s], (last / ring) & 1, kWaitLimitNs)) ok = false;
    }
  }
  if (!ok) report_status(a.status, kStatusTimeout);

  // ---------------- partial sums -> the CTA that finishes each row ----------------
  // value (row, token): sum over this slice of c*q, minus the slice's sum of q
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int m0 = nt * 8 + 2 * t;                   // tokens m0, m0 + 1 of this thread
    if (m0 < M) {
      const int rs0 = sm.rsum[m0], rs1 = (m0 + 1 < M) ? sm.rsum[m0 + 1] : 0;
      int c[4];
#pragma unroll
      for (int r = 0; r < 4; ++r)
        c[r] = acc[0][nt][r] + (acc[1][nt][r] >> 2) + (acc[2][nt][r] >> 4) + (acc[3][nt][r] >> 6);
#pragma unroll
      for (int h = 0; h < 2; ++h) {                  // rows r0 and r0 + 8
        const int row = r0 + 8 * h;
        const int owner = row / R, rl = row - owner * R;
        int* dst = &sm.red[(crank * R + rl) * 16 + m0];
        const uint32_t v0 = static_cast<uint32_t>(c[2 * h] - rs0), v1 = static_cast<uint32_t>(c[2 * h + 1] - rs1);
        if (C == 1 || owner == crank) {
          dst[0] = static_cast<int>(v0);
          dst[1] = static_cast<int>(v1);
        } else {
          st_async_v2(mapa_u32(smem_u32(dst), owner), v0, v1, mapa_u32(smem_u32(&sm.bar_red), owner));
        }
      }
    }
  }
  __syncthreads();
  if (C > 1 && !mbar_wait(&sm.bar_red, 0, kWaitLimitNs)) report_status(a.status, kStatusTimeout);

  // ---------------- epilogue for this CTA's R rows ----------------
  for (int idx = threadIdx.x; idx < R * M; idx += kThreads) {
    const int m = idx / R, rl = idx - m * R;
    const int n = rb * kRowsPerCta + crank * R + rl;
    if (n >= N) continue;
    int accv = 0;
#pragma unroll
    for (int r = 0; r < C; ++r) accv += sm.red[(r * R + rl) * 16 + m];
    const float d = __fmul_rn(sm.sx[m], s_w);
    float y32 = __fdiv_rn(static_cast<float>(accv), d);
    if (a.bias) y32 = __fadd_rn(y32, bf16_bits_to_f32(sm.bias[rl]));
    const size_t o = static_cast<size_t>(m) * N + n;
    a.y[o] = f32_to_bf16_bits(y32);
    if (a.acc_out) a.acc_out[o] = accv;
    if (a.y32_out) a.y32_out[o] = y32;
  }
}

template <int NT, int C>
cudaError_t launch_c(const CUtensorMap& tm, const DecodeArgs& a, int row_blocks, size_t smem,
                     cudaStream_t stream) {
  auto kern = decode_kernel<NT, C>;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, row_blocks, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tm, a);
}

template <int NT>
cudaError_t launch_nt(const CUtensorMap& tm, const DecodeArgs& a, int C, int row_blocks, size_t smem,
                      cudaStream_t stream) {
  switch (C) {
    case 1: return launch_c<NT, 1>(tm, a, row_blocks, smem, stream);
    case 2: return launch_c<NT, 2>(tm, a, row_blocks, smem, stream);
    case 4: return launch_c<NT, 4>(tm, a, row_blocks, smem, stream);
    default: return launch_c<NT, 8>(tm, a, row_blocks, smem, stream);
  }
}

}  // namespace

DecodePlan plan_decode(int M, int N, int K, int num_sms) {
  DecodePlan p;
  const int nbox = (K + kBoxK - 1) / kBoxK;
  p.row_blocks = (N + kRowsPerCta - 1) / kRowsPerCta;
  const int ntok = M <= 8 ? 8 : 16;
  auto fill = [&](int c) {
    p.cluster = c;
    p.boxes_per_cta = (nbox + c - 1) / c;
    p.ring = p.boxes_per_cta < kMaxRing ? p.boxes_per_cta : kMaxRing;
    p.smem = smem_bytes(ntok, p.ring, p.boxes_per_cta);
  };
  int C = 1;
  fill(C);
  // split K over a cluster until the grid covers the SMs and a CTA fits twice per SM
  while (C < 8 && 2 * C <= nbox && (p.row_blocks * C < num_sms || p.smem > static_cast<size_t>(kSmemBudget))) {
    C *= 2;
    fill(C);
  }
  return p;
}

cudaError_t launch_decode(DecodeArgs a, int num_sms, cudaStream_t stream) {
  if (a.M <= 0) return cudaSuccess;
  const DecodePlan p = plan_decode(a.M, a.N, a.K, num_sms);
  a.boxes_per_cta = p.boxes_per_cta;
  a.ring = p.ring;
  a.xs_stride = p.boxes_per_cta * kBoxK + 16;
  if (p.smem > 227 * 1024) return cudaErrorInvalidValue;
  CUtensorMap tm;
  if (!encode_2d_u8(&tm, a.packed, static_cast<uint64_t>(a.K) / 4, static_cast<uint64_t>(a.N),
                    static_cast<uint64_t>(a.K) / 4, kBoxK / 4, kRowsPerCta, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  return a.M <= 8 ? launch_nt<1>(tm, a, p.cluster, p.row_blocks, p.smem, stream)
                  : launch_nt<2>(tm, a, p.cluster, p.row_blocks, p.smem, stream);
}

}  // namespace bitlinear
