// Decode engine (M <= 16 tokens): the ternary x int8 contraction of
// BitLinear.forward (Falcon-Edge blog, section "Falcon-Edge, a series of
// universal models"; F.linear followed by post_quant_process and the bias
// add), streamed from the 2-bit packed weights.
//
// Work split:
//   * a CTA owns 128 weight rows (8 warps x 16 rows) and a K-slice; the
//     CTAs of a thread-block cluster (up to 8, along K) own the slices of
//     the same 128 rows and reduce their partial sums through distributed
//     shared memory;
//   * a warp owns 16 rows and walks the slice in units of 256 k: per unit
//     each thread loads one 16-byte vector of row g and one of row g + 8
//     (64 weights each) with streaming loads, and the 64 bytes of x_q that
//     the same k cover for its token column.
// Contraction: mma.sync m16n8k32 with the weights as A (u8) and the tokens
// as B (s8, 8 per tile; a second tile for M > 8).  The 2-bit codes c = u + 1
// are fed without shifting: A_i = word & (0x03030303 << 2i) holds 4^i * c
// in each byte lane, so field i accumulates 4^i * sum(c * q) in its own
// int32 accumulator; the four are combined with exact arithmetic shifts.
// sum(c * q) - sum(q) = sum(u * q) removes the code offset.  Weight rows
// beyond N and k beyond K read as code 0 and x as 0, adding nothing.
//
// The k order inside a unit is permuted identically for A and B: thread
// (g, t) of the warp covers k = 64t .. 64t + 63 of the unit; register a0 of
// field i / pair p holds k = 64t + 32p + 4i + {0..3}, a2 holds the same + 16,
// and the matching B registers are the x words at byte offsets
// 64t + 32p + 4i and 64t + 32p + 16 + 4i.
#include <cooperative_groups.h>

#include "kernels.h"

namespace cg = cooperative_groups;

namespace bitlinear {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kRowsPerCta = 16 * kWarps;   // 128
constexpr int kUnitK = 256;                // k per unit
constexpr int kUnitBytes = kUnitK / 4;     // packed bytes per row per unit
constexpr uint32_t kCodeMask = 0x03030303u;

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int NT, int P>   // NT token tiles of 8; P units of weights in flight per warp
__global__ void __launch_bounds__(kThreads, 2) gemv_decode_kernel(const ForwardArgs a, int units_per_cta) {
  __shared__ int part[NT * 8][kRowsPerCta];   // partial sums [token][row]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int C = gridDim.x;                  // cluster size along K
  const int crank = blockIdx.x;
  const int rb = blockIdx.y;
  const int K = a.K, N = a.N, M = a.M;
  const int units_total = (K + kUnitK - 1) / kUnitK;
  const int u_begin = crank * units_per_cta;
  const int u_end = min(units_total, u_begin + units_per_cta);
  const int nunits = max(0, u_end - u_begin);
  const size_t row_bytes = static_cast<size_t>(K) / 4;

  const int row0 = rb * kRowsPerCta + warp * 16 + g;    // this thread's rows: row0, row0 + 8
  const bool v0 = row0 < N, v1 = row0 + 8 < N;
  const uint8_t* w0 = a.packed + static_cast<size_t>(v0 ? row0 : 0) * row_bytes + 16 * t;
  const uint8_t* w1 = a.packed + static_cast<size_t>(v1 ? row0 + 8 : 0) * row_bytes + 16 * t;

  uint32_t wv[P][2][4];
  auto load_w = [&](int slot, int ui) {
    const int u = u_begin + ui;
    const bool kin = ui < nunits && (u * kUnitK + 64 * t) < K;
    uint4 r0 = make_uint4(0, 0, 0, 0), r1 = make_uint4(0, 0, 0, 0);
    if (kin && v0) r0 = ld_stream_v4(w0 + static_cast<size_t>(u) * kUnitBytes);
    if (kin && v1) r1 = ld_stream_v4(w1 + static_cast<size_t>(u) * kUnitBytes);
    wv[slot][0][0] = r0.x; wv[slot][0][1] = r0.y; wv[slot][0][2] = r0.z; wv[slot][0][3] = r0.w;
    wv[slot][1][0] = r1.x; wv[slot][1][1] = r1.y; wv[slot][1][2] = r1.z; wv[slot][1][3] = r1.w;
  };

  // The packed weights do not depend on the activation kernel: start
  // streaming them before waiting for it.
#pragma unroll
  for (int p = 0; p < P; ++p) load_w(p, p);
  pdl_wait_primary();

  int acc[4][NT][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[i][nt][r] = 0;

  for (int base = 0; base < nunits; base += P) {
#pragma unroll
    for (int p = 0; p < P; ++p) {
      const int ui = base + p;
      if (ui < nunits) {
        const int u = u_begin + ui;
        const bool kin = (u * kUnitK + 64 * t) < K;
        uint32_t xw[NT][16];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int m = nt * 8 + g;
          const uint4* xp = reinterpret_cast<const uint4*>(a.xq + static_cast<size_t>(m < M ? m : 0) * K +
                                                           static_cast<size_t>(u) * kUnitK + 64 * t);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (kin && m < M) v = __ldg(xp + c);
            xw[nt][4 * c + 0] = v.x; xw[nt][4 * c + 1] = v.y;
            xw[nt][4 * c + 2] = v.z; xw[nt][4 * c + 3] = v.w;
          }
        }
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t mask = kCodeMask << (2 * i);
            const uint32_t a0 = wv[p][0][2 * pr] & mask;
            const uint32_t a1 = wv[p][1][2 * pr] & mask;
            const uint32_t a2 = wv[p][0][2 * pr + 1] & mask;
            const uint32_t a3 = wv[p][1][2 * pr + 1] & mask;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma_u8s8(acc[i][nt], a0, a1, a2, a3, xw[nt][8 * pr + i], xw[nt][8 * pr + 4 + i]);
          }
        }
        load_w(p, ui + P);   // refill this slot (zero beyond the slice)
      }
    }
  }

  // combine the four fields (exact: field i is a multiple of 4^i) and park
  // the partial sums in shared memory
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    int c[4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
      c[r] = acc[0][nt][r] + (acc[1][nt][r] >> 2) + (acc[2][nt][r] >> 4) + (acc[3][nt][r] >> 6);
    const int lr = warp * 16 + g;
    part[nt * 8 + 2 * t][lr] = c[0];
    part[nt * 8 + 2 * t + 1][lr] = c[1];
    part[nt * 8 + 2 * t][lr + 8] = c[2];
    part[nt * 8 + 2 * t + 1][lr + 8] = c[3];
  }

  cg::cluster_group cluster = cg::this_cluster();
  if (C > 1) cluster.sync(); else __syncthreads();

  // epilogue: CTA `crank` finishes rows [crank * R, (crank + 1) * R) of the block
  const int R = kRowsPerCta / C;
  const int r_off = crank * R;
  const int* peer[8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
    peer[r] = (r < C) ? (C > 1 ? cluster.map_shared_rank(&part[0][0], r) : &part[0][0]) : nullptr;
  const float s_w = *a.w_scale;
  for (int idx = threadIdx.x; idx < R * M; idx += kThreads) {
    const int m = idx / R, nn = idx - m * R;
    const int n = rb * kRowsPerCta + r_off + nn;
    if (n >= N) continue;
    int sum = 0;
    for (int r = 0; r < C; ++r) sum += peer[r][m * kRowsPerCta + r_off + nn];
    const int accv = sum - a.rowsum[m];
    const float d = __fmul_rn(a.s_x[m], s_w);
    float y32 = __fdiv_rn(static_cast<float>(accv), d);
    if (a.bias) y32 = __fadd_rn(y32, bf16_bits_to_f32(a.bias[n]));
    const size_t o = static_cast<size_t>(m) * N + n;
    a.y[o] = f32_to_bf16_bits(y32);
    if (a.acc_out) a.acc_out[o] = accv;
    if (a.y32_out) a.y32_out[o] = y32;
  }
  if (C > 1) cluster.sync();   // peers' shared memory must outlive their readers
}

template <int NT, int P>
cudaError_t launch_variant(const ForwardArgs& a, int C, int units_per_cta, int row_blocks,
                           cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, row_blocks, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemv_decode_kernel<NT, P>, a, units_per_cta);
}

}  // namespace

cudaError_t launch_gemv_decode(const ForwardArgs& a, int num_sms, cudaStream_t stream) {
  if (a.M <= 0) return cudaSuccess;
  const int units = (a.K + kUnitK - 1) / kUnitK;
  const int row_blocks = (a.N + kRowsPerCta - 1) / kRowsPerCta;
  // Split K over a cluster until there are about two CTAs per SM.
  int C = 1;
  while (C < 8 && 2 * C <= units && row_blocks * C < 2 * num_sms) C *= 2;
  const int upc = (units + C - 1) / C;
  if (a.M <= 8) return launch_variant<1, 4>(a, C, upc, row_blocks, stream);
  return launch_variant<2, 4>(a, C, upc, row_blocks, stream);
}

}  // namespace bitlinear
