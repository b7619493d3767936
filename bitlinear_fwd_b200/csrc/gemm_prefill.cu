// Prefill engine (M > 16 tokens): the ternary x int8 contraction of
// BitLinear.forward (Falcon-Edge blog, section "Falcon-Edge, a series of
// universal models": F.linear, then post_quant_process and the bias add) as
// a dense int8 GEMM on the 5th-generation tensor cores.
//
// Tile: 128 tokens x 256 weight rows, k-blocks of 128; one CTA per tile.
//   warp 0      TMA producer: x_q tile (128 x 128 int8, 128-byte swizzle) and
//               the packed weight tile (256 rows x 32 bytes) per k-block
//   warp 1      MMA issuer: 4 x tcgen05.mma.kind::i8 (M=128, N=256, K=32)
//               per k-block into a 128 x 256 int32 accumulator in tensor memory
//   warp 2      tensor-memory allocation
//   warps 4..7  unpack each packed tile into the K-major, 128-byte-swizzled
//               int8 operand (one 32-bit word -> one 16-byte chunk of codes
//               c = u + 1 in {0,1,2}); after the last k-block, the epilogue:
//               tcgen05.ld of the accumulator, acc - sum_k q (removes the code
//               offset), y = acc / (s_x * s_w) (+ bias), bf16 stores.
// A 4-stage ring of (x tile, packed tile, unpacked tile) with three mbarriers
// per stage: full (TMA bytes landed), ready (unpacked), empty (MMAs done).
// Out-of-range rows/columns of a tile are zero-filled by TMA, so a code 0
// or an activation 0 adds nothing; the epilogue masks rows >= M, cols >= N.
// Every wait is bounded in time; a wait that gives up sets the status word,
// and the CTA still drains its copies and MMAs before freeing tensor memory.
#include "kernels.h"

namespace bitlinear {

namespace {

constexpr int BM = 128, BN = 256, BK = 128, STAGES = 4;
constexpr int kThreads = 256;
constexpr uint32_t kABytes = BM * BK;          // 16 KB
constexpr uint32_t kBuBytes = BN * BK;         // 32 KB
constexpr uint32_t kBpBytes = BN * BK / 4;     // 8 KB
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffBu = kOffA + STAGES * kABytes;
constexpr uint32_t kOffBp = kOffBu + STAGES * kBuBytes;
constexpr uint32_t kOffBar = kOffBp + STAGES * kBpBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;   // barriers + alignment slack
constexpr uint32_t kCodeMask = 0x03030303u;

__global__ void __launch_bounds__(kThreads, 1)
    gemm_prefill_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                        const ForwardArgs a, uint64_t wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* ready = full + STAGES;
  uint64_t* empty = ready + STAGES;
  uint64_t* accum = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* failed = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int num_kb = (a.K + BK - 1) / BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], 4);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    *failed = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int kb = 0;
      for (; kb < num_kb; ++kb) {
        const int s = kb % STAGES, round = kb / STAGES;
        if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1, wait_ns)) {
          *failed = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[s], kABytes + kBpBytes);
        // packed weights do not depend on the activation kernel
        tma_load_2d(smem + kOffBp + s * kBpBytes, &tm_w, &full[s], kb * (BK / 4), n0);
        if (kb == 0) pdl_wait_primary();
        tma_load_2d(smem + kOffA + s * kABytes, &tm_x, &full[s], kb * BK, m0);
      }
      // drain: the last copy issued into each stage has landed
      for (int s = 0; s < STAGES; ++s) {
        const int cnt = kb > s ? (kb - 1 - s) / STAGES + 1 : 0;   // copies issued into stage s
        if (cnt > 0 && !mbar_wait(&full[s], (cnt - 1) & 1, wait_ns)) *failed = 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = umma_idesc_i8(BM, BN, true, true);
      for (int kb = 0; kb < num_kb; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(&ready[s], (kb / STAGES) & 1, wait_ns)) {
          *failed = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + kOffA + s * kABytes);
        const uint32_t b_addr = smem_u32(smem + kOffBu + s * kBuBytes);
#pragma unroll
        for (int j = 0; j < BK / 32; ++j)
          umma_i8(tmem_base, umma_desc_sw128(a_addr + 32 * j), umma_desc_sw128(b_addr + 32 * j), idesc,
                  (kb | j) != 0);
        umma_commit(&empty[s]);
      }
      umma_commit(accum);   // fires once every MMA issued above has completed
    }
  } else if (warp >= 4) {
    // ---------------- unpack ----------------
    const int ut = threadIdx.x - 128;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % STAGES;
      if (!mbar_wait(&full[s], (kb / STAGES) & 1, wait_ns)) {
        *failed = 1;
        break;
      }
      const uint8_t* bp = smem + kOffBp + s * kBpBytes;
      uint8_t* bu = smem + kOffBu + s * kBuBytes;
#pragma unroll
      for (int it = 0; it < (BN * 2) / 128; ++it) {
        const int idx = ut + 128 * it;
        const int row = idx >> 1, half = idx & 1;
        const uint4 q = *reinterpret_cast<const uint4*>(bp + row * 32 + half * 16);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = half * 4 + j;   // 16-byte chunk = k 16c .. 16c + 15 of the block
          const uint4 out = make_uint4(w[j] & kCodeMask, (w[j] >> 2) & kCodeMask, (w[j] >> 4) & kCodeMask,
                                       (w[j] >> 6) & kCodeMask);
          *reinterpret_cast<uint4*>(bu + row * 128 + ((c ^ (row & 7)) << 4)) = out;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ready[s]);
    }

    // ---------------- epilogue ----------------
    const int ew = warp - 4;                  // tensor-memory lanes 32*ew .. 32*ew + 31
    const bool acc_ok = mbar_wait(accum, 0, wait_ns);
    tc_fence_after();
    pdl_wait_primary();
    if (!acc_ok) *failed = 1;
    if (acc_ok && !*failed) {
      const int m = m0 + 32 * ew + lane;
      const bool mv = m < a.M;
      const float s_w = *a.w_scale;
      const float d = mv ? __fmul_rn(a.s_x[m], s_w) : 1.0f;
      const int rs = mv ? a.rowsum[m] : 0;
      const bool vec = (a.N & 7) == 0;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * ew) << 16) + 32 * c, r);
        tmem_wait_ld();
        const int nb = n0 + 32 * c;
        if (!mv || nb >= a.N) continue;
        const size_t o = static_cast<size_t>(m) * a.N + nb;
        uint32_t yb[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float v[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int accv = static_cast<int>(r[i + h]) - rs;
            float y32 = __fdiv_rn(static_cast<float>(accv), d);
            if (a.bias && nb + i + h < a.N) y32 = __fadd_rn(y32, bf16_bits_to_f32(a.bias[nb + i + h]));
            v[h] = y32;
            if (nb + i + h < a.N) {
              if (a.acc_out) a.acc_out[o + i + h] = accv;
              if (a.y32_out) a.y32_out[o + i + h] = y32;
            }
          }
          yb[i / 2] = static_cast<uint32_t>(f32_to_bf16_bits(v[0])) |
                      (static_cast<uint32_t>(f32_to_bf16_bits(v[1])) << 16);
        }
        if (vec && nb + 32 <= a.N) {
          uint4* dst = reinterpret_cast<uint4*>(a.y + o);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(yb[4 * q], yb[4 * q + 1], yb[4 * q + 2], yb[4 * q + 3]);
        } else {
          for (int i = 0; i < 32 && nb + i < a.N; ++i)
            a.y[o + i] = static_cast<uint16_t>((i & 1) ? (yb[i / 2] >> 16) : (yb[i / 2] & 0xFFFFu));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *failed) report_status(a.status, kStatusTimeout);
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_prefill(const ForwardArgs& a, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  if (a.M <= 0) return cudaSuccess;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(gemm_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  CUtensorMap tm_x, tm_w;
  if (!encode_2d_u8(&tm_x, a.xq, a.K, a.M, a.K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  if (!encode_2d_u8(&tm_w, a.packed, a.K / 4, a.N, a.K / 4, BK / 4, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.N + BN - 1) / BN, (a.M + BM - 1) / BM, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_prefill_kernel, tm_x, tm_w, a, kWaitLimitNs);
}

}  // namespace bitlinear
