// Prefill engine (M > 16 tokens): the ternary x int8 contraction of
// BitLinear.forward (Falcon-Edge blog, section "Falcon-Edge, a series of
// universal models": F.linear, then post_quant_process and the bias add) as
// a dense int8 GEMM on the 5th-generation tensor cores.
//
// The weights are the MMA's A operand and come from tensor memory; the
// tokens are the B operand and come from shared memory:
//   D[weight row n][token m] += A[n][k] * B[m][k],  M_mma = 128 weight rows,
//   N_mma = BT = 192 tokens, K = 32 per instruction.
// Tile shape.  Per 128 k the shared memory of an SM carries the x tile twice
// (written by TMA, read by the MMA) plus the 2-bit codes; with 192 tokens
// that is 56 KB against 384 cycles of MMA, where 128 tokens would be 40 KB
// against 256 cycles: the wider tile moves fewer bytes per MMA cycle.
// Tensor memory holds two 192-column accumulators (the epilogue of one tile
// runs while the MMAs of the next one fill the other) and two 64-column
// stages of unpacked weights: 512 columns.
// Stages of 256 k.  The MMA warp waits once and commits twice per stage, so
// a stage carries eight MMAs: a loop of four MMAs between one wait and two
// commits ran at 78% of the tensor rate on B200, eight at 100%.
// Persistent kernel: one CTA per SM walks the 128 x 192 tiles (weight tile
// fastest, so the CTAs running at the same time share the token tile in L2)
// through a 3-stage operand ring in shared memory:
//   warp 0       TMA producer: x tile (192 tokens x 256 int8 as two
//                128-byte-swizzled boxes of 128 k) + packed weight tile (128
//                rows x 64 bytes, 64-byte swizzle) per stage
//   warp 1       MMA issuer: 8 x tcgen05.mma.kind::i8 per stage (4 when its
//                second half lies beyond K), A from tensor-memory stage
//                (stage & 1), into accumulator buffer (tile & 1); commits free
//                the shared stage and the A stage
//   warp 2       tensor-memory allocation
//   warps 4..11  weight unpack, two warps per tensor-memory lane quarter, one
//                per 128-k half of a stage: thread = weight row; its 32
//                packed bytes of the half become 32 registers of codes c =
//                u + 1 (one word -> four registers of four consecutive k)
//                and one tcgen05.st of 32 columns; the swizzled rows keep a
//                quarter-warp's reads in distinct banks.  (One warp per
//                quarter took longer per stage than the stage's MMAs.)
//   warps 12..19 epilogue of the previous tile while the MMAs of the next one
//                run; warps w and w + 4 share a lane quarter of tensor memory
//                and take one half of the tile's tokens each: tcgen05.ld of a
//                row's 96 accumulators (the next 32 columns load while 32 are
//                processed), acc - sum_k q (code offset), y = acc / (s_x s_w)
//                (+ bias) as a product with the double 1 / (s_x s_w) of the
//                token, bf16 into a shared staging tile that one thread
//                stores with TMA (plain stores when y's rows are not 16-byte
//                multiples or a debug output is asked for); s_w is the scale
//                of the row's group (stacked layers)
// Registers: 20 warps launch at 96 per thread; then the warpgroups set
// their own budgets (setmaxnreg): 56 for warps 0..3, 72 for the unpack
// warps, 136 for the epilogue.
// Barriers: per shared stage full (TMA bytes landed) and empty (MMAs done);
// per A stage ready (written) and afree (MMAs done); per accumulator buffer
// acc_full (tile's MMAs done) and acc_empty (epilogue has read it).
// Out-of-range rows/columns are zero-filled by TMA, so a code 0 or an
// activation 0 adds nothing; the epilogue masks rows >= N and tokens >= M
// (the tile store clips them).
// Every wait is bounded in time; a wait that gives up sets the status word,
// and the CTA drains its copies and MMAs (with the fixed 1 s limit) before
// freeing tensor memory.
#include "kernels.h"

namespace bitlinear {

namespace {

#ifndef BITLINEAR_GEMM_BT
#define BITLINEAR_GEMM_BT 192
#endif
constexpr int BW = 128;                      // weight rows per tile (MMA M)
constexpr int BT = BITLINEAR_GEMM_BT;        // tokens per tile (MMA N)
constexpr int BK = 256;                      // k per block (stage)
constexpr int STAGES = 3;                    // shared-memory operand stages
constexpr int ASTAGES = 2;                   // tensor-memory stages of unpacked weights
constexpr int kThreads = 640;                // 20 warps: see the roles above
// Register budgets per warpgroup after the set-up (setmaxnreg): the TMA,
// MMA and allocation warps need few, the unpack warps hold 32 codes, the
// epilogue warps two 32-column accumulator chunks.  Launched at 96 per
// thread (640 x 96 = 61440 of the SM's 65536); the budgets below sum to
// 32 x (4 x 56 + 8 x 72 + 8 x 136) = 60416, within the launch's share, so
// the raise never waits on registers that no warpgroup gives back.
constexpr uint32_t kRegsRoles = 56, kRegsUnpack = 72, kRegsEpi = 136;
static_assert(4 * kRegsRoles + 8 * kRegsUnpack + 8 * kRegsEpi <= kThreads / 32 * 96,
              "the warpgroups' register budgets fit the launch's");
constexpr int kEpiWarps = 8;                 // two per tensor-memory lane quarter
constexpr int kEpiCols = BT / 2;             // tokens of a tile per epilogue warp
constexpr int kEpiChunks = kEpiCols / 32;
constexpr uint32_t kXHalf = BT * 128;        // one 128-k half of the x tile (a 128-byte-swizzled TMA box)
constexpr uint32_t kXBytes = 2 * kXHalf;     // x tile per stage
constexpr uint32_t kWpBytes = BW * BK / 4;   // 8 KB packed weights per stage (64-byte-swizzled rows)
constexpr uint32_t kACols = BK / 4;          // tensor-memory columns of one A stage
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kCodeMask = 0x03030303u;
static_assert(BT % 64 == 0 && BT <= 256, "two halves of whole 32-column chunks; MMA N <= 256");
static_assert(2 * BT + ASTAGES * kACols <= kTmemCols, "two accumulators and the A stages fit in tensor memory");
static_assert(kXHalf % 1024 == 0 && kWpBytes % 512 == 0, "swizzle atoms stay aligned");

constexpr uint32_t kStageBytes = BT * BW * 2;          // bf16 y tile [BT tokens][BW rows] for the TMA store
constexpr uint32_t kOffX = 0;
constexpr uint32_t kOffWp = kOffX + STAGES * kXBytes;
constexpr uint32_t kOffStage = (kOffWp + STAGES * kWpBytes + 1023) & ~1023u;
constexpr uint32_t kOffD = kOffStage + kStageBytes;          // per token: 1 / d in double [BT], or s_x
constexpr uint32_t kOffRs = kOffD + 8 * BT;                  // row sums per token [BT]
constexpr uint32_t kOffBar = kOffRs + 4 * BT;
constexpr uint32_t kSmemBytes = kOffBar + 512 + 1024;        // + barriers, alignment slack
// tcgen05.alloc of all 512 columns waits until the columns are free, with no
// time limit.  It never waits here because two CTAs of this kernel cannot
// share an SM (their shared memory exceeds the SM's 228 KB), and no other
// kernel of the library allocates tensor memory beside it (the int8 rate
// measurement runs on its own).
static_assert(2 * kSmemBytes > 228 * 1024, "one GEMM CTA per SM keeps the 512-column allocation uncontended");
static_assert(kSmemBytes <= 227 * 1024, "fits the shared memory of one CTA");
static_assert(kOffD % 16 == 0 && kOffRs % 16 == 0, "per-token values are read as 16-byte vectors");

__global__ void __launch_bounds__(kThreads, 1)
    gemm_prefill_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_y, const ForwardArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* empty = full + STAGES;
  uint64_t* ready = empty + STAGES;           // [ASTAGES]
  uint64_t* afree = ready + ASTAGES;          // [ASTAGES]
  uint64_t* acc_full = afree + ASTAGES;       // [2]
  uint64_t* acc_empty = acc_full + 2;         // [2]
  uint64_t* drain = acc_empty + 2;            // every issued MMA has completed
  uint64_t* stall_bar = drain + 1;            // never signalled (test hook)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stall_bar + 1);
  volatile int* failed = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* drain_bad = failed + 1;       // a drain gave up: MMAs may still run
  double* rcp_s = reinterpret_cast<double*>(smem + kOffD);   // per token, when the tile has one scale
  float* sx_s = reinterpret_cast<float*>(smem + kOffD);      // per token s_x, when it has several
  int* rs_s = reinterpret_cast<int*>(smem + kOffRs);
  uint16_t* stage = reinterpret_cast<uint16_t*>(smem + kOffStage);   // y tile, token-major
  const uint64_t wait_ns = a.wait_ns;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_kb = (a.K + BK - 1) / BK;
  const int wtiles = (a.N + BW - 1) / BW;
  const int ntiles = wtiles * ((a.M + BT - 1) / BT);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < ASTAGES; ++s) {
      mbar_init(&ready[s], 8);                     // the eight unpack warps
      mbar_init(&afree[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    mbar_init(stall_bar, 1);
    *failed = 0;
    *drain_bad = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    if (a.y_tma) tma_prefetch_desc(&tm_y);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_a = tmem_base + 2 * BT;     // A stages after the two accumulators

  // Each warpgroup sets its register budget at the head of its role (every
  // thread of the warpgroup, converged after the barrier above).
  if (warp < 4) {
   setmaxnreg_dec<kRegsRoles>();
   if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int g = 0;                                  // k-blocks issued by this CTA
      bool waited = false;
      for (int tile = blockIdx.x; tile < ntiles && !*failed; tile += gridDim.x) {
        const int n0 = (tile % wtiles) * BW, m0 = (tile / wtiles) * BT;
        for (int kb = 0; kb < num_kb; ++kb, ++g) {
          const int s = g % STAGES, round = g / STAGES;
          if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1, wait_ns)) {
            *failed = 1;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kXBytes + kWpBytes);
          // packed weights do not depend on the activation kernel
          tma_load_2d(smem + kOffWp + s * kWpBytes, &tm_w, &full[s], kb * (BK / 4), n0);
          if (!waited) {
            pdl_wait_primary();
            waited = true;
          }
          // two 128-k halves (a half beyond K arrives zero-filled)
          tma_load_2d(smem + kOffX + s * kXBytes, &tm_x, &full[s], kb * BK, m0);
          tma_load_2d(smem + kOffX + s * kXBytes + kXHalf, &tm_x, &full[s], kb * BK + 128, m0);
        }
      }
      // drain: the last copy issued into each stage has landed.  The drain
      // keeps the fixed limit whatever the main loop's limit is, so that no
      // copy is still writing shared memory when the CTA exits.
      for (int s = 0; s < STAGES; ++s) {
        const int cnt = g > s ? (g - 1 - s) / STAGES + 1 : 0;
        if (cnt > 0 && !mbar_wait(&full[s], (cnt - 1) & 1, kWaitLimitNs)) {
          *failed = 1;
          *drain_bad = 1;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = umma_idesc_i8(BW, BT, true, true);
      int g = 0, j = 0;
      // forced-timeout test: a wait that nothing completes runs out, and the
      // CTA takes the same path as after any wait that gives up
      if (a.stall && !mbar_wait(stall_bar, 0, wait_ns)) *failed = 1;
      for (int tile = blockIdx.x; tile < ntiles && !*failed; tile += gridDim.x, ++j) {
        const int b = j & 1;
        // the epilogue has read this buffer's previous tile (fresh barriers pass parity 1)
        if (!mbar_wait(&acc_empty[b], ((j >> 1) & 1) ^ 1, wait_ns)) {
          *failed = 1;
          break;
        }
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + b * BT;
        for (int kb = 0; kb < num_kb; ++kb, ++g) {
          const int s = g % STAGES, as = g % ASTAGES;
          // the A stage is written, which also means the x stage has landed
          if (!mbar_wait(&ready[as], (g / ASTAGES) & 1, wait_ns)) {
            *failed = 1;
            break;
          }
          tc_fence_after();
          const uint32_t x_addr = smem_u32(smem + kOffX + s * kXBytes);
          // eight MMAs per stage, four when its second half lies beyond K
          const int nmma = kb * BK + 128 < a.K ? 8 : 4;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
            if (jj < nmma)
              umma_i8_ts(tmem_d, tmem_a + as * kACols + 8 * jj,
                         umma_desc_sw128(x_addr + (jj >> 2) * kXHalf + 32 * (jj & 3)), idesc, (kb | jj) != 0);
          umma_commit(&empty[s]);                 // the shared stage can be refilled
          umma_commit(&afree[as]);                // the A stage can be rewritten
        }
        if (*failed) break;
        umma_commit(&acc_full[b]);                // the tile's accumulator is complete
      }
      // every MMA issued above has completed before tensor memory is freed
      // (fixed limit, as for the copies)
      umma_commit(drain);
      if (!mbar_wait(drain, 0, kWaitLimitNs)) {
        *failed = 1;
        *drain_bad = 1;
      }
    }
   }
  } else if (warp < 12) {
    setmaxnreg_dec<kRegsUnpack>();
    // ---------------- weight unpack into tensor memory ----------------
    // Two warps per tensor-memory lane quarter, one per 128-k half of a
    // stage (a single warp's chain of loads, unpacking, store and arrive
    // took longer than the stage's MMAs).
    const int q = warp & 3;
    const int hh = (warp - 4) >> 2;               // the half of each stage this warp unpacks
    const int row = 32 * q + lane;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    // The weight rows are 64 bytes with TMA's 64-byte swizzle: 16-byte piece
    // p of row r sits at piece p ^ ((r >> 1) & 3), so the eight rows of a
    // quarter-warp read piece p from eight different 4-bank groups.
    const int sw = (row >> 1) & 3;
    int g = 0;
    for (int tile = blockIdx.x; tile < ntiles && !*failed; tile += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb, ++g) {
        const int s = g % STAGES, as = g % ASTAGES;
        bool ok = mbar_wait(&full[s], (g / STAGES) & 1, wait_ns);
        if (ok && g >= ASTAGES) ok = mbar_wait(&afree[as], ((g / ASTAGES) - 1) & 1, wait_ns);
        if (!ok) {
          *failed = 1;
          break;
        }
        // a second half beyond K gets no MMA: nothing to write, but its
        // warp still arrives
        if (hh == 0 || kb * BK + 128 < a.K) {
          const uint4* wp = reinterpret_cast<const uint4*>(smem + kOffWp + s * kWpBytes + row * 64);
          const uint4 p0 = wp[(2 * hh) ^ sw], p1 = wp[(2 * hh + 1) ^ sw];
          tc_fence_after();
          const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
          uint32_t codes[32];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {        // word jj = k 16jj .. 16jj + 15 of the half
            codes[4 * jj + 0] = w[jj] & kCodeMask;
            codes[4 * jj + 1] = (w[jj] >> 2) & kCodeMask;
            codes[4 * jj + 2] = (w[jj] >> 4) & kCodeMask;
            codes[4 * jj + 3] = (w[jj] >> 6) & kCodeMask;
          }
          tmem_st_32x32b_x32(tmem_a + lane_base + as * kACols + 32 * hh, codes);
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ready[as]);
      }
    }
  } else {
    setmaxnreg_inc<kRegsEpi>();
    // ---------------- epilogue ----------------
    const int q = warp & 3;
    const int et = threadIdx.x - 384;             // 0..255
    const int half = (warp - 12) >> 2;            // which half of the tile's tokens
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    pdl_wait_primary();
    float swg[kMaxGroups];                         // s_w of each row group
#pragma unroll
    for (int g = 0; g < kMaxGroups; ++g) swg[g] = g < a.ngroups ? a.w_scale[g] : 0.0f;
    int j = 0;
    // acc = sum(c q) - sum(q) is exact in float32 and double below 2^24,
    // |acc| <= 127 K: such a K takes the conversion-free path
    const bool small_k = a.K <= (1 << 17);
    // The eight epilogue warps meet at named barriers (1 twice, 2 once per
    // tile); every one of them runs every iteration (a failure only skips
    // work), so the barriers always get their 256 threads.
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++j) {
      const int b = j & 1;
      const int n0 = (tile % wtiles) * BW, m0 = (tile / wtiles) * BT;
      // The tile's rows share one layer's scale unless a group boundary of
      // stacked layers falls inside it (rare: only grouped calls).
      const int nlast = min(n0 + BW, a.N) - 1;
      int g0 = 0, g1 = 0;
#pragma unroll
      for (int g = 0; g + 1 < kMaxGroups; ++g) {
        g0 += (g + 1 < a.ngroups && n0 >= a.group_end[g]) ? 1 : 0;
        g1 += (g + 1 < a.ngroups && nlast >= a.group_end[g]) ? 1 : 0;
      }
      const bool uniform = g0 == g1;
      float sw_tile = swg[0];
#pragma unroll
      for (int g = 1; g < kMaxGroups; ++g)
        if (g == g0) sw_tile = swg[g];
      // the previous tile's TMA store has read the staging buffer
      if (a.y_tma && et == 0) bulk_wait_read_all();
      // per-token s_x and row sums of this tile
      asm volatile("bar.sync 1, 256;" ::: "memory");   // previous tile's readers are done
      if (et < BT) {
        const int m = m0 + et;
        const float sx = m < a.M ? a.s_x[m] : 1.0f;
        if (uniform) {
          // d = s_x s_w (float32), or on a bf16 module bf16(bf16(s_w) s_x),
          // kept as the double 1 / d: RN_f32(a * (1/d)) with a the float32
          // (or bf16) numerator is RN_f32(a / d) -- a quotient of two floats
          // lies at least 2^-49 (relative) from every float32 midpoint, and
          // the double product is within 2^-52 of it.
          const float d = a.faithful ? bf16_round(__fmul_rn(bf16_round(sw_tile), sx)) : __fmul_rn(sx, sw_tile);
          rcp_s[et] = __drcp_rn(static_cast<double>(d));
        } else {
          sx_s[et] = sx;
        }
        rs_s[et] = m < a.M ? a.rowsum[m] : 0;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      bool ok = !__any_sync(0xffffffffu, *failed != 0);
      if (ok) ok = mbar_wait(&acc_full[b], (j >> 1) & 1, wait_ns);
      ok = __all_sync(0xffffffffu, ok);             // warp-uniform decision
      if (!ok) *failed = 1;
      const int row = 32 * q + lane;                // row of the tile
      const int n = n0 + row;
      const bool nv = n < a.N;
      if (ok) {
        tc_fence_after();
        const float bv = (a.bias && nv) ? bf16_bits_to_f32(a.bias[n]) : 0.0f;
        float s_w = swg[0];                        // this row's group scale (tiles with several)
#pragma unroll
        for (int g = 1; g < kMaxGroups; ++g)
          if (g < a.ngroups && n >= a.group_end[g - 1]) s_w = swg[g];
        if (a.faithful) s_w = bf16_round(s_w);     // a bf16 module holds s_w in bf16
        auto emit = [&](int mi, int accv, float y32) {
          if (a.y_tma) {
            stage[mi * BW + row] = f32_to_bf16_bits_alu(y32);   // tokens >= M are clipped by the store
            return;
          }
          if (m0 + mi >= a.M) return;
          const size_t o = static_cast<size_t>(m0 + mi) * a.N + n;
          if (a.y) a.y[o] = f32_to_bf16_bits(y32);
          if (a.acc_out) a.acc_out[o] = accv;
          if (a.y32_out) a.y32_out[o] = y32;
        };
        auto process = [&](const uint32_t (&r)[32], int c) {
          if (!nv) return;
          if (uniform && !a.faithful && small_k) {
            // per-token values as 16-byte vectors, 4 tokens at a time; the
            // int32 -> double conversion by the 1.5 * 2^52 + 2^31 bias
            // (exact for every int32), one rounding double -> float
#pragma unroll
            for (int i4 = 0; i4 < 32; i4 += 4) {
              const int mb = 32 * c + i4;
              const int4 rs = *reinterpret_cast<const int4*>(rs_s + mb);
              const double2 rc01 = *reinterpret_cast<const double2*>(rcp_s + mb);
              const double2 rc23 = *reinterpret_cast<const double2*>(rcp_s + mb + 2);
              const int rsv[4] = {rs.x, rs.y, rs.z, rs.w};
              const double rcv[4] = {rc01.x, rc01.y, rc23.x, rc23.y};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int accv = static_cast<int>(r[i4 + i]) - rsv[i];
                const double num = __hiloint2double(0x43380000, accv ^ static_cast<int>(0x80000000u)) -
                                   6755401588539392.0;
                float y32 = __double2float_rn(num * rcv[i]);
                if (a.bias) y32 = __fadd_rn(y32, bv);
                emit(mb + i, accv, y32);
              }
            }
          } else if (uniform && !a.faithful) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int mi = 32 * c + i;
              const int accv = static_cast<int>(r[i]) - rs_s[mi];
              float y32 = __double2float_rn(static_cast<double>(static_cast<float>(accv)) * rcp_s[mi]);
              if (a.bias) y32 = __fadd_rn(y32, bv);
              emit(mi, accv, y32);
            }
          } else if (uniform) {
            // bf16 module: the sum, the quotient and the bias add are each
            // rounded to bf16 (the scale product is in rcp_s)
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int mi = 32 * c + i;
              const int accv = static_cast<int>(r[i]) - rs_s[mi];
              float y32 = bf16_round(__double2float_rn(static_cast<double>(bf16_round(static_cast<float>(accv))) * rcp_s[mi]));
              if (a.bias) y32 = bf16_round(__fadd_rn(y32, bv));
              emit(mi, accv, y32);
            }
          } else if (!a.faithful) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int mi = 32 * c + i;
              const int accv = static_cast<int>(r[i]) - rs_s[mi];
              float y32 = __fdiv_rn(static_cast<float>(accv), __fmul_rn(sx_s[mi], s_w));
              if (a.bias) y32 = __fadd_rn(y32, bv);
              emit(mi, accv, y32);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int mi = 32 * c + i;
              const int accv = static_cast<int>(r[i]) - rs_s[mi];
              float y32 = bf16_round(__fdiv_rn(bf16_round(static_cast<float>(accv)), bf16_round(__fmul_rn(s_w, sx_s[mi]))));
              if (a.bias) y32 = bf16_round(__fadd_rn(y32, bv));
              emit(mi, accv, y32);
            }
          }
        };
        // the next 32 columns load while the current ones are processed; once
        // the last load has landed the whole accumulator half is in registers
        // and the buffer goes back to the MMA warp
        const uint32_t col0 = tmem_base + b * BT + lane_base + 32 * (half * kEpiChunks);
        uint32_t r0[32], r1[32];
        tmem_ld_32x32b_x32(col0, r0);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kEpiChunks; ++c) {
          const bool last = c + 1 == kEpiChunks;
          if (!last) tmem_ld_32x32b_x32(col0 + 32 * (c + 1), (c & 1) ? r0 : r1);
          if (last) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
          }
          process((c & 1) ? r1 : r0, half * kEpiChunks + c);
          if (!last) tmem_wait_ld();
        }
      }
      if (a.y_tma) {
        // every epilogue thread's staging writes are visible to the async
        // proxy; then one thread stores the tile (rows >= N and tokens >= M
        // are clipped by the tensor map's bounds)
        fence_proxy_async_smem();
        asm volatile("bar.sync 2, 256;" ::: "memory");
        if (et == 0 && !*failed) {
          tma_store_2d(&tm_y, stage, n0, m0);
          bulk_commit();
        }
      }
    }
    // the last stores have completed (their shared memory stays in use until then)
    if (a.y_tma && et == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *failed) report_status(a.status, kStatusTimeout);
  // Tensor memory is freed only when every MMA is known to have completed;
  // after a drain that gave up (never seen: it needs MMAs or copies stuck
  // for a whole second) the CTA exits without freeing it rather than free
  // it under a running MMA.
  if (warp == 2 && !*drain_bad) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_prefill(const ForwardArgs& args, int num_sms, cudaStream_t stream) {
  if (args.M <= 0) return cudaSuccess;
  ForwardArgs a = args;
  static unsigned long long attr_done = 0;        // one bit per device
  cudaError_t ea = set_smem_attr_once(gemm_prefill_kernel, static_cast<int>(kSmemBytes), &attr_done);
  if (ea != cudaSuccess) return ea;
  CUtensorMap tm_x, tm_w;
  if (!encode_2d_u8(&tm_x, a.xq, a.K, a.M, a.K, 128, BT, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  if (!encode_2d_u8(&tm_w, a.packed, a.K / 4, a.N, a.K / 4, BK / 4, BW, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  // y by TMA tile stores when its rows are 16-byte multiples at a 16-byte
  // aligned base and no debug output is asked for; else plain stores
  CUtensorMap tm_y;
  memset(&tm_y, 0, sizeof(tm_y));
  a.y_tma = a.y != nullptr && a.acc_out == nullptr && a.y32_out == nullptr && (a.N % 8) == 0 &&
            (reinterpret_cast<uintptr_t>(a.y) & 15) == 0 &&
            encode_2d_u16(&tm_y, a.y, a.N, a.M, static_cast<uint64_t>(a.N) * 2, BW, BT);
  const long tiles = static_cast<long>((a.N + BW - 1) / BW) * ((a.M + BT - 1) / BT);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles < num_sms ? tiles : num_sms), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_prefill_kernel, tm_x, tm_w, tm_y, a);
}

}  // namespace bitlinear
