// Decode engine (M <= 16 tokens): the whole BitLinear forward of the
// Falcon-Edge blog (section "Falcon-Edge, a series of universal models":
// activation_norm_quant, F.linear on the unpacked ternary weights,
// post_quant_process and the bias add) in one kernel that streams the 2-bit
// packed weights once.
//
// Work split.  The N weight rows form 16-row units; the grid is one wave of
// CTAs (one per SM; two per SM for the 8-token kernel on matrices of 8 or
// more units per SM) and CTA c owns a contiguous, balanced range of units
// over the whole of K.  CTAs never talk to each other.  K is cut into 512-k
// chunks (the last one maybe partial), and the chunks into rounds of eight
// (4096 k: the x of one round sits in shared memory as int8).
//
// Inside a CTA every one of the 8 warps streams and computes:
//   * An item is one chunk of two consecutive units in the 8-token kernel
//     (32 rows x 128 bytes: one wait, one cursor step and one x fragment
//     per 4 KB, and eight independent MMA chains) and of one unit in the
//     16-token kernel.  A round's items are numbered chunk-major, and warp w
//     takes the contiguous w-th eighth of them, so a warp's consecutive
//     items share a chunk (its x fragment is loaded once per chunk) and the
//     shares differ by at most one item.
//   * Each warp streams its own items through its own ring of shared-memory
//     slots: every lane copies 4 x 16 bytes of an item with cp.async, at
//     per-lane offsets fixed for the whole kernel (128-byte rows, written in
//     the 128-byte-swizzled order that keeps the fragment reads below
//     conflict-free), one copy group per item, up to `ring` items ahead;
//     pieces beyond N or K, and the missing unit of a CTA's last pair, are
//     zero-filled.  The warp waits for the oldest
//     group (once for all of them when its whole share fitted in the ring)
//     and refills its slot once it has read it.  No warp ever waits for
//     another warp's copies.  When the weights are resident the first
//     copies, the bias and the scales, the x-phase plan and an L2 prefetch
//     of x are issued before the wait on the previous kernel of the stream,
//     so they overlap its tail; after the wait only x-dependent work is left.
//   * bf16 x (M <= 8): all warps form each token's absmax over the row,
//     s_x = 127 / max(absmax, 1e-5) in float32, and q = round_half_even(x
//     s_x) as int8 into shared memory, one round at a time, with the sum of q
//     per token.  For K <= 4096 each lane's share of x (at most 8 x 32
//     bytes per token) is read once and held in registers between the two
//     steps; otherwise x is read again for the quantising step.  With one
//     token and a full round, warp w quantises exactly the chunk its own
//     items use, so no block barrier separates the quantising from the
//     items.  A lane's x fragment loads use offsets worked out once (lanes
//     of tokens that do not exist read 512 zero bytes).
//   * int8 x (above 8 tokens the act-quant kernel quantises x once; also the
//     pre-quantised and K-split calls): the scales and row sums are read, and
//     each warp loads its x fragments straight from global memory.
//   * Per item a thread takes one 16-byte vector of two weight rows per
//     256-k half and issues mma.sync m16n8k32 (weights as A, u8; tokens as B,
//     s8; a second 8-token tile for M > 8).  The codes c = u + 1 enter
//     unshifted: A_i = word & (0x03030303 << 2i) holds 4^i c per byte lane,
//     so field i accumulates 4^i sum(c q); the fields of one unit are
//     combined with exact shifts before the next unit's MMAs (one unit's
//     field accumulators live at a time) and added to the unit's int32 sums
//     in shared memory.
//   * Epilogue: acc = sum(c q) - sum(q) = sum(u q); y = acc / (s_x s_w)
//     (+ bias) -> bf16, with s_w the scale of the row's layer when several
//     layers are stacked, the division done as a product with the double
//     1 / (s_x s_w) of the token and layer (exactly the float32 quotient),
//     each output computing its own reciprocal.  The bf16-faithful mode (a
//     template parameter, so neither mode carries the other's branches)
//     rounds the scale, the products, the sum and the quotient to bf16 as a
//     bf16 module does.
// Rows beyond N and k beyond K are zero-filled (code 0), so they add
// nothing whatever the x bytes there are.
//
// Fragment layout.  MMA row g of a unit is box row pi(g) = (g >> 1) |
// ((g & 1) << 2) (and pi(g) + 8), so the two rows a quarter-warp reads
// differ in bit 2 and the 128-byte swizzle puts their chunks in disjoint bank
// groups.  Inside a sub-box, thread (g, t) covers k = 64t .. 64t + 63 of each
// 256-k half v: register a0 of field i / pair p holds k = 64t + 32p + 4i +
// {0..3}, a2 the same + 16; the B registers are the x words at byte offsets
// 64t + 32p + 4i and 64t + 32p + 16 + 4i.
#include "kernels.h"

namespace bitlinear {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kUnitRows = 16;
constexpr int kBoxK = 512;                            // k per chunk (sub-box)
constexpr int kSubBytes = kUnitRows * kBoxK / 4;      // 2 KB
constexpr int kRoundChunks = 8;                       // chunks per x round
constexpr int kChunkK = kRoundChunks * kBoxK;         // k per round
constexpr int kMaxUnits = 32;                         // units per CTA
constexpr int kXB = 8;                                // bf16 x loads in flight per lane (absmax)
constexpr int kQB = 2;                                // the same in the quantising pass
constexpr int kHold = 8;                              // 32-byte x chunks per lane and token held in
                                                      // registers by the one-pass path
constexpr uint32_t kCodeMask = 0x03030303u;
// units per item: two for the 8-token kernel (one wait, one cursor step and
// one x fragment per 4 KB, eight independent MMA chains); one for the
// 16-token kernel, whose accumulators and x fragments fill its registers
__host__ __device__ constexpr int units_per_item(int nt) { return nt == 1 ? 2 : 1; }
constexpr float kRoundMagic = 12582912.0f;            // 1.5 * 2^23

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// the same with a zero accumulator in (the first MMA of a chain): no
// register has to be cleared for it
__device__ __forceinline__ void mma_u8s8_first(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// floor(a / 2^(32 - sh)) + c on the multiply-add pipe (mad.hi: the high word
// of the 64-bit product a 2^sh, plus c); the field sums are multiples of the
// divisor, so this is their exact shift
__device__ __forceinline__ int mad_hi(int a, int b, int c) {
  int d;
  asm("mad.hi.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// 16-byte asynchronous copy global -> shared (L2 only); src_bytes = 0 writes
// zeros and reads nothing
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// waits until at most n of this thread's copy groups are still in flight
__device__ __forceinline__ void cp_async_wait(int n) {
  switch (n) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
    case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
    case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
    case 6: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 7;" ::: "memory"); break;
  }
}

__device__ __forceinline__ void red_shared_add(int* p, int v) {
  asm volatile("red.shared.add.s32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

// 16-byte chunk position in a token row of the x chunk: within every 16
// chunks, chunks 8..15 swap pairs (p ^ 2), so the four quad lanes t of a
// fragment load hit four different bank groups.
__device__ __forceinline__ int xs_chunk(int ch) { return ch ^ (((ch >> 3) & 1) << 1); }

__device__ __forceinline__ int mma_row_to_box(int g) { return (g >> 1) | ((g & 1) << 2); }

// Place of (row, token) in a unit's int32 sums [16 rows][ntok tokens]: the
// token index is rotated by a function of the row so that the 32 lanes of
// one red.shared (rows pi(g) or pi(g) + 8, tokens 2t or 2t + 1) hit 32
// different banks; a plain [row][token] layout put two (8 tokens) or four
// (16 tokens) rows in one bank group.
template <int NTOK>
__device__ __forceinline__ int sum_idx(int row, int m) {
  const int f = NTOK == 8 ? ((row >> 2) & 1) : (((row >> 1) & 1) + 8 * ((row >> 2) & 1));
  return row * NTOK + ((m + f) & (NTOK - 1));
}

// largest |x| of 16 bf16 values, as bf16 bits (finite values order like bits & 0x7FFF)
__device__ __forceinline__ uint32_t absmax16_bits(uint4 lo, uint4 hi) {
  uint32_t m = 0;
  m = __vmaxu2(m, lo.x & 0x7FFF7FFFu); m = __vmaxu2(m, lo.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, lo.z & 0x7FFF7FFFu); m = __vmaxu2(m, lo.w & 0x7FFF7FFFu);
  m = __vmaxu2(m, hi.x & 0x7FFF7FFFu); m = __vmaxu2(m, hi.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, hi.z & 0x7FFF7FFFu); m = __vmaxu2(m, hi.w & 0x7FFF7FFFu);
  return max(m & 0xFFFFu, m >> 16);
}

// Four bf16 values (two words) -> four int8 q = round_half_even(x * s), packed.
// p = x * s is rounded to float32 first; adding 1.5 * 2^23 then rounds p to an
// integer with ties to even (the sum lies in [2^23, 2^24), where the float
// spacing is 1, and the magic constant is even), and the low byte of the sum's
// bits is q as a two's-complement byte.  In float32 |p| <= 127 for finite x
// because s was formed from the row's absmax, so the [-128, 127] clamp never
// acts; the bf16-faithful path clamps explicitly.
__device__ __forceinline__ uint32_t quant4(uint32_t w01, uint32_t w23, float s, bool faithful) {
  float p[4] = {__fmul_rn(__uint_as_float(w01 << 16), s), __fmul_rn(__uint_as_float(w01 & 0xFFFF0000u), s),
                __fmul_rn(__uint_as_float(w23 << 16), s), __fmul_rn(__uint_as_float(w23 & 0xFFFF0000u), s)};
  if (faithful) {
    // the bf16 tensor x * scale; here the scale can exceed 127 / absmax by a
    // few bf16 ulps, so the product can round to 128 and the clamp acts
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = fminf(fmaxf(bf16_round(p[e]), -128.0f), 127.0f);
  }
  const uint32_t b0 = __float_as_uint(__fadd_rn(p[0], kRoundMagic));
  const uint32_t b1 = __float_as_uint(__fadd_rn(p[1], kRoundMagic));
  const uint32_t b2 = __float_as_uint(__fadd_rn(p[2], kRoundMagic));
  const uint32_t b3 = __float_as_uint(__fadd_rn(p[3], kRoundMagic));
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

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

// s_x from the row's absmax a: 127 / max(a, 1e-5) in float32, or, on a bf16
// module, PyTorch's evaluation of 127.0 / t: bf16(bf16(1 / t) * 127)
__device__ __forceinline__ float act_scale(float a, bool faithful) {
  return faithful ? bf16_round(__fmul_rn(bf16_round(__fdiv_rn(1.0f, fmaxf(a, bf16_round(1e-5f)))), 127.0f))
                  : __fdiv_rn(127.0f, fmaxf(a, 1e-5f));
}

__device__ __forceinline__ int bytesum16(uint4 v, int sum) {
  sum = __dp4a(static_cast<int>(v.x), 0x01010101, sum);
  sum = __dp4a(static_cast<int>(v.y), 0x01010101, sum);
  sum = __dp4a(static_cast<int>(v.z), 0x01010101, sum);
  return __dp4a(static_cast<int>(v.w), 0x01010101, sum);
}

struct SmemTail {
  uint4 zero[32];                    // 512 zero bytes: the x fragment of a token that does not exist
  uint64_t stall;                    // never signalled (forced-timeout test hook)
  uint32_t amax[16];                 // absmax per token (bf16 bits)
  int rsum[16];                      // sum of q per token
  float sx[16];                      // s_x per token
  double rcp[kMaxGroups * 16];       // 1 / (s_x s_w) per row group and token, [group][token]
  int failed;                        // a wait of this CTA timed out
};

struct SmemLayout {
  size_t ring, xs, acc, bias, tail, total;
};

// 8 warps' rings of `ring` slots of slot_bytes (1024-aligned base), x rows of
// one round for the M tokens, per-unit int32 sums [unit][row][8 * token
// tiles], bias, tail
// M tokens, of which xrows have their x staged in shared memory (M for bf16
// x, 0 for int8 x read straight from global memory)
__host__ __device__ SmemLayout smem_layout(int M, int xrows, int ring, size_t slot_bytes, int units) {
  const int ntok = M <= 8 ? 8 : 16;
  SmemLayout L;
  L.ring = 0;
  L.xs = L.ring + static_cast<size_t>(kWarps) * ring * slot_bytes;
  L.acc = L.xs + static_cast<size_t>(xrows) * (kChunkK + 16);
  L.bias = L.acc + static_cast<size_t>(units) * kUnitRows * ntok * 4;
  L.tail = (L.bias + static_cast<size_t>(units) * kUnitRows * 2 + 15) & ~size_t(15);
  L.total = 1024 + L.tail + sizeof(SmemTail);
  return L;
}

// The items of one warp, in order.  An item is one chunk of UP consecutive
// units (UP = 2 for the 8-token kernel, 1 for the 16-token one); a CTA's U
// units form PU = ceil(U / UP) unit groups, the last one maybe short.  A
// round's T = chunks x PU items are numbered chunk major (item j: chunk j /
// PU, group j % PU), and warp w takes the contiguous range [w T / 8, (w + 1)
// T / 8) of them.  The shares differ by at most one item, and the
// consecutive items of a warp mostly share a chunk, so its x fragment is
// loaded once per chunk.  The cursor moves by increments; only a new round
// costs divisions.
struct ItemCursor {
  int r, g, p, left;                               // round, item (chunk g, group p), items left in the round
  __device__ __forceinline__ static int chunks(int r, int nchunks) {
    return min(nchunks - kRoundChunks * r, kRoundChunks);
  }
  __device__ __forceinline__ void begin_round(int warp, int nchunks, int PU) {
    const int T = chunks(r, nchunks) * PU;
    const int jb = warp * T / kWarps;
    left = (warp + 1) * T / kWarps - jb;
    g = jb / PU;
    p = jb - g * PU;
  }
  // moves past empty rounds; true when the round changed
  __device__ __forceinline__ bool settle(int warp, int nround, int nchunks, int PU) {
    bool moved = false;
    while (r < nround && left == 0) {
      ++r;
      moved = true;
      if (r < nround) begin_round(warp, nchunks, PU);
    }
    return moved;
  }
  __device__ __forceinline__ void start(int warp, int nround, int nchunks, int PU) {
    r = 0;
    begin_round(warp, nchunks, PU);
    settle(warp, nround, nchunks, PU);
  }
  // next item; true when it is not the group after the current one in the
  // same chunk (a new chunk or a new round)
  __device__ __forceinline__ bool next(int warp, int nround, int nchunks, int PU) {
    --left;
    bool jump = false;
    if (++p == PU) {
      p = 0;
      ++g;
      jump = true;
    }
    return settle(warp, nround, nchunks, PU) || jump;
  }
};

template <int NT, bool FAITHFUL>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 2 : 1)
    decode_kernel(const DecodeArgs a) {
  constexpr int NTOK = NT * 8;
  constexpr int UP = units_per_item(NT);             // units per item
  constexpr int kSlotBytes = UP * kSubBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int ring = a.ring;
  // int8 x with its row sums is read straight from global memory (no x in
  // shared memory); bf16 x is quantised into shared memory
  const bool direct = a.xq != nullptr && a.rowsum != nullptr;
  const SmemLayout L = smem_layout(a.M, direct ? 0 : a.M, ring, kSlotBytes, a.units_max);
  int8_t* xs = reinterpret_cast<int8_t*>(base + L.xs);
  int* acc_s = reinterpret_cast<int*>(base + L.acc);            // [unit][row][token]
  uint16_t* bias_s = reinterpret_cast<uint16_t*>(base + L.bias);
  SmemTail& sm = *reinterpret_cast<SmemTail*>(base + L.tail);
  constexpr int S = kChunkK + 16;                    // bytes per token row of the x round

  pdl_launch_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.K, N = a.N, M = a.M;
  const int units_total = (N + kUnitRows - 1) / kUnitRows;
  const int u_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * units_total / gridDim.x);
  const int U = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * units_total / gridDim.x) - u_begin;
  const int PU = (U + UP - 1) / UP;                 // unit groups of this CTA
  const int nchunks = (K + kBoxK - 1) / kBoxK;       // 512-k chunks, the last maybe partial
  const int nround = (K + kChunkK - 1) / kChunkK;
  const uint32_t row_bytes = static_cast<uint32_t>(K) / 4;
  uint8_t* wring = base + L.ring + static_cast<size_t>(warp) * ring * kSlotBytes;   // this warp's ring

  if (threadIdx.x == 0) {
    mbar_init(&sm.stall, 1);
    sm.failed = 0;
  }
  fence_mbar_init();
  if (threadIdx.x < 16) {
    sm.amax[threadIdx.x] = 0u;
    sm.rsum[threadIdx.x] = 0;
  }
  if (threadIdx.x < 32) sm.zero[threadIdx.x] = make_uint4(0, 0, 0, 0);
  for (int i = threadIdx.x; i < U * kUnitRows * NTOK; i += kThreads) acc_s[i] = 0;
  __syncthreads();

  // ---- this warp's weight stream: every lane copies its own 16-byte
  // pieces of an item (row p >> 3, piece p & 7 of each 128-byte chunk row,
  // p = lane, lane + 32, ..., per unit of the item) into the slot's
  // 128-byte-swizzled layout; one copy group per item; pieces beyond N or K
  // and units beyond the CTA's range are zero-filled
  ItemCursor ic;                                     // next item to issue
  ic.start(warp, nround, nchunks, PU);
  const ItemCursor cstart = ic;                      // the first item, for the consumer
  int islot = 0;                                     // ring slot of the next copy
  // this lane's pieces of a unit: rows (lane >> 3) + 4 j, piece lane & 7 of
  // each row, j = 0..3; their source and destination offsets are fixed, only
  // the item's first row and chunk change
  const int prow = lane >> 3, pq = lane & 7;
  const uint32_t psrc = static_cast<uint32_t>(prow) * row_bytes + 16u * pq;   // + (16 e + 4 j) row_bytes
  const uint32_t pdst0 = prow * 128 + ((pq ^ prow) << 4);          // rows prow, prow + 8
  const uint32_t pdst1 = (prow + 4) * 128 + ((pq ^ (prow + 4)) << 4);   // rows prow + 4, prow + 12
  // rows of this CTA's units that exist (the last unit of the matrix may be short)
  const int lim0 = min(U * kUnitRows, N - u_begin * kUnitRows);
  auto issue_next = [&]() {
    if (ic.r < nround) {
      const int c = kRoundChunks * ic.r + ic.g;     // chunk of the item
      const int r0g = UP * kUnitRows * ic.p;         // first row of the item in the CTA's range
      const int lim = lim0 - r0g;                    // rows of the item's units that exist
      uint8_t* dst = wring + islot * kSlotBytes;
      const bool kin = static_cast<uint32_t>(c) * (kBoxK / 4) + 16u * pq < row_bytes;
      const uint8_t* src = a.packed + static_cast<size_t>(u_begin * kUnitRows + r0g) * row_bytes +
                           static_cast<uint32_t>(c) * (kBoxK / 4) + psrc;
      // an item wholly inside N and K (every item but a CTA's last group and
      // the chunk at K's end; the same for the whole warp) needs no checks
      if (lim >= UP * kUnitRows && static_cast<uint32_t>(c + 1) * (kBoxK / 4) <= row_bytes) {
#pragma unroll
        for (int e = 0; e < UP; ++e)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            cp_async16(dst + e * kSubBytes + ((j & 1) ? pdst1 : pdst0) + (j >> 1) * 1024,
                       src + static_cast<size_t>(kUnitRows * e + 4 * j) * row_bytes, 16u);
      } else {
#pragma unroll
        for (int e = 0; e < UP; ++e)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const bool valid = kin && kUnitRows * e + prow + 4 * j < lim;
            cp_async16(dst + e * kSubBytes + ((j & 1) ? pdst1 : pdst0) + (j >> 1) * 1024,
                       valid ? src + static_cast<size_t>(kUnitRows * e + 4 * j) * row_bytes : a.packed, valid ? 16u : 0u);
          }
      }
      islot = islot + 1 == ring ? 0 : islot + 1;
      ic.next(warp, nround, nchunks, PU);
    }
    cp_async_commit();                               // one group per call, empty when nothing is left
  };
  // the bias and the scales are read into registers as early as they may be
  // (with the weights when those are resident) and stored to shared memory
  // only before the epilogue, so no thread waits for them on the way to x
  uint16_t bvals[2] = {0, 0};
  // thread g M + m (< M x groups) forms 1 / (s_x s_w) of token m and row group g
  float swv = 0.0f;
  auto load_params = [&]() {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = threadIdx.x + k * kThreads;
      const int n = u_begin * kUnitRows + i;
      if (i < U * kUnitRows && a.bias && n < N) bvals[k] = a.bias[n];
    }
    if (threadIdx.x < M * a.ngroups) swv = a.w_scale[threadIdx.x / M];
  };
  if (a.weights_early) {
    for (int i = 0; i < ring; ++i) issue_next();
    load_params();
  }

  // ---- the x-phase plan, worked out while the previous kernel finishes:
  // warp w takes token(s) m = w / P (+ 8 / P, ...) and a 1/P share of the
  // row, P = max(1, 8 / M); in the one-pass path load i of a lane reads the
  // 16-element chunk part * 32 + lane + i * 32 P of its token
  const int cpr = K >> 4;                            // 16-element chunks per row
  const int P = M >= kWarps ? 1 : kWarps / M;
  const int part = warp % P, mstep = kWarps / P;
  const int C = (cpr + 32 * P - 1) / (32 * P);       // chunks per lane per token
  // One pass over x when the row is one round and this lane's share fits in
  // registers: the values loaded for the absmax are quantised in place.
  const bool single = a.x && nround == 1 && C <= kHold;
  const int ch_first = part * 32 + lane;             // first chunk of this lane
  const int xstep = 64 * P;                          // uint4 between a lane's loads
  const uint4* xl[NT];                               // this lane's first load, per token slot
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int m = min(warp / P + j * mstep, M - 1);
    xl[j] = reinterpret_cast<const uint4*>(a.x) + ((static_cast<size_t>(m) * K) >> 3) + 2 * ch_first;
  }

  // x into L2 while the previous kernel finishes: each CTA takes every
  // gridDim-th 128-byte line, so the lines are asked for once
  {
    const uint8_t* xb = a.x ? reinterpret_cast<const uint8_t*>(a.x) : reinterpret_cast<const uint8_t*>(a.xq);
    const size_t xbytes = static_cast<size_t>(M) * K * (a.x ? 2 : 1);
    for (size_t l = blockIdx.x + static_cast<size_t>(gridDim.x) * threadIdx.x; xb != nullptr && l * 128 < xbytes;
         l += static_cast<size_t>(gridDim.x) * kThreads)
      prefetch_l2(xb + l * 128);
  }
  pdl_wait_primary();
  if (!a.weights_early) {
    for (int i = 0; i < ring; ++i) issue_next();
    load_params();
  }
  if (a.status && blockIdx.x == 0 && threadIdx.x == 0) *a.status = 0u;

  bool ok = true;
  const int g = lane >> 2, t = lane & 3;

  // ---- per-token absmax over the whole row
  if (direct) {
    // int8 x from the act-quant kernel: the scales and row sums are read
    // here, the fragments straight from global memory in the item loop
    if (threadIdx.x < M) {
      sm.sx[threadIdx.x] = a.s_x[threadIdx.x];
      sm.rsum[threadIdx.x] = a.rowsum[threadIdx.x];
    }
  } else if (NT == 1 && single) {
    // warp w takes token m = w / P; a lane holds C <= kHold chunks of it
    const int m = warp / P;
    const bool mine = m < M;
    // (the loops leave at i = C, the same for every thread, so the unrolled
    // iterations beyond it cost one branch rather than being predicated off)
    uint4 v[kHold][2];
#pragma unroll
    for (int i = 0; i < kHold; ++i) {
      if (i >= C) break;
      const bool in = mine && ch_first + i * 32 * P < cpr;
      v[i][0] = in ? __ldg(xl[0] + i * xstep) : make_uint4(0, 0, 0, 0);
      v[i][1] = in ? __ldg(xl[0] + i * xstep + 1) : make_uint4(0, 0, 0, 0);
    }
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < kHold; ++i) {
      if (i >= C) break;
      mx = max(mx, absmax16_bits(v[i][0], v[i][1]));   // zeros where nothing was loaded
    }
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0 && mine) atomicMax(&sm.amax[m], mx);
    __syncthreads();
    const float sxm = act_scale(bf16_bits_to_f32(sm.amax[min(m, M - 1)]), FAITHFUL);
    if (threadIdx.x < M) {
      // warp 0 holds token 0's scale already
      const float sxv = threadIdx.x == 0 ? sxm : act_scale(bf16_bits_to_f32(sm.amax[threadIdx.x]), FAITHFUL);
      sm.sx[threadIdx.x] = sxv;
      if (blockIdx.x == 0 && a.sx_out) a.sx_out[threadIdx.x] = sxv;
    }
    int sum = 0;
#pragma unroll
    for (int i = 0; i < kHold; ++i) {
      const int ch = ch_first + i * 32 * P;
      if (i >= C) break;
      if (mine && ch < cpr) {
        const uint4 qv = quant16(v[i][0], v[i][1], sxm, sum, FAITHFUL);
        *reinterpret_cast<uint4*>(xs + m * S + 16 * xs_chunk(ch)) = qv;
        if (blockIdx.x == 0 && a.xq_out) *reinterpret_cast<uint4*>(a.xq_out + static_cast<size_t>(m) * K + 16 * ch) = qv;
      }
    }
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0 && mine) atomicAdd(&sm.rsum[m], sum);
  } else if (NT == 1 && a.x) {
    for (int m = warp / P; m < M; m += mstep) {
      const uint4* row = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(m) * K);
      uint32_t mx = 0;
      // kXB 32-byte loads in flight per lane before any is used
      for (int ch0 = part * 32 + lane; ch0 < cpr; ch0 += 32 * P * kXB) {
        // loads of this pass that start inside the row for the warp's first
        // lane (the same for every thread of the warp: the loops leave early
        // instead of running predicated-off iterations)
        const int nj = min(kXB, (cpr - (ch0 - lane) + 32 * P - 1) / (32 * P));
        uint4 v[kXB][2];
#pragma unroll
        for (int j = 0; j < kXB; ++j) {
          if (j >= nj) break;
          const int chu = ch0 + j * 32 * P;
          v[j][0] = v[j][1] = make_uint4(0, 0, 0, 0);
          if (chu < cpr) {
            v[j][0] = __ldg(row + 2 * chu);
            v[j][1] = __ldg(row + 2 * chu + 1);
          }
        }
#pragma unroll
        for (int j = 0; j < kXB; ++j) {
          if (j >= nj) break;
          mx = max(mx, absmax16_bits(v[j][0], v[j][1]));
        }
      }
      mx = __reduce_max_sync(0xffffffffu, mx);
      if (lane == 0) atomicMax(&sm.amax[m], mx);
    }
    __syncthreads();
    if (threadIdx.x < M) {
      const float sxv = act_scale(bf16_bits_to_f32(sm.amax[threadIdx.x]), FAITHFUL);
      sm.sx[threadIdx.x] = sxv;
      if (blockIdx.x == 0 && a.sx_out) a.sx_out[threadIdx.x] = sxv;
    }
  } else {
    if (threadIdx.x < M) sm.sx[threadIdx.x] = a.s_x[threadIdx.x];
  }
  // One token and a full round of 8 chunks in the one-pass path: warp w
  // quantised exactly chunk w, and its items are exactly the units of chunk
  // w, so it reads only x it wrote itself; the scales and row sums are read
  // after the barrier before the epilogue.
  if (NT == 1 && single && M == 1 && nchunks == kRoundChunks)
    __syncwarp();
  else
    __syncthreads();

  // forced-timeout test: a wait that nothing completes runs out, and the
  // CTA takes the same path as after any wait that gives up
  if (a.stall && !mbar_wait(&sm.stall, 0, a.wait_ns)) ok = false;
  ok = __all_sync(0xffffffffu, ok);

  const int r0 = mma_row_to_box(g);                  // sub-box rows r0 and r0 + 8
  ItemCursor cc = cstart;                            // next item to consume
  int cslot = 0;                                     // ring slot of the next item to consume
  // When the prologue requested every item of this warp (they fit in its
  // ring), one wait for all copies replaces the per-item waits.
  const bool per_item_wait = ic.r < nround;
  bool first_wait = true;
  int xchunk = -1;                                   // round-local chunk of the x fragment held
  // bf16 x (8 tokens at most): this lane's token row in shared memory, or
  // the zero bytes; the offsets of its pair-p pieces within a 256-k half
  const uint8_t* xtok = g < M ? reinterpret_cast<const uint8_t*>(xs) + g * S + 64 * t
                              : reinterpret_cast<const uint8_t*>(sm.zero);
  const int xpo[2] = {32 * (t >> 1), 32 * (1 ^ (t >> 1))};
  // [v][pair][token tile][field]: the two B words of the field's MMA (x
  // words i and 4 + i) side by side, as the MMA takes them
  uint2 xw[2][2][NT][4];
  for (int r = 0; r < nround; ++r) {
    const int c0 = r * kChunkK;
    const int ccpr = min(kChunkK, K - c0) >> 4;      // 16-element chunks of x in this round
    if (r > 0) __syncthreads();                      // every warp is done with the previous round's x
    // ---- x round -> int8 in shared memory (tokens < M only)
    for (int m = warp / P; m < ((NT == 2 || single || direct) ? 0 : M); m += mstep) {
      int8_t* xrow = xs + m * S;
      const float sxm = sm.sx[m];
      int sum = 0;
      const size_t roff = static_cast<size_t>(m) * K + c0;
      for (int ch0 = part * 32 + lane; ch0 < ccpr; ch0 += 32 * P * kQB) {
        if (a.x) {
          const uint4* src = reinterpret_cast<const uint4*>(a.x + roff);
          uint4 v[kQB][2];
#pragma unroll
          for (int j = 0; j < kQB; ++j) {
            const int chu = ch0 + j * 32 * P;
            if (chu < ccpr) {
              v[j][0] = __ldg(src + 2 * chu);
              v[j][1] = __ldg(src + 2 * chu + 1);
            }
          }
#pragma unroll
          for (int j = 0; j < kQB; ++j) {
            const int chu = ch0 + j * 32 * P;
            if (chu < ccpr) {
              const int ch = chu;
              const uint4 qv = quant16(v[j][0], v[j][1], sxm, sum, FAITHFUL);
              if (blockIdx.x == 0 && a.xq_out) *reinterpret_cast<uint4*>(a.xq_out + roff + 16 * ch) = qv;
              *reinterpret_cast<uint4*>(xrow + 16 * xs_chunk(ch)) = qv;
            }
          }
        } else {
          const uint4* src = reinterpret_cast<const uint4*>(a.xq + roff);
          uint4 v[kQB];
#pragma unroll
          for (int j = 0; j < kQB; ++j) {
            const int ch = ch0 + j * 32 * P;
            if (ch < ccpr) v[j] = __ldg(src + ch);
          }
#pragma unroll
          for (int j = 0; j < kQB; ++j) {
            const int ch = ch0 + j * 32 * P;
            if (ch < ccpr) {
              sum = bytesum16(v[j], sum);
              *reinterpret_cast<uint4*>(xrow + 16 * xs_chunk(ch)) = v[j];
            }
          }
        }
      }
      sum = __reduce_add_sync(0xffffffffu, sum);
      if (lane == 0) atomicAdd(&sm.rsum[m], sum);
    }
    if (!single && !direct) __syncthreads();
    xchunk = -1;

    // ---- this warp's items of round r
    while (ok && cc.r == r) {
      const int s = cslot;
      // this item's copies (the oldest group in flight) have landed, for
      // every lane of the warp
      if (per_item_wait) {
        cp_async_wait(ring - 1);
        __syncwarp();
      } else if (first_wait) {
        cp_async_wait(0);
        __syncwarp();
        first_wait = false;
      }
      const int ug = cc.p;                           // unit group of the item
      const int lc = cc.g;                           // round-local chunk of the item
      if (lc != xchunk) {
        if (NT == 2 || direct) {                    // bf16 x comes with 8 tokens at most
#pragma unroll
          for (int v = 0; v < 2; ++v)
#pragma unroll
            for (int pr = 0; pr < 2; ++pr)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                const int m = nt * 8 + g;
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                  // every lane loads (a token and chunk that exist where its
                  // own do not) and keeps zeros for missing tokens and k
                  const int xc = 32 * lc + 16 * v + 4 * t + 2 * pr + c2;    // 16-byte chunk in the round
                  const bool xin = m < M && 16 * xc < K - r * kChunkK;
                  const int mr = xin ? m : 0, xr = xin ? xc : 0;
                  uint4 xv = __ldg(reinterpret_cast<const uint4*>(a.xq + static_cast<size_t>(mr) * K + r * kChunkK) + xr);
                  if (!xin) xv = make_uint4(0, 0, 0, 0);
                  if (c2 == 0) {
                    xw[v][pr][nt][0].x = xv.x; xw[v][pr][nt][1].x = xv.y;
                    xw[v][pr][nt][2].x = xv.z; xw[v][pr][nt][3].x = xv.w;
                  } else {
                    xw[v][pr][nt][0].y = xv.x; xw[v][pr][nt][1].y = xv.y;
                    xw[v][pr][nt][2].y = xv.z; xw[v][pr][nt][3].y = xv.w;
                  }
                }
              }
        } else {
          // chunk lc of this lane's token in shared memory (the 512 zero
          // bytes for a token that does not exist); the 16-byte pieces are at
          // 256 v + 64 t + 32 (pr ^ (t >> 1)) + 16 c2, the swizzle of
          // xs_chunk written out for this lane
          const uint8_t* xb = xtok + (g < M ? 512 * lc : 0);
#pragma unroll
          for (int v = 0; v < 2; ++v)
#pragma unroll
            for (int pr = 0; pr < 2; ++pr)
#pragma unroll
              for (int c2 = 0; c2 < 2; ++c2) {
                const uint4 xv = *reinterpret_cast<const uint4*>(xb + xpo[pr] + 256 * v + 16 * c2);
                if (c2 == 0) {
                  xw[v][pr][0][0].x = xv.x; xw[v][pr][0][1].x = xv.y;
                  xw[v][pr][0][2].x = xv.z; xw[v][pr][0][3].x = xv.w;
                } else {
                  xw[v][pr][0][0].y = xv.x; xw[v][pr][0][1].y = xv.y;
                  xw[v][pr][0][2].y = xv.z; xw[v][pr][0][3].y = xv.w;
                }
              }
        }
        xchunk = lc;
      }
      // per unit: 16 MMAs in four independent chains (one per field), then
      // the fields -> one sum per output (4^i sum(c q) >> 2i is exact: 64 * 2
      // * 127 * 512 < 2^31); only one unit's field accumulators are live
      int cv[UP][NT][4];
      const uint8_t* box = wring + s * kSlotBytes;
#pragma unroll
      for (int e = 0; e < UP; ++e) {
        // the missing unit of a CTA's last group (odd unit count) is all
        // zeros: no MMAs for it (the same for the whole warp)
        if (UP > 1 && e > 0 && UP * ug + e >= U) break;
        int acc[4][NT][4];
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const int cw = 4 * v + t;                  // 16-byte chunk of the 128-byte row
          const uint4 wa = *reinterpret_cast<const uint4*>(box + e * kSubBytes + r0 * 128 + ((cw ^ r0) << 4));
          const uint4 wb = *reinterpret_cast<const uint4*>(box + e * kSubBytes + (r0 + 8) * 128 + ((cw ^ r0) << 4));
          const uint32_t w0[4] = {wa.x, wa.y, wa.z, wa.w};
          const uint32_t w1[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
          for (int pr = 0; pr < 2; ++pr)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t mask = kCodeMask << (2 * i);
              const uint32_t a0 = w0[2 * pr] & mask, a1 = w1[2 * pr] & mask;
              const uint32_t a2 = w0[2 * pr + 1] & mask, a3 = w1[2 * pr + 1] & mask;
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                if (v == 0 && pr == 0)
                  mma_u8s8_first(acc[i][nt], a0, a1, a2, a3, xw[v][pr][nt][i].x, xw[v][pr][nt][i].y);
                else
                  mma_u8s8(acc[i][nt], a0, a1, a2, a3, xw[v][pr][nt][i].x, xw[v][pr][nt][i].y);
              }
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int rr = 0; rr < 4; ++rr)
            cv[e][nt][rr] = mad_hi(acc[3][nt][rr], 1 << 26,
                                   mad_hi(acc[2][nt][rr], 1 << 28, mad_hi(acc[1][nt][rr], 1 << 30, acc[0][nt][rr])));
      }
      // the slot is read: refill it with this warp's next item
      __syncwarp();
      cslot = cslot + 1 == ring ? 0 : cslot + 1;
      cc.next(warp, nround, nchunks, PU);
      issue_next();
      // the units' sums; a short group's missing unit is skipped
#pragma unroll
      for (int e = 0; e < UP; ++e) {
        const int u = UP * ug + e;
        if (UP > 1 && u >= U) break;
        int* au = acc_s + u * kUnitRows * NTOK;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int m0 = nt * 8 + 2 * t;
          if (m0 < M) {
            red_shared_add(au + sum_idx<NTOK>(r0, m0), cv[e][nt][0]);
            red_shared_add(au + sum_idx<NTOK>(r0 + 8, m0), cv[e][nt][2]);
          }
          if (m0 + 1 < M) {
            red_shared_add(au + sum_idx<NTOK>(r0, m0 + 1), cv[e][nt][1]);
            red_shared_add(au + sum_idx<NTOK>(r0 + 8, m0 + 1), cv[e][nt][3]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int i = threadIdx.x + k * kThreads;
    if (i < U * kUnitRows) bias_s[i] = bvals[k];
  }
  if (threadIdx.x < M * a.ngroups) {
    // d = s_x s_w of the token and the group (on a bf16 module bf16(bf16(s_w)
    // s_x)), kept as the double 1 / d: RN_f32(a * (1/d)) is RN_f32(a / d) for
    // every float32 (or bf16) numerator a -- a quotient of two floats lies at
    // least 2^-49 (relative) from every float32 midpoint, and the double
    // product is within 2^-52 of it.  s_x of token m is in shared memory
    // since the x phase (for one token, written by this warp).
    const float sx = sm.sx[threadIdx.x % M];
    const float d = FAITHFUL ? bf16_round(__fmul_rn(bf16_round(swv), sx)) : __fmul_rn(sx, swv);
    sm.rcp[threadIdx.x] = __drcp_rn(static_cast<double>(d));
  }
  // every copy this thread issued has landed before the CTA exits
  cp_async_wait(0);
  if (!ok) {
    report_status(a.status, kStatusTimeout);
    if (lane == 0) sm.failed = 1;
  }
  __syncthreads();                                   // s_w, the bias and the sums are in shared memory

  // ---------------- epilogue: U units x 16 rows x M tokens ----------------
  // output idx = m rows + rl: thread t starts at idx = t and steps by
  // kThreads = dm rows + drl (no division per output)
  const int rows = U * kUnitRows;
  const int dm = kThreads / rows, drl = kThreads - dm * rows;
  int m = static_cast<int>(threadIdx.x) / rows, rl = static_cast<int>(threadIdx.x) - m * rows;
  for (; m < M; m += dm, rl += drl) {
    if (rl >= rows) {
      rl -= rows;
      ++m;
      if (m >= M) break;
    }
    const int n = u_begin * kUnitRows + rl;
    if (n >= N) continue;
    const int accv = acc_s[(rl >> 4) * kUnitRows * NTOK + sum_idx<NTOK>(rl & 15, m)] - sm.rsum[m];
    int gi = 0;                                      // the row's group (scale), when layers are stacked
    if (a.ngroups > 1) {
#pragma unroll
      for (int gg = 0; gg + 1 < kMaxGroups; ++gg) gi += (gg + 1 < a.ngroups && n >= a.group_end[gg]) ? 1 : 0;
    }
    const double r = sm.rcp[gi * M + m];
    float y32;
    if (!FAITHFUL) {
      y32 = __double2float_rn(static_cast<double>(static_cast<float>(accv)) * r);
      if (a.bias) y32 = __fadd_rn(y32, bf16_bits_to_f32(bias_s[rl]));
    } else {
      // bf16 module: F.linear's sum, the scale product, the quotient and the
      // bias add are each a bf16 tensor
      y32 = bf16_round(__double2float_rn(static_cast<double>(bf16_round(static_cast<float>(accv))) * r));
      if (a.bias) y32 = bf16_round(__fadd_rn(y32, bf16_bits_to_f32(bias_s[rl])));
    }
    const size_t o = static_cast<size_t>(m) * N + n;
    if (a.y) a.y[o] = f32_to_bf16_bits(y32);
    if (a.acc_out) a.acc_out[o] = accv;
    if (a.y32_out) a.y32_out[o] = y32;
  }
}

template <int NT, bool FAITHFUL>
cudaError_t launch_nt(const DecodeArgs& a, const DecodePlan& p, cudaStream_t stream) {
  auto kern = decode_kernel<NT, FAITHFUL>;
  static unsigned long long attr_done = 0;        // one bit per device
  cudaError_t ea = set_smem_attr_once(kern, 227 * 1024, &attr_done);
  if (ea != cudaSuccess) return ea;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace

// Items of one chunk (2 KB) and up to 4 items in flight per warp: 64 KB in
// flight per CTA.  A streaming probe on B200 (chained launches, all SMs)
// found 64 KB per CTA as fast as any deeper ring at every decode shape, and
// 128 KB per CTA slower.
#ifndef BITLINEAR_DECODE_RING
#define BITLINEAR_DECODE_RING 4     // largest ring per warp
#endif

DecodePlan plan_decode(int M, int N, int K, int num_sms, bool direct) {
  DecodePlan p;
  const int units_total = (N + kUnitRows - 1) / kUnitRows;
  // One CTA per SM leaves room for the next kernel of the stream to start
  // beside this one; on the widest matrices (8 units per SM or more) two
  // 8-token CTAs per SM, both computing, stream faster.
  const int cap = (M <= 8 && units_total >= 8 * num_sms) ? 2 * num_sms : num_sms;
  p.grid = units_total < cap ? units_total : cap;
  if ((units_total + p.grid - 1) / p.grid > kMaxUnits) p.grid = (units_total + kMaxUnits - 1) / kMaxUnits;
  p.units_max = (units_total + p.grid - 1) / p.grid;
  // items of one chunk (the copy offsets of a lane are fixed for that size)
  p.tail = (K % kBoxK) != 0;
  p.slot_bytes = static_cast<size_t>(units_per_item(M <= 8 ? 1 : 2)) * kSubBytes;
  // shared-memory budget: two CTAs per SM for the 8-token kernel (the next
  // kernel on the stream can start beside this one; the 16-token kernel's
  // registers allow one); int8 x is not staged in shared memory
  const int mx = direct ? 0 : M;
  const long long budget = M <= 8 ? 110 * 1024 : 220 * 1024;
  const long long room = budget - static_cast<long long>(smem_layout(M, mx, 0, p.slot_bytes, p.units_max).total);
  long long ring = room > 0 ? room / (static_cast<long long>(kWarps) * static_cast<long long>(p.slot_bytes)) : 0;
  ring = ring > BITLINEAR_DECODE_RING ? BITLINEAR_DECODE_RING : ring;
  p.ring = ring < 1 ? 1 : static_cast<int>(ring);
  p.smem = smem_layout(M, mx, p.ring, p.slot_bytes, p.units_max).total;
  return p;
}

cudaError_t launch_decode(DecodeArgs a, int num_sms, cudaStream_t stream) {
  if (a.M <= 0) return cudaSuccess;
  // above 8 tokens the activations come quantised, with their row sums
  if (a.M > 8 && (a.xq == nullptr || a.rowsum == nullptr)) return cudaErrorInvalidValue;
  if (a.xq != nullptr && a.rowsum == nullptr) return cudaErrorInvalidValue;
  const DecodePlan p = plan_decode(a.M, a.N, a.K, num_sms, a.xq != nullptr);
  a.ring = p.ring;
  a.units_max = p.units_max;
  a.tail = p.tail;
  if (p.smem > 227 * 1024) return cudaErrorInvalidValue;
  if (a.faithful) return a.M <= 8 ? launch_nt<1, true>(a, p, stream) : launch_nt<2, true>(a, p, stream);
  return a.M <= 8 ? launch_nt<1, false>(a, p, stream) : launch_nt<2, false>(a, p, stream);
}

}  // namespace bitlinear
