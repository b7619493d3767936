// CPU oracle of the BitNet b1.58 BitLinear forward, in plain C++.
//
// TEST INFRASTRUCTURE.  Only the tests, the smoke entry point and the CPU
// baseline legs of the benchmark may load this library.  It shares no code
// with the CUDA path: no header, helper, table or constant comes from there.
// The compile flags keep IEEE single-precision arithmetic as written
// (-ffp-contract=off, no fast-math), so every float operation below rounds
// once, to nearest even.
//
// Plain loops, one step per function, in the order of the source pages:
//
// * [FE-univ]  Falcon-LLM team, "Falcon-Edge: a series of powerful,
//   universal and fine-tunable 1.58bit language models" (blog), section
//   "Falcon-Edge, a series of universal models": activation_norm_quant,
//   class BitLinear (post_quant_process, forward) and _weight_quant with the
//   state-dict export loop.
// * [GN-BitNet] "BitNet: inference framework for 1-bit LLMs" (GeekNews),
//   Hacker News comments: weights stored in 2 bits (four codes).
// * [Era-1bit] "The Era of 1-bit LLMs" (aitrends.kr summary), TL;DR: every
//   weight is ternary {-1, 0, 1}.
//
// Readings where the pages leave a step open (the same as the numpy oracle's):
// round() is round-half-to-even; scales and the products x*s, w*s are
// float32; the clamp constant is the float32 1e-5f; mean|w| is the exact sum
// rounded once to float32 (last place never below 2^-149); F.linear on the
// integer operands is the exact integer sum; the epilogue is d = s_x*s_w,
// acc/d, + bias, each in float32, then one rounding to bfloat16; the packing
// stores u+1 in bit pair i of byte j of little-endian word g for
// k = 16g + 4i + j (code 3 is invalid).  The bf16-faithful mode rounds every
// tensor op of the listings to bfloat16, with 127/t evaluated as
// (1/t)*127 and the module's bf16 copy of s_w.  The export divides u by s_w
// in float32 and rounds once to bfloat16; a zero code exports as +0.
//
// Every entry point returns 0 on success or a negative status:
//   -1 bad argument (null pointer, negative size, K not a multiple of 16,
//      a weight outside {-1,0,1}, group rows that do not add up to N),
//   -2 a packed bit pair holds the unused code 3,
//   -3 a non-finite weight,
//   -4 a size beyond what the exact arithmetic below holds.
// All buffers are host memory owned by the caller; nothing is kept between
// calls.
//
// ORACLE_PLANT (default 0) exists only so that a test can build a copy with
// one known mistake and check that the pins catch it: 1 rounds down instead
// of to nearest in the activation quantisation, 2 multiplies instead of
// divides in the epilogue, 3 swaps i and j in the packing layout.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifndef ORACLE_PLANT
#define ORACLE_PLANT 0
#endif

namespace {

const int kOk = 0;
const int kBadArgument = -1;
const int kInvalidCode = -2;
const int kNonFinite = -3;
const int kTooLarge = -4;

const float kClampMin = 1e-5f;   // the listings' clamp_(min=1e-5)
const float kQmax = 127.0f;      // activation_norm_quant's 127.0

// ---------------------------------------------------------------------------
// bfloat16 storage (not part of the method)
// ---------------------------------------------------------------------------

float from_bf16(uint16_t bits) {
    uint32_t u = static_cast<uint32_t>(bits) << 16;
    float f;
    std::memcpy(&f, &u, sizeof f);
    return f;
}

// Nearest bfloat16, ties to even (finite inputs).
uint16_t to_bf16(float f) {
    uint32_t u;
    std::memcpy(&u, &f, sizeof u);
    uint64_t lsb = (u >> 16) & 1u;
    return static_cast<uint16_t>((static_cast<uint64_t>(u) + 0x7FFFu + lsb) >> 16);
}

float round_bf16(float f) { return from_bf16(to_bf16(f)); }

float clamp_q(float t, float lo, float hi) { return t < lo ? lo : (t > hi ? hi : t); }

// ---------------------------------------------------------------------------
// Step 1: per-token absmax quantisation  ([FE-univ] activation_norm_quant)
// ---------------------------------------------------------------------------

// For row m: a = max_k |x|, s_x = 127 / max(a, 1e-5), q = clamp(round(x*s_x),
// -128, 127).  bf16 mode: s_x = bf16(bf16(1 / max(a, bf16(1e-5))) * 127) and
// q = clamp(round(bf16(x*s_x)), -128, 127).
void act_quant_row(const uint16_t* x, int64_t K, bool bf16_mode, int8_t* q, float* s_x, int32_t* rowsum) {
    float a = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float v = std::fabs(from_bf16(x[k]));
        if (v > a) a = v;
    }
    float s;
    if (bf16_mode) {
        float lo = round_bf16(kClampMin);
        float inv = round_bf16(1.0f / (a > lo ? a : lo));
        s = round_bf16(inv * kQmax);
    } else {
        s = kQmax / (a > kClampMin ? a : kClampMin);
    }
    int64_t sum = 0;
    for (int64_t k = 0; k < K; ++k) {
        float t = from_bf16(x[k]) * s;
        if (bf16_mode) t = round_bf16(t);
        float r = clamp_q(ORACLE_PLANT == 1 ? std::floor(t) : std::nearbyint(t), -128.0f, 127.0f);
        q[k] = static_cast<int8_t>(r);
        sum += q[k];
    }
    *s_x = s;
    *rowsum = static_cast<int32_t>(sum);
}

// ---------------------------------------------------------------------------
// Step 2a: absmean  ([FE-univ] _weight_quant: w.abs().mean())
// ---------------------------------------------------------------------------

// An unsigned integer in 32-bit limbs, least significant first.  A finite
// |w| is below 2^128, i.e. below 2^277 units of 2^-149; a sum of fewer than
// 2^32 of them is below 2^309 units, so 12 limbs (384 bits) hold it.
const int kLimbs = 12;

void wide_add(uint32_t* limb, uint64_t value, int shift) {
    int i = shift / 32;
    uint64_t carry = value << (shift % 32);   // value < 2^24: below 2^56
    while (carry != 0) {
        uint64_t s = static_cast<uint64_t>(limb[i]) + (carry & 0xFFFFFFFFu);
        limb[i] = static_cast<uint32_t>(s);
        carry = (carry >> 32) + (s >> 32);
        ++i;
    }
}

int wide_bit(const uint32_t* limb, int b) { return (limb[b / 32] >> (b % 32)) & 1; }

int wide_bit_length(const uint32_t* limb) {
    for (int i = kLimbs - 1; i >= 0; --i)
        for (int b = 31; b >= 0; --b)
            if ((limb[i] >> b) & 1u) return 32 * i + b + 1;
    return 0;
}

// mean = S * 2^-149 / n, with S the exact sum of |w| in units of 2^-149,
// rounded to the nearest float32 (ties to even, last place >= 2^-149).
int absmean(const float* w, int64_t n, float* mean) {
    if (n <= 0) return kBadArgument;
    if (n >= (int64_t(1) << 32)) return kTooLarge;
    uint32_t S[kLimbs] = {0};
    for (int64_t i = 0; i < n; ++i) {
        uint32_t bits;
        std::memcpy(&bits, &w[i], sizeof bits);
        uint32_t e = (bits >> 23) & 0xFFu;
        if (e == 0xFFu) return kNonFinite;
        uint32_t m = bits & 0x7FFFFFu;
        if (e > 0) m |= 0x800000u;
        // |w| = m * 2^(max(e,1) - 150) = (m << (max(e,1) - 1)) units of 2^-149
        wide_add(S, m, (e > 0 ? static_cast<int>(e) : 1) - 1);
    }
    // Q = floor(S / n), r = S mod n (long division, most significant limb first)
    uint64_t den = static_cast<uint64_t>(n), r = 0;
    for (int i = kLimbs - 1; i >= 0; --i) {
        uint64_t cur = (r << 32) | S[i];
        S[i] = static_cast<uint32_t>(cur / den);
        r = cur % den;
    }
    int L = wide_bit_length(S);
    uint64_t R;
    int exp2;
    if (L <= 24) {
        // below 2^-125: the last place is 2^-149, round Q + r/n to an integer
        uint64_t Q = S[0];
        bool up = 2 * r > den || (2 * r == den && (Q & 1u));
        R = Q + (up ? 1 : 0);
        exp2 = -149;
    } else {
        // keep the top 24 bits of Q; the bits below and r decide the rounding
        int sh = L - 24;
        uint64_t top = 0;
        for (int b = L - 1; b >= sh; --b) top = (top << 1) | static_cast<uint64_t>(wide_bit(S, b));
        int half = wide_bit(S, sh - 1);
        bool sticky = r != 0;
        for (int b = 0; b < sh - 1 && !sticky; ++b) sticky = wide_bit(S, b) != 0;
        bool up = half && (sticky || (top & 1u));
        R = top + (up ? 1 : 0);
        exp2 = sh - 149;
    }
    *mean = static_cast<float>(std::ldexp(static_cast<double>(R), exp2));   // exact: R <= 2^24
    return kOk;
}

// s_w = 1 / max(mean, 1e-5)  ([FE-univ] _weight_quant)
float weight_scale(float mean) { return 1.0f / (mean > kClampMin ? mean : kClampMin); }

// u = clamp(round(w * s_w), -1, 1)  ([FE-univ] _weight_quant; [Era-1bit])
int8_t ternarise_one(float w, float s_w) {
    return static_cast<int8_t>(clamp_q(std::nearbyint(w * s_w), -1.0f, 1.0f));
}

// ---------------------------------------------------------------------------
// Step 2c: 2-bit packing ([GN-BitNet]); byte b = 4g + j of a row holds
// k = 16g + 4i + j in its bit pair i, for i = 0..3
// ---------------------------------------------------------------------------

int64_t k_of(int64_t byte, int i) {
    return ORACLE_PLANT == 3 ? 16 * (byte / 4) + 4 * (byte % 4) + i : 16 * (byte / 4) + 4 * i + byte % 4;
}

// ---------------------------------------------------------------------------
// Step 4: epilogue  ([FE-univ] BitLinear.post_quant_process, bias add)
// ---------------------------------------------------------------------------

void epilogue_one(int32_t acc, float s_x, float s_w, const uint16_t* bias, bool bf16_mode,
                  float* y32, uint16_t* y) {
    float v;
    if (bf16_mode) {
        float d = round_bf16(round_bf16(s_w) * s_x);
        v = round_bf16(round_bf16(static_cast<float>(acc)) / d);
        if (bias) v = round_bf16(v + from_bf16(*bias));
    } else {
        float d = s_x * s_w;
        v = ORACLE_PLANT == 2 ? static_cast<float>(acc) * d : static_cast<float>(acc) / d;
        if (bias) v = v + from_bf16(*bias);
    }
    *y32 = v;
    *y = to_bf16(v);
}

}  // namespace

extern "C" {

int oracle_bf16_to_f32(const uint16_t* bits, int64_t n, float* out) {
    if (n < 0 || (n > 0 && (!bits || !out))) return kBadArgument;
    for (int64_t i = 0; i < n; ++i) out[i] = from_bf16(bits[i]);
    return kOk;
}

int oracle_f32_to_bf16(const float* v, int64_t n, uint16_t* out) {
    if (n < 0 || (n > 0 && (!v || !out))) return kBadArgument;
    for (int64_t i = 0; i < n; ++i) out[i] = to_bf16(v[i]);
    return kOk;
}

// x: bf16 bits [M, K]; q: int8 [M, K]; s_x: float [M]; rowsum: int32 [M].
int oracle_act_quant(const uint16_t* x, int64_t M, int64_t K, int bf16_mode,
                     int8_t* q, float* s_x, int32_t* rowsum) {
    if (M < 0 || K < 0) return kBadArgument;
    if (M > 0 && (!s_x || !rowsum || (K > 0 && (!x || !q)))) return kBadArgument;
    for (int64_t m = 0; m < M; ++m)
        act_quant_row(x + m * K, K, bf16_mode != 0, q + m * K, &s_x[m], &rowsum[m]);
    return kOk;
}

int oracle_absmean(const float* w, int64_t n, float* mean) {
    if (!w || !mean) return kBadArgument;
    return absmean(w, n, mean);
}

float oracle_weight_scale(float mean) { return weight_scale(mean); }

int oracle_ternarise(const float* w, int64_t n, float s_w, int8_t* u) {
    if (n < 0 || (n > 0 && (!w || !u))) return kBadArgument;
    for (int64_t i = 0; i < n; ++i) u[i] = ternarise_one(w[i], s_w);
    return kOk;
}

// u: int8 [N, K] in {-1,0,1}, K % 16 == 0; packed: uint8 [N, K/4].
int oracle_pack(const int8_t* u, int64_t N, int64_t K, uint8_t* packed) {
    if (N < 0 || K < 0 || K % 16 != 0) return kBadArgument;
    if (N * K > 0 && (!u || !packed)) return kBadArgument;
    for (int64_t i = 0; i < N * K; ++i)
        if (u[i] < -1 || u[i] > 1) return kBadArgument;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < K / 4; ++b) {
            unsigned byte = 0;
            for (int i = 0; i < 4; ++i)
                byte |= static_cast<unsigned>(u[n * K + k_of(b, i)] + 1) << (2 * i);
            packed[n * (K / 4) + b] = static_cast<uint8_t>(byte);
        }
    return kOk;
}

int oracle_unpack(const uint8_t* packed, int64_t N, int64_t K, int8_t* u) {
    if (N < 0 || K < 0 || K % 16 != 0) return kBadArgument;
    if (N * K > 0 && (!u || !packed)) return kBadArgument;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < K / 4; ++b)
            for (int i = 0; i < 4; ++i) {
                unsigned code = (packed[n * (K / 4) + b] >> (2 * i)) & 3u;
                if (code == 3u) return kInvalidCode;
                u[n * K + k_of(b, i)] = static_cast<int8_t>(static_cast<int>(code) - 1);
            }
    return kOk;
}

// acc[m, n] = sum_k q[m, k] * u[n, k]  ([FE-univ] BitLinear.forward, F.linear)
int oracle_contract(const int8_t* q, const int8_t* u, int64_t M, int64_t N, int64_t K, int32_t* acc) {
    if (M < 0 || N < 0 || K < 0) return kBadArgument;
    if (M * N > 0 && (!acc || (K > 0 && (!q || !u)))) return kBadArgument;
    if (128 * K > INT32_MAX) return kTooLarge;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) s += static_cast<int64_t>(q[m * K + k]) * u[n * K + k];
            acc[m * N + n] = static_cast<int32_t>(s);
        }
    return kOk;
}

// acc, y32, y: [M, N]; s_x: [M]; bias: bf16 bits [N] or null.
int oracle_epilogue(const int32_t* acc, int64_t M, int64_t N, const float* s_x, float s_w,
                    const uint16_t* bias, int bf16_mode, float* y32, uint16_t* y) {
    if (M < 0 || N < 0) return kBadArgument;
    if (M * N > 0 && (!acc || !s_x || !y32 || !y)) return kBadArgument;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            epilogue_one(acc[m * N + n], s_x[m], s_w, bias ? &bias[n] : nullptr, bf16_mode != 0,
                         &y32[m * N + n], &y[m * N + n]);
    return kOk;
}

// [FE-univ] _weight_quant, then packing: w float [N, K] -> packed [N, K/4],
// s_w and mean.
int oracle_pack_weights(const float* w, int64_t N, int64_t K, uint8_t* packed, float* s_w, float* mean) {
    if (!w || !s_w || !mean || N < 0 || K < 0 || K % 16 != 0) return kBadArgument;
    int st = absmean(w, N * K, mean);
    if (st != kOk) return st;
    *s_w = weight_scale(*mean);
    std::vector<int8_t> u(static_cast<size_t>(N * K));
    for (int64_t i = 0; i < N * K; ++i) u[i] = ternarise_one(w[i], *s_w);
    return oracle_pack(u.data(), N, K, packed);
}

// [FE-univ] BitLinear.forward on packed weights, for one layer
// (ngroups = 1) or several layers that read the same x: group g covers the
// next group_rows[g] rows of the packed matrix and of the output columns,
// with scale s_w[g].  Every intermediate is returned: q [M,K], s_x [M],
// rowsum [M], acc [M,N], y32 [M,N], y [M,N] (bf16 bits).
int oracle_forward(const uint16_t* x, int64_t M, int64_t K, const uint8_t* packed, int64_t N,
                   int ngroups, const int64_t* group_rows, const float* s_w, const uint16_t* bias,
                   int bf16_mode, int8_t* q, float* s_x, int32_t* rowsum, int32_t* acc,
                   float* y32, uint16_t* y) {
    if (M < 0 || N < 0 || K < 0 || K % 16 != 0 || ngroups < 1 || !group_rows || !s_w) return kBadArgument;
    int64_t total = 0;
    for (int g = 0; g < ngroups; ++g) {
        if (group_rows[g] < 0) return kBadArgument;
        total += group_rows[g];
    }
    if (total != N) return kBadArgument;
    int st = oracle_act_quant(x, M, K, bf16_mode, q, s_x, rowsum);
    if (st != kOk) return st;
    std::vector<int8_t> u(static_cast<size_t>(N * K));
    st = oracle_unpack(packed, N, K, u.data());
    if (st != kOk) return st;
    st = oracle_contract(q, u.data(), M, N, K, acc);
    if (st != kOk) return st;
    int64_t n0 = 0;
    for (int g = 0; g < ngroups; ++g) {
        for (int64_t m = 0; m < M; ++m)
            for (int64_t n = n0; n < n0 + group_rows[g]; ++n)
                epilogue_one(acc[m * N + n], s_x[m], s_w[g], bias ? &bias[n] : nullptr, bf16_mode != 0,
                             &y32[m * N + n], &y[m * N + n]);
        n0 += group_rows[g];
    }
    return kOk;
}

// [FE-univ] state-dict export: param_value = u / param_scale as bfloat16.
// out: bf16 bits [N, K].
int oracle_dequant(const uint8_t* packed, int64_t N, int64_t K, float s_w, uint16_t* out) {
    if (N < 0 || K < 0 || K % 16 != 0) return kBadArgument;
    if (N * K > 0 && (!packed || !out)) return kBadArgument;
    std::vector<int8_t> u(static_cast<size_t>(N * K));
    int st = oracle_unpack(packed, N, K, u.data());
    if (st != kOk) return st;
    for (int64_t i = 0; i < N * K; ++i) {
        float v = static_cast<float>(u[i]) / s_w;    // +-1/s_w rounded once; 0/s_w = +0
        out[i] = to_bf16(v);
    }
    return kOk;
}

}  // extern "C"
