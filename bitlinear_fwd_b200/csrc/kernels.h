// Internal launch functions of the BitLinear kernels (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace bitlinear {

// ---- device check (api.cu): BITLINEAR_OK when the current GPU is sm_100 ----
int current_device_status();

// ---- TMA tensor maps (tensor_map.cu) ---------------------------------------
bool encode_2d_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                  uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);
// 2-D map over 16-bit elements (no swizzle), for tile stores
bool encode_2d_u16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                   uint32_t box_inner, uint32_t box_outer);

// ---- activation quantisation (act_quant.cu) --------------------------------
// pdl: launch as a programmatic dependent of the previous kernel on the stream
// (the kernel waits for it before touching memory).
// faithful: the bf16-module rounding of every step (scale = bf16(bf16(1/a) * 127),
// q = round(bf16(x * scale))) instead of float32 arithmetic
// absmax_in: the tokens' absmax over the whole row when x is one K-shard of
// it (null: the kernel forms it from x)
cudaError_t launch_act_quant(const uint16_t* x, int M, int K, int8_t* xq, float* s_x,
                             int32_t* rowsum, uint32_t* status_clear, bool pdl, cudaStream_t stream,
                             bool faithful = false, const float* absmax_in = nullptr);
// float32 max_k |x[m, k]| of each token over this x
cudaError_t launch_act_absmax(const uint16_t* x, int M, int K, float* absmax, cudaStream_t stream);

// ---- weight absmean + ternarise + pack (pack.cu) ----------------------------
// Workspace layout used by the pack kernels.
struct PackWorkspace {
  uint32_t* status;   // 1 word
  float* mean;        // 1 float
  uint64_t* bins;     // kAbsmeanBins exponent bins
};
// Exponent bins of the exact absmean sum: bin e holds a sum of 24-bit
// significands of weight 2^(max(e,1) - 150); the window sums' chunks reach
// exponents up to 254 - 36 + 72 = 290.
constexpr int kAbsmeanBins = 320;
constexpr size_t kPackWsBytes = 4096;
PackWorkspace pack_workspace(void* ws);
cudaError_t launch_pack(const float* w, int64_t N, int64_t K, uint8_t* packed, float* w_scale,
                        float* w_mean, const PackWorkspace& pws, cudaStream_t stream);
// The exact exponent-bin form of sum |w| over this w (bins[kAbsmeanBins] are
// overwritten): integer bins that add across shards.
cudaError_t launch_absmean_bins(const float* w, int64_t N, int64_t K, uint64_t* bins, cudaStream_t stream);
// s_w and the exact mean from bins summed over all shards (n_total weights
// in all), then the ternary codes of this w.
cudaError_t launch_pack_from_bins(const float* w, int64_t N, int64_t K, const uint64_t* bins, int64_t n_total,
                                  uint8_t* packed, float* w_scale, float* w_mean, const PackWorkspace& pws,
                                  cudaStream_t stream);

// ---- epilogue over summed partial accumulators (epilogue.cu) ---------------
constexpr int kMaxParts = 8;
struct EpilogueArgs {
  const int32_t* part[kMaxParts];  // [M, N] int32 partial sums, added in order
  int nparts;
  const float* absmax;    // [M] tokens' absmax over the whole K
  const float* w_scale;   // [1]
  const uint16_t* bias;   // [N] or null
  uint16_t* y;            // [M, N]
  int32_t* acc_out;       // [M, N] or null: the summed accumulators
  int64_t M, N;
  int faithful;
};
cudaError_t launch_epilogue(const EpilogueArgs& a, int num_sms, cudaStream_t stream);

// ---- shared forward arguments ----------------------------------------------
// Rows [group_end[g-1], group_end[g]) of the packed matrix form group g,
// scaled by w_scale[g] (one group for a plain layer).
constexpr int kMaxGroups = 8;

struct ForwardArgs {
  const int8_t* xq;       // [M, K]
  const float* s_x;       // [M]
  const int32_t* rowsum;  // [M]
  const uint8_t* packed;  // [N, K/4]
  const float* w_scale;   // [ngroups]
  const uint16_t* bias;   // [N] or null
  uint16_t* y;            // [M, N]
  int32_t* acc_out;       // [M, N] or null (debug)
  float* y32_out;         // [M, N] or null (debug)
  uint32_t* status;       // status word
  int M, N, K;
  int ngroups;
  int group_end[kMaxGroups];
  bool pdl;               // launched as a programmatic dependent of the act-quant kernel
  bool faithful;          // bf16-module epilogue: every step rounded to bf16
  uint64_t wait_ns;       // limit of the main-loop waits (drains keep kWaitLimitNs)
  int stall;              // test hook: first wait on a barrier nothing signals
  bool y_tma;             // set by the launcher: y tiles staged in shared memory and stored by TMA
};

// ---- bf16 export of packed weights (dequant.cu) ----------------------------
cudaError_t launch_dequant(const uint8_t* packed, int64_t N, int64_t K, const float* w_scale, uint16_t* w_bf16,
                           int num_sms, cudaStream_t stream);

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel and
// device (the attribute belongs to the device that is current at the call)
template <typename Kern>
cudaError_t set_smem_attr_once(Kern kern, int bytes, unsigned long long* done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (__atomic_load_n(done_mask, __ATOMIC_ACQUIRE) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) __atomic_fetch_or(done_mask, bit, __ATOMIC_RELEASE);
  return e;
}

// ---- the int8 tensor-core rate (tc_peak.cu), a measurement utility ---------
cudaError_t launch_tc_i8_peak(int iters, int num_sms, uint32_t* status, cudaStream_t stream);

// ---- decode engine, M <= 16 (gemv_decode.cu) --------------------------------
struct DecodeArgs {
  const uint16_t* x;      // bf16 [M, K], quantised inside the kernel; or null
  const int8_t* xq;       // int8 [M, K] with s_x and rowsum when x is null
  const float* s_x;       // [M]
  const int32_t* rowsum;  // [M] sum of q per token, with xq
  const uint8_t* packed;  // [N, K/4]
  const float* w_scale;   // [ngroups]
  const uint16_t* bias;   // [N] or null
  uint16_t* y;            // [M, N]
  int8_t* xq_out;         // [M, K] or null (debug, quantising path)
  float* sx_out;          // [M] or null (debug, quantising path)
  int32_t* acc_out;       // [M, N] or null (debug)
  float* y32_out;         // [M, N] or null (debug)
  uint32_t* status;       // status word or null
  int M, N, K;
  int ngroups;
  int group_end[kMaxGroups];
  int faithful;           // bf16-module rounding of the quantisation and the epilogue
  int ring, units_max, tail;      // set by launch_decode
  int weights_early;      // the packed weights, w_scale and bias may be read before the dependency wait
  uint64_t wait_ns;       // limit of the main-loop waits (drains keep kWaitLimitNs)
  int stall;              // test hook: first wait on a barrier nothing signals
};

// Main-loop wait limits: the default, and the short one used while the
// forced-timeout test hook is on.
constexpr uint64_t kTestWaitLimitNs = 1000ull * 1000ull;   // 1 ms
// Wait limit and stall flag for the next launch (the forced-timeout test hook
// of api.cu).
uint64_t launch_wait_ns();
int launch_stall();
struct DecodePlan {
  int grid, units_max, ring, tail;
  size_t slot_bytes, smem;
};
DecodePlan plan_decode(int M, int N, int K, int num_sms, bool direct);
cudaError_t launch_decode(DecodeArgs a, int num_sms, cudaStream_t stream);

// ---- prefill engine, tcgen05 GEMM (gemm_prefill.cu) -------------------------
cudaError_t launch_gemm_prefill(const ForwardArgs& a, int num_sms, cudaStream_t stream);

}  // namespace bitlinear
