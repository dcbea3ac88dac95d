// Shared device/host definitions of the MoE layer kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Cycles a bounded device wait spins before it records MOE_ERR_TIMEOUT and
// gives up (about one second at the B200's boost clock).
constexpr long long kWaitBudgetCycles = 2000000000LL;

// Where a timed-out wait records itself (low bits of the status word).
enum WaitSite : int32_t {
  kSiteProducerEmpty = 1,
  kSiteMmaFull = 2,
  kSiteMmaAccEmpty = 3,
  kSiteEpiAccFull = 4,
  kSiteDrain = 5,
  kSiteBadIndex = 6,  // an expert id / row index outside its range (skipped)
  kSiteSelfTest = 7,  // the wait of moe_check_wait_timeout
  kSiteRowCopy = 8,   // a row's bulk load in the row scatter
};

// status word: 0 = ok; else (MOE_ERR_TIMEOUT << 8) | site
__device__ __forceinline__ void record_timeout(int32_t* status, int site) {
  atomicCAS(status, 0, (MOE_ERR_TIMEOUT << 8) | site);
}

__device__ __forceinline__ void record_bad_index(int32_t* status) {
  if (status) atomicCAS(status, 0, (MOE_ERR_INVALID_ARG << 8) | kSiteBadIndex);
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ constexpr int64_t align_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Gated expert activations: the GEMM-1 epilogue computes act(g) * u from the
// gate projection g and the up projection u ("Experts backends": experts with
// a gated activation, silu / gelu / relu, i.e. SwiGLU / GeGLU / ReGLU).
enum Act : int { kActNone = 0, kActSilu = 1, kActGelu = 2, kActRelu = 3 };

template <int ACT>
__device__ __forceinline__ float gated(float g, float u) {
  if constexpr (ACT == kActSilu) {
    return __fdividef(g, 1.0f + __expf(-g)) * u;  // g * sigmoid(g)
  } else if constexpr (ACT == kActGelu) {
    return 0.5f * g * (1.0f + erff(g * 0.7071067811865476f)) * u;  // g * Phi(g), erf form
  } else {
    return fmaxf(g, 0.0f) * u;
  }
}

// Launch bookkeeping (defined in capi.cu).
void note_launch();

}  // namespace moe
