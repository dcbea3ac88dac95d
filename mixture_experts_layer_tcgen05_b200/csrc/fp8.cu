// Fine-grained FP8 quantisation kernels.
//
// "Fine-grained FP8" (HF Transformers docs), opening list: weights are
// quantised to 8 bits per 128 x 128 block; activations per token per group
// of 128 input channels, dynamically. Scale rule (both): s = amax / 448 in
// fp32 (IEEE division), or the smallest power of two >= it with UE8M0
// scales, s = 1 for an all-zero group, code = e4m3 of v / s
// rounded to nearest even (the hardware cvt with satfinite; |v / s| <= 448
// up to one rounding, so saturation never changes a value).
#include <cuda_fp8.h>

#include <algorithm>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

// ue8m0: power-of-two scales (the UE8M0 scale format of "Experts backends"):
// the smallest 2^p >= amax / 448 (that fp32 quotient), p clamped to
// [-127, 127]; dividing by it only shifts exponents.
__device__ __forceinline__ float group_scale(float amax, bool ue8m0) {
  if (!(amax > 0.0f)) return 1.0f;
  const float r = __fdiv_rn(amax, 448.0f);
  if (!ue8m0) return r;
  int e;
  const float m = frexpf(r, &e);  // r = m * 2^e, m in [0.5, 1)
  const int p2 = min(max(m == 0.5f ? e - 1 : e, -127), 127);
  return ldexpf(1.0f, p2);
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// One warp per row; each step covers two 128-column groups (lanes 0-15 and
// 16-31, eight values each). Gather form (SCATTER false): output row p reads
// input row row_map[p] (the expert permutation) or p when row_map is NULL.
// Scatter form: input row p is read once and its codes and scales are
// written to output rows row_map[p*k + j], j < k (the inverse permutation),
// so the permuted operand is produced without an unpermuted copy; rows
// outside [0, rows*k) set the status flag and the warp writes nothing.
constexpr int kQuantScatterMaxK = 16;  // lanes that hold the k output rows

template <bool SCATTER>
__global__ void __launch_bounds__(256, SCATTER ? 4 : 1) quant_act_kernel(
    const uint4* __restrict__ x, int64_t rows, int64_t cols, const int32_t* __restrict__ row_map,
    int k, uint2* __restrict__ q, float* __restrict__ s, bool ue8m0, int32_t* status) {
  const int64_t p = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (p >= rows) return;  // warp-uniform
  const int64_t vpr = cols / 8, groups = cols / 128;
  int64_t src = p;
  int mine = (int)p;  // scatter: lane j < k holds output row j of this input row
  if constexpr (SCATTER) {
    mine = lane < k ? row_map[p * k + lane] : 0;
    if (__any_sync(0xffffffffu, (unsigned)mine >= (unsigned)(rows * k))) {
      if (lane == 0) record_bad_index(status);
      return;
    }
  } else {
    src = row_map ? row_map[p] : p;
  }
  const uint4* xr = x + src * vpr;
  // four 256-column steps per pass: their loads are issued before any is used
  for (int64_t b0 = 0; b0 < vpr; b0 += 4 * 32) {
    uint4 ub[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t v = b0 + i * 32 + lane;
      ub[i] = v < vpr ? xr[v] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll 1
    for (int i = 0; i < 4; ++i) {
      const int64_t v0 = b0 + i * 32;
      if (v0 >= vpr) break;  // warp-uniform
      const int64_t v = v0 + lane;
      const bool on = v < vpr;  // a trailing single group leaves lanes 16-31 idle
      const uint4 u = ub[0];
      ub[0] = ub[1], ub[1] = ub[2], ub[2] = ub[3];  // constant indices: stays in registers
      const float f[8] = {bf16lo_to_f32(u.x), bf16hi_to_f32(u.x), bf16lo_to_f32(u.y), bf16hi_to_f32(u.y),
                          bf16lo_to_f32(u.z), bf16hi_to_f32(u.z), bf16lo_to_f32(u.w), bf16hi_to_f32(u.w)};
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const float sc = group_scale(amax, ue8m0);
      const uint2 code =
          make_uint2(e4m3x4(__fdiv_rn(f[0], sc), __fdiv_rn(f[1], sc), __fdiv_rn(f[2], sc), __fdiv_rn(f[3], sc)),
                     e4m3x4(__fdiv_rn(f[4], sc), __fdiv_rn(f[5], sc), __fdiv_rn(f[6], sc), __fdiv_rn(f[7], sc)));
      for (int j = 0; j < (SCATTER ? k : 1); ++j) {  // warp-uniform trip count
        const int64_t d = SCATTER ? __shfl_sync(0xffffffffu, mine, j) : mine;
        if (on) {
          q[d * vpr + v] = code;
          if ((lane & 15) == 0) s[d * groups + v / 16] = sc;
        }
      }
    }
  }
}

// The scatter form with the bulk-copy engine, for rows whose scales fill whole
// 16-byte units (cols % 512 == 0): each warp quantises its token's row as
// above into a shared buffer (the codes, then the row's scales), and lanes
// j < k each issue two bulk stores, the codes to row inv_perm[p*k + j] of q
// and the scales to the same row of s; before the buffer takes the next
// token the lanes wait until their stores have read it.
constexpr int kQBulkWarps = 4;

__global__ void __launch_bounds__(kQBulkWarps * 32) quant_act_scatter_bulk_kernel(
    const uint4* __restrict__ x, int64_t rows, int64_t cols, const int32_t* __restrict__ inv_perm,
    int k, unsigned char* __restrict__ q, float* __restrict__ s, bool ue8m0, int32_t* status) {
  extern __shared__ __align__(16) unsigned char qrows[];  // [kQBulkWarps][cols + groups * 4]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t vpr = cols / 8, groups = cols / 128;
  unsigned char* buf = qrows + (size_t)warp * (cols + groups * 4);
  const uint32_t sbuf = ptx::smem_addr(buf);
  const int64_t R = rows * k;
  for (int64_t p = (int64_t)blockIdx.x * kQBulkWarps + warp; p < rows;
       p += (int64_t)gridDim.x * kQBulkWarps) {
    const int mine = lane < k ? inv_perm[p * k + lane] : 0;
    if (__any_sync(0xffffffffu, (unsigned)mine >= (unsigned)R)) {
      if (lane == 0) record_bad_index(status);
      continue;
    }
    ptx::bulk_wait_read0();  // this lane's stores of the previous row have read the buffer
    __syncwarp();
    const uint4* xr = x + p * vpr;
    for (int64_t b0 = 0; b0 < vpr; b0 += 4 * 32) {
      uint4 ub[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t v = b0 + i * 32 + lane;
        ub[i] = v < vpr ? xr[v] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll 1
      for (int i = 0; i < 4; ++i) {
        const int64_t v0 = b0 + i * 32;
        if (v0 >= vpr) break;  // warp-uniform
        const int64_t v = v0 + lane;
        const bool on = v < vpr;
        const uint4 u = ub[0];
        ub[0] = ub[1], ub[1] = ub[2], ub[2] = ub[3];
        const float f[8] = {bf16lo_to_f32(u.x), bf16hi_to_f32(u.x), bf16lo_to_f32(u.y), bf16hi_to_f32(u.y),
                            bf16lo_to_f32(u.z), bf16hi_to_f32(u.z), bf16lo_to_f32(u.w), bf16hi_to_f32(u.w)};
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const float sc = group_scale(amax, ue8m0);
        if (on) {
          *reinterpret_cast<uint2*>(buf + v * 8) =
              make_uint2(e4m3x4(__fdiv_rn(f[0], sc), __fdiv_rn(f[1], sc), __fdiv_rn(f[2], sc), __fdiv_rn(f[3], sc)),
                         e4m3x4(__fdiv_rn(f[4], sc), __fdiv_rn(f[5], sc), __fdiv_rn(f[6], sc), __fdiv_rn(f[7], sc)));
          if ((lane & 15) == 0) *reinterpret_cast<float*>(buf + cols + (v / 16) * 4) = sc;
        }
      }
    }
    ptx::fence_proxy_async_smem();  // the generic-proxy writes -> visible to the bulk copies
    __syncwarp();
    if (lane < k) {
      ptx::bulk_store(q + (int64_t)mine * cols, sbuf, (uint32_t)cols);
      ptx::bulk_store(s + (int64_t)mine * groups, sbuf + (uint32_t)cols, (uint32_t)(groups * 4));
      ptx::bulk_commit();
    }
  }
  ptx::bulk_wait_all();  // every store has completed before the block's shared memory goes
}

// One block (256 threads) per 128 x 128 weight block.
__global__ void __launch_bounds__(256) quant_weight_kernel(const __nv_bfloat16* __restrict__ w,
                                                           int64_t rows, int64_t cols,
                                                           uint8_t* __restrict__ q,
                                                           float* __restrict__ s, bool ue8m0) {
  const int64_t RB = rows / 128, CB = cols / 128;
  const int64_t blk = blockIdx.x;
  const int64_t b = blk / (RB * CB), rb = (blk / CB) % RB, cb = blk % CB;
  const int64_t base = b * rows * cols + rb * 128 * cols + cb * 128;
  const uint16_t* wp = reinterpret_cast<const uint16_t*>(w);
  __shared__ float red[8];
  float amax = 0.0f;
  // thread t: row t / 2, columns (t % 2) * 64 .. +64
  const int r = threadIdx.x >> 1, c0 = (threadIdx.x & 1) * 64;
  const uint16_t* rowp = wp + base + (int64_t)r * cols + c0;
  float vals[64];
#pragma unroll
  for (int i = 0; i < 64; i += 8) {
    uint4 u = *reinterpret_cast<const uint4*>(rowp + i);
    vals[i + 0] = bf16lo_to_f32(u.x), vals[i + 1] = bf16hi_to_f32(u.x);
    vals[i + 2] = bf16lo_to_f32(u.y), vals[i + 3] = bf16hi_to_f32(u.y);
    vals[i + 4] = bf16lo_to_f32(u.z), vals[i + 5] = bf16hi_to_f32(u.z);
    vals[i + 6] = bf16lo_to_f32(u.w), vals[i + 7] = bf16hi_to_f32(u.w);
  }
#pragma unroll
  for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(vals[i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float sc = group_scale(amax, ue8m0);
  uint32_t* qp = reinterpret_cast<uint32_t*>(q + base + (int64_t)r * cols + c0);
#pragma unroll
  for (int i = 0; i < 64; i += 4)
    qp[i / 4] = e4m3x4(__fdiv_rn(vals[i], sc), __fdiv_rn(vals[i + 1], sc),
                       __fdiv_rn(vals[i + 2], sc), __fdiv_rn(vals[i + 3], sc));
  if (threadIdx.x == 0) s[blk] = sc;
}

cudaError_t launch_quant_act(const void* x, int64_t rows, int64_t cols, void* q, float* sc,
                             const int32_t* row_map, bool ue8m0, cudaStream_t s) {
  quant_act_kernel<false><<<(unsigned)ceil_div(rows, 8), 256, 0, s>>>(
      static_cast<const uint4*>(x), rows, cols, row_map, 1, static_cast<uint2*>(q), sc, ue8m0,
      nullptr);
  note_launch();
  return cudaGetLastError();
}

// x [rows, cols] quantised per row and 128-column group, each row's codes and
// scales written to the k permuted rows inv_perm[row*k + j].
cudaError_t launch_quant_act_scatter(const void* x, int64_t rows, int64_t cols,
                                     const int32_t* inv_perm, int k, void* q_perm, float* sc_perm,
                                     bool ue8m0, int32_t* status, cudaStream_t s) {
  if (k < 1 || k > kQuantScatterMaxK) return cudaErrorNotSupported;
  const size_t bulk_smem = (size_t)kQBulkWarps * (cols + cols / 128 * 4);
  if (cols % 512 == 0 && bulk_smem <= 64 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(quant_act_scatter_bulk_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bulk_smem);
    if (e != cudaSuccess) return e;
    int sms = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks = std::min<int64_t>(ceil_div(rows, kQBulkWarps), (int64_t)std::max(sms, 1) * 6);
    quant_act_scatter_bulk_kernel<<<(unsigned)std::max<int64_t>(blocks, 1), kQBulkWarps * 32, bulk_smem,
                                    s>>>(static_cast<const uint4*>(x), rows, cols, inv_perm, k,
                                         static_cast<unsigned char*>(q_perm), sc_perm, ue8m0, status);
  } else {
    quant_act_kernel<true><<<(unsigned)ceil_div(rows, 8), 256, 0, s>>>(
        static_cast<const uint4*>(x), rows, cols, inv_perm, k, static_cast<uint2*>(q_perm), sc_perm,
        ue8m0, status);
  }
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_quant_weight(const void* w, int64_t nb, int64_t rows, int64_t cols, void* q,
                                float* sc, bool ue8m0, cudaStream_t s) {
  const int64_t blocks = nb * (rows / 128) * (cols / 128);
  quant_weight_kernel<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), rows,
                                                       cols, static_cast<uint8_t*>(q), sc, ue8m0);
  note_launch();
  return cudaGetLastError();
}

// FP4 expert weights ("Experts backends", "FP8 and FP4 quantized experts":
// e2m1 codes packed two per byte with UE8M0 scales). One scale per row per
// 32 consecutive K elements (the OCP microscaling block): the smallest power
// of two >= amax / 6 (fp32 quotient), p clamped to [-127, 127], 1 for an
// all-zero block, stored as its biased exponent. Element 2i goes to the low
// nibble of byte i. The scale bytes are stored in the block-scaled GEMM's
// chunk layout: per 128 rows and 128 K one 512-byte chunk whose byte
// 16 r + 4 g + j is the scale of row 32 g + r for the K elements
// [32 j, 32 j + 32) of that chunk.

// e2m1 code of v (|v| <= 6 here): nearest of 0, 0.5, 1, 1.5, 2, 3, 4, 6, ties
// to the even code; larger magnitudes saturate to 6; the sign bit is kept.
__device__ __forceinline__ uint32_t e2m1_code(float v) {
  const float a = fabsf(v);
  uint32_t c;
  if (a <= 0.25f) c = 0;
  else if (a < 0.75f) c = 1;
  else if (a <= 1.25f) c = 2;
  else if (a < 1.75f) c = 3;
  else if (a <= 2.5f) c = 4;
  else if (a < 3.5f) c = 5;
  else if (a <= 5.0f) c = 6;
  else c = 7;
  return (signbit(v) ? 8u : 0u) | c;
}

// One thread per 32-element block: 64 bytes in, 16 bytes of codes and one
// scale byte out.
__global__ void __launch_bounds__(256) quant_weight_fp4_kernel(const uint4* __restrict__ w,
                                                               int64_t nblocks, int64_t cols,
                                                               uint4* __restrict__ q,
                                                               uint8_t* __restrict__ sc) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nblocks) return;
  const int64_t row = i / (cols / 32);  // over all nb matrices (rows % 128 == 0)
  const int b32 = (int)(i % (cols / 32));
  const int64_t chunk = (row >> 7) * (cols / 128) + (b32 >> 2);
  const int64_t sidx = chunk * 512 + 16 * (row & 31) + 4 * ((row >> 5) & 3) + (b32 & 3);
  float v[32];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 u = w[i * 4 + j];
    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      v[8 * j + 2 * t] = bf16lo_to_f32(uw[t]);
      v[8 * j + 2 * t + 1] = bf16hi_to_f32(uw[t]);
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
  float s = 1.0f;
  if (amax > 0.0f) {
    int e;
    const float m = frexpf(__fdiv_rn(amax, 6.0f), &e);
    s = ldexpf(1.0f, min(max(m == 0.5f ? e - 1 : e, -127), 127));
  }
  uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int j = 0; j < 32; ++j) out[j >> 3] |= e2m1_code(__fdiv_rn(v[j], s)) << (4 * (j & 7));
  q[i] = make_uint4(out[0], out[1], out[2], out[3]);
  sc[sidx] = (uint8_t)((__float_as_uint(s) >> 23) & 0xFFu);  // 2^-127 is the one code-0 (subnormal) scale
}

cudaError_t launch_quant_weight_fp4(const void* w, int64_t nb, int64_t rows, int64_t cols, void* q,
                                    uint8_t* sc, cudaStream_t s) {
  const int64_t nblocks = nb * rows * (cols / 32);
  quant_weight_fp4_kernel<<<(unsigned)ceil_div(nblocks, 256), 256, 0, s>>>(
      static_cast<const uint4*>(w), nblocks, cols, static_cast<uint4*>(q), sc);
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
