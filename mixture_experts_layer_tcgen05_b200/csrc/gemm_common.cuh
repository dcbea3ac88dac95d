// Pieces shared by the grouped GEMM kernels (bf16 and FP8): tile
// scheduling over the expert offsets, drain of in-flight TMA loads, and the
// host-side tensor-map encoding.
#pragma once

#include <cuda.h>

#include <algorithm>

#include "ptx.cuh"

namespace moe {
namespace gg {

constexpr int BM = 128;         // MMA M
constexpr int BK = 64;          // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int UK = 16;          // K per tcgen05.mma (16-bit inputs)
constexpr int kThreads = 192;
constexpr int kTileA = BM * BK * 2;  // 16 KB
constexpr int kMaxE = 1024;
constexpr int kSmemBudget = 200 * 1024;

struct Args {
  const int32_t* offsets;  // [E + 1]
  int E;
  int K;
  int ldc;         // output columns
  int NT;          // weight tiles per expert
  int b_rows;      // rows of B (weights) per expert
  int up_off;      // SwiGLU: row offset of the up half inside an expert
  int band;        // m-tiles per raster band (rows kernel)
  int M_total;     // rows of A (and C); stores never leave [0, M_total)
  const int32_t* a_rows;  // gather: source row of each routed row (nullptr: A is dense)
  const void* a_src;      // gather: source matrix [a_src_rows, K]
  int a_src_rows;
  float* tail_part;  // rows kernel: fp32 partial sums of a K-split last wave, or nullptr
  int ksplit;        // small-M kernel: K split into ksplit ranges, fp32 partials
  float* partial;    // [ksplit, M_total, pld] with pld = (SwiGLU ? 2 : 1) * ldc
  __nv_bfloat16* C;
  int32_t* status;
};

// ------------------------------------------------------------- scheduling
// tile_start[e] = sum_{e' < e} tiles(e'), tile_start[E] = total; soff[0..E]
// = offsets[0..E], a shared-memory copy every role decodes tiles from (no
// global-memory latency at a tile switch). Warp-wide.
template <int kRowsPerTile>
__device__ void build_tile_starts(const int32_t* offsets, int E, int NT, int32_t* tile_start,
                                  int32_t* soff) {
  const int lane = threadIdx.x & 31;
  for (int e = lane; e <= E; e += 32) soff[e] = offsets[e];
  int32_t carry = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    int e = e0 + lane;
    int32_t cnt = e < E ? max(offsets[e + 1] - offsets[e], 0) : 0;
    int32_t t = (int32_t)((cnt + kRowsPerTile - 1) / kRowsPerTile) * NT;
    int32_t incl = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int32_t v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (e < E) tile_start[e] = carry + incl - t;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) tile_start[E] = carry;
}

// Largest e with tile_start[e] <= tile (that expert is non-empty).
__device__ __forceinline__ int find_expert(const int32_t* tile_start, int E, int tile) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (tile_start[mid] <= tile) lo = mid;
    else hi = mid;
  }
  return lo;
}

// ------------------------------------------------------------------ utils
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 o;
    o.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    o.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    o.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    o.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = o;
  }
}

// Producer drain: wait for the last in-flight loads of the ring to land so no
// TMA write targets shared memory after the CTA has gone.
template <int STAGES>
__device__ void drain_loads(uint32_t full0, int64_t issued, int32_t* status) {
  for (int64_t i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i) {
    uint32_t bar = full0 + (uint32_t)(i % STAGES) * 8;
    ptx::mbar_wait(bar, (uint32_t)((i / STAGES) & 1), status, kSiteDrain);
  }
}

// ---------------------------------------------------------- row gather
// A-operand rows fetched by index instead of from a permuted copy: lane l of
// the producer warp loads tile rows 4l..4l+3 with one TMA tile::gather4
// (tensor map box one row high, 128-byte swizzle), 512 bytes at offset 512*l
// of the stage, so the 32 lanes fill the same 128-row layout a tile load
// leaves. Rows past M_total (or with an index out of range) get row index
// `src_rows`, outside the tensor, and are zero-filled.
__device__ __forceinline__ void gather4_tile_rows(const int32_t* row_map, int base, int M_total,
                                                  int src_rows, int lane, int (&out)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int r = base + 4 * lane + j;
    int t = src_rows;
    if (r >= 0 && r < M_total) {
      const int v = row_map[r];
      if ((unsigned)v < (unsigned)src_rows) t = v;
    }
    out[j] = t;
  }
}

}  // namespace gg

// ------------------------------------------------------------------ host
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline PFN_encodeTiled get_encode() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  }
  return fn;
}

// 2-D K-major operand [rows, K] with 128-byte swizzled boxes {64 (K), box_rows}.
inline bool make_tmap(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                      int64_t K, int64_t rows, int box_rows) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K * elem_bytes)};
  cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Packed 4-bit codes [rows, K] (two per byte, element 2i in the low nibble)
// loaded into the unpacked shared layout (16 codes per 16 bytes), 128 codes
// (one 128-byte swizzled row) by box_rows rows per box. Needs a 32-byte
// aligned base and K % 64 == 0.
inline bool make_tmap_fp4(CUtensorMap* m, const void* base, int64_t K, int64_t rows, int box_rows) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <typename KernelT>
inline cudaError_t set_smem(KernelT k, size_t bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace moe
