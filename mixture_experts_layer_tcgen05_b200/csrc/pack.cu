// One-time weight packing: logical expert weights -> the K-major layout the
// grouped GEMMs read.
//
// "Experts backends" (HF Transformers docs), backend table, grouped_mm row:
// each expert's gate/up projection maps H -> I and its down projection maps
// I -> H, stored logically as Wg, Wu [E, H, I] and Wd [E, I, H]. The GEMMs
// take every B operand as a row-major [rows, K] matrix (K contiguous), so
//   w13[e] rows [0, I)  = Wg[e]^T     ([I, H], K = H)
//   w13[e] rows [I, 2I) = Wu[e]^T
//   w2[e]               = Wd[e]^T     ([H, I], K = I)
// Each of the three is a batch of bf16 transposes.
#include "common.cuh"

namespace moe {

// dst[b][c][r] = src[b][r][c] for r < R, c < C (both multiples of 64).
// A 64 x 64 tile per block: 256 threads load it as 32-bit pairs of adjacent
// columns (coalesced rows of 128 bytes), and store the transposed tile as
// pairs of adjacent source rows, again 128 contiguous bytes per row.
constexpr int kPackTile = 64;

__global__ void __launch_bounds__(256) transpose_bf16_kernel(const uint16_t* __restrict__ src,
                                                             int64_t src_batch, int R, int C,
                                                             uint16_t* __restrict__ dst,
                                                             int64_t dst_batch) {
  __shared__ uint16_t tile[kPackTile][kPackTile + 2];  // +2: rows start on different banks
  const int64_t b = blockIdx.z;
  const int r0 = blockIdx.y * kPackTile, c0 = blockIdx.x * kPackTile;
  const uint16_t* s = src + b * src_batch;
  uint16_t* d = dst + b * dst_batch;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 column pairs x 8 rows
  for (int r = ty; r < kPackTile; r += 8) {
    const uint32_t v =
        *reinterpret_cast<const uint32_t*>(s + (int64_t)(r0 + r) * C + c0 + 2 * tx);
    tile[r][2 * tx] = (uint16_t)(v & 0xffffu);
    tile[r][2 * tx + 1] = (uint16_t)(v >> 16);
  }
  __syncthreads();
  // output row c (a source column), output columns r0 + 2*tx, +1 (two source rows)
  for (int c = ty; c < kPackTile; c += 8) {
    const uint32_t v = (uint32_t)tile[2 * tx][c] | ((uint32_t)tile[2 * tx + 1][c] << 16);
    *reinterpret_cast<uint32_t*>(d + (int64_t)(c0 + c) * R + r0 + 2 * tx) = v;
  }
}

static cudaError_t launch_transpose(const void* src, int64_t src_batch, int nb, int R, int C,
                                    void* dst, int64_t dst_batch, cudaStream_t s) {
  dim3 grid((unsigned)(C / kPackTile), (unsigned)(R / kPackTile), (unsigned)nb);
  transpose_bf16_kernel<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(src), src_batch, R, C,
                                             static_cast<uint16_t*>(dst), dst_batch);
  note_launch();
  return cudaGetLastError();
}

// Packs Wg, Wu [E, H, I] into w13 [E, 2I, H] and Wd [E, I, H] into w2 [E, H, I].
// H and I are multiples of 64; E <= 65535 (the grid's z extent).
cudaError_t launch_pack_weights(const void* wg, const void* wu, const void* wd, int E, int H,
                                int I, void* w13, void* w2, cudaStream_t s) {
  const int64_t HI = (int64_t)H * I;
  uint16_t* w13p = static_cast<uint16_t*>(w13);
  cudaError_t e = launch_transpose(wg, HI, E, H, I, w13p, 2 * HI, s);
  if (e == cudaSuccess) e = launch_transpose(wu, HI, E, H, I, w13p + HI, 2 * HI, s);
  if (e == cudaSuccess) e = launch_transpose(wd, HI, E, I, H, w2, HI, s);
  return e;
}

}  // namespace moe
