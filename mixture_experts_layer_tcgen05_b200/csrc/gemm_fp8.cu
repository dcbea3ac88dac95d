// Grouped GEMM with fine-grained FP8 operands on sm_100a tensor cores.
//
// "Fine-grained FP8" (HF Transformers docs), opening list: weights carry one
// fp32 scale per 128 x 128 block, activations one per (token, 128-channel
// group). With fp32 (not power-of-two) scales the product of the two scales
// cannot be folded into a block-scaled MMA, so each 128-wide K block is
// multiplied on the tensor cores into its own TMEM partial (tcgen05.mma
// kind::f8f6f4, e4m3 x e4m3 -> fp32) and promoted on CUDA cores:
//   acc[m, n] += P_kb[m, n] * a_scale[m, kb] * b_scale[n / 128, kb]
// The partials are double-buffered in TMEM so the tensor cores fill one while
// eight promotion warps drain the other.
//
// Warp roles (320 threads): warp 0 TMA producer, warp 1 TMEM allocator + MMA
// issuer, warps 2..9 promotion + epilogue. Warp w reads TMEM lane quarter
// w % 4; warps 2..5 take the first half of a row's columns, 6..9 the second.
// With the SwiGLU epilogue a thread holds matching gate and up columns, so
// silu(g) * u is formed in registers; the output can be re-quantised per
// (row, 128-column group) to e4m3 with scale amax/448 (the next GEMM's input).
#include <cuda_fp8.h>

#include <cstring>

#include "gemm_common.cuh"

namespace moe {
namespace gg8 {

constexpr int BM = 128;
constexpr int BK = 128;  // fp8 elements per stage = one 128-byte swizzle row = one scale block
constexpr int UK = 32;   // K per tcgen05.mma for 8-bit inputs
constexpr int BN = 256;
constexpr int kThreads = 320;
constexpr int kTileA = BM * BK;  // 16 KB
constexpr int kTileB = BN * BK;  // 32 KB
constexpr int kStage = kTileA + kTileB;
constexpr int kMaxE = 1024;
constexpr uint32_t kIdesc = ptx::make_idesc(BM, BN, 0, 0);  // e4m3 x e4m3 -> fp32
// The plain GEMM stages its bf16 output tile (128 x 256, 64 KB) in shared
// memory and writes it with tiled TMA stores, so the promotion warps go on
// to the next tile at once; that buffer takes the fourth ring stage. Each
// promotion warp owns 8 KB: its 32 rows x 128 columns as two boxes of 64
// columns in the 128-byte-swizzled layout (row r's 16-byte chunk c at
// r * 128 + ((c ^ (r % 8)) * 16)), which spreads the 32 rows a warp writes
// at once over all banks and is what the store's tensor map expects.
__host__ __device__ constexpr int stages_of(bool plain) { return plain ? 3 : 4; }
constexpr int kStgWarp = 32 * 128 * 2;  // bytes of one promotion warp's two boxes
__host__ __device__ constexpr int staging_of(bool plain) { return plain ? 8 * kStgWarp : 0; }
__host__ __device__ constexpr size_t smem_of(bool plain) {
  return 1024 + (size_t)stages_of(plain) * kStage + staging_of(plain) + 256 + 2 * (kMaxE + 1) * 4 +
         2 * 2 * BM * 4;
}

struct Args {
  const int32_t* offsets;
  int E, K, ldc, NT, b_rows, up_off, band, M_total;
  const int32_t* a_rows;  // gather: source row of each routed row (nullptr: A is dense)
  const void* a_src;      // gather: source matrix [a_src_rows, K] (e4m3)
  int a_src_rows;
  int kblocks;  // K / 128
  int b_nblk;   // 128-row blocks of B per expert
  void* C;      // bf16 [M_total, ldc], or e4m3 when c_scales != nullptr
  float* c_scales;
  const float* a_scales;  // [M_total, kblocks], or [a_src_rows, kblocks] with a gather
  const float* b_scales;  // [E, b_nblk, kblocks]
  int32_t* status;
};

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// ACT: gated activation of the epilogue (kActNone: plain GEMM).
template <int ACT, bool GATHER>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_rows_fp8_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmC, Args args) {
  constexpr bool SWIGLU = ACT != kActNone;
  constexpr int STAGES = stages_of(!SWIGLU);
  constexpr int kStaging = staging_of(!SWIGLU);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* staging = smem + STAGES * kStage;  // plain: [BM rows][BN cols] bf16
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + kStaging);
  // bars: full[STAGES], empty[STAGES], pfull[2], pempty[2], drain, redbar[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 7);
  int32_t* tile_start = reinterpret_cast<int32_t*>(staging + kStaging + 256);
  int32_t* soff = tile_start + kMaxE + 1;  // [E + 1] expert offsets, shared copy
  float* red = reinterpret_cast<float*>(soff + kMaxE + 1);  // [2 tiles][2 halves][BM]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t full0 = ptx::smem_addr(bars), empty0 = full0 + STAGES * 8;
  const uint32_t pfull0 = empty0 + STAGES * 8, pempty0 = pfull0 + 16, drain = pempty0 + 16;
  const uint32_t redbar0 = drain + 8;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full0 + s * 8, 1);
      ptx::mbar_init(empty0 + s * 8, 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(pfull0 + a * 8, 1);
      ptx::mbar_init(pempty0 + a * 8, 8);
    }
    ptx::mbar_init(drain, 1);
    ptx::mbar_init(redbar0, 256);
    ptx::mbar_init(redbar0 + 8, 256);
    ptx::fence_barrier_init();
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
    if (!SWIGLU) ptx::tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_slot), 512);
    ptx::tmem_relinquish();
  }
  if (warp == 2) gg::build_tile_starts<BM>(args.offsets, args.E, args.NT, tile_start, soff);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_start[args.E];
  const int nkb = args.kblocks;

  auto decode = [&](int tile, int& e, int& m, int& n) {
    e = gg::find_expert(tile_start, args.E, tile);
    const int local = tile - tile_start[e];
    const int cnt = soff[e + 1] - soff[e];
    const int mt = (cnt + BM - 1) / BM;
    const int bsz = args.band * args.NT;
    const int b = local / bsz;
    const int rows = min(args.band, mt - b * args.band);
    const int l2 = local - b * bsz;
    n = l2 / rows;
    m = b * args.band + l2 % rows;
  };

  if (warp == 0) {
    if (GATHER) {
      // all 32 lanes gather A rows (4 each); lane 0 also owns the barriers and the B loads
      int64_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, m, n;
        decode(tile, e, m, n);
        int src_row[4];
        gg::gather4_tile_rows(args.a_rows, soff[e] + m * BM, args.M_total, args.a_src_rows,
                             lane, src_row);
        int rb0, rb1;
        if (SWIGLU) {
          rb0 = e * args.b_rows + n * 128;
          rb1 = rb0 + args.up_off;
        } else {
          rb0 = e * args.b_rows + n * BN;
          rb1 = rb0 + 128;
        }
        for (int kb = 0; kb < nkb; ++kb, ++issued) {
          const int s = (int)(issued % STAGES);
          const uint32_t ph = (uint32_t)((issued / STAGES) & 1);
          int got = 1;
          if (lane == 0) got = ptx::mbar_wait(empty0 + s * 8, ph ^ 1, args.status, kSiteProducerEmpty);
          if (!__shfl_sync(0xffffffffu, got, 0)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + s * kStage, sb = sa + kTileA;
          if (lane == 0) {
            ptx::mbar_arrive_expect_tx(full0 + s * 8, kStage);
            ptx::tma_load_2d(sb, &tmB, kb * BK, rb0, full0 + s * 8);
            ptx::tma_load_2d(sb + 128 * 128, &tmB, kb * BK, rb1, full0 + s * 8);
          }
          __syncwarp();
          ptx::tma_gather4(sa + lane * 512, &tmA, kb * BK, src_row[0], src_row[1], src_row[2],
                           src_row[3], full0 + s * 8);
        }
      }
      __syncwarp();
      if (lane == 0) gg::drain_loads<STAGES>(full0, issued, args.status);
    } else if (lane == 0) {
      int64_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, m, n;
        decode(tile, e, m, n);
        const int row_a = soff[e] + m * BM;
        int rb0, rb1;
        if (SWIGLU) {
          rb0 = e * args.b_rows + n * 128;
          rb1 = rb0 + args.up_off;
        } else {
          rb0 = e * args.b_rows + n * BN;
          rb1 = rb0 + 128;
        }
        for (int kb = 0; kb < nkb; ++kb, ++issued) {
          const int s = (int)(issued % STAGES);
          const uint32_t ph = (uint32_t)((issued / STAGES) & 1);
          if (!ptx::mbar_wait(empty0 + s * 8, ph ^ 1, args.status, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + s * kStage, sb = sa + kTileA;
          ptx::mbar_arrive_expect_tx(full0 + s * 8, kStage);
          ptx::tma_load_2d(sa, &tmA, kb * BK, row_a, full0 + s * 8);
          ptx::tma_load_2d(sb, &tmB, kb * BK, rb0, full0 + s * 8);
          ptx::tma_load_2d(sb + 128 * 128, &tmB, kb * BK, rb1, full0 + s * 8);
        }
      }
      gg::drain_loads<STAGES>(full0, issued, args.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int64_t consumed = 0;  // stages, also the partial-buffer sequence
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        for (int kb = 0; kb < nkb; ++kb, ++consumed) {
          const int s = (int)(consumed % STAGES);
          const uint32_t ph = (uint32_t)((consumed / STAGES) & 1);
          const int pb = (int)(consumed & 1);
          const uint32_t pph = (uint32_t)((consumed >> 1) & 1);
          if (!ptx::mbar_wait(pempty0 + pb * 8, pph ^ 1, args.status, kSiteMmaAccEmpty) ||
              !ptx::mbar_wait(full0 + s * 8, ph, args.status, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa = sbase + s * kStage, sb = sa + kTileA;
          const uint64_t da = ptx::sw128_kmajor_desc(sa), db = ptx::sw128_kmajor_desc(sb);
          const uint32_t d = tmem_base + pb * 256;
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk)
            ptx::mma_f8(d, da + (uint64_t)(kk * UK / 16), db + (uint64_t)(kk * UK / 16), kIdesc,
                        kk != 0);
          ptx::mma_commit(empty0 + s * 8);
          ptx::mma_commit(pfull0 + pb * 8);
        }
      }
      ptx::mma_commit(drain);
      ptx::mbar_wait(drain, 0, args.status, kSiteDrain);
    }
  } else {
    const int half = (warp - 2) >> 2;
    const int q = warp & 3;
    const int rl = q * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
    int64_t seq = 0;
    int tile_iter = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tile_iter) {
      const int tile_par = tile_iter & 1;
      int e, m, n;
      decode(tile, e, m, n);
      const int row = soff[e] + m * BM + rl;
      const bool valid = row >= 0 && row < soff[e + 1] && row < args.M_total;
      const int row_c = min(max(row, 0), args.M_total - 1);
      int srow = row_c;
      if (GATHER) {
        srow = args.a_rows[row_c];
        if ((unsigned)srow >= (unsigned)args.a_src_rows) srow = 0;  // such rows are not stored
      }
      const float* sa_p = args.a_scales + (int64_t)srow * nkb;
      // B scale rows (128-row blocks of this expert's B) for this thread's columns
      int nb0, nb1;
      if (SWIGLU) {
        nb0 = n;                                // gate block
        nb1 = (args.up_off >> 7) + n;           // up block
      } else {
        nb0 = nb1 = n * 2 + half;
      }
      const float* sb0 = args.b_scales + ((int64_t)e * args.b_nblk + nb0) * nkb;
      const float* sb1 = args.b_scales + ((int64_t)e * args.b_nblk + nb1) * nkb;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
      bool ok = true;
      // plain GEMM: scales are read two k-blocks ahead of their use (measured
      // faster there; with SwiGLU the extra registers cost more than they save)
      // scales of k-block kb + 1 loaded while kb is promoted (rotated scalars)
      float a_n = sa_p[0], b0_n = sb0[0], b1_n = sb1[0];
      for (int kb = 0; kb < nkb; ++kb, ++seq) {
        const float s0 = a_n * b0_n, s1 = SWIGLU ? a_n * b1_n : s0;
        if (kb + 1 < nkb) {
          a_n = sa_p[kb + 1], b0_n = sb0[kb + 1];
          if (SWIGLU) b1_n = sb1[kb + 1];
        }
        const int pb = (int)(seq & 1);
        const uint32_t pph = (uint32_t)((seq >> 1) & 1);
        if (!ptx::mbar_wait(pfull0 + pb * 8, pph, args.status, kSiteEpiAccFull)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t pbase = lane_addr + pb * 256;
        if (SWIGLU) {
          // gate cols [half*64, +64) -> acc[0..64), up cols [128 + half*64, +64) -> acc[64..128)
#pragma unroll
          for (int c = 0; c < 64; c += 16) {
            uint32_t g[16], u[16];
            ptx::tmem_ld16(pbase + half * 64 + c, g);
            ptx::tmem_ld16(pbase + 128 + half * 64 + c, u);
            ptx::tmem_wait_ld();
            const float2 s0p = make_float2(s0, s0), s1p = make_float2(s1, s1);
#pragma unroll
            for (int i = 0; i < 16; i += 2) {  // paired FMAs: two IEEE fmas per instruction
              float2 a = __ffma2_rn(make_float2(__uint_as_float(g[i]), __uint_as_float(g[i + 1])), s0p,
                                    make_float2(acc[c + i], acc[c + i + 1]));
              acc[c + i] = a.x, acc[c + i + 1] = a.y;
              float2 b = __ffma2_rn(make_float2(__uint_as_float(u[i]), __uint_as_float(u[i + 1])), s1p,
                                    make_float2(acc[64 + c + i], acc[65 + c + i]));
              acc[64 + c + i] = b.x, acc[65 + c + i] = b.y;
            }
          }
        } else {
          const float2 s0p = make_float2(s0, s0);
#pragma unroll
          for (int c = 0; c < 128; c += 32) {
            uint32_t v0[16], v1[16];
            ptx::tmem_ld16(pbase + half * 128 + c, v0);
            ptx::tmem_ld16(pbase + half * 128 + c + 16, v1);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; i += 2) {  // paired FMAs: two IEEE fmas per instruction
              float2 a = __ffma2_rn(make_float2(__uint_as_float(v0[i]), __uint_as_float(v0[i + 1])), s0p,
                                    make_float2(acc[c + i], acc[c + i + 1]));
              acc[c + i] = a.x, acc[c + i + 1] = a.y;
              float2 b = __ffma2_rn(make_float2(__uint_as_float(v1[i]), __uint_as_float(v1[i + 1])), s0p,
                                    make_float2(acc[c + 16 + i], acc[c + 17 + i]));
              acc[c + 16 + i] = b.x, acc[c + 17 + i] = b.y;
            }
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(pempty0 + pb * 8);
      }
      if (!ok) break;
      if (SWIGLU) {
        float h[64];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          h[i] = gated<ACT>(acc[i], acc[64 + i]);
          amax = fmaxf(amax, fabsf(h[i]));
        }
        if (args.c_scales) {
          // exchange the two halves' row maxima (all 256 epilogue threads arrive)
          float* rb = red + tile_par * 2 * BM;
          rb[half * BM + rl] = amax;
          ptx::mbar_arrive(redbar0 + tile_par * 8);
          if (!ptx::mbar_wait(redbar0 + tile_par * 8, (uint32_t)((tile_iter >> 1) & 1), args.status,
                              kSiteEpiAccFull))
            break;
          amax = fmaxf(rb[rl], rb[BM + rl]);
          const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
          // one IEEE reciprocal per group, then products: h * (1/s) differs from
          // h / s by at most one fp32 ulp, which moves an e4m3 code only at a
          // rounding midpoint
          const float inv = __frcp_rn(sc);
          if (valid) {
            uint8_t* dst = static_cast<uint8_t*>(args.C) + (int64_t)row * args.ldc + n * 128 + half * 64;
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 o;
              o.x = e4m3x4(h[16 * v + 0] * inv, h[16 * v + 1] * inv,
                           h[16 * v + 2] * inv, h[16 * v + 3] * inv);
              o.y = e4m3x4(h[16 * v + 4] * inv, h[16 * v + 5] * inv,
                           h[16 * v + 6] * inv, h[16 * v + 7] * inv);
              o.z = e4m3x4(h[16 * v + 8] * inv, h[16 * v + 9] * inv,
                           h[16 * v + 10] * inv, h[16 * v + 11] * inv);
              o.w = e4m3x4(h[16 * v + 12] * inv, h[16 * v + 13] * inv,
                           h[16 * v + 14] * inv, h[16 * v + 15] * inv);
              d4[v] = o;
            }
            if (half == 0) args.c_scales[(int64_t)row * (args.ldc / 128) + n] = sc;
          }
        } else if (valid) {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(args.C) + (int64_t)row * args.ldc + n * 128 + half * 64;
          uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            d4[v] = make_uint4(pack_bf16x2(h[8 * v], h[8 * v + 1]), pack_bf16x2(h[8 * v + 2], h[8 * v + 3]),
                               pack_bf16x2(h[8 * v + 4], h[8 * v + 5]), pack_bf16x2(h[8 * v + 6], h[8 * v + 7]));
        }
      } else {
        // this warp's 32 rows x 128 columns: two swizzled 64-column boxes in its
        // staging region, then two tiled TMA stores issued by lane 0 when all 32
        // rows belong to the expert; a row group that runs past the expert's
        // rows stores its valid rows directly instead (a box store would
        // overwrite the first rows of the next expert's output)
        unsigned char* region = staging + (size_t)(warp - 2) * kStgWarp;
        if (tile_iter > 0) {  // the previous tile's stores have read the region
          if (lane == 0) ptx::bulk_wait_read0();
          __syncwarp();
        }
        const int g0 = soff[e] + m * BM + q * 32;
        const int nvalid = min(32, min(soff[e + 1], args.M_total) - g0);
        if (nvalid == 32) {
#pragma unroll
          for (int b = 0; b < 2; ++b)
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float* a8 = acc + b * 64 + c * 8;
              *reinterpret_cast<uint4*>(region + b * 4096 + lane * 128 + ((c ^ (lane & 7)) * 16)) =
                  make_uint4(pack_bf16x2(a8[0], a8[1]), pack_bf16x2(a8[2], a8[3]),
                             pack_bf16x2(a8[4], a8[5]), pack_bf16x2(a8[6], a8[7]));
            }
          ptx::fence_proxy_async_smem();  // the generic-proxy writes -> visible to the TMA store
          __syncwarp();
          if (lane == 0) {
            const uint32_t src = ptx::smem_addr(region);
            ptx::tma_store_2d(&tmC, src, n * BN + half * 128, g0);
            ptx::tma_store_2d(&tmC, src + 4096, n * BN + half * 128 + 64, g0);
            ptx::bulk_commit();
          }
        } else if (valid) {
          uint4* d4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.C) + (int64_t)row * args.ldc +
                                               n * BN + half * 128);
#pragma unroll
          for (int v = 0; v < 16; ++v)
            d4[v] = make_uint4(pack_bf16x2(acc[8 * v], acc[8 * v + 1]), pack_bf16x2(acc[8 * v + 2], acc[8 * v + 3]),
                               pack_bf16x2(acc[8 * v + 4], acc[8 * v + 5]), pack_bf16x2(acc[8 * v + 6], acc[8 * v + 7]));
        }
      }
    }
  }
  if (!SWIGLU && warp >= 2) ptx::bulk_wait_all();  // every output copy has landed
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace gg8

// A_rows != nullptr: routed row r of A (and of a_scales) is row A_rows[r] of
// A [A_src_rows, K] (and of a_scales [A_src_rows, K/128]).
cudaError_t launch_grouped_gemm_fp8(const void* A, const int32_t* A_rows, int A_src_rows,
                                    const float* a_scales, const void* B, const float* b_scales,
                                    const int32_t* offsets, int M_total, int E, int N, int K,
                                    int act, void* Cout, float* c_scales,
                                    int /*max_rows_per_expert*/, int32_t* status, cudaStream_t s,
                                    const char** why) {
  const bool swiglu = act != kActNone;
  const int b_rows = swiglu ? 2 * N : N;
  if (!swiglu && N % 256 != 0) {
    *why = "FP8 GEMM without SwiGLU needs N % 256 == 0";
    return cudaErrorInvalidValue;
  }
  CUtensorMap tmA, tmB, tmC;
  std::memset(&tmC, 0, sizeof(tmC));
  // a gathered A is read by tile::gather4 from a map whose box is one row high;
  // the plain GEMM's bf16 output is written in 64-column x 32-row swizzled boxes
  if (!make_tmap(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, A_rows ? A_src_rows : M_total,
                 A_rows ? 1 : 128) ||
      !make_tmap(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, (int64_t)E * b_rows, 128) ||
      (!swiglu && !make_tmap(&tmC, Cout, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M_total, 32))) {
    *why = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  gg8::Args a;
  a.offsets = offsets;
  a.E = E;
  a.K = K;
  a.ldc = N;
  a.NT = swiglu ? N / 128 : N / 256;
  a.b_rows = b_rows;
  a.up_off = swiglu ? N : 0;
  a.band = 8;
  a.M_total = M_total;
  a.a_rows = A_rows;
  a.a_src = A;
  a.a_src_rows = A_src_rows;
  a.kblocks = K / 128;
  a.b_nblk = b_rows / 128;
  a.C = Cout;
  a.c_scales = c_scales;
  a.a_scales = a_scales;
  a.b_scales = b_scales;
  a.status = status;
  const int64_t tiles_ub = ((int64_t)M_total / gg8::BM + (M_total < E ? M_total : E)) * a.NT;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(num_sms(), tiles_ub));
#define MOE_FP8(SW, G)                                                                    \
  do {                                                                                    \
    constexpr size_t smem = gg8::smem_of(SW == kActNone);                                 \
    cudaError_t e = set_smem(gg8::gemm_rows_fp8_kernel<SW, G>, smem);                     \
    if (e != cudaSuccess) return e;                                                       \
    gg8::gemm_rows_fp8_kernel<SW, G><<<grid, gg8::kThreads, smem, s>>>(tmA, tmB, tmC, a); \
  } while (0)
#define MOE_FP8_ACT(ACTV)           \
  do {                              \
    if (A_rows) MOE_FP8(ACTV, true); \
    else MOE_FP8(ACTV, false);      \
  } while (0)
  if (act == kActSilu) MOE_FP8_ACT(kActSilu);
  else if (act == kActGelu) MOE_FP8_ACT(kActGelu);
  else if (act == kActRelu) MOE_FP8_ACT(kActRelu);
  else MOE_FP8_ACT(kActNone);
#undef MOE_FP8_ACT
#undef MOE_FP8
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
