// Grouped GEMM with FP8 operands and power-of-two (UE8M0) block scales on the
// sm_100a block-scaled tensor-core path.
//
// "Experts backends" (HF Transformers docs), "FP8 and FP4 quantized experts"
// and "UE8M0 scale format": with scales stored as 8-bit exponents
// (float8_e8m0fnu) Blackwell's block-scaled MMA applies them itself, so
// nothing is promoted on CUDA cores: tcgen05.mma kind::mxf8f6f4.block_scale
// multiplies e4m3 x e4m3 with one E8M0 scale per row (of A) and per column
// (of B) per 32-wide K step, accumulating in fp32 across the whole K in TMEM.
// The layer's scales cover 128-wide K blocks (and 128-row weight blocks), so
// each 128-K stage repeats a row's scale over its four K steps.
//
// Scale factors reach TMEM by tcgen05.cp from a 512-byte shared chunk per
// 128 rows: the 16 bytes at offset 16*r hold, for rows r, r+32, r+64, r+96
// (in that order, 4 bytes each), the scales of the stage's four K steps; the
// copy (32 lanes x 128 bits, replicated to the four lane quarters) puts row
// group g in TMEM column g and K step j in byte j, which the MMA selects
// with its scale-factor ids.
//
// FP4 weights (BFP4): B holds packed e2m1 codes, two per byte, loaded by TMA
// into the 16-byte-aligned unpacked shared layout the f8f6f4 MMA reads (16
// codes per 16 bytes), so a stage still covers 128 K in 128-byte rows; A stays
// e4m3 (kind::mxf8f6f4 mixes the two formats). B's scales are e8m0 codes per
// (row, 32 K), stored already in the chunk layout above (one 512-byte chunk
// per 128 rows and 128 K), so each stage's two B chunks arrive by two bulk
// copies on the stage's barrier.
//
// Warp roles (320 threads): warp 0 TMA producer, all 32 lanes building the
// scale chunks; warp 1 TMEM allocator + MMA issuer; warps 2..9 epilogue.
// One accumulator (256 TMEM columns, the rest holds the scale-factor ring):
// the eight epilogue warps drain it into registers (warp w: lane quarter
// w % 4, column half (w - 2) / 4) and release it before the SwiGLU /
// re-quantisation math, so the next tile's MMAs overlap that work.
#include <cuda_fp8.h>

#include "gemm_common.cuh"

namespace moe {
namespace ggmx {

constexpr int BM = 128;
constexpr int BK = 128;  // fp8 elements per stage = one 128-byte swizzle row = one scale block
constexpr int UK = 32;   // K per block-scaled MMA (8-bit inputs)
constexpr int BN = 256;
constexpr int kThreads = 320;
constexpr int kTileA = BM * BK;  // 16 KB
constexpr int kTileB = BN * BK;  // 32 KB
constexpr int kStage = kTileA + kTileB;
constexpr int STAGES = 4;
constexpr int kPre = 4;       // stages of scales the producer loads ahead
constexpr int kSfA = 512;        // scale chunk bytes for 128 rows of A
constexpr int kSfStage = 3 * kSfA;  // A chunk + two B chunks
constexpr int kMaxE = 1024;
constexpr int kSfCol0 = 256;     // TMEM columns of the scale-factor ring
constexpr int kSfColsPerStage = 16;
// The plain GEMM stages its bf16 output tile in shared memory (rows 16 bytes
// apart beyond their 512, so a warp's 16-byte stores spread over the banks)
// and writes it with asynchronous bulk copies: the epilogue warps are free
// to drain the next accumulator at once. That buffer takes the fourth stage.
constexpr int kStgRow = BN * 2 + 16;
__host__ __device__ constexpr int mx_stages(bool plain) { return plain ? 3 : STAGES; }
__host__ __device__ constexpr size_t mx_smem(bool plain) {
  return 1024 + (size_t)mx_stages(plain) * (kStage + kSfStage) + (plain ? (size_t)BM * kStgRow : 0) +
         256 + 2 * (kMaxE + 1) * 4 + 2 * 2 * BM * 4;
}

struct Args {
  const int32_t* offsets;
  int E, K, ldc, NT, b_rows, up_off, band, M_total;
  int kblocks;            // K / 128
  int b_nblk;             // 128-row blocks of B per expert
  void* C;                // bf16 [M_total, ldc], or e4m3 when c_scales != nullptr
  float* c_scales;        // power-of-two scales of C's 128-groups
  const float* a_scales;  // [M_total, kblocks], powers of two
  const float* b_scales;  // [E, b_nblk, kblocks], powers of two (e4m3 B)
  const uint8_t* b_sf8;   // e2m1 B: e8m0 chunks [E * b_rows / 128][K / 128][512 bytes]
  int32_t* status;
};

// E8M0 code of a power-of-two fp32 scale (2^-127 is the one subnormal one).
__device__ __forceinline__ uint32_t e8m0_code(float s) {
  const uint32_t b = __float_as_uint(s);
  const uint32_t ex = (b >> 23) & 0xFFu;
  return ex ? ex : 0u;
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// Smallest power of two >= amax / 448 (fp32 quotient), 1 for an all-zero group.
__device__ __forceinline__ float pow2_scale(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  int e;
  const float m = frexpf(__fdiv_rn(amax, 448.0f), &e);
  return ldexpf(1.0f, min(max(m == 0.5f ? e - 1 : e, -127), 127));
}

// Shared-memory descriptor of a scale chunk for tcgen05.cp: K-major, no
// swizzle, 8-row core matrices of 16-byte rows stacked every 128 bytes.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);  // start address
  d |= (uint64_t)(128u >> 4) << 16;         // leading byte offset (one core matrix along K)
  d |= (uint64_t)(128u >> 4) << 32;         // stride byte offset: next 8 rows
  d |= (uint64_t)1u << 46;                  // descriptor version (sm_100)
  return d;                                 // layout bits 61-63 = 0: no swizzle
}

__device__ __forceinline__ void sf_copy(uint32_t tmem, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem), "l"(desc) : "memory");
}

// Block-scaled instruction descriptor: e4m3 x (e4m3 or e2m1), fp32
// accumulate, E8M0 scales, scale-factor ids (the K step) for A and B.
constexpr uint32_t kFmtE4M3 = 0, kFmtE2M1 = 5;
__host__ __device__ constexpr uint32_t mx_idesc(int M, int N, uint32_t sf_id, uint32_t b_fmt,
                                               uint32_t a_fmt = 0) {
  return (sf_id << 4)                    // B scale-factor id
         | (a_fmt << 7) | (b_fmt << 10)   // A, B formats: E4M3 (0) or E2M1 (5)
         | ((uint32_t)(N >> 3) << 17)     // N / 8
         | (1u << 23)                     // scale format E8M0
         | ((uint32_t)(M >> 4) << 24)     // M / 16
         | (sf_id << 29);                 // A scale-factor id
}

__device__ __forceinline__ void mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// ACT: gated activation of the epilogue (kActNone: plain GEMM); BFP4: B is
// packed e2m1 with e8m0 scales per (row, 32 K).
template <int ACT, bool BFP4>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   Args args) {
  constexpr bool SWIGLU = ACT != kActNone;
  constexpr int STAGES = mx_stages(!SWIGLU);
  constexpr int kStaging = SWIGLU ? 0 : BM * kStgRow;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sf = smem + STAGES * kStage;  // [STAGES][A chunk, B chunk 0, B chunk 1]
  unsigned char* staging = sf + STAGES * kSfStage;  // plain: [BM rows][kStgRow bytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + kStaging);
  // bars: full[STAGES], empty[STAGES], accf, acce, drain, redbar[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 6);
  int32_t* tile_start = reinterpret_cast<int32_t*>(staging + kStaging + 256);
  int32_t* soff = tile_start + kMaxE + 1;  // [E + 1] expert offsets, shared copy
  float* red = reinterpret_cast<float*>(soff + kMaxE + 1);  // [2 tiles][2 halves][BM]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = ptx::smem_addr(smem), sfbase = ptx::smem_addr(sf);
  const uint32_t full0 = ptx::smem_addr(bars), empty0 = full0 + STAGES * 8;
  const uint32_t accf = empty0 + STAGES * 8, acce = accf + 8, drain = acce + 8;
  const uint32_t redbar0 = drain + 8;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full0 + s * 8, 1);
      ptx::mbar_init(empty0 + s * 8, 1);
    }
    ptx::mbar_init(accf, 1);
    ptx::mbar_init(acce, 8);
    ptx::mbar_init(drain, 1);
    ptx::mbar_init(redbar0, 256);
    ptx::mbar_init(redbar0 + 8, 256);
    ptx::fence_barrier_init();
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
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
    // all lanes: scale chunks (lane l writes the 16 bytes of rows l + 32g);
    // lane 0: barriers and TMA loads
    int64_t issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      int e, m, n;
      decode(tile, e, m, n);
      const int row0 = soff[e] + m * BM, row_end = soff[e + 1];
      int rb0, rb1, nb0, nb1;  // B rows of the two 128-row boxes and their scale blocks
      if (SWIGLU) {
        rb0 = e * args.b_rows + n * 128;
        rb1 = rb0 + args.up_off;
        nb0 = n;
        nb1 = (args.up_off >> 7) + n;
      } else {
        rb0 = e * args.b_rows + n * BN;
        rb1 = rb0 + 128;
        nb0 = 2 * n;
        nb1 = 2 * n + 1;
      }
      const float* sb0 = args.b_scales + ((int64_t)e * args.b_nblk + nb0) * nkb;
      const float* sb1 = args.b_scales + ((int64_t)e * args.b_nblk + nb1) * nkb;
      const float* sa[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int r = row0 + g * 32 + lane;
        sa[g] = r < row_end ? args.a_scales + (int64_t)r * nkb : nullptr;  // rows past the expert: scale 1
      }
      // e2m1 B: the stage's scale chunks of the two 128-row boxes (rows rb0, rb1)
      const unsigned char* sfc0 = BFP4 ? args.b_sf8 + (int64_t)(rb0 >> 7) * nkb * kSfA : nullptr;
      const unsigned char* sfc1 = BFP4 ? args.b_sf8 + (int64_t)(rb1 >> 7) * nkb * kSfA : nullptr;
      // scales of the next kPre stages, loaded ahead so that their latency
      // overlaps the wait for a free stage
      float pa[kPre][4], pb[kPre][2];
      auto fetch = [&](int kb, float (&a)[4], float (&b)[2]) {
        if (kb < nkb) {
#pragma unroll
          for (int g = 0; g < 4; ++g) a[g] = sa[g] ? __ldg(sa[g] + kb) : 1.0f;
          if constexpr (!BFP4) {
            b[0] = __ldg(sb0 + kb);
            b[1] = __ldg(sb1 + kb);
          }
        }
      };
#pragma unroll
      for (int i = 0; i < kPre; ++i) fetch(i, pa[i], pb[i]);
      for (int kb = 0; kb < nkb; ++kb, ++issued) {
        const int s = (int)(issued % STAGES);
        const uint32_t ph = (uint32_t)((issued / STAGES) & 1);
        float ca[4] = {pa[0][0], pa[0][1], pa[0][2], pa[0][3]};
        const float cb0 = pb[0][0], cb1 = pb[0][1];
#pragma unroll
        for (int i = 0; i + 1 < kPre; ++i) {
#pragma unroll
          for (int g = 0; g < 4; ++g) pa[i][g] = pa[i + 1][g];
          pb[i][0] = pb[i + 1][0];
          pb[i][1] = pb[i + 1][1];
        }
        fetch(kb + kPre, pa[kPre - 1], pb[kPre - 1]);
        int got = 1;
        if (lane == 0) got = ptx::mbar_wait(empty0 + s * 8, ph ^ 1, args.status, kSiteProducerEmpty);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        // scale chunks of this stage
        uint32_t w[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) w[g] = e8m0_code(ca[g]) * 0x01010101u;  // same for the four K steps
        unsigned char* sfs = sf + s * kSfStage;
        *reinterpret_cast<uint4*>(sfs + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        if constexpr (!BFP4) {  // e2m1 B: its chunks arrive by bulk copy below
          const uint32_t c0 = e8m0_code(cb0) * 0x01010101u, c1 = e8m0_code(cb1) * 0x01010101u;
          *reinterpret_cast<uint4*>(sfs + kSfA + lane * 16) = make_uint4(c0, c0, c0, c0);
          *reinterpret_cast<uint4*>(sfs + 2 * kSfA + lane * 16) = make_uint4(c1, c1, c1, c1);
        }
        ptx::fence_proxy_async_smem();  // generic-proxy writes -> visible to tcgen05.cp
        __syncwarp();
        if (lane == 0) {
          const uint32_t sa_ = sbase + s * kStage, sb_ = sa_ + kTileA;
          // packed e2m1: the transaction counts the bytes read (two codes per byte)
          // plus the two scale chunks
          ptx::mbar_arrive_expect_tx(full0 + s * 8, BFP4 ? kTileA + kTileB / 2 + 2 * kSfA : kStage);
          ptx::tma_load_2d(sa_, &tmA, kb * BK, row0, full0 + s * 8);
          ptx::tma_load_2d(sb_, &tmB, kb * BK, rb0, full0 + s * 8);
          ptx::tma_load_2d(sb_ + 128 * 128, &tmB, kb * BK, rb1, full0 + s * 8);
          if constexpr (BFP4) {
            const uint32_t sfd = sfbase + s * kSfStage;
            ptx::bulk_load(sfd + kSfA, sfc0 + (int64_t)kb * kSfA, kSfA, full0 + s * 8);
            ptx::bulk_load(sfd + 2 * kSfA, sfc1 + (int64_t)kb * kSfA, kSfA, full0 + s * 8);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) gg::drain_loads<STAGES>(full0, issued, args.status);
  } else if (warp == 1) {
    if (lane == 0) {
      int64_t consumed = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        // the single accumulator: wait until the epilogue has drained the previous tile
        if (!ptx::mbar_wait(acce, acc_ph ^ 1, args.status, kSiteMmaAccEmpty)) break;
        acc_ph ^= 1;
        ptx::tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++consumed) {
          const int s = (int)(consumed % STAGES);
          const uint32_t ph = (uint32_t)((consumed / STAGES) & 1);
          if (!ptx::mbar_wait(full0 + s * 8, ph, args.status, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sfcol = tmem_base + kSfCol0 + s * kSfColsPerStage;
          const uint32_t sfs = sfbase + s * kSfStage;
          sf_copy(sfcol, sf_desc(sfs));                // A: columns 0..3
          sf_copy(sfcol + 4, sf_desc(sfs + kSfA));     // B rows 0..127: columns 4..7
          sf_copy(sfcol + 8, sf_desc(sfs + 2 * kSfA)); // B rows 128..255: columns 8..11
          const uint32_t sa_ = sbase + s * kStage, sb_ = sa_ + kTileA;
          const uint64_t da = ptx::sw128_kmajor_desc(sa_), db = ptx::sw128_kmajor_desc(sb_);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk)
            mma_mx(tmem_base, da + (uint64_t)(kk * UK / 16), db + (uint64_t)(kk * UK / 16),
                   mx_idesc(BM, BN, (uint32_t)kk, BFP4 ? kFmtE2M1 : kFmtE4M3), sfcol, sfcol + 4,
                   (kb | kk) != 0);
          ptx::mma_commit(empty0 + s * 8);
        }
        if (!ok) break;
        ptx::mma_commit(accf);
      }
      ptx::mma_commit(drain);
      ptx::mbar_wait(drain, 0, args.status, kSiteDrain);
    }
  } else {
    const int half = (warp - 2) >> 2;
    const int q = warp & 3;
    const int rl = q * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
    uint32_t acc_ph = 0;
    int tile_iter = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tile_iter) {
      const int tile_par = tile_iter & 1;
      int e, m, n;
      decode(tile, e, m, n);
      const int row = soff[e] + m * BM + rl;
      const bool valid = row >= 0 && row < soff[e + 1] && row < args.M_total;
      if (!ptx::mbar_wait(accf, acc_ph, args.status, kSiteEpiAccFull)) break;
      acc_ph ^= 1;
      ptx::tc_fence_after();
      // drain this thread's 128 accumulator columns, then release the accumulator
      float acc[128];
      if (SWIGLU) {
        // gate cols [half*64, +64) -> acc[0..64), up cols [128 + half*64, +64) -> acc[64..128);
        // all four loads in flight before one wait
        uint32_t raw[4][32];
        ptx::tmem_ld32(lane_addr + half * 64, raw[0]);
        ptx::tmem_ld32(lane_addr + half * 64 + 32, raw[1]);
        ptx::tmem_ld32(lane_addr + 128 + half * 64, raw[2]);
        ptx::tmem_ld32(lane_addr + 128 + half * 64 + 32, raw[3]);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[32 * j + i] = __uint_as_float(raw[j][i]);
      } else {
        uint32_t raw[4][32];
#pragma unroll
        for (int j = 0; j < 4; ++j) ptx::tmem_ld32(lane_addr + half * 128 + 32 * j, raw[j]);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[32 * j + i] = __uint_as_float(raw[j][i]);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acce);
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
          const float sc = pow2_scale(amax);
          const float inv = __frcp_rn(sc);  // exact: sc is a power of two
          if (valid) {
            uint8_t* dst = static_cast<uint8_t*>(args.C) + (int64_t)row * args.ldc + n * 128 + half * 64;
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 o;
              o.x = e4m3x4(h[16 * v + 0] * inv, h[16 * v + 1] * inv, h[16 * v + 2] * inv, h[16 * v + 3] * inv);
              o.y = e4m3x4(h[16 * v + 4] * inv, h[16 * v + 5] * inv, h[16 * v + 6] * inv, h[16 * v + 7] * inv);
              o.z = e4m3x4(h[16 * v + 8] * inv, h[16 * v + 9] * inv, h[16 * v + 10] * inv, h[16 * v + 11] * inv);
              o.w = e4m3x4(h[16 * v + 12] * inv, h[16 * v + 13] * inv, h[16 * v + 14] * inv, h[16 * v + 15] * inv);
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
        // this thread's 128 columns: into the staging tile, then one asynchronous bulk
        // copy of those 256 bytes to C (rows of the expert only)
        unsigned char* srow = staging + (size_t)rl * kStgRow + half * 256;
        if (tile_iter > 0) ptx::bulk_wait_read0();  // the previous tile's copy has read it
#pragma unroll
        for (int v = 0; v < 16; ++v)
          *reinterpret_cast<uint4*>(srow + v * 16) =
              make_uint4(pack_bf16x2(acc[8 * v], acc[8 * v + 1]), pack_bf16x2(acc[8 * v + 2], acc[8 * v + 3]),
                         pack_bf16x2(acc[8 * v + 4], acc[8 * v + 5]), pack_bf16x2(acc[8 * v + 6], acc[8 * v + 7]));
        ptx::fence_proxy_async_smem();  // the generic-proxy writes -> visible to the bulk copy
        if (valid) {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(args.C) + (int64_t)row * args.ldc + n * BN + half * 128;
          ptx::bulk_store(dst, ptx::smem_addr(srow), 256);
        }
        ptx::bulk_commit();
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


// ==========================================================================
// small-M (swap-AB) block-scaled kernel: weights in the MMA's M slot
// ==========================================================================
// For decode-sized batches an expert has a few rows, so the tokens-in-M
// kernel would load (and multiply) 128-row token tiles for them. Here the
// expert's weight rows take the MMA's M = 128 and its tokens the N = BNT
// (16, 32 or 64) slot, as in the bf16 small-M kernel: A = weights (e4m3 or
// e2m1, with their scale chunks), B = token rows (e4m3, power-of-two scales
// per row and 128-K block). A tile is (expert, token tile, 128 output
// columns); for a gated epilogue a stage holds the gate and the up rows of
// those columns and each K step issues two MMAs. The accumulator is
// transposed (TMEM lane = output column, column = token), double-buffered.
// Output: bf16, or for a gated epilogue with c_scales e4m3 + power-of-two
// scales per (row, 128 columns), the 128 columns of a tile being exactly one
// group (the group maximum is exchanged between the four epilogue warps).
template <int ACT, bool BFP4, int BNT>
struct MxSwapCfg {
  static constexpr bool SWIGLU = ACT != kActNone;
  static constexpr int kNA = SWIGLU ? 2 : 1;          // weight boxes per stage
  static constexpr int kTileW = 128 * BK;             // 16 KB (e2m1: unpacked layout)
  static constexpr int kTileT = BNT * BK;             // token rows of a stage
  static constexpr int kStage = kNA * kTileW + kTileT;  // a multiple of 1024
  static constexpr int kSf = (kNA + 1) * kSfA;        // weight chunk(s) + token chunk
  static constexpr int STAGES = (200 * 1024) / (kStage + kSf) > 8 ? 8 : (200 * 1024) / (kStage + kSf);
  static constexpr int kAccCols = kNA * BNT;          // per accumulator buffer
  static constexpr int kSfCol = 256;                  // scale-factor ring after the accumulators
  static constexpr size_t kSmem = 1024 + (size_t)STAGES * (kStage + kSf) + 256 +
                                  2 * (kMaxE + 1) * 4 + 2 * 4 * BNT * 4;
  // transaction bytes of a stage: packed e2m1 counts two codes per byte
  static constexpr uint32_t kTx = kNA * (BFP4 ? kTileW / 2 + kSfA : kTileW) + kTileT;
};

template <int ACT, bool BFP4, int BNT>
__global__ void __launch_bounds__(192, 1)
    gemm_mx_swap_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmT,
                        Args args) {
  using C = MxSwapCfg<ACT, BFP4, BNT>;
  constexpr bool SWIGLU = C::SWIGLU;
  constexpr int STAGES = C::STAGES;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sf = smem + STAGES * C::kStage;  // [STAGES][weight chunk(s), token chunk]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sf + STAGES * C::kSf);
  // bars: full[STAGES], empty[STAGES], accf[2], acce[2], drain, redbar[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 7);
  int32_t* tile_start = reinterpret_cast<int32_t*>(sf + STAGES * C::kSf + 256);
  int32_t* soff = tile_start + kMaxE + 1;  // [E + 1] expert offsets, shared copy
  float* red = reinterpret_cast<float*>(soff + kMaxE + 1);  // [2 tiles][4 warps][BNT]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = ptx::smem_addr(smem), sfbase = ptx::smem_addr(sf);
  const uint32_t full0 = ptx::smem_addr(bars), empty0 = full0 + STAGES * 8;
  const uint32_t accf0 = empty0 + STAGES * 8, acce0 = accf0 + 16, drain = acce0 + 16;
  const uint32_t redbar0 = drain + 8;  // group-maximum exchange, by tile parity

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full0 + s * 8, 1);
      ptx::mbar_init(empty0 + s * 8, 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(accf0 + a * 8, 1);
      ptx::mbar_init(acce0 + a * 8, 4);
      ptx::mbar_init(redbar0 + a * 8, 128);
    }
    ptx::mbar_init(drain, 1);
    ptx::fence_barrier_init();
    ptx::tma_prefetch_desc(&tmW);
    ptx::tma_prefetch_desc(&tmT);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_slot), 512);
    ptx::tmem_relinquish();
  }
  if (warp == 2) gg::build_tile_starts<BNT>(args.offsets, args.E, args.NT, tile_start, soff);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_start[args.E];
  const int nkb = args.kblocks;

  // tile -> expert, token tile, 128-column output tile
  auto decode = [&](int tile, int& e, int& tt, int& n) {
    e = gg::find_expert(tile_start, args.E, tile);
    const int local = tile - tile_start[e];
    tt = local / args.NT;
    n = local % args.NT;
  };

  if (warp == 0) {
    // all lanes: scale chunks; lane 0: barriers and TMA loads
    int64_t issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      int e, tt, n;
      decode(tile, e, tt, n);
      const int row0 = soff[e] + tt * BNT, row_end = soff[e + 1];
      const int rw0 = e * args.b_rows + n * 128;              // gate (or only) weight rows
      const int rw1 = SWIGLU ? rw0 + args.up_off : rw0;      // up weight rows
      const float* sw0 = args.b_scales + ((int64_t)e * args.b_nblk + (n * 128 >> 7)) * nkb;
      const float* sw1 = SWIGLU ? args.b_scales + ((int64_t)e * args.b_nblk + ((args.up_off + n * 128) >> 7)) * nkb
                                : sw0;
      const unsigned char* swc0 = BFP4 ? args.b_sf8 + (int64_t)(rw0 >> 7) * nkb * kSfA : nullptr;
      const unsigned char* swc1 = BFP4 ? args.b_sf8 + (int64_t)(rw1 >> 7) * nkb * kSfA : nullptr;
      // token rows lane and lane + 32 of the tile (scale 1 past the expert)
      const int r0 = row0 + lane, r1 = row0 + 32 + lane;
      const float* st0 = r0 < row_end ? args.a_scales + (int64_t)r0 * nkb : nullptr;
      const float* st1 = (BNT > 32 && r1 < row_end) ? args.a_scales + (int64_t)r1 * nkb : nullptr;
      for (int kb = 0; kb < nkb; ++kb, ++issued) {
        const int s = (int)(issued % STAGES);
        const uint32_t ph = (uint32_t)((issued / STAGES) & 1);
        const float t0s = st0 ? __ldg(st0 + kb) : 1.0f;
        const float t1s = st1 ? __ldg(st1 + kb) : 1.0f;
        float w0s = 1.0f, w1s = 1.0f;
        if constexpr (!BFP4) {
          w0s = __ldg(sw0 + kb);
          w1s = __ldg(sw1 + kb);
        }
        int got = 1;
        if (lane == 0) got = ptx::mbar_wait(empty0 + s * 8, ph ^ 1, args.status, kSiteProducerEmpty);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        unsigned char* sfs = sf + s * C::kSf;  // [weight chunk(s)][token chunk]
        const uint32_t tc0 = e8m0_code(t0s) * 0x01010101u, tc1 = e8m0_code(t1s) * 0x01010101u;
        *reinterpret_cast<uint4*>(sfs + C::kNA * kSfA + lane * 16) =
            make_uint4(tc0, tc1, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
        if constexpr (!BFP4) {  // one block scale per 128 x 128 weight block: the same code everywhere
          const uint32_t c0 = e8m0_code(w0s) * 0x01010101u, c1 = e8m0_code(w1s) * 0x01010101u;
          *reinterpret_cast<uint4*>(sfs + lane * 16) = make_uint4(c0, c0, c0, c0);
          if (SWIGLU) *reinterpret_cast<uint4*>(sfs + kSfA + lane * 16) = make_uint4(c1, c1, c1, c1);
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const uint32_t sw = sbase + s * C::kStage, st = sw + C::kNA * C::kTileW;
          ptx::mbar_arrive_expect_tx(full0 + s * 8, C::kTx);
          ptx::tma_load_2d(sw, &tmW, kb * BK, rw0, full0 + s * 8);
          if (SWIGLU) ptx::tma_load_2d(sw + C::kTileW, &tmW, kb * BK, rw1, full0 + s * 8);
          ptx::tma_load_2d(st, &tmT, kb * BK, row0, full0 + s * 8);
          if constexpr (BFP4) {
            const uint32_t sfd = sfbase + s * C::kSf;
            ptx::bulk_load(sfd, swc0 + (int64_t)kb * kSfA, kSfA, full0 + s * 8);
            if (SWIGLU) ptx::bulk_load(sfd + kSfA, swc1 + (int64_t)kb * kSfA, kSfA, full0 + s * 8);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) gg::drain_loads<STAGES>(full0, issued, args.status);
  } else if (warp == 1) {
    if (lane == 0) {
      int64_t consumed = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      constexpr uint32_t kWFmt = BFP4 ? kFmtE2M1 : kFmtE4M3;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        if (!ptx::mbar_wait(acce0 + acc * 8, acc_ph ^ 1, args.status, kSiteMmaAccEmpty)) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem_base + acc * C::kAccCols;
        for (int kb = 0; kb < nkb; ++kb, ++consumed) {
          const int s = (int)(consumed % STAGES);
          const uint32_t ph = (uint32_t)((consumed / STAGES) & 1);
          if (!ptx::mbar_wait(full0 + s * 8, ph, args.status, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          // scale-factor ring: weight chunk(s) at +0 (+4), token chunk at +8
          const uint32_t sfcol = tmem_base + C::kSfCol + s * 16;
          const uint32_t sfs = sfbase + s * C::kSf;
          sf_copy(sfcol, sf_desc(sfs));
          if (SWIGLU) sf_copy(sfcol + 4, sf_desc(sfs + kSfA));
          sf_copy(sfcol + 8, sf_desc(sfs + C::kNA * kSfA));
          const uint32_t sw = sbase + s * C::kStage, st = sw + C::kNA * C::kTileW;
          const uint64_t dw = ptx::sw128_kmajor_desc(sw), dt = ptx::sw128_kmajor_desc(st);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            const uint64_t ko = (uint64_t)(kk * UK / 16);
            const uint32_t idesc = mx_idesc(128, BNT, (uint32_t)kk, kFmtE4M3, kWFmt);
            mma_mx(d, dw + ko, dt + ko, idesc, sfcol, sfcol + 8, (kb | kk) != 0);
            if (SWIGLU)
              mma_mx(d + BNT, dw + (uint64_t)(C::kTileW >> 4) + ko, dt + ko, idesc, sfcol + 4,
                     sfcol + 8, (kb | kk) != 0);
          }
          ptx::mma_commit(empty0 + s * 8);
        }
        if (!ok) break;
        ptx::mma_commit(accf0 + acc * 8);
        acc ^= 1;
        if (acc == 0) acc_ph ^= 1;
      }
      ptx::mma_commit(drain);
      ptx::mbar_wait(drain, 0, args.status, kSiteDrain);
    }
  } else {
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_ph = 0;
    int tile_iter = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tile_iter) {
      int e, tt, n;
      decode(tile, e, tt, n);
      const int row0 = soff[e] + tt * BNT;
      const int nrows = min(min(BNT, soff[e + 1] - row0), args.M_total - row0);
      const int col = n * 128 + q * 32 + lane;  // output column owned by this thread
      if (!ptx::mbar_wait(accf0 + acc * 8, acc_ph, args.status, kSiteEpiAccFull)) break;
      ptx::tc_fence_after();
      const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::kAccCols;
      float v[BNT];
#pragma unroll
      for (int c = 0; c < BNT; c += 16) {
        uint32_t g[16], u[16];
        ptx::tmem_ld16(t0 + c, g);
        if (SWIGLU) ptx::tmem_ld16(t0 + BNT + c, u);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          v[c + i] = SWIGLU ? gated<ACT>(__uint_as_float(g[i]), __uint_as_float(u[i]))
                            : __uint_as_float(g[i]);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acce0 + acc * 8);
      acc ^= 1;
      if (acc == 0) acc_ph ^= 1;
      if (SWIGLU && args.c_scales) {
        // e4m3 output: the 128 columns of this tile are one group of each row
        float* rb = red + (tile_iter & 1) * 4 * BNT;
#pragma unroll
        for (int t = 0; t < BNT; ++t) {
          float m = fabsf(v[t]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (lane == 0) rb[q * BNT + t] = m;
        }
        // all 128 epilogue threads arrive; a bounded wait, so that a failed
        // pipeline cannot leave some of them waiting here for good
        ptx::mbar_arrive(redbar0 + (tile_iter & 1) * 8);
        if (!ptx::mbar_wait(redbar0 + (tile_iter & 1) * 8, (uint32_t)((tile_iter >> 1) & 1),
                            args.status, kSiteEpiAccFull))
          break;
        uint8_t* cq = static_cast<uint8_t*>(args.C);
#pragma unroll
        for (int t = 0; t < BNT; ++t) {
          if (t < nrows) {
            const float amax = fmaxf(fmaxf(rb[t], rb[BNT + t]), fmaxf(rb[2 * BNT + t], rb[3 * BNT + t]));
            const float sc = pow2_scale(amax);
            const float inv = __frcp_rn(sc);  // exact: sc is a power of two
            const uint32_t code =
                __nv_cvt_float2_to_fp8x2(make_float2(v[t] * inv, 0.0f), __NV_SATFINITE, __NV_E4M3) & 0xFFu;
            cq[(int64_t)(row0 + t) * args.ldc + col] = (uint8_t)code;
            if (q == 0 && lane == 0) args.c_scales[(int64_t)(row0 + t) * (args.ldc / 128) + n] = sc;
          }
        }
      } else {
        __nv_bfloat16* cb = static_cast<__nv_bfloat16*>(args.C);
#pragma unroll
        for (int t = 0; t < BNT; ++t)
          if (t < nrows) cb[(int64_t)(row0 + t) * args.ldc + col] = __float2bfloat16_rn(v[t]);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace ggmx

// ==========================================================================
// host side
// ==========================================================================
// Block-scaled FP8 grouped GEMM with power-of-two scales (see
// launch_grouped_gemm_fp8 for the operands; scales are fp32 powers of two).
cudaError_t launch_grouped_gemm_mx(const void* A, const float* a_scales, const void* B,
                                   const float* b_scales, const uint8_t* b_sf8,
                                   const int32_t* offsets, int M_total, int E, int N, int K, int act,
                                   void* Cout, float* c_scales, int32_t* status, cudaStream_t s,
                                   const char** why) {
  const bool swiglu = act != kActNone;
  const bool fp4 = b_sf8 != nullptr;
  const int b_rows = swiglu ? 2 * N : N;
  if (!swiglu && N % 256 != 0) {
    *why = "the block-scaled plain GEMM needs N % 256 == 0";
    return cudaErrorInvalidValue;
  }
  if (fp4 && ((reinterpret_cast<uintptr_t>(B) & 31) || (reinterpret_cast<uintptr_t>(b_sf8) & 15))) {
    *why = "packed FP4 weights must be 32-byte aligned and their scale chunks 16-byte aligned";
    return cudaErrorInvalidValue;
  }
  CUtensorMap tmA, tmB;
  const bool okB = fp4 ? make_tmap_fp4(&tmB, B, K, (int64_t)E * b_rows, 128)
                       : make_tmap(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, (int64_t)E * b_rows, 128);
  if (!make_tmap(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M_total, 128) || !okB) {
    *why = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  ggmx::Args a;
  a.offsets = offsets;
  a.E = E;
  a.K = K;
  a.ldc = N;
  a.NT = swiglu ? N / 128 : N / 256;
  a.b_rows = b_rows;
  a.up_off = swiglu ? N : 0;
  a.band = 8;
  a.M_total = M_total;
  a.kblocks = K / 128;
  a.b_nblk = b_rows / 128;
  a.C = Cout;
  a.c_scales = c_scales;
  a.a_scales = a_scales;
  a.b_scales = b_scales;
  a.b_sf8 = b_sf8;
  a.status = status;
  const int64_t tiles_ub = ((int64_t)M_total / ggmx::BM + (M_total < E ? M_total : E)) * a.NT;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(num_sms(), tiles_ub));
#define MOE_MX(ACTV, F4)                                                                      \
  do {                                                                                        \
    constexpr size_t smem = ggmx::mx_smem(ACTV == kActNone);                                  \
    cudaError_t e = set_smem(ggmx::gemm_mx_kernel<ACTV, F4>, smem);                           \
    if (e != cudaSuccess) return e;                                                           \
    ggmx::gemm_mx_kernel<ACTV, F4><<<grid, ggmx::kThreads, smem, s>>>(tmA, tmB, a);           \
  } while (0)
#define MOE_MX_ACT(F4)                         \
  do {                                         \
    if (act == kActSilu) MOE_MX(kActSilu, F4); \
    else if (act == kActGelu) MOE_MX(kActGelu, F4); \
    else if (act == kActRelu) MOE_MX(kActRelu, F4); \
    else MOE_MX(kActNone, F4);                 \
  } while (0)
  if (fp4) MOE_MX_ACT(true);
  else MOE_MX_ACT(false);
#undef MOE_MX_ACT
#undef MOE_MX
  note_launch();
  return cudaGetLastError();
}


// Small-M form of the block-scaled GEMM (weights in M): A = token rows (e4m3,
// a_scales), B = weights (e4m3 with b_scales, or packed e2m1 with b_sf8
// chunks); BNT from max_rows (the most rows an expert can have).
cudaError_t launch_grouped_gemm_mx_swap(const void* A, const float* a_scales, const void* B,
                                        const float* b_scales, const uint8_t* b_sf8,
                                        const int32_t* offsets, int M_total, int E, int N, int K,
                                        int act, void* Cout, float* c_scales, int max_rows,
                                        int32_t* status, cudaStream_t s, const char** why) {
  const bool swiglu = act != kActNone;
  const bool fp4 = b_sf8 != nullptr;
  const int b_rows = swiglu ? 2 * N : N;
  if (fp4 && ((reinterpret_cast<uintptr_t>(B) & 31) || (reinterpret_cast<uintptr_t>(b_sf8) & 15))) {
    *why = "packed FP4 weights must be 32-byte aligned and their scale chunks 16-byte aligned";
    return cudaErrorInvalidValue;
  }
  const int bnt = max_rows <= 16 ? 16 : max_rows <= 32 ? 32 : 64;
  CUtensorMap tmW, tmT;
  const bool okW = fp4 ? make_tmap_fp4(&tmW, B, K, (int64_t)E * b_rows, 128)
                       : make_tmap(&tmW, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, (int64_t)E * b_rows, 128);
  if (!okW || !make_tmap(&tmT, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M_total, bnt)) {
    *why = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  ggmx::Args a;
  a.offsets = offsets;
  a.E = E;
  a.K = K;
  a.ldc = N;
  a.NT = N / 128;  // 128-column output tiles per expert
  a.b_rows = b_rows;
  a.up_off = swiglu ? N : 0;
  a.band = 0;
  a.M_total = M_total;
  a.kblocks = K / 128;
  a.b_nblk = b_rows / 128;
  a.C = Cout;
  a.c_scales = c_scales;
  a.a_scales = a_scales;
  a.b_scales = b_scales;
  a.b_sf8 = b_sf8;
  a.status = status;
  const int64_t tiles_ub = ((int64_t)M_total / bnt + (M_total < E ? M_total : E)) * a.NT;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(num_sms(), tiles_ub));
#define MOE_MXS(ACTV, F4, BN)                                                                      \
  do {                                                                                             \
    using Cfg = ggmx::MxSwapCfg<ACTV, F4, BN>;                                                     \
    cudaError_t e = set_smem(ggmx::gemm_mx_swap_kernel<ACTV, F4, BN>, Cfg::kSmem);                 \
    if (e != cudaSuccess) return e;                                                                \
    ggmx::gemm_mx_swap_kernel<ACTV, F4, BN><<<grid, 192, Cfg::kSmem, s>>>(tmW, tmT, a);            \
  } while (0)
#define MOE_MXS_BN(ACTV, F4)                          \
  do {                                                \
    if (bnt == 16) MOE_MXS(ACTV, F4, 16);             \
    else if (bnt == 32) MOE_MXS(ACTV, F4, 32);        \
    else MOE_MXS(ACTV, F4, 64);                       \
  } while (0)
#define MOE_MXS_ACT(F4)                               \
  do {                                                \
    if (act == kActSilu) MOE_MXS_BN(kActSilu, F4);    \
    else if (act == kActGelu) MOE_MXS_BN(kActGelu, F4); \
    else if (act == kActRelu) MOE_MXS_BN(kActRelu, F4); \
    else MOE_MXS_BN(kActNone, F4);                    \
  } while (0)
  if (fp4) MOE_MXS_ACT(true);
  else MOE_MXS_ACT(false);
#undef MOE_MXS_ACT
#undef MOE_MXS_BN
#undef MOE_MXS
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
