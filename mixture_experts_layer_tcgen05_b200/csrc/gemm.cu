// Grouped GEMMs of the expert MLP on sm_100a tensor cores (tcgen05 + TMEM,
// operands staged by TMA), with the SwiGLU epilogue fused.
//
// "Experts backends" (HF Transformers docs), backend table: grouped_mm /
// deepgemm rows (tokens sorted by expert, one grouped GEMM for all experts)
// and deepgemm_megamoe row (gated MLP: gate/up projection, SwiGLU, down
// projection). Rows of expert e are [offsets[e], offsets[e+1]) of A; the
// offsets are read on the device, so nothing here waits for the host.
//
// Two kernels:
//  * gemm_rows_kernel  -- tokens in the MMA M slot (M = 128 rows), weights in
//    N (256 or 128). Persistent: one CTA per SM walks a linear tile list
//    (expert, band of m-tiles, n-tile, m-tile) so the CTAs running together
//    share weight strips and activation bands through L2.
//  * gemm_swap_kernel  -- the small-M variant: weight rows in the MMA M slot
//    (M = 128) and the few token rows of an expert in N (16, 32 or 64).
//    "AWS improves MoE model performance on Amazon SageMaker AI", section
//    "Swap-AB advantage in MoE workloads": with few tokens per expert the
//    large expert dimension fills the MMA's fixed-size M.
//
// Both use the same warp roles (192 threads):
//   warp 0      TMA producer (one lane) through a STAGES-deep smem ring
//   warp 1      TMEM allocator + MMA issuer (one lane)
//   warps 2..5  epilogue: TMEM -> registers -> (SwiGLU) -> bf16 -> global
// with two accumulator buffers in TMEM so the epilogue of one tile overlaps
// the mainloop of the next. Every wait is bounded (see ptx::mbar_wait).
#include <cmath>

#include "gemm_common.cuh"

namespace moe {
namespace gg {

// ==========================================================================
// tokens-in-M kernel
// ==========================================================================
template <int ACT, int BN>
struct RowsCfg {
  static constexpr int kTileB = BN * BK * 2;
  static constexpr int kStage = kTileA + kTileB;
  static constexpr int STAGES = kSmemBudget / kStage;
  static constexpr int kAccCols = 256;  // column stride between the two accumulators
  static constexpr uint32_t kIdesc = ptx::make_idesc(BM, BN, 1, 1);  // bf16 x bf16 -> fp32
  static constexpr size_t kSmem = 1024 + (size_t)STAGES * kStage + 256 + 2 * (kMaxE + 1) * 4;
};

// ACT: gated activation of the epilogue (kActNone: plain GEMM).
// GATHER: A rows are copied by index (args.a_rows) from args.a_src by the
// whole producer warp instead of being loaded from a permuted copy by TMA.
template <int ACT, int BN, bool GATHER>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_rows_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, Args args) {
  using C = RowsCfg<ACT, BN>;
  constexpr bool SWIGLU = ACT != kActNone;
  constexpr int STAGES = C::STAGES;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStage);
  // bars: full[STAGES], empty[STAGES], accf[2], acce[2], drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  int32_t* tile_start = reinterpret_cast<int32_t*>(smem + STAGES * C::kStage + 256);
  int32_t* soff = tile_start + kMaxE + 1;  // [E + 1] expert offsets, shared copy

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t full0 = ptx::smem_addr(bars), empty0 = full0 + STAGES * 8;
  const uint32_t accf0 = empty0 + STAGES * 8, acce0 = accf0 + 16, drain = acce0 + 16;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full0 + s * 8, 1);
      ptx::mbar_init(empty0 + s * 8, 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(accf0 + a * 8, 1);
      ptx::mbar_init(acce0 + a * 8, 4);
    }
    ptx::mbar_init(drain, 1);
    ptx::fence_barrier_init();
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_slot), 512);
    ptx::tmem_relinquish();
  }
  if (warp == 2) build_tile_starts<BM>(args.offsets, args.E, args.NT, tile_start, soff);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_start[args.E];
  const int nkb = args.K / BK;
  // Plain GEMM: when the tiles leave a last wave at most half full, each of
  // its tiles runs as two units over the two halves of K, so that wave ends in
  // about half the time. Units >= nfull are those halves; each leaves its fp32
  // accumulator in args.tail_part ([unit - nfull][128 rows][BN columns]) and
  // tail_reduce_kernel adds the two halves (measured: prefill GEMM-2 777 ->
  // 753 us; the gated GEMM-1 lost more in its epilogue than it gained).
  const int G = (int)gridDim.x;
  const int nfull = (total / G) * G, ntail = total - nfull;
  const bool split = !SWIGLU && !GATHER && args.tail_part && ntail > 0 && 2 * ntail <= G;
  const int units = split ? nfull + 2 * ntail : total;
  // unit -> tile and K half (0: all of K, 1 / 2: first / second half)
  auto unit_tile = [&](int u, int& half) {
    if (split && u >= nfull) {
      half = 1 + ((u - nfull) & 1);
      return nfull + ((u - nfull) >> 1);
    }
    half = 0;
    return u;
  };
  auto k_range = [&](int half, int& kb0, int& kb1) {
    kb0 = half == 2 ? nkb / 2 : 0;
    kb1 = half == 1 ? nkb / 2 : nkb;
  };

  auto decode = [&](int tile, int& e, int& m, int& n) {
    e = find_expert(tile_start, args.E, tile);
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
        gather4_tile_rows(args.a_rows, soff[e] + m * BM, args.M_total, args.a_src_rows, lane,
                         src_row);
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
          const uint32_t sa = sbase + s * C::kStage, sb = sa + kTileA;
          if (lane == 0) {
            ptx::mbar_arrive_expect_tx(full0 + s * 8, C::kStage);
            ptx::tma_load_2d(sb, &tmB, kb * BK, rb0, full0 + s * 8);
            if (BN == 256) ptx::tma_load_2d(sb + 128 * 128, &tmB, kb * BK, rb1, full0 + s * 8);
          }
          __syncwarp();
          ptx::tma_gather4(sa + lane * 512, &tmA, kb * BK, src_row[0], src_row[1], src_row[2],
                           src_row[3], full0 + s * 8);
        }
      }
      __syncwarp();
      if (lane == 0) drain_loads<STAGES>(full0, issued, args.status);
    } else if (lane == 0) {
      int64_t issued = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int half;
        const int tile = unit_tile(u, half);
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
        constexpr bool two_b = BN == 256;
        int kb0, kb1;
        k_range(half, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb, ++issued) {
          const int s = (int)(issued % STAGES);
          const uint32_t ph = (uint32_t)((issued / STAGES) & 1);
          if (!ptx::mbar_wait(empty0 + s * 8, ph ^ 1, args.status, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + s * C::kStage, sb = sa + kTileA;
          ptx::mbar_arrive_expect_tx(full0 + s * 8, two_b ? C::kStage : kTileA + 128 * 128);
          ptx::tma_load_2d(sa, &tmA, kb * BK, row_a, full0 + s * 8);
          ptx::tma_load_2d(sb, &tmB, kb * BK, rb0, full0 + s * 8);
          if (two_b) ptx::tma_load_2d(sb + 128 * 128, &tmB, kb * BK, rb1, full0 + s * 8);
        }
      }
      drain_loads<STAGES>(full0, issued, args.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int64_t consumed = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int half, kb0, kb1;
        unit_tile(u, half);
        k_range(half, kb0, kb1);
        if (!ptx::mbar_wait(acce0 + acc * 8, acc_ph ^ 1, args.status, kSiteMmaAccEmpty)) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem_base + acc * C::kAccCols;
        for (int kb = kb0; kb < kb1; ++kb, ++consumed) {
          const int s = (int)(consumed % STAGES);
          const uint32_t ph = (uint32_t)((consumed / STAGES) & 1);
          if (!ptx::mbar_wait(full0 + s * 8, ph, args.status, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa = sbase + s * C::kStage, sb = sa + kTileA;
          const uint64_t da = ptx::sw128_kmajor_desc(sa), db = ptx::sw128_kmajor_desc(sb);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk)
            ptx::mma_f16(d, da + (uint64_t)(kk * UK * 2 / 16), db + (uint64_t)(kk * UK * 2 / 16),
                         C::kIdesc, kb != kb0 || kk != 0);
          ptx::mma_commit(empty0 + s * 8);
        }
        if (!ok) break;
        ptx::mma_commit(accf0 + acc * 8);
        acc ^= 1;
        if (acc == 0) acc_ph ^= 1;
      }
      // every MMA this thread issued has completed once `drain` fires
      ptx::mma_commit(drain);
      ptx::mbar_wait(drain, 0, args.status, kSiteDrain);
    }
  } else {
    // epilogue warps 2..5 -> TMEM lane quarter warp % 4
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      int half;
      const int tile = unit_tile(u, half);
      int e, m, n;
      decode(tile, e, m, n);
      const int row = soff[e] + m * BM + q * 32 + lane;
      const bool valid = row >= 0 && row < soff[e + 1] && row < args.M_total;
      if (!ptx::mbar_wait(accf0 + acc * 8, acc_ph, args.status, kSiteEpiAccFull)) break;
      ptx::tc_fence_after();
      const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::kAccCols;
      if (half) {  // one K half of a last-wave tile: the raw fp32 accumulator row
        float4* dst = reinterpret_cast<float4*>(args.tail_part + ((int64_t)(u - nfull) * BM + q * 32 + lane) * BN);
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          ptx::tmem_ld32(t0 + c, v);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[c / 4 + i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                         __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        }
      } else if (SWIGLU) {
        __nv_bfloat16* dst = args.C + (int64_t)row * args.ldc + n * 128;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t g[32], u[32];
          ptx::tmem_ld32(t0 + c, g);
          ptx::tmem_ld32(t0 + 128 + c, u);
          ptx::tmem_wait_ld();
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) h[i] = gated<ACT>(__uint_as_float(g[i]), __uint_as_float(u[i]));
          if (valid) store_row32(dst + c, h);
        }
      } else {
        __nv_bfloat16* dst = args.C + (int64_t)row * args.ldc + n * BN;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          ptx::tmem_ld32(t0 + c, v);
          ptx::tmem_wait_ld();
          float y[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(v[i]);
          if (valid) store_row32(dst + c, y);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acce0 + acc * 8);
      acc ^= 1;
      if (acc == 0) acc_ph ^= 1;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 512);
  }
}


// ==========================================================================
// tokens-in-M kernel with two-half tiles
// ==========================================================================
// Plain GEMMs with a long K (>= 4096). A tile is 256 routed rows (two halves
// of 128) by 256 weight columns. Each K step loads the two A halves and ONE
// 256-row weight tile and issues the MMAs of both halves against it, so a
// stage (64 KB) carries two thirds of the bytes per FLOP of a 128-row tile
// and takes twice the MMA time to consume: the three-stage ring hides about
// 2000 cycles of load latency instead of 1500. A half with no rows of the
// expert is neither loaded nor multiplied. The two accumulators (128 lanes x
// 256 columns each) fill TMEM, so there is no second buffer: eight epilogue
// warps (four per half) drain the two halves in parallel, and the next
// tile's MMAs into a half start as soon as that half is drained. Measured
// (same box): Mixtral-shaped GEMM-2 (K = 14336) 718-725 vs 767-768 us with
// 128-row tiles; the gated GEMM-1 (K = 4096 or 7168) was 2-4 % slower, its
// shorter tiles exposing the undoubled epilogue, so it keeps 128-row tiles.
struct Rows2Cfg {
  static constexpr int BN = 256;
  static constexpr int kTileB = BN * BK * 2;            // 32 KB
  static constexpr int kStage = 2 * kTileA + kTileB;    // 64 KB
  static constexpr int STAGES = kSmemBudget / kStage;   // 3
  static constexpr int kThreads2 = 320;
  static constexpr uint32_t kIdesc = ptx::make_idesc(BM, BN, 1, 1);
  static constexpr size_t kSmem = 1024 + (size_t)STAGES * kStage + 256 + 2 * (kMaxE + 1) * 4;
};

__global__ void __launch_bounds__(Rows2Cfg::kThreads2, 1)
    gemm_rows2_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, Args args) {
  using C = Rows2Cfg;
  constexpr int STAGES = C::STAGES;
  constexpr int BM2 = 2 * BM;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStage);
  // bars: full[STAGES], empty[STAGES], accf, acce[2], drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  int32_t* tile_start = reinterpret_cast<int32_t*>(smem + STAGES * C::kStage + 256);
  int32_t* soff = tile_start + kMaxE + 1;  // [E + 1] expert offsets, shared copy

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t full0 = ptx::smem_addr(bars), empty0 = full0 + STAGES * 8;
  const uint32_t accf = empty0 + STAGES * 8, acce0 = accf + 8, drain = acce0 + 16;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full0 + s * 8, 1);
      ptx::mbar_init(empty0 + s * 8, 1);
    }
    ptx::mbar_init(accf, 1);
    ptx::mbar_init(acce0, 4);
    ptx::mbar_init(acce0 + 8, 4);
    ptx::mbar_init(drain, 1);
    ptx::fence_barrier_init();
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_slot), 512);
    ptx::tmem_relinquish();
  }
  if (warp == 2) build_tile_starts<BM2>(args.offsets, args.E, args.NT, tile_start, soff);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_start[args.E];
  const int nkb = args.K / BK;

  auto decode = [&](int tile, int& e, int& m, int& n) {
    e = find_expert(tile_start, args.E, tile);
    const int local = tile - tile_start[e];
    const int cnt = soff[e + 1] - soff[e];
    const int mt = (cnt + BM2 - 1) / BM2;
    const int bsz = args.band * args.NT;
    const int b = local / bsz;
    const int rows = min(args.band, mt - b * args.band);
    const int l2 = local - b * bsz;
    n = l2 / rows;
    m = b * args.band + l2 % rows;
  };
  // the tile's second half holds rows of its expert
  auto has_half1 = [&](int e, int m) {
    return min(soff[e + 1], args.M_total) - (soff[e] + m * BM2) > BM;
  };

  if (warp == 0) {
    if (lane == 0) {
      int64_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, m, n;
        decode(tile, e, m, n);
        const int row_a = soff[e] + m * BM2;
        const bool h1 = has_half1(e, m);
        const int rb0 = e * args.b_rows + n * C::BN, rb1 = rb0 + 128;
        for (int kb = 0; kb < nkb; ++kb, ++issued) {
          const int s = (int)(issued % STAGES);
          const uint32_t ph = (uint32_t)((issued / STAGES) & 1);
          if (!ptx::mbar_wait(empty0 + s * 8, ph ^ 1, args.status, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + s * C::kStage, sb = sa + 2 * kTileA;
          ptx::mbar_arrive_expect_tx(full0 + s * 8, (h1 ? 2 * kTileA : kTileA) + C::kTileB);
          ptx::tma_load_2d(sa, &tmA, kb * BK, row_a, full0 + s * 8);
          if (h1) ptx::tma_load_2d(sa + kTileA, &tmA, kb * BK, row_a + BM, full0 + s * 8);
          ptx::tma_load_2d(sb, &tmB, kb * BK, rb0, full0 + s * 8);
          ptx::tma_load_2d(sb + 128 * 128, &tmB, kb * BK, rb1, full0 + s * 8);
        }
      }
      drain_loads<STAGES>(full0, issued, args.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int64_t consumed = 0;
      bool ok = true;
      int t = 0;  // tiles of this CTA so far
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++t) {
        int e, m, n;
        decode(tile, e, m, n);
        const bool h1 = has_half1(e, m);
        // a half's accumulator is free once the epilogue has drained it for the previous tile
        const uint32_t par = (uint32_t)((t & 1) ^ 1);
        if (!ptx::mbar_wait(acce0, par, args.status, kSiteMmaAccEmpty)) break;
        ptx::tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++consumed) {
          const int s = (int)(consumed % STAGES);
          const uint32_t ph = (uint32_t)((consumed / STAGES) & 1);
          if (!ptx::mbar_wait(full0 + s * 8, ph, args.status, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa = sbase + s * C::kStage, sb = sa + 2 * kTileA;
          const uint64_t da0 = ptx::sw128_kmajor_desc(sa), db = ptx::sw128_kmajor_desc(sb);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk)
            ptx::mma_f16(tmem_base, da0 + (uint64_t)(kk * UK * 2 / 16),
                         db + (uint64_t)(kk * UK * 2 / 16), C::kIdesc, kb != 0 || kk != 0);
          if (h1) {
            if (kb == 0) {
              if (!ptx::mbar_wait(acce0 + 8, par, args.status, kSiteMmaAccEmpty)) {
                ok = false;
                break;
              }
              ptx::tc_fence_after();
            }
            const uint64_t da1 = ptx::sw128_kmajor_desc(sa + kTileA);
#pragma unroll
            for (int kk = 0; kk < BK / UK; ++kk)
              ptx::mma_f16(tmem_base + C::BN, da1 + (uint64_t)(kk * UK * 2 / 16),
                           db + (uint64_t)(kk * UK * 2 / 16), C::kIdesc, kb != 0 || kk != 0);
          }
          ptx::mma_commit(empty0 + s * 8);
        }
        if (!ok) break;
        ptx::mma_commit(accf);
      }
      // every MMA this thread issued has completed once `drain` fires
      ptx::mma_commit(drain);
      ptx::mbar_wait(drain, 0, args.status, kSiteDrain);
    }
  } else {
    // epilogue warps 2..9: half h = (warp - 2) / 4, TMEM lane quarter warp % 4
    const int h = (warp - 2) >> 2;
    const int q = warp & 3;
    int t = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++t) {
      int e, m, n;
      decode(tile, e, m, n);
      const int row0 = soff[e] + m * BM2 + h * BM;
      const int row = row0 + q * 32 + lane;
      const bool valid = row >= 0 && row < soff[e + 1] && row < args.M_total;
      const bool any = h == 0 || has_half1(e, m);
      if (!ptx::mbar_wait(accf, (uint32_t)(t & 1), args.status, kSiteEpiAccFull)) break;
      ptx::tc_fence_after();
      const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + h * C::BN;
      if (any) {
        __nv_bfloat16* dst = args.C + (int64_t)row * args.ldc + n * C::BN;
#pragma unroll 1
        for (int c = 0; c < C::BN; c += 32) {
          uint32_t v[32];
          ptx::tmem_ld32(t0 + c, v);
          ptx::tmem_wait_ld();
          float y[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(v[i]);
          if (valid) store_row32(dst + c, y);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acce0 + h * 8);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 512);
  }
}

// Finishes the K-split last wave of the plain gemm_rows_kernel: block (i, y)
// takes rows [16 y, 16 y + 16) of tail tile nfull + i (the same tile order,
// recomputed from the offsets with the GEMM's grid size G), adds its two K
// halves (first + second, fp32) and writes them as bf16.
template <int BN>
__global__ void __launch_bounds__(256) tail_reduce_kernel(Args args, int G) {
  __shared__ int32_t tile_start[kMaxE + 1];
  __shared__ int32_t soff[kMaxE + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) build_tile_starts<BM>(args.offsets, args.E, args.NT, tile_start, soff);
  __syncthreads();
  const int total = tile_start[args.E];
  const int nfull = (total / G) * G, ntail = total - nfull;
  if (!(ntail > 0 && 2 * ntail <= G) || (int)blockIdx.x >= ntail) return;
  const int tile = nfull + (int)blockIdx.x;
  const int e = find_expert(tile_start, args.E, tile);
  const int local = tile - tile_start[e];
  const int mt = (soff[e + 1] - soff[e] + BM - 1) / BM;
  const int bsz = args.band * args.NT;
  const int b = local / bsz;
  const int rows = min(args.band, mt - b * args.band);
  const int l2 = local - b * bsz;
  const int n = l2 / rows, m = b * args.band + l2 % rows;
  const float* p0 = args.tail_part + (int64_t)(2 * blockIdx.x) * BM * BN;
  const float* p1 = p0 + (int64_t)BM * BN;
  for (int r = (int)blockIdx.y * 16 + warp; r < (int)blockIdx.y * 16 + 16; r += 8) {
    const int row = soff[e] + m * BM + r;
    if (row >= soff[e + 1] || row >= args.M_total) break;
    const float* a0 = p0 + (int64_t)r * BN;
    const float* a1 = p1 + (int64_t)r * BN;
    for (int c = 4 * lane; c < BN; c += 128) {
      const float4 v0 = *reinterpret_cast<const float4*>(a0 + c);
      const float4 v1 = *reinterpret_cast<const float4*>(a1 + c);
      *reinterpret_cast<uint2*>(args.C + (int64_t)row * args.ldc + n * BN + c) =
          make_uint2(pack_bf16x2(__fadd_rn(v0.x, v1.x), __fadd_rn(v0.y, v1.y)),
                     pack_bf16x2(__fadd_rn(v0.z, v1.z), __fadd_rn(v0.w, v1.w)));
    }
  }
}

// ==========================================================================
// small-M (swap-AB) kernel: weights in M, tokens in N
// ==========================================================================
template <int ACT, int BNT>
struct SwapCfg {
  static constexpr bool SWIGLU = ACT != kActNone;
  static constexpr int kNA = SWIGLU ? 2 : 1;                 // weight tiles per stage
  static constexpr int kTileB = BNT * BK * 2;
  static constexpr int kStage = kNA * kTileA + kTileB;       // multiple of 1024
  static constexpr int STAGES = (kSmemBudget / kStage) > 12 ? 12 : (kSmemBudget / kStage);
  static constexpr int kAccCols = kNA * BNT;                 // per accumulator buffer
  static constexpr int kTmemCols = (2 * kAccCols) <= 32 ? 32 : (2 * kAccCols) <= 64 ? 64
                                   : (2 * kAccCols) <= 128 ? 128 : 256;
  static constexpr uint32_t kIdesc = ptx::make_idesc(BM, BNT, 1, 1);
  static constexpr size_t kSmem = 1024 + (size_t)STAGES * kStage + 256 + 2 * (kMaxE + 1) * 4;
};

// tmA: weights [E*b_rows, K]; tmB: activation rows [M_total, K].
// Tile = (expert e, token tile tt, weight tile n); order: e, tt, n.
template <int ACT, int BNT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_swap_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, Args args) {
  using C = SwapCfg<ACT, BNT>;
  constexpr bool SWIGLU = ACT != kActNone;
  constexpr int STAGES = C::STAGES;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStage);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  int32_t* tile_start = reinterpret_cast<int32_t*>(smem + STAGES * C::kStage + 256);
  int32_t* soff = tile_start + kMaxE + 1;  // [E + 1] expert offsets, shared copy

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t full0 = ptx::smem_addr(bars), empty0 = full0 + STAGES * 8;
  const uint32_t accf0 = empty0 + STAGES * 8, acce0 = accf0 + 16, drain = acce0 + 16;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full0 + s * 8, 1);
      ptx::mbar_init(empty0 + s * 8, 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(accf0 + a * 8, 1);
      ptx::mbar_init(acce0 + a * 8, 4);
    }
    ptx::mbar_init(drain, 1);
    ptx::fence_barrier_init();
    ptx::tma_prefetch_desc(&tmA);
    ptx::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_slot), C::kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 2) build_tile_starts<BNT>(args.offsets, args.E, args.NT, tile_start, soff);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // work unit = (tile, k range): with ksplit > 1 each tile's K is cut into
  // ksplit ranges that run as separate units and leave fp32 partial sums
  const int S = args.ksplit;
  const int total = tile_start[args.E] * S;
  const int nkb = args.K / BK / S;  // k-blocks per unit

  auto decode = [&](int unit, int& e, int& tt, int& n, int& kb0) {
    const int tile = unit / S;
    kb0 = (unit % S) * nkb;
    e = find_expert(tile_start, args.E, tile);
    const int local = tile - tile_start[e];
    tt = local / args.NT;
    n = local % args.NT;
  };

  if (warp == 0) {
    if (lane == 0) {
      int64_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, tt, n, kb0;
        decode(tile, e, tt, n, kb0);
        const int row_b = soff[e] + tt * BNT;
        const int ra = e * args.b_rows + n * 128;
        for (int kb = kb0; kb < kb0 + nkb; ++kb, ++issued) {
          const int s = (int)(issued % STAGES);
          const uint32_t ph = (uint32_t)((issued / STAGES) & 1);
          if (!ptx::mbar_wait(empty0 + s * 8, ph ^ 1, args.status, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + s * C::kStage, sb = sa + C::kNA * kTileA;
          ptx::mbar_arrive_expect_tx(full0 + s * 8, C::kStage);
          ptx::tma_load_2d(sa, &tmA, kb * BK, ra, full0 + s * 8);
          if (SWIGLU) ptx::tma_load_2d(sa + kTileA, &tmA, kb * BK, ra + args.up_off, full0 + s * 8);
          ptx::tma_load_2d(sb, &tmB, kb * BK, row_b, full0 + s * 8);
        }
      }
      drain_loads<STAGES>(full0, issued, args.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int64_t consumed = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        if (!ptx::mbar_wait(acce0 + acc * 8, acc_ph ^ 1, args.status, kSiteMmaAccEmpty)) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem_base + acc * C::kAccCols;
        for (int kb = 0; kb < nkb; ++kb, ++consumed) {  // kb counts within the unit
          const int s = (int)(consumed % STAGES);
          const uint32_t ph = (uint32_t)((consumed / STAGES) & 1);
          if (!ptx::mbar_wait(full0 + s * 8, ph, args.status, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa = sbase + s * C::kStage, sb = sa + C::kNA * kTileA;
          const uint64_t da = ptx::sw128_kmajor_desc(sa), db = ptx::sw128_kmajor_desc(sb);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            const uint64_t ko = (uint64_t)(kk * UK * 2 / 16);
            ptx::mma_f16(d, da + ko, db + ko, C::kIdesc, (kb | kk) != 0);
            if (SWIGLU)
              ptx::mma_f16(d + BNT, da + (uint64_t)(kTileA >> 4) + ko, db + ko, C::kIdesc,
                           (kb | kk) != 0);
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
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int e, tt, n, kb0;
      decode(tile, e, tt, n, kb0);
      const int row0 = soff[e] + tt * BNT;
      const int nrows = min(min(BNT, soff[e + 1] - row0), args.M_total - row0);
      const int col = n * 128 + q * 32 + lane;  // output column owned by this thread
      if (!ptx::mbar_wait(accf0 + acc * 8, acc_ph, args.status, kSiteEpiAccFull)) break;
      ptx::tc_fence_after();
      const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::kAccCols;
#pragma unroll 1
      for (int c = 0; c < BNT; c += 16) {
        uint32_t g[16], u[16];
        ptx::tmem_ld16(t0 + c, g);
        if (SWIGLU) ptx::tmem_ld16(t0 + BNT + c, u);
        ptx::tmem_wait_ld();
        if (S == 1) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (c + i < nrows && row0 + c + i >= 0) {
              float v = SWIGLU ? gated<ACT>(__uint_as_float(g[i]), __uint_as_float(u[i]))
                               : __uint_as_float(g[i]);
              args.C[(int64_t)(row0 + c + i) * args.ldc + col] = __float2bfloat16_rn(v);
            }
          }
        } else {  // partial sums of this K range: gate in [0, ldc), up in [ldc, 2 ldc)
          const int pld = (SWIGLU ? 2 : 1) * args.ldc;
          float* P = args.partial + (int64_t)(kb0 / nkb) * args.M_total * pld;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (c + i < nrows && row0 + c + i >= 0) {
              float* prow = P + (int64_t)(row0 + c + i) * pld;
              prow[col] = __uint_as_float(g[i]);
              if (SWIGLU) prow[args.ldc + col] = __uint_as_float(u[i]);
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acce0 + acc * 8);
      acc ^= 1;
      if (acc == 0) acc_ph ^= 1;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Sum of the ksplit fp32 partials of each output in split order, then the
// epilogue the unsplit kernel would have applied (SwiGLU or none), to bf16.
template <int ACT>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ partial,
                                                            int S, int M, int N,
                                                            __nv_bfloat16* __restrict__ C) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)M * N) return;
  constexpr bool SWIGLU = ACT != kActNone;
  const int64_t r = i / N, c = i % N;
  const int pld = (SWIGLU ? 2 : 1) * N;
  const int64_t slice = (int64_t)M * pld;
  float g = 0.0f, u = 0.0f;
  for (int s = 0; s < S; ++s) {
    g += partial[s * slice + r * pld + c];
    if (SWIGLU) u += partial[s * slice + r * pld + N + c];
  }
  C[i] = __float2bfloat16_rn(SWIGLU ? gated<ACT>(g, u) : g);
}

}  // namespace gg

// ==========================================================================
// host side
// ==========================================================================
// bf16 grouped GEMM. B: [E, b_rows, K]; for SWIGLU b_rows = 2N.
// A_rows != nullptr: routed row r of A is row A_rows[r] of A ([A_src_rows, K]).
// scratch (may be null): room for the small-M kernel's split-K partials.
cudaError_t launch_grouped_gemm_bf16(const void* A, const int32_t* A_rows, int A_src_rows,
                                     const void* B, const int32_t* offsets, int M_total, int E,
                                     int N, int K, int act, void* Cout,
                                     int max_rows_per_expert, int32_t* status, void* scratch,
                                     size_t scratch_bytes, cudaStream_t s, const char** why) {
  const bool swiglu = act != kActNone;
  const int b_rows = swiglu ? 2 * N : N;
  CUtensorMap tmA, tmB;
  gg::Args a;
  a.offsets = offsets;
  a.E = E;
  a.K = K;
  a.ldc = N;
  a.b_rows = b_rows;
  a.up_off = swiglu ? N : 0;
  a.C = static_cast<__nv_bfloat16*>(Cout);
  a.M_total = M_total;
  a.a_rows = A_rows;
  a.a_src = A;
  a.a_src_rows = A_src_rows;
  a.ksplit = 1;
  a.tail_part = nullptr;
  a.partial = nullptr;
  const int64_t a_tmap_rows = A_rows ? A_src_rows : M_total;
  a.status = status;
  const int mrpe = max_rows_per_expert > 0 ? max_rows_per_expert : M_total;
  const int sms = num_sms();
  if (mrpe <= 64 && !A_rows) {
    // small-M variant: A operand = weights, B operand = tokens
    const int bnt = mrpe <= 16 ? 16 : mrpe <= 32 ? 32 : 64;
    if (!make_tmap(&tmA, B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, (int64_t)E * b_rows, 128) ||
        !make_tmap(&tmB, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, M_total, bnt)) {
      *why = "cuTensorMapEncodeTiled failed";
      return cudaErrorInvalidValue;
    }
    a.NT = N / 128;
    a.band = 1;
    const int64_t tiles_ub = ((int64_t)M_total / bnt + (M_total < E ? M_total : E)) * a.NT;
    // Split K so the units fill whole waves of SMs: a weight-streaming kernel
    // with a partial last wave leaves HBM bandwidth unused.
    const int nkb = K / gg::BK;
    const int64_t pld = (int64_t)(swiglu ? 2 : 1) * N;
    // Splitting costs pipeline ramps and the fp32 partials, so it is used only
    // when the unsplit units leave at least a fifth of the SMs' time idle.
    auto wave_eff = [&](int S) {
      const double waves = (double)tiles_ub * S / sms;
      return waves / std::ceil(waves);
    };
    double best = wave_eff(1);
    if (best < 0.8) {
      for (int S = 2; S <= 8; S *= 2) {
        if (nkb % S || nkb / S < 8) continue;
        if (!scratch || (int64_t)S * M_total * pld * 4 > (int64_t)scratch_bytes) continue;
        if (wave_eff(S) > best + 0.05) {
          best = wave_eff(S);
          a.ksplit = S;
        }
      }
    }
    if (a.ksplit > 1) a.partial = static_cast<float*>(scratch);
    const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(sms, tiles_ub * a.ksplit));
#define MOE_SWAP(SW, BNT)                                                                \
  do {                                                                                   \
    auto k = gg::gemm_swap_kernel<SW, BNT>;                                              \
    cudaError_t e = set_smem(k, gg::SwapCfg<SW, BNT>::kSmem);                            \
    if (e != cudaSuccess) return e;                                                      \
    k<<<grid, gg::kThreads, gg::SwapCfg<SW, BNT>::kSmem, s>>>(tmA, tmB, a);              \
  } while (0)
#define MOE_SWAP_ACT(ACTV)               \
  do {                                   \
    if (bnt == 16) MOE_SWAP(ACTV, 16);   \
    else if (bnt == 32) MOE_SWAP(ACTV, 32); \
    else MOE_SWAP(ACTV, 64);             \
  } while (0)
    if (act == kActSilu) MOE_SWAP_ACT(kActSilu);
    else if (act == kActGelu) MOE_SWAP_ACT(kActGelu);
    else if (act == kActRelu) MOE_SWAP_ACT(kActRelu);
    else MOE_SWAP_ACT(kActNone);
#undef MOE_SWAP_ACT
#undef MOE_SWAP
    note_launch();
    if (a.ksplit > 1) {
      const int64_t n = (int64_t)M_total * N;
#define MOE_REDUCE(ACTV) \
  gg::splitk_reduce_kernel<ACTV><<<(unsigned)ceil_div(n, 256), 256, 0, s>>>(a.partial, a.ksplit, M_total, N, a.C)
      if (act == kActSilu) MOE_REDUCE(kActSilu);
      else if (act == kActGelu) MOE_REDUCE(kActGelu);
      else if (act == kActRelu) MOE_REDUCE(kActRelu);
      else MOE_REDUCE(kActNone);
#undef MOE_REDUCE
      note_launch();
    }
    return cudaGetLastError();
  }
  const int BN = swiglu ? 256 : (N % 256 == 0 ? 256 : 128);
  // a gathered A is read by tile::gather4 from a map whose box is one row high
  if (!make_tmap(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, a_tmap_rows, A_rows ? 1 : 128) ||
      !make_tmap(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, (int64_t)E * b_rows, 128)) {
    *why = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  a.NT = swiglu ? N / 128 : N / BN;
  a.band = 16;
  // Plain GEMMs with a long K take two-half (256-row) tiles; the gated GEMM and
  // short-K plain GEMMs keep 128-row tiles, whose second accumulator buffer
  // hides their epilogue (and whose last wave can split over K).
  if (!A_rows && !swiglu && BN == 256 && K >= 4096) {
    a.band = 4;
    const int64_t tiles2 = ((int64_t)M_total / (2 * gg::BM) + (M_total < E ? M_total : E)) * a.NT;
    const unsigned grid2 = (unsigned)std::max<int64_t>(1, std::min<int64_t>(sms, tiles2));
    cudaError_t e = set_smem(gg::gemm_rows2_kernel, gg::Rows2Cfg::kSmem);
    if (e != cudaSuccess) return e;
    gg::gemm_rows2_kernel<<<grid2, gg::Rows2Cfg::kThreads2, gg::Rows2Cfg::kSmem, s>>>(tmA, tmB, a);
    note_launch();
    return cudaGetLastError();
  }
  const int64_t tiles_ub = ((int64_t)M_total / gg::BM + (M_total < E ? M_total : E)) * a.NT;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(sms, tiles_ub));
  // plain GEMM: scratch for a K-split last wave, at most `grid` half-tile
  // partials of 128 x BN fp32
  const size_t tail_bytes = (size_t)grid * gg::BM * BN * sizeof(float);
  if (!swiglu && !A_rows && scratch && scratch_bytes >= tail_bytes)
    a.tail_part = static_cast<float*>(scratch);
#define MOE_ROWS(SW, BNV)                                                                \
  do {                                                                                   \
    auto k = a.a_rows ? gg::gemm_rows_kernel<SW, BNV, true> : gg::gemm_rows_kernel<SW, BNV, false>; \
    cudaError_t e = set_smem(k, gg::RowsCfg<SW, BNV>::kSmem);                            \
    if (e != cudaSuccess) return e;                                                      \
    k<<<grid, gg::kThreads, gg::RowsCfg<SW, BNV>::kSmem, s>>>(tmA, tmB, a);              \
  } while (0)
  if (act == kActSilu)
    MOE_ROWS(kActSilu, 256);
  else if (act == kActGelu)
    MOE_ROWS(kActGelu, 256);
  else if (act == kActRelu)
    MOE_ROWS(kActRelu, 256);
  else if (BN == 256)
    MOE_ROWS(kActNone, 256);
  else
    MOE_ROWS(kActNone, 128);
#undef MOE_ROWS
  note_launch();
  if (a.tail_part) {  // finishes the last wave's tiles if the kernel split them
    const dim3 rgrid(grid, gg::BM / 16);
    if (BN == 256) gg::tail_reduce_kernel<256><<<rgrid, 256, 0, s>>>(a, (int)grid);
    else gg::tail_reduce_kernel<128><<<rgrid, 256, 0, s>>>(a, (int)grid);
    note_launch();
  }
  return cudaGetLastError();
}

}  // namespace moe
