// Router: logits GEMV and softmax top-k selection with renormalised weights.
//
// "Mixture of Experts (MoE): a practical explanation of how expert models
// work" (lira-now.com), section 5, steps 1-5 and its pseudocode: the router
// maps each token vector to E logits, softmax turns them into probabilities,
// the k largest are kept and renormalised over the selected experts.
//
// The logits decide integers (the selected ids), so they are computed in a
// fixed order: the h range is cut into 8 contiguous blocks of H/8; each block
// is summed from zero, h ascending, one fp32 fused multiply-add per term (a
// bf16 x bf16 product is exact in fp32, so the FMA equals the rounded sum of
// the exact product); the 8 block sums are added left to right, then the
// bias. Every logit is thus a fixed function of the inputs, whichever kernel
// computes it (tall, narrow, wide, split or not). The work runs on CUDA cores;
// tensor cores are not used here because their internal accumulation order
// is not specified.
#include "gemm_common.cuh"  // num_sms
#include "ptx.cuh"

namespace moe {

// N consecutive bf16 from shared memory, widened to fp32 (vector loads).
template <int N>
__device__ __forceinline__ void load_bf16_vec(const uint16_t* p, float (&v)[N]) {
  if constexpr (N == 8) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    v[0] = bf16lo_to_f32(u.x), v[1] = bf16hi_to_f32(u.x), v[2] = bf16lo_to_f32(u.y);
    v[3] = bf16hi_to_f32(u.y), v[4] = bf16lo_to_f32(u.z), v[5] = bf16hi_to_f32(u.z);
    v[6] = bf16lo_to_f32(u.w), v[7] = bf16hi_to_f32(u.w);
  } else if constexpr (N == 4) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    v[0] = bf16lo_to_f32(u.x), v[1] = bf16hi_to_f32(u.x);
    v[2] = bf16lo_to_f32(u.y), v[3] = bf16hi_to_f32(u.y);
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = __uint_as_float((uint32_t)p[i] << 16);
  }
}

// Wide router (E > 32). A block covers 64 tokens x 256 experts (grid.y
// walks expert chunks of 256) with 8 warps = 2 token halves x 4 expert
// quarters; inside a warp, lane = (token group 0..3, expert group 0..7) and
// each thread owns 8 tokens x 8 experts. Chunks of KC h values are converted
// to fp32 while being staged in shared memory, double-buffered through
// registers: x as [h][token], Wr as [h][half][expert group][4] so that one
// 16-byte load per lane gives a warp 8 different expert groups without bank
// conflicts. Per h a warp then moves 4 shared wavefronts for 64 fmas per
// thread. The inner loop uses paired FMAs (__ffma2_rn: two independent IEEE
// fmas per instruction); each (token, expert) sum follows the fixed blocked
// order: one fp32 fma per h within each of the 8 h blocks, the block sums
// added left to right as the blocks end.
constexpr int kRouterBlocks = 8;  // h blocks of the fixed summation order
constexpr int kWideKC = 32;

// SPLIT: grid.z runs the 8 h blocks as separate CTAs, each writing its
// block sums to part[b][t][e] (the running total and the bias are then
// applied by topk_kernel<PER, true>, in the same order); for many more CTAs
// than the 64-token tiles give and without the running-total registers;
// two CTAs per SM (128 registers) for more warps to hide the FMA latency.
template <bool VEC, bool SPLIT>
__global__ void __launch_bounds__(256, SPLIT ? 2 : 1) router_wide_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wr,
    const float* __restrict__ bias, int T, int H, int E, float* __restrict__ logits,
    float* __restrict__ part) {
  constexpr int BT = 64, EC = 256, KC = kWideKC;
  constexpr int XVEC = BT * KC / 8 / 256;  // 16-byte x vectors per thread per chunk (1)
  constexpr int WVEC = KC * EC / 8 / 256;  // 16-byte Wr vectors per thread per chunk (4)
  static_assert(XVEC == 1 && WVEC == 4, "staging layout");
  extern __shared__ __align__(16) unsigned char router_smem[];
  float* xs = reinterpret_cast<float*>(router_smem);  // [2][KC][BT]
  float* ws = xs + 2 * KC * BT;                        // [2][KC][2][EC/8][4]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tok0 = (warp >> 2) * 32 + (lane >> 3) * 8;  // this thread's 8 tokens (in block)
  const int eg = (warp & 3) * 8 + (lane & 7);           // this thread's expert group (of 32)
  const int t0 = blockIdx.x * BT, e0 = blockIdx.y * EC;
  const uint16_t* xg = reinterpret_cast<const uint16_t*>(x);
  const uint16_t* wg = reinterpret_cast<const uint16_t*>(wr);

  uint4 xr, wreg[WVEC];
  // x staging: thread -> (token tid % 64, h-octet tid / 64): a warp stores 32
  // consecutive tokens of one h, conflict-free
  const int xt = tid % BT, xc8 = (tid / BT) * 8;
  auto load = [&](int k0) {
    xr = (t0 + xt < T) ? *reinterpret_cast<const uint4*>(xg + (int64_t)(t0 + xt) * H + k0 + xc8)
                       : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < WVEC; ++i) {
      const int v = tid + i * 256, h = v / (EC / 8), e8 = (v % (EC / 8)) * 8;
      if (VEC) {
        wreg[i] = (e0 + e8 < E) ? *reinterpret_cast<const uint4*>(wg + (int64_t)(k0 + h) * E + e0 + e8)
                                : make_uint4(0, 0, 0, 0);
      } else {
        uint16_t tmp[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          tmp[j] = (e0 + e8 + j < E) ? wg[(int64_t)(k0 + h) * E + e0 + e8 + j] : (uint16_t)0;
        wreg[i] = *reinterpret_cast<uint4*>(tmp);
      }
    }
  };
  auto store = [&](int b) {
    {
      float* d = xs + (b * KC + xc8) * BT + xt;
      d[0 * BT] = bf16lo_to_f32(xr.x), d[1 * BT] = bf16hi_to_f32(xr.x);
      d[2 * BT] = bf16lo_to_f32(xr.y), d[3 * BT] = bf16hi_to_f32(xr.y);
      d[4 * BT] = bf16lo_to_f32(xr.z), d[5 * BT] = bf16hi_to_f32(xr.z);
      d[6 * BT] = bf16lo_to_f32(xr.w), d[7 * BT] = bf16hi_to_f32(xr.w);
    }
#pragma unroll
    for (int i = 0; i < WVEC; ++i) {
      const int v = tid + i * 256, h = v / (EC / 8), g = v % (EC / 8);
      float* d = ws + (b * KC + h) * EC + g * 4;  // half 0 at +0, half 1 at +EC/2
      const uint4 u = wreg[i];
      *reinterpret_cast<float4*>(d) =
          make_float4(bf16lo_to_f32(u.x), bf16hi_to_f32(u.x), bf16lo_to_f32(u.y), bf16hi_to_f32(u.y));
      *reinterpret_cast<float4*>(d + EC / 2) =
          make_float4(bf16lo_to_f32(u.z), bf16hi_to_f32(u.z), bf16lo_to_f32(u.w), bf16hi_to_f32(u.w));
    }
  };

  // acc[a][p]: the current h block's sums of experts (2p, 2p+1) of token a;
  // tot[a][p]: the finished blocks' sums, added left to right (the fixed
  // blocked order: 8 contiguous h blocks, each summed from zero)
  float2 acc[8][4], tot[SPLIT ? 1 : 8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int p = 0; p < 4; ++p) acc[a][p] = make_float2(0.0f, 0.0f);
  if constexpr (!SPLIT) {
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int p = 0; p < 4; ++p) tot[a][p] = make_float2(0.0f, 0.0f);
  }
  const int L = H / kRouterBlocks;  // a multiple of 16, so blocks end on 16-h steps
  const int hbase = SPLIT ? (int)blockIdx.z * L : 0;  // SPLIT: L is a multiple of KC
  const int nchunks = (SPLIT ? L : H) / KC;
  int done = 0;                     // finished blocks
  auto fold = [&]() {
    if constexpr (SPLIT) return;
    else {
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        tot[a][p] = done == 0 ? acc[a][p]
                              : make_float2(__fadd_rn(tot[a][p].x, acc[a][p].x),
                                            __fadd_rn(tot[a][p].y, acc[a][p].y));
        acc[a][p] = make_float2(0.0f, 0.0f);
      }
    ++done;
    }
  };
  load(hbase);
  store(0);
  __syncthreads();
  for (int c = 0; c < nchunks; ++c) {
    const int b = c & 1;
    if (c + 1 < nchunks) load(hbase + (c + 1) * KC);
    const float* xb = xs + b * KC * BT + tok0;
    const float* wb = ws + b * KC * EC + eg * 4;
#pragma unroll 1
    for (int h0 = 0; h0 < KC; h0 += 16) {
#pragma unroll 4
      for (int h = h0; h < h0 + 16; ++h) {
        const float4 x0 = *reinterpret_cast<const float4*>(xb + h * BT);
        const float4 x1 = *reinterpret_cast<const float4*>(xb + h * BT + 4);
        const float4 w0 = *reinterpret_cast<const float4*>(wb + h * EC);
        const float4 w1 = *reinterpret_cast<const float4*>(wb + h * EC + EC / 2);
        const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        const float2 wv[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w),
                              make_float2(w1.x, w1.y), make_float2(w1.z, w1.w)};
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          const float2 xa = make_float2(xv[a], xv[a]);
#pragma unroll
          for (int p = 0; p < 4; ++p) acc[a][p] = __ffma2_rn(xa, wv[p], acc[a][p]);
        }
      }
      if (!SPLIT && (c * KC + h0 + 16) % L == 0) fold();
    }
    if (c + 1 < nchunks) store(b ^ 1);
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int t = t0 + tok0 + a;
    if (t >= T) continue;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int ee = e0 + eg * 8 + 2 * p;
      if constexpr (SPLIT) {
        float* d = part + ((int64_t)blockIdx.z * T + t) * E + ee;
        if (ee < E) d[0] = acc[a][p].x;
        if (ee + 1 < E) d[1] = acc[a][p].y;
      } else {
        if (ee < E) logits[(int64_t)t * E + ee] = __fadd_rn(tot[a][p].x, bias ? bias[ee] : 0.0f);
        if (ee + 1 < E)
          logits[(int64_t)t * E + ee + 1] = __fadd_rn(tot[a][p].y, bias ? bias[ee + 1] : 0.0f);
      }
    }
  }
}

// One warp per token. Lane l holds logits e = l + 32*i. k rounds of a warp
// argmax on (logit desc, index asc); slot j gets the j-th winner. Weights:
// w_j = exp(l_j - l_max) / sum_selected exp(l_i - l_max).
// PART: the logits are first formed from the 8 block sums part[b][t][e] of
// the split wide kernel, added left to right, then the bias (the fixed
// blocked order), and written to `logits`.
template <int PER, bool PART>
__global__ void __launch_bounds__(256) topk_kernel(float* __restrict__ logits,
                                                   const float* __restrict__ part,
                                                   const float* __restrict__ bias, int T, int E,
                                                   int k, int32_t* __restrict__ ids,
                                                   float* __restrict__ w) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  float* l = logits + (int64_t)warp * E;
  float v[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    int e = lane + 32 * i;
    if constexpr (PART) {
      if (e < E) {
        const float* p = part + (int64_t)warp * E + e;
        float s = p[0];
#pragma unroll
        for (int b = 1; b < kRouterBlocks; ++b) s = __fadd_rn(s, p[(int64_t)b * T * E]);
        s = __fadd_rn(s, bias ? bias[e] : 0.0f);
        l[e] = s;
        v[i] = s;
      } else {
        v[i] = -INFINITY;
      }
    } else {
      v[i] = e < E ? l[e] : -INFINITY;
    }
  }
  uint32_t taken = 0;  // bit i: v[i] already selected (or absent)
#pragma unroll
  for (int i = 0; i < PER; ++i)
    if (lane + 32 * i >= E) taken |= 1u << i;
  float sel_l = 0.0f, lmax = 0.0f;
  int sel_e = 0;
  float my_ex = 0.0f;
  int my_slot = -1;
  float denom = 0.0f;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      int e = lane + 32 * i;
      bool ok = !(taken >> i & 1u);
      if (ok && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    sel_l = bv;
    sel_e = be;
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (j == 0) lmax = sel_l;
    float ex = expf(sel_l - lmax);
    denom += ex;
    if (lane == j) {
      my_ex = ex;
      my_slot = j;
      ids[(int64_t)warp * k + j] = sel_e;
    }
  }
  if (my_slot >= 0) w[(int64_t)warp * k + my_slot] = __fdiv_rn(my_ex, denom);
}

// Top-k of one token's E <= 32 logits held in shared memory, by one warp
// (lane = expert): k rounds of a warp argmax on (logit desc, index asc); the
// renormalised weights are exp(l - l_max) over their sum.
__device__ __forceinline__ void warp_topk32(const float* lg, int E, int k, int64_t tt, int lane,
                                            int32_t* __restrict__ ids, float* __restrict__ topw) {
  const float v = lane < E ? lg[lane] : -INFINITY;
  bool taken = lane >= E;
  float lmax = 0.0f, denom = 0.0f, my_ex = 0.0f;
  int my_slot = -1;
  for (int j = 0; j < k; ++j) {
    float bv = taken ? -INFINITY : v;
    int be = taken ? 0x7fffffff : lane;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ov > bv || (ov == bv && oe < be)) bv = ov, be = oe;
    }
    if (be == lane) taken = true;
    if (j == 0) lmax = bv;
    const float ex = expf(bv - lmax);
    denom += ex;
    if (lane == j) {
      my_ex = ex;
      my_slot = j;
      ids[tt * k + j] = be;
    }
  }
  if (my_slot >= 0) topw[tt * k + my_slot] = __fdiv_rn(my_ex, denom);
}

// Narrow router with fused top-k (E <= 32). The logit sum runs in the fixed
// blocked order (8 contiguous h blocks, each summed from zero, then added
// left to right), and the 8 block sums of a (token, expert pair) are computed
// by 8 threads at once, so each sequential chain is H/8 paired FMAs long:
//  * compute thread (token, pair, block b), b in the low 3 bits of the
//    thread index: two sums (experts 2p, 2p+1) advanced together by paired
//    FMAs (__ffma2_rn, two IEEE fmas per instruction) over block b's h;
//  * each chunk covers 16 h of every block; four helper warps stream x rows and
//    Wr rows through a cp.async ring (raw bf16) and widen each chunk into
//    fp32 "ready" buffers laid out for the compute loop, b fastest: x as
//    {x_h, x_h, x_h+1, x_h+1} per (token, block), Wr as
//    {w_h,e, w_h,e+1, w_h+1,e, w_h+1,e+1} per (pair, block);
//  * the 8 block sums are combined in order through warp shuffles, and the
//    top-k selection runs per token over the E logits staged in shared
//    memory (k rounds of a warp argmax on (logit desc, index asc)).
constexpr int kNarrowSL = 16;          // h per block per chunk (chunk = 128 h)
constexpr int kNarrowNS = 4;           // raw chunks in flight
constexpr int kNarrowCT = 128;         // compute threads per CTA
constexpr int kNarrowHT = 128;         // helper threads per CTA
constexpr int kNarrowXP = 256 + 16;    // raw x bytes per token per chunk (8 blocks x 32 B), padded

__host__ __device__ constexpr size_t narrow_stage_bytes(int BT, int E) {
  return (size_t)BT * kNarrowXP + (size_t)kRouterBlocks * kNarrowSL * E * 2;
}
__host__ __device__ constexpr size_t narrow_smem_bytes(int BT, int EPP, int E) {
  return kNarrowNS * narrow_stage_bytes(BT, E) +
         2 * (size_t)(kNarrowSL / 2) * kRouterBlocks * 16 * (BT + EPP) + (size_t)BT * 32 * 4;
}

template <int EPP>  // expert pairs per token (power of two, 1..16)
__global__ void __launch_bounds__(kNarrowCT + kNarrowHT) router_narrow_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wr,
    const float* __restrict__ bias, int T, int H, int E, int k, float* __restrict__ logits,
    int32_t* __restrict__ ids, float* __restrict__ topw) {
  constexpr int NB = kRouterBlocks, SL = kNarrowSL, NS = kNarrowNS, XP = kNarrowXP;
  constexpr int BT = kNarrowCT / (EPP * NB);   // tokens per CTA (16 / EPP)
  constexpr int NH = kNarrowHT;
  constexpr int XV = BT * NB * 2;              // 16-byte raw x vectors per chunk
  constexpr int XI = (SL / 2) * BT * NB;       // x items (h pair, token, block) per chunk
  constexpr int WI = (SL / 2) * EPP * NB;      // Wr items (h pair, pair, block) per chunk
  extern __shared__ __align__(16) unsigned char narrow_smem[];
  const int tid = threadIdx.x;
  const bool helper = tid >= kNarrowCT;
  const int hid = tid - kNarrowCT;
  const int b = tid & (NB - 1), p = (tid >> 3) % EPP, tl = (tid >> 3) / EPP;
  const int t0 = blockIdx.x * BT;
  const int L = H / NB;                        // h per block (a multiple of 16)
  const int nchunks = L / SL;
  const size_t stage = narrow_stage_bytes(BT, E);
  unsigned char* ring = narrow_smem;
  float4* rx = reinterpret_cast<float4*>(narrow_smem + NS * stage);  // [2][SL/2][BT][NB]
  float4* rw = rx + 2 * (SL / 2) * BT * NB;                            // [2][SL/2][EPP][NB]
  float* slg = reinterpret_cast<float*>(rw + 2 * (SL / 2) * EPP * NB);  // [BT][32] logits
  const char* xg = reinterpret_cast<const char*>(x);
  const char* wg = reinterpret_cast<const char*>(wr);

  // helpers: raw chunk c -> ring slot c % NS: per token its 8 block slices of
  // 16 h (32 B each), then per block 16 Wr rows (one contiguous 32*E bytes)
  auto issue = [&](int c) {
    if (c < nchunks) {
      const uint32_t st = ptx::smem_addr(ring + (c % NS) * stage);
      for (int i = hid; i < XV; i += NH) {
        const int r = i / (NB * 2), bb = (i / 2) % NB, v = i & 1, t = t0 + r;
        const char* src = xg + ((int64_t)(t < T ? t : 0) * H + (int64_t)bb * L + c * SL) * 2 + v * 16;
        ptx::cp_async16(st + r * XP + (bb * 2 + v) * 16, src, t < T ? 16u : 0u);
      }
      const int wv = 2 * E;  // 16-byte vectors per block slice
      const uint32_t wdst = st + BT * XP;
      for (int i = hid; i < NB * wv; i += NH) {
        const int bb = i / wv, v = i % wv;
        const char* src = wg + ((int64_t)bb * L + c * SL) * E * 2 + v * 16;
        ptx::cp_async16(wdst + (bb * wv + v) * 16, src, 16u);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // helpers: widen raw chunk c into ready buffer c & 1
  auto convert = [&](int c) {
    const unsigned char* st = ring + (c % NS) * stage;
    float4* dx = rx + (c & 1) * (SL / 2) * BT * NB;
#pragma unroll
    for (int it = 0; it < (XI + NH - 1) / NH; ++it) {
      const int i = hid + it * NH;
      if (XI % NH != 0 && i >= XI) break;
      const int bb = i % NB, r = (i / NB) % BT, j = i / (NB * BT);
      const uint32_t u = *reinterpret_cast<const uint32_t*>(st + r * XP + bb * 32 + j * 4);
      const float lo = bf16lo_to_f32(u), hi = bf16hi_to_f32(u);
      dx[(j * BT + r) * NB + bb] = make_float4(lo, lo, hi, hi);
    }
    const unsigned char* sw = st + BT * XP;  // [NB][SL][E] bf16
    float4* dw = rw + (c & 1) * (SL / 2) * EPP * NB;
#pragma unroll
    for (int it = 0; it < (WI + NH - 1) / NH; ++it) {
      const int i = hid + it * NH;
      if (WI % NH != 0 && i >= WI) break;
      const int bb = i % NB, pp = (i / NB) % EPP, j = i / (NB * EPP), e0 = 2 * pp;
      const int o0 = (bb * SL + 2 * j) * E + e0, o1 = o0 + E;  // elements of rows 2j, 2j+1
      uint32_t u0, u1;
      if ((E & 1) == 0) {  // the pair is one aligned 32-bit word
        u0 = e0 < E ? *reinterpret_cast<const uint32_t*>(sw + 2 * o0) : 0u;
        u1 = e0 < E ? *reinterpret_cast<const uint32_t*>(sw + 2 * o1) : 0u;
      } else {
        const uint16_t* h16 = reinterpret_cast<const uint16_t*>(sw);
        u0 = (e0 < E ? (uint32_t)h16[o0] : 0u) | (e0 + 1 < E ? (uint32_t)h16[o0 + 1] << 16 : 0u);
        u1 = (e0 < E ? (uint32_t)h16[o1] : 0u) | (e0 + 1 < E ? (uint32_t)h16[o1 + 1] << 16 : 0u);
      }
      dw[(j * EPP + pp) * NB + bb] = make_float4(bf16lo_to_f32(u0), bf16hi_to_f32(u0),
                                                 bf16lo_to_f32(u1), bf16hi_to_f32(u1));
    }
  };

  if (helper) {
#pragma unroll 1
    for (int c = 0; c < NS; ++c) issue(c);
    asm volatile("cp.async.wait_group %0;" ::"n"(NS - 1) : "memory");
  }
  __syncthreads();
  if (helper) convert(0);
  float2 acc = make_float2(0.0f, 0.0f);  // compute threads: block b's sums of experts (2p, 2p+1)
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    // helpers' copies of chunk c+1 landed; the barrier publishes them and the
    // ready buffer of chunk c, and frees ring slot c % NS and buffer (c+1) & 1
    if (helper) asm volatile("cp.async.wait_group %0;" ::"n"(NS - 2) : "memory");
    __syncthreads();
    if (helper) {
      issue(c + NS);
      if (c + 1 < nchunks) convert(c + 1);
    } else {
      const float4* xb = rx + (c & 1) * (SL / 2) * BT * NB + tl * NB + b;
      const float4* wb = rw + (c & 1) * (SL / 2) * EPP * NB + p * NB + b;
#pragma unroll
      for (int j = 0; j < SL / 2; ++j) {
        const float4 xv = xb[j * BT * NB], wv = wb[j * EPP * NB];
        acc = __ffma2_rn(make_float2(xv.x, xv.y), make_float2(wv.x, wv.y), acc);
        acc = __ffma2_rn(make_float2(xv.z, xv.w), make_float2(wv.z, wv.w), acc);
      }
    }
  }
  if (helper) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    return;
  }

  // block sums -> logits, added left to right by the block-0 lane of each group
  const int lane = tid & 31;
  float s0 = acc.x, s1 = acc.y;
#pragma unroll
  for (int i = 1; i < NB; ++i) {
    const float a0 = __shfl_sync(0xffffffffu, acc.x, (lane & ~(NB - 1)) + i);
    const float a1 = __shfl_sync(0xffffffffu, acc.y, (lane & ~(NB - 1)) + i);
    s0 = __fadd_rn(s0, a0);
    s1 = __fadd_rn(s1, a1);
  }
  const int t = t0 + tl, e0 = 2 * p, e1 = 2 * p + 1;
  if (b == 0) {
    const float l0 = __fadd_rn(s0, bias ? bias[e0 < E ? e0 : 0] : 0.0f);
    const float l1 = __fadd_rn(s1, bias ? bias[e1 < E ? e1 : 0] : 0.0f);
    if (e0 < E) slg[tl * 32 + e0] = l0;
    if (e1 < E) slg[tl * 32 + e1] = l1;
    if (t < T && logits) {
      if (e0 < E) logits[(int64_t)t * E + e0] = l0;
      if (e1 < E) logits[(int64_t)t * E + e1] = l1;
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kNarrowCT) : "memory");  // compute warps only
  // top-k: warp w takes tokens w, w + 4, ...
  const int w = tid >> 5;
  for (int r = w; r < BT; r += kNarrowCT / 32) {
    if (t0 + r >= T) break;
    warp_topk32(slg + r * 32, E, k, t0 + r, lane, ids, topw);
  }
}


// Tall router with fused top-k (E <= 32, many tokens). The CTA holds the
// whole of Wr, widened to fp32, in shared memory ([H][EV]); warp b owns h
// block b and lane l token t0 + l, so every shared load of a Wr row is one
// broadcast to the 32 tokens of the warp. Each thread keeps the EV sums of
// its (token, block) in registers, one paired FMA per h and expert pair, and
// reads its x slice straight from global memory, 16 h (32 bytes) per step
// with two steps in flight. The 8 block sums of a (token, expert) meet in
// shared memory and are added left to right, then the bias.
template <int EV>  // experts padded to a power of two (2..32)
__global__ void __launch_bounds__(256, 1) router_tall_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wr,
    const float* __restrict__ bias, int T, int H, int E, int k, int BT, float* __restrict__ logits,
    int32_t* __restrict__ ids, float* __restrict__ topw) {
  constexpr int NB = kRouterBlocks;
  extern __shared__ __align__(16) float tall_smem[];
  const int L = H / NB;                  // a multiple of 16 (H % 128 == 0)
  float* sw = tall_smem;                 // [H][EV] Wr in fp32, padded experts zero
  float* part = sw + (size_t)H * EV;     // [NB][32][EV] block sums
  float* slg = part + NB * 32 * EV;      // [32][32] logits for the top-k
  const int tid = threadIdx.x, b = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * BT;
  const int tr = min(t0 + lane, T - 1);  // lanes past the last token read a valid row, never write
  const uint4* xp = reinterpret_cast<const uint4*>(x + (int64_t)tr * H + (int64_t)b * L);
  const int nsteps = L / 16;
  uint4 xa0 = __ldg(xp), xa1 = __ldg(xp + 1), xb0 = xa0, xb1 = xa1;
  if (nsteps > 1) xb0 = __ldg(xp + 2), xb1 = __ldg(xp + 3);

  // stage Wr: 8 bf16 per 16-byte load, several loads in flight per thread
  const uint4* w4 = reinterpret_cast<const uint4*>(wr);
  const int nvec = H * E / 8;
  if (E == EV) {  // no padding: the table is Wr widened in place, two 16-byte stores per load
#pragma unroll 4
    for (int v = tid; v < nvec; v += blockDim.x) {
      const uint4 u = __ldg(w4 + v);
      float4* d = reinterpret_cast<float4*>(sw + 8 * v);
      d[0] = make_float4(bf16lo_to_f32(u.x), bf16hi_to_f32(u.x), bf16lo_to_f32(u.y), bf16hi_to_f32(u.y));
      d[1] = make_float4(bf16lo_to_f32(u.z), bf16hi_to_f32(u.z), bf16lo_to_f32(u.w), bf16hi_to_f32(u.w));
    }
  } else {
#pragma unroll 4
  for (int v = tid; v < nvec; v += blockDim.x) {
    const uint4 u = __ldg(w4 + v);
    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
    int h = (8 * v) / E, e = (8 * v) % E;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      sw[h * EV + e] = (q & 1) ? bf16hi_to_f32(uw[q >> 1]) : bf16lo_to_f32(uw[q >> 1]);
      if (++e == E) e = 0, ++h;
    }
  }
  }
  if (E < EV) {
    const int pad = EV - E;
    for (int i = tid; i < H * pad; i += blockDim.x) sw[(i / pad) * EV + E + i % pad] = 0.0f;
  }
  __syncthreads();

  float2 acc[EV / 2];
#pragma unroll
  for (int i = 0; i < EV / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);
  const float* wb = sw + (size_t)b * L * EV;
#pragma unroll 1
  for (int st = 0; st < nsteps; ++st) {
    const uint32_t xw[8] = {xa0.x, xa0.y, xa0.z, xa0.w, xa1.x, xa1.y, xa1.z, xa1.w};
    xa0 = xb0, xa1 = xb1;
    if (st + 2 < nsteps) xb0 = __ldg(xp + 2 * st + 4), xb1 = __ldg(xp + 2 * st + 5);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const float xf = (q & 1) ? bf16hi_to_f32(xw[q >> 1]) : bf16lo_to_f32(xw[q >> 1]);
      const float2 xx = make_float2(xf, xf);
      const float* wh = wb + (st * 16 + q) * EV;
      if constexpr (EV >= 4) {
#pragma unroll
        for (int e4 = 0; e4 < EV / 4; ++e4) {
          const float4 wv = *reinterpret_cast<const float4*>(wh + 4 * e4);
          acc[2 * e4] = __ffma2_rn(xx, make_float2(wv.x, wv.y), acc[2 * e4]);
          acc[2 * e4 + 1] = __ffma2_rn(xx, make_float2(wv.z, wv.w), acc[2 * e4 + 1]);
        }
      } else {
        acc[0] = __ffma2_rn(xx, *reinterpret_cast<const float2*>(wh), acc[0]);
      }
    }
  }
  float* pp = part + (b * 32 + lane) * EV;
#pragma unroll
  for (int i = 0; i < EV / 2; ++i) *reinterpret_cast<float2*>(pp + 2 * i) = acc[i];
  __syncthreads();
  // block sums -> logits, added left to right, then the bias
  for (int i = tid; i < BT * E; i += blockDim.x) {
    const int tl = i / E, e = i % E;
    float sum = part[tl * EV + e];
#pragma unroll
    for (int bb = 1; bb < NB; ++bb) sum = __fadd_rn(sum, part[(bb * 32 + tl) * EV + e]);
    const float l = __fadd_rn(sum, bias ? bias[e] : 0.0f);
    slg[tl * 32 + e] = l;
    if (t0 + tl < T && logits) logits[(int64_t)(t0 + tl) * E + e] = l;
  }
  __syncthreads();
  const int nw = blockDim.x >> 5;
  for (int r = b; r < BT; r += nw) {
    if (t0 + r >= T) break;
    warp_topk32(slg + r * 32, E, k, t0 + r, lane, ids, topw);
  }
}

static size_t tall_smem_bytes(int H, int EV) {
  return ((size_t)H * EV + (size_t)kRouterBlocks * 32 * EV + 32 * 32) * 4;
}

// Pairs per token for the narrow router (E padded to a power of two >= 2).
static int narrow_pairs(int E) {
  const int ep = E <= 2 ? 2 : E <= 4 ? 4 : E <= 8 ? 8 : E <= 16 ? 16 : 32;
  return ep / 2;
}

cudaError_t launch_topk_part(float* logits, const float* part, const float* bias, int T, int E,
                             int k, int32_t* ids, float* w, cudaStream_t s);

// Logits and top-k of T tokens: for E <= 32 the fused tall kernel (many
// tokens, Wr fits shared memory) or the fused narrow kernel; else the wide
// logits kernel followed by the warp-per-token selection. With scratch for
// 8 T E floats (and H a multiple of 256) the wide kernel runs its 8 h blocks
// as separate CTAs and the selection adds the block sums in order.
constexpr int kTallMinT = 1024;
constexpr size_t kTallMaxSmem = 200 * 1024;
cudaError_t launch_route(const void* x, const void* wr, const float* bias, int T, int H, int E,
                         int k, float* logits, int32_t* ids, float* w, float* part,
                         size_t part_bytes, cudaStream_t s) {
  const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(x);
  const __nv_bfloat16* wp = static_cast<const __nv_bfloat16*>(wr);
  if (E <= 32 && T >= kTallMinT) {
    const int ev = 2 * narrow_pairs(E);
    // tokens per CTA (lanes of a warp): about one CTA per SM
    const int sms = num_sms();
    const int bt = std::min(32, std::max(1, (int)((T + sms - 1) / sms)));
    const size_t smem = tall_smem_bytes(H, ev);
    if (smem <= kTallMaxSmem) {
#define MOE_TALL(EVV)                                                                          \
  do {                                                                                         \
    cudaFuncSetAttribute(router_tall_kernel<EVV>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                         (int)smem);                                                           \
    router_tall_kernel<EVV><<<(unsigned)ceil_div(T, bt), 32 * kRouterBlocks, smem, s>>>(       \
        xp, wp, bias, T, H, E, k, bt, logits, ids, w);                                         \
  } while (0)
      if (ev == 2) MOE_TALL(2);
      else if (ev == 4) MOE_TALL(4);
      else if (ev == 8) MOE_TALL(8);
      else if (ev == 16) MOE_TALL(16);
      else MOE_TALL(32);
#undef MOE_TALL
      note_launch();
      return cudaGetLastError();
    }
  }
  if (E <= 32) {
    const int epp = narrow_pairs(E);
#define MOE_NARROW(P)                                                                         \
  do {                                                                                        \
    constexpr int BTV = kNarrowCT / (P * kRouterBlocks);                                      \
    const size_t smem = narrow_smem_bytes(BTV, P, E);                                         \
    cudaFuncSetAttribute(router_narrow_kernel<P>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                         (int)smem);                                                          \
    router_narrow_kernel<P><<<(unsigned)ceil_div(T, BTV), kNarrowCT + kNarrowHT, smem, s>>>(  \
        xp, wp, bias, T, H, E, k, logits, ids, w);                                            \
  } while (0)
    if (epp == 1) MOE_NARROW(1);
    else if (epp == 2) MOE_NARROW(2);
    else if (epp == 4) MOE_NARROW(4);
    else if (epp == 8) MOE_NARROW(8);
    else MOE_NARROW(16);
#undef MOE_NARROW
    note_launch();
    return cudaGetLastError();
  }
  const size_t smem = 2 * (size_t)kWideKC * (64 + 256) * 4;
  const bool split = part && part_bytes >= (size_t)kRouterBlocks * T * E * sizeof(float) &&
                     (H / kRouterBlocks) % kWideKC == 0;
  dim3 grid((unsigned)ceil_div(T, 64), (unsigned)ceil_div(E, 256), split ? kRouterBlocks : 1);
#define MOE_WIDE(VECV, SPLITV)                                                                   \
  do {                                                                                           \
    cudaFuncSetAttribute(router_wide_kernel<VECV, SPLITV>,                                        \
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                 \
    router_wide_kernel<VECV, SPLITV><<<grid, 256, smem, s>>>(xp, wp, bias, T, H, E, logits, part); \
  } while (0)
  if (E % 8 == 0) {
    if (split) MOE_WIDE(true, true);
    else MOE_WIDE(true, false);
  } else {
    if (split) MOE_WIDE(false, true);
    else MOE_WIDE(false, false);
  }
#undef MOE_WIDE
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_topk_part(logits, split ? part : nullptr, bias, T, E, k, ids, w, s);
}

// Selection of the top k of each token's E logits (a warp per token); with
// `part`, the logits are first formed from the split kernel's block sums.
cudaError_t launch_topk_part(float* logits, const float* part, const float* bias, int T, int E,
                             int k, int32_t* ids, float* w, cudaStream_t s) {
  int per = (E + 31) / 32;
  dim3 grid((unsigned)ceil_div((int64_t)T * 32, 256));
#define MOE_TOPK(P)                                                              \
  do {                                                                           \
    if (part) topk_kernel<P, true><<<grid, 256, 0, s>>>(logits, part, bias, T, E, k, ids, w); \
    else topk_kernel<P, false><<<grid, 256, 0, s>>>(logits, nullptr, nullptr, T, E, k, ids, w); \
  } while (0)
  if (per <= 1)
    MOE_TOPK(1);
  else if (per <= 2)
    MOE_TOPK(2);
  else if (per <= 4)
    MOE_TOPK(4);
  else if (per <= 8)
    MOE_TOPK(8);
  else if (per <= 16)
    MOE_TOPK(16);
  else
    MOE_TOPK(32);
#undef MOE_TOPK
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                        cudaStream_t s) {
  return launch_topk_part(const_cast<float*>(logits), nullptr, nullptr, T, E, k, ids, w, s);
}

}  // namespace moe
