// Router: logits GEMV and softmax top-k selection with renormalised weights.
//
// "Mixture of Experts (MoE): a practical explanation of how expert models
// work" (lira-now.com), section 5, steps 1-5 and its pseudocode: the router
// maps each token vector to E logits, softmax turns them into probabilities,
// the k largest are kept and renormalised over the selected experts.
//
// The logits decide integers (the selected ids), so they are computed in a
// fixed order: one fp32 accumulator per (token, expert), h ascending, one
// fused multiply-add per term. A bf16 x bf16 product is exact in fp32, so the
// FMA equals the rounded sum of the exact product and every logit is a fixed
// function of the inputs. The work is register-tiled on CUDA cores (each
// thread owns TT tokens x TE experts); tensor cores are not used here because
// their internal accumulation order is not specified.
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
// fmas per instruction), so each (token, expert) sum is still one fp32 fma
// per h in ascending order.
constexpr int kWideKC = 32;

template <bool VEC>
__global__ void __launch_bounds__(256, 2) router_wide_kernel(const __nv_bfloat16* __restrict__ x,
                                                             const __nv_bfloat16* __restrict__ wr,
                                                             const float* __restrict__ bias,
                                                             int T, int H, int E,
                                                             float* __restrict__ logits) {
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

  // acc[a][p] holds experts (2p, 2p+1) of token a
  float2 acc[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int p = 0; p < 4; ++p) acc[a][p] = make_float2(0.0f, 0.0f);
  const int nchunks = H / KC;
  load(0);
  store(0);
  __syncthreads();
  for (int c = 0; c < nchunks; ++c) {
    const int b = c & 1;
    if (c + 1 < nchunks) load((c + 1) * KC);
    const float* xb = xs + b * KC * BT + tok0;
    const float* wb = ws + b * KC * EC + eg * 4;
#pragma unroll 4
    for (int h = 0; h < KC; ++h) {
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
      if (ee < E) logits[(int64_t)t * E + ee] = __fadd_rn(acc[a][p].x, bias ? bias[ee] : 0.0f);
      if (ee + 1 < E) logits[(int64_t)t * E + ee + 1] = __fadd_rn(acc[a][p].y, bias ? bias[ee + 1] : 0.0f);
    }
  }
}

// One warp per token. Lane l holds logits e = l + 32*i. k rounds of a warp
// argmax on (logit desc, index asc); slot j gets the j-th winner. Weights:
// w_j = exp(l_j - l_max) / sum_selected exp(l_i - l_max).
template <int PER>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E,
                                                   int k, int32_t* __restrict__ ids,
                                                   float* __restrict__ w) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  const float* l = logits + (int64_t)warp * E;
  float v[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    int e = lane + 32 * i;
    v[i] = e < E ? l[e] : -INFINITY;
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

// Narrow router (E <= 32). One thread per (token, expert): one sequential
// sum each, so a block of 64 threads covers 64/EP tokens (EP = E padded to a
// power of two) and the T*E sums spread over as many warps as possible.
// These kernels are latency-bound, so nothing global sits on the critical
// path: the whole of Wr (bf16, [h][expert], rows padded to EP) is loaded into
// shared memory once, and the token rows stream through an NS-deep ring of
// cp.async copies, so each chunk of x landed long before its sums need it.
constexpr int kNarrowKC = 64;  // h per x chunk
constexpr int kNarrowNS = 8;   // x chunks in flight

template <int EP>  // experts per token, padded to a power of two (1..32)
__global__ void __launch_bounds__(64) router_narrow_kernel(const __nv_bfloat16* __restrict__ x,
                                                           const __nv_bfloat16* __restrict__ wr,
                                                           const float* __restrict__ bias, int T,
                                                           int H, int E,
                                                           float* __restrict__ logits) {
  constexpr int BT = 64 / EP;          // tokens per block
  constexpr int XROW = kNarrowKC * 2;  // bytes of one token's chunk
  constexpr int XSTAGE = BT * XROW;    // bytes of one ring stage
  extern __shared__ __align__(16) unsigned char narrow_smem[];
  unsigned char* xring = narrow_smem;                                              // [NS][BT][KC] bf16
  uint16_t* wsm = reinterpret_cast<uint16_t*>(narrow_smem + kNarrowNS * XSTAGE);  // [H][EP] bf16
  const int tid = threadIdx.x;
  const int e = tid % EP, tl = tid / EP;
  const int t0 = blockIdx.x * BT;
  const int nchunks = H / kNarrowKC;
  const char* xg = reinterpret_cast<const char*>(x);
  const uint16_t* wg = reinterpret_cast<const uint16_t*>(wr);

  // x chunk c -> ring stage c % NS: BT rows x 128 B, as 16-byte copies
  auto issue = [&](int c) {
    if (c < nchunks) {
      const uint32_t st = ptx::smem_addr(xring + (c % kNarrowNS) * XSTAGE);
      for (int i = tid; i < BT * (XROW / 16); i += 64) {
        const int r = i / (XROW / 16), v = i % (XROW / 16);
        const int t = t0 + r;
        const char* src = xg + ((int64_t)(t < T ? t : 0) * H + (int64_t)c * kNarrowKC) * 2 + v * 16;
        ptx::cp_async16(st + r * XROW + v * 16, src, t < T ? 16u : 0u);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
#pragma unroll
  for (int c = 0; c < kNarrowNS - 1; ++c) issue(c);
  // Wr -> shared memory, once. When the padded layout equals Wr's own (E = EP,
  // rows of 16-byte multiples) it is one stream of asynchronous copies.
  if (E == EP && (E * 2) % 16 == 0) {
    const uint32_t wdst = ptx::smem_addr(wsm);
    const char* wsrc = reinterpret_cast<const char*>(wr);
    for (int i = tid; i < H * E * 2 / 16; i += 64) ptx::cp_async16(wdst + i * 16, wsrc + i * 16, 16u);
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else {
    for (int i = tid; i < H * EP; i += 64) {
      const int h = i / EP, ee = i % EP;
      wsm[i] = ee < E ? wg[(int64_t)h * E + ee] : (uint16_t)0;
    }
  }
  float acc = 0.0f;
  for (int c = 0; c < nchunks; ++c) {
    issue(c + kNarrowNS - 1);
    asm volatile("cp.async.wait_group %0;" ::"n"(kNarrowNS - 1) : "memory");
    __syncthreads();  // chunk c (and, the first time, Wr) visible to all threads
    const uint4* xs = reinterpret_cast<const uint4*>(xring + (c % kNarrowNS) * XSTAGE + tl * XROW);
    const uint16_t* wc = wsm + (int64_t)c * kNarrowKC * EP + e;
#pragma unroll
    for (int v = 0; v < kNarrowKC / 8; ++v) {
      const uint4 u = xs[v];
      const float xf[8] = {bf16lo_to_f32(u.x), bf16hi_to_f32(u.x), bf16lo_to_f32(u.y), bf16hi_to_f32(u.y),
                           bf16lo_to_f32(u.z), bf16hi_to_f32(u.z), bf16lo_to_f32(u.w), bf16hi_to_f32(u.w)};
#pragma unroll
      for (int j = 0; j < 8; ++j)
        acc = __fmaf_rn(xf[j], __uint_as_float((uint32_t)wc[(v * 8 + j) * EP] << 16), acc);
    }
    __syncthreads();  // stage c % NS is refilled by the next iteration's issue
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  const int t = t0 + tl;
  if (t < T && e < E) logits[(int64_t)t * E + e] = __fadd_rn(acc, bias ? bias[e] : 0.0f);
}

template <int EP>
size_t narrow_smem_bytes(int H) {
  return (size_t)kNarrowNS * (64 / EP) * kNarrowKC * 2 + (size_t)H * EP * 2;
}

cudaError_t launch_router_logits(const void* x, const void* wr, const float* bias, int T, int H,
                                 int E, float* logits, cudaStream_t s) {
  const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(x);
  const __nv_bfloat16* wp = static_cast<const __nv_bfloat16*>(wr);
  if (E <= 32) {
    const int ep = E <= 1 ? 1 : E <= 2 ? 2 : E <= 4 ? 4 : E <= 8 ? 8 : E <= 16 ? 16 : 32;
    // the whole of Wr must fit in shared memory next to the x ring
    const size_t need = ep == 1 ? narrow_smem_bytes<1>(H) : ep == 2 ? narrow_smem_bytes<2>(H)
                        : ep == 4 ? narrow_smem_bytes<4>(H) : ep == 8 ? narrow_smem_bytes<8>(H)
                        : ep == 16 ? narrow_smem_bytes<16>(H) : narrow_smem_bytes<32>(H);
    if (need <= 200 * 1024) {
#define MOE_NARROW(EPV)                                                                        \
  do {                                                                                         \
    cudaFuncSetAttribute(router_narrow_kernel<EPV>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                         (int)need);                                                           \
    router_narrow_kernel<EPV><<<(unsigned)ceil_div(T, 64 / EPV), 64, need, s>>>(xp, wp, bias, T, H, \
                                                                               E, logits);     \
  } while (0)
      if (ep == 1) MOE_NARROW(1);
      else if (ep == 2) MOE_NARROW(2);
      else if (ep == 4) MOE_NARROW(4);
      else if (ep == 8) MOE_NARROW(8);
      else if (ep == 16) MOE_NARROW(16);
      else MOE_NARROW(32);
#undef MOE_NARROW
      note_launch();
      return cudaGetLastError();
    }
  }
  const size_t smem = 2 * (size_t)kWideKC * (64 + 256) * 4;
  dim3 grid((unsigned)ceil_div(T, 64), (unsigned)ceil_div(E, 256));
  if (E % 8 == 0) {
    cudaFuncSetAttribute(router_wide_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    router_wide_kernel<true><<<grid, 256, smem, s>>>(xp, wp, bias, T, H, E, logits);
  } else {
    cudaFuncSetAttribute(router_wide_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    router_wide_kernel<false><<<grid, 256, smem, s>>>(xp, wp, bias, T, H, E, logits);
  }
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                        cudaStream_t s) {
  int per = (E + 31) / 32;
  dim3 grid((unsigned)ceil_div((int64_t)T * 32, 256));
#define MOE_TOPK(P) topk_kernel<P><<<grid, 256, 0, s>>>(logits, T, E, k, ids, w)
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

}  // namespace moe
