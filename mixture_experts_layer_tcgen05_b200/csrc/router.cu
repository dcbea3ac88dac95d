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
#include "common.cuh"

namespace moe {

constexpr int kRouterKC = 64;  // h values staged per shared-memory chunk

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

// blockDim.x = NE * NTT threads; thread (te_grp = tid % NE, tt_grp = tid / NE)
// owns experts e0 + te_grp*TE + [0,TE) and tokens t0 + tt_grp*TT + [0,TT).
template <int TE, int TT>
__global__ void __launch_bounds__(256) router_logits_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const __nv_bfloat16* __restrict__ wr,
                                                            const float* __restrict__ bias, int T,
                                                            int H, int E, int NE, int NTT,
                                                            float* __restrict__ logits) {
  const int EC = NE * TE;   // experts per block
  const int BT = NTT * TT;  // tokens per block
  extern __shared__ __align__(16) unsigned char router_smem[];
  // xs[h][t] (token contiguous) and ws[h][e] (expert contiguous), bf16 bits
  uint16_t* xs = reinterpret_cast<uint16_t*>(router_smem);
  uint16_t* ws = xs + kRouterKC * BT;

  const int tid = threadIdx.x;
  const int te_grp = tid % NE, tt_grp = tid / NE;
  const int t0 = blockIdx.x * BT;
  const int e0 = blockIdx.y * EC;
  const uint16_t* xg = reinterpret_cast<const uint16_t*>(x);
  const uint16_t* wg = reinterpret_cast<const uint16_t*>(wr);

  float acc[TT][TE];
#pragma unroll
  for (int a = 0; a < TT; ++a)
#pragma unroll
    for (int b = 0; b < TE; ++b) acc[a][b] = 0.0f;

  const int nthreads = NE * NTT;
  for (int k0 = 0; k0 < H; k0 += kRouterKC) {
    // stage x[t0.., k0..k0+KC) transposed, 8 bf16 (16 B) per load
    for (int i = tid; i < BT * (kRouterKC / 8); i += nthreads) {
      int t = i / (kRouterKC / 8), c8 = (i % (kRouterKC / 8)) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t0 + t < T) v = *reinterpret_cast<const uint4*>(xg + (int64_t)(t0 + t) * H + k0 + c8);
      const uint16_t* pv = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
      for (int j = 0; j < 8; ++j) xs[(c8 + j) * BT + t] = pv[j];
    }
    // stage wr[k0.., e0..e0+EC), zero beyond E
    for (int i = tid; i < kRouterKC * EC; i += nthreads) {
      int h = i / EC, e = i % EC;
      ws[h * EC + e] = (e0 + e < E) ? wg[(int64_t)(k0 + h) * E + e0 + e] : (uint16_t)0;
    }
    __syncthreads();
#pragma unroll 4
    for (int h = 0; h < kRouterKC; ++h) {
      float xv[TT], wv[TE];
      const uint16_t* xp = xs + h * BT + tt_grp * TT;
      const uint16_t* wp = ws + h * EC + te_grp * TE;
      load_bf16_vec<TT>(xp, xv);
      load_bf16_vec<TE>(wp, wv);
#pragma unroll
      for (int a = 0; a < TT; ++a)
#pragma unroll
        for (int b = 0; b < TE; ++b) acc[a][b] = __fmaf_rn(xv[a], wv[b], acc[a][b]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < TT; ++a) {
    int t = t0 + tt_grp * TT + a;
    if (t >= T) continue;
#pragma unroll
    for (int b = 0; b < TE; ++b) {
      int e = e0 + te_grp * TE + b;
      if (e < E) logits[(int64_t)t * E + e] = __fadd_rn(acc[a][b], bias ? bias[e] : 0.0f);
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

struct RouterShape {
  int TE, TT, NE, NTT;
};

static RouterShape router_shape(int E) {
  if (E <= 32) return {8, 1, (E + 7) / 8, 64};
  int ne = (E + 7) / 8;
  if (ne > 32) ne = 32;
  return {8, 4, ne, 256 / ne};
}

cudaError_t launch_router_logits(const void* x, const void* wr, const float* bias, int T, int H,
                                 int E, float* logits, cudaStream_t s) {
  RouterShape rs = router_shape(E);
  int EC = rs.NE * rs.TE, BT = rs.NTT * rs.TT;
  dim3 grid((unsigned)ceil_div(T, BT), (unsigned)ceil_div(E, EC));
  size_t smem = (size_t)kRouterKC * (BT + EC) * 2;
  int threads = rs.NE * rs.NTT;
  const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(x);
  const __nv_bfloat16* wp = static_cast<const __nv_bfloat16*>(wr);
  if (rs.TT == 1)
    router_logits_kernel<8, 1><<<grid, threads, smem, s>>>(xp, wp, bias, T, H, E, rs.NE, rs.NTT,
                                                           logits);
  else
    router_logits_kernel<8, 4><<<grid, threads, smem, s>>>(xp, wp, bias, T, H, E, rs.NE, rs.NTT,
                                                           logits);
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
