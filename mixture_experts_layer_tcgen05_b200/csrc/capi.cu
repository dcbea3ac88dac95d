// C ABI of the MoE layer (include/moe.h): argument validation, workspace
// layout, device check and the launch sequence of each entry point. Every
// step of the layer runs in this library's kernels; nothing here computes
// on the host.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "common.cuh"
#include "permute.cuh"

namespace moe {

// kernels (router.cu, permute.cu, gemm.cu, fp8.cu)
cudaError_t launch_route(const void* x, const void* wr, const float* bias, int T, int H, int E,
                         int k, float* logits, int32_t* ids, float* w, float* part,
                         size_t part_bytes, cudaStream_t s);
cudaError_t launch_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                        cudaStream_t s);
int64_t permute_scratch_bytes(int T, int E);
cudaError_t launch_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets,
                           int32_t* perm_token, int32_t* inv_perm, void* scratch, int32_t* status,
                           cudaStream_t s);
cudaError_t launch_gather_rows(const void* x, const int32_t* perm_token, int R, int T,
                               int row_bytes, void* x_perm, int32_t* status, cudaStream_t s);
cudaError_t launch_scatter_rows(const void* x, const int32_t* inv_perm, int T, int k,
                                int row_bytes, void* x_perm, int32_t* status, cudaStream_t s);
cudaError_t launch_permute_gather_small(const int32_t* ids, int T, int E, int k, int32_t* offsets,
                                        int32_t* perm_token, int32_t* inv_perm, const void* x,
                                        int row_bytes, void* x_perm, const void* x2,
                                        int row2_bytes, void* x2_perm, int32_t* status,
                                        cudaStream_t s);
cudaError_t launch_combine(const void* y_perm, const float* w, const int32_t* inv_perm, int T,
                           int H, int k, void* out, int32_t* status, cudaStream_t s);
cudaError_t launch_grouped_gemm_bf16(const void* A, const int32_t* A_rows, int A_src_rows,
                                     const void* B, const int32_t* offsets, int M_total, int E,
                                     int N, int K, int act, void* C,
                                     int max_rows_per_expert, int32_t* status, void* scratch,
                                     size_t scratch_bytes, cudaStream_t s, const char** why);
cudaError_t launch_grouped_gemm_fp8(const void* A, const int32_t* A_rows, int A_src_rows,
                                    const float* a_scales, const void* B, const float* b_scales,
                                    const int32_t* offsets, int M_total, int E, int N, int K,
                                    int act, void* C, float* c_scales,
                                    int max_rows_per_expert, int32_t* status, cudaStream_t s,
                                    const char** why);
cudaError_t launch_grouped_gemm_mx(const void* A, const float* a_scales, const void* B,
                                   const float* b_scales, const uint8_t* b_sf8,
                                   const int32_t* offsets, int M_total, int E, int N, int K, int act,
                                   void* Cout, float* c_scales, int32_t* status, cudaStream_t s,
                                   const char** why);
cudaError_t launch_wait_selftest(int32_t* status, long long budget, cudaStream_t s);
cudaError_t launch_grouped_gemm_mx_swap(const void* A, const float* a_scales, const void* B,
                                        const float* b_scales, const uint8_t* b_sf8,
                                        const int32_t* offsets, int M_total, int E, int N, int K,
                                        int act, void* Cout, float* c_scales, int max_rows,
                                        int32_t* status, cudaStream_t s, const char** why);
cudaError_t launch_quant_weight_fp4(const void* w, int64_t nb, int64_t rows, int64_t cols, void* q,
                                    uint8_t* sc, cudaStream_t s);
cudaError_t launch_quant_act(const void* x, int64_t rows, int64_t cols, void* q, float* sc,
                             const int32_t* row_map, bool ue8m0, cudaStream_t s);
cudaError_t launch_quant_act_scatter(const void* x, int64_t rows, int64_t cols,
                                     const int32_t* inv_perm, int k, void* q_perm, float* sc_perm,
                                     bool ue8m0, int32_t* status, cudaStream_t s);
cudaError_t launch_quant_weight(const void* w, int64_t nb, int64_t rows, int64_t cols, void* q,
                                float* sc, bool ue8m0, cudaStream_t s);

int64_t ep_plan_ints(int E, int G);
cudaError_t launch_ep_plan(const int32_t* cnt, int G, int E, int rank, int32_t* plan, cudaStream_t s);
cudaError_t launch_ep_dispatch(const void* x_perm, const int32_t* offsets, const int32_t* plan,
                               int E, int G, int R, int row_bytes, const uint64_t* dst_bufs,
                               int64_t dst_rows, int32_t* status, cudaStream_t s);
cudaError_t launch_ep_return(const void* y_loc, const int32_t* plan, int E, int G, int64_t cap,
                             int row_bytes, const uint64_t* src_bufs, int64_t src_rows,
                             int32_t* status, cudaStream_t s);
cudaError_t launch_pack_weights(const void* wg, const void* wu, const void* wd, int E, int H,
                                int I, void* w13, void* w2, cudaStream_t s);

int64_t noalloc_scratch_capacity();
cudaError_t launch_permute_noalloc(const int32_t* ids, int T, int H, int E, int k, int32_t* offsets,
                                   int32_t* perm_token, int32_t* inv_perm, const void* x,
                                   void* x_perm, cudaStream_t s);
cudaError_t noalloc_status(int32_t* out, bool clear);

static std::atomic<int64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

}  // namespace moe

using namespace moe;

namespace {

thread_local std::string t_err;
thread_local void* t_events[6] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
thread_local bool t_events_on = false;

moe_status_t fail(moe_status_t st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
moe_status_t fail(moe_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_err = buf;
  return st;
}

moe_status_t ok() {
  t_err.clear();
  return MOE_OK;
}

moe_status_t cuda_fail(cudaError_t e, const char* where) {
  return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t check_dims(moe_dims_t d, bool need_I) {
  if (d.T < 1) return fail(MOE_ERR_INVALID_ARG, "T must be >= 1 (got %d)", d.T);
  if (d.H < 128 || d.H % 128)
    return fail(MOE_ERR_INVALID_ARG, "H must be a positive multiple of 128 (got %d)", d.H);
  if (need_I && (d.I < 128 || d.I % 128))
    return fail(MOE_ERR_INVALID_ARG, "I must be a positive multiple of 128 (got %d)", d.I);
  if (d.E < 1 || d.E > 1024) return fail(MOE_ERR_INVALID_ARG, "E must be in [1, 1024] (got %d)", d.E);
  if (d.k < 1 || d.k > 16 || d.k > d.E)
    return fail(MOE_ERR_INVALID_ARG, "k must be in [1, min(E, 16)] (got k=%d, E=%d)", d.k, d.E);
  if ((int64_t)d.T * d.k >= (int64_t)1 << 31)
    return fail(MOE_ERR_INVALID_ARG, "T*k must be < 2^31");
  return MOE_OK;
}

moe_status_t check_ptr(const void* p, const char* name, bool allow_null = false) {
  if (!p) {
    if (allow_null) return MOE_OK;
    return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
  }
  if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return MOE_OK;
}

#define MOE_TRY(x)                      \
  do {                                  \
    moe_status_t _st = (x);             \
    if (_st != MOE_OK) return _st;      \
  } while (0)

moe_status_t check_device() {
  const char* fake = getenv("MOE_FAKE_CC");
  int major = 0, minor = 0;
  if (fake) {
    major = atoi(fake) / 10;
    minor = atoi(fake) % 10;
  } else {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(MOE_ERR_UNSUPPORTED_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
    static int cache_major[64] = {0}, cache_minor[64] = {0};
    if (dev < 64 && cache_major[dev]) {
      major = cache_major[dev];
      minor = cache_minor[dev];
    } else {
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
      if (dev < 64) {
        cache_major[dev] = major;
        cache_minor[dev] = minor;
      }
    }
  }
  if (major != 10 || minor != 0)
    return fail(MOE_ERR_UNSUPPORTED_DEVICE,
                "this library is built for sm_100a (compute capability 10.0); device is %d.%d",
                major, minor);
  return MOE_OK;
}

// Workspace layout shared by every entry point.
moe_ws_layout_t layout(moe_dims_t d, moe_dtype_t dt) {
  moe_ws_layout_t L;
  int64_t off = 0;
  auto take = [&](int64_t bytes) {
    int64_t o = off;
    off += align_up(bytes > 0 ? bytes : 0, 256);
    return o;
  };
  const int64_t T = d.T, H = d.H, I = d.I, E = d.E, k = d.k, R = T * k;
  L.status = take(256);
  L.logits = take(T * E * 4);
  L.topk_ids = take(R * 4);
  L.topk_w = take(R * 4);
  L.offsets = take((E + 1) * 4);
  L.perm_token = take(R * 4);
  L.inv_perm = take(R * 4);
  L.scratch = take(permute_scratch_bytes((int)T, (int)E));
  if (dt == MOE_DTYPE_BF16) {
    L.x_perm = take(R * H * 2);
    L.xq = L.xs = L.xq_perm = L.xs_perm = -1;
    L.h = take(R * I * 2);
    L.hq = L.hs = -1;
    // split-K partials of the small-M (decode) kernels: up to 8 fp32 slices
    L.splitk = T <= 64 ? take(8 * R * std::max(2 * I, H) * 4) : -1;
  } else {
    L.x_perm = -1;
    L.xq = take(T * H);
    L.xs = take(T * (H / 128) * 4);
    L.xq_perm = take(R * H);
    L.xs_perm = take(R * (H / 128) * 4);
    L.h = -1;
    L.hq = take(R * I);
    L.hs = take(R * (I / 128) * 4);
    L.splitk = -1;
  }
  L.y_perm = take(R * H * 2);
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, int64_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

void record(cudaStream_t s, int i) {
  if (t_events_on && t_events[i]) cudaEventRecord(static_cast<cudaEvent_t>(t_events[i]), s);
}

moe_status_t check_ws(moe_dims_t d, moe_dtype_t dt, const void* ws, size_t ws_bytes,
                      size_t extra = 0) {
  MOE_TRY(check_ptr(ws, "ws"));
  size_t need = (size_t)layout(d, dt).total + extra;
  if (ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_last_error(void) { return t_err.c_str(); }

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

int64_t moe_launch_count(void) { return g_launches.load(); }

size_t moe_workspace_size(moe_dims_t d, moe_dtype_t dt) {
  if (check_dims(d, true) != MOE_OK) return 0;
  if (dt < MOE_DTYPE_BF16 || dt > MOE_DTYPE_FP4_E2M1) return 0;
  return (size_t)layout(d, dt).total;
}

moe_status_t moe_workspace_layout(moe_dims_t d, moe_dtype_t dt, moe_ws_layout_t* out) {
  MOE_TRY(check_dims(d, true));
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  if (dt < MOE_DTYPE_BF16 || dt > MOE_DTYPE_FP4_E2M1) return fail(MOE_ERR_INVALID_ARG, "bad dtype");
  *out = layout(d, dt);
  return ok();
}

moe_status_t moe_route_topk(const void* x, const void* wr, const float* bias, moe_dims_t d,
                            float* logits, int32_t* ids, float* w, void* ws, size_t ws_bytes,
                            void* stream) {
  MOE_TRY(check_dims(d, false));
  MOE_TRY(check_ptr(x, "x"));
  MOE_TRY(check_ptr(wr, "w_router"));
  MOE_TRY(check_ptr(bias, "bias", true));
  MOE_TRY(check_ptr(logits, "logits", true));
  MOE_TRY(check_ptr(ids, "topk_ids"));
  MOE_TRY(check_ptr(w, "topk_w"));
  if (!logits) {
    moe_dims_t d2 = d;
    d2.I = 128;
    MOE_TRY(check_ws(d2, MOE_DTYPE_BF16, ws, ws_bytes));
    logits = at<float>(ws, layout(d2, MOE_DTYPE_BF16).logits);
  }
  MOE_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_route(x, wr, bias, d.T, d.H, d.E, d.k, logits, ids, w, nullptr, 0, s);
  if (e != cudaSuccess) return cuda_fail(e, "router");
  return ok();
}

moe_status_t moe_topk_from_logits(const float* logits, moe_dims_t d, int32_t* ids, float* w,
                                  void* stream) {
  if (d.T < 1 || d.E < 1 || d.E > 1024 || d.k < 1 || d.k > 16 || d.k > d.E)
    return fail(MOE_ERR_INVALID_ARG, "bad dims (T=%d E=%d k=%d)", d.T, d.E, d.k);
  MOE_TRY(check_ptr(logits, "logits"));
  MOE_TRY(check_ptr(ids, "topk_ids"));
  MOE_TRY(check_ptr(w, "topk_w"));
  MOE_TRY(check_device());
  cudaError_t e = launch_topk(logits, d.T, d.E, d.k, ids, w, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "top-k");
  return ok();
}

moe_status_t moe_permute(const int32_t* ids, moe_dims_t d, int32_t* offsets, int32_t* perm_token,
                         int32_t* inv_perm, const void* x, void* x_perm, void* ws,
                         size_t ws_bytes, void* stream) {
  moe_dims_t d2 = d;
  if (d2.I < 128) d2.I = 128;
  MOE_TRY(check_dims(d2, true));
  MOE_TRY(check_ptr(ids, "topk_ids"));
  MOE_TRY(check_ptr(offsets, "expert_offsets"));
  MOE_TRY(check_ptr(perm_token, "perm_token"));
  MOE_TRY(check_ptr(inv_perm, "inv_perm"));
  if ((x == nullptr) != (x_perm == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "x and x_perm must both be given or both be NULL");
  MOE_TRY(check_ptr(x, "x", true));
  MOE_TRY(check_ptr(x_perm, "x_perm", true));
  MOE_TRY(check_ws(d2, MOE_DTYPE_BF16, ws, ws_bytes));
  MOE_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  moe_ws_layout_t L = layout(d2, MOE_DTYPE_BF16);
  // decode-sized batches: one launch for the permutation and the gather
  cudaError_t e = launch_permute_gather_small(ids, d.T, d.E, d.k, offsets, perm_token, inv_perm, x,
                                              d.H * 2, x_perm, nullptr, 0, nullptr,
                                              at<int32_t>(ws, L.status), s);
  if (e == cudaSuccess) return ok();
  if (e != cudaErrorNotSupported) return cuda_fail(e, "permute");
  e = launch_permute(ids, d.T, d.E, d.k, offsets, perm_token, inv_perm,
                     at<char>(ws, L.scratch), at<int32_t>(ws, L.status), s);
  if (e != cudaSuccess) return cuda_fail(e, "permute");
  if (x) {
    e = launch_scatter_rows(x, inv_perm, d.T, d.k, d.H * 2, x_perm, at<int32_t>(ws, L.status), s);
    if (e != cudaSuccess) return cuda_fail(e, "row scatter");
  }
  return ok();
}

moe_status_t moe_permute_noalloc(const int32_t* ids, moe_dims_t d, int32_t* offsets,
                                 int32_t* perm_token, int32_t* inv_perm, const void* x,
                                 void* x_perm, void* stream) {
  moe_dims_t d2 = d;
  if (d2.I < 128) d2.I = 128;
  MOE_TRY(check_dims(d2, true));
  MOE_TRY(check_ptr(ids, "topk_ids"));
  MOE_TRY(check_ptr(offsets, "expert_offsets"));
  MOE_TRY(check_ptr(perm_token, "perm_token"));
  MOE_TRY(check_ptr(inv_perm, "inv_perm"));
  if ((x == nullptr) != (x_perm == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "x and x_perm must both be given or both be NULL");
  MOE_TRY(check_ptr(x, "x", true));
  MOE_TRY(check_ptr(x_perm, "x_perm", true));
  const int64_t need = permute_scratch_bytes(d.T, d.E);
  if (need > noalloc_scratch_capacity())
    return fail(MOE_ERR_INVALID_ARG,
                "T=%d, E=%d need %lld bytes of permutation scratch; the fixed array holds %lld "
                "(MOE_NOALLOC_SCRATCH_BYTES); use moe_permute with a workspace",
                d.T, d.E, (long long)need, (long long)noalloc_scratch_capacity());
  MOE_TRY(check_device());
  cudaError_t e = launch_permute_noalloc(ids, d.T, d.H, d.E, d.k, offsets, perm_token, inv_perm, x,
                                         x_perm, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "permute (fixed scratch)");
  return ok();
}

moe_status_t moe_permute_noalloc_status(int32_t* status_out, int32_t clear) {
  if (!status_out) return fail(MOE_ERR_INVALID_ARG, "status_out is NULL");
  MOE_TRY(check_device());
  cudaError_t e = noalloc_status(status_out, clear != 0);
  if (e != cudaSuccess) return cuda_fail(e, "read the fixed array's status word");
  return ok();
}

moe_status_t moe_grouped_gemm(const void* A, const int32_t* a_rows, int32_t a_src_rows,
                              const void* B, const int32_t* offsets,
                              int32_t M_total, int32_t E, int32_t N, int32_t K, moe_dtype_t dt,
                              moe_epilogue_t ep, void* C, const float* a_scales,
                              const float* b_scales, float* c_scales, int32_t max_rows_per_expert,
                              void* ws, size_t ws_bytes, void* stream) {
  if (M_total < 1) return fail(MOE_ERR_INVALID_ARG, "M_total must be >= 1");
  if (E < 1 || E > 1024) return fail(MOE_ERR_INVALID_ARG, "E must be in [1, 1024]");
  if (N < 128 || N % 128 || K < 128 || K % 128)
    return fail(MOE_ERR_INVALID_ARG, "N and K must be positive multiples of 128 (N=%d K=%d)", N, K);
  if (ep < MOE_EPILOGUE_NONE || ep > MOE_EPILOGUE_REGLU) return fail(MOE_ERR_INVALID_ARG, "bad epilogue");
  if (dt == MOE_DTYPE_FP4_E2M1)
    return fail(MOE_ERR_INVALID_ARG, "FP4 weights take moe_grouped_gemm_fp4 (e8m0 scale bytes)");
  if (dt < MOE_DTYPE_BF16 || dt > MOE_DTYPE_FP8_E4M3_UE8M0) return fail(MOE_ERR_INVALID_ARG, "bad dtype");
  if (dt == MOE_DTYPE_FP8_E4M3_UE8M0 && a_rows)
    return fail(MOE_ERR_INVALID_ARG, "the block-scaled GEMM takes no row gather");
  MOE_TRY(check_ptr(A, "A"));
  MOE_TRY(check_ptr(a_rows, "a_rows", true));
  if (a_rows && a_src_rows < 1) return fail(MOE_ERR_INVALID_ARG, "a_src_rows must be >= 1 with a_rows");
  MOE_TRY(check_ptr(B, "B"));
  MOE_TRY(check_ptr(offsets, "expert_offsets"));
  MOE_TRY(check_ptr(C, "C"));
  if (dt != MOE_DTYPE_BF16) {
    MOE_TRY(check_ptr(a_scales, "a_scales"));
    MOE_TRY(check_ptr(b_scales, "b_scales"));
    MOE_TRY(check_ptr(c_scales, "c_scales", true));
    if (c_scales && ep == MOE_EPILOGUE_NONE)
      return fail(MOE_ERR_INVALID_ARG, "c_scales (quantised output) needs a gated epilogue");
  }
  MOE_TRY(check_ptr(ws, "ws"));
  if (ws_bytes < 256) return fail(MOE_ERR_WORKSPACE, "workspace too small: %zu bytes", ws_bytes);
  MOE_TRY(check_device());
  const char* why = "";
  cudaError_t e;
  if (dt == MOE_DTYPE_BF16)
    e = launch_grouped_gemm_bf16(A, a_rows, a_rows ? a_src_rows : M_total, B, offsets, M_total, E,
                                 N, K, (int)ep, C,
                                 max_rows_per_expert, at<int32_t>(ws, 0), at<char>(ws, 256),
                                 ws_bytes - 256, static_cast<cudaStream_t>(stream), &why);
  else if (dt == MOE_DTYPE_FP8_E4M3)
    e = launch_grouped_gemm_fp8(A, a_rows, a_rows ? a_src_rows : M_total, a_scales, B, b_scales,
                                offsets, M_total, E, N, K,
                                (int)ep, C, c_scales, max_rows_per_expert,
                                at<int32_t>(ws, 0), static_cast<cudaStream_t>(stream), &why);
  else if (max_rows_per_expert > 0 && max_rows_per_expert <= 64)  // decode sizes: weights in M
    e = launch_grouped_gemm_mx_swap(A, a_scales, B, b_scales, nullptr, offsets, M_total, E, N, K,
                                    (int)ep, C, c_scales, max_rows_per_expert, at<int32_t>(ws, 0),
                                    static_cast<cudaStream_t>(stream), &why);
  else
    e = launch_grouped_gemm_mx(A, a_scales, B, b_scales, nullptr, offsets, M_total, E, N, K,
                               (int)ep, C, c_scales, at<int32_t>(ws, 0),
                               static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "grouped GEMM: %s %s", cudaGetErrorString(e), why);
  return ok();
}

moe_status_t moe_grouped_gemm_fp4(const void* A, const float* a_scales, const void* B,
                                  const uint8_t* b_scales, const int32_t* offsets, int32_t M_total,
                                  int32_t E, int32_t N, int32_t K, moe_epilogue_t ep, void* C,
                                  float* c_scales, int32_t max_rows_per_expert, void* ws,
                                  size_t ws_bytes, void* stream) {
  if (M_total < 1) return fail(MOE_ERR_INVALID_ARG, "M_total must be >= 1");
  if (E < 1 || E > 1024) return fail(MOE_ERR_INVALID_ARG, "E must be in [1, 1024]");
  if (N < 128 || N % 128 || K < 128 || K % 128)
    return fail(MOE_ERR_INVALID_ARG, "N and K must be positive multiples of 128 (N=%d K=%d)", N, K);
  if (ep < MOE_EPILOGUE_NONE || ep > MOE_EPILOGUE_REGLU) return fail(MOE_ERR_INVALID_ARG, "bad epilogue");
  const bool small = max_rows_per_expert > 0 && max_rows_per_expert <= 64;
  if (ep == MOE_EPILOGUE_NONE && N % 256 && !small)
    return fail(MOE_ERR_INVALID_ARG, "the plain tokens-in-M FP4 GEMM needs N %% 256 == 0 (N=%d)", N);
  MOE_TRY(check_ptr(A, "A"));
  MOE_TRY(check_ptr(a_scales, "a_scales"));
  MOE_TRY(check_ptr(B, "B"));
  if (reinterpret_cast<uintptr_t>(B) & 31) return fail(MOE_ERR_INVALID_ARG, "B must be 32-byte aligned");
  MOE_TRY(check_ptr(b_scales, "b_scales"));
  MOE_TRY(check_ptr(offsets, "expert_offsets"));
  MOE_TRY(check_ptr(C, "C"));
  MOE_TRY(check_ptr(c_scales, "c_scales", true));
  if (c_scales && ep == MOE_EPILOGUE_NONE)
    return fail(MOE_ERR_INVALID_ARG, "c_scales (quantised output) needs a gated epilogue");
  MOE_TRY(check_ptr(ws, "ws"));
  if (ws_bytes < 256) return fail(MOE_ERR_WORKSPACE, "workspace too small: %zu bytes", ws_bytes);
  MOE_TRY(check_device());
  const char* why = "";
  cudaError_t e =
      small
          ? launch_grouped_gemm_mx_swap(A, a_scales, B, nullptr, b_scales, offsets, M_total, E, N, K,
                                        (int)ep, C, c_scales, max_rows_per_expert, at<int32_t>(ws, 0),
                                        static_cast<cudaStream_t>(stream), &why)
          : launch_grouped_gemm_mx(A, a_scales, B, nullptr, b_scales, offsets, M_total, E, N, K,
                                   (int)ep, C, c_scales, at<int32_t>(ws, 0),
                                   static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "FP4 grouped GEMM: %s %s", cudaGetErrorString(e), why);
  return ok();
}

moe_status_t moe_gather_rows(const void* src, int64_t src_rows, const int32_t* rows, int64_t n,
                             int64_t row_bytes, void* dst, void* ws, void* stream) {
  if (n < 0 || src_rows < 0 || n > INT32_MAX || src_rows > INT32_MAX)
    return fail(MOE_ERR_INVALID_ARG, "n and src_rows must be in [0, 2^31)");
  if (row_bytes < 4 || row_bytes % 4 || row_bytes > (1 << 20))
    return fail(MOE_ERR_INVALID_ARG, "row_bytes must be a multiple of 4 in [4, 2^20] (got %lld)",
                (long long)row_bytes);
  if (n == 0) return ok();
  MOE_TRY(check_ptr(src, "src"));
  MOE_TRY(check_ptr(rows, "rows"));
  MOE_TRY(check_ptr(dst, "dst"));
  MOE_TRY(check_ptr(ws, "ws", true));
  MOE_TRY(check_device());
  cudaError_t e = launch_gather_rows(src, rows, (int)n, (int)src_rows, (int)row_bytes, dst,
                                     ws ? static_cast<int32_t*>(ws) : nullptr,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "row gather");
  return ok();
}

moe_status_t moe_combine(const void* y_perm, const float* w, const int32_t* inv_perm, moe_dims_t d,
                         void* out, void* stream) {
  moe_dims_t d2 = d;
  if (d2.I < 128) d2.I = 128;
  MOE_TRY(check_dims(d2, true));
  MOE_TRY(check_ptr(y_perm, "y_perm"));
  MOE_TRY(check_ptr(w, "topk_w"));
  MOE_TRY(check_ptr(inv_perm, "inv_perm"));
  MOE_TRY(check_ptr(out, "out"));
  MOE_TRY(check_device());
  cudaError_t e = launch_combine(y_perm, w, inv_perm, d.T, d.H, d.k, out, nullptr,
                                 static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "combine");
  return ok();
}

static moe_status_t forward_impl(const void* x, const void* wr, const float* bias, const void* w13,
                                 const float* w13s, const void* w2, const float* w2s, moe_dims_t d,
                                 int act, void* out, void* ws, moe_dtype_t dt, cudaStream_t s) {
  const moe_ws_layout_t L = layout(d, dt);
  const int T = d.T, H = d.H, I = d.I, E = d.E, k = d.k, R = T * k;
  int32_t* status = at<int32_t>(ws, L.status);
  float* logits = at<float>(ws, L.logits);
  int32_t* ids = at<int32_t>(ws, L.topk_ids);
  float* tw = at<float>(ws, L.topk_w);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm_token = at<int32_t>(ws, L.perm_token);
  int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
  void* y_perm = at<void>(ws, L.y_perm);
  const char* why = "";
  cudaError_t e;
  record(s, 0);
  // the E > 32 router may use the y_perm region (idle until GEMM-2) for its
  // per-h-block sums
  if ((e = launch_route(x, wr, bias, T, H, E, k, logits, ids, tw, at<float>(ws, L.y_perm),
                        (size_t)(L.total - L.y_perm), s)) != cudaSuccess)
    return cuda_fail(e, "router");
  record(s, 1);
  // The permuted copy of x feeds GEMM1's TMA tile loads (a gather inside the
  // GEMM costs the tensor cores more than this copy costs). Decode-sized
  // batches permute and gather in one launch; larger ones use the chunked
  // permutation, then write each token's row to its k positions.
  const bool small = R <= kSmallPermRows && E <= 1024;
  auto permute_large = [&]() {
    return launch_permute(ids, T, E, k, offsets, perm_token, inv_perm, at<char>(ws, L.scratch),
                          status, s);
  };
  if (dt == MOE_DTYPE_BF16) {
    void* x_perm = at<void>(ws, L.x_perm);
    void* h = at<void>(ws, L.h);
    if (small)
      e = launch_permute_gather_small(ids, T, E, k, offsets, perm_token, inv_perm, x, H * 2, x_perm,
                                      nullptr, 0, nullptr, status, s);
    else if ((e = permute_large()) == cudaSuccess)
      e = launch_scatter_rows(x, inv_perm, T, k, H * 2, x_perm, status, s);
    if (e != cudaSuccess) return cuda_fail(e, "permute");
    record(s, 2);
    // GEMM scratch: the split-K partials of the small-M kernels (decode), or
    // the K-split last wave of the plain tokens-in-M GEMM-2, in a region the
    // GEMM does not touch (x_perm, read by GEMM-1 only)
    void* splitk = L.splitk >= 0 ? at<void>(ws, L.splitk) : nullptr;
    const size_t splitk_bytes = L.splitk >= 0 ? (size_t)(L.y_perm - L.splitk) : 0;
    const size_t rows_bytes = (size_t)R * H * 2;
    if ((e = launch_grouped_gemm_bf16(x_perm, nullptr, R, w13, offsets, R, E, I, H, act, h, T,
                                      status, splitk, splitk_bytes, s, &why)) != cudaSuccess)
      return fail(MOE_ERR_CUDA, "GEMM1: %s %s", cudaGetErrorString(e), why);
    record(s, 3);
    if ((e = launch_grouped_gemm_bf16(h, nullptr, R, w2, offsets, R, E, H, I, 0, y_perm, T,
                                      status, splitk ? splitk : x_perm, splitk ? splitk_bytes : rows_bytes,
                                      s, &why)) != cudaSuccess)
      return fail(MOE_ERR_CUDA, "GEMM2: %s %s", cudaGetErrorString(e), why);
    record(s, 4);
  } else {
    void* xq = at<void>(ws, L.xq);
    float* xs = at<float>(ws, L.xs);
    void* xq_perm = at<void>(ws, L.xq_perm);
    float* xs_perm = at<float>(ws, L.xs_perm);
    void* hq = at<void>(ws, L.hq);
    float* hs = at<float>(ws, L.hs);
    // x is quantised once per token. Decode-sized batches quantise into xq /
    // xs, then permute and gather codes and scales in one launch; larger ones
    // permute first and quantise each token straight into its k permuted rows.
    const bool fp4 = dt == MOE_DTYPE_FP4_E2M1;  // w13s / w2s hold e8m0 bytes then
    const bool ue8m0 = dt == MOE_DTYPE_FP8_E4M3_UE8M0 || fp4;
    if (small) {
      if ((e = launch_quant_act(x, T, H, xq, xs, nullptr, ue8m0, s)) != cudaSuccess)
        return cuda_fail(e, "activation quantisation");
      if ((e = launch_permute_gather_small(ids, T, E, k, offsets, perm_token, inv_perm, xq, H,
                                           xq_perm, xs, (H / 128) * 4, xs_perm, status, s)) !=
          cudaSuccess)
        return cuda_fail(e, "permute");
    } else {
      if ((e = permute_large()) != cudaSuccess) return cuda_fail(e, "permute");
      if ((e = launch_quant_act_scatter(x, T, H, inv_perm, k, xq_perm, xs_perm, ue8m0, status, s)) !=
          cudaSuccess)
        return cuda_fail(e, "activation quantisation");
    }
    record(s, 2);
    if (ue8m0) {
      // power-of-two scales: the block-scaled tensor-core path, no promotion
      const float* f13 = fp4 ? nullptr : w13s;
      const float* f2 = fp4 ? nullptr : w2s;
      const uint8_t* b13 = fp4 ? reinterpret_cast<const uint8_t*>(w13s) : nullptr;
      const uint8_t* b2 = fp4 ? reinterpret_cast<const uint8_t*>(w2s) : nullptr;
      // the tokens-in-M kernel at every batch size: at decode sizes the
      // weights-in-M form measured no faster (weight streaming bounds both)
      if ((e = launch_grouped_gemm_mx(xq_perm, xs_perm, w13, f13, b13, offsets, R, E, I, H, act, hq,
                                      hs, status, s, &why)) != cudaSuccess)
        return fail(MOE_ERR_CUDA, "%s GEMM1: %s %s", fp4 ? "FP4" : "FP8", cudaGetErrorString(e), why);
      record(s, 3);
      if ((e = launch_grouped_gemm_mx(hq, hs, w2, f2, b2, offsets, R, E, H, I, 0, y_perm, nullptr,
                                      status, s, &why)) != cudaSuccess)
        return fail(MOE_ERR_CUDA, "%s GEMM2: %s %s", fp4 ? "FP4" : "FP8", cudaGetErrorString(e), why);
    } else {
      if ((e = launch_grouped_gemm_fp8(xq_perm, nullptr, R, xs_perm, w13, w13s, offsets, R, E, I, H,
                                       act, hq, hs, T, status, s, &why)) != cudaSuccess)
        return fail(MOE_ERR_CUDA, "FP8 GEMM1: %s %s", cudaGetErrorString(e), why);
      record(s, 3);
      if ((e = launch_grouped_gemm_fp8(hq, nullptr, R, hs, w2, w2s, offsets, R, E, H, I, 0, y_perm,
                                       nullptr, T, status, s, &why)) != cudaSuccess)
        return fail(MOE_ERR_CUDA, "FP8 GEMM2: %s %s", cudaGetErrorString(e), why);
    }
    record(s, 4);
  }
  if ((e = launch_combine(y_perm, tw, inv_perm, T, H, k, out, status, s)) != cudaSuccess)
    return cuda_fail(e, "combine");
  record(s, 5);
  return ok();
}

static moe_status_t check_act(moe_epilogue_t act) {
  if (act < MOE_EPILOGUE_SWIGLU || act > MOE_EPILOGUE_REGLU)
    return fail(MOE_ERR_INVALID_ARG, "the expert activation must be SWIGLU, GEGLU or REGLU (got %d)",
                (int)act);
  return MOE_OK;
}

moe_status_t moe_forward_gated(const void* x, const void* wr, const float* bias, const void* w13,
                               const void* w2, moe_dims_t d, moe_epilogue_t act, void* out, void* ws,
                               size_t ws_bytes, void* stream) {
  MOE_TRY(check_dims(d, true));
  MOE_TRY(check_act(act));
  MOE_TRY(check_ptr(x, "x"));
  MOE_TRY(check_ptr(wr, "w_router"));
  MOE_TRY(check_ptr(bias, "bias", true));
  MOE_TRY(check_ptr(w13, "w13"));
  MOE_TRY(check_ptr(w2, "w2"));
  MOE_TRY(check_ptr(out, "out"));
  MOE_TRY(check_ws(d, MOE_DTYPE_BF16, ws, ws_bytes));
  MOE_TRY(check_device());
  return forward_impl(x, wr, bias, w13, nullptr, w2, nullptr, d, (int)act, out, ws, MOE_DTYPE_BF16,
                      static_cast<cudaStream_t>(stream));
}

moe_status_t moe_forward(const void* x, const void* wr, const float* bias, const void* w13,
                         const void* w2, moe_dims_t d, void* out, void* ws, size_t ws_bytes,
                         void* stream) {
  return moe_forward_gated(x, wr, bias, w13, w2, d, MOE_EPILOGUE_SWIGLU, out, ws, ws_bytes, stream);
}

moe_status_t moe_forward_fp8_gated(const void* x, const void* wr, const float* bias,
                                   const void* w13q, const float* w13s, const void* w2q,
                                   const float* w2s, moe_dims_t d, moe_epilogue_t act, void* out,
                                   void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_dims(d, true));
  MOE_TRY(check_act(act));
  MOE_TRY(check_ptr(x, "x"));
  MOE_TRY(check_ptr(wr, "w_router"));
  MOE_TRY(check_ptr(bias, "bias", true));
  MOE_TRY(check_ptr(w13q, "w13q"));
  MOE_TRY(check_ptr(w13s, "w13s"));
  MOE_TRY(check_ptr(w2q, "w2q"));
  MOE_TRY(check_ptr(w2s, "w2s"));
  MOE_TRY(check_ptr(out, "out"));
  if (d.H % 256) return fail(MOE_ERR_INVALID_ARG, "the FP8 layer needs H %% 256 == 0 (got %d)", d.H);
  MOE_TRY(check_ws(d, MOE_DTYPE_FP8_E4M3, ws, ws_bytes));
  MOE_TRY(check_device());
  return forward_impl(x, wr, bias, w13q, w13s, w2q, w2s, d, (int)act, out, ws, MOE_DTYPE_FP8_E4M3,
                      static_cast<cudaStream_t>(stream));
}

moe_status_t moe_forward_fp8_ue8m0(const void* x, const void* wr, const float* bias,
                                   const void* w13q, const float* w13s, const void* w2q,
                                   const float* w2s, moe_dims_t d, moe_epilogue_t act, void* out,
                                   void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_dims(d, true));
  MOE_TRY(check_act(act));
  MOE_TRY(check_ptr(x, "x"));
  MOE_TRY(check_ptr(wr, "w_router"));
  MOE_TRY(check_ptr(bias, "bias", true));
  MOE_TRY(check_ptr(w13q, "w13q"));
  MOE_TRY(check_ptr(w13s, "w13s"));
  MOE_TRY(check_ptr(w2q, "w2q"));
  MOE_TRY(check_ptr(w2s, "w2s"));
  MOE_TRY(check_ptr(out, "out"));
  if (d.H % 256) return fail(MOE_ERR_INVALID_ARG, "the FP8 layer needs H %% 256 == 0 (got %d)", d.H);
  MOE_TRY(check_ws(d, MOE_DTYPE_FP8_E4M3_UE8M0, ws, ws_bytes));
  MOE_TRY(check_device());
  return forward_impl(x, wr, bias, w13q, w13s, w2q, w2s, d, (int)act, out, ws,
                      MOE_DTYPE_FP8_E4M3_UE8M0, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_forward_fp4(const void* x, const void* wr, const float* bias, const void* w13q,
                             const uint8_t* w13s, const void* w2q, const uint8_t* w2s, moe_dims_t d,
                             moe_epilogue_t act, void* out, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_dims(d, true));
  MOE_TRY(check_act(act));
  MOE_TRY(check_ptr(x, "x"));
  MOE_TRY(check_ptr(wr, "w_router"));
  MOE_TRY(check_ptr(bias, "bias", true));
  MOE_TRY(check_ptr(w13q, "w13q"));
  MOE_TRY(check_ptr(w2q, "w2q"));
  if ((reinterpret_cast<uintptr_t>(w13q) | reinterpret_cast<uintptr_t>(w2q)) & 31)
    return fail(MOE_ERR_INVALID_ARG, "packed FP4 weights must be 32-byte aligned");
  MOE_TRY(check_ptr(w13s, "w13s"));
  MOE_TRY(check_ptr(w2s, "w2s"));
  MOE_TRY(check_ptr(out, "out"));
  if (d.H % 256) return fail(MOE_ERR_INVALID_ARG, "the FP4 layer needs H %% 256 == 0 (got %d)", d.H);
  MOE_TRY(check_ws(d, MOE_DTYPE_FP4_E2M1, ws, ws_bytes));
  MOE_TRY(check_device());
  return forward_impl(x, wr, bias, w13q, reinterpret_cast<const float*>(w13s), w2q,
                      reinterpret_cast<const float*>(w2s), d, (int)act, out, ws, MOE_DTYPE_FP4_E2M1,
                      static_cast<cudaStream_t>(stream));
}

moe_status_t moe_forward_fp8(const void* x, const void* wr, const float* bias, const void* w13q,
                             const float* w13s, const void* w2q, const float* w2s, moe_dims_t d,
                             void* out, void* ws, size_t ws_bytes, void* stream) {
  return moe_forward_fp8_gated(x, wr, bias, w13q, w13s, w2q, w2s, d, MOE_EPILOGUE_SWIGLU, out, ws,
                               ws_bytes, stream);
}

moe_status_t moe_forward_hostio(const void* x_host, const void* wr, const float* bias,
                                const void* w13, const void* w2, moe_dims_t d, void* out_host,
                                void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_dims(d, true));
  if (!x_host || !out_host) return fail(MOE_ERR_INVALID_ARG, "x_host and out_host must be given");
  MOE_TRY(check_ptr(wr, "w_router"));
  MOE_TRY(check_ptr(bias, "bias", true));
  MOE_TRY(check_ptr(w13, "w13"));
  MOE_TRY(check_ptr(w2, "w2"));
  const size_t io = (size_t)d.T * d.H * 2;
  const size_t io_al = (size_t)align_up((int64_t)io, 256);
  MOE_TRY(check_ws(d, MOE_DTYPE_BF16, ws, ws_bytes, 2 * io_al));
  MOE_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t base = layout(d, MOE_DTYPE_BF16).total;
  void* x_dev = at<void>(ws, base);
  void* out_dev = at<void>(ws, base + (int64_t)io_al);
  cudaError_t e = cudaMemcpyAsync(x_dev, x_host, io, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "copy x to device");
  MOE_TRY(forward_impl(x_dev, wr, bias, w13, nullptr, w2, nullptr, d, MOE_EPILOGUE_SWIGLU, out_dev, ws,
                       MOE_DTYPE_BF16, s));
  e = cudaMemcpyAsync(out_host, out_dev, io, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "copy out to host");
  return ok();
}

moe_status_t moe_quantize_act_fp8_fmt(const void* x, int64_t rows, int64_t cols, void* q, float* sc,
                                      moe_scale_fmt_t fmt, void* stream) {
  if (rows < 1 || cols < 128 || cols % 128) return fail(MOE_ERR_INVALID_ARG, "rows >= 1, cols a multiple of 128");
  if (fmt != MOE_SCALE_F32 && fmt != MOE_SCALE_UE8M0) return fail(MOE_ERR_INVALID_ARG, "bad scale format");
  MOE_TRY(check_ptr(x, "x"));
  MOE_TRY(check_ptr(q, "q"));
  MOE_TRY(check_ptr(sc, "s"));
  MOE_TRY(check_device());
  cudaError_t e = launch_quant_act(x, rows, cols, q, sc, nullptr, fmt == MOE_SCALE_UE8M0,
                                   static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "activation quantisation");
  return ok();
}

moe_status_t moe_quantize_act_fp8(const void* x, int64_t rows, int64_t cols, void* q, float* sc,
                                  void* stream) {
  return moe_quantize_act_fp8_fmt(x, rows, cols, q, sc, MOE_SCALE_F32, stream);
}

moe_status_t moe_quantize_weight_fp8_fmt(const void* w, int64_t nb, int64_t rows, int64_t cols,
                                         void* q, float* sc, moe_scale_fmt_t fmt, void* stream) {
  if (nb < 1 || rows < 128 || rows % 128 || cols < 128 || cols % 128)
    return fail(MOE_ERR_INVALID_ARG, "nb >= 1, rows and cols multiples of 128");
  if (fmt != MOE_SCALE_F32 && fmt != MOE_SCALE_UE8M0) return fail(MOE_ERR_INVALID_ARG, "bad scale format");
  MOE_TRY(check_ptr(w, "w"));
  MOE_TRY(check_ptr(q, "q"));
  MOE_TRY(check_ptr(sc, "s"));
  MOE_TRY(check_device());
  cudaError_t e = launch_quant_weight(w, nb, rows, cols, q, sc, fmt == MOE_SCALE_UE8M0,
                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "weight quantisation");
  return ok();
}

moe_status_t moe_quantize_weight_fp8(const void* w, int64_t nb, int64_t rows, int64_t cols, void* q,
                                     float* sc, void* stream) {
  return moe_quantize_weight_fp8_fmt(w, nb, rows, cols, q, sc, MOE_SCALE_F32, stream);
}

moe_status_t moe_quantize_weight_fp4(const void* w, int64_t nb, int64_t rows, int64_t cols,
                                     void* q, uint8_t* sc, void* stream) {
  if (nb < 1 || rows < 128 || rows % 128 || cols < 128 || cols % 128)
    return fail(MOE_ERR_INVALID_ARG, "nb >= 1, rows and cols multiples of 128");
  MOE_TRY(check_ptr(w, "w"));
  MOE_TRY(check_ptr(q, "q"));
  MOE_TRY(check_ptr(sc, "s"));
  MOE_TRY(check_device());
  cudaError_t e = launch_quant_weight_fp4(w, nb, rows, cols, q, sc, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "FP4 weight quantisation");
  return ok();
}

moe_status_t moe_pack_weights(const void* wg, const void* wu, const void* wd, int32_t E, int32_t H,
                              int32_t I, void* w13, void* w2, void* stream) {
  if (E < 1 || E > 65535) return fail(MOE_ERR_INVALID_ARG, "E must be in [1, 65535] (got %d)", E);
  if (H < 128 || H % 128)
    return fail(MOE_ERR_INVALID_ARG, "H must be a positive multiple of 128 (got %d)", H);
  if (I < 128 || I % 128)
    return fail(MOE_ERR_INVALID_ARG, "I must be a positive multiple of 128 (got %d)", I);
  MOE_TRY(check_ptr(wg, "wg"));
  MOE_TRY(check_ptr(wu, "wu"));
  MOE_TRY(check_ptr(wd, "wd"));
  MOE_TRY(check_ptr(w13, "w13"));
  MOE_TRY(check_ptr(w2, "w2"));
  // the outputs must not overlap any input (the transposes read and write concurrently)
  const uint64_t hi = (uint64_t)H * I * 2 * E;
  auto lo_of = [](const void* p) { return reinterpret_cast<uint64_t>(p); };
  auto overlap = [&](const void* a, uint64_t na, const void* b, uint64_t nb) {
    return lo_of(a) < lo_of(b) + nb && lo_of(b) < lo_of(a) + na;
  };
  const void* ins[3] = {wg, wu, wd};
  for (const void* in : ins)
    if (overlap(w13, 2 * hi, in, hi) || overlap(w2, hi, in, hi))
      return fail(MOE_ERR_INVALID_ARG, "w13 / w2 overlap an input weight");
  if (overlap(w13, 2 * hi, w2, hi)) return fail(MOE_ERR_INVALID_ARG, "w13 and w2 overlap");
  MOE_TRY(check_device());
  cudaError_t e = launch_pack_weights(wg, wu, wd, E, H, I, w13, w2, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "weight packing");
  return ok();
}

namespace {
moe_status_t check_ep(int32_t E, int32_t G, int32_t rank) {
  if (G < 1 || G > 64) return fail(MOE_ERR_INVALID_ARG, "G must be in [1, 64] (got %d)", G);
  if (E < 1 || E > 1024 || E % G)
    return fail(MOE_ERR_INVALID_ARG, "E must be in [1, 1024] and a multiple of G (E=%d, G=%d)", E, G);
  if (rank < 0 || rank >= G) return fail(MOE_ERR_INVALID_ARG, "rank must be in [0, G) (got %d)", rank);
  return MOE_OK;
}
}  // namespace

size_t moe_ep_plan_bytes(int32_t E, int32_t G) {
  if (check_ep(E, G, 0) != MOE_OK) return 0;
  return (size_t)ep_plan_ints(E, G) * sizeof(int32_t);
}

moe_status_t moe_ep_plan(const int32_t* counts_all, int32_t G, int32_t rank, int32_t E,
                         int32_t* plan, void* stream) {
  MOE_TRY(check_ep(E, G, rank));
  MOE_TRY(check_ptr(counts_all, "counts_all"));
  MOE_TRY(check_ptr(plan, "plan"));
  MOE_TRY(check_device());
  cudaError_t e = launch_ep_plan(counts_all, G, E, rank, plan, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "expert-parallel plan");
  return ok();
}

moe_status_t moe_ep_dispatch(const void* x_perm, const int32_t* offsets, const int32_t* plan,
                             int32_t E, int32_t G, int32_t R, int64_t row_bytes,
                             const uint64_t* dst_bufs, int64_t dst_rows, void* ws, void* stream) {
  MOE_TRY(check_ep(E, G, 0));
  if (R < 0) return fail(MOE_ERR_INVALID_ARG, "R must be >= 0 (got %d)", R);
  if (row_bytes < 16 || row_bytes % 16 || row_bytes > (int64_t)1 << 30)
    return fail(MOE_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 16 (got %lld)",
                (long long)row_bytes);
  if (dst_rows < 0) return fail(MOE_ERR_INVALID_ARG, "dst_rows must be >= 0");
  MOE_TRY(check_ptr(x_perm, "x_perm", R == 0));
  MOE_TRY(check_ptr(offsets, "offsets"));
  MOE_TRY(check_ptr(plan, "plan"));
  MOE_TRY(check_ptr(dst_bufs, "dst_bufs"));
  MOE_TRY(check_ptr(ws, "ws", true));
  MOE_TRY(check_device());
  cudaError_t e = launch_ep_dispatch(x_perm, offsets, plan, E, G, R, (int)row_bytes, dst_bufs,
                                     dst_rows, static_cast<int32_t*>(ws),
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "expert-parallel dispatch");
  return ok();
}

moe_status_t moe_ep_return(const void* y_loc, const int32_t* plan, int32_t E, int32_t G,
                           int64_t cap_rows, int64_t row_bytes, const uint64_t* src_bufs,
                           int64_t src_rows, void* ws, void* stream) {
  MOE_TRY(check_ep(E, G, 0));
  if (cap_rows < 0 || cap_rows > ((int64_t)1 << 31) * 8)
    return fail(MOE_ERR_INVALID_ARG, "cap_rows out of range");
  if (row_bytes < 16 || row_bytes % 16 || row_bytes > (int64_t)1 << 30)
    return fail(MOE_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 16 (got %lld)",
                (long long)row_bytes);
  if (src_rows < 0) return fail(MOE_ERR_INVALID_ARG, "src_rows must be >= 0");
  MOE_TRY(check_ptr(y_loc, "y_loc", cap_rows == 0));
  MOE_TRY(check_ptr(plan, "plan"));
  MOE_TRY(check_ptr(src_bufs, "src_bufs"));
  MOE_TRY(check_ptr(ws, "ws", true));
  MOE_TRY(check_device());
  cudaError_t e = launch_ep_return(y_loc, plan, E, G, cap_rows, (int)row_bytes, src_bufs, src_rows,
                                   static_cast<int32_t*>(ws), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "expert-parallel return");
  return ok();
}

moe_status_t moe_get_device_status(const void* ws, int32_t* status_out) {
  MOE_TRY(check_ptr(ws, "ws"));
  if (!status_out) return fail(MOE_ERR_INVALID_ARG, "status_out is NULL");
  int32_t v = 0;
  cudaError_t e = cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  *status_out = v;
  return ok();
}

moe_status_t moe_check_wait_timeout(void* ws, int64_t budget_cycles, void* stream) {
  MOE_TRY(check_ptr(ws, "ws"));
  if (budget_cycles < 1000 || budget_cycles > 2000000000LL)
    return fail(MOE_ERR_INVALID_ARG, "budget_cycles must be in [1000, 2e9] (got %lld)",
                (long long)budget_cycles);
  MOE_TRY(check_device());
  cudaError_t e = launch_wait_selftest(static_cast<int32_t*>(ws), (long long)budget_cycles,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "wait self-test");
  return ok();
}

moe_status_t moe_clear_device_status(void* ws, void* stream) {
  MOE_TRY(check_ptr(ws, "ws"));
  cudaError_t e = cudaMemsetAsync(ws, 0, 4, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  return ok();
}

moe_status_t moe_set_stage_events(void* const* events, int32_t n) {
  if (!events) {
    t_events_on = false;
    return ok();
  }
  if (n != 6) return fail(MOE_ERR_INVALID_ARG, "expected 6 events (got %d)", n);
  for (int i = 0; i < 6; ++i) t_events[i] = events[i];
  t_events_on = true;
  return ok();
}

}  // extern "C"
