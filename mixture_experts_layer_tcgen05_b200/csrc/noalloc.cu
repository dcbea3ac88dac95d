// moe_permute_noalloc: the permutation by expert with its scratch in a
// fixed device array that this library owns, for callers that cannot hand
// the library a workspace.
//
// The scratch is a file-scope __device__ array, so it exists once per device
// that loads the library and stays allocated until the process exits. In host
// code its name only stands in for the symbol (it is not a device address),
// so the address the kernels receive comes from cudaGetSymbolAddress, looked
// up once per device with that device current.
#include <mutex>

#include "common.cuh"

namespace moe {

cudaError_t launch_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets,
                           int32_t* perm_token, int32_t* inv_perm, void* scratch, int32_t* status,
                           cudaStream_t s);
cudaError_t launch_scatter_rows(const void* x, const int32_t* inv_perm, int T, int k,
                                int row_bytes, void* x_perm, int32_t* status, cudaStream_t s);

// The fixed array: its first 256 bytes hold a status word (the same encoding
// as a workspace's), the rest is the permutation's scratch.
constexpr int64_t kNoAllocBytes = MOE_NOALLOC_SCRATCH_BYTES;
constexpr int64_t kNoAllocStatusBytes = 256;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of the array on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

// Bytes of the array left for the permutation's scratch (after the status word).
int64_t noalloc_scratch_capacity() { return kNoAllocBytes - kNoAllocStatusBytes; }

// Same kernels as moe_permute, with the status word and the scratch taken from
// the fixed array.
cudaError_t launch_permute_noalloc(const int32_t* ids, int T, int H, int E, int k, int32_t* offsets,
                                   int32_t* perm_token, int32_t* inv_perm, const void* x,
                                   void* x_perm, cudaStream_t s) {
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return e;
  int32_t* status = static_cast<int32_t*>(base);
  void* scratch = static_cast<char*>(base) + kNoAllocStatusBytes;
  // Every scratch word the permutation reads is written earlier in the same
  // call (chunk masks, chunk bases, counts), so the scratch needs no clearing.
  // The status word is not cleared either: like a workspace's, it keeps the
  // first failure until moe_permute_noalloc_status clears it.
  e = launch_permute(ids, T, E, k, offsets, perm_token, inv_perm, scratch, status, s);
  if (e == cudaSuccess && x) e = launch_scatter_rows(x, inv_perm, T, k, H * 2, x_perm, status, s);
  return e;
}

// Reads the status word of the current device's array (a blocking copy, after
// all work on the device) and, if `clear`, sets it back to zero.
cudaError_t noalloc_status(int32_t* out, bool clear) {
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return e;
  e = cudaDeviceSynchronize();  // work on every stream, blocking or not, has finished
  if (e == cudaSuccess) e = cudaMemcpy(out, base, sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && clear) e = cudaMemset(base, 0, sizeof(int32_t));
  if (e == cudaSuccess && clear) e = cudaDeviceSynchronize();
  return e;
}

}  // namespace moe
