// Expert-parallel exchange of routed rows between ranks, planned and moved on
// the device (no host round trip for the counts).
//
// "Experts backends" (HF Transformers docs), backend table, deepgemm_megamoe
// row: the experts are spread over ranks and each token's rows travel to the
// ranks that own their experts and back. Here G ranks own E / G consecutive
// experts each (rank g: experts [g*El, (g+1)*El), El = E / G). After every
// rank has routed and permuted its own tokens (rows expert-major), the G x E
// matrix cnt[s][e] of rows rank s holds for expert e (an all-gather of the
// permutation's counts) fixes every row's destination:
//
//  * rank g's receive buffer is expert-major: local expert j, then source
//    rank s ascending, then the source's own row order; so the grouped GEMMs
//    run on it directly with offsets loc_off[j];
//  * source r's rows for expert e start at
//      send_base[e] = sum_{j' < j} sum_s cnt[s][g*El + j'] + sum_{s < r} cnt[s][e]
//    in rank g = e / El's buffer (j = e % El);
//  * back at the source, the expert output of those rows goes to the same
//    positions of the source's y_perm they were sent from: for local expert j
//    and source s, ret_dst[j*G + s] = sum_{e' < r*El + j} cnt[s][e'].
//
// Rows move by plain stores through the destination pointers (the buffers of
// the other ranks mapped into this process, e.g. symmetric memory), 16 bytes
// per lane; no TMA copies touch peer memory. Each warp ends with a system-scope fence so
// its stores are visible to the other ranks once the stream's next
// cross-rank synchronisation (a collective) has run.
#include "common.cuh"

namespace moe {

// Plan (int32): loc_off[El + 1] at the start (so it is as aligned as the plan,
// for the grouped GEMMs), then send_base[E] at ep_plan_send_off(El), then
// ret_lb[El*G + 1], ret_dst[El*G]. One block of 1024 threads; E <= 1024 and
// G <= 64 (checked by the host).
__host__ __device__ constexpr int ep_plan_send_off(int El) { return (El + 1 + 3) / 4 * 4; }

__global__ void __launch_bounds__(1024) ep_plan_kernel(const int32_t* __restrict__ cnt, int G, int E,
                                                       int rank, int32_t* __restrict__ plan) {
  __shared__ int32_t colsum[1024];
  __shared__ int32_t scan[1025];  // exclusive scan of colsum over all E experts
  const int El = E / G;
  int32_t* loc_off = plan;
  int32_t* send_base = plan + ep_plan_send_off(El);
  int32_t* ret_lb = send_base + E;
  int32_t* ret_dst = ret_lb + El * G + 1;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t c = 0;
    for (int s = 0; s < G; ++s) c += cnt[(int64_t)s * E + e];
    colsum[e] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // E <= 1024 additions: serial is cheap and exact
    int32_t run = 0;
    for (int e = 0; e < E; ++e) {
      scan[e] = run;
      run += colsum[e];
    }
    scan[E] = run;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int g = e / El;
    int32_t pre = 0;  // rows of lower source ranks for this expert
    for (int s = 0; s < rank; ++s) pre += cnt[(int64_t)s * E + e];
    send_base[e] = scan[e] - scan[g * El] + pre;
  }
  const int e0 = rank * El;
  for (int j = threadIdx.x; j <= El; j += blockDim.x) loc_off[j] = scan[e0 + j] - scan[e0];
  // return blocks, (local expert j, source s) in receive order
  for (int b = threadIdx.x; b < El * G; b += blockDim.x) {
    const int j = b / G, s = b % G;
    int32_t lb = scan[e0 + j] - scan[e0];
    for (int s2 = 0; s2 < s; ++s2) lb += cnt[(int64_t)s2 * E + e0 + j];
    ret_lb[b] = lb;
    int32_t dst = 0;  // the source's own offset of expert e0 + j
    for (int e = 0; e < e0 + j; ++e) dst += cnt[(int64_t)s * E + e];
    ret_dst[b] = dst;
  }
  if (threadIdx.x == 0) ret_lb[El * G] = scan[e0 + El] - scan[e0];
}

// Dispatch: row p of this rank's x_perm (expert-major, offsets[E + 1]) goes to
// rank g = e / El at row send_base[e] + (p - offsets[e]). One warp per row.
__global__ void __launch_bounds__(256) ep_dispatch_kernel(
    const uint4* __restrict__ x_perm, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ plan, int E, int G, int R, int vec_per_row,
    const uint64_t* __restrict__ dst_bufs, int64_t dst_rows, int32_t* status) {
  const int p = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (p >= R || p >= offsets[E]) return;  // warp-uniform
  // expert of row p: the last e with offsets[e] <= p
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offsets[mid] <= p) lo = mid;
    else hi = mid;
  }
  const int e = lo, El = E / G;
  const int64_t pos = (int64_t)plan[ep_plan_send_off(El) + e] + (p - offsets[e]);
  if (pos < 0 || pos >= dst_rows) {
    if (lane == 0) record_bad_index(status);
    return;
  }
  uint4* dst = reinterpret_cast<uint4*>(dst_bufs[e / El]) + pos * vec_per_row;
  const uint4* src = x_perm + (int64_t)p * vec_per_row;
  for (int v = lane; v < vec_per_row; v += 32) dst[v] = src[v];
  __threadfence_system();
}

// Return: local row q (receive order) of y_loc goes back to its source s at
// row ret_dst[b] + (q - ret_lb[b]) of the source's y_perm, b = (j, s) the
// block holding q. One warp per row; rows past loc_off[El] do nothing.
__global__ void __launch_bounds__(256) ep_return_kernel(
    const uint4* __restrict__ y_loc, const int32_t* __restrict__ plan, int E, int G,
    int64_t cap, int vec_per_row, const uint64_t* __restrict__ src_bufs, int64_t src_rows,
    int32_t* status) {
  const int El = E / G;
  const int32_t* ret_lb = plan + ep_plan_send_off(El) + E;
  const int32_t* ret_dst = ret_lb + El * G + 1;
  const int64_t q = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int nb = El * G;
  if (q >= cap || q >= ret_lb[nb]) return;  // warp-uniform
  int lo = 0, hi = nb;  // last b with ret_lb[b] <= q (empty blocks share a start)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ret_lb[mid] <= q) lo = mid;
    else hi = mid;
  }
  const int b = lo, s = b % G;
  const int64_t pos = (int64_t)ret_dst[b] + (q - ret_lb[b]);
  if (pos < 0 || pos >= src_rows) {
    if (lane == 0) record_bad_index(status);
    return;
  }
  uint4* dst = reinterpret_cast<uint4*>(src_bufs[s]) + pos * vec_per_row;
  const uint4* src = y_loc + q * vec_per_row;
  for (int v = lane; v < vec_per_row; v += 32) dst[v] = src[v];
  __threadfence_system();
}

int64_t ep_plan_ints(int E, int G) {
  const int El = E / G;
  return (int64_t)ep_plan_send_off(El) + E + (El * G + 1) + El * G;
}

cudaError_t launch_ep_plan(const int32_t* cnt, int G, int E, int rank, int32_t* plan,
                           cudaStream_t s) {
  ep_plan_kernel<<<1, 1024, 0, s>>>(cnt, G, E, rank, plan);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const void* x_perm, const int32_t* offsets, const int32_t* plan,
                               int E, int G, int R, int row_bytes, const uint64_t* dst_bufs,
                               int64_t dst_rows, int32_t* status, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  ep_dispatch_kernel<<<(unsigned)ceil_div(R, 8), 256, 0, s>>>(
      static_cast<const uint4*>(x_perm), offsets, plan, E, G, R, row_bytes / 16, dst_bufs,
      dst_rows, status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_ep_return(const void* y_loc, const int32_t* plan, int E, int G, int64_t cap,
                             int row_bytes, const uint64_t* src_bufs, int64_t src_rows,
                             int32_t* status, cudaStream_t s) {
  if (cap == 0) return cudaSuccess;
  ep_return_kernel<<<(unsigned)ceil_div(cap, 8), 256, 0, s>>>(
      static_cast<const uint4*>(y_loc), plan, E, G, cap, row_bytes / 16, src_bufs, src_rows,
      status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
