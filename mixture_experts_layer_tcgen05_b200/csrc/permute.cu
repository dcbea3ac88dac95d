// Permutation of routed (token, slot) pairs by expert, the row gather, and
// the weighted combine.
//
// "Experts backends" (HF Transformers docs), backend table, grouped_mm row:
// the routed tokens are sorted by chosen expert so one grouped GEMM covers
// every expert. The order is expert-major, then token ascending; a token
// holds each expert at most once, so this order is unique. It is built
// without atomics on the order itself:
//   1. per 32-token chunk (one warp), a bitmask per expert of the chunk's
//      lanes (tokens) that chose it;
//   2. per expert, an exclusive scan of popcount(mask) over chunks, and the
//      expert totals;
//   3. offsets = exclusive scan of the totals over experts; the row of
//      (token t, slot j) with expert e is
//        offsets[e] + chunk_base[chunk(t)][e] + popc(mask[chunk(t)][e] & lanes below t).
#include <algorithm>

#include "common.cuh"
#include "permute.cuh"
#include "ptx.cuh"

namespace moe {

// ---- 1. chunk masks ---------------------------------------------------------
// grid: one warp per chunk of 32 tokens, 4 warps per block; smem E words per warp.
__global__ void __launch_bounds__(128) permute_mask_kernel(const int32_t* __restrict__ ids, int T,
                                                           int E, int k, int nchunks,
                                                           uint32_t* __restrict__ masks,
                                                           int32_t* status) {
  extern __shared__ uint32_t pm_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * 4 + warp;
  uint32_t* m = pm_smem + warp * E;
  for (int e = lane; e < E; e += 32) m[e] = 0;
  __syncwarp();
  if (chunk < nchunks) {
    int t = chunk * 32 + lane;
    if (t < T)
      for (int j = 0; j < k; ++j) {
        const int e = ids[(int64_t)t * k + j];
        if ((unsigned)e >= (unsigned)E) record_bad_index(status);
        else if (atomicOr(&m[e], 1u << lane) & (1u << lane))  // bit already set: a repeat
          record_bad_index(status);
      }
  }
  __syncwarp();
  if (chunk < nchunks)
    for (int e = lane; e < E; e += 32) masks[(int64_t)chunk * E + e] = m[e];
}

// ---- 2. per-expert scan over chunks ----------------------------------------
// block: 32 experts (lanes) x 32 warps; warp w scans chunks [w*S, (w+1)*S).
__global__ void __launch_bounds__(1024) permute_scan_kernel(const uint32_t* __restrict__ masks,
                                                            int E, int nchunks,
                                                            int32_t* __restrict__ chunk_base,
                                                            int32_t* __restrict__ counts) {
  __shared__ int32_t seg_total[32][33];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 32 + lane;
  const int S = (nchunks + 31) / 32;
  const int c0 = warp * S, c1 = min(nchunks, c0 + S);
  int32_t run = 0;
  if (e < E)
    for (int c = c0; c < c1; ++c) run += __popc(masks[(int64_t)c * E + e]);
  seg_total[warp][lane] = run;
  __syncthreads();
  int32_t base = 0;
  for (int w = 0; w < warp; ++w) base += seg_total[w][lane];
  if (e < E) {
    for (int c = c0; c < c1; ++c) {
      chunk_base[(int64_t)c * E + e] = base;
      base += __popc(masks[(int64_t)c * E + e]);
    }
    if (warp == 31) counts[e] = base;
  }
}

// ---- 3. offsets + scatter ---------------------------------------------------
// Each block first scans the E totals into offsets (block 0 stores them),
// then one warp per chunk places its (token, slot) pairs.
__global__ void __launch_bounds__(128) permute_scatter_kernel(
    const int32_t* __restrict__ ids, const uint32_t* __restrict__ masks,
    const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ counts, int T, int E,
    int k, int nchunks, int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token,
    int32_t* __restrict__ inv_perm, int32_t* status) {
  extern __shared__ int32_t off_smem[];  // E + 1
  __shared__ int32_t warp_sums[4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // exclusive scan of counts over E with 128 threads: each owns a contiguous slice
  const int per = (E + 127) / 128;
  const int lo = threadIdx.x * per, hi = min(E, lo + per);
  int32_t local = 0;
  for (int e = lo; e < hi; ++e) local += counts[e];
  int32_t incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int32_t v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  int32_t wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += warp_sums[w];
  int32_t run = wbase + incl - local;
  for (int e = lo; e < hi; ++e) {
    off_smem[e] = run;
    run += counts[e];
  }
  if (threadIdx.x == 127) off_smem[E] = wbase + incl;
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e <= E; e += 128) offsets[e] = off_smem[e];

  const int chunk = blockIdx.x * 4 + warp;
  if (chunk >= nchunks) return;
  const int t = chunk * 32 + lane;
  if (t >= T) return;
  const uint32_t below = (1u << lane) - 1u;
  for (int j = 0; j < k; ++j) {
    int e = ids[(int64_t)t * k + j];
    if ((unsigned)e >= (unsigned)E) continue;  // recorded by the mask kernel
    uint32_t m = masks[(int64_t)chunk * E + e];
    int32_t p = off_smem[e] + chunk_base[(int64_t)chunk * E + e] + __popc(m & below);
    if ((unsigned)p >= (unsigned)(T * k)) {  // only for invalid ids (recorded by the mask kernel)
      record_bad_index(status);
      continue;
    }
    perm_token[p] = t;
    inv_perm[(int64_t)t * k + j] = p;
  }
}

// ---- row gather: x_perm[p, :] = x[perm_token[p], :] --------------------------
// one warp per row, 16-byte vectors (4-byte words for rows that are not a
// multiple of 16 bytes, e.g. a few fp32 scales)
template <typename V>
__global__ void __launch_bounds__(256) gather_rows_kernel(const V* __restrict__ x,
                                                          const int32_t* __restrict__ perm_token,
                                                          int R, int T, int vec_per_row,
                                                          V* __restrict__ x_perm, int32_t* status) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= R) return;
  const int t = perm_token[row];
  if ((unsigned)t >= (unsigned)T) {
    if (lane == 0) record_bad_index(status);
    return;
  }
  const V* src = x + (int64_t)t * vec_per_row;
  V* dst = x_perm + (int64_t)row * vec_per_row;
  for (int v = lane; v < vec_per_row; v += 32) dst[v] = src[v];
}

// ---- token-major row scatter: x_perm[inv_perm[t, j], :] = x[t, :] -----------
// The same bytes as the gather, visited from the source side: one warp per
// token reads its row once and writes it to the row's k positions, so x
// crosses HBM once however many experts the token chose (the gather reads a
// row k times, from HBM again once the output stream has evicted it from L2).
// Four vectors per lane are loaded before their stores, for more loads in
// flight. k <= 16 (the largest k the entry points accept); destinations
// outside [0, T*k) set the status flag and the warp writes nothing.
constexpr int kScatterMaxK = 16;

template <typename V>
__global__ void __launch_bounds__(256) scatter_rows_kernel(const V* __restrict__ x,
                                                           const int32_t* __restrict__ inv_perm,
                                                           int T, int k, int vec_per_row,
                                                           V* __restrict__ x_perm, int32_t* status) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= T) return;  // warp-uniform
  const int R = T * k;
  const int mine = lane < k ? inv_perm[(int64_t)t * k + lane] : 0;
  if (__any_sync(0xffffffffu, (unsigned)mine >= (unsigned)R)) {
    if (lane == 0) record_bad_index(status);
    return;
  }
  V* dst[kScatterMaxK];
#pragma unroll
  for (int j = 0; j < kScatterMaxK; ++j)
    dst[j] = x_perm + (int64_t)__shfl_sync(0xffffffffu, mine, j) * vec_per_row;
  const V* src = x + (int64_t)t * vec_per_row;
  for (int v0 = lane; v0 < vec_per_row; v0 += 4 * 32) {
    V u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (v0 + i * 32 < vec_per_row) u[i] = src[v0 + i * 32];
#pragma unroll
    for (int j = 0; j < kScatterMaxK; ++j) {
      if (j >= k) break;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (v0 + i * 32 < vec_per_row) dst[j][v0 + i * 32] = u[i];
    }
  }
}

// The same scatter with the bulk-copy engine (rows a multiple of 16 bytes):
// each warp loads its token's row into shared memory with one asynchronous
// bulk copy, waits for it on an mbarrier (bounded), and lanes j < k each issue
// one bulk store of the whole row to position inv_perm[t, j]; before the
// buffer takes the next row, the lanes wait until their stores have read it.
// The warp issues a handful of copy instructions per row instead of 32 vector
// stores per lane per 2 KB, and the copies run while it waits.
constexpr int kBulkWarps = 4;

__global__ void __launch_bounds__(kBulkWarps * 32) scatter_rows_bulk_kernel(
    const unsigned char* __restrict__ x, const int32_t* __restrict__ inv_perm, int T, int k,
    int row_bytes, unsigned char* __restrict__ x_perm, int32_t* status) {
  extern __shared__ __align__(128) unsigned char bulk_rows[];  // [kBulkWarps][row_bytes]
  __shared__ __align__(8) uint64_t bar[kBulkWarps];
  __shared__ int32_t local_status;  // the waits' status word when the caller passes none
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) local_status = 0;
  if (lane == 0) ptx::mbar_init(ptx::smem_addr(&bar[warp]), 1);
  ptx::fence_barrier_init();
  __syncthreads();
  int32_t* st = status ? status : &local_status;
  const uint32_t buf = ptx::smem_addr(bulk_rows + (size_t)warp * row_bytes);
  const uint32_t b = ptx::smem_addr(&bar[warp]);
  const int R = T * k;
  uint32_t phase = 0;
  for (int t = blockIdx.x * kBulkWarps + warp; t < T; t += gridDim.x * kBulkWarps) {
    const int mine = lane < k ? inv_perm[(int64_t)t * k + lane] : 0;
    if (__any_sync(0xffffffffu, (unsigned)mine >= (unsigned)R)) {
      if (lane == 0) record_bad_index(status);
      continue;
    }
    ptx::bulk_wait_read0();  // this lane's stores of the previous row have read the buffer
    __syncwarp();
    int ok = 1;
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(b, (uint32_t)row_bytes);
      ptx::bulk_load(buf, x + (int64_t)t * row_bytes, (uint32_t)row_bytes, b);
      ok = ptx::mbar_wait(b, phase, st, kSiteRowCopy);
    }
    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    phase ^= 1;
    if (lane < k) {
      ptx::bulk_store(x_perm + (int64_t)mine * row_bytes, buf, (uint32_t)row_bytes);
      ptx::bulk_commit();
    }
  }
  ptx::bulk_wait_all();  // every store has completed before the block's shared memory goes
}

// ---- small batches: permutation and row gather in one launch ---------------
// For R = T*k <= 1024 routed rows (decode-sized batches) the three launches of
// the chunked permutation plus the gather cost more than the work. Here block
// b handles routed pair b = (token b / k, slot b % k): every block histograms
// all R expert ids in shared memory (counts, hence offsets, do not depend on
// the order of the atomic adds), takes the exclusive scan, ranks its pair
// among the earlier pairs of the same expert (the pairs are in token order, so
// that rank is the token-ascending position) and copies its token's row(s)
// to the permuted position. The result equals the chunked permutation's.
constexpr int kSmallPermThreads = 128;

__global__ void __launch_bounds__(kSmallPermThreads) permute_gather_small_kernel(
    const int32_t* __restrict__ ids, int T, int E, int k, int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm_token, int32_t* __restrict__ inv_perm, const uint4* __restrict__ x,
    int x_vecs, uint4* __restrict__ x_perm, const uint32_t* __restrict__ x2, int x2_words,
    uint32_t* __restrict__ x2_perm, int32_t* status) {
  extern __shared__ int32_t small_smem[];
  const int R = T * k;
  int32_t* sid = small_smem;        // [R] expert of each pair (-1: out of range)
  int32_t* soff = small_smem + R;   // [E + 1] counts, then exclusive offsets
  __shared__ int32_t red[kSmallPermThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e <= E; e += kSmallPermThreads) soff[e] = 0;
  __syncthreads();
  for (int i = tid; i < R; i += kSmallPermThreads) {
    int e = ids[i];
    if ((unsigned)e >= (unsigned)E) {
      if (blockIdx.x == 0) record_bad_index(status);
      e = -1;
    } else {
      atomicAdd(&soff[e], 1);
    }
    sid[i] = e;
  }
  __syncthreads();
  // exclusive scan of soff[0..E) (E <= 1024): each thread sums a run of
  // consecutive experts, the runs are scanned across the block
  {
    constexpr int NT = kSmallPermThreads;
    const int per = (E + NT - 1) / NT, lo = min(tid * per, E), hi = min(lo + per, E);
    int run = 0;
    for (int e = lo; e < hi; ++e) run += soff[e];
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += red[w];
    int acc = base + incl - run;  // exclusive prefix of this run
    __syncthreads();
    for (int e = lo; e < hi; ++e) {
      const int c = soff[e];
      soff[e] = acc;
      acc += c;
    }
    if (tid == NT - 1) soff[E] = acc;
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = tid; e <= E; e += kSmallPermThreads) offsets[e] = soff[e];
  const int b = blockIdx.x, t = b / k, e = sid[b];
  if (e < 0) return;
  if (tid == 0)  // an expert repeated within the token is recorded (once, by its later slot)
    for (int p = t * k; p < b; ++p)
      if (sid[p] == e) {
        record_bad_index(status);
        break;
      }
  // rank of pair b among the earlier pairs that chose the same expert
  int cnt = 0;
  for (int p = tid; p < b; p += kSmallPermThreads) cnt += sid[p] == e;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  __syncthreads();
  if (lane == 0) red[warp] = cnt;
  __syncthreads();
  int rank = 0;
#pragma unroll
  for (int w = 0; w < kSmallPermThreads / 32; ++w) rank += red[w];
  const int pos = soff[e] + rank;
  if (tid == 0) {
    perm_token[pos] = t;
    inv_perm[b] = pos;
  }
  if (x) {
    const uint4* src = x + (int64_t)t * x_vecs;
    uint4* dst = x_perm + (int64_t)pos * x_vecs;
    for (int v = tid; v < x_vecs; v += kSmallPermThreads) dst[v] = src[v];
  }
  if (x2) {
    const uint32_t* src = x2 + (int64_t)t * x2_words;
    uint32_t* dst = x2_perm + (int64_t)pos * x2_words;
    for (int v = tid; v < x2_words; v += kSmallPermThreads) dst[v] = src[v];
  }
}

// ---- weighted combine ---------------------------------------------------------
// "Mixture of Experts (MoE): a practical explanation", section 5 pseudocode
// `y = sum_i weights_i * expert_i(x)`:
//   out[t, c] = sum_{j ascending} w[t, j] * y_perm[inv_perm[t, j], c]  (fp32) -> bf16
// Each thread owns 8 consecutive columns (one 16-byte vector) of one token.
// The routed rows are read four at a time, all four loads issued before the
// first is used; the sums still run in ascending j.
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y_perm,
                                                      const float* __restrict__ w,
                                                      const int32_t* __restrict__ inv_perm, int T,
                                                      int vec_per_row, int k,
                                                      uint4* __restrict__ out, int32_t* status) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)T * vec_per_row) return;
  const int t = (int)(i / vec_per_row), v = (int)(i % vec_per_row);
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
  for (int j0 = 0; j0 < k; j0 += 4) {
    uint4 y[4];
    float wj[4];
    bool use[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u;
      use[u] = false;
      if (j < k) {
        wj[u] = __ldg(w + (int64_t)t * k + j);
        const int p = __ldg(inv_perm + (int64_t)t * k + j);
        if ((unsigned)p >= (unsigned)(T * k)) {
          record_bad_index(status);
        } else {
          y[u] = __ldg(y_perm + (int64_t)p * vec_per_row + v);
          use[u] = true;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (!use[u]) continue;
      acc[0] = __fmaf_rn(wj[u], bf16lo_to_f32(y[u].x), acc[0]);
      acc[1] = __fmaf_rn(wj[u], bf16hi_to_f32(y[u].x), acc[1]);
      acc[2] = __fmaf_rn(wj[u], bf16lo_to_f32(y[u].y), acc[2]);
      acc[3] = __fmaf_rn(wj[u], bf16hi_to_f32(y[u].y), acc[3]);
      acc[4] = __fmaf_rn(wj[u], bf16lo_to_f32(y[u].z), acc[4]);
      acc[5] = __fmaf_rn(wj[u], bf16hi_to_f32(y[u].z), acc[5]);
      acc[6] = __fmaf_rn(wj[u], bf16lo_to_f32(y[u].w), acc[6]);
      acc[7] = __fmaf_rn(wj[u], bf16hi_to_f32(y[u].w), acc[7]);
    }
  }
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  out[i] = o;
}

// ---- launchers ------------------------------------------------------------------
int64_t permute_scratch_bytes(int T, int E) {
  int64_t nchunks = ceil_div(T, 32);
  return align_up(nchunks * E * 4, 256) * 2 + align_up((int64_t)E * 4, 256);
}

cudaError_t launch_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets,
                           int32_t* perm_token, int32_t* inv_perm, void* scratch,
                           int32_t* status, cudaStream_t s) {
  const int nchunks = (int)ceil_div(T, 32);
  char* sp = static_cast<char*>(scratch);
  uint32_t* masks = reinterpret_cast<uint32_t*>(sp);
  sp += align_up((int64_t)nchunks * E * 4, 256);
  int32_t* chunk_base = reinterpret_cast<int32_t*>(sp);
  sp += align_up((int64_t)nchunks * E * 4, 256);
  int32_t* counts = reinterpret_cast<int32_t*>(sp);

  const unsigned nblk = (unsigned)ceil_div(nchunks, 4);
  permute_mask_kernel<<<nblk, 128, 4 * E * sizeof(uint32_t), s>>>(ids, T, E, k, nchunks, masks,
                                                                  status);
  note_launch();
  permute_scan_kernel<<<(unsigned)ceil_div(E, 32), 1024, 0, s>>>(masks, E, nchunks, chunk_base,
                                                                   counts);
  note_launch();
  permute_scatter_kernel<<<nblk, 128, (E + 1) * sizeof(int32_t), s>>>(
      ids, masks, chunk_base, counts, T, E, k, nchunks, offsets, perm_token, inv_perm, status);
  note_launch();
  return cudaGetLastError();
}

// Permutation plus the gather of one or two row payloads (row_bytes a
// multiple of 16; row2_bytes a multiple of 4) in one launch, for
// R = T*k <= 1024 and E <= 1024; returns cudaErrorNotSupported otherwise.
cudaError_t launch_permute_gather_small(const int32_t* ids, int T, int E, int k, int32_t* offsets,
                                        int32_t* perm_token, int32_t* inv_perm, const void* x,
                                        int row_bytes, void* x_perm, const void* x2,
                                        int row2_bytes, void* x2_perm, int32_t* status,
                                        cudaStream_t s) {
  const int R = T * k;
  if (R > kSmallPermRows || E > 1024 || (x && row_bytes % 16) || (x2 && row2_bytes % 4))
    return cudaErrorNotSupported;
  const size_t smem = (size_t)(R + E + 1) * sizeof(int32_t);
  permute_gather_small_kernel<<<(unsigned)R, kSmallPermThreads, smem, s>>>(
      ids, T, E, k, offsets, perm_token, inv_perm, static_cast<const uint4*>(x), row_bytes / 16,
      static_cast<uint4*>(x_perm), static_cast<const uint32_t*>(x2), row2_bytes / 4,
      static_cast<uint32_t*>(x2_perm), status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* x, const int32_t* perm_token, int R, int T,
                               int row_bytes, void* x_perm, int32_t* status, cudaStream_t s) {
  if (row_bytes % 16 == 0)
    gather_rows_kernel<uint4><<<(unsigned)ceil_div(R, 8), 256, 0, s>>>(
        static_cast<const uint4*>(x), perm_token, R, T, row_bytes / 16,
        static_cast<uint4*>(x_perm), status);
  else
    gather_rows_kernel<uint32_t><<<(unsigned)ceil_div(R, 8), 256, 0, s>>>(
        static_cast<const uint32_t*>(x), perm_token, R, T, row_bytes / 4,
        static_cast<uint32_t*>(x_perm), status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_scatter_rows(const void* x, const int32_t* inv_perm, int T, int k,
                                int row_bytes, void* x_perm, int32_t* status, cudaStream_t s) {
  if (k > kScatterMaxK) return cudaErrorNotSupported;
  const size_t bulk_smem = (size_t)kBulkWarps * row_bytes;
  if (row_bytes % 16 == 0 && bulk_smem <= 64 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(scatter_rows_bulk_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bulk_smem);
    if (e != cudaSuccess) return e;
    int sms = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks = std::min<int64_t>(ceil_div(T, kBulkWarps), (int64_t)std::max(sms, 1) * 3);
    scatter_rows_bulk_kernel<<<(unsigned)std::max<int64_t>(blocks, 1), kBulkWarps * 32, bulk_smem, s>>>(
        static_cast<const unsigned char*>(x), inv_perm, T, k, row_bytes,
        static_cast<unsigned char*>(x_perm), status);
  } else if (row_bytes % 16 == 0)
    scatter_rows_kernel<uint4><<<(unsigned)ceil_div(T, 8), 256, 0, s>>>(
        static_cast<const uint4*>(x), inv_perm, T, k, row_bytes / 16, static_cast<uint4*>(x_perm),
        status);
  else
    scatter_rows_kernel<uint32_t><<<(unsigned)ceil_div(T, 8), 256, 0, s>>>(
        static_cast<const uint32_t*>(x), inv_perm, T, k, row_bytes / 4,
        static_cast<uint32_t*>(x_perm), status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_combine(const void* y_perm, const float* w, const int32_t* inv_perm, int T,
                           int H, int k, void* out, int32_t* status, cudaStream_t s) {
  const int vpr = H / 8;
  const int64_t n = (int64_t)T * vpr;
  combine_kernel<<<(unsigned)ceil_div(n, 256), 256, 0, s>>>(
      static_cast<const uint4*>(y_perm), w, inv_perm, T, vpr, k, static_cast<uint4*>(out), status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
