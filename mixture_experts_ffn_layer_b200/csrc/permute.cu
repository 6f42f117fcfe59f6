// Token permutation grouped by expert, the row gather, and the weighted combine.
//
// The torchtitan GPT-OSS guide ("grouped matrix multiplication") feeds the
// grouped GEMMs with rows sorted by expert and offsets = cumsum of
// num_tokens_per_expert, computed without a device-to-host sync. Here the
// R = T*k assignments a = t*k + j are sorted stably by expert in two launches:
//   1. per-block histograms of kPermChunk assignments (shared-memory counters);
//   2. each block derives its per-expert base from the histograms of the
//      blocks before it plus the exclusive scan over experts, then ranks its
//      assignments in order with warp match/popc and per-warp counts -- the
//      position of every assignment is fixed by (expert, a), never by atomics.
// The combine (from-scratch GPT-OSS write-up, "weighted combination") is a
// gather: every output row sums its k expert rows in slot order.
#include "common.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(kPermThreads) perm_hist_kernel(const int32_t* __restrict__ idx, int64_t R, int E,
                                                                 int32_t* __restrict__ block_counts, int* status) {
  __shared__ int cnt[256];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int64_t a0 = static_cast<int64_t>(blockIdx.x) * kPermChunk;
  const int64_t a1 = min(a0 + kPermChunk, R);
  for (int64_t a = a0 + threadIdx.x; a < a1; a += blockDim.x) {
    int e = idx[a];
    if (e >= 0 && e < E)
      atomicAdd(&cnt[e], 1);
    else
      record_status(status, MOE_ERR_DEVICE_BOUNDS);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) block_counts[static_cast<int64_t>(blockIdx.x) * E + e] = cnt[e];
}

__global__ void __launch_bounds__(kPermThreads) perm_scatter_kernel(const int32_t* __restrict__ idx, int64_t R, int E,
                                                                    const int32_t* __restrict__ block_counts,
                                                                    int32_t* __restrict__ counts,
                                                                    int32_t* __restrict__ offsets,
                                                                    int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  constexpr int kWarps = kPermThreads / 32;
  __shared__ int tot[256];
  __shared__ int base[256];
  __shared__ int wcnt[kWarps][256];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int nblk = gridDim.x, blk = blockIdx.x;

  // Per-expert totals and this block's prefix over the blocks before it.
  int pre = 0;
  if (tid < E) {
    int total = 0;
    for (int b = 0; b < nblk; ++b) {
      int c = block_counts[static_cast<int64_t>(b) * E + tid];
      if (b < blk) pre += c;
      total += c;
    }
    tot[tid] = total;
  }
  __syncthreads();
  if (tid < E) {
    int off = 0;
    for (int e = 0; e < tid; ++e) off += tot[e];
    base[tid] = off + pre;
    if (blk == 0) {
      counts[tid] = tot[tid];
      offsets[tid] = off;
      if (tid == E - 1) offsets[E] = off + tot[tid];
    }
  }
  __syncthreads();

  const int64_t a0 = static_cast<int64_t>(blk) * kPermChunk;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int sub = 0; sub < kPermChunk; sub += kPermThreads) {
    for (int i = tid; i < kWarps * 256; i += kPermThreads) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    const int64_t a = a0 + sub + tid;
    int e = a < R ? idx[a] : -1;
    const bool valid = e >= 0 && e < E;
    const int key = valid ? e : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int rank = __popc(peers & lt_mask);
    if (valid && rank == 0) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    if (valid) {
      int pos = base[e] + rank;
      for (int w = 0; w < warp; ++w) pos += wcnt[w][e];
      perm[pos] = static_cast<int32_t>(a);
      inv[a] = pos;
    } else if (a < R) {
      inv[a] = -1;
    }
    __syncthreads();
    if (tid < E) {
      int s = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += wcnt[w][tid];
      base[tid] += s;
    }
    __syncthreads();
    if (a0 + sub + kPermThreads >= R) break;
  }
}

// x_perm[r, :] = x[perm[r] / k, :], one 16-byte vector per thread.
__global__ void gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm, uint4* __restrict__ x_perm,
                                   int64_t R, int k, int T, int vec_per_row, int* status) {
  const int64_t n = R * vec_per_row;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / vec_per_row;
    const int c = static_cast<int>(i - r * vec_per_row);
    const int32_t a = perm[r];
    uint4 v = make_uint4(0, 0, 0, 0);
    if (a >= 0 && a < R) {
      v = x[static_cast<int64_t>(a / k) * vec_per_row + c];
    } else if (c == 0) {
      record_status(status, MOE_ERR_DEVICE_BOUNDS);
    }
    x_perm[i] = v;
  }
}

// y[t, :] = bf16( sum_j o_perm[inv[t*k + j], :] ), fp32 sum in slot order;
// one thread per 8 outputs (two 16-byte fp32 loads per slot, one bf16 store).
__global__ void combine_kernel(const float4* __restrict__ o_perm, const int32_t* __restrict__ inv,
                               uint4* __restrict__ y, int T, int k, int64_t R, int vec_per_row, int* status) {
  const int64_t n = static_cast<int64_t>(T) * vec_per_row;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / vec_per_row;
    const int c = static_cast<int>(i - t * vec_per_row);
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int32_t r = inv[t * k + j];
      if (r < 0 || r >= R) {
        if (c == 0) record_status(status, MOE_ERR_DEVICE_BOUNDS);
        continue;
      }
      const float4* src = o_perm + (static_cast<int64_t>(r) * vec_per_row + c) * 2;
      const float4 v0 = src[0], v1 = src[1];
      acc[0] += v0.x;
      acc[1] += v0.y;
      acc[2] += v0.z;
      acc[3] += v0.w;
      acc[4] += v1.x;
      acc[5] += v1.y;
      acc[6] += v1.z;
      acc[7] += v1.w;
    }
    uint4 out;
    out.x = pack_bf16x2(acc[0], acc[1]);
    out.y = pack_bf16x2(acc[2], acc[3]);
    out.z = pack_bf16x2(acc[4], acc[5]);
    out.w = pack_bf16x2(acc[6], acc[7]);
    y[i] = out;
  }
}

int grid_for(int64_t n, int threads) {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  int64_t blocks = (n + threads - 1) / threads;
  int64_t cap = static_cast<int64_t>(sms) * 8;
  return static_cast<int>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace

cudaError_t launch_permute(const moe_dims_t& d, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* inv, int32_t* block_counts, int* status, cudaStream_t s) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  const int nblk = perm_blocks(R);
  perm_hist_kernel<<<nblk, kPermThreads, 0, s>>>(topk_idx, R, d.E, block_counts, status);
  perm_scatter_kernel<<<nblk, kPermThreads, 0, s>>>(topk_idx, R, d.E, block_counts, counts, offsets, perm, inv);
  return cudaGetLastError();
}

cudaError_t launch_gather(const moe_dims_t& d, const uint16_t* x, const int32_t* perm, uint16_t* x_perm, int* status,
                          cudaStream_t s) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  const int vpr = d.D / 8;
  const int threads = 256;
  gather_rows_kernel<<<grid_for(R * vpr, threads), threads, 0, s>>>(reinterpret_cast<const uint4*>(x), perm,
                                                                     reinterpret_cast<uint4*>(x_perm), R, d.k, d.T,
                                                                     vpr, status);
  return cudaGetLastError();
}

cudaError_t launch_combine(const moe_dims_t& d, const float* o_perm, const int32_t* inv, uint16_t* y, int* status,
                           cudaStream_t s) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  const int vpr = d.D / 8;
  const int threads = 256;
  combine_kernel<<<grid_for(static_cast<int64_t>(d.T) * vpr, threads), threads, 0, s>>>(
      reinterpret_cast<const float4*>(o_perm), inv, reinterpret_cast<uint4*>(y), d.T, d.k, R, vpr, status);
  return cudaGetLastError();
}

}  // namespace moe

// ---------------------------------------------------------------------------
// moe_permute_noalloc: the permutation for callers that cannot allocate.
//
// The only scratch the permutation needs is the per-block expert histogram
// (one int32 per (block of kPermChunk assignments, expert)). Here it lives in
// a fixed array in the library's own device memory instead of a caller
// workspace. Every GPU that loads the library holds this array until the
// process exits. Calls share it: each call overwrites every entry it reads
// (the histogram kernel writes all of its block's counts, so nothing has to
// start at zero), and two calls whose kernels overlap on the GPU -- on two
// streams, or on two host threads -- race on it.
#include <mutex>

namespace moe {
namespace {

// 65536 int32 = 256 KB: enough for ceil(T*k / 2048) * E <= 65536, e.g.
// T*k <= 4M assignments at E = 32, or <= 512K at E = 256.
constexpr int64_t kNoAllocScratchInts = int64_t(1) << 16;
__device__ __align__(256) int32_t g_noalloc_block_counts[kNoAllocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
int32_t* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. The host-side
// name of a __device__ array is only a stand-in, so the address is looked up
// once per device (with that device current) and cached.
moe_status_t noalloc_scratch(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_block_counts) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_permute_noalloc(moe_dims_t d, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                                            int32_t* perm, int32_t* inv, void* stream) {
  using namespace moe;
  const moe_status_t dims_ok = moe_check_dims(d);
  if (dims_ok != MOE_OK) return dims_ok;
  if (!topk_idx || !counts || !offsets || !perm || !inv) return MOE_ERR_INVALID_ARG;
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  if (static_cast<int64_t>(perm_blocks(R)) * d.E > kNoAllocScratchInts) return MOE_ERR_UNSUPPORTED;
  int32_t* scratch = nullptr;
  const moe_status_t st = noalloc_scratch(&scratch);
  if (st != MOE_OK) return st;
  return launch_permute(d, topk_idx, counts, offsets, perm, inv, scratch, nullptr, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
