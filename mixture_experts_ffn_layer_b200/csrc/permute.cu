// Token permutation grouped by expert, the row gather, and the weighted combine.
//
// The torchtitan GPT-OSS guide ("grouped matrix multiplication") feeds the
// grouped GEMMs with rows sorted by expert and offsets = cumsum of
// num_tokens_per_expert, computed without a device-to-host sync. Here the
// R = T*k assignments a = t*k + j are sorted stably by expert in three launches:
//   1. per-block histograms of `chunk` assignments (shared-memory counters);
//   2. a column scan per expert turns the histograms into per-block prefixes
//      and per-expert totals (counts);
//   3. each block takes its per-expert base from its prefix plus the
//      exclusive scan of the totals over experts, then ranks its assignments
//      in order with warp match/popc and per-warp counts -- the position of
//      every assignment is fixed by (expert, a), never by atomics.
// The combine (from-scratch GPT-OSS write-up, "weighted combination") is a
// gather: every output row sums its k expert rows in slot order.
#include "common.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(kPermThreads) perm_hist_kernel(const int32_t* __restrict__ idx, int64_t R, int E,
                                                                 int chunk, int32_t* __restrict__ block_counts,
                                                                 int* status) {
  __shared__ int cnt[256];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int64_t a0 = static_cast<int64_t>(blockIdx.x) * chunk;
  const int64_t a1 = min(a0 + chunk, R);
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

// Column scan of the block histograms, one CTA per expert e: block_counts[b][e]
// becomes the number of assignments to e in blocks before b (exclusive prefix
// over blocks, in place), and counts[e] the total.
__global__ void __launch_bounds__(kPermThreads) perm_scan_kernel(int32_t* __restrict__ block_counts, int nblk, int E,
                                                                 int32_t* __restrict__ counts) {
  constexpr int kWarps = kPermThreads / 32;
  __shared__ int wsum[kWarps];
  const int e = blockIdx.x, tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  int carry = 0;
  for (int b0 = 0; b0 < nblk; b0 += kPermThreads) {
    const int b = b0 + tid;
    const int v = b < nblk ? block_counts[static_cast<int64_t>(b) * E + e] : 0;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += u;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int ws = wsum[w];
      if (w < warp) before += ws;
      total += ws;
    }
    if (b < nblk) block_counts[static_cast<int64_t>(b) * E + e] = carry + before + incl - v;
    carry += total;
    __syncthreads();
  }
  if (tid == 0) counts[e] = carry;
}

// Stable ranking of the assignments [a0, a0 + n) into perm / inv, in order,
// kPermThreads at a time: base[e] (shared) holds the next position for expert
// e and advances past each group; wcnt is per-warp scratch. Warp match/popc
// and per-warp counts fix each position from (expert, a), never by atomics.
// Every thread of the block calls it.
__device__ void rank_assignments(const int32_t* __restrict__ idx, int64_t R, int E, int64_t a0, int n, int* base,
                                 int (*wcnt)[256], int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  constexpr int kWarps = kPermThreads / 32;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int sub = 0; sub < n; sub += kPermThreads) {
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

// Exclusive scan of c (one value per thread, E <= 256 = the block size) over
// the experts: returns thread tid's prefix. scratch: kPermThreads / 32 ints.
__device__ int expert_prefix(int c, int* scratch) {
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  int incl = c;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += u;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += scratch[w];
  __syncthreads();
  return before + incl - c;
}

__global__ void __launch_bounds__(kPermThreads) perm_scatter_kernel(const int32_t* __restrict__ idx, int64_t R, int E,
                                                                    int chunk, const int32_t* __restrict__ block_pre,
                                                                    const int32_t* __restrict__ counts,
                                                                    int32_t* __restrict__ offsets,
                                                                    int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  constexpr int kWarps = kPermThreads / 32;
  __shared__ int base[256];
  __shared__ int wcnt[kWarps][256];
  const int tid = threadIdx.x;
  const int blk = blockIdx.x;
  // Expert offsets (exclusive scan of the totals over experts) plus this
  // block's prefix over the blocks before it.
  const int c = tid < E ? counts[tid] : 0;
  const int off = expert_prefix(c, &wcnt[0][0]);
  if (tid < E) {
    base[tid] = off + block_pre[static_cast<int64_t>(blk) * E + tid];
    if (blk == 0) {
      offsets[tid] = off;
      if (tid == E - 1) offsets[E] = off + c;
    }
  }
  __syncthreads();
  rank_assignments(idx, R, E, static_cast<int64_t>(blk) * chunk, chunk, base, wcnt, perm, inv);
}

// The whole permutation in one block, for batches of at most kPermSingleMax
// assignments (decode-sized): histogram in shared memory, counts and offsets,
// then the same stable ranking over all R assignments -- one launch instead
// of three, the same perm / inv / counts / offsets.
constexpr int kPermSingleMax = 1024;

__global__ void __launch_bounds__(kPermThreads) perm_single_kernel(const int32_t* __restrict__ idx, int64_t R, int E,
                                                                   int32_t* __restrict__ counts,
                                                                   int32_t* __restrict__ offsets,
                                                                   int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                                   int* status) {
  constexpr int kWarps = kPermThreads / 32;
  __shared__ int base[256];
  __shared__ int wcnt[kWarps][256];
  const int tid = threadIdx.x;
  for (int e = tid; e < 256; e += kPermThreads) base[e] = 0;
  __syncthreads();
  for (int64_t a = tid; a < R; a += kPermThreads) {
    const int e = idx[a];
    if (e >= 0 && e < E)
      atomicAdd(&base[e], 1);
    else
      record_status(status, MOE_ERR_DEVICE_BOUNDS);
  }
  __syncthreads();
  const int c = tid < E ? base[tid] : 0;
  const int off = expert_prefix(c, &wcnt[0][0]);
  if (tid < E) {
    counts[tid] = c;
    offsets[tid] = off;
    if (tid == E - 1) offsets[E] = off + c;
    base[tid] = off;
  }
  __syncthreads();
  rank_assignments(idx, R, E, 0, static_cast<int>(R), base, wcnt, perm, inv);
}

// x_perm[r, :] = x[perm[r] / k, :]. Grid (row, chunk block): each thread
// copies one 32-byte vector (16 bf16) of one row.
__global__ void gather_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm,
                                   uint16_t* __restrict__ x_perm, int64_t R, int k, int D, int* status) {
  const int64_t r = blockIdx.x;
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= D / 16) return;
  const int32_t a = perm[r];
  uint32_t v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (a >= 0 && a < R)
    sm100::ld_global_v8u(x + static_cast<int64_t>(a / k) * D + 16 * c, v);
  else if (c == 0)
    record_status(status, MOE_ERR_DEVICE_BOUNDS);
  sm100::st_global_v8u(x_perm + r * D + 16 * c, v);
}

// y[t, :] = bf16( sum_j o_perm[inv[t*k + j], :] ), fp32 sum in slot order.
// Grid (token, chunk block): each thread sums k 32-byte fp32 vectors and
// stores 8 bf16.
__global__ void combine_kernel(const float* __restrict__ o_perm, const int32_t* __restrict__ inv,
                               uint16_t* __restrict__ y, int k, int64_t R, int D, int* status) {
  const int64_t t = blockIdx.x;
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= D / 8) return;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int j = 0; j < k; ++j) {
    const int32_t r = __ldg(inv + t * k + j);
    if (r < 0 || r >= R) {
      if (c == 0) record_status(status, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    float v[8];
    sm100::ld_global_v8f(o_perm + static_cast<int64_t>(r) * D + 8 * c, v);
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] += v[q];
  }
  uint4 out;
  out.x = pack_bf16x2(acc[0], acc[1]);
  out.y = pack_bf16x2(acc[2], acc[3]);
  out.z = pack_bf16x2(acc[4], acc[5]);
  out.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4*>(y + t * D + 8 * c) = out;
}

// Threads per block for n vectors per row: a multiple of 32, at most 256.
int row_block(int n) { return n >= 256 ? 256 : (n + 31) / 32 * 32; }


}  // namespace

cudaError_t launch_permute(const moe_dims_t& d, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* inv, int32_t* block_counts, int* status, cudaStream_t s,
                           int chunk) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  if (R <= kPermSingleMax) {
    perm_single_kernel<<<1, kPermThreads, 0, s>>>(topk_idx, R, d.E, counts, offsets, perm, inv, status);
    return cudaGetLastError();
  }
  const int nblk = static_cast<int>((R + chunk - 1) / chunk);
  perm_hist_kernel<<<nblk, kPermThreads, 0, s>>>(topk_idx, R, d.E, chunk, block_counts, status);
  perm_scan_kernel<<<d.E, kPermThreads, 0, s>>>(block_counts, nblk, d.E, counts);
  perm_scatter_kernel<<<nblk, kPermThreads, 0, s>>>(topk_idx, R, d.E, chunk, block_counts, counts, offsets, perm,
                                                    inv);
  return cudaGetLastError();
}

cudaError_t launch_gather(const moe_dims_t& d, const uint16_t* x, const int32_t* perm, uint16_t* x_perm, int* status,
                          cudaStream_t s) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  const int n = d.D / 16, bs = row_block(n);
  const dim3 grid(static_cast<unsigned>(R), (n + bs - 1) / bs);
  gather_rows_kernel<<<grid, bs, 0, s>>>(x, perm, x_perm, R, d.k, d.D, status);
  return cudaGetLastError();
}

cudaError_t launch_combine(const moe_dims_t& d, const float* o_perm, const int32_t* inv, uint16_t* y, int* status,
                           cudaStream_t s) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  const int n = d.D / 8, bs = row_block(n);
  combine_kernel<<<dim3(static_cast<unsigned>(d.T), (n + bs - 1) / bs), bs, 0, s>>>(o_perm, inv, y, d.k, R, d.D,
                                                                                    status);
  return cudaGetLastError();
}

}  // namespace moe

// ---------------------------------------------------------------------------
// moe_permute_noalloc: the permutation for callers that cannot allocate.
//
// The only scratch the permutation needs is the per-block expert histogram
// (one int32 per (block of kPermChunkNoAlloc = 2048 assignments, expert)). Here it lives in
// a fixed array in the library's own device memory instead of a caller
// workspace. Every GPU that loads the library holds this array until the
// process exits. Calls share it: each call overwrites every entry it reads
// (the histogram kernel writes all of its block's counts, so nothing has to
// start at zero), and two calls whose kernels overlap on the GPU -- on two
// streams, or on two host threads -- race on it.
#include <cudaTypedefs.h>

#include <mutex>

namespace moe {
namespace {

// 65536 int32 = 256 KB: enough for ceil(T*k / 2048) * E <= 65536, e.g.
// T*k <= 4M assignments at E = 32, or <= 512K at E = 256.
constexpr int64_t kNoAllocScratchInts = int64_t(1) << 16;
__device__ __align__(256) int32_t g_noalloc_block_counts[kNoAllocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct ScratchAddr {
  unsigned long long ctx_id;  // the CUDA context the address belongs to (0 = none yet)
  int32_t* ptr;
};
ScratchAddr g_noalloc_addr[kMaxDevices] = {};

// Unique id of the calling thread's current CUDA context (cuCtxGetId: never
// reused within the process), fetched through the runtime's driver entry
// point query so the library needs no libcuda link.
bool current_ctx_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  if (!get_current || !get_id) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess || !a)
      return false;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess || !b)
      return false;
    get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(a);
    get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(b);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current device's context. The
// host-side name of a __device__ array is only a stand-in, so the address is
// looked up with the device current, once per context, and cached. A new
// context on the device (after cudaDeviceReset, for instance, the module is
// loaded again and the array may move) has a new id and gets a new lookup.
moe_status_t noalloc_scratch(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  unsigned long long id = 0;
  const bool have_ctx = current_ctx_id(&id) && id != 0;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  ScratchAddr& a = g_noalloc_addr[dev];
  if (!have_ctx || a.ctx_id != id || !a.ptr) {
    // the lookup also binds the device's primary context to this thread if
    // no runtime call has done so yet
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_block_counts) != cudaSuccess || !p) return MOE_ERR_CUDA;
    if (!current_ctx_id(&id) || id == 0) return MOE_ERR_CUDA;
    a.ptr = static_cast<int32_t*>(p);
    a.ctx_id = id;
  }
  *out = a.ptr;
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
  if (static_cast<int64_t>(perm_blocks(R, kPermChunkNoAlloc)) * d.E > kNoAllocScratchInts) return MOE_ERR_UNSUPPORTED;
  int32_t* scratch = nullptr;
  const moe_status_t st = noalloc_scratch(&scratch);
  if (st != MOE_OK) return st;
  return launch_permute(d, topk_idx, counts, offsets, perm, inv, scratch, nullptr, static_cast<cudaStream_t>(stream),
                        kPermChunkNoAlloc) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
