// Router linear + top-k + softmax over the chosen logits.
//
// The router is a linear layer with bias (torchtitan GPT-OSS guide, HuggingFace
// weight adapter section: moe.router.gate.weight/bias); the from-scratch GPT-OSS
// write-up's model flow routes each token to its top-4 experts. Gate weights
// are the softmax of the k chosen logits; ties go to the lower expert index.
//
// One CTA handles kTok tokens: the logits tile (kTok x E) is accumulated in
// fp32 registers from bf16 tiles of x and Wr staged in shared memory, then one
// warp per token selects the top k with warp shuffles and writes the
// normalised weights. HBM traffic is x once plus Wr (L2-resident).
#include "common.cuh"

#include <float.h>

namespace moe {
namespace {

constexpr int kTok = 32;      // tokens per CTA
constexpr int kDc = 32;       // reduction chunk staged in shared memory
constexpr int kThreads = 256; // 16 x 16 thread grid: tokens x expert groups

template <int EJ>  // experts per thread: E <= 16 * EJ
__global__ void __launch_bounds__(kThreads) route_kernel(int T, int D, int E, int k, const uint16_t* __restrict__ x,
                                                         const uint16_t* __restrict__ Wr,
                                                         const uint16_t* __restrict__ br, int32_t* __restrict__ topk_idx,
                                                         float* __restrict__ topk_w) {
  constexpr int EP = 16 * EJ;
  constexpr int kWsFloats = EP * (kDc + 1), kLgFloats = kTok * (EP + 1);
  __shared__ float xs[kTok][kDc + 1];
  // The Wr tile and, after the reduction, the logits tile share this buffer.
  __shared__ float buf[kWsFloats > kLgFloats ? kWsFloats : kLgFloats];
  float (*ws)[kDc + 1] = reinterpret_cast<float (*)[kDc + 1]>(buf);
  float (*lg)[EP + 1] = reinterpret_cast<float (*)[EP + 1]>(buf);

  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int t0 = blockIdx.x * kTok;

  float acc[2][EJ];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < EJ; ++j) acc[i][j] = 0.f;

  for (int d0 = 0; d0 < D; d0 += kDc) {
    // x tile: kTok x kDc bf16 = 128 vectors of 8
    if (tid < kTok * kDc / 8) {
      int r = tid / (kDc / 8), c = (tid % (kDc / 8)) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t0 + r < T) v = *reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t0 + r) * D + d0 + c);
      const uint16_t* p = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
      for (int q = 0; q < 8; ++q) xs[r][c + q] = bf16_bits_to_float(p[q]);
    }
    // Wr tile: EP x kDc
    for (int v_id = tid; v_id < EP * kDc / 8; v_id += kThreads) {
      int r = v_id / (kDc / 8), c = (v_id % (kDc / 8)) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < E) v = *reinterpret_cast<const uint4*>(Wr + static_cast<int64_t>(r) * D + d0 + c);
      const uint16_t* p = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
      for (int q = 0; q < 8; ++q) ws[r][c + q] = bf16_bits_to_float(p[q]);
    }
    __syncthreads();
#pragma unroll 8
    for (int dd = 0; dd < kDc; ++dd) {
      float xv0 = xs[ty][dd], xv1 = xs[ty + 16][dd];
#pragma unroll
      for (int j = 0; j < EJ; ++j) {
        float wv = ws[tx + 16 * j][dd];
        acc[0][j] = fmaf(xv0, wv, acc[0][j]);
        acc[1][j] = fmaf(xv1, wv, acc[1][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < EJ; ++j) {
    int e = tx + 16 * j;
    float b = e < E ? bf16_bits_to_float(br[e]) : 0.f;
    lg[ty][e] = acc[0][j] + b;
    lg[ty + 16][e] = acc[1][j] + b;
  }
  __syncthreads();

  // Top-k: one warp per token, lanes own experts lane, lane+32, ...
  const int warp = tid / 32, lane = tid % 32;
  constexpr int kPer = (EP + 31) / 32;
  for (int r = warp; r < kTok; r += kThreads / 32) {
    const int t = t0 + r;
    if (t >= T) break;
    float v[kPer];
#pragma unroll
    for (int m = 0; m < kPer; ++m) {
      int e = lane + 32 * m;
      v[m] = e < E ? lg[r][e] : -FLT_MAX;
    }
    bool taken[kPer];
#pragma unroll
    for (int m = 0; m < kPer; ++m) taken[m] = (lane + 32 * m) >= E;
    float sel_v = 0.f, v0 = 0.f, denom = 0.f;
    int sel_e = 0;
    for (int j = 0; j < k; ++j) {
      // local best among untaken: (value desc, index asc)
      float bv = -FLT_MAX;
      int be = 0x7fffffff;
#pragma unroll
      for (int m = 0; m < kPer; ++m) {
        int e = lane + 32 * m;
        if (!taken[m] && (v[m] > bv || (v[m] == bv && e < be))) {
          bv = v[m];
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
#pragma unroll
      for (int m = 0; m < kPer; ++m)
        if (lane + 32 * m == be) taken[m] = true;
      if (j == 0) v0 = bv;
      float ex = __expf(bv - v0);
      denom += ex;
      if (lane == j) {
        sel_v = ex;
        sel_e = be;
      }
    }
    if (lane < k) {
      topk_idx[static_cast<int64_t>(t) * k + lane] = sel_e;
      topk_w[static_cast<int64_t>(t) * k + lane] = sel_v / denom;
    }
  }
}

}  // namespace

cudaError_t launch_route(const moe_dims_t& d, const uint16_t* x, const uint16_t* Wr, const uint16_t* br,
                         int32_t* topk_idx, float* topk_w, cudaStream_t s) {
  dim3 grid((d.T + kTok - 1) / kTok);
  if (d.E <= 16)
    route_kernel<1><<<grid, kThreads, 0, s>>>(d.T, d.D, d.E, d.k, x, Wr, br, topk_idx, topk_w);
  else if (d.E <= 32)
    route_kernel<2><<<grid, kThreads, 0, s>>>(d.T, d.D, d.E, d.k, x, Wr, br, topk_idx, topk_w);
  else if (d.E <= 64)
    route_kernel<4><<<grid, kThreads, 0, s>>>(d.T, d.D, d.E, d.k, x, Wr, br, topk_idx, topk_w);
  else if (d.E <= 128)
    route_kernel<8><<<grid, kThreads, 0, s>>>(d.T, d.D, d.E, d.k, x, Wr, br, topk_idx, topk_w);
  else
    route_kernel<16><<<grid, kThreads, 0, s>>>(d.T, d.D, d.E, d.k, x, Wr, br, topk_idx, topk_w);
  return cudaGetLastError();
}

}  // namespace moe
