// Router linear + top-k + softmax over the chosen logits, on the tensor cores.
//
// The router is a linear layer with bias (torchtitan GPT-OSS guide, HuggingFace
// weight adapter section: moe.router.gate.weight/bias); the from-scratch GPT-OSS
// write-up's model flow routes each token to its top-4 experts. Gate weights
// are the softmax of the k chosen logits; ties go to the lower expert index.
//
// The logits are a dense contraction (T x D) . (D x E), so each CTA computes a
// 128-token tile of them with tcgen05.mma (M=128, N=E rounded up to 16, K=D)
// into TMEM, fed by TMA (x rows and all of Wr, 64-wide K slices, 128-byte
// swizzle, a ring as deep as shared memory allows: only T/128 CTAs stream x). Its epilogue is one thread per token (= TMEM lane):
// it streams the token's E logits out of TMEM, adds the bias, keeps a sorted
// top-k in registers and writes the normalised gate weights. x is read once
// from HBM; Wr stays L2-resident.
// With fewer 128-token tiles than SMs (decode batches) the contraction is also
// split along K across CTAs so that the SMs all stream x: each split writes
// its fp32 partial logits, and a second kernel (one block per token) sums the
// splits in a fixed order, adds the bias and takes the same top-k / softmax,
// so the result is deterministic for given sizes.
#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

#include <float.h>

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = 128, BK = 64, kMaxStages = 12, kThreads = 192, kMaxK = 8;
// Two warps issue the MMAs, each into its own accumulator (even / odd 16-wide
// K slices), added in that order by the epilogue: a tcgen05.commit stalls the
// issuing warp's MMA stream, and with N = E these MMAs are short.
constexpr int kIssuers = 2;
constexpr int kABytes = BM * BK * 2;
constexpr uint64_t kWaitNs = 1000000000ull;

struct RouteParams {
  int T, D, E, k;
  int n_pad;        // MMA N: E rounded up to a multiple of 16
  int stages;       // TMA ring depth (as many as fit: few CTAs stream all of x)
  uint32_t tmem_cols;
  int kb_per;       // K blocks per split (all of them when there is one split)
  int ksplit;       // number of K splits (gridDim.y)
  float* partial;   // (ksplit, T, n_pad) fp32 partial logits when ksplit > 1
  const uint16_t* br;
  int32_t* topk_idx;
  float* topk_w;
  int* status;
};

__global__ void __launch_bounds__(kThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const RouteParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t stage_bytes = kABytes + p.n_pad * BK * 2;
  const int kStages = p.stages;
  uint8_t* ctrl = smem + kStages * stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctrl);  // full[S] empty[S] tfull done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * (2 * kMaxStages + 2));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x / 32), 0), lane = threadIdx.x % 32;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kMaxStages + s); };
  const uint32_t tfull_bar = bar0 + 8u * (2 * kMaxStages);
  const uint32_t done_bar = bar0 + 8u * (2 * kMaxStages + 1);
  const int t0 = blockIdx.x * BM;
  const int KB = (p.D + BK - 1) / BK;
  const int kb0 = blockIdx.y * p.kb_per, kb1 = min(KB, kb0 + p.kb_per);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kIssuers);
    }
    mbar_init(tfull_bar, kIssuers);
    mbar_init(done_bar, kIssuers);
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // TMA producer
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool failed = false;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, kWaitNs)) {
          failed = true;
          break;
        }
        const uint32_t a_dst = smem_u32(smem + stage * stage_bytes);
        mbar_arrive_expect_tx(full_bar(stage), stage_bytes);
        tma_load_2d(a_dst, &tmX, full_bar(stage), kb * BK, t0);
        tma_load_2d(a_dst + kABytes, &tmW, full_bar(stage), kb * BK, 0);
        ++issued;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (failed) {
        record_status(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        const int n = issued < kStages ? issued : kStages;
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < n; ++i) {
          if (--s < 0) {
            s = kStages - 1;
            ph ^= 1u;
          }
          mbar_wait_bounded(full_bar(s), ph, nullptr, kWaitNs);
        }
      }
    }
  } else {
    if (warp <= kIssuers) {
      // ---- MMA issuers (warps 1, 2): whole warp, one lane elected, operands
      // warp-uniform; issuer i takes the K slices kk = i, i + 2 of each block
      const int i = warp - 1;
      const uint32_t idesc = idesc_bf16_f32(BM, p.n_pad);
      const uint32_t dacc = tmem_base + i * p.n_pad;
      int stage = 0;
      uint32_t phase = 0;
      bool failed = false;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(full_bar(stage), phase, abort_flag, kWaitNs))) {
          failed = true;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + stage * stage_bytes);
        const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
        for (int kk = i; kk < BK / 16; kk += kIssuers)
          mma_bf16_elect(dacc, desc_kmajor_sw128(a_addr + kk * 32), desc_kmajor_sw128(b_addr + kk * 32), idesc,
                         (kb != kb0 || kk != i) ? 1u : 0u);
        tc_commit_elect(empty_bar(stage));
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (failed) {
        if (lane == 0) {
          record_status(p.status, MOE_ERR_TIMEOUT);
          *abort_flag = 1;
        }
      } else {
        tc_commit_elect(tfull_bar);
      }
      tc_commit_elect(done_bar);
      mbar_wait_bounded(done_bar, 0, nullptr, kWaitNs);
    }
    if (warp >= 2) {
    // epilogue: thread = token = TMEM lane
    const int q = warp & 3;
    const int t = t0 + q * 32 + lane;
    const bool ok = mbar_wait_bounded(tfull_bar, 0, abort_flag, kWaitNs);
    if (__all_sync(0xffffffffu, ok) && p.ksplit > 1) {
      // partial logits of this K split: the token's n_pad accumulator columns
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      float* dst = p.partial + (static_cast<int64_t>(blockIdx.y) * p.T + t) * p.n_pad;
      for (int c0 = 0; c0 < p.n_pad; c0 += 32) {
        uint32_t v[32], w[32];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (c0 + 8 * j < p.n_pad) {
            tmem_ld_x8(tbase + c0 + 8 * j, v + 8 * j);
            tmem_ld_x8(tbase + p.n_pad + c0 + 8 * j, w + 8 * j);
          }
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(w[i]));
        if (t < p.T) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (c0 + 4 * j < p.n_pad)
              *reinterpret_cast<uint4*>(dst + c0 + 4 * j) = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      }
    } else if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      float topv[kMaxK];
      int tope[kMaxK];
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        topv[j] = -FLT_MAX;
        tope[j] = 0x7fffffff;
      }
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      for (int c0 = 0; c0 < p.n_pad; c0 += 32) {
        uint32_t v[32], w[32];
        // up to four 8-column loads of each accumulator in flight per wait
        // (warp-uniform bounds); the two are added in issuer order
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (c0 + 8 * j < p.n_pad) {
            tmem_ld_x8(tbase + c0 + 8 * j, v + 8 * j);
            tmem_ld_x8(tbase + p.n_pad + c0 + 8 * j, w + 8 * j);
          }
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(w[i]));
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int e = c0 + i;
          if (e < p.E) {
            float cv = __uint_as_float(v[i]) + bf16_bits_to_float(__ldg(p.br + e));
            int ce = e;
            // insert into the sorted list: experts arrive in increasing index,
            // so an equal logit never overtakes (lower index wins ties)
            bool moved = false;
#pragma unroll
            for (int j = 0; j < kMaxK; ++j) {
              if (j < p.k && (moved || cv > topv[j])) {
                const float tv = topv[j];
                const int te = tope[j];
                topv[j] = cv;
                tope[j] = ce;
                cv = tv;
                ce = te;
                moved = true;
              }
            }
          }
        }
      }
      if (t < p.T) {
        float ex[kMaxK], denom = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
          ex[j] = j < p.k ? __expf(topv[j] - topv[0]) : 0.f;
          denom += ex[j];
        }
        const float inv = 1.0f / denom;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
          if (j < p.k) {
            p.topk_idx[static_cast<int64_t>(t) * p.k + j] = tope[j];
            p.topk_w[static_cast<int64_t>(t) * p.k + j] = ex[j] * inv;
          }
        }
      }
    } else if (lane == 0) {
      record_status(p.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

// Sum of the K splits' partial logits, bias, top-k and softmax over the
// chosen logits; one 256-thread block per token. Thread (e, part) sums the
// splits part, part + nparts, ... in increasing order, the parts are added
// in part order (a fixed order: deterministic for given sizes), then warp 0
// selects the top k with lanes over experts. Ties go to the lower expert
// index, as in the fused epilogue.
__global__ void __launch_bounds__(256) route_reduce_topk_kernel(const RouteParams p) {
  __shared__ float part_sum[256];
  __shared__ float logit[256];
  const int t = blockIdx.x;
  const int ep = (p.E + 31) / 32 * 32;  // experts per part, padded to a warp multiple (<= 256)
  const int nparts = 256 / ep;
  const int e = threadIdx.x % ep, part = threadIdx.x / ep;
  float acc = 0.f;
  if (part < nparts && e < p.E) {
    const float* src = p.partial + static_cast<int64_t>(t) * p.n_pad + e;
    const int64_t stride = static_cast<int64_t>(p.T) * p.n_pad;
    int sp = part;
    for (; sp + 3 * nparts < p.ksplit; sp += 4 * nparts) {  // four loads in flight, added in order
      const float a0 = src[sp * stride], a1 = src[(sp + nparts) * stride];
      const float a2 = src[(sp + 2 * nparts) * stride], a3 = src[(sp + 3 * nparts) * stride];
      acc += a0;
      acc += a1;
      acc += a2;
      acc += a3;
    }
    for (; sp < p.ksplit; sp += nparts) acc += src[sp * stride];
  }
  part_sum[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x < ep) {
    float l = 0.f;
    for (int q = 0; q < nparts; ++q) l += part_sum[q * ep + threadIdx.x];
    logit[threadIdx.x] = threadIdx.x < p.E ? l + bf16_bits_to_float(__ldg(p.br + threadIdx.x)) : -FLT_MAX;
  }
  __syncthreads();
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  constexpr int kPerLane = 8;  // E <= 256
  float v[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) v[i] = lane + 32 * i < p.E ? logit[lane + 32 * i] : -FLT_MAX;
  uint32_t taken = 0;
  float topv[kMaxK];
  int tope[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    topv[j] = -FLT_MAX;
    tope[j] = 0x7fffffff;
    if (j >= p.k) continue;
    // this lane's best untaken candidate, then the warp's (value desc, index asc)
    float bv = -FLT_MAX;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int ei = lane + 32 * i;
      if (ei < p.E && !(taken >> i & 1u) && v[i] > bv) {  // strict: lower index wins ties
        bv = v[i];
        be = ei;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    topv[j] = bv;
    tope[j] = be;
    if (be != 0x7fffffff && (be & 31) == lane) taken |= 1u << (be >> 5);
  }
  if (lane == 0) {
    float ex[kMaxK], denom = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      ex[j] = j < p.k ? __expf(topv[j] - topv[0]) : 0.f;
      denom += ex[j];
    }
    const float inv = 1.0f / denom;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < p.k) {
        p.topk_idx[static_cast<int64_t>(t) * p.k + j] = tope[j];
        p.topk_w[static_cast<int64_t>(t) * p.k + j] = ex[j] * inv;
      }
    }
  }
}

}  // namespace

int route_splits(const moe_dims_t& d) {
  // With few token tiles, enough K splits that tiles x splits cover the SMs
  // (one wave of 148 on B200); fixed by the sizes, so results do not depend on
  // the device. Measured on B200: at 64 tiles (8192 tokens) two splits cost
  // more (partials + second launch) than they save, at 1 tile (64 tokens)
  // 45 splits save ~5 us; so only batches of at most 18 tiles split.
  const int tiles = (d.T + BM - 1) / BM, KB = (d.D + BK - 1) / BK;
  if (tiles * 8 > 148) return 1;
  int sp = 148 / tiles;
  if (sp > KB) sp = KB;
  if (sp < 1) sp = 1;
  const int per = (KB + sp - 1) / sp;
  return (KB + per - 1) / per;
}

cudaError_t launch_route(const moe_dims_t& d, const uint16_t* x, const uint16_t* Wr, const uint16_t* br,
                         int32_t* topk_idx, float* topk_w, float* partial, int* status, cudaStream_t s) {
  RouteParams p{};
  p.T = d.T;
  p.D = d.D;
  p.E = d.E;
  p.k = d.k;
  p.n_pad = (d.E + 15) / 16 * 16;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(kIssuers * p.n_pad)) cols <<= 1;  // one accumulator per issuer
  p.tmem_cols = cols;
  p.br = br;
  p.topk_idx = topk_idx;
  p.topk_w = topk_w;
  p.status = status;
  const int KB = (d.D + BK - 1) / BK;
  p.ksplit = route_splits(d);
  p.kb_per = (KB + p.ksplit - 1) / p.ksplit;
  p.partial = partial;
  if (p.ksplit > 1 && !partial) return cudaErrorInvalidValue;
  CUtensorMap tx, tw;
  if (!make_tmap_bf16(&tx, x, d.D, d.T, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tw, Wr, d.D, d.E, p.n_pad)) return cudaErrorInvalidValue;
  const size_t stage_bytes = kABytes + static_cast<size_t>(p.n_pad) * BK * 2;
  p.stages = static_cast<int>((200 * 1024) / stage_bytes);
  if (p.stages > kMaxStages) p.stages = kMaxStages;
  if (p.stages > p.kb_per) p.stages = p.kb_per < 2 ? 2 : p.kb_per;
  const size_t smem = 1024 + p.stages * stage_bytes + 8 * (2 * kMaxStages + 2) + 16;
  cudaError_t e = cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  route_tc_kernel<<<dim3((d.T + BM - 1) / BM, p.ksplit), kThreads, smem, s>>>(tx, tw, p);
  if (p.ksplit > 1) route_reduce_topk_kernel<<<d.T, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace moe
