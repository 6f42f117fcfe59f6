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
#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

#include <float.h>

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = 128, BK = 64, kMaxStages = 12, kThreads = 192, kMaxK = 8;
constexpr int kABytes = BM * BK * 2;
constexpr uint64_t kWaitNs = 1000000000ull;

struct RouteParams {
  int T, D, E, k;
  int n_pad;        // MMA N: E rounded up to a multiple of 16
  int stages;       // TMA ring depth (as many as fit: few CTAs stream all of x)
  uint32_t tmem_cols;
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

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kMaxStages + s); };
  const uint32_t tfull_bar = bar0 + 8u * (2 * kMaxStages);
  const uint32_t done_bar = bar0 + 8u * (2 * kMaxStages + 1);
  const int t0 = blockIdx.x * BM;
  const int KB = (p.D + BK - 1) / BK;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(done_bar, 1);
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
      for (int kb = 0; kb < KB; ++kb) {
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
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issuer: one 128 x n_pad accumulator over all of K
      const uint32_t idesc = idesc_bf16_f32(BM, p.n_pad);
      int stage = 0;
      uint32_t phase = 0;
      bool failed = false;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag, kWaitNs)) {
          failed = true;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + stage * stage_bytes);
        const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          mma_bf16(tmem_base, desc_kmajor_sw128(a_addr + kk * 32), desc_kmajor_sw128(b_addr + kk * 32), idesc,
                   (kb | kk) != 0 ? 1u : 0u);
        tc_commit(empty_bar(stage));
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (failed) {
        record_status(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
      } else {
        tc_commit(tfull_bar);
      }
      tc_commit(done_bar);
      mbar_wait_bounded(done_bar, 0, nullptr, kWaitNs);
    }
  } else {
    // epilogue: thread = token = TMEM lane
    const int q = warp & 3;
    const int t = t0 + q * 32 + lane;
    const bool ok = mbar_wait_bounded(tfull_bar, 0, abort_flag, kWaitNs);
    if (__all_sync(0xffffffffu, ok)) {
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
        uint32_t v[32];
        // up to four 8-column loads in flight per wait (warp-uniform bounds)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (c0 + 8 * j < p.n_pad) tmem_ld_x8(tbase + c0 + 8 * j, v + 8 * j);
        tmem_ld_wait();
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

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace

cudaError_t launch_route(const moe_dims_t& d, const uint16_t* x, const uint16_t* Wr, const uint16_t* br,
                         int32_t* topk_idx, float* topk_w, int* status, cudaStream_t s) {
  RouteParams p{};
  p.T = d.T;
  p.D = d.D;
  p.E = d.E;
  p.k = d.k;
  p.n_pad = (d.E + 15) / 16 * 16;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(p.n_pad)) cols <<= 1;
  p.tmem_cols = cols;
  p.br = br;
  p.topk_idx = topk_idx;
  p.topk_w = topk_w;
  p.status = status;
  CUtensorMap tx, tw;
  if (!make_tmap_bf16(&tx, x, d.D, d.T, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tw, Wr, d.D, d.E, p.n_pad)) return cudaErrorInvalidValue;
  const size_t stage_bytes = kABytes + static_cast<size_t>(p.n_pad) * BK * 2;
  p.stages = static_cast<int>((200 * 1024) / stage_bytes);
  if (p.stages > kMaxStages) p.stages = kMaxStages;
  const size_t smem = 1024 + p.stages * stage_bytes + 8 * (2 * kMaxStages + 2) + 16;
  cudaError_t e = cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  route_tc_kernel<<<(d.T + BM - 1) / BM, kThreads, smem, s>>>(tx, tw, p);
  return cudaGetLastError();
}

}  // namespace moe
