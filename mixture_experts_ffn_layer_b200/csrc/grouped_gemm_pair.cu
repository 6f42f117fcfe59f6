// Grouped mlp1 / mlp2 on SM pairs: tcgen05.mma.cta_group::2, 256-row tiles.
//
// Same layer step as grouped_gemm.cu (torchtitan GPT-OSS guide, "grouped
// matrix multiplication": per-expert GEMMs over the expert-sorted rows, K-major
// weights, bias, SwiGLU between mlp1 and mlp2), with one tile computed by a
// cluster of two CTAs on two SMs:
//
//   - each CTA loads its own 128 rows of A and HALF of the B tile (for mlp1
//     CTA 0 holds the gate rows [n, n+Nh) and CTA 1 the up rows [I+n, I+n+Nh);
//     for mlp2 the two halves of the N tile), 64-wide K slices, 128-byte
//     swizzle; both CTAs' copies complete on the leader CTA's stage barrier;
//   - the leader's MMA thread issues tcgen05.mma.cta_group::2 (M = 256,
//     N = full tile); the hardware reads both CTAs' shared memory, and each
//     CTA's TMEM receives its own 128 rows x N columns;
//   - stage release, accumulator-ready and completion are committed to both
//     CTAs' barriers at once (tcgen05.commit multicast); each CTA's epilogue
//     drains its own TMEM and arrives on the leader's accumulator-free barrier.
// Per SM and K slice this moves A (16 KB) + half of B instead of A + all of
// B, so more of the tensor core's time is fed from the same L2 bandwidth, at
// the price of 256-row tile granularity on ragged expert segments. No TMA
// multicast is used: every CTA loads its own data.
#include "gemm_common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BMP = 256;              // rows per pair tile (128 per CTA)
constexpr int BK = 64;
constexpr int kMaxStages = 8;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccStride = 256;
constexpr int kABytes = 128 * BK * 2;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr int kCtrlBytes = 256;
constexpr size_t kMaxSmem = 232448;   // 227 KB per CTA

struct PairParams {
  GemmParams g;
  int n_half;    // B rows held by each CTA
  int stages;
  int b_off1;    // row offset of CTA 1's B half relative to CTA 0's
};

template <bool kSwiGLU>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const PairParams pp) {
  const GemmParams& p = pp.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = pp.stages;
  const uint32_t stage_bytes = kABytes + pp.n_half * BK * 2;
  uint8_t* ctrl = smem + S * stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctrl);  // full[8] empty[8] tfull[2] tempty[2] done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * (2 * kMaxStages + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* total_s = reinterpret_cast<int*>(tmem_slot + 2);
  int* bad_s = reinterpret_cast<int*>(tmem_slot + 3);
  int* seg = reinterpret_cast<int*>(ctrl + kCtrlBytes);
  int* tpre = seg + (p.E + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kMaxStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kMaxStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kMaxStages + 2 + b); };
  const uint32_t done_bar = bar0 + 8u * (2 * kMaxStages + 4);

  // ---- prologue: segment table, tile prefix (256-row tiles), barriers, TMEM
  if (threadIdx.x == 0) {
    *bad_s = 0;
    *abort_flag = 0;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
    const int o = p.offsets[e];
    seg[e] = o;
    if (o < 0 || o > p.R || (e == 0 && o != 0)) atomicOr(bad_s, 1);
  }
  __syncthreads();
  if (warp == 0) {
    const int per = (p.E + 31) / 32;
    const int e0 = lane * per;
    int local = 0;
    for (int e = e0; e < e0 + per && e < p.E; ++e) {
      const int cnt = seg[e + 1] - seg[e];
      if (cnt < 0) atomicOr(bad_s, 1);
      local += cnt > 0 ? (cnt + BMP - 1) / BMP * p.NT : 0;
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int run = incl - local;
    for (int e = e0; e < e0 + per && e < p.E; ++e) {
      tpre[e] = run;
      const int cnt = seg[e + 1] - seg[e];
      run += cnt > 0 ? (cnt + BMP - 1) / BMP * p.NT : 0;
    }
    if (lane == 31) tpre[p.E] = incl;
    __syncwarp();
    if (lane == 0) {
      const int bad = *bad_s;
      if (bad && leader) record_status(p.status, MOE_ERR_DEVICE_BOUNDS);
      *total_s = bad ? 0 : tpre[p.E];
      for (int s = 0; s < S; ++s) {
        mbar_init(full_bar(s), 1);
        mbar_init(empty_bar(s), 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(tfull_bar(b), 1);
        mbar_init(tempty_bar(b), 8);  // 4 epilogue warps in each CTA of the pair
      }
      mbar_init(done_bar, 1);
      fence_mbar_init();
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
    }
  } else if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = *total_s;
  const int KB = (p.K + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer (both CTAs)
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool failed = false;
      for (int tile = pair; tile < total && !failed; tile += npairs) {
        int e, nt, mt;
        decode_tile(tile, tpre, seg, p.E, BMP, e, nt, mt);
        const int row0 = seg[e] + mt * BMP + 128 * static_cast<int>(rank);
        const int brow = e * p.b_rows + nt * p.n_tile + (leader ? 0 : pp.b_off1);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, kWaitNs)) {
            failed = true;
            break;
          }
          const uint32_t a_dst = smem_u32(smem + stage * stage_bytes);
          const uint32_t bar_leader = mapa_shared(full_bar(stage), 0);
          if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * stage_bytes);
          tma_load_2d_pair(a_dst, &tmA, bar_leader, kb * BK, row0);
          tma_load_2d_pair(a_dst + kABytes, &tmB, bar_leader, kb * BK, brow);
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (failed) {
        record_status(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        if (leader) {
          // the leader's stage barriers count both CTAs' copies: drain them
          const int n = issued < S ? issued : S;
          int s = stage;
          uint32_t ph = phase;
          for (int i = 0; i < n; ++i) {
            if (--s < 0) {
              s = S - 1;
              ph ^= 1u;
            }
            mbar_wait_bounded(full_bar(s), ph, nullptr, kWaitNs);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------------------------------------------------- MMA issuer (leader)
      const uint32_t idesc = idesc_bf16_f32(BMP, p.mma_n);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool failed = false;
      for (int tile = pair; tile < total && !failed; tile += npairs) {
        if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, kWaitNs)) {
          failed = true;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccStride;
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
            mma_bf16_pair(d_tmem, desc_kmajor_sw128(a_addr + kk * 32), desc_kmajor_sw128(b_addr + kk * 32), idesc,
                          (kb | kk) != 0 ? 1u : 0u);
          tc_commit_pair(empty_bar(stage), 0x3);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (failed) break;
        tc_commit_pair(tfull_bar(acc), 0x3);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (failed) {
        record_status(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc_commit_pair(done_bar, 0x1);
      mbar_wait_bounded(done_bar, 0, nullptr, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int row_in_tile = 128 * static_cast<int>(rank) + q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total; tile += npairs) {
      int e, nt, mt;
      decode_tile(tile, tpre, seg, p.E, BMP, e, nt, mt);
      const bool ok = mbar_wait_bounded(tfull_bar(acc), acc_phase, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) {
          record_status(p.status, MOE_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(seg[e]) + mt * BMP + row_in_tile;
      const bool valid = row < seg[e + 1];
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccStride;
      epilogue_tile<kSwiGLU>(p, tbase, e, nt, row, valid);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its pair may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <bool kSwiGLU>
moe_status_t launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, PairParams pp, cudaStream_t s) {
  const size_t fixed = 1024 + kCtrlBytes + 2 * (pp.g.E + 1) * sizeof(int);
  const size_t stage_bytes = kABytes + static_cast<size_t>(pp.n_half) * BK * 2;
  int stages = static_cast<int>((kMaxSmem - fixed) / stage_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return MOE_ERR_UNSUPPORTED;
  pp.stages = stages;
  const size_t smem = fixed + stages * stage_bytes;
  if (cudaFuncSetAttribute(grouped_gemm_pair_kernel<kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int64_t max_tiles = ((pp.g.R + BMP - 1) / BMP + pp.g.E) * static_cast<int64_t>(pp.g.NT);
  int pairs = num_sms() / 2;
  if (max_tiles < pairs) pairs = static_cast<int>(max_tiles);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel<kSwiGLU>, ta, tb, pp) != cudaSuccess) return MOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int pick_tile(int n, int max_tile, int step) {
  for (int t = max_tile; t >= step; t -= step)
    if (n % t == 0) return t;
  return 0;
}

}  // namespace

moe_status_t launch_mlp1_pair(const moe_dims_t& d, const uint16_t* x_perm, const int32_t* offsets,
                              const uint16_t* W1, const uint16_t* b1, uint16_t* h, int* status, cudaStream_t s) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  const int nh = pick_tile(d.I, 128, 8);  // gate rows per tile (= up rows): CTA 0 gate, CTA 1 up
  if (nh == 0) return MOE_ERR_UNSUPPORTED;
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, x_perm, d.D, R, 128)) return MOE_ERR_CUDA;
  if (!make_tmap_bf16(&tb, W1, d.D, static_cast<uint64_t>(d.E) * 2 * d.I, nh)) return MOE_ERR_CUDA;
  PairParams pp{};
  GemmParams& p = pp.g;
  p.E = d.E;
  p.K = d.D;
  p.n_out = d.I;
  p.n_tile = nh;
  p.mma_n = 2 * nh;
  p.NT = d.I / nh;
  p.b_rows = 2 * d.I;
  p.R = R;
  p.offsets = offsets;
  p.bias = b1;
  p.act = act_of(d);
  p.out = h;
  p.status = status;
  pp.n_half = nh;
  pp.b_off1 = d.I;  // CTA 1 loads the up rows
  return launch_pair<true>(ta, tb, pp, s);
}

moe_status_t launch_mlp2_pair(const moe_dims_t& d, const uint16_t* h, const int32_t* perm, const int32_t* offsets,
                              const float* topk_w, const uint16_t* W2, const uint16_t* b2, float* o_perm,
                              int* status, cudaStream_t s) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  const int nt = pick_tile(d.D, 256, 16);  // N tile; each CTA holds half of it
  if (nt == 0) return MOE_ERR_UNSUPPORTED;
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, h, d.I, R, 128)) return MOE_ERR_CUDA;
  if (!make_tmap_bf16(&tb, W2, d.I, static_cast<uint64_t>(d.E) * d.D, nt / 2)) return MOE_ERR_CUDA;
  PairParams pp{};
  GemmParams& p = pp.g;
  p.E = d.E;
  p.K = d.I;
  p.n_out = d.D;
  p.n_tile = nt;
  p.mma_n = nt;
  p.NT = d.D / nt;
  p.b_rows = d.D;
  p.R = R;
  p.offsets = offsets;
  p.bias = b2;
  p.perm = perm;
  p.topk_w = topk_w;
  p.out = o_perm;
  p.status = status;
  pp.n_half = nt / 2;
  pp.b_off1 = nt / 2;  // CTA 1 loads the second half of the N tile
  return launch_pair<false>(ta, tb, pp, s);
}

}  // namespace moe
