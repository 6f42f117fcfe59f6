// Grouped expert GEMMs mlp1 (+bias, SwiGLU) and mlp2 (+bias, gate weight) on
// the sm_100a tensor cores.
//
// The torchtitan GPT-OSS guide ("grouped matrix multiplication") expresses the
// expert FFN as two grouped GEMMs over the expert-sorted rows: mlp1 with
// weights (E, 2I, D) and mlp2 with weights (E, D, I), both stored (num_experts,
// out_dim, in_dim), i.e. K-major, each with a per-expert bias, and a SwiGLU
// between them. This file is one persistent, warp-specialised kernel for both:
//
//   warp 0      TMA producer: A rows [seg_start + 128*mt, +128) and the B
//               weight rows of the tile, 64-wide K slices, 128-byte swizzle,
//               into a 4-stage shared-memory ring (mbarrier full/empty).
//   warp 1      allocates 512 TMEM columns and issues tcgen05.mma (M=128,
//               N=mma_n, K=16 per instruction) into one of two TMEM
//               accumulators, committing stage releases and tile completion.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (one row per thread),
//               bias + SwiGLU (mlp1, bf16 h) or bias * gate weight (mlp2,
//               fp32 expert outputs), stores masked to the expert segment. Double-buffered TMEM lets
//               the epilogue of tile i overlap the MMAs of tile i+1.
//
// Tiles are (expert, column tile, row tile), numbered expert-major and read
// from the device-side offsets -- no host sync, no per-expert launch. For
// mlp1 the B tile stacks gate rows [n, n+Nh) over up rows [I+n, I+n+Nh), so
// SwiGLU pairs columns c and Nh+c of the same accumulator.
//
// Every mbarrier wait is bounded (1 s); on timeout the kernel records
// MOE_ERR_TIMEOUT, stops issuing, waits for its in-flight copies and MMAs,
// frees TMEM and returns.
#include "common.cuh"
#include "gemm_common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = 128;               // rows per tile = TMEM lanes
constexpr int BK = 64;                // K per stage: one 128-byte swizzle row of bf16
constexpr int kStages = 4;
// Experts with at most this many rows (one m-tile) get HBM-bound tiles: each
// column tile streams its weight slab for few rows. (Counting two-m-tile
// experts in as well measured slower on the skewed 120B shape.)
constexpr int kLightRows = BM;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccStride = 256;  // TMEM columns per accumulator buffer
constexpr int kABytes = BM * BK * 2;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr int kCtrlBytes = 256;

template <bool kSwiGLU>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t stage_bytes = kABytes + p.mma_n * BK * 2;
  uint8_t* ctrl = smem + kStages * stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctrl);  // full[S] empty[S] tfull[2] tempty[2] done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * (2 * kStages + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* total_s = reinterpret_cast<int*>(tmem_slot + 2);
  int* bad_s = reinterpret_cast<int*>(tmem_slot + 3);
  int* seg = reinterpret_cast<int*>(ctrl + kCtrlBytes);  // E+1 segment starts
  int* tpre = seg + (p.E + 1);                           // E+1 tile prefix, experts with > kLightRows rows
  int* tpre1 = tpre + (p.E + 1);                         // E+1 tile prefix, experts with 1..kLightRows rows

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
  const uint32_t done_bar = bar0 + 8u * (2 * kStages + 4);

  // ---- prologue: segment table, tile prefix, barriers, TMEM
  if (threadIdx.x == 0) {
    *bad_s = 0;
    *abort_flag = 0;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
    int o = p.offsets[e];
    seg[e] = o;
    if (o < 0 || o > p.R || (e == 0 && o != 0)) atomicOr(bad_s, 1);
  }
  __syncthreads();
  if (warp == 0) {
    // tile counts per expert, exclusive scan across the warp (E <= 256)
    const int per = (p.E + 31) / 32;
    const int e0 = lane * per;
    // two tile lists: experts with more than kLightRows rows (tensor-bound)
    // and experts with 1..kLightRows rows (HBM-bound)
    int local = 0, local1 = 0;
    for (int e = e0; e < e0 + per && e < p.E; ++e) {
      const int cnt = seg[e + 1] - seg[e];
      if (cnt < 0) atomicOr(bad_s, 1);
      if (cnt > kLightRows)
        local += (cnt + BM - 1) / BM * p.NT;
      else if (cnt > 0)
        local1 += (cnt + BM - 1) / BM * p.NT;
    }
    int incl = local, incl1 = local1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off), v1 = __shfl_up_sync(0xffffffffu, incl1, off);
      if (lane >= off) {
        incl += v;
        incl1 += v1;
      }
    }
    int run = incl - local, run1 = incl1 - local1;
    for (int e = e0; e < e0 + per && e < p.E; ++e) {
      tpre[e] = run;
      tpre1[e] = run1;
      const int cnt = seg[e + 1] - seg[e];
      if (cnt > kLightRows)
        run += (cnt + BM - 1) / BM * p.NT;
      else if (cnt > 0)
        run1 += (cnt + BM - 1) / BM * p.NT;
    }
    if (lane == 31) {
      tpre[p.E] = incl;
      tpre1[p.E] = incl1;
    }
    __syncwarp();
    if (lane == 0) {
      const int bad = *bad_s;
      if (bad) record_status(p.status, MOE_ERR_DEVICE_BOUNDS);
      *total_s = bad ? 0 : tpre[p.E] + tpre1[p.E];
      for (int s = 0; s < kStages; ++s) {
        mbar_init(full_bar(s), 1);
        mbar_init(empty_bar(s), 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(tfull_bar(b), 1);
        mbar_init(tempty_bar(b), 4);
      }
      mbar_init(done_bar, 1);
      fence_mbar_init();
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
    }
  } else if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = *total_s;
  const int KB = (p.K + BK - 1) / BK;
  // Schedule position -> tile. The light experts' tiles are spread
  // evenly among the others (position i takes the next one of them when
  // floor((i+1) C / total) steps, C their number), so that every wave of
  // concurrent tiles mixes HBM-bound and tensor-bound work; each list keeps
  // its own order (consecutive tiles of an expert share its weights in L2).
  const int n_single = tpre1[p.E];
  auto schedule = [&](int i, int& e, int& nt, int& mt) {
    const int64_t c0 = static_cast<int64_t>(i) * n_single / total;
    const int64_t c1 = static_cast<int64_t>(i + 1) * n_single / total;
    if (c1 > c0)
      decode_tile(static_cast<int>(c0), tpre1, seg, p.E, BM, e, nt, mt);
    else
      decode_tile(i - static_cast<int>(c0), tpre, seg, p.E, BM, e, nt, mt);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool failed = false;
      for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
        int e, nt, mt;
        schedule(tile, e, nt, mt);
        const int row0 = seg[e] + mt * BM;
        const int brow = e * p.b_rows + nt * p.n_tile;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, kWaitNs)) {
            failed = true;
            break;
          }
          const uint32_t a_dst = smem_u32(smem + stage * stage_bytes);
          const uint32_t b_dst = a_dst + kABytes;
          mbar_arrive_expect_tx(full_bar(stage), stage_bytes);
          tma_load_2d(a_dst, &tmA, full_bar(stage), kb * BK, row0);
          tma_load_2d(b_dst, &tmB, full_bar(stage), kb * BK, brow);
          if (kSwiGLU) tma_load_2d(b_dst + p.n_tile * BK * 2, &tmB, full_bar(stage), kb * BK, brow + p.n_out);
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (failed) {
        record_status(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        // let the copies still in flight land before the CTA can exit
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
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(BM, p.mma_n);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool failed = false;
      for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
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
          for (int kk = 0; kk < BK / 16; ++kk) {
            mma_bf16(d_tmem, desc_kmajor_sw128(a_addr + kk * 32), desc_kmajor_sw128(b_addr + kk * 32), idesc,
                     (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (failed) break;
        tc_commit(tfull_bar(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (failed) {
        record_status(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      // all MMAs issued by this thread complete before TMEM is released
      tc_commit(done_bar);
      mbar_wait_bounded(done_bar, 0, nullptr, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_in_tile = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int e, nt, mt;
      schedule(tile, e, nt, mt);
      const bool ok = mbar_wait_bounded(tfull_bar(acc), acc_phase, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) {
          record_status(p.status, MOE_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(seg[e]) + mt * BM + row_in_tile;
      const bool valid = row < seg[e + 1];
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccStride;
      epilogue_tile<kSwiGLU>(p, tbase, e, nt, row, valid);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
int pick_tile(int n, int max_tile, int step) {
  for (int t = max_tile; t >= step; t -= step)
    if (n % t == 0) return t;
  return 0;
}

size_t smem_bytes(int mma_n, int E) {
  return 1024 + static_cast<size_t>(kStages) * (kABytes + mma_n * BK * 2) + kCtrlBytes + 3 * (E + 1) * sizeof(int);
}

template <bool kSwiGLU>
moe_status_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p, cudaStream_t s) {
  const size_t smem = smem_bytes(p.mma_n, p.E);
  if (cudaFuncSetAttribute(grouped_gemm_kernel<kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int64_t max_tiles = ((p.R + BM - 1) / BM + p.E) * static_cast<int64_t>(p.NT);
  const int grid = static_cast<int>(max_tiles < num_sms() ? max_tiles : num_sms());
  grouped_gemm_kernel<kSwiGLU><<<grid, kThreads, smem, s>>>(ta, tb, p);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

moe_status_t launch_mlp1(const moe_dims_t& d, const uint16_t* x_perm, const int32_t* offsets, const uint16_t* W1,
                         const uint16_t* b1, uint16_t* h, int* status, cudaStream_t s) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  const int nh = pick_tile(d.I, 128, 8);
  if (nh == 0) return MOE_ERR_UNSUPPORTED;
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, x_perm, d.D, R, BM)) return MOE_ERR_CUDA;
  if (!make_tmap_bf16(&tb, W1, d.D, static_cast<uint64_t>(d.E) * 2 * d.I, nh)) return MOE_ERR_CUDA;
  GemmParams p{};
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
  return launch_gemm<true>(ta, tb, p, s);
}

moe_status_t launch_mlp2(const moe_dims_t& d, const uint16_t* h, const int32_t* perm, const int32_t* offsets,
                         const float* topk_w, const uint16_t* W2, const uint16_t* b2, float* o_perm, int* status,
                         cudaStream_t s) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  const int nt = pick_tile(d.D, 256, 16);
  if (nt == 0) return MOE_ERR_UNSUPPORTED;
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, h, d.I, R, BM)) return MOE_ERR_CUDA;
  if (!make_tmap_bf16(&tb, W2, d.I, static_cast<uint64_t>(d.E) * d.D, nt)) return MOE_ERR_CUDA;
  GemmParams p{};
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
  return launch_gemm<false>(ta, tb, p, s);
}

}  // namespace moe
