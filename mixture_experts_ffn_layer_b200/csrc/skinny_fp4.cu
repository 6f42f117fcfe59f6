// Grouped expert GEMMs with MXFP4 weights when each expert sees few rows
// (decode-like batches).
//
// MXFP4 (GPT-OSS in Transformers blog, MXFP4 paragraph): E2M1 4-bit values,
// one E8M0 scale per 32 consecutive elements of the reduction dim. With a
// handful of routed rows per expert the layer is bound by streaming the
// 4.25-bit weights from HBM, and a 128-row tensor-core tile would be almost
// all padding. So the weights are the "M" side here: each warp owns 16 weight
// rows of one expert and streams their codes once (32 bytes per row per
// 64-element K step), decodes them straight into mma.sync A fragments with
// the hardware E2M1 -> f16 conversion (exact: every E2M1 value is an f16),
// and multiplies them against up to 32 routed rows (the N side, f16). Each
// 32-element block's partial product comes out of the tensor core in fp32 and
// is scaled there by 2^(s-127), so every E8M0 scale is applied exactly.
//
// The codes reach shared memory by TMA (one producer warp, 8-stage ring of
// 128-row x 64-element boxes), so each SM keeps tens of KB in flight.
// mlp1: rows [n, n+16) (gate) and [I+n, I+n+16) (up) of W1[e] in one warp,
//       epilogue h = bf16(silu(gate + b1) * (up + b1')).
// mlp2: rows [n, n+16) of W2[e], epilogue o = w * (acc + b2), fp32.
// The routed rows enter as bf16 and are converted to f16 on load, times a
// power of two (mlp2 reads h * 2^-8 so that |h| up to 2^24 stays finite in
// f16); the accumulator is multiplied back.
#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;        // compute warps: 8 x 16 = 128 weight rows per CTA
constexpr int kStages = 8;       // 64-element K steps of codes in flight per CTA
constexpr int kMaxChunks = 4;    // up to 4 x 8 = 32 routed rows per pass over the weights
constexpr int kRowsPerCta = kWarps * 16;
constexpr uint64_t kWaitNs = 1000000000ull;

struct SkinnyParams {
  int E, K;
  int n_out;   // output columns: I (mlp1) or D (mlp2)
  int b_rows;  // weight rows per expert: 2I or D
  int64_t R;
  const int32_t* offsets;
  const uint8_t* scales;  // (E, b_rows, K/32)
  const uint16_t* bias;   // (E, b_rows) bf16
  const uint16_t* in;     // routed rows (R, K) bf16
  float in_scale;         // power of two applied to the routed rows in f16
  const int32_t* perm;    // mlp2: gate weight of row r is topk_w[perm[r]]
  const float* topk_w;
  void* out;              // h (R, I) bf16 or o_perm (R, D) fp32
  int* status;
};

__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t d;
  const unsigned short b = static_cast<unsigned short>(byte & 0xffu);
  asm("{\n\t.reg .b8 t;\n\tmov.b16 {t, _}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(d) : "h"(b));
  return d;
}

// bf16 pair -> f16 pair times s (exact for |v*s| in the f16 normal range)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, float s) {
  const float lo = __uint_as_float(w << 16) * s, hi = __uint_as_float(w & 0xffff0000u) * s;
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float e8m0(uint32_t s) {
  if (s == 255u) return __uint_as_float(0x7fc00000u);
  if (s == 0u) return __uint_as_float(0x00400000u);
  return __uint_as_float(s << 23);
}

// A fragments of the two 16-element halves of 32-element block `blk` of a
// 64-element step, for the rows whose 32 code bytes start at r0 (row g) and
// r1 (row g + 8) in shared memory. Element 2j, 2j+1 = byte j.
__device__ __forceinline__ void a_frags(const uint8_t* r0, const uint8_t* r1, int blk, int t, uint32_t (&a)[4],
                                        uint32_t (&b)[4]) {
  const uint4 w0 = *reinterpret_cast<const uint4*>(r0 + 16 * blk);
  const uint4 w1 = *reinterpret_cast<const uint4*>(r1 + 16 * blk);
  const int sh = 8 * t;
  // half 0: elements 0..15 of the block = bytes 0..7 (words x, y); half 1: words z, w
  a[0] = e2m1x2_to_f16x2(w0.x >> sh);
  a[1] = e2m1x2_to_f16x2(w1.x >> sh);
  a[2] = e2m1x2_to_f16x2(w0.y >> sh);
  a[3] = e2m1x2_to_f16x2(w1.y >> sh);
  b[0] = e2m1x2_to_f16x2(w0.z >> sh);
  b[1] = e2m1x2_to_f16x2(w1.z >> sh);
  b[2] = e2m1x2_to_f16x2(w0.w >> sh);
  b[3] = e2m1x2_to_f16x2(w1.w >> sh);
}

// Warp kWarps (lane 0) streams the CTA's 128 weight rows (and, for mlp1, the
// matching 128 up rows) one 64-element step at a time by TMA into a
// kStages ring; warps 0..kWarps-1 each compute 16 of those rows.
template <bool kSwiGLU>
__global__ void __launch_bounds__((kWarps + 1) * 32) skinny_fp4_kernel(const __grid_constant__ CUtensorMap tmCodes,
                                                                       const SkinnyParams p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  constexpr uint32_t kBox = kRowsPerCta * 32;  // bytes of one 128-row box
  constexpr uint32_t kStageBytes = kSwiGLU ? 2 * kBox : kBox;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * kStages);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };

  const int e = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int seg0 = p.offsets[e], seg1 = p.offsets[e + 1];
  if (seg0 < 0 || seg1 < seg0 || seg1 > p.R) {
    if (threadIdx.x == 0) record_status(p.status, MOE_ERR_DEVICE_BOUNDS);
    return;
  }
  const int n_rows = seg1 - seg0;
  if (n_rows == 0) return;
  const int ksteps = p.K / 64;
  const int npass = (n_rows + 8 * kMaxChunks - 1) / (8 * kMaxChunks);
  const int64_t wrow_g = static_cast<int64_t>(e) * p.b_rows + blockIdx.x * kRowsPerCta;  // first row of the box
  const int64_t wrow_u = wrow_g + p.n_out;                                                // mlp1 up rows

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kWarps) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool failed = false;
      for (int pass = 0; pass < npass && !failed; ++pass) {
        for (int ks = 0; ks < ksteps; ++ks) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, kWaitNs)) {
            failed = true;
            break;
          }
          const uint32_t dst = smem_u32(smem + stage * kStageBytes);
          mbar_arrive_expect_tx(full_bar(stage), kStageBytes);
          tma_load_2d(dst, &tmCodes, full_bar(stage), ks * 32, static_cast<int32_t>(wrow_g));
          if (kSwiGLU) tma_load_2d(dst + kBox, &tmCodes, full_bar(stage), ks * 32, static_cast<int32_t>(wrow_u));
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
    return;
  }

  // ------------------------------------------------------------ compute warps
  const int g = lane >> 2, t = lane & 3;
  const int col_base = blockIdx.x * kRowsPerCta + warp * 16;  // first output column of this warp
  const bool active = col_base < p.n_out;
  const int64_t nsc = p.K / 32;
  const uint8_t* sc_g = p.scales + (wrow_g + warp * 16 + g) * nsc;  // row g; row g+8 is 8*nsc further
  const uint8_t* sc_u = p.scales + (wrow_u + warp * 16 + g) * nsc;
  int stage = 0;
  uint32_t phase = 0;
  for (int pass = 0; pass < npass; ++pass) {
    const int base = pass * 8 * kMaxChunks;
    const int nch = min(kMaxChunks, (n_rows - base + 7) / 8);
    float acc_g[kMaxChunks][4], acc_u[kMaxChunks][4];
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc_g[c][i] = acc_u[c][i] = 0.f;
    const uint16_t* brow[kMaxChunks];
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int n = base + 8 * c + g;
      brow[c] = p.in + static_cast<int64_t>(seg0 + (n < n_rows ? n : 0)) * p.K;
    }
    bool failed = false;
    for (int ks = 0; ks < ksteps; ++ks) {
      const bool ok = mbar_wait_bounded(full_bar(stage), phase, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        failed = true;
        break;
      }
      if (active) {
        const uint8_t* box = smem + stage * kStageBytes;
        const uint8_t* rg0 = box + (warp * 16 + g) * 32;
        const uint8_t* rg1 = rg0 + 8 * 32;
        const uint32_t sg0 = __ldg(reinterpret_cast<const unsigned short*>(sc_g + 2 * ks));
        const uint32_t sg1 = __ldg(reinterpret_cast<const unsigned short*>(sc_g + 8 * nsc + 2 * ks));
        uint32_t su0 = 0, su1 = 0;
        if (kSwiGLU) {
          su0 = __ldg(reinterpret_cast<const unsigned short*>(sc_u + 2 * ks));
          su1 = __ldg(reinterpret_cast<const unsigned short*>(sc_u + 8 * nsc + 2 * ks));
        }
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          uint32_t ag0[4], ag1[4], au0[4], au1[4];
          a_frags(rg0, rg1, blk, t, ag0, ag1);
          if (kSwiGLU) a_frags(rg0 + kBox, rg1 + kBox, blk, t, au0, au1);
          const float fg0 = e8m0((sg0 >> (8 * blk)) & 0xffu), fg1 = e8m0((sg1 >> (8 * blk)) & 0xffu);
          const float fu0 = e8m0((su0 >> (8 * blk)) & 0xffu), fu1 = e8m0((su1 >> (8 * blk)) & 0xffu);
#pragma unroll
          for (int c = 0; c < kMaxChunks; ++c) {
            if (c < nch) {
              const uint16_t* b = brow[c] + ks * 64 + blk * 32 + 2 * t;
              const uint32_t b00 = bf16x2_to_f16x2(__ldg(reinterpret_cast<const uint32_t*>(b)), p.in_scale);
              const uint32_t b01 = bf16x2_to_f16x2(__ldg(reinterpret_cast<const uint32_t*>(b + 8)), p.in_scale);
              const uint32_t b10 = bf16x2_to_f16x2(__ldg(reinterpret_cast<const uint32_t*>(b + 16)), p.in_scale);
              const uint32_t b11 = bf16x2_to_f16x2(__ldg(reinterpret_cast<const uint32_t*>(b + 24)), p.in_scale);
              float tg[4] = {0.f, 0.f, 0.f, 0.f};
              mma_f16_16816(tg, ag0, b00, b01);
              mma_f16_16816(tg, ag1, b10, b11);
              acc_g[c][0] = fmaf(fg0, tg[0], acc_g[c][0]);
              acc_g[c][1] = fmaf(fg0, tg[1], acc_g[c][1]);
              acc_g[c][2] = fmaf(fg1, tg[2], acc_g[c][2]);
              acc_g[c][3] = fmaf(fg1, tg[3], acc_g[c][3]);
              if (kSwiGLU) {
                float tu[4] = {0.f, 0.f, 0.f, 0.f};
                mma_f16_16816(tu, au0, b00, b01);
                mma_f16_16816(tu, au1, b10, b11);
                acc_u[c][0] = fmaf(fu0, tu[0], acc_u[c][0]);
                acc_u[c][1] = fmaf(fu0, tu[1], acc_u[c][1]);
                acc_u[c][2] = fmaf(fu1, tu[2], acc_u[c][2]);
                acc_u[c][3] = fmaf(fu1, tu[3], acc_u[c][3]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(stage));
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
      return;
    }
    if (!active) continue;

    // epilogue: acc[c][0,1] = weight row g, routed rows 2t, 2t+1 of chunk c;
    //           acc[c][2,3] = weight row g+8, same routed rows
    const float undo = 1.0f / p.in_scale;
    const int64_t brow_g = wrow_g + warp * 16 + g;
    const float bg0 = bf16_bits_to_float(p.bias[brow_g]);
    const float bg1 = bf16_bits_to_float(p.bias[brow_g + 8]);
    float bu0 = 0.f, bu1 = 0.f;
    if (kSwiGLU) {
      bu0 = bf16_bits_to_float(p.bias[brow_g + p.n_out]);
      bu1 = bf16_bits_to_float(p.bias[brow_g + p.n_out + 8]);
    }
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      if (c >= nch) continue;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int n = base + 8 * c + 2 * t + (i & 1);
        if (n >= n_rows) continue;
        const int64_t row = seg0 + n;
        const int col = col_base + g + (i >= 2 ? 8 : 0);
        const float vg = acc_g[c][i] * undo + (i >= 2 ? bg1 : bg0);
        if (kSwiGLU) {
          const float vu = acc_u[c][i] * undo + (i >= 2 ? bu1 : bu0);
          const float hv = __fdividef(vg, 1.0f + __expf(-vg)) * vu;
          static_cast<uint16_t*>(p.out)[row * p.n_out + col] = float_to_bf16_bits(hv);
        } else {
          const int32_t a = p.perm[row];
          float wgt = 0.f;
          if (a >= 0 && a < p.R)
            wgt = p.topk_w[a];
          else
            record_status(p.status, MOE_ERR_DEVICE_BOUNDS);
          static_cast<float*>(p.out)[row * p.n_out + col] = wgt * vg;
        }
      }
    }
  }
}

// (E * rows, K/2) bytes of codes, loaded as 32-byte x 128-row boxes.
bool make_tmap_codes(CUtensorMap* map, const uint8_t* codes, uint64_t rows, uint64_t half_k) {
  auto fn = tma_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {half_k, rows};
  cuuint64_t strides[1] = {half_k};
  cuuint32_t box[2] = {32u, static_cast<cuuint32_t>(kRowsPerCta)};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kSwiGLU>
moe_status_t launch_skinny(const CUtensorMap& tm, const SkinnyParams& p, int E, cudaStream_t s) {
  const size_t stage_bytes = (kSwiGLU ? 2 : 1) * kRowsPerCta * 32;
  const size_t smem = 128 + kStages * stage_bytes + 2 * kStages * 8 + 16;
  if (cudaFuncSetAttribute(skinny_fp4_kernel<kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_CUDA;
  const dim3 grid((p.n_out + kRowsPerCta - 1) / kRowsPerCta, E);
  skinny_fp4_kernel<kSwiGLU><<<grid, (kWarps + 1) * 32, smem, s>>>(tm, p);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

bool skinny_fp4_applies(const moe_dims_t& d) {
  // few routed rows per expert: at most 16 on average
  return d.wfmt == MOE_W_MXFP4 && static_cast<int64_t>(d.T) * d.k <= 16LL * d.E;
}

moe_status_t launch_mlp1_fp4_skinny(const moe_dims_t& d, const uint16_t* x_perm, const int32_t* offsets,
                                    const uint8_t* codes, const uint8_t* scales, const uint16_t* b1, uint16_t* h,
                                    int* status, cudaStream_t s) {
  SkinnyParams p{};
  p.E = d.E;
  p.K = d.D;
  p.n_out = d.I;
  p.b_rows = 2 * d.I;
  p.R = static_cast<int64_t>(d.T) * d.k;
  p.offsets = offsets;
  p.scales = scales;
  p.bias = b1;
  p.in = x_perm;
  p.in_scale = 1.0f;
  p.out = h;
  p.status = status;
  CUtensorMap tm;
  if (!make_tmap_codes(&tm, codes, static_cast<uint64_t>(d.E) * 2 * d.I, d.D / 2)) return MOE_ERR_CUDA;
  return launch_skinny<true>(tm, p, d.E, s);
}

moe_status_t launch_mlp2_fp4_skinny(const moe_dims_t& d, const uint16_t* h, const int32_t* perm,
                                    const int32_t* offsets, const float* topk_w, const uint8_t* codes,
                                    const uint8_t* scales, const uint16_t* b2, float* o_perm, int* status,
                                    cudaStream_t s) {
  SkinnyParams p{};
  p.E = d.E;
  p.K = d.I;
  p.n_out = d.D;
  p.b_rows = d.D;
  p.R = static_cast<int64_t>(d.T) * d.k;
  p.offsets = offsets;
  p.scales = scales;
  p.bias = b2;
  p.in = h;
  p.in_scale = 1.0f / 256.0f;
  p.perm = perm;
  p.topk_w = topk_w;
  p.out = o_perm;
  p.status = status;
  CUtensorMap tm;
  if (!make_tmap_codes(&tm, codes, static_cast<uint64_t>(d.E) * d.D, d.I / 2)) return MOE_ERR_CUDA;
  return launch_skinny<false>(tm, p, d.E, s);
}

}  // namespace moe
