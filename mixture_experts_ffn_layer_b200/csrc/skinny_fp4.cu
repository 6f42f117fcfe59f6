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
// The codes and the routed rows reach shared memory by TMA (one producer
// warp, a ring of 64-element K steps), so each SM keeps tens of KB in flight
// and no global load sits inside the math loop.
// mlp1: rows [n, n+16) (gate) and [I+n, I+n+16) (up) of W1[e] in one warp,
//       epilogue h = bf16(silu(gate + b1) * (up + b1')).
// mlp2: rows [n, n+16) of W2[e], epilogue o = w * (acc + b2), fp32.
// The routed rows are converted once to f16 in the workspace, times a power
// of two (mlp2 uses h * 2^-8 so that |h| up to 2^24 stays finite in f16);
// the accumulator is multiplied back.
#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;        // compute warps: 8 x 16 = 128 weight rows per CTA
constexpr int kMaxChunks = 4;    // up to 4 x 8 = 32 routed rows per pass over the weights
constexpr int kRowsPerCta = kWarps * 16;
constexpr int kTokRows = 8 * kMaxChunks;
constexpr int kStepK = 128;                       // K elements per pipeline step (4 scale blocks)
constexpr uint32_t kBox = kRowsPerCta * kStepK / 2;  // one 128-row x 128-element box of codes (64 B rows)
constexpr uint32_t kTokBox = kTokRows * 128;      // 32 routed rows x 64 f16, 128-byte swizzle (two per step)
constexpr uint64_t kWaitNs = 1000000000ull;

template <bool kSwiGLU>
struct Cfg {
  static constexpr int kStages = kSwiGLU ? 3 : 6;  // two CTAs per SM
  static constexpr uint32_t kStageBytes = (kSwiGLU ? 2 : 1) * kBox + 2 * kTokBox;  // multiple of 1024
};

struct SkinnyParams {
  int E, K;
  int n_out;   // output columns: I (mlp1) or D (mlp2)
  int b_rows;  // weight rows per expert: 2I or D
  int64_t R;
  const int32_t* offsets;
  const uint8_t* scales;  // (E, b_rows, K/32)
  const uint16_t* bias;   // (E, b_rows) bf16
  float in_scale;         // power of two the routed rows were scaled by in f16
  const int32_t* perm;    // mlp2: gate weight of row r is topk_w[perm[r]]
  const float* topk_w;
  void* out;              // h (R, I) bf16 or o_perm (R, D) fp32
  int* status;
};

// Four E2M1 pairs (one 32-bit word = 8 codes) to four f16 pairs, in byte order.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t (&d)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(w));
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// E8M0 scale 2^(s-127); s = 0 is 2^-127 (s = 255, NaN in the format, reads as inf).
__device__ __forceinline__ float e8m0(uint32_t s) {
  return s ? __uint_as_float(s << 23) : __uint_as_float(0x00400000u);
}

// K order inside each 32-element scale block. The dot product does not depend
// on the order in which K is visited, so lane t of a quad takes the 8
// consecutive elements [8t, 8t+8) of the block for both operands: its A
// fragment is one 32-bit word of codes (4 hardware conversions) and its B
// fragment one 16-byte load. Element pairs (8t+2u, 8t+2u+1), u = 0..3, feed
// the mma.m16n8k16 fragment slots "k = 2t" (u=0) and "k = 2t+8" (u=1) of the
// block's first 16-wide mma and the same slots of its second (u = 2, 3).

// Warp kWarps (lane 0) streams, per 128-element K step, the CTA's 128 weight
// rows of codes (and for mlp1 the matching 128 up rows) plus the 32 routed
// rows of the pass by TMA into a shared-memory ring; warps 0..kWarps-1 each
// compute 16 of the weight rows. Block scales are copied to shared memory
// once per CTA.
template <bool kSwiGLU>
__global__ void __launch_bounds__((kWarps + 1) * 32) skinny_fp4_kernel(const __grid_constant__ CUtensorMap tmCodes,
                                                                       const __grid_constant__ CUtensorMap tmTok,
                                                                       const SkinnyParams p) {
  using namespace sm100;
  constexpr int kStages = Cfg<kSwiGLU>::kStages;
  constexpr uint32_t kStageBytes = Cfg<kSwiGLU>::kStageBytes;
  constexpr uint32_t kTokOff = (kSwiGLU ? 2 : 1) * kBox;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * kStages);
  uint8_t* sc_smem = reinterpret_cast<uint8_t*>(bars + 2 * kStages + 2);  // rows x K/32 scale bytes
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
  const int ksteps = (p.K + kStepK - 1) / kStepK;  // a ragged last step reads zeros past K
  const int npass = (n_rows + kTokRows - 1) / kTokRows;
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
      tma_prefetch_desc(&tmCodes);
      tma_prefetch_desc(&tmTok);
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
          tma_load_2d(dst, &tmCodes, full_bar(stage), ks * (kStepK / 2), static_cast<int32_t>(wrow_g));
          if (kSwiGLU)
            tma_load_2d(dst + kBox, &tmCodes, full_bar(stage), ks * (kStepK / 2), static_cast<int32_t>(wrow_u));
          tma_load_2d(dst + kTokOff, &tmTok, full_bar(stage), ks * kStepK, seg0 + pass * kTokRows);
          tma_load_2d(dst + kTokOff + kTokBox, &tmTok, full_bar(stage), ks * kStepK + 64, seg0 + pass * kTokRows);
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
  // block scales of the CTA's rows (gate rows, then up rows): each set of 128
  // consecutive rows is one contiguous run of 128 * K/32 bytes, copied with
  // batched 16-byte loads (rows past the end of the tensor read as zero)
  const int nsc = p.K / 32;
  const int64_t total_bytes = static_cast<int64_t>(p.E) * p.b_rows * nsc;
  const int vec_per_set = kRowsPerCta * nsc / 16;  // 128 * nsc is a multiple of 16 since K % 64 == 0
  for (int set = 0; set < (kSwiGLU ? 2 : 1); ++set) {
    const int64_t first = (set == 0 ? wrow_g : wrow_u) * nsc;
    const uint4* src = reinterpret_cast<const uint4*>(p.scales + first);
    uint4* dst = reinterpret_cast<uint4*>(sc_smem + set * kRowsPerCta * nsc);
    for (int i0 = threadIdx.x; i0 < vec_per_set; i0 += 4 * kWarps * 32) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kWarps * 32;
        v[u] = make_uint4(0, 0, 0, 0);
        if (i < vec_per_set && first + 16 * (i + 1) <= total_bytes) v[u] = __ldg(src + i);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kWarps * 32;
        if (i < vec_per_set) dst[i] = v[u];
      }
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");

  const int g = lane >> 2, t = lane & 3;
  const int col_base = blockIdx.x * kRowsPerCta + warp * 16;  // first output column of this warp
  const bool active = col_base < p.n_out;
  const uint8_t* scg0 = sc_smem + (warp * 16 + g) * nsc;
  const uint8_t* scg1 = scg0 + 8 * nsc;
  const uint8_t* scu0 = scg0 + kRowsPerCta * nsc;
  const uint8_t* scu1 = scu0 + 8 * nsc;
  int stage = 0;
  uint32_t phase = 0;
  for (int pass = 0; pass < npass; ++pass) {
    const int base = pass * kTokRows;
    const int nch = min(kMaxChunks, (n_rows - base + 7) / 8);
    float acc_g[kMaxChunks][4], acc_u[kMaxChunks][4];
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc_g[c][i] = acc_u[c][i] = 0.f;
    bool failed = false;
    for (int ks = 0; ks < ksteps; ++ks) {
      const bool ok = mbar_wait_bounded(full_bar(stage), phase, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        failed = true;
        break;
      }
      if (active) {
        const uint8_t* box = smem + stage * kStageBytes;
        const uint8_t* rg0 = box + (warp * 16 + g) * (kStepK / 2) + 4 * t;  // row g, word t of each block
        const uint8_t* rg1 = rg0 + 8 * (kStepK / 2);                        // row g + 8
#pragma unroll
        for (int blk = 0; blk < kStepK / 32; ++blk) {
          const int sj = (kStepK / 32) * ks + blk;  // scale block index along K
          if (sj >= nsc) break;                     // ragged last step
          const uint8_t* tok = box + kTokOff + (blk >> 1) * kTokBox;
          uint32_t ga[4], gb[4], ua[4], ub[4];  // f16 pairs of rows g and g+8 (gate, up)
          e2m1x8_to_f16x2x4(*reinterpret_cast<const uint32_t*>(rg0 + 16 * blk), ga);
          e2m1x8_to_f16x2x4(*reinterpret_cast<const uint32_t*>(rg1 + 16 * blk), gb);
          if (kSwiGLU) {
            e2m1x8_to_f16x2x4(*reinterpret_cast<const uint32_t*>(rg0 + kBox + 16 * blk), ua);
            e2m1x8_to_f16x2x4(*reinterpret_cast<const uint32_t*>(rg1 + kBox + 16 * blk), ub);
          }
          const float fg0 = e8m0(scg0[sj]), fg1 = e8m0(scg1[sj]);
          const float fu0 = kSwiGLU ? e8m0(scu0[sj]) : 0.f, fu1 = kSwiGLU ? e8m0(scu1[sj]) : 0.f;
#pragma unroll
          for (int c = 0; c < kMaxChunks; ++c) {
            if (c < nch) {
              // routed row n = 8c + g, elements [32 blk + 8t, +8): one 16-byte chunk of the swizzled box
              const int n = 8 * c + g;
              const uint4 bv = *reinterpret_cast<const uint4*>(tok + n * 128 + (((4 * (blk & 1) + t) ^ (n & 7)) << 4));
              float tg[4] = {0.f, 0.f, 0.f, 0.f};
              mma_f16_16816(tg, ga[0], gb[0], ga[1], gb[1], bv.x, bv.y);
              mma_f16_16816(tg, ga[2], gb[2], ga[3], gb[3], bv.z, bv.w);
              acc_g[c][0] = fmaf(fg0, tg[0], acc_g[c][0]);
              acc_g[c][1] = fmaf(fg0, tg[1], acc_g[c][1]);
              acc_g[c][2] = fmaf(fg1, tg[2], acc_g[c][2]);
              acc_g[c][3] = fmaf(fg1, tg[3], acc_g[c][3]);
              if (kSwiGLU) {
                float tu[4] = {0.f, 0.f, 0.f, 0.f};
                mma_f16_16816(tu, ua[0], ub[0], ua[1], ub[1], bv.x, bv.y);
                mma_f16_16816(tu, ua[2], ub[2], ua[3], ub[3], bv.z, bv.w);
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

// The routed rows in f16, times a power of two: 8 elements per thread.
__global__ void to_f16_scaled_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, int64_t n8, float s) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 v = in[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float lo = __uint_as_float(w[q] << 16) * s, hi = __uint_as_float(w[q] & 0xffff0000u) * s;
      asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(o[q]) : "f"(hi), "f"(lo));
    }
    out[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// (E * rows, K/2) bytes of codes, loaded as 64-byte x 128-row boxes.
bool make_tmap_codes(CUtensorMap* map, const uint8_t* codes, uint64_t rows, uint64_t half_k) {
  auto fn = tma_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {half_k, rows};
  cuuint64_t strides[1] = {half_k};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kStepK / 2), static_cast<cuuint32_t>(kRowsPerCta)};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kSwiGLU>
moe_status_t launch_skinny(const CUtensorMap& tm, const uint16_t* in, uint16_t* in16, const SkinnyParams& p,
                           cudaStream_t s) {
  // routed rows -> f16 (x in_scale) once, then TMA boxes of them feed the mma B operand
  const int64_t n8 = p.R * p.K / 8;
  const int64_t blocks = (n8 + 255) / 256;
  to_f16_scaled_kernel<<<static_cast<int>(blocks < 4096 ? blocks : 4096), 256, 0, s>>>(
      reinterpret_cast<const uint4*>(in), reinterpret_cast<uint4*>(in16), n8, p.in_scale);
  CUtensorMap tt;
  if (!make_tmap_bf16(&tt, in16, p.K, p.R, kTokRows)) return MOE_ERR_CUDA;
  const int srows = (kSwiGLU ? 2 : 1) * kRowsPerCta;
  const size_t smem = 1024 + Cfg<kSwiGLU>::kStages * Cfg<kSwiGLU>::kStageBytes +
                      (2 * Cfg<kSwiGLU>::kStages + 2) * 8 + static_cast<size_t>(srows) * (p.K / 32);
  if (cudaFuncSetAttribute(skinny_fp4_kernel<kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_CUDA;
  const dim3 grid((p.n_out + kRowsPerCta - 1) / kRowsPerCta, p.E);
  skinny_fp4_kernel<kSwiGLU><<<grid, (kWarps + 1) * 32, smem, s>>>(tm, tt, p);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

bool skinny_fp4_applies(const moe_dims_t& d) {
  // few routed rows per expert: at most 16 on average
  return d.wfmt == MOE_W_MXFP4 && static_cast<int64_t>(d.T) * d.k <= 16LL * d.E;
}

moe_status_t launch_mlp1_fp4_skinny(const moe_dims_t& d, const uint16_t* x_perm, const int32_t* offsets,
                                    const uint8_t* codes, const uint8_t* scales, const uint16_t* b1, uint16_t* h,
                                    uint16_t* tok16, int* status, cudaStream_t s) {
  SkinnyParams p{};
  p.E = d.E;
  p.K = d.D;
  p.n_out = d.I;
  p.b_rows = 2 * d.I;
  p.R = static_cast<int64_t>(d.T) * d.k;
  p.offsets = offsets;
  p.scales = scales;
  p.bias = b1;
  p.in_scale = 1.0f;
  p.out = h;
  p.status = status;
  CUtensorMap tm;
  if (!make_tmap_codes(&tm, codes, static_cast<uint64_t>(d.E) * 2 * d.I, d.D / 2)) return MOE_ERR_CUDA;
  return launch_skinny<true>(tm, x_perm, tok16, p, s);
}

moe_status_t launch_mlp2_fp4_skinny(const moe_dims_t& d, const uint16_t* h, const int32_t* perm,
                                    const int32_t* offsets, const float* topk_w, const uint8_t* codes,
                                    const uint8_t* scales, const uint16_t* b2, float* o_perm, uint16_t* tok16,
                                    int* status, cudaStream_t s) {
  SkinnyParams p{};
  p.E = d.E;
  p.K = d.I;
  p.n_out = d.D;
  p.b_rows = d.D;
  p.R = static_cast<int64_t>(d.T) * d.k;
  p.offsets = offsets;
  p.scales = scales;
  p.bias = b2;
  p.in_scale = 1.0f / 256.0f;
  p.perm = perm;
  p.topk_w = topk_w;
  p.out = o_perm;
  p.status = status;
  CUtensorMap tm;
  if (!make_tmap_codes(&tm, codes, static_cast<uint64_t>(d.E) * d.D, d.I / 2)) return MOE_ERR_CUDA;
  return launch_skinny<false>(tm, h, tok16, p, s);
}

}  // namespace moe
