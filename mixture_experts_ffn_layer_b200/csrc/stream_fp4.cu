// Grouped expert GEMMs with MXFP4 weights for decode-sized batches, on tcgen05.
//
// MXFP4 (GPT-OSS in Transformers blog, MXFP4 paragraph): E2M1 4-bit values
// with one E8M0 scale per 32 consecutive elements of the reduction dim. With a
// few routed rows per expert the layer is bound by streaming the 4.25-bit
// weights from HBM once, so the weights are the MMA's M side (128 weight rows
// per tile) and the expert's routed rows its N side (32 per pass):
//
//   warp 0      bulk copy of the tile's block scales, then TMA: a deep ring
//               of code stages, each the 128-row block's codes for 128 K
//               elements (64-byte swizzle; for mlp1 also the 128 up rows)
//               plus the 32 routed rows (f16, 128-byte swizzle) for them;
//   warps 5..   converters, two (mlp2) or four (mlp1) per TMEM lane
//               quarter, each thread half a weight row of a stage: decode the
//               codes with the hardware E2M1 -> f16 conversion, times
//               2^(s_block - s_row) where s_row is the row's largest block
//               scale (so every value is exact in f16 and none exceeds 6),
//               and store them to tensor memory;
//   warps 1..4  tcgen05.mma with A read from tensor memory (M = 128 weight
//               rows, K = 16) and B the routed rows from shared memory
//               (N = 32); four issuers with an accumulator each (a commit
//               stalls only its own issuer's MMA stream), each warp-wide with
//               one lane elected (operands warp-uniform), one commit per stage;
//   first four converter warps, epilogue: TMEM lane = output column; add the
//               partial accumulators, multiply back
//               2^(s_row - 127), add the bias, SwiGLU (mlp1) or gate weight
//               (mlp2); for each routed row the 32 lanes of a warp store 32
//               consecutive outputs.
// The decoded f16 tiles never touch shared memory: through it they would cost
// 4 bytes of shared-memory traffic per weight element (store, then the MMA's
// read), more than the SM can move at HBM speed. Only the codes (half a byte
// per element) and the routed rows pass through shared memory.
// The routed rows are converted once to f16 in the workspace, times a power of
// two (mlp2 uses h * 2^-8 so that |h| up to 2^24 stays finite in f16); the
// accumulator is multiplied back. A block whose scale is more than 14 binades
// below its row's largest one is flushed to zero (its terms are below 2^-14 of
// the row's scale; a row's scales span a few binades in practice).
#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int kRows = 128;                          // weight rows per tile: MMA M
constexpr int kTok = 32;                            // routed rows per pass: MMA N
constexpr int kCodeK = 128;                         // K elements per code stage
constexpr uint32_t kCodeTile = kRows * kCodeK / 2;  // 8 KB of codes per 128-row block (64-byte swizzle)
constexpr uint32_t kTokBox = kTok * 64 * 2;         // 64 K of f16 routed rows (128-byte swizzle)
constexpr uint32_t kTmemCols = 512;
constexpr int kMmaWarps = 4;                        // MMA issuers, one accumulator each
constexpr int kConv0 = 1 + kMmaWarps;               // first converter warp
constexpr uint32_t kAcol0 = kMmaWarps * kTok;       // TMEM columns [0, 128): accumulators; then the A ring
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr size_t kSmemLimit = 227 * 1024;

template <bool kSwiGLU>
struct Cfg {
  static constexpr int kTiles = kSwiGLU ? 2 : 1;  // gate and up weight blocks for mlp1
  // converter warps, a multiple of four (one group per TMEM lane quarter);
  // each thread converts half a weight row of one block per stage
  static constexpr int kConvWarps = kSwiGLU ? 16 : 8;
  static constexpr int kThreads = (kConv0 + kConvWarps) * 32;
  static constexpr int kMaxCodeStages = kSwiGLU ? 8 : 10;
  static constexpr int kAStages = kSwiGLU ? 3 : 4;  // (512 - 128) / (64 columns per tile)
  // code stage: [2 routed-row boxes][kTiles code tiles], 1024-byte aligned
  static constexpr uint32_t kCodeStageBytes = 2 * kTokBox + kTiles * kCodeTile;
  static_assert(kAcol0 + kAStages * kTiles * 64 <= kTmemCols, "A ring exceeds tensor memory");
};

struct StreamParams {
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
  void* out;              // h (R, I) bf16 (f16 with h_f16) or o_perm (R, D) fp32
  int* status;
  Act act;     // mlp1's activation
  bool h_f16;  // mlp1: store h as f16(bf16(h) * 2^-8), mlp2's input form, instead of bf16
  int stages;  // pipeline depth that fits shared memory next to the block scales
};

// Four E2M1 pairs (one 32-bit word = 8 codes, element 2j in the low nibble of
// byte j) to four f16 pairs.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t (&d)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(w));
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// f16 pair (2^delta, 2^delta) for delta <= 0; 0 below 2^-14 (a block that
// far below its row's largest one adds under 2^-14 of the row's scale).
__device__ __forceinline__ uint32_t pow2_f16x2(int delta) {
  const uint32_t h = static_cast<uint32_t>(max(delta + 15, 0)) << 10;
  return h | (h << 16);
}

// E8M0 scale value: 2^(s-127); 0 is 2^-127, 255 is NaN.
__device__ __forceinline__ float e8m0_value(int s) {
  if (s == 255) return __uint_as_float(0x7fc00000u);
  if (s == 0) return __uint_as_float(0x00400000u);
  return __uint_as_float(static_cast<uint32_t>(s) << 23);
}

// Instruction descriptor: kind::f16 with A = B = f16, D = fp32, K-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

template <bool kSwiGLU>
__global__ void __launch_bounds__(Cfg<kSwiGLU>::kThreads, 1) stream_fp4_kernel(const __grid_constant__ CUtensorMap tmCodes,
                                                                 const __grid_constant__ CUtensorMap tmTok,
                                                                 const StreamParams p) {
  using C = Cfg<kSwiGLU>;
  constexpr int SA = C::kAStages;
  const int SC = p.stages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nsc = p.K / 32;
  // [code ring][block scales kTiles x 128 x K/32][row reference scales][barriers][TMEM slot, abort]
  uint8_t* code_ring = smem;
  uint8_t* sc_smem = code_ring + SC * C::kCodeStageBytes;
  int* sref_smem = reinterpret_cast<int*>(sc_smem + C::kTiles * kRows * nsc);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sref_smem + C::kTiles * kRows);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * SC + 2 * SA + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  auto code_full = [&](int s) { return bar0 + 8u * s; };
  // code_empty: the converter warps release a code stage once the MMA that read
  // its routed rows has completed (seen as the A-ring slot SA stages later
  // coming free), so the MMA warps commit only to a_empty
  auto code_empty = [&](int s) { return bar0 + 8u * (SC + s); };
  auto a_conv = [&](int s) { return bar0 + 8u * (2 * SC + s); };
  auto a_empty = [&](int s) { return bar0 + 8u * (2 * SC + SA + s); };
  const uint32_t accf_bar = bar0 + 8u * (2 * SC + 2 * SA), acce_bar = accf_bar + 8u, done_bar = accf_bar + 16u,
                 sc_bar = accf_bar + 24u;

  const int e = blockIdx.y;
  // broadcast from lane 0 so the compiler knows the warp index is warp-uniform
  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x / 32), 0), lane = threadIdx.x % 32;
  const int seg0 = p.offsets[e], seg1 = p.offsets[e + 1];
  if (seg0 < 0 || seg1 < seg0 || seg1 > p.R) {
    if (threadIdx.x == 0) record_status(p.status, MOE_ERR_DEVICE_BOUNDS);
    return;
  }
  const int n_rows = seg1 - seg0;
  if (n_rows == 0) return;
  const int ncode = (p.K + kCodeK - 1) / kCodeK;
  const int npass = (n_rows + kTok - 1) / kTok;
  const int64_t wrow_g = static_cast<int64_t>(e) * p.b_rows + blockIdx.x * kRows;
  const int64_t wrow_u = wrow_g + p.n_out;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < SC; ++s) {
      mbar_init(code_full(s), 1);
      mbar_init(code_empty(s), C::kConvWarps);
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(a_conv(s), C::kConvWarps);
      mbar_init(a_empty(s), kMmaWarps);
    }
    mbar_init(accf_bar, kMmaWarps);
    mbar_init(acce_bar, 4);
    mbar_init(done_bar, kMmaWarps);
    mbar_init(sc_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // All 512 columns are allocated, so the allocation starts at lane 0, column 0.
  // Addressing from the constant keeps every TMEM operand warp-uniform (the
  // tcgen05 instructions take them in uniform registers).
  const uint32_t tmem_got = *tmem_slot;
  constexpr uint32_t tmem_base = 0;
  if (tmem_got != tmem_base) {
    if (threadIdx.x == 0) record_status(p.status, MOE_ERR_CUDA);
  } else if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer: scales, then codes + routed rows
      tma_prefetch_desc(&tmCodes);
      tma_prefetch_desc(&tmTok);
      {
        // the tile's block scales are 128 contiguous rows of K/32 bytes; rows
        // past the end of the tensor (the last up block) are not copied
        const int64_t total_rows = static_cast<int64_t>(p.E) * p.b_rows;
        uint32_t bytes[2] = {0, 0};
        for (int t = 0; t < C::kTiles; ++t) {
          const int64_t w0 = t == 0 ? wrow_g : wrow_u;
          const int64_t rows = total_rows - w0 < kRows ? total_rows - w0 : kRows;
          bytes[t] = rows > 0 ? static_cast<uint32_t>(rows * nsc) : 0u;
        }
        mbar_arrive_expect_tx(sc_bar, bytes[0] + bytes[1]);
        for (int t = 0; t < C::kTiles; ++t)
          if (bytes[t])
            bulk_load(smem_u32(sc_smem + t * kRows * nsc), p.scales + (t == 0 ? wrow_g : wrow_u) * nsc, bytes[t],
                      sc_bar);
      }
      int cs = 0, issued = 0;
      uint32_t cph = 0;
      bool failed = false;
      for (int pass = 0; pass < npass && !failed; ++pass) {
        for (int q = 0; q < ncode; ++q) {
          if (!mbar_wait_bounded(code_empty(cs), cph ^ 1u, abort_flag, kWaitNs)) {
            failed = true;
            break;
          }
          const int nh = p.K - q * kCodeK > 64 ? 2 : 1;  // 64-element routed-row boxes inside K
          const uint32_t tok = smem_u32(code_ring + cs * C::kCodeStageBytes), codes = tok + 2 * kTokBox;
          mbar_arrive_expect_tx(code_full(cs), C::kTiles * kCodeTile + nh * kTokBox);
          tma_load_2d(codes, &tmCodes, code_full(cs), q * (kCodeK / 2), static_cast<int32_t>(wrow_g));
          if (kSwiGLU)
            tma_load_2d(codes + kCodeTile, &tmCodes, code_full(cs), q * (kCodeK / 2), static_cast<int32_t>(wrow_u));
          for (int h = 0; h < nh; ++h)
            tma_load_2d(tok + h * kTokBox, &tmTok, code_full(cs), q * kCodeK + h * 64, seg0 + pass * kTok);
          ++issued;
          if (++cs == SC) {
            cs = 0;
            cph ^= 1u;
          }
        }
      }
      // the scale copy must have landed before the CTA can exit
      const bool sc_ok = mbar_wait_bounded(sc_bar, 0, nullptr, kWaitNs);
      if (failed || !sc_ok) {
        record_status(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        const int n = issued < SC ? issued : SC;  // wait for the copies still in flight
        for (int i = 0; i < n; ++i) {
          if (--cs < 0) {
            cs = SC - 1;
            cph ^= 1u;
          }
          mbar_wait_bounded(code_full(cs), cph, nullptr, kWaitNs);
        }
      }
    }
  } else if (warp >= 1 && warp <= kMmaWarps) {
    // ------------------------------------------------------------ MMA issuers (whole warp, one lane elected)
    // Four issuing warps, each with its own accumulator and its own commits:
    // a commit holds up its own warp's MMA stream for a long time, and with
    // 32 routed rows an MMA is short, so a single issuer would spend most of
    // each stage waiting. mlp1: issuer m takes tile m / 2 (gate, up) and the
    // K slices of parity m % 2; mlp2: the K slices kk = m mod 4. The
    // epilogue adds the partial accumulators in a fixed order.
    const int m = warp - 1;
    const int t = kSwiGLU ? m >> 1 : 0;
    const int kk0 = kSwiGLU ? m & 1 : m, kstep = kSwiGLU ? 2 : 4;
    const uint32_t idesc = idesc_f16_f32(kRows, kTok);
    const uint32_t dacc = tmem_base + m * kTok;
    int cs = 0, as = 0;
    uint32_t cph = 0, aph = 0;
    bool failed = false;
    for (int pass = 0; pass < npass && !failed; ++pass) {
      // the epilogue has read the previous pass's accumulators
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(acce_bar, (pass & 1) ^ 1u, abort_flag, kWaitNs))) {
        failed = true;
        break;
      }
      for (int q = 0; q < ncode; ++q) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(code_full(cs), cph, abort_flag, kWaitNs) &&
                                         mbar_wait_bounded(a_conv(as), aph, abort_flag, kWaitNs))) {
          failed = true;
          break;
        }
        tc_fence_after();
        const uint64_t bdesc = desc_kmajor_sw128(smem_u32(code_ring + cs * C::kCodeStageBytes));
        const uint32_t a0 = tmem_base + kAcol0 + (as * C::kTiles + t) * 64;
        const int nk = p.K - q * kCodeK >= kCodeK ? kCodeK / 16 : 4;  // K is a multiple of 64
        for (int kk = kk0; kk < nk; kk += kstep) {
          // routed-row box kk / 4, 32-byte K slice kk % 4 (descriptor address field counts 16 bytes)
          const uint64_t bd = bdesc + static_cast<uint64_t>(((kk >> 2) * kTokBox + (kk & 3) * 32) >> 4);
          mma_f16_tmem_a_elect(dacc, a0 + kk * 8, bd, idesc, (q != 0 || kk != kk0) ? 1u : 0u);
        }
        tc_commit_elect(a_empty(as));
        if (++as == SA) {
          as = 0;
          aph ^= 1u;
        }
        if (++cs == SC) {
          cs = 0;
          cph ^= 1u;
        }
      }
      if (failed) break;
      tc_commit_elect(accf_bar);
    }
    if (failed && lane == 0) {
      record_status(p.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    tc_commit_elect(done_bar);
    mbar_wait_bounded(done_bar, 0, nullptr, kWaitNs);
  } else {
    // ------------------------------------------------------------ converters (+ epilogue on the first four)
    const int cw = warp - kConv0;
    const int quarter = warp & 3;  // TMEM lanes this warp may touch: [32 * quarter, 32 * quarter + 32)
    const int r = quarter * 32 + lane;  // weight row within the tile
    // the warps of a lane quarter split a stage: mlp1 (gate | up) x (two K halves), mlp2 two K halves
    const int t = kSwiGLU ? (cw >> 2) & 1 : 0;
    const int e_lo = kSwiGLU ? (cw >> 3) * 64 : (cw >> 2) * 64;
    constexpr int kNel = kCodeK / 2;
    bool failed = !__all_sync(0xffffffffu, mbar_wait_bounded(sc_bar, 0, abort_flag, kWaitNs));
    const uint8_t* sc_row = sc_smem + (t * kRows + r) * nsc;
    int sref = 0;
    if (!failed) {
      uint32_t m = 0;
      const uint16_t* s2 = reinterpret_cast<const uint16_t*>(sc_row);  // K/32 is even: rows start on even bytes
      for (int b = 0; b < nsc / 2; ++b) {
        const uint32_t v = s2[b];
        m = max(m, max(v & 0xffu, v >> 8));
      }
      sref = static_cast<int>(m);
      sref_smem[t * kRows + r] = sref;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(C::kConvWarps * 32) : "memory");
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int swz = (r >> 1) & 3;  // 64-byte swizzle: 16-byte chunk c of row r sits at c ^ ((r / 2) % 4)

    int cs = 0, as = 0, g = 0;  // g: stage count over all passes
    uint32_t cph = 0, aph = 0;
    for (int pass = 0; pass < npass && !failed; ++pass) {
      for (int q = 0; q < ncode; ++q, ++g) {
        if (!__all_sync(0xffffffffu, mbar_wait_backoff(code_full(cs), cph, abort_flag, kWaitNs) &&
                                         mbar_wait_backoff(a_empty(as), aph ^ 1u, abort_flag, kWaitNs))) {
          failed = true;
          break;
        }
        tc_fence_after();
        if (g >= SA && lane == 0) {
          // A slot `as` free again: the MMA of stage g - SA has completed, so
          // that stage's code slot (codes read by this warp long ago, routed
          // rows read by that MMA) may be refilled
          const int rs = cs - SA < 0 ? cs - SA + SC : cs - SA;
          mbar_arrive(code_empty(rs));
        }
        const uint8_t* crow = code_ring + cs * C::kCodeStageBytes + 2 * kTokBox + t * kCodeTile + r * (kCodeK / 2);
        const uint32_t acol = tmem_base + lane_addr + kAcol0 + (as * C::kTiles + t) * 64;
        const int kq = min(kCodeK, p.K - q * kCodeK);
#pragma unroll
        for (int bi = 0; bi < kNel / 32; ++bi) {
          const int b = e_lo / 32 + bi;  // 32-element scale block within the stage
          if (b * 32 < kq) {
            const uint4 w = *reinterpret_cast<const uint4*>(crow + ((b ^ swz) << 4));
            const uint32_t f = pow2_f16x2(static_cast<int>(sc_row[q * 4 + b]) - sref);
            const uint32_t words[4] = {w.x, w.y, w.z, w.w};
            uint32_t v[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t d[4];
              e2m1x8_to_f16x2x4(words[c], d);
#pragma unroll
              for (int u = 0; u < 4; ++u) v[4 * c + u] = hmul2(d[u], f);
            }
            tmem_st_x16(acol + b * 16, v);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(a_conv(as));
        if (++as == SA) {
          as = 0;
          aph ^= 1u;
        }
        if (++cs == SC) {
          cs = 0;
          cph ^= 1u;
        }
      }
      if (failed || cw >= 4) continue;

      // ---------------------------------------------------------- epilogue (the first four converter warps)
      if (!__all_sync(0xffffffffu, mbar_wait_backoff(accf_bar, pass & 1, abort_flag, kWaitNs))) {
        failed = true;
        break;
      }
      tc_fence_after();
      const int col = blockIdx.x * kRows + r;  // TMEM lane = weight row = output column
      const bool live = col < p.n_out;
      const float undo = 1.0f / p.in_scale;
      const float fg = e8m0_value(sref_smem[r]) * undo;
      const float bg = live ? bf16_bits_to_float(p.bias[wrow_g + r]) : 0.f;
      float fu = 0.f, bu = 0.f;
      if (kSwiGLU) {
        fu = e8m0_value(sref_smem[kRows + r]) * undo;
        bu = live ? bf16_bits_to_float(p.bias[wrow_u + r]) : 0.f;
      }
      const int nb = min(kTok, n_rows - pass * kTok);
#pragma unroll
      for (int c = 0; c < kTok / 8; ++c) {  // eight routed rows per TMEM load
        // the four partial accumulators: mlp1 gate = 0 + 1, up = 2 + 3; mlp2 0 + 1 + 2 + 3
        uint32_t v0[8], v1[8], v2[8], v3[8];
        tmem_ld_x8(tmem_base + lane_addr + 0 * kTok + 8 * c, v0);
        tmem_ld_x8(tmem_base + lane_addr + 1 * kTok + 8 * c, v1);
        tmem_ld_x8(tmem_base + lane_addr + 2 * kTok + 8 * c, v2);
        tmem_ld_x8(tmem_base + lane_addr + 3 * kTok + 8 * c, v3);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int jr = 8 * c + i;
          if (!live || jr >= nb) continue;
          const int64_t row = seg0 + pass * kTok + jr;
          const float a01 = __uint_as_float(v0[i]) + __uint_as_float(v1[i]);
          const float a23 = __uint_as_float(v2[i]) + __uint_as_float(v3[i]);
          const float g = (kSwiGLU ? a01 : a01 + a23) * fg + bg;
          if (kSwiGLU) {
            const float u = a23 * fu + bu;
            const uint16_t hb = float_to_bf16_bits(glu_act(g, u, p.act));
            static_cast<uint16_t*>(p.out)[row * p.n_out + col] =
                p.h_f16 ? __half_as_ushort(__float2half_rn(bf16_bits_to_float(hb) * (1.0f / 256.0f))) : hb;
          } else {
            const int32_t a = p.perm[row];
            float wgt = 0.f;
            if (a >= 0 && a < p.R)
              wgt = p.topk_w[a];
            else
              record_status(p.status, MOE_ERR_DEVICE_BOUNDS);
            static_cast<float*>(p.out)[row * p.n_out + col] = wgt * g;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_bar);  // the accumulators may be overwritten
    }
    if (failed && lane == 0) {
      record_status(p.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_got, kTmemCols);
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

// (E * rows, K/2) bytes of codes, loaded as 64-byte x 128-row boxes with the
// 64-byte swizzle (conflict-free 16-byte reads when each thread takes a row).
bool make_tmap_codes(CUtensorMap* map, const uint8_t* codes, uint64_t rows, uint64_t half_k) {
  auto fn = tma_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {half_k, rows};
  cuuint64_t strides[1] = {half_k};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kCodeK / 2), static_cast<cuuint32_t>(kRows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kSwiGLU>
moe_status_t launch_stream(const CUtensorMap& tm, const uint16_t* in, uint16_t* in16, bool in_f16,
                           const StreamParams& p, cudaStream_t s) {
  using C = Cfg<kSwiGLU>;
  // routed rows -> f16 (x in_scale) once, then TMA boxes of them are the MMA's
  // B operand; in_f16: `in` already holds them in that form
  if (in_f16) {
    in16 = const_cast<uint16_t*>(in);
  } else {
    const int64_t n8 = p.R * p.K / 8;
    const int64_t blocks = (n8 + 255) / 256;
    to_f16_scaled_kernel<<<static_cast<int>(blocks < 4096 ? blocks : 4096), 256, 0, s>>>(
        reinterpret_cast<const uint4*>(in), reinterpret_cast<uint4*>(in16), n8, p.in_scale);
  }
  CUtensorMap tt;
  if (!make_tmap_bf16(&tt, in16, p.K, p.R, kTok)) return MOE_ERR_CUDA;
  const size_t fixed = 1024 + 16 + static_cast<size_t>(C::kTiles) * kRows * (p.K / 32) +
                       static_cast<size_t>(C::kTiles) * kRows * 4 + (2 * C::kAStages + 4) * 8;
  int stages = C::kMaxCodeStages;
  auto bytes = [&](int st) { return fixed + static_cast<size_t>(st) * C::kCodeStageBytes + 2 * st * 8; };
  // the code ring must be deeper than the A ring (a code stage is released SA
  // stages after it was converted)
  while (stages > C::kAStages + 1 && bytes(stages) > kSmemLimit) --stages;
  if (bytes(stages) > kSmemLimit) return MOE_ERR_UNSUPPORTED;
  StreamParams q = p;
  q.stages = stages;
  const size_t smem = bytes(stages);
  if (cudaFuncSetAttribute(stream_fp4_kernel<kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_CUDA;
  const dim3 grid((p.n_out + kRows - 1) / kRows, p.E);
  stream_fp4_kernel<kSwiGLU><<<grid, C::kThreads, smem, s>>>(tm, tt, q);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

bool stream_fp4_applies(const moe_dims_t& d) {
  // few routed rows per expert: at most 16 on average
  return d.wfmt == MOE_W_MXFP4 && static_cast<int64_t>(d.T) * d.k <= 16LL * d.E;
}

moe_status_t launch_mlp1_fp4_stream(const moe_dims_t& d, const uint16_t* x_perm, const int32_t* offsets,
                                    const uint8_t* codes, const uint8_t* scales, const uint16_t* b1, uint16_t* h,
                                    uint16_t* tok16, int* status, cudaStream_t s, bool in_f16, bool h_f16) {
  StreamParams p{};
  p.E = d.E;
  p.K = d.D;
  p.n_out = d.I;
  p.b_rows = 2 * d.I;
  p.R = static_cast<int64_t>(d.T) * d.k;
  p.offsets = offsets;
  p.scales = scales;
  p.bias = b1;
  p.in_scale = 1.0f;
  p.act = act_of(d);
  p.h_f16 = h_f16;
  p.out = h;
  p.status = status;
  CUtensorMap tm;
  if (!make_tmap_codes(&tm, codes, static_cast<uint64_t>(d.E) * 2 * d.I, d.D / 2)) return MOE_ERR_CUDA;
  return launch_stream<true>(tm, x_perm, tok16, in_f16, p, s);
}

moe_status_t launch_mlp2_fp4_stream(const moe_dims_t& d, const uint16_t* h, const int32_t* perm,
                                    const int32_t* offsets, const float* topk_w, const uint8_t* codes,
                                    const uint8_t* scales, const uint16_t* b2, float* o_perm, uint16_t* tok16,
                                    int* status, cudaStream_t s, bool in_f16) {
  StreamParams p{};
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
  return launch_stream<false>(tm, h, tok16, in_f16, p, s);
}

}  // namespace moe
