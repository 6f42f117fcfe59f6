// Grouped expert GEMMs with MXFP4 expert weights on block-scaled tcgen05 MMA.
//
// MXFP4 (GPT-OSS in Transformers blog, MXFP4 paragraph): E2M1 4-bit values
// with one E8M0 scale per 32 consecutive elements of the reduction dim; the
// torchtitan GPT-OSS guide ("grouped matrix multiplication") runs the expert
// FFN as two grouped GEMMs over the expert segments of the routed rows.
//
// The sm_100a tensor cores multiply MX operands directly
// (tcgen05.mma kind::mxf8f6f4.block_scale: per-32-element E8M0 scales for
// both operands, read from tensor memory), but both operands must be MX
// types. The weights stay E2M1 as stored; the bf16 activations (routed rows,
// then h) are quantised to MX E4M3 as a PAIR of terms per element, hi + lo,
// each with its own E8M0 scale per 32 elements:
//   hi = e4m3(v / 2^(e-7)),  lo = e4m3((v - hi*2^(e-7)) / 2^(e_r-7)),
// e and e_r the binary exponents of the block's largest |v| and largest
// residual. hi keeps 4 significant bits, lo the next 4, so the pair carries
// ~8 bits like bf16 itself (one E4M3 alone would leave errors of ~2^-5 per
// element, too coarse for the layer's output). The two MMAs (hi, lo) per K
// block accumulate into the same fp32 accumulator; every weight byte crosses
// HBM and L2 at 4.25 bits per element and is never expanded.
//
// One persistent, warp-specialised kernel for mlp1 (+bias, SwiGLU) and mlp2
// (+bias, gate weight); tiles are (expert, column tile, 128-row tile) over
// the device-side expert offsets, as in the bf16 grouped GEMM:
//   warp 0      activation-side producer, per 128-K stage: the tile's 128
//               rows, hi and lo E4M3 planes in one 3-D TMA box (128-byte
//               swizzle), and their 1 KB of scale factors (TMA);
//   warp 6      weight-side producer: the weight rows' E2M1 codes, gate and
//               up halves in one TMA box of the 16U4_ALIGN16B type (which
//               unpacks every 8 bytes of codes into the 16-byte slot the MMA's
//               E2M1 operand layout wants), and their 1 KB of scale factors;
//   warp 1      MMA: tcgen05.cp of the stage's scale factors into tensor
//               memory, then per 32-K block two block-scaled MMAs (hi, lo),
//               M = 128 rows, N = the tile's weight rows; whole warp, one
//               elected lane issuing;
//   warps 2..5  epilogue: bias + SwiGLU into h (bf16, or straight into the
//               quantised hi/lo form mlp2 reads), or bias * gate weight into
//               the fp32 expert outputs.
// A thread that issues a TMA copy cannot issue the next for ~60 ns whatever
// its size, so each operand of a stage is one copy and two threads share the
// copies; each completes its own full barrier, and the MMA warp waits on both.
//
// Scale factors reach tensor memory through tcgen05.cp, which reads 128 rows'
// scales of 4 K blocks as a 32 x 16-byte shared-memory atom (row m's scale
// of block kb at byte (m % 32) * 16 + (m / 32) * 4 + kb). Both operands'
// scales are stored in that form in global memory, so a stage moves them
// with one copy each:
//  - activations, tile-blocked: for m-tile g (the 128-row tiles of all
//    experts, numbered expert by expert) and stage q, a 2 KB block at
//    (g * nst + q) * 2048 (hi atom, lo atom, the small-expert kernel's atom),
//    written by the quantiser / mlp1's epilogue;
//  - weights, per (expert, column tile, stage): 1 KB (two atoms, rows 0..127
//    and 128..255 of the tile), written from the (E, N, K/32) scales by a
//    preparation pass, per call for the experts a call routes to (13 MB read
//    at the 20B shape) or once for all experts (moe_mxfp4_prepare).
// The codes are read either as stored, (E, N, K/2) bytes (each stage a
// 64-byte piece of every row, rows K/2 bytes apart; TMA's 4-bit type needs
// K to be a multiple of 128, so for K % 128 = 64 (GPT-OSS: 2880) the per-call
// pass writes each weight row's last 64 codes padded with zeros to a
// 128-element row, loaded through a second tensor map), or from the
// prepare-once copy, K-block-major (E, nst, N, 64 bytes) with the last block
// padded, where a stage's rows are one contiguous run per half: 64-byte
// pieces of rows 1.4 KB apart leave DRAM at about half its bandwidth.
//
// Every mbarrier wait is bounded (1 s); on timeout the kernel records
// MOE_ERR_TIMEOUT, stops issuing, waits for its in-flight copies and MMAs,
// frees TMEM and returns.
#include <cuda_fp16.h>

#include <cstring>

#include "common.cuh"
#include "gemm_common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int BM = 128;                                   // token rows per tile = TMEM lanes
constexpr int BKE = 128;                                  // K elements per stage (4 scale blocks)
constexpr int kStages = 3;
constexpr int kThreads = 224;                             // 2 producers, MMA, 4 epilogue warps
constexpr int kWProducerWarp = 6;                         // the weight-side producer
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccStride = 256;                      // accumulators at columns 0 and 256
// Two 16-column scale-factor regions, used by alternate stages: after
// accumulator 0 (columns 240..255) and after accumulator 1 (496..511).
constexpr uint32_t kSfCol0 = 240, kSfCol1 = 496;
constexpr int kMaxN = 240;                                // MMA N (weight rows per tile) at most
constexpr uint32_t kAOpBytes = BM * BKE;                  // one E4M3 operand box: 16 KB
constexpr uint32_t kAStageBytes = 2 * kAOpBytes + 1024;   // hi, lo, their scale atoms
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr int kCtrlBytes = 256;

struct MxParams {
  GemmParams g;            // sizes, bias, perm / gate weights, output, status, activation
  int nst;                 // 128-K stages
  int kfull;               // K rounded down to a multiple of 128 (the rest comes from the tail rows)
  int wprep;               // codes from the prepared copy (K-block-major), else from the weights as stored
  const uint8_t* a_sf;     // activation scales, tile-blocked (nst stages)
  uint8_t* hq;             // mlp1, optional: h quantised, hi (R, I) then lo (R, I) E4M3
  uint8_t* h_sf;           // and its scales, tile-blocked with h_nst stages
  int h_nst;
  int small_max;           // experts with 1..small_max rows are left to the small-expert kernel (0: none)
};

// One stage: A hi, A lo, A scale atoms, the B operand (mma_n rows of 128
// bytes), B scale atoms (two of 512 bytes), rounded up to 1 KB.
__host__ __device__ constexpr uint32_t stage_bytes(int mma_n) {
  return kAStageBytes + (static_cast<uint32_t>(mma_n) * 128 + 1024 + 1023) / 1024 * 1024;
}

__device__ __forceinline__ uint32_t sf_atom_off(int m, int kb) {
  return static_cast<uint32_t>((m & 31) * 16 + (m >> 5) * 4 + kb);
}

// Activation scales, per (m-tile g, 128-K stage q), a kSfBlock-byte block:
//   [0, 512)     hi atom of the tile's 128 rows,
//   [512, 1024)  lo atom,
//   [1024, 1536) the small-expert kernel's 64-row atom of rows 0..31: line m
//                holds row m's 4 hi scales, then its 4 lo scales (MMA rows m
//                and 32 + m of its hi-over-lo operand).
constexpr uint32_t kSfBlock = 2048;

// Store row m's (of its 128-row tile) hi and lo scales of K block kb of a stage.
__device__ __forceinline__ void store_act_sf(uint8_t* block, int m, int kb, uint32_t sfh, uint32_t sfl) {
  const uint32_t o = sf_atom_off(m, kb);
  block[o] = static_cast<uint8_t>(sfh);
  block[512 + o] = static_cast<uint8_t>(sfl);
  if (m < 32) {
    block[1024 + m * 16 + kb] = static_cast<uint8_t>(sfh);
    block[1024 + m * 16 + 4 + kb] = static_cast<uint8_t>(sfl);
  }
}

// ---------------------------------------------------------------- E4M3 hi/lo quantisation
// Two fp32 -> two E4M3 (round to nearest even, saturating), `a` in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

// Two E4M3 (low byte first) -> their exact values.
__device__ __forceinline__ float2 e4m3x2_value(uint32_t v) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(v)));
  return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

// 32 consecutive values of one row -> their hi and lo E4M3 codes (32 bytes
// each, element i in byte i) and E8M0 scale bytes. A block whose largest |v|
// is below 2^-119 is taken as zero (its terms are below 2^-119 * sum|w|); a
// non-finite value makes the whole block NaN, which the MMA propagates.
__device__ __forceinline__ void quant32(const float (&v)[32], uint32_t (&hi)[8], uint32_t (&lo)[8], uint32_t& sfh,
                                        uint32_t& sfl) {
  float amax = 0.f, chk = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    amax = fmaxf(amax, fabsf(v[i]));
    chk += v[i] * 0.f;  // NaN if any value is inf or NaN
  }
  if (chk != 0.f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) hi[i] = lo[i] = 0x7f7f7f7fu;
    sfh = sfl = 127;
    return;
  }
  if (!(amax >= 0x1p-119f)) {
#pragma unroll
    for (int i = 0; i < 8; ++i) hi[i] = lo[i] = 0u;
    sfh = sfl = 127;
    return;
  }
  // scale 2^(e-7) puts the block's largest value in [128, 256), inside E4M3's 448
  const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127;
  const float mul = __uint_as_float(static_cast<uint32_t>(127 + 7 - e) << 23);
  const float back = __uint_as_float(static_cast<uint32_t>(127 + e - 7) << 23);
  sfh = static_cast<uint32_t>(e + 120);
  float r[32];
  float rmax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t q = e4m3x2(v[2 * i] * mul, v[2 * i + 1] * mul);
    const float2 d = e4m3x2_value(q);
    r[2 * i] = v[2 * i] - d.x * back;
    r[2 * i + 1] = v[2 * i + 1] - d.y * back;
    rmax = fmaxf(rmax, fmaxf(fabsf(r[2 * i]), fabsf(r[2 * i + 1])));
    if (i & 1)
      hi[i >> 1] |= q << 16;
    else
      hi[i >> 1] = q;
  }
  if (!(rmax >= 0x1p-119f)) {
#pragma unroll
    for (int i = 0; i < 8; ++i) lo[i] = 0u;
    sfl = 127;
    return;
  }
  const int er = static_cast<int>((__float_as_uint(rmax) >> 23) & 0xffu) - 127;
  const float mul2 = __uint_as_float(static_cast<uint32_t>(127 + 7 - er) << 23);
  sfl = static_cast<uint32_t>(er + 120);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t q = e4m3x2(r[2 * i] * mul2, r[2 * i + 1] * mul2);
    if (i & 1)
      lo[i >> 1] |= q << 16;
    else
      lo[i >> 1] = q;
  }
}

// Expert segment table and m-tile prefix (numbering of the 128-row tiles of
// all experts, expert by expert) from the offsets, into shared memory, by one
// warp; returns false (and records the status) for offsets out of order or
// range. mpre has E+1 entries.
__device__ bool load_segments(const int32_t* offsets, int E, int64_t R, int* seg, int* mpre, int* status) {
  const int lane = threadIdx.x & 31;
  bool bad = false;
  for (int e = lane; e <= E; e += 32) {
    const int o = offsets[e];
    seg[e] = o;
    if (o < 0 || o > R || (e == 0 && o != 0)) bad = true;
  }
  __syncwarp();
  const int per = (E + 31) / 32;
  const int e0 = lane * per;
  int local = 0;
  for (int e = e0; e < e0 + per && e < E; ++e) {
    const int cnt = seg[e + 1] - seg[e];
    if (cnt < 0) bad = true;
    local += cnt > 0 ? (cnt + BM - 1) / BM : 0;
  }
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += u;
  }
  int run = incl - local;
  for (int e = e0; e < e0 + per && e < E; ++e) {
    mpre[e] = run;
    const int cnt = seg[e + 1] - seg[e];
    run += cnt > 0 ? (cnt + BM - 1) / BM : 0;
  }
  if (lane == 31) mpre[E] = incl;
  __syncwarp();
  bad = __any_sync(0xffffffffu, bad);
  if (bad && lane == 0) record_status(status, MOE_ERR_DEVICE_BOUNDS);
  return !bad;
}

// Tile prefix for a kernel's schedule, by one warp: tpre[e] = sum over
// experts e' < e of tiles(e'), with tiles(e) = per_expert(count of e).
template <class F>
__device__ void schedule_prefix(const int* seg, int E, int* tpre, F per_expert) {
  const int lane = threadIdx.x & 31;
  const int per = (E + 31) / 32;
  const int e0 = lane * per;
  int local = 0;
  for (int e = e0; e < e0 + per && e < E; ++e) local += per_expert(seg[e + 1] - seg[e]);
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += u;
  }
  int run = incl - local;
  for (int e = e0; e < e0 + per && e < E; ++e) {
    tpre[e] = run;
    run += per_expert(seg[e + 1] - seg[e]);
  }
  if (lane == 31) tpre[E] = incl;
  __syncwarp();
}

// ---------------------------------------------------------------- quantiser kernel
// Rows of `src` (bf16; with `perm`, row r is x[perm[r] / k], the gather of
// the routed rows) -> hi (R, K) and lo (R, K) E4M3 at dst and dst + R*K, and
// their scales in the tile-blocked layout. One thread per 32-element block.
__global__ void __launch_bounds__(256) mx_quant_kernel(const uint16_t* __restrict__ src, const int32_t* __restrict__ perm,
                                                       int k, int64_t R, int K, const int32_t* __restrict__ offsets,
                                                       int E, int nst, uint8_t* __restrict__ dst,
                                                       uint8_t* __restrict__ sf, int* status) {
  __shared__ int seg[257], mpre[257];
  __shared__ int ok_s;
  if (threadIdx.x < 32) {
    const bool ok = load_segments(offsets, E, R, seg, mpre, status);
    if (threadIdx.x == 0) ok_s = ok;
  }
  __syncthreads();
  if (!ok_s) return;
  const int nb = K / 32;
  const int64_t total = R * nb;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / nb;
    const int b = static_cast<int>(i - r * nb);
    int64_t srow = r;
    if (perm) {
      const int32_t a = perm[r];
      if (a < 0 || a >= R) {
        if (b == 0) record_status(status, MOE_ERR_DEVICE_BOUNDS);
        continue;
      }
      srow = a / k;
    }
    uint32_t w[16];
    ld_global_v8u(src + srow * K + 32 * b, *reinterpret_cast<uint32_t(*)[8]>(w));
    ld_global_v8u(src + srow * K + 32 * b + 16, *reinterpret_cast<uint32_t(*)[8]>(w + 8));
    float v[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
    uint32_t hi[8], lo[8], sfh, sfl;
    quant32(v, hi, lo, sfh, sfl);
    st_global_v8u(dst + r * K + 32 * b, hi);
    st_global_v8u(dst + R * K + r * K + 32 * b, lo);
    // the row's expert (last e with seg[e] <= r among non-empty ones) and tile
    int lo_e = 0, hi_e = E - 1;
    while (lo_e < hi_e) {
      const int mid = (lo_e + hi_e + 1) >> 1;
      if (seg[mid] <= r)
        lo_e = mid;
      else
        hi_e = mid - 1;
    }
    const int local = static_cast<int>(r - seg[lo_e]);
    const int64_t g = mpre[lo_e] + local / BM;
    store_act_sf(sf + (g * nst + b / 4) * kSfBlock, local % BM, b % 4, sfh, sfl);
  }
}

// ---------------------------------------------------------------- weight preparation
// The weight scales in the atom layout the MMA's scale copies read, and the
// codes in the form the GEMM kernels load, for the experts each kernel takes:
//  - big-tile kernel (more than small_max rows): 1 KB per (expert, column
//    tile, stage), two atoms for the tile's mma_n weight rows;
//  - small-expert kernel (1..small_max rows): 512 B per (expert, weight tile,
//    stage), one atom for its 128 weight rows (mlp1: 64 gate, 64 up);
//  - per call (codes read as stored, row by row): with K % 128 = 64, each
//    weight row's last 64 codes padded with zeros to a 128-element row (64
//    bytes), for the 4-bit TMA type;
//  - prepare-once form: the codes K-block-major, (E, nst, N, 64 bytes), the
//    128 codes of every row for K block q side by side and the ragged last
//    block padded with zeros. A stage's weight rows are then one contiguous
//    run per gate / up half (whole DRAM pages, where reading 64-byte pieces of
//    rows K/2 bytes apart leaves DRAM at a fraction of its bandwidth).
// With all_experts set (the prepare-once form) every expert gets both atom
// sets and its codes; otherwise only what this call's routing uses, and the
// tail rows. One CTA per (expert, tile), per 256 weight rows of an expert, or
// per (expert, K block, 64 weight rows).
struct PrepArgs {
  const uint8_t* codes;
  const uint8_t* scales;
  int E, b_rows, K, n_out, n_tile, mma_n, NT, NT2, nst, swiglu;
  const int32_t* offsets;
  int small_max, all_experts;
  uint8_t* w_sf;
  uint8_t* w_sf_small;
  uint8_t* tail;       // per call with K % 128 != 0, else null
  uint8_t* codes_out;  // prepare-once form, else null
};

__global__ void __launch_bounds__(256) mx_prep_weights_kernel(const PrepArgs a) {
  const int nsc = a.K / 32, half_k = a.K / 2, kfull = a.K / BKE * BKE;
  const int64_t wrows_all = static_cast<int64_t>(a.E) * a.b_rows;
  const int n_big = a.E * a.NT, n_small = a.small_max > 0 ? a.E * a.NT2 : 0;
  const int rblocks = (a.b_rows + 255) / 256;
  const int n_tail = a.tail ? a.E * rblocks : 0;
  int blk = blockIdx.x;
  // the 4 scale bytes of a weight row for stage q (127 = 1.0 past K or past the tensor)
  auto sc4 = [&](int64_t row, int q) -> uint32_t {
    if (row >= wrows_all) return 0x7f7f7f7fu;
    const uint16_t* s2 = reinterpret_cast<const uint16_t*>(a.scales + row * nsc + q * 4);
    const uint32_t lo16 = __ldg(s2);
    const uint32_t hi16 = q * 4 + 2 < nsc ? static_cast<uint32_t>(__ldg(s2 + 1)) : 0x7f7fu;
    return lo16 | (hi16 << 16);
  };
  auto count = [&](int e) { return a.all_experts ? -1 : __ldg(a.offsets + e + 1) - __ldg(a.offsets + e); };
  if (blk < n_big) {
    const int e = blk / a.NT, nt = blk - e * a.NT;
    const int c = count(e);
    if (!a.all_experts && c <= a.small_max) return;
    uint8_t* out = a.w_sf + static_cast<int64_t>(blk) * a.nst * 1024;
    for (int i = threadIdx.x; i < a.nst * a.mma_n; i += blockDim.x) {
      const int q = i / a.mma_n, j = i - q * a.mma_n;
      const int64_t row = static_cast<int64_t>(e) * a.b_rows +
                          (a.swiglu ? (j < a.n_tile ? nt * a.n_tile + j : a.n_out + nt * a.n_tile + (j - a.n_tile))
                                    : nt * a.n_tile + j);
      *reinterpret_cast<uint32_t*>(out + q * 1024 + (j >> 7) * 512 + sf_atom_off(j & 127, 0)) = sc4(row, q);
    }
    return;
  }
  blk -= n_big;
  if (blk < n_small) {
    const int e = blk / a.NT2, wt = blk - e * a.NT2;
    const int c = count(e);
    if (!a.all_experts && (c < 1 || c > a.small_max)) return;
    uint8_t* out = a.w_sf_small + static_cast<int64_t>(blk) * a.nst * 512;
    for (int i = threadIdx.x; i < a.nst * 128; i += blockDim.x) {
      const int q = i >> 7, j = i & 127;
      const int64_t row = static_cast<int64_t>(e) * a.b_rows +
                          (a.swiglu ? (j < 64 ? wt * 64 + j : a.n_out + wt * 64 + (j - 64)) : wt * 128 + j);
      *reinterpret_cast<uint32_t*>(out + q * 512 + sf_atom_off(j, 0)) = sc4(row, q);
    }
    return;
  }
  blk -= n_small;
  if (blk < n_tail) {
    const int e = blk / rblocks, rb = blk - e * rblocks;
    if (!a.all_experts && count(e) <= 0) return;
    for (int i = threadIdx.x; i < 256 * 4; i += blockDim.x) {
      const int r = rb * 256 + (i >> 2), piece = i & 3;
      if (r >= a.b_rows) break;
      const int64_t row = static_cast<int64_t>(e) * a.b_rows + r;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (piece < 2) v = __ldg(reinterpret_cast<const uint4*>(a.codes + row * half_k + kfull / 2 + piece * 16));
      *reinterpret_cast<uint4*>(a.tail + row * 64 + piece * 16) = v;
    }
    return;
  }
  blk -= n_tail;
  if (a.codes_out) {
    // 64 rows of K block q of expert e, 16 bytes per thread
    const int rchunks = (a.b_rows + 63) / 64;
    const int e = blk / (a.nst * rchunks), rem = blk - e * (a.nst * rchunks);
    const int q = rem / rchunks, rc = rem - q * rchunks;
    if (e >= a.E) return;
    const int r = rc * 64 + (threadIdx.x >> 2), piece = threadIdx.x & 3;
    if (r >= a.b_rows) return;
    const int64_t row = static_cast<int64_t>(e) * a.b_rows + r;
    const int byte = q * 64 + piece * 16;  // within the stored row of K/2 bytes
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (byte < half_k) v = __ldg(reinterpret_cast<const uint4*>(a.codes + row * half_k + byte));
    *reinterpret_cast<uint4*>(a.codes_out + ((static_cast<int64_t>(e) * a.nst + q) * a.b_rows + r) * 64 + piece * 16) = v;
  }
}

// ---------------------------------------------------------------- the block-scaled grouped GEMM
template <bool kSwiGLU>
__global__ void __launch_bounds__(kThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAsf,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmBtail,
                   const __grid_constant__ CUtensorMap tmBsf, const MxParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const GemmParams& gp = p.g;
  const uint32_t sst = stage_bytes(gp.mma_n);
  constexpr uint32_t kBOff = kAStageBytes;                                 // B operand within a stage
  const uint32_t sfb_off = kBOff + static_cast<uint32_t>(gp.mma_n) * 128;  // B scale atoms within a stage
  uint8_t* ring = smem;
  uint8_t* ctrl = ring + kStages * sst;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctrl);
  constexpr int kBars = 3 * kStages + 5;
  static_assert(8 * kBars + 16 <= kCtrlBytes, "control block overflow");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* total_s = reinterpret_cast<int*>(tmem_slot + 2);
  int* seg = reinterpret_cast<int*>(ctrl + kCtrlBytes);
  int* mpre = seg + (gp.E + 1);
  int* tpre = mpre + (gp.E + 1);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x / 32), 0), lane = threadIdx.x % 32;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };                // activation side landed
  auto full_w = [&](int s) { return bar0 + 8u * (kStages + s); };      // weight side landed
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
  auto tfull = [&](int b) { return bar0 + 8u * (3 * kStages + b); };
  auto tempty = [&](int b) { return bar0 + 8u * (3 * kStages + 2 + b); };
  const uint32_t done_bar = bar0 + 8u * (3 * kStages + 4);

  // ---- prologue: segments, tile prefixes, barriers, TMEM
  if (warp == 0) {
    const bool ok = load_segments(gp.offsets, gp.E, gp.R, seg, mpre, gp.status);
    // mpre numbers the 128-row tiles of all experts (the activation scales'
    // layout); the schedule leaves out experts the small-expert kernel takes
    const int small_max = p.small_max, NT = gp.NT;
    schedule_prefix(seg, gp.E, tpre, [small_max, NT](int cnt) {
      return (cnt > small_max) ? (cnt + BM - 1) / BM * NT : 0;
    });
    if (lane == 0) {
      *abort_flag = 0;
      *total_s = ok ? tpre[gp.E] : 0;
    }
  }
  __syncthreads();
  // A CTA without a tile (on decode-sized batches every expert may go to the
  // small-expert kernel) leaves before it allocates tensor memory.
  if (static_cast<int>(blockIdx.x) >= *total_s) return;
  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(full_bar(s), 1);
        mbar_init(full_w(s), 1);
        mbar_init(empty_bar(s), 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(tfull(b), 1);
        mbar_init(tempty(b), 4);
      }
      mbar_init(done_bar, 1);
      fence_mbar_init();
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmAsf);
      if (p.wprep || p.kfull > 0) tma_prefetch_desc(&tmB);
      if (!p.wprep && p.kfull < gp.K) tma_prefetch_desc(&tmBtail);
      tma_prefetch_desc(&tmBsf);
    }
  } else if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // All 512 columns are allocated, so the allocation starts at lane 0, column
  // 0; TMEM is addressed from that constant (warp-uniform operands).
  const uint32_t tmem_got = *tmem_slot;
  constexpr uint32_t tmem_base = 0;
  if (tmem_got != tmem_base && threadIdx.x == 0) record_status(gp.status, MOE_ERR_CUDA);
  const int total = tmem_got == tmem_base ? *total_s : 0;
  const int nst = p.nst;
  const int nfull = p.kfull / BKE;  // stages whose codes come from the weights; the last, if ragged, from the tail rows

  if (warp == 0 || warp == kWProducerWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------- producers
      // A thread that issues a TMA copy waits ~60 ns before it can issue the
      // next, whatever the copy's size, so a stage takes one copy per operand
      // (hi and lo planes in one 3-D box; gate and up halves in one box) and
      // two threads share them: warp 0 the activation side, warp 6 the weight
      // side, each completing its own full barrier.
      const bool wside = warp == kWProducerWarp;
      const uint32_t stage_tx =
          wside ? static_cast<uint32_t>(gp.mma_n) * (BKE / 2) + 1024 : 2 * kAOpBytes + 1024;
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool failed = false;
      for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
        int e, nt, mt;
        decode_tile(tile, tpre, seg, gp.E, BM, e, nt, mt);
        const int row0 = seg[e] + mt * BM;
        const int64_t g = mpre[e] + mt;
        const int brow = nt * gp.n_tile;  // the tile's first (gate) row within the expert
        const int64_t wsf_row = (static_cast<int64_t>(e) * gp.NT + nt) * nst;
        for (int q = 0; q < nst; ++q) {
          if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, kWaitNs)) {
            failed = true;
            break;
          }
          const uint32_t st = smem_u32(ring + s * sst);
          const uint32_t fb = wside ? full_w(s) : full_bar(s);
          mbar_arrive_expect_tx(fb, stage_tx);
          if (!wside) {
            tma_load_3d(st, &tmA, fb, q * BKE, row0, 0);                                  // hi, lo planes
            tma_load_2d(st + 2 * kAOpBytes, &tmAsf, fb, 0, static_cast<int32_t>(g * nst + q));  // their scales
          } else {
            if (p.wprep)
              tma_load_4d(st + kBOff, &tmB, fb, 0, brow, 0, e * nst + q);
            else if (q < nfull)
              tma_load_4d(st + kBOff, &tmB, fb, q * BKE, e * gp.b_rows + brow, 0, 0);
            else
              tma_load_4d(st + kBOff, &tmBtail, fb, 0, e * gp.b_rows + brow, 0, 0);
            tma_load_2d(st + sfb_off, &tmBsf, fb, 0, static_cast<int32_t>(wsf_row + q));
          }
          ++issued;
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (failed) {
        record_status(gp.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        const int n = issued < kStages ? issued : kStages;  // this thread's copies still in flight
        for (int i = 0; i < n; ++i) {
          if (--s < 0) {
            s = kStages - 1;
            ph ^= 1u;
          }
          mbar_wait_bounded(wside ? full_w(s) : full_bar(s), ph, nullptr, kWaitNs);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop and one elected lane issues each tcgen05
    // instruction, so every operand is warp-uniform.
    const uint32_t idesc = idesc_mx(0 /* E4M3 */, 5 /* E2M1 */, gp.mma_n);
    int s = 0, acc = 0, sfr = 0;
    uint32_t ph = 0, pacc = 0;
    bool failed = false;
    for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(tempty(acc), pacc ^ 1u, abort_flag, kWaitNs))) {
        failed = true;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * kAccStride;
      for (int q = 0; q < nst; ++q) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(full_bar(s), ph, abort_flag, kWaitNs) &&
                                         mbar_wait_bounded(full_w(s), ph, abort_flag, kWaitNs))) {
          failed = true;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(ring + s * sst);
        const uint32_t b = st + kBOff;
        const uint32_t tsf = tmem_base + (sfr ? kSfCol1 : kSfCol0);
        sfr ^= 1;
        tc_cp_sf_elect(tsf + 0, desc_noswizzle(st + 2 * kAOpBytes, 128));
        tc_cp_sf_elect(tsf + 4, desc_noswizzle(st + 2 * kAOpBytes + 512, 128));
        tc_cp_sf_elect(tsf + 8, desc_noswizzle(st + sfb_off, 128));
        if (gp.mma_n > 128) tc_cp_sf_elect(tsf + 12, desc_noswizzle(st + sfb_off + 512, 128));
        const int kleft = gp.K - q * BKE;
        const int nkb = kleft >= BKE ? 4 : kleft / 32;
        for (int kb = 0; kb < nkb; ++kb) {
          const uint64_t bd = desc_kmajor_sw128(b + kb * 32);
          mma_mx_elect(d_tmem, desc_kmajor_sw128(st + kb * 32), bd, idesc, kb, tsf + 0, tsf + 8,
                       (q | kb) != 0 ? 1u : 0u);
          mma_mx_elect(d_tmem, desc_kmajor_sw128(st + kAOpBytes + kb * 32), bd, idesc, kb, tsf + 4, tsf + 8, 1u);
        }
        tc_commit_elect(empty_bar(s));
        if (++s == kStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (failed) break;
      tc_commit_elect(tfull(acc));
      if (++acc == 2) {
        acc = 0;
        pacc ^= 1u;
      }
    }
    if (failed && lane == 0) {
      record_status(gp.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    tc_commit_elect(done_bar);
    mbar_wait_bounded(done_bar, 0, nullptr, kWaitNs);
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------ epilogue
    const int qd = warp & 3;  // TMEM lane quarter this warp may access
    const int m = qd * 32 + lane;
    int acc = 0;
    uint32_t pacc = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int e, nt, mt;
      decode_tile(tile, tpre, seg, gp.E, BM, e, nt, mt);
      const bool ok = mbar_wait_bounded(tfull(acc), pacc, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) {
          record_status(gp.status, MOE_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(seg[e]) + mt * BM + m;
      const bool valid = row < seg[e + 1];
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) + acc * kAccStride;
      if (kSwiGLU && p.hq != nullptr) {
        // bias + activation, h rounded to bf16, then straight into mlp2's
        // operand form: hi/lo E4M3 + scales (the quantiser's arithmetic)
        const uint16_t* bg = gp.bias + static_cast<int64_t>(e) * gp.b_rows + nt * gp.n_tile;
        const uint16_t* bu = bg + gp.n_out;
        const int64_t g = mpre[e] + mt;
        for (int c0 = 0; c0 < gp.n_tile; c0 += 32) {
          float v[32];
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {  // 16 columns at a time keeps the registers in check
            uint32_t ga[16], ua[16];
            tmem_ld_x8(tbase + c0 + 16 * hf, ga);
            tmem_ld_x8(tbase + c0 + 16 * hf + 8, ga + 8);
            tmem_ld_x8(tbase + gp.n_tile + c0 + 16 * hf, ua);
            tmem_ld_x8(tbase + gp.n_tile + c0 + 16 * hf + 8, ua + 8);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              float gb[8], ub[8];
              unpack8(__ldg(reinterpret_cast<const uint4*>(bg + c0 + 16 * hf + 8 * j)), gb);
              unpack8(__ldg(reinterpret_cast<const uint4*>(bu + c0 + 16 * hf + 8 * j)), ub);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float hv = glu_act(__uint_as_float(ga[8 * j + i]) + gb[i],
                                         __uint_as_float(ua[8 * j + i]) + ub[i], gp.act);
                v[16 * hf + 8 * j + i] = bf16_bits_to_float(float_to_bf16_bits(hv));
              }
            }
          }
          if (valid) {
            uint32_t hi[8], lo[8], sfh, sfl;
            quant32(v, hi, lo, sfh, sfl);
            const int col = nt * gp.n_tile + c0;
            st_global_v8u(p.hq + row * gp.n_out + col, hi);
            st_global_v8u(p.hq + gp.R * gp.n_out + row * gp.n_out + col, lo);
            store_act_sf(p.h_sf + (g * p.h_nst + col / BKE) * kSfBlock, m, (col % BKE) / 32, sfh, sfl);
          }
        }
      } else {
        epilogue_tile<kSwiGLU>(gp, tbase, e, nt, row, valid);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty(acc));
      if (++acc == 2) {
        acc = 0;
        pacc ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_got, kTmemCols);
  }
}

// ---------------------------------------------------------------- small-expert kernel
// Experts with at most kSmallRows routed rows (decode-sized batches): the
// weights are the MMA's M side, 128 weight rows per tile (mlp1: 64 gate rows
// over the 64 matching up rows; mlp2: 128 output rows), and the expert's rows
// its N side, hi rows over lo rows (N = 64), one MMA per 32-K block. Each tile
// streams its weight rows once through a deep ring of small stages: every
// weight byte crosses HBM once, at 4.25 bits per element.
//   warps 0, 9  weight-side producers (even / odd stages): the weight codes
//               (one TMA box, 16U4_ALIGN16B, both mlp1 halves) and the weight
//               rows' scale atom (TMA, from the preparation pass);
//   warps 6, 10 row-side producers (likewise): the expert's hi and lo rows
//               (one 3-D TMA box of 32 rows x 2 planes) and their 64-row scale
//               atom (TMA, from the activation scales);
//   warps 1,7,8 MMA: two scale copies into tensor memory and 4 block-scaled
//               MMAs per stage; warp i takes the stages q = i mod 3 into its
//               own accumulator. Each tcgen05 instruction holds its issuing
//               warp for ~50 ns (~0.4 us for a stage's seven), so the stages
//               are spread over three issuing warps;
//   warps 2..5  epilogue (lane = weight row): the issuers' hi + lo parts
//               added per row in a fixed order, then SwiGLU with the up half
//               from the other two warps via shared memory and h quantised
//               across the warp's 32 columns, or bias * gate weight into the
//               fp32 expert outputs.
// Nothing here writes shared memory for the tensor core but TMA, so no proxy
// fence sits on the pipeline.
constexpr int kSmallRows = 32;
constexpr int kSN = 2 * kSmallRows;                  // the expert's hi rows, then its lo rows
constexpr int kSIssuers = 3;
// Producers per side. Producer i fills the stages n with n mod kSProducers =
// i, and the ring depth is a multiple of kSProducers, so every ring slot is
// always filled by the same thread: a producer's parity wait on a slot's
// empty barrier is then never two phases behind (the slot's previous fill was
// its own, issued after the phase before completed). With slots rotating
// among producers one could run a ring ahead of another and pass a wait on
// the stale parity.
constexpr int kSProducers = 2;
// warps: 0, 6 producers; 1, 7, 8 issuers; 2..5 epilogue; 9.. the other producers
constexpr int kSThreads = 32 * (9 + 2 * (kSProducers - 1));
__device__ __forceinline__ int small_issuer_of(int warp) { return warp == 1 ? 0 : warp == 7 ? 1 : warp == 8 ? 2 : -1; }
// producer id: side * kSProducers + i (side 1: the row side), producer i
// taking the stages n with n mod kSProducers = i; -1 for other warps
static_assert(kSThreads / 32 == 9 + 2 * (kSProducers - 1), "every producer id has a warp");
__device__ __forceinline__ int small_producer_of(int warp) {
  if (warp == 0) return 0;
  if (warp == 6) return kSProducers;
  if (warp >= 9 && warp < 9 + 2 * (kSProducers - 1)) {
    const int j = warp - 9;
    return (j & 1) ? kSProducers + 1 + j / 2 : 1 + j / 2;
  }
  return -1;
}
constexpr uint32_t kSA = 128 * 128;                  // weight operand: 128 rows x 128 B
constexpr uint32_t kSB = kSN * 128;                  // row operand: 64 rows x 128 B
constexpr uint32_t kSStage = kSA + kSB + 1024;       // + weight scale atom, row scale atom (512 B each)
constexpr uint32_t kSAccStride = 64;                 // accumulator (issuer i, buffer b) at (2i + b) * 64
constexpr uint32_t kSSfBase = 384;                   // scale regions (issuer i, r) at 384 + (2i + r) * 8
static_assert(kSSfBase >= 2 * kSIssuers * kSAccStride && kSSfBase + 16 * kSIssuers <= 512, "TMEM columns");
constexpr int kSMaxStages = 8;
constexpr int kXStride = 33;                         // floats per row of the up-half exchange buffer

// Control block: 3 * stages + 9 mbarriers, then the TMEM slot, abort flag and
// tile total (16 bytes).
__host__ __device__ constexpr uint32_t small_ctrl_bytes(int stages) {
  return (8u * static_cast<uint32_t>(3 * stages + 9) + 16u + 15u) / 16u * 16u;
}

struct SmallParams {
  GemmParams g;           // E, K, n_out, b_rows, R, offsets, bias, perm, topk_w, out, status, act
  int nst, kfull;
  int NT2;                // weight tiles per expert
  int stages;             // ring depth
  int wprep;              // codes from the prepared copy (K-block-major), else from the weights as stored
  uint8_t* hq;
  uint8_t* h_sf;
  int h_nst;
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// quant32's arithmetic with the 32 values spread over the warp's lanes (lane
// i holds element i): this lane's hi and lo codes and the block's scales.
__device__ __forceinline__ void quant32_warp(float v, uint32_t& qh, uint32_t& ql, uint32_t& sfh, uint32_t& sfl) {
  const bool bad = __any_sync(0xffffffffu, v * 0.f != 0.f);
  const float amax = warp_max(fabsf(v));
  if (bad) {
    qh = ql = 0x7fu;
    sfh = sfl = 127;
    return;
  }
  if (!(amax >= 0x1p-119f)) {
    qh = ql = 0u;
    sfh = sfl = 127;
    return;
  }
  const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127;
  const float mul = __uint_as_float(static_cast<uint32_t>(127 + 7 - e) << 23);
  const float back = __uint_as_float(static_cast<uint32_t>(127 + e - 7) << 23);
  sfh = static_cast<uint32_t>(e + 120);
  qh = e4m3x2(v * mul, 0.f) & 0xffu;
  const float r = v - e4m3x2_value(qh).x * back;
  const float rmax = warp_max(fabsf(r));
  if (!(rmax >= 0x1p-119f)) {
    ql = 0u;
    sfl = 127;
    return;
  }
  const int er = static_cast<int>((__float_as_uint(rmax) >> 23) & 0xffu) - 127;
  const float mul2 = __uint_as_float(static_cast<uint32_t>(127 + 7 - er) << 23);
  sfl = static_cast<uint32_t>(er + 120);
  ql = e4m3x2(r * mul2, 0.f) & 0xffu;
}

template <bool kSwiGLU>
__global__ void __launch_bounds__(kSThreads, 1)
    mx_small_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmWtail,
                    const __grid_constant__ CUtensorMap tmWsf, const __grid_constant__ CUtensorMap tmX,
                    const __grid_constant__ CUtensorMap tmXsf, const SmallParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const GemmParams& gp = p.g;
  const int S = p.stages;
  uint8_t* ring = smem;
  float* xbuf = reinterpret_cast<float*>(ring + S * kSStage);  // 64 x kXStride
  uint8_t* ctrl = reinterpret_cast<uint8_t*>(xbuf + 64 * kXStride);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctrl);
  const int nbars = 3 * S + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * nbars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* total_s = reinterpret_cast<int*>(tmem_slot + 2);
  int* seg = reinterpret_cast<int*>(ctrl + small_ctrl_bytes(S));
  int* mpre = seg + (gp.E + 1);
  int* tpre = mpre + (gp.E + 1);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x / 32), 0), lane = threadIdx.x % 32;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };            // weight side landed
  auto full_x = [&](int s) { return bar0 + 8u * (S + s); };         // row side landed
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * S + s); };
  auto tfull = [&](int b) { return bar0 + 8u * (3 * S + b); };
  auto tempty = [&](int b) { return bar0 + 8u * (3 * S + 2 + b); };
  const uint32_t done_bar = bar0 + 8u * (3 * S + 4);
  const uint32_t xfull = bar0 + 8u * (3 * S + 5), xempty = bar0 + 8u * (3 * S + 6);  // up-half exchange

  if (warp == 0) {
    const bool ok = load_segments(gp.offsets, gp.E, gp.R, seg, mpre, gp.status);
    const int NT2 = p.NT2;
    schedule_prefix(seg, gp.E, tpre, [NT2](int cnt) { return (cnt >= 1 && cnt <= kSmallRows) ? NT2 : 0; });
    if (lane == 0) {
      *abort_flag = 0;
      *total_s = ok ? tpre[gp.E] : 0;
    }
  }
  __syncthreads();
  // A CTA without a tile (on large batches no expert may have 1..32 rows)
  // leaves before it allocates tensor memory.
  if (static_cast<int>(blockIdx.x) >= *total_s) return;
  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < S; ++s) {
        mbar_init(full_bar(s), 1);
        mbar_init(full_x(s), 1);
        mbar_init(empty_bar(s), 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(tfull(b), kSIssuers);
        mbar_init(tempty(b), 4);
      }
      mbar_init(done_bar, kSIssuers);
      mbar_init(xfull, 2);
      mbar_init(xempty, 2);
      fence_mbar_init();
      if (p.wprep || p.kfull > 0) tma_prefetch_desc(&tmW);
      if (!p.wprep && p.kfull < gp.K) tma_prefetch_desc(&tmWtail);
      tma_prefetch_desc(&tmWsf);
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmXsf);
    }
  } else if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_got = *tmem_slot;
  constexpr uint32_t tmem_base = 0;
  if (tmem_got != tmem_base && threadIdx.x == 0) record_status(gp.status, MOE_ERR_CUDA);
  const int total = tmem_got == tmem_base ? *total_s : 0;
  const int nst = p.nst, nfull = p.kfull / BKE;
  // tile -> (expert, weight tile)
  auto decode = [&](int tile, int& e, int& wt) {
    int lo = 0, hi = gp.E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tpre[mid] <= tile)
        lo = mid;
      else
        hi = mid - 1;
    }
    e = lo;
    wt = tile - tpre[e];
  };

  if (small_producer_of(warp) >= 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producers
      // One TMA copy per operand per stage; a thread waits ~60 ns after each
      // copy it issues, so each side is split over kSProducers threads taking
      // the stages in turn (each always the same ring slots: S is a multiple
      // of kSProducers).
      const int pid = small_producer_of(warp);
      const bool xside = pid >= kSProducers;
      const int par = pid % kSProducers;
      const uint32_t stage_tx = xside ? kSB + 512 : 128 * (BKE / 2) + 512;
      int s = 0, n = 0;
      uint32_t ph = 0;
      bool failed = false;
      for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
        int e, wt;
        decode(tile, e, wt);
        const int row0 = seg[e];
        const int64_t g = mpre[e];
        const int wrow = kSwiGLU ? wt * 64 : wt * 128;  // the tile's first (gate) row within the expert
        const int64_t wsf_row = (static_cast<int64_t>(e) * p.NT2 + wt) * nst;
        for (int q = 0; q < nst; ++q) {
          if (n % kSProducers == par) {
            if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, kWaitNs)) {
              failed = true;
              break;
            }
            const uint32_t st = smem_u32(ring + s * kSStage);
            const uint32_t fb = xside ? full_x(s) : full_bar(s);
            mbar_arrive_expect_tx(fb, stage_tx);
            if (xside) {
              tma_load_3d(st + kSA, &tmX, fb, q * BKE, row0, 0);  // hi rows over lo rows
              tma_load_2d(st + kSA + kSB + 512, &tmXsf, fb, 0, static_cast<int32_t>(g * nst + q));
            } else {
              if (p.wprep)
                tma_load_4d(st, &tmW, fb, 0, wrow, 0, e * nst + q);
              else if (q < nfull)
                tma_load_4d(st, &tmW, fb, q * BKE, e * gp.b_rows + wrow, 0, 0);
              else
                tma_load_4d(st, &tmWtail, fb, 0, e * gp.b_rows + wrow, 0, 0);
              tma_load_2d(st + kSA + kSB, &tmWsf, fb, 0, static_cast<int32_t>(wsf_row + q));
            }
          }
          ++n;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (failed) {
        record_status(gp.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        // this thread's copies still in flight: its stages among the last S
        for (int i = 1; i <= S && i <= n; ++i) {
          if (--s < 0) {
            s = S - 1;
            ph ^= 1u;
          }
          if ((n - i) % kSProducers == par) mbar_wait_bounded(xside ? full_x(s) : full_bar(s), ph, nullptr, kWaitNs);
        }
      }
    }
  } else if (small_issuer_of(warp) >= 0) {
    // ------------------------------------------------------------ MMA issuers (whole warp, one lane elected)
    // Issuer i takes the stages q = i, i + 3, ... of every tile; all track
    // the ring position of every stage.
    const int iss = small_issuer_of(warp);
    const uint32_t idesc = idesc_mx(5 /* E2M1 weights */, 0 /* E4M3 rows */, kSN);
    int s = 0, acc = 0, sfr = 0;
    uint32_t ph = 0, pacc = 0;
    bool failed = false;
    for (int tile = blockIdx.x; tile < total && !failed; tile += gridDim.x) {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(tempty(acc), pacc ^ 1u, abort_flag, kWaitNs))) {
        failed = true;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (2 * iss + acc) * kSAccStride;
      for (int q = 0; q < nst; ++q) {
        if (q % kSIssuers == iss) {
          // The slot's previous stage may have been another issuer's: wait
          // for it to be consumed first, so that the parity waits on the full
          // barriers cannot match that older phase.
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, kWaitNs) &&
                                           mbar_wait_bounded(full_bar(s), ph, abort_flag, kWaitNs) &&
                                           mbar_wait_bounded(full_x(s), ph, abort_flag, kWaitNs))) {
            failed = true;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(ring + s * kSStage);
          const uint32_t tsf = tmem_base + kSSfBase + (2 * iss + sfr) * 8;
          sfr ^= 1;
          // (each copy fills 4 columns and must start on a multiple of 4)
          tc_cp_sf_elect(tsf + 0, desc_noswizzle(st + kSA + kSB, 128));        // weight rows' scales
          tc_cp_sf_elect(tsf + 4, desc_noswizzle(st + kSA + kSB + 512, 128));  // the 64 operand rows' scales
          const int kleft = gp.K - q * BKE;
          const int nkb = kleft >= BKE ? 4 : kleft / 32;
          for (int kb = 0; kb < nkb; ++kb)
            mma_mx_elect(d_tmem, desc_kmajor_sw128(st + kb * 32), desc_kmajor_sw128(st + kSA + kb * 32), idesc, kb,
                         tsf + 0, tsf + 4, (q != iss || kb != 0) ? 1u : 0u);
          tc_commit_elect(empty_bar(s));
        }
        if (++s == S) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (failed) break;
      tc_commit_elect(tfull(acc));  // an issuer with no stage in the tile (short K) arrives at once
      if (++acc == 2) {
        acc = 0;
        pacc ^= 1u;
      }
    }
    if (failed && lane == 0) {
      record_status(gp.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    tc_commit_elect(done_bar);
    mbar_wait_bounded(done_bar, 0, nullptr, kWaitNs);
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------ epilogue (lane = weight row)
    const int qd = warp & 3;  // TMEM lane quarter
    const int m = qd * 32 + lane;
    int acc = 0, ti = 0;
    uint32_t pacc = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int e, wt;
      decode(tile, e, wt);
      const int row0 = seg[e], cnt = seg[e + 1] - seg[e];
      const bool ok = mbar_wait_bounded(tfull(acc), pacc, abort_flag, kWaitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) {
          record_status(gp.status, MOE_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) + acc * kSAccStride;
      // row t's value: issuer 0's (hi + lo) part, then those of the issuers
      // that had stages in this tile (issuer i when nst > i), added in that order
      float v[kSmallRows];
      {
        uint32_t hv[32], lv[32];
        tmem_ld_x32(tb, hv);
        tmem_ld_x32(tb + kSmallRows, lv);
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < kSmallRows; ++t) v[t] = __uint_as_float(hv[t]) + __uint_as_float(lv[t]);
        for (int i = 1; i < kSIssuers && i < nst; ++i) {
          tmem_ld_x32(tb + 2 * i * kSAccStride, hv);
          tmem_ld_x32(tb + 2 * i * kSAccStride + kSmallRows, lv);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < kSmallRows; ++t) v[t] += __uint_as_float(hv[t]) + __uint_as_float(lv[t]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty(acc));  // the accumulator is in registers now
      if (++acc == 2) {
        acc = 0;
        pacc ^= 1u;
      }
      if (kSwiGLU) {
        // lanes 64..127 hold the up half: hand it to the gate warps through
        // shared memory (bounded waits on two mbarriers, one phase per tile)
        bool xok = true;
        if (qd >= 2) {
          xok = __all_sync(0xffffffffu, mbar_wait_bounded(xempty, (ti & 1) ^ 1u, abort_flag, kWaitNs));
          if (xok) {
#pragma unroll
            for (int t = 0; t < kSmallRows; ++t) xbuf[(m - 64) * kXStride + t] = v[t];
            __syncwarp();
            if (lane == 0) mbar_arrive(xfull);
          }
        } else {
          xok = __all_sync(0xffffffffu, mbar_wait_bounded(xfull, ti & 1, abort_flag, kWaitNs));
          if (xok) {
            const int col = wt * 64 + m;  // h column
            const float bg = bf16_bits_to_float(gp.bias[static_cast<int64_t>(e) * gp.b_rows + col]);
            const float bu = bf16_bits_to_float(gp.bias[static_cast<int64_t>(e) * gp.b_rows + gp.n_out + col]);
            const int64_t g = mpre[e];
            const int col0 = wt * 64 + qd * 32;  // the warp's 32-column scale block
            float u[kSmallRows];
#pragma unroll
            for (int t = 0; t < kSmallRows; ++t) u[t] = xbuf[m * kXStride + t];
            __syncwarp();
            if (lane == 0) mbar_arrive(xempty);
#pragma unroll
            for (int t = 0; t < kSmallRows; ++t) {
              if (t >= cnt) break;  // warp-uniform
              const float hb = bf16_bits_to_float(float_to_bf16_bits(glu_act(v[t] + bg, u[t] + bu, gp.act)));
              const int64_t r = row0 + t;
              if (p.hq != nullptr) {
                uint32_t qh, ql, sfh, sfl;
                quant32_warp(hb, qh, ql, sfh, sfl);
                p.hq[r * gp.n_out + col] = static_cast<uint8_t>(qh);
                p.hq[gp.R * gp.n_out + r * gp.n_out + col] = static_cast<uint8_t>(ql);
                if (lane == 0)
                  store_act_sf(p.h_sf + (g * p.h_nst + col0 / BKE) * kSfBlock, t, (col0 % BKE) / 32, sfh, sfl);
              } else {
                static_cast<uint16_t*>(gp.out)[r * gp.n_out + col] = float_to_bf16_bits(hb);
              }
            }
          }
        }
        if (!xok) {
          if (lane == 0) {
            record_status(gp.status, MOE_ERR_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
        ++ti;
      } else {
        const int col = wt * 128 + m;  // output column
        if (col < gp.n_out) {
          const float bb = bf16_bits_to_float(gp.bias[static_cast<int64_t>(e) * gp.b_rows + col]);
#pragma unroll
          for (int t = 0; t < kSmallRows; ++t) {
            if (t >= cnt) break;
            const int64_t r = row0 + t;
            const int32_t a = gp.perm[r];
            float wgt = 0.f;
            if (a >= 0 && a < gp.R)
              wgt = gp.topk_w[a];
            else
              record_status(gp.status, MOE_ERR_DEVICE_BOUNDS);
            static_cast<float*>(gp.out)[r * gp.n_out + col] = wgt * (v[t] + bb);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_got, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
// Tensor maps (cuTensorMapEncodeTiled through the runtime's driver entry
// point); a false return becomes MOE_ERR_CUDA.

// The hi and lo E4M3 planes, (R, K) bytes each with lo right after hi, as one
// 3-D tensor (K, R, 2) loaded in 128-byte x box_rows x 2 boxes with the
// 128-byte swizzle: a stage's hi rows, then its lo rows, in shared memory.
bool make_tmap_act(CUtensorMap* map, const uint8_t* hi, uint64_t K, uint64_t R, uint32_t box_rows) {
  auto fn = tma_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {K, R, 2};
  cuuint64_t strides[2] = {K, R * K};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(BKE), box_rows, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(hi), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E2M1 codes as a 4-D tensor (elements, rows, halves, K blocks): `inner`
// elements per row (a multiple of 128), rows `row_bytes` apart, `halves` (2:
// mlp1's gate rows and the matching up rows) `half_bytes` apart, `kblocks`
// blocks `kblock_bytes` apart. Loaded as 128-element x box_rows x halves x 1
// boxes, unpacked by TMA into the MMA's E2M1 operand layout (every 8 bytes of
// codes padded to 16) with the 128-byte swizzle: the gate rows, then the up
// rows, in shared memory. Base 32-byte aligned, strides multiples of 32.
//  - weights as stored: (K rounded down to 128, E * N, halves, 1), rows K/2 bytes apart;
//  - their tail rows: (128, E * N, halves, 1), rows 64 bytes apart;
//  - the prepared copy: (128, rows per half, halves, E * nst), rows 64 bytes apart.
bool make_tmap_codes(CUtensorMap* map, const uint8_t* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                     uint32_t halves, uint64_t half_bytes, uint64_t kblocks, uint64_t kblock_bytes,
                     uint32_t box_rows) {
  auto fn = tma_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {inner, rows, halves, kblocks};
  cuuint64_t strides[3] = {row_bytes, half_bytes, kblock_bytes};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(BKE), box_rows, halves, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 4, const_cast<uint8_t*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// `count` scale atoms of atom_bytes (512 or 1024) bytes, `stride` bytes
// apart, one atom per load, copied as is.
bool make_tmap_atoms(CUtensorMap* map, const uint8_t* base, uint32_t atom_bytes, uint64_t count, uint64_t stride) {
  auto fn = tma_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {atom_bytes / 4u, count};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {atom_bytes / 4u, 1};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t smem_bytes(int mma_n, int E) {
  return 1024 + static_cast<size_t>(kStages) * stage_bytes(mma_n) + kCtrlBytes +
         3 * static_cast<size_t>(E + 1) * sizeof(int);
}

int pick_tile(int n, int max_tile, int step) {
  for (int t = max_tile; t >= step; t -= step)
    if (n % t == 0) return t;
  return 0;
}

// Tile sizes of the two GEMMs: mlp1 h columns per tile a multiple of 32
// (whole scale blocks of mlp2's K), gate and up halves stacked in one MMA of
// N = 2 * n_tile <= 240; mlp2 N = n_tile <= 240.
int mlp1_ntile(const moe_dims_t& d) { return pick_tile(d.I, kMaxN / 2 / 32 * 32, 32); }
int mlp2_ntile(const moe_dims_t& d) { return pick_tile(d.D, kMaxN, 16); }


size_t small_smem_bytes(int stages, int E) {
  return 1024 + static_cast<size_t>(stages) * kSStage + 64 * kXStride * sizeof(float) + small_ctrl_bytes(stages) +
         3 * static_cast<size_t>(E + 1) * sizeof(int);
}

// The preparation region of one GEMM: big-tile atoms, small-tile atoms, then
// either (per call) the tail rows or (prepare-once form) the K-block-major codes.
struct PrepLayout {
  size_t big, small, rest, tail, codes;
  size_t per_call() const { return rest + tail; }
  size_t prepared() const { return rest + codes; }
};
PrepLayout prep_layout(int E, int b_rows, int K, int NT, int NT2) {
  PrepLayout L{};
  const int nst = (K + BKE - 1) / BKE;
  L.big = 0;
  L.small = align_up(static_cast<size_t>(E) * NT * nst * 1024, 256);
  L.rest = L.small + align_up(static_cast<size_t>(E) * NT2 * nst * 512, 256);
  L.tail = K % BKE ? align_up(static_cast<size_t>(E) * b_rows * 64, 256) : 0;
  L.codes = align_up(static_cast<size_t>(E) * nst * b_rows * 64, 256);
  return L;
}

// The small-expert kernel's geometry for a GEMM: weight tiles per expert,
// ring depth, and whether it runs at all (else every expert takes big tiles).
struct SmallGeom {
  int NT2, stages;
  bool ok;
};
template <bool kSwiGLU>
SmallGeom small_geom(const GemmParams& g) {
  SmallGeom sg{};
  sg.NT2 = kSwiGLU ? g.n_out / 64 : (g.n_out + 127) / 128;
  // (a multiple of kSProducers: each ring slot keeps one producer)
  sg.stages = kSMaxStages / kSProducers * kSProducers;
  while (sg.stages >= kSProducers && small_smem_bytes(sg.stages, g.E) > 227 * 1024) sg.stages -= kSProducers;
  sg.ok = sg.stages >= 3 && sg.stages % kSProducers == 0 && (!kSwiGLU || g.n_out % 64 == 0);
  return sg;
}

// The preparation pass into `out` for the given routing (offsets) or, with
// all_experts, for every expert (the prepare-once form).
template <bool kSwiGLU>
moe_status_t run_prep(const MxParams& p, const uint8_t* codes, const uint8_t* scales, uint8_t* out, bool all_experts,
                      cudaStream_t s) {
  const GemmParams& g = p.g;
  const SmallGeom sg = small_geom<kSwiGLU>(g);
  const PrepLayout L = prep_layout(g.E, g.b_rows, g.K, g.NT, sg.NT2);
  uint8_t* tail = (!all_experts && g.K % BKE) ? out + L.rest : nullptr;
  uint8_t* codes_out = all_experts ? out + L.rest : nullptr;
  PrepArgs pa{codes, scales, g.E, g.b_rows, g.K, g.n_out, g.n_tile, g.mma_n, g.NT, sg.NT2, p.nst, kSwiGLU ? 1 : 0,
              g.offsets, sg.ok ? kSmallRows : 0, all_experts ? 1 : 0, out + L.big, out + L.small, tail, codes_out};
  const int64_t blocks = static_cast<int64_t>(g.E) * g.NT + (sg.ok ? static_cast<int64_t>(g.E) * sg.NT2 : 0) +
                         (tail ? static_cast<int64_t>(g.E) * ((g.b_rows + 255) / 256) : 0) +
                         (codes_out ? static_cast<int64_t>(g.E) * p.nst * ((g.b_rows + 63) / 64) : 0);
  if (blocks > 0x7fffffff) return MOE_ERR_UNSUPPORTED;
  mx_prep_weights_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(pa);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <bool kSwiGLU>
PrepLayout layout_of(const MxParams& p) {
  return prep_layout(p.g.E, p.g.b_rows, p.g.K, p.g.NT, small_geom<kSwiGLU>(p.g).NT2);
}

// One grouped GEMM with MXFP4 weights: the preparation pass (unless `prep`
// already holds the prepare-once form), then the small-expert kernel (experts
// with 1..kSmallRows rows) and the big-tile kernel (the others), each
// skipping the other's experts.
template <bool kSwiGLU>
moe_status_t launch_mx_gemm(const uint8_t* aq, const uint8_t* codes, const uint8_t* scales, uint8_t* prep,
                            bool prepared, MxParams p, cudaStream_t s) {
  const GemmParams& g = p.g;
  p.kfull = g.K / BKE * BKE;
  p.wprep = prepared ? 1 : 0;
  const SmallGeom sg = small_geom<kSwiGLU>(g);
  const PrepLayout L = prep_layout(g.E, g.b_rows, g.K, g.NT, sg.NT2);
  if (!prepared) {
    const moe_status_t st = run_prep<kSwiGLU>(p, codes, scales, prep, false, s);
    if (st != MOE_OK) return st;
  }
  const int nst = p.nst;
  const uint64_t wrows = static_cast<uint64_t>(g.E) * g.b_rows;
  const uint64_t row_bytes = static_cast<uint64_t>(g.K) / 2;
  const uint32_t halves = kSwiGLU ? 2 : 1;
  const uint64_t m_tiles = static_cast<uint64_t>((g.R + BM - 1) / BM + g.E);  // what the activation scales hold
  // the weight codes (and, per call with a ragged K, the tail rows) in boxes of box_rows rows per half
  auto codes_maps = [&](CUtensorMap* m, CUtensorMap* t, uint32_t box_rows) -> bool {
    memset(m, 0, sizeof(*m));
    memset(t, 0, sizeof(*t));
    if (prepared)
      return make_tmap_codes(m, prep + L.rest, BKE, g.n_out, 64, halves, static_cast<uint64_t>(g.n_out) * 64,
                             static_cast<uint64_t>(g.E) * nst, static_cast<uint64_t>(g.b_rows) * 64, box_rows);
    if (p.kfull > 0 && !make_tmap_codes(m, codes, p.kfull, wrows, row_bytes, halves, g.n_out * row_bytes, 1,
                                        wrows * row_bytes, box_rows))
      return false;
    if (p.kfull < g.K && !make_tmap_codes(t, prep + L.rest, BKE, wrows, 64, halves, static_cast<uint64_t>(g.n_out) * 64,
                                          1, wrows * 64, box_rows))
      return false;
    return true;
  };

  if (sg.ok) {
    SmallParams sp{};
    sp.g = g;
    sp.nst = nst;
    sp.kfull = p.kfull;
    sp.NT2 = sg.NT2;
    sp.stages = sg.stages;
    sp.wprep = p.wprep;
    sp.hq = p.hq;
    sp.h_sf = p.h_sf;
    sp.h_nst = p.h_nst;
    CUtensorMap tw, twt, twsf, tx, txsf;
    if (!codes_maps(&tw, &twt, kSwiGLU ? 64 : 128) ||
        !make_tmap_atoms(&twsf, prep + L.small, 512, static_cast<uint64_t>(g.E) * sg.NT2 * nst, 512) ||
        !make_tmap_act(&tx, aq, g.K, g.R, kSmallRows) ||
        !make_tmap_atoms(&txsf, p.a_sf + 1024, 512, m_tiles * nst, kSfBlock))
      return MOE_ERR_CUDA;
    const size_t smem = small_smem_bytes(sp.stages, g.E);
    if (cudaFuncSetAttribute(mx_small_kernel<kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return MOE_ERR_CUDA;
    const int64_t max_tiles = static_cast<int64_t>(g.E) * sp.NT2;
    const int grid = static_cast<int>(max_tiles < num_sms() ? max_tiles : num_sms());
    mx_small_kernel<kSwiGLU><<<grid, kSThreads, smem, s>>>(tw, twt, twsf, tx, txsf, sp);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  p.small_max = sg.ok ? kSmallRows : 0;

  CUtensorMap ta, tasf, tb, tt, tbsf;
  if (!make_tmap_act(&ta, aq, g.K, g.R, BM) || !make_tmap_atoms(&tasf, p.a_sf, 1024, m_tiles * nst, kSfBlock) ||
      !codes_maps(&tb, &tt, static_cast<uint32_t>(kSwiGLU ? g.n_tile : g.mma_n)) ||
      !make_tmap_atoms(&tbsf, prep + L.big, 1024, static_cast<uint64_t>(g.E) * g.NT * nst, 1024))
    return MOE_ERR_CUDA;
  const size_t smem = smem_bytes(g.mma_n, g.E);
  if (smem > 227 * 1024) return MOE_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(mx_gemm_kernel<kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int64_t max_tiles = ((g.R + BM - 1) / BM + g.E) * static_cast<int64_t>(g.NT);
  const int grid = static_cast<int>(max_tiles < num_sms() ? max_tiles : num_sms());
  mx_gemm_kernel<kSwiGLU><<<grid, kThreads, smem, s>>>(ta, tasf, tb, tt, tbsf, p);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

size_t mx_sf_bytes(const moe_dims_t& d, int K) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  return static_cast<size_t>((R + BM - 1) / BM + d.E) * ((K + BKE - 1) / BKE) * kSfBlock;
}

moe_status_t launch_mx_quant(const moe_dims_t& d, const uint16_t* src, const int32_t* perm, int K,
                             const int32_t* offsets, uint8_t* dst, uint8_t* sf, int* status, cudaStream_t s) {
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  const int64_t total = R * (K / 32);
  const int64_t blocks = (total + 255) / 256;
  const int grid = static_cast<int>(blocks < 8 * num_sms() ? blocks : 8 * num_sms());
  mx_quant_kernel<<<grid, 256, 0, s>>>(src, perm, d.k, R, K, offsets, d.E, (K + BKE - 1) / BKE, dst, sf, status);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

MxParams mlp1_params(const moe_dims_t& d) {
  MxParams p{};
  GemmParams& g = p.g;
  g.E = d.E;
  g.K = d.D;
  g.n_out = d.I;
  g.n_tile = mlp1_ntile(d);
  g.mma_n = 2 * g.n_tile;
  g.NT = g.n_tile ? d.I / g.n_tile : 0;
  g.b_rows = 2 * d.I;
  g.R = static_cast<int64_t>(d.T) * d.k;
  g.act = act_of(d);
  p.nst = (d.D + BKE - 1) / BKE;
  p.h_nst = (d.I + BKE - 1) / BKE;
  return p;
}

MxParams mlp2_params(const moe_dims_t& d) {
  MxParams p{};
  GemmParams& g = p.g;
  g.E = d.E;
  g.K = d.I;
  g.n_out = d.D;
  g.n_tile = mlp2_ntile(d);
  g.mma_n = g.n_tile;
  g.NT = g.n_tile ? d.D / g.n_tile : 0;
  g.b_rows = d.D;
  g.R = static_cast<int64_t>(d.T) * d.k;
  p.nst = (d.I + BKE - 1) / BKE;
  return p;
}

moe_status_t launch_mlp1_mx(const moe_dims_t& d, const uint8_t* xq, const uint8_t* x_sf, const int32_t* offsets,
                            const uint8_t* codes, const uint8_t* scales, const uint8_t* prepared, const uint16_t* b1,
                            uint16_t* h, uint8_t* hq, uint8_t* h_sf, uint8_t* prep, int* status, cudaStream_t s) {
  MxParams p = mlp1_params(d);
  if (p.g.n_tile == 0) return MOE_ERR_UNSUPPORTED;
  p.g.offsets = offsets;
  p.g.bias = b1;
  p.g.out = h;
  p.g.status = status;
  p.a_sf = x_sf;
  p.hq = hq;
  p.h_sf = h_sf;
  return launch_mx_gemm<true>(xq, codes, scales, prepared ? const_cast<uint8_t*>(prepared) : prep, prepared != nullptr,
                              p, s);
}

moe_status_t launch_mlp2_mx(const moe_dims_t& d, const uint8_t* hq, const uint8_t* h_sf, const int32_t* perm,
                            const int32_t* offsets, const float* topk_w, const uint8_t* codes, const uint8_t* scales,
                            const uint8_t* prepared, const uint16_t* b2, float* o_perm, uint8_t* prep, int* status,
                            cudaStream_t s) {
  MxParams p = mlp2_params(d);
  if (p.g.n_tile == 0) return MOE_ERR_UNSUPPORTED;
  p.g.offsets = offsets;
  p.g.bias = b2;
  p.g.perm = perm;
  p.g.topk_w = topk_w;
  p.g.out = o_perm;
  p.g.status = status;
  p.a_sf = h_sf;
  return launch_mx_gemm<false>(hq, codes, scales, prepared ? const_cast<uint8_t*>(prepared) : prep, prepared != nullptr,
                               p, s);
}

size_t mx_prepared_bytes(const moe_dims_t& d, int which) {
  if (which == 1) {
    const MxParams p = mlp1_params(d);
    return p.g.n_tile ? layout_of<true>(p).prepared() : 0;
  }
  if (which == 2) {
    const MxParams p = mlp2_params(d);
    return p.g.n_tile ? layout_of<false>(p).prepared() : 0;
  }
  return 0;
}

size_t mx_prep_bytes(const moe_dims_t& d) {
  const MxParams p1 = mlp1_params(d), p2 = mlp2_params(d);
  if (p1.g.n_tile == 0 || p2.g.n_tile == 0) return 0;
  const size_t b1 = layout_of<true>(p1).per_call(), b2 = layout_of<false>(p2).per_call();
  return align_up(b1 > b2 ? b1 : b2, 256);
}

moe_status_t mx_prepare(const moe_dims_t& d, int which, const uint8_t* codes, const uint8_t* scales, uint8_t* out,
                        cudaStream_t s) {
  if (which == 1) return run_prep<true>(mlp1_params(d), codes, scales, out, true, s);
  return run_prep<false>(mlp2_params(d), codes, scales, out, true, s);
}

}  // namespace moe
