// MXFP4 expert weights expanded to bf16.
//
// The GPT-OSS in Transformers blog (MXFP4 paragraph) stores expert weights as
// 4-bit floats laid out E2M1 (1 sign, 2 exponent, 1 mantissa bit) with one
// shared scale per 32-element block. Read here as: exponent bias 1, exponent
// field 0 subnormal (0.m), scale an E8M0 power of two 2^(s-127); codes packed
// two per byte along the reduction dim, even element in the low nibble.
// Every E2M1 value times a power of two in the normal range is exact in bf16,
// so this expansion loses nothing and the bf16 tensor-core GEMMs then compute
// the MXFP4 layer exactly as they compute the bf16 one.
#include "common.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float e2m1_magnitude(uint32_t c) {
  const uint32_t ex = (c >> 1) & 3u, m = c & 1u;
  // exponent 0: 0.m ; exponent 1..3: 2^(ex-1) * 1.m
  return ex == 0 ? 0.5f * static_cast<float>(m) : __uint_as_float((126u + ex) << 23) * (1.0f + 0.5f * m);
}

__device__ __forceinline__ float e8m0_value(uint32_t s) {
  if (s == 255u) return __uint_as_float(0x7fc00000u);
  if (s == 0u) return __uint_as_float(0x00400000u);  // 2^-127
  return __uint_as_float(s << 23);
}

// One thread expands 16 consecutive elements (8 code bytes, one scale) into
// one 32-byte store.
__global__ void dequant_mxfp4_kernel(const uint2* __restrict__ codes, const uint8_t* __restrict__ scales,
                                     uint16_t* __restrict__ out, int64_t n16) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint2 w2 = __ldg(codes + i);
    const float sc = e8m0_value(__ldg(scales + (i >> 1)));  // 16 elements per thread, 32 per scale
    uint32_t packed[8];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t w = h ? w2.y : w2.x;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t c0 = (w >> (8 * q)) & 0xfu, c1 = (w >> (8 * q + 4)) & 0xfu;
        const float m0 = e2m1_magnitude(c0) * sc, m1 = e2m1_magnitude(c1) * sc;
        packed[4 * h + q] = pack_bf16x2((c0 & 8u) ? -m0 : m0, (c1 & 8u) ? -m1 : m1);
      }
    }
    sm100::st_global_v8u(out + 16 * i, packed);
  }
}

}  // namespace

cudaError_t launch_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales, int64_t E, int64_t N, int64_t K,
                                 uint16_t* out, cudaStream_t s) {
  const int64_t n16 = E * N * K / 16;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int threads = 256;
  int64_t blocks = (n16 + threads - 1) / threads;
  if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
  if (blocks < 1) blocks = 1;
  dequant_mxfp4_kernel<<<static_cast<int>(blocks), threads, 0, s>>>(reinterpret_cast<const uint2*>(codes), scales,
                                                                     out, n16);
  return cudaGetLastError();
}

}  // namespace moe
