// Shared device/host helpers of the MoE layer's CUDA path.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Workspace header: the device status word lives at byte 0 of ws.
constexpr size_t kWsHeader = 256;

__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(float_to_bf16_bits(lo)) | (static_cast<uint32_t>(float_to_bf16_bits(hi)) << 16);
}

// Launch helpers shared by the host side of every .cu file.
struct Launch {
  cudaStream_t stream;
  int* status;  // device status word (may be null for kernels that never record)
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Permutation: assignments per histogram/scatter block (a multiple of the
// block size), and the larger chunk of the workspace-free variant (its fixed
// histogram array bounds ceil(T*k / chunk) * E).
constexpr int kPermChunk = 512;
constexpr int kPermChunkNoAlloc = 2048;
constexpr int kPermThreads = 256;

inline int perm_blocks(int64_t R, int chunk = kPermChunk) { return static_cast<int>((R + chunk - 1) / chunk); }

// The activation between mlp1 and mlp2 on gate g and up u (moe_act_t in
// moe.h): plain SwiGLU silu(g) * u, or the GPT-OSS variant with the gate
// clamped from above at `limit`, sigmoid(alpha * gate), up clipped to
// [-limit, limit] plus 1.
struct Act {
  int kind;
  float alpha, limit;
};

__device__ __forceinline__ float glu_act(float g, float u, const Act& a) {
  if (a.kind == MOE_ACT_SWIGLU) return __fdividef(g, 1.0f + __expf(-g)) * u;
  const float gc = fminf(g, a.limit);
  const float uc = fminf(fmaxf(u, -a.limit), a.limit);
  return __fdividef(gc, 1.0f + __expf(-a.alpha * gc)) * (uc + 1.0f);
}

inline Act act_of(const moe_dims_t& d) { return Act{d.act, d.act_alpha, d.act_limit}; }

// Kernel launchers (defined in the .cu files).
// Router (route.cu). With route_splits(d) > 1 the contraction is split along
// K and `partial` holds route_splits(d) * T * n_pad fp32 (n_pad = E rounded
// up to 16).
int route_splits(const moe_dims_t& d);
cudaError_t launch_route(const moe_dims_t& d, const uint16_t* x, const uint16_t* Wr, const uint16_t* br,
                         int32_t* topk_idx, float* topk_w, float* partial, int* status, cudaStream_t s);
cudaError_t launch_permute(const moe_dims_t& d, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                           int32_t* perm, int32_t* inv, int32_t* block_counts, int* status, cudaStream_t s,
                           int chunk = kPermChunk);
cudaError_t launch_gather(const moe_dims_t& d, const uint16_t* x, const int32_t* perm, uint16_t* x_perm,
                          int* status, cudaStream_t s);
cudaError_t launch_combine(const moe_dims_t& d, const float* o_perm, const int32_t* inv, uint16_t* y,
                           int* status, cudaStream_t s);

// Grouped GEMMs (grouped_gemm.cu). Return MOE_OK or an error code.
moe_status_t launch_mlp1(const moe_dims_t& d, const uint16_t* x_perm, const int32_t* offsets,
                         const uint16_t* W1, const uint16_t* b1, uint16_t* h, int* status, cudaStream_t s);
moe_status_t launch_mlp2(const moe_dims_t& d, const uint16_t* h, const int32_t* perm, const int32_t* offsets,
                         const float* topk_w, const uint16_t* W2, const uint16_t* b2, float* o_perm,
                         int* status, cudaStream_t s);

// The same GEMMs on SM pairs, 256-row tiles (grouped_gemm_pair.cu).
moe_status_t launch_mlp1_pair(const moe_dims_t& d, const uint16_t* x_perm, const int32_t* offsets,
                              const uint16_t* W1, const uint16_t* b1, uint16_t* h, int* status, cudaStream_t s);
moe_status_t launch_mlp2_pair(const moe_dims_t& d, const uint16_t* h, const int32_t* perm, const int32_t* offsets,
                              const float* topk_w, const uint16_t* W2, const uint16_t* b2, float* o_perm,
                              int* status, cudaStream_t s);

// MXFP4 expert weights on block-scaled tcgen05 MMA (mx_gemm.cu). The
// activations (routed rows, h) are quantised to hi/lo E4M3 pairs with E8M0
// scales per 32 elements; the scales are stored tile-blocked, mx_sf_bytes
// bytes for a reduction length K.
size_t mx_sf_bytes(const moe_dims_t& d, int K);
// Workspace each MX GEMM needs for its weights' per-stage scale atoms (and,
// with a ragged K, the padded last codes of every weight row); one region
// serves mlp1 and mlp2 in turn.
size_t mx_prep_bytes(const moe_dims_t& d);
// src rows (with perm: the gather x[perm[r] / k]) -> dst = hi (R, K) then lo (R, K), sf.
moe_status_t launch_mx_quant(const moe_dims_t& d, const uint16_t* src, const int32_t* perm, int K,
                             const int32_t* offsets, uint8_t* dst, uint8_t* sf, int* status, cudaStream_t s);
// mlp1 from quantised rows; h in bf16 (h non-null) or quantised for mlp2 (hq,
// h_sf). prepared: the weight's prepare-once form (mx_prepare) or null, in
// which case prep (workspace, mx_prep_bytes) receives this call's preparation.
moe_status_t launch_mlp1_mx(const moe_dims_t& d, const uint8_t* xq, const uint8_t* x_sf, const int32_t* offsets,
                            const uint8_t* codes, const uint8_t* scales, const uint8_t* prepared, const uint16_t* b1,
                            uint16_t* h, uint8_t* hq, uint8_t* h_sf, uint8_t* prep, int* status, cudaStream_t s);
moe_status_t launch_mlp2_mx(const moe_dims_t& d, const uint8_t* hq, const uint8_t* h_sf, const int32_t* perm,
                            const int32_t* offsets, const float* topk_w, const uint8_t* codes, const uint8_t* scales,
                            const uint8_t* prepared, const uint16_t* b2, float* o_perm, uint8_t* prep, int* status,
                            cudaStream_t s);
// The prepare-once form of an MXFP4 weight (which = 1: W1, 2: W2): its size
// (0 for unsupported sizes) and the pass that writes it.
size_t mx_prepared_bytes(const moe_dims_t& d, int which);
moe_status_t mx_prepare(const moe_dims_t& d, int which, const uint8_t* codes, const uint8_t* scales, uint8_t* out,
                        cudaStream_t s);

}  // namespace moe
