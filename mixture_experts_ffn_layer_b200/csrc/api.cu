// The C ABI of include/moe.h: argument validation, workspace layout, and the
// enqueueing of the kernels of route.cu, permute.cu, grouped_gemm.cu,
// grouped_gemm_pair.cu and mx_gemm.cu on the caller's stream.
// No host synchronisation except in moe_read_device_status.
#include <cmath>

#include "common.cuh"

#include <stdint.h>

namespace moe {
namespace {

struct WsLayout {
  size_t block_counts, topk_idx, topk_w, counts, offsets, perm, inv, x_perm, h, o_perm, xq, x_sf, hq, h_sf,
      mx_prep, route_partial, total;
};

WsLayout ws_layout(const moe_dims_t& d) {
  WsLayout L{};
  const int64_t R = static_cast<int64_t>(d.T) * d.k;
  size_t off = kWsHeader;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  L.block_counts = take(static_cast<size_t>(perm_blocks(R)) * d.E * 4);
  L.topk_idx = take(R * 4);
  L.topk_w = take(R * 4);
  L.counts = take(static_cast<size_t>(d.E) * 4);
  L.offsets = take(static_cast<size_t>(d.E + 1) * 4);
  L.perm = take(R * 4);
  L.inv = take(R * 4);
  L.x_perm = take(static_cast<size_t>(R) * d.D * 2);
  L.h = take(static_cast<size_t>(R) * d.I * 2);
  L.o_perm = take(static_cast<size_t>(R) * d.D * 4);
  if (route_splits(d) > 1)  // K-split router: fp32 partial logits per split
    L.route_partial = take(static_cast<size_t>(route_splits(d)) * d.T * ((d.E + 15) / 16 * 16) * 4);
  if (d.wfmt == MOE_W_MXFP4) {
    // block-scaled MMA operands: the routed rows and h as hi/lo E4M3 pairs
    // plus their tile-blocked E8M0 scales (the expert weights are used as stored)
    L.xq = take(static_cast<size_t>(R) * d.D * 2);
    L.x_sf = take(mx_sf_bytes(d, d.D));
    L.hq = take(static_cast<size_t>(R) * d.I * 2);
    L.h_sf = take(mx_sf_bytes(d, d.I));
    L.mx_prep = take(mx_prep_bytes(d));
  }
  L.total = off;
  return L;
}

// Every tensor must be 32-byte aligned: the memory-bound kernels move 32-byte
// vectors and TMA needs 16.
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

int* status_word(void* ws) { return static_cast<int*>(ws); }

moe_status_t check_ws(const moe_dims_t& d, void* ws, size_t ws_bytes) {
  if (!ws || !aligned32(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < ws_layout(d).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

moe_status_t check_weight(const moe_dims_t& d, const moe_weight_t& w) {
  if (w.prepared) {
    // the prepare-once form holds everything the MXFP4 GEMMs read: data and
    // scales may be null
    if (d.wfmt != MOE_W_MXFP4 || (reinterpret_cast<uintptr_t>(w.prepared) & 255u)) return MOE_ERR_INVALID_ARG;
    if ((w.data && !aligned32(w.data)) || (w.scales && !aligned32(w.scales))) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
  }
  if (!w.data || !aligned32(w.data)) return MOE_ERR_INVALID_ARG;
  if (d.wfmt == MOE_W_MXFP4 && (!w.scales || !aligned32(w.scales))) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

const uint8_t* prepared_of(const moe_weight_t& w) { return static_cast<const uint8_t*>(w.prepared); }

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// SM-pair GEMM tiles (256 rows) feed the tensor cores ~3% better per executed
// FLOP than single-SM tiles (128 rows) but round every expert segment up to
// 256 rows; measured on B200 they win only when segments are long. So pairs
// are used when experts average at least 2048 routed rows (padding <= ~6%).
bool use_pair(const moe_dims_t& d) { return static_cast<int64_t>(d.T) * d.k >= 2048LL * d.E; }

#define MOE_TRY(expr)                      \
  do {                                     \
    moe_status_t _st = (expr);             \
    if (_st != MOE_OK) return _st;         \
  } while (0)

#define MOE_REQUIRE(cond)                         \
  do {                                            \
    if (!(cond)) return MOE_ERR_INVALID_ARG;      \
  } while (0)

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status_t moe_check_dims(moe_dims_t d) {
  if (d.T <= 0 || d.D <= 0 || d.E <= 0 || d.k <= 0 || d.I <= 0) return MOE_ERR_INVALID_ARG;
  if (d.k > d.E) return MOE_ERR_INVALID_ARG;
  if (d.wfmt != MOE_W_BF16 && d.wfmt != MOE_W_MXFP4) return MOE_ERR_INVALID_ARG;
  if (d.act != MOE_ACT_SWIGLU && d.act != MOE_ACT_GPTOSS) return MOE_ERR_INVALID_ARG;
  // GPT-OSS variant: a finite alpha and a limit > 0 (+inf allowed: no clamping)
  if (d.act == MOE_ACT_GPTOSS && (!std::isfinite(d.act_alpha) || !(d.act_limit > 0.0f))) return MOE_ERR_INVALID_ARG;
  if (d.E > 256 || d.k > 8) return MOE_ERR_UNSUPPORTED;
  if (d.D % 64 || d.I % 64 || d.D > 16384 || d.I > 16384) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d.T) * d.k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

size_t moe_workspace_bytes(moe_dims_t d) {
  if (moe_check_dims(d) != MOE_OK) return 0;
  return ws_layout(d).total;
}

moe_status_t moe_route(moe_dims_t d, const uint16_t* x, const uint16_t* Wr, const uint16_t* br, int32_t* topk_idx,
                       float* topk_w, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(moe_check_dims(d));
  MOE_REQUIRE(x && Wr && br && topk_idx && topk_w);
  MOE_REQUIRE(aligned32(x) && aligned32(Wr));
  MOE_TRY(check_ws(d, ws, ws_bytes));
  const WsLayout L = ws_layout(d);
  float* partial = route_splits(d) > 1 ? at<float>(ws, L.route_partial) : nullptr;
  return cuda_status(
      launch_route(d, x, Wr, br, topk_idx, topk_w, partial, status_word(ws), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_permute(moe_dims_t d, const int32_t* topk_idx, int32_t* counts, int32_t* offsets, int32_t* perm,
                         int32_t* inv, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(moe_check_dims(d));
  MOE_REQUIRE(topk_idx && counts && offsets && perm && inv);
  MOE_TRY(check_ws(d, ws, ws_bytes));
  const WsLayout L = ws_layout(d);
  return cuda_status(launch_permute(d, topk_idx, counts, offsets, perm, inv, at<int32_t>(ws, L.block_counts),
                                    status_word(ws), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_gather(moe_dims_t d, const uint16_t* x, const int32_t* perm, uint16_t* x_perm, void* ws,
                        size_t ws_bytes, void* stream) {
  MOE_TRY(moe_check_dims(d));
  MOE_REQUIRE(x && perm && x_perm && aligned32(x) && aligned32(x_perm));
  MOE_TRY(check_ws(d, ws, ws_bytes));
  return cuda_status(launch_gather(d, x, perm, x_perm, status_word(ws), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_mlp1(moe_dims_t d, const uint16_t* x_perm, const int32_t* offsets, moe_weight_t W1,
                      const uint16_t* b1, uint16_t* h, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(moe_check_dims(d));
  MOE_REQUIRE(x_perm && offsets && b1 && h && aligned32(x_perm) && aligned32(b1) && aligned32(h));
  MOE_TRY(check_weight(d, W1));
  MOE_TRY(check_ws(d, ws, ws_bytes));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(d);
  if (d.wfmt == MOE_W_MXFP4) {
    // the routed rows to hi/lo E4M3 + scales, then the block-scaled GEMM (h in bf16)
    MOE_TRY(launch_mx_quant(d, x_perm, nullptr, d.D, offsets, at<uint8_t>(ws, L.xq), at<uint8_t>(ws, L.x_sf),
                            status_word(ws), s));
    return launch_mlp1_mx(d, at<uint8_t>(ws, L.xq), at<uint8_t>(ws, L.x_sf), offsets,
                          static_cast<const uint8_t*>(W1.data), W1.scales, prepared_of(W1), b1, h, nullptr, nullptr,
                          at<uint8_t>(ws, L.mx_prep), status_word(ws), s);
  }
  const uint16_t* w1 = static_cast<const uint16_t*>(W1.data);
  if (use_pair(d)) return launch_mlp1_pair(d, x_perm, offsets, w1, b1, h, status_word(ws), s);
  return launch_mlp1(d, x_perm, offsets, w1, b1, h, status_word(ws), s);
}

moe_status_t moe_mlp2(moe_dims_t d, const uint16_t* h, const int32_t* perm, const int32_t* offsets,
                      const float* topk_w, moe_weight_t W2, const uint16_t* b2, float* o_perm, void* ws,
                      size_t ws_bytes, void* stream) {
  MOE_TRY(moe_check_dims(d));
  MOE_REQUIRE(h && perm && offsets && topk_w && b2 && o_perm && aligned32(h) && aligned32(b2) && aligned32(o_perm));
  MOE_TRY(check_weight(d, W2));
  MOE_TRY(check_ws(d, ws, ws_bytes));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(d);
  if (d.wfmt == MOE_W_MXFP4) {
    MOE_TRY(launch_mx_quant(d, h, nullptr, d.I, offsets, at<uint8_t>(ws, L.hq), at<uint8_t>(ws, L.h_sf),
                            status_word(ws), s));
    return launch_mlp2_mx(d, at<uint8_t>(ws, L.hq), at<uint8_t>(ws, L.h_sf), perm, offsets, topk_w,
                          static_cast<const uint8_t*>(W2.data), W2.scales, prepared_of(W2), b2, o_perm, at<uint8_t>(ws, L.mx_prep),
                          status_word(ws), s);
  }
  const uint16_t* w2 = static_cast<const uint16_t*>(W2.data);
  if (use_pair(d)) return launch_mlp2_pair(d, h, perm, offsets, topk_w, w2, b2, o_perm, status_word(ws), s);
  return launch_mlp2(d, h, perm, offsets, topk_w, w2, b2, o_perm, status_word(ws), s);
}

moe_status_t moe_ffn_grouped(moe_dims_t d, const uint16_t* x, const int32_t* perm, const int32_t* offsets,
                             const float* topk_w, moe_weight_t W1, const uint16_t* b1, moe_weight_t W2,
                             const uint16_t* b2, float* o_perm, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(moe_check_dims(d));
  MOE_REQUIRE(x && perm && offsets && topk_w && b1 && b2 && o_perm);
  MOE_TRY(check_ws(d, ws, ws_bytes));
  const WsLayout L = ws_layout(d);
  uint16_t* x_perm = at<uint16_t>(ws, L.x_perm);
  uint16_t* h = at<uint16_t>(ws, L.h);
  if (d.wfmt == MOE_W_MXFP4) {
    // x_perm and h are internal here: the gather writes the routed rows
    // straight into their hi/lo E4M3 form and mlp1 writes h in the same form
    // (the same values the stage-by-stage entry points produce)
    MOE_REQUIRE(x && aligned32(x) && aligned32(b1) && aligned32(b2) && aligned32(o_perm));
    MOE_TRY(check_weight(d, W1));
    MOE_TRY(check_weight(d, W2));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* xq = at<uint8_t>(ws, L.xq);
    uint8_t* hq = at<uint8_t>(ws, L.hq);
    MOE_TRY(launch_mx_quant(d, x, perm, d.D, offsets, xq, at<uint8_t>(ws, L.x_sf), status_word(ws), s));
    MOE_TRY(launch_mlp1_mx(d, xq, at<uint8_t>(ws, L.x_sf), offsets, static_cast<const uint8_t*>(W1.data), W1.scales,
                           prepared_of(W1), b1, nullptr, hq, at<uint8_t>(ws, L.h_sf), at<uint8_t>(ws, L.mx_prep), status_word(ws), s));
    return launch_mlp2_mx(d, hq, at<uint8_t>(ws, L.h_sf), perm, offsets, topk_w, static_cast<const uint8_t*>(W2.data),
                          W2.scales, prepared_of(W2), b2, o_perm, at<uint8_t>(ws, L.mx_prep), status_word(ws), s);
  }
  MOE_TRY(moe_gather(d, x, perm, x_perm, ws, ws_bytes, stream));
  MOE_TRY(moe_mlp1(d, x_perm, offsets, W1, b1, h, ws, ws_bytes, stream));
  return moe_mlp2(d, h, perm, offsets, topk_w, W2, b2, o_perm, ws, ws_bytes, stream);
}

moe_status_t moe_combine(moe_dims_t d, const float* o_perm, const int32_t* inv, uint16_t* y, void* ws,
                         size_t ws_bytes, void* stream) {
  MOE_TRY(moe_check_dims(d));
  MOE_REQUIRE(o_perm && inv && y && aligned32(o_perm) && aligned32(y));
  MOE_TRY(check_ws(d, ws, ws_bytes));
  return cuda_status(launch_combine(d, o_perm, inv, y, status_word(ws), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_forward(moe_dims_t d, const uint16_t* x, const uint16_t* Wr, const uint16_t* br, moe_weight_t W1,
                         const uint16_t* b1, moe_weight_t W2, const uint16_t* b2, uint16_t* y, void* ws,
                         size_t ws_bytes, void* stream) {
  MOE_TRY(moe_check_dims(d));
  MOE_REQUIRE(x && Wr && br && b1 && b2 && y);
  MOE_TRY(check_weight(d, W1));
  MOE_TRY(check_weight(d, W2));
  MOE_TRY(check_ws(d, ws, ws_bytes));
  const WsLayout L = ws_layout(d);
  int32_t* topk_idx = at<int32_t>(ws, L.topk_idx);
  float* topk_w = at<float>(ws, L.topk_w);
  int32_t* counts = at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv = at<int32_t>(ws, L.inv);
  float* o_perm = at<float>(ws, L.o_perm);
  MOE_TRY(moe_route(d, x, Wr, br, topk_idx, topk_w, ws, ws_bytes, stream));
  MOE_TRY(moe_permute(d, topk_idx, counts, offsets, perm, inv, ws, ws_bytes, stream));
  MOE_TRY(moe_ffn_grouped(d, x, perm, offsets, topk_w, W1, b1, W2, b2, o_perm, ws, ws_bytes, stream));
  return moe_combine(d, o_perm, inv, y, ws, ws_bytes, stream);
}

size_t moe_mxfp4_prepared_bytes(moe_dims_t d, int32_t which) {
  if (moe_check_dims(d) != MOE_OK || d.wfmt != MOE_W_MXFP4 || (which != 1 && which != 2)) return 0;
  return mx_prepared_bytes(d, which);
}

moe_status_t moe_mxfp4_prepare(moe_dims_t d, int32_t which, moe_weight_t W, void* out, size_t out_bytes,
                               void* stream) {
  MOE_TRY(moe_check_dims(d));
  MOE_REQUIRE(d.wfmt == MOE_W_MXFP4 && (which == 1 || which == 2) && out);
  MOE_REQUIRE((reinterpret_cast<uintptr_t>(out) & 255u) == 0);
  W.prepared = nullptr;
  MOE_TRY(check_weight(d, W));
  const size_t need = mx_prepared_bytes(d, which);
  if (need == 0) return MOE_ERR_UNSUPPORTED;
  if (out_bytes < need) return MOE_ERR_WORKSPACE;
  return mx_prepare(d, which, static_cast<const uint8_t*>(W.data), W.scales, static_cast<uint8_t*>(out),
                    static_cast<cudaStream_t>(stream));
}

moe_status_t moe_read_device_status(void* ws, void* stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0) {
    if (cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return static_cast<moe_status_t>(v);
}

const char* moe_status_str(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported sizes";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_TIMEOUT: return "device: bounded wait timed out";
    case MOE_ERR_DEVICE_BOUNDS: return "device: index or offset out of range";
  }
  return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Self-test of the bounded wait every tcgen05 kernel uses: one thread waits on
// an mbarrier that nothing will arrive on, gives up after limit_ns and
// records MOE_ERR_TIMEOUT in the status word, exactly as a stalled pipeline
// would. The context stays usable.
#include "sm100.cuh"

namespace moe {
namespace {

__global__ void wait_timeout_selftest_kernel(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = sm100::smem_u32(&bar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    sm100::fence_mbar_init();
    if (!sm100::mbar_wait_bounded(b, 0, nullptr, limit_ns)) record_status(status, MOE_ERR_TIMEOUT);
  }
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_selftest_wait_timeout(void* ws, uint64_t limit_ns, void* stream) {
  if (!ws || limit_ns == 0 || limit_ns > 2000000000ull) return MOE_ERR_INVALID_ARG;
  moe::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<int*>(ws), limit_ns);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
