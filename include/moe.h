/*
 * moe.h -- C ABI of the B200 (sm_100a) GPT-OSS-style MoE feed-forward layer.
 *
 * The layer (per token t of x, T x D):
 *   logits = x[t] . Wr^T + br                       router linear with bias
 *   idx    = the k largest logits, ordered by (logit desc, expert index asc)
 *   w      = softmax over those k logits
 *   for each chosen expert e = idx[j]:
 *     u    = W1[e] . x[t] + b1[e]                   mlp1, 2I outputs
 *     h    = silu(u[0:I]) * u[I:2I]                 SwiGLU, rounded to bf16
 *     o_j  = W2[e] . h + b2[e]                      mlp2, D outputs
 *   y[t]   = sum_j w_j * o_j                        weighted combine, bf16
 * Sources: the torchtitan GPT-OSS guide (sections "grouped matrix
 * multiplication" -- mlp1/mlp2 as grouped GEMMs over per-expert token
 * segments with offsets = cumsum(num_tokens_per_expert), weights stored
 * (num_experts, out_dim, in_dim), and "HuggingFace weight adapter" -- router
 * gate weight and bias, MXFP4 expert blocks); the from-scratch GPT-OSS
 * write-up ("model flow" diagram: expert routing top-4, expert compute,
 * weighted combination); the GPT-OSS in Transformers blog (MXFP4 paragraph:
 * E2M1 values with one scale per 32-element block).
 *
 * Conventions for every entry point:
 *  - All pointers are DEVICE pointers unless stated otherwise; every tensor
 *    is dense, row-major, and at least 32-byte aligned (a misaligned pointer
 *    is an argument error). bf16 tensors are passed as uint16_t bit patterns.
 *  - The caller owns every buffer and the stream. The library allocates
 *    nothing; scratch lives in the caller's workspace `ws` of `ws_bytes`
 *    bytes (at least moe_workspace_bytes(d)), zero-filled once before its
 *    first use. One workspace serves one stream at a time.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls
 *    only enqueue work: no host synchronisation, counts stay on the device.
 *  - Argument errors are returned synchronously (nothing is enqueued).
 *    Errors found on the device (an index out of range, a bounded wait that
 *    gave up) are recorded in a status word inside `ws` and read with
 *    moe_read_device_status(); when one is recorded the outputs are
 *    unspecified, but every memory access stayed inside the given buffers.
 *  - Supported sizes: T >= 1, 1 <= k <= E <= 256, k <= 8, D and I multiples
 *    of 64, D <= 16384, I <= 16384, T*k < 2^31. Other sizes return
 *    MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, k > E, pointer not 32-byte aligned */
  MOE_ERR_UNSUPPORTED = 2,   /* sizes outside the supported set above */
  MOE_ERR_WORKSPACE = 3,     /* ws_bytes < moe_workspace_bytes(d) */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed (launch, tensor map) */
  MOE_ERR_TIMEOUT = 5,       /* device: a bounded wait in a kernel gave up */
  MOE_ERR_DEVICE_BOUNDS = 6  /* device: an expert index, row index or offset out of range */
} moe_status_t;

typedef enum { MOE_W_BF16 = 0, MOE_W_MXFP4 = 1 } moe_wfmt_t;

/* T tokens, D model dim, E experts, top-k, I expert intermediate dim, and the
 * expert-weight format (moe_wfmt_t). R = T*k routed rows. */
/* Activation between mlp1 and mlp2, on the gate half g and up half u of mlp1's
 * output (rows [0,I) and [I,2I) of W1):
 *   MOE_ACT_SWIGLU:  h = silu(g) * u, silu(g) = g / (1 + e^-g)
 *   MOE_ACT_GPTOSS:  the GPT-OSS variant (torchtitan GPT-OSS guide, paragraph
 *     on the grouped experts' SwiGLU variant): gc = min(g, act_limit),
 *     uc = min(max(u, -act_limit), act_limit), h = gc * sigmoid(act_alpha * gc) * (uc + 1).
 *     The pages do not give alpha and limit; the caller does (act_limit may be
 *     +inf for no clamping). Ignored for MOE_ACT_SWIGLU. */
typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_GPTOSS = 1 } moe_act_t;

typedef struct {
  int32_t T, D, E, k, I, wfmt;
  int32_t act;                /* moe_act_t */
  float act_alpha, act_limit; /* MOE_ACT_GPTOSS only */
} moe_dims_t;

/* An expert weight tensor of logical shape (E, N, K), K the reduction dim.
 * MOE_W_BF16:  data = (E, N, K) bf16, scales = NULL, prepared = NULL.
 * MOE_W_MXFP4: data = (E, N, K/2) bytes of E2M1 codes, two per byte along K
 *              with the even element in the low nibble; scales = (E, N, K/32)
 *              E8M0 bytes, value 2^(s-127), one per 32 consecutive K;
 *              prepared = NULL, or the output of moe_mxfp4_prepare() for this
 *              weight and these dims: the GEMMs then read only the prepared
 *              copy (no per-call preparation pass), and data and scales may
 *              be NULL. */
typedef struct {
  const void* data;
  const uint8_t* scales;
  const void* prepared;
} moe_weight_t;

/* Bytes of workspace every entry point below needs for dims d (0 if d is
 * invalid). Holds the device status word, the permutation scratch and, for
 * moe_forward, the routed intermediates (indices, gate weights, counts,
 * offsets, perm, inv, gathered rows, h, expert outputs). */
MOE_API size_t moe_workspace_bytes(moe_dims_t d);

/* Validate d against the supported set (MOE_OK, INVALID_ARG or UNSUPPORTED). */
MOE_API moe_status_t moe_check_dims(moe_dims_t d);

/* Router linear + top-k + softmax over the chosen logits.
 * Defined by: torchtitan GPT-OSS guide, "HuggingFace weight adapter" (the
 * router is a linear layer with weight and bias, one logit per expert);
 * from-scratch GPT-OSS write-up, "model flow" (expert routing, top-4 of 32
 * experts); the softmax is taken over the k chosen logits only.
 *   x (T,D) bf16, Wr (E,D) bf16, br (E) bf16
 *   -> topk_idx (T,k) int32, ordered by (logit desc, expert asc);
 *      topk_w (T,k) fp32, softmax of the chosen logits (sums to 1).
 * Logits are accumulated in fp32 from the bf16 products (tcgen05 tensor
 * cores, one 128-token tile per CTA; batches of at most 18 tiles also split
 * the reduction over D across CTAs and sum the fp32 partials in a fixed
 * order, kept in ws). Deterministic for given sizes. */
MOE_API moe_status_t moe_route(moe_dims_t d, const uint16_t* x, const uint16_t* Wr, const uint16_t* br,
                       int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, void* stream);

/* Group the R = T*k assignments a = t*k + j by expert (stable in a).
 * Defined by: torchtitan GPT-OSS guide, "grouped matrix multiplication"
 * (tokens sorted by expert, num_tokens_per_expert, offsets = cumsum of it,
 * computed without a device-to-host sync).
 *   topk_idx (T,k) int32
 *   -> counts (E) int32 tokens per expert; offsets (E+1) int32 exclusive
 *      prefix sums (offsets[0] = 0, offsets[E] = R); perm (R) int32, row r of
 *      the expert-sorted order holds assignment perm[r]; inv (R) int32 with
 *      inv[perm[r]] = r (inv[a] = -1 for an out-of-range index, which also
 *      records MOE_ERR_DEVICE_BOUNDS).
 * Deterministic: no atomics decide any output position. */
MOE_API moe_status_t moe_permute(moe_dims_t d, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                         int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes, void* stream);

/* Gather the routed rows: x_perm[r] = x[perm[r] / k], x_perm (R,D) bf16.
 * Defined by: torchtitan GPT-OSS guide, "grouped matrix multiplication"
 * (the grouped GEMM's input is the token rows in expert-sorted order). */
MOE_API moe_status_t moe_gather(moe_dims_t d, const uint16_t* x, const int32_t* perm, uint16_t* x_perm,
                        void* ws, size_t ws_bytes, void* stream);

/* Grouped mlp1 + bias + SwiGLU over the expert segments of x_perm.
 * Defined by: torchtitan GPT-OSS guide, "grouped matrix multiplication"
 * (mlp1 as one grouped GEMM over the expert segments given by offsets,
 * weights stored (num_experts, out_dim, in_dim) with a per-expert bias,
 * then the SwiGLU; the guide's GPT-OSS variant is moe_act_t's second
 * form) and "expert-parallel sharding" (mlp1 weight E x 2I x D, bias E x 2I).
 * for r in [offsets[e], offsets[e+1]):
 *   u = W1[e] . x_perm[r] + b1[e] (fp32 accumulate), h[r,i] = bf16(act(u[i], u[I+i]))
 *   with act = d.act (plain SwiGLU or the GPT-OSS variant, see moe_act_t).
 *   x_perm (R,D) bf16, offsets (E+1), W1 (E,2I,D), b1 (E,2I) bf16 -> h (R,I) bf16.
 * tcgen05 tensor-core grouped GEMM, persistent over (expert, row tile, column tile).
 * MXFP4 weights: the codes are multiplied as stored on block-scaled tensor
 * cores (tcgen05 kind::mxf8f6f4); x_perm is first quantised in ws to a hi +
 * lo pair of E4M3 terms per element with an E8M0 scale per 32 elements each
 * (about 8 significant bits, like bf16). Experts with 1..32 rows take a
 * kernel with the weights on the MMA's M side, the others 128-row tiles. A
 * block of 32 values whose largest magnitude is below 2^-119 is taken as
 * zero; a non-finite value makes its block NaN. */
MOE_API moe_status_t moe_mlp1(moe_dims_t d, const uint16_t* x_perm, const int32_t* offsets, moe_weight_t W1,
                      const uint16_t* b1, uint16_t* h, void* ws, size_t ws_bytes, void* stream);

/* Grouped mlp2 + bias + gate weight over the expert segments of h.
 * Defined by: torchtitan GPT-OSS guide, "grouped matrix multiplication"
 * (mlp2 as the second grouped GEMM, weights E x D x I with bias E x D) and
 * the write-up's "weighted combination" (each expert output scaled by its
 * routing weight; here inside mlp2's epilogue).
 *   o_perm[r] = topk_w[perm[r]] * (W2[e] . h[r] + b2[e]), stored fp32.
 *   h (R,I) bf16, perm (R), offsets (E+1), topk_w (T*k) fp32, W2 (E,D,I),
 *   b2 (E,D) bf16 -> o_perm (R,D) fp32. The expert outputs stay fp32 so that
 *   the combine rounds each y element to bf16 once. */
MOE_API moe_status_t moe_mlp2(moe_dims_t d, const uint16_t* h, const int32_t* perm, const int32_t* offsets,
                      const float* topk_w, moe_weight_t W2, const uint16_t* b2, float* o_perm,
                      void* ws, size_t ws_bytes, void* stream);

/* Defined by: torchtitan GPT-OSS guide, "grouped matrix multiplication" (the
 * whole grouped-experts forward: gather, mlp1 + SwiGLU, mlp2).
 * The expert FFN of all routed rows: moe_gather, moe_mlp1, moe_mlp2 with the
 * gathered rows and h kept in ws. o_perm (R,D) fp32 as moe_mlp2. */
MOE_API moe_status_t moe_ffn_grouped(moe_dims_t d, const uint16_t* x, const int32_t* perm, const int32_t* offsets,
                             const float* topk_w, moe_weight_t W1, const uint16_t* b1, moe_weight_t W2,
                             const uint16_t* b2, float* o_perm, void* ws, size_t ws_bytes, void* stream);

/* Weighted combine back to token order (the gate weight is already applied).
 * Defined by: from-scratch GPT-OSS write-up, "model flow" (weighted
 * combination of the top-4 expert outputs per token).
 *   y[t] = bf16( sum_{j<k} o_perm[inv[t*k+j]] ), o_perm (R,D) fp32, summed in
 *   fp32 in j order. A gather: each output row is written once, no atomics,
 *   bitwise deterministic. */
MOE_API moe_status_t moe_combine(moe_dims_t d, const float* o_perm, const int32_t* inv, uint16_t* y,
                         void* ws, size_t ws_bytes, void* stream);

/* The whole layer in one call: route, permute, gather, mlp1, mlp2, combine,
 * as the write-up's "model flow" (routing, expert compute, weighted
 * combination) and the torchtitan guide's grouped-experts forward define it;
 * enqueued on `stream` with every intermediate in ws.
 *   x (T,D) bf16, Wr (E,D), br (E), W1/b1, W2/b2 as above -> y (T,D) bf16. */
MOE_API moe_status_t moe_forward(moe_dims_t d, const uint16_t* x, const uint16_t* Wr, const uint16_t* br,
                         moe_weight_t W1, const uint16_t* b1, moe_weight_t W2, const uint16_t* b2,
                         uint16_t* y, void* ws, size_t ws_bytes, void* stream);

/* The MXFP4 expert weights are multiplied as stored (E2M1 codes with E8M0
 * block scales, GPT-OSS in Transformers blog, MXFP4 paragraph) on block-scaled
 * tensor-core MMAs, which read the scales in their own layout: each MXFP4 GEMM
 * first rewrites the scales of the experts a call routes to into that layout
 * (and, when K is not a multiple of 128, the last 64 codes of every weight
 * row padded to 128), into ws. The weights are static, so a caller can do it
 * once instead, which also stores the codes K-block-major -- for each block
 * of 128 K, every row's 64 code bytes side by side, the ragged last block
 * padded with zeros -- so the GEMMs read them as contiguous runs rather than
 * as 64-byte pieces of rows K/2 bytes apart (about twice the delivered HBM
 * bandwidth on decode-sized batches). The form takes about the size of the
 * codes plus 2.4x the scales (the atoms of both GEMM kernels); once it
 * exists, the original data and scales are not read again. moe_mxfp4_prepare() writes the complete form for one weight
 * (which = 1: W1 (E, 2I, D); which = 2: W2 (E, D, I)) into `out` (device
 * memory of at least moe_mxfp4_prepared_bytes(d, which) bytes, 256-byte
 * aligned, owned by the caller), enqueued on `stream`; pass it as that
 * weight's moe_weight_t.prepared in every later call with the same dims
 * (T may differ). The form depends on D, I and E only. Returns INVALID_ARG
 * for a null pointer, a bf16 weight format or which outside {1, 2},
 * WORKSPACE if out_bytes is too small. */
MOE_API size_t moe_mxfp4_prepared_bytes(moe_dims_t d, int32_t which);
MOE_API moe_status_t moe_mxfp4_prepare(moe_dims_t d, int32_t which, moe_weight_t W, void* out, size_t out_bytes,
                               void* stream);

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory -- e.g. code running where the memory budget is fixed up front by a
 * host framework or serving runtime, or on a latency-critical path that must
 * not call cudaMalloc (which can synchronise the device). This entry point
 * has no counterpart in the layer's description; it is a deployment aid.
 * Same arguments and outputs as moe_permute, minus ws: the per-block expert
 * histogram it needs is kept in a fixed 256 KB array inside the library
 * (held on every GPU that loads the library until the process exits), so it
 * allocates nothing. Limit: ceil(T*k / 2048) * E <= 65536 (e.g. T*k <= 4M at
 * E = 32, <= 512K at E = 256); larger sizes return MOE_ERR_UNSUPPORTED
 * without enqueueing anything. The first call on each device looks up the
 * array's device address with that device current; make that first call
 * before any stream capture. Calls share the array, so two calls that overlap
 * on the GPU (other streams or host threads) race. With no workspace there is
 * no device status word: an out-of-range expert index shows up only as
 * inv[a] = -1 and a missing count. */
MOE_API moe_status_t moe_permute_noalloc(moe_dims_t d, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                                 int32_t* perm, int32_t* inv, void* stream);

/* Synchronise `stream`, return the device status recorded in ws since the
 * last read (MOE_OK if none) and clear it. */
MOE_API moe_status_t moe_read_device_status(void* ws, void* stream);

/* Self-test of the device-side failure detection: enqueue a one-thread
 * kernel that waits on an mbarrier nothing will arrive on, using the same
 * bounded wait as every tcgen05 kernel, gives up after limit_ns (at most 2 s)
 * and records MOE_ERR_TIMEOUT in ws's status word. Read it with
 * moe_read_device_status(); the context stays usable. */
MOE_API moe_status_t moe_selftest_wait_timeout(void* ws, uint64_t limit_ns, void* stream);

/* Static description of a status code. */
MOE_API const char* moe_status_str(moe_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
