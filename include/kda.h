/*
 * kda.h - C ABI of libkda.so, the B200 (sm_100a) implementation of the Kimi Delta Attention
 * (KDA) gated delta-rule recurrence used by GLM-5.3's linear_attention layers.
 *
 * The operation (GLM-5.3-Flash model card, the Kimi Delta Attention snippet of
 * Glm5NextTextLinearAttention): every (sequence, head) keeps a state S of shape [dk, dv], row c
 * being key channel c. For each token t, in order,
 *
 *     S      = diag(g_t) S                 g_t = exp(log_g_t), one gate per key channel
 *     m      = k_t^T S
 *     delta  = beta_t (v_t - m)
 *     S      = S + k_t delta^T
 *     o_t    = S^T q_t                     (read-out after the write; no 1/sqrt(dk) scale)
 *
 * Packed variable-length input restarts the state at every document boundary (NeMo AutoModel
 * glm5_next layers page: the docstring of `_torch_recurrent_kda(q, k, v, g, beta, cu_seqlens)`
 * says the state resets at packed boundaries, and `Glm5NextLinearAttention.forward` keeps KDA
 * within each document). The gate arrives in log space as float32: `Glm5NextKDAFp32Params.forward`
 * returns log-decay gates shaped [batch, sequence, heads, head_dim].
 * Decode advances a per-sequence state by one token (metrale glm5next_layer page: KDA decode
 * takes a KdaSeqState).
 *
 * Conventions for every entry point
 *   - All tensors are dense, contiguous, row-major, in DEVICE memory unless stated otherwise, and
 *     every base pointer must be 16-byte aligned.
 *   - The caller owns all memory. The library allocates no device memory, keeps no per-call
 *     state and is safe to call from several host threads on different streams. The one thing it
 *     creates: on the first segmented split-path kda_fwd call (see kda_fwd) from a host thread on
 *     a device, one internal stream and 17 events for that thread and device, kept for the
 *     thread's lifetime.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default stream).
 *   - Problems visible on the host (null or misaligned pointers, bad sizes, unsupported
 *     combinations) return an error before anything is launched. Problems only the device can
 *     see (malformed cu_seqlens, a pipeline wait that timed out) are recorded in a sticky device
 *     error word that kda_get_device_error() reports and clears.
 *   - No C++ exception crosses this interface.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* kda_stream_t; /* identical to cudaStream_t */

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, negative or inconsistent size       */
    KDA_ERR_UNSUPPORTED = 2,  /* valid request this build has no kernel for (see kda_fwd)     */
    KDA_ERR_CUDA = 3,         /* a CUDA runtime call failed; kda_last_error() has the text     */
    KDA_ERR_TIMEOUT = 4,      /* device: a bounded pipeline wait expired (kernel gave up)      */
    KDA_ERR_BAD_SEQLENS = 5,  /* device: cu_seqlens not non-decreasing from 0 to T             */
    KDA_ERR_RANGE = 6         /* reserved: no longer raised (steep decays take a direct path)  */
} kda_status_t;

typedef enum {
    KDA_F32 = 0,   /* float32 */
    KDA_BF16 = 1   /* bfloat16 */
} kda_dtype_t;

/* Algorithm selector for kda_fwd (field `chunk_size`). */
enum {
    KDA_CHUNK_AUTO = 0,      /* 64 for bf16 with dk = dv = 128, else the per-token walk */
    KDA_CHUNK_PER_TOKEN = 1, /* per-token walk: exact fp32 recurrence, any dtype, dk,dv <= 256 */
    KDA_CHUNK_64 = 64        /* chunked WY/UT form on tcgen05 tensor cores: bf16, dk = dv = 128 */
};

/*
 * Problem description for kda_fwd.
 *   B, T, H, dk, dv : batch, tokens per row, heads, key and value head dims.
 *   num_seqs        : number of independent sequences N. Without cu_seqlens N must equal B;
 *                     with cu_seqlens, B must be 1 and N = len(cu_seqlens) - 1.
 *   dtype           : element type of q, k, v, beta and o. log_g, h0 and hT are always float32.
 *   chunk_size      : KDA_CHUNK_AUTO, KDA_CHUNK_PER_TOKEN or KDA_CHUNK_64. For float32 inputs
 *                     any value selects the per-token walk (the exact path).
 */
typedef struct {
    int B, T, H, dk, dv;
    int num_seqs;
    kda_dtype_t dtype;
    int chunk_size;
} kda_fwd_desc_t;

/*
 * kda_fwd - prefill: run the recurrence over whole sequences or packed documents.
 *
 *   q, k    : [B, T, H, dk]  dtype           v, o : [B, T, H, dv] dtype
 *   log_g   : [B, T, H, dk]  float32 (log of the per-channel decay; must be <= 0 and finite)
 *   beta    : [B, T, H]      dtype
 *   h0      : [N, H, dk, dv] float32, or NULL for a zero initial state
 *   cu_seqlens : int32 [N + 1], device, or NULL. Offsets into the packed token axis of a B = 1
 *             row; must start at 0, be non-decreasing and end at T. Empty documents are allowed
 *             (their final state equals their initial state).
 *   o       : output, written for every token.
 *   hT      : [N, H, dk, dv] float32 final state of every sequence/document, or NULL to skip.
 *   workspace, workspace_bytes : scratch owned by the caller (device memory, 16-byte aligned).
 *             With at least kda_fwd_workspace_size(desc) bytes the chunked path runs split: an
 *             intra-chunk kernel computes every chunk's WY factors in parallel over all chunks
 *             and heads and stores them here (about 72.5 KiB per 64-token chunk and head), then a
 *             state pass walks each sequence's chunks. For equal-length sequences of more than
 *             64 chunks the two run in chunk segments of at least 32 chunks (up to 12;
 *             KDA_SPLIT_SEGMENTS, 1-16, overrides): the state pass of one segment runs on an
 *             internal high-priority stream while the intra-chunk kernel works on the next, and
 *             the caller's stream waits for both before the call's later work; the state between
 *             segments (64 KiB per sequence and head) is kept in the workspace. Equal-length sequences with few chains
 *             (sequences x heads) and enough chunks instead run a two-level state pass (see
 *             kda_fwd_scan_segments): the chunks are cut into P segments; the map from a
 *             segment's initial to its final state is affine, S -> A S + B, so the state pass
 *             computes A and B of the inner segments beside segment 0, chains the segments'
 *             initial states in fp32, and then runs every segment at once (3 P - 5 states of
 *             64 KiB per sequence and head in the workspace). With less workspace (but at least
 *             kda_fwd_workspace_size_min(desc), which is 0 unless documents are packed) one fused
 *             kernel per (sequence, head) does both, with no intermediate storage. Both give the
 *             same result up to bf16 rounding of the stored factors. May be NULL when the minimum
 *             is 0.
 *
 * The chunked path (KDA_CHUNK_64) computes in bf16 tensor-core products with fp32 accumulation
 * and an fp32 state. Its fast within-chunk factorisation holds while the summed decay of any 8
 * consecutive tokens inside a 16-token sub-chunk stays above about -69 nats per key channel;
 * a chunk with a steeper decay (a decay product below 1e-30) is evaluated directly instead
 * (cumulative log decay, A_kk and A_qk summed with one exponential per term), at a few times the
 * cost of a fast chunk. Any finite log_g <= 0 is therefore accepted on every path.
 * Returns KDA_OK once the work is enqueued. T = 0 or N = 0 is a valid no-op (hT = h0 or 0).
 */
kda_status_t kda_fwd(const kda_fwd_desc_t* desc, const void* q, const void* k, const void* v,
                     const float* log_g, const void* beta, const float* h0,
                     const int32_t* cu_seqlens, void* o, float* hT, void* workspace,
                     size_t workspace_bytes, kda_stream_t stream);

/*
 * Gated per-head RMSNorm of the output (NeMo glm5_next layers, _TorchRMSNormGated: normalise
 * [batch, sequence, heads, head_dim], then gate with a sigmoid; its base Glm5NextRMSNorm keeps
 * the variance in fp32 and a weight of head_dim entries; metrale glm5next_layer: every norm is
 * x * w / rms). Per (token, head):
 *     y = x / sqrt(mean over head_dim of x^2 + eps) * weight * sigmoid(gate).
 *   gate   : same shape and dtype as the output it gates, device.
 *   weight : [dv] float32, device, shared by all heads.
 *   eps    : >= 0.
 */
typedef struct {
    const void* gate;
    const float* weight;
    float eps;
} kda_out_norm_t;

/*
 * kda_fwd_normed - kda_fwd followed by the gated RMSNorm above, writing y (shaped like o)
 * instead of o: the prefill writes o into y, then one bandwidth-bound pass normalises y in
 * place. The norm sees o rounded to the output dtype, as a separate norm module would. Same
 * arguments, layouts, workspace and errors as kda_fwd; dv <= 256. NULL norm is
 * KDA_ERR_INVALID_ARG.
 */
kda_status_t kda_fwd_normed(const kda_fwd_desc_t* desc, const void* q, const void* k,
                            const void* v, const float* log_g, const void* beta,
                            const float* h0, const int32_t* cu_seqlens,
                            const kda_out_norm_t* norm, void* y, float* hT, void* workspace,
                            size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_bwd - gradients of the recurrence, for training (NeMo glm5_next layers,
 * `_torch_recurrent_kda` is a differentiable reference KDA; this is the derivative of kda_fwd's
 * recurrence). For
 * upstream gradients do (of o) and dhT (of the final states), computes the gradients of
 * L = sum <do, o> + <dhT, hT>:
 *   dq, dk    : [B, T, H, dk] float32      dv       : [B, T, H, dv] float32
 *   dlog_g    : [B, T, H, dk] float32      dbeta    : [B, T, H] float32
 *   dh0       : [N, H, dk, dv] float32, or NULL to skip.
 * The forward arguments (desc, q, k, v, log_g, beta, h0, cu_seqlens) are as for kda_fwd; do has
 * the layout and dtype of o; dhT is [N, H, dk, dv] float32 or NULL (zero). dk = dv = 128
 * (KDA_ERR_UNSUPPORTED otherwise); desc->chunk_size is ignored. Every gradient is computed in
 * fp32 from the exact per-token recurrence; 16 warps per (sequence or document, head), one per 8
 * value columns, run the forward storing the state every 64 tokens, then walk each 64-token chunk
 * backwards after re-running its forward. The workspace (kda_bwd_workspace_size bytes, 16-byte
 * aligned, device) holds those states. dq, dk, dlog_g and dbeta are sums over the value columns:
 * the call zeroes them on the stream and the 16 warps add their parts atomically, in no fixed
 * order, so their last bits may differ between runs (dv and dh0 are written once).
 * Host-checkable errors return before any launch; a malformed cu_seqlens is reported through
 * kda_get_device_error.
 */
kda_status_t kda_bwd(const kda_fwd_desc_t* desc, const void* q, const void* k, const void* v,
                     const float* log_g, const void* beta, const float* h0,
                     const int32_t* cu_seqlens, const void* dout, const float* dhT, float* dq,
                     float* dk, float* dv, float* dlog_g, float* dbeta, float* dh0,
                     void* workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * Workspace bytes kda_bwd needs for `desc`: per (sequence or document, head), one 64 KiB state
 * per 64 tokens of T plus one, one 64-token chunk of states and its read-outs. Host-only; 0 for
 * a rejected description or no tokens.
 */
size_t kda_bwd_workspace_size(const kda_fwd_desc_t* desc);

/*
 * kda_out_norm_gated - the gated RMSNorm on its own: `vectors` vectors of dv elements (for o of
 * shape [B, T, H, dv], vectors = B * T * H), x and gate in dtype, y in dtype (y may equal x).
 * dv <= 256. Host-checkable errors return before any launch.
 */
kda_status_t kda_out_norm_gated(long long vectors, int dv, kda_dtype_t dtype, const void* x,
                                const void* gate, const float* weight, float eps, void* y,
                                kda_stream_t stream);

/*
 * kda_short_conv - the input prologue of the recurrence: the short causal convolution of q, k or
 * v with a reset at packed-document boundaries, an optional SiLU and an optional L2 norm per
 * group of channels, in one pass (NeMo glm5_next layers, _TorchShortConvolution: a depthwise
 * causal Conv1d over [batch, sequence, channels] that resets at packed boundaries;
 * Glm5NextLinearAttention holds one each for q, k and v, of linear_conv_kernel_dim taps). Per
 * channel c and token t of a document starting at s:
 *     y[t, c] = sum_{j < W} weight[c, j] x[t - (W - 1) + j, c]     (positions before s: zero)
 * then, with act = KDA_ACT_SILU, y <- y * sigmoid(y), and, with norm_group = g > 0,
 * y <- y / sqrt(sum over its group of y^2 + eps) for every group of g consecutive channels
 * (g = head_dim normalises each head vector, the form in which q and k enter kda_fwd).
 *   x, y       : [B, T, C] in dtype (C = heads * head_dim), device, 16-byte aligned; y must not
 *                overlap x.
 *   weight     : [C, W] float32, device; 1 <= W <= 8.
 *   cu_seqlens : int32 [num_seqs + 1] on the device (B must be 1), or NULL (each batch row is
 *                one document).
 *   C % 4 == 0; norm_group is 0 or one of 4, 8, ..., 128 and divides C.
 * Host-checkable errors return before any launch; a malformed cu_seqlens sets
 * KDA_ERR_BAD_SEQLENS in the device error word. The pages do not print the activation: it is
 * off unless asked for.
 */
typedef enum { KDA_ACT_NONE = 0, KDA_ACT_SILU = 1 } kda_activation_t;
kda_status_t kda_short_conv(int B, int T, int C, int W, kda_dtype_t dtype, const void* x,
                            const float* weight, const int32_t* cu_seqlens, int num_seqs,
                            kda_activation_t act, int norm_group, float eps, void* y,
                            kda_stream_t stream);

/*
 * Path kda_fwd takes for `desc` (has_cu_seqlens: whether cu_seqlens will be non-NULL):
 * KDA_CHUNK_PER_TOKEN or KDA_CHUNK_64, or the negated kda_status_t when the description is
 * rejected. Host-only, no CUDA calls.
 */
int kda_fwd_algorithm(const kda_fwd_desc_t* desc, int has_cu_seqlens);

/*
 * Number of chunk segments kda_fwd's split chunked path runs for `desc` (each one launch of the
 * intra-chunk kernel and one of the state pass): 1 for packed documents, short sequences or the
 * per-token path, else as described under kda_fwd's workspace. Reads KDA_SPLIT_SEGMENTS like
 * kda_fwd does. Host-only, no CUDA calls; the negated kda_status_t for a rejected description.
 */
int kda_fwd_split_segments(const kda_fwd_desc_t* desc, int has_cu_seqlens);

/*
 * Segments P of kda_fwd's two-level state pass for `desc` (equal-length sequences): P >= 3 when
 * the call runs it (with kda_fwd_workspace_size(desc) bytes of workspace), 1 for the plain state
 * pass (packed documents, many chains, short sequences, the per-token path). P is chosen from a
 * cost model of the phases; KDA_SCAN_SEGMENTS (read per call) overrides it: 0 or 1 = the plain
 * pass, 3 to 32 = that many segments of ceil(chunks / P) chunks (fewer when that leaves a
 * segment empty). Results differ from the plain pass's only by rounding (the segments' initial
 * states are products of fp32 maps whose factors were rounded to bf16 like the state's).
 * Host-only, no CUDA calls; the negated kda_status_t for a rejected description.
 */
int kda_fwd_scan_segments(const kda_fwd_desc_t* desc, int has_cu_seqlens);

/*
 * Workspace bytes for the fastest path kda_fwd has for `desc` (the split chunked path when it
 * applies; 0 when nothing needs scratch). With B == 1 the size allows for cu_seqlens. Host-only,
 * no CUDA calls; 0 for a rejected description.
 */
size_t kda_fwd_workspace_size(const kda_fwd_desc_t* desc);

/*
 * Smallest workspace kda_fwd accepts for `desc`: the fused chunked path's document order (one
 * int32 per packed document, rounded up to 256 bytes; 0 without packed documents). Host-only.
 */
size_t kda_fwd_workspace_size_min(const kda_fwd_desc_t* desc);

/*
 * kda_fwd_no_alloc - kda_fwd for callers that cannot allocate device memory.
 *
 * The source pages have no counterpart for this entry point. It exists for callers that cannot
 * call cudaMalloc, or any allocator, when they run the prefill. Examples: an engine that reserves
 * all device memory at start-up and hands kernels only fixed buffers; a plugin host that exposes
 * no allocator; a serving loop that may not allocate (an allocation can synchronise the device
 * or fail under memory pressure).
 *
 * Same arguments as kda_fwd, without the workspace. The caller still passes every input and
 * output buffer. The scratch kda_fwd would take from the workspace comes from a static device
 * array built into the library: KDA_NO_ALLOC_MAX_DOCS int32 document slots (8 KiB), held by
 * every GPU that loads the library until the process exits. A packed call (cu_seqlens != NULL)
 * with more documents than that returns KDA_ERR_INVALID_ARG before anything is launched.
 *
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current. Make that first call before any stream capture.
 *
 * All calls on a device share the one array, which keeps the last call's contents. Every call
 * rewrites the slots it uses before reading them, so nothing needs to start at zero. Calls that
 * overlap on the GPU (concurrent streams, or several host threads) race on the array: serialise
 * them, or use kda_fwd with a workspace per stream. The array is too small for the split
 * chunked path's workspace, so this entry point runs kda_fwd's fused chunked path: the same
 * result as kda_fwd given kda_fwd_workspace_size_min bytes, and the same as the split path up to
 * bf16 rounding of the factors that path stores.
 * This function allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
#define KDA_NO_ALLOC_MAX_DOCS 2048
kda_status_t kda_fwd_no_alloc(const kda_fwd_desc_t* desc, const void* q, const void* k,
                              const void* v, const float* log_g, const void* beta,
                              const float* h0, const int32_t* cu_seqlens, void* o, float* hT,
                              kda_stream_t stream);

/*
 * kda_decode_step - advance N sequences by one token each, updating the state in place.
 *
 *   q, k, log_g : [N, H, dk] (q, k in dtype, log_g float32)    v, o : [N, H, dv] dtype
 *   beta        : [N, H] dtype
 *   S_inout     : [N, H, dk, dv] float32, read and overwritten with the new state.
 *   o           : output [N, H, dv].
 * S_inout must not alias any other argument. dk, dv <= 256.
 */
kda_status_t kda_decode_step(int N, int H, int dk, int dv, kda_dtype_t dtype, const void* q,
                             const void* k, const void* v, const float* log_g, const void* beta,
                             float* S_inout, void* o, kda_stream_t stream);

/*
 * kda_decode_tokens - advance N sequences by T tokens each from their decode state, in place:
 * the recurrence of the GLM-5.3-Flash model card's Kimi Delta Attention snippet, token by token,
 * starting from S_inout and leaving the final state there. It serves rows that run against a
 * decode state several at a time, such as the verify rows of batched decoding (metrale
 * glm5next_layer, decoder-layer invariants: decode_batched gives verify row t its own slot).
 * For d = 128 the state crosses HBM once per call (read once, updated T times in registers,
 * written once), so T tokens cost about what one decode step costs.
 *
 *   q, k, log_g : [N, T, H, dk] (q, k in dtype, log_g float32)    v, o : [N, T, H, dv] dtype
 *   beta        : [N, T, H] dtype
 *   S_inout     : [N, H, dk, dv] float32, read and overwritten with the state after token T.
 *   o           : output [N, T, H, dv], row t the read-out after token t.
 * T = 1 is kda_decode_step (same layouts, same arithmetic order); T = 0 or N = 0 does nothing.
 * S_inout must not alias any other argument. dk, dv <= 256. Host-checkable errors return before
 * any launch.
 */
kda_status_t kda_decode_tokens(int N, int H, int T, int dk, int dv, kda_dtype_t dtype,
                               const void* q, const void* k, const void* v, const float* log_g,
                               const void* beta, float* S_inout, void* o, kda_stream_t stream);

/*
 * kda_get_device_error - synchronise `stream`, then return and clear the sticky device error
 * word (KDA_OK, KDA_ERR_BAD_SEQLENS or KDA_ERR_TIMEOUT), or KDA_ERR_CUDA if
 * the synchronisation itself failed. The word is per device and shared by all streams.
 */
kda_status_t kda_get_device_error(kda_stream_t stream);

/* Static description of a status code. */
const char* kda_status_string(kda_status_t status);

/* Text of the last error raised on this host thread ("" if none). Valid until the next call. */
const char* kda_last_error(void);

/* Library version as major * 10000 + minor * 100 + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
