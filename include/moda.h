/*
 * moda.h -- C ABI of the B200 (sm_100a) mixture-of-depths attention (MoDA) library.
 *
 * The operator (hyper.ai summary of arXiv 2603.15619, section "Mixture-of-Depths
 * Attention (MoDA)"): every query head attends in ONE softmax, with all scores
 * normalised together, to
 *   (a) the sequence keys/values of its GQA group at the current layer, causally, and
 *   (b) the L depth keys/values that preceding attention and FFN sublayers wrote for the
 *       query's own token position.
 * For row (b, h, t) with g = h / (Hq / Hkv):
 *   out[b,h,t] = softmax over { scale*<q,k[b,g,s]> : s <= t } U { scale*<q,kd[b,g,t,j]> : j < L }
 *                applied to the matching values v[b,g,s] / vd[b,g,t,j]
 *   lse[b,h,t] = natural log of the softmax normaliser (sum of exp of the scaled logits).
 * The same page's section "Hardware-efficient implementation" describes the depth cache
 * flattened along one axis of length T*L so that each query reads one contiguous
 * range, and a chunk/group-aware tiling; the [B,Hkv,T,L,d] layout below is that
 * flattening per (batch, KV head).
 *
 * Tensors (all row-major and contiguous, all pointers DEVICE pointers, 16-byte aligned):
 *   q, out, dout, dq : bf16 [B][Hq][T][d]
 *   k, v, dk, dv     : bf16 [B][Hkv][T][d]
 *   kd, vd, dkd, dvd : bf16 [B][Hkv][T][L][d]     (may be NULL when L == 0)
 *   lse              : fp32 [B][Hq][T]
 * Sizes: B, T >= 1; Hq, Hkv >= 1 with Hq % Hkv == 0 and Hq / Hkv <= 64; L >= 0;
 * d in {64, 128}.  scale is applied to every logit (typically 1/sqrt(d)) and must be
 * finite.  Violations give MODA_ERR_INVALID_ARGUMENT, except d outside {64, 128}, a
 * group Hq / Hkv above 64, and problems beyond the kernels' index ranges
 * (B*Hq*T > 2^31 rows, B*Hkv > 65535, T > 2^30 or L > 65535), which give
 * MODA_ERR_UNSUPPORTED.  Output buffers must not overlap any input or each other
 * (MODA_ERR_INVALID_ARGUMENT).
 * causal != 0: sequence key s is visible to token t iff s <= t; causal == 0: every
 * sequence key is visible.  Depth keys are always the query's own token's only.
 *
 * Ownership: the caller allocates and owns every buffer (including the backward
 * workspace).  Calls are asynchronous and stream-ordered on `stream`; the library keeps
 * no per-call state and never allocates caller-visible memory.  Thread-safe.
 *
 * Errors: argument checks run before any launch and nothing is launched on failure.
 * No entry point aborts or throws.  Kernels that detect an internal failure (a bounded
 * wait that ran out, an index check) record it in a per-device error word that
 * moda_check_device_errors() reads and clears.
 *
 * Fault injection (for testing a caller's error handling; not on the paper): when the
 * environment variable MODA_FAULT_INJECT is "validate", every compute entry point returns
 * MODA_ERR_INVALID_ARGUMENT before its argument checks; when it is "launch", it returns
 * MODA_ERR_CUDA once its argument checks have passed, in place of the device query and
 * the launch.  Nothing is launched in either case.  The variable is read on every call.
 */
#ifndef MODA_H_
#define MODA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MODA_OK = 0,
    MODA_ERR_INVALID_ARGUMENT = 1, /* null/misaligned pointer, bad size, aliasing output */
    MODA_ERR_UNSUPPORTED = 2,      /* d not in {64,128}, group too large, not sm_100 */
    MODA_ERR_CUDA = 3,             /* a CUDA runtime/driver call failed */
    MODA_ERR_TIMEOUT = 4,          /* a kernel's bounded wait ran out */
    MODA_ERR_INTERNAL = 5          /* a kernel's internal consistency check failed */
} moda_status_t;

/* Opaque stream handle: a cudaStream_t (CUstream); NULL is the legacy default stream. */
typedef void *moda_stream_t;

/*
 * Forward pass.  Writes out (bf16) and lse (fp32, natural log).  Definition: see the
 * header comment (one joint softmax over causal sequence keys and own-token depth keys).
 * kd/vd may be NULL iff L == 0, in which case this is plain causal GQA attention.
 * Returns MODA_OK once the kernel is enqueued on `stream`.
 */
moda_status_t moda_forward(const void *q, const void *k, const void *v, const void *kd,
                           const void *vd, void *out, float *lse, int B, int Hq, int Hkv,
                           int T, int L, int d, float scale, int causal,
                           moda_stream_t stream);

/*
 * moda_forward with the depth path chosen by the caller; the result is the same
 * operator either way (hyper.ai summary of arXiv 2603.15619, section "Hardware-efficient
 * implementation": the depth logits enter the same on-chip softmax state as the
 * sequence logits).  depth_path:
 *   0  automatic: the choice moda_forward makes (dense depth blocks whenever L > 0 and
 *      Hq/Hkv divides 128; the fold otherwise);
 *   1  CUDA-core fold: each query tile's depth rows are folded into the softmax state on
 *      CUDA cores before its sequence blocks;
 *   2  dense depth blocks: the depth rows run through the tensor-core pipeline as extra
 *      128-key blocks of (token, entry) rows, each query row masked to its own token's
 *      entries.  Needs Hq/Hkv to divide 128 (MODA_ERR_UNSUPPORTED otherwise).
 * The two paths round differently (the fold's logits are fp32 CUDA-core dot products,
 * the dense path's come from the tensor cores), so results agree to rounding, not bits.
 * Any other depth_path value: MODA_ERR_INVALID_ARGUMENT.  Everything else as moda_forward.
 */
moda_status_t moda_forward_depth_path(const void *q, const void *k, const void *v,
                                      const void *kd, const void *vd, void *out, float *lse,
                                      int B, int Hq, int Hkv, int T, int L, int d,
                                      float scale, int causal, int depth_path,
                                      moda_stream_t stream);

/*
 * Depth-only attention forward: the pages' other operator (hyper.ai summary of arXiv
 * 2603.15619, section "Depth-stream mechanisms": a layer's input is attention over the
 * key/value pairs that earlier layers wrote for the same token position; the
 * shijienb.com article, first half, calls its kernel Flash Depth Attention).  It is the
 * MoDA definition with no sequence keys:
 *   y_j = scale * <q[b,h,t], kd[b,g,t,j]>  (j < L),  out = sum_j softmax(y)_j vd[b,g,t,j],
 *   lse = ln sum_j exp(y_j).
 * Arguments as moda_forward without k, v and causal; L >= 1 (MODA_ERR_INVALID_ARGUMENT
 * otherwise).  Same kernel as moda_forward with its sequence blocks removed.
 */
moda_status_t moda_depth_attention_forward(const void *q, const void *kd, const void *vd,
                                           void *out, float *lse, int B, int Hq, int Hkv,
                                           int T, int L, int d, float scale,
                                           moda_stream_t stream);

/*
 * Depth-only attention backward: dq (bf16), dkd, dvd (bf16) of moda_depth_attention_forward
 * given dout, from its out and lse.  Workspace as for moda_backward (size from
 * moda_backward_workspace_size with the same sizes).  L >= 1.  Two launches: the depth
 * part (row terms, dkd, dvd, fp32 dq) and the dq conversion; dq is deterministic here.
 */
moda_status_t moda_depth_attention_backward(const void *q, const void *kd, const void *vd,
                                            const void *out, const float *lse,
                                            const void *dout, void *dq, void *dkd, void *dvd,
                                            void *workspace, size_t workspace_bytes, int B,
                                            int Hq, int Hkv, int T, int L, int d, float scale,
                                            moda_stream_t stream);

/*
 * Single-token decode: the forward's row for the newest token of each sequence.  The
 * K/V cache holds S sequence keys/values, the last of them the newest token's own; its
 * query row sees all S of them (the causal row of position S-1) and its own L depth
 * keys, in one joint softmax (hyper.ai summary of arXiv 2603.15619, section
 * "Mixture-of-Depths Attention (MoDA)").  The pages do not describe decoding; this is
 * that definition restricted to one query token per sequence.
 *   q, out: [B, Hq, d]    k, v: [B, Hkv, S, d]    kd, vd: [B, Hkv, L, d] (NULL iff L == 0)
 *   lse: [B, Hq] fp32     workspace: >= moda_decode_workspace_size(...) bytes, 256-byte
 *   aligned, owned by the caller, contents irrelevant between calls.
 * Groups above 16 heads run the split launch once per 16 heads (each reading the cache
 * again).  The sequence is split over CTAs
 * (a function of the sizes only) and the partial softmax states are combined by a second
 * launch.  Other argument rules as moda_forward.
 */
size_t moda_decode_workspace_size(int B, int Hq, int Hkv, int S, int L, int d);
moda_status_t moda_decode(const void *q, const void *k, const void *v, const void *kd,
                          const void *vd, void *out, float *lse, void *workspace,
                          size_t workspace_bytes, int B, int Hq, int Hkv, int S, int L, int d,
                          float scale, moda_stream_t stream);

/*
 * Fused depth-stream write: the projection that produces a sublayer's depth key/value
 * pair, with the depth cache as its output (hyper.ai summary of arXiv 2603.15619,
 * section "Hardware-efficient implementation": every layer appends its K/V to the
 * depth stream, kept as [B, Hkv, T, L, d] so that token t's entries are contiguous).
 *   x:  [B, T, hidden] bf16 (the sublayer's input hidden states)
 *   w:  [2*Hkv*d, hidden] bf16 (rows 0..Hkv*d-1 project K, the rest V; nn.Linear layout)
 *   kd, vd: [B, Hkv, T, L, d] bf16; slot l of each receives
 *           kd[b,g,t,l,:] = (x[b,t,:] . w[g*d + c, :])_c,  vd likewise with rows Hkv*d + ...
 *           computed with fp32 accumulation and rounded to bf16; other slots are untouched.
 * Requirements: B, T, hidden, Hkv, L >= 1 and 0 <= slot < L; x, w, kd, vd non-NULL and
 * 16-byte aligned; kd and vd overlapping neither x, w nor each other
 * (MODA_ERR_INVALID_ARGUMENT otherwise).  d in {64, 128}, Hkv*d a multiple of 128,
 * hidden a multiple of 8 and B*T < 2^31 - 256 (MODA_ERR_UNSUPPORTED otherwise).  One tcgen05 GEMM launch; no
 * workspace.
 */
moda_status_t moda_depth_kv_write(const void *x, const void *w, void *kd, void *vd, int B,
                                  int T, int hidden, int Hkv, int d, int L, int slot,
                                  moda_stream_t stream);

/*
 * Bytes of device workspace moda_backward needs for these sizes (fp32 dQ accumulator
 * [B][Hq][T][d] plus the fp32 row terms: D = <dO, out> as [B][Hq][T] at d = 64, and at
 * d = 128 both -lse*log2(e) and -D per query tile of floor(128 / G) tokens, 1 KB per tile
 * and (batch, KV head); for groups Hq / Hkv above 16 also fp32 dkd and dvd accumulators,
 * 2 x [B][Hkv][T][L][d]).  0 for invalid sizes.
 */
size_t moda_backward_workspace_size(int B, int Hq, int Hkv, int T, int L, int d);

/*
 * Backward pass: gradients of sum(out * dout) w.r.t. q, k, v, kd, vd.  Recomputes the
 * softmax weights P = exp(scale*logit - lse) from the forward's lse, with
 * D = <dout, out> per row and dS = P * (<dout, value> - D):
 *   dq = scale * sum dS * key,  dk/dkd = scale * sum dS * q,  dv/dvd = sum P * dout.
 * The pages give no backward design; this is the exact gradient of the definition.
 * Groups above 16 heads run the depth part once per 16 heads, summing dkd and dvd in fp32
 * accumulators that the workspace then also holds.  dq is summed with fp32 atomics, and
 * dk and dv add the two 64-row halves of each query tile in the order their products
 * reach the tensor cores, so the last bits of dq, dk and dv may differ between runs;
 * dkd and dvd are deterministic.
 * `out` and `lse` must be the forward's outputs for the same inputs.  `workspace`
 * (device, >= moda_backward_workspace_size bytes, 256-byte aligned) is scratch owned
 * by the caller; its contents on entry do not matter.
 */
moda_status_t moda_backward(const void *q, const void *k, const void *v, const void *kd,
                            const void *vd, const void *out, const float *lse,
                            const void *dout, void *dq, void *dk, void *dv, void *dkd,
                            void *dvd, void *workspace, size_t workspace_bytes, int B,
                            int Hq, int Hkv, int T, int L, int d, float scale, int causal,
                            moda_stream_t stream);

/*
 * moda_backward split into its three launches, for callers that schedule or time them
 * separately.  `stages` is a non-empty bit mask:
 *   1  row terms D = <dout, out> (into the workspace), the depth gradients dkd and dvd,
 *      and the depth share of dq, which initialises the workspace's fp32 dq accumulator;
 *   2  the sequence part: dk and dv, plus the sequence share of dq added to the
 *      accumulator (needs stage 1's workspace contents);
 *   4  dq (bf16) from the accumulator (needs stages 1 and 2).
 * Running 1, 2 and 4 in that order on one stream (with the same arguments and workspace)
 * equals one moda_backward call; moda_backward is stages = 7.  Arguments, checks and
 * errors are moda_backward's; an invalid mask gives MODA_ERR_INVALID_ARGUMENT.
 */
moda_status_t moda_backward_stages(const void *q, const void *k, const void *v,
                                   const void *kd, const void *vd, const void *out,
                                   const float *lse, const void *dout, void *dq, void *dk,
                                   void *dv, void *dkd, void *dvd, void *workspace,
                                   size_t workspace_bytes, int B, int Hq, int Hkv, int T,
                                   int L, int d, float scale, int causal, unsigned stages,
                                   moda_stream_t stream);

/*
 * The backward of moda_backward for callers that cannot allocate device memory: those
 * whose device memory is owned by another allocator or by a fixed memory plan that hands
 * out only the tensors it planned, and those calling through a plain C binding with no
 * device allocation API.  (The paper has no counterpart; this is an interface addition.)
 *
 * Same arguments and results as moda_backward, without the workspace: the library takes
 * it from a static device array of 64 MiB that every GPU loading the library holds until
 * the process exits.  Neither the caller nor the library allocates anything.
 *   - Sizes whose moda_backward_workspace_size() exceeds 64 MiB are rejected with
 *     MODA_ERR_UNSUPPORTED (about B*Hq*T <= 128000 rows at d = 128).
 *   - Argument checks come first and need no device: a bad pointer or size is refused
 *     (MODA_ERR_INVALID_ARGUMENT, or MODA_ERR_UNSUPPORTED for sizes beyond 64 MiB)
 *     before anything touches the GPU.
 *   - The first call on a device (the calling thread's current device) looks up the
 *     array's device address with cudaGetSymbolAddress and caches it for the process;
 *     make that first call before any stream capture begins.  A cudaDeviceReset()
 *     between calls is not supported (the cached address would be stale).
 *   - Every call on a device shares the one array and leaves its contents behind.  The
 *     backward writes every workspace element it reads before reading it, so nothing has
 *     to be cleared between calls, but calls that may overlap on the GPU (different
 *     streams, or concurrent host threads) race on the array and must be serialised by
 *     the caller.
 */
moda_status_t moda_backward_noalloc(const void *q, const void *k, const void *v,
                                    const void *kd, const void *vd, const void *out,
                                    const float *lse, const void *dout, void *dq, void *dk,
                                    void *dv, void *dkd, void *dvd, int B, int Hq, int Hkv,
                                    int T, int L, int d, float scale, int causal,
                                    moda_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the calling device's kernel error word.
 * *flags (may be NULL) receives the raw bits: 1 = a bounded wait ran out, 2 = an
 * internal index/consistency check failed.  Returns MODA_ERR_TIMEOUT / MODA_ERR_INTERNAL
 * if the corresponding bit was set, MODA_ERR_CUDA if synchronisation failed, else MODA_OK.
 */
moda_status_t moda_check_device_errors(moda_stream_t stream, uint32_t *flags);

/*
 * TEST ONLY: exercises the kernels' failure detection without a real fault.  Sets, on the
 * calling thread's current device, the limit every bounded kernel wait uses and a fault
 * the kernels inject on purpose:
 *   fault 0  none (the normal state);
 *   fault 1  the forward kernel's TMA producer issues no loads, so every wait for that
 *            data runs out after wait_limit_ns: each CTA records the timeout in the
 *            device error word, lets the operations it has in flight finish, releases its
 *            tensor memory and exits (its out and lse are then meaningless), and
 *            moda_check_device_errors() returns MODA_ERR_TIMEOUT.
 * wait_limit_ns: 0 restores the default limit (2 s), otherwise 1e5..1e10 ns.  Call it
 * with no kernel of this library in flight on the device, and call it again with (0, 0)
 * afterwards.  MODA_ERR_INVALID_ARGUMENT for other values, MODA_ERR_CUDA or
 * MODA_ERR_UNSUPPORTED from the device check.  Not part of the paper's operator.
 */
moda_status_t moda_test_set_device_fault(int fault, uint64_t wait_limit_ns);

/*
 * TEST ONLY: y[i] = 2^x[i] for 0 <= i < n, computed by the forward kernel's FMA-pipe
 * exponential (the one that takes a quarter of the exponentials of unmasked sequence
 * blocks off the exponent unit, in the softmax of the fused kernel of the hyper.ai
 * summary of arXiv 2603.15619, section "Hardware-efficient implementation").  x and y:
 * device arrays of n
 * fp32 values, 4-byte aligned, owned by the caller; y may not overlap x.  Enqueued on
 * `stream`.  Accuracy: relative error at most 8e-5 for x in [-125, 8]; below -125 the
 * result is that of -125 (about 2.35e-38).  MODA_ERR_INVALID_ARGUMENT for n outside
 * [0, 2^30], NULL or misaligned pointers (checked before any CUDA call); MODA_ERR_CUDA
 * or MODA_ERR_UNSUPPORTED from the device check or the launch.  Not part of the paper's
 * operator.
 */
moda_status_t moda_test_exp2_fma(const float *x, float *y, int n, moda_stream_t stream);

/* Static English description of a status code.  Never NULL. */
const char *moda_status_string(moda_status_t status);

/* Description of the last failure on the calling host thread (or ""). Never NULL. */
const char *moda_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* MODA_H_ */
