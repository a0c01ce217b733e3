/*
 * kda_decode.h -- C ABI of the B200 (sm_100a) KDA layer-half decode step.
 *
 * One call advances a batch of sequences by one token through the
 * linear-attention ("KDA") half of a layer:
 *
 *   q, k, v   = W_q x, W_k x, W_v x      FP8 E4M3 weights, fp32 128x128 block scales
 *   beta_h    = sigmoid(W_b x)_h          bf16 weights [num_heads, hidden]
 *   alpha     = exp(-softplus(W_a_up W_a_down x))   bf16, low rank alpha_rank
 *   k^_h      = k_h / ||k_h||_2           (a zero k_h gives k^_h = 0)
 *   S_h      <- (I - beta_h k^ k^T) diag(alpha_h) S_h + beta_h k^ v_h^T
 *   o_h       = S_h^T q_h                 (read out after the update)
 *   out       = W_o concat_h(o_h)         FP8 E4M3, fp32 128x128 block scales
 *
 * Sources.  The layer and its fixed-size per-sequence recurrent state, updated
 * in place by one decode kernel, are named by the TrnRT listing ("The
 * interesting bit": linear attention with fixed-size state), the TrnRT story
 * ("KDA (linear attention)", one fused kernel per layer half whose working set
 * stays on chip so that only inputs, outputs and streamed weights cross HBM)
 * and the Kiln post ("The decode kernels, and why they are opt-in": KDA decode
 * as one kernel updating each sequence's recurrent state in place; "How was
 * Kiln measured": FP8 weights with 128 x 128 block scales; "Expert parallelism
 * without an all-to-all": one scale per kernel tile).  The pages print no
 * equations; the gated delta rule above is the decode benchmark's stated
 * workload, read with S_h stored dk x dv (key index first).
 *
 * Conventions for every entry point:
 *   - Return value: KDA_OK (0) or one of the KDA_ERR_* codes below.  No C++
 *     exception crosses this boundary.  kda_status_string() names a code and
 *     kda_decode_last_error() gives the handle's last detailed message.
 *   - Every tensor pointer is DEVICE memory owned by the caller (cudaMalloc,
 *     torch, ...) unless the name says _host.  All tensors are dense and
 *     row-major with the shapes given; base addresses must be 16-byte aligned.
 *   - Work is enqueued asynchronously on the handle's stream.  Errors found on
 *     the host (null or misaligned pointers, sizes) are returned before
 *     anything is enqueued.  A device-side bounded wait that gives up sets a
 *     status word that the next kda_decode_step / kda_decode_sync returns as
 *     KDA_ERR_DEVICE_TIMEOUT.  Steps enqueued after the one that timed out,
 *     before the error was returned, stop without doing their work: after
 *     KDA_ERR_DEVICE_TIMEOUT treat every step enqueued since the last
 *     successful kda_decode_sync as not run (outputs and state unwritten).
 *     If an aborted kernel also could not drain its own copies in flight, the
 *     handle is unusable: every later call on it returns
 *     KDA_ERR_DEVICE_TIMEOUT; destroy it and create a new one.
 *   - The handle belongs to the device that was current at kda_decode_init;
 *     that device must be current whenever the handle enqueues work (a call
 *     that would enqueue work on another current device returns
 *     KDA_ERR_INVALID_ARG and enqueues nothing).
 *   - There is no CPU fallback: without a usable sm_100 device every call
 *     fails with KDA_ERR_NO_DEVICE or KDA_ERR_CUDA.
 *   - A handle is not thread-safe; use one handle per stream.
 */
#ifndef KDA_DECODE_H_
#define KDA_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_DECODE_ABI_VERSION 1

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

/* status codes */
#define KDA_OK 0
#define KDA_ERR_INVALID_ARG 1       /* null / misaligned pointer, batch outside [1, max_batch], bad enum   */
#define KDA_ERR_UNSUPPORTED_SHAPE 2 /* dimensions the kernels do not cover (see kda_decode_init)           */
#define KDA_ERR_CUDA 3              /* a CUDA runtime call failed; kda_decode_last_error() has the text     */
#define KDA_ERR_DEVICE_TIMEOUT 4    /* a bounded device-side wait expired; outputs of that step are invalid */
#define KDA_ERR_NO_DEVICE 5         /* no CUDA device, or the current device is not sm_100                  */
#define KDA_ERR_OUT_OF_MEMORY 6     /* device scratch allocation failed                                     */

/* out dtypes */
#define KDA_OUT_F32 0  /* out is fp32 [B, hidden] (default)    */
#define KDA_OUT_BF16 1 /* out is bf16 [B, hidden], RNE rounded */

/* engines (kda_config.engine) */
#define KDA_ENGINE_AUTO 0   /* pick per shape and batch                                        */
#define KDA_ENGINE_SIMPLE 1 /* five plain CUDA-core kernels; the correctness baseline          */
#define KDA_ENGINE_FUSED 2  /* one persistent kernel: TMA weight stream + tcgen05 projections   */

typedef struct kda_config {
    int hidden;      /* H: model width; multiple of 128                                        */
    int num_heads;   /* nh                                                                     */
    int head_dk;     /* dk: key/query width per head; 64 or 128                                */
    int head_dv;     /* dv: value width per head; 64 or 128                                    */
    int alpha_rank;  /* r: inner width of the low-rank alpha projection; multiple of 16, <= 256 */
    int max_batch;   /* largest batch a step may pass; 1..256; sizes the handle's scratch      */
    int out_dtype;   /* KDA_OUT_F32 or KDA_OUT_BF16                                           */
    int engine;      /* KDA_ENGINE_*                                                          */
    int reserved[8]; /* must be zero                                                          */
} kda_config;

/*
 * Layer weights (device pointers, caller-owned, read-only for the library).
 * FP8 matrices are E4M3 ("fn": bias 7, no infinities) codes, row-major
 * [out_features, in_features]; the dequantised weight is
 *   W[i][j] = decode(code[i][j]) * scale[i / 128][j / 128]
 * with scale row-major [ceil(out/128), ceil(in/128)] fp32.
 * bf16 matrices are raw bf16 bit patterns, row-major [out, in].
 */
typedef struct kda_weights {
    const uint8_t *wq;       /* [nh*dk, H]  */
    const uint8_t *wk;       /* [nh*dk, H]  */
    const uint8_t *wv;       /* [nh*dv, H]  */
    const uint8_t *wo;       /* [H, nh*dv]  */
    const float *sq;         /* [nh*dk/128, H/128]  */
    const float *sk;         /* [nh*dk/128, H/128]  */
    const float *sv;         /* [nh*dv/128, H/128]  */
    const float *so;         /* [H/128, nh*dv/128]  */
    const uint16_t *wa_down; /* bf16 [r, H]      */
    const uint16_t *wa_up;   /* bf16 [nh*dk, r]  */
    const uint16_t *wb;      /* bf16 [nh, H]     */
} kda_weights;

typedef struct kda_handle_s *kda_handle;

/* Creates a handle on the CURRENT CUDA device.  Validates the shape
 * (hidden % 128 == 0, dk and dv in {64, 128}, nh*dk and nh*dv multiples of
 * 128, alpha_rank a multiple of 16 in [16, 256], 1 <= max_batch <= 256) and allocates the
 * handle's device scratch (activations between stages, a status word) with
 * cudaMalloc.  No weights are copied.  On failure *out_handle is set to NULL. */
KDA_API int kda_decode_init(const kda_config *cfg, kda_handle *out_handle);

/* Binds a cudaStream_t (passed as void*) for all later work; NULL = legacy default stream. */
KDA_API int kda_decode_set_stream(kda_handle h, void *cuda_stream);

/*
 * One decode step for `batch` sequences, enqueued on the handle's stream.
 *   x            bf16 [batch, H]                       hidden state of the new token
 *   w            weights as above (the struct itself is read on the host during the call)
 *   state_inout  fp32 [batch, nh, dk, dv]              recurrent state, updated in place
 *   out          [batch, H] fp32 or bf16 (cfg.out_dtype)
 * state_inout must not overlap x, out or the weights.  Rows >= batch of any
 * buffer are never read or written.  Returns KDA_ERR_DEVICE_TIMEOUT if an
 * earlier step recorded a device-side timeout (the status is then cleared).
 */
KDA_API int kda_decode_step(kda_handle h, const void *x, const kda_weights *w, float *state_inout, void *out, int batch);

/*
 * Same step with x and out in HOST memory (pinned memory gives asynchronous
 * copies): copies x to the handle's device staging buffer, runs the step and
 * copies out back, all on the handle's stream, then waits for the stream.
 * The weights and the state stay in device memory.
 */
KDA_API int kda_decode_step_host(kda_handle h, const void *x_host, const kda_weights *w, float *state_inout,
                         void *out_host, int batch);

/*
 * The same step from host buffers, without waiting: for a loop that feeds steps from the
 * host and reads every result.  x is copied in and out is copied back on two copy streams of
 * the handle (created with two device staging slots on the first call), so the copies of one
 * step overlap the neighbouring steps' kernels; the steps themselves stay in order on the
 * handle's stream.  x_host and out_host should be page-locked (pageable memory makes the
 * copies synchronous).  x_host may be reused, and out_host read, only after kda_decode_sync(h),
 * which waits for all of the handle's streams.  Same arguments and errors as kda_decode_step_host, plus
 * KDA_ERR_OUT_OF_MEMORY if the staging cannot be allocated.
 */
KDA_API int kda_decode_step_host_async(kda_handle h, const void *x_host, const kda_weights *w, float *state_inout,
                                       void *out_host, int batch);

/*
 * Several tokens per sequence in one call: `tokens` consecutive tokens of each of `batch`
 * sequences, as in the verify step of multi-token (speculative) decoding that the Kiln post
 * ("What did we measure that did not pay?") and the TileRT README (MTP) describe.
 *   x            bf16 [batch * tokens, H]; row b * tokens + t is token t of sequence b
 *   state_inout  fp32 [batch, nh, dk, dv]; advanced by `tokens` steps, token by token
 *   out          [batch * tokens, H] (cfg.out_dtype); row b * tokens + t is the output of
 *                token t, read out after token t's update
 * The projections read the weights once for all batch * tokens rows.  Requires
 * tokens >= 1 and batch * tokens <= max_batch.  tokens == 1 is kda_decode_step.  With up
 * to 8 tokens and batch * tokens <= 64 rows the fused engine runs the step as one kernel:
 * each of its state units keeps its sequence's state in registers and applies the tokens in
 * order.  Otherwise (or with KDA_ENGINE_SIMPLE) the five-kernel engine runs it, with one
 * state kernel that applies the tokens in order; its result then equals `tokens` successive
 * kda_decode_step calls on that engine bit for bit.  kda_decode_tokens_engine says which
 * engine a (batch, tokens) step uses.  Same errors and ordering as kda_decode_step.
 */
KDA_API int kda_decode_step_tokens(kda_handle h, const void *x, const kda_weights *w, float *state_inout, void *out,
                                   int batch, int tokens);

/*
 * Prefill: `tokens` consecutive tokens of each of `batch` sequences (a prompt), through the
 * chunked form of the recurrence -- the parallel-in-time prefill form that the Kiln post names
 * among its KDA kernels ("What moved the number...", "The token mixers' collectives...").
 *   x            bf16 [batch * tokens, H]; row b * tokens + t is token t of sequence b
 *   state_inout  fp32 [batch, nh, dk, dv]; advanced by all `tokens` tokens
 *   out          [batch * tokens, H] (cfg.out_dtype); row b * tokens + t is the output of
 *                token t, read out after token t's update
 *   chunk        tokens per chunk: 16, 32 or 64 (0: 32)
 * Each head's state goes through the tokens `chunk` at a time: inside a chunk the tokens'
 * updates are one unit lower-triangular system and dense products (decays taken in log space,
 * log alpha clamped at -30).  Two kernels: the first prepares every chunk of every head at
 * once (normalised keys, decays, the inverse of the chunk's triangular matrix); the second
 * walks the chunks in order, one CTA per sequence, head and slice of value columns.  The
 * projections are bf16 tensor-core GEMMs (cuBLASLt): each FP8 weight, scaled by its block
 * scale, is split into two bf16 parts (hi + lo, about 2^-17 of the weight), as are the fp32
 * activations o and t, so the products keep fp32-level accuracy.  batch and tokens are not
 * limited by max_batch: the handle keeps a workspace (the activations of batch * tokens rows,
 * the bf16 splits of the weights, one record per chunk), allocated (cudaMalloc; waiting for the
 * device when it grows) on the first call that needs it and freed by kda_decode_destroy.
 * Same errors and stream ordering as kda_decode_step; KDA_ERR_OUT_OF_MEMORY if the workspace
 * cannot grow; a record copy that does not land within the wait limit is reported as
 * KDA_ERR_DEVICE_TIMEOUT by the next call or kda_decode_sync.
 */
KDA_API int kda_prefill(kda_handle h, const void *x, const kda_weights *w, float *state_inout, void *out, int batch,
                        int tokens, int chunk);

/*
 * Recurrent-state checkpoint and restore (the Kiln post's prefix cache keeps checkpoints of
 * linear-attention state in a host tier: "What is Kiln?"; its "What could only a device
 * show?" is the lesson that such a copy must be ordered behind the queued work).  Both are
 * enqueued on the handle's stream, after every step enqueued before them and before every
 * step enqueued after them, so a checkpoint holds exactly the state those steps produced
 * and a restore is what the next step reads.
 *   state     device fp32 [*, nh, dk, dv] (the state_inout of the steps)
 *   seq0, nseq  sequences [seq0, seq0 + nseq): seq0 >= 0, nseq >= 1, seq0 + nseq <=
 *               max_batch, and inside the caller's state buffer
 *   host      host memory of nseq * nh * dk * dv * 4 bytes, sequence-major (page-locked
 *             memory makes the copy asynchronous; pageable memory makes the call wait)
 * The host buffer must not be read (checkpoint) or reused (restore) before the stream has
 * passed the copy: kda_decode_sync(h) or any later wait on the stream.
 */
KDA_API int kda_state_checkpoint(kda_handle h, const float *state, int seq0, int nseq, void *host_dst);
KDA_API int kda_state_restore(kda_handle h, const void *host_src, float *state, int seq0, int nseq);

/*
 * Launch overlap between consecutive steps (on by default).  A fused-engine step is
 * launched with programmatic stream serialization: its kernel may start on the SMs the
 * kernel enqueued just before it frees, and there, before that kernel has finished, it
 * already streams the first weight tiles of the step into shared memory.  It touches x,
 * the state and its scratch only after the preceding kernel has completed, so only the
 * weights are read early: a kernel that WRITES a step's weights must not be enqueued on the
 * stream immediately before that step while the overlap is on.  on = 0 restores strict
 * stream order (the step then also uses a cooperative launch, which makes the runtime check
 * that every CTA of the step can be resident at once).  Applies to later steps.
 */
KDA_API int kda_decode_set_launch_overlap(kda_handle h, int on);

/*
 * Tensor parallelism by heads with the out all-reduce inside the fused kernel.
 *
 * The TrnRT story runs decode tensor-parallel and folds each collective that would block the
 * next kernel into the kernel itself (its third rule).  For this layer half a head split
 * needs one exchange: rank g of `world` holds the rows of W_q, W_k, W_v, W_a_up and W_b for
 * its heads, their state, the matching column block of W_o and a whole W_a_down, and its
 * step forms the partial out = W_o[:, its heads] o; the layer's out is the sum over ranks.
 * Configured handles do that sum in the step's own kernel: as soon as a block of 32 output
 * rows is final, each rank stores its partial rows into every rank's exchange region over
 * peer memory (NVLink), raises that block's flag there (release, system scope), and then
 * adds the ranks' partials in rank order, so every rank writes the same out bits.  Each
 * rank's handle is created with its own shard's shape (num_heads = heads per rank).
 *
 * kda_tp_configure(h, rank, world, handle_out): allocates this rank's exchange region on
 *   the handle's device (2 x world x max_batch x hidden fp32 partials and 2 x world x
 *   hidden / 32 flags; two parities so that a step never overwrites rows a peer may still
 *   read) and writes its CUDA IPC handle (KDA_TP_HANDLE_BYTES bytes) to handle_out when
 *   world > 1 (handle_out may be NULL when world = 1).  1 <= world <= 8, 0 <= rank < world.
 *   Needs the fused engine (KDA_ERR_UNSUPPORTED_SHAPE otherwise); a handle is configured
 *   once (KDA_ERR_INVALID_ARG on a second call).
 * kda_tp_set_peer(h, peer, handle): maps rank `peer`'s exchange region from the handle that
 *   rank's kda_tp_configure wrote (cudaIpcOpenMemHandle; the two devices must have peer
 *   access).  Steps return KDA_ERR_INVALID_ARG until every peer is mapped.
 * After configuration every step of the handle (kda_decode_step, kda_decode_step_tokens)
 *   returns the whole out, and must take the fused engine (KDA_ERR_UNSUPPORTED_SHAPE, with
 *   nothing enqueued, for a batch it does not cover).  kda_prefill is not a step of the
 *   group: on a configured handle it still returns this rank's partial out (its heads' share),
 *   which the caller sums over the ranks (a prompt's out is large and leaves the kernel anyway).  All ranks must issue the same steps
 *   in the same order: a step's kernel waits (bounded by the handle's timeout) for the
 *   matching step of every peer.  A timed-out wait leaves the group out of step; destroy
 *   and recreate the handles of every rank.  The regions are freed (peers unmapped) by
 *   kda_decode_destroy.
 */
#define KDA_TP_HANDLE_BYTES 64
KDA_API int kda_tp_configure(kda_handle h, int rank, int world, void *handle_out);
KDA_API int kda_tp_set_peer(kda_handle h, int peer, const void *handle);

/* Waits for the handle's stream (and its copy streams, if kda_decode_step_host_async made them);
 * returns the device status of the steps since the last check (KDA_OK or
 * KDA_ERR_DEVICE_TIMEOUT) and clears it. */
KDA_API int kda_decode_sync(kda_handle h);

/* Frees the handle's scratch.  Waits for its stream first.  NULL is accepted. */
KDA_API int kda_decode_destroy(kda_handle h);

/* Engine the handle runs for `batch` (KDA_ENGINE_SIMPLE or KDA_ENGINE_FUSED). */
KDA_API int kda_decode_engine(kda_handle h, int batch);

/* Engine a kda_decode_step_tokens(batch, tokens) call runs (negative on bad arguments). */
KDA_API int kda_decode_tokens_engine(kda_handle h, int batch, int tokens);

/* Number of kernels one kda_decode_step(batch) launches. */
KDA_API int kda_decode_launches_per_step(kda_handle h, int batch);

/* Bytes of device scratch kda_decode_init allocates for cfg (host-only query). */
KDA_API int kda_decode_scratch_bytes(const kda_config *cfg, size_t *bytes);

/* Static name of a status code ("KDA_OK", ...); never NULL. */
KDA_API const char *kda_status_string(int status);

/* Last detailed error message recorded on the handle (empty string if none); never NULL. */
KDA_API const char *kda_decode_last_error(kda_handle h);

/* Intermediates of the most recent step, for stage-by-stage diagnosis (which =):      */
#define KDA_DEBUG_Q 0        /* fp32 [batch, nh*dk]  q = W_q x                            */
#define KDA_DEBUG_K 1        /* fp32 [batch, nh*dk]  k = W_k x (before normalisation)     */
#define KDA_DEBUG_V 2        /* fp32 [batch, nh*dv]  v = W_v x                            */
#define KDA_DEBUG_BETA_PRE 3 /* fp32 [batch, nh]     W_b x (before the sigmoid)           */
#define KDA_DEBUG_T 4        /* fp32 [batch, r]      W_a_down x                           */
#define KDA_DEBUG_TRACE 5    /* uint64 [num_SMs][32] fused-kernel timeline stamps (ns); only in
                                libraries built with -DKDA_TRACE, else KDA_ERR_INVALID_ARG */

/* Copies `bytes` of intermediate `which` of the last step into device buffer `dst`,
 * ordered on the handle's stream (bytes must not exceed the tensor's size at max_batch). */
KDA_API int kda_decode_debug_copy(kda_handle h, int which, void *dst, size_t bytes);

/* KDA_DECODE_ABI_VERSION of the loaded library. */
KDA_API int kda_decode_abi_version(void);

/*
 * kda_decode_step_noalloc -- the same decode step for callers that may not
 * allocate device memory.  The pages describe no such entry point; it is a
 * deployment convenience of this library.  It serves runtimes that own all
 * device memory themselves (a pre-reserved pool that no library may grow) and
 * serving loops that cannot afford the implicit device synchronisation of
 * cudaMalloc / cudaFree.  It takes no handle and allocates no device memory
 * (it calls no cudaMalloc, cudaFree or allocating library).
 *
 * It runs the five-kernel (KDA_ENGINE_SIMPLE) path, whatever cfg->engine says,
 * with its fp32 activations in one file-scope device array of
 * KDA_NOALLOC_MAX_SCRATCH_BYTES per device.  The activations of `batch`
 * sequences take batch * (3 nh dk + 2 nh dv + nh + r) * 4 bytes, each of the
 * seven arrays rounded up to 256 bytes; a step that needs more is rejected
 * with KDA_ERR_UNSUPPORTED_SHAPE before anything is enqueued (for example
 * batch 12 at hidden 4096, 32 heads of 128 x 128, r 64 fits; batch 64 at
 * 48 heads of 128 x 128 does not).  Every stage writes its whole output
 * before the next reads it, so nothing in the array needs to start at zero
 * and nothing is cleared.
 *
 *   cfg          shape and out dtype as for kda_decode_init (validated the
 *                same way; max_batch and engine are ignored, not checked)
 *   x, w, state_inout, out   as for kda_decode_step (device memory)
 *   batch        1 .. any, within the scratch limit above
 *   cuda_stream  cudaStream_t passed as void* (NULL = legacy default stream)
 *
 * Set-up: the first call in each CUDA context (normally a device's primary
 * context, bound with cudaSetDevice), with that context current, looks up the
 * array's device address (cudaGetSymbolAddress, which may also load the
 * library's device code on that device) and caches it under the context;
 * later calls only read the cache.  Make that first call before any stream
 * capture begins.
 *
 * All calls on one device share the one array: two calls that can run at the
 * same time (on different streams, or from host threads without ordering)
 * race on it and corrupt each other's activations.  Order them (one stream,
 * or events).  The set-up itself is thread-safe.  The cached address belongs to
 * the context of the set-up: once that context is destroyed (cudaDeviceReset,
 * cuCtxDestroy) the entry is stale, and this entry point must not be called
 * again in the process.
 */
#define KDA_NOALLOC_MAX_SCRATCH_BYTES (1u << 20)
KDA_API int kda_decode_step_noalloc(const kda_config *cfg, const void *x, const kda_weights *w, float *state_inout,
                                    void *out, int batch, void *cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_DECODE_H_ */
