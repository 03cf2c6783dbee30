/*
 * dm05_suffix_attn.h -- C ABI of the B200 (sm_100a) suffix attention of the
 * DM0.5 action expert.
 *
 * The operation (page "TensorRT+Triton+FlexAttention: OpenDM VLA
 * 快速推理加速栈深度剖析", section 2.2 "Triton 大 Kernel"): the action-chunk
 * queries attend at once over the prefix KV cache and over the suffix's own
 * K/V, under the prefix-visibility mask, with a softmax and a value-weighted
 * sum.  The same section's shape table gives head_dim 256 and 8 query heads
 * over 4 KV heads (GQA).  The prefix cache is padded to a length bucket
 * (same page, section 3; page "DM05 推理指南", section "Fast Backend 约束"),
 * so each sample carries a valid prefix length.
 *
 * For every sample b, query head h (KV head g = h / (Hq / Hkv)) and suffix
 * query i:
 *   visible keys  = prefix rows j with j < clamp(prefix_valid_len[b], 0, P)
 *                   and (prefix_mask == NULL or prefix_mask[b*P + j] != 0),
 *                   plus every suffix row k < S (suffix keys are visible to
 *                   every suffix query);
 *   logit(x)      = <q[b,h,i,:], K_x> / sqrt(D);
 *   lse[b,h,i]    = ln sum_x exp(logit(x))           (natural log, fp32);
 *   out[b,h,i,:]  = sum_x exp(logit(x) - lse) V_x     (rounded once to bf16).
 *
 * Layouts: every tensor is dense, row-major, with the last dimension
 * contiguous.  All device pointers are addresses in the memory of the CUDA
 * device that is current on the calling thread.
 *
 * Ownership: the caller owns every tensor.  The library keeps no pointer
 * after a call returns.  The library owns an error word per device and, per
 * (device, stream), a workspace for the partial results of split calls (at
 * most dm05_suffix_attn_workspace_bytes); for the handle cudaStreamPerThread
 * the calling thread is part of the key, since that handle names a different
 * stream on every thread.  They are created by
 * dm05_suffix_attn_reserve or by a dm05_suffix_attn that runs outside stream
 * capture, grow only outside capture, and are freed by dm05_release.
 *
 * Errors: every entry point returns a dm05_status.  Arguments are checked on
 * the host before anything is launched; a failed check launches nothing.
 * Nothing on the success path synchronises the host.
 */
#ifndef DM05_SUFFIX_ATTN_H
#define DM05_SUFFIX_ATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DM05_OK = 0,
    DM05_ERR_NULL = -1,        /* a required pointer is NULL */
    DM05_ERR_SHAPE = -2,       /* B, Hq, Hkv, S < 1, P < 0, Hq % Hkv != 0, or sizes too large */
    DM05_ERR_UNSUPPORTED = -3, /* D != 256, or (Hq/Hkv)*S > 128 */
    DM05_ERR_ALIGN = -4,       /* a bf16 tensor base is not 16-byte aligned */
    DM05_ERR_WORKSPACE = -5,   /* no workspace on this device and the stream is capturing */
    DM05_ERR_CUDA = -6         /* a CUDA call failed (launch, attribute, allocation) */
} dm05_status;

/* Bits of the device error word (dm05_get_error_word). */
#define DM05_EW_VALID_LEN_CLAMPED 0x1u /* a prefix_valid_len value was outside [0, P] and was clamped */
#define DM05_EW_WAIT_TIMEOUT      0x2u /* a kernel wait gave up after its time limit; outputs invalid */
#define DM05_EW_BAD_SPLIT         0x4u /* a kernel was launched with a split count it cannot merge (the
                                          host never does this); outputs invalid */

/*
 * dm05_suffix_attn -- one suffix-attention call, asynchronous on `stream`.
 *
 *   q                 bf16  [B, Hq, S, D]    suffix queries
 *   k_prefix          bf16  [B, Hkv, P, D]   bucket-padded prefix key cache (NULL allowed iff P == 0)
 *   v_prefix          bf16  [B, Hkv, P, D]   prefix value cache              (NULL allowed iff P == 0)
 *   prefix_valid_len  int32 [B]     device; NULL = every prefix row is in range.  Values
 *                                   outside [0, P] are clamped and flagged in the error word.
 *   prefix_mask       uint8 [B, P]  device; 1 = visible, 0 = hidden; NULL = no extra mask.
 *   k_suffix          bf16  [B, Hkv, S, D]   suffix keys
 *   v_suffix          bf16  [B, Hkv, S, D]   suffix values
 *   out               bf16  [B, Hq, S, D]    result (written)
 *   lse               fp32  [B, Hq, S]       natural-log LSE of the scaled logits; NULL = not written
 *   B, Hq, Hkv, P, S, D  sizes; query head h reads KV head h / (Hq / Hkv).
 *   stream            CUDA stream (0 = legacy default stream).
 *
 * Supported: D == 256 and (Hq / Hkv) * S <= 128; P >= 0.  Bases of q,
 * k_prefix, v_prefix, k_suffix, v_suffix and out must be 16-byte aligned.
 * Prefix rows at or past the valid length are never used: they may hold any
 * bits, NaN included.  Hidden rows inside the valid range must hold finite
 * values (they are multiplied by an exact zero weight).
 *
 * The call is deterministic for fixed inputs and sizes, does not
 * synchronise, and may be captured into a CUDA graph once the device has a
 * workspace (dm05_suffix_attn_reserve).  Consecutive calls on one stream may
 * overlap their start-up with the previous kernel (programmatic dependent
 * launch); each call still waits for all earlier work on the stream before
 * it reads an input or writes an output.
 */
int dm05_suffix_attn(const void *q, const void *k_prefix, const void *v_prefix,
                     const int32_t *prefix_valid_len, const uint8_t *prefix_mask,
                     const void *k_suffix, const void *v_suffix,
                     void *out, float *lse,
                     int B, int Hq, int Hkv, int P, int S, int D,
                     cudaStream_t stream);

/*
 * dm05_suffix_attn_ex -- dm05_suffix_attn with option flags (0 gives exactly
 * dm05_suffix_attn).  Unknown bits return DM05_ERR_SHAPE.
 *
 * DM05_FLAG_PREFIX_STATIC: the caller promises that the kernel launched
 * right before this call on `stream` writes none of k_prefix, v_prefix,
 * prefix_valid_len and prefix_mask (they were written earlier, as the pages'
 * static, address-stable prefix KV cache is: page "TensorRT+Triton+
 * FlexAttention: OpenDM VLA 快速推理加速栈深度剖析", section 3, where the cache
 * is filled by the prefix graph and then read, unchanged, by every suffix
 * step).  The call may then start reading them while that kernel is still
 * running (programmatic dependent launch); q, k_suffix, v_suffix and the
 * outputs are still ordered after it.  Breaking the promise gives wrong
 * results.
 */
#define DM05_FLAG_PREFIX_STATIC 0x1u
int dm05_suffix_attn_ex(const void *q, const void *k_prefix, const void *v_prefix,
                        const int32_t *prefix_valid_len, const uint8_t *prefix_mask,
                        const void *k_suffix, const void *v_suffix,
                        void *out, float *lse,
                        int B, int Hq, int Hkv, int P, int S, int D, unsigned flags,
                        cudaStream_t stream);

/*
 * Multi-step calls -- N suffix-attention calls over one prefix cache, run by
 * one launch.  The pages' runtime captures the suffix-decode step of every
 * prefix-length bucket into a CUDA graph at start-up and replays it per
 * request, for the diffusion_steps denoising steps (page "TensorRT+Triton+
 * FlexAttention: OpenDM VLA 快速推理加速栈深度剖析", section 3; page "DM05
 * 推理指南", section 6: diffusion_steps defaults to 10 and is fixed after
 * capture); every step reads the same, unchanged prefix cache.
 *
 * dm05_suffix_attn_steps_create captures n_steps calls, in order, each one
 * exactly a dm05_suffix_attn_ex call with the shared prefix arguments and its
 * own dm05_step, into a CUDA graph owned by the returned handle (with its own
 * workspace for split partial results).  Consecutive calls are ordered as on
 * one stream: call t + 1 reads its inputs only after call t has written its
 * outputs, so a step's q may be an earlier step's out.  With
 * DM05_FLAG_PREFIX_STATIC every call may request its prefix tiles while the
 * previous call finishes (the prefix arguments must not be written by any
 * step).  The pointers are baked into the graph: every launch reads and
 * writes the same buffers.  Create outside any stream capture; the device
 * current at creation must be current at every launch.
 *
 * dm05_suffix_attn_steps_launch enqueues all n_steps calls on `stream` with
 * one graph launch (asynchronous).  Launches of one handle must not overlap
 * on the GPU (they share its workspace).
 *
 * dm05_suffix_attn_steps_destroy waits for the device and frees the handle.
 */
typedef struct {
    const void *q;        /* bf16 [B, Hq, S, D] */
    const void *k_suffix; /* bf16 [B, Hkv, S, D] */
    const void *v_suffix; /* bf16 [B, Hkv, S, D] */
    void *out;            /* bf16 [B, Hq, S, D] */
    float *lse;           /* fp32 [B, Hq, S] or NULL */
} dm05_step;
typedef struct dm05_steps_s *dm05_steps_handle;
int dm05_suffix_attn_steps_create(const dm05_step *steps, int n_steps, const void *k_prefix, const void *v_prefix,
                                  const int32_t *prefix_valid_len, const uint8_t *prefix_mask,
                                  int B, int Hq, int Hkv, int P, int S, int D, unsigned flags,
                                  dm05_steps_handle *handle);
int dm05_suffix_attn_steps_launch(dm05_steps_handle handle, cudaStream_t stream);
int dm05_suffix_attn_steps_destroy(dm05_steps_handle handle);

/* Upper bound of the device workspace dm05_suffix_attn uses for these sizes:
 * the error word plus the partial results of the largest split (16 CTAs per
 * (sample, KV head)).  0 if the sizes are invalid.
 *
 * The pages' fast path preallocates its work buffers once
 * (DM05BigKernelBuffers, page "TensorRT+Triton+FlexAttention: OpenDM VLA
 * 快速推理加速栈深度剖析", section 2.2) so that no request allocates device
 * memory; this call tells a caller how much this library's equivalent needs. */
size_t dm05_suffix_attn_workspace_bytes(int B, int Hq, int Hkv, int P, int S, int D);

/* Creates the workspace of (current device, `stream`) for these sizes and
 * sets the kernel attributes, outside any stream capture.  Call it before
 * capturing dm05_suffix_attn on `stream` into a CUDA graph.  `stream` must not
 * be capturing.
 *
 * This is the step the pages take at start-up: the prefix KV cache has a
 * static address and every bucket's graph is captured once, then replayed
 * per request (same page, section 3).  A graph captured after this call
 * stays valid while the workspace lives (until dm05_release). */
int dm05_suffix_attn_reserve(int B, int Hq, int Hkv, int P, int S, int D, cudaStream_t stream);

/* Work decomposition the next call with these sizes will use: the number of
 * CTAs (one thread-block cluster) per (sample, KV head, query block), the key
 * rows per tile, and the number of query blocks each (sample, KV head)'s S
 * queries are cut into.  Any output pointer may be NULL. */
int dm05_suffix_attn_plan(int B, int Hq, int Hkv, int P, int S, int D,
                          int *splits_per_head, int *tile_rows, int *row_blocks);

/* Forces the number of CTAs per (sample, KV head) for later calls on this
 * process: 1 to 16; 0 restores the automatic choice.  For tuning and tests.
 * Returns DM05_ERR_SHAPE for any other value. */
int dm05_set_split_override(int splits_per_head);

/* Forces the number of query blocks each (sample, KV head)'s S queries are
 * cut into, for later split calls on this process: 1 to 16; 0 restores the
 * automatic choice.  Blocks hold ceil(S / row_blocks) queries per head (the
 * last one fewer), at least 8, and (Hq/Hkv) * (block rounded up to 8) <= 128
 * rows; a count that breaks this, that another count already gives the same
 * blocks, or a call that runs unsplit, uses one block.  dm05_suffix_attn_plan
 * reports what a call will use.  For tuning and tests.  Returns
 * DM05_ERR_SHAPE for any other value. */
int dm05_set_row_block_override(int row_blocks);

/*
 * dm05_prefix_prefill_attn -- the prefix stage's attention under the
 * prefix-causal mask, asynchronous on `stream`.
 *
 * The operation (page "TensorRT+Triton+FlexAttention: OpenDM VLA
 * 快速推理加速栈深度剖析", section 2.3 "FlexAttention"): the prefix stage runs
 * its attention with a custom causal mask mapping
 * (_make_prefix_causal_mask_mapping), with the prefix decoder's 8 / 4 GQA
 * heads and head_dim 256 (section 2.2 shape table).  The queries are the P
 * prefix positions, the keys and values the prefix K/V of the same call (the
 * tensors that then form the prefix KV cache read by dm05_suffix_attn).  For
 * sample b, query head h (KV head h / (Hq / Hkv)) and prefix position
 * i < clamp(valid_len[b], 0, P):
 *   visible keys  = prefix positions j <= i   (causal; j < valid length follows);
 *   lse[b,h,i]    = ln sum_j exp(<q[b,h,i,:], k[b,g,j,:]> / sqrt(D));
 *   out[b,h,i,:]  = sum_j exp(logit(j) - lse) v[b,g,j,:]   (rounded once to bf16).
 * Positions i at or past the valid length are bucket padding: their out and
 * lse rows are not written.
 *
 *   q          bf16  [B, Hq, P, D]
 *   k, v       bf16  [B, Hkv, P, D]
 *   valid_len  int32 [B]  device; NULL = every position in range; values
 *                         outside [0, P] are clamped and flagged in the error word
 *   out        bf16  [B, Hq, P, D]   (rows < valid length written)
 *   lse        fp32  [B, Hq, P]      (rows < valid length written); NULL = not written
 *
 * Supported: D == 256 and (Hq / Hkv) * 8 <= 128; P >= 1; 16-byte aligned
 * bases.  Workspace, capture, errors and determinism as in dm05_suffix_attn;
 * the same per-(device, stream) workspace serves both calls.  Before
 * capturing this call into a CUDA graph, create it with
 * dm05_prefix_prefill_reserve.
 */
int dm05_prefix_prefill_attn(const void *q, const void *k, const void *v, const int32_t *valid_len,
                             void *out, float *lse, int B, int Hq, int Hkv, int P, int D,
                             cudaStream_t stream);

/* Creates the workspace of (current device, `stream`) that a
 * dm05_prefix_prefill_attn call with these sizes needs, outside any stream
 * capture (as dm05_suffix_attn_reserve does for the suffix call). */
int dm05_prefix_prefill_reserve(int B, int Hq, int Hkv, int P, int D, cudaStream_t stream);

/* Work plan of a dm05_prefix_prefill_attn call with these sizes: CTAs per
 * (sample, KV head, query block), query positions per head in a block, and
 * the number of blocks.  Any output pointer may be NULL. */
int dm05_prefix_prefill_plan(int B, int Hq, int Hkv, int P, int D, int *splits_per_head, int *query_block,
                             int *row_blocks);

/*
 * dm05_suffix_qkv_prologue -- the step right before the suffix attention:
 * QKV projection, QK-Norm and RoPE of the action tokens in one kernel,
 * asynchronous on `stream`.
 *
 * The operation (page "TensorRT+Triton+FlexAttention: OpenDM VLA
 * 快速推理加速栈深度剖析", section 2.2: "QKV projection + QK-Norm + RoPE done
 * at once" is one of the fused steps; the action expert's shape table gives
 * hidden 1024, head_dim 256, 8 / 4 heads).  For token t = b * S + i and head
 * hd of w's row order (Hq query heads, then Hkv key heads, then Hkv value
 * heads):
 *   y        = w[hd*D : (hd+1)*D, :] x[t, :]                         (fp32 accumulation)
 *   query / key heads: y' = y / sqrt(mean(y^2) + eps) * nw  (nw = q_norm_w or k_norm_w),
 *                      then RoPE in the rotate-half pairing (d, d + D/2) by the
 *                      angle positions[t] * theta^(-2d/D);
 *   value heads: the projection y unchanged;
 * written (rounded once to bf16) to q [B,Hq,S,D], k [B,Hkv,S,D], v [B,Hkv,S,D]:
 * exactly the q / k_suffix / v_suffix layout dm05_suffix_attn reads.
 *
 *   x          bf16  [B*S, H]                  hidden states of the action tokens
 *   w          bf16  [(Hq + 2*Hkv) * D, H]     QKV weight (row-major)
 *   q_norm_w, k_norm_w  bf16 [D]               QK-Norm weights
 *   positions  int32 [B*S]                     RoPE position of each token (the angle is
 *                                              accurate to ~1e-6 rad for positions in
 *                                              [0, 65536); larger ones lose precision)
 *   q, k, v    bf16  outputs as above
 *   eps > 0, theta > 1                          norm epsilon and RoPE base
 *
 * Supported: D == 256, H a multiple of 64.  x, w, q, k, v 16-byte aligned,
 * the norm weights 2-byte and positions 4-byte aligned.  Errors, capture
 * and determinism as dm05_suffix_attn (the first call on a device creates
 * the error word and must run outside stream capture).
 */
int dm05_suffix_qkv_prologue(const void *x, const void *w, const void *q_norm_w, const void *k_norm_w,
                             const int32_t *positions, void *q, void *k, void *v,
                             int B, int S, int H, int Hq, int Hkv, int D, float eps, float theta,
                             cudaStream_t stream);

/*
 * dm05_post_attention -- the step right after the suffix attention in an
 * action-expert layer: output projection + residual, Adarms time
 * modulation, GEGLU gate-up, MLP down + gated residual; asynchronous on
 * `stream` (five kernel launches).
 *
 * The operation (page "TensorRT+Triton+FlexAttention: OpenDM VLA
 * 快速推理加速栈深度剖析", section 2.2: after the three attention stages the
 * suffix path chains the time modulation Adarms, the GEGLU gate-up and the
 * MLP down; hidden 1024, intermediate 4096).  For token t = b * S + i:
 *   a_t  = the attention output of the token, its Hq heads concatenated (Hq * D)
 *   h1   = h[t] + wo a_t
 *   u    = h1 / sqrt(mean(h1^2) + eps) * (1 + scale[b]) + shift[b]
 *   m    = gelu_tanh(wgu[0:F] u) * (wgu[F:2F] u)
 *   out[t] = h1 + gate[b] * (wd m)              (rounded once to bf16)
 * gelu_tanh(z) = z / 2 (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))).
 *
 *   attn   bf16 [B, Hq, S, D]   the suffix attention's output (its `out`)
 *   h      bf16 [B*S, Hd]       residual stream entering the layer
 *   scale, shift, gate  bf16 [B, Hd]   time modulation of each sample
 *   wo     bf16 [Hd, Hq*D], wgu bf16 [2F, Hd] (gate rows, then up rows),
 *   wd     bf16 [Hd, F]
 *   out    bf16 [B*S, Hd]
 *
 * Supported: D and F multiples of 64, Hd a multiple of 128.  attn, h, the
 * weights and out 16-byte aligned; scale, shift, gate 8-byte aligned.  The
 * intermediates (h1 fp32, u and m bf16, and fp32 split-K partial sums) live
 * in a library workspace per (device, stream), created by the first call
 * outside stream capture or by dm05_post_attention_reserve (call it before
 * capturing); results are deterministic (the split-K partial sums are added
 * in a fixed order).  Errors as dm05_suffix_attn.
 */
int dm05_post_attention(const void *attn, const void *h, const void *scale, const void *shift, const void *gate,
                        const void *wo, const void *wgu, const void *wd, void *out,
                        int B, int S, int Hq, int D, int Hd, int F, float eps, cudaStream_t stream);
int dm05_post_attention_reserve(int B, int S, int Hq, int D, int Hd, int F, cudaStream_t stream);

/*
 * dm05_suffix_attn_noalloc -- the same attention as dm05_suffix_attn, for
 * callers that must not allocate device memory.  The source pages have no
 * counterpart of this entry point; it exists for embedding.
 *
 * Who needs it: a process whose device memory is carved up in advance (a
 * serving stack that reserves almost all of HBM for its KV cache, or an
 * arena-only deployment where every byte is budgeted), and a real-time
 * control loop that cannot afford cudaMalloc's implicit device
 * synchronisation and unbounded latency.  Such a caller still passes every
 * input and output; the kernel's scratch (its error word and the partial
 * results of split calls) lives in a fixed array of
 * DM05_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU that
 * loads the library holds until exit.
 *
 * Arguments, layouts, supported sizes and results are those of
 * dm05_suffix_attn.  This entry point never calls cudaMalloc, cudaFree or any
 * allocating routine.  When the automatic split would need more partial
 * scratch than the array holds, the call splits each (sample, KV head) over
 * fewer CTAs (down to one, which needs none), so valid sizes always fit;
 * DM05_ERR_WORKSPACE is returned only if the error word itself did not fit.
 *
 * Set-up: the first call on each device looks up the array's device address
 * and clears its error word (enqueued on `stream`, then the host waits for
 * it), so make that first call before any stream capture on that device; a
 * first call on a capturing stream returns DM05_ERR_WORKSPACE and does
 * nothing.
 *
 * Sharing: every call on a device uses the same array and it keeps what the
 * last call left there.  A call writes all the partial results it later
 * reads.  The array's error word collects the same bits as the allocating
 * entry points' word (a clamped prefix_valid_len, a wait time-out) and
 * keeps them until dm05_get_error_word reads and clears them (it reads this
 * word too).  After a time-out the call's outputs are invalid.  Calls whose
 * kernels overlap on the GPU (for example on two streams) race on the array
 * and may corrupt each other's results: serialise them.
 */
#define DM05_NOALLOC_SCRATCH_BYTES (8u << 20)
int dm05_suffix_attn_noalloc(const void *q, const void *k_prefix, const void *v_prefix,
                             const int32_t *prefix_valid_len, const uint8_t *prefix_mask,
                             const void *k_suffix, const void *v_suffix,
                             void *out, float *lse,
                             int B, int Hq, int Hkv, int P, int S, int D,
                             cudaStream_t stream);

/*
 * dm05_suffix_attn_host -- the same attention with every tensor in HOST
 * memory: the call for a caller whose inputs are on the host and who wants
 * the result back there (one request at a time, as a control loop issues
 * them).  The source pages have no counterpart; it exists so that a whole
 * request (copies in, attention, copies out) is one library call.
 *
 * Arguments, sizes and results are those of dm05_suffix_attn, but q,
 * k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix, v_suffix,
 * out and lse are host addresses; no alignment is required.  The call
 * enqueues on `stream`, in order: host-to-device copies of the inputs into a
 * staging buffer the library owns per (device, stream), the attention
 * kernel, and device-to-host copies of out (and of lse unless it is NULL).
 *
 * prefix_valid_len is read on the host during the call: only the prefix
 * rows [0, clamp(prefix_valid_len[b], 0, P)) of each sample are copied
 * (every row when it is NULL), since no other row is used.  The clamp is
 * flagged in the error word as in dm05_suffix_attn.
 *
 * With page-locked host buffers (cudaHostAlloc / cudaHostRegister) every
 * copy is asynchronous: the inputs must stay unchanged, and out / lse must
 * not be read, until `stream` has passed the call (cudaStreamSynchronize).
 * Pageable buffers also work, but the CUDA runtime then blocks the host
 * inside the copies.
 *
 * When out (16-byte aligned) and lse (if not NULL) are page-locked memory
 * that the device can address (cudaHostAlloc / cudaMallocHost on a 64-bit
 * system, or cudaHostRegister with cudaHostRegisterMapped), the kernel
 * stores O and the LSE into them directly and no copy back is enqueued;
 * otherwise both come back from the staging buffer by copies.  out and lse
 * must each lie inside one allocation.
 *
 * The staging buffer is allocated (cudaMalloc) by the first call with these
 * sizes on the stream, grows when sizes grow (cudaFree, which waits for the
 * device) and is freed by dm05_release.  The call cannot be captured into a
 * CUDA graph (it reads valid lengths on the host): on a capturing stream it
 * returns DM05_ERR_UNSUPPORTED and enqueues nothing.
 */
int dm05_suffix_attn_host(const void *q, const void *k_prefix, const void *v_prefix,
                          const int32_t *prefix_valid_len, const uint8_t *prefix_mask,
                          const void *k_suffix, const void *v_suffix,
                          void *out, float *lse,
                          int B, int Hq, int Hkv, int P, int S, int D,
                          cudaStream_t stream);

/* Bytes one dm05_suffix_attn_host call with these arguments copies to the
 * device (*h2d_bytes) and back to the host (*d2h_bytes).  prefix_valid_len
 * is the same host array (or NULL); has_prefix_mask and want_lse say whether
 * prefix_mask and lse would be non-NULL.  Host-only: touches no device.
 * Either output pointer may be NULL. */
int dm05_suffix_attn_host_copy_bytes(const int32_t *prefix_valid_len, int has_prefix_mask, int want_lse,
                                     int B, int Hq, int Hkv, int P, int S, int D,
                                     size_t *h2d_bytes, size_t *d2h_bytes);

/*
 * dm05_selftest_wait_timeout -- exercises the failure detection without a
 * GPU fault.  It launches, on `stream`, one thread that waits on a barrier
 * nothing completes, with the same bounded wait every kernel wait uses but a
 * limit of limit_ms milliseconds (1..2000); the wait gives up and sets
 * DM05_EW_WAIT_TIMEOUT in the device error word, as an attention kernel
 * whose wait ran out does, and the kernel returns normally.  Read the word
 * with dm05_get_error_word.  Creates the error word if needed, so it must not
 * be called on a capturing stream (DM05_ERR_UNSUPPORTED).  Returns
 * DM05_ERR_SHAPE for a limit out of range.
 */
int dm05_selftest_wait_timeout(int limit_ms, cudaStream_t stream);

/* Synchronises `stream`, then returns in *host_word the error bits
 * (DM05_EW_*) that kernels on the current device set since the last read,
 * and clears them: the word of dm05_suffix_attn / dm05_suffix_attn_host /
 * dm05_selftest_wait_timeout and the word in the fixed array of
 * dm05_suffix_attn_noalloc, ORed together.  Allocates nothing. */
int dm05_get_error_word(cudaStream_t stream, uint32_t *host_word);

/* Human-readable name of a dm05_status value. */
const char *dm05_status_string(int status);

/* Frees every workspace and staging buffer the library holds (all
 * devices).  No call may be in flight. */
void dm05_release(void);

#ifdef __cplusplus
}
#endif

#endif /* DM05_SUFFIX_ATTN_H */
