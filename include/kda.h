/*
 * kda.h -- C ABI of the B200 (sm_100a) forward pass of the modality-aware
 * short convolution followed by the Kimi Delta Attention (KDA) scan.
 *
 * What is computed (sources are the pages about "Chimera: Designing and
 * Chinchilla-Scaling Hybrid Visual Diffusion Transformers"):
 *
 *  - Token stream: per batch item, text_len text tokens followed by the visual
 *    tokens of a (grid_t, grid_h, grid_w) latent grid in time-major raster
 *    order, N = text_len + grid_t*grid_h*grid_w
 *    (paper.rainbus.top, section 核心方法 and 方法步骤详情 step (2)).
 *  - Short convolution, per modality, depthwise, separately on q, k and v
 *    (genai-atlas, section "How it works"; paper.rainbus.top, section 核心方法):
 *      text token t:  x'[t,c] = sum_{j<text_k} w_text[c][j] * x[t-(text_k-1)+j, c]
 *                     (positions before the first token read 0);
 *      visual token (t,h,w):
 *                     x' = sum_{a,b,e} w_vis[c][(a*kh+b)*kw+e] * x(t+a-pt, h+b-ph, w+e-pw)
 *                     with ph=(kh-1)/2, pw=(kw-1)/2, pt=(kt-1)/2, or pt=kt-1 when
 *                     KDA_FLAG_VIS_CAUSAL_T is set; positions outside the grid
 *                     read 0; text and visual tokens never read each other.
 *  - KDA scan (paper.rainbus.top, section 方法步骤详情 step (5), and section
 *    前置知识 "Kimi Delta Attention"), per (batch item, head), in stream order:
 *      S_t = (I - beta_t k'_t k'_t^T) Diag(alpha_t) S_{t-1} + beta_t k'_t v'_t^T,
 *      o_t = S_t^T q'_t            (alpha_t = exp(log_alpha_t), no scale on q)
 *    with S_{-1} = initial_state (or 0).  The scan is evaluated in chunks of
 *    `chunk` tokens (the chunked KDA form named in section 复现评估); the result
 *    does not depend on the chunk length beyond rounding.
 *
 *  - Batch items with fewer text tokens than text_len: place an item's text at
 *    the end of the text span and fill the leading positions with zero tokens
 *    (q = k = v = 0, log_alpha = 0, beta = 0).  A zero token leaves the state
 *    unchanged and is what the causal text conv reads before the first token,
 *    so the real tokens' outputs and the final state are exactly those of the
 *    unpadded item; the padding positions' outputs are zero.
 *
 * Layouts (row-major, contiguous):
 *    q, k, log_alpha : [B, N, H, dk]      v, o : [B, N, H, dv]      beta : [B, N, H]
 *    w_text : [3][H*dk][text_k]           w_vis : [3][H*dk][vis_kt*vis_kh*vis_kw]
 *             (slot 0 for q, 1 for k, 2 for v; fp32)
 *    initial_state, final_state : [B, H, dk, dv] fp32
 * q, k, v, beta and o have the element type `dtype`; log_alpha is always fp32
 * and must be finite and <= 0.
 *
 * Conventions for every entry point:
 *  - All data pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or synchronises (kda_read_status excepted, which
 *    synchronises the given stream).  `stream` is a cudaStream_t (NULL = the
 *    legacy default stream); work is enqueued asynchronously on it.
 *  - Argument errors are detected on the host and returned WITHOUT launching
 *    anything: a NULL required pointer, a non-positive size, an unsupported
 *    size (dk, dv, chunk, kernel extents), a data pointer that is not 16-byte
 *    aligned, or a workspace smaller than kda_workspace_bytes().
 *  - Outputs must not alias inputs.
 *  - Device-side conditions (bounded waits that gave up; the gate range check
 *    of the backward pass) are recorded in a status word at the start of the
 *    workspace; read it with kda_read_status() once the stream has reached the
 *    call.  Kernels never trap.  The forward pass accepts any finite
 *    log_alpha <= 0: its decay factors are products of gates alpha <= 1.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1,    /* NULL pointer, non-positive or inconsistent size */
  KDA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. dk != dv, dk not 64/128) */
  KDA_ERR_MISALIGNED = 3,     /* a data pointer is not 16-byte aligned */
  KDA_ERR_WORKSPACE = 4,      /* workspace NULL or smaller than kda_workspace_bytes() */
  KDA_ERR_CUDA = 5,           /* a CUDA runtime call failed (launch, copy) */
  KDA_ERR_TIMEOUT = 6,        /* device: a bounded wait gave up */
  KDA_ERR_DEVICE_ASSERT = 7,  /* device: an internal consistency check failed */
  KDA_ERR_RANGE = 8           /* device: a chunk's gate decay exceeds what the backward pass handles */
} kda_status;

typedef enum { KDA_DT_BF16 = 0, KDA_DT_F32 = 1 } kda_dtype;

/* Temporal taps of the 3D conv cover frames t-kt+1..t instead of being centred. */
#define KDA_FLAG_VIS_CAUSAL_T 1u
/* kda_chunk_fwd only (the other entry points reject it): the workspace still holds the
 * intermediate block records that the previous kda_chunk_fwd call on it computed from the
 * same q, k, v, log_alpha, beta, problem and dtype, on the same stream, with no other call on
 * this workspace in between.  Only the serial state pass runs again, from the new
 * initial_state: the map from initial to final state is affine, so a caller can evaluate it
 * at several initial states (sequence sharding) for the price of one full pass.  Paths that
 * keep no records (fp32, d = 64) recompute everything; the result is the same. */
#define KDA_FLAG_REUSE_RECORDS 2u
/* bf16 problems with d = 128 only (otherwise KDA_ERR_UNSUPPORTED): the convolved q', k', v'
 * are fp16 instead of bf16 -- the outputs of kda_shortconv_fwd and the q, k, v inputs of
 * kda_chunk_fwd / kda_chunk_fwd_noalloc.  fp16 is the operand type of the tensor-core scan
 * and keeps three more mantissa bits than bf16 (kda_fwd keeps its intermediates in fp16
 * anyway and rejects the flag); callers that split the pass into the two calls use it to
 * get kda_fwd's accuracy.  beta and o stay bf16. */
#define KDA_FLAG_QKV_F16 4u

typedef struct {
  int32_t B, H, dk, dv;             /* batch items, heads, key and value head dims */
  int64_t text_len;                 /* text tokens per item (>= 0), same for all items */
  int32_t grid_t, grid_h, grid_w;   /* visual grid (each >= 0; all 0 or all > 0) */
  int32_t text_k;                   /* causal text kernel length, 1..8 */
  int32_t vis_kt, vis_kh, vis_kw;   /* 3D kernel extents; only 3,3,3 is implemented */
  int32_t chunk;                    /* scan chunk length: 16, 32 or 64 for fp32 and for bf16 with
                                       d = 64; exactly 64 for bf16 with d = 128 (the tensor-core
                                       path's 64-token sub-chunks); anything else, 128 included,
                                       returns KDA_ERR_UNSUPPORTED */
  uint32_t flags;                   /* KDA_FLAG_* */
} kda_problem;

/* Tokens per batch item, N = text_len + grid_t*grid_h*grid_w, or -1 if the
 * problem is inconsistent. */
int64_t kda_tokens(const kda_problem* p);

/* Bytes of device workspace any entry point below needs for problem p and
 * element type dtype (0 if p is invalid).  The workspace must be 256-byte
 * aligned; its first 256 bytes hold the status word. */
size_t kda_workspace_bytes(const kda_problem* p, kda_dtype dtype);

/* Short convolution only: q_out = conv_q(q), k_out = conv_k(k), v_out = conv_v(v),
 * all [B, N, H, d] of `dtype` (fp32 accumulation, one rounding to dtype).
 * Returns a kda_status. */
int kda_shortconv_fwd(const kda_problem* p, kda_dtype dtype,
                      const void* q, const void* k, const void* v,
                      const float* w_text, const float* w_vis,
                      void* q_out, void* k_out, void* v_out, void* stream);

/* KDA scan only, on already-convolved q', k', v'.  initial_state may be NULL
 * (zero state); final_state may be NULL (not written).  Returns a kda_status.
 * On the bf16 d = 128 tensor-core path the scan writes per-block records (and, after them, one
 * flag word per record) to the workspace.  With at most a fifth as many (batch item, head) pairs
 * as SMs it is one cooperative launch, whose state-pass CTAs wait for the record CTAs' flags (all
 * its CTAs are resident at once, so it may start only once the whole grid fits on the device);
 * otherwise, and when the device refuses a cooperative launch of that size, the record kernel and
 * then the state-pass kernel. */
int kda_chunk_fwd(const kda_problem* p, kda_dtype dtype,
                  const void* q, const void* k, const void* v,
                  const float* log_alpha, const void* beta,
                  const float* initial_state, void* o, float* final_state,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Short convolution followed by the KDA scan.  Returns a kda_status. */
int kda_fwd(const kda_problem* p, kda_dtype dtype,
            const void* q, const void* k, const void* v,
            const float* log_alpha, const void* beta,
            const float* w_text, const float* w_vis,
            const float* initial_state, void* o, float* final_state,
            void* workspace, size_t workspace_bytes, void* stream);

/* kda_fwd on host-resident tensors, with the host<->device copies overlapped with the kernels.
 * The pages describe no host interface; this is the call for data that lives in host memory.
 *   q, k, v, log_alpha, beta: host pointers, layouts as in kda_fwd; o: host pointer [B, N, H, d].
 *     Page-locked (pinned) memory lets the copies run asynchronously; pageable memory works but
 *     each copy then blocks the calling thread.  They must stay valid and unchanged until the
 *     stream has passed the call.
 *   w_text, w_vis, initial_state, final_state: device pointers, as in kda_fwd.
 *   seg_frames >= 1: visual frames per segment.  Each batch item's token stream is cut into
 *     segments of seg_frames frames (its text prefix goes with the first); a segment's inputs are
 *     copied in on copy_in_stream, its conv and scan run on stream (the scan entering with the
 *     state the previous segment left, so o and final_state equal kda_fwd's up to the rounding
 *     of the scan's chunking at segment starts), and its o is copied out on copy_out_stream.
 *     Copies of one segment overlap the kernels of its neighbours.
 *   stream, copy_in_stream, copy_out_stream: caller-owned streams (three distinct streams for
 *     the overlap).  The copies in wait for the work enqueued on `stream` before the call; once
 *     `stream` has passed the call, o is in host memory and final_state is written.
 * The call creates and releases a few CUDA events; it allocates no memory and does not
 * synchronise.  Workspace: kda_fwd_host_workspace_bytes(p, dtype, seg_frames) device bytes,
 * 256-byte aligned (the inputs and o staged in full, the conv outputs, two states and the scan
 * records of one segment).  Flags as in kda_fwd.  Returns a kda_status. */
size_t kda_fwd_host_workspace_bytes(const kda_problem* p, kda_dtype dtype, int32_t seg_frames);
int kda_fwd_host(const kda_problem* p, kda_dtype dtype,
                 const void* q, const void* k, const void* v,
                 const float* log_alpha, const void* beta,
                 const float* w_text, const float* w_vis,
                 const float* initial_state, void* o, float* final_state, int32_t seg_frames,
                 void* workspace, size_t workspace_bytes, void* stream,
                 void* copy_in_stream, void* copy_out_stream);

/* Backward pass of kda_fwd: the gradients of the loss sum(d_o * o) + sum(d_final_state * S_N)
 * (o and S_N as kda_fwd computes them from the same arguments) with respect to every input.
 * The pages describe only the forward pass; the gradients are the chain rule applied to it
 * (the conv is linear, its adjoint is its transpose; the recurrence is differentiated in its
 * chunked form over 64-token chunks: the state entering every chunk is stored by a forward
 * pass, the gradient reaching every chunk's exit by a reverse pass, and each chunk's token
 * gradients follow from the two).  The products run on the tensor cores: for fp32 problems in
 * tf32 split into two terms per operand (three products, fp32 accuracy); for bf16 problems one
 * tf32 product of rounded operands in the per-chunk passes and fp16 operands and additive terms
 * with fp32 accumulation in the passes over chunks (the state itself kept in fp32).
 *   d_o                    [B, N, H, d] of dtype; d_final_state [B, H, d, d] fp32 or NULL (zero)
 *   dq, dk, dv             [B, N, H, d] of dtype: gradients of the raw (unconvolved) q, k, v
 *   d_log_alpha            [B, N, H, d] fp32;  d_beta [B, N, H] of dtype
 *   d_w_text, d_w_vis      [3][H*d][text_k], [3][H*d][kt*kh*kw] fp32
 *   d_initial_state        [B, H, d, d] fp32 or NULL (not written)
 * The workspace is kda_bwd_workspace_bytes(p, dtype) bytes, 256-byte aligned.  Flags:
 * KDA_FLAG_VIS_CAUSAL_T as in kda_fwd; the other flags are rejected.  The conv weight
 * gradients are summed over tokens with atomic adds, so their last bits depend on the order of
 * the additions.  Device status KDA_ERR_RANGE: within a chunk the running log-decay moved more
 * than 60 nats away from its value at the chunk's token 31 (the fp32 factors of the pairwise
 * decays would overflow); the gradients are then not valid.  Returns a kda_status. */
size_t kda_bwd_workspace_bytes(const kda_problem* p, kda_dtype dtype);
int kda_bwd(const kda_problem* p, kda_dtype dtype,
            const void* q, const void* k, const void* v,
            const float* log_alpha, const void* beta,
            const float* w_text, const float* w_vis, const float* initial_state,
            const void* d_o, const float* d_final_state,
            void* dq, void* dk, void* dv, float* d_log_alpha, void* d_beta,
            float* d_w_text, float* d_w_vis, float* d_initial_state,
            void* workspace, size_t workspace_bytes, void* stream);

/* kda_chunk_fwd without a workspace, for callers that cannot allocate device
 * memory (code running inside an allocator or memory-pool callback, runtimes
 * that forbid allocation after start-up, plugins handed only their input and
 * output buffers).  The pages describe no counterpart; this is an interface
 * convenience.
 *
 * Same operation, arguments and errors as kda_chunk_fwd, with these differences:
 *  - Scratch comes from a static device array of 64 MiB that the library holds
 *    on every GPU that loads it, until the process exits.  A problem whose
 *    scratch exceeds it (256 B + 128 KiB per (batch item, head, 128-token block)
 *    on the bf16 d=128 tensor-core path) returns KDA_ERR_WORKSPACE without
 *    launching anything.
 *  - The first call on a device looks up that array's device address (once per
 *    device); make it before any stream capture.  The address belongs to the
 *    device's primary context: do not use this entry point on a device again
 *    after cudaDeviceReset in the same process.
 *  - Calls share the array: calls whose GPU work overlaps (other streams, other
 *    host threads on the same device) race.  Run them on one stream.
 *  - Device-side conditions (see kda_read_status) are written to *device_status
 *    (a 4-byte-aligned device word, cleared at the start of the call) when it is
 *    not NULL, otherwise to a word inside the static array that callers cannot
 *    read.
 *  - No cudaMalloc, cudaFree or other allocating call is made. */
int kda_chunk_fwd_noalloc(const kda_problem* p, kda_dtype dtype,
                          const void* q, const void* k, const void* v,
                          const float* log_alpha, const void* beta,
                          const float* initial_state, void* o, float* final_state,
                          uint32_t* device_status, void* stream);

/* Self-test of the bounded device waits; the pages have no counterpart.  Every wait of the kernels
 * (for an asynchronous copy, a tensor-core product or another warp) gives up after a time limit and
 * records KDA_ERR_TIMEOUT instead of hanging the GPU; this call makes one such wait run out on purpose
 * so that a test can check the give-up path without faulting or hanging anything.  It runs
 * kda_chunk_fwd's kernels on a bf16 problem with dk = dv = 128 (the tensor-core path; other problems
 * return KDA_ERR_UNSUPPORTED) with every device wait limited to wait_us microseconds (>= 1), and one
 * asynchronous load that is never issued:
 *   stage 1: the first k/q/v tile load of the first CTA of the block-record kernel;
 *   stage 2: the first record load of the first CTA of the serial state pass.
 * The CTA whose wait gives up records KDA_ERR_TIMEOUT in the workspace status word, waits (bounded)
 * for its other copies, frees its tensor memory and returns; CTAs and kernels that start later skip
 * their work.  o is not valid afterwards.  Arguments as in kda_chunk_fwd (no states).  Returns
 * KDA_OK once the work is enqueued; kda_read_status then reports KDA_ERR_TIMEOUT. */
int kda_selftest_wait_timeout(const kda_problem* p, kda_dtype dtype,
                              const void* q, const void* k, const void* v,
                              const float* log_alpha, const void* beta, void* o,
                              void* workspace, size_t workspace_bytes,
                              int32_t stage, uint32_t wait_us, void* stream);

/* Synchronises `stream`, then returns and clears the device status word kept
 * in `workspace` (KDA_OK if no device-side condition was recorded). */
int kda_read_status(void* workspace, void* stream);

/* Static description of a kda_status value. */
const char* kda_status_str(int status);

/* Number of kernel launches the most recent successful call on this host
 * thread enqueued (for launch accounting in benchmarks). */
int kda_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
