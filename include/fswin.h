/*
 * fswin — fused Swin windowed self-attention with window-local learnable 2D RoPE
 * on B200 (sm_100a): forward and backward behind a plain C ABI.
 *
 * The operation is the one the FlashSwin paper introduces ("FLASHSWIN: Unlocking
 * Large Windows and Dense Tokens in Swin Vision Transformers with Memory Efficient
 * Attention"; arxivdaily.com/papers/2610.04664, English abstract; and
 * thelatestinai.com/papers/2610.04664, Figure 1B and Figure S4): exact softmax
 * attention inside every M x M window of a cyclically shifted token grid, computed
 * without materialising the M^2 x M^2 score matrix, with queries and keys rotated
 * by a window-local 2D RoPE whose inverse frequencies theta are learnable.
 *
 * Conventions (readings of the paper where it is silent):
 *  - tensors q, k, v, o, dout, dq, dk, dv are bf16, contiguous [B, H, W, heads, d]
 *    (d = 32 or 64), 16-byte aligned, in DEVICE memory;
 *  - theta and dtheta are fp32 [heads, 2, d/4]; axis 0 (x) rotates channel pairs
 *    (2k, 2k+1) of the first d/2 channels by j * theta[h][0][k], axis 1 (y) the pairs
 *    of the last d/2 channels by i * theta[h][1][k], where (i, j) is the token's
 *    row and column inside its window (0 .. M-1, in the rolled frame);
 *  - H or W that is not a multiple of M is padded at the bottom and right to
 *    Hp = ceil(H/M)*M, Wp = ceil(W/M)*M with zero tokens, as a Swin layer pads its
 *    input before the shift; everything below then refers to the padded grid
 *    (Hp = H, Wp = W for multiples), padded tokens take part in the softmax, and
 *    only the H x W real tokens are read or written;
 *  - the shift takes rolled token (r, c) from original position ((r+s) mod Hp,
 *    (c+s) mod Wp); outputs are written back at original positions;
 *  - with s > 0 a query attends a key of its window only when both carry the same
 *    Swin shift-region label, built from the row/column slices [0, Hp-M),
 *    [Hp-M, Hp-s), [Hp-s, Hp); masked scores are -infinity;
 *  - softmax scale 1/sqrt(d); lse is the natural-log log-sum-exp per query, fp32
 *    [B, H, W, heads];
 *  - gradients are those of sum(o * dout).
 *
 * Ownership and ordering: the caller owns every buffer.  The library never
 * allocates device memory and never synchronises; all work is enqueued on the
 * given stream (a cudaStream_t; NULL is the legacy default stream).
 *
 * Per-device state (the device status word's address, the kernels' shared-memory
 * opt-in) is set up on the first call on each device and kept for the life of the
 * process, so the library must not be used on a device after cudaDeviceReset.
 *
 * Errors: invalid arguments return a status and launch nothing.  A kernel whose
 * internal wait runs past its time limit stops and records FS_ERR_TIMEOUT in a
 * device status word that fs_device_status() reads (after the stream is
 * synchronised by the caller).
 */
#ifndef FSWIN_H
#define FSWIN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FS_API __attribute__((visibility("default")))
#else
#define FS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FS_OK = 0,
    FS_ERR_NULL = 1,      /* a required pointer is NULL */
    FS_ERR_SHAPE = 2,     /* unsupported or inconsistent shape (see fs_winattn_shape) */
    FS_ERR_ALIGN = 3,     /* a pointer is not 16-byte aligned */
    FS_ERR_WORKSPACE = 4, /* workspace missing, misaligned or too small */
    FS_ERR_CUDA = 5,      /* a CUDA runtime/driver call failed */
    FS_ERR_TIMEOUT = 6,   /* a device-side wait ran out of time */
    FS_ERR_ARCH = 7       /* the current device is not sm_100 */
} fs_status;

/*
 * Problem shape.  Supported: d == 32 or d == 64; M in {4, 8, 16, 32, 64}; H >= M and W >= M
 * (not necessarily multiples of M: the grid is then padded, see above; a grid
 * smaller than the window is the caller's to clamp, as Swin clamps the window);
 * 0 <= s < M with s a multiple of 4; heads >= 1; B >= 0 (B == 0 is a valid empty
 * problem).  Anything else returns FS_ERR_SHAPE.
 * Heads of d = 64 (16 RoPE pairs per axis) run their own kernels, plain
 * one-tile pipelines; their backward's workspace holds an fp32 dQ accumulator
 * (256 bytes per token-head) besides the d theta partials.
 */
typedef struct {
    int B, H, W, heads, d, M, s;
} fs_winattn_shape;

typedef struct CUstream_st* fs_stream_t; /* same type as cudaStream_t */

/* Returns FS_OK when the shape is supported, without touching the device. */
FS_API fs_status fs_winattn_check_shape(const fs_winattn_shape* shape);

/*
 * Forward.  In: q, k, v (bf16 [B,H,W,heads,d]), theta (fp32 [heads,2,d/4]).
 * Out: o (bf16 [B,H,W,heads,d]) and lse (fp32 [B,H,W,heads], natural log);
 * both overwritten.  lse may be NULL: an inference forward that writes o only
 * (the workload of FlashSwin's inference-throughput figure, thelatestinai.com
 * Fig. S1); the backward needs lse, so a training forward passes it.
 * Exact softmax attention per window, with no score matrix in device memory
 * (the FlashSwin abstract).
 */
FS_API fs_status fs_winattn_fwd(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                         const float* theta, void* o, float* lse, fs_stream_t stream);

/*
 * Forward of the whole window-attention block of a Swin layer, for inference
 * (the attention module of a FlashSwin block, thelatestinai.com 2610.04664,
 * Figure 1B, with its two linear maps):
 *   qkv = x W_qkv^T + b_qkv, split in (3, heads, d) along the channels;
 *   o = fs_winattn_fwd's attention of (q, k, v) with theta, M, s;
 *   y = o W_o^T + b_o, o taken as [B,H,W,C].
 * In: x bf16 [B,H,W,C] with C = heads * d; w_qkv bf16 [3C, C] (output channels
 * q of every head, then k, then v); b_qkv fp32 [3C]; w_o bf16 [C, C]; b_o
 * fp32 [C]; theta fp32 [heads,2,d/4].  Out: y bf16 [B,H,W,C], overwritten.  d == 32 only.
 * q, k, v and o never reach device memory.  Supported: the shapes of
 * fs_winattn_check_shape with M*M < 128 (windows inside one 128-token tile)
 * and heads <= 3; anything else returns FS_ERR_SHAPE.  On a padded grid (H or W
 * not a multiple of M) the padded tokens of x are zero, as the Swin layer pads x
 * before its qkv map, so their q, k, v equal the bias.  x, w_qkv, w_o, y
 * 16-byte aligned (FS_ERR_ALIGN); no pointer may be NULL (FS_ERR_NULL).
 */
FS_API fs_status fs_winattn_block_fwd(const fs_winattn_shape* shape, const void* x, const void* w_qkv,
                               const float* b_qkv, const void* w_o, const float* b_o, const float* theta,
                               void* y, fs_stream_t stream);

/*
 * Workspace the backward needs, in bytes.  It depends on the token count of the
 * padded grid, B*Hp*Wp*heads, only: for H and W multiples of M it does not depend
 * on the window size (memory flat in M, FlashSwin Table S1).
 */
FS_API size_t fs_winattn_bwd_workspace_bytes(const fs_winattn_shape* shape);

/*
 * Backward (recompute-based: the probabilities are rebuilt from lse, never stored).
 * In: q, k, v, o (the forward output), dout, lse, theta.  Out: dq, dk, dv (bf16
 * [B,H,W,heads,d]) and dtheta (fp32 [heads,2,d/4]); all overwritten.  workspace:
 * device scratch of at least fs_winattn_bwd_workspace_bytes(shape) bytes, 256-byte
 * aligned; its contents on entry are ignored.
 */
FS_API fs_status fs_winattn_bwd(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                         const void* o, const void* dout, const float* lse, const float* theta, void* dq,
                         void* dk, void* dv, float* dtheta, void* workspace, size_t workspace_bytes,
                         fs_stream_t stream);

/*
 * Windowed attention with a low-rank additive bias (the FlashBias-T variant of
 * the same pages: thelatestinai.com 2610.04664, Table 2 and Table S1 captions,
 * a trainable rank-16 factorization of an additive attention bias whose
 * parameters grow with M).  Reading where the pages are silent: per head h the
 * bias of a window's (query position t, key position u) pair is
 * U[h][t] . W[h][u], t = i*M + j the window-local position in the rolled frame,
 * the same for every window of the batch, added to the scaled score before the
 * shift mask:  S_tu = q'_t . k'_u / sqrt(d) + U[h][t] . W[h][u].
 *
 * Shapes: those of fs_winattn_check_shape with d == 32 (else FS_ERR_SHAPE);
 * rank == 16 (else FS_ERR_SHAPE).  u, w: fp32 [heads][M*M][16], 16-byte aligned.
 * theta may be NULL: no rotation (q' = q, k' = k), and the backward then takes
 * dtheta == NULL too; with theta the RoPE of fs_winattn_fwd applies.  Other
 * arguments, layouts, ownership and errors as fs_winattn_fwd / fs_winattn_bwd.
 *
 * Forward: o and lse (lse may be NULL: inference), overwritten.
 * Backward: dq, dk, dv, dtheta (when theta is given), du and dw (fp32
 * [heads][M*M][16], the gradients summed over every window of the batch, in a
 * fixed order), all overwritten.  dq, du and the query side of dtheta are
 * accumulated in fp32 with vector reductions whose order varies from run to
 * run; dk, dv and dw do not vary.  workspace: at least fs_winattn_lrbias_bwd_workspace_bytes(shape)
 * bytes, 256-byte aligned (about 276 bytes per token-head on the padded grid,
 * plus a few KB per head).  The kernels are plain one-tile pipelines.
 */
FS_API fs_status fs_winattn_lrbias_fwd(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                                       const float* theta, const float* u, const float* w, int rank, void* o,
                                       float* lse, fs_stream_t stream);
FS_API size_t fs_winattn_lrbias_bwd_workspace_bytes(const fs_winattn_shape* shape);
FS_API fs_status fs_winattn_lrbias_bwd(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                                       const void* o, const void* dout, const float* lse, const float* theta,
                                       const float* u, const float* w, int rank, void* dq, void* dk, void* dv,
                                       float* dtheta, float* du, float* dw, void* workspace, size_t workspace_bytes,
                                       fs_stream_t stream);

/*
 * Training pair.  fs_winattn_fwd_train is fs_winattn_fwd (lse required) that
 * also leaves, in `workspace` (the backward's: at least
 * fs_winattn_bwd_workspace_bytes(shape) bytes, 256-byte aligned), the rotated
 * q', k' tiles the backward needs; fs_winattn_bwd_train is fs_winattn_bwd that
 * takes them from there instead of rotating q and k again.  The forward of
 * windows of >= 128 tokens (d == 32) then reads its Q', K' tiles from those
 * images, rotating each row once instead of once per query tile of the window.
 * Same results as fs_winattn_fwd / fs_winattn_bwd.  Contract: the backward gets
 * the workspace of the training forward of the same shape, q, k and theta,
 * unchanged in between (otherwise its gradients are wrong; nothing checks it).
 * For windows of fewer than 128 tokens and for d == 64 the pair behaves as
 * fs_winattn_fwd / fs_winattn_bwd (the forward writes nothing to the workspace).
 * Errors as those of fs_winattn_fwd and fs_winattn_bwd; the forward also
 * returns FS_ERR_WORKSPACE for a missing, misaligned or short workspace.
 */
FS_API fs_status fs_winattn_fwd_train(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                                      const float* theta, void* o, float* lse, void* workspace,
                                      size_t workspace_bytes, fs_stream_t stream);
FS_API fs_status fs_winattn_bwd_train(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                                      const void* o, const void* dout, const float* lse, const float* theta,
                                      void* dq, void* dk, void* dv, float* dtheta, void* workspace,
                                      size_t workspace_bytes, fs_stream_t stream);

/* Human-readable name of a status. */
FS_API const char* fs_status_string(fs_status status);

/*
 * Reads and clears the device status word of the current device.  *code receives 0
 * when no kernel reported a failure, else (status << 24) | where.  Synchronous.
 */
FS_API fs_status fs_device_status(unsigned int* code);

/* Time limit of every device-side wait, in nanoseconds (default 10 s). */
FS_API fs_status fs_set_wait_limit_ns(uint64_t limit_ns);

/*
 * Self-test of the bounded-wait path: launches one CTA that waits on a barrier no
 * thread ever arrives on, with the given limit.  Afterwards (stream synchronised)
 * fs_device_status() reports FS_ERR_TIMEOUT.  The GPU context stays usable.
 */
FS_API fs_status fs_selftest_bounded_wait(uint64_t limit_ns, fs_stream_t stream);

/*
 * Backward that allocates nothing and takes no workspace (the paper has no
 * counterpart; this is a convenience of this library).  For callers that cannot
 * allocate device memory when they call the backward, for example code that
 * runs inside a memory pool that is already fully handed out, or a runtime that
 * forbids cudaMalloc after start-up.  The scratch is one array inside the
 * library, fs_winattn_bwd_noalloc_max_bytes() bytes (64 MiB) on every GPU that
 * loads the library, held until the process exits.  Problems whose
 * fs_winattn_bwd_workspace_bytes() exceeds that size return FS_ERR_WORKSPACE and
 * launch nothing.  Arguments and results are those of fs_winattn_bwd.
 *
 * The first call on a device looks up the array's device address (once per
 * device).  All calls on a device share the array: calls whose kernels may overlap on the GPU (other
 * streams or host threads without ordering between them) race on it.
 * The address is kept for the life of the process: do not use this entry point
 * (or any other of this library, whose device status word is looked up the same
 * way) on a device after cudaDeviceReset.
 */
FS_API fs_status fs_winattn_bwd_noalloc(const fs_winattn_shape* shape, const void* q, const void* k, const void* v,
                                        const void* o, const void* dout, const float* lse, const float* theta,
                                        void* dq, void* dk, void* dv, float* dtheta, fs_stream_t stream);

/* Size of the scratch array fs_winattn_bwd_noalloc uses, in bytes. */
FS_API size_t fs_winattn_bwd_noalloc_max_bytes(void);

/*
 * Profiling hook.  events: `n` caller-created cudaEvent_t handles (as void*), or
 * n == 0 to switch the hook off.  While set, fs_winattn_fwd records events[0]
 * before and events[1] after its kernel (n >= 2), and fs_winattn_bwd records
 * events[0] before its first kernel and events[1 + i] after its kernel i
 * (prep, main, post, dtheta reduction; n >= 5), on the call's stream; the
 * low-rank-bias entry points record the same marks (the backward's last one
 * after the dtheta, du and dw sums).  The
 * handles are kept by value; the hook is process-wide and not thread-safe.
 */
FS_API fs_status fs_set_phase_events(void* const* events, int n);

#ifdef __cplusplus
}
#endif

#endif /* FSWIN_H */
