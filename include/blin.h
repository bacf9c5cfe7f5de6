/*
 * blin — block-causal ReLU linear attention with 3D RoPE (numerator only) and
 * a constant-size (S, z) cache, for NVIDIA B200 (sm_100a).
 *
 * The operation (SANA-Video pages):
 *   - "SANA-Video: Efficient Video Generation with Block Linear Diffusion
 *     Transformer [ICLR 2026, Oral]" talk transcript, linear-attention state
 *     review: the state is d x d whatever the sequence length; block i adds its
 *     contribution K_i^T V_i to the cached state; block b attends to itself and
 *     every earlier block; 3D RoPE is used inside linear attention.
 *   - "四库全闻快报 ... SANA-Video" news article, positional-encoding paragraph:
 *     RoPE is kept in the numerator and removed from the denominator.
 *
 * For one head, with phi = ReLU and R_n the 3D rotation at token n:
 *   S_<=b = S_0 + sum_{m in blocks <= b} (R_m phi(k_m)) v_m^T      (d x d)
 *   z_<=b = z_0 + sum_{m in blocks <= b} phi(k_m)                   (d)
 *   o_n   = (R_n phi(q_n))^T S_<=b(n) / (phi(q_n) . z_<=b(n) + eps)
 *
 * Conventions (readings of points the pages leave open):
 *   - Tensors are contiguous [B][H][N][d], d innermost; N = T * Hgt * Wid with
 *     tokens ordered t-major, then y, then x.
 *   - Frame t of a call has absolute index t_abs = t0 + t, t0 being the cache's
 *     frame count (0 without a cache).  Blocks group F = block_frames absolute
 *     frames: block(t_abs) = t_abs / F, so a call that starts inside a block
 *     first finishes that block.  Attention is full inside a block.
 *   - RoPE: rope_split = (d_t, d_y, d_x), even, summing to d.  Axis sections
 *     are consecutive (t, then y, then x); pair (2j, 2j+1) of an axis section
 *     turns by p_axis * theta^(-2j/d_axis) with p = (t_abs, y, x).
 *   - No 1/sqrt(d) scale.  eps is added after the denominator's dot product.
 *   - States are fp32: S[B][H][d][d] (row = rotated key feature, column =
 *     value feature) and z[B][H][d].  Outputs have the input dtype.
 *
 * Ownership: the caller owns q, k, v, o and any workspace (device memory).
 * The library owns a state's S, z and block-step scratch, allocated in
 * blin_state_init / blin_state_reserve / the first blin_block_step that needs
 * more scratch, and freed in blin_state_free.  All work is enqueued
 * asynchronously on the given stream (a cudaStream_t; NULL = legacy default).
 *
 * Errors: arguments are checked on the host before any launch; a check that
 * fails returns a negative blin_status and sets a thread-local message
 * (blin_last_error).  CUDA launch failures return BLIN_ERR_CUDA.  Kernel
 * waits are bounded: a wait that exceeds its limit records a code readable by
 * blin_device_status and the kernel returns instead of hanging.
 */
#ifndef BLIN_H
#define BLIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BLIN_API __attribute__((visibility("default")))
#else
#define BLIN_API
#endif

typedef void *blin_stream; /* a cudaStream_t */

typedef enum {
    BLIN_OK = 0,
    BLIN_ERR_INVALID_ARG = -1, /* null pointer, non-positive size, bad flag, eps/theta out of range */
    BLIN_ERR_SHAPE = -2,       /* d not 32/64, bad rope split, a block step across blocks, size or launch limits */
    BLIN_ERR_DTYPE = -3,       /* unknown dtype */
    BLIN_ERR_ALIGN = -4,       /* q/k/v/o/workspace not 16-byte aligned */
    BLIN_ERR_WORKSPACE = -5,   /* workspace missing or too small; state scratch that would grow during capture */
    BLIN_ERR_STATE = -6,       /* freed/foreign state, B/H/d mismatch, wrong device, wrong byte count */
    BLIN_ERR_CUDA = -7,        /* a CUDA runtime/driver call failed */
    BLIN_ERR_DEVICE = -8       /* a kernel's bounded wait ran out (see blin_device_status) */
} blin_status;

typedef enum { BLIN_F32 = 0, BLIN_BF16 = 1 } blin_dtype;

/* Latent grid and method constants of one call.
 *   T, Hgt, Wid   latent frames, height and width of this call (N = T*Hgt*Wid)
 *   block_frames  F, latent frames per causal block (>= 1)
 *   rope_split    dims of the t, y, x RoPE sections (even, sum = d)
 *   theta         RoPE base (> 0), eps  denominator offset (>= 0, finite) */
typedef struct {
    int T, Hgt, Wid;
    int block_frames;
    int rope_split[3];
    float theta;
    float eps;
} blin_geom;

/* Memory layout of one [B][H][N][d] operand: element (b, h, n, j) sits at
 * base + b*batch + h*head + n*token + j, strides in elements (d is innermost,
 * stride 1).  Each stride must be >= d and a multiple of 16 bytes (for bf16: a
 * multiple of 8 elements); a stride of a dimension of extent 1 is ignored.
 * Example, a fused QKV projection output [B][N][3][H][d]:
 *   q = base, k = base + H*d, v = base + 2*H*d,
 *   {token = 3*H*d, head = d, batch = N*3*H*d}.
 * Contiguous [B][H][N][d] is {d, N*d, H*N*d}. */
typedef struct {
    long long token, head, batch;
} blin_layout;

typedef struct blin_state blin_state; /* opaque (S, z) cache on one device */

/* ---------------------------------------------------------------- state */

/* Allocate a zeroed cache S[B][H][d][d], z[B][H][d] (fp32) on the current
 * device, t_next = 0.  Memory stays constant however many blocks pass through
 * it (talk transcript: constant KV-cache memory for any video length). */
BLIN_API blin_status blin_state_init(int B, int H, int d, blin_stream stream, blin_state **out);

/* Free the cache and its scratch.  Waits for the last call that used the state
 * (on whatever stream it ran) to finish first; other work on the device is not
 * waited for.  Calls captured into a CUDA graph are not tracked: the caller
 * must let every launch of such a graph finish before freeing the state.
 * NULL is a no-op. */
BLIN_API blin_status blin_state_free(blin_state *st);

/* Zero S and z (on stream) and set t_next = 0. */
BLIN_API blin_status blin_state_reset(blin_state *st, blin_stream stream);

/* Device pointers of S and z and the next absolute frame index.  Any output
 * pointer may be NULL.  The pointers stay valid until blin_state_free. */
BLIN_API blin_status blin_state_tensors(const blin_state *st, float **S, float **z, int *t_next);

/* Bytes of one host copy of the cache: B*H*(d*d + d)*4 (S then z). */
BLIN_API size_t blin_state_bytes(const blin_state *st);

/* Copy S then z into host memory (bytes must equal blin_state_bytes).  The
 * copy is enqueued on stream; synchronise before reading host. */
BLIN_API blin_status blin_state_copy_to_host(const blin_state *st, void *host, size_t bytes, blin_stream stream);

/* Restore S then z from host memory and set t_next (checkpoint resume).  The
 * host buffer must stay valid until the stream reaches the copy. */
BLIN_API blin_status blin_state_copy_from_host(blin_state *st, const void *host, size_t bytes, int t_next,
                                      blin_stream stream);

/* Pre-size the block-step scratch for blocks of up to max_block_tokens tokens
 * (Hgt*Wid*frames), so that later blin_block_step calls allocate nothing
 * (for instance before capturing them in a CUDA graph). */
BLIN_API blin_status blin_state_reserve(blin_state *st, long max_block_tokens, blin_stream stream);

/* ---------------------------------------------------------------- prefill */

/* Workspace bytes blin_prefill needs for this shape (0 on invalid input).  A
 * call uses its workspace until its last kernel has finished: calls that may
 * run at the same time (on different streams) need separate workspaces. */
BLIN_API size_t blin_prefill_workspace_size(int B, int H, int d, const blin_geom *g);

/* Block-causal linear attention over a whole latent video (or a continuation).
 *   q, k, v  device [B][H][N][d] of dtype dt;  o  device [B][H][N][d] output,
 *            which must not overlap q, k or v
 *   st       optional cache.  NULL: start from S = 0, z = 0, t0 = 0.
 *            Otherwise start from its (S, z) with t0 = its t_next, and on
 *            return (in stream order) it holds the final (S, z) with
 *            t_next += T.
 *   workspace device scratch of at least blin_prefill_workspace_size bytes,
 *            16-byte aligned; contents on entry are ignored.
 * T = 0 is valid and does nothing.  Splitting the frames into several calls
 * at block boundaries gives the same rows as one call, and the final (S, z) is
 * bitwise equal to the one blin_block_step reaches over the same blocks.  A
 * call that ends inside a block lets that block's rows see only the frames
 * given so far; the next call's rows of the same block see the whole block.
 * Per-call limits (BLIN_ERR_SHAPE beyond them, before any launch): on the
 * tensor-core path fewer than 2^31 - 2^20 (head, state chunk) and (head, query
 * group) work units; on the CUDA-core path at most 65535 heads (B*H) and 65535
 * causal blocks.  Larger jobs split over heads or frames. */
BLIN_API blin_status blin_prefill(const void *q, const void *k, const void *v, void *o, blin_dtype dt,
                         int B, int H, int d, const blin_geom *g, blin_state *st,
                         void *workspace, size_t ws_bytes, blin_stream stream);

/* blin_prefill on operands in any strided layout (see blin_layout), so a
 * QKV projection's [B][N][H*d] output (news article, SVDQuant paragraph: the
 * QKV projections feed this attention) is read in place, with no transpose
 * into [B][H][N][d]: the tensor-core path addresses it through 4D tensor maps.
 * qkv_layout applies to q, k and v alike, o_layout to o; NULL means
 * contiguous [B][H][N][d].  Results are those of blin_prefill on the same
 * values, bit for bit.  Errors as for blin_prefill, plus BLIN_ERR_SHAPE /
 * BLIN_ERR_ALIGN for strides that break the rules of blin_layout.  o's rows
 * must not overlap each other or the inputs. */
BLIN_API blin_status blin_prefill_strided(const void *q, const void *k, const void *v, void *o, blin_dtype dt,
                                          int B, int H, int d, const blin_geom *g, const blin_layout *qkv_layout,
                                          const blin_layout *o_layout, blin_state *st, void *workspace,
                                          size_t ws_bytes, blin_stream stream);

/* ---------------------------------------------------------------- decode */

/* One autoregressive block, or the part of one that is ready (talk
 * transcript, block-causal walk-through: the new block reads the cached state
 * plus its own contribution; the sum is cached for the next block).
 *   q, k, v, o  device [B][H][g->T * g->Hgt * g->Wid][d] of dtype dt
 *   g           g->T = latent frames of this call (>= 1), g->block_frames = F,
 *               the causal block length; rope_split, theta, eps as for prefill
 *   commit      1: S += the call's K~^T V, z += sum phi(k), t_next += T.
 *               0: read-only pass (a denoising step of the same block);
 *                  the cache is left unchanged.
 * Positions continue from the cache: t_abs = t_next + t.  The call's frames
 * must lie in one causal block: (t_next % F) + T <= F, else BLIN_ERR_SHAPE
 * (a call that would cross a block boundary is rejected, never regrouped).
 * A call that starts a block and covers it whole reduces its keys exactly as
 * blin_prefill does, so a block-by-block stream gives bitwise the outputs and
 * the final (S, z) of one prefill over the same frames.  Needs scratch owned
 * by the state; the first call with a larger block grows it (allocation on
 * stream), blin_state_reserve avoids that.  Inside stream capture (a CUDA
 * graph) the scratch cannot grow: such a call returns BLIN_ERR_WORKSPACE, so
 * reserve (or run one block step) before capturing.  Per-call limits as for
 * blin_prefill. */
BLIN_API blin_status blin_block_step(const void *q, const void *k, const void *v, void *o, blin_dtype dt,
                            int B, int H, int d, const blin_geom *g, blin_state *st, int commit,
                            blin_stream stream);

/* blin_block_step on strided operands (see blin_prefill_strided). */
BLIN_API blin_status blin_block_step_strided(const void *q, const void *k, const void *v, void *o, blin_dtype dt,
                                             int B, int H, int d, const blin_geom *g, const blin_layout *qkv_layout,
                                             const blin_layout *o_layout, blin_state *st, int commit,
                                             blin_stream stream);

/* ---------------------------------------------------------------- NVFP4 inputs */

/* One NVFP4 operand [B][H][N][d] (news article, NVFP4 / SVDQuant paragraph: the
 * QKV projections run in NVFP4).  Element i of a token's d-vector is
 *   e2m1(code_i) * e4m3(scale[i / 16]) * global_scale
 * with code_i the E2M1 nibble i of the token's d/2 data bytes (even elements
 * in the low nibble; bit 3 sign, bits 2..1 exponent, bit 0 mantissa) and
 * scale the token's d/16 E4M3 bytes (one per 16 consecutive elements).
 *   data   device [B][H][N][d/2] bytes, 16-byte aligned
 *   scale  device [B][H][N][d/16] bytes, 16-byte aligned; the allocation must
 *          be a whole number of 16-byte units (scale bytes are copied in
 *          aligned 16-byte runs)
 *   global_scale  finite, > 0 */
typedef struct {
    const void *data;
    const void *scale;
    float global_scale;
} blin_nvfp4;

/* blin_prefill on NVFP4 q, k, v; o is bf16 [B][H][N][d].  The tensor-core
 * kernels decode the 4-bit values in shared memory (E2M1 x E4M3 products are
 * exact in bf16) and apply the global scales in fp32, so a token-head moves
 * 3 * (d/2 + d/16) + 2d bytes instead of 8d.  Needs the tensor-core path (the
 * compiled RoPE splits), else BLIN_ERR_SHAPE.  Workspace and state as for
 * blin_prefill; with power-of-two global scales the results are bitwise those
 * of blin_prefill on the decoded bf16 values. */
BLIN_API blin_status blin_prefill_nvfp4(const blin_nvfp4 *q, const blin_nvfp4 *k, const blin_nvfp4 *v, void *o,
                                        int B, int H, int d, const blin_geom *g, blin_state *st, void *workspace,
                                        size_t ws_bytes, blin_stream stream);

/* blin_block_step on NVFP4 q, k, v (see blin_prefill_nvfp4); o is bf16. */
BLIN_API blin_status blin_block_step_nvfp4(const blin_nvfp4 *q, const blin_nvfp4 *k, const blin_nvfp4 *v, void *o,
                                           int B, int H, int d, const blin_geom *g, blin_state *st, int commit,
                                           blin_stream stream);

/* ---------------------------------------------------------------- causal temporal convolution */

/* The Mix-FFN's causal block temporal convolution and its one-frame cache
 * (talk transcript, causal-FFN passage: in causal training a zero token sits
 * between two blocks, so no block sees the next one; a block sees the
 * previous block through that block's last token, which is cached and put in
 * front of the block).  Per batch entry, pixel and channel c, with taps
 * w[c] = (previous, current, next):
 *   y[t] = w[c][0] * x[t-1] + w[c][1] * x[t] + w[c][2] * x[t+1] + bias[c]
 * x[t-1] is the previous frame: from the call, or for the call's first frame
 * from the cache (zero before the video's first frame); x[t+1] counts only when
 * it lies in the same block of F = block_frames frames and in the call, else
 * zero.  Accumulation in fp32 in the order bias, previous, current, next;
 * outputs have the input dtype (bf16 rounded to nearest even). */
typedef struct blin_tconv_state blin_tconv_state; /* the last frame seen, [B][Hgt*Wid][C], and t_next */

/* Allocate a zeroed cache on the current device (t_next = 0).  C must be a
 * multiple of 8.  Its size is fixed: one frame, whatever the video length. */
BLIN_API blin_status blin_tconv_state_init(int B, int C, int Hgt, int Wid, blin_dtype dt, blin_stream stream,
                                           blin_tconv_state **out);
/* Free the cache (waits for the last call that used it).  NULL is a no-op. */
BLIN_API blin_status blin_tconv_state_free(blin_tconv_state *st);
/* Zero the cache and set t_next = 0 (a new video). */
BLIN_API blin_status blin_tconv_state_reset(blin_tconv_state *st, blin_stream stream);
/* Device pointer of the cached frame and the next absolute frame index (either may be NULL). */
BLIN_API blin_status blin_tconv_state_frame(const blin_tconv_state *st, void **frame, int *t_next);
/* Bytes of the cached frame: B * Hgt * Wid * C * element size. */
BLIN_API size_t blin_tconv_state_bytes(const blin_tconv_state *st);

/* Temporal convolution of frames [t0, t0 + g->T) of a latent video.
 *   x, y   device [B][g->T * g->Hgt * g->Wid][C] tokens (frame-major, channels
 *          innermost) of dtype dt, 16-byte aligned; y must not overlap x
 *   taps   device fp32 [C][3]; bias device fp32 [C] or NULL
 *   g      T, Hgt, Wid and block_frames are used (the RoPE fields are not)
 *   st     NULL: the call is the start of a video (t0 = 0).  Otherwise t0 =
 *          st's t_next and the call's first frame sees the cached frame.
 *   commit 1 (needs st): the cache takes the call's last frame, t_next += T;
 *          0: the cache is only read (a denoising pass of the same block).
 * Calls split at block boundaries, each committed, give bitwise the outputs of
 * one call over the same frames.  A call that ends inside a block gives its
 * last frame no next neighbour (that frame is not given yet). */
BLIN_API blin_status blin_tconv(const void *x, const float *taps, const float *bias, void *y, blin_dtype dt, int B,
                                int C, const blin_geom *g, blin_tconv_state *st, int commit, blin_stream stream);

/* ---------------------------------------------------------------- no allocation */

/* blin_prefill for callers that cannot allocate device memory (the method on
 * the SANA-Video pages has no counterpart; this is a library convenience).
 * Some callers have no device allocator of their own -- for example a plugin
 * inside a host framework that owns all device memory and hands out no
 * scratch buffers -- so they cannot pass the workspace blin_prefill needs.
 * This entry point takes the same arguments minus the workspace and uses a
 * fixed scratch area of blin_prefill_static_capacity() bytes (32 MiB) that is
 * part of the library's own device memory: every GPU that loads the library
 * holds it until the process exits, and nothing is allocated per call.
 *   - Shapes whose blin_prefill_workspace_size exceeds the capacity are
 *     rejected with BLIN_ERR_WORKSPACE and a message naming both sizes.
 *   - The first call in each CUDA context (normally one per device: the
 *     primary context) looks up the scratch area's device address
 *     (cudaGetSymbolAddress with that context current) and caches it under
 *     the context's unique id; make that first call before any stream capture.
 *     Another context made current later, or a new primary context after
 *     cudaDeviceReset, gets its own lookup.
 *   - All calls on a device share the one scratch area and it keeps the last
 *     call's contents.  Nothing in it needs to start at zero (each call writes
 *     everything it reads), but calls that overlap on the GPU, e.g. on two
 *     streams at once, race on it: serialise them.
 *   - Results are those of blin_prefill on the same arguments, bit for bit. */
BLIN_API blin_status blin_prefill_static(const void *q, const void *k, const void *v, void *o, blin_dtype dt,
                                         int B, int H, int d, const blin_geom *g, blin_state *st,
                                         blin_stream stream);

/* Bytes of blin_prefill_static's fixed scratch area. */
BLIN_API size_t blin_prefill_static_capacity(void);

/* ---------------------------------------------------------------- status */

/* Thread-local message for the last non-OK status of this thread ("" if none). */
BLIN_API const char *blin_last_error(void);

/* Which kernels this thread's last blin_prefill / blin_block_step that
 * launched any ran (a call rejected before launch leaves it unchanged):
 *   BLIN_PATH_TENSOR_CORE  bf16 storage with a compiled RoPE split whose
 *                          RoPE table fits shared memory: tcgen05/TMA kernels
 *   BLIN_PATH_CUDA_CORE    otherwise (fp32 storage, other splits): fp32 FMA
 *                          kernels.  Both compute the same function. */
typedef enum { BLIN_PATH_NONE = 0, BLIN_PATH_TENSOR_CORE = 1, BLIN_PATH_CUDA_CORE = 2 } blin_path;
BLIN_API int blin_last_path(void);

/* Read (synchronously) and clear the current device's kernel watchdog word:
 * 0 = no bounded wait ran out since the last call; otherwise a code naming the
 * wait that gave up.  Returns BLIN_ERR_DEVICE when the word was non-zero. */
BLIN_API blin_status blin_device_status(int *code);

/* Per-launch timing (profiling aid).  When `events` is non-NULL, the calling
 * thread's next blin_prefill / blin_block_step calls record events[2*i] just
 * before and events[2*i+1] just after launch slot i on the call's stream
 * (n >= 8 cudaEvent_t handles, owned by the caller): 0 RoPE table (CUDA-core
 * path only), 1 partial states, 2 block scan, 3 output.  NULL turns recording
 * off. */
BLIN_API blin_status blin_set_timing_events(void *const *events, int n);

/* Number of kernels this library has launched in this process so far (all
 * threads and devices; a profiling aid: the difference across a region counts
 * its launches).  A tensor-core prefill or block step launches 3 (partial
 * states, block scan, output; plus a 16-byte memset of its work counters),
 * the CUDA-core path 4 (RoPE table first). */
BLIN_API unsigned long long blin_launch_count(void);

/* Library version string. */
BLIN_API const char *blin_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BLIN_H */
