/*
 * gspn.h -- C ABI of libgspn, the GSPN 2D line-scan propagation on NVIDIA
 * B200 (sm_100a).
 *
 * The operator (cited by page title and section):
 *
 *   For one (batch b, channel c) plane and one scan direction, lines are
 *   visited in scan order and every line i is computed from the previous one:
 *
 *       h_i[j] = sum_{k=0..2} w_{i,j,k} * h_{i-1}[j+k-1] + lambda_i[j] * x_i[j]
 *
 *   "Parallel Sequence Modeling via Generalized Spatial Propagation Network"
 *   (GSPN, CVPR 2025 reading notes), Key design 1: the recurrence
 *   h_i = w_i h_{i-1} + lambda_i (.) x_i with row-stochastic w_i, made so by a
 *   sigmoid on the non-zero entries of each row and a normalisation of the
 *   row; Key design 2: w_i is tridiagonal (each pixel reads the three
 *   adjacent pixels of the previous row or column), four scan directions;
 *   Key design 3: the local variant propagates each of g groups on its own.
 *   "GSPN-2: Efficient Parallel Sequence Modeling", Justification for
 *   Channel-Agnostic Propagation: one tap set shared by all channels
 *   (W kron I(C)) with per-channel gains lambda.
 *
 *   Readings this library fixes (the pages leave them open):
 *   - weights: s_k = sigmoid(logit_k) for the taps whose source j+k-1 lies in
 *     the line, w_k = s_k / sum of the valid s; taps outside the line have
 *     w = 0 and their logits are ignored;
 *   - h_{-1} = 0, so the first line of a scan (and of each local group) is
 *     lambda * x;
 *   - the four directions are merged by an unweighted sum;
 *   - local groups cut the scan axis into g equal parts; taps still span the
 *     whole line.
 *
 * Directions and coordinates.  Bit d of dir_mask enables direction d:
 *   GSPN_DIR_T2B (lines = rows, top to bottom),    GSPN_DIR_B2T (bottom to top),
 *   GSPN_DIR_L2R (lines = columns, left to right), GSPN_DIR_R2L (right to left).
 * Tap k of a pixel reads the neighbour at offset k-1 along the line (column
 * offset for row scans, row offset for column scans) in the previous line.
 * The logits of a pixel's taps are stored at that pixel.
 *
 * Layouts (dense, row-major, element type `dtype`):
 *   x, out, dout, dx   [B, C, H, W]
 *   lambda, dlambda    [D, B, C, H, W]
 *   logits, dlogits    [D, B, Cw, 3, H, W]   Cw = 1 when shared_weights, else C
 * D = popcount(dir_mask); the D axis lists the enabled directions in the bit
 * order T2B, B2T, L2R, R2L.  Arithmetic is fp32 throughout; bf16 outputs are
 * rounded to nearest-even once, at the store.
 *
 * Ownership and streams.  Every pointer is a device pointer owned by the
 * caller, including the workspace.  gspn_fwd and gspn_bwd allocate no memory,
 * keep no state between calls and never synchronise the stream (unless
 * gspn_set_sync_check is on); calls are asynchronous on `stream` (a
 * cudaStream_t; NULL = legacy default stream).  The one exception is
 * gspn_fwd_noalloc, whose scratch is a fixed device array of the library
 * itself (see there).  Process-wide settings: the device wait limit, the
 * synchronous check and the stall test hook below.
 * Outputs are overwritten, never accumulated into.  Inputs and outputs must
 * not alias.  Concurrent calls on different streams may not share a
 * workspace.
 *
 * Errors.  Arguments are checked on the host before any launch; a rejected
 * call launches nothing and returns:
 *   GSPN_ERR_INVALID_ARG  null descriptor or pointer, a dimension < 1, a
 *                         dir_mask of 0 or with bits above 8, groups < 1, or
 *                         groups not dividing the scan length of an enabled
 *                         direction (H for T2B/B2T, W for L2R/R2L), or an
 *                         element count that overflows;
 *   GSPN_ERR_UNSUPPORTED  an unknown dtype;
 *   GSPN_ERR_ALIGNMENT    a tensor pointer not 16-byte aligned;
 *   GSPN_ERR_WORKSPACE    workspace smaller than gspn_workspace_size();
 *   GSPN_ERR_CUDA         a CUDA runtime error at or before launch (the
 *                         runtime's own error is left for cudaGetLastError);
 *   GSPN_ERR_SCRATCH_LIMIT  (gspn_fwd_noalloc only) the problem does not fit
 *                         the library's fixed scratch.
 * Device-side timeouts.  The TMA-fed kernels (the compact 64x64 and 128x128
 * paths, which gspn_variant_name names "compact*_tma_*", and the compact
 * large-plane kernels, "large_compact_*") hand data between warps through
 * shared-memory barriers.  Every such wait is bounded (2 s by default,
 * gspn_set_wait_limit_ns); when one runs out, the kernel records an error
 * word in its workspace, waits for its own copies in flight, frees its tensor
 * memory and returns, so the GPU stays usable but the outputs are not
 * valid.  The launching call has already returned GSPN_OK by then; the caller
 * learns of the timeout with gspn_device_status (or gspn_noalloc_status),
 * which synchronises the stream and returns
 *   GSPN_ERR_TIMEOUT      a bounded device wait of the last call that used
 *                         this workspace ran out.
 * With gspn_set_sync_check(1) every gspn_fwd / gspn_bwd / gspn_fwd_noalloc
 * synchronises its stream itself and returns GSPN_ERR_TIMEOUT directly (a
 * debugging mode: it serialises the host with the GPU).
 * No exception or signal crosses the ABI.
 */
#ifndef GSPN_H_
#define GSPN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GSPN_OK = 0,
    GSPN_ERR_INVALID_ARG = 1,
    GSPN_ERR_UNSUPPORTED = 2,
    GSPN_ERR_ALIGNMENT = 3,
    GSPN_ERR_WORKSPACE = 4,
    GSPN_ERR_CUDA = 5,
    GSPN_ERR_TIMEOUT = 6,
    GSPN_ERR_SCRATCH_LIMIT = 7
} gspn_status;

typedef enum { GSPN_F32 = 0, GSPN_BF16 = 1 } gspn_dtype;

enum { GSPN_DIR_T2B = 1, GSPN_DIR_B2T = 2, GSPN_DIR_L2R = 4, GSPN_DIR_R2L = 8 };

typedef struct {
    int64_t B, C, H, W;      /* batch, channels, rows, columns; each >= 1 */
    uint32_t dir_mask;        /* OR of GSPN_DIR_* */
    int32_t groups;           /* local groups along each scan axis; 1 = global scan */
    int32_t shared_weights;   /* 1: one tap set per (b, pixel, direction) for all channels */
    int32_t dtype;            /* gspn_dtype of every tensor */
} gspn_desc;

/* Bytes of device workspace a gspn_fwd (backward = 0) or gspn_bwd
 * (backward = 1) call with this descriptor needs; 0 if none.  Returns 0 for a
 * descriptor gspn_fwd/gspn_bwd would reject.  The workspace must be 256-byte
 * aligned.  Its contents on entry are irrelevant. */
size_t gspn_workspace_size(const gspn_desc* desc, int backward);

/* Forward: out = sum over enabled directions d of h^(d), the line scan above
 * ("Parallel Sequence Modeling via Generalized Spatial Propagation Network",
 * Key designs 1-3; "GSPN-2: Efficient Parallel Sequence Modeling",
 * channel-shared taps).  x: [B,C,H,W]; logits: [D,B,Cw,3,H,W] raw
 * (pre-sigmoid) tap logits; lambda: [D,B,C,H,W]; out: [B,C,H,W].
 * workspace/ws_bytes: device scratch of at least gspn_workspace_size(desc, 0)
 * bytes (may be NULL when that is 0). */
gspn_status gspn_fwd(const gspn_desc* desc, const void* x, const void* logits, const void* lambda, void* out,
                     void* workspace, size_t ws_bytes, void* stream);

/* Backward of gspn_fwd for upstream gradient dout ([B,C,H,W]): writes
 * dx = dL/dx ([B,C,H,W], summed over directions), dlogits = dL/dlogits
 * ([D,B,Cw,3,H,W]; summed over channels when shared_weights; zero for the
 * logits of group-start lines and of taps outside the line) and
 * dlambda = dL/dlambda ([D,B,C,H,W]).  The same kernel-launch design as the
 * forward ("GSPN-2: Efficient Parallel Sequence Modeling", Backward
 * Benchmark): each direction's lines are recomputed on chip and its adjoint
 * h-gradient is run from the last line back to the first.
 * workspace: at least gspn_workspace_size(desc, 1) bytes. */
gspn_status gspn_bwd(const gspn_desc* desc, const void* x, const void* logits, const void* lambda,
                     const void* dout, void* dx, void* dlogits, void* dlambda, void* workspace, size_t ws_bytes,
                     void* stream);

/* Forward without any caller-provided workspace and without allocating.
 *
 * No counterpart in the GSPN pages: this is a convenience of this library for
 * callers that cannot allocate device memory -- code that runs under a host
 * framework which owns all device memory through its own pool and forbids
 * direct cudaMalloc, code on a latency-critical path where cudaMalloc/cudaFree
 * would block or synchronize the device, and plugins handed only the tensors
 * they read and write.  Such callers pass inputs and outputs only.
 *
 * The scratch this forward needs (an error word and the normalised tap-weight
 * table, 128 KB per batch image) lives in a fixed array in the library's
 * device memory, 4 MiB + 256 bytes, which every GPU that loads the library
 * holds until the process exits.  Hence the limits: only descriptors that run
 * the compact 64x64 forward (bf16, shared_weights = 1, dir_mask = 15,
 * H = W = 64, C a multiple of 8) are accepted, with B <= 32.  Larger batches
 * return GSPN_ERR_SCRATCH_LIMIT and other descriptors GSPN_ERR_UNSUPPORTED,
 * both before any launch; argument errors are reported as by gspn_fwd.
 *
 * Every call looks up the array's device address in the current context
 * (cudaGetSymbolAddress; in host code the array's name is not a device
 * address), so a context torn down and recreated (cudaDeviceReset) gets the
 * new address.  With lazy module loading (the CUDA 12 default) the first call
 * on a device also makes the runtime load the module, which places the array:
 * make that first call before any stream capture begins.  All calls share the
 * one array and each call rewrites what it reads, so results never depend on
 * an earlier call, but calls whose execution overlaps on the GPU (different
 * streams, or graphs replayed concurrently) race on it: serialise them.
 * Beyond that first module load, nothing is allocated or freed, here or in
 * any library routine this calls.  gspn_noalloc_status reads the array's
 * error word. */
gspn_status gspn_fwd_noalloc(const gspn_desc* desc, const void* x, const void* logits, const void* lambda,
                             void* out, void* stream);

/* Synchronises `stream`, then reports how the last gspn_fwd (backward = 0)
 * or gspn_bwd (backward = 1) call with this descriptor and this workspace
 * ended on the device: GSPN_ERR_TIMEOUT if one of its bounded waits ran out
 * (its outputs are then invalid), GSPN_ERR_CUDA if the stream reports a CUDA
 * error, else GSPN_OK.  Kernel families without device-side waits always
 * give GSPN_OK after the synchronisation.  workspace: the one that call
 * used (may be NULL only for those families).  No counterpart in the GSPN
 * pages: it is how a caller learns of a timeout (see "Device-side timeouts"
 * above). */
gspn_status gspn_device_status(const gspn_desc* desc, int backward, const void* workspace, void* stream);

/* The same for the last gspn_fwd_noalloc call: synchronises `stream` and reads
 * the error word of the library's fixed scratch. */
gspn_status gspn_noalloc_status(void* stream);

/* Sets the limit, in nanoseconds, of every device-side wait of the TMA-fed
 * kernels on data, a pipeline stage or another warp, for launches made after
 * the call, process-wide; 0 restores the default of 2 s.  Returns the
 * previous limit.  Waits that only drain a kernel's own copies or release its
 * tensor memory keep fixed bounds (0.1 s and 20 s).  Thread-safe. */
uint64_t gspn_set_wait_limit_ns(uint64_t limit_ns);

/* on != 0: every later gspn_fwd, gspn_bwd and gspn_fwd_noalloc call
 * synchronises its stream and returns GSPN_ERR_TIMEOUT itself when a wait ran
 * out (a debugging mode).  Returns the previous setting.  Process-wide. */
int gspn_set_sync_check(int on);

/* Test hook for the timeout path.  on != 0: in every later launch of a
 * TMA-fed kernel, one warp of the first CTA begins with a wait on a barrier
 * that only its own final arrival can complete, so that wait runs out after
 * the wait limit and the kernel ends through its error path (the other warps'
 * waits then run out in turn).  No fault, trap or unbounded wait is involved.
 * Returns the previous setting.  Process-wide; off by default. */
int gspn_set_stall_test(int on);

/* ---- Compressed propagation block --------------------------------------------
 *
 * y = U . RMSNorm_k( sum_d alpha[d,k] scan_d(V . x) ) . gamma, per pixel:
 *   xp[b,k]  = sum_c V[k,c] x[b,c]                  proxy projection to Cp channels
 *   h_d[b,k] = the GSPN scan of xp[b,k] in direction d (channel-shared taps,
 *              per-channel lambda, local groups as in gspn_fwd)
 *   m[b,k]   = sum_d alpha[d,k] h_d[b,k]             learnable merger
 *   n[b,k]   = gamma[k] m[b,k] / sqrt(mean_k m[b,k]^2 + eps)   (norm = 1; n = m if 0)
 *   y[b,c]   = sum_k U[c,k] n[b,k]                   projection back to C channels
 * Sources: "GSPN-2: Efficient Parallel Sequence Modeling" (OpenReview response,
 * "Relate Compressive Proxy Dimension to Low-rank Approximation": a linear
 * layer to C_proxy channels, the recurrence there, the projection back);
 * "Parallel Sequence Modeling via Generalized Spatial Propagation Network",
 * Key design 2 (the four directions aggregated by a learnable merger);
 * "Scaling Parallel Sequence Models to Vision Foundation Models", abstract (a
 * compressed latent-space propagation block with fused normalisation).  The
 * pages give neither the merger's nor the normalisation's formula: this
 * library reads them as one weight per (direction, proxy channel) and as an
 * RMS normalisation over the proxy channels of each pixel with a per-channel
 * gain (a LayerNorm over 2 proxy channels would collapse to +-1).
 *
 * Layouts (dense, row-major): x, y [B,C,H,W] bf16; v_proj [Cp,C] bf16;
 * u_proj [C,Cp] bf16; lambda [4,B,Cp,H,W] bf16; logits [4,B,1,3,H,W] bf16
 * (one tap set per pixel and direction for all proxy channels); alpha [4,Cp]
 * fp32; gamma [Cp] fp32.  The 4 axis is T2B, B2T, L2R, R2L.  Arithmetic is
 * fp32 (the projections on the tensor cores with bf16 operands: x, V and U as
 * stored, n rounded to bf16 once); y is rounded to bf16 once.
 * Limits (else GSPN_ERR_UNSUPPORTED): 1 <= Cp <= 32, H and W <= 128, C, H and
 * W multiples of 8, C <= 3072 (Cp <= 16) or 1536 (Cp <= 32).
 * Errors and ownership as for gspn_fwd; a bounded device wait that runs out
 * is reported by gspn_block_device_status. */
typedef struct {
    int64_t B, C, H, W;  /* batch, channels, rows, columns; each >= 1 */
    int32_t Cp;          /* proxy channels */
    int32_t groups;      /* local groups along each scan axis; 1 = global scan */
    int32_t norm;        /* 1: RMS normalisation over the proxy channels */
    float eps;           /* 0 <= eps <= 1, added to the mean square */
} gspn_block_desc;

/* Bytes of device workspace (256-byte aligned) gspn_block_fwd needs; 0 for a
 * descriptor it would reject. */
size_t gspn_block_workspace_size(const gspn_block_desc* desc);

gspn_status gspn_block_fwd(const gspn_block_desc* desc, const void* x, const void* v_proj, const void* logits,
                           const void* lambda, const float* alpha, const float* gamma, const void* u_proj, void* y,
                           void* workspace, size_t ws_bytes, void* stream);

/* As gspn_device_status, for the last gspn_block_fwd with this workspace. */
gspn_status gspn_block_device_status(const gspn_block_desc* desc, const void* workspace, void* stream);

/* Number of kernel launches one gspn_fwd (backward = 0) / gspn_bwd
 * (backward = 1) call with this descriptor issues; 0 for a descriptor the
 * call would reject. */
int gspn_launches_per_call(const gspn_desc* desc, int backward);

/* Name of the forward (backward = 0) or backward (backward = 1) kernel
 * variant this descriptor dispatches to, for logs and benchmarks; a static
 * string, "invalid" for a rejected descriptor. */
const char* gspn_variant_name(const gspn_desc* desc, int backward);

/* Static, human-readable text of a status code. */
const char* gspn_status_string(gspn_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int gspn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GSPN_H_ */
