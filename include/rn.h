/*
 * rn.h -- C ABI of librn: batch-invariant zero-centred and gated RMSNorm,
 * forward and backward, for NVIDIA B200 (sm_100a).
 *
 * The operators
 * -------------
 * RL-Kernel PR #468, "[WS1][CUDA][Qwen3-Next] Gated RMSNorm CUDA kernel for the
 * GDN block", section "Summary" defines, per row x of width H:
 *
 *   rstd = rsqrt(mean_j(x_j^2) + eps)
 *   zero-centred:  y_j = x_j * rstd * (1 + w_j)         (weight offset 1)
 *   gated:         y_j = x_j * rstd * w_j * silu(z_j)   (weight offset 0,
 *                  norm before gate, one group per row, silu = z * sigmoid(z))
 *
 * and, in general (the displayed formula and the "Activation" bullet of the
 * same section), with a weight offset and a gate activation a:
 *
 *   y_j = x_j * rstd * u_j * a(z_j),  u_j = w_j + offset,  a = silu or sigmoid
 *
 * where the offset is added only when it is nonzero, so with offset 0 a -0.0
 * weight keeps its sign (the "Signed zero" bullet of that page's "Changes to
 * existing code, in detail").  The zero-centred operator is offset 1 with no
 * gate, the gated one offset 0 with silu; rmsnorm_fwd / rmsnorm_bwd take both
 * as arguments.
 *
 * The backward (the "Backward" bullet of the same section, and the calculus
 * of the forward), with g_j = 1 + w_j or w_j * silu(z_j) (in general
 * g_j = u_j * a(z_j), dz_j = dy_j * x_j * rstd * u_j * a'(z_j) and
 * dw_j sums dy_j * x_j * rstd * a(z_j)):
 *
 *   m     = mean_j(g_j * dy_j * x_j * rstd)
 *   dx_j  = rstd * (g_j * dy_j - x_j * rstd * m)
 *   dz_j  = dy_j * x_j * rstd * w_j * s_j * (1 + z_j * (1 - s_j))  (gated)
 *   dw_j  = sum over rows of dy_j * x_j * rstd [* silu(z_j) when gated]
 *
 * Numerical contract (RL-Kernel RFC #415, section 4 "Numerical contract"):
 *   - every sum accumulates in fp32 and every intermediate is fp32; the only
 *     narrowing is the round-to-nearest-even store of y, dx, dz (and of h,
 *     the residual sum, in rmsnorm_add_fwd);
 *   - the addition order depends on the width and dtype only: each thread
 *     adds its own elements in ascending order, a fixed xor butterfly joins
 *     the lanes of a row, a fixed pairwise tree joins the warps of a row.
 *     It never depends on the row count, the row's position, the launch
 *     geometry or the SM count, so a row's y, rstd, dx and dz are bitwise the
 *     same alone or inside any batch;
 *   - dw uses no atomics: rows are folded in ascending order inside 32-row
 *     leaves, and leaves are joined by a level-by-level pairwise tree whose
 *     shape depends on the row count only (rn_describe prints it); it is
 *     bitwise the same across runs and launch geometries, and a row left out
 *     by a row mask stands for the tree's identity (-0.0);
 *   - unsupported shapes fail closed with a status; there is no fallback.
 *
 * Data layout and ownership
 * -------------------------
 * x, z, dy, y, dx, dz: row-major contiguous [rows, width] of dtype `dt`
 *   (RN_BF16, RN_F16 or RN_F32); y, dx, dz take the dtype of x.
 * w: fp32 [width].  rstd: fp32 [rows].  dw: fp32 [width].
 * All pointers are DEVICE pointers on the device that is current when the
 * call is made, and `stream` is a cudaStream_t of that device (NULL = the
 * legacy default stream).  The caller owns all memory; the library never
 * allocates, frees or synchronises.  Every call only enqueues work on
 * `stream` and returns; results are ready when the stream reaches them.
 *
 * Errors
 * ------
 * Every argument is checked before anything is enqueued.  A failed check
 * returns its status and enqueues nothing:
 *   RN_E_ARG       rows < 0 or > 2^36, eps negative or not finite, the
 *                  weight offset not finite, an unknown activation, a
 *                  required pointer is NULL (or z / dz given without a
 *                  gate), or an output overlaps an input or another output
 *                  (except the in-place forms the residual-add calls allow);
 *   RN_E_DTYPE     dt is not RN_BF16, RN_F16 or RN_F32;
 *   RN_E_WIDTH     width is not a multiple of 8 in [8, 16384];
 *   RN_E_ALIGN     a tensor pointer is not 16-byte aligned (rstd: 4 bytes;
 *                  row_mask: any address);
 *   RN_E_WORKSPACE the backward's workspace is NULL or smaller than
 *                  norm_bwd_workspace_bytes(rows, width);
 *   RN_E_CUDA      a launch failed (rn_last_cuda_error() gives the code).
 * rows == 0 is valid: the forward enqueues nothing and the backward sets
 * every element of dw to -0.0, the empty sum (see rmsnorm_bwd's row_mask:
 * the same value as a call whose mask leaves out every row).
 */
#ifndef RN_H_
#define RN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RN_OK = 0,
    RN_E_ARG = 1,
    RN_E_DTYPE = 2,
    RN_E_WIDTH = 3,
    RN_E_ALIGN = 4,
    RN_E_WORKSPACE = 5,
    RN_E_CUDA = 6
} rn_status;

typedef enum {
    RN_F32 = 0,
    RN_BF16 = 1,
    RN_F16 = 2
} rn_dtype;

/* Gate activation a(z) (PR #468 Summary, "Activation" bullet; "swish" is
 * another name for silu).  RN_ACT_NONE: the ungated operator, no z. */
typedef enum {
    RN_ACT_NONE = 0,
    RN_ACT_SILU = 1,       /* a(z) = z * s(z),  s(z) = 1 / (1 + exp(-z)) */
    RN_ACT_SIGMOID = 2     /* a(z) = s(z) */
} rn_act;

/* A cudaStream_t, passed as a plain pointer so this header needs no CUDA. */
typedef void* rn_stream;

/*
 * General forward (PR #468 Summary, the displayed formula):
 *   y[r, j] = x[r, j] * rstd[r] * u[j] * a(z[r, j]),
 *   u[j] = w[j] + weight_offset when weight_offset != 0, else w[j] itself.
 * act selects a; with RN_ACT_NONE the factor a(z) is absent and z must be
 * NULL.  x, z: [rows, width] dt, read.  w: [width] fp32, read.
 * y: [rows, width] dt, written.  rstd: [rows] fp32, written, or NULL.
 * rstd depends on x, eps and width only: bitwise the same for every
 * activation and offset.
 */
rn_status rmsnorm_fwd(int64_t rows, int32_t width, float eps, float weight_offset,
                      rn_act act, rn_dtype dt, const void* x, const void* z,
                      const float* w, void* y, float* rstd, rn_stream stream);

/*
 * General backward, the gradient of sum(y * dy) for rmsnorm_fwd's y:
 *   g = u * a(z),  m = mean_j(g_j * dy_j * xh_j),  xh = x * rstd,
 *   dx = rstd * (g * dy - xh * m),  dz = dy * xh * u * a'(z),
 *   dw[j] = sum over rows of dy * xh * a(z)   (the offset is a constant).
 * row_mask: [rows] bytes, read, or NULL.  Rows with row_mask[r] == 0 are left
 *   out of dw (they add nothing, whatever their values -- padding may hold
 *   anything); dx and dz are written for every row.  A left-out row stands
 *   for the additive identity (-0.0) in dw's fixed tree, so the tree's shape
 *   still depends on the row count only.  dw over no contributing row is the
 *   empty sum, -0.0 in every column, whether every row is left out or
 *   rows == 0.  (PR #468 Notes: the dw entry point takes a mask.)
 * With RN_ACT_NONE, z and dz must be NULL.  Arguments otherwise as
 * gated_norm_bwd (workspace: norm_bwd_workspace_bytes).
 */
rn_status rmsnorm_bwd(int64_t rows, int32_t width, float eps, float weight_offset,
                      rn_act act, rn_dtype dt, const void* x, const void* z,
                      const float* w, const void* dy, const float* rstd,
                      const uint8_t* row_mask, void* dx, void* dz, float* dw,
                      void* ws, size_t ws_bytes, rn_stream stream);

/*
 * Residual-add forward (PR #468 Notes mention a norm that also adds a
 * residual; read as the usual fused form):
 *   h[r, j] = fmt(x[r, j] + r_in[r, j])   fp32 sum, rounded once to dt, written;
 *   y = rmsnorm_fwd of h (the stored, rounded h), rstd likewise.
 * x, r: [rows, width] dt, read.  h, y: [rows, width] dt, written; h may be
 * exactly x or exactly r (an in-place update of the residual stream), any
 * other overlap is RN_E_ARG.  Other arguments as rmsnorm_fwd.
 */
rn_status rmsnorm_add_fwd(int64_t rows, int32_t width, float eps, float weight_offset,
                          rn_act act, rn_dtype dt, const void* x, const void* r,
                          const void* z, const float* w, void* h, void* y, float* rstd,
                          rn_stream stream);

/*
 * Residual-add backward: h (from rmsnorm_add_fwd) takes x's place in
 * rmsnorm_bwd, and the gradient reaching h is the norm's plus dh, the
 * gradient of the residual output; x and r both receive it:
 *   dx = fmt(dnorm(h; dy) + dh)   (fp32 sum, one rounding);  dz, dw as rmsnorm_bwd.
 * dh: [rows, width] dt, read, or NULL (no gradient into h beyond the norm's);
 * dx may be exactly dh.  Other arguments as rmsnorm_bwd.
 */
rn_status rmsnorm_add_bwd(int64_t rows, int32_t width, float eps, float weight_offset,
                          rn_act act, rn_dtype dt, const void* h, const void* z,
                          const float* w, const void* dy, const void* dh,
                          const float* rstd, const uint8_t* row_mask, void* dx, void* dz,
                          float* dw, void* ws, size_t ws_bytes, rn_stream stream);

/*
 * Zero-centred RMSNorm forward (PR #468 Summary, with weight offset 1):
 * rmsnorm_fwd with weight_offset = 1 and RN_ACT_NONE.
 *   y[r, j] = x[r, j] * rstd[r] * (1 + w[j]).
 * x: [rows, width] dt, read.  w: [width] fp32, read.  y: [rows, width] dt,
 * written.  rstd: [rows] fp32, written, or NULL to skip it.
 */
rn_status norm_fwd(int64_t rows, int32_t width, float eps, rn_dtype dt,
                   const void* x, const float* w, void* y, float* rstd,
                   rn_stream stream);

/*
 * Gated RMSNorm forward (PR #468 Summary, weight offset 0, act = silu):
 * rmsnorm_fwd with weight_offset = 0 and RN_ACT_SILU.
 *   y[r, j] = x[r, j] * rstd[r] * w[j] * silu(z[r, j]).
 * The offset is never added, so a -0.0 weight keeps its sign.  rstd is
 * bitwise identical to norm_fwd's for the same x (same reduction).
 * x, z: [rows, width] dt.  w: [width] fp32.  y: [rows, width] dt.
 * rstd: [rows] fp32 or NULL.
 */
rn_status gated_norm_fwd(int64_t rows, int32_t width, float eps, rn_dtype dt,
                         const void* x, const void* z, const float* w, void* y,
                         float* rstd, rn_stream stream);

/*
 * Bytes of device workspace the backward needs for `rows` x `width`
 * (fp32 dw partials; independent of dtype and of the launch geometry).
 * 0 when rows <= 0 or width is unsupported.
 */
size_t norm_bwd_workspace_bytes(int64_t rows, int32_t width);

/*
 * Zero-centred RMSNorm backward.
 * x, dy: [rows, width] dt, read.  w: [width] fp32, read.
 * rstd: [rows] fp32 from norm_fwd, read; or NULL to recompute it (bitwise
 *   the same value norm_fwd writes).
 * dx: [rows, width] dt, written.  dw: [width] fp32, written (overwritten,
 *   not accumulated).
 * ws: device workspace of ws_bytes >= norm_bwd_workspace_bytes(rows, width),
 *   16-byte aligned; its contents on entry do not matter and are garbage on
 *   return.
 */
rn_status norm_bwd(int64_t rows, int32_t width, float eps, rn_dtype dt,
                   const void* x, const float* w, const void* dy,
                   const float* rstd, void* dx, float* dw,
                   void* ws, size_t ws_bytes, rn_stream stream);

/*
 * Gated RMSNorm backward: as norm_bwd, plus z ([rows, width] dt, read) and
 * dz ([rows, width] dt, written).  dz keeps the sign of a -0.0 weight.
 */
rn_status gated_norm_bwd(int64_t rows, int32_t width, float eps, rn_dtype dt,
                         const void* x, const void* z, const float* w,
                         const void* dy, const float* rstd, void* dx, void* dz,
                         float* dw, void* ws, size_t ws_bytes, rn_stream stream);

/*
 * Data-parallel dw (RFC #415 section 4: the result must not depend on rank
 * placement).  dw's declared tree over 32-row leaves is, from its third level
 * up, the same level-by-level pairwise tree over 256-row chunks, whose node for
 * chunk c is the tree over leaves 8c .. 8c+7 (fewer for a ragged last chunk).
 * So when a batch is split across ranks in row order on 256-row boundaries
 * (every rank but the last holds a multiple of 256 rows), each rank can return
 * its chunk partials, and the tree over all ranks' chunk partials in rank
 * order is bitwise the dw of one call over the whole batch.
 *
 * rmsnorm_bwd_chunk_count: ceil(rows / 256), the chunk partials of `rows`
 * rows (0 for rows < 0 or > 2^36).
 *
 * rmsnorm_bwd_chunks: rmsnorm_bwd (same arguments, same dx and dz, same
 * workspace), except that dw_chunks [rmsnorm_bwd_chunk_count(rows)][width]
 * fp32, written, receives the chunk partials instead of their fold.  rows == 0
 * writes nothing (dw_chunks may then be NULL).  A left-out row (row_mask) is
 * the identity -0.0, as in rmsnorm_bwd.
 */
int64_t rmsnorm_bwd_chunk_count(int64_t rows);
rn_status rmsnorm_bwd_chunks(int64_t rows, int32_t width, float eps, float weight_offset,
                             rn_act act, rn_dtype dt, const void* x, const void* z,
                             const float* w, const void* dy, const float* rstd,
                             const uint8_t* row_mask, void* dx, void* dz, float* dw_chunks,
                             void* ws, size_t ws_bytes, rn_stream stream);

/*
 * The level-by-level pairwise tree over n >= 1 rows of fp32 partials, in row
 * order (node 2i + node 2i+1 at each level, an odd last node carried up):
 * out[width] = tree(in[0], ..., in[n-1]).  Folding the chunk partials of
 * rmsnorm_bwd_chunks gives that call's dw bits; folding several ranks' chunk
 * partials concatenated in rank order gives the dw of the whole batch.
 * in: [n][width] fp32 device, read.  out: [width] fp32 device, written.
 * ws: device workspace of ws_bytes >= rn_fold_tree_workspace_bytes(n, width),
 * 16-byte aligned, contents irrelevant.  No overlap between in, out and ws.
 * RN_E_ARG for n < 1 or > 2^36; other errors as the backward's.
 */
size_t rn_fold_tree_workspace_bytes(int64_t n, int32_t width);
rn_status rn_fold_tree(int64_t n, int32_t width, const float* in, float* out, void* ws,
                       size_t ws_bytes, rn_stream stream);

/*
 * Joins n rows of fp32 dw partials with the same level-by-level pairwise tree
 * the backward uses: out[width] = tree(in[0], ..., in[n-1]), in row order.
 * A backward call's dw is the root of that tree over its 32-row leaves, so
 * when a batch is split across data-parallel ranks in order and every rank
 * holds the same power-of-two number of leaves, folding the ranks' dw in rank
 * order gives exactly (bitwise) the dw of one call over the whole batch.
 * in: [n][width] fp32 device, read; out: [width] fp32 device, written; no
 * workspace.  1 <= n <= 256, else RN_E_ARG; out must not overlap in.
 */
rn_status rn_fold_rows(int64_t n, int32_t width, const float* in, float* out,
                       rn_stream stream);

/*
 * Gated RMSNorm backward that allocates nothing: the same computation,
 * arguments and results as gated_norm_bwd, but the dw-partial scratch is a
 * fixed 8 MiB block of static device memory inside this library instead of a
 * caller-supplied workspace.  (RFC #415 and PR #468 have no counterpart of
 * this call; it is an addition of this library.)
 *
 * Who needs it: hosts that hand a library only the input and output buffers of
 * each call and own every other byte of device memory -- plugin interfaces,
 * runtimes with a fixed memory plan, code that must not call cudaMalloc
 * because it would synchronise the device or fall outside the host's memory
 * accounting.  Such a caller has no workspace to pass and cannot allocate one.
 *
 * Limits and sharing:
 *  - the scratch holds 8 MiB (8388608 bytes), so a call needs
 *    norm_bwd_workspace_bytes(rows, width) <= 8388608 (e.g. 262144 rows of
 *    width 128 use 4.7 MiB); larger shapes return RN_E_WORKSPACE and enqueue
 *    nothing;
 *  - every GPU on which this library runs kernels keeps the 8 MiB until the
 *    process exits;
 *  - the first call on each device looks up the scratch's device address (with
 *    that device current) and keeps it; make that first call before any
 *    stream capture.  The address kept is that of the device's context at
 *    the time: after cudaDeviceReset (or any other reset of that context)
 *    the library's device memory is set up anew and the kept address is
 *    stale, so do not use this call on a device after resetting it;
 *  - all calls on a device share the one scratch, which keeps whatever the last
 *    call left there (nothing in it needs to start at zero).  Calls that can
 *    run at the same time on the GPU -- on different streams, or from several
 *    host threads -- race on it and give wrong dw; order them on one stream.
 * The call never allocates or frees memory (no cudaMalloc/cudaFree, no
 * allocating library routine).
 */
rn_status gated_norm_bwd_static_ws(int64_t rows, int32_t width, float eps, rn_dtype dt,
                                   const void* x, const void* z, const float* w,
                                   const void* dy, const float* rstd, void* dx, void* dz,
                                   float* dw, rn_stream stream);

/*
 * Provenance record (RFC #415 section 4, point 8): a static, NUL-terminated
 * string naming the kernels, the reduction schedule and tree, and the
 * accumulator for (width, dt); "unsupported" for an invalid pair.  The
 * pointer stays valid until the next rn_describe call on the same thread.
 */
const char* rn_describe(int32_t width, rn_dtype dt);

/*
 * Number of kernels one norm_bwd / gated_norm_bwd call with these sizes
 * enqueues under the current geometry (the backward kernel plus its dw fold
 * passes); 1 when rows == 0 (the kernel that sets dw to -0.0); 0 when the
 * shape is unsupported.  The forward always enqueues one kernel when rows > 0.
 */
int32_t rn_bwd_launches(int64_t rows, int32_t width, rn_dtype dt);

/* Short message for a status code (static string). */
const char* rn_status_string(rn_status s);

/* The cudaError_t behind this thread's last RN_E_CUDA (0 if none). */
int rn_last_cuda_error(void);

/*
 * Number of kernels the last call made on this thread enqueued (forward,
 * backward, chunk backward, rn_fold_tree, rn_fold_rows; 0 after a failed
 * check or in validate-only mode).  For bookkeeping: a benchmark counts the
 * library's kernels per step with it.
 */
int32_t rn_last_launches(void);

/*
 * Test knobs (process-wide; not for production use).  They change how work
 * is mapped to CTAs -- never the arithmetic -- so results must not change:
 *   max_ctas        cap on every grid (CTAs loop over the rest); 0 = default.
 *   leaves_per_cta  32-row leaves one backward CTA folds together (a power
 *                   of two, clamped to what the width allows); 0 = default.
 *   fold_rows       rows of partials one fold CTA reduces per pass (a power
 *                   of two in [8, 256]); 0 = default.
 * Returns RN_E_ARG for a negative value or a non-power-of-two.
 */
rn_status rn_test_set_geometry(int32_t max_ctas, int32_t leaves_per_cta,
                               int32_t fold_rows);

/*
 * Test knob: when on, every entry point runs its argument checks and returns
 * their status without touching the GPU (no CUDA call at all), so the checks
 * can be exercised on a machine without one.  Off by default.
 */
void rn_test_set_validate_only(int32_t on);

/*
 * Test entry point: out[i] = the reciprocal the sigmoid uses, for inputs
 * d[i] in [1, 2] (n floats, device pointers; steps = 1 or 2 Newton steps;
 * RN_E_ARG otherwise).  Lets a test compare it with IEEE division over every
 * float in [1, 2].
 */
rn_status rn_test_rcp_1to2(int64_t n, const float* d, float* out, int32_t steps,
                           rn_stream stream);

/*
 * Test entry point: out[i] = the gate's sigmoid 1 / (1 + e^{-z[i]}) as the
 * row kernels evaluate it (n floats, device pointers; e^{-|z|} from CUDA's
 * expf, the reciprocal of rn_test_rcp_1to2 with one step); RN_E_ARG for n < 0
 * or a NULL pointer with n > 0.  Lets a test bound it against the exact
 * function, subnormal tail included.
 */
rn_status rn_test_sigmoid(int64_t n, const float* z, float* out, rn_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* RN_H_ */
