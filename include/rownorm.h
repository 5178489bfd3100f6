/*
 * rownorm.h -- fused last-axis row normalization on NVIDIA B200 (sm_100a).
 *
 * C ABI of librownorm.so. Every entry point takes plain pointers and sizes;
 * no C++ or framework types cross this boundary.
 *
 * Operations (what each computes is stated with the function):
 *   rn_rms_norm            RMSNorm    -- "Emily.Fast", rms_norm/3, and the
 *                                        composed RMSNorm of "Fused
 *                                        transformer kernels on Emily",
 *                                        Part 1.
 *   rn_layer_norm          LayerNorm  -- "Emily.Fast", layer_norm/4.
 *   rn_dual_head_rms_norm  query/key head RMSNorm, both outputs from one
 *                          launch -- "norm_fusion.rs" (mlx_c_rust compile),
 *                          MlxCompiledDualHeadNorm and
 *                          apply_compiled_dual_head_norm.
 *
 * Common conventions
 *   Views. A tensor is passed as an rn_view: `rows` rows of `dim` elements,
 *   the elements of a row contiguous (unit stride), consecutive rows
 *   `row_stride` elements apart (row_stride >= dim). Any leading dimensions
 *   of a tensor are folded into `rows`. Normalization always runs over the
 *   last axis ("Emily.Bumblebee.FastKernels", What's not rewritten: only
 *   norms over the last axis are fused).
 *   Element types. RN_F32 (IEEE binary32) or RN_BF16 (bfloat16). Inputs,
 *   outputs, weights and biases of one call share one element type. All
 *   arithmetic is binary32 with binary32 accumulation; the result is rounded
 *   once (round to nearest even) to the output element type.
 *   eps. A binary32 value >= 0, finite (norm_fusion.rs keeps the epsilon as
 *   f32 bits). It is added to the mean square (RMSNorm) or the variance
 *   (LayerNorm) inside the square root.
 *   Memory. Every pointer is a device pointer on the calling thread's current
 *   CUDA device (memory from cudaMalloc or a framework allocator). The
 *   caller owns all memory; the library allocates nothing and keeps no
 *   per-call state. Base pointers must be aligned to the element size.
 *   Streams. `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   Calls are asynchronous: they enqueue one kernel launch and return.
 *   Aliasing. An output view may be identical to its input view (same data
 *   pointer and row stride: in place). Any other overlap between an output
 *   and any input or other output is rejected with RN_ERR_OVERLAP.
 *   Errors. Every argument is validated on the host before anything is
 *   enqueued; a rejected call launches nothing and returns a nonzero
 *   rn_status. There is no fallback to another implementation: inputs the
 *   kernels do not support are rejected, never silently degraded.
 *   rows == 0 is valid and enqueues nothing.
 *   Determinism. The summation order of every row is fixed by (element type,
 *   dim, and the 16-byte phase of the row's address); repeated calls on the
 *   same data and addresses return bit-identical results, independently of
 *   the grid size. rn_dual_head_rms_norm returns exactly the bits of two
 *   rn_rms_norm calls on the same views.
 */
#ifndef ROWNORM_H_
#define ROWNORM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define RN_API __attribute__((visibility("default")))
#else
#define RN_API
#endif

#define RN_ABI_VERSION 3

/* Widest rows the register kernels hold (every op): a row stays on chip
 * between reading and writing, so x is read from HBM exactly once. The fused
 * ops reject wider rows with RN_ERR_UNSUPPORTED. rn_rms_norm and
 * rn_layer_norm take wider rows, up to RN_MAX_DIM_STREAM, through streaming
 * kernels that read each row once per pass (two passes for RMSNorm, three for
 * LayerNorm; the later ones from L2 while the rows in flight fit there). */
#define RN_MAX_DIM_BF16 32768
#define RN_MAX_DIM_F32 16384
#define RN_MAX_DIM_STREAM 4194304
/* rn_dual_head_rms_norm: both head dims at most this (one launch keeps the
 * query and key rows in one warp-level kernel). */
#define RN_MAX_HEAD_DIM 1024

typedef enum rn_dtype { RN_F32 = 0, RN_BF16 = 1 } rn_dtype;

typedef enum rn_status {
    RN_OK = 0,
    RN_ERR_NULL = 1,        /* a required pointer is NULL                     */
    RN_ERR_SHAPE = 2,       /* rows < 0, dim < 1, row_stride < dim, or views  */
                            /* of one call disagree in rows/dim               */
    RN_ERR_DTYPE = 3,       /* unknown element type or mixed element types    */
    RN_ERR_EPS = 4,         /* eps is negative, NaN or infinite               */
    RN_ERR_ALIGN = 5,       /* a pointer not aligned to its element size      */
    RN_ERR_OVERLAP = 6,     /* an output partially overlaps an input/output  */
    RN_ERR_UNSUPPORTED = 7, /* dim beyond RN_MAX_DIM_STREAM (RMSNorm,         */
                            /* LayerNorm) or RN_MAX_DIM_BF16/F32 (fused ops), */
                            /* or a dual head dim beyond RN_MAX_HEAD_DIM      */
    RN_ERR_CUDA = 8         /* the CUDA runtime reported an error (device    */
                            /* query or launch); see rn_last_error()          */
} rn_status;

/*
 * A [rows, dim] view whose last axis is contiguous. Rows either sit
 * row_stride elements apart (inner_rows = 0), or form blocks of inner_rows
 * rows: row r starts at (r / inner_rows) * outer_stride + (r % inner_rows)
 * * row_stride elements from data. The second form describes head rows
 * sliced out of a packed buffer, e.g. the query heads [tokens, Hq, D] of a
 * [tokens, (Hq + 2 Hk) * D] QKV projection ("kernel_micro_ab.rs", section 2:
 * the packed QKV op writes the head buffers): inner_rows = Hq, row_stride =
 * D, outer_stride = (Hq + 2 Hk) * D. The norm stays on the last axis
 * ("Emily.Bumblebee.FastKernels", What's not rewritten); only the row layout
 * widens.
 */
typedef struct rn_view {
    void *data;           /* device pointer to element [0, 0]                 */
    int64_t rows;         /* number of rows, >= 0                              */
    int64_t dim;          /* elements per row (the normalized axis), >= 1      */
    int64_t row_stride;   /* elements between the starts of consecutive rows  */
                          /* (of one block when inner_rows > 0)               */
    int32_t dtype;        /* rn_dtype                                          */
    int64_t inner_rows;   /* 0: one row stride; > 0: rows per block            */
    int64_t outer_stride; /* inner_rows > 0: elements between block starts;   */
                          /* >= (inner_rows - 1) * row_stride + dim            */
} rn_view;

/*
 * RMSNorm of every row:  y[r, j] = x[r, j] * rsqrt(mean_i(x[r, i]^2) + eps) * w[j]
 * ("Emily.Fast", rms_norm/3; composed form x / sqrt(mean(x^2) + eps) * w in
 * "Fused transformer kernels on Emily", Part 1).
 *   x       input view.
 *   weight  device pointer to dim elements of x's type, or NULL (all ones).
 *   eps     binary32, >= 0 and finite.
 *   y       output view, same rows, dim and dtype as x (row_stride may
 *           differ); may be x itself.
 * Returns RN_OK or an rn_status; nothing is enqueued on error.
 */
RN_API int rn_rms_norm(const rn_view *x, const void *weight, float eps,
                       const rn_view *y, void *stream);

/*
 * LayerNorm of every row:
 *   mean = mean_i x[r, i];  var = mean_i (x[r, i] - mean)^2   (population)
 *   y[r, j] = (x[r, j] - mean) * rsqrt(var + eps) * w[j] + b[j]
 * ("Emily.Fast", layer_norm/4).
 *   weight, bias  device pointers to dim elements of x's type, or NULL
 *                 (weight all ones / bias all zeros).
 * Other arguments as rn_rms_norm. A row whose elements are all equal returns
 * exactly the bias (its deviations are exactly zero).
 */
RN_API int rn_layer_norm(const rn_view *x, const void *weight, const void *bias,
                         float eps, const rn_view *y, void *stream);

/*
 * Dual-output query/key head RMSNorm in ONE kernel launch
 * ("norm_fusion.rs", MlxCompiledDualHeadNorm / apply_compiled_dual_head_norm):
 *   yq = rms_norm(q, wq, eps),  yk = rms_norm(k, wk, eps)
 * Queries first, keys second; one eps shared by both. q [T*Hq, Dq] and
 * k [T*Hk, Dk] are the head rows (leading dims folded into rows); Dq and Dk
 * may differ and must each be <= RN_MAX_HEAD_DIM. q and k share one dtype.
 *   wq, wk  device pointers to Dq / Dk elements; both REQUIRED (non-NULL).
 *   yq, yk  outputs shaped like q and k; each may be its own input.
 * The bits of yq and yk equal those of rn_rms_norm(q, wq, eps, yq) and
 * rn_rms_norm(k, wk, eps, yk).
 */
RN_API int rn_dual_head_rms_norm(const rn_view *q, const rn_view *k,
                                 const void *wq, const void *wk, float eps,
                                 const rn_view *yq, const rn_view *yk,
                                 void *stream);

/*
 * Residual add + RMSNorm in one pass ("norm_fusion.rs", module doc comment:
 * the elementwise-producer fusion kept composed until a kernel pins the
 * summation order; this library's order is fixed and documented):
 *   h[r, j] = x[r, j] + residual[r, j], rounded once (nearest, ties to even)
 *             to the element type and STORED;
 *   y[r, j] = h[r, j] * rsqrt(mean_i(h[r, i]^2) + eps) * w[j]
 * The row statistics use the stored h, so y equals rn_rms_norm applied to
 * h bit for bit (one pass instead of an add kernel, a store and a reload).
 *   x, residual  input views of one shape and dtype.
 *   weight       device pointer to dim elements, or NULL (all ones).
 *   y            output view like x; may be x itself (then not also h).
 *   h            output view like x for the stored sum; may be x or the
 *                residual exactly (an in-place residual stream).
 * Every row of residual and h must start at the same 16-byte phase as the
 * matching row of x (true for equal shapes and strides); otherwise
 * RN_ERR_ALIGN. Any other overlap is RN_ERR_OVERLAP. Other errors as
 * rn_rms_norm; nothing is enqueued on error.
 */
RN_API int rn_add_rms_norm(const rn_view *x, const rn_view *residual,
                           const void *weight, float eps, const rn_view *y,
                           const rn_view *h, void *stream);

/*
 * Gated RMSNorm: the output RMS normalization chained into the SwiGLU-style
 * gate ("norm_fusion.rs", module doc comment), in one pass:
 *   y[r, j] = ((x[r, j] * rsqrt(mean_i(x[r, i]^2) + eps)) * w[j]) * silu(z[r, j])
 *   silu(t) = t / (1 + exp(-t)), in binary32, rounded once to the output.
 *   x, z    input views of one shape and dtype; every row of z starts at the
 *           same 16-byte phase as the matching row of x (else RN_ERR_ALIGN).
 *   weight  device pointer to dim elements, or NULL (all ones).
 *   y       output view like x; may be x itself, must not overlap z.
 * Other arguments and errors as rn_rms_norm.
 */
RN_API int rn_gated_rms_norm(const rn_view *x, const rn_view *z,
                             const void *weight, float eps, const rn_view *y,
                             void *stream);

/*
 * RoPE schedule for rn_dual_head_rms_norm_rope ("Emily.Fast", rope/3 and
 * rope_with_freqs/4). Head rows are token-major: row r of q is token
 * r / heads_q (likewise k), at position offset + token. For plane i <
 * dims / 2 the rotation angle is theta_i(pos); the planes are (i, i + dims/2)
 * (split-half) or (2i, 2i + 1) (traditional, interleaved). Columns from dims
 * on pass through unrotated.
 */
typedef struct rn_rope {
    const float *table;   /* device, [n_pos][dims] binary32: cos theta_i(pos) */
                          /* at [pos][i], sin theta_i(pos) at [pos][dims/2+i] */
                          /* (build it with rn_rope_table); caller-owned       */
    int64_t n_pos;        /* rows of the table (positions 0 .. n_pos - 1)      */
    int64_t offset;       /* position of token 0 (0 for a prompt, the cache    */
                          /* length in decode); offset + tokens <= n_pos       */
    int32_t dims;         /* rotated columns: even, <= both head dims          */
    int32_t traditional;  /* 1: planes (2i, 2i + 1); 0: (i, i + dims / 2)     */
    int32_t heads_q;      /* q rows per token                                  */
    int32_t heads_k;      /* k rows per token                                  */
} rn_rope;

/*
 * Fill a HOST buffer `table` ([n_pos][dims] binary32) with the cos / sin of
 * theta_i(pos) = pos * scale * f_i for every position and plane, where
 * f_i = base^(-2i / dims), or inv_freq[i] when inv_freq (host, dims / 2
 * binary32 values) is not NULL (rope_with_freqs/4: Llama-3, LongRoPE, linear
 * or dynamic schedules precomputed by the caller). Angles are formed and
 * evaluated in double and rounded once, so large positions keep full
 * binary32 accuracy. Copy the table to the device once per model.
 * Returns RN_OK, RN_ERR_SHAPE (odd dims, n_pos < 0), RN_ERR_NULL, RN_ERR_EPS
 * (base <= 0 or non-finite base / scale).
 */
RN_API int rn_rope_table(int32_t dims, float base, float scale,
                         const float *inv_freq, int64_t n_pos, float *table);

/*
 * Dual q/k head RMSNorm followed by RoPE, in ONE launch (the dual head norm
 * of "norm_fusion.rs" with the rotary embedding that follows it in these
 * models):
 *   o = rms_norm(q, wq, eps) (binary32, not rounded), yq = rope(o); the same
 *   for k with wk; y_a = o_a cos - o_b sin, y_b = o_b cos + o_a sin per plane.
 * Arguments as rn_dual_head_rms_norm, plus the schedule `rope`. q and k must
 * hold the same number of tokens. Errors: RN_ERR_NULL (rope or its table),
 * RN_ERR_SHAPE (heads, tokens, dims or positions), RN_ERR_ALIGN (table),
 * RN_ERR_OVERLAP (an output over the table); others as the dual head norm.
 */
RN_API int rn_dual_head_rms_norm_rope(const rn_view *q, const rn_view *k,
                                      const void *wq, const void *wk, float eps,
                                      const rn_rope *rope, const rn_view *yq,
                                      const rn_view *yk, void *stream);

/* Static text for an rn_status value ("unknown status" otherwise). */
RN_API const char *rn_status_string(int status);

/* Detail of the most recent failed call on the calling thread (which
 * argument, which CUDA error). Valid until the thread's next call. */
RN_API const char *rn_last_error(void);

/* RN_ABI_VERSION of the loaded library. */
RN_API int rn_abi_version(void);

/* ---------------------------------------------------------------------------
 * Launch introspection and testing controls.
 */

typedef struct rn_launch_info {
    int32_t family;         /* 0: a group of lanes of one warp per row;    */
                            /* 1: one thread block (CTA) per row;          */
                            /* 2: one block per row, streaming (rows wider */
                            /* than the register kernels hold)             */
    int32_t threads_per_row;/* lanes sharing one row                        */
    int32_t chunks_per_thread; /* 16-byte chunks of a row each thread holds */
    int32_t smem_bytes;     /* dynamic shared memory per block: realigned   */
                            /* weight/bias of each thread's chunks (rows   */
                            /* off the 16-byte grid) and prefetch slots    */
    int32_t block_threads;  /* threads per block                            */
    int32_t grid_blocks;    /* blocks launched (persistent: <= SMs x blocks */
                            /* resident per SM)                             */
    int32_t blocks_per_sm;  /* resident blocks per SM for this kernel       */
    int32_t vector_y;       /* 1: y rows share x's 16-byte phase (16-byte   */
                            /* stores); 0: y written element by element     */
    int32_t phase_period;   /* distinct 16-byte phases among x's rows       */
    int32_t exact;          /* layout class: 0 any; 1 every row of x and y, */
                            /* the weight and the bias start 16-byte        */
                            /* aligned and dim fills whole 16-byte chunks;  */
                            /* 2 as 1, and those chunks divide evenly over  */
                            /* the row's threads (no slot is ever empty)    */
    int32_t staged;         /* 1: rows come through rings of shared-memory */
                            /* stages filled by bulk copies, one ring per  */
                            /* warp (family 0) or per block (family 1);    */
                            /* 0: per-thread loads                         */
    int32_t stages;         /* staged: stages per ring                      */
    int32_t stage_bytes;    /* staged: bytes per stage (a tile of rows, or  */
                            /* one row's full 16-byte chunks)              */
} rn_launch_info;

enum { RN_OP_RMS = 0, RN_OP_LN = 1, RN_OP_DUAL = 2, RN_OP_ADD_RMS = 3, RN_OP_GATED_RMS = 4 };

/*
 * The launch the library would make for op (RN_OP_*) on these arguments,
 * without launching. For RN_OP_DUAL, x/y are q/yq and x2/y2 are k/yk (the
 * weight and bias arguments are wq and wk); for RN_OP_ADD_RMS x2/y2 are the
 * residual and h; for RN_OP_GATED_RMS x2 is the gate; otherwise x2/y2 are
 * ignored.
 * Queries the current device (SM count, occupancy), so it needs a GPU.
 */
RN_API int rn_plan(int op, const rn_view *x, const rn_view *y,
                   const rn_view *x2, const rn_view *y2, const void *weight,
                   const void *bias, rn_launch_info *info);

/* Testing control: launch exactly `blocks` blocks (> 0) instead of the
 * automatic persistent grid; 0 restores the automatic choice. Results do not
 * depend on it (rows are statically strided over blocks). A test hook: it
 * applies to every thread of the process (an atomic setting). */
RN_API int rn_set_grid_override(int blocks);

/* Kernel choice: 0 automatic; 1 register-resident kernels loading rows
 * directly; 2 the bulk-copy rings wherever the shape allows (RMSNorm and
 * LayerNorm rows, and the dual head norm with or without in-thread RoPE:
 * rows of up to 2048 bf16 or 1024 binary32 columns in 16-byte aligned
 * layouts through a ring of shared-memory stages per warp, wider rows
 * through a ring per block; all
 * filled with cp.async.bulk), the register kernels elsewhere; 3
 * register-resident kernels with a per-thread prefetch of the rows ahead
 * through shared memory (cp.async), also where the planner would not
 * prefetch. The per-row arithmetic is identical in every kind of
 * kernel, so results do not depend on it. A test hook for tests and
 * measurements: it applies to every thread of the process (an atomic
 * setting). */
RN_API int rn_set_path_override(int path);

/* Testing control for the ring kernels' bounded waits: with on = 1 every
 * ring launch announces 16 bytes more per stage than its copies bring, so no
 * stage ever completes; each warp (or block) gives up its first wait after
 * 1 ms, waits at most 2 ms per stage for its copies (which all land), counts
 * the timeout (rn_device_error_count) and stops, leaving its outputs
 * unwritten. Nothing faults and the CUDA context stays usable. on = 0
 * restores the normal limits (2 s per wait). A test hook: it applies to
 * every thread of the process (an atomic setting). Returns RN_OK, or
 * RN_ERR_SHAPE for another value. */
RN_API int rn_set_ring_wait_test(int on);

/* Number of stage waits in the ring kernels that gave up after their time
 * limit (2 s). Each makes its warp stop early, after waiting for the bulk
 * copies it still has in flight, so a nonzero count means some outputs were
 * not written. Reading synchronizes the current device; reset != 0 clears
 * the counter. Needs a GPU. */
RN_API int rn_device_error_count(unsigned int *count, int reset);

#ifdef __cplusplus
}
#endif

#endif /* ROWNORM_H_ */
