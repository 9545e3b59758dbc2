/*
 * tl_gemm.h -- C ABI of the B200 (sm_100a) fused tensor-core GEMM library
 *              (libtlgemm.so).
 *
 * The operation, as the TileLang pages define it:
 *
 *   C = epilogue(A . B)
 *
 *   - "Designing High-Performance GPU Kernels with TileLang" (blog retelling),
 *     Step 4 (Tensor-Core GEMM): A is M x K, B is K x N, both row-major (the
 *     shared tiles are block_M x block_K and block_K x block_N); the inputs
 *     are 16-bit floats and the accumulator is float32.
 *   - TileLang GPU kernel design article, paragraph 5 (fused GEMM epilogue):
 *     optionally add a per-column bias and apply GELU to the float32
 *     accumulator before the single write of C, so no intermediate reaches
 *     global memory.  GELU is the exact form x * Phi(x) =
 *     0.5 x (1 + erf(x / sqrt 2)), or on request its tanh form (see
 *     tl_epilogue).
 *
 * The result is rounded once, to nearest even, from float32 to the input
 * dtype (or kept as float32 with tl_gemm_ex's c_float32 option).  The library
 * also holds the tutorial's adjacent kernels: tl_attention_fwd,
 * tl_softmax_rows and tl_vector_add.  Sums are accumulated in float32 on the
 * tensor cores; the order of the sum is fixed by the kernel configuration and
 * the work split (tl_gemm_plan), so two calls with the same plan give
 * bit-identical results (the raster group changes only which tiles run
 * together).
 *
 * All calls are host functions.  None of them allocates memory that outlives
 * the call; a call that must re-lay out an operand, or whose last round of
 * tiles is cut along K (see tl_gemm), takes a stream-ordered temporary from a
 * library-owned CUDA memory pool and returns it on the same stream.
 *
 * Threads: every entry point may be called from several host threads at
 * once, each on its own stream (or the same one).  The library's host state
 * (per device: the memory pool, the kernels' shared-memory limits and their
 * occupancy figures) is guarded by a lock held only while that state is
 * read or first set, never across a launch; tensor maps are encoded per call.
 * The results of concurrent calls equal those of the same calls made one at
 * a time.
 */
#ifndef TL_GEMM_H
#define TL_GEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* major * 1000 + minor.  2.0: tl_gemm_options gained raster_group and
 * force_split, and tl_plan gained tail_units, num_slots and raster_group; both
 * structs grew, so callers built against 1.x must be rebuilt.               */
#define TL_VERSION 2000

#if defined(__GNUC__)
#define TL_API __attribute__((visibility("default")))
#else
#define TL_API
#endif

typedef enum { TL_F16 = 0, TL_BF16 = 1 } tl_dtype;

/* The epilogue applied to the fp32 accumulator before C's only store (the
 * TileLang GPU kernel design article, paragraph 5: bias add, then GELU).
 * GELU is the exact form x Phi(x) = 0.5 x (1 + erf(x / sqrt 2)); GELU_TANH is
 * the tanh approximation 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) of
 * the GELU paper (Hendrycks and Gimpel), PyTorch's approximate="tanh".      */
typedef enum {
    TL_EPI_NONE = 0,            /* C = A.B                                   */
    TL_EPI_BIAS_GELU = 1,       /* C = GELU(A.B + bias[col]), exact erf GELU */
    TL_EPI_BIAS = 2,            /* C = A.B + bias[col]                       */
    TL_EPI_GELU = 3,            /* C = GELU(A.B)                             */
    TL_EPI_BIAS_GELU_TANH = 4,  /* C = GELU_TANH(A.B + bias[col])            */
    TL_EPI_GELU_TANH = 5        /* C = GELU_TANH(A.B)                        */
} tl_epilogue;

typedef enum {
    TL_OK = 0,
    TL_ERR_INVALID_ARG = 1,     /* null pointer, size <= 0, bad enum, missing bias */
    TL_ERR_UNSUPPORTED = 2,     /* size beyond the 32-bit coordinate range, no sm_100 device */
    TL_ERR_MISALIGNED = 3,      /* a pointer not aligned to its 2-byte element */
    TL_ERR_CUDA = 4,            /* a CUDA runtime or driver call failed */
    TL_ERR_DEVICE_TIMEOUT = 5,  /* a bounded wait inside a kernel ran out (see tl_check_device) */
    TL_ERR_SCRATCH_LIMIT = 6    /* tl_gemm_noalloc: the call needs more workspace than TL_NOALLOC_SCRATCH_BYTES */
} tl_status;

/* A cudaStream_t, passed as an opaque pointer; NULL is the legacy default stream. */
typedef void *tl_stream;

/*
 * tl_gemm -- C = epilogue(A . B) on the current CUDA device, asynchronously on
 * `stream`.
 *
 *   A     device pointer, M x K, row-major (leading dimension K), `dtype`
 *   B     device pointer, K x N, row-major (leading dimension N), `dtype`
 *   bias  device pointer to N values of `dtype`; required when epi is
 *         TL_EPI_BIAS_GELU, TL_EPI_BIAS or TL_EPI_BIAS_GELU_TANH, ignored (may
 *         be NULL) otherwise
 *   C     device pointer, M x N, row-major (leading dimension N), `dtype`
 *         (float32 with tl_gemm_ex's c_float32 option); written, never read.
 *         C must not overlap A, B or bias (not checked).
 *   M, N, K   sizes, each in [1, 2^31 - 1]
 *
 * Layout requirements: every pointer must be aligned to 2 bytes.  Nothing
 * else is required.  When a row stride of A or B is not a multiple of 16
 * bytes (K or N not a multiple of 8) or its base is not 16-byte aligned, the
 * call first copies that operand into a zero-padded temporary with rows of a
 * whole number of 128-byte lines (64 elements); when C's rows
 * are not 16-byte aligned the epilogue stores element by element instead of
 * through the tensor-memory-access unit.  Both are slower than the aligned
 * path but give the same numbers.
 *
 * Work split: output tiles are dealt to persistent units (one SM, or a pair
 * of SMs); when the last round of tiles would leave units idle for much of a
 * tile's time, its k-blocks are spread evenly over all units instead, and
 * each partly computed tile is finished by the unit that completes its last
 * part, which adds the parts' float32 partial sums in k order (a fixed order:
 * results stay bit-reproducible).  The partial sums live in the same
 * stream-ordered temporary (tl_gemm_plan's workspace_bytes).  No part of the
 * kernel waits for another unit, so concurrent calls on several streams
 * cannot stall one another.
 *
 * Ownership: the caller owns every buffer and must keep them alive until the
 * work on `stream` completes.  The call does not synchronize.
 *
 * Returns TL_OK once the work is enqueued.  Argument errors are reported
 * before anything is enqueued.  A fault found by the kernel itself (a bounded
 * wait that ran out) is reported later by tl_check_device.
 */
TL_API tl_status tl_gemm(const void *A, const void *B, const void *bias, void *C,
                  int64_t M, int64_t N, int64_t K,
                  tl_dtype dtype, tl_epilogue epi, tl_stream stream);

/*
 * tl_gemm_noalloc -- tl_gemm for callers that must not allocate device memory.
 *
 * The TileLang pages have no counterpart to this call; it exists for users of
 * this library whose code cannot allocate at the moment it runs a GEMM: a
 * plugin whose execute step an inference engine forbids from allocating, a
 * service that reserves all of its device memory up front under a fixed
 * budget, or code that must not call cudaMalloc because it would synchronize
 * the device or fail inside a stream capture.  tl_gemm may take a temporary
 * from a memory pool when an operand has to be copied into a zero-padded
 * layout (K or N not a multiple of 8, or a base that is not 16-byte aligned);
 * tl_gemm_noalloc instead uses a fixed scratch area of
 * TL_NOALLOC_SCRATCH_BYTES that the library declares statically: each GPU the
 * library is used on holds that much device memory until the process exits.
 *
 * What goes into the scratch area is everything tl_gemm would put in its
 * temporary: the zero-padded copies of A and/or B, and, for a shape whose
 * last round of tiles is split along K, the fp32 partial sums of the split
 * tiles and their arrival words.  tl_gemm_plan reports the bytes a call needs
 * as workspace_bytes; every call with workspace_bytes > 0 uses the scratch
 * area, aligned shapes that split included, and a call with workspace_bytes
 * == 0 does not touch it.
 *
 * Arguments, layout rules, results and errors are those of tl_gemm, plus
 * TL_ERR_SCRATCH_LIMIT when the call needs more workspace than
 * TL_NOALLOC_SCRATCH_BYTES.  Nothing is enqueued in that case.
 *
 * The scratch area is shared by all calls on a device and keeps what the last
 * call wrote; each call writes every byte of it that it later reads (partial
 * sums and arrival words are tagged with the launch's own stamp, so nothing a
 * previous call left behind is ever taken for this call's data).  Calls that
 * use the scratch area and whose work can overlap on the GPU (different
 * streams with no ordering between them) race on it and can give wrong
 * results -- padded copies and split partial sums alike: order them on one
 * stream, or with events.
 *
 * The first call on each device does a one-time set-up with that device
 * current: it looks up the device address of the scratch area, raises the
 * kernels' shared-memory limits and records a few bytes of host bookkeeping.
 * Make that first call before any stream capture begins.  After it, a call
 * allocates nothing, on the device or on the host.
 */
#define TL_NOALLOC_SCRATCH_BYTES (64ull << 20)

TL_API tl_status tl_gemm_noalloc(const void *A, const void *B, const void *bias, void *C,
                         int64_t M, int64_t N, int64_t K,
                         tl_dtype dtype, tl_epilogue epi, tl_stream stream);

/*
 * tl_attention_fwd -- attention forward with an online softmax on the tensor
 * cores (the TileLang GPU kernel design article, paragraph 6: query, key and
 * value tiles, running maximum, normaliser and rescaling, the score matrix
 * never written to global memory, checked against PyTorch's scaled
 * dot-product attention):
 *
 *   O[b,h,i,:] = sum_j softmax_j(scale * Q[b,h,i,:] . K[b,h,j,:]) V[b,h,j,:]
 *   lse[b,h,i] = log sum_j exp(scale * Q[b,h,i,:] . K[b,h,j,:])
 *
 * with j over all keys, or over j <= i when `causal` (PyTorch's is_causal).
 *
 *   Q    device pointer, [batch][heads][seq_q][head_dim], `dtype`, contiguous
 *   K, V device pointers, [batch][heads][seq_k][head_dim], `dtype`, contiguous
 *   O    device pointer, [batch][heads][seq_q][head_dim], `dtype`; written
 *   lse  device pointer to batch*heads*seq_q floats, or NULL; written
 *   head_dim        64 or 128
 *   batch * heads   at most 65535 (non-causal) or 2^31 - 1 (causal);
 *   seq_q           at most 65535 * 256 when causal
 *   softmax_scale   > 0, or 0 for 1 / sqrt(head_dim)
 *
 * The products run on 16-bit inputs with fp32 accumulation; the softmax
 * weights are rounded to `dtype` before the product with V (as in
 * FlashAttention); O is rounded once.  Q, K, V, O must be 16-byte aligned
 * (TL_ERR_MISALIGNED otherwise), lse 4-byte aligned.  Asynchronous on
 * `stream`; allocates nothing; bounded waits report through tl_check_device.
 */
TL_API tl_status tl_attention_fwd(const void *Q, const void *K, const void *V, void *O, float *lse,
                          int64_t batch, int64_t heads, int64_t seq_q, int64_t seq_k, int64_t head_dim,
                          tl_dtype dtype, int32_t causal, float softmax_scale, tl_stream stream);

/*
 * tl_softmax_rows -- Y[r, :] = softmax(X[r, :]) for each of `rows` rows of
 * `cols` values (the TileLang GPU kernel design article, paragraph 5: a
 * row-wise softmax with max and sum reductions).  X and Y are device pointers
 * to rows x cols row-major `dtype` values (2-byte aligned; 16-byte aligned with
 * cols a multiple of 8 for the vectorised path); Y may equal X.  Computed in
 * fp32 with the row maximum subtracted, rounded once to `dtype`;
 * probabilities below 2^-126 are returned as 0.  rows, cols >= 1.
 * Asynchronous on `stream`; allocates nothing.  Rows of up to ~110,000 values
 * are read into shared memory by bulk copies whose wait is bounded; a wait
 * that runs out is reported by tl_check_device (bit 6).
 */
TL_API tl_status tl_softmax_rows(const void *X, void *Y, int64_t rows, int64_t cols, tl_dtype dtype,
                         tl_stream stream);

/*
 * tl_vector_add -- C[i] = A[i] + B[i] for i < n, float32 (the same article,
 * paragraph 3, and the blog retelling's Step 3: a bandwidth-bound kernel).
 * Device pointers, 4-byte aligned (16-byte aligned for the vectorised path);
 * n >= 1.  Asynchronous on `stream`; allocates nothing.
 */
TL_API tl_status tl_vector_add(const float *A, const float *B, float *C, int64_t n, tl_stream stream);

/* Options for tl_gemm_ex.  Zero-initialise, then set what you need. */
typedef struct {
    int32_t config;       /* 0: the library's choice for the shape; k > 0: kernel
                             configuration k - 1 (see tl_num_configs)            */
    int32_t inject_fault; /* test hook, 0 in production: 1 makes the copy warp
                             (of both CTAs, with a CTA pair) skip its first
                             stage without issuing the copy, so the MMA warp's
                             bounded wait runs out and the kernel drains what
                             it issued and returns with TL_ERR_DEVICE_TIMEOUT
                             recorded (bit 1 of the detail word; the copy and
                             epilogue warps then wait up to 2 x timeout_ns, so
                             the MMA warp's wait is the one that runs out); 2 makes
                             the host treat the encoding of A's tensor map as
                             failed: the call returns TL_ERR_CUDA and the GEMM
                             kernel is not launched (padding copies the shape
                             needs may already be enqueued; their temporary is
                             released on the stream)                             */
    uint64_t timeout_ns;  /* bound on every wait inside the kernel; 0 = 10 s     */
    int32_t no_split;     /* 1: never cut the tiles of a short last round along K */
    int32_t b_layout;     /* 0: B is K x N row-major (leading dimension N);
                             1: B is given transposed, N x K row-major (leading
                             dimension K) -- the layout of a weight W in A.W^T */
    int32_t c_float32;    /* 0: C has the inputs' type, rounded once from fp32;
                             1: C is float32, the epilogue's fp32 result itself
                             (4-byte aligned; 16-byte aligned rows take vector
                             stores).  C is then stored without the TMA unit.  */
    int32_t raster_group; /* output-tile rows per rasterisation group (tiles are
                             visited column by column inside a group of this
                             many tile rows, so that the tiles running together
                             share operands in L2); 0: the library's choice     */
    int32_t force_split;  /* 1: cut a partial last round along K whenever it is
                             possible (every unit gets at least 4 k-blocks),
                             even where the library's cost rule says it does
                             not pay -- for tests and sweeps; not with no_split */
} tl_gemm_options;

/* tl_gemm with options (NULL options == tl_gemm).  Same arguments and errors;
 * TL_ERR_INVALID_ARG also for a configuration index out of range.             */
TL_API tl_status tl_gemm_ex(const void *A, const void *B, const void *bias, void *C,
                     int64_t M, int64_t N, int64_t K,
                     tl_dtype dtype, tl_epilogue epi, tl_stream stream,
                     const tl_gemm_options *options);

/*
 * tl_check_device -- synchronize `stream`, then read and clear the error word
 * the kernels of this library set on the current device when a bounded wait
 * runs out.  Returns TL_ERR_DEVICE_TIMEOUT if it was set (the kernel stopped
 * early, C is incomplete), TL_ERR_CUDA if the synchronization failed, TL_OK
 * otherwise.  `detail`, if not NULL, receives the raw error word (which waits
 * gave up: bit 0 copy warp, bit 1 MMA warp on data, bit 2 MMA warp on the
 * accumulator, bit 3 epilogue warps, bit 4 final drain, bit 5 a part of a
 * split tile that could not record its arrival, bit 6 the row softmax waiting
 * for a row's copy into shared memory, bit 7 -- in the checked build
 * libtlgemm_checked.so only -- an index invariant of the GEMM kernel failed).
 */
TL_API tl_status tl_check_device(tl_stream stream, uint32_t *detail);

/*
 * tl_gemm_plan -- the host-side decision tl_gemm would take for these
 * arguments, without launching anything (no GPU needed when num_sms > 0).
 * Validation is the same as tl_gemm's and returns the same status.
 */
typedef struct {
    int32_t config;          /* kernel configuration index                     */
    int32_t block_m, block_n, block_k, stages;
    int32_t tiles_m, tiles_n;
    int32_t grid;            /* persistent CTAs launched                       */
    int32_t cluster_ctas;    /* 1, or 2 when pairs of CTAs share each tile     */
    int32_t split;           /* the last, partial round of tiles has its k-blocks
                                spread evenly over all units, so one tile can be
                                shared by several units: the most units sharing
                                one tile (1: nothing is split)                  */
    int32_t full_tiles;      /* tiles computed whole by one unit; the rest form
                                the split last round                           */
    int32_t pad_a, pad_b;    /* 1 when the operand is first copied to a padded temporary */
    int32_t direct_store;    /* 1 when C is stored element by element          */
    int32_t smem_bytes;      /* dynamic shared memory per CTA                  */
    int64_t workspace_bytes; /* stream-ordered temporary the call takes        */
    int32_t tail_units;      /* units the split last round is spread over (0: no
                                split); unit u < tail_units takes the last
                                round's k-blocks [u T / tail_units, (u + 1) T /
                                tail_units), T = (tiles - full_tiles) * k-blocks
                                per tile, tiles in order, each tile's k-blocks in
                                order                                           */
    int32_t num_slots;       /* partial-sum slots in the workspace (slot u + r:
                                unit u's part of last-round tile r)             */
    int32_t raster_group;    /* output-tile rows per rasterisation group       */
    int32_t reserved;        /* 0                                              */
} tl_plan;

TL_API tl_status tl_gemm_plan(const void *A, const void *B, const void *bias, void *C,
                       int64_t M, int64_t N, int64_t K,
                       tl_dtype dtype, tl_epilogue epi, int32_t num_sms,
                       const tl_gemm_options *options, tl_plan *plan);

/* Number of compiled kernel configurations, and the name of configuration i
 * ("bm128_bn256_bk64_s4" ...; NULL when i is out of range).                   */
TL_API int32_t tl_num_configs(void);
TL_API const char *tl_config_name(int32_t i);

/* Human-readable name of a status code (never NULL). */
TL_API const char *tl_status_string(tl_status s);

/* TL_VERSION of the built library. */
TL_API int32_t tl_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TL_GEMM_H */
