/*
 * dlrm_sparse.h -- C ABI of the DLRMv1 sparse/interaction stage on B200.
 *
 * The stage has two steps (luminal compare main...vanilla-pytorch):
 *   1. a multi-table EmbeddingBag in sum mode that pools every table's bag of
 *      row ids into a (B, F, D) f32 tensor (embedding_bag.rs, module doc
 *      comment and multi-table section doc comment);
 *   2. the strict-lower-triangular pairwise dot over [dense, pooled_0 ..
 *      pooled_{F-1}], (F+1)F/2 dots per sample in torch.tril_indices(F+1,
 *      F+1, -1) order (dlrm_interact.rs, module doc comment, pair-table
 *      comment, and the stacked-kernel doc comment that puts the dense vector
 *      first).
 *
 * Conventions shared by every entry point:
 *   - Pointers marked "dev" are device pointers on the current CUDA device;
 *     "host" pointers are read during the call only. The caller owns every
 *     buffer: the library allocates nothing and keeps no state between calls.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default
 *     stream). No call synchronises, none copies host memory to the device
 *     except dlrm_sparse_interact_host, so all others can be captured into a
 *     CUDA graph.
 *   - Outputs must not alias inputs.
 *   - A negative return value is a dlrm_status_t; host-side checks run before
 *     anything is launched, so on such an error nothing has been enqueued.
 *   - Indices and offsets are int32 (the pages' kernels take Int indices and
 *     narrow int64 ones; movement.rs, translate_embedding_bag_forward_only).
 *     Row addresses are computed in 64 bits, so tables of any size work.
 *   - Tables, dense and outputs are f32, row-major, with 4-byte aligned
 *     pointers. When D % 4 == 0 and every float pointer is 16-byte aligned the
 *     kernels use 128-bit loads; otherwise a scalar path gives the same bits.
 *
 * Index layout: `indices` holds F segments of B*L entries, table-major:
 * entry t of table k is indices[k*B*L + t]. `offsets` is (F, B): bag b of table
 * k is [offsets[k*B+b], next) where next is offsets[k*B+b+1], or B*L for the
 * last bag (torch.nn.EmbeddingBag with include_last_offset=False, relative to
 * the table's own segment). Fixed-stride offsets b*L give bags of exactly L.
 * An empty bag pools to +0.0. The pooled sum of every column is taken in f32,
 * from 0.0f, in bag order, one rounding per addition, as the pages' kernels
 * sum (embedding_bag.rs, single- and multi-table kernels): pooled outputs are
 * bit-identical to that sequential sum.
 */
#ifndef DLRM_SPARSE_H
#define DLRM_SPARSE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols of the shared library (everything else is hidden). */
#if defined(__GNUC__)
#define DLRM_API __attribute__((visibility("default")))
#else
#define DLRM_API
#endif

/* Same type as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st* dlrm_stream_t;

/* Largest table count F. The F table pointers travel in the kernel's
 * parameter block, so no device-side pointer array has to be staged. */
#define DLRM_MAX_TABLES 256

typedef enum {
    DLRM_OK = 0,
    DLRM_ERR_NULL = -1,            /* a required pointer is NULL */
    DLRM_ERR_SHAPE = -2,           /* B < 1, L < 0, D < 1, B*L > INT32_MAX, or
                                      the interaction's per-sample features do
                                      not fit in one block's shared memory */
    DLRM_ERR_ALIGN = -3,           /* a float/int32 pointer is not 4-byte aligned */
    DLRM_ERR_TOO_MANY_TABLES = -4, /* F < 1 or F > DLRM_MAX_TABLES */
    DLRM_ERR_INDEX_OOB = -5,       /* (device flag) an index outside [0, rows[k]) */
    DLRM_ERR_OFFSETS = -6,         /* (device flag) a bag with start > end, start < 0
                                      or end > B*L */
    DLRM_ERR_CUDA = -7,            /* a CUDA runtime call or launch failed; see
                                      dlrm_last_cuda_error() */
    DLRM_ERR_TIMEOUT = -8,         /* (device flag) a bounded wait on an asynchronous
                                      copy ran out; the results are not valid */
    DLRM_ERR_ARG = -9,             /* any other invalid argument (e.g. count < 0) */
    DLRM_ERR_SCRATCH = -10         /* the call needs more device staging than the
                                      library's fixed array holds
                                      (dlrm_sparse_interact_host_static) */
} dlrm_status_t;

/* Bits that the checked (_ex) entry points OR into *status_dev. */
#define DLRM_FLAG_INDEX_OOB 1
#define DLRM_FLAG_OFFSETS 2
#define DLRM_FLAG_TIMEOUT 4

/* Gather paths (dlrm_set_gather_path). Earlier builds also offered a TMA
 * tile::gather4 path (2), a persistent pipelined register-load path (3) and a
 * persistent shared-memory ring path; each lost to DLRM_PATH_LDG on every
 * measured workload and was removed. Those values are now rejected. */
#define DLRM_PATH_AUTO 0 /* the path measured fastest on B200: DLRM_PATH_LDG */
#define DLRM_PATH_LDG 1  /* one block per batch of bags (fused: of samples), register
                            (128-bit ld.global.nc) loads; serves every call */

/* Pooling of a bag's rows (torch.nn.EmbeddingBag modes). The pages implement
 * only SUM and name the others as what a later model would need (movement.rs,
 * translate_embedding_bag_forward_only). */
typedef enum {
    DLRM_POOL_SUM = 0,  /* sum in bag order, one rounding per add; with
                           per-sample weights one fused multiply-add per entry */
    DLRM_POOL_MEAN = 1, /* the SUM result divided once by the entry count */
    DLRM_POOL_MAX = 2   /* first entry, then (x > acc ? x : acc) in bag order */
} dlrm_pool_mode_t;     /* an empty bag gives 0 in every mode */

/* Element type of the tables. A bf16 table holds the upper 16 bits of each
 * f32 value; rows are widened to f32 exactly and pooled in f32. */
typedef enum { DLRM_TABLE_F32 = 0, DLRM_TABLE_BF16 = 1 } dlrm_table_dtype_t;

/* General bag description (ragged bags, weights, modes).
 *   indices  : dev int32, F segments of T entries (entry t of table k at
 *              indices[k*T + t]); may be NULL iff T == 0.
 *   offsets  : dev int32, (F, B), or (F, B+1) when include_last_offset != 0.
 *              Bag b of table k is [offsets[k][b], end) with end =
 *              offsets[k][b+1], or T for the last bag when
 *              include_last_offset == 0. Entries outside every bag are never
 *              read.
 *   per_sample_weights : dev f32 (F, T), same layout as indices, or NULL.
 *              Only with DLRM_POOL_SUM (else DLRM_ERR_ARG).
 *   T        : entries per table, 0 <= T <= INT32_MAX.
 *   mode     : dlrm_pool_mode_t. */
typedef struct {
    const int32_t* indices;
    const int32_t* offsets;
    const float* per_sample_weights;
    int64_t T;
    int include_last_offset;
    int mode;
} dlrm_bags_t;

/*
 * embbag_sum_multi -- one launch pools all F tables.
 *   weights : host array[F] of dev pointers; table k is (rows_k, D) f32.
 *             Tables may have different row counts (embedding_bag.rs,
 *             multi-table section doc comment).
 *   indices : dev int32, F*B*L entries (see layout above); may be NULL iff L == 0.
 *   offsets : dev int32, (F, B).
 *   out     : dev f32, (B, F, D); out[(b*F + k)*D + d].
 * Indices are trusted, as in the pages' kernels: an index outside its table
 * reads outside it. A bag whose offsets are invalid (start < 0, start > end or
 * end > B*L) is pooled as empty, so bad offsets never cause an out-of-range
 * read; the _ex variant also reports it.
 */
DLRM_API int embbag_sum_multi(const float* const* weights, const int32_t* indices,
                              const int32_t* offsets, int B, int F, int L, int D, float* out,
                              dlrm_stream_t stream);

/*
 * embbag_sum_multi_ex -- embbag_sum_multi with device-side checks.
 *   rows       : host array[F], row count of every table (required).
 *   status_dev : dev int32 or NULL. It is set to 0 on `stream` before the
 *                launch; the kernel ORs DLRM_FLAG_* into it. An index outside
 *                [0, rows[k]) is skipped (adds nothing); a bag with invalid
 *                offsets is pooled as empty. dlrm_status_from_flags() maps the
 *                value, once the stream has reached it, to a status.
 */
DLRM_API int embbag_sum_multi_ex(const float* const* weights, const int64_t* rows,
                                 const int32_t* indices, const int32_t* offsets, int B, int F,
                                 int L, int D, float* out, int32_t* status_dev,
                                 dlrm_stream_t stream);

/*
 * embbag_pool_multi -- the general multi-table EmbeddingBag in one launch.
 *   weights     : host array[F] of dev pointers; table k is (rows_k, D) of
 *                 table_dtype (dlrm_table_dtype_t).
 *   rows        : host array[F] of row counts, or NULL. If given, indices
 *                 outside [0, rows[k]) are skipped (they add nothing and do not
 *                 count toward a mean) and flagged; if NULL, indices are
 *                 trusted.
 *   bags        : host pointer to the bag description, read during the call.
 *   out         : dev f32 (B, F, D).
 *   status_dev  : dev int32 or NULL; zeroed on `stream`, then DLRM_FLAG_* are
 *                 OR-ed in (bad offsets always, bad indices when rows != NULL).
 * A bag with invalid offsets (start < 0, start > end, end > T) pools as empty.
 * With 16-byte aligned tables and output, f32 rows use 128-bit loads when
 * D % 4 == 0 and bf16 rows when D % 8 == 0; otherwise scalar loads, same bits.
 */
DLRM_API int embbag_pool_multi(const void* const* weights, int table_dtype, const int64_t* rows,
                               const dlrm_bags_t* bags, int B, int F, int D, float* out,
                               int32_t* status_dev, dlrm_stream_t stream);

/*
 * interact_lower_tri -- the pairwise-dot interaction alone.
 *   dense : dev f32 (B, D), feature 0.
 *   emb   : dev f32 (B, F, D), features 1..F.
 *   out   : dev f32 (B, P), P = (F+1)F/2; out[b*P + p] = v_i . v_j with (i, j)
 *           the p-th pair of the strict lower triangle, row-major (i > j).
 * Dots are f32 with any summation order: |out - exact| <= 1e-5 * sum_d |v_i v_j|
 * for D <= 128 (the error of D f32 multiply-adds is at most about D * 2^-24
 * times that sum).
 * Needs (4*ceil((F+1)/4)) * (4*ceil(D/4) + 4) * 4 bytes of shared memory per
 * sample, at most the device's per-block limit (227 KB on B200); else
 * DLRM_ERR_SHAPE.
 */
DLRM_API int interact_lower_tri(const float* dense, const float* emb, int B, int F, int D,
                                float* out, dlrm_stream_t stream);

/*
 * dlrm_sparse_interact -- both steps in one launch. Each block gathers its
 * samples' F bags straight into shared memory next to the dense vector, then
 * computes the dots there; only the pooled vectors (if asked) and the
 * interaction rows are written to HBM.
 *   weights, indices, offsets, B, F, L, D : as for embbag_sum_multi.
 *   dense        : dev f32 (B, D).
 *   pooled_out   : dev f32 (B, F, D), or NULL to skip writing the pooled vectors.
 *   inter_out    : dev f32, (B, P) if concat_dense == 0, else (B, D + P) with
 *                  row b = [dense[b] | dots of b] (the concatenation a DLRMv1
 *                  top MLP consumes).
 * Pooled values are bit-identical to embbag_sum_multi's; dots as for
 * interact_lower_tri; the dense part of a concatenated row is copied exactly.
 * Shared memory as for interact_lower_tri.
 */
DLRM_API int dlrm_sparse_interact(const float* const* weights, const int32_t* indices,
                                  const int32_t* offsets, const float* dense, int B, int F, int L,
                                  int D, float* pooled_out, float* inter_out, int concat_dense,
                                  dlrm_stream_t stream);

/* dlrm_sparse_interact with the device-side checks of embbag_sum_multi_ex. */
DLRM_API int dlrm_sparse_interact_ex(const float* const* weights, const int64_t* rows,
                                     const int32_t* indices, const int32_t* offsets,
                                     const float* dense, int B, int F, int L, int D,
                                     float* pooled_out, float* inter_out, int concat_dense,
                                     int32_t* status_dev, dlrm_stream_t stream);

/*
 * dlrm_sparse_interact_pool -- the fused stage with the general bag
 * description: arguments as for embbag_pool_multi, plus dense, pooled_out
 * (nullable), inter_out and concat_dense as for dlrm_sparse_interact.
 */
DLRM_API int dlrm_sparse_interact_pool(const void* const* weights, int table_dtype,
                                       const int64_t* rows, const dlrm_bags_t* bags,
                                       const float* dense, int B, int F, int D, float* pooled_out,
                                       float* inter_out, int concat_dense, int32_t* status_dev,
                                       dlrm_stream_t stream);

/*
 * dlrm_sparse_interact_host -- the whole stage from host memory, for callers
 * whose per-batch inputs live on the host. Tables stay resident on the device.
 * On `stream`, in order: copy indices, offsets and dense host -> dev staging,
 * launch dlrm_sparse_interact, copy the interaction rows (and the pooled
 * vectors if pooled_host != NULL) dev -> host. Returns once everything is
 * enqueued; host outputs are valid after the stream has reached this point.
 * Host buffers should be page-locked for the copies to be asynchronous. When
 * indices, offsets and dense follow each other with no gap both on the host
 * and in the device staging (indices first), they go over in one copy.
 *   indices_host, offsets_host, dense_host : host, layouts as above.
 *   indices_dev, offsets_dev, dense_dev    : dev staging of the same sizes.
 *   pooled_dev   : dev (B, F, D) or NULL; if given the kernel writes the
 *                  pooled vectors there. Required if pooled_host != NULL.
 *   inter_dev    : dev staging for the interaction rows.
 *   pooled_host  : host (B, F, D) or NULL; inter_host : host rows.
 */
DLRM_API int dlrm_sparse_interact_host(const float* const* weights, const int32_t* indices_host,
                                       const int32_t* offsets_host, const float* dense_host, int B,
                                       int F, int L, int D, int concat_dense, int32_t* indices_dev,
                                       int32_t* offsets_dev, float* dense_dev, float* pooled_dev,
                                       float* inter_dev, float* pooled_host, float* inter_host,
                                       dlrm_stream_t stream);

/*
 * dlrm_sparse_interact_host_static -- dlrm_sparse_interact_host for callers
 * that cannot allocate device memory: the device staging is a fixed array of
 * DLRM_STATIC_SCRATCH_BYTES inside this library, so the caller passes only
 * host buffers and the call makes no cudaMalloc, cudaFree or other
 * allocation. The paper and pages this library follows have no counterpart;
 * it is an interface addition. Who needs it: a plugin or callback run by a
 * host framework that owns the device's memory (a serving runtime, or a
 * PyTorch process whose caching allocator already holds the free memory, so
 * a raw cudaMalloc fails or fragments it); code running while a CUDA graph is
 * being captured elsewhere on the device, where cudaMalloc is not allowed;
 * and latency-critical loops, where cudaMalloc/cudaFree would synchronise the
 * device on every batch.
 *   weights, B, F, L, D, concat_dense : as for dlrm_sparse_interact.
 *   indices_host, offsets_host, dense_host : host inputs, layouts as above.
 *   pooled_host  : host (B, F, D) or NULL (then the pooled vectors are not
 *                  written anywhere).
 *   inter_host   : host interaction rows, (B, P) or (B, D + P).
 * On `stream`: the inputs are copied into the array, the fused kernel runs
 * there, and the interaction rows (and pooled vectors) are copied back. It
 * returns once that is enqueued; host outputs are valid when the stream has
 * reached that point. Page-locked host buffers keep the copies asynchronous.
 * Results are bit-identical to dlrm_sparse_interact_host's.
 * Limit: the staging of one call, [indices | offsets | dense] then the
 * interaction rows then the pooled vectors (these two on 256-byte
 * boundaries), must fit in DLRM_STATIC_SCRATCH_BYTES, else DLRM_ERR_SCRATCH
 * and nothing is enqueued. Every GPU that loads the library keeps the array
 * until the process exits.
 * Sharing: every call on a device uses the same array, and the array keeps
 * what the last call left there (nothing in it has to start at zero: a call
 * writes every byte it reads). Calls whose work overlaps on the GPU (two
 * host threads, or two streams with no ordering between them) race on it and
 * corrupt each other's results: run them on one stream, or order them.
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current), which may load the
 * library's code onto the device. Make that first call before any stream
 * capture on that device.
 */
#define DLRM_STATIC_SCRATCH_BYTES (32u << 20)
DLRM_API int dlrm_sparse_interact_host_static(const float* const* weights,
                                              const int32_t* indices_host,
                                              const int32_t* offsets_host,
                                              const float* dense_host, int B, int F, int L, int D,
                                              int concat_dense, float* pooled_host,
                                              float* inter_host, dlrm_stream_t stream);

/*
 * dlrm_pair_decode -- the kernels' flat-index decoder, exposed so it can be
 * checked exhaustively. For p in [p0, p0 + count): (i, j) of the p-th pair of
 * the strict lower triangle, i = floor((1 + sqrt(1 + 8p)) / 2) and
 * j = p - i(i-1)/2, from an f32 square root followed by an exact integer
 * correction (dlrm_interact.rs, stacked-kernel layout comment). For
 * p < 2^24 this runs the 32-bit decoder that the interaction and fused
 * kernels apply to their pair-tile index (a tile index is below 2145 at
 * DLRM_MAX_TABLES); from 2^24 on, a 64-bit form of the same steps.
 *   i_out, j_out : dev int32 arrays of `count` entries. Needs p0 >= 0,
 *                  count >= 0 and p0 + count <= 2^31 (else DLRM_ERR_ARG).
 */
DLRM_API int dlrm_pair_decode(int64_t p0, int64_t count, int32_t* i_out, int32_t* j_out,
                              dlrm_stream_t stream);

/*
 * dlrm_set_gather_path -- which gather serves later gather and fused calls of
 * this process (all threads): DLRM_PATH_AUTO (default) or DLRM_PATH_LDG.
 * Returns the previous setting, or DLRM_ERR_ARG for any other value.
 */
DLRM_API int dlrm_set_gather_path(int path);

/* The path (DLRM_PATH_LDG) that served the calling thread's last gather or
 * fused launch; 0 before the first one. */
DLRM_API int dlrm_last_gather_path(void);

/* Status of a *status_dev value written by an _ex call (DLRM_OK if 0). */
DLRM_API int dlrm_status_from_flags(int32_t flags);

/* Static, human-readable name of a status code. */
DLRM_API const char* dlrm_status_string(int status);

/* cudaError_t of the last failing CUDA call made by this thread in the library. */
DLRM_API int dlrm_last_cuda_error(void);

/* Number of kernels this library has launched in this process (all threads). */
DLRM_API int64_t dlrm_launch_count(void);

/*
 * dlrm_probe_bounded_wait -- failure-detection check. One thread of one block
 * waits on a shared-memory mbarrier that nothing ever completes, with the same
 * bounded wait the asynchronous kernels use (the MLP layers wait that way on
 * their TMA copies and tensor-core work). After about
 * `limit_cycles` clock cycles (clamped to [1000, 2e8]) the wait gives up, the
 * kernel ORs DLRM_FLAG_TIMEOUT into *status_dev (dev int32, required) and
 * returns normally: the CUDA context stays usable. Asynchronous on `stream`.
 */
DLRM_API int dlrm_probe_bounded_wait(int64_t limit_cycles, int32_t* status_dev,
                                     dlrm_stream_t stream);

/*
 * dlrm_probe_row_gather -- measurement aid: the device's rate of random row
 * reads for rows of `row_bytes` bytes, without the stage's offset and index
 * loads (the roofline that the gather's row reads meet). No counterpart on the
 * pages. `count` rows of `table` are read, row n (0 <= n < count) at row id
 * splitmix64(seed + n) mod rows, each row by row_bytes/16 lanes with one
 * 128-bit load per lane that does not allocate in L1, eight rows in flight per
 * lane. The XOR of every word read is folded into one value per thread, which
 * is written to *sink_dev only if it equals a fixed constant (so the reads
 * cannot be left out; the sink's content is otherwise unspecified). Time the
 * call with events on `stream` to get rows/s.
 *   table    : dev, `rows` rows of `row_bytes` bytes, 16-byte aligned; read only.
 *   rows     : >= 1.
 *   row_bytes: 16, 32, 64, 128, 256 or 512 (DLRM_ERR_SHAPE otherwise).
 *   count    : >= 0 rows to read.
 *   sink_dev : dev uint32, 4-byte aligned, required.
 * Asynchronous on `stream`.
 */
DLRM_API int dlrm_probe_row_gather(const void* table, int64_t rows, int row_bytes,
                                   int64_t count, uint64_t seed, uint32_t* sink_dev,
                                   dlrm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DLRM_SPARSE_H */
