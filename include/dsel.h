/*
 * dsel.h -- C ABI of the B200 (sm_100a) batched row-wise TopK library.
 *
 * The operation (what every entry point computes)
 * -----------------------------------------------
 * For each row r of a batch, select the k largest entries (k <= 4096) and return
 * their indices, and optionally their values.  This is the selection kernel of
 * DeepSeek Sparse Attention's Lightning Indexer (bfloat16 scores, tuned for
 * k = 512) and of the sampler (float32 logits, vocabulary ~129,280):
 *   - "Inside DeepSeek V4.1's New Open Inference Toolkit", section "DeepSelect: a
 *     fast, deliberately narrow TopK" (dtypes, k <= 4096, row alignment, options,
 *     NaN policy);
 *   - "DeepSeek releases DeepSelect, a TopK kernel for sparse attention and
 *     sampling" (narracomm): the method paragraph (threshold T, contiguous blocks
 *     of size B in random order, candidate buffer, radix select back to k when the
 *     buffer reaches k + B2), the coverage paragraph (bf16 / f32, int32 / int64
 *     indices), the paragraph on install and switches (stride requirement,
 *     sorted_index, return_value) and the NaN paragraph;
 *   - "DeepSeek 在 GitHub 发布 DeepSelect v1.0.0" (aifluxnews), section "PyTorch 接口与
 *     CUDA 环境要求" (per-row `end`, output stride constraints, NaN trap).
 *
 * Result definition: the k entries of row r that come first in the total order
 * "value descending, then index ascending", where -0.0 equals +0.0 and both
 * infinities are ordinary values.  The result is therefore unique and the library
 * is deterministic (the pages promise stable results: "DeepSeek开源DeepSelect：
 * 比torch.topk快二十倍！", section "DeepSelect 的差异化设计").
 *
 * Layout and ownership (all entry points)
 * ---------------------------------------
 *   x            device pointer, rows x row_stride elements, row-major, rows
 *                contiguous in the last dimension; 16-byte aligned.
 *   row_stride   elements between row starts; a multiple of
 *                dsel_stride_requirement(dtype) (the caller pads).
 *   end          device pointer to int32[rows] or NULL.  Row r's valid range is
 *                [0, end[r]); NULL means every row is row_stride long.  Entries at
 *                or past end[r] are never read as candidates.
 *   indices_out  device pointer, rows x k, contiguous (row stride k), int32 or
 *                int64 per index_dtype; indices are relative to the row start.
 *   values_out   device pointer, rows x k, contiguous, same dtype as x, holding the
 *                selected elements' original bits; NULL iff return_value == 0.
 *   stream       a cudaStream_t passed as void* (NULL = legacy default stream).
 * The caller owns all memory.  Calls are asynchronous on `stream` and never
 * synchronise the host.  Plans that split one row over several thread-block
 * clusters (rows longer than sixteen 128 KB slices) use a per-(device, stream)
 * workspace that the library allocates on first use and grows in stream order
 * (cudaMallocAsync / cudaFreeAsync on `stream`); it never allocates inside a stream
 * capture (such a call returns DSEL_ERR_WORKSPACE: make the first call of a
 * split-row shape on a stream before capturing).  At most 16 streams per device
 * keep a workspace; a further stream evicts the least recently used one with
 * cudaFree, which waits for the device.  All other plans allocate nothing;
 * dsel_topk_noalloc never allocates.
 *
 * Special rows and sentinel values
 *   - end[r] <= k ("short row"): all end[r] entries are returned, in index order
 *     (DSEL_ORDER_VALUE: value descending, equal values by index), and the NaN
 *     check is skipped (narracomm NaN paragraph); slots end[r]..k-1 hold index
 *     DSEL_IDX_PAD and value -inf.
 *   - a NaN in a row with end[r] > k: DSEL_NAN_TRAP (default, the pages'
 *     abort_when_nan_found=True) executes the PTX `trap` instruction, which
 *     aborts the CUDA context; DSEL_NAN_FLAG instead writes DSEL_IDX_NAN in every
 *     index slot of that row and a quiet NaN in every value slot.
 *   - end[r] < 0 or end[r] > row_stride: DSEL_NAN_FLAG writes DSEL_IDX_BAD_END
 *     (values quiet NaN); DSEL_NAN_TRAP clamps end[r] to [0, row_stride].
 *
 * Errors: every argument check runs on the host before any launch; a failed
 * check returns a negative DSEL_ERR_* code and launches nothing.
 */
#ifndef DSEL_H_
#define DSEL_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSEL_API __attribute__((visibility("default")))

/* dtype */
#define DSEL_BF16 0
#define DSEL_F32 1
/* index_dtype */
#define DSEL_I32 0
#define DSEL_I64 1
/* nan_mode */
#define DSEL_NAN_TRAP 0
#define DSEL_NAN_FLAG 1
/* sorted_index: 0 = unspecified order, 1 = ascending index,
 * 2 = value descending (ties by ascending index), float32 only (narracomm: sorting
 * by value is limited to the float32 CUDA path). */
#define DSEL_ORDER_NONE 0
#define DSEL_ORDER_INDEX 1
#define DSEL_ORDER_VALUE 2

/* sentinel indices */
#define DSEL_IDX_PAD (-1)
#define DSEL_IDX_NAN (-2)
#define DSEL_IDX_BAD_END (-3)

/* status codes */
#define DSEL_OK 0
#define DSEL_ERR_DTYPE (-1)        /* dtype not DSEL_BF16 / DSEL_F32 */
#define DSEL_ERR_INDEX_DTYPE (-2)  /* index_dtype not DSEL_I32 / DSEL_I64 */
#define DSEL_ERR_K (-3)            /* k < 1 or k > 4096 */
#define DSEL_ERR_ROWS (-4)         /* rows < 0 */
#define DSEL_ERR_STRIDE (-5)       /* row_stride < 1, > INT32_MAX, or not a multiple of the requirement */
#define DSEL_ERR_ALIGN (-6)        /* x not 16-byte aligned */
#define DSEL_ERR_NULL (-7)         /* x or indices_out is NULL (with rows > 0) */
#define DSEL_ERR_VALUES (-8)       /* return_value set with values_out NULL, or the reverse */
#define DSEL_ERR_NAN_MODE (-9)     /* nan_mode not DSEL_NAN_TRAP / DSEL_NAN_FLAG */
#define DSEL_ERR_ORDER (-10)       /* sorted_index out of range, or value order on bf16 */
#define DSEL_ERR_DEVICE (-11)      /* current device is not sm_100 */
#define DSEL_ERR_WORKSPACE (-12)   /* the split-row workspace could not be allocated (or the stream is capturing) */
#define DSEL_ERR_CUDA (-13)        /* a CUDA runtime call failed (launch error forwarded) */
#define DSEL_ERR_DEVICE_TIMEOUT (-14) /* a kernel gave up a bounded wait (see dsel_device_status) */
#define DSEL_ERR_UNAVAILABLE (-15) /* the entry point is not part of this build */
#define DSEL_ERR_SCRATCH_LIMIT (-16) /* dsel_topk_noalloc: the call needs more than its static scratch */

/* Size of the static device scratch behind dsel_topk_noalloc (512 KiB per device). */
#define DSEL_NOALLOC_SCRATCH_BYTES (512 * 1024)

/* Launch plan chosen for a call (see dsel_plan). */
typedef struct {
  int32_t threads;       /* threads per CTA: 512 (one CTA per SM); with at least as many rows as
                            SMs, 256 for the row-resident kernel (rows of at most 32 KB, four
                            CTAs per SM), 128 for other short rows (several CTAs per SM) or 256
                            for long rows with k <= 1024 (two CTAs per SM); the slice kernel:
                            512 for slices of four 16 KB chunks or more, else 256 */
  int32_t cluster;       /* CTAs per thread-block cluster working on one row */
  int32_t groups;        /* clusters per row (> 1: split-row plan with a merge launch) */
  int32_t block;         /* B: elements per contiguous block visited in random order */
  int32_t b2;            /* B2: the buffer is cut back to k when it holds k + B2 */
  int32_t round;         /* elements the CTA filters between two buffer checks */
  int32_t capacity;      /* candidate-buffer slots per CTA: k + B2 + slack (512 threads: 4096, or
                            2048 for k > 1024; 128 or 256 threads: 1024), at least next_pow2(k)
                            and 4096; the row-resident kernel: next_pow2(k) */
  int32_t stages;        /* blocks kept in flight per CTA (shared-memory ring) */
  int32_t idx_bits;      /* bits of the in-row index used to break ties */
  int32_t smem_bytes;    /* dynamic shared memory per CTA */
  int64_t workspace_bytes; /* split-row workspace (0 unless groups > 1) */
  int32_t kernel;        /* DSEL_KERNEL_STREAM, or DSEL_KERNEL_RESIDENT: at least as many rows as
                            SMs and rows of at most 32 KB, one 256-thread CTA per row holding the
                            whole row in shared memory (block = the 4 KB bulk-copy chunk,
                            round = row_stride, stages = chunks per row, b2 = 0), or
                            DSEL_KERNEL_SLICE: rows cut into `cluster` slices of at most 128 KB,
                            one CTA per slice holding it whole in shared memory, the slices of
                            a row in one cluster (up to 8 to fill idle SMs, up to 16 when the
                            row needs that many slices) (round = slice elements, block =
                            elements per 16 KB bulk-copy chunk, stages = chunks per slice,
                            capacity = candidate-list entries of each CTA, b2 = 0); index
                            order and unspecified order only */
} dsel_plan_t;

#define DSEL_KERNEL_STREAM 0
#define DSEL_KERNEL_RESIDENT 1
#define DSEL_KERNEL_SLICE 2

/*
 * dsel_topk -- batched row-wise TopK (the operation described at the top).
 *   dtype        DSEL_BF16 or DSEL_F32
 *   rows         number of rows (0 is a no-op)
 *   row_stride   see above
 *   end          see above (device, may be NULL)
 *   k            1..4096
 *   sorted_index DSEL_ORDER_NONE / DSEL_ORDER_INDEX / DSEL_ORDER_VALUE
 *   return_value 0 or 1
 *   index_dtype  DSEL_I32 or DSEL_I64
 *   nan_mode     DSEL_NAN_TRAP (default behaviour of the pages) or DSEL_NAN_FLAG
 * Returns DSEL_OK or a DSEL_ERR_* code.
 */
DSEL_API int dsel_topk(const void* x, int dtype, int64_t rows, int64_t row_stride,
                       const int32_t* end, int32_t k, int sorted_index, int return_value,
                       int index_dtype, int nan_mode, void* values_out, void* indices_out,
                       void* stream);

/*
 * dsel_topk_noalloc -- dsel_topk for callers that cannot let a library allocate
 * device memory (for example engines that own the device heap through their own
 * allocator and budget, hosts that forbid side allocations by plug-ins, or
 * latency-critical loops where cudaMalloc / cudaFree, which may synchronise the
 * device, are not acceptable).  The pages have no counterpart to this entry
 * point; it is an interface addition of this library.
 *
 * Arguments, layout, results, sentinels and errors are those of dsel_topk.  The
 * difference is the split-row workspace: instead of a lazily allocated buffer it
 * uses a static device array of DSEL_NOALLOC_SCRATCH_BYTES that every GPU loading
 * the library holds until the process exits.  The call never calls cudaMalloc,
 * cudaFree or any allocating routine.
 *   - It plans a long row's split as dsel_plan does (clusters of up to 8), not
 *     with dsel_topk's split fitted to the device's cluster capacity, so the
 *     scratch a call needs is known on the host: a call whose plan (dsel_plan's
 *     workspace_bytes) needs more than the array returns DSEL_ERR_SCRATCH_LIMIT
 *     and launches nothing (on a 148-SM B200 this happens only for k >= 3640, on
 *     at most nine long rows split over several clusters).
 *   - The first call on a device, whatever its shape, looks up the array's
 *     device address (cudaGetSymbolAddress); the first call of each kernel shape
 *     also sets that kernel's attributes.  Make those first calls before any
 *     stream capture.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents (no slot has to start at zero: each call writes every slot it
 *     reads).  Calls whose work overlaps on the GPU (different streams, not
 *     ordered) race on it: order them.
 */
DSEL_API int dsel_topk_noalloc(const void* x, int dtype, int64_t rows, int64_t row_stride,
                               const int32_t* end, int32_t k, int sorted_index, int return_value,
                               int index_dtype, int nan_mode, void* values_out, void* indices_out,
                               void* stream);

/*
 * dsel_topk_sample -- TopK of float32 sampler logits followed, in the same
 * launch, by a sampling draw among each row's k candidates.
 *
 * The pages name this use ("DeepSeek releases DeepSelect, a TopK kernel for
 * sparse attention and sampling", paragraph "Why rewrite TopK at all?": during
 * sampling TopK picks the candidate tokens out of a large vocabulary) and list
 * temperature and top-p among the generation settings (deepseek-recipe page,
 * section "deepseek-recipe: the protocol layer is real engineering"), but print
 * no formula for the draw.  This library's reading, per row, on the candidates
 * z_1 >= z_2 >= ... (value order, ties by ascending index):
 *   - weights e_i = exp((z_i - z_1) / temperature), and e_i = 1 wherever
 *     z_i == z_1 (so +-inf logits stay meaningful); temperature <= 0 (or NaN)
 *     draws greedily: the first candidate;
 *   - top-p: keep the shortest prefix whose weight sum E_c reaches top_p times
 *     the total; top_p >= 1 (or NaN) keeps every candidate;
 *   - the token is the first kept candidate whose prefix sum exceeds u[r] * E_c;
 *     its probability is e / E_c.
 * Arithmetic is float32 (expf, float32 sums); a different summation order can
 * change the token only where u[r] * E_c or top_p times the total falls within
 * rounding distance of a prefix sum.
 *
 *   x, rows, row_stride, end, k, nan_mode
 *                as for dsel_topk, with dtype DSEL_F32 (x holds float32 logits)
 *   temperature, top_p   as above
 *   u            device float32 [rows]: the caller's uniform draws in [0, 1), one
 *                per row (values outside [0, 1) clamp to the first / last kept
 *                candidate)
 *   values_out, indices_out
 *                both NULL (only the draw is wanted) or both set: the TopK result
 *                as dsel_topk gives it with sorted_index = DSEL_ORDER_VALUE,
 *                return_value = 1 and int64 indices
 *   token_out    device int64 [rows]: the drawn index within the row, or a
 *                negative row code: DSEL_IDX_PAD for an empty row (end = 0),
 *                DSEL_IDX_NAN for a NaN row in DSEL_NAN_FLAG mode, DSEL_IDX_BAD_END
 *                for an invalid end in DSEL_NAN_FLAG mode
 *   prob_out     device float32 [rows] or NULL: the drawn token's probability
 *                (NaN on rows with a negative code)
 * NaN policy: as dsel_topk, except that rows of length <= k are checked for NaN
 * too (TopK skips the check there, but a softmax over a NaN has no meaning).
 * Returns DSEL_OK or a DSEL_ERR_* code (DSEL_ERR_NULL when x, u or token_out is
 * NULL, DSEL_ERR_VALUES when exactly one of values_out / indices_out is NULL);
 * asynchronous on `stream`, allocation behaviour as dsel_topk.
 */
DSEL_API int dsel_topk_sample(const void* x, int64_t rows, int64_t row_stride, const int32_t* end, int32_t k,
                              float temperature, float top_p, const float* u, int nan_mode, void* values_out,
                              void* indices_out, int64_t* token_out, float* prob_out, void* stream);

/*
 * Row split over several shards (one per GPU).  A row too long for one GPU is
 * cut into `shards` contiguous pieces of shard_len elements; each piece's TopK
 * (dsel_topk with sorted_index = DSEL_ORDER_INDEX, return_value = 1, int64
 * indices relative to the piece) is exchanged (one all-gather: shard-major
 * [shards][rows][k]), and the row's TopK is the TopK of the shards' candidates:
 * none of the row's k largest can be missing from its own shard's k largest.
 * The pages keep a whole row on one device; this is the library's extension of
 * their multi-CTA split to several GPUs.  Requires shard_len >= k, so every
 * shard contributes k real candidates and no padding competes with them.
 *
 * dsel_shard_stack lays the gathered candidates out as one row per input row:
 *   vals_in     device [shards][rows][k] values (dtype), as gathered
 *   idx_in      device int64 [shards][rows][k] indices relative to each shard
 *   out_stride  elements per output row: >= shards * k, a multiple of
 *               dsel_stride_requirement(dtype)
 *   vals_out    device [rows][out_stride]: candidate j of shard s at column
 *               s * k + j; columns from shards * k on hold -inf
 *   idx_out     device int64 [rows][out_stride]: the candidate's index in the
 *               whole row (idx_in + s * shard_len; negative codes pass through)
 * Concatenating in shard order keeps the positions in index order, so
 * dsel_topk on vals_out breaks ties exactly as on the whole row; -inf padding
 * sits after every real candidate and is never preferred to one.
 * Returns DSEL_OK, DSEL_ERR_DTYPE / _K / _ROWS / _STRIDE / _NULL, or
 * DSEL_ERR_CUDA.  Asynchronous on `stream`.
 */
DSEL_API int dsel_shard_stack(const void* vals_in, const int64_t* idx_in, int dtype, int64_t rows, int32_t k,
                              int32_t shards, int64_t shard_len, int64_t out_stride, void* vals_out,
                              int64_t* idx_out, void* stream);

/*
 * dsel_take_index -- out[r][j] = table[r][pos[r][j]] for pos >= 0, pos itself
 * (a sentinel code) otherwise: maps the positions returned by dsel_topk on a
 * dsel_shard_stack row back to indices in the whole row.
 *   table        device int64 [rows][table_stride]
 *   pos          device [rows][k], int32 or int64 (pos_dtype: DSEL_I32 / DSEL_I64):
 *                each entry a negative code or a position < table_stride (what
 *                dsel_topk returns on rows of table_stride elements); the kernel
 *                reads table[r][pos] without a further check
 *   indices_out  device [rows][k], int32 or int64 (index_dtype)
 * Returns DSEL_OK, DSEL_ERR_K / _ROWS / _INDEX_DTYPE / _NULL, or DSEL_ERR_CUDA.
 */
DSEL_API int dsel_take_index(const int64_t* table, int64_t table_stride, const void* pos, int pos_dtype, int64_t rows,
                             int32_t k, int index_dtype, void* indices_out, void* stream);

/* Row-stride requirement in elements for `dtype` (the pages' get_stride_requirement,
 * narracomm paragraph on install and switches): 16 for both dtypes, so every row
 * start is 32-byte (bf16) or 64-byte (f32) aligned.  Returns -1 for a bad dtype. */
DSEL_API int64_t dsel_stride_requirement(int dtype);

/* Human-readable text for a status code (static storage, never NULL). */
DSEL_API const char* dsel_status_string(int status);

/* Host-only planner: the plan dsel_topk would use for these arguments on a device
 * with `num_sms` SMs, `smem_optin` bytes of opt-in shared memory per CTA and
 * clusters of up to `max_cluster` CTAs.  Makes no CUDA call.  Returns DSEL_OK or
 * a DSEL_ERR_* code for invalid arguments. */
DSEL_API int dsel_plan(int dtype, int64_t rows, int64_t row_stride, int32_t k,
                       int32_t num_sms, int32_t smem_optin, int32_t max_cluster,
                       dsel_plan_t* out);

/* dsel_plan for a given output order: the plan dsel_topk would use with this
 * sorted_index (value order, DSEL_ORDER_VALUE, and the sampling call never use the
 * slice kernel; pass DSEL_ORDER_VALUE for the plan of dsel_topk_sample).  Makes no
 * CUDA call.  Returns DSEL_OK or a DSEL_ERR_* code (DSEL_ERR_ORDER for a bad
 * order). */
DSEL_API int dsel_plan_for(int dtype, int64_t rows, int64_t row_stride, int32_t k, int sorted_index,
                           int32_t num_sms, int32_t smem_optin, int32_t max_cluster, dsel_plan_t* out);

/* dsel_plan_for with a given cluster capacity: cluster_fit[c], for c = 0..16 (17
 * entries; index 0 unused), is how many clusters of c streaming CTAs (512 threads,
 * all opt-in shared memory) the device holds at once, as the occupancy calculator
 * reports it; 0 where a size cannot be launched.  A row split over the streaming
 * kernel's clusters then takes the cluster size and group count with the most CTAs
 * whose clusters all fit at once, as dsel_plan_device does with the device's own
 * counts.  Host only, no CUDA call.  Returns DSEL_OK, DSEL_ERR_NULL for a NULL
 * array or out, or a DSEL_ERR_* code for invalid arguments. */
DSEL_API int dsel_plan_fit(int dtype, int64_t rows, int64_t row_stride, int32_t k, int sorted_index,
                           int32_t num_sms, int32_t smem_optin, const int32_t* cluster_fit, dsel_plan_t* out);

/* The plan dsel_topk would use with this sorted_index on the current device (pass
 * DSEL_ORDER_VALUE for the plan of dsel_topk_sample): dsel_plan_for with the
 * device's SM count and opt-in shared memory, the slice kernel's cluster size the
 * device can schedule, and a long row split over the streaming kernel's clusters
 * (any size up to 16) and groups chosen for the most CTAs whose clusters the
 * occupancy calculator says the device holds all at once (one wave).
 * Queries the device; launches nothing.  Returns DSEL_OK, DSEL_ERR_CUDA,
 * DSEL_ERR_NULL for a NULL out, or a DSEL_ERR_* code for invalid arguments. */
DSEL_API int dsel_plan_device(int dtype, int64_t rows, int64_t row_stride, int32_t k, int sorted_index,
                              dsel_plan_t* out);

/* Reads and clears the device-side status word that kernels set when a bounded
 * wait runs out (it should never happen).  Synchronises `stream`.  *status_out
 * receives 0 or DSEL_ERR_DEVICE_TIMEOUT.  Returns DSEL_OK or DSEL_ERR_CUDA. */
DSEL_API int dsel_device_status(int* status_out, void* stream);

/* Per-CTA counters of the last streaming launch, for tuning.  Only builds made
 * with -DDSEL_STATS record them; other builds return DSEL_ERR_UNAVAILABLE.
 * host_out receives n_ctas x 16 uint64 (CTA = blockIdx.x of the streaming kernel):
 * stream cycles, final-phase cycles, compaction cycles, compactions, candidates
 * appended, screened vectors sent to the exact test, rounds, final buffer count,
 * then cycle times (from kernel start, thread 0) of: set-up done, prologue
 * issued, first round filtered, first round barrier, first compaction done,
 * stream done; then thread 0's cycles waiting for blocks, and total cycles.
 * With n_ctas == -1, host_out instead receives the per-round timeline of CTA 0:
 * 16 warps x 12 rounds x 10 int64 cycle times from kernel start (round start,
 * screened, counted, append barrier, written, after compaction, prefixed,
 * seeded, blocks arrived, seed returned; 0 = not reached).  With n_ctas <= -2,
 * later launches record the timeline of CTA -n_ctas - 2 instead of CTA 0
 * (host_out is not used).
 * Synchronises `stream`. */
DSEL_API int dsel_debug_stats(uint64_t* host_out, int64_t n_ctas, void* stream);

/* Library version string. */
DSEL_API const char* dsel_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSEL_H_ */
