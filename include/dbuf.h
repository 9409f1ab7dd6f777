/*
 * dbuf.h -- C-ABI of the ragged-bucket optimizer step for B200 (sm_100a).
 *
 * What the library does (veScale-FSDP: Flexible and High-Performance FSDP at
 * Scale, MLSys 2026, as the notes.yuuk.io and gist.science pages summarise
 * it):
 *
 *   RaggedShard (paper Sec. 3, page section "1. RaggedShard"): every tensor is
 *     cut into whole blocks of k rows; a block is the unit of block-wise
 *     quantisation and never straddles two devices' shards.
 *   Structure-aware planning (paper Sec. 4, page section "2. Structure-aware
 *     planning algorithm"): the tensors of one communication bucket are sorted
 *     by block size, largest first, and given offsets so that every boundary
 *     between the m equal per-device slices falls on a block edge, with
 *     padding only between tensors.  Runs once, on the host.
 *   DBuffer (paper Sec. 5, page section "3. DBuffer"): the bucket is one flat
 *     buffer per kind (batch-allocated once); tensors are zero-copy views;
 *     group-level operations run once over the whole bucket instead of once
 *     per tensor; streams are ordered explicitly (no record_stream).
 *   8-bit Adam case study (paper Sec. 6.3): block-wise quantised optimizer
 *     states, each device quantising its own blocks with no communication.
 *     A dbuf holds all m slices of a bucket (m devices simulated on one), or,
 *     from dbuf_plan_rank, a single device's slice with only that slice's
 *     optimizer state.
 *
 * Conventions of every entry point:
 *   - Status codes are returned; on failure dbuf_last_error() gives a
 *     thread-local message.  Nothing aborts the process.
 *   - "stream" is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Device work is enqueued on it and is asynchronous; no entry
 *     point synchronises except dbuf_get_device_status and
 *     dbuf_adam8_step_host's callers' own sync.  record_stream is never used.
 *   - Device calls must be made with the device that created the dbuf
 *     current; otherwise DBUF_EINVAL.
 *   - A dbuf is not safe for concurrent calls from several host threads.
 *   - Element offsets are in elements of the array in question; the bucket
 *     holds m*s elements of each kind, s = slice size.
 */
#ifndef DBUF_H
#define DBUF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A tensor of the bucket: row-major rows x cols.  The layout unit (the
 * RaggedShard block) is k whole rows, the last one possibly shorter.  A 1-D
 * tensor of length L is rows=L, cols=1, k=L (one block).
 *
 * Quantisation blocks: block_cols = 0 (or >= cols): each k-row block is one
 * quantisation block.  Otherwise each k-row block is cut into tiles of
 * block_cols columns, the last one narrower, each with its own scales: the
 * 2-D blocks (e.g. 32x32 elements, k = block_cols = 32) that the pages' 8-bit
 * Adam case study allows per parameter (page section "case study: 8-bit Adam
 * and distributed Muon", paper Sec. 6.3).  Tiles require block_cols a power
 * of two in [16, 4096] and cols a multiple of 16.
 *
 * Requires rows, cols, k >= 1, k <= rows, block_cols >= 0. */
typedef struct {
    int64_t rows, cols, k;
    int64_t block_cols;
} dbuf_tensor_desc;

typedef struct dbuf_plan_s dbuf_plan_t; /* host-only layout, owned by the caller */
typedef struct dbuf_s dbuf_t;           /* device bucket, owned by the caller   */

typedef enum {
    DBUF_OK = 0,
    DBUF_EINVAL = 1,      /* bad argument (message says which)                 */
    DBUF_EINFEASIBLE = 2, /* no layout within max_bucket_elems                 */
    DBUF_ENOMEM = 3,      /* host or device allocation failed                  */
    DBUF_ECUDA = 4,       /* a CUDA runtime call failed (message has the name) */
    DBUF_EDEVICE = 5      /* a kernel reported an error in its status word     */
} dbuf_status;

/* Plan the layout of one bucket (host only, no CUDA).
 *   descs[n]          tensors in the caller's order (copied; not retained)
 *   m                 number of equal slices (devices), >= 1
 *   align_elems       every tensor start and s are multiples of it, >= 1;
 *                     dbuf_create needs a multiple of 16 (128-bit accesses)
 *   max_bucket_elems  0 = no cap; otherwise m*s above it -> DBUF_EINFEASIBLE
 * Order: block size k*cols descending, then element count descending, then
 * input position.  s is the smallest multiple of align_elems, at least
 * ceil(sum/m), for which earliest-start placement in that order puts every
 * tensor so that each slice boundary inside a tensor is on a block edge.
 * n = 0 gives an empty plan (s = 0).  *out is NULL on failure. */
dbuf_status dbuf_plan(const dbuf_tensor_desc* descs, int32_t n, int32_t m, int64_t align_elems,
                      int64_t max_bucket_elems, dbuf_plan_t** out);

/* Read a plan.  Any output pointer may be NULL.  offsets[n] (caller-owned)
 * receives each tensor's start in the caller's order.  n_blocks counts the
 * quantisation blocks; blocks are numbered in bucket order (tensors by
 * ascending offset, k-row blocks top to bottom, tiles left to right inside
 * a k-row block), which is the index of their scales. */
dbuf_status dbuf_plan_info(const dbuf_plan_t* plan, int64_t* slice_elems, int64_t* bucket_elems,
                           int64_t* padding_elems, int64_t* n_blocks, int64_t* offsets);

void dbuf_plan_free(dbuf_plan_t* plan); /* NULL is a no-op */

/* Number of tensors and of slices of a plan (the sizes of the caller-owned
 * arrays that dbuf_plan_info, dbuf_plan_shards and dbuf_unpack_views fill).
 * Either output may be NULL.  Host only. */
dbuf_status dbuf_plan_dims(const dbuf_plan_t* plan, int32_t* n_tensors, int32_t* m);

/* RaggedShard placement of a plan (paper Sec. 3; page section
 * "1. RaggedShard": devices hold different numbers of whole blocks): the
 * rows of each tensor that each rank's slice holds.  out[i*m + r] (host
 * array of n*m entries) gets rows [row_begin, row_end) of tensor i in slice
 * r, an empty range when it holds none.  The ranges of a tensor increase with
 * r and cover all its rows, and every boundary between two ranks is a k-row
 * block edge, so each rank quantises its own blocks.  Host only. */
typedef struct {
    int64_t row_begin, row_end;
} dbuf_shard_rows;
dbuf_status dbuf_plan_shards(const dbuf_plan_t* plan, dbuf_shard_rows* out);

/* The bucket one rank holds, as a plan of its own (page section "1.
 * RaggedShard" and paper Sec. 3: each device quantises the whole blocks of
 * its slice, with no exchange): slice `rank` = [rank*s, (rank+1)*s) of the
 * bucket, with m = 1 and slice = bucket = s.  Its tensors are the non-empty
 * row ranges dbuf_plan_shards gives for that rank, in the parent's caller
 * order (tensors with no rows there are left out). Each range keeps cols,
 * k and block_cols and sits at its parent offset minus rank*s; a range
 * shorter than k rows is the tensor's last block.  Its blocks are the parent's
 * blocks inside the slice in the same order, so a dbuf created from it, given
 * slice `rank` of the gradient bucket and stepped with the same
 * hyperparameters and grad_scale, holds slice `rank` of the parent's bucket
 * bit for bit. It stores the fp32 master weights, codes and scales of that
 * one slice only.  *first_block (may be NULL) receives the parent's index of
 * its block 0.  rank in [0, m); *out (freed with dbuf_plan_free) is NULL on
 * failure.  DBUF_EINVAL for a rank out of range, or if a slice boundary cuts
 * a block (which no plan from dbuf_plan does).  Host only. */
dbuf_status dbuf_plan_rank(const dbuf_plan_t* plan, int32_t rank, dbuf_plan_t** out, int64_t* first_block);

/* Bytes of device memory dbuf_create needs for this plan (one allocation:
 * fp32 master, bf16 param, bf16 grad, int8 m codes, uint8 sqrt(v) codes,
 * per-block scales, work tables, status word), 256-byte aligned parts.
 * 0 if plan is NULL. */
size_t dbuf_required_bytes(const dbuf_plan_t* plan);

/* Create the device bucket of a plan (the plan is copied; it may be freed
 * afterwards).  device_base = NULL: one cudaMalloc of dbuf_required_bytes,
 * freed by dbuf_destroy.  Otherwise the caller's device memory, at least
 * dbuf_required_bytes long (base_bytes says how long) and 256-byte aligned;
 * it stays the caller's.  The whole region is zeroed on `stream` and the
 * work tables are copied in, both asynchronously: the bucket is ready for
 * work ordered after them on that stream.  DBUF_EINVAL if the plan's
 * alignment is not a multiple of 16. */
dbuf_status dbuf_create(const dbuf_plan_t* plan, void* device_base, size_t base_bytes, void* stream,
                        dbuf_t** out);

/* Copy-in gather, the per-parameter copy of row-wise FSDP that the
 * zero-copy bucket removes (page section "Importance of zero-copy
 * communication"): for every tensor i,
 *   grad[offset_i + j] = bf16(float(grads_bf16[i][j]) * scale), j < rows*cols.
 * grads_bf16[n] are device pointers in the caller's order (host array,
 * read during the call only); the device memory they point to must stay
 * valid until the copy completes on `stream`.  Padding is not touched. */
dbuf_status dbuf_pack_grads(dbuf_t* db, const void* const* grads_bf16, float scale, void* stream);

/* Gradient accumulation across micro-batches, the DBuffer group "add"
 * (paper Sec. 5; gist.science "Technische samenvatting" 2C: identical
 * operations such as add, scale and zero are fused across the tensors of a
 * bucket): for every tensor i, one launch for the whole bucket,
 *   grad[offset_i + j] = bf16(float(grad[offset_i + j]) + float(grads_bf16[i][j]) * scale).
 * Arguments and lifetimes as in dbuf_pack_grads.  Padding is not touched. */
dbuf_status dbuf_accumulate_grads(dbuf_t* db, const void* const* grads_bf16, float scale, void* stream);

typedef struct {
    float lr, beta1, beta2, eps, weight_decay;
    int64_t step; /* 1-based step number t used in the bias corrections */
} dbuf_adam_hparams;

/* One block-wise 8-bit Adam step over the whole bucket, zero-copy: reads the
 * bf16 gradient bucket in place, one grouped kernel launch.  Per element
 * (fp32, each operation rounded separately, in this order):
 *   g = grad * grad_scale;  m_old = qm * scale_m / 127;  s = qv * scale_v / 255;
 *   m = b1*m_old + (1-b1)*g;  v = b2*s*s + (1-b2)*g*g;  r = sqrt(v);
 *   p = p*(1 - lr*wd) - step_hat * m / (r + eps_hat);
 *   param_bf16 = round-to-nearest-even(p)
 * with the bias corrections folded into step_hat = lr*sqrt(1-b2^t)/(1-b1^t)
 * and eps_hat = eps*sqrt(1-b2^t) (the same Adam step in exact arithmetic);
 * per block: scale_m = max|m|, scale_v = max r, qm = rint(m*127/scale_m)
 * clamped to [-127,127], qv = rint(r*255/scale_v) clamped to [0,255] (codes
 * 0 where the scale is 0).  Per-step scalars are formed in double, rounded to
 * float once.  The bf16 param bucket is set to 0 on every padding element.
 * grad_scale is typically 1/m (the reduce-scatter average). */
dbuf_status dbuf_adam8_step(dbuf_t* db, const dbuf_adam_hparams* hp, float grad_scale, void* stream);

/* Global L2 norm of the gradient bucket as the step would scale it:
 * sqrt(sum over the bucket of (float(grad) * grad_scale)^2), each scaled
 * value rounded to float as in the step, squares summed in double in a
 * fixed order (deterministic on a given device; padding holds zeros).
 * Writes the norm (double) to device memory norm_dev on `stream`.  Uses the
 * bucket's own scratch memory; calls on one bucket must not overlap. */
dbuf_status dbuf_grad_norm(dbuf_t* db, float grad_scale, double* norm_dev, void* stream);

/* The gradient norm of dbuf_grad_norm for callers that cannot allocate
 * device memory: code running where cudaMalloc is not allowed or not wanted
 * (inside a custom allocator or memory-pool callback, a runtime that owns
 * every byte of device memory, a latency-critical loop that must not touch
 * the allocator).  It needs no dbuf: grad_bf16 (device, 16-byte aligned) and
 * n_elems are the input, norm_dev (device, one double) the output:
 *   sqrt(sum over i < n_elems of (float(grad_bf16[i]) * grad_scale)^2).
 * No counterpart in the paper: an addition for such callers.
 * It allocates nothing.  Its scratch (one partial sum per 2^20 elements,
 * 2048 sums) is a file-scope device array of the library that every GPU
 * loading the library holds until the process exits; so n_elems is at most
 * 2^31 and larger sizes return DBUF_EINVAL.  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress): make that
 * first call before any stream capture.  Every call shares the one array,
 * so calls whose work overlaps on the GPU race and give wrong results;
 * serialise them (one stream, or events).  Summation order differs from
 * dbuf_grad_norm's, so results agree to fp64 rounding, not bit for bit. */
dbuf_status dbuf_grad_norm_noalloc(const void* grad_bf16, int64_t n_elems, float grad_scale, double* norm_dev,
                                   void* stream);

/* dbuf_adam8_step with global-norm clipping, without a host round trip:
 * the norm is computed as in dbuf_grad_norm, then the step runs with
 * grad_scale * min(1, max_norm / (norm + 1e-6)) (formed in double on the
 * device, rounded to float once; the convention of
 * torch.nn.utils.clip_grad_norm_).  norm_dev may be NULL; otherwise it
 * receives the norm.  max_norm > 0. */
dbuf_status dbuf_adam8_step_clipped(dbuf_t* db, const dbuf_adam_hparams* hp, float grad_scale, float max_norm,
                                    double* norm_dev, void* stream);

/* The same step with host buffers at both ends (the end-to-end path): copies
 * grads_host (bucket_elems bf16, caller's host memory, pinned for overlap)
 * into the grad bucket, runs the step, and copies the bf16 param bucket back
 * to params_bf16_host (bucket_elems bf16).  On buckets of more than 4M
 * elements this is a pipeline over up to 16 chunks of the bucket:
 *   - a chunk's gradients come in on a copy stream of the dbuf's own;
 *   - the chunk is stepped on `stream` once they have landed;
 *   - its params go out on a second internal stream while later chunks
 *     are still coming in;
 * so the two copy directions and the step overlap.  The results equal
 * dbuf_adam8_step's bit for bit.  Everything is ordered after the work
 * already queued on `stream`, and work queued on `stream` afterwards runs
 * after the last copy out.  The caller synchronises `stream` before reading
 * the output. */
dbuf_status dbuf_adam8_step_host(dbuf_t* db, const dbuf_adam_hparams* hp, float grad_scale,
                                 const void* grads_host, void* params_bf16_host, void* stream);

typedef enum {
    DBUF_MASTER_F32 = 0, /* float  */
    DBUF_PARAM_BF16 = 1, /* bf16   (the all-gather buffer) */
    DBUF_GRAD_BF16 = 2,  /* bf16   (the reduce-scatter buffer) */
    DBUF_M_I8 = 3,       /* int8   codes of m */
    DBUF_V_U8 = 4        /* uint8  codes of sqrt(v) */
} dbuf_which;

typedef struct {
    void* ptr; /* device pointer to the tensor's first element */
    int64_t rows, cols, offset_elems;
} dbuf_view;

/* Zero-copy views: out[n] (caller-owned) gets each tensor's place in the
 * chosen bucket array, in the caller's tensor order.  Pure pointer
 * arithmetic; pointers are borrowed and valid until dbuf_destroy. */
dbuf_status dbuf_unpack_views(const dbuf_t* db, dbuf_which which, dbuf_view* out);

/* Whole bucket array of one kind (e.g. for an in-place all-gather or
 * reduce-scatter of slice r = [r*s, (r+1)*s)).  Borrowed pointer. */
dbuf_status dbuf_bucket(const dbuf_t* db, dbuf_which which, void** ptr, int64_t* elems);

/* Per-block scales, interleaved: scales[2j] = scale of m, scales[2j+1] =
 * scale of sqrt(v), for block j in bucket order.  Borrowed device pointer. */
dbuf_status dbuf_scales(const dbuf_t* db, float** scales, int64_t* n_blocks);

/* Read (and synchronise `stream` for) the device status word that the
 * kernels set instead of trapping: 0 = fine; 1 = a bounded wait on a copy
 * ran out; 2 = a work-table entry was out of range; 3 = a copy-in source
 * pointer was not 2-byte aligned. */
dbuf_status dbuf_get_device_status(dbuf_t* db, int32_t* code, void* stream);

/* One entry of the step kernel's work table (introspection for tests and
 * tools; the kernel's own table holds the same entries).  kind 0: up to 254
 * whole blocks of one tensor, at most 4096 elements counted from the
 * 16-element boundary at or below first_elem; kind 1: one block longer than
 * that, streamed twice; kind 2: a padding range whose bf16 copy is zeroed;
 * kind 3: columns [c0, c0 + n_elems) of the n_blocks rows of one k-row block
 * of a tiled tensor (first_elem = row 0, column c0; block_elems = row
 * stride; reserved = tile width; first_block = scale index of the first
 * tile), streamed twice. */
typedef struct {
    int64_t first_elem, first_block, n_elems;
    int32_t block_elems, kind, n_blocks, reserved;
} dbuf_work_item;

/* Copy the work table that dbuf_create would build for `plan` into out[cap]
 * (host memory; may be NULL when cap = 0) and its length into *n. */
dbuf_status dbuf_work_table(const dbuf_plan_t* plan, dbuf_work_item* out, int64_t cap, int64_t* n);

/* Set the status word back to 0 (asynchronous, on `stream`). */
dbuf_status dbuf_clear_device_status(dbuf_t* db, void* stream);

void dbuf_destroy(dbuf_t* db); /* NULL is a no-op; frees only what it allocated */

/* ---------------------------------------------------------- distributed Muon
 *
 * Muon on the bucket's 2-D tensors (veScale-FSDP pages, case study "8-bit
 * Adam and distributed Muon", paper Sec. 6.3: each 2-D parameter is gathered
 * whole on one rank, Muon's Newton-Schulz preconditioner runs there, and the
 * result returns to the original placement).  In a bucket every tensor is
 * whole, so the gather is the tensor's own view; on several GPUs it is a
 * gather of the tensor's slices to one rank.  The iteration is Muon as its
 * authors published it (the pages name it without coefficients):
 *   t = float(grad) * grad_scale;  mom = momentum * mom + t;
 *   U = t + momentum * mom  (nesterov != 0)  or  U = mom;
 *   X = U / (||U||_F + eps), then ns_steps times on the orientation with
 *       rows <= cols:  A = X X^T;  B = b A + c A A;  X = a X + B X,
 *       (a, b, c) = (3.4445, -4.7750, 2.0315);
 *   master = master * (1 - lr * weight_decay) - lr * sqrt(max(1, rows/cols)) * X;
 *   param = bf16(master).
 * Momentum and its norm are fp32 with fp64 sums (deterministic); the
 * iteration is bf16 with fp32 accumulation, its matrix products cuBLAS GEMMs
 * on the tensor cores. */
typedef struct dbuf_muon_s dbuf_muon_t;

typedef struct {
    float lr, momentum, weight_decay, eps;
    int32_t ns_steps; /* >= 1 */
    int32_t nesterov;
} dbuf_muon_hparams;

/* Muon state for the tensors ids[n] (indices in the plan's caller order;
 * each with rows, cols >= 2) of db: fp32 momentum per tensor (zeroed on
 * `stream`), bf16 workspaces sized for the largest tensor, a cuBLAS handle.
 * One cudaMalloc besides cuBLAS's own; the call waits for the zeroing.  db
 * must outlive the state.  DBUF_EINVAL for a bad or repeated id. */
dbuf_status dbuf_muon_create(dbuf_t* db, const int32_t* ids, int32_t n, void* stream, dbuf_muon_t** out);

/* One Muon step of every listed tensor, in list order, on `stream`: reads
 * the bucket's bf16 grads, updates the momentum, fp32 master weights and
 * bf16 params in place.  The state is bound to db's device; calls on one
 * state must not overlap. */
dbuf_status dbuf_muon_step(dbuf_muon_t* mu, const dbuf_muon_hparams* hp, float grad_scale, void* stream);

/* The orthogonalisation alone: x_bf16 = NS_steps(u / (||u||_F + eps)) for a
 * row-major fp32 rows x cols matrix u (device pointers; rows*cols and
 * min(rows, cols)^2 within the state's workspace, else DBUF_EINVAL). */
dbuf_status dbuf_muon_orthogonalize(dbuf_muon_t* mu, const float* u, int64_t rows, int64_t cols, int32_t ns_steps,
                                    float eps, void* x_bf16, void* stream);

/* Device pointer and length of listed tensor i's momentum (row-major fp32). */
dbuf_status dbuf_muon_momentum(const dbuf_muon_t* mu, int32_t i, float** ptr, int64_t* n);

void dbuf_muon_destroy(dbuf_muon_t* mu); /* NULL is a no-op */

/* ------------------------------------------------ row-wise baseline layout
 *
 * The layout RaggedShard replaces, for measuring what it saves: row-wise even
 * sharding as in FSDP2 / Megatron-FSDP (veScale-FSDP pages, comparison of
 * sharding formats; section on the importance of zero-copy communication:
 * per-parameter copy-in and copy-out with interleaved addresses cost 12-31%
 * of communication time).  Tensor i (rows_i x cols_i, row-major bf16) is
 * cut along dim 0 into m shards of q_i = ceil(rows_i / m) rows, the last
 * ones shorter or empty, each padded to q_i rows in the communication
 * buffer.  Rank r's chunk concatenates its padded shards of tensors 0..n-1;
 * a gathered buffer holds the m chunks in rank order, m * chunk_elems bf16
 * elements.  The k of each descriptor is ignored (it must still be valid). */
typedef struct dbuf_rowwise_s dbuf_rowwise_t;

/* The layout alone, on the host (no CUDA call): chunk_elems, and when not
 * NULL shard_rows[n] (q_i) and offsets[n] (element offset of tensor i's
 * shard in a chunk).  DBUF_EINVAL for n < 1 or m < 1 or an invalid
 * descriptor. */
dbuf_status dbuf_rowwise_layout(const dbuf_tensor_desc* tensors, int32_t n, int32_t m, int64_t* chunk_elems,
                                int64_t* shard_rows, int64_t* offsets);

/* Build the layout and its device copy table (one cudaMalloc, freed by
 * dbuf_rowwise_destroy; the table is copied in on `stream`, and the call
 * waits for that copy).  DBUF_EINVAL for n < 1 or m < 1 or an invalid
 * descriptor. */
dbuf_status dbuf_rowwise_create(const dbuf_tensor_desc* tensors, int32_t n, int32_t m, void* stream,
                                dbuf_rowwise_t** out);

/* chunk_elems: elements per rank chunk.  shard_rows[n] (q_i) and
 * offsets[n] (element offset of tensor i's shard in a chunk) are filled when
 * not NULL (host arrays). */
dbuf_status dbuf_rowwise_info(const dbuf_rowwise_t* rw, int64_t* chunk_elems, int64_t* shard_rows,
                              int64_t* offsets);

/* Interleaved copy-out after an AllGather: for every tensor i and rank r,
 *   params_bf16[i][r*q_i*cols_i + j] = gathered_bf16[r*chunk + offsets_i + j],
 *   j < (min(rows_i, (r+1)*q_i) - r*q_i) * cols_i  (bits copied as they are).
 * gathered_bf16: device, m * chunk_elems elements.  params_bf16[n]: device
 * pointers in tensor order (host array, read during the call).  Any 2-byte
 * alignment; the memory must stay valid until the copy completes on
 * `stream`. */
dbuf_status dbuf_rowwise_copy_out(dbuf_rowwise_t* rw, const void* gathered_bf16, void* const* params_bf16,
                                  void* stream);

/* Interleaved copy-in before a ReduceScatter: the inverse placement of
 * dbuf_rowwise_copy_out with every element scaled,
 *   rs_input_bf16[r*chunk + offsets_i + j] = bf16(float(grads_bf16[i][r*q_i*cols_i + j]) * scale),
 * and the padding rows of every shard set to 0.  rs_input_bf16: device,
 * m * chunk_elems elements.  Arguments and lifetimes as above. */
dbuf_status dbuf_rowwise_copy_in(dbuf_rowwise_t* rw, const void* const* grads_bf16, float scale,
                                 void* rs_input_bf16, void* stream);

/* Status word of the copy kernels, read after the work queued on `stream`
 * (waits for it): 0 = fine, 2 = a malformed copy-table entry was skipped. */
dbuf_status dbuf_rowwise_status(dbuf_rowwise_t* rw, int32_t* code, void* stream);

void dbuf_rowwise_destroy(dbuf_rowwise_t* rw); /* NULL is a no-op */

/* Message of the last failure on this host thread ("" if none). */
const char* dbuf_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DBUF_H */
