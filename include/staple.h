/*
 * staple.h -- C ABI of the STAPLE embedding-augmented SwiGLU FFN layer on
 * NVIDIA B200 (sm_100a).
 *
 * The layer (paper: "STAPLE: Static Sparse Upcycling of Pretrained
 * Checkpoints via Embedding Modules", arXiv 2610.12599; abstract, and the
 * ai4snews summary's Interpretation section) keeps the pretrained SwiGLU FFN
 * and adds a token-indexed row of a vocab x d_ff table E to the output of the
 * up-projection:
 *
 *     g = W_gate x,  u = W_up x,  h = u + E[id],  z = SiLU(g) * h,  y = W_down z
 *
 * E starts at zero, which gives back the dense FFN exactly.  The tables live
 * in host DRAM, the ~5% most frequent rows are cached in HBM, only the rows of
 * the batch's distinct ids reach the GPU, and the table gradient exists for
 * those rows only (abstract; thelatestinai listing, Figure 4 caption and the
 * retrieval-path table; AI Radio episode, paper summary).
 *
 * Conventions for every call below
 *  - Every function returns a staple_status; nothing else crosses the ABI.
 *  - Device work is asynchronous on the caller's stream (a cudaStream_t passed
 *    as staple_stream; NULL = the legacy default stream).  Errors detected on
 *    the device (an id >= V, a kernel wait that ran out of time) are recorded
 *    in the context's device error word; staple_get_error() reads it.
 *  - The caller owns every tensor.  The library allocates device memory only
 *    in staple_context_create and staple_cache_build (and events in
 *    staple_trace_enable); the per-step calls allocate nothing and take
 *    scratch from a caller workspace sized by staple_workspace_bytes().
 *  - Pointers are device pointers unless the argument says "host".
 *    Matrices are row-major and dense (leading dimension = row length).
 *    bf16 tensors are passed as raw 16-bit storage.
 *  - Data-dependent counts (U distinct ids, the miss count) are written to
 *    device int32 words, so the host never waits inside a step; outputs whose
 *    length depends on them are sized for the capacity T.
 */
#ifndef STAPLE_H
#define STAPLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define STAPLE_ABI_VERSION 1

typedef struct CUstream_st* staple_stream; /* same handle as cudaStream_t */

typedef enum staple_status {
  STAPLE_OK = 0,
  STAPLE_EINVAL = -1,       /* bad argument: null pointer, size, alignment, flags */
  STAPLE_EIDRANGE = -2,     /* (device-detected) a token id was outside [0, V) */
  STAPLE_ECUDA = -3,        /* a CUDA runtime call failed */
  STAPLE_ENOMEM = -4,       /* device or pinned-host allocation failed.  For tests,
                               STAPLE_FAIL_ALLOC=<site> in the environment fails
                               that allocation ("context_err", "cache_rows",
                               "cache_hash", "cache_hot", or "all") */
  STAPLE_ETIMEOUT = -5,     /* (device-detected) a bounded kernel wait ran out */
  STAPLE_EUNSUPPORTED = -6, /* valid request this build does not implement */
  STAPLE_ENODEV = -7        /* no usable sm_100 device */
} staple_status;

typedef enum staple_dtype {
  STAPLE_BF16 = 0, /* bf16 storage, fp32 accumulation, tcgen05 tensor cores */
  STAPLE_F32 = 1   /* fp32 storage and arithmetic (CUDA cores) */
} staple_dtype;

typedef struct staple_context staple_context;
typedef struct staple_table staple_table;
typedef struct staple_cache staple_cache;

/* ---------------------------------------------------------------- context */

/* ABI version compiled into the library (STAPLE_ABI_VERSION). */
int staple_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* staple_status_string(staple_status s);

/* Create a context on `device` (makes it current for the calling thread).
 * Allocates the 4-byte device error word.  EINVAL if out == NULL, ENODEV if
 * the device is not compute capability 10.x. */
staple_status staple_context_create(int device, staple_context** out);

/* Free the context.  NULL is accepted. */
staple_status staple_context_destroy(staple_context* ctx);

/* Synchronize `stream`, copy the device error word to *device_error (a
 * staple_status value: STAPLE_OK when no kernel reported an error) and clear
 * it.  The only call that waits for the device. */
staple_status staple_get_error(staple_context* ctx, staple_stream stream, int32_t* device_error);

/* Bound of every wait inside the library's kernels launched for this context
 * from now on (an mbarrier wait for a copy or an MMA, a spin on a flag another
 * block raises), in nanoseconds of the GPU's global timer; default 4 s.  A
 * kernel whose wait runs out records STAPLE_ETIMEOUT in the device error word,
 * stops its remaining work, lets the copies and MMAs it already issued finish,
 * frees its tensor memory and returns, so the context stays usable; its
 * outputs are then undefined.  After STAPLE_ETIMEOUT from a decode-sized call
 * (see staple_ffn_fwd) zero the workspace's counter head again
 * (staple_workspace_bytes) before the next such call.  This is the library's
 * failure detection: no kernel waits without a bound.  EINVAL unless
 * 1 <= limit_ns <= 60 s.  Host-only; takes effect for later launches (a
 * captured CUDA graph keeps the limit it was captured with). */
staple_status staple_set_wait_limit(staple_context* ctx, int64_t limit_ns);

/* SMs that the tiled (persistent) GEMM kernels of this context leave free
 * from now on, for kernels running beside them on other streams.  Each GEMM
 * block keeps an SM's shared memory to itself, so a kernel queued on another
 * stream (the next batch's dedup, which holds one SM's shared memory for a
 * whole batch) otherwise takes an SM a GEMM block was due to start on, and
 * that block, with its fixed share of the tiles, finishes late.  Default 0;
 * EINVAL unless 0 <= sms <= a quarter of the SMs.  Host-only. */
staple_status staple_set_sm_reserve(staple_context* ctx, int32_t sms);

/* Per-kernel timing.  With tracing enabled, every kernel the library launches
 * for this context is bracketed by two CUDA events on its launch stream (a
 * record costs well under a microsecond of device time).  staple_trace_read
 * waits for the recorded events, writes up to `capacity` records in launch
 * order into out[], stores their number in *count, and forgets them (records
 * beyond capacity are dropped).  Enabling allocates 2 * 65536 events once. */
typedef struct staple_trace_record {
  char kernel[40]; /* kernel name, e.g. "k5_gateup" */
  float ms;        /* event-to-event device time of the launch */
} staple_trace_record;

staple_status staple_trace_enable(staple_context* ctx, int enable);
staple_status staple_trace_read(staple_context* ctx, staple_trace_record* out, int32_t capacity,
                                int32_t* count);

/* ------------------------------------------------------------------ tables */

#define STAPLE_TABLE_DEVICE 1u        /* `base` is device memory (the whole table in HBM) */
#define STAPLE_TABLE_HOST_PINNED 2u   /* `base` is pinned, mapped host memory (cudaHostAlloc) */
#define STAPLE_TABLE_HOST_REGISTER 4u /* `base` is pageable host memory: page-lock and map it
                                         (cudaHostRegister) until staple_table_unregister */

/* Describe a table of V rows.  Each row holds `groups` adjacent layers'
 * d_ff-wide rows back to back (token-major grouping of adjacent tables:
 * thelatestinai listing, retrieval-path table, Decode row), so the element
 * (v, layer-in-group l, f) sits at base[(v * groups + l) * F + f].
 * `bytes` must be >= V * groups * F * sizeof(dtype).  Exactly one location
 * flag.  The caller keeps ownership of `base`.  EINVAL on a bad argument,
 * ECUDA if registration fails. */
staple_status staple_table_register(staple_context* ctx, void* base, size_t bytes, int64_t V,
                                    int32_t F, int32_t groups, staple_dtype dtype, uint32_t flags,
                                    staple_table** out);

/* Undo staple_table_register (unregisters host memory it registered). */
staple_status staple_table_unregister(staple_table* table);

/* ------------------------------------------------------------------- cache */

/* Frequency-aware hot-row cache (abstract: about 5% of the embeddings cached
 * on the GPU; AI Radio episode: 5-6% of the vocabulary, ~80% hit rate).
 * Chooses the K = ceil(frac * V) rows with the largest freq[v] (ties: smaller
 * id first; slot k = rank k), allocates K * groups * F elements of HBM, copies
 * those rows from the table, and builds an open-addressing id -> slot hash
 * (capacity: the next power of two >= 2K).  `freq` is a host array of V
 * counts.  frac in [0, 1]; frac = 0 gives an empty cache (every lookup
 * misses).  Synchronizes `stream` before returning. */
staple_status staple_cache_build(staple_context* ctx, const staple_table* table,
                                 const int64_t* freq, double frac, staple_stream stream,
                                 staple_cache** out);

/* Number of cached rows and hash capacity. */
staple_status staple_cache_info(const staple_cache* cache, int32_t* K, int32_t* hash_capacity);

/* Copy the cached ids in slot order into the host array hot_ids[K]. */
staple_status staple_cache_hot_ids(const staple_cache* cache, int32_t* hot_ids);

/* Device address of the cache rows ([K][groups * F], table dtype). */
staple_status staple_cache_rows(const staple_cache* cache, const void** rows);

staple_status staple_cache_free(staple_cache* cache);

/* --------------------------------------------------------------- workspace */

/* Bytes of caller-owned device scratch the per-step calls need for T tokens,
 * d_model D, d_ff F (flags reserved, pass 0).  Zero-fill the workspace once
 * (e.g. cudaMemset) before its first use: its first bytes hold the decode
 * kernel's ready flags and the table-gradient reduction's counters, which
 * every call leaves at zero again (after a call that reported an error,
 * zero-fill it again).  A
 * workspace of this size (or larger), 256-byte aligned, may be reused by
 * every call with the same D and F and the same or smaller T, one call at a
 * time per workspace. */
size_t staple_workspace_bytes(int32_t T, int32_t D, int32_t F, uint32_t flags);

/* ------------------------------------------------------- retrieval (K1..K4) */

/* Deduplicate the batch's token ids once; the inverse map serves every
 * augmented layer (retrieval-path table, Prefill row).
 *   ids[T]          token ids, each in [0, V)
 *   unique[T]       out: the U distinct ids ascending (entries >= U untouched)
 *   inverse[T]      out: unique[inverse[i]] == ids[i]
 *   seg_off[T+1]    out: tokens with id unique[j] are
 *                        sorted_pos[seg_off[j] .. seg_off[j+1]-1]; entries > U untouched
 *   sorted_pos[T]   out: token positions ordered by (id, position)
 *   U_dev           out: U (device int32)
 * T in [0, 32768] and V in [1, 2^31).  An id outside [0, V) sets the error
 * word to STAPLE_EIDRANGE (outputs are then unspecified).  Radix sort by id
 * with warp-ballot run detection, one thread block. */
staple_status staple_dedup(staple_context* ctx, const int32_t* ids, int32_t T, int64_t V,
                           int32_t* unique, int32_t* inverse, int32_t* seg_off,
                           int32_t* sorted_pos, int32_t* U_dev, staple_stream stream);

/* Rows of the batch's distinct ids, reusing a dedup: probe the hot-row cache
 * per distinct id (slot[j] = cache slot or -1), list the misses
 * (miss_list[0..miss_count) = positions j in unique order), copy hit rows from
 * the cache on `stream`, and read miss rows straight from the mapped host
 * table with 16-byte loads on `side` (which then waits for `stream` first and
 * makes `stream` wait for it at the end; pass side = stream to serialise).
 * rows[T][groups * F] receives row j of the batch at rows[j]; all of a row's
 * grouped layers are fetched together.  cache may be NULL (all misses); a
 * DEVICE table needs no cache (all rows read from HBM). */
staple_status staple_gather_unique_rows(staple_context* ctx, const staple_cache* cache,
                                        const staple_table* table, const int32_t* unique,
                                        const int32_t* U_dev, int32_t T, int32_t* slot,
                                        int32_t* miss_list, int32_t* miss_count, void* rows,
                                        staple_stream stream, staple_stream side);

/* staple_gather_unique_rows with the misses taken the bulk way, the pages'
 * prefill path (retrieval-path table, Prefill row): the miss rows are packed
 * on the host into a page-locked staging buffer and copied to the device in
 * bulk by the copy engine (chunk by chunk, each chunk's copy starting as soon
 * as it is packed), then placed into rows by a scatter kernel.  No SM reads
 * host memory.  The calling thread waits for the probe (the host needs the
 * miss list), packs with `threads` host threads (<= 0: all), and returns once
 * the copies and the scatter are queued on `stream`; call it from a helper
 * thread to overlap it with other work.  Not while `stream` is captured.
 *   staging_host  page-locked, >= T * groups * F elements
 *   staging_dev   device, >= T * groups * F elements, 16-byte aligned
 *   list_host     page-locked int32 [1 + 2T] (miss count, miss list, ids)
 *   chunk_rows    rows per bulk copy (>= 1; a value above the miss count
 *                 means one copy of all misses)
 * The buffers may be reused by the next call on the same stream.  The table
 * must be in host memory (HOST_PINNED or HOST_REGISTER).  Same results as
 * staple_gather_unique_rows, bit for bit.  A miss whose id lies outside
 * [0, V) is not read: its row is zero-filled and the call returns
 * STAPLE_EIDRANGE (after queuing the rest). */
staple_status staple_gather_unique_rows_bulk(staple_context* ctx, const staple_cache* cache,
                                             const staple_table* table, const int32_t* unique,
                                             const int32_t* U_dev, int32_t T, int32_t* slot,
                                             int32_t* miss_list, int32_t* miss_count, void* rows,
                                             void* staging_host, void* staging_dev,
                                             int32_t* list_host, int32_t chunk_rows,
                                             int32_t threads, staple_stream stream);

/* Cache write-back after the table rows changed on the host (an optimizer
 * step on the host tables, where the pages keep them together with their
 * AdamW moments: Table 4's caption, ai4snews summary): the cached copies of
 * the listed distinct ids are read again from the table, so the cache keeps
 * serving the current rows.
 *   unique, slot, U_dev   device, from staple_gather_unique_rows (slot[j] =
 *                         the cache slot of unique[j], -1 when not cached)
 * Every grouped layer of a row is copied.  EINVAL if the cache was not built
 * from this table's row shape. */
staple_status staple_cache_refresh(staple_context* ctx, staple_cache* cache,
                                   const staple_table* table, const int32_t* unique,
                                   const int32_t* slot, const int32_t* U_dev,
                                   staple_stream stream);

/* staple_dedup followed by staple_gather_unique_rows (ids -> unique/inverse,
 * hit/miss map, U rows). */
staple_status staple_gather_rows(staple_context* ctx, const staple_cache* cache,
                                 const staple_table* table, const int32_t* ids, int32_t T,
                                 int32_t* unique, int32_t* inverse, int32_t* seg_off,
                                 int32_t* sorted_pos, int32_t* U_dev, int32_t* slot,
                                 int32_t* miss_list, int32_t* miss_count, void* rows,
                                 staple_stream stream, staple_stream side);

/* ------------------------------------------------------------ FFN forward */

typedef enum staple_embed_mode {
  STAPLE_EMBED_NONE = 0,  /* dense FFN: h = u (the E path disabled) */
  STAPLE_EMBED_TABLE = 1, /* h = u + base[index[t] * row_pitch + f], index = token ids,
                             n_rows = V (ids checked against it); a table in HBM */
  STAPLE_EMBED_ROWS = 2   /* h = u + base[index[t] * row_pitch + f], index = inverse map,
                             base = gathered rows; n_rows = capacity */
} staple_embed_mode;

/* staple_embed.flags */
#define STAPLE_EMBED_REPLACE_UP 1u  /* STEM, the variant STAPLE builds on (abstract: STEM replaces
                                       the FFN up-projections with token-indexed embeddings;
                                       ai4snews summary, Interpretation): the row takes the
                                       up-projection's place, h = E[id], and w_up is not read
                                       (may be NULL).  Needs mode TABLE or ROWS. */

typedef struct staple_embed {
  int32_t mode;          /* staple_embed_mode */
  uint32_t flags;        /* 0 (STAPLE: the row is added) or STAPLE_EMBED_REPLACE_UP (STEM) */
  const void* base;      /* device; points at this layer's first element (group offset applied) */
  int64_t row_pitch;     /* elements between consecutive rows (groups * F) */
  const int32_t* index;  /* device [T] */
  int64_t n_rows;        /* rows addressable through index */
} staple_embed;

/* Forward pass of one layer: the pretrained SwiGLU FFN with the token-indexed
 * row E[id] added to the up-projection's output, inside the SiLU gate
 * (abstract: the embeddings join the FFN as a residual pathway; ai4snews
 * summary, Interpretation: the zero-initialised table leaves the seed FFN's
 * output unchanged, and the gate makes the added row context-dependent):
 *     g = W_gate x,  h = W_up x + E[id],  z = SiLU(g) * h,  y = W_down z.
 * With embed->flags = STAPLE_EMBED_REPLACE_UP it computes STEM instead,
 * h = E[id] (w_up not read, may be NULL).
 *   x[T][D], w_gate[F][D], w_up[F][D], w_down[D][F]   inputs (dtype)
 *   z[T][F]     out: SiLU(g) * h, the down projection's input (kept for dW_down)
 *   y[T][D]     out: layer output
 *   g_save, h_save [T][F]  out (training): g and h for the backward pass;
 *               both NULL for inference
 * bf16 needs D and F multiples of 64 and 16-byte aligned pointers;
 * T >= 0.  fp32 needs F a multiple of 8.
 * bf16 with 1 <= T <= 256 (decode sizes; the pages serve at batch 64 on one
 * B200: thelatestinai listing, Table 4) runs one persistent kernel that
 * streams both projections' weights across the SMs and needs the workspace
 * (staple_workspace_bytes, zero-filled once); larger T runs the tiled GEMMs
 * and ignores it.  The down projection's split-k pieces are summed either by
 * a second, small kernel, or, when the layer has enough down tiles (128-row
 * blocks of d_model; e.g. d_model 4096), inside the same launch by clusters
 * of 4 blocks through distributed shared memory.  The persistent kernel's
 * blocks wait on one another, so its whole grid must be resident at once:
 * STAPLE_EUNSUPPORTED when the device cannot hold it (the grid exceeds what
 * the device holds at once, in blocks or in clusters). */
staple_status staple_ffn_fwd(staple_context* ctx, staple_dtype dtype, int32_t T, int32_t D,
                             int32_t F, const void* x, const staple_embed* embed,
                             const void* w_gate, const void* w_up, const void* w_down, void* z,
                             void* y, void* g_save, void* h_save, void* workspace,
                             size_t workspace_bytes, staple_stream stream);

/* ----------------------------------------------------------- FFN backward */

/* Table gradient of one layer: dY -> one gradient row per distinct id of the
 * batch (AI Radio episode, paper summary: during training only the U x d_ff
 * rows of the batch's distinct ids exist on the GPU, as the trainable leaf,
 * so each gets one accumulated gradient row; thelatestinai listing,
 * retrieval-path table: the one dedup's inverse map serves every layer).
 * Computes dz = dY W_down, dh = dz * SiLU(g), dg = dz * h * SiLU'(g) into
 * dgh[T][2F] (dg in columns [0, F), dh in [F, 2F)), then
 *   dE[j][f] = sum of dh[i][f] over the tokens i of segment j (seg_off /
 *              sorted_pos from staple_dedup), accumulated in fp32 in
 *              ascending token position, for j < U (U read from U_dev).
 * dE is fp32 [T][F] (capacity T rows; rows >= U untouched).  With
 * dE == NULL only dgh is produced (the dense run).  With dE, T is at most
 * what one staple_dedup takes (32768; else STAPLE_EUNSUPPORTED). */
staple_status staple_embed_bwd(staple_context* ctx, staple_dtype dtype, int32_t T, int32_t D,
                               int32_t F, const void* dy, const void* g_save, const void* h_save,
                               const void* w_down, const int32_t* sorted_pos,
                               const int32_t* inverse, const int32_t* seg_off,
                               const int32_t* U_dev, void* dgh, float* dE, void* workspace,
                               size_t workspace_bytes, staple_stream stream);

/* The table-gradient half of staple_embed_bwd on its own: dE from a dh that
 * staple_embed_bwd (called with dE == NULL) left in dgh, so that the
 * reduction can run on another stream, next to the rest of the backward pass.
 *   dh          device, T rows of F values (dtype), row pitch ld elements
 *               (the dh half of dgh: dgh + F elements, ld = 2F)
 *   sorted_pos, inverse, seg_off, U_dev   from staple_dedup for the same ids
 *   dE          out, fp32 [>= U][F]; rows >= U untouched
 *   workspace   as for staple_embed_bwd (staple_workspace_bytes(T, D, F)
 *               bytes; of its head only the reduction's counters are used,
 *               and left at zero).  Two calls that overlap on the GPU need
 *               two workspaces.  T at most 32768 (STAPLE_EUNSUPPORTED).
 * Same result, bit for bit, as the reduction inside staple_embed_bwd. */
staple_status staple_embed_grad(staple_context* ctx, staple_dtype dtype, int32_t T, int32_t D,
                                int32_t F, const void* dh, int64_t ld, const int32_t* sorted_pos,
                                const int32_t* inverse, const int32_t* seg_off,
                                const int32_t* U_dev, float* dE, void* workspace,
                                size_t workspace_bytes, staple_stream stream);

/* Return one layer's table gradient to host memory, where the tables and
 * their optimizer live (the pages keep the tables in host DRAM and
 * materialise only the U active rows of a batch: AI Radio episode, paper
 * summary; Table 4's caption for the 12 offloaded tables).
 *   dE          device, fp32 [capacity][F] from staple_embed_bwd
 *   unique      device, int32 [capacity] from staple_dedup
 *   U_dev       device int32: the number of rows to return
 *   host_dE     out, host fp32 [capacity][F]: rows [0, U) written
 *   host_unique out, host int32 [capacity]: ids [0, U) written
 *   host_U      out, host int32: U
 * The three host buffers must be page-locked and mapped into the device's
 * address space (cudaHostAlloc, or cudaHostRegister with the mapped flag);
 * otherwise STAPLE_EINVAL.  U is read on the device, so only U rows cross the
 * host link and the host never waits for U.  F a multiple of 4, dE and
 * host_dE 16-byte aligned.  Asynchronous on `stream`: the host buffers hold
 * the result once the stream's work up to this call has completed. */
staple_status staple_embed_grad_to_host(staple_context* ctx, int32_t F, int32_t capacity,
                                        const float* dE, const int32_t* unique,
                                        const int32_t* U_dev, float* host_dE,
                                        int32_t* host_unique, int32_t* host_U,
                                        staple_stream stream);

/* Rest of the layer backward, consuming dgh from staple_embed_bwd:
 *   dx[T][D]       = dg W_gate + dh W_up                      (dtype)
 *   dw_gate[F][D]  = sum_t dg_t x_t^T       (fp32; NULL: not computed)
 *   dw_up[F][D]    = sum_t dh_t x_t^T       (fp32; NULL: frozen up-projection,
 *                    the warmup recipe of the ai4snews summary, Interpretation)
 *   dw_down[D][F]  = sum_t dY_t z_t^T       (fp32; NULL: not computed)
 * w_up == NULL (with dw_up == NULL) is the STEM layer, which has no
 * up-projection (STAPLE_EMBED_REPLACE_UP): dx = dg W_gate.
 * Gradients are written, not accumulated. */
staple_status staple_ffn_bwd(staple_context* ctx, staple_dtype dtype, int32_t T, int32_t D,
                             int32_t F, const void* dy, const void* x, const void* z,
                             const void* dgh, const void* w_gate, const void* w_up, void* dx,
                             float* dw_gate, float* dw_up, float* dw_down, void* workspace,
                             size_t workspace_bytes, staple_stream stream);

/* ------------------------------------------------ host optimizer (AdamW) */

typedef struct staple_adamw {
  float lr;
  float beta1;
  float beta2;
  float eps;
  float weight_decay;   /* decoupled: w -= lr * weight_decay * w */
  int32_t step;         /* t >= 1: bias corrections 1 - beta^t */
} staple_adamw;

/* AdamW on the U table rows a step touched, on the host, where the tables
 * and their fp32 moments live (the pages offload the tables with their AdamW
 * moments to host DRAM: Table 4's caption; ai4snews summary).  For each
 * j < U, row r = ids[j]:
 *   m[r] = b1 m[r] + (1 - b1) g_j,   v[r] = b2 v[r] + (1 - b2) g_j^2
 *   w[r] -= lr (m[r] / (1 - b1^t) / (sqrt(v[r] / (1 - b2^t)) + eps) + weight_decay w[r])
 * computed in fp32 (Loshchilov & Hutter, decoupled weight decay); a bf16
 * table is rounded to nearest, ties to even.
 *   table      host, rows of F values (dtype), row pitch table_pitch elements
 *              (a grouped table's layer: base + layer * F, pitch groups * F)
 *   ids        host int32 [U], distinct, each in [0, V) (e.g. staple_embed_grad_to_host's
 *              ids); a negative id returns STAPLE_EINVAL before anything changes
 *   grad       host fp32 [U][grad_pitch]: row j is the gradient of row ids[j]
 *   m, v       host fp32 [V][moment_pitch], indexed by row id
 *   threads    host threads to use (<= 0: all hardware threads)
 * Plain host code (no device, no context); returns when done. */
staple_status staple_adamw_rows(void* table, int64_t table_pitch, staple_dtype dtype, int32_t F,
                                const int32_t* ids, int32_t U, const float* grad,
                                int64_t grad_pitch, float* m, float* v, int64_t moment_pitch,
                                const staple_adamw* hp, int32_t threads);

/* ------------------------------------------- allocation-free table gradient */

/* dE from dh without any device allocation, by the caller or the library.
 * The paper has no counterpart: this is the table-gradient reduction of
 * staple_embed_bwd (same kernels, same result) for callers that cannot
 * allocate device memory -- a process whose device memory is all owned by
 * another allocator, code that must not call cudaMalloc because it
 * synchronizes the device, or a plug-in host that only passes its input and
 * output buffers.  Its partial-sum scratch is a 16 MiB array built into the
 * library's device image, which every GPU that loads the library holds until
 * the process exits.
 *   dh          device, T rows of F values (dtype) with row pitch ld elements
 *               (e.g. the dh half of staple_embed_bwd's dgh: base + F, ld = 2F)
 *   sorted_pos, inverse, seg_off   from staple_dedup for the same ids
 *   dE          out, fp32 [>= U][F]; rows >= U untouched
 * Runs on the current device, on `stream`.  The first call in each CUDA
 * context of a device looks up the array's device address
 * (cudaGetSymbolAddress) and keeps it for that context; make that first call
 * before any stream capture (and again after a cudaDeviceReset, which starts
 * a new context).  Every call shares the one array (and a small array of
 * counters beside it, zero at load and left at zero by every call), so calls
 * that overlap on the GPU race; nothing else needs to start at zero.
 * Returns STAPLE_EUNSUPPORTED, before any pointer is looked at, for a size
 * beyond the array or beyond one dedup: T <= 32768 and
 * 2 * ceil(T / 64) * F * 4 bytes <= 16 MiB (T <= 16384 at F = 8192), and
 * STAPLE_EINVAL for other bad arguments.  F must be a multiple of 8. */
staple_status staple_embed_grad_static(staple_dtype dtype, int32_t T, int32_t F, const void* dh,
                                       int64_t ld, const int32_t* sorted_pos,
                                       const int32_t* inverse, const int32_t* seg_off, float* dE,
                                       staple_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* STAPLE_H */
