/*
 * liteattn.h -- C ABI of the B200 (sm_100a) LiteAttention library.
 *
 * LiteAttention runs temporally sparse self-attention across the denoising
 * steps of a video diffusion transformer.  A persistent skip mask holds one
 * bit per (batch, head, query tile, key tile).  Each step loads and multiplies
 * only the key/value tiles that are still live.  Inside the online softmax a
 * QK-Skip test kills a tile whose maximum logit falls more than a threshold
 * below the running maximum.  Dead tiles stay dead in later steps.
 * Sources: "LiteAttention: Temporal Sparse Attention for Diffusion
 * Transformers" (skill page), sections "Core Concept" (T denoising steps,
 * QK-Skip, mask propagated forward) and "Architecture Overview" (Skip-Mask
 * bitmask or skip-list, QK-Skip inside the softmax pipeline, per-step error
 * budget, persistent propagation); "LiteAttention: A Temporal Sparse
 * Attention for Diffusion Transformers", abstract (skip decisions are marked
 * early and propagated forward).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Return value: LITE_OK (0) or a negative LITE_ERR_* code.  No exception
 *   crosses the ABI.  Argument checks run synchronously on the host; kernels
 *   run asynchronously on the given stream, and device-side failures (a
 *   bounded wait that ran out) surface through lite_attn_stats().
 * - Tensors q, k, v, o: device pointers to contiguous bf16 arrays of layout
 *   [B][H][N][d] (row-major, head-major), or [B][N][H][d] (token-major, the
 *   layout of a transformer's QKV projection) for plans made with
 *   LITE_LAYOUT_BNHD; 16-byte aligned, owned by the caller.  o has the
 *   layout of q and must not overlap q, k or v.
 * - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *   default stream), a stream of the plan's device.  A plan and its masks
 *   must not be used from two streams at once.
 * - Devices: a plan belongs to the device that was current when it was
 *   created, and its masks to the same device.  Every call on a plan or mask
 *   makes that device current for its duration and restores the caller's
 *   current device before returning, so plans on several devices can be
 *   driven from one thread.  Tensor pointers must be memory of the plan's
 *   device (INVALID_ARG otherwise).
 * - Threshold tau: natural-log domain, tau <= 0, or -inf (never skip).  A
 *   key tile j dies for query tile i when, for every valid query row r,
 *   (max over the tile's valid keys of the logit) - (running max of row r)
 *   < tau, where logits are q.k / sqrt(d).
 * - Mask bits: word j>>5, bit j&31 of a row of W = ceil(Tk/32) uint32
 *   words; 1 = live; bits >= Tk are 0.  Row index (b*H + h)*Tq + i.
 */
#ifndef LITEATTN_H
#define LITEATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct lite_attn_plan *lite_attn_plan_t;
typedef struct lite_attn_mask *lite_attn_mask_t;

enum {
    LITE_OK = 0,
    LITE_ERR_INVALID_ARG = -1,    /* null/misaligned/overlapping pointer, bad shape, step out of range, tau NaN or > 0 */
    LITE_ERR_UNSUPPORTED = -2,    /* (d, Br, Bc) other than (64,64,64) or (128,128,128); N outside [1, 2^20] */
    LITE_ERR_PLAN_MISMATCH = -3,  /* a mask used with a plan that did not create it */
    LITE_ERR_ALLOC = -4,          /* device or host allocation failed */
    LITE_ERR_CUDA = -5,           /* CUDA runtime or launch error, or no sm_100 device */
    LITE_ERR_DEVICE_TIMEOUT = -6, /* a kernel's bounded wait ran out; its outputs are invalid */
    LITE_ERR_DEVICE_CHECK = -7    /* debug builds (LITE_DEBUG_CHECKS): a work item failed its device-side checks */
};

typedef struct {
    int64_t tiles_total;    /* B*H*Tq*Tk */
    int64_t live_in;        /* live tiles of the incoming mask of the step that wrote this mask (= QK tiles) */
    int64_t qk_tiles;       /* tiles whose Q K^T was computed in that step (= live_in) */
    int64_t pv_tiles;       /* tiles whose softmax and P V were computed in that step (= live_out) */
    int64_t newly_dead;     /* tiles killed by the QK-Skip test in that step */
    int64_t live_out;       /* live tiles currently held by this mask */
    double skip_fraction;   /* 1 - live_out / tiles_total */
    double executed_flops;  /* 2*Br*Bc*d*(qk_tiles + pv_tiles) of that step: the algorithmic work.  With
                               Br = 64 the kernel issues 128-row MMAs over a pair of query tiles whenever
                               either tile needs the key tile, so the issued MMA work can exceed this (up to
                               2x where the pair's two live sets differ); with Br = 128 the two are equal. */
    double dense_flops;     /* 4*B*H*N*N*d */
    int64_t cum_qk_tiles;   /* plan-wide totals over all steps since plan creation */
    int64_t cum_pv_tiles;
    int64_t cum_steps;
    int32_t device_status;  /* LITE_OK, LITE_ERR_DEVICE_TIMEOUT or LITE_ERR_DEVICE_CHECK (sticky for the plan) */
    int32_t last_step;      /* step index that produced this mask; -1 after reset or import */
} lite_attn_stats_t;

/* Create a plan for a fixed problem shape and a T-step threshold schedule.
 * Passage: skill page, "Core Concept" (T denoising steps) and "Architecture
 * Overview" (Accumulated-Error Calibration: a per-step error budget, here a
 * caller-given per-step threshold).
 *   out     : receives the plan handle (owned by the caller; free with
 *             lite_attn_plan_destroy).
 *   B, H, N : batch, heads, tokens; d : head dim; Br, Bc : query / key tile.
 *   threshold_schedule : host array of T floats, copied; tau_t for step t.
 * Runs on the current CUDA device, which must be sm_100 (B200).  Allocates a
 * small device status block.  Errors: INVALID_ARG, UNSUPPORTED, ALLOC, CUDA. */
int lite_attn_plan_create(lite_attn_plan_t *out, int B, int H, int N, int d, int Br, int Bc,
                          const float *threshold_schedule, int T);

/* Tensor layouts of a plan (lite_attn_plan_create_ex). */
#define LITE_LAYOUT_BHND 0   /* [B][H][N][d]: the layout of lite_attn_plan_create */
#define LITE_LAYOUT_BNHD 1   /* [B][N][H][d] */

/* lite_attn_plan_create with the tensor geometry chosen explicitly.  Neither
 * option has a counterpart in the pages, which fix no layout and no device
 * count.
 *   layout      : LITE_LAYOUT_BHND or LITE_LAYOUT_BNHD, else INVALID_ARG.  A
 *                 transformer block produces [B][N][H][d] from its QKV
 *                 projection; this layout spares it a transpose before and
 *                 after the call.
 *   heads_total : heads in the tensors, >= H (0 means H, else INVALID_ARG).
 *                 The plan then covers H consecutive heads of tensors with
 *                 heads_total heads: the pointers given to lite_attn_step
 *                 point at the plan's first head (tensor + h0*N*d elements for
 *                 BHND, + h0*d for BNHD) and only those H heads are read or
 *                 written.  Work items are independent across heads, so plans
 *                 over disjoint head ranges (one per GPU, say) compute exactly
 *                 what one plan over all heads computes, with no exchange.
 *                 lite_attn_output_error needs heads_total == H.
 * Masks, lists and statistics do not depend on either option, and neither do
 * the results (bit for bit).  Other arguments, ownership and errors as
 * lite_attn_plan_create. */
int lite_attn_plan_create_ex(lite_attn_plan_t *out, int B, int H, int N, int d, int Br, int Bc,
                             const float *threshold_schedule, int T, int layout, int heads_total);

/* A plan over a batch of B sequences of different lengths (no counterpart in
 * the pages; an integration form for batches of videos of different sizes).
 * The tensors are packed token-major: q, k, v, o are [total][H][d] bf16 with
 * total = sum of seq_lens, sequence b occupying tokens [off_b, off_b +
 * seq_lens[b]), off_b = seq_lens[0] + ... + seq_lens[b-1]; the pointers given
 * to lite_attn_step point at token 0.  Each sequence attends within itself.
 *   seq_lens : host [B] int32, each >= 1 (copied); N = max(seq_lens) sets the
 *              tile geometry (Tq, Tk, W, G of lite_attn_plan_info), and the
 *              tiles a shorter sequence lacks are dead in every mask (reset
 *              leaves them dead; import rejects masks that set them).
 * Results for each sequence are those of a fixed-length plan on that sequence
 * alone (bit for bit).  Other arguments, ownership and errors as
 * lite_attn_plan_create (INVALID_ARG for a null or non-positive length;
 * UNSUPPORTED for N beyond 2^20 or 2^31 tokens in total). */
int lite_attn_plan_create_varlen(lite_attn_plan_t *out, int B, int H, const int32_t *seq_lens, int d, int Br,
                                 int Bc, const float *threshold_schedule, int T);

/* Skip predicates of a plan (lite_attn_plan_predicate). */
#define LITE_PRED_THRESHOLD 0   /* QK-Skip against a per-step threshold tau (the plans above) */
#define LITE_PRED_RECALL 1      /* fixed recall p per step (lite_attn_plan_create_recall) */

/* A plan whose skip predicate keeps a fixed recall of the attention mass
 * instead of testing a fixed threshold.  Passage: "Training-free sparse
 * attention based on cumulative energy filtering", abstract (a fixed recall
 * rate is enough for accuracy; a dynamic threshold reaches it inside the
 * FlashAttention pass, with no separate masking stage).  The page gives no
 * formula; the test computed here:
 *   per query row, l = its kept softmax mass so far and z = an upper bound on
 *   the mass of the key tiles it skipped so far (both relative to its running
 *   max m).  A key tile live in mask_in, with w valid keys and per-row maxima
 *   m_loc, is skipped for the query tile when every valid row has
 *       z + w * exp(m_loc - m) <= ((1 - p) / p) * l,
 *   i.e. when its max-logit gap lies under the row's dynamic threshold
 *   ln(((1 - p) / p * l - z) / w).  A skipped tile gets no softmax and no P V,
 *   its bound joins z, and it is cleared in mask_out (dead in later steps, as
 *   for QK-Skip).  Every valid row therefore keeps at least a fraction p of
 *   the softmax mass of the tiles it was offered; p = 1 skips nothing.  The
 *   bound w * exp(m_loc - m) over-counts a tile's mass, so the recall reached
 *   is usually well above p.
 *   recall_schedule : host array of T floats, copied; p_t in (0, 1] for step t
 *                     (INVALID_ARG otherwise).
 * Other arguments, layouts, ownership and errors as lite_attn_plan_create_ex. */
int lite_attn_plan_create_recall(lite_attn_plan_t *out, int B, int H, int N, int d, int Br, int Bc,
                                 const float *recall_schedule, int T, int layout, int heads_total);

/* The plan's skip predicate: LITE_PRED_THRESHOLD or LITE_PRED_RECALL. */
int lite_attn_plan_predicate(lite_attn_plan_t plan, int *predicate);

/* Options of lite_attn_plan_create_opts.  Zero-initialised options give the
 * plan of lite_attn_plan_create. */
typedef struct {
    int layout;       /* LITE_LAYOUT_BHND (0) or LITE_LAYOUT_BNHD */
    int heads_total;  /* heads in the tensors, >= H; 0 means H (see lite_attn_plan_create_ex) */
    int predicate;    /* LITE_PRED_THRESHOLD (schedule = thresholds tau) or LITE_PRED_RECALL (recall targets p) */
    int pair_stride;  /* which query tiles share a work item; 0 or 1: adjacent tiles (2p, 2p+1) */
} lite_attn_plan_options_t;

/* Plan creation with every option at once.  The pages fix no work
 * decomposition; the pairing is this library's scheduling choice:
 *   pair_stride s : each work item (one CTA) runs two query tiles that share
 *                   every key/value tile load over the union of their live
 *                   lists.  With s > 1 the Tq query tiles of a head go in
 *                   blocks of 2s and tile r of a block pairs with tile r + s (a
 *                   last, shorter block of m tiles pairs r with r + ceil(m/2)).
 *                   For video tokens in (frame, y, x) order, s = the tiles per
 *                   frame (Y*X/Br rounded down) pairs each query tile with the
 *                   one a frame later, whose live key tiles overlap its own
 *                   more than those of its neighbour along the scan line: fewer
 *                   union entries that only one tile of the pair needs, so
 *                   less idle time at high skip rates.  Outputs, masks and
 *                   statistics do not depend on s (bit for bit); only the
 *                   compacted lists (lite_attn_mask_export_lists) and the time
 *                   do.  s > 1 needs Br = 128 (UNSUPPORTED otherwise);
 *                   negative s: INVALID_ARG.
 * Other arguments as lite_attn_plan_create_ex / lite_attn_plan_create_recall;
 * NULL opts: INVALID_ARG. */
int lite_attn_plan_create_opts(lite_attn_plan_t *out, int B, int H, int N, int d, int Br, int Bc,
                               const float *schedule, int T, const lite_attn_plan_options_t *opts);

/* The two query tiles of work item `pair` (0 <= pair < ceil(Tq/2)) of every
 * (batch, head) of the plan; *tile_b = -1 when the item has one tile. */
int lite_attn_plan_pair_tiles(lite_attn_plan_t plan, int pair, int *tile_a, int *tile_b);

/* Free a plan (synchronises the device first).  Masks of the plan must be
 * destroyed before it.  NULL is accepted and ignored. */
int lite_attn_plan_destroy(lite_attn_plan_t plan);

/* Tile counts of a plan: Tq = ceil(N/Br), Tk = ceil(N/Bc), W = ceil(Tk/32) words
 * per mask row, G = B*H*ceil(Tq/2) query-tile pairs (the kernel's work items;
 * which tiles pair up: lite_attn_plan_pair_tiles). */
int lite_attn_plan_info(lite_attn_plan_t plan, int *Tq, int *Tk, int *W, int *G);

/* Create a skip mask of the plan (device memory: bitmask, compacted live
 * lists, counts, work order, stats).  It starts all-live (synchronously).
 * Passage: skill page, "Architecture Overview" (Skip-Mask data structure:
 * bitmask, or a skip-list for high sparsity). */
int lite_attn_mask_create(lite_attn_plan_t plan, lite_attn_mask_t *out);
int lite_attn_mask_destroy(lite_attn_mask_t mask);

/* Set every valid tile live (asynchronous on `stream`).  Calling this before
 * each step gives recompute-every-step mode. */
int lite_attn_mask_reset(lite_attn_mask_t mask, void *stream);

/* Load a bitmask from host memory ([B*H*Tq][W] uint32, bits >= Tk must be 0,
 * else INVALID_ARG) and rebuild the live lists.  The host buffer may be
 * reused when the call returns (the copy is synchronous w.r.t. the host
 * buffer).  Used to resume a denoising run from a checkpointed mask. */
int lite_attn_mask_import(lite_attn_mask_t mask, const uint32_t *host_bits, void *stream);

/* Copy the bitmask to host memory ([B*H*Tq][W] uint32).  Synchronises `stream`. */
int lite_attn_mask_export(lite_attn_mask_t mask, uint32_t *host_bits, void *stream);

/* Copy the compacted live lists to host memory (for inspection and tests).
 *   host_list : [G][Tk] uint32 entries j | (flags << 30), ascending j, flags
 *               bit 0 = live for the pair's first query tile, bit 1 = for the
 *               second (tiles of pair p: lite_attn_plan_pair_tiles; adjacent
 *               tiles 2p, 2p + 1 unless the plan has a pair stride); entries
 *               past the count are unspecified.
 *   host_cnt  : [G] int32 entry counts.   host_order : [G] int32 work order:
 *               pairs sorted by descending count, or, when one head's K and V
 *               exceed 32 MB (4*N*d bytes), the pairs in index (head-by-head)
 *               order, which keeps each head's K and V in L2 while its pairs
 *               run.  Any pointer may be NULL.
 * Synchronises `stream`. */
int lite_attn_mask_export_lists(lite_attn_mask_t mask, uint32_t *host_list, int32_t *host_cnt,
                                int32_t *host_order, void *stream);

/* Divergence of two masks of one plan: the number of tiles live in `a` and
 * not in `b`, and live in `b` and not in `a`.
 * Passage: skill page, "Core Concept" (the mask is updated only if the
 * attention pattern diverges significantly) and "Architecture Overview"
 * (Persistent Propagation: decisions carry forward unless the attention
 * distribution shifts).  A caller measures the shift by running a probe step
 * from an all-live mask into a second mask and comparing it with the
 * propagated one: tiles live only in the probe are the ones propagation would
 * never revive.
 *   a, b   : masks of the same plan (else PLAN_MISMATCH); a == b gives 0, 0.
 *   only_a : host out, tiles live in a and dead in b;  only_b : the converse.
 * Runs one small kernel on `stream` and synchronises it (scratch: two
 * counters in the plan's device block, so calls on one plan must not overlap).
 * Errors: INVALID_ARG, PLAN_MISMATCH, CUDA. */
int lite_attn_mask_compare(lite_attn_mask_t a, lite_attn_mask_t b, int64_t *only_a, int64_t *only_b,
                           void *stream);

/* One denoising step (the hot path).
 * Passage: skill page, "Core Concept" and "Architecture Overview" (QK-Skip
 * inside the FlashAttention softmax pipeline; persistent propagation);
 * abstract (skip decisions propagated forward).
 *   q, k, v : device bf16 [B][H][N][d] ([B][N][H][d] for LITE_LAYOUT_BNHD plans;
 *             the plan's first head of [B][heads_total][N][d] tensors for
 *             head-range plans, see lite_attn_plan_create_ex);
 *   o       : device bf16, same layout (out).
 *   mask_in : live tiles entering the step (only its live lists are read).
 *   mask_out: receives mask_in AND (not killed in this step); its live lists
 *             are rebuilt after the attention kernel.  mask_out == mask_in
 *             is allowed (in-place propagation).
 *   step    : 0 <= step < T, selects tau_step from the schedule.
 * Enqueues the attention kernel and the compaction kernel on `stream`.
 * Rows of o are fully overwritten; a query tile with no live key tile gets
 * zeros.  Errors: INVALID_ARG, PLAN_MISMATCH, CUDA. */
int lite_attn_step(lite_attn_plan_t plan, const void *q, const void *k, const void *v, void *o,
                   lite_attn_mask_t mask_in, lite_attn_mask_t mask_out, int step, void *stream);

/* Error of an attention output against a reference output of the plan's
 * shape (e.g. the dense output of a tau = -inf plan on the same inputs).  For
 * calibrating thresholds against per-step error budgets; not part of a step.
 * Passage: skill page, "Architecture Overview" (Accumulated-Error
 * Calibration: variable error budgets per timestep, early steps tolerating
 * less error).
 *   o, o_ref : device bf16, B*H*N*d elements each in the plan's layout.
 *   out      : host, 3 doubles: sum |o - o_ref|, max |o - o_ref|, sum |o_ref|
 *              (differences of the bf16 values, summed in fp64).
 * Runs one kernel on `stream` and synchronises it (scratch in the plan's
 * device block: calls on one plan must not overlap).
 * Errors: INVALID_ARG, CUDA. */
int lite_attn_output_error(lite_attn_plan_t plan, const void *o, const void *o_ref, double *out, void *stream);

/* Statistics of a mask plus plan-wide totals.  Blocks until the plan's last
 * step and the last call that wrote this mask (step, reset, import) have
 * finished on their streams, then reads the counters back on a stream of the
 * plan's own; work on other streams of the device is not waited for. */
int lite_attn_stats(lite_attn_plan_t plan, lite_attn_mask_t mask, lite_attn_stats_t *out);

/* Optional per-kernel timing with CUDA events on the step's stream.
 * enable != 0 starts recording (clearing previous records).
 * lite_attn_timing_read() synchronises, returns the summed milliseconds of
 * the attention kernels and of whole steps recorded since enabling, and the
 * number of steps; it then clears the records. */
int lite_attn_timing_enable(lite_attn_plan_t plan, int enable);
int lite_attn_timing_read(lite_attn_plan_t plan, double *attn_ms, double *step_ms, int64_t *n_steps);

/* Compaction without allocation.  This entry point has no counterpart in the
 * pages; it exists for callers that cannot call cudaMalloc: code whose device
 * memory is owned by another allocator (a framework's caching allocator or a
 * preallocated arena) and serving loops that must not allocate after start-up
 * (cudaMalloc can synchronise the device).  It rebuilds the compacted live lists
 * of a caller-owned bitmask into caller-owned buffers, exactly as the mask
 * store does after a step or an import, and allocates nothing: the kernel's
 * scratch (per-block partial counts and a completion counter) lives in a fixed
 * array inside this library.
 *   bits       : device [B*H*Tq][W] uint32, layout as above; bits >= Tk are ignored.
 *   list       : device out [G][Tk] uint32 entries j | (flags << 30) (as in
 *                lite_attn_mask_export_lists); entries past the count unspecified.
 *   cnt, order : device out [G] int32 (order = pairs by descending count).
 *   live_total : device out, one int64: number of live tiles in `bits`.
 *   Shapes: (Br, Bc) in {(64, 64), (128, 128)}, 1 <= N <= 2^20, and at most
 *   LITE_NOALLOC_MAX_PAIRS query-tile pairs G = B*H*ceil(Tq/2); larger shapes
 *   return LITE_ERR_UNSUPPORTED.
 * Checks before launching (INVALID_ARG otherwise): every buffer is memory of
 * the current device inside one allocation and at least the size above, bits,
 * list, cnt and order 4-byte aligned and live_total 8-byte aligned; no two of
 * the five buffers overlap; a non-NULL stream belongs to the current device.
 * The first call on a device (or on a thread whose current device is new)
 * looks up the scratch array's device address and keeps it for the life of
 * the process; make that first call before any stream capture.  A device
 * reset (cudaDeviceReset, or a primary context torn down and made again)
 * invalidates that address: do not call this entry point after one.  All calls
 * share the one scratch array: calls whose kernels overlap on the GPU (other
 * streams, other host threads) race and must be serialised by the caller.
 * Asynchronous on `stream`; errors: INVALID_ARG, UNSUPPORTED, CUDA. */
#define LITE_NOALLOC_MAX_PAIRS 65536
int lite_attn_compact_noalloc(const uint32_t *bits, int B, int H, int N, int Br, int Bc, uint32_t *list,
                              int32_t *cnt, int32_t *order, int64_t *live_total, void *stream);

/* Kernel launches issued by this library in the calling process so far. */
int64_t lite_attn_launch_count(void);

/* Static description of an error code (never NULL). */
const char *lite_attn_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* LITEATTN_H */
