/*
 * tide.h - C ABI of libtide.so: layout-aware reduce-scatter and all-gather
 * placement for FSDP2-style per-parameter storage.
 *
 * Source of the method: "The Endgame of FSDP Communication: Layout-Aware
 * Collectives on Copy Engines, RDMA, and NVSwitch" (weekinpapers.com, Abstract)
 * and the kongchang.com article "The Endgame of FSDP Communication: TIDE
 * Zero-Copy Collective Communication Optimization" (sections "The Root of FSDP2
 * Communication Overhead" and "TIDE's Design Approach").  TIDE computes the
 * final address of every shard element inside the collective itself: the
 * all-gather result lands directly in per-parameter storage (TIDE-AG) and the
 * reduce-scatter reads per-parameter bf16 gradients where they are and writes
 * fp32 shards (TIDE-RS), so neither a copy-out nor a packed fp32 staging
 * buffer exists.  This library implements the per-rank arithmetic and
 * addressing of those two collectives with the network taken out: the W
 * data-parallel ranks are W sets of buffers that the calling GPU's kernels
 * read, its own memory or, through CUDA IPC (tide_ipc_*), other processes'
 * buffers, with one-rank plans (tide_plan_group_rank) for a process that holds
 * one rank.  Gradients FSDP2 keeps in fp32 (accumulated with gradient sync off)
 * have calls of their own: tide_rs_reduce_f32, tide_rs_stage_one_f32 and
 * tide_rs_reduce_slots_f32.
 *
 * Layout (the pages leave it open; this is the reading every call follows):
 *   param i has shape (d0_i, ...) with inner_i = product of the trailing dims;
 *   S_i = ceil(d0_i / W) rows per shard, c_i = S_i * inner_i elements per chunk;
 *   rank r owns rows [r*S_i, min((r+1)*S_i, d0_i)); rows d0_i .. W*S_i-1 are pad;
 *   inside a rank's shard, params follow the group order with no gaps:
 *   off_i = sum_{j<i} c_j, Ns = sum_i c_i; a rank-major buffer is [W][Ns].
 *
 * Conventions for every call:
 *   - The caller owns every data buffer.  All pointers to data are device
 *     pointers of the plan's device; pointer ARRAYS (grads, params, slots) and
 *     numel arrays are host arrays that are only read during the call.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronize the device, except tide_plan_group,
 *     tide_plan_destroy, tide_plan_check and tide_plan_errors where stated.
 *   - All arguments are validated on the host before anything is enqueued; on
 *     any error status nothing has been enqueued.
 *   - A plan keeps small device tables (tile list, pointer tables, an error
 *     word, and two counters with which the reduction's CTAs claim tiles on long
 *     launches; the launch's last CTA puts them back to zero, so two reductions of
 *     one plan must never run at the same time: they would share the counters).  A pointer table is re-uploaded, stream-ordered, only when its
 *     contents change.  One plan must be used from one stream at a time (or the
 *     caller orders the streams) and from one host thread at a time; different
 *     plans are independent.
 *   - bf16 buffers must be 2-byte aligned and fp32 buffers 4-byte aligned; any
 *     such alignment is accepted (16-byte alignment gives the fast path).
 *   - No call allocates device memory except tide_plan_group.
 *   - The plan-based calls (tide_ag_place, tide_rs_reduce, tide_rs_stage,
 *     tide_rs_reduce_slots, tide_rs_reduce_pipelined; tested) can be captured into a
 *     CUDA graph once the same buffers have been used in an uncaptured call on
 *     the same plan (that call uploads the pointer tables and creates the
 *     pipeline's events and the copy-engine streams; a capture that needs an
 *     upload fails with TIDE_ERR_CUDA).  Replays read the buffers' current
 *     contents.
 *   - TIDE_ENGINE_CE calls spread their memcpys over 8 streams that the plan
 *     creates on first use (no device memory), forked from the call's stream
 *     with an event and joined back to it before the call returns; work
 *     enqueued on the call's stream afterwards sees every copy.  The copies
 *     are issued by the calling thread and 3 host threads that the plan starts
 *     on its first copy-engine call (they sleep between calls and are joined
 *     by tide_plan_destroy); the call returns once every copy is enqueued.
 *   - A TIDE_ENGINE_CE placement (tide_ag_place, tide_ag_gather_place) made
 *     outside any stream capture records its copies once as a CUDA graph (on a
 *     private stream of the plan) the first time its set of buffer addresses
 *     is seen, and then launches that graph on the call's stream, for this
 *     call and every later one with the same addresses: one graph launch
 *     instead of one host call per copy.  The plan keeps the 4 most recently
 *     used recordings and frees them in tide_plan_destroy.  A call on a stream
 *     that is being captured issues its copies directly into that capture.
 *     Slot-Reuse staging on the copy engines always issues its copies directly.
 */
#ifndef TIDE_H
#define TIDE_H

#include <stdint.h>

#if defined(__GNUC__)
#define TIDE_API __attribute__((visibility("default")))
#else
#define TIDE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TIDE_OK = 0,
    TIDE_ERR_INVALID_ARG = -1,  /* null pointer, bad enum, bad shape, aliasing */
    TIDE_ERR_ALIGNMENT = -2,    /* buffer not aligned to its element size */
    TIDE_ERR_SIZE = -3,         /* a buffer is smaller than the plan needs */
    TIDE_ERR_CUDA = -4,         /* a CUDA runtime call or launch failed */
    TIDE_ERR_NOMEM = -5,        /* host or device allocation failed */
    TIDE_ERR_DEVICE = -6,       /* wrong current device, or a host-only plan */
    TIDE_ERR_KERNEL_CHECK = -7  /* a kernel's own range check rejected a tile */
} tide_status_t;

enum { TIDE_ENGINE_SM = 0, TIDE_ENGINE_CE = 1 };
enum { TIDE_ORDER_RANK = 0, TIDE_ORDER_TREE = 1 };
enum { TIDE_SCALE_NONE = 0, TIDE_SCALE_INV_WORLD = 1 };
enum {
    TIDE_PLAN_HOST_ONLY = 1, /* flag: build the tables on the host only (no CUDA calls) */
    TIDE_PLAN_TMA = 2,       /* flag: reduce with the bulk-copy (TMA) kernel where it applies */
    /* flag, test hook for the timeout path: with TIDE_PLAN_TMA, CTA 0 of every
     * bulk-copy launch withholds its first stage (no arrival, no copy), so its
     * consumers' bounded wait gives up after about 1 s; the CTA stops, the
     * launch sets TIDE_KCHECK_TIMEOUT and its result is incomplete.  Nothing
     * faults or hangs.  Not for use outside tests. */
    TIDE_PLAN_TEST_TMA_TIMEOUT = 4,
    /* flag: short-lived CTAs (kongchang.com, "TIDE's Design Approach": node-local
     * accumulation by short-lived CTAs; weekinpapers.com Abstract).  The SM
     * kernels (every kernel but the bulk-copy ones) launch one CTA per unit of
     * work -- per tile, or per (tile, rank) for Slot-Reuse staging -- that does
     * that unit and exits, instead of a persistent grid; max_ctas must then be
     * 0 (TIDE_ERR_INVALID_ARG otherwise).  Each CTA holds its SM for a few
     * microseconds, so when work of a higher-priority stream (say a GEMM) is
     * waiting for SMs it gets them as CTAs finish, instead of waiting for the
     * whole reduction.  Same results, same bits. */
    TIDE_PLAN_SHORT_CTAS = 8
};

#define TIDE_MAX_WORLD 256
#define TIDE_TILE_ELEMS 8192
#define TIDE_NOALLOC_SCRATCH_BYTES (1 << 20)

/* One parameter: dim 0 and the product of the remaining dims (1 for a 1-D param). */
typedef struct {
    int64_t dim0;
    int64_t inner;
} tide_param_t;

/*
 * One unit of kernel work: elements [e0, e0 + n_total) of the chunk of param
 * `param` that rank `rank` owns, with e0 a multiple of TIDE_TILE_ELEMS.
 *   src_off = rank*c_i + e0        offset into the param's own tensor
 *   dst_off = rank*Ns + off_i + e0 offset into a rank-major [W][Ns] buffer
 *             (off_i + e0, inside the rank's own shard, in a one-rank plan)
 *   the first n_valid elements hold data; the remaining ones are padding.
 */
typedef struct {
    int64_t src_off;
    int64_t dst_off;
    int32_t param;
    int32_t rank;
    int32_t n_valid;
    int32_t n_total;
} tide_tile_t;

typedef struct tide_plan tide_plan_t;

/*
 * Build the address tables of a parameter group for W = `world` ranks: per
 * param S_i, c_i, off_i; per (param, rank) chunk the valid and pad lengths; the
 * tile list the kernels walk.  These tables are where the per-parameter layout
 * enters the collective's address computation (weekinpapers.com Abstract),
 * built once per group.  1 <= world <= TIDE_MAX_WORLD, 0 <= n_params, dims >= 0.
 * Unless flags has TIDE_PLAN_HOST_ONLY, the tables are uploaded to `device`
 * (cudaMalloc + synchronous copies; the current device is restored).
 * On success *out_plan owns the tables; free it with tide_plan_destroy.
 */
TIDE_API tide_status_t tide_plan_group(const tide_param_t* params, int32_t n_params, int32_t world,
                              int32_t device, uint32_t flags, tide_plan_t** out_plan);

/*
 * A plan for ONE output rank of a group (0 <= rank < world): the same layout,
 * but only rank `rank`'s tiles, with output offsets inside its own shard.  It
 * is the plan a real data-parallel rank uses to reduce-scatter (weekinpapers.com
 * Abstract, TIDE-RS: each rank's shard is reduced from every rank's
 * gradients): tide_rs_reduce with it reads chunk `rank` of every rank's
 * gradients, which may be peer pointers (other processes' or GPUs' memory
 * mapped into this one), and writes out[0 .. Ns):
 *   out[off_i + e] = s * fl32(sum_k fp32(g_{k,i}[rank*c_i + e])),  +0.0 at pads,
 * the same bits as rows [rank*Ns, (rank+1)*Ns) of the all-rank call.  Only
 * tide_rs_reduce without slots accepts such a plan; the other data calls
 * return TIDE_ERR_INVALID_ARG for it.  Arguments and errors as tide_plan_group.
 */
TIDE_API tide_status_t tide_plan_group_rank(const tide_param_t* params, int32_t n_params,
                                            int32_t world, int32_t rank, int32_t device,
                                            uint32_t flags, tide_plan_t** out_plan);

/* Free a plan (NULL is accepted).  Synchronizes the plan's device first, so
 * that no enqueued call can still read the tables. */
TIDE_API void tide_plan_destroy(tide_plan_t* plan);

/* Group-level sizes.  Any output pointer may be NULL.  workspace_bytes counts
 * every byte of device memory the plan holds (tables only: no staging). */
TIDE_API tide_status_t tide_plan_info(const tide_plan_t* plan, int32_t* world, int32_t* n_params,
                             int64_t* shard_numel, int64_t* n_tiles, int64_t* workspace_bytes);

/* Per-param layout: S_i, off_i, padded numel W*c_i, and c_i.  Any output may be NULL. */
TIDE_API tide_status_t tide_plan_query(const tide_plan_t* plan, int32_t param, int64_t* shard_rows,
                              int64_t* shard_offset, int64_t* padded_numel, int64_t* chunk_numel);

/* Copy up to `capacity` tiles into out (host array); *n_written gets the count.
 * Tiles are listed chunk by chunk: param 0's chunks of ranks 0..W-1, then
 * param 1's, and so on; within a chunk by position. */
TIDE_API tide_status_t tide_plan_tiles(const tide_plan_t* plan, tide_tile_t* out, int64_t capacity,
                              int64_t* n_written);

/*
 * TIDE-AG placement (weekinpapers.com Abstract, TIDE-AG; kongchang.com
 * "TIDE's Design Approach"): the rank-major all-gather buffer ag_buf (bf16
 * [W][Ns], ag_numel >= W*Ns) is written straight into per-parameter padded
 * storage: param_storage[i] (bf16, param_numel[i] >= W*c_i) receives
 *   param_i[r*c_i + e] = ag[r*Ns + off_i + e]  for r*c_i + e < d0_i*inner_i,
 *   param_i[r*c_i + e] = +0                    for the pad rows.
 * Pad positions of ag_buf are never read.  engine: TIDE_ENGINE_SM (one kernel
 * launch, at most max_ctas CTAs, 0 = as many as fit) or TIDE_ENGINE_CE (copy
 * engine memcpys and memsets only; max_ctas is ignored).  ag_buf must not
 * overlap any param storage.
 */
TIDE_API tide_status_t tide_ag_place(const tide_plan_t* plan, const void* ag_buf, int64_t ag_numel,
                            void* const* param_storage, const int64_t* param_numel,
                            int32_t engine, int32_t max_ctas, void* stream);

/*
 * TIDE-AG placement from per-rank shards (weekinpapers.com Abstract, TIDE-AG:
 * shards land in parameter storage; kongchang.com "TIDE's Design Approach"):
 * the same result as tide_ag_place, but rank r's shard is its own buffer
 * shards[r] (bf16, shard_numel >= Ns elements each) instead of row r of one
 * rank-major buffer, so each rank can place every peer's shard straight from
 * that peer's memory (peer pointers):
 *   param_i[r*c_i + e] = shards[r][off_i + e]  for valid rows, +0 for pad rows.
 * shards is a host array of W device pointers; shards are only read, and no
 * shard may overlap any parameter storage.  engine: TIDE_ENGINE_SM (one kernel
 * launch) or TIDE_ENGINE_CE (one copy per (param, rank) chunk with data plus
 * one memset per padded param).  Needs an all-rank plan.
 */
TIDE_API tide_status_t tide_ag_gather_place(const tide_plan_t* plan, const void* const* shards,
                                            int64_t shard_numel, void* const* param_storage,
                                            const int64_t* param_numel, int32_t engine,
                                            int32_t max_ctas, void* stream);

/*
 * TIDE-RS (weekinpapers.com Abstract, TIDE-RS and the two-phase pipeline;
 * kongchang.com "TIDE's Design Approach"): per-parameter bf16 gradients are
 * reduced straight into fp32 rank-major shards with no packed fp32 buffer.
 * grads is a host array of W*P device pointers, grads[k*P + i] = rank k's
 * unpadded gradient of param i (grad_numel[k*P+i] >= d0_i*inner_i).  out is
 * fp32 [W][Ns] (out_numel >= W*Ns); rank r's shard is out[r*Ns, (r+1)*Ns):
 *   out[r*Ns + off_i + e] = s * fl32(sum_{k=0..W-1} fp32(g_{k,i}[r*c_i + e]))
 * for r*c_i + e < d0_i*inner_i, and +0.0 at pad positions.  scale_mode
 * TIDE_SCALE_INV_WORLD multiplies once by fl32(1/W) after the sum; NONE skips it.
 * order TIDE_ORDER_RANK adds in rank order 0..W-1 (bit-exact against the stock
 * pack-then-reduce result); TIDE_ORDER_TREE adds adjacent ranks pairwise, level
 * by level, an odd last one carried to the next level (every kernel gives the
 * same bits; within |err| <= 1e-6 * sum|terms| of the exact sum for W <= 64).
 * With a one-rank plan (tide_plan_group_rank) out is that rank's shard only:
 * fp32 [Ns], out_numel >= Ns.
 * slots == NULL: one kernel launch.  slots != NULL: Slot-Reuse, the two phases
 * of tide_rs_stage (with `engine`) and tide_rs_reduce_slots run back to back;
 * slots is a host array of W device pointers to bf16 [W][Ns] buffers
 * (slot_numel elements each, >= W*Ns) whose contents are overwritten.
 * out must not overlap grads or slots; slots must not overlap grads.
 */
TIDE_API tide_status_t tide_rs_reduce(const tide_plan_t* plan, const void* const* grads,
                             const int64_t* grad_numel, float* out, int64_t out_numel,
                             int32_t scale_mode, int32_t order, void* const* slots,
                             int64_t slot_numel, int32_t engine, int32_t max_ctas, void* stream);

/*
 * Slot-Reuse phase 1 (weekinpapers.com Abstract: gradients staged in vacated
 * all-gather slots; gradient reads are the pipeline's first phase): rank k's
 * gradients are copied, still bf16, into slot k in the all-gather layout,
 *   slot_k[r*Ns + off_i + e] = g_{k,i}[r*c_i + e]  for valid positions;
 * pad positions of the slots are not written.  engine SM (one launch) or CE.
 */
TIDE_API tide_status_t tide_rs_stage(const tide_plan_t* plan, const void* const* grads,
                            const int64_t* grad_numel, void* const* slots, int64_t slot_numel,
                            int32_t engine, int32_t max_ctas, void* stream);

/*
 * Slot-Reuse phase 1 for the one rank a process holds (same passages): that
 * rank's gradients alone are copied, still bf16, into its own slot,
 *   slot[r*Ns + off_i + e] = g_i[r*c_i + e]  for valid positions, every r;
 * pad positions of the slot are not written.  This is tide_rs_stage's copy for
 * one source rank (its result does not depend on which rank that is): each
 * process stages its own gradients, and the slots then reach the other ranks as
 * peer memory.  grads is a host array of P device pointers (grad_numel[i] >=
 * d0_i*inner_i), slot one bf16 buffer of slot_numel >= W*Ns elements, which
 * must not overlap any gradient.  engine SM (one launch) or CE.  Needs an
 * all-rank plan.
 */
TIDE_API tide_status_t tide_rs_stage_one(const tide_plan_t* plan, const void* const* grads,
                                         const int64_t* grad_numel, void* slot, int64_t slot_numel,
                                         int32_t engine, int32_t max_ctas, void* stream);

/*
 * Slot-Reuse phase 2: out[r*Ns + j] = s * fl32(sum_k fp32(slot_k[r*Ns + j])) at
 * valid positions (from the plan), +0.0 at pad positions.  One kernel launch.
 * With a one-rank plan (rank r) out is that rank's shard only, fp32 [Ns]
 * (out_numel >= Ns): out[j] = s * fl32(sum_k fp32(slot_k[r*Ns + j])); the
 * slots may then be peers' memory.
 */
TIDE_API tide_status_t tide_rs_reduce_slots(const tide_plan_t* plan, const void* const* slots,
                                   int64_t slot_numel, float* out, int64_t out_numel,
                                   int32_t scale_mode, int32_t order, int32_t max_ctas,
                                   void* stream);

/*
 * Slot-Reuse for fp32 gradients.  While gradient sync is off, FSDP2 keeps
 * gradients in its fp32 reduce dtype across micro-batches and packs those at the
 * next synced backward; the layout-aware reduction applies to them unchanged
 * (weekinpapers.com, Abstract: gradients read where they lie, reduced into fp32
 * shards), with 4-byte slot words and no bf16 widening.  Rank order only.
 *
 * tide_rs_stage_one_f32: slot[r*Ns + off_i + e] = g_i[r*c_i + e] for every rank
 * r and valid e, a copy of the 4-byte words; pad positions of the slot are not
 * written.  grads: host array of P device pointers to fp32 gradients
 * (grad_numel[i] >= d0_i*inner_i, 4-byte aligned); slot: one device buffer of
 * fp32 [W][Ns] (slot_numel >= W*Ns), overlapping no gradient.  engine SM (one
 * kernel launch) or CE (per param one 2-D copy plus at most one 1-D copy on the
 * copy engines, no kernel).  Needs an all-rank plan (TIDE_ERR_INVALID_ARG
 * otherwise).
 *
 * tide_rs_reduce_slots_f32: out[r*Ns + j] = s * fl32(sum_{k=0..W-1}
 * slot_k[r*Ns + j]), summed in rank order from slot_0 in fp32 (round to nearest
 * even, no fused multiply-add), s = fl32(1/W) under TIDE_SCALE_INV_WORLD; +0.0
 * at pad positions.  slots: host array of W device pointers to fp32 [W][Ns]
 * buffers of slot_numel >= W*Ns elements each (read only; peers' memory is
 * accepted).  out: fp32 [W][Ns], or fp32 [Ns] with a one-rank plan (rank r),
 * whose sums then read rows [r*Ns, (r+1)*Ns) of every slot.  out must not
 * overlap a slot.  One kernel launch.
 *
 * Both: errors as tide_rs_stage_one / tide_rs_reduce_slots (TIDE_ERR_ALIGNMENT
 * for a buffer that is not 4-byte aligned); nothing is enqueued on error; the
 * caller owns every buffer.
 */
/*
 * TIDE-RS on fp32 gradients read where they lie (no slot, no packed buffer):
 * out[r*Ns + off_i + e] = s * fl32(sum_{k=0..W-1} g_{k,i}[r*c_i + e]) in rank
 * order from g_0 (fp32, round to nearest even), +0.0 at pad positions; with a
 * one-rank plan (rank r) out is that rank's fp32 [Ns] shard.  grads: host array
 * of W*P device pointers to fp32 gradients, index k*P + i (grad_numel[k*P+i] >=
 * d0_i*inner_i; 4-byte aligned; peers' memory accepted); out must overlap no
 * gradient.  One kernel launch.  Errors as tide_rs_reduce.
 */
TIDE_API tide_status_t tide_rs_reduce_f32(const tide_plan_t* plan, const float* const* grads,
                                          const int64_t* grad_numel, float* out, int64_t out_numel,
                                          int32_t scale_mode, int32_t max_ctas, void* stream);
TIDE_API tide_status_t tide_rs_stage_one_f32(const tide_plan_t* plan, const float* const* grads,
                                             const int64_t* grad_numel, float* slot, int64_t slot_numel,
                                             int32_t engine, int32_t max_ctas, void* stream);
TIDE_API tide_status_t tide_rs_reduce_slots_f32(const tide_plan_t* plan, const float* const* slots,
                                                int64_t slot_numel, float* out, int64_t out_numel,
                                                int32_t scale_mode, int32_t max_ctas, void* stream);

/*
 * Slot-Reuse with the two phases overlapped (weekinpapers.com Abstract: the
 * two-phase pipeline keeps gradient reads apart from the reduction's
 * progress, and copy engines move the gradients).  Same result as
 * tide_rs_reduce with the same slots (same bits).  The (param, rank) chunks,
 * taken param by param and within a param rank by rank, are cut into
 * n_segments contiguous groups of about equal valid elements
 * (1 <= n_segments <= W; a group may be empty).  For each group, phase 1
 * stages its chunks from every source rank into the slots with copy-engine
 * memcpys on `copy_stream`, then phase 2 reduces them on `stream` (one kernel
 * launch per group) while the copy engines already stage the next group.
 * Work enqueued on `stream` before the call is ordered before the copies;
 * work enqueued on `stream` after it sees the complete result.  `copy_stream`
 * may equal `stream` (the phases then run one after the other).  The plan
 * creates its pacing events (no device memory) on first use.
 * With a one-rank plan (rank r) the call is that rank's share of the
 * exchange: out is its fp32 shard [Ns] (out_numel >= Ns), and slots[k] receives
 * rank k's row r only (slot_numel >= Ns each): chunk r of rank k's gradient of
 * param i lands at slots[k] + off_i.  The gradients may be peers' memory, so
 * the copy engines carry the transfer and the SMs reduce from local slots;
 * the result equals the one-rank tide_rs_reduce (same bits).
 */
TIDE_API tide_status_t tide_rs_reduce_pipelined(const tide_plan_t* plan, const void* const* grads,
                                                const int64_t* grad_numel, float* out,
                                                int64_t out_numel, int32_t scale_mode,
                                                int32_t order, void* const* slots,
                                                int64_t slot_numel, int32_t n_segments,
                                                int32_t max_ctas, void* stream, void* copy_stream);

/* Bits of a plan's device error word. */
enum {
    TIDE_KCHECK_TILE = 1,    /* a tile descriptor pointed outside its buffers; the tile was skipped */
    TIDE_KCHECK_TIMEOUT = 2  /* a bounded wait of the bulk-copy kernel gave up (about 1 s); that CTA stopped */
};

/*
 * Read and clear the plan's device error word: synchronizes `stream`, then
 * returns TIDE_ERR_KERNEL_CHECK if a kernel enqueued before it set any bit
 * (a rejected tile is skipped, nothing outside the buffers is touched; a
 * timed-out CTA leaves its remaining tiles unwritten), else TIDE_OK.
 */
TIDE_API tide_status_t tide_plan_check(tide_plan_t* plan, void* stream);

/* tide_plan_check that also stores the bits it read (TIDE_KCHECK_*, 0 if none)
 * in *bits. */
TIDE_API tide_status_t tide_plan_errors(tide_plan_t* plan, void* stream, int32_t* bits);

/*
 * Allocation-free rank-order reduction.  The paper has no counterpart: this
 * entry point exists for callers that cannot allocate device memory, which
 * tide_plan_group does.  Examples: a training runtime whose caching allocator
 * has already reserved the GPU's memory for its own arena (a foreign
 * cudaMalloc then fails or fragments it), or a hot loop that cannot afford the
 * device-wide synchronisation cudaMalloc/cudaFree may cause.
 * Computes exactly what tide_rs_reduce computes with slots == NULL and
 * TIDE_ORDER_RANK (same bits), for the group given directly by params /
 * n_params / world instead of a plan; grads, grad_numel, out, out_numel,
 * scale_mode, max_ctas and stream mean what they mean there.
 * It calls no cudaMalloc, cudaFree or other allocating routine.  Its tables
 * (32*P + 8*W*P bytes) live in one file-scope device array of
 * TIDE_NOALLOC_SCRATCH_BYTES (1 MiB) that every GPU loading this library
 * holds until the process exits; a larger group is rejected with
 * TIDE_ERR_SIZE before anything is enqueued.  The first call on each device
 * looks up that device's address of the array; make that first call before
 * any stream capture.  That address is kept for the life of the process:
 * after cudaDeviceReset on a device, do not call this entry point on that
 * device again.  The tables are copied in from one host array that the next
 * call reuses, so a call on a stream that is being captured is refused with
 * TIDE_ERR_INVALID_ARG (nothing enqueued).  Every call rewrites the tables its
 * kernel reads, so no state carries over, but all calls share the one array:
 * calls that may overlap on the GPU (on streams the caller does not order)
 * race and must not be issued.
 */
TIDE_API tide_status_t tide_rs_reduce_noalloc(const tide_param_t* params, int32_t n_params,
                                              int32_t world, const void* const* grads,
                                              const int64_t* grad_numel, float* out,
                                              int64_t out_numel, int32_t scale_mode,
                                              int32_t max_ctas, void* stream);

/* The number of CTAs a kernel call with this max_ctas would launch (0 if that
 * kernel cannot run on this plan; the unit count under TIDE_PLAN_SHORT_CTAS).  kernel: 0 = RS reduce (load/store kernel),
 * 1 = AG place, 2 = Slot-Reuse stage, 3 = slot reduce (load/store), 4 = RS
 * reduce with bulk-copy staging, 5 = slot reduce with bulk-copy staging,
 * 6 = RS reduce with 32-byte loads, 7 = slot reduce with 32-byte loads,
 * 8 = RS reduce in tree order, 9 = slot reduce in tree order,
 * 10 = AG placement from per-rank shards (tide_ag_gather_place),
 * 11 = RS reduce in tree order with 32-byte loads, 12 = slot reduce in tree
 * order with 32-byte loads, 13 = Slot-Reuse stage of fp32 gradients
 * (tide_rs_stage_one_f32), 14 = slot reduce of fp32 slots (tide_rs_reduce_slots_f32),
 * 15 = RS reduce of fp32 gradients (tide_rs_reduce_f32).
 * The reductions use kernels 4/5 (one CTA per SM, TMA loads into shared memory)
 * when the plan was built with TIDE_PLAN_TMA, every tile starts on an
 * 8-element boundary and every source and the output are 16-byte aligned.
 * Otherwise they use the 32-byte kernels (rank order 6/7 when W = 2 or W >= 5,
 * tree order 11/12 when W is 2, 4, 8 or 16) if every tile starts on a 16-element
 * boundary and every source and the output are 32-byte aligned; else kernels
 * 0/3 (rank order) or 8/9 (tree order).
 * Kernels of the same order give the same bits.  With the whole grid the
 * load/store kernels are the faster ones on B200; the bulk-copy kernels move
 * more bytes per CTA, which matters when max_ctas is small. */
TIDE_API tide_status_t tide_launch_ctas(const tide_plan_t* plan, int32_t kernel, int32_t max_ctas,
                               int32_t* ctas);

/* The kernel id (as in tide_launch_ctas; -1 for copy-engine calls or none yet)
 * and CTA count of the plan's most recent kernel launch. */
TIDE_API tide_status_t tide_plan_last_launch(const tide_plan_t* plan, int32_t* kernel,
                                             int32_t* ctas);

/*
 * Peer buffers across processes (CUDA IPC), for the exchange between ranks that
 * run as one process per GPU: each rank reduces its own shard from every
 * rank's gradients and places every rank's shard (weekinpapers.com Abstract,
 * TIDE-RS and TIDE-AG; kongchang.com "TIDE's Design Approach"), so the
 * pointer tables of tide_rs_reduce / tide_ag_gather_place name other ranks'
 * buffers.  The allocation must come from cudaMalloc (PyTorch's default
 * caching allocator qualifies; its expandable segments do not).
 *
 * tide_ipc_export: for the device buffer dev_ptr, writes the IPC handle of the
 * allocation that holds it (TIDE_IPC_HANDLE_BYTES bytes into the host buffer
 * `handle`), dev_ptr's byte offset inside that allocation (*offset), and, if
 * device is not NULL, the allocation's device (*device).  The handle stays
 * valid while the allocation lives.  TIDE_ERR_INVALID_ARG for a NULL or
 * non-device pointer.
 * tide_ipc_open: in another process, maps the exported allocation for use by
 * kernels on `device` (made current for the call, then restored), enabling
 * peer access from `device` to the owner's GPU as needed; *base receives the
 * mapping's address, to which the exporter's offset is added.  The same
 * allocation may be opened once per process and device.  TIDE_ERR_CUDA when the
 * runtime refuses (no peer access between the two GPUs, a handle from this
 * same process, an expired allocation).
 * tide_ipc_close: unmaps a base returned by tide_ipc_open (same device), after
 * every call that reads it has completed.
 * tide_peer_access: *can_access = 1 when kernels on `device` can read `peer`'s
 * memory directly (always for device == peer), else 0.
 * None of these synchronizes other processes: the caller orders ranks' writes
 * and reads with host barriers.
 */
#define TIDE_IPC_HANDLE_BYTES 64
TIDE_API tide_status_t tide_ipc_export(const void* dev_ptr, void* handle, int64_t* offset,
                                       int32_t* device);
TIDE_API tide_status_t tide_ipc_open(const void* handle, int32_t device, void** base);
TIDE_API tide_status_t tide_ipc_close(void* base, int32_t device);
TIDE_API tide_status_t tide_peer_access(int32_t device, int32_t peer, int32_t* can_access);

/*
 * Ordering between ranks on the device, with bounded waits (weekinpapers.com,
 * Abstract: each rank's collectives read the other ranks' buffers in place, so
 * a rank may read a peer's buffer only after the peer wrote it, and overwrite
 * its own only after every peer read it).  Both calls are stream-ordered on
 * the current device and need no plan; flags are 32-bit words in device
 * memory, this process's own or a peer's mapped with tide_ipc_open.
 *
 * tide_flag_signal: one kernel thread makes every earlier write of this device
 * visible to the whole system, then stores `value` into *flag with release
 * semantics.  TIDE_ERR_INVALID_ARG for a NULL flag, TIDE_ERR_ALIGNMENT if it
 * is not 4-byte aligned.
 *
 * tide_flag_wait: one CTA polls the n flags (flags: a host array of n device
 * pointers, 1 <= n <= TIDE_MAX_WORLD) with acquire loads until each holds
 * `value` or a later epoch (flag - value, as a signed 32-bit difference, >= 0),
 * or until timeout_ns (1 ns .. 60 s) has passed; it then writes *status (a
 * device int32): 0 if every flag got there, else 1 + the index of the first
 * one that did not.  The wait always ends: at the time limit, and as a second
 * bound after an iteration cap.  Work queued after it on the stream runs when
 * it ends, whatever the status, so the caller reads *status before trusting
 * that work.  A waiting kernel must not be the only way its flag can be set
 * on the same GPU (no two launches that wait on one another share a GPU).
 * TIDE_ERR_INVALID_ARG / TIDE_ERR_ALIGNMENT for bad arguments, checked before
 * anything is enqueued.
 */
TIDE_API tide_status_t tide_flag_signal(void* flag, uint32_t value, void* stream);
TIDE_API tide_status_t tide_flag_wait(const void* const* flags, int32_t n, uint32_t value,
                                      int64_t timeout_ns, int32_t* status, void* stream);

TIDE_API const char* tide_status_string(tide_status_t status);
TIDE_API int32_t tide_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TIDE_H */
