// tide_internal.h - plan object and kernel launchers shared by the libtide.so
// translation units (not part of the public ABI; see include/tide.h).
#pragma once

#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "tide.h"

// Kernel ids (match tide_launch_ctas and tide_plan_last_launch).
enum : int32_t {
    K_RS = 0, K_AG = 1, K_STAGE = 2, K_SLOT_RS = 3, K_RS_TMA = 4, K_SLOT_RS_TMA = 5,
    K_RS_V32 = 6, K_SLOT_RS_V32 = 7, K_RS_TREE = 8, K_SLOT_RS_TREE = 9, K_AG_GATHER = 10,
    K_RS_TREE_V32 = 11, K_SLOT_RS_TREE_V32 = 12, K_STAGE_F32 = 13, K_SLOT_RS_F32 = 14,
    K_RS_F32 = 15, K_COUNT = 16
};

// A device pointer table with a host mirror: re-uploaded only when it changes.
struct PtrTable {
    const void** dev = nullptr;          // device array of `capacity` pointers
    std::vector<const void*> host;       // last uploaded contents
    int64_t capacity = 0;
    bool valid = false;                  // host mirror matches the device copy
    bool aligned16 = false;              // every pointer in it is 16-byte aligned
    bool aligned32 = false;              // every pointer in it is 32-byte aligned
};

struct tide_plan {
    int32_t device = -1;
    int32_t world = 0;
    int32_t rank = -1;                   // >= 0: the plan covers only this output rank's shard
    int32_t n_params = 0;
    uint32_t flags = 0;
    int64_t shard_numel = 0;             // Ns
    std::vector<int64_t> dim0, inner, numel, rows, chunk, offset;   // per param: d0, inner, d0*inner, S, c, off
    std::vector<tide_tile_t> tiles;
    std::vector<int64_t> chunk_tile_begin;  // [P*W+1]: chunk (i, r) holds tiles [begin[i*W+r], begin[i*W+r+1])
    bool tiles_aligned8 = true;          // every tile starts on 8-element boundaries (src and dst)
    bool tiles_aligned16 = true;         // ... and on 16-element boundaries
    std::vector<cudaEvent_t> seg_events; // pacing events of tide_rs_reduce_pipelined (created on first use)
    std::vector<cudaStream_t> ce_streams;  // copy-engine fan-out streams (created on first use)
    std::vector<cudaEvent_t> ce_events;    // their fork event [0] and join events [1..]
    struct CeIssuer* ce_issuer = nullptr;  // host threads that issue the copies (created on first use)
    // Copy-engine calls recorded as CUDA graphs, keyed by call kind, chunk range and
    // every buffer address of the call; replayed when the same buffers come back.
    struct CeGraph {
        int32_t kind = 0;
        int64_t j0 = 0, j1 = 0;
        std::vector<const void*> key;
        cudaGraphExec_t exec = nullptr;
        uint64_t last_use = 0;
    };
    std::vector<CeGraph> ce_graphs;
    uint64_t ce_clock = 0;
    cudaStream_t ce_capture_stream = nullptr;  // private stream the recordings are made on

    // device tables (absent for TIDE_PLAN_HOST_ONLY)
    tide_tile_t* d_tiles = nullptr;
    int64_t* d_numel = nullptr;
    int32_t* d_err = nullptr;
    unsigned long long* d_counter = nullptr;  // the reduction's tile claim counters (2 words)
    PtrTable grad_tab, param_tab, slot_tab, shard_tab;
    int64_t workspace_bytes = 0;

    int32_t sm_count = 0;
    int32_t blocks_per_sm[K_COUNT] = {};
    int32_t last_kernel = -1;            // kernel id of the last launch (-1: none or copy engines)
    int32_t last_ctas = 0;
};

namespace tide {

constexpr int kThreads = 256;

// Occupancy (resident CTAs per SM) of each kernel at kThreads threads.
int rs_blocks_per_sm(int world, bool slot, int order, bool v32);
bool rs_v32_applies(int world, int order);  // whether a 32-byte variant exists for this W and order
int rs_tma_blocks_per_sm(int world);  // also opts the TMA kernels in to their shared memory
int ag_blocks_per_sm(bool gather);
int stage_blocks_per_sm();
int stage_f32_blocks_per_sm();
int reduce_f32_blocks_per_sm(bool slot);

// Kernel launches; return the launch's cudaError_t.
// The RS launchers work on the plan's tiles [t0, t1) (t1 < 0: to the end).
cudaError_t launch_rs_reduce(const tide_plan* p, const void* const* d_src_tab, bool slot,
                             int64_t src_bound, float* out, int64_t out_numel, float scale,
                             bool do_scale, int order, int grid, cudaStream_t stream,
                             bool v32 = false, int64_t t0 = 0, int64_t t1 = -1);
cudaError_t launch_rs_reduce_tma(const tide_plan* p, const void* const* d_src_tab, bool slot,
                                 int64_t src_bound, float* out, int64_t out_numel, float scale,
                                 bool do_scale, int order, int grid, cudaStream_t stream,
                                 int64_t t0 = 0, int64_t t1 = -1);
cudaError_t launch_ag_place(const tide_plan* p, const uint16_t* ag, int64_t ag_numel,
                            const void* const* d_param_tab, int grid, cudaStream_t stream);
// Placement from W per-rank shards (d_shard_tab[r]: rank r's [Ns] shard).
cudaError_t launch_ag_gather(const tide_plan* p, const void* const* d_shard_tab, int64_t shard_numel,
                             const void* const* d_param_tab, int grid, cudaStream_t stream);
// Stages `sources` source ranks: W (d_grad_tab [W*P], d_slot_tab [W]) or 1 (one
// rank's gradients, d_grad_tab [P], into the one slot d_slot_tab[0]).
cudaError_t launch_slot_stage(const tide_plan* p, const void* const* d_grad_tab,
                              const void* const* d_slot_tab, int64_t slot_numel, int grid,
                              cudaStream_t stream, int32_t sources);

// fp32 gradients: one source rank's P gradients (d_grad_tab [P]) into its slot, and
// the rank-order reduction of W fp32 slots (d_slot_tab [W], advanced to the plan's
// first row; src_bound elements readable from each).  v8: every slot and out are
// 32-byte aligned.
cudaError_t launch_stage_f32(const tide_plan* p, const void* const* d_grad_tab, void* slot,
                             int64_t slot_numel, int grid, cudaStream_t stream);
cudaError_t launch_reduce_slots_f32(const tide_plan* p, const void* const* d_slot_tab, int64_t src_bound,
                                    float* out, int64_t out_numel, float scale, bool do_scale, bool v8,
                                    int grid, cudaStream_t stream);
// TIDE-RS on fp32 gradients read in place (d_grad_tab [W*P], k*P + i); v8: every
// gradient and out are 32-byte aligned.
cudaError_t launch_reduce_f32(const tide_plan* p, const void* const* d_grad_tab, float* out,
                              int64_t out_numel, float scale, bool do_scale, bool v8, int grid,
                              cudaStream_t stream);

// Copy-engine variants (no kernels).
cudaError_t ce_ag_place(tide_plan* p, const uint16_t* ag, void* const* params,
                        cudaStream_t stream);
// Placement from W per-rank shards (shards[r]: rank r's [Ns] shard).
cudaError_t ce_ag_gather(tide_plan* p, const void* const* shards, void* const* params,
                         cudaStream_t stream);
// Stages the chunks [j0, j1) (numbered i*W + r as in chunk_tile_begin; j1 < 0:
// all) from every source rank k into slot k.  The copies are issued directly
// (`record` = false): a recorded graph of them measured slower (Wan2.2 group:
// 3.55 against 4.07 TB/s; within 2 % elsewhere).  one_source: grads holds one
// rank's P gradients and slots one slot, which receives them.  esize: bytes per
// element of the gradients and slots (2: bf16, 4: fp32).
cudaError_t ce_slot_stage(tide_plan* p, const void* const* grads, void* const* slots,
                          cudaStream_t stream, int64_t j0 = 0, int64_t j1 = -1, bool record = false,
                          bool one_source = false, int esize = 2);
// A one-rank plan's phase 1: chunk `rank` of every rank k's gradients into
// slots[k] (that rank's row only, Ns elements), for the chunks [j0, j1).
cudaError_t ce_rank_stage(tide_plan* p, const void* const* grads, void* const* slots,
                          cudaStream_t stream, int64_t j0, int64_t j1);
// Stops and frees the plan's copy-issuing threads and recorded graphs.
void ce_release(tide_plan* p);

}  // namespace tide
