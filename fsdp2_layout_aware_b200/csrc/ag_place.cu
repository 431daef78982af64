// ag_place.cu - TIDE-AG placement kernel and the Slot-Reuse staging kernel (sm_100a).
//
// AG placement ("The Endgame of FSDP Communication", weekinpapers.com,
// Abstract, TIDE-AG; kongchang.com, "TIDE's Design Approach"): shards arrive
// in parameter storage, not in a flat buffer that a copy-out pass rearranges.
// On one GPU the arrival is this kernel: tile by tile it copies the valid part
// of rank r's chunk of param i from the rank-major buffer,
//   param_i[r*c_i + e] = ag[r*Ns + off_i + e],
// and writes +0 to the chunk's pad rows; pad positions of ag are never read.
//
// Slot-Reuse staging (same Abstract, the two-phase pipeline's gradient-read
// phase with Slot-Reuse): rank k's gradients are copied, unconverted, into
// slot k in the all-gather layout, slot_k[r*Ns + off_i + e] = g_{k,i}[r*c_i + e];
// pad positions of the slot are not written.
//
// Both are pure copies (2 bytes read + 2 written per element): HBM-bound.
// Each CTA walks the plan's tiles round-robin and moves a tile with 32-byte
// streaming loads/stores (sm_100 vector width), two in flight per thread;
// 16-byte vectors measured 5-8 % slower on B200.  (Measured
// alternatives that were slower on B200: a bulk L2 prefetch of the next tile,
// every thread loading the descriptor itself with no barrier, and thread 0
// prefetching the next descriptor into a double-buffered slot.)
#include "device_common.cuh"
#include "tide_internal.h"

namespace tide {
namespace {

constexpr int kCopyU = 2;  // 32-byte vectors in flight per thread (64 bytes, as 4 x 16 before)

struct AgParams {
    const tide_tile_t* tiles;
    int64_t n_tiles;
    const uint16_t* ag;            // rank-major source [W][Ns] (placement)
    int64_t ag_numel;              // its length; for gathering, each shard's length
    const void* const* shard_tab;  // gathering: [W] per-rank shards of Ns elements
    int64_t shard_numel;           // Ns
    int32_t world;
    const void* const* param_tab;  // [P] padded param storage
    const int64_t* numel;          // [2P]: unpadded numel, then padded numel
    int32_t n_params;
    int32_t* err;
};

// GATHER: the source of rank r's chunk is rank r's own shard (shard_tab[r], of
// which the chunk starts at off_i), not row r of one rank-major buffer; the
// shards may live in other processes' or GPUs' memory (peer pointers).
template <bool GATHER>
__global__ void __launch_bounds__(kThreads) ag_place_kernel(const AgParams a) {
    __shared__ tide_tile_t s_tile;
    for (int64_t t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
        __syncthreads();
        if (threadIdx.x == 0) s_tile = a.tiles[t];
        __syncthreads();
        const tide_tile_t tl = s_tile;
        const bool param_ok = tl.param >= 0 && tl.param < a.n_params;
        // offset of the tile's first element in its source buffer
        const int64_t src = GATHER ? tl.dst_off - (int64_t)tl.rank * a.shard_numel : tl.dst_off;
        const bool ok = param_ok && tl.n_valid >= 0 && tl.n_valid <= tl.n_total &&
                        tl.src_off >= 0 && tl.src_off + tl.n_total <= a.numel[a.n_params + tl.param] &&
                        (!GATHER || (tl.rank >= 0 && tl.rank < a.world)) &&
                        src >= 0 && src + tl.n_valid <= a.ag_numel;
        if (!ok) {
            if (threadIdx.x == 0) atomicOr(a.err, TIDE_KCHECK_TILE);
            continue;
        }
        const uint16_t* from = GATHER ? static_cast<const uint16_t*>(a.shard_tab[tl.rank]) + src : a.ag + src;
        uint16_t* dst = static_cast<uint16_t*>(const_cast<void*>(a.param_tab[tl.param])) + tl.src_off;
        block_copy_bf16_v32<kCopyU, kThreads>(from, dst, tl.n_valid);
        if (tl.n_total > tl.n_valid) block_zero_bf16<kThreads>(dst + tl.n_valid, tl.n_total - tl.n_valid);
    }
}

struct StageParams {
    const tide_tile_t* tiles;
    int64_t n_tiles;
    const void* const* grad_tab;  // [world*P], k*P + i
    const void* const* slot_tab;  // [world]
    const int64_t* numel;         // [P] unpadded numel
    int64_t slot_numel;
    int32_t world;                // source ranks in the tables: W, or 1 for one rank's gradients
    int32_t n_params;
    int32_t* err;
};

__global__ void __launch_bounds__(kThreads) slot_stage_kernel(const StageParams a) {
    __shared__ tide_tile_t s_tile;
    const int64_t units = a.n_tiles * a.world;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t t = u / a.world;
        const int k = (int)(u - t * a.world);
        __syncthreads();
        if (threadIdx.x == 0) s_tile = a.tiles[t];
        __syncthreads();
        const tide_tile_t tl = s_tile;
        const bool param_ok = tl.param >= 0 && tl.param < a.n_params;
        // (an all-pad tile copies nothing; its gradient offset may lie past the tensor)
        const bool ok = param_ok && tl.n_valid >= 0 && tl.n_valid <= tl.n_total &&
                        (tl.n_valid == 0 ||
                         (tl.src_off >= 0 && tl.src_off + tl.n_valid <= a.numel[tl.param] &&
                          tl.dst_off >= 0 && tl.dst_off + tl.n_valid <= a.slot_numel));
        if (!ok) {
            if (threadIdx.x == 0) atomicOr(a.err, TIDE_KCHECK_TILE);
            continue;
        }
        if (tl.n_valid == 0) continue;
        const uint16_t* src =
            static_cast<const uint16_t*>(a.grad_tab[(int64_t)k * a.n_params + tl.param]) + tl.src_off;
        uint16_t* dst = static_cast<uint16_t*>(const_cast<void*>(a.slot_tab[k])) + tl.dst_off;
        block_copy_bf16_v32<kCopyU, kThreads>(src, dst, tl.n_valid);
    }
}

}  // namespace

int ag_blocks_per_sm(bool gather) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, gather ? ag_place_kernel<true> : ag_place_kernel<false>, kThreads, 0) != cudaSuccess)
        return 0;
    return n;
}

int stage_blocks_per_sm() {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, slot_stage_kernel, kThreads, 0) != cudaSuccess)
        return 0;
    return n;
}

cudaError_t launch_ag_place(const tide_plan* p, const uint16_t* ag, int64_t ag_numel,
                            const void* const* d_param_tab, int grid, cudaStream_t stream) {
    if (p->tiles.empty() || grid <= 0) return cudaSuccess;
    AgParams a;
    a.tiles = p->d_tiles;
    a.n_tiles = (int64_t)p->tiles.size();
    a.ag = ag;
    a.ag_numel = ag_numel;
    a.shard_tab = nullptr;
    a.shard_numel = p->shard_numel;
    a.world = p->world;
    a.param_tab = d_param_tab;
    a.numel = p->d_numel;
    a.n_params = p->n_params;
    a.err = p->d_err;
    (void)cudaGetLastError();  // drop an error left by an earlier failed runtime call
    ag_place_kernel<false><<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_ag_gather(const tide_plan* p, const void* const* d_shard_tab, int64_t shard_numel,
                             const void* const* d_param_tab, int grid, cudaStream_t stream) {
    if (p->tiles.empty() || grid <= 0) return cudaSuccess;
    AgParams a;
    a.tiles = p->d_tiles;
    a.n_tiles = (int64_t)p->tiles.size();
    a.ag = nullptr;
    a.ag_numel = shard_numel;
    a.shard_tab = d_shard_tab;
    a.shard_numel = p->shard_numel;
    a.world = p->world;
    a.param_tab = d_param_tab;
    a.numel = p->d_numel;
    a.n_params = p->n_params;
    a.err = p->d_err;
    (void)cudaGetLastError();  // drop an error left by an earlier failed runtime call
    ag_place_kernel<true><<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_slot_stage(const tide_plan* p, const void* const* d_grad_tab,
                              const void* const* d_slot_tab, int64_t slot_numel, int grid,
                              cudaStream_t stream, int32_t sources) {
    if (p->tiles.empty() || grid <= 0) return cudaSuccess;
    StageParams a;
    a.tiles = p->d_tiles;
    a.n_tiles = (int64_t)p->tiles.size();
    a.grad_tab = d_grad_tab;
    a.slot_tab = d_slot_tab;
    a.numel = p->d_numel;
    a.slot_numel = slot_numel;
    a.world = sources;  // the kernel's source ranks: its units are (tile, source) pairs
    a.n_params = p->n_params;
    a.err = p->d_err;
    (void)cudaGetLastError();  // drop an error left by an earlier failed runtime call
    slot_stage_kernel<<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace tide
