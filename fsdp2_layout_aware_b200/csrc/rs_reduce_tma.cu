// rs_reduce_tma.cu - TIDE-RS reduction with bulk-copy (TMA) staging, sm_100a.
//
// Same result as rs_reduce_kernel (rank order: bit-identical; tree order: the
// same tree), for groups whose chunks start on 8-element boundaries and whose
// buffers are 16-byte aligned; used when the plan asks for it (TIDE_PLAN_TMA).
// The difference is how the bytes move: one producer warp streams every rank's
// piece of the current tile into shared memory with cp.async.bulk (the copy
// engine inside each SM), kStages pieces ahead, and eight consumer warps reduce
// from shared memory and write the fp32 shard with 16-byte streaming stores.
// A piece holds `sub` elements of each of the W ranks (sub * W * 2 bytes = one
// 64 KB stage), so a CTA keeps up to kStages * 64 KB of loads in flight without
// spending registers or threads on them.  One persistent CTA per SM walks the
// plan's tile list round-robin.
//
// Measured on B200 against the load/store kernel (same workloads, whole grid):
// 6.76 vs 6.82 TB/s on the Llama-3.1-70B group (W=8), 6.52 vs 6.86 on Wan2.2
// (W=16), 2.8 vs 7.0 on W=64 (pieces of 256 B per rank are too small), so the
// load/store kernel is the default.  What this kernel offers is bandwidth per
// CTA: with a handful of CTAs (the short-lived accumulation CTAs of the TIDE
// design) each SM moves far more than a load/store CTA can.
//
// Synchronisation: per stage a `full` mbarrier (one producer arrival plus the
// bulk-copy transaction bytes) and an `empty` mbarrier (one arrival per
// consumer warp).  Every wait is bounded (tma.cuh); on a timeout the CTA sets
// the plan's error word, stops, waits (bounded) for its own copies still in
// flight, and returns.
#include "device_common.cuh"
#include "reduce_ranks.cuh"
#include "tide_internal.h"
#include "tma.cuh"

namespace tide {
namespace {

#ifndef TIDE_TMA_STAGES
#define TIDE_TMA_STAGES 3
#endif
#ifndef TIDE_TMA_STAGE_KB
#define TIDE_TMA_STAGE_KB 64
#endif

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kTmaThreads = 32 + kConsumers;
constexpr int kStages = TIDE_TMA_STAGES;
constexpr int kStageBytes = TIDE_TMA_STAGE_KB * 1024;
constexpr int kPtrsPerLane = TIDE_MAX_WORLD / 32;  // producer lane k keeps ranks k, k+32, ...

struct StageHdr {
    int64_t dst_off;  // output offset of the piece
    int32_t n_piece;  // elements in the piece (valid + pad)
    int32_t n_valid;  // leading valid elements
    int32_t n_bulk;   // leading valid elements delivered to shared memory (multiple of 8)
    int32_t unused;
};

struct TmaParams {
    const tide_tile_t* tiles;
    int64_t n_tiles;
    const void* const* src_tab;  // plain: [W*P] grads (k*P + i); slot mode: [W] slots
    const int64_t* numel;        // [P] unpadded numel
    int64_t slot_numel;
    float* out;
    int64_t out_numel;
    int32_t world;
    int32_t n_params;
    int32_t sub;                 // elements per rank per stage (multiple of 8)
    float scale;
    int32_t do_scale;
    int32_t withhold;            // test hook: CTA 0 withholds its first stage (its wait then runs out)
    int32_t* err;
};

__device__ __forceinline__ bool tile_ok(const TmaParams& a, const tide_tile_t& tl, bool slot) {
    const bool param_ok = tl.param >= 0 && tl.param < a.n_params;
    const int64_t src_off = slot ? tl.dst_off : tl.src_off;
    const int64_t src_lim = slot ? a.slot_numel : (param_ok ? a.numel[tl.param] : -1);
    return param_ok && tl.n_valid >= 0 && tl.n_valid <= tl.n_total && tl.n_total >= 0 &&
           tl.dst_off >= 0 && tl.dst_off + tl.n_total <= a.out_numel &&
           (tl.n_valid == 0 || (src_off >= 0 && src_off + tl.n_valid <= src_lim));
}

template <bool SLOT, bool TREE>
__global__ void __launch_bounds__(kTmaThreads, 1) rs_reduce_tma_kernel(const TmaParams a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ volatile int s_abort;
    const int W = a.world, sub = a.sub;
    uint16_t* data = reinterpret_cast<uint16_t*>(smem);
    StageHdr* hdr = reinterpret_cast<StageHdr*>(smem + (size_t)kStages * W * sub * 2);
    const uint16_t** srcs = reinterpret_cast<const uint16_t**>(hdr + kStages);  // [kStages][W]
    uint64_t* full = reinterpret_cast<uint64_t*>(srcs + kStages * W);
    uint64_t* empty = full + kStages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        mbar_init_fence();
        s_abort = 0;
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        int stage = 0;
        uint32_t phase = 0;
        uint32_t pending = 0;     // stages whose last issue carried bulk bytes
        uint32_t pend_par = 0;    // parity of that issue, per stage bit
        bool aborted = false;
        bool withhold = a.withhold != 0 && blockIdx.x == 0;  // warp-uniform
        int64_t t = blockIdx.x;
        tide_tile_t next = t < a.n_tiles ? a.tiles[t] : tide_tile_t{};
        for (; t < a.n_tiles && !aborted; t += gridDim.x) {
            const tide_tile_t tl = next;
            if (t + gridDim.x < a.n_tiles) next = a.tiles[t + gridDim.x];  // in flight meanwhile
            if (!tile_ok(a, tl, SLOT)) {
                if (lane == 0) atomicOr(a.err, TIDE_KCHECK_TILE);
                continue;
            }
            // this tile's source pointers: lane keeps ranks lane, lane+32, ...
            const int64_t src_off = SLOT ? tl.dst_off : tl.src_off;
            const uint16_t* base[kPtrsPerLane];
            bool aligned = true;
#pragma unroll
            for (int j = 0; j < kPtrsPerLane; ++j) {
                const int k = lane + 32 * j;
                base[j] = nullptr;
                if (k < W) {
                    base[j] = static_cast<const uint16_t*>(
                                  a.src_tab[SLOT ? k : (int64_t)k * a.n_params + tl.param]) + src_off;
                    aligned &= (reinterpret_cast<uintptr_t>(base[j]) & 15) == 0;
                }
            }
            // piece starts advance by sub (a multiple of 8 elements = 16 bytes)
            aligned = __all_sync(0xffffffffu, aligned) &&
                      (reinterpret_cast<uintptr_t>(a.out + tl.dst_off) & 15) == 0;
            for (int e0 = 0; e0 < tl.n_total; e0 += sub) {
                const int n_piece = min(sub, tl.n_total - e0);
                const int n_val = max(0, min(n_piece, tl.n_valid - e0));
                const int n_bulk = aligned ? (n_val & ~7) : 0;
                // the whole warp takes the same branch (a lane that gave up aborts all)
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[stage], phase ^ 1, &s_abort))) {
                    aborted = true;
                    break;
                }
#pragma unroll
                for (int j = 0; j < kPtrsPerLane; ++j) {
                    const int k = lane + 32 * j;
                    if (k < W) srcs[stage * W + k] = base[j] + e0;
                }
                if (lane == 0) {
                    StageHdr h;
                    h.dst_off = tl.dst_off + e0;
                    h.n_piece = n_piece;
                    h.n_valid = n_val;
                    h.n_bulk = n_bulk;
                    h.unused = 0;
                    hdr[stage] = h;
                }
                __syncwarp();
                if (lane == 0 && !withhold) {
                    if (n_bulk > 0) mbar_arrive_expect_tx(&full[stage], (uint32_t)(W * n_bulk * 2));
                    else mbar_arrive(&full[stage]);
                }
                __syncwarp();
                if (n_bulk > 0 && !withhold) {
#pragma unroll
                    for (int j = 0; j < kPtrsPerLane; ++j) {
                        const int k = lane + 32 * j;
                        if (k < W)
                            bulk_g2s(data + ((size_t)stage * W + k) * sub, base[j] + e0,
                                     (uint32_t)(n_bulk * 2), &full[stage]);
                    }
                    pending |= 1u << stage;
                    pend_par = (pend_par & ~(1u << stage)) | (phase << stage);
                } else {
                    pending &= ~(1u << stage);
                }
                withhold = false;
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        if (aborted && lane == 0) {
            atomicOr(a.err, TIDE_KCHECK_TIMEOUT);
            s_abort = 1;
        }
        // Before the CTA exits, every bulk copy it issued must have landed.
        for (int s = 0; s < kStages; ++s) {
            if ((pending >> s) & 1) {
                if (!mbar_wait(&full[s], (pend_par >> s) & 1, nullptr) && lane == 0)
                    atomicOr(a.err, TIDE_KCHECK_TIMEOUT);
            }
        }
    } else {
        // ---------------------------------------------------------------- consumers
        const int ctid = threadIdx.x - 32;
        int stage = 0;
        uint32_t phase = 0;
        bool aborted = false;
        for (int64_t t = blockIdx.x; t < a.n_tiles && !aborted; t += gridDim.x) {
            const tide_tile_t tl = a.tiles[t];
            if (!tile_ok(a, tl, SLOT)) continue;
            for (int e0 = 0; e0 < tl.n_total; e0 += sub) {
                if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, &s_abort))) {
                    aborted = true;
                    break;
                }
                const StageHdr h = hdr[stage];
                float* __restrict__ dst = a.out + h.dst_off;
                const uint16_t* sbase = data + (size_t)stage * W * sub;
                const uint16_t* const* psrc = srcs + stage * W;
                const int nv = h.n_bulk >> 3;
                for (int v = ctid; v < nv; v += kConsumers) {
                    float acc[8];
                    auto load = [&](int k) {
                        return *reinterpret_cast<const uint4*>(sbase + (size_t)k * sub + 8 * v);
                    };
                    if (TREE && W <= 8) tree_one_group<8, 8, uint4>(W, load, acc);
                    else reduce_ranks<8, 8, TREE, uint4>(W, load, acc);
                    if (a.do_scale) {
#pragma unroll
                        for (int l = 0; l < 8; ++l) acc[l] = __fmul_rn(acc[l], a.scale);
                    }
                    float* o = dst + 8 * v;
                    st_stream_f4(o, acc[0], acc[1], acc[2], acc[3]);
                    st_stream_f4(o + 4, acc[4], acc[5], acc[6], acc[7]);
                }
                for (int e = h.n_bulk + ctid; e < h.n_valid; e += kConsumers) {
                    float acc[1];
                    auto load = [&](int k) { return (uint32_t)ld_stream_u16(psrc[k] + e); };
                    if (TREE && W <= 8) tree_one_group<8, 1, uint32_t>(W, load, acc);
                    else reduce_ranks<8, 1, TREE, uint32_t>(W, load, acc);
                    if (a.do_scale) acc[0] = __fmul_rn(acc[0], a.scale);
                    dst[e] = acc[0];
                }
                for (int e = h.n_valid + ctid; e < h.n_piece; e += kConsumers) dst[e] = 0.0f;
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        if (aborted && lane == 0) {
            atomicOr(a.err, TIDE_KCHECK_TIMEOUT);
            s_abort = 1;
        }
    }
    __syncthreads();
}

using TmaKernelFn = void (*)(const TmaParams);

TmaKernelFn select_tma(bool slot, int order) {
    const bool tree = order == TIDE_ORDER_TREE;
    if (slot) return tree ? rs_reduce_tma_kernel<true, true> : rs_reduce_tma_kernel<true, false>;
    return tree ? rs_reduce_tma_kernel<false, true> : rs_reduce_tma_kernel<false, false>;
}

int sub_for(int world) {
    int sub = (kStageBytes / (2 * world)) & ~7;
    return sub > TIDE_TILE_ELEMS ? TIDE_TILE_ELEMS : sub;
}

size_t smem_for(int world) {
    return (size_t)kStages * world * sub_for(world) * 2 + kStages * sizeof(StageHdr) +
           (size_t)kStages * world * sizeof(void*) + 2 * kStages * sizeof(uint64_t);
}

// The largest dynamic shared memory any world size needs: the kernels are
// opted in to this once, so plans of different world sizes can coexist.
size_t smem_max() {
    size_t m = 0;
    for (int w = 1; w <= TIDE_MAX_WORLD; ++w) m = smem_for(w) > m ? smem_for(w) : m;
    return m;
}

}  // namespace

// Opt in to the dynamic shared memory the TMA kernels need for this world size
// and return their resident CTAs per SM (0 if they cannot run).
int rs_tma_blocks_per_sm(int world) {
    const size_t smem = smem_for(world);
    int n = 0;
    for (bool slot : {false, true})
        for (int order : {TIDE_ORDER_RANK, TIDE_ORDER_TREE}) {
            if (cudaFuncSetAttribute(select_tma(slot, order), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem_max()) != cudaSuccess)
                return 0;
        }
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, select_tma(false, TIDE_ORDER_RANK), kTmaThreads,
                                                      smem) != cudaSuccess)
        return 0;
    return n;
}

cudaError_t launch_rs_reduce_tma(const tide_plan* p, const void* const* d_src_tab, bool slot,
                                 int64_t src_bound, float* out, int64_t out_numel, float scale,
                                 bool do_scale, int order, int grid, cudaStream_t stream, int64_t t0,
                                 int64_t t1) {
    if (t1 < 0) t1 = (int64_t)p->tiles.size();
    if (t1 <= t0 || grid <= 0) return cudaSuccess;
    TmaParams a;
    a.tiles = p->d_tiles + t0;
    a.n_tiles = t1 - t0;
    a.src_tab = d_src_tab;
    a.numel = p->d_numel;
    a.slot_numel = src_bound;
    a.out = out;
    a.out_numel = out_numel;
    a.world = p->world;
    a.n_params = p->n_params;
    a.sub = sub_for(p->world);
    a.scale = scale;
    a.do_scale = do_scale ? 1 : 0;
    a.withhold = (p->flags & TIDE_PLAN_TEST_TMA_TIMEOUT) ? 1 : 0;
    a.err = p->d_err;
    (void)cudaGetLastError();  // drop an error left by an earlier failed runtime call
    select_tma(slot, order)<<<grid, kTmaThreads, smem_for(p->world), stream>>>(a);
    return cudaGetLastError();
}

}  // namespace tide
