// f32_grads.cu - Slot-Reuse staging and reduction of fp32 gradients (sm_100a).
//
// While gradient sync is off, FSDP2 keeps a parameter's gradients in its fp32
// reduce dtype across micro-batches and packs those fp32 gradients at the next
// synced backward.  The layout-aware reduction applies to them as to bf16 ones
// ("The Endgame of FSDP Communication", weekinpapers.com, Abstract: gradients
// read where they lie, reduced into fp32 shards; the Slot-Reuse option of the
// two-phase pipeline): the same tiles, the same rank-order fp32 sum and scale,
// the same pads, only without the bf16 widening and with 4-byte slot words.
//   stage:  slot[r*Ns + off_i + e] = g_i[r*c_i + e] for valid e (one source
//           rank, every row of its slot; slot pads are not written);
//   reduce: out[j] = s * fl32(sum_{k=0..W-1} slot_k[row0 + j]) from slot_0 in
//           rank order, +0.0 at pads (row0 = rank*Ns for a one-rank plan,
//           applied by the host to the slot pointers);
//   direct: out[r*Ns + off_i + e] = s * fl32(sum_k g_{k,i}[r*c_i + e]), TIDE-RS
//           itself on fp32 gradients read where they lie (no slot).
// Both are HBM-bound (stage: 4 + 4 bytes per element; reduce: 4W + 4).  CTAs
// walk the plan's tiles round-robin.  Each thread keeps four 32-byte vectors in
// flight: the staging loads four before storing them, the reduction issues one
// rank's four loads before adding them.  A tile that is not 32-byte aligned
// takes 16-byte vectors or the element loop (coalesced 4-byte accesses).
#include "device_common.cuh"
#include "tide_internal.h"

namespace tide {
namespace {

constexpr int kVecU = 4;   // 32-byte vectors per thread per step of the reduction
constexpr int kCopyU = 4;  // 32-byte vectors in flight per thread in the staging copy

struct StageF32Params {
    const tide_tile_t* tiles;
    int64_t n_tiles;
    const void* const* grad_tab;  // [P] the one source rank's fp32 gradients
    void* slot;                   // fp32 [W][Ns]
    const int64_t* numel;         // [P] unpadded numel
    int64_t slot_numel;
    int32_t n_params;
    int32_t* err;
};

struct ReduceF32Params {
    const tide_tile_t* tiles;
    int64_t n_tiles;
    const void* const* slot_tab;  // [W] fp32 slots, already advanced to the plan's first row
    int64_t src_bound;            // elements readable from each of those pointers
    const void* const* grad_tab;  // direct: [W*P] fp32 gradients, k*P + i
    const int64_t* numel;         // direct: [P] unpadded numel
    int32_t n_params;
    float* out;
    int64_t out_numel;
    int32_t world;
    float scale;
    int32_t do_scale;
    int32_t v8;                   // every slot and out 32-byte aligned
    int32_t* err;
};

// Block-wide copy of n 4-byte words.  When source and destination share their
// offset modulo 32 (or 16) bytes, a scalar head aligns both and the body moves
// 32-byte (16-byte) vectors; otherwise every word is moved on its own.
__device__ __forceinline__ void block_copy_words(const uint32_t* __restrict__ src,
                                                 uint32_t* __restrict__ dst, int64_t n) {
    const uintptr_t sa = reinterpret_cast<uintptr_t>(src), da = reinterpret_cast<uintptr_t>(dst);
    const int vbytes = ((sa ^ da) & 31) == 0 ? 32 : ((sa ^ da) & 15) == 0 ? 16 : 4;
    int64_t head = 0;
    if (vbytes > 4) {
        head = (int64_t)(((vbytes - (int)(da & (vbytes - 1))) & (vbytes - 1)) >> 2);
        if (head > n) head = n;
    }
    for (int64_t e = threadIdx.x; e < head; e += kThreads) dst[e] = src[e];
    int64_t done = head;
    if (vbytes == 32) {
        // kCopyU vectors per thread per step, all loaded before the first is stored
        const int64_t nv = (n - head) >> 3;
        for (int64_t v0 = threadIdx.x; v0 < nv; v0 += (int64_t)kThreads * kCopyU) {
            V8 x[kCopyU];
#pragma unroll
            for (int u = 0; u < kCopyU; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nv) x[u] = ld_stream_v8(src + head + 8 * v);
            }
#pragma unroll
            for (int u = 0; u < kCopyU; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nv) st_stream_v8(dst + head + 8 * v, x[u]);
            }
        }
        done = head + 8 * nv;
    } else if (vbytes == 16) {
        const int64_t nv = (n - head) >> 2;
        for (int64_t v = threadIdx.x; v < nv; v += kThreads)
            st_stream_v4(dst + head + 4 * v, ld_stream_v4(src + head + 4 * v));
        done = head + 4 * nv;
    }
    for (int64_t e = done + threadIdx.x; e < n; e += kThreads) dst[e] = src[e];
}

// Every thread reads the tile descriptors itself (the same 32 bytes for the whole CTA, one
// broadcast load per warp) and has the next one in flight while it copies the current
// tile, so no barrier stands between tiles.  (With a descriptor in shared memory the
// barriers around it were a third of the stalls on the sweep W=8 group; without them the
// throughput barely moved, 6.06 -> 6.10 TB/s on the 70B group.)
__global__ void __launch_bounds__(kThreads) stage_f32_kernel(const StageF32Params a) {
    if ((int64_t)blockIdx.x >= a.n_tiles) return;
    tide_tile_t next = a.tiles[blockIdx.x];
    for (int64_t t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
        const tide_tile_t tl = next;
        if (t + gridDim.x < a.n_tiles) next = a.tiles[t + gridDim.x];
        // (an all-pad tile copies nothing; its gradient offset may lie past the tensor)
        const bool ok = tl.param >= 0 && tl.param < a.n_params && tl.n_valid >= 0 &&
                        tl.n_valid <= tl.n_total &&
                        (tl.n_valid == 0 ||
                         (tl.src_off >= 0 && tl.src_off + tl.n_valid <= a.numel[tl.param] &&
                          tl.dst_off >= 0 && tl.dst_off + tl.n_valid <= a.slot_numel));
        if (!ok) {
            if (threadIdx.x == 0) atomicOr(a.err, TIDE_KCHECK_TILE);
            continue;
        }
        if (tl.n_valid == 0) continue;
        // (block_copy_words has no barrier: each thread moves its own words)
        const uint32_t* src = static_cast<const uint32_t*>(a.grad_tab[tl.param]) + tl.src_off;
        uint32_t* dst = static_cast<uint32_t*>(a.slot) + tl.dst_off;
        block_copy_words(src, dst, tl.n_valid);
    }
}

__device__ __forceinline__ void add8(float (&acc)[8], const V8& v) {
#pragma unroll
    for (int l = 0; l < 8; ++l) acc[l] = __fadd_rn(acc[l], __uint_as_float(v.w[l]));
}

// SLOT: the sources are the W slots, read at the output position (tile dst_off).
// Otherwise (direct): the sources are the W ranks' gradients of the tile's param,
// read at the tile's src_off, with no staging at all; their pointers are put in
// shared memory tile by tile.  s_src[k] + src0 is rank k's first element of the tile.
template <bool SLOT>
__global__ void __launch_bounds__(kThreads) reduce_f32_kernel(const ReduceF32Params a) {
    __shared__ const float* s_src[TIDE_MAX_WORLD];
    __shared__ tide_tile_t s_tile;
    const int W = a.world;
    if (SLOT)
        for (int k = threadIdx.x; k < W; k += kThreads) s_src[k] = static_cast<const float*>(a.slot_tab[k]);
    for (int64_t t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
        __syncthreads();
        if (threadIdx.x == 0) s_tile = a.tiles[t];
        __syncthreads();
        const tide_tile_t tl = s_tile;
        const int64_t base = tl.dst_off;
        bool ok = tl.n_valid >= 0 && tl.n_valid <= tl.n_total && base >= 0 && base + tl.n_total <= a.out_numel;
        if (SLOT)
            ok = ok && base + tl.n_valid <= a.src_bound;
        else
            ok = ok && tl.param >= 0 && tl.param < a.n_params &&
                 (tl.n_valid == 0 || (tl.src_off >= 0 && tl.src_off + tl.n_valid <= a.numel[tl.param]));
        if (!ok) {
            if (threadIdx.x == 0) atomicOr(a.err, TIDE_KCHECK_TILE);
            continue;
        }
        const int64_t src0 = SLOT ? base : tl.src_off;
        if (!SLOT) {
            // (every thread has finished the previous tile: the barriers above lie between)
            for (int k = threadIdx.x; k < W; k += kThreads)
                s_src[k] = static_cast<const float*>(a.grad_tab[(int64_t)k * a.n_params + tl.param]);
            __syncthreads();
        }
        // whole 32-byte vectors of valid elements, then the element loop for the rest
        const int64_t nv = (a.v8 && ((base | src0) & 7) == 0) ? (tl.n_valid >> 3) : 0;
        for (int64_t v0 = threadIdx.x; v0 < nv; v0 += (int64_t)kThreads * kVecU) {
            float acc[kVecU][8];
#pragma unroll
            for (int u = 0; u < kVecU; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nv) {
                    const V8 x = ld_stream_v8(s_src[0] + src0 + 8 * v);
#pragma unroll
                    for (int l = 0; l < 8; ++l) acc[u][l] = __uint_as_float(x.w[l]);
                }
            }
            for (int k = 1; k < W; ++k) {
                V8 x[kVecU];
#pragma unroll
                for (int u = 0; u < kVecU; ++u) {
                    const int64_t v = v0 + (int64_t)u * kThreads;
                    if (v < nv) x[u] = ld_stream_v8(s_src[k] + src0 + 8 * v);
                }
#pragma unroll
                for (int u = 0; u < kVecU; ++u)
                    if (v0 + (int64_t)u * kThreads < nv) add8(acc[u], x[u]);
            }
#pragma unroll
            for (int u = 0; u < kVecU; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nv) {
                    if (a.do_scale) {
#pragma unroll
                        for (int l = 0; l < 8; ++l) acc[u][l] = __fmul_rn(acc[u][l], a.scale);
                    }
                    st_stream_f8(a.out + base + 8 * v, acc[u]);
                }
            }
        }
        for (int64_t e = 8 * nv + threadIdx.x; e < tl.n_total; e += kThreads) {
            float r = 0.0f;
            if (e < tl.n_valid) {
                r = s_src[0][src0 + e];
                for (int k = 1; k < W; ++k) r = __fadd_rn(r, s_src[k][src0 + e]);
                if (a.do_scale) r = __fmul_rn(r, a.scale);
            }
            a.out[base + e] = r;
        }
    }
}

}  // namespace

int stage_f32_blocks_per_sm() {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, stage_f32_kernel, kThreads, 0) != cudaSuccess)
        return 0;
    return n;
}

int reduce_f32_blocks_per_sm(bool slot) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, slot ? reduce_f32_kernel<true> : reduce_f32_kernel<false>, kThreads, 0) != cudaSuccess)
        return 0;
    return n;
}

cudaError_t launch_stage_f32(const tide_plan* p, const void* const* d_grad_tab, void* slot,
                             int64_t slot_numel, int grid, cudaStream_t stream) {
    if (p->tiles.empty() || grid <= 0) return cudaSuccess;
    StageF32Params a;
    a.tiles = p->d_tiles;
    a.n_tiles = (int64_t)p->tiles.size();
    a.grad_tab = d_grad_tab;
    a.slot = slot;
    a.numel = p->d_numel;
    a.slot_numel = slot_numel;
    a.n_params = p->n_params;
    a.err = p->d_err;
    (void)cudaGetLastError();  // drop an error left by an earlier failed runtime call
    stage_f32_kernel<<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_reduce_slots_f32(const tide_plan* p, const void* const* d_slot_tab, int64_t src_bound,
                                    float* out, int64_t out_numel, float scale, bool do_scale, bool v8,
                                    int grid, cudaStream_t stream) {
    if (p->tiles.empty() || grid <= 0) return cudaSuccess;
    ReduceF32Params a;
    a.tiles = p->d_tiles;
    a.n_tiles = (int64_t)p->tiles.size();
    a.slot_tab = d_slot_tab;
    a.src_bound = src_bound;
    a.out = out;
    a.out_numel = out_numel;
    a.world = p->world;
    a.scale = scale;
    a.do_scale = do_scale ? 1 : 0;
    a.v8 = v8 ? 1 : 0;
    a.err = p->d_err;
    a.grad_tab = nullptr;
    a.numel = nullptr;
    a.n_params = p->n_params;
    (void)cudaGetLastError();
    reduce_f32_kernel<true><<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_reduce_f32(const tide_plan* p, const void* const* d_grad_tab, float* out,
                              int64_t out_numel, float scale, bool do_scale, bool v8, int grid,
                              cudaStream_t stream) {
    if (p->tiles.empty() || grid <= 0) return cudaSuccess;
    ReduceF32Params a;
    a.tiles = p->d_tiles;
    a.n_tiles = (int64_t)p->tiles.size();
    a.slot_tab = nullptr;
    a.src_bound = 0;
    a.grad_tab = d_grad_tab;
    a.numel = p->d_numel;
    a.n_params = p->n_params;
    a.out = out;
    a.out_numel = out_numel;
    a.world = p->world;
    a.scale = scale;
    a.do_scale = do_scale ? 1 : 0;
    a.v8 = v8 ? 1 : 0;
    a.err = p->d_err;
    (void)cudaGetLastError();
    reduce_f32_kernel<false><<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace tide
