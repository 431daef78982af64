// rs_reduce.cu - TIDE-RS reduction kernel for sm_100a.
//
// Method: "The Endgame of FSDP Communication" (weekinpapers.com, Abstract,
// TIDE-RS): per-parameter bf16 gradients are consumed where they lie and
// reduced into fp32 shards, with no fp32 packing buffer in between.  Here the
// W ranks are W sets of buffers on this GPU; one launch produces every rank's
// fp32 shard:
//   out[r*Ns + off_i + e] = s * fl32(sum_{k=0..W-1} fp32(g_{k,i}[r*c_i + e]))
// and +0.0 at pad positions.  In Slot-Reuse mode the sources are the W staged
// slots in the all-gather layout, read at the output position itself.
//
// Design (HBM-bound: W*2 bytes read and 4 bytes written per output element,
// ~(W-1)/(2W+4) flop/byte, so no tensor cores):
//   - a persistent grid, at most max_ctas CTAs, walks the plan's tile list
//     round-robin, or on long launches claims tiles from a counter as CTAs
//     finish them; a tile is a piece of one (param, rank) chunk of up to
//     TIDE_TILE_ELEMS elements, so tiny MoE chunks and huge dense chunks mix;
//   - per tile the W source addresses are staged in shared memory once (one
//     barrier per tile; the next tile's descriptor is already in registers);
//   - each thread owns 8 consecutive outputs per step: W independent 16-byte
//     streaming loads (in groups of G ranks to bound registers), an fp32 sum
//     with __fadd_rn (no contraction), the optional __fmul_rn scale, two 16-byte
//     streaming stores; for W = 2 or W >= 5 and 32-byte aligned groups, 16
//     outputs per step with 32-byte loads and stores instead;
//   - tiles whose addresses are not all 16-byte aligned (possible only when
//     the group's sizes break alignment) fall back to coalesced scalar loads;
//   - ragged tile ends and pad rows are finished element by element.
// Rank order (ORDER_RANK) adds g_0 + g_1 + ... exactly as the stock
// pack-then-reduce does, so the result is bit-identical to it.  Tree order
// adds adjacent ranks pairwise inside each group of G and merges group sums
// with a binary counter (a pairwise tree over groups).
#include "device_common.cuh"
#include "reduce_ranks.cuh"
#include "tide_internal.h"


namespace tide {
namespace {

// The 32-byte path measured faster for W >= 5 (70B W=8: 7.03 vs 6.89 TB/s;
// Qwen3 W=8: 7.08 vs 6.87; Wan2.2 W=16: 6.93 vs 6.90; the sweep's W = 32 and 64
// groups: 6.90 vs 6.68 and 6.85 vs 6.71; 16 x 1536x4096 at W = 24: 6.88 vs
// 6.54; 16 x 1024x4096 at W = 128: 6.89 vs 6.65).  At W = 2 it beats the
// 16-byte two-rank kernel by 20-27 % (67 MB to 1.1 GB groups: 3.41 vs 2.73,
// 5.02 vs 3.95, 5.31 vs 4.45 TB/s), and its two-rank form at 4 CTAs per SM
// beats its eight-rank form by 6-24 % (the sweep's 67 MB group: 4.17 vs 3.43;
// 134 MB: 6.24 vs 5.03; 1 GB: 5.79 vs 5.45).  At W = 3 and 4 neither form wins
// on the large groups (1 GB: 6.12 vs 6.24 and 6.12 vs 6.39 for the four-rank
// form), so they keep 16-byte loads.  Its registers do not grow with W: the
// ranks are loaded 8 at a time and added in order.
constexpr int kV32MaxWorld = TIDE_MAX_WORLD;

struct RsParams {
    const tide_tile_t* tiles;
    int64_t n_tiles;
    const void* const* src_tab;  // plain: [W*P] grads, index k*P + i; slot mode: [W] slots
    const int64_t* numel;        // [P] unpadded numel (plain-mode source bound)
    int64_t slot_numel;          // slot-mode source bound
    float* out;
    int64_t out_numel;
    int32_t world;
    int32_t n_params;
    float scale;
    int32_t do_scale;
    int32_t* err;
    // dynamic != 0: after its first tile (blockIdx.x) each CTA claims the next unclaimed
    // tile from counter[0]; counter[1] counts finished CTAs.  Both are zero at launch.
    int32_t dynamic;
    unsigned long long* counter;
};

// V32: 32-byte loads and stores (16 outputs per thread per step); the host
// picks it only when every tile's sources and output are 32-byte aligned
// (a tile that is not falls back to the element loop, never faults).
// NG selects how the tree order is formed (rank order ignores it):
//   NG = -1: W <= G at run time, one group (tree_one_group), no merge stack;
//   NG =  0: any W at run time, groups of G merged through reduce_ranks' stack;
//   NG >= 1: W = NG * G exactly, the whole tree fixed at compile time
//            (tree_groups): no merge stack and no run-time W.
// The 32-byte tree kernels are NG = 1 and 2 (W = 8, 16).  A first 32-byte
// version kept W at run time; up to 8 ranks' unpacked lanes then stayed live
// and spilled (276 and 708 bytes) at the 128 registers of 2 CTAs per SM.
// The 16-byte NG = 4 (W = 32) kernel keeps 2 CTAs per SM by loading one group
// at a time; NG = 8 (W = 64) spilled 300-320 bytes that way and runs at one
// CTA per SM instead (153 registers, no spill): 6.74 TB/s against 6.18 for the
// merge-stack kernel on the sweep's W = 64 group.
// The 16-byte NG = -1 kernels are held to 3 CTAs per SM (80 registers, a
// spill of 88 bytes per thread at G = 8): left free they take 128 registers
// and 2 CTAs per SM, 4 % slower on B200 (70B W=8: 6.52 vs 6.28 TB/s; Qwen3:
// 6.47 vs 6.19).  The 32-byte tree kernels are held to 2 CTAs per SM, the
// rank-order 32-byte kernel's occupancy.  The others keep the compiler's
// choice (an explicit minimum of 1 CTA raised the rank-order kernels'
// registers and cost bandwidth).
template <int G, int U, bool SLOT, bool TREE, bool V32, int NG>
__global__ void __launch_bounds__(kThreads, (TREE && NG == 8) ? 1 : (TREE && (V32 || NG == 4)) ? 2 : (TREE && NG == -1) ? 3 : 0)
rs_reduce_kernel(const RsParams a) {
    // s_src is double-buffered: tile i writes buffer i&1 while no thread can
    // still be reading the same buffer from tile i-2 (a barrier lies between).
    __shared__ const uint16_t* s_src[2][TIDE_MAX_WORLD];
    const int tid = threadIdx.x;
    const int W = a.world;

    // Every thread keeps the next tile's descriptor in registers: its load is
    // in flight while the current tile is reduced, so no tile waits on it.  The
    // next tile is t + gridDim.x, or, with dynamic claiming, one claimed from
    // the counter at the start of the current tile (the claim is in flight
    // while the tile's sources are staged, and read after the tile's barrier).
    __shared__ int64_t s_next[2];
    // (claiming is compiled only into the kernels of W > 4 outside the one-group tree: those
    // run at 3-4 CTAs per SM on 64-80 registers, which the claim's registers would push
    // into spills; the host's flag is then ignored and they keep the fixed stride)
    constexpr bool kClaim = G >= 8 && !(TREE && NG == -1);
    const bool dyn = kClaim && a.dynamic;
    int64_t t = blockIdx.x;
    tide_tile_t next = t < a.n_tiles ? a.tiles[t] : tide_tile_t{};
    for (int buf = 0; t < a.n_tiles; buf ^= 1) {
        const tide_tile_t tl = next;
        int64_t nt = t + gridDim.x;
        if (dyn) {
            if (tid == 0) s_next[buf] = (int64_t)gridDim.x + (int64_t)atomicAdd(a.counter, 1ull);
        } else if (nt < a.n_tiles) {
            next = a.tiles[nt];
        }

        // Range check of the descriptor against the buffers the host validated.
        const bool param_ok = tl.param >= 0 && tl.param < a.n_params;
        const int64_t src_off = SLOT ? tl.dst_off : tl.src_off;
        const int64_t src_lim = SLOT ? a.slot_numel : (param_ok ? a.numel[tl.param] : -1);
        // (an all-pad tile reads nothing, so its source offset may lie past the tensor)
        const bool ok = param_ok && tl.n_valid >= 0 && tl.n_valid <= tl.n_total &&
                        tl.dst_off >= 0 && tl.dst_off + tl.n_total <= a.out_numel &&
                        (tl.n_valid == 0 || (src_off >= 0 && src_off + tl.n_valid <= src_lim));
        if (!ok && tid == 0) atomicOr(a.err, TIDE_KCHECK_TILE);

        const uint16_t** srcs = s_src[buf];
        bool misaligned = false;
        for (int k = tid; ok && k < W; k += kThreads) {
            const void* base = a.src_tab[SLOT ? k : (int64_t)k * a.n_params + tl.param];
            const uint16_t* p = static_cast<const uint16_t*>(base) + src_off;
            srcs[k] = p;
            misaligned |= (reinterpret_cast<uintptr_t>(p) & 15) != 0;
        }
        float* __restrict__ dst = a.out + tl.dst_off;
        misaligned |= (reinterpret_cast<uintptr_t>(dst) & 15) != 0;
        if (V32) {
            for (int k = tid; ok && k < W; k += kThreads)
                misaligned |= (reinterpret_cast<uintptr_t>(srcs[k]) & 31) != 0;
            misaligned |= (reinterpret_cast<uintptr_t>(dst) & 31) != 0;
        }
        const bool scalar_only = __syncthreads_or(misaligned);
        if (dyn) {
            nt = s_next[buf];
            if (nt < a.n_tiles) next = a.tiles[nt];
        }
        if (!ok) {  // skipped after the barrier, so every tile keeps exactly one
            t = nt;
            continue;
        }

        int nv;  // 8-element units covered by the vector body
        if (V32) {
            // 16 outputs per thread per step: W 32-byte loads, two 32-byte stores.
            const int nv16 = scalar_only ? 0 : (tl.n_valid >> 4);
            for (int v = tid; v < nv16; v += kThreads) {
                float acc[16];
                auto load = [&](int k) { return ld_stream_v8(srcs[k] + 16 * (int64_t)v); };
                // (the 32-byte tree kernels run only for W = NG * G, tree fixed at compile time)
                if constexpr (!TREE) reduce_ranks<G, 16, false, V8>(W, load, acc);
                else tree_groups<G, (NG > 0 ? NG : 1), 16, V8>(load, acc);
                if (a.do_scale) {
#pragma unroll
                    for (int l = 0; l < 16; ++l) acc[l] = __fmul_rn(acc[l], a.scale);
                }
                float* o = dst + 16 * (int64_t)v;
                st_stream_f8(o, *reinterpret_cast<const float(*)[8]>(&acc[0]));
                st_stream_f8(o + 8, *reinterpret_cast<const float(*)[8]>(&acc[8]));
            }
            nv = 2 * nv16;
        } else {
            nv = scalar_only ? 0 : (tl.n_valid >> 3);
        }
        // Vector body: 8 outputs per thread per unit, U units per step.
        for (int v0 = 0; !V32 && v0 < nv; v0 += kThreads * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + u * kThreads + tid;
                if (v < nv) {
                    // (the four-group tree re-reads each source address from shared memory at
                    // its use, in order, rather than keeping all W addresses in registers)
                    auto load = [&](int k) {
                        if constexpr (TREE && NG == 4) {
                            const uint16_t* p = const_cast<const uint16_t* const volatile*>(srcs)[k];
                            return ld_stream_v4_ordered(p + 8 * (int64_t)v);
                        } else {
                            return ld_stream_v4(srcs[k] + 8 * (int64_t)v);
                        }
                    };
                    if constexpr (TREE && NG == -1) tree_one_group<G, 8, uint4>(W, load, acc[u]);
                    else if constexpr (TREE && NG > 0) tree_groups<G, NG, 8, uint4>(load, acc[u]);
                    else reduce_ranks<G, 8, TREE, uint4>(W, load, acc[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + u * kThreads + tid;
                if (v < nv) {
                    if (a.do_scale) {
#pragma unroll
                        for (int l = 0; l < 8; ++l) acc[u][l] = __fmul_rn(acc[u][l], a.scale);
                    }
                    float* o = dst + 8 * (int64_t)v;
                    st_stream_f4(o, acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
                    st_stream_f4(o + 4, acc[u][4], acc[u][5], acc[u][6], acc[u][7]);
                }
            }
        }
        // Remaining valid elements one by one (ragged end, or a misaligned tile).
        for (int e = 8 * nv + tid; e < tl.n_valid; e += kThreads) {
            float acc[1];
            auto load = [&](int k) { return (uint32_t)ld_stream_u16(srcs[k] + e); };
            if constexpr (TREE && NG == -1) tree_one_group<G, 1, uint32_t>(W, load, acc);
            else if constexpr (TREE && NG > 0) tree_groups<G, NG, 1, uint32_t>(load, acc);
            else reduce_ranks<G, 1, TREE, uint32_t>(W, load, acc);
            if (a.do_scale) acc[0] = __fmul_rn(acc[0], a.scale);
            dst[e] = acc[0];
        }
        // Pad positions are +0.0.
        for (int e = tl.n_valid + tid; e < tl.n_total; e += kThreads) dst[e] = 0.0f;
        t = nt;
    }
    // With dynamic claiming the last CTA to finish puts both counters back to zero for the
    // next launch on the stream (each CTA's claims precede its count, fenced).
    if (dyn && tid == 0) {
        __threadfence();
        if (atomicAdd(a.counter + 1, 1ull) == (unsigned long long)gridDim.x - 1) {
            a.counter[0] = 0;
            a.counter[1] = 0;
            __threadfence();
        }
    }
}

using KernelFn = void (*)(const RsParams);

template <bool SLOT, bool TREE>
KernelFn pick(int world, bool v32) {
    // (in the tree order every W <= G is one group, so G < 8 kernels never merge)
    if constexpr (!TREE) {
        // W = 2 in rank order: the 32-byte kernel over one group of two ranks (64
        // registers, 4 CTAs per SM; the group of 8 held 119 registers and 2 CTAs per SM)
        if (v32 && world == 2) return rs_reduce_kernel<2, 1, SLOT, false, true, 0>;
    }
    // (for W <= 2 the tree is one add, the same as rank order, so the rank-order
    // kernels serve it)
    if constexpr (TREE) {
        if (world <= 2) return pick<SLOT, false>(world, v32);
    }
    if (world <= 2) return rs_reduce_kernel<2, 4, SLOT, false, false, 0>;
    if constexpr (TREE) {
        // W = 4: the 32-byte tree over one group of 4 (6.13 against 4.93 TB/s on the
        // sweep's W = 4 group with the 16-byte kernel)
        if (v32 && world == 4) return rs_reduce_kernel<4, 1, SLOT, true, true, 1>;
    }
    if (world <= 4) return rs_reduce_kernel<4, 2, SLOT, TREE, false, TREE ? -1 : 0>;
    if constexpr (TREE) {
        // 32-byte tree kernels: exactly one group (W = 8) or two groups (W = 16) of 8
        if (v32 && (world == 8 || world == 16))
            return world == 8 ? rs_reduce_kernel<8, 1, SLOT, true, true, 1>
                              : rs_reduce_kernel<8, 1, SLOT, true, true, 2>;
        if (world <= 8) return rs_reduce_kernel<8, 1, SLOT, true, false, -1>;
        // 16-byte trees fixed at compile time for W = 16, 32 and 64
        if (world == 16) return rs_reduce_kernel<8, 1, SLOT, true, false, 2>;
        if (world == 32) return rs_reduce_kernel<8, 1, SLOT, true, false, 4>;
        if (world == 64) return rs_reduce_kernel<8, 1, SLOT, true, false, 8>;
        return rs_reduce_kernel<8, 1, SLOT, true, false, 0>;
    } else {
        if (v32 && world <= kV32MaxWorld) return rs_reduce_kernel<8, 1, SLOT, false, true, 0>;
        return rs_reduce_kernel<8, 1, SLOT, false, false, 0>;
    }
}

KernelFn select(int world, bool slot, int order, bool v32) {
    const bool tree = order == TIDE_ORDER_TREE;
    if (slot) return tree ? pick<true, true>(world, v32) : pick<true, false>(world, v32);
    return tree ? pick<false, true>(world, v32) : pick<false, false>(world, v32);
}

}  // namespace

bool rs_v32_applies(int world, int order) {
    if (order == TIDE_ORDER_TREE) return world == 2 || world == 4 || world == 8 || world == 16;
    return world == 2 || (world > 4 && world <= kV32MaxWorld);
}

int rs_blocks_per_sm(int world, bool slot, int order, bool v32) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, select(world, slot, order, v32), kThreads, 0) !=
        cudaSuccess)
        return 0;
    return n;
}

cudaError_t launch_rs_reduce(const tide_plan* p, const void* const* d_src_tab, bool slot,
                             int64_t src_bound, float* out, int64_t out_numel, float scale,
                             bool do_scale, int order, int grid, cudaStream_t stream, bool v32,
                             int64_t t0, int64_t t1) {
    if (t1 < 0) t1 = (int64_t)p->tiles.size();
    if (t1 <= t0 || grid <= 0) return cudaSuccess;
    RsParams a;
    a.tiles = p->d_tiles + t0;
    a.n_tiles = t1 - t0;
    a.src_tab = d_src_tab;
    a.numel = p->d_numel;
    a.slot_numel = src_bound;
    a.out = out;
    a.out_numel = out_numel;
    a.world = p->world;
    a.n_params = p->n_params;
    a.scale = scale;
    a.do_scale = do_scale ? 1 : 0;
    a.err = p->d_err;
    // Claiming tiles as CTAs finish evens out CTAs that run slower than others (their end
    // is the launch's tail): 70B W=8 7.06 -> 7.18 TB/s, Wan2.2 W=16 6.94 -> 7.17, the
    // sweep's W = 64 group 6.86 -> 7.14.  A claim costs a global atomic per tile, hidden by
    // a second CTA on the SM; with few tiles per CTA there is no tail to even out and the
    // claims cost more than they save (sweep W=2: -10 %, W=8: -1 %), so launches with under
    // 2 CTAs per SM or under 16 tiles per CTA keep the fixed stride, and so does W <= 4.
    a.dynamic = (p->world > 4 && grid >= 2 * p->sm_count && t1 - t0 >= 16 * (int64_t)grid) ? 1 : 0;
    a.counter = p->d_counter;
    (void)cudaGetLastError();  // drop an error left by an earlier failed runtime call
    select(p->world, slot, order, v32)<<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace tide
