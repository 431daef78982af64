// reduce_ranks.cuh - the fp32 reduction over W ranks shared by the RS kernels.
//
// Given a loader that returns rank k's raw bf16 bits (a 16-byte vector of 8,
// or a single element), reduce_ranks produces the fp32 sum in one of two
// orders.  bf16 -> fp32 is exact; every add is __fadd_rn, so no contraction
// or reassociation can change the bits.
#pragma once

#include <cstdint>

#include "device_common.cuh"

namespace tide {

constexpr int kMaxTreeLevels = 6;  // binary counter over ceil(W/G) <= 63 groups

// Lane l (0..7) of a 16-byte vector of 8 bf16, or the single bf16 of a scalar,
// as fp32 (exact).  l is a compile-time constant after unrolling.
__device__ __forceinline__ float lane(const uint4& x, int l) {
    const uint32_t w = l < 2 ? x.x : l < 4 ? x.y : l < 6 ? x.z : x.w;
    return (l & 1) ? bf16_hi(w) : bf16_lo(w);
}
__device__ __forceinline__ float lane(uint32_t x, int) { return __uint_as_float(x << 16); }
// Lane l (0..15) of a 32-byte vector of 16 bf16.
__device__ __forceinline__ float lane(const V8& x, int l) {
    return (l & 1) ? bf16_hi(x.w[l >> 1]) : bf16_lo(x.w[l >> 1]);
}

// Reduce W ranks for L lanes (L = 8: one 16-byte vector per rank; L = 1: one
// element).  load(k) returns rank k's raw bf16 bits; loads are issued G ranks
// at a time, before any add, and converted to fp32 inside the adds.
//   Rank order: acc = g_0, then acc = acc + g_k for k = 1..W-1, one add per
//   rank in order (grouping only batches the loads, never the adds).
//   Tree: within a group, adjacent ranks are added pairwise level by level (an
//   unpaired last one is carried); group sums are merged pairwise through a
//   binary counter, which is a balanced tree when the group count is a power
//   of two.
template <int G, int L, bool TREE, class Raw, class Load>
__device__ __forceinline__ void reduce_ranks(int W, Load load, float (&acc)[L]) {
    float stack[TREE ? kMaxTreeLevels : 1][L];
    int gidx = 0;
    for (int k0 = 0; k0 < W; k0 += G, ++gidx) {
        Raw x[G];
        const int n_in = min(G, W - k0);
#pragma unroll
        for (int j = 0; j < G; ++j) {
            if (j < n_in) x[j] = load(k0 + j);
        }
        if (!TREE) {
#pragma unroll
            for (int j = 0; j < G; ++j) {
                if (j < n_in) {
                    if (k0 + j == 0) {
#pragma unroll
                        for (int l = 0; l < L; ++l) acc[l] = lane(x[0], l);
                    } else {
#pragma unroll
                        for (int l = 0; l < L; ++l) acc[l] = __fadd_rn(acc[l], lane(x[j], l));
                    }
                }
            }
        } else {
            // level 1 straight from the raw values, then in place
            constexpr int H = (G + 1) / 2;
            float f[H][L];
#pragma unroll
            for (int j = 0; j < G; j += 2) {
#pragma unroll
                for (int l = 0; l < L; ++l) {
                    if (j + 1 < n_in) f[j / 2][l] = __fadd_rn(lane(x[j], l), lane(x[j + 1], l));
                    else if (j < n_in) f[j / 2][l] = lane(x[j], l);
                }
            }
            const int n_half = (n_in + 1) / 2;
#pragma unroll
            for (int step = 1; step < H; step <<= 1) {
#pragma unroll
                for (int j = 0; j + step < H; j += 2 * step) {
                    if (j + step < n_half) {
#pragma unroll
                        for (int l = 0; l < L; ++l) f[j][l] = __fadd_rn(f[j][l], f[j + step][l]);
                    }
                }
            }
            // push the group sum as a level-0 node; merge while the counter carries
#pragma unroll
            for (int lvl = 0; lvl < kMaxTreeLevels; ++lvl) {
                if ((gidx >> lvl) & 1) {
#pragma unroll
                    for (int l = 0; l < L; ++l) f[0][l] = __fadd_rn(stack[lvl][l], f[0][l]);
                } else {
#pragma unroll
                    for (int l = 0; l < L; ++l) stack[lvl][l] = f[0][l];
                    break;
                }
            }
        }
    }
    if (TREE) {
        // gidx is now the group count; occupied levels are its set bits
        bool have = false;
#pragma unroll
        for (int lvl = 0; lvl < kMaxTreeLevels; ++lvl) {
            if ((gidx >> lvl) & 1) {
#pragma unroll
                for (int l = 0; l < L; ++l)
                    acc[l] = have ? __fadd_rn(stack[lvl][l], acc[l]) : stack[lvl][l];
                have = true;
            }
        }
    }
}

// The tree order when all W <= G ranks fit in one group: the same adds as
// reduce_ranks<G, L, true> makes for such a W (so the same bits), without the
// group-merge stack.
template <int G, int L, class Raw, class Load>
__device__ __forceinline__ void tree_one_group(int W, Load load, float (&acc)[L]) {
    Raw x[G];
#pragma unroll
    for (int j = 0; j < G; ++j) {
        if (j < W) x[j] = load(j);
    }
    constexpr int H = (G + 1) / 2;
    float f[H][L];
#pragma unroll
    for (int j = 0; j < G; j += 2) {
#pragma unroll
        for (int l = 0; l < L; ++l) {
            if (j + 1 < W) f[j / 2][l] = __fadd_rn(lane(x[j], l), lane(x[j + 1], l));
            else if (j < W) f[j / 2][l] = lane(x[j], l);
        }
    }
    const int n_half = (W + 1) / 2;
#pragma unroll
    for (int step = 1; step < H; step <<= 1) {
#pragma unroll
        for (int j = 0; j + step < H; j += 2 * step) {
            if (j + step < n_half) {
#pragma unroll
                for (int l = 0; l < L; ++l) f[j][l] = __fadd_rn(f[j][l], f[j + step][l]);
            }
        }
    }
#pragma unroll
    for (int l = 0; l < L; ++l) acc[l] = f[0][l];
}

// The tree order when W = NG * G exactly, NG a power of two, fixed at compile
// time: the two halves' trees, then one add that joins them, recursively down
// to single groups.  For W a power of two this is the balanced binary tree,
// which is what adjacent pairs level by level make (no odd one is ever carried)
// and what reduce_ranks<G, L, true> makes by merging group sums through its
// binary counter -- the same bits, with no merge stack and no run-time W.  The
// second half is loaded only after the first is reduced, so at most one
// group's raw vectors are live beside log2(NG) partial sums.
template <int G, int NG, int L, class Raw, class Load>
__device__ __forceinline__ void tree_groups(Load load, float (&acc)[L]) {
    static_assert(NG >= 1 && (NG & (NG - 1)) == 0, "group count must be a power of two");
    if constexpr (NG == 1) {
        tree_one_group<G, L, Raw>(G, load, acc);
    } else {
        float first[L];
        tree_groups<G, NG / 2, L, Raw>(load, first);
        // the first half's sums exist before the second half's loads are issued (with
        // ordered loads, see ld_stream_v4_ordered, the compiler cannot hoist them above)
#pragma unroll
        for (int l = 0; l < L; ++l) asm volatile("" : "+f"(first[l]));
        tree_groups<G, NG / 2, L, Raw>([&](int k) { return load(NG / 2 * G + k); }, acc);
#pragma unroll
        for (int l = 0; l < L; ++l) acc[l] = __fadd_rn(first[l], acc[l]);
    }
}

}  // namespace tide
