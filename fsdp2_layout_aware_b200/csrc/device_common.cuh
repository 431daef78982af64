// device_common.cuh - memory helpers shared by the libtide.so kernels.
//
// Everything here moves bytes: streaming 16-byte loads that skip L1 (each
// input byte is read exactly once), streaming stores, and a block-wide
// segmented copy with an aligned vector body.  All sizes come from tiles that
// the caller has already range-checked.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace tide {

// 16-byte load of data read once: no L1 allocation, 256-byte L2 prefetch.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

__device__ __forceinline__ uint16_t ld_stream_u16(const uint16_t* p) {
    unsigned short v;
    asm("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// 16-byte store of data nobody re-reads soon (evict-first in L2).
__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};"
                 :
                 : "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_stream_f4(float* p, float a, float b, float c, float d) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};"
                 :
                 : "l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_one(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

__device__ __forceinline__ void unpack8(const uint4& x, float f[8]) {
    f[0] = bf16_lo(x.x); f[1] = bf16_hi(x.x);
    f[2] = bf16_lo(x.y); f[3] = bf16_hi(x.y);
    f[4] = bf16_lo(x.z); f[5] = bf16_hi(x.z);
    f[6] = bf16_lo(x.w); f[7] = bf16_hi(x.w);
}

// Block-wide copy of n bf16 elements.  When source and destination share
// their offset modulo 16 bytes, a short scalar head brings both to a 16-byte
// boundary and the body moves 16-byte vectors, U per thread per step (all U
// loads issued before the first store); otherwise every element is moved on
// its own (still coalesced).
template <int U, int NT>
__device__ __forceinline__ void block_copy_bf16(const uint16_t* __restrict__ src,
                                                uint16_t* __restrict__ dst, int n) {
    const int tid = threadIdx.x;
    const uintptr_t sa = reinterpret_cast<uintptr_t>(src), da = reinterpret_cast<uintptr_t>(dst);
    int done = 0;
    if (((sa ^ da) & 15) == 0) {
        int head = (int)(((16 - (da & 15)) & 15) >> 1);
        if (head > n) head = n;
        if (tid < head) dst[tid] = ld_stream_u16(src + tid);
        const int nv = (n - head) >> 3;
        const uint16_t* s = src + head;
        uint16_t* d = dst + head;
        for (int v0 = 0; v0 < nv; v0 += NT * U) {
            uint4 x[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + u * NT + tid;
                if (v < nv) x[u] = ld_stream_v4(s + 8 * (int64_t)v);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + u * NT + tid;
                if (v < nv) st_stream_v4(d + 8 * (int64_t)v, x[u]);
            }
        }
        done = head + 8 * nv;
    }
    for (int e = done + tid; e < n; e += NT) dst[e] = ld_stream_u16(src + e);
}

// Block-wide zero fill of n bf16 elements.
template <int NT>
__device__ __forceinline__ void block_zero_bf16(uint16_t* dst, int n) {
    const int tid = threadIdx.x;
    const uintptr_t da = reinterpret_cast<uintptr_t>(dst);
    int head = (int)(((16 - (da & 15)) & 15) >> 1);
    if (head > n) head = n;
    if (tid < head) dst[tid] = 0;
    const int nv = (n - head) >> 3;
    for (int v = tid; v < nv; v += NT) st_stream_v4(dst + head + 8 * (int64_t)v, make_uint4(0, 0, 0, 0));
    for (int e = head + 8 * nv + tid; e < n; e += NT) dst[e] = 0;
}

}  // namespace tide
