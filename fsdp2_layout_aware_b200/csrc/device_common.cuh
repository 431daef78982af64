// device_common.cuh - memory helpers shared by the libtide.so kernels.
//
// Everything here moves bytes: streaming 16- and 32-byte loads that skip L1
// (each input byte is read exactly once), streaming stores, and a block-wide
// segmented copy with an aligned vector body.  All sizes come from tiles that
// the caller has already range-checked.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace tide {

// Loads of data read exactly once: no L1 allocation.  (An L2 256-byte
// prefetch hint measured 0.5-1 % slower on B200; an evict-first hint, 3-6 %.)

// 16-byte load; p must be 16-byte aligned.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// ld_stream_v4 that the compiler keeps in program order with other volatile asm
// (a wide tree loads one group of ranks at a time this way, so registers hold
// one group's raw vectors, not all of them).
__device__ __forceinline__ uint4 ld_stream_v4_ordered(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 32 bytes (16 bf16) as eight 32-bit words.
struct V8 {
    uint32_t w[8];
};

// 32-byte load (a single sm_100 vector load); p must be 32-byte aligned.
__device__ __forceinline__ V8 ld_stream_v8(const void* p) {
    V8 v;
    asm("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]), "=r"(v.w[5]),
          "=r"(v.w[6]), "=r"(v.w[7])
        : "l"(p));
    return v;
}

// 32-byte streaming store of 8 floats; p must be 32-byte aligned.  (Plain and
// L1::no_allocate stores measured within 1 % of this on B200.)
__device__ __forceinline__ void st_stream_f8(float* p, const float (&f)[8]) {
    asm volatile("st.global.cs.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :
                 : "l"(p), "f"(f[0]), "f"(f[1]), "f"(f[2]), "f"(f[3]), "f"(f[4]), "f"(f[5]),
                   "f"(f[6]), "f"(f[7])
                 : "memory");
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

// 32-byte streaming store of eight 32-bit words; p must be 32-byte aligned.
__device__ __forceinline__ void st_stream_v8(void* p, const V8& v) {
    asm volatile("st.global.cs.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :
                 : "l"(p), "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]),
                   "r"(v.w[5]), "r"(v.w[6]), "r"(v.w[7])
                 : "memory");
}

// As block_copy_bf16 with 32-byte vectors: source and destination must share
// their offset modulo 32 bytes for the vector body (otherwise the 16-byte copy
// above takes over).
template <int U, int NT>
__device__ __forceinline__ void block_copy_bf16_v32(const uint16_t* __restrict__ src,
                                                    uint16_t* __restrict__ dst, int n) {
    const uintptr_t sa = reinterpret_cast<uintptr_t>(src), da = reinterpret_cast<uintptr_t>(dst);
    if (((sa ^ da) & 31) != 0) {
        block_copy_bf16<2 * U, NT>(src, dst, n);
        return;
    }
    const int tid = threadIdx.x;
    int head = (int)(((32 - (da & 31)) & 31) >> 1);
    if (head > n) head = n;
    if (tid < head) dst[tid] = ld_stream_u16(src + tid);
    const int nv = (n - head) >> 4;
    const uint16_t* s = src + head;
    uint16_t* d = dst + head;
    for (int v0 = 0; v0 < nv; v0 += NT * U) {
        V8 x[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int v = v0 + u * NT + tid;
            if (v < nv) x[u] = ld_stream_v8(s + 16 * (int64_t)v);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int v = v0 + u * NT + tid;
            if (v < nv) st_stream_v8(d + 16 * (int64_t)v, x[u]);
        }
    }
    for (int e = head + 16 * nv + tid; e < n; e += NT) dst[e] = ld_stream_u16(src + e);
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
