// ce.cpp - copy-engine (SM-free) variants of AG placement and Slot-Reuse staging.
//
// "The Endgame of FSDP Communication" (weekinpapers.com, Abstract; kongchang.com,
// "TIDE's Design Approach") places all-gather shards without using SMs and
// moves gradients with copy engines.  On one GPU the same placement is a set
// of device-to-device memcpys that the copy engines execute: per parameter one
// 2-D copy covers every rank whose chunk is entirely valid (source rows Ns
// apart in the rank-major buffer, destination rows c_i apart in parameter
// storage), one 1-D copy covers a partially valid chunk, and one memset clears
// the pad rows, which are contiguous at the end of the padded storage.  No
// kernel is launched.  One cudaMemcpyAsync (or 2-D variant) per copy keeps the
// API surface to the plain asynchronous calls.
#include <algorithm>

#include "tide_internal.h"

namespace tide {
namespace {

// Copy `rows` rows of `width` bytes; falls back to one 1-D copy per row when a
// pitch exceeds the device limit.
cudaError_t copy_rows(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width,
                      int64_t rows, size_t max_pitch, cudaStream_t stream) {
    if (rows <= 0 || width == 0) return cudaSuccess;
    if (rows == 1) return cudaMemcpyAsync(dst, src, width, cudaMemcpyDeviceToDevice, stream);
    if (dpitch <= max_pitch && spitch <= max_pitch)
        return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, (size_t)rows,
                                 cudaMemcpyDeviceToDevice, stream);
    for (int64_t r = 0; r < rows; ++r) {
        cudaError_t e = cudaMemcpyAsync(static_cast<char*>(dst) + r * dpitch,
                                        static_cast<const char*>(src) + r * spitch, width,
                                        cudaMemcpyDeviceToDevice, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

size_t device_max_pitch(int device) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxPitch, device) != cudaSuccess || v <= 0) return 0;
    return (size_t)v;
}

}  // namespace

cudaError_t ce_ag_place(const tide_plan* p, const uint16_t* ag, void* const* params,
                        cudaStream_t stream) {
    const int64_t W = p->world, Ns = p->shard_numel;
    const size_t max_pitch = device_max_pitch(p->device);
    for (int32_t i = 0; i < p->n_params; ++i) {
        const int64_t c = p->chunk[i], n = p->numel[i];
        if (c == 0) continue;
        uint16_t* dst = static_cast<uint16_t*>(params[i]);
        const uint16_t* src = ag + p->offset[i];
        const int64_t full = std::min(W, n / c);
        cudaError_t e = copy_rows(dst, 2 * c, src, 2 * Ns, 2 * c, full, max_pitch, stream);
        if (e != cudaSuccess) return e;
        const int64_t rem = n - full * c;
        if (rem > 0 && full < W) {
            e = cudaMemcpyAsync(dst + full * c, src + full * Ns, 2 * rem, cudaMemcpyDeviceToDevice,
                                stream);
            if (e != cudaSuccess) return e;
        }
        if (W * c > n) {
            e = cudaMemsetAsync(dst + n, 0, 2 * (W * c - n), stream);
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

// Stage the chunks that output ranks [r0, r1) need (r1 < 0: up to W) from every
// source rank k into slot k.
cudaError_t ce_slot_stage(const tide_plan* p, const void* const* grads, void* const* slots,
                          cudaStream_t stream, int64_t r0, int64_t r1) {
    const int64_t W = p->world, P = p->n_params, Ns = p->shard_numel;
    if (r1 < 0) r1 = W;
    const size_t max_pitch = device_max_pitch(p->device);
    for (int64_t k = 0; k < W; ++k) {
        uint16_t* slot = static_cast<uint16_t*>(slots[k]);
        for (int64_t i = 0; i < P; ++i) {
            const int64_t c = p->chunk[i], n = p->numel[i];
            if (c == 0 || n == 0) continue;
            const uint16_t* g = static_cast<const uint16_t*>(grads[k * P + i]);
            uint16_t* dst = slot + p->offset[i];
            const int64_t full = std::min(W, n / c);  // ranks [0, full) hold whole chunks
            const int64_t fr1 = std::min(full, r1);
            if (fr1 > r0) {
                cudaError_t e = copy_rows(dst + r0 * Ns, 2 * Ns, g + r0 * c, 2 * c, 2 * c, fr1 - r0,
                                          max_pitch, stream);
                if (e != cudaSuccess) return e;
            }
            const int64_t rem = n - full * c;       // rank `full` holds a partial chunk
            if (rem > 0 && full < W && full >= r0 && full < r1) {
                cudaError_t e = cudaMemcpyAsync(dst + full * Ns, g + full * c, 2 * rem,
                                                cudaMemcpyDeviceToDevice, stream);
                if (e != cudaSuccess) return e;
            }
        }
    }
    return cudaSuccess;
}

}  // namespace tide
