// rs_reduce_noalloc.cu - tide_rs_reduce_noalloc: the rank-order TIDE-RS reduction
// without any device (or host heap) allocation.
//
// Why it exists: tide_rs_reduce needs a plan, and tide_plan_group allocates
// the plan's device tables with cudaMalloc.  Some callers cannot do that: a
// training runtime whose caching allocator has already reserved the GPU's
// memory for its own arena (a foreign cudaMalloc then fails or fragments that
// arena), or a hot loop that cannot afford the device-wide synchronisation a
// cudaMalloc/cudaFree may cause.  This entry point takes the parameter shapes
// directly and keeps the small per-call tables (per-parameter layout and the
// gradient pointer table) in one fixed device array that is part of the
// library's module, so it allocates nothing.
//
// Contract (also in include/tide.h):
//   - Scratch: `g_noalloc_scratch`, TIDE_NOALLOC_SCRATCH_BYTES (1 MiB), a
//     file-scope __device__ array; every GPU that loads libtide.so holds it
//     until the process exits.  A call needs 32*P + 8*W*P bytes of it; larger
//     groups are rejected with TIDE_ERR_SIZE before anything happens.
//   - The first call on each device looks up that device's address of the
//     array (cudaGetSymbolAddress, with the device current) and caches it; make
//     that first call before any stream capture.  The cached address lives as
//     long as the process; after cudaDeviceReset on a device (which unloads
//     this module there) the entry point must not be called on that device.
//   - A call on a stream that is being captured is refused with
//     TIDE_ERR_INVALID_ARG before anything is enqueued: the tables are copied
//     from one host array that every later call overwrites, so a recorded copy
//     would replay another call's tables.
//   - Every call rewrites every byte of the array that its kernel reads (the
//     previous call's tables are left beyond that and never read), so nothing
//     depends on earlier contents.  Calls that may overlap on the GPU
//     (different streams, not ordered by the caller) race on the array and
//     must not be issued.
//   - The tables are copied from a fixed host array with one pageable
//     cudaMemcpyAsync on `stream`; the runtime has consumed the host array when
//     that call returns, so the host array is reused by the next call.
//   - No cudaMalloc, cudaFree, host malloc or library allocation is made.
#include <cstring>
#include <mutex>

#include "device_common.cuh"
#include "tide_internal.h"

namespace {

constexpr int64_t kScratchBytes = TIDE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// One row of the per-parameter table.
struct NaParam {
    int64_t numel;       // d0 * inner (unpadded gradient length)
    int64_t chunk;       // c = ceil(d0 / W) * inner
    int64_t offset;      // off inside a rank's shard
    int64_t tile_begin;  // first tile index of this param (tiles of all ranks)
};

struct NaArgs {
    unsigned char* scratch;  // device address of g_noalloc_scratch on this device
    int32_t n_params;
    int32_t world;
    int64_t shard_numel;
    int64_t n_tiles;
    float* out;
    int64_t out_numel;
    float scale;
    int32_t do_scale;
};

__device__ __forceinline__ float lane_of(const uint4& x, int l) {
    const uint32_t w = l < 2 ? x.x : l < 4 ? x.y : l < 6 ? x.z : x.w;
    return (l & 1) ? tide::bf16_hi(w) : tide::bf16_lo(w);
}

__global__ void __launch_bounds__(tide::kThreads) rs_reduce_noalloc_kernel(const NaArgs a) {
    constexpr int G = 8;
    constexpr int TILE = TIDE_TILE_ELEMS;
    __shared__ const uint16_t* s_src[TIDE_MAX_WORLD];
    __shared__ int64_t s_desc[4];  // src_off, dst_off, n_valid, n_total
    const int tid = threadIdx.x;
    const int W = a.world, P = a.n_params;
    const NaParam* prm = reinterpret_cast<const NaParam*>(a.scratch);
    const void* const* tab = reinterpret_cast<const void* const*>(prm + P);

    for (int64_t t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
        __syncthreads();
        if (tid == 0) {
            // the param whose tile range holds t (tile_begin is non-decreasing)
            int lo = 0, hi = P - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (prm[mid].tile_begin <= t) lo = mid; else hi = mid - 1;
            }
            const NaParam q = prm[lo];
            const int64_t per_rank = (q.chunk + TILE - 1) / TILE;
            const int64_t local = t - q.tile_begin;
            const int64_t r = per_rank > 0 ? local / per_rank : 0;
            const int64_t e0 = (local - r * per_rank) * TILE;
            const int64_t n_total = min((int64_t)TILE, q.chunk - e0);
            const int64_t valid = min(q.chunk, max((int64_t)0, q.numel - r * q.chunk));
            const int64_t n_valid = min(n_total, max((int64_t)0, valid - e0));
            const int64_t dst_off = r * a.shard_numel + q.offset + e0;
            // holds by construction of the tables; a failing tile is skipped
            const bool ok = per_rank > 0 && r < W && n_total > 0 && dst_off >= 0 &&
                            dst_off + n_total <= a.out_numel;
            s_desc[0] = r * q.chunk + e0;
            s_desc[1] = dst_off;
            s_desc[2] = ok ? n_valid : 0;
            s_desc[3] = ok ? n_total : 0;
            for (int k = 0; k < W; ++k) {
                const void* base = tab[(int64_t)k * P + lo];
                s_src[k] = static_cast<const uint16_t*>(base) + s_desc[0];
            }
        }
        __syncthreads();
        const int n_valid = (int)s_desc[2], n_total = (int)s_desc[3];
        float* __restrict__ dst = a.out + s_desc[1];
        bool mis = false;
        for (int k = tid; k < W; k += tide::kThreads) mis |= (reinterpret_cast<uintptr_t>(s_src[k]) & 15) != 0;
        mis |= (reinterpret_cast<uintptr_t>(dst) & 15) != 0;
        const bool scalar_only = __syncthreads_or(mis);

        const int nv = scalar_only ? 0 : (n_valid >> 3);
        for (int v = tid; v < nv; v += tide::kThreads) {
            float acc[8];
            for (int k0 = 0; k0 < W; k0 += G) {
                uint4 x[G];
                const int n_in = min(G, W - k0);
#pragma unroll
                for (int j = 0; j < G; ++j)
                    if (j < n_in) x[j] = tide::ld_stream_v4(s_src[k0 + j] + 8 * (int64_t)v);
#pragma unroll
                for (int j = 0; j < G; ++j) {
                    if (j < n_in) {
#pragma unroll
                        for (int l = 0; l < 8; ++l)
                            acc[l] = (k0 + j == 0) ? lane_of(x[0], l) : __fadd_rn(acc[l], lane_of(x[j], l));
                    }
                }
            }
            if (a.do_scale) {
#pragma unroll
                for (int l = 0; l < 8; ++l) acc[l] = __fmul_rn(acc[l], a.scale);
            }
            float* o = dst + 8 * (int64_t)v;
            tide::st_stream_f4(o, acc[0], acc[1], acc[2], acc[3]);
            tide::st_stream_f4(o + 4, acc[4], acc[5], acc[6], acc[7]);
        }
        for (int e = 8 * nv + tid; e < n_valid; e += tide::kThreads) {
            float acc = tide::bf16_one(tide::ld_stream_u16(s_src[0] + e));
            for (int k = 1; k < W; ++k) acc = __fadd_rn(acc, tide::bf16_one(tide::ld_stream_u16(s_src[k] + e)));
            if (a.do_scale) acc = __fmul_rn(acc, a.scale);
            dst[e] = acc;
        }
        for (int e = n_valid + tid; e < n_total; e += tide::kThreads) dst[e] = 0.0f;
    }
}

// Host side: the cached device address of the scratch array, per device, and
// the fixed host array the tables are built in.
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
alignas(256) unsigned char g_host_stage[kScratchBytes];

bool ranges_overlap(const void* a, int64_t abytes, const void* b, int64_t bbytes) {
    if (a == nullptr || b == nullptr || abytes <= 0 || bbytes <= 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + (uintptr_t)bbytes && b0 < a0 + (uintptr_t)abytes;
}

}  // namespace

extern "C" tide_status_t tide_rs_reduce_noalloc(const tide_param_t* params, int32_t n_params,
                                                int32_t world, const void* const* grads,
                                                const int64_t* grad_numel, float* out,
                                                int64_t out_numel, int32_t scale_mode,
                                                int32_t max_ctas, void* stream) {
    if (n_params < 0 || (n_params > 0 && params == nullptr)) return TIDE_ERR_INVALID_ARG;
    if (world < 1 || world > TIDE_MAX_WORLD || max_ctas < 0) return TIDE_ERR_INVALID_ARG;
    if (scale_mode != TIDE_SCALE_NONE && scale_mode != TIDE_SCALE_INV_WORLD) return TIDE_ERR_INVALID_ARG;
    const int64_t W = world, P = n_params;
    if (P * (int64_t)sizeof(NaParam) + W * P * 8 > kScratchBytes) return TIDE_ERR_SIZE;
    if (W * P > 0 && (grads == nullptr || grad_numel == nullptr)) return TIDE_ERR_INVALID_ARG;

    // layout and size checks (no allocation: everything is recomputed in place)
    int64_t Ns = 0, n_tiles = 0;
    for (int64_t i = 0; i < P; ++i) {
        const int64_t d0 = params[i].dim0, in = params[i].inner;
        if (d0 < 0 || in < 0 || (in > 0 && d0 > INT64_MAX / in)) return TIDE_ERR_INVALID_ARG;
        const int64_t c = (d0 / W + (d0 % W != 0)) * in;
        if (Ns > INT64_MAX / 2 - c) return TIDE_ERR_SIZE;
        Ns += c;
        n_tiles += W * ((c + TIDE_TILE_ELEMS - 1) / TIDE_TILE_ELEMS);
    }
    if (Ns > 0 && W > INT64_MAX / 4 / Ns) return TIDE_ERR_SIZE;
    const int64_t n_out = W * Ns;
    if (n_out > 0) {
        if (out == nullptr) return TIDE_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(out) % 4 != 0) return TIDE_ERR_ALIGNMENT;
        if (out_numel < n_out) return TIDE_ERR_SIZE;
    }
    for (int64_t k = 0; k < W; ++k)
        for (int64_t i = 0; i < P; ++i) {
            const int64_t n = params[i].dim0 * params[i].inner;
            const void* g = grads[k * P + i];
            if (n == 0) continue;
            if (g == nullptr) return TIDE_ERR_INVALID_ARG;
            if (reinterpret_cast<uintptr_t>(g) % 2 != 0) return TIDE_ERR_ALIGNMENT;
            if (grad_numel[k * P + i] < n) return TIDE_ERR_SIZE;
            if (ranges_overlap(out, 4 * n_out, g, 2 * n)) return TIDE_ERR_INVALID_ARG;
        }
    if (n_tiles == 0) return TIDE_OK;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &capture) != cudaSuccess) {
        (void)cudaGetLastError();
        return TIDE_ERR_CUDA;
    }
    if (capture != cudaStreamCaptureStatusNone) return TIDE_ERR_INVALID_ARG;

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TIDE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TIDE_ERR_DEVICE;

    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        // set-up, once per device, with that device current
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            (void)cudaGetLastError();
            return TIDE_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    unsigned char* scratch = static_cast<unsigned char*>(g_scratch_ptr[dev]);

    // build the tables in the fixed host array: per-param rows, then the pointers
    NaParam* prm = reinterpret_cast<NaParam*>(g_host_stage);
    int64_t off = 0, tb = 0;
    for (int64_t i = 0; i < P; ++i) {
        const int64_t d0 = params[i].dim0, in = params[i].inner;
        const int64_t c = (d0 / W + (d0 % W != 0)) * in;
        prm[i].numel = d0 * in;
        prm[i].chunk = c;
        prm[i].offset = off;
        prm[i].tile_begin = tb;
        off += c;
        tb += W * ((c + TIDE_TILE_ELEMS - 1) / TIDE_TILE_ELEMS);
    }
    const void** tab = reinterpret_cast<const void**>(prm + P);
    for (int64_t j = 0; j < W * P; ++j) tab[j] = grads[j];
    const size_t bytes = (size_t)(P * (int64_t)sizeof(NaParam) + W * P * 8);
    if (cudaMemcpyAsync(scratch, g_host_stage, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
        (void)cudaGetLastError();
        return TIDE_ERR_CUDA;
    }

    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rs_reduce_noalloc_kernel, tide::kThreads, 0) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return TIDE_ERR_CUDA;
    int64_t grid = (int64_t)per_sm * sms;
    if (max_ctas > 0 && grid > max_ctas) grid = max_ctas;
    if (grid > n_tiles) grid = n_tiles;
    if (grid < 1) grid = 1;

    NaArgs a;
    a.scratch = scratch;
    a.n_params = n_params;
    a.world = world;
    a.shard_numel = Ns;
    a.n_tiles = n_tiles;
    a.out = out;
    a.out_numel = out_numel;
    a.scale = 1.0f / (float)world;
    a.do_scale = scale_mode == TIDE_SCALE_INV_WORLD ? 1 : 0;
    (void)cudaGetLastError();  // drop an error left by an earlier failed runtime call
    rs_reduce_noalloc_kernel<<<(unsigned)grid, tide::kThreads, 0, s>>>(a);
    return cudaGetLastError() == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}
