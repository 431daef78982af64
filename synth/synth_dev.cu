// synth_dev.cu - device twin of synth.c: the same seeded bf16 values, written
// straight into device buffers so that multi-GB workloads need no host pass.
// The recipe (and its provenance) is documented in synth.c; this file must stay
// bit-identical to it, which the generator tests check on sampled indices.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint64_t sm64(uint64_t x) {
    uint64_t z = x + 0x9e3779b97f4a7c15ULL;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

__device__ __forceinline__ uint16_t value_at(uint64_t key, uint64_t idx, float mul) {
    uint64_t h = sm64(key ^ idx);
    int32_t s = (int32_t)(h & 0xffff) + (int32_t)((h >> 16) & 0xffff) +
                (int32_t)((h >> 32) & 0xffff) + (int32_t)(h >> 48) - 131070;
    float x = __fmul_rn((float)s, mul);
    uint32_t u = __float_as_uint(x);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

__global__ void fill_kernel(uint16_t* __restrict__ out, int64_t n, uint64_t idx0,
                            uint64_t key, float mul) {
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += stride)
        out[j] = value_at(key, idx0 + (uint64_t)j, mul);
}

}  // namespace

extern "C" uint64_t synth_dev_key(uint64_t seed, uint64_t stream, uint64_t rank, uint64_t param) {
    auto h = [](uint64_t x) {
        uint64_t z = x + 0x9e3779b97f4a7c15ULL;
        z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
        z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
        return z ^ (z >> 31);
    };
    return h(h(seed) ^ ((stream << 48) ^ (rank << 32) ^ param));
}

// Fill a device buffer; returns a cudaError_t value (0 = success).
extern "C" int synth_dev_fill_bf16(void* out, int64_t n, uint64_t idx0, uint64_t seed,
                                   uint64_t stream, uint64_t rank, uint64_t param,
                                   float mul, void* cuda_stream) {
    if (n <= 0) return 0;
    if (out == nullptr) return (int)cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (n + 255) / 256;
    int64_t cap = (int64_t)sms * 8;
    if (blocks > cap) blocks = cap;
    uint64_t key = synth_dev_key(seed, stream, rank, param);
    fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)cuda_stream>>>(
        (uint16_t*)out, n, idx0, key, mul);
    return (int)cudaGetLastError();
}
