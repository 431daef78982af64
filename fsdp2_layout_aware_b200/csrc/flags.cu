// flags.cu - ordering between ranks on the device, with bounded waits.
//
// Across GPUs a rank's reduction may read a peer's gradients only once the
// peer has written them, and a rank may overwrite its buffers only once every
// peer has read them (weekinpapers.com, Abstract: the collectives read peers'
// buffers in place).  The host can order this with barriers; these two calls
// order it on the device instead, stream-ordered, without a host round trip:
//   - tide_flag_signal: one thread makes every earlier write of this device
//     visible system-wide, then stores `value` into a flag (its own memory or a
//     peer's, mapped through CUDA IPC) with release semantics;
//   - tide_flag_wait: one CTA polls n flags with acquire loads until each holds
//     `value` or later (epoch arithmetic modulo 2^32), then writes a status
//     word: 0, or 1 + the index of the first flag that did not get there in
//     time.  Every poll loop ends: at the time limit (globaltimer) and, as a
//     second bound, after an iteration cap.  Work queued after the wait on
//     the same stream starts when it ends, so the caller checks the status
//     before trusting what that work read.
#include <climits>
#include <cstdint>

#include "tide_internal.h"
#include "tma.cuh"

namespace {

constexpr int kWaitThreads = 256;
constexpr int64_t kMaxTimeoutNs = 60ll * 1000 * 1000 * 1000;
constexpr uint32_t kPollSleepNs = 200;

struct WaitArgs {
    const uint32_t* flags[TIDE_MAX_WORLD];
    int32_t n;
    uint32_t value;
    uint64_t timeout_ns;
    uint64_t max_polls;
    int32_t* status;
};

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__global__ void flag_signal_kernel(uint32_t* flag, uint32_t value) {
    __threadfence_system();
    asm volatile("st.release.sys.global.u32 [%0], %1;" : : "l"(flag), "r"(value) : "memory");
}

__global__ void __launch_bounds__(kWaitThreads) flag_wait_kernel(const WaitArgs a) {
    __shared__ int first_late;
    if (threadIdx.x == 0) first_late = INT_MAX;
    __syncthreads();
    const uint64_t t0 = tide::global_ns();
    for (int k = threadIdx.x; k < a.n; k += kWaitThreads) {
        bool reached = false;
        for (uint64_t polls = 0; polls < a.max_polls; ++polls) {
            if ((int32_t)(ld_acquire_sys(a.flags[k]) - a.value) >= 0) {
                reached = true;
                break;
            }
            if (tide::global_ns() - t0 > a.timeout_ns) break;
            __nanosleep(kPollSleepNs);
        }
        if (!reached) atomicMin(&first_late, k);
    }
    __syncthreads();
    if (threadIdx.x == 0) *a.status = first_late == INT_MAX ? 0 : first_late + 1;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

}  // namespace

extern "C" tide_status_t tide_flag_signal(void* flag, uint32_t value, void* stream) {
    if (flag == nullptr) return TIDE_ERR_INVALID_ARG;
    if (!aligned4(flag)) return TIDE_ERR_ALIGNMENT;
    (void)cudaGetLastError();  // drop an error left by an earlier failed runtime call
    flag_signal_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(flag), value);
    return cudaGetLastError() == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}

extern "C" tide_status_t tide_flag_wait(const void* const* flags, int32_t n, uint32_t value,
                                        int64_t timeout_ns, int32_t* status, void* stream) {
    if (flags == nullptr || status == nullptr || n < 1 || n > TIDE_MAX_WORLD) return TIDE_ERR_INVALID_ARG;
    if (timeout_ns <= 0 || timeout_ns > kMaxTimeoutNs) return TIDE_ERR_INVALID_ARG;
    if (!aligned4(status)) return TIDE_ERR_ALIGNMENT;
    WaitArgs a;
    for (int32_t k = 0; k < n; ++k) {
        if (flags[k] == nullptr) return TIDE_ERR_INVALID_ARG;
        if (!aligned4(flags[k])) return TIDE_ERR_ALIGNMENT;
        a.flags[k] = static_cast<const uint32_t*>(flags[k]);
    }
    a.n = n;
    a.value = value;
    a.timeout_ns = (uint64_t)timeout_ns;
    // the second bound: a poll (a system-scope acquire load, then a sleep that may be
    // shorter than asked) takes well over 16 ns, so this many polls outlast the time limit
    a.max_polls = (uint64_t)timeout_ns / 16 + 1000;
    a.status = status;
    (void)cudaGetLastError();
    flag_wait_kernel<<<1, kWaitThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return cudaGetLastError() == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}
