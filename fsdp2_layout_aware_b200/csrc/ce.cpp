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
//
// The copies are spread over kFanout plan-owned streams (forked from the
// caller's stream with an event and joined back before the call returns), so
// that several copy engines work at once: on one stream the copies run one
// after another, which holds them to about half of HBM bandwidth.
//
// Issuing a copy costs the host about 3 us, which bounds the calls on groups of
// many small parameters.  So the first placement call with a given set of
// buffers (outside any stream capture) records its copies once as a CUDA graph,
// on a private stream, and every call with the same buffers launches that graph
// on the caller's stream: one launch instead of hundreds of copy calls.  A call
// on a stream that is being captured issues its copies directly, into the
// caller's capture.  Measured on B200 against direct issue (TB/s): placement
// 6.55 / 3.29 / 3.72 against 6.27 / 3.25 / 3.68 on the 70B / Qwen3 / Wan2.2
// groups; placement from per-rank shards (one copy per chunk) 6.48 / 1.90 /
// 4.55 against 6.12 / 0.70 / 2.60.  Slot-Reuse staging stays on direct issue
// (see ce_slot_stage).
#include <algorithm>
#include <condition_variable>
#include <functional>
#include <mutex>
#include <thread>

#include "tide_internal.h"

// Host threads that issue the copies of one call, the caller included.  On
// groups of many small parameters the calls are bound by the host's cost per
// copy call (about 3 us), not by the copy engines, and the CUDA runtime takes
// calls on different streams from several threads at once.  Measured on B200
// (ms, 1 / 4 / 8 threads): Qwen3 group, AG placement 1.39 / 0.76 / 0.76, slot
// staging 10.6 / 5.96 / 5.95; the 70B and Wan2.2 groups, whose copies are few
// and large, within 1 %.
constexpr int kIssueThreads = 4;

// One planned copy-engine operation.
struct CeOp {
    enum Kind { kRows, kMemset } kind;
    void* dst;
    size_t dpitch;
    const void* src;
    size_t spitch;
    size_t width;   // bytes per row (kMemset: bytes to clear)
    int64_t rows;
};

// Persistent worker threads: run() executes job(t) for t = 0..n-1, t = 0 on the
// calling thread, and returns when all have finished.
struct CeIssuer {
    int device = 0;
    std::vector<std::thread> threads;
    std::mutex mu;
    std::condition_variable start_cv, done_cv;
    const std::function<void(int)>* job = nullptr;
    uint64_t generation = 0;
    int pending = 0;
    bool stop = false;
    std::vector<std::vector<CeOp>> lists;  // per fan-out stream, reused across calls

    int size() const { return (int)threads.size() + 1; }

    void worker(int idx) {
        cudaSetDevice(device);
        uint64_t seen = 0;
        std::unique_lock<std::mutex> lk(mu);
        while (true) {
            start_cv.wait(lk, [&] { return stop || generation != seen; });
            if (stop) return;
            seen = generation;
            const std::function<void(int)>* f = job;
            lk.unlock();
            (*f)(idx);
            lk.lock();
            if (--pending == 0) done_cv.notify_all();
        }
    }

    void run(const std::function<void(int)>& f) {
        {
            std::lock_guard<std::mutex> lk(mu);
            job = &f;
            pending = (int)threads.size();
            ++generation;
        }
        start_cv.notify_all();
        f(0);
        std::unique_lock<std::mutex> lk(mu);
        done_cv.wait(lk, [&] { return pending == 0; });
    }

    ~CeIssuer() {
        {
            std::lock_guard<std::mutex> lk(mu);
            stop = true;
        }
        start_cv.notify_all();
        for (auto& t : threads) t.join();
    }
};

namespace tide {
namespace {

// Rows at least this wide go as one 1-D copy each.  Measured on B200: 2-D
// device-to-device copies stay near 3.4 TB/s whatever the number of streams,
// while 1-D copies on several streams reach HBM bandwidth; below a few MB a row,
// the fixed cost of each extra copy call (about 3 us) outweighs that.  Staging
// for Slot-Reuse (70B / Qwen3 / Wan2.2 groups, ms): all 2-D 7.72 / 10.78 / 6.63;
// split from 256 KB 4.31 / 79.4 / 10.9; from 1 MB 4.31 / 11.3 / 11.1; from
// 4 MB 4.38 / 10.8 / 5.57.
constexpr size_t kRowSplitBytes = size_t(4) << 20;

// Copy `rows` rows of `width` bytes: one 2-D copy, or one 1-D copy per row when
// the rows are wide or a pitch exceeds the device limit.
cudaError_t copy_rows(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width,
                      int64_t rows, size_t max_pitch, cudaStream_t stream) {
    if (rows <= 0 || width == 0) return cudaSuccess;
    if (rows == 1) return cudaMemcpyAsync(dst, src, width, cudaMemcpyDeviceToDevice, stream);
    if (dpitch <= max_pitch && spitch <= max_pitch && width < kRowSplitBytes)
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

// Measured on B200 (AG placement, 70B / Qwen3 / Wan2.2 groups, TB/s): one
// stream 3.41 / 1.03 / 2.68; 2 streams 3.32 / 1.79 / 2.96; 4: 3.32 / 1.81 / 3.10;
// 8: 6.32 / 1.69 / 3.07; 16: 6.29 / 1.65 / 2.23.  Large parameters are cut by
// ranks over the streams, so with 8 streams each rank row of a big parameter is
// one 1-D copy on its own stream.
constexpr int kFanout = 8;

// Create the fan-out streams and events once, then make them wait for
// everything enqueued on `s` so far.
cudaError_t fork(tide_plan* p, cudaStream_t s) {
    while ((int)p->ce_streams.size() < kFanout) {
        cudaStream_t st = nullptr;
        cudaError_t e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
        if (e != cudaSuccess) return e;
        p->ce_streams.push_back(st);
    }
    while ((int)p->ce_events.size() < kFanout + 1) {
        cudaEvent_t ev = nullptr;
        cudaError_t e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
        p->ce_events.push_back(ev);
    }
    cudaError_t e = cudaEventRecord(p->ce_events[0], s);
    for (int j = 0; e == cudaSuccess && j < kFanout; ++j)
        e = cudaStreamWaitEvent(p->ce_streams[j], p->ce_events[0], 0);
    return e;
}

// Make `s` wait for everything enqueued on the fan-out streams.
cudaError_t join(tide_plan* p, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    for (int j = 0; e == cudaSuccess && j < kFanout; ++j) {
        e = cudaEventRecord(p->ce_events[1 + j], p->ce_streams[j]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, p->ce_events[1 + j], 0);
    }
    return e;
}

// Parameters below this size go whole to one stream; larger ones are cut by ranks.
constexpr int64_t kSplitBytes = 8 << 20;

// The plan's issuer, created on first use with kIssueThreads - 1 worker
// threads (fewer if the system refuses more); nullptr only if even the empty
// issuer cannot be allocated.
CeIssuer* issuer(tide_plan* p) {
    if (p->ce_issuer != nullptr) return p->ce_issuer;
    CeIssuer* q = new (std::nothrow) CeIssuer;
    if (q == nullptr) return nullptr;
    q->device = p->device;
    q->lists.resize(kFanout);
    for (int t = 1; t < kIssueThreads; ++t) {
        try {
            q->threads.emplace_back(&CeIssuer::worker, q, t);
        } catch (...) {
            break;  // run with the threads that started
        }
    }
    p->ce_issuer = q;
    return q;
}

cudaError_t issue(const CeOp& op, size_t max_pitch, cudaStream_t st) {
    if (op.kind == CeOp::kMemset) return cudaMemsetAsync(op.dst, 0, op.width, st);
    return copy_rows(op.dst, op.dpitch, op.src, op.spitch, op.width, op.rows, max_pitch, st);
}

// Issue every planned list on its fan-out stream, the lists spread over the
// issuer's threads (list j on thread j mod threads); the first error wins.
cudaError_t issue_all(tide_plan* p, CeIssuer* q, size_t max_pitch) {
    const int n = q->size();
    std::vector<cudaError_t> err(n, cudaSuccess);
    const std::function<void(int)> job = [&](int t) {
        for (int j = t; j < kFanout; j += n) {
            for (const CeOp& op : q->lists[j]) {
                cudaError_t e = issue(op, max_pitch, p->ce_streams[j]);
                if (e != cudaSuccess) {
                    err[t] = e;
                    return;
                }
            }
        }
    };
    if (n == 1) job(0);
    else q->run(job);
    for (cudaError_t e : err)
        if (e != cudaSuccess) return e;
    return cudaSuccess;
}

CeOp rows_op(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width, int64_t rows) {
    return CeOp{CeOp::kRows, dst, dpitch, src, spitch, width, rows};
}

// Recorded graphs kept per plan (the least recently used one is replaced).
constexpr size_t kMaxCeGraphs = 4;

enum { kCallPlace = 1, kCallGather = 2, kCallStage = 3, kCallRankStage = 4, kCallStageF32 = 5 };

// Issue the planned lists (q->lists) as one call on `stream`: replay the graph
// recorded for (kind, j0, j1, key) if there is one, else record it now and
// replay it; if the stream is being captured, or recording fails, fork, issue
// and join directly on `stream`.  `plan` fills q->lists; it runs only when the
// copies are issued or recorded.
cudaError_t run_call(tide_plan* p, cudaStream_t stream, int kind, int64_t j0, int64_t j1,
                     std::vector<const void*>&& key, bool record,
                     const std::function<void(CeIssuer*)>& plan) {
    CeIssuer* q = issuer(p);
    if (q == nullptr) return cudaErrorMemoryAllocation;
    const size_t max_pitch = device_max_pitch(p->device);
    cudaStreamCaptureStatus capturing = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &capturing) != cudaSuccess) {
        (void)cudaGetLastError();
        capturing = cudaStreamCaptureStatusActive;  // treat as captured: issue directly
    }
    if (record && capturing == cudaStreamCaptureStatusNone) {
        for (auto& g : p->ce_graphs) {
            if (g.kind == kind && g.j0 == j0 && g.j1 == j1 && g.key == key) {
                g.last_use = ++p->ce_clock;
                return cudaGraphLaunch(g.exec, stream);
            }
        }
        // record the call on the private stream: fork, issue, join, as below
        bool ok = p->ce_capture_stream != nullptr ||
                  cudaStreamCreateWithFlags(&p->ce_capture_stream, cudaStreamNonBlocking) == cudaSuccess;
        cudaGraph_t graph = nullptr;
        cudaGraphExec_t exec = nullptr;
        if (ok) {
            for (auto& l : q->lists) l.clear();
            plan(q);
            cudaStream_t cap = p->ce_capture_stream;
            ok = cudaStreamBeginCapture(cap, cudaStreamCaptureModeRelaxed) == cudaSuccess;
            if (ok) {
                cudaError_t e = fork(p, cap);
                if (e == cudaSuccess) e = issue_all(p, q, max_pitch);
                cudaError_t j = join(p, cap);
                cudaError_t end = cudaStreamEndCapture(cap, &graph);  // ends the capture in every case
                ok = e == cudaSuccess && j == cudaSuccess && end == cudaSuccess && graph != nullptr &&
                     cudaGraphInstantiate(&exec, graph, 0) == cudaSuccess;
                if (graph != nullptr) cudaGraphDestroy(graph);
            }
        }
        if (ok) {
            if (p->ce_graphs.size() >= kMaxCeGraphs) {
                auto lru = std::min_element(p->ce_graphs.begin(), p->ce_graphs.end(),
                                            [](const tide_plan::CeGraph& a, const tide_plan::CeGraph& b) {
                                                return a.last_use < b.last_use;
                                            });
                cudaGraphExecDestroy(lru->exec);
                p->ce_graphs.erase(lru);
            }
            tide_plan::CeGraph g;
            g.kind = kind;
            g.j0 = j0;
            g.j1 = j1;
            g.key = std::move(key);
            g.exec = exec;
            g.last_use = ++p->ce_clock;
            p->ce_graphs.push_back(std::move(g));
            return cudaGraphLaunch(exec, stream);
        }
        if (exec != nullptr) cudaGraphExecDestroy(exec);
        (void)cudaGetLastError();  // fall back to issuing the copies directly
    }
    for (auto& l : q->lists) l.clear();
    plan(q);
    cudaError_t e = fork(p, stream);
    if (e != cudaSuccess) return e;
    e = issue_all(p, q, max_pitch);
    cudaError_t j = join(p, stream);
    return e != cudaSuccess ? e : j;
}

}  // namespace

cudaError_t ce_ag_place(tide_plan* p, const uint16_t* ag, void* const* params, cudaStream_t stream) {
    const int64_t W = p->world, Ns = p->shard_numel;
    std::vector<const void*> key;
    key.reserve((size_t)p->n_params + 1);
    key.push_back(ag);
    for (int32_t i = 0; i < p->n_params; ++i) key.push_back(params[i]);
    return run_call(p, stream, kCallPlace, 0, 0, std::move(key), true, [&](CeIssuer* q) {
        int next = 0;  // round-robin over the fan-out streams for whole (small) params
        for (int32_t i = 0; i < p->n_params; ++i) {
            const int64_t c = p->chunk[i], n = p->numel[i];
            if (c == 0) continue;
            uint16_t* dst = static_cast<uint16_t*>(params[i]);
            const uint16_t* src = ag + p->offset[i];
            const int64_t full = std::min(W, n / c);
            // ranks [0, full) hold whole chunks: one 2-D copy, cut by ranks over the streams if large
            const int parts = (2 * n >= kSplitBytes) ? (int)std::min<int64_t>(kFanout, full) : 1;
            for (int j = 0; j < parts; ++j) {
                const int64_t r0 = full * j / parts, r1 = full * (j + 1) / parts;
                if (r1 > r0)
                    q->lists[(next + j) % kFanout].push_back(
                        rows_op(dst + r0 * c, 2 * c, src + r0 * Ns, 2 * Ns, 2 * c, r1 - r0));
            }
            auto& l = q->lists[next % kFanout];
            next = (next + parts) % kFanout;
            const int64_t rem = n - full * c;
            if (rem > 0 && full < W) l.push_back(rows_op(dst + full * c, 0, src + full * Ns, 0, 2 * rem, 1));
            if (W * c > n)
                l.push_back(CeOp{CeOp::kMemset, dst + n, 0, nullptr, 0, (size_t)(2 * (W * c - n)), 0});
        }
    });
}

// Gathering placement: rank r's chunk of param i comes from rank r's own shard
// (shards[r] + off_i), one 1-D copy per chunk with data, on the fan-out stream
// of its source rank; each param's pad tail is one memset.
cudaError_t ce_ag_gather(tide_plan* p, const void* const* shards, void* const* params,
                         cudaStream_t stream) {
    const int64_t W = p->world;
    std::vector<const void*> key;
    key.reserve((size_t)(W + p->n_params));
    for (int64_t r = 0; r < W; ++r) key.push_back(shards[r]);
    for (int32_t i = 0; i < p->n_params; ++i) key.push_back(params[i]);
    return run_call(p, stream, kCallGather, 0, 0, std::move(key), true, [&](CeIssuer* q) {
        for (int32_t i = 0; i < p->n_params; ++i) {
            const int64_t c = p->chunk[i], n = p->numel[i];
            if (c == 0) continue;
            uint16_t* dst = static_cast<uint16_t*>(params[i]);
            for (int64_t r = 0; r < W; ++r) {
                const int64_t valid = std::min(c, std::max<int64_t>(0, n - r * c));
                if (valid == 0) break;  // later ranks hold only pad rows
                const uint16_t* src = static_cast<const uint16_t*>(shards[r]) + p->offset[i];
                q->lists[r % kFanout].push_back(rows_op(dst + r * c, 0, src, 0, 2 * valid, 1));
            }
            if (W * c > n)
                q->lists[i % kFanout].push_back(
                    CeOp{CeOp::kMemset, dst + n, 0, nullptr, 0, (size_t)(2 * (W * c - n)), 0});
        }
    });
}

// Stage the chunks [j0, j1) (chunk i*W + r: rank r's rows of param i) from
// every source rank k into slot k.  Within one param the chunks of a range are
// consecutive ranks, so each (k, param) pair takes one 2-D copy plus at most
// one 1-D copy for a partial chunk.  esize: bytes per element (2 for bf16
// gradients and slots, 4 for fp32).
cudaError_t ce_slot_stage(tide_plan* p, const void* const* grads, void* const* slots,
                          cudaStream_t caller, int64_t j0, int64_t j1, bool record, bool one_source,
                          int esize) {
    const int64_t W = p->world, P = p->n_params, Ns = p->shard_numel, e = esize;
    const int64_t sources = one_source ? 1 : W;
    if (j1 < 0) j1 = P * W;
    if (j1 <= j0) return cudaSuccess;
    std::vector<const void*> key;
    if (record) {
        key.reserve((size_t)(sources * P + sources + 1));
        for (int64_t j = 0; j < sources * P; ++j) key.push_back(grads[j]);
        for (int64_t k = 0; k < sources; ++k) key.push_back(slots[k]);
        key.push_back(reinterpret_cast<const void*>(sources));
    }
    const int kind = esize == 4 ? kCallStageF32 : kCallStage;
    return run_call(p, caller, kind, j0, j1, std::move(key), record, [&](CeIssuer* q) {
        for (int64_t k = 0; k < sources; ++k) {
            char* slot = static_cast<char*>(slots[k]);
            for (int64_t i = j0 / W; i <= (j1 - 1) / W; ++i) {
                // one source rank per stream at a time; one rank's params spread over the streams
                auto& l = q->lists[(one_source ? i : k) % kFanout];
                const int64_t c = p->chunk[i], n = p->numel[i];
                if (c == 0 || n == 0) continue;
                const int64_t r0 = std::max<int64_t>(0, j0 - i * W), r1 = std::min<int64_t>(W, j1 - i * W);
                const char* g = static_cast<const char*>(grads[k * P + i]);
                char* dst = slot + e * p->offset[i];
                const int64_t full = std::min(W, n / c);  // ranks [0, full) hold whole chunks
                const int64_t fr1 = std::min(full, r1);
                if (fr1 > r0)
                    l.push_back(rows_op(dst + e * r0 * Ns, e * Ns, g + e * r0 * c, e * c, e * c, fr1 - r0));
                const int64_t rem = n - full * c;       // rank `full` holds a partial chunk
                if (rem > 0 && full < W && full >= r0 && full < r1)
                    l.push_back(rows_op(dst + e * full * Ns, 0, g + e * full * c, 0, e * rem, 1));
            }
        }
    });
}

// One rank's Slot-Reuse phase 1 (a one-rank plan, rank r): for the chunks
// [j0, j1) that are rank r's (chunk i*W + r), chunk r of every source rank k's
// gradient of param i goes to slots[k] + off_i, one 1-D copy per (k, i) with
// data, on the fan-out stream of the source rank.  The sources may be peers'
// memory, so the copy engines carry the transfer.
cudaError_t ce_rank_stage(tide_plan* p, const void* const* grads, void* const* slots,
                          cudaStream_t caller, int64_t j0, int64_t j1) {
    const int64_t W = p->world, P = p->n_params, r = p->rank;
    return run_call(p, caller, kCallRankStage, j0, j1, {}, false, [&](CeIssuer* q) {
        for (int64_t i = j0 / W; i < P && i * W + r < j1; ++i) {
            if (i * W + r < j0) continue;
            const int64_t c = p->chunk[i];
            const int64_t valid = std::min(c, std::max<int64_t>(0, p->numel[i] - r * c));
            if (valid == 0) continue;
            for (int64_t k = 0; k < W; ++k) {
                const uint16_t* g = static_cast<const uint16_t*>(grads[k * P + i]) + r * c;
                uint16_t* dst = static_cast<uint16_t*>(slots[k]) + p->offset[i];
                q->lists[k % kFanout].push_back(rows_op(dst, 0, g, 0, 2 * valid, 1));
            }
        }
    });
}

void ce_release(tide_plan* p) {
    delete p->ce_issuer;
    p->ce_issuer = nullptr;
    for (auto& g : p->ce_graphs) cudaGraphExecDestroy(g.exec);
    p->ce_graphs.clear();
    if (p->ce_capture_stream != nullptr) cudaStreamDestroy(p->ce_capture_stream);
    p->ce_capture_stream = nullptr;
}

}  // namespace tide
