// api.cpp - the launch entry points of libtide.so: host-side validation,
// pointer-table upload and dispatch to the kernels or the copy engines.
//
// Every check runs before anything is enqueued, so an error status means the
// stream is untouched.  Checks: plan usable on the current device, enum
// values, null pointers (a NULL buffer is accepted only where it would hold
// zero elements), element alignment, buffer sizes against the plan, and
// overlap between any written buffer and any other buffer of the call.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "tide_internal.h"

namespace {

// An NVTX range over one API call, named after it, for Nsight Systems
// timelines (with no tool attached it costs a check of a function pointer).
struct ApiRange {
    explicit ApiRange(const char* name) { nvtxRangePushA(name); }
    ~ApiRange() { nvtxRangePop(); }
    ApiRange(const ApiRange&) = delete;
    ApiRange& operator=(const ApiRange&) = delete;
};

struct Span {
    uintptr_t lo, hi;
    bool write;
};

// True if a written span overlaps any other span (read spans may overlap each other).
bool overlaps(std::vector<Span>& spans) {
    size_t n_write = 0;
    for (const Span& s : spans) n_write += (s.write && s.lo != s.hi) ? 1 : 0;
    if (n_write <= 16) {
        // few written spans (one output, or a few slots): test each against every span
        for (size_t i = 0; i < spans.size(); ++i) {
            const Span& w = spans[i];
            if (!w.write || w.lo == w.hi) continue;
            for (size_t j = 0; j < spans.size(); ++j) {
                const Span& o = spans[j];
                if (j != i && o.lo != o.hi && o.lo < w.hi && w.lo < o.hi) return true;
            }
        }
        return false;
    }
    std::sort(spans.begin(), spans.end(), [](const Span& a, const Span& b) { return a.lo < b.lo; });
    uintptr_t max_hi = 0, max_hi_write = 0;
    for (const Span& s : spans) {
        if (s.lo == s.hi) continue;
        if (s.lo < max_hi_write) return true;
        if (s.write && s.lo < max_hi) return true;
        max_hi = std::max(max_hi, s.hi);
        if (s.write) max_hi_write = std::max(max_hi_write, s.hi);
    }
    return false;
}

void add_span(std::vector<Span>& v, const void* p, int64_t bytes, bool write) {
    if (p == nullptr || bytes <= 0) return;
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    v.push_back({lo, lo + (uintptr_t)bytes, write});
}

// A host-only plan passes here (so that argument validation can run without a
// GPU) and is refused by `launchable` once the arguments have been checked.
tide_status_t check_plan(const tide_plan* p) {
    if (p == nullptr) return TIDE_ERR_INVALID_ARG;
    if (p->flags & TIDE_PLAN_HOST_ONLY) return TIDE_OK;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return TIDE_ERR_CUDA;
    if (cur != p->device) return TIDE_ERR_DEVICE;
    return TIDE_OK;
}

tide_status_t launchable(const tide_plan* p) {
    return (p->flags & TIDE_PLAN_HOST_ONLY) ? TIDE_ERR_DEVICE : TIDE_OK;
}

// Calls that need every rank's tiles refuse a one-rank plan.
tide_status_t all_ranks(const tide_plan* p) { return p->rank >= 0 ? TIDE_ERR_INVALID_ARG : TIDE_OK; }

// A device buffer of `need` elements of size `esize` at `ptr` with `have` elements.
tide_status_t check_buf(const void* ptr, int64_t have, int64_t need, int esize) {
    if (need == 0) return TIDE_OK;
    if (ptr == nullptr) return TIDE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(ptr) % (uintptr_t)esize != 0) return TIDE_ERR_ALIGNMENT;
    if (have < need) return TIDE_ERR_SIZE;
    return TIDE_OK;
}

tide_status_t check_grads(const tide_plan* p, const void* const* grads, const int64_t* grad_numel,
                          std::vector<Span>& spans) {
    const int64_t W = p->world, P = p->n_params;
    if (W * P > 0 && (grads == nullptr || grad_numel == nullptr)) return TIDE_ERR_INVALID_ARG;
    for (int64_t k = 0; k < W; ++k)
        for (int64_t i = 0; i < P; ++i) {
            const int64_t j = k * P + i;
            tide_status_t st = check_buf(grads[j], grad_numel[j], p->numel[i], 2);
            if (st != TIDE_OK) return st;
            add_span(spans, grads[j], 2 * p->numel[i], false);
        }
    return TIDE_OK;
}

tide_status_t check_slots(const tide_plan* p, void* const* slots, int64_t slot_numel,
                          std::vector<Span>& spans) {
    const int64_t W = p->world, need = W * p->shard_numel;
    if (slots == nullptr) return TIDE_ERR_INVALID_ARG;
    for (int64_t k = 0; k < W; ++k) {
        tide_status_t st = check_buf(slots[k], slot_numel, need, 2);
        if (st != TIDE_OK) return st;
        add_span(spans, slots[k], 2 * need, true);
    }
    return TIDE_OK;
}

tide_status_t check_enums(const tide_plan* p, int32_t engine, int32_t max_ctas) {
    if (engine != TIDE_ENGINE_SM && engine != TIDE_ENGINE_CE) return TIDE_ERR_INVALID_ARG;
    if (max_ctas < 0) return TIDE_ERR_INVALID_ARG;
    // short-lived CTAs: one per unit of work, so no cap on the grid
    if ((p->flags & TIDE_PLAN_SHORT_CTAS) && max_ctas != 0) return TIDE_ERR_INVALID_ARG;
    return TIDE_OK;
}

tide_status_t check_reduce_modes(int32_t scale_mode, int32_t order) {
    if (scale_mode != TIDE_SCALE_NONE && scale_mode != TIDE_SCALE_INV_WORLD) return TIDE_ERR_INVALID_ARG;
    if (order != TIDE_ORDER_RANK && order != TIDE_ORDER_TREE) return TIDE_ERR_INVALID_ARG;
    return TIDE_OK;
}

// Upload a pointer table unless the device copy already holds these pointers.
tide_status_t sync_table(PtrTable& t, const void* const* ptrs, int64_t n, cudaStream_t stream) {
    if (n == 0) return TIDE_OK;
    if (n > t.capacity || t.dev == nullptr) return TIDE_ERR_INVALID_ARG;
    if (t.valid && (int64_t)t.host.size() == n &&
        std::memcmp(t.host.data(), ptrs, sizeof(void*) * (size_t)n) == 0)
        return TIDE_OK;
    t.host.assign(ptrs, ptrs + n);
    t.aligned16 = t.aligned32 = true;
    for (int64_t j = 0; j < n; ++j) {
        if ((reinterpret_cast<uintptr_t>(ptrs[j]) & 15) != 0) t.aligned16 = false;
        if ((reinterpret_cast<uintptr_t>(ptrs[j]) & 31) != 0) t.aligned32 = false;
    }
    // Pageable source: the runtime stages it before returning, so the host
    // mirror may change afterwards; the device copy is stream-ordered.
    cudaError_t e = cudaMemcpyAsync(t.dev, t.host.data(), sizeof(void*) * (size_t)n,
                                    cudaMemcpyHostToDevice, stream);
    t.valid = (e == cudaSuccess);
    return e == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}

int grid_for(const tide_plan* p, int kernel, int32_t max_ctas) {
    int32_t g = 0;
    tide_launch_ctas(p, kernel, max_ctas, &g);
    return g;
}

float inv_world(int32_t world) { return 1.0f / (float)world; }

// The bulk-copy (TMA) reduction runs when the plan asks for it and every tile
// starts on an 8-element boundary with 16-byte aligned sources and output;
// otherwise the load/store kernel runs.
bool use_tma(const tide_plan* p, const PtrTable& src, const float* out, int kernel) {
    return (p->flags & TIDE_PLAN_TMA) && p->tiles_aligned8 && p->blocks_per_sm[kernel] > 0 &&
           src.aligned16 && (reinterpret_cast<uintptr_t>(out) & 15) == 0;
}

// The 32-byte load/store variant needs 32-byte aligned sources and output at
// every tile: 16-element tile offsets plus 32-byte aligned base pointers.
bool use_v32(const tide_plan* p, const PtrTable& src, const float* out, int kernel) {
    return p->tiles_aligned16 && p->blocks_per_sm[kernel] > 0 && src.aligned32 &&
           (reinterpret_cast<uintptr_t>(out) & 31) == 0;
}

// Launch the reduction over `tab` on the chosen kernel, for the plan's tiles
// [t0, t1) (t1 < 0: all), and record it in the plan.
cudaError_t launch_reduce(tide_plan* p, PtrTable& tab, bool slot, int64_t bound, float* out,
                          int64_t out_numel, int32_t scale_mode, int32_t order, int32_t max_ctas,
                          cudaStream_t s, int64_t t0 = 0, int64_t t1 = -1) {
    const bool tree = order == TIDE_ORDER_TREE;
    const int k_tma = slot ? K_SLOT_RS_TMA : K_RS_TMA;
    const int k_v32 = tree ? (slot ? K_SLOT_RS_TREE_V32 : K_RS_TREE_V32) : (slot ? K_SLOT_RS_V32 : K_RS_V32);
    const bool tma = use_tma(p, tab, out, k_tma);
    const bool v32 = !tma && use_v32(p, tab, out, k_v32);
    const int kernel = tma ? k_tma : v32 ? k_v32 : tree ? (slot ? K_SLOT_RS_TREE : K_RS_TREE)
                                                        : (slot ? K_SLOT_RS : K_RS);
    if (t1 < 0) t1 = (int64_t)p->tiles.size();
    const int grid = (int)std::min<int64_t>(grid_for(p, kernel, max_ctas), t1 - t0);
    p->last_kernel = kernel;
    p->last_ctas = grid;
    const float scale = inv_world(p->world);
    const bool do_scale = scale_mode == TIDE_SCALE_INV_WORLD;
    return tma ? tide::launch_rs_reduce_tma(p, tab.dev, slot, bound, out, out_numel, scale, do_scale,
                                            order, grid, s, t0, t1)
               : tide::launch_rs_reduce(p, tab.dev, slot, bound, out, out_numel, scale, do_scale,
                                        order, grid, s, v32, t0, t1);
}

tide_status_t stage_impl(tide_plan* p, const void* const* grads, void* const* slots,
                         int64_t slot_numel, int32_t engine, int32_t max_ctas, cudaStream_t s) {
    if (p->tiles.empty()) return TIDE_OK;
    cudaError_t e;
    if (engine == TIDE_ENGINE_CE) {
        p->last_kernel = -1;
        p->last_ctas = 0;
        e = tide::ce_slot_stage(p, grads, slots, s);
    } else {
        tide_status_t st = sync_table(p->grad_tab, grads, (int64_t)p->world * p->n_params, s);
        if (st == TIDE_OK)
            st = sync_table(p->slot_tab, const_cast<const void* const*>(slots), p->world, s);
        if (st != TIDE_OK) return st;
        p->last_kernel = K_STAGE;
        p->last_ctas = grid_for(p, K_STAGE, max_ctas);
        e = tide::launch_slot_stage(p, p->grad_tab.dev, p->slot_tab.dev, slot_numel, p->last_ctas, s,
                                    p->world);
    }
    return e == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}

tide_status_t reduce_slots_impl(tide_plan* p, void* const* slots, int64_t slot_numel, float* out,
                                int64_t out_numel, int32_t scale_mode, int32_t order,
                                int32_t max_ctas, cudaStream_t s) {
    if (p->tiles.empty()) return TIDE_OK;
    // A one-rank plan's tiles address its shard from 0; its rows of every slot start at
    // rank * Ns, so the kernel gets each slot from there on.
    const int64_t row0 = p->rank >= 0 ? (int64_t)p->rank * p->shard_numel : 0;
    std::vector<const void*> from((size_t)p->world);
    for (int64_t k = 0; k < p->world; ++k) from[k] = static_cast<const uint16_t*>(slots[k]) + row0;
    tide_status_t st = sync_table(p->slot_tab, from.data(), p->world, s);
    if (st != TIDE_OK) return st;
    cudaError_t e = launch_reduce(p, p->slot_tab, true, slot_numel - row0, out, out_numel, scale_mode,
                                  order, max_ctas, s);
    return e == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}

// Cut the chunks, in tile order (chunk i*W + r), into n contiguous segments
// that hold about equal numbers of valid elements, so that the copy engines
// stage about the same bytes for each.  Segment s is [b[s], b[s+1]).  Cut this
// way, a segment copies only the params it holds: about W*(P + n) copies in
// all, where cutting by output ranks would copy every param in every segment
// (W*P*n copies, which is what limits groups of many small params).
std::vector<int64_t> segment_bounds(const tide_plan* p, int32_t n) {
    const int64_t W = p->world, J = (int64_t)p->n_params * W;
    auto valid = [&](int64_t j) {
        const int64_t i = j / W, r = j % W, c = p->chunk[i];
        return std::min(c, std::max<int64_t>(0, p->numel[i] - r * c));
    };
    long double total = 0;
    for (int64_t i = 0; i < p->n_params; ++i) total += (long double)p->numel[i];
    std::vector<int64_t> b((size_t)n + 1, J);
    b[0] = 0;
    long double acc = 0;
    int64_t j = 0;
    for (int32_t s = 1; s < n; ++s) {
        const long double target = total * s / n;
        while (j < J && acc < target) acc += (long double)valid(j++);
        b[s] = j;
    }
    return b;
}

}  // namespace

extern "C" tide_status_t tide_ag_place(const tide_plan_t* cplan, const void* ag_buf,
                                       int64_t ag_numel, void* const* param_storage,
                                       const int64_t* param_numel, int32_t engine,
                                       int32_t max_ctas, void* stream) {
    ApiRange range("tide_ag_place");
    tide_plan* p = const_cast<tide_plan*>(cplan);
    tide_status_t st = check_plan(p);
    if (st != TIDE_OK) return st;
    if ((st = all_ranks(p)) != TIDE_OK) return st;
    if ((st = check_enums(p, engine, max_ctas)) != TIDE_OK) return st;
    const int64_t W = p->world, P = p->n_params;
    std::vector<Span> spans;
    spans.reserve((size_t)p->world * (p->n_params + 1) + p->n_params + 2);
    if ((st = check_buf(ag_buf, ag_numel, W * p->shard_numel, 2)) != TIDE_OK) return st;
    add_span(spans, ag_buf, 2 * W * p->shard_numel, false);
    if (P > 0 && (param_storage == nullptr || param_numel == nullptr)) return TIDE_ERR_INVALID_ARG;
    for (int64_t i = 0; i < P; ++i) {
        if ((st = check_buf(param_storage[i], param_numel[i], W * p->chunk[i], 2)) != TIDE_OK) return st;
        add_span(spans, param_storage[i], 2 * W * p->chunk[i], true);
    }
    if (overlaps(spans)) return TIDE_ERR_INVALID_ARG;
    if ((st = launchable(p)) != TIDE_OK) return st;
    if (p->tiles.empty()) return TIDE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (engine == TIDE_ENGINE_CE) {
        p->last_kernel = -1;
        p->last_ctas = 0;
        e = tide::ce_ag_place(p, static_cast<const uint16_t*>(ag_buf), param_storage, s);
    } else {
        if ((st = sync_table(p->param_tab, const_cast<const void* const*>(param_storage), P, s)) != TIDE_OK)
            return st;
        p->last_kernel = K_AG;
        p->last_ctas = grid_for(p, K_AG, max_ctas);
        e = tide::launch_ag_place(p, static_cast<const uint16_t*>(ag_buf), ag_numel, p->param_tab.dev,
                                  p->last_ctas, s);
    }
    return e == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}

extern "C" tide_status_t tide_ag_gather_place(const tide_plan_t* cplan, const void* const* shards,
                                              int64_t shard_numel, void* const* param_storage,
                                              const int64_t* param_numel, int32_t engine,
                                              int32_t max_ctas, void* stream) {
    ApiRange range("tide_ag_gather_place");
    tide_plan* p = const_cast<tide_plan*>(cplan);
    tide_status_t st = check_plan(p);
    if (st != TIDE_OK) return st;
    if ((st = all_ranks(p)) != TIDE_OK) return st;
    if ((st = check_enums(p, engine, max_ctas)) != TIDE_OK) return st;
    const int64_t W = p->world, P = p->n_params, Ns = p->shard_numel;
    std::vector<Span> spans;
    spans.reserve((size_t)p->world * (p->n_params + 1) + p->n_params + 2);
    if (W > 0 && shards == nullptr) return TIDE_ERR_INVALID_ARG;
    for (int64_t r = 0; r < W; ++r) {
        if ((st = check_buf(shards[r], shard_numel, Ns, 2)) != TIDE_OK) return st;
        add_span(spans, shards[r], 2 * Ns, false);
    }
    if (P > 0 && (param_storage == nullptr || param_numel == nullptr)) return TIDE_ERR_INVALID_ARG;
    for (int64_t i = 0; i < P; ++i) {
        if ((st = check_buf(param_storage[i], param_numel[i], W * p->chunk[i], 2)) != TIDE_OK) return st;
        add_span(spans, param_storage[i], 2 * W * p->chunk[i], true);
    }
    if (overlaps(spans)) return TIDE_ERR_INVALID_ARG;
    if ((st = launchable(p)) != TIDE_OK) return st;
    if (p->tiles.empty()) return TIDE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (engine == TIDE_ENGINE_CE) {
        p->last_kernel = -1;
        p->last_ctas = 0;
        e = tide::ce_ag_gather(p, shards, param_storage, s);
    } else {
        if ((st = sync_table(p->shard_tab, shards, W, s)) != TIDE_OK) return st;
        if ((st = sync_table(p->param_tab, const_cast<const void* const*>(param_storage), P, s)) != TIDE_OK)
            return st;
        p->last_kernel = K_AG_GATHER;
        p->last_ctas = grid_for(p, K_AG_GATHER, max_ctas);
        e = tide::launch_ag_gather(p, p->shard_tab.dev, shard_numel, p->param_tab.dev, p->last_ctas, s);
    }
    return e == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}

extern "C" tide_status_t tide_rs_reduce(const tide_plan_t* cplan, const void* const* grads,
                                        const int64_t* grad_numel, float* out, int64_t out_numel,
                                        int32_t scale_mode, int32_t order, void* const* slots,
                                        int64_t slot_numel, int32_t engine, int32_t max_ctas,
                                        void* stream) {
    ApiRange range("tide_rs_reduce");
    tide_plan* p = const_cast<tide_plan*>(cplan);
    tide_status_t st = check_plan(p);
    if (st != TIDE_OK) return st;
    if ((st = check_enums(p, engine, max_ctas)) != TIDE_OK) return st;
    if ((st = check_reduce_modes(scale_mode, order)) != TIDE_OK) return st;
    if (slots != nullptr && (st = all_ranks(p)) != TIDE_OK) return st;
    // a one-rank plan writes only its own shard
    const int64_t W = p->world, P = p->n_params, n_out = (p->rank >= 0 ? 1 : W) * p->shard_numel;
    std::vector<Span> spans;
    spans.reserve((size_t)p->world * (p->n_params + 1) + p->n_params + 2);
    if ((st = check_grads(p, grads, grad_numel, spans)) != TIDE_OK) return st;
    if ((st = check_buf(out, out_numel, n_out, 4)) != TIDE_OK) return st;
    add_span(spans, out, 4 * n_out, true);
    if (slots != nullptr && (st = check_slots(p, slots, slot_numel, spans)) != TIDE_OK) return st;
    if (overlaps(spans)) return TIDE_ERR_INVALID_ARG;
    if ((st = launchable(p)) != TIDE_OK) return st;
    if (p->tiles.empty()) return TIDE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (slots != nullptr) {
        st = stage_impl(p, grads, slots, slot_numel, engine, max_ctas, s);
        if (st != TIDE_OK) return st;
        return reduce_slots_impl(p, slots, slot_numel, out, out_numel, scale_mode, order, max_ctas, s);
    }
    if ((st = sync_table(p->grad_tab, grads, W * P, s)) != TIDE_OK) return st;
    cudaError_t e = launch_reduce(p, p->grad_tab, false, 0, out, out_numel, scale_mode, order, max_ctas, s);
    return e == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}

extern "C" tide_status_t tide_rs_stage(const tide_plan_t* cplan, const void* const* grads,
                                       const int64_t* grad_numel, void* const* slots,
                                       int64_t slot_numel, int32_t engine, int32_t max_ctas,
                                       void* stream) {
    ApiRange range("tide_rs_stage");
    tide_plan* p = const_cast<tide_plan*>(cplan);
    tide_status_t st = check_plan(p);
    if (st != TIDE_OK) return st;
    if ((st = all_ranks(p)) != TIDE_OK) return st;
    if ((st = check_enums(p, engine, max_ctas)) != TIDE_OK) return st;
    std::vector<Span> spans;
    spans.reserve((size_t)p->world * (p->n_params + 1) + p->n_params + 2);
    if ((st = check_grads(p, grads, grad_numel, spans)) != TIDE_OK) return st;
    if ((st = check_slots(p, slots, slot_numel, spans)) != TIDE_OK) return st;
    if (overlaps(spans)) return TIDE_ERR_INVALID_ARG;
    if ((st = launchable(p)) != TIDE_OK) return st;
    return stage_impl(p, grads, slots, slot_numel, engine, max_ctas, static_cast<cudaStream_t>(stream));
}

extern "C" tide_status_t tide_rs_stage_one(const tide_plan_t* cplan, const void* const* grads,
                                           const int64_t* grad_numel, void* slot, int64_t slot_numel,
                                           int32_t engine, int32_t max_ctas, void* stream) {
    ApiRange range("tide_rs_stage_one");
    tide_plan* p = const_cast<tide_plan*>(cplan);
    tide_status_t st = check_plan(p);
    if (st != TIDE_OK) return st;
    if ((st = all_ranks(p)) != TIDE_OK) return st;
    if ((st = check_enums(p, engine, max_ctas)) != TIDE_OK) return st;
    const int64_t W = p->world, P = p->n_params;
    std::vector<Span> spans;
    spans.reserve((size_t)P + 1);
    if (P > 0 && (grads == nullptr || grad_numel == nullptr)) return TIDE_ERR_INVALID_ARG;
    for (int64_t i = 0; i < P; ++i) {
        if ((st = check_buf(grads[i], grad_numel[i], p->numel[i], 2)) != TIDE_OK) return st;
        add_span(spans, grads[i], 2 * p->numel[i], false);
    }
    if ((st = check_buf(slot, slot_numel, W * p->shard_numel, 2)) != TIDE_OK) return st;
    add_span(spans, slot, 2 * W * p->shard_numel, true);
    if (overlaps(spans)) return TIDE_ERR_INVALID_ARG;
    if ((st = launchable(p)) != TIDE_OK) return st;
    if (p->tiles.empty()) return TIDE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void* const slots[1] = {slot};
    cudaError_t e;
    if (engine == TIDE_ENGINE_CE) {
        p->last_kernel = -1;
        p->last_ctas = 0;
        e = tide::ce_slot_stage(p, grads, slots, s, 0, -1, false, true);
    } else {
        if ((st = sync_table(p->grad_tab, grads, P, s)) != TIDE_OK) return st;
        if ((st = sync_table(p->slot_tab, const_cast<const void* const*>(slots), 1, s)) != TIDE_OK)
            return st;
        p->last_kernel = K_STAGE;
        // one source rank: one unit per tile
        p->last_ctas = (int)std::min<int64_t>(grid_for(p, K_STAGE, max_ctas), (int64_t)p->tiles.size());
        e = tide::launch_slot_stage(p, p->grad_tab.dev, p->slot_tab.dev, slot_numel, p->last_ctas, s, 1);
    }
    return e == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}

extern "C" tide_status_t tide_rs_reduce_slots(const tide_plan_t* cplan, const void* const* slots,
                                              int64_t slot_numel, float* out, int64_t out_numel,
                                              int32_t scale_mode, int32_t order, int32_t max_ctas,
                                              void* stream) {
    ApiRange range("tide_rs_reduce_slots");
    tide_plan* p = const_cast<tide_plan*>(cplan);
    tide_status_t st = check_plan(p);
    if (st != TIDE_OK) return st;
    if ((st = check_enums(p, TIDE_ENGINE_SM, max_ctas)) != TIDE_OK) return st;
    if ((st = check_reduce_modes(scale_mode, order)) != TIDE_OK) return st;
    const int64_t n_out = (p->rank >= 0 ? 1 : (int64_t)p->world) * p->shard_numel;
    std::vector<Span> spans;
    spans.reserve((size_t)p->world * (p->n_params + 1) + p->n_params + 2);
    if ((st = check_slots(p, const_cast<void* const*>(slots), slot_numel, spans)) != TIDE_OK) return st;
    // slots are only read in this phase: re-tag them as read spans
    for (Span& sp : spans) sp.write = false;
    if ((st = check_buf(out, out_numel, n_out, 4)) != TIDE_OK) return st;
    add_span(spans, out, 4 * n_out, true);
    if (overlaps(spans)) return TIDE_ERR_INVALID_ARG;
    if ((st = launchable(p)) != TIDE_OK) return st;
    return reduce_slots_impl(p, const_cast<void* const*>(slots), slot_numel, out, out_numel, scale_mode,
                             order, max_ctas, static_cast<cudaStream_t>(stream));
}

extern "C" tide_status_t tide_rs_stage_one_f32(const tide_plan_t* cplan, const float* const* grads,
                                               const int64_t* grad_numel, float* slot, int64_t slot_numel,
                                               int32_t engine, int32_t max_ctas, void* stream) {
    ApiRange range("tide_rs_stage_one_f32");
    tide_plan* p = const_cast<tide_plan*>(cplan);
    tide_status_t st = check_plan(p);
    if (st != TIDE_OK) return st;
    if ((st = all_ranks(p)) != TIDE_OK) return st;
    if ((st = check_enums(p, engine, max_ctas)) != TIDE_OK) return st;
    const int64_t W = p->world, P = p->n_params;
    std::vector<Span> spans;
    spans.reserve((size_t)P + 1);
    if (P > 0 && (grads == nullptr || grad_numel == nullptr)) return TIDE_ERR_INVALID_ARG;
    for (int64_t i = 0; i < P; ++i) {
        if ((st = check_buf(grads[i], grad_numel[i], p->numel[i], 4)) != TIDE_OK) return st;
        add_span(spans, grads[i], 4 * p->numel[i], false);
    }
    if ((st = check_buf(slot, slot_numel, W * p->shard_numel, 4)) != TIDE_OK) return st;
    add_span(spans, slot, 4 * W * p->shard_numel, true);
    if (overlaps(spans)) return TIDE_ERR_INVALID_ARG;
    if ((st = launchable(p)) != TIDE_OK) return st;
    if (p->tiles.empty()) return TIDE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (engine == TIDE_ENGINE_CE) {
        p->last_kernel = -1;
        p->last_ctas = 0;
        void* const slots[1] = {slot};
        cudaError_t e = tide::ce_slot_stage(p, reinterpret_cast<const void* const*>(grads), slots, s, 0, -1,
                                            false, true, 4);
        return e == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
    }
    if ((st = sync_table(p->grad_tab, reinterpret_cast<const void* const*>(grads), P, s)) != TIDE_OK)
        return st;
    p->last_kernel = K_STAGE_F32;
    p->last_ctas = grid_for(p, K_STAGE_F32, max_ctas);
    cudaError_t e = tide::launch_stage_f32(p, p->grad_tab.dev, slot, slot_numel, p->last_ctas, s);
    return e == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}

extern "C" tide_status_t tide_rs_reduce_slots_f32(const tide_plan_t* cplan, const float* const* slots,
                                                  int64_t slot_numel, float* out, int64_t out_numel,
                                                  int32_t scale_mode, int32_t max_ctas, void* stream) {
    ApiRange range("tide_rs_reduce_slots_f32");
    tide_plan* p = const_cast<tide_plan*>(cplan);
    tide_status_t st = check_plan(p);
    if (st != TIDE_OK) return st;
    if ((st = check_enums(p, TIDE_ENGINE_SM, max_ctas)) != TIDE_OK) return st;
    if ((st = check_reduce_modes(scale_mode, TIDE_ORDER_RANK)) != TIDE_OK) return st;
    const int64_t W = p->world, need = W * p->shard_numel;
    const int64_t n_out = (p->rank >= 0 ? 1 : W) * p->shard_numel;
    std::vector<Span> spans;
    spans.reserve((size_t)W + 1);
    if (slots == nullptr) return TIDE_ERR_INVALID_ARG;
    for (int64_t k = 0; k < W; ++k) {
        if ((st = check_buf(slots[k], slot_numel, need, 4)) != TIDE_OK) return st;
        add_span(spans, slots[k], 4 * need, false);
    }
    if ((st = check_buf(out, out_numel, n_out, 4)) != TIDE_OK) return st;
    add_span(spans, out, 4 * n_out, true);
    if (overlaps(spans)) return TIDE_ERR_INVALID_ARG;
    if ((st = launchable(p)) != TIDE_OK) return st;
    if (p->tiles.empty()) return TIDE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // a one-rank plan's tiles address its shard from 0; its rows of every slot start at rank * Ns
    const int64_t row0 = p->rank >= 0 ? (int64_t)p->rank * p->shard_numel : 0;
    std::vector<const void*> from((size_t)W);
    for (int64_t k = 0; k < W; ++k) from[k] = slots[k] + row0;
    if ((st = sync_table(p->slot_tab, from.data(), W, s)) != TIDE_OK) return st;
    const bool v8 = p->slot_tab.aligned32 && (reinterpret_cast<uintptr_t>(out) & 31) == 0;
    p->last_kernel = K_SLOT_RS_F32;
    p->last_ctas = grid_for(p, K_SLOT_RS_F32, max_ctas);
    cudaError_t e = tide::launch_reduce_slots_f32(p, p->slot_tab.dev, slot_numel - row0, out, out_numel,
                                                  inv_world(p->world), scale_mode == TIDE_SCALE_INV_WORLD,
                                                  v8, p->last_ctas, s);
    return e == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}

extern "C" tide_status_t tide_rs_reduce_f32(const tide_plan_t* cplan, const float* const* grads,
                                            const int64_t* grad_numel, float* out, int64_t out_numel,
                                            int32_t scale_mode, int32_t max_ctas, void* stream) {
    ApiRange range("tide_rs_reduce_f32");
    tide_plan* p = const_cast<tide_plan*>(cplan);
    tide_status_t st = check_plan(p);
    if (st != TIDE_OK) return st;
    if ((st = check_enums(p, TIDE_ENGINE_SM, max_ctas)) != TIDE_OK) return st;
    if ((st = check_reduce_modes(scale_mode, TIDE_ORDER_RANK)) != TIDE_OK) return st;
    const int64_t W = p->world, P = p->n_params;
    const int64_t n_out = (p->rank >= 0 ? 1 : W) * p->shard_numel;
    std::vector<Span> spans;
    spans.reserve((size_t)(W * P) + 1);
    if (W * P > 0 && (grads == nullptr || grad_numel == nullptr)) return TIDE_ERR_INVALID_ARG;
    for (int64_t k = 0; k < W; ++k)
        for (int64_t i = 0; i < P; ++i) {
            const int64_t j = k * P + i;
            if ((st = check_buf(grads[j], grad_numel[j], p->numel[i], 4)) != TIDE_OK) return st;
            add_span(spans, grads[j], 4 * p->numel[i], false);
        }
    if ((st = check_buf(out, out_numel, n_out, 4)) != TIDE_OK) return st;
    add_span(spans, out, 4 * n_out, true);
    if (overlaps(spans)) return TIDE_ERR_INVALID_ARG;
    if ((st = launchable(p)) != TIDE_OK) return st;
    if (p->tiles.empty()) return TIDE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = sync_table(p->grad_tab, reinterpret_cast<const void* const*>(grads), W * P, s)) != TIDE_OK)
        return st;
    const bool v8 = p->grad_tab.aligned32 && (reinterpret_cast<uintptr_t>(out) & 31) == 0;
    p->last_kernel = K_RS_F32;
    p->last_ctas = grid_for(p, K_RS_F32, max_ctas);
    cudaError_t e = tide::launch_reduce_f32(p, p->grad_tab.dev, out, out_numel, inv_world(p->world),
                                            scale_mode == TIDE_SCALE_INV_WORLD, v8, p->last_ctas, s);
    return e == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
}

extern "C" tide_status_t tide_rs_reduce_pipelined(const tide_plan_t* cplan, const void* const* grads,
                                                  const int64_t* grad_numel, float* out,
                                                  int64_t out_numel, int32_t scale_mode,
                                                  int32_t order, void* const* slots,
                                                  int64_t slot_numel, int32_t n_segments,
                                                  int32_t max_ctas, void* stream, void* copy_stream) {
    ApiRange range("tide_rs_reduce_pipelined");
    tide_plan* p = const_cast<tide_plan*>(cplan);
    tide_status_t st = check_plan(p);
    if (st != TIDE_OK) return st;
    if ((st = check_enums(p, TIDE_ENGINE_SM, max_ctas)) != TIDE_OK) return st;
    if ((st = check_reduce_modes(scale_mode, order)) != TIDE_OK) return st;
    if (n_segments < 1 || n_segments > p->world) return TIDE_ERR_INVALID_ARG;
    // a one-rank plan (rank r) stages and reduces rank r's rows only: out is [Ns] and each
    // slot holds one source rank's row r ([Ns]); an all-rank plan's slots are [W][Ns]
    const bool one = p->rank >= 0;
    const int64_t W = p->world, n_out = (one ? 1 : W) * p->shard_numel;
    std::vector<Span> spans;
    spans.reserve((size_t)p->world * (p->n_params + 1) + p->n_params + 2);
    if ((st = check_grads(p, grads, grad_numel, spans)) != TIDE_OK) return st;
    if ((st = check_buf(out, out_numel, n_out, 4)) != TIDE_OK) return st;
    add_span(spans, out, 4 * n_out, true);
    if (!one) {
        if ((st = check_slots(p, slots, slot_numel, spans)) != TIDE_OK) return st;
    } else {
        if (slots == nullptr) return TIDE_ERR_INVALID_ARG;
        for (int64_t k = 0; k < W; ++k) {
            if ((st = check_buf(slots[k], slot_numel, p->shard_numel, 2)) != TIDE_OK) return st;
            add_span(spans, slots[k], 2 * p->shard_numel, true);
        }
    }
    if (overlaps(spans)) return TIDE_ERR_INVALID_ARG;
    if ((st = launchable(p)) != TIDE_OK) return st;
    if (p->tiles.empty()) return TIDE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream), cs = static_cast<cudaStream_t>(copy_stream);
    // pacing events, one per segment plus one for the start (created once per plan)
    while ((int64_t)p->seg_events.size() < (int64_t)n_segments + 1) {
        cudaEvent_t ev = nullptr;
        if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) {
            (void)cudaGetLastError();
            return TIDE_ERR_CUDA;
        }
        p->seg_events.push_back(ev);
    }
    if ((st = sync_table(p->slot_tab, const_cast<const void* const*>(slots), W, s)) != TIDE_OK) return st;
    // the copies may start once everything enqueued on `stream` so far is done
    cudaEvent_t start = p->seg_events[n_segments];
    if (cudaEventRecord(start, s) != cudaSuccess || cudaStreamWaitEvent(cs, start, 0) != cudaSuccess)
        return TIDE_ERR_CUDA;
    const std::vector<int64_t> bounds = segment_bounds(p, n_segments);
    for (int32_t seg = 0; seg < n_segments; ++seg) {
        const int64_t j0 = bounds[seg], j1 = bounds[seg + 1];
        if (j1 == j0) continue;
        // phase 1 of these chunks on the copy engines ...
        if ((one ? tide::ce_rank_stage(p, grads, slots, cs, j0, j1)
                 : tide::ce_slot_stage(p, grads, slots, cs, j0, j1, false)) != cudaSuccess)
            return TIDE_ERR_CUDA;
        cudaEvent_t done = p->seg_events[seg];
        if (cudaEventRecord(done, cs) != cudaSuccess || cudaStreamWaitEvent(s, done, 0) != cudaSuccess)
            return TIDE_ERR_CUDA;
        // ... phase 2 of them on the SMs, while the next segment is being copied
        if (launch_reduce(p, p->slot_tab, true, slot_numel, out, out_numel, scale_mode, order, max_ctas,
                          s, p->chunk_tile_begin[j0], p->chunk_tile_begin[j1]) != cudaSuccess)
            return TIDE_ERR_CUDA;
    }
    return TIDE_OK;
}

extern "C" tide_status_t tide_plan_errors(tide_plan_t* p, void* stream, int32_t* bits) {
    if (bits != nullptr) *bits = 0;
    tide_status_t st = check_plan(p);
    if (st != TIDE_OK) return st;
    if ((st = launchable(p)) != TIDE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t h = 0;
    if (cudaMemcpyAsync(&h, p->d_err, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return TIDE_ERR_CUDA;
    if (bits != nullptr) *bits = h;
    if (h == 0) return TIDE_OK;
    if (cudaMemsetAsync(p->d_err, 0, sizeof(int32_t), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return TIDE_ERR_CUDA;
    return TIDE_ERR_KERNEL_CHECK;
}

extern "C" tide_status_t tide_plan_check(tide_plan_t* p, void* stream) {
    return tide_plan_errors(p, stream, nullptr);
}
