// plan.cpp - tide_plan_group and the plan queries.
//
// A plan turns a parameter group into the address tables the kernels walk:
// per param the shard rows S_i = ceil(d0_i / W), chunk c_i = S_i * inner_i and
// offset off_i inside a rank's shard (tightly packed in group order), and a
// tile list that cuts every (param, rank) chunk into pieces of at most
// TIDE_TILE_ELEMS elements, ordered by their position in the rank-major
// buffer.  Each tile records how many of its elements hold data; the rest are
// pad rows.  Tiles have equal size apart from chunk ends, so a static
// round-robin over CTAs balances thousands of small MoE chunks and a few huge
// dense ones alike.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>

#include "tide_internal.h"

namespace {

constexpr int64_t kI64Max = INT64_MAX;

bool mul_ok(int64_t a, int64_t b) { return a == 0 || b <= kI64Max / a; }

template <class T>
cudaError_t dev_alloc(T** p, int64_t count, int64_t* total) {
    *p = nullptr;
    if (count <= 0) return cudaSuccess;
    cudaError_t e = cudaMalloc(reinterpret_cast<void**>(p), sizeof(T) * (size_t)count);
    if (e == cudaSuccess) *total += (int64_t)sizeof(T) * count;
    return e;
}

void free_device(tide_plan* p) {
    cudaFree(p->d_tiles);
    cudaFree(p->d_numel);
    cudaFree(p->d_err);
    cudaFree(p->d_counter);
    cudaFree(p->grad_tab.dev);
    cudaFree(p->param_tab.dev);
    cudaFree(p->slot_tab.dev);
    cudaFree(p->shard_tab.dev);
    p->d_tiles = nullptr;
    p->d_numel = nullptr;
    p->d_err = nullptr;
    p->d_counter = nullptr;
    p->grad_tab.dev = p->param_tab.dev = p->slot_tab.dev = p->shard_tab.dev = nullptr;
}

tide_status_t upload(tide_plan* p) {
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) {
        (void)cudaGetLastError();
        return TIDE_ERR_CUDA;
    }
    if (cudaSetDevice(p->device) != cudaSuccess) {
        (void)cudaGetLastError();
        return TIDE_ERR_DEVICE;
    }
    tide_status_t st = TIDE_OK;
    int64_t total = 0;
    const int64_t W = p->world, P = p->n_params, T = (int64_t)p->tiles.size();
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = dev_alloc(&p->d_tiles, T, &total);
    if (e == cudaSuccess) e = dev_alloc(&p->d_numel, 2 * P, &total);
    if (e == cudaSuccess) e = dev_alloc(&p->d_err, 1, &total);
    if (e == cudaSuccess) e = dev_alloc(&p->d_counter, 2, &total);
    if (e == cudaSuccess) e = dev_alloc(&p->grad_tab.dev, W * P, &total);
    if (e == cudaSuccess) e = dev_alloc(&p->param_tab.dev, P, &total);
    if (e == cudaSuccess) e = dev_alloc(&p->slot_tab.dev, W, &total);
    if (e == cudaSuccess) e = dev_alloc(&p->shard_tab.dev, W, &total);
    if (e != cudaSuccess) {
        st = (e == cudaErrorMemoryAllocation) ? TIDE_ERR_NOMEM : TIDE_ERR_CUDA;
    }
    p->grad_tab.capacity = W * P;
    p->param_tab.capacity = P;
    p->slot_tab.capacity = W;
    p->shard_tab.capacity = W;
    if (st == TIDE_OK && T > 0)
        e = cudaMemcpy(p->d_tiles, p->tiles.data(), sizeof(tide_tile_t) * T, cudaMemcpyHostToDevice);
    if (st == TIDE_OK && e == cudaSuccess && P > 0) {
        std::vector<int64_t> n2(2 * P);
        for (int64_t i = 0; i < P; ++i) {
            n2[i] = p->numel[i];
            n2[P + i] = W * p->chunk[i];
        }
        e = cudaMemcpy(p->d_numel, n2.data(), sizeof(int64_t) * 2 * P, cudaMemcpyHostToDevice);
    }
    if (st == TIDE_OK && e == cudaSuccess) e = cudaMemset(p->d_err, 0, sizeof(int32_t));
    if (st == TIDE_OK && e == cudaSuccess)
        e = cudaMemset(p->d_counter, 0, 2 * sizeof(unsigned long long));
    if (st == TIDE_OK && e == cudaSuccess)
        e = cudaDeviceGetAttribute(&p->sm_count, cudaDevAttrMultiProcessorCount, p->device);
    if (st == TIDE_OK && e != cudaSuccess) st = TIDE_ERR_CUDA;
    if (st == TIDE_OK) {
        p->blocks_per_sm[K_RS] = tide::rs_blocks_per_sm(p->world, false, TIDE_ORDER_RANK, false);
        p->blocks_per_sm[K_SLOT_RS] = tide::rs_blocks_per_sm(p->world, true, TIDE_ORDER_RANK, false);
        if (tide::rs_v32_applies(p->world, TIDE_ORDER_RANK)) {
            p->blocks_per_sm[K_RS_V32] = tide::rs_blocks_per_sm(p->world, false, TIDE_ORDER_RANK, true);
            p->blocks_per_sm[K_SLOT_RS_V32] = tide::rs_blocks_per_sm(p->world, true, TIDE_ORDER_RANK, true);
        }
        if (tide::rs_v32_applies(p->world, TIDE_ORDER_TREE)) {
            p->blocks_per_sm[K_RS_TREE_V32] = tide::rs_blocks_per_sm(p->world, false, TIDE_ORDER_TREE, true);
            p->blocks_per_sm[K_SLOT_RS_TREE_V32] =
                tide::rs_blocks_per_sm(p->world, true, TIDE_ORDER_TREE, true);
        }
        p->blocks_per_sm[K_RS_TREE] = tide::rs_blocks_per_sm(p->world, false, TIDE_ORDER_TREE, false);
        p->blocks_per_sm[K_SLOT_RS_TREE] = tide::rs_blocks_per_sm(p->world, true, TIDE_ORDER_TREE, false);
        p->blocks_per_sm[K_AG] = tide::ag_blocks_per_sm(false);
        p->blocks_per_sm[K_AG_GATHER] = tide::ag_blocks_per_sm(true);
        p->blocks_per_sm[K_STAGE] = tide::stage_blocks_per_sm();
        p->blocks_per_sm[K_STAGE_F32] = tide::stage_f32_blocks_per_sm();
        p->blocks_per_sm[K_SLOT_RS_F32] = tide::reduce_f32_blocks_per_sm(true);
        p->blocks_per_sm[K_RS_F32] = tide::reduce_f32_blocks_per_sm(false);
        for (int k : {K_RS, K_AG, K_STAGE, K_SLOT_RS, K_RS_TREE, K_SLOT_RS_TREE, K_AG_GATHER, K_STAGE_F32,
                      K_SLOT_RS_F32, K_RS_F32})
            if (p->blocks_per_sm[k] <= 0) st = TIDE_ERR_CUDA;
        // 0 here (not enough shared memory) only disables the bulk-copy path
        p->blocks_per_sm[K_RS_TMA] = p->blocks_per_sm[K_SLOT_RS_TMA] = tide::rs_tma_blocks_per_sm(p->world);
        (void)cudaGetLastError();
    }
    p->workspace_bytes = total;
    if (st != TIDE_OK) free_device(p);
    cudaSetDevice(prev);
    if (st != TIDE_OK) (void)cudaGetLastError();  // leave no stale error for later launches
    return st;
}

// Builds a plan for all ranks (rank < 0) or for one output rank.
tide_status_t make_plan(const tide_param_t* params, int32_t n_params, int32_t world, int32_t rank,
                        int32_t device, uint32_t flags, tide_plan_t** out_plan) {
    if (out_plan == nullptr) return TIDE_ERR_INVALID_ARG;
    *out_plan = nullptr;
    if (n_params < 0 || (n_params > 0 && params == nullptr)) return TIDE_ERR_INVALID_ARG;
    if (world < 1 || world > TIDE_MAX_WORLD) return TIDE_ERR_INVALID_ARG;
    if (rank >= world) return TIDE_ERR_INVALID_ARG;
    if ((flags & ~(uint32_t)(TIDE_PLAN_HOST_ONLY | TIDE_PLAN_TMA | TIDE_PLAN_TEST_TMA_TIMEOUT |
                             TIDE_PLAN_SHORT_CTAS)) != 0)
        return TIDE_ERR_INVALID_ARG;
    if (!(flags & TIDE_PLAN_HOST_ONLY) && device < 0) return TIDE_ERR_DEVICE;

    tide_plan* p = new (std::nothrow) tide_plan;
    if (p == nullptr) return TIDE_ERR_NOMEM;
    p->device = device;
    p->world = world;
    p->rank = rank;
    p->n_params = n_params;
    p->flags = flags;
    const int64_t W = world;
    try {
        p->dim0.resize(n_params);
        p->inner.resize(n_params);
        p->numel.resize(n_params);
        p->rows.resize(n_params);
        p->chunk.resize(n_params);
        p->offset.resize(n_params);
        int64_t acc = 0;
        for (int32_t i = 0; i < n_params; ++i) {
            const int64_t d0 = params[i].dim0, in = params[i].inner;
            if (d0 < 0 || in < 0 || !mul_ok(d0, in)) { delete p; return TIDE_ERR_INVALID_ARG; }
            const int64_t S = d0 / W + (d0 % W != 0);
            if (!mul_ok(S, in) || !mul_ok(W, S * in)) { delete p; return TIDE_ERR_SIZE; }
            p->dim0[i] = d0;
            p->inner[i] = in;
            p->numel[i] = d0 * in;
            p->rows[i] = S;
            p->chunk[i] = S * in;
            p->offset[i] = acc;
            if (acc > kI64Max - S * in) { delete p; return TIDE_ERR_SIZE; }
            acc += S * in;
        }
        if (!mul_ok(W, acc)) { delete p; return TIDE_ERR_SIZE; }
        p->shard_numel = acc;
        // tiles in chunk order: param, then rank, then position; the chunk
        // (i, r) is number i*W + r and holds tiles [begin[i*W+r], begin[i*W+r+1]).
        // A one-rank plan keeps only its rank's chunks, at offsets in its shard.
        p->chunk_tile_begin.assign((size_t)n_params * W + 1, 0);
        for (int32_t i = 0; i < n_params; ++i) {
            for (int64_t r = 0; r < W; ++r) {
                p->chunk_tile_begin[(size_t)i * W + r] = (int64_t)p->tiles.size();
                if (rank >= 0 && r != rank) continue;
                const int64_t c = p->chunk[i];
                const int64_t valid = std::min(c, std::max<int64_t>(0, p->numel[i] - r * c));
                for (int64_t e0 = 0; e0 < c; e0 += TIDE_TILE_ELEMS) {
                    tide_tile_t t;
                    t.src_off = r * c + e0;
                    t.dst_off = (rank >= 0 ? 0 : r * acc) + p->offset[i] + e0;
                    t.param = i;
                    t.rank = (int32_t)r;
                    t.n_total = (int32_t)std::min<int64_t>(TIDE_TILE_ELEMS, c - e0);
                    t.n_valid = (int32_t)std::min<int64_t>(t.n_total, std::max<int64_t>(0, valid - e0));
                    if ((t.src_off & 7) != 0 || (t.dst_off & 7) != 0) p->tiles_aligned8 = false;
                    if ((t.src_off & 15) != 0 || (t.dst_off & 15) != 0) p->tiles_aligned16 = false;
                    p->tiles.push_back(t);
                }
            }
        }
        p->chunk_tile_begin[(size_t)n_params * W] = (int64_t)p->tiles.size();
    } catch (const std::bad_alloc&) {
        delete p;
        return TIDE_ERR_NOMEM;
    }
    if (!(flags & TIDE_PLAN_HOST_ONLY)) {
        tide_status_t st = upload(p);
        if (st != TIDE_OK) {
            delete p;
            return st;
        }
    }
    *out_plan = p;
    return TIDE_OK;
}

}  // namespace

extern "C" tide_status_t tide_plan_group(const tide_param_t* params, int32_t n_params,
                                         int32_t world, int32_t device, uint32_t flags,
                                         tide_plan_t** out_plan) {
    return make_plan(params, n_params, world, -1, device, flags, out_plan);
}

extern "C" tide_status_t tide_plan_group_rank(const tide_param_t* params, int32_t n_params,
                                              int32_t world, int32_t rank, int32_t device,
                                              uint32_t flags, tide_plan_t** out_plan) {
    if (rank < 0) {
        if (out_plan != nullptr) *out_plan = nullptr;
        return TIDE_ERR_INVALID_ARG;
    }
    return make_plan(params, n_params, world, rank, device, flags, out_plan);
}

extern "C" void tide_plan_destroy(tide_plan_t* plan) {
    if (plan == nullptr) return;
    tide::ce_release(plan);
    if (!(plan->flags & TIDE_PLAN_HOST_ONLY)) {
        int prev = -1;
        cudaGetDevice(&prev);
        if (cudaSetDevice(plan->device) == cudaSuccess) {
            cudaDeviceSynchronize();
            free_device(plan);
            for (cudaEvent_t ev : plan->seg_events) cudaEventDestroy(ev);
            plan->seg_events.clear();
            for (cudaStream_t st : plan->ce_streams) cudaStreamDestroy(st);
            for (cudaEvent_t ev : plan->ce_events) cudaEventDestroy(ev);
            plan->ce_streams.clear();
            plan->ce_events.clear();
        }
        if (prev >= 0) cudaSetDevice(prev);
    }
    delete plan;
}

extern "C" tide_status_t tide_plan_info(const tide_plan_t* plan, int32_t* world,
                                        int32_t* n_params, int64_t* shard_numel,
                                        int64_t* n_tiles, int64_t* workspace_bytes) {
    if (plan == nullptr) return TIDE_ERR_INVALID_ARG;
    if (world) *world = plan->world;
    if (n_params) *n_params = plan->n_params;
    if (shard_numel) *shard_numel = plan->shard_numel;
    if (n_tiles) *n_tiles = (int64_t)plan->tiles.size();
    if (workspace_bytes) *workspace_bytes = plan->workspace_bytes;
    return TIDE_OK;
}

extern "C" tide_status_t tide_plan_query(const tide_plan_t* plan, int32_t param,
                                         int64_t* shard_rows, int64_t* shard_offset,
                                         int64_t* padded_numel, int64_t* chunk_numel) {
    if (plan == nullptr || param < 0 || param >= plan->n_params) return TIDE_ERR_INVALID_ARG;
    if (shard_rows) *shard_rows = plan->rows[param];
    if (shard_offset) *shard_offset = plan->offset[param];
    if (padded_numel) *padded_numel = (int64_t)plan->world * plan->chunk[param];
    if (chunk_numel) *chunk_numel = plan->chunk[param];
    return TIDE_OK;
}

extern "C" tide_status_t tide_plan_tiles(const tide_plan_t* plan, tide_tile_t* out,
                                         int64_t capacity, int64_t* n_written) {
    if (plan == nullptr || n_written == nullptr || capacity < 0) return TIDE_ERR_INVALID_ARG;
    const int64_t n = std::min<int64_t>(capacity, (int64_t)plan->tiles.size());
    if (n > 0 && out == nullptr) return TIDE_ERR_INVALID_ARG;
    if (n > 0) std::memcpy(out, plan->tiles.data(), sizeof(tide_tile_t) * (size_t)n);
    *n_written = n;
    return TIDE_OK;
}

extern "C" tide_status_t tide_launch_ctas(const tide_plan_t* plan, int32_t kernel,
                                          int32_t max_ctas, int32_t* ctas) {
    if (plan == nullptr || ctas == nullptr || kernel < 0 || kernel >= K_COUNT || max_ctas < 0)
        return TIDE_ERR_INVALID_ARG;
    if (plan->flags & TIDE_PLAN_HOST_ONLY) return TIDE_ERR_DEVICE;
    int64_t units = (int64_t)plan->tiles.size();
    if (kernel == K_STAGE) units *= plan->world;
    if (kernel >= K_RS_TMA && plan->blocks_per_sm[kernel] <= 0) {
        *ctas = 0;
        return TIDE_OK;
    }
    if ((plan->flags & TIDE_PLAN_SHORT_CTAS) && kernel != K_RS_TMA && kernel != K_SLOT_RS_TMA) {
        // one short-lived CTA per unit of work
        *ctas = (int32_t)std::min<int64_t>(units, INT32_MAX);
        return TIDE_OK;
    }
    int64_t grid = (int64_t)plan->blocks_per_sm[kernel] * plan->sm_count;
    if (max_ctas > 0) grid = std::min<int64_t>(grid, max_ctas);
    grid = std::min(grid, units);
    *ctas = (int32_t)std::max<int64_t>(grid, 0);
    return TIDE_OK;
}

extern "C" tide_status_t tide_plan_last_launch(const tide_plan_t* plan, int32_t* kernel,
                                               int32_t* ctas) {
    if (plan == nullptr || kernel == nullptr || ctas == nullptr) return TIDE_ERR_INVALID_ARG;
    *kernel = plan->last_kernel;
    *ctas = plan->last_ctas;
    return TIDE_OK;
}

extern "C" const char* tide_status_string(tide_status_t s) {
    switch (s) {
        case TIDE_OK: return "ok";
        case TIDE_ERR_INVALID_ARG: return "invalid argument";
        case TIDE_ERR_ALIGNMENT: return "misaligned buffer";
        case TIDE_ERR_SIZE: return "buffer too small or size overflow";
        case TIDE_ERR_CUDA: return "CUDA error";
        case TIDE_ERR_NOMEM: return "out of memory";
        case TIDE_ERR_DEVICE: return "wrong device or host-only plan";
        case TIDE_ERR_KERNEL_CHECK: return "a kernel range check failed";
    }
    return "unknown status";
}

extern "C" int32_t tide_abi_version(void) { return 1; }
