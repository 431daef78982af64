/*
 * tide_oracle.c - plain CPU oracle for the TIDE data-parallel hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline / reference arm may load this library.  The CUDA
 * path shares no code with it and never calls it.
 *
 * What it computes is the *stock* FSDP2 layout conversion that TIDE removes,
 * written out step by step:
 *   - all-gather copy-out: the rank-major all-gather output is copied into
 *     the per-parameter tensors ("The Endgame of FSDP Communication",
 *     weekinpapers.com, Abstract; kongchang.com article of the same title,
 *     section "The Root of FSDP2 Communication Overhead", where the rank-major
 *     buffer is explained);
 *   - gradient pack: each rank's per-parameter bf16 gradients are converted
 *     and packed into one fp32 rank-major buffer covering the whole group
 *     (same Abstract);
 *   - reduce-scatter: the packed buffers are summed over ranks and rank r
 *     keeps the r-th shard (kongchang.com, "The Root of FSDP2 Communication
 *     Overhead", the reduce-scatter explanation).  TIDE-RS has to produce the
 *     same fp32 shards while reading the bf16 gradients where they lie, with
 *     no packed copy (weekinpapers.com, Abstract; kongchang.com, "TIDE's Design
 *     Approach").
 *
 * Readings the pages leave open (each is a choice, stated once here):
 *   - Sharding: every parameter is split along dim 0 into W contiguous blocks
 *     of S = ceil(d0 / W) rows; rank r owns rows [r*S, min((r+1)*S, d0)); rows
 *     d0 .. W*S-1 are padding (FSDP2's chunk-then-pad).
 *   - Flat layout: parameters follow the group order, tightly packed (no
 *     alignment gaps): param i starts at off_i = sum_{j<i} S_j * inner_j inside
 *     each rank's shard of Ns = sum_i S_i * inner_i elements; rank r's shard is
 *     [r*Ns, (r+1)*Ns) of any rank-major buffer.
 *   - Sum: rank order 0..W-1 starting from fp32(g_0), IEEE fp32
 *     round-to-nearest-even, no fused multiply-add; bf16 -> fp32 is exact.
 *   - Optional scale: after the sum, one fp32 multiply by fl32(1/W).
 *   - Tree order (an optional mode of the reduction, not on the pages): the W
 *     fp32 values of a position are added in adjacent pairs, level by level,
 *     an odd last value carried unchanged to the next level, until one is
 *     left; then the optional scale.
 *   - Pads: +0.0 in the fp32 shards and in padded parameter rows; source pads
 *     of the all-gather buffer are never read.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math (x86-64 SSE arithmetic).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Shard layout of a parameter group.  Returns 0, or -1 on a bad argument. */
int orc_layout(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
               int64_t* S, int64_t* c, int64_t* off, int64_t* Ns) {
    if (W < 1 || P < 0) return -1;
    int64_t acc = 0;
    for (int64_t i = 0; i < P; ++i) {
        if (d0[i] < 0 || inner[i] < 0) return -1;
        S[i] = (d0[i] + W - 1) / W;
        c[i] = S[i] * inner[i];
        off[i] = acc;
        acc += c[i];
    }
    *Ns = acc;
    return 0;
}

/*
 * Stock all-gather copy-out.  ag is the rank-major buffer [W][Ns]; params[i]
 * receives W*S_i rows of inner_i elements.  Valid rows are copied, pad rows are
 * zero-filled, source pad positions are not touched.
 */
int orc_ag_copyout(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                   const uint16_t* ag, uint16_t* const* params) {
    int64_t *S = malloc(sizeof(int64_t) * (P + 1)), *c = malloc(sizeof(int64_t) * (P + 1)),
            *off = malloc(sizeof(int64_t) * (P + 1)), Ns = 0;
    if (!S || !c || !off) { free(S); free(c); free(off); return -1; }
    orc_layout(W, P, d0, inner, S, c, off, &Ns);
    for (int64_t i = 0; i < P; ++i) {
        for (int64_t r = 0; r < W; ++r) {
            for (int64_t s = 0; s < S[i]; ++s) {
                int64_t row = r * S[i] + s;
                uint16_t* dst = params[i] + row * inner[i];
                if (row < d0[i]) {
                    const uint16_t* src = ag + r * Ns + off[i] + s * inner[i];
                    for (int64_t t = 0; t < inner[i]; ++t) dst[t] = src[t];
                } else {
                    for (int64_t t = 0; t < inner[i]; ++t) dst[t] = 0;
                }
            }
        }
    }
    free(S); free(c); free(off);
    return 0;
}

/*
 * Stock gradient pack of ONE rank: its P unpadded bf16 gradients g[i] go into a
 * full-group fp32 rank-major buffer buf[W][Ns]; every pad position is +0.0.
 */
static void pack_f32(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                     const int64_t* S, const int64_t* off, int64_t Ns,
                     const uint16_t* const* g, float* buf) {
    for (int64_t r = 0; r < W; ++r) {
        for (int64_t i = 0; i < P; ++i) {
            for (int64_t s = 0; s < S[i]; ++s) {
                int64_t row = r * S[i] + s;
                float* dst = buf + r * Ns + off[i] + s * inner[i];
                for (int64_t t = 0; t < inner[i]; ++t)
                    dst[t] = row < d0[i] ? bf16_to_f32(g[i][row * inner[i] + t]) : 0.0f;
            }
        }
    }
}

int orc_pack_f32(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                 const uint16_t* const* g, float* buf) {
    int64_t *S = malloc(sizeof(int64_t) * (P + 1)), *c = malloc(sizeof(int64_t) * (P + 1)),
            *off = malloc(sizeof(int64_t) * (P + 1)), Ns = 0;
    if (!S || !c || !off) { free(S); free(c); free(off); return -1; }
    orc_layout(W, P, d0, inner, S, c, off, &Ns);
    pack_f32(W, P, d0, inner, S, off, Ns, g, buf);
    free(S); free(c); free(off);
    return 0;
}

/*
 * Stock reduce-scatter over W simulated ranks.  grads[k*P + i] is rank k's
 * gradient of param i.  For k = 0..W-1: pack rank k into a full-group fp32
 * buffer, then add it into the running sum (rank 0's pack starts the sum).
 * Finally multiply by fl32(1/W) when scale_mode is 1.  out is [W][Ns]; rank r's
 * shard is out[r*Ns .. (r+1)*Ns).  Only one packed buffer is live at a time.
 */
int orc_rs_reduce(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                  const uint16_t* const* grads, int32_t scale_mode, float* out) {
    int64_t *S = malloc(sizeof(int64_t) * (P + 1)), *c = malloc(sizeof(int64_t) * (P + 1)),
            *off = malloc(sizeof(int64_t) * (P + 1)), Ns = 0;
    if (!S || !c || !off) { free(S); free(c); free(off); return -1; }
    orc_layout(W, P, d0, inner, S, c, off, &Ns);
    int64_t n = W * Ns;
    float* packed = malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    if (!packed) { free(S); free(c); free(off); return -1; }
    for (int64_t k = 0; k < W; ++k) {
        if (k == 0) {
            pack_f32(W, P, d0, inner, S, off, Ns, grads, out);
        } else {
            pack_f32(W, P, d0, inner, S, off, Ns, grads + k * P, packed);
            for (int64_t j = 0; j < n; ++j) out[j] = out[j] + packed[j];
        }
    }
    if (scale_mode == 1) {
        float s = 1.0f / (float)W;
        for (int64_t j = 0; j < n; ++j) out[j] = out[j] * s;
    }
    free(packed); free(S); free(c); free(off);
    return 0;
}

/*
 * Slot-Reuse phase 1 for ONE rank: its bf16 gradients are copied, unconverted,
 * into an all-gather buffer whose contents are no longer needed; that slot has
 * the all-gather layout [W][Ns] ("The Endgame of FSDP Communication",
 * weekinpapers.com, Abstract, the Slot-Reuse option of the two-phase pipeline).
 * Pad positions are left as they were.
 */
int orc_slot_stage(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                   const uint16_t* const* g, uint16_t* slot) {
    int64_t *S = malloc(sizeof(int64_t) * (P + 1)), *c = malloc(sizeof(int64_t) * (P + 1)),
            *off = malloc(sizeof(int64_t) * (P + 1)), Ns = 0;
    if (!S || !c || !off) { free(S); free(c); free(off); return -1; }
    orc_layout(W, P, d0, inner, S, c, off, &Ns);
    for (int64_t r = 0; r < W; ++r)
        for (int64_t i = 0; i < P; ++i)
            for (int64_t s = 0; s < S[i]; ++s) {
                int64_t row = r * S[i] + s;
                if (row >= d0[i]) continue;
                for (int64_t t = 0; t < inner[i]; ++t)
                    slot[r * Ns + off[i] + s * inner[i] + t] = g[i][row * inner[i] + t];
            }
    free(S); free(c); free(off);
    return 0;
}

/*
 * Slot-Reuse phase 2: the W staged slots are summed in rank order into fp32
 * shards, then scaled; positions that are padding in the layout are +0.0.
 */
int orc_rs_reduce_slots(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                        const uint16_t* const* slots, int32_t scale_mode, float* out) {
    int64_t *S = malloc(sizeof(int64_t) * (P + 1)), *c = malloc(sizeof(int64_t) * (P + 1)),
            *off = malloc(sizeof(int64_t) * (P + 1)), Ns = 0;
    if (!S || !c || !off) { free(S); free(c); free(off); return -1; }
    orc_layout(W, P, d0, inner, S, c, off, &Ns);
    float s = 1.0f / (float)W;
    for (int64_t r = 0; r < W; ++r)
        for (int64_t i = 0; i < P; ++i)
            for (int64_t e = 0; e < c[i]; ++e) {
                int64_t j = r * Ns + off[i] + e;
                int64_t row = r * S[i] + (inner[i] ? e / inner[i] : 0);
                if (row >= d0[i]) { out[j] = 0.0f; continue; }
                float acc = bf16_to_f32(slots[0][j]);
                for (int64_t k = 1; k < W; ++k) acc = acc + bf16_to_f32(slots[k][j]);
                out[j] = scale_mode == 1 ? acc * s : acc;
            }
    free(S); free(c); free(off);
    return 0;
}

/*
 * fp32 gradients.  While gradient sync is off, FSDP2 keeps a parameter's
 * gradients in its fp32 reduce dtype, and the next synced backward packs those
 * fp32 gradients as they are: the same pack into the fp32 rank-major buffer
 * with no conversion, then the same reduce-scatter (weekinpapers.com,
 * Abstract: the gradients that TIDE-RS reads in place are the ones the stock
 * path packs).  These three functions are the bf16 ones above with fp32
 * inputs: pack, then the rank-order sum from rank 0's pack, then the optional
 * multiply; Slot-Reuse staging as a copy of the 4-byte words, pads untouched.
 */
static void pack_f32_of_f32(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                            const int64_t* S, const int64_t* off, int64_t Ns,
                            const float* const* g, float* buf) {
    for (int64_t r = 0; r < W; ++r) {
        for (int64_t i = 0; i < P; ++i) {
            for (int64_t s = 0; s < S[i]; ++s) {
                int64_t row = r * S[i] + s;
                float* dst = buf + r * Ns + off[i] + s * inner[i];
                for (int64_t t = 0; t < inner[i]; ++t)
                    dst[t] = row < d0[i] ? g[i][row * inner[i] + t] : 0.0f;
            }
        }
    }
}

int orc_rs_reduce_f32(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                      const float* const* grads, int32_t scale_mode, float* out) {
    int64_t *S = malloc(sizeof(int64_t) * (P + 1)), *c = malloc(sizeof(int64_t) * (P + 1)),
            *off = malloc(sizeof(int64_t) * (P + 1)), Ns = 0;
    if (!S || !c || !off) { free(S); free(c); free(off); return -1; }
    orc_layout(W, P, d0, inner, S, c, off, &Ns);
    int64_t n = W * Ns;
    float* packed = malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    if (!packed) { free(S); free(c); free(off); return -1; }
    pack_f32_of_f32(W, P, d0, inner, S, off, Ns, grads, out);
    for (int64_t k = 1; k < W; ++k) {
        pack_f32_of_f32(W, P, d0, inner, S, off, Ns, grads + k * P, packed);
        for (int64_t j = 0; j < n; ++j) out[j] += packed[j];
    }
    if (scale_mode == 1) {
        float sc = 1.0f / (float)W;
        for (int64_t j = 0; j < n; ++j) out[j] = out[j] * sc;
    }
    free(packed); free(S); free(c); free(off);
    return 0;
}

int orc_slot_stage_f32(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                       const uint32_t* const* g, uint32_t* slot) {
    int64_t *S = malloc(sizeof(int64_t) * (P + 1)), *c = malloc(sizeof(int64_t) * (P + 1)),
            *off = malloc(sizeof(int64_t) * (P + 1)), Ns = 0;
    if (!S || !c || !off) { free(S); free(c); free(off); return -1; }
    orc_layout(W, P, d0, inner, S, c, off, &Ns);
    for (int64_t r = 0; r < W; ++r)
        for (int64_t i = 0; i < P; ++i)
            for (int64_t s = 0; s < S[i]; ++s) {
                const int64_t src_row = r * S[i] + s;      /* row of the param, rank r's s-th */
                if (src_row >= d0[i]) continue;            /* a pad row: the slot keeps its words */
                for (int64_t t = 0; t < inner[i]; ++t)
                    slot[r * Ns + off[i] + s * inner[i] + t] = g[i][src_row * inner[i] + t];
            }
    free(S); free(c); free(off);
    return 0;
}

int orc_rs_reduce_slots_f32(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                            const float* const* slots, int32_t scale_mode, float* out) {
    int64_t *S = malloc(sizeof(int64_t) * (P + 1)), *c = malloc(sizeof(int64_t) * (P + 1)),
            *off = malloc(sizeof(int64_t) * (P + 1)), Ns = 0;
    if (!S || !c || !off) { free(S); free(c); free(off); return -1; }
    orc_layout(W, P, d0, inner, S, c, off, &Ns);
    float sc = 1.0f / (float)W;
    for (int64_t r = 0; r < W; ++r)
        for (int64_t i = 0; i < P; ++i)
            for (int64_t e = 0; e < c[i]; ++e) {
                int64_t j = r * Ns + off[i] + e;
                int64_t row = r * S[i] + (inner[i] ? e / inner[i] : 0);
                if (row >= d0[i]) { out[j] = 0.0f; continue; }
                float acc = slots[0][j];
                for (int64_t k = 1; k < W; ++k) acc = acc + slots[k][j];
                out[j] = scale_mode == 1 ? acc * sc : acc;
            }
    free(S); free(c); free(off);
    return 0;
}

/*
 * The tree order on one position: v[0..n) are replaced, level by level, by the
 * sums of adjacent pairs (v[0]+v[1], v[2]+v[3], ...), an odd last value carried
 * unchanged, until one value is left.  fp32 adds, round-to-nearest-even.
 */
static float tree_of(float* v, int64_t n) {
    while (n > 1) {
        int64_t m = 0;
        for (int64_t j = 0; j + 1 < n; j += 2) v[m++] = v[j] + v[j + 1];
        if (n % 2 == 1) v[m++] = v[n - 1];
        n = m;
    }
    return v[0];
}

/* Tree-order sum of one position's W bf16 values, then the optional scale. */
float orc_sum_ranks_tree(int64_t W, const uint16_t* vals, int32_t scale_mode) {
    float* v = malloc(sizeof(float) * (size_t)(W > 0 ? W : 1));
    if (!v) return 0.0f;
    for (int64_t k = 0; k < W; ++k) v[k] = bf16_to_f32(vals[k]);
    float acc = tree_of(v, W);
    free(v);
    if (scale_mode == 1) acc = acc * (1.0f / (float)W);
    return acc;
}

/*
 * The reduce-scatter in tree order, position by position straight from the
 * per-parameter gradients (the definition written out; no packed buffer):
 *   out[r*Ns + off_i + e] = s * tree_k(fp32(g_{k,i}[r*c_i + e])) for valid
 * positions, +0.0 at pads.
 */
int orc_rs_reduce_tree(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                       const uint16_t* const* grads, int32_t scale_mode, float* out) {
    int64_t *S = malloc(sizeof(int64_t) * (P + 1)), *c = malloc(sizeof(int64_t) * (P + 1)),
            *off = malloc(sizeof(int64_t) * (P + 1)), Ns = 0;
    float* v = malloc(sizeof(float) * (size_t)(W > 0 ? W : 1));
    if (!S || !c || !off || !v) { free(S); free(c); free(off); free(v); return -1; }
    orc_layout(W, P, d0, inner, S, c, off, &Ns);
    const float s = 1.0f / (float)W;
    for (int64_t r = 0; r < W; ++r)
        for (int64_t i = 0; i < P; ++i)
            for (int64_t e = 0; e < c[i]; ++e) {
                int64_t j = r * Ns + off[i] + e, src = r * c[i] + e;
                if (src >= d0[i] * inner[i]) { out[j] = 0.0f; continue; }
                for (int64_t k = 0; k < W; ++k) v[k] = bf16_to_f32(grads[k * P + i][src]);
                float acc = tree_of(v, W);
                out[j] = scale_mode == 1 ? acc * s : acc;
            }
    free(S); free(c); free(off); free(v);
    return 0;
}

/*
 * Exact (fp64) sums for the tree-order tolerance check: E[j] = sum_k g and
 * A[j] = sum_k |g| over the same positions as the reduce-scatter.  bf16 values
 * carry 8 significant bits, so for the generated magnitudes and W <= 64 every
 * partial sum is exact in fp64.  Pads give 0.
 */
int orc_exact_f64(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                  const uint16_t* const* grads, double* E, double* A) {
    int64_t *S = malloc(sizeof(int64_t) * (P + 1)), *c = malloc(sizeof(int64_t) * (P + 1)),
            *off = malloc(sizeof(int64_t) * (P + 1)), Ns = 0;
    if (!S || !c || !off) { free(S); free(c); free(off); return -1; }
    orc_layout(W, P, d0, inner, S, c, off, &Ns);
    for (int64_t r = 0; r < W; ++r)
        for (int64_t i = 0; i < P; ++i)
            for (int64_t e = 0; e < c[i]; ++e) {
                int64_t j = r * Ns + off[i] + e, src = r * c[i] + e;
                double sum = 0.0, mag = 0.0;
                if (src < d0[i] * inner[i])
                    for (int64_t k = 0; k < W; ++k) {
                        double v = (double)bf16_to_f32(grads[k * P + i][src]);
                        sum += v;
                        mag += v < 0 ? -v : v;
                    }
                E[j] = sum;
                A[j] = mag;
            }
    free(S); free(c); free(off);
    return 0;
}

/*
 * Where output position j of rank r's shard comes from: returns 1 and sets
 * *param / *src_idx (index into that param's unpadded tensor) for a valid
 * position, 0 for a pad position, -1 if j is outside the shard.
 */
int orc_locate(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
               int64_t r, int64_t j, int64_t* param, int64_t* src_idx) {
    int64_t start = 0;
    for (int64_t i = 0; i < P; ++i) {
        int64_t S = (d0[i] + W - 1) / W, c = S * inner[i];
        if (j >= start && j < start + c) {
            int64_t e = j - start, row = r * S + e / inner[i];
            *param = i;
            *src_idx = r * c + e;
            return row < d0[i] ? 1 : 0;
        }
        start += c;
    }
    return -1;
}

/* fp32 rank-order sum of one position's W bf16 values, then the optional scale. */
float orc_sum_ranks(int64_t W, const uint16_t* vals, int32_t scale_mode) {
    float acc = bf16_to_f32(vals[0]);
    for (int64_t k = 1; k < W; ++k) acc = acc + bf16_to_f32(vals[k]);
    if (scale_mode == 1) acc = acc * (1.0f / (float)W);
    return acc;
}

/*
 * Where element q of param i's padded storage comes from in the rank-major
 * all-gather buffer: returns 1 and sets *ag_idx (flat index into [W][Ns]) for
 * a valid row, 0 for a pad row, -1 if q is outside the padded storage.
 */
int orc_ag_source(int64_t W, int64_t P, const int64_t* d0, const int64_t* inner,
                  int64_t i, int64_t q, int64_t* ag_idx) {
    int64_t off = 0, Ns = 0;
    for (int64_t j = 0; j < P; ++j) {
        int64_t c = ((d0[j] + W - 1) / W) * inner[j];
        if (j < i) off += c;
        Ns += c;
    }
    int64_t S = (d0[i] + W - 1) / W, c = S * inner[i];
    if (c == 0 || q < 0 || q >= W * c) return -1;
    int64_t r = q / c, e = q % c, row = r * S + e / inner[i];
    *ag_idx = r * Ns + off + e;
    return row < d0[i] ? 1 : 0;
}
