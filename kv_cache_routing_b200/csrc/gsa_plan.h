// Host-side descriptor validation and launch plans (split counts, workspace
// layout).  Every quantity is a function of the descriptor alone, so results
// are bit-identical for a given descriptor on any device.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include <algorithm>

#include <cuda_runtime.h>

#include "gsa.h"

namespace gsa {

constexpr size_t kWsErrOffset = 0;          // u32 error word
constexpr size_t kWsCntOffset = 64;         // u32 tickets [2][rows]
constexpr int kTargetGistCtas = 296;        // 2 resident gist-pass CTAs per SM on 148 SMs
constexpr int kTargetUnfoldCtas = 444;      // 3 resident unfold-pass CTAs per SM
constexpr int kMaxSplits = 256;

// Library-wide device state shared between the source files (host side).
cudaError_t prefill_error_word(uint32_t** addr);        // gsa_prefill.cu
cudaError_t set_cross_cta_wait_limit(uint64_t ns);      // gsa_fused.cu (0 restores the default)

// A paged raw cache: chunk j of sequence b is page table[b * N + j] of the
// pools k_pages / v_pages [n_pages][Hkv][c][d] (one page: one chunk of every
// KV head); sequence b has nch[b] chunks (nch null: all N).  Dense callers
// pass no Paging.
struct Paging {
    const int32_t* table;
    const int32_t* nch;
    int n_pages;
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

inline int elem_bytes(int dtype) { return dtype == GSA_F32 ? 4 : 2; }
// keys per pipeline stage (one 16 KiB stage per tensor)
inline int stage_keys(int dtype, int head_dim) { return 16384 / (head_dim * elem_bytes(dtype)); }

inline gsa_status validate_decode(const gsa_decode_desc* d) {
    if (!d) return GSA_ERR_ARG;
    if (d->dtype != GSA_F32 && d->dtype != GSA_BF16) return GSA_ERR_DTYPE;
    if (d->mode != GSA_ALL_GISTS && d->mode != GSA_SELECTED_PAIRS && d->mode != GSA_SR_ONLY &&
        d->mode != GSA_UNSELECTED_GISTS)
        return GSA_ERR_ARG;
    if (d->batch < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1) return GSA_ERR_SHAPE;
    if (d->n_q_heads % d->n_kv_heads != 0) return GSA_ERR_SHAPE;
    const int G = d->n_q_heads / d->n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return GSA_ERR_SHAPE;
    if (d->head_dim != 64 && d->head_dim != 128) return GSA_ERR_SHAPE;
    if (d->n_chunks < 0 || d->chunk < 1 || d->tail_len < 0) return GSA_ERR_ARG;
    if (d->top_k < 0 || d->top_k > d->n_chunks) return GSA_ERR_ARG;
    const int64_t rows = (int64_t)d->batch * d->n_kv_heads;
    const int64_t unit = (int64_t)d->chunk + (d->mode == GSA_SELECTED_PAIRS ? 1 : 0);
    const int64_t kb = (int64_t)d->top_k * unit + d->tail_len;
    // element counts must fit the kernels' 32-bit per-row key arithmetic
    if (kb > INT32_MAX / 2 || (int64_t)d->n_chunks * d->chunk > INT32_MAX / 2) return GSA_ERR_SHAPE;
    if (rows > 65535) return GSA_ERR_SHAPE;   // grid.y
    // gists in the context: all, the selected ones (counted in kb), none, or the unselected ones
    const int64_t gists = d->mode == GSA_ALL_GISTS ? d->n_chunks
                        : d->mode == GSA_UNSELECTED_GISTS ? (int64_t)d->n_chunks - d->top_k : 0;
    const int64_t ctx = gists + kb;
    if (ctx <= 0) return GSA_ERR_ARG;         // empty attention context
    return GSA_OK;
}

struct DecodePlan {
    int rows, G, tile;
    int SA, tprA;          // gist pass
    int SB, tprB, KB, U;   // unfold pass
    int64_t candA;         // candidates per row
    size_t off_err, off_cnt, off_scores, off_cand_key, off_cand_idx, off_idx;
    size_t off_partA, off_mlA, off_partB, off_mlB, total;
};

inline int split_len(int s, int S, int tpr, int tile, int n) {
    const int t0 = (int)((int64_t)s * tpr / S), t1 = (int)((int64_t)(s + 1) * tpr / S);
    return std::min(t1 * tile, n) - t0 * tile;
}

inline DecodePlan make_decode_plan(const gsa_decode_desc& d) {
    DecodePlan p{};
    p.rows = d.batch * d.n_kv_heads;
    p.G = d.n_q_heads / d.n_kv_heads;
    p.tile = stage_keys(d.dtype, d.head_dim);
    const int N = d.n_chunks;
    p.tprA = (N + p.tile - 1) / p.tile;
    p.SA = p.tprA == 0 ? 0 : std::min({p.tprA, std::max(1, kTargetGistCtas / p.rows), kMaxSplits});
    p.U = d.chunk + (d.mode == GSA_SELECTED_PAIRS ? 1 : 0);
    p.KB = d.top_k * p.U + d.tail_len;
    p.tprB = (p.KB + p.tile - 1) / p.tile;
    p.SB = std::max(1, std::min({p.tprB, std::max(1, kTargetUnfoldCtas / p.rows), kMaxSplits}));
    p.candA = 0;
    for (int s = 0; s < p.SA; ++s) p.candA += std::min(d.top_k, split_len(s, p.SA, p.tprA, p.tile, N));
    const size_t rows = (size_t)p.rows;
    size_t o = 0;
    p.off_err = kWsErrOffset;
    p.off_cnt = kWsCntOffset;
    o = round256(kWsCntOffset + 2 * rows * 4);
    p.off_scores = o;
    o = round256(o + rows * (size_t)N * 4);
    p.off_cand_key = o;
    o = round256(o + rows * (size_t)p.candA * 4);
    p.off_cand_idx = o;
    o = round256(o + rows * (size_t)p.candA * 4);
    p.off_idx = o;
    o = round256(o + rows * (size_t)d.top_k * 4);
    p.off_partA = o;
    o = round256(o + rows * (size_t)p.SA * p.G * d.head_dim * 4);
    p.off_mlA = o;
    o = round256(o + rows * (size_t)p.SA * p.G * 2 * 4);
    p.off_partB = o;
    o = round256(o + rows * (size_t)p.SB * p.G * d.head_dim * 4);
    p.off_mlB = o;
    o = round256(o + rows * (size_t)p.SB * p.G * 2 * 4);
    p.total = o;
    return p;
}

}  // namespace gsa

namespace gsa {

inline gsa_status validate_hier(const gsa_hier_desc* h) {
    if (!h) return GSA_ERR_ARG;
    gsa_status st = validate_decode(&h->l1);
    if (st != GSA_OK) return st;
    const gsa_decode_desc& d = h->l1;
    if (d.mode != GSA_ALL_GISTS) return GSA_ERR_ARG;
    if (h->group < 1 || d.n_chunks < 1) return GSA_ERR_ARG;
    if (h->n_l2 != (d.n_chunks + h->group - 1) / h->group) return GSA_ERR_SHAPE;
    if (h->top_k2 < 1 || h->top_k2 > h->n_l2) return GSA_ERR_ARG;
    if ((int64_t)h->top_k2 * h->group > INT32_MAX / 2) return GSA_ERR_SHAPE;
    // k1 must not exceed the fewest candidates the level-2 selection can yield
    const int64_t last = d.n_chunks - (int64_t)(h->n_l2 - 1) * h->group;
    if (d.top_k > (int64_t)(h->top_k2 - 1) * h->group + last) return GSA_ERR_ARG;
    return GSA_OK;
}

struct HierPlan {
    gsa_decode_desc l2desc;   // level-2 pass as a flat descriptor (N = n_l2, k = k2)
    DecodePlan l2, l1;        // l2: pass 1; l1: unfold pass of the level-1 descriptor
    int Nv1, tprA1, SA1, SA2;
    size_t off_scores2, off_scores1, off_cand_key, off_cand_idx, off_idx2, off_idx1;
    size_t off_partA, off_mlA, off_partB, off_mlB, total;
};

inline HierPlan make_hier_plan(const gsa_hier_desc& h) {
    HierPlan p{};
    const gsa_decode_desc& d = h.l1;
    p.l2desc = d;
    p.l2desc.n_chunks = h.n_l2;
    p.l2desc.top_k = h.top_k2;
    p.l2 = make_decode_plan(p.l2desc);
    p.l1 = make_decode_plan(d);
    p.SA2 = p.l2.SA;
    p.Nv1 = h.top_k2 * h.group;
    p.tprA1 = (p.Nv1 + p.l1.tile - 1) / p.l1.tile;
    p.SA1 = std::min({p.tprA1, std::max(1, kTargetGistCtas / p.l1.rows), kMaxSplits});
    const size_t rows = (size_t)p.l1.rows;
    const int G = p.l1.G, D = d.head_dim;
    size_t o = round256(kWsCntOffset + 2 * rows * 4);
    p.off_scores2 = o;
    o = round256(o + rows * (size_t)h.n_l2 * 4);
    p.off_scores1 = o;
    o = round256(o + rows * (size_t)p.Nv1 * 4);
    p.off_cand_key = o;
    o = round256(o + rows * (size_t)p.l2.candA * 4);
    p.off_cand_idx = o;
    o = round256(o + rows * (size_t)p.l2.candA * 4);
    p.off_idx2 = o;
    o = round256(o + rows * (size_t)h.top_k2 * 4);
    p.off_idx1 = o;
    o = round256(o + rows * (size_t)d.top_k * 4);
    p.off_partA = o;
    o = round256(o + rows * (size_t)(p.SA2 + p.SA1) * G * D * 4);
    p.off_mlA = o;
    o = round256(o + rows * (size_t)(p.SA2 + p.SA1) * G * 2 * 4);
    p.off_partB = o;
    o = round256(o + rows * (size_t)p.l1.SB * G * D * 4);
    p.off_mlB = o;
    o = round256(o + rows * (size_t)p.l1.SB * G * 2 * 4);
    p.total = o;
    return p;
}

}  // namespace gsa

namespace gsa {

// Gists per level of a hierarchy of any depth: n[0] = N, n[i+1] = ceil(n[i] / group[i]).
inline void level_counts(const gsa_levels_desc& h, int* n) {
    n[0] = h.l1.n_chunks;
    for (int i = 0; i + 1 < h.levels; ++i) n[i + 1] = (n[i] + h.group[i] - 1) / h.group[i];
}
// Selection size at level lv + 1 (lv = 0: level 1).
inline int level_k(const gsa_levels_desc& h, int lv) { return lv == 0 ? h.l1.top_k : h.top_k[lv - 1]; }

inline gsa_status validate_levels(const gsa_levels_desc* h) {
    if (!h) return GSA_ERR_ARG;
    gsa_status st = validate_decode(&h->l1);
    if (st != GSA_OK) return st;
    if (h->l1.mode != GSA_ALL_GISTS || h->l1.n_chunks < 1) return GSA_ERR_ARG;
    if (h->levels < 2 || h->levels > GSA_MAX_LEVELS) return GSA_ERR_ARG;
    for (int i = 0; i + 1 < h->levels; ++i)
        if (h->group[i] < 1 || h->top_k[i] < 1) return GSA_ERR_ARG;
    int n[GSA_MAX_LEVELS];
    level_counts(*h, n);
    const int L = h->levels;
    if (level_k(*h, L - 1) > n[L - 1]) return GSA_ERR_ARG;
    for (int lv = L - 2; lv >= 0; --lv) {
        // fewest candidates: k full groups of the level above but the shortest (its last) one
        const int g = h->group[lv], kp = level_k(*h, lv + 1);
        const int64_t last = n[lv] - (int64_t)(n[lv + 1] - 1) * g;
        if ((int64_t)kp * g > INT32_MAX / 2) return GSA_ERR_SHAPE;
        if (level_k(*h, lv) > (int64_t)(kp - 1) * g + last) return GSA_ERR_ARG;
    }
    return GSA_OK;
}

// Passes: the top level flat (pass 0), each lower level over the children
// of the selection above (passes 1 .. L-1, level L-1 down to 1), then the
// unfold pass of the level-1 descriptor.
struct LevelsPlan {
    int L, n[GSA_MAX_LEVELS];
    gsa_decode_desc topdesc;       // the top level as a flat descriptor
    DecodePlan top, l1;            // pass 0; the unfold pass
    int Nv[GSA_MAX_LEVELS], tpr[GSA_MAX_LEVELS], SA[GSA_MAX_LEVELS];   // by level index (0 = level 1)
    int slot_base[GSA_MAX_LEVELS], slots;
    size_t off_scores[GSA_MAX_LEVELS], off_idx[GSA_MAX_LEVELS];
    size_t off_cand_key, off_cand_idx, off_partA, off_mlA, off_partB, off_mlB, total;
};

inline LevelsPlan make_levels_plan(const gsa_levels_desc& h) {
    LevelsPlan p{};
    const gsa_decode_desc& d = h.l1;
    p.L = h.levels;
    level_counts(h, p.n);
    const int top = p.L - 1;
    p.topdesc = d;
    p.topdesc.n_chunks = p.n[top];
    p.topdesc.top_k = level_k(h, top);
    p.top = make_decode_plan(p.topdesc);
    p.l1 = make_decode_plan(d);
    const int rows = p.l1.rows, tile = p.l1.tile;
    p.Nv[top] = p.n[top];
    p.tpr[top] = p.top.tprA;
    p.SA[top] = p.top.SA;
    p.slot_base[top] = 0;
    p.slots = p.SA[top];
    for (int lv = top - 1; lv >= 0; --lv) {
        p.Nv[lv] = level_k(h, lv + 1) * h.group[lv];
        p.tpr[lv] = (p.Nv[lv] + tile - 1) / tile;
        p.SA[lv] = std::min({p.tpr[lv], std::max(1, kTargetGistCtas / rows), kMaxSplits});
        p.slot_base[lv] = p.slots;
        p.slots += p.SA[lv];
    }
    const size_t R = (size_t)rows;
    const int G = p.l1.G, D = d.head_dim;
    size_t o = round256(kWsCntOffset + 2 * R * 4);
    for (int lv = 0; lv < p.L; ++lv) {
        p.off_scores[lv] = o;
        o = round256(o + R * (size_t)p.Nv[lv] * 4);
        p.off_idx[lv] = o;
        o = round256(o + R * (size_t)level_k(h, lv) * 4);
    }
    p.off_cand_key = o;
    o = round256(o + R * (size_t)p.top.candA * 4);
    p.off_cand_idx = o;
    o = round256(o + R * (size_t)p.top.candA * 4);
    p.off_partA = o;
    o = round256(o + R * (size_t)p.slots * G * D * 4);
    p.off_mlA = o;
    o = round256(o + R * (size_t)p.slots * G * 2 * 4);
    p.off_partB = o;
    o = round256(o + R * (size_t)p.l1.SB * G * D * 4);
    p.off_mlB = o;
    o = round256(o + R * (size_t)p.l1.SB * G * 2 * 4);
    p.total = o;
    return p;
}

}  // namespace gsa
