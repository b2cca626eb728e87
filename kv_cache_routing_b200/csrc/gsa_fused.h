// Host interface of the fused tensor-core decode step (bf16, head_dim 128).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "gsa_plan.h"

namespace gsa {

constexpr int kFusedCtas = 148;   // at most one persistent CTA per B200 SM (the work split is fixed by this, not the device)
constexpr int kSelCap = 2048;     // largest top_k of the tensor-core path (selection kept in shared memory)
constexpr int kMaxTpc = 8;        // largest number of gathered tiles one unfold item takes

struct FusedPlan {
    int rows, G, tg, tt, upr, grid;   // units per row, Stream-K grid (one launch)
    int T;                            // units in all
    int maxs;                         // most CTAs meeting one row (its key/value partial slots)
    int nrows_g, nbt, tpc, cb;        // unfold: gathered rows / tiles per row, tiles per item, items per row
    int items;                        // unfold items in all (rows * cb)
    int slot_stride;                  // maxs + unfold partial slots
    int sel_direct;                   // the selection is taken from the scores (else from per-CTA candidates)
    int attn_gists;                   // gist tiles are attended (ALL_GISTS)
    int tmem_cols;                    // TMEM columns a CTA allocates (S, O^T, kept logits and maxima)
    size_t off_scores, off_cand_key, off_cand_idx, off_idx, off_part, off_ml, total;
    size_t off_idx1;                  // hierarchy: level-1 selection (when the caller passes none)
};

namespace fused {
struct Params {
    CUtensorMap tm_kg, tm_vg;      // gists  [rows][N][d], box {64, 128, 1}
    CUtensorMap tm_kt, tm_vt;      // tail   [rows][W][d], box {64, 128, 1}
    CUtensorMap tm_kr, tm_vr;      // raw [rows][N c][d], or pages [n_pages Hkv][c][d]; box {64, c, 1} (chunk gathers by TMA)
    CUtensorMap tm_kc, tm_vc;      // hierarchy: level-1 gists [rows][N1][d], box {64, group, 1}
    const uint16_t* q;             // [B][Hq][d]
    const uint8_t* kr;             // raw K/V and gist K/V base pointers (gathered tiles)
    const uint8_t* vr;
    const uint8_t* kgp;
    const uint8_t* vgp;
    uint16_t* out;                 // [B][Hq][d]
    float* lse;                    // [B][Hq] or null
    float* scores;                 // [rows][N]
    int32_t* idx;                  // [rows][K]: written by the selection, or given
    uint32_t* err;
    uint32_t* cnt;                 // [rows] tickets: partials written
    uint32_t* kdone;               // [rows] CTAs whose key stretch over the row is done
    uint32_t* cand_key;            // [rows][N] local top-k candidates (orderable score keys)
    int32_t* cand_idx;             // [rows][N] their gist indices
    float* part;                   // [rows][slot_stride][G][d]
    float* ml;                     // [rows][slot_stride][G][4]: (m, l, unused, unused)
    int rows, Hkv, G, N, NA, C, K, W, mode;
    int tg, upr, grid, slot_stride, maxs;
    int nrows_g, nbt, tpc, cb, items;
    int T;                         // units in all
    int tma_raw;                   // chunks are gathered by TMA (c % 8 == 0 and c divides 128)
    int tma_children;              // the children groups are gathered by TMA (same rule for group)
    int tmem_cols;                 // TMEM columns a CTA allocates
    float c2;
    int do_score, do_topk, do_attn_gists, sel_direct;
    int mask_sel;                  // given selection, UNSELECTED_GISTS: its gists are masked in the key stretch
    // paged raw cache (table != null): chunk j of sequence b is page table[b N + j] of the
    // pools [n_pages][Hkv][c][d]; nch (may be null) holds each sequence's chunk count
    const int32_t* table;
    const int32_t* nch;
    int n_pages;
    // hierarchy (keys/values: level-2 gists; unfold: children tile, then raw tile)
    int hier, group, N1, K1;       // K = k2, N = NA = n_l2; group, level-1 gists, k1
    int32_t* idx1;                 // [rows][k1]
    // any depth: L = levels (2 for the two-level step; K, N are the top level's);
    // grp[l - 1] level-l gists per level-(l + 1) gist; the middle levels 2 .. L-1:
    // gist counts, selection sizes, selection outputs, gist maps (box {64, grp[l - 1], 1})
    int levels;
    int grp[3];
    int midN[2], midK[2];
    int32_t* midIdx[2];
    CUtensorMap tm_kcm[2], tm_vcm[2];
};
}  // namespace fused

bool fused_supported(const gsa_decode_desc& d);
// The hierarchy on the same kernel: the children of the selected groups must
// fit one 128-row tile, and so must the raw tokens of the k1 chunks.
bool fused_hier_supported(const gsa_hier_desc& h);
FusedPlan make_fused_hier_plan(const gsa_hier_desc& h);
// Any depth on the same kernel (up to 4 levels): each level's children of the
// selection above must fit one 128-row tile (by TMA: the groups are whole
// 16-byte-aligned runs), and so must the raw tokens of the level-1 selection.
bool fused_levels_supported(const gsa_levels_desc& h);
FusedPlan make_fused_levels_plan(const gsa_levels_desc& h);
// kg / vg: host arrays of the L levels' gist tensors, level 1 first; idx_out:
// null or a host array of L nullable selection outputs.
gsa_status fused_levels_launch(const gsa_levels_desc& h, const FusedPlan& f, const void* q, const void* const* kg,
                               const void* const* vg, const void* kr, const void* vr, const void* kt, const void* vt,
                               int32_t* const* idx_out, void* out, void* ws, cudaStream_t st);
gsa_status fused_hier_launch(const gsa_hier_desc& h, const FusedPlan& f, const void* q, const void* k_g2,
                             const void* v_g2, const void* k_g1, const void* v_g1, const void* kr, const void* vr,
                             const void* kt, const void* vt, int32_t* idx2_out, int32_t* idx1_out, void* out,
                             void* ws, cudaStream_t st);
// given: the selection is supplied (gsa_unfold_attn), so nothing is scored.
FusedPlan make_fused_plan(const gsa_decode_desc& d, bool given = false);
// Enqueue the fused decode step (one launch).  idx_given != null: attend over
// that selection (no scores, no selection); else select and write idx_out (or
// the workspace copy) and scores_out (or the workspace copy).
// pg (may be null): kr / vr are page pools and the chunks are found through pg's table.
gsa_status fused_launch(const gsa_decode_desc& d, const FusedPlan& f, const void* q, const void* kg, const void* vg,
                        const void* kr, const void* vr, const void* kt, const void* vt, const int32_t* idx_given,
                        int32_t* idx_out, float* scores_out, void* out, float* lse, void* ws, cudaStream_t st,
                        const Paging* pg = nullptr);

}  // namespace gsa
