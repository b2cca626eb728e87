// Flat GSA decode on B200: routing scores, top-k, selective unfolding and the
// hybrid attention, as two kernels chained by programmatic dependent launch.
//
//   gist pass   grid (S_A splits, B*Hkv rows).  Streams the split's gist keys
//               (and, in ALL_GISTS mode, gist values) once through a TMA ring.
//               Writes the routing score of every gist, accumulates the
//               attention of the G heads over these gists, keeps the split's
//               local top-k, and the row's last CTA (atomic ticket) merges the
//               local candidates into the row's exact top-k.
//   unfold pass grid (S_B splits, rows).  After the gist pass completes, bulk-
//               copies the selected chunks' raw K/V (and, in SELECTED_PAIRS
//               mode, the selected gists) plus the tail, attends over them, and
//               the row's last CTA merges every partial (log-sum-exp) into out.
//
// Method: gist.science explainer (EN), section 2 "Methodology": gist as
// routing signals, selective unfolding, hybrid attention; Taki-lab slides
// page 6 (score every gist, take top-k, restore chunks with their gists) and
// page 17 (AG+SR / SG+SR context rules).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "gsa_attn.cuh"
#include "gsa_fused.h"
#include "gsa_plan.h"

namespace gsa {

__device__ uint32_t g_err_sink;   // error word for entry points without a workspace

// ------------------------------------------------------------------ params --
struct PassParams {
    int rows, Hkv, N, C, K, W, mode;
    float c2;                         // softmax scale * log2(e)
    const uint8_t* q;                 // [B][Hq][d]
    const uint8_t* kg;                // [rows][N][d]
    const uint8_t* vg;
    const uint8_t* kr;                // [rows][N][c][d]
    const uint8_t* vr;
    const uint8_t* kt;                // [rows][W][d]
    const uint8_t* vt;
    const int32_t* idx_in;            // selection read by the unfold pass
    float* scores;                    // [rows][N]
    int32_t* idx_out;                 // [rows][K] written by the gist pass
    uint8_t* out;                     // [B][Hq][d]
    float* lse;                       // [B][Hq] or null
    uint32_t* err;
    uint32_t* cntA;
    uint32_t* cntB;
    uint32_t* cand_key;               // [rows][candA]
    int32_t* cand_idx;
    float* partA;                     // [rows][SA][G][d]
    float* mlA;                       // [rows][SA][G][2]
    float* partB;
    float* mlB;
    int SA, tprA;                     // gist pass: splits, stages per row
    int SB, tprB, KB, U;              // unfold pass: splits, stages, keys per row, keys per unit
    int64_t candA;
    int do_score, do_attn, do_topk;   // gist pass work
    int mask_sel;                     // do_attn with a given selection (idx_in) whose gists leave the context
    int local_topk;                   // 1: per-split candidates then merge; 0: last CTA selects from all scores
    int merge_a;                      // unfold pass merges the gist-pass partials
    // gist-pass source: the virtual gist list of a row has Nv entries.  Flat:
    // entry v is gist v.  Gathered (parent_idx != null): entry v is gist
    // parent_idx[row][v / group] * group + v % group (children of selected
    // parent groups, ascending); entries past the row's valid count are empty.
    int Nv;
    const int32_t* parent_idx;        // [rows][parent_k]
    int parent_k, group;
    int slot_base, slot_stride;       // gist-pass partial slots: [rows][slot_stride], this pass at slot_base + s
    // paged raw cache (table != null): chunk j of sequence b is page table[b N + j] of the
    // pools kr / vr [n_pages][Hkv][c][d]; nch (may be null) holds each sequence's chunk count
    const int32_t* table;
    const int32_t* nch;
    int n_pages;
    // selection rows: blockIdx.y = kv row * S + position (S = 1 for a decode step).  causal: the
    // tail of position p is its first p + 1 tokens (a suffix attending to itself); q / out are
    // [B][S][Hq][d]
    int S, causal;
};

// --------------------------------------------------------- shared memory --
template <typename T, int D, int G, int NS>
struct Smem {
    using C = Cfg<T, D, G>;
    alignas(128) uint8_t stage[NS][2][STAGE_TENSOR_BYTES];  // [slot][K|V]
    uint64_t full[NS];
    uint64_t empty[NS];
    WarpScratch<G, C::TW> warp[NCW];
    uint32_t topk[256 + 8 + NTHREADS / 32 + 8];
    int flag;
};

// Combine area inside the (then idle) stage ring.
template <int D, int G>
struct CombineView {
    float* cm;   // [NCW][G]
    float* cl;   // [NCW][G]
    float* co;   // [NCW][G][D]
    __device__ CombineView(uint8_t* base) {
        co = reinterpret_cast<float*>(base);
        cm = co + NCW * G * D;
        cl = cm + NCW * G;
    }
};

// Gist-pass split s of a row covers stages [s*tpr/S, (s+1)*tpr/S).
__device__ __forceinline__ void split_range(int s, int S, int tpr, int& t0, int& t1) {
    t0 = (int)((int64_t)s * tpr / S);
    t1 = (int)((int64_t)(s + 1) * tpr / S);
}

// ============================================================ gist pass ====
// Physical gist index of virtual entry v of a row.
__device__ __forceinline__ int gist_of(const PassParams& p, int row, int v) {
    if (p.parent_idx == nullptr) return v;
    const int u = v / p.group;
    return __ldcg(p.parent_idx + (size_t)row * p.parent_k + u) * p.group + (v - u * p.group);
}

// Chunks of sequence b: nch[b] clamped into [0, N] (a value outside is
// flagged when err is given), or N.
__device__ __forceinline__ int seq_chunks(const int32_t* nch, uint32_t* err, int b, int N) {
    if (nch == nullptr) return N;
    const int n = __ldg(nch + b);
    if (n < 0 || n > N) {
        if (err != nullptr) atomicOr(err, kErrIndex);
        return n < 0 ? 0 : N;
    }
    return n;
}

// Valid entries of a row's virtual gist list.
__device__ __forceinline__ int valid_entries(const PassParams& p, int row, int b) {
    if (p.parent_idx == nullptr) return seq_chunks(p.nch, p.err, b, p.Nv);
    if (p.parent_k == 0) return 0;
    const int last = __ldcg(p.parent_idx + (size_t)row * p.parent_k + p.parent_k - 1);
    return (p.parent_k - 1) * p.group + min(p.group, p.N - last * p.group);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(NTHREADS, 2) gist_pass_kernel(const __grid_constant__ PassParams p) {
    using C = Cfg<T, D, G>;
    constexpr int NS = 3;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    auto& sm = *reinterpret_cast<Smem<T, D, G, NS>*>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int s = blockIdx.x, row = blockIdx.y;        // row: the selection row
    const int kv = row / p.S, pos = row - kv * p.S;    // its K/V row and query position
    const int b = kv / p.Hkv, hk = kv % p.Hkv;
    const bool attn = p.do_attn != 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], NCW);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();                 // previous grid on the stream (parent selection, workspace reuse)
    pdl_launch_dependents();

    int t0, t1;
    split_range(s, p.SA, p.tprA, t0, t1);
    const int nvalid = valid_entries(p, row, b);
    const int j0 = t0 * C::TILE;
    const int j1 = min(t1 * C::TILE, nvalid);
    const int ntiles = j1 > j0 ? (j1 - j0 + C::TILE - 1) / C::TILE : 0;
    const size_t gist_row = (size_t)kv * p.N;       // physical gist rows of this (b, hk)
    const size_t score_row = (size_t)row * p.Nv;     // virtual score entries

    if (warp == NCW) {
        // ------------------------------------------------------- producer --
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            for (int t = 0; t < ntiles; ++t) {
                const int slot = t % NS;
                if (t >= NS && !mbar_wait(&sm.empty[slot], ((t / NS) - 1) & 1, p.err)) break;
                const int g0 = j0 + t * C::TILE;
                const int nk = min(C::TILE, j1 - g0);
                const uint32_t bytes = (uint32_t)nk * C::ROWB;
                mbar_arrive_expect_tx(&sm.full[slot], attn ? 2 * bytes : bytes);
                uint8_t* dk = sm.stage[slot][0];
                uint8_t* dv = sm.stage[slot][1];
                for (int v = g0; v < g0 + nk;) {
                    int run = g0 + nk - v;
                    if (p.parent_idx != nullptr) run = min(run, p.group - v % p.group);
                    const int j = gist_of(p, row, v);
                    const size_t o = (gist_row + j) * C::ROWB;
                    bulk_g2s(dk, p.kg + o, (uint32_t)run * C::ROWB, &sm.full[slot], pol);
                    if (attn) bulk_g2s(dv, p.vg + o, (uint32_t)run * C::ROWB, &sm.full[slot], pol);
                    dk += run * C::ROWB;
                    dv += run * C::ROWB;
                    v += run;
                }
            }
            // drain: the last use of every slot must have landed before exit
            for (int t = max(0, ntiles - NS); t < ntiles; ++t) mbar_wait(&sm.full[t % NS], (t / NS) & 1, p.err);
        }
    } else {
        // ------------------------------------------------------ consumers --
        WarpAttn<T, D, G> wa;
        wa.load_q(reinterpret_cast<const T*>(p.q + (((size_t)b * p.S + pos) * p.Hkv * G + (size_t)hk * G) * C::ROWB),
                  lane);
        auto& ws = sm.warp[warp];
        for (int t = 0; t < ntiles; ++t) {
            const int slot = t % NS;
            if (!mbar_wait(&sm.full[slot], (t / NS) & 1, p.err)) break;
            const int g0 = j0 + t * C::TILE;
            const int nk = min(C::TILE, j1 - g0);
            const int nv = min(C::TW, nk - warp * C::TW);
            if (nv > 0) {
                const uint8_t* kt = sm.stage[slot][0] + warp * C::TW * C::ROWB;
                wa.qk(kt, ws, lane);
                if (p.do_score) {
                    const float sc = wa.score(ws, lane);
                    if (lane < nv) p.scores[score_row + g0 + warp * C::TW + lane] = sc;
                }
                if (p.mask_sel) {
                    // UNSELECTED_GISTS with a given selection: its gists get no weight
                    if (lane < nv) {
                        const int j = gist_of(p, row, g0 + warp * C::TW + lane);
                        bool hit = false;
                        for (int u = 0; u < p.K && !hit; ++u) hit = __ldg(p.idx_in + (size_t)row * p.K + u) == j;
                        if (hit) {
#pragma unroll
                            for (int h = 0; h < G; ++h) ws.lg[lane * G + h] = kNegInf;
                        }
                    }
                    __syncwarp();
                }
                if (attn) wa.softmax_pv(sm.stage[slot][1] + warp * C::TW * C::ROWB, ws, nv, p.c2, lane);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[slot]);
        }
        if (attn) {
            // all consumers are past their last stage read once this barrier passes
            asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
            CombineView<D, G> cv(&sm.stage[0][0][0]);
            wa.finish(cv.cm + warp * G, cv.cl + warp * G, cv.co + warp * G * D, lane);
        }
    }
    __syncthreads();
    if (p.do_score && p.nch != nullptr) {
        // gists past the sequence's chunk count do not exist: score -inf
        for (int j = max(j0, nvalid) + threadIdx.x; j < min(t1 * C::TILE, p.Nv); j += NTHREADS)
            p.scores[score_row + j] = kNegInf;
    }

    if (attn) {
        CombineView<D, G> cv(&sm.stage[0][0][0]);
        const size_t slot = (size_t)row * p.slot_stride + p.slot_base + s;
        cta_combine<D, G>(cv.cm, cv.cl, cv.co, p.partA + slot * G * D, p.mlA + slot * G * 2);
    }
    if (!p.do_topk) return;

    if (p.local_topk) {
        // --------------------------------------- local top-k of this split --
        __syncthreads();   // scores of this split written by this CTA are visible
        int64_t off = 0;   // candidates of earlier splits
        for (int s2 = 0; s2 < s; ++s2) {
            int a0, a1;
            split_range(s2, p.SA, p.tprA, a0, a1);
            const int len = max(0, min(a1 * C::TILE, nvalid) - a0 * C::TILE);
            off += min(p.K, len);
        }
        const float* sc = p.scores + score_row + j0;
        uint32_t* ck = p.cand_key + (size_t)row * p.candA + off;
        int32_t* ci = p.cand_idx + (size_t)row * p.candA + off;
        block_topk<NTHREADS>(
            j1 - j0, p.K, [&](int i) { return order_key(sc[i]); },
            [&](int r, int i) {
                ck[r] = order_key(sc[i]);
                ci[r] = j0 + i;
            },
            sm.topk);
    }
    // ---------------------------------- row ticket: last CTA selects top-k --
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t ticket = atomicAdd(&p.cntA[row], 1u);
        sm.flag = (ticket == (uint32_t)p.SA - 1);
    }
    __syncthreads();
    if (!sm.flag) return;
    __threadfence();
    int32_t* out = p.idx_out + (size_t)row * p.K;
    if (p.local_topk) {
        const uint32_t* ck = p.cand_key + (size_t)row * p.candA;
        const int32_t* ci = p.cand_idx + (size_t)row * p.candA;
        // candidates the splits left (all of candA unless the sequence is short)
        int ncand = 0;
        for (int s2 = 0; s2 < p.SA; ++s2) {
            int a0, a1;
            split_range(s2, p.SA, p.tprA, a0, a1);
            ncand += min(p.K, max(0, min(a1 * C::TILE, nvalid) - a0 * C::TILE));
        }
        block_topk<NTHREADS>(
            ncand, p.K, [&](int i) { return __ldcg(ck + i); },
            [&](int r, int i) { out[r] = gist_of(p, row, __ldcg(ci + i)); }, sm.topk);
        // a sequence shorter than k: its other places are empty
        for (int r = min(p.K, ncand) + threadIdx.x; r < p.K; r += NTHREADS) out[r] = -1;
    } else {
        const float* sc = p.scores + score_row;
        block_topk<NTHREADS>(
            nvalid, p.K, [&](int i) { return order_key(__ldcg(sc + i)); },
            [&](int r, int i) { out[r] = gist_of(p, row, i); }, sm.topk);
    }
    if (threadIdx.x == 0) p.cntA[row] = 0;   // leave the ticket zero for the next pass
}

// ========================================================== unfold pass ====
// First raw row of chunk j of `row`: in the dense cache [rows][N][c], or in
// the page pool [n_pages][Hkv][c] (a page outside the pool is clamped into it
// and flagged).  An empty place reads page 0, which always exists.
__device__ __forceinline__ size_t raw_first_row(const PassParams& p, int row, int j, bool empty) {
    if (p.table == nullptr) return ((size_t)row * p.N + j) * p.C;
    const int b = row / p.Hkv, hk = row - b * p.Hkv;
    int pg = 0;
    if (!empty) {
        pg = __ldg(p.table + (size_t)b * p.N + j);
        if (pg < 0 || pg >= p.n_pages) {
            atomicOr(p.err, kErrIndex);
            pg = pg < 0 ? 0 : p.n_pages - 1;
        }
    }
    return ((size_t)pg * p.Hkv + hk) * p.C;
}

// Unfolded keys of a row, in order: for each selected chunk u (idx order) its
// c raw tokens (then its gist in SELECTED_PAIRS mode), then the W tail tokens.
template <int ROWB>
__device__ __forceinline__ void unfold_issue(const PassParams& p, int row, int kv, int x, int xe, uint8_t* dk,
                                             uint8_t* dv, uint64_t* bar, uint64_t pol) {
    const int kU = p.K * p.U;
    while (x < xe) {
        const uint8_t *sk, *sv;
        int run;
        if (x < kU) {
            const int u = x / p.U, r = x % p.U;
            int j = __ldcg(p.idx_in + (size_t)row * p.K + u);
            const bool empty = j == -1;
            if (empty) {
                j = 0;   // an empty place of a variable-size selection: copied, then masked
            } else if (j < 0 || j >= p.N) {
                atomicOr(p.err, kErrIndex);
                j = j < 0 ? 0 : p.N - 1;
            }
            if (r < p.C) {
                run = min(p.C - r, xe - x);
                const size_t o = (raw_first_row(p, kv, j, empty) + r) * ROWB;
                sk = p.kr + o;
                sv = p.vr + o;
            } else {
                run = 1;
                const size_t o = ((size_t)kv * p.N + j) * ROWB;
                sk = p.kg + o;
                sv = p.vg + o;
            }
        } else {
            const int tt = x - kU;
            run = min(p.W - tt, xe - x);
            const size_t o = ((size_t)kv * p.W + tt) * ROWB;
            sk = p.kt + o;
            sv = p.vt + o;
        }
        bulk_g2s(dk, sk, (uint32_t)run * ROWB, bar, pol);
        bulk_g2s(dv, sv, (uint32_t)run * ROWB, bar, pol);
        dk += run * ROWB;
        dv += run * ROWB;
        x += run;
    }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(NTHREADS, 3) unfold_pass_kernel(const __grid_constant__ PassParams p) {
    using C = Cfg<T, D, G>;
    constexpr int NS = 2;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    auto& sm = *reinterpret_cast<Smem<T, D, G, NS>*>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int s = blockIdx.x, row = blockIdx.y;        // row: the selection row
    const int kv = row / p.S, pos = row - kv * p.S;    // its K/V row and query position
    const int b = kv / p.Hkv, hk = kv % p.Hkv;
    // keys of this row: the unfolded units, then its tail (causal: tokens 0..pos)
    const int KB = p.causal ? p.K * p.U + pos + 1 : p.KB;
    int t0, t1;
    split_range(s, p.SB, p.tprB, t0, t1);
    const int x0 = t0 * C::TILE;
    const int x1 = min(t1 * C::TILE, KB);
    const int ntiles = x1 > x0 ? (x1 - x0 + C::TILE - 1) / C::TILE : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], NCW);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();                 // the gist pass (selection, partials) is complete
    pdl_launch_dependents();

    if (warp == NCW) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            for (int t = 0; t < ntiles; ++t) {
                const int slot = t % NS;
                if (t >= NS && !mbar_wait(&sm.empty[slot], ((t / NS) - 1) & 1, p.err)) break;
                const int xa = x0 + t * C::TILE;
                const int nk = min(C::TILE, x1 - xa);
                mbar_arrive_expect_tx(&sm.full[slot], 2u * nk * C::ROWB);
                unfold_issue<C::ROWB>(p, row, kv, xa, xa + nk, sm.stage[slot][0], sm.stage[slot][1],
                                      &sm.full[slot], pol);
            }
            for (int t = max(0, ntiles - NS); t < ntiles; ++t) mbar_wait(&sm.full[t % NS], (t / NS) & 1, p.err);
        }
    } else {
        WarpAttn<T, D, G> wa;
        wa.load_q(reinterpret_cast<const T*>(p.q + (((size_t)b * p.S + pos) * p.Hkv * G + (size_t)hk * G) * C::ROWB),
                  lane);
        auto& ws = sm.warp[warp];
        for (int t = 0; t < ntiles; ++t) {
            const int slot = t % NS;
            if (!mbar_wait(&sm.full[slot], (t / NS) & 1, p.err)) break;
            const int xa = x0 + t * C::TILE;
            const int nk = min(C::TILE, x1 - xa);
            const int nv = min(C::TW, nk - warp * C::TW);
            if (nv > 0) {
                // keys of an empty place (-1) of the selection take no part
                const int x = xa + warp * C::TW + lane;
                const bool gone = lane < nv && x < p.K * p.U && __ldcg(p.idx_in + (size_t)row * p.K + x / p.U) == -1;
                const uint32_t vmask = ~__ballot_sync(0xFFFFFFFFu, gone);
                wa.qk(sm.stage[slot][0] + warp * C::TW * C::ROWB, ws, lane);
                wa.softmax_pv(sm.stage[slot][1] + warp * C::TW * C::ROWB, ws, nv, p.c2, lane, vmask);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[slot]);
        }
        asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
        CombineView<D, G> cv(&sm.stage[0][0][0]);
        wa.finish(cv.cm + warp * G, cv.cl + warp * G, cv.co + warp * G * D, lane);
    }
    __syncthreads();
    {
        CombineView<D, G> cv(&sm.stage[0][0][0]);
        const size_t slot = (size_t)row * p.SB + s;
        cta_combine<D, G>(cv.cm, cv.cl, cv.co, p.partB + slot * G * D, p.mlB + slot * G * 2);
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t ticket = atomicAdd(&p.cntB[row], 1u);
        sm.flag = (ticket == (uint32_t)p.SB - 1);
    }
    __syncthreads();
    if (!sm.flag) return;
    __threadfence();

    // ------------------------------------- final log-sum-exp merge of a row --
    const int na = p.merge_a ? p.slot_stride : 0;
    const int nslots = na + p.SB;
    float* wgt = reinterpret_cast<float*>(&sm.stage[0][0][0]);   // [nslots][G]
    float* fin = wgt + nslots * G;                                // [G][2]: M, L
    auto ml_of = [&](int sl, int h, int which) -> float {
        return sl < na ? __ldcg(p.mlA + (((size_t)row * p.slot_stride + sl) * G + h) * 2 + which)
                       : __ldcg(p.mlB + (((size_t)row * p.SB + (sl - na)) * G + h) * 2 + which);
    };
    for (int h = warp; h < G; h += NCW + 1) {
        float M = kNegInf;
        for (int sl = lane; sl < nslots; sl += 32) M = fmaxf(M, ml_of(sl, h, 0));
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
        float L = 0.f;
        for (int sl = lane; sl < nslots; sl += 32) {
            const float m = ml_of(sl, h, 0);
            const float w = (m == kNegInf) ? 0.f : exp2f(m - M);
            wgt[sl * G + h] = w;
            L += ml_of(sl, h, 1) * w;
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, o);
        if (lane == 0) {
            fin[h * 2 + 0] = M;
            fin[h * 2 + 1] = L;
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * D; i += NTHREADS) {
        const int h = i / D, e = i % D;
        float acc = 0.f;
        for (int sl = 0; sl < nslots; ++sl) {
            const float w = wgt[sl * G + h];
            const float v = sl < na ? __ldcg(p.partA + (((size_t)row * p.slot_stride + sl) * G + h) * D + e)
                                    : __ldcg(p.partB + (((size_t)row * p.SB + (sl - na)) * G + h) * D + e);
            acc = fmaf(w, v, acc);
        }
        const float r = acc / fin[h * 2 + 1];
        const size_t oi = ((((size_t)b * p.S + pos) * p.Hkv + hk) * G + h) * D + e;
        if constexpr (sizeof(T) == 4) {
            reinterpret_cast<float*>(p.out)[oi] = r;
        } else {
            reinterpret_cast<uint16_t*>(p.out)[oi] = f32_to_bf16_rne(r);
        }
    }
    if (p.lse != nullptr && threadIdx.x < G) {
        const int h = threadIdx.x;
        p.lse[(((size_t)b * p.S + pos) * p.Hkv + hk) * G + h] = (fin[h * 2] + log2f(fin[h * 2 + 1])) * 0.69314718055994531f;
    }
    if (threadIdx.x == 0) p.cntB[row] = 0;
}

// =============================================================== top-k =====
// Standalone selection: one CTA per row over the row's N scores, or over the
// first nch[b] of them (nch may be null) with the places past those empty (-1).
__global__ void __launch_bounds__(NTHREADS) topk_kernel(const float* __restrict__ scores, int N, int K,
                                                        int32_t* __restrict__ idx, const int32_t* __restrict__ nch,
                                                        int Hkv) {
    __shared__ uint32_t sh[256 + 8 + NTHREADS / 32 + 8];
    const int row = blockIdx.x;
    const float* sc = scores + (size_t)row * N;
    int32_t* out = idx + (size_t)row * K;
    pdl_wait();
    const int n = seq_chunks(nch, nullptr, row / Hkv, N);
    block_topk<NTHREADS>(
        n, K, [&](int i) { return order_key(sc[i]); }, [&](int r, int i) { out[r] = i; }, sh);
    for (int r = min(K, n) + threadIdx.x; r < K; r += NTHREADS) out[r] = -1;
}

// =============================================================== top-p =====
// Top-p selection, one CTA per row: the row's softmax weights w = 2^((s -
// max) c2) and their sum Z; the exact top-kmax by the block radix select (in
// index order); each of those ranked in score order (higher score, then the
// lower index) by counting; the weights placed in rank order and prefix-summed
// (a block scan over contiguous segments); the cut is the first rank at which
// the prefix reaches p Z.  The selected positions are written ascending, then
// -1 up to kmax, and their number to count.  NaN scores weigh nothing.
constexpr int kToppMax = 2048;   // largest kmax of gsa_topp
__global__ void __launch_bounds__(NTHREADS) topp_kernel(const float* __restrict__ scores, int N, int kmax, float p,
                                                        float c2, int32_t* __restrict__ idx, int32_t* count) {
    extern __shared__ __align__(16) uint32_t dyn[];   // pos, key, rank [kmax] and weights in rank order [kmax]
    __shared__ uint32_t sh[256 + 8 + NTHREADS / 32 + 8];
    __shared__ float red[NTHREADS / 32];
    __shared__ int cut;
    const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = NTHREADS / 32;
    const float* sc = scores + (size_t)row * N;
    int32_t* pos = reinterpret_cast<int32_t*>(dyn);
    uint32_t* key = dyn + kmax;
    int32_t* rnk = reinterpret_cast<int32_t*>(dyn + 2 * kmax);
    float* wr = reinterpret_cast<float*>(dyn + 3 * kmax);
    pdl_wait();
    const int kk = min(kmax, N);
    // the row's maximum and the softmax normaliser
    float mx = kNegInf;
    for (int i = tid; i < N; i += NTHREADS) mx = fmaxf(mx, sc[i]);
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = red[0];
    for (int w = 1; w < NW; ++w) mx = fmaxf(mx, red[w]);
    __syncthreads();
    auto weight = [&](float x) { return x == x ? exp2f((x - mx) * c2) : 0.f; };
    float z = 0.f;
    for (int i = tid; i < N; i += NTHREADS) z += weight(sc[i]);
    for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, o);
    if (lane == 0) red[warp] = z;
    __syncthreads();
    z = 0.f;
    for (int w = 0; w < NW; ++w) z += red[w];
    const float target = p * z;
    // the top-kmax, in index order
    block_topk<NTHREADS>(
        N, kk, [&](int i) { return order_key(sc[i]); }, [&](int r, int i) { pos[r] = i; }, sh);
    __syncthreads();
    for (int r = tid; r < kk; r += NTHREADS) key[r] = order_key(sc[pos[r]]);
    __syncthreads();
    // rank in score order (pos is ascending, so r' < r means a lower index)
    for (int r = tid; r < kk; r += NTHREADS) {
        const uint32_t kr = key[r];
        int rank = 0;
        for (int q = 0; q < kk; ++q) rank += (key[q] > kr || (key[q] == kr && q < r)) ? 1 : 0;
        rnk[r] = rank;
        wr[rank] = weight(sc[pos[r]]);
    }
    if (tid == 0) cut = kk;
    __syncthreads();
    // prefix sums of the weights in rank order: contiguous segments, then a scan of their totals
    const int seg = (kk + NTHREADS - 1) / NTHREADS;
    const int lo = min(kk, tid * seg), hi = min(kk, lo + seg);
    float part = 0.f;
    for (int t = lo; t < hi; ++t) part += wr[t];
    float incl = part;
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    float before = incl - part;
    for (int w = 0; w < warp; ++w) before += red[w];
    float acc = before;
    for (int t = lo; t < hi; ++t) {
        acc += wr[t];
        if (acc >= target) {
            atomicMin(&cut, t + 1);
            break;
        }
    }
    __syncthreads();
    const int m = max(1, cut);
    // the selected positions (rank < m), ascending, then -1
    uint32_t n_sel = 0;
    for (int t = lo; t < hi; ++t) n_sel += rnk[t] < m ? 1u : 0u;
    uint32_t tot;
    uint32_t at = block_exclusive_scan<NTHREADS>(n_sel, sh, &tot);
    int32_t* out = idx + (size_t)row * kmax;
    for (int t = lo; t < hi; ++t)
        if (rnk[t] < m) out[at++] = pos[t];
    for (int t = m + tid; t < kmax; t += NTHREADS) out[t] = -1;
    if (count != nullptr && tid == 0) count[row] = m;
}

// ============================================================ host side ====
template <typename T, int D, int G>
size_t gist_smem() {
    return sizeof(Smem<T, D, G, 3>);
}
template <typename T, int D, int G>
size_t unfold_smem() {
    return sizeof(Smem<T, D, G, 2>);
}

static cudaError_t launch(const void* fn, dim3 grid, size_t smem, cudaStream_t st, const PassParams& p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {const_cast<PassParams*>(&p)};
    return cudaLaunchKernelExC(&cfg, fn, args);
}

template <typename T, int D, int G>
struct Launcher {
    static void set_attrs() {
        static bool done = false;
        if (!done) {
            cudaFuncSetAttribute(gist_pass_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gist_smem<T, D, G>());
            cudaFuncSetAttribute(unfold_pass_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)unfold_smem<T, D, G>());
            done = true;
        }
    }
    static cudaError_t gist(const PassParams& p, cudaStream_t st) {
        set_attrs();
        if (p.SA <= 0) return cudaSuccess;
        return launch((const void*)gist_pass_kernel<T, D, G>, dim3(p.SA, p.rows), gist_smem<T, D, G>(), st, p);
    }
    static cudaError_t unfold(const PassParams& p, cudaStream_t st) {
        set_attrs();
        return launch((const void*)unfold_pass_kernel<T, D, G>, dim3(p.SB, p.rows), unfold_smem<T, D, G>(), st, p);
    }
};

struct Kernels {
    cudaError_t (*gist)(const PassParams&, cudaStream_t);
    cudaError_t (*unfold)(const PassParams&, cudaStream_t);
};

template <typename T, int D>
static Kernels pick_g(int G) {
    switch (G) {
        case 1: return {Launcher<T, D, 1>::gist, Launcher<T, D, 1>::unfold};
        case 2: return {Launcher<T, D, 2>::gist, Launcher<T, D, 2>::unfold};
        case 4: return {Launcher<T, D, 4>::gist, Launcher<T, D, 4>::unfold};
        default: return {Launcher<T, D, 8>::gist, Launcher<T, D, 8>::unfold};
    }
}

static Kernels pick_kernels(int dtype, int D, int G) {
    if (dtype == GSA_F32) return D == 64 ? pick_g<float, 64>(G) : pick_g<float, 128>(G);
    return D == 64 ? pick_g<bf16_t, 64>(G) : pick_g<bf16_t, 128>(G);
}

static cudaError_t run_passes(const PassParams& p, int dtype, int D, int G, bool gist, bool unfold,
                              cudaStream_t st) {
    Kernels k = pick_kernels(dtype, D, G);
    cudaError_t e = cudaSuccess;
    if (gist && (e = k.gist(p, st)) != cudaSuccess) return e;
    if (unfold) e = k.unfold(p, st);
    return e;
}

// Fill PassParams from a validated descriptor and plan.
static PassParams make_params(const DecodePlan& pl, const gsa_decode_desc& d, const void* q, const void* kg,
                              const void* vg, const void* kr, const void* vr, const void* kt, const void* vt,
                              void* ws) {
    PassParams p;
    std::memset(&p, 0, sizeof(p));
    p.rows = pl.rows;
    p.Hkv = d.n_kv_heads;
    p.N = d.n_chunks;
    p.C = d.chunk;
    p.K = d.top_k;
    p.W = d.tail_len;
    p.mode = d.mode;
    const double scale = d.scale > 0 ? (double)d.scale : 1.0 / std::sqrt((double)d.head_dim);
    p.c2 = (float)(scale * 1.4426950408889634);
    p.q = static_cast<const uint8_t*>(q);
    p.kg = static_cast<const uint8_t*>(kg);
    p.vg = static_cast<const uint8_t*>(vg);
    p.kr = static_cast<const uint8_t*>(kr);
    p.vr = static_cast<const uint8_t*>(vr);
    p.kt = static_cast<const uint8_t*>(kt);
    p.vt = static_cast<const uint8_t*>(vt);
    uint8_t* w = static_cast<uint8_t*>(ws);
    if (w != nullptr) {
        p.err = reinterpret_cast<uint32_t*>(w + pl.off_err);
        p.cntA = reinterpret_cast<uint32_t*>(w + pl.off_cnt);
        p.cntB = p.cntA + pl.rows;
        p.scores = reinterpret_cast<float*>(w + pl.off_scores);
        p.cand_key = reinterpret_cast<uint32_t*>(w + pl.off_cand_key);
        p.cand_idx = reinterpret_cast<int32_t*>(w + pl.off_cand_idx);
        p.idx_out = reinterpret_cast<int32_t*>(w + pl.off_idx);
        p.partA = reinterpret_cast<float*>(w + pl.off_partA);
        p.mlA = reinterpret_cast<float*>(w + pl.off_mlA);
        p.partB = reinterpret_cast<float*>(w + pl.off_partB);
        p.mlB = reinterpret_cast<float*>(w + pl.off_mlB);
    }
    p.SA = pl.SA;
    p.tprA = pl.tprA;
    p.SB = pl.SB;
    p.tprB = pl.tprB;
    p.KB = pl.KB;
    p.U = pl.U;
    p.candA = pl.candA;
    p.local_topk = 1;
    p.Nv = d.n_chunks;
    p.slot_base = 0;
    p.slot_stride = pl.SA;
    p.S = 1;
    p.causal = 0;
    return p;
}

static void set_paging(PassParams& p, const Paging* pg) {
    if (pg == nullptr) return;
    p.table = pg->table;
    p.nch = pg->nch;
    p.n_pages = pg->n_pages;
}

// Workspace bytes of a flat decode descriptor on the path it will take.
static size_t decode_ws_bytes(const gsa_decode_desc& d) {
    return fused_supported(d) ? std::max(make_fused_plan(d).total, make_fused_plan(d, true).total)
                              : make_decode_plan(d).total;
}

// UNSELECTED_GISTS decode step: where the scores and the selection go when the
// caller passes no buffers for them.  Both plans keep score and selection
// regions that the given-selection pass does not use.
// (also the top-p step's, which runs the same three kernels)
static void unselected_scratch(const gsa_decode_desc& d, size_t& off_scores, size_t& off_idx) {
    if (fused_supported(d)) {
        const FusedPlan f = make_fused_plan(d, true);
        off_scores = f.off_scores;
        off_idx = f.off_idx;
    } else {
        const DecodePlan pl = make_decode_plan(d);
        off_scores = pl.off_scores;
        off_idx = pl.off_idx;
    }
}

}  // namespace gsa

// ================================================================ C ABI ====
using namespace gsa;

extern "C" {

size_t gsa_decode_workspace_size(const gsa_decode_desc* desc) {
    if (validate_decode(desc) != GSA_OK) return 0;
    return decode_ws_bytes(*desc);
}

static gsa_status score_impl(const gsa_decode_desc* desc, const void* q, const void* k_gist, float* scores,
                             void* stream, const Paging* pg) {
    gsa_status st = validate_decode(desc);
    if (st != GSA_OK) return st;
    if (!q || (desc->n_chunks > 0 && (!k_gist || !scores))) return GSA_ERR_ARG;
    if (!aligned16(q) || !aligned16(k_gist) || !aligned16(scores)) return GSA_ERR_ALIGN;
    if (desc->n_chunks == 0) return GSA_OK;
    DecodePlan pl = make_decode_plan(*desc);
    PassParams p = make_params(pl, *desc, q, k_gist, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
    uint32_t* sink = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&sink), g_err_sink) != cudaSuccess) return GSA_ERR_CUDA;
    p.err = sink;
    p.scores = scores;
    p.do_score = 1;
    if (pg != nullptr) p.nch = pg->nch;
    cudaError_t e = run_passes(p, desc->dtype, desc->head_dim, desc->n_q_heads / desc->n_kv_heads, true, false,
                               static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

gsa_status gsa_score(const gsa_decode_desc* desc, const void* q, const void* k_gist, float* scores,
                     void* stream) {
    return score_impl(desc, q, k_gist, scores, stream, nullptr);
}

static gsa_status topk_impl(const gsa_decode_desc* desc, const float* scores, int32_t* idx, void* stream,
                            const int32_t* nch) {
    gsa_status st = validate_decode(desc);
    if (st != GSA_OK) return st;
    if (desc->top_k == 0) return GSA_OK;
    if (!scores || !idx) return GSA_ERR_ARG;
    if (!aligned16(scores) || !aligned16(idx)) return GSA_ERR_ALIGN;
    const int rows = desc->batch * desc->n_kv_heads;
    topk_kernel<<<rows, NTHREADS, 0, static_cast<cudaStream_t>(stream)>>>(scores, desc->n_chunks, desc->top_k,
                                                                         idx, nch, desc->n_kv_heads);
    return cudaGetLastError() == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

gsa_status gsa_topk(const gsa_decode_desc* desc, const float* scores, int32_t* idx, void* stream) {
    return topk_impl(desc, scores, idx, stream, nullptr);
}

gsa_status gsa_topp(const gsa_decode_desc* desc, float top_p, const float* scores, int32_t* idx, int32_t* count,
                    void* stream) {
    gsa_status st = validate_decode(desc);
    if (st != GSA_OK) return st;
    if (!(top_p > 0.f && top_p <= 1.f) || desc->top_k < 1) return GSA_ERR_ARG;
    if (desc->top_k > kToppMax) return GSA_ERR_SHAPE;
    if (!scores || !idx) return GSA_ERR_ARG;
    if (!aligned16(scores) || !aligned16(idx) || (reinterpret_cast<uintptr_t>(count) & 3u)) return GSA_ERR_ALIGN;
    const int rows = desc->batch * desc->n_kv_heads;
    const double scale = desc->scale > 0 ? (double)desc->scale : 1.0 / std::sqrt((double)desc->head_dim);
    const size_t smem = (size_t)desc->top_k * 16;
    topp_kernel<<<rows, NTHREADS, smem, static_cast<cudaStream_t>(stream)>>>(
        scores, desc->n_chunks, desc->top_k, top_p, (float)(scale * 1.4426950408889634), idx, count);
    return cudaGetLastError() == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

static gsa_status check_tensors(const gsa_decode_desc* d, const void* q, const void* kg, const void* vg,
                                const void* kr, const void* vr, const void* kt, const void* vt, const void* out) {
    const bool gists_needed = d->n_chunks > 0;
    const bool raw_needed = d->top_k > 0;
    const bool tail_needed = d->tail_len > 0;
    if (!q || !out) return GSA_ERR_ARG;
    const bool gist_attn = d->mode == GSA_ALL_GISTS || d->mode == GSA_UNSELECTED_GISTS;
    if (gists_needed && (!kg || (gist_attn && !vg))) return GSA_ERR_ARG;
    if (raw_needed && (!kr || !vr || (d->mode == GSA_SELECTED_PAIRS && (!kg || !vg)))) return GSA_ERR_ARG;
    if (tail_needed && (!kt || !vt)) return GSA_ERR_ARG;
    const void* all[] = {q, kg, vg, kr, vr, kt, vt, out};
    for (const void* x : all)
        if (!aligned16(x)) return GSA_ERR_ALIGN;
    return GSA_OK;
}

static gsa_status check_ws(size_t need, const void* ws, size_t ws_bytes) {
    if (!ws || ws_bytes < need) return GSA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return GSA_ERR_WORKSPACE;
    return GSA_OK;
}

static gsa_status unfold_impl(const gsa_decode_desc* desc, const void* q, const void* k_gist, const void* v_gist,
                              const void* k_raw, const void* v_raw, const void* k_tail, const void* v_tail,
                              const int32_t* idx, void* out, float* lse, void* ws, size_t ws_bytes, void* stream,
                              const Paging* pg) {
    gsa_status st = validate_decode(desc);
    if (st != GSA_OK) return st;
    if ((st = check_tensors(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, out)) != GSA_OK) return st;
    if (desc->top_k > 0 && (!idx || !aligned16(idx))) return idx ? GSA_ERR_ALIGN : GSA_ERR_ARG;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return GSA_ERR_ALIGN;
    if ((st = check_ws(decode_ws_bytes(*desc), ws, ws_bytes)) != GSA_OK) return st;
    if (fused_supported(*desc))
        return fused_launch(*desc, make_fused_plan(*desc, true), q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, idx,
                            nullptr, nullptr, out, lse, ws, static_cast<cudaStream_t>(stream), pg);
    DecodePlan pl = make_decode_plan(*desc);
    PassParams p = make_params(pl, *desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, ws);
    set_paging(p, pg);
    p.idx_in = idx;
    p.out = static_cast<uint8_t*>(out);
    p.lse = lse;
    p.do_attn = (desc->mode == GSA_ALL_GISTS || desc->mode == GSA_UNSELECTED_GISTS);
    p.mask_sel = (desc->mode == GSA_UNSELECTED_GISTS);
    p.merge_a = p.do_attn && desc->n_chunks > 0;
    cudaError_t e = run_passes(p, desc->dtype, desc->head_dim, desc->n_q_heads / desc->n_kv_heads, p.merge_a != 0,
                               true, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

gsa_status gsa_unfold_attn(const gsa_decode_desc* desc, const void* q, const void* k_gist, const void* v_gist,
                           const void* k_raw, const void* v_raw, const void* k_tail, const void* v_tail,
                           const int32_t* idx, void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
    return unfold_impl(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, idx, out, lse, ws, ws_bytes, stream,
                       nullptr);
}

static gsa_status step_impl(const gsa_decode_desc* desc, const void* q, const void* k_gist, const void* v_gist,
                            const void* k_raw, const void* v_raw, const void* k_tail, const void* v_tail,
                            int32_t* idx_out, float* scores_out, void* out, void* ws, size_t ws_bytes, void* stream,
                            const Paging* pg) {
    gsa_status st = validate_decode(desc);
    if (st != GSA_OK) return st;
    if ((st = check_tensors(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, out)) != GSA_OK) return st;
    if (!aligned16(idx_out) || !aligned16(scores_out)) return GSA_ERR_ALIGN;
    if ((st = check_ws(decode_ws_bytes(*desc), ws, ws_bytes)) != GSA_OK) return st;
    if (desc->mode == GSA_UNSELECTED_GISTS && desc->top_k > 0) {
        // the gist attention needs the selection first: score, select, then
        // attend with the selection given (its gists masked out).  The scores
        // and the selection go to the caller's buffers or to workspace
        // regions the given-selection pass leaves unused.
        uint8_t* w = static_cast<uint8_t*>(ws);
        size_t off_s, off_i;
        unselected_scratch(*desc, off_s, off_i);
        float* sc = scores_out ? scores_out : reinterpret_cast<float*>(w + off_s);
        int32_t* ix = idx_out ? idx_out : reinterpret_cast<int32_t*>(w + off_i);
        if ((st = score_impl(desc, q, k_gist, sc, stream, pg)) != GSA_OK) return st;
        if ((st = topk_impl(desc, sc, ix, stream, pg ? pg->nch : nullptr)) != GSA_OK) return st;
        return unfold_impl(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, ix, out, nullptr, ws, ws_bytes,
                           stream, pg);
    }
    if (fused_supported(*desc))
        return fused_launch(*desc, make_fused_plan(*desc), q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, nullptr,
                            idx_out, scores_out, out, nullptr, ws, static_cast<cudaStream_t>(stream), pg);
    DecodePlan pl = make_decode_plan(*desc);
    PassParams p = make_params(pl, *desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, ws);
    set_paging(p, pg);
    if (scores_out) p.scores = scores_out;
    if (idx_out) p.idx_out = idx_out;
    p.idx_in = p.idx_out;
    p.out = static_cast<uint8_t*>(out);
    p.do_score = 1;
    p.do_topk = 1;
    p.do_attn = (desc->mode == GSA_ALL_GISTS || desc->mode == GSA_UNSELECTED_GISTS);   // (k = 0 here: nothing to mask)
    p.merge_a = p.do_attn && desc->n_chunks > 0;
    cudaError_t e = run_passes(p, desc->dtype, desc->head_dim, desc->n_q_heads / desc->n_kv_heads,
                               desc->n_chunks > 0, true, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

gsa_status gsa_decode_step(const gsa_decode_desc* desc, const void* q, const void* k_gist, const void* v_gist,
                           const void* k_raw, const void* v_raw, const void* k_tail, const void* v_tail,
                           int32_t* idx_out, float* scores_out, void* out, void* ws, size_t ws_bytes,
                           void* stream) {
    return step_impl(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, idx_out, scores_out, out, ws, ws_bytes,
                     stream, nullptr);
}

gsa_status gsa_decode_step_paged(const gsa_decode_desc* desc, const void* q, const void* k_gist, const void* v_gist,
                                 const void* k_pages, const void* v_pages, int32_t n_pages,
                                 const int32_t* block_table, const int32_t* seq_chunks, const void* k_tail,
                                 const void* v_tail, int32_t* idx_out, float* scores_out, void* out, void* ws,
                                 size_t ws_bytes, void* stream) {
    gsa_status st = validate_decode(desc);
    if (st != GSA_OK) return st;
    if (n_pages < 1 || !block_table) return GSA_ERR_ARG;
    // a short sequence keeps the tail as its context, so the tail may not be empty
    if (seq_chunks && desc->tail_len < 1) return GSA_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_chunks) & 3u))
        return GSA_ERR_ALIGN;
    // pool rows are addressed with 32-bit arithmetic
    if ((int64_t)n_pages * desc->n_kv_heads * desc->chunk > INT32_MAX / 2) return GSA_ERR_SHAPE;
    const Paging pg{block_table, seq_chunks, n_pages};
    return step_impl(desc, q, k_gist, v_gist, k_pages, v_pages, k_tail, v_tail, idx_out, scores_out, out, ws,
                     ws_bytes, stream, &pg);
}


gsa_status gsa_decode_step_topp(const gsa_decode_desc* desc, float top_p, const void* q, const void* k_gist,
                                const void* v_gist, const void* k_raw, const void* v_raw, const void* k_tail,
                                const void* v_tail, int32_t* idx_out, int32_t* count_out, float* scores_out,
                                void* out, void* ws, size_t ws_bytes, void* stream) {
    gsa_status st = validate_decode(desc);
    if (st != GSA_OK) return st;
    if (!(top_p > 0.f && top_p <= 1.f) || desc->top_k < 1) return GSA_ERR_ARG;
    if (desc->top_k > kToppMax) return GSA_ERR_SHAPE;
    if ((st = check_tensors(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, out)) != GSA_OK) return st;
    if (!aligned16(idx_out) || !aligned16(scores_out) || (reinterpret_cast<uintptr_t>(count_out) & 3u))
        return GSA_ERR_ALIGN;
    if ((st = check_ws(decode_ws_bytes(*desc), ws, ws_bytes)) != GSA_OK) return st;
    uint8_t* w = static_cast<uint8_t*>(ws);
    size_t off_s, off_i;
    unselected_scratch(*desc, off_s, off_i);
    float* sc = scores_out ? scores_out : reinterpret_cast<float*>(w + off_s);
    int32_t* ix = idx_out ? idx_out : reinterpret_cast<int32_t*>(w + off_i);
    if ((st = gsa_score(desc, q, k_gist, sc, stream)) != GSA_OK) return st;
    if ((st = gsa_topp(desc, top_p, sc, ix, count_out, stream)) != GSA_OK) return st;
    return gsa_unfold_attn(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, ix, out, nullptr, ws, ws_bytes,
                           stream);
}

// Hierarchical decode ([EN-2] "Hierarchical Extension (H-GSA)"; slide page 11):
// gist pass over the level-2 gists (scores, attention, top-k2), gist pass over
// the children of the selected groups (scores, attention, top-k1), unfold pass
// over the raw tokens of the k1 chunks and the tail, merging all partials.
size_t gsa_hier_workspace_size(const gsa_hier_desc* desc) {
    if (validate_hier(desc) != GSA_OK) return 0;
    return fused_hier_supported(*desc) ? make_fused_hier_plan(*desc).total : make_hier_plan(*desc).total;
}

gsa_status gsa_hier_decode(const gsa_hier_desc* desc, const void* q, const void* k_g2, const void* v_g2,
                           const void* k_g1, const void* v_g1, const void* k_raw, const void* v_raw,
                           const void* k_tail, const void* v_tail, int32_t* idx2_out, int32_t* idx1_out, void* out,
                           void* ws, size_t ws_bytes, void* stream) {
    gsa_status st = validate_hier(desc);
    if (st != GSA_OK) return st;
    const gsa_decode_desc& d = desc->l1;
    if (!q || !k_g2 || !v_g2 || !k_g1 || !v_g1 || !out) return GSA_ERR_ARG;
    if (d.top_k > 0 && (!k_raw || !v_raw)) return GSA_ERR_ARG;
    if (d.tail_len > 0 && (!k_tail || !v_tail)) return GSA_ERR_ARG;
    const void* all[] = {q, k_g2, v_g2, k_g1, v_g1, k_raw, v_raw, k_tail, v_tail, idx2_out, idx1_out, out};
    for (const void* x : all)
        if (!aligned16(x)) return GSA_ERR_ALIGN;
    if (fused_hier_supported(*desc)) {
        // tensor-core path: level-2 gists and tail streamed, then per row the
        // children tile (scored and attended) and the raw tile of the k1 chunks
        const FusedPlan f = make_fused_hier_plan(*desc);
        if (!ws || ws_bytes < f.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return GSA_ERR_WORKSPACE;
        return fused_hier_launch(*desc, f, q, k_g2, v_g2, k_g1, v_g1, k_raw, v_raw, k_tail, v_tail, idx2_out,
                                 idx1_out, out, ws, static_cast<cudaStream_t>(stream));
    }
    const HierPlan hp = make_hier_plan(*desc);
    if (!ws || ws_bytes < hp.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return GSA_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(ws);
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    const int G = d.n_q_heads / d.n_kv_heads;
    int32_t* idx2 = idx2_out ? idx2_out : reinterpret_cast<int32_t*>(w + hp.off_idx2);
    int32_t* idx1 = idx1_out ? idx1_out : reinterpret_cast<int32_t*>(w + hp.off_idx1);

    // pass 1: level-2 gists, flat
    PassParams p = make_params(hp.l2, hp.l2desc, q, k_g2, v_g2, nullptr, nullptr, nullptr, nullptr, ws);
    p.cntA = reinterpret_cast<uint32_t*>(w + hp.l2.off_cnt);
    p.scores = reinterpret_cast<float*>(w + hp.off_scores2);
    p.cand_key = reinterpret_cast<uint32_t*>(w + hp.off_cand_key);
    p.cand_idx = reinterpret_cast<int32_t*>(w + hp.off_cand_idx);
    p.idx_out = idx2;
    p.partA = reinterpret_cast<float*>(w + hp.off_partA);
    p.mlA = reinterpret_cast<float*>(w + hp.off_mlA);
    p.slot_base = 0;
    p.slot_stride = hp.SA2 + hp.SA1;
    p.do_score = p.do_attn = p.do_topk = 1;
    Kernels kern = pick_kernels(d.dtype, d.head_dim, G);
    if (kern.gist(p, strm) != cudaSuccess) return GSA_ERR_CUDA;

    // pass 2: children of the selected level-2 groups
    PassParams c = p;
    c.N = d.n_chunks;
    c.K = d.top_k;
    c.kg = static_cast<const uint8_t*>(k_g1);
    c.vg = static_cast<const uint8_t*>(v_g1);
    c.Nv = hp.Nv1;
    c.parent_idx = idx2;
    c.parent_k = desc->top_k2;
    c.group = desc->group;
    c.SA = hp.SA1;
    c.tprA = hp.tprA1;
    c.scores = reinterpret_cast<float*>(w + hp.off_scores1);
    c.idx_out = idx1;
    c.local_topk = 0;
    c.slot_base = hp.SA2;
    if (kern.gist(c, strm) != cudaSuccess) return GSA_ERR_CUDA;

    // pass 3: raw tokens of the selected level-1 chunks + tail, final merge
    PassParams u = make_params(hp.l1, d, q, k_g1, v_g1, k_raw, v_raw, k_tail, v_tail, ws);
    u.cntB = reinterpret_cast<uint32_t*>(w + hp.l2.off_cnt) + hp.l2.rows;
    u.partA = p.partA;
    u.mlA = p.mlA;
    u.partB = reinterpret_cast<float*>(w + hp.off_partB);
    u.mlB = reinterpret_cast<float*>(w + hp.off_mlB);
    u.idx_in = idx1;
    u.out = static_cast<uint8_t*>(out);
    u.merge_a = 1;
    u.slot_stride = hp.SA2 + hp.SA1;
    if (kern.unfold(u, strm) != cudaSuccess) return GSA_ERR_CUDA;
    return GSA_OK;
}

// ------------------------------------------------ no-allocation variant ----
// Scratch for gsa_decode_step_noalloc: a fixed device array that lives as long
// as the library is loaded, so that callers who may not allocate device memory
// can still run a decode step.  Its size is the largest workspace the variant
// accepts.
constexpr size_t kStaticWsBytes = size_t(8) << 20;   // 8 MiB
static __device__ __align__(256) uint8_t g_static_ws[kStaticWsBytes];

// The CUDA context current on this thread (driver entry point; null if none).
static CUcontext current_context() {
    static std::once_flag once;
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 4000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    });
    CUcontext c = nullptr;
    if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

// Device address of g_static_ws on each device, resolved with that device
// current the first time it is needed there.  (In host code the symbol itself
// is only a stand-in.)  The address is kept together with the context it was
// resolved in: after a device reset the module is loaded again, possibly
// elsewhere, and the address is resolved anew.
static void* static_ws_address(int device, bool resolve = true) {
    static std::mutex mu;
    static void* addr[128] = {};
    static CUcontext ctx[128] = {};
    if (device < 0 || device >= 128) return nullptr;
    const CUcontext cur = current_context();
    std::lock_guard<std::mutex> lock(mu);
    if (addr[device] == nullptr || ctx[device] != cur) {
        if (!resolve) return nullptr;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess) return nullptr;
        addr[device] = p;
        ctx[device] = cur;
    }
    return addr[device];
}

gsa_status gsa_decode_step_noalloc(const gsa_decode_desc* desc, const void* q, const void* k_gist,
                                   const void* v_gist, const void* k_raw, const void* v_raw, const void* k_tail,
                                   const void* v_tail, int32_t* idx_out, float* scores_out, void* out,
                                   void* stream) {
    gsa_status st = validate_decode(desc);
    if (st != GSA_OK) return st;
    if ((st = check_tensors(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, out)) != GSA_OK) return st;
    if (!aligned16(idx_out) || !aligned16(scores_out)) return GSA_ERR_ALIGN;
    const size_t need = decode_ws_bytes(*desc);
    if (need > kStaticWsBytes) return GSA_ERR_WORKSPACE;
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess) return GSA_ERR_CUDA;
    void* ws = static_ws_address(device);
    if (ws == nullptr) return GSA_ERR_CUDA;
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    // the tickets (the words between the error word and the first data region)
    // must start at zero; the error word is kept until gsa_device_error reads it
    const size_t head = fused_supported(*desc) ? make_fused_plan(*desc).off_scores : make_decode_plan(*desc).off_scores;
    if (cudaMemsetAsync(static_cast<uint8_t*>(ws) + kWsCntOffset, 0, head - kWsCntOffset, strm) != cudaSuccess)
        return GSA_ERR_CUDA;
    return gsa_decode_step(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, idx_out, scores_out, out, ws,
                           need, stream);
}

// One decode step with host-side query and output: the query is copied to
// the device, the step runs, and the output (and the selection, when asked)
// is copied back, all enqueued on `stream` in one call.
gsa_status gsa_decode_step_host(const gsa_decode_desc* desc, const void* q_host, void* q, const void* k_gist,
                                const void* v_gist, const void* k_raw, const void* v_raw, const void* k_tail,
                                const void* v_tail, int32_t* idx_out, int32_t* idx_host, void* out, void* out_host,
                                void* ws, size_t ws_bytes, void* stream) {
    gsa_status st = validate_decode(desc);
    if (st != GSA_OK) return st;
    if (!q_host || !out_host || (idx_host && !idx_out)) return GSA_ERR_ARG;
    const size_t qn = (size_t)desc->batch * desc->n_q_heads * desc->head_dim * elem_bytes(desc->dtype);
    const size_t in = (size_t)desc->batch * desc->n_kv_heads * desc->top_k * sizeof(int32_t);
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    // the device-side arguments are checked by the step before anything is enqueued
    if ((st = check_tensors(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, out)) != GSA_OK) return st;
    if (!aligned16(idx_out)) return GSA_ERR_ALIGN;
    if ((st = check_ws(decode_ws_bytes(*desc), ws, ws_bytes)) != GSA_OK) return st;
    if (cudaMemcpyAsync(q, q_host, qn, cudaMemcpyHostToDevice, strm) != cudaSuccess) return GSA_ERR_CUDA;
    if ((st = gsa_decode_step(desc, q, k_gist, v_gist, k_raw, v_raw, k_tail, v_tail, idx_out, nullptr, out, ws,
                              ws_bytes, stream)) != GSA_OK)
        return st;
    if (cudaMemcpyAsync(out_host, out, qn, cudaMemcpyDeviceToHost, strm) != cudaSuccess) return GSA_ERR_CUDA;
    if (idx_host && in > 0 && cudaMemcpyAsync(idx_host, idx_out, in, cudaMemcpyDeviceToHost, strm) != cudaSuccess)
        return GSA_ERR_CUDA;
    return GSA_OK;
}

// Hierarchy of any depth ([EN-2] "Hierarchical Extension (H-GSA)"): the
// top-level gist pass, one gathered gist pass per lower level (the children
// of the selection above: scores, attention, top-k), then the unfold pass
// over the raw tokens of the level-1 selection and the tail, merging the
// partials of every pass.
size_t gsa_levels_workspace_size(const gsa_levels_desc* desc) {
    if (validate_levels(desc) != GSA_OK) return 0;
    return fused_levels_supported(*desc) ? make_fused_levels_plan(*desc).total : make_levels_plan(*desc).total;
}

gsa_status gsa_levels_decode(const gsa_levels_desc* desc, const void* q, const void* const* k_gists,
                             const void* const* v_gists, const void* k_raw, const void* v_raw, const void* k_tail,
                             const void* v_tail, int32_t* const* idx_out, void* out, void* ws, size_t ws_bytes,
                             void* stream) {
    gsa_status st = validate_levels(desc);
    if (st != GSA_OK) return st;
    const gsa_decode_desc& d = desc->l1;
    const int L = desc->levels;
    if (!q || !k_gists || !v_gists || !out) return GSA_ERR_ARG;
    if (d.top_k > 0 && (!k_raw || !v_raw)) return GSA_ERR_ARG;
    if (d.tail_len > 0 && (!k_tail || !v_tail)) return GSA_ERR_ARG;
    for (int lv = 0; lv < L; ++lv) {
        if (!k_gists[lv] || !v_gists[lv]) return GSA_ERR_ARG;
        if (!aligned16(k_gists[lv]) || !aligned16(v_gists[lv])) return GSA_ERR_ALIGN;
        if (idx_out && !aligned16(idx_out[lv])) return GSA_ERR_ALIGN;
    }
    const void* all[] = {q, k_raw, v_raw, k_tail, v_tail, out};
    for (const void* x : all)
        if (!aligned16(x)) return GSA_ERR_ALIGN;
    if (fused_levels_supported(*desc)) {
        // tensor-core path: the top level and the tail streamed, then per row one
        // children tile per lower level and the raw tile, in one launch
        const FusedPlan f = make_fused_levels_plan(*desc);
        if (!ws || ws_bytes < f.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return GSA_ERR_WORKSPACE;
        return fused_levels_launch(*desc, f, q, k_gists, v_gists, k_raw, v_raw, k_tail, v_tail, idx_out, out, ws,
                                   static_cast<cudaStream_t>(stream));
    }
    const LevelsPlan lp = make_levels_plan(*desc);
    if (!ws || ws_bytes < lp.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return GSA_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(ws);
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    const int G = d.n_q_heads / d.n_kv_heads;
    int32_t* idx[GSA_MAX_LEVELS];
    for (int lv = 0; lv < L; ++lv)
        idx[lv] = (idx_out && idx_out[lv]) ? idx_out[lv] : reinterpret_cast<int32_t*>(w + lp.off_idx[lv]);
    Kernels kern = pick_kernels(d.dtype, d.head_dim, G);
    uint32_t* cnt = reinterpret_cast<uint32_t*>(w + kWsCntOffset);
    float* partA = reinterpret_cast<float*>(w + lp.off_partA);
    float* mlA = reinterpret_cast<float*>(w + lp.off_mlA);

    // pass 0: every top-level gist
    const int top = L - 1;
    PassParams p = make_params(lp.top, lp.topdesc, q, k_gists[top], v_gists[top], nullptr, nullptr, nullptr,
                               nullptr, ws);
    p.cntA = cnt;
    p.scores = reinterpret_cast<float*>(w + lp.off_scores[top]);
    p.cand_key = reinterpret_cast<uint32_t*>(w + lp.off_cand_key);
    p.cand_idx = reinterpret_cast<int32_t*>(w + lp.off_cand_idx);
    p.idx_out = idx[top];
    p.partA = partA;
    p.mlA = mlA;
    p.slot_base = lp.slot_base[top];
    p.slot_stride = lp.slots;
    p.do_score = p.do_attn = p.do_topk = 1;
    if (kern.gist(p, strm) != cudaSuccess) return GSA_ERR_CUDA;

    // passes 1 .. L-1: the children of the selection one level up
    for (int lv = top - 1; lv >= 0; --lv) {
        PassParams c = p;
        c.N = lp.n[lv];
        c.K = level_k(*desc, lv);
        c.kg = static_cast<const uint8_t*>(k_gists[lv]);
        c.vg = static_cast<const uint8_t*>(v_gists[lv]);
        c.Nv = lp.Nv[lv];
        c.parent_idx = idx[lv + 1];
        c.parent_k = level_k(*desc, lv + 1);
        c.group = desc->group[lv];
        c.SA = lp.SA[lv];
        c.tprA = lp.tpr[lv];
        c.scores = reinterpret_cast<float*>(w + lp.off_scores[lv]);
        c.idx_out = idx[lv];
        c.local_topk = 0;
        c.slot_base = lp.slot_base[lv];
        if (kern.gist(c, strm) != cudaSuccess) return GSA_ERR_CUDA;
    }

    // raw tokens of the level-1 selection + tail, final merge of every partial
    PassParams u = make_params(lp.l1, d, q, k_gists[0], v_gists[0], k_raw, v_raw, k_tail, v_tail, ws);
    u.cntB = cnt + lp.l1.rows;
    u.partA = partA;
    u.mlA = mlA;
    u.partB = reinterpret_cast<float*>(w + lp.off_partB);
    u.mlB = reinterpret_cast<float*>(w + lp.off_mlB);
    u.idx_in = idx[0];
    u.out = static_cast<uint8_t*>(out);
    u.merge_a = 1;
    u.slot_stride = lp.slots;
    if (kern.unfold(u, strm) != cudaSuccess) return GSA_ERR_CUDA;
    return GSA_OK;
}

int gsa_levels_launch_count(const gsa_levels_desc* desc) {
    if (validate_levels(desc) != GSA_OK) return -1;
    return fused_levels_supported(*desc) ? 1 : desc->levels + 1;
}

// Stage-2 selective-finetuning forward ([EN-2] "Training Procedure";
// slide page 10): every suffix position is a selection row of the CUDA-core
// passes (its own scores and top-k, shared by the G heads of a KV head), the
// suffix tokens 0..p its causal tail.  The plan is the decode plan of a
// batch of B * S rows.
static gsa_decode_desc suffix_rows_desc(const gsa_decode_desc& d) {
    gsa_decode_desc v = d;
    v.batch = d.batch * d.tail_len;
    return v;
}

static gsa_status validate_suffix(const gsa_decode_desc* desc) {
    gsa_status st = validate_decode(desc);
    if (st != GSA_OK) return st;
    if (desc->tail_len < 1) return GSA_ERR_ARG;
    if ((int64_t)desc->batch * desc->tail_len * desc->n_kv_heads > 65535) return GSA_ERR_SHAPE;   // grid.y
    return GSA_OK;
}

size_t gsa_suffix_workspace_size(const gsa_decode_desc* desc) {
    if (validate_suffix(desc) != GSA_OK) return 0;
    return make_decode_plan(suffix_rows_desc(*desc)).total;
}

int gsa_suffix_launch_count(const gsa_decode_desc* desc) {
    if (validate_suffix(desc) != GSA_OK) return -1;
    return desc->mode == GSA_UNSELECTED_GISTS && desc->top_k > 0 ? 3 : 2;
}

gsa_status gsa_suffix_attn(const gsa_decode_desc* desc, const void* q, const void* k_gist, const void* v_gist,
                           const void* k_raw, const void* v_raw, const void* k_suffix, const void* v_suffix,
                           int32_t* idx_out, float* scores_out, void* out, void* ws, size_t ws_bytes, void* stream) {
    gsa_status st = validate_suffix(desc);
    if (st != GSA_OK) return st;
    if ((st = check_tensors(desc, q, k_gist, v_gist, k_raw, v_raw, k_suffix, v_suffix, out)) != GSA_OK) return st;
    if (!aligned16(idx_out) || !aligned16(scores_out)) return GSA_ERR_ALIGN;
    const gsa_decode_desc v = suffix_rows_desc(*desc);
    const DecodePlan pl = make_decode_plan(v);
    if ((st = check_ws(pl.total, ws, ws_bytes)) != GSA_OK) return st;
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    PassParams p = make_params(pl, v, q, k_gist, v_gist, k_raw, v_raw, k_suffix, v_suffix, ws);
    p.S = desc->tail_len;
    p.causal = 1;
    if (scores_out) p.scores = scores_out;
    if (idx_out) p.idx_out = idx_out;
    p.idx_in = p.idx_out;
    p.out = static_cast<uint8_t*>(out);
    p.do_score = 1;
    p.do_topk = 1;
    const int G = desc->n_q_heads / desc->n_kv_heads;
    const bool gists = desc->mode == GSA_ALL_GISTS || desc->mode == GSA_UNSELECTED_GISTS;
    Kernels kern = pick_kernels(desc->dtype, desc->head_dim, G);
    if (desc->mode == GSA_UNSELECTED_GISTS && desc->top_k > 0) {
        // the gist attention needs the selection first: select, then attend
        // with the selection's gists masked out
        if (kern.gist(p, strm) != cudaSuccess) return GSA_ERR_CUDA;
        p.do_score = 0;
        p.do_topk = 0;
        p.do_attn = 1;
        p.mask_sel = 1;
    } else {
        p.do_attn = gists ? 1 : 0;
    }
    p.merge_a = p.do_attn && desc->n_chunks > 0;
    cudaError_t e = run_passes(p, desc->dtype, desc->head_dim, G, desc->n_chunks > 0, true, strm);
    return e == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

int gsa_hier_launch_count(const gsa_hier_desc* desc) {
    if (validate_hier(desc) != GSA_OK) return -1;
    return fused_hier_supported(*desc) ? 1 : 3;
}

int gsa_decode_launch_count(const gsa_decode_desc* desc) {
    if (validate_decode(desc) != GSA_OK) return -1;
    // the attention pass: one fused launch, or the gist pass (if any gists) and the unfold pass
    const bool gist_attn = desc->mode == GSA_ALL_GISTS || desc->mode == GSA_UNSELECTED_GISTS;
    const int attn = fused_supported(*desc) ? 1 : (desc->n_chunks > 0 ? 1 : 0) + 1;
    if (desc->mode == GSA_UNSELECTED_GISTS && desc->top_k > 0)
        return 2 + (fused_supported(*desc) ? 1 : (gist_attn && desc->n_chunks > 0 ? 1 : 0) + 1);
    return attn;
}

gsa_status gsa_device_error(uint32_t* flags_out, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess) return GSA_ERR_CUDA;
    uint32_t* words[3] = {nullptr, nullptr, nullptr};
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&words[0]), g_err_sink) != cudaSuccess ||
        prefill_error_word(&words[1]) != cudaSuccess)
        return GSA_ERR_CUDA;
    // the scratch array's word, if gsa_decode_step_noalloc has run in this context
    words[2] = static_cast<uint32_t*>(static_ws_address(device, false));
    uint32_t got[3] = {0u, 0u, 0u};
    for (int i = 0; i < 3; ++i) {
        if (words[i] == nullptr) continue;
        if (cudaMemcpyAsync(&got[i], words[i], 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
            cudaMemsetAsync(words[i], 0, 4, st) != cudaSuccess)
            return GSA_ERR_CUDA;
    }
    if (cudaStreamSynchronize(st) != cudaSuccess) return GSA_ERR_CUDA;
    const uint32_t f = got[0] | got[1] | got[2];
    if (flags_out) *flags_out = f;
    if (f & kErrTimeout) return GSA_ERR_TIMEOUT;
    if (f & kErrIndex) return GSA_ERR_ARG;
    return GSA_OK;
}

gsa_status gsa_set_wait_limit_ns(uint64_t ns) {
    return set_cross_cta_wait_limit(ns) == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

gsa_status gsa_workspace_error(const void* ws, uint32_t* flags_out, void* stream) {
    if (!ws) return GSA_ERR_WORKSPACE;
    uint32_t f = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&f, static_cast<const uint8_t*>(ws) + kWsErrOffset, 4, cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return GSA_ERR_CUDA;
    if (flags_out) *flags_out = f;
    if (f & kErrTimeout) return GSA_ERR_TIMEOUT;
    if (f & kErrIndex) return GSA_ERR_ARG;
    return GSA_OK;
}

}  // extern "C"
