// GSA decode step on the 5th-generation tensor cores (bf16, d = 128).
//
// Two launches of one persistent kernel per decode step (one CTA per SM),
// chained by programmatic dependent launch:
//
//  phase A  (launch 1) Stream-K over the units of all rows, a row being one
//           (b, kv-head): 128-gist tiles (routing scores; in ALL_GISTS mode
//           also attention) and 128-token tail tiles (attention).  Each CTA
//           takes a contiguous range of units; a maximal run of one row's
//           units is a segment, whose attention state leaves as one partial
//           (M, L, O).  Each CTA then takes the exact top-k of the gists it
//           scored, the candidates of the row's selection.
//  phase B  (launch 2) Each row's unfolded rows (the selected chunks' raw
//           tokens, and in SELECTED_PAIRS mode the selected gists) are packed
//           into 128-row tiles, and the tiles are spread over CTAs.  Each CTA
//           of a row selects the row's top-k from the candidates, gathers its
//           tiles with every thread's cp.async, attends over them and leaves
//           one partial; the row's last CTA (atomic ticket) merges all of the
//           row's partials (log-sum-exp) into out.
//
// Method: gist.science explainer (EN), section 2 "Methodology": gist as
// routing signals, selective unfolding, hybrid attention; Taki-lab slides
// pages 6 and 17 (AG+SR / SG+SR context rules).
//
// Warp roles: warps 0-3 run the softmax (thread t owns key row t of a tile and,
// for O^T, TMEM lane t = output dimension t); warp 4 issues the loads; warp 5
// owns TMEM and issues the MMAs.  Per tile:
//   S   = K_tile . Q^T     M = 128 keys, N = 16 (G heads, rest zero), K = d
//   O^T += V_tile^T . P^T  M = 128 = d,  N = 16 heads,                K = 128 keys
// S is double buffered in TMEM, O^T has one accumulator per segment parity,
// P^T (bf16) and Q are double buffered in shared memory; O^T is rescaled
// lazily (only when a head's running maximum grows by more than 2^8).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "gsa_fused.h"
#include "gsa_tc.cuh"

namespace gsa {
namespace fused {

constexpr int NT = 192;
constexpr int NS = 3;
constexpr int D = 128;
constexpr int TILE = 128;
constexpr uint32_t KV_BYTES = 32768;         // one tensor of one stage
constexpr uint32_t STAGE_BYTES = 2 * KV_BYTES;
constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 16, 0, 0);
constexpr uint32_t IDESC_PV = tc::idesc_bf16(128, 16, 1, 0);
constexpr float kRescaleLog2 = 8.f;
constexpr int kSelStageCap = 12288;   // keys a selection stages in shared memory (keys, result, 2 lists, bitmaps)

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t SM_STAGE = 0;
constexpr uint32_t SM_Q = NS * STAGE_BYTES;          // 2 x 4 KiB: [16 rows][128 B] x 2 K blocks
constexpr uint32_t SM_P = SM_Q + 2 * 4096;           // 2 x 4 KiB: P^T [16 heads][128 keys]
constexpr uint32_t SM_WMAX = SM_P + 2 * 4096;        // [2][4 warps][16] floats
constexpr uint32_t SM_LRED = SM_WMAX + 2 * 4 * 16 * 4;
constexpr uint32_t SM_TOPK = SM_LRED + 4 * 16 * 4;   // block top-k scratch
constexpr uint32_t SM_MISC = SM_TOPK + 2048;         // finalized-row list
constexpr uint32_t SM_SCORE = SM_MISC + 1024;        // phase A: this CTA's routing scores
constexpr int kScoreCap = 3072;                      // scores kept in shared memory
constexpr uint32_t SM_SEL = SM_SCORE;                // phase B: the row's selection [kSelCap]
constexpr uint32_t SM_ROWTAB = SM_SEL + kSelCap * 4; // phase B: source of each gathered row [kMaxTpc][128]
// hierarchy, phase B: the level-2 selection at SM_SEL [k2 <= 512], the children
// tile's score keys [128] and the level-1 selection [k1 <= 128] after it
constexpr uint32_t SM_CKEY = SM_SEL + 512 * 4;
constexpr uint32_t SM_SEL1 = SM_CKEY + TILE * 4;
static_assert(SM_SEL1 + TILE * 4 <= SM_ROWTAB, "hierarchy tables overflow the selection buffer");
static_assert(kSelCap * 4 + kMaxTpc * TILE * 4 <= kScoreCap * 4, "phase-B tables overflow the score buffer");
constexpr uint32_t SM_UB = SM_SCORE + kScoreCap * 4;  // first unit of every phase-A CTA [kFusedCtas + 1]
constexpr uint32_t SM_BAR = SM_UB + 640;
static_assert((kFusedCtas + 1) * 4 <= 640, "unit table overflow");
constexpr uint32_t SMEM_BYTES = SM_BAR + 512 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "dynamic shared memory above the per-block limit");

struct Bars {
    uint64_t full[NS], empty[NS];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full[2], o_done[2];
    uint64_t q_ready[2];
    uint32_t tmem;
};

// A unit of work: 128 keys of one row.
struct Unit {
    int row;
    int kind;      // 0 gist tile, 1 tail tile, 2 gathered tile (raw chunks [+ gists])
    int t;         // tile index within its kind
    int lt;        // gathered tiles: index into the shared row table
    int nvalid;    // kinds 0/1: leading valid rows
    bool score, attn;
};

// Phase-A CTA c takes units [ub[c], ub[c + 1]), ub[c] = floor(c * T / grid),
// a table every CTA builds in shared memory at start.
__device__ __forceinline__ int unit_begin(const int* ub, int c) { return ub[c]; }
// The phase-A CTA whose range holds unit u (binary search of the table).
__device__ __forceinline__ int cta_of(const int* ub, int grid, int u) {
    int lo = 0, hi = grid - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ub[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Unit i of the current pipeline: phase A (row < 0) walks the CTA's unit range
// starting at u0; phase B walks the gathered tiles of `row` from tile u0.
__device__ __forceinline__ Unit unit_at(const Params& p, int u0, int row, int i) {
    Unit x;
    if (row < 0) {
        const int u = u0 + i;
        x.row = (int)(u / p.upr);
        const int t = (int)(u % p.upr);
        if (t < p.tg) {
            x.kind = 0;
            x.t = t;
            x.nvalid = min(TILE, p.NA - t * TILE);
            x.score = p.do_score != 0;
            x.attn = p.do_attn_gists != 0;
        } else {
            x.kind = 1;
            x.t = t - p.tg;
            x.nvalid = min(TILE, p.W - x.t * TILE);
            x.score = false;
            x.attn = true;
        }
    } else {
        x.row = row;
        x.kind = 2;
        x.t = u0 + i;
        x.lt = i;
        x.nvalid = 0;
        x.score = p.hier != 0 && x.t == 0;   // the hierarchy's children tile (tile 0) is scored
        x.attn = true;
    }
    return x;
}

// Is key row r of the gathered tile with row-table index lt valid?  (The
// table marks an empty row with -1.)
__device__ __forceinline__ bool gathered_valid(const uint8_t* base, int lt, int r) {
    return reinterpret_cast<const int32_t*>(base + SM_ROWTAB)[lt * TILE + r] != -1;
}

// Copy 16-byte piece c16 of gathered row r into the swizzled K and V operand
// tiles ks / vs.  e is the row's source: raw row e (e >= 0), gist row -e - 2
// (e <= -2), or none (e == -1: V is zeroed so that the row's zero weight
// cannot meet a stale NaN pattern).
__device__ __forceinline__ void gather_piece(const Params& p, uint8_t* ks, uint8_t* vs, int e, int r, int c16) {
    const uint32_t off = (uint32_t)(c16 >> 3) * 16384u + (uint32_t)r * 128u + ((uint32_t)((c16 & 7) ^ (r & 7)) << 4);
    if (e != -1) {
        const size_t y = e >= 0 ? (size_t)e : (size_t)(-(long long)e - 2);
        const size_t src = y * (D * 2) + (size_t)c16 * 16;
        cp_async16(ks + off, (e >= 0 ? p.kr : p.kgp) + src);
        cp_async16(vs + off, (e >= 0 ? p.vr : p.vgp) + src);
    } else {
        cp_async16_zero(vs + off, p.vr);
    }
}

struct Ctx {
    uint8_t* base;
    uint32_t sbase;
    Bars* bars;
    uint32_t tmem;
    int warp, lane;
    // role counters (each role keeps its own copy; all roles see the same unit sequence)
    int tiles, segs, atiles;
    int first_attn;   // MMA role: the next attention tile starts its segment
    // softmax role: running state of the current segment
    float m_run[16];
    float l_part[16];
    int had_attn, cur_row, cur_slot;
    int gtiles;     // softmax role: score tiles so far (index into the shared score buffer)
};

// ------------------------------------------------------------ producer --
// Called by all 32 lanes of the producer warp: lane 0 issues the large boxes
// of gist / tail tiles; the 8-row boxes of a gathered tile are spread over
// the lanes (box lane % 16, K for lanes < 16, V above), so their issue runs
// in parallel.
__device__ __forceinline__ void produce(const Params& p, Ctx& cx, const Unit& u) {
    const int gi = cx.tiles;
    const int stage = gi % NS;
    cx.tiles = gi + 1;
    if (gi >= NS && !mbar_wait(&cx.bars->empty[stage], ((gi / NS) - 1) & 1, p.err)) return;
    uint8_t* ks = cx.base + SM_STAGE + stage * STAGE_BYTES;
    uint8_t* vs = ks + KV_BYTES;
    uint64_t* bar = &cx.bars->full[stage];
    if (u.kind < 2) {
        if (cx.lane == 0) {
            const CUtensorMap* mk = u.kind == 0 ? &p.tm_kg : &p.tm_kt;
            const CUtensorMap* mv = u.kind == 0 ? &p.tm_vg : &p.tm_vt;
            const int y = u.t * TILE;
            mbar_arrive_expect_tx(bar, u.attn ? STAGE_BYTES : KV_BYTES);
            tc::tma_load_3d(ks, mk, 0, y, u.row, bar);
            tc::tma_load_3d(ks + 16384, mk, 64, y, u.row, bar);
            if (u.attn) {
                tc::tma_load_3d(vs, mv, 0, y, u.row, bar);
                tc::tma_load_3d(vs + 16384, mv, 64, y, u.row, bar);
            }
        }
    } else if (gi >= NS) {
        // a gathered tile beyond the ones every thread issued up front: the
        // producer warp copies it from the shared row table; its 32 lanes'
        // completions and one arrival for the other NT - 32 threads complete
        // the stage's phase (the barrier counts NT in phase B)
        const int32_t* tab = reinterpret_cast<const int32_t*>(cx.base + SM_ROWTAB) + gi * TILE;
        for (int q = cx.lane; q < TILE * 16; q += 32) gather_piece(p, ks, vs, tab[q >> 4], q >> 4, q & 15);
        cp_async_arrive_noinc(bar);
        __syncwarp();
        if (cx.lane == 0) mbar_arrive_cnt(bar, NT - 32);
    }
}

// ----------------------------------------------------------------- MMA --
// The MMA thread runs an event loop over its units: it issues a unit's S
// product as soon as the unit's data, a free S buffer and (for a new segment)
// its Q are there, and a pending P.V as soon as its P is there, whichever
// comes first.  A stage is thus released right after its own P.V, not after
// the next unit's data has arrived.
struct PendingPV {
    int stage, obuf, first, pj;
};

__device__ __forceinline__ void issue_pv(Ctx& cx, const PendingPV& r) {
    const uint32_t vs = cx.sbase + SM_STAGE + r.stage * STAGE_BYTES + KV_BYTES;
    const uint32_t pt = cx.sbase + SM_P + (r.pj & 1) * 4096;
    const uint32_t dO = cx.tmem + 32 + r.obuf * 16;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        tc::mma_bf16(dO, tc::sdesc_sw128(vs + kk * 2048, 16384, 1024),
                     tc::sdesc_sw128(pt + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024), IDESC_PV,
                     (r.first && kk == 0) ? 0u : 1u);
    }
    tc::commit(&cx.bars->o_done[r.pj & 1]);
    tc::commit(&cx.bars->empty[r.stage]);
}

__device__ __forceinline__ void mma_loop(const Params& p, Ctx& cx, int u0, int row, int n) {
    PendingPV ring[4];
    int head = 0, tail = 0;   // pending P.V products [head, tail)
    int next = 0;             // next unit whose S product is due
    int prev_row = -1;
    uint64_t t_last = global_ns();
    while (next < n || head != tail) {
        bool prog = false;
        if (next < n && tail - head < 4) {
            const Unit u = unit_at(p, u0, row, next);
            const bool ns = u.row != prev_row;
            const int gi = cx.tiles, stage = gi % NS, sb = gi & 1;
            const bool ready = (!ns || mbar_test(&cx.bars->q_ready[cx.segs & 1], (cx.segs >> 1) & 1)) &&
                               mbar_test(&cx.bars->full[stage], (gi / NS) & 1) &&
                               (gi < 2 || mbar_test(&cx.bars->s_free[sb], ((gi - 2) >> 1) & 1));
            if (ready) {
                tc::fence_after();
                if (ns) {
                    cx.segs++;
                    cx.first_attn = 1;
                }
                cx.tiles = gi + 1;
                if (u.kind == 2) tc::fence_async_smem();   // cp.async (generic proxy) writes -> tensor core reads
                const uint32_t ks = cx.sbase + SM_STAGE + stage * STAGE_BYTES;
                const uint32_t qb = cx.sbase + SM_Q + ((cx.segs - 1) & 1) * 4096;
                const uint32_t dS = cx.tmem + sb * 16;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t ka = (kk >> 2) * 16384 + (kk & 3) * 32;
                    const uint32_t qa = (kk >> 2) * 2048 + (kk & 3) * 32;
                    tc::mma_bf16(dS, tc::sdesc_sw128(ks + ka, 16, 1024), tc::sdesc_sw128(qb + qa, 16, 1024), IDESC_S,
                                 kk > 0 ? 1u : 0u);
                }
                tc::commit(&cx.bars->s_full[sb]);
                if (!u.attn) tc::commit(&cx.bars->empty[stage]);
                if (u.attn) {
                    ring[tail & 3] = PendingPV{stage, (cx.segs - 1) & 1, cx.first_attn, cx.atiles};
                    ++tail;
                    cx.first_attn = 0;
                    cx.atiles++;
                }
                prev_row = u.row;
                ++next;
                prog = true;
            }
        }
        if (head != tail) {
            const PendingPV& r = ring[head & 3];
            if (mbar_test(&cx.bars->p_full[r.pj & 1], (r.pj >> 1) & 1)) {
                tc::fence_after();
                issue_pv(cx, r);
                ++head;
                prog = true;
            }
        }
        if (prog) {
            t_last = global_ns();
        } else {
            __nanosleep(20);   // leave the issue slots to the softmax warp sharing this scheduler
            if (global_ns() - t_last > kWaitLimitNs) {
                atomicOr(p.err, kErrTimeout);
                return;
            }
        }
    }
}

// ------------------------------------------------------------- softmax --
// Write Q of `row` into the Q buffer of the next segment (rows >= G stay zero).
template <int G>
__device__ __forceinline__ void write_q(const Params& p, Ctx& cx, int row) {
    const int t = threadIdx.x;            // 0..127: head t/16, 16-byte chunk t%16
    const int h = t >> 4, c = t & 15;
    uint8_t* qb = cx.base + SM_Q + (cx.segs & 1) * 4096;
    if (h < G) {
        const uint4 v = *reinterpret_cast<const uint4*>(p.q + ((size_t)row * G + h) * D + c * 8);
        *reinterpret_cast<uint4*>(qb + (c >> 3) * 2048 + h * 128 + (((c & 7) ^ (h & 7)) << 4)) = v;
    }
    tc::fence_async_smem();
    mbar_arrive(&cx.bars->q_ready[cx.segs & 1]);
    cx.segs++;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Close the current segment (its O^T accumulator is `obuf`): write its
// partial (M, L, O) to slot cur_slot of cur_row.
template <int G>
__device__ __forceinline__ void finalize_segment(const Params& p, Ctx& cx, uint32_t obuf) {
    const int t = threadIdx.x;
    float O[G];
    if (cx.had_attn) {
        const int pj = cx.atiles - 1;
        mbar_wait(&cx.bars->o_done[pj & 1], (pj >> 1) & 1, p.err);
        tc::fence_after();
        uint32_t r[G];
        tc::ldn<G>(cx.tmem + 32 + obuf * 16 + ((uint32_t)(cx.warp * 32) << 16), r);
        tc::wait_ld();
#pragma unroll
        for (int h = 0; h < G; ++h) O[h] = __uint_as_float(r[h]);
    } else {
#pragma unroll
        for (int h = 0; h < G; ++h) O[h] = 0.f;
    }
    float* lred = reinterpret_cast<float*>(cx.base + SM_LRED);
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float s = warp_sum(cx.l_part[h]);
        if (cx.lane == 0) lred[cx.warp * 16 + h] = s;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const size_t slot = (size_t)cx.cur_row * p.slot_stride + cx.cur_slot;
    float* part = p.part + slot * G * D;
#pragma unroll
    for (int h = 0; h < G; ++h) part[h * D + t] = O[h];
    if (t < G) {
        float L = 0.f;
        for (int w = 0; w < 4; ++w) L += lred[w * 16 + t];
        float m = cx.m_run[0];
#pragma unroll
        for (int h = 1; h < G; ++h) m = (h == t) ? cx.m_run[h] : m;
        p.ml[(slot * G + t) * 4 + 0] = m;   // 16 bytes per head: (m, l, -, -)
        p.ml[(slot * G + t) * 4 + 1] = L;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

template <int G>
__device__ __forceinline__ void softmax_tile(const Params& p, Ctx& cx, const Unit& u, bool new_seg, int slot) {
    const int t = threadIdx.x;
    if (new_seg) {
        // publish the new segment's Q first: the MMA thread issues the pending
        // P.V of the closing segment only after the S of this tile
        const uint32_t prev_obuf = (cx.segs - 1) & 1;
        write_q<G>(p, cx, u.row);
        if (cx.cur_row >= 0) finalize_segment<G>(p, cx, prev_obuf);
        cx.cur_row = u.row;
        cx.cur_slot = slot;
        cx.had_attn = 0;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            cx.m_run[h] = -INFINITY;
            cx.l_part[h] = 0.f;
        }
    }
    const int gi = cx.tiles;
    const int sb = gi & 1;
    cx.tiles = gi + 1;
    if (!mbar_wait(&cx.bars->s_full[sb], (gi >> 1) & 1, p.err)) return;
    tc::fence_after();
    uint32_t r[G];
    const uint32_t lane_off = (uint32_t)(cx.warp * 32) << 16;
    tc::ldn<G>(cx.tmem + sb * 16 + lane_off, r);
    tc::wait_ld();
    tc::fence_before();
    mbar_arrive(&cx.bars->s_free[sb]);
    const bool valid = u.kind < 2 ? (t < u.nvalid) : gathered_valid(cx.base, u.lt, t);
    float score = 0.f;
    if (u.score) {
#pragma unroll
        for (int h = 0; h < G; ++h) score += __uint_as_float(r[h]);
    }
    if (u.attn) {
        const int pj = cx.atiles;
        const int pb = pj & 1;
        float* wmax = reinterpret_cast<float*>(cx.base + SM_WMAX) + pb * 64;
        float x[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            x[h] = valid ? __uint_as_float(r[h]) * p.c2 : -INFINITY;
            float m;
            asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(x[h]));
            if (cx.lane == 0) wmax[cx.warp * 16 + h] = m;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        float alpha[G];
        bool need = false;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            alpha[h] = 1.f;
            const float mt = fmaxf(fmaxf(wmax[h], wmax[16 + h]), fmaxf(wmax[32 + h], wmax[48 + h]));
            if (mt > -INFINITY) {
                if (cx.m_run[h] == -INFINITY) {
                    cx.m_run[h] = mt;   // nothing accumulated yet for this head
                } else if (mt > cx.m_run[h] + kRescaleLog2) {
                    alpha[h] = exp2f(cx.m_run[h] - mt);
                    cx.m_run[h] = mt;
                    need = true;
                }
            }
        }
        if (need && cx.had_attn) {
            // O^T holds the P.V of this segment's earlier tiles: wait for the last, rescale columns
            mbar_wait(&cx.bars->o_done[(pj - 1) & 1], ((pj - 1) >> 1) & 1, p.err);
            tc::fence_after();
            uint32_t o[G];
            const uint32_t ta = cx.tmem + 32 + ((cx.segs - 1) & 1) * 16 + lane_off;
            tc::ldn<G>(ta, o);
            tc::wait_ld();
#pragma unroll
            for (int h = 0; h < G; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
            tc::stn<G>(ta, o);
            tc::wait_st();
        }
        // P^T buffer pb was last read by the P.V of attention tile pj-2
        if (pj >= 2) mbar_wait(&cx.bars->o_done[pb], ((pj - 2) >> 1) & 1, p.err);
        uint8_t* pt = cx.base + SM_P + pb * 4096;
        const int kb = t >> 6, c16 = (t & 63) >> 3, e = t & 7;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float pv = (x[h] == -INFINITY) ? 0.f : exp2f(x[h] - cx.m_run[h]);
            cx.l_part[h] = cx.l_part[h] * alpha[h] + pv;
            *reinterpret_cast<uint16_t*>(pt + kb * 2048 + h * 128 + ((c16 ^ (h & 7)) << 4) + e * 2) =
                f32_to_bf16_rne(pv);
        }
        tc::fence_async_smem();
        tc::fence_before();
        mbar_arrive(&cx.bars->p_full[pb]);
        cx.atiles = pj + 1;
        cx.had_attn = 1;
    }
    // the routing score leaves after the tile is handed to the tensor core
    if (u.score && u.kind == 2) {
        // hierarchy: the level-1 scores of the children tile, as keys for the k1 selection
        reinterpret_cast<uint32_t*>(cx.base + SM_CKEY)[t] = valid ? order_key(score) : 0u;
    } else if (u.score) {
        if (valid) {
            p.scores[(size_t)u.row * p.NA + u.t * TILE + t] = score;
            if (cx.gtiles < kScoreCap / TILE)
                reinterpret_cast<float*>(cx.base + SM_SCORE)[cx.gtiles * TILE + t] = score;
        }
        cx.gtiles++;
    }
}

// Run the three roles over n units (phase A: row < 0, from unit u0; phase B:
// the gathered tiles of `row` from tile u0).  A new segment starts where the
// row changes; its partial goes to slot c - first CTA of the row (phase A) or
// to slot `slot_b` (phase B).  Ends with every segment written out.
template <int G>
__device__ __forceinline__ void run_pipeline(const Params& p, Ctx& cx, int u0, int row, int n,
                                             int slot_b) {
    if (cx.warp == 4) {
        for (int i = 0; i < n; ++i) produce(p, cx, unit_at(p, u0, row, i));
    } else if (cx.warp == 5) {
        if (cx.lane == 0) mma_loop(p, cx, u0, row, n);
    } else {
        int prev_row = -1;
        for (int i = 0; i < n; ++i) {
            const Unit u = unit_at(p, u0, row, i);
            const bool ns = u.row != prev_row;
            const int slot =
                row >= 0 ? slot_b
                         : (int)blockIdx.x - cta_of(reinterpret_cast<const int*>(cx.base + SM_UB), p.grid,
                                                    u.row * p.upr);
            softmax_tile<G>(p, cx, u, ns, slot);
            prev_row = u.row;
        }
        if (cx.cur_row >= 0) finalize_segment<G>(p, cx, (cx.segs - 1) & 1);
        cx.cur_row = -1;
    }
    __syncthreads();
}

// Top-k of n keys in shared memory into res[0..min(k, n)) (ascending
// positions).  One out-of-line copy serves both phases, so the code that
// phase A runs is the code phase B finds in the instruction cache.
__device__ __noinline__ void select_staged(const uint32_t* keys, int n, int k, int32_t* res, uint32_t* scratch) {
    if (k >= n) {
        for (int i = threadIdx.x; i < n; i += NT) res[i] = i;
    } else {
        bool done = false;
        if (k <= 32 && n <= NT * 16) done = threshold_topk<NT, 16>(keys, n, k, res, scratch);
        else if (k <= 32 && n <= NT * 32) done = threshold_topk<NT, 32>(keys, n, k, res, scratch);
        if (!done) smem_topk<NT>(keys, n, k, res, scratch);
    }
    __syncthreads();
}

// Top-k of n keys staged (by `key_of`) into shared memory; `emit(r, pos)` for
// the k selected positions in ascending order.  Falls back to a radix
// select straight from global memory when n exceeds the staging capacity.
template <class KeyOf, class Emit>
__device__ __forceinline__ void select_keys(uint8_t* base, int n, int k, KeyOf key_of, Emit emit) {
    if (n <= kSelStageCap) {
        uint32_t* keys = reinterpret_cast<uint32_t*>(base + SM_STAGE);
        int32_t* res = reinterpret_cast<int32_t*>(keys + ((n + 31) & ~31));
        uint32_t* scratch = reinterpret_cast<uint32_t*>(res + ((min(k, n) + 31) & ~31));
#pragma unroll 1
        for (int i = threadIdx.x; i < n; i += NT) keys[i] = key_of(i);
        __syncthreads();
        select_staged(keys, n, k, res, scratch);
#pragma unroll 1
        for (int r = threadIdx.x; r < min(k, n); r += NT) emit(r, res[r]);
    } else {
        block_topk<NT>(n, k, key_of, emit, reinterpret_cast<uint32_t*>(base + SM_TOPK));
    }
    __syncthreads();
}

// Local top-k of this CTA's gists [g0, g1) of `row` (scores in the shared
// buffer from `soff`, or in global memory), written as candidates at `off`
// of the row's candidate list, in index order.
__device__ __forceinline__ void local_topk(const Params& p, uint8_t* base, int row, int g0, int g1, int soff, int off,
                                        bool in_smem) {
    const float* ss = reinterpret_cast<const float*>(base + SM_SCORE) + soff;
    const float* sg = p.scores + (size_t)row * p.NA + g0;
    uint32_t* ck = p.cand_key + (size_t)row * p.NA + off;
    int32_t* ci = p.cand_idx + (size_t)row * p.NA + off;
    const uint32_t* keys = reinterpret_cast<const uint32_t*>(base + SM_STAGE);
    select_keys(
        base, g1 - g0, p.K, [&](int i) { return order_key(in_smem ? ss[i] : __ldcg(sg + i)); },
        [&](int r, int pos) {
            ck[r] = g1 - g0 <= kSelStageCap ? keys[pos] : order_key(__ldcg(sg + pos));
            ci[r] = g0 + pos;
        });
}

// The row's exact top-k from the candidates that every phase-A CTA meeting
// the row left (n of them), into the shared selection sel[0..k) and, when
// `publish`, into the row's idx output.
__device__ __forceinline__ void merge_select(const Params& p, uint8_t* base, int row, int n, bool publish) {
    const uint32_t* ck = p.cand_key + (size_t)row * p.NA;
    const int32_t* ci = p.cand_idx + (size_t)row * p.NA;
    int32_t* out = p.idx + (size_t)row * p.K;
    int32_t* sel = reinterpret_cast<int32_t*>(base + SM_SEL);
    select_keys(
        base, n, p.K, [&](int i) { return __ldcg(ck + i); },
        [&](int r, int pos) {
            const int32_t j = __ldcg(ci + pos);
            sel[r] = j;
            if (publish) out[r] = j;
        });
}

// The row's exact top-k straight from its n = N routing scores (small N and
// k): the scores are staged with all loads of a thread in flight at once.
template <int U>   // n <= U * NT
__device__ __forceinline__ void direct_select_u(const Params& p, uint8_t* base, int row, bool publish) {
    const int n = p.NA, k = p.K;
    const float* sg = p.scores + (size_t)row * p.NA;
    uint32_t* keys = reinterpret_cast<uint32_t*>(base + SM_STAGE);
    int32_t* res = reinterpret_cast<int32_t*>(keys + ((n + 31) & ~31));
    uint32_t* scratch = reinterpret_cast<uint32_t*>(res + ((min(k, n) + 31) & ~31));
    float v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int i = threadIdx.x + u * NT;
        v[u] = i < n ? __ldcg(sg + i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int i = threadIdx.x + u * NT;
        if (i < n) keys[i] = order_key(v[u]);
    }
    __syncthreads();
    select_staged(keys, n, k, res, scratch);
    int32_t* sel = reinterpret_cast<int32_t*>(base + SM_SEL);
    int32_t* out = p.idx + (size_t)row * p.K;
    for (int r = threadIdx.x; r < min(k, n); r += NT) {
        sel[r] = res[r];
        if (publish) out[r] = res[r];
    }
    __syncthreads();
}

__device__ __forceinline__ void direct_select(const Params& p, uint8_t* base, int row, bool publish) {
    if (p.NA <= 16 * NT) direct_select_u<16>(p, base, row, publish);
    else direct_select_u<32>(p, base, row, publish);
}

// A given selection (gsa_unfold_attn) into sel[0..k); an index outside
// [0, N) is clamped into range and flagged in the error word.
__device__ __forceinline__ void load_selection(const Params& p, uint8_t* base, int row) {
    int32_t* sel = reinterpret_cast<int32_t*>(base + SM_SEL);
    for (int r = threadIdx.x; r < p.K; r += NT) {
        int32_t j = __ldcg(p.idx + (size_t)row * p.K + r);
        if (j < 0 || j >= p.N) {
            atomicOr(p.err, kErrIndex);
            j = j < 0 ? 0 : p.N - 1;
        }
        sel[r] = j;
    }
    __syncthreads();
}

// Phase B, before the pipeline: the source of every row of this CTA's
// gathered tiles [t0, t0 + ntl) into the shared row table, then every thread
// issues its share of the first min(ntl, NS) tiles' copies (stage i = tile
// t0 + i) and arrives on each of those stages once its copies have landed.
__device__ __forceinline__ void gather_prologue(const Params& p, uint8_t* base, Bars* bars, int row, int t0, int ntl) {
    const int32_t* sel = reinterpret_cast<const int32_t*>(base + SM_SEL);
    int32_t* tab = reinterpret_cast<int32_t*>(base + SM_ROWTAB);
    const int kc = p.K * p.C;
    for (int i = threadIdx.x; i < ntl * TILE; i += NT) {
        const int gr = t0 * TILE + i;
        int32_t e = -1;
        if (gr < kc) {
            const int sidx = gr / p.C, tok = gr - sidx * p.C;
            e = (int32_t)(((long long)row * p.N + sel[sidx]) * p.C + tok);
        } else if (gr < p.nrows_g) {
            e = (int32_t)(-((long long)row * p.N + sel[gr - kc]) - 2);
        }
        tab[i] = e;
    }
    __syncthreads();
    const int npre = min(ntl, NS);
#pragma unroll 1
    for (int q = threadIdx.x; q < npre * TILE * 16; q += NT) {
        const int lt = q >> 11, r = (q >> 4) & (TILE - 1);
        uint8_t* ks = base + SM_STAGE + lt * STAGE_BYTES;
        gather_piece(p, ks, ks + KV_BYTES, tab[lt * TILE + r], r, q & 15);
    }
    for (int lt = 0; lt < npre; ++lt) cp_async_arrive_noinc(&bars->full[lt]);
}

// Hierarchy, phase B: every thread issues its share of the gathered tile
// described by row-table entries [0, 128) into `stage`, and arrives on that
// stage's barrier once its copies have landed.
__device__ __forceinline__ void gather_issue(const Params& p, uint8_t* base, Bars* bars, int stage) {
    const int32_t* tab = reinterpret_cast<const int32_t*>(base + SM_ROWTAB);
    uint8_t* ks = base + SM_STAGE + stage * STAGE_BYTES;
#pragma unroll 1
    for (int q = threadIdx.x; q < TILE * 16; q += NT) gather_piece(p, ks, ks + KV_BYTES, tab[q >> 4], q >> 4, q & 15);
    cp_async_arrive_noinc(&bars->full[stage]);
}

// Hierarchy, phase B: the row table of the children tile: the level-1 gists
// of the k2 selected groups, group after group (a short last group leaves
// empty rows).
__device__ __forceinline__ void hier_children_table(const Params& p, uint8_t* base, int row) {
    const int32_t* sel2 = reinterpret_cast<const int32_t*>(base + SM_SEL);
    int32_t* tab = reinterpret_cast<int32_t*>(base + SM_ROWTAB);
    for (int r = threadIdx.x; r < TILE; r += NT) {
        int32_t e = -1;
        if (r < p.K * p.group) {
            const int child = sel2[r / p.group] * p.group + r % p.group;
            if (child < p.N1) e = (int32_t)(-((long long)row * p.N1 + child) - 2);
        }
        tab[r] = e;
    }
    __syncthreads();
}

// Hierarchy, phase B: the exact top-k1 of the children tile's scores (ties to
// the lower level-1 index: the tile holds the children in ascending order),
// published as idx1 and kept in shared memory, then the row table of the
// raw tokens of those k1 chunks.
__device__ __forceinline__ void hier_select_children(const Params& p, uint8_t* base, int row) {
    const uint32_t* keys = reinterpret_cast<const uint32_t*>(base + SM_CKEY);
    const int32_t* sel2 = reinterpret_cast<const int32_t*>(base + SM_SEL);
    int32_t* sel1 = reinterpret_cast<int32_t*>(base + SM_SEL1);
    int32_t* res = reinterpret_cast<int32_t*>(base + SM_STAGE);   // stage 0 is free once its tile is done
    uint32_t* scratch = reinterpret_cast<uint32_t*>(base + SM_STAGE + 1024);
    const int n = min(TILE, p.K * p.group);
    select_staged(keys, n, p.K1, res, scratch);
    for (int r = threadIdx.x; r < p.K1; r += NT) {
        const int pos = res[r];
        const int child = sel2[pos / p.group] * p.group + pos % p.group;
        sel1[r] = child;
        p.idx1[(size_t)row * p.K1 + r] = child;
    }
    __syncthreads();
    int32_t* tab = reinterpret_cast<int32_t*>(base + SM_ROWTAB);
    for (int r = threadIdx.x; r < TILE; r += NT) {
        int32_t e = -1;
        if (r < p.K1 * p.C) {
            const int sl = r / p.C;
            e = (int32_t)(((long long)row * p.N1 + sel1[sl]) * p.C + (r - sl * p.C));
        }
        tab[r] = e;
    }
    __syncthreads();
}

// Final log-sum-exp merge of a row: phase-A slots [0, na) and phase-B slots
// [maxs, maxs + nb).  The partials are brought into shared memory with
// cp.async in groups (one memory round trip per group).  Per group, warp h
// finds head h's largest slot maximum M_g and each slot's weight
// 2^(m_s - M_g) and the weighted sum L_g of the l_s; each output is then a
// plain weighted sum over the slots (independent products, no dependent
// rescaling chain), folded into a running (M, L, acc) once per group.
template <int G>
__device__ __forceinline__ void merge_row(const Params& p, uint8_t* base, int row, int na, int nb) {
    constexpr int NW = NT / 32;
    const int nsl = na + nb;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int PER = (G * D + NT - 1) / NT;          // outputs per thread
    constexpr int GS = (int)((STAGE_BYTES * NS - 256) / ((G * D + 5 * G) * 4));   // slots per group
    float* so = reinterpret_cast<float*>(base + SM_STAGE);              // [GS][G][D]
    float* sml = so + GS * G * D;                                       // [GS][G][4]: (m, l, -, -)
    float* wgt = sml + GS * G * 4;                                      // [GS][G]
    float* gml = wgt + GS * G;                                          // [G][2]: (M_g, L_g)
    float M[PER], L[PER], acc[PER];
#pragma unroll
    for (int q = 0; q < PER; ++q) {
        M[q] = -INFINITY;
        L[q] = 0.f;
        acc[q] = 0.f;
    }
#pragma unroll 1
    for (int s0 = 0; s0 < nsl; s0 += GS) {
        const int cnt = min(GS, nsl - s0);
        // slot s0 + i of the row lives at slot index sidx(i) of its slot array
        auto sidx = [&](int i) { const int sl = s0 + i; return row * p.slot_stride + (sl < na ? sl : p.maxs + (sl - na)); };
#pragma unroll 1
        for (int q = threadIdx.x; q < cnt * (G * D / 4); q += NT) {
            const int i = q / (G * D / 4), e4 = q - i * (G * D / 4);
            cp_async16(so + (size_t)i * G * D + e4 * 4, p.part + (size_t)sidx(i) * G * D + e4 * 4);
        }
#pragma unroll 1
        for (int q = threadIdx.x; q < cnt * G; q += NT) {
            const int i = q / G, h = q - i * G;
            cp_async16(sml + (i * G + h) * 4, p.ml + ((size_t)sidx(i) * G + h) * 4);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
#pragma unroll 1
        for (int h = warp; h < G; h += NW) {
            float mx = -INFINITY;
            for (int sl = lane; sl < cnt; sl += 32) mx = fmaxf(mx, sml[(sl * G + h) * 4]);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
            float ls = 0.f;
            for (int sl = lane; sl < cnt; sl += 32) {
                const float m = sml[(sl * G + h) * 4];
                const float wv = m > -INFINITY ? exp2f(m - mx) : 0.f;
                wgt[sl * G + h] = wv;
                ls += sml[(sl * G + h) * 4 + 1] * wv;
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) ls += __shfl_xor_sync(0xFFFFFFFFu, ls, o);
            if (lane == 0) {
                gml[h * 2] = mx;
                gml[h * 2 + 1] = ls;
            }
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const int i = threadIdx.x + q * NT;
            if (i < G * D) {
                const int h = i / D;
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
                int sl = 0;
#pragma unroll 1
                for (; sl + 4 <= cnt; sl += 4) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) a4[e] += wgt[(sl + e) * G + h] * so[(sl + e) * G * D + i];
                }
                for (; sl < cnt; ++sl) a4[0] += wgt[sl * G + h] * so[sl * G * D + i];
                const float ag = (a4[0] + a4[1]) + (a4[2] + a4[3]);
                const float Mg = gml[h * 2], Lg = gml[h * 2 + 1];
                if (Mg > -INFINITY) {
                    const float Mn = fmaxf(M[q], Mg);
                    const float a = (M[q] == -INFINITY) ? 0.f : exp2f(M[q] - Mn), wg = exp2f(Mg - Mn);
                    L[q] = L[q] * a + Lg * wg;
                    acc[q] = acc[q] * a + ag * wg;
                    M[q] = Mn;
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int q = 0; q < PER; ++q) {
        const int i = threadIdx.x + q * NT;
        if (i < G * D) {
            const int h = i / D, e = i % D;
            p.out[((size_t)row * G + h) * D + e] = f32_to_bf16_rne(acc[q] / L[q]);
            if (p.lse != nullptr && e == 0) p.lse[(size_t)row * G + h] = (M[q] + log2f(L[q])) * 0.69314718055994531f;
        }
    }
    if (threadIdx.x == 0) p.cnt[row] = 0;   // leave the ticket zero for the next call
}

// ---------------------------------------------------------------- kernel --
template <int G>
__global__ void __launch_bounds__(NT, 1) fused_decode_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    Ctx cx;
    cx.base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    cx.sbase = smem_u32(cx.base);
    cx.bars = reinterpret_cast<Bars*>(cx.base + SM_BAR);
    cx.warp = threadIdx.x >> 5;
    cx.lane = threadIdx.x & 31;
    cx.tiles = cx.segs = cx.atiles = 0;
    cx.had_attn = 0;
    cx.first_attn = 1;
    cx.cur_row = -1;
    cx.cur_slot = 0;
    cx.gtiles = 0;

    // the Q and P^T rows of heads >= G must be zero (K/V stages need no
    // clearing: TMA zero-fills past a row's end, and a gathered tile zeroes
    // the V rows it leaves empty)
    for (uint32_t o = SM_Q + threadIdx.x * 16; o < SM_WMAX; o += NT * 16)
        *reinterpret_cast<uint4*>(cx.base + o) = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        Bars* b = cx.bars;
        for (int i = 0; i < NS; ++i) {
            // phase A: one arrival with the TMA byte count; phase B: one
            // cp.async completion arrival per thread
            mbar_init(&b->full[i], p.phase == 0 ? 1u : (uint32_t)NT);
            mbar_init(&b->empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&b->s_full[i], 1);
            mbar_init(&b->s_free[i], 128);
            mbar_init(&b->p_full[i], 128);
            mbar_init(&b->o_done[i], 1);
            mbar_init(&b->q_ready[i], 128);
        }
        fence_mbar_init();
    }
    if (threadIdx.x == 32 * 4) {
        // fetch the phase-A tensor maps' descriptors ahead of the first loads
        if (p.tg > 0) asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_kg) : "memory");
        if (p.tg > 0 && p.do_attn_gists) asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_vg) : "memory");
        if (p.W > 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_kt) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_vt) : "memory");
        }
    }
    if (p.grid > 0)
        for (int i = threadIdx.x; i <= p.grid; i += NT)
            reinterpret_cast<int*>(cx.base + SM_UB)[i] = (int)((long long)i * p.T / p.grid);
    tc::fence_async_smem();
    if (cx.warp == 5) {
        tc::tmem_alloc(&cx.bars->tmem, 64);
        tc::tmem_relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    cx.tmem = cx.bars->tmem;
    pdl_wait();                  // the previous step on this stream is complete (workspace reuse)
    pdl_launch_dependents();

    const int c = blockIdx.x;
    // gists of `row` scored by phase-A CTA cc: [g0, g1)
    const int* ub = reinterpret_cast<const int*>(cx.base + SM_UB);
    auto gists_of = [&](int cc, int row, int& g0, int& g1) {
        const int ru0 = row * p.upr;
        const int a = max(unit_begin(ub, cc), ru0), b = min(unit_begin(ub, cc + 1), ru0 + p.tg);
        g0 = (a - ru0) * TILE;
        g1 = b > a ? min((b - ru0) * TILE, p.NA) : g0;
    };
    // the pipeline has one call site for both phases: phase B runs the code
    // that phase A left in this SM's instruction cache
    int pu0 = 0, prow = -1, pn = 0, pslot = 0;
    int row = 0, j = 0, na = 0;
    // the hierarchy's phase B runs two rounds in one CTA per row: the
    // children tile (scored and attended), then the raw tile of the k1 chunks
    const int rounds = (p.phase == 1 && p.hier) ? (p.K1 > 0 ? 2 : 1) : 1;
    for (int rd = 0; rd < rounds; ++rd) {
        if (p.phase == 0) {
            pu0 = unit_begin(ub, c);
            pn = unit_begin(ub, c + 1) - pu0;
        } else {
            // phase B: this CTA takes tiles [t0, t0 + ntl) of `row`
            row = c / p.cb;
            j = c % p.cb;
            const int t0 = p.hier ? rd : j * p.tpc;
            const int ntl = p.hier ? 1 : max(0, min(p.nbt, t0 + p.tpc) - t0);
            const int ru0 = row * p.upr;
            const int cf = p.T > 0 ? cta_of(ub, p.grid, ru0) : 0;
            na = p.T > 0 ? cta_of(ub, p.grid, ru0 + p.upr - 1) - cf + 1 : 0;   // phase-A slots
            if (rd == 1) {
                hier_select_children(p, cx.base, row);
            } else if (ntl > 0) {
                if (p.do_topk && p.sel_direct) {
                    direct_select(p, cx.base, row, j == 0);
                } else if (p.do_topk) {
                    int n = 0;
                    for (int cc = cf; cc < cf + na; ++cc) {
                        int a0, a1;
                        gists_of(cc, row, a0, a1);
                        n += min(p.K, max(0, a1 - a0));
                    }
                    merge_select(p, cx.base, row, n, j == 0);
                } else {
                    load_selection(p, cx.base, row);
                }
                if (p.hier) hier_children_table(p, cx.base, row);
            }
            if (p.hier) {
                gather_issue(p, cx.base, cx.bars, rd % NS);
            } else if (ntl > 0) {
                gather_prologue(p, cx.base, cx.bars, row, t0, ntl);
            }
            pu0 = t0;
            prow = row;
            pn = ntl;
            pslot = p.maxs + (p.hier ? rd : j);
        }
        run_pipeline<G>(p, cx, pu0, prow, pn, pslot);
    }
    if (p.phase == 0) {
        if (p.do_topk && !p.sel_direct) {
            // local top-k of every segment, from the scores this CTA kept
            const int u0 = pu0, u1 = pu0 + pn;
            const int row_first = u0 / p.upr, row_last = (u1 - 1) / p.upr;
            int sfirst = 0;   // score-tile offset of the segment in the shared buffer
            int ntiles = 0;
            for (int r = row_first; r <= row_last; ++r) {
                int a0, a1;
                gists_of(c, r, a0, a1);
                ntiles += (a1 - a0 + TILE - 1) / TILE;
            }
            const bool fits = ntiles <= kScoreCap / TILE;
            for (int r = row_first; r <= row_last; ++r) {
                int g0, g1;
                gists_of(c, r, g0, g1);
                if (g1 <= g0) continue;
                const int cf = cta_of(ub, p.grid, r * p.upr);
                int off = 0;
                for (int cc = cf; cc < c; ++cc) {
                    int a0, a1;
                    gists_of(cc, r, a0, a1);
                    off += min(p.K, max(0, a1 - a0));
                }
                local_topk(p, cx.base, r, g0, g1, sfirst * TILE, off, fits);
                sfirst += (g1 - g0 + TILE - 1) / TILE;
            }
        }
    } else {
        // the row's last CTA merges all of its partials
        int* misc = reinterpret_cast<int*>(cx.base + SM_MISC);
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) misc[0] = atomicAdd(&p.cnt[row], 1u) == (uint32_t)(p.cb - 1) ? 1 : 0;
        __syncthreads();
        if (misc[0]) {
            __threadfence();
            merge_row<G>(p, cx.base, row, na, p.hier ? rounds : (p.nbt > 0 ? p.cb : 0));
        }
    }
    tc::fence_before();
    __syncthreads();
    if (cx.warp == 5) {
        tc::fence_after();
        tc::tmem_dealloc(cx.tmem, 64);
    }
}

// ============================================================ host side ====
static PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// 3-D bf16 map over [rows][len][d = 128], box {64, 128, 1}, 128-byte swizzle:
// a tile that runs past `len` is zero-filled instead of reading the next
// (batch, kv-head) row's entries. An operand the call never reads gets a zeroed map.
static bool map3d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t len) {
    if (rows == 0 || len == 0 || base == nullptr) {
        std::memset(m, 0, sizeof(*m));
        return true;
    }
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {D, len, rows};
    cuuint64_t strides[2] = {D * 2, len * D * 2};
    cuuint32_t box[3] = {64, TILE, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G>
static cudaError_t launch_g(const Params& p, int grid, cudaStream_t st) {
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(fused_decode_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fused_decode_kernel<G>, p);
}

}  // namespace fused

bool fused_supported(const gsa_decode_desc& d) {
    // gathered rows are addressed by a 32-bit row number; the selection lives in shared memory
    const long long raw_rows = (long long)d.batch * d.n_kv_heads * d.n_chunks * d.chunk;
    // phase-A units are counted in 32 bits
    const long long units = (long long)d.batch * d.n_kv_heads * ((d.n_chunks + 127) / 128 + (d.tail_len + 127) / 128);
    return d.dtype == GSA_BF16 && d.head_dim == 128 && d.top_k <= kSelCap && raw_rows < INT32_MAX - 2 &&
           units < (1LL << 30);
}

FusedPlan make_fused_plan(const gsa_decode_desc& d, bool given) {
    FusedPlan f{};
    const bool pairs = d.mode == GSA_SELECTED_PAIRS;
    f.rows = d.batch * d.n_kv_heads;
    f.G = d.n_q_heads / d.n_kv_heads;
    // with a given selection in SELECTED_PAIRS mode no gist is scored or attended in phase A
    f.tg = (given && pairs) ? 0 : (d.n_chunks + 127) / 128;
    f.tt = (d.tail_len + 127) / 128;
    f.upr = f.tg + f.tt;
    f.T = f.rows * f.upr;
    f.grid = std::min(f.T, kFusedCtas);
    // phase-A slots of a row: the CTAs whose range meets the row
    int maxs = 0;
    if (f.T > 0) {
        for (int r = 0; r < f.rows; ++r) {
            const long long a = (long long)r * f.upr, b = a + f.upr - 1;
            const int ca = (int)(((a + 1) * f.grid + f.T - 1) / f.T) - 1;
            const int cb = (int)(((b + 1) * f.grid + f.T - 1) / f.T) - 1;
            maxs = std::max(maxs, cb - ca + 1);
        }
    }
    f.maxs = maxs;
    // small selections are taken in phase B straight from the scores; larger
    // ones from per-CTA candidates that phase A leaves
    f.sel_direct = (d.top_k <= 32 && d.n_chunks <= 32 * fused::NT) ? 1 : 0;
    // phase B: the row's gathered rows packed into 128-row tiles, spread over
    // as many CTAs per row as fill the GPU (at most kMaxTpc tiles each)
    f.nrows_g = d.top_k * d.chunk + (pairs ? d.top_k : 0);
    f.nbt = (f.nrows_g + 127) / 128;
    if (f.nbt == 0) {
        f.tpc = 0;
        f.cb = 1;   // the row's merge still runs
    } else {
        const int cpr = std::max(1, kFusedCtas / f.rows);
        f.tpc = std::min(kMaxTpc, (f.nbt + std::min(cpr, f.nbt) - 1) / std::min(cpr, f.nbt));
        f.cb = (f.nbt + f.tpc - 1) / f.tpc;
    }
    f.grid_b = f.rows * f.cb;
    f.slot_stride = maxs + f.cb;
    const size_t rows = (size_t)f.rows, N = (size_t)d.n_chunks;
    size_t o = round256(kWsCntOffset + rows * 4);
    f.off_scores = o;
    o = round256(o + rows * N * 4);
    f.off_cand_key = o;
    o = round256(o + rows * N * 4);
    f.off_cand_idx = o;
    o = round256(o + rows * N * 4);
    f.off_idx = o;
    o = round256(o + rows * (size_t)d.top_k * 4);
    f.off_part = o;
    o = round256(o + rows * (size_t)f.slot_stride * f.G * 128 * 4);
    f.off_ml = o;
    o = round256(o + rows * (size_t)f.slot_stride * f.G * 4 * 4);
    f.total = o;
    return f;
}

gsa_status fused_launch(const gsa_decode_desc& d, const FusedPlan& f, const void* q, const void* kg, const void* vg,
                        const void* kr, const void* vr, const void* kt, const void* vt, const int32_t* idx_given,
                        int32_t* idx_out, float* scores_out, void* out, float* lse, void* ws, cudaStream_t st) {
    using namespace fused;
    if (f.grid_b <= 0) return GSA_ERR_ARG;
    Params p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t rows = (uint64_t)f.rows, N = (uint64_t)d.n_chunks;
    const bool pairs = d.mode == GSA_SELECTED_PAIRS;
    bool ok = map3d(&p.tm_kg, kg, rows, N) && map3d(&p.tm_vg, pairs ? nullptr : vg, rows, N) &&
              map3d(&p.tm_kt, kt, rows, (uint64_t)d.tail_len) && map3d(&p.tm_vt, vt, rows, (uint64_t)d.tail_len);
    if (!ok) return GSA_ERR_CUDA;
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.q = static_cast<const uint16_t*>(q);
    p.kr = static_cast<const uint8_t*>(kr);
    p.vr = static_cast<const uint8_t*>(vr);
    p.kgp = static_cast<const uint8_t*>(kg);
    p.vgp = static_cast<const uint8_t*>(vg);
    p.out = static_cast<uint16_t*>(out);
    p.lse = lse;
    p.err = reinterpret_cast<uint32_t*>(w + kWsErrOffset);
    p.cnt = reinterpret_cast<uint32_t*>(w + kWsCntOffset);
    p.scores = scores_out ? scores_out : reinterpret_cast<float*>(w + f.off_scores);
    p.idx = idx_given ? const_cast<int32_t*>(idx_given) : (idx_out ? idx_out : reinterpret_cast<int32_t*>(w + f.off_idx));
    p.cand_key = reinterpret_cast<uint32_t*>(w + f.off_cand_key);
    p.cand_idx = reinterpret_cast<int32_t*>(w + f.off_cand_idx);
    p.part = reinterpret_cast<float*>(w + f.off_part);
    p.ml = reinterpret_cast<float*>(w + f.off_ml);
    p.rows = f.rows;
    p.Hkv = d.n_kv_heads;
    p.G = f.G;
    p.N = d.n_chunks;
    p.NA = d.n_chunks;
    p.C = d.chunk;
    p.K = d.top_k;
    p.W = d.tail_len;
    p.mode = d.mode;
    p.tg = f.tg;
    p.upr = f.upr;
    p.T = f.T;
    p.grid = f.grid;
    p.slot_stride = f.slot_stride;
    p.maxs = f.maxs;
    p.nrows_g = f.nrows_g;
    p.nbt = f.nbt;
    p.tpc = f.tpc;
    p.cb = f.cb;
    const double scale = d.scale > 0 ? (double)d.scale : 1.0 / std::sqrt(128.0);
    p.c2 = (float)(scale * 1.4426950408889634);
    p.do_score = idx_given ? 0 : 1;
    p.do_topk = idx_given ? 0 : 1;
    p.do_attn_gists = pairs ? 0 : 1;
    p.sel_direct = f.sel_direct;
    auto launch = [&](int grid) {
        switch (f.G) {
            case 1: return launch_g<1>(p, grid, st);
            case 2: return launch_g<2>(p, grid, st);
            case 4: return launch_g<4>(p, grid, st);
            default: return launch_g<8>(p, grid, st);
        }
    };
    cudaError_t e = cudaSuccess;
    if (f.grid > 0) {
        p.phase = 0;
        e = launch(f.grid);
    }
    if (e == cudaSuccess) {
        p.phase = 1;
        e = launch(f.grid_b);
    }
    return e == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

// --------------------------------------------------------- hierarchy ----
bool fused_hier_supported(const gsa_hier_desc& h) {
    const gsa_decode_desc& d = h.l1;
    const long long rows = (long long)d.batch * d.n_kv_heads;
    const long long units = rows * ((h.n_l2 + 127) / 128 + (d.tail_len + 127) / 128);
    return d.dtype == GSA_BF16 && d.head_dim == 128 && (long long)h.top_k2 * h.group <= 128 &&
           (long long)d.top_k * d.chunk <= 128 && rows * d.n_chunks * d.chunk < INT32_MAX - 2 &&
           rows * d.n_chunks < INT32_MAX - 2 && units < (1LL << 30);
}

FusedPlan make_fused_hier_plan(const gsa_hier_desc& h) {
    // phase A and the level-2 selection are the flat step over the level-2 gists
    gsa_decode_desc l2 = h.l1;
    l2.n_chunks = h.n_l2;
    l2.top_k = h.top_k2;
    l2.mode = GSA_ALL_GISTS;
    FusedPlan f = make_fused_plan(l2);
    // phase B: one CTA per row, two partial slots (children tile, raw tile)
    f.nbt = 2;
    f.tpc = 2;
    f.cb = 1;
    f.grid_b = f.rows;
    f.slot_stride = f.maxs + 2;
    const size_t rows = (size_t)f.rows;
    size_t o = f.off_part;
    o = round256(o + rows * (size_t)f.slot_stride * f.G * 128 * 4);
    f.off_ml = o;
    o = round256(o + rows * (size_t)f.slot_stride * f.G * 4 * 4);
    f.off_idx1 = o;
    o = round256(o + rows * (size_t)h.l1.top_k * 4);
    f.total = o;
    return f;
}

gsa_status fused_hier_launch(const gsa_hier_desc& h, const FusedPlan& f, const void* q, const void* k_g2,
                             const void* v_g2, const void* k_g1, const void* v_g1, const void* kr, const void* vr,
                             const void* kt, const void* vt, int32_t* idx2_out, int32_t* idx1_out, void* out,
                             void* ws, cudaStream_t st) {
    using namespace fused;
    const gsa_decode_desc& d = h.l1;
    if (f.grid <= 0 || f.grid_b <= 0) return GSA_ERR_ARG;
    Params p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t rows = (uint64_t)f.rows;
    bool ok = map3d(&p.tm_kg, k_g2, rows, (uint64_t)h.n_l2) && map3d(&p.tm_vg, v_g2, rows, (uint64_t)h.n_l2) &&
              map3d(&p.tm_kt, kt, rows, (uint64_t)d.tail_len) && map3d(&p.tm_vt, vt, rows, (uint64_t)d.tail_len);
    if (!ok) return GSA_ERR_CUDA;
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.q = static_cast<const uint16_t*>(q);
    p.kr = static_cast<const uint8_t*>(kr);
    p.vr = static_cast<const uint8_t*>(vr);
    p.kgp = static_cast<const uint8_t*>(k_g1);   // gathered "gist" rows are the level-1 gists
    p.vgp = static_cast<const uint8_t*>(v_g1);
    p.out = static_cast<uint16_t*>(out);
    p.lse = nullptr;
    p.err = reinterpret_cast<uint32_t*>(w + kWsErrOffset);
    p.cnt = reinterpret_cast<uint32_t*>(w + kWsCntOffset);
    p.scores = reinterpret_cast<float*>(w + f.off_scores);
    p.idx = idx2_out ? idx2_out : reinterpret_cast<int32_t*>(w + f.off_idx);
    p.idx1 = idx1_out ? idx1_out : reinterpret_cast<int32_t*>(w + f.off_idx1);
    p.cand_key = reinterpret_cast<uint32_t*>(w + f.off_cand_key);
    p.cand_idx = reinterpret_cast<int32_t*>(w + f.off_cand_idx);
    p.part = reinterpret_cast<float*>(w + f.off_part);
    p.ml = reinterpret_cast<float*>(w + f.off_ml);
    p.rows = f.rows;
    p.Hkv = d.n_kv_heads;
    p.G = f.G;
    p.N = h.n_l2;
    p.NA = h.n_l2;
    p.C = d.chunk;
    p.K = h.top_k2;
    p.W = d.tail_len;
    p.mode = GSA_ALL_GISTS;
    p.tg = f.tg;
    p.upr = f.upr;
    p.T = f.T;
    p.grid = f.grid;
    p.slot_stride = f.slot_stride;
    p.maxs = f.maxs;
    p.nrows_g = 0;
    p.nbt = f.nbt;
    p.tpc = f.tpc;
    p.cb = f.cb;
    const double scale = d.scale > 0 ? (double)d.scale : 1.0 / std::sqrt(128.0);
    p.c2 = (float)(scale * 1.4426950408889634);
    p.do_score = 1;
    p.do_topk = 1;
    p.do_attn_gists = 1;
    p.sel_direct = f.sel_direct;
    p.hier = 1;
    p.group = h.group;
    p.N1 = d.n_chunks;
    p.K1 = d.top_k;
    auto launch = [&](int grid) {
        switch (f.G) {
            case 1: return launch_g<1>(p, grid, st);
            case 2: return launch_g<2>(p, grid, st);
            case 4: return launch_g<4>(p, grid, st);
            default: return launch_g<8>(p, grid, st);
        }
    };
    p.phase = 0;
    cudaError_t e = launch(f.grid);
    if (e == cudaSuccess) {
        p.phase = 1;
        e = launch(f.grid_b);
    }
    return e == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

}  // namespace gsa
