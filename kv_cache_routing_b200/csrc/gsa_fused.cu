// GSA decode step on the 5th-generation tensor cores (bf16, d = 128).
//
// One persistent launch per decode step: at most 148 CTAs, one per SM, all
// resident at once.  A row is one (b, kv-head).  Every CTA runs three stretches,
// the last two side by side:
//
//  keys     Its Stream-K share of the phase-A units, a contiguous range of the
//           units of all rows (a unit is a 128-gist tile or a 128-token tail
//           tile of one row).  Only K is read: S = K . Q^T gives each gist's
//           routing score (summed over the G heads of the group) and the scaled
//           attention logits, which stay in tensor memory (TMEM).  A maximal
//           run of one row's units is a segment; its exact per-head maximum M
//           goes to TMEM too.  The streaming warps then hand the stretch to the
//           unfold warps through a named barrier, and those count the CTA done
//           on every row it met.
//  values   (streaming warps) V of the units whose logits the key stretch
//           kept: P = 2^(x - M) against the segment's exact maximum (nothing
//           is ever rescaled), O^T += V^T . P^T, one partial (M, L, O) per
//           segment.  Then the gathered tiles of the CTA's unfold items, with
//           an online softmax, one partial per item.
//  unfold   (unfold warps, beside the value stretch) Its phase-B item(s):
//           once every CTA that met the item's row has counted itself done (a
//           bounded wait on the row's counter), the row's top-k is taken, and
//           the selected chunks' raw tokens (and in SELECTED_PAIRS mode the
//           selected gists) are gathered into 128-row tiles in the ring: whole
//           chunks by TMA boxes, other rows by cp.async.
// Every partial is counted on its row's ticket; the row's first unfold CTA
// waits (bounded) for the full count and merges the partials (log-sum-exp)
// into out.
//
// Method: gist.science explainer (EN), section 2 "Methodology": gist as
// routing signals, selective unfolding, hybrid attention; Taki-lab slides
// pages 6 and 17 (AG+SR / SG+SR context rules).
//
// Warp roles: warps 0-3 run the softmax (thread t owns key row t of a tile and,
// for O^T, TMEM lane t = output dimension t); warp 4 issues the loads; warp 5
// owns TMEM and issues the MMAs; warps 6-9 (the unfold warps) select, build
// the row tables and issue the gathers.  Shared memory holds a ring of six 32 KiB
// slots; a key-stretch tile takes one (K), a value-stretch tile one (V), a
// gathered tile two (K, V).  Per tile:
//   S   = K_tile . Q^T     M = 128 keys, N = 16 (G heads, rest zero), K = d
//   O^T += V_tile^T . P^T  M = 128 = d,  N = 16 heads,                K = 128 keys
// S is double buffered in TMEM, O^T has one accumulator per segment parity,
// P^T (bf16) and Q are double buffered in shared memory.  TMEM columns:
// S [0, 32), O^T [32, 64), then the logits of the CTA's attended units (G
// columns each) and the maxima of its attended segments (G columns each).
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

// Limit of the waits of one CTA on others (default kWaitLimitNs; a
// diagnostics setter shortens it so that tests can make such a wait run out).
__device__ unsigned long long g_cross_wait_ns = kWaitLimitNs;

constexpr int NT = 192;                      // streaming warps 0-5: softmax 0-3, loads 4, MMA 5
constexpr int NU = 128;                      // unfold warps 6-9: selection, row tables, gathers
constexpr int UFIRST = NT;                   // first unfold thread
constexpr int NTHR = NT + NU;
constexpr int BAR_SOFT = 1, BAR_UNF = 2, BAR_PIPE = 3;   // named barriers (0 is the whole block)
constexpr int BAR_KEYS = 4;                  // the key stretch is done (streaming warps arrive, unfold warps wait)
constexpr int NSL = 4;                       // ring slots
constexpr int PD = 4;                        // P^T buffers (the softmax runs up to PD value tiles ahead of the MMA)
constexpr int D = 128;
constexpr int TILE = 128;
constexpr uint32_t SLOT_BYTES = 32768;       // one 128 x 128 bf16 tensor tile
constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 16, 0, 0);
constexpr uint32_t IDESC_PV = tc::idesc_bf16(128, 16, 1, 0);
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kLogitCol = 64;           // first TMEM column of the kept logits

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t SM_STAGE = 0;
constexpr uint32_t SM_Q = NSL * SLOT_BYTES;          // 2 x 4 KiB: [16 rows][128 B] x 2 K blocks
constexpr uint32_t SM_P = SM_Q + 2 * 4096;           // PD x 4 KiB: P^T [16 heads][128 keys]
constexpr uint32_t SM_WMAX = SM_P + PD * 4096;       // [2][4 warps][16] floats
constexpr uint32_t SM_LRED = SM_WMAX + 2 * 4 * 16 * 4;
constexpr uint32_t SM_TOPK = SM_LRED + 4 * 16 * 4;   // selection scratch
constexpr uint32_t SM_MISC = SM_TOPK + 2048;         // a threshold selection's positions [<= 32], or a radix select's bitmaps [2][<= 128]
constexpr uint32_t SM_SCORE = SM_MISC + 1024;        // key stretch: this CTA's routing scores
constexpr int kScoreCap = 3072;                      // scores kept in shared memory
constexpr uint32_t SM_SEL = SM_SCORE;                // unfold stretch: the row's selection [kSelCap]
constexpr uint32_t SM_ROWTAB = SM_SEL + kSelCap * 4; // unfold stretch: source of each gathered row [kMaxTpc][128]
// hierarchy: the top level's selection at SM_SEL [<= 512], the children tile's
// score keys [128], a lower level's selection [<= 128] (rounds alternate
// between SM_SEL1 and SM_SEL), the children top-k's result [128] and scratch
// after it
constexpr uint32_t SM_CKEY = SM_SEL + 512 * 4;
constexpr uint32_t SM_SEL1 = SM_CKEY + TILE * 4;
constexpr uint32_t SM_HRES = SM_SEL1 + TILE * 4;
constexpr uint32_t SM_HSCR = SM_HRES + TILE * 4;
static_assert(SM_HSCR + 4608 <= SM_ROWTAB, "hierarchy tables overflow the selection buffer");
static_assert(kSelCap * 4 + kMaxTpc * TILE * 4 <= kScoreCap * 4, "unfold tables overflow the score buffer");
constexpr uint32_t SM_UB = SM_SCORE + kScoreCap * 4;  // first unit of every CTA [kFusedCtas + 1]
constexpr uint32_t SM_TMASK = SM_UB + 640;             // key stretch: the tile's gists of a given selection (UNSELECTED_GISTS) [4] u32
constexpr uint32_t SM_BAR = SM_TMASK + 16;
static_assert((kFusedCtas + 1) * 4 <= 640, "unit table overflow");
constexpr uint32_t SMEM_BYTES = SM_BAR + 512 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "dynamic shared memory above the per-block limit");

struct Bars {
    uint64_t full[NSL], empty[NSL];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full[PD], o_done[PD];
    uint64_t q_ready[2];
    uint64_t gdone;              // a gathered stretch is closed (its row table and children keys are free)
    uint64_t gready;             // the first NSL gathered slots are free (their key / value tiles consumed)
    uint32_t tmem;
};
static_assert(sizeof(Bars) <= 512, "mbarriers overflow their shared-memory region");
// a gathered tile takes two consecutive slots from the CTA's first gathered
// one, so with an even ring a tile's slots are both handed over or neither
static_assert(NSL % 2 == 0, "the gathered slots' hand-over assumes an even ring");

// A tile of work: 128 keys of one row.
struct Tile {
    int row;
    int kind;      // 0 gist tile, 1 tail tile, 2 gathered tile (raw chunks [+ gists])
    int t;         // tile index within its kind
    int u;         // kinds 0/1: the unit's index (its logits block)
    int lt;        // gathered tiles: index into the shared row table
    int nvalid;    // kinds 0/1: leading valid rows
    bool score, attn;
};

// A stretch of one role loop.
enum : int { RUN_K = 0, RUN_V = 1, RUN_G = 2 };
struct Run {
    int kind;
    int u0, n;     // RUN_K / RUN_V: units [u0, u0 + n); RUN_G: n tiles of `row` from tile t0
    int row, t0;
    int seq0;      // slot sequence number: RUN_K unit i at seq0 + i; RUN_G tile i at seq0 + 2i (K), + 1 (V)
    int npre;      // RUN_K: value tiles issued early; RUN_V: of those, how many; RUN_G: tiles all threads issued
    int vseq0;     // RUN_K: sequence number of the first early value tile
    int gap;       // RUN_V: value tile j at seq0 + j (j < npre) or seq0 + gap + j
    int slot_b;    // RUN_G: the partial slot
    int score;     // RUN_G: the tile is scored (the hierarchy's children tile)
    int gfirst;    // RUN_V: the first gathered tile's slot sequence number
    int gwait;     // RUN_V: slots from gfirst the producer waits free for the unfold warps
};

// CTA c takes units [ub[c], ub[c + 1]), ub[c] = floor(c * T / grid), a table
// every CTA builds in shared memory at start.
__device__ __forceinline__ int unit_begin(const int* ub, int c) { return ub[c]; }
// The CTA whose range holds unit u (binary search of the table).
__device__ __forceinline__ int cta_of(const int* ub, int grid, int u) {
    int lo = 0, hi = grid - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ub[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ Tile unit_tile(const Params& p, int u) {
    Tile x;
    x.u = u;
    x.row = u / p.upr;
    const int t = u - x.row * p.upr;
    x.lt = 0;
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
    return x;
}

__device__ __forceinline__ Tile gathered_tile(int row, int t, int lt, bool score) {
    Tile x;
    x.row = row;
    x.kind = 2;
    x.t = t;
    x.u = 0;
    x.lt = lt;
    x.nvalid = 0;
    x.score = score;
    x.attn = true;
    return x;
}

// value tile j of a RUN_V stretch: its slot sequence number
__device__ __forceinline__ int value_seq(const Run& r, int j) { return j < r.npre ? r.seq0 + j : r.seq0 + r.gap + j; }

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
    // role counters (each role keeps its own copy; all roles see the same tile sequence)
    int stiles;    // S products so far (S buffer and its barrier phases)
    int ptiles;    // P^T tiles so far (P buffer, p_full / o_done phases)
    int qsegs;     // segments that needed Q (Q buffer, q_ready phases)
    int osegs;     // segments that accumulate O^T (O buffer)
    // softmax role: running state of the current segment
    float m_run[8];
    float l_part[8];
    int had_attn, cur_row, cur_slot;
    int gtiles;    // softmax role: score tiles so far (index into the shared score buffer)
    int ai, aseg;  // softmax role: attended units / attended segments so far (TMEM columns)
    uint32_t mcol; // first TMEM column of the segment maxima
};

// Is slot sequence number `seq` free to fill (its previous use consumed)?
__device__ __forceinline__ bool slot_free(const Params& p, Bars* b, int seq) {
    return seq < NSL || mbar_wait(&b->empty[seq % NSL], ((seq / NSL) - 1) & 1, p.err);
}

// ------------------------------------------------------------ producer --
// One TMA tensor (K or V) of unit tile u into slot `seq` (lane 0 of the producer warp).
__device__ __forceinline__ void load_tensor(const Params& p, Ctx& cx, const Tile& u, int seq, bool v) {
    const int s = seq % NSL;
    uint8_t* dst = cx.base + SM_STAGE + s * SLOT_BYTES;
    uint64_t* bar = &cx.bars->full[s];
    const CUtensorMap* m = v ? (u.kind == 0 ? &p.tm_vg : &p.tm_vt) : (u.kind == 0 ? &p.tm_kg : &p.tm_kt);
    const int y = u.t * TILE;
    mbar_arrive_expect_tx(bar, SLOT_BYTES);
    tc::tma_load_3d(dst, m, 0, y, u.row, bar);
    tc::tma_load_3d(dst + 16384, m, 64, y, u.row, bar);
}

// Gathered tile i of the row table into slots k_seq and k_seq + 1 by the 32
// lanes of the producer warp; each lane holds both phases open until its
// copies land, lane 0 then gives the one expected arrival.
__device__ __forceinline__ void gather_warp(const Params& p, Ctx& cx, int i, int k_seq) {
    const int sk = k_seq % NSL, sv = (k_seq + 1) % NSL;
    uint8_t* ks = cx.base + SM_STAGE + sk * SLOT_BYTES;
    uint8_t* vs = cx.base + SM_STAGE + sv * SLOT_BYTES;
    const int32_t* tab = reinterpret_cast<const int32_t*>(cx.base + SM_ROWTAB) + i * TILE;
    for (int q = cx.lane; q < TILE * 16; q += 32) gather_piece(p, ks, vs, tab[q >> 4], q >> 4, q & 15);
    cp_async_arrive_hold(&cx.bars->full[sk]);
    cp_async_arrive_hold(&cx.bars->full[sv]);
    __syncwarp();
    if (cx.lane == 0) {
        mbar_arrive(&cx.bars->full[sk]);
        mbar_arrive(&cx.bars->full[sv]);
    }
}

__device__ __forceinline__ void produce_run(const Params& p, Ctx& cx, const Run& r) {
    if (r.kind == RUN_K) {
        for (int i = 0; i < r.n; ++i) {
            const int seq = r.seq0 + i;
            if (!slot_free(p, cx.bars, seq)) return;
            if (cx.lane == 0) load_tensor(p, cx, unit_tile(p, r.u0 + i), seq, false);
        }
        // the first value tiles of the CTA, ahead of the unfold stretch
        int j = 0;
        for (int i = 0; i < r.n && j < r.npre; ++i) {
            const Tile u = unit_tile(p, r.u0 + i);
            if (!u.attn) continue;
            const int seq = r.vseq0 + j;
            ++j;
            if (!slot_free(p, cx.bars, seq)) return;
            if (cx.lane == 0) load_tensor(p, cx, u, seq, true);
        }
    } else if (r.kind == RUN_V) {
        int j = 0;
        for (int i = 0; i < r.n; ++i) {
            const Tile u = unit_tile(p, r.u0 + i);
            if (!u.attn) continue;
            if (j >= r.npre) {
                const int seq = value_seq(r, j);
                if (!slot_free(p, cx.bars, seq)) return;
                if (cx.lane == 0) load_tensor(p, cx, u, seq, true);
            }
            ++j;
        }
        // The first gathered tiles take slots whose previous use was a key or
        // value tile many ring turns back, too far for a parity wait by the
        // unfold warps (a phase parity names only the current or the
        // previous phase).  The producer, which walks the ring in order, waits
        // them free and hands them over through one mbarrier.
        if (r.gwait > 0) {
            for (int q = 0; q < r.gwait; ++q)
                if (!slot_free(p, cx.bars, r.gfirst + q)) return;
            if (cx.lane == 0) mbar_arrive(&cx.bars->gready);
        }
    } else {
        // gathered tiles beyond the ones every thread issued up front
        for (int i = r.npre; i < r.n; ++i) {
            const int sk = r.seq0 + 2 * i;
            if (!slot_free(p, cx.bars, sk) || !slot_free(p, cx.bars, sk + 1)) return;
            gather_warp(p, cx, i, sk);
        }
    }
}

// ----------------------------------------------------------------- MMA --
// The MMA thread runs an event loop over a stretch: it issues a tile's S
// product as soon as the tile's K, a free S buffer and (for a new segment)
// its Q are there, and a pending P.V as soon as its P and V are there,
// whichever comes first.
struct PendingPV {
    int vslot, vpar, obuf, first, pj;
};

// The descriptors of the 8 K-steps differ only in the start-address field
// (address / 16, bits 0-13), which never carries out for addresses inside
// shared memory: each is the first one plus a constant.
__device__ __forceinline__ void issue_pv(Ctx& cx, const PendingPV& r) {
    const uint32_t vs = cx.sbase + SM_STAGE + r.vslot * SLOT_BYTES;
    const uint32_t pt = cx.sbase + SM_P + (r.pj % PD) * 4096;
    const uint32_t dO = cx.tmem + 32 + r.obuf * 16;
    const uint64_t a0 = tc::sdesc_sw128(vs, 16384, 1024), b0 = tc::sdesc_sw128(pt, 16, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        tc::mma_bf16(dO, a0 + (uint64_t)(kk * (2048 >> 4)), b0 + (uint64_t)((kk >> 2) * (2048 >> 4) + (kk & 3) * 2),
                     IDESC_PV, (r.first && kk == 0) ? 0u : 1u);
    tc::commit(&cx.bars->o_done[r.pj % PD]);
    tc::commit(&cx.bars->empty[r.vslot]);
}

// S = K_tile . Q^T into TMEM columns dS (8 K-steps of 16 over d = 128).
__device__ __forceinline__ void issue_s(uint32_t dS, uint32_t ks, uint32_t qb) {
    const uint64_t a0 = tc::sdesc_sw128(ks, 16, 1024), b0 = tc::sdesc_sw128(qb, 16, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        tc::mma_bf16(dS, a0 + (uint64_t)((kk >> 2) * (16384 >> 4) + (kk & 3) * 2),
                     b0 + (uint64_t)((kk >> 2) * (2048 >> 4) + (kk & 3) * 2), IDESC_S, kk > 0 ? 1u : 0u);
}

__device__ __forceinline__ void mma_run(const Params& p, Ctx& cx, const Run& r) {
    PendingPV ring[4];
    int head = 0, tail = 0;   // pending P.V products [head, tail)
    int i = 0;                // next tile of the stretch
    int j = 0;                // RUN_V: value tiles so far
    int prev_row = -1;
    uint64_t t_last = sm_cycles();
    int ui = -1;              // the tile whose info `u` holds
    Tile u{};
    for (;;) {
        if (r.kind == RUN_V) {
            while (i < r.n) {
                if (ui != i) {
                    u = unit_tile(p, r.u0 + i);
                    ui = i;
                }
                if (u.attn) break;
                ++i;
            }
        }
        if (i >= r.n && head == tail) break;
        bool prog = false;
        if (i < r.n && tail - head < 4) {
            if (ui != i) {
                u = r.kind == RUN_G ? gathered_tile(r.row, r.t0 + i, i, false) : unit_tile(p, r.u0 + i);
                ui = i;
            }
            const bool ns = u.row != prev_row;
            if (r.kind == RUN_V) {
                // the value tile's data is waited for with its P
                if (ns) cx.osegs++;
                const int seq = value_seq(r, j);
                ring[tail & 3] = PendingPV{seq % NSL, (seq / NSL) & 1, (cx.osegs - 1) & 1, ns ? 1 : 0, cx.ptiles};
                ++tail;
                cx.ptiles++;
                ++j;
                prev_row = u.row;
                ++i;
                prog = true;
            } else {
                const int kseq = r.kind == RUN_K ? r.seq0 + i : r.seq0 + 2 * i;
                const int ks_ = kseq % NSL;
                const int sb = cx.stiles & 1;
                const bool ready = (!ns || mbar_test(&cx.bars->q_ready[cx.qsegs & 1], (cx.qsegs >> 1) & 1)) &&
                                   mbar_test(&cx.bars->full[ks_], (kseq / NSL) & 1) &&
                                   (cx.stiles < 2 || mbar_test(&cx.bars->s_free[sb], ((cx.stiles - 2) >> 1) & 1));
                if (ready) {
                    tc::fence_after();
                    if (ns) cx.qsegs++;
                    if (r.kind == RUN_G) tc::fence_async_smem();   // cp.async (generic proxy) writes -> tensor core reads
                    const uint32_t ks = cx.sbase + SM_STAGE + ks_ * SLOT_BYTES;
                    const uint32_t qb = cx.sbase + SM_Q + ((cx.qsegs - 1) & 1) * 4096;
                    issue_s(cx.tmem + sb * 16, ks, qb);
                    tc::commit(&cx.bars->s_full[sb]);
                    tc::commit(&cx.bars->empty[ks_]);
                    cx.stiles++;
                    if (r.kind == RUN_G) {
                        if (ns) cx.osegs++;
                        const int vseq = kseq + 1;
                        ring[tail & 3] =
                            PendingPV{vseq % NSL, (vseq / NSL) & 1, (cx.osegs - 1) & 1, ns ? 1 : 0, cx.ptiles};
                        ++tail;
                        cx.ptiles++;
                    }
                    prev_row = u.row;
                    ++i;
                    prog = true;
                }
            }
        }
        if (head != tail) {
            const PendingPV& q = ring[head & 3];
            if (mbar_test(&cx.bars->p_full[q.pj % PD], (q.pj / PD) & 1) &&
                mbar_test(&cx.bars->full[q.vslot], q.vpar)) {
                tc::fence_after();
                if (r.kind == RUN_G) tc::fence_async_smem();
                issue_pv(cx, q);
                ++head;
                prog = true;
            }
        }
        if (prog) {
            t_last = sm_cycles();
        } else {
            __nanosleep(20);   // leave the issue slots to the softmax warp sharing this scheduler
            if (sm_cycles() - t_last > kWaitLimitCycles) {
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
    uint8_t* qb = cx.base + SM_Q + (cx.qsegs & 1) * 4096;
    if (h < G) {
        const uint4 v = *reinterpret_cast<const uint4*>(p.q + ((size_t)row * G + h) * D + c * 8);
        *reinterpret_cast<uint4*>(qb + (c >> 3) * 2048 + h * 128 + (((c & 7) ^ (h & 7)) << 4)) = v;
    }
    tc::fence_async_smem();
    mbar_arrive(&cx.bars->q_ready[cx.qsegs & 1]);
    cx.qsegs++;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Close the current attention segment (its O^T accumulator is `obuf`): write
// its partial (M, L, O) to slot cur_slot of cur_row.
template <int G>
__device__ __forceinline__ void finalize_segment(const Params& p, Ctx& cx, uint32_t obuf) {
    const int t = threadIdx.x;
    float O[G];
    if (cx.had_attn) {
        const int pj = cx.ptiles - 1;
        mbar_wait(&cx.bars->o_done[pj % PD], (pj / PD) & 1, p.err);
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
    group_sync<128, BAR_SOFT>();
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
    group_sync<128, BAR_SOFT>();
}

// Close the current key-stretch segment: its exact per-head maximum of the
// scaled logits goes to the partial's m; a segment without attention (gists
// scored only) leaves its whole, empty partial here.
template <int G>
__device__ __forceinline__ void key_close(const Params& p, Ctx& cx) {
    const int t = threadIdx.x;
    float* wmax = reinterpret_cast<float*>(cx.base + SM_WMAX);
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float m;
        asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(cx.m_run[h]));
        if (cx.lane == 0) wmax[cx.warp * 16 + h] = m;
    }
    group_sync<128, BAR_SOFT>();
    if (cx.had_attn) {
        // every lane keeps the maxima of the segment in its TMEM lane
        uint32_t mr[G];
#pragma unroll
        for (int h = 0; h < G; ++h)
            mr[h] = __float_as_uint(fmaxf(fmaxf(wmax[h], wmax[16 + h]), fmaxf(wmax[32 + h], wmax[48 + h])));
        tc::stn<G>(cx.tmem + ((uint32_t)(cx.warp * 32) << 16) + cx.mcol + cx.aseg * G, mr);
        cx.aseg++;
    } else {
        // scored only: the segment's partial is empty
        const size_t slot = (size_t)cx.cur_row * p.slot_stride + cx.cur_slot;
        if (t < G) {
            p.ml[(slot * G + t) * 4 + 0] = -INFINITY;
            p.ml[(slot * G + t) * 4 + 1] = 0.f;
        }
        float* part = p.part + slot * G * D;
#pragma unroll
        for (int h = 0; h < G; ++h) part[h * D + t] = 0.f;
    }
    group_sync<128, BAR_SOFT>();
}

// Chunks of the sequence of `row`: nch[b] clamped into [0, N] (a value
// outside is flagged), or N.
__device__ __forceinline__ int seq_chunks(const Params& p, int row) {
    if (p.nch == nullptr) return p.N;
    const int n = __ldg(p.nch + row / p.Hkv);
    if (n < 0 || n > p.N) {
        atomicOr(p.err, kErrIndex);
        return n < 0 ? 0 : p.N;
    }
    return n;
}

// First raw row of chunk j of `row`: in the dense cache [rows][N][c], or in
// the page pool [n_pages][Hkv][c] (a page outside the pool is clamped into
// it and flagged).
__device__ __forceinline__ long long raw_first(const Params& p, int row, int j) {
    if (p.table == nullptr) return ((long long)row * p.N + j) * p.C;
    const int b = row / p.Hkv, hk = row - b * p.Hkv;
    int pg = __ldg(p.table + (size_t)b * p.N + j);
    if (pg < 0 || pg >= p.n_pages) {
        atomicOr(p.err, kErrIndex);
        pg = pg < 0 ? 0 : p.n_pages - 1;
    }
    return ((long long)pg * p.Hkv + hk) * p.C;
}

// Key stretch, one unit: routing score and scaled logits of key row t.
template <int G, bool PG>
__device__ __forceinline__ void key_tile(const Params& p, Ctx& cx, const Tile& u, bool new_seg, int slot) {
    const int t = threadIdx.x;
    if (new_seg) {
        write_q<G>(p, cx, u.row);
        if (cx.cur_row >= 0) key_close<G>(p, cx);
        cx.cur_row = u.row;
        cx.cur_slot = slot;
        cx.had_attn = 0;
#pragma unroll
        for (int h = 0; h < G; ++h) cx.m_run[h] = -INFINITY;
    }
    const int sb = cx.stiles & 1;
    const bool ok = mbar_wait(&cx.bars->s_full[sb], (cx.stiles >> 1) & 1, p.err);
    cx.stiles++;
    if (!ok) return;
    tc::fence_after();
    uint32_t r[G];
    tc::ldn<G>(cx.tmem + sb * 16 + ((uint32_t)(cx.warp * 32) << 16), r);
    tc::wait_ld();
    tc::fence_before();
    mbar_arrive(&cx.bars->s_free[sb]);
    const bool in_row = t < u.nvalid;
    // gists past the sequence's chunk count do not exist: no weight, score -inf
    bool exists = in_row;
    if constexpr (PG) exists = exists && (p.nch == nullptr || u.kind != 0 || u.t * TILE + t < seq_chunks(p, u.row));
    bool valid = exists;
    if (p.mask_sel && u.kind == 0) {
        // the given selection's gists are not in the context: a 128-bit mask
        // of the tile's selected gists (every thread reads the selection)
        uint32_t* tm = reinterpret_cast<uint32_t*>(cx.base + SM_TMASK);
        if (t < 4) tm[t] = 0u;
        group_sync<128, BAR_SOFT>();
        for (int j = t; j < p.K; j += 128) {
            const int o = __ldg(p.idx + (size_t)u.row * p.K + j) - u.t * TILE;
            if (o >= 0 && o < TILE) atomicOr(&tm[o >> 5], 1u << (o & 31));
        }
        group_sync<128, BAR_SOFT>();
        valid = valid && !((tm[t >> 5] >> (t & 31)) & 1u);
        group_sync<128, BAR_SOFT>();
    }
    if (u.attn) {
        uint32_t xr[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float x = valid ? __uint_as_float(r[h]) * p.c2 : -INFINITY;
            xr[h] = __float_as_uint(x);
            cx.m_run[h] = fmaxf(cx.m_run[h], x);
        }
        tc::stn<G>(cx.tmem + ((uint32_t)(cx.warp * 32) << 16) + kLogitCol + cx.ai * G, xr);
        cx.ai++;
        cx.had_attn = 1;
    }
    if (u.score) {
        float score = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) score += __uint_as_float(r[h]);
        if (in_row) {
            if constexpr (PG) {
                if (!exists) score = -INFINITY;
            }
            p.scores[(size_t)u.row * p.NA + u.t * TILE + t] = score;
            if (cx.gtiles < kScoreCap / TILE)
                reinterpret_cast<float*>(cx.base + SM_SCORE)[cx.gtiles * TILE + t] = score;
        }
        cx.gtiles++;
    }
}

// Value stretch, one unit: P^T = 2^(x - M) from the kept logits x (this
// thread's key row) and the segment's exact maximum M.
template <int G>
__device__ __forceinline__ void value_tile(const Params& p, Ctx& cx, const Tile& u, bool new_seg, int slot,
                                           const float (&x)[G], const float (&M)[G]) {
    const int t = threadIdx.x;
    if (new_seg) {
        if (cx.cur_row >= 0) finalize_segment<G>(p, cx, (cx.osegs - 1) & 1);
        cx.osegs++;
        cx.cur_row = u.row;
        cx.cur_slot = slot;
        cx.had_attn = 1;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            cx.m_run[h] = M[h];
            cx.l_part[h] = 0.f;
        }
    }
    const int pj = cx.ptiles, pb = pj % PD;
    // P^T buffer pb was last read by the P.V of tile pj - PD
    if (pj >= PD) mbar_wait(&cx.bars->o_done[pb], ((pj - PD) / PD) & 1, p.err);
    uint8_t* pt = cx.base + SM_P + pb * 4096;
    const int kb = t >> 6, c16 = (t & 63) >> 3, e = t & 7;
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float pv = (x[h] == -INFINITY || cx.m_run[h] == -INFINITY) ? 0.f : exp2f(x[h] - cx.m_run[h]);
        cx.l_part[h] += pv;
        *reinterpret_cast<uint16_t*>(pt + kb * 2048 + h * 128 + ((c16 ^ (h & 7)) << 4) + e * 2) = f32_to_bf16_rne(pv);
    }
    tc::fence_async_smem();
    tc::fence_before();
    mbar_arrive(&cx.bars->p_full[pb]);
    cx.ptiles = pj + 1;
}

// Unfold stretch, one gathered tile: online softmax (the maximum is not
// known ahead), O^T rescaled lazily when a head's maximum grows by more
// than 2^8.
template <int G>
__device__ __forceinline__ void gathered_softmax(const Params& p, Ctx& cx, const Tile& u, bool new_seg, int slot) {
    const int t = threadIdx.x;
    if (new_seg) {
        write_q<G>(p, cx, u.row);
        if (cx.cur_row >= 0) finalize_segment<G>(p, cx, (cx.osegs - 1) & 1);
        cx.osegs++;
        cx.cur_row = u.row;
        cx.cur_slot = slot;
        cx.had_attn = 0;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            cx.m_run[h] = -INFINITY;
            cx.l_part[h] = 0.f;
        }
    }
    const int sb = cx.stiles & 1;
    const bool ok = mbar_wait(&cx.bars->s_full[sb], (cx.stiles >> 1) & 1, p.err);
    cx.stiles++;
    if (!ok) return;
    tc::fence_after();
    uint32_t r[G];
    const uint32_t lane_off = (uint32_t)(cx.warp * 32) << 16;
    tc::ldn<G>(cx.tmem + sb * 16 + lane_off, r);
    tc::wait_ld();
    tc::fence_before();
    mbar_arrive(&cx.bars->s_free[sb]);
    const bool valid = gathered_valid(cx.base, u.lt, t);
    const int pj = cx.ptiles;
    const int pb = pj % PD;
    float* wmax = reinterpret_cast<float*>(cx.base + SM_WMAX) + (pj & 1) * 64;
    float x[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        x[h] = valid ? __uint_as_float(r[h]) * p.c2 : -INFINITY;
        float m;
        asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(x[h]));
        if (cx.lane == 0) wmax[cx.warp * 16 + h] = m;
    }
    group_sync<128, BAR_SOFT>();
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
        mbar_wait(&cx.bars->o_done[(pj - 1) % PD], ((pj - 1) / PD) & 1, p.err);
        tc::fence_after();
        uint32_t o[G];
        const uint32_t ta = cx.tmem + 32 + ((cx.osegs - 1) & 1) * 16 + lane_off;
        tc::ldn<G>(ta, o);
        tc::wait_ld();
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
        tc::stn<G>(ta, o);
        tc::wait_st();
    }
    if (pj >= PD) mbar_wait(&cx.bars->o_done[pb], ((pj - PD) / PD) & 1, p.err);
    uint8_t* pt = cx.base + SM_P + pb * 4096;
    const int kb = t >> 6, c16 = (t & 63) >> 3, e = t & 7;
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float pv = (x[h] == -INFINITY) ? 0.f : exp2f(x[h] - cx.m_run[h]);
        cx.l_part[h] = cx.l_part[h] * alpha[h] + pv;
        *reinterpret_cast<uint16_t*>(pt + kb * 2048 + h * 128 + ((c16 ^ (h & 7)) << 4) + e * 2) = f32_to_bf16_rne(pv);
    }
    tc::fence_async_smem();
    tc::fence_before();
    mbar_arrive(&cx.bars->p_full[pb]);
    cx.ptiles = pj + 1;
    cx.had_attn = 1;
    if (u.score) {
        // hierarchy: the scores of the children tile, as keys for the next level's selection
        float score = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) score += __uint_as_float(r[h]);
        reinterpret_cast<uint32_t*>(cx.base + SM_CKEY)[t] = valid ? order_key(score) : 0u;
    }
}

template <int G, bool PG>
__device__ __forceinline__ void softmax_run(const Params& p, Ctx& cx, const Run& r) {
    const int* ub = reinterpret_cast<const int*>(cx.base + SM_UB);
    const int c = blockIdx.x;
    auto seg_slot = [&](int row) { return c - cta_of(ub, p.grid, row * p.upr); };
    if (r.kind == RUN_K) {
        int prev_row = -1;
        for (int i = 0; i < r.n; ++i) {
            const Tile u = unit_tile(p, r.u0 + i);
            const bool ns = u.row != prev_row;
            key_tile<G, PG>(p, cx, u, ns, ns ? seg_slot(u.row) : cx.cur_slot);
            prev_row = u.row;
        }
        if (cx.cur_row >= 0) key_close<G>(p, cx);
        tc::wait_st();   // the kept logits and maxima are in TMEM before the value stretch reads them
    } else if (r.kind == RUN_V) {
        // the logits of value tile j and the maxima of attended segment s were
        // kept in this thread's TMEM lane by the key stretch
        const uint32_t lane_off = (uint32_t)(cx.warp * 32) << 16;
        int prev_row = -1, j = 0, sg = 0;
        float M[G];
#pragma unroll
        for (int h = 0; h < G; ++h) M[h] = -INFINITY;
        for (int i = 0; i < r.n; ++i) {
            const Tile u = unit_tile(p, r.u0 + i);
            if (!u.attn) continue;
            const bool ns = u.row != prev_row;
            uint32_t xr[G], mr[G];
            tc::ldn<G>(cx.tmem + lane_off + kLogitCol + j * G, xr);
            if (ns) tc::ldn<G>(cx.tmem + lane_off + cx.mcol + sg * G, mr);
            tc::wait_ld();
            float x[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                x[h] = __uint_as_float(xr[h]);
                if (ns) M[h] = __uint_as_float(mr[h]);
            }
            value_tile<G>(p, cx, u, ns, ns ? seg_slot(u.row) : cx.cur_slot, x, M);
            sg += ns ? 1 : 0;
            prev_row = u.row;
            ++j;
        }
        if (j > 0) finalize_segment<G>(p, cx, (cx.osegs - 1) & 1);
    } else {
        for (int i = 0; i < r.n; ++i)
            gathered_softmax<G>(p, cx, gathered_tile(r.row, r.t0 + i, i, r.score != 0), i == 0, r.slot_b);
        if (r.n > 0) finalize_segment<G>(p, cx, (cx.osegs - 1) & 1);
        mbar_arrive(&cx.bars->gdone);   // the row table (and the children keys) may be rewritten
    }
    cx.cur_row = -1;
}

// Run the three roles over one stretch.  Ends with the streaming warps
// synchronised and every segment of the stretch closed.
template <int G, bool PG>
__device__ __forceinline__ void run_pipeline(const Params& p, Ctx& cx, const Run& r) {
    if (cx.warp == 4) {
        produce_run(p, cx, r);
    } else if (cx.warp == 5) {
        if (cx.lane == 0) mma_run(p, cx, r);
    } else {
        softmax_run<G, PG>(p, cx, r);
    }
    group_sync<NT, BAR_PIPE>();
}

// ----------------------------------------------------------- selection --
// Everything from here to the merge runs on the unfold warps (threads
// [NT, NT + NU), named barrier BAR_UNF), beside the streaming warps.

__device__ __forceinline__ int utid() { return (int)threadIdx.x - UFIRST; }
__device__ __forceinline__ void usync() { group_sync<NU, BAR_UNF>(); }

// Where a selection reads its keys.
enum : int { SRC_GSCORE = 0, SRC_SSCORE = 1, SRC_GKEY = 2, SRC_SKEY = 3 };

__device__ __forceinline__ uint32_t load_key_bits(const void* src, int kind, int i) {
    switch (kind) {
        case SRC_GSCORE: return __float_as_uint(__ldcg(static_cast<const float*>(src) + i));
        case SRC_SSCORE: return __float_as_uint(static_cast<const float*>(src)[i]);
        case SRC_GKEY: return __ldcg(static_cast<const uint32_t*>(src) + i);
        default: return static_cast<const uint32_t*>(src)[i];
    }
}
// scores are mapped to orderable keys; keys pass through
__device__ __forceinline__ uint32_t key_of_bits(uint32_t bits, int kind) {
    return (kind == SRC_GSCORE || kind == SRC_SSCORE) ? order_key(__uint_as_float(bits)) : bits;
}

// Thread t takes positions t, t + NU, t + 2 NU, ...: every warp-wide load is
// one contiguous line.  k <= 32: the threshold selection; otherwise, or when
// equal keys flood the threshold's bound, the radix select on the same
// registers.
template <int U, class Emit>
__device__ __forceinline__ void select_regs(const void* src, int kind, int n, int k, int32_t* tmp, uint32_t* w,
                                            uint32_t* bm, Emit emit) {
    const int lo = utid();
    const int mine = lo < n ? (n - lo + NU - 1) / NU : 0;
    uint32_t key[U];
#pragma unroll
    for (int i = 0; i < U; ++i) key[i] = i < mine ? load_key_bits(src, kind, lo + i * NU) : 0u;   // all loads first
#pragma unroll
    for (int i = 0; i < U; ++i) key[i] = i < mine ? key_of_bits(key[i], kind) : 0u;
    if (k <= 32 && threshold_topk_regs<NU, U, BAR_UNF, UFIRST>(key, lo, NU, mine, k, tmp, w)) {
        for (int r = utid(); r < k; r += NU) emit(r, tmp[r]);
        return;
    }
    radix_topk_regs<NU, U, BAR_UNF, UFIRST>(key, mine, n, k, w, bm, emit);
}

// Exact top-k of n keys (read from `src` as `kind` says), ties to the lower
// position, the selected positions in ascending order: into res[0..k), or,
// when `ck` is given, as candidates (ck[r] = key, ci[r] = pos0 + pos).  n <= 32
// NU: every thread's keys in registers (all loaded at once), the threshold
// selection for k <= 32, else the radix select on those registers (also when
// equal keys flood the threshold's bound); larger n: the radix select reading
// the keys where they are.  Neither res nor the scratch may overlap the keys.
// Every caller goes through this one body (the unfold path runs once per
// launch, cold, so its code is kept small).
__device__ __forceinline__ void unfold_topk(const void* src, int kind, int n, int k, int32_t* res, uint32_t* w,
                                            int32_t* tmp, uint32_t* ck, int32_t* ci, int pos0) {
    auto emit = [&](int r, int pos) {
        if (ck != nullptr) {
            ck[r] = key_of_bits(load_key_bits(src, kind, pos), kind);
            ci[r] = pos0 + pos;
        } else {
            res[r] = pos;
        }
    };
    if (k >= n) {
        for (int i = utid(); i < n; i += NU) emit(i, i);
    } else {
        // the radix select's bitmaps (2 ceil(n / 32) words) share the tmp buffer
        uint32_t* bm = reinterpret_cast<uint32_t*>(tmp);
        if (n <= 16 * NU) {
            select_regs<16>(src, kind, n, k, tmp, w, bm, emit);
        } else if (n <= 32 * NU) {
            select_regs<32>(src, kind, n, k, tmp, w, bm, emit);
        } else {
            block_topk<NU, BAR_UNF, UFIRST>(
                n, k, [&](int i) { return key_of_bits(load_key_bits(src, kind, i), kind); }, emit, w);
        }
    }
    usync();
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
    // the candidates go straight to global memory: nothing is written over
    // the scores while they are read
    unfold_topk(in_smem ? (const void*)ss : (const void*)sg, in_smem ? SRC_SSCORE : SRC_GSCORE, g1 - g0, p.K,
                nullptr, reinterpret_cast<uint32_t*>(base + SM_TOPK), reinterpret_cast<int32_t*>(base + SM_MISC), ck,
                ci, g0);
}

// The row's exact top-k into the shared selection sel[0..k) and, when
// `publish`, into the row's idx output: from the candidates that every CTA
// meeting the row left (n of them), or straight from its routing scores.
template <bool PG>
__device__ __forceinline__ void merge_select(const Params& p, uint8_t* base, int row, int n, bool publish) {
    const int32_t* ci = p.cand_idx + (size_t)row * p.NA;
    int32_t* out = p.idx + (size_t)row * p.K;
    int32_t* sel = reinterpret_cast<int32_t*>(base + SM_SEL);
    unfold_topk(p.cand_key + (size_t)row * p.NA, SRC_GKEY, n, p.K, sel, reinterpret_cast<uint32_t*>(base + SM_TOPK),
                reinterpret_cast<int32_t*>(base + SM_MISC), nullptr, nullptr, 0);
    const int nb = PG ? seq_chunks(p, row) : p.N;
    for (int r = utid(); r < min(p.K, n); r += NU) {
        int32_t j = __ldcg(ci + sel[r]);
        if (PG && j >= nb) j = -1;   // a sequence shorter than k: the place is empty
        sel[r] = j;
        if (publish) out[r] = j;
    }
    usync();
}

template <bool PG>
__device__ __forceinline__ void direct_select(const Params& p, uint8_t* base, int row, bool publish) {
    int32_t* out = p.idx + (size_t)row * p.K;
    int32_t* sel = reinterpret_cast<int32_t*>(base + SM_SEL);
    unfold_topk(p.scores + (size_t)row * p.NA, SRC_GSCORE, p.NA, p.K, sel, reinterpret_cast<uint32_t*>(base + SM_TOPK),
                reinterpret_cast<int32_t*>(base + SM_MISC), nullptr, nullptr, 0);
    if (PG && p.nch != nullptr) {
        const int nb = seq_chunks(p, row);
        for (int r = utid(); r < p.K; r += NU)
            if (sel[r] >= nb) sel[r] = -1;   // a sequence shorter than k: the place is empty
        usync();
    }
    if (publish)
        for (int r = utid(); r < min(p.K, p.NA); r += NU) out[r] = sel[r];
}

// A given selection (gsa_unfold_attn) into sel[0..k); -1 is an empty place
// (a variable-size selection such as top-p's), any other index outside
// [0, N) is clamped into range and flagged in the error word.
__device__ __forceinline__ void load_selection(const Params& p, uint8_t* base, int row) {
    int32_t* sel = reinterpret_cast<int32_t*>(base + SM_SEL);
    for (int r = utid(); r < p.K; r += NU) {
        int32_t j = __ldcg(p.idx + (size_t)row * p.K + r);
        if (j != -1 && (j < 0 || j >= p.N)) {
            atomicOr(p.err, kErrIndex);
            j = j < 0 ? 0 : p.N - 1;
        }
        sel[r] = j;
    }
    usync();
}

// The source of every row of the gathered tiles [t0, t0 + ntl) of `row` into
// the shared row table.
template <bool PG>
__device__ __forceinline__ void build_table(const Params& p, uint8_t* base, int row, int t0, int ntl) {
    const int32_t* sel = reinterpret_cast<const int32_t*>(base + SM_SEL);
    int32_t* tab = reinterpret_cast<int32_t*>(base + SM_ROWTAB);
    const int kc = p.K * p.C;
    for (int i = utid(); i < ntl * TILE; i += NU) {
        const int gr = t0 * TILE + i;
        int32_t e = -1;
        if (gr < kc) {
            const int sidx = gr / p.C, tok = gr - sidx * p.C;
            if (sel[sidx] >= 0)
                e = (int32_t)((PG ? raw_first(p, row, sel[sidx]) : ((long long)row * p.N + sel[sidx]) * p.C) + tok);
        } else if (gr < p.nrows_g) {
            if (sel[gr - kc] >= 0) e = (int32_t)(-((long long)row * p.N + sel[gr - kc]) - 2);
        }
        tab[i] = e;
    }
    usync();
}

// Hierarchy levels (1-based: level 1 has one gist per chunk, level L is the
// top): gist count, selection size and selection output of level l.
__device__ __forceinline__ int lvl_n(const Params& p, int l) {
    return l == 1 ? p.N1 : l == p.levels ? p.N : p.midN[l - 2];
}
__device__ __forceinline__ int lvl_k(const Params& p, int l) {
    return l == 1 ? p.K1 : l == p.levels ? p.K : p.midK[l - 2];
}
__device__ __forceinline__ int32_t* lvl_idx(const Params& p, int l) {
    return l == 1 ? p.idx1 : l == p.levels ? p.idx : p.midIdx[l - 2];
}
// Tile lt of the row table into slots seq, seq + 1 (K, V) once the slots'
// previous contents are consumed.  Its first tma_rows rows are runs of h
// consecutive source rows (selected chunks, or the children of selected
// groups) starting at multiples of h: one thread moves each run with four TMA
// boxes (K and V, two 64-column halves each) that land in the swizzled
// layout, h being a multiple of 8; the other rows (selected gists, empty rows)
// are copied by every unfold thread with cp.async.  The copiers hold each
// phase open until their copies have landed, the TMA bytes are expected on
// it, and one thread then gives the one expected arrival.
template <bool PG>
__device__ __forceinline__ void gather_tile(const Params& p, uint8_t* base, Bars* bars, int lt, int seq, int row,
                                            int tma_rows, int h, bool children, int gfirst, int cl) {
    if (seq < gfirst + NSL) {
        // handed over by the producer (see the value stretch)
        mbar_wait(&bars->gready, 0, p.err);
    } else {
        // the previous use of these slots is this CTA's own gathered tile
        // NSL / 2 tiles back: one phase behind, so a parity wait is exact
        slot_free(p, bars, seq);
        slot_free(p, bars, seq + 1);
    }
    const int sk = seq % NSL, sv = (seq + 1) % NSL;
    uint8_t* ks = base + SM_STAGE + sk * SLOT_BYTES;
    uint8_t* vs = base + SM_STAGE + sv * SLOT_BYTES;
    const int32_t* tab = reinterpret_cast<const int32_t*>(base + SM_ROWTAB) + lt * TILE;
    // lane 0 of each unfold warp issues every fourth run (TMA issue, not the
    // copy, sets the pace: about 45 ns an instruction), expecting its own
    // bytes first; the phase cannot complete before the final arrival below
    const int uw = utid() >> 5;
    if (tma_rows > 0 && (utid() & 31) == 0 && uw * h < tma_rows) {
        // runs of empty places (-1 in the table) are not loaded: their V rows
        // are zeroed below with the other rows that are not whole runs
        int runs = 0;
        for (int r = uw * h; r < tma_rows; r += (NU / 32) * h) runs += tab[r] != -1 ? 1 : 0;
        const uint32_t bytes = (uint32_t)(runs * h) * (D * 2);
        mbar_expect_tx(&bars->full[sk], bytes);
        mbar_expect_tx(&bars->full[sv], bytes);
        // children of level cl: level 1's own maps, the middle levels' from their arrays
        const CUtensorMap* mk = children ? (cl == 1 ? &p.tm_kc : &p.tm_kcm[cl - 2]) : &p.tm_kr;
        const CUtensorMap* mv = children ? (cl == 1 ? &p.tm_vc : &p.tm_vcm[cl - 2]) : &p.tm_vr;
        const long long nch = children ? (long long)lvl_n(p, cl) : 0;
        for (int r = uw * h; r < tma_rows; r += (NU / 32) * h) {
            const long long e = tab[r];
            if (e == -1) continue;
            // the run's source: a whole chunk (box {64, c, 1} at chunk e / c of
            // the raw map), or the first child of a group in the row's level-1 gists
            int y, z;
            if (children) {
                y = (int)(-e - 2 - (long long)row * nch);
                z = row;
            } else if (PG && p.table != nullptr) {
                // pool rows are below 2^31 (checked on the host): 32-bit division
                z = (int)((uint32_t)e / (uint32_t)p.C);
                y = (int)e - z * p.C;
            } else {
                // dense: token chunk * c of the row's raw rows
                z = row;
                y = (int)(e - (long long)row * (p.hier ? p.N1 : p.N) * p.C);
            }
            tc::tma_load_3d(ks + r * 128, mk, 0, y, z, &bars->full[sk]);
            tc::tma_load_3d(ks + 16384 + r * 128, mk, 64, y, z, &bars->full[sk]);
            tc::tma_load_3d(vs + r * 128, mv, 0, y, z, &bars->full[sv]);
            tc::tma_load_3d(vs + 16384 + r * 128, mv, 64, y, z, &bars->full[sv]);
        }
    }
#pragma unroll 4
    for (int q = utid(); q < (TILE - tma_rows) * 16; q += NU) {
        const int r = tma_rows + (q >> 4);
        gather_piece(p, ks, vs, tab[r], r, q & 15);
    }
    // runs skipped above (an empty place of a variable-size selection): their
    // V rows zeroed.  One table read per run (a broadcast), so a tile with no
    // empty place costs a handful of loads, not a pass over its pieces
    for (int r0 = 0; r0 < tma_rows; r0 += h) {
        if (tab[r0] != -1) continue;
        for (int q = utid(); q < h * 16; q += NU) gather_piece(p, ks, vs, -1, r0 + (q >> 4), q & 15);
    }
    cp_async_arrive_hold(&bars->full[sk]);
    cp_async_arrive_hold(&bars->full[sv]);
    usync();
    if (utid() == 0) {
        mbar_arrive(&bars->full[sk]);
        mbar_arrive(&bars->full[sv]);
    }
}

// The selection made at the start of unfold round rd (round 0: the top
// level's), kept in shared memory; consecutive rounds alternate buffers, so a
// round's selection never overwrites the parents it is read against.
__device__ __forceinline__ int32_t* round_sel(uint8_t* base, int rd) {
    return reinterpret_cast<int32_t*>(base + ((rd & 1) ? SM_SEL1 : SM_SEL));
}

// Hierarchy, round rd < L - 1: the row table of the children tile, the
// level-(L-1-rd) gists of the groups that round rd's selection (one level up)
// picked, group after group (a short last group leaves empty rows).
__device__ __forceinline__ void hier_children_table(const Params& p, uint8_t* base, int row, int rd) {
    const int cl = p.levels - 1 - rd;                 // the children's level
    const int32_t* par = round_sel(base, rd);
    const int kp = lvl_k(p, cl + 1), g = p.grp[cl - 1], nch = lvl_n(p, cl);
    int32_t* tab = reinterpret_cast<int32_t*>(base + SM_ROWTAB);
    for (int r = utid(); r < TILE; r += NU) {
        int32_t e = -1;
        if (r < kp * g) {
            const int child = par[r / g] * g + r % g;
            if (child < nch) e = (int32_t)(-((long long)row * nch + child) - 2);
        }
        tab[r] = e;
    }
    usync();
}

// Hierarchy, round rd >= 1: the exact top-k of the children tile that round
// rd - 1 attended and scored (level L - rd; ties to the lower index: the tile
// holds the children in ascending order), published and kept as round rd's
// selection; then the next table: that level's children, or at level 1 the
// raw tokens of the selected chunks.
__device__ __forceinline__ void hier_select_children(const Params& p, uint8_t* base, int row, int rd) {
    const int lv = p.levels - rd;                     // the level selected here
    const uint32_t* keys = reinterpret_cast<const uint32_t*>(base + SM_CKEY);
    const int32_t* par = round_sel(base, rd - 1);
    int32_t* sel1 = round_sel(base, rd);
    int32_t* res = reinterpret_cast<int32_t*>(base + SM_HRES);
    uint32_t* scratch = reinterpret_cast<uint32_t*>(base + SM_HSCR);
    const int g = p.grp[lv - 1];
    const int n = min(TILE, lvl_k(p, lv + 1) * g);
    const int k = lvl_k(p, lv);
    int32_t* out = lvl_idx(p, lv);
    unfold_topk(keys, SRC_SKEY, n, k, res, scratch, reinterpret_cast<int32_t*>(base + SM_MISC), nullptr, nullptr, 0);
    for (int r = utid(); r < k; r += NU) {
        const int pos = res[r];
        const int child = par[pos / g] * g + pos % g;
        sel1[r] = child;
        out[(size_t)row * k + r] = child;
    }
    usync();
    if (lv > 1) {
        hier_children_table(p, base, row, rd);
        return;
    }
    int32_t* tab = reinterpret_cast<int32_t*>(base + SM_ROWTAB);
    for (int r = utid(); r < TILE; r += NU) {
        int32_t e = -1;
        if (r < k * p.C) {
            const int sl = r / p.C;
            e = (int32_t)(((long long)row * p.N1 + sel1[sl]) * p.C + (r - sl * p.C));
        }
        tab[r] = e;
    }
    usync();
}

// Wait (bounded) until counter `ctr` reaches `target`; the writes published
// before it are then visible to the whole group.  The comparison is
// wrap-aware (the signed difference), so a counter word that holds a value
// half the 32-bit range away never reaches the target: the wait then runs
// out, flags kErrTimeout and the kernel carries on to its normal end.
template <int GN, int GBAR>
__device__ __forceinline__ void wait_count(const Params& p, const uint32_t* ctr, uint32_t target, bool leader) {
    if (leader) {
        const uint64_t t0 = global_ns();
        const uint64_t limit = g_cross_wait_ns;
        while ((int32_t)(ld_acquire_u32(ctr) - target) < 0) {
            __nanosleep(100);
            if (global_ns() - t0 > limit) {
                atomicOr(p.err, kErrTimeout);
                break;
            }
        }
    }
    group_sync<GN, GBAR>();
}

// Final log-sum-exp merge of a row: slots [0, na) of the CTAs that met the
// row and slots [maxs, maxs + nb) of its unfold partials.  The partials are
// brought into shared memory with cp.async in groups (one memory round trip
// per group).  Per group, warp h finds head h's largest slot maximum M_g and
// each slot's weight 2^(m_s - M_g) and the weighted sum L_g of the l_s; each
// output is then a plain weighted sum over the slots (independent products,
// no dependent rescaling chain), folded into a running (M, L, acc) once per
// group.  Leaves the row's ticket and key counter zero for the next call.
template <int G>
__device__ __forceinline__ void merge_row(const Params& p, uint8_t* base, int row, int na, int nb) {
    constexpr int NW = NTHR / 32;
    const int nsl = na + nb;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int PER = (G * D + NTHR - 1) / NTHR;          // outputs per thread
    constexpr int GS = (int)((SLOT_BYTES * NSL - 256) / ((G * D + 5 * G) * 4));   // slots per group
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
        for (int q = threadIdx.x; q < cnt * (G * D / 4); q += NTHR) {
            const int i = q / (G * D / 4), e4 = q - i * (G * D / 4);
            cp_async16(so + (size_t)i * G * D + e4 * 4, p.part + (size_t)sidx(i) * G * D + e4 * 4);
        }
#pragma unroll 1
        for (int q = threadIdx.x; q < cnt * G; q += NTHR) {
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
            const int i = threadIdx.x + q * NTHR;
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
        const int i = threadIdx.x + q * NTHR;
        if (i < G * D) {
            const int h = i / D, e = i % D;
            p.out[((size_t)row * G + h) * D + e] = f32_to_bf16_rne(acc[q] / L[q]);
            if (p.lse != nullptr && e == 0) p.lse[(size_t)row * G + h] = (M[q] + log2f(L[q])) * 0.69314718055994531f;
        }
    }
    if (threadIdx.x == 0) {
        p.cnt[row] = 0;
        p.kdone[row] = 0;
    }
}

// ---------------------------------------------------------------- kernel --
// PG: the raw cache is paged or the sequences have their own chunk counts
template <int G, bool PG>
__global__ void __launch_bounds__(NTHR, 1) fused_decode_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    Ctx cx;
    cx.base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    cx.sbase = smem_u32(cx.base);
    cx.bars = reinterpret_cast<Bars*>(cx.base + SM_BAR);
    cx.warp = threadIdx.x >> 5;
    cx.lane = threadIdx.x & 31;
    cx.stiles = cx.ptiles = cx.qsegs = cx.osegs = 0;
    cx.had_attn = 0;
    cx.cur_row = -1;
    cx.cur_slot = 0;
    cx.gtiles = 0;
    cx.ai = cx.aseg = 0;

    // the Q and P^T rows of heads >= G must be zero (slots need no clearing:
    // TMA zero-fills past a row's end, and a gathered tile zeroes the V rows
    // it leaves empty)
    for (uint32_t o = SM_Q + threadIdx.x * 16; o < SM_WMAX; o += NTHR * 16)
        *reinterpret_cast<uint4*>(cx.base + o) = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        Bars* b = cx.bars;
        for (int i = 0; i < NSL; ++i) {
            // one expected arrival per fill: the TMA issuer's (with the byte
            // count), or the gatherer's after every copier holds the phase
            mbar_init(&b->full[i], 1);
            mbar_init(&b->empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&b->s_full[i], 1);
            mbar_init(&b->s_free[i], 128);
            mbar_init(&b->q_ready[i], 128);
        }
        for (int i = 0; i < PD; ++i) {
            mbar_init(&b->p_full[i], 128);
            mbar_init(&b->o_done[i], 1);
        }
        mbar_init(&b->gdone, 128);
        mbar_init(&b->gready, 1);
        fence_mbar_init();
    }
    if (threadIdx.x == 32 * 4) {
        // fetch the tensor maps' descriptors ahead of the first loads
        if (p.tg > 0) asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_kg) : "memory");
        if (p.tg > 0 && p.do_attn_gists) asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_vg) : "memory");
        if (p.W > 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_kt) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_vt) : "memory");
        }
    }
    if (threadIdx.x == UFIRST) {
        // and those of the gathers
        if (p.tma_raw) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_kr) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_vr) : "memory");
        }
        if (p.tma_children) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_kc) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(&p.tm_vc) : "memory");
        }
    }
    for (int i = threadIdx.x; i <= p.grid; i += NTHR)
        reinterpret_cast<int*>(cx.base + SM_UB)[i] = (int)((long long)i * p.T / p.grid);
    tc::fence_async_smem();
    if (cx.warp == 5) {
        tc::tmem_alloc(&cx.bars->tmem, (uint32_t)p.tmem_cols);
        tc::tmem_relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    cx.tmem = cx.bars->tmem;
    pdl_wait();                  // the previous step on this stream is complete (workspace reuse)
    pdl_launch_dependents();

    const int c = blockIdx.x;
    const int* ub = reinterpret_cast<const int*>(cx.base + SM_UB);
    const int u0 = unit_begin(ub, c);
    const int n1 = unit_begin(ub, c + 1) - u0;
    // the CTAs whose ranges meet `row` (their count, the first one)
    auto row_ctas = [&](int row, int& cf) {
        if (p.T == 0) {
            cf = 0;
            return 0;
        }
        const int ru0 = row * p.upr;
        cf = cta_of(ub, p.grid, ru0);
        return cta_of(ub, p.grid, ru0 + p.upr - 1) - cf + 1;
    };
    // gists of `row` scored by CTA cc: [g0, g1)
    auto gists_of = [&](int cc, int row, int& g0, int& g1) {
        const int ru0 = row * p.upr;
        const int a = max(unit_begin(ub, cc), ru0), b = min(unit_begin(ub, cc + 1), ru0 + p.tg);
        g0 = (a - ru0) * TILE;
        g1 = b > a ? min((b - ru0) * TILE, p.NA) : g0;
    };
    // the hierarchy's rounds: one children tile per level below the top, then
    // the raw tile of the level-1 selection (none when k1 = 0)
    const int rounds = p.hier ? (p.K1 > 0 ? p.levels : p.levels - 1) : 1;
    // gathered tiles of unfold item `it`, round rd: [t0, t0 + ntl) of its row
    auto item_tiles = [&](int it, int rd, int& t0) {
        if (p.hier) {
            t0 = rd;
            return 1;
        }
        t0 = (it % p.cb) * p.tpc;
        return max(0, min(p.nbt, t0 + p.tpc) - t0);
    };
    int n2 = 0;   // attended units of this CTA (its value tiles)
    for (int i = 0; i < n1; ++i) n2 += unit_tile(p, u0 + i).attn ? 1 : 0;
    cx.mcol = kLogitCol + (uint32_t)(n2 * G);
    const int row_first = n1 > 0 ? u0 / p.upr : 0;
    const int row_last = n1 > 0 ? (u0 + n1 - 1) / p.upr : -1;
    // slots: keys [0, n1), values [n1, n1 + n2), then two per gathered tile
    const int gseq0 = n1 + n2;
    int gtiles_total = 0;   // gathered tiles of this CTA's unfold items
    for (int it = c; it < p.items; it += p.grid)
        for (int rd = 0; rd < rounds; ++rd) {
            int t0;
            gtiles_total += max(0, item_tiles(it, rd, t0));
        }

    // ------------------------------------------------------ key stretch --
    if (cx.warp < 6) {
        Run rk{};
        rk.kind = RUN_K;
        rk.u0 = u0;
        rk.n = n1;
        rk.seq0 = 0;
        rk.npre = min(n2, NSL);   // the first value tiles follow the keys without a gap
        rk.vseq0 = n1;
        run_pipeline<G, PG>(p, cx, rk);
        // the scores are written (global and shared memory): hand them to the
        // unfold warps, which publish them, and go on without waiting
        asm volatile("bar.arrive %0, %1;" ::"n"(BAR_KEYS), "n"(NTHR) : "memory");
        // ------------------------------------------------ value stretch --
        Run rv{};
        rv.kind = RUN_V;
        rv.u0 = u0;
        rv.n = n1;
        rv.seq0 = n1;
        rv.npre = min(n2, NSL);
        rv.gap = 0;
        rv.gfirst = gseq0;
        rv.gwait = min(NSL, 2 * gtiles_total);
        run_pipeline<G, PG>(p, cx, rv);
        // ------------------------------------ gathered tiles, item by item --
        int gseq = gseq0;
        for (int it = c; it < p.items; it += p.grid) {
            for (int rd = 0; rd < rounds; ++rd) {
                int t0;
                const int ntl = item_tiles(it, rd, t0);
                if (ntl <= 0) continue;
                Run rg{};
                rg.kind = RUN_G;
                rg.row = it / p.cb;
                rg.t0 = t0;
                rg.n = ntl;
                rg.seq0 = gseq;
                rg.npre = ntl;   // every tile is gathered by the unfold warps
                rg.slot_b = p.maxs + (p.hier ? rd : it % p.cb);
                rg.score = (p.hier && rd < p.levels - 1) ? 1 : 0;   // children tiles are scored
                run_pipeline<G, PG>(p, cx, rg);
                gseq += 2 * ntl;
            }
        }
    } else {
        // ----------------------------------------------- unfold warps --
        const bool lead = utid() == 0;
        asm volatile("bar.sync %0, %1;" ::"n"(BAR_KEYS), "n"(NTHR) : "memory");
        if (p.do_topk && !p.sel_direct) {
            // local top-k of every segment, from the scores this CTA kept
            int ntiles = 0;
            for (int r = row_first; r <= row_last; ++r) {
                int a0, a1;
                gists_of(c, r, a0, a1);
                ntiles += (a1 - a0 + TILE - 1) / TILE;
            }
            const bool fits = ntiles <= kScoreCap / TILE;
            int sfirst = 0;   // score-tile offset of the segment in the shared buffer
            for (int r = row_first; r <= row_last; ++r) {
                int g0, g1;
                gists_of(c, r, g0, g1);
                if (g1 <= g0) continue;
                int cf;
                row_ctas(r, cf);
                int off = 0;
                for (int cc = cf; cc < c; ++cc) {
                    int a0, a1;
                    gists_of(cc, r, a0, a1);
                    off += min(p.K, max(0, a1 - a0));
                }
                local_topk(p, cx.base, r, g0, g1, sfirst * TILE, off, fits);
                sfirst += (g1 - g0 + TILE - 1) / TILE;
            }
            usync();
        }
        // scores (and candidates) of every row this CTA met are out.  The
        // lead's fence is cumulative: it orders before the counters the
        // streaming warps' scores and the unfold warps' candidates, which the
        // barriers above made visible to it.
        if (lead) {
            __threadfence();
            for (int r = row_first; r <= row_last; ++r) atomicAdd(p.kdone + r, 1u);
        }
        int gseq = gseq0, runs = 0;
        for (int it = c; it < p.items; it += p.grid) {
            const int row = it / p.cb, j = it % p.cb;
            int cf;
            const int na = row_ctas(row, cf);
            if (p.do_topk) wait_count<NU, BAR_UNF>(p, p.kdone + row, (uint32_t)na, lead);
            for (int rd = 0; rd < rounds; ++rd) {
                int t0;
                const int ntl = item_tiles(it, rd, t0);
                if (ntl <= 0) continue;
                // the previous gathered stretch is closed: its row table (and
                // the hierarchy's children keys) are free
                if (runs > 0) {
                    if (lead) mbar_wait(&cx.bars->gdone, (runs - 1) & 1, p.err);
                    usync();
                }
                if (rd >= 1) {
                    hier_select_children(p, cx.base, row, rd);
                } else {
                    if (p.do_topk && p.sel_direct) {
                        direct_select<PG>(p, cx.base, row, j == 0);
                    } else if (p.do_topk) {
                        int n = 0;
                        for (int cc = cf; cc < cf + na; ++cc) {
                            int a0, a1;
                            gists_of(cc, row, a0, a1);
                            n += min(p.K, max(0, a1 - a0));
                        }
                        merge_select<PG>(p, cx.base, row, n, j == 0);
                    } else {
                        load_selection(p, cx.base, row);
                    }
                    if (p.hier) hier_children_table(p, cx.base, row, 0);
                    else build_table<PG>(p, cx.base, row, t0, ntl);
                }
                for (int lt = 0; lt < ntl; ++lt) {
                    // leading rows that are whole runs of consecutive source rows
                    int tma_rows = 0, h = p.C;
                    const bool children = p.hier && rd < p.levels - 1;
                    const int cl = children ? p.levels - 1 - rd : 0;   // the children's level
                    if (children) {
                        h = p.grp[cl - 1];
                        tma_rows = p.tma_children ? min(TILE, lvl_k(p, cl + 1) * h) : 0;
                    } else if (p.tma_raw) {
                        // rows of the selected chunks in this tile (the hierarchy's raw
                        // round keeps its one tile at table index 0)
                        const int kc = (p.hier ? p.K1 : p.K) * p.C;
                        const int tile = p.hier ? lt : t0 + lt;
                        tma_rows = max(0, min(TILE, kc - tile * TILE));
                    }
                    gather_tile<PG>(p, cx.base, cx.bars, lt, gseq + 2 * lt, row, tma_rows, h, children, gseq0, cl);
                }
                gseq += 2 * ntl;
                ++runs;
            }
        }
    }

    // ---------------------------------------------------------- tickets --
    // every partial of this CTA is out: count each on its row's ticket (each
    // counting thread's fence is cumulative over the partials the barrier
    // made visible to it)
    __syncthreads();
    {
        const int nA = row_last - row_first + 1;
        const int nI = c < p.items ? (p.items - 1 - c) / p.grid + 1 : 0;
        if (threadIdx.x < nA + nI) __threadfence();
        for (int q = threadIdx.x; q < nA + nI; q += NTHR) {
            const int row = q < nA ? row_first + q : (c + (q - nA) * p.grid) / p.cb;
            atomicAdd(p.cnt + row, 1u);
        }
    }
    // the first unfold item's CTA of a row merges it once every partial is counted
    const int nb = p.hier ? rounds : (p.nbt > 0 ? p.cb : 0);
    for (int it = c; it < p.items; it += p.grid) {
        if (it % p.cb != 0) continue;
        const int row = it / p.cb;
        int cf;
        const int na = row_ctas(row, cf);
        wait_count<NTHR, 0>(p, p.cnt + row, (uint32_t)(na + p.cb), threadIdx.x == 0);
        merge_row<G>(p, cx.base, row, na, nb);
        __syncthreads();
    }
    tc::fence_before();
    __syncthreads();
    if (cx.warp == 5) {
        tc::fence_after();
        tc::tmem_dealloc(cx.tmem, (uint32_t)p.tmem_cols);
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

// 3-D bf16 map over [rows][len][d = 128], box {64, box_rows, 1}, 128-byte
// swizzle: a box that runs past `len` is zero-filled instead of reading the
// next (batch, kv-head) row's entries.  An operand the call never reads gets a
// zeroed map.
// The last few encoded maps are kept per host thread (a decode step encodes
// up to six, and callers reuse the same buffers call after call).
struct MapCacheEntry {
    const void* base;
    uint64_t rows, len;
    uint32_t box_rows;
    bool valid;
    CUtensorMap map;
};
static bool map3d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t len, uint32_t box_rows = TILE) {
    if (rows == 0 || len == 0 || base == nullptr) {
        std::memset(m, 0, sizeof(*m));
        return true;
    }
    constexpr int kMapCache = 32;
    thread_local MapCacheEntry cache[kMapCache];
    thread_local int next = 0;
    for (int i = 0; i < kMapCache; ++i) {
        const MapCacheEntry& c = cache[i];
        if (c.valid && c.base == base && c.rows == rows && c.len == len && c.box_rows == box_rows) {
            *m = c.map;
            return true;
        }
    }
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {D, len, rows};
    cuuint64_t strides[2] = {D * 2, len * D * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    MapCacheEntry& c = cache[next];
    next = (next + 1) % kMapCache;
    c.base = base;
    c.rows = rows;
    c.len = len;
    c.box_rows = box_rows;
    c.map = *m;
    c.valid = true;
    return true;
}

// Runs of h consecutive source rows are gathered by TMA when each run starts
// on a 1 KiB boundary of the swizzled tile (h a multiple of 8) and runs never
// straddle tiles (h divides 128).
static bool chunk_runs(int h) { return h >= 8 && h % 8 == 0 && TILE % h == 0; }

// The CTAs of one launch wait on one another (a row's unfold item waits for
// the key stretches of the CTAs that met the row), so all of them must be
// resident at once: the launch is refused on a device that cannot hold `grid`.
template <int G, bool PG>
static cudaError_t launch_g(const Params& p, int grid, cudaStream_t st) {
    static int resident = -1;
    if (resident < 0) {
        cudaError_t e = cudaFuncSetAttribute(fused_decode_kernel<G, PG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 0, per_sm = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused_decode_kernel<G, PG>, NTHR, SMEM_BYTES)) !=
            cudaSuccess)
            return e;
        resident = sms * per_sm;
    }
    if (grid > resident) return cudaErrorCooperativeLaunchTooLarge;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTHR);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fused_decode_kernel<G, PG>, p);
}

static cudaError_t launch(const Params& p, int G, int grid, cudaStream_t st) {
    if (p.table != nullptr || p.nch != nullptr) {
        switch (G) {
            case 1: return launch_g<1, true>(p, grid, st);
            case 2: return launch_g<2, true>(p, grid, st);
            case 4: return launch_g<4, true>(p, grid, st);
            default: return launch_g<8, true>(p, grid, st);
        }
    }
    switch (G) {
        case 1: return launch_g<1, false>(p, grid, st);
        case 2: return launch_g<2, false>(p, grid, st);
        case 4: return launch_g<4, false>(p, grid, st);
        default: return launch_g<8, false>(p, grid, st);
    }
}

}  // namespace fused

cudaError_t set_cross_cta_wait_limit(uint64_t ns) {
    const unsigned long long v = ns ? (unsigned long long)ns : (unsigned long long)kWaitLimitNs;
    return cudaMemcpyToSymbol(fused::g_cross_wait_ns, &v, sizeof(v));
}

bool fused_supported(const gsa_decode_desc& d) {
    // gathered rows are addressed by a 32-bit row number; the selection lives in shared memory
    const long long raw_rows = (long long)d.batch * d.n_kv_heads * d.n_chunks * d.chunk;
    // units are counted in 32 bits
    const long long units = (long long)d.batch * d.n_kv_heads * ((d.n_chunks + 127) / 128 + (d.tail_len + 127) / 128);
    if (!(d.dtype == GSA_BF16 && d.head_dim == 128 && d.top_k <= kSelCap && raw_rows < INT32_MAX - 2 &&
          units < (1LL << 30) && d.n_q_heads % d.n_kv_heads == 0))
        return false;
    // the kept logits and maxima of every CTA's range fit tensor memory
    return make_fused_plan(d).tmem_cols <= 512;
}

// Grid and partial slots once the rows' unfold items (cb per row) are known:
// every unfold item and every unit has a CTA (at most one per SM); the
// phase-A slots of a row are the CTAs whose range meets it.
static void place_ctas(FusedPlan& f, int nb_slots) {
    f.items = f.rows * f.cb;
    f.grid = std::min(kFusedCtas, std::max(f.T, f.items));
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
    f.slot_stride = maxs + nb_slots;
    // TMEM: S and O^T (64 columns), then per CTA G columns for each attended
    // unit and each attended segment of its range (its rows, few per CTA)
    int need = 64;
    for (int c = 0; c < f.grid && f.T > 0; ++c) {
        const long long u0 = (long long)c * f.T / f.grid, u1 = (long long)(c + 1) * f.T / f.grid;
        if (u1 <= u0) continue;
        long long units = 0, segs = 0;
        for (long long row = u0 / f.upr; row <= (u1 - 1) / f.upr; ++row) {
            // the row's attended units: all of them, or its tail tiles
            const long long a0 = row * f.upr + (f.attn_gists ? 0 : f.tg), a1 = (row + 1) * f.upr;
            const long long n = std::max(0LL, std::min(a1, u1) - std::max(a0, u0));
            units += n;
            segs += n > 0 ? 1 : 0;
        }
        need = (int)std::max<long long>(need, 64 + (units + segs) * f.G);
    }
    f.tmem_cols = need <= 64 ? 64 : need <= 128 ? 128 : need <= 256 ? 256 : need <= 512 ? 512 : 1024;
}

// Workspace: tickets and key counters [2][rows], scores, candidates, idx,
// partials, (m, l) (and the hierarchy's lower-level selections).
static void layout_ws(FusedPlan& f, size_t N, size_t top_k, size_t k1) {
    const size_t rows = (size_t)f.rows;
    size_t o = round256(kWsCntOffset + 2 * rows * 4);
    f.off_scores = o;
    o = round256(o + rows * N * 4);
    f.off_cand_key = o;
    o = round256(o + rows * N * 4);
    f.off_cand_idx = o;
    o = round256(o + rows * N * 4);
    f.off_idx = o;
    o = round256(o + rows * top_k * 4);
    f.off_part = o;
    o = round256(o + rows * (size_t)f.slot_stride * f.G * 128 * 4);
    f.off_ml = o;
    o = round256(o + rows * (size_t)f.slot_stride * f.G * 4 * 4);
    f.off_idx1 = o;
    o = round256(o + rows * k1 * 4);
    f.total = o;
}

static FusedPlan build_fused_plan(const gsa_decode_desc& d, bool given);

// Plans are a pure function of the descriptor; the last few are kept per host
// thread (one decode call asks for the plan several times).
FusedPlan make_fused_plan(const gsa_decode_desc& d, bool given) {
    struct Entry {
        gsa_decode_desc d;
        bool given, valid;
        FusedPlan f;
    };
    constexpr int kPlanCache = 8;
    thread_local Entry cache[kPlanCache];
    thread_local int next = 0;
    for (int i = 0; i < kPlanCache; ++i)
        if (cache[i].valid && cache[i].given == given && std::memcmp(&cache[i].d, &d, sizeof(d)) == 0)
            return cache[i].f;
    Entry& e = cache[next];
    next = (next + 1) % kPlanCache;
    e.d = d;
    e.given = given;
    e.f = build_fused_plan(d, given);
    e.valid = true;
    return e.f;
}

static FusedPlan build_fused_plan(const gsa_decode_desc& d, bool given) {
    FusedPlan f{};
    const bool pairs = d.mode == GSA_SELECTED_PAIRS;
    // gists attended by the stream: all of them, or all but the given
    // selection (UNSELECTED_GISTS, masked in the key stretch); SELECTED_PAIRS
    // gathers its gists with the raw rows and SR_ONLY attends none
    f.attn_gists = (d.mode == GSA_ALL_GISTS || d.mode == GSA_UNSELECTED_GISTS) ? 1 : 0;
    f.rows = d.batch * d.n_kv_heads;
    f.G = d.n_q_heads / d.n_kv_heads;
    // with a given selection in SELECTED_PAIRS mode no gist is scored or attended
    f.tg = (given && !f.attn_gists) ? 0 : (d.n_chunks + 127) / 128;
    f.tt = (d.tail_len + 127) / 128;
    f.upr = f.tg + f.tt;
    f.T = f.rows * f.upr;
    // small selections are taken straight from the scores; larger ones from
    // per-CTA candidates the key stretch leaves
    f.sel_direct = (d.top_k <= 32 && d.n_chunks <= 32 * fused::NU) ? 1 : 0;
    // unfold: the row's gathered rows packed into 128-row tiles, spread over
    // as many CTAs per row as fill the GPU (at most kMaxTpc tiles each)
    f.nrows_g = d.top_k * d.chunk + (pairs ? d.top_k : 0);
    f.nbt = (f.nrows_g + 127) / 128;
    if (f.nbt == 0) {
        f.tpc = 0;
        f.cb = 1;   // the row's ticket is still taken
    } else {
        const int cpr = std::max(1, kFusedCtas / f.rows);
        f.tpc = std::min(kMaxTpc, (f.nbt + std::min(cpr, f.nbt) - 1) / std::min(cpr, f.nbt));
        f.cb = (f.nbt + f.tpc - 1) / f.tpc;
    }
    place_ctas(f, f.cb);
    layout_ws(f, (size_t)d.n_chunks, (size_t)d.top_k, 0);
    return f;
}

static void fill_common(fused::Params& p, const FusedPlan& f, const gsa_decode_desc& d, uint8_t* w) {
    p.err = reinterpret_cast<uint32_t*>(w + kWsErrOffset);
    p.cnt = reinterpret_cast<uint32_t*>(w + kWsCntOffset);
    p.kdone = p.cnt + f.rows;
    p.cand_key = reinterpret_cast<uint32_t*>(w + f.off_cand_key);
    p.cand_idx = reinterpret_cast<int32_t*>(w + f.off_cand_idx);
    p.part = reinterpret_cast<float*>(w + f.off_part);
    p.ml = reinterpret_cast<float*>(w + f.off_ml);
    p.rows = f.rows;
    p.Hkv = d.n_kv_heads;
    p.G = f.G;
    p.C = d.chunk;
    p.W = d.tail_len;
    p.tg = f.tg;
    p.upr = f.upr;
    p.T = f.T;
    p.grid = f.grid;
    p.items = f.items;
    p.slot_stride = f.slot_stride;
    p.maxs = f.maxs;
    p.nbt = f.nbt;
    p.tpc = f.tpc;
    p.cb = f.cb;
    p.sel_direct = f.sel_direct;
    p.tmem_cols = f.tmem_cols;
    const double scale = d.scale > 0 ? (double)d.scale : 1.0 / std::sqrt(128.0);
    p.c2 = (float)(scale * 1.4426950408889634);
}

gsa_status fused_launch(const gsa_decode_desc& d, const FusedPlan& f, const void* q, const void* kg, const void* vg,
                        const void* kr, const void* vr, const void* kt, const void* vt, const int32_t* idx_given,
                        int32_t* idx_out, float* scores_out, void* out, float* lse, void* ws, cudaStream_t st,
                        const Paging* pg) {
    using namespace fused;
    if (f.grid <= 0) return GSA_ERR_ARG;
    Params p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t rows = (uint64_t)f.rows, N = (uint64_t)d.n_chunks;
    bool ok = map3d(&p.tm_kg, kg, rows, N) && map3d(&p.tm_vg, f.attn_gists ? vg : nullptr, rows, N) &&
              map3d(&p.tm_kt, kt, rows, (uint64_t)d.tail_len) && map3d(&p.tm_vt, vt, rows, (uint64_t)d.tail_len);
    p.tma_raw = chunk_runs(d.chunk) && f.nbt > 0 ? 1 : 0;
    // the raw cache: [rows][N c][d] dense; [n_pages Hkv][c][d] (pages as rows) paged
    const uint64_t mrows = pg && pg->table ? (uint64_t)pg->n_pages * (uint64_t)d.n_kv_heads : rows;
    const uint64_t mlen = pg && pg->table ? (uint64_t)d.chunk : N * (uint64_t)d.chunk;
    if (p.tma_raw)
        ok = ok && map3d(&p.tm_kr, kr, mrows, mlen, (uint32_t)d.chunk) &&
             map3d(&p.tm_vr, vr, mrows, mlen, (uint32_t)d.chunk);
    if (!ok) return GSA_ERR_CUDA;
    uint8_t* w = static_cast<uint8_t*>(ws);
    fill_common(p, f, d, w);
    p.q = static_cast<const uint16_t*>(q);
    p.kr = static_cast<const uint8_t*>(kr);
    p.vr = static_cast<const uint8_t*>(vr);
    p.kgp = static_cast<const uint8_t*>(kg);
    p.vgp = static_cast<const uint8_t*>(vg);
    p.out = static_cast<uint16_t*>(out);
    p.lse = lse;
    p.scores = scores_out ? scores_out : reinterpret_cast<float*>(w + f.off_scores);
    p.idx = idx_given ? const_cast<int32_t*>(idx_given) : (idx_out ? idx_out : reinterpret_cast<int32_t*>(w + f.off_idx));
    p.N = d.n_chunks;
    p.NA = d.n_chunks;
    p.K = d.top_k;
    p.mode = d.mode;
    p.nrows_g = f.nrows_g;
    p.do_score = idx_given ? 0 : 1;
    p.do_topk = idx_given ? 0 : 1;
    p.do_attn_gists = f.attn_gists;
    // a given selection in UNSELECTED_GISTS mode: its gists leave the context
    p.mask_sel = (idx_given != nullptr && d.mode == GSA_UNSELECTED_GISTS) ? 1 : 0;
    if (pg != nullptr) {
        p.table = pg->table;
        p.nch = pg->nch;
        p.n_pages = pg->n_pages;
    }
    return launch(p, f.G, f.grid, st) == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

// --------------------------------------------------------- hierarchy ----
bool fused_hier_supported(const gsa_hier_desc& h) {
    const gsa_decode_desc& d = h.l1;
    const long long rows = (long long)d.batch * d.n_kv_heads;
    const long long units = rows * ((h.n_l2 + 127) / 128 + (d.tail_len + 127) / 128);
    if (!(d.dtype == GSA_BF16 && d.head_dim == 128 && (long long)h.top_k2 * h.group <= 128 &&
          (long long)d.top_k * d.chunk <= 128 && rows * d.n_chunks * d.chunk < INT32_MAX - 2 &&
          rows * d.n_chunks < INT32_MAX - 2 && units < (1LL << 30) && d.n_q_heads % d.n_kv_heads == 0))
        return false;
    return make_fused_hier_plan(h).tmem_cols <= 512;
}

FusedPlan make_fused_hier_plan(const gsa_hier_desc& h) {
    // the key and value stretches and the level-2 selection are the flat
    // step over the level-2 gists
    gsa_decode_desc l2 = h.l1;
    l2.n_chunks = h.n_l2;
    l2.top_k = h.top_k2;
    l2.mode = GSA_ALL_GISTS;
    FusedPlan f = make_fused_plan(l2);
    // unfold: one item per row, two partial slots (children tile, raw tile)
    f.nbt = 2;
    f.tpc = 2;
    f.cb = 1;
    place_ctas(f, 2);
    layout_ws(f, (size_t)h.n_l2, (size_t)h.top_k2, (size_t)h.l1.top_k);
    return f;
}

gsa_status fused_hier_launch(const gsa_hier_desc& h, const FusedPlan& f, const void* q, const void* k_g2,
                             const void* v_g2, const void* k_g1, const void* v_g1, const void* kr, const void* vr,
                             const void* kt, const void* vt, int32_t* idx2_out, int32_t* idx1_out, void* out,
                             void* ws, cudaStream_t st) {
    using namespace fused;
    const gsa_decode_desc& d = h.l1;
    if (f.grid <= 0) return GSA_ERR_ARG;
    Params p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t rows = (uint64_t)f.rows;
    bool ok = map3d(&p.tm_kg, k_g2, rows, (uint64_t)h.n_l2) && map3d(&p.tm_vg, v_g2, rows, (uint64_t)h.n_l2) &&
              map3d(&p.tm_kt, kt, rows, (uint64_t)d.tail_len) && map3d(&p.tm_vt, vt, rows, (uint64_t)d.tail_len);
    p.tma_raw = chunk_runs(d.chunk) && d.top_k > 0 ? 1 : 0;
    p.tma_children = chunk_runs(h.group) ? 1 : 0;
    const uint64_t n1 = (uint64_t)d.n_chunks;
    if (p.tma_raw)
        ok = ok && map3d(&p.tm_kr, kr, rows, n1 * (uint64_t)d.chunk, (uint32_t)d.chunk) &&
             map3d(&p.tm_vr, vr, rows, n1 * (uint64_t)d.chunk, (uint32_t)d.chunk);
    if (p.tma_children)
        ok = ok && map3d(&p.tm_kc, k_g1, rows, n1, (uint32_t)h.group) && map3d(&p.tm_vc, v_g1, rows, n1, (uint32_t)h.group);
    if (!ok) return GSA_ERR_CUDA;
    uint8_t* w = static_cast<uint8_t*>(ws);
    fill_common(p, f, d, w);
    p.q = static_cast<const uint16_t*>(q);
    p.kr = static_cast<const uint8_t*>(kr);
    p.vr = static_cast<const uint8_t*>(vr);
    p.kgp = static_cast<const uint8_t*>(k_g1);   // gathered "gist" rows are the level-1 gists
    p.vgp = static_cast<const uint8_t*>(v_g1);
    p.out = static_cast<uint16_t*>(out);
    p.lse = nullptr;
    p.scores = reinterpret_cast<float*>(w + f.off_scores);
    p.idx = idx2_out ? idx2_out : reinterpret_cast<int32_t*>(w + f.off_idx);
    p.idx1 = idx1_out ? idx1_out : reinterpret_cast<int32_t*>(w + f.off_idx1);
    p.N = h.n_l2;
    p.NA = h.n_l2;
    p.K = h.top_k2;
    p.mode = GSA_ALL_GISTS;
    p.nrows_g = 0;
    p.do_score = 1;
    p.do_topk = 1;
    p.do_attn_gists = 1;
    p.hier = 1;
    p.group = h.group;
    p.N1 = d.n_chunks;
    p.K1 = d.top_k;
    p.levels = 2;
    p.grp[0] = h.group;
    return launch(p, f.G, f.grid, st) == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

// --------------------------------------------------- hierarchy, any depth ----
constexpr int kFusedMaxLevels = 4;   // the middle levels' maps in Params (levels 2 .. L-1)

bool fused_levels_supported(const gsa_levels_desc& h) {
    using namespace fused;
    const gsa_decode_desc& d = h.l1;
    const int L = h.levels;
    if (L < 2 || L > kFusedMaxLevels) return false;
    if (L > 2 && h.l1.top_k < 1) return false;   // (no raw round: the CUDA-core passes)
    int n[GSA_MAX_LEVELS];
    level_counts(h, n);
    const long long rows = (long long)d.batch * d.n_kv_heads;
    const long long units = rows * ((n[L - 1] + 127) / 128 + (d.tail_len + 127) / 128);
    if (!(d.dtype == GSA_BF16 && d.head_dim == 128 && (long long)d.top_k * d.chunk <= 128 &&
          rows * d.n_chunks * d.chunk < INT32_MAX - 2 && rows * d.n_chunks < INT32_MAX - 2 && units < (1LL << 30) &&
          d.n_q_heads % d.n_kv_heads == 0))
        return false;
    // every level's children of the selection above: one tile, gathered in whole
    // groups by TMA (the two-level step also takes other groups, by cp.async)
    for (int l = 1; l < L; ++l) {
        const int g = h.group[l - 1];
        if ((long long)level_k(h, l) * g > 128 || (L > 2 && !chunk_runs(g))) return false;
    }
    return make_fused_levels_plan(h).tmem_cols <= 512;
}

FusedPlan make_fused_levels_plan(const gsa_levels_desc& h) {
    const int L = h.levels;
    int n[GSA_MAX_LEVELS];
    level_counts(h, n);
    // the key and value stretches and the top selection are the flat step
    // over the top level's gists
    gsa_decode_desc top = h.l1;
    top.n_chunks = n[L - 1];
    top.top_k = level_k(h, L - 1);
    top.mode = GSA_ALL_GISTS;
    FusedPlan f = make_fused_plan(top);
    // unfold: one item per row, a partial slot per round (a children tile per
    // level below the top, the raw tile)
    f.nbt = L;
    f.tpc = L;
    f.cb = 1;
    place_ctas(f, L);
    // the lower levels' selections when the caller passes none: level 1, then 2 .. L-1
    size_t lower = 0;
    for (int l = 0; l < L - 1; ++l) lower += (size_t)level_k(h, l);
    layout_ws(f, (size_t)n[L - 1], (size_t)top.top_k, lower);
    return f;
}

gsa_status fused_levels_launch(const gsa_levels_desc& h, const FusedPlan& f, const void* q, const void* const* kg,
                               const void* const* vg, const void* kr, const void* vr, const void* kt, const void* vt,
                               int32_t* const* idx_out, void* out, void* ws, cudaStream_t st) {
    using namespace fused;
    const gsa_decode_desc& d = h.l1;
    const int L = h.levels;
    if (f.grid <= 0 || L > kFusedMaxLevels) return GSA_ERR_ARG;
    int n[GSA_MAX_LEVELS];
    level_counts(h, n);
    Params p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t rows = (uint64_t)f.rows;
    bool ok = map3d(&p.tm_kg, kg[L - 1], rows, (uint64_t)n[L - 1]) &&
              map3d(&p.tm_vg, vg[L - 1], rows, (uint64_t)n[L - 1]) &&
              map3d(&p.tm_kt, kt, rows, (uint64_t)d.tail_len) && map3d(&p.tm_vt, vt, rows, (uint64_t)d.tail_len);
    p.tma_raw = chunk_runs(d.chunk) && d.top_k > 0 ? 1 : 0;
    p.tma_children = chunk_runs(h.group[0]) ? 1 : 0;   // (every group, from three levels on)
    const uint64_t n1 = (uint64_t)d.n_chunks;
    if (p.tma_raw)
        ok = ok && map3d(&p.tm_kr, kr, rows, n1 * (uint64_t)d.chunk, (uint32_t)d.chunk) &&
             map3d(&p.tm_vr, vr, rows, n1 * (uint64_t)d.chunk, (uint32_t)d.chunk);
    if (p.tma_children)
        ok = ok && map3d(&p.tm_kc, kg[0], rows, n1, (uint32_t)h.group[0]) &&
             map3d(&p.tm_vc, vg[0], rows, n1, (uint32_t)h.group[0]);
    for (int l = 2; l < L; ++l)
        ok = ok && map3d(&p.tm_kcm[l - 2], kg[l - 1], rows, (uint64_t)n[l - 1], (uint32_t)h.group[l - 1]) &&
             map3d(&p.tm_vcm[l - 2], vg[l - 1], rows, (uint64_t)n[l - 1], (uint32_t)h.group[l - 1]);
    if (!ok) return GSA_ERR_CUDA;
    uint8_t* w = static_cast<uint8_t*>(ws);
    fill_common(p, f, d, w);
    p.q = static_cast<const uint16_t*>(q);
    p.kr = static_cast<const uint8_t*>(kr);
    p.vr = static_cast<const uint8_t*>(vr);
    p.kgp = static_cast<const uint8_t*>(kg[0]);   // gathered "gist" rows are level-1 gists (two levels, cp.async)
    p.vgp = static_cast<const uint8_t*>(vg[0]);
    p.out = static_cast<uint16_t*>(out);
    p.lse = nullptr;
    p.scores = reinterpret_cast<float*>(w + f.off_scores);
    // selections: the caller's, else workspace (level 1, then 2 .. L-1, after the top level's)
    auto sel_of = [&](int l, size_t& off) -> int32_t* {
        int32_t* given = idx_out ? idx_out[l - 1] : nullptr;
        int32_t* mine = reinterpret_cast<int32_t*>(w + f.off_idx1 + off);
        off += (size_t)f.rows * level_k(h, l - 1) * 4;
        return given ? given : mine;
    };
    size_t off = 0;
    p.idx1 = sel_of(1, off);
    for (int l = 2; l < L; ++l) p.midIdx[l - 2] = sel_of(l, off);
    p.idx = (idx_out && idx_out[L - 1]) ? idx_out[L - 1] : reinterpret_cast<int32_t*>(w + f.off_idx);
    p.N = n[L - 1];
    p.NA = n[L - 1];
    p.K = level_k(h, L - 1);
    p.mode = GSA_ALL_GISTS;
    p.nrows_g = 0;
    p.do_score = 1;
    p.do_topk = 1;
    p.do_attn_gists = 1;
    p.hier = 1;
    p.group = h.group[0];
    p.N1 = d.n_chunks;
    p.K1 = d.top_k;
    p.levels = L;
    for (int l = 1; l < L; ++l) p.grp[l - 1] = h.group[l - 1];
    for (int l = 2; l < L; ++l) {
        p.midN[l - 2] = n[l - 1];
        p.midK[l - 2] = level_k(h, l - 1);
    }
    return launch(p, f.G, f.grid, st) == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

}  // namespace gsa
