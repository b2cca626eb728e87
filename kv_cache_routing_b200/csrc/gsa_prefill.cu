// Gist-causal prefill on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Mask (gist.science explainer EN, section 2 "Interleaved Gist Tokens";
// Taki-lab slides page 7 "Gist token", page 9): position p belongs to chunk
// p / (c+1) and is a gist iff p % (c+1) == c; query p attends key t <= p iff
// t == p, or t is a gist of an earlier chunk, or t is a raw token of p's own
// chunk.
//
// Tiling.  A query tile is QC = floor(128 / (c+1)) whole chunks in their
// interleaved order (119 rows for c = 16; rows past the tile are idle).  Its
// keys are
//   * the gists of earlier chunks, read as a compact list straight from the
//     interleaved K/V through a strided tensor map (row stride (c+1)*d), in
//     tiles of 128 gists; only the tile holding the staircase g < chunk(p)
//     needs a mask;
//   * one local tile: the 128 positions starting at the query tile, masked
//     to "same chunk and t <= p" (this covers every raw-token and self key).
// So the work is ~ (earlier gists + 128) per 119 queries instead of the full
// causal triangle.
//
// Per CTA: one query tile of TWO query heads of the same KV head (grouped-
// query attention), which see the same keys under the same mask, so every
// K/V tile is loaded once for both.  Warps 0-3 run the online softmax of head
// A, warps 4-7 that of head B (thread = query row = TMEM lane), warp 8 issues
// the TMA loads and warp 9 the MMAs from one thread.  TMEM (512 columns): S_A
// [0,128), S_B [128,256), O_A [256,384), O_B [384,512); each head's P (bf16,
// two per column) overwrites the first 64 columns of its S once read and is
// the A operand of its P.V product straight from TMEM.  The tensor core
// alternates between the heads (S_A, S_B, P.V_A, S_A', P.V_B, S_B', ...), so
// one head's softmax overlaps the other head's products.  K/V tiles are double
// buffered; O is rescaled lazily (only when a row's running maximum grows by
// more than 2^8).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "gsa_plan.h"
#include "gsa_tc.cuh"

namespace gsa {

constexpr int PF_THREADS = 384;   // three warpgroups: softmax A, softmax B, loads + MMA
// Register split (setmaxnreg): launched at 168 a thread (384 x 168 = 64,512),
// the load/MMA warpgroup gives back down to 72 and the two softmax warpgroups
// grow to 216: 2 x 128 x 216 + 128 x 72 = 64,512, the same total.
constexpr uint32_t PF_REG_SOFTMAX = 216, PF_REG_OTHER = 72;
static_assert(2 * 128 * PF_REG_SOFTMAX + 128 * PF_REG_OTHER == PF_THREADS * 168, "register split must add up");
constexpr int PF_D = 128;
constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
constexpr uint32_t IDESC_PV = tc::idesc_bf16(128, 128, 0, 1);  // P (TMEM, K-major) x V (MN-major)
constexpr float kRescaleLog2 = 8.f;

// Error word of the prefill's bounded waits (the prefill takes no workspace).
__device__ uint32_t g_prefill_err;

struct PrefillParams {
    CUtensorMap tm_q;    // [B*Hq][P][d]
    CUtensorMap tm_k;    // [B*Hkv][P][d]
    CUtensorMap tm_v;
    CUtensorMap tm_kg;   // gist rows of k: [B*Hkv][N][d], row stride (c+1)*d
    CUtensorMap tm_vg;
    uint16_t* out;       // [B*Hq][P][d] bf16
    float* lse;          // [B*Hq][P] or null
    int B, Hq, Hkv, G, NPAIR, N, C, P, QC, n_qt;
    float c2;            // scale * log2(e)
};

// 2^x on the special-function unit (ex2.approx.ftz: -inf -> +0), a
// three-input maximum, and packed two-wide fp32 arithmetic (sm_100).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unf2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t SM_Q = 0;                  // 2 heads x 32 KiB
constexpr uint32_t SM_KV = 65536;             // 2 stages x (K 32 KiB + V 32 KiB)
constexpr uint32_t SM_BAR = SM_KV + 2 * 65536; // barriers and the TMEM address
constexpr uint32_t PF_SMEM = SM_BAR + 256 + 1024;

struct PfBars {
    uint64_t q_full, q_free, kv_full[2], kv_empty[2], s_full[2], p_full[2], o_done[2], o_free[2];
    uint32_t tmem;
};

// A work item: one query tile of one head pair.  Items are numbered heaviest
// query tiles first (most earlier gists), then (batch, kv head, head pair).
struct PfItem {
    int bkv, hkv, bhA, j0, p0, n_gt, n_kv;
    bool hasB;
};

__device__ __forceinline__ PfItem pf_item(const PrefillParams& p, int item) {
    PfItem x;
    const int nw = p.B * p.Hkv * p.NPAIR;
    const int wi = item % nw;
    const int t = p.n_qt - 1 - item / nw;
    const int hp = wi % p.NPAIR;
    x.bkv = wi / p.NPAIR;   // b * Hkv + kv head
    const int b = x.bkv / p.Hkv;
    x.hkv = x.bkv % p.Hkv;
    const int hA = x.hkv * p.G + 2 * hp;
    x.hasB = 2 * hp + 1 < p.G;
    x.bhA = b * p.Hq + hA;
    x.j0 = t * p.QC;
    x.p0 = x.j0 * (p.C + 1);
    const int j_last = min(x.j0 + p.QC, p.N) - 1;   // last chunk of the tile
    x.n_gt = (j_last + 127) / 128;                  // tiles of earlier gists
    x.n_kv = x.n_gt + 1;
    return x;
}

// Persistent: CTA c takes items c, c + grid, ...  Every barrier's phases run
// on across items; the K/V ring, the S / P / O hand-offs and the softmax state
// are as for one item, and two more barriers join consecutive items: q_free
// (the item's last S products are done with Q, so the next Q may load) and
// o_free[h] (the epilogue has read head h's O, so the next item's first P.V
// may overwrite it).  The next item's loads and first S products thus run
// under the current item's epilogue.
__global__ void __launch_bounds__(PF_THREADS, 1) gist_prefill_kernel(const __grid_constant__ PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(base);
    PfBars& bars = *reinterpret_cast<PfBars*>(base + SM_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = p.n_qt * p.B * p.Hkv * p.NPAIR;

    if (threadIdx.x == 0) {
        mbar_init(&bars.q_full, 1);
        mbar_init(&bars.q_free, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.kv_full[i], 1);
            mbar_init(&bars.kv_empty[i], 1);
            mbar_init(&bars.s_full[i], 1);
            mbar_init(&bars.p_full[i], 128);
            mbar_init(&bars.o_done[i], 1);
            mbar_init(&bars.o_free[i], 128);
        }
        fence_mbar_init();
    }
    if (warp == 9) {
        tc::tmem_alloc(&bars.tmem, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars.tmem;
    uint32_t* err = &g_prefill_err;   // waits below are bounded; a timeout abandons the item

    if (warp >= 8) {
    // --------------------------------- load / MMA warpgroup (warps 8-11) ----
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(PF_REG_OTHER));
    if (warp == 8) {
        if (lane == 0) {
            // --------------------------------------------------- TMA loads --
            int g = 0, it = 0;   // K/V tiles and items so far
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++it) {
                const PfItem x = pf_item(p, item);
                // the previous item's S products are done with the Q buffer
                if (it > 0 && !mbar_wait(&bars.q_free, (it - 1) & 1, err)) break;
                mbar_arrive_expect_tx(&bars.q_full, x.hasB ? 65536 : 32768);
                tc::tma_load_3d(base + SM_Q, &p.tm_q, 0, x.p0, x.bhA, &bars.q_full);
                tc::tma_load_3d(base + SM_Q + 16384, &p.tm_q, 64, x.p0, x.bhA, &bars.q_full);
                if (x.hasB) {
                    tc::tma_load_3d(base + SM_Q + 32768, &p.tm_q, 0, x.p0, x.bhA + 1, &bars.q_full);
                    tc::tma_load_3d(base + SM_Q + 49152, &p.tm_q, 64, x.p0, x.bhA + 1, &bars.q_full);
                }
                for (int i = 0; i < x.n_kv; ++i, ++g) {
                    const int s = g & 1;
                    if (g >= 2 && !mbar_wait(&bars.kv_empty[s], ((g - 2) >> 1) & 1, err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* ks = base + SM_KV + s * 65536;
                    uint8_t* vs = ks + 32768;
                    mbar_arrive_expect_tx(&bars.kv_full[s], 65536);
                    const CUtensorMap* mk = i < x.n_gt ? &p.tm_kg : &p.tm_k;
                    const CUtensorMap* mv = i < x.n_gt ? &p.tm_vg : &p.tm_v;
                    const int y = i < x.n_gt ? i * 128 : x.p0;
                    tc::tma_load_3d(ks, mk, 0, y, x.bkv, &bars.kv_full[s]);
                    tc::tma_load_3d(ks + 16384, mk, 64, y, x.bkv, &bars.kv_full[s]);
                    tc::tma_load_3d(vs, mv, 0, y, x.bkv, &bars.kv_full[s]);
                    tc::tma_load_3d(vs + 16384, mv, 64, y, x.bkv, &bars.kv_full[s]);
                }
            }
        }
    } else if (warp == 9) {
        if (lane == 0) {
            // ----------------------------------------------------- MMA issue --
            // S_h = Q_h . K^T into TMEM columns 128 h; P_h . V into 256 + 128 h
            auto issue_s = [&](int h, int g) {
                const uint32_t ks = sbase + SM_KV + (g & 1) * 65536;
                const uint32_t qs = sbase + SM_Q + h * 32768;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    tc::mma_bf16(tmem + h * 128, tc::sdesc_sw128(qs + off, 16, 1024),
                                 tc::sdesc_sw128(ks + off, 16, 1024), IDESC_S, kk > 0);
                }
                tc::commit(&bars.s_full[h]);
            };
            auto issue_pv = [&](int h, int g, bool first) {
                const uint32_t vs = sbase + SM_KV + (g & 1) * 65536 + 32768;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16_ts(tmem + 256 + h * 128, tmem + h * 128 + kk * 8,
                                    tc::sdesc_sw128(vs + kk * 2048, 16384, 1024), IDESC_PV, (!first || kk > 0));
                tc::commit(&bars.o_done[h]);
            };
            int g = 0, it = 0;
            int pc0 = 0, pc1 = 0;   // P tiles per head so far (p_full phases)
            int itB = 0;            // items with a head B so far (o_free[1] phases; head A: every item)
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++it) {
                const PfItem x = pf_item(p, item);
                const int nh = x.hasB ? 2 : 1;
                ok = mbar_wait(&bars.q_full, it & 1, err) && mbar_wait(&bars.kv_full[g & 1], (g >> 1) & 1, err);
                tc::fence_after();
                if (!ok) break;
                issue_s(0, g);
                if (x.hasB) issue_s(1, g);
                if (x.n_kv == 1) tc::commit(&bars.q_free);   // the item's last S products are issued
                for (int i = 0; ok && i < x.n_kv; ++i) {
                    const bool more = i + 1 < x.n_kv;
                    for (int h = 0; ok && h < nh; ++h) {
                        // P_h of tile i (which also means S_h of tile i has been read)
                        const int pc = h == 0 ? pc0++ : pc1++;
                        ok = mbar_wait(&bars.p_full[h], pc & 1, err);
                        // the first P.V of an item overwrites O_h: the previous
                        // item's epilogue must have read it
                        const int ih = h == 0 ? it : itB;
                        if (ok && i == 0 && ih > 0) ok = mbar_wait(&bars.o_free[h], (ih - 1) & 1, err);
                        if (!ok) break;
                        tc::fence_after();
                        issue_pv(h, g + i, i == 0);
                        if (h == nh - 1) tc::commit(&bars.kv_empty[(g + i) & 1]);
                        if (more) {
                            if (h == 0) {
                                ok = mbar_wait(&bars.kv_full[(g + i + 1) & 1], ((g + i + 1) >> 1) & 1, err);
                                if (!ok) break;
                                tc::fence_after();
                            }
                            issue_s(h, g + i + 1);
                            if (i + 2 == x.n_kv && h == nh - 1) tc::commit(&bars.q_free);
                        }
                    }
                }
                g += x.n_kv;
                itB += x.hasB ? 1 : 0;
            }
        }
    }
    } else {
        // ------------------------------------------------ softmax warps ----
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(PF_REG_SOFTMAX));
        const int h = warp >> 2;                         // 0: head A, 1: head B
        const int r = threadIdx.x & 127;                 // query row = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t ts = tmem + h * 128 + lane_off, to = tmem + 256 + h * 128 + lane_off;
        int sc = 0;                                      // S tiles of this head so far
        for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
            const PfItem x = pf_item(p, item);
            if (h == 1 && !x.hasB) continue;             // (only with an odd group: the last pair is one head)
            const int qp = x.p0 + r;
            const bool valid = r < p.QC * (p.C + 1) && qp < p.P;
            const int jq = valid ? x.j0 + r / (p.C + 1) : -1;
            float m_run = -INFINITY, l_run = 0.f;
            bool ok = true;
            for (int i = 0; i < x.n_kv; ++i, ++sc) {
                if (!mbar_wait(&bars.s_full[h], sc & 1, err)) {
                    ok = false;
                    break;
                }
                tc::fence_after();
                // allowed key columns [lo, hi] of this row in this tile
                int lo, hi;
                if (i < x.n_gt) {
                    lo = 0;
                    hi = valid ? min(127, jq - i * 128 - 1) : -1;
                } else {
                    lo = valid ? jq * (p.C + 1) - x.p0 : 1;
                    hi = valid ? r : 0;
                }
                // the row's 128 scores in registers (all four loads in flight)
                uint32_t uu[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tc::ld32(ts + c * 32, uu[c]);
                tc::wait_ld();
                uint32_t* u = &uu[0][0];
                // the row maximum of the allowed columns; the scale is applied to
                // the maximum (it is positive); a warp whose rows all see the
                // whole tile takes the unmasked path
                const bool full = __all_sync(0xFFFFFFFFu, lo == 0 && hi >= 127);
                if (!full) {
#pragma unroll
                    for (int jj = 0; jj < 128; ++jj)
                        if (jj < lo || jj > hi) u[jj] = __float_as_uint(-INFINITY);
                }
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int jj = 0; jj < 128; jj += 8) {
                    m4[0] = max3(m4[0], __uint_as_float(u[jj]), __uint_as_float(u[jj + 1]));
                    m4[1] = max3(m4[1], __uint_as_float(u[jj + 2]), __uint_as_float(u[jj + 3]));
                    m4[2] = max3(m4[2], __uint_as_float(u[jj + 4]), __uint_as_float(u[jj + 5]));
                    m4[3] = max3(m4[3], __uint_as_float(u[jj + 6]), __uint_as_float(u[jj + 7]));
                }
                const float mt = max3(fmaxf(m4[0], m4[1]), m4[2], m4[3]) * p.c2;
                bool need = false;
                float m_new = m_run;
                if (mt > -INFINITY) {
                    if (m_run == -INFINITY) {
                        m_new = mt;
                    } else if (mt > m_run + kRescaleLog2) {
                        m_new = mt;
                        need = true;
                    }
                }
                const float alpha = need ? exp2f(m_run - m_new) : 1.f;
                if (__any_sync(0xFFFFFFFFu, need) && i > 0) {
                    // O holds P.V of tiles < i: wait for the last of them, then rescale
                    mbar_wait(&bars.o_done[h], (sc - 1) & 1, err);
                    tc::fence_after();
#pragma unroll 1
                    for (int c = 0; c < 8; ++c) {
                        uint32_t o[16];
                        tc::ld16(to + c * 16, o);
                        tc::wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) o[jj] = __float_as_uint(__uint_as_float(o[jj]) * alpha);
                        tc::st16(to + c * 16, o);
                    }
                }
                m_run = m_new;
                // P (bf16 pairs) over the first 64 columns of S (all of S is in
                // registers); the P.V of the previous tile finished before this S
                // was written.  x * c2 - m in pairs (fma.f32x2), 2^x on the SFU
                // (masked: -inf -> 0), pair sums (add.f32x2)
                // (a row with nothing allowed yet subtracts 0: its masked -inf stay -inf)
                const float ms = m_run == -INFINITY ? 0.f : m_run;
                const uint64_t c22 = f2(p.c2, p.c2), nm2 = f2(-ms, -ms);
                uint64_t acc2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int jj = c * 32 + 2 * e;
                        float xa, xb;
                        unf2(ffma2(f2(__uint_as_float(u[jj]), __uint_as_float(u[jj + 1])), c22, nm2), xa, xb);
                        const float a = ex2(xa), bb = ex2(xb);
                        acc2[e & 1] = fadd2(acc2[e & 1], f2(a, bb));
                        w[e] = tc::pack_bf16x2(a, bb);
                    }
                    tc::st16(ts + c * 16, w);
                }
                float sa, sb;
                unf2(fadd2(acc2[0], acc2[1]), sa, sb);
                const float sum = m_run == -INFINITY ? 0.f : sa + sb;
                l_run = l_run * alpha + sum;
                tc::wait_st();
                tc::fence_before();
                mbar_arrive(&bars.p_full[h]);
            }
            if (!ok) break;
            // -------------------------------------------------- epilogue ----
            // O of the item's last tile, all 128 columns into registers; then
            // O_h is released to the next item's first P.V
            mbar_wait(&bars.o_done[h], (sc - 1) & 1, err);
            tc::fence_after();
            uint32_t ov[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::ld32(to + c * 32, ov[c]);
            tc::wait_ld();
            tc::fence_before();
            mbar_arrive(&bars.o_free[h]);
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            const int bh = x.bhA + h;
            uint16_t* orow = p.out + ((size_t)bh * p.P + qp) * PF_D;
            if (valid) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint4 v;
                        v.x = tc::pack_bf16x2(__uint_as_float(ov[c][j]) * inv, __uint_as_float(ov[c][j + 1]) * inv);
                        v.y = tc::pack_bf16x2(__uint_as_float(ov[c][j + 2]) * inv, __uint_as_float(ov[c][j + 3]) * inv);
                        v.z = tc::pack_bf16x2(__uint_as_float(ov[c][j + 4]) * inv, __uint_as_float(ov[c][j + 5]) * inv);
                        v.w = tc::pack_bf16x2(__uint_as_float(ov[c][j + 6]) * inv, __uint_as_float(ov[c][j + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + c * 32 + j) = v;
                    }
                }
                if (p.lse != nullptr) p.lse[(size_t)bh * p.P + qp] = (m_run + log2f(l_run)) * 0.69314718055994531f;
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 9) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ============================================================ host side ====
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// 3-D bf16 map: dims {d, rows, slabs}, box {64, 128, 1}, 128-byte swizzle.
static bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t slabs, uint64_t row_stride_bytes,
                     uint64_t slab_stride_bytes) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {PF_D, rows, slabs};
    cuuint64_t strides[2] = {row_stride_bytes, slab_stride_bytes};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static gsa_status validate_prefill(const gsa_prefill_desc* d) {
    if (!d) return GSA_ERR_ARG;
    if (d->dtype != GSA_BF16) return GSA_ERR_DTYPE;
    if (d->batch < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1 || d->n_q_heads % d->n_kv_heads) return GSA_ERR_SHAPE;
    if (d->head_dim != PF_D) return GSA_ERR_SHAPE;
    if (d->n_chunks < 1 || d->chunk < 1) return GSA_ERR_ARG;
    if (d->chunk + 1 > 128) return GSA_ERR_SHAPE;   // a query tile holds at least one whole chunk
    const int64_t P = (int64_t)d->n_chunks * (d->chunk + 1);
    if (P > INT32_MAX / 2 || (int64_t)d->batch * d->n_q_heads > 65535 * 64) return GSA_ERR_SHAPE;
    return GSA_OK;
}

// Device address of the prefill's error word on the current device (read and
// cleared by gsa_device_error).
cudaError_t prefill_error_word(uint32_t** addr) {
    return cudaGetSymbolAddress(reinterpret_cast<void**>(addr), g_prefill_err);
}

}  // namespace gsa

using namespace gsa;

extern "C" gsa_status gsa_gist_prefill(const gsa_prefill_desc* desc, const void* q, const void* k, const void* v,
                                       void* out, float* lse, void* stream) {
    gsa_status st = validate_prefill(desc);
    if (st != GSA_OK) return st;
    if (!q || !k || !v || !out) return GSA_ERR_ARG;
    const void* all[] = {q, k, v, out};
    for (const void* x : all)
        if (!aligned16(x)) return GSA_ERR_ALIGN;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return GSA_ERR_ALIGN;
    const int B = desc->batch, Hq = desc->n_q_heads, Hkv = desc->n_kv_heads, N = desc->n_chunks, C = desc->chunk;
    const uint64_t P = (uint64_t)N * (C + 1);
    const uint64_t rowb = PF_D * 2;
    PrefillParams p;
    std::memset(&p, 0, sizeof(p));
    bool ok = make_map(&p.tm_q, q, P, (uint64_t)B * Hq, rowb, P * rowb) &&
              make_map(&p.tm_k, k, P, (uint64_t)B * Hkv, rowb, P * rowb) &&
              make_map(&p.tm_v, v, P, (uint64_t)B * Hkv, rowb, P * rowb) &&
              make_map(&p.tm_kg, static_cast<const uint8_t*>(k) + (size_t)C * rowb, N, (uint64_t)B * Hkv,
                       (C + 1) * rowb, P * rowb) &&
              make_map(&p.tm_vg, static_cast<const uint8_t*>(v) + (size_t)C * rowb, N, (uint64_t)B * Hkv,
                       (C + 1) * rowb, P * rowb);
    if (!ok) return GSA_ERR_CUDA;
    p.out = static_cast<uint16_t*>(out);
    p.lse = lse;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.NPAIR = (p.G + 1) / 2;
    p.N = N;
    p.C = C;
    p.P = (int)P;
    p.QC = 128 / (C + 1);
    p.n_qt = (N + p.QC - 1) / p.QC;
    const double scale = desc->scale > 0 ? (double)desc->scale : 1.0 / std::sqrt((double)PF_D);
    p.c2 = (float)(scale * 1.4426950408889634);
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(gist_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PF_SMEM) !=
            cudaSuccess)
            return GSA_ERR_CUDA;
        attr = true;
    }
    // persistent: one CTA per SM (the work split does not depend on the device beyond the grid)
    static int n_sm = 0;
    if (n_sm == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0)
            return GSA_ERR_CUDA;
    }
    const long long items = (long long)p.n_qt * (B * Hkv * p.NPAIR);
    const unsigned grid = (unsigned)std::min<long long>(items, n_sm);
    gist_prefill_kernel<<<grid, PF_THREADS, PF_SMEM, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}
