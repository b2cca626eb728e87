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
// Per CTA (one query tile of one head): warp 4 allocates TMEM, issues the
// TMA loads and the MMAs from one thread; warps 0-3 own one query row each
// (TMEM lane = row) and run the online softmax.  S = Q.K^T lands in TMEM
// columns [0,128), O accumulates in columns [128,256).  K/V tiles are double
// buffered, P (bf16, written by the softmax warps in the MMA's swizzled
// K-major layout) is double buffered, and O is rescaled lazily: only when a
// row's running maximum grows by more than 2^8.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "gsa_plan.h"
#include "gsa_tc.cuh"

namespace gsa {

constexpr int PF_THREADS = 160;
constexpr int PF_D = 128;
constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
constexpr uint32_t IDESC_PV = tc::idesc_bf16(128, 128, 0, 1);  // P (K-major) x V (MN-major)
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
    int BH, Hq, G, N, C, P, QC, n_qt;
    float c2;            // scale * log2(e)
};

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t SM_Q = 0;                  // 32 KiB
constexpr uint32_t SM_KV = 32768;             // 2 stages x (K 32 KiB + V 32 KiB)
constexpr uint32_t SM_P = SM_KV + 2 * 65536;  // 2 x 32 KiB
constexpr uint32_t SM_BAR = SM_P + 2 * 32768; // barriers and the TMEM address
constexpr uint32_t PF_SMEM = SM_BAR + 256 + 1024;

struct PfBars {
    uint64_t q_full, kv_full[2], kv_empty[2], s_full, s_free, p_full[2], o_done[2];
    uint32_t tmem;
};

__global__ void __launch_bounds__(PF_THREADS, 1) gist_prefill_kernel(const __grid_constant__ PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(base);
    PfBars& bars = *reinterpret_cast<PfBars*>(base + SM_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int bid = blockIdx.x;
    const int bh = bid % p.BH;
    const int t = p.n_qt - 1 - bid / p.BH;          // heaviest query tiles first
    const int b = bh / p.Hq, h = bh % p.Hq;
    const int bkv = b * (p.Hq / p.G) + h / p.G;
    const int j0 = t * p.QC;
    const int p0 = j0 * (p.C + 1);
    const int j_last = min(j0 + p.QC, p.N) - 1;      // last chunk of the tile
    const int n_gt = (j_last + 127) / 128;          // tiles of earlier gists
    const int n_kv = n_gt + 1;

    if (threadIdx.x == 0) {
        mbar_init(&bars.q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.kv_full[i], 1);
            mbar_init(&bars.kv_empty[i], 1);
            mbar_init(&bars.p_full[i], 128);
            mbar_init(&bars.o_done[i], 1);
        }
        mbar_init(&bars.s_full, 1);
        mbar_init(&bars.s_free, 128);
        fence_mbar_init();
    }
    if (warp == 4) {
        tc::tmem_alloc(&bars.tmem, 256);
        tc::tmem_relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = bars.tmem;
    const uint32_t tmem_s = tmem, tmem_o = tmem + 128;
    uint32_t* err = &g_prefill_err;   // waits below are bounded; a timeout abandons the tile

    if (warp == 4) {
        if (lane == 0) {
            // ---------------------------------------------- TMA + MMA issue --
            auto load_kv = [&](int i, int s) {
                uint8_t* ks = base + SM_KV + s * 65536;
                uint8_t* vs = ks + 32768;
                mbar_arrive_expect_tx(&bars.kv_full[s], 65536);
                if (i < n_gt) {
                    const int g0 = i * 128;
                    tc::tma_load_3d(ks, &p.tm_kg, 0, g0, bkv, &bars.kv_full[s]);
                    tc::tma_load_3d(ks + 16384, &p.tm_kg, 64, g0, bkv, &bars.kv_full[s]);
                    tc::tma_load_3d(vs, &p.tm_vg, 0, g0, bkv, &bars.kv_full[s]);
                    tc::tma_load_3d(vs + 16384, &p.tm_vg, 64, g0, bkv, &bars.kv_full[s]);
                } else {
                    tc::tma_load_3d(ks, &p.tm_k, 0, p0, bkv, &bars.kv_full[s]);
                    tc::tma_load_3d(ks + 16384, &p.tm_k, 64, p0, bkv, &bars.kv_full[s]);
                    tc::tma_load_3d(vs, &p.tm_v, 0, p0, bkv, &bars.kv_full[s]);
                    tc::tma_load_3d(vs + 16384, &p.tm_v, 64, p0, bkv, &bars.kv_full[s]);
                }
            };
            auto issue_s = [&](int i) {
                const uint32_t ks = sbase + SM_KV + (i & 1) * 65536;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    tc::mma_bf16(tmem_s, tc::sdesc_sw128(sbase + SM_Q + off, 16, 1024),
                                 tc::sdesc_sw128(ks + off, 16, 1024), IDESC_S, kk > 0);
                }
                tc::commit(&bars.s_full);
            };
            mbar_arrive_expect_tx(&bars.q_full, 32768);
            tc::tma_load_3d(base + SM_Q, &p.tm_q, 0, p0, bh, &bars.q_full);
            tc::tma_load_3d(base + SM_Q + 16384, &p.tm_q, 64, p0, bh, &bars.q_full);
            for (int i = 0; i < min(2, n_kv); ++i) load_kv(i, i);
            bool ok = mbar_wait(&bars.q_full, 0, err) && mbar_wait(&bars.kv_full[0], 0, err);
            tc::fence_after();
            if (ok) issue_s(0);
            for (int i = 0; ok && i < n_kv; ++i) {
                if (i + 1 < n_kv) {
                    ok = mbar_wait(&bars.kv_full[(i + 1) & 1], ((i + 1) >> 1) & 1, err) &&
                         mbar_wait(&bars.s_free, i & 1, err);
                    tc::fence_after();
                    if (!ok) break;
                    issue_s(i + 1);
                }
                if (!mbar_wait(&bars.p_full[i & 1], (i >> 1) & 1, err)) break;
                tc::fence_after();
                const uint32_t pb = sbase + SM_P + (i & 1) * 32768;
                const uint32_t vs = sbase + SM_KV + (i & 1) * 65536 + 32768;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
                    tc::mma_bf16(tmem_o, tc::sdesc_sw128(pb + aoff, 16, 1024),
                                 tc::sdesc_sw128(vs + kk * 2048, 16384, 1024), IDESC_PV, (i > 0 || kk > 0));
                }
                tc::commit(&bars.o_done[i & 1]);
                tc::commit(&bars.kv_empty[i & 1]);
                if (i + 2 < n_kv) {
                    if (!mbar_wait(&bars.kv_empty[i & 1], (i >> 1) & 1, err)) break;
                    load_kv(i + 2, i & 1);
                }
            }
        }
    } else {
        // ------------------------------------------------ softmax warps ----
        const int r = threadIdx.x;                       // query row = TMEM lane
        const int qp = p0 + r;
        const bool valid = r < p.QC * (p.C + 1) && qp < p.P;
        const int jq = valid ? j0 + r / (p.C + 1) : -1;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        float m_run = -INFINITY, l_run = 0.f;
        float s[128];
        for (int i = 0; i < n_kv; ++i) {
            if (!mbar_wait(&bars.s_full, i & 1, err)) break;
            tc::fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t u[32];
                tc::ld32(tmem_s + lane_off + c * 32, u);
                tc::wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) s[c * 32 + j] = __uint_as_float(u[j]);
            }
            tc::fence_before();
            mbar_arrive(&bars.s_free);
            // allowed key columns [lo, hi] of this row in this tile
            int lo, hi;
            if (i < n_gt) {
                lo = 0;
                hi = valid ? min(127, jq - i * 128 - 1) : -1;
            } else {
                lo = valid ? jq * (p.C + 1) - p0 : 1;
                hi = valid ? r : 0;
            }
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < 128; ++j) {
                s[j] = (j >= lo && j <= hi) ? s[j] * p.c2 : -INFINITY;
                mt = fmaxf(mt, s[j]);
            }
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
                mbar_wait(&bars.o_done[(i - 1) & 1], ((i - 1) >> 1) & 1, err);
                tc::fence_after();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t u[32];
                    tc::ld32(tmem_o + lane_off + c * 32, u);
                    tc::wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(__uint_as_float(u[j]) * alpha);
                    tc::st32(tmem_o + lane_off + c * 32, u);
                }
                tc::wait_st();
            }
            m_run = m_new;
            // the P buffer of this tile was last read by the P.V MMA of tile i-2
            if (i >= 2) mbar_wait(&bars.o_done[i & 1], ((i - 2) >> 1) & 1, err);
            uint8_t* prow = base + SM_P + (i & 1) * 32768 + r * 128;
            float sum = 0.f;
#pragma unroll
            for (int c16 = 0; c16 < 16; ++c16) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = c16 * 8 + 2 * e;
                    const float a = (m_run == -INFINITY) ? 0.f : exp2f(s[j] - m_run);
                    const float bb = (m_run == -INFINITY) ? 0.f : exp2f(s[j + 1] - m_run);
                    sum += a + bb;
                    w[e] = tc::pack_bf16x2(a, bb);
                }
                const int kb = c16 >> 3, ch = c16 & 7;
                *reinterpret_cast<uint4*>(prow + kb * 16384 + ((ch ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            l_run = l_run * alpha + sum;
            tc::fence_async_smem();
            tc::fence_before();
            mbar_arrive(&bars.p_full[i & 1]);
        }
        // ------------------------------------------------------ epilogue ----
        mbar_wait(&bars.o_done[(n_kv - 1) & 1], ((n_kv - 1) >> 1) & 1, err);
        tc::fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        uint16_t* orow = p.out + ((size_t)bh * p.P + qp) * PF_D;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t u[32];
            tc::ld32(tmem_o + lane_off + c * 32, u);
            tc::wait_ld();
            if (valid) {
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    uint4 v;
                    v.x = tc::pack_bf16x2(__uint_as_float(u[j]) * inv, __uint_as_float(u[j + 1]) * inv);
                    v.y = tc::pack_bf16x2(__uint_as_float(u[j + 2]) * inv, __uint_as_float(u[j + 3]) * inv);
                    v.z = tc::pack_bf16x2(__uint_as_float(u[j + 4]) * inv, __uint_as_float(u[j + 5]) * inv);
                    v.w = tc::pack_bf16x2(__uint_as_float(u[j + 6]) * inv, __uint_as_float(u[j + 7]) * inv);
                    *reinterpret_cast<uint4*>(orow + c * 32 + j) = v;
                }
            }
        }
        if (valid && p.lse != nullptr)
            p.lse[(size_t)bh * p.P + qp] = (m_run + log2f(l_run)) * 0.69314718055994531f;
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 4) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, 256);
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
    p.BH = B * Hq;
    p.Hq = Hq;
    p.G = Hq / Hkv;
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
    const unsigned grid = (unsigned)p.n_qt * (unsigned)p.BH;
    gist_prefill_kernel<<<grid, PF_THREADS, PF_SMEM, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}
