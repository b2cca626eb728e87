// Warp-level streaming attention engine used by every decode kernel.
//
// A CTA has NCW consumer warps and one producer warp.  The producer fills a
// ring of NS shared-memory stages with key/value rows through 1-D bulk copies
// (TMA engine); each stage holds TILE keys, TW per consumer warp.  A consumer
// warp owns the d-slice [sub*VEC, sub*VEC+VEC) of every key its lane group
// reads (16 bytes per lane), so one warp instruction covers KPI keys with
// conflict-free shared loads, and the G query heads of the KV head sit in
// registers.  The G partial dot products of ITS iterations are reduced across
// the key's LPK lanes with a transposing butterfly (each level halves the
// values a lane holds), the routing score is the sum of the G head logits, and
// the online softmax keeps (m, l, o) per head in the base-2 domain.
#pragma once

#include "gsa_device.cuh"

namespace gsa {

constexpr int NCW = 4;                 // consumer warps per CTA
constexpr int NTHREADS = (NCW + 1) * 32;
constexpr int STAGE_TENSOR_BYTES = 16384;  // keys of one tensor per stage
constexpr float kNegInf = -__builtin_huge_valf();

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

template <typename T, int D, int G>
struct Cfg {
    static constexpr int VEC = 16 / sizeof(T);          // elements per lane per key
    static constexpr int LPK = D / VEC;                 // lanes per key
    static constexpr int KPI = 32 / LPK;                // keys per warp iteration
    static constexpr int ITS = 8;                       // iterations per warp tile
    static constexpr int TW = KPI * ITS;                // keys per warp tile
    static constexpr int NV = ITS * G;                  // partial sums per lane
    static constexpr int LOG_LPK = ilog2(LPK);
    static constexpr int LOG_NV = ilog2(NV);
    static constexpr int NF = NV >= LPK ? NV / LPK : 1; // reduced values per lane
    static constexpr int ROWB = D * (int)sizeof(T);     // bytes per key row
    static constexpr int TILE = NCW * TW;               // keys per stage
    static constexpr int PT = G * TW;                   // (key, head) pairs per warp tile
    static constexpr int PPL = PT >= 32 ? PT / 32 : 1;  // pairs per lane (softmax phase)
    static constexpr int ACT = PT / PPL;                // lanes active in the softmax phase
    static constexpr int LPH = TW / PPL;                // lanes per head (softmax phase)
    static_assert(LPK * VEC == D && LPK <= 32, "head_dim / vector width");
    static_assert(TILE * ROWB == STAGE_TENSOR_BYTES, "stage size");
    static_assert(TW <= 32, "routing-score phase uses one lane per key");
};

// Reduce v[] across the LPK lanes of a key group.  Afterwards, with
// sub = lane & (LPK-1), v[t] (t < NF) is the total of value index
// sub*NF + t when NV >= LPK, else (t = 0) of index sub >> (LOG_LPK-LOG_NV).
template <int N, int O>
struct TReduce {
    template <int NV>
    __device__ __forceinline__ static void run(float (&v)[NV], int lane) {
        if constexpr (O >= 1) {
            if constexpr (N > 1) {
                constexpr int H = N / 2;
                const bool up = (lane & O) != 0;
#pragma unroll
                for (int i = 0; i < H; ++i) {
                    float send = up ? v[i] : v[i + H];
                    float keep = up ? v[i + H] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, O);
                }
                TReduce<H, O / 2>::run(v, lane);
            } else {
                v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], O);
                TReduce<1, O / 2>::run(v, lane);
            }
        }
    }
};

// arr[i] for a runtime i without dynamic register indexing.
template <int N>
__device__ __forceinline__ float pick(const float (&arr)[N], int i) {
    float r = arr[0];
#pragma unroll
    for (int t = 1; t < N; ++t) r = (i == t) ? arr[t] : r;
    return r;
}

// Per-warp scratch in shared memory.
template <int G, int TW>
struct WarpScratch {
    float lg[TW * G];   // raw dot products, [key][head]
    float pk[TW * G];   // softmax numerators, [key][head]
    float mt[G > 4 ? G : 4];
};

template <typename T, int D, int G>
struct WarpAttn {
    using C = Cfg<T, D, G>;
    float q[G][C::VEC];
    float o[G][C::VEC];
    float m[G];
    float lp;           // this lane's share of l for head (lane / LPH)

    __device__ __forceinline__ void load_q(const T* qrow_base /* q[b][hk*G] */, int lane) {
        const int sub = lane & (C::LPK - 1);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const uint4 r = *reinterpret_cast<const uint4*>(
                reinterpret_cast<const uint8_t*>(qrow_base) + (size_t)h * C::ROWB + sub * 16);
            float x[C::VEC];
            Vec16<T>::unpack(r, x);
#pragma unroll
            for (int e = 0; e < C::VEC; ++e) q[h][e] = x[e];
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = kNegInf;
#pragma unroll
            for (int e = 0; e < C::VEC; ++e) o[h][e] = 0.f;
        }
        lp = 0.f;
    }

    // Dot products of the warp tile's keys with every head; writes lg[key][h].
    __device__ __forceinline__ void qk(const uint8_t* kt /* warp tile K rows */, WarpScratch<G, C::TW>& ws,
                                       int lane) const {
        const int sub = lane & (C::LPK - 1);
        const int hf = lane >> C::LOG_LPK;
        float part[C::NV];
#pragma unroll
        for (int it = 0; it < C::ITS; ++it) {
            const int key = it * C::KPI + hf;
            const uint4 r = *reinterpret_cast<const uint4*>(kt + key * C::ROWB + sub * 16);
            float x[C::VEC];
            Vec16<T>::unpack(r, x);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float acc = 0.f;
#pragma unroll
                for (int e = 0; e < C::VEC; ++e) acc = fmaf(q[h][e], x[e], acc);
                part[it * G + h] = acc;
            }
        }
        TReduce<C::NV, C::LPK / 2>::run(part, lane);
        if constexpr (C::NV >= C::LPK) {
#pragma unroll
            for (int t = 0; t < C::NF; ++t) {
                const int i = sub * C::NF + t;       // value index = it*G + h
                const int it = i / G, h = i % G;
                ws.lg[(it * C::KPI + hf) * G + h] = part[t];
            }
        } else {
            constexpr int SH = C::LOG_LPK - C::LOG_NV;
            if ((sub & ((1 << SH) - 1)) == 0) {
                const int i = sub >> SH;
                const int it = i / G, h = i % G;
                ws.lg[(it * C::KPI + hf) * G + h] = part[0];
            }
        }
        __syncwarp();
    }

    // Routing score of each valid key: sum over the heads of the raw dots.
    __device__ __forceinline__ float score(const WarpScratch<G, C::TW>& ws, int lane) const {
        float s = 0.f;
        if (lane < C::TW) {
#pragma unroll
            for (int h = 0; h < G; ++h) s += ws.lg[lane * G + h];
        }
        return s;
    }

    // Online softmax over the warp tile (first nv keys valid) and P.V.
    // (vmask: keys of the tile that take part; a key outside it gets no weight)
    __device__ __forceinline__ void softmax_pv(const uint8_t* vt /* warp tile V rows */,
                                               WarpScratch<G, C::TW>& ws, int nv, float c2, int lane,
                                               uint32_t vmask = 0xFFFFFFFFu) {
        const int sub = lane & (C::LPK - 1);
        const int hf = lane >> C::LOG_LPK;
        const int hl = lane / C::LPH;                     // this lane's head (softmax phase)
        float x[C::PPL];
        float mt = kNegInf;
#pragma unroll
        for (int u = 0; u < C::PPL; ++u) {
            const int pi = lane * C::PPL + u;             // head-major pair index
            const int key = pi % C::TW;
            x[u] = (lane < C::ACT && key < nv && ((vmask >> key) & 1u)) ? ws.lg[key * G + hl] * c2 : kNegInf;
            mt = fmaxf(mt, x[u]);
        }
#pragma unroll
        for (int off = 1; off < C::LPH; off <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, off));
        if (lane < C::ACT && (lane % C::LPH) == 0) ws.mt[hl] = mt;
        __syncwarp();
        float alpha[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float mn = fmaxf(m[h], ws.mt[h]);
            alpha[h] = (mn == kNegInf) ? 1.f : exp2f(m[h] - mn);
            m[h] = mn;
        }
        if (lane < C::ACT) {
            const float mh = pick(m, hl);
            float sum = 0.f;
#pragma unroll
            for (int u = 0; u < C::PPL; ++u) {
                const int pi = lane * C::PPL + u;
                const int key = pi % C::TW;
                const float p = (x[u] == kNegInf) ? 0.f : exp2f(x[u] - mh);
                sum += p;
                ws.pk[key * G + hl] = p;
            }
            lp = lp * pick(alpha, hl) + sum;
        }
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < C::VEC; ++e) o[h][e] *= alpha[h];
        __syncwarp();
#pragma unroll
        for (int it = 0; it < C::ITS; ++it) {
            const int key = it * C::KPI + hf;
            if (key < nv) {
                const uint4 r = *reinterpret_cast<const uint4*>(vt + key * C::ROWB + sub * 16);
                float v[C::VEC];
                Vec16<T>::unpack(r, v);
                float p[G];
#pragma unroll
                for (int h = 0; h < G; ++h) p[h] = ws.pk[key * G + h];
#pragma unroll
                for (int h = 0; h < G; ++h)
#pragma unroll
                    for (int e = 0; e < C::VEC; ++e) o[h][e] = fmaf(p[h], v[e], o[h][e]);
            }
        }
        __syncwarp();
    }

    // Reduce the warp's state and store it for the CTA combine:
    // cm[h], cl[h] and co[h][0..D) of this warp.
    __device__ __forceinline__ void finish(float* cm, float* cl, float* co, int lane) {
        const int sub = lane & (C::LPK - 1);
        const int hf = lane >> C::LOG_LPK;
#pragma unroll
        for (int off = C::LPK; off < 32; off <<= 1)
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < C::VEC; ++e) o[h][e] += __shfl_xor_sync(0xFFFFFFFFu, o[h][e], off);
        float l = lp;
#pragma unroll
        for (int off = 1; off < C::LPH; off <<= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
        if (hf == 0) {
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < C::VEC; ++e) co[h * D + sub * C::VEC + e] = o[h][e];
        }
        if (lane < C::ACT && (lane % C::LPH) == 0) cl[lane / C::LPH] = l;
        if (lane == 0) {   // m is warp-uniform
#pragma unroll
            for (int h = 0; h < G; ++h) cm[h] = m[h];
        }
    }
};

// Combine the NCW warps' (m, l, o) into one partial (M, L, O) per head and
// write it to part[h][0..D), ml[h][0..2).  cm: [NCW][G], cl: [NCW][G],
// co: [NCW][G][D].  Called by all threads after a __syncthreads.
template <int D, int G>
__device__ __forceinline__ void cta_combine(const float* cm, const float* cl, const float* co, float* part,
                                            float* ml) {
    for (int i = threadIdx.x; i < G * D; i += NTHREADS) {
        const int h = i / D, e = i % D;
        float M = kNegInf;
#pragma unroll
        for (int w = 0; w < NCW; ++w) M = fmaxf(M, cm[w * G + h]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w) {
            const float mw = cm[w * G + h];
            const float s = (mw == kNegInf) ? 0.f : exp2f(mw - M);
            L += cl[w * G + h] * s;
            O += co[(w * G + h) * D + e] * s;
        }
        part[h * D + e] = O;
        if (e == 0) {
            ml[h * 2 + 0] = M;
            ml[h * 2 + 1] = L;
        }
    }
}

}  // namespace gsa
