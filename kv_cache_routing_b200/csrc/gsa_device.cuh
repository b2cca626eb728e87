// Device building blocks shared by the GSA kernels (sm_100a).
//
//  - thin inline-PTX wrappers: mbarrier, 1-D bulk copy (TMA engine),
//    programmatic dependent launch;
//  - bounded waits that record an error flag instead of hanging;
//  - the orderable 32-bit key of an fp32 score and a block-wide exact top-k
//    by radix select (lowest index wins ties, output in index order).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gsa {

constexpr uint32_t kErrTimeout = 1u;   // matches GSA_WS_ERR_TIMEOUT
constexpr uint32_t kErrIndex = 2u;     // matches GSA_WS_ERR_INDEX
// A bounded wait gives up after this many nanoseconds of %globaltimer time.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier --
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    // make barrier initialisation visible to the async (TMA) proxy
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Raise the transaction count of the current phase without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    // the suspend-time hint (ns) lets the thread sleep until the phase
    // completes instead of spinning on the issue slots
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}

// Non-blocking probe: has phase `parity` of `bar` completed?
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of `bar` to complete; after kWaitLimitNs it gives
// up, ORs kErrTimeout into *err and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, kErrTimeout);
            return false;
        }
    }
    return true;
}

// ------------------------------------------------------------- bulk copies --
// 1-D bulk copy global -> shared through the TMA engine; completion is
// signalled as transaction bytes on `bar`.  dst, src 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// L2 policy for data read once per step (KV caches): evict first.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// -------------------------------------------------- programmatic launches --
// Wait until the preceding grid in the stream has completed and its memory
// is visible (no-op when the launch was not programmatic).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next grid in the stream to begin launching.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------ conversions --
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 16 bytes of elements -> fp32 (8 bf16 or 4 fp32).
template <typename T>
struct Vec16;
template <>
struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(const uint4& r, float (&x)[4]) {
        x[0] = __uint_as_float(r.x);
        x[1] = __uint_as_float(r.y);
        x[2] = __uint_as_float(r.z);
        x[3] = __uint_as_float(r.w);
    }
};
struct bf16_t {
    uint16_t bits;
};
template <>
struct Vec16<bf16_t> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(const uint4& r, float (&x)[8]) {
        x[0] = bf16lo(r.x);
        x[1] = bf16hi(r.x);
        x[2] = bf16lo(r.y);
        x[3] = bf16hi(r.y);
        x[4] = bf16lo(r.z);
        x[5] = bf16hi(r.z);
        x[6] = bf16lo(r.w);
        x[7] = bf16hi(r.w);
    }
};

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    // round-to-nearest-even on the upper half (finite inputs)
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7F800000u) == 0x7F800000u) return static_cast<uint16_t>((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
    u += 0x7FFFu + ((u >> 16) & 1u);
    return static_cast<uint16_t>(u >> 16);
}

// ---------------------------------------------------------- ordering keys --
// Monotone map fp32 -> u32 (larger score -> larger key).  -0 and +0 share a
// key; NaN maps to 0, below every number.
// Written with selects only, so that a key computed from a load does not
// put a branch between that load and the next.
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = f == 0.0f ? 0u : __float_as_uint(f);
    const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return f != f ? 0u : k;
}

// ------------------------------------------------------------ thread groups --
// The block-wide helpers below run on a group of NT threads: threads
// [FIRST, FIRST + NT) of the block, synchronised by named barrier BAR (0: the
// whole block, NT == blockDim.x).  FIRST is a multiple of 32.
template <int NT, int BAR>
__device__ __forceinline__ void group_sync() {
    if constexpr (BAR == 0) __syncthreads();
    else asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
}

// -------------------------------------------------------------- block scan --
// Exclusive prefix sum over the group; returns this thread's prefix and
// writes the group total to *total.  `sh` holds >= NT/32 + 1 words.
template <int NT, int BAR = 0, int FIRST = 0>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* sh, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = (threadIdx.x - FIRST) >> 5;
    constexpr int NW = NT / 32;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    group_sync<NT, BAR>();
    if (warp == 0) {
        uint32_t w = lane < NW ? sh[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < NW) sh[lane] = w;  // inclusive warp totals
    }
    group_sync<NT, BAR>();
    uint32_t before = (warp > 0 ? sh[warp - 1] : 0u) + x - v;
    *total = sh[NW - 1];
    group_sync<NT, BAR>();
    return before;
}

// ----------------------------------------------------------- block top-k --
// Exact top-k of n keys given in position order: the k largest keys, equal
// keys taken in position order (so with keys built from scores and positions
// in index order, ties go to the lowest index).  Calls emit(rank, pos) for
// every selected position, rank = 0..k-1 in position order.
// Radix select over the 32-bit key, 8 bits per pass, then one ordered
// compaction.  `sh` holds >= 256 + NT/32 + 8 words of shared memory.
// All NT threads of the block must call it.
template <int NT, int BAR = 0, int FIRST = 0, class KeyF, class Emit>
__device__ void block_topk(int n, int k, KeyF key, Emit emit, uint32_t* sh) {
    const int tid = threadIdx.x - FIRST;
    if (k <= 0 || n <= 0) return;
    if (k >= n) {
        for (int i = tid; i < n; i += NT) emit(i, i);
        return;
    }
    uint32_t* hist = sh;              // 256
    uint32_t* res = sh + 256;         // [0] digit, [1] count above
    uint32_t* scan = sh + 256 + 4;    // NT/32 + 1
    uint32_t prefix = 0, pmask = 0;
    uint32_t kk = static_cast<uint32_t>(k);
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += NT) hist[i] = 0;
        group_sync<NT, BAR>();
        // warp-aggregated histogram: float keys crowd a few bins in the high
        // digits, so lanes with the same bin add once per warp instruction
        for (int i0 = tid - (tid & 31); i0 < n; i0 += NT) {
            const int i = i0 + (tid & 31);
            uint32_t bin = 0xFFFFFFFFu;
            if (i < n) {
                const uint32_t u = key(i);
                if ((u & pmask) == prefix) bin = (u >> shift) & 255u;
            }
            const uint32_t same = __match_any_sync(0xFFFFFFFFu, bin);
            if (bin != 0xFFFFFFFFu && (tid & 31) == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
        }
        group_sync<NT, BAR>();
        if (tid < 32) {
            // lane l owns bins 255-8l .. 248-8l (descending)
            const int lane = tid;
            uint32_t cnt[8], tot = 0;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                cnt[t] = hist[255 - 8 * lane - t];
                tot += cnt[t];
            }
            uint32_t incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += y;
            }
            uint32_t above = incl - tot;  // keys in higher bins than this lane's
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                if (above < kk && above + cnt[t] >= kk) {
                    res[0] = static_cast<uint32_t>(255 - 8 * lane - t);
                    res[1] = above;
                }
                above += cnt[t];
            }
        }
        group_sync<NT, BAR>();
        uint32_t digit = res[0];
        kk -= res[1];
        prefix |= digit << shift;
        pmask |= 255u << shift;
        group_sync<NT, BAR>();
    }
    // threshold key T = prefix: take every key > T and the first kk keys == T.
    const uint32_t T = prefix;
    const int seg = (n + NT - 1) / NT;
    const int lo = min(n, tid * seg), hi = min(n, lo + seg);
    uint32_t n_eq = 0;
    for (int i = lo; i < hi; ++i) n_eq += (key(i) == T);
    uint32_t tot;
    uint32_t eq_before = block_exclusive_scan<NT, BAR, FIRST>(n_eq, scan, &tot);
    uint32_t n_sel = 0, e = eq_before;
    for (int i = lo; i < hi; ++i) {
        uint32_t u = key(i);
        if (u > T) ++n_sel;
        else if (u == T) { if (e < kk) ++n_sel; ++e; }
    }
    uint32_t sel_before = block_exclusive_scan<NT, BAR, FIRST>(n_sel, scan, &tot);
    uint32_t r = sel_before;
    e = eq_before;
    for (int i = lo; i < hi; ++i) {
        uint32_t u = key(i);
        bool take = false;
        if (u > T) take = true;
        else if (u == T) { take = e < kk; ++e; }
        if (take) emit(static_cast<int>(r++), i);
    }
}


// ------------------------------------------------- shared-memory top-k --
// Exact top-k of n orderable keys held in shared memory (keys[i] for
// position i): the k largest keys, equal keys taken lowest position first.
// Writes the k selected positions to out[0..k) in ascending order.
// Radix select, 8 bits per digit, compacting the candidates after every
// digit (keys above the threshold digit are selected at once, keys on it
// stay candidates), so only the first digit reads all n keys; the selection
// is kept as a bitmap and emitted in position order by a popcount prefix.
// Scratch `w` (shared): >= 256 + 16 + 2*NT/32 + (n+31)/32 * 2 + 2*n words
// (histogram, control, scan, two bitmaps, two candidate lists).
// All NT threads of the block call it.
template <int NT, int BAR = 0, int FIRST = 0>
__device__ void smem_topk(const uint32_t* keys, int n, int k, int32_t* out, uint32_t* w) {
    const int tid = threadIdx.x - FIRST, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = NT / 32;
    if (k <= 0 || n <= 0) return;
    if (k >= n) {
        for (int i = tid; i < n; i += NT) out[i] = i;
        return;
    }
    const int nw = (n + 31) >> 5;
    uint32_t* hist = w;                   // 256
    uint32_t* ctl = w + 256;              // [0] digit, [1] above, [2] next count, [3] done flag
    uint32_t* scan = ctl + 16;            // 2 * NW
    uint32_t* sel = scan + 2 * NW;        // nw words: selected positions
    uint32_t* tie = sel + nw;             // nw words: candidates left after the last digit
    uint32_t* cand = tie + nw;            // candidate positions (unordered), read list
    uint32_t* next = cand + n;            // write list; the two swap after every digit
    for (int i = tid; i < nw; i += NT) {
        sel[i] = 0;
        tie[i] = 0;
    }
    uint32_t kk = (uint32_t)k;
    int m = n;                            // candidates: all positions on the first digit
    bool all = true;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += NT) hist[i] = 0;
        if (tid == 0) ctl[2] = 0;
        group_sync<NT, BAR>();
        for (int i0 = tid - lane; i0 < m; i0 += NT) {
            const int i = i0 + lane;
            uint32_t bin = 0xFFFFFFFFu;
            if (i < m) bin = (keys[all ? i : cand[i]] >> shift) & 255u;
            const uint32_t same = __match_any_sync(0xFFFFFFFFu, bin);
            if (bin != 0xFFFFFFFFu && lane == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
        }
        group_sync<NT, BAR>();
        if (warp == 0) {
            // lane l owns bins 255-8l .. 248-8l (descending)
            uint32_t cnt[8], tot = 0;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                cnt[t] = hist[255 - 8 * lane - t];
                tot += cnt[t];
            }
            uint32_t incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += y;
            }
            uint32_t above = incl - tot;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                if (above < kk && above + cnt[t] >= kk) {
                    ctl[0] = 255u - 8u * lane - t;
                    ctl[1] = above;
                }
                above += cnt[t];
            }
        }
        group_sync<NT, BAR>();
        const uint32_t D = ctl[0], above = ctl[1];
        const bool last = shift == 0;
        // keys above the threshold digit are selected; keys on it stay
        // candidates (warp-aggregated: one atomic per warp and predicate)
        for (int i0 = tid - lane; i0 < m; i0 += NT) {
            const int i = i0 + lane;
            int pos = 0;
            uint32_t dg = 0;
            if (i < m) {
                pos = all ? i : (int)cand[i];
                dg = (keys[pos] >> shift) & 255u;
            }
            const bool up = i < m && dg > D, eq = i < m && dg == D;
            const uint32_t mup = __ballot_sync(0xFFFFFFFFu, up);
            const uint32_t meq = __ballot_sync(0xFFFFFFFFu, eq);
            if (all) {
                // positions i0..i0+31 are exactly one bitmap word (i0 is a multiple of 32)
                if (lane == 0) {
                    if (mup) sel[i0 >> 5] |= mup;
                    if (last && meq) tie[i0 >> 5] |= meq;
                }
            } else {
                if (up) atomicOr(&sel[pos >> 5], 1u << (pos & 31));
                if (last && eq) atomicOr(&tie[pos >> 5], 1u << (pos & 31));
            }
            if (!last && meq) {
                uint32_t base = 0;
                if (lane == 0) base = atomicAdd(&ctl[2], (uint32_t)__popc(meq));
                base = __shfl_sync(0xFFFFFFFFu, base, 0);
                if (eq) next[base + __popc(meq & ((1u << lane) - 1u))] = (uint32_t)pos;
            }
        }
        group_sync<NT, BAR>();
        kk -= above;
        m = (int)ctl[2];
        all = false;
        {
            uint32_t* t = cand;
            cand = next;
            next = t;
        }
        group_sync<NT, BAR>();
        if (!last && (uint32_t)m == kk) {
            // every remaining candidate is selected
            for (int i = tid; i < m; i += NT) atomicOr(&sel[cand[i] >> 5], 1u << (cand[i] & 31));
            kk = 0;
            group_sync<NT, BAR>();
            break;
        }
    }
    // equal keys on the threshold: the kk lowest positions (tie bitmap in position order)
    if (kk > 0) {
        uint32_t c = 0;
        const int per = (nw + NT - 1) / NT, lo = tid * per, hi = min(nw, lo + per);
        for (int i = lo; i < hi; ++i) c += __popc(tie[i]);
        uint32_t tot;
        uint32_t before = block_exclusive_scan<NT, BAR, FIRST>(c, scan, &tot);
        for (int i = lo; i < hi; ++i) {
            uint32_t bits = tie[i];
            while (bits) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1;
                if (before < kk) atomicOr(&sel[i], 1u << b);
                ++before;
            }
        }
        group_sync<NT, BAR>();
    }
    // emit the selection in ascending position order
    {
        uint32_t c = 0;
        const int per = (nw + NT - 1) / NT, lo = tid * per, hi = min(nw, lo + per);
        for (int i = lo; i < hi; ++i) c += __popc(sel[i]);
        uint32_t tot;
        uint32_t r = block_exclusive_scan<NT, BAR, FIRST>(c, scan, &tot);
        for (int i = lo; i < hi; ++i) {
            uint32_t bits = sel[i];
            while (bits) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1;
                out[r++] = i * 32 + b;
            }
        }
    }
}


// --------------------------------------------------- threshold top-k --
// Exact top-k for k <= 32 of n <= NT * M keys: the k largest keys, equal keys
// taken lowest position first; out[0..k) receives the positions in ascending
// order.  Thread t holds the keys of positions lo + i * step, i < mine, in
// registers (key[i]); the positions of the threads may interleave in any way
// (step NT: every warp-wide load is one contiguous line).
//  1. In each warp, the k-th largest of the 32 lane maxima bounds the k-th
//     largest key of the whole set from below (k distinct keys reach it), so
//     the largest such bound over the warps, tau, does as well.
//  2. The keys >= tau (k of them at least, and rarely many more) are appended,
//     in any order, to a shared list as 64-bit composites (key, ~position): a
//     larger composite is a larger key, or the same key at a lower position.
//  3. Each candidate counts the composites above its own; those with fewer
//     than k above are selected, the count being the key rank.  The k
//     selected positions, one per rank, are sorted ascending by one warp.
// Returns false without writing anything when more than NT keys reach tau
// (a flood of equal keys): the caller then runs a general selection.
// Scratch `w` (shared, 16-byte aligned): >= 16 + 2 * NT + 2 + 32 words.
// All NT threads call it; it ends with the block synchronised.
template <int NT, int M, int BAR = 0, int FIRST = 0>
__device__ bool threshold_topk_regs(const uint32_t (&key)[M], int lo, int step, int mine, int k, int32_t* out,
                                    uint32_t* w) {
    constexpr int NW = NT / 32;
    static_assert(NW + 1 <= 16, "warp bound table overflow");
    const int tid = threadIdx.x - FIRST, lane = tid & 31, warp = tid >> 5;
    uint32_t tmax = 0u;
#pragma unroll
    for (int i = 0; i < M; ++i) tmax = max(tmax, i < mine ? key[i] : 0u);
    // the k-th largest of the warp's 32 lane maxima is the warp's bound (a
    // lane without keys offers 0, the smallest key, which can only weaken
    // it): a bitonic sort of the lane maxima, descending, leaves it in lane k-1
    uint32_t v = tmax;
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const uint32_t o = __shfl_xor_sync(0xFFFFFFFFu, v, stride);
            // descending runs where (lane & size) == 0, the final pass descending
            const bool desc = ((lane & size) == 0) || size == 32;
            const bool lower = (lane & stride) == 0;
            v = (lower == desc) ? max(v, o) : min(v, o);
        }
    }
    const uint32_t tau_w = __shfl_sync(0xFFFFFFFFu, v, k - 1);
    if (lane == 0) w[warp] = tau_w;
    if (tid == 0) w[NW] = 0u;
    group_sync<NT, BAR>();
    uint32_t tau = w[0];
#pragma unroll
    for (int i = 1; i < NW; ++i) tau = max(tau, w[i]);
    // append this thread's candidates: one atomic per warp
    uint32_t c = 0;
#pragma unroll
    for (int i = 0; i < M; ++i) c += (i < mine && key[i] >= tau) ? 1u : 0u;
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    uint32_t base = 0;
    if (lane == 31 && incl > 0) base = atomicAdd(&w[NW], incl);
    base = __shfl_sync(0xFFFFFFFFu, base, 31);
    uint32_t off = base + incl - c;
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(w + 16);
#pragma unroll
    for (int i = 0; i < M; ++i)
        if (i < mine && key[i] >= tau) {
            if (off < (uint32_t)NT)
                cand[off] = ((unsigned long long)key[i] << 32) | (unsigned long long)(~(uint32_t)(lo + i * step));
            ++off;
        }
    group_sync<NT, BAR>();
    const uint32_t total = w[NW];
    if (total > (uint32_t)NT) return false;       // the same on every thread
    unsigned long long mc = 0ull;
    uint32_t* selpos = reinterpret_cast<uint32_t*>(w + 16 + 2 * NT + 2);   // [k]: position of key rank r
    if ((uint32_t)tid < total) {
        mc = cand[tid];
        // pad to an even count with 0 (never above a candidate: keys of
        // candidates are >= tau and positions are complemented)
        if (tid == 0 && (total & 1)) cand[total] = 0ull;
    }
    group_sync<NT, BAR>();
    if ((uint32_t)tid < total) {
        const ulonglong2* c2 = reinterpret_cast<const ulonglong2*>(cand);
        int a = 0;
#pragma unroll 4
        for (uint32_t j = 0; j < (total + 1) / 2; ++j) {
            const ulonglong2 v = c2[j];
            a += (v.x > mc ? 1 : 0) + (v.y > mc ? 1 : 0);
        }
        if (a < k) selpos[a] = ~(uint32_t)mc;   // ranks of the selected are 0..k-1, each once
    }
    group_sync<NT, BAR>();
    // the k selected positions, ascending: a bitonic sort in the first warp
    if (warp == 0) {
        // (rolled: one warp runs this once per call, and unrolled its
        // instruction fetch, not its arithmetic, set its latency)
        uint32_t v = lane < k ? selpos[lane] : 0xFFFFFFFFu;
#pragma unroll 1
        for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll 1
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                const uint32_t o = __shfl_xor_sync(0xFFFFFFFFu, v, stride);
                const bool asc = ((lane & size) == 0) || size == 32;
                const bool lower = (lane & stride) == 0;
                v = (lower == asc) ? min(v, o) : max(v, o);
            }
        }
        if (lane < k) out[lane] = (int32_t)v;
    }
    group_sync<NT, BAR>();
    return true;
}

// The same selection with the keys in shared memory (keys[i] for position i).
template <int NT, int M, int BAR = 0, int FIRST = 0>
__device__ bool threshold_topk(const uint32_t* keys, int n, int k, int32_t* out, uint32_t* w) {
    const int m = (n + NT - 1) / NT;
    const int lo = (threadIdx.x - FIRST) * m;
    const int mine = max(0, min(m, n - lo));
    uint32_t key[M];
#pragma unroll
    for (int i = 0; i < M; ++i) key[i] = i < mine ? keys[lo + i] : 0u;
    return threshold_topk_regs<NT, M, BAR, FIRST>(key, lo, 1, mine, k, out, w);
}

// ----------------------------------------------------- per-thread copies --
// 16-byte global -> shared copy that bypasses L1 (cp.async, tracked per thread).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// Zero 16 bytes of shared memory through the same path (source size 0 reads nothing).
__device__ __forceinline__ void cp_async16_zero(void* dst, const void* any_global) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, 0;" ::"r"(smem_u32(dst)), "l"(any_global) : "memory");
}
// One arrival on `bar` once every cp.async this thread issued so far has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Hold the current phase of `bar` open until every cp.async this thread issued
// so far has landed (the pending count is raised now and lowered on landing;
// the phase's own expected arrivals are still needed to complete it).
__device__ __forceinline__ void cp_async_arrive_hold(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Acquire load of a counter other CTAs publish with a release.
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// `count` arrivals on `bar` at once.
__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

}  // namespace gsa
