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

// SM cycle counter: cheap to read (%globaltimer costs tens of nanoseconds a
// read), so spin loops keep their time budget in cycles.  The budget of a
// wait of kWaitLimitNs is taken at 2 cycles per ns (the clock is at most
// 1.965 GHz), so the limit is reached after at most about that time at the
// highest clock, and later at lower clocks.
__device__ __forceinline__ uint64_t sm_cycles() { return (uint64_t)clock64(); }
constexpr uint64_t kWaitLimitCycles = 2ull * kWaitLimitNs;

// Wait for phase `parity` of `bar` to complete; after kWaitLimitCycles it
// gives up, ORs kErrTimeout into *err and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = sm_cycles();
    while (!mbar_try_wait(bar, parity)) {
        if (sm_cycles() - t0 > kWaitLimitCycles) {
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
        // plain shared-memory atomics: same-bin updates serialise, but a
        // warp-wide match of the bins costs far more
        for (int i = tid; i < n; i += NT) {
            const uint32_t u = key(i);
            if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
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


// --------------------------------------------------- threshold top-k --
// Exact top-k for k <= 32 of n <= NT * M keys: the k largest keys, equal keys
// taken lowest position first; out[0..k) receives the positions in ascending
// order.  Thread t holds the keys of positions lo + i * step, i < mine, in
// registers (key[i]); the positions of the threads may interleave in any way
// (step NT: every warp-wide load is one contiguous line).
//  1. In each warp, the k-th largest of the 32 lane maxima bounds the k-th
//     largest key of the whole set from below (k distinct keys reach it), so
//     the largest such bound over the warps, tau, does as well.
//  2. The keys >= tau (k of them at least, and rarely many more) go to a
//     shared list as 64-bit composites (key, ~position), each thread's after
//     those of the lower threads (a warp scan of the counts, then the warp
//     totals): a larger composite is a larger key, or the same key at a lower
//     position.
//  3. Each candidate counts the composites above its own; those with fewer
//     than k above are selected, the count being the key rank.  Each of the
//     k selected positions, one per rank, then counts the selected positions
//     below it: its place in the ascending output.
// Returns false without writing anything when more than NT keys reach tau
// (a flood of equal keys): the caller then runs a general selection.
// Scratch `w` (shared, 16-byte aligned): >= 16 + 2 * NT + 2 + 32 words.
// All NT threads call it; it ends with the block synchronised.
template <int NT, int M, int BAR = 0, int FIRST = 0>
__device__ bool threshold_topk_regs(const uint32_t (&key)[M], int lo, int step, int mine, int k, int32_t* out,
                                    uint32_t* w) {
    constexpr int NW = NT / 32;
    static_assert(2 * NW <= 16, "warp table overflow");
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
    group_sync<NT, BAR>();
    uint32_t tau = w[0];
#pragma unroll
    for (int i = 1; i < NW; ++i) tau = max(tau, w[i]);
    // this thread's candidates: counted, then placed after those of the lower
    // lanes and warps (warp totals through shared memory, no atomics)
    uint32_t c = 0;
#pragma unroll
    for (int i = 0; i < M; ++i) c += (i < mine && key[i] >= tau) ? 1u : 0u;
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) w[NW + warp] = incl;
    group_sync<NT, BAR>();
    uint32_t base = 0, total = 0;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
        const uint32_t x = w[NW + i];
        base += i < warp ? x : 0u;
        total += x;
    }
    if (total > (uint32_t)NT) {                   // the same on every thread
        group_sync<NT, BAR>();                    // all have read the table before the caller reuses w
        return false;
    }
    uint32_t off = base + incl - c;
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(w + 16);
#pragma unroll
    for (int i = 0; i < M; ++i)
        if (i < mine && key[i] >= tau) {
            cand[off] = ((unsigned long long)key[i] << 32) | (unsigned long long)(~(uint32_t)(lo + i * step));
            ++off;
        }
    // pad to an even count with 0 (never above a candidate: keys of
    // candidates are >= tau and positions are complemented)
    if (tid == 0 && (total & 1)) cand[total] = 0ull;
    group_sync<NT, BAR>();
    // key rank of each candidate: the composites above it; with at most NT/2
    // candidates two neighbouring threads split the count
    uint32_t* selpos = reinterpret_cast<uint32_t*>(w + 16 + 2 * NT + 2);   // [k]: position of key rank r
    {
        const bool two = total <= (uint32_t)(NT / 2);
        const uint32_t ci = two ? (uint32_t)(tid >> 1) : (uint32_t)tid;
        const uint32_t np = (total + 1) / 2, mid = np / 2;
        const uint32_t j0 = (two && (tid & 1)) ? mid : 0u, j1 = (two && !(tid & 1)) ? mid : np;
        const ulonglong2* c2 = reinterpret_cast<const ulonglong2*>(cand);
        unsigned long long mc = 0ull;
        int a = 0;
        if (ci < total) {
            mc = cand[ci];
#pragma unroll 4
            for (uint32_t j = j0; j < j1; ++j) {
                const ulonglong2 v = c2[j];
                a += (v.x > mc ? 1 : 0) + (v.y > mc ? 1 : 0);
            }
        }
        if (two) a += __shfl_xor_sync(0xFFFFFFFFu, a, 1);
        // ranks of the selected are 0..k-1, each once
        if (ci < total && (!two || !(tid & 1)) && a < k) selpos[a] = ~(uint32_t)mc;
    }
    group_sync<NT, BAR>();
    // the k selected positions, ascending: each goes to the count of selected
    // positions below it (they are distinct)
    if (tid < k) {
        const uint32_t me = selpos[tid];
        int r = 0;
#pragma unroll 8
        for (int j = 0; j < k; ++j) r += selpos[j] < me ? 1 : 0;
        out[r] = (int32_t)me;
    }
    group_sync<NT, BAR>();
    return true;
}

// Exact top-k (any 0 < k < n) of n keys held in registers: thread t holds
// positions t + i * NT for i < mine (key[i]).  Radix select on digits of up
// to 8 bits from the top, starting below the bits every key shares: each pass
// counts, in a 256-bin histogram (shared-memory atomics), the keys that share
// the prefix found so far, and the digit on which the k-th largest falls
// joins the prefix.  The k-th largest key T is then known; the keys above T
// are selected, and of the keys equal to T the lowest positions (a popcount
// scan of a bitmap in position order).  emit(r, pos) for the selected positions,
// ascending.  Scratch: w >= 288 + 2 NT / 32 words; bm >= max(256, 2 ceil(n /
// 32)) words (a histogram during the passes, then the bitmaps).  All NT
// threads of the group call it.
template <int NT, int U, int BAR = 0, int FIRST = 0, class Emit>
__device__ void radix_topk_regs(const uint32_t (&key)[U], int mine, int n, int k, uint32_t* w, uint32_t* bm,
                                Emit emit) {
    const int tid = threadIdx.x - FIRST, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = NT / 32;
    uint32_t* ctl = w + 256;     // [0] digit, [1] keys above it
    uint32_t* scan = w + 272;    // NT / 32 + 1
    uint32_t* mm = w + 288;      // [NW] smallest, [NW] largest key of each warp
    // the leading bits that every key shares (those of the smallest and the
    // largest key) need no pass: score keys share their sign and most of
    // their exponent
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
    for (int i = 0; i < U; ++i) {
        if (i < mine) {
            kmin = min(kmin, key[i]);
            kmax = max(kmax, key[i]);
        }
    }
    kmin = __reduce_min_sync(0xFFFFFFFFu, kmin);
    kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
    if (lane == 0) {
        mm[warp] = kmin;
        mm[NW + warp] = kmax;
    }
    for (int i = tid; i < 256; i += NT) w[i] = 0;
    group_sync<NT, BAR>();
#pragma unroll
    for (int i = 0; i < NW; ++i) {
        kmin = min(kmin, mm[i]);
        kmax = max(kmax, mm[NW + i]);
    }
    const int common = __clz(kmin ^ kmax);   // 32 when every key is the same
    uint32_t pmask = common > 0 ? (0xFFFFFFFFu << (32 - common)) : 0u;
    uint32_t prefix = kmax & pmask, kk = (uint32_t)k;
    // digits of up to 8 bits below the common prefix; the two histograms (w
    // and bm) alternate, so the next one is cleared during this pass
    int left = 32 - common, par = 0;
#pragma unroll 1
    while (left > 0) {
        const int width = min(8, left), shift = left - width;
        const uint32_t dmask = (1u << width) - 1u;
        uint32_t* hist = par ? bm : w;
        uint32_t* next = par ? w : bm;
#pragma unroll
        for (int i = 0; i < U; ++i) {
            if (i < mine && (key[i] & pmask) == prefix) atomicAdd(&hist[(key[i] >> shift) & dmask], 1u);
        }
        for (int i = tid; i < 256; i += NT) next[i] = 0;
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
        // (ctl is next written after the following pass's first barrier,
        // which every thread reaches only after reading it here)
        prefix |= ctl[0] << shift;
        pmask |= dmask << shift;
        kk -= ctl[1];
        left -= width;
        par ^= 1;
    }
    // T = prefix; take every key > T and the kk lowest positions of the keys == T
    const int nw = (n + 31) >> 5;
    uint32_t* sel = bm;
    uint32_t* eq = bm + nw;
    for (int i = tid; i < 2 * nw; i += NT) bm[i] = 0;
    group_sync<NT, BAR>();
#pragma unroll
    for (int i = 0; i < U; ++i) {
        if (i < mine) {
            const int pos = tid + i * NT;
            if (key[i] > prefix) atomicOr(&sel[pos >> 5], 1u << (pos & 31));
            else if (key[i] == prefix) atomicOr(&eq[pos >> 5], 1u << (pos & 31));
        }
    }
    group_sync<NT, BAR>();
    const int per = (nw + NT - 1) / NT, lo = tid * per, hi = min(nw, lo + per);
    {
        uint32_t c = 0;
        for (int i = lo; i < hi; ++i) c += __popc(eq[i]);
        uint32_t tot;
        uint32_t before = block_exclusive_scan<NT, BAR, FIRST>(c, scan, &tot);
        for (int i = lo; i < hi; ++i) {
            uint32_t bits = eq[i];
            while (bits) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1;
                if (before < kk) atomicOr(&sel[i], 1u << b);
                ++before;
            }
        }
    }
    group_sync<NT, BAR>();
    {
        uint32_t c = 0;
        for (int i = lo; i < hi; ++i) c += __popc(sel[i]);
        uint32_t tot;
        uint32_t r = block_exclusive_scan<NT, BAR, FIRST>(c, scan, &tot);
        for (int i = lo; i < hi; ++i) {
            uint32_t bits = sel[i];
            while (bits) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1;
                emit((int)r++, i * 32 + b);
            }
        }
    }
    group_sync<NT, BAR>();
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
