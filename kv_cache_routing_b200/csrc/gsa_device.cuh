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
// try_wait suspends the thread for a hardware-chosen interval per probe; this
// many probes bound one wait to well under a few seconds.
constexpr uint32_t kSpinLimit = 1u << 22;

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

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete; gives up after kSpinLimit
// probes, ORs kErrTimeout into *err and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
    for (uint32_t i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    atomicOr(err, kErrTimeout);
    return false;
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
__device__ __forceinline__ uint32_t order_key(float f) {
    if (f != f) return 0u;
    if (f == 0.0f) f = 0.0f;
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// -------------------------------------------------------------- block scan --
// Exclusive prefix sum over the block; returns this thread's prefix and
// writes the block total to *total.  `sh` holds >= NT/32 + 1 words.
template <int NT>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* sh, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NW = NT / 32;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < NW ? sh[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < NW) sh[lane] = w;  // inclusive warp totals
    }
    __syncthreads();
    uint32_t before = (warp > 0 ? sh[warp - 1] : 0u) + x - v;
    *total = sh[NW - 1];
    __syncthreads();
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
template <int NT, class KeyF, class Emit>
__device__ void block_topk(int n, int k, KeyF key, Emit emit, uint32_t* sh) {
    const int tid = threadIdx.x;
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
        __syncthreads();
        for (int i = tid; i < n; i += NT) {
            uint32_t u = key(i);
            if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
        }
        __syncthreads();
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
        __syncthreads();
        uint32_t digit = res[0];
        kk -= res[1];
        prefix |= digit << shift;
        pmask |= 255u << shift;
        __syncthreads();
    }
    // threshold key T = prefix: take every key > T and the first kk keys == T.
    const uint32_t T = prefix;
    const int seg = (n + NT - 1) / NT;
    const int lo = min(n, tid * seg), hi = min(n, lo + seg);
    uint32_t n_eq = 0;
    for (int i = lo; i < hi; ++i) n_eq += (key(i) == T);
    uint32_t tot;
    uint32_t eq_before = block_exclusive_scan<NT>(n_eq, scan, &tot);
    uint32_t n_sel = 0, e = eq_before;
    for (int i = lo; i < hi; ++i) {
        uint32_t u = key(i);
        if (u > T) ++n_sel;
        else if (u == T) { if (e < kk) ++n_sel; ++e; }
    }
    uint32_t sel_before = block_exclusive_scan<NT>(n_sel, scan, &tot);
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

}  // namespace gsa
