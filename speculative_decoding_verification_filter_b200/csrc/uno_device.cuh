// uno_device.cuh -- device helpers of libuno_filter: sortable keys, the
// counter-based RNG, and warp-level select / compact / sort primitives that
// the row kernels use.  Everything here runs on sm_100a.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace uno {

constexpr int kThreads = 256;              // threads per row CTA
constexpr int kWarps = kThreads / 32;      // warps per row CTA
constexpr unsigned kFull = 0xffffffffu;
constexpr int kMaxSplits = 16;             // CTAs that may share one row

// Draw identifiers (third Philox counter word).
constexpr uint32_t kDrawProposal = 0, kDrawAccept = 1, kDrawResidual = 2, kDrawTarget = 3;

// Flag bits, as in the public header.
constexpr uint32_t kFlagNonfinite = 1u, kFlagDraftNotInSupport = 2u, kFlagResidualEmpty = 4u, kFlagTimeout = 8u,
                   kFlagBadParams = 32u;

// ---------------------------------------------------------------------------
// Sortable 64-bit keys.  High word: the logit's binary32 bits mapped so that
// unsigned order equals numeric order; low word: ~token id, so that among
// equal logits the lower id has the larger key.  Larger key = ranked first
// by (logit desc, id asc).  Distinct tokens have distinct keys.  -0.0 is
// folded into +0.0 before a key is made.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ord_of_float(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float float_of_ord(uint32_t o) {
    uint32_t u = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
    return __uint_as_float(u);
}
__device__ __forceinline__ uint64_t make_key(float v, uint32_t id) {
    return ((uint64_t)ord_of_float(__fadd_rn(v, 0.0f)) << 32) | (uint64_t)(~id);
}
__device__ __forceinline__ float key_value(uint64_t k) { return float_of_ord((uint32_t)(k >> 32)); }
__device__ __forceinline__ int32_t key_id(uint64_t k) { return (int32_t)(~(uint32_t)k); }

// ord(-inf): every key of a real (finite) logit has a larger high word.
constexpr uint32_t kOrdNegInf = 0x007fffffu;

// Value below which an element cannot enter the top-k, for the cheap
// per-vector test: the logit value of threshold key tau (or -inf).
__device__ __forceinline__ float tau_value(uint64_t tau) {
    uint32_t hi = (uint32_t)(tau >> 32);
    if (hi <= kOrdNegInf) return -__int_as_float(0x7f800000);
    float v = float_of_ord(hi);
    return (v != v) ? -__int_as_float(0x7f800000) : v;
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC'11): ten rounds of two 32x32->64 multiplies with the
// Philox multipliers, the round key bumped by the Weyl constants between
// rounds.  The uniform of a decision: key = seed, counter = (request,
// position, draw, cycle), u = (x0 * 2^21 + (x1 >> 11)) * 2^-53 in [0, 1).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void philox4x32_10(uint32_t& c0, uint32_t& c1, uint32_t& c2, uint32_t& c3, uint32_t k0,
                                              uint32_t k1) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
        const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
        const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
    }
}

__device__ __forceinline__ double uniform53(uint64_t seed, uint32_t request, uint32_t position, uint32_t draw,
                                            uint32_t cycle) {
    uint32_t c0 = request, c1 = position, c2 = draw, c3 = cycle;
    philox4x32_10(c0, c1, c2, c3, (uint32_t)seed, (uint32_t)(seed >> 32));
    const uint64_t m = ((uint64_t)c0 << 21) | (uint64_t)(c1 >> 11);
    return (double)m * 0x1p-53;
}

// ---------------------------------------------------------------------------
// Bulk asynchronous copies (TMA, no multicast) into shared memory with
// mbarrier completion.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// global -> this CTA's shared memory; addresses 16-byte aligned, bytes a
// multiple of 16
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// plain arrival (release semantics at CTA scope)
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Every wait is bounded: try_wait suspends for a hardware-chosen time per
// attempt, so this limit is seconds, far beyond any real copy; on expiry the
// caller flags the row instead of hanging.
constexpr uint32_t kMaxWaitTries = 1u << 22;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    for (uint32_t it = 0; it < kMaxWaitTries; ++it)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// ---------------------------------------------------------------------------
// Warp-level primitives over a key array in shared memory.  All 32 lanes of
// the warp call them together; n is warp-uniform.
// ---------------------------------------------------------------------------

// Keep the keys >= t, in place, preserving order.  Returns the new count.
__device__ __forceinline__ int warp_keep_ge(uint64_t* buf, int n, uint64_t t, int lane) {
    int w = 0;
    for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        const bool act = i < n;
        const uint64_t key = act ? buf[i] : 0ull;
        const bool keep = act && key >= t;
        const unsigned bal = __ballot_sync(kFull, keep);
        // Every lane has read its slot of this 32-block before any write, and
        // writes land below base + 32, so the in-place copy is safe.
        if (keep) buf[w + __popc(bal & lanemask_lt())] = key;
        w += __popc(bal);
    }
    __syncwarp();
    return w;
}

// Largest x such that at least k keys of buf[0..n) have a high word >= x
// (1 <= k <= n): the k-th largest high word.  Bitwise binary search, one warp
// count per bit (a warp reduction, no atomics).  Each lane holds its keys'
// high words in registers (M per lane) so the 32 rounds touch no memory.
template <int M>
__device__ __forceinline__ uint32_t kth_high_regs(const uint64_t* buf, int n, int k, int lane) {
    uint32_t v[M];
#pragma unroll
    for (int j = 0; j < M; ++j) {
        const int i = lane + 32 * j;
        v[j] = i < n ? (uint32_t)(buf[i] >> 32) : 0u;  // 0 is below every real key
    }
    uint32_t x = 0;
#pragma unroll 1
    for (int b = 31; b >= 0; --b) {
        const uint32_t t = x | (1u << b);
        uint32_t c = 0;
#pragma unroll
        for (int j = 0; j < M; ++j) c += (v[j] >= t) ? 1u : 0u;
        if (__reduce_add_sync(kFull, c) >= (uint32_t)k) x = t;
    }
    return x;
}

__device__ __noinline__ uint32_t warp_kth_high(const uint64_t* buf, int n, int k, int lane) {
    if (n <= 64) return kth_high_regs<2>(buf, n, k, lane);
    if (n <= 128) return kth_high_regs<4>(buf, n, k, lane);
    if (n <= 256) return kth_high_regs<8>(buf, n, k, lane);
    if (n <= 512) return kth_high_regs<16>(buf, n, k, lane);
    uint32_t x = 0;  // large n: count from shared memory
#pragma unroll 1
    for (int b = 31; b >= 0; --b) {
        const uint32_t t = x | (1u << b);
        uint32_t c = 0;
        for (int i = lane; i < n; i += 32) c += ((uint32_t)(buf[i] >> 32) >= t) ? 1u : 0u;
        if (__reduce_add_sync(kFull, c) >= (uint32_t)k) x = t;
    }
    return x;
}

// The need-th largest low word among keys whose high word is x (registers,
// M per lane; 1 <= need <= that count).
template <int M>
__device__ __forceinline__ uint32_t kth_low_regs(const uint64_t* buf, int n, uint32_t x, uint32_t need, int lane) {
    uint32_t lo[M];
    bool in[M];
#pragma unroll
    for (int j = 0; j < M; ++j) {
        const int i = lane + 32 * j;
        const uint64_t key = i < n ? buf[i] : 0ull;
        in[j] = i < n && (uint32_t)(key >> 32) == x;
        lo[j] = (uint32_t)key;
    }
    uint32_t y = 0;
#pragma unroll 1
    for (int b = 31; b >= 0; --b) {
        const uint32_t t = y | (1u << b);
        uint32_t c = 0;
#pragma unroll
        for (int j = 0; j < M; ++j) c += (in[j] && lo[j] >= t) ? 1u : 0u;
        if (__reduce_add_sync(kFull, c) >= need) y = t;
    }
    return y;
}

// Exact k-th largest key among buf[0..n) (1 <= k <= n, keys distinct):
// returns t such that exactly k keys are >= t.  The high word first; if the
// keys sharing the k-th high word are not all needed, the low word decides.
__device__ __noinline__ uint64_t warp_select_kth(const uint64_t* buf, int n, int k, int lane) {
    const uint32_t x = warp_kth_high(buf, n, k, lane);
    uint32_t cgt = 0, ceq = 0;
    for (int i = lane; i < n; i += 32) {
        const uint32_t h = (uint32_t)(buf[i] >> 32);
        cgt += (h > x) ? 1u : 0u;
        ceq += (h == x) ? 1u : 0u;
    }
    cgt = __reduce_add_sync(kFull, cgt);
    ceq = __reduce_add_sync(kFull, ceq);
    const uint32_t need = (uint32_t)k - cgt;  // 1 <= need <= ceq
    if (need == ceq) return (uint64_t)x << 32;
    uint32_t y;
    if (n <= 64) {
        y = kth_low_regs<2>(buf, n, x, need, lane);
    } else if (n <= 256) {
        y = kth_low_regs<8>(buf, n, x, need, lane);
    } else if (n <= 512) {
        y = kth_low_regs<16>(buf, n, x, need, lane);
    } else {
        y = 0;
#pragma unroll 1
        for (int b = 31; b >= 0; --b) {
            const uint32_t t = y | (1u << b);
            uint32_t c = 0;
            for (int i = lane; i < n; i += 32) {
                const uint64_t key = buf[i];
                c += ((uint32_t)(key >> 32) == x && (uint32_t)key >= t) ? 1u : 0u;
            }
            if (__reduce_add_sync(kFull, c) >= need) y = t;
        }
    }
    return ((uint64_t)x << 32) | (uint64_t)y;
}

// Sequential sum of w[0..n) in index order (the defined rounding order), with
// loads issued ahead of the dependent adds.
__device__ __forceinline__ double serial_sum(const double* w, int n) {
    double s = 0.0;
    int j = 0;
    for (; j + 8 <= n; j += 8) {
        double b[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) b[q] = w[j + q];
#pragma unroll
        for (int q = 0; q < 8; ++q) s += b[q];
    }
    for (; j < n; ++j) s += w[j];
    return s;
}

// Bitonic sort of buf[0..npow2) in shared memory by one warp; descending when
// desc.  npow2 is a power of two; callers pad with a key that sorts last.
__device__ __noinline__ void warp_bitonic_sort(uint64_t* buf, int npow2, bool desc, int lane) {
    for (int size = 2; size <= npow2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = lane; i < (npow2 >> 1); i += 32) {
                const int a = 2 * i - (i & (stride - 1));
                const int b = a + stride;
                // at the last stage (size == npow2) every pair uses `desc`
                const bool dir = ((a & size) == 0) ? desc : !desc;
                const uint64_t x = buf[a], y = buf[b];
                const bool swap = dir ? (x < y) : (x > y);
                if (swap) {
                    buf[a] = y;
                    buf[b] = x;
                }
            }
            __syncwarp();
        }
    }
}

__host__ __device__ __forceinline__ int next_pow2(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

// Inverse-CDF pick over weights w[0..n) (ascending-id order) by one thread:
// S = sum in order, x = u*S, first j with x < prefix_j, else the last j with
// a positive weight; -1 when every weight is zero.
__device__ __forceinline__ int inv_cdf_serial(const double* w, int n, double u) {
    const double S = serial_sum(w, n);
    if (!(S > 0.0)) return -1;
    const double x = u * S;
    double c = 0.0;
    int j = 0;
    for (; j + 8 <= n; j += 8) {
        double b[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) b[q] = w[j + q];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            c += b[q];
            if (x < c) return j + q;
        }
    }
    for (; j < n; ++j) {
        c += w[j];
        if (x < c) return j;
    }
    for (j = n - 1; j >= 0; --j)
        if (w[j] > 0.0) return j;
    return -1;
}

}  // namespace uno
