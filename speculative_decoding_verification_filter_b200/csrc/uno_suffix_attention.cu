// uno_suffix_attention.cu -- tree-suffix attention of a request's V tree
// nodes, merged with the prefix attention state by log-sum-exp (the cascade
// split of EAGLE's tree verification that the UNO pull request fuses into one
// kernel; section "Modifications").
//
// One CTA per (request, key/value head).  The CTA stages the K and V rows of
// its head for the request's nodes in shared memory, rows padded to d + 1
// floats so that lanes reading different rows hit different banks, and
// builds each node's ancestor bit mask (V <= 128 bits) from the parent array.
// A warp then takes one (query head, node) pair at a time.
// - Scores: lane i owns keys i, i + 32, ...; it computes scale * <q, k_i> for
//   the keys the node may see, with q broadcast from shared memory.
// - Softmax statistics: warp max and sum by shuffles.
// - Output: lane t owns columns t, t + 32, ...; it accumulates p_i * v_i[t]
//   over the visible keys, whose weights are broadcast by shuffle.
// - Merge: the suffix state (o_s, l_s) is combined with the prefix state in
//   registers and written once.
// For tree sizes (V <= 128) the contraction is small; the kernel is bound by
// latency, not by HBM or the tensor cores.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <cmath>

#include "uno_filter.h"

namespace uno_sa {

constexpr int kWarps = 4;
constexpr int kMaxD = 256;
constexpr int kMaskWords = (UNO_MAX_TREE_NODES + 31) / 32;
constexpr unsigned kFull = 0xffffffffu;

struct Job {
    const void* q;
    const void* k;
    const void* v;
    int32_t bf16;
    int32_t R, V, H, Hkv, d, G;  // G = H / Hkv query heads per key/value head
    float scale;
    const int32_t* parent;
    const int32_t* num_nodes;
    const float* o_prefix;
    const float* lse_prefix;
    float* out_o;
    float* out_lse;
    uint32_t* out_flags;
};

__device__ __forceinline__ float load_elem(const void* base, int32_t bf16, size_t idx) {
    if (bf16) return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[idx]);
    return static_cast<const float*>(base)[idx];
}

// Ancestor masks of the first n nodes of one request: node j's mask holds j
// and its ancestors, found by walking up the parent links from j.  A link
// must point to an earlier node, and node 0's parent is -1; a node whose link
// breaks that rule keeps itself alone (the walk from any node below it stops
// there) and sets *s_bad.  Each thread walks its own nodes; s_par (n entries)
// is shared scratch.  Every thread of the block calls it; the caller
// synchronises the block before reading anc or *s_bad.
__device__ void build_ancestor_masks(const int32_t* parent, int n, uint32_t* anc, int32_t* s_par, int* s_bad,
                                     int tid, int nthreads) {
    for (int j = tid; j < n; j += nthreads) s_par[j] = parent[j];
    if (tid == 0) *s_bad = 0;
    __syncthreads();
    for (int j = tid; j < n; j += nthreads) {
        uint32_t mk[kMaskWords];
#pragma unroll
        for (int w = 0; w < kMaskWords; ++w) mk[w] = (j >> 5) == w ? 1u << (j & 31) : 0u;
        int cur = j;
        for (int step = 0; step < n; ++step) {  // links only go down, so at most j steps
            const int p = s_par[cur];
            const bool ok = cur == 0 ? p == -1 : (p >= 0 && p < cur);
            if (!ok && cur == j) *s_bad = 1;
            if (!ok || cur == 0) break;
#pragma unroll
            for (int w = 0; w < kMaskWords; ++w) mk[w] |= (p >> 5) == w ? 1u << (p & 31) : 0u;
            cur = p;
        }
#pragma unroll
        for (int w = 0; w < kMaskWords; ++w) anc[j * kMaskWords + w] = mk[w];
    }
}

__global__ void __launch_bounds__(32 * kWarps) suffix_attention_kernel(const __grid_constant__ Job J) {
    extern __shared__ float smem[];
    const int r = blockIdx.x, g = blockIdx.y;
    const int V = J.V, d = J.d, ld = d + 1;
    float* sk = smem;                                                    // [V][d + 1]
    float* sv = sk + (size_t)V * ld;                                     // [V][d + 1]
    float* sq = sv + (size_t)V * ld;                                     // [kWarps][d]
    uint32_t* anc = reinterpret_cast<uint32_t*>(sq + (size_t)kWarps * d);  // [V][kMaskWords]
    __shared__ int s_bad;
    __shared__ int32_t s_par[UNO_MAX_TREE_NODES];

    int n = J.num_nodes[r];
    n = n < 1 ? 1 : (n > V ? V : n);

    for (int e = threadIdx.x; e < n * d; e += blockDim.x) {
        const int i = e / d, t = e - i * d;
        const size_t src = (((size_t)r * V + i) * J.Hkv + g) * d + t;
        sk[i * ld + t] = load_elem(J.k, J.bf16, src);
        sv[i * ld + t] = load_elem(J.v, J.bf16, src);
    }
    build_ancestor_masks(J.parent + (size_t)r * V, n, anc, s_par, &s_bad, threadIdx.x, blockDim.x);
    __syncthreads();
    if (threadIdx.x == 0 && g == 0 && J.out_flags != nullptr) J.out_flags[r] = s_bad ? UNO_FLAG_BAD_TREE : 0u;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* qw = sq + (size_t)warp * d;
    for (int pair = warp; pair < J.G * n; pair += kWarps) {
        const int hl = pair / n, j = pair - hl * n;
        const int h = g * J.G + hl;
        const size_t row = ((size_t)r * V + j) * J.H + h;  // (request, node, query head)
        for (int t = lane; t < d; t += 32) qw[t] = load_elem(J.q, J.bf16, row * d + t);
        __syncwarp();

        const uint32_t* a = anc + j * kMaskWords;
        float s[kMaskWords];
        float m = -INFINITY;
#pragma unroll
        for (int c = 0; c < kMaskWords; ++c) {
            const int i = lane + 32 * c;
            s[c] = -INFINITY;
            if (i < n && ((a[c] >> lane) & 1u)) {
                const float* kr = sk + (size_t)i * ld;
                float acc = 0.0f;
                for (int t = 0; t < d; ++t) acc = fmaf(qw[t], kr[t], acc);
                s[c] = acc * J.scale;
                m = fmaxf(m, s[c]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
        float sum = 0.0f;
#pragma unroll
        for (int c = 0; c < kMaskWords; ++c) {
            s[c] = s[c] == -INFINITY ? 0.0f : expf(s[c] - m);
            sum += s[c];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);

        float oacc[kMaxD / 32];
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) oacc[u] = 0.0f;
#pragma unroll
        for (int c = 0; c < kMaskWords; ++c) {
            uint32_t bits = a[c];  // the same for every lane: the loop is warp-uniform
            while (bits) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1;
                const float w = __shfl_sync(kFull, s[c], b);
                const float* vr = sv + (size_t)(32 * c + b) * ld;
#pragma unroll
                for (int u = 0; u < kMaxD / 32; ++u) {
                    const int t = lane + 32 * u;
                    if (t < d) oacc[u] = fmaf(w, vr[t], oacc[u]);
                }
            }
        }

        const float lse_s = m + logf(sum);
        const float lp = J.lse_prefix[row];
        const bool has_prefix = lp != -INFINITY;
        const float M = has_prefix ? fmaxf(lp, lse_s) : lse_s;
        const float w1 = has_prefix ? expf(lp - M) : 0.0f;
        const float w2 = expf(lse_s - M);
        const float inv = 1.0f / (w1 + w2);
        const float inv_sum = 1.0f / sum;
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) {
            const int t = lane + 32 * u;
            if (t < d) {
                const float os = oacc[u] * inv_sum;
                const float o = has_prefix ? (w1 * J.o_prefix[row * d + t] + w2 * os) * inv : os;
                J.out_o[row * d + t] = o;
            }
        }
        if (lane == 0) J.out_lse[row] = M + logf(w1 + w2);
        __syncwarp();  // qw is rewritten by the next pair
    }

    // nodes past num_nodes: o = 0, lse = -inf, for this CTA's query heads
    const int pad = V - n;
    for (int e = threadIdx.x; e < pad * J.G * d; e += blockDim.x) {
        const int t = e % d, rest = e / d, hl = rest % J.G, j = n + rest / J.G;
        const size_t row = ((size_t)r * V + j) * J.H + g * J.G + hl;
        J.out_o[row * d + t] = 0.0f;
        if (t == 0) J.out_lse[row] = -INFINITY;
    }
}

// ---------------------------------------------------------------------------
// Tensor-core form: bf16 inputs, d a multiple of 16 up to 256.
//
// One CTA of four warps per (request, key/value head, tile of 128 stacked
// rows).  The rows of a tile are (query head, node) pairs of the G query
// heads that read this key/value head, row m = hl * V + j, so the G heads
// share one K and one V and the contraction has M = 128 (G = 4 heads of a
// V = 32 tree fill one tile exactly).
// - Staging: the tile's Q rows, the head's K rows and V transposed go to
//   shared memory in the tensor cores' K-major layout without swizzle: core
//   matrices of 8 rows x 16 bytes, the 16-byte chunks of a core matrix's
//   rows adjacent, core matrices along K 128 bytes apart (LBO) and groups of
//   8 rows 16 K bytes apart (SBO).  Nodes are padded to Np = V rounded up
//   to 16 with zeros.
// - S = Q K^T: one thread issues tcgen05.mma (kind::f16, bf16 in, f32
//   accumulate; M = 128, N = Np, d / 16 steps of K = 16) into TMEM columns
//   [0, Np); tcgen05.commit signals an mbarrier.
// - Thread t owns TMEM lane t, i.e. row t of the tile: it reads its row of S
//   (tcgen05.ld), applies the ancestor mask, takes the maximum and the sum
//   of exp, and writes its unnormalised weights P to shared memory as three
//   bf16 parts (hi + mid + lo carry P to a relative 2^-24, so the second
//   contraction is as accurate as one in binary32).
// - O = P V: three accumulating chains of tcgen05.mma (M = 128, N = d,
//   K = Np) into TMEM columns [128, 128 + d).
// - Epilogue: each thread reads its row of O, divides by the sum and merges
//   with the prefix state.
// Every wait on the mbarrier is bounded; on expiry the request is flagged
// UNO_FLAG_TIMEOUT, and the TMEM is freed after a second bounded wait.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

constexpr int kTcRows = 128;
constexpr int kTcThreads = 128;
constexpr uint32_t kTcColO = 128;  // TMEM column of O
constexpr uint32_t kTcMaxTries = 1u << 22;
constexpr int kTcBatch = 8;  // staging loads in flight per thread

// byte offset of bf16 element (row, k) of a K-major operand whose rows hold K elements
__device__ __forceinline__ uint32_t kmajor_off(int row, int k, int K) {
    return (uint32_t)((row >> 3) * (K * 16) + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}
// shared-memory matrix descriptor of such an operand starting at `addr`:
// start >> 4 in bits 0-13, LBO = 128 B in bits 16-29, SBO = 16 K bytes in
// bits 32-45, descriptor version 1 in bits 46-47, no swizzle (bits 61-63 = 0)
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr, int K) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) |
           ((uint64_t)(((uint32_t)K * 16u >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// instruction descriptor, kind::f16: f32 accumulator (bits 4-5 = 1), bf16 A
// and B (bits 7-9 = 1, 10-12 = 1), both K-major, N >> 3 in bits 17-22,
// M >> 4 in bits 24-28
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
// 16 consecutive f32 columns of this thread's TMEM lane (warp-collective)
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t x[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]), "=r"(x[4]), "=r"(x[5]), "=r"(x[6]), "=r"(x[7]),
          "=r"(x[8]), "=r"(x[9]), "=r"(x[10]), "=r"(x[11]), "=r"(x[12]), "=r"(x[13]), "=r"(x[14]), "=r"(x[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(x[i]);
}
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity) {
    for (uint32_t it = 0; it < kTcMaxTries; ++it)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}
__device__ __forceinline__ uint32_t bf16_bits(float x) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// shared-memory bytes of the tensor-core form: the operands (the
// epilogue's O blocks of 128 x (cb + 4) floats reuse their area and the
// ancestor masks), then a block of 128 x cb prefix floats that arrives by
// asynchronous copies while the block before it is worked on
__host__ __device__ inline int tc_block_cols(int d) { return d < 64 ? d : 64; }
__host__ __device__ inline size_t tc_prefetch_offset(int V, int d) {
    const int Np = (V + 15) / 16 * 16;
    const size_t ops = (size_t)kTcRows * d * 2 + (size_t)Np * d * 2 * 2 + (size_t)3 * kTcRows * Np * 2 +
                       (size_t)V * kMaskWords * 4;
    const size_t out = (size_t)kTcRows * (tc_block_cols(d) + 4) * 4;
    return ops > out ? ops : out;
}
__host__ __device__ inline size_t tc_smem_bytes(int V, int d) {
    return tc_prefetch_offset(V, d) + (size_t)kTcRows * tc_block_cols(d) * 4;
}
// 16 bytes global -> shared, asynchronously (both addresses 16-byte aligned)
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(kTcThreads) suffix_attention_tc_kernel(const __grid_constant__ Job J) {
    extern __shared__ __align__(1024) unsigned char sm[];
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    __shared__ int s_bad;
    __shared__ int32_t s_par[UNO_MAX_TREE_NODES];
    const int r = blockIdx.x, g = blockIdx.y, m0 = blockIdx.z * kTcRows;
    const int V = J.V, d = J.d, G = J.G, rows = G * V;
    const int Np = (V + 15) / 16 * 16;
    unsigned char* sQ = sm;                                   // [128][d]
    unsigned char* sK = sQ + (size_t)kTcRows * d * 2;         // [Np][d]
    unsigned char* sVt = sK + (size_t)Np * d * 2;             // [d][Np]
    unsigned char* sP = sVt + (size_t)d * Np * 2;             // 3 x [128][Np]
    uint32_t* anc = reinterpret_cast<uint32_t*>(sP + (size_t)3 * kTcRows * Np * 2);  // [V][kMaskWords]
    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t ncols = kTcColO + (uint32_t)d <= 256u ? 256u : 512u;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_base)),
                     "r"(ncols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    int n = J.num_nodes[r];
    n = n < 1 ? 1 : (n > V ? V : n);

    // staging: 16-byte chunks (8 elements).  Q and K go straight to their
    // K-major places by asynchronous copies (absent rows are zeroed); V is
    // transposed through registers, kTcBatch loads in flight per thread.
    const int cpr = d >> 3;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (int e = tid; e < kTcRows * cpr; e += kTcThreads) {
        const int ml = e / cpr, c = e - ml * cpr, m = m0 + ml;
        const int hl = m / V, j = m - hl * V;
        unsigned char* dst = sQ + kmajor_off(ml, c * 8, d);
        if (m < rows && j < n) {
            const size_t row = ((size_t)r * V + j) * J.H + (size_t)g * G + hl;
            cp_async16(dst, static_cast<const __nv_bfloat16*>(J.q) + row * d + c * 8);
        } else {
            *reinterpret_cast<uint4*>(dst) = zero;
        }
    }
    for (int e = tid; e < Np * cpr; e += kTcThreads) {
        const int i = e / cpr, c = e - i * cpr;
        unsigned char* dst = sK + kmajor_off(i, c * 8, d);
        if (i < n)
            cp_async16(dst, static_cast<const __nv_bfloat16*>(J.k) + (((size_t)r * V + i) * J.Hkv + g) * d + c * 8);
        else
            *reinterpret_cast<uint4*>(dst) = zero;
    }
    cp_async_commit();
    // the first block of the prefix state, for the epilogue: it lands while
    // the products run (rows past num_nodes and past the stack are skipped)
    const int cb = tc_block_cols(d);
    float* sPre = reinterpret_cast<float*>(sm + tc_prefetch_offset(V, d));  // [128][cb]
    auto prefetch = [&](int b0) {
        const int f4 = cb >> 2;
        for (int e = tid; e < kTcRows * f4; e += kTcThreads) {
            const int pl = e / f4, c4 = e - pl * f4, pm = m0 + pl;
            const int ph = pm / V, pj = pm - ph * V;
            if (pm < rows && pj < n) {
                const size_t orow = ((size_t)r * V + pj) * J.H + (size_t)g * G + ph;
                cp_async16(sPre + (size_t)pl * cb + 4 * c4, J.o_prefix + orow * d + b0 + 4 * c4);
            }
        }
        cp_async_commit();
    };
    prefetch(0);
    for (int e0 = tid; e0 < Np * cpr; e0 += kTcThreads * (kTcBatch / 2)) {
        uint4 vx[kTcBatch / 2];
#pragma unroll
        for (int u = 0; u < kTcBatch / 2; ++u) {
            const int e = e0 + u * kTcThreads, i = e / cpr, c = e - i * cpr;
            vx[u] = zero;
            if (e < Np * cpr && i < n) {
                const size_t src = (((size_t)r * V + i) * J.Hkv + g) * d;
                vx[u] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(J.v) + src) + c);
            }
        }
#pragma unroll
        for (int u = 0; u < kTcBatch / 2; ++u) {
            const int e = e0 + u * kTcThreads, i = e / cpr, c = e - i * cpr;
            if (e >= Np * cpr) continue;
            const uint32_t w[4] = {vx[u].x, vx[u].y, vx[u].z, vx[u].w};
#pragma unroll
            for (int q = 0; q < 8; ++q)  // V^T: element (column t of V, node i)
                *reinterpret_cast<uint16_t*>(sVt + kmajor_off(c * 8 + q, i, Np)) =
                    (uint16_t)((q & 1) ? (w[q >> 1] >> 16) : (w[q >> 1] & 0xffffu));
        }
    }
    build_ancestor_masks(J.parent + (size_t)r * V, n, anc, s_par, &s_bad, tid, kTcThreads);
    cp_async_wait<1>();   // Q and K have landed (the prefix block may still be in flight)
    fence_proxy_async();  // the staged operands, for the tensor cores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tmem_base;

    // S = Q K^T
    if (tid == 0) {
        const uint32_t id1 = idesc_bf16(kTcRows, Np), aq = smem_u32(sQ), ak = smem_u32(sK);
        for (int s = 0; s < d / 16; ++s)
            tc_mma(tb, kmajor_desc(aq + 256u * s, d), kmajor_desc(ak + 256u * s, d), id1, s > 0 ? 1u : 0u);
        tc_commit(&bar);
    }
    bool ok = tc_wait(&bar, 0);
    tc_fence_after();

    // this thread's row: masked softmax statistics and the weights P
    const int ml = tid, m = m0 + ml;
    const int hl = m / V, j = m - hl * V;
    const bool live = m < rows && j < n;
    const uint32_t lane_addr = tb + ((uint32_t)(warp * 32) << 16);
    const uint32_t* a = anc + (live ? j : 0) * kMaskWords;
    float mx = -INFINITY;
    for (int c0 = 0; c0 < Np; c0 += 16) {
        float sv[16];
        tc_ld16(lane_addr + (uint32_t)c0, sv);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int i = c0 + q;
            if (live && i < n && ((a[i >> 5] >> (i & 31)) & 1u)) mx = fmaxf(mx, sv[q] * J.scale);
        }
    }
    float sum = 0.0f;
    for (int c0 = 0; c0 < Np; c0 += 16) {
        float sv[16];
        tc_ld16(lane_addr + (uint32_t)c0, sv);
        uint32_t part[3][8];
#pragma unroll
        for (int q = 0; q < 16; q += 2) {
            float pr[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = c0 + q + h;
                pr[h] = (live && i < n && ((a[i >> 5] >> (i & 31)) & 1u)) ? expf(sv[q + h] * J.scale - mx) : 0.0f;
                sum += pr[h];
            }
            // three bf16 parts of each weight
            float r0 = pr[0], r1 = pr[1];
#pragma unroll
            for (int t = 0; t < 3; ++t) {
                const uint32_t b0 = bf16_bits(r0), b1 = bf16_bits(r1);
                part[t][q >> 1] = b0 | (b1 << 16);
                r0 -= __uint_as_float(b0 << 16);
                r1 -= __uint_as_float(b1 << 16);
            }
        }
#pragma unroll
        for (int t = 0; t < 3; ++t) {
            unsigned char* base = sP + (size_t)t * kTcRows * Np * 2;
            *reinterpret_cast<uint4*>(base + kmajor_off(ml, c0, Np)) =
                make_uint4(part[t][0], part[t][1], part[t][2], part[t][3]);
            *reinterpret_cast<uint4*>(base + kmajor_off(ml, c0 + 8, Np)) =
                make_uint4(part[t][4], part[t][5], part[t][6], part[t][7]);
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // O = P V, three accumulating parts
    if (tid == 0) {
        const uint32_t id2 = idesc_bf16(kTcRows, d), av = smem_u32(sVt);
        uint32_t acc = 0u;
        for (int t = 0; t < 3; ++t) {
            const uint32_t ap = smem_u32(sP + (size_t)t * kTcRows * Np * 2);
            for (int s = 0; s < Np / 16; ++s) {
                tc_mma(tb + kTcColO, kmajor_desc(ap + 256u * s, Np), kmajor_desc(av + 256u * s, Np), id2, acc);
                acc = 1u;
            }
        }
        tc_commit(&bar);
    }
    ok = tc_wait(&bar, 1) && ok;
    tc_fence_after();

    // epilogue: the suffix state merged with the prefix state.  The operand
    // area is free now; O goes through it in blocks of cb columns so that the
    // prefix reads and the output writes are whole rows per warp.
    __shared__ float s_c1[kTcRows], s_c2[kTcRows];
    __shared__ long long s_row[kTcRows];  // output row, -1: none; -2 - row: a node past num_nodes
    {
        const size_t orow = ((size_t)r * V + j) * J.H + (size_t)g * G + hl;
        float c1 = 0.0f, c2 = 0.0f;
        if (live) {
            const float lse_s = mx + logf(sum);
            const float lp = J.lse_prefix[orow];
            const bool has_prefix = lp != -INFINITY;
            const float M = has_prefix ? fmaxf(lp, lse_s) : lse_s;
            const float w1 = has_prefix ? expf(lp - M) : 0.0f;
            const float w2 = expf(lse_s - M);
            const float inv = 1.0f / (w1 + w2);
            c1 = w1 * inv;
            c2 = w2 * inv / sum;
            J.out_lse[orow] = M + logf(w1 + w2);
        } else if (m < rows) {
            J.out_lse[orow] = -INFINITY;  // a node past num_nodes
        }
        s_c1[ml] = c1;
        s_c2[ml] = c2;
        s_row[ml] = live ? (long long)orow : (m < rows ? -2 - (long long)orow : -1);
    }
    const int ld = cb + 4;
    float* sO = reinterpret_cast<float*>(sm);  // [128][cb + 4]
    for (int b0 = 0; b0 < d; b0 += cb) {
        tc_fence_before();
        __syncthreads();  // the operands (first block) or the previous block are consumed
        if (b0 > 0) prefetch(b0);  // its copies land while O leaves the tensor memory
        for (int c0 = 0; c0 < cb; c0 += 16) {
            float ov[16];
            tc_ld16(lane_addr + kTcColO + (uint32_t)(b0 + c0), ov);
            const float c2 = s_c2[ml];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<float4*>(sO + (size_t)ml * ld + c0 + 4 * q) =
                    make_float4(ov[4 * q] * c2, ov[4 * q + 1] * c2, ov[4 * q + 2] * c2, ov[4 * q + 3] * c2);
        }
        cp_async_wait<0>();
        __syncthreads();
        const int f4 = cb >> 2;
        for (int e0 = tid; e0 < kTcRows * f4; e0 += kTcThreads * 4) {
            float4 pv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * kTcThreads, row = e / f4, c4 = e - row * f4;
                pv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (e < kTcRows * f4 && s_row[row] >= 0 && s_c1[row] != 0.0f)
                    pv[u] = *reinterpret_cast<const float4*>(sPre + (size_t)row * cb + 4 * c4);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * kTcThreads, row = e / f4, c4 = e - row * f4;
                if (e >= kTcRows * f4 || s_row[row] == -1) continue;
                float4* out;
                float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
                if (s_row[row] >= 0) {
                    const float c1 = s_c1[row];
                    const float4 sv = *reinterpret_cast<const float4*>(sO + (size_t)row * ld + 4 * c4);
                    o = make_float4(c1 * pv[u].x + sv.x, c1 * pv[u].y + sv.y, c1 * pv[u].z + sv.z,
                                    c1 * pv[u].w + sv.w);
                    out = reinterpret_cast<float4*>(J.out_o + (size_t)s_row[row] * d + b0) + c4;
                } else {
                    out = reinterpret_cast<float4*>(J.out_o + (size_t)(-2 - s_row[row]) * d + b0) + c4;
                }
                *out = o;
            }
        }
    }
    if (tid == 0 && g == 0 && blockIdx.z == 0 && J.out_flags != nullptr)
        J.out_flags[r] = (s_bad ? UNO_FLAG_BAD_TREE : 0u) | (ok ? 0u : UNO_FLAG_TIMEOUT);
    if (!ok) tc_wait(&bar, 1);  // a second bounded wait before the TMEM is freed
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tb), "r"(ncols) : "memory");
}

}  // namespace uno_sa

extern "C" uno_status uno_tree_suffix_attention_merge(const void* q, const void* k, const void* v, uno_dtype dt,
                                                      int32_t R, int32_t V, int32_t H, int32_t Hkv, int32_t d,
                                                      float scale, const int32_t* node_parent,
                                                      const int32_t* num_nodes, const float* o_prefix,
                                                      const float* lse_prefix, float* out_o, float* out_lse,
                                                      uint32_t* out_flags, void* stream) {
    using namespace uno_sa;
    if (!q || !k || !v || !node_parent || !num_nodes || !o_prefix || !lse_prefix || !out_o || !out_lse)
        return UNO_ERR_INVALID_ARG;
    if (R <= 0 || V <= 0 || H <= 0 || Hkv <= 0 || d <= 0) return UNO_ERR_INVALID_ARG;
    if (V > UNO_MAX_TREE_NODES || H % Hkv != 0 || Hkv > 65535) return UNO_ERR_INVALID_ARG;
    if (dt != UNO_F32 && dt != UNO_BF16) return UNO_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return UNO_ERR_INVALID_ARG;
    const size_t esz = dt == UNO_F32 ? 4 : 2;
    auto aligned = [](const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; };
    if (!aligned(q, esz) || !aligned(k, esz) || !aligned(v, esz)) return UNO_ERR_INVALID_ARG;
    if (!aligned(o_prefix, 4) || !aligned(lse_prefix, 4) || !aligned(out_o, 4) || !aligned(out_lse, 4) ||
        !aligned(node_parent, 4) || !aligned(num_nodes, 4) || (out_flags && !aligned(out_flags, 4)))
        return UNO_ERR_INVALID_ARG;
    if (d > kMaxD) return UNO_ERR_UNSUPPORTED;
    // bf16 rows with d a multiple of 16 take the tensor cores; the rest the
    // CUDA-core kernel.  The tensor-core kernel moves q, k, v, o_prefix and
    // out_o 16 bytes at a time (rows of d a multiple of 16 keep that
    // alignment), so arrays that start off a 16-byte boundary go to the
    // CUDA-core kernel, which reads and writes single elements.
    const size_t tc_smem = tc_smem_bytes(V, d);
    const bool tc = dt == UNO_BF16 && d % 16 == 0 && tc_smem <= 220 * 1024 && aligned(q, 16) && aligned(k, 16) &&
                    aligned(v, 16) && aligned(o_prefix, 16) && aligned(out_o, 16);
    const size_t smem = ((size_t)2 * V * (d + 1) + (size_t)kWarps * d) * 4 + (size_t)V * kMaskWords * 4;
    if (!tc && smem > 227 * 1024) return UNO_ERR_UNSUPPORTED;
    Job J{};
    J.q = q;
    J.k = k;
    J.v = v;
    J.bf16 = dt == UNO_BF16 ? 1 : 0;
    J.R = R;
    J.V = V;
    J.H = H;
    J.Hkv = Hkv;
    J.d = d;
    J.G = H / Hkv;
    J.scale = scale;
    J.parent = node_parent;
    J.num_nodes = num_nodes;
    J.o_prefix = o_prefix;
    J.lse_prefix = lse_prefix;
    J.out_o = out_o;
    J.out_lse = out_lse;
    J.out_flags = out_flags;
    if (tc) {
        if (tc_smem > 48 * 1024 &&
            cudaFuncSetAttribute(suffix_attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tc_smem) != cudaSuccess)
            return UNO_ERR_CUDA;
        const int tiles = (J.G * V + kTcRows - 1) / kTcRows;
        suffix_attention_tc_kernel<<<dim3((unsigned)R, (unsigned)Hkv, (unsigned)tiles), kTcThreads, tc_smem,
                                     static_cast<cudaStream_t>(stream)>>>(J);
        return cudaGetLastError() == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
    }
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(suffix_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
        return UNO_ERR_CUDA;
    suffix_attention_kernel<<<dim3((unsigned)R, (unsigned)Hkv), 32 * kWarps, smem,
                              static_cast<cudaStream_t>(stream)>>>(J);
    return cudaGetLastError() == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}
