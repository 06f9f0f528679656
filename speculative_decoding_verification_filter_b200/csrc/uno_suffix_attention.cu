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

__global__ void __launch_bounds__(32 * kWarps) suffix_attention_kernel(const __grid_constant__ Job J) {
    extern __shared__ float smem[];
    const int r = blockIdx.x, g = blockIdx.y;
    const int V = J.V, d = J.d, ld = d + 1;
    float* sk = smem;                                                    // [V][d + 1]
    float* sv = sk + (size_t)V * ld;                                     // [V][d + 1]
    float* sq = sv + (size_t)V * ld;                                     // [kWarps][d]
    uint32_t* anc = reinterpret_cast<uint32_t*>(sq + (size_t)kWarps * d);  // [V][kMaskWords]
    __shared__ int s_bad;

    int n = J.num_nodes[r];
    n = n < 1 ? 1 : (n > V ? V : n);

    for (int e = threadIdx.x; e < n * d; e += blockDim.x) {
        const int i = e / d, t = e - i * d;
        const size_t src = (((size_t)r * V + i) * J.Hkv + g) * d + t;
        sk[i * ld + t] = load_elem(J.k, J.bf16, src);
        sv[i * ld + t] = load_elem(J.v, J.bf16, src);
    }
    if (threadIdx.x == 0) {
        // ancestors in node order: a parent precedes its child
        const int32_t* par = J.parent + (size_t)r * V;
        int bad = 0;
        for (int j = 0; j < n; ++j) {
            const int p = par[j];
            const bool ok = j == 0 ? p == -1 : (p >= 0 && p < j);
            uint32_t* a = anc + j * kMaskWords;
            for (int w = 0; w < kMaskWords; ++w) a[w] = (ok && j > 0) ? anc[p * kMaskWords + w] : 0u;
            a[j >> 5] |= 1u << (j & 31);
            bad |= ok ? 0 : 1;
        }
        s_bad = bad;
    }
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
    const size_t smem = ((size_t)2 * V * (d + 1) + (size_t)kWarps * d) * 4 + (size_t)V * kMaskWords * 4;
    if (smem > 227 * 1024) return UNO_ERR_UNSUPPORTED;
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
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(suffix_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
        return UNO_ERR_CUDA;
    suffix_attention_kernel<<<dim3((unsigned)R, (unsigned)Hkv), 32 * kWarps, smem,
                              static_cast<cudaStream_t>(stream)>>>(J);
    return cudaGetLastError() == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}
