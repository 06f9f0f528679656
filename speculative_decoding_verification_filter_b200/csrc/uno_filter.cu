// uno_filter.cu -- libuno_filter: UNO's per-cycle sampling and verification
// step on sm_100a, behind the C ABI of include/uno_filter.h.
//
// Hot path.  Every entry point that reads logits runs one row kernel: a CTA
// (or `S` CTAs, for few rows) streams one row of vocabulary logits from HBM
// exactly once with 16-byte non-allocating loads, keeps only the elements that
// can still be among the row's top_k (a per-warp candidate buffer in shared
// memory behind a threshold the warps share), and finishes the row with an
// exact top-k select, a double-precision softmax over the kept support, the
// top-p cut and renormalisation, and then, depending on the entry point:
//   * filter:  write the compact row (and the dense row / one draw);
//   * linear:  write the compact target row to the workspace; the last CTA of
//              a request runs the request's accept / residual / bonus steps;
//   * tree:    the same, the last CTA walks the request's tree.
// No tensor cores: nothing on this path is a contraction.  The filter order
// (top-k, renormalise, then top-p) follows the UNO PR page's review thread;
// the verification rules follow its "Motivation" and "Modifications"
// sections (see include/uno_filter.h for the full statement).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <climits>
#include <cmath>
#include <cstddef>
#include <mutex>

#include "uno_filter.h"
#include "uno_device.cuh"

namespace uno {

enum Mode { kModeFilter = 0, kModeLinear = 1, kModeTree = 2, kModeCycle = 3 };


struct RowJob {
    // logits and shape
    const unsigned char* logits;
    int64_t rows, vocab, row_stride;  // row_stride in elements
    int32_t rpr;                      // rows per request
    int32_t S;                        // CTAs per row
    // sampling parameters
    float temperature, top_p;
    int32_t k;                        // min(top_k, vocab); with per-request parameters, min(top_k_max, vocab)
    // per-request sampling parameters (nullable: the scalars above apply)
    const float* rq_T;
    const int32_t* rq_k;
    const float* rq_p;
    int32_t joint;                    // 1: the top-p cut on the full-vocabulary softmax
    double2* row_ms;                  // joint order: per row, (largest finite logit, sum of exp)
    int32_t hw, cap_w;                // warp buffer high-water mark / capacity
    int32_t merge_cap;                // entries of the merge area
    int32_t fin_off;                  // shared-memory offset of the finishing area (0: the ring)
    int32_t tail_off, tail_bytes;     // shared-memory scratch of the request tails
    int32_t nst, fin_stride;          // pipelined kernel: ring stages, bytes per finishing warp
    int32_t defer_tails;              // verifiers: the request tails run in tail_kernel afterwards
    // filter outputs
    int32_t* out_ids;
    float* out_probs;
    int32_t* out_count;
    int32_t cap;
    float* out_dense;
    int32_t* out_sample;
    uint32_t* out_flags;
    int32_t has_rng;
    uint64_t seed;
    uint32_t cycle;
    const uint32_t* cycle_word;  // nullable: the cycle word, read from device memory at run time
    uint32_t first_request;  // global index of request 0 of this call
    // workspace
    uint32_t* row_ticket;
    uint32_t* req_ticket;
    uint64_t* part_keys;   // [rows*S][k]
    int32_t* part_count;   // [rows*S]
    uint32_t* part_flags;  // [rows*S]
    uint64_t* part_spec;   // pipelined kernel: the predicted threshold each piece used
    double2* part_ms;      // pipelined kernel, joint order: each piece's pair (m, s)
    int32_t* redo;         // pipelined kernel: rows each CTA reads again (rows + grid entries)
    uint32_t* dyn;         // pipelined kernel: rows handed out at run time (nullable; see kDyn*)
    uint64_t* hint;        // pipelined kernel: per CTA, the prediction carried to the next call
    int32_t* c_ids;        // [rows][ks]  compact target rows (verifiers)
    float* c_probs;        // [rows][ks]
    int32_t ks;            // their row stride: k rounded up to a multiple of 4 (16-byte rows)
    int32_t* c_count;      // [rows]
    uint32_t* c_flags;     // [rows]
    // a whole cycle in one launch: rows [0, nq2) are draft rows from `logits`
    // (filtered, one proposal drawn each), rows [nq2, rows) target rows from
    // `logits2` (rows past nq2 count from its start)
    const unsigned char* logits2;
    int64_t nq2;
    // linear verification
    int32_t B;
    int32_t sh;                  // 1: the two-pass layout (x_0 untested, target row i-1 tests x_i)
    const uint32_t* q_flags;     // flags of the draft rows (nullable)
    const int32_t* draft_ids;
    const int32_t* q_ids;
    const float* q_probs;
    const int32_t* q_count;
    int32_t q_cap;
    int32_t* out_tokens;
    int32_t* out_accept_len;
    int32_t* out_num_tokens;
    uint32_t* out_req_flags;
    // tree verification
    int32_t V;
    const int32_t* node_token;
    const int32_t* node_parent;
    const int32_t* num_nodes;
    int32_t* out_path_nodes;
};

// The cycle word of the counter-based RNG: the by-value one, or the one in
// device memory when the call gave its address (a captured CUDA graph replays
// the same arguments every cycle; the word it reads there changes).
__device__ __forceinline__ uint32_t cycle_of(const RowJob& J) {
    return J.cycle_word != nullptr ? __ldg(J.cycle_word) : J.cycle;
}

// The request a row belongs to: a cycle's draft rows come B per request,
// its target rows B + 1 (generic layout) or B (two-pass layout) per request.
template <int MODE>
__device__ __forceinline__ int32_t request_of(const RowJob& J, int64_t row) {
    if (MODE == kModeCycle)
        return (int32_t)(row < J.nq2 ? row / J.B : (row - J.nq2) / (J.B + 1 - J.sh));
    return (int32_t)(row / J.rpr);
}

// A row's sampling parameters: the call's scalars, or its request's entries
// of the per-request arrays.  Entries outside the valid ranges (or a top_k
// above the call's bound) make `ok` false.
struct RowParams {
    float T, p;
    int k;
    bool ok;
};
template <int MODE>
__device__ __forceinline__ RowParams row_params(const RowJob& J, int64_t row) {
    RowParams r{J.temperature, J.top_p, J.k, true};
    if (J.rq_T != nullptr) {
        const int32_t q = request_of<MODE>(J, row);
        r.T = J.rq_T[q];
        r.p = J.rq_p[q];
        const int32_t kq = J.rq_k[q];
        const int64_t kv = (int64_t)kq < J.vocab ? (int64_t)kq : J.vocab;
        r.ok = r.T >= 0.0f && r.T < __int_as_float(0x7f800000) && kq >= 1 && r.p > 0.0f && r.p <= 1.0f &&
               kv <= (int64_t)J.k;
        r.k = kv < 1 ? 1 : (kv > J.k ? J.k : (int)kv);
    }
    return r;
}

// The joint order's normaliser is carried as a pair (m, s): a running
// maximum m of the row's finite logits and s = sum of 2^((l - m) * c) over
// them, c = log2(e) / T.  The exponent (l - m) * c is formed with c split
// into two floats (hi + lo), so that the rounding of c does not bias every
// term alike.
struct JointScale {
    float hi, lo;
};
__device__ __forceinline__ JointScale joint_scale(float T) {
    const double c = 1.4426950408889634 / (double)T;  // log2(e) / T
    JointScale k;
    k.hi = (float)c;
    k.lo = (float)(c - (double)k.hi);
    return k;
}
__device__ __forceinline__ float joint_term(float v, float m, JointScale c) {
    const float d = v - m;
    return exp2f(fmaf(d, c.hi, d * c.lo));
}
// The same term from the hardware base-2 exponential (PTX ex2.approx.ftz:
// relative error about 2^-22; results below 2^-126 flush to zero, which
// leaves a row's sum unchanged at float precision).
__device__ __forceinline__ float joint_term_fast(float v, float m, JointScale c) {
    const float d = v - m;
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(fmaf(d, c.hi, d * c.lo)));
    return y;
}
// (m, s) with s relative to m: raise m to at least x, rescaling s
__device__ __forceinline__ void joint_raise(float& m, double& s, float x, JointScale c) {
    if (x > m) {
        const double d = (double)m - (double)x;
        s *= exp2(d * ((double)c.hi + (double)c.lo));
        m = x;
    }
}
__device__ __forceinline__ void joint_merge(float& m, double& s, float m2, double s2, JointScale c) {
    const float M = m > m2 ? m : m2;
    const double cc = (double)c.hi + (double)c.lo;
    s = s * exp2(((double)m - (double)M) * cc) + s2 * exp2(((double)m2 - (double)M) * cc);
    m = M;
}

// ---------------------------------------------------------------------------
// Element traits.  A lane examines 16-byte units (8 bf16 or 4 fp32), four
// per ring stage.
// ---------------------------------------------------------------------------
constexpr int kUnits = 4;  // 16-byte units per lane per stage

template <typename T>
struct Elem;

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kPerUnit = 8;
    static constexpr int kBytes = 2;
    typedef __nv_bfloat162 Tau;
    __device__ static Tau make_tau(float t) {
        const __nv_bfloat16 b = __float2bfloat16_rd(t);  // largest bf16 <= t
        return __halves2bfloat162(b, b);
    }
    __device__ static __nv_bfloat162 w2(uint32_t w) { return *reinterpret_cast<const __nv_bfloat162*>(&w); }
    // elementwise maximum of a unit (NaN propagates)
    __device__ static __nv_bfloat162 umax(const uint4& r) {
        return __hmax2_nan(__hmax2_nan(w2(r.x), w2(r.y)), __hmax2_nan(w2(r.z), w2(r.w)));
    }
    // true when some element of the unit may be >= tau, or is NaN
    __device__ static bool maybe(const uint4& r, Tau tau) { return !__hblt2(umax(r), tau); }
    __device__ static float get(const uint4& r, int e) {
        const uint32_t w = (e < 2) ? r.x : (e < 4) ? r.y : (e < 6) ? r.z : r.w;
        return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
    }
    // bit e set when element e is finite and >= t; *bad when some element is NaN or +inf
    __device__ static uint32_t elem_mask(const uint4& r, float t, uint32_t& bad) {
        uint32_t m = 0;
#pragma unroll
        for (int e = 0; e < kPerUnit; ++e) {
            const float v = get(r, e);
            const bool nonfinite = (v != v) || v == __int_as_float(0x7f800000);
            bad |= nonfinite ? 1u : 0u;
            m |= (!nonfinite && v >= t && v != -__int_as_float(0x7f800000)) ? (1u << e) : 0u;
        }
        return m;
    }
    __device__ static float load_scalar(const unsigned char* p) {
        const uint16_t h = *reinterpret_cast<const uint16_t*>(p);
        return __uint_as_float((uint32_t)h << 16);
    }
    __device__ static uint4 neg_inf_unit() { return make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u); }
    // Running top-2 of a lane's elements (per bf16x2 half); NaN is skipped
    // by the min/max, the -inf fill never counts, and +inf only arises in a
    // row that is flagged non-finite anyway.
    typedef __nv_bfloat162 Top;
    __device__ static Top top_init() {
        const __nv_bfloat16 ninf = __ushort_as_bfloat16((unsigned short)0xff80u);
        return __halves2bfloat162(ninf, ninf);
    }
    // running maximum of a unit's elements (NaN skipped)
    __device__ static void max_update(Top& m1, const uint4& r) {
        m1 = __hmax2(__hmax2(m1, __hmax2(w2(r.x), w2(r.y))), __hmax2(w2(r.z), w2(r.w)));
    }
    __device__ static uint32_t lane_max_ord(Top m1) {
        const float f = fmaxf(__low2float(m1), __high2float(m1));
        return (f > -__int_as_float(0x7f800000)) ? ord_of_float(__fadd_rn(f, 0.0f)) : 0u;
    }
    __device__ static void top2_update(Top& m1, Top& m2, const uint4* c) {
#pragma unroll
        for (int u = 0; u < kUnits; ++u) {
            const uint32_t w[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const __nv_bfloat162 x = w2(w[q]);
                const __nv_bfloat162 t = __hmin2(m1, x);
                m1 = __hmax2(m1, x);
                m2 = __hmax2(m2, t);
            }
        }
    }
    // ordered bits of the lane's two largest tracked elements (0 = none)
    __device__ static void lane_top2_ord(Top m1, Top m2, uint32_t& t1, uint32_t& t2) {
        const float a1 = __low2float(m1), b1 = __high2float(m1), a2 = __low2float(m2), b2 = __high2float(m2);
        const float first = fmaxf(a1, b1);
        const float second = fmaxf(fminf(a1, b1), fmaxf(a2, b2));
        t1 = (first > -__int_as_float(0x7f800000)) ? ord_of_float(__fadd_rn(first, 0.0f)) : 0u;
        t2 = (second > -__int_as_float(0x7f800000)) ? ord_of_float(__fadd_rn(second, 0.0f)) : 0u;
    }
    // bit u*8+e set when element e of unit u is >= tau (rounded down) or NaN
    __device__ static unsigned cand_mask4(const uint4* c, Tau tau) {
        unsigned m = 0;
#pragma unroll
        for (int u = 0; u < kUnits; ++u) {
            if (maybe(c[u], tau)) {
                const uint32_t w[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const unsigned g = __hgeu2_mask(w2(w[q]), tau);
                    m |= ((g & 1u) | ((g >> 15) & 2u)) << (u * 8 + 2 * q);
                }
            }
        }
        return m;
    }
};

template <>
struct Elem<float> {
    static constexpr int kPerUnit = 4;
    static constexpr int kBytes = 4;
    typedef float Tau;
    __device__ static Tau make_tau(float t) { return t; }
    __device__ static float max_nan(float a, float b) {
        float r;
        asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
        return r;
    }
    __device__ static float umax(const uint4& r) {
        return max_nan(max_nan(__uint_as_float(r.x), __uint_as_float(r.y)),
                       max_nan(__uint_as_float(r.z), __uint_as_float(r.w)));
    }
    __device__ static bool maybe(const uint4& r, Tau tau) { return !(umax(r) < tau); }
    __device__ static float get(const uint4& r, int e) {
        const uint32_t w = (e == 0) ? r.x : (e == 1) ? r.y : (e == 2) ? r.z : r.w;
        return __uint_as_float(w);
    }
    __device__ static uint32_t elem_mask(const uint4& r, float t, uint32_t& bad) {
        uint32_t m = 0;
#pragma unroll
        for (int e = 0; e < kPerUnit; ++e) {
            const float v = get(r, e);
            const bool nonfinite = (v != v) || v == __int_as_float(0x7f800000);
            bad |= nonfinite ? 1u : 0u;
            m |= (!nonfinite && v >= t && v != -__int_as_float(0x7f800000)) ? (1u << e) : 0u;
        }
        return m;
    }
    __device__ static float load_scalar(const unsigned char* p) { return *reinterpret_cast<const float*>(p); }
    __device__ static uint4 neg_inf_unit() { return make_uint4(0xff800000u, 0xff800000u, 0xff800000u, 0xff800000u); }
    typedef float Top;
    __device__ static Top top_init() { return -__int_as_float(0x7f800000); }
    __device__ static void max_update(Top& m1, const uint4& r) {
        m1 = fmaxf(fmaxf(m1, fmaxf(__uint_as_float(r.x), __uint_as_float(r.y))),
                   fmaxf(__uint_as_float(r.z), __uint_as_float(r.w)));
    }
    __device__ static uint32_t lane_max_ord(Top m1) {
        return (m1 > -__int_as_float(0x7f800000)) ? ord_of_float(__fadd_rn(m1, 0.0f)) : 0u;
    }
    __device__ static void top2_update(Top& m1, Top& m2, const uint4* c) {
#pragma unroll
        for (int u = 0; u < kUnits; ++u) {
            const float x[4] = {__uint_as_float(c[u].x), __uint_as_float(c[u].y), __uint_as_float(c[u].z),
                                __uint_as_float(c[u].w)};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float t = fminf(m1, x[q]);
                m1 = fmaxf(m1, x[q]);
                m2 = fmaxf(m2, t);
            }
        }
    }
    __device__ static void lane_top2_ord(Top m1, Top m2, uint32_t& t1, uint32_t& t2) {
        t1 = (m1 > -__int_as_float(0x7f800000)) ? ord_of_float(__fadd_rn(m1, 0.0f)) : 0u;
        t2 = (m2 > -__int_as_float(0x7f800000)) ? ord_of_float(__fadd_rn(m2, 0.0f)) : 0u;
    }
    // bit u*4+e set when element e of unit u is >= tau or NaN
    __device__ static unsigned cand_mask4(const uint4* c, Tau tau) {
        unsigned m = 0;
#pragma unroll
        for (int u = 0; u < kUnits; ++u) {
            const float x[4] = {__uint_as_float(c[u].x), __uint_as_float(c[u].y), __uint_as_float(c[u].z),
                                __uint_as_float(c[u].w)};
#pragma unroll
            for (int q = 0; q < 4; ++q) m |= (!(x[q] < tau) ? 1u : 0u) << (u * 4 + q);
        }
        return m;
    }
};


// Per-warp streaming state.  Candidates are appended by single lanes with a
// shared-memory counter (*wcnt); cnt is the warp-uniform copy of it.
struct WarpState {
    uint64_t* buf;    // candidate keys (shared memory)
    int* wcnt;        // this warp's candidate count (shared memory)
    int cnt;          // warp-uniform copy of *wcnt
    uint64_t tau;     // threshold key (warp-uniform): every key < tau is out
    uint32_t bad;     // this lane saw NaN / +inf
};

struct Compacted {
    int cnt;
    uint64_t tau;
};

// Drop candidates below the threshold, cut to the k best if more remain, and
// publish the threshold to the CTA.  Every threshold a warp holds is a lower
// bound of the CTA's k-th best key, so dropping below it loses nothing.
// Rare; kept out of line so the streaming loop stays small.
__device__ __noinline__ Compacted warp_compact(uint64_t* buf, int* wcnt, int cnt, uint64_t tau, int k,
                                               unsigned long long* s_tau, int lane) {
    cnt = warp_keep_ge(buf, cnt, tau, lane);
    if (cnt > k) {
        const uint64_t t = warp_select_kth(buf, cnt, k, lane);
        cnt = warp_keep_ge(buf, cnt, t, lane);
        if (t > tau) tau = t;
        if (lane == 0) atomicMax(s_tau, (unsigned long long)tau);
    }
    if (lane == 0) *wcnt = cnt;
    __syncwarp();
    return Compacted{cnt, tau};
}

// Geometry of a row: `head` scalar elements up to the first 16-byte boundary,
// then nunit aligned 16-byte units, then the tail.
struct RowGeom {
    const unsigned char* base;  // first element of the row
    int64_t head, nunit, tail_begin;
};

template <typename T>
__device__ __forceinline__ RowGeom row_geom(const RowJob& J, int64_t row) {
    RowGeom g;
    g.base = (J.logits2 == nullptr || row < J.nq2)
                 ? J.logits + (size_t)row * (size_t)J.row_stride * Elem<T>::kBytes
                 : J.logits2 + (size_t)(row - J.nq2) * (size_t)J.row_stride * Elem<T>::kBytes;
    const uintptr_t addr = reinterpret_cast<uintptr_t>(g.base);
    int64_t head = (int64_t)(((16u - (addr & 15u)) & 15u) / Elem<T>::kBytes);
    if (head > J.vocab) head = J.vocab;
    g.head = head;
    g.nunit = (J.vocab - head) / Elem<T>::kPerUnit;
    g.tail_begin = head + g.nunit * Elem<T>::kPerUnit;
    return g;
}


// Element j (0 .. kUnits*kPerUnit-1) of a lane's units, j not known at compile time.
template <typename T>
__device__ __forceinline__ float lane_elem(const uint4* c, int j) {
    const int u = j / Elem<T>::kPerUnit;
    const uint4 r = (u == 0) ? c[0] : (u == 1) ? c[1] : (u == 2) ? c[2] : c[3];
    const int e = j % Elem<T>::kPerUnit;
    if (Elem<T>::kBytes == 2) {
        const int q = e >> 1;
        const uint32_t w = (q == 0) ? r.x : (q == 1) ? r.y : (q == 2) ? r.z : r.w;
        return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
    }
    const uint32_t w = (e == 0) ? r.x : (e == 1) ? r.y : (e == 2) ? r.z : r.w;
    return __uint_as_float(w);
}

// Streaming ring of the CTA.  A stage is kStageBytes of consecutive logits,
// brought in by ONE bulk copy (TMA, no multicast) with an mbarrier tracking
// its bytes.  Warp w owns bytes [w*2KB, (w+1)*2KB) of a stage: four rows of
// 32 16-byte units, lane l taking unit l of each row (conflict-free shared
// loads).  The last warp to finish with a stage refills it (a shared-memory
// arrival counter: no warp ever waits for another to release a stage).
constexpr int kStages = 2;
constexpr int kStageBytes = 16384;
constexpr int kStageUnits = kStageBytes / 16;         // 16-byte units per stage
constexpr int kWarpUnits = kStageUnits / kWarps;      // 128 per warp per stage
constexpr int kRowsPerWarp = kWarpUnits / 32;         // 4 = kUnits
static_assert(kRowsPerWarp == kUnits, "one unit per lane per row");
// Stages whose elements seed the CTA threshold; the CTA reads them twice
// (seed, then select), the second time from L2.
constexpr int kBootStages = 4;
// Elements per lane handled at a time when a burst of candidates arrives.
constexpr int kPiece = 4;

struct Ring {
    unsigned char* stages;  // [kStages][kStageBytes]
    uint64_t* full;         // [kStages] mbarriers (bytes arrived)
    int* done;              // [kStages] warps finished with the stage
    const unsigned char* ubase;
    int ub, ue;             // the CTA's 16-byte units
    int nA, total;          // sequence: nA seed stages, then every stage
};

__device__ __forceinline__ int ring_stage_index(const Ring& R, int q) { return q < R.nA ? q : q - R.nA; }

// one thread: start copying sequence element q into its stage buffer
__device__ __forceinline__ void ring_issue(const Ring& R, int q) {
    const int u0 = R.ub + ring_stage_index(R, q) * kStageUnits;
    const int nu = (R.ue - u0) < kStageUnits ? (R.ue - u0) : kStageUnits;
    const uint32_t bytes = (uint32_t)nu * 16u;
    uint64_t* bar = R.full + (q % kStages);
    mbar_expect_tx(bar, bytes);
    bulk_g2s(R.stages + (q % kStages) * kStageBytes, R.ubase + (size_t)u0 * 16, bytes, bar);
}

// Wait for sequence element q and load this warp's lane units (the -inf fill
// past the end of the slice).  Returns false if the wait gave up.
template <typename T>
__device__ __forceinline__ bool ring_take(const Ring& R, int q, int warp, int lane, uint4* c) {
    uint64_t* bar = R.full + (q % kStages);
    const uint32_t par = (uint32_t)((q / kStages) & 1);
    uint32_t got = 0;  // lane 0 polls; the warp learns the outcome
    if (lane == 0) got = (mbar_try_wait(bar, par) || mbar_wait_bounded(bar, par)) ? 1u : 0u;
    const bool ok = __shfl_sync(kFull, got, 0) != 0;
    const int u0 = R.ub + ring_stage_index(R, q) * kStageUnits + warp * kWarpUnits + lane;
    const uint4* sp = reinterpret_cast<const uint4*>(R.stages + (q % kStages) * kStageBytes) + warp * kWarpUnits + lane;
#pragma unroll
    for (int u = 0; u < kUnits; ++u) c[u] = (ok && u0 + u * 32 < R.ue) ? sp[u * 32] : Elem<T>::neg_inf_unit();
    return ok;
}

// After every lane of the warp has used its units (its shared loads are
// complete): count the warp out of the stage; the last warp refills it.
__device__ __forceinline__ void ring_release(const Ring& R, int q, int lane) {
    __syncwarp();
    if (lane == 0) {
        int* d = R.done + (q % kStages);
        if (atomicAdd(d, 1) == kWarps - 1) {
            atomicExch(d, 0);
            if (q + kStages < R.total) ring_issue(R, q + kStages);
        }
    }
}

// After a timeout: wait (bounded) for the copies that may still be in flight.
__device__ __forceinline__ void ring_drain(const Ring& R, int q) {
    for (int d = q; d < R.total && d < q + kStages; ++d)
        (void)mbar_wait_bounded(R.full + (d % kStages), (uint32_t)((d / kStages) & 1));
}

// Element id of bit j of a lane's mask (unit j / kPerUnit, element j % kPerUnit).
template <typename T>
__device__ __forceinline__ uint32_t lane_id(uint32_t uid0, int j) {
    return (uid0 + (uint32_t)(j / Elem<T>::kPerUnit) * 32u) * Elem<T>::kPerUnit + (uint32_t)(j % Elem<T>::kPerUnit);
}

// Append the candidates of mask cm (bit j = element j of the lane's units;
// uid0 = the lane's first unit, relative to element 0 of the row's units).
template <typename T>
__device__ __forceinline__ void append_mask(WarpState& ws, unsigned cm, const uint4* c, uint32_t id_base,
                                            uint32_t uid0) {
    while (cm) {
        const int j = __ffs(cm) - 1;
        cm &= cm - 1;
        const float x = lane_elem<T>(c, j);
        if (x != x || x == __int_as_float(0x7f800000)) {
            ws.bad |= 1u;
        } else if (x != -__int_as_float(0x7f800000)) {
            const uint64_t key = make_key(x, id_base + lane_id<T>(uid0, j));
            if (key > ws.tau) ws.buf[atomicAdd(ws.wcnt, 1)] = key;
        }
    }
}

// Stream this CTA's share of the row: 16-byte units [ub, ue) plus, for split
// 0, the head and tail scalars.  All threads of the CTA call it.  ws.bad gets
// bit 0 for a NaN / +inf logit, bit 1 when a wait gave up.
//
// Phase A (threshold seed): every lane tracks the two largest elements of its
// share of the first kBootStages stages; the k-th largest of those (real,
// distinct) elements is a valid lower bound of the CTA's k-th largest
// (k <= 2*kThreads).
// Phase B (select): every stage again; a lane whose units may hold an element
// >= the threshold (or a NaN) appends its candidates; a warp whose buffer
// passes the high-water mark cuts it to its best k, which raises the
// threshold for the whole CTA.
template <typename T>
__device__ void scan_slice(const RowJob& J, const RowGeom& g, int64_t ub64, int64_t ue64, bool do_scalars,
                           WarpState& ws, unsigned long long* s_tau, const Ring& ring_in, uint64_t* boot, int warp,
                           int lane) {
    typedef typename Elem<T>::Tau Tau;
    constexpr int NE = kUnits * Elem<T>::kPerUnit;  // elements per lane per stage
    Ring R = ring_in;
    R.ubase = g.base + (size_t)g.head * Elem<T>::kBytes;  // 16-byte aligned
    R.ub = (int)ub64;                                     // unit indices fit in 32 bits
    R.ue = (int)ue64;
    const int nstage = (R.ue - R.ub + kStageUnits - 1) / kStageUnits;
    R.nA = nstage < kBootStages ? nstage : kBootStages;
    R.total = R.nA + nstage;
    const uint32_t id_base = (uint32_t)g.head;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(R.full + s, 1);
            R.done[s] = 0;
        }
        fence_mbar_init();
        for (int q = 0; q < kStages && q < R.total; ++q) ring_issue(R, q);
    }
    __syncthreads();

    bool ok = true;
    int q = 0;
    // ---- phase A: seed the threshold
    {
        typename Elem<T>::Top m1 = Elem<T>::top_init(), m2 = m1;
        for (; q < R.nA; ++q) {
            uint4 c[kUnits];
            ok = ring_take<T>(R, q, warp, lane, c);
            if (!ok) break;
            Elem<T>::top2_update(m1, m2, c);
            ring_release(R, q, lane);
        }
        uint32_t t1, t2;
        Elem<T>::lane_top2_ord(m1, m2, t1, t2);
        // the k-th largest lane maximum: at least k (distinct) elements are
        // >= it, so it is a valid lower bound of the CTA's k-th largest
        uint32_t* bv = reinterpret_cast<uint32_t*>(boot);
        bv[threadIdx.x] = t1;  // 0: no element
        __syncthreads();
        if (J.k <= kThreads && t1 > kOrdNegInf) {
            int gt = 0, ge = 0;
            for (int j = 0; j < kThreads; j += 8) {
                const uint4 a = *reinterpret_cast<const uint4*>(bv + j);
                const uint4 b = *reinterpret_cast<const uint4*>(bv + j + 4);
                const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    gt += v[q] > t1;
                    ge += v[q] >= t1;
                }
            }
            if (gt < J.k && J.k <= ge) *s_tau = (uint64_t)t1 << 32;  // every writer holds the same value
        }
        (void)t2;
        __syncthreads();
        ws.tau = *reinterpret_cast<volatile unsigned long long*>(s_tau);
    }

    // row head / tail scalars (split 0, warp 0)
    if (do_scalars && warp == 0) {
        const int64_t ntail = J.vocab - g.tail_begin;
        const int64_t nsc = g.head + ntail;  // < 2 * 8 = 16
        if (lane < nsc) {
            const int64_t id = (lane < g.head) ? (int64_t)lane : g.tail_begin + (lane - g.head);
            const float v = Elem<T>::load_scalar(g.base + (size_t)id * Elem<T>::kBytes);
            if (v != v || v == __int_as_float(0x7f800000)) {
                ws.bad |= 1u;
            } else if (v != -__int_as_float(0x7f800000)) {
                const uint64_t key = make_key(v, (uint32_t)id);
                if (key > ws.tau) ws.buf[atomicAdd(ws.wcnt, 1)] = key;
            }
        }
        __syncwarp();
        ws.cnt = *reinterpret_cast<volatile int*>(ws.wcnt);
    }

    // ---- phase B: select
    Tau tau_v = Elem<T>::make_tau(tau_value(ws.tau));
    float tau_f = tau_value(ws.tau);
    for (; ok && q < R.total; ++q) {
        uint4 c[kUnits];
        ok = ring_take<T>(R, q, warp, lane, c);
        if (!ok) break;
        bool need = false;
#pragma unroll
        for (int u = 0; u < kUnits; ++u) need |= Elem<T>::maybe(c[u], tau_v);
        if (__any_sync(kFull, need)) {
            const uint32_t uid0 = (uint32_t)(R.ub + ring_stage_index(R, q) * kStageUnits + warp * kWarpUnits + lane);
            unsigned cm = need ? Elem<T>::cand_mask4(c, tau_v) : 0u;
            const int nc = (int)__reduce_add_sync(kFull, (unsigned)__popc(cm));
            if (ws.cnt + nc <= J.cap_w) {
                append_mask<T>(ws, cm, c, id_base, uid0);
                __syncwarp();
                ws.cnt = *reinterpret_cast<volatile int*>(ws.wcnt);
            } else {
                // a burst: kPiece elements per lane at a time, compacting between
#pragma unroll 1
                for (int p = 0; p < NE; p += kPiece) {
                    if (ws.cnt > J.hw) {
                        const Compacted cp = warp_compact(ws.buf, ws.wcnt, ws.cnt, ws.tau, J.k, s_tau, lane);
                        ws.cnt = cp.cnt;
                        ws.tau = cp.tau;
                        tau_v = Elem<T>::make_tau(tau_value(ws.tau));
                        tau_f = tau_value(ws.tau);
                    }
                    unsigned pm = 0;
                    for (int e = 0; e < kPiece; ++e) pm |= (!(lane_elem<T>(c, p + e) < tau_f) ? 1u : 0u) << (p + e);
                    append_mask<T>(ws, pm, c, id_base, uid0);
                    __syncwarp();
                    ws.cnt = *reinterpret_cast<volatile int*>(ws.wcnt);
                }
            }
            if (ws.cnt > J.hw) {
                const Compacted cp = warp_compact(ws.buf, ws.wcnt, ws.cnt, ws.tau, J.k, s_tau, lane);
                ws.cnt = cp.cnt;
                ws.tau = cp.tau;
                tau_v = Elem<T>::make_tau(tau_value(ws.tau));
                tau_f = tau_value(ws.tau);
            }
        }
        ring_release(R, q, lane);
        // adopt a better threshold found by another warp of this CTA
        const unsigned long long st = *reinterpret_cast<volatile unsigned long long*>(s_tau);
        if (st > ws.tau) {
            ws.tau = st;
            tau_v = Elem<T>::make_tau(tau_value(ws.tau));
            tau_f = tau_value(ws.tau);
        }
    }
    if (!ok) {
        ring_drain(R, q);
        ws.bad |= 2u;
    }
}

// ---------------------------------------------------------------------------
// Request tails (one warp of the last CTA of a request).
// ---------------------------------------------------------------------------

// Probability of `tok` in a compact row with ascending ids (binary search).
__device__ __forceinline__ double lookup_sorted(const int32_t* ids, const float* probs, int n, int32_t tok) {
    int lo = 0, hi = n - 1;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        const int32_t m = __ldcg(ids + mid);
        if (m == tok) return (double)__ldcg(probs + mid);
        if (m < tok)
            lo = mid + 1;
        else
            hi = mid - 1;
    }
    return 0.0;
}

// A compact row's count as the request tails use it: a value outside [0, k]
// (only a row that was never written holds one) reads as an empty row.
__device__ __forceinline__ int clamp_count(int c, int k) { return (c < 0 || c > k) ? 0 : c; }

// Linear verification of request r from global memory (one warp): any k, any
// B.  Generic layout (sh = 0): target row i tests proposal x_i, row B gives
// the bonus.  Two-pass layout (sh = 1): x_0 is emitted untested, row i - 1
// tests x_i, row B - 1 gives the bonus.
__device__ __noinline__ void linear_tail(const RowJob& J, int32_t r, double* wd, int lane) {
    const int32_t B = J.B;
    const int sh = J.sh;
    const int64_t base = (int64_t)r * (B + 1 - sh);
    uint32_t flags = 0;
    for (int i = lane; i <= B - sh; i += 32) flags |= __ldcg(J.c_flags + base + i);
    if (J.q_flags != nullptr)
        for (int i = lane; i < B; i += 32) flags |= __ldcg(J.q_flags + (int64_t)r * B + i);
    flags = __reduce_or_sync(kFull, flags);
    int32_t acc = B, ntok = B + 1;
    int32_t* toks = J.out_tokens + (size_t)r * (B + 1);
    for (int i = lane; i <= B; i += 32) toks[i] = -1;
    __syncwarp();
    bool stopped = false;
    if (sh == 1) {
        // the base-weights token, untested
        if (__ldcg(J.q_count + (int64_t)r * B) > 0) {
            if (lane == 0) toks[0] = __ldcg(J.draft_ids + (size_t)r * B);
        } else {
            acc = 0;
            ntok = 0;
            stopped = true;
        }
    }
    for (int i = sh; i < B && !stopped; ++i) {
        const int pc = clamp_count(__ldcg(J.c_count + base + i - sh), J.k);
        const int32_t* pid = J.c_ids + (size_t)(base + i - sh) * J.ks;
        const float* ppr = J.c_probs + (size_t)(base + i - sh) * J.ks;
        if (pc == 0) {
            acc = i;
            ntok = i;
            stopped = true;
            break;
        }
        const int64_t qrow = (int64_t)r * B + i;
        int qc = __ldcg(J.q_count + qrow);
        qc = qc < 0 ? 0 : (qc > J.q_cap ? J.q_cap : qc);
        const int32_t* qid = J.q_ids + (size_t)qrow * J.q_cap;
        const float* qpr = J.q_probs + (size_t)qrow * J.q_cap;
        const int32_t x = __ldcg(J.draft_ids + (size_t)r * B + i);
        const bool xin = x >= 0 && (int64_t)x < J.vocab;
        const double a = xin ? lookup_sorted(qid, qpr, qc, x) : 0.0;
        const double px = xin ? lookup_sorted(pid, ppr, pc, x) : 0.0;
        bool accept = false;
        if (a > 0.0) {
            const double u = uniform53(J.seed, J.first_request + (uint32_t)r, (uint32_t)i, kDrawAccept, cycle_of(J));
            accept = (u * a < px);
        } else {
            flags |= kFlagDraftNotInSupport;
        }
        if (accept) {
            if (lane == 0) toks[i] = x;
            continue;
        }
        // residual max(0, p - q_i) over supp p (ascending ids)
        for (int j = lane; j < pc; j += 32) {
            const double d = (double)__ldcg(ppr + j) - lookup_sorted(qid, qpr, qc, __ldcg(pid + j));
            wd[j] = d > 0.0 ? d : 0.0;
        }
        __syncwarp();
        int pick = -1;
        if (lane == 0) {
            double tot = 0.0;
            for (int j = 0; j < pc; ++j) tot += wd[j];
            if (!(tot > 0.0)) {
                flags |= kFlagResidualEmpty;
                for (int j = 0; j < pc; ++j) wd[j] = (double)__ldcg(ppr + j);
            }
            const double u = uniform53(J.seed, J.first_request + (uint32_t)r, (uint32_t)i, kDrawResidual, cycle_of(J));
            pick = inv_cdf_serial(wd, pc, u);
            toks[i] = pick >= 0 ? __ldcg(pid + pick) : -1;
        }
        flags = __shfl_sync(kFull, flags, 0);
        __syncwarp();
        acc = i;
        ntok = i + 1;
        stopped = true;
    }
    if (!stopped) {
        const int pc = clamp_count(__ldcg(J.c_count + base + B - sh), J.k);
        if (pc == 0) {
            ntok = B;
        } else if (lane == 0) {
            const int32_t* pid = J.c_ids + (size_t)(base + B - sh) * J.ks;
            const float* ppr = J.c_probs + (size_t)(base + B - sh) * J.ks;
            for (int j = 0; j < pc; ++j) wd[j] = (double)__ldcg(ppr + j);
            const double u = uniform53(J.seed, J.first_request + (uint32_t)r, (uint32_t)B, kDrawTarget, cycle_of(J));
            const int pick = inv_cdf_serial(wd, pc, u);
            toks[B] = pick >= 0 ? __ldcg(pid + pick) : -1;
        }
    }
    if (lane == 0) {
        J.out_accept_len[r] = acc > sh ? acc - sh : 0;
        J.out_num_tokens[r] = ntok;
        J.out_req_flags[r] = flags;
    }
}

__device__ __noinline__ void tree_tail(const RowJob& J, int32_t r, double* wd, int lane) {
    const int32_t B = J.B, V = J.V;
    const int64_t base = (int64_t)r * V;
    int32_t n = J.num_nodes[r];
    n = n < 1 ? 1 : (n > V ? V : n);
    const int32_t* tk = J.node_token + (size_t)r * V;
    const int32_t* pa = J.node_parent + (size_t)r * V;
    uint32_t flags = 0;
    for (int j = lane; j < n; j += 32) flags |= __ldcg(J.c_flags + base + j);
    flags = __reduce_or_sync(kFull, flags);
    int32_t* toks = J.out_tokens + (size_t)r * (B + 1);
    int32_t* path = J.out_path_nodes + (size_t)r * (B + 1);
    for (int t = lane; t <= B; t += 32) {
        toks[t] = -1;
        path[t] = -1;
    }
    __syncwarp();
    int32_t j = 0, t = 0, acc = 0, ntok = 0;
    for (;;) {
        const int pc = clamp_count(__ldcg(J.c_count + base + j), J.k);
        if (pc == 0) {
            if (lane == 0) path[t] = j;
            ntok = t;
            acc = t;
            break;
        }
        int32_t y = -1;
        if (lane == 0) {
            const int32_t* pid = J.c_ids + (size_t)(base + j) * J.ks;
            const float* ppr = J.c_probs + (size_t)(base + j) * J.ks;
            for (int q = 0; q < pc; ++q) wd[q] = (double)__ldcg(ppr + q);
            const double u = uniform53(J.seed, J.first_request + (uint32_t)r, (uint32_t)j, kDrawTarget, cycle_of(J));
            const int pick = inv_cdf_serial(wd, pc, u);
            y = pick >= 0 ? __ldcg(pid + pick) : -1;
            toks[t] = y;
            path[t] = j;
        }
        y = __shfl_sync(kFull, y, 0);
        __syncwarp();
        ++t;
        ntok = t;
        acc = t - 1;
        // the lowest-index child of j carrying token y
        int32_t next = -1;
        for (int c0 = 1; c0 < n && next < 0; c0 += 32) {
            const int c = c0 + lane;
            const bool hit = c < n && pa[c] == j && tk[c] == y;
            const unsigned bal = __ballot_sync(kFull, hit);
            if (bal) next = c0 + __ffs(bal) - 1;
        }
        if (next < 0 || t > B) break;
        j = next;
    }
    if (lane == 0) {
        J.out_accept_len[r] = acc;
        J.out_num_tokens[r] = ntok;
        J.out_req_flags[r] = flags;
    }
}

// ---------------------------------------------------------------------------
// Warp-level finishing for k <= 64: lane l holds ranks l and l + 32.  Sums
// and scans run as warp reductions (a fixed order; it differs from a serial
// sum only in the last bits, which can flip a decision only within the
// boundary margin the library documents).
// ---------------------------------------------------------------------------
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}
__device__ __forceinline__ double warp_incl_scan_d(double v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += t;
    }
    return v;
}
// Ascending bitonic sort of 64 keys, element e = lane in a, e = lane + 32 in b.
// The loops stay rolled: this runs once per row beside the streaming loop,
// and a small body stays in the instruction cache where an unrolled one
// would be fetched cold every time.
__device__ __forceinline__ void warp_sort64(uint64_t& a, uint64_t& b, int lane) {
#pragma unroll 1
    for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll 1
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride == 32) {
                const uint64_t lo = a < b ? a : b, hi = a < b ? b : a;
                a = lo;
                b = hi;
            } else {
                const uint64_t pa = __shfl_xor_sync(kFull, a, stride), pb = __shfl_xor_sync(kFull, b, stride);
                const bool lower = (lane & stride) == 0;
                const bool upa = size == 64 || (lane & size) == 0;
                const bool upb = size == 64 || ((lane + 32) & size) == 0;
                a = (lower == upa) ? (a < pa ? a : pa) : (a < pa ? pa : a);
                b = (lower == upb) ? (b < pb ? b : pb) : (b < pb ? pb : b);
            }
        }
    }
}

// First j (of weights wa at index lane, wb at lane + 32; ascending id order)
// with u * S < prefix_j, else the last positive weight; -1 if all are zero.
__device__ __forceinline__ int warp_inv_cdf(double wa, double wb, double u, int lane) {
    const double S = warp_sum_d(wa + wb);
    if (!(S > 0.0)) return -1;
    const double x = u * S;
    const double ia = warp_incl_scan_d(wa, lane);
    const double ta = __shfl_sync(kFull, ia, 31);
    const double ib = warp_incl_scan_d(wb, lane) + ta;
    const unsigned ba = __ballot_sync(kFull, x < ia), bb = __ballot_sync(kFull, x < ib);
    if (ba) return __ffs(ba) - 1;
    if (bb) return 32 + __ffs(bb) - 1;
    const unsigned pa = __ballot_sync(kFull, wa > 0.0), pb = __ballot_sync(kFull, wb > 0.0);
    if (pb) return 32 + 31 - __clz(pb);
    if (pa) return 31 - __clz(pa);
    return -1;
}

// ---------------------------------------------------------------------------
// Request tails from shared memory (k <= 64): the last CTA of a request first
// copies the request's compact rows into its idle ring buffer with all
// lanes, then runs the sequential decisions with warp-parallel lookups and
// inverse-CDF draws.  They return false (and the callers fall back to the
// tails above) when the rows do not fit.
// ---------------------------------------------------------------------------


// Probability of token x in a compact row with ascending ids (one lane,
// binary search in shared memory).
__device__ __forceinline__ double smem_lookup(const int32_t* ids, const float* pr, int n, int32_t x) {
    int lo = 0, hi = n - 1;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        const int32_t m = ids[mid];
        if (m == x) return (double)pr[mid];
        if (m < x)
            lo = mid + 1;
        else
            hi = mid - 1;
    }
    return 0.0;
}

// One warp copies rows [0, nrows) x [0, width) of (ids, probs) from global
// memory (row stride gs) into shared arrays (row stride ss).  Loads are
// staged in registers, eight per lane, so that they are all in flight
// together (a shared store between them could alias a later load and
// serialise the round trips).  Entries past a row's count are copied too and
// never read.  CG: through L2 only (rows written by this kernel).
template <bool CG>
__device__ __forceinline__ void warp_copy_rows(const int32_t* gid, const float* gpr, int64_t gs, int nrows, int width,
                                               int32_t* sid, float* spr, int ss, int lane) {
    constexpr int RB = 8;
    const int total = nrows * width;
    for (int b0 = 0; b0 < total; b0 += 32 * RB) {
        int32_t vi[RB];
        float vp[RB];
#pragma unroll
        for (int t = 0; t < RB; ++t) {
            const int idx = b0 + t * 32 + lane;
            if (idx < total) {
                const int i = idx / width, j = idx - i * width;
                const size_t g = (size_t)i * (size_t)gs + (size_t)j;
                vi[t] = CG ? __ldcg(gid + g) : __ldg(gid + g);
                vp[t] = CG ? __ldcg(gpr + g) : __ldg(gpr + g);
            }
        }
#pragma unroll
        for (int t = 0; t < RB; ++t) {
            const int idx = b0 + t * 32 + lane;
            if (idx < total) {
                const int i = idx / width, j = idx - i * width;
                sid[i * ss + j] = vi[t];
                spr[i * ss + j] = vp[t];
            }
        }
    }
}

__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Whole warp: bounded wait for a tail's bulk copies (phase 0 of bar).  Every
// lane waits on the barrier itself, so that every lane sees the copied data.
// On expiry a second bounded wait lets copies in flight land first.
__device__ __forceinline__ bool tail_copies_wait(uint64_t* bar, int lane) {
    bool got = mbar_try_wait(bar, 0) || mbar_wait_bounded(bar, 0);
    const bool ok = __all_sync(kFull, got);
    if (!ok && !got) (void)mbar_wait_bounded(bar, 0);
    __syncwarp();
    if (ok && lane == 0) mbar_inval(bar);
    return ok;
}

// A request's outputs when its tail could not get its rows in time.
__device__ __forceinline__ void tail_timeout(const RowJob& J, int32_t r, int lane) {
    int32_t* toks = J.out_tokens + (size_t)r * (J.B + 1);
    for (int t = lane; t <= J.B; t += 32) toks[t] = -1;
    if (J.out_path_nodes != nullptr)
        for (int t = lane; t <= J.B; t += 32) J.out_path_nodes[(size_t)r * (J.B + 1) + t] = -1;
    if (lane == 0) {
        J.out_accept_len[r] = 0;
        J.out_num_tokens[r] = 0;
        J.out_req_flags[r] = kFlagTimeout;
    }
}

// Bytes of the 16-byte-aligned middle of the byte range [src, src + n).
__device__ __forceinline__ uint32_t range_bulk_bytes(const unsigned char* src, uint32_t n) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(src), a1 = a0 + n;
    const uintptr_t m0 = (a0 + 15u) & ~(uintptr_t)15u, m1 = a1 & ~(uintptr_t)15u;
    return m1 > m0 ? (uint32_t)(m1 - m0) : 0u;
}

// Bring the 4-byte-aligned byte range [src, src + n) of global memory into
// shared memory at dst (the same address modulo 16: dst is a 16-aligned
// region plus src % 16): lane 0 bulk-copies the 16-byte-aligned middle on
// bar (lane 0 has already added range_bulk_bytes to the barrier's expected
// count), lanes 1..6 copy the at most three words at each edge.  Nothing
// outside the range is read.
__device__ __forceinline__ void copy_range_async(unsigned char* dst, const unsigned char* src, uint32_t n,
                                                 uint64_t* bar, int lane) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(src), a1 = a0 + n;
    const uintptr_t m0 = (a0 + 15u) & ~(uintptr_t)15u, m1 = a1 & ~(uintptr_t)15u;
    if (m1 > m0 && lane == 0) bulk_g2s(dst + (m0 - a0), reinterpret_cast<const void*>(m0), (uint32_t)(m1 - m0), bar);
    // edge words: [a0, min(m0, a1)) and [max(m1, m0), a1)
    const uintptr_t h1 = m0 < a1 ? m0 : a1, t0 = m1 > m0 ? m1 : (m0 < a1 ? m0 : a1);
    const int nh = (int)((h1 - a0) / 4), nt = (int)((a1 - t0) / 4);
    if (lane >= 1 && lane <= nh) {
        const uintptr_t a = a0 + 4u * (uintptr_t)(lane - 1);
        *reinterpret_cast<uint32_t*>(dst + (a - a0)) = *reinterpret_cast<const uint32_t*>(a);
    } else if (lane >= 4 && lane < 4 + nt) {
        const uintptr_t a = t0 + 4u * (uintptr_t)(lane - 4);
        *reinterpret_cast<uint32_t*>(dst + (a - a0)) = *reinterpret_cast<const uint32_t*>(a);
    }
}

__device__ __noinline__ bool linear_tail_fast(const RowJob& J, int32_t r, unsigned char* sm, int lane) {
    const int32_t B = J.B;
    const int kc = J.k, ks = J.ks;
    constexpr int QS = 64;  // q entries kept per row
    if (kc > 64 || B > 31) return false;
    const int sh = J.sh;      // 1: two-pass layout (x_0 untested, target row i-1 tests x_i)
    const int P = B + 1 - sh;  // target rows per request
    const size_t need = 16 + (size_t)(B + 1) * ks * 8 + 2 * ((size_t)B * QS * 4 + 16) + (size_t)(4 * B + 2) * 4;
    if (need > (size_t)J.tail_bytes) return false;
    // the draft rows as one byte range per array (stride q_cap) when short
    const bool qflat = J.q_cap <= QS;
    const int qs = qflat ? J.q_cap : QS;
    const uint32_t qn = (uint32_t)B * (uint32_t)J.q_cap * 4u;
    const unsigned char* qsi = reinterpret_cast<const unsigned char*>(J.q_ids + (size_t)r * B * J.q_cap);
    const unsigned char* qsp = reinterpret_cast<const unsigned char*>(J.q_probs + (size_t)r * B * J.q_cap);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm);                              // the copies' mbarrier
    int32_t* pid = reinterpret_cast<int32_t*>(sm + 16);                           // [B+1][ks]
    float* ppr = reinterpret_cast<float*>(pid + (B + 1) * ks);                    // [B+1][ks]
    unsigned char* qreg_i = reinterpret_cast<unsigned char*>(ppr + (B + 1) * ks);  // 16-aligned regions
    unsigned char* qreg_p = qreg_i + ((size_t)B * QS * 4 + 16);
    int32_t* qid = reinterpret_cast<int32_t*>(qflat ? qreg_i + (reinterpret_cast<uintptr_t>(qsi) & 15u) : qreg_i);  // [B][qs]
    float* qpr = reinterpret_cast<float*>(qflat ? qreg_p + (reinterpret_cast<uintptr_t>(qsp) & 15u) : qreg_p);     // [B][qs]
    int32_t* pcnt = reinterpret_cast<int32_t*>(qreg_p + ((size_t)B * QS * 4 + 16));  // [B+1]
    int32_t* qcnt = pcnt + (B + 1);                                                  // [B]
    int32_t* dft = qcnt + B;                                                         // [B]
    int32_t* otok = dft + B;                                                         // [B+1] emitted tokens
    const int64_t base = (int64_t)r * P;
    const uint32_t req = J.first_request + (uint32_t)r;
    // The request's compact target rows and draft rows arrive by bulk copies
    // (TMA) on one mbarrier: one round trip, whatever the memory system's
    // queueing; counts, flags and drafts load alongside.
    if (lane == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        const uint32_t pb = (uint32_t)(P * ks * 4);
        const uint32_t qb = qflat ? range_bulk_bytes(qsi, qn) + range_bulk_bytes(qsp, qn) : 0u;
        mbar_expect_tx(bar, 2 * pb + qb);  // before any copy is issued
        bulk_g2s(pid, J.c_ids + (size_t)base * ks, pb, bar);
        bulk_g2s(ppr, J.c_probs + (size_t)base * ks, pb, bar);
    }
    if (qflat) {
        copy_range_async(reinterpret_cast<unsigned char*>(qid), qsi, qn, bar, lane);
        copy_range_async(reinterpret_cast<unsigned char*>(qpr), qsp, qn, bar, lane);
    }
    int pc_l = 0, qc_l = 0, d_l = 0;
    uint32_t f_l = 0;
    if (lane < P) {
        pc_l = clamp_count(__ldcg(J.c_count + base + lane), J.k);
        f_l = __ldcg(J.c_flags + base + lane);
    }
    if (lane < B) {
        qc_l = __ldcg(J.q_count + (int64_t)r * B + lane);
        d_l = __ldcg(J.draft_ids + (size_t)r * B + lane);
        if (J.q_flags != nullptr) f_l |= __ldcg(J.q_flags + (int64_t)r * B + lane);
    }
    if (!qflat)
        warp_copy_rows<false>(J.q_ids + (size_t)r * B * J.q_cap, J.q_probs + (size_t)r * B * J.q_cap, J.q_cap, B, QS,
                              qid, qpr, QS, lane);
    // the decisions' uniforms, one position per lane
    double ua = 0.0, ur = 0.0;
    if (lane < B) {
        ua = uniform53(J.seed, req, (uint32_t)lane, kDrawAccept, cycle_of(J));
        ur = uniform53(J.seed, req, (uint32_t)lane, kDrawResidual, cycle_of(J));
    } else if (lane == B) {
        ur = uniform53(J.seed, req, (uint32_t)B, kDrawTarget, cycle_of(J));
    }
    const bool copied = tail_copies_wait(bar, lane);
    if (!copied) {
        tail_timeout(J, r, lane);
        return true;
    }
    qc_l = qc_l < 0 ? 0 : (qc_l > J.q_cap ? J.q_cap : qc_l);
    if (__any_sync(kFull, lane < B && qc_l > QS)) return false;
    uint32_t flags = __reduce_or_sync(kFull, f_l);
    if (lane <= B) otok[lane] = -1;
    if (lane < P) pcnt[lane] = pc_l;
    if (lane < B) {
        qcnt[lane] = qc_l;
        dft[lane] = d_l;
    }
    __syncwarp();

    int32_t* toks = J.out_tokens + (size_t)r * (B + 1);
    // Every position's accept test at once (lane i: position i).  The walk
    // stops at the first position whose target row is empty or whose draft
    // is rejected; the positions before it are accepted, so deciding them
    // all in parallel and taking the first stop gives the sequential result.
    bool stop_i = false, empty_i = false, notin_i = false;
    int32_t x_i = -1;
    if (lane < B) {
        x_i = dft[lane];
        if (lane < sh) {
            // the base-weights token is emitted untested (none when its row is empty)
            stop_i = empty_i = qcnt[0] == 0;
        } else {
            const int pr = lane - sh;  // the target row that tests position `lane`
            const int pc = pcnt[pr];
            if (pc == 0) {
                stop_i = empty_i = true;  // a non-finite target row
            } else {
                const bool xin = x_i >= 0 && (int64_t)x_i < J.vocab;
                const double a = xin ? smem_lookup(qid + lane * qs, qpr + lane * qs, qcnt[lane], x_i) : 0.0;
                const double px = xin ? smem_lookup(pid + pr * ks, ppr + pr * ks, pc, x_i) : 0.0;
                notin_i = !(a > 0.0);
                stop_i = notin_i || !(ua * a < px);
            }
        }
    }
    const unsigned stops = __ballot_sync(kFull, stop_i);
    const int istop = stops ? __ffs(stops) - 1 : B;  // first stopping position (B: none)
    if (lane < istop) otok[lane] = x_i;             // accepted drafts
    int32_t acc = B, ntok = B + 1;
    if (istop < B) {
        const bool empty = __shfl_sync(kFull, empty_i, istop);
        acc = istop;
        ntok = empty ? istop : istop + 1;
        if (!empty) {
            if (__shfl_sync(kFull, notin_i, istop)) flags |= kFlagDraftNotInSupport;
            // residual max(0, p - q_i) over supp p, ascending ids (p: the
            // target row that tests position i)
            const int i = istop, pc = pcnt[i - sh];
            const int32_t* pi = pid + (i - sh) * ks;
            const float* pp = ppr + (i - sh) * ks;
            const int32_t* qi = qid + i * qs;
            const float* qp = qpr + i * qs;
            double ra = 0.0, rb = 0.0, pa = 0.0, pb = 0.0;
            if (lane < pc) {
                pa = (double)pp[lane];
                const double d = pa - smem_lookup(qi, qp, qcnt[i], pi[lane]);
                ra = d > 0.0 ? d : 0.0;
            }
            if (lane + 32 < pc) {
                pb = (double)pp[lane + 32];
                const double d = pb - smem_lookup(qi, qp, qcnt[i], pi[lane + 32]);
                rb = d > 0.0 ? d : 0.0;
            }
            const double u = __shfl_sync(kFull, ur, i);
            int pick = warp_inv_cdf(ra, rb, u, lane);
            if (pick < 0) {  // the residual is empty: draw from p_i
                flags |= kFlagResidualEmpty;
                pick = warp_inv_cdf(pa, pb, u, lane);
            }
            if (lane == 0) otok[i] = pick >= 0 ? pi[pick] : -1;
        }
    } else {
        const int pc = pcnt[B - sh];  // the bonus row
        if (pc == 0) {
            ntok = B;
        } else {
            const float* pp = ppr + (B - sh) * ks;
            const double wa = lane < pc ? (double)pp[lane] : 0.0, wb = lane + 32 < pc ? (double)pp[lane + 32] : 0.0;
            const double u = __shfl_sync(kFull, ur, B);
            const int pick = warp_inv_cdf(wa, wb, u, lane);
            if (lane == 0) otok[B] = pick >= 0 ? pid[(B - sh) * ks + pick] : -1;
        }
    }
    __syncwarp();
    for (int t = lane; t <= B; t += 32) toks[t] = otok[t];
    if (lane == 0) {
        J.out_accept_len[r] = acc > sh ? acc - sh : 0;  // accepted proposals (x_0 of the two-pass layout is not one)
        J.out_num_tokens[r] = ntok;
        J.out_req_flags[r] = flags;
    }
    return true;
}

__device__ __noinline__ bool tree_tail_fast(const RowJob& J, int32_t r, unsigned char* sm, int lane) {
    const int32_t B = J.B, V = J.V;
    const int kc = J.k, ks = J.ks;
    if (kc > 64) return false;
    int32_t n = J.num_nodes[r];
    n = n < 1 ? 1 : (n > V ? V : n);
    const size_t need = 16 + (size_t)n * ks * 8 + (size_t)n * 12 + (size_t)(B + 1) * 8;
    if (need > (size_t)J.tail_bytes) return false;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm);           // the copies' mbarrier
    int32_t* nid = reinterpret_cast<int32_t*>(sm + 16);        // [n][ks]
    float* npr = reinterpret_cast<float*>(nid + n * ks);       // [n][ks]
    int32_t* ncnt = reinterpret_cast<int32_t*>(npr + n * ks);  // [n]
    int32_t* tk = ncnt + n;                                    // [n]
    int32_t* pa = tk + n;                                      // [n]
    int32_t* otok = pa + n;                                    // [B+1] emitted tokens
    int32_t* opath = otok + (B + 1);                           // [B+1] nodes that drew them
    const int64_t base = (int64_t)r * V;
    // the nodes' compact target rows by bulk copies (one round trip)
    if (lane == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        const uint32_t nb = (uint32_t)(n * ks * 4);
        mbar_expect_tx(bar, 2 * nb);
        bulk_g2s(nid, J.c_ids + (size_t)base * ks, nb, bar);
        bulk_g2s(npr, J.c_probs + (size_t)base * ks, nb, bar);
    }
    uint32_t flags = 0;
    for (int j = lane; j < n; j += 32) {
        ncnt[j] = clamp_count(__ldcg(J.c_count + base + j), J.k);
        flags |= __ldcg(J.c_flags + base + j);
        tk[j] = J.node_token[(size_t)r * V + j];
        pa[j] = J.node_parent[(size_t)r * V + j];
    }
    for (int q = lane; q <= B; q += 32) {
        otok[q] = -1;
        opath[q] = -1;
    }
    flags = __reduce_or_sync(kFull, flags);
    if (!tail_copies_wait(bar, lane)) {
        tail_timeout(J, r, lane);
        return true;
    }
    int32_t* toks = J.out_tokens + (size_t)r * (B + 1);
    int32_t* path = J.out_path_nodes + (size_t)r * (B + 1);
    const uint32_t req = J.first_request + (uint32_t)r;
    int32_t j = 0, t = 0, acc = 0, ntok = 0;
    for (;;) {
        const int pc = ncnt[j];
        if (pc == 0) {
            if (lane == 0) opath[t] = j;
            ntok = t;
            acc = t;
            break;
        }
        const float* pp = npr + j * ks;
        const double wa = lane < pc ? (double)pp[lane] : 0.0, wb = lane + 32 < pc ? (double)pp[lane + 32] : 0.0;
        const double u = uniform53(J.seed, req, (uint32_t)j, kDrawTarget, cycle_of(J));
        const int pick = warp_inv_cdf(wa, wb, u, lane);
        const int32_t y = pick >= 0 ? nid[j * ks + pick] : -1;
        if (lane == 0) {
            otok[t] = y;
            opath[t] = j;
        }
        ++t;
        ntok = t;
        acc = t - 1;
        int32_t next = -1;  // the lowest-index child of j carrying y
        for (int c0 = 1; c0 < n && next < 0; c0 += 32) {
            const int c = c0 + lane;
            const bool hit = c < n && pa[c] == j && tk[c] == y;
            const unsigned bal = __ballot_sync(kFull, hit);
            if (bal) next = c0 + __ffs(bal) - 1;
        }
        if (next < 0 || t > B) break;
        j = next;
    }
    __syncwarp();
    for (int q = lane; q <= B; q += 32) {
        toks[q] = otok[q];
        path[q] = opath[q];
    }
    if (lane == 0) {
        J.out_accept_len[r] = acc;
        J.out_num_tokens[r] = ntok;
        J.out_req_flags[r] = flags;
    }
    return true;
}

template <int MODE>
__device__ __forceinline__ void request_tail(const RowJob& J, int32_t req, double* wd, unsigned char* tail_smem,
                                             int lane) {
    if (MODE == kModeLinear || MODE == kModeCycle) {
        if (!linear_tail_fast(J, req, tail_smem, lane)) linear_tail(J, req, wd, lane);
    } else {
        if (!tree_tail_fast(J, req, tail_smem, lane)) tree_tail(J, req, wd, lane);
    }
}

// One warp: count a finished row of request req; the warp that counts the
// request's last row runs the request's tail.
template <int MODE>
__device__ __forceinline__ void request_arrive(const RowJob& J, int32_t req, double* wd, unsigned char* tail_smem,
                                               int lane) {
    __syncwarp();
    int last = 0;
    if (lane == 0) {
        __threadfence();
        const uint32_t t = atomicAdd(J.req_ticket + req, 1u);
        last = (t == (uint32_t)(J.rpr - 1));
        if (last) {
            atomicExch(J.req_ticket + req, 0u);
            __threadfence();
        }
    }
    last = __shfl_sync(kFull, last, 0);
    if (last) request_tail<MODE>(J, req, wd, tail_smem, lane);
}


// ---------------------------------------------------------------------------
// Finishing a row (all threads of the CTA).
// ---------------------------------------------------------------------------
struct FinishShared {
    double S, W;
    int kept, last, n;
};

// Exact top k of the unique keys uni[0..U): each key's rank is the number of
// larger keys; ranks below k land in sel[rank], so sel comes out sorted
// (descending).  All threads call it.
__device__ __forceinline__ void cta_rank_topk(const uint64_t* uni, int U, int k, uint64_t* sel) {
    for (int i = threadIdx.x; i < U; i += kThreads) {
        const uint64_t key = uni[i];
        int rank = 0;
        int j = 0;
        for (; j + 8 <= U; j += 8) {  // independent loads ahead of the compares
            ulonglong2 p[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) p[q] = *reinterpret_cast<const ulonglong2*>(uni + j + 2 * q);
#pragma unroll
            for (int q = 0; q < 4; ++q) rank += (p[q].x > key) + (p[q].y > key);
        }
        for (; j < U; ++j) rank += (uni[j] > key);
        if (rank < k) sel[rank] = key;
    }
}

// The joint order's normaliser of a row whose largest value is v0:
// sum over every finite logit of exp((l - v0) / T), from the row's pair.
__device__ __forceinline__ double joint_sum(const RowJob& J, int64_t row, double v0, double inv_t) {
    const double2 ms = J.row_ms[row];
    return ms.y * exp((ms.x - v0) * inv_t);
}

// A row's flags: bit 0 of rowbad: NaN / +inf (or no finite logit); bit 1: a
// wait gave up; badp: its request's parameters are out of range.
__device__ __forceinline__ uint32_t row_flags(bool bad, uint32_t rowbad, bool badp) {
    if (!bad) return 0u;
    if (badp) return kFlagBadParams | ((rowbad & 1u) ? kFlagNonfinite : 0u) | ((rowbad & 2u) ? kFlagTimeout : 0u);
    return (rowbad & 2u) ? (kFlagTimeout | ((rowbad & 1u) ? kFlagNonfinite : 0u)) : kFlagNonfinite;
}

// jms: the row's joint-order pair when the caller accumulated it (else the
// normaliser pass left it in J.row_ms).
template <int MODE, int PR>
__device__ void finish_row_warp(const RowJob& J, int64_t row, int32_t req, int n, uint32_t rowbad,
                                const uint64_t* sel, double* wd, unsigned char* tail_smem, FinishShared& fs, int lane,
                                uint64_t* pairs, const double2* jms) {
    const RowParams rp = PR ? row_params<MODE>(J, row) : RowParams{J.temperature, J.top_p, J.k, true};
    if (n > rp.k) n = rp.k;  // sel[] holds the best min(top_k_max, vocab), descending
    const bool bad = rowbad != 0u || n == 0 || !rp.ok;
    int kept = 0;
    uint64_t oa = ~0ull, ob = ~0ull;  // (id, prob) pairs, ascending id after the sort
    if (!bad) {
        const uint64_t ka = lane < n ? sel[lane] : 0ull, kb = lane + 32 < n ? sel[lane + 32] : 0ull;
        double wa = 0.0, wb = 0.0;
        if (rp.T == 0.0f) {
            kept = 1;
            wa = lane == 0 ? 1.0 : 0.0;
        } else {
            const double v0 = (double)key_value(sel[0]);
            const double inv_t = 1.0 / (double)rp.T;
            if (lane < n) wa = exp(((double)key_value(ka) - v0) * inv_t);
            if (lane + 32 < n) wb = exp(((double)key_value(kb) - v0) * inv_t);
            if (rp.p >= 1.0f) {
                kept = n;
            } else {
                const double S = !(PR && J.joint) ? warp_sum_d(wa + wb)
                                 : jms != nullptr ? jms->y * exp((jms->x - v0) * inv_t) : joint_sum(J, row, v0, inv_t);
                const double inv_s = 1.0 / S;
                const double pa = wa * inv_s, pb = wb * inv_s;
                // mass before rank j
                const double ia = warp_incl_scan_d(pa, lane);
                const double ta = __shfl_sync(kFull, ia, 31);
                const double ib = warp_incl_scan_d(pb, lane) + ta;
                double ea = __shfl_up_sync(kFull, ia, 1), eb = __shfl_up_sync(kFull, ib, 1);
                if (lane == 0) {
                    ea = 0.0;
                    eb = ta;
                }
                const double tp = (double)rp.p;
                const bool keepa = lane < n && (lane == 0 || ea < tp);
                const bool keepb = lane + 32 < n && eb < tp;
                kept = __popc(__ballot_sync(kFull, keepa)) + __popc(__ballot_sync(kFull, keepb));
            }
        }
        const double ra = lane < kept ? wa : 0.0, rb = lane + 32 < kept ? wb : 0.0;
        const double inv_w = 1.0 / warp_sum_d(ra + rb);
        if (lane < kept)
            oa = ((uint64_t)(uint32_t)key_id(ka) << 32) | (uint64_t)__float_as_uint((float)(wa * inv_w));
        if (lane + 32 < kept)
            ob = ((uint64_t)(uint32_t)key_id(kb) << 32) | (uint64_t)__float_as_uint((float)(wb * inv_w));
        // ascending id order: each pair goes to its rank among the kept ids
        // (distinct), counted against sel[] in shared memory
        const uint32_t ida = (uint32_t)key_id(ka), idb = (uint32_t)key_id(kb);
        int pa = 0, pb = 0;
#pragma unroll 4
        for (int j = 0; j < kept; ++j) {
            const uint32_t x = (uint32_t)key_id(sel[j]);
            pa += x < ida ? 1 : 0;
            pb += x < idb ? 1 : 0;
        }
        __syncwarp();
        if (lane < kept) pairs[pa] = oa;
        if (lane + 32 < kept) pairs[pb] = ob;
        __syncwarp();
        oa = lane < kept ? pairs[lane] : ~0ull;
        ob = lane + 32 < kept ? pairs[lane + 32] : ~0ull;
    }
    const uint32_t rflags = row_flags(bad, rowbad, !rp.ok);
    if (MODE == kModeFilter || (MODE == kModeCycle && row < J.nq2)) {
        int32_t* ids = J.out_ids + (size_t)row * J.cap;
        float* pr = J.out_probs + (size_t)row * J.cap;
        // lanes write their own two slots, then the rest of the row's slots
        if (lane < J.cap) {
            ids[lane] = lane < kept ? (int32_t)(oa >> 32) : -1;
            pr[lane] = lane < kept ? __uint_as_float((uint32_t)oa) : 0.0f;
        }
        if (lane + 32 < J.cap) {
            ids[lane + 32] = lane + 32 < kept ? (int32_t)(ob >> 32) : -1;
            pr[lane + 32] = lane + 32 < kept ? __uint_as_float((uint32_t)ob) : 0.0f;
        }
        for (int j = 64 + lane; j < J.cap; j += 32) {
            ids[j] = -1;
            pr[j] = 0.0f;
        }
        if (J.out_dense != nullptr) {
            float* d = J.out_dense + (size_t)row * (size_t)J.vocab;
            if (lane < kept) d[(int32_t)(oa >> 32)] = __uint_as_float((uint32_t)oa);
            if (lane + 32 < kept) d[(int32_t)(ob >> 32)] = __uint_as_float((uint32_t)ob);
        }
        int32_t tok = -1;
        if (J.has_rng && kept > 0) {
            const double u = uniform53(J.seed, J.first_request + (uint32_t)(row / J.rpr), (uint32_t)(row % J.rpr),
                                       kDrawProposal, cycle_of(J));
            const double wa = lane < kept ? (double)__uint_as_float((uint32_t)oa) : 0.0;
            const double wb = lane + 32 < kept ? (double)__uint_as_float((uint32_t)ob) : 0.0;
            const int pick = warp_inv_cdf(wa, wb, u, lane);
            if (pick >= 0) tok = (int32_t)(__shfl_sync(kFull, pick < 32 ? oa : ob, pick & 31) >> 32);
        }
        if (lane == 0) {
            J.out_count[row] = kept;
            J.out_flags[row] = rflags;
            if (J.has_rng) J.out_sample[row] = tok;
        }
    } else {
        if (MODE == kModeCycle) row -= J.nq2;  // the cycle's target rows
        int32_t* ids = J.c_ids + (size_t)row * J.ks;
        float* pr = J.c_probs + (size_t)row * J.ks;
        if (lane < kept) {
            ids[lane] = (int32_t)(oa >> 32);
            pr[lane] = __uint_as_float((uint32_t)oa);
        }
        if (lane + 32 < kept) {
            ids[lane + 32] = (int32_t)(ob >> 32);
            pr[lane + 32] = __uint_as_float((uint32_t)ob);
        }
        if (lane == 0) {
            J.c_count[row] = kept;
            J.c_flags[row] = rflags;
        }
        if (!J.defer_tails) request_arrive<MODE>(J, req, wd, tail_smem, lane);
    }
}

// Softmax in double over the sorted top n, top-p cut, renormalise, and write
// the row (filter: output; verifiers: workspace + request tail).
template <int MODE>
__device__ void finish_row(const RowJob& J, int64_t row, int32_t req, int n, uint32_t rowbad, const uint64_t* sel,
                           uint64_t* outk, double* wd, double* pd, unsigned char* tail_smem, FinishShared& fs, int warp,
                           int lane) {
    const int tid = threadIdx.x;
    const RowParams rp = row_params<MODE>(J, row);
    if (n > rp.k) n = rp.k;  // sel[] holds the best min(top_k_max, vocab), descending
    const bool bad = rowbad != 0u || n == 0 || !rp.ok;
    int kept = 0;
    if (!bad) {
        const double v0 = (double)key_value(sel[0]);
        if (rp.T == 0.0f) {
            kept = 1;
            if (tid == 0) fs.W = 1.0;
            if (tid == 0) wd[0] = 1.0;
        } else {
            const double temp = (double)rp.T;
            for (int j = tid; j < n; j += kThreads) wd[j] = exp(((double)key_value(sel[j]) - v0) / temp);
            __syncthreads();
            // the defined (descending) order; the joint order's normaliser
            // covers the whole row
            if (tid == 0) fs.S = J.joint ? joint_sum(J, row, v0, 1.0 / temp) : serial_sum(wd, n);
            __syncthreads();
            const double S = fs.S;
            for (int j = tid; j < n; j += kThreads) pd[j] = wd[j] / S;
            __syncthreads();
            if (tid == 0) {
                int kk = 0;
                if (rp.p >= 1.0f) {
                    kk = n;
                } else {
                    const double tp = (double)rp.p;
                    double m = 0.0;
                    int j = 0;
                    for (; j + 8 <= n; j += 8) {  // loads ahead of the dependent walk
                        double b[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) b[q] = pd[j + q];
                        bool stop = false;
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            if (!stop) {
                                if (j + q > 0 && !(m < tp)) {
                                    stop = true;
                                } else {
                                    m += b[q];
                                    ++kk;
                                }
                            }
                        }
                        if (stop) break;
                    }
                    if (kk == j) {
                        for (; j < n; ++j) {
                            if (j > 0 && !(m < tp)) break;
                            m += pd[j];
                            ++kk;
                        }
                    }
                }
                fs.kept = kk;
                fs.W = serial_sum(wd, kk);
            }
        }
        __syncthreads();
        if (rp.T != 0.0f) kept = fs.kept;
        const double W = fs.W;
        // (id, prob) pairs in ascending id order
        for (int j = tid; j < kept; j += kThreads) {
            const float p = (float)(wd[j] / W);
            const uint32_t id = (uint32_t)key_id(sel[j]);
            int r = 0;
            int i = 0;
            for (; i + 8 <= kept; i += 8) {
                uint64_t b[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) b[q] = sel[i + q];
#pragma unroll
                for (int q = 0; q < 8; ++q) r += ((uint32_t)key_id(b[q]) < id);
            }
            for (; i < kept; ++i) r += ((uint32_t)key_id(sel[i]) < id);
            outk[r] = ((uint64_t)id << 32) | (uint64_t)__float_as_uint(p);
        }
        __syncthreads();
    }
    const uint32_t rflags = row_flags(bad, rowbad, !rp.ok);

    if (MODE == kModeFilter) {
        int32_t* ids = J.out_ids + (size_t)row * J.cap;
        float* pr = J.out_probs + (size_t)row * J.cap;
        for (int j = tid; j < J.cap; j += kThreads) {
            if (j < kept) {
                ids[j] = (int32_t)(outk[j] >> 32);
                pr[j] = __uint_as_float((uint32_t)outk[j]);
            } else {
                ids[j] = -1;
                pr[j] = 0.0f;
            }
        }
        if (J.out_dense != nullptr) {
            float* d = J.out_dense + (size_t)row * (size_t)J.vocab;
            for (int j = tid; j < kept; j += kThreads) d[(int32_t)(outk[j] >> 32)] = __uint_as_float((uint32_t)outk[j]);
        }
        if (tid == 0) {
            J.out_count[row] = kept;
            J.out_flags[row] = rflags;
            if (J.has_rng) {
                int32_t tok = -1;
                if (kept > 0) {
                    for (int j = 0; j < kept; ++j) wd[j] = (double)__uint_as_float((uint32_t)outk[j]);
                    const double u = uniform53(J.seed, J.first_request + (uint32_t)(row / J.rpr),
                                               (uint32_t)(row % J.rpr), kDrawProposal, cycle_of(J));
                    const int pick = inv_cdf_serial(wd, kept, u);
                    tok = pick >= 0 ? (int32_t)(outk[pick] >> 32) : -1;
                }
                J.out_sample[row] = tok;
            }
        }
    } else {
        int32_t* ids = J.c_ids + (size_t)row * J.ks;
        float* pr = J.c_probs + (size_t)row * J.ks;
        for (int j = tid; j < kept; j += kThreads) {
            ids[j] = (int32_t)(outk[j] >> 32);
            pr[j] = __uint_as_float((uint32_t)outk[j]);
        }
        if (tid == 0) {
            J.c_count[row] = kept;
            J.c_flags[row] = rflags;
        }
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            const uint32_t t = atomicAdd(J.req_ticket + req, 1u);
            fs.last = (t == (uint32_t)(J.rpr - 1));
            if (fs.last) {
                atomicExch(J.req_ticket + req, 0u);
                __threadfence();
            }
        }
        __syncthreads();
        if (fs.last && warp == 0) request_tail<MODE>(J, req, wd, tail_smem, lane);
    }
}

// ---------------------------------------------------------------------------
// The row kernel.
// ---------------------------------------------------------------------------
template <typename T, int MODE>
__global__ void __launch_bounds__(kThreads, 4) row_kernel(const __grid_constant__ RowJob J) {
    extern __shared__ __align__(128) unsigned char smem[];
    // streaming: ring stages | barriers | counters | warp buffers
    unsigned char* stages = smem;                                                   // [kStages][kStageBytes]
    uint64_t* full = reinterpret_cast<uint64_t*>(stages + kStages * kStageBytes);   // [kStages]
    int* done = reinterpret_cast<int*>(full + kStages);                             // [kStages] (+pad)
    uint64_t* wbufs = reinterpret_cast<uint64_t*>(full + 2 * kStages);
    // finishing (after streaming): in the ring stages when it fits there
    unsigned char* fin = J.fin_off ? smem + J.fin_off : smem;
    uint64_t* uni = reinterpret_cast<uint64_t*>(fin);   // [merge_cap]
    uint64_t* sel = uni + J.merge_cap;                  // [k]
    uint64_t* outk = sel + J.k;                         // [k]
    double* wd = reinterpret_cast<double*>(outk + J.k); // [k]
    double* pd = wd + J.k;                              // [k]

    __shared__ unsigned long long s_tau;
    __shared__ int s_wcnt[kWarps];
    __shared__ int s_cnt[kWarps];
    __shared__ uint32_t s_bad;
    __shared__ FinishShared fs;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x / J.S;
    const int split = (int)(blockIdx.x % J.S);
    const int32_t req = (int32_t)(row / J.rpr);

    // Tree rows past the request's node count are neither read nor used.
    if (MODE == kModeTree) {
        int32_t nn = J.num_nodes[req];
        nn = nn < 1 ? 1 : (nn > J.V ? J.V : nn);
        if ((int32_t)(row % J.V) >= nn) {
            if (split != 0) return;
            if (threadIdx.x == 0) {
                __threadfence();
                const uint32_t t = atomicAdd(J.req_ticket + req, 1u);
                fs.last = (t == (uint32_t)(J.rpr - 1));
                if (fs.last) {
                    atomicExch(J.req_ticket + req, 0u);
                    __threadfence();
                }
            }
            __syncthreads();
            if (fs.last && warp == 0) request_tail<kModeTree>(J, req, wd, smem + J.tail_off, lane);
            return;
        }
    }

    if (threadIdx.x == 0) {
        s_tau = 0ull;
        s_bad = 0u;
    }
    if (threadIdx.x < kWarps) s_wcnt[threadIdx.x] = 0;

    const RowGeom g = row_geom<T>(J, row);
    const int64_t per = (g.nunit + J.S - 1) / J.S;
    const int64_t vb = per * split < g.nunit ? per * split : g.nunit;
    const int64_t ve = vb + per < g.nunit ? vb + per : g.nunit;

    // Zero the dense row over this CTA's element range before any value is
    // written (the last CTA of the row writes the values after the ticket).
    if (MODE == kModeFilter && J.out_dense != nullptr) {
        const int64_t e0 = (split == 0) ? 0 : g.head + vb * Elem<T>::kPerUnit;
        const int64_t e1 = (split == J.S - 1) ? J.vocab : g.head + ve * Elem<T>::kPerUnit;
        float* d = J.out_dense + (size_t)row * (size_t)J.vocab;
        for (int64_t e = e0 + threadIdx.x; e < e1; e += kThreads) d[e] = 0.0f;
    }
    __syncthreads();

    WarpState ws;
    ws.buf = wbufs + (size_t)warp * J.cap_w;
    ws.wcnt = &s_wcnt[warp];
    ws.cnt = 0;
    ws.tau = 0ull;
    ws.bad = 0u;
    Ring ring;
    ring.stages = stages;
    ring.full = full;
    ring.done = done;
    scan_slice<T>(J, g, vb, ve, split == 0, ws, &s_tau, ring, wbufs, warp, lane);

    // each warp drops what the CTA's threshold has ruled out
    {
        const unsigned long long st = *reinterpret_cast<volatile unsigned long long*>(&s_tau);
        if (st > ws.tau) ws.tau = st;
        ws.cnt = warp_keep_ge(ws.buf, ws.cnt, ws.tau, lane);
    }
    const uint32_t wbad = __reduce_or_sync(kFull, ws.bad);
    if (lane == 0) {
        s_cnt[warp] = ws.cnt;
        if (wbad) atomicOr(&s_bad, wbad);
    }
    __syncthreads();
    int U = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) U += s_cnt[w];
    if (U > J.merge_cap) {  // rare: cut every warp to its own best k first
        const Compacted cp = warp_compact(ws.buf, ws.wcnt, ws.cnt, ws.tau, J.k, &s_tau, lane);
        ws.cnt = cp.cnt;
        if (lane == 0) s_cnt[warp] = ws.cnt;
        __syncthreads();
        U = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) U += s_cnt[w];
    }
    {
        int off = 0;
        for (int w = 0; w < warp; ++w) off += s_cnt[w];
        for (int i = lane; i < ws.cnt; i += 32) uni[off + i] = ws.buf[i];
    }
    __syncthreads();
    cta_rank_topk(uni, U, J.k, sel);
    int n = U < J.k ? U : J.k;
    uint32_t rowbad = s_bad;
    __syncthreads();

    // Split rows: publish this CTA's best k; the last CTA of the row merges.
    if (J.S > 1) {
        const size_t pslot = (size_t)row * J.S + split;
        uint64_t* pk = J.part_keys + pslot * J.k;
        for (int i = threadIdx.x; i < n; i += kThreads) pk[i] = sel[i];
        __syncthreads();
        if (threadIdx.x == 0) {
            J.part_count[pslot] = n;
            J.part_flags[pslot] = rowbad;
            __threadfence();
            const uint32_t t = atomicAdd(J.row_ticket + row, 1u);
            fs.last = (t == (uint32_t)(J.S - 1));
            if (fs.last) {
                atomicExch(J.row_ticket + row, 0u);
                __threadfence();
            }
        }
        __syncthreads();
        if (!fs.last) return;
        U = 0;
        rowbad = 0;
        for (int s = 0; s < J.S; ++s) {
            const size_t ps = (size_t)row * J.S + s;
            const int c = __ldcg(J.part_count + ps);
            rowbad |= __ldcg(J.part_flags + ps);
            const unsigned long long* src = reinterpret_cast<const unsigned long long*>(J.part_keys + ps * J.k);
            for (int i = threadIdx.x; i < c; i += kThreads) uni[U + i] = __ldcg(src + i);
            U += c;
        }
        __syncthreads();
        cta_rank_topk(uni, U, J.k, sel);
        n = U < J.k ? U : J.k;
        __syncthreads();
    }

    if (J.k <= 64) {
        if (warp == 0)
            finish_row_warp<MODE, 1>(J, row, req, n, rowbad, sel, wd, smem + J.tail_off, fs, lane, outk, nullptr);
    } else {
        finish_row<MODE>(J, row, req, n, rowbad, sel, outk, wd, pd, smem + J.tail_off, fs, warp, lane);
    }
}

// ---------------------------------------------------------------------------
// The pipelined row kernel (k <= 64, no dense row): one persistent CTA per
// SM.  The rows are laid end to end as one sequence of 16-byte units and
// CTA b of G streams the b-th G-th of it (balanced pieces, below), so every
// CTA moves the same number of bytes.
//
//   warp 0      producer: lane 0 keeps a ring of `nst` 16 KB stages filled
//               with bulk copies (TMA, no multicast), running across piece
//               boundaries, each stage tracked by a `full` mbarrier, a fill
//               tag and an `empty` mbarrier;
//   warps 1..8  consumers: ring element q goes to consumer q % 8, whatever
//               piece it belongs to.  A consumer reads each of its stages
//               once, as it lands: the maxima of its units, then every
//               element at or above the piece's threshold into its
//               candidate buffer of the piece's slot (lane-parallel, one
//               warp scan for the write positions);
//   warps 9..10 finishers: finisher f takes the pieces whose ordinal in the
//               CTA's list is f mod 2 from slot f: it gathers the keys at or
//               above the piece's final threshold, hands the slot back, and
//               selects the exact top-k from its copy; a split row's pieces
//               publish their partial top-k and the last one merges; then
//               the softmax / top-p / output work of the row.
//
// Thresholds.  A piece runs in one of two modes.
//   * boot: the piece's first stages (up to 8) wait until the k-th largest
//     of their lane maxima is known, then every stage is filtered by it.
//     The k-th largest of any set of disjoint group maxima of a row is at
//     most the row's k-th largest element, so this loses nothing.  A CTA's
//     first piece runs this way.
//   * predicted: the piece is filtered by the CTA's latest prediction, with
//     no waiting: a value that about 2.5 k elements of a row reach,
//     extrapolated from the k/2-th and k-th values of the last finished row
//     of the same row set (or, at the start, the prediction the CTA left in
//     the workspace at the end of the previous call).  The first consumer to
//     start a piece fixes its mode.  Decoding cycles give rows of one
//     distribution, so the prediction holds almost always; it is checked
//     exactly: the row's k-th kept key must be at or above every threshold
//     its pieces used, which means at least k elements of the row reach them
//     and nothing of the top k was dropped.  A row that fails the check is
//     re-read whole, in boot mode, at the end of the CTA's list (the redo
//     pass), before the kernel exits.
// Consumers raise the piece's threshold as their candidate buffers fill (a
// buffer over its high-water mark is cut to its k best), and the finisher
// gathers by the highest threshold any of them posted, so it sorts about k
// keys.
//
// Every wait is bounded; a wait that gives up sets the CTA's abort word,
// every role stops at its next check, and rows that were not finished are
// written with UNO_FLAG_TIMEOUT.
// ---------------------------------------------------------------------------
constexpr int kPipeConsumers = 8;
constexpr int kPipeFinishers = 2;
// Rows handed out at run time: the producer of each CTA takes the next row
// from a counter in the workspace and posts it in a queue that the CTA's
// consumers and finishers read in order.  Counter words (zero between calls):
constexpr int kDynNext = 0;      // next row
constexpr int kDynDone = 1;      // CTAs that have exited
constexpr int kDynRetryPut = 2;  // rows posted for a second read
constexpr int kDynRetryGet = 3;  // of those, taken
constexpr int kDynFinished = 4;  // rows finished
constexpr int kDynWords = 8;     // then one word per posted retry (row + 1; 0 = not yet written)
constexpr int kDynOffset = 1024; // counter words start here in the row-ticket area
constexpr int kDynQ = 64;        // queue entries (the producer runs at most a few rows ahead)
constexpr int kTicketAhead = 3;  // stages before a row's last copy at which the next ticket is taken
constexpr int kPipeSlots = kPipeFinishers;
constexpr int kPipeWarps = 1 + kPipeConsumers + kPipeFinishers;
constexpr int kPipeThreads = 32 * kPipeWarps;
constexpr int kPipeMaxK = 64;
// A pipelined stage is 16 KB (1024 units); its owner's lane l takes units
// l, l + 32, ... (conflict-free shared loads), 32 units per lane.
constexpr int kPStageBytes = 16384;
constexpr int kPStageUnits = kPStageBytes / 16;                 // 1024
constexpr int kPLaneUnits = kPStageUnits / 32;                  // 32 per lane per stage
constexpr int kPGroups = 4;                                     // groups of 8 units per lane (one-stage seed)
constexpr int kPBootStages = 8;                                 // stages of a piece's seed
constexpr int kPGather = 256;                                   // keys a finisher gathers for its select
constexpr int kPipeMinStages = 6, kPipeMaxStages = 12;
// The largest grid: part slots of split rows are sized for it.
constexpr int kPipeMaxGrid = 256;
// A piece of a row is at least this many units when rows are few.  A split
// row costs a merge across CTAs after its pieces (about 8 us: the pieces'
// keys published, a ticket, the last piece reading them back); a piece of
// 19 stages (304 KB) streams about as long on one SM, so shorter pieces do
// not pay for the merge (16 bf16 rows of 151,936 logits: 24.6 us whole
// against 32.8 us in pieces of 4 stages).
constexpr int64_t kPipeMinPieceUnits = 19 * kPStageUnits;
// A row is cut into at most this many pieces (one merge warp).
constexpr int kPipeMaxPieces = 32;
// Suspend hint of the off-path waits (ns): the waiting thread sleeps until
// the phase completes or the hint runs out, instead of polling.
constexpr uint32_t kNapNs = 2000;

struct __align__(16) PipeShared {
    uint64_t full[kPipeMaxStages];          // stage bytes arrived
    uint64_t empty[kPipeMaxStages];         // the stage's owner warp is done with it
    uint32_t fill[kPipeMaxStages];          // ring element each buffer holds or is receiving
    uint64_t slot_full[kPipeSlots];         // every consumer warp is done with the slot's piece
    uint64_t slot_empty[kPipeSlots];        // the finisher is done with the slot's buffers
    unsigned long long tau[kPipeSlots];     // CTA threshold key of the slot's piece
    unsigned long long used[kPipeSlots];    // largest predicted threshold the piece was filtered by
    __align__(16) uint32_t boot[kPipeSlots][kPBootStages * 32];  // lane maxima of the seed stages
    int boot_cnt[kPipeSlots];               // seed stages done
    uint32_t boot_ready[kPipeSlots];        // the seed is in tau
    uint32_t mode[kPipeSlots];              // the piece's mode, set by its first consumer (1 predicted, 2 not)
    int cnt[kPipeSlots][kPipeConsumers];    // candidates per consumer warp of the slot's piece
    float jm[kPipeSlots][kPipeConsumers];   // joint order: per consumer warp, its pair (m, s) for the piece
    double js[kPipeSlots][kPipeConsumers];
    int wcnt[kPipeConsumers];               // candidate counts (compaction bookkeeping)
    uint32_t bad[kPipeSlots];               // NaN / +inf (bit 0) or gave-up (bit 1) of the slot's piece
    unsigned long long spec[2];             // the latest prediction (a threshold key), per row set
    uint32_t spec_set[2];                   // a prediction exists
    long long qrow[kDynQ];                  // run-time rows: the row (bit 62: a second read), -1 at the end
    uint32_t qseq[kDynQ];                   // entry i % kDynQ holds item i when it reads i + 1
    int fin_done;                           // finishers done with the CTA's list
    int redo_n;                             // rows of the redo pass
    uint32_t redo_ready;                    // redo_n is final
    int abort;
};

// A cycle's draft rows (0) and target rows (1) differ in scale.
template <int MODE>
__device__ __forceinline__ int row_set(const RowJob& J, int64_t row) {
    return (MODE == kModeCycle && row >= J.nq2) ? 1 : 0;
}

template <int MODE>
__device__ __forceinline__ bool item_active(const RowJob& J, int64_t row) {
    if (MODE != kModeTree) return true;
    int32_t nn = J.num_nodes[row / J.rpr];
    nn = nn < 1 ? 1 : (nn > J.V ? J.V : nn);
    return (int32_t)(row % J.V) < nn;
}

// ---------------------------------------------------------------------------
// Balanced pieces.  Row r owns the virtual units [r*nu, (r+1)*nu) of a
// sequence of T = rows*nu, nu = floor(vocab / elements per unit) (a row's
// real unit count is nu or nu - 1, by its alignment; units past it are
// empty).  CTA b of G takes [b*T/G, (b+1)*T/G).  A row that a CTA boundary
// cuts is split; each of its pieces publishes its partial top-k in a part
// slot of its CTA (2b for the CTA's first row, 2b + 1 for its last) and
// takes a ticket at the row's first CTA, which no other split row shares.
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int64_t part_start(int64_t b, int64_t T, int64_t G) { return b * T / G; }
// the CTA whose range holds virtual unit x (the largest b with start(b) <= x)
__host__ __device__ __forceinline__ int64_t part_cta(int64_t x, int64_t T, int64_t G) {
    return ((x + 1) * G + T - 1) / T - 1;
}

struct Piece {
    RowGeom g;
    const unsigned char* ubase;  // unit 0 of the row (16-byte aligned)
    int ub, ue, nstage;          // the piece: units [ub, ue) of the row
    int seg, np;                 // index of the piece in its row; pieces of the row
    int64_t first_cta;           // CTA of the row's first piece
};

struct CtaRange {
    int64_t nu, T, G, b, s, e, row0, row1;  // rows [row0, row1]
};

template <typename T>
__device__ __forceinline__ CtaRange cta_range(const RowJob& J) {
    CtaRange c;
    const int64_t nu = J.vocab / Elem<T>::kPerUnit;
    c.nu = nu > 0 ? nu : 1;
    c.T = J.rows * c.nu;
    c.G = gridDim.x;
    c.b = blockIdx.x;
    c.s = part_start(c.b, c.T, c.G);
    c.e = part_start(c.b + 1, c.T, c.G);
    c.row0 = c.s / c.nu;
    c.row1 = c.e > c.s ? (c.e - 1) / c.nu : c.row0 - 1;
    return c;
}

template <typename T>
__device__ __forceinline__ Piece piece_of(const RowJob& J, const CtaRange& c, int64_t row) {
    Piece p;
    p.g = row_geom<T>(J, row);
    p.ubase = p.g.base + (size_t)p.g.head * Elem<T>::kBytes;
    const int64_t r0 = row * c.nu;
    const int64_t vb = (c.s > r0 ? c.s : r0) - r0;
    const int64_t ve = (c.e < r0 + c.nu ? c.e : r0 + c.nu) - r0;
    p.ub = (int)(vb < p.g.nunit ? vb : p.g.nunit);
    p.ue = (int)(ve < p.g.nunit ? ve : p.g.nunit);
    p.nstage = (p.ue - p.ub + kPStageUnits - 1) / kPStageUnits;
    p.first_cta = part_cta(r0, c.T, c.G);
    p.seg = (int)(c.b - p.first_cta);
    p.np = (int)(part_cta(r0 + c.nu - 1, c.T, c.G) - p.first_cta + 1);
    return p;
}

// A whole row as one piece (the redo pass).
template <typename T>
__device__ __forceinline__ Piece whole_row(const RowJob& J, const CtaRange& c, int64_t row) {
    Piece p;
    p.g = row_geom<T>(J, row);
    p.ubase = p.g.base + (size_t)p.g.head * Elem<T>::kBytes;
    p.ub = 0;
    p.ue = (int)p.g.nunit;
    p.nstage = (p.ue + kPStageUnits - 1) / kPStageUnits;
    p.first_cta = c.b;
    p.seg = 0;
    p.np = 1;
    return p;
}

// Part slot of row `row`'s piece in CTA b.
__device__ __forceinline__ int64_t part_slot(const CtaRange& c, int64_t b, int64_t row) {
    return 2 * b + ((part_start(b, c.T, c.G) / c.nu) == row ? 0 : 1);
}

__device__ __forceinline__ bool pipe_aborted(const PipeShared& P) {
    return *reinterpret_cast<const volatile int*>(&P.abort) != 0;
}

__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Bounded wait that also gives up once the CTA has aborted.  The first probe
// returns at once; later ones sleep in the barrier until the phase completes
// (or the hint runs out), so waiting threads leave the issue slots and the
// shared-memory pipe to the others.  Every thread that calls it polls; call
// it with the whole warp converged.
__device__ __forceinline__ bool pipe_wait(uint64_t* bar, uint32_t parity, const PipeShared& P) {
    if (mbar_try_wait(bar, parity)) return true;
    for (uint32_t it = 0; it < (kMaxWaitTries >> 4); ++it) {
        if (mbar_try_wait_hint(bar, parity, kNapNs)) return true;
        if (pipe_aborted(P)) return false;
    }
    return false;
}

__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait by polling with short naps: the waiter sees the phase within
// a few tens of nanoseconds of its completion (a suspending try_wait can
// sleep well past it).  For the waits on the streaming path.
constexpr uint32_t kSpinTries = 1u << 25;  // about a second at the nap below
__device__ __forceinline__ bool pipe_spin(uint64_t* bar, uint32_t parity, const PipeShared& P) {
    for (uint32_t it = 0; it < kSpinTries; ++it) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((it & 255u) == 255u && pipe_aborted(P)) return false;
        __nanosleep(20);
    }
    return false;
}

__device__ __forceinline__ bool pipe_wait_warp(uint64_t* bar, uint32_t parity, const PipeShared& P) {
    return __all_sync(kFull, pipe_wait(bar, parity, P));
}

__device__ __forceinline__ uint32_t ld_acquire_shared(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_shared(uint32_t* p, uint32_t v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

// Whole warp: wait until ring element qq has landed in its buffer.  A buffer
// may still hold an older element that another warp has not released (the
// stages of an item go to different warps), and a parity wait cannot tell
// that phase from qq's, so the buffer's fill tag must name qq first; the
// producer stores the tag (release) before it arms the barrier for qq.
__device__ __forceinline__ bool pipe_wait_stage(PipeShared& P, uint32_t qq, uint32_t nst) {
    const uint32_t b = qq % nst;
    bool ok = ld_acquire_shared(&P.fill[b]) == qq;
    for (uint32_t it = 0; !ok && it < kMaxWaitTries; ++it) {
        __nanosleep(64);
        ok = ld_acquire_shared(&P.fill[b]) == qq;
        if (!ok && (it & 15u) == 15u && pipe_aborted(P)) break;
    }
    if (!__all_sync(kFull, ok)) return false;
    return __all_sync(kFull, pipe_spin(&P.full[b], (qq / nst) & 1u, P));
}

// Hand a stage back to the producer.  The warp's shared loads of it have
// completed (their values decided the warp's branches), so a plain arrival
// orders them before the producer's next copy into the stage.
__device__ __forceinline__ void pipe_release(PipeShared& P, uint32_t b, int lane) {
    __syncwarp();
    if (lane == 0) mbar_arrive(&P.empty[b]);
}

// The largest x with a zero low half such that at least k of the warp's
// values (PER ordered keys per lane; 0 = no element) are >= x; 0 when fewer
// than k are nonzero.  Two bits per step: the counts of three trial values
// travel packed in one warp reduction (10 bits each).
template <int PER>
__device__ __forceinline__ uint32_t warp_kth_hi16(const uint32_t (&v)[PER], int k) {
    static_assert(PER * 32 < 1024, "packed 10-bit counts");
    uint32_t p = 0;  // high bits of the answer found so far
#pragma unroll 1
    for (int sh = 14; sh >= 0; sh -= 2) {
        const uint32_t t1 = (p | (1u << sh)) << 16, t2 = (p | (2u << sh)) << 16, t3 = (p | (3u << sh)) << 16;
        uint32_t c = 0;
#pragma unroll
        for (int j = 0; j < PER; ++j)
            c += (v[j] >= t1 ? 1u : 0u) + (v[j] >= t2 ? (1u << 10) : 0u) + (v[j] >= t3 ? (1u << 20) : 0u);
        c = __reduce_add_sync(kFull, c);
        const uint32_t kk = (uint32_t)k;
        const uint32_t d = ((c >> 20) >= kk) ? 3u : (((c >> 10) & 1023u) >= kk) ? 2u : ((c & 1023u) >= kk) ? 1u : 0u;
        p |= d << sh;
    }
    return p << 16;
}

// A 16-byte load from shared memory by its shared-window address.
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
    return r;
}

// One pass over a lane's 32 units of a stage (unit u = stage unit lane + 32u,
// present when 32u < left): the units' maxima in registers (NaN propagates,
// absent units are -inf) and the ordered maxima of its four groups of eight
// units (NaN skipped; 0 = no finite element).
template <typename T>
struct StageScan;

template <>
struct StageScan<__nv_bfloat16> {
    typedef __nv_bfloat162 B2;
    typedef __nv_bfloat162 Cmp;
    __device__ __forceinline__ static B2 w2(uint32_t w) { return *reinterpret_cast<const B2*>(&w); }
    __device__ __forceinline__ static uint32_t gkey(B2 m) {
        const float f = fmaxf(__low2float(m), __high2float(m));
        return (f > -__int_as_float(0x7f800000)) ? ord_of_float(__fadd_rn(f, 0.0f)) : 0u;
    }
    __device__ __forceinline__ static B2 ninf2() { return w2(0xff80ff80u); }
    // NaN or +inf in either half of a NaN-propagating maximum
    __device__ __forceinline__ static bool nonfinite(B2 m) {
        return !(__low2float(m) < __int_as_float(0x7f800000)) || !(__high2float(m) < __int_as_float(0x7f800000));
    }
    // The lane's units of a stage (unit u = stage unit lane + 32u, present when
    // 32u < left), one pass: bit u of the result is set when unit u is present
    // and some element of it is >= tau or NaN; lm gets the ordered key of the
    // lane's largest finite element (0: none), `bad` whether some element is
    // NaN or +inf.
    __device__ __forceinline__ static uint32_t flags_fused(const uint4* lsp, int left, Cmp tau, uint32_t& lm,
                                                           bool& bad) {
        const uint32_t sa = smem_u32(lsp);
        const uint4 ninf = Elem<__nv_bfloat16>::neg_inf_unit();
        uint32_t ub = 0;
        B2 mx = ninf2(), nn = ninf2();
        if (left >= 32 * kPLaneUnits) {  // every unit of the lane is present (all but a row's last stage)
#pragma unroll 4
            for (int u = 0; u < kPLaneUnits; ++u) {
                const B2 m = Elem<__nv_bfloat16>::umax(lds128(sa + (uint32_t)u * 512u));
                nn = __hmax2_nan(nn, m);
                mx = __hmax2(mx, m);
                ub |= (__hgeu2_mask(m, tau) != 0u ? 1u : 0u) << u;
            }
        } else {
#pragma unroll 4
            for (int u = 0; u < kPLaneUnits; ++u) {
                const bool here = 32 * u < left;
                const uint4 x = lds128(sa + (uint32_t)u * 512u);
                const uint4 r = here ? x : ninf;
                const B2 m = Elem<__nv_bfloat16>::umax(r);
                nn = __hmax2_nan(nn, m);
                mx = __hmax2(mx, m);
                ub |= (here && __hgeu2_mask(m, tau) != 0u ? 1u : 0u) << u;
            }
        }
        lm = gkey(mx);
        bad = nonfinite(nn);
        return ub;
    }
    // Statistics only (the threshold is not known yet): the ordered maxima of
    // the lane's four groups of eight units; returns the lane's maximum key.
    __device__ __forceinline__ static uint32_t stats(const uint4* lsp, int left, uint32_t (&gk)[kPGroups], bool& bad) {
        const uint32_t sa = smem_u32(lsp);
        const uint4 ninf = Elem<__nv_bfloat16>::neg_inf_unit();
        B2 nn = ninf2();
        uint32_t lm = 0;
#pragma unroll
        for (int g = 0; g < kPGroups; ++g) {
            B2 mx = ninf2();
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int u = 8 * g + v;
                const uint4 x = lds128(sa + (uint32_t)u * 512u);
                const uint4 r = (32 * u < left) ? x : ninf;
                const B2 m = Elem<__nv_bfloat16>::umax(r);
                nn = __hmax2_nan(nn, m);
                mx = __hmax2(mx, m);
            }
            gk[g] = gkey(mx);
            lm = gk[g] > lm ? gk[g] : lm;
        }
        bad = nonfinite(nn);
        return lm;
    }
    // Flags only (a second pass once the threshold is known).
    __device__ __forceinline__ static uint32_t flags(const uint4* lsp, int left, Cmp tau) {
        const uint32_t sa = smem_u32(lsp);
        uint32_t ub = 0;
#pragma unroll 4
        for (int u = 0; u < kPLaneUnits; ++u) {
            const bool here = 32 * u < left;
            const uint4 x = lds128(sa + (uint32_t)u * 512u);
            const uint4 r = here ? x : Elem<__nv_bfloat16>::neg_inf_unit();
            ub |= (here && __hgeu2_mask(Elem<__nv_bfloat16>::umax(r), tau) != 0u ? 1u : 0u) << u;
        }
        return ub;
    }
    // the unit comparand of a threshold value (rounded down to bf16)
    __device__ __forceinline__ static Cmp unit_cmp(float t) { return Elem<__nv_bfloat16>::make_tau(t); }
    // the element comparand of a threshold value: rounded down to bf16, and
    // never below the lowest finite value (so -inf elements stay out)
    __device__ __forceinline__ static Cmp cmp_of(float t) {
        const float lo = -3.3895313892515355e38f;  // lowest finite bf16
        const __nv_bfloat16 b = __float2bfloat16_rd(t > lo ? t : lo);
        return __halves2bfloat162(b, b);
    }
    // bit e: element e of the unit is >= c (NaN is not)
    __device__ __forceinline__ static uint32_t ge_mask(const uint4& r, Cmp c) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
        uint32_t m = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t g = __hge2_mask(w2(w[q]), c);
            m |= ((g & 1u) | ((g >> 15) & 2u)) << (2 * q);
        }
        return m;
    }
};

template <>
struct StageScan<float> {
    typedef float Cmp;
    __device__ __forceinline__ static uint32_t gkey(float f) {
        return (f > -__int_as_float(0x7f800000)) ? ord_of_float(__fadd_rn(f, 0.0f)) : 0u;
    }
    __device__ __forceinline__ static uint32_t flags_fused(const uint4* lsp, int left, Cmp tau, uint32_t& lm,
                                                           bool& bad) {
        const uint32_t sa = smem_u32(lsp);
        uint32_t ub = 0;
        float mx = -__int_as_float(0x7f800000), nn = -__int_as_float(0x7f800000);
        if (left >= 32 * kPLaneUnits) {  // every unit of the lane is present (all but a row's last stage)
#pragma unroll 4
            for (int u = 0; u < kPLaneUnits; ++u) {
                const float m = Elem<float>::umax(lds128(sa + (uint32_t)u * 512u));
                nn = Elem<float>::max_nan(nn, m);
                mx = fmaxf(mx, m);
                ub |= (!(m < tau) ? 1u : 0u) << u;
            }
        } else {
#pragma unroll 4
            for (int u = 0; u < kPLaneUnits; ++u) {
                const bool here = 32 * u < left;
                const uint4 x = lds128(sa + (uint32_t)u * 512u);
                const uint4 r = here ? x : Elem<float>::neg_inf_unit();
                const float m = Elem<float>::umax(r);
                nn = Elem<float>::max_nan(nn, m);
                mx = fmaxf(mx, m);
                ub |= (here && !(m < tau) ? 1u : 0u) << u;
            }
        }
        lm = gkey(mx);
        bad = !(nn < __int_as_float(0x7f800000));
        return ub;
    }
    __device__ __forceinline__ static uint32_t stats(const uint4* lsp, int left, uint32_t (&gk)[kPGroups], bool& bad) {
        const uint32_t sa = smem_u32(lsp);
        float nn = -__int_as_float(0x7f800000);
        uint32_t lm = 0;
#pragma unroll
        for (int g = 0; g < kPGroups; ++g) {
            float mx = -__int_as_float(0x7f800000);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int u = 8 * g + v;
                const uint4 x = lds128(sa + (uint32_t)u * 512u);
                const uint4 r = (32 * u < left) ? x : Elem<float>::neg_inf_unit();
                const float m = Elem<float>::umax(r);
                nn = Elem<float>::max_nan(nn, m);
                mx = fmaxf(mx, m);
            }
            gk[g] = gkey(mx);
            lm = gk[g] > lm ? gk[g] : lm;
        }
        bad = !(nn < __int_as_float(0x7f800000));
        return lm;
    }
    __device__ __forceinline__ static uint32_t flags(const uint4* lsp, int left, Cmp tau) {
        const uint32_t sa = smem_u32(lsp);
        uint32_t ub = 0;
#pragma unroll 4
        for (int u = 0; u < kPLaneUnits; ++u) {
            const bool here = 32 * u < left;
            const uint4 x = lds128(sa + (uint32_t)u * 512u);
            const uint4 r = here ? x : Elem<float>::neg_inf_unit();
            ub |= (here && !(Elem<float>::umax(r) < tau) ? 1u : 0u) << u;
        }
        return ub;
    }
    __device__ __forceinline__ static Cmp unit_cmp(float t) { return t; }
    __device__ __forceinline__ static Cmp cmp_of(float t) { return t > -3.402823466e38f ? t : -3.402823466e38f; }
    __device__ __forceinline__ static uint32_t ge_mask(const uint4& r, Cmp c) {
        return (__uint_as_float(r.x) >= c ? 1u : 0u) | (__uint_as_float(r.y) >= c ? 2u : 0u) |
               (__uint_as_float(r.z) >= c ? 4u : 0u) | (__uint_as_float(r.w) >= c ? 8u : 0u);
    }
};

// One consumer warp's candidates of one stage: every element of the lane's
// eight units that is >= the threshold (or NaN) is re-read from the stage
// and appended; one element per lane per round, positions by ballot.  The
// warp state travels by value (it stays in registers in the caller).
struct AppendState {
    int cnt;
    uint64_t tau;
    uint32_t bad;
};

template <typename T>
__device__ __noinline__ AppendState pipe_append(uint64_t* buf, int* wcnt, AppendState st, uint64_t m,
                                                const unsigned char* wstage, uint32_t id0, int hw, int k,
                                                unsigned long long* s_tau, int lane) {
    constexpr int KPU = Elem<T>::kPerUnit;
    const unsigned lt = lanemask_lt();
    while (__any_sync(kFull, m != 0ull)) {
        uint64_t key = 0ull;
        bool has = false;
        if (m != 0ull) {
            const int j = __ffsll((long long)m) - 1;
            m &= m - 1ull;
            const int u = j / KPU, e = j % KPU;
            const float v = Elem<T>::load_scalar(wstage + (size_t)(u * 32) * 16 + (size_t)e * Elem<T>::kBytes);
            if (v != v || v == __int_as_float(0x7f800000)) {
                st.bad |= 1u;
            } else if (v != -__int_as_float(0x7f800000)) {
                key = make_key(v, id0 + (uint32_t)(u * 32 * KPU + e));
                has = key > st.tau;
            }
        }
        const unsigned bal = __ballot_sync(kFull, has);
        if (has) buf[st.cnt + __popc(bal & lt)] = key;
        st.cnt += __popc(bal);
        if (st.cnt > hw) {
            __syncwarp();
            const Compacted cp = warp_compact(buf, wcnt, st.cnt, st.tau, k, s_tau, lane);
            st.cnt = cp.cnt;
            st.tau = cp.tau;
        }
    }
    __syncwarp();
    return st;
}

// The candidates of one stage (ub = the lane's units, of its 32, whose
// maximum may reach the threshold): each round every lane with a unit
// left re-reads it from the stage, masks its finite elements >= the
// threshold, and writes them at positions from bit-sliced ballots of the
// per-lane counts.  A round that would overflow the buffer goes one element
// per lane at a time with compaction in between (pipe_append).
template <typename T>
__device__ __noinline__ AppendState pipe_units(uint64_t* buf, int* wcnt, AppendState st, uint32_t ub,
                                               const uint4* sp, uint32_t id0, int hw, int cap_w, int k,
                                               unsigned long long* s_tau, int lane) {
    constexpr int KPU = Elem<T>::kPerUnit;
    const unsigned lt = lanemask_lt();
    while (__any_sync(kFull, ub != 0u)) {
        const float tf = tau_value(st.tau);
        uint32_t em = 0;
        uint4 r = make_uint4(0u, 0u, 0u, 0u);
        int u = 0;
        if (ub != 0u) {
            u = __ffs(ub) - 1;
            ub &= ub - 1u;
            r = sp[u * 32];
            em = Elem<T>::elem_mask(r, tf, st.bad);
        }
        const uint32_t c = (uint32_t)__popc(em);  // <= 8
        const unsigned b0 = __ballot_sync(kFull, c & 1u), b1 = __ballot_sync(kFull, c & 2u);
        const unsigned b2 = __ballot_sync(kFull, c & 4u), b3 = __ballot_sync(kFull, c & 8u);
        const int tot = __popc(b0) + 2 * __popc(b1) + 4 * __popc(b2) + 8 * __popc(b3);
        if (tot == 0) continue;
        if (st.cnt + tot > cap_w) {
            st = pipe_append<T>(buf, wcnt, st, (uint64_t)em, reinterpret_cast<const unsigned char*>(sp + u * 32),
                                id0 + (uint32_t)(u * 32 * KPU), hw, k, s_tau, lane);
            continue;
        }
        int pos = st.cnt + __popc(b0 & lt) + 2 * __popc(b1 & lt) + 4 * __popc(b2 & lt) + 8 * __popc(b3 & lt);
        const uint32_t idu = id0 + (uint32_t)(u * 32 * KPU);
        while (em != 0u) {
            const int e = __ffs(em) - 1;
            em &= em - 1u;
            buf[pos++] = make_key(Elem<T>::get(r, e), idu + (uint32_t)e);
        }
        st.cnt += tot;
        if (st.cnt > hw) {
            __syncwarp();
            const Compacted cp = warp_compact(buf, wcnt, st.cnt, st.tau, k, s_tau, lane);
            st.cnt = cp.cnt;
            st.tau = cp.tau;
        }
    }
    __syncwarp();
    return st;
}

// The candidates of one stage, lane-parallel: every lane counts the
// elements >= the threshold value in its flagged units, one warp scan gives
// each lane its write position, and each lane writes its own keys.  Returns
// the new count, or -1 (nothing written) when they would not fit in cap_w.
template <typename T>
__device__ __forceinline__ int extract_fast(uint64_t* buf, int cnt, uint32_t ub, const uint4* lsp, uint64_t tau,
                                            uint32_t id0, int cap_w, int lane) {
    typedef StageScan<T> SS;
    constexpr int KPU = Elem<T>::kPerUnit;
    const typename SS::Cmp cmp = SS::cmp_of(tau_value(tau));
    int c = 0;
    const uint32_t sa = smem_u32(lsp);
    for (uint32_t m = ub; m != 0u; m &= m - 1u) c += __popc(SS::ge_mask(lds128(sa + (uint32_t)(__ffs(m) - 1) * 512u), cmp));
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += t;
    }
    const int total = __shfl_sync(kFull, incl, 31);
    if (cnt + total > cap_w) return -1;
    int pos = cnt + incl - c;
    for (uint32_t m = ub; m != 0u; m &= m - 1u) {
        const int u = __ffs(m) - 1;
        const uint4 r = lds128(sa + (uint32_t)u * 512u);
        uint32_t em = SS::ge_mask(r, cmp);
        const uint32_t idu = id0 + (uint32_t)(u * 32 * KPU);
        while (em != 0u) {
            const int e = __ffs(em) - 1;
            em &= em - 1u;
            buf[pos++] = make_key(Elem<T>::get(r, e), idu + (uint32_t)e);
        }
    }
    __syncwarp();
    return cnt + total;
}

// The CTA threshold of a piece, read once and given to the whole warp (so
// that every lane takes the same branches).
__device__ __forceinline__ uint64_t read_tau(const unsigned long long* s_tau) {
    uint64_t v = 0ull;
    if ((threadIdx.x & 31) == 0) v = *reinterpret_cast<const volatile unsigned long long*>(s_tau);
    return __shfl_sync(kFull, v, 0);
}

// Whole warp or one thread: wait until a shared flag is set (acquire).
__device__ __forceinline__ bool wait_flag(const uint32_t* f, const PipeShared& P) {
    for (uint32_t it = 0; it < kMaxWaitTries; ++it) {
        if (ld_acquire_shared(f) != 0u) return true;
        if ((it & 15u) == 15u && pipe_aborted(P)) return false;
        __nanosleep(64);
    }
    return false;
}

// The CTA's list of items: one per row its range touches (main items), then
// the rows of its redo pass.  Every role walks it in the same order.
struct PipeList {
    CtaRange cr;
    int64_t nmain, rbase;  // main items; the redo rows' offset in J.redo
    bool rot;              // the last row is cut by the CTA's end: it goes first
    int64_t nredo;         // known after the main items (-1 before)
    int64_t full_units;    // units of a whole row (for "big" pieces)
    bool spec_ok;          // rows are long enough for predictions
    bool dyn;              // rows handed out at run time (whole rows; nmain known at the end)
};

template <typename T>
__device__ __forceinline__ PipeList pipe_list(const RowJob& J) {
    PipeList L;
    L.cr = cta_range<T>(J);
    L.nmain = L.cr.row1 - L.cr.row0 + 1;
    L.rbase = L.cr.row0 + L.cr.b;
    // a row split across two CTAs is merged by the one that finishes its
    // piece last; taking the CTA's last (split) row first, as the next CTA
    // takes it first too, keeps merges away from the end of the kernel
    L.rot = L.nmain > 1 && (L.cr.e % L.cr.nu) != 0;
    L.nredo = -1;
    L.full_units = L.cr.nu;
    // predictions read the spacing of a row's k best values; rows must hold
    // several times k elements
    L.spec_ok = J.k >= 8 && L.cr.nu * Elem<T>::kPerUnit >= (int64_t)16 * J.k;
    L.dyn = J.dyn != nullptr;
    if (L.dyn) {
        L.nmain = -1;
        L.rot = false;
    }
    return L;
}

// The piece of an item: a whole row when it is read again or rows are
// handed out at run time, else the CTA's share of it.
template <typename T>
__device__ __forceinline__ Piece item_piece(const RowJob& J, const PipeList& L, int64_t row, bool redo) {
    return (redo || L.dyn) ? whole_row<T>(J, L.cr, row) : piece_of<T>(J, L.cr, row);
}

// Row of main item i.
__device__ __forceinline__ int64_t main_row(const PipeList& L, int64_t i) {
    if (!L.rot) return L.cr.row0 + i;
    return i == 0 ? L.cr.row1 : L.cr.row0 + i - 1;
}

// A main piece whose group maxima publish a prediction: at least a quarter
// of a row.
__device__ __forceinline__ bool piece_big(const PipeList& L, const Piece& p) {
    return L.spec_ok && (int64_t)(p.ue - p.ub) * 4 >= L.full_units;
}

// Producer (one thread).
template <typename T, int MODE>
__device__ void pipe_produce(const RowJob& J, PipeShared& P, unsigned char* ring) {
    PipeList L = pipe_list<T>(J);
    const uint32_t nst = (uint32_t)J.nst;
    uint32_t q = 0;
    bool ok = true;
    // ticket: when not null, the next row's ticket is taken kTicketAhead
    // stages before this piece's last copy (its answer is needed only then)
    auto issue = [&](const Piece& p, uint32_t* ticket) {
        const int at = p.nstage > kTicketAhead ? p.nstage - kTicketAhead : 0;
        // a piece with no stage (a row of head and tail scalars only) still takes its ticket
        if (ticket != nullptr && p.nstage == 0) *ticket = atomicAdd(J.dyn + kDynNext, 1u);
        for (int st = 0; ok && st < p.nstage; ++st) {
            if (ticket != nullptr && st == at) *ticket = atomicAdd(J.dyn + kDynNext, 1u);
            const uint32_t b = q % nst;
            if (q >= nst && !pipe_spin(&P.empty[b], ((q / nst) - 1u) & 1u, P)) {
                ok = false;
                break;
            }
            if (pipe_aborted(P)) {
                ok = false;
                break;
            }
            const int u0 = p.ub + st * kPStageUnits;
            const int nu = (p.ue - u0) < kPStageUnits ? (p.ue - u0) : kPStageUnits;
            st_release_shared(&P.fill[b], q);  // the buffer now belongs to element q
            mbar_expect_tx(&P.full[b], (uint32_t)nu * 16u);
            bulk_g2s(ring + (size_t)b * kPStageBytes, p.ubase + (size_t)u0 * 16, (uint32_t)nu * 16u, &P.full[b]);
            ++q;
        }
    };
    if (L.dyn) {
        // take rows until none is left: first the counter's, then rows that a
        // finisher posted for a second read; a row is done once some finisher
        // has finished it, so the producers stop when every row is
        auto post = [&](int64_t i, long long e) {
            P.qrow[i % kDynQ] = e;
            st_release_shared(&P.qseq[i % kDynQ], (uint32_t)(i + 1));
        };
        uint32_t* dc = J.dyn;
        int64_t i = 0;
        // the counter only grows, so once past the rows it stays past them
        uint32_t r = atomicAdd(dc + kDynNext, 1u);
        for (; ok; ++i) {
            if ((int64_t)r < J.rows) {
                post(i, (long long)r);
                uint32_t nx = 0xffffffffu;
                issue(whole_row<T>(J, L.cr, (int64_t)r), &nx);
                r = nx;
                continue;
            }
            long long e = -1;
            bool found = false;
            for (uint32_t it = 0; it < kMaxWaitTries && !pipe_aborted(P); ++it) {
                // the three counters in one round trip.  Every row finished
                // means no retry is outstanding (a posted row counts as
                // finished only once its second read has finished it).
                const uint32_t put0 = *reinterpret_cast<volatile uint32_t*>(dc + kDynRetryPut);
                uint32_t t = *reinterpret_cast<volatile uint32_t*>(dc + kDynRetryGet);
                const uint32_t fin0 = *reinterpret_cast<volatile uint32_t*>(dc + kDynFinished);
                if (t >= put0 && fin0 >= (uint32_t)J.rows) break;
                // claim the next posted retry: the taken count only moves from t
                // to t + 1 while t is below the posted count (which only grows)
                bool claimed = false;
                while (t < *reinterpret_cast<volatile uint32_t*>(dc + kDynRetryPut)) {
                    const uint32_t seen = atomicCAS(dc + kDynRetryGet, t, t + 1u);
                    if (seen == t) {
                        claimed = true;
                        break;
                    }
                    t = seen;
                }
                if (claimed) {
                    // the poster writes the entry after taking its index: wait for it
                    volatile uint32_t* slot = dc + kDynWords + t;
                    uint32_t v = 0;
                    for (uint32_t w = 0; w < kMaxWaitTries && (v = *slot) == 0u; ++w) __nanosleep(32);
                    if (v != 0u) {
                        *slot = 0u;  // back to zero for the next call
                        e = (long long)(v - 1u) | (1ll << 62);
                        found = true;
                    }
                    break;
                }
                __nanosleep(64);
            }
            if (!found) break;
            post(i, e);
            issue(whole_row<T>(J, L.cr, (int64_t)(e & ((1ll << 62) - 1))), nullptr);
        }
        post(i, -1);
        if (!ok) atomicExch(&P.abort, 1);
        for (uint32_t d = q > nst ? q - nst : 0u; d < q; ++d) (void)mbar_wait_bounded(&P.full[d % nst], (d / nst) & 1u);
        return;
    }
    for (int64_t i = 0; ok && i < L.nmain; ++i) {
        const int64_t row = main_row(L, i);
        if (item_active<MODE>(J, row)) issue(piece_of<T>(J, L.cr, row), nullptr);
    }
    // the redo pass: rows whose prediction failed, read whole
    if (ok && wait_flag(&P.redo_ready, P)) {
        const int n = *reinterpret_cast<volatile int*>(&P.redo_n);
        for (int j = 0; ok && j < n; ++j)
            issue(whole_row<T>(J, L.cr, (int64_t)__ldcg(J.redo + L.rbase + j)), nullptr);
    } else {
        ok = false;
    }
    if (!ok) atomicExch(&P.abort, 1);
    // the copies still in flight land before the CTA may exit (bounded)
    for (uint32_t d = q > nst ? q - nst : 0u; d < q; ++d) (void)mbar_wait_bounded(&P.full[d % nst], (d / nst) & 1u);
}

// The item of ordinal i for a consumer or finisher warp (whole warp): false
// past the end of the list.  Waits for the redo list at the end of the main
// items.
template <typename T>
__device__ __forceinline__ bool pipe_item(const RowJob& J, PipeShared& P, PipeList& L, int64_t i, int64_t& row,
                                          bool& redo) {
    if (L.dyn) {
        // run-time rows: entry i of the queue (the producer posts -1 at the end)
        const uint32_t* seq = &P.qseq[i % kDynQ];
        bool ok = true;
        if (__shfl_sync(kFull, ld_acquire_shared(seq), 0) != (uint32_t)(i + 1)) {
            ok = false;
            for (uint32_t it = 0; it < kMaxWaitTries; ++it) {
                if (ld_acquire_shared(seq) == (uint32_t)(i + 1)) {
                    ok = true;
                    break;
                }
                if ((it & 15u) == 15u && pipe_aborted(P)) break;
                __nanosleep(64);
            }
            ok = __all_sync(kFull, ok);
        }
        if (!ok) return false;
        const long long e = *reinterpret_cast<const volatile long long*>(&P.qrow[i % kDynQ]);
        if (e < 0) return false;
        row = (int64_t)(e & ((1ll << 62) - 1));
        redo = (e >> 62) != 0;
        return true;
    }
    if (i < L.nmain) {
        row = main_row(L, i);
        redo = false;
        return true;
    }
    if (L.nredo < 0) {
        const bool ok = __all_sync(kFull, wait_flag(&P.redo_ready, P));
        L.nredo = ok ? (int64_t)*reinterpret_cast<volatile int*>(&P.redo_n) : 0;
        L.nredo = __shfl_sync(kFull, L.nredo, 0);
    }
    if (i >= L.nmain + L.nredo) return false;
    row = (int64_t)__ldcg(J.redo + L.rbase + (i - L.nmain));
    redo = true;
    return true;
}

// A piece's seed from the lane maxima of its first nA stages (32 per
// stage; stage j's at bv[32 j .. 32 j + 31]).  Distinct lanes of distinct
// stages hold distinct elements, so at least k elements are >= the result.
__device__ __forceinline__ uint32_t boot_threshold(const uint32_t* bv, int nA, int k, int lane) {
    uint32_t v[kPBootStages];
    const bool mine = (lane * kPBootStages) / 32 < nA;  // lane's values belong to stage lane / 4
#pragma unroll
    for (int j = 0; j < kPBootStages; j += 4) {
        const uint4 x = mine ? reinterpret_cast<const uint4*>(bv + lane * kPBootStages)[j / 4] : make_uint4(0, 0, 0, 0);
        v[j] = x.x;
        v[j + 1] = x.y;
        v[j + 2] = x.z;
        v[j + 3] = x.w;
    }
    return warp_kth_hi16<kPBootStages>(v, k);
}


// Consumer warp c (0 .. kPipeConsumers-1): ring elements q with q % 8 == c.
// Joint order: add a stage's elements to the lane's pair (m, s).  lm is the
// ordered key of the lane's largest finite element in the stage (0: none).
// The stage's terms go to four float sums (independent chains of at most 64
// terms each), then to s in double.
template <typename T>
__device__ __forceinline__ void joint_stage(const uint4* lsp, int left, uint32_t lm, JointScale c, float& m,
                                            double& s) {
    if (lm != 0u) joint_raise(m, s, float_of_ord(lm), c);
    float t[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 4
    for (int u = 0; u < kPLaneUnits; ++u) {
        if (32 * u < left) {
            const uint4 r = lsp[u * 32];
#pragma unroll
            for (int e = 0; e < Elem<T>::kPerUnit; ++e) t[e & 3] += joint_term_fast(Elem<T>::get(r, e), m, c);
        }
    }
    s += (double)((t[0] + t[1]) + (t[2] + t[3]));
}

// A warp's pairs merged into every lane.
__device__ __forceinline__ void joint_warp_merge(float& m, double& s, JointScale c) {
#pragma unroll 1
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(kFull, m, o);
        const double s2 = __shfl_xor_sync(kFull, s, o);
        joint_merge(m, s, m2, s2, c);
    }
}

constexpr float kLowestFloat = -3.402823466e38f;

template <typename T, int MODE, int PR>
__device__ void pipe_consume(const RowJob& J, PipeShared& P, const unsigned char* ring, uint64_t* slots, int c,
                             int lane) {
    typedef StageScan<T> SS;
    constexpr int KPU = Elem<T>::kPerUnit;
    PipeList L = pipe_list<T>(J);
    const uint32_t nst = (uint32_t)J.nst;
    const int k = J.k, hw = J.hw, cap_w = J.cap_w;
    uint32_t q = 0;              // ring element of the piece's first stage
    uint32_t used = 0, par = 0;  // per slot: used before; parity of its current use
    bool fail = false;
    int64_t row = 0;
    bool redo = false;
    for (int64_t i = 0; pipe_item<T>(J, P, L, i, row, redo); ++i) {
        if (!item_active<MODE>(J, row)) continue;
        const int slot = (int)(i % kPipeSlots);
        const uint32_t sb = 1u << slot;
        // the finisher is done with this slot's previous piece
        if ((used & sb) && !pipe_wait_warp(&P.slot_empty[slot], (par & sb) ? 0u : 1u, P)) fail = true;
        const Piece p = item_piece<T>(J, L, row, redo);
        // joint order: the piece's pair (m, s) over every element it reads
        bool jon = false;
        JointScale jc{0.0f, 0.0f};
        if (PR && J.joint) {
            const RowParams rp = row_params<MODE>(J, row);
            jon = rp.ok && rp.T > 0.0f;
            if (jon) jc = joint_scale(rp.T);
        }
        float jm = kLowestFloat;
        double js = 0.0;
        // a cycle's draft rows and target rows keep separate predictions
        const int pset = row_set<MODE>(J, row);
        // the first consumer warp to start the piece fixes its mode: predicted
        // when a prediction exists by then (nobody waits for one)
        uint32_t mode = 0;
        if (lane == 0) {
            const uint32_t want = (!redo && L.spec_ok && ld_acquire_shared(&P.spec_set[pset]) != 0u) ? 1u : 2u;
            const uint32_t old = atomicCAS(&P.mode[slot], 0u, want);
            mode = old == 0u ? want : old;
        }
        const bool predicted = __shfl_sync(kFull, mode, 0) == 1u;
        const int nA = p.nstage < kPBootStages ? p.nstage : kPBootStages;
        // a seed from lane maxima needs about 2k lanes that hold elements
        // (a short last stage has fewer); else each stage seeds itself
        int lanes = 0;
        for (int st = 0; st < nA; ++st) {
            const int u = p.ue - (p.ub + st * kPStageUnits);
            lanes += u < 32 ? u : 32;
        }
        const bool boot = !predicted && lanes >= 2 * k;
        unsigned long long* s_tau = &P.tau[slot];

        WarpState ws;
        ws.buf = slots + ((size_t)slot * kPipeConsumers + c) * cap_w;
        ws.wcnt = &P.wcnt[c];
        ws.cnt = 0;
        ws.bad = 0u;
        if (c == 1 && p.seg == 0) {
            // row head / tail scalars (fewer than 16): every finite one
            const int64_t ntail = J.vocab - p.g.tail_begin;
            const int64_t nsc = p.g.head + ntail;
            uint64_t key = 0ull;
            bool has = false;
            if (lane < nsc) {
                const int64_t id = (lane < p.g.head) ? (int64_t)lane : p.g.tail_begin + (lane - p.g.head);
                const float v = Elem<T>::load_scalar(p.g.base + (size_t)id * Elem<T>::kBytes);
                if (v != v || v == __int_as_float(0x7f800000)) {
                    ws.bad |= 1u;
                } else if (v != -__int_as_float(0x7f800000)) {
                    key = make_key(v, (uint32_t)id);
                    has = true;
                    if (jon) {
                        joint_raise(jm, js, v, jc);
                        js += (double)joint_term(v, jm, jc);
                    }
                }
            }
            const unsigned bal = __ballot_sync(kFull, has);
            if (has) ws.buf[__popc(bal & lanemask_lt())] = key;
            ws.cnt = __popc(bal);
        }
        ws.tau = read_tau(s_tau);
        if (predicted) {
            // the latest prediction of this CTA
            const uint64_t t = read_tau(&P.spec[pset]);
            if (t > ws.tau) ws.tau = t;
            if (lane == 0) {
                atomicMax(&P.used[slot], (unsigned long long)t);
                atomicMax(s_tau, (unsigned long long)t);
            }
        }

        const uint32_t id_base = (uint32_t)p.g.head;
        const int st0 = (int)((uint32_t)(c + kPipeConsumers) - q % kPipeConsumers) % kPipeConsumers;
        for (int st = st0; st < p.nstage && !fail; st += kPipeConsumers) {
            const uint32_t qq = q + st;
            const uint32_t b = qq % nst;
            if (!pipe_wait_stage(P, qq, nst)) {
                fail = true;
                break;
            }
            const int su = p.ub + st * kPStageUnits;  // the stage's first unit in the row
            const int left = (p.ue - su) - lane;       // the lane's unit u is present when 32 u < left
            const uint4* lsp = reinterpret_cast<const uint4*>(ring + (size_t)b * kPStageBytes) + lane;
            uint32_t ub, lm;
            bool nonfin = false;
            if (predicted) {
                // one pass: the threshold is known
                {
                    const uint64_t stv = read_tau(s_tau);
                    if (stv > ws.tau) ws.tau = stv;
                }
                ub = SS::flags_fused(lsp, left, SS::unit_cmp(tau_value(ws.tau)), lm, nonfin);
            } else {
                uint32_t gk[kPGroups];
                lm = SS::stats(lsp, left, gk, nonfin);
                if (boot) {
                    // the piece's seed: lane maxima of its first nA stages; the
                    // consumer that completes them searches, every stage waits
                    if (st < nA) {
                        P.boot[slot][st * 32 + lane] = lm;
                        __threadfence_block();
                        __syncwarp();
                        int last = 0;
                        if (lane == 0) last = atomicAdd(&P.boot_cnt[slot], 1) == nA - 1;
                        if (__shfl_sync(kFull, last, 0)) {
                            __threadfence_block();
                            const uint64_t t = (uint64_t)boot_threshold(P.boot[slot], nA, k, lane) << 32;
                            if (lane == 0) {
                                atomicMax(s_tau, (unsigned long long)t);
                                // until a big piece completes, its seed is the CTA's
                                // prediction (about 2.6 k elements of a row reach it)
                                if (!redo && piece_big(L, p) && P.spec_set[pset] == 0u) {
                                    P.spec[pset] = t;
                                    __threadfence_block();
                                    st_release_shared(&P.spec_set[pset], 1u);
                                }
                                st_release_shared(&P.boot_ready[slot], 1u);
                            }
                        }
                    }
                    if (!__all_sync(kFull, wait_flag(&P.boot_ready[slot], P))) fail = true;
                } else {
                    // one-stage seed: the k-th largest of this stage's group maxima
                    const uint32_t th = (uint32_t)(ws.tau >> 32);
                    uint32_t n = 0;
#pragma unroll
                    for (int g = 0; g < kPGroups; ++g) n += gk[g] > th ? 1u : 0u;
                    if (__reduce_add_sync(kFull, n) >= (uint32_t)k) {
                        const uint64_t t = (uint64_t)warp_kth_hi16<kPGroups>(gk, k) << 32;
                        if (t > ws.tau) {
                            ws.tau = t;
                            if (lane == 0) atomicMax(s_tau, (unsigned long long)t);
                        }
                    }
                }
                {
                    const uint64_t stv = read_tau(s_tau);
                    if (stv > ws.tau) ws.tau = stv;
                }
                ub = SS::flags(lsp, left, SS::unit_cmp(tau_value(ws.tau)));
            }
            if (nonfin) ws.bad |= 1u;
            if (jon) joint_stage<T>(lsp, left, lm, jc, jm, js);
            if (__any_sync(kFull, ub != 0u)) {
                const uint32_t id0 = id_base + (uint32_t)(su + lane) * KPU;
                const int nc = extract_fast<T>(ws.buf, ws.cnt, ub, lsp, ws.tau, id0, cap_w, lane);
                if (nc >= 0) {
                    ws.cnt = nc;
                    if (ws.cnt > hw) {
                        const Compacted cp = warp_compact(ws.buf, ws.wcnt, ws.cnt, ws.tau, k, s_tau, lane);
                        ws.cnt = cp.cnt;
                        ws.tau = cp.tau;
                    }
                } else {  // rare: the stage's candidates overflow the buffer; append with compaction
                    const AppendState r = pipe_units<T>(ws.buf, ws.wcnt, AppendState{ws.cnt, ws.tau, 0u}, ub, lsp,
                                                        id0, hw, cap_w, k, s_tau, lane);
                    ws.cnt = r.cnt;
                    ws.tau = r.tau;
                }
            }
            pipe_release(P, b, lane);
        }
        {
            const uint64_t stv = read_tau(s_tau);
            if (stv > ws.tau) ws.tau = stv;
            ws.cnt = warp_keep_ge(ws.buf, ws.cnt, ws.tau, lane);
        }
        const uint32_t wb = __reduce_or_sync(kFull, ws.bad | (fail ? 2u : 0u));
        if (jon) joint_warp_merge(jm, js, jc);
        if (lane == 0) {
            P.jm[slot][c] = jm;
            P.js[slot][c] = js;
            P.cnt[slot][c] = ws.cnt;
            if (wb) atomicOr(&P.bad[slot], wb);
            mbar_arrive(&P.slot_full[slot]);
        }
        if (fail && lane == 0) atomicExch(&P.abort, 1);
        q += (uint32_t)p.nstage;
        par ^= sb;
        used |= sb;
    }
}

// Ascending bitonic merge of a bitonic sequence of 64 keys (element e = lane
// in a, e = lane + 32 in b).
__device__ __forceinline__ void warp_merge64(uint64_t& a, uint64_t& b, int lane) {
    {
        const uint64_t lo = a < b ? a : b, hi = a < b ? b : a;
        a = lo;
        b = hi;
    }
#pragma unroll 1
    for (int stride = 16; stride > 0; stride >>= 1) {
        const uint64_t pa = __shfl_xor_sync(kFull, a, stride), pb = __shfl_xor_sync(kFull, b, stride);
        const bool lower = (lane & stride) == 0;
        a = lower ? (a < pa ? a : pa) : (a < pa ? pa : a);
        b = lower ? (b < pb ? b : pb) : (b < pb ? pb : b);
    }
}

// The best min(k, U) of U distinct keys get(0 .. U-1) (k <= 64), written to
// sel[] in descending order; one warp.  Chunks of 64 are sorted and merged
// into a running best 64 (the 64 smallest complements).
template <class Get>
__device__ __forceinline__ int warp_topk64(int U, int k, const Get& get, uint64_t* sel, int lane) {
    uint64_t ra = ~0ull, rb = ~0ull;
    for (int base = 0; base < U; base += 64) {
        uint64_t xa = base + lane < U ? ~get(base + lane) : ~0ull;
        uint64_t xb = base + 32 + lane < U ? ~get(base + 32 + lane) : ~0ull;
        warp_sort64(xa, xb, lane);
        if (base == 0) {
            ra = xa;
            rb = xb;
        } else {
            // element e pairs with chunk element 63 - e
            const uint64_t ca = __shfl_xor_sync(kFull, xb, 31), cb = __shfl_xor_sync(kFull, xa, 31);
            ra = ra < ca ? ra : ca;
            rb = rb < cb ? rb : cb;
            warp_merge64(ra, rb, lane);
        }
    }
    const int n = U < k ? U : k;
    if (lane < n) sel[lane] = ~ra;
    if (lane + 32 < n) sel[lane + 32] = ~rb;
    __syncwarp();
    return n;
}

// The best min(k, U) of U distinct keys g[0..U) (U <= kPGather), into
// sel[] in descending order, by rank: each key's rank is the number of
// larger keys, counted against g[] in shared memory (independent loads, no
// shuffle chain).  One warp.
__device__ __noinline__ int warp_rank_topk(const uint64_t* g, int U, int k, uint64_t* sel, int lane) {
    for (int i0 = 0; i0 < U; i0 += 64) {
        const int ia = i0 + lane, ib = i0 + 32 + lane;
        const uint64_t ka = ia < U ? g[ia] : ~0ull, kb = ib < U ? g[ib] : ~0ull;
        int ra = 0, rb = 0;
#pragma unroll 4
        for (int j = 0; j < U; ++j) {
            const uint64_t x = g[j];
            ra += x > ka ? 1 : 0;
            rb += x > kb ? 1 : 0;
        }
        if (ia < U && ra < k) sel[ra] = ka;
        if (ib < U && rb < k) sel[rb] = kb;
    }
    __syncwarp();
    return U < k ? U : k;
}

// The best min(k, U) of U distinct keys g[0..U) (U <= kPGather), into
// sel[] in descending order: first cut g to the keys whose high half lies in
// the k-th largest one's bucket or above, then rank the rest.  The buckets
// split the keys' range of high halves [bot, top] into at most 64 classes
// of 2^shift values each, counted into hist[64] (shared memory).  Whole
// buckets are kept, so the cut keeps the best k and at least k keys.
__device__ __noinline__ int warp_select_topk(uint64_t* g, int U, int k, uint64_t* sel, uint32_t* hist, int lane) {
    if (U > k + 8) {
        constexpr int PER = kPGather / 32;
        uint32_t v[PER];
        uint32_t vmax = 0u, vmin = 0xffffffffu;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const bool here = lane + 32 * j < U;
            v[j] = here ? (uint32_t)(g[lane + 32 * j] >> 32) : 0u;
            vmax = here && v[j] > vmax ? v[j] : vmax;
            vmin = here && v[j] < vmin ? v[j] : vmin;
        }
        const uint32_t top = __reduce_max_sync(kFull, vmax), bot = __reduce_min_sync(kFull, vmin);
        const uint32_t span = top - bot;
        const int shift = span < 64u ? 0 : 26 - __clz(span);  // span >> shift < 64
        hist[lane] = 0u;
        hist[lane + 32] = 0u;
        __syncwarp();
#pragma unroll
        for (int j = 0; j < PER; ++j)
            if (lane + 32 * j < U) atomicAdd(&hist[(top - v[j]) >> shift], 1u);  // bucket 0 holds top
        __syncwarp();
        // running counts from the top: lane l holds buckets 2l and 2l + 1
        const uint32_t c0 = hist[2 * lane], c1 = hist[2 * lane + 1];
        uint32_t incl = c0 + c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += t;
        }
        const bool first_half = incl - c1 >= (uint32_t)k;
        const unsigned reach = __ballot_sync(kFull, incl >= (uint32_t)k);  // a suffix of the lanes (U >= k)
        const int L = __ffs(reach) - 1;
        const int bstar = 2 * L + (__shfl_sync(kFull, first_half, L) ? 0 : 1);
        // keep the keys of buckets 0..bstar: top - hi < (bstar + 1) << shift
        int64_t lo = (int64_t)top - ((int64_t)(bstar + 1) << shift) + 1;
        lo = lo < 0 ? 0 : lo;
        __syncwarp();
        U = warp_keep_ge(g, U, (uint64_t)lo << 32, lane);
    }
    return warp_rank_topk(g, U, k, sel, lane);
}

// The CTA's next prediction from a finished row's best keys sel[0..n)
// (descending): the value that about 2.5 k elements of a row like it reach.
// Near the top of a row the values fall about linearly in the log of the
// rank, so the drop from rank k/2 to rank k, scaled by log(2.5k / k) /
// log(k / (k/2)), extrapolates to rank 2.5 k.  A row that failed its
// prediction (fewer than k kept at or above it) lowers the next one below
// its last kept value by twice the same spread.  0 when there is no basis.
__device__ __forceinline__ uint64_t next_prediction(const uint64_t* sel, int n, int k, bool held) {
    if (n < 2) return 0ull;
    const int last = (held ? k : n) - 1;
    const int mid = last / 2;
    const float vl = key_value(sel[last]), vm = key_value(sel[mid]);
    const float d = vm - vl;
    if (!(d > 0.0f)) return 0ull;
    const float f = held ? logf(2.5f * (float)(last + 1)) - logf((float)(last + 1)) : 2.0f * logf((float)(last + 1) / (float)(mid + 1));
    const float v = vl - d * f / logf((float)(last + 1) / (float)(mid + 1));
    if (!(v > -3.0e38f) || !(v < 3.0e38f)) return 0ull;
    return (uint64_t)ord_of_float(__fadd_rn(v, 0.0f)) << 32;
}

// The last finishing warp of a split row: the best min(k, U) keys of the U
// keys its pieces published, into sel[] (descending); rowbad gets the OR of
// the pieces' flags and `spec` the largest predicted threshold any piece
// was filtered by.  Piece t's keys sit in part slot slot_t and occupy
// indices [excl_t, excl_t + count_t) of the merged order (lane t holds
// both; at most kPipeMaxPieces pieces).
struct Merged {
    int n;
    uint32_t rowbad;
    uint64_t spec;
    float jm;  // joint order: the row's pair (m, s) from its pieces' pairs
    double js;
};
__device__ __noinline__ Merged merge_pieces(const RowJob& J, int64_t T, int64_t G, int64_t nu, int64_t row,
                                            int64_t first_cta, int np, uint64_t* sel, int lane, bool jon,
                                            JointScale jc) {
    CtaRange c;
    c.T = T;
    c.G = G;
    c.nu = nu;
    const int64_t myslot = lane < np ? part_slot(c, first_cta + lane, row) : 0;
    const int c_l = lane < np ? __ldcg(J.part_count + myslot) : 0;
    const uint32_t rowbad = __reduce_or_sync(kFull, lane < np ? __ldcg(J.part_flags + myslot) : 0u);
    uint64_t sp = lane < np ? (uint64_t)__ldcg(reinterpret_cast<const unsigned long long*>(J.part_spec) + myslot) : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t t = __shfl_xor_sync(kFull, sp, o);
        sp = t > sp ? t : sp;
    }
    int incl = c_l;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += t;
    }
    const int U = __shfl_sync(kFull, incl, 31);
    const int excl = incl - c_l;
    const int kk = J.k;
    const unsigned long long* pbase = reinterpret_cast<const unsigned long long*>(J.part_keys);
    uint64_t ra = ~0ull, rb = ~0ull;
    for (int base = 0; base < U; base += 64) {
        const int ga = base + lane, gb = base + 32 + lane;
        int sa = 0, sg = 0;
        for (int t = 1; t < np; ++t) {
            const int e = __shfl_sync(kFull, excl, t);
            sa = (e <= ga) ? t : sa;
            sg = (e <= gb) ? t : sg;
        }
        const int ea = __shfl_sync(kFull, excl, sa), eb = __shfl_sync(kFull, excl, sg);
        const int64_t pa = __shfl_sync(kFull, myslot, sa), pb = __shfl_sync(kFull, myslot, sg);
        uint64_t xa = ga < U ? ~(uint64_t)__ldcg(pbase + (size_t)pa * kk + (ga - ea)) : ~0ull;
        uint64_t xb = gb < U ? ~(uint64_t)__ldcg(pbase + (size_t)pb * kk + (gb - eb)) : ~0ull;
        warp_sort64(xa, xb, lane);
        if (base == 0) {
            ra = xa;
            rb = xb;
        } else {
            const uint64_t ca = __shfl_xor_sync(kFull, xb, 31), cb = __shfl_xor_sync(kFull, xa, 31);
            ra = ra < ca ? ra : ca;
            rb = rb < cb ? rb : cb;
            warp_merge64(ra, rb, lane);
        }
    }
    const int n = U < kk ? U : kk;
    if (lane < n) sel[lane] = ~ra;
    if (lane + 32 < n) sel[lane + 32] = ~rb;
    __syncwarp();
    float jm = kLowestFloat;
    double js = 0.0;
    if (jon) {
        if (lane < np) {
            const double2 v = __ldcg(J.part_ms + myslot);
            jm = (float)v.x;
            js = v.y;
        }
        joint_warp_merge(jm, js, jc);
    }
    return Merged{n, rowbad, sp, jm, js};
}

// The slot's per-piece state starts afresh for its next piece (one thread).
__device__ __forceinline__ void slot_reset(PipeShared& P, int slot) {
    P.bad[slot] = 0u;
    P.tau[slot] = 0ull;
    P.used[slot] = 0ull;
    P.boot_cnt[slot] = 0;
    P.boot_ready[slot] = 0u;
    P.mode[slot] = 0u;
}

// Finishing warp f.
template <typename T, int MODE, int PR>
__device__ void pipe_finish(const RowJob& J, PipeShared& P, const uint64_t* slots, unsigned char* scratch, int f,
                            int lane) {
    uint64_t* sel = reinterpret_cast<uint64_t*>(scratch);            // [kPipeMaxK]
    double* wd = reinterpret_cast<double*>(sel + kPipeMaxK);         // [kPipeMaxK]
    uint64_t* gat = reinterpret_cast<uint64_t*>(wd + kPipeMaxK);     // [kPGather]
    unsigned char* tail = reinterpret_cast<unsigned char*>(gat + kPGather);
    FinishShared unused_fs;
    PipeList L = pipe_list<T>(J);
    const int slot = f;
    const uint64_t* sbuf = slots + (size_t)slot * kPipeConsumers * J.cap_w;
    uint32_t use = 0;
    int64_t row = 0;
    bool redo = false;
    for (int64_t i = 0;; ++i) {
        if (i == L.nmain) {
            // this finisher's main items are done (their failed rows recorded):
            // the second one to get here opens the redo pass
            if (lane == 0 && atomicAdd(&P.fin_done, 1) == kPipeFinishers - 1) {
                __threadfence_block();
                st_release_shared(&P.redo_ready, 1u);
            }
            __syncwarp();
        }
        if (!pipe_item<T>(J, P, L, i, row, redo)) break;
        if ((int)(i % kPipeSlots) != slot) continue;
        if (!item_active<MODE>(J, row)) continue;  // nothing to filter (the tails run afterwards)
        const int32_t req = (int32_t)(row / J.rpr);
        uint32_t rowbad = 2u;
        uint64_t spec = 0ull;
        int n = 0;
        bool jon = false;  // joint order: the piece's and then the row's pair (m, s)
        JointScale jc{0.0f, 0.0f};
        if (PR && J.joint) {
            const RowParams rp = row_params<MODE>(J, row);
            jon = rp.ok && rp.T > 0.0f;
            if (jon) jc = joint_scale(rp.T);
        }
        float jm = kLowestFloat;
        double js = 0.0;
        const bool ok = pipe_wait_warp(&P.slot_full[slot], use & 1u, P);
        ++use;
        if (ok) {
            // gather the keys at or above the piece's best threshold into this
            // warp's scratch, hand the slot back, then select from the copy
            const uint64_t tf = P.tau[slot];
            rowbad = P.bad[slot];
            spec = P.used[slot];
            if (jon) {
                if (lane < kPipeConsumers) {
                    jm = P.jm[slot][lane];
                    js = P.js[slot][lane];
                }
                joint_warp_merge(jm, js, jc);
            }
            int U = 0;
            for (int w = 0; w < kPipeConsumers; ++w) {
                const int cw = P.cnt[slot][w];
                const uint64_t* wb = sbuf + (size_t)w * J.cap_w;
                for (int base = 0; base < cw; base += 32) {
                    const uint64_t key = base + lane < cw ? wb[base + lane] : 0ull;
                    const bool keep = base + lane < cw && key >= tf;
                    const unsigned bal = __ballot_sync(kFull, keep);
                    const int at = U + __popc(bal & lanemask_lt());
                    if (keep && at < kPGather) gat[at] = key;
                    U += __popc(bal);
                }
            }
            __syncwarp();
            if (U <= kPGather) {
                if (lane == 0) {
                    slot_reset(P, slot);
                    mbar_arrive(&P.slot_empty[slot]);
                }
                n = warp_select_topk(gat, U, J.k, sel, reinterpret_cast<uint32_t*>(wd), lane);
            } else {  // more keys than the scratch holds: select from the slot itself
                int cw[kPipeConsumers];
                U = 0;
#pragma unroll
                for (int w = 0; w < kPipeConsumers; ++w) {
                    cw[w] = P.cnt[slot][w];
                    U += cw[w];
                }
                const int cap_w = J.cap_w;
                auto get = [&](int g) -> uint64_t {
                    int w = 0, off = g;
#pragma unroll
                    for (int t = 0; t < kPipeConsumers - 1; ++t) {
                        if (w == t && off >= cw[t]) {
                            off -= cw[t];
                            w = t + 1;
                        }
                    }
                    return sbuf[(size_t)w * cap_w + off];
                };
                n = warp_topk64(U, J.k, get, sel, lane);
                __syncwarp();
                if (lane == 0) {
                    slot_reset(P, slot);
                    mbar_arrive(&P.slot_empty[slot]);
                }
            }
        } else if (lane == 0) {
            atomicExch(&P.abort, 1);
        }
        const Piece p = item_piece<T>(J, L, row, redo);
        if (p.np > 1) {
            // publish this piece's best; the last piece of the row merges
            const int64_t ps = part_slot(L.cr, L.cr.b, row);
            uint64_t* pk = J.part_keys + ps * J.k;
            if (lane < n) pk[lane] = sel[lane];
            if (lane + 32 < n) pk[lane + 32] = sel[lane + 32];
            __syncwarp();
            int last = 0;
            if (lane == 0) {
                J.part_count[ps] = n;
                J.part_flags[ps] = rowbad;
                J.part_spec[ps] = spec;
                if (jon) J.part_ms[ps] = make_double2((double)jm, js);
                __threadfence();
                const uint32_t t = atomicAdd(J.row_ticket + p.first_cta, 1u);
                last = (t == (uint32_t)(p.np - 1));
                if (last) {
                    atomicExch(J.row_ticket + p.first_cta, 0u);
                    __threadfence();
                }
            }
            last = __shfl_sync(kFull, last, 0);
            if (!last) continue;
            const Merged m = merge_pieces(J, L.cr.T, L.cr.G, L.cr.nu, row, p.first_cta, p.np, sel, lane, jon, jc);
            n = m.n;
            rowbad = m.rowbad;
            spec = m.spec;
            jm = m.jm;
            js = m.js;
        }
        // a predicted threshold holds when the row's k-th kept key reaches it:
        // then at least k elements of the row do, and none of the top k was
        // dropped.  Otherwise the row is read again, whole, in the redo pass.
        const bool held = !(spec != 0ull && rowbad == 0u && (n < J.k || sel[J.k - 1] < spec));
        if (L.spec_ok && rowbad == 0u && lane == 0) {
            // the row's best values set the prediction of the pieces that follow
            // (and of the next call).  A prediction that failed is dropped (it
            // may come from rows of another scale, carried over from an earlier
            // call): the pieces that follow seed themselves, exactly, until a
            // row finished with its own seed sets a new one.
            const uint64_t t = next_prediction(sel, n, J.k, held);
            if (t != 0ull) {
                const int pset = row_set<MODE>(J, row);
                P.spec[pset] = t;
                __threadfence_block();
                st_release_shared(&P.spec_set[pset], 1u);
            }
        }
        if (!held) {
            if (lane == 0) {
                if (L.dyn) {
                    // post the row for a second read, by whichever producer takes it
                    const uint32_t at = atomicAdd(J.dyn + kDynRetryPut, 1u);
                    atomicExch(J.dyn + kDynWords + at, (uint32_t)row + 1u);
                } else {
                    const int at = atomicAdd(&P.redo_n, 1);
                    J.redo[L.rbase + at] = (int32_t)row;
                }
                __threadfence();
            }
            __syncwarp();
            continue;
        }
        const double2 jms = make_double2((double)jm, js);
        finish_row_warp<MODE, PR>(J, row, req, n, rowbad, sel, wd, tail, unused_fs, lane, gat, &jms);
        if (L.dyn && lane == 0) {
            __threadfence();
            atomicAdd(J.dyn + kDynFinished, 1u);
        }
    }
}

// PR: 1 when the call has per-request parameters (and may use the joint
// order), 0 for the call's scalar parameters, which compiles neither in.
template <typename T, int MODE, int PR>
__global__ void __launch_bounds__(kPipeThreads, 1) pipe_kernel(const __grid_constant__ RowJob J) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ PipeShared P;
    unsigned char* ring = smem;                                                           // [nst][kPStageBytes]
    uint64_t* slots = reinterpret_cast<uint64_t*>(smem + (size_t)J.nst * kPStageBytes);  // [slots][consumers][cap_w]
    unsigned char* fin = reinterpret_cast<unsigned char*>(slots + (size_t)kPipeSlots * kPipeConsumers * J.cap_w);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < J.nst; ++s) {
            mbar_init(&P.full[s], 1);
            mbar_init(&P.empty[s], 1);
            P.fill[s] = 0xffffffffu;  // no element yet
        }
        for (int s = 0; s < kPipeSlots; ++s) {
            mbar_init(&P.slot_full[s], kPipeConsumers);
            mbar_init(&P.slot_empty[s], 1);
            slot_reset(P, s);
        }
        // the predictions this CTA left at the end of the previous call
        for (int t = 0; t < 2; ++t) {
            const uint64_t h = J.hint != nullptr ? J.hint[(size_t)t * kPipeMaxGrid + blockIdx.x] : 0ull;
            P.spec[t] = h;
            P.spec_set[t] = h != 0ull ? 1u : 0u;
        }
        for (int e = 0; e < kDynQ; ++e) P.qseq[e] = 0u;
        P.fin_done = 0;
        P.redo_n = 0;
        P.redo_ready = 0u;
        P.abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == 0) {
        if (lane == 0) pipe_produce<T, MODE>(J, P, ring);
    } else if (warp <= kPipeConsumers) {
        pipe_consume<T, MODE, PR>(J, P, ring, slots, warp - 1, lane);
    } else {
        const int f = warp - 1 - kPipeConsumers;
        pipe_finish<T, MODE, PR>(J, P, slots, fin + (size_t)f * J.fin_stride, f, lane);
    }
    // carry this CTA's latest prediction to the next call (a hint only: the
    // rows it predicts are checked exactly)
    __syncthreads();
    if (threadIdx.x < 2 && J.hint != nullptr && P.spec_set[threadIdx.x] != 0u && P.abort == 0)
        J.hint[(size_t)threadIdx.x * kPipeMaxGrid + blockIdx.x] = P.spec[threadIdx.x];
    // run-time rows: the request-tail kernel that follows puts the counters
    // back to zero; without one, the last CTA to exit does (every other CTA
    // has stopped touching them)
    if (MODE == kModeFilter && J.dyn != nullptr && threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(J.dyn + kDynDone, 1u) == gridDim.x - 1) {
            for (int w = 0; w < kDynWords; ++w) atomicExch(J.dyn + w, 0u);
            __threadfence();
        }
    }
}

// ---------------------------------------------------------------------------
// Request tails after the pipelined kernel: one warp per request, with its
// own shared-memory scratch.  Run on their own, the tails' reads of the
// compact rows hit L2 without queueing behind streaming copies.
// ---------------------------------------------------------------------------
constexpr int kTailWarps = 4;

template <int MODE>
__global__ void __launch_bounds__(32 * kTailWarps) tail_kernel(const __grid_constant__ RowJob J, int64_t nreq) {
    extern __shared__ __align__(128) unsigned char smem[];
    // The job in shared memory: the tails read many of its fields once each,
    // and one parallel copy beats a chain of cold parameter-cache misses.
    __shared__ __align__(16) RowJob sJ;
    static_assert(sizeof(RowJob) % 4 == 0, "copied by words");
    for (int i = threadIdx.x; i < (int)(sizeof(RowJob) / 4); i += blockDim.x)
        reinterpret_cast<uint32_t*>(&sJ)[i] = reinterpret_cast<const uint32_t*>(&J)[i];
    // the row kernel's run-time row counters, back to zero for the next call
    if (blockIdx.x == 0 && threadIdx.x < kDynWords && J.dyn != nullptr) J.dyn[threadIdx.x] = 0u;
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * kTailWarps + warp;
    if (r >= nreq) return;
    unsigned char* mine = smem + (size_t)warp * sJ.fin_stride;
    double* wd = reinterpret_cast<double*>(mine);  // [k] (the global-memory path)
    request_tail<MODE>(sJ, (int32_t)r, wd, mine + (size_t)kPipeMaxK * 8, lane);
}

// ---------------------------------------------------------------------------
// The joint filter order's normaliser, one CTA per row, before the row
// kernels: the row's largest finite logit m and sum_j exp((l_j - m) / T) over
// its finite logits, in one read of the row.  Each thread keeps a running
// maximum and rescales its sum when the maximum rises.  The exponent
// (l - m) / T is formed as (l - m) * c with c = log2(e) / T split into two
// floats (hi + lo), so that the rounding of c does not bias every term alike;
// a unit's terms are added in float, units in double.
// ---------------------------------------------------------------------------
constexpr int kJointThreads = 256;

template <typename T, int MODE>
__global__ void __launch_bounds__(kJointThreads) joint_norm_kernel(const __grid_constant__ RowJob J) {
    const int64_t row = blockIdx.x;
    if (!item_active<MODE>(J, row)) return;
    const RowParams rp = row_params<MODE>(J, row);
    if (!(rp.T > 0.0f) || !rp.ok) {  // greedy rows and rows with bad parameters need no normaliser
        if (threadIdx.x == 0) J.row_ms[row] = make_double2(0.0, 0.0);
        return;
    }
    const JointScale c = joint_scale(rp.T);
    const RowGeom g = row_geom<T>(J, row);
    constexpr int KPU = Elem<T>::kPerUnit;
    float m = -3.402823466e38f;  // lowest finite float
    double s = 0.0;
    const uint4* units = reinterpret_cast<const uint4*>(g.base + (size_t)g.head * Elem<T>::kBytes);
    for (int64_t i = threadIdx.x; i < g.nunit; i += kJointThreads) {
        const uint4 r = __ldg(units + i);
        float um = m;
#pragma unroll
        for (int e = 0; e < KPU; ++e) {
            const float v = Elem<T>::get(r, e);
            um = v > um ? v : um;
        }
        joint_raise(m, s, um, c);
        float t = 0.0f;
#pragma unroll
        for (int e = 0; e < KPU; ++e) t += joint_term(Elem<T>::get(r, e), m, c);
        s += (double)t;
    }
    // the head and tail scalars (fewer than one unit each)
    const int64_t ntail = J.vocab - g.tail_begin;
    if (threadIdx.x < g.head + ntail) {
        const int64_t id = threadIdx.x < g.head ? (int64_t)threadIdx.x : g.tail_begin + (threadIdx.x - g.head);
        const float v = Elem<T>::load_scalar(g.base + (size_t)id * Elem<T>::kBytes);
        joint_raise(m, s, v, c);
        s += (double)joint_term(v, m, c);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(kFull, m, o);
        const double s2 = __shfl_xor_sync(kFull, s, o);
        joint_merge(m, s, m2, s2, c);
    }
    __shared__ float wm[kJointThreads / 32];
    __shared__ double wsum[kJointThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        wm[warp] = m;
        wsum[warp] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kJointThreads / 32; ++w) joint_merge(m, s, wm[w], wsum[w], c);
        J.row_ms[row] = make_double2((double)m, s);
    }
}

// ---------------------------------------------------------------------------
// Tree expansion: one CTA per request.  Its warps extract the top-K of the B
// marginals side by side; warp 0 then expands the tree.
// ---------------------------------------------------------------------------
struct TreeJob {
    const int32_t* q_ids;
    const float* q_probs;
    const int32_t* q_count;
    int32_t q_cap, R, B, K, V, sort_cap;
    int32_t* node_token;
    int32_t* node_parent;
    int32_t* node_depth;
    float* node_score;
    int32_t* num_nodes;
};

constexpr int kTreeMaxWarps = 16;
constexpr int kTreeRankMax = 256;  // rows up to this many entries are ranked, longer ones sorted

__global__ void __launch_bounds__(32 * kTreeMaxWarps) tree_expand_kernel(const __grid_constant__ TreeJob J) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int B = J.B, K = J.K, V = J.V;
    const int nwarps = blockDim.x >> 5;
    double* nscore = reinterpret_cast<double*>(smem);                  // [V]
    uint64_t* sortbufs = reinterpret_cast<uint64_t*>(nscore + V);      // [nwarps][sort_cap]
    int32_t* cand_id = reinterpret_cast<int32_t*>(sortbufs + (size_t)nwarps * J.sort_cap);  // [B*K]
    float* cand_p = reinterpret_cast<float*>(cand_id + B * K);         // [B*K]
    int32_t* ncand = reinterpret_cast<int32_t*>(cand_p + B * K);       // [B]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x;

    // 1. top-K of each marginal by (prob desc, id asc), one row per warp at a
    // time.  Keys are distinct (ids are), so an entry's place is the number
    // of larger keys in its row.
    uint64_t* sortbuf = sortbufs + (size_t)warp * J.sort_cap;
    for (int d = warp; d < B; d += nwarps) {
        const int64_t row = (int64_t)r * B + d;
        int c = J.q_count[row];
        c = c < 0 ? 0 : (c > J.q_cap ? J.q_cap : c);
        const int np2 = c <= kTreeRankMax ? c : next_pow2(c);
        for (int i = lane; i < np2; i += 32) {
            uint64_t key = 0ull;
            if (i < c) {
                const float p = __fadd_rn(J.q_probs[(size_t)row * J.q_cap + i], 0.0f);
                const int32_t id = J.q_ids[(size_t)row * J.q_cap + i];
                key = ((uint64_t)ord_of_float(p) << 32) | (uint64_t)(~(uint32_t)id);
            }
            sortbuf[i] = key;
        }
        __syncwarp();
        const int nk = c < K ? c : K;
        if (c <= kTreeRankMax) {
            for (int i = lane; i < c; i += 32) {
                const uint64_t key = sortbuf[i];
                int rank = 0;
                for (int j = 0; j < c; ++j) rank += sortbuf[j] > key ? 1 : 0;
                if (rank < nk) {
                    cand_id[d * K + rank] = key_id(key);
                    cand_p[d * K + rank] = float_of_ord((uint32_t)(key >> 32));
                }
            }
        } else {
            warp_bitonic_sort(sortbuf, np2, true, lane);
            for (int i = lane; i < nk; i += 32) {
                cand_id[d * K + i] = key_id(sortbuf[i]);
                cand_p[d * K + i] = float_of_ord((uint32_t)(sortbuf[i] >> 32));
            }
        }
        if (lane == 0) ncand[d] = nk;
        __syncwarp();
    }
    __syncthreads();
    if (warp != 0) return;

    int32_t* tok = J.node_token + (size_t)r * V;
    int32_t* par = J.node_parent + (size_t)r * V;
    int32_t* dep = J.node_depth + (size_t)r * V;
    float* sco = J.node_score + (size_t)r * V;
    for (int j = lane; j < V; j += 32) {
        tok[j] = -1;
        par[j] = -1;
        dep[j] = -1;
        sco[j] = 0.0f;
    }
    __syncwarp();

    // 2. best-first expansion with a lazy frontier: a tree node keeps only its
    // best unexpanded child in the frontier; popping a child brings in its own
    // first child and its next sibling.  Scores never rise along those links
    // and the tie order never falls, so this pops nodes in the same order as
    // a frontier that holds every child.  The frontier holds at most as many
    // entries as the tree has nodes (V <= 128): entry j lives in registers of
    // lane j % 32, slot j / 32, as its score and its tie key (depth << 24 |
    // parent << 12 | rank; lower ranks first at equal scores).  An empty slot
    // holds score 0 and the largest tie key, so every entry ranks above it.
    constexpr int kSlots = (UNO_MAX_TREE_NODES + 31) / 32;
    double fs[kSlots];
    uint32_t ft[kSlots];
    fs[0] = fs[1] = fs[2] = fs[3] = 0.0;  // empty
    ft[0] = ft[1] = ft[2] = ft[3] = 0xffffffffu;
    auto tie_of = [](int d, int p, int rk) -> uint32_t {
        return ((uint32_t)d << 24) | ((uint32_t)p << 12) | (uint32_t)rk;
    };
    // entry j := (score, tie), by its owner lane (unrolled, so that the
    // slots stay in registers)
#define UNO_TREE_SLOT(t_)                                     \
    fs[t_] = (own_ && (pj_ >> 5) == (t_)) ? psc_ : fs[t_];    \
    ft[t_] = (own_ && (pj_ >> 5) == (t_)) ? ptk_ : ft[t_];
#define UNO_TREE_PUT(j_, sc_, tk_)                            \
    do {                                                      \
        const int pj_ = (j_);                                 \
        const double psc_ = (sc_);                            \
        const uint32_t ptk_ = (tk_);                          \
        const bool own_ = lane == (pj_ & 31);                 \
        UNO_TREE_SLOT(0) UNO_TREE_SLOT(1) UNO_TREE_SLOT(2) UNO_TREE_SLOT(3) \
    } while (0)
    static_assert(kSlots == 4, "four frontier slots per lane");
    if (lane == 0) {
        nscore[0] = 1.0;
        tok[0] = -1;
        par[0] = -1;
        dep[0] = 0;
        sco[0] = 1.0f;
    }
    __syncwarp();
    int nf = 0;
    if (ncand[0] > 0) {
        UNO_TREE_PUT(0, 1.0 * (double)cand_p[0], tie_of(1, 0, 0));
        nf = 1;
    }
    int n = 1;
    while (n < V && nf > 0) {
        // the lane's best entry, then the warp's: the highest score, and among
        // equal scores the smallest tie key
        double bs = fs[0];
        uint32_t bt = ft[0];
        int bslot = 0;
#define UNO_TREE_BEST(t_)                                          \
        if (fs[t_] > bs || (fs[t_] == bs && ft[t_] < bt)) {        \
            bs = fs[t_];                                           \
            bt = ft[t_];                                           \
            bslot = t_;                                            \
        }
        UNO_TREE_BEST(1) UNO_TREE_BEST(2) UNO_TREE_BEST(3)
#undef UNO_TREE_BEST
        // scores are >= 0, so their bit patterns order as their values: the
        // warp's best is the largest high word, then low word, then the
        // smallest tie key (three 32-bit warp reductions)
        const uint64_t bb = (uint64_t)__double_as_longlong(bs);
        const uint32_t bh = (uint32_t)(bb >> 32), bl = (uint32_t)bb;
        const uint32_t mh = __reduce_max_sync(kFull, bh);
        const uint32_t ml = __reduce_max_sync(kFull, bh == mh ? bl : 0u);
        const bool best = bh == mh && bl == ml;
        const double ms = __longlong_as_double((long long)(((uint64_t)mh << 32) | ml));
        const uint32_t mt = __reduce_min_sync(kFull, best ? bt : 0xffffffffu);
        const unsigned own = __ballot_sync(kFull, best && bt == mt);
        const int owner = __ffs(own) - 1;
        const int jo = owner + 32 * __shfl_sync(kFull, bslot, owner);
        const double sp = ms;
        const int d = (int)(mt >> 24), pp = (int)((mt >> 12) & 0xfffu), rk = (int)(mt & 0xfffu);
        // remove it: the last entry moves into its place
        const int jl = nf - 1;
        const int jt = jl >> 5;
        double ls = jt == 0 ? fs[0] : jt == 1 ? fs[1] : jt == 2 ? fs[2] : fs[3];
        uint32_t lt = jt == 0 ? ft[0] : jt == 1 ? ft[1] : jt == 2 ? ft[2] : ft[3];
        ls = __shfl_sync(kFull, ls, jl & 31);
        lt = __shfl_sync(kFull, lt, jl & 31);
        // everything the pushes below read, loaded at once (nothing of it is
        // written in this step: the parent pp was stored steps ago)
        const int nc_child = d < B ? ncand[d] : 0;
        const float p_child = d < B ? cand_p[d * K] : 0.0f;
        const int nc_sib = ncand[d - 1];
        const float p_sib = rk + 1 < K ? cand_p[(d - 1) * K + rk + 1] : 0.0f;
        const double s_par = nscore[pp];
        const int32_t t_new = cand_id[(d - 1) * K + rk];
        UNO_TREE_PUT(jl, 0.0, 0xffffffffu);
        if (jo != jl) UNO_TREE_PUT(jo, ls, lt);
        nf = jl;
        // the popped entry becomes node n
        const int idx = n;
        if (lane == 0) {
            nscore[idx] = sp;
            tok[idx] = t_new;
            par[idx] = pp;
            dep[idx] = d;
            sco[idx] = (float)sp;
        }
        __syncwarp();
        if (nc_child > 0) {  // its first child
            UNO_TREE_PUT(nf, sp * (double)p_child, tie_of(d + 1, idx, 0));
            ++nf;
        }
        if (rk + 1 < nc_sib) {  // its next sibling
            UNO_TREE_PUT(nf, s_par * (double)p_sib, tie_of(d, pp, rk + 1));
            ++nf;
        }
        ++n;
    }
    if (lane == 0) J.num_nodes[r] = n;
#undef UNO_TREE_PUT
#undef UNO_TREE_SLOT
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
static int sm_count() {
    static int cached[64];
    static std::once_flag flags[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::call_once(flags[dev], [dev]() {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    });
    return cached[dev];
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Largest split count the workspace is sized for.
static int split_bound(int64_t rows) {
    if (rows <= 0) return 1;
    int64_t s = 4096 / rows;
    if (s < 1) s = 1;
    if (s > kMaxSplits) s = kMaxSplits;
    return (int)s;
}

// Workspace layout.  The first kCounterBytes hold the library's arrival
// counters: row counters (split rows) in the first half, request counters in
// the second.  Every call leaves them at zero, and nothing else is ever
// written there, so one zero-fill serves every later call of any entry point
// and size.  Scratch (partial selections, compact target rows) follows.
constexpr int64_t kCounterWords = UNO_WORKSPACE_COUNTER_BYTES / 4;
constexpr int64_t kRowCounterWords = kCounterWords / 2;

struct WsLayout {
    size_t row_ticket, req_ticket, part_keys, part_count, part_flags, part_spec, part_ms, redo, row_ms, c_ids,
        c_probs, c_count, c_flags, total;
};

static WsLayout ws_layout(int64_t rows, int32_t k, bool compact) {
    WsLayout L{};
    const int sb = split_bound(rows);
    // part slots: split rows of the general kernel (rows x splits) or of the
    // pipelined kernel (two per CTA)
    size_t nslot = sb > 1 ? (size_t)rows * sb : 0;
    if (nslot < (size_t)2 * kPipeMaxGrid) nslot = (size_t)2 * kPipeMaxGrid;
    L.row_ticket = 0;
    L.req_ticket = (size_t)kRowCounterWords * 4;
    size_t off = (size_t)UNO_WORKSPACE_COUNTER_BYTES + UNO_WORKSPACE_HINT_BYTES;
    L.part_keys = off;
    off = align_up(off + nslot * (size_t)k * 8, 256);
    L.part_count = off;
    off = align_up(off + nslot * 4, 256);
    L.part_flags = off;
    off = align_up(off + nslot * 4, 256);
    L.part_spec = off;
    off = align_up(off + nslot * 8, 256);
    L.part_ms = off;
    off = align_up(off + nslot * 16, 256);
    L.redo = off;
    off = align_up(off + ((size_t)rows + kPipeMaxGrid) * 4, 256);
    L.row_ms = off;
    off = align_up(off + (size_t)rows * 16, 256);
    L.c_ids = off;
    const size_t crow = compact ? (size_t)rows : 0;
    const size_t ks = (size_t)((k + 3) & ~3);
    off = align_up(off + crow * ks * 4, 256);
    L.c_probs = off;
    off = align_up(off + crow * ks * 4, 256);
    L.c_count = off;
    off = align_up(off + crow * 4, 256);
    L.c_flags = off;
    off = align_up(off + crow * 4, 256);
    L.total = off;
    return L;
}

// A cycle's workspace: the verifier layout over all its rows, then the draft
// rows' compact arrays (ids and probs [nq][ks], count, flags, drafts [nq]).
struct CycleLayout {
    WsLayout w;
    size_t q_ids, q_probs, q_count, q_flags, q_draft, total;
};
static CycleLayout cycle_layout(int32_t R, int32_t B, int32_t k, int32_t layout) {
    CycleLayout C{};
    const int64_t nq = (int64_t)R * B, np = (int64_t)R * (B + 1 - layout);
    C.w = ws_layout(nq + np, k, true);
    const size_t ks = (size_t)((k + 3) & ~3);
    size_t off = C.w.total;
    C.q_ids = off;
    off = align_up(off + (size_t)nq * ks * 4, 256);
    C.q_probs = off;
    off = align_up(off + (size_t)nq * ks * 4, 256);
    C.q_count = off;
    off = align_up(off + (size_t)nq * 4, 256);
    C.q_flags = off;
    off = align_up(off + (size_t)nq * 4, 256);
    C.q_draft = off;
    off = align_up(off + (size_t)nq * 4, 256);
    C.total = off;
    return C;
}

static bool params_ok(const uno_sampling_params& sp) {
    if (!(sp.temperature >= 0.0f) || std::isinf(sp.temperature)) return false;
    if (sp.top_k < 1) return false;
    if (!(sp.top_p > 0.0f && sp.top_p <= 1.0f)) return false;
    return true;
}

// Shared memory of the streaming phase; the finishing area reuses the ring
// stages when it fits there, else it is appended (fin_off).
template <typename T, int MODE>
static size_t row_smem_bytes(RowJob& J) {
    const size_t stream = (size_t)kStages * kStageBytes + 32 + (size_t)kWarps * J.cap_w * 8;
    const size_t finish = (size_t)J.merge_cap * 8 + (size_t)J.k * 32;
    const size_t ring = (size_t)kStages * kStageBytes;
    // the request tails use the rest of the ring
    if (finish <= ring) {
        J.fin_off = 0;
        J.tail_off = (int32_t)((finish + 127) / 128 * 128);
        J.tail_bytes = J.tail_off < (int32_t)ring ? (int32_t)ring - J.tail_off : 0;
        return stream;
    }
    J.fin_off = (int32_t)((stream + 127) / 128 * 128);
    J.tail_off = 0;
    J.tail_bytes = (int32_t)ring;
    return (size_t)J.fin_off + finish;
}

// The joint order's per-row normalisers, ahead of the row kernels.
template <typename T, int MODE>
static uno_status launch_joint(const RowJob& J, cudaStream_t stream) {
    if (!J.joint || J.rows <= 0) return UNO_OK;
    joint_norm_kernel<T, MODE><<<(unsigned)J.rows, kJointThreads, 0, stream>>>(J);
    return cudaGetLastError() == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}

// The pipelined kernel: grid (balanced pieces or run-time rows), ring depth
// and shared memory.  Returns UNO_ERR_UNSUPPORTED (nothing launched) when it
// does not fit.
template <typename T, int MODE>
static uno_status launch_pipe(RowJob J, cudaStream_t stream) {
    J.hw = J.k + 16 > 64 ? J.k + 16 : 64;
    J.cap_w = J.hw + 32;  // a stage's candidates that fit are written at once, else appended with compaction
    // one CTA per SM; with fewer rows than SMs, pieces of at least
    // kPipeMinPieceUnits and at most kPipeMaxPieces per row
    int64_t grid = sm_count() < kPipeMaxGrid ? sm_count() : kPipeMaxGrid;
    if (J.rows < grid) {
        const int64_t nu = J.vocab / Elem<T>::kPerUnit > 0 ? J.vocab / Elem<T>::kPerUnit : 1;
        int64_t g = J.rows * nu / kPipeMinPieceUnits;
        if (g > J.rows * (kPipeMaxPieces - 2)) g = J.rows * (kPipeMaxPieces - 2);
        if (g < J.rows) g = J.rows;
        if (g < grid) grid = g;
    }
    J.S = 1;
    // With several rows per CTA, rows are handed out at run time (whole rows,
    // one counter), so that CTAs whose stream runs slower take fewer; tree
    // mode keeps the fixed pieces (its inactive node rows are skipped).
    J.dyn = nullptr;
    if (MODE != kModeTree && J.rows >= 4 * grid && J.rows + kDynOffset + kDynWords <= kRowCounterWords)
        J.dyn = J.row_ticket + kDynOffset;
    if (J.hint != nullptr) J.hint += (size_t)MODE * 2 * kPipeMaxGrid;  // each entry point keeps its own
    // shared memory: ring | candidate slots | per finisher: sel, wd, tail
    const size_t slot_bytes = (size_t)kPipeSlots * kPipeConsumers * J.cap_w * 8;
    size_t tail = 0;
    if (MODE == kModeLinear || MODE == kModeCycle)
        tail = 16 + (size_t)(J.B + 1) * J.ks * 8 + 2 * ((size_t)J.B * 64 * 4 + 16) + (size_t)(4 * J.B + 2) * 4;
    else if (MODE == kModeTree)
        tail = 16 + (size_t)J.V * J.ks * 8 + (size_t)J.V * 12 + (size_t)(J.B + 1) * 8;
    const size_t dyn_max = 227 * 1024 - sizeof(PipeShared);
    auto stride_of = [](size_t tb) { return align_up((size_t)2 * kPipeMaxK * 8 + (size_t)kPGather * 8 + tb, 128); };
    auto stages_of = [&](size_t tb) -> int64_t {
        const size_t fixed = slot_bytes + (size_t)kPipeFinishers * stride_of(tb);
        return fixed >= dyn_max ? 0 : (int64_t)((dyn_max - fixed) / kPStageBytes);
    };
    int64_t nst = stages_of(0);  // the request tails run in their own kernel
    if (nst > kPipeMaxStages) nst = kPipeMaxStages;
    if (nst < kPipeMinStages) return UNO_ERR_UNSUPPORTED;
    J.nst = (int32_t)nst;
    J.tail_bytes = 0;
    J.fin_stride = (int32_t)stride_of(0);
    J.defer_tails = 1;
    const size_t dyn = (size_t)nst * kPStageBytes + slot_bytes + (size_t)kPipeFinishers * J.fin_stride;
    auto kern = J.rq_T != nullptr ? pipe_kernel<T, MODE, 1> : pipe_kernel<T, MODE, 0>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) != cudaSuccess)
        return UNO_ERR_CUDA;
    if (grid <= 0) return UNO_OK;
    kern<<<(unsigned)grid, kPipeThreads, dyn, stream>>>(J);
    if (cudaGetLastError() != cudaSuccess) return UNO_ERR_CUDA;
    if (MODE == kModeFilter) return UNO_OK;
    // the request tails: shared-memory rows when they fit in 48 KB a warp
    RowJob TJ = J;
    TJ.tail_bytes = tail <= 48 * 1024 ? (int32_t)tail : 0;
    TJ.fin_stride = (int32_t)align_up((size_t)kPipeMaxK * 8 + (size_t)TJ.tail_bytes, 128);
    const int64_t nreq = MODE == kModeCycle ? J.nq2 / J.B : J.rows / J.rpr;
    const size_t tsm = (size_t)kTailWarps * TJ.fin_stride;
    auto tkern = tail_kernel<MODE>;
    if (tsm > 48 * 1024 &&
        cudaFuncSetAttribute(tkern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm) != cudaSuccess)
        return UNO_ERR_CUDA;
    tkern<<<(unsigned)((nreq + kTailWarps - 1) / kTailWarps), 32 * kTailWarps, tsm, stream>>>(TJ, nreq);
    return cudaGetLastError() == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}

template <typename T, int MODE>
static uno_status launch_rows(RowJob J, cudaStream_t stream) {
    // the pipelined kernel forms the joint order's normalisers as it reads
    // the rows; the general one takes them from a pass of their own
    if (J.k <= kPipeMaxK && J.out_dense == nullptr) {
        const uno_status st = launch_pipe<T, MODE>(J, stream);
        if (st != UNO_ERR_UNSUPPORTED) return st;
    }
    const uno_status sj = launch_joint<T, MODE>(J, stream);
    if (sj != UNO_OK) return sj;
    // warp buffer: high-water mark, plus room for one piece of appends from
    // every lane; it also holds the threshold seed (2 keys per thread)
    J.hw = J.k + 16 > 64 ? J.k + 16 : 64;
    J.cap_w = J.hw + 32 * kPiece;
    // split count: fill the GPU when rows are few (each split streams at
    // least two stages)
    const int64_t nunit_row = J.vocab / Elem<T>::kPerUnit;
    const int64_t slots = (int64_t)sm_count() * 4;
    int S = 1;
    if (J.rows < slots && J.rows <= kRowCounterWords) {
        int64_t s = slots / J.rows;
        const int64_t by_work = nunit_row / (2 * kStageUnits);
        if (s > by_work) s = by_work;
        if (s > split_bound(J.rows)) s = split_bound(J.rows);
        S = s < 1 ? 1 : (int)s;
    }
    // fewer splits if the merge area would not fit in shared memory
    size_t smem = 0;
    for (;;) {
        J.S = S;
        J.merge_cap = (S > kWarps ? S : kWarps) * J.k;
        smem = row_smem_bytes<T, MODE>(J);
        if (smem <= 227 * 1024 || S <= kWarps) break;
        --S;
    }
    if (smem > 227 * 1024) return UNO_ERR_UNSUPPORTED;
    auto kern = row_kernel<T, MODE>;
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return UNO_ERR_CUDA;
    }
    const int64_t grid = J.rows * S;
    if (grid <= 0) return UNO_OK;
    if (grid > INT_MAX) return UNO_ERR_UNSUPPORTED;
    kern<<<(unsigned)grid, kThreads, smem, stream>>>(J);
    return cudaGetLastError() == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}

static void bind_workspace(RowJob& J, void* ws, const WsLayout& L) {
    unsigned char* b = static_cast<unsigned char*>(ws);
    J.row_ticket = reinterpret_cast<uint32_t*>(b + L.row_ticket);
    J.req_ticket = reinterpret_cast<uint32_t*>(b + L.req_ticket);
    J.part_keys = reinterpret_cast<uint64_t*>(b + L.part_keys);
    J.part_count = reinterpret_cast<int32_t*>(b + L.part_count);
    J.part_flags = reinterpret_cast<uint32_t*>(b + L.part_flags);
    J.part_spec = reinterpret_cast<uint64_t*>(b + L.part_spec);
    J.part_ms = reinterpret_cast<double2*>(b + L.part_ms);
    J.redo = reinterpret_cast<int32_t*>(b + L.redo);
    J.row_ms = reinterpret_cast<double2*>(b + L.row_ms);
    J.hint = reinterpret_cast<uint64_t*>(b + UNO_WORKSPACE_COUNTER_BYTES);
    J.c_ids = reinterpret_cast<int32_t*>(b + L.c_ids);
    J.ks = (J.k + 3) & ~3;
    J.c_probs = reinterpret_cast<float*>(b + L.c_probs);
    J.c_count = reinterpret_cast<int32_t*>(b + L.c_count);
    J.c_flags = reinterpret_cast<uint32_t*>(b + L.c_flags);
}

// Per-request parameters: the call's sampling parameters for its checks and
// sizes (top_k = the bound), the arrays for the rows.
static bool request_params_ok(const uno_request_params* rp) {
    if (rp == nullptr || !rp->temperature || !rp->top_k || !rp->top_p) return false;
    if ((reinterpret_cast<uintptr_t>(rp->temperature) | reinterpret_cast<uintptr_t>(rp->top_k) |
         reinterpret_cast<uintptr_t>(rp->top_p)) % 4 != 0)
        return false;
    if (rp->top_k_max < 1) return false;
    return rp->order == UNO_ORDER_TOPK_FIRST || rp->order == UNO_ORDER_JOINT;
}
static uno_sampling_params bound_params(const uno_request_params* rp) {
    uno_sampling_params sp;
    sp.temperature = 1.0f;
    sp.top_k = rp->top_k_max;
    sp.top_p = 1.0f;
    return sp;
}
static void apply_request_params(RowJob& J, const uno_request_params* rp) {
    if (rp == nullptr) return;
    J.rq_T = rp->temperature;
    J.rq_k = rp->top_k;
    J.rq_p = rp->top_p;
    J.joint = rp->order == UNO_ORDER_JOINT ? 1 : 0;
}

}  // namespace uno

using namespace uno;

extern "C" {

const char* uno_status_string(uno_status s) {
    switch (s) {
        case UNO_OK: return "ok";
        case UNO_ERR_INVALID_ARG: return "invalid argument";
        case UNO_ERR_UNSUPPORTED: return "unsupported argument";
        case UNO_ERR_CUDA: return "CUDA launch error";
        case UNO_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

size_t uno_filter_softmax_workspace_bytes(int64_t rows, int64_t vocab, int32_t top_k) {
    if (rows <= 0 || vocab <= 0 || top_k < 1) return 0;
    const int32_t k = (int32_t)(top_k < vocab ? top_k : vocab);
    return ws_layout(rows, k, false).total;
}

size_t uno_linear_verify_workspace_bytes(int32_t R, int32_t B, int64_t vocab, int32_t top_k) {
    if (R <= 0 || B <= 0 || vocab <= 0 || top_k < 1) return 0;
    const int32_t k = (int32_t)(top_k < vocab ? top_k : vocab);
    return ws_layout((int64_t)R * (B + 1), k, true).total;
}

size_t uno_tree_verify_workspace_bytes(int32_t R, int32_t V, int64_t vocab, int32_t top_k) {
    if (R <= 0 || V <= 0 || vocab <= 0 || top_k < 1) return 0;
    const int32_t k = (int32_t)(top_k < vocab ? top_k : vocab);
    return ws_layout((int64_t)R * V, k, true).total;
}

static bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
// a device cycle word, when given, is a 4-byte aligned uint32_t
static bool rng_ok(const uno_rng& r) { return r.cycle_word == nullptr || aligned_to(r.cycle_word, 4); }

static uno_status filter_softmax_impl(const void* logits, uno_dtype dt, int64_t rows, int64_t vocab, int64_t row_stride,
                              int32_t rows_per_request, uno_sampling_params sp, const uno_request_params* rp, int32_t cap, int32_t* out_ids,
                              float* out_probs, int32_t* out_count, float* out_dense, const uno_rng* rng,
                              int32_t* out_sample, uint32_t* out_flags, void* workspace, size_t workspace_bytes,
                              void* stream) {
    if (!logits || !out_ids || !out_probs || !out_count || !out_flags) return UNO_ERR_INVALID_ARG;
    if (rows <= 0 || vocab <= 0 || vocab > INT32_MAX || row_stride < vocab || rows_per_request < 1)
        return UNO_ERR_INVALID_ARG;
    if (dt != UNO_F32 && dt != UNO_BF16) return UNO_ERR_INVALID_ARG;
    if (!params_ok(sp)) return UNO_ERR_INVALID_ARG;
    if (rng && !rng_ok(*rng)) return UNO_ERR_INVALID_ARG;
    if (rng && !out_sample) return UNO_ERR_INVALID_ARG;
    if (!aligned_to(logits, dt == UNO_F32 ? 4 : 2)) return UNO_ERR_INVALID_ARG;
    if (sp.top_k > UNO_MAX_TOP_K) return UNO_ERR_UNSUPPORTED;
    const int32_t k = (int32_t)(sp.top_k < vocab ? sp.top_k : vocab);
    if (cap < k) return UNO_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(rows, k, false);
    if (!workspace || workspace_bytes < L.total || !aligned_to(workspace, 16)) return UNO_ERR_WORKSPACE;

    RowJob J{};
    J.logits = static_cast<const unsigned char*>(logits);
    J.rows = rows;
    J.vocab = vocab;
    J.row_stride = row_stride;
    J.rpr = rows_per_request;
    J.temperature = sp.temperature;
    J.top_p = sp.top_p;
    J.k = k;
    apply_request_params(J, rp);
    J.out_ids = out_ids;
    J.out_probs = out_probs;
    J.out_count = out_count;
    J.cap = cap;
    J.out_dense = out_dense;
    J.out_sample = out_sample;
    J.out_flags = out_flags;
    J.has_rng = rng ? 1 : 0;
    J.seed = rng ? rng->seed : 0;
    J.cycle = rng ? rng->cycle : 0;
    J.cycle_word = rng ? rng->cycle_word : nullptr;
    J.first_request = rng ? rng->first_request : 0;
    bind_workspace(J, workspace, L);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return dt == UNO_BF16 ? launch_rows<__nv_bfloat16, kModeFilter>(J, s) : launch_rows<float, kModeFilter>(J, s);
}

static uno_status linear_verify_impl(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int64_t vocab,
                             uno_sampling_params sp, const uno_request_params* rp, const int32_t* draft_ids, const int32_t* q_ids,
                             const float* q_probs, const int32_t* q_count, int32_t q_cap, uno_rng rng,
                             int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_num_tokens,
                             uint32_t* out_flags, void* workspace, size_t workspace_bytes, void* stream) {
    if (!target_logits || !draft_ids || !q_ids || !q_probs || !q_count || !out_tokens || !out_accept_len ||
        !out_num_tokens || !out_flags)
        return UNO_ERR_INVALID_ARG;
    if (R <= 0 || B <= 0 || vocab <= 0 || vocab > INT32_MAX || q_cap < 1) return UNO_ERR_INVALID_ARG;
    if (dt != UNO_F32 && dt != UNO_BF16) return UNO_ERR_INVALID_ARG;
    if (!params_ok(sp)) return UNO_ERR_INVALID_ARG;
    if (!rng_ok(rng)) return UNO_ERR_INVALID_ARG;
    if (!aligned_to(target_logits, dt == UNO_F32 ? 4 : 2)) return UNO_ERR_INVALID_ARG;
    if (sp.top_k > UNO_MAX_TOP_K) return UNO_ERR_UNSUPPORTED;
    const int32_t k = (int32_t)(sp.top_k < vocab ? sp.top_k : vocab);
    const int64_t rows = (int64_t)R * (B + 1);
    if ((int64_t)R > kCounterWords - kRowCounterWords) return UNO_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(rows, k, true);
    if (!workspace || workspace_bytes < L.total || !aligned_to(workspace, 16)) return UNO_ERR_WORKSPACE;

    RowJob J{};
    J.logits = static_cast<const unsigned char*>(target_logits);
    J.rows = rows;
    J.vocab = vocab;
    J.row_stride = vocab;
    J.rpr = B + 1;
    J.temperature = sp.temperature;
    J.top_p = sp.top_p;
    J.k = k;
    apply_request_params(J, rp);
    J.seed = rng.seed;
    J.cycle = rng.cycle;
    J.cycle_word = rng.cycle_word;
    J.first_request = rng.first_request;
    J.B = B;
    J.draft_ids = draft_ids;
    J.q_ids = q_ids;
    J.q_probs = q_probs;
    J.q_count = q_count;
    J.q_cap = q_cap;
    J.out_tokens = out_tokens;
    J.out_accept_len = out_accept_len;
    J.out_num_tokens = out_num_tokens;
    J.out_req_flags = out_flags;
    bind_workspace(J, workspace, L);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return dt == UNO_BF16 ? launch_rows<__nv_bfloat16, kModeLinear>(J, s) : launch_rows<float, kModeLinear>(J, s);
}

size_t uno_linear_cycle_workspace_bytes(int32_t R, int32_t B, int64_t vocab, int32_t top_k, int32_t layout) {
    if (R <= 0 || B <= 0 || vocab <= 0 || top_k < 1 || (layout != UNO_LAYOUT_GENERIC && layout != UNO_LAYOUT_TWO_PASS))
        return 0;
    const int32_t k = (int32_t)(top_k < vocab ? top_k : vocab);
    return cycle_layout(R, B, k, layout).total;
}

static uno_status linear_cycle_impl(const void* draft_logits, const void* target_logits, uno_dtype dt, int32_t R, int32_t B,
                            int64_t vocab, int32_t layout, uno_sampling_params sp, const uno_request_params* rp, uno_rng rng, int32_t* out_tokens,
                            int32_t* out_num_accepted, int32_t* out_num_tokens, uint32_t* out_flags,
                            int32_t* out_draft_ids, void* workspace, size_t workspace_bytes, void* stream) {
    if (!draft_logits || !target_logits || !out_tokens || !out_num_accepted || !out_num_tokens || !out_flags)
        return UNO_ERR_INVALID_ARG;
    if (R <= 0 || B <= 0 || vocab <= 0 || vocab > INT32_MAX) return UNO_ERR_INVALID_ARG;
    if (layout != UNO_LAYOUT_GENERIC && layout != UNO_LAYOUT_TWO_PASS) return UNO_ERR_INVALID_ARG;
    if (dt != UNO_F32 && dt != UNO_BF16) return UNO_ERR_INVALID_ARG;
    if (!params_ok(sp)) return UNO_ERR_INVALID_ARG;
    if (!rng_ok(rng)) return UNO_ERR_INVALID_ARG;
    const size_t esz = dt == UNO_F32 ? 4 : 2;
    if (!aligned_to(draft_logits, esz) || !aligned_to(target_logits, esz)) return UNO_ERR_INVALID_ARG;
    if (sp.top_k > UNO_MAX_TOP_K) return UNO_ERR_UNSUPPORTED;
    if ((int64_t)R > kCounterWords - kRowCounterWords) return UNO_ERR_UNSUPPORTED;
    const int32_t k = (int32_t)(sp.top_k < vocab ? sp.top_k : vocab);
    const int64_t nq = (int64_t)R * B, np = (int64_t)R * (B + 1 - layout);
    const CycleLayout C = cycle_layout(R, B, k, layout);
    if (!workspace || workspace_bytes < C.total || !aligned_to(workspace, 16)) return UNO_ERR_WORKSPACE;
    unsigned char* wb = static_cast<unsigned char*>(workspace);
    int32_t* q_ids = reinterpret_cast<int32_t*>(wb + C.q_ids);
    float* q_probs = reinterpret_cast<float*>(wb + C.q_probs);
    int32_t* q_count = reinterpret_cast<int32_t*>(wb + C.q_count);
    uint32_t* q_flags = reinterpret_cast<uint32_t*>(wb + C.q_flags);
    int32_t* drafts = out_draft_ids != nullptr ? out_draft_ids : reinterpret_cast<int32_t*>(wb + C.q_draft);
    const int32_t ks = (k + 3) & ~3;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    RowJob J{};
    J.vocab = vocab;
    J.row_stride = vocab;
    J.temperature = sp.temperature;
    J.top_p = sp.top_p;
    J.k = k;
    apply_request_params(J, rp);
    J.seed = rng.seed;
    J.cycle = rng.cycle;
    J.cycle_word = rng.cycle_word;
    J.first_request = rng.first_request;
    // the draft rows' outputs: compact rows, flags and one proposal each
    J.out_ids = q_ids;
    J.out_probs = q_probs;
    J.out_count = q_count;
    J.out_flags = q_flags;
    J.cap = ks;
    J.has_rng = 1;
    J.out_sample = drafts;
    // the verification
    J.B = B;
    J.sh = layout;
    J.draft_ids = drafts;
    J.q_ids = q_ids;
    J.q_probs = q_probs;
    J.q_count = q_count;
    J.q_cap = ks;
    J.q_flags = q_flags;
    J.out_tokens = out_tokens;
    J.out_accept_len = out_num_accepted;
    J.out_num_tokens = out_num_tokens;
    J.out_req_flags = out_flags;
    bind_workspace(J, workspace, C.w);
    if (k <= kPipeMaxK) {
        // one launch over the cycle's draft and target rows, then the request tails
        J.logits = static_cast<const unsigned char*>(draft_logits);
        J.logits2 = static_cast<const unsigned char*>(target_logits);
        J.nq2 = nq;
        J.rows = nq + np;
        J.rpr = B;
        const uno_status st = dt == UNO_BF16 ? launch_pipe<__nv_bfloat16, kModeCycle>(J, s)
                                             : launch_pipe<float, kModeCycle>(J, s);
        if (st != UNO_ERR_UNSUPPORTED) return st;
    }
    // the draft rows, then the target rows with the request tails
    RowJob Q = J;
    Q.logits = static_cast<const unsigned char*>(draft_logits);
    Q.rows = nq;
    Q.rpr = B;
    uno_status st = dt == UNO_BF16 ? launch_rows<__nv_bfloat16, kModeFilter>(Q, s) : launch_rows<float, kModeFilter>(Q, s);
    if (st != UNO_OK) return st;
    RowJob V = J;
    V.logits = static_cast<const unsigned char*>(target_logits);
    V.rows = np;
    V.rpr = B + 1 - layout;
    V.has_rng = 0;
    return dt == UNO_BF16 ? launch_rows<__nv_bfloat16, kModeLinear>(V, s) : launch_rows<float, kModeLinear>(V, s);
}

uno_status uno_tree_topk_expand(const int32_t* q_ids, const float* q_probs, const int32_t* q_count, int32_t q_cap,
                                int32_t R, int32_t B, int32_t K, int32_t V, int32_t* node_token,
                                int32_t* node_parent, int32_t* node_depth, float* node_score, int32_t* num_nodes,
                                void* stream) {
    if (!q_ids || !q_probs || !q_count || !node_token || !node_parent || !node_depth || !node_score || !num_nodes)
        return UNO_ERR_INVALID_ARG;
    if (R <= 0 || B <= 0 || K <= 0 || V <= 0 || q_cap < 1) return UNO_ERR_INVALID_ARG;
    if (V < B || V > UNO_MAX_TREE_NODES || (int64_t)V * K > UNO_MAX_TREE_FRONTIER) return UNO_ERR_INVALID_ARG;
    if (q_cap > 4096) return UNO_ERR_UNSUPPORTED;
    TreeJob J{};
    J.q_ids = q_ids;
    J.q_probs = q_probs;
    J.q_count = q_count;
    J.q_cap = q_cap;
    J.R = R;
    J.B = B;
    J.K = K;
    J.V = V;
    J.sort_cap = q_cap <= kTreeRankMax ? q_cap : next_pow2(q_cap);
    J.node_token = node_token;
    J.node_parent = node_parent;
    J.node_depth = node_depth;
    J.node_score = node_score;
    J.num_nodes = num_nodes;
    const size_t fixed = (size_t)V * 8 + (size_t)B * K * 8 + (size_t)B * 4;
    const size_t per_warp = align_up((size_t)J.sort_cap * 8, 8);
    // warps: one per marginal up to kTreeMaxWarps, as many as fit 200 KB
    int nw = B < kTreeMaxWarps ? B : kTreeMaxWarps;
    while (nw > 1 && fixed + (size_t)nw * per_warp > 200 * 1024) --nw;
    const size_t smem = fixed + (size_t)nw * per_warp;
    if (smem > 227 * 1024) return UNO_ERR_UNSUPPORTED;
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(tree_expand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return UNO_ERR_CUDA;
    }
    tree_expand_kernel<<<(unsigned)R, 32 * nw, smem, static_cast<cudaStream_t>(stream)>>>(J);
    return cudaGetLastError() == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}

static uno_status tree_verify_impl(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int32_t V, int64_t vocab,
                           uno_sampling_params sp, const uno_request_params* rp, const int32_t* node_token, const int32_t* node_parent,
                           const int32_t* num_nodes, uno_rng rng, int32_t* out_tokens, int32_t* out_accept_len,
                           int32_t* out_num_tokens, int32_t* out_path_nodes, uint32_t* out_flags, void* workspace,
                           size_t workspace_bytes, void* stream) {
    if (!target_logits || !node_token || !node_parent || !num_nodes || !out_tokens || !out_accept_len ||
        !out_num_tokens || !out_path_nodes || !out_flags)
        return UNO_ERR_INVALID_ARG;
    if (R <= 0 || B <= 0 || V <= 0 || vocab <= 0 || vocab > INT32_MAX) return UNO_ERR_INVALID_ARG;
    if (V < B || V > UNO_MAX_TREE_NODES) return UNO_ERR_INVALID_ARG;
    if (dt != UNO_F32 && dt != UNO_BF16) return UNO_ERR_INVALID_ARG;
    if (!params_ok(sp)) return UNO_ERR_INVALID_ARG;
    if (!rng_ok(rng)) return UNO_ERR_INVALID_ARG;
    if (!aligned_to(target_logits, dt == UNO_F32 ? 4 : 2)) return UNO_ERR_INVALID_ARG;
    if (sp.top_k > UNO_MAX_TOP_K) return UNO_ERR_UNSUPPORTED;
    const int32_t k = (int32_t)(sp.top_k < vocab ? sp.top_k : vocab);
    const int64_t rows = (int64_t)R * V;
    if ((int64_t)R > kCounterWords - kRowCounterWords) return UNO_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(rows, k, true);
    if (!workspace || workspace_bytes < L.total || !aligned_to(workspace, 16)) return UNO_ERR_WORKSPACE;

    RowJob J{};
    J.logits = static_cast<const unsigned char*>(target_logits);
    J.rows = rows;
    J.vocab = vocab;
    J.row_stride = vocab;
    J.rpr = V;
    J.temperature = sp.temperature;
    J.top_p = sp.top_p;
    J.k = k;
    apply_request_params(J, rp);
    J.seed = rng.seed;
    J.cycle = rng.cycle;
    J.cycle_word = rng.cycle_word;
    J.first_request = rng.first_request;
    J.B = B;
    J.V = V;
    J.node_token = node_token;
    J.node_parent = node_parent;
    J.num_nodes = num_nodes;
    J.out_tokens = out_tokens;
    J.out_accept_len = out_accept_len;
    J.out_num_tokens = out_num_tokens;
    J.out_path_nodes = out_path_nodes;
    J.out_req_flags = out_flags;
    bind_workspace(J, workspace, L);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return dt == UNO_BF16 ? launch_rows<__nv_bfloat16, kModeTree>(J, s) : launch_rows<float, kModeTree>(J, s);
}

// ---------------------------------------------------------------------------
// The entry points: one set with the call's sampling parameters, one with
// per-request parameter arrays and a filter order.
// ---------------------------------------------------------------------------
uno_status uno_filter_softmax(const void* logits, uno_dtype dt, int64_t rows, int64_t vocab, int64_t row_stride,
                              int32_t rows_per_request, uno_sampling_params sp, int32_t cap, int32_t* out_ids,
                              float* out_probs, int32_t* out_count, float* out_dense, const uno_rng* rng,
                              int32_t* out_sample, uint32_t* out_flags, void* workspace, size_t workspace_bytes,
                              void* stream) {
    return filter_softmax_impl(logits, dt, rows, vocab, row_stride, rows_per_request, sp, nullptr, cap, out_ids,
                               out_probs, out_count, out_dense, rng, out_sample, out_flags, workspace,
                               workspace_bytes, stream);
}

uno_status uno_filter_softmax_params(const void* logits, uno_dtype dt, int64_t rows, int64_t vocab,
                                     int64_t row_stride, int32_t rows_per_request, const uno_request_params* rp,
                                     int32_t cap, int32_t* out_ids, float* out_probs, int32_t* out_count,
                                     float* out_dense, const uno_rng* rng, int32_t* out_sample, uint32_t* out_flags,
                                     void* workspace, size_t workspace_bytes, void* stream) {
    if (!request_params_ok(rp)) return UNO_ERR_INVALID_ARG;
    return filter_softmax_impl(logits, dt, rows, vocab, row_stride, rows_per_request, bound_params(rp), rp, cap,
                               out_ids, out_probs, out_count, out_dense, rng, out_sample, out_flags, workspace,
                               workspace_bytes, stream);
}

uno_status uno_linear_verify(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int64_t vocab,
                             uno_sampling_params sp, const int32_t* draft_ids, const int32_t* q_ids,
                             const float* q_probs, const int32_t* q_count, int32_t q_cap, uno_rng rng,
                             int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_num_tokens,
                             uint32_t* out_flags, void* workspace, size_t workspace_bytes, void* stream) {
    return linear_verify_impl(target_logits, dt, R, B, vocab, sp, nullptr, draft_ids, q_ids, q_probs, q_count, q_cap,
                              rng, out_tokens, out_accept_len, out_num_tokens, out_flags, workspace, workspace_bytes,
                              stream);
}

uno_status uno_linear_verify_params(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int64_t vocab,
                                    const uno_request_params* rp, const int32_t* draft_ids, const int32_t* q_ids,
                                    const float* q_probs, const int32_t* q_count, int32_t q_cap, uno_rng rng,
                                    int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_num_tokens,
                                    uint32_t* out_flags, void* workspace, size_t workspace_bytes, void* stream) {
    if (!request_params_ok(rp)) return UNO_ERR_INVALID_ARG;
    return linear_verify_impl(target_logits, dt, R, B, vocab, bound_params(rp), rp, draft_ids, q_ids, q_probs,
                              q_count, q_cap, rng, out_tokens, out_accept_len, out_num_tokens, out_flags, workspace,
                              workspace_bytes, stream);
}

uno_status uno_linear_cycle(const void* draft_logits, const void* target_logits, uno_dtype dt, int32_t R, int32_t B,
                            int64_t vocab, int32_t layout, uno_sampling_params sp, uno_rng rng, int32_t* out_tokens,
                            int32_t* out_num_accepted, int32_t* out_num_tokens, uint32_t* out_flags,
                            int32_t* out_draft_ids, void* workspace, size_t workspace_bytes, void* stream) {
    return linear_cycle_impl(draft_logits, target_logits, dt, R, B, vocab, layout, sp, nullptr, rng, out_tokens,
                             out_num_accepted, out_num_tokens, out_flags, out_draft_ids, workspace, workspace_bytes,
                             stream);
}

uno_status uno_linear_cycle_params(const void* draft_logits, const void* target_logits, uno_dtype dt, int32_t R,
                                   int32_t B, int64_t vocab, int32_t layout, const uno_request_params* rp,
                                   uno_rng rng, int32_t* out_tokens, int32_t* out_num_accepted,
                                   int32_t* out_num_tokens, uint32_t* out_flags, int32_t* out_draft_ids,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    if (!request_params_ok(rp)) return UNO_ERR_INVALID_ARG;
    return linear_cycle_impl(draft_logits, target_logits, dt, R, B, vocab, layout, bound_params(rp), rp, rng,
                             out_tokens, out_num_accepted, out_num_tokens, out_flags, out_draft_ids, workspace,
                             workspace_bytes, stream);
}

uno_status uno_tree_verify(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int32_t V, int64_t vocab,
                           uno_sampling_params sp, const int32_t* node_token, const int32_t* node_parent,
                           const int32_t* num_nodes, uno_rng rng, int32_t* out_tokens, int32_t* out_accept_len,
                           int32_t* out_num_tokens, int32_t* out_path_nodes, uint32_t* out_flags, void* workspace,
                           size_t workspace_bytes, void* stream) {
    return tree_verify_impl(target_logits, dt, R, B, V, vocab, sp, nullptr, node_token, node_parent, num_nodes, rng,
                            out_tokens, out_accept_len, out_num_tokens, out_path_nodes, out_flags, workspace,
                            workspace_bytes, stream);
}

uno_status uno_tree_verify_params(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int32_t V,
                                  int64_t vocab, const uno_request_params* rp, const int32_t* node_token,
                                  const int32_t* node_parent, const int32_t* num_nodes, uno_rng rng,
                                  int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_num_tokens,
                                  int32_t* out_path_nodes, uint32_t* out_flags, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    if (!request_params_ok(rp)) return UNO_ERR_INVALID_ARG;
    return tree_verify_impl(target_logits, dt, R, B, V, vocab, bound_params(rp), rp, node_token, node_parent,
                            num_nodes, rng, out_tokens, out_accept_len, out_num_tokens, out_path_nodes, out_flags,
                            workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// uno_linear_verify_noalloc: uno_linear_verify with library-owned scratch.
//
// Some callers cannot hand the library a workspace: a serving loop that has
// already given all free device memory to its KV-cache pool, or a host
// program that loads this library as a plugin and offers it no allocator.
// For them the scratch lives in a file-scope device array that every GPU
// which loads the library holds until the process exits.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[UNO_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current context.  In host code
// the array's name is only a stand-in: each context that loads the library's
// module (a device's primary context, a driver-API context of a plugin host,
// the primary context again after cudaDeviceReset) holds its own copy at its
// own address.  Outside stream capture the address is looked up on every call
// (cudaGetSymbolAddress, cheap once the module is loaded), so a stale address
// is never used; the result is remembered per CUcontext for calls made while
// `s` is being captured, where a context cannot be reset.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

static CUcontext current_context() {
    static CtxGetCurrentFn fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<CtxGetCurrentFn>(f);
    }();
    CUcontext c = nullptr;
    if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

static uno_status noalloc_scratch(cudaStream_t s, unsigned char** out) {
    static std::mutex mu;
    constexpr int kSlots = 64;
    static CUcontext ctx[kSlots] = {nullptr};
    static unsigned char* addr[kSlots] = {nullptr};
    static int next = 0;
    const CUcontext c = current_context();
    if (c == nullptr) return UNO_ERR_CUDA;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return UNO_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    int at = -1;
    for (int i = 0; i < kSlots; ++i)
        if (ctx[i] == c) at = i;
    if (cs != cudaStreamCaptureStatusNone && at >= 0) {
        *out = addr[at];
        return UNO_OK;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return UNO_ERR_CUDA;
    if (at < 0) {
        at = next;
        next = (next + 1) % kSlots;
        ctx[at] = c;
    }
    addr[at] = static_cast<unsigned char*>(p);
    *out = addr[at];
    return UNO_OK;
}

uno_status uno_linear_verify_noalloc(const void* target_logits, uno_dtype dt, int32_t R, int32_t B, int64_t vocab,
                                     uno_sampling_params sp, const int32_t* draft_ids, const int32_t* q_ids,
                                     const float* q_probs, const int32_t* q_count, int32_t q_cap, uno_rng rng,
                                     int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_num_tokens,
                                     uint32_t* out_flags, void* stream) {
    if (!target_logits || !draft_ids || !q_ids || !q_probs || !q_count || !out_tokens || !out_accept_len ||
        !out_num_tokens || !out_flags)
        return UNO_ERR_INVALID_ARG;
    if (R <= 0 || B <= 0 || vocab <= 0 || vocab > INT32_MAX || q_cap < 1) return UNO_ERR_INVALID_ARG;
    if (dt != UNO_F32 && dt != UNO_BF16) return UNO_ERR_INVALID_ARG;
    if (!params_ok(sp)) return UNO_ERR_INVALID_ARG;
    if (!rng_ok(rng)) return UNO_ERR_INVALID_ARG;
    if (!aligned_to(target_logits, dt == UNO_F32 ? 4 : 2)) return UNO_ERR_INVALID_ARG;
    if (sp.top_k > UNO_MAX_TOP_K) return UNO_ERR_UNSUPPORTED;
    if ((int64_t)R > kCounterWords - kRowCounterWords) return UNO_ERR_UNSUPPORTED;
    const int32_t k = (int32_t)(sp.top_k < vocab ? sp.top_k : vocab);
    const int64_t rows = (int64_t)R * (B + 1);
    const WsLayout L = ws_layout(rows, k, true);
    if (L.total > (size_t)UNO_NOALLOC_SCRATCH_BYTES) return UNO_ERR_UNSUPPORTED;  // beyond the fixed scratch
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char* scratch = nullptr;
    const uno_status st = noalloc_scratch(s, &scratch);
    if (st != UNO_OK) return st;
    // the array keeps the last call's contents: clear the counters this call
    // may use: request tickets, and the tickets of split rows, which the
    // general kernel keys by row (rows <= kRowCounterWords only) and the
    // pipelined kernel by the row's first CTA (below kPipeMaxGrid), and the
    // pipelined kernel's run-time row counters (kDynOffset on)
    if (cudaMemsetAsync(scratch + L.req_ticket, 0, (size_t)R * 4, s) != cudaSuccess) return UNO_ERR_CUDA;
    int64_t nrow_words = kDynOffset + kDynWords + (rows > kPipeMaxGrid ? rows : kPipeMaxGrid);
    if (nrow_words > kRowCounterWords) nrow_words = kRowCounterWords;
    if (cudaMemsetAsync(scratch + L.row_ticket, 0, (size_t)nrow_words * 4, s) != cudaSuccess) return UNO_ERR_CUDA;

    RowJob J{};
    J.logits = static_cast<const unsigned char*>(target_logits);
    J.rows = rows;
    J.vocab = vocab;
    J.row_stride = vocab;
    J.rpr = B + 1;
    J.temperature = sp.temperature;
    J.top_p = sp.top_p;
    J.k = k;
    J.seed = rng.seed;
    J.cycle = rng.cycle;
    J.cycle_word = rng.cycle_word;
    J.first_request = rng.first_request;
    J.B = B;
    J.draft_ids = draft_ids;
    J.q_ids = q_ids;
    J.q_probs = q_probs;
    J.q_count = q_count;
    J.q_cap = q_cap;
    J.out_tokens = out_tokens;
    J.out_accept_len = out_accept_len;
    J.out_num_tokens = out_num_tokens;
    J.out_req_flags = out_flags;
    bind_workspace(J, scratch, L);
    return dt == UNO_BF16 ? launch_rows<__nv_bfloat16, kModeLinear>(J, s) : launch_rows<float, kModeLinear>(J, s);
}

}  // extern "C"
