// verify_full.cu — lossless block verify without top-k: softmax over the whole
// vocabulary, optionally followed by top-p.
//
// Same verify rule as the top-k path (LoopUno project page, "How it works" and "Training
// is self-distillation"; uno-qwen3-8B model card, "Evaluation protocol"); this path serves
// the unfiltered and the top-p-only sampler settings (the LoopUno runs use temperature 1.0
// and top-p 0.95 without top-k).
//
// Two launches. The rows pass handles every row (verifier rows 0..K-1 and drafter rows
// 1..K-1 of every sequence):
//   1. per chunk of CH elements, the maximum and the sum of exp(z - max) (z = logit / T);
//      from them the row's max M and sum S;
//   2. with top-p, the exact cut: the cut value tau, the mass above it and how many of the
//      tokens equal to tau are kept (the lowest ids: ties are ordered by id);
//   3. per chunk, the surviving mass and the number of tokens equal to tau.
// It has two forms. rows_cluster_kernel (bf16 rows, V a multiple of 8): a thread-block
// cluster per row, each CTA holding a slice of whole chunks in shared memory (one bulk copy,
// the next row's copied in meanwhile), row-wide reductions through distributed shared
// memory; the cut comes from counts per bf16 value (one exp per distinct value) where the
// values near the max span few keys. rows_kernel (any row): one CTA per row reading the row
// from global memory in every pass; the cut comes from a histogram of the mass over 1/8-nat
// bins below the max, then radix histograms over the order-preserving logit key (bits
// 31..24, then 23..16, ...: 2 levels for bf16 logits, 4 for fp32) restricted at each level
// to the crossing bin.
// seq_kernel: one CTA per sequence, one warp per block position for the draws, the
// probabilities and the acceptance, then the whole CTA for the residual and the TV.
// Draws (inverse CDF over ascending ids) walk the chunk table and then scan one chunk in
// id order; probabilities of single tokens need the token's rank among the tau-ties, from
// the table and a scan of its chunk. The correction token's residual max(0, p - q) and the
// optional TV take one more pass over the two rows involved.
// Sums are fp32 within a chunk and fp64 across chunks.
#include <cuda_bf16.h>

#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <type_traits>

#include "verify_common.cuh"

namespace uno {
namespace vfull {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kVecPerLane = 8;  // 16-byte vectors per lane per chunk

struct RowInfo {
    float M;        // max of z = logit / T
    int c_tie;      // number of tokens equal to tau that survive (top-p)
    uint32_t tau;   // key of the cut value (0: no cut, every token survives)
    int pad;
    double S;       // sum exp(z - M) over the row
    double Z;       // surviving mass (sum over survivors of exp(z - M))
    double w_tau;   // exp(z_tau - M)
};

struct Params {
    VerifyArgs a;
    int rows_per_seq;
    int nchunks;
    double* cmass;    // [B * rows_per_seq * nchunks] surviving mass per chunk (rel. to M)
    int* cties;       // [B * rows_per_seq * nchunks] tokens equal to tau per chunk
    double* cres;     // [B * nchunks] scratch: residual mass per chunk
    RowInfo* infos;   // [B * rows_per_seq]
    uint32_t* status; // device status word (bounded waits that give up)
};

template <typename T>
struct Chunk {
    static constexpr int VEC = Elem<T>::VEC;
    static constexpr int CH = 32 * VEC * kVecPerLane;  // elements per chunk
};

// element (vector j, lane, slot e) of chunk c in id order: c*CH + j*32*VEC + lane*VEC + e
template <typename T>
__device__ __forceinline__ uint4 load_vec(const T* row, int V, int c, int j, int lane, int& nv) {
    constexpr int VEC = Elem<T>::VEC;
    const int64_t e0 = (int64_t)c * Chunk<T>::CH + (int64_t)j * 32 * VEC + lane * VEC;
    nv = (int)max((int64_t)0, min((int64_t)VEC, (int64_t)V - e0));
    const bool aligned = ((reinterpret_cast<uintptr_t>(row + e0) & 15u) == 0);
    return nv > 0 ? load_raw<T>(row, e0, nv, aligned && nv == VEC) : make_uint4(0, 0, 0, 0);
}

// Full bf16 vectors: the 8 elements in id order, and packed tests that let a vector whose
// elements cannot pass a pass's test skip the per-element work (the exact test still
// decides every element of a vector that is not skipped).
__device__ __forceinline__ void unpack8(const uint4& v, float (&x)[8]) {
    x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x); x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
    x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z); x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
}
__device__ __forceinline__ __nv_bfloat162 as_b2(uint32_t w) { return *reinterpret_cast<__nv_bfloat162*>(&w); }
// some element >= lo
__device__ __forceinline__ bool any_ge(const uint4& v, __nv_bfloat162 lo) {
    const __nv_bfloat162 m = __hmax2(__hmax2(as_b2(v.x), as_b2(v.y)), __hmax2(as_b2(v.z), as_b2(v.w)));
    return __hge2_mask(m, lo) != 0u;
}
// some element in [lo, hi]
__device__ __forceinline__ bool any_in(const uint4& v, __nv_bfloat162 lo, __nv_bfloat162 hi) {
    const uint32_t m = (__hge2_mask(as_b2(v.x), lo) & __hle2_mask(as_b2(v.x), hi)) |
                       (__hge2_mask(as_b2(v.y), lo) & __hle2_mask(as_b2(v.y), hi)) |
                       (__hge2_mask(as_b2(v.z), lo) & __hle2_mask(as_b2(v.z), hi)) |
                       (__hge2_mask(as_b2(v.w), lo) & __hle2_mask(as_b2(v.w), hi));
    return m != 0u;
}
template <typename T>
constexpr bool kIsBf16 = sizeof(T) == 2;

// Order-preserving 16-bit keys of the two bf16 values of w (the top 16 bits of float_key of
// each): h ^ 0x8000 for a value >= +0, ~h for a negative one; -0 is taken as +0 first.
__device__ __forceinline__ uint32_t bf16x2_keys(uint32_t w) {
    w &= ~__vcmpeq2(w, 0x80008000u);
    return w ^ 0x80008000u ^ (((w >> 15) & 0x00010001u) * 0x7FFFu);
}

__device__ __forceinline__ double cta_sum_f64(double v, double* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum_f64(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < kWarps; ++w) t += red[w];
    __syncthreads();
    return t;
}

__device__ __forceinline__ float cta_max_f32(float v, float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_max(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = -INFINITY;
    for (int w = 0; w < kWarps; ++w) t = fmaxf(t, red[w]);
    __syncthreads();
    return t;
}

// ---------------------------------------------------------------------------------------
// where a row's elements come from, and which CTAs share the work of a row
// ---------------------------------------------------------------------------------------
// The whole row in global memory (per-row kernel).
template <typename T>
struct GlobalRow {
    const T* row;
    int V;
    __device__ __forceinline__ uint4 load(int c, int j, int lane, int& nv) const {
        return load_vec<T>(row, V, c, j, lane, nv);
    }
};

// This CTA's slice of a bf16 row in shared memory, starting at chunk c0 (cluster kernel;
// V is a multiple of 8, so every 8-element vector is either whole or past the end).
struct SharedSlice {
    const uint16_t* slice;
    int c0, V;
    __device__ __forceinline__ uint4 load(int c, int j, int lane, int& nv) const {
        constexpr int CH = Chunk<__nv_bfloat16>::CH;
        const int e0 = c * CH + j * 256 + lane * 8;
        nv = e0 < V ? 8 : 0;
        return nv ? lds128(slice + (e0 - c0 * CH)) : make_uint4(0u, 0u, 0u, 0u);
    }
};

__device__ __forceinline__ uint32_t cl_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cl_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cl_index() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cl_count() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// One CTA per row: the group is the CTA.
struct CtaGroup {
    __device__ __forceinline__ int size() const { return 1; }
    __device__ __forceinline__ void sync() const { __syncthreads(); }
    template <class X>
    __device__ __forceinline__ const X* peer(const X* p, int) const { return p; }
};

// A thread-block cluster per row: barriers are cluster barriers (release / acquire), and
// peer(p, r) is the generic address of p's counterpart in the shared memory of CTA r.
struct ClusterGroup {
    int n;
    __device__ __forceinline__ int size() const { return n; }
    __device__ __forceinline__ void sync() const {
        asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    }
    template <class X>
    __device__ __forceinline__ const X* peer(const X* p, int r) const {
        uint64_t q;
        asm volatile("mapa.u64 %0, %1, %2;" : "=l"(q) : "l"(reinterpret_cast<uint64_t>(p)), "r"(r));
        return reinterpret_cast<const X*>(q);
    }
};

// What each CTA of a group publishes for a row-wide reduction: its partials, read by every
// CTA of the group after a group barrier. Two areas are used in turn, so that one barrier
// per exchange suffices (area e is rewritten at exchange e + 2, after every CTA has passed
// the barrier of exchange e + 1 and so has finished reading it).
struct Xchg {
    double mass[256];
    uint32_t cnt[256];
    double s;
    float m;
    int pad;
};

// Units of the cluster kernel's balanced passes: vector row j of a chunk, one 16-byte vector
// per lane (a CTA's slice has at most kMaxUnits of them).
constexpr int kMaxUnits = 192;
constexpr int kUB = 4;  // units (or vectors) a warp (thread) works on at a time in the slice passes
// Keys of the exact cut histogram (bf16 values: 16-bit keys; 16 per thread of the first 256).
constexpr int kKeyBins = 4096;

struct RowShared {
    float hist_f[256 * kWarps];   // per-warp histograms; the group's key counts (as uint32)
    uint32_t hist_n[256 * kWarps];  // per-warp histograms; this CTA's key counts
    double comb_m[256];           // the group's histogram; key-mass partial sums
    uint32_t comb_n[256];
    double dred[kWarps];
    float fred[kWarps];
    float ustat[kMaxUnits];       // per unit: max (then survivor mass)
    float usum[kMaxUnits];        // per unit: sum of exps
    int uties[kMaxUnits];         // per unit: tokens equal to the cut
    float cmx[kMaxUnits / kVecPerLane];  // per chunk of the slice: max
    Xchg x[2];
};
static_assert(kKeyBins <= 256 * kWarps, "key counts live in the histogram arrays");

// ---------------------------------------------------------------------------------------
// per row: statistics, top-p cut, per-chunk survivor table (a CTA, or a cluster of CTAs each
// holding a slice of the row)
// ---------------------------------------------------------------------------------------
// Chunks [c0, c1) of the row are this CTA's; cmass and cties are indexed by the row's chunk
// index; info (written if not null) receives the row's RowInfo, which every CTA of the group
// computes identically (every CTA combines the same partials in the same order). xe counts
// the exchanges made so far.
template <typename T, typename Src, typename Grp>
__device__ void prepare_row(const Src& src, const VerifyArgs& a, int c0, int c1, double* cmass, int* cties,
                            RowInfo* info, RowShared& sh, const Grp& grp, int& xe) {
    constexpr int NLEVELS = sizeof(T) == 2 ? 2 : 4;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int V = a.V;
    const float invT = 1.0f / a.temperature;

    constexpr bool kSlice = std::is_same<Src, SharedSlice>::value;
    constexpr int CH = Chunk<T>::CH;
    const int U = (c1 - c0) * kVecPerLane;  // units of this CTA (slice form)

    // 1. per chunk max and sum; row max and sum
    float lmax = -INFINITY;
    if constexpr (kSlice) {
        // balanced over the warps: unit u = vector row u % 8 of chunk c0 + u / 8; each warp
        // takes UB of its units at a time, so that their loads and reductions overlap
        for (int ub = warp; ub < U; ub += kUB * kWarps) {
            float m[kUB];
#pragma unroll
            for (int k = 0; k < kUB; ++k) {
                const int u = ub + k * kWarps;
                m[k] = -INFINITY;
                if (u < U) {
                    int nv;
                    const uint4 v = src.load(c0 + u / kVecPerLane, u % kVecPerLane, lane, nv);
                    if (nv == 8) {
                        const __nv_bfloat162 m2 =
                            __hmax2(__hmax2(as_b2(v.x), as_b2(v.y)), __hmax2(as_b2(v.z), as_b2(v.w)));
                        m[k] = fmaxf(__low2float(m2), __high2float(m2)) * invT;
                    }
                }
            }
#pragma unroll
            for (int off = 16; off; off >>= 1)
#pragma unroll
                for (int k = 0; k < kUB; ++k) m[k] = fmaxf(m[k], __shfl_xor_sync(kFullMask, m[k], off));
            if (lane == 0)
#pragma unroll
                for (int k = 0; k < kUB; ++k)
                    if (ub + k * kWarps < U) sh.ustat[ub + k * kWarps] = m[k];
        }
        __syncthreads();
        for (int c = c0 + threadIdx.x; c < c1; c += kThreads) {
            const float* um = sh.ustat + (c - c0) * kVecPerLane;
            float cm = um[0];
            for (int k = 1; k < kVecPerLane; ++k) cm = fmaxf(cm, um[k]);
            sh.cmx[c - c0] = cm;
        }
        __syncthreads();
        for (int ub = warp; ub < U; ub += kUB * kWarps) {
            float cs[kUB];
#pragma unroll
            for (int k = 0; k < kUB; ++k) {
                const int u = ub + k * kWarps;
                cs[k] = 0.f;
                if (u < U) {
                    int nv;
                    const uint4 v = src.load(c0 + u / kVecPerLane, u % kVecPerLane, lane, nv);
                    if (nv == 8) {
                        const float cm = sh.cmx[u / kVecPerLane];
                        float x[8];
                        unpack8(v, x);
#pragma unroll
                        for (int e = 0; e < 8; ++e) cs[k] += __expf(x[e] * invT - cm);
                    }
                }
            }
#pragma unroll
            for (int off = 16; off; off >>= 1)
#pragma unroll
                for (int k = 0; k < kUB; ++k) cs[k] += __shfl_xor_sync(kFullMask, cs[k], off);
            if (lane == 0)
#pragma unroll
                for (int k = 0; k < kUB; ++k)
                    if (ub + k * kWarps < U) sh.usum[ub + k * kWarps] = cs[k];
        }
        __syncthreads();
        for (int c = c0 + threadIdx.x; c < c1; c += kThreads) {
            const int u0 = (c - c0) * kVecPerLane;
            const float cm = sh.cmx[c - c0];
            double cs = 0.0;
            for (int k = 0; k < kVecPerLane; ++k) cs += (double)sh.usum[u0 + k];
            cmass[c] = cs;                             // relative to the chunk max for now
            reinterpret_cast<float*>(cties)[c] = cm;  // chunk max parked in the ties slot
            lmax = fmaxf(lmax, cm);
        }
    } else
    for (int c = c0 + warp; c < c1; c += kWarps) {
        float cm = -INFINITY;
        for (int j = 0; j < kVecPerLane; ++j) {
            int nv;
            uint4 v = src.load(c, j, lane, nv);
            if constexpr (kIsBf16<T>) {
                if (nv == 8) {
                    const __nv_bfloat162 m2 = __hmax2(__hmax2(as_b2(v.x), as_b2(v.y)), __hmax2(as_b2(v.z), as_b2(v.w)));
                    cm = fmaxf(cm, fmaxf(__low2float(m2), __high2float(m2)) * invT);
                    continue;
                }
            }
            for (int e = 0; e < nv; ++e) cm = fmaxf(cm, raw_get<T>(v, e) * invT);
        }
        cm = warp_max(cm);
        float cs = 0.f;
        for (int j = 0; j < kVecPerLane; ++j) {
            int nv;
            uint4 v = src.load(c, j, lane, nv);
            if constexpr (kIsBf16<T>) {
                if (nv == 8) {
                    float x[8];
                    unpack8(v, x);
#pragma unroll
                    for (int e = 0; e < 8; ++e) cs += __expf(x[e] * invT - cm);
                    continue;
                }
            }
            for (int e = 0; e < nv; ++e) cs += __expf(raw_get<T>(v, e) * invT - cm);
        }
        cs = warp_sum(cs);
        if (lane == 0) {
            cmass[c] = (double)cs;               // relative to the chunk max for now
            reinterpret_cast<float*>(cties)[c] = cm;  // chunk max parked in the ties slot
        }
        lmax = fmaxf(lmax, cm);
    }
    // this CTA's max and its sum relative to it; then the group's M and S
    const float mc = cta_max_f32(lmax, sh.fred);
    double part = 0.0;
    for (int c = c0 + threadIdx.x; c < c1; c += kThreads)
        part += cmass[c] * exp((double)reinterpret_cast<float*>(cties)[c] - (double)mc);
    const double sc = cta_sum_f64(part, sh.dred);
    float M;
    double S = 0.0;
    {
        Xchg& xo = sh.x[xe++ & 1];
        if (threadIdx.x == 0) {
            xo.m = mc;
            xo.s = sc;
        }
        grp.sync();
        // every warp combines the group's partials, lane r taking CTA r's (a CTA without
        // chunks sends 0 and -inf); the fixed lane order makes the sums identical everywhere
        float mr = -INFINITY;
        double sr = 0.0;
        if (lane < grp.size()) {
            const Xchg* xr = grp.peer(&xo, lane);
            mr = xr->m;
            sr = xr->s;
        }
        M = warp_max(mr);
        S = warp_sum_f64(lane < grp.size() ? sr * exp((double)mr - (double)M) : 0.0);
    }
    for (int c = c0 + threadIdx.x; c < c1; c += kThreads) {
        cmass[c] = cmass[c] * exp((double)reinterpret_cast<float*>(cties)[c] - (double)M);
        cties[c] = 0;
    }
    RowInfo ri{};
    ri.M = M;
    ri.S = S;
    ri.Z = S;
    ri.tau = 0u;
    ri.c_tie = 0;
    ri.w_tau = 0.0;
    if (a.top_p < 1.0f) {
        // 2. exact top-p cut by radix histograms of the mass over the logit keys
        const double target = (double)a.top_p * S;
        // level A: mass by distance below the max, 1/8-nat bins (the radix levels below,
        // restricted to the crossing bin, then fix the exact cut). Binning by value spreads
        // the elements over many bins, where the first radix level over the key's top bits
        // would put most of them in a few.
        auto vbin = [&](float x) {
            const float d = M - x * invT;
            return d < 31.875f ? (int)(d * 8.f) : 255;
        };
        // Only elements within D nats of the max are binned: those further down weigh at
        // most V e^-D together, which is below the mass top-p leaves out when
        // D >= ln(V / ((1 - top_p) S)), so the cut lies within D (a full pass is the
        // fallback for rounding).
        // (D is a whole number of bins, so that a bin is either binned in full or not at all)
        const double dcut = log((double)V / ((1.0 - (double)a.top_p) * S)) + 0.5;
        float D = dcut > 31.875 ? 31.875f : (dcut < 0.125 ? 0.125f : ceilf((float)dcut * 8.f) * 0.125f);
        uint32_t tau = 0u;      // key of the cut value
        double above = 0.0;     // mass of the keys above it
        uint32_t count_at = 0;  // tokens equal to it (0: no cut, every token survives)
        bool have_cut = false;
        if constexpr (kSlice) {
            // Exact cut from counts per bf16 value: every token with the same value has the same
            // weight, so the mass of a value is its count times one exp (fp64). The values within
            // D of the max span at most kKeyBins 16-bit keys unless the range reaches close to 0;
            // otherwise (or if rounding leaves the target unmet) the histograms below decide.
            const float hiv = __bfloat162float(__float2bfloat16_ru(M * a.temperature));  // >= the max logit
            const float lov = __bfloat162float(__float2bfloat16_rd((M - D) * a.temperature));
            const uint32_t hi16 = float_key(hiv) >> 16, lo16 = float_key(lov) >> 16;
            const uint32_t R = hi16 >= lo16 ? hi16 - lo16 + 1u : 0u;
            if (R > 0u && R <= (uint32_t)kKeyBins) {
                uint32_t* kc = sh.hist_n;                                // this CTA's counts (read by the group)
                uint32_t* tot = reinterpret_cast<uint32_t*>(sh.hist_f);  // the group's counts
                auto key_weight = [&](uint32_t k16) {  // a token's weight exp(z - M), for a bf16 key
                    const uint32_t k = (k16 << 16) | ((k16 & 0x8000u) ? 0x0000u : 0xFFFFu);
                    return (double)__expf(key_float(k) * invT - M);
                };
                for (int i = threadIdx.x; i < (int)R; i += kThreads) kc[i] = 0u;
                __syncthreads();
                const __nv_bfloat162 lo2 = __float2bfloat162_rn(lov);  // lov is a bf16 value
                const int nvec = c1 > c0 ? (int)((min((int64_t)V, (int64_t)c1 * CH) - (int64_t)c0 * CH) / 8) : 0;
                for (int i0 = threadIdx.x; i0 < nvec; i0 += kUB * kThreads) {
                    uint4 vb[kUB];
#pragma unroll
                    for (int k = 0; k < kUB; ++k) {
                        const int i = i0 + k * kThreads;
                        vb[k] = i < nvec ? lds128(src.slice + (size_t)i * 8) : make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                    for (int k = 0; k < kUB; ++k) {
                        if (i0 + k * kThreads >= nvec || !any_ge(vb[k], lo2)) continue;
                        const uint32_t w4[4] = {vb[k].x, vb[k].y, vb[k].z, vb[k].w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint32_t k2 = bf16x2_keys(w4[q]);
                            const uint32_t ka = (k2 & 0xFFFFu) - lo16, kb = (k2 >> 16) - lo16;
                            if (ka < R) atomicAdd(&kc[ka], 1u);
                            if (kb < R) atomicAdd(&kc[kb], 1u);
                        }
                    }
                }
                grp.sync();  // every CTA's counts are complete
                for (int i = threadIdx.x; i < (int)R; i += kThreads) {
                    uint32_t n = 0;
                    for (int r = 0; r < grp.size(); ++r) n += grp.peer(kc, r)[i];
                    tot[i] = n;
                }
                __syncthreads();
                // mass of 16 keys per thread (threads 0..255), from the top key down
                constexpr int KPT = kKeyBins / 256;
                if (threadIdx.x < 256) {
                    double msum = 0.0;
                    for (int q = 0; q < KPT; ++q) {
                        const int idx = (int)R - 1 - ((int)threadIdx.x * KPT + q);
                        if (idx >= 0 && tot[idx]) msum += (double)tot[idx] * key_weight(lo16 + (uint32_t)idx);
                    }
                    sh.comb_m[threadIdx.x] = msum;
                }
                __syncthreads();
                if (warp == 0) {
                    double cum = 0.0, t_excl = 0.0;
                    int t_hit = -1;
                    for (int t0 = 0; t0 < 256 && t_hit < 0; t0 += 32) {
                        const double m = sh.comb_m[t0 + lane];
                        const double incl = warp_scan_f64(m, lane);
                        const unsigned hit = __ballot_sync(kFullMask, cum + incl >= target && m > 0.0);
                        if (hit) {
                            const int hl = __ffs(hit) - 1;
                            t_hit = t0 + hl;
                            t_excl = cum + __shfl_sync(kFullMask, incl - m, hl);
                        }
                        cum += __shfl_sync(kFullMask, incl, 31);
                    }
                    if (lane == 0) {
                        // the key within that thread's range where the mass reaches the target
                        // (the last non-empty one if rounding leaves it a hair short)
                        int idx_hit = -1;
                        double ab = 0.0, c = t_excl;
                        uint32_t n_hit = 0;
                        for (int q = 0; t_hit >= 0 && q < KPT; ++q) {
                            const int idx = (int)R - 1 - (t_hit * KPT + q);
                            if (idx < 0) break;
                            const uint32_t n = tot[idx];
                            if (!n) continue;
                            const double w = (double)n * key_weight(lo16 + (uint32_t)idx);
                            idx_hit = idx;
                            ab = c;
                            n_hit = n;
                            if (c + w >= target) break;
                            c += w;
                        }
                        sh.dred[0] = ab;
                        sh.dred[1] = (double)idx_hit;
                        sh.dred[2] = (double)n_hit;
                    }
                }
                __syncthreads();
                const int idx_hit = (int)sh.dred[1];
                if (idx_hit >= 0) {
                    have_cut = true;
                    const uint32_t k16 = lo16 + (uint32_t)idx_hit;
                    tau = (k16 << 16) | ((k16 & 0x8000u) ? 0x0000u : 0xFFFFu);
                    above = sh.dred[0];
                    count_at = (uint32_t)sh.dred[2];
                }
                __syncthreads();
            }
        }
        if (!have_cut) {
        int vchosen = -1;
        double vabove = 0.0;
        for (int attempt = 0; attempt < 2 && vchosen < 0; ++attempt) {
            if (attempt == 1) D = INFINITY;  // every element
            for (int i = threadIdx.x; i < 256 * kWarps; i += kThreads) sh.hist_f[i] = 0.f;
            __syncthreads();
            float* hf = sh.hist_f + warp * 256;
            // packed prefilter: a logit below (M - D) T - 1/16 (rounded down) cannot pass
            const __nv_bfloat162 alo = D == INFINITY
                                           ? __float2bfloat162_rn(-INFINITY)
                                           : __bfloat162bfloat162(__float2bfloat16_rd(((M - D) - 0.0625f) * a.temperature));
            for (int c = c0 + warp; c < c1; c += kWarps) {
                for (int j = 0; j < kVecPerLane; ++j) {
                    int nv;
                    uint4 v = src.load(c, j, lane, nv);
                    if constexpr (kIsBf16<T>) {
                        if (nv == 8) {
                            if (!any_ge(v, alo)) continue;
                            float x[8];
                            unpack8(v, x);
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                if (M - x[e] * invT < D) atomicAdd(&hf[vbin(x[e])], __expf(x[e] * invT - M));
                            continue;
                        }
                    }
                    for (int e = 0; e < nv; ++e) {
                        const float x = raw_get<T>(v, e);
                        if (M - x * invT < D) atomicAdd(&hf[vbin(x)], __expf(x * invT - M));
                    }
                }
            }
            __syncthreads();
            {
                Xchg& xo = sh.x[xe++ & 1];
                for (int bin = threadIdx.x; bin < 256; bin += kThreads) {
                    double m = 0.0;
                    for (int w = 0; w < kWarps; ++w) m += (double)sh.hist_f[w * 256 + bin];
                    xo.mass[bin] = m;
                }
                grp.sync();
                for (int bin = threadIdx.x; bin < 256; bin += kThreads) {
                    double m = 0.0;
                    for (int r = 0; r < grp.size(); ++r) m += grp.peer(&xo, r)->mass[bin];
                    sh.comb_m[bin] = m;
                }
                __syncthreads();
            }
            if (warp == 0) {
            double cum = 0.0;
            int chosen = -1;
            double chosen_above = 0.0;
            for (int b0 = 0; b0 < 256 && chosen < 0; b0 += 32) {
                const int bin = b0 + lane;
                const double m = sh.comb_m[bin];
                const double incl = warp_scan_f64(m, lane);
                // (a bin whose elements all underflow to 0 cannot be where the mass crosses)
                const unsigned hit = __ballot_sync(kFullMask, cum + incl >= target && m > 0.0);
                if (hit) {
                    const int hl = __ffs(hit) - 1;
                    chosen = b0 + hl;
                    chosen_above = cum + __shfl_sync(kFullMask, incl - m, hl);
                }
                cum += __shfl_sync(kFullMask, incl, 31);
            }
            if (lane == 0) {
                sh.dred[0] = chosen_above;
                sh.dred[1] = (double)chosen;
            }
            }
            __syncthreads();
            vchosen = (int)sh.dred[1];  // -1: the binned mass falls short of the target
            vabove = sh.dred[0];
            __syncthreads();
        }
        uint32_t prefix = 0;     // key bits fixed so far
        above = vchosen >= 0 ? vabove : 0.0;  // mass of keys above the current prefix bin
        count_at = 0;
        // packed prefilter of the radix levels: the logits of the chosen bin lie within
        // [(M - (b + 1) / 8) T, (M - b / 8) T], widened by 1/16 and rounded outwards
        const float vlo = (M - (vchosen + 1) * 0.125f - 0.0625f) * a.temperature;
        const float vhi = (M - vchosen * 0.125f + 0.0625f) * a.temperature;
        const __nv_bfloat162 rlo = vchosen == 255 ? __float2bfloat162_rn(-INFINITY)
                                                  : __bfloat162bfloat162(__float2bfloat16_rd(vlo));
        const __nv_bfloat162 rhi = __bfloat162bfloat162(__float2bfloat16_ru(vhi));
        for (int level = 0; level < NLEVELS && vchosen >= 0; ++level) {
            const int shift = 24 - 8 * level;
            const uint32_t hi_mask = level == 0 ? 0u : (~0u << (shift + 8));
            for (int i = threadIdx.x; i < 256 * kWarps; i += kThreads) {
                sh.hist_f[i] = 0.f;
                sh.hist_n[i] = 0u;
            }
            __syncthreads();
            float* hf = sh.hist_f + warp * 256;
            uint32_t* hn = sh.hist_n + warp * 256;
            for (int c = c0 + warp; c < c1; c += kWarps) {
                for (int j = 0; j < kVecPerLane; ++j) {
                    int nv;
                    uint4 v = src.load(c, j, lane, nv);
                    if constexpr (kIsBf16<T>) {
                        if (nv == 8) {
                            if (!any_in(v, rlo, rhi)) continue;
                            float x[8];
                            unpack8(v, x);
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const uint32_t key = float_key(x[e]);
                                if ((key & hi_mask) == prefix && vbin(x[e]) == vchosen) {
                                    const uint32_t bin = (key >> shift) & 0xFFu;
                                    atomicAdd(&hf[bin], __expf(x[e] * invT - M));
                                    atomicAdd(&hn[bin], 1u);
                                }
                            }
                            continue;
                        }
                    }
                    for (int e = 0; e < nv; ++e) {
                        const float x = raw_get<T>(v, e);
                        const uint32_t key = float_key(x);
                        if ((key & hi_mask) == prefix && vbin(x) == vchosen) {
                            const uint32_t bin = (key >> shift) & 0xFFu;
                            atomicAdd(&hf[bin], __expf(x * invT - M));
                            atomicAdd(&hn[bin], 1u);
                        }
                    }
                }
            }
            __syncthreads();
            // combine the warps' histograms, then the group's; walk bins from the top
            {
                Xchg& xo = sh.x[xe++ & 1];
                for (int bin = threadIdx.x; bin < 256; bin += kThreads) {
                    double m = 0.0;
                    uint32_t n = 0;
                    for (int w = 0; w < kWarps; ++w) {
                        m += (double)sh.hist_f[w * 256 + bin];
                        n += sh.hist_n[w * 256 + bin];
                    }
                    xo.mass[bin] = m;
                    xo.cnt[bin] = n;
                }
                grp.sync();
                for (int bin = threadIdx.x; bin < 256; bin += kThreads) {
                    double m = 0.0;
                    uint32_t n = 0;
                    for (int r = 0; r < grp.size(); ++r) {
                        const Xchg* xr = grp.peer(&xo, r);
                        m += xr->mass[bin];
                        n += xr->cnt[bin];
                    }
                    sh.comb_m[bin] = m;
                    sh.comb_n[bin] = n;
                }
                __syncthreads();
            }
            if (warp == 0) {
                double cum = above;
                int chosen = -1;
                double chosen_above = above;
                uint32_t chosen_n = 0;
                for (int b0 = 255; b0 >= 0 && chosen < 0; b0 -= 32) {
                    const int bin = b0 - lane;
                    const double m = sh.comb_m[bin];
                    const uint32_t n = sh.comb_n[bin];
                    const double incl = warp_scan_f64(m, lane);
                    const unsigned hit = __ballot_sync(kFullMask, cum + incl >= target && n > 0);
                    if (hit) {
                        const int hl = __ffs(hit) - 1;
                        chosen = b0 - hl;
                        chosen_above = cum + __shfl_sync(kFullMask, incl - m, hl);
                        chosen_n = __shfl_sync(kFullMask, n, hl);
                    }
                    cum += __shfl_sync(kFullMask, incl, 31);
                }
                if (chosen < 0) {  // rounding: the whole mass falls short of the target; keep everything
                    chosen = -2;
                }
                if (lane == 0) {
                    sh.dred[0] = chosen_above;
                    sh.dred[1] = (double)chosen;
                    sh.dred[2] = (double)chosen_n;
                }
            }
            __syncthreads();
            const int chosen = (int)sh.dred[1];
            if (chosen == -2) {
                prefix = 0;
                above = 0.0;
                count_at = 0;
                break;
            }
            above = sh.dred[0];
            count_at = (uint32_t)sh.dred[2];
            prefix |= (uint32_t)chosen << shift;
            __syncthreads();
        }
        if (count_at > 0) {
            // the cut value; for bf16 logits the low 16 key bits follow from the sign
            tau = prefix;
            if (NLEVELS == 2) tau |= (tau & 0x80000000u) ? 0x0000u : 0xFFFFu;
        }
        }  // !have_cut
        if (count_at > 0) {
            const double w_tau = exp((double)key_float(tau) / (double)a.temperature - (double)M);
            double need = (target - above) / w_tau;
            int c_tie = (int)ceil(need - 1e-12);
            c_tie = c_tie < 1 ? 1 : (c_tie > (int)count_at ? (int)count_at : c_tie);
            ri.tau = tau;
            ri.c_tie = c_tie;
            ri.w_tau = w_tau;
            ri.Z = above + (double)c_tie * w_tau;
            // 3. per chunk: mass of keys above tau, and the number of tokens equal to tau
            if constexpr (kSlice) {
                const __nv_bfloat162 tlo = __float2bfloat162_rn(key_float(tau));  // tau is a bf16 value here
                for (int ub = warp; ub < U; ub += kUB * kWarps) {
                    float mg[kUB];
                    int nt[kUB];
#pragma unroll
                    for (int k = 0; k < kUB; ++k) {
                        const int u = ub + k * kWarps;
                        mg[k] = 0.f;
                        nt[k] = 0;
                        if (u < U) {
                            int nv;
                            const uint4 v = src.load(c0 + u / kVecPerLane, u % kVecPerLane, lane, nv);
                            if (nv == 8 && any_ge(v, tlo)) {
                                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    // IEEE comparisons of bf16 values order them as their keys
                                    // do (-0 equal to +0)
                                    const uint32_t gt = __hgt2_mask(as_b2(w4[q]), tlo);
                                    const uint32_t eq = __heq2_mask(as_b2(w4[q]), tlo);
                                    if (gt & 0xFFFFu) mg[k] += __expf(bf16_lo(w4[q]) * invT - M);
                                    if (gt >> 16) mg[k] += __expf(bf16_hi(w4[q]) * invT - M);
                                    nt[k] += (int)((eq & 1u) + (eq >> 31));
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int off = 16; off; off >>= 1)
#pragma unroll
                        for (int k = 0; k < kUB; ++k) {
                            mg[k] += __shfl_xor_sync(kFullMask, mg[k], off);
                            nt[k] += __shfl_xor_sync(kFullMask, nt[k], off);
                        }
                    if (lane == 0)
#pragma unroll
                        for (int k = 0; k < kUB; ++k)
                            if (ub + k * kWarps < U) {
                                sh.ustat[ub + k * kWarps] = mg[k];
                                sh.uties[ub + k * kWarps] = nt[k];
                            }
                }
                __syncthreads();
                for (int c = c0 + threadIdx.x; c < c1; c += kThreads) {
                    const int u0 = (c - c0) * kVecPerLane;
                    double m = 0.0;
                    int n = 0;
                    for (int k = 0; k < kVecPerLane; ++k) {
                        m += (double)sh.ustat[u0 + k];
                        n += sh.uties[u0 + k];
                    }
                    cmass[c] = m;
                    cties[c] = n;
                }
            } else
            for (int c = c0 + warp; c < c1; c += kWarps) {
                float mg = 0.f;
                int nt = 0;
                const __nv_bfloat162 tlo = __float2bfloat162_rn(key_float(tau));  // tau is a bf16 value here
                for (int j = 0; j < kVecPerLane; ++j) {
                    int nv;
                    uint4 v = src.load(c, j, lane, nv);
                    if constexpr (kIsBf16<T>) {
                        if (nv == 8) {
                            if (!any_ge(v, tlo)) continue;
                            float x[8];
                            unpack8(v, x);
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const uint32_t key = float_key(x[e]);
                                if (key > tau) mg += __expf(x[e] * invT - M);
                                nt += key == tau;
                            }
                            continue;
                        }
                    }
                    for (int e = 0; e < nv; ++e) {
                        const float x = raw_get<T>(v, e);
                        const uint32_t key = float_key(x);
                        if (key > tau) mg += __expf(x * invT - M);
                        nt += key == tau;
                    }
                }
                mg = warp_sum(mg);
                nt = warp_sum(nt);
                if (lane == 0) {
                    cmass[c] = (double)mg;
                    cties[c] = nt;
                }
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && info) *info = ri;
    __syncthreads();
}

// ---------------------------------------------------------------------------------------
// warp-level walks over one row
// ---------------------------------------------------------------------------------------
// surviving mass of chunk c given the ties that precede it
__device__ __forceinline__ double chunk_surv(const RowInfo& ri, const double* cmass, const int* cties, int c,
                                             int ties_before) {
    if (ri.tau == 0u) return cmass[c];
    const int kept = max(0, min(ri.c_tie - ties_before, cties[c]));
    return cmass[c] + (double)kept * ri.w_tau;
}

// Scan chunk c of the row in id order; for every element calls f(id, z, survivor weight,
// lane) — all lanes call f for their elements of each 32-lane vector in turn.
template <typename T, typename F>
__device__ __forceinline__ void scan_chunk(const T* row, const VerifyArgs& a, const RowInfo& ri, int c,
                                           int ties_before, int lane, F f) {
    constexpr int VEC = Elem<T>::VEC;
    const float invT = 1.0f / a.temperature;
    int carry = ties_before;
    for (int j = 0; j < kVecPerLane; ++j) {
        int nv;
        const uint4 v = load_vec<T>(row, a.V, c, j, lane, nv);
        int nt = 0;
        for (int e = 0; e < nv; ++e) nt += float_key(raw_get<T>(v, e)) == ri.tau;
        const int incl = warp_inclusive_scan(nt, lane);
        int rank = carry + incl - nt;
        const int64_t id0 = (int64_t)c * Chunk<T>::CH + (int64_t)j * 32 * VEC + lane * VEC;
        double wv[Elem<T>::VEC];
        for (int e = 0; e < VEC; ++e) {
            wv[e] = 0.0;
            if (e < nv) {
                const float x = raw_get<T>(v, e);
                const uint32_t key = float_key(x);
                bool surv = ri.tau == 0u || key > ri.tau;
                if (ri.tau != 0u && key == ri.tau) surv = rank++ < ri.c_tie;
                if (surv) wv[e] = (double)__expf(x * invT - ri.M);
            }
        }
        f(id0, wv, nv, j);
        carry += __shfl_sync(kFullMask, incl, 31);
    }
}

// Scan chunk c of two rows (verifier p, drafter q) together in id order; for every vector
// of 32 lanes calls f(id0, wp, wq, nv) with the lane's normalised survivor probabilities
// of both rows (reciprocals of the rows' surviving masses taken once).
template <typename T, typename F>
__device__ __forceinline__ void scan_pair_chunk(const T* prow, const T* qrow, const VerifyArgs& a, const RowInfo& rp,
                                                const RowInfo& rq, int c, int tbp, int tbq, int lane, F f) {
    constexpr int VEC = Elem<T>::VEC;
    const float invT = 1.0f / a.temperature;
    const double izp = 1.0 / rp.Z, izq = 1.0 / rq.Z;
    int carp = tbp, carq = tbq;
    for (int j = 0; j < kVecPerLane; ++j) {
        int nv;
        const uint4 vp = load_vec<T>(prow, a.V, c, j, lane, nv);
        const uint4 vq = load_vec<T>(qrow, a.V, c, j, lane, nv);
        int ntp = 0, ntq = 0;
        for (int e = 0; e < nv; ++e) {
            ntp += float_key(raw_get<T>(vp, e)) == rp.tau;
            ntq += float_key(raw_get<T>(vq, e)) == rq.tau;
        }
        const int ip = warp_inclusive_scan(ntp, lane), iq = warp_inclusive_scan(ntq, lane);
        int rkp = carp + ip - ntp, rkq = carq + iq - ntq;
        const int64_t id0 = (int64_t)c * Chunk<T>::CH + (int64_t)j * 32 * VEC + lane * VEC;
        double wp[VEC], wq[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            wp[e] = 0.0;
            wq[e] = 0.0;
            if (e < nv) {
                const float xp = raw_get<T>(vp, e), xq = raw_get<T>(vq, e);
                const uint32_t kp = float_key(xp), kq = float_key(xq);
                bool sp = rp.tau == 0u || kp > rp.tau, sq = rq.tau == 0u || kq > rq.tau;
                if (rp.tau != 0u && kp == rp.tau) sp = rkp++ < rp.c_tie;
                if (rq.tau != 0u && kq == rq.tau) sq = rkq++ < rq.c_tie;
                if (sp) wp[e] = (double)__expf(xp * invT - rp.M) * izp;
                if (sq) wq[e] = (double)__expf(xq * invT - rq.M) * izq;
            }
        }
        f(id0, wp, wq, nv);
        carp += __shfl_sync(kFullMask, ip, 31);
        carq += __shfl_sync(kFullMask, iq, 31);
    }
}

// inverse-CDF draw over the row's survivors with uniform u (one warp)
template <typename T>
__device__ int warp_row_draw(const T* row, const VerifyArgs& a, const RowInfo& ri, const double* cmass,
                             const int* cties, int nchunks, double u, int lane) {
    const double target = u * ri.Z;
    double carry = 0.0;
    int tcarry = 0;
    int cstar = -1, tstar = 0;
    double before = 0.0;
    for (int c0 = 0; c0 < nchunks && cstar < 0; c0 += 32) {
        const int c = c0 + lane;
        const int nt = c < nchunks ? cties[c] : 0;
        const int tincl = warp_inclusive_scan(nt, lane);
        const double m = c < nchunks ? chunk_surv(ri, cmass, cties, c, tcarry + tincl - nt) : 0.0;
        const double incl = warp_scan_f64(m, lane);
        const unsigned hit = __ballot_sync(kFullMask, c < nchunks && m > 0.0 && carry + incl > target);
        if (hit) {
            const int src = __ffs(hit) - 1;
            cstar = c0 + src;
            tstar = tcarry + __shfl_sync(kFullMask, tincl - nt, src);
            before = carry + __shfl_sync(kFullMask, incl - m, src);
        }
        carry += __shfl_sync(kFullMask, incl, 31);
        tcarry += __shfl_sync(kFullMask, tincl, 31);
    }
    double tgt = target;
    if (cstar < 0) {  // rounding left no crossing: the answer is the row's last survivor
        for (int c = nchunks - 1; c >= 0; --c) {
            int tb = 0;
            for (int q = 0; q < c; ++q) tb += cties[q];
            if (chunk_surv(ri, cmass, cties, c, tb) > 0.0) {
                cstar = c;
                tstar = tb;
                break;
            }
        }
        if (cstar < 0) return -1;
        tgt = INFINITY;  // no element crosses: the scan below reports the chunk's last survivor
    }
    const double target2 = tgt;
    int found = -1, last = -1;
    double cum = before;
    scan_chunk<T>(row, a, ri, cstar, tstar, lane, [&](int64_t id0, const double* wv, int nv, int) {
        double s = 0.0;
        for (int e = 0; e < nv; ++e) s += wv[e];
        const double incl = warp_scan_f64(s, lane);
        if (found < 0) {
            const unsigned hit = __ballot_sync(kFullMask, s > 0.0 && cum + incl > target2);
            if (hit) {
                const int src = __ffs(hit) - 1;
                int tok = -1;
                if (lane == src) {
                    double cc = cum + incl - s;
                    for (int e = 0; e < nv; ++e) {
                        if (wv[e] <= 0.0) continue;
                        cc += wv[e];
                        tok = (int)(id0 + e);
                        if (cc > target2) break;
                    }
                }
                found = __shfl_sync(kFullMask, tok, src);
            }
            const unsigned pos = __ballot_sync(kFullMask, s > 0.0);
            if (pos) {
                const int src = 31 - __clz(pos);
                int tl = -1;
                if (lane == src)
                    for (int e = 0; e < nv; ++e)
                        if (wv[e] > 0.0) tl = (int)(id0 + e);
                last = __shfl_sync(kFullMask, tl, src);
            }
        }
        cum += __shfl_sync(kFullMask, incl, 31);
    });
    return found >= 0 ? found : last;
}

// probability of token t under the row's distribution (one warp)
template <typename T>
__device__ double warp_row_prob(const T* row, const VerifyArgs& a, const RowInfo& ri, const int* cties, int t,
                                int lane) {
    if (t < 0 || t >= a.V) return 0.0;
    constexpr int CH = Chunk<T>::CH;
    const int c = t / CH;
    int tb = 0;
    if (ri.tau != 0u) {
        for (int q = lane; q < c; q += 32) tb += cties[q];
        tb = warp_sum(tb);
    }
    double w = 0.0;
    scan_chunk<T>(row, a, ri, c, tb, lane, [&](int64_t id0, const double* wv, int nv, int) {
        if (t >= id0 && t < id0 + nv) w = wv[t - id0];
    });
    // the owning lane holds w; share it
    unsigned own = __ballot_sync(kFullMask, w != 0.0);
    if (own) w = __shfl_sync(kFullMask, w, __ffs(own) - 1);
    return w / ri.Z;
}

// ---------------------------------------------------------------------------------------
// CTA-level passes over a pair of rows: residual mass per chunk, or TV
// ---------------------------------------------------------------------------------------
template <typename T, typename F>
__device__ void pair_pass(const T* prow, const T* qrow, const VerifyArgs& a, const RowInfo& rp, const RowInfo& rq,
                          const int* ctp, const int* ctq, int nchunks, F per_chunk) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int c = warp; c < nchunks; c += kWarps) {
        int tbp = 0, tbq = 0;
        if (rp.tau != 0u || rq.tau != 0u) {
            for (int q = lane; q < c; q += 32) {
                tbp += ctp[q];
                tbq += ctq[q];
            }
            tbp = warp_sum(tbp);
            tbq = warp_sum(tbq);
        }
        double acc = 0.0;
        scan_pair_chunk<T>(prow, qrow, a, rp, rq, c, tbp, tbq, lane,
                           [&](int64_t, const double* wp, const double* wq, int nv) {
                               for (int e = 0; e < nv; ++e) acc += per_chunk(wp[e], wq[e]);
                           });
        acc = warp_sum_f64(acc);
        (void)acc;
    }
}

// ---------------------------------------------------------------------------------------
// the kernel: one CTA per sequence
// ---------------------------------------------------------------------------------------
// Row g = b * R + r of the work: verifier rows r < K, then drafter rows 1..K-1.
template <typename T>
__device__ __forceinline__ const T* work_row(const VerifyArgs& a, int R, int64_t g) {
    const int b = (int)(g / R), r = (int)(g % R);
    const bool isP = r < a.K;
    const int pos = isP ? r : r - a.K + 1;
    return reinterpret_cast<const T*>(isP ? a.P : a.Q) + ((int64_t)b * a.K + pos) * a.V;
}

// One CTA per row (every row of every sequence): the row's chunk table and RowInfo, the
// row read from global memory (HBM once, then L2) by every pass.
template <typename T>
__global__ void __launch_bounds__(kThreads) rows_kernel(Params p) {
    __shared__ RowShared sh;
    const int NC = p.nchunks;
    const int64_t g = blockIdx.x;
    int xe = 0;
    const GlobalRow<T> src{work_row<T>(p.a, p.rows_per_seq, g), p.a.V};
    prepare_row<T>(src, p.a, 0, NC, p.cmass + g * NC, p.cties + g * NC, p.infos + g, sh, CtaGroup{}, xe);
}

// Cluster form for bf16 rows whose length is a multiple of 8 (16-byte aligned rows): a
// cluster of CL CTAs owns one row at a time, CTA r holding chunks [r cpc, (r + 1) cpc) of
// it in shared memory, so the row is read from HBM exactly once and every pass runs from
// shared memory; the row-wide reductions go through distributed shared memory (ClusterGroup).
// Persistent: cluster i takes rows i, i + #clusters, ...; the next row's slice is copied in
// (one bulk copy per CTA, completion counted on an mbarrier) while this row is processed.
constexpr int kBulkAlign = 128;
inline size_t cluster_dyn_smem(int cpc) {
    return kBulkAlign + 2 * (size_t)cpc * Chunk<__nv_bfloat16>::CH * sizeof(uint16_t);
}

__global__ void __launch_bounds__(kThreads, 1) rows_cluster_kernel(Params p, int cpc) {
    extern __shared__ __align__(128) unsigned char dsm[];
    __shared__ RowShared sh;
    constexpr int CH = Chunk<__nv_bfloat16>::CH;
    const VerifyArgs& a = p.a;
    const int tid = threadIdx.x;
    const int rank = (int)cl_rank();
    const ClusterGroup grp{(int)cl_size()};
    uint64_t* full = reinterpret_cast<uint64_t*>(dsm);  // [2]: a buffer's slice has landed
    uint16_t* buf = reinterpret_cast<uint16_t*>(dsm + kBulkAlign);
    const int64_t buf_elems = (int64_t)cpc * CH;
    const int V = a.V, NC = p.nchunks, R = p.rows_per_seq;
    const int c0 = min(NC, rank * cpc), c1 = min(NC, c0 + cpc);
    const int64_t e_lo = min((int64_t)V, (int64_t)c0 * CH), e_hi = min((int64_t)V, (int64_t)c1 * CH);
    const uint32_t bytes = (uint32_t)((e_hi - e_lo) * 2);  // a multiple of 16; 0 without chunks
    const int64_t rows = (int64_t)a.B * R;
    const int64_t first = cl_index(), step = cl_count();
    uint32_t issued[2] = {0u, 0u}, done[2] = {0u, 0u};  // copies per buffer (thread 0)
    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    auto issue = [&](int64_t g, int bi) {
        ++issued[bi];
        if (bytes == 0) {
            mbar_arrive(&full[bi]);
            return;
        }
        mbar_arrive_expect_tx(&full[bi], bytes);
        bulk_g2s(buf + bi * buf_elems, work_row<__nv_bfloat16>(a, R, g) + e_lo, bytes, &full[bi]);
    };
    bool failed = false;
    if (tid == 0 && first < rows) issue(first, 0);
    int xe = 0;
    int it = 0;
    for (int64_t g = first; g < rows; g += step, ++it) {
        const int bi = it & 1;
        __syncthreads();  // every warp is done with the other buffer (the previous row)
        if (tid == 0 && !failed && g + step < rows) {
            fence_proxy_async_smem();
            issue(g + step, bi ^ 1);
        }
        if (!failed) {
            if (mbar_wait(&full[bi], (uint32_t)(it >> 1) & 1u)) {
                if (tid == 0) ++done[bi];
            } else {
                failed = true;
                record_device_status(p.status, UNO_ERR_TIMEOUT);
            }
        }
        // (after a timeout the CTA keeps taking part in the cluster's barriers; its results
        // are not valid, and the status word says so)
        const SharedSlice src{buf + bi * buf_elems, c0, V};
        prepare_row<__nv_bfloat16>(src, a, c0, c1, p.cmass + g * NC, p.cties + g * NC,
                                   rank == 0 ? p.infos + g : nullptr, sh, grp, xe);
    }
    // no CTA leaves while another may still read its exchange areas
    grp.sync();
    if (tid == 0)  // copies still in flight after a timeout: wait for them (bounded)
        for (int bi = 0; bi < 2; ++bi)
            while (done[bi] < issued[bi] && mbar_wait(&full[bi], done[bi] & 1u)) ++done[bi];
}

template <typename T>
__global__ void __launch_bounds__(kThreads) seq_kernel(Params p) {
    __shared__ double dred[kWarps];
    __shared__ int s_tok[32];
    __shared__ double s_p[32], s_q[32], s_tv[32];
    __shared__ int s_acc[32];
    const VerifyArgs& a = p.a;
    const int b = blockIdx.x, K = a.K, V = a.V, NC = p.nchunks;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int R = p.rows_per_seq;
    const int64_t rbase = (int64_t)b * R;
    auto rowp = [&](int r) -> const T* {
        const bool isP = r < K;
        const int pos = isP ? r : r - K + 1;
        return reinterpret_cast<const T*>(isP ? a.P : a.Q) + ((int64_t)b * K + pos) * V;
    };
    // the rows' tables come from rows_kernel (earlier on the stream)

    // per position: draws, probabilities, acceptance (warp per position)
    for (int i = warp; i < K; i += kWarps) {
        const RowInfo rp = p.infos[rbase + i];
        const double* cmp = p.cmass + (rbase + i) * NC;
        const int* ctp = p.cties + (rbase + i) * NC;
        const float* u = a.u + ((int64_t)b * K + i) * 3;
        int tok;
        double pi = 0.0, qi = 0.0;
        int acc = 1;
        if (i == 0) {
            tok = a.pos0 && a.pos0[b] >= 0 ? a.pos0[b]
                                           : warp_row_draw<T>(rowp(0), a, rp, cmp, ctp, NC, (double)u[0], lane);
            pi = warp_row_prob<T>(rowp(0), a, rp, ctp, tok, lane);
        } else {
            const int rq_i = K + i - 1;
            const RowInfo rq = p.infos[rbase + rq_i];
            const double* cmq = p.cmass + (rbase + rq_i) * NC;
            const int* ctq = p.cties + (rbase + rq_i) * NC;
            tok = a.drafts ? a.drafts[(int64_t)b * K + i] : warp_row_draw<T>(rowp(rq_i), a, rq, cmq, ctq, NC, (double)u[0], lane);
            pi = warp_row_prob<T>(rowp(i), a, rp, ctp, tok, lane);
            qi = warp_row_prob<T>(rowp(rq_i), a, rq, ctq, tok, lane);
            acc = (double)u[1] * qi < pi;
        }
        if (lane == 0) {
            s_tok[i] = tok;
            s_p[i] = pi;
            s_q[i] = qi;
            s_acc[i] = acc;
            s_tv[i] = 0.0;
        }
    }
    __syncthreads();
    int n = K;
    for (int i = 1; i < K; ++i)
        if (!s_acc[i]) {
            n = i;
            break;
        }

    // optional TV per position (i >= 1): 1/2 sum |p - q| over the whole vocabulary
    if (a.out_tv) {
        for (int i = 1; i < K; ++i) {
            const int rq_i = K + i - 1;
            double part = 0.0;
            const RowInfo rp = p.infos[rbase + i], rq = p.infos[rbase + rq_i];
            const int* ctp = p.cties + (rbase + i) * NC;
            const int* ctq = p.cties + (rbase + rq_i) * NC;
            pair_pass<T>(rowp(i), rowp(rq_i), a, rp, rq, ctp, ctq, NC, [&](double pv, double qv) {
                part += fabs(pv - qv);
                return 0.0;
            });
            const double tv = 0.5 * cta_sum_f64(part, dred);
            if (threadIdx.x == 0) s_tv[i] = tv;
            __syncthreads();
        }
    }

    // the correction token: residual max(0, p_n - q_n) (whole CTA for the per-chunk table)
    int nxt = -1;
    if (n < K) {
        const int rq_n = K + n - 1;
        const RowInfo rp = p.infos[rbase + n], rq = p.infos[rbase + rq_n];
        const double* cmp = p.cmass + (rbase + n) * NC;
        const int* ctp = p.cties + (rbase + n) * NC;
        const int* ctq = p.cties + (rbase + rq_n) * NC;
        double* cres = p.cres + (int64_t)b * NC;
        const T* prow = rowp(n);
        const T* qrow = rowp(rq_n);
        // residual mass per chunk (warp per chunk)
        for (int c = warp; c < NC; c += kWarps) {
            int tbp = 0, tbq = 0;
            for (int q = lane; q < c; q += 32) {
                tbp += ctp[q];
                tbq += ctq[q];
            }
            tbp = warp_sum(tbp);
            tbq = warp_sum(tbq);
            double acc = 0.0;
            scan_pair_chunk<T>(prow, qrow, a, rp, rq, c, tbp, tbq, lane,
                               [&](int64_t, const double* wp, const double* wq, int nv) {
                                   for (int e = 0; e < nv; ++e) {
                                       const double d = wp[e] - wq[e];
                                       acc += d > 0.0 ? d : 0.0;
                                   }
                               });
            acc = warp_sum_f64(acc);
            if (lane == 0) cres[c] = acc;
        }
        __syncthreads();
        if (warp == 0) {
            const double uu = (double)a.u[((int64_t)b * K + n) * 3 + 2];
            double Rtot = 0.0;
            for (int c = lane; c < NC; c += 32) Rtot += cres[c];
            Rtot = warp_sum_f64(Rtot);
            if (!(Rtot > 0.0)) {
                nxt = warp_row_draw<T>(prow, a, rp, cmp, ctp, NC, uu, lane);
            } else {
                // walk the residual table, then scan the crossing chunk
                const double target = uu * Rtot;
                double carry = 0.0, before = 0.0;
                int cstar = -1;
                for (int c0 = 0; c0 < NC && cstar < 0; c0 += 32) {
                    const int c = c0 + lane;
                    const double m = c < NC ? cres[c] : 0.0;
                    const double incl = warp_scan_f64(m, lane);
                    const unsigned hit = __ballot_sync(kFullMask, c < NC && m > 0.0 && carry + incl > target);
                    if (hit) {
                        const int src = __ffs(hit) - 1;
                        cstar = c0 + src;
                        before = carry + __shfl_sync(kFullMask, incl - m, src);
                    }
                    carry += __shfl_sync(kFullMask, incl, 31);
                }
                if (cstar < 0)
                    for (int c = NC - 1; c >= 0 && cstar < 0; --c)
                        if (cres[c] > 0.0) {
                            cstar = c;
                            before = target;
                        }
                int tbp = 0, tbq = 0;
                for (int q = lane; q < cstar; q += 32) {
                    tbp += ctp[q];
                    tbq += ctq[q];
                }
                tbp = warp_sum(tbp);
                tbq = warp_sum(tbq);
                int found = -1, last = -1;
                double cum = before;
                scan_pair_chunk<T>(prow, qrow, a, rp, rq, cstar, tbp, tbq, lane,
                                   [&](int64_t id0, const double* wp, const double* wq, int nv) {
                    double r[Elem<T>::VEC];
                    double s = 0.0;
                    for (int e = 0; e < Elem<T>::VEC; ++e) {
                        const double d = e < nv ? wp[e] - wq[e] : 0.0;
                        r[e] = d > 0.0 ? d : 0.0;
                        s += r[e];
                    }
                    const double incl = warp_scan_f64(s, lane);
                    if (found < 0) {
                        const unsigned hit = __ballot_sync(kFullMask, s > 0.0 && cum + incl > target);
                        if (hit) {
                            const int src = __ffs(hit) - 1;
                            int tk = -1;
                            if (lane == src) {
                                double cc = cum + incl - s;
                                for (int e = 0; e < nv; ++e) {
                                    if (r[e] <= 0.0) continue;
                                    cc += r[e];
                                    tk = (int)(id0 + e);
                                    if (cc > target) break;
                                }
                            }
                            found = __shfl_sync(kFullMask, tk, src);
                        }
                        const unsigned pos = __ballot_sync(kFullMask, s > 0.0);
                        if (pos) {
                            const int src = 31 - __clz(pos);
                            int tl = -1;
                            if (lane == src)
                                for (int e = 0; e < nv; ++e)
                                    if (r[e] > 0.0) tl = (int)(id0 + e);
                            last = __shfl_sync(kFullMask, tl, src);
                        }
                    }
                    cum += __shfl_sync(kFullMask, incl, 31);
                });
                nxt = found >= 0 ? found : last;
            }
        }
    }

    if (warp == 0) {
        const int i = lane;
        if (i < K) {
            const int64_t o = (int64_t)b * K + i;
            a.out_tokens[o] = i < n ? s_tok[i] : -1;
            if (a.out_p) a.out_p[o] = (float)s_p[i];
            if (a.out_q) a.out_q[o] = (float)s_q[i];
            if (a.out_tv) a.out_tv[o] = (float)s_tv[i];
        }
        if (lane == 0) {
            a.out_count[b] = n;
            if (a.out_next) a.out_next[b] = n < K ? nxt : -1;
        }
    }
}

struct Layout {
    int nchunks, rows_per_seq;
    size_t off_cmass, off_cties, off_cres, off_infos, total;
};

inline Layout layout(const VerifyArgs& a) {
    Layout L{};
    const int CH = a.dtype == UNO_BF16 ? Chunk<__nv_bfloat16>::CH : Chunk<float>::CH;
    L.nchunks = (a.V + CH - 1) / CH;
    L.rows_per_seq = 2 * a.K - 1;
    const size_t rows = (size_t)a.B * L.rows_per_seq;
    L.off_cmass = 0;
    L.off_cties = align_up(rows * L.nchunks * 8, 256);
    L.off_cres = align_up(L.off_cties + rows * L.nchunks * 4, 256);
    L.off_infos = align_up(L.off_cres + (size_t)a.B * L.nchunks * 8, 256);
    L.total = align_up(L.off_infos + rows * sizeof(RowInfo), 256);
    return L;
}

// Cluster size for the rows: UNO_VERIFY_FULL_CLUSTER (1, 2, 4, 8 or 16) if set, else the
// smallest size whose two slice buffers fit in shared memory next to RowShared.
inline bool cluster_fits(int nchunks, int c, size_t room) {
    const int cpc = (nchunks + c - 1) / c;
    return cpc * kVecPerLane <= kMaxUnits && cluster_dyn_smem(cpc) <= room;
}
inline int choose_cluster(int nchunks, size_t room) {
    if (const char* e = getenv("UNO_VERIFY_FULL_CLUSTER")) {
        const int c = atoi(e);
        if (c == 1 || c == 2 || c == 4 || c == 8 || c == 16) return cluster_fits(nchunks, c, room) ? c : 0;
    }
    for (int c = 1; c <= 16; c *= 2)
        if (cluster_fits(nchunks, c, room)) return c;
    return 0;
}

struct ClusterDevice {
    bool ready = false;
    size_t dyn_max = 0;  // dynamic shared memory a CTA may use beside the kernel's static part
    std::map<std::pair<int, size_t>, int> max_clusters;  // (cluster size, dynamic smem) -> co-resident clusters
};
std::mutex g_cluster_mu;
ClusterDevice g_cluster_dev[64];

// Launch rows_cluster_kernel when it applies (bf16, V a multiple of 8, 16-byte aligned
// logits, a cluster that fits) and UNO_VERIFY_FULL is not "rows"; returns false to fall back
// to the per-row kernel. UNO_VERIFY_FULL=cluster makes a case that cannot take the cluster
// form an error (UNO_ERR_UNSUPPORTED) instead of a fallback.
bool launch_rows_cluster(const Params& p, cudaStream_t stream, uno_status& st) {
    const VerifyArgs& a = p.a;
    const char* mode = getenv("UNO_VERIFY_FULL");
    if (mode && strcmp(mode, "rows") == 0) return false;
    const bool required = mode && strcmp(mode, "cluster") == 0;
    auto no = [&](const char* why) {
        if (required) st = set_error(UNO_ERR_UNSUPPORTED, "verify (full vocabulary): no cluster form: %s", why);
        return required;
    };
    if (a.dtype != UNO_BF16 || a.V % 8 != 0) return no("bf16 rows whose length is a multiple of 8 only");
    if ((reinterpret_cast<uintptr_t>(a.P) | reinterpret_cast<uintptr_t>(a.Q)) & 15u)
        return no("logits must be 16-byte aligned");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return no("no current device");
    std::lock_guard<std::mutex> lock(g_cluster_mu);
    ClusterDevice& di = g_cluster_dev[dev];
    if (!di.ready) {
        int optin = 0;
        cudaFuncAttributes fa{};
        if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaFuncGetAttributes(&fa, rows_cluster_kernel) != cudaSuccess || optin <= (int)fa.sharedSizeBytes) {
            cudaGetLastError();
            return no("shared memory attributes unavailable");
        }
        const int dyn_max = optin - (int)fa.sharedSizeBytes;
        if (cudaFuncSetAttribute(rows_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max) !=
                cudaSuccess ||
            cudaFuncSetAttribute(rows_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess) {
            cudaGetLastError();
            return no("kernel attributes refused");
        }
        di.dyn_max = (size_t)dyn_max;
        di.ready = true;
    }
    const int c = choose_cluster(p.nchunks, di.dyn_max);
    if (c == 0) return no("the row slices do not fit in the shared memory of this cluster size");
    const int cpc = (p.nchunks + c - 1) / c;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = cluster_dyn_smem(cpc);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const auto key = std::make_pair(c, cfg.dynamicSmemBytes);
    int maxc = 0;
    const auto found = di.max_clusters.find(key);
    if (found != di.max_clusters.end()) {
        maxc = found->second;
    } else {
        cudaLaunchConfig_t q = cfg;
        q.gridDim = dim3((unsigned)c);
        if (cudaOccupancyMaxActiveClusters(&maxc, rows_cluster_kernel, &q) != cudaSuccess) {
            cudaGetLastError();
            maxc = 0;
        }
        di.max_clusters[key] = maxc;
    }
    if (maxc <= 0) return no("no cluster of this size can be resident");
    const int64_t rows = (int64_t)a.B * p.rows_per_seq;
    const int64_t clusters = std::min<int64_t>(rows, (int64_t)maxc);
    cfg.gridDim = dim3((unsigned)(clusters * c));
    st = check_cuda(cudaLaunchKernelEx(&cfg, rows_cluster_kernel, p, cpc), "launch(verify full rows, cluster)");
    return true;
}

}  // namespace vfull

size_t verify_full_workspace_bytes(const VerifyArgs& a) { return vfull::layout(a).total; }

uno_status verify_full_launch(const VerifyArgs& a, void* workspace, cudaStream_t stream) {
    const vfull::Layout L = vfull::layout(a);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    vfull::Params p{};
    p.a = a;
    p.rows_per_seq = L.rows_per_seq;
    p.nchunks = L.nchunks;
    p.cmass = reinterpret_cast<double*>(ws + L.off_cmass);
    p.cties = reinterpret_cast<int*>(ws + L.off_cties);
    p.cres = reinterpret_cast<double*>(ws + L.off_cres);
    p.infos = reinterpret_cast<vfull::RowInfo*>(ws + L.off_infos);
    p.status = device_status_ptr();
    const unsigned rows = (unsigned)((int64_t)a.B * L.rows_per_seq);
    if (a.dtype == UNO_BF16) {
        uno_status st = UNO_OK;
        if (!vfull::launch_rows_cluster(p, stream, st))
            vfull::rows_kernel<__nv_bfloat16><<<rows, vfull::kThreads, 0, stream>>>(p);
        else if (st != UNO_OK)
            return st;
        vfull::seq_kernel<__nv_bfloat16><<<(unsigned)a.B, vfull::kThreads, 0, stream>>>(p);
    } else {
        vfull::rows_kernel<float><<<rows, vfull::kThreads, 0, stream>>>(p);
        vfull::seq_kernel<float><<<(unsigned)a.B, vfull::kThreads, 0, stream>>>(p);
    }
    return check_cuda(cudaGetLastError(), "launch(verify full)");
}

}  // namespace uno
