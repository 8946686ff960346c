// verify_topk.cu — lossless block verify with top-k on (optionally followed by top-p).
//
// Lossless verification of a drafted block: LoopUno project page, "How it works" (the
// unmodified model verifies the block, keeps the longest correct prefix, position 0 is the
// exact AR token) and "Training is self-distillation" (acceptance probability 1 - TV);
// sampler settings from the uno-qwen3-8B model card, "Evaluation protocol" (temperature
// 1.0, top-k 50, top-p 0.95, block 16).
//
// Two launches, neither of which waits on another CTA:
//   1. stream: the logit rows (verifier rows 0..K-1 and drafter rows 1..K-1 of every
//      sequence) are read once with 16-byte coalesced loads; every warp keeps the exact
//      top-k of its own run of the row (among the elements at or above a sampled guess)
//      and writes it out. bf16 rows that are 16-byte aligned take the persistent row
//      kernel; the rest one CTA per row segment (or the TMA-fed variant);
//   2. finish: CTAs of 16 warps, a warp per row, merge each row's lists into its exact
//      top-k (redoing the row when the guess could have hidden part of it), apply softmax
//      and top-p in fp64 and store the survivors sorted by token id; the CTA that completes
//      a sequence's rows (per-sequence counters) then runs its draft sampling, acceptance,
//      longest accepted prefix and residual resample, one warp per block position.
#include <cuda_bf16.h>

#include <cstdlib>
#include <cstring>
#include <type_traits>
#include <algorithm>

#include "select.cuh"
#include "verify_common.cuh"

namespace uno {
namespace vtopk {

constexpr int kUnroll = 4;
constexpr int kStreamWarps = 8;  // warps per CTA of the streaming kernel
constexpr int kGuessPerWarp = 8; // sample maxima each warp contributes to the guess

template <int KCAP>
constexpr int cap_entries() { return KCAP + 576; }


struct Params {
    VerifyArgs a;
    int S;               // segments per row (one streaming CTA each)
    int rows_per_seq;    // 2K - 1
    int lists_per_row;   // S * kStreamWarps
    uint64_t* lists;     // [rows * lists_per_row][kcap]
    int32_t* counts;     // [rows * lists_per_row]
    uint32_t* guesses;   // [rows * lists_per_row] ordered key of the guess each list was taken with
    unsigned char* recs;
    int kcap;
    unsigned long long* trace;  // UNO_VERIFY_TRACE: phase timestamps of the finish (profiling aid), or NULL
    uint32_t* seq_done;         // [B] rows finished per sequence (zeroed by the streaming kernel)
};

// Zero the per-sequence counters of the finish kernel (CTA 0 of the streaming kernel, which
// runs before it in the stream).
__device__ __forceinline__ void zero_seq_counters(const Params& p) {
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < p.a.B; i += blockDim.x) p.seq_done[i] = 0u;
}

// finish kernel, CTA 0: slot (warp, event)
__device__ __forceinline__ void fin_mark(const Params& p, int warp, int e) {
    if (p.trace != nullptr && blockIdx.x == 0 && (threadIdx.x & 31) == 0) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        p.trace[warp * 8 + e] = t;
    }
}

template <typename T>
struct KeyBits;
template <>
struct KeyBits<__nv_bfloat16> { static constexpr int value = 16; };
template <>
struct KeyBits<float> { static constexpr int value = 32; };

// Descending bitonic sort of one 32-bit key per lane across the warp.
__device__ __forceinline__ uint32_t warp_sort32_desc(uint32_t v, int lane) {
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            uint32_t o = __shfl_xor_sync(kFullMask, v, stride);
            bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0);
            v = keep_max ? max(v, o) : min(v, o);
        }
    }
    return v;
}

// Packed lane-chunk tests. hit(): does any element x satisfy x >= lo and x > thr?
// mask(): which elements do (bit j = element j), for the nvalid first elements.
template <typename T>
struct LaneOps;

template <>
struct LaneOps<__nv_bfloat16> {
    using Thr = __nv_bfloat162;
    __device__ static __forceinline__ Thr thr(float f) { return __float2bfloat162_rn(f); }  // f is a bf16 value
    __device__ static __forceinline__ __nv_bfloat162 w2(uint32_t w) { return *reinterpret_cast<__nv_bfloat162*>(&w); }
    __device__ static __forceinline__ bool hit(const uint4& v, Thr lo, Thr th) {
        __nv_bfloat162 m = __hmax2(__hmax2(w2(v.x), w2(v.y)), __hmax2(w2(v.z), w2(v.w)));
        return (__hge2_mask(m, lo) & __hgt2_mask(m, th)) != 0u;
    }
    __device__ static __forceinline__ uint32_t mask(const uint4& v, int nvalid, Thr lo, Thr th) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t m = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t t = __hge2_mask(w2(w[q]), lo) & __hgt2_mask(w2(w[q]), th);
            m |= ((t & 1u) << (2 * q)) | (((t >> 16) & 1u) << (2 * q + 1));
        }
        return nvalid >= 8 ? m : (m & ((1u << nvalid) - 1u));
    }
};

template <>
struct LaneOps<float> {
    using Thr = float;
    __device__ static __forceinline__ Thr thr(float f) { return f; }
    __device__ static __forceinline__ bool hit(const uint4& v, Thr lo, Thr th) {
        float m = raw_max<float>(v);
        return m >= lo && m > th;
    }
    __device__ static __forceinline__ uint32_t mask(const uint4& v, int nvalid, Thr lo, Thr th) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t m = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float x = __uint_as_float(w[q]);
            m |= (uint32_t)(q < nvalid && x >= lo && x > th) << q;
        }
        return m;
    }
};

// Per-warp candidate state, in shared memory so that the rare out-of-line paths can
// update it. The buffer is always in ascending token-id order.
struct WarpSlot {
    int count;
    int have_k;
    float thr;  // the buffer's k-th value once it has been cut to k (-inf before)
};

template <int KB>
__device__ __noinline__ void warp_shrink(uint64_t* buf, uint32_t* hist, WarpSlot* ws, uint32_t* bound, int k,
                                         int lane) {
    uint32_t tau;
    int need;
    warp_select_key<KB>(buf, ws->count, k, hist, lane, tau, need);
    const int n = warp_compact_key<KB>(buf, ws->count, tau, need, lane);
    const uint32_t key = key32_of_radix<KB>(tau);
    __syncwarp();
    if (lane == 0) {
        ws->count = n;
        ws->have_k = 1;
        ws->thr = key_float(key);
        atomicMax(bound, key);
    }
    __syncwarp();
}

// Cut an unordered buffer to its exact top-k by the packed (value desc, id asc) order.
__device__ __noinline__ void warp_shrink_packed(uint64_t* buf, uint32_t* hist, WarpSlot* ws, int k, int lane) {
    const int n0 = ws->count;
    const uint64_t T = warp_select(buf, n0, k, hist, lane);
    uint64_t mn;
    const int n = warp_compact(buf, n0, T, lane, &mn);
    __syncwarp();
    if (lane == 0) {
        ws->count = n;
        ws->have_k = 1;
        ws->thr = key_float(candidate_key(mn));
    }
    __syncwarp();
}

// Lane-local append (no warp collectives): the lane's elements of chunk v that pass
// x >= lo and x > th go to the warp's unordered buffer through a shared-memory atomic.
template <typename T>
__device__ __forceinline__ void lane_append(const uint4& v, int nvalid, uint32_t id0, typename LaneOps<T>::Thr lo,
                                            typename LaneOps<T>::Thr th, uint64_t* buf, WarpSlot* ws) {
    uint32_t m = LaneOps<T>::mask(v, nvalid, lo, th);
    int pos = atomicAdd(&ws->count, __popc(m));
    while (m) {
        const int j = __ffs(m) - 1;
        buf[pos++] = pack_candidate(float_key(raw_get<T>(v, j)), id0 + (uint32_t)j);
        m &= m - 1u;
    }
}

// Append the elements of this lane's chunk that pass the current bounds (every lane of
// the warp calls it; lanes with nothing to add pass through).
template <typename T, int CAP>
__device__ __noinline__ void warp_append(const uint4 v, int nvalid, uint32_t id0, uint64_t* buf, uint32_t* hist,
                                         WarpSlot* ws, uint32_t* bound, float guess, int k, int lane) {
    using Ops = LaneOps<T>;
    constexpr int VEC = Elem<T>::VEC;
    const float lo = fmaxf(guess, key_float(*reinterpret_cast<volatile uint32_t*>(bound)));
    const float th = ws->have_k ? ws->thr : -INFINITY;
    uint32_t m = nvalid > 0 ? Ops::mask(v, nvalid, Ops::thr(lo), Ops::thr(th)) : 0u;
    const int c = __popc(m);
    const int incl = warp_inclusive_scan(c, lane);
    const int total = __shfl_sync(kFullMask, incl, 31);
    int pos = ws->count + incl - c;
    while (m) {
        const int j = __ffs(m) - 1;
        buf[pos++] = pack_candidate(float_key(raw_get<T>(v, j)), id0 + (uint32_t)j);
        m &= m - 1u;
    }
    __syncwarp();
    if (lane == 0) ws->count += total;
    __syncwarp();
    if (ws->count > CAP - 32 * VEC) warp_shrink<KeyBits<T>::value>(buf, hist, ws, bound, k, lane);
}

// One chunk of the bulk loop: lanes whose part of the chunk passes the bounds append
// their candidates (every lane of the warp calls it; the buffer is cut first when it may
// not have room for the whole chunk).
template <int CAP>
__device__ __forceinline__ void handle_chunk(const uint4 v, uint32_t id0, uint64_t* buf, uint32_t* hist, WarpSlot* ws,
                                             uint32_t* bound, const float* guess, int k, int lane,
                                             __nv_bfloat162& lo, __nv_bfloat162& th) {
    using Ops = LaneOps<__nv_bfloat16>;
    bool h = Ops::hit(v, lo, th);
    if (!__any_sync(kFullMask, h)) return;
    if (ws->count > CAP - 256) {  // room for a whole chunk (uniform)
        warp_shrink<16>(buf, hist, ws, bound, k, lane);
        lo = Ops::thr(fmaxf(*guess, key_float(*reinterpret_cast<volatile uint32_t*>(bound))));
        th = Ops::thr(ws->have_k ? ws->thr : -INFINITY);
        h = Ops::hit(v, lo, th);
    }
    if (h) lane_append<__nv_bfloat16>(v, 8, id0, lo, th, buf, ws);
    __syncwarp();
}

// The bulk of a warp's run over an aligned bf16 row: full chunks [cb, cf) (at least two
// groups of kUnroll), 16-byte loads two groups ahead, one test of each lane's maximum per
// group, lane-local appends for the rare lanes that hold a candidate. The thresholds are
// kept in registers and refreshed after appends (a stale, lower threshold only admits
// more candidates). Returns the first chunk not processed.
template <int CAP>
__device__ __noinline__ int stream_full_bf16(const uint4* lp, int cb, int cf, uint64_t* buf, uint32_t* hist,
                                             WarpSlot* ws, uint32_t* bound, const float* guess, int k, int lane) {
    using Ops = LaneOps<__nv_bfloat16>;
    constexpr int CH = 256;  // elements per warp chunk
    const volatile uint32_t* vb = bound;
    __nv_bfloat162 lo = Ops::thr(fmaxf(*guess, key_float(*vb))), th = Ops::thr(ws->have_k ? ws->thr : -INFINITY);
    uint4 a0 = ld_stream_v4(lp), a1 = ld_stream_v4(lp + 32), a2 = ld_stream_v4(lp + 64), a3 = ld_stream_v4(lp + 96);
    for (; cb + kUnroll <= cf; cb += kUnroll) {
        const bool more = cb + 2 * kUnroll <= cf;
        uint4 b0, b1, b2, b3;
        if (more) {
            b0 = ld_stream_v4(lp + 128);
            b1 = ld_stream_v4(lp + 160);
            b2 = ld_stream_v4(lp + 192);
            b3 = ld_stream_v4(lp + 224);
        }
        const __nv_bfloat162 m01 = __hmax2(__hmax2(__hmax2(Ops::w2(a0.x), Ops::w2(a0.y)), __hmax2(Ops::w2(a0.z), Ops::w2(a0.w))),
                                           __hmax2(__hmax2(Ops::w2(a1.x), Ops::w2(a1.y)), __hmax2(Ops::w2(a1.z), Ops::w2(a1.w))));
        const __nv_bfloat162 m23 = __hmax2(__hmax2(__hmax2(Ops::w2(a2.x), Ops::w2(a2.y)), __hmax2(Ops::w2(a2.z), Ops::w2(a2.w))),
                                           __hmax2(__hmax2(Ops::w2(a3.x), Ops::w2(a3.y)), __hmax2(Ops::w2(a3.z), Ops::w2(a3.w))));
        const __nv_bfloat162 mall = __hmax2(m01, m23);
        if (__any_sync(kFullMask, (__hge2_mask(mall, lo) & __hgt2_mask(mall, th)) != 0u)) {
            handle_chunk<CAP>(a0, (uint32_t)(cb * CH + lane * 8), buf, hist, ws, bound, guess, k, lane, lo, th);
            handle_chunk<CAP>(a1, (uint32_t)((cb + 1) * CH + lane * 8), buf, hist, ws, bound, guess, k, lane, lo, th);
            handle_chunk<CAP>(a2, (uint32_t)((cb + 2) * CH + lane * 8), buf, hist, ws, bound, guess, k, lane, lo, th);
            handle_chunk<CAP>(a3, (uint32_t)((cb + 3) * CH + lane * 8), buf, hist, ws, bound, guess, k, lane, lo, th);
            // another warp's cut may have raised the shared bound
            lo = Ops::thr(fmaxf(*guess, key_float(*vb)));
        }
        if (!more) {
            cb += kUnroll;
            break;
        }
        a0 = b0;
        a1 = b1;
        a2 = b2;
        a3 = b3;
        lp += 128;
    }
    return cb;
}

// ---------------------------------------------------------------------------------------
// Kernel 1: stream the logit rows once. Every warp walks its own contiguous run of chunks
// in token-id order and keeps the run's exact top-k (ties to the lower id). Warps share
// only a lower bound on the segment's k-th value (any warp's k-th value is one), used as
// a non-strict filter; they never wait for one another.
//   - first bound: the k-th largest of the warp's first 32 * kUnroll lane-chunk maxima
//     (distinct elements, so at least k elements are >= it);
//   - once a warp's buffer has been cut to its exact top-k, later (higher id) elements
//     are appended only when strictly above its k-th value.
// ---------------------------------------------------------------------------------------
template <typename T, int KCAP>
__global__ void __launch_bounds__(kStreamWarps * 32, 3)
stream_kernel(Params p) {
    zero_seq_counters(p);
    using Ops = LaneOps<T>;
    constexpr int VEC = Elem<T>::VEC;
    constexpr int CAP = cap_entries<KCAP>();
    constexpr int CH = 32 * VEC;  // elements per warp step (one chunk)
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint64_t* wbuf = reinterpret_cast<uint64_t*>(smem_raw);
    uint32_t* whist = reinterpret_cast<uint32_t*>(wbuf + kStreamWarps * CAP);
    __shared__ uint32_t s_bound;
    __shared__ float s_guess;
    __shared__ WarpSlot s_slot[kStreamWarps];
    __shared__ uint64_t s_top[kStreamWarps * kGuessPerWarp];
    __shared__ int s_nsample[kStreamWarps];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const VerifyArgs& a = p.a;
    const int S = p.S, k = a.top_k, V = a.V;
    const int grow = blockIdx.x / S, seg = blockIdx.x % S;
    const int b = grow / p.rows_per_seq, r = grow % p.rows_per_seq;
    const bool isP = r < a.K;
    const int pos = isP ? r : r - a.K + 1;
    const T* row = reinterpret_cast<const T*>(isP ? a.P : a.Q) + ((int64_t)b * a.K + pos) * V;
    const bool aligned = ((reinterpret_cast<uintptr_t>(row) & 15u) == 0);

    const int nchunks = (V + CH - 1) / CH;
    const int full_chunks = aligned ? V / CH : 0;  // chunks read with plain 16-byte loads
    const int sc0 = (int)((int64_t)nchunks * seg / S), sc1 = (int)((int64_t)nchunks * (seg + 1) / S);
    const int c0 = sc0 + (int)((int64_t)(sc1 - sc0) * warp / kStreamWarps);
    const int c1 = sc0 + (int)((int64_t)(sc1 - sc0) * (warp + 1) / kStreamWarps);

    uint64_t* buf = wbuf + warp * CAP;
    uint32_t* hist = whist + warp * 256;
    WarpSlot* ws = &s_slot[warp];
    if (threadIdx.x == 0) {
        s_bound = 0x007FFFFFu;  // ordered key of -inf
        s_guess = -INFINITY;
    }
    if (lane == 0) {
        ws->count = 0;
        ws->have_k = 0;
        ws->thr = -INFINITY;
    }
    __syncthreads();
    volatile uint32_t* vbound = &s_bound;

    uint4 raw[kUnroll];
    int nv[kUnroll];
    auto load = [&](int cb) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int c = cb + u;
            const int64_t e0 = (int64_t)c * CH + lane * VEC;
            if (c < full_chunks && c < c1) {
                nv[u] = VEC;
                raw[u] = ld_stream_v4(row + e0);
            } else {
                nv[u] = (c < c1) ? (int)max((int64_t)0, min((int64_t)VEC, (int64_t)V - e0)) : 0;
                raw[u] = nv[u] > 0 ? load_raw<T>(row, e0, nv[u], aligned) : make_uint4(0, 0, 0, 0);
            }
        }
    };
    auto offer = [&](int cb) {
        const typename Ops::Thr lo = Ops::thr(fmaxf(s_guess, key_float(*vbound)));
        const typename Ops::Thr th = Ops::thr(ws->have_k ? ws->thr : -INFINITY);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const bool hit = nv[u] > 0 && Ops::hit(raw[u], lo, th);
            if (__any_sync(kFullMask, hit))
                warp_append<T, CAP>(raw[u], hit ? nv[u] : 0, (uint32_t)((cb + u) * CH + lane * VEC), buf, hist, ws,
                                    &s_bound, s_guess, k, lane);
        }
    };

    // ---- prologue (every warp, also those with an empty run) ----
    load(c0);
    {
        // Sample of the segment: the lane-chunk maxima of every warp's first loads
        // (key 0 = no element). (a) The k-th largest of a warp's maxima is a lower bound on
        // the k-th value (they are distinct elements): shared in s_bound. (b) A guess tau_g
        // from the CTA's whole sample, expected to leave about 3.7k candidates in the row;
        // rows that end with fewer than k candidates are redone exactly by the finish
        // kernel, so the guess never changes the result.
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            buf[u * 32 + lane] =
                ((uint64_t)(nv[u] > 0 ? float_key(raw_max<T>(raw[u])) : 0u) << 32) | (uint32_t)(u * 32 + lane);
        __syncwarp();
        warp_sort_desc(buf, 32 * kUnroll, lane);
        if (k <= 32 * kUnroll) {
            const uint32_t key = (uint32_t)(buf[k - 1] >> 32);
            if (lane == 0) atomicMax(&s_bound, key < 0x007FFFFFu ? 0x007FFFFFu : key);
        }
        if (lane < kGuessPerWarp) s_top[warp * kGuessPerWarp + lane] = buf[lane] | ((uint64_t)warp << 16);
        int nvalid = 0;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) nvalid += nv[u];
        nvalid = warp_sum(nvalid);
        if (lane == 0) s_nsample[warp] = nvalid;
        __syncthreads();
        if (warp == 0) {
            int ns = 0;
            for (int w = 0; w < kStreamWarps; ++w) ns += s_nsample[w];
            uint64_t* tb = buf;  // warp 0's buffer is still free
            for (int j = lane; j < kStreamWarps * kGuessPerWarp; j += 32) tb[j] = s_top[j];
            __syncwarp();
            warp_sort_desc(tb, kStreamWarps * kGuessPerWarp, lane);
            // expected number of sample elements among the row's top-k: k * ns / V
            const int m = (int)(3.0 * k * (double)ns / (double)V) + 2;
            uint32_t g = 0u;
            if (m <= kStreamWarps * kGuessPerWarp && ns < V) g = (uint32_t)(tb[m - 1] >> 32);
            if (lane == 0) s_guess = key_float(g < 0x007FFFFFu ? 0x007FFFFFu : g);
            __syncwarp();
        }
        __syncthreads();
    }
    offer(c0);

    // ---- stream the rest of the warp's run ----
    int cb = c0 + kUnroll;
    if constexpr (VEC == 8) {
        const int cf = max(cb, min(c1, full_chunks));
        if (cb + 2 * kUnroll <= cf)
            cb = stream_full_bf16<CAP>(reinterpret_cast<const uint4*>(row) + (int64_t)cb * 32 + lane, cb, cf, buf,
                                       hist, ws, &s_bound, &s_guess, k, lane);
    }
    for (; cb < c1; cb += kUnroll) {
        load(cb);
        offer(cb);
    }
    if (ws->count > k) warp_shrink<KeyBits<T>::value>(buf, hist, ws, &s_bound, k, lane);

    const int64_t list = ((int64_t)grow * S + seg) * kStreamWarps + warp;
    uint64_t* out = p.lists + list * KCAP;
    const int cnt = ws->count;
    for (int j = lane; j < cnt; j += 32) out[j] = buf[j];
    if (lane == 0) {
        p.counts[list] = cnt;
        p.guesses[list] = float_key(s_guess);
    }
}

// ---------------------------------------------------------------------------------------
// Kernel 2: one warp per row. Merge the row's lists into its exact top-k, softmax in
// fp64, top-p, and write the survivor record sorted by token id.
// ---------------------------------------------------------------------------------------
// ---------------------------------------------------------------------------------------
// Kernel 1 (rows whose start is 16-byte aligned): persistent, fed by TMA.
// One CTA per SM; its warps take the grid's work items (row segments) in turn and each
// warp keeps the exact top-k of its run of every item (its 1/kTmaWarps share of the
// segment) among the elements >= its own guess g (see below). Each warp owns a ring of
// kStages shared-memory stages filled by bulk async copies that one lane issues ahead
// without regard to item boundaries, so the next item's data is already arriving while
// the current one finishes. An mbarrier per stage counts the arriving bytes. Warps never
// wait for one another. Every wait is bounded: on timeout the warp records
// UNO_ERR_TIMEOUT in the device status word, waits (bounded) for its copies still in
// flight, and stops.
// The guess g: from the first stage of its run the warp takes the maxima of its 32 lanes
// and sets g to the m-th largest, m chosen so that g is very unlikely to exceed the row's
// k-th value. The row's result is exact whenever its k-th value is >= every
// warp's g (then every element that can be in the top-k was a candidate); the finish
// kernel checks that and otherwise redoes the row exactly.
// ---------------------------------------------------------------------------------------
constexpr int kTmaWarps = 4;       // warps per CTA; several CTAs share an SM
constexpr int kTmaCtasPerSm = 4;
constexpr int kStageChunks = 4;    // 512-byte chunks per stage (2 KB)
constexpr int kStages = 4;
constexpr int kChunkBytes = 512;
constexpr int kTmaGuessPerWarp = 16;
constexpr int kFlushChunks = 2;             // chunks between flushes of the flagged list
constexpr int kHitCap = 32 * kFlushChunks;  // lane-chunks that can be flagged between flushes

template <int KCAP>
constexpr int tma_cap() { return KCAP + 320; }  // 32 flagged lane-chunks (<= 256 elements) fit after a cut to k

template <int KCAP>
constexpr size_t tma_smem_bytes() {
    return (size_t)kTmaWarps * kStages * kStageChunks * kChunkBytes   // rings
           + (size_t)kTmaWarps * tma_cap<KCAP>() * 8                  // candidate buffers
           + (size_t)kTmaWarps * kHitCap * 16                         // flagged chunks (data)
           + (size_t)kTmaWarps * kHitCap * 4                          // flagged chunks (first id)
           + (size_t)kTmaWarps * 256 * 4                              // histograms
           + (size_t)kTmaWarps * kStages * 8;                         // mbarriers
}

struct RunGeom {
    int c0, ct, c1, nst;  // chunks [c0, ct) by TMA in nst stages, [ct, c1) by plain loads
};

template <int CH>
__device__ __forceinline__ RunGeom run_geom(int item, int warp, int S, int V) {
    const int seg = item % S;
    const int nchunks = (V + CH - 1) / CH, full_chunks = V / CH;
    const int sc0 = (int)((int64_t)nchunks * seg / S), sc1 = (int)((int64_t)nchunks * (seg + 1) / S);
    RunGeom g;
    g.c0 = sc0 + (sc1 - sc0) * warp / kTmaWarps;
    g.c1 = sc0 + (sc1 - sc0) * (warp + 1) / kTmaWarps;
    g.ct = max(g.c0, min(g.c1, full_chunks));
    g.nst = (g.ct - g.c0 + kStageChunks - 1) / kStageChunks;
    return g;
}

template <typename T>
__device__ __forceinline__ const T* item_row(const Params& p, int item) {
    const VerifyArgs& a = p.a;
    const int grow = item / p.S;
    const int b = grow / p.rows_per_seq, r = grow % p.rows_per_seq;
    const bool isP = r < a.K;
    const int pos = isP ? r : r - a.K + 1;
    return reinterpret_cast<const T*>(isP ? a.P : a.Q) + ((int64_t)b * a.K + pos) * a.V;
}

// Unpack the flagged lane-chunks hv[0..nh) (first token ids hid[]) and append their
// elements that pass x >= lo and x > th to the warp's buffer, 32 chunks at a time; the
// buffer is cut to its exact top-k whenever another 32 chunks might not fit.
template <typename T, int CAP>
__device__ __noinline__ void warp_flush_hits(const uint4* hv, const uint32_t* hid, int nh, int nvalid, float lo_f,
                                             uint64_t* buf, uint32_t* hist, WarpSlot* ws, int k, int lane) {
    using Ops = LaneOps<T>;
    constexpr int VEC = Elem<T>::VEC;
    for (int h0 = 0; h0 < nh; h0 += 32) {
        if (ws->count > CAP - 32 * VEC) warp_shrink_packed(buf, hist, ws, k, lane);
        const typename Ops::Thr lo = Ops::thr(lo_f);
        const typename Ops::Thr th = Ops::thr(ws->have_k ? ws->thr : -INFINITY);
        const int h = h0 + lane;
        uint4 v = make_uint4(0, 0, 0, 0);
        uint32_t m = 0, id0 = 0;
        if (h < nh) {
            v = hv[h];
            id0 = hid[h];
            m = Ops::mask(v, nvalid, lo, th);
        }
        const int c = __popc(m);
        const int incl = warp_inclusive_scan(c, lane);
        const int total = __shfl_sync(kFullMask, incl, 31);
        int pos = ws->count + incl - c;
        while (m) {
            const int j = __ffs(m) - 1;
            buf[pos++] = pack_candidate(float_key(raw_get<T>(v, j)), id0 + (uint32_t)j);
            m &= m - 1u;
        }
        __syncwarp();
        if (lane == 0) ws->count += total;
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------------------
// Kernel 1 (rows whose start is 16-byte aligned): persistent, fed by TMA.
// kTmaCtasPerSm CTAs per SM, each taking the grid's work items (row segments) in turn;
// each of a CTA's warps keeps the exact top-k of its run of the item (its 1/kTmaWarps
// share) among the elements >= the item's guess g. Each warp owns a ring of kStages
// shared-memory stages filled by bulk async copies that one lane issues ahead without
// regard to item boundaries, so the next item's data is already arriving while the
// current one finishes; an mbarrier per stage counts the arriving bytes. Testing a
// lane-chunk against the thresholds is a few packed bf16x2 operations; a lane whose
// chunk passes only records it, and after each stage the warp unpacks all recorded chunks
// together into its candidate buffer. The buffer is cut to its exact top-k (packed
// value/id order) when more might not fit; after the cut, later (higher id) elements of
// the warp's run are kept only when strictly above the k-th value.
// The guess g: the CTA sorts the lane maxima of its warps' first stages and takes the
// m-th largest, m chosen so that g is very unlikely to exceed the row's k-th value. The
// result is exact whenever the row's k-th value is >= g (every element that can be in the
// top-k was then a candidate); the finish kernel checks that and otherwise redoes the row.
// Every wait is bounded: on timeout the warp records UNO_ERR_TIMEOUT in the device status
// word, waits (bounded) for its copies still in flight, and stops.
// ---------------------------------------------------------------------------------------
template <typename T, int KCAP>
__global__ void __launch_bounds__(kTmaWarps * 32, kTmaCtasPerSm)
stream_tma_kernel(Params p, int n_items, uint32_t* status) {
    zero_seq_counters(p);
    using Ops = LaneOps<T>;
    constexpr int VEC = Elem<T>::VEC;
    constexpr int CAP = tma_cap<KCAP>();
    constexpr int CH = 32 * VEC;  // elements per chunk (512 bytes)
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char* rings = smem_raw;
    uint4* hvs = reinterpret_cast<uint4*>(rings + (size_t)kTmaWarps * kStages * kStageChunks * kChunkBytes);
    uint64_t* wbuf = reinterpret_cast<uint64_t*>(hvs + kTmaWarps * kHitCap);
    uint32_t* hids = reinterpret_cast<uint32_t*>(wbuf + kTmaWarps * CAP);
    uint32_t* whist = hids + kTmaWarps * kHitCap;
    uint64_t* bars = reinterpret_cast<uint64_t*>(whist + kTmaWarps * 256);
    __shared__ WarpSlot s_slot[kTmaWarps];
    __shared__ int s_nhit[kTmaWarps];
    __shared__ uint64_t s_top[kTmaWarps * kTmaGuessPerWarp];
    __shared__ int s_nsample[kTmaWarps];
    __shared__ float s_guess;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int S = p.S, k = p.a.top_k, V = p.a.V;
    unsigned char* ring = rings + (size_t)warp * kStages * kStageChunks * kChunkBytes;
    uint64_t* bar = bars + warp * kStages;
    uint64_t* buf = wbuf + warp * CAP;
    uint4* hv = hvs + warp * kHitCap;
    uint32_t* hid = hids + warp * kHitCap;
    uint32_t* hist = whist + warp * 256;
    WarpSlot* ws = &s_slot[warp];
    int* nhit = &s_nhit[warp];

    if (lane == 0) {
        for (int j = 0; j < kStages; ++j) mbar_init(&bar[j], 1);
        fence_mbar_init();
        *nhit = 0;
    }
    __syncwarp();

    // producer state (lane 0): the next stage to issue, as (item, stage within the run)
    int pi = blockIdx.x, pt = 0;
    RunGeom pg = pi < n_items ? run_geom<CH>(pi, warp, S, V) : RunGeom{0, 0, 0, 0};
    int issued = 0;  // stages issued so far (all items), lane 0's count
    auto issue_next = [&]() {  // lane 0
        while (pi < n_items && pt >= pg.nst) {  // skip to the next stage that exists
            pi += gridDim.x;
            pt = 0;
            if (pi < n_items) pg = run_geom<CH>(pi, warp, S, V);
        }
        if (pi >= n_items) return;
        const int slot = issued % kStages;
        const uint32_t bytes = (uint32_t)min(kStageChunks, pg.ct - (pg.c0 + pt * kStageChunks)) * kChunkBytes;
        const unsigned char* src = reinterpret_cast<const unsigned char*>(item_row<T>(p, pi)) +
                                   (int64_t)(pg.c0 + pt * kStageChunks) * kChunkBytes;
        mbar_arrive_expect_tx(&bar[slot], bytes);
        bulk_g2s(ring + (size_t)slot * kStageChunks * kChunkBytes, src, bytes, &bar[slot]);
        ++pt;
        ++issued;
    };
    if (lane == 0)
        for (int j = 0; j < kStages; ++j) issue_next();
    __syncwarp();

    int consumed = 0;  // stages consumed so far (all items)
    bool ok = true;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const RunGeom g = run_geom<CH>(item, warp, S, V);
        const T* row = item_row<T>(p, item);
        if (lane == 0) {
            ws->count = 0;
            ws->have_k = 0;
            ws->thr = -INFINITY;
        }
        // ---- the item's guess from every warp's first stage (two CTA barriers per item) ----
        int slot = consumed % kStages;
        if (g.nst > 0) ok = ok && __all_sync(kFullMask, mbar_wait(&bar[slot], (uint32_t)((consumed / kStages) & 1)));
        {
            const int nc0 = (g.nst > 0 && ok) ? min(kStageChunks, g.ct - g.c0) : 0;
            const unsigned char* stg = ring + (size_t)slot * kStageChunks * kChunkBytes;
            float lm = -INFINITY;
            for (int j = 0; j < nc0; ++j) lm = fmaxf(lm, raw_max<T>(lds128(stg + j * kChunkBytes + lane * 16)));
            const uint32_t sorted = warp_sort32_desc(nc0 > 0 ? float_key(lm) : 0u, lane);
            if (lane < kTmaGuessPerWarp)
                s_top[warp * kTmaGuessPerWarp + lane] = ((uint64_t)sorted << 32) | (uint32_t)(warp * 32 + lane);
            if (lane == 0) s_nsample[warp] = nc0 * CH;
            __syncthreads();
            if (warp == 0) {
                int ns = 0;
                for (int w = 0; w < kTmaWarps; ++w) ns += s_nsample[w];
                uint64_t* tb = buf;  // warp 0's buffer is empty at an item's start
                for (int j = lane; j < kTmaWarps * kTmaGuessPerWarp; j += 32) tb[j] = s_top[j];
                __syncwarp();
                warp_sort_desc(tb, kTmaWarps * kTmaGuessPerWarp, lane);
                // lambda = expected number of sample elements among the row's top-k; the
                // m-th largest lane maximum with m = 3 lambda + 8 exceeds the row's k-th
                // value only with negligible probability on exchangeable data
                const int m = (int)(3.0 * k * (double)ns / (double)V) + 8;
                uint32_t gk = 0u;
                if (m <= kTmaWarps * kTmaGuessPerWarp && ns < V) gk = (uint32_t)(tb[m - 1] >> 32);
                if (lane == 0) s_guess = key_float(gk < 0x007FFFFFu ? 0x007FFFFFu : gk);
                __syncwarp();
            }
            __syncthreads();
        }
        const float guess = s_guess;
        const typename Ops::Thr lo = Ops::thr(guess);

        for (int t = 0; t < g.nst && ok; ++t) {
            slot = consumed % kStages;
            if (t > 0) ok = __all_sync(kFullMask, mbar_wait(&bar[slot], (uint32_t)((consumed / kStages) & 1)));
            if (!ok) break;
            const unsigned char* stg = ring + (size_t)slot * kStageChunks * kChunkBytes;
            const int nc = min(kStageChunks, g.ct - (g.c0 + t * kStageChunks));
#pragma unroll
            for (int j0 = 0; j0 < kStageChunks; j0 += kFlushChunks) {
                const typename Ops::Thr th = Ops::thr(ws->have_k ? ws->thr : -INFINITY);
#pragma unroll
                for (int j = j0; j < j0 + kFlushChunks; ++j) {
                    if (j < nc) {
                        const uint4 v = lds128(stg + j * kChunkBytes + lane * 16);
                        if (Ops::hit(v, lo, th)) {
                            const int h = atomicAdd(nhit, 1);
                            hv[h] = v;
                            hid[h] = (uint32_t)((g.c0 + t * kStageChunks + j) * CH + lane * VEC);
                        }
                    }
                }
                __syncwarp();
                const int nh = *nhit;
                if (nh > 0) {
                    warp_flush_hits<T, CAP>(hv, hid, nh, VEC, guess, buf, hist, ws, k, lane);
                    if (lane == 0) *nhit = 0;
                    __syncwarp();
                }
            }
            // every lane's reads of this slot are complete (their values fed the tests above
            // and the warp has passed __syncwarp): the slot can be refilled
            ++consumed;
            if (lane == 0) issue_next();
            __syncwarp();
        }
        if (!ok) break;
        // the row's last, partial chunk (not a multiple of 16 bytes long) by plain loads
        for (int c = g.ct; c < g.c1; ++c) {
            const int64_t e0 = (int64_t)c * CH + lane * VEC;
            const int nv = (int)max((int64_t)0, min((int64_t)VEC, (int64_t)V - e0));
            const uint4 v = nv > 0 ? load_raw<T>(row, e0, nv, nv == VEC) : make_uint4(0, 0, 0, 0);
            const typename Ops::Thr th = Ops::thr(ws->have_k ? ws->thr : -INFINITY);
            if (ws->count > CAP - 32 * VEC) warp_shrink_packed(buf, hist, ws, k, lane);
            if (nv > 0 && Ops::hit(v, lo, th)) lane_append<T>(v, nv, (uint32_t)e0, lo, th, buf, ws);
            __syncwarp();
        }
        if (ws->count > k) warp_shrink_packed(buf, hist, ws, k, lane);
        const int64_t list = (int64_t)item * kTmaWarps + warp;
        uint64_t* out = p.lists + list * KCAP;
        const int cnt = ws->count;
        for (int j = lane; j < cnt; j += 32) out[j] = buf[j];
        if (lane == 0) {
            p.counts[list] = cnt;
            p.guesses[list] = float_key(guess);
        }
        __syncwarp();
    }
    if (!ok) {
        // wait (bounded) for the copies still in flight, then stop
        const int n_issued = __shfl_sync(kFullMask, issued, 0);
        for (int t = consumed; t < n_issued; ++t) mbar_wait(&bar[t % kStages], (uint32_t)((t / kStages) & 1), 1u << 16);
        if (lane == 0) record_device_status(status, (uint32_t)UNO_ERR_TIMEOUT);
    }
}

// Exact top-k of a whole row by one warp, with no guess (the finish kernel's fallback).
// Leaves the k largest (ties to the lower id) in buf[0..return) in ascending id order.
template <typename T, int CAP>
__device__ __noinline__ int warp_exact_row(const T* row, int V, uint64_t* buf, uint32_t* hist, WarpSlot* ws,
                                           uint32_t* bound, int k, int lane) {
    constexpr int VEC = Elem<T>::VEC;
    constexpr int CH = 32 * VEC;
    using Ops = LaneOps<T>;
    const bool aligned = ((reinterpret_cast<uintptr_t>(row) & 15u) == 0);
    if (lane == 0) {
        ws->count = 0;
        ws->have_k = 0;
        ws->thr = -INFINITY;
        *bound = 0x007FFFFFu;
    }
    __syncwarp();
    const int nchunks = (V + CH - 1) / CH;
    for (int c = 0; c < nchunks; ++c) {
        const int64_t e0 = (int64_t)c * CH + lane * VEC;
        const int nv = (int)max((int64_t)0, min((int64_t)VEC, (int64_t)V - e0));
        const uint4 v = nv > 0 ? load_raw<T>(row, e0, nv, aligned) : make_uint4(0, 0, 0, 0);
        const bool hit = nv > 0 && Ops::hit(v, Ops::thr(-INFINITY), Ops::thr(ws->have_k ? ws->thr : -INFINITY));
        if (__any_sync(kFullMask, hit))
            warp_append<T, CAP>(v, hit ? nv : 0, (uint32_t)(c * CH + lane * VEC), buf, hist, ws, bound, -INFINITY, k,
                                lane);
    }
    if (ws->count > k) warp_shrink<KeyBits<T>::value>(buf, hist, ws, bound, k, lane);
    return ws->count;
}

// capacity of the finish kernel's exact fallback buffer (it reuses the row's candidate
// area of lists_per_row * KCAP >= kStreamWarps * KCAP entries)
template <int KCAP>
constexpr int fallback_cap() { return KCAP + 320; }
static_assert(fallback_cap<64>() <= 8 * 64 && fallback_cap<256>() <= 8 * 256 && fallback_cap<1024>() <= 8 * 1024,
              "fallback buffer must fit the candidate area");
static_assert(fallback_cap<64>() - 256 >= 64, "fallback buffer must hold k + one chunk");

template <int KCAP>
constexpr size_t finish_bytes_per_warp(int lists_per_row) {
    return (size_t)lists_per_row * KCAP * 8 + 2 * KCAP * 8 + 256 * 4 + 32;
}

// The row's top-k cand[0..n), in ascending id order -> its survivor record. Sorted copy sb
// (value desc, id asc) gives the fp64 softmax weights relative to the largest value and the
// top-p cut (the shortest prefix of that order whose mass reaches top_p); the survivors are
// then taken from cand in id order (values above the cut value, and the first of the ties at
// it), so no second sort is needed. One warp.
__device__ __forceinline__ void write_survivors_ids(const VerifyArgs& a, uint64_t* cand, int n, uint64_t* sb, double* w,
                                                    RecView rec, int lane) {
    const double Td = (double)a.temperature;
    int np = 1;
    while (np < n) np <<= 1;
    for (int j = lane; j < np; j += 32) sb[j] = j < n ? cand[j] : 0ull;
    __syncwarp();
    warp_sort_desc(sb, np, lane);
    const double zmax = (double)key_float(candidate_key(sb[0])) / Td;
    double part = 0.0;
    for (int j = lane; j < n; j += 32) {
        w[j] = exp((double)key_float(candidate_key(sb[j])) / Td - zmax);
        part += w[j];
    }
    __syncwarp();
    int c = n;
    if (a.top_p < 1.0f) {
        const double Ssum = warp_sum_f64(part), tp = (double)a.top_p;
        double carry = 0.0;
        c = -1;
        for (int b0 = 0; b0 < n && c < 0; b0 += 32) {
            int j = b0 + lane;
            double x = j < n ? w[j] / Ssum : 0.0;
            double incl = warp_scan_f64(x, lane);
            unsigned hit = __ballot_sync(kFullMask, j < n && carry + incl >= tp);
            if (hit) c = b0 + __ffs(hit);
            carry += __shfl_sync(kFullMask, incl, 31);
        }
        if (c < 0) c = n;
    }
    // the cut key and how many of its ties survive (those in sb[0..c))
    const uint32_t kc = c > 0 ? candidate_key(sb[c - 1]) : 0xFFFFFFFFu;
    int above = 0;
    for (int j = lane; j < c; j += 32) above += candidate_key(sb[j]) > kc;
    above = warp_sum(above);
    const int tkeep = c - above;
    int out = 0, ties = 0;
    double z = 0.0;
    for (int b0 = 0; b0 < n; b0 += 32) {
        const int j = b0 + lane;
        const uint64_t x = j < n ? cand[j] : 0ull;
        const uint32_t key = candidate_key(x);
        const bool tie = j < n && key == kc;
        const unsigned tb = __ballot_sync(kFullMask, tie);
        const bool keep = j < n && (key > kc || (tie && ties + __popc(tb & ((1u << lane) - 1u)) < tkeep));
        const unsigned kb = __ballot_sync(kFullMask, keep);
        if (keep) {
            const int o = out + __popc(kb & ((1u << lane) - 1u));
            const double wj = exp((double)key_float(key) / Td - zmax);  // the same weight as in w
            rec.id[o] = (int32_t)candidate_id(x);
            rec.w[o] = wj;
            z += wj;
        }
        out += __popc(kb);
        ties += __popc(tb);
    }
    z = warp_sum_f64(z);
    if (lane == 0) {
        *rec.Z = z;
        *rec.n = out;
    }
}

// Finish row `grow` (one warp): gather its lists, select the exact top-k (redoing the row
// exactly when the streaming guess could have hidden part of it) and write the survivor
// record. `base` is the warp's finish_bytes_per_warp(L) bytes of shared memory.
template <typename T, int KCAP>
__device__ void finish_row(const Params& p, int64_t grow, unsigned char* base, int lane) {
    const VerifyArgs& a = p.a;
    const int k = a.top_k, L = p.lists_per_row;
    uint64_t* cand = reinterpret_cast<uint64_t*>(base);      // [L * KCAP], ascending id
    uint64_t* sb = cand + (size_t)L * KCAP;                  // [np] (value desc, id asc)
    double* w = reinterpret_cast<double*>(sb + KCAP);        // [KCAP]
    uint32_t* hist = reinterpret_cast<uint32_t*>(sb + 2 * KCAP);
    WarpSlot* ws = reinterpret_cast<WarpSlot*>(hist + 256);
    uint32_t* bound = reinterpret_cast<uint32_t*>(ws + 1);

    // gather the row's lists in (segment, warp) order: ascending token id overall. Every
    // list's count and guess is loaded at once (lane l: lists l, l + 32, ...), then every
    // entry, so the gather costs two dependent rounds of loads whatever the list count.
    int n = 0;
    uint32_t G = 0u;  // the largest guess any list was taken with
    for (int l0 = 0; l0 < L; l0 += 32) {
        const int l = l0 + lane;
        const int64_t list = grow * L + l;
        const int cnt = l < L ? __ldcg(p.counts + list) : 0;
        if (l < L) G = max(G, __ldcg(p.guesses + list));
        const int incl = warp_inclusive_scan(cnt, lane);
        const int tot = __shfl_sync(kFullMask, incl, 31);
        const int excl = incl - cnt;
        for (int e0 = 0; e0 < tot; e0 += 32) {
            const int e = e0 + lane;
            // the list holding entry e: the number of lists whose inclusive count is <= e
            int li = 0;
#pragma unroll
            for (int b = 16; b > 0; b >>= 1)
                if (__shfl_sync(kFullMask, incl, li + b - 1) <= e) li += b;
            const int first = __shfl_sync(kFullMask, excl, li & 31);
            if (e < tot) cand[n + e] = __ldcg(p.lists + (grow * L + l0 + li) * KCAP + (e - first));
        }
        n += tot;
    }
    for (int o = 16; o > 0; o >>= 1) G = max(G, __shfl_xor_sync(kFullMask, G, o));
    __syncwarp();
    fin_mark(p, threadIdx.x >> 5, 1);
    // the exact top-k in id order: radix selection over the value keys, ties to the lower id
    const int n_all = n;
    if (n > k) {
        uint32_t tau;
        int need;
        warp_select_key<KeyBits<T>::value>(cand, n, k, hist, lane, tau, need);
        n = warp_compact_key<KeyBits<T>::value>(cand, n, tau, need, lane);
    }
    uint32_t kmin = 0xFFFFFFFFu;
    for (int j = lane; j < n; j += 32) kmin = min(kmin, candidate_key(cand[j]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmin = min(kmin, __shfl_xor_sync(kFullMask, kmin, o));
    // exact iff the k-th value is >= every guess: then every element that can be in the
    // top-k was >= its warp's guess and so was a candidate
    if (n_all < k || kmin < G) {
        // the streaming guess left fewer than k candidates: redo this row exactly
        const int b = (int)(grow / p.rows_per_seq), r = (int)(grow % p.rows_per_seq);
        const bool isP = r < a.K;
        const int pos = isP ? r : r - a.K + 1;
        const T* row = reinterpret_cast<const T*>(isP ? a.P : a.Q) + ((int64_t)b * a.K + pos) * a.V;
        n = warp_exact_row<T, fallback_cap<KCAP>()>(row, a.V, cand, hist, ws, bound, k, lane);
    }
    fin_mark(p, threadIdx.x >> 5, 2);
    // cand[0..n): the row's top-k in id order
    write_survivors_ids(a, cand, n, sb, w, rec_view(p.recs, p.kcap, grow), lane);
    fin_mark(p, threadIdx.x >> 5, 3);
}

// ---------------------------------------------------------------------------------------
// Kernel 2: warp w of CTA c finishes row c fw + w: merges its lists into the exact top-k,
// applies softmax and top-p in fp64 and writes the survivor record sorted by token id. The
// CTA then adds its rows to each of their sequences' counters (after a fence); the CTA that
// completes a sequence runs its draft sampling, acceptance, longest accepted prefix and
// residual resample. Spreading the rows over many CTAs keeps every SM busy; no CTA waits for
// another.
// ---------------------------------------------------------------------------------------
constexpr int kFinWarps = 16;

template <typename T, int KCAP>
__global__ void __launch_bounds__(kFinWarps * 32)
finish_seq_kernel(Params p, int fw, int n_rows, size_t smem_bytes) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ int s_done[kFinWarps], s_nd;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rps = p.rows_per_seq;
    const int64_t r0 = (int64_t)blockIdx.x * fw, r1 = min(r0 + fw, (int64_t)n_rows);
    // launched as a programmatic dependent of the streaming kernel: its CTAs may start while
    // the last rows stream; the lists are read only after that grid has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");
    fin_mark(p, warp, 0);
    if (warp < fw && r0 + warp < r1) {
        unsigned char* base = smem_raw + (size_t)warp * finish_bytes_per_warp<KCAP>(p.lists_per_row);
        finish_row<T, KCAP>(p, r0 + warp, base, lane);
        __threadfence();  // the record is visible to the CTA that verifies its sequence
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int nd = 0;
        for (int64_t r = r0; r < r1;) {
            const int b = (int)(r / rps);
            const int64_t e = min(r1, (int64_t)(b + 1) * rps);
            const unsigned add = (unsigned)(e - r);
            if (atomicAdd(&p.seq_done[b], add) + add == (unsigned)rps) s_done[nd++] = b;
            r = e;
        }
        s_nd = nd;
        if (nd) __threadfence();
    }
    __syncthreads();
    fin_mark(p, warp, 4);
    for (int j = 0; j < s_nd; ++j) {
        sequence_verify<kFinWarps>(p.a, p.recs, KCAP, s_done[j], rps, smem_raw, smem_bytes);
        __syncthreads();
    }
    fin_mark(p, warp, 5);
}

// ---------------------------------------------------------------------------------------
// Kernel 1 (bf16 rows, 16-byte aligned, V a multiple of 8, k <= 256): persistent over rows.
// kRowsCtasPerSm CTAs of kRowsWarps warps per SM take the rows in turn, so no SM idles
// through a last partial wave. Each warp streams its 1/kRowsWarps run of the row with
// 16-byte register loads one group of kGroup chunks ahead (a chunk is 32 lanes x 8
// elements, a group gives each lane 64 elements to test); a group costs a few packed
// bf16x2 maxima and one vote. A lane whose chunk holds an element at or above the
// threshold only records the chunk (one 16-byte shared store); once 32 chunks are recorded
// the warp unpacks them together into its candidate buffer (cut to its exact top-k, packed
// value/id order, when more might not fit; after a cut, later elements of the run are kept
// only when strictly above the k-th value). The threshold starts at a guess g: every warp
// offers the four largest lane maxima of its first group, and g is the m-th largest of
// those 32 offers, m = 3 lambda + 4 with lambda the expected number of the row's top-k
// among the sampled elements. g exceeds the row's k-th value only with negligible
// probability on exchangeable data; the finish kernel checks every row (its k-th value
// must be >= g, so that every element that can be in the top-k was a candidate) and redoes
// the rare failures exactly. The next row's first group is loaded before this row's lists
// are written, so the warp's loads stay in flight across rows. No CTA waits for another.
// ---------------------------------------------------------------------------------------
constexpr int kRowsWarps = 8;
constexpr int kRowsCtasPerSm = 2;
constexpr int kGroup = 8;                        // chunks per group
constexpr int kHitSlots = 32 + 32 * kGroup;      // recorded chunks: < 32 carried + one group
constexpr uint32_t kNegInfPair = 0xFF80FF80u;    // two bf16 -inf

template <int KCAP>
constexpr int rows_cap() { return KCAP + 320; }  // a flush of 32 chunks (<= 256 elements) fits after a cut

// shared memory: recorded chunks [warp][kHitSlots] (16 bytes + id each), candidate buffers
// [warp][rows_cap], histograms [warp][256]
template <int KCAP>
constexpr size_t rows_smem_bytes() {
    return (size_t)kRowsWarps * ((size_t)kHitSlots * (16 + 4) + (size_t)rows_cap<KCAP>() * 8 + 256 * 4);
}

__device__ __forceinline__ __nv_bfloat162 bf2_of(uint32_t w) { return *reinterpret_cast<const __nv_bfloat162*>(&w); }
__device__ __forceinline__ __nv_bfloat162 bf2_max4(const uint4& v) {
    return __hmax2(__hmax2(bf2_of(v.x), bf2_of(v.y)), __hmax2(bf2_of(v.z), bf2_of(v.w)));
}

template <int KCAP>
__global__ void __launch_bounds__(kRowsWarps * 32, kRowsCtasPerSm)
stream_rows_kernel(Params p, int n_items) {
    zero_seq_counters(p);
    constexpr int CAP = rows_cap<KCAP>();
    constexpr int CH = 256;  // elements per chunk
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint4* hvs = reinterpret_cast<uint4*>(smem_raw);
    uint64_t* wbuf = reinterpret_cast<uint64_t*>(hvs + kRowsWarps * kHitSlots);
    uint32_t* hids = reinterpret_cast<uint32_t*>(wbuf + kRowsWarps * CAP);
    uint32_t* whist = hids + kRowsWarps * kHitSlots;
    __shared__ WarpSlot s_slot[kRowsWarps];
    __shared__ uint32_t s_top[kRowsWarps * 4];
    __shared__ int s_nsample[kRowsWarps];
    __shared__ float s_guess;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const VerifyArgs& a = p.a;
    const int k = a.top_k, V = a.V;
    const int V8 = V >> 3;
    const int nchunks = (V + CH - 1) / CH;
    uint4* hv = hvs + warp * kHitSlots;
    uint32_t* hid = hids + warp * kHitSlots;
    uint64_t* buf = wbuf + warp * CAP;
    uint32_t* hist = whist + warp * 256;
    WarpSlot* ws = &s_slot[warp];

    // the warp's chunk run [c0, c1) of a row
    auto run_of = [&](int& c0, int& c1) {
        c0 = nchunks * warp / kRowsWarps;
        c1 = nchunks * (warp + 1) / kRowsWarps;
    };
    auto row_of = [&](int grow) -> const __nv_bfloat16* {
        const int b = grow / p.rows_per_seq, r = grow % p.rows_per_seq;
        const bool isP = r < a.K;
        const int pos = isP ? r : r - a.K + 1;
        return reinterpret_cast<const __nv_bfloat16*>(isP ? a.P : a.Q) + ((int64_t)b * a.K + pos) * V;
    };
    // chunk c of the run: this lane's 8 elements, or two -inf pairs past the run or the row
    auto load = [&](const uint4* r4, int c, int c1) -> uint4 {
        const int idx = c * 32 + lane;
        return (c < c1 && idx < V8) ? ld_stream_v4(r4 + idx) : make_uint4(kNegInfPair, kNegInfPair, kNegInfPair, kNegInfPair);
    };

    int item = blockIdx.x;
    int c0 = 0, c1 = 0;
    uint4 cur[kGroup];
    const uint4* r4 = nullptr;
    if (item < n_items) {
        run_of(c0, c1);
        r4 = reinterpret_cast<const uint4*>(row_of(item));
#pragma unroll
        for (int u = 0; u < kGroup; ++u) cur[u] = load(r4, c0 + u, c1);
    }
    for (; item < n_items; item += gridDim.x) {
        const int grow = item;
        if (lane == 0) {
            ws->count = 0;
            ws->have_k = 0;
            ws->thr = -INFINITY;
        }
        // ---- the guess, from every warp's first group ----
        {
            float lm = -INFINITY;
            int nv = 0;
#pragma unroll
            for (int u = 0; u < kGroup; ++u) {
                const int c = c0 + u;
                if (c < c1 && c * 32 + lane < V8) {
                    const __nv_bfloat162 m2 = bf2_max4(cur[u]);
                    lm = fmaxf(lm, fmaxf(__low2float(m2), __high2float(m2)));
                    nv += 8;
                }
            }
            uint32_t key = nv > 0 ? float_key(lm) : 0u;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                uint32_t mx = key;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(kFullMask, mx, o));
                if (lane == 0) s_top[warp * 4 + t] = mx;
                const unsigned owner = __ballot_sync(kFullMask, key == mx);
                if (lane == __ffs(owner) - 1) key = 0u;
            }
            nv = warp_sum(nv);
            if (lane == 0) s_nsample[warp] = nv;
            __syncthreads();
            if (warp == 0) {
                int ns = 0;
                for (int w = 0; w < kRowsWarps; ++w) ns += s_nsample[w];
                const uint32_t sorted = warp_sort32_desc(s_top[lane], lane);
                const int m = (int)(3.0 * k * (double)ns / (double)V) + 4;
                uint32_t g = 0u;
                const uint32_t gm = __shfl_sync(kFullMask, sorted, (m - 1) & 31);
                if (m <= 32 && ns < V) g = gm;
                if (lane == 0) s_guess = key_float(g < 0x007FFFFFu ? 0x007FFFFFu : g);
            }
            __syncthreads();
        }
        const float guess = s_guess;
        __nv_bfloat162 lo2 = __float2bfloat162_rn(guess);  // the guess is a bf16 value (or -inf)
        int nh = 0;
        // ---- stream the run ----
        int c = c0;
        while (true) {
            if (nh >= 32) {  // unpack the recorded chunks (the next group's loads are not out yet)
                __syncwarp();
                warp_flush_hits<__nv_bfloat16, CAP>(hv, hid, nh, 8, guess, buf, hist, ws, k, lane);
                nh = 0;
                const float th = ws->have_k ? ws->thr : -INFINITY;
                lo2 = __float2bfloat162_rn(fmaxf(guess, th));
            }
            const bool more = c + kGroup < c1;
            uint4 nxt[kGroup];
            if (more) {
#pragma unroll
                for (int u = 0; u < kGroup; ++u) nxt[u] = load(r4, c + kGroup + u, c1);
            }
            __nv_bfloat162 mu[kGroup];
#pragma unroll
            for (int u = 0; u < kGroup; ++u) mu[u] = bf2_max4(cur[u]);
            __nv_bfloat162 gm2 = mu[0];
#pragma unroll
            for (int u = 1; u < kGroup; ++u) gm2 = __hmax2(gm2, mu[u]);
            if (__any_sync(kFullMask, __hge2_mask(gm2, lo2) != 0u)) {
#pragma unroll
                for (int u = 0; u < kGroup; ++u) {
                    const int cc = c + u;
                    const bool f = cc < c1 && cc * 32 + lane < V8 && __hge2_mask(mu[u], lo2) != 0u;
                    const unsigned bal = __ballot_sync(kFullMask, f);
                    if (f) {
                        const int pos = nh + __popc(bal & ((1u << lane) - 1u));
                        hv[pos] = cur[u];
                        hid[pos] = (uint32_t)(cc * CH + lane * 8);
                    }
                    nh += __popc(bal);
                }
            }
            if (!more) break;
#pragma unroll
            for (int u = 0; u < kGroup; ++u) cur[u] = nxt[u];
            c += kGroup;
        }
        // ---- the warp's list: its exact top-k among the candidates ----
        __syncwarp();
        if (nh > 0) warp_flush_hits<__nv_bfloat16, CAP>(hv, hid, nh, 8, guess, buf, hist, ws, k, lane);
        if (ws->count > k) warp_shrink_packed(buf, hist, ws, k, lane);
        const int64_t list = (int64_t)grow * kRowsWarps + warp;
        uint64_t* out = p.lists + list * KCAP;
        const int cnt = ws->count;
        for (int j = lane; j < cnt; j += 32) out[j] = buf[j];
        if (lane == 0) {
            p.counts[list] = cnt;
            p.guesses[list] = float_key(guess);
        }
        __syncwarp();
        // ---- the next row's first group ----
        const int next = item + gridDim.x;
        if (next < n_items) {
            run_of(c0, c1);
            r4 = reinterpret_cast<const uint4*>(row_of(next));
#pragma unroll
            for (int u = 0; u < kGroup; ++u) cur[u] = load(r4, c0 + u, c1);
        }
    }
    // this CTA's rows are written: the finish kernel may be scheduled
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

inline int num_sms() {
    static int n[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (n[dev] == 0) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : 148;
    }
    return n[dev];
}

struct Layout {
    int kcap, S, rows_per_seq, lists_per_row;
    size_t off_lists, off_counts, off_guesses, off_recs, off_seq, off_trace, total;
};

// The streaming kernel a batch takes: UNO_VERIFY_STREAM=warps (one CTA per row segment,
// any dtype and alignment) or =tma (TMA-fed, 16-byte aligned rows) select one; by default
// bf16 rows that are 16-byte aligned with V a multiple of 8 and k <= 256 take the
// persistent row-segment kernel, the rest the per-segment CTAs.
enum class StreamKind { kRows, kWarps, kTma };
inline StreamKind stream_kind(const VerifyArgs& a) {
    const bool aligned = ((reinterpret_cast<uintptr_t>(a.P) | reinterpret_cast<uintptr_t>(a.Q)) & 15u) == 0;
    const size_t esz = a.dtype == UNO_BF16 ? 2 : 4;
    const bool rows_aligned = aligned && ((size_t)a.V * esz) % 16 == 0;
    const char* sel = getenv("UNO_VERIFY_STREAM");
    if (sel && strcmp(sel, "warps") == 0) return StreamKind::kWarps;
    if (sel && strcmp(sel, "tma") == 0) return rows_aligned ? StreamKind::kTma : StreamKind::kWarps;
    return (a.dtype == UNO_BF16 && rows_aligned && a.top_k <= 256) ? StreamKind::kRows : StreamKind::kWarps;
}

// Segments per row: the persistent kernel takes whole rows; the per-segment CTAs one each
// unless UNO_VERIFY_SEGMENTS=s forces s.
inline int choose_segments(int V, StreamKind kind) {
    if (kind == StreamKind::kRows) return 1;
    int forced = 0;
    if (const char* e = getenv("UNO_VERIFY_SEGMENTS")) forced = atoi(e);
    int S = forced > 0 ? forced : 1;
    int nchunks = (V + 255) / 256;
    if (S > nchunks) S = nchunks;
    if (S > 8) S = 8;
    return S < 1 ? 1 : S;
}

inline Layout layout(const VerifyArgs& a) {
    Layout L{};
    L.kcap = a.top_k <= 64 ? 64 : (a.top_k <= 256 ? 256 : 1024);
    L.S = choose_segments(a.V, stream_kind(a));
    // a finishing warp holds a row's lists in shared memory: fewer segments where they
    // would not fit
    while (L.S > 1 && ((size_t)L.S * 8 * L.kcap * 8 + 2 * (size_t)L.kcap * 8 + 256 * 4 + 32) > 220 * 1024) --L.S;
    L.rows_per_seq = 2 * a.K - 1;
    // sized for the streaming kernel with the most warps; the launch sets the actual count
    L.lists_per_row = L.S * (kTmaWarps > kStreamWarps ? kTmaWarps : kStreamWarps);
    size_t rows = (size_t)a.B * L.rows_per_seq;
    L.off_lists = 0;
    L.off_counts = align_up(rows * L.lists_per_row * L.kcap * 8, 256);
    L.off_guesses = align_up(L.off_counts + rows * L.lists_per_row * 4, 256);
    L.off_recs = align_up(L.off_guesses + rows * L.lists_per_row * 4, 256);
    L.off_seq = align_up(L.off_recs + rows * rec_bytes(L.kcap), 256);
    L.total = align_up(L.off_seq + (size_t)a.B * 4, 256);
    L.off_trace = L.total;
    if (getenv("UNO_VERIFY_TRACE")) L.total += 32 * 8 * 8;
    return L;
}

template <typename F>
uno_status set_smem(F* fn, size_t bytes, bool& done, const char* what) {
    if (done) return UNO_OK;
    uno_status s = check_cuda(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes), what);
    if (s == UNO_OK) done = true;
    return s;
}

template <typename T, int KCAP>
uno_status launch_t(const VerifyArgs& a, const Layout& L, unsigned char* ws, cudaStream_t stream) {
    Params p{};
    p.a = a;
    p.S = L.S;
    p.rows_per_seq = L.rows_per_seq;
    p.lists_per_row = L.lists_per_row;
    p.lists = reinterpret_cast<uint64_t*>(ws + L.off_lists);
    p.counts = reinterpret_cast<int32_t*>(ws + L.off_counts);
    p.guesses = reinterpret_cast<uint32_t*>(ws + L.off_guesses);
    p.recs = ws + L.off_recs;
    p.seq_done = reinterpret_cast<uint32_t*>(ws + L.off_seq);
    p.trace = getenv("UNO_VERIFY_TRACE") ? reinterpret_cast<unsigned long long*>(ws + L.off_trace) : nullptr;
    p.kcap = KCAP;
    const int n_rows = a.B * L.rows_per_seq;
    const StreamKind kind = stream_kind(a);
    const bool use_tma = kind == StreamKind::kTma && tma_smem_bytes<KCAP>() <= 227 * 1024;
    const bool use_rows = kind == StreamKind::kRows && std::is_same<T, __nv_bfloat16>::value && KCAP <= 256;
    p.lists_per_row = L.S * (use_tma ? kTmaWarps : (use_rows ? kRowsWarps : kStreamWarps));
    static bool a1 = false, a2 = false;
    const size_t smem1 = (size_t)kStreamWarps * cap_entries<KCAP>() * 8 + (size_t)kStreamWarps * 256 * 4;
    // the finish: as many warps finishing rows at once as their lists fit in shared memory
    // (the kernel's static shared memory takes the rest of the 227 KB)
    constexpr size_t kFinSmem = 220 * 1024;
    const size_t per_warp = finish_bytes_per_warp<KCAP>(p.lists_per_row);
    if (per_warp > kFinSmem) return set_error(UNO_ERR_UNSUPPORTED, "verify: too many segments for top_k %d", a.top_k);
    const int fw = (int)std::min<size_t>(kFinWarps, kFinSmem / per_warp);
    const size_t smem2 = std::max<size_t>((size_t)fw * per_warp, (size_t)2 * 12 * KCAP);

    uno_status s;
    if ((s = set_smem(finish_seq_kernel<T, KCAP>, kFinSmem, a2, "cudaFuncSetAttribute(verify finish)")) != UNO_OK)
        return s;
    const int n_items = n_rows * L.S;
    if (use_rows) {
        if constexpr (KCAP <= 256) {
            static bool a0 = false;
            constexpr size_t smem0 = rows_smem_bytes<KCAP>();
            if ((s = set_smem(stream_rows_kernel<KCAP>, smem0, a0, "cudaFuncSetAttribute(verify rows)")) != UNO_OK)
                return s;
            const int grid = std::min(n_rows, num_sms() * kRowsCtasPerSm);
            stream_rows_kernel<KCAP><<<(unsigned)grid, kRowsWarps * 32, smem0, stream>>>(p, n_rows);
        }
    } else if (use_tma) {
        static bool a0 = false;
        const size_t smem0 = tma_smem_bytes<KCAP>();
        if ((s = set_smem(stream_tma_kernel<T, KCAP>, smem0, a0, "cudaFuncSetAttribute(verify stream tma)")) != UNO_OK)
            return s;
        const int grid = n_items < num_sms() * kTmaCtasPerSm ? n_items : num_sms() * kTmaCtasPerSm;
        stream_tma_kernel<T, KCAP><<<(unsigned)grid, kTmaWarps * 32, smem0, stream>>>(p, n_items, device_status_ptr());
    } else {
        if ((s = set_smem(stream_kernel<T, KCAP>, smem1, a1, "cudaFuncSetAttribute(verify stream)")) != UNO_OK) return s;
        stream_kernel<T, KCAP><<<(unsigned)(n_rows * L.S), kStreamWarps * 32, smem1, stream>>>(p);
    }
    if ((s = check_cuda(cudaGetLastError(), "launch(verify stream)")) != UNO_OK) return s;
    // a programmatic dependent launch (UNO_VERIFY_PDL=0: an ordinary one)
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.gridDim = dim3((unsigned)((n_rows + fw - 1) / fw));
    cfg.blockDim = dim3(kFinWarps * 32);
    cfg.dynamicSmemBytes = smem2;
    cfg.stream = stream;
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    const char* pe = getenv("UNO_VERIFY_PDL");
    cfg.numAttrs = (pe && strcmp(pe, "0") == 0) ? 0 : 1;
    return check_cuda(cudaLaunchKernelEx(&cfg, finish_seq_kernel<T, KCAP>, p, fw, n_rows, smem2), "launch(verify finish)");
}

}  // namespace vtopk

size_t verify_topk_workspace_bytes(const VerifyArgs& a) { return vtopk::layout(a).total; }

uno_status verify_topk_launch(const VerifyArgs& a, void* workspace, cudaStream_t stream) {
    vtopk::Layout L = vtopk::layout(a);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const bool bf = a.dtype == UNO_BF16;
    switch (L.kcap) {
        case 64:
            return bf ? vtopk::launch_t<__nv_bfloat16, 64>(a, L, ws, stream) : vtopk::launch_t<float, 64>(a, L, ws, stream);
        case 256:
            return bf ? vtopk::launch_t<__nv_bfloat16, 256>(a, L, ws, stream) : vtopk::launch_t<float, 256>(a, L, ws, stream);
        default:
            return bf ? vtopk::launch_t<__nv_bfloat16, 1024>(a, L, ws, stream) : vtopk::launch_t<float, 1024>(a, L, ws, stream);
    }
}

}  // namespace uno
