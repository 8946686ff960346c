// verify_topk.cu — lossless block verify with top-k on (optionally followed by top-p).
//
// Lossless verification of a drafted block: LoopUno project page, "How it works" (the
// unmodified model verifies the block, keeps the longest correct prefix, position 0 is the
// exact AR token) and "Training is self-distillation" (acceptance probability 1 - TV);
// sampler settings from the uno-qwen3-8B model card, "Evaluation protocol" (temperature
// 1.0, top-k 50, top-p 0.95, block 16).
//
// One launch does the whole step. The logit rows (verifier rows 0..K-1 and drafter rows
// 1..K-1 of every sequence) are cut into S segments; one CTA streams one segment once
// with 16-byte coalesced loads and keeps the segment's exact top-k:
//   - a CTA-wide lower bound tau0 = k-th largest of the per-thread maxima of the first
//     loads (k distinct elements are >= it, so nothing below it can be in the top-k);
//   - each warp walks its sub-range in token-id order and appends candidates to its own
//     shared-memory buffer; once the buffer has been cut to its exact top-k, later (higher
//     id) elements are appended only when strictly above the k-th value, which keeps the
//     ties-to-lower-id rule exact;
//   - the warps' lists are merged with a CTA radix select and written to the workspace.
// The last CTA to finish a row (atomic counter, no waiting) merges the S lists, applies
// softmax and top-p in fp64 and stores the survivor list sorted by token id. The last row
// of a sequence to finish runs the per-sequence verify (draft sampling, acceptance,
// prefix, residual resample) in one warp, one lane per block position.
#include <cuda_bf16.h>

#include <cstdlib>

#include "select.cuh"
#include "verify_common.cuh"

namespace uno {
namespace vtopk {

constexpr int kUnroll = 4;

template <int KCAP>
struct Cfg;
template <>
struct Cfg<64> { static constexpr int WARPS = 16, MIN_CTAS = 2; };
template <>
struct Cfg<256> { static constexpr int WARPS = 8, MIN_CTAS = 2; };
template <>
struct Cfg<1024> { static constexpr int WARPS = 4, MIN_CTAS = 2; };

template <int KCAP>
constexpr int cap_entries() { return KCAP + 384; }

template <typename T, int KCAP>
constexpr size_t smem_bytes() {
    constexpr int W = Cfg<KCAP>::WARPS;
    return (size_t)W * cap_entries<KCAP>() * 8 + (size_t)W * KCAP * 8 + (size_t)W * 256 * 4 + 256 * 4;
}

struct Params {
    VerifyArgs a;
    int S;
    int rows_per_seq;
    uint32_t* row_counter;
    uint32_t* seq_counter;
    uint64_t* seg_lists;
    unsigned char* recs;
    int kcap;
};

struct WarpState {
    uint64_t* buf;
    uint32_t* hist;
    int count;
    bool have_k;
    float thr;
};

__device__ __forceinline__ void warp_shrink(WarpState& s, int k, int lane) {
    uint64_t T = warp_select(s.buf, s.count, k, s.hist, lane);
    uint64_t mn;
    s.count = warp_compact(s.buf, s.count, T, lane, &mn);
    s.have_k = true;
    s.thr = key_float(candidate_key(mn));
    __syncwarp();
}

// Offer one lane-chunk (raw vector v with nvalid elements, token ids id0..) to the warp's
// candidate buffer. Only lanes whose maximum passes both thresholds unpack the vector.
template <typename T, int CAP>
__device__ __forceinline__ void warp_offer(WarpState& s, const uint4& v, int nvalid, uint32_t id0, float tau0,
                                           int k, int lane) {
    constexpr int VEC = Elem<T>::VEC;
    const float vmax = raw_max<T>(v);
    bool hit = nvalid > 0 && vmax >= tau0 && (!s.have_k || vmax > s.thr);
    if (!__any_sync(kFullMask, hit)) return;
    int c = 0;
    uint32_t mask = 0;
    if (hit) {
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            float x = raw_get<T>(v, j);
            bool t = j < nvalid && x >= tau0 && (!s.have_k || x > s.thr);
            mask |= (uint32_t)t << j;
            c += t;
        }
    }
    int incl = warp_inclusive_scan(c, lane);
    int total = __shfl_sync(kFullMask, incl, 31);
    int pos = s.count + incl - c;
#pragma unroll
    for (int j = 0; j < VEC; ++j)
        if ((mask >> j) & 1u) s.buf[pos++] = pack_candidate(float_key(raw_get<T>(v, j)), id0 + (uint32_t)j);
    s.count += total;
    __syncwarp();
    if (s.count > CAP - 32 * VEC) warp_shrink(s, k, lane);
}

template <typename T, int KCAP>
__global__ void __launch_bounds__(Cfg<KCAP>::WARPS * 32, Cfg<KCAP>::MIN_CTAS)
rows_kernel(Params p) {
    constexpr int VEC = Elem<T>::VEC;
    constexpr int WARPS = Cfg<KCAP>::WARPS;
    constexpr int NT = WARPS * 32;
    constexpr int CAP = cap_entries<KCAP>();
    constexpr int CH = 32 * VEC;  // elements per warp step (one "chunk")

    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint64_t* wbuf = reinterpret_cast<uint64_t*>(smem_raw);
    uint64_t* merged = wbuf + WARPS * CAP;
    uint32_t* whist = reinterpret_cast<uint32_t*>(merged + WARPS * KCAP);
    uint32_t* chist = whist + WARPS * 256;
    __shared__ uint64_t bc[4];
    __shared__ int s_cnt[WARPS];
    __shared__ int s_w;
    __shared__ int s_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const VerifyArgs& a = p.a;
    const int S = p.S, k = a.top_k, V = a.V;
    const int grow = blockIdx.x / S, seg = blockIdx.x % S;
    const int b = grow / p.rows_per_seq, r = grow % p.rows_per_seq;
    const bool isP = r < a.K;
    const int pos = isP ? r : r - a.K + 1;
    const int64_t row_elem0 = ((int64_t)b * a.K + pos) * V;
    const T* row = reinterpret_cast<const T*>(isP ? a.P : a.Q) + row_elem0;
    const bool aligned = ((reinterpret_cast<uintptr_t>(row) & 15u) == 0);

    const int nchunks = (V + CH - 1) / CH;
    const int sc0 = (int)((int64_t)nchunks * seg / S), sc1 = (int)((int64_t)nchunks * (seg + 1) / S);
    const int c0 = sc0 + (int)((int64_t)(sc1 - sc0) * warp / WARPS);
    const int c1 = sc0 + (int)((int64_t)(sc1 - sc0) * (warp + 1) / WARPS);

    WarpState st{wbuf + warp * CAP, whist + warp * 256, 0, false, 0.f};

    // ---- prologue: the first kUnroll chunks of each warp; CTA lower bound tau0 ----
    uint4 raw[kUnroll];
    int nv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        int c = c0 + u;
        int64_t e0 = (int64_t)c * CH + lane * VEC;
        nv[u] = (c < c1) ? (int)max((int64_t)0, min((int64_t)VEC, (int64_t)V - e0)) : 0;
        raw[u] = nv[u] > 0 ? load_raw<T>(row, e0, nv[u], aligned) : make_uint4(0, 0, 0, 0);
    }
    float tmax = -INFINITY;
    bool tany = false;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        if (nv[u] > 0) {
            tmax = fmaxf(tmax, raw_max<T>(raw[u]));
            tany = true;
        }
    }
    float tau0 = -INFINITY;
    {
        int have = __syncthreads_count(tany);
        if (have >= k) {
            merged[tid] = tany ? pack_candidate(float_key(tmax), (uint32_t)tid) : 0ull;
            __syncthreads();
            uint64_t T0 = cta_select<NT>(merged, NT, k, chist, bc);
            uint32_t key = candidate_key(T0);
            tau0 = key_float(key < 0x007FFFFFu ? 0x007FFFFFu : key);
        }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
        warp_offer<T, CAP>(st, raw[u], nv[u], (uint32_t)((c0 + u) * CH + lane * VEC), tau0, k, lane);

    // ---- stream the rest of the warp's range ----
    for (int cb = c0 + kUnroll; cb < c1; cb += kUnroll) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            int c = cb + u;
            int64_t e0 = (int64_t)c * CH + lane * VEC;
            nv[u] = (c < c1) ? (int)max((int64_t)0, min((int64_t)VEC, (int64_t)V - e0)) : 0;
            raw[u] = nv[u] > 0 ? load_raw<T>(row, e0, nv[u], aligned) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            warp_offer<T, CAP>(st, raw[u], nv[u], (uint32_t)((cb + u) * CH + lane * VEC), tau0, k, lane);
    }
    if (st.count > k) warp_shrink(st, k, lane);

    // ---- merge the warps' lists: the segment's exact top-k ----
    if (lane == 0) s_cnt[warp] = st.count;
    __syncthreads();
    int off = 0, total = 0;
    for (int w = 0; w < WARPS; ++w) {
        off += (w < warp) ? s_cnt[w] : 0;
        total += s_cnt[w];
    }
    for (int j = lane; j < st.count; j += 32) merged[off + j] = st.buf[j];
    if (tid == 0) s_w = 0;
    __syncthreads();
    uint64_t T1 = 0;
    if (total > k) T1 = cta_select<NT>(merged, total, k, chist, bc);
    uint64_t* out = p.seg_lists + ((int64_t)grow * S + seg) * KCAP;
    for (int j = tid; j < total; j += NT) {
        uint64_t v = merged[j];
        if (v >= T1) out[atomicAdd(&s_w, 1)] = v;
    }
    __syncthreads();
    for (int j = s_w + tid; j < KCAP; j += NT) out[j] = 0ull;

    // ---- last CTA of the row: survivors of the warped row ----
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&p.row_counter[grow], 1u) == (unsigned)(S - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int n = S * KCAP;
    const uint64_t* lists = p.seg_lists + (int64_t)grow * S * KCAP;
    for (int j = tid; j < n; j += NT) merged[j] = __ldcg(lists + j);
    __syncthreads();
    uint64_t T2 = cta_select<NT>(merged, n, k, chist, bc);
    int np = 1;
    while (np < k) np <<= 1;
    uint64_t* sb = wbuf;                                       // [np] selected, sorted
    double* w = reinterpret_cast<double*>(wbuf + KCAP);        // [KCAP] weights
    uint64_t* ib = wbuf + 2 * KCAP;                            // [np] id-sort keys
    if (tid == 0) s_w = 0;
    __syncthreads();
    for (int j = tid; j < n; j += NT) {
        uint64_t v = merged[j];
        if (v >= T2) sb[atomicAdd(&s_w, 1)] = v;
    }
    __syncthreads();
    for (int j = k + tid; j < np; j += NT) sb[j] = 0ull;
    __syncthreads();
    cta_sort_desc<NT>(sb, np);
    const double Td = (double)a.temperature;
    const double zmax = (double)key_float(candidate_key(sb[0])) / Td;
    for (int j = tid; j < k; j += NT) w[j] = exp((double)key_float(candidate_key(sb[j])) / Td - zmax);
    __syncthreads();
    if (tid == 0) {
        int c = k;
        if (a.top_p < 1.0f) {
            double Ssum = 0.0;
            for (int j = 0; j < k; ++j) Ssum += w[j];
            double cum = 0.0, tp = (double)a.top_p;
            for (int j = 0; j < k; ++j) {
                cum += w[j] / Ssum;
                if (cum >= tp) {
                    c = j + 1;
                    break;
                }
            }
        }
        s_w = c;
    }
    __syncthreads();
    const int nsurv = s_w;
    int np2 = 1;
    while (np2 < nsurv) np2 <<= 1;
    for (int j = tid; j < np2; j += NT)
        ib[j] = j < nsurv ? ((uint64_t)(0xFFFFFFFFu - candidate_id(sb[j])) << 32) | (uint64_t)j : 0ull;
    __syncthreads();
    cta_sort_desc<NT>(ib, np2);
    RecView rec = rec_view(p.recs, p.kcap, grow);
    for (int j = tid; j < nsurv; j += NT) {
        uint64_t e = ib[j];
        rec.id[j] = (int32_t)(0xFFFFFFFFu - (uint32_t)(e >> 32));
        rec.w[j] = w[(uint32_t)(e & 0xFFFFFFFFu)];
    }
    __syncthreads();
    if (tid == 0) {
        double Z = 0.0;
        for (int j = 0; j < nsurv; ++j) Z += __ldcg(rec.w + j);
        *rec.Z = Z;
        *rec.n = nsurv;
    }

    // ---- last row of the sequence: the verify decisions ----
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&p.seq_counter[b], 1u) == (unsigned)(p.rows_per_seq - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (warp == 0) sequence_verify(a, p.recs, p.kcap, b, p.rows_per_seq, lane);
}

struct Layout {
    int kcap, S, rows_per_seq;
    size_t off_row_cnt, off_seq_cnt, off_lists, off_recs, total;
};

inline int choose_segments(int V, int warps) {
    static int forced = -1;
    if (forced < 0) {
        const char* e = getenv("UNO_VERIFY_SEGMENTS");
        forced = e ? atoi(e) : 0;
    }
    int S = forced > 0 ? forced : V / 49152;
    if (S < 1) S = 1;
    if (S > warps) S = warps;
    return S;
}

inline Layout layout(const VerifyArgs& a) {
    Layout L{};
    L.kcap = a.top_k <= 64 ? 64 : (a.top_k <= 256 ? 256 : 1024);
    int warps = L.kcap == 64 ? Cfg<64>::WARPS : (L.kcap == 256 ? Cfg<256>::WARPS : Cfg<1024>::WARPS);
    L.S = choose_segments(a.V, warps);
    L.rows_per_seq = 2 * a.K - 1;
    size_t rows = (size_t)a.B * L.rows_per_seq;
    L.off_row_cnt = 0;
    L.off_seq_cnt = align_up(rows * 4, 16);
    L.off_lists = align_up(L.off_seq_cnt + (size_t)a.B * 4, 256);
    L.off_recs = align_up(L.off_lists + rows * L.S * L.kcap * 8, 256);
    L.total = align_up(L.off_recs + rows * rec_bytes(L.kcap), 256);
    return L;
}

template <typename T, int KCAP>
uno_status launch_t(const VerifyArgs& a, const Layout& L, unsigned char* ws, cudaStream_t stream) {
    Params p{};
    p.a = a;
    p.S = L.S;
    p.rows_per_seq = L.rows_per_seq;
    p.row_counter = reinterpret_cast<uint32_t*>(ws + L.off_row_cnt);
    p.seq_counter = reinterpret_cast<uint32_t*>(ws + L.off_seq_cnt);
    p.seg_lists = reinterpret_cast<uint64_t*>(ws + L.off_lists);
    p.recs = ws + L.off_recs;
    p.kcap = KCAP;
    constexpr size_t smem = smem_bytes<T, KCAP>();
    static bool attr = false;
    if (!attr) {
        uno_status s = check_cuda(cudaFuncSetAttribute(rows_kernel<T, KCAP>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                                  "cudaFuncSetAttribute(verify top-k)");
        if (s != UNO_OK) return s;
        attr = true;
    }
    uno_status s = check_cuda(cudaMemsetAsync(ws, 0, L.off_lists, stream), "cudaMemsetAsync(verify counters)");
    if (s != UNO_OK) return s;
    int64_t grid = (int64_t)a.B * L.rows_per_seq * L.S;
    rows_kernel<T, KCAP><<<(unsigned)grid, Cfg<KCAP>::WARPS * 32, smem, stream>>>(p);
    return check_cuda(cudaGetLastError(), "launch(verify top-k)");
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
