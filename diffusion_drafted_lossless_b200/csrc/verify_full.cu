// verify_full.cu — lossless block verify without top-k: softmax over the whole vocabulary,
// optionally followed by top-p, with the top-p cut decided exactly.
//
// The verify rule is the top-k path's (LoopUno project page, "How it works" and "Training is
// self-distillation"; uno-qwen3-8B model card, "Evaluation protocol"); this path serves the
// unfiltered and the top-p-only sampler settings (the LoopUno runs use temperature 1.0 and
// top-p 0.95 without top-k).
//
// Work is split by block position. Item (b, i) owns the verifier row P_i and, for i >= 1, the
// drafter row Q_i of sequence b, and everything it decides depends on those rows alone:
//   i = 0:  x_0 (drawn from P_0 unless supplied) and P_0(x_0);
//   i >= 1: d_i (drawn from Q_i unless supplied), P_i(d_i), Q_i(d_i), the acceptance test
//           u * Q_i(d_i) < P_i(d_i), TV(P_i, Q_i), and a draw from the residual
//           normalise(max(0, P_i - Q_i)) with the position's resample uniform, which is the
//           correction token if i turns out to be the first rejection.
// Items write small records; assemble_kernel then takes each sequence's longest accepted
// prefix. Nothing waits on another item.
//
// Exact cut. With bf16 logits a row is fixed by how many tokens hold each 16-bit value, so
// every mass the verify needs is a sum over distinct values of count * exp(value / T - max),
// one fp64 exp per distinct value rather than one per token. pair_kernel counts the values
// whose magnitude lies within 2048 bf16 steps of the row's largest magnitude (both signs: all
// but tiny magnitudes); the few tokens below that band have their fp64 weights summed one by
// one. The cut is then the value at which the mass from the top first reaches top_p * S, and
// the ties at that value are kept lowest id first, as the sorted order (probability desc, id
// asc) keeps them. Sums run in fp64 in a different order from a sequential sum, so results
// agree with an exact evaluation up to fp64 rounding.
//
// pair_kernel (bf16, V a multiple of 8, 16-byte aligned logits): a thread-block cluster of CL
// CTAs owns an item at a time, CTA r holding elements [r L, (r + 1) L) of both rows in shared
// memory (one bulk copy per row, so each row crosses HBM once). Each CTA runs two teams of
// eight warps on alternate items, so one team computes while the other waits for its copy or
// for a cluster exchange. Per item and team: (1) the largest value and magnitude of each row;
// (2) the per-value counts; (3) each CTA sums the cluster's counts for its share of the values
// and their masses; (4) every CTA finds the same cut from the exchanged masses; (5) the CTA
// holding the boundary among the tied tokens finds it; (6) one pass over the rows sums, per
// warp part, the masses the draws walk (drafter survivors, verifier survivors, residual);
// (7) the CTAs that hold the drawn tokens find them. Exchanges are one-sided: each CTA stores
// its partials into every CTA's shared memory and arrives on that CTA's mbarrier.
// item_generic_kernel (any dtype and layout, and any item pair_kernel could not decide, e.g.
// a cut among the tiny-magnitude tokens): one CTA per item reading the rows from global
// memory in every pass, an fp64 exp per token, the cut by radix selection over the
// order-preserving 32-bit keys with fp64 masses per bin.
// Every wait is bounded; on timeout a kernel records UNO_ERR_TIMEOUT and stops.
#include <cuda_bf16.h>

#include <algorithm>
#include <climits>
#include <cstdlib>
#include <cstring>
#include <map>
#include <tuple>
#include <mutex>

#include "select.cuh"
#include "verify_common.cuh"

namespace uno {
namespace vfull {

// One record per item (b, i).
struct Rec {
    int32_t tok;    // x_0 (i = 0) or d_i
    int32_t res;    // residual draw (i >= 1), -1 at i = 0
    int32_t acc;    // acceptance of d_i (1 at i = 0)
    int32_t state;  // kDone, or kRedo for the generic kernel
    double p, q;    // P_i(tok), Q_i(tok) (q = 0 at i = 0)
    double tv;      // TV(P_i, Q_i) (0 at i = 0)
    double pad;
};
static_assert(sizeof(Rec) == 48, "record layout");
constexpr int32_t kDone = 1, kRedo = 2;

struct Params {
    const void* P;
    const void* Q;
    int B, K, V;
    double T;       // temperature
    double top_p;   // used when cut != 0
    int cut;        // top-p < 1
    int top_k;      // 0: off
    int need_p0;    // P_0(x_0) is an output: P_0 is needed even when x_0 is supplied
    const int32_t* drafts;
    const int32_t* pos0;
    const float* u;
    Rec* recs;
    uint32_t* status;
    unsigned long long* trace;  // UNO_VERIFY_TRACE: phase timestamps of cluster 0 (profiling aid), or NULL
};

// trace slot of (cluster rank, team, item number j < 32, event e < 16) in cluster 0
__device__ __forceinline__ void trace_mark(const Params& p, int cid, uint32_t crank, int team, uint32_t j, int e) {
    if (p.trace != nullptr && cid == 0 && j < 32u) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        p.trace[((crank * 2u + (uint32_t)team) * 32u + j) * 16u + (uint32_t)e] = t;
    }
}
constexpr size_t kTraceBytes = 16 * 2 * 32 * 16 * 8;

__device__ __forceinline__ bool pos0_given(const Params& p, int b) { return p.pos0 && p.pos0[b] >= 0; }
// an item with nothing to compute: x_0 supplied and P_0(x_0) not wanted
__device__ __forceinline__ bool trivial_item(const Params& p, int b, int i) {
    return i == 0 && pos0_given(p, b) && !p.need_p0;
}
__device__ __forceinline__ void write_trivial(const Params& p, int item, int b) {
    Rec r;
    r.tok = p.pos0[b];
    r.res = -1;
    r.acc = 1;
    r.state = kDone;
    r.p = 0.0;
    r.q = 0.0;
    r.tv = 0.0;
    r.pad = 0.0;
    p.recs[item] = r;
}

// =======================================================================================
// generic kernel: one CTA per item, rows read from global memory in every pass
// =======================================================================================
namespace gen {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

template <typename TL>
__device__ __forceinline__ float val(const TL* row, int v);
template <>
__device__ __forceinline__ float val<__nv_bfloat16>(const __nv_bfloat16* row, int v) {
    return __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(row)[v] << 16);
}
template <>
__device__ __forceinline__ float val<float>(const float* row, int v) {
    return row[v];
}

struct Row {
    double zmax;     // max of logit / T
    double Sk;       // surviving mass: sum over survivors of exp(logit / T - zmax)
    uint32_t kap_k;  // top-k: tokens with a larger order key survive it, and those with this key
    int th_k;        //   and an id below th_k (kap_k = 0: top-k off)
    uint32_t kap_p;  // top-p within the top-k survivors, the same way (kap_p = 0: top-p off)
    int th_p;
};

struct Shared {
    double red[kWarps];
    float fred[kWarps];
    int ired[kWarps];
    double binm[256];
    unsigned binc[256];
    int sel, sel2, mode;
    double dsel;
};

__device__ double block_sum(double v, Shared& s) {
    v = warp_sum_f64(v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) s.red[threadIdx.x >> 5] = v;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < kWarps; ++w) t += s.red[w];  // same order in every thread
    return t;
}

__device__ float block_max(float v, Shared& s) {
    v = warp_max(v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) s.fred[threadIdx.x >> 5] = v;
    __syncthreads();
    float t = -INFINITY;
    for (int w = 0; w < kWarps; ++w) t = fmaxf(t, s.fred[w]);
    return t;
}

__device__ __forceinline__ bool in_topk(const Row& r, uint32_t key, int v) {
    return key > r.kap_k || (key == r.kap_k && v < r.th_k);
}
__device__ __forceinline__ bool survives(const Row& r, uint32_t key, int v) {
    return in_topk(r, key, v) && (key > r.kap_p || (key == r.kap_p && v < r.th_p));
}

// Radix selection over the order-preserving 32-bit keys of the tokens `in(v, key)`, 8 bits at
// a time from the top: the largest key at which the running total of amount(v, x) from the
// top reaches `target`. Returns the key, the total of the tokens strictly above it and how
// many tokens hold it. If rounding leaves the target unmet, the smallest key present.
template <typename TL, typename In, typename Amt>
__device__ void radix_select(const TL* row, int V, In in, Amt amount, double target, Shared& s, uint32_t& key,
                             double& above, unsigned& count) {
    const int tid = threadIdx.x;
    uint32_t prefix = 0u, mask = 0u;
    double cb = 0.0;
    unsigned cnt = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int j = tid; j < 256; j += kThreads) {
            s.binm[j] = 0.0;
            s.binc[j] = 0u;
        }
        __syncthreads();
        for (int v = tid; v < V; v += kThreads) {
            const float x = val(row, v);
            const uint32_t k = float_key(x);
            if ((k & mask) == prefix && in(v, k)) {
                const int bin = (int)((k >> shift) & 0xFFu);
                atomicAdd(&s.binm[bin], amount(v, x));
                atomicAdd(&s.binc[bin], 1u);
            }
        }
        __syncthreads();
        if (tid == 0) {
            double c = cb;
            int bin = -1;
            for (int j = 255; j >= 0; --j) {
                if (s.binc[j] == 0u) continue;
                if (c + s.binm[j] >= target) {
                    bin = j;
                    break;
                }
                c += s.binm[j];
            }
            if (bin < 0) {
                for (int j = 0; j < 256 && bin < 0; ++j)
                    if (s.binc[j]) bin = j;
                c = cb;
                for (int j = 255; j > bin; --j) c += s.binm[j];
            }
            s.sel = bin;
            s.dsel = c;
        }
        __syncthreads();
        const int bin = s.sel;
        cb = s.dsel;
        cnt = s.binc[bin];
        prefix |= (uint32_t)bin << shift;
        mask |= 0xFFu << shift;
        __syncthreads();
    }
    key = prefix;
    above = cb;
    count = cnt;
}

// The id of the t-th (1-based, id order) token with `in(v, key)` and this key.
template <typename TL, typename In>
__device__ int tie_id(const TL* row, int V, In in, uint32_t key, long long t, Shared& s) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int seg = (V + kWarps - 1) / kWarps;
    const int v0 = warp * seg, v1 = min(V, v0 + seg);
    int c = 0;
    for (int v = v0 + lane; v < v1; v += 32) {
        const uint32_t k = float_key(val(row, v));
        c += (k == key && in(v, k));
    }
    c = warp_sum(c);
    __syncthreads();
    if (lane == 0) s.ired[warp] = c;
    __syncthreads();
    if (tid == 0) {
        long long before = 0;
        int w = 0;
        for (; w < kWarps; ++w) {
            if (before + s.ired[w] >= t) break;
            before += s.ired[w];
        }
        s.sel = w;
        s.sel2 = (int)(t - before);  // rank within that warp's part (1-based)
    }
    __syncthreads();
    if (warp == s.sel) {
        int need = s.sel2, found = -1;
        for (int base = v0; base < v1 && found < 0; base += 32) {
            const int v = base + lane;
            bool hit = false;
            if (v < v1) {
                const uint32_t k = float_key(val(row, v));
                hit = k == key && in(v, k);
            }
            const unsigned bal = __ballot_sync(kFullMask, hit);
            const int nb = __popc(bal);
            if (nb >= need) {
                unsigned b = bal;
                for (int q = 1; q < need; ++q) b &= b - 1;
                found = base + __ffs(b) - 1;
            }
            need -= nb;
        }
        if (lane == 0) s.sel = found;
    }
    __syncthreads();
    const int id = s.sel;
    __syncthreads();
    return id;
}

// Row statistics, the top-k cut and the top-p cut of one row.
template <typename TL>
__device__ void row_stats(const TL* row, const Params& p, Shared& s, Row& out) {
    const int V = p.V, tid = threadIdx.x;
    float m = -INFINITY;
    for (int v = tid; v < V; v += kThreads) m = fmaxf(m, val(row, v));
    m = block_max(m, s);
    Row r;
    r.zmax = (double)m / p.T;  // the largest logit survives both cuts
    r.kap_k = 0u;
    r.th_k = INT_MAX;
    r.kap_p = 0u;
    r.th_p = INT_MAX;
    const double zmax = r.zmax, T = p.T;
    auto all = [&](int, uint32_t) { return true; };
    if (p.top_k > 0) {
        // the k largest values, ties to the lower id
        uint32_t key;
        double above;
        unsigned cnt;
        radix_select(row, V, all, [](int, float) { return 1.0; }, (double)p.top_k, s, key, above, cnt);
        long long t = (long long)p.top_k - (long long)above;
        if (t < 1) t = 1;
        if (t > (long long)cnt) t = cnt;
        r.kap_k = key;
        if (t < (long long)cnt) r.th_k = tie_id(row, V, all, key, t, s) + 1;
    }
    const Row rk = r;
    auto in_k = [&](int v, uint32_t k) { return in_topk(rk, k, v); };
    double acc = 0.0;
    for (int v = tid; v < V; v += kThreads) {
        const float x = val(row, v);
        if (in_topk(r, float_key(x), v)) acc += exp((double)x / T - zmax);
    }
    const double S = block_sum(acc, s);
    r.Sk = S;
    if (p.cut) {
        // the mass from the top first reaches top_p * S: the fewest (at least one) of the
        // tokens at that value, lowest ids first, that bring it there
        const double target = p.top_p * S;
        uint32_t key;
        double cb;
        unsigned cnt;
        radix_select(row, V, in_k, [&](int, float x) { return exp((double)x / T - zmax); }, target, s, key, cb, cnt);
        const double wk = exp((double)key_float(key) / T - zmax);
        long long t = (long long)ceil((target - cb) / wk);
        if (t < 1) t = 1;
        if (t > (long long)cnt) t = cnt;
        while (t > 1 && cb + (double)(t - 1) * wk >= target) --t;
        while (t < (long long)cnt && cb + (double)t * wk < target) ++t;
        r.kap_p = key;
        r.Sk = cb + (double)t * wk;
        if (t < (long long)cnt) r.th_p = tie_id(row, V, in_k, key, t, s) + 1;
    }
    out = r;
}

template <typename TL>
__device__ __forceinline__ double kept_weight(const TL* row, const Row& r, const Params& p, int v) {
    const float x = val(row, v);
    return survives(r, float_key(x), v) ? exp((double)x / p.T - r.zmax) : 0.0;
}

// Inverse-CDF draw over ascending ids: the first id whose cumulative weight exceeds target;
// if rounding leaves no crossing, the last id with positive weight. -1 if no weight at all.
template <typename F>
__device__ int draw(int V, double target, F wfn, Shared& s) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int seg = (V + kWarps - 1) / kWarps;
    const int v0 = warp * seg, v1 = min(V, v0 + seg);
    double part = 0.0;
    for (int v = v0 + lane; v < v1; v += 32) part += wfn(v);
    part = warp_sum_f64(part);
    __syncthreads();
    if (lane == 0) s.red[warp] = part;
    __syncthreads();
    if (tid == 0) {
        double c = 0.0, clast = 0.0;
        int wd = -1, last = -1;
        for (int w = 0; w < kWarps; ++w) {
            if (!(s.red[w] > 0.0)) continue;
            last = w;
            clast = c;
            if (c + s.red[w] > target) {
                wd = w;
                break;
            }
            c += s.red[w];
        }
        s.mode = wd < 0;
        s.sel = wd < 0 ? last : wd;
        s.dsel = wd < 0 ? clast : c;
    }
    __syncthreads();
    const int wsel = s.sel;
    if (wsel < 0) return -1;
    if (warp == wsel) {
        const bool last_mode = s.mode;
        double carry = s.dsel;
        int res = -1, lastpos = -1;
        const int stop = last_mode ? v1 : V;
        for (int base = v0; base < stop; base += 32) {
            const int v = base + lane;
            const double x = v < stop ? wfn(v) : 0.0;
            const double incl = warp_scan_f64(x, lane);
            const unsigned hit = last_mode ? 0u : __ballot_sync(kFullMask, x > 0.0 && carry + incl > target);
            if (hit) {
                res = base + __ffs(hit) - 1;
                break;
            }
            const unsigned pos = __ballot_sync(kFullMask, x > 0.0);
            if (pos) lastpos = base + 31 - __clz(pos);
            carry += __shfl_sync(kFullMask, incl, 31);
        }
        if (lane == 0) s.sel2 = res >= 0 ? res : lastpos;
    }
    __syncthreads();
    const int out = s.sel2;
    __syncthreads();
    return out;
}

template <typename TL>
__global__ void __launch_bounds__(kThreads) item_kernel(Params p, int only_redo) {
    __shared__ Shared s;
    const int n_items = p.B * p.K;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        if (only_redo && p.recs[item].state == kDone) continue;
        const int b = item / p.K, i = item % p.K;
        if (trivial_item(p, b, i)) {
            if (threadIdx.x == 0) write_trivial(p, item, b);
            continue;
        }
        const TL* P = static_cast<const TL*>(p.P) + (int64_t)item * p.V;
        const float* u = p.u + (int64_t)item * 3;
        Row rp;
        row_stats(P, p, s, rp);
        auto wP = [&](int v) { return kept_weight(P, rp, p, v); };
        if (i == 0) {
            const int x0 = pos0_given(p, b) ? p.pos0[b] : draw(p.V, (double)u[0] * rp.Sk, wP, s);
            const double px = (x0 >= 0 && x0 < p.V) ? wP(x0) / rp.Sk : 0.0;
            if (threadIdx.x == 0) {
                Rec r;
                r.tok = x0;
                r.res = -1;
                r.acc = 1;
                r.state = kDone;
                r.p = px;
                r.q = 0.0;
                r.tv = 0.0;
                r.pad = 0.0;
                p.recs[item] = r;
            }
            __syncthreads();
            continue;
        }
        const TL* Q = static_cast<const TL*>(p.Q) + (int64_t)item * p.V;
        Row rq;
        row_stats(Q, p, s, rq);
        auto wQ = [&](int v) { return kept_weight(Q, rq, p, v); };
        const int d = p.drafts ? p.drafts[item] : draw(p.V, (double)u[0] * rq.Sk, wQ, s);
        const bool in = d >= 0 && d < p.V;
        const double pd = in ? wP(d) / rp.Sk : 0.0, qd = in ? wQ(d) / rq.Sk : 0.0;
        const int acc = (double)u[1] * qd < pd;
        auto resid = [&](int v) {
            const double dl = wP(v) / rp.Sk - wQ(v) / rq.Sk;
            return dl > 0.0 ? dl : 0.0;
        };
        double rs = 0.0, ts = 0.0;
        for (int v = threadIdx.x; v < p.V; v += kThreads) {
            const double dl = wP(v) / rp.Sk - wQ(v) / rq.Sk;
            if (dl > 0.0) rs += dl;
            ts += fabs(dl);
        }
        const double R = block_sum(rs, s);
        const double tv = 0.5 * block_sum(ts, s);
        const int res = R > 0.0 ? draw(p.V, (double)u[2] * R, resid, s) : draw(p.V, (double)u[2] * rp.Sk, wP, s);
        if (threadIdx.x == 0) {
            Rec r;
            r.tok = d;
            r.res = res;
            r.acc = acc;
            r.state = kDone;
            r.p = pd;
            r.q = qd;
            r.tv = tv;
            r.pad = 0.0;
            p.recs[item] = r;
        }
        __syncthreads();
    }
}

}  // namespace gen

// =======================================================================================
// pair_kernel: one cluster per item, the rows' slices resident in shared memory
// =======================================================================================
namespace pk {

constexpr int kTeams = 2;
constexpr int kTeamWarps = 8;
constexpr int kTeamThreads = kTeamWarps * 32;
constexpr int kThreads = kTeams * kTeamThreads;
constexpr int kWords = 2048;   // full mode: counted magnitudes per row, a_top - d for d < kWords
constexpr int kWinK = 256;     // top-k mode: counted values per row, the 256 largest bf16 values from the max down
constexpr int kLut = 512;      // tabulated survivor weights per row (positive values, d < kLut)
constexpr int kMaxCL = 16;
constexpr int kMaxTopK = 256;  // top-k mode: largest k

// shared-memory layout of one team (byte offsets from the team's base); host and device
struct Layout {
    int CL;          // CTAs per cluster
    int L;           // slice length in elements (a multiple of 8)
    int hw;          // histogram words per row (kWords, or kWinK in top-k mode)
    int OW;          // histogram words owned by each CTA: hw / CL
    int KL;          // top-k mode: survivor list capacity per row (a power of two >= k)
    uint32_t off_hist, off_own, off_lut, off_list, off_x1, off_x2, off_x3, off_misc, team_bytes;
};

struct RowStat {
    double zmax;      // max of logit / T
    double S;         // total mass
    double Sk;        // surviving mass
    double wk;        // weight of the cut value
    float M;          // max value
    uint32_t atop;    // largest magnitude (bf16 bits without the sign)
    uint32_t kM;      // order key of the max value (top-k mode)
    uint32_t kbits;   // bf16 bits of the cut value
    int kd, kneg;     // cut value as (word d, sign)
    int tkeep;        // ties kept, cluster-wide
    int theta;        // ties with id < theta survive (this CTA's slice)
    int lut_n;        // lut holds the weights of positive values with d < lut_n
};

struct TeamShared {
    RowStat rs[2];
    double wpart[kTeamWarps][3];  // per-warp part masses: draw row, verifier survivors, residual
    double dred[kTeamWarps][6];
    uint32_t ured[kTeamWarps][4];
    int ipart[kTeamWarps];
    int redo, abort_;
    int sel, sel2, mode;
    double dsel;
    unsigned lcnt[2];   // top-k mode: survivors appended to this CTA's lists (when it is the head)
    int np[2];          // top-k mode: survivors of the top-p cut
    double Z[2];        // top-k mode: their mass
};

// ---- PTX wrappers for the cluster ----
__device__ __forceinline__ uint32_t ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t mapa(const void* local, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
    return a;
}
__device__ __forceinline__ void st_remote_f64(uint32_t addr, double v) {
    asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(addr), "d"(v) : "memory");
}
__device__ __forceinline__ void st_remote_u64(uint32_t addr, unsigned long long v) {
    asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_remote_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t atom_remote_add(uint32_t addr, uint32_t v) {
    uint32_t old;
    asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ uint2 ld_remote_v2(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared::cluster.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void arrive_remote(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void fence_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }
__device__ __forceinline__ bool wait_cluster(uint64_t* bar, uint32_t parity) {
    for (uint32_t k = 0; k < kWaitLimit; ++k) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred q;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 q, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    return false;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void team_sync(int team) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "n"(kTeamThreads) : "memory");
}

__device__ __forceinline__ float bf(uint32_t h16) { return __uint_as_float(h16 << 16); }

// weight of a bf16 value relative to the row's max: exp(v / T - zmax)
__device__ __forceinline__ double wexp(uint32_t h16, const RowStat& r, double T) {
    return exp((double)bf(h16) / T - r.zmax);
}

// value of histogram word d with the given sign
__device__ __forceinline__ uint32_t word_bits(const RowStat& r, int d, int neg) {
    return (r.atop - (uint32_t)d) | (neg ? 0x8000u : 0u);
}

// survivor weight of one element (value bits h16, token id v), 0 if it does not survive
__device__ __forceinline__ double surv_weight(uint32_t h16, int v, const RowStat& r, const double* lut, double T,
                                              int cut) {
    const float x = bf(h16);
    if (cut) {
        const float kx = bf(r.kbits);
        if (x < kx || (x == kx && v >= r.theta) || x != x) return 0.0;
    }
    const uint32_t d = r.atop - h16;  // positive values only (sign bit clear)
    if (!(h16 & 0x8000u) && d < (uint32_t)r.lut_n) return lut[d];
    if (!(fabsf(x) < INFINITY)) return 0.0;
    return exp((double)x / T - r.zmax);
}

// the element's 16 bits from a shared-memory slice
__device__ __forceinline__ uint32_t elem(const uint16_t* buf, int e) { return buf[e]; }

// 16-bit order key of a bf16 value (larger value, larger key) and back
__device__ __forceinline__ uint32_t key16(uint32_t h) { return (h & 0x8000u) ? (~h & 0xFFFFu) : (h | 0x8000u); }
__device__ __forceinline__ uint32_t bits16(uint32_t k) { return (k & 0x8000u) ? (k & 0x7FFFu) : (~k & 0xFFFFu); }
__device__ __forceinline__ __nv_bfloat162 as_bf2(uint32_t w) { return *reinterpret_cast<const __nv_bfloat162*>(&w); }

// TOPK = false: full-vocabulary mode (top-p over the whole row, or no cut). TOPK = true:
// top-k (k <= kMaxTopK), then top-p over the k survivors.
template <bool TOPK>
__global__ void __launch_bounds__(kThreads, 1) pair_kernel(Params p, Layout Ly) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bars[kTeams][5];

    const int team = threadIdx.x / kTeamThreads, tt = threadIdx.x % kTeamThreads;
    const int tw = tt >> 5, lane = tt & 31;
    const int CL = Ly.CL;
    const uint32_t crank = ctarank();
    const int cid = blockIdx.x / CL, NC = gridDim.x / CL;
    const int n_items = p.B * p.K;
    const double T = p.T;

    unsigned char* base = smem + (size_t)team * Ly.team_bytes;
    uint16_t* bufs[2] = {reinterpret_cast<uint16_t*>(base), reinterpret_cast<uint16_t*>(base) + Ly.L};
    uint32_t* hist = reinterpret_cast<uint32_t*>(base + Ly.off_hist);      // [2][hw]
    uint2* own = reinterpret_cast<uint2*>(base + Ly.off_own);              // [2][OW]: (+count, -count)
    double* lut = reinterpret_cast<double*>(base + Ly.off_lut);            // [2][kLut] (full mode)
    uint64_t* list = reinterpret_cast<uint64_t*>(base + Ly.off_list);      // top-k mode: [2][KL] survivors,
    uint64_t* ltmp = list + 2 * Ly.KL;                                     //   [2][KL] scratch,
    double* lw = reinterpret_cast<double*>(ltmp + 2 * Ly.KL);              //   [2][KL] weights,
    int32_t* lid = reinterpret_cast<int32_t*>(lw + 2 * Ly.KL);             //   [2][KL] ids
    unsigned long long* x1 = reinterpret_cast<unsigned long long*>(base + Ly.off_x1);  // [kMaxCL]
    double* x2 = reinterpret_cast<double*>(base + Ly.off_x2);              // [kMaxCL][6]
    double* x3 = reinterpret_cast<double*>(base + Ly.off_x3);              // [kMaxCL][3]
    TeamShared& ts = *reinterpret_cast<TeamShared*>(base + Ly.off_misc);
    uint64_t* full = &bars[team][0];
    uint64_t* xb1 = &bars[team][1];
    uint64_t* xb2a = &bars[team][2];
    uint64_t* xb2b = &bars[team][3];
    uint64_t* xb3 = &bars[team][4];

    if (tt == 0) {
        mbar_init(full, 1);
        mbar_init(xb1, CL);
        mbar_init(xb2a, CL);
        mbar_init(xb2b, CL);
        mbar_init(xb3, CL);
        ts.abort_ = 0;
        fence_mbar_init();
    }
    __syncthreads();
    cluster_sync_all();  // every CTA's barriers exist before any remote arrive

    const int lo = (int)crank * Ly.L;
    const int n = max(0, min(Ly.L, p.V - lo));
    const int nvec = n >> 3;
    const int pv = (nvec + kTeamWarps - 1) / kTeamWarps;  // vectors per warp part
    const int wv0 = min(nvec, tw * pv), wv1 = min(nvec, wv0 + pv);
    const int step = kTeams * NC;

    // the leader (tt == 0) issues the bulk copies of the team's next item
    int issued = -1, inflight = 0;
    auto needs_rows = [&](int it) { return !trivial_item(p, it / p.K, it % p.K); };
    auto issue = [&](int it) {
        const int i = it % p.K;
        const int nrows = i > 0 ? 2 : 1;
        if (n > 0) {
            mbar_arrive_expect_tx(full, (uint32_t)(n * 2 * nrows));
            const __nv_bfloat16* Prow = static_cast<const __nv_bfloat16*>(p.P) + (int64_t)it * p.V + lo;
            bulk_g2s(bufs[0], Prow, (uint32_t)(n * 2), full);
            if (i > 0) {
                const __nv_bfloat16* Qrow = static_cast<const __nv_bfloat16*>(p.Q) + (int64_t)it * p.V + lo;
                bulk_g2s(bufs[1], Qrow, (uint32_t)(n * 2), full);
            }
        } else {
            mbar_arrive(full);
        }
        issued = it;
        inflight = 1;
    };

    uint32_t xph = 0, lph = 0;  // phases of the exchange barriers and of the buffer barrier
    uint32_t hph = 0;           // top-k mode: items this CTA has been the head of (its xb3 phase)
    for (int item = cid + team * NC; item < n_items; item += step) {
        const int b = item / p.K, i = item % p.K;
        if (!needs_rows(item)) {
            if (crank == 0 && tt == 0) write_trivial(p, item, b);
            continue;
        }
        const int nrows = i > 0 ? 2 : 1;
        if (tt == 0) trace_mark(p, cid, crank, team, xph, 0);
        if (tt == 0 && issued != item) issue(item);
        if (tw == 0) {
            const bool ok = mbar_wait(full, lph & 1);
            if (!ok && lane == 0) ts.abort_ = 1;
        }
        ++lph;
        if (tt == 0) inflight = 0;
        team_sync(team);
        if (ts.abort_) break;
        if (tt == 0) trace_mark(p, cid, crank, team, xph, 1);

        // ---- (1) largest value and magnitude of each row slice ----
        {
            __nv_bfloat162 mx[2], mg[2];
            for (int r = 0; r < 2; ++r) {
                mx[r] = __floats2bfloat162_rn(-INFINITY, -INFINITY);
                mg[r] = __floats2bfloat162_rn(0.f, 0.f);
            }
            for (int r = 0; r < nrows; ++r) {
                const uint4* v4 = reinterpret_cast<const uint4*>(bufs[r]);
                for (int j = tt; j < nvec; j += kTeamThreads) {
                    const uint4 v = v4[j];
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        mx[r] = __hmax2(mx[r], *reinterpret_cast<const __nv_bfloat162*>(&w[q]));
                        if (!TOPK) {  // the largest magnitude sets the counted band (full mode)
                            const uint32_t a = w[q] & 0x7FFF7FFFu;
                            mg[r] = __hmax2(mg[r], *reinterpret_cast<const __nv_bfloat162*>(&a));
                        }
                    }
                }
            }
            float fm[2], fa[2];
            for (int r = 0; r < 2; ++r) {
                fm[r] = warp_max(fmaxf(__low2float(mx[r]), __high2float(mx[r])));
                fa[r] = warp_max(fmaxf(__low2float(mg[r]), __high2float(mg[r])));
            }
            if (lane == 0) {
                ts.dred[tw][0] = fm[0];
                ts.dred[tw][1] = fa[0];
                ts.dred[tw][2] = fm[1];
                ts.dred[tw][3] = fa[1];
            }
            // clear the counts (nobody reads them before the exchange below)
            for (int j = tt; j < 2 * Ly.hw; j += kTeamThreads) hist[j] = 0u;
            if (TOPK && tt < 2 && (int)crank == item % CL) ts.lcnt[tt] = 0u;
            team_sync(team);
            if (tw == 0) {
                float m0 = -INFINITY, a0 = 0.f, m1 = -INFINITY, a1 = 0.f;
                for (int w = 0; w < kTeamWarps; ++w) {
                    m0 = fmaxf(m0, (float)ts.dred[w][0]);
                    a0 = fmaxf(a0, (float)ts.dred[w][1]);
                    m1 = fmaxf(m1, (float)ts.dred[w][2]);
                    a1 = fmaxf(a1, (float)ts.dred[w][3]);
                }
                const unsigned long long pk = (unsigned long long)(__float_as_uint(m0) >> 16) |
                                              ((unsigned long long)(__float_as_uint(a0) >> 16) << 16) |
                                              ((unsigned long long)(__float_as_uint(m1) >> 16) << 32) |
                                              ((unsigned long long)(__float_as_uint(a1) >> 16) << 48);
                if (lane < CL) {
                    st_remote_u64(mapa(&x1[crank], (uint32_t)lane), pk);
                    arrive_remote(mapa(xb1, (uint32_t)lane));
                }
                const bool ok = wait_cluster(xb1, xph & 1);
                if (!ok && lane == 0) ts.abort_ = 1;
                if (lane < 2) {
                    float M = -INFINITY;
                    uint32_t A = 0;
                    for (int r = 0; r < CL; ++r) {
                        const unsigned long long v = x1[r] >> (32 * lane);
                        M = fmaxf(M, bf((uint32_t)(v & 0xFFFFu)));
                        A = max(A, (uint32_t)((v >> 16) & 0xFFFFu));
                    }
                    RowStat& rs = ts.rs[lane];
                    if (M == 0.f) M = 0.f;  // +0, at or above every zero in key order
                    rs.M = M;
                    rs.atop = A;
                    rs.kM = key16(__float_as_uint(M) >> 16);
                    rs.zmax = (double)M / T;
                }
            }
            team_sync(team);
            if (ts.abort_) break;
        }

        if (tt == 0) trace_mark(p, cid, crank, team, xph, 2);
        // ---- (2) counts per value: full mode, every magnitude within kWords steps of the
        //      largest (the rest weighed one by one); top-k mode, the kWinK largest values ----
        if constexpr (TOPK) {
            for (int r = 0; r < nrows; ++r) {
                const uint32_t kM = ts.rs[r].kM;
                const uint32_t kf = kM >= (uint32_t)(kWinK - 1) ? kM - (uint32_t)(kWinK - 1) : 0u;
                const uint32_t hf = bits16(kf);
                const __nv_bfloat162 f2 = as_bf2(hf | (hf << 16));
                uint32_t* h = hist + r * Ly.hw;
                const uint4* v4 = reinterpret_cast<const uint4*>(bufs[r]);
                for (int j = tt; j < nvec; j += kTeamThreads) {
                    const uint4 v = v4[j];
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t m = __hge2_mask(as_bf2(w[q]), f2);
                        if (m) {
                            // (-0 passes a +0 floor but lies below it in key order: d checked)
                            const uint32_t dl = kM - key16(w[q] & 0xFFFFu), dh = kM - key16(w[q] >> 16);
                            if ((m & 0xFFFFu) && dl < (uint32_t)kWinK) atomicAdd(&h[dl], 1u);
                            if ((m >> 16) && dh < (uint32_t)kWinK) atomicAdd(&h[dh], 1u);
                        }
                    }
                }
            }
            if (lane == 0) {
                ts.dred[tw][4] = 0.0;
                ts.dred[tw][5] = 0.0;
            }
            team_sync(team);
            if (tw == 0) {
                fence_cluster();
                if (lane < CL) arrive_remote(mapa(xb2a, (uint32_t)lane));
                const bool ok = wait_cluster(xb2a, xph & 1);
                if (!ok && lane == 0) ts.abort_ = 1;
            }
            team_sync(team);
            if (ts.abort_) break;
        } else {
            double below[2] = {0.0, 0.0};  // fp64 weights of the tokens under the counted band
            for (int r = 0; r < nrows; ++r) {
                const RowStat rs = ts.rs[r];
                uint32_t* h = hist + r * Ly.hw;
                const uint4* v4 = reinterpret_cast<const uint4*>(bufs[r]);
                for (int j = tt; j < nvec; j += kTeamThreads) {
                    const uint4 v = v4[j];
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t hl = w[q] & 0xFFFFu, hh = w[q] >> 16;
                        const uint32_t dl = rs.atop - (hl & 0x7FFFu), dh = rs.atop - (hh & 0x7FFFu);
                        if (dl < (uint32_t)kWords) atomicAdd(&h[dl], (hl & 0x8000u) ? 0x10000u : 1u);
                        else if (fabsf(bf(hl)) < INFINITY) below[r] += wexp(hl, rs, T);
                        if (dh < (uint32_t)kWords) atomicAdd(&h[dh], (hh & 0x8000u) ? 0x10000u : 1u);
                        else if (fabsf(bf(hh)) < INFINITY) below[r] += wexp(hh, rs, T);
                    }
                }
            }
            below[0] = warp_sum_f64(below[0]);
            below[1] = warp_sum_f64(below[1]);
            if (lane == 0) {
                ts.dred[tw][4] = below[0];
                ts.dred[tw][5] = below[1];
            }
            team_sync(team);
            if (tw == 0) {
                fence_cluster();
                if (lane < CL) arrive_remote(mapa(xb2a, (uint32_t)lane));
                const bool ok = wait_cluster(xb2a, xph & 1);
                if (!ok && lane == 0) ts.abort_ = 1;
            }
            team_sync(team);
            if (ts.abort_) break;
        }

        if (tt == 0) trace_mark(p, cid, crank, team, xph, 3);
        // ---- (3) this CTA's share of the values: cluster-wide counts, and (full mode) their
        //      masses ----
        {
            const int w0 = (int)crank * Ly.OW;
            double pm[2] = {0.0, 0.0}, nm[2] = {0.0, 0.0};
            for (int r = 0; r < nrows; ++r) {
                const RowStat rs = ts.rs[r];
                for (int k = tt; k < Ly.OW; k += kTeamThreads) {
                    const int d = w0 + k;
                    uint32_t cp = 0, cn = 0;
                    for (int q = 0; q < CL; ++q) {
                        const uint32_t c = ld_remote_u32(mapa(&hist[r * Ly.hw + d], (uint32_t)q));
                        if constexpr (TOPK) {
                            cp += c;
                        } else {
                            cp += c & 0xFFFFu;
                            cn += c >> 16;
                        }
                    }
                    own[r * Ly.OW + k] = make_uint2(cp, cn);
                    if constexpr (TOPK) {
                        pm[r] += (double)cp;
                    } else {
                        if (cp) pm[r] += (double)cp * wexp(word_bits(rs, d, 0), rs, T);
                        if (cn) nm[r] += (double)cn * wexp(word_bits(rs, d, 1), rs, T);
                    }
                }
            }
            for (int r = 0; r < 2; ++r) {
                pm[r] = warp_sum_f64(pm[r]);
                nm[r] = warp_sum_f64(nm[r]);
            }
            team_sync(team);  // dred[.][0..3] of step (1) are no longer read
            if (lane == 0) {
                ts.dred[tw][0] = pm[0];
                ts.dred[tw][1] = nm[0];
                ts.dred[tw][2] = pm[1];
                ts.dred[tw][3] = nm[1];
            }
            team_sync(team);
            if (tw == 0) {
                double v6[6] = {0, 0, 0, 0, 0, 0};
                for (int w = 0; w < kTeamWarps; ++w) {
                    v6[0] += ts.dred[w][0];
                    v6[1] += ts.dred[w][1];
                    v6[2] += ts.dred[w][4];
                    v6[3] += ts.dred[w][2];
                    v6[4] += ts.dred[w][3];
                    v6[5] += ts.dred[w][5];
                }
                if (lane < CL) {
                    const uint32_t slot = mapa(&x2[crank * 6], (uint32_t)lane);
                    for (int k = 0; k < 6; ++k) st_remote_f64(slot + 8u * k, v6[k]);
                    arrive_remote(mapa(xb2b, (uint32_t)lane));
                }
                const bool ok = wait_cluster(xb2b, xph & 1);
                if (!ok && lane == 0) ts.abort_ = 1;
            }
            team_sync(team);
            if (ts.abort_) break;
        }

        if (tt == 0) trace_mark(p, cid, crank, team, xph, 4);
        // ---- (4) the cut of each row, identical in every CTA ----
        if (TOPK && tw < nrows) {  // warp r finds the k-th largest value of row r
            const int r = tw;
            RowStat& rs = ts.rs[r];
            rs.S = 0.0;
            rs.Sk = 0.0;
            rs.kbits = 0xFF80u;
            rs.kd = -1;
            rs.kneg = 0;
            rs.tkeep = 0;
            rs.theta = INT_MAX;
            const double target = (double)p.top_k;
            double c = 0.0;
            int part = -1;
            for (int q = 0; q < CL && part < 0; ++q) {
                const double m = x2[q * 6 + 3 * r];
                if (m > 0.0 && c + m >= target) part = q;
                else c += m;
            }
            int redo = part < 0;  // fewer than k tokens among the counted values
            if (!redo) {
                const int w0 = part * Ly.OW;
                int kd = -1;
                double cb = 0.0;
                for (int k0 = 0; k0 < Ly.OW && kd < 0; k0 += 32) {
                    const int k = k0 + lane;
                    const uint32_t cnt = k < Ly.OW ? ld_remote_v2(mapa(&own[r * Ly.OW + k], (uint32_t)part)).x : 0u;
                    const double m = (double)cnt;
                    const double incl = warp_scan_f64(m, lane);
                    const unsigned hit = __ballot_sync(kFullMask, cnt > 0 && c + incl >= target);
                    if (hit) {
                        const int src = __ffs(hit) - 1;
                        kd = w0 + k0 + src;
                        cb = c + __shfl_sync(kFullMask, incl - m, src);
                    }
                    c += __shfl_sync(kFullMask, incl, 31);
                }
                if (kd < 0) {
                    redo = 1;
                } else {
                    rs.kd = kd;
                    rs.kbits = bits16(rs.kM - (uint32_t)kd);
                    rs.tkeep = (int)(target - cb);  // the tokens at the k-th value that are kept
                    // +0 and -0 are one value but two keys: leave such a cut to the generic kernel
                    if ((rs.kbits & 0x7FFFu) == 0u) redo = 1;
                }
            }
            if (lane == 0) ts.dred[r][0] = redo;
        }
        if (!TOPK && tw < nrows) {  // warp r decides row r
            const int r = tw;
            RowStat& rs = ts.rs[r];
            double S = 0.0;
            for (int q = 0; q < CL; ++q) S += x2[q * 6 + 3 * r + 0];
            for (int q = 0; q < CL; ++q) S += x2[q * 6 + 3 * r + 2];
            for (int q = 0; q < CL; ++q) S += x2[q * 6 + 3 * r + 1];
            rs.S = S;
            rs.Sk = S;
            rs.kbits = 0xFF80u;  // -inf: no cut
            rs.kd = -1;
            rs.kneg = 0;
            rs.tkeep = 0;
            rs.theta = INT_MAX;
            int redo = !(S > 0.0) || !(S < INFINITY);
            if (p.cut && !redo) {
                const double target = p.top_p * S;
                // value order: positive parts of CTAs 0..CL-1, the uncounted band, negative
                // parts of CTAs CL-1..0
                double c = 0.0;
                int part = -1, neg = 0;
                for (int q = 0; q < CL && part < 0; ++q) {
                    const double m = x2[q * 6 + 3 * r + 0];
                    if (m > 0.0 && c + m >= target) part = q;
                    else c += m;
                }
                if (part < 0) {
                    double zb = 0.0;
                    for (int q = 0; q < CL; ++q) zb += x2[q * 6 + 3 * r + 2];
                    if (zb > 0.0 && c + zb >= target) redo = 1;  // the cut lies among uncounted tokens
                    c += zb;
                    for (int q = CL - 1; q >= 0 && part < 0 && !redo; --q) {
                        const double m = x2[q * 6 + 3 * r + 1];
                        if (m > 0.0 && c + m >= target) {
                            part = q;
                            neg = 1;
                        } else {
                            c += m;
                        }
                    }
                    if (part < 0) redo = 1;  // rounding left the target unmet
                }
                if (!redo) {
                    // scan the owner's words in value order
                    const int w0 = part * Ly.OW;
                    int kd = -1;
                    uint32_t kc = 0;
                    double cb = 0.0, wk = 0.0;
                    for (int k0 = 0; k0 < Ly.OW && kd < 0; k0 += 32) {
                        const int k = k0 + lane;
                        const int kk = neg ? Ly.OW - 1 - k : k;
                        uint32_t cnt = 0;
                        double w = 0.0;
                        if (k < Ly.OW) {
                            const uint2 c2 = ld_remote_v2(mapa(&own[r * Ly.OW + kk], (uint32_t)part));
                            cnt = neg ? c2.y : c2.x;
                            if (cnt) w = wexp(word_bits(rs, w0 + kk, neg), rs, T);
                        }
                        const double m = (double)cnt * w;
                        const double incl = warp_scan_f64(m, lane);
                        const unsigned hit = __ballot_sync(kFullMask, cnt > 0 && c + incl >= target);
                        if (hit) {
                            const int src = __ffs(hit) - 1;
                            kd = w0 + (neg ? Ly.OW - 1 - (k0 + src) : k0 + src);
                            kc = __shfl_sync(kFullMask, cnt, src);
                            wk = __shfl_sync(kFullMask, w, src);
                            cb = c + __shfl_sync(kFullMask, incl - m, src);
                        }
                        c += __shfl_sync(kFullMask, incl, 31);
                    }
                    if (kd < 0) {
                        redo = 1;
                    } else {
                        long long t = (long long)ceil((target - cb) / wk);
                        if (t < 1) t = 1;
                        if (t > (long long)kc) t = kc;
                        while (t > 1 && cb + (double)(t - 1) * wk >= target) --t;
                        while (t < (long long)kc && cb + (double)t * wk < target) ++t;
                        rs.kd = kd;
                        rs.kneg = neg;
                        rs.kbits = word_bits(rs, kd, neg);
                        rs.wk = wk;
                        rs.tkeep = (int)t;
                        rs.Sk = cb + (double)t * wk;
                        // +0 and -0 are one value but two counts: leave such a cut to the
                        // generic kernel
                        if ((rs.kbits & 0x7FFFu) == 0u) redo = 1;
                    }
                }
            }
            if (lane == 0) ts.dred[r][0] = redo;  // dred[0..1][0] are free here
        }
        team_sync(team);
        {
            const int redo = (int)ts.dred[0][0] | (nrows > 1 ? (int)ts.dred[1][0] : 0);
            team_sync(team);
            if (redo) {
                if (crank == 0 && tt == 0) p.recs[item].state = kRedo;
                // full mode: the exchange of step (6) still runs so that every barrier keeps its
                // phase; top-k mode: every CTA skips steps (5) to (7) alike
            }
            const bool cutting = TOPK || p.cut;
            // survivor weights of the top positive values (full mode)
            for (int r = 0; r < nrows && !TOPK; ++r) {
                RowStat& rs = ts.rs[r];
                int ln = kLut;
                if (p.cut && rs.kd >= 0 && !rs.kneg) ln = min(kLut, rs.kd + 1);
                for (int d = tt; d < ln; d += kTeamThreads)
                    lut[r * kLut + d] = ((int)rs.atop - d >= 0) ? wexp(word_bits(rs, d, 0), rs, T) : 0.0;
                if (tt == 0) rs.lut_n = (int)min((uint32_t)ln, rs.atop + 1u);
            }

            if (tt == 0) trace_mark(p, cid, crank, team, xph, 5);
            // ---- (5) where the kept ties end: counts of the tie value in lower-ranked CTAs ----
            if (cutting && !redo && tw < nrows) {
                const int r = tw;
                RowStat& rs = ts.rs[r];
                long long before = 0;
                uint32_t mine = 0;
                for (int q = 0; q < CL; ++q) {
                    uint32_t c = 0;
                    if (lane == 0) c = ld_remote_u32(mapa(&hist[r * Ly.hw + rs.kd], (uint32_t)q));
                    if (!TOPK) c = rs.kneg ? (c >> 16) : (c & 0xFFFFu);
                    if (q < (int)crank) before += c;
                    if (q == (int)crank) mine = c;
                }
                if (lane == 0) {
                    const long long keep = min((long long)mine, max(0LL, (long long)rs.tkeep - before));
                    ts.ured[r][0] = (uint32_t)keep;
                    ts.ured[r][1] = mine;
                }
            }
            team_sync(team);
            for (int r = 0; r < nrows && cutting && !redo; ++r) {
                RowStat& rs = ts.rs[r];
                const uint32_t keep = ts.ured[r][0], mine = ts.ured[r][1];
                if (keep == mine) {
                    if (tt == 0) rs.theta = INT_MAX;
                } else if (keep == 0) {
                    if (tt == 0) rs.theta = 0;
                } else {
                    // this CTA holds the boundary: find its keep-th tie in id order
                    const uint16_t* buf = bufs[r];
                    int c = 0;
                    for (int e = wv0 * 8 + lane; e < wv1 * 8; e += 32) c += elem(buf, e) == rs.kbits;
                    c = warp_sum(c);
                    if (lane == 0) ts.ipart[tw] = c;
                    team_sync(team);
                    int before = 0, wt = 0;
                    for (; wt < kTeamWarps; ++wt) {
                        if (before + ts.ipart[wt] >= (int)keep) break;
                        before += ts.ipart[wt];
                    }
                    if (tw == wt) {
                        int need = (int)keep - before, found = -1;
                        for (int e0 = wv0 * 8; e0 < wv1 * 8 && found < 0; e0 += 32) {
                            const int e = e0 + lane;
                            const unsigned bal = __ballot_sync(kFullMask, e < wv1 * 8 && elem(buf, e) == rs.kbits);
                            const int nb = __popc(bal);
                            if (nb >= need) {
                                unsigned bb = bal;
                                for (int q = 1; q < need; ++q) bb &= bb - 1;
                                found = e0 + __ffs(bb) - 1;
                            }
                            need -= nb;
                        }
                        if (lane == 0) rs.theta = lo + found + 1;
                    }
                }
                team_sync(team);
            }
            team_sync(team);

            if constexpr (TOPK) {
                if (!redo) {
                    const int head = item % CL;
                    // ---- (6) the top-k survivors, appended to the head CTA's lists ----
                    for (int r = 0; r < nrows; ++r) {
                        const RowStat rs = ts.rs[r];
                        const __nv_bfloat162 k2 = as_bf2(rs.kbits | (rs.kbits << 16));
                        const float kx = bf(rs.kbits);
                        const uint32_t cnt_addr = mapa(&ts.lcnt[r], (uint32_t)head);
                        const uint32_t list_addr = mapa(&list[r * Ly.KL], (uint32_t)head);
                        const uint4* v4 = reinterpret_cast<const uint4*>(bufs[r]);
                        for (int j = tt; j < nvec; j += kTeamThreads) {
                            const uint4 v = v4[j];
                            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const uint32_t m = __hge2_mask(as_bf2(w[q]), k2);
                                if (!m) continue;
#pragma unroll
                                for (int hh = 0; hh < 2; ++hh) {
                                    if (!((m >> (16 * hh)) & 1u)) continue;
                                    const uint32_t h16 = (w[q] >> (16 * hh)) & 0xFFFFu;
                                    const float x = bf(h16);
                                    const int id = lo + j * 8 + 2 * q + hh;
                                    if (x == kx && id >= rs.theta) continue;  // a tie past the kept ones
                                    const uint32_t slot = atom_remote_add(cnt_addr, 1u);
                                    if (slot < (uint32_t)Ly.KL)
                                        st_remote_u64(list_addr + 8u * slot, pack_candidate(float_key(x), (uint32_t)id));
                                }
                            }
                        }
                    }
                    team_sync(team);
                    if (tt == 0) {
                        fence_cluster();
                        arrive_remote(mapa(xb3, (uint32_t)head));
                    }
                    // ---- (7) the head: softmax and top-p over the survivors, the draws, the tests ----
                    if ((int)crank == head) {
                        if (tw == 0) {
                            const bool ok = wait_cluster(xb3, hph & 1);
                            if (!ok && lane == 0) ts.abort_ = 1;
                        }
                        ++hph;
                        team_sync(team);
                        if (ts.abort_) break;
                        if (tw < nrows) {  // warp r: row r's survivor record
                            const int r = tw;
                            const int nk = (int)min(ts.lcnt[r], (unsigned)Ly.KL);
                            uint64_t* Lr = list + r * Ly.KL;
                            uint64_t* Tr = ltmp + r * Ly.KL;
                            double* Wr = lw + r * Ly.KL;
                            int32_t* Ir = lid + r * Ly.KL;
                            int n2 = 32;
                            while (n2 < nk) n2 <<= 1;
                            for (int j = nk + lane; j < n2; j += 32) Lr[j] = 0ull;
                            __syncwarp();
                            warp_sort_desc(Lr, n2, lane);  // (value desc, id asc)
                            const double zmax = ts.rs[r].zmax;
                            double S1 = 0.0;
                            for (int j = lane; j < nk; j += 32) {
                                const double w = exp((double)key_float(candidate_key(Lr[j])) / T - zmax);
                                Tr[j] = __double_as_longlong(w);
                                S1 += w;
                            }
                            S1 = warp_sum_f64(S1);
                            __syncwarp();
                            // top-p: the shortest prefix of that order whose mass reaches top_p
                            int np = nk;
                            if (p.cut) {
                                double carry = 0.0;
                                for (int j0 = 0; j0 < nk; j0 += 32) {
                                    const int j = j0 + lane;
                                    const double x = j < nk ? __longlong_as_double(Tr[j]) / S1 : 0.0;
                                    const double incl = warp_scan_f64(x, lane);
                                    const unsigned hit = __ballot_sync(kFullMask, j < nk && carry + incl >= p.top_p);
                                    if (hit) {
                                        np = j0 + __ffs(hit);
                                        break;
                                    }
                                    carry += __shfl_sync(kFullMask, incl, 31);
                                }
                            }
                            // the survivors in id order, with their weights
                            int sid[kMaxTopK / 32];
                            double sw[kMaxTopK / 32];
                            for (int j = lane, t = 0; j < n2; j += 32, ++t) {
                                const uint32_t id = j < np ? candidate_id(Lr[j]) : 0xFFFFFFFFu;
                                sid[t] = (int)id;
                                sw[t] = j < np ? __longlong_as_double(Tr[j]) : 0.0;
                            }
                            __syncwarp();
                            for (int j = lane, t = 0; j < n2; j += 32, ++t)
                                Lr[j] = j < np ? (((uint64_t)(0xFFFFFFFFu - (uint32_t)sid[t]) << 32) | (uint32_t)j) : 0ull;
                            for (int j = lane, t = 0; j < n2; j += 32, ++t) Tr[j] = __double_as_longlong(sw[t]);
                            __syncwarp();
                            warp_sort_desc(Lr, n2, lane);  // ascending id
                            double Z = 0.0;
                            for (int j = lane; j < np; j += 32) {
                                const uint32_t src = (uint32_t)(Lr[j] & 0xFFFFFFFFu);
                                Ir[j] = (int32_t)(0xFFFFFFFFu - (uint32_t)(Lr[j] >> 32));
                                Wr[j] = __longlong_as_double(Tr[src]);
                                Z += Wr[j];
                            }
                            Z = warp_sum_f64(Z);
                            if (lane == 0) {
                                ts.np[r] = np;
                                ts.Z[r] = Z;
                            }
                        }
                        team_sync(team);
                        if (tw == 0) {
                            const float* u = p.u + (int64_t)item * 3;
                            SRec P;
                            P.w = lw;
                            P.id = lid;
                            P.n = ts.np[0];
                            P.Z = ts.Z[0];
                            Rec rec;
                            rec.state = kDone;
                            rec.pad = 0.0;
                            if (i == 0) {
                                const int x0 = pos0_given(p, b) ? p.pos0[b] : srec_inv_cdf(P, (double)u[0], lane);
                                rec.tok = x0;
                                rec.res = -1;
                                rec.acc = 1;
                                rec.p = (x0 >= 0 && x0 < p.V) ? srec_prob(P, x0) : 0.0;
                                rec.q = 0.0;
                                rec.tv = 0.0;
                            } else {
                                SRec Q;
                                Q.w = lw + Ly.KL;
                                Q.id = lid + Ly.KL;
                                Q.n = ts.np[1];
                                Q.Z = ts.Z[1];
                                const int d = p.drafts ? p.drafts[item] : srec_inv_cdf(Q, (double)u[0], lane);
                                const bool in = d >= 0 && d < p.V;
                                rec.tok = d;
                                rec.p = in ? srec_prob(P, d) : 0.0;
                                rec.q = in ? srec_prob(Q, d) : 0.0;
                                rec.acc = (double)u[1] * rec.q < rec.p;
                                rec.tv = srec_tv(P, Q, lane);
                                rec.res = srec_residual(P, Q, (double)u[2], lane);
                            }
                            if (lane == 0) p.recs[item] = rec;
                        }
                    }
                }
            } else {
            if (tt == 0) trace_mark(p, cid, crank, team, xph, 6);
            // ---- (6) masses per warp part: draw row, verifier survivors, residual ----
            const int draw_row = i > 0 ? 1 : 0;
            const RowStat rp = ts.rs[0];
            const RowStat rq = ts.rs[nrows > 1 ? 1 : 0];
            const double iSp = 1.0 / rp.Sk, iSq = 1.0 / rq.Sk;
            double sd = 0.0, sp = 0.0, sr = 0.0;
            if (!redo) {
                const uint32_t kp = rp.kbits | (rp.kbits << 16), kq = rq.kbits | (rq.kbits << 16);
                const uint4* vp = reinterpret_cast<const uint4*>(bufs[0]);
                const uint4* vq = reinterpret_cast<const uint4*>(bufs[1]);
                for (int j = wv0 + lane; j < wv1; j += 32) {
                    const uint4 a = vp[j];
                    const uint32_t wa[4] = {a.x, a.y, a.z, a.w};
                    uint32_t ma = 0, mb = 0;
                    uint32_t wb[4] = {0, 0, 0, 0};
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        ma |= __hge2_mask(*reinterpret_cast<const __nv_bfloat162*>(&wa[q]),
                                          *reinterpret_cast<const __nv_bfloat162*>(&kp));
                    if (nrows > 1) {
                        const uint4 bq = vq[j];
                        wb[0] = bq.x;
                        wb[1] = bq.y;
                        wb[2] = bq.z;
                        wb[3] = bq.w;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            mb |= __hge2_mask(*reinterpret_cast<const __nv_bfloat162*>(&wb[q]),
                                              *reinterpret_cast<const __nv_bfloat162*>(&kq));
                    }
                    if (!(ma | mb)) continue;
                    const int e0 = lo + j * 8;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const uint32_t hp = (wa[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
                        const double wp = surv_weight(hp, e0 + e, rp, lut, T, p.cut);
                        double wq = 0.0;
                        if (nrows > 1) {
                            const uint32_t hq = (wb[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
                            wq = surv_weight(hq, e0 + e, rq, lut + kLut, T, p.cut);
                        }
                        sd += draw_row ? wq : wp;
                        sp += wp;
                        if (wp > 0.0) {
                            const double dl = wp * iSp - wq * iSq;
                            if (dl > 0.0) sr += dl;
                        }
                    }
                }
            }
            sd = warp_sum_f64(sd);
            sp = warp_sum_f64(sp);
            sr = warp_sum_f64(sr);
            if (lane == 0) {
                ts.wpart[tw][0] = sd;
                ts.wpart[tw][1] = sp;
                ts.wpart[tw][2] = sr;
            }
            team_sync(team);
            if (tw == 0) {
                double v3[3] = {0, 0, 0};
                for (int w = 0; w < kTeamWarps; ++w)
                    for (int k = 0; k < 3; ++k) v3[k] += ts.wpart[w][k];
                if (lane < CL) {
                    const uint32_t slot = mapa(&x3[crank * 3], (uint32_t)lane);
                    for (int k = 0; k < 3; ++k) st_remote_f64(slot + 8u * k, v3[k]);
                    arrive_remote(mapa(xb3, (uint32_t)lane));
                }
                const bool ok = wait_cluster(xb3, xph & 1);
                if (!ok && lane == 0) ts.abort_ = 1;
            }
            team_sync(team);
            if (ts.abort_) break;

            if (tt == 0) trace_mark(p, cid, crank, team, xph, 7);
            // ---- (7) the draws: the CTA and warp part holding each target, then its token ----
            if (!redo) {
                const float* u = p.u + (int64_t)item * 3;
                // mode 0: the draw row's survivors, 1: verifier survivors, 2: residual
                auto weight_at = [&](int mode, int e) -> double {  // e: element of this slice
                    const uint32_t hp = elem(bufs[0], e);
                    const double wp = surv_weight(hp, lo + e, rp, lut, T, p.cut);
                    if (mode == 1 || (mode == 0 && !draw_row)) return wp;
                    const double wq = surv_weight(elem(bufs[1], e), lo + e, rq, lut + kLut, T, p.cut);
                    if (mode == 0) return wq;
                    if (!(wp > 0.0)) return 0.0;
                    const double dl = wp * iSp - wq * iSq;
                    return dl > 0.0 ? dl : 0.0;
                };
                // returns the token id (only meaningful in the owning CTA), or -1 elsewhere;
                // identical owner choice in every CTA from the exchanged totals
                auto find = [&](int mode, double target) -> int {
                    double c = 0.0, clast = 0.0;
                    int owner = -1, last = -1;
                    for (int q = 0; q < CL; ++q) {
                        const double m = x3[q * 3 + mode];
                        if (!(m > 0.0)) continue;
                        last = q;
                        clast = c;
                        if (c + m > target) {
                            owner = q;
                            break;
                        }
                        c += m;
                    }
                    const bool last_mode = owner < 0;
                    if (last_mode) {
                        owner = last;
                        c = clast;
                    }
                    if (owner != (int)crank) return -1;
                    double c2 = c, c2last = c;
                    int wsel = -1, wlast = -1;
                    for (int w = 0; w < kTeamWarps; ++w) {
                        const double m = ts.wpart[w][mode];
                        if (!(m > 0.0)) continue;
                        wlast = w;
                        c2last = c2;
                        if (!last_mode && c2 + m > target) {
                            wsel = w;
                            break;
                        }
                        c2 += m;
                    }
                    const bool lm = last_mode || wsel < 0;
                    if (wsel < 0) {
                        wsel = wlast;
                        c2 = c2last;
                    }
                    int res = -1;
                    if (tw == wsel) {
                        const int v0 = min(nvec, wsel * pv) * 8, v1 = min(nvec, wsel * pv + pv) * 8;
                        double carry = c2;
                        int lastpos = -1;
                        for (int base = v0; base < v1 && res < 0; base += 32) {
                            const int e = base + lane;
                            const double x = e < v1 ? weight_at(mode, e) : 0.0;
                            const double incl = warp_scan_f64(x, lane);
                            const unsigned hit = lm ? 0u : __ballot_sync(kFullMask, x > 0.0 && carry + incl > target);
                            if (hit) res = lo + base + __ffs(hit) - 1;
                            const unsigned pos = __ballot_sync(kFullMask, x > 0.0);
                            if (pos) lastpos = lo + base + 31 - __clz(pos);
                            carry += __shfl_sync(kFullMask, incl, 31);
                        }
                        if (res < 0) res = lastpos;
                    }
                    return res;
                };
                // the item's token: drawn, or supplied
                int tok = -1;
                bool tok_here = false;
                if (i == 0 ? !pos0_given(p, b) : !p.drafts) {
                    const double target = (double)u[0] * (draw_row ? rq.Sk : rp.Sk);
                    tok = find(0, target);
                    tok_here = tok >= 0;
                } else {
                    tok = i == 0 ? p.pos0[b] : p.drafts[item];
                    const bool in = tok >= 0 && tok < p.V;
                    tok_here = in ? (tok >= lo && tok < lo + n) : crank == 0;
                    tok_here = tok_here && tw == 0;
                }
                if (tok_here && lane == 0) {
                    const bool in = tok >= 0 && tok < p.V;
                    double pd = 0.0, qd = 0.0;
                    if (in) {
                        pd = surv_weight(elem(bufs[0], tok - lo), tok, rp, lut, T, p.cut) * iSp;
                        if (i > 0) qd = surv_weight(elem(bufs[1], tok - lo), tok, rq, lut + kLut, T, p.cut) * iSq;
                    }
                    Rec& rec = p.recs[item];
                    rec.tok = tok;
                    rec.p = pd;
                    rec.q = qd;
                    rec.acc = i == 0 ? 1 : ((double)u[1] * qd < pd);
                }
                if (i > 0) {
                    double R = 0.0;
                    for (int q = 0; q < CL; ++q) R += x3[q * 3 + 2];
                    const int mode = R > 0.0 ? 2 : 1;
                    const int res = find(mode, (double)u[2] * (R > 0.0 ? R : rp.Sk));
                    if (res >= 0 && lane == 0) p.recs[item].res = res;
                    if (crank == 0 && tt == 0) {
                        p.recs[item].tv = R;
                        p.recs[item].state = kDone;
                    }
                } else if (crank == 0 && tt == 0) {
                    p.recs[item].res = -1;
                    p.recs[item].tv = 0.0;
                    p.recs[item].state = kDone;
                }
            }
            }  // full mode
        }
        if (tt == 0) trace_mark(p, cid, crank, team, xph, 8);
        ++xph;
        team_sync(team);  // the buffer is free
        if (tt == 0) {
            int nx = item + step;
            while (nx < n_items && !needs_rows(nx)) nx += step;
            if (nx < n_items) issue(nx);
        }
    }
    // a copy issued for an item this team will not process (after an abort): let it land
    if (tt == 0 && inflight) mbar_wait(full, lph & 1, 1u << 16);
    __syncthreads();
    cluster_sync_all();  // no CTA leaves while another may still read its shared memory
    if (tt == 0 && ts.abort_) record_device_status(p.status, (uint32_t)UNO_ERR_TIMEOUT);
}


// ---------------------------------------------------------------------------------------
// topk_local_kernel: top-k (k <= kMaxLocalK) with no cluster-wide cut. Each CTA takes the
// exact top-k of its own slice of each row (the k largest values, ties to the lower id):
// the row's top-k is among those CL lists, since a token outside its slice's top-k has k
// better tokens in that slice alone. A head CTA, rotating over the cluster from item to
// item, merges the lists, then applies softmax and top-p and takes the draws and the tests.
// Per item the only cluster traffic is each CTA's sorted list stored into the head's shared
// memory and one arrive on the head's barrier; the head acknowledges once it has read the
// lists, and a CTA waits for that only before its next push to the same head, CL items
// later, by when it is normally long done. Items whose slice top-k lies outside the 256
// largest values of the slice are left to the generic kernel.
// ---------------------------------------------------------------------------------------
constexpr int kMaxLocalK = 128;

struct LLayout {
    int CL;   // CTAs per cluster
    int L;    // slice length in elements (a multiple of 8)
    int KL;   // list capacity: a power of two >= k, >= 32
    uint32_t off_hist, off_loc, off_cand, off_cnt, off_merged, off_w, off_id, off_tmp, off_misc, team_bytes;
};

struct LShared {
    float fred[kTeamWarps][2];
    float M[2];
    int kd[2], tkeep[2], theta[2], take_all[2], redo[2], mine[2];
    uint32_t kbits[2];
    unsigned loc_n[2];
    int ipart[kTeamWarps];
    int np[2];
    double Z[2];
    int abort_, any_redo;
};

__global__ void __launch_bounds__(kThreads, 1) topk_local_kernel(Params p, LLayout Ly) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bars[kTeams][2 + kMaxCL];

    const int team = threadIdx.x / kTeamThreads, tt = threadIdx.x % kTeamThreads;
    const int tw = tt >> 5, lane = tt & 31;
    const int CL = Ly.CL, KL = Ly.KL;
    const uint32_t crank = ctarank();
    const int cid = blockIdx.x / CL, NC = gridDim.x / CL;
    const int n_items = p.B * p.K;
    const double T = p.T;

    unsigned char* base = smem + (size_t)team * Ly.team_bytes;
    uint16_t* bufs[2] = {reinterpret_cast<uint16_t*>(base), reinterpret_cast<uint16_t*>(base) + Ly.L};
    uint32_t* hist = reinterpret_cast<uint32_t*>(base + Ly.off_hist);      // [2][kWinK]
    uint64_t* loc = reinterpret_cast<uint64_t*>(base + Ly.off_loc);        // [2][KL] this slice's top-k
    uint64_t* cand = reinterpret_cast<uint64_t*>(base + Ly.off_cand);      // [2][CL][KL] lists (as head)
    int* cnt = reinterpret_cast<int*>(base + Ly.off_cnt);                  // [2][kMaxCL] list lengths, -1: redo
    uint64_t* merged = reinterpret_cast<uint64_t*>(base + Ly.off_merged);  // [2][KL] the row's top-k
    double* lw = reinterpret_cast<double*>(base + Ly.off_w);               // [2][KL] survivor weights, id order
    int32_t* lid = reinterpret_cast<int32_t*>(base + Ly.off_id);           // [2][KL] survivor ids
    uint64_t* ltmp = reinterpret_cast<uint64_t*>(base + Ly.off_tmp);       // [2][KL] scratch
    LShared& ls = *reinterpret_cast<LShared*>(base + Ly.off_misc);
    uint64_t* full = &bars[team][0];
    uint64_t* ein = &bars[team][1];     // the lists of an item this CTA heads have landed
    uint64_t* freeb = &bars[team][2];   // [kMaxCL]: head q has read the lists this CTA pushed to it

    if (tt == 0) {
        mbar_init(full, 1);
        mbar_init(ein, CL);
        for (int q = 0; q < CL; ++q) mbar_init(&freeb[q], 1);
        ls.abort_ = 0;
        fence_mbar_init();
    }
    __syncthreads();
    cluster_sync_all();

    const int lo = (int)crank * Ly.L;
    const int n = max(0, min(Ly.L, p.V - lo));
    const int nvec = n >> 3;
    const int pv = (nvec + kTeamWarps - 1) / kTeamWarps;
    const int wv0 = min(nvec, tw * pv), wv1 = min(nvec, wv0 + pv);
    const int step = kTeams * NC;
    const int kk = min(p.top_k, n);  // this slice's share of the list

    int issued = -1, inflight = 0;
    auto needs_rows = [&](int it) { return !trivial_item(p, it / p.K, it % p.K); };
    auto issue = [&](int it) {
        const int i = it % p.K;
        const int nrows = i > 0 ? 2 : 1;
        if (n > 0) {
            mbar_arrive_expect_tx(full, (uint32_t)(n * 2 * nrows));
            bulk_g2s(bufs[0], static_cast<const __nv_bfloat16*>(p.P) + (int64_t)it * p.V + lo, (uint32_t)(n * 2), full);
            if (i > 0)
                bulk_g2s(bufs[1], static_cast<const __nv_bfloat16*>(p.Q) + (int64_t)it * p.V + lo, (uint32_t)(n * 2),
                         full);
        } else {
            mbar_arrive(full);
        }
        issued = it;
        inflight = 1;
    };

    uint32_t lph = 0, hph = 0, jitem = 0;
    uint32_t pushes = 0;  // bit q, per head q: parity of this CTA's completed pushes there (see below)
    uint32_t pushed_once = 0;
    for (int item = cid + team * NC; item < n_items; item += step) {
        const int b = item / p.K, i = item % p.K;
        if (!needs_rows(item)) {
            if (crank == 0 && tt == 0) write_trivial(p, item, b);
            continue;
        }
        const int nrows = i > 0 ? 2 : 1;
        const int head = (int)(jitem % (uint32_t)CL);
        const uint32_t jm = jitem++;
        if (tt == 0) trace_mark(p, cid, crank, team, jm, 0);
        if (tt == 0 && issued != item) issue(item);
        if (tw == 0) {
            const bool ok = mbar_wait(full, lph & 1);
            if (!ok && lane == 0) ls.abort_ = 1;
        }
        ++lph;
        if (tt == 0) inflight = 0;
        team_sync(team);
        if (ls.abort_) break;

        if (tt == 0) trace_mark(p, cid, crank, team, jm, 1);
        // ---- (1) this slice's largest value per row ----
        {
            __nv_bfloat162 mx[2] = {__floats2bfloat162_rn(-INFINITY, -INFINITY), __floats2bfloat162_rn(-INFINITY, -INFINITY)};
            for (int r = 0; r < nrows; ++r) {
                const uint4* v4 = reinterpret_cast<const uint4*>(bufs[r]);
                for (int j = tt; j < nvec; j += kTeamThreads) {
                    const uint4 v = v4[j];
                    mx[r] = __hmax2(mx[r], __hmax2(__hmax2(as_bf2(v.x), as_bf2(v.y)), __hmax2(as_bf2(v.z), as_bf2(v.w))));
                }
            }
            const float m0 = warp_max(fmaxf(__low2float(mx[0]), __high2float(mx[0])));
            const float m1 = warp_max(fmaxf(__low2float(mx[1]), __high2float(mx[1])));
            if (lane == 0) {
                ls.fred[tw][0] = m0;
                ls.fred[tw][1] = m1;
            }
            for (int j = tt; j < 2 * kWinK; j += kTeamThreads) hist[j] = 0u;
            if (tt < 2) ls.loc_n[tt] = 0u;
            team_sync(team);
            if (tt < 2) {
                float M = -INFINITY;
                for (int w = 0; w < kTeamWarps; ++w) M = fmaxf(M, ls.fred[w][tt]);
                if (M == 0.f) M = 0.f;  // +0, at or above every zero in key order
                ls.M[tt] = M;
            }
            team_sync(team);
        }
        if (tt == 0) trace_mark(p, cid, crank, team, jm, 2);
        // ---- (2) counts of the slice's 256 largest values ----
        for (int r = 0; r < nrows; ++r) {
            const uint32_t kM = key16(__float_as_uint(ls.M[r]) >> 16);
            const uint32_t kf = kM >= (uint32_t)(kWinK - 1) ? kM - (uint32_t)(kWinK - 1) : 0u;
            const uint32_t hf = bits16(kf);
            const __nv_bfloat162 f2 = as_bf2(hf | (hf << 16));
            uint32_t* h = hist + r * kWinK;
            const uint4* v4 = reinterpret_cast<const uint4*>(bufs[r]);
            for (int j = tt; j < nvec; j += kTeamThreads) {
                const uint4 v = v4[j];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t m = __hge2_mask(as_bf2(w[q]), f2);
                    if (m) {
                        const uint32_t dl = kM - key16(w[q] & 0xFFFFu), dh = kM - key16(w[q] >> 16);
                        if ((m & 0xFFFFu) && dl < (uint32_t)kWinK) atomicAdd(&h[dl], 1u);
                        if ((m >> 16) && dh < (uint32_t)kWinK) atomicAdd(&h[dh], 1u);
                    }
                }
            }
        }
        team_sync(team);
        if (tt == 0) trace_mark(p, cid, crank, team, jm, 3);
        // ---- (3) warp r: the slice's k-th largest value of row r, and how many of its ties count ----
        if (tw < nrows) {
            const int r = tw;
            const uint32_t kM = key16(__float_as_uint(ls.M[r]) >> 16);
            int take_all = kk >= n, redo = 0, kd = -1, tkeep = 0, mine = 0;
            if (!take_all && kk > 0) {
                int c = 0;
                for (int d0 = 0; d0 < kWinK && kd < 0; d0 += 32) {
                    const int cn = (int)hist[r * kWinK + d0 + lane];
                    const int incl = warp_inclusive_scan(cn, lane);
                    const unsigned hit = __ballot_sync(kFullMask, cn > 0 && c + incl >= kk);
                    if (hit) {
                        const int src = __ffs(hit) - 1;
                        kd = d0 + src;
                        mine = __shfl_sync(kFullMask, cn, src);
                        tkeep = kk - (c + __shfl_sync(kFullMask, incl - cn, src));
                    }
                    c += __shfl_sync(kFullMask, incl, 31);
                }
                if (kd < 0) redo = 1;  // fewer than k of the slice's tokens among its 256 largest values
            }
            const uint32_t kb = kd >= 0 ? bits16(kM - (uint32_t)kd) : 0xFF80u;
            // +0 and -0 are one value under two keys: leave such a cut to the generic kernel
            if (kd >= 0 && (kb & 0x7FFFu) == 0u) redo = 1;
            if (lane == 0) {
                ls.take_all[r] = take_all || kk == 0;
                ls.redo[r] = redo;
                ls.kd[r] = kd;
                ls.kbits[r] = kb;
                ls.tkeep[r] = tkeep;
                ls.mine[r] = mine;
                ls.theta[r] = INT_MAX;
            }
        }
        team_sync(team);
        if (tt == 0) trace_mark(p, cid, crank, team, jm, 4);
        // ---- (4) the last tie that counts, in id order (when only some ties count) ----
        for (int r = 0; r < nrows; ++r) {
            if (ls.take_all[r] || ls.redo[r] || ls.tkeep[r] >= ls.mine[r]) continue;
            const uint16_t* buf = bufs[r];
            const uint32_t kb = ls.kbits[r];
            const int keep = ls.tkeep[r];
            int c = 0;
            for (int e = wv0 * 8 + lane; e < wv1 * 8; e += 32) c += elem(buf, e) == kb;
            c = warp_sum(c);
            if (lane == 0) ls.ipart[tw] = c;
            team_sync(team);
            int before = 0, wt = 0;
            for (; wt < kTeamWarps; ++wt) {
                if (before + ls.ipart[wt] >= keep) break;
                before += ls.ipart[wt];
            }
            if (tw == wt) {
                int need = keep - before, found = -1;
                for (int e0 = wv0 * 8; e0 < wv1 * 8 && found < 0; e0 += 32) {
                    const int e = e0 + lane;
                    const unsigned bal = __ballot_sync(kFullMask, e < wv1 * 8 && elem(buf, e) == kb);
                    const int nb = __popc(bal);
                    if (nb >= need) {
                        unsigned bb = bal;
                        for (int q = 1; q < need; ++q) bb &= bb - 1;
                        found = e0 + __ffs(bb) - 1;
                    }
                    need -= nb;
                }
                if (lane == 0) ls.theta[r] = lo + found + 1;
            }
            team_sync(team);
        }
        if (tt == 0) trace_mark(p, cid, crank, team, jm, 5);
        // ---- (5) the slice's top-k of each row, gathered locally ----
        for (int r = 0; r < nrows; ++r) {
            if (ls.redo[r]) continue;
            const bool all = ls.take_all[r];
            const uint32_t kb = ls.kbits[r];
            const __nv_bfloat162 k2 = as_bf2(kb | (kb << 16));
            const float kx = bf(kb);
            const int theta = ls.theta[r];
            uint64_t* Lr = loc + r * KL;
            const uint4* v4 = reinterpret_cast<const uint4*>(bufs[r]);
            for (int j = tt; j < nvec; j += kTeamThreads) {
                const uint4 v = v4[j];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t m = all ? 0xFFFFFFFFu : __hge2_mask(as_bf2(w[q]), k2);
                    if (!m) continue;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        if (!((m >> (16 * hh)) & 1u)) continue;
                        const uint32_t h16 = (w[q] >> (16 * hh)) & 0xFFFFu;
                        const float x = bf(h16);
                        const int id = lo + j * 8 + 2 * q + hh;
                        if (!all && x == kx && id >= theta) continue;
                        const unsigned slot = atomicAdd(&ls.loc_n[r], 1u);
                        if (slot < (unsigned)KL) Lr[slot] = pack_candidate(float_key(x), (uint32_t)id);
                    }
                }
            }
        }
        team_sync(team);
        if (tt == 0) trace_mark(p, cid, crank, team, jm, 6);
        // ---- (6) warp r sorts row r's list (value desc, id asc) ----
        if (tw < nrows) {
            const int r = tw;
            uint64_t* Lr = loc + r * KL;
            const int c = ls.redo[r] ? 0 : (int)min(ls.loc_n[r], (unsigned)KL);
            for (int j = c + lane; j < KL; j += 32) Lr[j] = 0ull;
            __syncwarp();
            warp_sort_desc(Lr, KL, lane);
        }
        team_sync(team);
        if (tt == 0) trace_mark(p, cid, crank, team, jm, 7);
        // ---- (7) push the lists into the head's shared memory ----
        if (tw == 0) {
            const uint32_t hbit = 1u << head;
            if (pushed_once & hbit) {  // the head has read what this CTA pushed there last time
                const bool ok = wait_cluster(&freeb[head], (pushes >> head) & 1u);
                if (!ok && lane == 0) ls.abort_ = 1;
                pushes ^= hbit;
            }
            pushed_once |= hbit;
            for (int r = 0; r < nrows; ++r) {
                // odd ranks store their list reversed (ascending), so that the head's lists
                // alternate in direction, as a bitonic merge network takes them
                const uint32_t dst = mapa(&cand[(r * CL + (int)crank) * KL], (uint32_t)head);
                const bool rev = (crank & 1u) != 0u;
                for (int j = lane; j < KL; j += 32)
                    st_remote_u64(dst + 8u * (uint32_t)(rev ? KL - 1 - j : j), loc[r * KL + j]);
                if (lane == 0) {
                    const int c = ls.redo[r] ? -1 : (int)min(ls.loc_n[r], (unsigned)KL);
                    asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(mapa(&cnt[r * kMaxCL + (int)crank], (uint32_t)head)),
                                 "r"(c)
                                 : "memory");
                }
            }
            __syncwarp();
            if (lane == 0) {
                fence_cluster();
                arrive_remote(mapa(ein, (uint32_t)head));
            }
            if (lane == 0) trace_mark(p, cid, crank, team, jm, 8);
        }
        // ---- (8) the head merges the lists, cuts, draws and tests ----
        if ((int)crank == head) {
            if (tw == 0) {
                const bool ok = wait_cluster(ein, hph & 1);
                if (!ok && lane == 0) ls.abort_ = 1;
            }
            ++hph;
            team_sync(team);
            if (tt == 0) trace_mark(p, cid, crank, team, jm, 9);
            if (ls.abort_) break;
            if (tt == 0) {
                int rd = 0;
                for (int r = 0; r < nrows; ++r)
                    for (int q = 0; q < CL; ++q) rd |= cnt[r * kMaxCL + q] < 0;
                ls.any_redo = rd;
            }
            team_sync(team);
            const bool redo = ls.any_redo;
            if (!redo) {
                // the CL sorted lists of each row (alternately descending and ascending) form
                // bitonic runs: the merge phases of a bitonic sort (run lengths 2 KL ... CL KL)
                // leave each row's CL KL entries in descending order
                const int nall = CL * KL;
                for (int size = 2 * KL; size <= nall; size <<= 1) {
                    for (int stride = size >> 1; stride > 0; stride >>= 1) {
                        for (int t = tt; t < nrows * (nall >> 1); t += kTeamThreads) {
                            const int r = t / (nall >> 1), tr = t % (nall >> 1);
                            uint64_t* A = cand + r * nall;
                            const int lo2 = 2 * tr - (tr & (stride - 1));
                            const int hi2 = lo2 + stride;
                            const bool desc = (lo2 & size) == 0;
                            const uint64_t x = A[lo2], y = A[hi2];
                            if ((x < y) == desc) {
                                A[lo2] = y;
                                A[hi2] = x;
                            }
                        }
                        team_sync(team);
                    }
                }
            }
            if (!redo && tw < nrows) {  // warp r: softmax, top-p, survivors by id
                const int r = tw;
                int total = 0;
                for (int q = 0; q < CL; ++q) total += cnt[r * kMaxCL + q];
                const int nk = min(p.top_k, total);
                uint64_t* Mr = merged + r * KL;
                for (int j = lane; j < KL; j += 32) Mr[j] = j < nk ? cand[r * CL * KL + j] : 0ull;
                __syncwarp();
                uint64_t* Tr = ltmp + r * KL;
                double* Wr = lw + r * KL;
                int32_t* Ir = lid + r * KL;
                // the row's largest value is the first of the merged list
                const double zm = (double)key_float(candidate_key(Mr[0])) / T;
                double S1 = 0.0;
                for (int j = lane; j < nk; j += 32) {
                    const double w = exp((double)key_float(candidate_key(Mr[j])) / T - zm);
                    Tr[j] = __double_as_longlong(w);
                    S1 += w;
                }
                S1 = warp_sum_f64(S1);
                __syncwarp();
                int np = nk;
                if (p.cut) {
                    double carry = 0.0;
                    for (int j0 = 0; j0 < nk; j0 += 32) {
                        const int j = j0 + lane;
                        const double x = j < nk ? __longlong_as_double(Tr[j]) / S1 : 0.0;
                        const double incl = warp_scan_f64(x, lane);
                        const unsigned hit = __ballot_sync(kFullMask, j < nk && carry + incl >= p.top_p);
                        if (hit) {
                            np = j0 + __ffs(hit);
                            break;
                        }
                        carry += __shfl_sync(kFullMask, incl, 31);
                    }
                }
                // the survivors in id order: sort (id asc) the first np entries
                for (int j = lane; j < KL; j += 32)
                    Mr[j] = j < np ? (((uint64_t)(0xFFFFFFFFu - candidate_id(Mr[j])) << 32) | (uint32_t)j) : 0ull;
                __syncwarp();
                warp_sort_desc(Mr, KL, lane);
                double Z = 0.0;
                for (int j = lane; j < np; j += 32) {
                    const uint32_t src = (uint32_t)(Mr[j] & 0xFFFFFFFFu);
                    Ir[j] = (int32_t)(0xFFFFFFFFu - (uint32_t)(Mr[j] >> 32));
                    Wr[j] = __longlong_as_double(Tr[src]);
                    Z += Wr[j];
                }
                Z = warp_sum_f64(Z);
                if (lane == 0) {
                    ls.np[r] = np;
                    ls.Z[r] = Z;
                }
            }
            team_sync(team);
            if (tt == 0) trace_mark(p, cid, crank, team, jm, 10);
            // the lists are read: acknowledge to every CTA
            if (tw == 1 && lane < CL) arrive_remote(mapa(&freeb[crank], (uint32_t)lane));
            if (tw == 0) {
                if (redo) {
                    if (lane == 0) p.recs[item].state = kRedo;
                } else {
                    const float* u = p.u + (int64_t)item * 3;
                    SRec P;
                    P.w = lw;
                    P.id = lid;
                    P.n = ls.np[0];
                    P.Z = ls.Z[0];
                    Rec rec;
                    rec.state = kDone;
                    rec.pad = 0.0;
                    if (i == 0) {
                        const int x0 = pos0_given(p, b) ? p.pos0[b] : srec_inv_cdf(P, (double)u[0], lane);
                        rec.tok = x0;
                        rec.res = -1;
                        rec.acc = 1;
                        rec.p = (x0 >= 0 && x0 < p.V) ? srec_prob(P, x0) : 0.0;
                        rec.q = 0.0;
                        rec.tv = 0.0;
                    } else {
                        SRec Q;
                        Q.w = lw + KL;
                        Q.id = lid + KL;
                        Q.n = ls.np[1];
                        Q.Z = ls.Z[1];
                        const int d = p.drafts ? p.drafts[item] : srec_inv_cdf(Q, (double)u[0], lane);
                        const bool in = d >= 0 && d < p.V;
                        rec.tok = d;
                        rec.p = in ? srec_prob(P, d) : 0.0;
                        rec.q = in ? srec_prob(Q, d) : 0.0;
                        rec.acc = (double)u[1] * rec.q < rec.p;
                        rec.tv = srec_tv(P, Q, lane);
                        rec.res = srec_residual(P, Q, (double)u[2], lane);
                    }
                    if (lane == 0) p.recs[item] = rec;
                }
            }
        }
        team_sync(team);  // the buffer and the local lists are free
        if (tt == 0) trace_mark(p, cid, crank, team, jm, 11);
        if (tt == 0) {
            int nx = item + step;
            while (nx < n_items && !needs_rows(nx)) nx += step;
            if (nx < n_items) issue(nx);
        }
    }
    if (tt == 0 && inflight) mbar_wait(full, lph & 1, 1u << 16);
    __syncthreads();
    cluster_sync_all();
    if (tt == 0 && ls.abort_) record_device_status(p.status, (uint32_t)UNO_ERR_TIMEOUT);
}

}  // namespace pk

// =======================================================================================
// Row streaming (bf16 rows, V a multiple of 8, 16-byte aligned, top-k off): two persistent
// kernels, each reading every logit once.
//
// row_kernel, one row per CTA at a time (the verifier rows and the drafter rows i >= 1).
// Streaming the row it takes the largest value M, counts exactly how many tokens hold each
// of the kWin largest order keys from an anchor a little above a sampled maximum (one count
// array per warp), and sums the weight exp((x - F) / T) of every element below that window
// (F its lowest value) in fp32 (ex2.approx) into an fp64 total, with a rigorous bound E on
// that sum's error: the measured ex2 error, the three roundings of the argument and the
// fp32 partial sums. Z = sum over the window of count * exp(v / T - M / T) in fp64 plus the
// rescaled rest sum, known to within E. The top-p cut (the value at which the mass from the
// top first reaches top_p * Z, and how many of the tokens at that value it keeps, lowest
// ids first) is decided from the window's counts for top_p * (Z - E) and top_p * (Z + E):
// when both give the same cut it is the exact one, and every mass the item pass needs (the
// survivors lie inside the window) is a count times an fp64 weight. Otherwise (the bound
// straddles a token boundary, the cut lies below the window, the row has no cut, an element
// lies above the window, the window would reach non-positive values, a non-finite weight)
// the CTA recounts the row exactly: counts per (sign, magnitude) for the kMagWin magnitudes
// below the largest and an fp64 weight for every tinier element. A row whose cut cannot be decided that way (or whose
// largest value is not finite) sends its item to the generic kernel.
//
// item_kernel_rs, one item per CTA at a time: streams the item's rows again, each warp its
// run of chunks in id order, and sums per group of chunks the masses the draws walk (the
// draw row's survivors, the verifier's survivors, the residual max(0, p - q)) and |p - q|.
// A draw finds the group holding its target from those sums and rescans that group alone.
// Tokens at a cut value survive by rank among the row's tokens at that value (the row
// record holds how many precede each warp's run).
// =======================================================================================
namespace rs {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kCtasPerSm = 2;         // item pass
constexpr int kRowCtasPerSm = 3;      // row pass (UNO_VERIFY_ROW_CTAS=2: two, with more registers each)
constexpr int kGroup = 4;             // chunks per group of the row pass (a chunk: 32 lanes x 8 elements)
constexpr int kCh = 256;              // elements per chunk
constexpr int kWin = 320;             // counted keys: the anchor and the kWin - 1 below it
constexpr int kAbove = 96;            // the anchor: this many keys above the sampled maximum
constexpr int kLutMax = 512;          // tabulated survivor weights per row
constexpr int kMagWin = 2048;         // recount: counted magnitudes (both signs) from the largest down
constexpr int kListCap = 4096;        // candidate list entries per warp run (beyond: the row has no list)
constexpr int kStage = 512;           // staged entries per warp before a list flush
constexpr int kMaxListV = 196608;     // list path: V up to this (the item pass's bitmap size)
constexpr double kEx2Err = 0x1p-22;   // bound on ex2.approx.ftz.f32's relative error (2^-22.7 measured)
constexpr double kU = 0x1p-24;        // fp32 unit roundoff
constexpr double kLn2 = 0.6931471805599453;

// A row's statistics (written by row_kernel, read by item_kernel_rs).
struct RowRec {
    double zmax;              // largest logit / T
    double S;                 // surviving mass, relative to zmax
    uint32_t kM;              // order key of the largest value
    uint32_t kc;              // order key of the cut value: smaller keys do not survive
    int cut;                  // 0: every token survives
    int tie_t;                // tokens at the cut value that survive (the first tie_t by id)
    int tie_before[kWarps];   // tokens at the cut value before each warp's run
    int lut_n;                // lut[j]: weight of key kM - j, for j < lut_n (0 where absent)
    int state;                // kDone, or kRedo (the item goes to the generic kernel)
    int list_ok;              // the candidate lists hold every survivor (window path, no overflow)
    uint32_t A15;             // the window's anchor (bf16 bits): an entry's window bin is A15 - its bits
    int dcut;                 // the cut value's window bin (list path)
    int list_n[kWarps];       // entries in each warp run's list
    int theta;                // list path: a token at the cut value survives when its id is below theta
    double lut[kLutMax];
};

typedef unsigned long long f2;
__device__ __forceinline__ f2 pk(float lo, float hi) {
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float lo_of(f2 v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi_of(f2 v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
    f2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2 sub2(f2 a, f2 b) {
    f2 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
    f2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
    f2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float bfv(uint32_t h16) { return __uint_as_float(h16 << 16); }
__device__ __forceinline__ f2 widen(uint32_t w) { return pk(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)); }
__device__ __forceinline__ __nv_bfloat162 bf2(uint32_t w) { return *reinterpret_cast<const __nv_bfloat162*>(&w); }
// 16-bit order key of a bf16 value and back
__device__ __forceinline__ uint32_t okey(uint32_t h) { return (h & 0x8000u) ? (~h & 0xFFFFu) : (h | 0x8000u); }
__device__ __forceinline__ uint32_t obits(uint32_t k) { return (k & 0x8000u) ? (k & 0x7FFFu) : (~k & 0xFFFFu); }

// rows of the item space: r < n_items the verifier row of item r, else the drafter row of
// item r - n_items
__device__ __forceinline__ bool row_needed(const Params& p, int r) {
    const int n = p.B * p.K;
    if (r < n) return !trivial_item(p, r / p.K, r % p.K);
    return (r - n) % p.K > 0;
}
__device__ __forceinline__ const uint4* row_ptr(const Params& p, int r) {
    const int n = p.B * p.K;
    const __nv_bfloat16* base = r < n ? static_cast<const __nv_bfloat16*>(p.P) + (int64_t)r * p.V
                                      : static_cast<const __nv_bfloat16*>(p.Q) + (int64_t)(r - n) * p.V;
    return reinterpret_cast<const uint4*>(base);
}

// the warp's run of chunks
__device__ __forceinline__ void warp_run(int V, int warp, int& c0, int& c1) {
    const int nchunks = (V + kCh - 1) / kCh;
    c0 = nchunks * warp / kWarps;
    c1 = nchunks * (warp + 1) / kWarps;
}

// UNO_VERIFY_TRACE (profiling aid): phase timestamps of CTA 0's first 32 rows / items
// (kernel 0: rows, 1: items), and counters of recounted rows (slot 0) and generic items (1)
__device__ __forceinline__ void rs_mark(const Params& p, int kernel, int j, int e) {
    if (p.trace != nullptr && blockIdx.x == 0 && threadIdx.x == 0 && j < 32) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        p.trace[((kernel * 2) * 32 + j) * 16 + e] = t;
    }
}
// (kernel 0: rows, 1: items, 2: list items; the end time of each CTA at 6144 + CTA for rows,
// 7168 + CTA for list items, 8192 + CTA for items)
__device__ __forceinline__ void rs_end(const Params& p, int base) {
    if (p.trace != nullptr && threadIdx.x == 0 && blockIdx.x < 1024) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        p.trace[base + blockIdx.x] = t;
    }
}
__device__ __forceinline__ void rs_count(const Params& p, int slot) {
    if (p.trace != nullptr && threadIdx.x == 0) atomicAdd(&p.trace[(15 * 2 * 32) * 16 + slot], 1ull);
}

__device__ __forceinline__ double cta_sum(double v, double* red) {
    v = warp_sum_f64(v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < kWarps; ++w) t += red[w];  // the same order in every thread
    return t;
}

struct RowShared {
    uint32_t hw[kWarps][kWin + 1];  // per-warp counts of the window keys (anchor - d); the last slot takes
                                    // counted values above the anchor (the window is then void)
    uint32_t hc[kWin];           // their sum
    double wd[kWin];             // weight of window key d (where present), relative to zmax
    uint32_t hr[2 * kMagWin];    // recount: counts of (sign, magnitude largest - d)
    uint32_t stage[kWarps][kStage];  // counted elements (bits << 16 | (0xFFFF - (id - c0 256))) on their way to the list
    float fmax[kWarps];
    double dz[kWarps], db[kWarps], red[kWarps];
    int ties[kWarps];
    int ln[kWarps];              // entries each warp's list has taken
    int next[2];                 // the next row (alternate rows use alternate slots)
    int d_cut, tie_t, ok, theta;
    double S;
};

// The recount's bins in value order: VC over the positive magnitudes (largest first), VC2
// over the negative ones (smallest first).
struct VC {
    const uint32_t* hr;
    __device__ uint32_t operator[](int v) const { return hr[v]; }
};
struct VC2 {
    const uint32_t* hr;
    __device__ uint32_t operator[](int v) const { return hr[2 * kMagWin - 1 - v]; }
};

// The cut for `target` over bins [0, n) of masses cnt[d] * w[d] in value order (one warp,
// every lane gets the answer): the first bin at which the running mass reaches the target
// and how many of its tokens are kept (the fewest, at least one, that bring it there).
// Returns false if the bins' total does not reach the target.
template <typename C, typename W>
__device__ bool warp_cut(C cnt, W w, int n, double target, int lane, int& dcut, long long& t, double& cb) {
    const int per = (n + 31) / 32;
    double s = 0.0;
    for (int j = 0; j < per; ++j) {
        const int d = lane * per + j;
        if (d < n && cnt[d]) s += (double)cnt[d] * w(d);
    }
    const double incl = warp_scan_f64(s, lane);
    const unsigned hit = __ballot_sync(kFullMask, s > 0.0 && incl >= target);
    if (!hit) return false;
    const int L = __ffs(hit) - 1;
    double c = __shfl_sync(kFullMask, incl - s, L);
    int found = -1;
    for (int j = 0; j < per && found < 0; ++j) {
        const int d = L * per + j;
        if (d >= n || !cnt[d]) continue;
        const double m = (double)cnt[d] * w(d);
        if (c + m >= target) found = d;
        else c += m;
    }
    if (found < 0) return false;  // rounding between the two summation orders
    const double wk = w(found);
    const long long kc = cnt[found];
    long long tt = (long long)ceil((target - c) / wk);
    if (tt < 1) tt = 1;
    if (tt > kc) tt = kc;
    while (tt > 1 && c + (double)(tt - 1) * wk >= target) --tt;
    while (tt < kc && c + (double)tt * wk < target) ++tt;
    dcut = found;
    t = tt;
    cb = c;
    return true;
}

constexpr int kLT = 128;  // entries per list tile: lane l holds entries 4l .. 4l + 3 (one 16-byte load)
constexpr int kLB = 8;    // tiles per batch: the 16-byte loads each lane has in flight

// The id of the kk-th entry (0-based, id order) of a warp's list of n entries whose bits are
// hcut (entries: bits << 16 | (0xFFFF - (id - id0))); INT_MAX if there are not that many.
__device__ int find_tie(const uint32_t* list, int n, uint32_t hcut, int kk, int id0, int lane) {
    int cnt = 0;
    for (int t0 = 0; t0 < n; t0 += kLT * kLB) {
        uint4 v[kLB];
#pragma unroll
        for (int u = 0; u < kLB; ++u) {
            const int j = t0 + u * kLT + lane * 4;
            v[u] = j < n ? __ldcg(reinterpret_cast<const uint4*>(list + j)) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kLB; ++u) {
            const int j = t0 + u * kLT + lane * 4;
            const uint32_t e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t tie = 0u;
#pragma unroll
            for (int k = 0; k < 4; ++k) tie |= (uint32_t)(j + k < n && (e[k] >> 16) == hcut) << k;
            const int nt = __popc(tie);
            const int tot = (int)__reduce_add_sync(kFullMask, (unsigned)nt);
            if (cnt + tot > kk) {  // the same in every lane
                const int incl = warp_inclusive_scan(nt, lane);
                const int r = kk - cnt;  // its rank among this tile's ties
                const bool mine = incl > r && incl - nt <= r;
                int id = 0;
                if (mine) {
                    int q = r - (incl - nt);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if ((tie >> k) & 1u) {
                            if (q == 0) id = id0 + 0xFFFF - (int)(e[k] & 0xFFFFu);
                            --q;
                        }
                }
                return __shfl_sync(kFullMask, id, __ffs(__ballot_sync(kFullMask, mine)) - 1);
            }
            cnt += tot;
        }
    }
    return INT_MAX;
}

template <int CPS>
__global__ void __launch_bounds__(kThreads, CPS) row_kernel(Params p, RowRec* rows, uint32_t* lists, uint32_t* ctr) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RowShared& sh = *reinterpret_cast<RowShared*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int V = p.V, V8 = V >> 3;
    int c0, c1;
    warp_run(V, warp, c0, c1);
    const int n_rows = 2 * p.B * p.K;
    const double T = p.T;
    const float cT = (float)(1.4426950408889634 / T);  // log2(e) / T

    int jr = 0;  // rows this CTA has taken (trace)
    // rows are taken from a counter (after each CTA's first, blockIdx.x): a row that needs the
    // recount holds up only the CTA that has it
    int par = 0;
    for (int r = blockIdx.x; r < n_rows; r = sh.next[par], par ^= 1) {
        if (tid == 0) sh.next[par] = gridDim.x + (int)atomicAdd(ctr, 1u);  // read after this row's last barrier
        if (!row_needed(p, r)) {  // the same in every thread
            __syncthreads();
            continue;
        }
        const uint4* r4 = row_ptr(p, r);
        RowRec& out = rows[r];
        const int jm = jr++;
        rs_mark(p, 0, jm, 0);
        for (int j = lane; j <= kWin; j += 32) sh.hw[warp][j] = 0u;
        auto valid = [&](int c) { return c < c1 && c * 32 + lane < V8; };
        uint4 cur[kGroup];
#pragma unroll
        for (int u = 0; u < kGroup; ++u) cur[u] = valid(c0 + u) ? ld_stream_v4(r4 + (c0 + u) * 32 + lane) : make_uint4(0, 0, 0, 0);

        // ---- the anchor: kAbove keys above the largest value of every warp's first group ----
        {
            float lm = -INFINITY;
#pragma unroll
            for (int u = 0; u < kGroup; ++u) {
                if (!valid(c0 + u)) continue;
                const uint4 v = cur[u];
                const __nv_bfloat162 m2 = __hmax2(__hmax2(bf2(v.x), bf2(v.y)), __hmax2(bf2(v.z), bf2(v.w)));
                lm = fmaxf(lm, fmaxf(__low2float(m2), __high2float(m2)));
            }
            lm = warp_max(lm);
            if (lane == 0) sh.fmax[warp] = lm;
        }
        __syncthreads();
        float smax = -INFINITY;
        for (int w = 0; w < kWarps; ++w) smax = fmaxf(smax, sh.fmax[w]);
        uint32_t A15 = 0x7F80u, F15 = 0x7F80u;  // no window: every element to the rest sum
        bool fast = false;
        if (smax < INFINITY && smax > -INFINITY) {
            const uint32_t akey = min(okey(__float_as_uint(smax) >> 16) + (uint32_t)kAbove, 0xFF7Fu);
            if (akey >= 0x8000u + (uint32_t)kWin) {  // the window's lowest value is positive
                fast = true;
                A15 = akey - 0x8000u;
                F15 = A15 - (uint32_t)(kWin - 1);
            }
        }
        const float Fv = bfv(F15);
        const __nv_bfloat162 F2 = bf2(F15 | (F15 << 16));
        const f2 Ff = pk(Fv, Fv), C2 = pk(cT, cT);

        rs_mark(p, 0, jm, 1);
        // ---- stream the row ----
        // Every counted element (x >= F) goes, in id order, to the warp's stage as
        // bits << 16 | (0xFFFF - (id - c0 256)) (so one unsigned comparison with a per-row
        // threshold tells a survivor); each flush of the stage counts its entries' window
        // bins and appends them to the warp's candidate list.
        __nv_bfloat162 mx2 = __floats2bfloat162_rn(-INFINITY, -INFINITY);
        double zr = 0.0;  // rest weights exp((x - F) / T)
        // rest weights times their ex2 argument, which is negative for every rest element: the
        // error bound's sum of weights times |argument| is minus this (counted elements add 0)
        f2 zb2 = pk(0.f, 0.f);
        uint32_t* hwp = sh.hw[warp];
        uint32_t* stg = sh.stage[warp];
        uint32_t* gl = lists ? lists + ((int64_t)r * kWarps + warp) * kListCap : nullptr;
        int lq = 0, gn = 0;  // staged entries, entries this warp's list has taken (both warp-uniform)
        auto flush = [&](int n) {  // the first n staged entries (n <= 256)
            __syncwarp();
            for (int j = lane; j < n; j += 32) {
                const uint32_t s = stg[j];
                atomicAdd(&hwp[min(A15 - (s >> 16), (uint32_t)kWin)], 1u);  // above the anchor: last slot
                if (gl != nullptr && gn + n <= kListCap) gl[gn + j] = s;
            }
            gn += n;
            __syncwarp();
        };
        int c = c0;
        while (true) {
            const bool more = c + kGroup < c1;
            uint4 nxt[kGroup];
            if (more) {
#pragma unroll
                for (int u = 0; u < kGroup; ++u)
                    nxt[u] = valid(c + kGroup + u) ? ld_stream_v4(r4 + (c + kGroup + u) * 32 + lane) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kGroup; ++u) {
                if (c + u >= c1) continue;  // the same in every lane
                const bool ok = valid(c + u);
                const uint32_t w4[4] = {cur[u].x, cur[u].y, cur[u].z, cur[u].w};
                uint32_t cm = 0u;  // this lane's counted elements (bit e: element e of its 8)
                if (ok) {
                    f2 acc = pk(0.f, 0.f);
                    uint32_t mq[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t wq = w4[q];
                        const uint32_t m = __hge2_mask(bf2(wq), F2);  // x >= F: counted (0xFFFF per half)
                        mq[q] = m;
                        mx2 = __hmax2(mx2, bf2(wq));
                        const f2 a = mul2(sub2(widen(wq), Ff), C2);
                        const bool in0 = (m & 0xFFFFu) != 0u, in1 = (m >> 16) != 0u;
                        const float x0 = ex2f(lo_of(a)), x1 = ex2f(hi_of(a));
                        const f2 e = pk(in0 ? 0.f : x0, in1 ? 0.f : x1);
                        acc = add2(acc, e);
                        zb2 = fma2(e, a, zb2);
                    }
                    // bit 2q, 2q + 1: the halves of word q. One byte of each half (0x00 or
                    // 0xFF), four to a word, then each byte's low bit moved to bit 24 + its
                    // index by one multiply (the partial products do not overlap)
                    const uint32_t b0 = __byte_perm(mq[0], mq[1], 0x6420u) & 0x01010101u;
                    const uint32_t b1 = __byte_perm(mq[2], mq[3], 0x6420u) & 0x01010101u;
                    cm = ((b0 * 0x01020408u) >> 24) | (((b1 * 0x01020408u) >> 24) << 4);
                    zr += (double)lo_of(acc) + (double)hi_of(acc);
                }
                // this chunk's counted elements, in id order (lane, element), to the stage
                const int cnt = __popc(cm);
                const int incl = warp_inclusive_scan(cnt, lane);
                const int tot = __shfl_sync(kFullMask, incl, 31);
                if (tot) {
                    int pos = lq + incl - cnt;
                    const uint32_t base = 0xFFFFu - (uint32_t)((c + u - c0) * kCh + lane * 8);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if ((cm >> e) & 1u)
                            stg[pos++] = __byte_perm(w4[e >> 1], base - (uint32_t)e, (e & 1) ? 0x3254u : 0x1054u);
                    lq += tot;
                    if (lq >= 256) {  // (lq < 512: the rest moves from [256, lq) to the front)
                        flush(256);
                        for (int j = lane; j < lq - 256; j += 32) stg[j] = stg[256 + j];
                        __syncwarp();
                        lq -= 256;
                    }
                }
            }
            if (!more) break;
#pragma unroll
            for (int u = 0; u < kGroup; ++u) cur[u] = nxt[u];
            c += kGroup;
        }
        if (lq > 0) flush(lq);
        if (lane == 0) {
            out.list_n[warp] = gn;
            sh.ln[warp] = gn;
        }
        rs_mark(p, 0, jm, 2);
        {
            float lm = fmaxf(__low2float(mx2), __high2float(mx2));
            lm = warp_max(lm);
            zr = warp_sum_f64(zr);
            const double zbd = warp_sum_f64(-((double)lo_of(zb2) + (double)hi_of(zb2)));
            __syncthreads();  // every thread has read the anchor's maxima
            if (lane == 0) {
                sh.fmax[warp] = lm;
                sh.dz[warp] = zr;
                sh.db[warp] = zbd;
            }
        }
        __syncthreads();
        float M = -INFINITY;
        double ZR = 0.0, ZB = 0.0;
        for (int w = 0; w < kWarps; ++w) {
            M = fmaxf(M, sh.fmax[w]);
            ZR += sh.dz[w];
            ZB += sh.db[w];
        }
        if (M == 0.f) M = 0.f;  // +0
        // a value above the anchor was not counted: the window is void
        const int OVF = fast && (__float_as_uint(M) >> 16) > A15;
        const bool finite_max = M < INFINITY && M > -INFINITY;
        const double zmax = (double)M / T;
        const uint32_t kM = okey(__float_as_uint(M) >> 16);
        bool exact = fast && !OVF && p.cut && finite_max && ZR < INFINITY && ZB < INFINITY;  // NaN fails

        // ---- the window's masses, Z within E, and the cut ----
        if (exact) {
            double zw = 0.0;
            for (int d = tid; d < kWin; d += kThreads) {
                uint32_t cnt = 0;
                for (int w = 0; w < kWarps; ++w) cnt += sh.hw[w][d];
                sh.hc[d] = cnt;
                const double wv = cnt ? exp((double)bfv(A15 - (uint32_t)d) / T - zmax) : 0.0;
                sh.wd[d] = wv;
                zw += (double)cnt * wv;
            }
            zw = cta_sum(zw, sh.red);
            const double fz = exp((double)Fv / T - zmax);
            const double Zr = ZR * fz;
            const double Z = zw + Zr;
            const double E = 1.01 * ((kEx2Err + 3.0 * kU) * ZR + 3.0 * kU * kLn2 * ZB) * fz + 1e-14 * Z;
            if (warp == 0) {
                int d_lo = -1, d_hi = -2;
                long long t_lo = 0, t_hi = -1;
                double cb_lo = 0.0, cb_hi = 0.0;
                auto wwin = [&](int d) { return sh.wd[d]; };
                const bool a = warp_cut(sh.hc, wwin, kWin, p.top_p * (Z - E), lane, d_lo, t_lo, cb_lo);
                const bool b = warp_cut(sh.hc, wwin, kWin, p.top_p * (Z + E), lane, d_hi, t_hi, cb_hi);
                if (lane == 0) {
                    sh.ok = a && b && d_lo == d_hi && t_lo == t_hi;
                    sh.d_cut = d_hi;
                    sh.tie_t = (int)t_hi;
                    sh.S = cb_hi + (double)t_hi * sh.wd[max(d_hi, 0)];
                }
            }
            __syncthreads();
            exact = sh.ok;
        }
        rs_mark(p, 0, jm, 3);
        if (exact) {
            const int dcut = sh.d_cut;
            const int d0 = (int)(A15 - (__float_as_uint(M) >> 16));  // the largest value's bin
            const int lut_n = dcut - d0 + 1;
            for (int j = tid; j < lut_n; j += kThreads) out.lut[j] = sh.wd[d0 + j];
            if (tid == 0) {
                out.zmax = zmax;
                out.S = sh.S;
                out.kM = kM;
                out.kc = (A15 - (uint32_t)dcut) | 0x8000u;
                out.cut = 1;
                out.tie_t = sh.tie_t;
                int before = 0;
                for (int w = 0; w < kWarps; ++w) {
                    out.tie_before[w] = before;
                    before += (int)sh.hw[w][dcut];
                }
                out.lut_n = lut_n;
                out.state = kDone;
                out.A15 = A15;
                out.dcut = dcut;
            }
            // The lists are complete when every warp's fits. Then the tie at the cut of rank
            // tie_t (id order), the first that does not survive, is found in its warp's list:
            // a tie survives exactly when its id is below that tie's id (theta).
            int lok = lists != nullptr && V <= kMaxListV && lut_n <= 255;  // (table indices fit a byte)
            for (int w = 0; w < kWarps; ++w) lok &= sh.ln[w] <= kListCap;
            if (lok) {
                const int tt = sh.tie_t;
                int wb = -1, kk = 0, before = 0;
                for (int w = 0; w < kWarps; ++w) {
                    const int cw = (int)sh.hw[w][dcut];
                    if (wb < 0 && tt < before + cw) {
                        wb = w;
                        kk = tt - before;
                    }
                    before += cw;
                }
                if (warp == (wb < 0 ? 0 : wb)) {
                    const int th = wb < 0 ? INT_MAX : find_tie(gl, gn, A15 - (uint32_t)dcut, kk, c0 * kCh, lane);
                    if (lane == 0) sh.theta = th;
                }
            }
            __syncthreads();
            if (tid == 0) {
                out.list_ok = lok;
                out.theta = lok ? sh.theta : INT_MAX;
            }
            __syncthreads();  // the window counts are reused by the next row
            continue;
        }

        // ---- exact recount ----
        rs_count(p, 0);
        if (tid == 0) out.list_ok = 0;
        if (!finite_max) {
            if (tid == 0) out.state = kRedo;
            __syncthreads();
            continue;
        }
        // the largest magnitude (pass 1), then counts per (sign, magnitude) for the kMagWin
        // magnitudes below it and fp64 weights for the tinier ones (pass 2)
        for (int d = tid; d < 2 * kMagWin; d += kThreads) sh.hr[d] = 0u;
        uint32_t am = 0u;
        for (int cb = c0; cb < c1; cb += kGroup) {
            uint4 vv[kGroup];
#pragma unroll
            for (int u = 0; u < kGroup; ++u) vv[u] = valid(cb + u) ? ld_stream_v4(r4 + (cb + u) * 32 + lane) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < kGroup; ++u) {
                const uint32_t w4[4] = {vv[u].x, vv[u].y, vv[u].z, vv[u].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) am = max(am, max(w4[q] & 0x7FFFu, (w4[q] >> 16) & 0x7FFFu));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(kFullMask, am, o));
        if (lane == 0) sh.ties[warp] = (int)am;
        __syncthreads();
        uint32_t atop = 0u;
        for (int w = 0; w < kWarps; ++w) atop = max(atop, (uint32_t)sh.ties[w]);
        double zo = 0.0;
        for (int cb = c0; cb < c1; cb += kGroup) {
            uint4 vv[kGroup];
#pragma unroll
            for (int u = 0; u < kGroup; ++u) vv[u] = valid(cb + u) ? ld_stream_v4(r4 + (cb + u) * 32 + lane) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < kGroup; ++u) {
                if (!valid(cb + u)) continue;
                const uint32_t w4[4] = {vv[u].x, vv[u].y, vv[u].z, vv[u].w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t h = (w4[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
                    const uint32_t d = atop - (h & 0x7FFFu);
                    if (d < (uint32_t)kMagWin) atomicAdd(&sh.hr[(h >> 15) * kMagWin + d], 1u);
                    else zo += exp((double)bfv(h) / T - zmax);
                }
            }
        }
        __syncthreads();
        // value order: positive magnitudes from the top, the tiny ones, negative magnitudes
        // from the bottom; virtual bin v < kMagWin is (+, d = v), v >= kMagWin (-, d = 2 kMagWin - 1 - v)
        auto vcnt = [&](int v) -> uint32_t {
            return v < kMagWin ? sh.hr[v] : sh.hr[kMagWin + (2 * kMagWin - 1 - v)];
        };
        auto vbits = [&](int v) -> uint32_t {
            return v < kMagWin ? atop - (uint32_t)v : 0x8000u | (atop - (uint32_t)(2 * kMagWin - 1 - v));
        };
        auto vw = [&](int v) -> double { return (atop >= (uint32_t)(v < kMagWin ? v : 2 * kMagWin - 1 - v)) ? exp((double)bfv(vbits(v)) / T - zmax) : 0.0; };
        double zp = 0.0, zn = 0.0;  // masses of the positive and the negative bins
        for (int v = tid; v < 2 * kMagWin; v += kThreads) {
            const uint32_t cnt = vcnt(v);
            if (!cnt) continue;
            const double m = (double)cnt * vw(v);
            if (v < kMagWin) zp += m;
            else zn += m;
        }
        rs_mark(p, 0, jm, 4);
        zp = cta_sum(zp, sh.red);
        zn = cta_sum(zn, sh.red);
        zo = cta_sum(zo, sh.red);
        const double Z = zp + zo + zn;
        if (warp == 0) {
            int v = -1;
            long long tt = 0;
            double cb = 0.0;
            bool ok = Z > 0.0 && Z < INFINITY;
            if (ok && p.cut) {
                const double target = p.top_p * Z;
                VC vc{sh.hr};
                if (warp_cut(vc, vw, kMagWin, target, lane, v, tt, cb)) {
                    // the cut among the positive magnitudes
                } else if (target <= zp + zo) {
                    ok = false;  // among the tiniest magnitudes: the generic kernel decides
                } else {
                    // among the negative magnitudes (virtual bins kMagWin ..)
                    auto vw2 = [&](int x) { return vw(x + kMagWin); };
                    VC2 vc2{sh.hr};
                    ok = warp_cut(vc2, vw2, kMagWin, target - zp - zo, lane, v, tt, cb);
                    if (ok) {
                        v += kMagWin;
                        cb += zp + zo;
                    }
                }
                // +0 and -0 are one value under two keys: leave such a cut to the generic kernel
                if (ok && (vbits(v) & 0x7FFFu) == 0u) ok = false;
            }
            if (lane == 0) {
                sh.ok = ok;
                sh.d_cut = v;
                sh.tie_t = (int)tt;
                sh.S = p.cut ? (ok ? cb + (double)tt * vw(v) : 0.0) : Z;
            }
        }
        __syncthreads();
        if (!sh.ok) {
            if (tid == 0) out.state = kRedo;
            rs_count(p, 1);
            __syncthreads();
            continue;
        }
        const int dcut = sh.d_cut;
        const uint32_t kc = p.cut ? okey(vbits(dcut)) : 0u;
        // tokens at the cut value in each warp's run
        if (p.cut) {
            int cnt = 0;
            for (int cb = c0; cb < c1; cb += kGroup) {
                uint4 vv[kGroup];
#pragma unroll
                for (int u = 0; u < kGroup; ++u) vv[u] = valid(cb + u) ? ld_stream_v4(r4 + (cb + u) * 32 + lane) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int u = 0; u < kGroup; ++u) {
                    if (!valid(cb + u)) continue;
                    const uint32_t w4[4] = {vv[u].x, vv[u].y, vv[u].z, vv[u].w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) cnt += okey((w4[e >> 1] >> (16 * (e & 1))) & 0xFFFFu) == kc;
                }
            }
            cnt = warp_sum(cnt);
            if (lane == 0) sh.ties[warp] = cnt;
        }
        const int lut_n = p.cut ? (int)min((uint32_t)kLutMax, kM - kc + 1u) : kLutMax;
        for (int j = tid; j < lut_n; j += kThreads)
            out.lut[j] = kM >= (uint32_t)j ? exp((double)bfv(obits(kM - (uint32_t)j)) / T - zmax) : 0.0;
        // The candidate lists hold every element at or above the window's floor F, so they
        // serve the list item pass when the cut value is at or above F (the recount only
        // decided what the bounded sums could not); theta as on the window path.
        __syncthreads();  // every warp's tie count has landed
        const uint32_t hcut = p.cut ? obits(kc) : 0u;
        int lok = p.cut && fast && lists != nullptr && V <= kMaxListV && lut_n <= 255 && !(hcut & 0x8000u) &&
                  hcut >= F15;
        for (int w = 0; w < kWarps; ++w) lok &= sh.ln[w] <= kListCap;
        if (lok) {
            const int tt = sh.tie_t;
            int wb = -1, kk = 0, before = 0;
            for (int w = 0; w < kWarps; ++w) {
                const int cw = sh.ties[w];
                if (wb < 0 && tt < before + cw) {
                    wb = w;
                    kk = tt - before;
                }
                before += cw;
            }
            if (warp == (wb < 0 ? 0 : wb)) {
                const int th = wb < 0 ? INT_MAX : find_tie(gl, gn, hcut, kk, c0 * kCh, lane);
                if (lane == 0) sh.theta = th;
            }
        }
        __syncthreads();
        if (tid == 0) {
            out.list_ok = lok;
            out.theta = lok ? sh.theta : INT_MAX;
            out.A15 = A15;
            out.dcut = (int)(A15 - hcut);
            out.zmax = zmax;
            out.S = sh.S;
            out.kM = kM;
            out.kc = kc;
            out.cut = p.cut;
            out.tie_t = sh.tie_t;
            int before = 0;
            for (int w = 0; w < kWarps; ++w) {
                out.tie_before[w] = before;
                before += p.cut ? sh.ties[w] : 0;
            }
            out.lut_n = lut_n;
            out.state = kDone;
        }
        __syncthreads();
    }
    rs_end(p, 6144);
}

// ---------------------------------------------------------------------------------------
// item pass
// ---------------------------------------------------------------------------------------
struct RowView {
    double zmax, iS, S;
    uint32_t kM, kc;
    int cut, tie_t, tie_before, lut_n;
    const double* lut;  // shared memory
};

// survivor weight of value bits h (relative to zmax) if it survives by value alone, or is
// at the cut value (the caller ranks those); 0 otherwise
__device__ __noinline__ double weight_far(uint32_t h, double T, double zmax) { return exp((double)bfv(h) / T - zmax); }
__device__ __forceinline__ double weight_of(const RowView& R, uint32_t h, double T) {
    const uint32_t j = R.kM - okey(h);
    return j < (uint32_t)R.lut_n ? R.lut[j] : weight_far(h, T, R.zmax);
}

// the 8-bit masks of this lane's 8 elements strictly above / equal to the cut value
__device__ __forceinline__ void cut_masks(const uint4& v, const RowView& R, uint32_t& gt, uint32_t& eq) {
    gt = 0u;
    eq = 0u;
    if (!R.cut) {
        gt = 0xFFu;
        return;
    }
    const uint32_t cb = obits(R.kc);
    const __nv_bfloat162 c2 = bf2(cb | (cb << 16));
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t g = __hgt2_mask(bf2(w4[q]), c2), e = __heq2_mask(bf2(w4[q]), c2);
        gt |= ((g & 1u) << (2 * q)) | (((g >> 16) & 1u) << (2 * q + 1));
        eq |= ((e & 1u) << (2 * q)) | (((e >> 16) & 1u) << (2 * q + 1));
    }
    // +0 and -0 compare equal as bf16 but the cut is never at zero (those go to the generic kernel)
}

// Keep the ties (eq) this lane holds whose rank among the row's tokens at the cut value is
// below tie_t; seen: ties before this chunk in the warp's run (updated; the same in all lanes).
__device__ __forceinline__ uint32_t rank_ties(uint32_t eq, const RowView& R, int& seen, int lane) {
    const int ce = __popc(eq);
    const int incl = warp_inclusive_scan(ce, lane);
    const int base = R.tie_before + seen + incl - ce;
    seen += __shfl_sync(kFullMask, incl, 31);
    int keep = R.tie_t - base;
    if (keep <= 0) return 0u;
    uint32_t kept = 0u, m = eq;
    while (m && keep > 0) {
        const uint32_t bit = m & (0u - m);
        kept |= bit;
        m ^= bit;
        --keep;
    }
    return kept;
}

constexpr int kIG = 4;              // chunks per group of the item pass
constexpr int kMaxIGroups = 128;    // its groups per warp run (V <= kWarps * kMaxIGroups * kIG * kCh)
constexpr int kQueue = 32 + 4 * 32;  // word pairs queued per warp: < 32 carried + one chunk

struct ItemShared {
    double lut[2][kLutMax];
    double gs[kWarps][kMaxIGroups][3];   // per group: draw row, verifier survivors, residual
    int gseen[kWarps][kMaxIGroups][2];   // ties seen before the group (verifier, drafter)
    uint4 queue[kWarps][kQueue];         // word pairs with a kept token: (verifier, drafter, masks, first id)
    double wt[kWarps][3];                // per warp run: the totals of gs
    int ng[kWarps];                      // groups per warp run
    double red[kWarps];
    int sel_w, sel_g, mode;
    double sel_c;
    int tok_found;
};

// survivor masks of one chunk for both rows (ties ranked)
__device__ __forceinline__ void chunk_survivors(const uint4& vp, const uint4& vq, bool two, const RowView& P,
                                                const RowView& Q, int& seen_p, int& seen_q, int lane, uint32_t& sp,
                                                uint32_t& sq) {
    uint32_t gp, ep, gq = 0u, eq = 0u;
    cut_masks(vp, P, gp, ep);
    if (two) cut_masks(vq, Q, gq, eq);
    if (__any_sync(kFullMask, ep != 0u)) gp |= rank_ties(ep, P, seen_p, lane);
    if (two && __any_sync(kFullMask, eq != 0u)) gq |= rank_ties(eq, Q, seen_q, lane);
    sp = gp;
    sq = gq;
}

// the per-element masses of one chunk for the draw modes (0: draw row, 1: verifier, 2: residual)
__device__ __forceinline__ void chunk_masses(const uint4& vp, const uint4& vq, uint32_t mp, uint32_t mq, bool two,
                                             const RowView& P, const RowView& Q, double T, int mode, double (&x)[8]) {
    const uint32_t wp4[4] = {vp.x, vp.y, vp.z, vp.w};
    const uint32_t wq4[4] = {vq.x, vq.y, vq.z, vq.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const double wp = (mp >> e) & 1u ? weight_of(P, (wp4[e >> 1] >> (16 * (e & 1))) & 0xFFFFu, T) : 0.0;
        const double wq = (mq >> e) & 1u ? weight_of(Q, (wq4[e >> 1] >> (16 * (e & 1))) & 0xFFFFu, T) : 0.0;
        double v;
        if (mode == 1) v = wp;
        else if (mode == 0) v = two ? wq : wp;
        else {
            const double dl = wp * P.iS - wq * Q.iS;
            v = dl > 0.0 ? dl : 0.0;
        }
        x[e] = v;
    }
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm) item_kernel_rs(Params p, const RowRec* rows) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ItemShared& sh = *reinterpret_cast<ItemShared*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int V = p.V, V8 = V >> 3;
    int c0, c1;
    warp_run(V, warp, c0, c1);
    const int n_items = p.B * p.K;
    const double T = p.T;

    int ji = 0;  // items this CTA has taken (trace)
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int b = item / p.K, i = item % p.K;
        if (trivial_item(p, b, i)) {
            if (tid == 0) write_trivial(p, item, b);
            continue;
        }
        const int jm = ji++;
        rs_mark(p, 1, jm, 0);
        const bool two = i > 0;
        const RowRec& rp = rows[item];
        const RowRec& rq = rows[n_items + item];
        if (rp.state != kDone || (two && rq.state != kDone)) {
            if (tid == 0) p.recs[item].state = kRedo;
            continue;
        }
        if (rp.list_ok && (!two || rq.list_ok)) continue;  // item_list_kernel decides it
        RowView P, Q;
        auto view = [&](const RowRec& rr, int slot, RowView& R) {
            R.zmax = rr.zmax;
            R.S = rr.S;
            R.iS = 1.0 / rr.S;
            R.kM = rr.kM;
            R.kc = rr.kc;
            R.cut = rr.cut;
            R.tie_t = rr.tie_t;
            R.tie_before = rr.tie_before[warp];
            R.lut_n = rr.lut_n;
            R.lut = sh.lut[slot];
            for (int j = tid; j < rr.lut_n; j += kThreads) sh.lut[slot][j] = rr.lut[j];
        };
        __syncthreads();  // the previous item is done with the tables
        view(rp, 0, P);
        if (two) view(rq, 1, Q);
        else Q = P;
        __syncthreads();
        rs_mark(p, 1, jm, 1);

        const uint4* p4 = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.P) + (int64_t)item * V);
        const uint4* q4 = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.Q) + (int64_t)item * V);
        auto valid = [&](int c) { return c < c1 && c * 32 + lane < V8; };
        auto ldp = [&](int c) { return valid(c) ? ld_stream_v4(p4 + c * 32 + lane) : make_uint4(0, 0, 0, 0); };
        auto ldq = [&](int c) { return (two && valid(c)) ? ld_stream_v4(q4 + c * 32 + lane) : make_uint4(0, 0, 0, 0); };

        // ---- per-group masses in id order (the next group's loads in flight) ----
        // Word pairs (two tokens of each row) holding a token at or above a row's cut value
        // are queued in id order with the masks of those tokens; 32 queued pairs are weighed
        // at a time, one per lane, tokens at the cut value ranked among the row's as they come.
        const uint32_t cbp = P.cut ? obits(P.kc) : 0u, cbq = Q.cut ? obits(Q.kc) : 0u;
        const __nv_bfloat162 cp2 = bf2(cbp | (cbp << 16)), cq2 = bf2(cbq | (cbq << 16));
        uint4* qu = sh.queue[warp];
        int seen_p = 0, seen_q = 0, g = 0, nq = 0;
        double acc_d = 0.0, acc_v = 0.0, acc_r = 0.0;  // this lane's masses of the current group
        // tokens at a cut value in entries of lower lanes and before element e: kept while their
        // rank is below tie_t (m: the row's 2-bit mask of this entry, updated)
        auto rank2 = [&](uint32_t w, uint32_t& m, uint32_t cb, const RowView& R, int& seen) {
            const uint32_t t0 = (m & 1u) && (w & 0xFFFFu) == cb, t1 = ((m >> 1) & 1u) && (w >> 16) == cb;
            const unsigned any = __ballot_sync(kFullMask, t0 | t1);
            if (!any) return;
            const int c = (int)(t0 + t1);
            const int incl = warp_inclusive_scan(c, lane);
            const int r0 = R.tie_before + seen + incl - c;
            if (t0 && r0 >= R.tie_t) m &= ~1u;
            if (t1 && r0 + (int)t0 >= R.tie_t) m &= ~2u;
            seen += __shfl_sync(kFullMask, incl, 31);
        };
        // weigh queue entries [off, off + n) (n <= 32): one per lane
        auto weigh = [&](int off, int n) {
            const uint4 e = lane < n ? qu[off + lane] : make_uint4(0u, 0u, 0u, 0u);
            uint32_t mp = e.z & 3u, mq = (e.z >> 2) & 3u;
            if (P.cut) rank2(e.x, mp, cbp, P, seen_p);
            if (two && Q.cut) rank2(e.y, mq, cbq, Q, seen_q);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const double wp = (mp >> h) & 1u ? weight_of(P, (e.x >> (16 * h)) & 0xFFFFu, T) : 0.0;
                const double wq = (mq >> h) & 1u ? weight_of(Q, (e.y >> (16 * h)) & 0xFFFFu, T) : 0.0;
                acc_v += wp;
                acc_d += two ? wq : wp;
                const double dl = wp * P.iS - wq * Q.iS;
                acc_r += dl > 0.0 ? dl : 0.0;
            }
        };
        double tw[3] = {0.0, 0.0, 0.0};
        if (c0 < c1) {
            uint4 cp[kIG], cq[kIG];
#pragma unroll
            for (int u = 0; u < kIG; ++u) {
                cp[u] = ldp(c0 + u);
                cq[u] = ldq(c0 + u);
            }
            for (int c = c0;; c += kIG, ++g) {
                const bool more = c + kIG < c1;
                uint4 np[kIG], nq4[kIG];
                if (more) {
#pragma unroll
                    for (int u = 0; u < kIG; ++u) {
                        np[u] = ldp(c + kIG + u);
                        nq4[u] = ldq(c + kIG + u);
                    }
                }
                if (lane == 0) {
                    sh.gseen[warp][g][0] = seen_p;
                    sh.gseen[warp][g][1] = seen_q;
                }
#pragma unroll
                for (int u = 0; u < kIG; ++u) {
                    if (c + u >= c1) continue;  // the same in every lane
                    // this lane's word pairs with a token at or above a row's cut value
                    const uint32_t wp4[4] = {cp[u].x, cp[u].y, cp[u].z, cp[u].w};
                    const uint32_t wq4[4] = {cq[u].x, cq[u].y, cq[u].z, cq[u].w};
                    uint32_t mk[4];
                    int cnt = 0;
                    const bool ok = valid(c + u);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t a = P.cut ? (__hge2_mask(bf2(wp4[q]), cp2) >> 15) & 3u : 3u;
                        const uint32_t b2 = two ? (Q.cut ? (__hge2_mask(bf2(wq4[q]), cq2) >> 15) & 3u : 3u) : 0u;
                        mk[q] = ok ? (a | (b2 << 2)) : 0u;
                        cnt += mk[q] != 0u;
                    }
                    const int incl = warp_inclusive_scan(cnt, lane);
                    int pos = nq + incl - cnt;
                    const uint32_t id0 = (uint32_t)((c + u) * kCh + lane * 8);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (mk[q]) qu[pos++] = make_uint4(wp4[q], wq4[q], mk[q], id0 + 2 * q);
                    nq += __shfl_sync(kFullMask, incl, 31);
                    __syncwarp();
                    // weigh whole rounds of 32; the rest moves to the front
                    int done = 0;
                    for (; nq - done >= 32; done += 32) weigh(done, 32);
                    if (done > 0) {
                        const int rest = nq - done;
                        const uint4 v = lane < rest ? qu[done + lane] : make_uint4(0u, 0u, 0u, 0u);
                        __syncwarp();
                        if (lane < rest) qu[lane] = v;
                        __syncwarp();
                        nq = rest;
                    }
                }
                // the group's last queued tokens, then its masses
                if (nq > 0) {
                    weigh(0, nq);
                    nq = 0;
                }
                __syncwarp();
                const double sd = warp_sum_f64(acc_d), sv = warp_sum_f64(acc_v), sr = warp_sum_f64(acc_r);
                acc_d = acc_v = acc_r = 0.0;
                tw[0] += sd;
                tw[1] += sv;
                tw[2] += sr;
                if (lane == 0) {
                    sh.gs[warp][g][0] = sd;
                    sh.gs[warp][g][1] = sv;
                    sh.gs[warp][g][2] = sr;
                }
                if (!more) {
                    ++g;
                    break;
                }
#pragma unroll
                for (int u = 0; u < kIG; ++u) {
                    cp[u] = np[u];
                    cq[u] = nq4[u];
                }
            }
        }
        if (lane == 0) {
            sh.ng[warp] = g;
            for (int k = 0; k < 3; ++k) sh.wt[warp][k] = tw[k];
        }
        __syncthreads();
        rs_mark(p, 1, jm, 2);

        // ---- draws: the group holding the target, then the token within it ----
        // The first token whose running mass (id order) exceeds the target; if rounding
        // leaves no crossing, the last token with positive mass; -1 if there is none.
        auto draw = [&](int mode, double target) -> int {
            if (warp == 0) {
                // the warp run, then (lanes over its groups) the group
                double cacc = 0.0, clast = 0.0;
                int sw = -1, lw = -1;
                for (int w = 0; w < kWarps; ++w) {
                    const double m = sh.wt[w][mode];
                    if (!(m > 0.0)) continue;
                    lw = w;
                    clast = cacc;
                    if (cacc + m > target) {
                        sw = w;
                        break;
                    }
                    cacc += m;
                }
                const bool last_mode = sw < 0;
                const int w = last_mode ? lw : sw;
                double base = last_mode ? clast : cacc;
                int sg = -1;
                if (w >= 0) {
                    const int n = sh.ng[w];
                    const int per = (n + 31) / 32;
                    double s = 0.0;
                    int lastg = -1;
                    for (int j = 0; j < per; ++j) {
                        const int gg = lane * per + j;
                        if (gg < n && sh.gs[w][gg][mode] > 0.0) {
                            s += sh.gs[w][gg][mode];
                            lastg = gg;
                        }
                    }
                    const double incl = warp_scan_f64(s, lane);
                    const unsigned hit = last_mode ? 0u : __ballot_sync(kFullMask, s > 0.0 && base + incl > target);
                    int L;
                    if (hit) {
                        L = __ffs(hit) - 1;
                    } else {  // the last lane with mass
                        const unsigned any = __ballot_sync(kFullMask, s > 0.0);
                        L = any ? 31 - __clz(any) : -1;
                    }
                    if (L >= 0) {
                        double cg = base + __shfl_sync(kFullMask, incl - s, L);
                        int pick = -1;
                        const int lg = __shfl_sync(kFullMask, lastg, L);
                        for (int j = 0; j < per && pick < 0 && hit; ++j) {
                            const int gg = L * per + j;
                            if (gg >= n) break;
                            const double m = sh.gs[w][gg][mode];
                            if (!(m > 0.0)) continue;
                            if (cg + m > target) pick = gg;
                            else cg += m;
                        }
                        if (pick < 0) {  // no crossing (rounding, or past the end): the last group with mass
                            pick = lg;
                            cg = base + __shfl_sync(kFullMask, incl - s, L);
                            for (int j = 0; j < per; ++j) {
                                const int gg = L * per + j;
                                if (gg >= pick) break;
                                const double m = sh.gs[w][gg][mode];
                                if (m > 0.0) cg += m;
                            }
                            sh.mode = 1;
                        } else {
                            sh.mode = last_mode;
                        }
                        sg = pick;
                        base = cg;
                    }
                }
                if (lane == 0) {
                    sh.sel_w = sg >= 0 ? w : -1;
                    sh.sel_g = sg;
                    sh.sel_c = base;
                    sh.tok_found = -1;
                }
            }
            __syncthreads();
            const int sw = sh.sel_w;
            if (sw < 0) return -1;
            if (warp == sw) {
                const bool last_mode = sh.mode;
                const int sg = sh.sel_g;
                int seen_pp = sh.gseen[sw][sg][0], seen_qq = sh.gseen[sw][sg][1];
                double carry = sh.sel_c;
                int res = -1, lastpos = -1;
                const int cs = c0 + sg * kIG;
                uint4 gp[kIG], gq[kIG];
#pragma unroll
                for (int u = 0; u < kIG; ++u) {
                    gp[u] = ldp(cs + u);
                    gq[u] = ldq(cs + u);
                }
#pragma unroll
                for (int u = 0; u < kIG; ++u) {
                    const int cc = cs + u;
                    if (cc >= c1 || res >= 0) continue;  // the same in every lane
                    uint32_t mp, mq;
                    chunk_survivors(gp[u], gq[u], two, P, Q, seen_pp, seen_qq, lane, mp, mq);
                    if (!valid(cc)) mp = mq = 0u;
                    double x[8];
                    chunk_masses(gp[u], gq[u], mp, mq, two, P, Q, T, mode, x);
                    double lsum = 0.0;
#pragma unroll
                    for (int e = 0; e < 8; ++e) lsum += x[e];
                    const double incl = warp_scan_f64(lsum, lane);
                    const double before = carry + incl - lsum;
                    const unsigned hit = last_mode ? 0u : __ballot_sync(kFullMask, lsum > 0.0 && carry + incl > target);
                    if (hit) {
                        const int L = __ffs(hit) - 1;
                        int pos = -1;
                        if (lane == L) {
                            double cc2 = before;
                            for (int e = 0; e < 8 && pos < 0; ++e) {
                                if (x[e] > 0.0 && cc2 + x[e] > target) pos = e;
                                cc2 += x[e];
                            }
                            if (pos < 0)  // rounding: the lane's last positive element
                                for (int e = 7; e >= 0 && pos < 0; --e)
                                    if (x[e] > 0.0) pos = e;
                        }
                        pos = __shfl_sync(kFullMask, pos, L);
                        res = cc * kCh + L * 8 + pos;
                    }
                    unsigned posm = 0u;
#pragma unroll
                    for (int e = 0; e < 8; ++e) posm |= (x[e] > 0.0 ? 1u : 0u) << e;
                    const unsigned anyp = __ballot_sync(kFullMask, posm != 0u);
                    if (anyp) {
                        const int L = 31 - __clz(anyp);
                        const int e = 31 - __clz(__shfl_sync(kFullMask, posm, L));
                        lastpos = cc * kCh + L * 8 + e;
                    }
                    carry += __shfl_sync(kFullMask, incl, 31);
                }
                if (res < 0) res = lastpos;
                if (lane == 0) sh.tok_found = res;
            }
            __syncthreads();
            const int out = sh.tok_found;
            __syncthreads();
            return out;
        };

        const float* u = p.u + (int64_t)item * 3;
        Rec rec;
        rec.state = kDone;
        rec.pad = 0.0;
        int tok;
        if (!two) tok = pos0_given(p, b) ? p.pos0[b] : draw(0, (double)u[0] * P.S);
        else tok = p.drafts ? p.drafts[item] : draw(0, (double)u[0] * Q.S);
        rs_mark(p, 1, jm, 3);
        rec.tok = tok;
        rec.res = -1;
        rec.acc = 1;
        rec.tv = 0.0;
        rec.p = 0.0;
        rec.q = 0.0;
        // P(tok) and Q(tok): value, survival (a token at the cut value is ranked by the count
        // of those before it, one pass by the whole CTA)
        {
            const bool in = tok >= 0 && tok < V;
            double pr[2] = {0.0, 0.0};
            for (int rr = 0; rr < (two ? 2 : 1); ++rr) {
                const RowView& R = rr == 0 ? P : Q;
                const uint4* r4 = rr == 0 ? p4 : q4;
                uint32_t h = 0u;
                int state = 0;  // 0: not a survivor, 1: survivor, 2: at the cut value (rank it)
                if (in) {
                    h = reinterpret_cast<const uint16_t*>(r4)[tok];
                    if (!R.cut) state = 1;
                    else {
                        const uint32_t k = okey(h);
                        state = k > R.kc ? 1 : (k == R.kc ? 2 : 0);
                    }
                }
                if (state == 2) {
                    const uint32_t cbits = obits(R.kc);
                    int cnt = 0;
                    for (int v = tid; v < tok; v += kThreads) cnt += reinterpret_cast<const uint16_t*>(r4)[v] == cbits;
                    const double tot = cta_sum((double)cnt, sh.red);
                    state = tot < (double)R.tie_t ? 1 : 0;
                }
                if (state == 1) pr[rr] = weight_of(R, h, T) * R.iS;
            }
            rec.p = pr[0];
            rec.q = pr[1];
        }
        rs_mark(p, 1, jm, 4);
        if (two) {
            rec.acc = (double)u[1] * rec.q < rec.p;
            double R = 0.0;
            for (int w = 0; w < kWarps; ++w) R += sh.wt[w][2];
            rec.tv = R;  // TV(p, q) = sum of max(0, p - q), both distributions summing to 1
            rec.res = R > 0.0 ? draw(2, (double)u[2] * R) : draw(1, (double)u[2] * P.S);
        }
        rs_mark(p, 1, jm, 5);
        if (tid == 0) p.recs[item] = rec;
    }
    rs_end(p, 8192);
}


// ---------------------------------------------------------------------------------------
// item pass over the candidate lists (items whose rows both have complete lists)
// ---------------------------------------------------------------------------------------
// Warp w works on list segment w of both rows, which covers the same ids [c0 256, c1 256) in
// both. A list entry is bits << 16 | (0xFFFF - (id - id0)) (id0 = c0 256, bits the logit's
// bf16 bits, positive); it survives when it is above the row's threshold: its value above
// the cut value, or at it with an id below theta. The drafter's survivors go to a bitmap of
// their ids and a byte array of their table indices (id order, found through per-word
// prefix counts), which the verifier's survivors look up to weigh max(0, p - q). Each pass
// also keeps every 128-entry tile's masses, so a draw reads one tile of one segment.
constexpr int kBitWords = kMaxListV / 32;
constexpr int kMaxTiles = kListCap / kLT;

struct ListShared {
    double lut[2][kLutMax];                  // weights by table index (hM - bits): verifier, drafter
    double tm[kWarps][kMaxTiles][3];         // per tile: drafter mass, verifier mass, residual mass
    uint32_t qbits[kBitWords];               // drafter survivors by id
    uint16_t wpre[kBitWords];                // drafter survivors before each bitmap word (within its warp run)
    uint8_t qd[kWarps][kListCap];            // drafter survivors' table indices, id order, per warp run
    double ws[kWarps][3];                    // per warp run: the tiles' masses summed in order
    double sel_c;
    int sel_w, tok_found;
    int next[2];                             // the next item (alternate items use alternate slots)
};

struct ListRow {
    const uint32_t* list;   // this warp's segment
    int n;                  // its entries
    uint32_t thr;           // survivors: entries above thr
    int hM;                 // bits of the row's largest value (table index = hM - bits)
    int idtop;              // id0 + 0xFFFF (id = idtop - low half)
    int hcut, theta;        // the cut value's bits; ties survive below theta
    double iS, S;
    __device__ __forceinline__ int tix(uint32_t e) const { return hM - (int)(e >> 16); }
    __device__ __forceinline__ int id(uint32_t e) const { return idtop - (int)(e & 0xFFFFu); }
};

// a batch of kLB tiles of a segment from entry t0 (entries past n read as 0, which never
// survives: thr >= 2^16 - 1)
__device__ __forceinline__ void load_batch(const ListRow& R, int t0, uint4 (&v)[kLB], int lane) {
#pragma unroll
    for (int u = 0; u < kLB; ++u) {
        const int j = t0 + u * kLT + lane * 4;
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (j < R.n) {
            x = __ldcg(reinterpret_cast<const uint4*>(R.list + j));
            if (j + 1 >= R.n) x.y = 0u;
            if (j + 2 >= R.n) x.z = 0u;
            if (j + 3 >= R.n) x.w = 0u;
        }
        v[u] = x;
    }
}

__global__ void __launch_bounds__(kThreads, 2) item_list_kernel(Params p, const RowRec* rows, const uint32_t* lists,
                                                                 uint32_t* ctr) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ListShared& sh = *reinterpret_cast<ListShared*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int V = p.V;
    int c0, c1;
    warp_run(V, warp, c0, c1);
    const int w0 = c0 * (kCh / 32), w1 = c1 * (kCh / 32);  // this warp run's bitmap words
    const int n_items = p.B * p.K;
    int jr = 0;  // items this CTA has taken (trace)

    // items are taken from a counter (after each CTA's first, blockIdx.x)
    int par = 0;
    for (int item = blockIdx.x; item < n_items; item = sh.next[par], par ^= 1) {
        if (tid == 0) sh.next[par] = gridDim.x + (int)atomicAdd(ctr, 1u);  // read after this item's last barrier
        const int b = item / p.K, i = item % p.K;
        const bool two = i > 0;
        const RowRec& rp = rows[item];
        const RowRec& rq = rows[n_items + item];
        // trivial items: the row-reading pass writes them; items without lists: item_kernel_rs
        if (trivial_item(p, b, i) || rp.state != kDone || !rp.list_ok ||
            (two && (rq.state != kDone || !rq.list_ok))) {
            __syncthreads();
            continue;
        }
        __syncthreads();  // the previous item is done with the shared tables
        const int jm = jr++;
        rs_mark(p, 2, jm, 0);
        auto view = [&](const RowRec& rr, int r, int slot) {
            ListRow R;
            R.list = lists + ((int64_t)r * kWarps + warp) * kListCap;
            R.n = rr.list_n[warp];
            R.hM = (int)(obits(rr.kM) & 0x7FFFu);
            R.idtop = c0 * kCh + 0xFFFF;
            R.hcut = (int)(rr.A15 - (uint32_t)rr.dcut);
            R.theta = rr.theta;
            const long long trel = min(max((long long)rr.theta - (long long)c0 * kCh, 0ll), 0x10000ll);
            R.thr = (uint32_t)(((long long)R.hcut << 16) + 0xFFFF - trel);
            R.S = rr.S;
            R.iS = 1.0 / rr.S;
            for (int j = tid; j < rr.lut_n; j += kThreads) sh.lut[slot][j] = rr.lut[j];
            return R;
        };
        const ListRow P = view(rp, item, 0);
        const ListRow Q = two ? view(rq, n_items + item, 1) : P;
        for (int j = w0 + lane; j < w1; j += 32) sh.qbits[j] = 0u;
        __syncthreads();

        // ---- the drafter's survivors: bitmap, table indices in id order, tile masses ----
        if (two) {
            int nq = 0, tile = 0;
            for (int t0 = 0; t0 < Q.n; t0 += kLT * kLB) {
                uint4 v[kLB];
                load_batch(Q, t0, v, lane);
#pragma unroll
                for (int u = 0; u < kLB; ++u) {
                    if (t0 + u * kLT >= Q.n) break;  // the same in every lane
                    const uint32_t e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    uint32_t keep = 0u;
#pragma unroll
                    for (int k = 0; k < 4; ++k) keep |= (uint32_t)(e[k] > Q.thr) << k;
                    const int c = __popc(keep);
                    const int incl = warp_inclusive_scan(c, lane);
                    int pos = nq + incl - c;
                    double m = 0.0;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const bool s = (keep >> k) & 1u;
                        const uint32_t id = (uint32_t)Q.id(e[k]);
                        const int ti = Q.tix(e[k]);
                        if (s) {
                            atomicOr(&sh.qbits[id >> 5], 1u << (id & 31u));
                            sh.qd[warp][pos] = (uint8_t)ti;
                        }
                        pos += s;
                        m += s ? sh.lut[1][s ? ti : 0] : 0.0;
                    }
                    m = warp_sum_f64(m);
                    if (lane == 0) sh.tm[warp][tile][0] = m;
                    ++tile;
                    nq += __shfl_sync(kFullMask, incl, 31);
                }
            }
            __syncwarp();
            // survivors before each word of this warp run
            const int nw = w1 - w0, per = (nw + 31) / 32;
            int cnt = 0;
            for (int k = 0; k < per; ++k) {
                const int wd = w0 + lane * per + k;
                if (wd < w1) cnt += __popc(sh.qbits[wd]);
            }
            int run = warp_inclusive_scan(cnt, lane) - cnt;
            for (int k = 0; k < per; ++k) {
                const int wd = w0 + lane * per + k;
                if (wd < w1) {
                    sh.wpre[wd] = (uint16_t)run;
                    run += __popc(sh.qbits[wd]);
                }
            }
            __syncwarp();
        }
        rs_mark(p, 2, jm, 1);
        // the drafter's weight of a verifier survivor's id (0 if the drafter does not keep it;
        // s false: not a survivor, and the entry may be padding, whose id is out of range)
        auto q_of = [&](uint32_t e, bool s) -> double {
            const uint32_t id = s ? (uint32_t)P.id(e) : (uint32_t)(c0 * kCh);
            const uint32_t word = sh.qbits[id >> 5], bit = 1u << (id & 31u);
            const bool has = s && (word & bit);
            const int kq = has ? sh.wpre[id >> 5] + __popc(word & (bit - 1u)) : 0;
            const double wq = sh.lut[1][sh.qd[warp][kq]];
            return has ? wq : 0.0;
        };

        // ---- the verifier's survivors: tile masses and residual masses (branch-free) ----
        {
            int tile = 0;
            for (int t0 = 0; t0 < P.n; t0 += kLT * kLB) {
                uint4 v[kLB];
                load_batch(P, t0, v, lane);
#pragma unroll
                for (int u = 0; u < kLB; ++u) {
                    if (t0 + u * kLT >= P.n) break;
                    const uint32_t e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    double mp = 0.0, mr = 0.0;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const bool s = e[k] > P.thr;
                        const double wp = sh.lut[0][s ? P.tix(e[k]) : 0];
                        mp += s ? wp : 0.0;
                        if (two) {
                            const double dl = wp * P.iS - q_of(e[k], s) * Q.iS;
                            mr += (s && dl > 0.0) ? dl : 0.0;
                        }
                    }
                    mp = warp_sum_f64(mp);
                    if (two) mr = warp_sum_f64(mr);
                    if (lane == 0) {
                        sh.tm[warp][tile][1] = mp;
                        sh.tm[warp][tile][2] = mr;
                    }
                    ++tile;
                }
            }
            __syncwarp();
            if (lane < 3) {  // the warp run's masses: its tiles' in order
                const int nt = (lane == 0 ? Q.n : P.n) + kLT - 1;
                double s = 0.0;
                if (lane != 2 || two)
                    for (int u = 0; u < nt / kLT; ++u) s += sh.tm[warp][u][lane];
                sh.ws[warp][lane] = s;
            }
        }
        __syncthreads();
        rs_mark(p, 2, jm, 2);

        // ---- draws: the warp run, then the tile, holding the target; then the token ----
        // col 0: the drafter's survivors, 1: the verifier's, 2: the residual. The first token
        // whose running mass (id order) exceeds the target; if rounding leaves no crossing,
        // the last token with positive mass; -1 if there is none.
        auto draw = [&](int col, double target) -> int {
            if (tid == 0) {
                double cacc = 0.0, clast = 0.0;
                int sw = -1, lw = -1;
                for (int w = 0; w < kWarps; ++w) {
                    const double m = sh.ws[w][col];
                    if (!(m > 0.0)) continue;
                    lw = w;
                    clast = cacc;
                    if (cacc + m > target) {
                        sw = w;
                        break;
                    }
                    cacc += m;
                }
                sh.sel_w = sw < 0 ? lw : sw;
                sh.sel_c = sw < 0 ? clast : cacc;
                sh.tok_found = -1;
            }
            __syncthreads();
            if (warp == sh.sel_w) {
                const ListRow R = col == 0 ? Q : P;  // (a copy: both stay in registers)
                const int nt = (R.n + kLT - 1) / kLT;
                double carry = sh.sel_c;
                int tf = -1, tl = -1;  // the tile with the crossing; the last tile with mass
                for (int u = 0; u < nt; ++u) {
                    const double m = sh.tm[warp][u][col];
                    if (!(m > 0.0)) continue;
                    tl = u;
                    if (carry + m > target) {
                        tf = u;
                        break;
                    }
                    carry += m;
                }
                int res = -1;
                const int u = tf >= 0 ? tf : tl;
                if (u >= 0) {
                    const int j = u * kLT + lane * 4;
                    uint4 x4 = make_uint4(0u, 0u, 0u, 0u);
                    if (j < R.n) {
                        x4 = __ldcg(reinterpret_cast<const uint4*>(R.list + j));
                        if (j + 1 >= R.n) x4.y = 0u;
                        if (j + 2 >= R.n) x4.z = 0u;
                        if (j + 3 >= R.n) x4.w = 0u;
                    }
                    const uint32_t e[4] = {x4.x, x4.y, x4.z, x4.w};
                    double x[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const bool s = e[k] > R.thr;
                        const double w = sh.lut[col == 0 ? 1 : 0][s ? R.tix(e[k]) : 0];
                        double m = s ? w : 0.0;
                        if (col == 2) {
                            const double dl = w * P.iS - q_of(e[k], s) * Q.iS;
                            m = (s && dl > 0.0) ? dl : 0.0;
                        }
                        x[k] = m;
                    }
                    const double s = (x[0] + x[1]) + (x[2] + x[3]);
                    const double incl = warp_scan_f64(s, lane);
                    int cross = -1, lastk = -1;
                    double run = carry + (incl - s);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (x[k] > 0.0) {
                            run += x[k];
                            lastk = R.id(e[k]);
                            if (cross < 0 && run > target) cross = lastk;
                        }
                    const unsigned hit = tf >= 0 ? __ballot_sync(kFullMask, cross >= 0) : 0u;
                    const unsigned pos = __ballot_sync(kFullMask, lastk >= 0);
                    if (hit) res = __shfl_sync(kFullMask, cross, __ffs(hit) - 1);
                    else if (pos) res = __shfl_sync(kFullMask, lastk, 31 - __clz(pos));
                }
                if (lane == 0) sh.tok_found = res;
            }
            __syncthreads();
            const int out = sh.tok_found;
            __syncthreads();
            return out;
        };

        const float* u = p.u + (int64_t)item * 3;
        double Rm = 0.0;  // TV(p, q) = sum of max(0, p - q), both distributions summing to 1
        for (int w = 0; w < kWarps; ++w) Rm += sh.ws[w][2];
        Rec rec;
        rec.state = kDone;
        rec.pad = 0.0;
        rec.res = -1;
        rec.tv = two ? Rm : 0.0;
        const bool given = !two ? pos0_given(p, b) : p.drafts != nullptr;
        int tok = !given ? -1 : (!two ? p.pos0[b] : p.drafts[item]);
        // the draws (one call site keeps the code small): s = 0 the token, unless it is given;
        // s = 1 the residual draw (two rows), from p itself if max(0, p - q) has no mass
        for (int s = 0; s < 2; ++s) {
            if (s == 0 && given) continue;
            if (s == 1 && !two) break;
            const int col = s == 0 ? (two ? 0 : 1) : (Rm > 0.0 ? 2 : 1);
            const double target = s == 0 ? (double)u[0] * (two ? Q.S : P.S) : (double)u[2] * (Rm > 0.0 ? Rm : P.S);
            const int got = draw(col, target);
            if (s == 0) tok = got;
            else rec.res = got;
        }
        rs_mark(p, 2, jm, 3);
        rec.tok = tok;
        // p(tok), q(tok) from the logits: survivors by the same rule as the lists'
        auto prob = [&](const ListRow& R, int r, int slot) -> double {
            if (tok < 0 || tok >= V) return 0.0;
            const __nv_bfloat16* row = r < n_items ? static_cast<const __nv_bfloat16*>(p.P) + (int64_t)r * V
                                                   : static_cast<const __nv_bfloat16*>(p.Q) + (int64_t)(r - n_items) * V;
            const int h = (int)reinterpret_cast<const uint16_t*>(row)[tok];
            if (h & 0x8000) return 0.0;  // negative: below the window (whose floor is positive)
            if (h < R.hcut || (h == R.hcut && tok >= R.theta) || h > R.hM) return 0.0;
            return sh.lut[slot][R.hM - h] * R.iS;
        };
        rec.p = prob(P, item, 0);
        rec.q = two ? prob(Q, n_items + item, 1) : 0.0;
        rec.acc = two ? (double)u[1] * rec.q < rec.p : 1;
        if (tid == 0) p.recs[item] = rec;
        rs_mark(p, 2, jm, 4);
    }
    rs_end(p, 7168);
}

}  // namespace rs

// =======================================================================================
// per sequence: the longest accepted prefix and the outputs
// =======================================================================================
__global__ void assemble_kernel(Params p, int32_t* out_tokens, int32_t* out_count, int32_t* out_next, float* out_p,
                                float* out_q, float* out_tv) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= p.B) return;
    const int K = p.K;
    const Rec* r = p.recs + (int64_t)b * K;
    int n = 1;
    while (n < K && r[n].acc) ++n;
    for (int i = 0; i < K; ++i) {
        const int64_t o = (int64_t)b * K + i;
        out_tokens[o] = i < n ? r[i].tok : -1;
        if (out_p) out_p[o] = (float)r[i].p;
        if (out_q) out_q[o] = (float)r[i].q;
        if (out_tv) out_tv[o] = (float)r[i].tv;
    }
    out_count[b] = n;
    if (out_next) out_next[b] = n < K ? r[n].res : -1;
}

// =======================================================================================
// host side
// =======================================================================================
inline bool tracing() { return getenv("UNO_VERIFY_TRACE") != nullptr; }
// the records, then (UNO_VERIFY_TRACE set) the phase-timestamp trace
inline size_t recs_bytes(const VerifyArgs& a) {
    return align_up((size_t)a.B * a.K * sizeof(Rec), 256) + (tracing() ? kTraceBytes : 0);
}

// the team layout for cluster size CL; top_k > 0 selects the top-k mode
pk::Layout make_layout(int V, int CL, int top_k) {
    pk::Layout Ly{};
    Ly.CL = CL;
    Ly.L = (int)(((int64_t)V + (int64_t)CL * 8 - 1) / ((int64_t)CL * 8) * 8);
    Ly.hw = top_k > 0 ? pk::kWinK : pk::kWords;
    Ly.OW = Ly.hw / CL;
    Ly.KL = 0;
    if (top_k > 0) {
        Ly.KL = 32;
        while (Ly.KL < top_k) Ly.KL <<= 1;
    }
    uint32_t off = (uint32_t)align_up((size_t)Ly.L * 2 * 2, 16);
    Ly.off_hist = off;
    off += (uint32_t)(2 * Ly.hw * 4);
    Ly.off_own = off;
    off += (uint32_t)(2 * Ly.OW * 8);
    Ly.off_lut = off;
    off += top_k > 0 ? 0u : 2u * pk::kLut * 8u;
    Ly.off_list = off;
    off += (uint32_t)(2 * Ly.KL * (8 + 8 + 8 + 4));
    off = (uint32_t)align_up(off, 16);
    Ly.off_x1 = off;
    off += pk::kMaxCL * 8;
    Ly.off_x2 = off;
    off += pk::kMaxCL * 6 * 8;
    Ly.off_x3 = off;
    off += pk::kMaxCL * 3 * 8;
    Ly.off_misc = off;
    off += (uint32_t)align_up(sizeof(pk::TeamShared), 16);
    Ly.team_bytes = (uint32_t)align_up(off, 128);
    return Ly;
}

// the team layout of topk_local_kernel for cluster size CL
pk::LLayout make_llayout(int V, int CL, int top_k) {
    pk::LLayout Ly{};
    Ly.CL = CL;
    Ly.L = (int)(((int64_t)V + (int64_t)CL * 8 - 1) / ((int64_t)CL * 8) * 8);
    Ly.KL = 32;
    while (Ly.KL < top_k) Ly.KL <<= 1;
    const uint32_t KL = (uint32_t)Ly.KL;
    uint32_t off = (uint32_t)align_up((size_t)Ly.L * 2 * 2, 16);
    Ly.off_hist = off;
    off += 2 * pk::kWinK * 4;
    Ly.off_loc = off;
    off += 2 * KL * 8;
    Ly.off_cand = off;
    off += 2 * (uint32_t)CL * KL * 8;
    Ly.off_cnt = off;
    off += 2 * pk::kMaxCL * 4;
    Ly.off_merged = off;
    off += 2 * KL * 8;
    Ly.off_w = off;
    off += 2 * KL * 8;
    Ly.off_id = off;
    off += 2 * KL * 4;
    off = (uint32_t)align_up(off, 16);
    Ly.off_tmp = off;
    off += 2 * KL * 8;
    Ly.off_misc = off;
    off += (uint32_t)align_up(sizeof(pk::LShared), 16);
    Ly.team_bytes = (uint32_t)align_up(off, 128);
    return Ly;
}

struct DeviceInfo {
    bool ready = false;
    size_t dyn_max = 0;
    std::map<std::tuple<int, int, size_t>, int> max_clusters;  // (mode, cluster size, smem) -> resident clusters
};
std::mutex g_mu;
DeviceInfo g_dev[64];

struct DeviceInfo;
bool launch_local(const VerifyArgs& a, const Params& p, cudaStream_t stream, uno_status& st, DeviceInfo& di,
                  int forced, bool required);

template <bool TOPK>
bool set_attributes(int dyn_max) {
    return cudaFuncSetAttribute(pk::pair_kernel<TOPK>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max) ==
               cudaSuccess &&
           cudaFuncSetAttribute(pk::pair_kernel<TOPK>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
               cudaSuccess;
}

// Launch pair_kernel where it applies; false (with st untouched) to leave every item to the
// generic kernel. UNO_VERIFY_FULL=generic always leaves them; UNO_VERIFY_FULL=cluster makes a
// case the pair kernel cannot take an error. UNO_VERIFY_FULL_CLUSTER=c forces the cluster size.
bool launch_pairs(const VerifyArgs& a, const Params& p, cudaStream_t stream, uno_status& st) {
    const char* mode = getenv("UNO_VERIFY_FULL");
    if (mode && strcmp(mode, "generic") == 0) return false;
    const bool required = mode && strcmp(mode, "cluster") == 0;
    auto no = [&](const char* why) {
        if (required) st = set_error(UNO_ERR_UNSUPPORTED, "verify: no cluster form: %s", why);
        return required;
    };
    if (a.dtype != UNO_BF16 || a.V % 8 != 0) return no("bf16 rows whose length is a multiple of 8 only");
    if (a.top_k > pk::kMaxTopK) return no("top-k above 256");
    if ((reinterpret_cast<uintptr_t>(a.P) | reinterpret_cast<uintptr_t>(a.Q)) & 15u)
        return no("logits must be 16-byte aligned");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return no("no current device");
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& di = g_dev[dev];
    if (!di.ready) {
        int optin = 0;
        cudaFuncAttributes fa{}, fb{};
        if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaFuncGetAttributes(&fa, pk::pair_kernel<false>) != cudaSuccess ||
            cudaFuncGetAttributes(&fb, pk::pair_kernel<true>) != cudaSuccess) {
            cudaGetLastError();
            return no("shared memory attributes unavailable");
        }
        cudaFuncAttributes fc{};
        if (cudaFuncGetAttributes(&fc, pk::topk_local_kernel) != cudaSuccess) {
            cudaGetLastError();
            return no("shared memory attributes unavailable");
        }
        const int stat = (int)std::max(std::max(fa.sharedSizeBytes, fb.sharedSizeBytes), fc.sharedSizeBytes);
        if (optin <= stat) return no("shared memory attributes unavailable");
        const int dyn_max = optin - stat;
        if (!set_attributes<false>(dyn_max) || !set_attributes<true>(dyn_max) ||
            cudaFuncSetAttribute(pk::topk_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max) !=
                cudaSuccess ||
            cudaFuncSetAttribute(pk::topk_local_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess) {
            cudaGetLastError();
            return no("kernel attributes refused");
        }
        di.dyn_max = (size_t)dyn_max;
        di.ready = true;
    }
    int forced = 0;
    if (const char* e = getenv("UNO_VERIFY_FULL_CLUSTER")) forced = atoi(e);
    // top-k up to kMaxLocalK: per-CTA top-k lists merged by a head CTA (UNO_VERIFY_TOPK=window
    // selects the cluster-wide cut of pair_kernel instead)
    const char* tmode = getenv("UNO_VERIFY_TOPK");
    if (a.top_k > 0 && a.top_k <= pk::kMaxLocalK && !(tmode && strcmp(tmode, "window") == 0))
        return launch_local(a, p, stream, st, di, forced, required);
    int CL = 0;
    pk::Layout Ly{};
    for (int c = 1; c <= pk::kMaxCL; c *= 2) {
        if (forced && c != forced) continue;
        const pk::Layout t = make_layout(a.V, c, a.top_k);
        if (t.L >= 65536) continue;  // per-CTA counts are 16-bit
        if ((size_t)t.team_bytes * pk::kTeams <= di.dyn_max) {
            CL = c;
            Ly = t;
            break;
        }
    }
    if (CL == 0) return no("the row slices do not fit in the shared memory of any cluster size");
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(pk::kThreads);
    cfg.dynamicSmemBytes = (size_t)Ly.team_bytes * pk::kTeams;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const bool topk = a.top_k > 0;
    const auto key = std::make_tuple((int)topk, CL, cfg.dynamicSmemBytes);
    int maxc = 0;
    const auto found = di.max_clusters.find(key);
    if (found != di.max_clusters.end()) {
        maxc = found->second;
    } else {
        cudaLaunchConfig_t q = cfg;
        q.gridDim = dim3((unsigned)CL);
        const cudaError_t e = topk ? cudaOccupancyMaxActiveClusters(&maxc, pk::pair_kernel<true>, &q)
                                   : cudaOccupancyMaxActiveClusters(&maxc, pk::pair_kernel<false>, &q);
        if (e != cudaSuccess) {
            cudaGetLastError();
            maxc = 0;
        }
        di.max_clusters[key] = maxc;
    }
    if (maxc <= 0) return no("no cluster of this size can be resident");
    const int64_t items = (int64_t)a.B * a.K;
    const int64_t clusters = std::min<int64_t>((items + pk::kTeams - 1) / pk::kTeams, (int64_t)maxc);
    cfg.gridDim = dim3((unsigned)(clusters * CL));
    const cudaError_t e = topk ? cudaLaunchKernelEx(&cfg, pk::pair_kernel<true>, p, Ly)
                               : cudaLaunchKernelEx(&cfg, pk::pair_kernel<false>, p, Ly);
    st = check_cuda(e, "launch(verify, pairs)");
    return true;
}

// topk_local_kernel: the smallest cluster size whose two team layouts fit
bool launch_local(const VerifyArgs& a, const Params& p, cudaStream_t stream, uno_status& st, DeviceInfo& di,
                  int forced, bool required) {
    auto no = [&](const char* why) {
        if (required) st = set_error(UNO_ERR_UNSUPPORTED, "verify: no cluster form: %s", why);
        return required;
    };
    int CL = 0;
    pk::LLayout Ly{};
    for (int c = 1; c <= pk::kMaxCL; c *= 2) {
        if (forced && c != forced) continue;
        const pk::LLayout t = make_llayout(a.V, c, a.top_k);
        if ((size_t)t.team_bytes * pk::kTeams <= di.dyn_max) {
            CL = c;
            Ly = t;
            break;
        }
    }
    if (CL == 0) return no("the row slices do not fit in the shared memory of any cluster size");
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(pk::kThreads);
    cfg.dynamicSmemBytes = (size_t)Ly.team_bytes * pk::kTeams;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const auto key = std::make_tuple(2, CL, cfg.dynamicSmemBytes);
    int maxc = 0;
    const auto found = di.max_clusters.find(key);
    if (found != di.max_clusters.end()) {
        maxc = found->second;
    } else {
        cudaLaunchConfig_t q = cfg;
        q.gridDim = dim3((unsigned)CL);
        if (cudaOccupancyMaxActiveClusters(&maxc, pk::topk_local_kernel, &q) != cudaSuccess) {
            cudaGetLastError();
            maxc = 0;
        }
        di.max_clusters[key] = maxc;
    }
    if (maxc <= 0) return no("no cluster of this size can be resident");
    const int64_t items = (int64_t)a.B * a.K;
    const int64_t clusters = std::min<int64_t>((items + pk::kTeams - 1) / pk::kTeams, (int64_t)maxc);
    cfg.gridDim = dim3((unsigned)(clusters * CL));
    st = check_cuda(cudaLaunchKernelEx(&cfg, pk::topk_local_kernel, p, Ly), "launch(verify, local top-k)");
    return true;
}

// The row-streaming path takes bf16 rows, 16-byte aligned, V a multiple of 8 (and at most
// the groups its item pass keeps sums for), top-k off; UNO_VERIFY_FULL=generic or =cluster
// selects another path.
bool rs_applies(const VerifyArgs& a) {
    const char* mode = getenv("UNO_VERIFY_FULL");
    if (mode && (strcmp(mode, "generic") == 0 || strcmp(mode, "cluster") == 0)) return false;
    const int64_t vmax = (int64_t)rs::kWarps * rs::kMaxIGroups * rs::kIG * rs::kCh;
    return a.top_k == 0 && a.dtype == UNO_BF16 && a.V % 8 == 0 && (int64_t)a.V <= vmax &&
           ((reinterpret_cast<uintptr_t>(a.P) | reinterpret_cast<uintptr_t>(a.Q)) & 15u) == 0;
}

int num_sms();

uno_status launch_rs(const VerifyArgs& a, const Params& p, rs::RowRec* rows, uint32_t* ctr, uint32_t* lists,
                     cudaStream_t stream) {
    static std::mutex mu;
    static bool ready[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return set_error(UNO_ERR_CUDA, "verify: no device");
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!ready[dev]) {
            uno_status s;
            if ((s = check_cuda(cudaFuncSetAttribute(rs::row_kernel<rs::kRowCtasPerSm>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(rs::RowShared)),
                                "cudaFuncSetAttribute(verify rows)")) != UNO_OK)
                return s;
            if ((s = check_cuda(cudaFuncSetAttribute(rs::row_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)sizeof(rs::RowShared)),
                                "cudaFuncSetAttribute(verify rows)")) != UNO_OK)
                return s;
            if ((s = check_cuda(cudaFuncSetAttribute(rs::item_kernel_rs, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)sizeof(rs::ItemShared)),
                                "cudaFuncSetAttribute(verify items)")) != UNO_OK)
                return s;
            if ((s = check_cuda(cudaFuncSetAttribute(rs::item_list_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)sizeof(rs::ListShared)),
                                "cudaFuncSetAttribute(verify list items)")) != UNO_OK)
                return s;
            ready[dev] = true;
        }
    }
    const int items = a.B * a.K;
    const int slots = num_sms() * rs::kCtasPerSm;
    // UNO_VERIFY_LISTS=off: every item weighed from the logits by item_kernel_rs
    const char* lm = getenv("UNO_VERIFY_LISTS");
    if (lists == nullptr || a.V > rs::kMaxListV || (lm && strcmp(lm, "off") == 0)) lists = nullptr;
    uno_status s = check_cuda(cudaMemsetAsync(ctr, 0, 2 * sizeof(uint32_t), stream), "verify: counters");
    if (s != UNO_OK) return s;
    const char* rc = getenv("UNO_VERIFY_ROW_CTAS");
    if (rc && strcmp(rc, "2") == 0)
        rs::row_kernel<2><<<(unsigned)std::min(2 * items, num_sms() * 2), rs::kThreads, sizeof(rs::RowShared), stream>>>(
            p, rows, lists, ctr);
    else
        rs::row_kernel<rs::kRowCtasPerSm><<<(unsigned)std::min(2 * items, num_sms() * rs::kRowCtasPerSm), rs::kThreads,
                                            sizeof(rs::RowShared), stream>>>(p, rows, lists, ctr);
    if ((s = check_cuda(cudaGetLastError(), "launch(verify rows)")) != UNO_OK) return s;
    if (lists != nullptr) {
        rs::item_list_kernel<<<(unsigned)std::min(items, 2 * num_sms()), rs::kThreads, sizeof(rs::ListShared), stream>>>(
            p, rows, lists, ctr + 1);
        if ((s = check_cuda(cudaGetLastError(), "launch(verify list items)")) != UNO_OK) return s;
    }
    rs::item_kernel_rs<<<(unsigned)std::min(items, slots), rs::kThreads, sizeof(rs::ItemShared), stream>>>(p, rows);
    return check_cuda(cudaGetLastError(), "launch(verify items)");
}

int num_sms() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 1;
    }
    return n;
}

}  // namespace vfull

// the row records of the row-streaming path and its two work counters
inline size_t rs_rows_bytes(const VerifyArgs& a) {
    return align_up((size_t)2 * a.B * a.K * sizeof(vfull::rs::RowRec) + 2 * sizeof(uint32_t), 256);
}

// the records, then (top-k off) the row records of the row-streaming path and, with
// with_lists, the rows' candidate lists (without them every item is weighed from the logits)
size_t verify_full_workspace_bytes(const VerifyArgs& a, bool with_lists) {
    size_t n = align_up(vfull::recs_bytes(a), 256);
    if (a.top_k == 0) {
        n += rs_rows_bytes(a);
        if (with_lists && a.V <= vfull::rs::kMaxListV)
            n += (size_t)2 * a.B * a.K * vfull::rs::kWarps * vfull::rs::kListCap * 4;
    }
    return n;
}

// The item path: pair_kernel where it applies, the generic kernel for the rest, then the
// per-sequence assembly. With allow_generic false (top-k on: the streaming path serves the
// cases pair_kernel does not take) nothing is launched unless pair_kernel takes the batch.
uno_status verify_full_launch(const VerifyArgs& a, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                              bool allow_generic, bool* taken) {
    vfull::Params p{};
    p.P = a.P;
    p.Q = a.Q;
    p.B = a.B;
    p.K = a.K;
    p.V = a.V;
    p.T = (double)a.temperature;
    p.cut = a.top_p < 1.0f;
    p.top_p = (double)a.top_p;
    p.top_k = a.top_k;
    p.need_p0 = a.out_p != nullptr;
    p.drafts = a.drafts;
    p.pos0 = a.pos0;
    p.u = a.u;
    p.recs = static_cast<vfull::Rec*>(workspace);
    p.status = device_status_ptr();
    p.trace = vfull::tracing() ? reinterpret_cast<unsigned long long*>(
                                     static_cast<unsigned char*>(workspace) +
                                     align_up((size_t)a.B * a.K * sizeof(vfull::Rec), 256))
                               : nullptr;
    uno_status st = UNO_OK;
    int only_redo = 0;
    if (vfull::rs_applies(a)) {
        unsigned char* w8 = static_cast<unsigned char*>(workspace) + align_up(vfull::recs_bytes(a), 256);
        auto* rows = reinterpret_cast<vfull::rs::RowRec*>(w8);
        auto* ctr = reinterpret_cast<uint32_t*>(w8 + (size_t)2 * a.B * a.K * sizeof(vfull::rs::RowRec));
        auto* lists = workspace_bytes >= verify_full_workspace_bytes(a, true)
                          ? reinterpret_cast<uint32_t*>(w8 + rs_rows_bytes(a))
                          : nullptr;
        if ((st = vfull::launch_rs(a, p, rows, ctr, lists, stream)) != UNO_OK) return st;
        only_redo = 1;
    } else if (vfull::launch_pairs(a, p, stream, st)) {
        if (st != UNO_OK) return st;
        only_redo = 1;
    } else if (!allow_generic) {
        *taken = false;
        return UNO_OK;
    }
    *taken = true;
    const int items = a.B * a.K;
    const unsigned grid = (unsigned)std::min(items, 2 * vfull::num_sms());
    if (a.dtype == UNO_BF16)
        vfull::gen::item_kernel<__nv_bfloat16><<<grid, vfull::gen::kThreads, 0, stream>>>(p, only_redo);
    else
        vfull::gen::item_kernel<float><<<grid, vfull::gen::kThreads, 0, stream>>>(p, only_redo);
    if ((st = check_cuda(cudaGetLastError(), "launch(verify, generic)")) != UNO_OK) return st;
    vfull::assemble_kernel<<<(unsigned)((a.B + 127) / 128), 128, 0, stream>>>(p, a.out_tokens, a.out_count, a.out_next,
                                                                             a.out_p, a.out_q, a.out_tv);
    return check_cuda(cudaGetLastError(), "launch(verify, assemble)");
}

}  // namespace uno
