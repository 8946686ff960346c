// tv_loss.cu — TV self-distillation loss and its gradient w.r.t. the student logits.
//
// LoopUno project page, "Training is self-distillation": the loss is the total-variation
// distance between the frozen teacher's next-token distribution (clean copy) and the
// student's (model + LoRA on the block-noised copy) on the response tokens.
//   p = softmax(teacher), q = softmax(student); TV = 1/2 sum |p - q|
//   mean = sum_{masked} TV / N_mask
//   dmean/dstudent_v = q_v (s_v - sum_w q_w s_w) / N_mask,  s = 1/2 sign(q - p)
//
// Three kernels compute the same thing.
//
// cluster_kernel (bf16 rows whose length is a multiple of 8 elements, the common case):
// a thread-block cluster of CL CTAs owns one (teacher, student) row pair at a time, each
// CTA holding a 1/CL slice of both rows in shared memory, so every logit is read from HBM
// exactly once. The slices arrive by bulk copies (mbarrier completion) issued one row
// ahead, so the next row streams in while this one is computed. Per row: warp maxima and
// exps of both rows -> cluster reduction of the (max, sum) pairs; A = sum of q over q > p
// and P = sum of p over q > p -> cluster reduction; gradient. Each reduction is a per-warp
// st.async of its partial into every CTA of the cluster. Rows overlap: row i's second
// reduction is in flight while the warps take row i + 1's maxima and exps, and row i + 1's
// first while they write row i's gradient. exp(student) is either kept in shared memory
// from the exp pass to the A, P pass (KEEP: 4 exponentials per element pair, 12 bytes of
// shared memory per element) or recomputed there too (5 exponentials, 8 bytes, so a
// smaller cluster fits: clusters of 6 at a 152k vocabulary). 6 bytes of HBM traffic per
// element pair either way.
//
// team_kernel: the cluster kernel's computation with two teams of warps per CTA on
// alternate rows (a variant; see its own comment).
//
// rows_kernel (fp32 rows, unaligned rows, rows too long for the cluster's shared memory):
// one CTA per token row. Pass 1 streams both rows from HBM once and keeps per-thread
// online (max, sum); pass 2 re-reads them (L2) for sum |p - q| and c = sum q s; pass 3
// re-reads them and writes the gradient.
//
// A tiny pre-kernel counts the mask; the CTA that finishes the last row (atomic counter,
// no waiting) writes the mean.
#include <cuda_bf16.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "tv_loss.cuh"
#include "verify_common.cuh"

namespace uno {
namespace tvk {

constexpr int kThreads = 1024;

struct Work {
    double sum_tv;
    uint32_t n_mask;
    uint32_t done;
};

struct Params {
    TVArgs a;
    Work* work;
    uint32_t* status;
};

__global__ void count_mask_kernel(const uint8_t* mask, int64_t N, Work* work) {
    __shared__ uint32_t s;
    if (threadIdx.x == 0) s = 0;
    __syncthreads();
    uint32_t c = 0;
    for (int64_t i = threadIdx.x; i < N; i += blockDim.x) c += mask ? (mask[i] != 0) : 1u;
    atomicAdd(&s, c);
    __syncthreads();
    if (threadIdx.x == 0) {
        work->n_mask = s;
        work->sum_tv = 0.0;
        work->done = 0;
    }
}

__device__ __forceinline__ void online_add(float& m, float& s, float x) {
    if (x > m) {
        s = s * __expf(m - x) + 1.0f;
        m = x;
    } else {
        s += __expf(x - m);
    }
}

__device__ __forceinline__ void combine(float& m, float& s, float m2, float s2) {
    if (m2 > m) {
        s = s * __expf(m - m2) + s2;
        m = m2;
    } else if (m2 > -INFINITY) {
        s += s2 * __expf(m2 - m);
    }
}

template <typename T>
__device__ __forceinline__ void lane_load(const T* row, int64_t e0, int nvalid, bool aligned, float (&x)[Elem<T>::VEC]) {
    float vm;
    load_lane<T>(row, e0, nvalid, aligned, x, vm);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) rows_kernel(Params p) {
    using E = Elem<T>;
    constexpr int VEC = E::VEC;
    constexpr int NW = kThreads / 32;
    const TVArgs& a = p.a;
    const int64_t r = blockIdx.x;
    const int64_t V = a.V;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const T* trow = reinterpret_cast<const T*>(a.teacher) + r * V;
    const T* srow = reinterpret_cast<const T*>(a.student) + r * V;
    const bool aligned = ((reinterpret_cast<uintptr_t>(trow) | reinterpret_cast<uintptr_t>(srow)) & 15u) == 0;
    const int64_t nvec = (V + VEC - 1) / VEC;

    __shared__ float s_m[2][NW], s_s[2][NW];
    __shared__ double s_d[NW], s_c[NW];
    __shared__ float s_stat[4];
    __shared__ double s_red[2];

    // ---- pass 1: online max / sum of exp for teacher and student ----
    float mt = -INFINITY, st = 0.f, ms = -INFINITY, ss = 0.f;
    for (int64_t v = tid; v < nvec; v += kThreads) {
        int64_t e0 = v * VEC;
        int nv = (int)min((int64_t)VEC, V - e0);
        float xt[VEC], xs[VEC];
        lane_load<T>(trow, e0, nv, aligned, xt);
        lane_load<T>(srow, e0, nv, aligned, xs);
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            if (j < nv) {
                online_add(mt, st, xt[j]);
                online_add(ms, ss, xs[j]);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        combine(mt, st, __shfl_xor_sync(kFullMask, mt, o), __shfl_xor_sync(kFullMask, st, o));
        combine(ms, ss, __shfl_xor_sync(kFullMask, ms, o), __shfl_xor_sync(kFullMask, ss, o));
    }
    if (lane == 0) {
        s_m[0][warp] = mt; s_s[0][warp] = st;
        s_m[1][warp] = ms; s_s[1][warp] = ss;
    }
    __syncthreads();
    if (warp == 0) {
        for (int h = 0; h < 2; ++h) {
            float m = lane < NW ? s_m[h][lane] : -INFINITY;
            float s = lane < NW ? s_s[h][lane] : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                combine(m, s, __shfl_xor_sync(kFullMask, m, o), __shfl_xor_sync(kFullMask, s, o));
            if (lane == 0) {
                s_stat[2 * h] = m;
                s_stat[2 * h + 1] = 1.0f / s;
            }
        }
    }
    __syncthreads();
    const float Mt = s_stat[0], iSt = s_stat[1], Ms = s_stat[2], iSs = s_stat[3];

    // ---- pass 2: sum |p - q| and c = sum q * s ----
    float d = 0.f, c = 0.f;
    for (int64_t v = tid; v < nvec; v += kThreads) {
        int64_t e0 = v * VEC;
        int nv = (int)min((int64_t)VEC, V - e0);
        float xt[VEC], xs[VEC];
        lane_load<T>(trow, e0, nv, aligned, xt);
        lane_load<T>(srow, e0, nv, aligned, xs);
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            if (j < nv) {
                float pv = __expf(xt[j] - Mt) * iSt;
                float qv = __expf(xs[j] - Ms) * iSs;
                d += fabsf(pv - qv);
                c += qv > pv ? 0.5f * qv : (qv < pv ? -0.5f * qv : 0.f);
            }
        }
    }
    d = warp_sum(d);
    c = warp_sum(c);
    if (lane == 0) {
        s_d[warp] = d;
        s_c[warp] = c;
    }
    __syncthreads();
    if (warp == 0) {
        double dd = lane < NW ? s_d[lane] : 0.0, cc = lane < NW ? s_c[lane] : 0.0;
        dd = warp_sum(dd);
        cc = warp_sum(cc);
        if (lane == 0) {
            s_red[0] = 0.5 * dd;
            s_red[1] = cc;
        }
    }
    __syncthreads();
    const double tv = s_red[0];
    const float cq = (float)s_red[1];
    const bool on = a.mask == nullptr || a.mask[r] != 0;
    const uint32_t n_mask = p.work->n_mask;

    // ---- pass 3: gradient ----
    if (a.grad) {
        const float f = (on && n_mask > 0) ? a.grad_scale / (float)n_mask : 0.f;
        T* grow = reinterpret_cast<T*>(a.grad) + r * V;
        const bool galigned = aligned && ((reinterpret_cast<uintptr_t>(grow) & 15u) == 0);
        for (int64_t v = tid; v < nvec; v += kThreads) {
            int64_t e0 = v * VEC;
            int nv = (int)min((int64_t)VEC, V - e0);
            float xt[VEC], xs[VEC], g[VEC];
            if (f != 0.f) {
                lane_load<T>(trow, e0, nv, aligned, xt);
                lane_load<T>(srow, e0, nv, aligned, xs);
#pragma unroll
                for (int j = 0; j < VEC; ++j) {
                    float pv = __expf(xt[j] - Mt) * iSt;
                    float qv = __expf(xs[j] - Ms) * iSs;
                    float sg = qv > pv ? 0.5f : (qv < pv ? -0.5f : 0.f);
                    g[j] = f * qv * (sg - cq);
                }
            } else {
#pragma unroll
                for (int j = 0; j < VEC; ++j) g[j] = 0.f;
            }
            if (nv == VEC && galigned) {
                if constexpr (VEC == 8) {
                    uint4 o;
                    __nv_bfloat162 h0 = __floats2bfloat162_rn(g[0], g[1]);
                    __nv_bfloat162 h1 = __floats2bfloat162_rn(g[2], g[3]);
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(g[4], g[5]);
                    __nv_bfloat162 h3 = __floats2bfloat162_rn(g[6], g[7]);
                    o.x = *reinterpret_cast<uint32_t*>(&h0);
                    o.y = *reinterpret_cast<uint32_t*>(&h1);
                    o.z = *reinterpret_cast<uint32_t*>(&h2);
                    o.w = *reinterpret_cast<uint32_t*>(&h3);
                    __stcs(reinterpret_cast<uint4*>(grow + e0), o);
                } else {
                    __stcs(reinterpret_cast<float4*>(grow + e0), make_float4(g[0], g[1], g[2], g[3]));
                }
            } else {
                for (int j = 0; j < nv; ++j) {
                    if constexpr (VEC == 8) grow[e0 + j] = __float2bfloat16_rn(g[j]);
                    else reinterpret_cast<float*>(grow)[e0 + j] = g[j];
                }
            }
        }
    }

    // ---- per-token TV and the masked mean (last CTA) ----
    if (tid == 0) {
        a.out_tv[r] = (float)tv;
        if (on) atomicAdd(&p.work->sum_tv, tv);
        __threadfence();
        uint32_t prev = atomicAdd(&p.work->done, 1u);
        if (prev == (uint32_t)(a.N - 1)) {
            __threadfence();
            double s = atomicAdd(&p.work->sum_tv, 0.0);
            *a.out_mean = n_mask > 0 ? (float)(s / (double)n_mask) : 0.f;
        }
    }
}

__global__ void empty_mean_kernel(float* out_mean) { *out_mean = 0.f; }

// =====================================================================================
// cluster kernel
// =====================================================================================
namespace cl {

constexpr int kWarps = 16;                   // compute warps
constexpr int kThreads = (kWarps + 1) * 32;  // + one producer warp
constexpr float kLog2e = 1.4426950408889634f;

// Shared memory: a header of mbarriers and reduction slots, two input buffers of
// (teacher, student) bf16 row slices, and exp(student) of the current row in fp32.
//   mbarriers: full[2] (an input buffer has landed), empty[2] (every compute warp is done
//   with an input buffer), red[2] (every warp of the cluster has sent its partial of
//   reduction 0 / 1); then the per-warp partials, [ncta][kWarps] float4 (reduction 0:
//   max and sum of exp for both rows) and [ncta][kWarps] float2 (reduction 1).
__host__ __device__ inline size_t header_bytes(int ncta) {
    return ((size_t)64 + (size_t)ncta * kWarps * (16 + 8) + 127) / 128 * 128;
}
// Elements of a row slice: a multiple of 8 (16-byte bulk copies and 8-element units).
inline int64_t slice_elems(int64_t V, int cl) { return ((V + cl - 1) / cl + 7) / 8 * 8; }
// two (teacher, student) buffers, and with `keep` exp(student) of the current row in fp32
inline size_t smem_bytes(int64_t n, int ncta, bool keep) {
    return header_bytes(ncta) + (size_t)n * (2 * 2 * 2 + (keep ? 4 : 0));
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t num_clusters() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    __syncwarp();
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_rank(const void* local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    return remote;
}
// stores into another CTA's shared memory, counted in bytes on that CTA's mbarrier
__device__ __forceinline__ void st_async_v4(uint32_t dst, uint32_t bar, float a, float b, float c, float d) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     dst),
                 "f"(a), "f"(b), "f"(c), "f"(d), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t dst, uint32_t bar, float a, float b) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(dst),
                 "f"(a), "f"(b), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// bulk copy shared -> global (16-byte aligned addresses, size a multiple of 16), tracked
// by this thread's bulk groups
__device__ __forceinline__ void bulk_s2g(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every committed group has finished reading its shared-memory source
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// every committed group has completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// packed pairs of fp32 (Blackwell's two-wide fp32 pipe)
typedef unsigned long long f2;
__device__ __forceinline__ f2 pk(float lo, float hi) {
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float lo_of(f2 v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi_of(f2 v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
    f2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
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
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
    f2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// the two bf16 values of a 32-bit word, widened (exact)
__device__ __forceinline__ f2 widen(uint32_t w) { return pk(bf16_lo(w), bf16_hi(w)); }

template <bool KEEP>
__global__ void __launch_bounds__(kThreads, 1) cluster_kernel(Params p, int64_t n) {
    extern __shared__ __align__(128) unsigned char smem[];
    const TVArgs& a = p.a;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = cluster_rank(), ncta = cluster_size();
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + 2;
    uint64_t* red = full + 4;  // [2]
    float4* slots0 = reinterpret_cast<float4*>(smem + 64);                              // [ncta][kWarps]
    float2* slots1 = reinterpret_cast<float2*>(smem + 64 + (size_t)ncta * kWarps * 16);  // [ncta][kWarps]
    const size_t hdr = header_bytes((int)ncta);
    uint16_t* inbuf = reinterpret_cast<uint16_t*>(smem + hdr);  // [2][teacher, student][n]
    // (KEEP) unit u keeps its 8 exps at es[u*4 ..+4) and es[half + u*4 ..+4)
    float* es = reinterpret_cast<float*>(smem + hdr + (size_t)n * 8);
    const int half = (int)(n / 2);
    const int64_t N = a.N, V = a.V;
    const int64_t lo = (int64_t)rank * n;
    const int cnt = (int)max((int64_t)0, min(n, V - lo));  // elements of this CTA's slice
    const uint32_t bytes = (uint32_t)cnt * 2u;
    const int units = cnt / 8;
    const uint32_t red0_bytes = ncta * kWarps * 16u, red1_bytes = ncta * kWarps * 8u;
    const __nv_bfloat16* T = reinterpret_cast<const __nv_bfloat16*>(a.teacher);
    const __nv_bfloat16* S = reinterpret_cast<const __nv_bfloat16*>(a.student);
    __nv_bfloat16* G = reinterpret_cast<__nv_bfloat16*>(a.grad);
    const uint32_t n_mask = p.work->n_mask;
    uint32_t* status = p.status;
    const int64_t first = cluster_id(), step = num_clusters();
    bool failed = false;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
        if (!mbar_wait(bar, parity)) {
            failed = true;
            record_device_status(status, UNO_ERR_TIMEOUT);
        }
    };

    // Cluster-wide reductions of a row's per-warp partials (every lane of the warp passes the
    // same value): each warp stores its partial into slot [rank][warp] of every CTA of the
    // cluster (st.async, counted in bytes on that CTA's barrier); once all have landed, every
    // warp combines them. Rows overlap (see the compute loop), yet one slot array and one
    // barrier per reduction suffice, because of the order of the sends: a warp sends its
    // partial of reduction 1 for row i only after reading the slots of reduction 0 for row
    // i, and its partial of reduction 0 for row i + 1 only after reading the slots of
    // reduction 1 for row i; so no CTA can send a row's partial into slots that another CTA
    // is still reading, or count it on a barrier phase that is still open. Thread 0 arms a
    // barrier's next phase right after its own wait, before it sends anything further.
    // After a failed wait the later reduction waits are skipped (the call reports an error).
    auto wait_red = [&](uint64_t* bar, uint32_t parity) {
        if (!failed) wait(bar, parity);
    };
    // 0: (max t, sum exp(t - max t), max s, sum exp(s - max s)) -> row maxima and sums
    auto send0 = [&](float4 part) {
        if ((uint32_t)lane < ncta)
            st_async_v4(map_rank(&slots0[rank * kWarps + warp], lane), map_rank(&red[0], lane), part.x, part.y,
                        part.z, part.w);
    };
    auto recv0 = [&](uint32_t parity, bool arm_next) -> float4 {
        wait_red(&red[0], parity);
        float Mt = -INFINITY, Ms = -INFINITY;
        for (uint32_t j = lane; j < ncta * kWarps; j += 32) {
            const float4 w = slots0[j];
            Mt = fmaxf(Mt, w.x);
            Ms = fmaxf(Ms, w.z);
        }
        Mt = warp_max(Mt);
        Ms = warp_max(Ms);
        float Zt = 0.f, Zs = 0.f;
        for (uint32_t j = lane; j < ncta * kWarps; j += 32) {
            const float4 w = slots0[j];
            if (w.y > 0.f) Zt += w.y * ex2((w.x - Mt) * kLog2e);
            if (w.w > 0.f) Zs += w.w * ex2((w.z - Ms) * kLog2e);
        }
        if (tid == 0 && arm_next) mbar_arrive_expect_tx(&red[0], red0_bytes);
        return make_float4(Mt, warp_sum(Zt), Ms, warp_sum(Zs));
    };
    // 1: (A, P) sums
    auto send1 = [&](float2 part) {
        if ((uint32_t)lane < ncta)
            st_async_v2(map_rank(&slots1[rank * kWarps + warp], lane), map_rank(&red[1], lane), part.x, part.y);
    };
    auto recv1 = [&](uint32_t parity, bool arm_next) -> float2 {
        wait_red(&red[1], parity);
        float x = 0.f, y = 0.f;
        for (uint32_t j = lane; j < ncta * kWarps; j += 32) {
            const float2 w = slots1[j];
            x += w.x;
            y += w.y;
        }
        if (tid == 0 && arm_next) mbar_arrive_expect_tx(&red[1], red1_bytes);
        return make_float2(warp_sum(x), warp_sum(y));
    };

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&empty[0], kWarps);
        mbar_init(&empty[1], kWarps);
        mbar_init(&red[0], 1);
        mbar_init(&red[1], 1);
        fence_mbar_init();
        // armed one row ahead, so that no partial can arrive before its phase is armed
        if (first < N) {
            mbar_arrive_expect_tx(&red[0], red0_bytes);
            mbar_arrive_expect_tx(&red[1], red1_bytes);
        }
    }
    // every CTA's mbarriers are initialised and armed before any CTA sends to them
    cluster_sync();

    if (warp == kWarps) {
        // ---------------- producer: one row ahead, each buffer refilled once released ----
        // A released buffer holds the gradient of its row in place of the teacher slice:
        // stream that out first, then refill the buffer.
        if (lane == 0 && cnt > 0) {
            uint32_t k = 0;
            for (int64_t r = first; r < N; r += step, ++k) {
                const int b = k & 1;
                uint16_t* dst = inbuf + (size_t)b * 2 * n;
                if (k >= 2) {
                    wait(&empty[b], ((k >> 1) - 1) & 1);
                    if (G != nullptr) {
                        bulk_s2g(G + (r - 2 * step) * V + lo, dst, bytes);
                        bulk_commit();
                        bulk_wait_read();  // the slice has been read out before it is refilled
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&full[b], 2u * bytes);
                bulk_g2s(dst, T + r * V + lo, bytes, &full[b]);
                bulk_g2s(dst + n, S + r * V + lo, bytes, &full[b]);
            }
            // the last two rows' gradients
            for (uint32_t j = (k >= 2 ? k - 2 : 0); j < k; ++j) {
                const int b = j & 1;
                wait(&empty[b], (j >> 1) & 1);
                if (G != nullptr) {
                    bulk_s2g(G + (first + (int64_t)j * step) * V + lo, inbuf + (size_t)b * 2 * n, bytes);
                    bulk_commit();
                }
            }
            bulk_wait_all();  // every gradient store has completed
        }
        __syncwarp();
    } else {
        // ---------------- compute warps ----------------
        // Rows overlap: row i's reduction 1 is in flight while the warps take row i + 1's
        // maxima and exps, and row i + 1's reduction 0 while they write row i's gradient:
        //   [combine 0 (i)] [A, P (i); send 1 (i)] [maxima, exps (i + 1)]
        //   [combine 1 (i); send 0 (i + 1)] [gradient (i)] ...
        // Row i + 1's exps overwrite the kept exp(student) of row i, so the gradient pass
        // recomputes exp(student) (4 exponentials per element pair).
        double tv_sum = 0.0;  // this cluster's masked TV (rank 0, thread 0)
        uint32_t rows_done = 0;
        const f2 L2E = pk(kLog2e, kLog2e);
        // maxima and exps of the row in buffer b: this warp's (max t, sum, max s, sum), with
        // exp(s - warp max) kept; lt, ls are the warp maxima x log2(e) (0 for a warp with no
        // elements: its sums are 0 and it never reads its factors)
        float mt = -INFINITY, ms = -INFINITY, lt = 0.f, ls = 0.f;
        auto maxima_exps = [&](int b) -> float4 {
            const uint16_t* tin = inbuf + (size_t)b * 2 * n;
            const uint16_t* sin = tin + n;
            __nv_bfloat162 mt2 = __floats2bfloat162_rn(-INFINITY, -INFINITY), ms2 = mt2;
            for (int u = tid; u < units; u += kWarps * 32) {
                const uint4 wt = lds128(tin + u * 8), ws = lds128(sin + u * 8);
                const uint32_t at4[4] = {wt.x, wt.y, wt.z, wt.w}, as4[4] = {ws.x, ws.y, ws.z, ws.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    mt2 = __hmax2(mt2, *reinterpret_cast<const __nv_bfloat162*>(&at4[j]));
                    ms2 = __hmax2(ms2, *reinterpret_cast<const __nv_bfloat162*>(&as4[j]));
                }
            }
            mt = warp_max(fmaxf(__low2float(mt2), __high2float(mt2)));
            ms = warp_max(fmaxf(__low2float(ms2), __high2float(ms2)));
            lt = (mt == -INFINITY ? 0.f : mt) * kLog2e;
            ls = (ms == -INFINITY ? 0.f : ms) * kLog2e;
            const f2 NLT = pk(-lt, -lt), NLS = pk(-ls, -ls);
            f2 zt2 = pk(0.f, 0.f), zs2 = zt2;
            for (int u = tid; u < units; u += kWarps * 32) {
                const uint4 wt = lds128(tin + u * 8), ws = lds128(sin + u * 8);
                const uint32_t at4[4] = {wt.x, wt.y, wt.z, wt.w}, as4[4] = {ws.x, ws.y, ws.z, ws.w};
                float e[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const f2 xt = fma2(widen(at4[j]), L2E, NLT), xs = fma2(widen(as4[j]), L2E, NLS);
                    zt2 = add2(zt2, pk(ex2(lo_of(xt)), ex2(hi_of(xt))));
                    e[2 * j] = ex2(lo_of(xs));
                    e[2 * j + 1] = ex2(hi_of(xs));
                    zs2 = add2(zs2, pk(e[2 * j], e[2 * j + 1]));
                }
                if constexpr (KEEP) {
                    *reinterpret_cast<float4*>(es + u * 4) = make_float4(e[0], e[1], e[2], e[3]);
                    *reinterpret_cast<float4*>(es + half + u * 4) = make_float4(e[4], e[5], e[6], e[7]);
                }
            }
            return make_float4(mt, warp_sum(lo_of(zt2) + hi_of(zt2)), ms, warp_sum(lo_of(zs2) + hi_of(zs2)));
        };

        if (first < N) {
            if (cnt > 0) wait(&full[0], 0);
            send0(maxima_exps(0));
        }
        uint32_t it = 0;
        for (int64_t r = first; r < N; r += step, ++it) {
            const int b = it & 1;
            const uint32_t par = it & 1;
            const bool more = r + step < N;
            const uint16_t* tin = inbuf + (size_t)b * 2 * n;
            const uint16_t* sin = tin + n;
            // this row's warp maxima (the next row's maxima_exps replaces them)
            const float rmt = mt, rms = ms, rlt = lt, rls = ls;

            const float4 st = recv0(par, more);
            const float Mt = st.x, Zt = st.y, Ms = st.z, Zs = st.w;
            // p = exp(t - wmt) * at, q = exp(s - wms) * as: this warp's maxima folded into at,
            // as (the same arithmetic for both rows: identical rows give p == q).
            // q > p is decided in the log domain, exact up to the rounding of one threshold:
            //   q > p  <=>  s - t > K = (Ms + ln Zs) - (Mt + ln Zt)
            // (Ms - Mt is exact; Zs / Zt is near 1 in practice, so its log is accurate to ~1e-7)
            const float at = rmt == -INFINITY ? 0.f : ex2(rlt - Mt * kLog2e) / Zt;
            const float as = rms == -INFINITY ? 0.f : ex2(rls - Ms * kLog2e) / Zs;
            const float K = (Ms - Mt) + logf(Zs / Zt);
            const f2 NLT = pk(-rlt, -rlt), NLS = pk(-rls, -rls);

            // ---- A = sum of q over q > p, P = sum of p over q > p ----
            // TV = A - P and sum_v q_v sign(q_v - p_v) / 2 = A - 1/2 (both rows sum to 1)
            float Araw = 0.f, Praw = 0.f;
            for (int u = tid; u < units; u += kWarps * 32) {
                const uint4 wt = lds128(tin + u * 8), ws = lds128(sin + u * 8);
                const uint32_t at4[4] = {wt.x, wt.y, wt.z, wt.w}, as4[4] = {ws.x, ws.y, ws.z, ws.w};
                float qe[8];
                if constexpr (KEEP) {
                    const float4 k0 = *reinterpret_cast<const float4*>(es + u * 4);
                    const float4 k1 = *reinterpret_cast<const float4*>(es + half + u * 4);
                    qe[0] = k0.x, qe[1] = k0.y, qe[2] = k0.z, qe[3] = k0.w;
                    qe[4] = k1.x, qe[5] = k1.y, qe[6] = k1.z, qe[7] = k1.w;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const f2 t2 = widen(at4[j]), s2 = widen(as4[j]);
                    const f2 dl = sub2(s2, t2);
                    const f2 xt = fma2(t2, L2E, NLT), xs = fma2(s2, L2E, NLS);
                    if (lo_of(dl) > K) {
                        Araw += KEEP ? qe[2 * j] : ex2(lo_of(xs));
                        Praw += ex2(lo_of(xt));
                    }
                    if (hi_of(dl) > K) {
                        Araw += KEEP ? qe[2 * j + 1] : ex2(hi_of(xs));
                        Praw += ex2(hi_of(xt));
                    }
                }
            }
            send1(make_float2(warp_sum(Araw * as), warp_sum(Praw * at)));

            // ---- the next row's maxima and exps, while reduction 1 is in flight ----
            float4 next_part = make_float4(0.f, 0.f, 0.f, 0.f);
            if (more) {
                if (cnt > 0) wait(&full[b ^ 1], ((it + 1) >> 1) & 1);
                next_part = maxima_exps(b ^ 1);
            }
            const float2 ap = recv1(par, more);
            const float Af = ap.x, Pf = ap.y;
            if (more) send0(next_part);
            const bool on = a.mask == nullptr || a.mask[r] != 0;

            // ---- gradient: f q (1 - A) where q > p, -f q A elsewhere ----
            // written as bf16 in place of the teacher slice (each unit by the thread that read
            // it); the producer warp streams the slice out once every warp is done
            if (G != nullptr) {
                const bool grad_on = on && n_mask > 0;
                const float f = grad_on ? a.grad_scale / (float)n_mask : 0.f;
                const float kp = f * (1.f - Af) * as, kn = -f * Af * as;
                uint16_t* gout = const_cast<uint16_t*>(tin);
                for (int u = tid; u < units; u += kWarps * 32) {
                    uint4 o = make_uint4(0u, 0u, 0u, 0u);
                    if (grad_on) {
                        const uint4 wt = lds128(tin + u * 8), ws = lds128(sin + u * 8);
                        const uint32_t at4[4] = {wt.x, wt.y, wt.z, wt.w}, as4[4] = {ws.x, ws.y, ws.z, ws.w};
                        uint32_t ow[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const f2 s2 = widen(as4[j]);
                            const f2 dl = sub2(s2, widen(at4[j]));
                            const f2 xs = fma2(s2, L2E, NLS);
                            const f2 fac = pk(lo_of(dl) > K ? kp : kn, hi_of(dl) > K ? kp : kn);
                            const f2 g = mul2(pk(ex2(lo_of(xs)), ex2(hi_of(xs))), fac);
                            __nv_bfloat162 hv = __floats2bfloat162_rn(lo_of(g), hi_of(g));
                            ow[j] = *reinterpret_cast<uint32_t*>(&hv);
                        }
                        o = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    }
                    *reinterpret_cast<uint4*>(gout + u * 8) = o;
                }
                fence_proxy_async_smem();  // the bulk store reads these through the async proxy
            }
            // this warp is done with the input buffer
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[b]);
            if (rank == 0 && tid == 0) {
                const double tv = (double)Af - (double)Pf;
                a.out_tv[r] = (float)tv;
                if (on) tv_sum += tv;
                ++rows_done;
            }
        }
        // this cluster's share of the masked mean; the cluster that completes the last row
        // writes it
        if (rank == 0 && tid == 0 && rows_done > 0) {
            atomicAdd(&p.work->sum_tv, tv_sum);
            __threadfence();
            const uint32_t prev = atomicAdd(&p.work->done, rows_done);
            if (prev + rows_done == (uint32_t)N) {
                __threadfence();
                const double s = atomicAdd(&p.work->sum_tv, 0.0);
                *a.out_mean = n_mask > 0 ? (float)(s / (double)n_mask) : 0.f;
            }
        }
    }
    // no CTA leaves while a store into its shared memory may be in flight
    cluster_sync();
}

// ---------------------------------------------------------------------------------------
// team_kernel: the same computation with two teams of eight warps per CTA on alternate rows.
// A team waits for its cluster reductions and its copies while the other team computes, so
// those latencies overlap instead of adding up. Each team holds one (teacher, student) slice
// pair (the gradient replaces the teacher slice and is streamed out by the team's leader,
// who then brings in the team's next row). KEEP: exp(student) of the team's row is kept in
// fp32 beside its slices (3 exponentials per element pair, 12 bytes of shared memory per
// element and team, so clusters of 16 at a 152k vocabulary); otherwise it is recomputed
// where it is needed (5 exponentials per element pair, 4 bytes per element and team).
// Reductions: each warp stores its partial into slot [rank][warp] of every CTA of the
// cluster and arrives on that CTA's barrier.
// ---------------------------------------------------------------------------------------
constexpr int kTeams = 2;
constexpr int kTeamWarps = 8;
constexpr int kTeamThreads = kTeamWarps * 32;
constexpr int kTeamKernelThreads = kTeams * kTeamThreads;
constexpr int kMaxCL = 16;

// a team's (teacher, student) slices, and with `keep` its exp(student) in fp32
__host__ __device__ inline size_t team_slice_bytes(int64_t n, bool keep) {
    return ((size_t)n * (keep ? 8 : 4) + 127) / 128 * 128;
}
__host__ __device__ inline size_t team_bytes(int64_t n, bool keep) {
    return team_slice_bytes(n, keep) + (size_t)kMaxCL * kTeamWarps * (16 + 8);
}

__device__ __forceinline__ void team_sync(int team) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "n"(kTeamThreads) : "memory");
}
__device__ __forceinline__ void st_remote_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
__device__ __forceinline__ void st_remote_v2(uint32_t addr, float a, float b) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void arrive_remote(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
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

template <bool KEEP>
__global__ void __launch_bounds__(kTeamKernelThreads, 1) team_kernel(Params p, int64_t n) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bars[kTeams][3];  // slices landed, reduction 0, reduction 1
    __shared__ double s_tv[kTeams];
    __shared__ uint32_t s_rows[kTeams];
    __shared__ int s_abort[kTeams];
    const TVArgs& a = p.a;
    const int team = threadIdx.x / kTeamThreads, tt = threadIdx.x % kTeamThreads;
    const int tw = tt >> 5, lane = tt & 31;
    const uint32_t rank = cluster_rank(), ncta = cluster_size();
    unsigned char* base = smem + (size_t)team * team_bytes(n, KEEP);
    uint16_t* tin = reinterpret_cast<uint16_t*>(base);  // teacher slice, then the gradient
    uint16_t* sin = tin + n;                            // student slice
    // (KEEP) unit u's 8 values of exp(s - warp max) at es[u*4 ..+4) and es[half + u*4 ..+4)
    float* es = reinterpret_cast<float*>(base + (size_t)n * 4);
    const int half = (int)(n / 2);
    float4* s0 = reinterpret_cast<float4*>(base + team_slice_bytes(n, KEEP));  // [kMaxCL][kTeamWarps]
    float2* s1 = reinterpret_cast<float2*>(s0 + kMaxCL * kTeamWarps);     // [kMaxCL][kTeamWarps]
    uint64_t* full = &bars[team][0];
    uint64_t* red0 = &bars[team][1];
    uint64_t* red1 = &bars[team][2];
    const int64_t N = a.N, V = a.V;
    const int64_t lo = (int64_t)rank * n;
    const int cnt = (int)max((int64_t)0, min(n, V - lo));
    const uint32_t bytes = (uint32_t)cnt * 2u;
    const int units = cnt / 8;
    const __nv_bfloat16* T = reinterpret_cast<const __nv_bfloat16*>(a.teacher);
    const __nv_bfloat16* S = reinterpret_cast<const __nv_bfloat16*>(a.student);
    __nv_bfloat16* G = reinterpret_cast<__nv_bfloat16*>(a.grad);
    const uint32_t n_mask = p.work->n_mask;
    const int64_t NC = num_clusters();
    const int64_t step = kTeams * NC;
    const int64_t r0 = (int64_t)cluster_id() + team * NC;

    if (tt == 0) {
        mbar_init(full, 1);
        mbar_init(red0, ncta * kTeamWarps);
        mbar_init(red1, ncta * kTeamWarps);
        s_tv[team] = 0.0;
        s_rows[team] = 0u;
        s_abort[team] = 0;
        fence_mbar_init();
    }
    __syncthreads();
    cluster_sync();  // every CTA's barriers exist before any remote arrive

    auto issue = [&](int64_t r) {  // the leader brings in row r's slices
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(full, 2u * bytes);
        bulk_g2s(tin, T + r * V + lo, bytes, full);
        bulk_g2s(sin, S + r * V + lo, bytes, full);
    };
    if (tt == 0 && cnt > 0 && r0 < N) issue(r0);

    uint32_t k = 0;
    for (int64_t r = r0; r < N; r += step, ++k) {
        const uint32_t par = k & 1;
        if (cnt > 0 && tw == 0) {
            const bool ok = mbar_wait(full, par);
            if (!ok && lane == 0) s_abort[team] = 1;
        }
        team_sync(team);
        if (s_abort[team]) break;

        // ---- this warp's maxima, then its sums of exp(x - warp max) ----
        __nv_bfloat162 mt2 = __floats2bfloat162_rn(-INFINITY, -INFINITY), ms2 = mt2;
        for (int u = tt; u < units; u += kTeamThreads) {
            const uint4 wt = lds128(tin + u * 8), ws = lds128(sin + u * 8);
            const uint32_t at4[4] = {wt.x, wt.y, wt.z, wt.w}, as4[4] = {ws.x, ws.y, ws.z, ws.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                mt2 = __hmax2(mt2, *reinterpret_cast<const __nv_bfloat162*>(&at4[j]));
                ms2 = __hmax2(ms2, *reinterpret_cast<const __nv_bfloat162*>(&as4[j]));
            }
        }
        const float mt = warp_max(fmaxf(__low2float(mt2), __high2float(mt2)));
        const float ms = warp_max(fmaxf(__low2float(ms2), __high2float(ms2)));
        const float lt = (mt == -INFINITY ? 0.f : mt) * kLog2e, ls = (ms == -INFINITY ? 0.f : ms) * kLog2e;
        const f2 L2E = pk(kLog2e, kLog2e), NLT = pk(-lt, -lt), NLS = pk(-ls, -ls);
        f2 zt2 = pk(0.f, 0.f), zs2 = zt2;
        for (int u = tt; u < units; u += kTeamThreads) {
            const uint4 wt = lds128(tin + u * 8), ws = lds128(sin + u * 8);
            const uint32_t at4[4] = {wt.x, wt.y, wt.z, wt.w}, as4[4] = {ws.x, ws.y, ws.z, ws.w};
            float e[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const f2 xt = fma2(widen(at4[j]), L2E, NLT), xs = fma2(widen(as4[j]), L2E, NLS);
                zt2 = add2(zt2, pk(ex2(lo_of(xt)), ex2(hi_of(xt))));
                e[2 * j] = ex2(lo_of(xs));
                e[2 * j + 1] = ex2(hi_of(xs));
                zs2 = add2(zs2, pk(e[2 * j], e[2 * j + 1]));
            }
            if constexpr (KEEP) {
                *reinterpret_cast<float4*>(es + u * 4) = make_float4(e[0], e[1], e[2], e[3]);
                *reinterpret_cast<float4*>(es + half + u * 4) = make_float4(e[4], e[5], e[6], e[7]);
            }
        }
        const float zt = warp_sum(lo_of(zt2) + hi_of(zt2)), zs = warp_sum(lo_of(zs2) + hi_of(zs2));
        // ---- reduction 0: row maxima and sums ----
        if ((uint32_t)lane < ncta) {
            st_remote_v4(map_rank(&s0[rank * kTeamWarps + tw], lane), mt, zt, ms, zs);
            arrive_remote(map_rank(red0, lane));
        }
        if (!wait_cluster(red0, par) && lane == 0) s_abort[team] = 1;
        float Mt = -INFINITY, Ms = -INFINITY;
        for (uint32_t j = lane; j < ncta * kTeamWarps; j += 32) {
            const float4 w = s0[j];
            Mt = fmaxf(Mt, w.x);
            Ms = fmaxf(Ms, w.z);
        }
        Mt = warp_max(Mt);
        Ms = warp_max(Ms);
        float Zt = 0.f, Zs = 0.f;
        for (uint32_t j = lane; j < ncta * kTeamWarps; j += 32) {
            const float4 w = s0[j];
            if (w.y > 0.f) Zt += w.y * ex2((w.x - Mt) * kLog2e);
            if (w.w > 0.f) Zs += w.w * ex2((w.z - Ms) * kLog2e);
        }
        Zt = warp_sum(Zt);
        Zs = warp_sum(Zs);
        // p = exp(t - wmt) at, q = exp(s - wms) as; q > p  <=>  s - t > K (see cluster_kernel)
        const float at = mt == -INFINITY ? 0.f : ex2(lt - Mt * kLog2e) / Zt;
        const float as = ms == -INFINITY ? 0.f : ex2(ls - Ms * kLog2e) / Zs;
        const float K = (Ms - Mt) + logf(Zs / Zt);

        // ---- A = sum of q over q > p, P = sum of p over q > p ----
        float Araw = 0.f, Praw = 0.f;
        for (int u = tt; u < units; u += kTeamThreads) {
            const uint4 wt = lds128(tin + u * 8), ws = lds128(sin + u * 8);
            const uint32_t at4[4] = {wt.x, wt.y, wt.z, wt.w}, as4[4] = {ws.x, ws.y, ws.z, ws.w};
            float qe[8];
            if constexpr (KEEP) {
                const float4 k0 = *reinterpret_cast<const float4*>(es + u * 4);
                const float4 k1 = *reinterpret_cast<const float4*>(es + half + u * 4);
                qe[0] = k0.x, qe[1] = k0.y, qe[2] = k0.z, qe[3] = k0.w;
                qe[4] = k1.x, qe[5] = k1.y, qe[6] = k1.z, qe[7] = k1.w;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const f2 t2 = widen(at4[j]), s2 = widen(as4[j]);
                const f2 dl = sub2(s2, t2);
                const f2 xt = fma2(t2, L2E, NLT), xs = fma2(s2, L2E, NLS);
                if (lo_of(dl) > K) {
                    Araw += KEEP ? qe[2 * j] : ex2(lo_of(xs));
                    Praw += ex2(lo_of(xt));
                }
                if (hi_of(dl) > K) {
                    Araw += KEEP ? qe[2 * j + 1] : ex2(hi_of(xs));
                    Praw += ex2(hi_of(xt));
                }
            }
        }
        const float Aw = warp_sum(Araw * as), Pw = warp_sum(Praw * at);
        if ((uint32_t)lane < ncta) {
            st_remote_v2(map_rank(&s1[rank * kTeamWarps + tw], lane), Aw, Pw);
            arrive_remote(map_rank(red1, lane));
        }
        if (!wait_cluster(red1, par) && lane == 0) s_abort[team] = 1;
        float Af = 0.f, Pf = 0.f;
        for (uint32_t j = lane; j < ncta * kTeamWarps; j += 32) {
            const float2 w = s1[j];
            Af += w.x;
            Pf += w.y;
        }
        Af = warp_sum(Af);
        Pf = warp_sum(Pf);
        const bool on = a.mask == nullptr || a.mask[r] != 0;

        // ---- gradient f q (1 - A) where q > p, -f q A elsewhere, over the teacher slice ----
        if (G != nullptr) {
            const bool grad_on = on && n_mask > 0;
            const float f = grad_on ? a.grad_scale / (float)n_mask : 0.f;
            const float kp = f * (1.f - Af) * as, kn = -f * Af * as;
            for (int u = tt; u < units; u += kTeamThreads) {
                uint4 o = make_uint4(0u, 0u, 0u, 0u);
                if (grad_on) {
                    const uint4 wt = lds128(tin + u * 8), ws = lds128(sin + u * 8);
                    const uint32_t at4[4] = {wt.x, wt.y, wt.z, wt.w}, as4[4] = {ws.x, ws.y, ws.z, ws.w};
                    float qe[8];
                    if constexpr (KEEP) {
                        const float4 k0 = *reinterpret_cast<const float4*>(es + u * 4);
                        const float4 k1 = *reinterpret_cast<const float4*>(es + half + u * 4);
                        qe[0] = k0.x, qe[1] = k0.y, qe[2] = k0.z, qe[3] = k0.w;
                        qe[4] = k1.x, qe[5] = k1.y, qe[6] = k1.z, qe[7] = k1.w;
                    }
                    uint32_t ow[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const f2 s2 = widen(as4[j]);
                        const f2 dl = sub2(s2, widen(at4[j]));
                        const f2 xs = fma2(s2, L2E, NLS);
                        const f2 fac = pk(lo_of(dl) > K ? kp : kn, hi_of(dl) > K ? kp : kn);
                        const f2 qv = KEEP ? pk(qe[2 * j], qe[2 * j + 1]) : pk(ex2(lo_of(xs)), ex2(hi_of(xs)));
                        const f2 g = mul2(qv, fac);
                        __nv_bfloat162 hv = __floats2bfloat162_rn(lo_of(g), hi_of(g));
                        ow[j] = *reinterpret_cast<uint32_t*>(&hv);
                    }
                    o = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                }
                *reinterpret_cast<uint4*>(tin + u * 8) = o;
            }
            fence_proxy_async_smem();  // the bulk store reads these through the async proxy
        }
        team_sync(team);  // the slices are no longer read; the gradient is complete
        if (rank == 0 && tt == 0) {
            const double tv = (double)Af - (double)Pf;
            a.out_tv[r] = (float)tv;
            if (on) s_tv[team] += tv;
            s_rows[team] += 1u;
        }
        if (tt == 0 && cnt > 0) {
            if (G != nullptr) {
                bulk_s2g(G + r * V + lo, tin, bytes);
                bulk_commit();
                bulk_wait_read();  // the slice has been read out before it is refilled
            }
            if (r + step < N) issue(r + step);
        }
    }
    if (tt == 0) {
        if (s_abort[team]) {
            // a copy issued for a row this team will not process: let it land
            mbar_wait(full, k & 1, 1u << 16);
            record_device_status(p.status, UNO_ERR_TIMEOUT);
        }
        bulk_wait_all();  // every gradient store has completed
        // this team's share of the masked mean; whoever completes the last row writes it
        if (rank == 0 && s_rows[team] > 0) {
            atomicAdd(&p.work->sum_tv, s_tv[team]);
            __threadfence();
            const uint32_t prev = atomicAdd(&p.work->done, s_rows[team]);
            if (prev + s_rows[team] == (uint32_t)N) {
                __threadfence();
                const double sum = atomicAdd(&p.work->sum_tv, 0.0);
                *a.out_mean = n_mask > 0 ? (float)(sum / (double)n_mask) : 0.f;
            }
        }
    }
    __syncthreads();
    cluster_sync();  // no CTA leaves while a store into its shared memory may be in flight
}

}  // namespace cl

}  // namespace tvk

size_t tv_loss_workspace_bytes(int64_t N, int64_t V, uno_dtype dtype) {
    (void)N;
    (void)V;
    (void)dtype;
    return 256;
}

namespace {

struct DeviceInfo {
    bool ready = false;
    int smem_optin = 0;
    std::map<std::pair<int, size_t>, int> max_clusters;  // (cluster size, smem) -> co-resident clusters
};
std::mutex g_mu;
DeviceInfo g_dev[64];

// Co-resident clusters of the cluster kernel at cluster size c (cached per device).
int cluster_capacity(DeviceInfo& di, int c, bool keep, int64_t n) {
    cudaLaunchConfig_t q = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    q.blockDim = dim3(tvk::cl::kThreads);
    q.dynamicSmemBytes = tvk::cl::smem_bytes(n, c, keep);
    q.attrs = attr;
    q.numAttrs = 1;
    q.gridDim = dim3((unsigned)c);
    auto key = std::make_pair(c + (keep ? 32 : 0), q.dynamicSmemBytes);
    auto found = di.max_clusters.find(key);
    if (found != di.max_clusters.end()) return found->second;
    int maxc = 0;
    if (cudaOccupancyMaxActiveClusters(&maxc, keep ? tvk::cl::cluster_kernel<true> : tvk::cl::cluster_kernel<false>,
                                       &q) != cudaSuccess) {
        cudaGetLastError();
        maxc = 0;
    }
    di.max_clusters[key] = maxc;
    return maxc;
}

// Cluster form for N rows of V bf16 elements: a cluster size c (1 to 8, or 16) whose slices
// fit in one CTA's shared memory, with exp(student) kept (12 bytes per element) or
// recomputed (8 bytes per element, 5 exponentials per element pair instead of 4, so a
// smaller c fits). Among those that fit, the one with the least estimated time: the rows
// each co-resident cluster takes in turn x the slice each CTA works through, x 1.02 when
// exp(student) is kept (its shared-memory traffic measured costlier than the extra
// exponentials: at V = 151936, clusters of 8 took 0.438 ms per 1024 rows keeping it and
// 0.430 ms recomputing it; clusters of 6, which only the recomputing form fits, 0.361 ms:
// no more than 15 clusters of 8 are co-resident, 120 of the 148 SMs). UNO_TV_CLUSTER=c
// forces c where it fits; UNO_TV_KEEP=0 forces the recomputing form and UNO_TV_KEEP=1 the
// keeping one. Returns c = 0 when none fits.
std::pair<int, bool> choose_cluster(DeviceInfo& di, int64_t N, int64_t V) {
    int forced = 0;
    if (const char* e = getenv("UNO_TV_CLUSTER")) forced = atoi(e);
    const char* ke = getenv("UNO_TV_KEEP");
    const bool allow_keep = !(ke && ke[0] == '0'), allow_recompute = !(ke && ke[0] == '1');
    std::pair<int, bool> best{0, false};
    double best_cost = 0.0;
    static const int kSizes[] = {1, 2, 3, 4, 5, 6, 7, 8, 16};
    // pass 0: the forced size only (if any); pass 1: every size
    for (int pass = forced != 0 ? 0 : 1; pass < 2 && best.first == 0; ++pass) {
        for (int c : kSizes) {
            if (pass == 0 && c != forced) continue;
            const int64_t n = tvk::cl::slice_elems(V, c);
            for (int k = 0; k < 2; ++k) {
                const bool keep = k == 0;
                if ((keep && !allow_keep) || (!keep && !allow_recompute)) continue;
                if (tvk::cl::smem_bytes(n, c, keep) > (size_t)di.smem_optin) continue;
                const int maxc = cluster_capacity(di, c, keep, n);
                if (maxc <= 0) continue;
                const double cost = (double)((N + maxc - 1) / maxc) * (double)n * (keep ? 1.02 : 1.0);
                if (best.first == 0 || cost < best_cost) {
                    best = {c, keep};
                    best_cost = cost;
                }
            }
        }
    }
    return best;
}

// The two-team kernel: the smallest cluster size whose two teams' slices fit, keeping
// exp(student) where some cluster size lets it fit (UNO_TV_CLUSTER forces a size, and
// UNO_TV_KEEP=0 recomputes exp(student) instead).
bool launch_teams(const tvk::Params& p, cudaStream_t stream, uno_status& st, DeviceInfo& di) {
    const TVArgs& a = p.a;
    const size_t room = (size_t)di.smem_optin - 256;  // the kernel's static shared memory
    auto fits = [&](int c, bool keep) {
        return 2 * tvk::cl::team_bytes(tvk::cl::slice_elems(a.V, c), keep) <= room;
    };
    int forced = 0;
    if (const char* e = getenv("UNO_TV_CLUSTER")) {
        const int f = atoi(e);
        if (f == 1 || f == 2 || f == 4 || f == 8 || f == 16) forced = f;
    }
    const char* ke = getenv("UNO_TV_KEEP");
    const bool allow_keep = !(ke && ke[0] == '0');
    int c = 0;
    bool keep = false;
    for (int pass = allow_keep ? 0 : 1; pass < 2 && c == 0; ++pass) {
        keep = pass == 0;
        if (forced != 0) {
            if (fits(forced, keep)) c = forced;
        } else {
            for (int t = 1; t <= 16 && c == 0; t *= 2)
                if (fits(t, keep)) c = t;
        }
    }
    if (c == 0) return false;
    const int64_t n = tvk::cl::slice_elems(a.V, c);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(tvk::cl::kTeamKernelThreads);
    cfg.dynamicSmemBytes = 2 * tvk::cl::team_bytes(n, keep);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    auto kernel = keep ? tvk::cl::team_kernel<true> : tvk::cl::team_kernel<false>;
    auto key = std::make_pair(-(c + (keep ? 32 : 0)), cfg.dynamicSmemBytes);
    auto found = di.max_clusters.find(key);
    int maxc = 0;
    if (found != di.max_clusters.end()) {
        maxc = found->second;
    } else {
        cudaLaunchConfig_t q = cfg;
        q.gridDim = dim3((unsigned)c);
        if (cudaOccupancyMaxActiveClusters(&maxc, kernel, &q) != cudaSuccess) {
            cudaGetLastError();
            maxc = 0;
        }
        di.max_clusters[key] = maxc;
    }
    if (maxc <= 0) return false;
    const int64_t clusters = std::min<int64_t>((a.N + 1) / 2, (int64_t)maxc);
    cfg.gridDim = dim3((unsigned)(clusters * c));
    st = check_cuda(cudaLaunchKernelEx(&cfg, kernel, p, n), "launch(tv teams)");
    return true;
}

// Launch the cluster kernel; returns false (nothing launched) when it cannot run here.
bool launch_cluster(const tvk::Params& p, cudaStream_t stream, uno_status& st) {
    const TVArgs& a = p.a;
    if (a.dtype != UNO_BF16 || a.V % 8 != 0) return false;
    const uintptr_t al = reinterpret_cast<uintptr_t>(a.teacher) | reinterpret_cast<uintptr_t>(a.student) |
                         reinterpret_cast<uintptr_t>(a.grad);
    if (al & 15u) return false;
    bool teams = false;
    if (const char* e = getenv("UNO_TV_KERNEL")) {
        if (strcmp(e, "rows") == 0) return false;
        teams = strcmp(e, "teams") == 0;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& di = g_dev[dev];
    if (!di.ready) {
        if (cudaDeviceGetAttribute(&di.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return false;
        if (cudaFuncSetAttribute(tvk::cl::cluster_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 di.smem_optin) != cudaSuccess ||
            cudaFuncSetAttribute(tvk::cl::cluster_kernel<true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess ||
            cudaFuncSetAttribute(tvk::cl::cluster_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 di.smem_optin) != cudaSuccess ||
            cudaFuncSetAttribute(tvk::cl::cluster_kernel<false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess ||
            cudaFuncSetAttribute(tvk::cl::team_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 di.smem_optin - 256) != cudaSuccess ||
            cudaFuncSetAttribute(tvk::cl::team_kernel<false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess ||
            cudaFuncSetAttribute(tvk::cl::team_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 di.smem_optin - 256) != cudaSuccess ||
            cudaFuncSetAttribute(tvk::cl::team_kernel<true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        di.ready = true;
    }
    if (teams) return launch_teams(p, stream, st, di);
    const std::pair<int, bool> choice = choose_cluster(di, a.N, a.V);
    const int c = choice.first;
    const bool keep = choice.second;
    if (c == 0) return false;
    const int64_t n = tvk::cl::slice_elems(a.V, c);
    const int maxc = cluster_capacity(di, c, keep, n);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(tvk::cl::kThreads);
    cfg.dynamicSmemBytes = tvk::cl::smem_bytes(n, c, keep);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int64_t clusters = std::min<int64_t>(a.N, (int64_t)maxc);
    cfg.gridDim = dim3((unsigned)(clusters * c));
    st = check_cuda(cudaLaunchKernelEx(&cfg, keep ? tvk::cl::cluster_kernel<true> : tvk::cl::cluster_kernel<false>,
                                       p, n),
                    "launch(tv cluster)");
    return true;
}

}  // namespace

uno_status tv_loss_launch(const TVArgs& a, void* workspace, cudaStream_t stream) {
    if (a.N == 0) {
        tvk::empty_mean_kernel<<<1, 1, 0, stream>>>(a.out_mean);
        return check_cuda(cudaGetLastError(), "launch(tv mean)");
    }
    tvk::Params p{a, static_cast<tvk::Work*>(workspace), device_status_ptr()};
    tvk::count_mask_kernel<<<1, 1024, 0, stream>>>(a.mask, a.N, p.work);
    uno_status s = check_cuda(cudaGetLastError(), "launch(tv mask count)");
    if (s != UNO_OK) return s;
    if (launch_cluster(p, stream, s)) return s;
    if (a.dtype == UNO_BF16) tvk::rows_kernel<__nv_bfloat16><<<(unsigned)a.N, tvk::kThreads, 0, stream>>>(p);
    else tvk::rows_kernel<float><<<(unsigned)a.N, tvk::kThreads, 0, stream>>>(p);
    return check_cuda(cudaGetLastError(), "launch(tv rows)");
}

}  // namespace uno
