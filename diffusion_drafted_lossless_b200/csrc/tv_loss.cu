// tv_loss.cu — TV self-distillation loss and its gradient w.r.t. the student logits.
//
// LoopUno project page, "Training is self-distillation": the loss is the total-variation
// distance between the frozen teacher's next-token distribution (clean copy) and the
// student's (model + LoRA on the block-noised copy) on the response tokens.
//   p = softmax(teacher), q = softmax(student); TV = 1/2 sum |p - q|
//   mean = sum_{masked} TV / N_mask
//   dmean/dstudent_v = q_v (s_v - sum_w q_w s_w) / N_mask,  s = 1/2 sign(q - p)
//
// One CTA per token row. Pass 1 streams both rows from HBM once and keeps per-thread
// online (max, sum); pass 2 re-reads them (L2) for sum |p - q| and c = sum q s; pass 3
// re-reads them and writes the bf16 gradient. A tiny pre-kernel counts the mask; the last
// CTA to finish (atomic counter, no waiting) writes the mean.
#include <cuda_bf16.h>

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

}  // namespace tvk

size_t tv_loss_workspace_bytes(int64_t N, int64_t V, uno_dtype dtype) {
    (void)N;
    (void)V;
    (void)dtype;
    return 256;
}

uno_status tv_loss_launch(const TVArgs& a, void* workspace, cudaStream_t stream) {
    if (a.N == 0) {
        tvk::empty_mean_kernel<<<1, 1, 0, stream>>>(a.out_mean);
        return check_cuda(cudaGetLastError(), "launch(tv mean)");
    }
    tvk::Params p{a, static_cast<tvk::Work*>(workspace)};
    tvk::count_mask_kernel<<<1, 1024, 0, stream>>>(a.mask, a.N, p.work);
    uno_status s = check_cuda(cudaGetLastError(), "launch(tv mask count)");
    if (s != UNO_OK) return s;
    if (a.dtype == UNO_BF16) tvk::rows_kernel<__nv_bfloat16><<<(unsigned)a.N, tvk::kThreads, 0, stream>>>(p);
    else tvk::rows_kernel<float><<<(unsigned)a.N, tvk::kThreads, 0, stream>>>(p);
    return check_cuda(cudaGetLastError(), "launch(tv rows)");
}

}  // namespace uno
