// verify_common.cuh — pieces shared by the block-verify kernels: logit access, survivor
// records, and the per-sequence verify decisions (draft sampling, acceptance, longest
// accepted prefix, residual resample).
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "verify.cuh"

namespace uno {

template <typename T>
struct Elem;

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int VEC = 8;  // elements per 16-byte vector
};

template <>
struct Elem<float> {
    static constexpr int VEC = 4;
};

// Load this lane's VEC elements starting at element e0 (a multiple of VEC) of `row` as
// one raw 16-byte vector; nvalid of them exist and the missing slots read -inf. A full,
// aligned lane-chunk is one 16-byte streaming load.
template <typename T>
__device__ __forceinline__ uint4 load_raw(const T* row, int64_t e0, int nvalid, bool aligned);

template <>
__device__ __forceinline__ uint4 load_raw<__nv_bfloat16>(const __nv_bfloat16* row, int64_t e0, int nvalid,
                                                          bool aligned) {
    if (nvalid == 8 && aligned) return ld_stream_v4(row + e0);
    const uint16_t* h = reinterpret_cast<const uint16_t*>(row) + e0;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t lo = (2 * q < nvalid) ? h[2 * q] : 0xFF80u;
        uint32_t hi = (2 * q + 1 < nvalid) ? h[2 * q + 1] : 0xFF80u;
        w[q] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <>
__device__ __forceinline__ uint4 load_raw<float>(const float* row, int64_t e0, int nvalid, bool aligned) {
    if (nvalid == 4 && aligned) return ld_stream_v4(row + e0);
    const uint32_t* f = reinterpret_cast<const uint32_t*>(row) + e0;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = q < nvalid ? f[q] : 0xFF800000u;
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename T>
__device__ __forceinline__ float raw_max(const uint4& v);
template <>
__device__ __forceinline__ float raw_max<__nv_bfloat16>(const uint4& v) {
    __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
    __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
    __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162*>(&v.z);
    __nv_bfloat162 d = *reinterpret_cast<const __nv_bfloat162*>(&v.w);
    __nv_bfloat162 m = __hmax2(__hmax2(a, b), __hmax2(c, d));
    return fmaxf(__low2float(m), __high2float(m));
}
template <>
__device__ __forceinline__ float raw_max<float>(const uint4& v) {
    return fmaxf(fmaxf(__uint_as_float(v.x), __uint_as_float(v.y)), fmaxf(__uint_as_float(v.z), __uint_as_float(v.w)));
}

template <typename T>
__device__ __forceinline__ float raw_get(const uint4& v, int j);
template <>
__device__ __forceinline__ float raw_get<__nv_bfloat16>(const uint4& v, int j) {
    uint32_t w = j < 2 ? v.x : (j < 4 ? v.y : (j < 6 ? v.z : v.w));
    return (j & 1) ? bf16_hi(w) : bf16_lo(w);
}
template <>
__device__ __forceinline__ float raw_get<float>(const uint4& v, int j) {
    return __uint_as_float(j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w)));
}

// Unpacked variant (kept for the kernels that use every element).
template <typename T>
__device__ __forceinline__ void load_lane(const T* row, int64_t e0, int nvalid, bool aligned,
                                          float (&x)[Elem<T>::VEC], float& vmax) {
    uint4 v = load_raw<T>(row, e0, nvalid, aligned);
    vmax = raw_max<T>(v);
#pragma unroll
    for (int j = 0; j < Elem<T>::VEC; ++j) x[j] = raw_get<T>(v, j);
}

// ------------------------------------------------------------------------------------
// survivor records (top-k path): the warped row's surviving tokens sorted by id, with
// unnormalised fp64 weights and their total Z (summed in id order).
//   [int32 n][pad][double Z][double w[kcap]][int32 id[kcap]]
// ------------------------------------------------------------------------------------
struct RecView {
    int32_t* n;
    double* Z;
    double* w;
    int32_t* id;
};

__host__ __device__ inline size_t rec_bytes(int kcap) { return ((size_t)16 + 12 * (size_t)kcap + 15) / 16 * 16; }

__device__ inline RecView rec_view(unsigned char* recs, int kcap, int64_t row) {
    unsigned char* base = recs + row * (int64_t)rec_bytes(kcap);
    RecView r;
    r.n = reinterpret_cast<int32_t*>(base);
    r.Z = reinterpret_cast<double*>(base + 8);
    r.w = reinterpret_cast<double*>(base + 16);
    r.id = reinterpret_cast<int32_t*>(base + 16 + 8 * (size_t)kcap);
    return r;
}

// ------------------------------------------------------------------------------------
// Warp-cooperative use of a record staged in shared memory (ids ascending, fp64 weights).
// ------------------------------------------------------------------------------------
struct SRec {
    double* w;
    int32_t* id;
    int n;
    double Z;
};

__device__ __forceinline__ double warp_scan_f64(double v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        double t = __shfl_up_sync(kFullMask, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFullMask, v, o);
    return v;
}

// copy a global record into the warp's slice (w, id arrays of capacity kcap)
__device__ inline SRec warp_stage_rec(unsigned char* recs, int kcap, int64_t row, double* w, int32_t* id, int lane) {
    RecView R = rec_view(recs, kcap, row);
    SRec s;
    s.w = w;
    s.id = id;
    s.n = __ldcg(R.n);
    s.Z = __ldcg(R.Z);
    for (int j = lane; j < s.n; j += 32) {
        w[j] = __ldcg(R.w + j);
        id[j] = __ldcg(R.id + j);
    }
    __syncwarp();
    return s;
}

// probability of token t (0 if not a survivor); every lane gets the same answer
__device__ __forceinline__ double srec_prob(const SRec& R, int t) {
    int lo = 0, hi = R.n - 1;
    while (lo <= hi) {
        int mid = (lo + hi) >> 1;
        int v = R.id[mid];
        if (v == t) return R.w[mid] / R.Z;
        if (v < t) lo = mid + 1;
        else hi = mid - 1;
    }
    return 0.0;
}

// inverse-CDF draw over weights x_j (ascending id order): the first j whose cumulative
// weight exceeds target; the last j with positive weight if rounding leaves no crossing.
template <typename F>
__device__ __forceinline__ int warp_inv_cdf_gen(int n, double target, int lane, F weight) {
    double carry = 0.0;
    int last = -1;
    for (int base = 0; base < n; base += 32) {
        int j = base + lane;
        double x = j < n ? weight(j) : 0.0;
        double incl = warp_scan_f64(x, lane);
        unsigned hit = __ballot_sync(kFullMask, x > 0.0 && carry + incl > target);
        if (hit) return base + __ffs(hit) - 1;
        unsigned pos = __ballot_sync(kFullMask, x > 0.0);
        if (pos) last = base + 31 - __clz(pos);
        carry += __shfl_sync(kFullMask, incl, 31);
    }
    return last;
}

__device__ __forceinline__ int srec_inv_cdf(const SRec& R, double u, int lane) {
    int j = warp_inv_cdf_gen(R.n, u * R.Z, lane, [&](int i) { return R.w[i]; });
    return j >= 0 ? R.id[j] : -1;
}

// TV(p, q) = 1/2 (sum over p's survivors |p - q| + q's mass outside p's survivors)
__device__ __forceinline__ double srec_tv(const SRec& P, const SRec& Q, int lane) {
    double s = 0.0;
    for (int j = lane; j < P.n; j += 32) s += fabs(P.w[j] / P.Z - srec_prob(Q, P.id[j]));
    for (int j = lane; j < Q.n; j += 32)
        if (srec_prob(P, Q.id[j]) == 0.0) s += Q.w[j] / Q.Z;
    return 0.5 * warp_sum_f64(s);
}

// residual draw: normalise(max(0, p - q)) over p's survivors; p itself if that is empty
__device__ __forceinline__ int srec_residual(const SRec& P, const SRec& Q, double u, int lane) {
    auto r = [&](int j) {
        double d = P.w[j] / P.Z - srec_prob(Q, P.id[j]);
        return d > 0.0 ? d : 0.0;
    };
    double R = 0.0;
    for (int j = lane; j < P.n; j += 32) R += r(j);
    R = warp_sum_f64(R);
    if (!(R > 0.0)) return srec_inv_cdf(P, u, lane);
    int j = warp_inv_cdf_gen(P.n, u * R, lane, r);
    return j >= 0 ? P.id[j] : -1;
}

// Per-sequence verify by the whole CTA (NW warps, the first FW of them with two record
// slices each in `region`): warp w evaluates block positions w, w + FW, ...; warp 0 then
// takes the longest accepted prefix, writes the outputs and draws the correction token.
template <int NW>
__device__ void sequence_verify(const VerifyArgs& a, unsigned char* recs, int kcap, int b, int rows_per_seq,
                                unsigned char* region, size_t region_bytes) {
    __shared__ int s_tok[32];
    __shared__ double s_p[32], s_q[32], s_tv[32];
    __shared__ int s_acc[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = a.K;
    const size_t slice = (size_t)kcap * 12;
    int FW = (int)(region_bytes / (2 * slice));
    FW = FW < NW ? FW : NW;
    const int64_t rbase = (int64_t)b * rows_per_seq;
    double* w0 = reinterpret_cast<double*>(region + (size_t)warp * 2 * slice);
    int32_t* i0 = reinterpret_cast<int32_t*>(region + (size_t)warp * 2 * slice + (size_t)kcap * 8);
    double* w1 = reinterpret_cast<double*>(region + (size_t)warp * 2 * slice + slice);
    int32_t* i1 = reinterpret_cast<int32_t*>(region + (size_t)warp * 2 * slice + slice + (size_t)kcap * 8);
    if (warp < FW) {
        for (int i = warp; i < K; i += FW) {
            const float* u = a.u + ((int64_t)b * K + i) * 3;
            SRec P = warp_stage_rec(recs, kcap, rbase + i, w0, i0, lane);
            int tok;
            double pi = 0.0, qi = 0.0, tv = 0.0;
            int acc = 1;
            if (i == 0) {
                tok = a.pos0 && a.pos0[b] >= 0 ? a.pos0[b] : srec_inv_cdf(P, (double)u[0], lane);
                pi = (tok >= 0 && tok < a.V) ? srec_prob(P, tok) : 0.0;
            } else {
                SRec Q = warp_stage_rec(recs, kcap, rbase + K + i - 1, w1, i1, lane);
                tok = a.drafts ? a.drafts[(int64_t)b * K + i] : srec_inv_cdf(Q, (double)u[0], lane);
                bool in = tok >= 0 && tok < a.V;
                pi = in ? srec_prob(P, tok) : 0.0;
                qi = in ? srec_prob(Q, tok) : 0.0;
                acc = (double)u[1] * qi < pi;
                if (a.out_tv) tv = srec_tv(P, Q, lane);
            }
            if (lane == 0) {
                s_tok[i] = tok;
                s_p[i] = pi;
                s_q[i] = qi;
                s_tv[i] = tv;
                s_acc[i] = acc;
            }
            __syncwarp();
        }
    }
    __syncthreads();
    if (warp == 0) {
        const int i = lane;
        const bool act = i < K;
        unsigned rej = __ballot_sync(kFullMask, act && !s_acc[act ? i : 0]);
        const int n = rej ? (__ffs(rej) - 1) : K;
        if (act) {
            int64_t o = (int64_t)b * K + i;
            a.out_tokens[o] = i < n ? s_tok[i] : -1;
            if (a.out_p) a.out_p[o] = (float)s_p[i];
            if (a.out_q) a.out_q[o] = (float)s_q[i];
            if (a.out_tv) a.out_tv[o] = (float)s_tv[i];
        }
        if (lane == 0) a.out_count[b] = n;
        if (a.out_next) {
            int nxt = -1;
            if (n < K) {
                SRec P = warp_stage_rec(recs, kcap, rbase + n, w0, i0, lane);
                SRec Q = warp_stage_rec(recs, kcap, rbase + K + n - 1, w1, i1, lane);
                nxt = srec_residual(P, Q, (double)a.u[((int64_t)b * K + n) * 3 + 2], lane);
            }
            if (lane == 0) a.out_next[b] = nxt;
        }
    }
}

size_t verify_topk_workspace_bytes(const VerifyArgs& a);
uno_status verify_topk_launch(const VerifyArgs& a, void* workspace, cudaStream_t stream);
size_t verify_full_workspace_bytes(const VerifyArgs& a, bool with_lists);
uno_status verify_full_launch(const VerifyArgs& a, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                              bool allow_generic, bool* taken);

}  // namespace uno
