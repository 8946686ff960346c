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

// probability of token t under the record's distribution (0 if not a survivor)
__device__ inline double rec_prob(const RecView& R, int t) {
    int n = __ldcg(R.n);
    int lo = 0, hi = n - 1;
    while (lo <= hi) {
        int mid = (lo + hi) >> 1;
        int v = __ldcg(R.id + mid);
        if (v == t) return __ldcg(R.w + mid) / __ldcg(R.Z);
        if (v < t) lo = mid + 1;
        else hi = mid - 1;
    }
    return 0.0;
}

// inverse-CDF draw: smallest id (ascending) whose cumulative weight exceeds u * Z
__device__ inline int rec_inv_cdf(const RecView& R, double u) {
    int n = __ldcg(R.n);
    double target = u * __ldcg(R.Z);
    double cum = 0.0;
    int last = -1;
    for (int j = 0; j < n; ++j) {
        double w = __ldcg(R.w + j);
        if (w <= 0.0) continue;
        cum += w;
        last = __ldcg(R.id + j);
        if (cum > target) return last;
    }
    return last;
}

// residual draw: normalise(max(0, p - q)) over p's survivors (q's tokens outside p's
// survivors have p = 0 and so no residual mass); p itself if the residual is empty
__device__ inline int rec_residual(const RecView& P, const RecView& Q, double u) {
    int n = __ldcg(P.n);
    double Zp = __ldcg(P.Z);
    double R = 0.0;
    for (int j = 0; j < n; ++j) {
        double d = __ldcg(P.w + j) / Zp - rec_prob(Q, __ldcg(P.id + j));
        R += d > 0.0 ? d : 0.0;
    }
    if (!(R > 0.0)) return rec_inv_cdf(P, u);
    double target = u * R, cum = 0.0;
    int last = -1;
    for (int j = 0; j < n; ++j) {
        int id = __ldcg(P.id + j);
        double d = __ldcg(P.w + j) / Zp - rec_prob(Q, id);
        if (!(d > 0.0)) continue;
        cum += d;
        last = id;
        if (cum > target) return id;
    }
    return last;
}

// TV(p, q) = 1/2 (sum over p's survivors |p - q| + q's mass outside p's survivors)
__device__ inline double rec_tv(const RecView& P, const RecView& Q) {
    double s = 0.0;
    int np = __ldcg(P.n), nq = __ldcg(Q.n);
    double Zp = __ldcg(P.Z), Zq = __ldcg(Q.Z);
    for (int j = 0; j < np; ++j) s += fabs(__ldcg(P.w + j) / Zp - rec_prob(Q, __ldcg(P.id + j)));
    for (int j = 0; j < nq; ++j)
        if (rec_prob(P, __ldcg(Q.id + j)) == 0.0) s += __ldcg(Q.w + j) / Zq;
    return 0.5 * s;
}

// Per-sequence verify, one warp, lane i = block position i (K <= 32). Rows of sequence b:
// records rbase + i are the verifier rows i = 0..K-1, rbase + K + i - 1 the drafter rows.
__device__ inline void sequence_verify(const VerifyArgs& a, unsigned char* recs, int kcap, int b,
                                       int rows_per_seq, int lane) {
    const int K = a.K;
    const int64_t rbase = (int64_t)b * rows_per_seq;
    const int i = lane;
    const bool act = i < K;
    int tok = -1;
    bool acc = true;
    double pi = 0.0, qi = 0.0, tv = 0.0;
    if (act) {
        RecView P = rec_view(recs, kcap, rbase + i);
        const float* u = a.u + ((int64_t)b * K + i) * 3;
        if (i == 0) {
            tok = a.pos0 ? a.pos0[b] : rec_inv_cdf(P, (double)u[0]);
            pi = (tok >= 0 && tok < a.V) ? rec_prob(P, tok) : 0.0;
        } else {
            RecView Qr = rec_view(recs, kcap, rbase + K + i - 1);
            tok = a.drafts ? a.drafts[(int64_t)b * K + i] : rec_inv_cdf(Qr, (double)u[0]);
            bool in = tok >= 0 && tok < a.V;
            pi = in ? rec_prob(P, tok) : 0.0;
            qi = in ? rec_prob(Qr, tok) : 0.0;
            acc = (double)u[1] * qi < pi;
            if (a.out_tv) tv = rec_tv(P, Qr);
        }
    }
    unsigned rej = __ballot_sync(kFullMask, act && !acc);
    const int n = rej ? (__ffs(rej) - 1) : K;
    if (act) {
        int64_t o = (int64_t)b * K + i;
        a.out_tokens[o] = i < n ? tok : -1;
        if (a.out_p) a.out_p[o] = (float)pi;
        if (a.out_q) a.out_q[o] = (float)qi;
        if (a.out_tv) a.out_tv[o] = (float)tv;
    }
    if (lane == 0) {
        a.out_count[b] = n;
        if (a.out_next && n == K) a.out_next[b] = -1;
    }
    if (n < K && lane == n && a.out_next) {
        RecView P = rec_view(recs, kcap, rbase + n);
        RecView Qr = rec_view(recs, kcap, rbase + K + n - 1);
        a.out_next[b] = rec_residual(P, Qr, (double)a.u[((int64_t)b * K + n) * 3 + 2]);
    }
}

size_t verify_topk_workspace_bytes(const VerifyArgs& a);
uno_status verify_topk_launch(const VerifyArgs& a, void* workspace, cudaStream_t stream);
size_t verify_full_workspace_bytes(const VerifyArgs& a);
uno_status verify_full_launch(const VerifyArgs& a, void* workspace, cudaStream_t stream);

}  // namespace uno
