// gated_lora.cu — row-gated LoRA linear on the 5th-generation tensor cores (tcgen05).
//
//   Y = X W0^T + scale * diag(g) (X A^T) B^T
//
// LoopUno project page, "How it works" (one LoRA switched on only for noise positions) and
// "Setup / Recipe" (gated LoRA on all seven projections, noise rows only); uno-qwen3-8B
// model card introduction (seed, prefill, verification and AR rows use the frozen base
// weights).
//
// Three steps on the caller's stream:
//   1. down:  X A^T split over K across CTAs, each split's fp32 partial in its own slice;
//   2. gate:  T = bf16(scale * g[m] * sum of the partials[m, :])   (rows with g = 0 give 0);
//   3. main:  Y = [X | T] [W0 | B]^T — the K loop runs over d_in columns of (X, W0) and then
//             over the r columns of (T, B), accumulating both into one TMEM accumulator.
// Steps 1 and 3 use one warp-specialised kernel: warp 0 issues TMA tile loads into a
// ring of shared-memory stages, warp 1 owns the TMEM accumulator and issues
// tcgen05.mma (kind::f16, bf16 x bf16 -> fp32, 128 x BN x 16 per instruction) from one
// thread, and warps 2-5 read the accumulator back with tcgen05.ld for the epilogue.
// Every mbarrier wait is bounded; on timeout the kernel records UNO_ERR_TIMEOUT in the
// device status word, lets its in-flight copies and MMAs drain (bounded), frees its TMEM
// and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "gated_lora.cuh"

namespace uno {
namespace glora {

constexpr int BM = 128;         // rows per tile (UMMA M)
constexpr int BK = 64;          // K elements per stage: one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;
constexpr int kThreads = 192;   // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: epilogue
constexpr int kSmemBudget = 200 * 1024;

struct Params {
    int M, N;               // output extent
    int kt0, kt1;           // K tiles of segment 0 (X, W0) and segment 1 (T, B)
    int kt_per_split;       // split-K: K tiles per z-slice of the grid (segment 0 only)
    void* out;              // bf16 or fp32 [M, ldo]
    int ldo;
    int out_f32;
    float* red;             // if set: this split's fp32 partial into red[blockIdx.z][M, ldo] instead of out
    uint32_t* status;
};

// ---------------------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// K-major operand tile in shared memory written by TMA with 128-byte swizzling: rows of
// 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);        // start address
    d |= (uint64_t)1u << 16;                        // leading byte offset (unused with this swizzle)
    d |= (uint64_t)(1024u >> 4) << 32;              // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1u << 46;                        // descriptor version (tcgen05)
    d |= (uint64_t)2u << 61;                        // 128-byte swizzle
    return d;
}

// kind::f16 instruction descriptor: bf16 A and B (K-major), fp32 accumulator, M x N
__host__ __device__ constexpr uint32_t instr_desc_bf16(int M, int N) {
    return (1u << 4)                      // D format: f32
           | (1u << 7)                    // A format: bf16
           | (1u << 10)                   // B format: bf16
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <int BN>
constexpr int tmem_cols() { return BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256)); }

template <int BN>
constexpr int stages() {
    return (kSmemBudget - 1024) / (BM * BK * 2 + BN * BK * 2) < 8 ? (kSmemBudget - 1024) / (BM * BK * 2 + BN * BK * 2) : 8;
}

template <int BN>
constexpr size_t smem_bytes() { return (size_t)stages<BN>() * (BM * BK * 2 + BN * BK * 2) + 1024; }

// ---------------------------------------------------------------------------------------
// the GEMM kernel: C[m0:m0+128, n0:n0+BN] over K tiles of segment 0 then segment 1
// ---------------------------------------------------------------------------------------
template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tB0,
            const __grid_constant__ CUtensorMap tA1, const __grid_constant__ CUtensorMap tB1, Params p) {
    constexpr int ST = stages<BN>();
    constexpr uint32_t A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2;
    constexpr uint32_t TCOLS = tmem_cols<BN>();
    extern __shared__ unsigned char smem_dyn[];
    __shared__ __align__(8) uint64_t full[ST], empty[ST], accum;
    __shared__ uint32_t tmem_holder;
    __shared__ int s_abort;

    // 128-byte swizzled tiles need 1024-byte aligned shared-memory addresses
    unsigned char* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    unsigned char* sA = smem;
    unsigned char* sB = smem + (size_t)ST * A_BYTES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
    // K tiles of this CTA: split-K slices cover segment 0 only
    int kb = 0, ke = p.kt0 + p.kt1;
    if (p.kt_per_split > 0) {
        kb = blockIdx.z * p.kt_per_split;
        ke = min(p.kt0, kb + p.kt_per_split);
    }
    const int nk = max(0, ke - kb);

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&accum, 1);
        s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {  // TMEM accumulator: TCOLS fp32 columns x 128 lanes
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_holder)),
                     "r"(TCOLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tA0);
        prefetch_tmap(&tB0);
        if (p.kt1 > 0) {
            prefetch_tmap(&tA1);
            prefetch_tmap(&tB1);
        }
    }
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    const uint32_t tmem = tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer ----
            int it = 0;
            for (; it < nk; ++it) {
                const int s = it % ST;
                if (it >= ST && !mbar_wait(&empty[s], (uint32_t)(((it / ST) & 1) ^ 1))) {
                    s_abort = 1;
                    break;
                }
                if (*reinterpret_cast<volatile int*>(&s_abort)) break;
                const int kt = kb + it;
                mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES);
                if (kt < p.kt0) {
                    tma_load_2d(sA + (size_t)s * A_BYTES, &tA0, kt * BK, m0, &full[s]);
                    tma_load_2d(sB + (size_t)s * B_BYTES, &tB0, kt * BK, n0, &full[s]);
                } else {
                    tma_load_2d(sA + (size_t)s * A_BYTES, &tA1, (kt - p.kt0) * BK, m0, &full[s]);
                    tma_load_2d(sB + (size_t)s * B_BYTES, &tB1, (kt - p.kt0) * BK, n0, &full[s]);
                }
            }
            // drain: wait (bounded) for the loads that no MMA will consume
            if (*reinterpret_cast<volatile int*>(&s_abort))
                for (int j = max(0, it - ST); j < it; ++j) mbar_wait(&full[j % ST], (uint32_t)((j / ST) & 1), 1u << 16);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer (one thread) ----
            constexpr uint32_t idesc = instr_desc_bf16(BM, BN);
            int it = 0;
            for (; it < nk; ++it) {
                const int s = it % ST;
                if (!mbar_wait(&full[s], (uint32_t)((it / ST) & 1))) {
                    s_abort = 1;
                    break;
                }
                tmem_fence_after();
                const uint32_t a0 = smem_u32(sA + (size_t)s * A_BYTES), b0 = smem_u32(sB + (size_t)s * B_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                    const uint32_t off = kk * UMMA_K * 2;  // bytes along K within the 128-byte row
                    umma_bf16(tmem, smem_desc_sw128(a0 + off), smem_desc_sw128(b0 + off), idesc,
                              (it > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&empty[s]);  // the stage is free once these MMAs have read it
            }
            umma_commit(&accum);  // the accumulator is final once every MMA has completed
        }
    } else {
        // ---- epilogue: TMEM -> registers -> global ----
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int row = m0 + q * 32 + lane;
        const bool okw = mbar_wait(&accum, 0);
        tmem_fence_after();
        if (!okw) {
            if (lane == 0) s_abort = 1;
        } else if (nk > 0) {
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t r[32];
                __syncwarp();  // tcgen05.ld is .sync.aligned: the whole warp, converged
                tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, r);
                const int col0 = n0 + c0;
                if (row >= p.M || col0 >= p.N) continue;
                const int ncol = min(32, p.N - col0);
                if (p.red) {
                    // split-K partial: this z-slice's own [M, ldo] fp32 slice, plain stores
                    float* dst = p.red + ((size_t)blockIdx.z * p.M + row) * p.ldo + col0;
                    if (ncol == 32) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4*>(dst + j) = make_float4(
                                __uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                __uint_as_float(r[j + 3]));
                    } else {
                        for (int j = 0; j < ncol; ++j) dst[j] = __uint_as_float(r[j]);
                    }
                } else if (p.out_f32) {
                    float* dst = reinterpret_cast<float*>(p.out) + (size_t)row * p.ldo + col0;
                    if (ncol == 32) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4*>(dst + j) = make_float4(
                                __uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                __uint_as_float(r[j + 3]));
                    } else {
                        for (int j = 0; j < ncol; ++j) dst[j] = __uint_as_float(r[j]);
                    }
                } else {
                    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)row * p.ldo + col0;
                    if (ncol == 32) {
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            uint4 o;
                            __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(r[j]), __uint_as_float(r[j + 1]));
                            __nv_bfloat162 h1 = __floats2bfloat162_rn(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[j + 4]), __uint_as_float(r[j + 5]));
                            __nv_bfloat162 h3 = __floats2bfloat162_rn(__uint_as_float(r[j + 6]), __uint_as_float(r[j + 7]));
                            o.x = *reinterpret_cast<uint32_t*>(&h0);
                            o.y = *reinterpret_cast<uint32_t*>(&h1);
                            o.z = *reinterpret_cast<uint32_t*>(&h2);
                            o.w = *reinterpret_cast<uint32_t*>(&h3);
                            *reinterpret_cast<uint4*>(dst + j) = o;
                        }
                    } else {
                        for (int j = 0; j < ncol; ++j) dst[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
                    }
                }
            }
        } else if (row < p.M) {
            // no K tiles: the product (or this split's partial) is zero
            for (int col = n0; col < min(n0 + BN, p.N); ++col) {
                if (p.red) p.red[((size_t)blockIdx.z * p.M + row) * p.ldo + col] = 0.f;
                else if (p.out_f32) reinterpret_cast<float*>(p.out)[(size_t)row * p.ldo + col] = 0.f;
                else reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)row * p.ldo + col] = __float2bfloat16_rn(0.f);
            }
        }
    }

    tmem_fence_before();
    __syncthreads();
    if (warp == 1) {
        tmem_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS) : "memory");
    }
    if (threadIdx.x == 0 && s_abort) record_device_status(p.status, (uint32_t)UNO_ERR_TIMEOUT);
}

// ---------------------------------------------------------------------------------------
// small element-wise kernels
// ---------------------------------------------------------------------------------------
// T[m, j] = bf16(scale * g[m] * sum_s Tpart[s, m, j])   (r a multiple of 8)
__global__ void gate_kernel(const float* __restrict__ tpart, int splits, const float* __restrict__ gate, float scale,
                            int M, int r, __nv_bfloat16* __restrict__ t) {
    const int64_t n4 = (int64_t)M * r / 4, slice = (int64_t)M * r;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const int m = (int)(i * 4 / r);
        const float g = gate ? scale * gate[m] : 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (g != 0.f)
            for (int s = 0; s < splits; ++s) {
                const float4 v = reinterpret_cast<const float4*>(tpart + s * slice)[i];
                acc.x += v.x;
                acc.y += v.y;
                acc.z += v.z;
                acc.w += v.w;
            }
        __nv_bfloat162 h0 = __floats2bfloat162_rn(g * acc.x, g * acc.y), h1 = __floats2bfloat162_rn(g * acc.z, g * acc.w);
        reinterpret_cast<uint2*>(t)[i] = make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
    }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = __float2bfloat16_rn(src[i]);
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// row-major [rows, cols] bf16 matrix, box of 64 columns x box_rows rows, 128-byte swizzle
uno_status make_tmap(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return set_error(UNO_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(UNO_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return UNO_OK;
}

template <int BN>
uno_status launch_gemm(const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1, const CUtensorMap& b1,
                       const Params& p, dim3 grid, cudaStream_t stream) {
    static bool attr = false;
    if (!attr) {
        uno_status s = check_cuda(cudaFuncSetAttribute(gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)smem_bytes<BN>()),
                                  "cudaFuncSetAttribute(gemm)");
        if (s != UNO_OK) return s;
        attr = true;
    }
    gemm_kernel<BN><<<grid, kThreads, smem_bytes<BN>(), stream>>>(a0, b0, a1, b1, p);
    return check_cuda(cudaGetLastError(), "launch(gated lora gemm)");
}

uno_status launch_bn(int BN, const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1,
                     const CUtensorMap& b1, const Params& p, dim3 grid, cudaStream_t stream) {
    switch (BN) {
        case 16: return launch_gemm<16>(a0, b0, a1, b1, p, grid, stream);
        case 32: return launch_gemm<32>(a0, b0, a1, b1, p, grid, stream);
        case 64: return launch_gemm<64>(a0, b0, a1, b1, p, grid, stream);
        case 128: return launch_gemm<128>(a0, b0, a1, b1, p, grid, stream);
        case 256: return launch_gemm<256>(a0, b0, a1, b1, p, grid, stream);
    }
    return set_error(UNO_ERR_UNSUPPORTED, "tile width %d", BN);
}

int down_bn(int64_t rank) {
    int r16 = (int)((rank + 15) / 16 * 16);
    return r16 <= 16 ? 16 : (r16 <= 32 ? 32 : (r16 <= 64 ? 64 : (r16 <= 128 ? 128 : 256)));
}

// split-K of the down-projection: about one wave of CTAs over the M tiles, each split
// at least one K tile
struct DownSplit {
    int splits, per;
};
DownSplit down_split(int64_t M, int64_t d_in) {
    const int m_tiles = (int)((M + BM - 1) / BM), kt0 = (int)(d_in / BK);
    int splits = 148 / m_tiles;
    splits = splits < 1 ? 1 : (splits > kt0 ? kt0 : splits);
    const int per = (kt0 + splits - 1) / splits;
    return {(kt0 + per - 1) / per, per};
}

struct WsLayout {
    size_t tacc, t, x, w0, a, b, total;
};

WsLayout ws_layout(int64_t M, int64_t d_in, int64_t d_out, int64_t rank, uno_dtype dtype) {
    WsLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    L.tacc = take((size_t)down_split(M, d_in).splits * M * rank * 4);  // per-split partials
    L.t = take((size_t)M * rank * 2);
    if (dtype == UNO_F32) {
        L.x = take((size_t)M * d_in * 2);
        L.w0 = take((size_t)d_out * d_in * 2);
        L.a = take((size_t)rank * d_in * 2);
        L.b = take((size_t)d_out * rank * 2);
    }
    L.total = off;
    return L;
}

}  // namespace glora

size_t gated_lora_workspace_bytes(int64_t M, int64_t d_in, int64_t d_out, int64_t rank, uno_dtype dtype) {
    return glora::ws_layout(M, d_in, d_out, rank, dtype).total;
}

uno_status gated_lora_launch(const GatedLoraArgs& g, void* workspace, cudaStream_t stream) {
    using namespace glora;
    const WsLayout L = ws_layout(g.M, g.d_in, g.d_out, g.rank, g.dtype);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    float* tacc = reinterpret_cast<float*>(ws + L.tacc);
    __nv_bfloat16* t = reinterpret_cast<__nv_bfloat16*>(ws + L.t);
    const void *x = g.x, *w0 = g.w0, *a = g.a, *b = g.b;
    uno_status s;
    if (g.dtype == UNO_F32) {  // round the fp32 operands to bf16 once
        struct { const void* src; size_t off; int64_t n; } cv[4] = {
            {g.x, L.x, g.M * g.d_in}, {g.w0, L.w0, g.d_out * g.d_in}, {g.a, L.a, g.rank * g.d_in}, {g.b, L.b, g.d_out * g.rank}};
        for (auto& c : cv) {
            f32_to_bf16_kernel<<<592, 256, 0, stream>>>(static_cast<const float*>(c.src),
                                                      reinterpret_cast<__nv_bfloat16*>(ws + c.off), c.n);
            if ((s = check_cuda(cudaGetLastError(), "launch(f32->bf16)")) != UNO_OK) return s;
        }
        x = ws + L.x;
        w0 = ws + L.w0;
        a = ws + L.a;
        b = ws + L.b;
    }
    const int M = (int)g.M, din = (int)g.d_in, dout = (int)g.d_out, r = (int)g.rank;
    const int m_tiles = (M + BM - 1) / BM;
    uint32_t* status = device_status_ptr();

    // ---- 1. down: per-split partials of X A^T (fp32, plain stores) ----
    CUtensorMap tX, tA, tW0, tT, tBl;
    const int bnd = down_bn(r);
    if ((s = make_tmap(&tX, x, M, din, BM)) != UNO_OK) return s;
    if ((s = make_tmap(&tA, a, r, din, bnd)) != UNO_OK) return s;
    const int kt0 = din / BK;
    const DownSplit ds = down_split(M, din);
    Params pd{};
    pd.M = M;
    pd.N = r;
    pd.kt0 = kt0;
    pd.kt1 = 0;
    pd.kt_per_split = ds.per;
    pd.red = tacc;
    pd.ldo = r;
    pd.status = status;
    if ((s = launch_bn(bnd, tX, tA, tX, tA, pd, dim3(1, m_tiles, ds.splits), stream)) != UNO_OK) return s;

    // ---- 2. gate: T = bf16(scale * g * sum of the partials) ----
    {
        const int64_t n4 = (int64_t)M * r / 4;
        const int blocks = (int)((n4 + 255) / 256 < 1184 ? (n4 + 255) / 256 : 1184);
        gate_kernel<<<blocks, 256, 0, stream>>>(tacc, ds.splits, g.gate, g.scale, M, r, t);
        if ((s = check_cuda(cudaGetLastError(), "launch(gate)")) != UNO_OK) return s;
    }

    // ---- 3. main: Y = [X | T] [W0 | B]^T ----
    int BN = 256;
    while (BN > 64 && (int64_t)m_tiles * ((dout + BN - 1) / BN) < 120) BN >>= 1;
    if ((s = make_tmap(&tW0, w0, dout, din, BN)) != UNO_OK) return s;
    if ((s = make_tmap(&tT, t, M, r, BM)) != UNO_OK) return s;
    if ((s = make_tmap(&tBl, b, dout, r, BN)) != UNO_OK) return s;
    Params pm{};
    pm.M = M;
    pm.N = dout;
    pm.kt0 = kt0;
    pm.kt1 = (r + BK - 1) / BK;
    pm.kt_per_split = 0;
    pm.out = g.y;
    pm.ldo = dout;
    pm.out_f32 = g.dtype == UNO_F32;
    pm.red = nullptr;
    pm.status = status;
    return launch_bn(BN, tX, tW0, tT, tBl, pm, dim3((dout + BN - 1) / BN, m_tiles, 1), stream);
}

}  // namespace uno
