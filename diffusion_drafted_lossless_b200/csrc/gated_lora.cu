// gated_lora.cu — row-gated LoRA linear on the 5th-generation tensor cores (tcgen05).
//
//   Y = X W0^T + scale * diag(g) (X A^T) B^T
//
// LoopUno project page, "How it works" (one LoRA switched on only for noise positions) and
// "Setup / Recipe" (gated LoRA on all seven projections, noise rows only); uno-qwen3-8B
// model card introduction (seed, prefill, verification and AR rows use the frozen base
// weights).
//
// One persistent kernel per call, one CTA per SM, as many CTAs as can be resident at once
// (a cooperative launch where the runtime takes it). CTA c takes the work items
// c, c + G, c + 2G, ... (G CTAs):
//   1. adapter items (m, s), first in the list: the fp32 product X A^T of row tile m over
//      the s-th range of K. With one range it is written at once as
//      T = bf16(scale * g * (X A^T)); with several, each stores an fp32 partial and the item
//      that completes row tile m last (a ticket) sums the partials into T. Row tile m's T is
//      then published with a release flag carrying this call's epoch.
//   2. output tiles (m, n): Y[m, n] = [X | T] [W0 | B]^T. The K loop runs over the d_in
//      columns of (X, W0) and then over the r columns of (T, B), all into one TMEM
//      accumulator; the loads of (T, B) wait (bounded) for row tile m's flag, by which
//      time the adapter items, scheduled first everywhere, have normally long finished.
// Warp roles: warp 0 issues TMA tile loads into a ring of shared-memory stages that runs on
// across items; warp 1 owns TMEM (two accumulators) and issues tcgen05.mma (kind::f16,
// bf16 x bf16 -> fp32, 128 x N x 16) from one thread; warps 2-5 drain one accumulator to
// global memory while the next item accumulates into the other.
// A second form (UNO_LORA_CG=2) runs each item on a cluster of two CTAs: one tcgen05.mma
// stream with cta_group::2 issued by the leader computes a 256 x N tile, each CTA holding
// its 128 rows of A and half of B, the TMA loads of both completing on the leader's
// mbarriers (plain loads, no multicast).
// Every wait is bounded; on timeout the kernel records UNO_ERR_TIMEOUT in the device status
// word, stops issuing work, lets in-flight copies drain (bounded), frees its TMEM and
// returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <chrono>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "gated_lora.cuh"

namespace uno {
namespace glora {

constexpr int BM = 128;          // rows per tile (UMMA M)
constexpr int BK = 64;           // K elements per stage: one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;
constexpr int kThreads = 192;    // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: epilogue
constexpr int kEpiThreads = 128;
constexpr int kMaxStages = 8;
constexpr int kSmemBudget = 220 * 1024;
constexpr uint32_t A_BYTES = BM * BK * 2;
constexpr uint32_t kFlagPolls = 1u << 22;  // polls of a T flag, each after a short sleep

struct Params {
    int M, N, r;                  // rows, d_out, rank
    int kt0, kt1;                 // K tiles of (X, W0) and of (T, B)
    int m_tiles;                  // 128-row tiles (T flags, tickets)
    int m_units;                  // row units of the work items: 128 x CG rows
    int splits, per;              // adapter items: m_units x splits, `per` K tiles each (one T partial each)
    int n_adapter, n_items;       // adapter items, all items
    int n_tiles;                  // column tiles of the output
    int ksplit, kper;             // output items per tile (split over K), K tiles of (X, W0) each
    int rb;                       // adapter accumulator width: r rounded up to 16 x CG
    int stages;                   // shared-memory ring depth
    uint32_t b_bytes;             // bytes of one B-operand K slab (max(BN, rb) rows of 64 elements)
    int ws;                       // K slabs per main K step (1 or 2: X/W0/A loads are 3-D boxes of ws slabs)
    int tws;                      // K slabs per (T, B) step; T and B are 3-D maps when r is a multiple of 64
    int t3d;
    uint32_t cb;                  // TMEM columns of one accumulator
    void* y;                      // [M, N] bf16 or fp32
    int out_f32;
    float* ypart;                 // [ksplit][M][N] fp32 partials of the output (ksplit > 1)
    unsigned long long* otickets; // [m_tiles * n_tiles]: (epoch << 16) | output partials stored
    __nv_bfloat16* t;             // [splits][M][r] bf16 T partials (their sum is T)
    const float* gate;            // [M] or NULL (all zero)
    float scale;
    unsigned long long* flags;    // [m_tiles][splits]: the epoch once row tile m's T partial s is written
    unsigned long long* header;   // [5]: the next execution's epoch and exit counter (see Header)
    unsigned long long host_tag;  // lower bound for this execution's epoch (fresh per host call), < 2^48
    uint32_t flag_polls;          // polls of a T flag before the wait gives up
    int epi_tma;                  // bf16 output tiles leave through shared memory and TMA stores
    uint32_t epi_off;             // byte offset of the epilogue staging buffers in dynamic smem
    int withhold_flags;           // test switch: adapter items do not publish T (every wait on it runs out)
    long long* trace;             // UNO_LORA_TRACE (profiling aid): per-K-step SM clocks of three CTAs, or NULL
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

// a 3-D box (x fastest): here 64 columns x rows x K slabs of a row-major matrix, landing in
// shared memory slab after slab
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// TMA store of a 2-D box from shared memory (bulk group of this thread)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, const void* src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(smem_u32(src))
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most N of this thread's bulk groups still read their shared-memory source
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

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


__device__ __forceinline__ void named_sync_epilogue() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); }

__device__ __forceinline__ bool wait_flag(const unsigned long long* f, unsigned long long epoch, uint32_t polls) {
    for (uint32_t i = 0; i < polls; ++i) {
        unsigned long long v;
        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(f) : "memory");
        if (v == epoch) {
            // T was written through the generic proxy; the TMA loads read it through the async one
            asm volatile("fence.proxy.async.global;" ::: "memory");
            return true;
        }
        __nanosleep(64);
    }
    return false;
}

// Wait for an mbarrier phase (bounded), giving up early once another role of this CTA has
// aborted: a role that waits for work the aborted one will never deliver stops at once.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 0; i < kWaitLimit; i += 256) {
        if (mbar_wait(bar, parity, 256)) return true;
        if (*abort_flag) return false;
    }
    return false;
}

// one more partial of row tile m stored; true for the one that completes the tile
__device__ __forceinline__ bool take_ticket(unsigned long long* t, unsigned long long epoch, int splits) {
    unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(t), now = 0;
    for (int i = 0; i < 1 << 20; ++i) {
        now = (old >> 16) == epoch ? old + 1 : ((epoch << 16) | 1ull);
        const unsigned long long seen = atomicCAS(t, old, now);
        if (seen == old) break;
        old = seen;
    }
    __threadfence();
    return (int)(now & 0xFFFFull) == splits;
}

constexpr unsigned long long kEpochMask = 0xFFFFFFFFFFFFull;

// The workspace header: [0] the next execution's epoch, [1] its complement (the header is
// valid only when they match), [2] which exit counter the next execution uses (0 or 1),
// [3..4] the two exit counters. The counter a valid header names is zero when the execution
// starts: the previous execution's last CTA cleared it.
struct Header {
    unsigned long long epoch, check, slot, count[2];
};

// This execution's epoch and exit counter. Each CTA reads the header when it starts, and
// only the last CTA of the grid to finish rewrites it (retire_epoch), so all CTAs see the
// same values. The epoch is the larger of the header's stored one and the host's tag, so
// it is above every epoch this workspace has seen: a CUDA-graph replay, whose host tag is
// frozen at capture, still gets a fresh epoch, and no flag or ticket left by an earlier
// execution (or unrelated data in a fresh workspace, which fails the check) can match it.
// slot = -1: the header was not valid; the CTAs then count their exits with a tagged
// compare-and-swap ticket instead (contended, but only on a workspace's first use).
__device__ __forceinline__ unsigned long long read_epoch(const unsigned long long* hdr, unsigned long long host_tag,
                                                         int* slot) {
    const Header* h = reinterpret_cast<const Header*>(hdr);
    const unsigned long long e = __ldcg(&h->epoch), chk = __ldcg(&h->check), sl = __ldcg(&h->slot);
    const bool valid = chk == ~e && sl <= 1ull;
    *slot = valid ? (int)sl : -1;
    const unsigned long long stored = valid ? (e & kEpochMask) : 0ull;
    const unsigned long long ep = stored > host_tag ? stored : host_tag;
    return ep == 0 ? 1ull : ep;
}

// Called once per CTA after all of its work: the last CTA to finish stores epoch + 1 and the
// other exit counter, cleared, for the next execution on this workspace.
__device__ __forceinline__ void retire_epoch(unsigned long long* hdr, unsigned long long epoch, int slot, int ctas) {
    Header* h = reinterpret_cast<Header*>(hdr);
    __threadfence();
    bool last;
    if (slot >= 0) {
        last = atomicAdd(&h->count[slot], 1ull) + 1ull == (unsigned long long)ctas;
    } else {
        last = take_ticket(&h->count[0], epoch, ctas);
    }
    if (last) {
        const int next = slot == 0 ? 1 : 0;
        unsigned long long nx = (epoch + 1) & kEpochMask;
        if (nx == 0) nx = 1;
        h->count[next] = 0ull;
        h->slot = (unsigned long long)next;
        h->epoch = nx;
        h->check = ~nx;
        __threadfence();
    }
}

struct Item {
    bool adapter;
    int m, j;    // row unit (128 x CG rows); split (adapter) or column tile (output)
    int s;       // output: K split (the last one also runs the (T, B) columns)
    int kb, ke;  // K tiles [kb, ke)
};

__device__ __forceinline__ Item decode(const Params& p, int item) {
    Item it;
    if (item < p.n_adapter) {
        it.adapter = true;
        it.m = item % p.m_units;
        it.j = item / p.m_units;
        it.s = 0;
        it.kb = it.j * p.per;
        it.ke = min(p.kt0, it.kb + p.per);
    } else {
        const int q = item - p.n_adapter;
        it.adapter = false;
        it.m = q % p.m_units;  // row units fastest: concurrent tiles share W0's column block
        const int js = q / p.m_units;
        it.s = js % p.ksplit;
        it.j = js / p.ksplit;
        it.kb = it.s * p.kper;
        it.ke = it.s == p.ksplit - 1 ? p.kt0 + p.splits * p.kt1 : it.kb + p.kper;
    }
    return it;
}

// ---- pair (cta_group::2) forms: one MMA over the two CTAs of a cluster ----
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t map_to_rank(const void* local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    return remote;
}
__device__ __forceinline__ void pair_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA load into this CTA's shared memory whose completed bytes count on the leader CTA's
// mbarrier (cluster address `bar`)
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8, %9, %10, %11, %12}, p;\n\t}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u),
        "r"(0u), "r"(0u));
}
// arrive on the mbarrier at this offset in both CTAs of the pair once the MMAs complete
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"((unsigned short)3)
        : "memory");
}
// arrive on this CTA's mbarrier once the pair's MMAs issued so far complete
__device__ __forceinline__ void umma_commit_pair_local(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

// UNO_LORA_TRACE: SM clock at event e (0: loads issued, 1: stage landed, 2: MMAs committed)
// of K step g, for CTAs 0, 20 and 100
__device__ __forceinline__ void gl_mark(const Params& p, int e, uint32_t g) {
    if (p.trace == nullptr || g >= 512) return;
    const int slot = blockIdx.x == 0 ? 0 : (blockIdx.x == 20 ? 1 : (blockIdx.x == 100 ? 2 : -1));
    if (slot >= 0) p.trace[(slot * 6 + e) * 512 + g] = clock64();
}

// CG = 1: one CTA computes a 128 x N tile. CG = 2: the two CTAs of a cluster compute a
// 256 x N tile with one MMA stream issued by the leader (rank 0): each CTA holds its 128
// rows of A and half of the N rows of B, and its own 128-lane accumulator.
template <int BN, int CG>
__global__ void __launch_bounds__(kThreads, 1)
lora_gemm_kernel(const __grid_constant__ CUtensorMap tX, const __grid_constant__ CUtensorMap tW0,
                 const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tT,
                 const __grid_constant__ CUtensorMap tB, const __grid_constant__ CUtensorMap tY, Params p) {
    extern __shared__ unsigned char smem_dyn[];
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages], tfull[2], tempty[2], drain;
    __shared__ uint32_t tmem_holder;
    __shared__ int s_abort, s_last;
    __shared__ unsigned long long s_epoch;
    __shared__ int s_slot;

    // 128-byte swizzled tiles need 1024-byte aligned shared-memory addresses
    unsigned char* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
    const int ST = p.stages;
    const int WS = p.ws;                               // K slabs per main K step
    const int TWS = p.tws, t3d = p.t3d;                // K slabs per (T, B) step; 3-D maps for T and B
    const uint32_t a_stage = (uint32_t)WS * A_BYTES;  // bytes of a stage's A tiles
    unsigned char* sA = smem;
    unsigned char* sB = smem + (size_t)ST * a_stage;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &s_abort;
    if constexpr (CG == 2) {
        // the pair form needs its two-CTA cluster: a launch that arrives without it (a
        // profiler may run a cooperative cluster launch as single CTAs) records an error and
        // returns before any cta_group::2 instruction (the test is uniform over the grid)
        uint32_t nct;
        asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(nct));
        if (nct != 2u) {
            if (threadIdx.x == 0 && blockIdx.x == 0) record_device_status(p.status, (uint32_t)UNO_ERR_UNSUPPORTED);
            return;
        }
    }
    const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int unit0 = blockIdx.x / CG, units = gridDim.x / CG;  // this CTA's pair and the pair count

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], CG * kEpiThreads / 32);
        }
        mbar_init(&drain, 1);
        s_abort = 0;
        s_epoch = read_epoch(p.header, p.host_tag, &s_slot);
        fence_mbar_init();
    }
    if (warp == 1) {  // two accumulators of cb fp32 columns x 128 lanes (in each CTA of a pair)
        if constexpr (CG == 2) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(&tmem_holder)),
                         "r"(2 * p.cb)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(&tmem_holder)),
                         "r"(2 * p.cb)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tX);
        prefetch_tmap(&tW0);
        prefetch_tmap(&tA);
        prefetch_tmap(&tT);
        prefetch_tmap(&tB);
        if (p.epi_tma) prefetch_tmap(&tY);
    }
    tmem_fence_before();
    __syncthreads();
    if constexpr (CG == 2) pair_sync();  // the peer's mbarriers exist before any remote arrive
    tmem_fence_after();
    const uint32_t tmem = tmem_holder;
    const unsigned long long epoch = s_epoch;

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer (each CTA loads its own rows of A and its half of B) ----
            const uint32_t lead_full0 = CG == 2 ? map_to_rank(&full[0], 0) : 0u;
            // (the parameters the loop reads, in registers: every asm statement below clobbers memory)
            const int kt0 = p.kt0, kt1 = p.kt1, M = p.M, splits = p.splits, rb = p.rb;
            const uint32_t bbytes = (uint32_t)WS * p.b_bytes, polls = p.flag_polls;
            unsigned long long* const flags = p.flags;
            uint32_t g = 0;       // K steps issued by this CTA, across items
            int s = 0;            // their stage: g mod ST
            uint32_t ph = 0;      // and its pass over the ring, mod 2
            for (int item = unit0; item < p.n_items && !*abort_flag; item += units) {
                const Item w = decode(p, item);
                const int m0 = w.m * BM * CG + (int)rank * BM;
                const int nrows = w.adapter ? rb : BN;  // B rows of the whole (pair) tile
                const int n0 = w.adapter ? (int)rank * (nrows / CG) : w.j * BN + (int)rank * (BN / CG);
                const uint32_t tx1 = CG * A_BYTES + (uint32_t)nrows * 128u;  // bytes of one K slab
                int ts = 0, tk = 0;  // the (T, B) K tiles run over T's partials in turn: partial ts, its K tile tk
                for (int kt = w.kb; kt < w.ke; ++kt, ++g) {
                    gl_mark(p, 5, g);
                    if (g >= (uint32_t)ST && !mbar_wait(&empty[s], ph ^ 1u)) {
                        *abort_flag = 1;
                        break;
                    }
                    const bool tpart = !w.adapter && kt >= kt0;
                    // rows past M have no T (their loads are zero-filled or not stored): nothing to wait for
                    if (tpart && tk == 0 && m0 < M && !wait_flag(&flags[(m0 / BM) * splits + ts], epoch, polls)) {
                        *abort_flag = 1;
                        break;
                    }
                    if (*abort_flag) break;
                    unsigned char* a = sA + (size_t)s * a_stage;
                    unsigned char* b = sB + (size_t)s * bbytes;
                    const CUtensorMap* ma = tpart ? &tT : &tX;
                    const CUtensorMap* mb = w.adapter ? &tA : (tpart ? &tB : &tW0);
                    const int kx = (tpart ? tk * TWS : kt) * BK;  // (2-D (T, B) loads)
                    const int kz = tpart ? tk * TWS : kt * WS;      // (3-D loads: the first K slab)
                    const int ma_row = tpart ? ts * M + m0 : m0;  // partial ts's rows follow the earlier partials
                    if (tpart && ++tk == kt1) {
                        tk = 0;
                        ++ts;
                    }
                    const int st = s;
                    if (++s == ST) {
                        s = 0;
                        ph ^= 1u;
                    }
                    gl_mark(p, 3, g);
                    if (leader) mbar_arrive_expect_tx(&full[st], (uint32_t)(tpart ? TWS : WS) * tx1);
                    // every operand is a 3-D map (64 columns x rows x K slabs, several slabs per
                    // box), except T and B when r is not a multiple of 64
                    const bool two_d = tpart && !t3d;
                    if constexpr (CG == 2) {
                        const uint32_t bar = lead_full0 + (uint32_t)st * 8u;
                        if (two_d) {
                            tma_load_2d_pair(a, ma, kx, ma_row, bar);
                            tma_load_2d_pair(b, mb, kx, n0, bar);
                        } else {
                            tma_load_3d_pair(a, ma, 0, ma_row, kz, bar);
                            tma_load_3d_pair(b, mb, 0, n0, kz, bar);
                        }
                    } else {
                        if (two_d) {
                            tma_load_2d(a, ma, kx, ma_row, &full[st]);
                            gl_mark(p, 4, g);
                            tma_load_2d(b, mb, kx, n0, &full[st]);
                        } else {
                            tma_load_3d(a, ma, 0, ma_row, kz, &full[st]);
                            gl_mark(p, 4, g);
                            tma_load_3d(b, mb, 0, n0, kz, &full[st]);
                        }
                    }
                    gl_mark(p, 0, g);
                }
            }
            // on abort: wait (bounded) for the loads that no MMA will consume
            if (*abort_flag && leader) {
                const uint32_t lo = g > (uint32_t)ST ? g - ST : 0;
                for (uint32_t j = lo; j < g; ++j) mbar_wait(&full[j % ST], (j / ST) & 1, 1u << 16);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---- MMA issuer (one thread of the leader CTA) ----
            const uint32_t cb = p.cb, rb = (uint32_t)p.rb, bbytes = (uint32_t)WS * p.b_bytes;
            const int kt0 = p.kt0;
            const uint64_t da0 = smem_desc_sw128(smem_u32(sA)), db0 = smem_desc_sw128(smem_u32(sB));
            uint32_t g = 0, li = 0;
            int s = 0;        // stage of K step g
            uint32_t ph = 0;  // its pass over the ring, mod 2
            for (int item = unit0; item < p.n_items && !*abort_flag; item += units, ++li) {
                const Item w = decode(p, item);
                const int buf = li & 1;
                if (li >= 2 && !wait_or_abort(&tempty[buf], ((li >> 1) & 1) ^ 1, abort_flag)) {
                    *abort_flag = 1;
                    break;
                }
                tmem_fence_after();
                const uint32_t d = tmem + (uint32_t)buf * cb;
                const uint32_t idesc = instr_desc_bf16(BM * CG, w.adapter ? (int)rb : BN);
                bool ok = true;
                for (int kt = w.kb; kt < w.ke; ++kt, ++g) {
                    if (!wait_or_abort(&full[s], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    gl_mark(p, 1, g);
                    tmem_fence_after();
                    // descriptors of this stage's tiles: the start-address field (address >> 4)
                    // of the ring's base plus the stage offset (no carry: shared addresses < 2^18)
                    const uint64_t da = da0 + (uint64_t)(((uint32_t)s * a_stage) >> 4);
                    const uint64_t db = db0 + (uint64_t)(((uint32_t)s * bbytes) >> 4);
                    // a main step holds WS K slabs (slab j of B at j x its box rows x 128 bytes);
                    // a (T, B) step one
                    const int slabs = (!w.adapter && kt >= kt0) ? TWS : WS;
                    const uint32_t bslab = ((w.adapter ? rb : (uint32_t)BN) / CG * 128u) >> 4;
                    for (int sl = 0; sl < slabs; ++sl) {
#pragma unroll
                        for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                            const uint64_t off = (uint64_t)((kk * UMMA_K * 2) >> 4);  // 32 bytes along K per step
                            const uint32_t acc = (kt > w.kb || sl > 0 || kk > 0) ? 1u : 0u;
                            const uint64_t oa = off + (uint64_t)sl * (A_BYTES >> 4), ob = off + (uint64_t)sl * bslab;
                            if constexpr (CG == 2)
                                umma_bf16_pair(d, da + oa, db + ob, idesc, acc);
                            else
                                umma_bf16(d, da + oa, db + ob, idesc, acc);
                        }
                    }
                    // the stage is free (in both CTAs) once these MMAs have read it
                    if constexpr (CG == 2) umma_commit_pair(&empty[s]);
                    else umma_commit(&empty[s]);
                    gl_mark(p, 2, g);
                    if (++s == ST) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
                // the accumulator is final once every MMA has completed
                if constexpr (CG == 2) umma_commit_pair(&tfull[buf]);
                else umma_commit(&tfull[buf]);
            }
            if (*abort_flag) {
                // let every MMA issued so far complete before the accumulators are freed
                if constexpr (CG == 2) umma_commit_pair_local(&drain);
                else umma_commit(&drain);
                mbar_wait(&drain, 0, 1u << 16);
            }
        }
    } else {
        // ---- epilogue: TMEM -> registers -> global, four warps, one TMEM lane quarter each ----
        const int q = warp & 3;
        const int et = threadIdx.x - 64;  // 0..127 across the epilogue warps
        const uint32_t lead_tempty0 = CG == 2 ? map_to_rank(&tempty[0], 0) : 0u;
        // TMA-store epilogue: two 32 x 32 bf16 staging boxes per warp (64-byte swizzle)
        unsigned char* stage_box = smem + p.epi_off + (size_t)q * 4096;
        uint32_t chunk = 0;  // boxes this warp has stored
        uint32_t li = 0;
        for (int item = unit0; item < p.n_items; item += units, ++li) {
            const Item w = decode(p, item);
            const int buf = li & 1;
            const int m0 = w.m * BM * CG + (int)rank * BM;
            const int row = m0 + q * 32 + lane;
            bool ok = !*abort_flag && wait_or_abort(&tfull[buf], (li >> 1) & 1, abort_flag);
            tmem_fence_after();
            if (!ok) *abort_flag = 1;
            const uint32_t taddr = tmem + (uint32_t)buf * p.cb + ((uint32_t)(q * 32) << 16);
            if (ok && w.adapter) {
                const float gs = (row < p.M && p.gate) ? p.scale * p.gate[row] : 0.f;
                for (int c0 = 0; c0 < p.rb; c0 += 32) {
                    uint32_t r[32];
                    __syncwarp();
                    tmem_ld32(taddr + (uint32_t)c0, r);
                    if (row >= p.M || c0 >= p.r) continue;
                    const int ncol = min(32, p.r - c0);  // a multiple of 8
                    {
                        __nv_bfloat16* dst = p.t + ((size_t)w.j * p.M + row) * p.r + c0;
                        for (int j = 0; j < ncol; j += 8) {
                            __nv_bfloat162 h0 = __floats2bfloat162_rn(gs * __uint_as_float(r[j]), gs * __uint_as_float(r[j + 1]));
                            __nv_bfloat162 h1 = __floats2bfloat162_rn(gs * __uint_as_float(r[j + 2]), gs * __uint_as_float(r[j + 3]));
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(gs * __uint_as_float(r[j + 4]), gs * __uint_as_float(r[j + 5]));
                            __nv_bfloat162 h3 = __floats2bfloat162_rn(gs * __uint_as_float(r[j + 6]), gs * __uint_as_float(r[j + 7]));
                            *reinterpret_cast<uint4*>(dst + j) =
                                make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                                           *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
                        }
                    }
                }
            } else if (ok) {
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t r[32];
                    __syncwarp();
                    tmem_ld32(taddr + (uint32_t)c0, r);
                    const int col0 = w.j * BN + c0;
                    // (the TMA-store path keeps every lane: the store leaves rows past M out)
                    if (col0 >= p.N || (row >= p.M && !p.epi_tma)) continue;
                    const int ncol = min(32, p.N - col0);  // a multiple of 32: N is a multiple of 64
                    if (p.ksplit > 1) {  // this split's fp32 partial
                        float* dst = p.ypart + ((size_t)w.s * p.M + row) * p.N + col0;
                        for (int j = 0; j < ncol; j += 4)
                            *reinterpret_cast<float4*>(dst + j) =
                                make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                            __uint_as_float(r[j + 3]));
                    } else if (p.out_f32) {
                        float* dst = reinterpret_cast<float*>(p.y) + (size_t)row * p.N + col0;
                        for (int j = 0; j < ncol; j += 4)
                            *reinterpret_cast<float4*>(dst + j) =
                                make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                            __uint_as_float(r[j + 3]));
                    } else if (p.epi_tma) {
                        // row `lane` of this warp's 32-row box: four 16-byte chunks, chunk c at
                        // c ^ ((lane >> 1) & 3) (the 64-byte swizzle the tensor map names)
                        unsigned char* box = stage_box + (chunk & 1) * 2048;
                        if (chunk >= 2) {  // the store issued from this box two chunks ago has read it
                            if (lane == 0) bulk_wait_read<1>();
                            __syncwarp();
                        }
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(r[j]), __uint_as_float(r[j + 1]));
                            __nv_bfloat162 h1 = __floats2bfloat162_rn(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[j + 4]), __uint_as_float(r[j + 5]));
                            __nv_bfloat162 h3 = __floats2bfloat162_rn(__uint_as_float(r[j + 6]), __uint_as_float(r[j + 7]));
                            const int c = (j >> 3) ^ ((lane >> 1) & 3);
                            *reinterpret_cast<uint4*>(box + lane * 64 + c * 16) =
                                make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                                           *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tY, col0, m0 + q * 32, box);
                            bulk_commit_group();
                        }
                        ++chunk;
                    } else {
                        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.y) + (size_t)row * p.N + col0;
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(r[j]), __uint_as_float(r[j + 1]));
                            __nv_bfloat162 h1 = __floats2bfloat162_rn(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[j + 4]), __uint_as_float(r[j + 5]));
                            __nv_bfloat162 h3 = __floats2bfloat162_rn(__uint_as_float(r[j + 6]), __uint_as_float(r[j + 7]));
                            *reinterpret_cast<uint4*>(dst + j) =
                                make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                                           *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
                        }
                    }
                }
            }
            // the accumulator may be refilled (the leader's MMA waits for both CTAs' warps)
            tmem_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (CG == 2) mbar_arrive_remote(lead_tempty0 + (uint32_t)buf * 8u);
                else mbar_arrive(&tempty[buf]);
            }

            if (!w.adapter && p.ksplit > 1) {
                // the split that stores a tile's partials last (a ticket) sums them into Y
                // (all four warps take every barrier)
                const int tile = (m0 / BM) * p.n_tiles + w.j;
                __threadfence();
                named_sync_epilogue();
                if (et == 0)
                    s_last = (ok && !*abort_flag && m0 < p.M) ? take_ticket(&p.otickets[tile], epoch, p.ksplit) : 0;
                named_sync_epilogue();
                if (s_last) {
                    // four float4 per thread at a time, every split's loads issued together
                    constexpr int n4 = BN / 4;
                    const size_t plane = (size_t)p.M * p.N;
                    for (int idx0 = et; idx0 < BM * n4; idx0 += 4 * kEpiThreads) {
                        float4 acc[4];
                        size_t off[4];
                        bool valid[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int idx = idx0 + u * kEpiThreads;
                            const int rr = m0 + idx / n4, c = w.j * BN + (idx % n4) * 4;
                            valid[u] = idx < BM * n4 && rr < p.M && c < p.N;
                            off[u] = valid[u] ? (size_t)rr * p.N + c : 0;
                            acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                        for (int k = 0; k < p.ksplit; ++k) {
                            float4 v[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                v[u] = valid[u] ? __ldcg(reinterpret_cast<const float4*>(p.ypart + k * plane + off[u]))
                                                : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                acc[u].x += v[u].x;
                                acc[u].y += v[u].y;
                                acc[u].z += v[u].z;
                                acc[u].w += v[u].w;
                            }
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            if (!valid[u]) continue;
                            if (p.out_f32) {
                                *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.y) + off[u]) = acc[u];
                            } else {
                                __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[u].x, acc[u].y);
                                __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[u].z, acc[u].w);
                                *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.y) + off[u]) =
                                    make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
                            }
                        }
                    }
                }
                named_sync_epilogue();
            }
            if (w.adapter) {
                // publish this CTA's 128 rows of T partial w.j (all four warps take every barrier)
                const int tile = m0 / BM;
                asm volatile("fence.proxy.async.global;" ::: "memory");
                __threadfence();
                named_sync_epilogue();
                if (et == 0 && ok && m0 < p.M && !p.withhold_flags)
                    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(&p.flags[tile * p.splits + w.j]), "l"(epoch)
                                 : "memory");
            }
        }
        if (p.epi_tma && lane == 0) bulk_wait_all();  // this warp's output stores have completed
    }

    tmem_fence_before();
    __syncthreads();
    if constexpr (CG == 2) pair_sync();  // nothing of the pair still reaches this CTA
    if (warp == 1) {
        tmem_fence_after();
        if constexpr (CG == 2)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * p.cb) : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * p.cb) : "memory");
    }
    if (threadIdx.x == 0) {
        if (s_abort) record_device_status(p.status, (uint32_t)UNO_ERR_TIMEOUT);
        retire_epoch(p.header, epoch, s_slot, (int)gridDim.x);
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

// row-major [rows, cols] bf16 matrix (cols a multiple of 64) seen as 64 columns x rows x
// cols / 64 K slabs: a box of 64 columns x box_rows rows x slabs, 128-byte swizzle
uno_status make_tmap3(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int box_rows, int slabs) {
    auto fn = encode_fn();
    if (!fn) return set_error(UNO_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t gdim[3] = {(cuuint64_t)BK, (cuuint64_t)rows, (cuuint64_t)(cols / BK)};
    cuuint64_t gstride[2] = {(cuuint64_t)cols * 2, (cuuint64_t)BK * 2};
    cuuint32_t box[3] = {(cuuint32_t)BK, (cuuint32_t)box_rows, (cuuint32_t)slabs};
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), gdim, gstride, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(UNO_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d)", (int)r);
    return UNO_OK;
}

// row-major [rows, cols] bf16 output, 32 x 32 boxes with 64-byte swizzle (the epilogue's
// staging layout)
uno_status make_tmap_store(CUtensorMap* m, void* ptr, int64_t rows, int64_t cols) {
    auto fn = encode_fn();
    if (!fn) return set_error(UNO_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, gdim, gstride, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(UNO_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", (int)r);
    return UNO_OK;
}


// The launch plan of one call (also sizes the workspace).
struct Plan {
    int CG, BN, rb, cb, m_tiles, m_units, n_tiles, kt0, kt1, splits, per, n_adapter, n_items, stages, ws, tws, t3d;
    int ksplit, kper;
    int epi_tma;
    uint32_t b_bytes, epi_off;
    size_t smem;
    // workspace offsets
    size_t header, flags, t, ypart, otickets, x, w0, a, b, trace, total;
};

int num_sms_cached();

Plan make_plan(int64_t M, int64_t d_in, int64_t d_out, int64_t rank, uno_dtype dtype) {
    Plan P{};
    P.m_tiles = (int)((M + BM - 1) / BM);
    // The CTA-pair form (256 x 256 tiles, one MMA stream over two SMs, each loading half of
    // B: a third less operand traffic per FLOP) when there are 40 or more of its tiles;
    // otherwise single-CTA 128 x BN tiles. With two K slabs per load the pair form measured
    // 12-18% faster on the Qwen3-8B q/o/gate/up/down and the looped-3B gate/up/down
    // projections (64 pair tiles or more), 11% faster on the looped-3B gate/up at M = 256
    // (43 pair tiles), and slower on the narrow k/v ones, on q/k/v/o/down at M = 256 (8 to
    // 16 pair tiles) and on Qwen3-8B k and v as one call (32 pair tiles: 42.0 against 39.7 us). Narrower pair tiles (UNO_LORA_BN=64 or 128 with UNO_LORA_CG=2) measured
    // slower than single CTAs on every narrow projection (Qwen3-8B k: 37.7 against 31.6 us).
    // UNO_LORA_CG=1 or 2 fixes the form.
    const bool pair_ok = M >= 2 * BM && d_out % 64 == 0;
    const int64_t pair_tiles = d_out % 256 == 0 ? ((M + 2 * BM - 1) / (2 * BM)) * (d_out / 256) : 0;
    P.CG = pair_ok && pair_tiles >= 40 ? 2 : 1;
    if (const char* e = getenv("UNO_LORA_CG")) {
        const int c = atoi(e);
        if (c == 1 || (c == 2 && pair_ok)) P.CG = c;
    }
    P.m_units = (int)((M + (int64_t)BM * P.CG - 1) / ((int64_t)BM * P.CG));
    if (P.CG == 2) {
        P.BN = d_out % 256 == 0 ? 256 : d_out % 128 == 0 ? 128 : 64;
        // UNO_LORA_BN (64, 128 or 256, dividing d_out) fixes the pair tile width, for measurements
        if (const char* e = getenv("UNO_LORA_BN")) {
            const int bn = atoi(e);
            if ((bn == 64 || bn == 128 || bn == 256) && d_out % bn == 0) P.BN = bn;
        }
    } else {
        // A K step takes about as long at every tile width (its operand loads set the pace),
        // so the width is the one with the fewest waves of items over the SMs, the wider on a
        // tie (ranked by waves x (1 + BN / 1024)); two adapter items per row tile count too.
        const int sms = num_sms_cached();
        double best = 0.0;
        for (int bn = 256; bn >= 64; bn >>= 1) {
            const int64_t items = (int64_t)P.m_tiles * ((d_out + bn - 1) / bn + 2);
            const double cost = (double)((items + sms - 1) / sms) * (1.0 + bn / 1024.0);
            if (bn == 256 || cost < best) {
                best = cost;
                P.BN = bn;
            }
        }
        // UNO_LORA_BN (64, 128 or 256) fixes the tile width, for measurements
        if (const char* e = getenv("UNO_LORA_BN")) {
            const int bn = atoi(e);
            if (bn == 64 || bn == 128 || bn == 256) P.BN = bn;
        }
    }
    P.n_tiles = (int)((d_out + P.BN - 1) / P.BN);
    const int rq = 16 * P.CG;  // each CTA of a pair holds rb / 2 rows of A: a multiple of 16
    P.rb = (int)((rank + rq - 1) / rq * rq);
    const int w = P.BN > P.rb ? P.BN : P.rb;  // N of the widest MMA
    P.cb = 32;
    while (P.cb < w) P.cb <<= 1;
    // Main K steps of WS = 2 slabs of 64 (one 3-D TMA box per operand): a stage lands about
    // every thousand SM clocks whatever its bytes (a per-load cost, measured with
    // UNO_LORA_TRACE at 24 to 48 KB per stage), so two slabs per load nearly halve the count
    // of loads. UNO_LORA_WIDE=0 keeps one slab per step.
    P.ws = (d_in / BK) % 2 == 0 ? 2 : 1;
    if (const char* e = getenv("UNO_LORA_WIDE"))
        if (atoi(e) == 0) P.ws = 1;
    P.kt0 = (int)(d_in / BK) / P.ws;
    // (T, B) steps: two slabs when r is a multiple of 128 (and main steps take two)
    P.t3d = rank % BK == 0;
    P.tws = (P.t3d && P.ws == 2 && (rank / BK) % 2 == 0) ? 2 : 1;
    P.kt1 = (int)((rank + BK - 1) / BK) / P.tws;
    // The adapter product X A^T of a row unit is split over K into `splits` items, each of
    // which writes its own bf16 partial of T; the output tiles run the (T, B) K tiles once
    // per partial, so no partial is ever summed on its own. Two partials measured fastest
    // on every Qwen3-8B and looped-3B projection (an adapter item streams the unit's rows of
    // X and all of A through one SM; halving that keeps it off the output tiles' critical
    // path, while more partials add (T, B) K tiles to every output tile, or a wave of items).
    // UNO_LORA_SPLITS=n fixes it.
    int splits = P.kt0 >= 2 ? 2 : 1;
    if (const char* e = getenv("UNO_LORA_SPLITS")) splits = atoi(e);
    splits = splits < 1 ? 1 : (splits > P.kt0 ? P.kt0 : splits);
    P.per = (P.kt0 + splits - 1) / splits;
    P.splits = (P.kt0 + P.per - 1) / P.per;
    P.n_adapter = P.m_units * P.splits;
    // Output tiles split over K (UNO_LORA_KSPLIT=n, single-CTA tiles only): each split stores
    // an fp32 partial and the split that finishes a tile last sums them. Meant for small M,
    // where few tiles leave SMs idle; on the looped-3B shapes at M = 256 it measured slower
    // (the summing of the partials costs more than the shorter K loops save), so it is off
    // by default.
    int ks = 1;
    if (const char* e = getenv("UNO_LORA_KSPLIT"))
        if (P.CG == 1) ks = atoi(e);
    ks = ks < 1 ? 1 : (ks > P.kt0 ? P.kt0 : ks);
    P.kper = (P.kt0 + ks - 1) / ks;
    P.ksplit = (P.kt0 + P.kper - 1) / P.kper;  // every split has K tiles of (X, W0); the last also (T, B)
    P.n_items = P.n_adapter + P.m_units * P.n_tiles * P.ksplit;
    P.b_bytes = (uint32_t)(w / P.CG) * 128u;
    // bf16 output tiles of single CTAs leave through 16 KB of shared-memory staging boxes and
    // TMA stores (measured 2-5 % faster than per-lane row stores on the Qwen3-8B and looped-3B
    // shapes; on CTA pairs the two measured the same, within 0.5 %, so pairs keep the row
    // stores); UNO_LORA_EPI=rows selects the row stores, which fp32 outputs and split K use
    P.epi_tma = dtype == UNO_BF16 && P.ksplit == 1 && P.CG == 1;
    if (const char* e = getenv("UNO_LORA_EPI"))
        if (strcmp(e, "rows") == 0) P.epi_tma = 0;
    const uint32_t epi_bytes = P.epi_tma ? 4u * 4096u : 0u;
    P.stages = (int)((kSmemBudget - 1024 - epi_bytes) / ((uint32_t)P.ws * (A_BYTES + P.b_bytes)));
    if (P.stages > kMaxStages) P.stages = kMaxStages;
    // UNO_LORA_STAGES=n (2 up to what fits) shortens the ring, for measurements
    if (const char* e = getenv("UNO_LORA_STAGES")) {
        const int st = atoi(e);
        if (st >= 2 && st < P.stages) P.stages = st;
    }
    P.epi_off = (uint32_t)align_up((size_t)P.stages * P.ws * (A_BYTES + P.b_bytes), 1024);
    P.smem = (size_t)P.epi_off + epi_bytes + 1024;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    P.header = take(sizeof(unsigned long long) * 5);
    P.flags = take((size_t)P.m_tiles * P.splits * 8);
    P.t = take((size_t)P.splits * M * rank * 2);
    P.ypart = P.ksplit > 1 ? take((size_t)P.ksplit * M * d_out * 4) : 0;
    P.otickets = P.ksplit > 1 ? take((size_t)P.m_tiles * P.n_tiles * 8) : 0;
    if (dtype == UNO_F32) {
        P.x = take((size_t)M * d_in * 2);
        P.w0 = take((size_t)d_out * d_in * 2);
        P.a = take((size_t)rank * d_in * 2);
        P.b = take((size_t)d_out * rank * 2);
    }
    P.trace = getenv("UNO_LORA_TRACE") ? take((size_t)3 * 6 * 512 * 8) : 0;
    P.total = off;
    return P;
}

// A fresh host tag per call (48 bits, never 0), starting from a time-derived value; the
// kernel takes the larger of it and the workspace header's stored epoch (read_epoch).
unsigned long long next_epoch() {
    static std::atomic<unsigned long long> counter{
        (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() * 2654435761ull};
    unsigned long long e;
    do {
        e = counter.fetch_add(1) & 0xFFFFFFFFFFFFull;
    } while (e == 0);
    return e;
}

int num_sms_cached() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 1;
    }
    return n;
}

template <int BN, int CG>
uno_status launch_t(const CUtensorMap (&maps)[6], Params& p, const Plan& P, cudaStream_t stream) {
    static bool attr = false;
    if (!attr) {
        uno_status s = check_cuda(cudaFuncSetAttribute(lora_gemm_kernel<BN, CG>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)(kSmemBudget + 1024)),
                                  "cudaFuncSetAttribute(gated lora)");
        if (s != UNO_OK) return s;
        attr = true;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attrs[2];
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = stream;
    cfg.attrs = attrs;
    int n_attr = 0;
    attrs[n_attr].id = cudaLaunchAttributeClusterDimension;
    attrs[n_attr].val.clusterDim.x = CG;
    attrs[n_attr].val.clusterDim.y = 1;
    attrs[n_attr].val.clusterDim.z = 1;
    ++n_attr;
    cfg.numAttrs = n_attr;
    // resident units (CTAs or CTA pairs): an output tile may wait for its row unit's T
    // (the occupancy query costs tens of microseconds of host time: cached per device and
    // shared-memory size)
    int resident = 0;
    {
        static std::mutex mu;
        static std::map<std::pair<int, size_t>, int> cache;
        int dev = 0;
        cudaGetDevice(&dev);
        const auto key = std::make_pair(dev, (size_t)P.smem);
        std::lock_guard<std::mutex> lock(mu);
        const auto found = cache.find(key);
        if (found != cache.end()) {
            resident = found->second;
        } else {
            cudaLaunchConfig_t q = cfg;
            q.gridDim = dim3(CG);
            q.numAttrs = 1;  // the cluster shape alone
            uno_status s = check_cuda(cudaOccupancyMaxActiveClusters(&resident, lora_gemm_kernel<BN, CG>, &q),
                                      "cudaOccupancyMaxActiveClusters(gated lora)");
            if (s != UNO_OK) return s;
            cache[key] = resident;
        }
    }
    if (resident < 1) return set_error(UNO_ERR_CUDA, "gated lora kernel does not fit on the GPU");
    const int units = p.n_items < resident ? p.n_items : resident;
    cfg.gridDim = dim3((unsigned)(units * CG));
    // Ask for a cooperative launch (every CTA resident, as the waits on T assume); where the
    // runtime does not take it together with clusters, the grid is sized to what is
    // resident at once, which an otherwise idle GPU runs in full. UNO_LORA_COOP=0 leaves the
    // attribute out (Nsight Compute runs a cooperative launch with clusters as single CTAs).
    const char* coop_env = getenv("UNO_LORA_COOP");
    const bool coop = !(coop_env && coop_env[0] == '0');
    attrs[n_attr].id = cudaLaunchAttributeCooperative;
    attrs[n_attr].val.cooperative = 1;
    cfg.numAttrs = coop ? n_attr + 1 : n_attr;
    cudaError_t e = cudaLaunchKernelEx(&cfg, lora_gemm_kernel<BN, CG>, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], p);
    if (e != cudaSuccess && coop) {
        cudaGetLastError();
        cfg.numAttrs = n_attr;
        e = cudaLaunchKernelEx(&cfg, lora_gemm_kernel<BN, CG>, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], p);
    }
    return check_cuda(e, "launch(gated lora)");
}

}  // namespace glora

size_t gated_lora_workspace_bytes(int64_t M, int64_t d_in, int64_t d_out, int64_t rank, uno_dtype dtype) {
    return glora::make_plan(M, d_in, d_out, rank, dtype).total;
}

uno_status gated_lora_launch(const GatedLoraArgs& g, void* workspace, cudaStream_t stream) {
    using namespace glora;
    const Plan P = make_plan(g.M, g.d_in, g.d_out, g.rank, g.dtype);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const void *x = g.x, *w0 = g.w0, *a = g.a, *b = g.b;
    uno_status s;
    if (g.dtype == UNO_F32) {  // round the fp32 operands to bf16 once
        struct { const void* src; size_t off; int64_t n; } cv[4] = {
            {g.x, P.x, g.M * g.d_in}, {g.w0, P.w0, g.d_out * g.d_in}, {g.a, P.a, g.rank * g.d_in}, {g.b, P.b, g.d_out * g.rank}};
        for (auto& c : cv) {
            f32_to_bf16_kernel<<<592, 256, 0, stream>>>(static_cast<const float*>(c.src),
                                                      reinterpret_cast<__nv_bfloat16*>(ws + c.off), c.n);
            if ((s = check_cuda(cudaGetLastError(), "launch(f32->bf16)")) != UNO_OK) return s;
        }
        x = ws + P.x;
        w0 = ws + P.w0;
        a = ws + P.a;
        b = ws + P.b;
    }
    const int M = (int)g.M, din = (int)g.d_in, dout = (int)g.d_out, r = (int)g.rank;
    __nv_bfloat16* t = reinterpret_cast<__nv_bfloat16*>(ws + P.t);
    CUtensorMap maps[6];
    const int cg = P.CG;
    // X, W0, A: boxes of P.ws K slabs (each CTA of a pair loads half of the B rows)
    if ((s = make_tmap3(&maps[0], x, M, din, BM, P.ws)) != UNO_OK) return s;
    if ((s = make_tmap3(&maps[1], w0, dout, din, P.BN / cg, P.ws)) != UNO_OK) return s;
    if ((s = make_tmap3(&maps[2], a, r, din, P.rb / cg, P.ws)) != UNO_OK) return s;
    if (P.t3d) {  // T partials, B: boxes of P.tws K slabs
        if ((s = make_tmap3(&maps[3], t, (int64_t)P.splits * M, r, BM, P.tws)) != UNO_OK) return s;
        if ((s = make_tmap3(&maps[4], b, dout, r, P.BN / cg, P.tws)) != UNO_OK) return s;
    } else {
        if ((s = make_tmap(&maps[3], t, (int64_t)P.splits * M, r, BM)) != UNO_OK) return s;  // T partials
        if ((s = make_tmap(&maps[4], b, dout, r, P.BN / cg)) != UNO_OK) return s;      // B
    }
    if (P.epi_tma) {
        if ((s = make_tmap_store(&maps[5], g.y, M, dout)) != UNO_OK) return s;     // Y (stores)
    } else {
        maps[5] = maps[0];  // not read
    }
    Params p{};
    p.M = M;
    p.N = dout;
    p.r = r;
    p.kt0 = P.kt0;
    p.kt1 = P.kt1;
    p.m_tiles = P.m_tiles;
    p.m_units = P.m_units;
    p.splits = P.splits;
    p.per = P.per;
    p.n_adapter = P.n_adapter;
    p.n_items = P.n_items;
    p.n_tiles = P.n_tiles;
    p.ksplit = P.ksplit;
    p.kper = P.kper;
    p.ypart = P.ksplit > 1 ? reinterpret_cast<float*>(ws + P.ypart) : nullptr;
    p.otickets = P.ksplit > 1 ? reinterpret_cast<unsigned long long*>(ws + P.otickets) : nullptr;
    p.rb = P.rb;
    p.stages = P.stages;
    p.b_bytes = P.b_bytes;
    p.ws = P.ws;
    p.tws = P.tws;
    p.t3d = P.t3d;
    p.cb = (uint32_t)P.cb;
    p.y = g.y;
    p.out_f32 = g.dtype == UNO_F32;
    p.t = t;
    p.gate = g.gate;
    p.scale = g.scale;
    p.flags = reinterpret_cast<unsigned long long*>(ws + P.flags);
    p.header = reinterpret_cast<unsigned long long*>(ws + P.header);
    p.host_tag = next_epoch();
    // UNO_LORA_TEST_WITHHOLD_FLAGS=1 (tests of the failure path only): the adapter items keep
    // T to themselves and the output tiles' waits for it give up after a few thousand polls;
    // the call must then end with UNO_ERR_TIMEOUT in the device status word
    p.epi_tma = P.epi_tma;
    p.epi_off = P.epi_off;
    p.withhold_flags = 0;
    p.flag_polls = kFlagPolls;
    if (const char* e = getenv("UNO_LORA_TEST_WITHHOLD_FLAGS"))
        if (atoi(e) == 1) {
            p.withhold_flags = 1;
            p.flag_polls = 4096;
        }
    p.status = device_status_ptr();
    p.trace = getenv("UNO_LORA_TRACE") ? reinterpret_cast<long long*>(ws + P.trace) : nullptr;
    if (P.CG == 2) {
        switch (P.BN) {
            case 64: return launch_t<64, 2>(maps, p, P, stream);
            case 128: return launch_t<128, 2>(maps, p, P, stream);
            case 256: return launch_t<256, 2>(maps, p, P, stream);
        }
        return set_error(UNO_ERR_UNSUPPORTED, "pair tile width %d", P.BN);
    }
    switch (P.BN) {
        case 64: return launch_t<64, 1>(maps, p, P, stream);
        case 128: return launch_t<128, 1>(maps, p, P, stream);
        case 256: return launch_t<256, 1>(maps, p, P, stream);
    }
    return set_error(UNO_ERR_UNSUPPORTED, "tile width %d", P.BN);
}

}  // namespace uno
