// select.cuh — exact selection of the k largest 64-bit packed candidates (radix select
// over 8-bit digits, most significant first) at warp and CTA scope, plus a CTA bitonic
// sort. Candidates are distinct (the low 32 bits encode the token id), so "the k largest"
// is unique.
#pragma once

#include "common.cuh"

namespace uno {

// Find the digit bin in which the k_rem-th largest entry lies. `c` holds, for this lane,
// the counts of bins 255-8*lane .. 255-8*lane-7 (descending). Returns (bin, count of
// entries in higher bins, count in the bin) in all lanes.
__device__ __forceinline__ void warp_find_bin(const uint32_t* hist, uint32_t k_rem, int lane,
                                              int& bin, uint32_t& above, uint32_t& cnt) {
    uint32_t c[8];
    uint32_t s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - 8 * lane - j];
        s += c[j];
    }
    uint32_t incl = warp_inclusive_scan(s, lane);
    uint32_t excl = incl - s;
    bool mine = excl < k_rem && k_rem <= incl;
    unsigned ball = __ballot_sync(kFullMask, mine);
    int src = __ffs(ball) - 1;
    int b = 0;
    uint32_t a = excl, n = 0;
    if (mine) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (a + c[j] >= k_rem) {
                b = 255 - 8 * lane - j;
                n = c[j];
                break;
            }
            a += c[j];
        }
    }
    bin = __shfl_sync(kFullMask, b, src);
    above = __shfl_sync(kFullMask, a, src);
    cnt = __shfl_sync(kFullMask, n, src);
}

// Warp scope: returns T such that exactly k of buf[0..n) are >= T (1 <= k <= n).
// `hist` is 256 words of this warp's shared memory.
static __device__ __noinline__ uint64_t warp_select(const uint64_t* buf, int n, int k, uint32_t* hist, int lane) {
    uint64_t prefix = 0;
    uint32_t k_rem = (uint32_t)k;
    for (int shift = 56; shift >= 0; shift -= 8) {
        const uint64_t hi_mask = shift == 56 ? 0ull : (~0ull << (shift + 8));
#pragma unroll
        for (int j = 0; j < 8; ++j) hist[lane * 8 + j] = 0u;
        __syncwarp();
        for (int i = lane; i < n; i += 32) {
            uint64_t x = buf[i];
            if ((x & hi_mask) == prefix) atomicAdd(&hist[(uint32_t)(x >> shift) & 0xFFu], 1u);
        }
        __syncwarp();
        int bin;
        uint32_t above, cnt;
        warp_find_bin(hist, k_rem, lane, bin, above, cnt);
        __syncwarp();
        prefix |= (uint64_t)bin << shift;
        k_rem -= above;
        if (cnt == k_rem) return prefix;
    }
    return prefix;
}

// Warp scope: keep the entries >= T in place (order not kept); returns the new count.
// *min_kept = smallest kept entry (~0 if none).
__device__ __forceinline__ int warp_compact(uint64_t* buf, int n, uint64_t T, int lane, uint64_t* min_kept) {
    int out = 0;
    uint64_t mn = ~0ull;
    for (int base = 0; base < n; base += 32) {
        int i = base + lane;
        uint64_t x = i < n ? buf[i] : 0ull;
        bool keep = i < n && x >= T;
        unsigned ball = __ballot_sync(kFullMask, keep);
        __syncwarp();
        if (keep) {
            buf[out + __popc(ball & ((1u << lane) - 1u))] = x;
            mn = x < mn ? x : mn;
        }
        out += __popc(ball);
        __syncwarp();
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        uint64_t t = __shfl_xor_sync(kFullMask, mn, o);
        mn = t < mn ? t : mn;
    }
    *min_kept = mn;
    return out;
}

// CTA scope (all NT threads call): returns T such that exactly k of v[0..n) are >= T.
// `hist` is 256 words of shared memory; `bc` is 4 words of shared memory.
template <int NT>
static __device__ __noinline__ uint64_t cta_select(const uint64_t* v, int n, int k, uint32_t* hist, uint64_t* bc) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint64_t prefix = 0;
    uint32_t k_rem = (uint32_t)k;
    for (int shift = 56; shift >= 0; shift -= 8) {
        const uint64_t hi_mask = shift == 56 ? 0ull : (~0ull << (shift + 8));
        for (int j = tid; j < 256; j += NT) hist[j] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += NT) {
            uint64_t x = v[i];
            if ((x & hi_mask) == prefix) atomicAdd(&hist[(uint32_t)(x >> shift) & 0xFFu], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            int bin;
            uint32_t above, cnt;
            warp_find_bin(hist, k_rem, lane, bin, above, cnt);
            if (lane == 0) {
                bc[0] = prefix | ((uint64_t)bin << shift);
                bc[1] = k_rem - above;
                bc[2] = (cnt == k_rem - above) ? 1ull : 0ull;
            }
        }
        __syncthreads();
        prefix = bc[0];
        k_rem = (uint32_t)bc[1];
        bool done = bc[2] != 0;
        __syncthreads();
        if (done) return prefix;
    }
    return prefix;
}

// CTA bitonic sort of n (power of two, <= 2 * NT * 8) 64-bit keys, descending.
template <int NT>
__device__ void cta_sort_desc(uint64_t* a, int n) {
    const int tid = threadIdx.x;
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = tid; t < n / 2; t += NT) {
                int lo = 2 * t - (t & (stride - 1));
                int hi = lo + stride;
                bool desc = ((lo & size) == 0);
                uint64_t x = a[lo], y = a[hi];
                if ((x < y) == desc) {
                    a[lo] = y;
                    a[hi] = x;
                }
            }
            __syncthreads();
        }
    }
}

}  // namespace uno

namespace uno {

// Warp bitonic sort of n (power of two) 64-bit keys in shared memory, descending.
__device__ __forceinline__ void warp_sort_desc(uint64_t* a, int n, int lane) {
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = lane; t < n / 2; t += 32) {
                int lo = 2 * t - (t & (stride - 1));
                int hi = lo + stride;
                bool desc = ((lo & size) == 0);
                uint64_t x = a[lo], y = a[hi];
                if ((x < y) == desc) {
                    a[lo] = y;
                    a[hi] = x;
                }
            }
            __syncwarp();
        }
    }
}

}  // namespace uno

namespace uno {

// ------------------------------------------------------------------------------------
// Selection on the value key only, for buffers kept in ascending token-id order.
// Candidates are packed (key32 << 32 | ~id). KEYBITS = 16 for bf16 values (the low 16
// bits of a widened bf16 key are fixed by its sign), 32 for fp32.
// warp_select_key finds the key of the k-th largest entry (tau) and how many entries
// equal to tau belong to the top-k (need); because the buffer is in id order, those are
// the first `need` entries equal to tau, which warp_compact_key keeps (stable).
// ------------------------------------------------------------------------------------
template <int KEYBITS>
__device__ __forceinline__ uint32_t radix_of(uint64_t c) {
    return (uint32_t)(c >> (64 - KEYBITS));
}

template <int KEYBITS>
__device__ __forceinline__ uint32_t key32_of_radix(uint32_t r) {
    if (KEYBITS == 32) return r;
    return (r << 16) | ((r & 0x8000u) ? 0x0000u : 0xFFFFu);
}

template <int KEYBITS>
__device__ __forceinline__ void warp_select_key(const uint64_t* buf, int n, int k, uint32_t* hist, int lane,
                                                uint32_t& tau_radix, int& need) {
    uint32_t prefix = 0;
    uint32_t k_rem = (uint32_t)k;
#pragma unroll 1
    for (int shift = KEYBITS - 8; shift >= 0; shift -= 8) {
        const uint32_t hi_mask = (shift + 8 >= 32) ? 0u : (~0u << (shift + 8));
#pragma unroll
        for (int j = 0; j < 8; ++j) hist[lane * 8 + j] = 0u;
        __syncwarp();
        for (int i = lane; i < n; i += 32) {
            uint32_t x = radix_of<KEYBITS>(buf[i]);
            if ((x & hi_mask) == prefix) atomicAdd(&hist[(x >> shift) & 0xFFu], 1u);
        }
        __syncwarp();
        int bin;
        uint32_t above, cnt;
        warp_find_bin(hist, k_rem, lane, bin, above, cnt);
        __syncwarp();
        prefix |= (uint32_t)bin << shift;
        k_rem -= above;
        (void)cnt;
    }
    tau_radix = prefix;
    need = (int)k_rem;
}

// keep entries with radix > tau, and the first `need` (in buffer order) equal to tau
template <int KEYBITS>
__device__ __forceinline__ int warp_compact_key(uint64_t* buf, int n, uint32_t tau, int need, int lane) {
    int out = 0, ties = 0;
    for (int base = 0; base < n; base += 32) {
        int i = base + lane;
        uint64_t x = i < n ? buf[i] : 0ull;
        uint32_t r = radix_of<KEYBITS>(x);
        bool tie = i < n && r == tau;
        unsigned tball = __ballot_sync(kFullMask, tie);
        bool keep = i < n && (r > tau || (tie && ties + __popc(tball & ((1u << lane) - 1u)) < need));
        unsigned ball = __ballot_sync(kFullMask, keep);
        __syncwarp();
        if (keep) buf[out + __popc(ball & ((1u << lane) - 1u))] = x;
        out += __popc(ball);
        ties += __popc(tball);
        __syncwarp();
    }
    return out;
}

}  // namespace uno
