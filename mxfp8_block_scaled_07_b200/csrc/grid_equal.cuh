// Byte-for-byte grid comparison: the check that synchronized sampler weights, scales and kernel
// layouts equal the learner's quantization ("End-to-End MXFP8 Reinforcement Learning on
// Blackwell", abstract and Table 11, byte comparison; Table 13 lists the violations it must see).
//
// Result per compared pair, on the device: the number of differing bytes and the index of the
// first one (-1 if none). One small launch resets the result words; the comparison kernel splits
// all pairs into 32 KB work units (one tile space over every pair, so one launch covers a whole
// model's weights, elements and scales), reads both sides once with 16-byte streaming loads (8 in
// flight per side per thread), reduces per warp, and only a warp that saw a difference touches
// the results (one atomicAdd and one atomicMin).
#pragma once
#include <cstdint>

namespace mx {

constexpr int kGeThreads = 256;
constexpr int kGeChunksPerThread = 8;                                    // 16-byte chunks per side
constexpr int64_t kGeUnitBytes = int64_t(kGeThreads) * kGeChunksPerThread * 16;   // 32 KB
constexpr int kGeMaxPairs = 512;       // pairs per launch (kernel parameters < 32 KB)

__device__ __forceinline__ uint4 ld_stream_v4_ge(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Nonzero bytes of x -> 0x01 in that byte.
__device__ __forceinline__ uint32_t nonzero_bytes(uint32_t x) {
    x |= x >> 4;
    x |= x >> 2;
    x |= x >> 1;
    return x & 0x01010101u;
}

struct CmpPair {
    const uint8_t* a;
    const uint8_t* b;
    int64_t nbytes;
    int64_t unit_start;       // first work unit of this pair
    int vec;                  // both sides 16-byte aligned
};

template <int NP>
struct CmpArgs {
    int n;
    int64_t total_units;
    unsigned long long* counts;   // [n]
    long long* firsts;            // [n]
    CmpPair p[NP];
};

__global__ void grid_equal_reset_kernel(unsigned long long* counts, long long* firsts, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        counts[i] = 0ull;
        firsts[i] = -1ll;     // all ones: the largest value for the unsigned atomicMin below
    }
}

template <int NP>
__global__ void __launch_bounds__(kGeThreads) grid_equal_kernel(const __grid_constant__ CmpArgs<NP> g) {
    const int lane = threadIdx.x & 31;
    for (int64_t u = blockIdx.x; u < g.total_units; u += gridDim.x) {
        int pi = 0;
        if constexpr (NP > 1) {
            int lo = 0, hi = g.n - 1;      // largest pair with unit_start <= u
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (g.p[mid].unit_start <= u) lo = mid; else hi = mid - 1;
            }
            pi = lo;
        }
        const CmpPair& P = g.p[pi];
        const int64_t off = (u - P.unit_start) * kGeUnitBytes;
        const int64_t len = min(kGeUnitBytes, P.nbytes - off);
        unsigned long long cnt = 0, first = ~0ull;
        if (P.vec && len == kGeUnitBytes) {
            const uint4* va = reinterpret_cast<const uint4*>(P.a + off);
            const uint4* vb = reinterpret_cast<const uint4*>(P.b + off);
            uint4 xa[kGeChunksPerThread], xb[kGeChunksPerThread];
#pragma unroll
            for (int j = 0; j < kGeChunksPerThread; ++j) {
                xa[j] = ld_stream_v4_ge(va + j * kGeThreads + threadIdx.x);
                xb[j] = ld_stream_v4_ge(vb + j * kGeThreads + threadIdx.x);
            }
#pragma unroll
            for (int j = 0; j < kGeChunksPerThread; ++j) {
                const uint32_t d0 = nonzero_bytes(xa[j].x ^ xb[j].x), d1 = nonzero_bytes(xa[j].y ^ xb[j].y);
                const uint32_t d2 = nonzero_bytes(xa[j].z ^ xb[j].z), d3 = nonzero_bytes(xa[j].w ^ xb[j].w);
                if ((d0 | d1 | d2 | d3) != 0) {
                    cnt += __popc(d0) + __popc(d1) + __popc(d2) + __popc(d3);
                    const uint64_t lo = static_cast<uint64_t>(d0) | (static_cast<uint64_t>(d1) << 32);
                    const uint64_t hi = static_cast<uint64_t>(d2) | (static_cast<uint64_t>(d3) << 32);
                    const int byte = lo ? (__ffsll(static_cast<long long>(lo)) - 1) / 8
                                        : 8 + (__ffsll(static_cast<long long>(hi)) - 1) / 8;
                    const unsigned long long idx =
                        static_cast<unsigned long long>(off + (int64_t(j) * kGeThreads + threadIdx.x) * 16 + byte);
                    first = idx < first ? idx : first;
                }
            }
        } else {
            // Partial last unit, or buffers that are not 16-byte aligned: bytewise.
            for (int64_t k = threadIdx.x; k < len; k += kGeThreads) {
                if (P.a[off + k] != P.b[off + k]) {
                    ++cnt;
                    const unsigned long long idx = static_cast<unsigned long long>(off + k);
                    first = idx < first ? idx : first;
                }
            }
        }
        if (__any_sync(0xFFFFFFFFu, cnt != 0)) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, o);
                const unsigned long long f = __shfl_xor_sync(0xFFFFFFFFu, first, o);
                first = f < first ? f : first;
            }
            if (lane == 0) {
                atomicAdd(&g.counts[pi], cnt);
                atomicMin(reinterpret_cast<unsigned long long*>(&g.firsts[pi]), first);
            }
        }
    }
}

}  // namespace mx
