// Byte-for-byte grid comparison: the check that synchronized sampler weights, scales and kernel
// layouts equal the learner's quantization ("End-to-End MXFP8 Reinforcement Learning on
// Blackwell", abstract and Table 11, byte comparison; Table 13 lists the violations it must see).
//
// Result on the device: the number of differing bytes and the index of the first one (-1 if
// none). One small launch resets the two result words, then a streaming kernel reads both
// buffers once (16-byte loads, 4 in flight per buffer per thread), reduces per block and merges
// with one atomicAdd and one atomicMin per block.
#pragma once
#include <cstdint>

namespace mx {

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

__global__ void grid_equal_reset_kernel(unsigned long long* count, long long* first) {
    *count = 0ull;
    *first = -1ll;   // all ones: the largest value for the unsigned atomicMin below
}

constexpr int kGeThreads = 256;
constexpr int kGeUnroll = 4;

__global__ void __launch_bounds__(kGeThreads) grid_equal_kernel(const uint8_t* __restrict__ a,
                                                                const uint8_t* __restrict__ b, int64_t nbytes,
                                                                int vector_ok, unsigned long long* count,
                                                                long long* first) {
    unsigned long long cnt = 0;
    unsigned long long first_local = ~0ull;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t tail_start = 0;
    if (vector_ok) {
        const int64_t nvec = nbytes / 16;
        const uint4* va = reinterpret_cast<const uint4*>(a);
        const uint4* vb = reinterpret_cast<const uint4*>(b);
        // Main loop: kGeUnroll chunks per thread per iteration, strided by the grid.
        int64_t i = tid;
        for (; i + (kGeUnroll - 1) * nthreads < nvec; i += kGeUnroll * nthreads) {
            uint4 xa[kGeUnroll], xb[kGeUnroll];
#pragma unroll
            for (int u = 0; u < kGeUnroll; ++u) {
                xa[u] = ld_stream_v4_ge(va + i + u * nthreads);
                xb[u] = ld_stream_v4_ge(vb + i + u * nthreads);
            }
#pragma unroll
            for (int u = 0; u < kGeUnroll; ++u) {
                const uint32_t d0 = nonzero_bytes(xa[u].x ^ xb[u].x), d1 = nonzero_bytes(xa[u].y ^ xb[u].y);
                const uint32_t d2 = nonzero_bytes(xa[u].z ^ xb[u].z), d3 = nonzero_bytes(xa[u].w ^ xb[u].w);
                const uint32_t n = __popc(d0) + __popc(d1) + __popc(d2) + __popc(d3);
                if (n) {
                    cnt += n;
                    const uint64_t mask = static_cast<uint64_t>(d0) | (static_cast<uint64_t>(d1) << 32);
                    const uint64_t mask2 = static_cast<uint64_t>(d2) | (static_cast<uint64_t>(d3) << 32);
                    const int off = mask ? (__ffsll(static_cast<long long>(mask)) - 1) / 8
                                         : 8 + (__ffsll(static_cast<long long>(mask2)) - 1) / 8;
                    const unsigned long long idx = static_cast<unsigned long long>((i + u * nthreads) * 16 + off);
                    first_local = idx < first_local ? idx : first_local;
                }
            }
        }
        for (; i < nvec; i += nthreads) {
            const uint4 xa = ld_stream_v4_ge(va + i), xb = ld_stream_v4_ge(vb + i);
            const uint32_t d0 = nonzero_bytes(xa.x ^ xb.x), d1 = nonzero_bytes(xa.y ^ xb.y);
            const uint32_t d2 = nonzero_bytes(xa.z ^ xb.z), d3 = nonzero_bytes(xa.w ^ xb.w);
            const uint32_t n = __popc(d0) + __popc(d1) + __popc(d2) + __popc(d3);
            if (n) {
                cnt += n;
                const uint64_t mask = static_cast<uint64_t>(d0) | (static_cast<uint64_t>(d1) << 32);
                const uint64_t mask2 = static_cast<uint64_t>(d2) | (static_cast<uint64_t>(d3) << 32);
                const int off = mask ? (__ffsll(static_cast<long long>(mask)) - 1) / 8
                                     : 8 + (__ffsll(static_cast<long long>(mask2)) - 1) / 8;
                const unsigned long long idx = static_cast<unsigned long long>(i * 16 + off);
                first_local = idx < first_local ? idx : first_local;
            }
        }
        tail_start = nvec * 16;
    }
    // Bytes not covered by 16-byte chunks (all of them when the buffers are not 16-byte aligned).
    for (int64_t j = tail_start + tid; j < nbytes; j += nthreads) {
        if (a[j] != b[j]) {
            ++cnt;
            const unsigned long long idx = static_cast<unsigned long long>(j);
            first_local = idx < first_local ? idx : first_local;
        }
    }

    // Block reduction.
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, o);
        const unsigned long long f = __shfl_xor_sync(0xFFFFFFFFu, first_local, o);
        first_local = f < first_local ? f : first_local;
    }
    __shared__ unsigned long long s_cnt[kGeThreads / 32], s_first[kGeThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        s_cnt[warp] = cnt;
        s_first[warp] = first_local;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long c = 0, f = ~0ull;
        for (int w = 0; w < kGeThreads / 32; ++w) {
            c += s_cnt[w];
            f = s_first[w] < f ? s_first[w] : f;
        }
        if (c) {
            atomicAdd(count, c);
            atomicMin(reinterpret_cast<unsigned long long*>(first), f);
        }
    }
}

}  // namespace mx
