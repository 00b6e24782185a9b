// fwht.cuh -- fast Walsh-Hadamard transform building blocks (device code).
//
// H_B is the normalised Sylvester matrix; the fast transform applies the
// butterfly (a, b) -> (a + b, a - b) for every stride 1, 2, ..., B/2 (the
// strides commute).  A group of T = B/E threads owns one block, E consecutive
// entries per thread: strides below E in registers, strides E .. 16E by warp
// shuffles, longer strides through padded shared memory four at a time.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

namespace qlk {

__device__ __forceinline__ bool sign_neg(const uint32_t* bits, int i) { return (bits[i >> 5] >> (i & 31)) & 1u; }
__device__ __forceinline__ int pad16(int i) { return i + (i >> 4); }

// One radix-2^LOGR pass at stride h = 2^logh: group gi holds the entries
// base + q h, q < 2^LOGR (h and B are powers of two, so no divisions).
template <int LOGR>
__device__ __forceinline__ void fwht_pass(float* buf, int B, int logh, int tid, int nthreads) {
    constexpr int R = 1 << LOGR;
    const int groups = B >> LOGR;
    const int hmask = (1 << logh) - 1;
    for (int gi = tid; gi < groups; gi += nthreads) {
        const int base = ((gi >> logh) << (logh + LOGR)) + (gi & hmask);
        const int h = 1 << logh;
        float v[R];
#pragma unroll
        for (int q = 0; q < R; ++q) v[q] = buf[pad16(base + q * h)];
#pragma unroll
        for (int s = 0; s < LOGR; ++s) {
#pragma unroll
            for (int q = 0; q < R; ++q) {
                if (!(q & (1 << s))) {
                    const float a = v[q], b = v[q | (1 << s)];
                    v[q] = a + b;
                    v[q | (1 << s)] = a - b;
                }
            }
        }
#pragma unroll
        for (int q = 0; q < R; ++q) buf[pad16(base + q * h)] = v[q];
    }
}

// Strides E.. of the remaining FWHT through shared memory (padded layout) by
// the `nthreads` threads of the group, starting at stride h0; ends with a
// CTA barrier after every pass.
// Threads with active == false touch no memory but take part in every barrier.
__device__ __forceinline__ void fwht_smem_passes(float* buf, int B, int h0, int tid, int nthreads, bool active) {
    int logh = 31 - __clz(h0);
    const int logb = 31 - __clz(B);
    while (logh < logb) {
        const int rem = logb - logh;
        if (rem >= 4) {
            if (active) fwht_pass<4>(buf, B, logh, tid, nthreads);
            logh += 4;
        } else if (rem == 3) {
            if (active) fwht_pass<3>(buf, B, logh, tid, nthreads);
            logh += 3;
        } else if (rem == 2) {
            if (active) fwht_pass<2>(buf, B, logh, tid, nthreads);
            logh += 2;
        } else {
            if (active) fwht_pass<1>(buf, B, logh, tid, nthreads);
            logh += 1;
        }
        __syncthreads();
    }
}

// Full FWHT of a group's block: v holds the thread's E consecutive entries
// (thread tid of T owns entries [tid*E, tid*E + E)); on return v holds the
// same positions of the transformed block.  `buf` is the group's shared
// memory (B + B/16 floats), used only when T > 32.  Every thread of the CTA
// must call this with the same B (it contains CTA barriers when T > 32);
// threads with use_smem == false (spare threads outside any group) skip the
// shared-memory traffic but keep the barriers.
template <int E>
__device__ __forceinline__ void fwht_block(float (&v)[E], int B, int tid, int T, float* buf, bool use_smem = true) {
#pragma unroll
    for (int s = 1; s < E; s <<= 1) {
#pragma unroll
        for (int q = 0; q < E; ++q) {
            if (!(q & s)) {
                const float a = v[q], b = v[q | s];
                v[q] = a + b;
                v[q | s] = a - b;
            }
        }
    }
    const int lanes = T < 32 ? T : 32;
    const int lane = threadIdx.x & 31;
    for (int j = 1; j < lanes; j <<= 1) {
        const bool upper = lane & j;
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const float o = __shfl_xor_sync(0xffffffffu, v[q], j);
            v[q] = upper ? (o - v[q]) : (v[q] + o);
        }
    }
    if (T > 32) {
        if (use_smem) {
#pragma unroll
            for (int q = 0; q < E; ++q) buf[pad16(tid * E + q)] = v[q];
        }
        __syncthreads();
        fwht_smem_passes(buf, B, 32 * E, tid, T, use_smem);
        if (use_smem) {
#pragma unroll
            for (int q = 0; q < E; ++q) v[q] = buf[pad16(tid * E + q)];
        }
    }
}

}  // namespace qlk
