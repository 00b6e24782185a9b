// xstep.cuh -- the x' operand layout of the decode-GEMV, and a blockwise fast
// Walsh-Hadamard transform that all threads of a CTA run over a shared-memory
// buffer.
//
// The decode-GEMV multiplies one 32-bit A word per (weight row, trellis step)
// by one 32-bit B word per (batch row, step) in m16n8k16 MMAs: the two fp16
// halves of a word sit in two consecutive K slots.
//   V = 1: the A word's two halves sum to the step's weight (the "split" form
//          of a code, see gemv.cu), and the B word holds x' of the step's
//          column twice;
//   V = 2: the A word holds the step's two weights, the B word x' of its two
//          columns.
// Lane (g, c) of a warp owns steps [c*64/V, (c+1)*64/V) of every 256-column
// block; its B words for its steps 4*u2 .. 4*u2+3 (MMAs 2*u2 and 2*u2+1) form
// one 16-byte group, and the groups of the four lanes c of one (block, u2,
// batch row) are contiguous:
//     word  (((j * (16/V) + u2) * batch + b) * 4 + c) * 4 + r % 4
// for step r (within the lane's run) of block j, batch row b.  A batch row
// takes n / V words.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "fwht.cuh"

namespace qlk {

__host__ __device__ __forceinline__ size_t xstep_word(int j, int c, int r, int b, int batch, int V) {
    return ((((size_t)j * (16 / V) + (r >> 2)) * batch + b) * 4 + c) * 4 + (r & 3);
}

// The word of column `col` (V = 1), or of the step holding columns col and
// col + 1 (V = 2, col even), of batch row b.
__host__ __device__ __forceinline__ size_t xstep_word_of_col(int col, int b, int batch, int V) {
    const int j = col >> 8, within = col & 255;
    return xstep_word(j, within >> 6, (within & 63) / V, b, batch, V);
}

__device__ __forceinline__ uint32_t half2_bits(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Writes x' of columns col .. col+3 (col % 4 == 0) of batch row b, already
// scaled, as step words: one 16-byte group (V = 1) or two words (V = 2).
template <int V>
__device__ __forceinline__ void store_xstep4(uint32_t* words, int col, int b, int batch, const float (&v)[4]) {
    const size_t w = xstep_word_of_col(col, b, batch, V);
    if constexpr (V == 1) {
        *reinterpret_cast<uint4*>(words + w) =
            make_uint4(half2_bits(v[0], v[0]), half2_bits(v[1], v[1]), half2_bits(v[2], v[2]), half2_bits(v[3], v[3]));
    } else {
        *reinterpret_cast<uint2*>(words + w) = make_uint2(half2_bits(v[0], v[1]), half2_bits(v[2], v[3]));
    }
}

template <int E>
__device__ __forceinline__ void fwht_regs(float (&v)[E]) {
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
}

// The FWHT of every B-entry block of a padded shared buffer of `count`
// entries (count % B == 0, B a power of two >= 8), by all threads of the CTA.
// load8(i, v) supplies entries i .. i+7 (i % 8 == 0); store4(i, v) receives the
// transformed entries i .. i+3.  Strides 1..4 run in registers, the rest in
// radix-16 passes over the buffer with a CTA barrier after each.  Every thread
// of the CTA must call this; the caller synchronises before reusing `buf`.
// U > 1: each thread issues the loads of U chunks before transforming any of
// them (more loads in flight when the source is global memory).
template <int U = 1, typename Load8, typename Store4>
__device__ __forceinline__ void fwht_blocks_smem(float* buf, int count, int B, Load8&& load8, Store4&& store4) {
    const int tid = threadIdx.x, nt = blockDim.x;
    for (int i0 = tid * 8; i0 < count; i0 += nt * 8 * U) {
        float v[U][8];
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (i0 + u * nt * 8 < count) load8(i0 + u * nt * 8, v[u]);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * nt * 8;
            if (i >= count) break;
            fwht_regs<8>(v[u]);
#pragma unroll
            for (int q = 0; q < 8; ++q) buf[pad16(i + q)] = v[u][q];
        }
    }
    __syncthreads();
    int logh = 3;
    const int logb = 31 - __clz(B);
    while (logh < logb) {
        const int rem = logb - logh;
        if (rem >= 4) {
            fwht_pass<4>(buf, count, logh, tid, nt);
            logh += 4;
        } else if (rem == 3) {
            fwht_pass<3>(buf, count, logh, tid, nt);
            logh += 3;
        } else if (rem == 2) {
            fwht_pass<2>(buf, count, logh, tid, nt);
            logh += 2;
        } else {
            fwht_pass<1>(buf, count, logh, tid, nt);
            logh += 1;
        }
        __syncthreads();
    }
    for (int i = tid * 4; i < count; i += nt * 4) {
        float v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = buf[pad16(i + q)];
        store4(i, v);
    }
}

// x' = H_B (s_in * x) / sqrt(B) of `batch` rows of x (fp16 [batch][n],
// 16-byte aligned), per block of B consecutive entries, written as step words
// to `xs` (shared memory, the layout above) by every thread of the CTA.
// Groups of T = B / E threads (a power of two, at most blockDim.x) take one
// block each, E consecutive entries a thread: strides below E in registers,
// then warp shuffles, then `scratch` (floor(blockDim.x / T) * (B + B / 16)
// floats of shared memory) when T > 32.  All threads of the CTA must call
// this; it ends with a CTA barrier.
template <int VX, int E>
__device__ __forceinline__ void xstep_transform_cta(const __half* __restrict__ x, int n, int B,
                                                    const uint32_t* __restrict__ sin_bits, int batch, uint32_t* xs,
                                                    float* scratch) {
    const int T = B / E;
    const int G = blockDim.x / T;
    const int grp = threadIdx.x / T, tid = threadIdx.x % T;
    const bool member = grp < G;
    const int per_row = n / B, items = batch * per_row;
    const float scale = rsqrtf((float)B);
    auto load = [&](int item, float (&v)[E]) {  // entries tid*E .. +E-1 of item, signs applied (0 past the end)
        if (!member || item >= items) {
#pragma unroll
            for (int q = 0; q < E; ++q) v[q] = 0.f;
            return;
        }
        const int b = item / per_row, col = (item % per_row) * B + tid * E;
        const uint32_t sw = sin_bits[col >> 5] >> (col & 31);  // E <= 32 consecutive sign bits
#pragma unroll
        for (int q = 0; q < E; q += 8) {
            const uint4 raw = *reinterpret_cast<const uint4*>(x + (size_t)b * n + col + q);
            const __half* hv = reinterpret_cast<const __half*>(&raw);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float f = __half2float(hv[e]);
                v[q + e] = ((sw >> (q + e)) & 1u) ? -f : f;
            }
        }
    };
    auto store = [&](int item, float (&v)[E]) {
        if (!member || item >= items) return;
        const int b = item / per_row, col = (item % per_row) * B + tid * E;
#pragma unroll
        for (int q = 0; q < E; q += 4) {
            const float o[4] = {v[q] * scale, v[q + 1] * scale, v[q + 2] * scale, v[q + 3] * scale};
            store_xstep4<VX>(xs, col + q, b, batch, o);
        }
    };
    float* buf = scratch + (size_t)(member ? grp : 0) * (B + B / 16);
    for (int i0 = 0; i0 < items; i0 += G) {
        const int item = i0 + grp;
        float v[E];
        load(item, v);
        fwht_block<E>(v, B, tid, T, buf, member && item < items);
        store(item, v);
        if (T > 32) __syncthreads();  // buf is written again by the next round
    }
    __syncthreads();
}

}  // namespace qlk
