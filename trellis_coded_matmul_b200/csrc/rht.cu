// rht.cu -- the random-sign Hadamard transforms around the contraction
// (QuIP# page, Fig. 2: incoherence processing with a randomized Hadamard
// transform; QTIP discussion, "Incoherence Processing (W2)").
//
//   input:  x' = H_n diag(s_in) x      (per block of B_n consecutive entries)
//   output: y  = alpha diag(s_out) H_m z
//
// H_B is the normalised Sylvester matrix.  The fast transform applies the
// butterfly (a, b) -> (a + b, a - b) for every stride 1, 2, ..., B/2 (the
// strides commute).  A group of T = B/E threads owns one block, E consecutive
// entries per thread:
//   * strides 1 .. E/2 inside a thread's registers,
//   * strides E .. 16E by warp shuffles (lane bit j <-> stride E*2^j),
//   * the remaining strides (blocks of more than 32E entries) through shared
//     memory, four strides per pass (a thread takes 16 entries base + q*h),
//     with one word of padding per 16 so the passes are free of bank
//     conflicts.
// The 1/sqrt(B) normalisation is applied once, at the end, in fp32.  A CTA
// holds several groups when blocks are small.  Both kernels are launched as
// programmatic dependents: they wait for the previous kernel before touching
// their inputs.  The output kernel also re-zeroes the z entries it consumed,
// so the accumulation buffer is ready for the next forward without a memset.
#include <cuda_fp16.h>

#include "fwht.cuh"
#include "internal.h"
#include "xstep.cuh"

namespace qlk {

struct RhtGeometry {
    int B;        // Hadamard block size
    int per_row;  // Hadamard blocks per batch row (d / B)
    int total;    // batch * per_row
    int groups;   // Hadamard blocks per CTA
    int tpg;      // threads per group (B / E)
};

// E entries per thread (B / E <= 1024 threads).
static RhtGeometry rht_geometry(int d, int B, int batch, int E) {
    RhtGeometry g;
    g.B = B;
    g.per_row = d / B;
    g.total = batch * g.per_row;
    g.tpg = B / E < 1 ? 1 : B / E;
    g.groups = g.tpg >= 256 ? 1 : 256 / g.tpg;
    if (g.groups > g.total) g.groups = g.total;
    return g;
}

// Output layouts of x': row-major [batch][n], or the tensor-core operand
// tiles (64-column K stages of npad rows of 128 bytes, 16-byte chunk c of row
// b stored at chunk c ^ (b % 8)).  (The decode-GEMV's step words come from
// rht_in_block_kernel below.)
enum { kXpRowMajor = 1, kXpUmma = 2, kXpUmmaDup = 3 };

// batches from which the tensor-core operand tiles come from the lean input
// transform (measured on a B200: 1.4 us faster at batch 256, 0.7-1.3 us slower
// at batch 16-64, where the older kernel stays)
constexpr int kLeanInMinBatch = 128;

// The 16-byte chunk holding K indices kk .. kk + 7 (kk % 8 == 0) of row b, in halves.
__device__ __forceinline__ size_t umma_chunk_index(int kk, int b, int npad) {
    const int s = kk >> 6, chunk = ((kk & 63) >> 3) ^ (b & 7);
    return (((size_t)s * npad + b) * 128 + chunk * 16) / 2;
}

// Columns col .. col + 3 (col % 4 == 0) of row b, each value twice along K,
// as one 16-byte store.
__device__ __forceinline__ void store_umma_dup4(__half* out, int col, int b, int npad, __half2 lo, __half2 hi) {
    const __half2 d0 = __half2(__low2half(lo), __low2half(lo));
    const __half2 d1 = __half2(__high2half(lo), __high2half(lo));
    const __half2 d2 = __half2(__low2half(hi), __low2half(hi));
    const __half2 d3 = __half2(__high2half(hi), __high2half(hi));
    *reinterpret_cast<uint4*>(out + umma_chunk_index(2 * col, b, npad)) =
        make_uint4(*reinterpret_cast<const uint32_t*>(&d0), *reinterpret_cast<const uint32_t*>(&d1),
                   *reinterpret_cast<const uint32_t*>(&d2), *reinterpret_cast<const uint32_t*>(&d3));
}

__device__ __forceinline__ size_t umma_tile_index4(int col, int b, int npad) {
    const int s = col >> 6, kin = col & 63;
    const int chunk = (kin >> 3) ^ (b & 7);
    return (((size_t)s * npad + b) * 128 + chunk * 16 + (kin & 7) * 2) / 2;  // in halves
}

// B / E threads for one Hadamard block: up to 1024 threads per CTA for
// E >= 16 (the launch bound keeps those within 64 registers per thread), up
// to 512 for E = 8.
template <int MODE, int E>
__global__ void __launch_bounds__(E == 8 ? 512 : 1024) rht_in_kernel(const __half* __restrict__ x, int batch, int n, RhtGeometry geo,
                              const uint32_t* __restrict__ sin_bits, __half* __restrict__ out, int npad) {
    extern __shared__ float smem[];
    const int B = geo.B;
    const int grp = threadIdx.x / geo.tpg, tid = threadIdx.x % geo.tpg;
    const int item = blockIdx.x * geo.groups + grp;
    const bool active = item < geo.total;
    float* buf = smem + (size_t)grp * (B + B / 16);
    const int b = active ? item / geo.per_row : 0;
    const int col = (active ? (item % geo.per_row) * B : 0) + tid * E;
    // the sign bits are written once at create time: read before the wait
    const uint32_t sw = active ? sin_bits[col >> 5] >> (col & 31) : 0u;  // E <= 32 consecutive sign bits
    grid_dependency_wait();
    float v[E];
    if (active) {
        const __half* xs = x + (size_t)b * n + col;
#pragma unroll
        for (int q = 0; q < E; q += 8) {
            const uint4 raw = *reinterpret_cast<const uint4*>(xs + q);
            const __half* hv = reinterpret_cast<const __half*>(&raw);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float f = __half2float(hv[e]);
                v[q + e] = ((sw >> (q + e)) & 1u) ? -f : f;
            }
        }
    } else {
#pragma unroll
        for (int q = 0; q < E; ++q) v[q] = 0.f;
    }
    fwht_block<E>(v, B, tid, geo.tpg, buf);
    grid_launch_dependents();
    if (!active) return;
    const float scale = rsqrtf((float)B);
#pragma unroll
    for (int q = 0; q < E; q += 4) {
        const __half2 lo = __floats2half2_rn(v[q] * scale, v[q + 1] * scale);
        const __half2 hi = __floats2half2_rn(v[q + 2] * scale, v[q + 3] * scale);
        uint2 w;
        w.x = *reinterpret_cast<const uint32_t*>(&lo);
        w.y = *reinterpret_cast<const uint32_t*>(&hi);
        if (MODE == kXpUmmaDup)
            store_umma_dup4(out, col + q, b, npad, lo, hi);
        else if (MODE == kXpUmma)
            *reinterpret_cast<uint2*>(out + umma_tile_index4(col + q, b, npad)) = w;
        else
            *reinterpret_cast<uint2*>(out + (size_t)b * n + col + q) = w;
    }
}

template <int MODE, int E>
static cudaError_t launch_rht_in_e(const Layer& L, const void* x, int batch, void* xp, int npad, cudaStream_t st) {
    const RhtGeometry geo = rht_geometry(L.n, L.B_n, batch, E);
    const size_t smem = geo.tpg > 32 ? (size_t)geo.groups * (geo.B + geo.B / 16) * sizeof(float) : 0;
    auto kern = rht_in_kernel<MODE, E>;
    cudaError_t e = ensure_smem_limit<rht_in_kernel<MODE, E>>((kMaxHadamard + kMaxHadamard / 16) * 4);
    if (e != cudaSuccess) return e;
    const int grid = (geo.total + geo.groups - 1) / geo.groups;
    return launch_pdl(kern, dim3(grid), dim3(geo.groups * geo.tpg), smem, st, (const __half*)x, batch, L.n, geo,
                      (const uint32_t*)L.sin_bits, (__half*)xp, npad);
}

template <int MODE>
static cudaError_t launch_rht_in(const Layer& L, const void* x, int batch, void* xp, int npad, cudaStream_t st) {
    return L.B_n > 16384 ? launch_rht_in_e<MODE, 32>(L, x, batch, xp, npad, st)
                         : launch_rht_in_e<MODE, 16>(L, x, batch, xp, npad, st);
}

// x' for the decode-GEMV, one CTA per (256-column block j, batch row b).
// With B = B_n = 256 R, H_B = H_R (x) H_256 (Sylvester order: the high index
// bits go to H_R), so the block's 256 outputs are
//     x'[256 j + i] = H_256 w / sqrt(B),  w[t] = sum_a H_R[j mod R][a] u[B hb + 256 a + t]
// (u = s_in * x, hb = the Hadamard block of column 256 j): R signed sums per
// entry and one 256-point transform, so every block is computed by its own
// CTA in parallel instead of one CTA per Hadamard block.
template <int VX>
__global__ void __launch_bounds__(256) rht_in_block_kernel(const __half* __restrict__ x, int n, int B,
                                                          const uint32_t* __restrict__ sin_bits, int batch,
                                                          uint32_t* __restrict__ xstep) {
    __shared__ float w[256];
    __shared__ float buf[256 + 16];
    const int j = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
    const int R = B / 256, jr = j % R;
    const int base = (j / R) * B;  // first column of the Hadamard block
    grid_dependency_wait();
    const __half* xr = x + (size_t)b * n + base + t;
    const uint32_t* sr = sin_bits + ((base + t) >> 5);  // + 8 a: the sign word of column base + 256 a + t
    float acc = 0.f;
    for (int a0 = 0; a0 < R; a0 += 16) {  // R is a power of two: sixteen (or R) loads in flight
        const int na = R - a0 < 16 ? R - a0 : 16;
        float v[16];
        uint32_t sw[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            if (q < na) {
                v[q] = __half2float(__ldg(xr + 256 * (a0 + q)));
                sw[q] = __ldg(sr + 8 * (a0 + q));
            }
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            if (q < na) {
                const uint32_t neg = ((sw[q] >> (t & 31)) ^ (uint32_t)__popc(jr & (a0 + q))) & 1u;
                acc += neg ? -v[q] : v[q];
            }
        }
    }
    w[t] = acc;
    __syncthreads();
    grid_launch_dependents();
    const float scale = rsqrtf((float)B);
    fwht_blocks_smem(
        buf, 256, 256,
        [&](int i, float (&v)[8]) {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = w[i + e];
        },
        [&](int i, const float (&v)[4]) {
            const float o[4] = {v[0] * scale, v[1] * scale, v[2] * scale, v[3] * scale};
            store_xstep4<VX>(xstep, 256 * j + i, b, batch, o);
        });
}

cudaError_t launch_rht_in_xstep(const Layer& L, const void* x, int batch, void* xp, cudaStream_t st) {
    const dim3 grid(L.n / 256, batch);
    return L.V == 1 ? launch_pdl(rht_in_block_kernel<1>, grid, dim3(256), 0, st, (const __half*)x, L.n, L.B_n,
                                 (const uint32_t*)L.sin_bits, batch, (uint32_t*)xp)
                    : launch_pdl(rht_in_block_kernel<2>, grid, dim3(256), 0, st, (const __half*)x, L.n, L.B_n,
                                 (const uint32_t*)L.sin_bits, batch, (uint32_t*)xp);
}

// x' as tensor-core operand tiles with the lean scheme of the output
// transform (T = B / 16 threads per Hadamard block, 256 <= B <= 8192, one CTA
// per (block, batch row)): thread t loads columns t + T q (q < 16) with their
// signs and transforms over q in registers, one shared-memory transpose gives
// it columns 16 t .. 16 t + 15, transformed in registers, then the strides 16
// .. T / 2 by warp shuffles; it writes its 16 fp16 values as four 8-byte
// pieces of the swizzled tiles.
template <bool DUP>
__global__ void __launch_bounds__(512) rht_in_umma_lean_kernel(const __half* __restrict__ x, int n, int B,
                                                              const uint32_t* __restrict__ sin_bits, int npad,
                                                              __half* __restrict__ out) {
    extern __shared__ float buf[];  // B + B / 16 floats
    const int T = B >> 4, t = threadIdx.x;
    const int b = blockIdx.y;
    const int base = blockIdx.x * B;
    uint32_t sw[16];  // the sign word of each column t + T q (written at create time: read before the wait)
#pragma unroll
    for (int q = 0; q < 16; ++q) sw[q] = sin_bits[(base + T * q + t) >> 5];
    grid_dependency_wait();
    float v[16];
    const __half* xr = x + (size_t)b * n + base + t;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const float f = __half2float(xr[T * q]);
        v[q] = ((sw[q] >> ((base + T * q + t) & 31)) & 1u) ? -f : f;
    }
    fwht_regs<16>(v);
#pragma unroll
    for (int q = 0; q < 16; ++q) buf[pad16(T * q + t)] = v[q];
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = buf[pad16(16 * t + j)];
    fwht_regs<16>(v);
    const int lane = t & 31;
    for (int h = 1; h < T / 16; h <<= 1) {  // column stride 16 h
        const bool upper = lane & h;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float o = __shfl_xor_sync(0xffffffffu, v[j], h);
            v[j] = upper ? o - v[j] : v[j] + o;
        }
    }
    grid_launch_dependents();
    const float scale = rsqrtf((float)B);
    const int col0 = base + 16 * t;
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
        const __half2 lo = __floats2half2_rn(v[j] * scale, v[j + 1] * scale);
        const __half2 hi = __floats2half2_rn(v[j + 2] * scale, v[j + 3] * scale);
        if constexpr (DUP)
            store_umma_dup4(out, col0 + j, b, npad, lo, hi);
        else
            *reinterpret_cast<uint2*>(out + umma_tile_index4(col0 + j, b, npad)) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    }
}

static bool lean_in_ok(const Layer& L, int batch) { return L.B_n >= 256 && L.B_n <= 8192 && batch >= kLeanInMinBatch; }

cudaError_t launch_rht_in_umma(const Layer& L, const void* x, int batch, int npad, void* xt, cudaStream_t st,
                               bool dup) {
    if (lean_in_ok(L, batch)) {
        const dim3 grid(L.n / L.B_n, batch);
        const size_t smem = (size_t)(L.B_n + L.B_n / 16) * sizeof(float);
        auto kern = dup ? rht_in_umma_lean_kernel<true> : rht_in_umma_lean_kernel<false>;
        return launch_pdl(kern, grid, dim3(L.B_n / 16), smem, st, (const __half*)x, L.n, L.B_n,
                          (const uint32_t*)L.sin_bits, npad, (__half*)xt);
    }
    return dup ? launch_rht_in<kXpUmmaDup>(L, x, batch, xt, npad, st) : launch_rht_in<kXpUmma>(L, x, batch, xt, npad, st);
}

// Entries per thread of the output transform: B_m may be as small as 16.
template <bool F16, int E>
__global__ void __launch_bounds__(E == 8 ? 512 : 1024) rht_out_kernel(float* __restrict__ z, int batch, int m, RhtGeometry geo,
                               const uint32_t* __restrict__ sout_bits, float alpha, void* __restrict__ y) {
    extern __shared__ float smem[];
    const int B = geo.B;
    const int grp = threadIdx.x / geo.tpg, tid = threadIdx.x % geo.tpg;
    const int item = blockIdx.x * geo.groups + grp;
    const bool active = item < geo.total;
    float* buf = smem + (size_t)grp * (B + B / 16);
    const int b = active ? item / geo.per_row : 0;
    const int row = (active ? (item % geo.per_row) * B : 0) + tid * E;
    // the sign bits are written once at create time: read before the wait
    const uint32_t sw = active ? sout_bits[row >> 5] >> (row & 31) : 0u;
    const float scale = alpha * rsqrtf((float)B);
    grid_dependency_wait();
    float v[E];
    if (active) {
        float* zs = z + (size_t)b * m + row;
#pragma unroll
        for (int q = 0; q < E; q += 4) {
            const float4 t = *reinterpret_cast<const float4*>(zs + q);
            v[q] = t.x;
            v[q + 1] = t.y;
            v[q + 2] = t.z;
            v[q + 3] = t.w;
            *reinterpret_cast<float4*>(zs + q) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    } else {
#pragma unroll
        for (int q = 0; q < E; ++q) v[q] = 0.f;
    }
    fwht_block<E>(v, B, tid, geo.tpg, buf);
    grid_launch_dependents();
    if (!active) return;
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = ((sw >> q) & 1u) ? -v[q] * scale : v[q] * scale;
    if (F16) {
        __half* ys = (__half*)y + (size_t)b * m + row;
#pragma unroll
        for (int q = 0; q < E; q += 4) {
            const __half2 lo = __floats2half2_rn(v[q], v[q + 1]);
            const __half2 hi = __floats2half2_rn(v[q + 2], v[q + 3]);
            uint2 w;
            w.x = *reinterpret_cast<const uint32_t*>(&lo);
            w.y = *reinterpret_cast<const uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(ys + q) = w;
        }
    } else {
        float* ys = (float*)y + (size_t)b * m + row;
#pragma unroll
        for (int q = 0; q < E; q += 4) *reinterpret_cast<float4*>(ys + q) = make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
    }
}

template <bool F16, int E>
static cudaError_t launch_rht_out_e(const Layer& L, float* z, int batch, void* y, cudaStream_t st, float zscale) {
    const RhtGeometry geo = rht_geometry(L.m, L.B_m, batch, E);
    const size_t smem = geo.tpg > 32 ? (size_t)geo.groups * (geo.B + geo.B / 16) * sizeof(float) : 0;
    auto kern = rht_out_kernel<F16, E>;
    cudaError_t e = ensure_smem_limit<rht_out_kernel<F16, E>>((kMaxHadamard + kMaxHadamard / 16) * 4);
    if (e != cudaSuccess) return e;
    const int grid = (geo.total + geo.groups - 1) / geo.groups;
    return launch_pdl(kern, dim3(grid), dim3(geo.groups * geo.tpg), smem, st, z, batch, L.m, geo,
                      (const uint32_t*)L.sout_bits, L.alpha * zscale, y);
}

// The output transform with T = B / 16 threads per Hadamard block (256 <= B
// <= 8192, so T <= 512), one CTA per (block, batch row), 16 entries a thread:
//   1. thread t takes rows t + T q (q < 16) and transforms over q in registers
//      (the strides T, 2T, 4T, 8T);
//   2. one transpose through shared memory (one pad word per 16) gives it rows
//      16 t .. 16 t + 15, transformed in registers (strides 1, 2, 4, 8);
//   3. the strides 16 .. T / 2 pair threads t and t ^ (stride / 16): warp
//      shuffles, as T <= 512 keeps them inside a warp (none for T <= 16).
// SLOTS: z of a row is the sum of the row's tile's segment slots of the
// tensor-core GEMM's workspace (src = ws, [slot][npad][128]; needs every part's
// rows to be whole 128-row tiles, so that row r lies in global tile r / 128);
// else src = z ([batch][m] fp32), re-zeroed after it is read.  All loads of
// a thread are in flight at once (three slots of every entry; further slots,
// for layers with fewer units than the GEMM has CTAs, one by one).
template <bool F16, bool SLOTS>
__global__ void __launch_bounds__(512) rht_out_lean_kernel(float* __restrict__ src, int npad, int m, int B,
                                                           const int* __restrict__ tile_seg,
                                                           const uint32_t* __restrict__ sout_bits, float scale,
                                                           void* __restrict__ y) {
    extern __shared__ float buf[];  // B + B / 16 floats
    const int T = B >> 4, t = threadIdx.x;
    const int b = blockIdx.y;
    const int base = blockIdx.x * B;
    // the sign bits and the segment table are written once at create time: read before the wait
    const uint32_t sw = sout_bits[(base + 16 * t) >> 5] >> ((base + 16 * t) & 31);
    grid_dependency_wait();
    // every load of the 16 entries is issued before any of them is used
    float v[16];
    if constexpr (SLOTS) {
        const size_t stride = (size_t)npad * 128;
        int s0[16], ns[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int row = base + T * q + t;
            s0[q] = tile_seg[row >> 7];
            ns[q] = tile_seg[(row >> 7) + 1] - s0[q];
        }
        float a1[16], a2[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const float* p = src + ((size_t)s0[q] * npad + b) * 128 + ((base + T * q + t) & 127);
            v[q] = __ldcs(p);
            a1[q] = ns[q] > 1 ? __ldcs(p + stride) : 0.f;
            a2[q] = ns[q] > 2 ? __ldcs(p + 2 * stride) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            v[q] += a1[q] + a2[q];
            for (int k = 3; k < ns[q]; ++k)  // tiles of more than three segments (layers with few units)
                v[q] += __ldcs(src + ((size_t)(s0[q] + k) * npad + b) * 128 + ((base + T * q + t) & 127));
        }
    } else {
        float* p = src + (size_t)b * m + base + t;
#pragma unroll
        for (int q = 0; q < 16; ++q) v[q] = p[T * q];
#pragma unroll
        for (int q = 0; q < 16; ++q) p[T * q] = 0.f;
    }
    fwht_regs<16>(v);
#pragma unroll
    for (int q = 0; q < 16; ++q) buf[pad16(T * q + t)] = v[q];
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = buf[pad16(16 * t + j)];
    fwht_regs<16>(v);
    const int lane = t & 31;
    for (int h = 1; h < T / 16; h <<= 1) {  // row stride 16 h (the strides from T on were step 1)
        const bool upper = lane & h;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float o = __shfl_xor_sync(0xffffffffu, v[j], h);
            v[j] = upper ? o - v[j] : v[j] + o;
        }
    }
    grid_launch_dependents();
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = ((sw >> j) & 1u) ? -v[j] * scale : v[j] * scale;
    const size_t o = (size_t)b * m + base + 16 * t;
    if (F16) {
        __half* ys = (__half*)y + o;
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
            const __half2 lo = __floats2half2_rn(v[j], v[j + 1]);
            const __half2 hi = __floats2half2_rn(v[j + 2], v[j + 3]);
            *reinterpret_cast<uint2*>(ys + j) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
        }
    } else {
        float* ys = (float*)y + o;
#pragma unroll
        for (int j = 0; j < 16; j += 4) *reinterpret_cast<float4*>(ys + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    }
}

// The lean kernel covers 256 <= B_m <= 8192 (and, after the GEMM, layers whose
// parts are whole 128-row tiles).
static bool lean_out_ok(const Layer& L) { return L.B_m >= 256 && L.B_m <= 8192; }

static bool tc_tiles_whole(const Layer& L) {
    for (int i = 0; i < L.nparts; ++i)
        if (L.parts[i].rows % 128) return false;
    return true;
}

template <bool F16, bool SLOTS>
static cudaError_t launch_rht_out_lean(const Layer& L, float* src, int npad, int batch, void* y, float scale,
                                       cudaStream_t st) {
    const dim3 grid(L.m / L.B_m, batch);
    const size_t smem = (size_t)(L.B_m + L.B_m / 16) * sizeof(float);
    return launch_pdl(rht_out_lean_kernel<F16, SLOTS>, grid, dim3(L.B_m / 16), smem, st, src, npad, L.m, L.B_m,
                      L.tc_tile_seg, (const uint32_t*)L.sout_bits, scale, y);
}

cudaError_t launch_rht_out(const Layer& L, float* z, int batch, void* y, int y_dtype, cudaStream_t st, float zscale) {
    const bool f16 = y_dtype == QL_F16;
    // measured on a B200: the lean kernel wins when one or two CTAs do the whole
    // transform (batch 1 of a layer with one Hadamard block of rows); with more
    // blocks or batch rows the older kernel's shorter per-thread chains win
    if (lean_out_ok(L) && (long long)batch * (L.m / L.B_m) <= 2) {
        const float scale = L.alpha * zscale * rsqrtf((float)L.B_m);
        return f16 ? launch_rht_out_lean<true, false>(L, z, 0, batch, y, scale, st)
                   : launch_rht_out_lean<false, false>(L, z, 0, batch, y, scale, st);
    }
    // Small batches (a few CTAs, latency-bound): 8 entries per thread up to blocks
    // of 4096 (512 threads), shorter chains per thread.  Large batches (many
    // CTAs, bandwidth-bound): 16, fewer and fuller CTAs.
    if (L.B_m > 16384)
        return f16 ? launch_rht_out_e<true, 32>(L, z, batch, y, st, zscale)
                   : launch_rht_out_e<false, 32>(L, z, batch, y, st, zscale);
    if (L.B_m > 4096 || batch > kGemvMaxBatch)
        return f16 ? launch_rht_out_e<true, 16>(L, z, batch, y, st, zscale)
                   : launch_rht_out_e<false, 16>(L, z, batch, y, st, zscale);
    return f16 ? launch_rht_out_e<true, 8>(L, z, batch, y, st, zscale)
               : launch_rht_out_e<false, 8>(L, z, batch, y, st, zscale);
}

// Where the tensor-core GEMM's partial sums of a layer row live: row r of
// part p (rows row0[p] ..) is row (r - row0[p]) % 128 of the part's tile
// (r - row0[p]) / 128, which is global tile tile0[p] + that.
struct TcRowMap {
    int nparts;
    int row0[kMaxParts];
    int tile0[kMaxParts];
};

// y = alpha s_out (H_m z) with z read as the sum of each tile's segment slots
// of the GEMM's workspace (ws[slot][b][row in tile], npad columns per slot).
// The same groups and butterflies as rht_out_kernel; four rows (one float4 of
// every slot) are looked up at a time: a part's rows come in multiples of 16,
// so four aligned rows never straddle a tile.
template <bool F16, int E>
__global__ void __launch_bounds__(E == 8 ? 512 : 1024) rht_out_tc_kernel(const float* __restrict__ ws, int npad,
                                                                          int m, RhtGeometry geo, TcRowMap map,
                                                                          const int* __restrict__ tile_seg,
                                                                          const uint32_t* __restrict__ sout_bits,
                                                                          float alpha, void* __restrict__ y) {
    extern __shared__ float smem[];
    const int B = geo.B;
    const int grp = threadIdx.x / geo.tpg, tid = threadIdx.x % geo.tpg;
    const int item = blockIdx.x * geo.groups + grp;
    const bool active = item < geo.total;
    float* buf = smem + (size_t)grp * (B + B / 16);
    const int b = active ? item / geo.per_row : 0;
    const int row = (active ? (item % geo.per_row) * B : 0) + tid * E;
    // the sign bits and the segment table are written once at create time: read before the wait
    const uint32_t sw = active ? sout_bits[row >> 5] >> (row & 31) : 0u;
    int off[E / 4], s0[E / 4], s1[E / 4];
#pragma unroll
    for (int q = 0; q < E / 4; ++q) {
        const int r = row + 4 * q;
        int pi = 0;
        while (pi + 1 < map.nparts && r >= map.row0[pi + 1]) ++pi;
        const int rr = r - map.row0[pi];
        const int gt = map.tile0[pi] + (rr >> 7);
        off[q] = b * 128 + (rr & 127);
        s0[q] = active ? tile_seg[gt] : 0;
        s1[q] = active ? tile_seg[gt + 1] : 0;
    }
    const float scale = alpha * rsqrtf((float)B);
    grid_dependency_wait();
    // A tile has one to three segments unless the layer has fewer units than
    // the GEMM has CTAs.  E = 8: the first three slots of every float4 are
    // loaded at once (all loads in flight), further slots one by one; larger E
    // (64 registers a thread) take one slot of every float4 at a time.
    constexpr int kFirst = E == 8 ? 3 : 1;
    const size_t slot_stride = (size_t)npad * 128;
    float v[E];
    float4 t[E / 4][kFirst];
#pragma unroll
    for (int q = 0; q < E / 4; ++q) {
#pragma unroll
        for (int k = 0; k < kFirst; ++k)
            t[q][k] = s0[q] + k < s1[q] ? __ldcs(reinterpret_cast<const float4*>(ws + (s0[q] + k) * slot_stride + off[q]))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int q = 0; q < E / 4; ++q) {
        float4 acc = t[q][0];
#pragma unroll
        for (int k = 1; k < kFirst; ++k) {
            acc.x += t[q][k].x;
            acc.y += t[q][k].y;
            acc.z += t[q][k].z;
            acc.w += t[q][k].w;
        }
        for (int sl = s0[q] + kFirst; sl < s1[q]; ++sl) {
            const float4 u = __ldcs(reinterpret_cast<const float4*>(ws + sl * slot_stride + off[q]));
            acc.x += u.x;
            acc.y += u.y;
            acc.z += u.z;
            acc.w += u.w;
        }
        v[4 * q] = acc.x;
        v[4 * q + 1] = acc.y;
        v[4 * q + 2] = acc.z;
        v[4 * q + 3] = acc.w;
    }
    fwht_block<E>(v, B, tid, geo.tpg, buf);
    grid_launch_dependents();
    if (!active) return;
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = ((sw >> q) & 1u) ? -v[q] * scale : v[q] * scale;
    if (F16) {
        __half* ys = (__half*)y + (size_t)b * m + row;
#pragma unroll
        for (int q = 0; q < E; q += 4) {
            const __half2 lo = __floats2half2_rn(v[q], v[q + 1]);
            const __half2 hi = __floats2half2_rn(v[q + 2], v[q + 3]);
            uint2 w;
            w.x = *reinterpret_cast<const uint32_t*>(&lo);
            w.y = *reinterpret_cast<const uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(ys + q) = w;
        }
    } else {
        float* ys = (float*)y + (size_t)b * m + row;
#pragma unroll
        for (int q = 0; q < E; q += 4) *reinterpret_cast<float4*>(ys + q) = make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
    }
}

static TcRowMap tc_row_map(const Layer& L) {
    TcRowMap map = {};
    map.nparts = L.nparts;
    int tiles = 0;
    for (int i = 0; i < L.nparts; ++i) {
        map.row0[i] = L.parts[i].row0;
        map.tile0[i] = tiles;
        tiles += (L.parts[i].rows + 127) / 128;
    }
    return map;
}

template <bool F16, int E>
static cudaError_t launch_rht_out_tc_e(const Layer& L, const float* ws, int batch, int npad, void* y, cudaStream_t st,
                                       float zscale) {
    const RhtGeometry geo = rht_geometry(L.m, L.B_m, batch, E);
    const size_t smem = geo.tpg > 32 ? (size_t)geo.groups * (geo.B + geo.B / 16) * sizeof(float) : 0;
    cudaError_t e = ensure_smem_limit<rht_out_tc_kernel<F16, E>>((kMaxHadamard + kMaxHadamard / 16) * 4);
    if (e != cudaSuccess) return e;
    const int grid = (geo.total + geo.groups - 1) / geo.groups;
    return launch_pdl(rht_out_tc_kernel<F16, E>, dim3(grid), dim3(geo.groups * geo.tpg), smem, st, ws, npad, L.m, geo,
                      tc_row_map(L), L.tc_tile_seg, (const uint32_t*)L.sout_bits, L.alpha * zscale, y);
}

cudaError_t launch_rht_out_tc(const Layer& L, const float* ws, int batch, int npad, void* y, int y_dtype,
                              cudaStream_t st, float zscale) {
    const bool f16 = y_dtype == QL_F16;
    // measured on a B200: the lean kernel wins at the large batches (many CTAs,
    // throughput-bound: ~107 -> ~30 instructions per output), not at batch 16
    if (lean_out_ok(L) && tc_tiles_whole(L) && batch >= 32) {
        const float scale = L.alpha * zscale * rsqrtf((float)L.B_m);
        float* w = const_cast<float*>(ws);  // only read (SLOTS)
        return f16 ? launch_rht_out_lean<true, true>(L, w, npad, batch, y, scale, st)
                   : launch_rht_out_lean<false, true>(L, w, npad, batch, y, scale, st);
    }
    if (L.B_m > 16384)
        return f16 ? launch_rht_out_tc_e<true, 32>(L, ws, batch, npad, y, st, zscale)
                   : launch_rht_out_tc_e<false, 32>(L, ws, batch, npad, y, st, zscale);
    if (L.B_m > 4096)
        return f16 ? launch_rht_out_tc_e<true, 16>(L, ws, batch, npad, y, st, zscale)
                   : launch_rht_out_tc_e<false, 16>(L, ws, batch, npad, y, st, zscale);
    return f16 ? launch_rht_out_tc_e<true, 8>(L, ws, batch, npad, y, st, zscale)
               : launch_rht_out_tc_e<false, 8>(L, ws, batch, npad, y, st, zscale);
}

template <int MODE>
static cudaError_t prepare_rht_in(const Layer& L) {
    const int limit = (kMaxHadamard + kMaxHadamard / 16) * 4;
    return L.B_n > 16384 ? preload_kernel<rht_in_kernel<MODE, 32>>(limit) : preload_kernel<rht_in_kernel<MODE, 16>>(limit);
}

template <bool F16>
static cudaError_t prepare_rht_out(const Layer& L) {
    const int limit = (kMaxHadamard + kMaxHadamard / 16) * 4;
    if (lean_out_ok(L)) {
        cudaError_t e = preload_kernel<rht_out_lean_kernel<F16, false>>(0);
        if (e == cudaSuccess) e = preload_kernel<rht_out_lean_kernel<F16, true>>(0);
        if (e != cudaSuccess) return e;
    }
    if (L.B_m > 16384) {
        cudaError_t e = preload_kernel<rht_out_kernel<F16, 32>>(limit);
        return e == cudaSuccess ? preload_kernel<rht_out_tc_kernel<F16, 32>>(limit) : e;
    }
    cudaError_t e = preload_kernel<rht_out_kernel<F16, 16>>(limit);
    if (e == cudaSuccess && L.B_m <= 4096) e = preload_kernel<rht_out_kernel<F16, 8>>(limit);
    if (e == cudaSuccess) e = L.B_m > 4096 ? preload_kernel<rht_out_tc_kernel<F16, 16>>(limit)
                                           : preload_kernel<rht_out_tc_kernel<F16, 8>>(limit);
    return e;
}

// The transform kernels launch_rht_in_xstep, launch_rht_in_umma and
// launch_rht_out can pick for this layer.
cudaError_t prepare_rht_kernels(const Layer& L) {
    cudaError_t e = L.V == 1 ? preload_kernel<rht_in_block_kernel<1>>(0) : preload_kernel<rht_in_block_kernel<2>>(0);
    if (e == cudaSuccess) e = prepare_rht_in<kXpUmma>(L);
    if (e == cudaSuccess && L.B_n >= 256 && L.B_n <= 8192) e = preload_kernel<rht_in_umma_lean_kernel<false>>(0);
    if (e == cudaSuccess && L.B_n >= 256 && L.B_n <= 8192) e = preload_kernel<rht_in_umma_lean_kernel<true>>(0);
    if (e == cudaSuccess) e = prepare_rht_in<kXpUmmaDup>(L);
    if (e == cudaSuccess) e = prepare_rht_out<true>(L);
    if (e == cudaSuccess) e = prepare_rht_out<false>(L);
    return e;
}

}  // namespace qlk
