// rht.cu -- the random-sign Hadamard transforms around the contraction
// (QuIP# page, Fig. 2: incoherence processing with a randomized Hadamard
// transform; QTIP discussion, "Incoherence Processing (W2)").
//
//   input:  x' = H_n diag(s_in) x      (per block of B_n consecutive entries)
//   output: y  = alpha diag(s_out) H_m z
//
// H_B is the normalised Sylvester matrix; the in-place butterfly
// (a, b) -> (a + b, a - b) over strides 1, 2, 4, ... produces it in natural
// order, and the 1/sqrt(B) normalisation is applied once at the end.  One CTA
// transforms one Hadamard block of one batch row in shared memory (fp32).
#include <cuda_fp16.h>

#include "internal.h"

namespace qlk {

__device__ __forceinline__ bool sign_neg(const uint32_t* bits, int i) { return (bits[i >> 5] >> (i & 31)) & 1u; }

__device__ __forceinline__ void fwht_smem(float* buf, int B) {
    for (int hs = 1; hs < B; hs <<= 1) {
        for (int t = threadIdx.x; t < (B >> 1); t += blockDim.x) {
            const int i0 = ((t / hs) * 2 * hs) + (t % hs);
            const int i1 = i0 + hs;
            const float a = buf[i0], b = buf[i1];
            buf[i0] = a + b;
            buf[i1] = a - b;
        }
        __syncthreads();
    }
}

// Fragment layout of x' for the decode-GEMV: the 8-byte group
//   frag[((j*16 + u) * batch + b) * 4 + c] = x'[b][256 j + 64 c + 4 u + 0..3]
// is what lane (g = b, c) needs as its B operand for the u-th m16n8k16 MMA of
// block j (see gemv.cu).
__device__ __forceinline__ size_t frag_index(int col, int b, int batch) {
    const int j = col >> 8, within = col & 255;
    const int c = within >> 6, r = within & 63;
    const int u = r >> 2, e = r & 3;
    return ((((size_t)j * 16 + u) * batch + b) * 4 + c) * 4 + e;
}

template <bool FRAG>
__global__ void rht_in_kernel(const __half* __restrict__ x, int batch, int n, int B,
                              const uint32_t* __restrict__ sin_bits, __half* __restrict__ out) {
    extern __shared__ float buf[];
    const int blk = blockIdx.x, b = blockIdx.y;
    const __half* xb = x + (size_t)b * n + (size_t)blk * B;
    for (int i = threadIdx.x; i < B; i += blockDim.x) {
        float v = __half2float(xb[i]);
        buf[i] = sign_neg(sin_bits, blk * B + i) ? -v : v;
    }
    __syncthreads();
    fwht_smem(buf, B);
    const float scale = rsqrtf((float)B);
    for (int i = threadIdx.x; i < B; i += blockDim.x) {
        const int col = blk * B + i;
        const __half v = __float2half_rn(buf[i] * scale);
        if (FRAG)
            out[frag_index(col, b, batch)] = v;
        else
            out[(size_t)b * n + col] = v;
    }
}

template <bool FRAG>
static cudaError_t launch_rht_in(const Layer& L, const void* x, int batch, void* xp, cudaStream_t st) {
    const int B = L.B_n;
    const size_t smem = (size_t)B * sizeof(float);
    auto kern = rht_in_kernel<FRAG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(L.n / B, batch);
    const int threads = B >= 1024 ? 1024 : (B >= 64 ? B : 64);
    kern<<<grid, threads, smem, st>>>((const __half*)x, batch, L.n, B, L.sin_bits, (__half*)xp);
    return cudaGetLastError();
}

cudaError_t launch_rht_in_frag(const Layer& L, const void* x, int batch, void* xp, cudaStream_t st) {
    return launch_rht_in<true>(L, x, batch, xp, st);
}

cudaError_t launch_rht_in_rowmajor(const Layer& L, const void* x, int batch, void* xp, cudaStream_t st) {
    return launch_rht_in<false>(L, x, batch, xp, st);
}

template <bool F16>
__global__ void rht_out_kernel(const float* __restrict__ z, int batch, int m, int B,
                               const uint32_t* __restrict__ sout_bits, float alpha, void* __restrict__ y) {
    extern __shared__ float buf[];
    const int blk = blockIdx.x, b = blockIdx.y;
    const float* zb = z + (size_t)b * m + (size_t)blk * B;
    for (int i = threadIdx.x; i < B; i += blockDim.x) buf[i] = zb[i];
    __syncthreads();
    fwht_smem(buf, B);
    const float scale = alpha * rsqrtf((float)B);
    for (int i = threadIdx.x; i < B; i += blockDim.x) {
        const int row = blk * B + i;
        float v = buf[i] * scale;
        if (sign_neg(sout_bits, row)) v = -v;
        if (F16)
            ((__half*)y)[(size_t)b * m + row] = __float2half_rn(v);
        else
            ((float*)y)[(size_t)b * m + row] = v;
    }
}

cudaError_t launch_rht_out(const Layer& L, const float* z, int batch, void* y, int y_dtype, cudaStream_t st) {
    const int B = L.B_m;
    const size_t smem = (size_t)B * sizeof(float);
    auto kern = (y_dtype == QL_F16) ? rht_out_kernel<true> : rht_out_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(L.m / B, batch);
    const int threads = B >= 1024 ? 1024 : (B >= 64 ? B : 64);
    kern<<<grid, threads, smem, st>>>(z, batch, L.m, B, L.sout_bits, L.alpha, y);
    return cudaGetLastError();
}

}  // namespace qlk
