// prep.cu -- one-time kernels run by qlinear_create: re-layout of the code
// words, bit-packing of the sign vectors, copy of the HYB / codebook table.
#include <cuda_fp16.h>

#include "internal.h"
#include "layout.cuh"

namespace qlk {

// One thread per destination word of one part.  The source word of
// thread-row (h, lane) word w of unit (R, j) is word
//   (row_local * n * k + j * 256k + c * 64k) / 32 + w
//     = row_local * (n / 64) * K2 + j * 4 K2 + c * K2 + w      (c = lane % 4, K2 = 2k)
// of the part's stream, row_local = 16R + 8h + lane / 4.
__global__ void relayout_kernel(const uint32_t* __restrict__ src, uint32_t* __restrict__ dst,
                                size_t n_words, int k2, int nb, int n) {
    const size_t unit_words = 64u * (size_t)k2;
    for (size_t d = blockIdx.x * (size_t)blockDim.x + threadIdx.x; d < n_words;
         d += (size_t)gridDim.x * blockDim.x) {
        const size_t unit = d / unit_words;
        const uint32_t within = (uint32_t)(d % unit_words);
        int h, lane, w;
        unit_word_coords(k2, within, &h, &lane, &w);
        const size_t R = unit / nb, j = unit % nb;
        const size_t row = R * 16 + 8 * h + (lane >> 2);
        const size_t c = lane & 3;
        const size_t s = row * (size_t)(n / 64) * k2 + j * 4u * k2 + c * k2 + w;
        dst[d] = src[s];
    }
}

cudaError_t launch_relayout(const uint32_t* src, uint32_t* dst, const Part& part, int n, cudaStream_t st) {
    if (part.n_words == 0) return cudaSuccess;
    const int threads = 256;
    size_t blocks = (part.n_words + threads - 1) / threads;
    if (blocks > 65535u * 8u) blocks = 65535u * 8u;
    relayout_kernel<<<(unsigned)blocks, threads, 0, st>>>(src, dst + part.word_off, part.n_words, part.k2,
                                                          n / kT, n);
    return cudaGetLastError();
}

// One warp per 32 entries: bit i of word i/32 is set when s[i] == -1.
__global__ void pack_signs_kernel(const int8_t* __restrict__ s, int count, uint32_t* __restrict__ bits,
                                  int* status) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const int v = (i < count) ? (int)s[i] : 1;
    if (v != 1 && v != -1) atomicOr(status, kStatusBadSign);
    const unsigned word = __ballot_sync(0xffffffffu, v == -1);
    if ((threadIdx.x & 31) == 0 && i < count) bits[i >> 5] = word;
}

cudaError_t launch_pack_signs(const int8_t* s, int count, uint32_t* bits, int* status, cudaStream_t st) {
    const int threads = 256;
    pack_signs_kernel<<<(count + threads - 1) / threads, threads, 0, st>>>(s, count, bits, status);
    return cudaGetLastError();
}

// HYB table or codebook: 2^Q entries of V fp16 -> 2^Q words (V = 2: value 0 in the low
// half, value 1 in the high half; V = 1: the value in the low half).
__global__ void copy_lut_kernel(const uint16_t* __restrict__ lut, int entries, int V, uint32_t* __restrict__ dst) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= entries) return;
    dst[i] = (V == 2) ? ((uint32_t)lut[2 * i] | ((uint32_t)lut[2 * i + 1] << 16)) : (uint32_t)lut[i];
}

cudaError_t launch_copy_lut(const void* lut_f16, int Q, int V, uint32_t* dst, cudaStream_t st) {
    const int entries = 1 << Q;
    copy_lut_kernel<<<(entries + 255) / 256, 256, 0, st>>>((const uint16_t*)lut_f16, entries, V, dst);
    return cudaGetLastError();
}

}  // namespace qlk
