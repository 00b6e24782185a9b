// encode.cu -- trellis-coded quantization (encoding) on the GPU: for each block
// of 256 source values, the bits whose tail-biting walk on the bitshift
// trellis reproduces the block with the least squared error (QTIP
// discussion: encoding searches the fixed-length walks of the trellis for the
// least distortion; the stream format stores each step's kV-bit delta).
//
// The search is the two-pass tail-biting Viterbi: pass 1 runs the dynamic
// programme with a free first state and takes the low L-kV bits of its best
// final state as the block's wrap-around prefix; pass 2 runs it with the first
// state's high bits and the last state's low bits tied to that prefix, and
// traces the best walk back.  Costs are float32 with every operation rounded
// to nearest (difference, square, sum over the V values in order, addition to
// the path cost; no fused multiply-add); ties go to the smallest predecessor
// and the smallest final state.
//
// Bitshift structure: the 2^kV predecessors of state s = a*2^kV + c are
// a + h*G (G = 2^(L-kV), h < 2^kV), the same set for every c.  So a step is,
// for every group a, one minimum over its 2^kV predecessors (the choice h is
// recorded per group), then the 2^kV successors' costs.  One CTA encodes one
// block with both cost buffers and the code values in shared memory, which
// bounds L to 14.
#include <cuda_fp16.h>
#include <math.h>

#include "codes.cuh"
#include "internal.h"

namespace qlk {

constexpr int kEncThreads = 1024;
constexpr int kEncMaxL = 14;

struct EncodeArgs {
    int code, L, kV, V, Q;
    const uint32_t* lut;    // HYB table or codebook, 2^Q words (codebook: Q = L)
    const float* x;         // [blocks][256]
    int blocks;
    uint32_t* words;        // [blocks][256 k / 32], stream format
    float* err;             // [blocks] squared error of the reconstruction, or null
    uint8_t* choice;        // [blocks][T][G] predecessor choices (global scratch)
    int* status;
};

// Code values of state s into v[0..V).
__device__ __forceinline__ void code_values(const EncodeArgs& p, const uint32_t* lut_lane, uint32_t s, float* v) {
    if (p.V == 2) {
        const uint32_t w = p.code == kCodeTable ? code_v2<kCodeTable>(s, lut_lane, 0)
                                                : code_v2<kCodeHYB>(s, lut_lane, 32 - p.Q);
        v[0] = __half2float(__ushort_as_half((unsigned short)(w & 0xFFFF)));
        v[1] = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
        return;
    }
    uint32_t w;
    if (p.code == kCode1MAD) w = code_pair<kCode1MAD>(s, s, lut_lane, 0);
    else if (p.code == kCode3INST) w = code_pair<kCode3INST>(s, s, lut_lane, 0);
    else if (p.code == kCodeTable) w = code_pair<kCodeTable>(s, s, lut_lane, 0);
    else w = code_pair<kCodeHYB>(s, s, lut_lane, 32 - p.Q);
    v[0] = __half2float(__ushort_as_half((unsigned short)(w & 0xFFFF)));
}

// (value, index) minimum over the CTA, ties to the smaller index.
__device__ __forceinline__ void argmin_cta(float& val, int& idx, float* red_v, int* red_i) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_down_sync(0xffffffffu, val, o);
        const int oi = __shfl_down_sync(0xffffffffu, idx, o);
        if (ov < val || (ov == val && oi < idx)) val = ov, idx = oi;
    }
    if (lane == 0) red_v[w] = val, red_i[w] = idx;
    __syncthreads();
    if (w == 0) {
        val = lane < (int)(blockDim.x >> 5) ? red_v[lane] : INFINITY;
        idx = lane < (int)(blockDim.x >> 5) ? red_i[lane] : 0x7fffffff;
        for (int o = 16; o; o >>= 1) {
            const float ov = __shfl_down_sync(0xffffffffu, val, o);
            const int oi = __shfl_down_sync(0xffffffffu, idx, o);
            if (ov < val || (ov == val && oi < idx)) val = ov, idx = oi;
        }
        if (lane == 0) red_v[0] = val, red_i[0] = idx;
    }
    __syncthreads();
    val = red_v[0];
    idx = red_i[0];
    __syncthreads();
}

__global__ void __launch_bounds__(kEncThreads, 1) encode_kernel(EncodeArgs p) {
    extern __shared__ float esm[];
    const int L = p.L, kV = p.kV, V = p.V;
    const int S = 1 << L, G = S >> kV, C = 1 << kV;
    const int T = 256 / V;
    float* cost_a = esm;                // [S]
    float* cost_b = cost_a + S;         // [S]
    float* vals = cost_b + S;           // [S][V]
    float* xs = vals + S * V;           // [256]
    float* red_v = xs + 256;            // [32]
    int* red_i = reinterpret_cast<int*>(red_v + 32);
    uint32_t* lut_smem = reinterpret_cast<uint32_t*>(red_i + 32);  // table codes: 2^Q x 32 replicated words
    const int lane = threadIdx.x & 31;
    if (uses_table(p.code))
        for (int i = threadIdx.x; i < (32 << p.Q); i += blockDim.x) lut_smem[i] = p.lut[i >> 5];
    __syncthreads();
    const uint32_t* lut_lane = lut_smem + lane;
    for (int s = threadIdx.x; s < S; s += blockDim.x) {
        float v[2];
        code_values(p, lut_lane, (uint32_t)s, v);
        for (int e = 0; e < V; ++e) vals[s * V + e] = v[e];
    }
    uint8_t* choice = p.choice + (size_t)blockIdx.x * T * G;
    for (int blk = blockIdx.x; blk < p.blocks; blk += gridDim.x) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) xs[i] = p.x[(size_t)blk * 256 + i];
        __syncthreads();
        // step cost of state s at step t (the float32 rule)
        auto dist = [&](int t, int s) {
            float d = 0.f;
            for (int e = 0; e < V; ++e) {
                const float diff = __fsub_rn(xs[t * V + e], vals[s * V + e]);
                d = e ? __fadd_rn(d, __fmul_rn(diff, diff)) : __fmul_rn(diff, diff);
            }
            return d;
        };
        int prefix = 0;
        int last = 0;
        for (int pass = 0; pass < 2; ++pass) {
            float* old_c = cost_a;
            float* new_c = cost_b;
            for (int s = threadIdx.x; s < S; s += blockDim.x)
                old_c[s] = (pass == 0 || (s >> kV) == prefix) ? dist(0, s) : INFINITY;
            __syncthreads();
            for (int t = 1; t < T; ++t) {
                for (int a = threadIdx.x; a < G; a += blockDim.x) {
                    float m = old_c[a];
                    int hb = 0;
                    for (int h = 1; h < C; ++h) {
                        const float c = old_c[a + h * G];
                        if (c < m) m = c, hb = h;
                    }
                    if (pass == 1) choice[(size_t)t * G + a] = (uint8_t)hb;
                    for (int c = 0; c < C; ++c) {
                        const int s = a * C + c;
                        new_c[s] = __fadd_rn(m, dist(t, s));
                    }
                }
                __syncthreads();
                float* tmp = old_c;
                old_c = new_c;
                new_c = tmp;
            }
            // best final state (pass 2: only those whose low bits are the prefix)
            float bv = INFINITY;
            int bi = 0x7fffffff;
            for (int s = threadIdx.x; s < S; s += blockDim.x) {
                if (pass == 1 && (s & (G - 1)) != prefix) continue;
                const float c = old_c[s];
                if (c < bv || (c == bv && s < bi)) bv = c, bi = s;
            }
            argmin_cta(bv, bi, red_v, red_i);
            if (bi < 0 || bi >= S) {  // no finite walk (cannot happen for finite inputs)
                if (threadIdx.x == 0) atomicOr(p.status, kStatusBadInput);
                bi = 0;
            }
            if (pass == 0) prefix = bi & (G - 1);
            last = bi;
        }
        // trace back (one thread), pack the chunks MSB-first, score the reconstruction
        __threadfence_block();
        __syncthreads();
        if (threadIdx.x == 0) {
            const int words_per_block = T * kV / 32;
            uint32_t* out = p.words + (size_t)blk * words_per_block;
            for (int i = 0; i < words_per_block; ++i) out[i] = 0u;
            int s = last;
            float err = 0.f;
            for (int t = T - 1; t >= 0; --t) {
                const uint32_t chunk = (uint32_t)(s & (C - 1));
                const int bitpos = t * kV;  // chunk t covers bits [t kV, (t+1) kV) of the block
                for (int b = 0; b < kV; ++b) {
                    const int pos = bitpos + b;
                    const uint32_t bit = (chunk >> (kV - 1 - b)) & 1u;
                    out[pos >> 5] |= bit << (31 - (pos & 31));
                }
                for (int e = 0; e < V; ++e) {
                    const float diff = xs[t * V + e] - vals[s * V + e];
                    err += diff * diff;
                }
                if (t) {
                    const int a = s >> kV;
                    s = a + (int)choice[(size_t)t * G + a] * G;
                }
            }
            if (p.err) p.err[blk] = err;
        }
        __syncthreads();
    }
}

size_t encode_smem_bytes(int L, int V, int code, int Q) {
    const size_t S = (size_t)1 << L;
    size_t b = (2 * S + S * V + 256 + 32) * 4 + 32 * 4;
    if (uses_table(code)) b += ((size_t)32 << Q) * 4;
    return b;
}

cudaError_t launch_encode(int code, int L, int kv, int V, int Q, const uint32_t* lut, const float* x, int blocks,
                          uint32_t* words, float* err, uint8_t* choice, int grid, int* status, cudaStream_t st) {
    EncodeArgs a;
    a.code = code;
    a.L = L;
    a.kV = kv;
    a.V = V;
    a.Q = Q;
    a.lut = lut;
    a.x = x;
    a.blocks = blocks;
    a.words = words;
    a.err = err;
    a.choice = choice;
    a.status = status;
    const size_t smem = encode_smem_bytes(L, V, code, Q);
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(encode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcMaxSmem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    encode_kernel<<<grid, kEncThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace qlk
