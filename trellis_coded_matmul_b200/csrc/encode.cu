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
// recorded per group), then the 2^kV successors' costs.
//
// One CTA encodes one block whenever the group minima fit its shared memory
// (every case but L = 16 with kV = 1): it stores only M_t(a) = min_h
// cost_{t-1}(a + hG), 2^(L-kV) floats per buffer, and recomputes a state's
// cost M_t(s >> kV) + d(t, s) when it reads it (the same float32 operations
// as storing it), with the code values computed on the fly, or, at L = 13-16
// with one value and 2-4 bits per step, held in registers for the whole
// kernel (2^L / 512 states a thread).  L = 16 with
// kV = 1 splits the 2^16 states over a thread-block cluster of 4 CTAs,
// 16384 states each, which keep their costs and code values (fp16, which they
// are exactly) in shared memory and read the predecessors' costs from the
// other CTAs' shared memory; the cluster synchronises once per step.
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <math.h>

#include "codes.cuh"
#include "encode.h"
#include "internal.h"

namespace cg = cooperative_groups;

namespace qlk {

constexpr int kEncThreads = 1024;
constexpr int kEncMaxL = 14;           // above: the cluster kernel when the group minima do not fit
constexpr int kEncClusterStates = 16384;  // states per CTA of a cluster (L = 15, 16)

struct EncodeArgs {
    int code, L, kV, V, Q;
    const uint32_t* lut;    // HYB table or codebook, 2^Q words (codebook: Q = L)
    const float* x;         // [blocks][256]
    int blocks;
    uint32_t* words;        // [blocks][256 k / 32], stream format
    float* err;             // [blocks] squared error of the reconstruction, or null
    uint8_t* choice;        // [workers][T][G] predecessor choices (global scratch)
    int* status;
    int nc;                 // CTAs per cluster (cluster kernel)
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

// ---- group-minima search (one CTA per block): cost_t(s) = M_t(s >> kV) + d(t, s) ----
// Only the group minima M_t(a) = min_h cost_{t-1}(a + hG) are stored (2^(L-kV)
// floats per buffer); a state's cost is recomputed when it is read, with the
// same float32 operations as the stored form, and the code values are
// computed (or looked up in the replicated table) on the fly.
// fp32 values of state s (V of them), fp16-exact
template <int CODE, int V>
__device__ __forceinline__ void values_of(uint32_t s, const uint32_t* lut_lane, int qshift, float (&v)[V]) {
    uint32_t w;
    if constexpr (V == 2) w = code_v2<CODE>(s, lut_lane, qshift);
    else w = code_pair<CODE>(s, s, lut_lane, qshift);
    v[0] = __half2float(__ushort_as_half((unsigned short)(w & 0xFFFF)));
    if constexpr (V == 2) v[1] = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
}

// v - x for the fp16 v in the low (HI = false) or high half of a word and a
// float32 x, rounded to nearest once: the mixed-precision subtraction of
// sm_100, which widens v exactly.  Its square is the square of x - v bit for
// bit (rounding to nearest is symmetric in sign).  The word is split inside the
// asm so that the halves are not kept as separate registers.
template <bool HI>
__device__ __forceinline__ float sub_f16_f32(uint32_t w, float x) {
    float d;
    if constexpr (HI)
        asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tsub.rn.f32.f16 %0, hi, %2;\n\t}"
            : "=f"(d) : "r"(w), "f"(x));
    else
        asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tsub.rn.f32.f16 %0, lo, %2;\n\t}"
            : "=f"(d) : "r"(w), "f"(x));
    return d;
}

template <int V>
__device__ __forceinline__ float dist_of(const float* xt, const float (&v)[V]) {
    const float d0 = __fsub_rn(xt[0], v[0]);
    float d = __fmul_rn(d0, d0);
    if constexpr (V == 2) {
        const float d1 = __fsub_rn(xt[1], v[1]);
        d = __fadd_rn(d, __fmul_rn(d1, d1));
    }
    return d;
}

// Squared distance of state s's values (computed from the code) to xt[0..V),
// with the float32 rule of dist_of, each difference one mixed-precision
// subtraction on the fp16 value.
template <int CODE, int V>
__device__ __forceinline__ float dist_of_state(uint32_t s, const uint32_t* lut_lane, int qshift, const float* xt) {
    uint32_t w;
    if constexpr (V == 2) w = code_v2<CODE>(s, lut_lane, qshift);
    else w = code_pair<CODE>(s, s, lut_lane, qshift);
    const float d0 = sub_f16_f32<false>(w, xt[0]);
    float d = __fmul_rn(d0, d0);
    if constexpr (V == 2) {
        const float d1 = sub_f16_f32<true>(w, xt[1]);
        d = __fadd_rn(d, __fmul_rn(d1, d1));
    }
    return d;
}


template <int CODE, int KV, int V>
__global__ void __launch_bounds__(1024, 1) encode_gm_kernel(EncodeArgs p) {
    extern __shared__ __align__(16) unsigned char sm[];
    constexpr int C = 1 << KV;
    constexpr int T = 256 / V;
    const int L = p.L;
    const int S = 1 << L, G = S >> KV;  // p.kV == KV, p.V == V
    const int qshift = 32 - p.Q;
    float* Ma = reinterpret_cast<float*>(sm);
    float* Mb = Ma + G;
    float* xs = Mb + G;
    float* red_v = xs + 256;
    int* red_i = reinterpret_cast<int*>(red_v + 32);
    uint32_t* lut_smem = reinterpret_cast<uint32_t*>(red_i + 32);
    const int lane = threadIdx.x & 31;
    if (uses_table(CODE))
        for (int i = threadIdx.x; i < (32 << p.Q); i += blockDim.x) lut_smem[i] = p.lut[i >> 5];
    __syncthreads();
    const uint32_t* lut_lane = lut_smem + lane;
    uint8_t* choice = p.choice + (size_t)blockIdx.x * T * G;
    for (int blk = blockIdx.x; blk < p.blocks; blk += gridDim.x) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) xs[i] = p.x[(size_t)blk * 256 + i];
        __syncthreads();
        int prefix = 0, last = 0;
        for (int pass = 0; pass < 2; ++pass) {
            float* Mp = Ma;
            float* Mn = Mb;
            for (int a = threadIdx.x; a < G; a += blockDim.x) Mp[a] = (pass == 0 || a == prefix) ? 0.f : INFINITY;
            __syncthreads();
            for (int t = 1; t < T; ++t) {
                const float* xt = xs + (t - 1) * V;
                for (int a = threadIdx.x; a < G; a += blockDim.x) {
                    float m = INFINITY;
                    int hb = 0;
#pragma unroll (C <= 16 ? C : 4)
                    for (int h = 0; h < C; ++h) {
                        const uint32_t q = (uint32_t)(a + h * G);
                        const float c = __fadd_rn(Mp[q >> KV], dist_of_state<CODE, V>(q, lut_lane, qshift, xt));
                        if (c < m) m = c, hb = h;
                    }
                    Mn[a] = m;
                    if (pass == 1) choice[(size_t)t * G + a] = (uint8_t)hb;
                }
                __syncthreads();
                float* tmp = Mp;
                Mp = Mn;
                Mn = tmp;
            }
            const float* xl = xs + (T - 1) * V;
            float bv = INFINITY;
            int bi = 0x7fffffff;
            for (int s = threadIdx.x; s < S; s += blockDim.x) {
                if (pass == 1 && (s & (G - 1)) != prefix) continue;
                float v[V];
                values_of<CODE, V>((uint32_t)s, lut_lane, qshift, v);
                const float c = __fadd_rn(Mp[s >> KV], dist_of<V>(xl, v));
                if (c < bv || (c == bv && s < bi)) bv = c, bi = s;
            }
            argmin_cta(bv, bi, red_v, red_i);
            if (bi < 0 || bi >= S) {
                if (threadIdx.x == 0) atomicOr(p.status, kStatusBadInput);
                bi = 0;
            }
            if (pass == 0) prefix = bi & (G - 1);
            last = bi;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            constexpr int words_per_block = T * KV / 32;
            uint32_t* out = p.words + (size_t)blk * words_per_block;
            for (int i = 0; i < words_per_block; ++i) out[i] = 0u;
            int s = last;
            float err = 0.f;
            for (int t = T - 1; t >= 0; --t) {
                const uint32_t chunk = (uint32_t)(s & (C - 1));
                for (int b = 0; b < KV; ++b) {
                    const int pos = t * KV + b;
                    out[pos >> 5] |= ((chunk >> (KV - 1 - b)) & 1u) << (31 - (pos & 31));
                }
                float v[V];
                values_of<CODE, V>((uint32_t)s, lut_lane, qshift, v);
                for (int e = 0; e < V; ++e) {
                    const float diff = xs[t * V + e] - v[e];
                    err += diff * diff;
                }
                if (t) {
                    const int a = s >> KV;
                    s = a + (int)choice[(size_t)t * G + a] * G;
                }
            }
            if (p.err) p.err[blk] = err;
        }
        __syncthreads();
    }
}


// ---- L = 15, 16: one cluster of nc CTAs per block ----

// Packed fp16 value word of state s (value 0 in the low half), the tables read
// from global memory (the values are computed once per CTA).
__device__ __forceinline__ uint32_t code_word_global(const EncodeArgs& p, uint32_t s) {
    if (p.code == kCode1MAD) return code_pair<kCode1MAD>(s, s, nullptr, 0);
    if (p.code == kCode3INST) return code_pair<kCode3INST>(s, s, nullptr, 0);
    if (p.code == kCodeTable) return p.lut[s];
    const uint32_t x = kAHYB * s + kBHYB;
    return p.lut[x >> (32 - p.Q)] ^ (x & 0x8000u);
}

struct ClusterSmem {
    int cost_a, cost_b, vals, xs, red_v, red_i, res, total;  // byte offsets
};
__host__ __device__ inline ClusterSmem cluster_smem(int V) {
    ClusterSmem s;
    s.cost_a = 0;
    s.cost_b = s.cost_a + kEncClusterStates * 4;
    s.vals = s.cost_b + kEncClusterStates * 4;
    s.xs = s.vals + kEncClusterStates * V * 2;
    s.red_v = s.xs + 256 * 4;
    s.red_i = s.red_v + 32 * 4;
    s.res = s.red_i + 32 * 4;  // this CTA's best final state: (value, index)
    s.total = s.res + 16;
    return s;
}

template <int KV>
__global__ void __launch_bounds__(kEncThreads, 1) encode_cluster_kernel(EncodeArgs p) {
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ __align__(16) unsigned char csm[];
    constexpr int C = 1 << KV;
    constexpr int SL = kEncClusterStates;  // states of this CTA: [s0, s0 + SL)
    constexpr int kLogSL = 14;
    constexpr int NA = SL >> KV;           // groups whose successors are this CTA's states
    const int L = p.L, V = p.V;
    const int S = 1 << L, G = S >> KV;
    const int NC = p.nc;
    const int T = 256 / V;
    const ClusterSmem lay = cluster_smem(V);
    float* cost_a = reinterpret_cast<float*>(csm + lay.cost_a);
    float* cost_b = reinterpret_cast<float*>(csm + lay.cost_b);
    __half* vals = reinterpret_cast<__half*>(csm + lay.vals);
    float* xs = reinterpret_cast<float*>(csm + lay.xs);
    float* red_v = reinterpret_cast<float*>(csm + lay.red_v);
    int* red_i = reinterpret_cast<int*>(csm + lay.red_i);
    float* res_v = reinterpret_cast<float*>(csm + lay.res);
    int* res_i = reinterpret_cast<int*>(csm + lay.res + 4);
    const int rank = (int)cluster.block_rank();
    const int s0 = rank * SL;
    const int a0 = s0 >> KV;
    for (int i = threadIdx.x; i < SL; i += blockDim.x) {
        const uint32_t w = code_word_global(p, (uint32_t)(s0 + i));
        vals[i * V] = __ushort_as_half((unsigned short)(w & 0xFFFF));
        if (V == 2) vals[i * V + 1] = __ushort_as_half((unsigned short)(w >> 16));
    }
    const int worker = blockIdx.x / NC, workers = gridDim.x / NC;
    uint8_t* choice = p.choice + (size_t)worker * T * G;
    // every CTA of a cluster runs the same iterations and barriers
    for (int blk = worker; blk < p.blocks; blk += workers) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) xs[i] = p.x[(size_t)blk * 256 + i];
        __syncthreads();
        auto dist = [&](int t, int sl) {  // the float32 rule, local state sl
            float d = 0.f;
            for (int e = 0; e < V; ++e) {
                const float diff = __fsub_rn(xs[t * V + e], __half2float(vals[sl * V + e]));
                d = e ? __fadd_rn(d, __fmul_rn(diff, diff)) : __fmul_rn(diff, diff);
            }
            return d;
        };
        int prefix = 0;
        int last = 0;
        for (int pass = 0; pass < 2; ++pass) {
            float* old_c = cost_a;
            float* new_c = cost_b;
            for (int i = threadIdx.x; i < SL; i += blockDim.x)
                old_c[i] = (pass == 0 || ((s0 + i) >> KV) == prefix) ? dist(0, i) : INFINITY;
            cluster.sync();
            for (int t = 1; t < T; ++t) {
                for (int ai = threadIdx.x; ai < NA; ai += blockDim.x) {
                    const int a = a0 + ai;
                    // first minimum over the predecessors a + h G (h ascending), which
                    // live in CTA (a + h G) / SL; CH loads in flight at a time
                    constexpr int CH = C < 4 ? C : 4;
                    float m = INFINITY;
                    int hb = 0;
#pragma unroll 4
                    for (int h0 = 0; h0 < C; h0 += CH) {
                        float c[CH];
#pragma unroll
                        for (int j = 0; j < CH; ++j) {
                            const int q = a + (h0 + j) * G;
                            c[j] = cluster.map_shared_rank(old_c, q >> kLogSL)[q & (SL - 1)];
                        }
#pragma unroll
                        for (int j = 0; j < CH; ++j)
                            if (c[j] < m) m = c[j], hb = h0 + j;
                    }
                    if (pass == 1) choice[(size_t)t * G + a] = (uint8_t)hb;
#pragma unroll 4
                    for (int cc = 0; cc < C; ++cc) {
                        const int sl = ai * C + cc;  // local index of state a C + cc
                        new_c[sl] = __fadd_rn(m, dist(t, sl));
                    }
                }
                cluster.sync();
                float* tmp = old_c;
                old_c = new_c;
                new_c = tmp;
            }
            // best final state of the cluster (pass 2: only those whose low bits are the prefix)
            float bv = INFINITY;
            int bi = 0x7fffffff;
            for (int i = threadIdx.x; i < SL; i += blockDim.x) {
                const int s = s0 + i;
                if (pass == 1 && (s & (G - 1)) != prefix) continue;
                const float cv = old_c[i];
                if (cv < bv || (cv == bv && s < bi)) bv = cv, bi = s;
            }
            argmin_cta(bv, bi, red_v, red_i);
            if (threadIdx.x == 0) {
                *res_v = bv;
                *res_i = bi;
            }
            cluster.sync();
            float gv = INFINITY;
            int gi = 0x7fffffff;
            for (int r = 0; r < NC; ++r) {  // the same combination, in rank order, in every CTA
                const float v = *cluster.map_shared_rank(res_v, r);
                const int i = *cluster.map_shared_rank(res_i, r);
                if (v < gv || (v == gv && i < gi)) gv = v, gi = i;
            }
            if (gi < 0 || gi >= S) {  // no finite walk (cannot happen for finite inputs)
                if (threadIdx.x == 0 && rank == 0) atomicOr(p.status, kStatusBadInput);
                gi = 0;
            }
            if (pass == 0) prefix = gi & (G - 1);
            last = gi;
            cluster.sync();  // every CTA has read the results before they are rewritten
        }
        // trace back (one thread of rank 0): choices from global memory (written
        // before the cluster barriers), code values from the owning CTA
        if (rank == 0 && threadIdx.x == 0) {
            const int words_per_block = T * KV / 32;
            uint32_t* out = p.words + (size_t)blk * words_per_block;
            for (int i = 0; i < words_per_block; ++i) out[i] = 0u;
            int s = last;
            float err = 0.f;
            for (int t = T - 1; t >= 0; --t) {
                const uint32_t chunk = (uint32_t)(s & (C - 1));
                const int bitpos = t * KV;
                for (int b = 0; b < KV; ++b) {
                    const int pos = bitpos + b;
                    const uint32_t bit = (chunk >> (KV - 1 - b)) & 1u;
                    out[pos >> 5] |= bit << (31 - (pos & 31));
                }
                const __half* vs = cluster.map_shared_rank(vals, s >> kLogSL) + (s & (SL - 1)) * V;
                for (int e = 0; e < V; ++e) {
                    const float diff = xs[t * V + e] - __half2float(vs[e]);
                    err += diff * diff;
                }
                if (t) {
                    const int a = s >> KV;
                    s = a + (int)choice[(size_t)t * G + a] * G;
                }
            }
            if (p.err) p.err[blk] = err;
        }
        cluster.sync();  // the next block rewrites the choices, costs and x
    }
}

// ---- L = 13..16, V = 1: the group-minima search with the code values in registers ----
// The same search, the same float32 operations and the same tie rules as
// encode_gm_kernel.  Each of the 512 threads owns runs ("units") of R
// consecutive groups a = base .. base + R - 1, R = min(2^kV, 8), base a
// multiple of R: all of them have the predecessor minima M(base >> kV + h
// G / 2^kV), so one shared-memory load per h serves R groups, and the unit's
// R new minima (and, in pass 2, its R choices) go out as one vector store.
// The fp16 values of the thread's 2^L / 512 states (128 at L = 16) stay in
// registers for the whole kernel instead of being recomputed 2 x 255 times
// per block.  Needs G >= 512 R (L = 16: kV <= 4; 15: kV <= 3; 13, 14: kV = 2).
constexpr int kEncRegThreads = 512;

template <int LL, int KV>
struct RegVals {
    static constexpr int G = (1 << LL) >> KV;
    static constexpr int C = 1 << KV;
    static constexpr int R = C < 8 ? C : 8;               // groups a unit
    static constexpr int NU = G / (kEncRegThreads * R);  // units a thread: unit j starts at (tid + 512 j) R
    static_assert(NU >= 1, "fewer groups than 512 units");
    uint32_t w[NU][R][C / 2];  // states base + r + h G and base + r + (h + 1) G (h even): low and high half
    __device__ __forceinline__ float at(int j, int r, int h) const {
        const uint32_t v = w[j][r][h >> 1];
        return __half2float(__ushort_as_half((unsigned short)((h & 1) ? (v >> 16) : (v & 0xFFFFu))));
    }
    // v(state) - x, see sub_f16_f32
    __device__ __forceinline__ float sub_at(int j, int r, int h, float x) const;
    __device__ __forceinline__ static int base(int j) { return ((int)threadIdx.x + j * kEncRegThreads) * R; }
};

template <int LL, int KV>
__device__ __forceinline__ float RegVals<LL, KV>::sub_at(int j, int r, int h, float x) const {
    return (h & 1) ? sub_f16_f32<true>(w[j][r][h >> 1], x) : sub_f16_f32<false>(w[j][r][h >> 1], x);
}

// One step for this thread's groups: Mn(a) = min_h cost_{t-1}(a + h G), the
// first minimum in ascending h, recorded in ch[a] in pass 2.  Pass 1 needs only
// the value, and fminf returns the same one: equal costs are the same float
// (no cost is -0), and both forms skip a NaN cost.
template <int LL, int KV, bool CHOICE>
__device__ __forceinline__ void reg_step(const RegVals<LL, KV>& rv, const float* __restrict__ Mp,
                                         float* __restrict__ Mn, float xt, uint8_t* __restrict__ ch) {
    using Rv = RegVals<LL, KV>;
    constexpr int R = Rv::R, C = Rv::C;
#pragma unroll
    for (int j = 0; j < Rv::NU; ++j) {
        const int b = Rv::base(j);
        float mp[C];
#pragma unroll
        for (int h = 0; h < C; ++h) mp[h] = Mp[(b >> KV) + h * (Rv::G >> KV)];
        float m[R];
        uint32_t hw[R / 4] = {};
#pragma unroll
        for (int r = 0; r < R; ++r) {
            m[r] = INFINITY;
            int hb = 0;
#pragma unroll
            for (int h = 0; h < C; ++h) {
                const float d0 = rv.sub_at(j, r, h, xt);
                const float c = __fadd_rn(mp[h], __fmul_rn(d0, d0));
                if constexpr (CHOICE) {
                    if (c < m[r]) m[r] = c, hb = h;
                } else {
                    m[r] = fminf(m[r], c);
                }
            }
            if constexpr (CHOICE) hw[r >> 2] |= (uint32_t)hb << (8 * (r & 3));
        }
#pragma unroll
        for (int q = 0; q < R; q += 4)
            *reinterpret_cast<float4*>(Mn + b + q) = make_float4(m[q], m[q + 1], m[q + 2], m[q + 3]);
        if constexpr (CHOICE) {
            if constexpr (R == 4) *reinterpret_cast<uint32_t*>(ch + b) = hw[0];
            else *reinterpret_cast<uint2*>(ch + b) = make_uint2(hw[0], hw[1]);
        }
    }
}

template <int LL, int KV>
__global__ void __launch_bounds__(kEncRegThreads, 1) encode_reg_kernel(EncodeArgs p) {
    extern __shared__ __align__(16) unsigned char sm[];
    using Rv = RegVals<LL, KV>;
    constexpr int S = 1 << LL, G = Rv::G, T = 256, R = Rv::R, C = Rv::C;
    float* Ma = reinterpret_cast<float*>(sm);
    float* Mb = Ma + G;
    float* xs = Mb + G;
    float* red_v = xs + 256;
    int* red_i = reinterpret_cast<int*>(red_v + 32);
    const int tid = threadIdx.x;
    Rv rv;
#pragma unroll
    for (int j = 0; j < Rv::NU; ++j)
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int h = 0; h < C; h += 2) {
                const uint32_t q = (uint32_t)(Rv::base(j) + r + h * G);
                rv.w[j][r][h >> 1] = __byte_perm(code_word_global(p, q), code_word_global(p, q + G), 0x5410);
            }
    uint8_t* choice = p.choice + (size_t)blockIdx.x * T * G;
    for (int blk = blockIdx.x; blk < p.blocks; blk += gridDim.x) {
        for (int i = tid; i < 256; i += blockDim.x) xs[i] = p.x[(size_t)blk * 256 + i];
        __syncthreads();
        int prefix = 0, last = 0;
        for (int pass = 0; pass < 2; ++pass) {
            float* Mp = Ma;
            float* Mn = Mb;
            for (int a = tid; a < G; a += blockDim.x) Mp[a] = (pass == 0 || a == prefix) ? 0.f : INFINITY;
            __syncthreads();
            for (int t = 1; t < T; ++t) {
                const float xt = xs[t - 1];
                if (pass == 0) reg_step<LL, KV, false>(rv, Mp, Mn, xt, nullptr);
                else reg_step<LL, KV, true>(rv, Mp, Mn, xt, choice + (size_t)t * G);
                __syncthreads();
                float* tmp = Mp;
                Mp = Mn;
                Mn = tmp;
            }
            // best final state (pass 2: only the states whose low bits, their group, are the prefix)
            const float xl = xs[T - 1];
            float bv = INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < Rv::NU; ++j)
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const int a = Rv::base(j) + r;
                    if (pass == 1 && a != prefix) continue;
#pragma unroll
                    for (int h = 0; h < C; ++h) {
                        const int s = a + h * G;
                        const float d0 = __fsub_rn(xl, rv.at(j, r, h));
                        const float c = __fadd_rn(Mp[s >> KV], __fmul_rn(d0, d0));
                        if (c < bv || (c == bv && s < bi)) bv = c, bi = s;
                    }
                }
            argmin_cta(bv, bi, red_v, red_i);
            if (bi < 0 || bi >= S) {
                if (tid == 0) atomicOr(p.status, kStatusBadInput);
                bi = 0;
            }
            if (pass == 0) prefix = bi & (G - 1);
            last = bi;
        }
        __syncthreads();
        if (tid == 0) {
            constexpr int words_per_block = T * KV / 32;
            uint32_t* out = p.words + (size_t)blk * words_per_block;
            for (int i = 0; i < words_per_block; ++i) out[i] = 0u;
            int s = last;
            float err = 0.f;
            for (int t = T - 1; t >= 0; --t) {
                const uint32_t chunk = (uint32_t)(s & (C - 1));
                for (int b = 0; b < KV; ++b) {
                    const int pos = t * KV + b;
                    out[pos >> 5] |= ((chunk >> (KV - 1 - b)) & 1u) << (31 - (pos & 31));
                }
                const float v = __half2float(__ushort_as_half((unsigned short)(code_word_global(p, (uint32_t)s) & 0xFFFFu)));
                const float diff = xs[t] - v;
                err += diff * diff;
                if (t) {
                    const int a = s >> KV;
                    s = a + (int)choice[(size_t)t * G + a] * G;
                }
            }
            if (p.err) p.err[blk] = err;
        }
        __syncthreads();
    }
}

static size_t reg_smem_bytes(int L, int kv) { return ((size_t)2 * ((size_t)1 << (L - kv)) + 256 + 64) * 4; }

template <int LL, int KV>
static cudaError_t launch_reg(const EncodeArgs& a, int workers, cudaStream_t st) {
    cudaError_t e = ensure_smem_limit<encode_reg_kernel<LL, KV>>(kTcMaxSmem);
    if (e != cudaSuccess) return e;
    encode_reg_kernel<LL, KV><<<workers, kEncRegThreads, reg_smem_bytes(LL, KV), st>>>(a);
    return cudaGetLastError();
}

static size_t gm_smem_bytes(int L, int kv, int code, int Q) {
    const size_t G = (size_t)1 << (L - kv);
    size_t b = (2 * G + 256 + 64) * 4;
    if (uses_table(code)) b += ((size_t)32 << Q) * 4;
    return b;
}

static bool use_gm(int L, int kv, int code, int Q) { return gm_smem_bytes(L, kv, code, Q) <= (size_t)kTcMaxSmem; }

// the register-cached search: one value per step, at least 2 bits per step
// and 512 units of groups (L = 16: kV 2..4, L = 15: 2..3, L = 13, 14: 2), where
// the group minima fit one CTA
static bool use_reg(int L, int kv, int V, int code, int Q) {
    const int R = kv >= 3 ? 8 : 4;
    return L >= 13 && L <= 16 && V == 1 && kv >= 2 && kv <= 4 && ((1 << (L - kv)) >= kEncRegThreads * R) &&
           use_gm(L, kv, code, Q);
}

size_t encode_smem_bytes(int L, int kv, int V, int code, int Q) {
    if (use_gm(L, kv, code, Q)) return gm_smem_bytes(L, kv, code, Q);
    if (L > kEncMaxL) return (size_t)cluster_smem(V).total;  // the cluster kernel reads tables from global memory
    return (size_t)-1;  // does not fit
}

static int encode_cluster_size(int L) { return L > kEncMaxL ? (1 << L) / kEncClusterStates : 1; }

template <int KV>
static cudaError_t cluster_config(int nc, int workers, size_t smem, cudaStream_t st, cudaLaunchConfig_t* cfg,
                                  cudaLaunchAttribute* attr) {
    cudaError_t e = ensure_smem_limit<encode_cluster_kernel<KV>>(kTcMaxSmem);
    if (e != cudaSuccess) return e;
    *cfg = cudaLaunchConfig_t{};
    cfg->gridDim = dim3(nc * workers);
    cfg->blockDim = dim3(kEncThreads);
    cfg->dynamicSmemBytes = smem;
    cfg->stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nc;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg->attrs = attr;
    cfg->numAttrs = 1;
    return cudaSuccess;
}

// Clusters that can be resident at once (each loops over its share of blocks).
template <int KV>
static cudaError_t cluster_workers(int nc, size_t smem, int* workers) {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    cudaError_t e = cluster_config<KV>(nc, 1, smem, 0, &cfg, attr);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveClusters(workers, encode_cluster_kernel<KV>, &cfg);
}

template <int KV>
static cudaError_t launch_cluster(const EncodeArgs& a, int workers, size_t smem, cudaStream_t st) {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    cudaError_t e = cluster_config<KV>(a.nc, workers, smem, st, &cfg, attr);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, encode_cluster_kernel<KV>, a);
}

cudaError_t encode_workers(int L, int kv, int V, int code, int Q, int blocks, int num_sms, int* workers) {
    int w = num_sms;
    if (!use_gm(L, kv, code, Q)) {
        const int nc = encode_cluster_size(L);
        const size_t smem = (size_t)cluster_smem(V).total;
        cudaError_t e = cudaErrorInvalidValue;
        switch (kv) {
            case 1: e = cluster_workers<1>(nc, smem, &w); break;
            case 2: e = cluster_workers<2>(nc, smem, &w); break;
            case 3: e = cluster_workers<3>(nc, smem, &w); break;
            case 4: e = cluster_workers<4>(nc, smem, &w); break;
            case 5: e = cluster_workers<5>(nc, smem, &w); break;
            case 6: e = cluster_workers<6>(nc, smem, &w); break;
            case 7: e = cluster_workers<7>(nc, smem, &w); break;
            case 8: e = cluster_workers<8>(nc, smem, &w); break;
        }
        if (e != cudaSuccess) return e;
        if (w < 1) return cudaErrorInvalidConfiguration;
    }
    *workers = blocks < w ? blocks : w;
    return cudaSuccess;
}

template <int CODE, int KV, int V>
static cudaError_t launch_gm(const EncodeArgs& a, int workers, size_t smem, cudaStream_t st) {
    auto kern = encode_gm_kernel<CODE, KV, V>;
    cudaError_t e = ensure_smem_limit<encode_gm_kernel<CODE, KV, V>>(kTcMaxSmem);
    if (e != cudaSuccess) return e;
    kern<<<workers, kEncThreads, smem, st>>>(a);
    return cudaGetLastError();
}

// (code, V, kv) -> the group-minima instance: V = 1 takes kv 1..4 (any code),
// V = 2 kv 2..8 (the table codes)
template <int CODE, int V>
static cudaError_t launch_gm_kv(const EncodeArgs& a, int kv, int workers, size_t smem, cudaStream_t st) {
    if constexpr (V == 1) {
        switch (kv) {
            case 1: return launch_gm<CODE, 1, 1>(a, workers, smem, st);
            case 2: return launch_gm<CODE, 2, 1>(a, workers, smem, st);
            case 3: return launch_gm<CODE, 3, 1>(a, workers, smem, st);
            case 4: return launch_gm<CODE, 4, 1>(a, workers, smem, st);
        }
    } else {
        switch (kv) {
            case 2: return launch_gm<CODE, 2, 2>(a, workers, smem, st);
            case 3: return launch_gm<CODE, 3, 2>(a, workers, smem, st);
            case 4: return launch_gm<CODE, 4, 2>(a, workers, smem, st);
            case 5: return launch_gm<CODE, 5, 2>(a, workers, smem, st);
            case 6: return launch_gm<CODE, 6, 2>(a, workers, smem, st);
            case 7: return launch_gm<CODE, 7, 2>(a, workers, smem, st);
            case 8: return launch_gm<CODE, 8, 2>(a, workers, smem, st);
        }
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_encode(int code, int L, int kv, int V, int Q, const uint32_t* lut, const float* x, int blocks,
                          uint32_t* words, float* err, uint8_t* choice, int workers, int* status, cudaStream_t st) {
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
    a.nc = encode_cluster_size(L);
    if (use_reg(L, kv, V, code, Q)) {
        switch (L * 8 + kv) {
            case 16 * 8 + 2: return launch_reg<16, 2>(a, workers, st);
            case 16 * 8 + 3: return launch_reg<16, 3>(a, workers, st);
            case 16 * 8 + 4: return launch_reg<16, 4>(a, workers, st);
            case 15 * 8 + 2: return launch_reg<15, 2>(a, workers, st);
            case 15 * 8 + 3: return launch_reg<15, 3>(a, workers, st);
            case 14 * 8 + 2: return launch_reg<14, 2>(a, workers, st);
            case 13 * 8 + 2: return launch_reg<13, 2>(a, workers, st);
        }
        return cudaErrorInvalidValue;
    }
    if (use_gm(L, kv, code, Q)) {
        const size_t smem = gm_smem_bytes(L, kv, code, Q);
        if (V == 1) {
            switch (code) {
                case kCode1MAD: return launch_gm_kv<kCode1MAD, 1>(a, kv, workers, smem, st);
                case kCode3INST: return launch_gm_kv<kCode3INST, 1>(a, kv, workers, smem, st);
                case kCodeHYB: return launch_gm_kv<kCodeHYB, 1>(a, kv, workers, smem, st);
                case kCodeTable: return launch_gm_kv<kCodeTable, 1>(a, kv, workers, smem, st);
            }
        } else {
            switch (code) {
                case kCodeHYB: return launch_gm_kv<kCodeHYB, 2>(a, kv, workers, smem, st);
                case kCodeTable: return launch_gm_kv<kCodeTable, 2>(a, kv, workers, smem, st);
            }
        }
        return cudaErrorInvalidValue;
    }
    const size_t smem = (size_t)cluster_smem(V).total;
    switch (kv) {
        case 1: return launch_cluster<1>(a, workers, smem, st);
        case 2: return launch_cluster<2>(a, workers, smem, st);
        case 3: return launch_cluster<3>(a, workers, smem, st);
        case 4: return launch_cluster<4>(a, workers, smem, st);
        case 5: return launch_cluster<5>(a, workers, smem, st);
        case 6: return launch_cluster<6>(a, workers, smem, st);
        case 7: return launch_cluster<7>(a, workers, smem, st);
        case 8: return launch_cluster<8>(a, workers, smem, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace qlk
