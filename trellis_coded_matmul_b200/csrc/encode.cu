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
// Up to L = 14 one CTA encodes one block with both cost vectors and the code
// values in its shared memory.  At L = 15 and 16 (the discussion's
// experiments use L = 16) the 2^L states are split over a thread-block
// cluster of 2 or 4 CTAs, 16384 states each: a CTA keeps its states' two cost
// vectors and code values (fp16, which they are exactly) in its shared
// memory, reads the predecessors' costs from the other CTAs' shared memory
// (distributed shared memory), and the cluster synchronises once per step.
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <math.h>

#include "codes.cuh"
#include "encode.h"
#include "internal.h"

namespace cg = cooperative_groups;

namespace qlk {

constexpr int kEncThreads = 1024;
constexpr int kEncMaxL = 14;           // single-CTA kernel
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

size_t encode_smem_bytes(int L, int V, int code, int Q) {
    if (L > kEncMaxL) return (size_t)cluster_smem(V).total;
    const size_t S = (size_t)1 << L;
    size_t b = (2 * S + S * V + 256 + 32) * 4 + 32 * 4;
    if (uses_table(code)) b += ((size_t)32 << Q) * 4;
    return b;
}

static int encode_cluster_size(int L) { return L > kEncMaxL ? (1 << L) / kEncClusterStates : 1; }

template <int KV>
static cudaError_t cluster_config(int nc, int workers, size_t smem, cudaStream_t st, cudaLaunchConfig_t* cfg,
                                  cudaLaunchAttribute* attr) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(encode_cluster_kernel<KV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kTcMaxSmem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
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

cudaError_t encode_workers(int L, int kv, int V, int blocks, int num_sms, int* workers) {
    int w = num_sms;
    if (L > kEncMaxL) {
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
    const size_t smem = encode_smem_bytes(L, V, code, Q);
    if (L > kEncMaxL) {
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
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(encode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcMaxSmem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    encode_kernel<<<workers, kEncThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace qlk
