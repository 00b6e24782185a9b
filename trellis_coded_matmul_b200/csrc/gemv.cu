// gemv.cu -- fused trellis decode + matrix-vector product for batch <= 8, and
// the decode / eval_code test kernels built on the same device functions.
//
// Decode follows the QTIP discussion: the bitshift trellis makes every state
// a window of the stored bits, so a lane can decode any run of steps on its
// own ("the bitshift trellis also enables parallel decoding"), and the codes
// are computed in INT32 ALU (1MAD, 3INST) or with a small table in banked
// shared memory (HYB).  Decoded weights stay in registers: they are the A
// operand of m16n8k16 half-precision MMAs whose B operand is x' (batch padded
// to 8 columns) and whose fp32 accumulators hold 16 rows x 8 batch columns.
//
// Work split: the m x n matrix is a grid of units (16 rows x 256 columns).
// Units are numbered row-tile-major; every warp of the grid takes one
// contiguous, equally sized range of units, accumulates while the row tile is
// unchanged and adds its partial sums into z with atomics when it moves on.
// The k-slot order inside an MMA is free (both operands use it): lane c
// feeds its own 4 consecutive columns per MMA, so every lane walks a
// contiguous run of trellis steps and the matching x' values are one 8-byte
// load (see the fragment layout in rht.cu).
#include <cuda_fp16.h>

#include "codes.cuh"
#include "fwht.cuh"
#include "internal.h"
#include "layout.cuh"

namespace qlk {

struct DecodeArgs {
    const uint32_t* words;  // part's words, kernel layout
    int rt;                 // row tiles in the part
    int nb;                 // blocks per row
    uint32_t lmask;         // (1 << L) - 1
    int qshift;             // HYB: 32 - Q
    const uint32_t* lut;    // HYB: 2^Q words in global memory
    int lut_entries;
};

__device__ __forceinline__ uint4 ldg_stream_v4(const uint32_t* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ uint2 ldg_stream_v2(const uint32_t* p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ldg_stream_v1(const uint32_t* p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

// Load lane's two thread-rows of one unit into w[h][0 .. K2-1] (K2 = 2k).
template <int K2>
__device__ __forceinline__ void load_unit(uint32_t (&w)[2][K2], const uint32_t* unit_base, int lane) {
    using UL = UnitLayout<K2>;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int q = 0; q < UL::NV; ++q) {
            const uint32_t* p = unit_base + ((h * UL::NV + q) * 32 + lane) * UL::VW;
            if (UL::VW == 4) {
                const uint4 v = ldg_stream_v4(p);
                w[h][q * 4 + 0] = v.x;
                w[h][q * 4 + 1] = v.y;
                w[h][q * 4 + 2] = v.z;
                w[h][q * 4 + 3] = v.w;
            } else if (UL::VW == 2) {
                const uint2 v = ldg_stream_v2(p);
                w[h][q * 2 + 0] = v.x;
                w[h][q * 2 + 1] = v.y;
            } else {
                w[h][q] = ldg_stream_v1(p);
            }
        }
    }
}

// Fill the per-lane replicated table (HYB, or the table code's codebook) in shared memory.
__device__ __forceinline__ void fill_lut_smem(uint32_t* smem, const uint32_t* lut, int entries) {
    for (int i = threadIdx.x; i < entries * 32; i += blockDim.x) smem[i] = lut[i >> 5];
}

// A operands of the 16 m16n8k16 MMAs of one unit.  MMA u takes, for each
// thread-row h (row g for h = 0, row g + 8 for h = 1), the lane's columns
// 4u .. 4u+3 of its run, i.e. steps 4u .. 4u+3 (V = 1) or 2u, 2u+1 (V = 2):
//   a[0] = row g, columns 4u, 4u+1      a[2] = row g, columns 4u+2, 4u+3
//   a[1] = row g+8, columns 4u, 4u+1    a[3] = row g+8, columns 4u+2, 4u+3
// Paired extraction (16 % kV == 0): steps t and t + 16/kV share one funnel
// shift, which pairs MMA u with MMA u + MP (MP = 16/kV/steps-per-MMA).
// K2 = 2k bits per two weights (k may be a half number when V = 2).
template <int CODE, int K2, int V, bool L16>
struct UnitDecoder {
    static_assert((K2 * V) % 2 == 0, "a step carries a whole number of bits");
    static constexpr int kV = K2 * V / 2;
    static constexpr int SPM = 4 / V;                  // steps per MMA per thread-row
    static constexpr bool kPair = (16 % kV) == 0;
    static constexpr int P = kPair ? 16 / kV : 1;      // step distance of paired windows
    static constexpr int MP = kPair ? P / SPM : 1;     // MMA distance of paired MMAs
    static constexpr int NW = K2 + 1;

    // states of steps [t0, t0 + SPM) into s[0..SPM) and, when paired, of
    // [t0 + P, t0 + P + SPM) into s2[0..SPM)
    static __device__ __forceinline__ void states(const uint32_t (&cw)[NW], int t0, uint32_t lmask,
                                                  uint32_t (&s)[SPM], uint32_t (&s2)[SPM]) {
#pragma unroll
        for (int q = 0; q < SPM; ++q) {
            if (kPair)
                state_pair<kV, L16>(cw, t0 + q, lmask, s[q], s2[q]);
            else
                s[q] = state_one<kV, L16>(cw, t0 + q, lmask);
        }
    }

    static __device__ __forceinline__ void codes(const uint32_t (&s)[SPM], uint32_t& lo, uint32_t& hi,
                                                 const uint32_t* lut_lane, int qshift) {
        if constexpr (V == 1) {
            lo = code_pair<CODE>(s[0], s[1], lut_lane, qshift);
            hi = code_pair<CODE>(s[2], s[3], lut_lane, qshift);
        } else {
            lo = code_v2<CODE>(s[0], lut_lane, qshift);
            hi = code_v2<CODE>(s[SPM - 1], lut_lane, qshift);
        }
    }

    // Operands of MMA u (and, when paired, of MMA u + MP into a2).
    static __device__ __forceinline__ void operands(const uint32_t (&cw)[2][NW], int u, uint32_t lmask,
                                                    const uint32_t* lut_lane, int qshift, uint32_t (&a)[4],
                                                    uint32_t (&a2)[4]) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t s[SPM], s2[SPM];
            states(cw[h], u * SPM, lmask, s, s2);
            codes(s, a[h], a[2 + h], lut_lane, qshift);
            if (kPair) codes(s2, a2[h], a2[2 + h], lut_lane, qshift);
        }
    }
};

// Calls f(u, a) for u = 0..15 with the A operands of MMA u, in the order
// that lets paired extraction share its funnel shifts.
template <int CODE, int K2, int V, bool L16, typename F>
__device__ __forceinline__ void for_each_mma(const uint32_t (&cw)[2][K2 + 1], uint32_t lmask,
                                             const uint32_t* lut_lane, int qshift, F&& f) {
    using D = UnitDecoder<CODE, K2, V, L16>;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        if (D::kPair && ((u / D::MP) & 1)) continue;  // produced together with MMA u - MP
        uint32_t a[4], a2[4];
        D::operands(cw, u, lmask, lut_lane, qshift, a, a2);
        f(u, a);
        if (D::kPair) f(u + D::MP, a2);
    }
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct GemvArgs {
    DecodeArgs dec;
    const uint2* xf;  // x' fragment layout in global memory (when x' is not computed in-kernel)
    int batch;        // 1..8
    float* z;         // [batch][m], all-zero on entry (the output transform re-zeroes it)
    int m;
    int row0;         // first layer row of the part
    // input transform in-kernel (XSMEM): x' = H_n diag(s_in) x into shared memory
    const __half* x;  // [batch][n]
    const uint32_t* sin_bits;
    int n, B_n;
    int groups_in;    // thread groups (B_n/8 threads each) of the in-kernel input transform
};

// x' = H_n diag(s_in) x for every column and batch row, fp16, into the
// fragment layout in shared memory.  Groups of B_n/kXinE threads take one
// (batch row, Hadamard block) at a time; all threads run the same rounds.
// prepare() runs before the wait for the previous kernel (the sign bits are
// written once at create time); run() reads x, which that kernel may produce.
constexpr int kXinE = 8;  // entries per thread of the in-kernel input transform
struct InputTransform {
    int B, T, G, grp, tid, per_row, total;
    uint32_t sw0;  // sign bits of the thread's entries in the first round
    __device__ __forceinline__ void prepare(const GemvArgs& p) {
        B = p.B_n;
        T = B / kXinE;
        G = p.groups_in;  // groups with their own FWHT scratch; spare threads only join barriers
        grp = threadIdx.x / T;
        tid = threadIdx.x - grp * T;
        per_row = p.n / B;
        total = p.batch * per_row;
        sw0 = 0;
        if (grp < G && grp < total) {
            const int col = (grp % per_row) * B + tid * kXinE;
            sw0 = p.sin_bits[col >> 5] >> (col & 31);
        }
    }
    __device__ __forceinline__ void run(const GemvArgs& p, __half* xs, float* fw) const {
        const float scale = rsqrtf((float)B);
        for (int r0 = 0; r0 < total; r0 += G) {
            const int item = r0 + grp;
            const bool active = grp < G && item < total;
            const int b = active ? item / per_row : 0;
            const int col = (active ? (item % per_row) * B : 0) + tid * kXinE;
            float v[kXinE];
            if (active) {
                const __half* src = p.x + (size_t)b * p.n + col;
                const uint32_t sw = r0 == 0 ? sw0 : p.sin_bits[col >> 5] >> (col & 31);
                const uint4 raw = *reinterpret_cast<const uint4*>(src);
                const __half* hv = reinterpret_cast<const __half*>(&raw);
#pragma unroll
                for (int e = 0; e < kXinE; ++e) {
                    const float f = __half2float(hv[e]);
                    v[e] = ((sw >> e) & 1u) ? -f : f;
                }
            } else {
#pragma unroll
                for (int e = 0; e < kXinE; ++e) v[e] = 0.f;
            }
            fwht_block<kXinE>(v, B, tid, T, fw + (size_t)(grp < G ? grp : 0) * (B + B / 16), grp < G);
            if (active) {
#pragma unroll
                for (int q = 0; q < kXinE; q += 4) {
                    const __half2 lo = __floats2half2_rn(v[q] * scale, v[q + 1] * scale);
                    const __half2 hi = __floats2half2_rn(v[q + 2] * scale, v[q + 3] * scale);
                    uint2 w;
                    w.x = *reinterpret_cast<const uint32_t*>(&lo);
                    w.y = *reinterpret_cast<const uint32_t*>(&hi);
                    *reinterpret_cast<uint2*>(xs + frag_index4(col + q, b, p.batch)) = w;
                }
            }
            __syncthreads();
        }
    }
};

// One CTA per SM.  CTA i takes units [U*i/G, U*(i+1)/G) of the part (G CTAs)
// and splits them evenly over its warps; the launcher sizes the CTA so that
// every warp gets the same whole number of units (to within one), which keeps
// every SM and every warp equally loaded.  Every thread runs every phase (no
// early exit), since the in-kernel transforms use CTA barriers.
template <int CODE, int K2, int V, bool L16, bool XSMEM>
__global__ void __launch_bounds__(kGemvMaxWarps * 32, 1) trellis_gemv_kernel(GemvArgs p, GemvSmem sm) {
    extern __shared__ uint32_t smem[];
    using UL = UnitLayout<K2>;
    uint32_t* lut_smem = smem;
    __half* xs = reinterpret_cast<__half*>(smem + sm.lut_words);
    float* fw = reinterpret_cast<float*>(smem + sm.lut_words + sm.xs_words);
    const int lane = threadIdx.x & 31;
    if (uses_table(CODE)) {
        fill_lut_smem(lut_smem, p.dec.lut, p.dec.lut_entries);
        __syncthreads();
    }
    const uint32_t* lut_lane = lut_smem + lane;
    const int nb = p.dec.nb;
    const long long U = (long long)p.dec.rt * nb;
    const long long c0 = U * blockIdx.x / gridDim.x, c1 = U * (blockIdx.x + 1) / gridDim.x;
    const int wpb = blockDim.x >> 5, w = threadIdx.x >> 5;
    const long long u0 = c0 + (c1 - c0) * w / wpb, u1 = c0 + (c1 - c0) * (w + 1) / wpb;

    const int g = lane >> 2, c = lane & 3;
    const int src_lane = (lane & ~3) | ((c + 3) & 3);
    const int batch = p.batch;

    uint32_t nxt[2][K2];
    if (u0 < u1) load_unit<K2>(nxt, p.dec.words + u0 * UL::UW, lane);
    // Programmatic dependent launch: the code words, the table and the
    // sign bits are written once at create time, so they are fetched before
    // waiting for the previous kernel (the producer of x or x', the consumer
    // of the last z).
    InputTransform xin;
    if (XSMEM) xin.prepare(p);
    grid_dependency_wait();
    if (XSMEM) xin.run(p, xs, fw);
    grid_launch_dependents();

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int R = (int)(u0 / nb), j = (int)(u0 % nb);
    int curR = R;
    auto flush = [&](int tile) {
        const int row = p.row0 + tile * kRowTile + g;
        const int b0 = 2 * c, b1 = 2 * c + 1;
        if (b0 < batch) {
            atomicAdd(p.z + (size_t)b0 * p.m + row, acc[0]);
            atomicAdd(p.z + (size_t)b0 * p.m + row + 8, acc[2]);
        }
        if (b1 < batch) {
            atomicAdd(p.z + (size_t)b1 * p.m + row, acc[1]);
            atomicAdd(p.z + (size_t)b1 * p.m + row + 8, acc[3]);
        }
    };

    for (long long unit = u0; unit < u1; ++unit) {
        uint32_t cw[2][K2 + 1];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < K2; ++i) cw[h][i + 1] = nxt[h][i];
        if (unit + 1 < u1) load_unit<K2>(nxt, p.dec.words + (unit + 1) * UL::UW, lane);
        if (R != curR) {
            flush(curR);
            acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
            curR = R;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) cw[h][0] = __shfl_sync(0xffffffffu, cw[h][K2], src_lane);

        const size_t xoff = (size_t)j * 16 * batch * 4 + g * 4 + c;
        for_each_mma<CODE, K2, V, L16>(cw, p.dec.lmask, lut_lane, p.dec.qshift, [&](int u, const uint32_t(&a)[4]) {
            uint2 bv = make_uint2(0u, 0u);
            if (g < batch) {
                if (XSMEM)
                    bv = reinterpret_cast<const uint2*>(xs)[xoff + (size_t)u * batch * 4];
                else
                    bv = __ldg(p.xf + xoff + (size_t)u * batch * 4);
            }
            mma_16816(acc, a, bv.x, bv.y);
        });
        if (++j == nb) {
            j = 0;
            ++R;
        }
    }
    if (u0 < u1) flush(curR);
}

// ---- decode-GEMV over all row parts of a layer in one launch ----
// Units are numbered part by part (each part's row tiles x blocks, as in the
// single-part kernel); a warp's contiguous range may cross into the next part,
// whose bitwidth it dispatches per unit.  x' comes in the fragment layout from
// the separate input-transform kernel.
struct GemvPartArgs {
    const uint32_t* words;  // the part's words, kernel layout
    int rt;                 // row tiles
    int row0;               // first layer row
    int k2;                 // 2k: bits per two weights
};
struct GemvMultiArgs {
    GemvPartArgs part[kMaxParts];
    int nparts, nb;
    uint32_t lmask;
    int qshift;
    const uint32_t* lut;
    int lut_entries;
    const uint2* xf;
    int batch;
    float* z;
    int m;
};

// Two thread-rows of one unit at K2 = 2k into w[h][0 .. K2-1].
template <int K2>
__device__ __forceinline__ void load_unit_into(uint32_t (&w)[2][8], const uint32_t* unit_base, int lane) {
    uint32_t t[2][K2];
    load_unit<K2>(t, unit_base, lane);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < K2; ++i) w[h][i] = t[h][i];
}
__device__ __forceinline__ void load_unit_k2(uint32_t (&w)[2][8], const uint32_t* unit_base, int k2, int lane) {
    switch (k2) {
        case 2: load_unit_into<2>(w, unit_base, lane); break;
        case 3: load_unit_into<3>(w, unit_base, lane); break;
        case 4: load_unit_into<4>(w, unit_base, lane); break;
        case 5: load_unit_into<5>(w, unit_base, lane); break;
        case 6: load_unit_into<6>(w, unit_base, lane); break;
        case 7: load_unit_into<7>(w, unit_base, lane); break;
        default: load_unit_into<8>(w, unit_base, lane); break;
    }
}

// One unit at K2 = 2k: take its words from nxt, start the next unit's load
// into nxt, then decode and multiply.
template <int CODE, int K2, int V, bool L16>
__device__ __forceinline__ void gemv_unit(uint32_t (&nxt)[2][8], const uint32_t* next_base, int next_k2, int lane,
                                          int src_lane, const GemvMultiArgs& p, const uint32_t* lut_lane,
                                          size_t xoff, bool use_x, float (&acc)[4]) {
    uint32_t cw[2][K2 + 1];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < K2; ++i) cw[h][i + 1] = nxt[h][i];
    if (next_base) load_unit_k2(nxt, next_base, next_k2, lane);
#pragma unroll
    for (int h = 0; h < 2; ++h) cw[h][0] = __shfl_sync(0xffffffffu, cw[h][K2], src_lane);
    for_each_mma<CODE, K2, V, L16>(cw, p.lmask, lut_lane, p.qshift, [&](int u, const uint32_t(&a)[4]) {
        uint2 bv = make_uint2(0u, 0u);
        if (use_x) bv = __ldg(p.xf + xoff + (size_t)u * p.batch * 4);
        mma_16816(acc, a, bv.x, bv.y);
    });
}

// The unit's bitwidth picks the decoder (V = 1 has whole bitwidths only).
template <int CODE, int V, bool L16>
__device__ __forceinline__ void gemv_unit_k2(int k2, uint32_t (&nxt)[2][8], const uint32_t* next_base, int next_k2,
                                             int lane, int src_lane, const GemvMultiArgs& p,
                                             const uint32_t* lut_lane, size_t xoff, bool use_x, float (&acc)[4]) {
    switch (k2) {
        case 2: gemv_unit<CODE, 2, V, L16>(nxt, next_base, next_k2, lane, src_lane, p, lut_lane, xoff, use_x, acc); break;
        case 3: if constexpr (V == 2) gemv_unit<CODE, 3, V, L16>(nxt, next_base, next_k2, lane, src_lane, p, lut_lane, xoff, use_x, acc); break;
        case 4: gemv_unit<CODE, 4, V, L16>(nxt, next_base, next_k2, lane, src_lane, p, lut_lane, xoff, use_x, acc); break;
        case 5: if constexpr (V == 2) gemv_unit<CODE, 5, V, L16>(nxt, next_base, next_k2, lane, src_lane, p, lut_lane, xoff, use_x, acc); break;
        case 6: gemv_unit<CODE, 6, V, L16>(nxt, next_base, next_k2, lane, src_lane, p, lut_lane, xoff, use_x, acc); break;
        case 7: if constexpr (V == 2) gemv_unit<CODE, 7, V, L16>(nxt, next_base, next_k2, lane, src_lane, p, lut_lane, xoff, use_x, acc); break;
        default: gemv_unit<CODE, 8, V, L16>(nxt, next_base, next_k2, lane, src_lane, p, lut_lane, xoff, use_x, acc); break;
    }
}

template <int CODE, int V, bool L16>
__global__ void __launch_bounds__(kGemvMaxWarps * 32, 1) trellis_gemv_multi_kernel(GemvMultiArgs p) {
    extern __shared__ uint32_t smem[];
    const int lane = threadIdx.x & 31;
    if (uses_table(CODE)) {
        fill_lut_smem(smem, p.lut, p.lut_entries);
        __syncthreads();
    }
    const uint32_t* lut_lane = smem + lane;
    const int nb = p.nb;
    long long U = 0;
    for (int i = 0; i < p.nparts; ++i) U += (long long)p.part[i].rt * nb;
    const long long c0 = U * blockIdx.x / gridDim.x, c1 = U * (blockIdx.x + 1) / gridDim.x;
    const int wpb = blockDim.x >> 5, w = threadIdx.x >> 5;
    const long long u0 = c0 + (c1 - c0) * w / wpb, u1 = c0 + (c1 - c0) * (w + 1) / wpb;
    const int g = lane >> 2, c = lane & 3;
    const int src_lane = (lane & ~3) | ((c + 3) & 3);
    const int batch = p.batch;

    // walker: part pt, row tile t within it, block j
    int pt = 0;
    long long rest = u0;
    while (pt + 1 < p.nparts && rest >= (long long)p.part[pt].rt * nb) rest -= (long long)p.part[pt++].rt * nb;
    int t = (int)(rest / nb), j = (int)(rest % nb);
    auto unit_base = [&](int part, int tile, int blk) {
        return p.part[part].words + ((size_t)tile * nb + blk) * 64 * p.part[part].k2;
    };
    uint32_t nxt[2][8];
    if (u0 < u1) load_unit_k2(nxt, unit_base(pt, t, j), p.part[pt].k2, lane);
    grid_dependency_wait();  // x' from the input transform; z consumed by the last output transform
    grid_launch_dependents();

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int cur_pt = pt, cur_t = t;
    auto flush = [&](int part, int tile) {
        const int row = p.part[part].row0 + tile * kRowTile + g;
        const int b0 = 2 * c, b1 = 2 * c + 1;
        if (b0 < batch) {
            atomicAdd(p.z + (size_t)b0 * p.m + row, acc[0]);
            atomicAdd(p.z + (size_t)b0 * p.m + row + 8, acc[2]);
        }
        if (b1 < batch) {
            atomicAdd(p.z + (size_t)b1 * p.m + row, acc[1]);
            atomicAdd(p.z + (size_t)b1 * p.m + row + 8, acc[3]);
        }
    };
    for (long long unit = u0; unit < u1; ++unit) {
        // the unit after this one, for the prefetch
        int npt = pt, nt = t, nj = j + 1;
        if (nj == nb) {
            nj = 0;
            if (++nt == p.part[npt].rt && npt + 1 < p.nparts) {
                nt = 0;
                ++npt;
            }
        }
        const uint32_t* next_base = unit + 1 < u1 ? unit_base(npt, nt, nj) : nullptr;
        if (pt != cur_pt || t != cur_t) {
            flush(cur_pt, cur_t);
            acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
            cur_pt = pt;
            cur_t = t;
        }
        const size_t xoff = (size_t)j * 16 * batch * 4 + g * 4 + c;
        const bool use_x = g < batch;
        gemv_unit_k2<CODE, V, L16>(p.part[pt].k2, nxt, next_base, p.part[npt].k2, lane, src_lane, p, lut_lane, xoff,
                                   use_x, acc);
        pt = npt;
        t = nt;
        j = nj;
    }
    if (u0 < u1) flush(cur_pt, cur_t);
}

template <int CODE, int V, bool L16>
static cudaError_t launch_gemv_multi_t(const GemvMultiArgs& a, int grid, int threads, size_t smem, cudaStream_t st) {
    auto kern = trellis_gemv_multi_kernel<CODE, V, L16>;
    cudaError_t e = ensure_smem_limit<trellis_gemv_multi_kernel<CODE, V, L16>>(kGemvMaxSmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(grid), dim3(threads), smem, st, a);
}

cudaError_t launch_gemv_multi(const Layer& L, const void* xp_frag, int batch, float* z, cudaStream_t st) {
    GemvMultiArgs a;
    a.nparts = L.nparts;
    a.nb = L.n / kT;
    long long units = 0;
    for (int i = 0; i < kMaxParts; ++i) {
        const Part& pt = L.parts[i < L.nparts ? i : 0];
        a.part[i].words = L.words + pt.word_off;
        a.part[i].rt = pt.rows / kRowTile;
        a.part[i].row0 = pt.row0;
        a.part[i].k2 = pt.k2;
        if (i < L.nparts) units += (long long)a.part[i].rt * a.nb;
    }
    a.lmask = (1u << L.L) - 1u;
    a.qshift = 32 - L.Q;
    a.lut = L.lut;
    a.lut_entries = uses_table(L.code) ? (1 << L.Q) : 0;
    a.xf = (const uint2*)xp_frag;
    a.batch = batch;
    a.z = z;
    a.m = L.m;
    // one CTA per SM, warps sized so that every warp gets the same whole number of units
    const int grid = (int)(units < L.num_sms ? units : L.num_sms);
    const long long per_cta = (units + grid - 1) / grid;
    const long long per_warp = (per_cta + kGemvMaxWarps - 1) / kGemvMaxWarps;
    const int threads = (int)((per_cta + per_warp - 1) / per_warp) * 32;
    const size_t smem = (size_t)a.lut_entries * 32 * 4;
    const bool l16 = L.L == 16;
    if (L.code == kCode1MAD && L.V == 1) return l16 ? launch_gemv_multi_t<kCode1MAD, 1, true>(a, grid, threads, smem, st)
                                                    : launch_gemv_multi_t<kCode1MAD, 1, false>(a, grid, threads, smem, st);
    if (L.code == kCode3INST && L.V == 1) return l16 ? launch_gemv_multi_t<kCode3INST, 1, true>(a, grid, threads, smem, st)
                                                     : launch_gemv_multi_t<kCode3INST, 1, false>(a, grid, threads, smem, st);
    if (L.code == kCodeHYB && L.V == 1) return l16 ? launch_gemv_multi_t<kCodeHYB, 1, true>(a, grid, threads, smem, st)
                                                   : launch_gemv_multi_t<kCodeHYB, 1, false>(a, grid, threads, smem, st);
    if (L.code == kCodeHYB && L.V == 2) return l16 ? launch_gemv_multi_t<kCodeHYB, 2, true>(a, grid, threads, smem, st)
                                                   : launch_gemv_multi_t<kCodeHYB, 2, false>(a, grid, threads, smem, st);
    if (L.code == kCodeTable && !l16) return L.V == 1 ? launch_gemv_multi_t<kCodeTable, 1, false>(a, grid, threads, smem, st)
                                                      : launch_gemv_multi_t<kCodeTable, 2, false>(a, grid, threads, smem, st);
    return cudaErrorInvalidValue;
}

// ---- qlinear_decode: one warp per unit, fp16 W_hat row-major ----
template <int CODE, int K2, int V, bool L16>
__global__ void __launch_bounds__(256) trellis_decode_kernel(DecodeArgs p, __half* __restrict__ w_hat, int n, int row0) {
    extern __shared__ uint32_t lut_smem[];
    using UL = UnitLayout<K2>;
    const int lane = threadIdx.x & 31;
    if (uses_table(CODE)) {
        fill_lut_smem(lut_smem, p.lut, p.lut_entries);
        __syncthreads();
    }
    const uint32_t* lut_lane = lut_smem + lane;
    const int g = lane >> 2, c = lane & 3;
    const int src_lane = (lane & ~3) | ((c + 3) & 3);
    const long long U = (long long)p.rt * p.nb;
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long unit = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); unit < U;
         unit += nwarps) {
        uint32_t w[2][K2];
        load_unit<K2>(w, p.words + unit * UL::UW, lane);
        uint32_t cw[2][K2 + 1];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int i = 0; i < K2; ++i) cw[h][i + 1] = w[h][i];
            cw[h][0] = __shfl_sync(0xffffffffu, w[h][K2 - 1], src_lane);
        }
        const int R = (int)(unit / p.nb), j = (int)(unit % p.nb);
        for_each_mma<CODE, K2, V, L16>(cw, p.lmask, lut_lane, p.qshift, [&](int u, const uint32_t(&a)[4]) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const size_t row = (size_t)row0 + R * kRowTile + 8 * h + g;
                uint2* dst = (uint2*)(w_hat + row * n + (size_t)j * kT + 64 * c + 4 * u);
                *dst = make_uint2(a[h], a[2 + h]);
            }
        });
    }
}

// ---- qlinear_eval_code ----
template <int CODE, int V>
__global__ void eval_code_kernel(const uint32_t* __restrict__ states, int count, uint32_t lmask, int qshift,
                                 const uint32_t* __restrict__ lut, int lut_entries, __half* __restrict__ out) {
    extern __shared__ uint32_t lut_smem[];
    const int lane = threadIdx.x & 31;
    if (uses_table(CODE)) {
        fill_lut_smem(lut_smem, lut, lut_entries);
        __syncthreads();
    }
    const uint32_t* lut_lane = lut_smem + lane;
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if constexpr (V == 2) {
        if (t < count) ((uint32_t*)out)[t] = code_v2<CODE>(states[t] & lmask, lut_lane, qshift);
    } else {
        const int i0 = 2 * t;
        if (i0 >= count) return;
        const uint32_t s0 = states[i0] & lmask;
        const uint32_t s1 = (i0 + 1 < count) ? (states[i0 + 1] & lmask) : s0;
        const uint32_t pr = code_pair<CODE>(s0, s1, lut_lane, qshift);
        const unsigned short* hv = (const unsigned short*)&pr;
        ((unsigned short*)out)[i0] = hv[0];
        if (i0 + 1 < count) ((unsigned short*)out)[i0 + 1] = hv[1];
    }
}

// ---- dispatch ----
template <template <int, int, int, bool> class F, bool L16, typename... Args>
static cudaError_t dispatch_l(int code, int k2, int V, Args&&... args);

template <template <int, int, int, bool> class F, typename... Args>
static cudaError_t dispatch(int code, int k2, int V, bool l16, Args&&... args) {
    return l16 ? dispatch_l<F, true>(code, k2, V, args...) : dispatch_l<F, false>(code, k2, V, args...);
}

// (code, k2 = 2k, V) -> the kernel instance.  V = 1 takes whole bitwidths
// (k2 even), V = 2 also half ones; the table code has no L = 16 instance
// (its codebook holds at most 2^9 entries).
template <template <int, int, int, bool> class F, int CODE, int V, bool L16, typename... Args>
static cudaError_t dispatch_k2(int k2, Args&&... args) {
    switch (k2) {
        case 2: return F<CODE, 2, V, L16>::run(args...);
        case 4: return F<CODE, 4, V, L16>::run(args...);
        case 6: return F<CODE, 6, V, L16>::run(args...);
        case 8: return F<CODE, 8, V, L16>::run(args...);
    }
    if constexpr (V == 2) {
        switch (k2) {
            case 3: return F<CODE, 3, V, L16>::run(args...);
            case 5: return F<CODE, 5, V, L16>::run(args...);
            case 7: return F<CODE, 7, V, L16>::run(args...);
        }
    }
    return cudaErrorInvalidValue;
}

template <template <int, int, int, bool> class F, bool L16, typename... Args>
static cudaError_t dispatch_l(int code, int k2, int V, Args&&... args) {
    if (code == kCode1MAD && V == 1) return dispatch_k2<F, kCode1MAD, 1, L16>(k2, args...);
    if (code == kCode3INST && V == 1) return dispatch_k2<F, kCode3INST, 1, L16>(k2, args...);
    if (code == kCodeHYB && V == 1) return dispatch_k2<F, kCodeHYB, 1, L16>(k2, args...);
    if (code == kCodeHYB && V == 2) return dispatch_k2<F, kCodeHYB, 2, L16>(k2, args...);
    if constexpr (!L16) {
        if (code == kCodeTable && V == 1) return dispatch_k2<F, kCodeTable, 1, false>(k2, args...);
        if (code == kCodeTable && V == 2) return dispatch_k2<F, kCodeTable, 2, false>(k2, args...);
    }
    return cudaErrorInvalidValue;
}

static DecodeArgs make_decode_args(const Layer& L, const Part& part) {
    DecodeArgs d;
    d.words = L.words + part.word_off;
    d.rt = part.rows / kRowTile;
    d.nb = L.n / kT;
    d.lmask = (1u << L.L) - 1u;
    d.qshift = 32 - L.Q;
    d.lut = L.lut;
    d.lut_entries = uses_table(L.code) ? (1 << L.Q) : 0;
    return d;
}

// The in-kernel input transform has instances for L = 16 and for the table code.
template <int CODE, int K2, int V, bool L16>
struct GemvLaunch {
    static cudaError_t run(const GemvArgs& a, const GemvSmem& sm, bool xsmem, int grid, int threads,
                           cudaStream_t st) {
        const size_t smem = (size_t)(sm.lut_words + sm.xs_words + sm.fw_words) * 4;
        if (xsmem) {
            if constexpr (L16 || CODE == kCodeTable) {
                auto kern = trellis_gemv_kernel<CODE, K2, V, L16, true>;
                cudaError_t e = ensure_smem_limit<trellis_gemv_kernel<CODE, K2, V, L16, true>>(kGemvMaxSmem);
                if (e != cudaSuccess) return e;
                return launch_pdl(kern, dim3(grid), dim3(threads), smem, st, a, sm);
            } else {
                return cudaErrorInvalidValue;
            }
        }
        auto kern = trellis_gemv_kernel<CODE, K2, V, L16, false>;
        cudaError_t e = ensure_smem_limit<trellis_gemv_kernel<CODE, K2, V, L16, false>>(kGemvMaxSmem);
        if (e != cudaSuccess) return e;
        return launch_pdl(kern, dim3(grid), dim3(threads), smem, st, a, sm);
    }
};

// CTA shape: one CTA per SM, warps sized so every warp gets the same whole
// number of units.  The input transform runs in-kernel (each CTA computes
// x' into its shared memory while its first code words are in flight) when
// x is small; otherwise a separate kernel writes x' to global memory.
GemvPlan plan_gemv(const Layer& L, const Part& part, int batch) {
    GemvPlan pl;
    const long long nb = L.n / kT;
    const long long units = (long long)(part.rows / kRowTile) * nb;
    pl.grid = (int)(units < L.num_sms ? units : L.num_sms);
    const long long per_cta = (units + pl.grid - 1) / pl.grid;
    const long long per_warp = (per_cta + kGemvMaxWarps - 1) / kGemvMaxWarps;
    int threads = (int)((per_cta + per_warp - 1) / per_warp) * 32;
    const int lut_words = uses_table(L.code) ? (32 << L.Q) : 0;
    const int budget = kGemvMaxSmem / 4 - lut_words;
    const int t_in = L.B_n / kXinE;
    const int xs_words = batch * L.n / 2;
    pl.xsmem = (L.L == 16 || L.code == kCodeTable) && L.nparts == 1 && (long long)batch * L.n <= kFuseInElems &&
               t_in <= kGemvMaxWarps * 32;
    int fw = 0;
    pl.groups_in = 0;
    const int threads_decode = threads;
    if (pl.xsmem) {
        if (threads < t_in) threads = t_in;
        // thread groups of B_n/kXinE threads; a group of more than a warp needs
        // its own FWHT scratch (B_n + B_n/16 floats)
        int g = threads / t_in;
        const int work = batch * (L.n / L.B_n);
        if (g > work) g = work;
        if (g < 1) g = 1;
        if (t_in > 32) {
            const int per = L.B_n + L.B_n / 16;
            while (g > 1 && xs_words + g * per > budget) --g;
            fw = g * per;
        }
        pl.groups_in = g;
        if (xs_words + fw > budget) pl.xsmem = false, fw = 0, pl.groups_in = 0;
        // every CTA runs the transform before its first MMA: only worth it when
        // it takes a single round (one group per (batch row, Hadamard block))
        if (g < work) pl.xsmem = false, fw = 0, pl.groups_in = 0;
        if (!pl.xsmem) threads = threads_decode;
    }
    pl.threads = threads;
    pl.sm.lut_words = lut_words;
    pl.sm.xs_words = pl.xsmem ? xs_words : 0;
    pl.sm.fw_words = fw;
    return pl;
}

cudaError_t launch_gemv(const Layer& L, const Part& part, const GemvPlan& pl, const void* x, const void* xp_frag,
                        int batch, float* z, cudaStream_t st) {
    GemvArgs a;
    a.dec = make_decode_args(L, part);
    a.xf = (const uint2*)xp_frag;
    a.batch = batch;
    a.z = z;
    a.m = L.m;
    a.row0 = part.row0;
    a.x = (const __half*)x;
    a.sin_bits = L.sin_bits;
    a.n = L.n;
    a.B_n = L.B_n;
    a.groups_in = pl.groups_in;
    return dispatch<GemvLaunch>(L.code, part.k2, L.V, L.L == 16, a, pl.sm, pl.xsmem, pl.grid, pl.threads, st);
}

template <int CODE, int K2, int V, bool L16>
struct DecodeLaunch {
    static cudaError_t run(const DecodeArgs& d, __half* w, int n, int row0, int grid, cudaStream_t st) {
        const size_t smem = (size_t)d.lut_entries * 32 * 4;
        auto kern = trellis_decode_kernel<CODE, K2, V, L16>;
        if (smem > 48 * 1024) {
            cudaError_t e = ensure_smem_limit<trellis_decode_kernel<CODE, K2, V, L16>>(32 * 512 * 4);
            if (e != cudaSuccess) return e;
        }
        kern<<<grid, 256, smem, st>>>(d, w, n, row0);
        return cudaGetLastError();
    }
};

cudaError_t launch_decode(const Layer& L, const Part& part, void* w_hat, cudaStream_t st) {
    DecodeArgs d = make_decode_args(L, part);
    const long long units = (long long)d.rt * d.nb;
    long long grid = (units + 7) / 8;
    if (grid > (long long)L.num_sms * 8) grid = (long long)L.num_sms * 8;
    return dispatch<DecodeLaunch>(L.code, part.k2, L.V, L.L == 16, d, (__half*)w_hat, L.n, part.row0, (int)grid, st);
}

template <int CODE, int K2, int V, bool L16>
struct EvalLaunch {
    static cudaError_t run(const uint32_t* states, int count, uint32_t lmask, int qshift, const uint32_t* lut,
                           int entries, __half* out, cudaStream_t st) {
        // one instance per (code, V) suffices: the code ignores k and L
        if (K2 != 2 || L16 == (CODE == kCodeTable)) return cudaErrorInvalidValue;
        const size_t smem = (size_t)entries * 32 * 4;
        auto kern = eval_code_kernel<CODE, V>;
        if (smem > 48 * 1024) {
            cudaError_t e = ensure_smem_limit<eval_code_kernel<CODE, V>>(32 * 512 * 4);
            if (e != cudaSuccess) return e;
        }
        const int items = V == 2 ? count : (count + 1) / 2;
        kern<<<(items + 255) / 256, 256, smem, st>>>(states, count, lmask, qshift, lut, entries, out);
        return cudaGetLastError();
    }
};

cudaError_t launch_eval_code(int code, int L, int V, int Q, const uint32_t* lut_words, const uint32_t* states,
                             int count, void* out, cudaStream_t st) {
    const uint32_t lmask = (1u << L) - 1u;
    const int entries = uses_table(code) ? (1 << Q) : 0;
    return dispatch<EvalLaunch>(code, 2, V, code != kCodeTable, states, count, lmask, 32 - Q, lut_words, entries,
                                (__half*)out, st);
}

}  // namespace qlk
