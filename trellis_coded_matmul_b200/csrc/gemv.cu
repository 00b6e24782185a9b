// gemv.cu -- fused trellis decode + matrix-vector product for batch <= 8 (the
// whole forward in one kernel when x is small), and the decode / eval_code
// test kernels built on the same device functions.
//
// Decode follows the QTIP discussion: the bitshift trellis makes every state
// a window of the stored bits, so a lane can decode any run of steps on its
// own ("the bitshift trellis also enables parallel decoding"), and the codes
// are computed in INT32 ALU (1MAD, 3INST) or with a small table in banked
// shared memory (HYB, and the palette's table code).  Decoded weights stay in
// registers: they are the A operand of m16n8k16 half-precision MMAs whose B
// operand is x' (batch padded to 8 columns) and whose fp32 accumulators hold
// 16 rows x 8 batch columns.
//
// One 32-bit A word per trellis step (xstep.cuh gives the matching B words):
//   V = 2: the code's table word, the step's two fp16 weights;
//   V = 1: the code's "split" word, two fp16 halves whose sum is the weight,
//          so the MMA adds them (h0 x' + h1 x' = (h0 + h1) x') and the decode
//          spends no instruction on the sum or on pairing weights:
//            3INST  the masked word m itself (value = m.lo + m.hi);
//            1MAD   one dp4a whose accumulator puts 1536 + d in the low half
//                   and -1536 in the high half (sum d, the byte sum minus
//                   510); the factor C1 is applied to z in the epilogue;
//            HYB / table  the table word (value in the low half, 0 above).
//   The product then carries the code value before its rounding to fp16
//   (qlinear_decode still returns the fp16-rounded values); the difference
//   is a relative 2^-12 per weight, independent from weight to weight.
//
// Work split: the m x n matrix is a grid of units (16 rows x 256 columns),
// numbered part by part, row tile by row tile.  Every warp of the grid takes
// one contiguous, equally sized range of units, accumulates while the row
// tile is unchanged and adds its partial sums into z with atomics when it
// moves on.  Lane (g, c) decodes rows g and g + 8 of a unit, one contiguous
// run of 64 / V trellis steps of each (see layout.cuh).
//
// Forward in one launch (batch <= 8):
//   1. code words of the first unit in flight, then the wait for the previous
//      kernel (programmatic dependent launch);
//   2. x' = H_n diag(s_in) x into shared memory at batch 1 when one thread
//      group holds a Hadamard block (every CTA computes all of it), else read
//      from the input-transform kernel's output;
//   3. decode + MMA over the warp's units, atomics into z;
//   4. when the whole output is small (batch * m <= 256), the output
//      transform (QuIP# page, Fig. 2; QTIP discussion, "Incoherence
//      Processing (W2)"): a CTA adds the units it finished in each output
//      Hadamard block to that block's ticket; the CTA that completes a ticket
//      owns the block, reads its z, applies y = alpha diag(s_out) H_B z,
//      writes y and returns z and the ticket to zero for the next forward.
//      No CTA waits for another.  Otherwise the output-transform kernel
//      follows.
#include <cuda_fp16.h>

#include "codes.cuh"
#include "fwht.cuh"
#include "internal.h"
#include "layout.cuh"
#include "xstep.cuh"

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


__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// (qlinear_decode uses code_pair / code_v2 of codes.cuh, which round each
// value to fp16; the forward's MMAs take the split words below.)

// The forward's decode ends with one instruction per step word that turns a
// "pre" word into the MMA's A word: 3INST (pre & MASK) ^ XOR; 1MAD one dp4a
// giving {1536 + d, -1536}; HYB the table word xor the hashed state's bit 15;
// the table code none.  That instruction runs inside the MMA's asm block, so
// the finished words are allocated as the MMA's operand registers (computed
// into arbitrary registers they would be copied into an aligned quad).
template <int CODE, int V>
__device__ __forceinline__ void step_pre(uint32_t s, const uint32_t* lut_lane, int qshift, uint32_t& pre,
                                         uint32_t& aux) {
    if constexpr (CODE == kCode1MAD) {
        pre = kA1MAD * s + kB1MAD;
    } else if constexpr (CODE == kCode3INST) {
        pre = kA3INST * s + kB3INST;
    } else if constexpr (CODE == kCodeHYB) {
        aux = kAHYB * s + kBHYB;
        pre = lut_lane[(aux >> qshift) * 32u];
    } else {
        pre = lut_lane[s * 32u];
    }
}

// 1MAD: {1536 + d, -1536} as two halves (0x6600 is 1536.0; 0xE600 is -1536.0).
constexpr uint32_t kDp4aSplitAcc = 0xE6006600u - 510u;
constexpr float kC1 = 443.0f / 65536.0f;  // the 1MAD scale

template <int CODE>
__device__ __forceinline__ void mma_step(float (&d)[4], const uint32_t (&pre)[4], const uint32_t (&aux)[4], uint32_t b0,
                                         uint32_t b1) {
#define QLK_MMA_TAIL \
    "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {a0,a1,a2,a3}, {%8,%9}, {%0,%1,%2,%3};\n\t}"
    if constexpr (CODE == kCode3INST) {
        asm volatile(
            "{\n\t.reg .b32 a0, a1, a2, a3;\n\t"
            "lop3.b32 a0, %4, %10, %11, 0x6a;\n\tlop3.b32 a1, %5, %10, %11, 0x6a;\n\t"
            "lop3.b32 a2, %6, %10, %11, 0x6a;\n\tlop3.b32 a3, %7, %10, %11, 0x6a;\n\t" QLK_MMA_TAIL
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(pre[0]), "r"(pre[1]), "r"(pre[2]), "r"(pre[3]), "r"(b0), "r"(b1), "n"(kMask3INST), "n"(kXor3INST));
    } else if constexpr (CODE == kCode1MAD) {
        asm volatile(
            "{\n\t.reg .b32 a0, a1, a2, a3;\n\t"
            "dp4a.u32.u32 a0, %4, %10, %11;\n\tdp4a.u32.u32 a1, %5, %10, %11;\n\t"
            "dp4a.u32.u32 a2, %6, %10, %11;\n\tdp4a.u32.u32 a3, %7, %10, %11;\n\t" QLK_MMA_TAIL
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(pre[0]), "r"(pre[1]), "r"(pre[2]), "r"(pre[3]), "r"(b0), "r"(b1), "n"(0x01010101u),
              "n"(kDp4aSplitAcc));
    } else if constexpr (CODE == kCodeHYB) {
        asm volatile(
            "{\n\t.reg .b32 a0, a1, a2, a3;\n\t"
            "lop3.b32 a0, %4, %10, %14, 0x78;\n\tlop3.b32 a1, %5, %11, %14, 0x78;\n\t"
            "lop3.b32 a2, %6, %12, %14, 0x78;\n\tlop3.b32 a3, %7, %13, %14, 0x78;\n\t" QLK_MMA_TAIL
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(pre[0]), "r"(pre[1]), "r"(pre[2]), "r"(pre[3]), "r"(b0), "r"(b1), "r"(aux[0]), "r"(aux[1]),
              "r"(aux[2]), "r"(aux[3]), "n"(0x8000u));
    } else {
        mma_16816(d, pre, b0, b1);
    }
#undef QLK_MMA_TAIL
}

// Decode + MMA of one unit: lane (g, c) holds, for thread-row h (row g + 8h),
// the 32 bits before its run in cw[h][0] and its run's K2 words in
// cw[h][1..K2].  MMA u takes the lane's steps 2u (K slots 2c, 2c+1) and 2u+1
// (slots 2c+8, 2c+9) of rows g (a[0], a[2]) and g + 8 (a[1], a[3]); its B
// words are word 2*(u%2) and 2*(u%2)+1 of the 16-byte group u/2.  When 16 is a
// multiple of kV, the windows of steps t and t + 16/kV are the two halves of
// one funnel shift, which pairs MMA u with MMA u + 8/kV.
template <int CODE, int K2, int V, bool L16>
struct StepMMAs {
    static constexpr int kV = K2 * V / 2;
    static constexpr bool kPair = (16 % kV) == 0;
    static constexpr int MP = kPair ? 8 / kV : 0;   // MMA distance of paired windows
    static constexpr bool kQuad = kPair && MP >= 2;  // an iteration covers MMAs u, u+1, u+MP, u+MP+1
    static constexpr int NM = 32 / V;                // MMAs per unit
    static constexpr int NW = K2 + 1;

    static __device__ __forceinline__ void run(const uint32_t (&cw)[2][NW], uint32_t lmask, const uint32_t* lut_lane,
                                               int qshift, const uint4* xsrc, int xstride, bool use_x,
                                               float (&acc)[2][4]) {
#pragma unroll
        for (int u = 0; u < NM; u += 2) {
            if (kQuad && ((u / (kQuad ? MP : 1)) & 1)) continue;  // produced together with MMAs u - MP, u - MP + 1
            uint32_t pre[4][4], aux[4][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = 2 * u + e;  // step of MMA u + e/2, register 2 (e % 2) + h
                    const int q = e >> 1, r = 2 * (e & 1) + h;
                    if constexpr (kQuad) {
                        uint32_t s, s2;
                        state_pair<kV, L16>(cw[h], t, lmask, s, s2);
                        step_pre<CODE, V>(s, lut_lane, qshift, pre[q][r], aux[q][r]);
                        step_pre<CODE, V>(s2, lut_lane, qshift, pre[2 + q][r], aux[2 + q][r]);
                    } else if constexpr (kPair) {  // MP == 1: step t pairs with step t + 2, of MMA u + 1
                        if (e < 2) {
                            uint32_t s, s2;
                            state_pair<kV, L16>(cw[h], t, lmask, s, s2);
                            step_pre<CODE, V>(s, lut_lane, qshift, pre[0][r], aux[0][r]);
                            step_pre<CODE, V>(s2, lut_lane, qshift, pre[1][r], aux[1][r]);
                        }
                    } else {
                        step_pre<CODE, V>(state_one<kV, L16>(cw[h], t, lmask), lut_lane, qshift, pre[q][r], aux[q][r]);
                    }
                }
            }
            uint4 b0 = make_uint4(0u, 0u, 0u, 0u), b1 = b0;
            if (use_x) {
                b0 = xsrc[(u >> 1) * xstride];
                if (kQuad) b1 = xsrc[((u + MP) >> 1) * xstride];
            }
            // two accumulators: two dependent MMA chains of half the length
            mma_step<CODE>(acc[0], pre[0], aux[0], b0.x, b0.y);
            mma_step<CODE>(acc[1], pre[1], aux[1], b0.z, b0.w);
            if (kQuad) {
                mma_step<CODE>(acc[0], pre[2], aux[2], b1.x, b1.y);
                mma_step<CODE>(acc[1], pre[3], aux[3], b1.z, b1.w);
            }
        }
    }
};

// The E8 code (V = 8): each 16-bit step gives 8 weights, four fp16 pairs;
// step t of the lane's run (the high half of word 1 + t/2 when t is even, the
// low half when odd) feeds MMAs 2t (pairs 0, 1) and 2t + 1 (pairs 2, 3), whose
// B words are the 16-byte group t.
template <int K2, bool L16>
struct StepMMAs<kCodeE8P, K2, 8, L16> {
    static constexpr int NW = K2 + 1;
    static __device__ __forceinline__ void run(const uint32_t (&cw)[2][NW], uint32_t, const uint32_t* lut_lane, int,
                                               const uint4* xsrc, int xstride, bool use_x, float (&acc)[2][4]) {
        static_assert(K2 == 4, "the E8 code stores 16 bits per 8 weights");
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            uint32_t p0[4], p1[4];  // rows g and g + 8
            const uint32_t w0 = cw[0][1 + t / 2], w1 = cw[1][1 + t / 2];
            e8p_pairs((t & 1) ? (w0 & 0xFFFFu) : (w0 >> 16), lut_lane, p0);
            e8p_pairs((t & 1) ? (w1 & 0xFFFFu) : (w1 >> 16), lut_lane, p1);
            uint4 b = make_uint4(0u, 0u, 0u, 0u);
            if (use_x) b = xsrc[t * xstride];
            const uint32_t a0[4] = {p0[0], p1[0], p0[1], p1[1]};
            const uint32_t a1[4] = {p0[2], p1[2], p0[3], p1[3]};
            mma_16816(acc[0], a0, b.x, b.y);
            mma_16816(acc[1], a1, b.z, b.w);
        }
    }
};

struct GemvPartArgs {
    const uint32_t* words;  // the part's words, kernel layout
    int rt;                 // row tiles
    int row0;               // first layer row
    int k2;                 // 2k: bits per two weights
};

struct GemvArgs {
    GemvPartArgs part[kMaxParts];
    int nparts;
    int nb;                 // 256-column blocks per row
    long long units;        // (row tile, block) units over all parts
    uint32_t lmask;         // (1 << L) - 1
    int qshift;             // HYB: 32 - Q
    const uint32_t* lut;    // HYB / table code / E8 shapes: 2^Q words
    int lut_entries;
    int batch;              // 1..8
    int m, n;
    const uint4* xstep;     // x' step words from the input-transform kernel (x_e == 0)
    const __half* x;        // x_e > 0: the input, transformed by every CTA into shared memory
    const uint32_t* sin_bits;
    int B_n;
    int x_e;                // entries per thread of that transform (8 or 16), 0: x' from xstep
    int xs_word0;           // first shared-memory word of x' (after the code table)
    float* z;               // [batch][m], all-zero on entry and on exit
    int* tickets;           // [m / B_m], all-zero on entry and on exit
    int B_m;
    const uint32_t* sout_bits;
    float out_scale;        // alpha (times C1 for 1MAD) / sqrt(B_m)
    void* y;                // [batch][m]
    int y_f16;
    int fuse_out;           // the output transform runs in this kernel (else a separate kernel after it)
    int smem_floats;        // dynamic shared memory of the launch, in 4-byte words
};

// Load one unit's K2 words per thread-row into w[h][0 .. K2-1] (runtime K2 <= 8).
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
// into nxt (NXW = K2: a one-part layer; NXW = 8: the next unit's own K2),
// then decode and multiply.
template <int CODE, int K2, int V, bool L16, int NXW>
__device__ __forceinline__ void gemv_unit(uint32_t (&nxt)[2][NXW], const uint32_t* next_base, int next_k2, int lane,
                                          int src_lane, const GemvArgs& p, const uint32_t* lut_lane, const uint4* xsrc,
                                          int xstride, bool use_x, float (&acc)[2][4]) {
    uint32_t cw[2][K2 + 1];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < K2; ++i) cw[h][i + 1] = nxt[h][i];
    if (next_base) {
        // NXW = 8 holds any bitwidth: the next unit may belong to a part of
        // another bitwidth (it follows its own next_k2); else a one-part layer
        if constexpr (NXW == 8)
            load_unit_k2(nxt, next_base, next_k2, lane);
        else
            load_unit<K2>(nxt, next_base, lane);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) cw[h][0] = __shfl_sync(0xffffffffu, cw[h][K2], src_lane);
    StepMMAs<CODE, K2, V, L16>::run(cw, p.lmask, lut_lane, p.qshift, xsrc, xstride, use_x, acc);
}

// The unit's bitwidth picks the decoder (V = 1 has whole bitwidths only).
template <int CODE, int V, bool L16>
__device__ __forceinline__ void gemv_unit_k2(int k2, uint32_t (&nxt)[2][8], const uint32_t* next_base, int next_k2,
                                             int lane, int src_lane, const GemvArgs& p, const uint32_t* lut_lane,
                                             const uint4* xsrc, int xstride, bool use_x, float (&acc)[2][4]) {
#define QLK_UNIT(K) gemv_unit<CODE, K, V, L16, 8>(nxt, next_base, next_k2, lane, src_lane, p, lut_lane, xsrc, \
                                                         xstride, use_x, acc)
    switch (k2) {
        case 2: QLK_UNIT(2); break;
        case 3: if constexpr (V == 2) QLK_UNIT(3); break;
        case 4: QLK_UNIT(4); break;
        case 5: if constexpr (V == 2) QLK_UNIT(5); break;
        case 6: QLK_UNIT(6); break;
        case 7: if constexpr (V == 2) QLK_UNIT(7); break;
        default: QLK_UNIT(8); break;
    }
#undef QLK_UNIT
}

// The output transform of Hadamard block hb for every batch row (as many rows
// at once as `buf` holds): y = out_scale * s_out (H z); z returns to zero.
// The block's B/32 sign words are staged in shared memory after the rows.
__device__ __forceinline__ void output_transform_block(const GemvArgs& p, int hb, float* buf) {
    const int B = p.B_m, m = p.m;
    const int w0 = (hb * B) >> 5, nw = ((hb * B + B - 1) >> 5) - w0 + 1;  // sign words of the block's rows
    int rows = (p.smem_floats - nw) / (B + B / 16);
    rows = rows < 1 ? 1 : (rows > p.batch ? p.batch : rows);
    uint32_t* sgn = reinterpret_cast<uint32_t*>(buf + rows * (B + B / 16));
    for (int i = threadIdx.x; i < nw; i += blockDim.x) sgn[i] = p.sout_bits[w0 + i];
    // (the barrier after the first load phase makes the sign words visible)
    for (int b0 = 0; b0 < p.batch; b0 += rows) {
        const int nr = p.batch - b0 < rows ? p.batch - b0 : rows;
        fwht_blocks_smem<2>(
            buf, nr * B, B,
            [&](int i, float (&v)[8]) {
                const int bb = b0 + i / B, r = hb * B + (i % B);
                float4* zp = reinterpret_cast<float4*>(p.z + (size_t)bb * m + r);
                const float4 t0 = __ldcg(zp), t1 = __ldcg(zp + 1);
                __stcg(zp, make_float4(0.f, 0.f, 0.f, 0.f));
                __stcg(zp + 1, make_float4(0.f, 0.f, 0.f, 0.f));
                v[0] = t0.x, v[1] = t0.y, v[2] = t0.z, v[3] = t0.w;
                v[4] = t1.x, v[5] = t1.y, v[6] = t1.z, v[7] = t1.w;
            },
            [&](int i, const float (&v)[4]) {
                const int bb = b0 + i / B, r = hb * B + (i % B);
                const uint32_t sw = sgn[(r >> 5) - w0] >> (r & 31);  // r % 4 == 0: bits r .. r+3 in one word
                float o[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) o[q] = ((sw >> q) & 1u) ? -v[q] * p.out_scale : v[q] * p.out_scale;
                if (p.y_f16) {
                    *reinterpret_cast<uint2*>((__half*)p.y + (size_t)bb * m + r) =
                        make_uint2(half2_bits(o[0], o[1]), half2_bits(o[2], o[3]));
                } else {
                    *reinterpret_cast<float4*>((float*)p.y + (size_t)bb * m + r) = make_float4(o[0], o[1], o[2], o[3]);
                }
            });
        __syncthreads();
    }
}

// After the CTA's last atomics into z: count its units into the tickets of the
// Hadamard blocks they touch and transform the blocks it completes.  The
// CTA's units are [c0, c1) of the row-tile-major walk (unit = T nb + j, T the
// global row tile).
constexpr int kEpiOwnedMax = 32;
__device__ __forceinline__ void output_epilogue(const GemvArgs& p, float* buf, long long c0, long long c1) {
    __shared__ int owned[kEpiOwnedMax];
    __shared__ int n_owned;
    __threadfence();  // this thread's atomics into z are visible device-wide before the ticket
    __syncthreads();
    if (c0 >= c1) return;  // uniform over the CTA
    const long long uph = (long long)(p.B_m / kRowTile) * p.nb;  // units per output Hadamard block
    const int hb_first = (int)(c0 / uph), hb_last = (int)((c1 - 1) / uph);
    for (int hb0 = hb_first; hb0 <= hb_last; hb0 += kEpiOwnedMax) {
        if (threadIdx.x == 0) {
            int cnt = 0;
            for (int hb = hb0; hb <= hb_last && hb < hb0 + kEpiOwnedMax; ++hb) {
                const long long lo = c0 > hb * uph ? c0 : hb * uph;
                const long long hi = c1 < (hb + 1) * uph ? c1 : (hb + 1) * uph;
                const int mine = (int)(hi - lo);
                const int prev = atomicAdd(p.tickets + hb, mine);
                if ((long long)(prev + mine) == uph) {
                    owned[cnt++] = hb;
                    p.tickets[hb] = 0;  // every unit of the block is in: no other CTA touches this ticket again
                }
            }
            n_owned = cnt;
            __threadfence();  // the other CTAs' z sums, published before their tickets, are read after this
        }
        __syncthreads();
        const int cnt = n_owned;
        for (int i = 0; i < cnt; ++i) output_transform_block(p, owned[i], buf);
        __syncthreads();
    }
}

// One CTA per SM (at most).  CTA i takes units [U*i/G, U*(i+1)/G) of the
// row-tile-major walk (unit = T nb + j over the global row tile T; partial
// sums accumulate over the blocks of a tile) and splits them evenly over its
// warps; x' comes from the input-transform kernel.  K2F: the bitwidth of a
// one-part layer (decoder fixed at compile time), 0 for several parts
// (decoder per unit).  Every thread runs the epilogue, which uses CTA
// barriers.
template <int CODE, int V, bool L16, int K2F>
__global__ void __launch_bounds__(kGemvMaxWarps * 32, 1) trellis_gemv_kernel(GemvArgs p) {
    extern __shared__ __align__(16) uint32_t smem[];
    constexpr int NXW = K2F ? K2F : 8;
    constexpr int VX = V == 1 ? 1 : 2;  // x' layout: one column per B word (V = 1) or two
    const int lane = threadIdx.x & 31;
    if (uses_table(CODE)) fill_lut_smem(smem, p.lut, p.lut_entries);
    const uint32_t* lut_lane = smem + lane;

    const int nb = p.nb;
    const long long U = p.units;
    const long long c0 = U * blockIdx.x / gridDim.x, c1 = U * (blockIdx.x + 1) / gridDim.x;
    const int wpb = blockDim.x >> 5, w = threadIdx.x >> 5;
    const long long u0 = c0 + (c1 - c0) * w / wpb, u1 = c0 + (c1 - c0) * (w + 1) / wpb;
    const int g = lane >> 2, c = lane & 3;
    const int src_lane = (lane & ~3) | ((c + 3) & 3);
    const int batch = p.batch;

    // walker over (part, row tile in the part, block)
    long long Tg = u0 / nb;
    int j = (int)(u0 % nb);
    int pt = 0;
    while (pt + 1 < p.nparts && Tg >= p.part[pt].rt) Tg -= p.part[pt++].rt;
    int t = (int)Tg;
    auto unit_base = [&](int part, int tile, int blk) {
        return p.part[part].words + ((size_t)tile * nb + blk) * 64 * p.part[part].k2;
    };
    // Programmatic dependent launch: the code words, the tables and the sign
    // bits are written once at create time, so the first unit's words are
    // fetched before waiting for the previous kernel (the producer of x or x',
    // the previous forward that used z).
    uint32_t nxt[2][NXW];
    if (u0 < u1) {
        if constexpr (K2F != 0)
            load_unit<K2F>(nxt, unit_base(pt, t, j), lane);
        else
            load_unit_k2(nxt, unit_base(pt, t, j), p.part[pt].k2, lane);
    }
    grid_dependency_wait();
    if (uses_table(CODE)) __syncthreads();
    grid_launch_dependents();

    const uint4* xbase = p.xstep;
    if (p.x_e) {  // x' of the whole batch in shared memory, computed by this CTA (x was just written)
        uint32_t* xs = smem + p.xs_word0;
        float* scratch = reinterpret_cast<float*>(xs + (size_t)batch * p.n / VX);
        if (p.x_e == 8)
            xstep_transform_cta<VX, 8>(p.x, p.n, p.B_n, p.sin_bits, batch, xs, scratch);
        else
            xstep_transform_cta<VX, 16>(p.x, p.n, p.B_n, p.sin_bits, batch, xs, scratch);
        xbase = reinterpret_cast<const uint4*>(xs);
    }
    const int xstride = batch * 4;  // uint4 groups between consecutive u2
    const bool use_x = g < batch;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    int cur_pt = pt, cur_t = t;
    auto flush = [&](int part, int tile) {
        const int row = p.part[part].row0 + tile * kRowTile + g;
        const int b0 = 2 * c, b1 = 2 * c + 1;
        if (b0 < batch) {
            atomicAdd(p.z + (size_t)b0 * p.m + row, acc[0][0] + acc[1][0]);
            atomicAdd(p.z + (size_t)b0 * p.m + row + 8, acc[0][2] + acc[1][2]);
        }
        if (b1 < batch) {
            atomicAdd(p.z + (size_t)b1 * p.m + row, acc[0][1] + acc[1][1]);
            atomicAdd(p.z + (size_t)b1 * p.m + row + 8, acc[0][3] + acc[1][3]);
        }
    };
    for (long long unit = u0; unit < u1; ++unit) {
        int npt = pt, nt = t, nj = j + 1;  // the unit after this one, for the prefetch
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
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[0][i] = acc[1][i] = 0.f;
            cur_pt = pt;
            cur_t = t;
        }
        const uint4* xsrc = xbase + ((size_t)j * (16 / VX) * batch + g) * 4 + c;
        if constexpr (K2F != 0)
            gemv_unit<CODE, K2F, V, L16, NXW>(nxt, next_base, K2F, lane, src_lane, p, lut_lane, xsrc, xstride,
                                                     use_x, acc);
        else
            gemv_unit_k2<CODE, V, L16>(p.part[pt].k2, nxt, next_base, p.part[npt].k2, lane, src_lane, p,
                                              lut_lane, xsrc, xstride, use_x, acc);
        pt = npt;
        t = nt;
        j = nj;
    }
    if (u0 < u1) flush(cur_pt, cur_t);
    if (p.fuse_out) output_epilogue(p, reinterpret_cast<float*>(smem), c0, c1);
}

// ---- the forward's launch plan and dispatch ----

GemvPlan plan_gemv(const Layer& L, int batch) {
    GemvPlan pl;
    long long rt_total = 0;
    for (int i = 0; i < L.nparts; ++i) rt_total += L.parts[i].rows / kRowTile;
    const long long units = rt_total * (L.n / kT);
    pl.grid = (int)(units < L.num_sms ? units : L.num_sms);
    const long long per_cta = (units + pl.grid - 1) / pl.grid;
    const long long per_warp = (per_cta + kGemvMaxWarps - 1) / kGemvMaxWarps;
    pl.threads = (int)((per_cta + per_warp - 1) / per_warp) * 32;
    const long long lut_words = uses_table(L.code) ? (32ll << L.Q) : 0;
    const long long budget = kGemvMaxSmem / 4;
    // the output transform in-kernel when all of it is small (measured: with
    // many output blocks, e.g. m = 11008 in blocks of 256, the drain before
    // the tickets and the per-CTA transforms cost more than the separate
    // kernel), as many batch rows of one Hadamard block at once as fit (plus
    // its sign words)
    pl.fuse_out = (long long)batch * L.m <= kFuseOutElems;
    const long long row_words = L.B_m + L.B_m / 16;
    const long long sign_words = L.B_m / 32 + 2;
    long long rows = (budget - sign_words) / row_words;
    if (rows > batch) rows = batch;
    if (rows < 1) rows = 1;
    const long long epi_words = pl.fuse_out ? rows * row_words + sign_words : 0;
    // the input transform in-kernel for the smallest batches: every CTA computes
    // all of x' into shared memory (groups of T = B_n / E threads, E = 8 or 16,
    // T a power of two within the CTA), in place of a kernel and its boundary
    pl.x_e = 0;
    pl.xs_word0 = (int)lut_words;
    long long main_words = lut_words;
    // with the whole batch-1 transform in-kernel, as many threads as give it
    // 8 entries each (shorter chains), when that does not raise the most
    // units a warp takes
    if (batch <= kXInKernelMaxBatch && L.B_n / 8 > pl.threads && L.B_n / 8 <= kGemvMaxWarps * 32 &&
        (per_cta + L.B_n / 256 - 1) / (L.B_n / 256) == per_warp)
        pl.threads = L.B_n / 8;
    int tmax = 32;
    while (tmax * 2 <= pl.threads) tmax *= 2;
    const int e = L.B_n / tmax < 8 ? 8 : L.B_n / tmax;
    const int T = L.B_n / e;
    const long long items = (long long)batch * (L.n / L.B_n);
    // measured: a transform of more than one block per group (rounds of loads
    // and barriers), or of blocks above 4096 entries, costs more in-kernel than
    // the input-transform kernel and its launch boundary
    const bool one_round = items <= pl.threads / T;
    if (batch <= kXInKernelMaxBatch && (e == 8 || e == 16) && T <= pl.threads && L.B_n <= 4096 && one_round) {
        const long long xs_words = (long long)batch * L.n / (L.V == 1 ? 1 : 2);
        const long long scratch = T > 32 ? (long long)(pl.threads / T) * (L.B_n + L.B_n / 16) : 0;
        if (xs_words * 4 <= kXInKernelMaxBytes && lut_words + xs_words + scratch <= budget) {
            pl.x_e = e;
            main_words = lut_words + xs_words + scratch;
        }
    }
    pl.smem_bytes = (int)((main_words > epi_words ? main_words : epi_words) * 4);
    return pl;
}

float gemv_z_scale(const Layer& L) { return L.code == kCode1MAD ? kC1 : 1.0f; }

size_t gemv_xstep_bytes(const Layer& L, int batch) { return (size_t)batch * L.n / (L.V == 1 ? 1 : 2) * 4; }

template <int CODE, int K2, int V, bool L16>
struct GemvLaunch {
    static cudaError_t run(const GemvArgs& a, const GemvPlan& pl, cudaStream_t st) {
        constexpr int K2F = K2 == 99 ? 0 : K2;
        cudaError_t e = ensure_smem_limit<trellis_gemv_kernel<CODE, V, L16, K2F>>(kGemvMaxSmem);
        if (e != cudaSuccess) return e;
        return launch_pdl(trellis_gemv_kernel<CODE, V, L16, K2F>, dim3(pl.grid), dim3(pl.threads),
                          (size_t)pl.smem_bytes, st, a);
    }
};

template <int CODE, int K2, int V, bool L16>
struct GemvPrepare {
    static cudaError_t run() {
        constexpr int K2F = K2 == 99 ? 0 : K2;
        return preload_kernel<trellis_gemv_kernel<CODE, V, L16, K2F>>(kGemvMaxSmem);
    }
};

// A multi-part layer takes the per-unit decoder (the "K2 = 99" instance).
template <int CODE, int V, bool L16>
static cudaError_t gemv_multi_dispatch(const GemvArgs& a, const GemvPlan& pl, cudaStream_t st) {
    return GemvLaunch<CODE, 99, V, L16>::run(a, pl, st);
}

template <bool L16>
static cudaError_t gemv_multi_prepare(int code, int V) {
    if (code == kCode1MAD && V == 1) return GemvPrepare<kCode1MAD, 99, 1, L16>::run();
    if (code == kCode3INST && V == 1) return GemvPrepare<kCode3INST, 99, 1, L16>::run();
    if (code == kCodeHYB && V == 1) return GemvPrepare<kCodeHYB, 99, 1, L16>::run();
    if (code == kCodeHYB && V == 2) return GemvPrepare<kCodeHYB, 99, 2, L16>::run();
    if constexpr (!L16) {
        if (code == kCodeTable && V == 1) return GemvPrepare<kCodeTable, 99, 1, false>::run();
        if (code == kCodeTable && V == 2) return GemvPrepare<kCodeTable, 99, 2, false>::run();
    }
    return cudaErrorInvalidValue;
}

template <bool L16>
static cudaError_t gemv_multi_l(int code, int V, const GemvArgs& a, const GemvPlan& pl, cudaStream_t st) {
    if (code == kCode1MAD && V == 1) return gemv_multi_dispatch<kCode1MAD, 1, L16>(a, pl, st);
    if (code == kCode3INST && V == 1) return gemv_multi_dispatch<kCode3INST, 1, L16>(a, pl, st);
    if (code == kCodeHYB && V == 1) return gemv_multi_dispatch<kCodeHYB, 1, L16>(a, pl, st);
    if (code == kCodeHYB && V == 2) return gemv_multi_dispatch<kCodeHYB, 2, L16>(a, pl, st);
    if constexpr (!L16) {
        if (code == kCodeTable && V == 1) return gemv_multi_dispatch<kCodeTable, 1, false>(a, pl, st);
        if (code == kCodeTable && V == 2) return gemv_multi_dispatch<kCodeTable, 2, false>(a, pl, st);
    }
    return cudaErrorInvalidValue;
}

// qlinear_decode: the fp16-rounded values of one unit in the order of 16
// m16n8k16 A operands (two weights per register).  MMA u takes, for each
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

// ---- qlinear_decode: one warp per unit, fp16 W_hat row-major ----
template <int CODE, int K2, int V, bool L16>
__global__ void __launch_bounds__(256) trellis_decode_kernel(DecodeArgs p, __half* __restrict__ w_hat, int n, int row0) {
    extern __shared__ __align__(16) uint32_t lut_smem[];
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
        if constexpr (CODE == kCodeE8P) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const size_t row = (size_t)row0 + R * kRowTile + 8 * h + g;
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    uint32_t pr[4];
                    const uint32_t wd = cw[h][1 + t / 2];
                    e8p_pairs((t & 1) ? (wd & 0xFFFFu) : (wd >> 16), lut_lane, pr);
                    *reinterpret_cast<uint4*>(w_hat + row * n + (size_t)j * kT + 64 * c + 8 * t) =
                        make_uint4(pr[0], pr[1], pr[2], pr[3]);
                }
            }
        } else {
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
}

// ---- qlinear_eval_code ----
template <int CODE, int V>
__global__ void eval_code_kernel(const uint32_t* __restrict__ states, int count, uint32_t lmask, int qshift,
                                 const uint32_t* __restrict__ lut, int lut_entries, __half* __restrict__ out) {
    extern __shared__ __align__(16) uint32_t lut_smem[];
    const int lane = threadIdx.x & 31;
    if (uses_table(CODE)) {
        fill_lut_smem(lut_smem, lut, lut_entries);
        __syncthreads();
    }
    const uint32_t* lut_lane = lut_smem + lane;
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if constexpr (CODE == kCodeE8P) {
        if (t < count) {
            uint32_t pr[4];
            e8p_pairs(states[t] & 0xFFFFu, lut_lane, pr);
            reinterpret_cast<uint4*>(out)[t] = make_uint4(pr[0], pr[1], pr[2], pr[3]);
        }
    } else if constexpr (V == 2) {
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
    } else {
        if (code == kCodeE8P && V == 8 && k2 == 4) return F<kCodeE8P, 4, 8, true>::run(args...);
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
struct DecodePrepare {
    static cudaError_t run() {
        const bool big = uses_table(CODE) && (32 << kMaxTableBits) * 4 > 48 * 1024;
        return preload_kernel<trellis_decode_kernel<CODE, K2, V, L16>>(big ? 32 * 512 * 4 : 0);
    }
};

template <int CODE, int K2, int V, bool L16>
struct EvalLaunch {
    static cudaError_t run(const uint32_t* states, int count, uint32_t lmask, int qshift, const uint32_t* lut,
                           int entries, __half* out, cudaStream_t st) {
        // one instance per (code, V) suffices: the code ignores k and L
        if (CODE != kCodeE8P && (K2 != 2 || L16 == (CODE == kCodeTable))) return cudaErrorInvalidValue;
        const size_t smem = (size_t)entries * 32 * 4;
        auto kern = eval_code_kernel<CODE, V>;
        if (smem > 48 * 1024) {
            cudaError_t e = ensure_smem_limit<eval_code_kernel<CODE, V>>(32 * 512 * 4);
            if (e != cudaSuccess) return e;
        }
        const int items = V >= 2 ? count : (count + 1) / 2;
        kern<<<(items + 255) / 256, 256, smem, st>>>(states, count, lmask, qshift, lut, entries, out);
        return cudaGetLastError();
    }
};

cudaError_t launch_eval_code(int code, int L, int V, int Q, const uint32_t* lut_words, const uint32_t* states,
                             int count, void* out, cudaStream_t st) {
    const uint32_t lmask = (1u << L) - 1u;
    const int entries = uses_table(code) ? (1 << Q) : 0;
    if (code == kCodeE8P)
        return EvalLaunch<kCodeE8P, 4, 8, true>::run(states, count, lmask, 32 - Q, lut_words, entries, (__half*)out, st);
    return dispatch<EvalLaunch>(code, 2, V, code != kCodeTable, states, count, lmask, 32 - Q, lut_words, entries,
                                (__half*)out, st);
}


cudaError_t launch_gemv(const Layer& L, const GemvPlan& pl, const void* x, const void* xstep, int batch, float* z,
                        int* tickets, void* y, int y_dtype, cudaStream_t st) {
    GemvArgs a;
    a.nparts = L.nparts;
    a.nb = L.n / kT;
    a.units = 0;
    for (int i = 0; i < kMaxParts; ++i) {
        const Part& pt = L.parts[i < L.nparts ? i : 0];
        a.part[i].words = L.words + pt.word_off;
        a.part[i].rt = pt.rows / kRowTile;
        a.part[i].row0 = pt.row0;
        a.part[i].k2 = pt.k2;
        if (i < L.nparts) a.units += (long long)a.part[i].rt * a.nb;
    }
    a.lmask = (1u << L.L) - 1u;
    a.qshift = 32 - L.Q;
    a.lut = L.lut;
    a.lut_entries = uses_table(L.code) ? (1 << L.Q) : 0;
    a.batch = batch;
    a.m = L.m;
    a.n = L.n;
    a.xstep = (const uint4*)xstep;
    a.x = (const __half*)x;
    a.sin_bits = L.sin_bits;
    a.B_n = L.B_n;
    a.x_e = pl.x_e;
    a.xs_word0 = pl.xs_word0;
    a.z = z;
    a.tickets = tickets;
    a.B_m = L.B_m;
    a.sout_bits = L.sout_bits;
    a.out_scale = L.alpha * gemv_z_scale(L) / sqrtf((float)L.B_m);
    a.y = y;
    a.y_f16 = y_dtype == QL_F16;
    a.fuse_out = pl.fuse_out;
    a.smem_floats = pl.smem_bytes / 4;
    const bool l16 = L.L == 16;
    if (L.nparts > 1) return l16 ? gemv_multi_l<true>(L.code, L.V, a, pl, st) : gemv_multi_l<false>(L.code, L.V, a, pl, st);
    return dispatch<GemvLaunch>(L.code, L.parts[0].k2, L.V, l16, a, pl, st);
}

cudaError_t prepare_gemv_kernels(const Layer& L) {
    const bool l16 = L.L == 16;
    cudaError_t e = L.nparts > 1 ? (l16 ? gemv_multi_prepare<true>(L.code, L.V) : gemv_multi_prepare<false>(L.code, L.V))
                                 : dispatch<GemvPrepare>(L.code, L.parts[0].k2, L.V, l16);
    for (int i = 0; i < L.nparts && e == cudaSuccess; ++i) e = dispatch<DecodePrepare>(L.code, L.parts[i].k2, L.V, l16);
    return e;
}

}  // namespace qlk
