// codes.cuh -- device-side trellis window extraction and the three codes.
//
// The codes (QTIP OpenReview discussion: "Inference speed analysis (W2)", the
// comment on HYB cost, "HYB Uniqueness (Q2)", "Bit Accounting (Q2)"):
//   1MAD : x = A*s + B; value = fp16(C1 * (byte0 + byte1 + byte2 + byte3 - 510))
//   3INST: x = A*s + B; m = (x & MASK) ^ XOR; value = fp16(half(m.lo) + half(m.hi))
//   HYB  : x = A*s + B; entry = lut[x >> (32 - Q)]; bit 15 of x negates value 0
//   TABLE: entry = lut[s]: the palette quantizers of the Q-Palette page (VQ for
//          V = 2, NUQ for V = 1, when L = kV; a trellis over an explicit
//          codebook when L > kV)
// Every value is rounded to fp16 exactly once:
//   * 1MAD: the byte sum is produced directly as the fp16 bit pattern of
//     1536 + d (one dp4a whose accumulator is 0x6400 + 512 - 510; the
//     pattern 0x6400 + t is the half 1024 + t for 0 <= t < 1024), then one
//     half-precision FMA computes (1536 + d)*C1 - 1536*C1 = d*C1 with a single
//     rounding.  C1 = 443 * 2^-16 has 9 significant bits, so C1 and 1536*C1
//     are exact halves.
//   * 3INST: the two halves are finite normal halves; one fp16 add rounds once.
//   * HYB: no arithmetic on values, only a sign-bit xor; TABLE: none at all.
// The constants are part of the stream format; they were chosen by a seeded
// search against the statistical properties the discussion states for the
// codes (approximately N(0,1) at L = 16, successors of a state decorrelated).
//
// Instruction balance on sm_100a: IMAD, IDP4A/IDP2A and the packed-half
// HADD2/HFMA2 issue to one pipe, LOP3/PRMT/SHF to another, each at half the
// issue rate; the decode below splits its work between the two.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

namespace qlk {

constexpr int kCode1MAD = 0;
constexpr int kCode3INST = 1;
constexpr int kCodeHYB = 2;
constexpr int kCodeTable = 3;
constexpr int kCodeE8P = 4;

// Codes whose values come from a table in shared memory (2^Q words; the
// table code's Q is L; the E8 code's 256 shapes take 2 words each, Q = 9).
__host__ __device__ constexpr bool uses_table(int code) {
    return code == kCodeHYB || code == kCodeTable || code == kCodeE8P;
}
constexpr int kMaxTableBits = 9;  // 2^9 entries x 32 lanes x 4 bytes = 64 KiB replicated

constexpr uint32_t kA1MAD = 0x61616D4Bu, kB1MAD = 0xE29B5692u;
constexpr uint32_t kA3INST = 0x6C9FB67Bu, kB3INST = 0xA1E8CAB9u;
constexpr uint32_t kMask3INST = 0x9CFF8FFFu, kXor3INST = 0x20003000u;
constexpr uint32_t kAHYB = 0xBB6071B9u, kBHYB = 0x989D49ADu;

// 3INST masks applied after regrouping two states' low halves (resp. high
// halves) into one register: the low-half mask/xor in both halves, and the
// high-half mask/xor in both halves.
constexpr uint32_t kMask3Lo2 = (kMask3INST & 0xFFFFu) * 0x10001u;
constexpr uint32_t kXor3Lo2 = (kXor3INST & 0xFFFFu) * 0x10001u;
constexpr uint32_t kMask3Hi2 = (kMask3INST >> 16) * 0x10001u;
constexpr uint32_t kXor3Hi2 = (kXor3INST >> 16) * 0x10001u;

// 1MAD constants as half2 bit patterns: C1 = 443*2^-16 = 0x1EEC, -1536*C1 = -10.3828125 = 0xC931.
constexpr uint32_t kC1x2 = 0x1EEC1EECu;
constexpr uint32_t kNegBiasC1x2 = 0xC931C931u;
constexpr uint32_t kDp4aAcc = 0x6600u - 510u;

__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Low / high 16 bits of r through the dot-product unit (the FMA pipe), so
// that the extraction does not compete with the LOP3/PRMT/SHF work.
// (Inline PTX keeps the compiler from rewriting the dot product with a
// constant operand into shifts and masks on the other pipe.)
__device__ __forceinline__ uint32_t half_lo(uint32_t r) {
    uint32_t d;
    asm volatile("dp2a.lo.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(r), "r"(0x0001u), "r"(0u));
    return d;
}
__device__ __forceinline__ uint32_t half_hi(uint32_t r) {
    uint32_t d;
    asm volatile("dp2a.lo.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(r), "r"(0x0100u), "r"(0u));
    return d;
}

// Two V=1 states -> their two fp16 values packed (state a in the low half).
template <int CODE>
__device__ __forceinline__ uint32_t code_pair(uint32_t sa, uint32_t sb, const uint32_t* lut_lane, int qshift);

template <>
__device__ __forceinline__ uint32_t code_pair<kCode1MAD>(uint32_t sa, uint32_t sb, const uint32_t*, int) {
    const uint32_t xa = kA1MAD * sa + kB1MAD;
    const uint32_t xb = kA1MAD * sb + kB1MAD;
    const uint32_t ra = __dp4a(xa, 0x01010101u, kDp4aAcc);
    const uint32_t rb = __dp4a(xb, 0x01010101u, kDp4aAcc);
    return hfma2_u32(__byte_perm(ra, rb, 0x5410), kC1x2, kNegBiasC1x2);
}

template <>
__device__ __forceinline__ uint32_t code_pair<kCode3INST>(uint32_t sa, uint32_t sb, const uint32_t*, int) {
    const uint32_t xa = kA3INST * sa + kB3INST;
    const uint32_t xb = kA3INST * sb + kB3INST;
    const uint32_t lo = (__byte_perm(xa, xb, 0x5410) & kMask3Lo2) ^ kXor3Lo2;
    const uint32_t hi = (__byte_perm(xa, xb, 0x7632) & kMask3Hi2) ^ kXor3Hi2;
    return hadd2_u32(lo, hi);
}

// HYB: the table is replicated per lane in shared memory: entry i of lane l
// is word i*32 + l, so 32 lanes with arbitrary indices never share a bank.
__device__ __forceinline__ uint32_t hyb_word(uint32_t x, const uint32_t* lut_lane, int qshift) {
    return lut_lane[(x >> qshift) * 32u] ^ (x & 0x8000u);
}

// HYB with V = 1: table words hold the fp16 value in their low half.
template <>
__device__ __forceinline__ uint32_t code_pair<kCodeHYB>(uint32_t sa, uint32_t sb, const uint32_t* lut_lane, int qshift) {
    const uint32_t ea = hyb_word(kAHYB * sa + kBHYB, lut_lane, qshift);
    const uint32_t eb = hyb_word(kAHYB * sb + kBHYB, lut_lane, qshift);
    return __byte_perm(ea, eb, 0x5410);
}

// Table code with V = 1: entry s of the table, value in the low half.
template <>
__device__ __forceinline__ uint32_t code_pair<kCodeTable>(uint32_t sa, uint32_t sb, const uint32_t* lut_lane, int) {
    return __byte_perm(lut_lane[sa * 32u], lut_lane[sb * 32u], 0x5410);
}

// V = 2 (HYB or the table code): one state -> one table word (value 0 low, value 1 high).
template <int CODE>
__device__ __forceinline__ uint32_t code_v2(uint32_t s, const uint32_t* lut_lane, int qshift) {
    static_assert(CODE == kCodeHYB || CODE == kCodeTable, "V = 2 needs a table code");
    if (CODE == kCodeHYB) return hyb_word(kAHYB * s + kBHYB, lut_lane, qshift);
    return lut_lane[s * 32u];
}

// E8 code (V = 8, one 16-bit state per 8 values): the fp16 pairs of the
// state's codeword, coordinates 2p and 2p + 1 in pair p.  The state holds the
// shape index a (bits 8..15), the signs of coordinates 0..6 (bits 1..7: set =
// negative) and the shift (bit 0: +1/4, else -1/4).  Shape a is table words
// 2a (coordinates 0..3) and 2a + 1 (4..7), one byte per coordinate: the high
// byte of its magnitude in fp16 (the low byte is zero); bit 31 of word 2a + 1
// is the shape's parity bit, (sum of 2|T_i|) / 2 mod 2.  The sign of
// coordinate 7 is that bit xor the parity of the other seven signs, which
// makes the signed shape's coordinate sum even: a point of E8.
__device__ __forceinline__ void e8p_pairs(uint32_t s, const uint32_t* lut_lane, uint32_t (&pr)[4]) {
    const uint32_t a = s >> 8;
    const uint32_t w0 = lut_lane[(2u * a) * 32u], w1 = lut_lane[(2u * a + 1u) * 32u];
    const uint32_t sb = (s >> 1) & 0x7Fu;
    const uint32_t x = sb | ((__popc(sb) & 1u) << 7);  // sign bits of coordinates 0..7 (bit 7: the parity)
    const uint32_t d = (s & 1u) ? 0x34003400u : 0xB400B400u;  // +1/4 or -1/4 in both halves
    // bit 2p of x to bit 15, bit 2p + 1 to bit 31: one multiply by 2^15 + 2^30
    pr[0] = hadd2_u32(__byte_perm(w0, 0u, 0x1404) ^ ((x * 0x40008000u) & 0x80008000u), d);
    pr[1] = hadd2_u32(__byte_perm(w0, 0u, 0x3424) ^ (((x >> 2) * 0x40008000u) & 0x80008000u), d);
    pr[2] = hadd2_u32(__byte_perm(w1, 0u, 0x1404) ^ (((x >> 4) * 0x40008000u) & 0x80008000u), d);
    pr[3] = hadd2_u32(__byte_perm(w1, 0u, 0x3424) ^ (((x >> 6) * 0x40008000u) & 0x80008000u), d);
}

// Fill the per-lane replicated table (HYB, the table code's codebook, the E8
// code's shapes) in shared memory: word 32 i + l holds entry i for lane l.
// Thread k reads entries k and k + blockDim (both loads first) and writes each
// one's 32 copies (128 contiguous bytes) as eight 16-byte stores, starting at
// chunk i % 8 so that eight consecutive threads cover all 32 banks.
__device__ __forceinline__ void fill_lut_smem(uint32_t* smem, const uint32_t* lut, int entries) {
    const int bd = blockDim.x;
    for (int i = threadIdx.x; i < entries; i += 2 * bd) {
        const bool two = i + bd < entries;
        const uint32_t v0 = __ldg(lut + i), v1 = two ? __ldg(lut + i + bd) : 0u;
        uint4* d0 = reinterpret_cast<uint4*>(smem + 32 * i);
#pragma unroll
        for (int q = 0; q < 8; ++q) d0[(q + i) & 7] = make_uint4(v0, v0, v0, v0);
        if (two) {
            uint4* d1 = reinterpret_cast<uint4*>(smem + 32 * (i + bd));
#pragma unroll
            for (int q = 0; q < 8; ++q) d1[(q + i + bd) & 7] = make_uint4(v1, v1, v1, v1);
        }
    }
}

// Bits [a, a + 32) of a thread-row's bit string (most significant bit first):
// cw[0] holds the 32 bits before the thread's own range, cw[1..] its words.
// `a` is a compile-time constant after unrolling.
template <int NW>
__device__ __forceinline__ uint32_t bits32(const uint32_t (&cw)[NW], int a) {
    const int w = a >> 5, o = a & 31;
    if (o == 0) return cw[w];
    return __funnelshift_l(cw[w + 1], cw[w], o);
}

// Trellis states of one thread-row: state t is the L-bit window ending at
// bit 32 + (t+1)*kV of the thread-row string (the low L bits of the 16-bit
// window, see the tail-biting rule in include/qlinear.h).
//
// When 16 is a multiple of kV, the windows of steps t and t + 16/kV are the
// two halves of one 32-bit funnel shift: one SHF serves two states.
template <int kV, bool L16, int NW>
__device__ __forceinline__ void state_pair(const uint32_t (&cw)[NW], int t, uint32_t lmask, uint32_t& s_t,
                                           uint32_t& s_t2) {
    const uint32_t r = bits32(cw, 32 + (t + 1) * kV - 16);
    if (L16) {
        s_t = half_hi(r);
        s_t2 = half_lo(r);
    } else {
        s_t = (r >> 16) & lmask;
        s_t2 = r & lmask;
    }
}

template <int kV, bool L16, int NW>
__device__ __forceinline__ uint32_t state_one(const uint32_t (&cw)[NW], int t, uint32_t lmask) {
    const uint32_t r = bits32(cw, 32 + (t + 1) * kV - 32);
    return L16 ? half_lo(r) : (r & lmask);
}

}  // namespace qlk
