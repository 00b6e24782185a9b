// layout.cuh -- how the handle stores code words for the decode kernels.
//
// The caller's stream is row-major (row r, then block j, then the block's bits).
// The decode kernels work on units of 16 rows x one 256-column block: lane
// (g, c) = (lane / 4, lane % 4) of a warp decodes rows g and g + 8 of the
// unit ("thread-row" h = 0 and 1), steps [c*P/4, (c+1)*P/4) of the block
// (P = 256 / V steps), i.e. the contiguous bit range [c*S/4, (c+1)*S/4) of
// each of its two blocks (S = 256*k bits, S/4 = 2k words).  k may be a half
// number of bits (odd kV with V = 2), so everything is counted in K2 = 2k,
// a whole number: the words of one thread-row.  Create re-lays the words so
// that one vector load per (h, chunk) by the 32 lanes reads one contiguous
// segment of 128, 256 or 512 bytes:
//
//   unit u = R * nb + j                      (R = row tile, j = block)
//   word  = u * 64 K2 + ((h * NV + q) * 32 + lane) * VW + e
//
// with VW = 4 words per vector when 4 divides K2 (16-byte loads), else 2
// when 2 does (8-byte loads), else 1, NV = K2 / VW vectors per thread-row,
// and thread-row word index w = q * VW + e.  The layout is a permutation of
// the words; sizes match.
#pragma once
#include <stdint.h>

namespace qlk {

__host__ __device__ constexpr int unit_vector_words(int k2) { return k2 % 4 == 0 ? 4 : (k2 % 2 == 0 ? 2 : 1); }

template <int K2>
struct UnitLayout {
    static constexpr int TW = K2;                        // words per thread-row
    static constexpr int VW = unit_vector_words(K2);     // words per vector load
    static constexpr int NV = TW / VW;                   // vector loads per thread-row
    static constexpr int UW = 64 * K2;                   // words per unit
};

// Runtime form (used by the re-layout kernel for any K2).
__host__ __device__ inline void unit_word_coords(int k2, uint32_t within, int* h, int* lane, int* w) {
    const int VW = unit_vector_words(k2);
    const int NV = k2 / VW;
    const int e = within % VW;
    const uint32_t v = within / VW;
    *lane = v % 32;
    const uint32_t hq = v / 32;
    *h = hq / NV;
    const int q = hq % NV;
    *w = q * VW + e;
}

}  // namespace qlk
