// layout.cuh -- how the handle stores code words for the decode kernels.
//
// The caller's stream is row-major (row r, then block j, then the block's bits).
// The decode kernels work on units of 16 rows x one 256-column block: lane
// (g, c) = (lane / 4, lane % 4) of a warp decodes rows g and g + 8 of the
// unit ("thread-row" h = 0 and 1), steps [c*P/4, (c+1)*P/4) of the block
// (P = 256 / V steps), i.e. the contiguous bit range [c*S/4, (c+1)*S/4) of
// each of its two blocks (S = 256*k bits, S/4 = 2k words).  Create re-lays the
// words so that one vector load per (h, chunk) by the 32 lanes reads one
// contiguous 256- or 512-byte segment:
//
//   unit u = R * nb + j                      (R = row tile, j = block)
//   word  = u * 128k + ((h * NV + q) * 32 + lane) * VW + e
//
// with VW = 4 words per vector for even k (16-byte loads), 2 for odd k
// (8-byte loads), NV = 2k / VW vectors per thread-row, and thread-row word
// index w = q * VW + e.  The layout is a permutation of the words; sizes match.
#pragma once
#include <stdint.h>

namespace qlk {

template <int K>
struct UnitLayout {
    static constexpr int TW = 2 * K;                 // words per thread-row
    static constexpr int VW = (K % 2 == 0) ? 4 : 2;  // words per vector load
    static constexpr int NV = TW / VW;               // vector loads per thread-row
    static constexpr int UW = 128 * K;               // words per unit
};

// Runtime form (used by the re-layout kernel for any k).
__host__ __device__ inline void unit_word_coords(int k, uint32_t within, int* h, int* lane, int* w) {
    const int VW = (k % 2 == 0) ? 4 : 2;
    const int NV = 2 * k / VW;
    const int e = within % VW;
    const uint32_t v = within / VW;
    *lane = v % 32;
    const uint32_t hq = v / 32;
    *h = hq / NV;
    const int q = hq % NV;
    *w = q * VW + e;
}

}  // namespace qlk
