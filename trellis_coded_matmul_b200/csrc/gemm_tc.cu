// gemm_tc.cu -- trellis decode into tensor memory + tcgen05 tensor-core GEMM
// for batches above 8: z[b][row] = sum_c W_hat[row][c] x'[b][c], as partial
// sums per stream-K segment (below).
//
// The contraction is dense (M = 128 rows of W_hat per tile, N = batch padded
// to 16, K = n), so it runs on the 5th-generation tensor cores: the fp16 A
// operand in tensor memory, B = x' in shared memory (K-major, 128-byte
// swizzle), fp32 accumulator in tensor memory, one thread issuing
// tcgen05.mma.  The A operand is produced on the fly by decoder warps from
// the trellis code words (QTIP discussion:
// decode with computed codes or a small table; the bitshift trellis makes any
// run of steps decodable from the bits around it), so decoded weights never
// reach HBM.
//
// Work split (stream-K): the (128-row tile, 256-column block) units of the
// layer are cut into one contiguous run per CTA, one CTA per SM, so every SM
// decodes the same number of weights whatever the tile count.  A CTA's run
// falls into segments of consecutive blocks of one tile; each segment is
// accumulated in tensor memory and written with plain stores to its own slot
// of a partial-sum workspace (slot = the segment's rank in unit order, so the
// one to three segments of a tile have consecutive slots); the output
// transform sums a tile's slots as it reads them.  No atomics, and nothing to
// re-zero between forwards.
//
// Warp roles (a warp runs on SM sub-partition warp % 4, and may only touch
// tensor-memory lanes 32 * (warp % 4) .. + 31):
//   16 decoders    four groups of 4; group g decodes quarter g (64 columns) of
//                  every 256-column block, i.e. every 4th stage; warp w of a
//                  group covers rows 32 (w % 4) .. + 31 of the tile, one row
//                  per lane, 64 consecutive trellis steps per lane, and writes
//                  the decoded fp16 pairs straight into the stage's A slot in
//                  tensor memory (tcgen05.st): decoded weights never touch
//                  shared memory;
//   4 epilogue     at the end of each segment, read the accumulator back (one
//     warps        lane quarter each) and store it to the segment's slot, while
//                  the decoders go on filling the A slots of the next segment;
//   MMA warp       allocates tensor memory (accumulator in columns [0, 256),
//                  A slots of 32 columns from 256 on); one lane issues the 4
//                  MMAs (K = 16 each, A from tensor memory, x' from shared
//                  memory) of a stage and commits them to the stage's "empty"
//                  barrier, and the last of a segment to "acc_full";
//   x' producer    bulk copy of each stage's x' tile (x' is stored
//                  pre-swizzled) into the stage's shared-memory slot;
//   code producer  bulk copies of the code words, one 256-column block of the
//                  tile's row tiles at a time, into a ring of blocks.
// A stage has one "full" barrier (4 decoder arrivals and the x' bytes) and
// one "empty" barrier (the MMA commit).  Every wait is bounded; on expiry the
// CTA records kStatusTimeout in the handle's status word, abandons its work
// and still frees its tensor memory.
#include <cuda_fp16.h>

#include <vector>

#include "codes.cuh"
#include "internal.h"
#include "layout.cuh"
#include "tc_ptx.cuh"

namespace qlk {

constexpr int kTcRows = 128;         // M of one tile
constexpr int kTcK = 64;             // K of one stage (one 128-byte swizzled row of fp16)
constexpr int kTcDecoders = 16;      // decoder warps: four groups of 4, group g decodes quarter g of each block
constexpr int kTcGroup = 4;          // decoder warps per group (one per 32-row lane quarter)
constexpr int kTcWarps = 23;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kWarpMma = 16, kWarpXProd = 17, kWarpCodeProd = 18;
constexpr int kWarpEpi0 = 19, kTcEpiWarps = 4;  // warps 19..22: lane quarters 3, 0, 1, 2
constexpr int kTcMaxStages = 8;      // stage slots (A in tensor memory, x' tile in shared memory)
constexpr uint32_t kTcTmemCols = 512;  // accumulator [0, 256) and up to 8 A slots of 32 columns
constexpr uint32_t kTcTmemA = 256;     // first A-slot column
// Split A words (computed codes at batch <= 128): each weight is one 32-bit
// word whose two fp16 halves sum to it, and x' sits twice along K, so the MMA
// does the sum (the decode-GEMV's form): a stage's A slot is 64 columns, from
// column 128 (the accumulator then has at most 128), and its x' tile is two
// 128-byte swizzled sub-tiles.
constexpr uint32_t kTcTmemASplit = 128;
constexpr int kTcMaxStagesSplit = 6;  // (512 - 128) / 64
constexpr int kTcMaxSplitN = 128;
constexpr int kTcMaxCodeSlots = 4;   // code-word blocks in flight
#ifndef QL_TC_XSPLIT
#define QL_TC_XSPLIT 1
#endif
constexpr int kTcXSplit = QL_TC_XSPLIT;  // bulk copies per x' tile (npad * 128 bytes, a multiple of 2 KB)
static_assert(kTcXSplit == 1 || kTcXSplit == 2 || kTcXSplit == 4 || kTcXSplit == 8, "x' split");
constexpr int kTcWaitTries = 4096;           // try_wait calls of up to kTcSuspendNs each (a few seconds in all)
constexpr uint32_t kTcSuspendNs = 1000000;   // before a wait is declared expired
// barriers: code_full[C], code_empty[C], full[S], empty[S], acc_full, acc_empty
static_assert(2 * kTcMaxCodeSlots + 2 * kTcMaxStages + 2 <= 60, "barrier area");

// decoder group (0..3 = the block quarter it decodes) and lane quarter of warp w
__device__ __forceinline__ bool decoder_role(int w, int& grp, int& qtr) {
    if (w >= kTcDecoders) return false;
    grp = w >> 2;
    qtr = w & 3;
    return true;
}

struct TcPart {
    const uint32_t* words;  // kernel layout
    int rt;                 // row tiles of 16 rows
    int k2;                 // 2k: bits per two weights
    int tiles;              // 128-row tiles
};

struct GemmArgs {
    TcPart part[kMaxParts];
    int nparts;
    int nb;                 // 256-column blocks per row
    int units;              // (tile, block) units of the layer: sum over parts of tiles * nb
    uint32_t lmask;
    int qshift;
    const uint32_t* lut;
    int lut_entries;
    const uint8_t* xt;      // x' tiles: [n / 64][npad][128 B, swizzled]
    int npad;               // MMA N: batch padded to a multiple of 16 (<= 256)
    int batch;              // valid columns
    float* ws;              // partial sums: [segment slot][npad][128 rows], columns < batch written
    const int* cta_seg;     // slot of each CTA's first segment
    int* status;
    int wait_tries;         // try_wait calls of up to kTcSuspendNs before a wait is declared expired
    int withhold;           // test hook: the x' producer withholds its first stage (its waits then expire)
    int stages;             // stage slots
    int code_slots;         // depth of the code-word ring
    int code_slot_words;    // words of one code-ring slot (8 units at the largest k2)
};

struct TcSmem {  // offsets in bytes from the 1024-aligned dynamic shared memory base
    int b, code, lut, bar, total;
};

__host__ __device__ inline TcSmem tc_smem_layout(int stages, int code_slots, int npad, int code_slot_words,
                                                  int lut_entries) {
    TcSmem s;
    s.b = 0;
    s.code = s.b + stages * npad * 128;
    s.lut = s.code + code_slots * code_slot_words * 4;
    s.bar = s.lut + lut_entries * 32 * 4;
    s.total = s.bar + 512;  // mbarriers, the TMEM base address and the abort flag
    return s;
}

// A CTA's run of units in order, walked without divisions (the roles' loops
// are latency-bound chains; the MMA issuer's especially).  Units are numbered
// part by part, tile by tile, block by block.
struct TcWalk {
    int u, pt, t, j;  // unit, part, 128-row tile within the part, block
    __device__ __forceinline__ TcWalk(const GemmArgs& p, int u0) : u(u0), pt(0), j(0) {
        int gt = u0 / p.nb;
        j = u0 - gt * p.nb;
        while (pt + 1 < p.nparts && gt >= p.part[pt].tiles) gt -= p.part[pt++].tiles;
        t = gt;
    }
    __device__ __forceinline__ void next(const GemmArgs& p) {
        ++u;
        if (++j == p.nb) {
            j = 0;
            if (++t == p.part[pt].tiles && pt + 1 < p.nparts) {
                t = 0;
                ++pt;
            }
        }
    }
    __device__ __forceinline__ int part(const GemmArgs&) const { return pt; }
    __device__ __forceinline__ int tile(const GemmArgs&) const { return t; }
};

// Slot and phase parity of a ring position, advanced without divisions.
struct TcRing {
    int slot;
    uint32_t phase;
    __device__ __forceinline__ TcRing(int pos, int n) : slot(pos), phase(0) {
        while (slot >= n) {
            slot -= n;
            phase ^= 1u;
        }
    }
    __device__ __forceinline__ void advance(int by, int n) {
        slot += by;
        while (slot >= n) {
            slot -= n;
            phase ^= 1u;
        }
    }
};
__device__ __forceinline__ int tc_tiles16(const TcPart& pt, int tile) {  // row tiles present (ragged last tile)
    const int n = pt.rt - tile * (kTcRows / kRowTile);
    return n < kTcRows / kRowTile ? n : kTcRows / kRowTile;
}

// One decoder thread's 32 weights of a stage: row r of its row tile, trellis
// steps [HQ * NS, (HQ + 1) * NS) (NS = 32 / V) of its quarter-block (64
// columns).  w[0] holds the 32 bits before the quarter, w[1..K2] its K2 words
// (K2 = 2k; with a half-integer k a run starts inside a word).  Output: 16
// half2 words, columns 2i and 2i + 1 of the run in word i.
template <int CODE, int K2, int V, bool L16, int HQ>
__device__ __forceinline__ void decode_run32_trellis(const uint32_t (&w)[K2 + 1], uint32_t lmask,
                                                     const uint32_t* lut_lane, int qshift, uint32_t (&out)[16]);

template <int CODE, int K2, int V, bool L16, int HQ>
__device__ __forceinline__ void decode_run32(const uint32_t (&w)[K2 + 1], uint32_t lmask, const uint32_t* lut_lane,
                                             int qshift, uint32_t (&out)[16]) {
    static_assert((K2 * V) % 2 == 0, "a step carries a whole number of bits");
    if constexpr (CODE == kCodeE8P) {  // four 16-bit steps of 8 weights: words 1 + 2 HQ and 2 + 2 HQ
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            uint32_t pr[4];
            const uint32_t wd = w[1 + 2 * HQ + t / 2];
            e8p_pairs((t & 1) ? (wd & 0xFFFFu) : (wd >> 16), lut_lane, pr);
#pragma unroll
            for (int q = 0; q < 4; ++q) out[4 * t + q] = pr[q];
        }
    } else {
        decode_run32_trellis<CODE, K2, V, L16, HQ>(w, lmask, lut_lane, qshift, out);
    }
}

template <int CODE, int K2, int V, bool L16, int HQ>
__device__ __forceinline__ void decode_run32_trellis(const uint32_t (&w)[K2 + 1], uint32_t lmask,
                                                     const uint32_t* lut_lane, int qshift, uint32_t (&out)[16]) {
    constexpr int kV = K2 * V / 2;
    constexpr int NS = 32 / V;
    constexpr int T0 = HQ * NS;
    constexpr bool kPair = (16 % kV) == 0;
    constexpr int P = kPair ? 16 / kV : 1;
    uint32_t s[NS];
#pragma unroll
    for (int t = 0; t < NS; ++t) {
        if (kPair) {
            if (((t / P) & 1) == 0) state_pair<kV, L16>(w, T0 + t, lmask, s[t], s[t + P]);
        } else {
            s[t] = state_one<kV, L16>(w, T0 + t, lmask);
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if constexpr (V == 1)
            out[i] = code_pair<CODE>(s[2 * i], s[2 * i + 1], lut_lane, qshift);
        else
            out[i] = code_v2<CODE>(s[i], lut_lane, qshift);
    }
}

// Bounded wait (at most `tries` suspending tries); returns false (and raises
// the CTA's abort flag) on expiry.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status,
                                         int tries) {
    if (mbar_test_wait(bar, parity)) return true;  // already complete: no suspension
    for (int i = 0; i < tries; ++i) {
        if (mbar_try_wait(bar, parity, kTcSuspendNs)) return true;
        if (*abort_flag) return false;
    }
    *abort_flag = 1;
    atomicOr(status, kStatusTimeout);
    return false;
}

// One decoder thread's share of a stage: row r = 32 qtr + lane of the tile,
// quarter q (64 steps) of the block whose row-tile units sit at shared address
// `code`.  The quarter's K2 = 2k words of the row are loaded with vector
// loads, plus the last word of the previous quarter (cyclically: tail-biting),
// then decoded in two runs of 32 columns; run hq becomes 16 packed fp16 pairs
// stored to tensor-memory columns a_col + 16 hq .. + 15 of the thread's lane.
template <int CODE, int K2, int V, bool L16>
__device__ __forceinline__ void decode_stage_tmem(uint32_t code, uint32_t a_taddr, int qtr, int q, int lane,
                                                  uint32_t lmask, const uint32_t* lut_lane, int qshift) {
    using UL = UnitLayout<K2>;
    const int r = 32 * qtr + lane;
    const int h = (r >> 3) & 1, g = r & 7;
    const uint32_t unit = code + (r >> 4) * UL::UW * 4;
    const int own = 4 * g + q;
    auto addr = [&](int slot_lane, int e) -> uint32_t {  // word e of (row half h, lane slot) in the unit layout
        return unit + 4 * (((h * UL::NV + e / UL::VW) * 32 + slot_lane) * UL::VW + (e % UL::VW));
    };
    uint32_t w[K2 + 1];
    w[0] = lds32(addr(4 * g + ((q + 3) & 3), K2 - 1));
#pragma unroll
    for (int c = 0; c < K2 / UL::VW; ++c) {
        if (UL::VW == 4)
            lds128(addr(own, 4 * c), w[1 + 4 * c], w[2 + 4 * c], w[3 + 4 * c], w[4 + 4 * c]);
        else if (UL::VW == 2)
            lds64(addr(own, 2 * c), w[1 + 2 * c], w[2 + 2 * c]);
        else
            w[1 + c] = lds32(addr(own, c));
    }
    uint32_t out[16];
    decode_run32<CODE, K2, V, L16, 0>(w, lmask, lut_lane, qshift, out);
    tmem_st16(a_taddr, out);
    decode_run32<CODE, K2, V, L16, 1>(w, lmask, lut_lane, qshift, out);
    tmem_st16(a_taddr + 16, out);
}

// A split word of one state: two fp16 halves whose sum is the code value (for
// 1MAD the value is 1536 + (byte sum - 510) - 1536, so the sum comes out in
// units of the 1MAD scale, which the output transform applies).
template <int CODE>
__device__ __forceinline__ uint32_t split_word(uint32_t s) {
    if constexpr (CODE == kCode3INST) {
        return ((kA3INST * s + kB3INST) & kMask3INST) ^ kXor3INST;
    } else {
        static_assert(CODE == kCode1MAD, "split words exist for the computed codes");
        return __dp4a(kA1MAD * s + kB1MAD, 0x01010101u, 0xE6000000u + kDp4aAcc);
    }
}

// decode_stage_tmem with split words: the quarter's 64 weights become 64
// words, tensor-memory columns a_col .. + 63 of the thread's lane (weight i of
// the quarter in column i).
template <int CODE, int K2, bool L16>
__device__ __forceinline__ void decode_stage_tmem_split(uint32_t code, uint32_t a_taddr, int qtr, int q, int lane,
                                                        uint32_t lmask) {
    using UL = UnitLayout<K2>;
    constexpr int kV = K2 / 2;  // V = 1
    constexpr bool kPair = (16 % kV) == 0;
    constexpr int P = kPair ? 16 / kV : 1;
    const int r = 32 * qtr + lane;
    const int h = (r >> 3) & 1, g = r & 7;
    const uint32_t unit = code + (r >> 4) * UL::UW * 4;
    const int own = 4 * g + q;
    auto addr = [&](int slot_lane, int e) -> uint32_t {
        return unit + 4 * (((h * UL::NV + e / UL::VW) * 32 + slot_lane) * UL::VW + (e % UL::VW));
    };
    uint32_t w[K2 + 1];
    w[0] = lds32(addr(4 * g + ((q + 3) & 3), K2 - 1));
#pragma unroll
    for (int c = 0; c < K2 / UL::VW; ++c) {
        if (UL::VW == 4)
            lds128(addr(own, 4 * c), w[1 + 4 * c], w[2 + 4 * c], w[3 + 4 * c], w[4 + 4 * c]);
        else if (UL::VW == 2)
            lds64(addr(own, 2 * c), w[1 + 2 * c], w[2 + 2 * c]);
        else
            w[1 + c] = lds32(addr(own, c));
    }
#pragma unroll
    for (int hq = 0; hq < 4; ++hq) {  // 16 steps (weights) per tensor-memory store
        uint32_t out[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const int step = 16 * hq + t;
            if (kPair) {
                if (((t / P) & 1) == 0) {
                    uint32_t s0, s1;
                    state_pair<kV, L16>(w, step, lmask, s0, s1);
                    out[t] = split_word<CODE>(s0);
                    if (t + P < 16) out[t + P] = split_word<CODE>(s1);
                }
            } else {
                out[t] = split_word<CODE>(state_one<kV, L16>(w, step, lmask));
            }
        }
        tmem_st16(a_taddr + 16 * hq, out);
    }
}

template <int CODE, bool L16>
__device__ __forceinline__ void decode_stage_split_k2(int k2, uint32_t code, uint32_t a_taddr, int qtr, int q,
                                                      int lane, uint32_t lmask) {
    switch (k2) {
        case 2: decode_stage_tmem_split<CODE, 2, L16>(code, a_taddr, qtr, q, lane, lmask); break;
        case 4: decode_stage_tmem_split<CODE, 4, L16>(code, a_taddr, qtr, q, lane, lmask); break;
        case 6: decode_stage_tmem_split<CODE, 6, L16>(code, a_taddr, qtr, q, lane, lmask); break;
        default: decode_stage_tmem_split<CODE, 8, L16>(code, a_taddr, qtr, q, lane, lmask); break;
    }
}

// The part's bitwidth picks the decoder (V = 1 has whole bitwidths only).
template <int CODE, int V, bool L16>
__device__ __forceinline__ void decode_stage_k2(int k2, uint32_t code, uint32_t a_taddr, int qtr, int q, int lane,
                                                uint32_t lmask, const uint32_t* lut_lane, int qshift) {
    if constexpr (V == 8) {  // the E8 code: 16 bits per 8 weights
        decode_stage_tmem<CODE, 4, V, L16>(code, a_taddr, qtr, q, lane, lmask, lut_lane, qshift);
        return;
    }
    switch (k2) {
        case 2: decode_stage_tmem<CODE, 2, V, L16>(code, a_taddr, qtr, q, lane, lmask, lut_lane, qshift); break;
        case 3: if constexpr (V == 2) decode_stage_tmem<CODE, 3, V, L16>(code, a_taddr, qtr, q, lane, lmask, lut_lane, qshift); break;
        case 4: decode_stage_tmem<CODE, 4, V, L16>(code, a_taddr, qtr, q, lane, lmask, lut_lane, qshift); break;
        case 5: if constexpr (V == 2) decode_stage_tmem<CODE, 5, V, L16>(code, a_taddr, qtr, q, lane, lmask, lut_lane, qshift); break;
        case 6: decode_stage_tmem<CODE, 6, V, L16>(code, a_taddr, qtr, q, lane, lmask, lut_lane, qshift); break;
        case 7: if constexpr (V == 2) decode_stage_tmem<CODE, 7, V, L16>(code, a_taddr, qtr, q, lane, lmask, lut_lane, qshift); break;
        default: decode_stage_tmem<CODE, 8, V, L16>(code, a_taddr, qtr, q, lane, lmask, lut_lane, qshift); break;
    }
}

template <int CODE, int V, bool L16, bool SPLIT>
__global__ void __launch_bounds__(kTcThreads, 1) trellis_gemm_kernel(GemmArgs p) {
    constexpr uint32_t kAcol0 = SPLIT ? kTcTmemASplit : kTcTmemA;  // first A-slot column
    constexpr uint32_t kAcols = SPLIT ? kTcK : kTcK / 2;            // columns of one A slot
    constexpr int kMmas = SPLIT ? 2 * kTcK / 16 : kTcK / 16;        // MMAs (K = 16) per stage
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base, derived by indexing the shared array so that
    // accesses through it stay shared-memory accesses
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int xrows = SPLIT ? 2 * p.npad : p.npad;  // 128-byte x' rows of one stage
    const TcSmem L = tc_smem_layout(p.stages, p.code_slots, xrows, p.code_slot_words, p.lut_entries);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
    const int S = p.stages, C = p.code_slots;
    const uint32_t bar0 = smem_u32(bars);
    auto code_full = [&](int i) { return bar0 + 8 * i; };
    auto code_empty = [&](int i) { return bar0 + 8 * (C + i); };
    auto full = [&](int i) { return bar0 + 8 * (2 * C + i); };
    auto empty = [&](int i) { return bar0 + 8 * (2 * C + S + i); };
    const uint32_t acc_full = bar0 + 8 * (2 * C + 2 * S);
    const uint32_t acc_empty = acc_full + 8;
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(bars + 2 * C + 2 * S + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's run of units
    const int u0 = (int)((long long)blockIdx.x * p.units / gridDim.x);
    const int u1 = (int)((long long)(blockIdx.x + 1) * p.units / gridDim.x);
    const uint32_t b_base = smem_u32(smem + L.b);
    const uint32_t code_base = smem_u32(smem + L.code);
    const uint32_t b_bytes = (uint32_t)xrows * 128;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C; ++i) {
            mbar_init(code_full(i), 1);
            mbar_init(code_empty(i), kTcDecoders);  // every decoder warp releases each block once
        }
        for (int i = 0; i < S; ++i) {
            mbar_init(full(i), kTcGroup + 1);  // one decoder group and the x' producer
            mbar_init(empty(i), 1);            // MMA commit
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kTcEpiWarps);
        *abort_flag = 0;
        mbar_fence_init();
    }
    uint32_t* lut_smem = reinterpret_cast<uint32_t*>(smem + L.lut);
    if (uses_table(CODE)) fill_lut_smem(lut_smem, p.lut, p.lut_entries);
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(tmem_base_smem), kTcTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;

    int grp = 0, qtr = 0;
    if (warp == kWarpXProd) {
        // ---------------- x' producer ----------------
        grid_dependency_wait();  // x' comes from the previous kernel
        TcRing r(0, S);
        bool ok = true;
        for (TcWalk w(p, u0); w.u < u1 && ok; w.next(p)) {
            const int j = w.j;
            for (int q = 0; q < 4; ++q, r.advance(1, S)) {
                const int st = r.slot;
                if (!wait_bar(empty(st), r.phase ^ 1u, abort_flag, p.status, p.wait_tries)) {
                    ok = false;
                    break;
                }
                // Test hook: the first stage's x' never arrives, so the MMA issuer's
                // wait on it expires (and with it every role's).
                if (p.withhold && w.u == u0 && q == 0) continue;
                // The tile goes in kTcXSplit pieces, one per lane, so that several
                // bulk copies are in flight at once.
                if (lane == 0) mbar_arrive_expect_tx(full(st), b_bytes);
                __syncwarp();
                if (lane < kTcXSplit) {
                    const uint32_t piece = b_bytes / kTcXSplit;
                    bulk_g2s(b_base + st * b_bytes + lane * piece,
                             p.xt + (size_t)(4 * j + q) * b_bytes + (size_t)lane * piece, piece, full(st));
                }
                __syncwarp();
            }
        }
    } else if (warp == kWarpCodeProd) {
        // ---------------- code-word producer ----------------
        TcRing r(0, C);
        for (TcWalk w(p, u0); w.u < u1; w.next(p), r.advance(1, C)) {
            const int slot = r.slot;
            const TcPart& pt = p.part[w.part(p)];
            const int tile = w.tile(p);
            const int ntiles16 = tc_tiles16(pt, tile);
            const int unit_words = 64 * pt.k2;
            if (!wait_bar(code_empty(slot), r.phase ^ 1u, abort_flag, p.status, p.wait_tries)) break;
            if (lane == 0) mbar_arrive_expect_tx(code_full(slot), (uint32_t)(ntiles16 * unit_words * 4));
            __syncwarp();
            if (lane < ntiles16) {
                const size_t unit = (size_t)(tile * (kTcRows / kRowTile) + lane) * p.nb + w.j;
                bulk_g2s(code_base + (uint32_t)(slot * p.code_slot_words + lane * unit_words) * 4,
                         reinterpret_cast<const uint8_t*>(pt.words) + unit * unit_words * 4,
                         (uint32_t)unit_words * 4, code_full(slot));
            }
            __syncwarp();
        }
    } else if (warp == kWarpMma) {
        // ---------------- MMA issuer ----------------
        // The descriptors of all stages differ only in the 14-bit start-address
        // field (low word, 16-byte units, no carry out of it below 256 KB):
        // build the words once and step the low word.
        const uint32_t idesc = idesc_f16_f32(kTcRows, p.npad);
        const uint64_t b_desc0 = smem_desc_k_sw128(b_base);
        const uint32_t b_hi = (uint32_t)(b_desc0 >> 32), b_lo0 = (uint32_t)b_desc0;
        const uint32_t b_step = b_bytes / 16;
        TcRing r(0, S);
        int seg = 0;
        for (TcWalk w(p, u0); w.u < u1; w.next(p)) {
            const bool first = w.u == u0 || w.j == 0;  // first block of a segment
            const bool last = w.u + 1 == u1 || w.j + 1 == p.nb;
            // the epilogue of the previous segment must have read the accumulator
            if (first && seg > 0 && !wait_bar(acc_empty, (seg - 1) & 1, abort_flag, p.status, p.wait_tries)) break;
            bool ok = true;
            for (int q = 0; q < 4; ++q, r.advance(1, S)) {
                const int st = r.slot;
                if (!wait_bar(full(st), r.phase, abort_flag, p.status, p.wait_tries)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one()) {
                    const uint32_t a_t = tmem + kAcol0 + (uint32_t)st * kAcols;
                    const uint32_t b_lo = b_lo0 + (uint32_t)st * b_step;
                    // K chunk kk: A columns 8 kk .. + 7; x' sub-tile kk / 4 (npad rows of 128
                    // bytes, 8 p.npad 16-byte units), 32 bytes per chunk within it
#pragma unroll
                    for (int kk = 0; kk < kMmas; ++kk)
                        tc_mma_f16_ts(tmem, a_t + kk * 8,
                                      ((uint64_t)b_hi << 32) | (b_lo + (kk >> 2) * 8 * p.npad + (kk & 3) * 2), idesc,
                                      (first && q == 0 && kk == 0) ? 0u : 1u);
                    tc_commit(empty(st));
                    if (last && q == 3) tc_commit(acc_full);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (last) ++seg;
        }
    } else if (decoder_role(warp, grp, qtr)) {
        // ---------------- decoders ----------------
        const uint32_t* lut_lane = lut_smem + lane;
        const uint32_t lane_base = (uint32_t)(qtr * 32) << 16;
        TcRing rc(0, C), rs(grp, S);  // code block i, stage 4 i + grp
        for (TcWalk w(p, u0); w.u < u1; w.next(p), rc.advance(1, C), rs.advance(4, S)) {
            const int slot = rc.slot;
            const TcPart& pt = p.part[w.part(p)];
            const uint32_t code = code_base + slot * p.code_slot_words * 4;
            if (!wait_bar(code_full(slot), rc.phase, abort_flag, p.status, p.wait_tries)) break;
            bool ok = true;
            {
                const int st = rs.slot;
                if (!wait_bar(empty(st), rs.phase ^ 1u, abort_flag, p.status, p.wait_tries)) {
                    ok = false;
                } else {
                    tc_fence_after();  // the MMAs that read this A slot have completed
                    // Rows of row tiles beyond a ragged last tile decode whatever the
                    // slot holds; their accumulator rows are never stored.
                    const uint32_t a_taddr = tmem + lane_base + kAcol0 + (uint32_t)st * kAcols;
                    if constexpr (SPLIT)
                        decode_stage_split_k2<CODE, L16>(pt.k2, code, a_taddr, qtr, grp, lane, p.lmask);
                    else
                        decode_stage_k2<CODE, V, L16>(pt.k2, code, a_taddr, qtr, grp, lane, p.lmask, lut_lane, p.qshift);
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(full(st));
                }
            }
            if (!ok) break;
            if (lane == 0) mbar_arrive(code_empty(slot));
        }
    } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + kTcEpiWarps) {
        // ---------------- epilogue: accumulator -> the segment's workspace slot ----------------
        const int qtr = warp & 3;
        const int rloc = qtr * 32 + lane;  // row within the tile
        const uint32_t tbase = tmem + ((uint32_t)(qtr * 32) << 16);
        int seg = 0;
        float* ws = nullptr;
        for (TcWalk w(p, u0); w.u < u1; w.next(p)) {
            if (w.u + 1 < u1 && w.j + 1 < p.nb) continue;  // not the last unit of a segment
            if (!ws) {
                grid_dependency_wait();  // the previous kernels may still read the workspace
                ws = p.ws + (size_t)p.cta_seg[blockIdx.x] * p.npad * kTcRows + rloc;
            }
            if (!wait_bar(acc_full, seg & 1, abort_flag, p.status, p.wait_tries)) break;
            tc_fence_after();
            float* dst = ws + (size_t)seg * p.npad * kTcRows;
            // (the epilogue warps share their sub-partitions with issue-bound
            // decoders: a full chunk is 16 plain stores at immediate offsets)
            auto store16 = [&](const uint32_t (&v)[16], int c0) {
                float* d = dst + (size_t)c0 * kTcRows;
                if (c0 + 16 <= p.batch) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) d[e * kTcRows] = __uint_as_float(v[e]);
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if (c0 + e < p.batch) d[e * kTcRows] = __uint_as_float(v[e]);
                }
            };
            // two register sets: the next chunk's load is in flight while this one is stored
            uint32_t va[16], vb[16];
            tmem_ld16(tbase, va);
            for (int c0 = 0; c0 < p.npad; c0 += 32) {
                tmem_ld_wait(va);
                const bool more = c0 + 16 < p.npad;
                if (more) tmem_ld16(tbase + (uint32_t)(c0 + 16), vb);
                store16(va, c0);
                if (!more) break;
                tmem_ld_wait(vb);
                if (c0 + 32 < p.npad) tmem_ld16(tbase + (uint32_t)(c0 + 32), va);
                store16(vb, c0 + 16);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
            ++seg;
        }
    }
    grid_launch_dependents();
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTcTmemCols);
    }
}

template <int CODE, int V, bool L16>
static cudaError_t launch_gemm_t(const GemmArgs& a, int grid, size_t smem, cudaStream_t st, bool split = false) {
    if constexpr (CODE == kCode1MAD || CODE == kCode3INST) {
        if (split) {
            cudaError_t e = ensure_smem_limit<trellis_gemm_kernel<CODE, V, L16, true>>(kTcMaxSmem);
            if (e != cudaSuccess) return e;
            return launch_pdl(trellis_gemm_kernel<CODE, V, L16, true>, dim3(grid), dim3(kTcThreads), smem, st, a);
        }
    }
    auto kern = trellis_gemm_kernel<CODE, V, L16, false>;
    cudaError_t e = ensure_smem_limit<trellis_gemm_kernel<CODE, V, L16, false>>(kTcMaxSmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(grid), dim3(kTcThreads), smem, st, a);
}

// Ring depths: a code ring of kTcMaxCodeSlots blocks (the code words come
// from HBM: a deep ring hides their latency) with as many stage slots as
// fit, if that leaves at least 4; else the most stage slots, then the deepest
// code ring that fit in shared memory.
size_t tc_smem_bytes(const Layer& L, int npad, int* stages, int* code_slots, bool split) {
    const int xrows = split ? 2 * npad : npad;  // 128-byte x' rows of one stage
    const int max_stages = split ? kTcMaxStagesSplit : kTcMaxStages;
    int k2max = 0;
    for (int i = 0; i < L.nparts; ++i) k2max = L.parts[i].k2 > k2max ? L.parts[i].k2 : k2max;
    const int code_slot_words = (kTcRows / kRowTile) * 64 * k2max;
    const int lut_entries = uses_table(L.code) ? (1 << L.Q) : 0;
    for (int s = max_stages; s >= 4; --s) {
        const TcSmem lay = tc_smem_layout(s, kTcMaxCodeSlots, xrows, code_slot_words, lut_entries);
        if (lay.total + 1024 <= kTcMaxSmem) {
            *stages = s;
            *code_slots = kTcMaxCodeSlots;
            return (size_t)lay.total + 1024;
        }
    }
    for (int s = max_stages; s >= 2; --s) {
        for (int c = kTcMaxCodeSlots; c >= 2; --c) {
            const TcSmem lay = tc_smem_layout(s, c, xrows, code_slot_words, lut_entries);
            if (lay.total + 1024 <= kTcMaxSmem) {
                *stages = s;
                *code_slots = c;
                return (size_t)lay.total + 1024;
            }
        }
    }
    *stages = *code_slots = 0;
    return 0;
}

int tc_units(const Layer& L) {
    int tiles = 0;
    for (int i = 0; i < L.nparts; ++i) tiles += (L.parts[i].rows + kTcRows - 1) / kTcRows;
    return tiles * (L.n / kT);
}

bool tc_split(const Layer& L, int npad) {
    return (L.code == kCode1MAD || L.code == kCode3INST) && L.V == 1 && npad <= kTcMaxSplitN;
}

int tc_grid(const Layer& L) {
    const int units = tc_units(L);
    return units < L.num_sms ? units : L.num_sms;
}

// The stream-K segments in unit order: CTA c runs units [c U / G, (c+1) U / G)
// and starts a new segment at its first unit and at every tile's first block.
// cta_seg[c] = slot of CTA c's first segment (c <= G, cta_seg[G] = all
// segments); tile_seg[t] = slot of tile t's first segment (t <= tiles).  The
// segments of tile t are the slots tile_seg[t] .. tile_seg[t + 1] - 1.
void tc_segments(const Layer& L, std::vector<int>& cta_seg, std::vector<int>& tile_seg) {
    const int nb = L.n / kT, units = tc_units(L), G = tc_grid(L);
    const int tiles = units / nb;
    cta_seg.assign(G + 1, 0);
    tile_seg.assign(tiles + 1, 0);
    int slot = 0;
    for (int c = 0; c < G; ++c) {
        const int u0 = (int)((long long)c * units / G), u1 = (int)((long long)(c + 1) * units / G);
        cta_seg[c] = slot;
        for (int u = u0; u < u1; ++u) {
            if (u == u0 || u % nb == 0) {
                if (u % nb == 0) tile_seg[u / nb] = slot;
                ++slot;
            }
        }
    }
    cta_seg[G] = slot;
    tile_seg[tiles] = slot;
}

cudaError_t launch_gemm_tc(const Layer& L, const void* xt, int batch, int npad, float* ws, cudaStream_t st) {
    GemmArgs a;
    int k2max = 0;
    a.nparts = L.nparts;
    a.nb = L.n / kT;
    int tiles = 0;
    for (int i = 0; i < L.nparts; ++i) {
        const Part& pt = L.parts[i];
        a.part[i].words = L.words + pt.word_off;
        a.part[i].rt = pt.rows / kRowTile;
        a.part[i].k2 = pt.k2;
        a.part[i].tiles = (pt.rows + kTcRows - 1) / kTcRows;
        tiles += a.part[i].tiles;
        k2max = pt.k2 > k2max ? pt.k2 : k2max;
    }
    for (int i = L.nparts; i < kMaxParts; ++i) a.part[i] = a.part[0];
    a.units = tiles * a.nb;
    a.lmask = (1u << L.L) - 1u;
    a.qshift = 32 - L.Q;
    a.lut = L.lut;
    a.lut_entries = uses_table(L.code) ? (1 << L.Q) : 0;
    a.xt = (const uint8_t*)xt;
    a.npad = npad;
    a.batch = batch;
    a.ws = ws;
    a.cta_seg = L.tc_seg;
    a.status = L.status;
    a.wait_tries = L.test_wait_tries > 0 ? L.test_wait_tries : kTcWaitTries;
    a.withhold = L.test_withhold;
    a.code_slot_words = (kTcRows / kRowTile) * 64 * k2max;
    const bool split = tc_split(L, npad);
    const size_t smem = tc_smem_bytes(L, npad, &a.stages, &a.code_slots, split);
    if (smem == 0) return cudaErrorInvalidValue;
    const int grid = tc_grid(L);
    const bool l16 = L.L == 16;
    if (L.code == kCode1MAD) return l16 ? launch_gemm_t<kCode1MAD, 1, true>(a, grid, smem, st, split)
                                        : launch_gemm_t<kCode1MAD, 1, false>(a, grid, smem, st, split);
    if (L.code == kCode3INST) return l16 ? launch_gemm_t<kCode3INST, 1, true>(a, grid, smem, st, split)
                                         : launch_gemm_t<kCode3INST, 1, false>(a, grid, smem, st, split);
    if (L.code == kCodeTable) {
        if (l16) return cudaErrorInvalidValue;  // codebooks hold at most 2^9 entries
        return L.V == 1 ? launch_gemm_t<kCodeTable, 1, false>(a, grid, smem, st)
                        : launch_gemm_t<kCodeTable, 2, false>(a, grid, smem, st);
    }
    if (L.code == kCodeE8P) return l16 ? launch_gemm_t<kCodeE8P, 8, true>(a, grid, smem, st) : cudaErrorInvalidValue;
    if (L.V == 1) return l16 ? launch_gemm_t<kCodeHYB, 1, true>(a, grid, smem, st)
                             : launch_gemm_t<kCodeHYB, 1, false>(a, grid, smem, st);
    return l16 ? launch_gemm_t<kCodeHYB, 2, true>(a, grid, smem, st) : launch_gemm_t<kCodeHYB, 2, false>(a, grid, smem, st);
}

cudaError_t prepare_gemm_kernels(const Layer& L) {
    const bool l16 = L.L == 16;
#define QLK_PREP(C, V_, L_) preload_kernel<trellis_gemm_kernel<C, V_, L_, false>>(kTcMaxSmem)
#define QLK_PREP2(C, L_) \
    (QLK_PREP(C, 1, L_) == cudaSuccess ? preload_kernel<trellis_gemm_kernel<C, 1, L_, true>>(kTcMaxSmem) : cudaErrorUnknown)
    if (L.code == kCode1MAD) return l16 ? QLK_PREP2(kCode1MAD, true) : QLK_PREP2(kCode1MAD, false);
    if (L.code == kCode3INST) return l16 ? QLK_PREP2(kCode3INST, true) : QLK_PREP2(kCode3INST, false);
    if (L.code == kCodeTable) {
        if (l16) return cudaErrorInvalidValue;
        return L.V == 1 ? QLK_PREP(kCodeTable, 1, false) : QLK_PREP(kCodeTable, 2, false);
    }
    if (L.code == kCodeE8P) return l16 ? QLK_PREP(kCodeE8P, 8, true) : cudaErrorInvalidValue;
    if (L.V == 1) return l16 ? QLK_PREP(kCodeHYB, 1, true) : QLK_PREP(kCodeHYB, 1, false);
    return l16 ? QLK_PREP(kCodeHYB, 2, true) : QLK_PREP(kCodeHYB, 2, false);
#undef QLK_PREP
#undef QLK_PREP2
}

}  // namespace qlk
