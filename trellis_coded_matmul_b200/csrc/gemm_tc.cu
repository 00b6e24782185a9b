// gemm_tc.cu -- decode-to-shared-memory + tcgen05 tensor-core GEMM for
// batches above 8: z[b][row] = sum_c W_hat[row][c] x'[b][c].
//
// The contraction is dense (M = 128 rows of W_hat per CTA, N = batch padded
// to 16, K = n), so it runs on the 5th-generation tensor cores: fp16 A and B
// operands in shared memory (K-major, 128-byte swizzle), fp32 accumulator in
// tensor memory, one thread issuing tcgen05.mma.  The A operand is produced
// on the fly by decoder warps from the trellis code words (QTIP discussion:
// decode with computed codes or a small table; the bitshift trellis makes any
// run of steps decodable from the bits around it), so decoded weights never
// reach HBM.  Warp roles, one 128-row tile per CTA:
//   MMA warp       allocates tensor memory; one lane issues the MMAs of a
//                  stage (4 x K=16) and commits them to the stages' "empty"
//                  barriers;
//   x' producer    bulk copy of the x' tile of each 64-column K stage (x' is
//                  stored pre-swizzled, one copy per stage);
//   code producer  bulk copies of the code words, one 256-column block of 8
//                  row tiles at a time, up to 4 blocks ahead;
//   16 decoders    two groups of 8 that take alternate stages; a warp decodes
//                  16 rows x 64 columns of its stage (lane = one row, 32
//                  consecutive trellis steps) into the A stage;
//   all warps      at the end read the accumulator back and store z.
// Every wait on an mbarrier is bounded; on expiry the CTA records
// kStatusTimeout in the handle's status word, abandons its tile and frees its
// tensor memory.
#include <cuda_fp16.h>

#include "codes.cuh"
#include "internal.h"
#include "layout.cuh"
#include "tc_ptx.cuh"

namespace qlk {

constexpr int kTcRows = 128;         // M of one tile
constexpr int kTcK = 64;             // K of one stage (one 128-byte swizzled row of fp16)
constexpr int kTcDecoders = 16;      // decoder warps: two groups of 8 decode alternate stages
constexpr int kTcGroup = 8;          // decoder warps per group (one per 16-row tile)
constexpr int kTcWarps = 20;         // 5 per SM sub-partition (a warp runs on sub-partition warp % 4)
constexpr int kTcThreads = kTcWarps * 32;
// Warp roles.  The MMA issuer shares its sub-partition only with the two
// producers and one decoder, so its short instruction sequence per stage is
// not starved of issue slots by the decoders.
constexpr int kWarpMma = 0, kWarpXProd = 4, kWarpCodeProd = 8, kWarpSpare = 16;
__device__ __forceinline__ int decoder_index(int w) {  // 0..15 for decoder warps, -1 otherwise
    if (w == kWarpMma || w == kWarpXProd || w == kWarpCodeProd || w == kWarpSpare) return -1;
    return w - 1 - (w > kWarpXProd) - (w > kWarpCodeProd) - (w > kWarpSpare);
}
constexpr int kTcAStages = 4;      // decoded A tiles in flight
constexpr int kTcMaxBStages = 8;   // x' tiles in flight (as many as shared memory allows)
constexpr int kTcMaxCodeSlots = 4;
constexpr int kTcWaitTries = 4096;           // try_wait calls of up to kTcSuspendNs each (a few seconds in all)
constexpr uint32_t kTcSuspendNs = 1000000;   // before a wait is declared expired

struct TcPart {
    const uint32_t* words;  // kernel layout
    int rt;                 // row tiles of 16 rows
    int row0;               // first layer row
    int k;                  // bits per weight
    int tiles;              // 128-row tiles
};

struct GemmArgs {
    TcPart part[2];
    int nparts;
    int nb;                 // 256-column blocks per row
    uint32_t lmask;
    int qshift;
    const uint32_t* lut;
    int lut_entries;
    const uint8_t* xt;      // x' tiles: [n / 64][npad][128 B, swizzled]
    int npad;               // MMA N: batch padded to a multiple of 16 (<= 256)
    int batch;              // valid columns
    float* z;               // [batch][m]
    int m;
    int* status;
    int a_stages;           // depth of the A (decoded tile) ring
    int b_stages;           // depth of the B (x' tile) ring
    int code_slots;         // depth of the code-word ring
    int code_slot_words;    // words of one code-ring slot (8 units at the largest k)
    uint32_t tmem_cols;
};

struct TcSmem {  // offsets in bytes from the 1024-aligned dynamic shared memory base
    int a, b, code, lut, bar, total;
};

__host__ __device__ inline TcSmem tc_smem_layout(int a_stages, int b_stages, int code_slots, int npad,
                                                  int code_slot_words, int lut_entries) {
    TcSmem s;
    s.a = 0;
    s.b = s.a + a_stages * kTcRows * 128;
    s.code = s.b + b_stages * npad * 128;
    s.lut = s.code + code_slots * code_slot_words * 4;
    s.bar = s.lut + lut_entries * 32 * 4;
    s.total = s.bar + 512;  // up to 33 mbarriers, the TMEM base address and the abort flag
    return s;
}

// One decoder thread's 32 weights of a stage: row r of its row tile, trellis
// steps [32 hq / V, 32 (hq + 1) / V) of the quarter-block (64 columns).
// cw[0] holds the 32 bits before the run, cw[1..K] its K words.  Output:
// 16 half2 words, columns 2i and 2i + 1 of the run in word i.
template <int CODE, int K, int V, bool L16>
__device__ __forceinline__ void decode_run32(const uint32_t (&cw)[K + 1], uint32_t lmask, const uint32_t* lut_lane,
                                             int qshift, uint32_t (&out)[16]) {
    constexpr int kV = K * V;
    constexpr int NS = 32 / V;
    constexpr bool kPair = (16 % kV) == 0;
    constexpr int P = kPair ? 16 / kV : 1;
    uint32_t s[NS];
#pragma unroll
    for (int t = 0; t < NS; ++t) {
        if (kPair) {
            if (((t / P) & 1) == 0) state_pair<kV, L16>(cw, t, lmask, s[t], s[t + P]);
        } else {
            s[t] = state_one<kV, L16>(cw, t, lmask);
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if (V == 1)
            out[i] = code_pair<CODE>(s[2 * i], s[2 * i + 1], lut_lane, qshift);
        else
            out[i] = code_hyb_v2(s[i], lut_lane, qshift);
    }
}

// Decode one stage (quarter q of the block whose 8 units sit at shared address
// `code`) for row tile `tdx` of the CTA into the swizzled A stage at `a_stage`.
template <int CODE, int K, int V, bool L16>
__device__ __forceinline__ void decode_stage(uint32_t code, uint32_t a_stage, int tdx, int q, int lane,
                                             uint32_t lmask, const uint32_t* lut_lane, int qshift) {
    using UL = UnitLayout<K>;
    const uint32_t unit = code + tdx * UL::UW * 4;
    const int r = lane & 15, hq = lane >> 4;
    const int h = r >> 3, g = r & 7;
    auto word = [&](int slot_lane, int e) -> uint32_t {
        return lds32(unit + 4 * (((h * UL::NV + e / UL::VW) * 32 + slot_lane) * UL::VW + (e % UL::VW)));
    };
    uint32_t cw[K + 1];
    const int own = 4 * g + q;
    cw[0] = hq ? word(own, K - 1) : word(4 * g + ((q + 3) & 3), 2 * K - 1);
#pragma unroll
    for (int e = 0; e < K; ++e) cw[1 + e] = word(own, hq * K + e);
    uint32_t out[16];
    decode_run32<CODE, K, V, L16>(cw, lmask, lut_lane, qshift, out);
    const int row = tdx * 16 + r;
    const uint32_t rowp = a_stage + row * 128;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int chunk = (4 * hq + i) ^ (row & 7);
        sts128(rowp + chunk * 16, out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
    }
}

// Bounded wait; returns false (and raises the CTA's abort flag) on expiry.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status) {
    if (mbar_test_wait(bar, parity)) return true;  // already complete: no suspension
    for (int i = 0; i < kTcWaitTries; ++i) {
        if (mbar_try_wait(bar, parity, kTcSuspendNs)) return true;
        if (*abort_flag) return false;
    }
    *abort_flag = 1;
    atomicOr(status, kStatusTimeout);
    return false;
}

template <int CODE, int V, bool L16>
__global__ void __launch_bounds__(kTcThreads, 1) gemm_tc_kernel(GemmArgs p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base, derived by indexing the shared array so that
    // accesses through it stay shared-memory accesses
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const TcSmem L = tc_smem_layout(p.a_stages, p.b_stages, p.code_slots, p.npad, p.code_slot_words, p.lut_entries);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
    // barrier slots: code_full[C], code_empty[C], a_full[SA], a_empty[SA], b_full[SB],
    // b_empty[SB], mma_done; then the tmem base address and the abort flag
    const int SA = p.a_stages, SB = p.b_stages, C = p.code_slots;
    const uint32_t bar0 = smem_u32(bars);
    auto code_full = [&](int i) { return bar0 + 8 * i; };
    auto code_empty = [&](int i) { return bar0 + 8 * (C + i); };
    auto a_full = [&](int i) { return bar0 + 8 * (2 * C + i); };
    auto a_empty = [&](int i) { return bar0 + 8 * (2 * C + SA + i); };
    auto b_full = [&](int i) { return bar0 + 8 * (2 * C + 2 * SA + i); };
    auto b_empty = [&](int i) { return bar0 + 8 * (2 * C + 2 * SA + SB + i); };
    const uint32_t mma_done = bar0 + 8 * (2 * C + 2 * SA + 2 * SB);
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(bars + 2 * C + 2 * SA + 2 * SB + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // which part and tile
    int pi = 0, tile = blockIdx.x;
    if (p.nparts > 1 && tile >= p.part[0].tiles) {
        tile -= p.part[0].tiles;
        pi = 1;
    }
    const TcPart part = p.part[pi];
    const int R0 = tile * (kTcRows / kRowTile);        // first row tile of this CTA
    int ntiles16 = part.rt - R0;                        // row tiles present (ragged last tile)
    if (ntiles16 > kTcRows / kRowTile) ntiles16 = kTcRows / kRowTile;
    const int k = part.k;
    const int unit_words = 128 * k;
    const int nstages = p.nb * 4;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C; ++i) {
            mbar_init(code_full(i), 1);
            mbar_init(code_empty(i), kTcDecoders);  // every decoder warp releases each block once
        }
        for (int i = 0; i < SA; ++i) {
            mbar_init(a_full(i), kTcGroup);  // one group fills a stage
            mbar_init(a_empty(i), 1);        // MMA commit
        }
        for (int i = 0; i < SB; ++i) {
            mbar_init(b_full(i), 1);
            mbar_init(b_empty(i), 1);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    uint32_t* lut_smem = reinterpret_cast<uint32_t*>(smem + L.lut);
    if (CODE == kCodeHYB)
        for (int i = threadIdx.x; i < p.lut_entries * 32; i += blockDim.x) lut_smem[i] = p.lut[i >> 5];
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(tmem_base_smem), p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;

    const int dec = decoder_index(warp);
    if (warp == kWarpXProd) {
        // ---------------- x' producer ----------------
        grid_dependency_wait();  // x' comes from the previous kernel
        for (int s = 0; s < nstages && !*abort_flag; ++s) {
            const int st = s % SB, round = s / SB;
            if (!wait_bar(b_empty(st), (round & 1) ^ 1, abort_flag, p.status)) break;
            if (lane == 0) {
                const uint32_t bytes = (uint32_t)p.npad * 128;
                mbar_arrive_expect_tx(b_full(st), bytes);
                bulk_g2s(smem_u32(smem + L.b) + st * bytes, p.xt + (size_t)s * bytes, bytes, b_full(st));
            }
            __syncwarp();
        }
    } else if (warp == kWarpCodeProd) {
        // ---------------- code-word producer ----------------
        const uint8_t* code_src = reinterpret_cast<const uint8_t*>(part.words);
        for (int j = 0; j < p.nb && !*abort_flag; ++j) {
            const int slot = j % C, round = j / C;
            if (!wait_bar(code_empty(slot), (round & 1) ^ 1, abort_flag, p.status)) break;
            if (lane == 0) mbar_arrive_expect_tx(code_full(slot), (uint32_t)(ntiles16 * unit_words * 4));
            __syncwarp();
            if (lane < ntiles16) {
                const size_t unit = (size_t)(R0 + lane) * p.nb + j;
                bulk_g2s(smem_u32(smem + L.code) + (uint32_t)(slot * p.code_slot_words + lane * unit_words) * 4,
                         code_src + unit * unit_words * 4, (uint32_t)unit_words * 4, code_full(slot));
            }
            __syncwarp();
        }
    } else if (warp == kWarpMma) {
        // ---------------- MMA issuer ----------------
        // The descriptors of all stages differ only in the 14-bit start-address
        // field (low word, 16-byte units, no carry out of it below 256 KB):
        // build the words once and step the low word.
        const uint32_t idesc = idesc_f16_f32(kTcRows, p.npad);
        const uint64_t a_desc0 = smem_desc_k_sw128(smem_u32(smem + L.a));
        const uint64_t b_desc0 = smem_desc_k_sw128(smem_u32(smem + L.b));
        const uint32_t a_hi = (uint32_t)(a_desc0 >> 32), b_hi = (uint32_t)(b_desc0 >> 32);
        const uint32_t a_lo0 = (uint32_t)a_desc0, b_lo0 = (uint32_t)b_desc0;
        const uint32_t b_step = (uint32_t)p.npad * 128 / 16;
        int sa = 0, sb = 0, pa = 0, pb = 0;
        for (int s = 0; s < nstages; ++s) {
            if (!wait_bar(a_full(sa), pa, abort_flag, p.status)) break;
            if (!wait_bar(b_full(sb), pb, abort_flag, p.status)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t a_lo = a_lo0 + (uint32_t)sa * (kTcRows * 128 / 16);
                const uint32_t b_lo = b_lo0 + (uint32_t)sb * b_step;
#pragma unroll
                for (int kk = 0; kk < kTcK / 16; ++kk) {
                    tc_mma_f16(tmem, ((uint64_t)a_hi << 32) | (a_lo + kk * 2), ((uint64_t)b_hi << 32) | (b_lo + kk * 2),
                               idesc, (s > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(a_empty(sa));
                tc_commit(b_empty(sb));
                if (s == nstages - 1) tc_commit(mma_done);
            }
            __syncwarp();
            if (++sa == SA) sa = 0, pa ^= 1;
            if (++sb == SB) sb = 0, pb ^= 1;
        }
    } else if (dec >= 0) {
        // ---------------- decoders ----------------
        const int grp = dec / kTcGroup, tdx = dec % kTcGroup;
        const uint32_t* lut_lane = lut_smem + lane;
        const uint32_t code_base = smem_u32(smem + L.code);
        for (int s = grp; s < nstages && !*abort_flag; s += 2) {
            const int j = s >> 2, q = s & 3;
            const int slot = j % C;
            if (q < 2 && !wait_bar(code_full(slot), (j / C) & 1, abort_flag, p.status)) break;
            const int st = s % SA, round = s / SA;
            if (!wait_bar(a_empty(st), (round & 1) ^ 1, abort_flag, p.status)) break;
            if (tdx < ntiles16) {
                const uint32_t code = code_base + slot * p.code_slot_words * 4;
                const uint32_t a_stage = smem_u32(smem + L.a) + st * kTcRows * 128;
                switch (k) {
                    case 1: decode_stage<CODE, 1, V, L16>(code, a_stage, tdx, q, lane, p.lmask, lut_lane, p.qshift); break;
                    case 2: decode_stage<CODE, 2, V, L16>(code, a_stage, tdx, q, lane, p.lmask, lut_lane, p.qshift); break;
                    case 3: decode_stage<CODE, 3, V, L16>(code, a_stage, tdx, q, lane, p.lmask, lut_lane, p.qshift); break;
                    default: decode_stage<CODE, 4, V, L16>(code, a_stage, tdx, q, lane, p.lmask, lut_lane, p.qshift); break;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(a_full(st));
                if (q >= 2) mbar_arrive(code_empty(slot));  // this group's last stage of the block
            }
        }
    }
    // ---------------- epilogue (all warps): TMEM -> z ----------------
    grid_dependency_wait();
    if (wait_bar(mma_done, 0, abort_flag, p.status)) {
        tc_fence_after();
        const int quarter = warp & 3;        // TMEM lanes this warp may read
        const int share = warp >> 2;         // kTcWarps / 4 warps per quarter split the columns
        const int per = kTcWarps / 4;
        const int row = part.row0 + R0 * kRowTile + quarter * 32 + lane;
        const bool row_ok = (R0 * kRowTile + quarter * 32 + lane) < part.rt * kRowTile;
        const int chunks = p.npad / 16;      // 16-column TMEM loads
        for (int ci = share * chunks / per; ci < (share + 1) * chunks / per; ++ci) {
            const int c0 = ci * 16;
            uint32_t v[16];
            tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0, v);
            tmem_ld_wait();
            if (row_ok) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (c0 + i < p.batch) p.z[(size_t)(c0 + i) * p.m + row] = __uint_as_float(v[i]);
            }
        }
    }
    grid_launch_dependents();
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, p.tmem_cols);
    }
}

template <int CODE, int V, bool L16>
static cudaError_t launch_gemm_t(const GemmArgs& a, int grid, size_t smem, cudaStream_t st) {
    auto kern = gemm_tc_kernel<CODE, V, L16>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcMaxSmem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    return launch_pdl(kern, dim3(grid), dim3(kTcThreads), smem, st, a);
}

// Ring depths: 4 A stages, then the deepest code ring (4..2 slots) and the
// deepest x' ring (8..2 stages) that fit in shared memory.
size_t tc_smem_bytes(const Layer& L, int npad, int* a_stages, int* b_stages, int* code_slots) {
    int kmax = 0;
    for (int i = 0; i < L.nparts; ++i) kmax = L.parts[i].k > kmax ? L.parts[i].k : kmax;
    const int code_slot_words = (kTcRows / kRowTile) * 128 * kmax;
    const int lut_entries = L.code == kCodeHYB ? (1 << L.Q) : 0;
    for (int sa = kTcAStages; sa >= 2; --sa) {
        for (int c = kTcMaxCodeSlots; c >= 2; --c) {
            for (int sb = kTcMaxBStages; sb >= 2; --sb) {
                const TcSmem lay = tc_smem_layout(sa, sb, c, npad, code_slot_words, lut_entries);
                if (lay.total + 1024 <= kTcMaxSmem && (sb >= 4 || c == 2)) {
                    *a_stages = sa;
                    *b_stages = sb;
                    *code_slots = c;
                    return (size_t)lay.total + 1024;
                }
            }
        }
    }
    *a_stages = *b_stages = *code_slots = 0;
    return 0;
}

cudaError_t launch_gemm_tc(const Layer& L, const void* xt, int batch, int npad, float* z, cudaStream_t st) {
    GemmArgs a;
    int kmax = 0;
    a.nparts = L.nparts;
    int grid = 0;
    for (int i = 0; i < L.nparts; ++i) {
        const Part& pt = L.parts[i];
        a.part[i].words = L.words + pt.word_off;
        a.part[i].rt = pt.rows / kRowTile;
        a.part[i].row0 = pt.row0;
        a.part[i].k = pt.k;
        a.part[i].tiles = (pt.rows + kTcRows - 1) / kTcRows;
        grid += a.part[i].tiles;
        kmax = pt.k > kmax ? pt.k : kmax;
    }
    if (L.nparts == 1) a.part[1] = a.part[0];
    a.nb = L.n / kT;
    a.lmask = (1u << L.L) - 1u;
    a.qshift = 32 - L.Q;
    a.lut = L.lut;
    a.lut_entries = L.code == kCodeHYB ? (1 << L.Q) : 0;
    a.xt = (const uint8_t*)xt;
    a.npad = npad;
    a.batch = batch;
    a.z = z;
    a.m = L.m;
    a.status = L.status;
    a.code_slot_words = (kTcRows / kRowTile) * 128 * kmax;
    uint32_t cols = 32;
    while (cols < (uint32_t)npad) cols <<= 1;
    a.tmem_cols = cols;
    const size_t smem = tc_smem_bytes(L, npad, &a.a_stages, &a.b_stages, &a.code_slots);
    if (smem == 0) return cudaErrorInvalidValue;
    const bool l16 = L.L == 16;
    if (L.code == kCode1MAD) return l16 ? launch_gemm_t<kCode1MAD, 1, true>(a, grid, smem, st)
                                        : launch_gemm_t<kCode1MAD, 1, false>(a, grid, smem, st);
    if (L.code == kCode3INST) return l16 ? launch_gemm_t<kCode3INST, 1, true>(a, grid, smem, st)
                                         : launch_gemm_t<kCode3INST, 1, false>(a, grid, smem, st);
    if (L.V == 1) return l16 ? launch_gemm_t<kCodeHYB, 1, true>(a, grid, smem, st)
                             : launch_gemm_t<kCodeHYB, 1, false>(a, grid, smem, st);
    return l16 ? launch_gemm_t<kCodeHYB, 2, true>(a, grid, smem, st) : launch_gemm_t<kCodeHYB, 2, false>(a, grid, smem, st);
}

}  // namespace qlk
