// internal.h -- the handle and the kernel launchers shared by the library's .cu files.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <vector>

#include "../../include/qlinear.h"

namespace qlk {

constexpr int kT = 256;            // columns per trellis block
constexpr int kRowTile = 16;       // rows per decode tile (the m16n8k16 M dimension)
constexpr int kMaxHadamard = 32768;

constexpr int kGemvMaxWarps = 16;        // decode-GEMV: warps of its one CTA per SM (<= 128 registers/thread)
constexpr int kGemvMaxSmem = 200 * 1024;  // decode-GEMV dynamic shared memory limit
constexpr int kFuseOutElems = 256;  // batch * m up to which the GEMV's last CTA per block does the output transform
constexpr int kXInKernelMaxBatch = 2;          // batches up to which every GEMV CTA computes x' itself
constexpr int kXInKernelMaxBytes = 48 * 1024;  // and x' fits in this much shared memory
constexpr int kMaxParts = 8;          // row parts of one layer (layers fused along m, own bitwidth each)
constexpr int kGemvMaxBatch = 8;      // larger batches use the tensor-core GEMM
constexpr int kTcMaxN = 256;          // tensor-core GEMM: batch columns per pass
constexpr int kTcMaxSmem = 232448;    // 227 KB of dynamic shared memory per CTA

// Device status word bits (qlinear_get_status).
constexpr int kStatusBadSign = 1;
constexpr int kStatusTimeout = 2;
constexpr int kStatusBounds = 4;
constexpr int kStatusBadInput = 8;   // the encoder found no finite walk (non-finite source values)

// One run of rows sharing a bitrate.  Its code words are stored re-laid out
// for the decode kernels (see layout.cuh) starting at word `word_off` of the
// handle's word buffer.  The bitrate k = kv / V bits per weight may be a half
// number; the kernels take it as k2 = 2k (a whole number of bits per two
// weights, which is also the code words of one thread-row of a unit).
struct Part {
    int row0;
    int rows;
    int kv;       // bits per trellis step
    int k2;       // 2k = 2 kv / V
    size_t word_off;
    size_t n_words;
};

struct Layer {
    int device;
    int m, n, L, V, code, Q;  // Q: table index bits of HYB and of the table code (= L), else 0
    float alpha;
    int B_n, B_m;
    int nparts;
    Part parts[kMaxParts];
    uint32_t* words;      // all parts, kernel layout
    uint32_t* sin_bits;   // bit i set <=> s_in[i] == -1
    uint32_t* sout_bits;
    uint32_t* lut;        // HYB / table code: 2^Q words (table code: Q = L) (V = 2: value 0 low half,
                          // value 1 high; V = 1: low half)
    int* status;          // device status word
    // scratch, grown on demand
    void* xp;             // transformed input x' (fp16)
    size_t xp_bytes;
    void* acc;            // the output-block tickets (int [m / B_m], padded to 256 bytes), then z = W_hat x'
                          // before the output transform (fp32 [batch][m]); all-zero between forwards
    size_t acc_bytes;
    int acc_dirty;        // z or a ticket may be non-zero (a forward failed part-way)
    int last_launches;    // kernels launched by the most recent forward
    int last_batch;       // batch of the most recent successful forward (0: none)
    void* host_stage;     // device staging for qlinear_forward_host (x then y)
    size_t host_stage_bytes;
    // tensor-core GEMM (batch > 8): its stream-K segment table (device, written at
    // create: the slot of each CTA's first segment [grid + 1], then the slot of
    // each 128-row tile's first segment [tiles + 1]) and the partial-sum workspace
    // ([segment slot][npad][128] fp32, grown on demand)
    int* tc_seg;
    const int* tc_tile_seg;
    int tc_slots;
    void* tcws;
    size_t tcws_bytes;
    int num_sms;
    // test hooks of the tensor-core GEMM (qlinear_test_stall): a shorter
    // limit on its bounded waits and a stage that never arrives
    int test_wait_tries;
    int test_withhold;
    // profiling ring (qlinear_profile_enable)
    cudaEvent_t* prof_ev;  // 2 * prof_cap events
    int prof_cap;
    int prof_next;
    int prof_count;
};

// Programmatic dependent launch (PDL): the kernel may start while the
// previous kernel on the stream is still running; it must call
// grid_dependency_wait() before touching anything that kernel (or any earlier
// work on the stream) writes, and calls grid_launch_dependents() to let the
// next kernel start early.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Raise kernel Kern's dynamic shared-memory limit to `bytes` on the current
// device, once per device (the attribute is per device context); devices
// numbered 64 and above set it on every call.  Safe to call from several
// host threads.
template <auto Kern>
cudaError_t ensure_smem_limit(int bytes) {
    static std::atomic<unsigned long long> done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// Load kernel Kern's code on the current device now and raise its
// shared-memory limit to `smem_limit` bytes (0: leave it).  Under lazy module
// loading a kernel is otherwise loaded at its first launch, which may
// allocate device memory and must not happen inside a stream capture; create
// calls this for every kernel a handle's forwards and decodes can launch.
template <auto Kern>
cudaError_t preload_kernel(int smem_limit) {
    cudaFuncAttributes attr;
    cudaError_t e = cudaFuncGetAttributes(&attr, Kern);
    if (e == cudaSuccess && smem_limit > 0) e = ensure_smem_limit<Kern>(smem_limit);
    return e;
}

// ---- launchers (return cudaError_t of the launch) ----
cudaError_t launch_relayout(const uint32_t* src, uint32_t* dst, const Part& part, int n, cudaStream_t st);
cudaError_t launch_pack_signs(const int8_t* s, int count, uint32_t* bits, int* status, cudaStream_t st);
cudaError_t launch_copy_lut(const void* lut_f16, int Q, int V, uint32_t* dst, cudaStream_t st);

// x (fp16 [batch][n]) -> x' as the decode-GEMV's step words (xstep.cuh).
cudaError_t launch_rht_in_xstep(const Layer& L, const void* x, int batch, void* xstep, cudaStream_t st);
// x (fp16 [batch][n]) -> x' as tensor-core operand tiles: [n/64][npad][128 B],
// the 16-byte chunk c of row b at chunk c ^ (b % 8) (rows >= batch untouched);
// with dup, every value twice along K ([2n/64][npad][128 B], K index 2c and
// 2c + 1 for column c).
cudaError_t launch_rht_in_umma(const Layer& L, const void* x, int batch, int npad, void* xt, cudaStream_t st,
                               bool dup = false);
// z (fp32 [batch][m]) -> y = alpha zscale s_out (H_m z), fp32 or fp16; re-zeroes the consumed z.
cudaError_t launch_rht_out(const Layer& L, float* z, int batch, void* y, int y_dtype, cudaStream_t st,
                           float zscale = 1.0f);
// The tensor-core GEMM's partial sums (launch_gemm_tc's workspace, npad
// columns per slot) -> y = alpha s_out (H_m z), z = the sum of each tile's
// segment slots; the workspace is only read.
cudaError_t launch_rht_out_tc(const Layer& L, const float* ws, int batch, int npad, void* y, int y_dtype,
                              cudaStream_t st, float zscale = 1.0f);

// How one decode-GEMV launch is shaped: grid and CTA size, whether the
// output transform runs in its epilogue, and its dynamic shared memory.
struct GemvPlan {
    int grid, threads;
    bool fuse_out;  // output transform in the GEMV's epilogue (else launch_rht_out after it)
    int x_e;        // > 0: every CTA computes x' from x into shared memory (E entries a thread), no input-transform kernel
    int xs_word0;   // first shared-memory word of that x'
    int smem_bytes;
};
GemvPlan plan_gemv(const Layer& L, int batch);
// Bytes of x' step words for `batch` rows (the input-transform kernel's output
// when the plan does not compute x' in-kernel).
size_t gemv_xstep_bytes(const Layer& L, int batch);
// The factor between the decode-GEMV's z and W_hat x' (the 1MAD code's C1, else 1).
float gemv_z_scale(const Layer& L);
// The forward for batch <= 8: decode-GEMV over all row parts into z, x' from
// x in the kernel itself (pl.x_e > 0) or from xstep (the input-transform
// kernel's output), and (pl.fuse_out) the output transform into y (fp32 or
// fp16) by the CTA that completes each output Hadamard block; else
// launch_rht_out follows.  z ([batch][m] fp32) and tickets ([m / B_m] int)
// must be all-zero on entry and are all-zero again when the forward is done.
cudaError_t launch_gemv(const Layer& L, const GemvPlan& pl, const void* x, const void* xstep, int batch, float* z,
                        int* tickets, void* y, int y_dtype, cudaStream_t st);
cudaError_t launch_decode(const Layer& L, const Part& part, void* w_hat, cudaStream_t st);
// W_hat x' for all parts, x' in tensor-core tiles with npad (multiple of 16,
// <= 256) rows, b < batch; the (128-row tile, 256-column block) units are
// split evenly over one CTA per SM (stream-K), and each CTA's segment (its
// units within one tile) is stored to workspace slot L.tc_seg[cta] + k:
// ws[slot][b][r] for the tile's row r < 128 (L.tc_slots slots of npad * 128
// floats).
cudaError_t launch_gemm_tc(const Layer& L, const void* xt, int batch, int npad, float* ws, cudaStream_t st);
// The GEMM's (128-row tile, 256-column block) units, its grid, and its
// segment table (slot of each CTA's first segment, grid + 1 entries; slot of
// each tile's first segment, tiles + 1 entries).
int tc_units(const Layer& L);
int tc_grid(const Layer& L);
// Whether the GEMM takes split A words at this padded batch (computed codes,
// V = 1, npad <= 128): x' tiles then hold every value twice along K
// (launch_rht_in_umma with dup), and the 1MAD sums come out in units of its
// scale (gemv_z_scale).
bool tc_split(const Layer& L, int npad);
void tc_segments(const Layer& L, std::vector<int>& cta_seg, std::vector<int>& tile_seg);
// Preload (preload_kernel) every kernel a handle can launch: decode-GEMV
// (both input-transform variants) and qlinear_decode (gemv.cu), the transform
// kernels (rht.cu), the tensor-core GEMM (gemm_tc.cu).
cudaError_t prepare_gemv_kernels(const Layer& L);
cudaError_t prepare_rht_kernels(const Layer& L);
cudaError_t prepare_gemm_kernels(const Layer& L);
cudaError_t launch_eval_code(int code, int L, int V, int Q, const uint32_t* lut_words,
                             const uint32_t* states, int count, void* out, cudaStream_t st);

}  // namespace qlk
