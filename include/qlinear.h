/*
 * qlinear.h -- C ABI of the trellis-coded quantized linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer computes
 *
 *     y = alpha * diag(s_out) * H_m^T * W_hat * H_n * diag(s_in) * x
 *
 * where H_d = I_{d/B} (x) H_B is the normalised Walsh-Hadamard transform on
 * consecutive blocks of B entries (B = the largest power of two dividing d),
 * s_in / s_out are random +-1 sign vectors and alpha is a per-layer scale.
 * This is incoherence processing with a randomized Hadamard transform as on
 * the QuIP# page (Fig. 2) and in the QTIP OpenReview discussion ("Incoherence
 * Processing (W2)").  W_hat (m x n) is never stored: it is decoded on the fly
 * from a bitshift-trellis bit stream (QTIP discussion, "Figure 2 (Q4)" and
 * "Ablations and fast inference (W1 and W2)") through one of four codes
 * (QTIP discussion, "Inference speed analysis (W2)" and the comment on HYB
 * cost, "Bit Accounting (Q2)"; the table code is the palette reading of the
 * Q-Palette page):
 *
 *   QL_CODE_1MAD   x = A*s + B mod 2^32; value = fp16(C1 * (sum of the 4 bytes of x - 510))
 *   QL_CODE_3INST  x = A*s + B mod 2^32; m = (x & MASK) ^ XOR;
 *                  value = fp16(float16(m & 0xffff) + float16(m >> 16))
 *   QL_CODE_HYB    x = A*s + B mod 2^32; entry = lut[x >> (32 - Q)] (V fp16 values);
 *                  bit 15 of x negates the entry's first value
 *   QL_CODE_TABLE  entry = lut[s] (V fp16 values of an explicit codebook of 2^L
 *                  entries).  With L = kV each step's own kV bits index the
 *                  codebook: vector quantization (V = 2) or a non-uniform
 *                  scalar quantizer (V = 1), the VQ / NUQ members of the
 *                  Q-Palette page's palette (a trellis with L = kV is plain
 *                  k-bit, V-dimensional VQ, as the QTIP discussion's ablation
 *                  reply notes); with L > kV, a trellis over the codebook.
 *   QL_CODE_E8P    the E8-lattice vector quantizer the QTIP discussion compares
 *                  the trellis codes with (QuIP# page: abstract, Fig. 3
 *                  caption; QTIP discussion, "Inference speed analysis
 *                  (W2)": 2^16 E8-based entries of dimension 8, stored as 256
 *                  table words): V = 8, L = kV = 16 (each step's own 16 bits
 *                  index the codebook), k = 2.  State s: shape a = s >> 8,
 *                  signs of coordinates 0..6 in bits 1..7 (set = negative),
 *                  shift bit 0; codeword = sigma * T[a] + (bit 0 ? 1/4 : -1/4)
 *                  in every coordinate, where T[a] is the a-th of the 256
 *                  vectors of nonnegative half-odd-integer coordinates of
 *                  smallest norm (ties: 2T in lexicographic order) and the
 *                  sign of coordinate 7 makes sum(sigma * T[a]) even, i.e.
 *                  sigma * T[a] lies in the E8 lattice.  The library builds
 *                  the table; code.lut is not read.  One part only.
 *
 * with the constants (A, B per code; C1 = 443 * 2^-16; MASK = 0x9CFF8FFF,
 * XOR = 0x20003000) fixed by this library's format.  Values are rounded to
 * fp16 exactly once.
 *
 * Stream format (the pages print only the bit string of the Figure 2 example;
 * this is the library's reading):
 *   - packed_codes is a uint32 array read as one bit string, most significant
 *     bit of each word first.
 *   - Every row is cut into blocks of T = 256 columns; block j of row r is an
 *     independent trellis of S = 256*k bits starting at bit r*n*k + j*S.
 *     k is kV / V bits per weight: a whole number, or with V = 2 and an odd
 *     kV a half number (the Q-Palette page's fractional bitwidths, e.g. 2.5
 *     bits = 5 bits per 2-value step); S and r*n*k stay whole numbers.
 *   - Step t of a block carries bits [t*kV, (t+1)*kV); its L-bit state is the
 *     window of the block's bits ending at bit (t+1)*kV, read cyclically
 *     (tail-biting), and yields the V values of columns 256*j + t*V + e.
 *   - A half-TCQ layer (Q-Palette's mixed-bitwidth layer) stores rows
 *     [0, m_top) at k_top bits per weight first, then rows [m_top, m) at
 *     k_bot bits per weight.
 *
 * Conventions for every entry point:
 *   - Return value: QL_OK (0) or a negative QL_E_* code; qlinear_strerror()
 *     names it.  Argument errors are detected on the host before any work.
 *   - Device pointers are CUDA global-memory pointers of the device that was
 *     current when the handle was created; "stream" is a cudaStream_t (NULL =
 *     the legacy default stream).  forward/decode/eval_code are asynchronous
 *     with respect to the host and ordered on that stream.
 *   - A handle may be used from one host thread at a time; calls on one
 *     handle must be ordered (one stream, or streams ordered by events),
 *     because they share the handle's scratch buffers.
 */
#ifndef QLINEAR_H
#define QLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QL_OK 0
#define QL_E_ARG (-1)          /* invalid argument (null pointer, bad size, bad value)   */
#define QL_E_UNSUPPORTED (-2)  /* valid for the format but not implemented by this library */
#define QL_E_CUDA (-3)         /* a CUDA runtime call failed                              */
#define QL_E_OOM (-4)          /* device allocation failed                                */
#define QL_E_TIMEOUT (-5)      /* a bounded device-side wait gave up                      */
#define QL_E_DEVICE (-6)       /* a device-side check failed (see qlinear_get_status)     */
#define QL_E_SCRATCH (-7)      /* sizes exceed the fixed scratch of qlinear_forward_noalloc */

#define QL_CODE_1MAD 0
#define QL_CODE_3INST 1
#define QL_CODE_HYB 2
#define QL_CODE_TABLE 3
#define QL_CODE_E8P 4

#define QL_F32 0
#define QL_F16 1

typedef struct qlinear_s* qlinear_t;

/* The code that maps a trellis state to V values.
 *   kind: QL_CODE_1MAD or QL_CODE_3INST (V must be 1), QL_CODE_HYB or
 *         QL_CODE_TABLE (V = 1 or 2), or QL_CODE_E8P (V = 8, L = 16, k = 2).
 *   Q:    HYB only, table index bits, 1..9 (the discussion uses Q = 9; "you can
 *         go down to Q~6").  Ignored by the table code, whose codebook has
 *         2^L entries (L = 1..9).
 *   lut:  HYB and table code, device pointer to 2^Q (table code: 2^L) x V fp16
 *         values, row-major (entry i = lut[i*V .. i*V+V-1]).  Copied by create. */
typedef struct {
    int kind;
    int Q;
    const void* lut;
} ql_code_t;

/* Facts about a handle (qlinear_info). */
typedef struct {
    int m, n, L, V, code, Q;
    int k_top, k_bot, m_top;   /* bits per weight of the first / last part (rounded
                                  down: see part_kv), rows of the first part   */
    int B_n, B_m;              /* Hadamard block sizes                           */
    size_t stream_bytes;       /* packed code words: m*n*k/8 (summed over parts) */
    size_t sign_bytes;         /* bit-packed signs: (n + m) bits, word-padded    */
    size_t lut_bytes;          /* HYB table / codebook: 2^Q (2^L) * V * 2 bytes  */
    size_t scratch_bytes;      /* device scratch currently held by the handle    */
    int last_launches;         /* kernels launched by the most recent forward    */
    int nparts;                /* row parts (1 uniform, 2 half-TCQ, up to 8)     */
    int part_rows[8];          /* rows of each part (entries >= nparts are 0)    */
    int part_kv[8];            /* bits per trellis step of each part (k = kv/V)  */
} ql_info_t;

/* Create a uniform-bitrate layer.
 *   m, n:         output and input sizes; n % 256 == 0, m % 16 == 0, and the
 *                 Hadamard block sizes B(n), B(m) must not exceed 32768.
 *   k:            bits per weight, 1..4.   L: state bits, k*V <= L <= 16.
 *   V:            values per trellis step (1 or 2, see ql_code_t).
 *   packed_codes: device pointer, n_words = m*n*k/32 uint32 in the stream format above.
 *   s_in, s_out:  device pointers, int8 +-1, n and m entries (any other value -> QL_E_ARG).
 *   alpha:        finite scale.
 * The handle copies codes (re-laid out for the kernels), signs (bit-packed)
 * and the HYB table into library-owned device memory; the caller may free its
 * buffers when create returns.  Synchronises the device before returning.
 * Errors: QL_E_ARG, QL_E_UNSUPPORTED, QL_E_OOM, QL_E_CUDA. */
int qlinear_create(qlinear_t* out, int m, int n, int k, int L, int V, ql_code_t code,
                   const uint32_t* packed_codes, size_t n_words,
                   const int8_t* s_in, const int8_t* s_out, float alpha);

/* Create a half-TCQ layer (Q-Palette page: two TCQ quantizers of different
 * bitwidth in one layer): rows [0, m_top) at k_top bits, rows [m_top, m) at
 * k_bot bits.  m_top % 16 == 0, 0 < m_top < m.  n_words = (m_top*k_top +
 * (m - m_top)*k_bot) * n / 32.  Otherwise as qlinear_create. */
int qlinear_create_mixed(qlinear_t* out, int m, int n, int m_top, int k_top, int k_bot,
                         int L, int V, ql_code_t code,
                         const uint32_t* packed_codes, size_t n_words,
                         const int8_t* s_in, const int8_t* s_out, float alpha);

/* Create a layer of several row parts, each with its own bitwidth: layers
 * that share their input fused along m (Q-Palette page: layer fusion of
 * layers that read the same input, and a palette of TCQ quantizers of
 * different bitwidths).  Part i covers rows [sum of part_rows[0..i), +
 * part_rows[i]) at part_k[i] bits; the parts' streams follow one another in
 * packed_codes, each in the stream format above.  One sign vector each for
 * the input and the (fused) output, one Hadamard transform of the fused m.
 *   nparts:     1..8;  part_rows, part_k: host arrays of nparts entries,
 *               part_rows[i] % 16 == 0, sum(part_rows) == m, part_k[i] in 1..4.
 *   n_words:    sum over parts of part_rows[i] * n * part_k[i] / 32.
 * Otherwise as qlinear_create (qlinear_create_mixed is the two-part case).
 * Errors: QL_E_ARG, QL_E_UNSUPPORTED, QL_E_OOM, QL_E_CUDA. */
int qlinear_create_parts(qlinear_t* out, int m, int n, int nparts, const int* part_rows, const int* part_k,
                         int L, int V, ql_code_t code,
                         const uint32_t* packed_codes, size_t n_words,
                         const int8_t* s_in, const int8_t* s_out, float alpha);

/* As qlinear_create_parts with each part's bitrate given as bits per trellis
 * step: part i stores part_kv[i] bits per step of V values, so k = kv / V
 * bits per weight, in [1, 4]; with V = 2 an odd kv gives a half-integer
 * bitwidth (Q-Palette page: fractional bitwidths such as 2.5 bits, and
 * half-TCQ's 2.75 bits from a 2.5-bit and a 3-bit quantizer).
 *   part_kv:  host array of nparts entries, V <= part_kv[i] <= 4V, L >= part_kv[i].
 *   n_words:  sum over parts of part_rows[i] * (n / V) * part_kv[i] / 32.
 * Errors: QL_E_ARG, QL_E_UNSUPPORTED, QL_E_OOM, QL_E_CUDA. */
int qlinear_create_kv(qlinear_t* out, int m, int n, int nparts, const int* part_rows, const int* part_kv,
                      int L, int V, ql_code_t code,
                      const uint32_t* packed_codes, size_t n_words,
                      const int8_t* s_in, const int8_t* s_out, float alpha);

/* y = W x for a batch of inputs.
 *   x: device pointer, fp16 [batch][n] row-major.
 *   y: device pointer, [batch][m] row-major, fp32 (y_dtype = QL_F32) or fp16 (QL_F16).
 *   batch >= 0 (0 is a no-op).  batch <= 8 runs the fused decode-GEMV kernel
 *   after an input-transform kernel, with the output transform inside it
 *   when batch * B(m) <= 256, else before an output-transform kernel; larger
 *   batches run the decode-to-tensor-memory tcgen05 GEMM between the two
 *   transform kernels.  x and y must be 16-byte aligned.
 * The first call with a batch larger than any before it allocates scratch;
 * make such a call before capturing forward into a CUDA graph.
 * Errors: QL_E_ARG, QL_E_OOM, QL_E_CUDA (launch failure). */
int qlinear_forward(qlinear_t h, const void* x, int batch, void* y, int y_dtype, void* stream);

/* As qlinear_forward, with x and y in host memory: copies x to the device,
 * runs forward and copies y back, all on `stream`, and waits for the stream
 * before returning (y is ready on return).  Pinned host memory makes the
 * copies asynchronous DMA transfers; pageable memory also works.  A y of at
 * most 64 KB in pinned host memory that the device can address (16-byte
 * aligned) is written there by the forward's last kernel instead of copied. */
int qlinear_forward_host(qlinear_t h, const void* x_host, int batch, void* y_host, int y_dtype,
                         void* stream);

/* As qlinear_forward for batch <= 8, without allocating or freeing any
 * memory.  None of the pages has a counterpart: this serves callers that
 * cannot let a library allocate while they run (cudaMalloc/cudaFree may
 * synchronise the whole device and stall a serving process's other streams;
 * runtimes that pre-carve all free HBM into their own pools leave no room).
 *   Scratch: the output-block tickets, the fp32 accumulator z and (when the
 *   input transform runs as its own kernel) x' live in one fixed array of
 *   QL_NOALLOC_SCRATCH_BYTES in the library's static device memory, per
 *   device: round_up(4*m/B(m), 256) + round_up(4*batch*m, 256) bytes from its
 *   start, plus x' (4*batch*n bytes at V = 1, 2*batch*n at V = 2 or 8) at its
 *   end, must fit, else QL_E_SCRATCH (before any device work).  Tickets and z
 *   are all-zero again after every successful call; a call clears them on
 *   `stream` first only when an earlier call failed or wrote x' where they
 *   now lie.
 *   Sharing: all handles on a device share the array, so calls that overlap
 *   in time (different streams or host threads) race and give wrong y; calls
 *   in order on one stream are safe.
 *   Set-up: a device's first call looks up the array's address
 *   (cudaGetSymbolAddress), which may load the library's device code; make
 *   that first call before any stream capture.
 *   Profiling slots (qlinear_profile_enable) are not recorded by this call.
 * Errors: QL_E_ARG, QL_E_UNSUPPORTED (batch > 8), QL_E_SCRATCH, QL_E_CUDA. */
#define QL_NOALLOC_SCRATCH_BYTES (2 * 1024 * 1024)
int qlinear_forward_noalloc(qlinear_t h, const void* x, int batch, void* y, int y_dtype, void* stream);

/* Write W_hat as fp16 [m][n] row-major to the device pointer w_hat (the code
 * values before alpha, signs and Hadamard transforms).  For testing. */
int qlinear_decode(qlinear_t h, void* w_hat, void* stream);

/* Evaluate a code on `count` states (device pointer, uint32, each < 2^L) and
 * write fp16 [count][V] to the device pointer out.  For testing the codes
 * exhaustively. */
int qlinear_eval_code(ql_code_t code, int L, int V, const uint32_t* states, int count, void* out,
                      void* stream);

/* Test hook for the tensor-core GEMM's bounded waits (no counterpart on the
 * pages; the waits themselves are the failure detection of the GEMM's
 * producer/consumer pipeline).  With enable != 0, every later forward with
 * batch > 8 on this handle runs the GEMM with each mbarrier wait limited to
 * wait_tries suspending tries (1..4096; each try suspends for at most about a
 * millisecond) and with the x' producer withholding the first stage of every
 * CTA, so the MMA issuer's wait on it runs out.  The CTAs then set
 * QL_E_TIMEOUT in the handle's status word (read by qlinear_get_status), drop
 * their work, free their tensor memory and exit: y of that forward is
 * undefined, and the next forward after qlinear_get_status reported the
 * timeout is correct again.  No fault and no unbounded wait is involved.
 * enable = 0 restores the normal limit (a few seconds) and stops withholding.
 * Errors: QL_E_ARG (null handle, wait_tries out of range when enabling). */
int qlinear_test_stall(qlinear_t h, int enable, int wait_tries);

/* Trellis-coded quantization: for each block of 256 source values, the bits
 * whose tail-biting walk on the bitshift trellis reproduces the block with the
 * least squared error (QTIP discussion: encoding searches the fixed-length
 * walks of the trellis for the least distortion; the discussion's "Table 1"
 * replies on i.i.d. Gaussian sources).  The search is a two-pass tail-biting
 * Viterbi: a free-start pass fixes the block's wrap-around L-kV bits from its
 * best final state, a second pass with both ends tied to them gives the bits;
 * float32 costs, every operation rounded to nearest, ties to the smallest
 * predecessor and final state.
 *   x:      device pointer, float32 [blocks][256] source values (e.g. a row-major
 *           m x n weight after incoherence processing and scaling, n % 256 == 0:
 *           its blocks in stream order).
 *   words:  device pointer, out, uint32 [blocks][256 k / 32] in the stream format
 *           (for a row-major m x n source, exactly qlinear_create's packed_codes).
 *   err:    device pointer or null, out, float32 [blocks]: squared error of each
 *           block's reconstruction.
 *   L <= 16, k*V <= 8; code as in qlinear_create (HYB and the table code: the
 *   fp16 table is read; the table code with L = kV is nearest-codeword VQ / NUQ).
 *   One CTA holds a block's whole dynamic programme (the group minima of its
 *   2^L states) in its shared memory whenever they fit, i.e. everything but
 *   L = 16 at one bit per step, where a thread-block cluster of 4 CTAs shares it
 *   (16384 states per CTA, predecessors' costs read from the other CTAs'
 *   shared memory).
 * Scratch (256/V * 2^(L-kV) bytes per CTA or cluster that runs at once, at
 * most about 620 MB) comes from a memory pool of the library on the current
 * device, which keeps it mapped for later calls until the process exits.
 * Returns when the result is ready (synchronises the stream).
 * Errors: QL_E_ARG, QL_E_UNSUPPORTED (L > 16, or too large for shared memory),
 * QL_E_OOM, QL_E_CUDA, QL_E_DEVICE (non-finite source values). */
int qlinear_encode(ql_code_t code, int L, int k, int V, const float* x, int blocks, uint32_t* words, float* err,
                   void* stream);

/* As qlinear_encode with the bitrate given as kv bits per trellis step
 * (V <= kv <= min(4V, 8), L >= kv): with V = 2 an odd kv is a half-integer
 * bitwidth (kv = 5: 2.5 bits per weight), the layout qlinear_create_kv reads.
 *   words: device pointer, out, uint32 [blocks][(256 / V) * kv / 32].
 * With the table code and L = kv this is nearest-codeword vector (V = 2) or
 * non-uniform scalar (V = 1) quantization.  Errors as qlinear_encode. */
int qlinear_encode_kv(ql_code_t code, int L, int kv, int V, const float* x, int blocks, uint32_t* words, float* err,
                      void* stream);

/* Read the handle's device status word (synchronises the device).  Returns
 * QL_OK, or QL_E_DEVICE / QL_E_TIMEOUT if a kernel recorded a failed check or
 * an expired bounded wait since the last call; reading clears the word. */
int qlinear_get_status(qlinear_t h);

/* Fill *info. */
int qlinear_info(qlinear_t h, ql_info_t* info);

/* Profiling: record a pair of CUDA events around the dominant kernel launch(es)
 * of every forward (the decode-GEMV, or the tensor-core GEMM) on the
 * forward's own stream.  Pairs go to a ring of `capacity` slots owned by the
 * handle (pair i of the ring is reused by launch i + capacity); capacity 0
 * stops recording and frees the events.  Recording works inside CUDA graph
 * capture: the captured graph re-records the same slots on every replay.
 * Errors: QL_E_ARG (capacity < 0 or > 65536), QL_E_CUDA. */
int qlinear_profile_enable(qlinear_t h, int capacity);

/* Timing: launch the forward's dominant kernel alone (the decode-GEMV for
 * batch <= 8, the tensor-core GEMM for the first 256 rows of a larger batch)
 * on `stream`, on the operands the handle's most recent forward left in its
 * scratch: that forward must have had this batch.  x (device, fp16
 * [batch][n], as in qlinear_forward) is read where the decode-GEMV computes
 * x' itself (batch <= 2 with x' of at most 48 KB); it may be null otherwise.  The kernel does exactly
 * the work it does inside a forward (same launch configuration, same code
 * words and x'), so back-to-back launches time it apart from the transforms
 * around it.  Its output is not a result: the decode-GEMV's fp32 sums stay in
 * the handle's accumulator (the next forward re-zeroes it first), and where
 * the decode-GEMV transforms its own output (batch * m <= 256) it writes y
 * (fp32 or fp16 [batch][m], y_dtype as in qlinear_forward); y is not used
 * otherwise and may then be null.  Works inside CUDA graph capture.
 * Errors: QL_E_ARG (batch < 1, a different batch than the last forward, no
 * forward yet, bad y_dtype, y null when written), QL_E_CUDA. */
int qlinear_launch_main_kernel(qlinear_t h, const void* x, int batch, void* y, int y_dtype, void* stream);

/* Synchronise the device and report the summed elapsed time of the recorded
 * slots (each slot counted once, with its most recent record) and how many
 * slots hold a record.  Slots keep their records; graph replays overwrite
 * them in place. */
int qlinear_profile_read(qlinear_t h, double* total_ms, int* slots);

/* Free the handle and its device memory (synchronises the device). */
int qlinear_destroy(qlinear_t h);

/* Name of a status code (static string). */
const char* qlinear_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* QLINEAR_H */
