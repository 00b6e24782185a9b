// qlinear_abi.cu -- the C ABI declared in include/qlinear.h (host side).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "codes.cuh"
#include "encode.h"
#include "internal.h"

using namespace qlk;

struct qlinear_s {
    Layer L;
};

namespace {

struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) {
            ok = false;
            return;
        }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
    }
    ~DeviceGuard() {
        int cur;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

int is_device_pointer(const void* p) {
    if (!p) return 0;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged;
}

int pow2_block(int d) { return d & -d; }

template <typename T>
int dev_alloc(T** p, size_t bytes) {
    *p = nullptr;
    if (bytes == 0) return QL_OK;
    if (cudaMalloc((void**)p, bytes) != cudaSuccess) {
        cudaGetLastError();
        *p = nullptr;
        return QL_E_OOM;
    }
    return QL_OK;
}

void free_profiling(Layer& L) {
    for (int i = 0; i < 2 * L.prof_cap; ++i) cudaEventDestroy(L.prof_ev[i]);
    delete[] L.prof_ev;
    L.prof_ev = nullptr;
    L.prof_cap = L.prof_next = L.prof_count = 0;
}

void free_layer(Layer& L) {
    free_profiling(L);
    cudaFree(L.words);
    cudaFree(L.sin_bits);
    cudaFree(L.sout_bits);
    cudaFree(L.lut);
    cudaFree(L.status);
    cudaFree(L.xp);
    cudaFree(L.acc);
    cudaFree(L.host_stage);
    cudaFree(L.tc_seg);
    cudaFree(L.tcws);
    std::memset(&L, 0, sizeof(L));
}

int check_code(const ql_code_t& code, int V, int L) {
    if (code.kind == QL_CODE_1MAD || code.kind == QL_CODE_3INST) return V == 1 ? QL_OK : QL_E_UNSUPPORTED;
    if (code.kind == QL_CODE_E8P) return V == 8 && L == 16 ? QL_OK : QL_E_UNSUPPORTED;
    if (code.kind != QL_CODE_HYB && code.kind != QL_CODE_TABLE) return QL_E_ARG;
    if (V != 1 && V != 2) return QL_E_ARG;
    if (code.kind == QL_CODE_HYB && (code.Q < 1 || code.Q > kMaxTableBits)) return QL_E_UNSUPPORTED;
    if (code.kind == QL_CODE_TABLE && (L < 1 || L > kMaxTableBits)) return QL_E_UNSUPPORTED;
    if (!is_device_pointer(code.lut)) return QL_E_ARG;
    return QL_OK;
}

// Index bits of the code's table in words (the table code's codebook has 2^L
// entries; the E8 code's 256 shapes take 2 words each).
int table_bits(const ql_code_t& code, int L) {
    return code.kind == QL_CODE_HYB ? code.Q : code.kind == QL_CODE_TABLE ? L : code.kind == QL_CODE_E8P ? 9 : 0;
}

// The E8 code's shape table (include/qlinear.h): the 256 vectors of
// nonnegative half-odd coordinates T = n/2 (n odd) with the smallest norm,
// ties broken by n in lexicographic order.  Shape a takes words 2a and 2a+1:
// byte i of the pair is the high byte of fp16(n_i / 2) (its low byte is
// zero), and bit 31 of word 2a+1 holds (sum of n_i) / 2 mod 2.
const std::array<uint32_t, 512>& e8p_shape_words() {
    static const std::array<uint32_t, 512> words = [] {
        std::vector<std::array<int, 9>> all;  // [sum of n_i^2, n_0 .. n_7]
        all.reserve(1 << 16);
        for (int code = 0; code < (1 << 16); ++code) {
            std::array<int, 9> v{};
            for (int i = 0; i < 8; ++i) {
                v[1 + i] = 2 * ((code >> (2 * (7 - i))) & 3) + 1;  // 1, 3, 5, 7
                v[0] += v[1 + i] * v[1 + i];
            }
            all.push_back(v);
        }
        std::sort(all.begin(), all.end());
        std::array<uint32_t, 512> w{};
        for (int a = 0; a < 256; ++a) {
            int sum = 0;
            for (int i = 0; i < 8; ++i) {
                const int nv = all[a][1 + i];
                sum += nv;
                const uint32_t hi = __half_as_ushort(__float2half_rn(0.5f * (float)nv)) >> 8;
                w[2 * a + i / 4] |= hi << (8 * (i % 4));
            }
            w[2 * a + 1] |= (uint32_t)((sum % 4) / 2) << 31;
        }
        return w;
    }();
    return words;
}

// Copies the code's table into `dst` (2^Q words) on stream st.
cudaError_t copy_code_table(const ql_code_t& code, int Q, int V, uint32_t* dst, cudaStream_t st) {
    if (code.kind == QL_CODE_E8P)
        return cudaMemcpyAsync(dst, e8p_shape_words().data(), 512 * 4, cudaMemcpyHostToDevice, st);
    return launch_copy_lut(code.lut, Q, V, dst, st);
}

// Shared by the create calls. parts: [(rows, kv)], host arrays; kv = bits per
// trellis step, k = kv / V bits per weight in [1, 4] (a half number when
// V = 2 and kv is odd).
int create_common(qlinear_t* out, int m, int n, int nparts, const int* part_rows, const int* part_kv, int L,
                  int V, ql_code_t code, const uint32_t* packed_codes, size_t n_words, const int8_t* s_in,
                  const int8_t* s_out, float alpha) {
    if (!out) return QL_E_ARG;
    *out = nullptr;
    if (m <= 0 || n <= 0 || !std::isfinite(alpha)) return QL_E_ARG;
    if (V != 1 && V != 2 && !(V == 8 && code.kind == QL_CODE_E8P)) return QL_E_ARG;
    if (code.kind == QL_CODE_E8P && (nparts != 1 || !part_kv || part_kv[0] != 16)) return QL_E_UNSUPPORTED;
    if (n % kT != 0 || m % kRowTile != 0) return QL_E_UNSUPPORTED;
    if (pow2_block(n) > kMaxHadamard || pow2_block(m) > kMaxHadamard) return QL_E_UNSUPPORTED;
    if (nparts < 1 || nparts > kMaxParts || !part_rows || !part_kv) return QL_E_ARG;
    size_t expect_words = 0;
    long long rows_sum = 0;
    for (int i = 0; i < nparts; ++i) {
        const int kv = part_kv[i];
        if (kv < V || kv > 4 * V) return QL_E_UNSUPPORTED;
        if (L < kv || L > 16) return QL_E_UNSUPPORTED;
        if (part_rows[i] <= 0 || part_rows[i] % kRowTile != 0) return QL_E_ARG;
        expect_words += (size_t)part_rows[i] * n / V * kv / 32;  // n / V: whole steps per row
        rows_sum += part_rows[i];
    }
    if (rows_sum != m || n_words != expect_words) return QL_E_ARG;
    int rc = check_code(code, V, L);
    if (rc != QL_OK) return rc;
    if (!is_device_pointer(packed_codes) || !is_device_pointer(s_in) || !is_device_pointer(s_out))
        return QL_E_ARG;

    qlinear_s* h = new (std::nothrow) qlinear_s;
    if (!h) return QL_E_OOM;
    std::memset(&h->L, 0, sizeof(Layer));
    Layer& Ly = h->L;
    cudaGetDevice(&Ly.device);
    cudaDeviceGetAttribute(&Ly.num_sms, cudaDevAttrMultiProcessorCount, Ly.device);
    Ly.m = m;
    Ly.n = n;
    Ly.L = L;
    Ly.V = V;
    Ly.code = code.kind;
    Ly.Q = table_bits(code, L);
    Ly.alpha = alpha;
    Ly.B_n = pow2_block(n);
    Ly.B_m = pow2_block(m);
    Ly.nparts = nparts;
    size_t off = 0;
    int row0 = 0;
    for (int i = 0; i < nparts; ++i) {
        Ly.parts[i].row0 = row0;
        Ly.parts[i].rows = part_rows[i];
        Ly.parts[i].kv = part_kv[i];
        Ly.parts[i].k2 = 2 * part_kv[i] / V;
        Ly.parts[i].word_off = off;
        Ly.parts[i].n_words = (size_t)part_rows[i] * n / V * part_kv[i] / 32;
        off += Ly.parts[i].n_words;
        row0 += part_rows[i];
    }

    rc = dev_alloc(&Ly.words, n_words * 4);
    if (rc == QL_OK) rc = dev_alloc(&Ly.sin_bits, (size_t)((n + 31) / 32) * 4);
    if (rc == QL_OK) rc = dev_alloc(&Ly.sout_bits, (size_t)((m + 31) / 32) * 4);
    if (rc == QL_OK) rc = dev_alloc(&Ly.status, sizeof(int));
    if (rc == QL_OK && uses_table(Ly.code)) rc = dev_alloc(&Ly.lut, ((size_t)1 << Ly.Q) * 4);
    std::vector<int> cta_seg, tile_seg;
    tc_segments(Ly, cta_seg, tile_seg);
    if (rc == QL_OK) rc = dev_alloc(&Ly.tc_seg, (cta_seg.size() + tile_seg.size()) * sizeof(int));
    if (rc != QL_OK) {
        free_layer(Ly);
        delete h;
        return rc;
    }
    cudaStream_t st = 0;
    cudaError_t e = cudaMemsetAsync(Ly.status, 0, sizeof(int), st);
    for (int i = 0; i < nparts && e == cudaSuccess; ++i)
        e = launch_relayout(packed_codes + Ly.parts[i].word_off, Ly.words, Ly.parts[i], n, st);
    if (e == cudaSuccess) e = launch_pack_signs(s_in, n, Ly.sin_bits, Ly.status, st);
    if (e == cudaSuccess) e = launch_pack_signs(s_out, m, Ly.sout_bits, Ly.status, st);
    if (e == cudaSuccess && uses_table(Ly.code)) e = copy_code_table(code, Ly.Q, V, Ly.lut, st);
    Ly.tc_tile_seg = Ly.tc_seg + cta_seg.size();
    Ly.tc_slots = cta_seg.back();
    if (e == cudaSuccess)
        e = cudaMemcpy(Ly.tc_seg, cta_seg.data(), cta_seg.size() * sizeof(int), cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
        e = cudaMemcpy(Ly.tc_seg + cta_seg.size(), tile_seg.data(), tile_seg.size() * sizeof(int),
                       cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    int status = 0;
    if (e == cudaSuccess) e = cudaMemcpy(&status, Ly.status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
        cudaGetLastError();
        free_layer(Ly);
        delete h;
        return QL_E_CUDA;
    }
    if (status & kStatusBadSign) {
        free_layer(Ly);
        delete h;
        return QL_E_ARG;
    }
    // load every kernel this layer can launch now, not at its first launch
    e = prepare_gemv_kernels(Ly);
    if (e == cudaSuccess) e = prepare_rht_kernels(Ly);
    if (e == cudaSuccess) e = prepare_gemm_kernels(Ly);
    if (e != cudaSuccess) {
        cudaGetLastError();
        free_layer(Ly);
        delete h;
        return QL_E_CUDA;
    }
    *out = h;
    return QL_OK;
}

// Record an event on st; inside stream capture it becomes an event-record
// node of the graph (so every replay re-records it) instead of a capture-
// internal dependency marker.
cudaError_t record_event(cudaEvent_t ev, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(st, &cs);
    if (e != cudaSuccess) return e;
    return cudaEventRecordWithFlags(ev, st, cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : 0);
}

// Grow a scratch buffer to at least `bytes`.
int ensure(void** buf, size_t* have, size_t bytes) {
    if (*have >= bytes) return QL_OK;
    if (*buf) cudaFree(*buf);
    *buf = nullptr;
    *have = 0;
    if (cudaMalloc(buf, bytes) != cudaSuccess) {
        cudaGetLastError();
        *buf = nullptr;
        return QL_E_OOM;
    }
    *have = bytes;
    return QL_OK;
}

// Bytes of the ticket array at the start of the accumulator buffer.
size_t ticket_bytes(const Layer& L) { return ((size_t)(L.m / L.B_m) * 4 + 255) / 256 * 256; }
int* tickets_of(void* acc) { return (int*)acc; }
float* z_of(const Layer& L, void* acc) { return (float*)((char*)acc + ticket_bytes(L)); }

// The decode-GEMV's accumulator (tickets and z) is all-zero between forwards:
// it is zeroed when allocated, and the kernel that consumes z re-zeroes it
// (the decode-GEMV's output-transform epilogue or the output-transform
// kernel after it).
int prepare_acc(Layer& L, size_t z_bytes, cudaStream_t st) {
    const size_t bytes = ticket_bytes(L) + z_bytes;
    if (L.acc_bytes >= bytes && !L.acc_dirty) return QL_OK;
    int rc = ensure(&L.acc, &L.acc_bytes, bytes);
    if (rc != QL_OK) return rc;
    if (cudaMemsetAsync(L.acc, 0, L.acc_bytes, st) != cudaSuccess) {
        cudaGetLastError();
        return QL_E_CUDA;
    }
    L.acc_dirty = 0;
    return QL_OK;
}

// batch <= 8: the decode-GEMV kernel does the whole forward (its input
// transform in-kernel for small x, else after a separate input-transform
// kernel; the output transform in its epilogue).
int forward_gemv(Layer& L, const void* x, int batch, void* y, int y_dtype, cudaStream_t st) {
    const GemvPlan pl = plan_gemv(L, batch);
    int rc = ensure(&L.xp, &L.xp_bytes, gemv_xstep_bytes(L, batch));
    if (rc == QL_OK) rc = prepare_acc(L, (size_t)batch * L.m * 4, st);
    if (rc != QL_OK) return rc;
    L.last_launches = (pl.x_e ? 1 : 2) + (pl.fuse_out ? 0 : 1);
    cudaError_t e = pl.x_e ? cudaSuccess : launch_rht_in_xstep(L, x, batch, L.xp, st);
    const int slot = L.prof_cap ? L.prof_next : -1;
    if (e == cudaSuccess && slot >= 0) e = record_event(L.prof_ev[2 * slot], st);
    if (e == cudaSuccess) e = launch_gemv(L, pl, x, L.xp, batch, z_of(L, L.acc), tickets_of(L.acc), y, y_dtype, st);
    if (e == cudaSuccess && slot >= 0) {
        e = record_event(L.prof_ev[2 * slot + 1], st);
        L.prof_next = (L.prof_next + 1) % L.prof_cap;
        if (L.prof_count < L.prof_cap) ++L.prof_count;
    }
    if (e == cudaSuccess && !pl.fuse_out) e = launch_rht_out(L, z_of(L, L.acc), batch, y, y_dtype, st, gemv_z_scale(L));
    if (e != cudaSuccess) {
        cudaGetLastError();
        L.acc_dirty = 1;  // a partial forward may have left sums in z or counts in the tickets
        return QL_E_CUDA;
    }
    return QL_OK;
}

// batch > 8: input transform into tensor-core operand tiles, tcgen05 GEMM
// into the partial-sum workspace, output transform summing a tile's partials;
// batches above 256 run in passes of 256.
int forward_tc(Layer& L, const void* x, int batch, void* y, int y_dtype, cudaStream_t st) {
    const int chunk = batch < kTcMaxN ? batch : kTcMaxN;
    const int npad_max = (chunk + 15) / 16 * 16;
    // x' tiles hold every value twice along K where the GEMM takes split A words
    const size_t xp_dup = tc_split(L, 16) ? 2 : 1;
    int rc = ensure(&L.xp, &L.xp_bytes, (size_t)npad_max * L.n * 2 * xp_dup);
    if (rc == QL_OK) rc = ensure(&L.tcws, &L.tcws_bytes, (size_t)L.tc_slots * npad_max * 128 * 4);
    if (rc != QL_OK) return rc;
    float* ws = (float*)L.tcws;
    const size_t ysz = y_dtype == QL_F16 ? 2 : 4;
    L.last_launches = 3 * ((batch + kTcMaxN - 1) / kTcMaxN);
    for (int b0 = 0; b0 < batch; b0 += kTcMaxN) {
        const int nb = batch - b0 < kTcMaxN ? batch - b0 : kTcMaxN;
        const int npad = (nb + 15) / 16 * 16;
        const void* xb = (const char*)x + (size_t)b0 * L.n * 2;
        void* yb = (char*)y + (size_t)b0 * L.m * ysz;
        const bool split = tc_split(L, npad);
        cudaError_t e = launch_rht_in_umma(L, xb, nb, npad, L.xp, st, split);
        const int slot = L.prof_cap ? L.prof_next : -1;
        if (e == cudaSuccess && slot >= 0) e = record_event(L.prof_ev[2 * slot], st);
        if (e == cudaSuccess) e = launch_gemm_tc(L, L.xp, nb, npad, ws, st);
        if (e == cudaSuccess && slot >= 0) {
            e = record_event(L.prof_ev[2 * slot + 1], st);
            L.prof_next = (L.prof_next + 1) % L.prof_cap;
            if (L.prof_count < L.prof_cap) ++L.prof_count;
        }
        if (e == cudaSuccess) e = launch_rht_out_tc(L, ws, nb, npad, yb, y_dtype, st, split ? gemv_z_scale(L) : 1.0f);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return QL_E_CUDA;
        }
    }
    return QL_OK;
}

int forward_device(Layer& L, const void* x, int batch, void* y, int y_dtype, cudaStream_t st) {
    const int rc = batch <= kGemvMaxBatch ? forward_gemv(L, x, batch, y, y_dtype, st)
                                          : forward_tc(L, x, batch, y, y_dtype, st);
    L.last_batch = rc == QL_OK ? batch : 0;
    return rc;
}

// The dominant kernel of a forward with this batch alone, on the scratch the
// last forward (same batch) left: qlinear_launch_main_kernel.
int launch_main(Layer& L, const void* x, int batch, void* y, int y_dtype, cudaStream_t st) {
    cudaError_t e;
    if (batch <= kGemvMaxBatch) {
        const GemvPlan pl = plan_gemv(L, batch);
        if ((pl.fuse_out && !y) || (pl.x_e && !x)) return QL_E_ARG;
        e = launch_gemv(L, pl, x, L.xp, batch, z_of(L, L.acc), tickets_of(L.acc), y, y_dtype, st);
        if (!pl.fuse_out) L.acc_dirty = 1;  // the sums stay in z
    } else {
        const int nb = batch < kTcMaxN ? batch : kTcMaxN;
        e = launch_gemm_tc(L, L.xp, nb, (nb + 15) / 16 * 16, (float*)L.tcws, st);
    }
    L.last_launches = 1;
    if (e != cudaSuccess) {
        cudaGetLastError();
        L.acc_dirty = 1;
        return QL_E_CUDA;
    }
    return QL_OK;
}

}  // namespace

extern "C" {

int qlinear_create(qlinear_t* out, int m, int n, int k, int L, int V, ql_code_t code, const uint32_t* packed_codes,
                   size_t n_words, const int8_t* s_in, const int8_t* s_out, float alpha) {
    if (!out) return QL_E_ARG;
    *out = nullptr;
    if (k < 1 || k > 4) return QL_E_UNSUPPORTED;
    if (V != 1 && V != 2 && !(V == 8 && code.kind == QL_CODE_E8P)) return QL_E_ARG;
    const int rows[1] = {m};
    const int kvs[1] = {k * V};
    return create_common(out, m, n, 1, rows, kvs, L, V, code, packed_codes, n_words, s_in, s_out, alpha);
}

int qlinear_create_mixed(qlinear_t* out, int m, int n, int m_top, int k_top, int k_bot, int L, int V,
                         ql_code_t code, const uint32_t* packed_codes, size_t n_words, const int8_t* s_in,
                         const int8_t* s_out, float alpha) {
    if (!out) return QL_E_ARG;
    *out = nullptr;
    if (m_top <= 0 || m_top >= m) return QL_E_ARG;
    if (k_top < 1 || k_top > 4 || k_bot < 1 || k_bot > 4) return QL_E_UNSUPPORTED;
    if (V != 1 && V != 2) return QL_E_ARG;
    const int rows[2] = {m_top, m - m_top};
    const int kvs[2] = {k_top * V, k_bot * V};
    return create_common(out, m, n, 2, rows, kvs, L, V, code, packed_codes, n_words, s_in, s_out, alpha);
}

int qlinear_create_parts(qlinear_t* out, int m, int n, int nparts, const int* part_rows, const int* part_k, int L,
                         int V, ql_code_t code, const uint32_t* packed_codes, size_t n_words, const int8_t* s_in,
                         const int8_t* s_out, float alpha) {
    if (!out) return QL_E_ARG;
    *out = nullptr;
    if (nparts < 1 || nparts > kMaxParts || !part_rows || !part_k) return QL_E_ARG;
    if (V != 1 && V != 2) return QL_E_ARG;
    int kvs[kMaxParts];
    for (int i = 0; i < nparts; ++i) {
        if (part_k[i] < 1 || part_k[i] > 4) return QL_E_UNSUPPORTED;
        kvs[i] = part_k[i] * V;
    }
    return create_common(out, m, n, nparts, part_rows, kvs, L, V, code, packed_codes, n_words, s_in, s_out, alpha);
}

int qlinear_create_kv(qlinear_t* out, int m, int n, int nparts, const int* part_rows, const int* part_kv, int L,
                      int V, ql_code_t code, const uint32_t* packed_codes, size_t n_words, const int8_t* s_in,
                      const int8_t* s_out, float alpha) {
    if (!out) return QL_E_ARG;
    *out = nullptr;
    return create_common(out, m, n, nparts, part_rows, part_kv, L, V, code, packed_codes, n_words, s_in, s_out, alpha);
}

int qlinear_forward(qlinear_t h, const void* x, int batch, void* y, int y_dtype, void* stream) {
    if (!h || batch < 0 || (y_dtype != QL_F32 && y_dtype != QL_F16)) return QL_E_ARG;
    if (batch == 0) return QL_OK;
    if (!x || !y) return QL_E_ARG;
    DeviceGuard g(h->L.device);
    if (!g.ok) return QL_E_CUDA;
    return forward_device(h->L, x, batch, y, y_dtype, (cudaStream_t)stream);
}

int qlinear_launch_main_kernel(qlinear_t h, const void* x, int batch, void* y, int y_dtype, void* stream) {
    if (!h || batch < 1 || (y_dtype != QL_F32 && y_dtype != QL_F16)) return QL_E_ARG;
    if (h->L.last_batch != batch) return QL_E_ARG;
    DeviceGuard g(h->L.device);
    if (!g.ok) return QL_E_CUDA;
    return launch_main(h->L, x, batch, y, y_dtype, (cudaStream_t)stream);
}

// outputs up to this size in pinned, device-addressable host memory are written
// there directly by the forward's last kernel
constexpr size_t kHostZeroCopyMaxBytes = 64 * 1024;

int qlinear_forward_host(qlinear_t h, const void* x_host, int batch, void* y_host, int y_dtype, void* stream) {
    if (!h || batch < 0 || (y_dtype != QL_F32 && y_dtype != QL_F16)) return QL_E_ARG;
    if (batch == 0) return QL_OK;
    if (!x_host || !y_host) return QL_E_ARG;
    Layer& L = h->L;
    DeviceGuard g(L.device);
    if (!g.ok) return QL_E_CUDA;
    const size_t xbytes = (size_t)batch * L.n * 2;
    const size_t ybytes = (size_t)batch * L.m * (y_dtype == QL_F16 ? 2 : 4);
    const size_t xoff = (ybytes + 255) / 256 * 256;
    int rc = ensure(&L.host_stage, &L.host_stage_bytes, xoff + xbytes);
    if (rc != QL_OK) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    char* stage = (char*)L.host_stage;
    if (cudaMemcpyAsync(stage + xoff, x_host, xbytes, cudaMemcpyHostToDevice, st) != cudaSuccess) {
        cudaGetLastError();
        return QL_E_CUDA;
    }
    // A small y in pinned host memory that the device can address is written
    // there by the forward's last kernel (no copy command after it).
    void* y_mapped = nullptr;
    if (ybytes <= kHostZeroCopyMaxBytes && ((uintptr_t)y_host & 15) == 0) {
        cudaPointerAttributes pa;
        if (cudaPointerGetAttributes(&pa, y_host) == cudaSuccess && pa.type == cudaMemoryTypeHost && pa.devicePointer)
            y_mapped = pa.devicePointer;
        else
            cudaGetLastError();
    }
    rc = forward_device(L, stage + xoff, batch, y_mapped ? y_mapped : (void*)stage, y_dtype, st);
    if (rc != QL_OK) return rc;
    if ((!y_mapped && cudaMemcpyAsync(y_host, stage, ybytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return QL_E_CUDA;
    }
    return QL_OK;
}

int qlinear_decode(qlinear_t h, void* w_hat, void* stream) {
    if (!h || !w_hat) return QL_E_ARG;
    DeviceGuard g(h->L.device);
    if (!g.ok) return QL_E_CUDA;
    for (int i = 0; i < h->L.nparts; ++i) {
        if (launch_decode(h->L, h->L.parts[i], w_hat, (cudaStream_t)stream) != cudaSuccess) {
            cudaGetLastError();
            return QL_E_CUDA;
        }
    }
    return QL_OK;
}

int qlinear_eval_code(ql_code_t code, int L, int V, const uint32_t* states, int count, void* out, void* stream) {
    if (count < 0 || L < 1 || L > 16) return QL_E_ARG;
    int rc = check_code(code, V, L);
    if (rc != QL_OK) return rc;
    if (count == 0) return QL_OK;
    if (!states || !out) return QL_E_ARG;
    uint32_t* lut_words = nullptr;
    cudaStream_t st = (cudaStream_t)stream;
    const int Q = table_bits(code, L);
    if (uses_table(code.kind)) {
        if (cudaMallocAsync((void**)&lut_words, ((size_t)1 << Q) * 4, st) != cudaSuccess) {
            cudaGetLastError();
            return QL_E_OOM;
        }
        if (copy_code_table(code, Q, V, lut_words, st) != cudaSuccess) {
            cudaGetLastError();
            cudaFreeAsync(lut_words, st);
            return QL_E_CUDA;
        }
    }
    cudaError_t e = launch_eval_code(code.kind, L, V, Q, lut_words, states, count, out, st);
    if (lut_words) cudaFreeAsync(lut_words, st);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return QL_E_CUDA;
    }
    return QL_OK;
}

int qlinear_encode(ql_code_t code, int L, int k, int V, const float* x, int blocks, uint32_t* words, float* err,
                   void* stream) {
    if (blocks < 0) return QL_E_ARG;
    if (k < 1 || k > 4 || V < 1 || V > 2) return QL_E_UNSUPPORTED;
    return qlinear_encode_kv(code, L, k * V, V, x, blocks, words, err, stream);
}

namespace {

constexpr int kEncodePoolMaxDevices = 64;
std::mutex g_encode_pool_mutex;
cudaMemPool_t g_encode_pool[kEncodePoolMaxDevices];

// The encoder's scratch pool on `device`: a memory pool of this library that
// keeps the memory it has mapped (release threshold: unlimited), so the
// search's choice buffer (148 x 256 x 2^14 bytes at L = 16, kV = 2) is mapped
// by the first call and reused by later ones instead of being mapped and
// unmapped at every call (measured: about 3.8 ms of a 13 ms call).
cudaError_t encode_pool(int device, cudaMemPool_t* pool) {
    if (device < 0 || device >= kEncodePoolMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_encode_pool_mutex);
    if (!g_encode_pool[device]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = device;
        cudaMemPool_t p = nullptr;
        cudaError_t e = cudaMemPoolCreate(&p, &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = UINT64_MAX;
        e = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) {
            cudaMemPoolDestroy(p);
            return e;
        }
        g_encode_pool[device] = p;
    }
    *pool = g_encode_pool[device];
    return cudaSuccess;
}

}  // namespace

int qlinear_encode_kv(ql_code_t code, int L, int kv, int V, const float* x, int blocks, uint32_t* words, float* err,
                      void* stream) {
    if (blocks < 0) return QL_E_ARG;
    if (V < 1 || V > 2 || kv < V || kv > 4 * V || kv > 8) return QL_E_UNSUPPORTED;
    if (L < kv || L > 16) return QL_E_UNSUPPORTED;
    int rc = check_code(code, V, L);
    if (rc != QL_OK) return rc;
    if (blocks == 0) return QL_OK;
    if (!is_device_pointer(x) || !is_device_pointer(words) || (err && !is_device_pointer(err))) return QL_E_ARG;
    const int Q = table_bits(code, L);
    if (encode_smem_bytes(L, kv, V, code.kind, Q) > (size_t)kTcMaxSmem) return QL_E_UNSUPPORTED;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return QL_E_CUDA;
    }
    int workers = 0;
    if (encode_workers(L, kv, V, code.kind, Q, blocks, sms, &workers) != cudaSuccess) {
        cudaGetLastError();
        return QL_E_CUDA;
    }
    const size_t choice_bytes = (size_t)workers * (256 / V) * ((size_t)1 << (L - kv));
    cudaStream_t st = (cudaStream_t)stream;
    cudaMemPool_t pool = nullptr;
    if (encode_pool(dev, &pool) != cudaSuccess) {
        cudaGetLastError();
        return QL_E_CUDA;
    }
    uint8_t* choice = nullptr;
    uint32_t* lut_words = nullptr;
    int* status = nullptr;
    auto release = [&]() {  // stream-ordered: back to the pool once the stream's work is done
        if (choice) cudaFreeAsync(choice, st);
        if (status) cudaFreeAsync(status, st);
        if (lut_words) cudaFreeAsync(lut_words, st);
    };
    if (cudaMallocFromPoolAsync((void**)&choice, choice_bytes, pool, st) != cudaSuccess ||
        cudaMallocFromPoolAsync((void**)&status, sizeof(int), pool, st) != cudaSuccess ||
        (uses_table(code.kind) &&
         cudaMallocFromPoolAsync((void**)&lut_words, ((size_t)1 << Q) * 4, pool, st) != cudaSuccess)) {
        cudaGetLastError();
        release();
        cudaStreamSynchronize(st);
        cudaGetLastError();
        return QL_E_OOM;
    }
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), st);
    if (e == cudaSuccess && uses_table(code.kind)) e = launch_copy_lut(code.lut, Q, V, lut_words, st);
    if (e == cudaSuccess)
        e = launch_encode(code.kind, L, kv, V, Q, lut_words, x, blocks, words, err, choice, workers, status, st);
    int dev_status = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&dev_status, status, sizeof(int), cudaMemcpyDeviceToHost, st);
    release();
    const cudaError_t es = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = es;
    if (e != cudaSuccess) cudaGetLastError();
    if (e != cudaSuccess) return QL_E_CUDA;
    return dev_status ? QL_E_DEVICE : QL_OK;
}

int qlinear_get_status(qlinear_t h) {
    if (!h) return QL_E_ARG;
    DeviceGuard g(h->L.device);
    int status = 0;
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(&status, h->L.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(h->L.status, 0, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return QL_E_CUDA;
    }
    if (status & kStatusTimeout) {
        h->L.acc_dirty = 1;  // an abandoned GEMM may have left partial sums in z
        return QL_E_TIMEOUT;
    }
    if (status) return QL_E_DEVICE;
    return QL_OK;
}

int qlinear_test_stall(qlinear_t h, int enable, int wait_tries) {
    if (!h || (enable && (wait_tries < 1 || wait_tries > 4096))) return QL_E_ARG;
    h->L.test_withhold = enable ? 1 : 0;
    h->L.test_wait_tries = enable ? wait_tries : 0;
    return QL_OK;
}

int qlinear_info(qlinear_t h, ql_info_t* info) {
    if (!h || !info) return QL_E_ARG;
    const Layer& L = h->L;
    std::memset(info, 0, sizeof(*info));
    info->m = L.m;
    info->n = L.n;
    info->L = L.L;
    info->V = L.V;
    info->code = L.code;
    info->Q = L.Q;
    info->k_top = L.parts[0].kv / L.V;
    info->k_bot = L.parts[L.nparts - 1].kv / L.V;
    info->m_top = L.parts[0].rows;
    info->B_n = L.B_n;
    info->B_m = L.B_m;
    size_t words = 0;
    for (int i = 0; i < L.nparts; ++i) words += L.parts[i].n_words;
    info->stream_bytes = words * 4;
    info->sign_bytes = (size_t)((L.n + 31) / 32 + (L.m + 31) / 32) * 4;
    info->lut_bytes = uses_table(L.code) ? ((size_t)1 << L.Q) * L.V * 2 : 0;
    info->scratch_bytes = L.xp_bytes + L.acc_bytes + L.host_stage_bytes + L.tcws_bytes;
    info->last_launches = L.last_launches;
    info->nparts = L.nparts;
    for (int i = 0; i < L.nparts; ++i) {
        info->part_rows[i] = L.parts[i].rows;
        info->part_kv[i] = L.parts[i].kv;
    }
    return QL_OK;
}

int qlinear_profile_enable(qlinear_t h, int capacity) {
    if (!h || capacity < 0 || capacity > 65536) return QL_E_ARG;
    Layer& L = h->L;
    DeviceGuard g(L.device);
    if (!g.ok) return QL_E_CUDA;
    cudaDeviceSynchronize();
    free_profiling(L);
    if (capacity == 0) return QL_OK;
    L.prof_ev = new (std::nothrow) cudaEvent_t[2 * (size_t)capacity];
    if (!L.prof_ev) return QL_E_OOM;
    for (int i = 0; i < 2 * capacity; ++i) {
        if (cudaEventCreate(&L.prof_ev[i]) != cudaSuccess) {
            cudaGetLastError();
            L.prof_cap = i / 2;
            for (int j = 2 * L.prof_cap; j < i; ++j) cudaEventDestroy(L.prof_ev[j]);
            free_profiling(L);
            return QL_E_CUDA;
        }
    }
    L.prof_cap = capacity;
    return QL_OK;
}

int qlinear_profile_read(qlinear_t h, double* total_ms, int* slots) {
    if (!h || !total_ms || !slots) return QL_E_ARG;
    Layer& L = h->L;
    DeviceGuard g(L.device);
    if (!g.ok || cudaDeviceSynchronize() != cudaSuccess) {
        cudaGetLastError();
        return QL_E_CUDA;
    }
    double sum = 0.0;
    for (int i = 0; i < L.prof_count; ++i) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, L.prof_ev[2 * i], L.prof_ev[2 * i + 1]) != cudaSuccess) {
            cudaGetLastError();
            return QL_E_CUDA;
        }
        sum += ms;
    }
    *total_ms = sum;
    *slots = L.prof_count;
    return QL_OK;
}

int qlinear_destroy(qlinear_t h) {
    if (!h) return QL_E_ARG;
    {
        DeviceGuard g(h->L.device);
        cudaDeviceSynchronize();
        free_layer(h->L);
    }
    delete h;
    return QL_OK;
}

const char* qlinear_strerror(int status) {
    switch (status) {
        case QL_OK: return "ok";
        case QL_E_ARG: return "invalid argument";
        case QL_E_UNSUPPORTED: return "unsupported configuration";
        case QL_E_CUDA: return "CUDA runtime error";
        case QL_E_OOM: return "device allocation failed";
        case QL_E_TIMEOUT: return "bounded device wait expired";
        case QL_E_DEVICE: return "device-side check failed";
        case QL_E_SCRATCH: return "request exceeds the fixed scratch of qlinear_forward_noalloc";
        default: return "unknown status";
    }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward without allocation.
//
// Some callers cannot let a library allocate device memory while they run:
// cudaMalloc and cudaFree may synchronise the whole device, which stalls every
// other stream of a serving process in the middle of its step, and runtimes
// that carve nearly all free HBM into their own pools at start-up (weights and
// a key/value cache) leave no room for a late allocation.  For them,
// qlinear_forward_noalloc keeps the decode-GEMV's scratch (x' and the fp32
// accumulator z) in one fixed array in the library's static device memory.
// The array is shared by every handle on a device, so calls that overlap in
// time (two streams, or two host threads) race on it; calls issued in order
// on one stream do not.

static __device__ __align__(256) unsigned char g_noalloc_scratch[QL_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_base[kNoAllocMaxDevices];
// Bytes from the array's start known to be all-zero (tickets and z of every
// call live there and are all-zero again after a successful call; x' is
// written at the array's end).  Starts whole: a __device__ array is
// zero-initialised.
size_t g_noalloc_clean[kNoAllocMaxDevices];
bool g_noalloc_clean_set[kNoAllocMaxDevices];

// The array's address on `device` (current on entry).  Looked up once per
// device, on that device's first call; the lookup may load the library's
// device code, which is why the first call belongs before any stream capture.
int noalloc_scratch(int device, void** base) {
    if (device < 0 || device >= kNoAllocMaxDevices) return QL_E_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_base[device]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return QL_E_CUDA;
        }
        g_noalloc_base[device] = p;
    }
    if (!g_noalloc_clean_set[device]) {
        g_noalloc_clean[device] = QL_NOALLOC_SCRATCH_BYTES;
        g_noalloc_clean_set[device] = true;
    }
    *base = g_noalloc_base[device];
    return QL_OK;
}

// Before a call whose tickets and z take the first `need` bytes and whose x'
// takes the last `xp` bytes: whether the first `need` bytes must be zeroed
// first; records the call's effect on the clean prefix.
bool noalloc_claim(int device, size_t need, size_t xp) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    size_t& clean = g_noalloc_clean[device];
    const bool zero = need > clean;
    if (zero) clean = need;
    const size_t xp_start = (size_t)QL_NOALLOC_SCRATCH_BYTES - xp;
    if (xp && xp_start < clean) clean = xp_start;  // not reached: need + xp fits
    return zero;
}

// A call failed part-way: sums or counts may be left anywhere.
void noalloc_taint(int device) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    g_noalloc_clean[device] = 0;
}

}  // namespace

extern "C" int qlinear_forward_noalloc(qlinear_t h, const void* x, int batch, void* y, int y_dtype, void* stream) {
    if (!h || batch < 0 || (y_dtype != QL_F32 && y_dtype != QL_F16)) return QL_E_ARG;
    if (batch == 0) return QL_OK;
    if (!x || !y) return QL_E_ARG;
    if (batch > kGemvMaxBatch) return QL_E_UNSUPPORTED;
    Layer& L = h->L;
    // array layout: output-block tickets and z from the start, x' at the end
    const GemvPlan pl = plan_gemv(L, batch);
    const size_t t_bytes = ticket_bytes(L);
    const size_t z_bytes = ((size_t)batch * L.m * 4 + 255) / 256 * 256;
    const size_t xp_bytes = (gemv_xstep_bytes(L, batch) + 255) / 256 * 256;
    if (t_bytes + z_bytes + xp_bytes > (size_t)QL_NOALLOC_SCRATCH_BYTES) return QL_E_SCRATCH;
    DeviceGuard g(L.device);
    if (!g.ok) return QL_E_CUDA;
    void* base = nullptr;
    const int rc = noalloc_scratch(L.device, &base);
    if (rc != QL_OK) return rc;
    int* tickets = (int*)base;
    float* z = (float*)((char*)base + t_bytes);
    void* xp = (char*)base + QL_NOALLOC_SCRATCH_BYTES - xp_bytes;
    cudaStream_t st = (cudaStream_t)stream;
    // tickets and z must start at zero: they are unless a failed call, or an
    // earlier call's x', left something there (then they are zeroed first)
    cudaError_t e = cudaSuccess;
    if (noalloc_claim(L.device, t_bytes + z_bytes, pl.x_e ? 0 : xp_bytes)) e = cudaMemsetAsync(base, 0, t_bytes + z_bytes, st);
    if (e == cudaSuccess && !pl.x_e) e = launch_rht_in_xstep(L, x, batch, xp, st);
    if (e == cudaSuccess) e = launch_gemv(L, pl, x, xp, batch, z, tickets, y, y_dtype, st);
    if (e == cudaSuccess && !pl.fuse_out) e = launch_rht_out(L, z, batch, y, y_dtype, st, gemv_z_scale(L));
    if (e != cudaSuccess) {
        cudaGetLastError();
        noalloc_taint(L.device);
        return QL_E_CUDA;
    }
    L.last_launches = (pl.x_e ? 1 : 2) + (pl.fuse_out ? 0 : 1);
    return QL_OK;
}
