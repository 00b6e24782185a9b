// encode.h -- the trellis-coded quantizer's launchers (encode.cu), used by the C ABI.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace qlk {

// Trellis-coded quantization of `blocks` blocks of 256 source values (two-pass
// tail-biting Viterbi, L <= 16, kv bits per step): words [blocks][8 kv / V] in
// the stream format, the squared error of each block's reconstruction into
// err (may be null).  Blocks are shared out over `workers`: one CTA per block
// whenever the group minima fit its shared memory, else (L = 16, kv = 1) a
// cluster of 4 CTAs per block (encode_workers gives how many run at once);
// choice: workers * (256/V) * 2^(L-kv) bytes of scratch.
size_t encode_smem_bytes(int L, int kv, int V, int code, int Q);
cudaError_t encode_workers(int L, int kv, int V, int code, int Q, int blocks, int num_sms, int* workers);
cudaError_t launch_encode(int code, int L, int kv, int V, int Q, const uint32_t* lut, const float* x, int blocks,
                          uint32_t* words, float* err, uint8_t* choice, int workers, int* status, cudaStream_t st);

}  // namespace qlk
