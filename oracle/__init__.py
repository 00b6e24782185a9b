"""CPU oracle for the trellis-coded quantized linear layer (test infrastructure).

This package is a plain, slow, float64 restatement of what the layer computes,
written from the QTIP OpenReview discussion ("QTIP: Quantization with Trellises
and Incoherence Processing", paperhub.cn/paper/7sdkLVuYCU) and the QuIP# page
(signal-papers.cortex.a2olabs.com/p/2402.04396, Fig. 2):

    y = alpha * diag(s_out) * H_m^T * W_hat * H_n * diag(s_in) * x

It exists only to check the CUDA library. Only tests/, __graft_entry__.smoke()
and bench.py's CPU-baseline leg may import it; the library never does, and it
shares no code, header, table or constant generator with the CUDA sources
(the code constants below were typed separately on each side from the format
specification).

Modules:
  fp16      IEEE binary16 decoding and round-to-nearest-even, from the definition
  bitstream MSB-first bit access and the canonical stream layout
  trellis   the bitshift-trellis state walk (QTIP discussion, "Figure 2 (Q4)")
  e8p       an E8-lattice codebook of 2^16 eight-dimensional entries (QuIP#
            page, abstract and Fig. captions: the E8P-style comparison VQ)
  codes     the 1MAD, 3INST and HYB codes ("Inference speed analysis", "HYB
            Uniqueness", "Bit Accounting") and the table code of the palette
            quantizers (VQ / NUQ, Q-Palette page)
  hadamard  dense normalised Walsh-Hadamard blocks and the random-sign RHT
            (QuIP# Fig. 2; QTIP discussion, "Incoherence Processing (W2)")
  qlinear   decode of W_hat and the forward pass (dense, naive), at whole or
            half-integer bits per weight
  encode    trellis-coded quantization (tail-biting Viterbi)
  stats     the statistics the pins use (moments, neighbour dependence)

Parity status: every function here is pinned by a -m "not gpu" test against
values or properties fixed by the pages or by mathematics (tests/test_oracle_*.py).
The code constants themselves are a reading (the pages do not print them); what
pins them is the set of properties the pages claim for the codes.
"""
from . import fp16, bitstream, trellis, e8p, codes, hadamard, qlinear, stats  # noqa: F401
