"""Planted mistakes in the oracle, on the CPU: each test swaps one oracle
function for a plausible wrong version (a dropped term, a wrong index or
order) and checks that the pin guarding that part of the oracle fails.
(The trellis walk's own planted mistakes are in test_oracle_trellis.py.)"""
import numpy as np
import pytest

import test_oracle_encode as t_encode
import test_oracle_palette as t_palette
import test_oracle_qlinear as t_qlinear
import workloads as wl
from oracle import bitstream, codes, encode, hadamard, qlinear


def _fails(pin, *args):
    with pytest.raises(AssertionError):
        pin(*args)


def test_dropped_input_signs_are_caught(monkeypatch):
    """x' = H_n x instead of H_n diag(s_in) x."""
    monkeypatch.setattr(qlinear.Layer, "input_transform",
                        lambda self, x: hadamard.apply_blockwise(np.asarray(x).astype(np.float64), self.B_n))
    _fails(t_qlinear.test_forward_equals_dense_weight, 48, 768, 3, wl.CODE_3INST, 1)


def test_dropped_output_signs_are_caught(monkeypatch):
    """y = alpha H_m z instead of alpha diag(s_out) H_m z."""
    def forward_blocks(self, x, out_blocks):
        xp = self.input_transform(x)
        out = {}
        for b in out_blocks:
            rows = np.arange(b * self.B_m, (b + 1) * self.B_m)
            out[b] = self.alpha * hadamard.apply_blockwise(xp @ self.decode_rows(rows).T, self.B_m)
        return out
    monkeypatch.setattr(qlinear.Layer, "forward_blocks", forward_blocks)
    _fails(t_qlinear.test_forward_equals_dense_weight, 48, 768, 3, wl.CODE_3INST, 1)


def test_unnormalised_hadamard_is_caught(monkeypatch):
    """H_B without its 1/sqrt(B)."""
    real = hadamard.dense
    monkeypatch.setattr(hadamard, "dense", lambda B, normalised=True, rows=None: real(B, False, rows))
    _fails(t_qlinear.test_forward_equals_dense_weight, 32, 512, 4, wl.CODE_HYB, 2)


def test_swapped_pair_order_of_the_table_code_is_caught(monkeypatch):
    """Value e = 1 of a codebook entry placed in column e = 0 and vice versa."""
    real = codes.table
    monkeypatch.setattr(codes, "table", lambda state, lut: real(state, lut)[..., ::-1])
    _fails(t_palette.test_memoryless_table_code_is_a_field_lookup, 5, 2)
    _fails(t_encode.test_vq_with_a_product_codebook_is_per_dimension_scalar_quantization)


def test_fractional_row_offsets_rounded_down_are_caught(monkeypatch):
    """Rows of a 2.5-bit layer laid out as if they held 2 bits per weight."""
    real = bitstream.bits
    monkeypatch.setattr(bitstream, "bits", lambda k, weights: real(int(k), weights))
    _fails(t_palette.test_fractional_states_are_cyclic_windows, 16, 2.5, 2)


def test_absolute_instead_of_squared_error_is_caught(monkeypatch):
    """The search scoring |x - v| instead of (x - v)^2."""
    def step_costs(x, values, dtype):
        x = x.astype(dtype)
        v = values.astype(dtype)
        d = np.zeros((x.shape[0], v.shape[0]), dtype=dtype)
        for e in range(x.shape[1]):
            d = (d + np.abs(x[:, e:e + 1] - v[None, :, e])).astype(dtype)
        return d
    monkeypatch.setattr(encode, "_step_costs", step_costs)
    _fails(t_encode.test_exact_viterbi_equals_brute_force, 4, 1, 1, wl.CODE_3INST, 8)


def test_round_half_up_instead_of_to_even_is_caught(monkeypatch):
    """fp16 rounding with ties away from zero (floor(x + 1/2)) instead of to even."""
    from oracle import fp16
    import test_oracle_fp16 as t_fp16

    def round_half_up(v):
        v = np.asarray(v, dtype=np.float64)
        a = np.abs(v)
        mant, ex = np.frexp(np.where(a > 0, a, 1.0))
        q = np.exp2((np.maximum(ex - 1, -14) - 10).astype(np.float64))
        r = np.where(a == 0, 0.0, np.floor(a / q + 0.5) * q)
        r = np.where(a >= 65520.0, np.inf, r)
        return np.copysign(r, v)
    monkeypatch.setattr(fp16, "round_rne", round_half_up)
    _fails(t_fp16.test_round_ties_to_even_and_overflow)


def test_reversed_steps_inside_a_block_are_caught(monkeypatch):
    """Decoded values placed at column 256 j + (T/V - 1 - t) V + e instead of 256 j + t V + e."""
    def decode_rows(self, rows, blocks=None):
        rows = np.asarray(rows, dtype=np.int64)
        from oracle import trellis
        states = trellis.block_states(self.words, rows, self.n, self.parts, self.L, self.V, blocks)
        vals = codes.evaluate(self.code, states, self.V, self.lut)[:, :, ::-1, :]
        return vals.reshape(len(rows), -1)
    monkeypatch.setattr(qlinear.Layer, "decode_rows", decode_rows)
    _fails(t_qlinear.test_element_order_inside_a_block)
    _fails(t_palette.test_memoryless_table_code_is_a_field_lookup, 3, 1)


def test_3inst_without_its_high_half_is_caught(monkeypatch):
    """3INST taking only the low half (one fp16 value) instead of the sum of both halves."""
    import test_oracle_codes as t_codes

    def low_half_only(state):
        from oracle import fp16
        x = codes.lcg(state, codes.A_3INST, codes.B_3INST).astype(np.int64)
        m = (x & codes.MASK_3INST) ^ codes.XOR_3INST
        return fp16.round_rne(fp16.decode_bits(m & 0xFFFF))
    monkeypatch.setattr(codes, "three_inst", low_half_only)
    _fails(t_codes.test_computed_code_is_close_to_standard_normal, codes.three_inst)


def test_e8_code_without_its_parity_sign_is_caught(monkeypatch):
    """The sign of coordinate 7 taken from nowhere (always +) instead of the
    even-sum rule: half the codewords leave the lattice."""
    import test_oracle_e8p as t_e8p
    from oracle import e8p

    def no_parity(state):
        s = np.asarray(state, dtype=np.int64)
        T = e8p.shape_table()[s >> 8]
        neg = np.stack([(s >> (i + 1)) & 1 for i in range(7)] + [np.zeros_like(s)], axis=-1)
        return (1.0 - 2.0 * neg) * T + np.where(s & 1, 0.25, -0.25)[..., None]
    monkeypatch.setattr(e8p, "codeword", no_parity)
    _fails(t_e8p.test_every_codeword_is_a_shifted_e8_point_and_the_set_is_symmetric)
