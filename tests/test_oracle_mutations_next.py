"""Planted mistakes in the oracle's block, RoPE, prefix and relative-position functions (CPU only):
each must fail one of the pins in test_oracle_block_pins, test_oracle_partial_pins and
test_oracle_relpos_pins. The mistakes are plausible slips of someone writing those functions:
swapped axes, a wrong frequency exponent, a flipped relative index, q and k columns exchanged,
LN2 applied to the wrong tensor, the prefix keys forgotten."""
import math

import numpy as np
import pytest

from oracle import sparsesam_oracle as O
from tests import test_oracle_block_pins as BP
from tests import test_oracle_partial_pins as PP
from tests import test_oracle_relpos_pins as RP


def _rope_variant(swap_axes=False, freq_exp=None):
    def rope(x, grid_h, grid_w, base):
        x = np.asarray(x, dtype=np.float64)
        U, T, H, D = x.shape
        half, quart = D // 2, D // 4
        pos = (np.arange(T) // grid_w, np.arange(T) % grid_w)
        if swap_axes:
            pos = pos[::-1]
        out = x.copy()
        for axis in (0, 1):
            for i in range(quart):
                d = axis * half + 2 * i
                e = freq_exp(i, D) if freq_exp else -i / quart
                phi = pos[axis] * float(base) ** e
                c, s = np.cos(phi)[None, :, None], np.sin(phi)[None, :, None]
                a, b = x[:, :, :, d], x[:, :, :, d + 1]
                out[:, :, :, d] = a * c - b * s
                out[:, :, :, d + 1] = a * s + b * c
        return out
    return rope


def test_mutation_rope_axes_swapped_caught(monkeypatch):
    monkeypatch.setattr(O, "rope_2d", _rope_variant(swap_axes=True))
    with pytest.raises(AssertionError):
        PP.test_rope_closed_form_angles()


def test_mutation_rope_frequency_caught(monkeypatch):
    # base^(-2i/dh) instead of base^(-i/(dh/4))
    monkeypatch.setattr(O, "rope_2d", _rope_variant(freq_exp=lambda i, D: -2 * i / D))
    with pytest.raises(AssertionError):
        PP.test_rope_closed_form_angles()


def test_mutation_relpos_index_flipped_caught(monkeypatch):
    def wrong(q, rel_h, rel_w, Hu, Wu):
        q = np.asarray(q, dtype=np.float64)
        U, N, H, D = q.shape
        y, x = np.arange(N) // Wu, np.arange(N) % Wu
        qh = np.einsum("unhd,rd->uhnr", q, np.asarray(rel_h, np.float64))
        qw = np.einsum("unhd,rd->uhnr", q, np.asarray(rel_w, np.float64))
        rows = np.arange(N)[:, None]
        return (qh[:, :, rows, y[None, :] - y[:, None] + Hu - 1]
                + qw[:, :, rows, x[None, :] - x[:, None] + Wu - 1])
    monkeypatch.setattr(O, "relpos_bias", wrong)
    with pytest.raises(AssertionError):
        RP.test_bias_hand_values_2x2()


def _block_variant(swap_qk=False, ln2_on_x=False):
    def block(x, prm, perm, keep, geo, heads, density):
        x = np.asarray(x, dtype=np.float64)
        C = x.shape[-1]
        dh = C // heads
        xu = O.to_units(O.layer_norm(x, prm.ln1_w, prm.ln1_b), geo)
        qkv = O._lin(xu, prm.w_qkv, prm.b_qkv)
        U, N, _ = qkv.shape
        q, k, v = (qkv[..., i * C:(i + 1) * C].reshape(U, N, heads, dh) for i in range(3))
        if swap_qk:
            q, k = k, q
        a = O.attention(q, k, v, perm, density).reshape(U, N, C)
        x1 = x + O.from_units(O._lin(a, prm.w_proj, prm.b_proj), geo)
        y = x1.copy()
        for b in range(x.shape[0]):
            rows = np.asarray(keep[b], dtype=np.int64)
            src = x if ln2_on_x else x1
            h = O.gelu(O._lin(O.layer_norm(src[b, rows], prm.ln2_w, prm.ln2_b), prm.w1, prm.b1))
            y[b, rows] = x1[b, rows] + O._lin(h, prm.w2, prm.b2)
        return y
    return block


def test_mutation_block_qk_exchanged_caught(monkeypatch):
    monkeypatch.setattr(O, "encoder_block", _block_variant(swap_qk=True))
    with pytest.raises(AssertionError):
        BP.test_block_at_density_one_is_the_dense_sam_block_global()


def test_mutation_block_ln2_on_input_caught(monkeypatch):
    monkeypatch.setattr(O, "encoder_block", _block_variant(ln2_on_x=True))
    with pytest.raises(AssertionError):
        BP.test_block_at_density_one_is_the_dense_sam_block_windowed()


def test_mutation_partial_prefix_keys_forgotten_caught(monkeypatch):
    real = O.attention_partial

    def wrong(q, k, v, perm, density, prefix, grid_h, grid_w, rope_base):
        y = real(q, k, v, perm, density, prefix, grid_h, grid_w, rope_base)
        # patch rows computed without the prefix keys
        qn = np.asarray(q, np.float64).copy()
        kn = np.asarray(k, np.float64).copy()
        if rope_base:
            qn[:, prefix:] = O.rope_2d(qn[:, prefix:], grid_h, grid_w, rope_base)
            kn[:, prefix:] = O.rope_2d(kn[:, prefix:], grid_h, grid_w, rope_base)
        y[:, prefix:] = O.attention(qn[:, prefix:], kn[:, prefix:],
                                    np.asarray(v, np.float64)[:, prefix:], perm, density)
        return y
    monkeypatch.setattr(O, "attention_partial", wrong)
    with pytest.raises(AssertionError):
        PP.test_partial_at_density_one_is_dense_attention_with_rope()
