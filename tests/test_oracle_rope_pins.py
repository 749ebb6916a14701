"""Pins for the oracle's rotary position embedding (``oracle.rope``).

Pinned to: values worked out by hand with ``math.cos``/``math.sin`` for tiny
head dims (so theta_j's exponent and the pairing are fixed), numpy complex
multiplication by exp(i p theta), the invariants of a rotation (pair norms,
position 0 = identity, untouched features past rot_dim, scores that depend
only on p - p'), and the decode offset (the new token's rows equal the
prefill rows of the last token).  ``planted`` edits a copy of the oracle's
source and checks that the pins notice.
"""

import inspect
import math

import numpy as np
import pytest

import oracle
from oracle import hd_oracle
from stream_sequence_attention_b200 import synth


def test_two_dims_rotate_by_position_radians():
    # rot_dim = 2: theta_0 = 1, so position p rotates by p radians.
    x = np.zeros((1, 4, 1, 2))
    x[..., 0] = 1.0
    out = oracle.rope(x, 2, base=12345.0, layout="half")
    for p in range(4):
        np.testing.assert_allclose(out[0, p, 0], [math.cos(p), math.sin(p)], atol=1e-15)


def test_four_dims_by_hand_both_layouts():
    # base 100, rot_dim 4: theta = (1, 100^(-1/2) = 0.1).  Position 2.
    x = np.zeros((1, 3, 1, 4))
    x[0, 2, 0] = [1.0, 0.0, 0.0, 1.0]
    half = oracle.rope(x, 4, base=100.0, layout="half")[0, 2, 0]
    # pairs (x0, x2) = (1, 0) by 2 rad; (x1, x3) = (0, 1) by 0.2 rad
    want = [math.cos(2), -math.sin(0.2), math.sin(2), math.cos(0.2)]
    np.testing.assert_allclose(half, want, atol=1e-15)
    inter = oracle.rope(x, 4, base=100.0, layout="interleaved")[0, 2, 0]
    # pairs (x0, x1) = (1, 0) by 2 rad; (x2, x3) = (0, 1) by 0.2 rad
    want = [math.cos(2), math.sin(2), -math.sin(0.2), math.cos(0.2)]
    np.testing.assert_allclose(inter, want, atol=1e-15)


def test_partial_rotary_uses_rot_dim_in_theta_and_keeps_the_rest():
    # rot_dim 4 of D 6, base 100: theta = (1, 0.1) as above; features 4, 5 untouched.
    x = np.zeros((1, 3, 1, 6))
    x[0, 2, 0] = [1.0, 0.0, 0.0, 1.0, 7.0, -3.0]
    out = oracle.rope(x, 4, base=100.0, layout="half")[0, 2, 0]
    np.testing.assert_allclose(out, [math.cos(2), -math.sin(0.2), math.sin(2), math.cos(0.2), 7.0, -3.0],
                               atol=1e-15)


@pytest.mark.parametrize("layout", ["half", "interleaved"])
@pytest.mark.parametrize("rot", [8, 16])
def test_complex_multiplication(layout, rot):
    B, P, H, D, base = 2, 9, 3, 16, 5000.0
    x = synth.normal((B, P, H, D), 3).astype(np.float64)
    out = oracle.rope(x, rot, base, layout)
    half = rot // 2
    if layout == "half":
        z = x[..., :half] + 1j * x[..., half:rot]
    else:
        z = x[..., 0:rot:2] + 1j * x[..., 1:rot:2]
    theta = np.array([base ** (-2 * j / rot) for j in range(half)])
    zr = z * np.exp(1j * np.arange(P)[None, :, None, None] * theta)
    if layout == "half":
        got = out[..., :half] + 1j * out[..., half:rot]
    else:
        got = out[..., 0:rot:2] + 1j * out[..., 1:rot:2]
    np.testing.assert_allclose(got, zr, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(out[..., rot:], x[..., rot:])


@pytest.mark.parametrize("layout", ["half", "interleaved"])
def test_rotation_invariants(layout):
    x = synth.normal((1, 20, 2, 8), 5).astype(np.float64)
    out = oracle.rope(x, 8, 10000.0, layout)
    np.testing.assert_array_equal(out[:, 0], x[:, 0])  # position 0: identity
    np.testing.assert_allclose(np.linalg.norm(out, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)


@pytest.mark.parametrize("layout", ["half", "interleaved"])
def test_scores_depend_only_on_relative_position(layout):
    D = 16
    q = synth.normal((1, 1, 1, D), 7).astype(np.float64)
    k = synth.normal((1, 1, 1, D), 8).astype(np.float64)

    def at(x, p):
        return oracle.rope(x, D, 10000.0, layout, pos_base=p)[0, 0, 0]

    for p, pk, c in [(5, 2, 11), (100, 37, 1000), (3, 3, 250)]:
        a = at(q, p) @ at(k, pk)
        b = at(q, p + c) @ at(k, pk + c)
        assert abs(a - b) < 1e-10


def test_expanded_positions_and_decode_offset():
    # Prefill row p = i*n + s sits at position p; the decode rows of the new
    # token T-1 (r = s) with pos_base = -n, pos_mult = n, pos0 = T land at
    # (T-1)*n + s -- the prefill rows of the last token.
    n, L, H, D = 3, 7, 2, 8
    x = synth.normal((2, n * L, H, D), 9).astype(np.float64)
    full = oracle.rope(x, D, 500.0)
    T = np.array([L, 4])
    for b in range(2):
        dec_in = x[b:b + 1, (T[b] - 1) * n:(T[b] - 1) * n + n]
        dec = oracle.rope(dec_in, D, 500.0, pos_base=-n, pos_mult=n, pos0=T[b:b + 1])
        np.testing.assert_allclose(dec[0], full[b, (T[b] - 1) * n:T[b] * n], rtol=1e-12, atol=1e-12)


_PLANTS = {
    "sin_sign": ("out[b, :, :, :half] = xa * c - xb * s", "out[b, :, :, :half] = xa * c + xb * s"),
    "theta_over_D": ("theta = float(base) ** (-2.0 * j / rot_dim)", "theta = float(base) ** (-1.0 * j / rot_dim)"),
    "pos_off_by_one": ("ang = rope_angles(start + np.arange(P), rot_dim, base)",
                       "ang = rope_angles(start + 1 + np.arange(P), rot_dim, base)"),
    "half_pairs_swapped": ("xa, xb = x[b, :, :, :half], x[b, :, :, half:rot_dim]",
                           "xb, xa = x[b, :, :, :half], x[b, :, :, half:rot_dim]"),
}


@pytest.mark.parametrize("kind", sorted(_PLANTS))
def test_planted_rope_mistakes_are_caught(kind, monkeypatch):
    src = inspect.getsource(hd_oracle.rope) + "\n" + inspect.getsource(hd_oracle.rope_angles)
    a, b = _PLANTS[kind]
    assert a in src
    ns = dict(vars(hd_oracle))
    exec(src.replace(a, b), ns)
    monkeypatch.setattr(oracle, "rope", ns["rope"])
    failed = False
    for t in (test_two_dims_rotate_by_position_radians, test_four_dims_by_hand_both_layouts,
              test_partial_rotary_uses_rot_dim_in_theta_and_keeps_the_rest):
        try:
            t()
        except AssertionError:
            failed = True
    assert failed
