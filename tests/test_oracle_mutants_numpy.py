"""Each plausible mistake planted in a copy of one of the oracle's numpy steps
(the bf16 rounding, the key-value projection, the 3x3 depthwise convolution,
the GLU and the Mix-FFN composition) must fail at least one pin, so the pins
constrain those steps as the C-source mutants show for the attention. A mutant
replaces one method on a fresh oracle instance; the oracle itself is never
modified. CPU only."""
import numpy as np
import pytest

from oracle import Oracle
from tests import pins


def _round_bits(x, bits, rounding):
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(rounding(np.ldexp(m, bits)), e - bits)


def _half_away(v):
    return np.sign(v) * np.floor(np.abs(v) + 0.5)


def _project(orc, X, Wk, Wv, H, rnd=True, k_from_v=False, interleave=False):
    X, Wk, Wv = (np.asarray(a, dtype=np.float64) for a in (X, Wk, Wv))
    B, N, _ = X.shape
    HD = Wk.shape[0]
    r = orc.round_bf16 if rnd else (lambda a: a)
    K = r(X @ (Wv if k_from_v else Wk).T)
    V = r(X @ Wv.T)
    if interleave:      # channel o read as head o % H, feature o // H
        return (K.reshape(B, N, HD // H, H).transpose(0, 1, 3, 2).copy(),
                V.reshape(B, N, HD // H, H).transpose(0, 1, 3, 2).copy())
    return K.reshape(B, N, H, HD // H), V.reshape(B, N, H, HD // H)


def _depthwise(U, Kdw, hw, pad="zero", taps=lambda K, dy, dx: K[:, dy, dx], x_major=False):
    U = np.asarray(U, dtype=np.float64)
    Kdw = np.asarray(Kdw, dtype=np.float64)
    Hg, W = hw
    B, N, Cc = U.shape
    if x_major:         # tokens read as n = x * Hg + y
        G0 = U.reshape(B, W, Hg, Cc).transpose(0, 2, 1, 3)
    else:
        G0 = U.reshape(B, Hg, W, Cc)
    G = np.pad(G0, ((0, 0), (1, 1), (1, 1), (0, 0)), mode="wrap" if pad == "wrap" else "constant")
    D = np.zeros((B, Hg, W, Cc))
    for dy in range(3):
        for dx in range(3):
            D += G[:, dy:dy + Hg, dx:dx + W, :] * taps(Kdw, dy, dx)
    if x_major:
        D = D.transpose(0, 2, 1, 3)
    return D.reshape(B, N, Cc)


def _mix_ffn(orc, X, W1, Kdw, W2, hw, gate="glu", round_u=True, round_z=True, depthwise=True):
    X, W1, W2 = (np.asarray(a, dtype=np.float64) for a in (X, W1, W2))
    Ch = W1.shape[0] // 2
    U = X @ W1.T
    if round_u:
        U = orc.round_bf16(U)
    D = orc.depthwise3x3(U, Kdw, hw) if depthwise else U
    a, g = D[..., :Ch], D[..., Ch:]
    sig = lambda t: 1.0 / (1.0 + np.exp(-t))
    Z = {"glu": a * sig(g), "swapped": sig(a) * g, "silu": a * g * sig(g)}[gate]
    if round_z:
        Z = orc.round_bf16(Z)
    return Z @ W2.T


def _glu_stage(orc, U, Kdw, hw, gate="glu", rnd=True):
    D = orc.depthwise3x3(U, Kdw, hw)
    Ch = D.shape[-1] // 2
    a, g = D[..., :Ch], D[..., Ch:]
    sig = lambda t: 1.0 / (1.0 + np.exp(-t))
    Z = {"glu": a * sig(g), "swapped": sig(a) * g, "silu": a * g * sig(g)}[gate]
    return orc.round_bf16(Z) if rnd else Z


# name -> (method replaced, factory of the replacement given the instance)
MUTANTS = {
    "round_truncates": ("round_bf16", lambda o: lambda x: _round_bits(x, 8, np.trunc)),
    "round_half_away_from_zero": ("round_bf16", lambda o: lambda x: _round_bits(x, 8, _half_away)),
    "round_keeps_9_bits": ("round_bf16", lambda o: lambda x: _round_bits(x, 9, np.round)),
    "projection_not_rounded": ("project_kv", lambda o: lambda X, Wk, Wv, H: _project(o, X, Wk, Wv, H, rnd=False)),
    "projection_K_from_Wv": ("project_kv", lambda o: lambda X, Wk, Wv, H: _project(o, X, Wk, Wv, H, k_from_v=True)),
    "projection_heads_interleaved": ("project_kv",
                                     lambda o: lambda X, Wk, Wv, H: _project(o, X, Wk, Wv, H, interleave=True)),
    "depthwise_wraps_around": ("depthwise3x3", lambda o: lambda U, K, hw: _depthwise(U, K, hw, pad="wrap")),
    "depthwise_taps_transposed": ("depthwise3x3",
                                  lambda o: lambda U, K, hw: _depthwise(U, K, hw, taps=lambda K_, dy, dx: K_[:, dx, dy])),
    "depthwise_kernel_flipped": ("depthwise3x3",
                                 lambda o: lambda U, K, hw: _depthwise(
                                     U, K, hw, taps=lambda K_, dy, dx: K_[:, 2 - dy, 2 - dx])),
    "depthwise_grid_x_major": ("depthwise3x3", lambda o: lambda U, K, hw: _depthwise(U, K, hw, x_major=True)),
    "glu_halves_swapped": ("mix_ffn", lambda o: lambda *a: _mix_ffn(o, *a, gate="swapped")),
    "glu_silu_gate": ("mix_ffn", lambda o: lambda *a: _mix_ffn(o, *a, gate="silu")),
    "mix_ffn_u_not_rounded": ("mix_ffn", lambda o: lambda *a: _mix_ffn(o, *a, round_u=False)),
    "mix_ffn_z_not_rounded": ("mix_ffn", lambda o: lambda *a: _mix_ffn(o, *a, round_z=False)),
    "mix_ffn_no_depthwise": ("mix_ffn", lambda o: lambda *a: _mix_ffn(o, *a, depthwise=False)),
    "stage_glu_halves_swapped": ("depthwise_glu", lambda o: lambda U, K, hw: _glu_stage(o, U, K, hw, gate="swapped")),
    "stage_glu_silu_gate": ("depthwise_glu", lambda o: lambda U, K, hw: _glu_stage(o, U, K, hw, gate="silu")),
    "stage_glu_not_rounded": ("depthwise_glu", lambda o: lambda U, K, hw: _glu_stage(o, U, K, hw, rnd=False)),
    "stage_expand_not_rounded": ("expand", lambda o: lambda X, W1: np.asarray(X, dtype=np.float64)
                                 @ np.asarray(W1, dtype=np.float64).T),
    "stage_expand_transposed_weights": ("expand", lambda o: lambda X, W1: o.round_bf16(
        np.asarray(X, dtype=np.float64) @ np.asarray(W1, dtype=np.float64).reshape(-1, W1.shape[0]))),
}


def test_unmutated_copies_pass_every_pin():
    """The copies the mutants are made from (with no mistake planted) agree with
    the oracle's own steps, so a failing pin below is the planted mistake."""
    orc = Oracle()
    rng = np.random.default_rng(7)
    x = rng.standard_normal(1000) * 3
    assert np.array_equal(_round_bits(x, 8, np.round), orc.round_bf16(x))
    X, Wk, Wv = rng.standard_normal((2, 5, 6)), rng.standard_normal((8, 6)), rng.standard_normal((8, 6))
    for got, want in zip(_project(orc, X, Wk, Wv, 2), orc.project_kv(X, Wk, Wv, 2)):
        assert np.array_equal(got, want)
    U, Kd = rng.standard_normal((2, 12, 4)), rng.standard_normal((4, 3, 3))
    assert np.allclose(_depthwise(U, Kd, (3, 4)), orc.depthwise3x3(U, Kd, (3, 4)), rtol=0, atol=1e-13)
    X2, W1, W2 = rng.standard_normal((1, 12, 5)), rng.standard_normal((6, 5)), rng.standard_normal((5, 3))
    Kd2 = rng.standard_normal((6, 3, 3))
    assert np.allclose(_mix_ffn(orc, X2, W1, Kd2, W2, (3, 4)), orc.mix_ffn(X2, W1, Kd2, W2, (3, 4)),
                       rtol=1e-13, atol=1e-13)
    U2 = orc.expand(X2, W1)
    assert np.array_equal(_glu_stage(orc, U2, Kd2, (3, 4)), orc.depthwise_glu(U2, Kd2, (3, 4)))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_numpy_mutant_is_caught(name):
    method, factory = MUTANTS[name]
    orc = Oracle()
    setattr(orc, method, factory(orc))
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, FloatingPointError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passes every pin"
