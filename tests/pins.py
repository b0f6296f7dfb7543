"""Pins for the fp64 oracle: checks against what the pages and the mathematics
fix, none of which reuses the oracle's own code.

Each ``pin_*`` function takes an oracle object (anything with ``state``,
``apply`` and ``forward`` like ``oracle.Oracle``) and raises AssertionError if
the oracle disagrees with the pin. ``tests/test_oracle_pins.py`` runs them on
the real oracle; ``tests/test_oracle_mutants.py`` runs them on copies of the
oracle with a planted mistake and requires each copy to fail at least one.

Passages:
  * normalised form phi(Q)(phi(K)^T V) / (phi(Q) phi(K)^T 1):
    "linear-diffusion-transformer-4k-efficient-generation" (blog.hotdry.top),
    section "核心架构：Linear Attention 与 DC-AE 的协同设计";
  * phi = ReLU and the d x d intermediate KV = phi(K)^T V, A = phi(Q) KV:
    "08_sana高效高分辨率生成" (papers-3lj.pages.dev), "Linear Attention 的原理";
  * the shared terms are computed once for all queries, which equals the
    per-query n x n form: "SANA: Efficient High-Resolution Image Synthesis with
    Linear Diffusion Transformers" (phd-frog.tistory.com/40), section 2.2,
    "선형 어텐션 블럭" (Eq. 1 prose).
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def bruteforce(Q, K, V, eps):
    """The quadratic definition: W = phi(Q) phi(K)^T (N x N per (b, h)),
    O = (W V) / (W 1 + eps). numpy fp64, per (b, h) slice of (B, N, H, d)."""
    Q, K, V = (np.asarray(x, dtype=np.float64) for x in (Q, K, V))
    B, N, H, d = Q.shape
    O = np.empty_like(Q)
    for b in range(B):
        for h in range(H):
            q = np.maximum(Q[b, :, h, :], 0.0)
            k = np.maximum(K[b, :, h, :], 0.0)
            W = q @ k.T
            O[b, :, h, :] = (W @ V[b, :, h, :]) / (W.sum(axis=1, keepdims=True) + eps)
    return O


def row_relerr(O, R):
    """normwise relative error per (b, n, h) row of length d; rows with a zero
    reference norm report the plain norm of O (so they must be exactly 0)."""
    num = np.linalg.norm(O - R, axis=-1)
    den = np.linalg.norm(R, axis=-1)
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), num)


def _rng_inputs(seed, B=2, N=33, H=3, d=8, scale=1.0):
    rng = np.random.default_rng(seed)
    return tuple(scale * rng.standard_normal((B, N, H, d)) for _ in range(3))


# --------------------------------------------------------------------- pins --

def pin_bruteforce(orc, Q, K, V, eps, tol=1e-12):
    """Reassociated oracle == explicit n x n form to tol (normwise per row);
    rows whose reference is exactly 0 must be exactly 0."""
    O = orc.forward(Q, K, V, eps)
    R = bruteforce(Q, K, V, eps)
    err = row_relerr(O, R)
    assert np.all(np.isfinite(O)), "oracle produced non-finite values"
    assert err.max() <= tol, f"max row rel err vs brute force {err.max():.3e} > {tol}"
    zero = np.linalg.norm(R, axis=-1) == 0
    assert np.all(O[zero] == 0.0), "rows with phi(Q)=0 must be exactly 0"


def exact_rational(Q, K, V, eps: Fraction):
    """The quadratic definition in exact rational arithmetic (small inputs)."""
    B, N, H, d = Q.shape
    M = K.shape[1]           # keys may be fewer than queries (a causal prefix)
    out = np.empty((B, N, H, d), dtype=object)
    relu = (lambda x: x if x > 0 else Fraction(0))
    for b in range(B):
        for h in range(H):
            for n in range(N):
                w = [sum((relu(Fraction(Q[b, n, h, i])) * relu(Fraction(K[b, m, h, i]))
                          for i in range(d)), Fraction(0)) for m in range(M)]
                den = sum(w, Fraction(0)) + eps
                for j in range(d):
                    num = sum((w[m] * Fraction(V[b, m, h, j]) for m in range(M)), Fraction(0))
                    out[b, n, h, j] = num / den
    return out


def pin_exact_integers(orc, seed=11):
    """Small-integer inputs with eps = 1/4: every product and sum the oracle
    forms is exact in fp64, so its result must equal the correctly rounded
    exact rational value, bit for bit."""
    rng = np.random.default_rng(seed)
    B, N, H, d = 2, 5, 2, 3
    Q, K, V = (rng.integers(-3, 4, size=(B, N, H, d)).astype(np.float64) for _ in range(3))
    Q[0, 1, 0, :] = -np.abs(Q[0, 1, 0, :]) - 1  # one all-negative query row
    eps = Fraction(1, 4)
    ref = exact_rational(Q, K, V, eps)
    O = orc.forward(Q, K, V, float(eps))
    want = np.vectorize(float)(ref).astype(np.float64)
    assert np.array_equal(O, want), f"oracle != exact rational result:\n{O}\n{want}"


def pin_hand_example(orc):
    """A hand-worked case (d = 2, N = 2, one head).
    phi(Q_0) = [1, 0]; phi(K) = [[1, 2], [3, 0]] -> weights w = [1, 3], sum 4.
    num = 1*[1, 2] + 3*[3, 4] = [10, 14].  eps = 0 -> [2.5, 3.5];
    eps = 1 -> [2, 2.8].  Query 1 = [-1, 2] -> phi = [0, 2]: w = [4, 0],
    num = 4*[1, 2] = [4, 8], den 4 -> [1, 2] (eps 0) or [0.8, 1.6] (eps 1)."""
    Q = np.array([[1.0, -1.0], [-1.0, 2.0]]).reshape(1, 2, 1, 2)
    K = np.array([[1.0, 2.0], [3.0, -1.0]]).reshape(1, 2, 1, 2)
    V = np.array([[1.0, 2.0], [3.0, 4.0]]).reshape(1, 2, 1, 2)
    O0 = orc.forward(Q, K, V, 0.0).reshape(2, 2)
    O1 = orc.forward(Q, K, V, 1.0).reshape(2, 2)
    assert np.array_equal(O0, np.array([[2.5, 3.5], [1.0, 2.0]])), O0
    assert np.allclose(O1, np.array([[2.0, 2.8], [0.8, 1.6]]), rtol=1e-15, atol=0), O1


def pin_single_token(orc, seed=3):
    """N = 1: O_n = V_0 * s / (s + eps) with s = phi(Q_n) . phi(K_0)."""
    Q, K, V = _rng_inputs(seed, B=2, N=1, H=3, d=8)
    Qm, _, _ = _rng_inputs(seed + 1, B=2, N=7, H=3, d=8)
    eps = 0.25
    O = orc.apply(Qm, orc.state(K, V), eps)
    s = np.einsum("bnhi,bhi->bnh", np.maximum(Qm, 0), np.maximum(K[:, 0], 0))
    want = V[:, 0][:, None, :, :] * (s / (s + eps))[..., None]
    assert np.allclose(O, want, rtol=1e-13, atol=1e-300), np.abs(O - want).max()


def pin_equal_keys(orc, seed=4):
    """All keys equal to one positive vector c: every query with phi(Q) != 0
    weights all tokens equally, so O_n = mean_m V_m (up to eps / den)."""
    Q, _, V = _rng_inputs(seed, B=2, N=40, H=2, d=8)
    c = np.abs(np.random.default_rng(seed + 9).standard_normal((2, 1, 2, 8))) + 0.5
    K = np.broadcast_to(c, Q.shape).copy()
    O, den = orc.forward(Q, K, V, 1e-15, return_den=True)
    mean = V.mean(axis=1, keepdims=True)
    live = den > 0
    err = np.abs(O - mean)[live]
    assert err.max() <= 1e-12 * max(1.0, np.abs(mean).max()), err.max()


def pin_one_hot(orc):
    """phi(Q_n) = e_{i_n} and one-hot keys K_m = e_{m mod d}: w_nm = [m mod d ==
    i_n], so O_n is the mean of the V rows whose key is hot at i_n."""
    B, N, H, d = 1, 23, 2, 4
    rng = np.random.default_rng(5)
    V = rng.standard_normal((B, N, H, d))
    K = np.full((B, N, H, d), -1.0)
    for m in range(N):
        K[0, m, :, m % d] = 2.0
    Q = np.full((B, N, H, d), -0.5)
    hot = rng.integers(0, d, size=N)
    for n in range(N):
        Q[0, n, :, hot[n]] = 1.5
    O = orc.forward(Q, K, V, 0.0)
    for n in range(N):
        sel = [m for m in range(N) if m % d == hot[n]]
        want = V[0, sel].mean(axis=0)
        assert np.allclose(O[0, n], want, rtol=1e-13, atol=1e-15), (n, O[0, n], want)


def pin_constant_column(orc, seed=6):
    """A constant V column c comes back as c * den / (den + eps): exactly c up to
    eps / den on rows with den > 0, and 0 on rows with den = 0."""
    Q, K, V = _rng_inputs(seed, B=2, N=50, H=3, d=8)
    Q[1, 3, 2, :] = -1.0  # a zero-weight row
    V[..., 5] = 0.375
    O, den = orc.forward(Q, K, V, 1e-15, return_den=True)
    live = den > 0
    assert np.allclose(O[..., 5][live], 0.375, rtol=1e-13, atol=0)
    assert np.all(O[..., 5][~live] == 0.0)


def pin_key_permutation(orc, seed=7):
    """Permuting the token order of (K, V) jointly leaves O unchanged."""
    Q, K, V = _rng_inputs(seed, B=2, N=41, H=3, d=8)
    perm = np.random.default_rng(seed).permutation(41)
    O1 = orc.forward(Q, K, V, 1e-15)
    O2 = orc.forward(Q, K[:, perm], V[:, perm], 1e-15)
    assert row_relerr(O2, O1).max() <= 1e-13


def pin_query_permutation_and_independence(orc, seed=8):
    """Permuting queries permutes output rows bit for bit; changing another
    (b, h) slice, or K/V of another head, leaves a head's output unchanged."""
    Q, K, V = _rng_inputs(seed, B=2, N=29, H=3, d=8)
    O = orc.forward(Q, K, V, 1e-15)
    perm = np.random.default_rng(seed).permutation(29)
    Op = orc.forward(Q[:, perm], K, V, 1e-15)
    assert np.array_equal(Op, O[:, perm])
    Q2, K2, V2 = Q.copy(), K.copy(), V.copy()
    Q2[:, :, 1] += 3.0
    K2[:, :, 1] *= -2.0
    V2[1] = 7.0
    O2 = orc.forward(Q2, K2, V2, 1e-15)
    assert np.array_equal(O2[0][:, [0, 2]], O[0][:, [0, 2]])


def pin_convex_hull(orc, seed=9):
    """Weights phi(Q_n).phi(K_m) >= 0, so each O_{n,i} is den/(den+eps) times a
    convex combination of column i of V: it stays in the hull of V[:, i] and 0."""
    Q, K, V = _rng_inputs(seed, B=2, N=64, H=3, d=8)
    O = orc.forward(Q, K, V, 1e-15)
    lo = np.minimum(V.min(axis=1, keepdims=True), 0.0)
    hi = np.maximum(V.max(axis=1, keepdims=True), 0.0)
    tol = 1e-12
    assert np.all(O >= lo - tol) and np.all(O <= hi + tol)


def pin_zero_query(orc, seed=10):
    """A query with phi(Q) = 0 gives num = den = 0 and O = 0 / eps = 0 exactly."""
    Q, K, V = _rng_inputs(seed, B=1, N=16, H=2, d=8)
    Q[..., 0] = np.abs(Q[..., 0]) + 0.1   # every other row keeps a live feature
    K[..., 0] = np.abs(K[..., 0]) + 0.1
    Q[0, [2, 9], :, :] = -np.abs(Q[0, [2, 9], :, :]) - 0.1
    O = orc.forward(Q, K, V, 1e-15)
    assert np.all(O[0, [2, 9]] == 0.0)
    assert np.all(np.linalg.norm(np.delete(O[0], [2, 9], axis=0), axis=-1) > 0)


def pin_scale_invariance(orc, seed=12):
    """With eps = 0, scaling Q or K by a power of two changes nothing, bit for bit
    (every product scales exactly and the ratio cancels)."""
    Q, K, V = _rng_inputs(seed, B=2, N=30, H=2, d=8)
    Q = np.abs(Q) + 0.01  # no zero rows, so no 0/0 with eps = 0
    O = orc.forward(Q, K, V, 0.0)
    assert np.array_equal(orc.forward(4.0 * Q, 0.5 * K, V, 0.0), O)


def pin_linearity_in_v(orc, seed=13):
    """O is linear in V: O(aV + bV') = a O(V) + b O(V')."""
    Q, K, V = _rng_inputs(seed, B=2, N=30, H=2, d=8)
    _, _, V2 = _rng_inputs(seed + 1, B=2, N=30, H=2, d=8)
    a, b = -1.5, 0.75
    lhs = orc.forward(Q, K, a * V + b * V2, 1e-15)
    rhs = a * orc.forward(Q, K, V, 1e-15) + b * orc.forward(Q, K, V2, 1e-15)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-13)


def pin_state_definition(orc, seed=14):
    """The state alone: column d is the per-feature sum of phi(K); the d x d
    block is phi(K)^T V, checked by an explicit outer-product sum per token."""
    Q, K, V = _rng_inputs(seed, B=2, N=17, H=3, d=5)
    S = orc.state(K, V)
    for b in range(2):
        for h in range(3):
            acc = np.zeros((5, 6))
            for n in range(17):
                k = np.maximum(K[b, n, h], 0.0)
                acc += np.outer(k, np.append(V[b, n, h], 1.0))
            assert np.allclose(S[b, h], acc, rtol=1e-13, atol=1e-13)


def tiny_inputs():
    """The 16x16-latent oracle check: B=1, N=256, H=4, d=32 from seed 0 (fp32)."""
    import torch  # noqa: F401  (the generator lives in the product package)
    from linear_attention_diffusion_relu_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS["tiny"]
    (_, src) = make_inputs(w, keep_source=True)
    return tuple(t.double().numpy() for t in src), w.eps


def pin_bruteforce_tiny(orc):
    (Q, K, V), eps = tiny_inputs()
    pin_bruteforce(orc, Q, K, V, eps)


def pin_bruteforce_random(orc, seed=15):
    Q, K, V = _rng_inputs(seed, B=2, N=37, H=3, d=6)
    pin_bruteforce(orc, Q, K, V, 1e-15)


# ------------------------------------------------------------ block-causal --
# "linear-diffusion-transformer-4k-efficient-generation", section
# "技术演进：从图像到视频与世界模型" (SANA-Video: block causal linear attention).
# Reading: blocks of L consecutive tokens; a query of block j sees the keys of
# blocks 0 .. j.

def bruteforce_block_causal(Q, K, V, L, eps):
    """The quadratic definition with a block mask: W[n, m] = phi(Q_n).phi(K_m)
    where m // L <= n // L, else 0; O = (W V) / (W 1 + eps)."""
    Q, K, V = (np.asarray(x, dtype=np.float64) for x in (Q, K, V))
    B, N, H, d = Q.shape
    blk = np.arange(N) // L
    mask = (blk[None, :] <= blk[:, None]).astype(np.float64)
    O = np.empty_like(Q)
    for b in range(B):
        for h in range(H):
            W = (np.maximum(Q[b, :, h, :], 0.0) @ np.maximum(K[b, :, h, :], 0.0).T) * mask
            O[b, :, h, :] = (W @ V[b, :, h, :]) / (W.sum(axis=1, keepdims=True) + eps)
    return O


def pin_block_causal_bruteforce(orc, seed=21):
    """Oracle == masked n x n form for several block lengths, including L = 1
    (token-causal), a ragged last block, and L >= N (no mask)."""
    Q, K, V = _rng_inputs(seed, B=2, N=37, H=3, d=8)
    Q[1, 12, 1, :] = -np.abs(Q[1, 12, 1, :]) - 0.1   # a zero-weight row
    for L in (1, 4, 10, 37, 64):
        O = orc.block_causal_forward(Q, K, V, L, 1e-15)
        R = bruteforce_block_causal(Q, K, V, L, 1e-15)
        err = row_relerr(O, R)
        assert err.max() <= 1e-12, (L, err.max())
        zero = np.linalg.norm(R, axis=-1) == 0
        assert np.all(O[zero] == 0.0)


def pin_block_causal_exact_integers(orc, seed=22):
    """Small integers, eps = 1/4, L = 2: equal to the correctly rounded exact
    rational value of the masked definition, block by block."""
    rng = np.random.default_rng(seed)
    B, N, H, d, L = 1, 5, 2, 3, 2
    Q, K, V = (rng.integers(-3, 4, size=(B, N, H, d)).astype(np.float64) for _ in range(3))
    O = orc.block_causal_forward(Q, K, V, L, 0.25)
    for n in range(N):
        end = (n // L + 1) * L
        want = exact_rational(Q[:, n:n + 1], K[:, :end], V[:, :end], Fraction(1, 4))
        assert np.array_equal(O[:, n:n + 1], np.vectorize(float)(want).astype(np.float64)), n


def pin_block_causal_reductions(orc, seed=23):
    """L >= N is the plain forward, bit for bit; the last prefix state is the
    full state; block 0 alone is the plain forward over block 0's tokens."""
    Q, K, V = _rng_inputs(seed, B=2, N=30, H=2, d=8)
    assert np.array_equal(orc.block_causal_forward(Q, K, V, 30, 1e-15), orc.forward(Q, K, V, 1e-15))
    P = orc.block_causal_state(K, V, 7)
    assert P.shape == (2, 2, 5, 8, 9)
    assert np.array_equal(P[:, :, -1], orc.state(K, V))
    assert np.array_equal(P[:, :, 0], orc.state(K[:, :7], V[:, :7]))
    O = orc.block_causal_forward(Q, K, V, 7, 1e-15)
    assert np.array_equal(O[:, :7], orc.forward(Q[:, :7], K[:, :7], V[:, :7], 1e-15))


def pin_block_causal_no_future(orc, seed=24):
    """Keys and values of later blocks never reach earlier blocks' outputs (bit
    for bit); those of the query's own block do."""
    Q, K, V = _rng_inputs(seed, B=1, N=40, H=2, d=8)
    L = 8
    O = orc.block_causal_forward(Q, K, V, L, 1e-15)
    K2, V2 = K.copy(), V.copy()
    K2[:, 24:] = 5.0 * np.abs(K2[:, 24:])
    V2[:, 24:] += 3.0
    O2 = orc.block_causal_forward(Q, K2, V2, L, 1e-15)
    assert np.array_equal(O2[:, :24], O[:, :24])
    assert np.all(np.abs(O2[:, 24:] - O[:, 24:]).max(axis=-1) > 0)
    K3 = K.copy()
    K3[:, 23] = 4.0 * np.abs(K3[:, 23])      # last token of block 2
    O3 = orc.block_causal_forward(Q, K3, V, L, 1e-15)
    assert np.array_equal(O3[:, :16], O[:, :16])
    assert np.all(np.abs(O3[:, 16:24] - O[:, 16:24]).max(axis=-1) > 0)


# ------------------------------------------------------------ feature maps --
# "08_sana高效高分辨率生成", section "Linear Attention 的原理": ELU+1 and cos are
# named as alternatives to ReLU. Reading: ELU with alpha = 1, plus one.

FEATURES_NP = {
    "relu": lambda x: np.maximum(x, 0.0),
    "elu1": lambda x: np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0))),
    "cos": np.cos,
}


def bruteforce_fm(Q, K, V, eps, feature):
    """The quadratic definition with feature map phi, in numpy."""
    Q, K, V = (np.asarray(x, dtype=np.float64) for x in (Q, K, V))
    phi = FEATURES_NP[feature]
    B, N, H, d = Q.shape
    O = np.empty_like(Q)
    for b in range(B):
        for h in range(H):
            W = phi(Q[b, :, h, :]) @ phi(K[b, :, h, :]).T
            O[b, :, h, :] = (W @ V[b, :, h, :]) / (W.sum(axis=1, keepdims=True) + eps)
    return O


def pin_feature_maps_bruteforce(orc, seed=31):
    """Each feature map against its n x n definition (1e-12 normwise per row;
    cos normalisers of random inputs stay far from zero here); ReLU through the
    feature-map entry equals the plain oracle bit for bit."""
    Q, K, V = _rng_inputs(seed, B=2, N=37, H=3, d=8)
    for feature in ("relu", "elu1", "cos"):
        O, den = orc.forward_fm(Q, K, V, feature, 1e-15, return_den=True)
        R = bruteforce_fm(Q, K, V, 1e-15, feature)
        assert row_relerr(O, R).max() <= 1e-12, (feature, row_relerr(O, R).max())
        if feature == "cos":
            assert np.abs(den).min() > 1.0
    assert np.array_equal(orc.forward_fm(Q, K, V, "relu", 1e-15), orc.forward(Q, K, V, 1e-15))


def pin_feature_maps_closed_forms(orc, seed=32):
    """Q = K = 0 gives phi = 1 for ELU+1 and cos, every weight equals d, so
    O = d * sum_m V_m / (N d + eps): the mean of V up to eps. ELU+1 at hand
    points: phi(1) = 2, phi(0) = 1, phi(-ln 2) = 1/2 (one head, d = 1)."""
    _, _, V = _rng_inputs(seed, B=1, N=20, H=2, d=4)
    Z = np.zeros_like(V)
    for feature in ("elu1", "cos"):
        O = orc.forward_fm(Z, Z, V, feature, 0.0)
        assert np.allclose(O, np.broadcast_to(V.mean(axis=1, keepdims=True), O.shape), rtol=1e-14, atol=1e-15)
    Q = np.array([1.0]).reshape(1, 1, 1, 1)
    K = np.array([1.0, 0.0, -np.log(2.0)]).reshape(1, 3, 1, 1)
    V = np.array([3.0, 5.0, 7.0]).reshape(1, 3, 1, 1)
    # phi(Q) = 2, phi(K) = [2, 1, 1/2]: weights [4, 2, 1] -> (12 + 10 + 7) / 7
    O = orc.forward_fm(Q, K, V, "elu1", 0.0)
    assert np.allclose(O.ravel(), [29.0 / 7.0], rtol=1e-15), O


def pin_feature_maps_symmetries(orc, seed=33):
    """cos is even: negating Q and K changes nothing, bit for bit. ELU+1 keeps
    every weight positive, so outputs stay in the hull of V (plus 0)."""
    Q, K, V = _rng_inputs(seed, B=1, N=30, H=2, d=8)
    assert np.array_equal(orc.forward_fm(-Q, -K, V, "cos", 1e-15), orc.forward_fm(Q, K, V, "cos", 1e-15))
    O = orc.forward_fm(Q, K, V, "elu1", 1e-15)
    lo = np.minimum(V.min(axis=1, keepdims=True), 0.0)
    hi = np.maximum(V.max(axis=1, keepdims=True), 0.0)
    assert np.all(O >= lo - 1e-12) and np.all(O <= hi + 1e-12)
    S = orc.state_fm(K, V, "elu1")
    assert np.allclose(S[..., -1], np.where(K > 0, K + 1, np.exp(np.minimum(K, 0))).sum(axis=1), rtol=1e-13)


# ------------------------------------------------- projection-fused state --
# Section 4 "On-Device Deployment" of the SANA walk-through: ReLU(K)^T V fused
# into the QKV projection.

def pin_round_bf16(orc):
    """The oracle's bf16 rounding equals torch's float32 -> bfloat16 cast
    (round to nearest even) on float32 values, including exact ties and values
    that carry into the next binade."""
    import torch
    rng = np.random.default_rng(41)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(3.0)
    ties = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 255.5 / 128.0, -(1.0 + 2.0 ** -8),
                     1.0 - 2.0 ** -10, 0.0, -0.0], dtype=np.float32)
    x = np.concatenate([x, ties])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = orc.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def pin_projected_state_integers(orc, seed=42):
    """Small-integer X and weights: the projections are exact integers; with
    |values| < 256 they are exact in bf16 too, so the projected state equals the
    state of the explicitly computed integer K and V (triple loop), bit for bit."""
    rng = np.random.default_rng(seed)
    B, N, H, d, C = 2, 9, 3, 4, 5
    X = rng.integers(-3, 4, size=(B, N, C)).astype(np.float64)
    Wk = rng.integers(-3, 4, size=(H * d, C)).astype(np.float64)
    Wv = rng.integers(-3, 4, size=(H * d, C)).astype(np.float64)
    K = np.zeros((B, N, H * d))
    V = np.zeros((B, N, H * d))
    for b in range(B):
        for n in range(N):
            for o in range(H * d):
                K[b, n, o] = sum(X[b, n, c] * Wk[o, c] for c in range(C))
                V[b, n, o] = sum(X[b, n, c] * Wv[o, c] for c in range(C))
    S = orc.projected_state(X, Wk, Wv, H)
    assert np.array_equal(S, orc.state(K.reshape(B, N, H, d), V.reshape(B, N, H, d)))
    # the rounding step is applied: a projection that is not a bf16 value
    X2 = np.ones((1, 1, 1))
    W2 = np.full((1, 1), 1.0 + 2.0 ** -9)      # 1 + 2^-9 rounds to 1 (tie to even)
    K2, _ = orc.project_kv(X2, W2, W2, 1)
    assert K2.ravel()[0] == 1.0


# ---------------------------------------------------------------- Mix-FFN --
# SANA walk-through, section 2.2: inverted residual + 3x3 depthwise conv + GLU.

def pin_depthwise_loops(orc, seed=51):
    """The depthwise 3x3 conv against explicit loops over taps with bounds
    checks, on a small non-square grid."""
    rng = np.random.default_rng(seed)
    B, Hg, W, Cc = 2, 3, 5, 4
    U = rng.standard_normal((B, Hg * W, Cc))
    Kd = rng.standard_normal((Cc, 3, 3))
    D = orc.depthwise3x3(U, Kd, (Hg, W))
    for b in range(B):
        for y in range(Hg):
            for x in range(W):
                for c in range(Cc):
                    acc = 0.0
                    for dy in range(3):
                        for dx in range(3):
                            yy, xx = y + dy - 1, x + dx - 1
                            if 0 <= yy < Hg and 0 <= xx < W:
                                acc += U[b, yy * W + xx, c] * Kd[c, dy, dx]
                    assert abs(D[b, y * W + x, c] - acc) <= 1e-12 * (1 + abs(acc))


def pin_depthwise_shift_and_identity(orc, seed=52):
    """A centre-only kernel returns U; a kernel with only the (dy, dx) = (0, 2)
    tap shifts the grid by (+1 row, -1 column) with zeros entering at the edges."""
    rng = np.random.default_rng(seed)
    B, Hg, W, Cc = 1, 4, 3, 2
    U = rng.standard_normal((B, Hg * W, Cc))
    ident = np.zeros((Cc, 3, 3)); ident[:, 1, 1] = 1.0
    assert np.array_equal(orc.depthwise3x3(U, ident, (Hg, W)), U)
    shift = np.zeros((Cc, 3, 3)); shift[:, 0, 2] = 1.0
    D = orc.depthwise3x3(U, shift, (Hg, W)).reshape(Hg, W, Cc)
    G = U.reshape(Hg, W, Cc)
    for y in range(Hg):
        for x in range(W):
            want = G[y - 1, x + 1] if (y >= 1 and x + 1 < W) else np.zeros(Cc)
            assert np.array_equal(D[y, x], want)


def pin_mix_ffn_gate(orc):
    """With identity-like weights and a centre-only kernel, the block reduces to
    the GLU: Y = bf16(a * sigmoid(g)) for the channel halves a, g of X. Small
    integer a and g: g = 0 halves a exactly; g = 40 passes a (sigmoid rounds to 1)."""
    C = Ch = 2
    X = np.array([[[3.0, -5.0], [7.0, 1.0], [2.0, 4.0]]])        # B=1, N=3 tokens, C=2
    W1 = np.zeros((2 * Ch, C)); W1[0, 0] = W1[1, 1] = 1.0          # a = X, g = 0
    ident = np.zeros((2 * Ch, 3, 3)); ident[:, 1, 1] = 1.0
    W2 = np.eye(C)
    Y = orc.mix_ffn(X, W1, ident, W2, (1, 3))
    assert np.array_equal(Y, X / 2.0)
    Xg = np.concatenate([X, np.full((1, 3, C), 40.0)], axis=-1)     # C_in = 4: a = X, g = 40
    W1c = np.zeros((2 * Ch, 4)); W1c[0, 0] = W1c[1, 1] = 1.0; W1c[2, 2] = W1c[3, 3] = 1.0
    Y2 = orc.mix_ffn(Xg, W1c, ident, W2, (1, 3))
    assert np.array_equal(Y2, X)


def pin_mix_ffn_bruteforce(orc, seed=53):
    """The whole block against explicit per-token loops (expand, 3x3 taps,
    sigmoid gate, project) with the same two bf16 roundings."""
    rng = np.random.default_rng(seed)
    B, Hg, W, C, Ch = 1, 3, 4, 5, 3
    X = rng.standard_normal((B, Hg * W, C))
    W1 = rng.standard_normal((2 * Ch, C)) / np.sqrt(C)
    Kd = rng.standard_normal((2 * Ch, 3, 3)) / 3.0
    W2 = rng.standard_normal((C, Ch)) / np.sqrt(Ch)
    Y = orc.mix_ffn(X, W1, Kd, W2, (Hg, W))
    rb = orc.round_bf16
    U = np.zeros((B, Hg * W, 2 * Ch))
    for n in range(Hg * W):
        for o in range(2 * Ch):
            U[0, n, o] = rb(sum(X[0, n, c] * W1[o, c] for c in range(C)))
    for n in range(Hg * W):
        y, x = divmod(n, W)
        z = []
        for c in range(Ch):
            da = dg = 0.0
            for dy in range(3):
                for dx in range(3):
                    yy, xx = y + dy - 1, x + dx - 1
                    if 0 <= yy < Hg and 0 <= xx < W:
                        da += U[0, yy * W + xx, c] * Kd[c, dy, dx]
                        dg += U[0, yy * W + xx, Ch + c] * Kd[Ch + c, dy, dx]
            z.append(rb(da * (1.0 / (1.0 + np.exp(-dg)))))
        for o in range(C):
            want = sum(z[c] * W2[o, c] for c in range(Ch))
            assert abs(Y[0, n, o] - want) <= 1e-12 * (1 + abs(want)), (n, o)


ALL_PINS = [
    pin_bruteforce_tiny, pin_bruteforce_random, pin_exact_integers, pin_hand_example,
    pin_single_token, pin_equal_keys, pin_one_hot, pin_constant_column,
    pin_key_permutation, pin_query_permutation_and_independence, pin_convex_hull,
    pin_zero_query, pin_scale_invariance, pin_linearity_in_v, pin_state_definition,
    pin_block_causal_bruteforce, pin_block_causal_exact_integers, pin_block_causal_reductions,
    pin_block_causal_no_future, pin_feature_maps_bruteforce, pin_feature_maps_closed_forms,
    pin_feature_maps_symmetries, pin_round_bf16, pin_projected_state_integers,
    pin_depthwise_loops, pin_depthwise_shift_and_identity, pin_mix_ffn_gate, pin_mix_ffn_bruteforce,
]
