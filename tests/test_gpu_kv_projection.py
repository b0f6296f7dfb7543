"""Parity of the key-value projection with the state in its epilogue (the
ReLU(K)^T V product fused into the QKV projection: SANA walk-through, section 4
"On-Device Deployment") with the oracle, through the C ABI.

The oracle projects in fp64 and rounds K and V to bf16; the kernel accumulates
the projection in fp32 before the same rounding, so a small fraction f (~1e-4
to 1e-3, growing with C; measured below) of K and V elements land one bf16
step (at most 2^-7 relative) apart ("flips"). A state entry sum_n t_n,
t_n = phi(K_ni) [V | 1]_nj, is therefore held to 1e-4 of sum_n |t_n| plus four
such steps of its largest term (an O(1) error from a wrong layout, head, token
or feature fails by orders of magnitude).

End to end the flips do not cancel the way the state's own terms do: a
numerator entry sum_n t_n over zero-mean V is a random walk of size
sqrt(N) rms(t), and the flips add sqrt(f N) 2^-8 rms(t) to it, so the output
rows move by about sqrt(f) 2^-8 of their norm (~1e-4 at f = 1e-3), which is as
large as the forward's own 1e-4 bar. So the end-to-end check has two parts:
apply() on the GPU's state is held to the forward's tolerance against the
oracle's apply of that same state, and the output against the oracle's
end-to-end forward is held to that tolerance plus the first-order propagation
of the state's measured deviation, |dO_i| <= (phi(Q) |dS[:, i]| +
|O_i| phi(Q) |dS[:, d]|) / (den + eps), whose entries the state check bounds."""
import numpy as np
import pytest
import torch

from linear_attention_diffusion_relu_b200 import ops
from tests.parity import check_output, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_diffusion_relu_b200 import build
    build.build()
    ops.load_library()


def _inputs(B, N, C, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn((B, N, C), generator=g).to(torch.bfloat16)
    # weights scaled like a trained linear layer (unit-variance outputs)
    Wk = (torch.randn((H * d, C), generator=g) / C ** 0.5).to(torch.bfloat16)
    Wv = (torch.randn((H * d, C), generator=g) / C ** 0.5).to(torch.bfloat16)
    return X.cuda(), Wk.cuda(), Wv.cuda()


def _max_term(K, V):
    """max_n |phi(K_ni)| |[V | 1]_nj| per state entry (B, H, d, d+1)."""
    B, N, H, d = K.shape
    out = np.zeros((B, H, d, d + 1))
    pk = np.maximum(K, 0.0)
    v1 = np.concatenate([np.abs(V), np.ones((B, N, H, 1))], axis=-1)
    for b in range(B):
        for h in range(H):
            for n0 in range(0, N, 512):
                t = pk[b, n0:n0 + 512, h, :, None] * v1[b, n0:n0 + 512, h, None, :]
                out[b, h] = np.maximum(out[b, h], t.max(axis=0))
    return out


def _bound(K, V, mag):
    return 1e-4 * mag + 4 * 2.0 ** -7 * _max_term(K, V) + 1e-30


def _check_state(oracle, S, X, Wk, Wv, H):
    K, V = oracle.project_kv(to_f64(X), to_f64(Wk), to_f64(Wv), H)
    ref = oracle.state(K, V)
    mag = oracle.state(K, np.abs(V))
    err = np.abs(to_f64(S) - ref)
    bound = _bound(K, V, mag)
    assert np.all(err <= bound), (err / bound).max()
    return K, V


SHAPES = [(1, 1, 64, 1, 32), (2, 300, 136, 6, 32), (1, 1000, 1152, 36, 32), (2, 513, 256, 4, 64),
          (20, 200, 128, 40, 32),      # 200 slabs: several per CTA
          (2, 4096, 2240, 70, 32)]     # the 2048px Sana-1.6B shape (C = 2240)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}N{}C{}H{}d{}".format(*s))
def test_projected_state_matches_oracle(oracle, shape):
    B, N, C, H, d = shape
    X, Wk, Wv = _inputs(B, N, C, H, d, seed=N + C)
    S = ops.kv_projection_state(X, Wk, Wv, H)
    torch.cuda.synchronize()
    _check_state(oracle, S, X, Wk, Wv, H)
    assert ops.device_error() == 0


def test_projected_state_end_to_end_and_deterministic(oracle):
    """apply() on the fused state meets the forward's tolerance against the
    oracle's apply of the same state; against the oracle's whole forward of the
    projected K and V it meets that tolerance plus the propagated state
    deviation; repeated calls give the same bits."""
    B, N, C, H, d = 2, 777, 512, 8, 32
    eps = 1e-15
    X, Wk, Wv = _inputs(B, N, C, H, d, seed=5)
    Q = torch.randn((B, N, H, d), generator=torch.Generator().manual_seed(6)).to(torch.bfloat16).cuda()
    S1 = ops.kv_projection_state(X, Wk, Wv, H)
    S2 = ops.kv_projection_state(X, Wk, Wv, H)
    O32 = ops.apply(Q, S1, out_dtype=torch.float32)
    O16 = ops.apply(Q, S1, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(S1.view(torch.int32), S2.view(torch.int32))
    Qd, Sd = to_f64(Q), to_f64(S1)
    _check_state(oracle, S1, X, Wk, Wv, H)
    # the apply on the GPU's own state: the forward's tolerance
    same = oracle.apply(Qd, Sd, eps)
    check_output(O32, same, "apply on the projected state (fp32 out)")
    check_output(O16, same, "apply on the projected state (bf16 out)")
    # end to end: that tolerance plus the state's deviation carried through the apply
    K, V = oracle.project_kv(to_f64(X), to_f64(Wk), to_f64(Wv), H)
    S_ref = oracle.state(K, V)
    ref, den = oracle.apply(Qd, S_ref, eps, return_den=True)
    dS = np.abs(Sd - S_ref)
    phiQ = np.maximum(Qd, 0.0)
    d_num = np.einsum("bnhk,bhki->bnhi", phiQ, dS[..., :d])
    d_den = np.einsum("bnhk,bhk->bnh", phiQ, dS[..., d])
    prop = (d_num + np.abs(ref) * d_den[..., None]) / (den + eps)[..., None]
    got = to_f64(O32)
    err = np.linalg.norm(got - ref, axis=-1)
    bound = 1e-4 * np.linalg.norm(ref, axis=-1) + 1.01 * np.linalg.norm(prop, axis=-1) + 1e-30
    assert np.all(err <= bound), (err / bound).max()


def test_flip_fraction_of_fp32_projection(oracle):
    """The mechanism behind the bounds above, measured: K from an fp32
    accumulation (cuBLAS bf16 matmul) against the oracle's fp64 projection,
    both rounded to bf16, differ in a small fraction of elements, each by one
    bf16 step of the value or, where the dot product cancels to near zero, by
    the fp32 accumulation error C 2^-24 sum |x w| carrying the rounding across
    a step (the bound of the Mix-FFN expand check)."""
    B, N, C, H, d = 2, 2048, 2240, 70, 32
    X, Wk, Wv = _inputs(B, N, C, H, d, seed=11)
    K = (X @ Wk.T).view(B, N, H, d)
    torch.cuda.synchronize()
    Xd, Wd = to_f64(X), to_f64(Wk)
    Kr, _ = oracle.project_kv(Xd, Wd, Wd, H)
    Kg = to_f64(K)
    diff = Kg != Kr
    f = float(diff.mean())
    assert f < 1e-2, f
    mag = (np.abs(Xd) @ np.abs(Wd).T).reshape(B, N, H, d)
    bound = 2.0 ** -7 * np.abs(Kr) + C * 2.0 ** -23 * mag
    assert np.all(np.abs(Kg - Kr) <= bound), (np.abs(Kg - Kr) / bound).max()


def test_projected_state_agrees_with_unfused_path():
    """Against the unfused pipeline on the GPU: K and V from a cuBLAS bf16
    matmul (stored), then kv_state. Both round fp32 sums to bf16, so they agree
    to the same 1e-4 bound."""
    B, N, C, H, d = 2, 2048, 1152, 36, 32
    X, Wk, Wv = _inputs(B, N, C, H, d, seed=7)
    S = ops.kv_projection_state(X, Wk, Wv, H)
    K = (X @ Wk.T).view(B, N, H, d).contiguous()
    V = (X @ Wv.T).view(B, N, H, d).contiguous()
    S_ref = ops.kv_state(K, V)
    mag = ops.kv_state(K, V.abs())
    torch.cuda.synchronize()
    err = to_f64(S - S_ref)
    bound = _bound(to_f64(K), to_f64(V), to_f64(mag))
    assert np.all(np.abs(err) <= bound), (np.abs(err) / bound).max()


def test_projected_state_4096px_every_head(oracle):
    """The bench's 4096px shape (B = 2, N = 16384, C = 2240, H = 70), in the
    launch configuration the bench times: every head's state against the
    oracle's projection and state of that head (ten heads at a time)."""
    B, N, C, H, d = 2, 16384, 2240, 70, 32
    X, Wk, Wv = _inputs(B, N, C, H, d, seed=N + C)
    S = ops.kv_projection_state(X, Wk, Wv, H)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    Xd = to_f64(X)
    Sd = to_f64(S)
    for h0 in range(0, H, 10):
        h1 = min(H, h0 + 10)
        rows = slice(h0 * d, h1 * d)
        K, V = oracle.project_kv(Xd, to_f64(Wk[rows]), to_f64(Wv[rows]), h1 - h0)
        ref = oracle.state(K, V)
        mag = oracle.state(K, np.abs(V))
        err = np.abs(Sd[:, h0:h1] - ref)
        bound = _bound(K, V, mag)
        assert np.all(err <= bound), (h0, (err / bound).max())
