"""Parity of the key-value projection with the state in its epilogue (the
ReLU(K)^T V product fused into the QKV projection: SANA walk-through, section 4
"On-Device Deployment") with the oracle, through the C ABI.

The oracle projects in fp64 and rounds K and V to bf16; the kernel accumulates
the projection in fp32 before the same rounding, so a small fraction (~1e-4 to
1e-3, growing with C) of K and V elements land one bf16 step (at most 2^-7
relative) apart. A state entry sum_n t_n, t_n = phi(K_ni) [V | 1]_nj, is
therefore held to 1e-4 of sum_n |t_n| plus four such steps of its largest term
(an O(1) error from a wrong layout, head, token or feature fails by orders of
magnitude). End to end, apply() on that state is held to 1e-3 per row (fp32)
and to the forward's bf16 output tolerance."""
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
    """apply() on the fused state meets the forward's output tolerance against
    the oracle forward of the projected K and V; repeated calls give the same bits."""
    B, N, C, H, d = 2, 777, 512, 8, 32
    X, Wk, Wv = _inputs(B, N, C, H, d, seed=5)
    Q = torch.randn((B, N, H, d), generator=torch.Generator().manual_seed(6)).to(torch.bfloat16).cuda()
    S1 = ops.kv_projection_state(X, Wk, Wv, H)
    S2 = ops.kv_projection_state(X, Wk, Wv, H)
    O32 = ops.apply(Q, S1, out_dtype=torch.float32)
    O16 = ops.apply(Q, S1, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(S1.view(torch.int32), S2.view(torch.int32))
    K, V = oracle.project_kv(to_f64(X), to_f64(Wk), to_f64(Wv), H)
    ref = oracle.forward(to_f64(Q), K, V, 1e-15)
    check_output(O16, ref, "projected state, end to end (bf16 out)")
    got = to_f64(O32)
    rel = np.linalg.norm(got - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)
    assert rel.max() <= 1e-3, rel.max()


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


def test_projected_state_4096px_sampled_heads(oracle):
    """The bench's 4096px shape (B = 2, N = 16384, C = 2240, H = 70), in the
    launch configuration the bench times: three heads' states (first, middle,
    last group) against the oracle's projection and state of those heads."""
    B, N, C, H, d = 2, 16384, 2240, 70, 32
    X, Wk, Wv = _inputs(B, N, C, H, d, seed=N + C)
    S = ops.kv_projection_state(X, Wk, Wv, H)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    Xd = to_f64(X)
    for h in (0, 37, H - 1):
        rows = slice(h * d, (h + 1) * d)
        K, V = oracle.project_kv(Xd, to_f64(Wk[rows]), to_f64(Wv[rows]), 1)
        ref = oracle.state(K, V)[:, 0]
        mag = oracle.state(K, np.abs(V))[:, 0]
        err = np.abs(to_f64(S[:, h]) - ref)
        bound = _bound(K, V, mag[:, None])[:, 0]
        assert np.all(err <= bound), (h, (err / bound).max())
