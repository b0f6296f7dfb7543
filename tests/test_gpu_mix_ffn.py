"""Parity of the Mix-FFN (1x1 expand, 3x3 depthwise conv + GLU fused, 1x1
project; SANA walk-through section 2.2) with the oracle, through the C ABI.

The workspace keeps the two bf16 intermediates (U after the expand, Z after
the depthwise conv and the GLU), so each stage is checked against the oracle
applied to the GPU's own input of that stage: the GEMMs accumulate in fp32
and the oracle in fp64 before the same bf16 rounding, so an element may land
one bf16 step (2^-7 relative) apart, or, where the sum cancels, differ by the
fp32 accumulation error; the project's output is held to one bf16 rounding plus
an fp32 accumulation bound. End to end, rows of Y are held to 2e-2
of their norm (the two intermediate roundings compound)."""
import numpy as np
import pytest
import torch

from linear_attention_diffusion_relu_b200 import ops
from tests.parity import to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_diffusion_relu_b200 import build
    build.build()
    ops.load_library()


def _inputs(B, Hg, Wg, C, Ch, seed):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn((B, Hg * Wg, C), generator=g).to(torch.bfloat16)
    W1 = (torch.randn((2 * Ch, C), generator=g) / C ** 0.5).to(torch.bfloat16)
    Kdw = (torch.randn((2 * Ch, 3, 3), generator=g) / 3.0).float()
    W2 = (torch.randn((C, Ch), generator=g) / Ch ** 0.5).to(torch.bfloat16)
    return X.cuda(), W1.cuda(), Kdw.cuda(), W2.cuda()


def _intermediates(ws, B, N, Ch):
    nU = B * N * 2 * Ch * 2
    offZ = (nU + 255) // 256 * 256
    U = ws[:nU].view(torch.bfloat16).view(B, N, 2 * Ch)
    Z = ws[offZ:offZ + B * N * Ch * 2].view(torch.bfloat16).view(B, N, Ch)
    return U, Z


# (1, 9, 70, 128, 104): a last channel group of 40, a 6-column and a 1-row tile
SHAPES = [(1, 4, 4, 64, 32), (2, 16, 24, 256, 320), (1, 32, 32, 1152, 2880), (2, 7, 5, 136, 24),
          (1, 9, 70, 128, 104)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}G{}x{}C{}Ch{}".format(*s))
def test_mix_ffn_stages_match_oracle(oracle, shape):
    B, Hg, Wg, C, Ch = shape
    N = Hg * Wg
    X, W1, Kdw, W2 = _inputs(B, Hg, Wg, C, Ch, seed=N + C)
    ws = torch.empty(ops.mix_ffn_workspace_bytes(B, Hg, Wg, C, Ch), dtype=torch.uint8, device="cuda")
    Y = ops.mix_ffn(X, W1, Kdw, W2, (Hg, Wg), workspace=ws)
    torch.cuda.synchronize()
    U, Z = (to_f64(t) for t in _intermediates(ws, B, N, Ch))
    Xd, W1d, Kd, W2d = to_f64(X), to_f64(W1), to_f64(Kdw), to_f64(W2)
    # expand: one bf16 step at most, on few elements
    U_ref = oracle.round_bf16(Xd @ W1d.T)
    dU = np.abs(U - U_ref)
    # one bf16 step, or (for sums that cancel) the fp32 accumulation error
    # K * 2^-24 * sum |x w| carrying the rounding across a boundary
    boundU = 2.0 ** -7 * np.abs(U_ref) + C * 2.0 ** -23 * (np.abs(Xd) @ np.abs(W1d).T) + 1e-30
    assert np.all(dU <= boundU), (dU / boundU).max()
    assert np.mean(dU > 0) < 1e-2
    # depthwise + GLU on the GPU's own U
    D = oracle.depthwise3x3(U, Kd, (Hg, Wg))
    Z_ref = oracle.round_bf16(D[..., :Ch] / (1.0 + np.exp(-D[..., Ch:])))
    mag = oracle.depthwise3x3(np.abs(U), np.abs(Kd), (Hg, Wg))[..., :Ch]
    dZ = np.abs(Z - Z_ref)
    assert np.all(dZ <= 2.0 ** -7 * np.abs(Z_ref) + 1e-5 * mag + 1e-30)
    assert np.mean(dZ > 0) < 1e-2
    # project on the GPU's own Z: one bf16 rounding plus fp32 accumulation
    Y_ref = Z @ W2d.T
    bound = 2.0 ** -8 * np.abs(Y_ref) + Ch * 2.0 ** -23 * (np.abs(Z) @ np.abs(W2d).T) + 1e-30
    assert np.all(np.abs(to_f64(Y) - Y_ref) <= bound)
    # end to end
    Y_e2e = oracle.mix_ffn(Xd, W1d, Kd, W2d, (Hg, Wg))
    rel = np.linalg.norm(to_f64(Y) - Y_e2e, axis=-1) / np.maximum(np.linalg.norm(Y_e2e, axis=-1), 1e-30)
    assert rel.max() <= 2e-2, rel.max()
    assert ops.device_error() == 0


def test_mix_ffn_deterministic():
    B, Hg, Wg, C, Ch = 2, 16, 24, 256, 320
    X, W1, Kdw, W2 = _inputs(B, Hg, Wg, C, Ch, seed=3)
    Y1 = ops.mix_ffn(X, W1, Kdw, W2, (Hg, Wg))
    Y2 = ops.mix_ffn(X, W1, Kdw, W2, (Hg, Wg))
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def test_mix_ffn_4096px_sampled_tokens(oracle):
    """The bench's 4096px Mix-FFN (B = 2, 128 x 128 grid, C = 2240, Ch = 5600), in
    the launch configuration the bench times, stage by stage on eight tokens
    (corners, edges, interior): U on each token's 3 x 3 neighbourhood against the
    oracle's expand of those rows; Z from the oracle's depthwise conv of the
    GPU's own U cropped to the neighbourhood (at the grid's edge the crop's zero
    padding is the grid's); Y from the GPU's own Z row. Same bounds as above."""
    B, Hg, Wg, C, Ch = 2, 128, 128, 2240, 5600
    N = Hg * Wg
    X, W1, Kdw, W2 = _inputs(B, Hg, Wg, C, Ch, seed=4096)
    ws = torch.empty(ops.mix_ffn_workspace_bytes(B, Hg, Wg, C, Ch), dtype=torch.uint8, device="cuda")
    Y = ops.mix_ffn(X, W1, Kdw, W2, (Hg, Wg), workspace=ws)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    U, Z = _intermediates(ws, B, N, Ch)
    W1d, Kd, W2d = to_f64(W1), to_f64(Kdw), to_f64(W2)
    samples = [(0, 0, 0), (0, 0, Wg - 1), (0, Hg - 1, 0), (1, Hg - 1, Wg - 1),
               (0, 63, 64), (1, 5, 77), (1, 64, 0), (0, 100, Wg - 1)]
    changed_u = changed_z = total_u = total_z = 0
    for b, y, x in samples:
        ys = list(range(max(0, y - 1), min(Hg, y + 2)))
        xs = list(range(max(0, x - 1), min(Wg, x + 2)))
        rows = [yy * Wg + xx for yy in ys for xx in xs]
        # expand on the neighbourhood
        Xr = to_f64(X[b, rows])
        U_ref = oracle.round_bf16(Xr @ W1d.T)
        Ur = to_f64(U[b, rows])
        dU = np.abs(Ur - U_ref)
        boundU = 2.0 ** -7 * np.abs(U_ref) + C * 2.0 ** -23 * (np.abs(Xr) @ np.abs(W1d).T) + 1e-30
        assert np.all(dU <= boundU), ((b, y, x), (dU / boundU).max())
        changed_u += int(np.sum(dU > 0))
        total_u += dU.size
        # depthwise + GLU at the token, on the GPU's U
        crop = Ur.reshape(1, len(rows), 2 * Ch)
        ci = (y - ys[0]) * len(xs) + (x - xs[0])
        D = oracle.depthwise3x3(crop, Kd, (len(ys), len(xs)))[0, ci]
        Z_ref = oracle.round_bf16(D[:Ch] / (1.0 + np.exp(-D[Ch:])))
        mag = oracle.depthwise3x3(np.abs(crop), np.abs(Kd), (len(ys), len(xs)))[0, ci, :Ch]
        Zg = to_f64(Z[b, y * Wg + x])
        dZ = np.abs(Zg - Z_ref)
        assert np.all(dZ <= 2.0 ** -7 * np.abs(Z_ref) + 1e-5 * mag + 1e-30), (b, y, x)
        changed_z += int(np.sum(dZ > 0))
        total_z += dZ.size
        # project on the GPU's Z row
        Y_ref = Zg @ W2d.T
        bound = 2.0 ** -8 * np.abs(Y_ref) + Ch * 2.0 ** -23 * (np.abs(Zg) @ np.abs(W2d).T) + 1e-30
        assert np.all(np.abs(to_f64(Y[b, y * Wg + x]) - Y_ref) <= bound), (b, y, x)
    assert changed_u / total_u < 1e-2 and changed_z / total_z < 1e-2
