"""Parity of the Mix-FFN (1x1 expand, 3x3 depthwise conv + GLU fused, 1x1
project; SANA walk-through section 2.2 "선형 어텐션 블럭") with the oracle,
through the C ABI.

The workspace keeps the two bf16 intermediates (U after the expand, Z after
the depthwise conv and the GLU), so each stage is checked against the oracle's
own stage function (``expand``, ``depthwise_glu``, then ``Z W2^T``) applied to
the GPU's input of that stage: the GEMMs accumulate in fp32 and the oracle in
fp64 before the same bf16 rounding, so an element may land one bf16 step (2^-7
relative) apart, or, where the sum cancels, differ by the fp32 accumulation
error; the project's output is held to one bf16 rounding (2^-8 relative) plus
an fp32 accumulation bound.

End to end, against ``oracle.mix_ffn`` (whose U and Z are its own), a row of Y
differs by
  * the output's bf16 rounding: at most 2^-8 of each element, so at most 2^-8
    of the row norm;
  * the intermediates that rounded to a neighbouring bf16 value on one side
    only ("flips"): a fraction f of Z's elements differs from the oracle's Z,
    each by about one bf16 step (<= 2^-7 relative); at random positions with
    random signs, their share of a row of Y = Z W2^T is about sqrt(f) 2^-7 of
    its norm. The bound allows four times that, with f measured on the rows
    checked.
So rows of Y are held to 2^-8 + 4 sqrt(f) 2^-7 (+ 1e-5 for the fp32
accumulation) of their norm, with f asserted below 1e-2."""
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


def _check_grid_rows(oracle, X, W1, Kdw, W2, U, Z, Y, b, y0, y1, Hg, Wg):
    """Stage-by-stage and end-to-end checks of grid rows y0 .. y1-1 of batch b
    (every column). U is checked on those rows and one halo row either side;
    the depthwise conv runs on that crop, whose zero padding at the grid's
    edges is the grid's own. Returns (U elements changed, U checked, Z elements
    differing from the oracle's end-to-end Z, Z checked)."""
    C = X.shape[-1]
    Ch = W2.shape[-1]
    W1d, Kd, W2d = to_f64(W1), to_f64(Kdw), to_f64(W2)
    ya, yb = max(0, y0 - 1), min(Hg, y1 + 1)
    Xr = to_f64(X[b, ya * Wg:yb * Wg])
    Ur = to_f64(U[b, ya * Wg:yb * Wg])
    # expand: one bf16 step at most, or the fp32 accumulation error K 2^-24
    # sum |x w| carrying the rounding across a boundary where the sum cancels
    U_ref = oracle.expand(Xr, W1d)
    dU = np.abs(Ur - U_ref)
    boundU = 2.0 ** -7 * np.abs(U_ref) + C * 2.0 ** -23 * (np.abs(Xr) @ np.abs(W1d).T) + 1e-30
    assert np.all(dU <= boundU), ((b, y0), (dU / boundU).max())
    # depthwise + GLU on the GPU's own U
    rows = slice((y0 - ya) * Wg, (y1 - ya) * Wg)
    hw = (yb - ya, Wg)
    Z_ref = oracle.depthwise_glu(Ur[None], Kd, hw)[0, rows]
    mag = oracle.depthwise3x3(np.abs(Ur)[None], np.abs(Kd), hw)[0, rows, :Ch]
    Zg = to_f64(Z[b, y0 * Wg:y1 * Wg])
    dZ = np.abs(Zg - Z_ref)
    assert np.all(dZ <= 2.0 ** -7 * np.abs(Z_ref) + 1e-5 * mag + 1e-30), (b, y0)
    # project on the GPU's own Z: one bf16 rounding plus fp32 accumulation
    Yg = to_f64(Y[b, y0 * Wg:y1 * Wg])
    Y_ref = Zg @ W2d.T
    bound = 2.0 ** -8 * np.abs(Y_ref) + Ch * 2.0 ** -23 * (np.abs(Zg) @ np.abs(W2d).T) + 1e-30
    assert np.all(np.abs(Yg - Y_ref) <= bound), (b, y0)
    # end to end against the oracle's own intermediates
    Z_e2e = oracle.depthwise_glu(U_ref[None], Kd, hw)[0, rows]
    Y_e2e = Z_e2e @ W2d.T
    f = float(np.mean(Zg != Z_e2e))
    tol = 2.0 ** -8 + 4.0 * np.sqrt(f) * 2.0 ** -7 + 1e-5
    rel = np.linalg.norm(Yg - Y_e2e, axis=-1) / np.maximum(np.linalg.norm(Y_e2e, axis=-1), 1e-30)
    assert rel.max() <= tol, ((b, y0), rel.max(), tol, f)
    return int(np.sum(dU > 0)), dU.size, int(np.sum(Zg != Z_e2e)), Zg.size


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
    U, Z = _intermediates(ws, B, N, Ch)
    cu = tu = cz = tz = 0
    for b in range(B):
        a = _check_grid_rows(oracle, X, W1, Kdw, W2, U, Z, Y, b, 0, Hg, Hg, Wg)
        cu, tu, cz, tz = cu + a[0], tu + a[1], cz + a[2], tz + a[3]
    assert cu / tu < 1e-2 and cz / tz < 1e-2, (cu / tu, cz / tz)
    # and the composition itself: the whole block against oracle.mix_ffn
    Y_e2e = oracle.mix_ffn(to_f64(X), to_f64(W1), to_f64(Kdw), to_f64(W2), (Hg, Wg))
    rel = np.linalg.norm(to_f64(Y) - Y_e2e, axis=-1) / np.maximum(np.linalg.norm(Y_e2e, axis=-1), 1e-30)
    assert rel.max() <= 2.0 ** -8 + 4.0 * np.sqrt(cz / tz) * 2.0 ** -7 + 1e-5, rel.max()
    assert ops.device_error() == 0


def test_mix_ffn_deterministic():
    B, Hg, Wg, C, Ch = 2, 16, 24, 256, 320
    X, W1, Kdw, W2 = _inputs(B, Hg, Wg, C, Ch, seed=3)
    Y1 = ops.mix_ffn(X, W1, Kdw, W2, (Hg, Wg))
    Y2 = ops.mix_ffn(X, W1, Kdw, W2, (Hg, Wg))
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def test_mix_ffn_4096px_grid_rows(oracle):
    """The bench's 4096px Mix-FFN (B = 2, 128 x 128 grid, C = 2240, Ch = 5600),
    in the launch configuration the bench times: four whole grid rows (the top
    and bottom edges and two interior rows, 512 tokens, both batches), stage by
    stage and end to end, with the bounds above."""
    B, Hg, Wg, C, Ch = 2, 128, 128, 2240, 5600
    N = Hg * Wg
    X, W1, Kdw, W2 = _inputs(B, Hg, Wg, C, Ch, seed=4096)
    ws = torch.empty(ops.mix_ffn_workspace_bytes(B, Hg, Wg, C, Ch), dtype=torch.uint8, device="cuda")
    Y = ops.mix_ffn(X, W1, Kdw, W2, (Hg, Wg), workspace=ws)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    U, Z = _intermediates(ws, B, N, Ch)
    cu = tu = cz = tz = 0
    for b, y in [(0, 0), (0, 63), (1, 100), (1, Hg - 1)]:
        a = _check_grid_rows(oracle, X, W1, Kdw, W2, U, Z, Y, b, y, y + 1, Hg, Wg)
        cu, tu, cz, tz = cu + a[0], tu + a[1], cz + a[2], tz + a[3]
    assert cu / tu < 1e-2 and cz / tz < 1e-2, (cu / tu, cz / tz)
