"""Every output element of the headline shapes against the fp64 oracle, in the
launch configuration the bench times (one fwd_fused_tc launch per forward).

* The 4096px Sana-1.6B-like step (B = 2, N = 16384, H = 70, d = 32) with
  phi = ReLU, ELU+1 and cos, bf16 and fp32 output: all 140 (b, h) pairs, all
  16384 tokens, every element ("08_sana高效高分辨率生成", "Linear Attention 的原理";
  the normalised form of "linear-diffusion-transformer-4k-efficient-generation",
  "核心架构"). The oracle rebuilds each batch's states from all tokens.
* The two longest sweep points (N = 262144 and N = 1048576, H = 36): every
  head, with the oracle's states built from all N tokens and the output checked
  on sampled rows (first, last and random ones); the heads go through the
  oracle a few at a time so the fp64 copies stay within a few GB of host memory.

Tolerances are those of ``tests/parity.py`` (fp32 output: 1e-4 of the row norm;
bf16 output: 2^-7 |ref| + 1e-3 per element; rows with phi(Q) = 0 exactly 0)."""
import numpy as np
import pytest
import torch

from linear_attention_diffusion_relu_b200 import ops
from linear_attention_diffusion_relu_b200.workloads import WORKLOADS, make_inputs
from tests.parity import check_output, to_f64

pytestmark = pytest.mark.gpu

OUT_DTYPES = [torch.float32, torch.bfloat16]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_diffusion_relu_b200 import build
    build.build()
    ops.load_library()


def _oracle_forward(oracle, feature, Q, K, V, eps):
    if feature == "relu":
        return oracle.forward(Q, K, V, eps)
    return oracle.forward_fm(Q, K, V, feature, eps)


@pytest.mark.parametrize("name", ["4096px", "4096px_elu1", "4096px_cos"])
def test_headline_every_element(oracle, name):
    w = WORKLOADS[name]
    Q, K, V = make_inputs(w, device="cuda")
    refs = [_oracle_forward(oracle, w.feature, *(to_f64(t[b:b + 1]) for t in (Q, K, V)), w.eps)
            for b in range(w.B)]
    for dtype in OUT_DTYPES:
        O = ops.forward(Q, K, V, out_dtype=dtype, eps=w.eps, feature_map=w.feature)
        torch.cuda.synchronize()
        for b in range(w.B):
            check_output(O[b:b + 1], refs[b], f"{name} batch {b} {dtype}")
    assert ops.device_error() == 0


def _sampled_rows(N, count, seed=0):
    rows = np.sort(np.random.default_rng(seed).choice(N, size=count, replace=False))
    rows[0], rows[-1] = 0, N - 1
    return rows


@pytest.mark.parametrize("name,count", [("sweep_N262144", 8192), ("sweep_N1048576", 4096)])
def test_longest_sweep_every_head(oracle, name, count):
    """All heads; states from all N tokens, outputs on sampled rows."""
    w = WORKLOADS[name]
    Q, K, V = make_inputs(w, device="cuda", generator_device="cuda")
    rows = _sampled_rows(w.N, count)
    rows_dev = torch.as_tensor(rows, device="cuda")
    outs = {}
    for dtype in OUT_DTYPES:
        O = ops.forward(Q, K, V, out_dtype=dtype, eps=w.eps)
        outs[dtype] = O[:, rows_dev]            # (B, rows, H, d) on the device
        del O
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    step = 4 if w.N > 300_000 else 12
    for h0 in range(0, w.H, step):
        h1 = min(w.H, h0 + step)
        S = oracle.state(to_f64(K[:, :, h0:h1]), to_f64(V[:, :, h0:h1]))
        ref = oracle.apply(to_f64(Q[:, rows_dev, h0:h1]), S, w.eps)
        for dtype in OUT_DTYPES:
            check_output(outs[dtype][:, :, h0:h1], ref, f"{name} heads {h0}..{h1 - 1} {dtype}")
