"""Parity of the ELU+1 and cos feature maps ("08_sana高效高分辨率生成", section
"Linear Attention 的原理": alternatives to ReLU) with the fp64 oracle, through the
C ABI: every element at small and mid-size shapes (ragged, head size 64, more
slabs than SMs; the 4096px shape is in test_gpu_headline_full.py), the states themselves,
forward == kv_state + apply bit for bit, and ReLU through the feature-map
entry points == the plain calls bit for bit."""
from dataclasses import replace

import numpy as np
import pytest
import torch

from linear_attention_diffusion_relu_b200 import ops
from linear_attention_diffusion_relu_b200.workloads import WORKLOADS, Workload, make_inputs
from tests.parity import check_output, to_f64

pytestmark = pytest.mark.gpu

OUT_DTYPES = [torch.float32, torch.bfloat16]
FEATURES = ["elu1", "cos"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_diffusion_relu_b200 import build
    build.build()
    ops.load_library()


def _dt(dtype):
    return "f32" if dtype == torch.float32 else "bf16"


SHAPES = [(1, 1, 1, 32), (1, 129, 5, 32), (2, 1000, 3, 32), (1, 4097, 2, 64), (3, 513, 7, 32),
          (2, 300, 18, 64), (5, 100, 150, 32), (2, 4096, 70, 32)]


@pytest.mark.parametrize("feature", FEATURES)
@pytest.mark.parametrize("dtype", OUT_DTYPES, ids=_dt)
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}N{}H{}d{}".format(*s))
def test_feature_map_every_element(oracle, shape, dtype, feature):
    B, N, H, d = shape
    Q, K, V = make_inputs(Workload("fm", B, N, H, d, seed=300 + N + H), device="cuda")
    O = ops.forward(Q, K, V, out_dtype=dtype, feature_map=feature)
    torch.cuda.synchronize()
    ref = oracle.forward_fm(to_f64(Q), to_f64(K), to_f64(V), feature, 1e-15)
    check_output(O, ref, f"{feature} {shape}")


@pytest.mark.parametrize("feature", FEATURES)
def test_feature_map_state(oracle, feature):
    """Each state entry within 1e-5 of the sum of |terms| it adds up (the
    bound sum_n |phi(K_ni)| |[V | 1]_nj| is formed here in numpy)."""
    w = replace(WORKLOADS["sweep_N16384"], H=5)
    _, K, V = make_inputs(w, device="cuda")
    S = ops.kv_state(K, V, feature_map=feature)
    torch.cuda.synchronize()
    Kd, Vd = to_f64(K), to_f64(V)
    ref = oracle.state_fm(Kd, Vd, feature)
    phi = np.abs(np.cos(Kd)) if feature == "cos" else np.where(Kd > 0, Kd + 1, np.exp(np.minimum(Kd, 0)))
    v1 = np.concatenate([np.abs(Vd), np.ones(Vd.shape[:-1] + (1,))], axis=-1)
    mag = np.einsum("bnhi,bnhj->bhij", phi, v1)
    err = np.abs(to_f64(S) - ref)
    assert np.all(err <= 1e-5 * mag + 1e-30), (err / (mag + 1e-30)).max()


@pytest.mark.parametrize("feature", FEATURES)
@pytest.mark.parametrize("shape", [(2, 1531, 6, 32), (5, 100, 150, 32), (16, 200, 20, 64)],
                         ids=lambda s: "B{}N{}H{}d{}".format(*s))
def test_feature_map_forward_equals_two_calls(shape, feature):
    B, N, H, d = shape
    Q, K, V = make_inputs(Workload("fmb", B, N, H, d, seed=7), device="cuda")
    for dtype in OUT_DTYPES:
        bits = torch.int32 if dtype == torch.float32 else torch.int16
        O1 = ops.forward(Q, K, V, out_dtype=dtype, feature_map=feature)
        O2 = ops.forward(Q, K, V, out_dtype=dtype, feature_map=feature)
        O3 = ops.apply(Q, ops.kv_state(K, V, feature_map=feature), out_dtype=dtype, feature_map=feature)
        torch.cuda.synchronize()
        assert torch.equal(O1.view(bits), O2.view(bits))
        assert torch.equal(O1.view(bits), O3.view(bits))


def test_relu_through_feature_map_entry_is_the_plain_call():
    """The plain C entry points and the *_fm ones with SANA_LA_FEATURE_RELU
    give the same bits."""
    B, N, H, d = 2, 1531, 6, 32
    Q, K, V = make_inputs(Workload("fmr", B, N, H, d, seed=8), device="cuda")
    lib = ops.load_library()
    O1 = torch.empty_like(Q)
    ws = ops.make_workspace(B, N, H, d, "cuda")
    st = lib.sana_linattn_forward(Q.data_ptr(), K.data_ptr(), V.data_ptr(), B, N, H, d, O1.data_ptr(),
                                  ops.OUT_BF16, 1e-15, ws.data_ptr(), ws.numel(),
                                  torch.cuda.current_stream().cuda_stream)
    assert st == ops.OK
    O2 = ops.forward(Q, K, V, feature_map="relu")
    torch.cuda.synchronize()
    assert torch.equal(O1.view(torch.int16), O2.view(torch.int16))
    assert ops.device_error() == 0
