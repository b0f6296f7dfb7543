"""Seeded random shapes through the C ABI against the fp64 oracle: batch,
token count (ragged, from 1), head count (including head counts that leave a
part-filled last head group), head size, feature map, output type, and for a
share of them the block-causal form with a random block length. Every case is
checked in every element, and the single launch against the two-call API bit
for bit (SANA walk-through, "Linear Attention 的原理" for the feature maps;
"linear-diffusion-transformer-4k-efficient-generation", "核心架构" for the
normalised form)."""
import numpy as np
import pytest
import torch

from linear_attention_diffusion_relu_b200 import ops
from linear_attention_diffusion_relu_b200.workloads import Workload, make_inputs
from tests.parity import check_output, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_diffusion_relu_b200 import build
    build.build()
    ops.load_library()


def _cases(n=40, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for k in range(n):
        d = int(rng.choice([32, 64]))
        B = int(rng.integers(1, 4))
        N = int(rng.choice([1, 2, 127, 128, 129]) if k % 5 == 0 else rng.integers(1, 3000))
        H = int(rng.integers(1, 13))
        feature = str(rng.choice(["relu", "relu", "elu1", "cos"]))
        dtype = torch.float32 if rng.random() < 0.5 else torch.bfloat16
        L = int(128 * rng.integers(1, 8)) if feature == "relu" and rng.random() < 0.3 else 0
        out.append((k, B, N, H, d, feature, dtype, L))
    return out


def _id(c):
    k, B, N, H, d, feature, dtype, L = c
    return f"{k}-B{B}N{N}H{H}d{d}-{feature}-{'f32' if dtype == torch.float32 else 'bf16'}" + (f"-L{L}" if L else "")


@pytest.mark.parametrize("case", _cases(), ids=_id)
def test_random_shape_against_oracle(oracle, case):
    k, B, N, H, d, feature, dtype, L = case
    Q, K, V = make_inputs(Workload("fuzz", B, N, H, d, seed=7000 + k), device="cuda")
    bits = torch.int32 if dtype == torch.float32 else torch.int16
    Qd, Kd, Vd = to_f64(Q), to_f64(K), to_f64(V)
    if L:
        O = ops.block_causal_forward(Q, K, V, L, out_dtype=dtype)
        O2 = ops.block_causal_apply(Q, ops.block_causal_kv_state(K, V, L), L, out_dtype=dtype)
        O3 = ops.block_causal_forward(Q, K, V, L, out_dtype=dtype, single_launch=True)
        torch.cuda.synchronize()
        ref = oracle.block_causal_forward(Qd, Kd, Vd, L, 1e-15)
        assert torch.equal(O3.view(bits), O.view(bits)), "single launch differs from the three kernels"
    else:
        O = ops.forward(Q, K, V, out_dtype=dtype, feature_map=feature)
        O2 = ops.apply(Q, ops.kv_state(K, V, feature_map=feature), out_dtype=dtype, feature_map=feature)
        torch.cuda.synchronize()
        ref = (oracle.forward(Qd, Kd, Vd, 1e-15) if feature == "relu"
               else oracle.forward_fm(Qd, Kd, Vd, feature, 1e-15))
    assert torch.equal(O.view(bits), O2.view(bits)), "forward differs from the two-call API"
    check_output(O, ref, _id(case))
    assert ops.device_error() == 0
