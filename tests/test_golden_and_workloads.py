"""CPU checks of the stored oracle record and of the seeded input generators."""
import json
import os

import numpy as np
import torch

from linear_attention_diffusion_relu_b200.workloads import NEG_ROWS, WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "oracle_small.json")


def test_oracle_matches_stored_record(oracle):
    with open(GOLDEN) as f:
        doc = json.load(f)
    shape = tuple(doc["shape_BNHd"])
    Q, K, V = (np.array(doc[k]).reshape(shape) for k in ("Q", "K", "V"))
    S = oracle.state(K, V)
    O = oracle.apply(Q, S, doc["eps"])
    B, N, H, d = shape
    assert np.array_equal(S.ravel(), np.array(doc["state_BHd_dp1"]))
    assert np.array_equal(O.ravel(), np.array(doc["O"]))
    assert np.all(O.reshape(shape)[0, 2, 1] == 0.0)


def test_workload_shapes_and_token_grids():
    # AE-F32C32P1: (px / 32)^2 tokens
    assert WORKLOADS["1024px"].N == (1024 // 32) ** 2
    assert WORKLOADS["2048px"].N == (2048 // 32) ** 2
    assert WORKLOADS["4096px"].N == (4096 // 32) ** 2
    assert WORKLOADS["4096px"].H * WORKLOADS["4096px"].d == 2240
    assert WORKLOADS["1024px"].H * WORKLOADS["1024px"].d == 1152
    w = WORKLOADS["4096px"]
    assert w.algorithmic_bytes(2) == 587_202_560
    assert w.algorithmic_bytes(4) == 734_003_200


def test_generators_are_deterministic_and_shaped():
    w = WORKLOADS["tiny"]
    (q1, k1, v1), (qs, ks, vs) = make_inputs(w, keep_source=True)
    q2, k2, v2 = make_inputs(w)
    for a, b in ((q1, q2), (k1, k2), (v1, v2)):
        assert a.dtype == torch.bfloat16 and a.shape == (1, 256, 4, 32)
        assert torch.equal(a, b)
    assert qs.dtype == torch.float32
    assert torch.equal(qs.to(torch.bfloat16), q1)
    # the forced rows are all-negative in every head, and only they are
    neg = (qs[0] <= 0).all(dim=-1).all(dim=-1)
    assert sorted(torch.nonzero(neg).flatten().tolist()) == list(NEG_ROWS)
    assert (q1[0, list(NEG_ROWS)].float() < 0).all()


def test_head_bias_recipe():
    from dataclasses import replace
    w = replace(WORKLOADS["2048px"], N=64)
    q, k, v = make_inputs(w)
    g = torch.Generator().manual_seed(w.seed)
    shape = (w.B, w.N, w.H, w.d)
    raw = [torch.randn(shape, generator=g) for _ in range(3)]
    bias = [0.1 * torch.randn((1, 1, w.H, 1), generator=g) for _ in range(3)]
    for t, r, b in zip((q, k, v), raw, bias):
        assert torch.equal(t, (0.5 * r + b).to(torch.bfloat16))
