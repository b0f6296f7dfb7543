"""Parity of the block-causal CUDA path (SANA-Video's block causal linear
attention, "linear-diffusion-transformer-4k-efficient-generation", section
"技术演进：从图像到视频与世界模型") with the fp64 oracle, through the C ABI.

Blocks of L tokens; a query of block j uses the prefix state of blocks 0 .. j.
Small and mid-size shapes compare every output element (ragged last blocks,
L >= N, more slabs than SMs, head size 64, block lengths whose tile counts
force few CTAs per slab); the 16-frame video shape compares sampled heads and
rows, including the first and last token of every block. The one-launch form
(running prefix states in the apply phase) is checked bit for bit against the
three-kernel forward at every shape. Also: the prefix states themselves,
forward == kv_state + apply bit for bit, determinism, and that later blocks
never reach earlier outputs."""
import numpy as np
import pytest
import torch

from linear_attention_diffusion_relu_b200 import ops
from linear_attention_diffusion_relu_b200.workloads import WORKLOADS, Workload, make_inputs
from tests.parity import check_output, head_slice, to_f64

pytestmark = pytest.mark.gpu

OUT_DTYPES = [torch.float32, torch.bfloat16]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_diffusion_relu_b200 import build
    build.build()
    ops.load_library()


def _dt(dtype):
    return "f32" if dtype == torch.float32 else "bf16"


SHAPES = [
    (1, 1024, 4, 32, 128),       # L = 128: one CTA per slab
    (2, 3572, 6, 32, 1024),      # ragged last block
    (1, 300, 3, 64, 128),        # head size 64, ragged
    (5, 1000, 150, 32, 384),     # more slabs than SMs: several slabs per CTA
    (16, 900, 20, 64, 256),
    (1, 777, 2, 64, 640),
    (1, 500, 3, 32, 1024),       # L > N: one block
    (1, 17281, 9, 32, 5760),     # L / 128 = 45: 4 x 9 CTAs per slab over 4 blocks
    (2, 16384, 70, 32, 1024),    # 16 frames of 32x32 tokens at the 1.6B width
    (1, 1280, 80, 32, 128),      # 7 CTAs per slab over 10 blocks: some take two
    (1, 4600, 120, 32, 1024),    # 2 x 2 CTAs per slab: 5 ragged blocks over 2, tiles split 2 ways
]


def _ids(s):
    return "B{}N{}H{}d{}L{}".format(*s)


@pytest.mark.parametrize("dtype", OUT_DTYPES, ids=_dt)
@pytest.mark.parametrize("shape", SHAPES, ids=_ids)
def test_block_causal_every_element(oracle, shape, dtype):
    B, N, H, d, L = shape
    Q, K, V = make_inputs(Workload("bc", B, N, H, d, seed=200 + N + L), device="cuda")
    O = ops.block_causal_forward(Q, K, V, L, out_dtype=dtype)
    O1 = ops.block_causal_forward(Q, K, V, L, out_dtype=dtype, single_launch=True)
    torch.cuda.synchronize()
    ref = oracle.block_causal_forward(to_f64(Q), to_f64(K), to_f64(V), L, 1e-15)
    check_output(O, ref, f"block-causal {shape}")
    bits = torch.int32 if dtype == torch.float32 else torch.int16
    assert torch.equal(O1.view(bits), O.view(bits)), "single launch differs from the three kernels"
    assert ops.device_error() == 0


def test_block_causal_prefix_states(oracle):
    """Each prefix-state entry within 1e-5 of the sum of |terms| it adds up."""
    B, N, H, d, L = 2, 3572, 6, 32, 1024
    _, K, V = make_inputs(Workload("bcs", B, N, H, d, seed=9), device="cuda")
    P = ops.block_causal_kv_state(K, V, L)
    torch.cuda.synchronize()
    Kd, Vd = to_f64(K), to_f64(V)
    ref = oracle.block_causal_state(Kd, Vd, L)
    mag = oracle.block_causal_state(Kd, np.abs(Vd), L)
    err = np.abs(to_f64(P) - ref)
    assert np.all(err <= 1e-5 * mag + 1e-30), (err / (mag + 1e-30)).max()


@pytest.mark.parametrize("shape", [SHAPES[1], SHAPES[3], SHAPES[4], SHAPES[7], SHAPES[10]], ids=_ids)
def test_block_causal_forward_equals_two_calls_and_is_deterministic(shape):
    B, N, H, d, L = shape
    Q, K, V = make_inputs(Workload("bcb", B, N, H, d, seed=3), device="cuda")
    for dtype in OUT_DTYPES:
        bits = torch.int32 if dtype == torch.float32 else torch.int16
        O1 = ops.block_causal_forward(Q, K, V, L, out_dtype=dtype)
        O2 = ops.block_causal_forward(Q, K, V, L, out_dtype=dtype)
        O3 = ops.block_causal_apply(Q, ops.block_causal_kv_state(K, V, L), L, out_dtype=dtype)
        O4 = ops.block_causal_forward(Q, K, V, L, out_dtype=dtype, single_launch=True)
        O5 = ops.block_causal_forward(Q, K, V, L, out_dtype=dtype, single_launch=True)
        torch.cuda.synchronize()
        assert torch.equal(O1.view(bits), O2.view(bits))
        assert torch.equal(O1.view(bits), O3.view(bits))
        assert torch.equal(O1.view(bits), O4.view(bits))
        assert torch.equal(O4.view(bits), O5.view(bits))


def test_block_causal_later_blocks_never_reach_earlier_outputs():
    B, N, H, d, L = 1, 4096, 8, 32, 1024
    Q, K, V = make_inputs(Workload("bcf", B, N, H, d, seed=4), device="cuda")
    O = ops.block_causal_forward(Q, K, V, L, out_dtype=torch.float32)
    K2, V2 = K.clone(), V.clone()
    K2[:, 2048:] = K2[:, 2048:].abs() * 3
    V2[:, 2048:] += 1
    O2 = ops.block_causal_forward(Q, K2, V2, L, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(O[:, :2048].view(torch.int32), O2[:, :2048].view(torch.int32))
    assert not torch.equal(O[:, 2048:], O2[:, 2048:])


def test_block_causal_one_block_matches_plain(oracle):
    """L >= N: the plain forward's result (to the output tolerance; the two
    paths sum the same tokens in different chunkings)."""
    w = Workload("bc1", 2, 2000, 6, 32, seed=12)
    Q, K, V = make_inputs(w, device="cuda")
    O = ops.block_causal_forward(Q, K, V, 2048, out_dtype=torch.float32)
    torch.cuda.synchronize()
    check_output(O, oracle.forward(to_f64(Q), to_f64(K), to_f64(V), 1e-15), "one block")


def test_video16f_1024px_every_element(oracle):
    w = WORKLOADS["video16f_1024px"]
    Q, K, V = make_inputs(w, device="cuda")
    ref = oracle.block_causal_forward(to_f64(Q), to_f64(K), to_f64(V), w.block, w.eps)
    for dtype in OUT_DTYPES:
        for single in (False, True):
            O = ops.block_causal_forward(Q, K, V, w.block, out_dtype=dtype, eps=w.eps, single_launch=single)
            torch.cuda.synchronize()
            check_output(O, ref, f"{w.name} {_dt(dtype)}" + (" single launch" if single else ""))


def test_video16f_4096px_sampled_heads_and_rows(oracle):
    """The 16 x 65,536-token video shape (inputs from the seeded CUDA
    generator): two heads' prefix states rebuilt by the oracle from all tokens,
    4,096 sampled rows plus the first and last row of every block checked."""
    w = WORKLOADS["video16f_4096px"]
    L = w.block
    Q, K, V = make_inputs(w, device="cuda", generator_device="cuda")
    heads = [1, w.H - 2]
    rows = set(np.random.default_rng(1).choice(w.N, size=4096, replace=False).tolist())
    for j in range(w.N // L):
        rows |= {j * L, j * L + L - 1}
    rows = np.array(sorted(rows))
    P = oracle.block_causal_state(head_slice(K, heads), head_slice(V, heads), L)
    Qh = head_slice(Q, heads)
    for dtype in OUT_DTYPES:
        O = ops.block_causal_forward(Q, K, V, L, out_dtype=dtype, eps=w.eps)
        O1 = ops.block_causal_forward(Q, K, V, L, out_dtype=dtype, eps=w.eps, single_launch=True)
        torch.cuda.synchronize()
        bits = torch.int32 if dtype == torch.float32 else torch.int16
        assert torch.equal(O1.view(bits), O.view(bits)), "single launch differs from the three kernels"
        del O1
        got = O[:, :, heads, :]
        for j in range(w.N // L):
            sel = rows[(rows >= j * L) & (rows < (j + 1) * L)]
            ref = oracle.apply(Qh[:, sel], P[:, :, j], w.eps)
            check_output(got[:, torch.as_tensor(sel, device=O.device)], ref,
                         f"{w.name} block {j} {_dt(dtype)}")
    assert ops.device_error() == 0
