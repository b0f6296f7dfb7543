"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Every output element is compared, from single tokens up to the N = 65536
sweep point (the 4096px shapes and the longest sweep points are in
test_gpu_headline_full.py). Also: determinism, forward == kv_state + apply bit
for bit, guard bands around outputs and workspace, streams, error paths."""
from dataclasses import replace

import numpy as np
import pytest
import torch

from linear_attention_diffusion_relu_b200 import ops
from linear_attention_diffusion_relu_b200.workloads import WORKLOADS, Workload, make_inputs
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


def _dt(dtype):
    return "f32" if dtype == torch.float32 else "bf16"


def _full_check(oracle, Q, K, V, eps, dtype, what):
    O = ops.forward(Q, K, V, out_dtype=dtype, eps=eps)
    torch.cuda.synchronize()
    ref = oracle.forward(to_f64(Q), to_f64(K), to_f64(V), eps)
    check_output(O, ref, what)
    return O, ref


SMALL = [(1, 1, 1, 32), (1, 7, 3, 32), (2, 31, 2, 64), (1, 129, 5, 32), (2, 1000, 3, 32),
         (1, 4097, 2, 64), (3, 513, 7, 32), (1, 2048, 70, 32), (2, 300, 18, 64),
         # two slab sets with an odd slab count: one position holds a single slab
         (1, 3000, 60, 32), (1, 1000, 68, 32),
         # more (b, head-group) slabs than CTAs: several segments per CTA
         (5, 100, 150, 32), (16, 200, 20, 64),
         # more than two segments per CTA: the three-kernel path
         (40, 64, 70, 32)]


@pytest.mark.parametrize("dtype", OUT_DTYPES, ids=_dt)
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B{}N{}H{}d{}".format(*s))
def test_small_shapes(oracle, shape, dtype):
    B, N, H, d = shape
    w = Workload("adhoc", B, N, H, d, seed=100 + N + H)
    Q, K, V = make_inputs(w, device="cuda")
    _full_check(oracle, Q, K, V, 1e-15, dtype, f"{shape}")


@pytest.mark.parametrize("dtype", OUT_DTYPES, ids=_dt)
@pytest.mark.parametrize("name", ["tiny", "1024px", "2048px"])
def test_named_configs_every_element(oracle, name, dtype):
    w = WORKLOADS[name]
    Q, K, V = make_inputs(w, device="cuda")
    O, ref = _full_check(oracle, Q, K, V, w.eps, dtype, name)
    if name == "tiny":
        rows = list(w.neg_rows)
        assert torch.all(O[0, rows] == 0)


FULL = ["ragged_N16381", "d64", "sweep_N1024", "sweep_N16384", "sweep_N65536"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_every_element(oracle, name):
    """Every element of the mid-size workloads (ragged N, head size 64, the
    sweep up to N = 65536) for both output dtypes; the 4096px shapes and the
    longest sweep points are in test_gpu_headline_full.py."""
    w = WORKLOADS[name]
    Q, K, V = make_inputs(w, device="cuda")
    ref = oracle.forward(to_f64(Q), to_f64(K), to_f64(V), w.eps)
    for dtype in OUT_DTYPES:
        O = ops.forward(Q, K, V, out_dtype=dtype, eps=w.eps)
        torch.cuda.synchronize()
        check_output(O, ref, f"{name} {dtype}")


def test_state_matches_oracle(oracle):
    """kv_state alone: each entry within 1e-5 of the sum of |terms| it adds up
    (an fp32 accumulation bound with ample margin), at a multi-chunk size."""
    w = replace(WORKLOADS["sweep_N16384"], H=5)
    Q, K, V = make_inputs(w, device="cuda")
    S = ops.kv_state(K, V)
    torch.cuda.synchronize()
    Kd, Vd = to_f64(K), to_f64(V)
    ref = oracle.state(Kd, Vd)
    mag = oracle.state(Kd, np.abs(Vd))
    err = np.abs(to_f64(S) - ref)
    assert np.all(err <= 1e-5 * mag + 1e-30), (err / (mag + 1e-30)).max()


@pytest.mark.parametrize("dtype", OUT_DTYPES, ids=_dt)
def test_deterministic_and_split_equals_forward(dtype):
    w = WORKLOADS["2048px"]
    Q, K, V = make_inputs(w, device="cuda")
    O1 = ops.forward(Q, K, V, out_dtype=dtype, eps=w.eps)
    O2 = ops.forward(Q, K, V, out_dtype=dtype, eps=w.eps)
    S = ops.kv_state(K, V)
    O3 = ops.apply(Q, S, out_dtype=dtype, eps=w.eps)
    torch.cuda.synchronize()
    bits = torch.int32 if dtype == torch.float32 else torch.int16
    assert torch.equal(O1.view(bits), O2.view(bits))
    assert torch.equal(O1.view(bits), O3.view(bits))
    S2 = ops.kv_state(K, V)
    assert torch.equal(S.view(torch.int32), S2.view(torch.int32))


BITWISE = [(1, 1, 1, 32), (2, 31, 2, 64), (2, 1531, 6, 32), (5, 100, 150, 32), (16, 200, 20, 64),
           (1, 16381, 36, 32), (1, 3000, 60, 32), (40, 64, 70, 32)]


@pytest.mark.parametrize("dtype", OUT_DTYPES, ids=_dt)
@pytest.mark.parametrize("shape", BITWISE, ids=lambda s: "B{}N{}H{}d{}".format(*s))
def test_single_launch_forward_equals_two_calls(shape, dtype):
    """forward (one launch: state phase, grid barrier, apply phase) gives the
    bits of kv_state followed by apply (three launches)."""
    B, N, H, d = shape
    w = Workload("bits", B, N, H, d, seed=31 + N)
    Q, K, V = make_inputs(w, device="cuda")
    O1 = ops.forward(Q, K, V, out_dtype=dtype)
    O2 = ops.apply(Q, ops.kv_state(K, V), out_dtype=dtype)
    torch.cuda.synchronize()
    bits = torch.int32 if dtype == torch.float32 else torch.int16
    assert torch.equal(O1.view(bits), O2.view(bits))


@pytest.mark.parametrize("dtype", OUT_DTYPES, ids=_dt)
def test_guard_bands(dtype):
    """Outputs and workspace are written only inside their extents."""
    B, N, H, d = 2, 1531, 6, 32
    w = Workload("guard", B, N, H, d, seed=7)
    Q, K, V = make_inputs(w, device="cuda")
    pad = 4096
    n_out = B * N * H * d
    big = torch.full((pad + n_out + pad,), 12345.0 if dtype == torch.float32 else 77.0,
                     dtype=dtype, device="cuda")
    O = big[pad:pad + n_out].view(B, N, H, d)
    wsb = ops.workspace_bytes(B, N, H, d)
    wsbig = torch.full((256 + wsb + 4096,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = wsbig[256:256 + wsb]
    ops.forward(Q, K, V, out_dtype=dtype, out=O, workspace=ws)
    torch.cuda.synchronize()
    sentinel = big[0].item()
    assert torch.all(big[:pad] == sentinel) and torch.all(big[pad + n_out:] == sentinel)
    assert torch.all(wsbig[:256] == 0xA5) and torch.all(wsbig[256 + wsb:] == 0xA5)


@pytest.mark.parametrize("dtype", OUT_DTYPES, ids=_dt)
def test_forward_in_cuda_graph(dtype):
    """A captured forward replays correctly with new inputs each time: the
    grid barrier's flags are cleared by the captured memset, not by a fresh
    epoch (which a replay cannot draw)."""
    B, N, H, d = 2, 3001, 9, 32
    w = Workload("graph", B, N, H, d, seed=41)
    Q, K, V = make_inputs(w, device="cuda")
    O = torch.empty((B, N, H, d), dtype=dtype, device="cuda")
    ws = ops.make_workspace(B, N, H, d, "cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        ops.forward(Q, K, V, out_dtype=dtype, out=O, workspace=ws)      # warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ops.forward(Q, K, V, out_dtype=dtype, out=O, workspace=ws)
    bits = torch.int32 if dtype == torch.float32 else torch.int16
    for seed in (1, 2, 3):
        Qn, Kn, Vn = make_inputs(Workload("graph", B, N, H, d, seed=seed), device="cuda")
        Q.copy_(Qn), K.copy_(Kn), V.copy_(Vn)
        O.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        ref = ops.forward(Qn, Kn, Vn, out_dtype=dtype)
        torch.cuda.synchronize()
        assert torch.equal(O.view(bits), ref.view(bits)), seed
    assert ops.device_error() == 0


def test_workspace_shared_across_shapes_and_calls():
    """One workspace, sized for the largest shape, serves forwards of several
    shapes interleaved with kv_state calls; each result equals a forward with a
    fresh workspace bit for bit (stale partial states or barrier flags of an
    earlier call never leak into a later one)."""
    shapes = [(2, 1531, 6, 32), (1, 16381, 36, 32), (3, 200, 5, 64), (2, 1531, 6, 32)]
    wsb = max(ops.workspace_bytes(*sh) for sh in shapes)
    ws = torch.randint(0, 256, (wsb,), dtype=torch.uint8, device="cuda",
                       generator=torch.Generator("cuda").manual_seed(5))
    for i, (B, N, H, d) in enumerate(shapes * 2):
        Q, K, V = make_inputs(Workload("shared", B, N, H, d, seed=60 + i), device="cuda")
        O = ops.forward(Q, K, V, out_dtype=torch.float32, workspace=ws[:ops.workspace_bytes(B, N, H, d)])
        ops.kv_state(K, V, workspace=ws[:ops.workspace_bytes(B, N, H, d)])
        ref = ops.forward(Q, K, V, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(O.view(torch.int32), ref.view(torch.int32)), (B, N, H, d)
    assert ops.device_error() == 0


def test_runs_on_caller_stream(oracle):
    w = Workload("stream", 1, 777, 3, 64, seed=9)
    Q, K, V = make_inputs(w, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        O = ops.forward(Q, K, V, out_dtype=torch.float32)
    s.synchronize()
    check_output(O, oracle.forward(to_f64(Q), to_f64(K), to_f64(V), 1e-15), "side stream")


def test_key_permutation_and_constant_column(oracle):
    w = Workload("inv", 1, 3000, 4, 32, seed=11)
    Q, K, V = make_inputs(w, device="cuda")
    V[..., 7] = 0.375
    O = ops.forward(Q, K, V, out_dtype=torch.float32)
    perm = torch.randperm(w.N, generator=torch.Generator().manual_seed(1)).cuda()
    Op = ops.forward(Q, K[:, perm].contiguous(), V[:, perm].contiguous(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.forward(to_f64(Q), to_f64(K), to_f64(V), 1e-15)
    check_output(Op, ref, "permuted keys")
    live = np.linalg.norm(ref, axis=-1) > 0
    col = to_f64(O)[..., 7][live]
    assert np.allclose(col, 0.375, rtol=1e-5, atol=0)


def test_error_paths_on_device():
    Q = torch.zeros((1, 64, 2, 32), dtype=torch.bfloat16, device="cuda")
    flat = torch.zeros(1 + Q.numel(), dtype=torch.bfloat16, device="cuda")
    mis = flat[1:].view(1, 64, 2, 32)          # 2-byte offset: misaligned
    with pytest.raises(ops.LinAttnError) as e:
        ops.forward(mis, Q, Q)
    assert e.value.status == ops.ERR_INVALID_ARG
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ops.LinAttnError) as e:
        ops.forward(Q, Q, Q, workspace=ws)
    assert e.value.status == ops.ERR_WORKSPACE
    x = torch.zeros((1, 64, 2, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.LinAttnError) as e:
        ops.forward(x, x, x, workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))
    assert e.value.status == ops.ERR_UNSUPPORTED


def test_bounded_wait_times_out_and_reports():
    """A wait on a barrier nothing arrives at gives up after its limit, records
    error code 1, and the context stays usable (a forward afterwards is correct)."""
    torch.cuda.synchronize()
    assert ops.device_error(clear=True) == 0
    ops.selftest_wait_timeout(20000)          # 20 ms limit
    torch.cuda.synchronize()
    assert ops.device_error(clear=True) == 1
    assert ops.device_error() == 0
    w = Workload("after_timeout", 1, 100, 3, 32, seed=5)
    Q, K, V = make_inputs(w, device="cuda")
    from oracle import default
    check_output(ops.forward(Q, K, V, out_dtype=torch.float32),
                 default().forward(to_f64(Q), to_f64(K), to_f64(V), 1e-15), "after timeout")


def test_no_kernel_recorded_an_error():
    """Every pipeline wait in the kernels is bounded; none ran out in this run."""
    torch.cuda.synchronize()
    assert ops.device_error() == 0
