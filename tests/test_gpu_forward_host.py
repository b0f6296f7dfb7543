"""The forward from host buffers (sana_linattn_forward_host and its block-causal
form): the library copies K and V in, computes the state (or the blocks'
prefix states), and streams Q through in chunks whose outputs are copied back
on its own stream while the next chunk comes in. The apply of a token does not
depend on the chunk it is in, so the result must be bit-identical to the
device forward on the same inputs, for every way the tokens are cut into
chunks; and the caller's stream must cover the last copy out."""
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


# chunks: one; pieces of a batch (ragged last); whole batches; several batches
# per chunk; the 4096px shape (16 chunks of 2048 tokens)
SHAPES = [(1, 256, 4, 32), (2, 5000, 6, 32), (3, 700, 5, 64), (8, 300, 4, 32), (2, 16384, 70, 32)]
BITS = {torch.float32: torch.int32, torch.bfloat16: torch.int16}


def _host(B, N, H, d, seed, pinned=True):
    Q, K, V = make_inputs(Workload("host", B, N, H, d, seed=seed))
    return tuple(t.pin_memory() if pinned else t for t in (Q, K, V))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}N{}H{}d{}".format(*s))
def test_forward_host_equals_device_forward(shape, dtype):
    B, N, H, d = shape
    hQ, hK, hV = _host(B, N, H, d, seed=N + H)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        O = ops.forward_host(hQ, hK, hV, out_dtype=dtype)
    side.synchronize()               # the caller's stream covers the copies out
    Od = ops.forward(hQ.cuda(), hK.cuda(), hV.cuda(), out_dtype=dtype)
    assert O.device.type == "cpu" and O.is_pinned()
    assert torch.equal(O.view(BITS[dtype]), Od.cpu().view(BITS[dtype]))
    assert ops.device_error() == 0


def test_forward_host_pageable_buffers_and_feature_map():
    B, N, H, d = 2, 3000, 3, 32
    hQ, hK, hV = _host(B, N, H, d, seed=5, pinned=False)
    out = torch.empty((B, N, H, d), dtype=torch.bfloat16)
    O = ops.forward_host(hQ, hK, hV, out=out, feature_map="elu1")
    torch.cuda.synchronize()
    Od = ops.forward(hQ.cuda(), hK.cuda(), hV.cuda(), feature_map="elu1")
    assert O.data_ptr() == out.data_ptr()
    assert torch.equal(O.view(torch.int16), Od.cpu().view(torch.int16))


def test_forward_host_matches_oracle(oracle):
    B, N, H, d = 2, 2500, 4, 32
    hQ, hK, hV = _host(B, N, H, d, seed=11)
    ws = torch.empty(ops.forward_host_workspace_bytes(B, N, H, d, torch.float32), dtype=torch.uint8, device="cuda")
    O = ops.forward_host(hQ, hK, hV, out_dtype=torch.float32, workspace=ws)
    torch.cuda.synchronize()
    ref = oracle.forward(to_f64(hQ), to_f64(hK), to_f64(hV), 1e-15)
    check_output(O, ref, "forward_host")


def test_forward_host_from_two_threads():
    """Two host threads, each on its own stream, call forward_host on the same
    device at the same time (they share the library's copy streams and events);
    both results are bit-identical to the device forward."""
    import threading
    shapes = [(2, 5000, 6, 32), (1, 9000, 4, 32)]
    inputs = [_host(*sh, seed=40 + i) for i, sh in enumerate(shapes)]
    outs = [None, None]
    errors = []

    def run(i):
        try:
            side = torch.cuda.Stream()
            with torch.cuda.stream(side):
                for _ in range(3):
                    outs[i] = ops.forward_host(*inputs[i])
            side.synchronize()
        except Exception as exc:      # reported below, on the main thread
            errors.append(exc)

    threads = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for i in range(2):
        hQ, hK, hV = inputs[i]
        Od = ops.forward(hQ.cuda(), hK.cuda(), hV.cuda())
        assert torch.equal(outs[i].view(torch.int16), Od.cpu().view(torch.int16))
    assert ops.device_error() == 0


# block-causal: one block per chunk (16 blocks); several blocks per chunk; a
# ragged last block; more blocks than chunks in two batches; N shorter than L
BLOCK_SHAPES = [(1, 16 * 1024, 4, 32, 1024), (1, 5000, 3, 32, 128), (2, 3000, 5, 64, 256),
                (3, 2000, 6, 32, 384), (1, 100, 4, 32, 128)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape", BLOCK_SHAPES, ids=lambda s: "B{}N{}H{}d{}L{}".format(*s))
def test_block_causal_forward_host_equals_device_forward(shape, dtype):
    B, N, H, d, L = shape
    hQ, hK, hV = _host(B, N, H, d, seed=N + L)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        O = ops.block_causal_forward_host(hQ, hK, hV, L, out_dtype=dtype)
    side.synchronize()
    Od = ops.block_causal_forward(hQ.cuda(), hK.cuda(), hV.cuda(), L, out_dtype=dtype)
    assert O.device.type == "cpu" and O.is_pinned()
    assert torch.equal(O.view(BITS[dtype]), Od.cpu().view(BITS[dtype]))
    assert ops.device_error() == 0


def test_block_causal_forward_host_matches_oracle(oracle):
    B, N, H, d, L = 2, 1300, 3, 32, 256
    hQ, hK, hV = _host(B, N, H, d, seed=17, pinned=False)
    O = ops.block_causal_forward_host(hQ, hK, hV, L, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.block_causal_forward(to_f64(hQ), to_f64(hK), to_f64(hV), L, 1e-15)
    check_output(O, ref, "block_causal_forward_host")
