"""sana_linattn_forward_noalloc: the forward for callers that cannot allocate
device memory (their host owns the allocator, their loop must not allocate
once running, or their interface carries no scratch buffer). Its scratch is a
fixed array inside the library instead of a caller workspace.

Called through the C ABI and compared with sana_linattn_forward (caller
workspace) on two calls in a row, within the parity tolerance and bit for bit.
This file is collected last so that a failure here stops a `-x` run only after
every other test has run."""
import ctypes

import pytest
import torch

from linear_attention_diffusion_relu_b200 import ops
from linear_attention_diffusion_relu_b200.workloads import WORKLOADS, make_inputs
from tests.parity import check_output, to_f64

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 16 << 20


def _noalloc_fn():
    lib = ops.load_library()
    fn = lib.sana_linattn_forward_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp, i, i, i, i, vp, i, ctypes.c_float, vp]
    fn.restype = ctypes.c_int
    return lib, fn


@pytest.fixture(scope="module")
def cuda_lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_attention_diffusion_relu_b200 import build
    build.build()
    return _noalloc_fn()


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_noalloc_matches_forward_twice(cuda_lib, out_dtype):
    lib, fn = cuda_lib
    w = WORKLOADS["4096px"]
    assert ops.workspace_bytes(w.B, w.N, w.H, w.d) <= STATIC_SCRATCH_BYTES
    inputs = [make_inputs(w, device="cuda")]
    Q, K, V = inputs[0]
    inputs.append((V.flip(1).contiguous(), Q, K))   # a second, different problem
    code = ops.OUT_F32 if out_dtype == torch.float32 else ops.OUT_BF16
    bits = torch.int32 if out_dtype == torch.float32 else torch.int16
    stream = torch.cuda.current_stream().cuda_stream
    for call, (q, k, v) in enumerate(inputs):       # two calls in a row
        ref = ops.forward(q, k, v, out_dtype=out_dtype, eps=w.eps)
        out = torch.full_like(ref, float("nan"))
        st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), w.B, w.N, w.H, w.d,
                out.data_ptr(), code, w.eps, stream)
        assert st == ops.OK, (call, lib.sana_linattn_last_error().decode())
        torch.cuda.synchronize()
        check_output(out, to_f64(ref), f"noalloc call {call}")
        assert torch.equal(out.view(bits), ref.view(bits)), f"call {call} differs from forward"


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_lib):
    lib, fn = cuda_lib
    B, N, H, d = 16, 65536, 70, 64
    assert ops.workspace_bytes(B, N, H, d) > STATIC_SCRATCH_BYTES
    fake = 1 << 20      # never dereferenced: the size check comes first
    st = fn(fake, fake, fake, B, N, H, d, fake, ops.OUT_BF16, 1e-15, None)
    assert st == ops.ERR_WORKSPACE
    assert "static scratch" in lib.sana_linattn_last_error().decode()
