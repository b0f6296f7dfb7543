"""The C-ABI library loads, exports every function the header declares, and
rejects bad arguments on the host before launching anything. No GPU needed:
every call here returns before any CUDA work is enqueued."""
import ctypes
import os
import re

import pytest

from linear_attention_diffusion_relu_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.load_library()


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(sana_linattn_\w+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("sana_linattn_kv_state", "sana_linattn_apply", "sana_linattn_forward",
                     "sana_linattn_workspace_bytes"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(ops.SYMBOLS) <= set(declared_functions())


def test_status_strings(lib):
    for code in range(5):
        s = lib.sana_linattn_status_string(code).decode()
        assert s and s != "unknown status"
    assert lib.sana_linattn_status_string(99).decode() == "unknown status"


def test_workspace_bytes(lib):
    ws = lib.sana_linattn_workspace_bytes
    assert ws(2, 16384, 70, 32) > 0
    assert ws(2, 16384, 70, 32) % 256 == 0
    assert ws(1, 1, 1, 32) > 0
    assert ws(1, 1, 1, 48) == 0          # unsupported head size
    assert ws(0, 16, 1, 32) == 0
    assert ws(1, 0, 1, 32) == 0
    assert ws(1, 16, -1, 64) == 0
    # at least the reduced state plus one partial per (b, h)
    assert ws(2, 16384, 70, 32) >= 2 * 70 * 32 * 33 * 4 * 2
    # does not grow without bound with N (chunk count is capped)
    assert ws(1, 1 << 20, 36, 32) < 64 << 20


FAKE = 1 << 20   # aligned, never dereferenced: every call below fails its host checks


def test_null_and_size_errors(lib):
    f = lib.sana_linattn_forward
    wsb = lib.sana_linattn_workspace_bytes(1, 64, 2, 32)
    assert f(None, FAKE, FAKE, 1, 64, 2, 32, FAKE, 1, 1e-15, FAKE, wsb, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 0, 64, 2, 32, FAKE, 1, 1e-15, FAKE, wsb, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 0, 2, 32, FAKE, 1, 1e-15, FAKE, wsb, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 64, 2, 48, FAKE, 1, 1e-15, FAKE, wsb, None) == ops.ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 1, 64, 2, 32, FAKE, 7, 1e-15, FAKE, wsb, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 64, 2, 32, FAKE, 1, -1.0, FAKE, wsb, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 64, 2, 32, FAKE, 1, float("nan"), FAKE, wsb, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 64, 2, 32, FAKE, 1, float("inf"), FAKE, wsb, None) == ops.ERR_INVALID_ARG
    assert f(FAKE + 2, FAKE, FAKE, 1, 64, 2, 32, FAKE, 1, 1e-15, FAKE, wsb, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 64, 2, 32, FAKE + 8, 1, 1e-15, FAKE, wsb, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 64, 2, 32, FAKE, 1, 1e-15, FAKE, wsb - 1, None) == ops.ERR_WORKSPACE
    # element count overflow
    assert f(FAKE, FAKE, FAKE, 1 << 30, 1 << 30, 1 << 10, 32, FAKE, 1, 0.0, FAKE, wsb, None) \
        == ops.ERR_INVALID_ARG


def test_kv_state_and_apply_errors(lib):
    ks, ap = lib.sana_linattn_kv_state, lib.sana_linattn_apply
    wsb = lib.sana_linattn_workspace_bytes(2, 100, 3, 64)
    assert ks(FAKE, None, 2, 100, 3, 64, FAKE, FAKE, wsb, None) == ops.ERR_INVALID_ARG
    assert ks(FAKE, FAKE, 2, 100, 3, 16, FAKE, FAKE, wsb, None) == ops.ERR_UNSUPPORTED
    assert ks(FAKE, FAKE, 2, 100, 3, 64, FAKE + 4, FAKE, wsb, None) == ops.ERR_INVALID_ARG
    assert ks(FAKE, FAKE, 2, 100, 3, 64, FAKE, FAKE, 0, None) == ops.ERR_WORKSPACE
    assert ap(None, FAKE, 2, 100, 3, 64, FAKE, 0, 0.0, None) == ops.ERR_INVALID_ARG
    assert ap(FAKE, FAKE, 2, 100, 3, 64, FAKE, 2, 0.0, None) == ops.ERR_INVALID_ARG
    assert ap(FAKE, FAKE, 2, 100, 3, 64, FAKE, 0, -1e-3, None) == ops.ERR_INVALID_ARG
    assert ap(FAKE, FAKE, 2, -100, 3, 64, FAKE, 0, 0.0, None) == ops.ERR_INVALID_ARG
    assert lib.sana_linattn_last_error().decode() == ""
    # self-test limits are checked before any launch
    assert lib.sana_linattn_selftest_wait_timeout(0, None) == ops.ERR_INVALID_ARG
    assert lib.sana_linattn_selftest_wait_timeout(20_000_000, None) == ops.ERR_INVALID_ARG


def test_binding_rejects_cpu_tensors(lib):
    import torch
    x = torch.zeros((1, 8, 1, 32), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        ops.forward(x, x, x)


def test_library_is_sm100a_only():
    """The build targets sm_100a and nothing else (no PTX for other archs)."""
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.NVCC_FLAGS)
    assert not any("compute_90" in f or "sm_90" in f for f in build.NVCC_FLAGS)


def test_block_causal_host_checks(lib):
    wsb = lib.sana_linattn_block_causal_workspace_bytes
    assert wsb(2, 3572, 6, 32, 1024) > 0
    assert wsb(2, 3572, 6, 32, 1024) % 256 == 0
    # the prefix states alone: B * H * nblk * d * (d+1) fp32
    assert wsb(2, 3572, 6, 32, 1024) >= 2 * 6 * 4 * 32 * 33 * 4
    assert wsb(2, 3572, 6, 32, 100) == 0          # not a multiple of 128
    assert wsb(2, 3572, 6, 32, 0) == 0
    assert wsb(2, 3572, 6, 48, 1024) == 0         # head size
    assert wsb(1, 1 << 24, 36, 32, 128) == 0      # partials beyond the 4 GiB cap
    assert wsb(1, 1 << 24, 36, 32, 65536) > 0
    n = lib.sana_linattn_block_causal_forward_launches
    assert n(2, 3572, 6, 32, 1024) == 3 and n(2, 3572, 6, 32, 96) == 0
    n1 = lib.sana_linattn_block_causal_forward_single_launches
    assert n1(2, 3572, 6, 32, 1024) == 1 and n1(2, 3572, 6, 32, 96) == 0
    f = lib.sana_linattn_block_causal_forward
    ws = wsb(1, 1024, 2, 32, 256)
    assert f(FAKE, FAKE, FAKE, 1, 1024, 2, 32, 100, FAKE, 1, 1e-15, FAKE, ws, None) == ops.ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 1, 1024, 2, 32, 0, FAKE, 1, 1e-15, FAKE, ws, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 1024, 2, 32, -128, FAKE, 1, 1e-15, FAKE, ws, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 1024, 2, 32, 256, FAKE, 1, 1e-15, FAKE, ws - 1, None) == ops.ERR_WORKSPACE
    assert f(None, FAKE, FAKE, 1, 1024, 2, 32, 256, FAKE, 1, 1e-15, FAKE, ws, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 1024, 2, 32, 256, FAKE, 1, -1.0, FAKE, ws, None) == ops.ERR_INVALID_ARG
    ks = lib.sana_linattn_block_causal_kv_state
    assert ks(FAKE, FAKE, 1, 1024, 2, 32, 192, FAKE, FAKE, ws, None) == ops.ERR_UNSUPPORTED
    assert ks(FAKE, FAKE, 1, 1024, 2, 32, 256, FAKE, FAKE, 0, None) == ops.ERR_WORKSPACE
    ap = lib.sana_linattn_block_causal_apply
    assert ap(FAKE, FAKE, 1, 1024, 2, 32, 200, FAKE, 0, 0.0, None) == ops.ERR_UNSUPPORTED
    assert ap(FAKE, FAKE, 1, 1024, 2, 32, 256, FAKE, 5, 0.0, None) == ops.ERR_INVALID_ARG


def test_feature_map_host_checks(lib):
    wsb = lib.sana_linattn_workspace_bytes(1, 64, 2, 32)
    f = lib.sana_linattn_forward_fm
    for bad in (-1, 3, 99):
        assert f(FAKE, FAKE, FAKE, 1, 64, 2, 32, bad, FAKE, 1, 1e-15, FAKE, wsb, None) == ops.ERR_INVALID_ARG
        assert lib.sana_linattn_kv_state_fm(FAKE, FAKE, 1, 64, 2, 32, bad, FAKE, FAKE, wsb, None) \
            == ops.ERR_INVALID_ARG
        assert lib.sana_linattn_apply_fm(FAKE, FAKE, 1, 64, 2, 32, bad, FAKE, 1, 0.0, None) == ops.ERR_INVALID_ARG
    # valid feature maps still get the ordinary checks
    for fm in ops.FEATURE_MAPS.values():
        assert f(FAKE, FAKE, FAKE, 1, 64, 2, 48, fm, FAKE, 1, 1e-15, FAKE, wsb, None) == ops.ERR_UNSUPPORTED
        assert f(FAKE, FAKE, FAKE, 1, 64, 2, 32, fm, FAKE, 1, 1e-15, FAKE, wsb - 1, None) == ops.ERR_WORKSPACE
    import torch
    x = torch.zeros((1, 8, 1, 32), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="feature_map"):
        ops.forward(x, x, x, feature_map="softmax")


def test_kv_projection_host_checks(lib):
    wsb = lib.sana_linattn_kv_projection_workspace_bytes
    assert wsb(2, 16384, 2240, 70, 32) > 0
    assert wsb(2, 16384, 2240, 70, 32) % 256 == 0
    assert wsb(2, 16384, 2244, 70, 32) == 0     # C not a multiple of 8
    assert wsb(2, 16384, 0, 70, 32) == 0
    assert wsb(2, 16384, 2240, 70, 48) == 0     # head size
    f = lib.sana_linattn_kv_projection_state
    ws = wsb(1, 300, 128, 4, 32)
    assert f(None, FAKE, FAKE, 1, 300, 128, 4, 32, FAKE, FAKE, ws, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 300, 124, 4, 32, FAKE, FAKE, ws, None) == ops.ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 1, 300, 128, 4, 48, FAKE, FAKE, ws, None) == ops.ERR_UNSUPPORTED
    assert f(FAKE, FAKE + 8, FAKE, 1, 300, 128, 4, 32, FAKE, FAKE, ws, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 300, 128, 4, 32, FAKE, FAKE, ws - 1, None) == ops.ERR_WORKSPACE
    assert lib.sana_linattn_kv_projection_state_launches(1, 300, 128, 4, 32) == 2
    assert lib.sana_linattn_kv_projection_state_launches(1, 300, 124, 4, 32) == 0


def test_mix_ffn_host_checks(lib):
    wsb = lib.sana_linattn_mix_ffn_workspace_bytes
    assert wsb(2, 128, 128, 2240, 5600) > 0
    assert wsb(2, 128, 128, 2244, 5600) == 0        # C not a multiple of 8
    assert wsb(2, 128, 128, 2240, 5604) == 0        # Ch not a multiple of 8
    assert wsb(0, 128, 128, 2240, 5600) == 0
    # U (2 Ch bf16) and Z (Ch bf16) per token
    assert wsb(1, 4, 4, 64, 32) >= 16 * (64 + 32) * 2
    f = lib.sana_linattn_mix_ffn
    ws = wsb(1, 4, 4, 64, 32)
    assert f(None, FAKE, FAKE, FAKE, 1, 4, 4, 64, 32, FAKE, FAKE, ws, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 4, 4, 60, 32, FAKE, FAKE, ws, None) == ops.ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE + 2, FAKE, 1, 4, 4, 64, 32, FAKE, FAKE, ws, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 4, 4, 64, 32, FAKE, FAKE, ws - 1, None) == ops.ERR_WORKSPACE
    assert lib.sana_linattn_mix_ffn_launches(1, 4, 4, 64, 32) == 3


def test_forward_host_host_checks(lib):
    wsb = lib.sana_linattn_forward_host_workspace_bytes
    n16 = wsb(2, 1000, 6, 32, ops.OUT_BF16)
    n32 = wsb(2, 1000, 6, 32, ops.OUT_F32)
    assert n16 > 0 and n16 % 256 == 0 and n32 > n16
    # at least the four device copies and the state
    assert n16 >= 4 * (2 * 1000 * 6 * 32 * 2) + 2 * 6 * 32 * 33 * 4
    assert wsb(2, 1000, 6, 48, ops.OUT_BF16) == 0
    assert wsb(2, 1000, 6, 32, 7) == 0
    n = lib.sana_linattn_forward_host_launches
    assert n(2, 16384, 70, 32) == 2 + 16         # 2048 tokens per chunk
    assert n(1, 256, 4, 32) == 3                 # one chunk
    assert n(8, 300, 4, 32) == 2 + 3             # three batches per chunk
    assert n(0, 1, 1, 32) == 0
    f = lib.sana_linattn_forward_host
    ws = wsb(1, 1024, 2, 32, ops.OUT_BF16)
    # argument errors come back before any CUDA call
    assert f(None, FAKE, FAKE, 1, 1024, 2, 32, 0, FAKE, 1, 1e-15, FAKE, ws, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 1024, 2, 32, 3, FAKE, 1, 1e-15, FAKE, ws, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 1024, 2, 32, 0, FAKE, 1, -1.0, FAKE, ws, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 1024, 2, 32, 0, FAKE, 5, 1e-15, FAKE, ws, None) == ops.ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 1, 1024, 2, 48, 0, FAKE, 1, 1e-15, FAKE, ws, None) == ops.ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 1, 1024, 2, 32, 0, FAKE, 1, 1e-15, FAKE, ws - 256, None) == ops.ERR_WORKSPACE
