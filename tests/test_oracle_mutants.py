"""Each plausible mistake planted in a copy of the oracle's C source must fail at
least one pin. This shows the pins constrain every term of the oracle: a
dropped feature map, a misplaced eps, a wrong normaliser column, a transposed
state, a wrong layout, an off-by-one token loop. CPU only; the real oracle
source is never modified."""
import os
import tempfile

import pytest

from oracle import Oracle, compile_library
from oracle.oracle import SOURCE
from tests import pins

# (name, text in the oracle source, replacement, which occurrence)
MUTANTS = [
    ("no_relu_on_K",
     "double k = relu(K[at_bnhd(b, n, h, i, N, H, d)]);",
     "double k = K[at_bnhd(b, n, h, i, N, H, d)];", 0),
    ("no_relu_on_Q_den",
     "den += relu(Q[at_bnhd(b, n, h, i, N, H, d)])",
     "den += (Q[at_bnhd(b, n, h, i, N, H, d)])", 0),
    ("no_relu_on_Q_num",
     "num += relu(Q[at_bnhd(b, n, h, i, N, H, d)])",
     "num += (Q[at_bnhd(b, n, h, i, N, H, d)])", 0),
    ("relu_on_V",
     "k * V[at_bnhd(b, n, h, j, N, H, d)]",
     "k * relu(V[at_bnhd(b, n, h, j, N, H, d)])", 0),
    ("no_eps",
     "] = num / (den + eps);", "] = num / (den);", 0),
    ("eps_outside_division",
     "] = num / (den + eps);", "] = num / den + eps;", 0),
    ("normaliser_from_V",
     "S[at_state(b, h, i, d, H, d)] += k * 1.0;",
     "S[at_state(b, h, i, d, H, d)] += k * V[at_bnhd(b, n, h, 0, N, H, d)];", 0),
    ("den_from_column_0",
     "* S[at_state(b, h, i, d, H, d)];", "* S[at_state(b, h, i, 0, H, d)];", 0),
    ("transposed_state_in_apply",
     "* S[at_state(b, h, i, j, H, d)];", "* S[at_state(b, h, j, i, H, d)];", 0),
    ("token_loop_off_by_one",
     "for (long n = 0; n < N; ++n) {", "for (long n = 0; n < N - 1; ++n) {", 0),
    ("layout_BHNd",
     "return (((size_t)b * N + n) * H + h) * d + i;",
     "return (((size_t)b * H + h) * N + n) * d + i;", 0),
    ("den_skips_last_feature",
     "for (long i = 0; i < d; ++i)\n                    den +=",
     "for (long i = 0; i < d - 1; ++i)\n                    den +=", 0),
    ("K_from_head_0",
     "double k = relu(K[at_bnhd(b, n, h, i, N, H, d)]);",
     "double k = relu(K[at_bnhd(b, n, 0, i, N, H, d)]);", 0),
    ("num_skips_first_feature",
     "for (long i = 0; i < d; ++i)\n                        num +=",
     "for (long i = 1; i < d; ++i)\n                        num +=", 0),
    # block-causal form
    ("bc_no_relu_on_K",
     "double k = relu(K[at_bnhd(b, n, h, i, N, H, d)]);",
     "double k = K[at_bnhd(b, n, h, i, N, H, d)];", 1),
    ("bc_block_drops_last_token",
     "const long end = (j + 1) * L < N ? (j + 1) * L : N;",
     "const long end = (j + 1) * L - 1 < N ? (j + 1) * L - 1 : N;", 0),
    ("bc_block_skips_first_token",
     "for (long n = j * L; n < end; ++n) {",
     "for (long n = j * L + 1; n < end; ++n) {", 0),
    ("bc_query_uses_previous_block",
     "const long j = n / L;",
     "const long j = n / L > 0 ? n / L - 1 : 0;", 0),
    ("bc_query_uses_next_block",
     "const long j = n / L;",
     "const long j = n / L < nblk - 1 ? n / L + 1 : n / L;", 0),
    ("bc_den_from_column_0",
     "* P[at_prefix(b, h, j, i, d, H, nblk, d)];",
     "* P[at_prefix(b, h, j, i, 0, H, nblk, d)];", 0),
    ("bc_no_eps",
     "] = num / (den + eps);", "] = num / (den);", 1),
    # feature maps
    ("elu_without_plus_one",
     "return x > 0.0 ? x + 1.0 : exp(x);", "return x > 0.0 ? x : exp(x) - 1.0;", 0),
    ("elu_branch_at_wrong_side",
     "return x > 0.0 ? x + 1.0 : exp(x);", "return x > 0.0 ? exp(x) : x + 1.0;", 0),
    ("cos_as_sin",
     "return cos(x);", "return sin(x);", 0),
    ("fm_normaliser_without_key_feature",
     "S[at_state(b, h, i, d, H, d)] += k * 1.0;", "S[at_state(b, h, i, d, H, d)] += 1.0;", 1),
    ("fm_query_feature_ignored_in_num",
     "num += feature(Q[at_bnhd(b, n, h, i, N, H, d)], fm)",
     "num += (Q[at_bnhd(b, n, h, i, N, H, d)])", 0),
]


def _code_only(text):
    """the source with /* */ comments blanked, so patterns only match code"""
    out, i = [], 0
    while True:
        j = text.find("/*", i)
        if j < 0:
            out.append(text[i:])
            return "".join(out)
        k = text.index("*/", j) + 2
        out.append(text[i:j] + " " * (k - j))
        i = k


def _replace_nth(text, old, new, nth):
    code, start = _code_only(text), -1
    for _ in range(nth + 1):
        start = code.find(old, start + 1)
        assert start >= 0, f"pattern not found: {old!r}"
    return text[:start] + new + text[start + len(old):]


@pytest.fixture(scope="module")
def source_text():
    with open(SOURCE) as f:
        return f.read()


@pytest.fixture(scope="module")
def build_dir():
    # one directory alive for the whole module: dlopen matches libraries by
    # inode, so a deleted and reused file could hand back an earlier mutant
    with tempfile.TemporaryDirectory() as tmp:
        yield tmp


@pytest.mark.parametrize("name,old,new,nth", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(source_text, build_dir, name, old, new, nth):
    assert source_text.count(old) >= nth + 1, f"{name}: pattern missing from the oracle"
    mutated = _replace_nth(source_text, old, new, nth)
    assert mutated != source_text
    src = os.path.join(build_dir, f"{name}.c")
    with open(src, "w") as f:
        f.write(mutated)
    orc = Oracle(compile_library(src, os.path.join(build_dir, f"lib{name}.so")))
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, FloatingPointError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passes every pin"
