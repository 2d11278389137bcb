"""The oracle's pins must catch plausible mistakes.

Each case copies attn_oracle.c to a temporary directory, plants one mistake
in the copy (a dropped term, a wrong sign, a swapped operand or index), builds
it, and reruns every pin of tests/test_oracle.py against the mutant.  The
committed oracle source is never modified.  Every mutant must fail at least
one pin; every planted change keeps memory accesses in bounds.
"""
import os
import re
import shutil
import tempfile

import pytest

import oracle
from tests import test_oracle as pins

# (name, function whose body is edited, old text, new text)
MUTANTS = [
    ("scores lose the scale", "row_probs", "p[j] = scale * dot;", "p[j] = dot;"),
    ("sum of exponentials skips the max", "row_probs",
     "l += exp(p[j] - m);", "l += exp(p[j]);"),
    ("probabilities not normalised", "row_probs",
     "p[j] = exp(p[j] - m) / l;", "p[j] = exp(p[j] - m);"),
    ("keys used as values", "fwd_row",
     "const double *vj = v + at(", "const double *vj = k + at("),
    ("LSE in base 2", "fwd_row", "*lse_out = m + log(l);", "*lse_out = m + log2(l);"),
    ("head and token strides swapped", "at",
     "(((size_t)b * N + n) * H + h)", "(((size_t)b * H + h) * N + n)"),
    ("dQ loses the scale", "oracle_attn_bwd_rows",
     "dqi[x] += scale * ds * kj[x];", "dqi[x] += ds * kj[x];"),
    ("D without the probabilities", "oracle_attn_bwd_rows", "Di += p[j] * dp[j];", "Di += dp[j];"),
    ("dS sign flipped", "oracle_attn_bwd_rows",
     "double ds = p[j] * (dp[j] - Di);", "double ds = p[j] * (Di - dp[j]);"),
    ("dV from dS instead of P", "oracle_attn_bwd_rows",
     "dvj[x] += p[j] * doi[x];", "dvj[x] += ds * doi[x];"),
    ("dK from K instead of Q", "oracle_attn_bwd_rows",
     "dkj[x] += scale * ds * qi[x];", "dkj[x] += scale * ds * kj[x];"),
    ("online sum not rescaled", "oracle_attn_fwd_online", "l[r] = l[r] * alpha;", "l[r] = l[r];"),
    ("online output not rescaled", "oracle_attn_fwd_online",
     "ar[x] = ar[x] * alpha;", "ar[x] = ar[x];"),
    ("online max never updated", "oracle_attn_fwd_online", "m[r] = m_new;", "(void)m_new;"),
    ("dS table without D", "oracle_attn_dscores",
     "row[j] = p[j] * (dp[j] - Di);", "row[j] = p[j] * dp[j];"),
    ("causal mask lets one future key through", "row_probs",
     "const int nk = causal ? i + 1 : N;", "const int nk = causal ? (i + 2 < N ? i + 2 : N) : N;"),
    ("causal mask hides the diagonal", "row_probs",
     "const int nk = causal ? i + 1 : N;", "const int nk = causal ? (i > 0 ? i : 1) : N;"),
    ("causal mask ignored by the backward", "oracle_attn_bwd_rows",
     "row_probs(q, k, b, h, i, N, H, d, scale, causal, p, &m, &l);",
     "row_probs(q, k, b, h, i, N, H, d, scale, 0, p, &m, &l);"),
]

# One representative argument set for each parametrised pin.
ARGS = {
    "check_online_recurrence_bit_equal_with_one_kv_block": [(7,)],
    "check_online_recurrence_bit_equal_when_max_is_in_first_block": [(7,)],
    "check_online_recurrence_equals_definition_to_rounding": [(16, 5)],
    "check_backward_matches_central_finite_differences": [(1, 5, 2, 3)],
}


def _function_span(src: str, name: str):
    m = re.search(r"^[^\n;]*\b" + re.escape(name) + r"\s*\([^;{]*\)\s*\{", src, flags=re.M)
    assert m, name
    depth, i = 0, m.end() - 1
    while True:
        if src[i] == "{":
            depth += 1
        elif src[i] == "}":
            depth -= 1
            if depth == 0:
                return m.start(), i + 1
        i += 1


def plant(src: str, func: str, old: str, new: str) -> str:
    a, b = _function_span(src, func)
    body = src[a:b]
    assert body.count(old) >= 1, (func, old)
    return src[:a] + body.replace(old, new) + src[b:]


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name,func,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_every_planted_mistake_fails_a_pin(workdir, name, func, old, new):
    src = open(oracle.SOURCE).read()
    mutated = plant(src, func, old, new)
    assert mutated != src
    tag = re.sub(r"\W+", "_", name)
    c_path = os.path.join(workdir, f"m_{tag}.c")
    with open(c_path, "w") as f:
        f.write(mutated)
    mutant = oracle.Oracle(oracle.compile_source(c_path, os.path.join(workdir, f"libm_{tag}.so")))
    caught = []
    for check in pins.CHECKS:
        for args in ARGS.get(check.__name__, [()]):
            try:
                check(mutant, *args)
            except AssertionError:
                caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake: {name}"


def test_unmodified_copy_passes_every_pin(workdir):
    # Control: the same build route with no mistake planted passes everything.
    c_path = os.path.join(workdir, "control.c")
    shutil.copy(oracle.SOURCE, c_path)
    ctrl = oracle.Oracle(oracle.compile_source(c_path, os.path.join(workdir, "libcontrol.so")))
    for check in pins.CHECKS:
        for args in ARGS.get(check.__name__, [()]):
            check(ctrl, *args)
