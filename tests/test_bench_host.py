"""Host-side pieces of bench.py that need no GPU."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_tokens_ignore_comments_and_layout():
    a = 'int f(int x) {  // add one\n  return x + 1; /* done */\n}\n'
    b = '/* header\n   lines */\nint f(int x) {\n\n  return x + 1;\n}  // trailing\n'
    assert bench._code_tokens(a) == bench._code_tokens(b)
    # a code change is seen
    assert bench._code_tokens(a) != bench._code_tokens(a.replace("x + 1", "x + 2"))


def test_code_tokens_keep_string_literals():
    # comment markers inside string and character literals are code
    src = 'const char* s = "http://x /* y */"; char c = \'/\'; asm("a; // b");\n'
    toks = bench._code_tokens(src)
    assert '"http://x /* y */"' in toks and "'/'" in toks and '"a; // b"' in toks



def test_reference_arm_prints_the_gpu_arms_config(capsys):
    import argparse
    import json

    import attn_inputs
    w = attn_inputs.WORKLOADS["c1"]
    args = argparse.Namespace(steps=1, warmup=0, gpus=1)
    assert bench.run_reference(args, w, 0) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == bench.workload_config(w, 1)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1


def test_io_bytes_count_each_tensor_once():
    import attn_inputs
    w = attn_inputs.WORKLOADS["c4"]  # [1, 8192, 8, 128] bf16
    elems = 8192 * 8 * 128
    assert bench.io_bytes(w, False) == 4 * elems * 2 + 4 * 8 * 8192
    assert bench.io_bytes(w, True) == 8 * elems * 2 + 4 * 8 * 8192
    w8 = attn_inputs.WORKLOADS["c4fp8"]  # E4M3 in, bf16 O
    assert bench.io_bytes(w8, False) == 3 * elems + 2 * elems + 4 * 8 * 8192


def test_oracle_timing_whole_and_sampled():
    import attn_inputs
    whole = bench.oracle_time_config(attn_inputs.WORKLOADS["c1"], 1.0, single_core=True)
    assert whole["sample"] == "whole configuration"
    assert abs(whole["gflop"] - attn_inputs.WORKLOADS["c1"].fwd_flop / 1e9) < 1e-9
    assert whole["single_core"]["seconds"] > 0
    w = attn_inputs.WORKLOADS["sweep1024"]  # 2.15 GFLOP: sampled at a 0.5 GFLOP budget
    part = bench.oracle_time_config(w, 0.5, single_core=False)
    rows = int(1024 * 0.5e9 / w.fwd_flop)
    assert part["sample"] == f"query rows [0,{rows}) of all 8 heads"
    assert abs(part["gflop"] - 4.0 * rows * 1024 * 64 * 8 / 1e9) < 1e-9
    assert part["extrapolated_seconds"] > part["seconds"]
