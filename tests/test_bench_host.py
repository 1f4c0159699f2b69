"""bench.py's host logic on CPU: algorithmic byte counts per cache format, and the
reference arm (the oracle) for every format and option, as the driver launches it."""
import io
import json
import os
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from compressed_domain_attention_b200 import synthetic as syn  # noqa: E402


def test_byte_counts_per_format():
    w = syn.Workload("x", 2, 32, 8, 128, [1000, 300], None, 0, n_append=1)
    code = 64 + 8  # D/2 code bytes + D/32 binary16 scales
    lens = [1001, 301]
    assert bench.split_bytes(w, lens, "int4") == sum(lens) * 8 * 2 * code
    assert bench.split_bytes(w, lens, "fp16") == sum(lens) * 8 * (code + 256)
    assert bench.decode_bytes(w, lens, "fp16") == bench.split_bytes(w, lens, "fp16")
    # delegated: cold tokens as fp16 (binary16 K + int4 V), hot tokens binary16 K and V
    W, F = syn.DELEGATED_WINDOW, syn.DELEGATED_FOLD
    cold = [0 if n <= W else -(-(n - W) // F) * F for n in lens]
    assert [bench.cold_count(n, "delegated") for n in lens] == cold
    assert bench.split_bytes(w, lens, "delegated") == sum(cold) * 8 * (code + 256)
    hot = sum(n - c for n, c in zip(lens, cold))
    assert bench.decode_bytes(w, lens, "delegated") == sum(cold) * 8 * (code + 256) + hot * 8 * 512
    # appends: raw K and V in; codes or binary16 out; folds for the delegated cache
    assert bench.append_bytes(w, 2, "int4") == 2 * 8 * 2 * (256 + code)
    assert bench.append_bytes(w, 2, "fp16") == 2 * 8 * ((256 + code) + (256 + 256))
    folds = sum(bench.cold_count(n + 1, "delegated") - bench.cold_count(n, "delegated") for n in w.seq_lens)
    assert bench.append_bytes(w, 2, "delegated") == 2 * 8 * ((256 + 256) + (256 + 256)) + folds * 8 * (256 + code)


@pytest.mark.parametrize("flags", [[], ["--k-format", "fp16"], ["--k-format", "delegated"], ["--lambda"],
                                   ["--sparse-v", "1e-3"], ["--k-format", "fp16", "--lambda", "--sparse-v", "1e-6"]])
def test_reference_arm_runs_every_format(flags, monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "1", "--workload", "llama3_8b_layer",
                         *flags])
    assert rc == 0
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["gpu_launches"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    cfg = line["config"]
    assert cfg["k_format"] == (flags[flags.index("--k-format") + 1] if "--k-format" in flags else "int4")
    assert cfg["lambda"] == ("--lambda" in flags)
