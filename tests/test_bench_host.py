"""Host-side arithmetic of bench.py (no GPU): the flop and byte
conventions of the measurement (causal counts; compulsory HBM bytes)."""

from __future__ import annotations

import importlib.util
from pathlib import Path

import pytest

from workloads import WORKLOADS

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_module", ROOT / "bench.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_causal_flop_convention(bench):
    w = WORKLOADS[2]  # GPT-2 124M layer, 16 x 12 x 1024 x 64
    fwd = 4 * w.B * w.H * w.T * w.T * w.D / 2
    assert bench.fwd_flops(w) == pytest.approx(fwd)
    assert bench.fwd_flops(w) == pytest.approx(25.77e9, rel=1e-3)
    assert bench.step_flops(w) == pytest.approx(3.5 * fwd)
    assert bench.step_flops(w) == pytest.approx(90.19e9, rel=1e-3)


def test_compulsory_bytes(bench):
    w = WORKLOADS[2]
    t = w.B * w.H * w.T * w.D * 2          # one bf16 (B,H,T,D) tensor: 25.17 MB
    v = w.B * w.H * w.T * 4                # one fp32 (B,H,T) vector: 0.79 MB
    # fwd: Q,K,V in, O + LSE out; pre: O, dO in, Delta out;
    # bwd: Q,K,V,dO,LSE,Delta in, dQ,dK,dV out
    assert bench.compulsory_bytes(w) == (3 * t + t + v) + (2 * t + v) + (4 * t + 2 * v + 3 * t)
    assert bench.compulsory_bytes(w) == pytest.approx(330e6, rel=0.01)


def test_kernel_algorithmic_units(bench):
    w = WORKLOADS[2]
    amount, unit, bound = bench.kernel_algorithmic(w, "bwd_kernel")
    assert (unit, bound) == ("flop", "tensor") and amount == pytest.approx(2.5 * bench.fwd_flops(w))
    amount, unit, bound = bench.kernel_algorithmic(w, "dq_convert_kernel")
    assert (unit, bound) == ("byte", "hbm")
    assert amount == w.B * w.H * w.T * w.D * 6   # fp32 read + bf16 write


def test_decode_bytes(bench):
    # GPT-2 layer as a cache: K and V of 16 x 12 heads x 1024 positions x 64
    # (bf16), plus one query row, one output row and one LSE per head
    kv = 2 * 16 * 12 * 1024 * 64 * 2
    assert bench.decode_bytes(16, 12, 1024, 64) == kv + 2 * 16 * 12 * 64 * 2 + 16 * 12 * 4
    assert bench.decode_bytes(16, 12, 1024, 64) == pytest.approx(50.4e6, rel=1e-3)
    assert bench.decode_bytes(1, 1, 1, 16, 1) == 2 * 16 * 2 + 2 * 16 * 2 + 4


def test_source_hash_ignores_comments_only(bench):
    a = "int f(int x) {  // doubles\n  return 2 * x;  /* twice */\n}\n"
    b = "// header\nint f(int x) {\n\n  return 2 * x;\n}\n"
    c = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(c)


def test_traffic_entries_are_well_formed(bench):
    """profiles/traffic.json: per kernel, DRAM bytes per launch = read +
    write, keyed to a code hash (bench.py reports the figure only while that
    hash matches the kernel's current code)"""
    import json
    import re as _re
    with open(bench.TRAFFIC_FILE) as f:
        tr = json.load(f)
    assert set(tr) == set(bench.KERNEL_SOURCES)
    for name, ent in tr.items():
        assert _re.fullmatch(r"[0-9a-f]{16}", ent["source_hash"]), name
        assert ent["bytes_per_launch"] == ent["dram_read_bytes"] + ent["dram_write_bytes"]
