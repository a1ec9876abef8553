"""The kernels' dropout mask code (csrc/philox.cuh) built for the host and
checked without a GPU: the byte-wise threshold compare over every byte,
position and threshold, the interleaved keep-word order, and the keep bits
that keep16 and keep32_il draw, bit for bit against the dropout oracle."""

from __future__ import annotations

import shutil
import subprocess
from pathlib import Path

import numpy as np
import pytest

import oracle.dropout as odrop

ROOT = Path(__file__).resolve().parents[1]
EMU = ROOT / "tests" / "emu"


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    out = tmp_path_factory.mktemp("philox") / "philox_host"
    cmd = [cxx, "-std=c++17", "-O2", "-fsanitize=undefined", "-fno-sanitize-recover=all",
           "-I", str(ROOT / "causal_self_attention_flash_b200" / "csrc"),
           str(EMU / "philox_host.cpp"), "-o", str(out)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        pytest.fail("build failed:\n" + r.stderr[-3000:])
    return out


def test_byte_compare_and_interleaved_order(exe):
    r = subprocess.run([str(exe), "swar"], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr


def _bits(hexstr, T):
    v = int(hexstr, 16)
    return np.array([(v >> j) & 1 for j in range(T)], dtype=bool)


@pytest.mark.parametrize("B,H,T,seed,offset,p", [
    (1, 2, 100, 0x1234_5678_9ABC_DEF0, 7, 0.2),
    (2, 1, 64, 99, 0, 0.5),
    (1, 3, 48, (1 << 64) - 1, 0xFFFFFFFF, 0.9),
    (1, 1, 37, 5, 3, 0.1),
])
def test_kernel_keep_bits_match_oracle(exe, B, H, T, seed, offset, p):
    r = subprocess.run([str(exe), "mask", str(B), str(H), str(T), str(seed), str(offset), str(p)],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    lines = r.stdout.split("\n")
    rows = {}
    for ln in lines:
        if ln.strip():
            bh, i, a, b = ln.split()
            rows[(int(bh), int(i))] = (_bits(a, T), _bits(b, T))
    assert len(rows) == B * H * T
    for b in range(B):
        for h in range(H):
            want = odrop.keep_mask_head(b, h, H, T, p, seed, offset)
            for i in range(T):
                a, il = rows[(b * H + h, i)]
                assert np.array_equal(a, want[i]), (b, h, i, "keep16")
                assert np.array_equal(il, want[i]), (b, h, i, "keep32_il")
