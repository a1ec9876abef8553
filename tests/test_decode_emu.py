"""The decode kernel's own source run on the CPU (tests/emu: each CUDA
thread a host thread, warp-level instructions and barriers emulated, the
CTAs of a cluster together), built with AddressSanitizer and UBSan over
exactly sized buffers.  Any out-of-bounds or misaligned access of the
kernel's indexing fails the run; the outputs are compared with the fp64
decode oracle.  This checks the
indexing and the split/merge logic on shapes the GPU tests do not reach,
without a GPU."""

from __future__ import annotations

import os
import shutil
import subprocess
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle.decode as odec
from parity_util import check_bf16, check_lse

ROOT = Path(__file__).resolve().parents[1]
EMU = ROOT / "tests" / "emu"


@pytest.fixture(scope="module")
def emu_exe(tmp_path_factory):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = tmp_path_factory.mktemp("emu") / "decode_emu"
    cmd = [cxx, "-std=c++20", "-O1", "-g", "-fsanitize=address,undefined",
           "-fno-sanitize-recover=all", "-pthread", "-I", str(EMU / "include"), "-I", str(EMU),
           "-I", str(ROOT / "causal_self_attention_flash_b200" / "csrc"),
           str(EMU / "decode_emu.cpp"), "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        pytest.fail("emulator build failed:\n" + r.stderr[-3000:])
    return exe


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# (B, H, Tq, L, D, layout, CTAs per head (the cluster size) or None for
# attn_decode's own choice); a count below the number of chunks makes each
# CTA walk several chunks (the cross-chunk merge)
@pytest.mark.parametrize("B,H,Tq,L,D,layout,ctas", [
    (1, 1, 1, 1, 16, 0, None), (2, 2, 1, 300, 64, 0, None), (1, 2, 3, 257, 128, 1, None),
    (1, 1, 8, 8, 32, 0, None), (2, 1, 8, 513, 16, 1, None), (1, 3, 2, 256, 64, 1, None),
    (1, 1, 5, 1000, 128, 0, None), (1, 2, 4, 37, 64, 0, None), (2, 1, 2, 70, 32, 1, None),
    (1, 1, 7, 520, 64, 1, None), (1, 1, 1, 255, 128, 1, None), (3, 1, 6, 129, 16, 0, None),
    (1, 2, 1, 1000, 64, 0, 1), (1, 1, 4, 700, 128, 1, 3), (2, 1, 8, 1100, 32, 0, 2),
    (1, 1, 3, 600, 16, 1, 1),
    # the last CTA of the cluster holds only key 32, after rows 0-6's
    # positions: its partial for those rows is empty (m = -inf)
    (1, 1, 8, 33, 128, 0, None),
    # Tq = L: row 0 sees key 0 only
    (1, 2, 8, 8, 64, 1, None),
    # clusters of 5 and 4 CTAs (7 asked for: 8 chunks give runs of 2)
    (1, 1, 3, 1000, 64, 0, 5), (1, 1, 8, 900, 16, 1, 7)])
def test_decode_kernels_on_the_host(emu_exe, tmp_path, B, H, Tq, L, D, layout, ctas):
    g = torch.Generator().manual_seed(1000 * L + D + Tq)
    Tmax = L       # a tight cache: a read past row L - 1 leaves the buffer
    q = torch.randn(B, H, Tq, D, generator=g).to(torch.bfloat16)
    if layout == 0:
        kst = torch.randn(B, H, Tmax, D, generator=g).to(torch.bfloat16)
        vst = torch.randn(B, H, Tmax, D, generator=g).to(torch.bfloat16)
        k, v = kst, vst
    else:
        kst = torch.randn(B, Tmax, H, D, generator=g).to(torch.bfloat16)
        vst = torch.randn(B, Tmax, H, D, generator=g).to(torch.bfloat16)
        k, v = kst.transpose(1, 2), vst.transpose(1, 2)
    scale = D ** -0.5
    inp, out = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(inp, "wb") as f:
        for t in (q, kst, vst):
            f.write(bf16_bits(t).tobytes())
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=0")
    extra = [] if ctas is None else [str(ctas)]
    r = subprocess.run([str(emu_exe), str(B), str(H), str(Tq), str(L), str(D), str(Tmax),
                        str(layout), repr(scale), str(inp), str(out)] + extra,
                       capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    raw = np.fromfile(out, dtype=np.uint8)
    n = B * H * Tq * D
    o = from_bits(raw[:2 * n].view(np.uint16)).reshape(B, H, Tq, D)
    lse = raw[2 * n:].view(np.float32).astype(np.float64).reshape(B, H, Tq)
    as64 = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    ro, rl = odec.decode_attention(as64(q), as64(k), as64(v), scale, L)
    check_bf16("o", o, ro)
    check_lse(lse, rl)
