"""Host-side marshalling of the Python binding, without a GPU: the
wrappers are driven with stand-in device tensors and a recording stand-in
for the C library, to check that valid calls reach the right C entry point
with the right sizes, strides and flags, and that invalid ones stop in
Python first."""

from __future__ import annotations

import types

import pytest
import torch

import causal_self_attention_flash_b200 as cattn

DEV = torch.device("cuda", 0)


class FakeDev:
    """Duck-typed CUDA tensor: shape, strides, dtype, a fake address."""

    _next = 1 << 20

    def __init__(self, shape, dtype=torch.bfloat16, strides=None, ptr=None):
        self.shape = torch.Size(shape)
        if strides is None:
            strides, acc = [], 1
            for n in reversed(shape):
                strides.insert(0, acc)
                acc *= n
        self._strides = tuple(strides)
        self.dtype = dtype
        self.is_cuda = True
        self.device = DEV
        if ptr is None:
            ptr = FakeDev._next
            FakeDev._next += 1 << 30
        self._ptr = ptr

    def dim(self):
        return len(self.shape)

    def stride(self, i=None):
        return self._strides if i is None else self._strides[i]

    def is_contiguous(self):
        return self._strides == FakeDev(self.shape, self.dtype, ptr=0)._strides

    def data_ptr(self):
        return self._ptr

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n

    def element_size(self):
        return torch.tensor([], dtype=self.dtype).element_size()


class FakeLib:
    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name.endswith("_workspace_bytes") or name.startswith("cattn_"):
            return getattr(self.real, name)     # pure host functions: the real ones

        def record(*args):
            self.calls.append((name, args))
            return 0
        return record


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib(cattn.LIB)
    monkeypatch.setattr(cattn, "LIB", lib)
    monkeypatch.setattr(cattn.torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(cattn, "_stream", lambda s: 0)
    return lib


def bufs(B, H, T, D, dtype=torch.bfloat16):
    return FakeDev((B, H, T, D), dtype)


def test_contiguous_calls(fake):
    B, H, T, D = 2, 3, 100, 64
    q, k, v, do, o, olo = (bufs(B, H, T, D) for _ in range(6))
    lse = FakeDev((B, H, T), torch.float32)
    cattn.attn_fwd(q, k, v, 0.125, o=o, lse=lse)
    cattn.attn_fwd_ex(q, k, v, 0.125, o=o, lse=lse, o_lo=olo)
    ws = FakeDev((cattn.attn_bwd_workspace_bytes(B, H, T, D),), torch.uint8)
    dq, dk, dv = (bufs(B, H, T, D) for _ in range(3))
    cattn.attn_bwd(q, k, v, o, lse, do, 0.125, dq=dq, dk=dk, dv=dv, workspace=ws)
    f32 = [bufs(B, H, T, D, torch.float32) for _ in range(3)]
    cattn.attn_bwd(q, k, v, o, lse, do, 0.125, dq=f32[0], dk=f32[1], dv=f32[2], workspace=ws,
                   o_lo=olo, grad_dtype=torch.float32)
    names = [c[0] for c in fake.calls]
    assert names == ["attn_fwd", "attn_fwd_ex", "attn_bwd", "attn_bwd_ex"]
    args = fake.calls[3][1]
    assert args[8:12] == (B, H, T, D) and args[15] == 1          # fp32 gradients flag
    assert args[17] == ws.numel()                                # workspace bytes


def test_strided_and_dropout_calls(fake):
    B, H, T, D = 2, 4, 64, 32
    C = H * D
    qkv = FakeDev((B, T, 3 * C))
    # views of the fused projection: (B, H, T, D) with strides (T*3C, D, 3C, 1)
    q, k, v = (FakeDev((B, H, T, D), strides=(T * 3 * C, D, 3 * C, 1),
                       ptr=qkv.data_ptr() + 2 * i * C) for i in range(3))
    o = FakeDev((B, H, T, D), strides=(T * C, D, C, 1))
    lse = FakeDev((B, H, T), torch.float32)
    cattn.attn_fwd_strided(q, k, v, 0.2, o=o, lse=lse)
    drop = cattn.dropout_params(0.2, seed=7, offset=3)
    cattn.attn_fwd_strided(q, k, v, 0.2, o=o, lse=lse, dropout=drop)
    ws = FakeDev((cattn.attn_bwd_workspace_bytes(B, H, T, D),), torch.uint8)
    g = [FakeDev((B, H, T, D), strides=(T * 3 * C, D, 3 * C, 1)) for _ in range(3)]
    cattn.attn_bwd_strided(q, k, v, o, lse, o, 0.2, dq=g[0], dk=g[1], dv=g[2], workspace=ws)
    cattn.attn_bwd_strided(q, k, v, o, lse, o, 0.2, dq=g[0], dk=g[1], dv=g[2], workspace=ws,
                           dropout=drop)
    names = [c[0] for c in fake.calls]
    assert names == ["attn_fwd_strided", "attn_fwd_dropout", "attn_bwd_strided",
                     "attn_bwd_dropout"]
    lq = fake.calls[0][1][1]
    assert (lq.b, lq.h, lq.t) == (T * 3 * C, D, 3 * C)
    lo = fake.calls[0][1][12]
    assert (lo.b, lo.h, lo.t) == (T * C, D, C)


def test_strided_calls_reject_mismatches(fake):
    B, H, T, D = 1, 2, 32, 64
    q = bufs(B, H, T, D)
    lse = FakeDev((B, H, T), torch.float32)
    with pytest.raises(ValueError, match="k: expected shape"):
        cattn.attn_fwd_strided(q, bufs(B, H, T - 1, D), q, lse=lse, o=bufs(B, H, T, D))
    with pytest.raises(ValueError, match="o: expected shape"):
        cattn.attn_fwd_strided(q, q, q, o=bufs(B, H, 2 * T, D), lse=lse)
    with pytest.raises(ValueError, match="lse must have shape"):
        cattn.attn_bwd_strided(q, q, q, q, FakeDev((B, H, 2 * T), torch.float32), q,
                               dq=q, dk=q, dv=q)
    with pytest.raises(ValueError, match="dk: expected shape"):
        cattn.attn_bwd_strided(q, q, q, q, lse, q, dq=bufs(B, H, T, D),
                               dk=bufs(B, H, T, 32), dv=bufs(B, H, T, D))
    assert fake.calls == []


def test_decode_call(fake):
    B, H, Tmax, D, L, Tq = 2, 3, 300, 128, 257, 2
    cache = FakeDev((B, Tmax, H, D))
    k = FakeDev((B, H, Tmax, D), strides=(Tmax * H * D, D, H * D, 1), ptr=cache.data_ptr())
    q = bufs(B, H, Tq, D)
    o, lse = bufs(B, H, Tq, D), FakeDev((B, H, Tq), torch.float32)
    ws = FakeDev((cattn.attn_decode_workspace_bytes(B, H, Tq, L, D),), torch.uint8)
    cattn.attn_decode(q, k, k, L, o=o, lse=lse, workspace=ws)
    name, args = fake.calls[0]
    assert name == "attn_decode"
    assert args[7:12] == (B, H, Tq, L, D)
    assert (args[3].b, args[3].h, args[3].t) == (Tmax * H * D, D, H * D)
    assert args[16] == ws.numel()
    with pytest.raises(ValueError, match="fewer than L"):
        cattn.attn_decode(q, k, k, Tmax + 1, o=o, lse=lse, workspace=ws)
    with pytest.raises(ValueError, match="matching q"):
        cattn.attn_decode(q, FakeDev((B, H + 1, Tmax, D)), k, L, o=o, lse=lse, workspace=ws)


def test_status_word_readers_take_device_workspaces_only():
    """cattn_last_device_status and the workspace self-test read a backward
    workspace's status words: a host tensor is refused in Python, before
    any C call."""
    host_ws = torch.zeros(4096, dtype=torch.uint8)
    with pytest.raises(ValueError, match="device memory"):
        cattn.cattn_last_device_status(host_ws)
    with pytest.raises(ValueError, match="device memory"):
        cattn.cattn_selftest_wait_timeout(1000, workspace=host_ws)
