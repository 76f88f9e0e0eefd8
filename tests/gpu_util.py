"""Helpers for the GPU parity tests: numpy <-> CUDA tensors and checks."""
import numpy as np
import ml_dtypes
import torch

BF16 = ml_dtypes.bfloat16


def to_dev(a, device="cuda"):
    """numpy bf16 / fp32 array -> CUDA tensor with the same bits."""
    a = np.ascontiguousarray(a)
    if a.dtype == BF16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    if a.dtype in (np.float32, np.uint8, np.int64):
        return torch.from_numpy(a).to(device)
    raise TypeError(a.dtype)


def to_np(t):
    """CUDA tensor -> numpy with the same bits (bf16 as ml_dtypes.bfloat16)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(BF16)
    return t.numpy()


def assert_bits_equal(got, want, what):
    got = np.ascontiguousarray(got)
    want = np.ascontiguousarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    g = got.view(np.uint8).reshape(-1)
    w = want.view(np.uint8).reshape(-1)
    bad = np.nonzero(g != w)[0]
    assert bad.size == 0, "%s: %d bytes differ, first at %s (got %s, want %s)" % (
        what, bad.size, bad[:5], g[bad[:5]], w[bad[:5]])


def assert_f32_equal_or_both_nan(got, want, what):
    got = np.asarray(got, np.float32)
    want = np.asarray(want, np.float32)
    both_nan = np.isnan(got) & np.isnan(want)
    same = got.view(np.uint32) == want.view(np.uint32)
    bad = np.nonzero(~(same | both_nan))
    assert bad[0].size == 0, "%s: %d values differ, first %s: got %s want %s" % (
        what, bad[0].size, [b[:3] for b in bad], got[bad][:3], want[bad][:3])
