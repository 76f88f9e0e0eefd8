"""The Python binding checks every caller-supplied buffer (dtype, contiguity,
element count, device) before a pointer reaches the C ABI, which cannot see
sizes. CPU only: the device check and the library are replaced by fakes, so
these tests show that a bad buffer raises and that no library call (hence no
launch) happens."""
import pytest
import torch

from mxfp4_block_quantization_quantizer_b200 import _binding as B


class FakeLib:
    """Records calls; every entry point returns MXFP4_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if not name.startswith("mxfp4_"):
            raise AttributeError(name)

        def fn(*args):
            self.calls.append(name)
            return 0
        return fn


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(B, "lib", lambda: lib)
    monkeypatch.setattr(B, "_on_device", lambda t, name, device=None: None)
    monkeypatch.setattr(B, "_stream", lambda device, stream=None: None)
    return lib


def u8(*shape):
    return torch.zeros(shape, dtype=torch.uint8)


X = torch.zeros((64, 96), dtype=torch.bfloat16)  # 6144 elements


def test_real_device_check_rejects_host_tensors():
    with pytest.raises(TypeError):
        B._on_device(torch.zeros(4), "t")
    with pytest.raises(TypeError):
        B._cuda2d(torch.zeros((2, 32)), "x")


def test_correct_buffers_reach_the_library(fake):
    B.quantize(X, out=(u8(64, 48), u8(64, 3)))
    B.quantize(X, axis=B.COLS, out=(u8(96, 32), u8(96, 2)))
    B.double_quantize(X, out=(u8(64, 48), u8(64, 3), u8(96, 32), u8(96, 2)))
    B.rht_quantize(X, out=(u8(64, 48), u8(64, 3), torch.zeros((64, 96))))
    B.dequantize(u8(64, 48), u8(64, 3), 64, 96, out=torch.zeros((64, 96), dtype=torch.bfloat16))
    assert fake.calls == ["mxfp4_quantize", "mxfp4_quantize", "mxfp4_double_quantize",
                          "mxfp4_rht_quantize", "mxfp4_dequantize"]


BAD_QUANT_OUTS = [
    (u8(64, 47), u8(64, 3)),                          # codes one column short
    (u8(64, 48), u8(64, 2)),                          # scales short
    (u8(64, 49), u8(64, 3)),                          # codes too long
    (torch.zeros((64, 48), dtype=torch.int16), u8(64, 3)),  # wrong dtype
    (u8(64, 96)[:, ::2], u8(64, 3)),                  # strided view of the right size
]


@pytest.mark.parametrize("out", BAD_QUANT_OUTS)
def test_quantize_rejects_bad_outputs(fake, out):
    with pytest.raises(ValueError):
        B.quantize(X, out=out)
    with pytest.raises(ValueError):
        B.quantize(X, oas=True, out=out)
    assert fake.calls == []


def test_double_quantize_rejects_bad_outputs(fake):
    good = [u8(64, 48), u8(64, 3), u8(96, 32), u8(96, 2)]
    for i in range(4):
        bad = list(good)
        bad[i] = u8(bad[i].numel() - 1)
        with pytest.raises(ValueError):
            B.double_quantize(X, out=tuple(bad))
    assert fake.calls == []


def test_rht_quantize_rejects_bad_outputs(fake):
    with pytest.raises(ValueError):
        B.rht_quantize(X, out=(u8(64, 48), u8(64, 3), torch.zeros((64, 95))))
    with pytest.raises(ValueError):
        B.rht_quantize(X, out=(u8(64, 48), u8(64, 3), torch.zeros((64, 96), dtype=torch.bfloat16)))
    with pytest.raises(ValueError):
        B.rht_quantize(X, out=(u8(64, 40), u8(64, 3), None))
    assert fake.calls == []


def test_dequantize_rejects_mismatched_inputs_and_outputs(fake):
    with pytest.raises(ValueError):   # codes do not hold rows*cols/2 bytes
        B.dequantize(u8(64, 47), u8(64, 3), 64, 96)
    with pytest.raises(ValueError):   # scales short
        B.dequantize(u8(64, 48), u8(64, 2), 64, 96)
    with pytest.raises(ValueError):   # rows/cols disagree with the buffers
        B.dequantize(u8(64, 48), u8(64, 3), 128, 96)
    with pytest.raises(ValueError):   # output too small
        B.dequantize(u8(64, 48), u8(64, 3), 64, 96,
                     out=torch.zeros((64, 95), dtype=torch.bfloat16))
    with pytest.raises(TypeError):    # output dtype the library cannot write
        B.dequantize(u8(64, 48), u8(64, 3), 64, 96, out=torch.zeros((64, 96), dtype=torch.float16))
    assert fake.calls == []


def test_qema_blocked_gemm_and_tracker_reject_bad_buffers(fake):
    w = torch.zeros((32, 64))
    with pytest.raises(ValueError):
        B.qema_quantize(w, torch.zeros((32, 64)), out=(u8(32, 31), u8(32, 2)))
    with pytest.raises(ValueError):
        B.scales_to_blocked(u8(130, 5), out=u8(256, 7))
    a, ab = u8(128, 64), u8(128, 4)
    with pytest.raises(ValueError):
        B.gemm(a, ab, a, ab, 128, out=torch.zeros((128, 127)))
    with pytest.raises(ValueError):
        B.osc_step(w, w.clone(), w.clone(), w.clone(),
                   n_flagged=torch.zeros(2, dtype=torch.int64))
    with pytest.raises(ValueError):
        B.qramp_step(w, w.clone(), w.clone(), w.clone(), w.clone(), w.clone(),
                     u8(32, 63), 0)
    with pytest.raises(ValueError):
        B.qramp_step(w, w.clone()[:, :32], w.clone(), w.clone(), w.clone(), w.clone(),
                     u8(32, 64), 0)
    assert fake.calls == []
    B.qramp_step(w, w.clone(), w.clone(), w.clone(), w.clone(), w.clone(), u8(32, 64), 0)
    fake.calls.clear()
    B.scales_to_blocked(u8(130, 5), out=u8(256, 8))
    B.gemm(a, ab, a, ab, 128, out=torch.zeros((128, 128)))
    assert fake.calls == ["mxfp4_scales_to_blocked", "mxfp4_gemm"]


def test_status_word_must_be_one_int32(fake):
    a, ab = u8(128, 64), u8(128, 4)
    for bad in (torch.zeros(2, dtype=torch.int32), torch.zeros(1, dtype=torch.int64),
                torch.zeros(1, dtype=torch.float32)):
        with pytest.raises(ValueError):
            B.gemm(a, ab, a, ab, 128, status=bad)
        with pytest.raises(ValueError):
            B.rht_quantize(X, status=bad)
    assert fake.calls == []
    B.gemm(a, ab, a, ab, 128, status=torch.zeros(1, dtype=torch.int32))
    B.rht_quantize(X, status=torch.zeros(1, dtype=torch.int32))
    assert fake.calls == ["mxfp4_gemm", "mxfp4_rht_quantize"]


def test_gemm_quantize_a_checks_its_buffers(fake):
    x = torch.zeros((128, 256), dtype=torch.bfloat16)
    bc, bb = u8(256, 128), u8(256, 8)
    with pytest.raises(TypeError):      # X must be bf16
        B.gemm_quantize_a(x.float(), bc, bb)
    with pytest.raises(ValueError):     # B codes of another k
        B.gemm_quantize_a(x, u8(256, 64), bb)
    with pytest.raises(ValueError):     # blocked scales short
        B.gemm_quantize_a(x, bc, u8(256, 7))
    with pytest.raises(ValueError):     # C short
        B.gemm_quantize_a(x, bc, bb, out=torch.zeros((128, 255)))
    with pytest.raises(ValueError):     # A codes short
        B.gemm_quantize_a(x, bc, bb, want_a=True,
                          out=(torch.zeros((128, 256)), u8(128, 127), u8(128, 8)))
    assert fake.calls == []
    c, ac, as_ = B.gemm_quantize_a(x, bc, bb, want_a=True)
    assert c.shape == (128, 256) and ac.shape == (128, 128) and as_.shape == (128, 8)
    assert fake.calls == ["mxfp4_gemm_quantize_a"]
