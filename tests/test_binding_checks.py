"""The Python binding's argument checks: the C ABI sees only pointers, so the
binding refuses token tensors whose shapes, dtypes or devices disagree (an
output of the wrong size would be written past its end) and per-channel
vectors that are not float32[C].  These checks run before the library or the
GPU is touched, so they are tested here on stand-ins for CUDA tensors."""
import pytest
import torch

import linear_complexity_vision_b200 as vk


class FakeCuda:
    """Just enough of a CUDA tensor for the binding's checks."""

    def __init__(self, shape, dtype=torch.bfloat16, device="cuda:0", contiguous=True):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self.is_cuda = self.device.type == "cuda"
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous

    def dim(self):
        return len(self.shape)

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n


B, T, C = 2, 196, 64


def tok(**kw):
    return FakeCuda((B, T, C), **kw)


def vec(n=C, dtype=torch.float32, device="cuda:0"):
    return FakeCuda((n,), dtype=dtype, device=device)


def test_matching_token_tensors_pass():
    vk._require_tokens(("k", tok()), ("v", tok()), ("out", tok()))
    vk._require_vec(vec(), C, torch.device("cuda:0"), "w")


@pytest.mark.parametrize("bad,msg", [
    (FakeCuda((B, T, C + 8)), "shape"),
    (FakeCuda((B, T, C), dtype=torch.float32), "dtype"),
    (FakeCuda((B, T, C), device="cuda:1"), "device"),
    (FakeCuda((B * T, C)), r"\(B, T, C\)"),
    (FakeCuda((B, T, C), contiguous=False), "contiguous"),
    (FakeCuda((B, T, C), device="cpu"), "CUDA"),
])
def test_mismatched_token_tensors_are_refused(bad, msg):
    with pytest.raises(ValueError, match=msg):
        vk._require_tokens(("k", tok()), ("out", bad))


@pytest.mark.parametrize("bad", [vec(C + 1), vec(dtype=torch.bfloat16), vec(device="cuda:1")])
def test_per_channel_vectors_must_be_float32_of_length_c(bad):
    with pytest.raises(ValueError, match="float32 tensor of 64 elements"):
        vk._require_vec(bad, C, torch.device("cuda:0"), "w")


def test_qshift_mu_vectors_are_checked():
    assert vk._qs_ptr(None, C, torch.device("cuda:0")) is None
    qs = vk.QShift(14, 14, 1, 0.25, mu_r=vec(), mu_k=vec(C // 2), mu_v=None)
    with pytest.raises(ValueError, match="qs.mu_k"):
        vk._qs_ptr(qs, C, torch.device("cuda:0"))


def test_public_calls_refuse_before_launch():
    k, v = tok(), tok()
    with pytest.raises(ValueError, match="u must be a float32"):
        vk.biwkv_fwd(k, v, vec(), vec(C - 1))
    with pytest.raises(ValueError, match="out must match"):
        vk.spatial_gate(k, k, k, vec(), vec(), out=FakeCuda((B, T + 1, C)))
    with pytest.raises(ValueError, match="gy must match"):
        vk.biwkv_bwd(k, v, vec(), vec(), FakeCuda((B, T, C), dtype=torch.float32))
    with pytest.raises(ValueError, match="out must match"):
        vk.channel_mix(tok(), out=FakeCuda((B, T, C), dtype=torch.float32))
    with pytest.raises(ValueError, match="mu must be a float32"):
        vk.qshift(tok(), 14, 14, mu=vec(dtype=torch.float64))
    w4 = tuple(FakeCuda((C, C)) for _ in range(3)) + (FakeCuda((C, C + 1)),)
    with pytest.raises(ValueError, match=r"weights\[3\]"):
        vk.spatial_mix_block(tok(), w4, vec(), vec(), vec(), vec(), vk.QShift(14, 14))


def test_backward_outputs_are_checked():
    k, v, g = tok(), tok(), tok()
    good_rows = FakeCuda((B, C), dtype=torch.float32)
    with pytest.raises(ValueError, match="gv must match"):
        vk.biwkv_bwd(k, v, vec(), vec(), g, out=(tok(), FakeCuda((B, T, C + 8)), good_rows, good_rows))
    with pytest.raises(ValueError, match="gw must be a contiguous float32"):
        vk.biwkv_bwd(k, v, vec(), vec(), g, out=(tok(), tok(), FakeCuda((B, C)), good_rows))
    with pytest.raises(ValueError, match="gu must be a contiguous float32"):
        vk.biwkv_bwd(k, v, vec(), vec(), g, out=(tok(), tok(), good_rows, FakeCuda((B, C + 1), dtype=torch.float32)))

