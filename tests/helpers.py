"""Shared helpers of the GPU parity tests: dtype round trips and the scaled
error metric.

Error metric.  Bi-WKV outputs are weighted means of v with signed v, so the
output can cancel to ~0 and a plain relative error is ill-posed.  The error
of wkv_t is therefore divided by S_t, the same weighted mean of |v| (eq. 5
weights), which bounds |wkv_t|; for gated outputs by sigma(r_t) * S_t.
"""
import numpy as np

TOL = {"f32": 1e-4, "bf16": 2e-2}


def torch_dtype(name):
    import torch
    return torch.float32 if name == "f32" else torch.bfloat16


def to_device(a, dtype_name, device="cuda"):
    """float64 numpy -> (device tensor in the I/O dtype, float64 numpy of the
    rounded values the device sees)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a)).to(torch_dtype(dtype_name))
    return t.to(device), t.to(torch.float64).numpy()


def vec_f32(a, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a)).to(torch.float32)
    return t.to(device), t.to(torch.float64).numpy()


def to_numpy(t):
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def scaled_error(got, want, scale):
    return float(np.max(np.abs(got - want) / np.maximum(scale, 1e-300)))


def biwkv_scale(oracle, k, v, w, u):
    """S_t: the eq. 5 weighted mean of |v| (computed by the RNN form)."""
    return oracle.biwkv_rnn(k, np.abs(v), w, u)


def plain_relative_error(got, want, floor=1e-6):
    """max |got - want| / max(|want|, floor): the plain relative error, for
    information (outputs that cancel to ~0 inflate it)."""
    return float(np.max(np.abs(got - want) / np.maximum(np.abs(want), floor)))
