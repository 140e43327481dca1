"""Shared helpers of the GPU tests: move seeded inputs to the device, call the
C ABI through the binding, and compare with the fp64 oracle."""
import ctypes

import numpy as np
import torch

from gated_delta_rule_81_b200 import gdn

# Output tolerance: |y_gpu - y_ref| <= OUT_TOL * rms(y_ref) + BF16_ULP * |y_ref| element-wise.
# The first term is the mixer's arithmetic tolerance; the second is the bf16 output
# format's own rounding (one bf16 ulp of the value: no bf16 result can be closer to
# the fp64 value than half an ulp, and large outputs reach |y| ~ 20 rms).
OUT_TOL = 1e-2
BF16_ULP = 2.0 ** -8
STATE_TOL = 5e-3   # ||S_gpu - S_ref||_F / ||S_ref||_F <= STATE_TOL per sequence


def device_inputs(inp, dev="cuda"):
    """Copy the per-token inputs and parameters to the device; returns (keep, GdnInputs)."""
    keep = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in inp.items()}
    s = gdn.make_inputs(keep["q"], keep["k"], keep["v"], keep["a"], keep["b"], keep["z"], keep["conv_w"],
                        keep["A_log"], keep["norm_w"], scale=keep.get("scale", 1.0))
    return keep, s


def err_word(dev="cuda"):
    return torch.zeros(1, dtype=torch.int32, device=dev)


def out_error(y_gpu, y_ref, heads=None):
    """max over elements of (|y_gpu - y_ref| - BF16_ULP |y_ref|) / rms(y_ref): the
    arithmetic error beyond the output format's rounding, in units of rms(y_ref)."""
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    r = np.asarray(y_ref)
    if heads is not None:
        y, r = y[:, heads], r[:, heads]
    rms = np.sqrt(np.mean(r * r))
    return float(np.max(np.abs(y - r) - BF16_ULP * np.abs(r)) / rms)


def raw_out_error(y_gpu, y_ref, heads=None):
    """plain max |y_gpu - y_ref| / rms(y_ref), reported beside out_error"""
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    r = np.asarray(y_ref)
    if heads is not None:
        y, r = y[:, heads], r[:, heads]
    return float(np.max(np.abs(y - r)) / np.sqrt(np.mean(r * r)))


def state_error(S_gpu, S_ref, heads=None):
    """max over sequences of ||S_gpu - S_ref||_F / ||S_ref||_F."""
    s = S_gpu.double().cpu().numpy()
    r = np.asarray(S_ref)
    if heads is not None:
        s, r = s[:, heads], r[:, heads]
    num = np.sqrt(((s - r) ** 2).reshape(s.shape[0], -1).sum(1))
    den = np.sqrt((r ** 2).reshape(r.shape[0], -1).sum(1))
    den = np.where(den == 0, 1.0, den)
    return float(np.max(num / den))


def selftest_lib():
    from gated_delta_rule_81_b200 import build

    lib = ctypes.CDLL(build.lib_path("libgdn_selftest.so"))
    lib.gdn_selftest_umma.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.gdn_selftest_umma.restype = ctypes.c_int
    return lib
