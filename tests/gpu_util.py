"""Helpers shared by the GPU parity tests: moving generator output to the
device and comparing the CUDA path with the oracle."""
import numpy as np
import torch

import oracle


def dev_bytes(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def host_bytes(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint8)


def host_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def assert_gemv_close(y_gpu: torch.Tensor, y_ref: np.ndarray, S: np.ndarray, what=""):
    y = y_gpu.detach().cpu().numpy().astype(np.float64)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    err = np.abs(y - y_ref)
    tol = oracle.gemv_tolerance(S)
    ok = err <= tol
    if not ok.all():
        i = np.unravel_index(np.argmax(err / tol), err.shape)
        raise AssertionError(f"{what}: {int((~ok).sum())} of {ok.size} outside 2e-3*S+1e-5; "
                             f"worst at {i}: gpu={y[i]!r} ref={y_ref[i]!r} S={S[i]!r}")
    return float((err / tol).max()) if err.size else 0.0


ATTN_TOL = 3e-3


def assert_attn_close(out_gpu: torch.Tensor, ref: np.ndarray, what=""):
    o = out_gpu.detach().cpu().numpy().astype(np.float64)
    assert o.shape == ref.shape, (o.shape, ref.shape)
    err = np.abs(o - ref)
    if not (err <= ATTN_TOL).all():
        i = np.unravel_index(np.argmax(err), err.shape)
        raise AssertionError(f"{what}: max |err| {err.max():.3e} > {ATTN_TOL} at {i}: "
                             f"gpu={o[i]!r} ref={ref[i]!r}")
    return float(err.max()) if err.size else 0.0
