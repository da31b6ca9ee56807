"""Helpers for the GPU parity tests: move bf16 bit patterns to and from the
device and compare attention outputs against the oracle with the stated
tolerances (max |err| <= 2e-2, mean |err| <= 2e-3 on N(0,1) inputs; plus a
relative L2 error <= 1e-2, a stricter internal check)."""

import numpy as np
import pytest
import torch

from oracle import bf16_bits_to_f64

ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
ATTN_REL_L2 = 1e-2


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def to_dev(bits):
    a = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def to_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t):
    return bf16_bits_to_f64(to_bits(t))


def attn_errors(got, ref):
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    return float(err.max()), float(err.mean()), float(rel)


def assert_attn_close(got, ref, what=""):
    mx, mean, rel = attn_errors(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert mx <= ATTN_MAX_ABS, f"{what}: max abs err {mx:.3g}"
    assert mean <= ATTN_MEAN_ABS, f"{what}: mean abs err {mean:.3g}"
    assert rel <= ATTN_REL_L2, f"{what}: rel L2 err {rel:.3g}"
    return mx, mean, rel
