"""Shared helpers of the test suite (no attention arithmetic here)."""
import numpy as np

import synth

ATOL = 2e-2
RTOL = 2e-2


def to_dev(bits, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).astype(np.uint16).view(np.int16)).view(torch.bfloat16).to(device)


def dev_to_f64(t):
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def f64(bits):
    return synth.bf16_bits_to_f64(bits)


def assert_close(got, ref, what, atol=ATOL, rtol=RTOL):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    excess = np.abs(got - ref) - (atol + rtol * np.abs(ref))
    worst = np.unravel_index(np.argmax(excess), excess.shape)
    assert excess.max() <= 0, (f"{what}: |err| exceeds {atol} + {rtol}|ref| at {worst}: got {got[worst]:.6f} "
                               f"ref {ref[worst]:.6f} (max abs err {np.abs(got - ref).max():.3e})")
    return float(np.abs(got - ref).max())


def tid(layer, role):
    return synth.tensor_id(layer, role)
