"""Seeded, counter-based synthetic inputs shared by the tests, the oracle and the bench.

This module holds no attention arithmetic.  It defines one value per
(seed, tensor id, index) so that the host can regenerate any slice of a tensor
that the device filled, bit for bit, without copying it back:

    key      = mix64((seed << 32) ^ tensor_id ^ 0x5851F42D4C957F2D)
    word(c)  = mix64(key + (c + 1) * 0x9E3779B97F4A7C15)       (SplitMix64 stream)
    u_0..u_11 = the four 16-bit fields of word(3i), word(3i+1), word(3i+2)
    value(i) = bf16_rne( (sum(u) - 393210) * 2^-16 * sigma )

``mix64`` is the SplitMix64 output function (Steele, Lea and Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014; constants as in
Vigna's splitmix64.c).  The sum of twelve uniforms minus its mean is the
Irwin-Hall approximation of a unit normal (variance 12 * 1/12 = 1, range +-6).
sigma must be a power of two, so every step before the final bf16 rounding is
exact in float32 and both sides round the same float32 value.

Logical indexing (independent of any cache layout): the element of a
per-token tensor at (batch b, head h, absolute position p, dim d) has index
((b * H + h) * 2^20 + p) * D + d, with D = 1 for the gate logits.

The device implementation is ``synth/synth.cu`` (``libspark_synth.so``), which also holds a
read-only bandwidth probe for the bench (``read_probe_gbs``), no part of the generator.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
KEY_SALT = 0x5851F42D4C957F2D
MEAN12 = 393210            # 12 * 65535 / 2
POS_STRIDE = 1 << 20       # positions are < 2^20

# tensor roles; tensor_id = (layer << 8) | role
ROLE_Q, ROLE_K, ROLE_V, ROLE_GATE = 1, 2, 3, 4


def tensor_id(layer: int, role: int) -> int:
    return ((layer & 0xFFFFFF) << 8) | role


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    z ^= z >> np.uint64(30)
    z *= np.uint64(0xBF58476D1CE4E5B9)
    z ^= z >> np.uint64(27)
    z *= np.uint64(0x94D049BB133111EB)
    z ^= z >> np.uint64(31)
    return z


def _key(seed: int, tid: int) -> np.uint64:
    k = ((int(seed) << 32) ^ int(tid) ^ KEY_SALT) & M64
    return _mix64(np.array([k], dtype=np.uint64))[0]


def values_f32(seed: int, tid: int, index: np.ndarray, sigma: float = 1.0) -> np.ndarray:
    """float32 values before bf16 rounding, at the given flat indices."""
    m, e = np.frexp(sigma)
    if m != 0.5:
        raise ValueError("sigma must be a power of two")
    idx = np.asarray(index, dtype=np.uint64)
    key = _key(seed, tid)
    acc = np.zeros(idx.shape, dtype=np.int64)
    with np.errstate(over="ignore"):
        for r in range(3):
            c = idx * np.uint64(3) + np.uint64(r)
            w = _mix64(key + (c + np.uint64(1)) * np.uint64(GAMMA))
            for f in range(4):
                acc += ((w >> np.uint64(16 * f)) & np.uint64(0xFFFF)).astype(np.int64)
    return (acc - MEAN12).astype(np.float32) * np.float32(2.0 ** -16 * sigma)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even float32 -> bf16 bit patterns (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_values(seed: int, tid: int, index: np.ndarray, sigma: float = 1.0) -> np.ndarray:
    """bf16 bit patterns (uint16) at the given flat indices (large requests run on a thread pool)."""
    idx = np.asarray(index, dtype=np.uint64)
    n = idx.size
    chunk = 1 << 20
    if n <= 2 * chunk:
        return f32_to_bf16_bits(values_f32(seed, tid, idx, sigma))
    from concurrent.futures import ThreadPoolExecutor
    flat = idx.reshape(-1)
    out = np.empty(n, dtype=np.uint16)

    def work(lo):
        out[lo:lo + chunk] = f32_to_bf16_bits(values_f32(seed, tid, flat[lo:lo + chunk], sigma))

    with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(work, range(0, n, chunk)))
    return out.reshape(idx.shape)


def token_index(B: int, H: int, D: int, pos: np.ndarray, b_idx=None, h_idx=None) -> np.ndarray:
    """Flat indices [B, T, H, D] of a per-token tensor at absolute positions pos [B, T]."""
    pos = np.asarray(pos, dtype=np.uint64)
    if pos.ndim == 1:
        pos = np.broadcast_to(pos[None, :], (B, pos.shape[0]))
    b = np.arange(B, dtype=np.uint64)[:, None, None, None] if b_idx is None else np.asarray(b_idx, np.uint64)
    h = np.arange(H, dtype=np.uint64)[None, None, :, None] if h_idx is None else np.asarray(h_idx, np.uint64)
    d = np.arange(D, dtype=np.uint64)[None, None, None, :]
    p = pos[:, :, None, None]
    return ((b * np.uint64(H) + h) * np.uint64(POS_STRIDE) + p) * np.uint64(D) + d


def token_tensor(seed: int, tid: int, B: int, H: int, D: int, pos, sigma: float = 1.0) -> np.ndarray:
    """bf16 bits [B, T, H, D] (D=1 squeezed for gates) at absolute positions pos ([T] or [B, T])."""
    out = bf16_values(seed, tid, token_index(B, H, D, pos), sigma)
    return out[..., 0] if D == 1 else out


def head_slice(seed: int, tid: int, b: int, h: int, H: int, D: int, pos, sigma: float = 1.0) -> np.ndarray:
    """bf16 bits [n, D] of one (batch, head) row at the positions ``pos`` [n]."""
    pos = np.asarray(pos, dtype=np.uint64)
    idx = ((np.uint64(b) * np.uint64(H) + np.uint64(h)) * np.uint64(POS_STRIDE) + pos[:, None]) * np.uint64(D) \
        + np.arange(D, dtype=np.uint64)[None, :]
    return bf16_values(seed, tid, idx, sigma)


# ---------------------------------------------------------------------------
# Device side (libspark_synth.so, built from synth/synth.cu)
# ---------------------------------------------------------------------------

_LIB = None


def lib_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspark_synth.so")


def load_lib():
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build()")
        lib = ctypes.CDLL(path)
        lib.spark_synth_fill_tokens.restype = ctypes.c_int
        lib.spark_synth_fill_tokens.argtypes = [
            ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_longlong, ctypes.c_ulonglong, ctypes.c_ulonglong, ctypes.c_float, ctypes.c_void_p]
        lib.spark_synth_fill_cache.restype = ctypes.c_int
        lib.spark_synth_fill_cache.argtypes = [
            ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_longlong, ctypes.c_int, ctypes.c_ulonglong, ctypes.c_ulonglong, ctypes.c_float,
            ctypes.c_void_p]
        lib.spark_synth_read_probe.restype = ctypes.c_int
        lib.spark_synth_read_probe.argtypes = [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p, ctypes.c_int,
                                               ctypes.c_void_p]
        _LIB = lib
    return _LIB


def read_probe_gbs(n_bytes: int = 8 << 30, reps: int = 10, warmup: int = 3) -> float:
    """Read-only HBM bandwidth (GB/s, 1e9 B/s) of one stream over a device buffer of n_bytes (far
    larger than L2), best of `reps` launches timed with CUDA events on the current stream.  Bench
    infrastructure: the ceiling its HBM-bound kernels, which only read the KV cache, are held to."""
    import torch
    buf = torch.ones(n_bytes, dtype=torch.uint8, device="cuda")
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    lib = load_lib()
    st = _stream_ptr(None)

    def launch():
        if lib.spark_synth_read_probe(buf.data_ptr(), n_bytes, sink.data_ptr(), sms, st) != 0:
            raise RuntimeError("spark_synth_read_probe failed")

    for _ in range(warmup):
        launch()
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        launch()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del buf
    torch.cuda.empty_cache()
    return n_bytes / (best * 1e-3) / 1e9


def _stream_ptr(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def fill_tokens(t, seed: int, tid: int, pos0: int, sigma: float = 1.0, stream=None) -> None:
    """Fill a contiguous bf16 CUDA tensor [B, T, H, D] (or [B, T, H] for gates) in place."""
    if t.dim() == 3:
        B, T, H = t.shape
        D = 1
    else:
        B, T, H, D = t.shape
    rc = load_lib().spark_synth_fill_tokens(t.data_ptr(), B, T, H, D, pos0, seed, tid, sigma, _stream_ptr(stream))
    if rc != 0:
        raise RuntimeError(f"spark_synth_fill_tokens failed ({rc})")


def fill_cache(t, seed: int, tid: int, n_pos: int, ring: bool, sigma: float = 1.0, stream=None) -> None:
    """Fill a bf16 cache [B, Hkv, cap, D] holding positions 0..n_pos-1.

    Linear cache: row r holds position r (rows >= n_pos are zero).  Ring
    (cap = 512): row s holds the largest p < n_pos with p % cap == s (zero if
    none).  The value at a position is the generator's value at that position.
    """
    B, H, cap, D = t.shape
    rc = load_lib().spark_synth_fill_cache(t.data_ptr(), B, H, cap, D, n_pos, int(ring), seed, tid, sigma,
                                           _stream_ptr(stream))
    if rc != 0:
        raise RuntimeError(f"spark_synth_fill_cache failed ({rc})")
