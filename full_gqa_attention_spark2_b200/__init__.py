"""Python binding of libspark_attn.so: the Spark2_5 hybrid GQA attention core on B200.

Argument marshalling only.  Every step of the computation runs in the CUDA
kernels of libspark_attn.so (C ABI in include/spark_attn.h); there is no CPU
or PyTorch fallback, and a missing library raises at import of the first call.
PyTorch supplies device memory and streams.  The function names are the C
entry points'; tensors replace (pointer, size) pairs.
"""
from __future__ import annotations

import ctypes
import os

import torch

SPARK_SLIDING = 0
SPARK_FULL = 1
SPARK_ROPE_FUSED = 1
SPARK_APPEND_FUSED = 2
SPARK_STATIC_SCRATCH_BYTES = 16 << 20
N_LAYERS = 36
N_Q_HEADS = 16
N_KV_HEADS = 4
HEAD_DIM = 256
WINDOW = 512
MAX_POSITION = 1 << 20

_STATUS = {0: "OK", -1: "INVALID_ARG", -2: "UNSUPPORTED", -3: "CUDA", -4: "TIMEOUT", -5: "DEVICE_ARG"}


class SparkError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"spark status {status} ({_STATUS.get(status, '?')}): {message}")
        self.status = status


class SparkLayerCfg(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("window", ctypes.c_int), ("rot_dim", ctypes.c_int),
                ("n_q", ctypes.c_int), ("n_kv", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("theta", ctypes.c_double), ("scale", ctypes.c_float)]


_LIB = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_LL = ctypes.c_longlong


class SparkPagedKV(ctypes.Structure):
    """spark_paged_kv of include/spark_attn.h; keeps the tensors it points to alive."""
    _fields_ = [("k", _P), ("v", _P), ("k_scales", _P), ("v_scales", _P), ("block_table", _P),
                ("page_size", _I), ("n_pages", _I), ("max_pages", _I)]


def lib_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspark_attn.so")


def _lib():
    global _LIB
    if _LIB is not None:
        return _LIB
    path = lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing; build it with __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    cfgp = ctypes.POINTER(SparkLayerCfg)
    sig = {
        "spark_layer_cfg_for_layer": (_I, [_I, cfgp]),
        "spark_layer_cfg_for_kind": (_I, [_I, cfgp]),
        "spark_kv_cache_bytes": (ctypes.c_longlong, [cfgp, _I, ctypes.c_longlong]),
        "spark_stack_kv_bytes": (ctypes.c_longlong, [_I, ctypes.c_longlong]),
        "spark_rope_apply": (_I, [_P, _I, _I, _I, _LL, _LL, _P, cfgp, _P]),
        "spark_kv_append": (_I, [_P, _P, _I, _P, _P, _I, _I, _LL, _LL, _P, cfgp, ctypes.c_uint, _P]),
        "spark_attn_prefill": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _LL, _LL, _LL, _LL, _P, cfgp,
                                    ctypes.c_uint, _P]),
        "spark_decode_workspace_bytes": (ctypes.c_size_t, [_I, _I, cfgp]),
        "spark_attn_decode": (_I, [_P, _P, _LL, _P, _P, _P, _I, _I, _P, cfgp, _P, ctypes.c_size_t, ctypes.c_uint,
                                   _P]),
        "spark_attn_decode_static": (_I, [_P, _P, _P, _P, _P, _I, _I, _P, cfgp, ctypes.c_uint, _P]),
        "spark_decode_fused_workspace_bytes": (ctypes.c_size_t, [_I, _I, cfgp]),
        "spark_attn_decode_fused": (_I, [_P, _P, _LL, _P, _P, _LL, _P, _P, _P, _I, _I, _P, cfgp, _P,
                                         ctypes.c_size_t, ctypes.c_uint, _P]),
        "spark_decode_static_plan": (ctypes.c_size_t, [_I, _I, cfgp, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
        "spark_kv_cache_q8_bytes": (ctypes.c_longlong, [cfgp, _I, ctypes.c_longlong]),
        "spark_kv_append_q8": (_I, [_P, _P, _P, _P, _I, _P, _P, _I, _I, _P, cfgp, ctypes.c_uint, _P]),
        "spark_decode_q8_workspace_bytes": (ctypes.c_size_t, [_I, _I, cfgp]),
        "spark_attn_decode_q8": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _P, cfgp, _P, ctypes.c_size_t,
                                      ctypes.c_uint, _P]),
        "spark_prefill_q8_workspace_bytes": (ctypes.c_size_t, [_I, _I, cfgp]),
        "spark_attn_prefill_q8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _LL, _LL, _LL, _LL, _P, cfgp,
                                       _P, ctypes.c_size_t, ctypes.c_uint, _P]),
        "spark_kv_append_paged": (_I, [ctypes.POINTER(SparkPagedKV), _P, _P, _I, _I, _P, cfgp, ctypes.c_uint, _P]),
        "spark_decode_paged_workspace_bytes": (ctypes.c_size_t, [_I, ctypes.POINTER(SparkPagedKV), cfgp]),
        "spark_attn_decode_paged": (_I, [_P, _P, _P, ctypes.POINTER(SparkPagedKV), _I, _P, cfgp, _P,
                                         ctypes.c_size_t, ctypes.c_uint, _P]),
        "spark_rope_apply_varlen": (_I, [_P, _I, _P, _I, _P, _I, cfgp, _P]),
        "spark_kv_append_varlen": (_I, [ctypes.POINTER(SparkPagedKV), _P, _P, _P, _I, _P, _I, cfgp, ctypes.c_uint,
                                        _P]),
        "spark_attn_prefill_varlen": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _P, ctypes.POINTER(SparkPagedKV), _I,
                                           cfgp, ctypes.c_uint, _P]),
        "spark_decode_cp_record_bytes": (ctypes.c_size_t, [_I]),
        "spark_kv_append_cp": (_I, [_P, _P, _I, _I, _P, _P, _I, _P, cfgp, ctypes.c_uint, _P]),
        "spark_attn_decode_cp_partial": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, cfgp, _P, ctypes.c_size_t,
                                              ctypes.c_uint, _P]),
        "spark_attn_decode_cp_merge": (_I, [_P, _P, _P, _I, _I, _P]),
        "spark_selftest_wait_timeout": (_I, [ctypes.c_ulonglong, _P]),
        "spark_check": (_I, [_P]),
        "spark_last_error": (ctypes.c_char_p, []),
        "spark_version": (_I, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def exported_symbols():
    """Names of the C entry points this binding expects the library to export."""
    return ["spark_layer_cfg_for_layer", "spark_layer_cfg_for_kind", "spark_kv_cache_bytes",
            "spark_stack_kv_bytes", "spark_rope_apply", "spark_kv_append", "spark_attn_prefill",
            "spark_decode_workspace_bytes", "spark_attn_decode", "spark_attn_decode_static", "spark_decode_static_plan",
            "spark_decode_fused_workspace_bytes", "spark_attn_decode_fused",
            "spark_kv_cache_q8_bytes", "spark_kv_append_q8", "spark_decode_q8_workspace_bytes",
            "spark_attn_decode_q8", "spark_prefill_q8_workspace_bytes", "spark_attn_prefill_q8",
            "spark_kv_append_paged", "spark_decode_paged_workspace_bytes",
            "spark_attn_decode_paged", "spark_rope_apply_varlen", "spark_kv_append_varlen",
            "spark_attn_prefill_varlen", "spark_decode_cp_record_bytes", "spark_kv_append_cp",
            "spark_attn_decode_cp_partial", "spark_attn_decode_cp_merge", "spark_selftest_wait_timeout",
            "spark_check", "spark_last_error", "spark_version"]


def _raise(rc: int):
    if rc != 0:
        raise SparkError(rc, spark_last_error())


def spark_last_error() -> str:
    return _lib().spark_last_error().decode(errors="replace")


def spark_version() -> int:
    return _lib().spark_version()


def spark_layer_cfg_for_layer(layer: int) -> SparkLayerCfg:
    c = SparkLayerCfg()
    _raise(_lib().spark_layer_cfg_for_layer(layer, ctypes.byref(c)))
    return c


def spark_layer_cfg_for_kind(kind: int) -> SparkLayerCfg:
    c = SparkLayerCfg()
    _raise(_lib().spark_layer_cfg_for_kind(kind, ctypes.byref(c)))
    return c


def spark_kv_cache_bytes(cfg: SparkLayerCfg, B: int, cap: int) -> int:
    return int(_lib().spark_kv_cache_bytes(ctypes.byref(cfg), B, cap))


def spark_stack_kv_bytes(B: int, ctx: int) -> int:
    return int(_lib().spark_stack_kv_bytes(B, ctx))


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=torch.bfloat16, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    return t.data_ptr()


def _tokens(t: torch.Tensor, name: str, heads: int, ndim: int = 4):
    """Pointer and (sequence, token) element strides of a bf16 token tensor [B, T, heads, 256] (ndim 4)
    or [B, heads, 256] (ndim 3, token stride 0) whose heads are contiguous rows of 256: a view of a
    wider projection output is accepted."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be torch.bfloat16, got {t.dtype}")
    if t.dim() != ndim or t.shape[-1] != 256 or t.shape[-2] != heads:
        raise ValueError(f"{name} must be [{'B, T, ' if ndim == 4 else 'B, '}{heads}, 256], got {tuple(t.shape)}")
    if t.stride(-1) != 1 or (heads > 1 and t.stride(-2) != 256):
        raise ValueError(f"{name}: heads must be contiguous rows of 256 elements")
    return t.data_ptr(), t.stride(0), (t.stride(1) if ndim == 4 else 0)


def spark_rope_apply(x: torch.Tensor, pos0: torch.Tensor, cfg: SparkLayerCfg, stream=None) -> None:
    """Rotate x [B, T, H, 256] bf16 in place (a strided view is allowed); token t of sequence b is at
    pos0[b] + t."""
    B, T, H = x.shape[0], x.shape[1], x.shape[2] if x.dim() == 4 else 0
    px, sB, sT = _tokens(x, "x", H)
    pp = _dev(pos0, "pos0", torch.int32, 1)
    _raise(_lib().spark_rope_apply(px, B, T, H, sB, sT, pp, ctypes.byref(cfg), _stream(stream)))


def spark_kv_append(k_cache, v_cache, k, v, pos0, cfg: SparkLayerCfg, flags: int = 0, stream=None) -> None:
    """Append k, v [B, T, 4, 256] (views with the same strides allowed) at positions pos0[b] + t into
    caches [B, 4, cap, 256]."""
    pkc, pvc = _dev(k_cache, "k_cache", ndim=4), _dev(v_cache, "v_cache", ndim=4)
    pk, sB, sT = _tokens(k, "k", 4)
    pv, vB, vT = _tokens(v, "v", 4)
    if (vB, vT) != (sB, sT) or k.shape != v.shape:
        raise ValueError("k and v must have the same shape and strides")
    pp = _dev(pos0, "pos0", torch.int32, 1)
    B, T = k.shape[0], k.shape[1]
    cap = k_cache.shape[2]
    _raise(_lib().spark_kv_append(pkc, pvc, cap, pk, pv, B, T, sB, sT, pp, ctypes.byref(cfg), flags,
                                  _stream(stream)))


def spark_attn_prefill(out, q, k, v, gate, k_cache, v_cache, pos0, cfg: SparkLayerCfg, flags: int = 0,
                       stream=None) -> None:
    """Gated GQA attention of a chunk of T queries per sequence (see include/spark_attn.h).  q, k, v may
    be strided views (e.g. slices of one fused projection output); out and gate are dense."""
    po = _dev(out, "out", ndim=4)
    pq, q_sB, q_sT = _tokens(q, "q", 16)
    pk, kv_sB, kv_sT = _tokens(k, "k", 4)
    pv, vB, vT = _tokens(v, "v", 4)
    if (vB, vT) != (kv_sB, kv_sT) or k.shape != v.shape or tuple(q.shape[:2]) != tuple(k.shape[:2]):
        raise ValueError("k and v must have the same shape and strides, and q the same [B, T]")
    pg = _dev(gate, "gate", ndim=3)
    pp = _dev(pos0, "pos0", torch.int32, 1)
    if k_cache is None:
        pkc = pvc = None
        cap = 0
    else:
        pkc, pvc = _dev(k_cache, "k_cache", ndim=4), _dev(v_cache, "v_cache", ndim=4)
        cap = k_cache.shape[2]
    B, T = q.shape[0], q.shape[1]
    _raise(_lib().spark_attn_prefill(po, pq, pk, pv, pg, pkc, pvc, cap, B, T, q_sB, q_sT, kv_sB, kv_sT, pp,
                                     ctypes.byref(cfg), flags, _stream(stream)))


def spark_decode_cp_record_bytes(B: int) -> int:
    """Bytes of one rank's context-parallel decode record for B sequences."""
    return int(_lib().spark_decode_cp_record_bytes(B))


def spark_kv_append_cp(k_cache, v_cache, key_off: int, k, v, pos, cfg: SparkLayerCfg, flags: int = 0,
                       stream=None) -> None:
    """Append k, v [B, 4, 256] at pos[b] into a rank's shard [B, 4, cap, 256] holding positions key_off.. (rows
    outside the shard are skipped)."""
    pkc, pvc = _dev(k_cache, "k_cache", ndim=4), _dev(v_cache, "v_cache", ndim=4)
    pk, pv = _dev(k, "k", ndim=3), _dev(v, "v", ndim=3)
    pp = _dev(pos, "pos", torch.int32, 1)
    _raise(_lib().spark_kv_append_cp(pkc, pvc, k_cache.shape[2], key_off, pk, pv, k.shape[0], pp, ctypes.byref(cfg),
                                     flags, _stream(stream)))


def spark_attn_decode_cp_partial(record, q, k_cache, v_cache, key_off: int, pos, cfg: SparkLayerCfg,
                                 workspace: torch.Tensor, flags: int = 0, stream=None) -> None:
    """A rank's record (fp32, spark_decode_cp_record_bytes(B) bytes) of decode over its shard of a full layer."""
    pr = _dev(record, "record", torch.float32)
    if record.numel() * 4 < spark_decode_cp_record_bytes(q.shape[0]):
        raise ValueError("record is too small")
    pq = _dev(q, "q", ndim=3)
    pkc, pvc = _dev(k_cache, "k_cache", ndim=4), _dev(v_cache, "v_cache", ndim=4)
    pp = _dev(pos, "pos", torch.int32, 1)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    _raise(_lib().spark_attn_decode_cp_partial(pr, pq, pkc, pvc, k_cache.shape[2], key_off, q.shape[0], pp,
                                               ctypes.byref(cfg), workspace.data_ptr(),
                                               workspace.numel() * workspace.element_size(), flags,
                                               _stream(stream)))


def spark_attn_decode_cp_merge(out, gate, records, stream=None) -> None:
    """out [B, 16, 256] from the records of G ranks (records: fp32 [G, record floats], rank order)."""
    po, pg = _dev(out, "out", ndim=3), _dev(gate, "gate", ndim=2)
    prs = _dev(records, "records", torch.float32, 2)
    B = out.shape[0]
    if records.shape[1] * 4 != spark_decode_cp_record_bytes(B):
        raise ValueError("records must be [G, spark_decode_cp_record_bytes(B) / 4]")
    _raise(_lib().spark_attn_decode_cp_merge(po, pg, prs, records.shape[0], B, _stream(stream)))


def spark_decode_workspace_bytes(B: int, cap: int, cfg: SparkLayerCfg) -> int:
    return int(_lib().spark_decode_workspace_bytes(B, cap, ctypes.byref(cfg)))


def spark_attn_decode(out, q, gate, k_cache, v_cache, pos, cfg: SparkLayerCfg, workspace: torch.Tensor,
                      flags: int = 0, stream=None) -> None:
    """Attention of one new token per sequence at pos[b] (its k/v already appended); q [B, 16, 256] may be
    a view with any sequence stride."""
    po = _dev(out, "out", ndim=3)
    pq, q_sB, _ = _tokens(q, "q", 16, ndim=3)
    pg = _dev(gate, "gate", ndim=2)
    pkc, pvc = _dev(k_cache, "k_cache", ndim=4), _dev(v_cache, "v_cache", ndim=4)
    pp = _dev(pos, "pos", torch.int32, 1)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    B = q.shape[0]
    cap = k_cache.shape[2]
    _raise(_lib().spark_attn_decode(po, pq, q_sB, pg, pkc, pvc, cap, B, pp, ctypes.byref(cfg),
                                    workspace.data_ptr(), ws_bytes, flags, _stream(stream)))


def spark_decode_fused_workspace_bytes(B: int, cap: int, cfg: SparkLayerCfg) -> int:
    return int(_lib().spark_decode_fused_workspace_bytes(B, cap, ctypes.byref(cfg)))


def spark_decode_fused_workspace(B: int, cap: int, cfg: SparkLayerCfg, device="cuda"):
    """A zero-filled workspace for spark_attn_decode_fused (it must hold zeros before its first use)."""
    return torch.zeros(spark_decode_fused_workspace_bytes(B, cap, cfg), dtype=torch.uint8, device=device)


def spark_attn_decode_fused(out, q, k, v, gate, k_cache, v_cache, pos, cfg: SparkLayerCfg, workspace,
                            flags: int = 0, stream=None) -> None:
    """Append the new token (k, v [B, 4, 256] or [B, 1, 4, 256]) and attend q [B, 16, 256] in one launch
    (see include/spark_attn.h); workspace from spark_decode_fused_workspace."""
    po = _dev(out, "out", ndim=3)
    pq, q_sB, _ = _tokens(q, "q", 16, ndim=3)
    if k.dim() == 4:
        k, v = k[:, 0], v[:, 0]
    pk, kv_sB, _ = _tokens(k, "k", 4, ndim=3)
    pv, v_sB, _ = _tokens(v, "v", 4, ndim=3)
    if v_sB != kv_sB:
        raise ValueError("k and v must have the same strides")
    pg = _dev(gate, "gate", ndim=2)
    pkc, pvc = _dev(k_cache, "k_cache", ndim=4), _dev(v_cache, "v_cache", ndim=4)
    pp = _dev(pos, "pos", torch.int32, 1)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    _raise(_lib().spark_attn_decode_fused(po, pq, q_sB, pk, pv, kv_sB, pg, pkc, pvc, k_cache.shape[2], q.shape[0],
                                          pp, ctypes.byref(cfg), workspace.data_ptr(), ws_bytes, flags,
                                          _stream(stream)))


def spark_attn_decode_static(out, q, gate, k_cache, v_cache, pos, cfg: SparkLayerCfg, flags: int = 0,
                             stream=None) -> None:
    """Decode like spark_attn_decode, but without a workspace: for callers that cannot allocate.

    The split partials live in the library's fixed device scratch array, shared
    by all calls; calls that overlap on the device race on it."""
    po, pq = _dev(out, "out", ndim=3), _dev(q, "q", ndim=3)
    pg = _dev(gate, "gate", ndim=2)
    pkc, pvc = _dev(k_cache, "k_cache", ndim=4), _dev(v_cache, "v_cache", ndim=4)
    pp = _dev(pos, "pos", torch.int32, 1)
    _raise(_lib().spark_attn_decode_static(po, pq, pg, pkc, pvc, k_cache.shape[2], q.shape[0], pp,
                                           ctypes.byref(cfg), flags, _stream(stream)))


def spark_decode_static_plan(B: int, cap: int, cfg: SparkLayerCfg, sm_count: int = 148):
    """(n_splits, tiles_per_split, bytes) of spark_attn_decode_static's split plan; bytes is 0 on bad
    arguments or a batch above the scratch array's limit."""
    ns, tps = _I(0), _I(0)
    nbytes = _lib().spark_decode_static_plan(B, cap, ctypes.byref(cfg), sm_count, ctypes.byref(ns), ctypes.byref(tps))
    return ns.value, tps.value, int(nbytes)


def spark_kv_cache_q8_bytes(cfg: SparkLayerCfg, B: int, cap: int) -> int:
    return int(_lib().spark_kv_cache_q8_bytes(ctypes.byref(cfg), B, cap))


def _q8_pair(codes, scales, name):
    pc = _dev(codes, f"{name}_codes", torch.uint8, 4)
    ps = _dev(scales, f"{name}_scales", torch.float16, 4)
    if tuple(scales.shape) != tuple(codes.shape[:3]) + (codes.shape[3] // 32,):
        raise ValueError(f"{name}_scales must be [B, 4, cap, 8] beside codes [B, 4, cap, 256]")
    return pc, ps


def spark_kv_append_q8(k_codes, k_scales, v_codes, v_scales, k, v, pos0, cfg: SparkLayerCfg, flags: int = 0,
                       stream=None) -> None:
    """Quantise and append k, v [B, T, 4, 256] bf16 into 8-bit caches: codes uint8 [B, 4, cap, 256] and
    scales float16 [B, 4, cap, 8] (see include/spark_attn.h)."""
    pkc, pks = _q8_pair(k_codes, k_scales, "k")
    pvc, pvs = _q8_pair(v_codes, v_scales, "v")
    pk, pv = _dev(k, "k", ndim=4), _dev(v, "v", ndim=4)
    pp = _dev(pos0, "pos0", torch.int32, 1)
    B, T = k.shape[0], k.shape[1]
    _raise(_lib().spark_kv_append_q8(pkc, pks, pvc, pvs, k_codes.shape[2], pk, pv, B, T, pp, ctypes.byref(cfg),
                                     flags, _stream(stream)))


def spark_decode_q8_workspace_bytes(B: int, cap: int, cfg: SparkLayerCfg) -> int:
    return int(_lib().spark_decode_q8_workspace_bytes(B, cap, ctypes.byref(cfg)))


def spark_attn_decode_q8(out, q, gate, k_codes, k_scales, v_codes, v_scales, pos, cfg: SparkLayerCfg,
                         workspace: torch.Tensor, flags: int = 0, stream=None) -> None:
    """spark_attn_decode over 8-bit caches (codes + scales per K and V)."""
    po, pq = _dev(out, "out", ndim=3), _dev(q, "q", ndim=3)
    pg = _dev(gate, "gate", ndim=2)
    pkc, pks = _q8_pair(k_codes, k_scales, "k")
    pvc, pvs = _q8_pair(v_codes, v_scales, "v")
    pp = _dev(pos, "pos", torch.int32, 1)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    _raise(_lib().spark_attn_decode_q8(po, pq, pg, pkc, pks, pvc, pvs, k_codes.shape[2], q.shape[0], pp,
                                       ctypes.byref(cfg), workspace.data_ptr(), ws_bytes, flags,
                                       _stream(stream)))


def spark_prefill_q8_workspace_bytes(B: int, cap: int, cfg: SparkLayerCfg) -> int:
    return int(_lib().spark_prefill_q8_workspace_bytes(B, cap, ctypes.byref(cfg)))


def spark_attn_prefill_q8(out, q, k, v, gate, k_codes, k_scales, v_codes, v_scales, pos0, cfg: SparkLayerCfg,
                          workspace: torch.Tensor, flags: int = 0, stream=None) -> None:
    """spark_attn_prefill with the history in 8-bit caches (codes + scales per K and V); workspace: a
    contiguous CUDA tensor of at least spark_prefill_q8_workspace_bytes(B, cap, cfg) bytes."""
    po = _dev(out, "out", ndim=4)
    pq, q_sB, q_sT = _tokens(q, "q", 16)
    pk, kv_sB, kv_sT = _tokens(k, "k", 4)
    pv, vB, vT = _tokens(v, "v", 4)
    if (vB, vT) != (kv_sB, kv_sT) or k.shape != v.shape or tuple(q.shape[:2]) != tuple(k.shape[:2]):
        raise ValueError("k and v must have the same shape and strides, and q the same [B, T]")
    pg = _dev(gate, "gate", ndim=3)
    pp = _dev(pos0, "pos0", torch.int32, 1)
    pkc, pks = _q8_pair(k_codes, k_scales, "k")
    pvc, pvs = _q8_pair(v_codes, v_scales, "v")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    B, T = q.shape[0], q.shape[1]
    _raise(_lib().spark_attn_prefill_q8(po, pq, pk, pv, pg, pkc, pks, pvc, pvs, k_codes.shape[2], B, T, q_sB, q_sT,
                                        kv_sB, kv_sT, pp, ctypes.byref(cfg), workspace.data_ptr(), ws_bytes, flags,
                                        _stream(stream)))


def paged_kv(k_pool, v_pool, block_table, k_scales=None, v_scales=None) -> SparkPagedKV:
    """Describe one layer's paged K/V: pools [n_pages, 4, page_size, 256] (bf16, or uint8 codes with
    float16 scales [n_pages, 4, page_size, 8]) and block_table int32 [B, max_pages]."""
    q8 = k_scales is not None
    dt = torch.uint8 if q8 else torch.bfloat16
    pk, pv = _dev(k_pool, "k_pool", dt, 4), _dev(v_pool, "v_pool", dt, 4)
    pt = _dev(block_table, "block_table", torch.int32, 2)
    if tuple(v_pool.shape) != tuple(k_pool.shape) or k_pool.shape[1] != 4 or k_pool.shape[3] != 256:
        raise ValueError("pools must be [n_pages, 4, page_size, 256]")
    pks = pvs = None
    if q8:
        pks, pvs = _q8_pair(k_pool, k_scales, "k")[1], _q8_pair(v_pool, v_scales, "v")[1]
    kv = SparkPagedKV(pk, pv, pks, pvs, pt, k_pool.shape[2], k_pool.shape[0], block_table.shape[1])
    kv._keep = (k_pool, v_pool, block_table, k_scales, v_scales)
    return kv


def spark_kv_append_paged(kv: SparkPagedKV, k, v, pos0, cfg: SparkLayerCfg, flags: int = 0, stream=None) -> None:
    """Append k, v [B, T, 4, 256] at positions pos0[b] + t into a paged pool (quantised if it is 8-bit)."""
    pk, pv = _dev(k, "k", ndim=4), _dev(v, "v", ndim=4)
    pp = _dev(pos0, "pos0", torch.int32, 1)
    _raise(_lib().spark_kv_append_paged(ctypes.byref(kv), pk, pv, k.shape[0], k.shape[1], pp, ctypes.byref(cfg),
                                        flags, _stream(stream)))


def spark_decode_paged_workspace_bytes(B: int, kv: SparkPagedKV, cfg: SparkLayerCfg) -> int:
    return int(_lib().spark_decode_paged_workspace_bytes(B, ctypes.byref(kv), ctypes.byref(cfg)))


def spark_attn_decode_paged(out, q, gate, kv: SparkPagedKV, pos, cfg: SparkLayerCfg, workspace: torch.Tensor,
                            flags: int = 0, stream=None) -> None:
    """spark_attn_decode over a paged pool."""
    po, pq = _dev(out, "out", ndim=3), _dev(q, "q", ndim=3)
    pg = _dev(gate, "gate", ndim=2)
    pp = _dev(pos, "pos", torch.int32, 1)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    _raise(_lib().spark_attn_decode_paged(po, pq, pg, ctypes.byref(kv), q.shape[0], pp, ctypes.byref(cfg),
                                          workspace.data_ptr(), ws_bytes, flags, _stream(stream)))


def _cu(cu_seqlens):
    pc = _dev(cu_seqlens, "cu_seqlens", torch.int32, 1)
    return pc, cu_seqlens.shape[0] - 1


def spark_rope_apply_varlen(x, cu_seqlens, max_seqlen: int, pos0, cfg: SparkLayerCfg, stream=None) -> None:
    """Rotate packed x [total, H, 256] in place; sequence b is rows cu_seqlens[b]:cu_seqlens[b+1]."""
    px = _dev(x, "x", ndim=3)
    pc, B = _cu(cu_seqlens)
    pp = _dev(pos0, "pos0", torch.int32, 1)
    _raise(_lib().spark_rope_apply_varlen(px, x.shape[1], pc, max_seqlen, pp, B, ctypes.byref(cfg),
                                          _stream(stream)))


def spark_kv_append_varlen(kv: SparkPagedKV, k, v, cu_seqlens, max_seqlen: int, pos0, cfg: SparkLayerCfg,
                           flags: int = 0, stream=None) -> None:
    """Append packed k, v [total, 4, 256] into a paged pool."""
    pk, pv = _dev(k, "k", ndim=3), _dev(v, "v", ndim=3)
    pc, B = _cu(cu_seqlens)
    pp = _dev(pos0, "pos0", torch.int32, 1)
    _raise(_lib().spark_kv_append_varlen(ctypes.byref(kv), pk, pv, pc, max_seqlen, pp, B, ctypes.byref(cfg), flags,
                                         _stream(stream)))


def spark_attn_prefill_varlen(out, q, k, v, gate, cu_seqlens, max_seqlen: int, pos0, history, cfg: SparkLayerCfg,
                              flags: int = 0, stream=None) -> None:
    """Prefill of a ragged batch: packed out/q [total, 16, 256], k/v [total, 4, 256], gate [total, 16];
    history: a paged pool (paged_kv) or None."""
    po, pq = _dev(out, "out", ndim=3), _dev(q, "q", ndim=3)
    pk, pv = _dev(k, "k", ndim=3), _dev(v, "v", ndim=3)
    pg = _dev(gate, "gate", ndim=2)
    pc, B = _cu(cu_seqlens)
    pp = _dev(pos0, "pos0", torch.int32, 1)
    hist = ctypes.byref(history) if history is not None else None
    _raise(_lib().spark_attn_prefill_varlen(po, pq, pk, pv, pg, pc, q.shape[0], max_seqlen, pp, hist, B,
                                            ctypes.byref(cfg), flags, _stream(stream)))


def spark_selftest_wait_timeout(timeout_ns: int, stream=None) -> None:
    """Launch a block whose bounded wait cannot complete; spark_check() then reports a timeout."""
    _raise(_lib().spark_selftest_wait_timeout(timeout_ns, _stream(stream)))


def spark_check(stream=None) -> None:
    """Synchronise the stream and raise SparkError if a kernel flagged a device-side error."""
    _raise(_lib().spark_check(_stream(stream)))
