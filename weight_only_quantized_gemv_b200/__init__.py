"""Python binding of ``libqlinear.so``: the weight-only-quantized linear layer on B200.

Argument marshalling only.  Every function here forwards to the C entry point of
the same name in ``include/qlinear.h``; device arguments are ``torch.Tensor``
objects on the current CUDA device (their ``data_ptr()`` is passed), host
arguments of the packers are NumPy arrays.  A non-OK status raises
``QLinearError``.  There is no fallback: if the shared library is missing, the
import fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_HERE, "libqlinear.so")

if not os.path.exists(LIBRARY_PATH):
    raise ImportError(
        f"{LIBRARY_PATH} is missing: build it with "
        "`python -c 'import __graft_entry__ as g; g.build()'` or "
        "`python weight_only_quantized_gemv_b200/build.py`")

_lib = ctypes.CDLL(LIBRARY_PATH)

QL_FMT_W2, QL_FMT_W3, QL_FMT_W4, QL_FMT_W8, QL_FMT_LUT4 = 2, 3, 4, 8, 16
QL_FMT_CB = 32  # the codebook in the tensor-core layout (workspace and plan queries)
FORMATS = {"w2": QL_FMT_W2, "w3": QL_FMT_W3, "w4": QL_FMT_W4, "w8": QL_FMT_W8,
           "lut4": QL_FMT_LUT4}
STATUS = {0: "QL_OK", 1: "QL_ERR_NULL", 2: "QL_ERR_SHAPE", 3: "QL_ERR_ALIGN",
          4: "QL_ERR_UNSUPPORTED", 5: "QL_ERR_WORKSPACE", 6: "QL_ERR_CUDA",
          7: "QL_ERR_LIBRARY"}

_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t


class ql_policy_entry(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int), ("N", ctypes.c_int), ("K", ctypes.c_int),
                ("m_lo", ctypes.c_int), ("m_hi", ctypes.c_int), ("strategy", ctypes.c_int),
                ("warps_per_unit", ctypes.c_int), ("ctas", ctypes.c_int)]


QL_STRATEGY_GEMV, QL_STRATEGY_PREFILL = 0, 1


class ql_plan(ctypes.Structure):
    _fields_ = [("ctas", ctypes.c_int), ("warps", ctypes.c_int), ("tiles_per_warp", ctypes.c_int),
                ("units", ctypes.c_longlong), ("m_bucket", ctypes.c_int),
                ("warps_per_unit", ctypes.c_int)]


_SIGS = {
    "ql_status_str": (ctypes.c_char_p, [_I]),
    "qlinear_packed_bytes": (_SZ, [_I, _I, _I]),
    "qlinear_params_bytes": (_SZ, [_I, _I, _I]),
    "qlinear_pack": (_I, [_I, _P, _P, _I, _I]),
    "qlinear_pack_params": (_I, [_I, _P, _P, _I, _I]),
    "qlinear_params_bytes_grouped": (_SZ, [_I, _I, _I, _I]),
    "qlinear_pack_params_grouped": (_I, [_I, _I, _P, _P, _I, _I]),
    "qlinear_pack_tilecoo": (_I, [_P, _P, _P, _I, _I, _P, _P, _P]),
    "qlinear_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "qlinear_w4a16": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _SZ, _P]),
    "qlinear_w2a16": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _SZ, _P]),
    "qlinear_w8a16": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _SZ, _P]),
    "qlinear_w3a16": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _SZ, _P]),
    "qlinear_lut4": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _SZ, _P]),
    "qlinear_w4a16_outlier": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _SZ, _P]),
    "qlinear_debug_unpack": (_I, [_I, _P, _P, _I, _I, _P]),
    "qlinear_debug_dequant": (_I, [_I, _P, _P, _P, _P, _I, _I, _P]),
    "qlinear_plan": (_I, [_I, _I, _I, _I, ctypes.POINTER(ql_plan)]),
    "qlinear_read_error": (_I, [_P, ctypes.POINTER(ctypes.c_uint32), _P]),
    "qlinear_debug_wait_test": (_I, [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32]),
    "qlinear_w4a16_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "qlinear_w4a16_noalloc_read_error": (_I, [ctypes.POINTER(ctypes.c_uint32), _P]),
    "qlinear_dequant_fp16": (_I, [_I, _P, _P, _P, _P, _I, _I, _P]),
    "qlinear_prefill": (_I, [_I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "qlinear_prefill_fused": (_I, [_I, _P, _P, _P, _P, _P, _I, _I, _I, _P, _SZ, _P]),
    "qlinear_prefill_workspace_bytes": (_SZ, [_I, _I, _I]),
    "qlinear_prefill_read_error": (_I, [ctypes.POINTER(ctypes.c_uint32), _P]),
    "qlinear_policy_set": (_I, [ctypes.POINTER(ql_policy_entry), _I]),
    "qlinear_policy_size": (_I, []),
    "qlinear_policy_lookup": (_I, [_I, _I, _I, _I, ctypes.POINTER(ql_policy_entry),
                                   ctypes.POINTER(_I)]),
    "qlinear_matmul": (_I, [_I, _P, _P, _P, _P, _P, _I, _I, _I, _P, _SZ, _P, _P]),
    "qlinear_pack_codebook": (_I, [_P, _P, _I, _I]),
    "qlinear_pack_codebook_scales": (_I, [_P, _P, _I, _I]),
    "qlinear_codebook_workspace_bytes": (_SZ, [_I, _I, _I]),
    "qlinear_codebook": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P, _SZ, _P]),
    "qlinear_pack_codebook_tc": (_I, [_P, _P, _I, _I]),
    "qlinear_codebook_tc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P, _SZ, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


class QLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.ql_status_str(status).decode()
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != 0:
        raise QLinearError(status, where)


def _ptr(t) -> Optional[int]:
    """Device pointer of a torch tensor, or None."""
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _np_ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# ---------------------------------------------------------------------------
# host packer (NumPy in, NumPy out)


def qlinear_packed_bytes(fmt: int, N: int, K: int) -> int:
    return int(_lib.qlinear_packed_bytes(fmt, N, K))


def qlinear_params_bytes(fmt: int, N: int, K: int) -> int:
    return int(_lib.qlinear_params_bytes(fmt, N, K))


def qlinear_pack(fmt: int, canonical: np.ndarray, N: int, K: int) -> np.ndarray:
    canonical = np.ascontiguousarray(canonical)
    out = np.empty(qlinear_packed_bytes(fmt, N, K), dtype=np.uint8)
    if out.size != canonical.nbytes:
        raise QLinearError(2, "qlinear_pack")
    _check(_lib.qlinear_pack(fmt, _np_ptr(canonical), _np_ptr(out), N, K), "qlinear_pack")
    return out


def qlinear_pack_params(fmt: int, canonical: np.ndarray, N: int, K: int) -> np.ndarray:
    canonical = np.ascontiguousarray(canonical)
    out = np.empty(canonical.shape, dtype=canonical.dtype)
    if canonical.nbytes != qlinear_params_bytes(fmt, N, K):
        raise QLinearError(2, "qlinear_pack_params")
    _check(_lib.qlinear_pack_params(fmt, _np_ptr(canonical), _np_ptr(out), N, K),
           "qlinear_pack_params")
    return out


def qlinear_params_bytes_grouped(fmt: int, group: int, N: int, K: int) -> int:
    return int(_lib.qlinear_params_bytes_grouped(fmt, group, N, K))


def qlinear_pack_params_grouped(fmt: int, group: int, canonical: np.ndarray, N: int,
                                K: int) -> np.ndarray:
    """fp16 [K / group, N] (or [1, N] for group = K) -> the kernel layout for that group."""
    canonical = np.ascontiguousarray(canonical, dtype=np.float16)
    rows = 1 if group == K else K // group
    if canonical.shape != (rows, N):
        raise QLinearError(2, "qlinear_pack_params_grouped")
    nbytes = qlinear_params_bytes_grouped(fmt, group, N, K)
    if nbytes == 0:
        raise QLinearError(2, "qlinear_pack_params_grouped")
    out = np.empty(nbytes // 2, dtype=np.float16)
    _check(_lib.qlinear_pack_params_grouped(fmt, group, _np_ptr(canonical), _np_ptr(out), N, K),
           "qlinear_pack_params_grouped")
    return out


def qlinear_pack_tilecoo(offsets: np.ndarray, rc: np.ndarray, vals: np.ndarray, N: int, K: int):
    offsets = np.ascontiguousarray(offsets, dtype=np.uint32)
    rc = np.ascontiguousarray(rc, dtype=np.uint8)
    vals = np.ascontiguousarray(vals).view(np.uint16)
    o2, r2, v2 = np.empty_like(offsets), np.empty_like(rc), np.empty_like(vals)
    _check(_lib.qlinear_pack_tilecoo(_np_ptr(offsets), _np_ptr(rc), _np_ptr(vals), N, K,
                                     _np_ptr(o2), _np_ptr(r2), _np_ptr(v2)), "qlinear_pack_tilecoo")
    return o2, r2, v2.view(np.float16)


# ---------------------------------------------------------------------------
# workspace / plan


def qlinear_workspace_bytes(fmt: int, M: int, N: int, K: int) -> int:
    return int(_lib.qlinear_workspace_bytes(fmt, M, N, K))


def qlinear_plan(fmt: int, M: int, N: int, K: int) -> ql_plan:
    p = ql_plan()
    _check(_lib.qlinear_plan(fmt, M, N, K, ctypes.byref(p)), "qlinear_plan")
    return p


def qlinear_debug_wait_test(wait_limit=0, producer_delay_us=0, consumer_hold_us=0) -> None:
    """Settings for tests of the bounded device waits; no arguments restores the defaults."""
    _check(_lib.qlinear_debug_wait_test(wait_limit, producer_delay_us, consumer_hold_us),
           "qlinear_debug_wait_test")


def qlinear_read_error(workspace, stream=None) -> int:
    """Sticky error flags of the calls that used `workspace` (then cleared); 0 = none."""
    flags = ctypes.c_uint32(0)
    _check(_lib.qlinear_read_error(_ptr(workspace), ctypes.byref(flags), _stream(stream)),
           "qlinear_read_error")
    return int(flags.value)


# ---------------------------------------------------------------------------
# hot path (torch tensors on the current device)


def _uniform(name, x, qweight, scales, zeros, y, M, N, K, workspace, stream, group=128):
    st = getattr(_lib, name)(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(y), M, N, K,
                             group, _ptr(workspace), workspace.numel() * workspace.element_size()
                             if workspace is not None else 0, _stream(stream))
    _check(st, name)
    return y


def qlinear_w4a16(x, qweight, scales, zeros, y, M, N, K, workspace, stream=None, group=128):
    return _uniform("qlinear_w4a16", x, qweight, scales, zeros, y, M, N, K, workspace, stream, group)


def qlinear_w2a16(x, qweight, scales, zeros, y, M, N, K, workspace, stream=None, group=128):
    return _uniform("qlinear_w2a16", x, qweight, scales, zeros, y, M, N, K, workspace, stream, group)


def qlinear_w8a16(x, qweight, scales, zeros, y, M, N, K, workspace, stream=None, group=128):
    return _uniform("qlinear_w8a16", x, qweight, scales, zeros, y, M, N, K, workspace, stream, group)


def qlinear_w3a16(x, qweight, scales, zeros, y, M, N, K, workspace, stream=None, group=128):
    return _uniform("qlinear_w3a16", x, qweight, scales, zeros, y, M, N, K, workspace, stream, group)


def qlinear_w4a16_noalloc(x, qweight, scales, zeros, y, M, N, K, stream=None, group=128):
    """qlinear_w4a16 with the library's fixed device scratch instead of a workspace."""
    _check(_lib.qlinear_w4a16_noalloc(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(y),
                                      M, N, K, group, _stream(stream)), "qlinear_w4a16_noalloc")
    return y


def qlinear_w4a16_noalloc_read_error(stream=None) -> int:
    """Sticky error flags of qlinear_w4a16_noalloc's scratch on the current device (then
    cleared); 0 = none."""
    flags = ctypes.c_uint32(0)
    _check(_lib.qlinear_w4a16_noalloc_read_error(ctypes.byref(flags), _stream(stream)),
           "qlinear_w4a16_noalloc_read_error")
    return int(flags.value)


def qlinear_lut4(x, codes, lut16, absmax, y, M, N, K, workspace, stream=None, block=64):
    st = _lib.qlinear_lut4(_ptr(x), _ptr(codes), _ptr(lut16), _ptr(absmax), _ptr(y), M, N, K, block,
                           _ptr(workspace), workspace.numel() * workspace.element_size()
                           if workspace is not None else 0, _stream(stream))
    _check(st, "qlinear_lut4")
    return y


def qlinear_w4a16_outlier(x, qweight, scales, zeros, tile_offsets, tile_rc, tile_vals, y, M, N, K,
                          workspace, stream=None, group=128):
    st = _lib.qlinear_w4a16_outlier(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(zeros),
                                    _ptr(tile_offsets), _ptr(tile_rc), _ptr(tile_vals), _ptr(y),
                                    M, N, K, group, _ptr(workspace),
                                    workspace.numel() * workspace.element_size()
                                    if workspace is not None else 0, _stream(stream))
    _check(st, "qlinear_w4a16_outlier")
    return y


def qlinear_debug_unpack(fmt, packed, codes, N, K, stream=None):
    _check(_lib.qlinear_debug_unpack(fmt, _ptr(packed), _ptr(codes), N, K, _stream(stream)),
           "qlinear_debug_unpack")
    return codes


def qlinear_debug_dequant(fmt, packed, p0, p1, w, N, K, stream=None):
    _check(_lib.qlinear_debug_dequant(fmt, _ptr(packed), _ptr(p0), _ptr(p1), _ptr(w), N, K,
                                      _stream(stream)), "qlinear_debug_dequant")
    return w


def qlinear_dequant_fp16(fmt, packed, p0, p1, w, N, K, stream=None):
    """Packed weights -> dense fp16 ``w[N, K]`` (see the C declaration for p0 / p1)."""
    _check(_lib.qlinear_dequant_fp16(fmt, _ptr(packed), _ptr(p0), _ptr(p1), _ptr(w), N, K,
                                     _stream(stream)), "qlinear_dequant_fp16")
    return w


def qlinear_prefill(fmt, x, packed, p0, p1, w_fp16, y, M, N, K, stream=None):
    """``y[M, N] = x[M, K] @ w_fp16[N, K]^T`` after dequantizing into ``w_fp16``."""
    _check(_lib.qlinear_prefill(fmt, _ptr(x), _ptr(packed), _ptr(p0), _ptr(p1), _ptr(w_fp16),
                                _ptr(y), M, N, K, _stream(stream)), "qlinear_prefill")
    return y


def qlinear_prefill_fused(fmt, x, packed, p0, p1, y, M, N, K, workspace=None, stream=None):
    """``y[M, N] = x[M, K] @ W^T`` with the weights dequantized inside the tensor-core GEMM;
    with a (zero-filled) workspace the k-blocks are shared out over the SMs (stream-K)."""
    _check(_lib.qlinear_prefill_fused(fmt, _ptr(x), _ptr(packed), _ptr(p0), _ptr(p1), _ptr(y),
                                      M, N, K, _ptr(workspace),
                                      workspace.numel() * workspace.element_size()
                                      if workspace is not None else 0, _stream(stream)),
           "qlinear_prefill_fused")
    return y


def qlinear_prefill_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.qlinear_prefill_workspace_bytes(M, N, K))


def qlinear_prefill_read_error(stream=None) -> int:
    """Sticky wait-timeout flags of the prefill GEMM kernels on the current device (then
    cleared); 0 = none."""
    flags = ctypes.c_uint32(0)
    _check(_lib.qlinear_prefill_read_error(ctypes.byref(flags), _stream(stream)),
           "qlinear_prefill_read_error")
    return int(flags.value)


# ---------------------------------------------------------------------------
# measured policy map and dispatcher


_ENTRY_KEYS = ("fmt", "N", "K", "m_lo", "m_hi", "strategy", "warps_per_unit", "ctas")


def qlinear_policy_set(entries) -> None:
    """Install a policy table: a sequence of dicts (or ql_policy_entry) with the entry's
    fields; an empty sequence clears it."""
    arr = (ql_policy_entry * max(len(entries), 1))()
    for i, e in enumerate(entries):
        arr[i] = e if isinstance(e, ql_policy_entry) else \
            ql_policy_entry(*[int(e.get(k, 0)) for k in _ENTRY_KEYS])
    _check(_lib.qlinear_policy_set(arr, len(entries)), "qlinear_policy_set")


def qlinear_policy_size() -> int:
    return int(_lib.qlinear_policy_size())


def qlinear_policy_lookup(fmt: int, M: int, N: int, K: int):
    """(decision as a dict, whether it came from the table)."""
    e = ql_policy_entry()
    ft = _I(0)
    _check(_lib.qlinear_policy_lookup(fmt, M, N, K, ctypes.byref(e), ctypes.byref(ft)),
           "qlinear_policy_lookup")
    return {k: getattr(e, k) for k in _ENTRY_KEYS}, bool(ft.value)


def default_policy_path() -> str:
    """The table measured on B200 for the Llama-shaped layers (the package's policy_b200.json,
    written by the tune module)."""
    return os.path.join(_HERE, "policy_b200.json")


def load_policy(path: Optional[str] = None) -> int:
    """Install the table of a JSON file written by the tune module (default: the B200 table);
    returns its size."""
    import json
    with open(path or default_policy_path()) as f:
        table = json.load(f)
    qlinear_policy_set(table["entries"])
    return qlinear_policy_size()


def qlinear_matmul(fmt, x, packed, p0, p1, y, M, N, K, workspace, w_fp16=None, stream=None):
    """y[M, N] = x[M, K] . W for any M, by the policy map (GEMV slices or prefill)."""
    st = _lib.qlinear_matmul(fmt, _ptr(x), _ptr(packed), _ptr(p0), _ptr(p1), _ptr(y), M, N, K,
                             _ptr(workspace), workspace.numel() * workspace.element_size()
                             if workspace is not None else 0, _ptr(w_fp16), _stream(stream))
    _check(st, "qlinear_matmul")
    return y


# ---------------------------------------------------------------------------
# codebook GEMV (Psumbook)


def qlinear_pack_codebook(codes: np.ndarray, N: int, K: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    if codes.size != K // 4 * N:
        raise QLinearError(2, "qlinear_pack_codebook")
    out = np.empty(codes.size, dtype=np.uint8)
    _check(_lib.qlinear_pack_codebook(_np_ptr(codes), _np_ptr(out), N, K), "qlinear_pack_codebook")
    return out


def qlinear_pack_codebook_scales(scales: np.ndarray, N: int, K: int) -> np.ndarray:
    scales = np.ascontiguousarray(scales).view(np.uint16)
    if scales.size != K // 128 * N:
        raise QLinearError(2, "qlinear_pack_codebook_scales")
    out = np.empty(scales.size, dtype=np.uint16)
    _check(_lib.qlinear_pack_codebook_scales(_np_ptr(scales), _np_ptr(out), N, K),
           "qlinear_pack_codebook_scales")
    return out


def qlinear_codebook_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.qlinear_codebook_workspace_bytes(M, N, K))


def qlinear_codebook(x, codes, scales, codebook, y, M, N, K, workspace, stream=None):
    st = _lib.qlinear_codebook(_ptr(x), _ptr(codes), _ptr(scales), _ptr(codebook), _ptr(y), M, N,
                               K, _ptr(workspace), workspace.numel() * workspace.element_size()
                               if workspace is not None else 0, _stream(stream))
    _check(st, "qlinear_codebook")
    return y


# codebook GEMV on the tensor cores (the GEMV kernel, codebook lookups as A fragments)


def qlinear_pack_codebook_tc(codes: np.ndarray, N: int, K: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    if codes.size != K // 4 * N:
        raise QLinearError(2, "qlinear_pack_codebook_tc")
    out = np.empty(codes.size, dtype=np.uint8)
    _check(_lib.qlinear_pack_codebook_tc(_np_ptr(codes), _np_ptr(out), N, K),
           "qlinear_pack_codebook_tc")
    return out


def qlinear_codebook_tc(x, codes, scales, codebook, y, M, N, K, workspace, stream=None):
    st = _lib.qlinear_codebook_tc(_ptr(x), _ptr(codes), _ptr(scales), _ptr(codebook), _ptr(y), M,
                                  N, K, _ptr(workspace), workspace.numel() * workspace.element_size()
                                  if workspace is not None else 0, _stream(stream))
    _check(st, "qlinear_codebook_tc")
    return y
