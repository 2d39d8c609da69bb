"""Device-resident quantized linear layers.

A layer takes the canonical arrays of one weight matrix (NumPy, host), packs them
with the library's host packer, uploads the packed arrays once, and owns a
zero-filled workspace.  ``forward`` enqueues the entry point on a stream.  The
class only moves and marshals data; every operation runs in ``libqlinear.so``.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import (QL_FMT_CB, QL_FMT_LUT4, QL_FMT_W2, QL_FMT_W3, QL_FMT_W4, QL_FMT_W8,
               qlinear_codebook, qlinear_codebook_tc, qlinear_codebook_workspace_bytes,
               qlinear_debug_dequant, qlinear_pack_codebook, qlinear_pack_codebook_scales,
               qlinear_pack_codebook_tc,
               qlinear_debug_unpack, qlinear_dequant_fp16, qlinear_lut4, qlinear_pack,
               qlinear_matmul, qlinear_pack_params, qlinear_pack_params_grouped,
               qlinear_prefill, qlinear_prefill_fused, qlinear_prefill_workspace_bytes,
               qlinear_read_error,
               qlinear_pack_tilecoo, qlinear_w2a16, qlinear_w3a16, qlinear_w4a16,
               qlinear_w4a16_outlier,
               qlinear_w8a16, qlinear_workspace_bytes)

_ENTRY = {QL_FMT_W2: qlinear_w2a16, QL_FMT_W3: qlinear_w3a16, QL_FMT_W4: qlinear_w4a16,
          QL_FMT_W8: qlinear_w8a16}


def _dev(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


class QuantLinear:
    """One quantized weight matrix [K, N] resident on a CUDA device."""

    def __init__(self, fmt: int, K: int, N: int, canonical_codes: np.ndarray,
                 p0: np.ndarray, p1: Optional[np.ndarray] = None,
                 tilecoo: Optional[tuple] = None, device="cuda", max_m: int = 16,
                 group: int = 128):
        self.fmt, self.K, self.N, self.group = fmt, K, N, group
        self.device = torch.device(device)
        packed = qlinear_pack(fmt, canonical_codes, N, K)
        self.qweight = _dev(packed, self.device)
        if fmt == QL_FMT_LUT4:
            self.p0 = _dev(np.asarray(p0, dtype=np.float16).view(np.uint16), self.device)  # lut16
            self.p1 = _dev(qlinear_pack_params(fmt, np.asarray(p1, dtype=np.float32), N, K),
                           self.device)  # absmax
        elif group != 128:
            self.p0 = _dev(qlinear_pack_params_grouped(fmt, group, p0, N, K).view(np.uint16),
                           self.device)  # scales, one per (sub-group, column)
            self.p1 = _dev(qlinear_pack_params_grouped(fmt, group, p1, N, K).view(np.uint16),
                           self.device)  # zeros
        else:
            self.p0 = _dev(qlinear_pack_params(fmt, np.asarray(p0, dtype=np.float16), N, K)
                           .view(np.uint16), self.device)  # scales
            self.p1 = _dev(qlinear_pack_params(fmt, np.asarray(p1, dtype=np.float16), N, K)
                           .view(np.uint16), self.device)  # zeros
        self.tile = None
        if tilecoo is not None:
            off, rc, vals = qlinear_pack_tilecoo(*tilecoo, N, K)
            self.tile = (_dev(off, self.device), _dev(rc, self.device),
                         _dev(vals.view(np.uint16), self.device))
        ws = max(qlinear_workspace_bytes(fmt, m, N, K) for m in (1, max_m))
        self.workspace = torch.zeros(max(ws, 256) // 4 + 64, dtype=torch.int32, device=self.device)

    @property
    def weight_bytes(self) -> int:
        b = self.qweight.numel() + self.p0.numel() * self.p0.element_size() + \
            self.p1.numel() * self.p1.element_size()
        if self.tile is not None:
            b += sum(t.numel() * t.element_size() for t in self.tile)
        return b

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """y[M, N] (fp16) = x[M, K] (fp16) . W."""
        M = x.shape[0]
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.float16, device=self.device)
        xv = x.view(torch.int16)
        yv = y.view(torch.int16)
        if self.tile is not None:
            qlinear_w4a16_outlier(xv, self.qweight, self.p0, self.p1, *self.tile, yv, M, self.N,
                                  self.K, self.workspace, stream)
        elif self.fmt == QL_FMT_LUT4:
            qlinear_lut4(xv, self.qweight, self.p0, self.p1, yv, M, self.N, self.K,
                         self.workspace, stream)
        else:
            _ENTRY[self.fmt](xv, self.qweight, self.p0, self.p1, yv, M, self.N, self.K,
                             self.workspace, stream, group=self.group)
        return y

    def read_error(self, stream=None) -> int:
        """Sticky error flags of the calls that used this layer's workspace (then cleared);
        0 = every device wait completed."""
        return qlinear_read_error(self.workspace, stream)

    def _group128(self, what: str) -> None:
        if self.group != 128:
            raise ValueError(f"{what} reads parameters packed for group 128")

    def dequant_fp16(self, w: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """The dense fp16 weights, ``w[N, K]`` (one row per output column)."""
        self._group128("dequant_fp16")
        if w is None:
            w = torch.empty((self.N, self.K), dtype=torch.float16, device=self.device)
        qlinear_dequant_fp16(self.fmt, self.qweight, self.p0, self.p1, w.view(torch.int16),
                             self.N, self.K, stream)
        return w

    def prefill(self, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                w_fp16: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """y[M, N] = x[M, K] . W for any M: dequantize into ``w_fp16`` ([N, K] fp16, kept
        by the layer when not given), then one dense GEMM.  Dense part only (no outliers)."""
        if self.tile is not None:
            raise ValueError("prefill covers the dense formats; the outlier layer has none")
        self._group128("prefill")
        M = x.shape[0]
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.float16, device=self.device)
        if w_fp16 is None:
            if getattr(self, "_w_fp16", None) is None:
                self._w_fp16 = torch.empty((self.N, self.K), dtype=torch.float16,
                                           device=self.device)
            w_fp16 = self._w_fp16
        qlinear_prefill(self.fmt, x.view(torch.int16), self.qweight, self.p0, self.p1,
                        w_fp16.view(torch.int16), y.view(torch.int16), M, self.N, self.K, stream)
        return y

    def prefill_fused(self, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                      stream=None, stream_k: bool = True) -> torch.Tensor:
        """y[M, N] = x[M, K] . W for any M, the weights dequantized inside the tensor-core
        GEMM (no fp16 weight matrix); stream_k shares the k-blocks out over the SMs through a
        workspace the layer keeps.  Dense part only (no outliers)."""
        if self.tile is not None:
            raise ValueError("prefill covers the dense formats; the outlier layer has none")
        self._group128("prefill")
        M = x.shape[0]
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.float16, device=self.device)
        ws = self._prefill_workspace(M) if stream_k else None
        qlinear_prefill_fused(self.fmt, x.view(torch.int16), self.qweight, self.p0, self.p1,
                              y.view(torch.int16), M, self.N, self.K, ws, stream)
        return y

    def _prefill_workspace(self, M: int) -> torch.Tensor:
        """The zero-filled stream-K workspace of the fused prefill, grown as M needs."""
        need = qlinear_prefill_workspace_bytes(M, self.N, self.K)
        ws = getattr(self, "_pf_ws", None)
        if ws is None or ws.numel() * 4 < need:
            ws = torch.zeros(need // 4 + 64, dtype=torch.int32, device=self.device)
            self._pf_ws = ws
        return ws

    def matmul(self, x: torch.Tensor, y: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
        """y[M, N] = x[M, K] . W for any M, dispatched by the library's policy map (the fused
        GEMV, over 16-row slices when M > 16, or the tensor-core prefill GEMM with the
        dequantization fused in)."""
        if self.tile is not None:
            raise ValueError("the policy map covers the dense formats")
        self._group128("matmul")
        M = x.shape[0]
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.float16, device=self.device)
        qlinear_matmul(self.fmt, x.view(torch.int16), self.qweight, self.p0, self.p1,
                       y.view(torch.int16), M, self.N, self.K, self.workspace, None, stream)
        return y

    def debug_unpack(self, stream=None) -> torch.Tensor:
        codes = torch.empty((self.K, self.N), dtype=torch.uint8, device=self.device)
        qlinear_debug_unpack(self.fmt, self.qweight, codes, self.N, self.K, stream)
        return codes

    def debug_dequant(self, stream=None) -> torch.Tensor:
        self._group128("debug_dequant")
        w = torch.empty((self.K, self.N), dtype=torch.float32, device=self.device)
        qlinear_debug_dequant(self.fmt, self.qweight, self.p0, self.p1, w, self.N, self.K, stream)
        return w


def from_uniform(layer, device="cuda", max_m: int = 16) -> QuantLinear:
    """From a ``synth.gen.UniformLayer``-like object (bits, K, N, qweight, scales, zeros and,
    optionally, group)."""
    return QuantLinear(layer.bits, layer.K, layer.N, layer.qweight, layer.scales, layer.zeros,
                       device=device, max_m=max_m, group=getattr(layer, "group", 128))


def from_lut4(layer, device="cuda", max_m: int = 16) -> QuantLinear:
    return QuantLinear(QL_FMT_LUT4, layer.K, layer.N, layer.qbytes, layer.lut, layer.absmax,
                       device=device, max_m=max_m)


def from_outlier(layer, device="cuda", max_m: int = 16) -> QuantLinear:
    d = layer.dense
    return QuantLinear(QL_FMT_W4, d.K, d.N, d.qweight, d.scales, d.zeros,
                       tilecoo=(layer.tile_offsets, layer.tile_rc, layer.tile_vals),
                       device=device, max_m=max_m)


class CodebookLinear:
    """A codebook-quantized weight matrix (m1v4g128: codes uint8 [K / 4][N], scales fp16
    [K / 128][N], codebook fp16 [256][4]) on the device, packed for both GEMV forms: the
    Psumbook form (``qlinear_codebook``, M <= 4, N % 32 == 0) and the tensor-core form
    (``qlinear_codebook_tc``, M <= 16, N % 16 == 0)."""

    def __init__(self, K: int, N: int, codes: np.ndarray, scales: np.ndarray,
                 codebook: np.ndarray, device="cuda", max_m: int = 16):
        self.K, self.N, self.device, self.max_m = K, N, torch.device(device), max_m
        scales16 = np.ascontiguousarray(scales).view(np.uint16)
        self.codebook = _dev(np.ascontiguousarray(codebook).view(np.int16), self.device)
        self.codes_tc = _dev(qlinear_pack_codebook_tc(codes, N, K), self.device)
        self.scales_tc = _dev(qlinear_pack_params(QL_FMT_W4, scales16, N, K).view(np.int16),
                              self.device)
        ws = max(qlinear_workspace_bytes(QL_FMT_CB, m, N, K) for m in (1, max_m))
        self.ws_tc = torch.zeros(max(ws, 256) // 4 + 64, dtype=torch.int32, device=self.device)
        self.psum_ok = N % 32 == 0
        if self.psum_ok:
            self.codes_ps = _dev(qlinear_pack_codebook(codes, N, K), self.device)
            self.scales_ps = _dev(qlinear_pack_codebook_scales(scales16, N, K).view(np.int16),
                                  self.device)
            ws = max(qlinear_codebook_workspace_bytes(m, N, K) for m in range(1, 5))
            self.ws_ps = torch.zeros(max(ws, 256) // 4 + 64, dtype=torch.int32,
                                     device=self.device)

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None,
                form: str = "tc") -> torch.Tensor:
        """y[M, N] (fp16) = x[M, K] (fp16) . W; form "tc" (tensor cores) or "psumbook"."""
        M = x.shape[0]
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.float16, device=self.device)
        xv, yv = x.view(torch.int16), y.view(torch.int16)
        if form == "tc":
            qlinear_codebook_tc(xv, self.codes_tc, self.scales_tc, self.codebook, yv, M, self.N,
                                self.K, self.ws_tc, stream)
        elif form == "psumbook":
            if not self.psum_ok:
                raise ValueError("the Psumbook form needs N % 32 == 0")
            qlinear_codebook(xv, self.codes_ps, self.scales_ps, self.codebook, yv, M, self.N,
                             self.K, self.ws_ps, stream)
        else:
            raise ValueError(f"unknown form {form!r}")
        return y

    def read_error(self, stream=None) -> int:
        """Sticky error flags of the tensor-core form's device waits (then cleared)."""
        return qlinear_read_error(self.ws_tc, stream)


def from_codebook(layer, device="cuda", max_m: int = 16) -> CodebookLinear:
    """From a ``synth.gen.CodebookLayer``-like object (K, N, codes, scales, codebook)."""
    return CodebookLinear(layer.K, layer.N, layer.codes, layer.scales, layer.codebook,
                          device=device, max_m=max_m)
