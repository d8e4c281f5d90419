"""Whole-layer driver over the C ABI: H accumulation -> factor preparation -> column loop.

``LayerQuantizer`` owns the device buffers for one layer shape so repeated calls allocate
nothing; every step runs in libgq's kernels (this module only sequences the three calls).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import gq as G


@dataclass
class LayerResult:
    codes: torch.Tensor    # m x ceil(n b / 32) packed uint32 (int32 view)
    scales: torch.Tensor   # m x groups fp32
    zeros: torch.Tensor    # m x groups uint8
    loss: torch.Tensor     # [proxy, damped, bound] fp64
    H: torch.Tensor        # n x n fp64
    U: torch.Tensor        # n x n fp32
    dead: torch.Tensor     # n uint8
    delta: torch.Tensor    # [1] fp64


class LayerQuantizer:
    def __init__(self, m: int, n: int, cfg: G.QuantCfg, device="cuda", damp: float = 0.01,
                 max_tokens: int = 65536, order: str | None = None):
        """``order``: None (natural, or reversed when ``cfg.reverse``), or a column order of
        gq_prepare_hinv_ordered: "act" or "given" (fill ``self.perm`` first)."""
        if order is not None and order not in ("act", "given"):
            raise ValueError(f"unknown order {order!r}")
        if order is not None and cfg.reverse:
            raise ValueError("an order replaces cfg.reverse")
        self.m, self.n, self.cfg, self.damp, self.order = m, n, cfg, damp, order
        self.max_tokens = max_tokens
        dev = torch.device(device)
        self.H = torch.zeros((n, n), dtype=torch.float64, device=dev)
        self.U = torch.empty((n, n), dtype=torch.float32, device=dev)
        self.dead = torch.empty(n, dtype=torch.uint8, device=dev)
        self.delta = torch.empty(1, dtype=torch.float64, device=dev)
        self.ws_hess = G.workspace(G.gq_hessian_workspace_size(max_tokens, n), dev)
        self.ws_prep = G.workspace(G.gq_prepare_workspace_size(n), dev)
        self.ws_quant = G.workspace(G.gq_quantize_workspace_size(m, n, cfg), dev)
        ng = 1 if cfg.group_size == 0 else -(-n // cfg.group_size)
        ncols = n if cfg.clip == "unbounded" else G.n_words(n, cfg.bits)
        self.codes = torch.empty((m, ncols), dtype=torch.int32, device=dev)
        self.scales = torch.empty((m, ng), dtype=torch.float32, device=dev)
        self.zeros = torch.empty((m, ng), dtype=torch.uint8, device=dev)
        self.loss = torch.empty(3, dtype=torch.float64, device=dev)
        self.perm = torch.arange(n, dtype=torch.int32, device=dev) if order else None

    def hessian(self, X: torch.Tensor, reset: bool = True, stream=None):
        if X.shape[0] < 1 and not reset:
            return
        if X.shape[0] > self.max_tokens:
            raise ValueError(f"{X.shape[0]} tokens exceed this quantizer's {self.max_tokens}")
        G.gq_hessian_accumulate(self.H, X, accumulate=not reset, ws=self.ws_hess, stream=stream)

    def prepare(self, stream=None):
        if self.order:
            G.gq_prepare_hinv_ordered(self.H, self.damp, self.order, self.perm, self.U, self.dead,
                                      self.delta, self.ws_prep, stream=stream)
        else:
            G.gq_prepare_hinv(self.H, self.damp, self.cfg.reverse, self.U, self.dead,
                              self.delta, self.ws_prep, stream=stream)

    def quantize(self, W: torch.Tensor, stream=None):
        if self.order:
            G.gq_quantize_layer_ordered(W, self.U, self.dead, self.delta, self.cfg, self.perm,
                                        self.codes, self.scales, self.zeros, self.loss,
                                        self.ws_quant, stream=stream)
        else:
            G.gq_quantize_layer(W, self.U, self.dead, self.delta, self.cfg, self.codes,
                                self.scales, self.zeros, self.loss, self.ws_quant, stream=stream)

    def run(self, W: torch.Tensor, X: torch.Tensor, stream=None) -> LayerResult:
        self.hessian(X, stream=stream)
        self.prepare(stream=stream)
        self.quantize(W, stream=stream)
        return self.result()

    def status(self):
        """(prepare status, quantize status, ladder rounds); synchronizes."""
        sp, _ = G.gq_workspace_status(self.ws_prep)
        sq, rounds = G.gq_workspace_status(self.ws_quant)
        return sp, sq, rounds

    def run_host(self, W_host: torch.Tensor, X_host: torch.Tensor, out: dict | None = None,
                 x_chunks: int = 2, stream=None) -> LayerResult:
        """The whole layer from pinned host tensors, transfers overlapped with the kernels.

        X goes to the device in ``x_chunks`` token slices on a copy stream while H accumulates
        slice by slice; W goes on the copy stream after X and is waited for only by the column
        loop; the results are copied into ``out`` (pinned host tensors named codes / scales /
        zeros / loss) on the compute stream.  Device copies of W and X are kept between calls.
        """
        dev = self.H.device
        cur = torch.cuda.current_stream(dev) if stream is None else stream
        if not hasattr(self, "_copy_stream"):
            self._copy_stream = torch.cuda.Stream(device=dev)
        if getattr(self, "_Wd", None) is None or self._Wd.shape != W_host.shape or self._Wd.dtype != W_host.dtype:
            self._Wd = torch.empty(W_host.shape, dtype=W_host.dtype, device=dev)
        if getattr(self, "_Xd", None) is None or self._Xd.shape != X_host.shape or self._Xd.dtype != X_host.dtype:
            self._Xd = torch.empty(X_host.shape, dtype=X_host.dtype, device=dev)
        cs = self._copy_stream
        T = X_host.shape[0]
        if T < 1:
            raise ValueError("run_host needs at least one calibration token")
        k = max(1, min(int(x_chunks), T))
        bounds = [(T * i) // k for i in range(k + 1)]
        cs.wait_stream(cur)  # the previous call's readers of the device copies are done
        evs = []
        with torch.cuda.stream(cs):
            for a, b in zip(bounds[:-1], bounds[1:]):
                self._Xd[a:b].copy_(X_host[a:b], non_blocking=True)
                e = torch.cuda.Event()
                e.record(cs)
                evs.append(e)
            self._Wd.copy_(W_host, non_blocking=True)
            ew = torch.cuda.Event()
            ew.record(cs)
        for i, ((a, b), e) in enumerate(zip(zip(bounds[:-1], bounds[1:]), evs)):
            cur.wait_event(e)
            if b > a:
                G.gq_hessian_accumulate(self.H, self._Xd[a:b], accumulate=i > 0,
                                        ws=self.ws_hess, stream=cur)
        self.prepare(stream=cur)
        cur.wait_event(ew)
        self.quantize(self._Wd, stream=cur)
        if out is not None:
            with torch.cuda.stream(cur):
                out["codes"].copy_(self.codes, non_blocking=True)
                out["scales"].copy_(self.scales, non_blocking=True)
                out["zeros"].copy_(self.zeros, non_blocking=True)
                out["loss"].copy_(self.loss, non_blocking=True)
        return self.result()

    def result(self) -> LayerResult:
        return LayerResult(self.codes, self.scales, self.zeros, self.loss, self.H, self.U,
                           self.dead, self.delta)

