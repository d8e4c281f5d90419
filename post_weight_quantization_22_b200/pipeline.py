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
                 max_tokens: int = 65536):
        self.m, self.n, self.cfg, self.damp = m, n, cfg, damp
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
        self.codes = torch.empty((m, G.n_words(n, cfg.bits)), dtype=torch.int32, device=dev)
        self.scales = torch.empty((m, ng), dtype=torch.float32, device=dev)
        self.zeros = torch.empty((m, ng), dtype=torch.uint8, device=dev)
        self.loss = torch.empty(3, dtype=torch.float64, device=dev)

    def hessian(self, X: torch.Tensor, reset: bool = True, stream=None):
        if X.shape[0] > self.max_tokens:
            raise ValueError(f"{X.shape[0]} tokens exceed this quantizer's {self.max_tokens}")
        G.gq_hessian_accumulate(self.H, X, accumulate=not reset, ws=self.ws_hess, stream=stream)

    def prepare(self, stream=None):
        G.gq_prepare_hinv(self.H, self.damp, self.cfg.reverse, self.U, self.dead, self.delta,
                          self.ws_prep, stream=stream)

    def quantize(self, W: torch.Tensor, stream=None):
        G.gq_quantize_layer(W, self.U, self.dead, self.delta, self.cfg, self.codes, self.scales,
                            self.zeros, self.loss, self.ws_quant, stream=stream)

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

    def result(self) -> LayerResult:
        return LayerResult(self.codes, self.scales, self.zeros, self.loss, self.H, self.U,
                           self.dead, self.delta)

