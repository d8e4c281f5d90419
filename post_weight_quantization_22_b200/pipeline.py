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
        gq_prepare_hinv_ordered: "act", "min_pivot" or "given" (fill ``self.perm`` first)."""
        if order is not None and order not in ("act", "min_pivot", "given"):
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



# ---------------------------------------------------------------------------------------------
# Several layers that share an input: one Hessian and one factor per input
# ---------------------------------------------------------------------------------------------

class BlockQuantizer:
    """Quantize a group of layers whose inputs are shared: the layers that read the same
    activations (q/k/v, gate/up) share one Hessian H = 2 X^T X and one factor U, so each input
    runs gq_hessian_accumulate and gq_prepare_hinv once and each layer runs gq_quantize_layer.

    ``layers``: sequence of (name, m, n, input_key); layers with the same input_key must have
    the same n.  Device buffers are allocated here, once; ``run`` allocates nothing.
    """

    def __init__(self, layers, cfg: G.QuantCfg, device="cuda", damp: float = 0.01,
                 max_tokens: int = 65536):
        self.layers = [tuple(l) for l in layers]
        self.cfg, self.damp, self.max_tokens = cfg, damp, max_tokens
        dev = torch.device(device)
        self.inputs = {}
        for name, m, n, key in self.layers:
            if key in self.inputs:
                if self.inputs[key]["n"] != n:
                    raise ValueError(f"layers of input {key!r} disagree on n")
                continue
            self.inputs[key] = dict(
                n=n, H=torch.zeros((n, n), dtype=torch.float64, device=dev),
                U=torch.empty((n, n), dtype=torch.float32, device=dev),
                dead=torch.empty(n, dtype=torch.uint8, device=dev),
                delta=torch.empty(1, dtype=torch.float64, device=dev),
                ws_hess=G.workspace(G.gq_hessian_workspace_size(max_tokens, n), dev),
                ws_prep=G.workspace(G.gq_prepare_workspace_size(n), dev))
        # one quantize workspace per layer shape (layers run one after another on one stream)
        self._ws_quant = {}
        self.out = {}
        for name, m, n, key in self.layers:
            if (m, n) not in self._ws_quant:
                self._ws_quant[(m, n)] = G.workspace(G.gq_quantize_workspace_size(m, n, cfg), dev)
            ng = 1 if cfg.group_size == 0 else -(-n // cfg.group_size)
            ncols = n if cfg.clip == "unbounded" else G.n_words(n, cfg.bits)
            self.out[name] = dict(
                codes=torch.empty((m, ncols), dtype=torch.int32, device=dev),
                scales=torch.empty((m, ng), dtype=torch.float32, device=dev),
                zeros=torch.empty((m, ng), dtype=torch.uint8, device=dev),
                loss=torch.empty(3, dtype=torch.float64, device=dev))

    def weights(self) -> int:
        return sum(m * n for _, m, n, _ in self.layers)

    def hessian(self, key: str, X: torch.Tensor, stream=None):
        """H = 2 X^T X of one input."""
        d = self.inputs[key]
        if X.shape[0] > self.max_tokens:
            raise ValueError(f"{X.shape[0]} tokens exceed {self.max_tokens}")
        G.gq_hessian_accumulate(d["H"], X, accumulate=False, ws=d["ws_hess"], stream=stream)

    def prepare(self, key: str, stream=None):
        """U (and the dead mask, the damping) of one input from its H."""
        d = self.inputs[key]
        G.gq_prepare_hinv(d["H"], self.damp, self.cfg.reverse, d["U"], d["dead"], d["delta"],
                          d["ws_prep"], stream=stream)

    def factor(self, key: str, X: torch.Tensor, stream=None):
        """H and U of one input."""
        self.hessian(key, X, stream=stream)
        self.prepare(key, stream=stream)

    def quantize(self, name: str, W: torch.Tensor, stream=None):
        _, m, n, key = next(l for l in self.layers if l[0] == name)
        d, o = self.inputs[key], self.out[name]
        G.gq_quantize_layer(W, d["U"], d["dead"], d["delta"], self.cfg, o["codes"], o["scales"],
                            o["zeros"], o["loss"], self._ws_quant[(m, n)], stream=stream)

    def run(self, Ws: dict, Xs: dict, names=None, stream=None) -> dict:
        """The factor of every input that the layers ``names`` (default: all) read, then those
        layers; returns {name: out buffers}."""
        names = [l[0] for l in self.layers] if names is None else list(names)
        keys = []
        for name, _, _, key in self.layers:
            if name in names and key not in keys:
                keys.append(key)
        for key in keys:
            self.factor(key, Xs[key], stream=stream)
        for name in names:
            self.quantize(name, Ws[name], stream=stream)
        return {name: self.out[name] for name in names}

    def status(self):
        """Worst device status over every workspace (0 if all are clean); synchronizes."""
        codes = []
        for d in self.inputs.values():
            codes.append(G.gq_workspace_status(d["ws_prep"])[0])
        for ws in self._ws_quant.values():
            codes.append(G.gq_workspace_status(ws)[0])
        bad = [c for c in codes if c != 0]
        return bad[0] if bad else 0


# ---------------------------------------------------------------------------------------------
# A sweep over many blocks with per-layer checkpoints
# ---------------------------------------------------------------------------------------------

class SweepCheckpoint:
    """Per-layer results of a long sweep on disk, so that an interrupted sweep resumes at the
    first layer without a result.  One file per (tag, block, layer): the layer's codes, scales,
    zeros and losses as host tensors (``torch.save``), written to a temporary name and renamed,
    so a file that exists is complete."""

    def __init__(self, directory: str, tag: str):
        import os
        self.dir, self.tag = directory, tag
        os.makedirs(directory, exist_ok=True)

    def path(self, block: int, layer: str) -> str:
        import os
        return os.path.join(self.dir, f"{self.tag}.b{block:03d}.{layer}.pt")

    def done(self, block: int, layer: str) -> bool:
        import os
        return os.path.exists(self.path(block, layer))

    def save(self, block: int, layer: str, tensors: dict):
        import os
        p = self.path(block, layer)
        host = {k: v.detach().to("cpu").clone() for k, v in tensors.items()}
        torch.save(host, p + ".tmp")
        os.replace(p + ".tmp", p)

    def load(self, block: int, layer: str) -> dict:
        return torch.load(self.path(block, layer))


def run_sweep(blocks, layers, make_inputs, quantize_block, ckpt: SweepCheckpoint,
              on_layer=None) -> int:
    """Quantize ``blocks`` (an iterable of block indices) of ``layers`` ((name, m, n,
    input_key) tuples), skipping every layer that ``ckpt`` already holds.

    ``make_inputs(block)`` returns (Ws, Xs) for one block; ``quantize_block(Ws, Xs, names)``
    quantizes the named layers (and the inputs they need) and returns {name: tensors}.  A block
    whose layers are all checkpointed is not regenerated.  Returns the number of layers run."""
    ran = 0
    for b in blocks:
        todo = [l[0] for l in layers if not ckpt.done(b, l[0])]
        if not todo:
            continue
        Ws, Xs = make_inputs(b)
        res = quantize_block(Ws, Xs, todo)
        for name in todo:
            ckpt.save(b, name, res[name])
            ran += 1
            if on_layer is not None:
                on_layer(b, name)
    return ran
