"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI, unpack codes."""
from __future__ import annotations

import numpy as np
import torch


def unpack_np(packed: np.ndarray, n: int, bits: int) -> np.ndarray:
    """LSB-first b-bit codes from uint32 words (the layout gq.h documents)."""
    p = packed.astype(np.uint64) & np.uint64(0xFFFFFFFF)
    pos = np.arange(n) * bits
    wi, off = pos // 32, (pos % 32).astype(np.uint64)
    lo = p[:, wi] >> off
    nxt = np.minimum(wi + 1, p.shape[1] - 1)
    hi = np.where((off + np.uint64(bits)) > 32, p[:, nxt] << (np.uint64(32) - off), 0)
    return ((lo | hi) & np.uint64((1 << bits) - 1)).astype(np.int64)


def run_gpu(W: torch.Tensor, X: torch.Tensor, bits: int, group: int = 0, reverse: bool = False,
            clip: bool = True, damp: float = 0.01, order=None, perm=None, spacing="uniform",
            ladder_max: int = 8):
    from post_weight_quantization_22_b200 import gq as G
    from post_weight_quantization_22_b200.pipeline import LayerQuantizer

    m, n = W.shape
    cfg = G.QuantCfg(bits=bits, group_size=group, reverse=reverse, clip=clip, spacing=spacing,
                     ladder_max=ladder_max)
    lq = LayerQuantizer(m, n, cfg, device="cuda", damp=damp, order=order)
    if perm is not None:
        lq.perm.copy_(torch.as_tensor(np.asarray(perm), dtype=torch.int32))
    res = lq.run(W.cuda().contiguous(), X.cuda().contiguous())
    torch.cuda.synchronize()
    sp, sq, rounds = lq.status()
    if clip == "unbounded":  # int32 codes, original column order
        packed = None
        codes = res.codes.cpu().numpy().astype(np.int64)
    else:
        packed = res.codes.cpu().numpy().view(np.uint32)
        codes = unpack_np(packed, n, bits)
    return dict(H=res.H.cpu().numpy(), U=res.U.cpu().numpy(), packed=packed,
                codes=codes, scales=res.scales.cpu().numpy(), codes_dev=res.codes,
                zeros=res.zeros.cpu().numpy().astype(np.int64), loss=res.loss.cpu().numpy(),
                dead=res.dead.cpu().numpy().astype(bool), delta=float(res.delta.item()),
                status=(sp, sq), rounds=rounds,
                perm=None if lq.perm is None else lq.perm.cpu().numpy().astype(np.int64),
                kappa=G.gq_zsic_spacing(res.U).cpu().numpy() if spacing == "zsic" else None)


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
