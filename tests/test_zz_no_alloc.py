"""gq_prepare_hinv_static: the factor preparation for callers that cannot allocate device memory
(fixed memory plans, graph capture that forbids cudaMalloc, hosts that pass only inputs and
outputs).  It must give what gq_prepare_hinv gives on the same H, call after call, although
all its calls share one scratch array built into the library.

This file is collected last on purpose, and passes both alone in a fresh process and after
the other tests.
"""
import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_22_b200 import synth
from tests.gpu_helpers import rel_fro

pytestmark = pytest.mark.gpu

U_REL = 1e-6  # the factor parity tolerance of the GPU tests (fp64 factor stored in fp32)


def _hessian(n, T, seed_m):
    from post_weight_quantization_22_b200 import gq as G
    _, X, _ = synth.workload("q_proj_4096x4096", m=seed_m, n=n, T=T)
    H = torch.zeros((n, n), dtype=torch.float64, device="cuda")
    G.gq_hessian_accumulate(H, X.cuda())
    return H


def test_static_scratch_matches_workspace_call_twice_in_a_row():
    from post_weight_quantization_22_b200 import gq as G
    cases = [(1000, 1200, False), (257, 300, True), (1024, 1100, False)]
    for n, T, reverse in cases:
        H = _hessian(n, T, 4)
        U1, dead1, delta1, ws = G.gq_prepare_hinv(H, 0.01, reverse)
        U2, dead2, delta2, status = G.gq_prepare_hinv_static(H, 0.01, reverse)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert G.gq_workspace_status(ws)[0] == 0
        assert rel_fro(np.triu(U2.cpu().numpy()), np.triu(U1.cpu().numpy())) <= U_REL
        assert torch.equal(dead1, dead2)
        assert abs(float(delta2.item()) - float(delta1.item())) <= 1e-12 * abs(float(delta1.item()))
        # and against the fp64 oracle's factor of the damped Hessian in the processing order
        # (last to first when reverse: the factor of the column-reversed matrix)
        hfix, _, _ = O.fix_dead_features(H.cpu().numpy(), np.zeros((1, n)))
        hd, _ = O.dampen(hfix, 0.01)
        if reverse:
            hd = hd[::-1, ::-1]
        assert rel_fro(np.triu(U2.cpu().numpy()), O.hinv_upper_factor(hd)) <= U_REL


def test_static_scratch_reports_status_and_rejects_large_n():
    from post_weight_quantization_22_b200 import gq as G
    H = -torch.eye(64, dtype=torch.float64, device="cuda")
    _, _, _, status = G.gq_prepare_hinv_static(H, 0.01)
    torch.cuda.synchronize()
    assert int(status.item()) == 2  # not positive definite
    H = _hessian(300, 400, 4)
    _, _, _, status = G.gq_prepare_hinv_static(H, 0.01)
    torch.cuda.synchronize()
    assert int(status.item()) == 0  # the earlier call's error does not persist
    big = torch.zeros((1025, 1025), dtype=torch.float64, device="cuda")
    with pytest.raises(G.GQError) as e:
        G.gq_prepare_hinv_static(big, 0.01)
    assert e.value.code == 1
