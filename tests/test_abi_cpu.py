"""The C-ABI library loads on a machine without a GPU and exports every declared entry point.

No compute call is made here (no GPU); only the size queries and string functions, which touch
no device, are exercised.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "gq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gq_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    from post_weight_quantization_22_b200 import gq as G
    names = _declared()
    assert "gq_hessian_accumulate" in names and "gq_quantize_layer" in names
    missing = [n for n in names if not hasattr(G.LIB, n)]
    assert not missing, missing
    assert set(G.EXPORTED) <= set(names)


def test_size_queries_and_strings_without_gpu():
    from post_weight_quantization_22_b200 import gq as G
    assert G.gq_version().startswith("gq ")
    assert G.LIB.gq_status_string(2) == b"damped Hessian is not positive definite"
    n = 4096
    ps = G.gq_prepare_workspace_size(n)
    assert ps >= 8 * n * n
    cfg = G.QuantCfg(bits=4, group_size=128)
    qs = G.gq_quantize_workspace_size(4096, 4096, cfg)
    assert qs >= 4 * 4096 * 4096
    assert G.gq_prepare_workspace_size(0) == 0
    assert G.gq_quantize_workspace_size(4096, 4096, G.QuantCfg(bits=9)) == 0
    assert G.gq_quantize_workspace_size(16, 16, G.QuantCfg(bits=3, group_size=64, reverse=True)) == 0
    # ZSIC spacing takes a per-row grid and the forward (or ordered) form
    assert G.gq_quantize_workspace_size(16, 16, G.QuantCfg(bits=3, group_size=16, spacing="zsic")) == 0
    assert G.gq_quantize_workspace_size(16, 16, G.QuantCfg(bits=3, reverse=True, spacing="zsic")) == 0
    assert G.gq_quantize_workspace_size(16, 16, G.QuantCfg(bits=3, spacing="zsic")) > 0
    assert G.LIB.gq_kernel_launches() == 0


def test_package_has_no_cpu_fallback():
    """The product path never imports the oracle."""
    pkg = os.path.join(ROOT, "post_weight_quantization_22_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", src, flags=re.M), f
                assert "gptq_oracle" not in src, f


def test_ordered_entry_points_reject_bad_arguments_without_gpu():
    """Argument checks of the ordered calls return before any device work."""
    from post_weight_quantization_22_b200 import gq as G
    L = G.LIB
    fake = ctypes.c_void_p(4096)
    # unknown order value
    assert L.gq_prepare_hinv_ordered(fake, 16, 0.01, 9, fake, fake, fake, fake, fake, 1 << 20,
                                     None) == 1
    # the min-pivot order writes the order: without a perm array it is rejected
    assert L.gq_prepare_hinv_ordered(fake, 16, 0.01, 3, None, fake, fake, fake, fake, 1 << 20,
                                     None) == 1
    # ACT without a perm array
    assert L.gq_prepare_hinv_ordered(fake, 16, 0.01, 2, None, fake, fake, fake, fake, 1 << 20,
                                     None) == 1
    cfg = G.QuantCfg(bits=4)
    c = cfg.c()
    # no perm, and reverse together with a perm
    assert L.gq_quantize_layer_ordered(fake, 0, 4, 16, fake, None, None, ctypes.byref(c), None,
                                       fake, fake, fake, fake, fake, 1 << 20, None) == 1
    c2 = G.QuantCfg(bits=4, reverse=True).c()
    assert L.gq_quantize_layer_ordered(fake, 0, 4, 16, fake, None, None, ctypes.byref(c2), fake,
                                       fake, fake, fake, fake, fake, 1 << 20, None) == 1


def test_quant_cfg_binding_matches_the_header_struct():
    """The ctypes mirror of gq_quant_cfg has the header's fields, in order, with matching types;
    the Python settings map to the C values (clip: clamp 1 / clip-free 0 / lattice 2;
    spacing: uniform 0 / ZSIC 1)."""
    from post_weight_quantization_22_b200 import gq as G
    text = open(os.path.join(ROOT, "include", "gq.h")).read()
    body = re.search(r"typedef struct \{(.*?)\} gq_quant_cfg;", text, flags=re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"\b(int|float)\s+(\w+)\s*;", body)
    assert [n for _, n in fields] == [n for n, _ in G._Cfg._fields_]
    ctype = {"int": ctypes.c_int, "float": ctypes.c_float}
    assert [ctype[t] for t, _ in fields] == [t for _, t in G._Cfg._fields_]
    c = G.QuantCfg(bits=3, clip="unbounded", spacing="zsic").c()
    assert (c.bits, c.clip, c.spacing) == (3, 2, 1)
    c = G.QuantCfg(bits=4, clip=False).c()
    assert (c.clip, c.spacing) == (0, 0)


def test_wait_test_setting_is_host_only_and_checked():
    from post_weight_quantization_22_b200 import gq as G
    assert G.LIB.gq_debug_wait_test(0, 2) == 1          # withhold must be 0 or 1
    assert G.LIB.gq_debug_wait_test(4096, 1) == 0       # a host-side setting: no GPU needed
    assert G.LIB.gq_debug_wait_test(0, 0) == 0          # back to the defaults


def test_ssqr_entry_rejects_bad_arguments_without_gpu():
    from post_weight_quantization_22_b200 import gq as G
    assert G.LIB.gq_ssqr_workspace_size(0, 16) == 0
    assert G.LIB.gq_ssqr_workspace_size(16, 16) > 0
    # density outside [0, 1], bits outside 2..8: rejected before any device work
    args = [None, 0, 16, 16, None, None, None]
    for bits, density in ((3, -0.1), (3, 1.5), (1, 0.1), (9, 0.1)):
        rc = G.LIB.gq_ssqr_quantize_layer(*args, bits, density, 20, 12, None, None, None, None,
                                          None, None, None, 0, None, None, 0, None)
        assert rc == 1, (bits, density, rc)


def test_hptq_entry_rejects_bad_arguments_without_gpu():
    from post_weight_quantization_22_b200 import gq as G
    assert G.LIB.gq_hptq_workspace_size(0, 16) == 0
    assert G.LIB.gq_hptq_workspace_size(16, 16) > G.LIB.gq_huffman_workspace_size(256)
    # budget not positive, bits outside 2..8, steps outside 0..60: rejected before any device work
    args = [None, 0, 16, 16, None, None, None]
    for bits, budget, steps in ((3, 0.0, 12), (3, -1.0, 12), (1, 3.0, 12), (9, 3.0, 12),
                                (3, 3.0, 61)):
        rc = G.LIB.gq_hptq_quantize_layer(*args, bits, budget, steps, 12, None, None, None,
                                          None, None, None, 0, None)
        assert rc == 1, (bits, budget, steps, rc)
