"""The C-ABI library builds, loads and exports every entry point include/lmoe.h declares.

No compute calls: these run without a GPU.
"""
import os
import re
import subprocess

import pytest

import latent_routing_quantile_b200 as lq
from latent_routing_quantile_b200 import build as lbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "lmoe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lmoe_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def built():
    lbuild.build()
    return lq.lib()


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for name in ("lmoe_create", "lmoe_forward", "lmoe_qb_update", "lmoe_destroy"):
        assert name in syms
    assert set(syms) == set(lq.EXPORTED)


def test_library_exports_every_declared_symbol(built):
    out = subprocess.run(["nm", "-D", "--defined-only", lbuild.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s+(lmoe_\w+)", out))
    missing = set(declared_symbols()) - exported
    assert not missing, missing
    for name in declared_symbols():
        assert hasattr(built, name)


def test_strerror(built):
    assert built.lmoe_strerror(0) == b"ok"
    assert built.lmoe_strerror(-1) == b"invalid argument"
    assert built.lmoe_strerror(-4) == b"unsupported shape"


def test_workspace_query_and_validation(built):
    # host-only entry point: sizes the workspace without touching a GPU
    n = lq.workspace_bytes(1024, 256, 256, 6, 256, 2048, lq.BF16, 8192)
    assert 100 << 20 < n < 1 << 31
    with pytest.raises(lq.LmoeError, match="unsupported"):
        lq.workspace_bytes(1000, 256, 256, 6, 256, 2048, lq.BF16, 8192)   # d not a multiple of 64
    with pytest.raises(lq.LmoeError, match="invalid"):
        lq.workspace_bytes(1024, 256, 256, 300, 256, 2048, lq.BF16, 8192)  # k > E
    with pytest.raises(lq.LmoeError, match="unsupported"):
        lq.workspace_bytes(1024, 256, 96, 6, 256, 2048, lq.BF16, 8192)    # E not a multiple of 64
    # MXFP8 experts: bf16 layers with l and h multiples of 128; the 8-bit expert weights need less
    n8 = lq.workspace_bytes(1024, 256, 256, 6, 256, 2048, lq.BF16, 8192, experts=lq.EXPERTS_MXFP8)
    assert 0 < n8 < n
    with pytest.raises(lq.LmoeError, match="unsupported"):
        lq.workspace_bytes(256, 64, 32, 4, 128, 512, lq.F32, 256, experts=lq.EXPERTS_MXFP8)
    with pytest.raises(lq.LmoeError, match="unsupported"):
        lq.workspace_bytes(1024, 192, 256, 6, 256, 2048, lq.BF16, 8192, experts=lq.EXPERTS_MXFP8)
    with pytest.raises(lq.LmoeError, match="invalid"):
        lq.workspace_bytes(1024, 256, 256, 6, 256, 2048, lq.BF16, 8192, experts=2)


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "latent_routing_quantile_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f


def test_binding_constants_match_the_header():
    """Every flag, mode and status bit the binding passes or reads has the header's value."""
    text = open(os.path.join(ROOT, "include", "lmoe.h")).read()
    defs = {m.group(1): int(m.group(2), 0)
            for m in re.finditer(r"#define\s+LMOE_([A-Z0-9_]+)\s+\(?(-?(?:0x)?[0-9a-fA-F]+)u?\)?", text)}
    pairs = {"F32": lq.F32, "BF16": lq.BF16, "RECORD_STATS": lq.RECORD_STATS, "UPDATE_BIAS": lq.UPDATE_BIAS,
             "ASYNC_OUTPUT": lq.ASYNC_OUTPUT, "QB_LITERAL": lq.QB_LITERAL, "BIAS_SIGN": lq.BIAS_SIGN,
             "STATUS_NAN_SCORE": lq.STATUS_NAN_SCORE, "STATUS_WATCHDOG": lq.STATUS_WATCHDOG,
             "STATUS_BAD_INDEX": lq.STATUS_BAD_INDEX, "NBINS": lq.NBINS,
             "EXPERTS_BF16": lq.EXPERTS_BF16, "EXPERTS_MXFP8": lq.EXPERTS_MXFP8}
    for name, value in pairs.items():
        assert defs.get(name) == value, (name, defs.get(name), value)
    # the forward flags are distinct bits, and the update's rule flags stay out of their way
    fwd = [defs["RECORD_STATS"], defs["UPDATE_BIAS"], defs["ASYNC_OUTPUT"]]
    assert len(set(fwd)) == 3 and all(f & (f - 1) == 0 for f in fwd)
