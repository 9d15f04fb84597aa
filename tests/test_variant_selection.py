"""KQ_VAR_AUTO's choice (host-only, through kq_select_variant): the table of
measured winners agrees with the committed sweep, bf16 matrices and fp32 without
the factored form always take the tensor core, and the KQ_VARIANT override
applies where the named variant can serve the call."""
from __future__ import annotations

import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SWEEP = os.path.join(ROOT, "profiles", "kq_quant_sweep.md")


@pytest.fixture(scope="module")
def kq():
    from mxfp4_activations_b200 import build

    build.build()
    import mxfp4_activations_b200 as m

    m.load()
    return m


def sweep_winners():
    """{(M, d): "butterfly" | "mma"} from the sweep table's KroQuant (butterfly) and
    tensor-core (fp32 K) columns, for the shape-sweep rows."""
    rows = {}
    header = None
    for line in open(SWEEP):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if header is None and "config" in cells and "M × d" in cells:
            header = cells
            continue
        if header is None or len(cells) != len(header) or cells[0] != "sweep":
            continue
        M, d = (int(v) for v in re.findall(r"\d+", cells[header.index("M × d")]))
        bfly = float(cells[header.index("kroquant µs")])
        mma = float(cells[header.index("mma µs")])
        rows[(M, d)] = "butterfly" if bfly <= mma else "mma"
    return rows


def test_auto_table_matches_the_committed_sweep(kq):
    win = sweep_winners()
    assert len(win) == 18
    for (M, d), v in win.items():
        assert kq.kq_select_variant(M, d) == v, (M, d)


def test_auto_fixed_choices(kq):
    import torch

    for M, d in [(1, 32), (64, 1152), (4608, 12288), (10**6, 65536)]:
        assert kq.kq_select_variant(M, d, torch.bfloat16) == "mma"
        assert kq.kq_select_variant(M, d, torch.float32, has_factored=False) == "mma"
    assert kq.kq_select_variant(4608, 3072, log2n=6) == "butterfly"
    lib = kq.load()
    import ctypes

    out = ctypes.c_int(-1)
    assert lib.kq_select_variant(4, 64, 6, 1, 1, ctypes.byref(out)) == 5   # 64-element blocks: fp32 only
    assert lib.kq_select_variant(4, 64, 8, 0, 1, ctypes.byref(out)) == 1
    assert lib.kq_select_variant(4, 64, 4, 0, 1, ctypes.byref(out)) == 0 and out.value == 2
    assert lib.kq_select_variant(-1, 64, 5, 0, 1, ctypes.byref(out)) == 1
    assert lib.kq_select_variant(4, 64, 5, 0, 1, None) == 1


@pytest.mark.parametrize("env,mdt,fac,want", [("mma", "f32", 1, "mma"), ("butterfly", "f32", 1, "butterfly"),
                                              ("butterfly", "bf16", 1, "mma"), ("butterfly", "f32", 0, "mma")])
def test_environment_override(kq, env, mdt, fac, want):
    code = ("import sys; sys.path.insert(0, %r)\n"
            "import torch, mxfp4_activations_b200 as kq\n"
            "print(kq.kq_select_variant(4608, 12288, torch.%s, has_factored=%d))\n") % (
                ROOT, "float32" if mdt == "f32" else "bfloat16", fac)
    out = subprocess.run([sys.executable, "-c", code], env={**os.environ, "KQ_VARIANT": env},
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip().splitlines()[-1] == want
