"""The C-ABI library builds, loads and exports every entry point the header
declares; host-side argument checks answer without touching a GPU."""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "gce.h")


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^GCE_API\s+[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared()
    for fn in ("ef_topk_step", "ef_randk_step", "powersgd_step", "accordion_select",
               "decompress_accumulate", "gce_table_create", "gce_workspace_bytes", "gce_status"):
        assert fn in names


def test_library_exports_every_declared_symbol():
    from gradient_compression_error_b200 import build
    lib = build.build()
    out = subprocess.run(["nm", "-D", "--defined-only", lib], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in declared() if n not in exported]
    assert not missing, missing
    # nothing beyond the header leaks out of the library
    extra = [n for n in exported if n not in declared()]
    assert not extra, extra


def test_binding_covers_the_header_and_loads():
    import gradient_compression_error_b200 as gce
    assert sorted(gce.SIGNATURES) == declared()
    L = gce.lib()
    for n in declared():
        assert getattr(L, n) is not None


def test_null_arguments_are_rejected_on_the_host():
    import gradient_compression_error_b200 as gce
    L = gce.lib()
    assert L.gce_table_create(None, 1, None) == -1
    assert L.ef_topk_step(None, 1, None, None, 0.1, None, None, None, None, 0, None) == -1
    assert L.ef_randk_step(None, 1, None, None, 0.1, None, 0, 0, None, None, None, 0, None) == -1
    assert L.powersgd_step(None, 1, None, None, 0.1, None, None, None, None, None, None, 0,
                           None) == -1
    assert L.decompress_accumulate(None, 1, None, None, None, None, None, 1.0, None, None, 0,
                                   None) == -1
    assert L.gce_set_bracket_sigma(C.c_double(float("nan"))) == -1
    assert L.decompress_apply(None, 1, None, None, None, None, None, 1.0, None, None, 0,
                              None) == -1
    assert L.powersgd_dp_step(None, 1, None, None, 0.1, None, None, None, None, None, 0,
                              None) == -1
    assert L.ef_sign_step(None, 1, None, None, 0.1, None, None, 0, None) == -1
    assert L.gce_set_randk_ahead(2) == -1
    assert L.gce_set_sign_ahead(-2) == -1 and L.gce_set_sign_ahead((1 << 20) + 1) == -1
    assert L.gce_set_sign_ahead(-1) == 0                           # back to the default
    assert L.gce_set_sign_emit_first(2) == -1 and L.gce_set_sign_emit_first(0) == 0
    assert L.decompress_vote(None, 1, None, 1.0, None, None) == -1
    v = C.c_double()
    assert L.gce_table_set_option(None, 0, 1.0) == -1
    assert L.gce_table_reset_option(None, 0) == -1
    assert L.gce_table_get_option(None, 0, C.byref(v)) == -1
    assert L.gce_set_bracket_sigma(C.c_double(100.0)) == -1
    assert L.gce_set_bracket_sigma(C.c_double(6.0)) == 0          # back to the default
    e = C.c_float()
    assert L.gce_memsgd_eta(0, 0.0, 1.0, C.byref(e)) == -1        # mu <= 0
    assert L.gce_memsgd_eta(3, 1.0, -3.0, C.byref(e)) == -1       # a + t <= 0
    assert L.gce_memsgd_eta(-1, 1.0, 5.0, C.byref(e)) == -1       # t < 0
    assert L.gce_memsgd_eta(0, 1.0, 1.0, None) == -1
    assert L.gce_error_string(-3) == b"workspace missing or too small"


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "gradient_compression_error_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "liboracle" not in text and "gce_oracle" not in text, f


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    import gradient_compression_error_b200 as gce
    monkeypatch.setattr(gce, "_lib", None)
    monkeypatch.setattr(gce, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError):
        gce.lib()


def test_memsgd_eta_matches_the_oracle():
    """The step-size helper is host code: checked here against the oracle."""
    import gradient_compression_error_b200 as gce
    from oracle import steps
    for t, mu, a in [(0, 1.0, 8.0), (7, 0.01, 1000.0), (123456, 3.5, 0.25), (1, 1e-3, 1.0)]:
        assert np.float32(gce.memsgd_eta(t, mu, a)) == steps.memsgd_eta(t, mu, a)
