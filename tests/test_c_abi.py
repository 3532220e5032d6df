"""The C ABI used from plain C: a small program compiled with gcc against include/rf2.h
and linked to librf2.so calls the host-only entry points and the host-side validation
(no GPU needed); its results must equal the oracle's and the documented status codes."""
import os
import shutil
import subprocess

import pytest

import oracle as O
from image_diffusion_dits_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_uses_the_abi(tmp_path):
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    exe = tmp_path / "c_abi_check"
    subprocess.run(["gcc", "-std=c99", "-O1", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", lib_dir, "-lrf2",
                    "-Wl,-rpath," + lib_dir, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    res = dict(ln.split(" ", 1) for ln in out.strip().splitlines())
    og = O.geom(B=1, heads=40, T=21, H=45, W=80, D=128, wt=2, wh=8, ww=8)
    assert int(res["kept"]) == O.kept_count(og, 0.8, True) == 132
    assert int(res["kept_additive"]) == O.kept_count(og, 0.8, True, sink_additive=True)
    flat = O.geom(B=1, heads=40, T=21, H=45, W=80, D=128, wt=2, wh=8, ww=8, no_permute=True)
    assert int(res["kept_no_permute"]) == O.kept_count(flat, 0.8, True) == 119
    assert res["ws_nonzero"] == "1"
    assert int(res["v1_kmax"]) == O.rf1.rf1_kmax(og, O.rf1.Rf1Params())
    assert int(res["v1_kmax_dynamic"]) == O.rf1.rf1_kmax(og, O.rf1.Rf1Params(dynamic=True))
    assert [int(x) for x in res["schedule"].split()] == [O.schedule_action(10, 0.15, 3, s) for s in range(10)]
    assert int(res["attention_null"]) == _lib.RF2_ERR_INVALID_ARG
    assert int(res["kept_bad_sparsity"]) == -_lib.RF2_ERR_INVALID_ARG
    assert int(res["kept_bad_D"]) == -_lib.RF2_ERR_UNSUPPORTED
    assert res["status_text"].startswith("unsupported shape")
