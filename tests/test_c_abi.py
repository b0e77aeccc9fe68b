"""include/tp.h compiles as strict C99 and a C program links against libtp.so and gets the
documented answers on every path that returns before a launch (CPU only: no call reaches the GPU)."""
import os
import shutil
import subprocess

import pytest

import tensor_sharded_matmul_b200 as tp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def c_output(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path_factory.mktemp("c_abi") / "c_abi_check")
    libdir = os.path.dirname(tp.LIB_PATH)
    cmd = [cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", exe, "-L", libdir, "-ltp", f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    return dict(line.split(" ", 1) for line in r.stdout.strip().splitlines())


def test_header_compiles_as_c99_and_links(c_output):
    assert c_output["status_ok"] == "ok"
    assert c_output["status_unknown"] == "unknown status"


def test_empty_inputs_and_validation_from_c(c_output):
    assert int(c_output["empty_rs"]) == tp.TP_OK
    assert int(c_output["empty_mlp"]) == tp.TP_OK
    assert int(c_output["bad_t"]) == tp.TP_EINVAL
    assert int(c_output["indivisible"]) == tp.TP_EDIVIS
    assert int(c_output["last_error_nonempty"]) == 1
    assert int(c_output["negative"]) == tp.TP_EINVAL
    assert int(c_output["empty_contraction"]) == tp.TP_EINVAL


def test_workspace_sizes_from_c(c_output):
    assert int(c_output["ws_case4_gather_w"]) == 0                 # W's pieces read in place
    assert int(c_output["ws_case4_gather_w_ragged"]) == 4 * 8192 * 384 * 2   # F/t = 96: gathered copy
    assert int(c_output["ws_case3_fused"]) == 0
    assert c_output["choose_case2"] == f"{tp.TP_OK} {tp.TP_CASE2_ALLGATHER}"
    assert c_output["choose_case4"] == f"{tp.TP_OK} {tp.TP_CASE4_GATHER_X}"
    assert int(c_output["choose_case3"]) == tp.TP_EUNSUPPORTED
