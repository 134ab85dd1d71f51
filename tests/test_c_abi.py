"""The boundary is a C ABI: a program built against include/nshb.h (as C11 and as C++17) and linked with
libnshb.so sees the same struct layouts, defaults, workspace sizes and argument errors as
the ctypes binding (CPU only: nothing here launches a kernel)."""
import ctypes
import pathlib
import shutil
import subprocess

import pytest

import newton_schulz_hyperball_b200 as nshb
from newton_schulz_hyperball_b200 import _abi

ROOT = pathlib.Path(__file__).resolve().parents[1]


def fake(shapes):
    arr = (nshb.nshb_matrix * len(shapes))()
    for i, ((r, c), base) in enumerate(zip(shapes, (0x10000000, 0x20000000, 0x30000000))):
        arr[i].rows, arr[i].cols, arr[i].ld, arr[i].w_dtype, arr[i].z_index = r, c, c, nshb.NSHB_BF16, -1
        arr[i].W, arr[i].G, arr[i].M = base, base + 0x4000000, base + 0x8000000
    arr._n = len(shapes)
    return arr


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c11"), ("g++", "-std=c++17")])
def test_c_program_sees_the_same_abi(tmp_path, compiler, std):
    if shutil.which(compiler) is None:
        pytest.skip(f"needs {compiler}")
    lib_dir = pathlib.Path(_abi.LIB_PATH).parent
    exe = tmp_path / "c_abi_check"
    lang = ["-x", "c++"] if compiler == "g++" else []
    subprocess.run([compiler, std, "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", str(ROOT / "include"),
                    *lang, str(ROOT / "tests" / "c_abi_check.c"), "-x", "none", "-L", str(lib_dir), "-lnshb",
                    f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert int(got["sizeof_matrix"]) == ctypes.sizeof(_abi.nshb_matrix)
    assert int(got["sizeof_params"]) == ctypes.sizeof(_abi.nshb_params)
    assert int(got["sizeof_adam"]) == ctypes.sizeof(_abi.nshb_adam_params)
    assert int(got["offset_coeffs"]) == _abi.nshb_params.coeffs.offset
    assert int(got["offset_rho"]) == _abi.nshb_params.rho.offset
    assert got["defaults"] == "0.9500 5 256 1 0.9990"
    mats = fake([(768, 768), (3072, 768), (5, 7)])
    p = nshb.params()
    assert int(got["ws_status"]) == nshb.NSHB_OK
    assert int(got["ws_bytes"]) == nshb.workspace_size(mats, p, nshb.NSHB_OP_HYPERBALL)
    assert int(got["adam_status"]) == nshb.NSHB_OK
    assert int(got["adam_bytes"]) == nshb.workspace_size(mats, p, nshb.NSHB_OP_ADAMH)
    assert got["null_ws"] == "NSHB_ERR_NULL"
    assert got["short_ws"] == "NSHB_ERR_WORKSPACE"
    assert got["bad_shape"] == "NSHB_ERR_SHAPE"
    assert int(got["version"]) == nshb.lib().nshb_version()
