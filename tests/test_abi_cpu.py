"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/nshb.h declares, and rejects bad arguments synchronously, before any
CUDA call is made."""
import ctypes
import pathlib
import re

import pytest

import newton_schulz_hyperball_b200 as nshb
from newton_schulz_hyperball_b200 import _abi

HEADER = pathlib.Path(__file__).resolve().parents[1] / "include" / "nshb.h"


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                                 text, flags=re.M)))


def test_library_exports_every_declared_function():
    lib = nshb.lib()
    names = declared_functions()
    assert {"muon_step", "hyperball_step", "radial_brake_step", "himuon_step", "newton_muon_step",
            "nshb_workspace_size", "nshb_fro_norms", "nshb_device_status", "nshb_status_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_abi.SIGNATURES)


def test_struct_layouts_match_header():
    assert ctypes.sizeof(_abi.nshb_matrix) == 64
    assert ctypes.sizeof(_abi.nshb_params) == 80
    assert _abi.nshb_params.coeffs.offset == 16 and _abi.nshb_params.rho.offset == 40


def test_defaults_and_strings():
    p = nshb.params()
    assert abs(p.beta - 0.95) < 1e-7 and p.nesterov == 1 and p.ns_steps == 5
    assert abs(p.ns_eps - 1e-7) < 1e-12 and abs(p.hb_eps - 1e-8) < 1e-13
    assert p.ns_precision == nshb.NSHB_BF16 and p.tile == 256 and p.ns_compensated == 2
    assert nshb.lib().nshb_status_string(nshb.NSHB_ERR_WORKSPACE) == b"NSHB_ERR_WORKSPACE"
    assert nshb.lib().nshb_version() >= 100


def fake_mats(shapes, dtype=nshb.NSHB_BF16, ld=None):
    arr = (nshb.nshb_matrix * len(shapes))()
    for i, (r, c) in enumerate(shapes):
        arr[i].rows, arr[i].cols = r, c
        arr[i].ld = c if ld is None else ld
        arr[i].w_dtype = dtype
        arr[i].z_index = -1
        base = 0x10000000 * (i + 1)
        arr[i].W, arr[i].G, arr[i].M = base, base + 0x4000000, base + 0x8000000
    arr._n = len(shapes)
    return arr


def ws_size(mats, p, op):
    return nshb.workspace_size(mats, p, op)


def test_workspace_size_grows_with_matrices_and_orientation():
    p = nshb.params()
    a = ws_size(fake_mats([(768, 768)]), p, nshb.NSHB_OP_HYPERBALL)
    b = ws_size(fake_mats([(768, 768), (3072, 768)]), p, nshb.NSHB_OP_HYPERBALL)
    c = ws_size(fake_mats([(768, 768), (768, 3072)]), p, nshb.NSHB_OP_HYPERBALL)
    assert 0 < a < b and b == c      # tall and wide matrices use the same wide-side buffers
    # bf16 NS keeps X twice (ping-pong) and the two r x r Gram/polynomial matrices.
    assert a >= 2 * 768 * 768 * 2 * 2
    f = nshb.params(ns_precision=nshb.NSHB_F32)
    assert ws_size(fake_mats([(768, 768)], nshb.NSHB_F32), f, nshb.NSHB_OP_HYPERBALL) >= 4 * 768 * 768 * 4


@pytest.mark.parametrize("shape,code", [((0, 5), nshb.NSHB_ERR_SHAPE), ((5, -1), nshb.NSHB_ERR_SHAPE)])
def test_bad_shapes(shape, code):
    with pytest.raises(nshb.NshbError) as e:
        ws_size(fake_mats([shape]), nshb.params(), nshb.NSHB_OP_MUON)
    assert e.value.status == code


def test_ld_smaller_than_cols():
    with pytest.raises(nshb.NshbError) as e:
        ws_size(fake_mats([(8, 16)], ld=8), nshb.params(), nshb.NSHB_OP_MUON)
    assert e.value.status == nshb.NSHB_ERR_SHAPE


def test_null_pointers():
    m = fake_mats([(8, 8)])
    m[0].G = None
    with pytest.raises(nshb.NshbError) as e:
        ws_size(m, nshb.params(), nshb.NSHB_OP_MUON)
    assert e.value.status == nshb.NSHB_ERR_NULL
    lib = nshb.lib()
    assert lib.muon_step(fake_mats([(8, 8)]), 1, None, None, 0, None) == nshb.NSHB_ERR_NULL
    assert lib.nshb_device_status(None, None, None) == nshb.NSHB_ERR_NULL


def test_bad_dtype():
    with pytest.raises(nshb.NshbError) as e:
        ws_size(fake_mats([(8, 8)], dtype=7), nshb.params(), nshb.NSHB_OP_MUON)
    assert e.value.status == nshb.NSHB_ERR_DTYPE
    with pytest.raises(nshb.NshbError) as e:
        ws_size(fake_mats([(8, 8)]), nshb.params(ns_precision=3), nshb.NSHB_OP_MUON)
    assert e.value.status == nshb.NSHB_ERR_DTYPE


@pytest.mark.parametrize("kw,op", [
    (dict(beta=1.0), nshb.NSHB_OP_MUON),
    (dict(beta=-0.1), nshb.NSHB_OP_MUON),
    (dict(ns_steps=0), nshb.NSHB_OP_MUON),
    (dict(ns_steps=33), nshb.NSHB_OP_MUON),
    (dict(ns_eps=0.0), nshb.NSHB_OP_MUON),
    (dict(hb_eps=0.0), nshb.NSHB_OP_HYPERBALL),
    (dict(eta=-1.0), nshb.NSHB_OP_HYPERBALL),
    (dict(brake_out=1.5), nshb.NSHB_OP_RADIAL_BRAKE),
    (dict(brake_in=-0.1), nshb.NSHB_OP_RADIAL_BRAKE),
    (dict(weight_decay=0.1), nshb.NSHB_OP_RADIAL_BRAKE),
    (dict(tile=100), nshb.NSHB_OP_HIMUON),
    (dict(ridge_rel=-1.0), nshb.NSHB_OP_NEWTON_MUON),
    (dict(coeffs=[(float("nan"), 0, 0)] * 5), nshb.NSHB_OP_MUON),
    (dict(ns_compensated=-1), nshb.NSHB_OP_MUON),
    (dict(ns_compensated=33), nshb.NSHB_OP_MUON),
])
def test_bad_params(kw, op):
    with pytest.raises(nshb.NshbError) as e:
        ws_size(fake_mats([(8, 8)]), nshb.params(**kw), op)
    assert e.value.status == nshb.NSHB_ERR_PARAM


def test_workspace_too_small_or_misaligned_is_rejected_before_launch():
    lib = nshb.lib()
    m = fake_mats([(64, 64)])
    p = nshb.params()
    for fn, op in ((lib.muon_step, nshb.NSHB_OP_MUON), (lib.hyperball_step, nshb.NSHB_OP_HYPERBALL),
                   (lib.radial_brake_step, nshb.NSHB_OP_RADIAL_BRAKE)):
        need = ws_size(m, p, op)
        assert fn(m, 1, ctypes.byref(p), 0x20000000, need - 256, None) == nshb.NSHB_ERR_WORKSPACE
        assert fn(m, 1, ctypes.byref(p), 0x20000010, need, None) == nshb.NSHB_ERR_WORKSPACE
        assert fn(m, 1, ctypes.byref(p), None, need, None) == nshb.NSHB_ERR_NULL


def test_zero_matrices_is_a_no_op():
    lib = nshb.lib()
    p = nshb.params()
    assert lib.hyperball_step(None, 0, ctypes.byref(p), None, 0, None) == nshb.NSHB_OK


def test_adam_params_layout_defaults_and_argument_errors():
    assert ctypes.sizeof(_abi.nshb_adam_params) == 16
    a = nshb.adam_params()
    assert abs(a.beta1 - 0.9) < 1e-7 and abs(a.beta2 - 0.999) < 1e-7 and abs(a.eps - 1e-8) < 1e-13 and a.step == 1
    mats = fake_mats([(64, 64), (100, 30)])
    p = nshb.params()
    n = nshb.workspace_size(mats, p, nshb.NSHB_OP_ADAMH)
    assert n > 0
    # RelativeUpdate adds the (||O||^2, <W,O>, ||W||^2) records to the Muon step's workspace
    assert nshb.workspace_size(mats, p, nshb.NSHB_OP_RELATIVE_UPDATE) >= nshb.workspace_size(mats, p, nshb.NSHB_OP_MUON)
    V = [0x30000000, 0x31000000]
    ws = (0x40000000, n)
    for bad in (dict(step=0), dict(beta1=1.0), dict(beta2=-0.1), dict(eps=0.0)):
        with pytest.raises(nshb.NshbError) as e:
            nshb.adamh_step(mats, V, nshb.adam_params(**bad), p, ws, stream=0)
        assert e.value.status == nshb.NSHB_ERR_PARAM
    with pytest.raises(nshb.NshbError) as e:
        nshb.adamh_step(mats, [0x30000000, None], a, p, ws, stream=0)
    assert e.value.status == nshb.NSHB_ERR_NULL
    with pytest.raises(nshb.NshbError) as e:
        nshb.adamh_step(mats, V, a, p, (0x40000000, n - 256), stream=0)
    assert e.value.status == nshb.NSHB_ERR_WORKSPACE


def test_chunked_step_workspace_bounds_are_checked_before_any_launch():
    mats = fake_mats([(768, 768), (3072, 768), (768, 3072), (256, 512)])
    p = nshb.params()
    full = nshb.workspace_size(mats, p, nshb.NSHB_OP_HYPERBALL)
    least = nshb.workspace_size_min(mats, p, nshb.NSHB_OP_HYPERBALL)
    assert 0 < least < full
    one = [nshb.workspace_size(fake_mats([s]), p, nshb.NSHB_OP_HYPERBALL)
           for s in [(768, 768), (3072, 768), (768, 3072), (256, 512)]]
    assert least == max(one)
    with pytest.raises(nshb.NshbError) as e:
        nshb.step_chunked(nshb.NSHB_OP_HYPERBALL, mats, p, (0x40000000, least - 256), stream=0)
    assert e.value.status == nshb.NSHB_ERR_WORKSPACE
    with pytest.raises(nshb.NshbError) as e:
        nshb.step_chunked(nshb.NSHB_OP_NEWTON_MUON, mats, p, (0x40000000, full), stream=0)
    assert e.value.status == nshb.NSHB_ERR_PARAM
    with pytest.raises(nshb.NshbError) as e:
        nshb.workspace_size_min(mats, p, nshb.NSHB_OP_ADAMH)
    assert e.value.status == nshb.NSHB_ERR_PARAM


@pytest.mark.parametrize("shape,ld", [(((1 << 20) + 1, 8), None), ((8, (1 << 20) + 1), None),
                                      ((8, 8), (1 << 30) + 1)])
def test_sizes_beyond_the_documented_limits_are_unsupported(shape, ld):
    with pytest.raises(nshb.NshbError) as e:
        ws_size(fake_mats([shape], ld=ld), nshb.params(), nshb.NSHB_OP_HYPERBALL)
    assert e.value.status == nshb.NSHB_ERR_UNSUPPORTED


def newton_mats(cols_list, z_index):
    m = fake_mats([(768, c) for c in cols_list])
    for i, zi in enumerate(z_index):
        m[i].z_index = zi
    return m


@pytest.mark.parametrize("z_rows,n_tokens,z_index,code", [
    ([768], 8100, [0], nshb.NSHB_ERR_SHAPE),          # tokens not a multiple of 64
    ([768], 0, [0], nshb.NSHB_ERR_SHAPE),
    ([768], (1 << 24) + 64, [0], nshb.NSHB_ERR_SHAPE),
    ([760], 8192, [0], nshb.NSHB_ERR_SHAPE),          # Z rows not a multiple of 64
    ([16384 + 64], 8192, [0], nshb.NSHB_ERR_SHAPE),
    ([768], 8192, [1], nshb.NSHB_ERR_PARAM),          # z_index outside [0, n_z)
    ([768], 8192, [-1], nshb.NSHB_ERR_PARAM),
    ([1536], 8192, [0], nshb.NSHB_ERR_SHAPE),         # Z rows != cols of the matrix
    ([], 8192, [0], nshb.NSHB_ERR_NULL),              # no Z at all
])
def test_newton_muon_argument_errors(z_rows, n_tokens, z_index, code):
    with pytest.raises(nshb.NshbError) as e:
        nshb.workspace_size(newton_mats([768], z_index), nshb.params(), nshb.NSHB_OP_NEWTON_MUON,
                            z_rows=z_rows, n_tokens=n_tokens)
    assert e.value.status == code


def test_newton_muon_workspace_and_step_checks_before_launch():
    p = nshb.params()
    m = newton_mats([768, 768, 3072], [0, 0, 1])
    a = nshb.workspace_size(m, p, nshb.NSHB_OP_NEWTON_MUON, z_rows=[768, 3072], n_tokens=4096)
    b = nshb.workspace_size(m, p, nshb.NSHB_OP_NEWTON_MUON, z_rows=[768, 3072], n_tokens=8192)
    # Z is read where the caller keeps it (no copy), so the workspace does not grow with the
    # token count
    assert b == a
    assert a > nshb.workspace_size(m, p, nshb.NSHB_OP_HYPERBALL)
    with pytest.raises(nshb.NshbError) as e:   # Newton-Muon runs the bf16 NS only
        nshb.workspace_size(m, nshb.params(ns_precision=nshb.NSHB_F32), nshb.NSHB_OP_NEWTON_MUON,
                            z_rows=[768, 3072], n_tokens=4096)
    assert e.value.status == nshb.NSHB_ERR_UNSUPPORTED
    lib = nshb.lib()
    zr = (ctypes.c_int64 * 2)(768, 3072)
    zp = (ctypes.c_void_p * 2)(0x30000000, 0x30000010)
    # Z NULL, a misaligned Z, a short workspace: all rejected before any CUDA call
    assert lib.newton_muon_step(m, 3, None, zr, 2, 4096, ctypes.byref(p), 0x20000000, a, None) == nshb.NSHB_ERR_NULL
    bad = (ctypes.c_void_p * 2)(0x30000000, 0x30000008)
    assert lib.newton_muon_step(m, 3, bad, zr, 2, 4096, ctypes.byref(p), 0x20000000, a, None) == nshb.NSHB_ERR_SHAPE
    assert lib.newton_muon_step(m, 3, zp, zr, 2, 4096, ctypes.byref(p), 0x20000000, a - 256, None) == \
        nshb.NSHB_ERR_WORKSPACE


def test_missing_library_fails_loudly(tmp_path):
    """Without libnshb.so there is no step at all: no CPU fallback, an ImportError that says so."""
    with pytest.raises(ImportError, match="no fallback"):
        _abi.load(str(tmp_path / "libnshb.so"))


def test_package_never_reaches_the_oracle():
    """The product package (binding, planner helpers, sharding) neither imports nor reads
    anything under oracle/: the oracle is test infrastructure only."""
    pkg = pathlib.Path(nshb.__file__).resolve().parent
    for f in sorted(pkg.rglob("*")):
        if f.suffix not in (".py", ".cu", ".cuh", ".h", ".cpp"):
            continue
        text = f.read_text()
        assert not re.search(r"^\s*(from|import)\s+oracle\b", text, flags=re.M), f
        assert "nshb_oracle" not in text, f


def test_matrices_checks_what_the_library_cannot_see():
    """The C ABI gets bare pointers, so the binding checks sizes, dtypes, strides and the
    device before any pointer reaches the library (here with CPU tensors: every error is
    raised before the device check, and a consistent CPU set is refused as not CUDA)."""
    import torch
    W = torch.zeros(8, 16, dtype=torch.bfloat16)
    G = torch.zeros_like(W)
    M = torch.zeros(8, 16)
    cases = [
        (ValueError, dict(G=[torch.zeros(4, 16, dtype=torch.bfloat16)])),          # G smaller than W
        (ValueError, dict(M=[torch.zeros(8, 8)])),                                  # M of another shape
        (TypeError, dict(G=[torch.zeros(8, 16)])),                                  # G fp32 with bf16 W
        (TypeError, dict(M=[torch.zeros(8, 16, dtype=torch.bfloat16)])),            # M not fp32
        (ValueError, dict(O=[torch.zeros(8, 8, dtype=torch.bfloat16)])),            # O_out too small
        (ValueError, dict(O=[torch.zeros(8, 16)])),                                 # O_out of another dtype
        (ValueError, dict(O=[torch.zeros(16, 8, dtype=torch.bfloat16).t()])),       # O_out not contiguous
        (ValueError, dict(W=[torch.zeros(16, 8, dtype=torch.bfloat16).t()])),       # W column stride != 1
        (ValueError, dict(G=[])),                                                   # list lengths differ
        (ValueError, dict()),                                                       # CPU tensors
    ]
    for exc, kw in cases:
        with pytest.raises(exc):
            nshb.matrices(kw.get("W", [W]), kw.get("G", [G]), kw.get("M", [M]), kw.get("O"))
    assert nshb.matrices([], [], [])._n == 0


def test_pointer_arguments_are_checked_before_the_library_sees_them():
    """rho, V, Z, out and the workspace become bare device pointers: host tensors, wrong
    dtypes, short arrays and mismatched lengths are refused by the binding."""
    import torch
    with pytest.raises(ValueError):
        nshb.params(rho=torch.ones(3))                               # rho on the host
    assert getattr(nshb.params(rho=0x30000000), "_rho_n", None) is None  # raw pointer: caller's word
    mats = fake_mats([(64, 64), (100, 30), (8, 8)])
    p = nshb.params()
    p._rho_n = 2                                                     # a 2-entry rho for 3 matrices
    ws = (0x40000000, nshb.workspace_size(mats, nshb.params(), nshb.NSHB_OP_HYPERBALL))
    for fn in (nshb.hyperball_step, nshb.muon_step, nshb.himuon_step, nshb.relative_update_step):
        with pytest.raises(ValueError, match="rho"):
            fn(mats, p, ws, stream=0)
    with pytest.raises(ValueError, match="rho"):
        nshb.step_chunked(nshb.NSHB_OP_HYPERBALL, mats, p, ws, stream=0)
    a = nshb.adam_params()
    with pytest.raises(ValueError):
        nshb.adamh_step(mats, [0x30000000], a, nshb.params(), ws, stream=0)          # V too short
    with pytest.raises(TypeError):
        nshb.adamh_step(mats, [torch.zeros(64, 64)] * 3, a, nshb.params(), ws, stream=0)  # V on the host
    with pytest.raises(ValueError):
        nshb.newton_muon_step(mats, [torch.zeros(64, 128, dtype=torch.bfloat16)], 128, nshb.params(), ws, stream=0)
    with pytest.raises(ValueError):
        nshb.fro_norms(mats, torch.zeros(3), ws, stream=0)           # out on the host
    with pytest.raises(ValueError):
        nshb.fro_norms_static(mats, torch.zeros(3), stream=0)
    with pytest.raises(ValueError):
        nshb.device_status(torch.zeros(256, dtype=torch.uint8))      # workspace on the host


@pytest.mark.parametrize("field,offset", [("W", 1), ("G", 1), ("M", 2)])
def test_pointers_not_element_aligned_are_refused(field, offset):
    """A misaligned element pointer would fault on the device: every entry point that plans a
    step refuses it with NSHB_ERR_SHAPE before anything is queued."""
    m = fake_mats([(64, 64)])
    setattr(m[0], field, getattr(m[0], field) + offset)
    for op in (nshb.NSHB_OP_MUON, nshb.NSHB_OP_HYPERBALL, nshb.NSHB_OP_HIMUON, nshb.NSHB_OP_ADAMH):
        with pytest.raises(nshb.NshbError) as e:
            ws_size(m, nshb.params(), op)
        assert e.value.status == nshb.NSHB_ERR_SHAPE, op
    if field == "W":
        assert nshb.lib().nshb_fro_norms_static(m, 1, 0x1000, None) == nshb.NSHB_ERR_SHAPE


def test_adam_second_moment_not_float_aligned_is_refused():
    m = fake_mats([(64, 64)])
    p = nshb.params()
    n = nshb.workspace_size(m, p, nshb.NSHB_OP_ADAMH)
    with pytest.raises(nshb.NshbError) as e:
        nshb.adamh_step(m, [0x30000002], nshb.adam_params(), p, (0x40000000, n), stream=0)
    assert e.value.status == nshb.NSHB_ERR_SHAPE


def test_misaligned_rho_is_refused():
    m = fake_mats([(64, 64)])
    for op in (nshb.NSHB_OP_HYPERBALL, nshb.NSHB_OP_ADAMH):
        with pytest.raises(nshb.NshbError) as e:
            ws_size(m, nshb.params(rho=0x30000002), op)
        assert e.value.status == nshb.NSHB_ERR_PARAM, op


def test_misaligned_norm_output_is_refused():
    lib = nshb.lib()
    m = fake_mats([(64, 64)])
    assert lib.nshb_fro_norms(m, 1, 0x30000002, 0x40000000, 1 << 20, None) == nshb.NSHB_ERR_SHAPE
    assert lib.nshb_fro_norms_static(m, 1, 0x30000002, None) == nshb.NSHB_ERR_SHAPE


def _no_cuda_device():
    import torch
    return not torch.cuda.is_available()


@pytest.mark.skipif(not _no_cuda_device(), reason="passes fake device pointers: only where no GPU exists")
def test_chunk_partition_is_the_greedy_longest_prefix():
    """nshb_step_chunked fixes its chunk boundaries on the host before its first CUDA call, so
    on a machine without a GPU the partition is reported and the call then stops with
    NSHB_ERR_CUDA.  Each chunk must be the longest run of matrices, from where the last one
    ended, whose workspace fits (brute force over the sizes nshb_workspace_size reports)."""
    shapes = [(768, 768), (3072, 768), (768, 3072), (256, 512), (768, 768), (1024, 256), (64, 64)]
    mats = fake_mats(shapes)
    p = nshb.params()

    def need(i, k):
        return nshb.workspace_size(fake_mats(shapes[i:i + k]), p, nshb.NSHB_OP_HYPERBALL)

    least = nshb.workspace_size_min(mats, p, nshb.NSHB_OP_HYPERBALL)
    full = nshb.workspace_size(mats, p, nshb.NSHB_OP_HYPERBALL)
    for ws_bytes in sorted({least, (least + full) // 2 // 256 * 256, full - 256, full}):
        expect, i = 0, 0
        while i < len(shapes):
            k = max(k for k in range(1, len(shapes) - i + 1) if need(i, k) <= ws_bytes)
            expect, i = expect + 1, i + k
        n = ctypes.c_int32(-1)
        st = nshb.lib().nshb_step_chunked(nshb.NSHB_OP_HYPERBALL, mats, len(shapes), ctypes.byref(p), 0x40000000,
                                          ws_bytes, None, ctypes.byref(n))
        assert st == nshb.NSHB_ERR_CUDA
        assert n.value == expect, (ws_bytes, n.value, expect)
    assert expect == 1   # the whole set fits in `full`
