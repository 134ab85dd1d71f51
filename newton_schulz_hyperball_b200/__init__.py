"""B200 (sm_100a) Muon / Hyperball optimizer step.

Python binding of libnshb.so (C ABI in include/nshb.h).  This module only marshals
arguments: the step itself -- momentum, Newton-Schulz, the weight-update rule -- runs in
the library's CUDA kernels.  PyTorch is used for device memory and streams only.

    import newton_schulz_hyperball_b200 as nshb
    mats = nshb.matrices(W_list, G_list, M_list)
    p = nshb.params(eta=0.02, rho=rho_dev)
    ws = nshb.workspace(mats, p, nshb.NSHB_OP_HYPERBALL)
    nshb.hyperball_step(mats, p, ws)
"""
from __future__ import annotations

import ctypes

from . import _abi
from ._abi import (  # noqa: F401  (re-exported constants)
    NSHB_BF16, NSHB_F32, NSHB_OK, NSHB_ERR_NULL, NSHB_ERR_SHAPE, NSHB_ERR_DTYPE, NSHB_ERR_PARAM,
    NSHB_ERR_WORKSPACE, NSHB_ERR_CUDA, NSHB_ERR_DEVICE_TIMEOUT, NSHB_ERR_NONFINITE, NSHB_ERR_ZERO_NORM,
    NSHB_ERR_UNSUPPORTED, NSHB_DEV_ZERO_NORM_FALLBACK, NSHB_DEV_NONFINITE, NSHB_DEV_TIMEOUT,
    NSHB_DEV_ZERO_RADIUS, NSHB_DEV_NOT_SPD, NSHB_OP_MUON, NSHB_OP_HYPERBALL, NSHB_OP_RADIAL_BRAKE,
    NSHB_OP_HIMUON, NSHB_OP_NEWTON_MUON, NSHB_OP_RELATIVE_UPDATE, NSHB_OP_ADAMH, nshb_matrix, nshb_params,
    nshb_adam_params,
)

_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded libnshb.so (raises ImportError if it was not built)."""
    global _LIB
    if _LIB is None:
        _LIB = _abi.load()
    return _LIB


class NshbError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {lib().nshb_status_string(status).decode()}"
        if status == NSHB_ERR_CUDA:
            msg += f" (cudaError {lib().nshb_last_cuda_error()})"
        super().__init__(msg)


def _check(status: int, where: str) -> None:
    if status != NSHB_OK:
        raise NshbError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _device_arg(t, what: str, dtype=None, min_numel: int = 0) -> None:
    """Checks a tensor that becomes a bare device pointer: on a CUDA device, contiguous, of
    `dtype` and at least `min_numel` elements.  Raw pointers (ints) and None pass unchecked."""
    if t is None or isinstance(t, int):
        return
    if t.device.type != "cuda":
        raise ValueError(f"{what} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if t.numel() < min_numel:
        raise ValueError(f"{what} has {t.numel()} elements, needs {min_numel}")


def _check_rho(p, n: int) -> None:
    """p.rho is read for every matrix of the call: a tensor must have an entry per matrix."""
    rn = getattr(p, "_rho_n", None)
    if rn is not None and rn < n:
        raise ValueError(f"rho has {rn} entries for {n} matrices")


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return NSHB_BF16
    if t.dtype == torch.float32:
        return NSHB_F32
    raise TypeError(f"unsupported weight dtype {t.dtype}")


def matrices(W, G, M, O_out=None, z_index=None):
    """ctypes array of nshb_matrix for lists of 2-D CUDA tensors (row-major, unit column stride).

    The library receives bare pointers and cannot see a tensor's size, so what the C
    header requires is checked here: G of W's shape, dtype and strides; M float32 of W's
    shape and strides; O_out[i] (when given, None entries allowed) contiguous with W's
    shape and dtype; every tensor on W[0]'s CUDA device."""
    import torch
    n = len(W)
    if len(G) != n or len(M) != n or (O_out is not None and len(O_out) != n) or \
            (z_index is not None and len(z_index) != n):
        raise ValueError("W, G, M (and O_out, z_index when given) must have one entry per matrix")
    arr = (nshb_matrix * max(n, 1))()
    dev = W[0].device if n else None
    for i in range(n):
        w, g, m = W[i], G[i], M[i]
        if w.dim() != 2 or g.shape != w.shape or m.shape != w.shape:
            raise ValueError(f"matrix {i}: W, G and M must be 2-D of one shape")
        if w.stride(1) != 1 or g.stride() != w.stride() or m.stride() != w.stride():
            raise ValueError(f"matrix {i}: W, G and M must have equal strides and unit column stride")
        if g.dtype != w.dtype or m.dtype != torch.float32:
            raise TypeError(f"matrix {i}: G must have W's dtype and M must be float32")
        o = O_out[i] if O_out is not None else None
        if o is not None and (o.shape != w.shape or o.dtype != w.dtype or not o.is_contiguous()):
            raise ValueError(f"matrix {i}: O_out must be a contiguous tensor of W's shape and dtype")
        if any(t.device != dev for t in (w, g, m) + ((o,) if o is not None else ())) or dev.type != "cuda":
            raise ValueError(f"matrix {i}: every tensor must be on one CUDA device")
        arr[i].rows, arr[i].cols = w.shape
        arr[i].ld = w.stride(0)
        arr[i].w_dtype = _dtype_code(w)
        arr[i].z_index = -1 if z_index is None else int(z_index[i])
        arr[i].W, arr[i].G, arr[i].M = _ptr(w), _ptr(g), _ptr(m)
        arr[i].O_out = _ptr(o)
    arr._n = n
    arr._keep = (W, G, M, O_out)
    return arr


def params(**kw) -> nshb_params:
    """nshb_params with the library defaults, overridden by keyword.  `coeffs` may be a
    list of (a, b, c) rows; `rho` a CUDA float32 tensor (or a raw device pointer)."""
    p = nshb_params()
    _check(lib().nshb_default_params(ctypes.byref(p)), "nshb_default_params")
    keep = []
    for k, v in kw.items():
        if k == "coeffs":
            if v is None:
                p.coeffs = None
            else:
                flat = [float(x) for row in v for x in row]
                buf = (ctypes.c_float * len(flat))(*flat)
                keep.append(buf)
                p.coeffs = ctypes.cast(buf, ctypes.POINTER(ctypes.c_float))
        elif k == "rho":
            import torch
            _device_arg(v, "rho", torch.float32)
            keep.append(v)
            p.rho = _ptr(v)
            p._rho_n = None if v is None or isinstance(v, int) else v.numel()
        elif k == "nesterov":
            p.nesterov = 1 if v else 0
        else:
            if not hasattr(p, k):
                raise KeyError(k)
            setattr(p, k, v)
    p._keep = keep
    return p


def _n(mats) -> int:
    return getattr(mats, "_n", len(mats))


def workspace_size(mats, p, op: int, z_rows=None, n_tokens: int = 0) -> int:
    out = ctypes.c_size_t(0)
    zr, nz = None, 0
    if z_rows is not None:
        nz = len(z_rows)
        zr = (ctypes.c_int64 * max(nz, 1))(*[int(x) for x in z_rows])
    _check(lib().nshb_workspace_size(mats, _n(mats), ctypes.byref(p), op, zr, nz, int(n_tokens),
                                     ctypes.byref(out)), "nshb_workspace_size")
    return out.value


def workspace(mats, p, op: int, device=None, z_rows=None, n_tokens: int = 0):
    """A device workspace (torch uint8 tensor, 256-byte aligned by the caching allocator)."""
    import torch
    nbytes = workspace_size(mats, p, op, z_rows, n_tokens)
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device or "cuda")


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ws(ws):
    if isinstance(ws, tuple):
        return ws
    _device_arg(ws, "workspace")
    return ws.data_ptr(), ws.numel() * ws.element_size()


def _step(name, mats, p, ws, stream):
    _check_rho(p, _n(mats))
    ptr, nbytes = _ws(ws)
    fn = getattr(lib(), name)
    _check(fn(mats, _n(mats), ctypes.byref(p), ptr, nbytes, _stream(stream)), name)


def muon_step(mats, p, ws, stream=None):
    _step("muon_step", mats, p, ws, stream)


def hyperball_step(mats, p, ws, stream=None):
    _step("hyperball_step", mats, p, ws, stream)


def radial_brake_step(mats, p, ws, stream=None):
    _step("radial_brake_step", mats, p, ws, stream)


def himuon_step(mats, p, ws, stream=None):
    _step("himuon_step", mats, p, ws, stream)


def workspace_size_min(mats, p, op: int) -> int:
    """Smallest workspace step_chunked accepts for these matrices (the largest single matrix's need)."""
    out = ctypes.c_size_t(0)
    _check(lib().nshb_workspace_size_min(mats, _n(mats), ctypes.byref(p), op, ctypes.byref(out)),
           "nshb_workspace_size_min")
    return out.value


def step_chunked(op: int, mats, p, ws, stream=None) -> int:
    """The step of kind `op` over the matrices in chunks that fit the workspace; returns the chunk count."""
    _check_rho(p, _n(mats))
    ptr, nbytes = _ws(ws)
    n = ctypes.c_int32(0)
    _check(lib().nshb_step_chunked(op, mats, _n(mats), ctypes.byref(p), ptr, nbytes, _stream(stream),
                                   ctypes.byref(n)), "nshb_step_chunked")
    return n.value


def relative_update_step(mats, p, ws, stream=None):
    _step("relative_update_step", mats, p, ws, stream)


def adam_params(**kw) -> "_abi.nshb_adam_params":
    """nshb_adam_params with the library defaults (0.9, 0.999, 1e-8, step 1), overridden by keyword."""
    a = _abi.nshb_adam_params()
    _check(lib().nshb_default_adam_params(ctypes.byref(a)), "nshb_default_adam_params")
    for k, v in kw.items():
        if not hasattr(a, k):
            raise KeyError(k)
        setattr(a, k, v)
    return a


def adamh_step(mats, V, a, p, ws, stream=None):
    """AdamH step; mats[i].M is the first moment, V[i] (CUDA fp32 tensor or pointer) the second,
    with W's shape and strides."""
    import torch
    n = _n(mats)
    if len(V) != n:
        raise ValueError("V needs one entry per matrix")
    W = getattr(mats, "_keep", (None,))[0]
    for i, v in enumerate(V):
        if v is None or isinstance(v, int):
            continue
        if v.device.type != "cuda" or v.dtype != torch.float32:
            raise TypeError(f"V[{i}] must be a CUDA float32 tensor")
        if W is not None and (v.shape != W[i].shape or v.stride() != W[i].stride()):
            raise ValueError(f"V[{i}] must have W's shape and strides")
    _check_rho(p, n)
    ptr, nbytes = _ws(ws)
    vp = (ctypes.c_void_p * max(n, 1))(*[_ptr(v) for v in V])
    _check(lib().adamh_step(mats, n, vp, ctypes.byref(a), ctypes.byref(p), ptr, nbytes, _stream(stream)),
           "adamh_step")


def newton_muon_step(mats, Z, n_tokens: int, p, ws, stream=None):
    """Newton-Muon step; Z[j] a contiguous bf16 CUDA tensor of z_rows x n_tokens."""
    import torch
    for j, z in enumerate(Z):
        _device_arg(z, f"Z[{j}]", torch.bfloat16)
        if z.dim() != 2 or z.shape[1] != n_tokens:
            raise ValueError(f"Z[{j}] must be 2-D with n_tokens = {n_tokens} columns")
    _check_rho(p, _n(mats))
    ptr, nbytes = _ws(ws)
    nz = len(Z)
    zp = (ctypes.c_void_p * max(nz, 1))(*[_ptr(z) for z in Z])
    zr = (ctypes.c_int64 * max(nz, 1))(*[int(z.shape[0]) for z in Z])
    _check(lib().newton_muon_step(mats, _n(mats), zp, zr, nz, int(n_tokens), ctypes.byref(p), ptr, nbytes,
                                  _stream(stream)), "newton_muon_step")


def fro_norms(mats, out, ws, stream=None):
    import torch
    _device_arg(out, "out", torch.float32, _n(mats))
    ptr, nbytes = _ws(ws)
    _check(lib().nshb_fro_norms(mats, _n(mats), _ptr(out), ptr, nbytes, _stream(stream)), "nshb_fro_norms")


def fro_norms_static(mats, out, stream=None):
    """||W_i||_F into `out` without a workspace (scratch is a fixed array in the library)."""
    import torch
    _device_arg(out, "out", torch.float32, _n(mats))
    _check(lib().nshb_fro_norms_static(mats, _n(mats), _ptr(out), _stream(stream)), "nshb_fro_norms_static")


def device_status(ws, stream=None) -> int:
    ptr, _ = _ws(ws)
    v = ctypes.c_uint32(0)
    _check(lib().nshb_device_status(ptr, _stream(stream), ctypes.byref(v)), "nshb_device_status")
    return v.value


def profile_enable(on: bool = True) -> None:
    _check(lib().nshb_profile_enable(1 if on else 0), "nshb_profile_enable")


def profile_read() -> dict:
    """{kind: (ms, launches)} summed since the last read (waits for the recorded events)."""
    n = _abi.NSHB_PROF_KINDS
    ms = (ctypes.c_float * n)()
    cnt = (ctypes.c_int32 * n)()
    _check(lib().nshb_profile_read(n, ms, cnt), "nshb_profile_read")
    return {_abi.NSHB_PROF_NAMES[k]: (ms[k], cnt[k]) for k in range(n) if cnt[k]}
