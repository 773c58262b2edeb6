"""MatMulNBits (weight-only int4, block-quantized) for NVIDIA B200 -- Python binding.

A thin ctypes layer over ``libmnb.so`` (the sm_100a kernels and their C ABI,
declared in ``include/mnb.h``).  Every function here has the name of the C
entry point it calls and only marshals arguments: torch tensors become device
pointers, dtypes become ``mnb_dtype`` values, the stream defaults to torch's
current stream.  All arithmetic runs in the CUDA kernels; there is no CPU path.
If the library cannot be loaded, importing this package raises.

Layout (see ``include/mnb.h``): packed uint8 [N, K/2] (element 2j in the low
nibble of byte j), scales fp32/fp16 [N, K/bs], zero points uint8
[N, ceil(K/bs/2)] (block b in byte b/2, low nibble for even b) or None (zp=8).
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MnbError", "MNB_F32", "MNB_F16", "MNB_FLAG_PDL", "lib_path",
    "mnb_last_error", "mnb_version", "mnb_packed_sizes", "mnb_quantize_rtn", "mnb_dequantize",
    "mnb_gemv", "mnb_gemm", "mnb_embed_gather", "mnb_device_status",
    "mnb_gemv_argmax", "mnb_gemv_argmax_workspace_bytes", "mnb_gemv_argmax_noalloc", "mnb_gemv_swiglu",
    "mnb_gemv_task", "mnb_gemv_chain_plan_bytes", "mnb_gemv_chain_workspace_bytes", "mnb_gemv_chain_plan",
    "mnb_gemv_chain", "mnb_matmul", "mnb_gptq_hessian", "mnb_gptq_workspace_bytes", "mnb_gptq_prepare",
    "mnb_gptq_quantize",
]

MNB_F32, MNB_F16 = 0, 1
MNB_FLAG_PDL = 1
_ERRORS = {-1: "MNB_ERR_INVALID_ARG", -2: "MNB_ERR_SHAPE", -3: "MNB_ERR_ALIGN",
           -4: "MNB_ERR_UNSUPPORTED", -5: "MNB_ERR_CUDA", -6: "MNB_ERR_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libmnb.so")


class MnbError(RuntimeError):
    def __init__(self, fn, code, msg):
        super().__init__(f"{fn} -> {_ERRORS.get(code, code)}: {msg}")
        self.code = code


class mnb_gemv_task(ctypes.Structure):
    """One GEMV of mnb_gemv_chain (the C struct of the same name)."""
    _fields_ = [("X", ctypes.c_void_p), ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("zp", ctypes.c_void_p), ("Y", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("wait", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def _load():
    # (Re)build in-tree when libmnb.so is missing or older than its sources;
    # a no-op otherwise.  Raises if nvcc fails: there is no fallback path.
    from . import build as _build

    _build.build()
    lib = ctypes.CDLL(lib_path)
    i64, i32, u32, vp, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_uint, ctypes.c_void_p, ctypes.c_size_t
    P = ctypes.POINTER
    sig = {
        "mnb_last_error": ([], ctypes.c_char_p),
        "mnb_version": ([], ctypes.c_char_p),
        "mnb_packed_sizes": ([i64, i64, i32, i32, i32, P(sz), P(sz), P(sz)], i32),
        "mnb_quantize_rtn": ([vp, i64, i64, i32, i32, vp, vp, i32, vp, vp], i32),
        "mnb_dequantize": ([vp, vp, i32, vp, i64, i64, i32, vp, i32, vp], i32),
        "mnb_gemv": ([vp, i32, vp, vp, i32, vp, vp, i64, i64, i64, i32, u32, vp], i32),
        "mnb_gemm": ([vp, i32, vp, vp, i32, vp, vp, i64, i64, i64, i32, u32, vp], i32),
        "mnb_matmul": ([vp, i32, vp, vp, i32, vp, vp, i64, i64, i64, i32, u32, vp], i32),
        "mnb_embed_gather": ([vp, vp, i64, i64, vp, i64, vp, i32, vp, vp], i32),
        "mnb_device_status": ([P(u32), i32], i32),
        "mnb_gemv_argmax_workspace_bytes": ([i64], sz),
        "mnb_gemv_swiglu": ([vp, vp, vp, i32, vp, vp, i64, i64, i64, i32, u32, vp], i32),
        "mnb_gemv_argmax": ([vp, vp, vp, i32, vp, vp, i64, i64, i64, i32, vp, vp, vp, sz, u32, vp], i32),
        "mnb_gemv_argmax_noalloc": ([vp, vp, vp, i32, vp, vp, i64, i64, i64, i32, vp, vp, u32, vp], i32),
        "mnb_gemv_chain_plan_bytes": ([i32], sz),
        "mnb_gemv_chain_workspace_bytes": ([i32], sz),
        "mnb_gemv_chain_plan": ([P(mnb_gemv_task), i32, i64, i32, vp, sz], i32),
        "mnb_gemv_chain": ([vp, vp, vp, sz, u32, vp], i32),
        "mnb_gptq_hessian": ([vp, i32, i64, i64, vp, i32, vp], i32),
        "mnb_gptq_workspace_bytes": ([i64], sz),
        "mnb_gptq_prepare": ([vp, i64, ctypes.c_float, vp, vp, vp, sz, P(ctypes.c_float), vp], i32),
        "mnb_gptq_quantize": ([vp, vp, vp, i64, i64, i32, i32, vp, vp, i32, vp, vp], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes, f.restype = args, res
    return lib


_lib = _load()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dt(t):
    if t.dtype == torch.float32:
        return MNB_F32
    if t.dtype == torch.float16:
        return MNB_F16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(fn, rc):
    if rc != 0:
        raise MnbError(fn, rc, _lib.mnb_last_error().decode())


def mnb_last_error() -> str:
    return _lib.mnb_last_error().decode()


def mnb_version() -> str:
    return _lib.mnb_version().decode()


def mnb_packed_sizes(N, K, bs, scale_dtype=torch.float16, has_zp=True):
    """(packed_bytes, scale_bytes, zp_bytes) of one [N, K] weight."""
    p, s, z = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    st = MNB_F16 if scale_dtype == torch.float16 else MNB_F32
    _check("mnb_packed_sizes", _lib.mnb_packed_sizes(N, K, bs, st, int(bool(has_zp)),
                                                     ctypes.byref(p), ctypes.byref(s), ctypes.byref(z)))
    return p.value, s.value, z.value


def mnb_quantize_rtn(W, N, K, bs, has_zp, packed, scales, zp, stream=None):
    """Block-wise RTN of fp32 W [N, K] into packed / scales / zp (all device tensors)."""
    _check("mnb_quantize_rtn", _lib.mnb_quantize_rtn(
        _ptr(W), N, K, bs, int(bool(has_zp)), _ptr(packed), _ptr(scales), _dt(scales),
        _ptr(zp), _stream(stream)))


def mnb_dequantize(packed, scales, zp, N, K, bs, W_out, stream=None):
    """W_out [N, K] (fp32 or fp16) = (q - zp) * scale, one rounding."""
    _check("mnb_dequantize", _lib.mnb_dequantize(
        _ptr(packed), _ptr(scales), _dt(scales), _ptr(zp), N, K, bs, _ptr(W_out), _dt(W_out),
        _stream(stream)))


def mnb_gemv(X, packed, scales, zp, Y, M, N, K, bs, flags=0, stream=None):
    """Y [M, N] = X [M, K] . dequant(W)^T for 1 <= M <= 16 (decode kernel)."""
    _check("mnb_gemv", _lib.mnb_gemv(
        _ptr(X), _dt(X), _ptr(packed), _ptr(scales), _dt(scales), _ptr(zp), _ptr(Y),
        M, N, K, bs, flags, _stream(stream)))


def mnb_gemv_swiglu(X, packed, scales, zp, Y, M, N, K, bs, flags=0, stream=None):
    """Y [M, N/2] = silu(gate) * up from gate/up rows interleaved in 8-row groups (fp16 X)."""
    _check("mnb_gemv_swiglu", _lib.mnb_gemv_swiglu(
        _ptr(X), _ptr(packed), _ptr(scales), _dt(scales), _ptr(zp), _ptr(Y), M, N, K, bs, flags,
        _stream(stream)))


def mnb_gemv_argmax_workspace_bytes(M) -> int:
    """Bytes of workspace mnb_gemv_argmax needs for M tokens on the current device."""
    return _lib.mnb_gemv_argmax_workspace_bytes(M)


def mnb_gemv_argmax(X, packed, scales, zp, Y, M, N, K, bs, ids, max_out, workspace, flags=0, stream=None):
    """Y as mnb_gemv (fp16 X), plus ids[m] = first argmax of Y[m] and max_out[m] its value.
    workspace: a zero-filled uint8 device tensor of mnb_gemv_argmax_workspace_bytes(M) bytes."""
    _check("mnb_gemv_argmax", _lib.mnb_gemv_argmax(
        _ptr(X), _ptr(packed), _ptr(scales), _dt(scales), _ptr(zp), _ptr(Y), M, N, K, bs, _ptr(ids),
        _ptr(max_out), _ptr(workspace), workspace.numel() * workspace.element_size(), flags, _stream(stream)))


def mnb_gemv_argmax_noalloc(X, packed, scales, zp, Y, M, N, K, bs, ids, max_out, flags=0, stream=None):
    """mnb_gemv_argmax with its scratch in a device array held by the library:
    for callers that cannot provide device memory.  Calls that may overlap on
    the GPU share that array and must be serialized."""
    _check("mnb_gemv_argmax_noalloc", _lib.mnb_gemv_argmax_noalloc(
        _ptr(X), _ptr(packed), _ptr(scales), _dt(scales), _ptr(zp), _ptr(Y), M, N, K, bs, _ptr(ids),
        _ptr(max_out), flags, _stream(stream)))


def mnb_gemv_chain_plan_bytes(ntasks) -> int:
    return _lib.mnb_gemv_chain_plan_bytes(ntasks)


def mnb_gemv_chain_workspace_bytes(ntasks) -> int:
    """Bytes of the (zero-filled) device workspace of a chain of ntasks GEMVs."""
    return _lib.mnb_gemv_chain_workspace_bytes(ntasks)


def mnb_gemv_chain_plan(tasks, M, bs):
    """Plan a chain of decode GEMVs for mnb_gemv_chain (host only).

    tasks: sequence of (X, packed, scales, zp, Y, N, K, wait) with device
    tensors (zp may be None).  Returns the plan as a 64-byte aligned uint8 CPU
    tensor; copy it unchanged to the device (e.g. ``plan.cuda()``) and pass both."""
    n = len(tasks)
    arr = (mnb_gemv_task * n)()
    for i, (X, packed, scales, zp, Y, N, K, wait) in enumerate(tasks):
        arr[i] = mnb_gemv_task(_ptr(X), _ptr(packed), _ptr(scales), _ptr(zp), _ptr(Y), N, K, int(wait), 0)
    nbytes = mnb_gemv_chain_plan_bytes(n)
    if nbytes == 0:
        raise MnbError("mnb_gemv_chain_plan", -1, f"ntasks={n} outside [1, 65536]")
    buf = torch.empty(nbytes + 64, dtype=torch.uint8)
    off = (-buf.data_ptr()) % 64
    plan = buf[off:off + nbytes]
    _check("mnb_gemv_chain_plan", _lib.mnb_gemv_chain_plan(arr, n, M, bs, plan.data_ptr(), nbytes))
    return plan


def mnb_gemv_chain(plan, plan_device, workspace, flags=0, stream=None):
    """Run a planned chain of decode GEMVs as one launch (plan: the host tensor
    from mnb_gemv_chain_plan; plan_device: its device copy; workspace:
    zero-filled uint8 device tensor of mnb_gemv_chain_workspace_bytes bytes)."""
    _check("mnb_gemv_chain", _lib.mnb_gemv_chain(
        _ptr(plan), _ptr(plan_device), _ptr(workspace), workspace.numel() * workspace.element_size(), flags,
        _stream(stream)))


def mnb_gemm(X, packed, scales, zp, Y, M, N, K, bs, flags=0, stream=None):
    """Y [M, N] = X [M, K] . dequant(W)^T on the tensor cores (fp16 X and Y)."""
    _check("mnb_gemm", _lib.mnb_gemm(
        _ptr(X), _dt(X), _ptr(packed), _ptr(scales), _dt(scales), _ptr(zp), _ptr(Y),
        M, N, K, bs, flags, _stream(stream)))


def mnb_matmul(X, packed, scales, zp, Y, M, N, K, bs, flags=0, stream=None):
    """Y [M, N] = X [M, K] . dequant(W)^T for any M, on the kernel that serves M best."""
    _check("mnb_matmul", _lib.mnb_matmul(
        _ptr(X), _dt(X), _ptr(packed), _ptr(scales), _dt(scales), _ptr(zp), _ptr(Y),
        M, N, K, bs, flags, _stream(stream)))


def mnb_embed_gather(table, row_scales, V, D, ids, T, out, status=None, stream=None):
    """out [T, D] = int8 table rows [ids] * row_scales[ids] (fp32 product, fp16 if out is fp16)."""
    _check("mnb_embed_gather", _lib.mnb_embed_gather(
        _ptr(table), _ptr(row_scales), V, D, _ptr(ids), T, _ptr(out), _dt(out), _ptr(status),
        _stream(stream)))


def mnb_device_status(clear=False) -> int:
    """The library's device status word (bit 0: a GEMM or GEMV wait timed out;
    bits 1-3: mnb_gemv_chain); synchronizes.  A timeout (MNB_ERR_TIMEOUT from
    the C call) is reported through the returned word, not raised."""
    v = ctypes.c_uint()
    rc = _lib.mnb_device_status(ctypes.byref(v), int(bool(clear)))
    if rc != -6:
        _check("mnb_device_status", rc)
    return v.value


def _contiguous(fn, *ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise MnbError(fn, -1, "tensors must be contiguous (row-major)")


def mnb_gptq_hessian(X, H, accumulate=False, stream=None):
    """H [K, K] fp32 (+)= X^T X for calibration inputs X [T, K] (fp32 or fp16)."""
    _contiguous("mnb_gptq_hessian", X, H)
    T, K = X.shape
    _check("mnb_gptq_hessian", _lib.mnb_gptq_hessian(_ptr(X), _dt(X), T, K, _ptr(H), int(bool(accumulate)),
                                                     _stream(stream)))


def mnb_gptq_workspace_bytes(K) -> int:
    return _lib.mnb_gptq_workspace_bytes(K)


def mnb_gptq_prepare(H, U, dead, workspace, percdamp=0.01, stream=None) -> float:
    """U [K, K] fp32 = upper Cholesky factor of the damped H^-1; dead [K] uint8.
    Synchronizes the stream; returns the damping that succeeded."""
    _contiguous("mnb_gptq_prepare", H, U, dead)
    K = H.shape[0]
    d = ctypes.c_float()
    _check("mnb_gptq_prepare", _lib.mnb_gptq_prepare(
        _ptr(H), K, percdamp, _ptr(U), _ptr(dead), _ptr(workspace), workspace.numel() * workspace.element_size(),
        ctypes.byref(d), _stream(stream)))
    return d.value


def mnb_gptq_quantize(W, U, dead, bs, has_zp, packed, scales, zp, stream=None):
    """GPTQ of fp32 W [N, K] into packed / scales / zp (the layout of mnb_quantize_rtn)."""
    _contiguous("mnb_gptq_quantize", W, U, dead, packed, scales, zp)
    N, K = W.shape
    _check("mnb_gptq_quantize", _lib.mnb_gptq_quantize(
        _ptr(W), _ptr(U), _ptr(dead), N, K, bs, int(bool(has_zp)), _ptr(packed), _ptr(scales), _dt(scales),
        _ptr(zp), _stream(stream)))

