"""CPU oracle for the MatMulNBits operator -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The product
path (``int4_block_quantized_matmulnbits_b200``) never imports, links or runs
it, and this package imports nothing from the product.

The arithmetic lives in ``mnb_oracle.c`` (plain C, compiled without FMA
contraction); this module is ctypes marshalling over numpy arrays only.  See
the header of ``mnb_oracle.c`` for the definitions, the page sections they
follow and the readings taken where the pages are silent.

Parity status of each function (what pins it, in ``tests/test_oracle.py``):
  packed_sizes   pinned: byte counts printed on the pages (tests/golden).
  quantize_rtn   pinned: round-trip bound, constructed exact blocks, ties,
                 idempotence on exactly representable blocks.
                 The no-zero-point variant (reading R8) is PARITY UNPINNED
                 by the pages: only its error bound is checked.
  dequantize     pinned: exhaustive (q, zp) sweep, zp default of 8.
  matmul         pinned: exact rational brute force, zero-contribution blocks,
                 block-64 == paired block-32.
  embed_gather   pinned: exact power-of-two scales, bad-id rows, table sizes.
  swiglu         pinned: closed forms (silu(0) = 0, silu(1) = 1/(1 + 1/e),
                 silu(x) - silu(-x) = x, the large-|x| limits).
  gptq_hessian   pinned: exact rational sums on small integer inputs.
  gptq_prepare   pinned: diagonal Hessians in closed form; U^T U H = I.
  gptq_quantize  pinned: a diagonal Hessian reduces it to RTN exactly; an
                 independent formulation (explicit inverse-Hessian downdates,
                 float64) gives the same codes; lower proxy loss than RTN on
                 correlated inputs; dead input features give zero weights.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            from . import build as _build

            _build.build()
        lib = ctypes.CDLL(_LIB_PATH)
        i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.orc_packed_sizes.argtypes = [i64, i64, i64, i64, i32, vp, vp, vp]
        lib.orc_quantize_rtn.argtypes = [vp, i64, i64, i64, i32, i32, vp, vp, vp]
        lib.orc_dequantize.argtypes = [vp, vp, i32, vp, i64, i64, i64, i32, vp]
        lib.orc_matmul.argtypes = [vp, i64, i64, vp, vp, i32, vp, i64, i64, vp, i64, vp]
        lib.orc_embed_gather.argtypes = [vp, vp, i64, i64, vp, i64, i32, vp]
        lib.orc_gptq_quantize.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, vp, vp, vp]
        for f in ("orc_packed_sizes", "orc_quantize_rtn", "orc_dequantize", "orc_matmul",
                  "orc_embed_gather", "orc_num_threads", "orc_gptq_quantize"):
            getattr(lib, f).restype = i32
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def num_threads() -> int:
    return _load().orc_num_threads()


def packed_sizes(N, K, bs, scale_dtype=np.float32, has_zp=True):
    """(packed, scales, zp) byte counts of one [N, K] weight."""
    p, s, z = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    rc = _load().orc_packed_sizes(N, K, bs, np.dtype(scale_dtype).itemsize, int(has_zp),
                                  ctypes.byref(p), ctypes.byref(s), ctypes.byref(z))
    if rc != 0:
        raise ValueError("bad shape")
    return p.value, s.value, z.value


def quantize_rtn(W, bs, has_zp=True, scale_dtype=np.float32):
    """Block-wise RTN of fp32 W [N, K] -> (packed u8 [N, K/2], scales [N, nb], zp u8 or None)."""
    W = _c(W, np.float32)
    N, K = W.shape
    if K % bs or bs % 2:
        raise ValueError("K must be a multiple of an even block size")
    nb = K // bs
    packed = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, nb), scale_dtype)
    zp = np.zeros((N, (nb + 1) // 2), np.uint8) if has_zp else None
    rc = _load().orc_quantize_rtn(_ptr(W), N, K, bs, int(has_zp),
                                  int(np.dtype(scale_dtype) == np.float16),
                                  _ptr(packed), _ptr(scales), _ptr(zp))
    if rc != 0:
        raise ValueError("bad shape")
    return packed, scales, zp


def dequantize(packed, scales, zp, K, bs, out_dtype=np.float64):
    """dequant(W) [N, K]; out_dtype float64 (exact), float32 or float16 (one rounding)."""
    packed = _c(packed, np.uint8)
    scales = np.ascontiguousarray(scales)
    N = packed.shape[0]
    kind = {np.dtype(np.float64): 0, np.dtype(np.float32): 1, np.dtype(np.float16): 2}[np.dtype(out_dtype)]
    out = np.zeros((N, K), out_dtype)
    zp = None if zp is None else _c(zp, np.uint8)
    rc = _load().orc_dequantize(_ptr(packed), _ptr(scales), int(scales.dtype == np.float16),
                                _ptr(zp), N, K, bs, kind, _ptr(out))
    if rc != 0:
        raise ValueError("bad shape")
    return out


def matmul(X, packed, scales, zp, K, bs, cols=None):
    """Y = X . dequant(W)^T in double.  X is converted to float64 exactly.
    cols: optional output columns to compute (then Y is [M, len(cols)])."""
    X = np.ascontiguousarray(np.asarray(X).astype(np.float64))
    M = X.shape[0]
    if X.shape[1] != K:
        raise ValueError("X has the wrong K")
    packed = _c(packed, np.uint8)
    scales = np.ascontiguousarray(scales)
    N = packed.shape[0]
    zp = None if zp is None else _c(zp, np.uint8)
    if cols is not None:
        cols = _c(np.asarray(cols, dtype=np.int64), np.int64)
        ncols = cols.shape[0]
    else:
        ncols = N
    Y = np.zeros((M, ncols), np.float64)
    rc = _load().orc_matmul(_ptr(X), M, K, _ptr(packed), _ptr(scales),
                            int(scales.dtype == np.float16), _ptr(zp), N, bs,
                            _ptr(cols), ncols, _ptr(Y))
    if rc != 0:
        raise ValueError("bad shape or column index")
    return Y


def swiglu(gate, up):
    """silu(gate) * up in float64 (the SwiGLU activation of a Qwen3 MLP:
    "Qwen3-ASR-1.7B ONNX", "Architecture"), silu(x) = x / (1 + exp(-x))."""
    g = np.asarray(gate, np.float64)
    u = np.asarray(up, np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * u


def embed_gather(table, row_scales, ids, out_dtype=np.float16):
    """out[t] = row_scales[id] * table[id] (fp32 product, then fp16 if asked); returns (out, status)."""
    table = _c(table, np.int8)
    row_scales = _c(row_scales, np.float32)
    ids = _c(ids, np.int32)
    V, D = table.shape
    T = ids.shape[0]
    out = np.zeros((T, D), out_dtype)
    st = _load().orc_embed_gather(_ptr(table), _ptr(row_scales), V, D, _ptr(ids), T,
                                  int(np.dtype(out_dtype) == np.float16), _ptr(out))
    return out, st


# ---- GPTQ ("Mega-ASR -- INT4 ONNX (GPTQ-calibrated)", "Conversion details" and
# "GPTQ calibration"; the published GPTQ algorithm, see mnb_oracle.c) --------

def gptq_hessian(X):
    """H = X^T X over calibration rows X [T, K] (float64, exact products of the
    given values): the raw sum.  The usual 2/T factor changes no result of the
    method (U scales by a constant that the error feedback cancels) and is
    left out."""
    X = np.asarray(X, np.float64)
    return X.T @ X


def gptq_prepare(H, percdamp=0.01):
    """(U, dead): dead input features (zero diagonal) get diagonal 1 and are
    flagged; the diagonal is damped by percdamp times its mean; U is the upper
    Cholesky factor of the inverse, H^-1 = U^T U.  float64."""
    H = np.array(H, np.float64, copy=True)
    K = H.shape[0]
    d = np.diag(H).copy()
    dead = d == 0
    d[dead] = 1.0
    H[np.arange(K), np.arange(K)] = d
    damp = percdamp * np.mean(d)
    H[np.arange(K), np.arange(K)] += damp
    Hinv = np.linalg.inv(H)
    U = np.ascontiguousarray(np.linalg.cholesky(Hinv).T)   # lower L with Hinv = L L^T; U = L^T, row-major
    return U, dead.astype(np.uint8)


def gptq_quantize(W, U, bs, has_zp=True, scale_dtype=np.float32, dead=None):
    """GPTQ of fp32 W [N, K] with the fp32 factor U [K, K] (row-major upper):
    (packed, scales, zp) in the layout of quantize_rtn."""
    W = _c(W, np.float32)
    U = _c(U, np.float32)
    N, K = W.shape
    if U.shape != (K, K) or K % bs or bs % 2:
        raise ValueError("bad shape")
    nb = K // bs
    packed = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, nb), scale_dtype)
    zp = np.zeros((N, (nb + 1) // 2), np.uint8) if has_zp else None
    dead = None if dead is None else _c(np.asarray(dead, np.uint8), np.uint8)
    rc = _load().orc_gptq_quantize(_ptr(W), _ptr(U), _ptr(dead), N, K, bs, int(has_zp),
                                   int(np.dtype(scale_dtype) == np.float16), _ptr(packed), _ptr(scales), _ptr(zp))
    if rc != 0:
        raise ValueError("bad shape")
    return packed, scales, zp

