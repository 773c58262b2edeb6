"""Host-side checks of the C ABI: the library loads without a GPU, exports every
entry point include/mnb.h declares, and rejects bad arguments with the
documented codes before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mnb.h")
TUNE_HEADER = os.path.join(ROOT, "include", "mnb_tune.h")

OK, INVALID, SHAPE, ALIGN, UNSUPPORTED = 0, -1, -2, -3, -4
F32, F16 = 0, 1
A = 1 << 20          # a 16-byte aligned fake device address (never dereferenced)


@pytest.fixture(scope="module")
def mnb():
    import int4_block_quantized_matmulnbits_b200 as m

    return m


@pytest.fixture(scope="module")
def lib(mnb):
    return mnb._lib


def declared_functions(path=HEADER):
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mnb_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for f in ["mnb_packed_sizes", "mnb_quantize_rtn", "mnb_dequantize", "mnb_gemv", "mnb_gemm",
              "mnb_embed_gather", "mnb_last_error", "mnb_device_status"]:
        assert f in names


def test_library_exports_every_declared_symbol(mnb):
    raw = ctypes.CDLL(mnb.lib_path)
    for name in declared_functions():
        assert hasattr(raw, name), name


def exported_functions(path):
    """Names of the mnb_* functions the shared library exports (nm -D)."""
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    return sorted({ln.split()[-1] for ln in out.splitlines() if ln.split() and ln.split()[-1].startswith("mnb_")})


def test_every_exported_symbol_is_declared(mnb):
    # the stable entry points in mnb.h, the tuning hooks in mnb_tune.h; nothing else
    declared = set(declared_functions()) | set(declared_functions(TUNE_HEADER))
    exported = exported_functions(mnb.lib_path)
    assert exported, "nm found no mnb_* symbols"
    assert sorted(set(exported) - declared) == []
    for name in declared_functions(TUNE_HEADER):
        assert name in exported, name


def test_version_and_empty_error(mnb):
    assert "sm_100a" in mnb.mnb_version()


@pytest.mark.parametrize("N,K,bs,sdt,zp", [(2048, 1024, 32, F32, 1), (151936, 1024, 64, F16, 1),
                                           (3, 96, 32, F16, 1), (5, 64, 64, F16, 0)])
def test_packed_sizes_agree_with_oracle(lib, N, K, bs, sdt, zp):
    p, s, z = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.mnb_packed_sizes(N, K, bs, sdt, zp, ctypes.byref(p), ctypes.byref(s), ctypes.byref(z)) == OK
    assert (p.value, s.value, z.value) == oracle.packed_sizes(N, K, bs, np.float16 if sdt else np.float32, bool(zp))


def test_packed_sizes_rejects(lib):
    p, s, z = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    args = (ctypes.byref(p), ctypes.byref(s), ctypes.byref(z))
    assert lib.mnb_packed_sizes(4, 96, 48, F16, 1, *args) == SHAPE
    assert lib.mnb_packed_sizes(4, 100, 32, F16, 1, *args) == SHAPE
    assert lib.mnb_packed_sizes(-1, 64, 32, F16, 1, *args) == INVALID
    assert lib.mnb_packed_sizes(4, 64, 32, 7, 1, *args) == INVALID
    assert lib.mnb_packed_sizes(4, 64, 32, F16, 1, None, None, None) == INVALID
    assert "NULL" in lib.mnb_last_error().decode()


def test_gemv_argument_checks(lib):
    g = lib.mnb_gemv
    assert g(A, F16, A, A, F16, A, A, 33, 64, 64, 32, 0, None) == UNSUPPORTED    # fp16: M <= 32
    assert g(A, F32, A, A, F32, A, A, 17, 64, 64, 32, 0, None) == UNSUPPORTED    # fp32: M <= 16
    assert g(A, F16, A, A, F16, A, A, 1, 64, 96, 64, 0, None) == SHAPE          # K % bs
    assert g(A, F16, A, A, F16, A, A, 1, 64, 64, 16, 0, None) == SHAPE          # bs
    assert g(None, F16, A, A, F16, A, A, 1, 64, 64, 32, 0, None) == INVALID
    assert g(A + 8, F16, A, A, F16, A, A, 1, 64, 64, 32, 0, None) == ALIGN
    assert g(A, F16, A, A + 1, F16, A, A, 1, 64, 64, 32, 0, None) == ALIGN     # fp16 scales, odd address
    assert g(A, F16, A, A, F16, A, A, -1, 64, 64, 32, 0, None) == INVALID
    assert g(A, 5, A, A, F16, A, A, 1, 64, 64, 32, 0, None) == INVALID
    assert g(A, F16, A, A, F16, A, A, 1, 64, 64, 32, 0x80, None) == INVALID   # unknown flag
    assert g(A, F16, A, A, F16, A, A, 0, 64, 64, 32, 0, None) == OK            # M = 0: nothing to do
    assert g(A, F16, A, A, F16, A, A, 1, 0, 64, 32, 0, None) == OK             # N = 0


def test_gemm_argument_checks(lib):
    g = lib.mnb_gemm
    assert g(A, F32, A, A, F16, A, A, 64, 128, 64, 32, 0, None) == UNSUPPORTED   # fp32 activations
    assert g(A, F16, A, A, F32, A, A, 64, 128, 64, 32, 0, None) == UNSUPPORTED   # fp32 scales (q4 + fp16 X)
    assert g(A, F16, A, A, F16, A, A, 64, 100, 64, 32, 0, None) == SHAPE          # N % 128
    assert g(A, F16, A, A, F16, A, A, 64, 128, 96, 32, 0, None) == SHAPE          # K % 64
    assert g(A, F16, A + 4, A, F16, A, A, 64, 128, 64, 32, 0, None) == ALIGN
    assert g(A, F16, A, A, F16, A, A, 0, 128, 64, 32, 0, None) == OK


def test_quantize_dequantize_embed_argument_checks(lib):
    assert lib.mnb_quantize_rtn(A, 4, 96, 64, 1, A, A, F16, A, None) == SHAPE
    assert lib.mnb_quantize_rtn(A, 4, 64, 32, 1, A, A, F16, None, None) == INVALID   # zp needed
    assert lib.mnb_quantize_rtn(A + 4, 4, 64, 32, 1, A, A, F16, A, None) == ALIGN
    assert lib.mnb_quantize_rtn(A, 0, 64, 32, 1, A, A, F16, A, None) == OK
    assert lib.mnb_dequantize(A, A, F16, None, 4, 64, 32, A + 2, F16, None) == ALIGN
    assert lib.mnb_dequantize(A, A, 3, None, 4, 64, 32, A, F16, None) == INVALID
    assert lib.mnb_embed_gather(A, A, 10, 24, A, 4, A, F16, None, None) == SHAPE    # D % 16
    assert lib.mnb_embed_gather(A, A, 10, 32, None, 4, A, F16, None, None) == INVALID
    assert lib.mnb_embed_gather(A, A, 10, 32, A, 4, A + 8, F16, None, None) == ALIGN
    assert lib.mnb_embed_gather(A, A, 10, 32, A, 0, A, F16, None, None) == OK
    assert lib.mnb_device_status(None, 0) == INVALID


def test_binding_raises_with_message(mnb):
    with pytest.raises(mnb.MnbError) as e:
        mnb.mnb_packed_sizes(4, 100, 32)
    assert "MNB_ERR_SHAPE" in str(e.value) and "K=100" in str(e.value)


def test_gemv_argmax_argument_checks(lib):
    fake = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced: every call below fails its checks
    ws = lib.mnb_gemv_argmax_workspace_bytes
    ws.restype, ws.argtypes = ctypes.c_size_t, [ctypes.c_int64]
    assert ws(0) == 0 and ws(17) == 0 and ws(1) > 0 and ws(16) > ws(1)
    f = lib.mnb_gemv_argmax
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] + [ctypes.c_void_p] * 2 + [ctypes.c_int64] * 3 + \
        [ctypes.c_int] + [ctypes.c_void_p] * 3 + [ctypes.c_size_t, ctypes.c_uint, ctypes.c_void_p]
    need = ws(1)
    # M outside [1, 16]
    assert f(fake, fake, fake, 1, fake, fake, 17, 256, 512, 32, fake, None, fake, ws(16), 0, None) == -4
    # NULL ids
    assert f(fake, fake, fake, 1, fake, fake, 1, 256, 512, 32, None, None, fake, need, 0, None) == -1
    # workspace too small
    assert f(fake, fake, fake, 1, fake, fake, 1, 256, 512, 32, fake, None, fake, need - 1, 0, None) == -1
    assert b"workspace" in lib.mnb_last_error()
    # misaligned workspace
    assert f(fake, fake, fake, 1, fake, fake, 1, 256, 512, 32, fake, None, ctypes.c_void_p((1 << 20) + 4), need, 0,
             None) == -3


def test_gemv_swiglu_argument_checks(lib):
    f = lib.mnb_gemv_swiglu
    assert f(A, A, A, F16, A, A, 17, 64, 64, 32, 0, None) == UNSUPPORTED      # M > 16
    assert f(A, A, A, F16, A, A, 1, 72, 64, 32, 0, None) == SHAPE            # N % 16
    assert f(A, A, A, F16, A, A, 1, 64, 96, 64, 0, None) == SHAPE            # K % bs
    assert f(A, A, A, F16, A, A, 1, 64, 64, 32, 0x80, None) == INVALID       # unknown flag
    assert f(A, A, A, F16, A, A, 0, 64, 64, 32, 0, None) == OK               # M = 0


def test_gemv_chain_argument_checks(mnb, lib):
    T = mnb.mnb_gemv_task
    assert mnb.mnb_gemv_chain_plan_bytes(0) == 0 and mnb.mnb_gemv_chain_plan_bytes(65537) == 0
    assert mnb.mnb_gemv_chain_plan_bytes(3) == 64 + 3 * 256
    assert mnb.mnb_gemv_chain_workspace_bytes(0) == 0 and mnb.mnb_gemv_chain_workspace_bytes(197) >= 198 * 4

    def task(N=2048, K=2048, X=A, packed=A, scales=A, zp=A, Y=A, wait=1, reserved=0):
        return T(X, packed, scales, zp, Y, N, K, wait, reserved)

    nbytes = mnb.mnb_gemv_chain_plan_bytes(2)
    buf = ctypes.create_string_buffer(nbytes + 128)
    plan = ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 64

    def rc(tasks, M=1, bs=32, size=nbytes, ptr=plan):
        arr = (T * len(tasks))(*tasks)
        return lib.mnb_gemv_chain_plan(arr, len(tasks), M, bs, ptr, size)

    assert rc([task(), task(N=72)]) == SHAPE                  # N % 16
    assert rc([task(), task(K=320)]) == SHAPE                 # K % 256
    assert rc([task(K=768)], bs=64) == SHAPE                  # block 64 with zero points: K % 512
    assert rc([task(), task(X=A + 8)]) == ALIGN               # X not 16-byte aligned
    assert rc([task(scales=A + 8)]) == ALIGN                  # block-32 scales not 16-byte aligned
    assert rc([task(zp=A + 2)]) == ALIGN
    assert rc([task(), task(zp=None)]) == UNSUPPORTED         # zero points in some tasks only
    assert rc([task()], M=9) == UNSUPPORTED
    assert rc([task()], M=0) == INVALID
    assert rc([task()], bs=48) == SHAPE
    assert rc([task(reserved=1)]) == INVALID
    assert rc([task(Y=None)]) == INVALID
    assert rc([task(), task()], size=nbytes - 1) == INVALID   # plan buffer too small
    assert rc([task()], ptr=plan + 16) == ALIGN               # plan buffer not 64-byte aligned
    assert rc([task(K=65536)], M=8) == SHAPE                  # X does not fit in shared memory
    # launch: the plan's header is checked before anything touches the device
    f = lib.mnb_gemv_chain
    ctypes.memset(plan, 0, nbytes)
    ws = mnb.mnb_gemv_chain_workspace_bytes(2)
    assert f(plan, A, A, ws, 0, None) == INVALID              # not a plan
    assert b"not a plan" in lib.mnb_last_error()
    assert f(None, A, A, ws, 0, None) == INVALID
    assert f(plan, A + 32, A, ws, 0, None) == ALIGN           # device plan not 64-byte aligned
    assert f(plan, A, A, ws, 0x80, None) == INVALID           # unknown flag


def test_matmul_argument_checks(lib):
    f = lib.mnb_matmul
    assert f(A, F16, A, A, F16, A, A, 17, 128, 96, 64, 0, None) == SHAPE        # K % bs
    assert f(A, F16, A, A, F16, A, A, 17, 128, 64, 48, 0, None) == SHAPE        # bs
    assert f(A + 8, F16, A, A, F16, A, A, 17, 128, 64, 32, 0, None) == ALIGN    # X not 16-byte aligned
    assert f(A, F16, A, A, F16, A, A, 17, 128, 64, 32, 0x80, None) == INVALID   # unknown flag
    assert f(A, 7, A, A, F16, A, A, 17, 128, 64, 32, 0, None) == INVALID        # dtype
    assert f(A, F16, A, A, F16, A, A, 0, 128, 64, 32, 0, None) == OK            # M = 0: nothing to do


def test_gptq_argument_checks(lib):
    vp = ctypes.c_void_p
    h = lib.mnb_gptq_hessian
    h.argtypes = [vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, vp, ctypes.c_int, vp]
    assert h(A, F32, 10, 0, A, 0, None) == SHAPE                 # K = 0
    assert h(A, F32, 10, 8193, A, 0, None) == SHAPE              # K above the limit
    assert h(None, F32, 10, 64, A, 0, None) == INVALID
    assert h(A, F32, 10, 64, A + 2, 0, None) == ALIGN
    assert h(A, 7, 10, 64, A, 0, None) == INVALID                # dtype
    wsb = lib.mnb_gptq_workspace_bytes
    wsb.argtypes, wsb.restype = [ctypes.c_int64], ctypes.c_size_t
    assert wsb(0) == 0 and wsb(8193) == 0 and wsb(64) >= 2 * 64 * 64 * 4
    p = lib.mnb_gptq_prepare
    p.argtypes = [vp, ctypes.c_int64, ctypes.c_float, vp, vp, vp, ctypes.c_size_t, vp, vp]
    need = wsb(64)
    assert p(A, 64, 0.01, A, A, A, need - 1, None, None) == INVALID   # workspace too small
    assert p(A, 64, -1.0, A, A, A, need, None, None) == INVALID       # percdamp
    assert p(A, 64, 0.01, A, None, A, need, None, None) == INVALID
    assert p(A, 64, 0.01, A, A, A + 4, need, None, None) == ALIGN
    q = lib.mnb_gptq_quantize
    q.argtypes = [vp, vp, vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int, vp, vp, ctypes.c_int,
                  vp, vp]
    assert q(A, A, None, 4, 96, 64, 1, A, A, F16, A, None) == SHAPE    # K % bs
    assert q(A, A, None, 4, 96, 48, 1, A, A, F16, A, None) == SHAPE    # bs
    assert q(A, A, None, 4, 64, 32, 1, A, A, F16, None, None) == INVALID   # zp missing
    assert q(A, A, None, 0, 64, 32, 1, A, A, F16, A, None) == OK       # nothing to do
