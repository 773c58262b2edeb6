"""The debug build (libmnb_debug.so): the same kernels with device-side index
checks that record a status bit and keep the access inside its buffer instead
of trapping.  On correct inputs no check may fire and the results must be the
release build's, bit for bit."""
import ctypes
import os

import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import assert_close, np_of, random_packed, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs(cuda_dev):
    import int4_block_quantized_matmulnbits_b200 as mnb
    from int4_block_quantized_matmulnbits_b200 import build

    path = build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for name in dir(mnb._lib):
        if name.startswith("mnb_"):
            f, g = getattr(dbg, name), getattr(mnb._lib, name)
            f.argtypes, f.restype = g.argtypes, g.restype
    return mnb, dbg


def _status(lib):
    v = ctypes.c_uint()
    rc = lib.mnb_device_status(ctypes.byref(v), 1)
    return rc, v.value


@pytest.mark.parametrize("N,K,bs,has_zp", [(2048, 2048, 32, True), (6144, 2048, 32, True), (2048, 6144, 32, True),
                                           (151936, 2048, 32, True), (777, 512, 64, False), (50, 256, 32, True)])
def test_debug_build_matches_release(libs, cuda_dev, N, K, bs, has_zp):
    mnb, dbg = libs
    rng = np.random.default_rng(N + K)
    packed, scales, zp = random_packed(rng, N, K, bs, has_zp, np.float16)
    dp, ds, dz = to_dev(packed, cuda_dev), to_dev(scales, cuda_dev), to_dev(zp, cuda_dev)
    X = torch.randn((1, K), generator=torch.Generator().manual_seed(K)).half().to(cuda_dev)
    _status(dbg)
    ys = []
    for lib in (mnb._lib, dbg):
        Y = torch.empty((1, N), dtype=torch.float16, device=cuda_dev)
        rc = lib.mnb_gemv(X.data_ptr(), 1, dp.data_ptr(), ds.data_ptr(), 1, None if dz is None else dz.data_ptr(),
                          Y.data_ptr(), 1, N, K, bs, 0, torch.cuda.current_stream().cuda_stream)
        assert rc == 0
        torch.cuda.synchronize()
        ys.append(Y)
    assert _status(dbg) == (0, 0), "an index check fired"
    assert torch.equal(ys[0], ys[1])
    assert_close(np_of(ys[1].float()), oracle.matmul(np_of(X.float()), packed, scales, zp, K, bs), "f16")
