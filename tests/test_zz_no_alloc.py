"""mnb_gemv_argmax_noalloc: greedy decoding with the scratch held by the library.

Some callers cannot give this library device memory (a plug-in whose host
owns every device allocation, a decode thread that must not call the
allocator between tokens).  For them the library keeps the scratch of
mnb_gemv_argmax in a device array of its own.  Checked here against
mnb_gemv_argmax with a caller workspace, on the same inputs, two calls in a
row (the second call finds the first call's leftovers in the shared array):
the outputs must be identical, and right against the oracle.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import assert_close, np_of, random_packed, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mnb(cuda_dev):
    import int4_block_quantized_matmulnbits_b200 as m

    return m


@pytest.mark.parametrize("M,N,K,bs,has_zp", [(1, 151936, 2048, 32, True), (16, 3000, 1024, 64, True),
                                             (5, 777, 512, 32, False)])
def test_noalloc_matches_workspace_entry_point(mnb, cuda_dev, M, N, K, bs, has_zp):
    rng = np.random.default_rng(N * 3 + M)
    packed, scales, zp = random_packed(rng, N, K, bs, has_zp, np.float16)
    dp, ds, dz = to_dev(packed, cuda_dev), to_dev(scales, cuda_dev), to_dev(zp, cuda_dev)
    ws = torch.zeros(mnb.mnb_gemv_argmax_workspace_bytes(M), dtype=torch.uint8, device=cuda_dev)
    for call in range(2):
        X = torch.randn((M, K), generator=torch.Generator().manual_seed(100 * call + M)).half().to(cuda_dev)
        outs = []
        for noalloc in (False, True):
            Y = torch.empty((M, N), dtype=torch.float16, device=cuda_dev)
            ids = torch.full((M,), -1, dtype=torch.int32, device=cuda_dev)
            mx = torch.empty((M,), dtype=torch.float32, device=cuda_dev)
            if noalloc:
                mnb.mnb_gemv_argmax_noalloc(X, dp, ds, dz, Y, M, N, K, bs, ids, mx)
            else:
                mnb.mnb_gemv_argmax(X, dp, ds, dz, Y, M, N, K, bs, ids, mx, ws)
            torch.cuda.synchronize()
            outs.append((Y, ids, mx))
        (y0, i0, m0), (y1, i1, m1) = outs
        # the same kernel on the same inputs: identical logits, tokens and maxima
        assert torch.equal(y1, y0)
        assert torch.equal(i1, i0)
        assert torch.equal(m1, m0)
        # and both right: the logits within tolerance of the oracle, the token
        # the first maximum of the logits, and a greedy choice for the oracle's
        yn, idn = np_of(y1.float()), np_of(i1)
        ref = oracle.matmul(np_of(X.float()), packed, scales, zp, K, bs)
        assert_close(yn, ref, "f16")
        assert np.array_equal(idn, np.argmax(yn, axis=1))
        assert np.array_equal(np_of(m1), yn[np.arange(M), idn])
        assert np.all(ref[np.arange(M), idn] >= ref.max(axis=1) - 2e-2)


def test_noalloc_rejects_requests_outside_its_limits(mnb, cuda_dev):
    X = torch.zeros((17, 256), dtype=torch.float16, device=cuda_dev)
    packed = torch.zeros((64, 128), dtype=torch.uint8, device=cuda_dev)
    scales = torch.ones((64, 8), dtype=torch.float16, device=cuda_dev)
    Y = torch.empty((17, 64), dtype=torch.float16, device=cuda_dev)
    ids = torch.empty((17,), dtype=torch.int32, device=cuda_dev)
    with pytest.raises(mnb.MnbError, match="outside"):
        mnb.mnb_gemv_argmax_noalloc(X, packed, scales, None, Y, 17, 64, 256, 32, ids, None)
