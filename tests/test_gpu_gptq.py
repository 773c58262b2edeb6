"""GPU parity of the GPTQ quantizer ("Mega-ASR -- INT4 ONNX (GPTQ-calibrated)",
"Conversion details": algo=GPTQ; "GPTQ calibration").

The column loop takes the same fp32 factor U on both sides (the oracle's), so
its codes, scales and zero points must be bit-exact.  The Hessian and the
factor are continuous quantities, checked within tolerance against the
oracle's float64.  End to end (the device's own Hessian and factor), the codes
may differ where a rounding decision sits within fp32 noise of a tie, so the
check is the proxy loss GPTQ minimizes and the share of equal codes.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import np_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mnb(cuda_dev):
    import int4_block_quantized_matmulnbits_b200 as m

    return m


def _calib(rng, T, K, corr=0.5):
    """Correlated calibration inputs: X = Z (I + corr G), fp32."""
    G = rng.standard_normal((K, K)) / np.sqrt(K)
    return (rng.standard_normal((T, K)) @ (np.eye(K) + corr * G)).astype(np.float32)


def _dev_prepare(mnb, H, dev, percdamp=0.01):
    K = H.shape[0]
    U = torch.empty((K, K), dtype=torch.float32, device=dev)
    dead = torch.empty((K,), dtype=torch.uint8, device=dev)
    ws = torch.empty((mnb.mnb_gptq_workspace_bytes(K),), dtype=torch.uint8, device=dev)
    used = mnb.mnb_gptq_prepare(H, U, dead, ws, percdamp)
    return U, dead, used


def _dev_quantize(mnb, W, U, dead, bs, has_zp, sdt, dev):
    N, K = W.shape
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, K // bs), dtype=sdt, device=dev)
    zp = torch.empty((N, (K // bs + 1) // 2), dtype=torch.uint8, device=dev) if has_zp else None
    mnb.mnb_gptq_quantize(W, U, dead, bs, has_zp, packed, scales, zp)
    torch.cuda.synchronize()
    return np_of(packed), np_of(scales), (np_of(zp) if has_zp else None)


@pytest.mark.parametrize("T,K,dtype", [(333, 200, torch.float32), (1024, 256, torch.float16), (7, 96, torch.float32)])
def test_gptq_hessian(mnb, cuda_dev, T, K, dtype):
    rng = np.random.default_rng(T + K)
    X = torch.from_numpy(_calib(rng, T, K)).to(dtype)
    H = torch.full((K, K), float("nan"), dtype=torch.float32, device=cuda_dev)
    mnb.mnb_gptq_hessian(X.to(cuda_dev), H)
    mnb.mnb_gptq_hessian(X.to(cuda_dev), H, accumulate=True)   # a second batch: the same rows again
    torch.cuda.synchronize()
    ref = 2.0 * oracle.gptq_hessian(X.float().numpy())
    got = np_of(H).astype(np.float64)
    assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref)
    assert np.array_equal(got, got.T) or np.allclose(got, got.T, rtol=1e-6, atol=0)


@pytest.mark.parametrize("K", [64, 256, 1000])
def test_gptq_prepare(mnb, cuda_dev, K):
    rng = np.random.default_rng(K)
    X = _calib(rng, 4 * K, K)
    X[:, K // 3] = 0.0                           # a feature the calibration never activates
    H = oracle.gptq_hessian(X)
    U, dead, used = _dev_prepare(mnb, torch.from_numpy(H.astype(np.float32)).to(cuda_dev), cuda_dev)
    Uo, deado = oracle.gptq_prepare(H.astype(np.float32).astype(np.float64))
    assert used == pytest.approx(0.01)
    assert np.array_equal(np_of(dead), deado)
    got = np_of(U).astype(np.float64)
    assert np.all(np.tril(got, -1) == 0)
    assert np.linalg.norm(got - Uo) <= 1e-4 * np.linalg.norm(Uo)


def test_gptq_prepare_retries_with_more_damping(mnb, cuda_dev):
    # an indefinite 2 x 2 block (eigenvalues 2.0005 and -0.0005) inside an
    # identity: undamped, the fp32 factorisation meets a negative pivot; the
    # first retry (damping 0.001 x mean diagonal = 0.001) succeeds
    K = 64
    H = np.eye(K, dtype=np.float32)
    H[10, 11] = H[11, 10] = 1.0005
    U, dead, used = _dev_prepare(mnb, torch.from_numpy(H).to(cuda_dev), cuda_dev, percdamp=0.0)
    assert used == pytest.approx(1e-3)
    Uo, _ = oracle.gptq_prepare(H.astype(np.float64), percdamp=1e-3)
    assert np.linalg.norm(np_of(U) - Uo) <= 1e-3 * np.linalg.norm(Uo)
    # with an eigenvalue of -1 no damping up to 0.1 helps: a clear error, no U
    H[10, 11] = H[11, 10] = 2.0
    with pytest.raises(mnb.MnbError, match="not positive definite"):
        _dev_prepare(mnb, torch.from_numpy(H).to(cuda_dev), cuda_dev, percdamp=0.0)


@pytest.mark.parametrize("N,K,bs,has_zp,sdt", [(64, 256, 32, True, np.float16), (33, 512, 64, True, np.float32),
                                               (17, 256, 32, False, np.float16), (5, 128, 64, False, np.float32),
                                               (2048, 2048, 32, True, np.float16)])
def test_gptq_quantize_bit_exact(mnb, cuda_dev, N, K, bs, has_zp, sdt):
    rng = np.random.default_rng(N * 3 + K)
    X = _calib(rng, max(2 * K, 256), K)
    X[:, 5] = 0.0
    Uo, deado = oracle.gptq_prepare(oracle.gptq_hessian(X))
    U32 = np.ascontiguousarray(Uo, dtype=np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[rng.random((N, K)) < 0.01] *= 8.0       # outliers
    ref = oracle.gptq_quantize(W, U32, bs, has_zp, sdt, deado)
    tdt = torch.float16 if sdt == np.float16 else torch.float32
    got = _dev_quantize(mnb, torch.from_numpy(W).to(cuda_dev), torch.from_numpy(U32).to(cuda_dev),
                        torch.from_numpy(deado).to(cuda_dev), bs, has_zp, tdt, cuda_dev)
    assert np.array_equal(got[0], ref[0])
    assert np.array_equal(got[1].view(np.uint8), ref[1].view(np.uint8))
    if has_zp:
        assert np.array_equal(got[2], ref[2])


def test_gptq_end_to_end(mnb, cuda_dev):
    # the device's own Hessian and factor: the proxy loss within 1% of the
    # oracle's GPTQ, almost all codes equal, and well below plain RTN
    rng = np.random.default_rng(5)
    N, K, T, bs = 256, 512, 2048, 32
    X = _calib(rng, T, K, corr=1.0)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    dev = cuda_dev
    Xd = torch.from_numpy(X).half().to(dev)
    H = torch.empty((K, K), dtype=torch.float32, device=dev)
    mnb.mnb_gptq_hessian(Xd, H)
    U, dead, _ = _dev_prepare(mnb, H, dev)
    got = _dev_quantize(mnb, torch.from_numpy(W).to(dev), U, dead, bs, True, torch.float16, dev)
    Xh = Xd.float().cpu().numpy().astype(np.float64)
    Uo, deado = oracle.gptq_prepare(oracle.gptq_hessian(Xh))
    ref = oracle.gptq_quantize(W, Uo.astype(np.float32), bs, True, np.float16, deado)
    rtn = oracle.quantize_rtn(W, bs, True, np.float16)

    def loss(q):
        Wq = oracle.dequantize(q[0], q[1], q[2], K, bs)
        return float(np.sum(((W.astype(np.float64) - Wq) @ Xh.T) ** 2))

    lg, lo, lr = loss(got), loss(ref), loss(rtn)
    assert abs(lg - lo) <= 0.01 * lo
    assert lg < 0.8 * lr
    codes_g = np.concatenate([got[0] & 15, got[0] >> 4])
    codes_o = np.concatenate([ref[0] & 15, ref[0] >> 4])
    assert np.mean(codes_g == codes_o) >= 0.99
