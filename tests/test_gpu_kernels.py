"""GPU parity of every kernel against the CPU oracle, through the C ABI binding.

Sizes are small enough for the oracle to finish in seconds while still spanning
several tiles and a ragged tail.  Bit-exact: packing, scales, zero points,
dequantized weights, embedding rows.  Tolerances (relative L2 over all outputs,
max absolute error): 1e-5 / 2e-2 for fp32 activations, 2e-3 / 2e-2 for fp16.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity_util import assert_close, np_of, random_packed, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mnb(cuda_dev):
    import int4_block_quantized_matmulnbits_b200 as m

    m.mnb_device_status(clear=True)
    return m


def _quantize_dev(mnb, W, bs, has_zp, sdt, dev):
    N, K = W.shape
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, K // bs), dtype=sdt, device=dev)
    zp = torch.empty((N, (K // bs + 1) // 2), dtype=torch.uint8, device=dev) if has_zp else None
    mnb.mnb_quantize_rtn(W.to(dev), N, K, bs, has_zp, packed, scales, zp)
    torch.cuda.synchronize()
    return packed, scales, zp


# ------------------------------------------------------------------ quantization

@pytest.mark.parametrize("N,K,bs", [(1, 32, 32), (37, 96, 32), (64, 256, 64), (130, 192, 64),
                                    (300, 1024, 32), (2048, 1024, 32)])
@pytest.mark.parametrize("has_zp", [True, False])
@pytest.mark.parametrize("sdt", [torch.float32, torch.float16])
def test_quantize_rtn_bit_exact(mnb, cuda_dev, N, K, bs, has_zp, sdt):
    g = torch.Generator().manual_seed(N * 7 + K + bs)
    W = torch.randn((N, K), generator=g) * 0.02
    W[::5] = W[::5] * 8.0                                   # outlier rows
    if N > 2:
        W[1, :bs] = 0.0                                     # an all-zero block
        W[2, :] = W[2, :].abs() + 0.01                      # all-positive blocks
    p_ref, s_ref, z_ref = oracle.quantize_rtn(W.numpy(), bs, has_zp,
                                              np.float16 if sdt == torch.float16 else np.float32)
    packed, scales, zp = _quantize_dev(mnb, W, bs, has_zp, sdt, cuda_dev)
    assert np.array_equal(np_of(packed), p_ref)
    assert np.array_equal(np_of(scales).view(np.uint8), s_ref.view(np.uint8))
    if has_zp:
        assert np.array_equal(np_of(zp), z_ref)


def test_quantize_rtn_ties_and_constructed_block(mnb, cuda_dev):
    W = np.zeros((3, 64), np.float32)
    W[0, :32] = np.repeat(np.arange(-7, 9) * 0.5, 2)          # scale 0.5, zp 7, exact
    W[1, 0], W[1, 1:16] = 15.0, np.arange(0.5, 15.0, 1.0)     # x.5 ties, scale 1
    W[2, :4] = [-7.0, 8.0, 0.5, -0.5]                          # tie after adding zp
    p_ref, s_ref, z_ref = oracle.quantize_rtn(W, 32)
    packed, scales, zp = _quantize_dev(mnb, torch.from_numpy(W), 32, True, torch.float32, cuda_dev)
    assert np.array_equal(np_of(packed), p_ref)
    assert np.array_equal(np_of(scales), s_ref)
    assert np.array_equal(np_of(zp), z_ref)


# ------------------------------------------------------------------ dequantization

@pytest.mark.parametrize("N,K,bs,has_zp", [(37, 96, 32, True), (64, 256, 64, True), (16, 128, 32, False)])
@pytest.mark.parametrize("sdt", [np.float32, np.float16])
@pytest.mark.parametrize("odt", [torch.float32, torch.float16])
def test_dequantize_bit_exact(mnb, cuda_dev, N, K, bs, has_zp, sdt, odt):
    rng = np.random.default_rng(N + K)
    packed, scales, zp = random_packed(rng, N, K, bs, has_zp, sdt, 0.001, 0.5)
    out = torch.empty((N, K), dtype=odt, device=cuda_dev)
    mnb.mnb_dequantize(to_dev(packed, cuda_dev), to_dev(scales, cuda_dev), to_dev(zp, cuda_dev),
                       N, K, bs, out)
    ref = oracle.dequantize(packed, scales, zp, K, bs, np.float16 if odt == torch.float16 else np.float32)
    assert np.array_equal(np_of(out).view(np.uint8), ref.view(np.uint8))


# ------------------------------------------------------------------ GEMV

GEMV_CASES = [
    # M, N, K, bs, has_zp, act, scale
    (1, 2048, 1024, 32, True, "f32", np.float32),
    (3, 37, 96, 32, True, "f32", np.float32),
    (16, 64, 128, 64, False, "f32", np.float16),
    (1, 37, 96, 32, True, "f16", np.float16),
    (1, 1024, 2048, 32, True, "f16", np.float16),
    (2, 3000, 1024, 64, True, "f16", np.float16),
    (5, 130, 6144, 32, True, "f16", np.float16),
    (8, 512, 3072, 32, False, "f16", np.float16),
    (9, 256, 2048, 64, True, "f16", np.float16),
    (16, 2048, 2048, 32, True, "f16", np.float16),
    (16, 48, 64, 32, True, "f16", np.float32),
    (4, 16, 32, 32, True, "f16", np.float16),
    # decoder-like shapes, ragged N, fp32 scales, no zero points
    (1, 4096, 2048, 32, True, "f16", np.float16),
    (1, 2048, 6144, 32, True, "f16", np.float16),
    (2, 1024, 3072, 32, True, "f16", np.float16),
    (3, 1000, 1024, 64, False, "f16", np.float32),
    (8, 777, 512, 32, True, "f16", np.float32),
    (1, 50, 256, 32, True, "f16", np.float16),
    (6, 2000, 2048, 64, True, "f16", np.float16),
    (1, 300, 4096, 64, False, "f16", np.float32),
    (4, 3333, 1024, 32, False, "f16", np.float16),
    # four MMA column groups (17 <= M <= 32)
    (17, 2048, 2048, 32, True, "f16", np.float16),
    (24, 1000, 6144, 32, True, "f16", np.float16),
    (32, 6144, 2048, 32, True, "f16", np.float16),
    (32, 300, 1024, 64, False, "f16", np.float32),
    (29, 151936 // 8, 1024, 32, True, "f16", np.float16),
]


def _run_gemv(mnb, dev, X, packed, scales, zp, M, N, K, bs, flags=0):
    Y = torch.empty((M, N), dtype=X.dtype, device=dev)
    mnb.mnb_gemv(X, to_dev(packed, dev), to_dev(scales, dev), to_dev(zp, dev), Y, M, N, K, bs, flags)
    torch.cuda.synchronize()
    return Y


@pytest.mark.parametrize("M,N,K,bs,has_zp,act,sdt", GEMV_CASES)
def test_gemv_parity(mnb, cuda_dev, M, N, K, bs, has_zp, act, sdt):
    rng = np.random.default_rng(M * 1000 + N + K)
    packed, scales, zp = random_packed(rng, N, K, bs, has_zp, sdt)
    tdt = torch.float16 if act == "f16" else torch.float32
    X = torch.randn((M, K), generator=torch.Generator().manual_seed(K)).to(tdt)
    ref = oracle.matmul(X.float().numpy(), packed, scales, zp, K, bs)
    Y = _run_gemv(mnb, cuda_dev, X.to(cuda_dev), packed, scales, zp, M, N, K, bs)
    assert_close(np_of(Y.float()), ref, act)


RESIDENT_CASES = [
    # N, K, bs, has_zp: the one-token kernel whose CTAs hold their weights in
    # shared memory (one tile per CTA, tiles cut between warps, several tiles
    # per CTA, the streamed lm_head shape, ragged N, block 64, no zero points)
    (2048, 2048, 32, True), (1024, 2048, 32, True), (6144, 2048, 32, True), (2048, 6144, 32, True),
    (151936, 2048, 32, True), (1000, 1024, 32, True), (3000, 1024, 64, True), (777, 512, 64, False),
    (50, 256, 32, True), (17, 2048, 32, False), (1, 256, 32, True), (4736, 3072, 64, True),
]


@pytest.mark.parametrize("N,K,bs,has_zp", RESIDENT_CASES)
def test_gemv_resident_one_token(mnb, cuda_dev, N, K, bs, has_zp):
    # M = 1 through the resident kernel (the default) and through the general
    # decode kernel: both against the oracle
    rng = np.random.default_rng(N + 7 * K)
    packed, scales, zp = random_packed(rng, N, K, bs, has_zp, np.float16)
    X = torch.randn((1, K), generator=torch.Generator().manual_seed(N)).half()
    ref = oracle.matmul(X.float().numpy(), packed, scales, zp, K, bs)
    for resident in (1, 0):
        assert mnb._lib.mnb_tune_gemv_resident(resident) == 0
        try:
            Y = _run_gemv(mnb, cuda_dev, X.to(cuda_dev), packed, scales, zp, 1, N, K, bs)
        finally:
            mnb._lib.mnb_tune_gemv_resident(1)
        assert_close(np_of(Y.float()), ref, "f16")
    assert mnb.mnb_device_status() == 0


@pytest.mark.parametrize("N,K,bs,has_zp", [(2048, 2048, 32, True), (6144, 2048, 32, True),
                                           (2048, 6144, 32, True), (4736, 3072, 64, True), (777, 512, 64, False)])
def test_gemv_resident_is_deterministic(mnb, cuda_dev, N, K, bs, has_zp):
    # consecutive one-token launches alternate between two launch shapes with
    # different warp counts; the sums are cut at the same places in both, so
    # every call returns the same bits (plain and with the SwiGLU epilogue)
    rng = np.random.default_rng(N + K + bs)
    packed, scales, zp = (to_dev(a, cuda_dev) for a in random_packed(rng, N, K, bs, has_zp, np.float16))
    X = torch.randn((1, K), generator=torch.Generator().manual_seed(K + 1)).half().to(cuda_dev)
    for swiglu in ((False, True) if N % 16 == 0 else (False,)):
        outs = []
        for _ in range(5):
            Y = torch.empty((1, N // 2 if swiglu else N), dtype=torch.float16, device=cuda_dev)
            if swiglu:
                mnb.mnb_gemv_swiglu(X, packed, scales, zp, Y, 1, N, K, bs)
            else:
                mnb.mnb_gemv(X, packed, scales, zp, Y, 1, N, K, bs)
            outs.append(Y)
        torch.cuda.synchronize()
        for Y in outs[1:]:
            assert torch.equal(Y, outs[0])
    assert mnb.mnb_device_status() == 0


def test_gemv_resident_large_inputs_and_pdl(mnb, cuda_dev):
    # activations far from unit scale (the raw-code sums grow with |x|), and a
    # chain of dependent PDL launches: each GEMV reads the previous one's output
    rng = np.random.default_rng(3)
    K = 2048
    # x ~ 50 N(0, 1) meets scales 50x smaller, so every output stays near unit
    # scale (a gain of ~1 per GEMV for uniform codes and zero points) while the
    # first GEMV's raw-code sums are 50x larger than usual
    ws = [random_packed(rng, K, K, 32, True, np.float16, 0.1 / np.sqrt(K) / (50 if i == 0 else 1),
                        0.2 / np.sqrt(K) / (50 if i == 0 else 1)) for i in range(4)]
    x = (torch.randn((1, K), generator=torch.Generator().manual_seed(9)) * 50).half()
    dev = [tuple(to_dev(a, cuda_dev) for a in w) for w in ws]
    bufs = [x.to(cuda_dev)] + [torch.full((1, K), float("nan"), dtype=torch.float16, device=cuda_dev) for _ in ws]
    for i, (p_, s_, z_) in enumerate(dev):
        mnb.mnb_gemv(bufs[i], p_, s_, z_, bufs[i + 1], 1, K, K, 32, mnb.MNB_FLAG_PDL)
    torch.cuda.synchronize()
    cur = x.float().numpy()
    for i, w in enumerate(ws):
        ref = oracle.matmul(cur, *w, K, 32)
        got = np_of(bufs[i + 1].float())
        assert np.abs(ref).max() < 16, "outputs must stay near unit scale for the absolute tolerance"
        assert_close(got, ref, "f16")
        cur = got   # the next GEMV read the fp16 values this one stored


@pytest.mark.parametrize("N,K", [(64, 256), (80, 1024)])
def test_gemv_q_equal_zp_gives_exact_zero(mnb, cuda_dev, N, K):
    bs, M = 32, 3
    z = np.random.default_rng(1).integers(0, 16, (N, K // bs))
    q = np.repeat(z, bs, axis=1)
    packed = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    zp = (z[:, 0::2] | (z[:, 1::2] << 4)).astype(np.uint8)
    scales = np.full((N, K // bs), 0.5, np.float16)
    for dt in (torch.float16, torch.float32):
        X = torch.randn((M, K)).to(dt).to(cuda_dev)
        Y = _run_gemv(mnb, cuda_dev, X, packed, scales, zp, M, N, K, bs)
        assert torch.count_nonzero(Y).item() == 0


def test_gemv_rtn_quantized_weights(mnb, cuda_dev):
    # the product path end to end: RTN on the device, GEMV on the device, oracle on its own RTN
    N, K, bs, M = 1024, 2048, 32, 1
    W = workloads.weight(2, 0, 4, N, K, outliers=True)
    p_ref, s_ref, z_ref = oracle.quantize_rtn(W.numpy(), bs, True, np.float16)
    packed, scales, zp = _quantize_dev(mnb, W, bs, True, torch.float16, cuda_dev)
    X = workloads.activations(2, M, K)
    Y = torch.empty((M, N), dtype=torch.float16, device=cuda_dev)
    mnb.mnb_gemv(X.to(cuda_dev), packed, scales, zp, Y, M, N, K, bs)
    ref = oracle.matmul(X.float().numpy(), p_ref, s_ref, z_ref, K, bs)
    assert_close(np_of(Y.float()), ref, "f16")


def test_gemv_pdl_chain_and_graph_match_eager(mnb, cuda_dev):
    # Y of one call is X of the next: the PDL launches must still see it
    rng = np.random.default_rng(9)
    K = 1024
    layers = [random_packed(rng, K, K, 32, True, np.float16, 0.003, 0.004) for _ in range(6)]
    dev_layers = [(to_dev(p, cuda_dev), to_dev(s, cuda_dev), to_dev(z, cuda_dev)) for p, s, z in layers]
    x0 = torch.randn((1, K)).half().to(cuda_dev)

    def chain(flags, bufs):
        x = x0
        for (p, s, z), y in zip(dev_layers, bufs):
            mnb.mnb_gemv(x, p, s, z, y, 1, K, K, 32, flags)
            x = y
        return x

    bufs_plain = [torch.empty((1, K), dtype=torch.float16, device=cuda_dev) for _ in layers]
    bufs_pdl = [torch.empty((1, K), dtype=torch.float16, device=cuda_dev) for _ in layers]
    ref = chain(0, bufs_plain).clone()
    for _ in range(3):
        got = chain(mnb.MNB_FLAG_PDL, bufs_pdl)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    # the same chain captured in a CUDA graph
    bufs_g = [torch.zeros((1, K), dtype=torch.float16, device=cuda_dev) for _ in layers]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        chain(mnb.MNB_FLAG_PDL, bufs_g)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(bufs_g[-1], ref)
    # first link against the oracle
    p, sc, z = layers[0]
    r0 = oracle.matmul(x0.float().cpu().numpy(), p, sc, z, K, 32)
    assert_close(np_of(bufs_plain[0].float()), r0, "f16")


# ------------------------------------------------------------------ GEMV + SwiGLU epilogue

def _interleave8(g, u):
    """Rows in groups of 16: 8 gate rows, then the 8 up rows of the same outputs."""
    I = g.shape[0]
    return np.stack([g.reshape(I // 8, 8, *g.shape[1:]), u.reshape(I // 8, 8, *u.shape[1:])],
                    axis=1).reshape(2 * I, *g.shape[1:])


@pytest.mark.parametrize("M,I,K,bs,has_zp,sdt", [(1, 6144, 2048, 32, True, np.float16),
                                                 (1, 1024, 2048, 32, True, np.float16),
                                                 (1, 3000, 1024, 64, False, np.float16),
                                                 (1, 1024, 6144, 32, True, np.float16),
                                                 (4, 3072, 1024, 32, True, np.float16),
                                                 (16, 1000, 1024, 64, True, np.float32),
                                                 (3, 8, 256, 32, False, np.float16),
                                                 (2, 1024, 6144, 32, True, np.float16)])
def test_gemv_swiglu(mnb, cuda_dev, M, I, K, bs, has_zp, sdt):
    rng = np.random.default_rng(I + K + M)
    pg, sg, zg = random_packed(rng, I, K, bs, has_zp, sdt)
    pu, su, zu = random_packed(rng, I, K, bs, has_zp, sdt)
    X = torch.randn((M, K), generator=torch.Generator().manual_seed(I)).half()
    ref = oracle.swiglu(oracle.matmul(X.float().numpy(), pg, sg, zg, K, bs),
                        oracle.matmul(X.float().numpy(), pu, su, zu, K, bs))
    packed, scales = _interleave8(pg, pu), _interleave8(sg, su)
    zp = _interleave8(zg, zu) if has_zp else None
    Y = torch.empty((M, I), dtype=torch.float16, device=cuda_dev)
    mnb.mnb_gemv_swiglu(X.to(cuda_dev), to_dev(packed, cuda_dev), to_dev(scales, cuda_dev), to_dev(zp, cuda_dev), Y,
                        M, 2 * I, K, bs)
    torch.cuda.synchronize()
    assert_close(np_of(Y.float()), ref, "f16")


def test_gemv_swiglu_layout_helper(mnb, cuda_dev):
    from int4_block_quantized_matmulnbits_b200.step import QLinear, swiglu_interleave

    K, I, M = 2048, 6144, 1
    g = QLinear.quantize(workloads.weight(2, 0, 4, I, K, outliers=True).to(cuda_dev), 32)
    u = QLinear.quantize(workloads.weight(2, 0, 5, I, K, outliers=True).to(cuda_dev), 32)
    gu = swiglu_interleave(g, u)
    X = workloads.activations(2, M, K).to(cuda_dev)
    Y = torch.empty((M, I), dtype=torch.float16, device=cuda_dev)
    gu.gemv_swiglu(X, Y)
    yg = torch.empty((M, I), dtype=torch.float16, device=cuda_dev)
    yu = torch.empty((M, I), dtype=torch.float16, device=cuda_dev)
    g.gemv(X, yg)
    u.gemv(X, yu)
    torch.cuda.synchronize()
    ref = oracle.swiglu(oracle.matmul(X.float().cpu().numpy(), np_of(g.packed), np_of(g.scales), np_of(g.zp), K, 32),
                        oracle.matmul(X.float().cpu().numpy(), np_of(u.packed), np_of(u.scales), np_of(u.zp), K, 32))
    assert_close(np_of(Y.float()), ref, "f16")
    assert_close(np_of(Y.float()), oracle.swiglu(np_of(yg.float()), np_of(yu.float())), "f16")


# ------------------------------------------------------------------ GEMV + greedy argmax

ARGMAX_CASES = [
    # M, N, K, bs, has_zp, scale
    (1, 151936, 2048, 32, True, np.float16),   # the 1.7B lm_head
    (1, 1000, 2048, 32, True, np.float16),     # one token: tiles cut between warps
    (1, 33, 256, 32, False, np.float16),
    (4, 5000, 1024, 64, True, np.float16),
    (3, 777, 512, 32, False, np.float32),
    (16, 1000, 2048, 32, True, np.float16),
    (8, 33, 256, 32, True, np.float16),
]


def _run_argmax(mnb, dev, X, packed, scales, zp, M, N, K, bs, ws=None):
    Y = torch.empty((M, N), dtype=torch.float16, device=dev)
    ids = torch.full((M,), -1, dtype=torch.int32, device=dev)
    mx = torch.empty((M,), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.zeros(mnb.mnb_gemv_argmax_workspace_bytes(M), dtype=torch.uint8, device=dev)
    mnb.mnb_gemv_argmax(X, to_dev(packed, dev), to_dev(scales, dev), to_dev(zp, dev), Y, M, N, K, bs, ids, mx, ws)
    torch.cuda.synchronize()
    return Y, ids, mx, ws


@pytest.mark.parametrize("M,N,K,bs,has_zp,sdt", ARGMAX_CASES)
def test_gemv_argmax(mnb, cuda_dev, M, N, K, bs, has_zp, sdt):
    rng = np.random.default_rng(N + M)
    packed, scales, zp = random_packed(rng, N, K, bs, has_zp, sdt)
    X = torch.randn((M, K), generator=torch.Generator().manual_seed(N)).half()
    Y, ids, mx, ws = _run_argmax(mnb, cuda_dev, X.to(cuda_dev), packed, scales, zp, M, N, K, bs)
    ref = oracle.matmul(X.float().numpy(), packed, scales, zp, K, bs)
    y = np_of(Y.float())
    assert_close(y, ref, "f16")
    ids_np, mx_np = np_of(ids), np_of(mx)
    # the token is the first maximum of the logits the kernel wrote ...
    assert np.array_equal(ids_np, np.argmax(y, axis=1))
    assert np.array_equal(mx_np, y[np.arange(M), ids_np])
    # ... and a valid greedy choice for the exact logits
    assert np.all(ref[np.arange(M), ids_np] >= ref.max(axis=1) - 2e-2)
    # the workspace counter is back at zero, so the same workspace serves again
    assert int(np_of(ws[:4].view(torch.int32))[0]) == 0
    Y2, ids2, mx2, _ = _run_argmax(mnb, cuda_dev, X.to(cuda_dev), packed, scales, zp, M, N, K, bs, ws)
    assert torch.equal(ids2, ids) and torch.equal(Y2, Y) and torch.equal(mx2, mx)


def test_gemv_argmax_ties_take_the_first_row(mnb, cuda_dev):
    N, K, bs, M = 300, 512, 32, 2
    rng = np.random.default_rng(5)
    packed = np.zeros((N, K // 2), np.uint8)
    zp = np.full((N, K // bs // 2), 0x88, np.uint8)      # zp = 8 in every block
    packed[:] = 0x88                                     # q = zp: logit exactly 0 for rows 0..99
    row = rng.integers(0, 256, K // 2, dtype=np.uint8)
    packed[100:] = row                                   # rows 100..299 identical
    scales = np.full((N, K // bs), 0.25, np.float16)
    X = torch.randn((M, K), generator=torch.Generator().manual_seed(11)).half()
    Y, ids, _, _ = _run_argmax(mnb, cuda_dev, X.to(cuda_dev), packed, scales, zp, M, N, K, bs)
    y = np_of(Y.float())
    for m in range(M):
        assert np.all(y[m, 100:] == y[m, 100])
        assert int(np_of(ids)[m]) == (100 if y[m, 100] > 0 else 0)


# ------------------------------------------------------------------ GEMM (tcgen05)

GEMM_CASES = [
    # M, N, K, bs, has_zp, scale
    (1, 128, 64, 32, True, np.float16),
    (16, 128, 128, 64, True, np.float16),
    (63, 256, 192, 32, False, np.float16),
    (64, 1024, 2048, 32, True, np.float16),
    (100, 384, 1024, 64, True, np.float16),
    (256, 512, 2048, 32, True, np.float16),
    (300, 128, 6144, 32, True, np.float16),
    (420, 2048, 1024, 32, True, np.float16),
    (1024, 256, 512, 64, False, np.float16),
    # more tilings: 48 tiles of 256 tokens, one tile per SM, more tiles than
    # SMs, ragged token tiles with block 64
    (1024, 1536, 1024, 32, True, np.float16),
    (256, 18944, 256, 32, True, np.float16),
    (256, 20480, 512, 32, True, np.float16),
    (260, 1280, 768, 64, True, np.float16),
]


@pytest.mark.parametrize("M,N,K,bs,has_zp,sdt", GEMM_CASES)
def test_gemm_parity(mnb, cuda_dev, M, N, K, bs, has_zp, sdt):
    rng = np.random.default_rng(M * 31 + N + K)
    packed, scales, zp = random_packed(rng, N, K, bs, has_zp, sdt)
    X = torch.randn((M, K), generator=torch.Generator().manual_seed(M + K)).half()
    Y = torch.full((M, N), float("nan"), dtype=torch.float16, device=cuda_dev)
    mnb.mnb_gemm(X.to(cuda_dev), to_dev(packed, cuda_dev), to_dev(scales, cuda_dev), to_dev(zp, cuda_dev),
                 Y, M, N, K, bs)
    torch.cuda.synchronize()
    assert mnb.mnb_device_status() == 0
    ref = oracle.matmul(X.float().numpy(), packed, scales, zp, K, bs)
    assert_close(np_of(Y.float()), ref, "f16")


def test_gemm_matches_dequantized_weights_exactly_where_exact(mnb, cuda_dev):
    # power-of-two scales and small integers: every product and sum is exact in fp32
    N, K, M, bs = 256, 512, 80, 32
    rng = np.random.default_rng(5)
    packed, _, zp = random_packed(rng, N, K, bs, True, np.float16)
    scales = (2.0 ** rng.integers(-6, -2, (N, K // bs))).astype(np.float16)
    X = torch.from_numpy(rng.integers(-4, 5, (M, K)).astype(np.float16))
    Y = torch.empty((M, N), dtype=torch.float16, device=cuda_dev)
    mnb.mnb_gemm(X.to(cuda_dev), to_dev(packed, cuda_dev), to_dev(scales, cuda_dev), to_dev(zp, cuda_dev),
                 Y, M, N, K, bs)
    ref = oracle.matmul(X.float().numpy(), packed, scales, zp, K, bs)
    assert np.array_equal(np_of(Y).astype(np.float64), ref.astype(np.float16).astype(np.float64))


@pytest.mark.parametrize("M,N,K", [(1024, 256, 512), (64, 1024, 2048), (256, 512, 2048), (1024, 1536, 1024)])
def test_gemm_split_k_is_deterministic(mnb, cuda_dev, M, N, K):
    # these shapes split K over 2- and 4-CTA clusters; the owner of each column
    # chunk adds the other ranks' partial sums in rank order, so repeated calls
    # give the same bits
    rng = np.random.default_rng(M + N)
    packed, scales, zp = random_packed(rng, N, K, 32, True, np.float16)
    dp, ds, dz = to_dev(packed, cuda_dev), to_dev(scales, cuda_dev), to_dev(zp, cuda_dev)
    X = torch.randn((M, K), generator=torch.Generator().manual_seed(N)).half().to(cuda_dev)
    outs = []
    for _ in range(3):
        Y = torch.empty((M, N), dtype=torch.float16, device=cuda_dev)
        mnb.mnb_gemm(X, dp, ds, dz, Y, M, N, K, 32)
        outs.append(Y)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    assert_close(np_of(outs[0].float()), oracle.matmul(np_of(X.float()), packed, scales, zp, K, 32), "f16")


def test_gemm_q_equal_zp_gives_exact_zero(mnb, cuda_dev):
    N, K, bs, M = 128, 256, 64, 70
    z = np.random.default_rng(2).integers(0, 16, (N, K // bs))
    q = np.repeat(z, bs, axis=1)
    packed = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    zp = (z[:, 0::2] | (z[:, 1::2] << 4)).astype(np.uint8)
    scales = np.full((N, K // bs), 0.25, np.float16)
    Y = torch.ones((M, N), dtype=torch.float16, device=cuda_dev)
    mnb.mnb_gemm(torch.randn((M, K)).half().to(cuda_dev), to_dev(packed, cuda_dev), to_dev(scales, cuda_dev),
                 to_dev(zp, cuda_dev), Y, M, N, K, bs)
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y).item() == 0


# ------------------------------------------------------------------ embedding gather

@pytest.mark.parametrize("M,N,K,bs,has_zp,act", [
    (1, 256, 512, 32, True, "f16"), (16, 384, 1024, 32, True, "f16"), (17, 384, 1024, 32, True, "f16"),
    (20, 256, 2048, 64, True, "f16"), (21, 256, 512, 32, False, "f16"), (33, 1024, 256, 32, True, "f16"),
    (64, 128, 1024, 32, True, "f16"), (130, 384, 512, 64, False, "f16"), (40, 200, 512, 32, True, "f16"),
    (17, 256, 512, 32, True, "f32"), (40, 130, 256, 64, True, "f32")])
def test_matmul_dispatch(mnb, cuda_dev, M, N, K, bs, has_zp, act):
    # one entry point for any M: GEMV launches of up to 16 tokens or the GEMM
    rng = np.random.default_rng(M * 7 + N + K)
    packed, scales, zp = random_packed(rng, N, K, bs, has_zp, np.float16)
    tdt = torch.float16 if act == "f16" else torch.float32
    X = torch.randn((M, K), generator=torch.Generator().manual_seed(M + K)).to(tdt)
    Y = torch.full((M, N), float("nan"), dtype=tdt, device=cuda_dev)
    mnb.mnb_matmul(X.to(cuda_dev), to_dev(packed, cuda_dev), to_dev(scales, cuda_dev), to_dev(zp, cuda_dev), Y,
                   M, N, K, bs)
    torch.cuda.synchronize()
    assert_close(np_of(Y.float()), oracle.matmul(X.float().numpy(), packed, scales, zp, K, bs), act)


@pytest.mark.parametrize("V,D,T", [(1000, 1024, 4096), (50, 16, 1), (300, 80, 37)])
@pytest.mark.parametrize("odt", [torch.float16, torch.float32])
def test_embed_gather_bit_exact(mnb, cuda_dev, V, D, T, odt):
    table, scales, ids = workloads.embed_inputs(7, V, D, T)
    ids = ids.clone()
    if T > 3:
        ids[1], ids[2] = -5, V         # out of range -> zero rows + status bit
    status = torch.zeros((1,), dtype=torch.int32, device=cuda_dev)
    out = torch.full((T, D), 7.0, dtype=odt, device=cuda_dev)
    mnb.mnb_embed_gather(table.to(cuda_dev), scales.to(cuda_dev), V, D, ids.to(cuda_dev), T, out, status)
    ref, st = oracle.embed_gather(table.numpy(), scales.numpy(), ids.numpy(),
                                  np.float16 if odt == torch.float16 else np.float32)
    assert np.array_equal(np_of(out).view(np.uint8), ref.view(np.uint8))
    assert int(status.item()) == st


def test_no_timeouts_recorded(mnb, cuda_dev):
    torch.cuda.synchronize()
    assert mnb.mnb_device_status() == 0
