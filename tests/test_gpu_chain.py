"""GPU parity of mnb_gemv_chain (a sequence of decode GEMVs in one launch).

Every task is checked against the oracle on the X it actually read.  Where a
task's X is the previous task's Y, the Y buffers start as NaN: a task that read
its X before the previous task had written it would carry NaNs or stale values
and fail the comparison.  Shapes cover both work splits of the kernel (a CTA
with fewer than 16 tiles cuts K over its warps; with 16 or more, each warp owns
whole tiles), ragged tile counts over the SMs, block 32 and 64, with and
without zero points, M from 1 to 8.
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

    m.mnb_device_status(clear=True)
    return m


def _weights(rng, N, K, bs, has_zp, dev):
    s = 1.0 / (6.5 * np.sqrt(K))   # keeps outputs near unit scale along a chain
    p, sc, z = random_packed(rng, N, K, bs, has_zp, np.float16, 0.5 * s, 1.5 * s)
    if not has_zp:
        # with the implicit zero point 8, uniform nibbles have mean q - 8 = -0.5,
        # a bias that grows along the chain; nibble 0 -> 8 makes the mean 0
        lo, hi = p & 15, p >> 4
        lo[lo == 0] = 8
        hi[hi == 0] = 8
        p = (lo | (hi << 4)).astype(np.uint8)
    return (p, sc, z), (to_dev(p, dev), to_dev(sc, dev), to_dev(z, dev))


def _run(mnb, tasks, M, bs, dev, times=1):
    plan = mnb.mnb_gemv_chain_plan(tasks, M, bs)
    plan_dev = plan.to(dev)
    ws = torch.zeros(mnb.mnb_gemv_chain_workspace_bytes(len(tasks)), dtype=torch.uint8, device=dev)
    for _ in range(times):
        mnb.mnb_gemv_chain(plan, plan_dev, ws)
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0, "the workspace must be zero again after a call"
    return plan, plan_dev, ws


@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("bs,has_zp", [(32, True), (32, False), (64, True)])
def test_chain_of_dependent_layers(mnb, cuda_dev, M, bs, has_zp):
    rng = np.random.default_rng(M * 100 + bs + has_zp)
    # (N, K, input): input = index of the task whose Y is this task's X (-1: x0).
    # 1024 and 2048 rows split K over warps; 6144 and 38400 rows give whole
    # tiles per warp; K = 6144 at M = 8 makes the plan use fewer warps.
    layers = [(2048, 1024, -1), (1024, 2048, 0), (6144, 1024, 1), (1024, 6144, 2), (38400, 1024, 3),
              (512, 1024, 3), (2048, 38400, 4)]
    x0 = torch.randn((M, 1024), generator=torch.Generator().manual_seed(M)).half().to(cuda_dev)
    hosts, tasks, Ys = [], [], []
    for N, K, src in layers:
        X = x0 if src < 0 else Ys[src]
        assert X.shape[1] == K
        host, dev_w = _weights(rng, N, K, bs, has_zp, cuda_dev)
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device=cuda_dev)
        tasks.append((X, *dev_w, Y, N, K, 1))
        hosts.append(host)
        Ys.append(Y)
    if M * 38400 * 2 > 100 * 1024:
        # X of 38400 fp16 per token does not fit in shared memory for M > 1
        with pytest.raises(Exception, match="MNB_ERR_SHAPE"):
            mnb.mnb_gemv_chain_plan(tasks, M, bs)
        tasks, layers = tasks[:-1], layers[:-1]
    _run(mnb, tasks, M, bs, cuda_dev)
    assert mnb.mnb_device_status() == 0
    for (N, K, src), (p, sc, z), t in zip(layers, hosts, tasks):
        xin = t[0]
        ref = oracle.matmul(np_of(xin.float()), p, sc, z, K, bs)
        assert_close(np_of(t[4].float()), ref, "f16")


def test_chain_tasks_sharing_x_without_waits(mnb, cuda_dev):
    # q, k, v read the same X: no task waits for another
    rng = np.random.default_rng(7)
    K, M = 2048, 1
    x = torch.randn((M, K), generator=torch.Generator().manual_seed(3)).half().to(cuda_dev)
    shapes = [2048, 1024, 1024, 16, 151936 // 4]
    tasks, ref = [], []
    for i, N in enumerate(shapes):
        host, dev_w = _weights(rng, N, K, 32, True, cuda_dev)
        Y = torch.empty((M, N), dtype=torch.float16, device=cuda_dev)
        tasks.append((x, *dev_w, Y, N, K, 0))
        ref.append((host, Y))
    _run(mnb, tasks, M, 32, cuda_dev)
    for (p, sc, z), Y in ref:
        assert_close(np_of(Y.float()), oracle.matmul(np_of(x.float()), p, sc, z, K, 32), "f16")


def test_chain_repeats_graph_and_pdl(mnb, cuda_dev):
    # the same plan launched again, with PDL, and replayed from a CUDA graph
    rng = np.random.default_rng(11)
    M, K = 2, 1024
    x0 = torch.randn((M, K), generator=torch.Generator().manual_seed(5)).half().to(cuda_dev)
    tasks, X, Ws = [], x0, []
    for _ in range(12):
        host, dev_w = _weights(rng, K, K, 32, True, cuda_dev)
        Y = torch.zeros((M, K), dtype=torch.float16, device=cuda_dev)
        tasks.append((X, *dev_w, Y, K, K, 1))
        Ws.append(host)
        X = Y
    plan, plan_dev, ws = _run(mnb, tasks, M, 32, cuda_dev)
    first = tasks[-1][4].clone()
    for _ in range(3):
        mnb.mnb_gemv_chain(plan, plan_dev, ws, mnb.MNB_FLAG_PDL)
    torch.cuda.synchronize()
    assert_close(np_of(tasks[-1][4].float()), np_of(first.float()), "f16")
    for t in tasks:
        t[4].zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        mnb.mnb_gemv_chain(plan, plan_dev, ws, mnb.MNB_FLAG_PDL, s)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0
    assert mnb.mnb_device_status() == 0
    xin = x0
    for (p, sc, z), t in zip(Ws, tasks):
        assert_close(np_of(t[4].float()), oracle.matmul(np_of(xin.float()), p, sc, z, K, 32), "f16")
        xin = t[4]


def test_chain_q_equal_zp_gives_exact_zero(mnb, cuda_dev):
    # every nibble equal to its block's zero point: every output is exactly 0
    M, N, K = 4, 4096, 2048
    rng = np.random.default_rng(2)
    zp = rng.integers(0, 16, (N, K // 64), dtype=np.uint8)
    zb = (zp & 15) | ((zp & 15) << 4)            # both blocks of a byte share one value
    nib = np.repeat(zb & 15, 64, axis=1)          # per element: its block's zero point
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    scales = rng.uniform(0.1, 1.0, (N, K // 32)).astype(np.float16)
    x = torch.randn((M, K)).half().to(cuda_dev)
    Y = torch.full((M, N), 7.0, dtype=torch.float16, device=cuda_dev)
    tasks = [(x, to_dev(packed, cuda_dev), to_dev(scales, cuda_dev), to_dev(zb, cuda_dev), Y, N, K, 0)]
    _run(mnb, tasks, M, 32, cuda_dev)
    assert int(Y.count_nonzero()) == 0


def test_chain_refuses_a_workspace_left_dirty(mnb, cuda_dev):
    # a failed call leaves the abort word set; the next call must run nothing
    # and say so, and run normally once the workspace is zero-filled again
    rng = np.random.default_rng(4)
    M, N, K = 1, 2048, 1024
    host, dev_w = _weights(rng, N, K, 32, True, cuda_dev)
    x = torch.randn((M, K), generator=torch.Generator().manual_seed(8)).half().to(cuda_dev)
    Y = torch.full((M, N), 7.0, dtype=torch.float16, device=cuda_dev)
    tasks = [(x, *dev_w, Y, N, K, 0)]
    plan = mnb.mnb_gemv_chain_plan(tasks, M, 32)
    plan_dev = plan.to(cuda_dev)
    ws = torch.zeros(mnb.mnb_gemv_chain_workspace_bytes(1), dtype=torch.uint8, device=cuda_dev)
    ws.view(torch.int32)[1] = 1   # the abort word follows the one task counter
    mnb.mnb_device_status(clear=True)
    mnb.mnb_gemv_chain(plan, plan_dev, ws)
    torch.cuda.synchronize()
    assert mnb.mnb_device_status(clear=True) & (1 << 3)
    assert bool((Y == 7.0).all()), "no task may run on a dirty workspace"
    ws.zero_()
    mnb.mnb_gemv_chain(plan, plan_dev, ws)
    torch.cuda.synchronize()
    assert mnb.mnb_device_status() == 0
    assert_close(np_of(Y.float()), oracle.matmul(np_of(x.float()), *host, K, 32), "f16")


def test_chain_task_wait_times_out_and_reports_it(mnb, cuda_dev):
    # fault made on the host: the test hook withholds task 0's completion count,
    # so task 1's bounded wait for its inputs runs out (after 5 ms here).  The
    # kernel must return, set status bit 2 and the abort word, leave the later
    # tasks' outputs untouched; the next call must refuse the dirty workspace
    # (bit 3); after zero-filling it, a normal call gives correct results.
    rng = np.random.default_rng(11)
    M, bs = 2, 32
    shapes = [(2048, 1024), (1024, 2048), (1024, 1024)]   # task j reads task j-1's Y
    x0 = torch.randn((M, 1024), generator=torch.Generator().manual_seed(12)).half().to(cuda_dev)
    host, tasks, Ys = [], [], []
    X = x0
    for j, (N, K) in enumerate(shapes):
        h, d = _weights(rng, N, K, bs, True, cuda_dev)
        Y = torch.full((M, N), 7.0, dtype=torch.float16, device=cuda_dev)
        tasks.append((X, *d, Y, N, K, 1 if j else 0))
        host.append(h)
        Ys.append(Y)
        X = Y
    plan = mnb.mnb_gemv_chain_plan(tasks, M, bs)
    plan_dev = plan.to(cuda_dev)
    ws = torch.zeros(mnb.mnb_gemv_chain_workspace_bytes(len(tasks)), dtype=torch.uint8, device=cuda_dev)
    mnb.mnb_device_status(clear=True)
    assert mnb._lib.mnb_test_chain_withhold(0, 5000) == 0
    try:
        mnb.mnb_gemv_chain(plan, plan_dev, ws)
        torch.cuda.synchronize()
    finally:
        assert mnb._lib.mnb_test_chain_withhold(-1, 0) == 0
    st = ctypes_status(mnb)
    assert st["rc"] == -6 and st["word"] & (1 << 2), st
    assert int(ws.view(torch.int32)[len(tasks)].item()) != 0, "the abort word must be raised"
    assert bool((Ys[1] == 7.0).all()) and bool((Ys[2] == 7.0).all()), "tasks after the timeout must not run"
    # the same workspace again: refused, nothing runs
    mnb.mnb_gemv_chain(plan, plan_dev, ws)
    torch.cuda.synchronize()
    st = ctypes_status(mnb)
    assert st["rc"] == 0 and st["word"] == (1 << 3), st
    assert bool((Ys[2] == 7.0).all())
    # zero-filled again: a normal call
    ws.zero_()
    mnb.mnb_gemv_chain(plan, plan_dev, ws)
    torch.cuda.synchronize()
    assert mnb.mnb_device_status() == 0
    assert int(ws.count_nonzero()) == 0
    X = np_of(x0.float())
    for (N, K), h, Y in zip(shapes, host, Ys):
        ref = oracle.matmul(X, *h, K, bs)
        assert_close(np_of(Y.float()), ref, "f16")
        X = np_of(Y.float())


def ctypes_status(mnb):
    """The C call's return code and the status word it read (then cleared)."""
    import ctypes

    v = ctypes.c_uint()
    rc = mnb._lib.mnb_device_status(ctypes.byref(v), 1)
    return {"rc": rc, "word": v.value}
