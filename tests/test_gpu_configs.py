"""Parity at the full workload sizes, in the launch configuration bench.py times.

Each workload's weights are generated and RTN-quantized on the device, then the
whole pass (decode-step GEMVs or prefill GEMMs, every projection, PDL launches,
captured in a CUDA graph) runs exactly as the benchmark runs it.  The oracle
re-quantizes the checked weight rows of every projection from the same fp32
weights (bit-exact check of packed bytes, scales and zero points, once per
model) and recomputes those output columns in double precision (tolerance
check, per pass).  Which rows: a seeded sample of every projection (always
with the first and last row), every row of the layers named in full_layers,
or every row of every projection (all_rows).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity_util import assert_close, np_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def step_mod(cuda_dev):
    from int4_block_quantized_matmulnbits_b200 import step

    return step


def _sample_rows(N, count, seed):
    if count >= N:
        return np.arange(N)
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=count - 2, replace=False).tolist())
    rows.update([0, N - 1])
    return np.array(sorted(rows))


_MODELS = {}


def model(step_mod, cfg_name, rows_per_proj, full_layers=(), all_rows=False):
    """build_model, cached per workload for the whole module."""
    key = (cfg_name, rows_per_proj, tuple(full_layers), all_rows)
    if key not in _MODELS:
        _MODELS.clear()
        torch.cuda.empty_cache()
        _MODELS[key] = build_model(step_mod, cfg_name, rows_per_proj, full_layers, all_rows)
    return _MODELS[key]


def build_model(step_mod, cfg_name, rows_per_proj, full_layers=(), all_rows=False, dev="cuda"):
    """QLinears of a workload, and per projection the checked rows with the
    oracle's own RTN of them (bit-compared here with the device's)."""
    cfg = workloads.CONFIGS[cfg_name]
    sdt = torch.float16 if cfg["scale"] == "f16" else torch.float32
    ndt = np.float16 if cfg["scale"] == "f16" else np.float32
    lins, samples = [], []
    for lin in workloads.config_linears(cfg_name):
        W = workloads.weight(cfg["seed"], lin.layer, lin.proj, lin.N, lin.K, cfg.get("outliers", False), device=dev)
        q = step_mod.QLinear.quantize(W, cfg["bs"], cfg["has_zp"], sdt, name=f"{lin.name}{lin.layer}")
        count = lin.N if (all_rows or lin.layer in full_layers) else rows_per_proj
        rows = _sample_rows(lin.N, count, lin.layer * 16 + lin.proj)
        idx = torch.from_numpy(rows).to(dev)
        pr, sr, zr = oracle.quantize_rtn(W[idx].cpu().numpy(), cfg["bs"], cfg["has_zp"], ndt)
        del W
        assert np.array_equal(np_of(q.packed[idx]), pr), q.name
        assert np.array_equal(np_of(q.scales[idx]).view(np.uint8), sr.view(np.uint8)), q.name
        if cfg["has_zp"]:
            assert np.array_equal(np_of(q.zp[idx]), zr), q.name
        samples.append((rows, pr, sr, zr))
        lins.append(q)
    torch.cuda.synchronize()
    return cfg, lins, samples


def check_pass(cfg, lins, samples, p, act, max_rows=None):
    """Checked output columns of every projection within tolerance.  max_rows
    thins each projection's checked rows to an evenly spaced subset."""
    for q, (rows, pr, sr, zr), X, Y in zip(lins, samples, p.X, p.Y):
        if max_rows is not None and len(rows) > max_rows:
            sel = np.unique(np.linspace(0, len(rows) - 1, max_rows).astype(np.int64))
            rows, pr, sr = rows[sel], pr[sel], sr[sel]
            zr = None if zr is None else zr[sel]
        ref = oracle.matmul(np_of(X.float()), pr, sr, zr, q.K, cfg["bs"])
        got = np_of(Y[:, torch.from_numpy(rows).to(Y.device)].float())
        assert_close(got, ref, act)


def _fill_inputs(p, seed, act_dtype):
    for i, x in enumerate(p.X):
        x.copy_(workloads.activations(seed, x.shape[0], x.shape[1], act_dtype, tag=i))


def _run_graph(p):
    p.capture()
    p.replay()
    torch.cuda.synchronize()


def test_single_gemv_fp32(step_mod, cuda_dev):
    cfg, lins, samples = build_model(step_mod, "single_gemv", 2048)
    p = step_mod.Pass(lins, 1, "gemv", torch.float32)
    _fill_inputs(p, cfg["seed"], torch.float32)
    _run_graph(p)
    check_pass(cfg, lins, samples, p, "f32")


def test_qwen3_0p6b_decode_step(step_mod, cuda_dev):
    cfg, lins, samples = build_model(step_mod, "qwen3_0p6b_decode", 96, full_layers=(0,))
    p = step_mod.Pass(lins, 1, "gemv", torch.float16)
    _fill_inputs(p, cfg["seed"], torch.float16)
    _run_graph(p)
    check_pass(cfg, lins, samples, p, "f16")


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16])
def test_qwen3_1p7b_decode_step(step_mod, cuda_dev, M):
    cfg, lins, samples = model(step_mod, "qwen3_1p7b_decode", 48, full_layers=(27,))
    p = step_mod.Pass(lins, M, "gemv", torch.float16)
    _fill_inputs(p, cfg["seed"] + M, torch.float16)
    _run_graph(p)
    check_pass(cfg, lins, samples, p, "f16")


@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_qwen3_1p7b_decode_step_one_launch(step_mod, cuda_dev, M):
    # the same 197 GEMVs as one mnb_gemv_chain launch, each waiting for the previous
    cfg, lins, samples = model(step_mod, "qwen3_1p7b_decode", 48, full_layers=(27,))
    p = step_mod.Pass(lins, M, "gemv", torch.float16, chain=True)
    assert p.launches == 1
    _fill_inputs(p, cfg["seed"] + M, torch.float16)
    _run_graph(p)
    check_pass(cfg, lins, samples, p, "f16")


@pytest.mark.parametrize("M", [1, 16])
def test_qwen3_1p7b_decode_step_fused_layout(step_mod, cuda_dev, M):
    # q|k|v and gate|up stored row-concatenated: one GEMV per group, same outputs
    cfg, lins, samples = model(step_mod, "qwen3_1p7b_decode", 48, full_layers=(27,))
    fused = step_mod.fuse_decoder(lins)
    assert len(fused) == 28 * 4 + 1
    p = step_mod.Pass(fused, M, "gemv", torch.float16)
    _fill_inputs(p, cfg["seed"] + M, torch.float16)
    _run_graph(p)

    class View:   # per-projection views of the fused pass, in the original order
        X, Y = [], []

    v = View()
    for f, x, y in zip(fused, p.X, p.Y):
        off = 0
        for _, n in getattr(f, "parts", [(f.name, f.N)]):
            v.X.append(x)
            v.Y.append(y[:, off:off + n])
            off += n
    check_pass(cfg, lins, samples, v, "f16")


@pytest.mark.parametrize("M", [64, 256, 420, 1024])
def test_qwen3_1p7b_prefill(step_mod, cuda_dev, M):
    # every output column of layer 0, 256 sampled columns of every other projection
    cfg, lins, samples = model(step_mod, "qwen3_1p7b_prefill", 256, full_layers=(0,))
    p = step_mod.Pass(lins, M, "gemm", torch.float16)
    _fill_inputs(p, cfg["seed"] + M, torch.float16)
    _run_graph(p)
    import int4_block_quantized_matmulnbits_b200 as mnb

    assert mnb.mnb_device_status() == 0
    check_pass(cfg, lins, samples, p, "f16")


def test_qwen3_1p7b_prefill_fused_layout(step_mod, cuda_dev):
    # q|k|v and gate|up row-concatenated: one GEMM per group, the same outputs
    cfg, lins, samples = model(step_mod, "qwen3_1p7b_prefill", 256, full_layers=(0,))
    fused = step_mod.fuse_decoder(lins)
    assert len(fused) == 28 * 4
    M = 420
    p = step_mod.Pass(fused, M, "gemm", torch.float16)
    _fill_inputs(p, cfg["seed"] + M, torch.float16)
    _run_graph(p)

    class View:   # per-projection views of the fused pass, in the original order
        X, Y = [], []

    v = View()
    for f, x, y in zip(fused, p.X, p.Y):
        off = 0
        for _, n in getattr(f, "parts", [(f.name, f.N)]):
            v.X.append(x)
            v.Y.append(y[:, off:off + n])
            off += n
    check_pass(cfg, lins, samples, v, "f16")


@pytest.mark.parametrize("M", [17, 20, 32, 63])
def test_qwen3_1p7b_cached_prefill(step_mod, cuda_dev, M):
    # mnb_matmul: GEMV launches of 16 tokens up to M = 20, the tensor-core GEMM above
    cfg, lins, samples = model(step_mod, "qwen3_1p7b_cached_prefill", 24)
    p = step_mod.Pass(lins, M, "matmul", torch.float16)
    _fill_inputs(p, cfg["seed"] + M, torch.float16)
    _run_graph(p)
    check_pass(cfg, lins, samples, p, "f16")


@pytest.mark.parametrize("M", [42, 390])
def test_audio_encoder_prefill(step_mod, cuda_dev, M):
    cfg, lins, samples = model(step_mod, "audio_encoder_prefill", 24)
    p = step_mod.Pass(lins, M, "gemm", torch.float16)
    _fill_inputs(p, cfg["seed"] + M, torch.float16)
    _run_graph(p)
    check_pass(cfg, lins, samples, p, "f16")


def test_qwen3_0p6b_decode_step_one_launch(step_mod, cuda_dev):
    cfg, lins, samples = build_model(step_mod, "qwen3_0p6b_decode", 96, full_layers=(0,))
    p = step_mod.Pass(lins, 1, "gemv", torch.float16, chain=True)
    _fill_inputs(p, cfg["seed"], torch.float16)
    _run_graph(p)
    check_pass(cfg, lins, samples, p, "f16")


@pytest.mark.parametrize("variant", ["qwen3_0p6b_bs64", "qwen3_0p6b_nozp"])
def test_layout_variants_one_launch(step_mod, cuda_dev, variant):
    cfg, lins, samples = build_model(step_mod, variant, 32)
    for M in [m for m in cfg["gemv_M"] if m <= 8]:
        p = step_mod.Pass(lins, M, "gemv", torch.float16, chain=True)
        _fill_inputs(p, cfg["seed"] + M, torch.float16)
        _run_graph(p)
        check_pass(cfg, lins, samples, p, "f16")


@pytest.mark.parametrize("variant", ["qwen3_0p6b_bs64", "qwen3_0p6b_nozp"])
def test_layout_variants(step_mod, cuda_dev, variant):
    # decode GEMVs: every output column of every projection; prefill GEMMs: 256
    # evenly spaced columns of every projection
    cfg, lins, samples = build_model(step_mod, variant, 0, all_rows=True)
    for M in cfg["gemv_M"]:
        p = step_mod.Pass(lins, M, "gemv", torch.float16)
        _fill_inputs(p, cfg["seed"] + M, torch.float16)
        _run_graph(p)
        check_pass(cfg, lins, samples, p, "f16")
        del p
    body = [l for l in lins if l.N != workloads.VOCAB]
    bsamp = [s for l, s in zip(lins, samples) if l.N != workloads.VOCAB]
    for M in cfg["gemm_M"]:
        p = step_mod.Pass(body, M, "gemm", torch.float16)
        _fill_inputs(p, cfg["seed"] + M, torch.float16)
        _run_graph(p)
        check_pass(cfg, body, bsamp, p, "f16", max_rows=256)
        del p


def test_embed_gather_full_table(cuda_dev):
    import int4_block_quantized_matmulnbits_b200 as mnb

    e = workloads.EMBED
    table, scales, ids = workloads.embed_inputs(e["seed"], e["V"], e["D"], e["T"])
    out = torch.empty((e["T"], e["D"]), dtype=torch.float16, device=cuda_dev)
    status = torch.zeros((1,), dtype=torch.int32, device=cuda_dev)
    mnb.mnb_embed_gather(table.to(cuda_dev), scales.to(cuda_dev), e["V"], e["D"], ids.to(cuda_dev), e["T"],
                         out, status)
    ref, st = oracle.embed_gather(table.numpy(), scales.numpy(), ids.numpy(), np.float16)
    assert np.array_equal(np_of(out).view(np.uint8), ref.view(np.uint8))
    assert int(status.item()) == st == 0
