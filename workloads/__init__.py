"""Seeded synthetic inputs and workload shapes for the MatMulNBits tests and benchmark.

This module holds no arithmetic of the method: it only draws random numbers
and names shapes.  Both the CPU oracle (via the tests) and the CUDA library
receive the tensors made here, so neither side computes its own inputs.

Shapes: the decoder linears of Qwen3-0.6B / Qwen3-1.7B-shaped ASR decoders
(28 layers, GQA with 8 KV heads of 128, SwiGLU MLP, a 151936-token vocabulary),
as described on "Qwen3-ASR-0.6B -- ONNX for the browser" ("Graph contracts")
and "Qwen3-ASR-1.7B ONNX" ("Architecture", "Shared").

Recipe (seeded, synthetic; no dataset, no trained weights):
  * weights    fp32 N(0, 0.02), one torch.Generator per (seed, layer, proj)
               seeded with seed * 1_000_003 + layer * 16 + proj
               (proj order q, k, v, o, gate, up, down; lm_head is layer 28,
               proj 0).  Optional outliers: each weight independently, with
               probability 0.01 drawn from the same generator, times 8.
  * activations N(0, 1), generator seed * 1_000_003 + 999 * 16 + tag.
  * embedding  int8 table uniform over [-128, 127], fp32 row scales
               U(0.001, 0.05), token ids uniform over [0, V) as int32.
"""
from __future__ import annotations

import dataclasses

import torch

PROJ_NAMES = ("q", "k", "v", "o", "gate", "up", "down")
N_LAYERS = 28
VOCAB = 151936


@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    layer: int
    proj: int
    N: int  # output features (weight rows)
    K: int  # input features


def decoder_linears(hidden: int, q_out: int, kv_out: int, inter: int,
                    lm_head: bool = True, layers: int = N_LAYERS):
    """The 7 projections of each layer (plus lm_head) as (N, K) weight shapes."""
    per_layer = [
        ("q", q_out, hidden), ("k", kv_out, hidden), ("v", kv_out, hidden),
        ("o", hidden, q_out), ("gate", inter, hidden), ("up", inter, hidden),
        ("down", hidden, inter),
    ]
    out = []
    for layer in range(layers):
        for p, (name, n, k) in enumerate(per_layer):
            out.append(Linear(name, layer, p, n, k))
    if lm_head:
        out.append(Linear("lm_head", N_LAYERS, 0, VOCAB, hidden))
    return out


def audio_encoder(layers=24, d=1024, ffn=4096):
    """A Whisper-style audio encoder's linears: per layer q, k, v, o (d -> d),
    fc1 (d -> ffn), fc2 (ffn -> d)."""
    per_layer = [("q", d, d), ("k", d, d), ("v", d, d), ("o", d, d), ("fc1", ffn, d), ("fc2", d, ffn)]
    return [Linear(name, layer, p, n, k) for layer in range(layers) for p, (name, n, k) in enumerate(per_layer)]


def qwen3_0p6b(lm_head=True, layers=N_LAYERS):
    """Qwen3-0.6B-shaped decoder: hidden 1024, q 2048, kv 1024, MLP 3072."""
    return decoder_linears(1024, 2048, 1024, 3072, lm_head, layers)


def qwen3_1p7b(lm_head=True, layers=N_LAYERS):
    """Qwen3-1.7B-shaped decoder: hidden 2048, q 2048, kv 1024, MLP 6144."""
    return decoder_linears(2048, 2048, 1024, 6144, lm_head, layers)


# The five workloads, and three more shapes of the same decoders.  'gemv_M'
# lists go to the decode kernel, 'gemm_M' to the tensor-core kernel, 'matmul_M'
# to mnb_matmul (which picks one).
CONFIGS = {
    "single_gemv": dict(desc="single GEMV M=1 K=1024 N=2048 bs32 zp, fp32 activations",
                        seed=0, bs=32, has_zp=True, act="f32", scale="f32",
                        linears=[Linear("single", 0, 0, 2048, 1024)], gemv_M=[1], gemm_M=[]),
    "qwen3_0p6b_decode": dict(desc="Qwen3-0.6B-shaped decode step, fp16, bs32 zp",
                              seed=1, bs=32, has_zp=True, act="f16", scale="f16",
                              model="0.6b", gemv_M=[1], gemm_M=[]),
    "qwen3_1p7b_decode": dict(desc="Qwen3-1.7B-shaped decode step, fp16, bs32 zp, 1% outliers x8",
                              seed=2, bs=32, has_zp=True, act="f16", scale="f16", outliers=True,
                              model="1.7b", gemv_M=[1, 2, 4, 8, 16], gemm_M=[]),
    "qwen3_1p7b_prefill": dict(desc="Qwen3-1.7B-shaped prefill, fp16, bs32 zp, no lm_head",
                               seed=3, bs=32, has_zp=True, act="f16", scale="f16",
                               model="1.7b", lm_head=False, gemv_M=[], gemm_M=[64, 256, 420, 1024]),
    "qwen3_0p6b_bs64": dict(desc="Qwen3-0.6B shapes, block 64 with zero points",
                            seed=4, bs=64, has_zp=True, act="f16", scale="f16",
                            model="0.6b", gemv_M=[1, 4, 16], gemm_M=[64, 390]),
    "qwen3_0p6b_nozp": dict(desc="Qwen3-0.6B shapes, block 32 without zero points (zp = 8)",
                            seed=4, bs=32, has_zp=False, act="f16", scale="f16",
                            model="0.6b", gemv_M=[1, 4, 16], gemm_M=[64, 390]),
    # a prompt appended to a cached one: a few to a few dozen new tokens through
    # the 1.7B decoder's projections, between the decode and prefill regimes
    "qwen3_1p7b_cached_prefill": dict(desc="Qwen3-1.7B-shaped prefill of 17-63 new tokens, fp16, bs32 zp, no lm_head",
                                      seed=6, bs=32, has_zp=True, act="f16", scale="f16",
                                      model="1.7b", lm_head=False, gemv_M=[], gemm_M=[],
                                      matmul_M=[17, 20, 24, 32, 48, 63]),
    # the encoder's linears over one clip's audio tokens: 42 for a 3.2 s command,
    # 390 for a 30 s clip (the audio-token count of "Building the prompt", step 2)
    "audio_encoder_prefill": dict(desc="24-layer Whisper-style audio encoder linears (d 1024, FFN 4096), fp16, bs32 zp",
                                  seed=5, bs=32, has_zp=True, act="f16", scale="f16",
                                  model="encoder", lm_head=False, gemv_M=[], gemm_M=[42, 390]),
}

EMBED = dict(seed=4, V=VOCAB, D=1024, T=4096)


def config_linears(name: str):
    c = CONFIGS[name]
    if "linears" in c:
        return list(c["linears"])
    if c["model"] == "encoder":
        return audio_encoder()
    f = qwen3_0p6b if c["model"] == "0.6b" else qwen3_1p7b
    return f(lm_head=c.get("lm_head", True))


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def weight(seed: int, layer: int, proj: int, N: int, K: int, outliers: bool = False,
           device="cpu") -> torch.Tensor:
    """fp32 [N, K] ~ N(0, 0.02), optionally with 1% of entries times 8."""
    g = _gen(seed * 1_000_003 + layer * 16 + proj, device)
    w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * 0.02
    if outliers:
        mask = torch.rand((N, K), generator=g, device=device) < 0.01
        w = torch.where(mask, w * 8.0, w)
    return w


def activations(seed: int, M: int, K: int, dtype=torch.float16, tag: int = 0,
                device="cpu") -> torch.Tensor:
    """X [M, K] ~ N(0, 1) in the activation dtype."""
    g = _gen(seed * 1_000_003 + 999 * 16 + tag, device)
    return torch.randn((M, K), generator=g, device=device, dtype=torch.float32).to(dtype)


def embed_inputs(seed: int, V: int, D: int, T: int, device="cpu"):
    """(int8 table [V, D], fp32 row scales [V], int32 ids [T])."""
    g = _gen(seed * 1_000_003 + 777, device)
    table = torch.randint(-128, 128, (V, D), generator=g, device=device, dtype=torch.int32).to(torch.int8)
    scales = (torch.rand((V,), generator=g, device=device, dtype=torch.float32) * (0.05 - 0.001) + 0.001)
    ids = torch.randint(0, V, (T,), generator=g, device=device, dtype=torch.int32)
    return table, scales, ids
