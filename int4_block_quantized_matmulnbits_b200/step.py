"""Quantized linears and the decoder-shaped passes that chain them.

The decoders of "Mega-ASR -- INT4 ONNX (GPTQ-calibrated)" and "Qwen3-ASR-0.6B
-- ONNX for the browser" spend ~95% of their work in MatMulNBits
("Compression vs original"): per token, 28 layers x 7 projections plus the
lm_head (decoder_step), and the same projections over all prompt tokens in
decoder_init / decoder_prefill.  These classes hold the packed weights in HBM
and issue the library calls of one such pass; every call is one CUDA kernel
of libmnb, optionally captured into a CUDA graph.
"""
from __future__ import annotations

import torch

from . import (MNB_FLAG_PDL, mnb_dequantize, mnb_embed_gather, mnb_gemm, mnb_gemv, mnb_gemv_argmax,
               mnb_gemv_argmax_workspace_bytes, mnb_gemv_chain, mnb_gemv_chain_plan, mnb_gemv_chain_workspace_bytes,
               mnb_gemv_swiglu, mnb_matmul, mnb_packed_sizes, mnb_quantize_rtn)


class QLinear:
    """One MatMulNBits weight [N, K]: packed uint8 [N, K/2], scales [N, K/bs], zp or None."""

    def __init__(self, N, K, bs, has_zp=True, scale_dtype=torch.float16, device="cuda", name=""):
        self.N, self.K, self.bs, self.has_zp, self.name = N, K, bs, has_zp, name
        pb, sb, zb = mnb_packed_sizes(N, K, bs, scale_dtype, has_zp)
        self.packed = torch.empty((N, K // 2), dtype=torch.uint8, device=device)
        self.scales = torch.empty((N, K // bs), dtype=scale_dtype, device=device)
        self.zp = torch.empty((N, (K // bs + 1) // 2), dtype=torch.uint8, device=device) if has_zp else None
        self.nbytes = pb + sb + zb

    @classmethod
    def quantize(cls, W, bs, has_zp=True, scale_dtype=torch.float16, name="", stream=None):
        """RTN-quantize an fp32 [N, K] device tensor with mnb_quantize_rtn."""
        N, K = W.shape
        q = cls(N, K, bs, has_zp, scale_dtype, W.device, name)
        mnb_quantize_rtn(W.contiguous(), N, K, bs, has_zp, q.packed, q.scales, q.zp, stream)
        return q

    def dequantize(self, dtype=torch.float16, stream=None):
        out = torch.empty((self.N, self.K), dtype=dtype, device=self.packed.device)
        mnb_dequantize(self.packed, self.scales, self.zp, self.N, self.K, self.bs, out, stream)
        return out

    def gemv(self, X, Y, flags=0, stream=None):
        mnb_gemv(X, self.packed, self.scales, self.zp, Y, X.shape[0], self.N, self.K, self.bs, flags, stream)

    def gemv_swiglu(self, X, Y, flags=0, stream=None):
        mnb_gemv_swiglu(X, self.packed, self.scales, self.zp, Y, X.shape[0], self.N, self.K, self.bs, flags, stream)

    def gemv_argmax(self, X, Y, ids, max_out, workspace, flags=0, stream=None):
        mnb_gemv_argmax(X, self.packed, self.scales, self.zp, Y, X.shape[0], self.N, self.K, self.bs, ids, max_out,
                        workspace, flags, stream)

    def gemm(self, X, Y, flags=0, stream=None):
        mnb_gemm(X, self.packed, self.scales, self.zp, Y, X.shape[0], self.N, self.K, self.bs, flags, stream)

    def matmul(self, X, Y, flags=0, stream=None):
        mnb_matmul(X, self.packed, self.scales, self.zp, Y, X.shape[0], self.N, self.K, self.bs, flags, stream)


def concat_linears(parts, name=""):
    """One QLinear whose rows are the rows of `parts` in order.

    Projections that read the same input (q, k, v; gate, up) are one
    MatMulNBits over their row-concatenated weights: the packed rows, scales and
    zero points are per row, so concatenation changes no stored value, and the
    outputs come out concatenated in the same order."""
    K, bs, has_zp = parts[0].K, parts[0].bs, parts[0].has_zp
    assert all(p.K == K and p.bs == bs and p.has_zp == has_zp for p in parts)
    N = sum(p.N for p in parts)
    q = QLinear(N, K, bs, has_zp, parts[0].scales.dtype, parts[0].packed.device, name)
    torch.cat([p.packed for p in parts], dim=0, out=q.packed)
    torch.cat([p.scales for p in parts], dim=0, out=q.scales)
    if has_zp:
        torch.cat([p.zp for p in parts], dim=0, out=q.zp)
    q.parts = [(p.name, p.N) for p in parts]
    return q


def swiglu_interleave(gate, up, name=""):
    """One QLinear [2I, K] for mnb_gemv_swiglu: rows in groups of 16, the 8 gate
    rows 8j..8j+7 followed by the 8 up rows of the same outputs.  Every stored
    quantity is per row, so interleaving changes no stored value."""
    assert gate.N == up.N and gate.K == up.K and gate.bs == up.bs and gate.has_zp == up.has_zp
    assert gate.N % 8 == 0
    I = gate.N
    q = QLinear(2 * I, gate.K, gate.bs, gate.has_zp, gate.scales.dtype, gate.packed.device, name)

    def inter(a, b, out):
        g = a.reshape(I // 8, 8, *a.shape[1:])
        u = b.reshape(I // 8, 8, *b.shape[1:])
        out.copy_(torch.stack([g, u], dim=1).reshape(2 * I, *a.shape[1:]))

    inter(gate.packed, up.packed, q.packed)
    inter(gate.scales, up.scales, q.scales)
    if gate.has_zp:
        inter(gate.zp, up.zp, q.zp)
    q.swiglu = True   # a decode pass runs it through mnb_gemv_swiglu: N / 2 outputs
    return q


def fuse_decoder(linears, swiglu=False):
    """Per layer [q, k, v, o, gate, up, down] -> [qkv, o, gate_up, down]; others kept.
    swiglu=True stores gate/up interleaved for the fused SwiGLU epilogue."""
    out, i = [], 0
    while i < len(linears):
        names = [l.name.rstrip("0123456789") for l in linears[i:i + 7]]
        if names == ["q", "k", "v", "o", "gate", "up", "down"]:
            L = linears[i:i + 7]
            layer = L[0].name[1:]
            gu = swiglu_interleave(L[4], L[5], f"gate_up{layer}") if swiglu else \
                concat_linears(L[4:6], f"gate_up{layer}")
            out += [concat_linears(L[0:3], f"qkv{layer}"), L[3], gu, L[6]]
            i += 7
        else:
            out.append(linears[i])
            i += 1
    return out


class Pass:
    """A chain of MatMulNBits calls with one X / Y buffer pair per linear.

    kind = "gemv" (decode step, M <= 32), "gemm" (prefill) or "matmul" (any M:
    mnb_matmul picks the kernel).  With pdl=True each
    launch may overlap the tail of the previous one (weights stream early, X is
    read after the previous kernel completes).  An optional int8 embedding
    gather of M token ids runs first, as in a decode step.
    """

    def __init__(self, linears, M, kind="gemv", act_dtype=torch.float16, pdl=True, embed=None, greedy=False,
                 chain=False, waits=None):
        self.linears, self.M, self.kind, self.pdl = list(linears), M, kind, pdl
        dev = self.linears[0].packed.device
        # one flat buffer each for all inputs and all outputs (views per linear,
        # 16-byte aligned), so a step's inputs and outputs move in one copy each
        xs = [M * l.K for l in self.linears]
        ys = [M * (l.N // 2 if getattr(l, "swiglu", False) else l.N) for l in self.linears]
        self.x_flat = torch.zeros((sum(xs),), dtype=act_dtype, device=dev)
        self.y_flat = torch.zeros((sum(ys),), dtype=act_dtype, device=dev)
        self.X, self.Y = [], []
        ox = oy = 0
        for l, nx, ny in zip(self.linears, xs, ys):
            self.X.append(self.x_flat[ox:ox + nx].view(M, l.K))
            self.Y.append(self.y_flat[oy:oy + ny].view(M, ny // M))
            ox, oy = ox + nx, oy + ny
        for t in self.X + self.Y:
            assert t.data_ptr() % 16 == 0
        self.embed = embed   # (table, row_scales, ids[M], out[M, D]) or None
        self.graph = None
        # greedy=True: the last linear (the lm_head) also picks each token's id
        self.greedy = greedy and kind == "gemv"
        if self.greedy:
            self.ids = torch.zeros((M,), dtype=torch.int32, device=dev)
            self.max_out = torch.zeros((M,), dtype=torch.float32, device=dev)
            self.ws = torch.zeros((mnb_gemv_argmax_workspace_bytes(M),), dtype=torch.uint8, device=dev)
        # chain=True: all GEMVs in one persistent launch (mnb_gemv_chain).  waits[i]
        # = 1 makes linear i read its X only after linears 0..i-1 are complete
        # (default: every linear waits, the dependencies of separate launches)
        self.chain = None
        if chain:
            assert kind == "gemv" and not self.greedy
            assert not any(getattr(l, "swiglu", False) for l in self.linears)
            n = len(self.linears)
            waits = [1] * n if waits is None else list(waits)
            tasks = [(x, l.packed, l.scales, l.zp, y, l.N, l.K, w)
                     for l, x, y, w in zip(self.linears, self.X, self.Y, waits)]
            plan = mnb_gemv_chain_plan(tasks, M, self.linears[0].bs)
            self.chain = (plan, plan.to(dev),
                          torch.zeros((mnb_gemv_chain_workspace_bytes(n),), dtype=torch.uint8, device=dev))

    @property
    def weight_bytes(self):
        return sum(l.nbytes for l in self.linears)

    @property
    def flops(self):
        return sum(2 * self.M * l.N * l.K for l in self.linears)

    @property
    def launches(self):
        n = 1 if self.chain is not None else len(self.linears)
        return n + (1 if self.embed is not None else 0)

    def run(self, stream=None):
        if self.embed is not None:
            table, rs, ids, out = self.embed
            mnb_embed_gather(table, rs, table.shape[0], table.shape[1], ids, ids.shape[0], out,
                             None, stream)
        flags = MNB_FLAG_PDL if self.pdl else 0
        if self.chain is not None:
            mnb_gemv_chain(*self.chain, flags, stream)
            return
        last = len(self.linears) - 1
        for i, (l, x, y) in enumerate(zip(self.linears, self.X, self.Y)):
            if self.kind == "gemv":
                if self.greedy and i == last:
                    l.gemv_argmax(x, y, self.ids, self.max_out, self.ws, flags, stream)
                elif getattr(l, "swiglu", False):
                    l.gemv_swiglu(x, y, flags, stream)
                else:
                    l.gemv(x, y, flags, stream)
            elif self.kind == "matmul":
                l.matmul(x, y, flags, stream)
            else:
                l.gemm(x, y, flags, stream)

    def capture(self):
        """Capture run() into a CUDA graph (replayed with replay())."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run(s)          # warm-up outside the graph (first-use attribute setup)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            self.run(s)
        self.graph = g
        return g

    def replay(self):
        self.graph.replay()
