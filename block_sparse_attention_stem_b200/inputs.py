"""Seeded synthetic inputs shaped like a Qwen3-8B long-context prefill layer.

This module only draws random numbers and rounds them to the input encodings
(bf16, or fp8 e4m3 with a per-head fp32 scale).  It holds none of the method's
arithmetic, so the CUDA library's tests and the fp64 oracle can both consume
exactly the same bytes.

Workloads (head_dim 128, 128-token blocks, stride 8 unless stated):

* ``tiny``       1 sequence of 2048 tokens, 2 Q / 2 KV heads, rho 0.5, mu 0.7,
                 beta 0.2, 1 sink block, 1 window block, seed 0.
* ``qwen32k``    1 x 32768 tokens, 32 Q / 8 KV heads (GQA 4:1), rho 0.25,
                 mu 0.7, 4 sink / 4 window blocks, first 4 keys pushed +3 sigma
                 along the mean-query direction of their KV group, seed 1.
* ``long128k``   as qwen32k at 131072 tokens, 1 sink / 2 window blocks, seed 2.
* ``sweep64k``   1 x 65536 tokens, 32 / 8 heads, mu 1.0, rho swept, seed 3.
* ``fp8_varlen`` 4 packed sequences {8192, 16384, 40960, 98304}, e4m3 with
                 per-head scale amax/448 of N(0,1) data (Q, K and V alike; no
                 value-norm scaling), rho 0.25, 36 layers with mu 1.0 for
                 layers 0-4 and 0.7 after, seed 4000 + layer.

Value rows are N(0,1) vectors scaled by exp(z), z ~ N(0, sigma^2), so their
norms are log-normal with sigma = ``v_norm_sigma`` (0.5; 0 leaves V at
N(0,1)).  Q and K entries are N(0,1).

``structure="topics"`` (used by the reconstruction-quality measurement) adds,
after the draws above, a block-level topic structure under which attention is
concentrated rather than near uniform: per KV head, 16 random unit topic
directions; every 128-token block gets one topic per KV head; Q rows (of the
group's query heads) and K rows get that direction times a, with
a^2 / sqrt(d) = 6, so a key of the query's topic scores about +6 higher; and
the V rows of each (KV head, block) are scaled by exp(0.8 z), z ~ N(0, 1), so
blocks differ in value magnitude.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

E4M3_MAX = 448.0


@dataclass
class Workload:
    name: str
    seqlens: list
    num_q_heads: int
    num_kv_heads: int
    head_dim: int = 128
    dtype: str = "bf16"  # "bf16" or "fp8"
    seed: int = 0
    sink_boost: bool = False
    v_norm_sigma: float = 0.5  # log-normal value-row norms; 0: plain N(0,1) rows
    # method parameters (values only)
    keep_ratio: float = 0.25
    mu: float = 0.7
    beta: float = 0.2
    sink_blocks: int = 4
    window_blocks: int = 4
    block_size: int = 128
    stride: int = 8
    chunk_size: int = 2048
    norm: float = 1.0
    softmax_scale: float = 0.0
    budget_mode: int = 0
    bonus_mode: int = 0
    list_mode: int = 0
    structure: str = "iid"  # "iid", or "topics" (block-level topic structure, see the module docstring)

    def params(self) -> dict:
        return dict(block_size=self.block_size, stride=self.stride, chunk_size=self.chunk_size,
                    norm=self.norm, beta=self.beta, keep_ratio=self.keep_ratio, mu=self.mu,
                    sink_blocks=self.sink_blocks, window_blocks=self.window_blocks,
                    softmax_scale=self.softmax_scale, budget_mode=self.budget_mode, bonus_mode=self.bonus_mode,
                    list_mode=self.list_mode)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    def cu_seqlens(self) -> list:
        out = [0]
        for L in self.seqlens:
            out.append(out[-1] + int(L))
        return out


def workload(name: str, **overrides) -> Workload:
    base = {
        "tiny": dict(seqlens=[2048], num_q_heads=2, num_kv_heads=2, seed=0, keep_ratio=0.5,
                     mu=0.7, beta=0.2, sink_blocks=1, window_blocks=1),
        "qwen32k": dict(seqlens=[32768], num_q_heads=32, num_kv_heads=8, seed=1, sink_boost=True,
                        keep_ratio=0.25, mu=0.7, sink_blocks=4, window_blocks=4),
        "long128k": dict(seqlens=[131072], num_q_heads=32, num_kv_heads=8, seed=2, sink_boost=True,
                         keep_ratio=0.25, mu=0.7, sink_blocks=1, window_blocks=2),
        "sweep64k": dict(seqlens=[65536], num_q_heads=32, num_kv_heads=8, seed=3, keep_ratio=0.25,
                         mu=1.0, sink_blocks=4, window_blocks=4),
        "fp8_varlen": dict(seqlens=[8192, 16384, 40960, 98304], num_q_heads=32, num_kv_heads=8,
                           dtype="fp8", seed=4000, keep_ratio=0.25, mu=0.7, sink_blocks=4,
                           window_blocks=4, v_norm_sigma=0.0),
    }[name]
    base.update(overrides)
    return Workload(name=name, **base)


def fp8_layer_mu(layer: int) -> float:
    """Per-layer decay schedule of the fp8 stack: 1.0 for 5 warm-up layers, then 0.7."""
    return 1.0 if layer < 5 else 0.7


def _draw(w: Workload, gen: torch.Generator):
    T, hq, hkv, d = w.total_tokens, w.num_q_heads, w.num_kv_heads, w.head_dim
    dev = gen.device
    q = torch.randn(T, hq, d, generator=gen, dtype=torch.float32, device=dev)
    k = torch.randn(T, hkv, d, generator=gen, dtype=torch.float32, device=dev)
    v = torch.randn(T, hkv, d, generator=gen, dtype=torch.float32, device=dev)
    if w.v_norm_sigma > 0:
        v *= torch.exp(w.v_norm_sigma * torch.randn(T, hkv, 1, generator=gen, dtype=torch.float32, device=dev))
    if w.sink_boost:
        G = hq // hkv
        cu = w.cu_seqlens()
        for s in range(len(w.seqlens)):
            o, e = cu[s], cu[s + 1]
            qm = q[o:e].reshape(e - o, hkv, G, d).mean(dim=(0, 2))  # [hkv, d]
            u = qm / qm.norm(dim=1, keepdim=True)
            n = min(4, e - o)
            k[o:o + n] += 3.0 * u[None]
    if w.structure == "topics":
        _add_topics(w, q, k, v, gen)
    return q, k, v


def _add_topics(w: Workload, q, k, v, gen: torch.Generator, ntopics: int = 16, logit_gap: float = 6.0):
    T, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    dev = gen.device
    a = (logit_gap * d ** 0.5) ** 0.5
    cu = w.cu_seqlens()
    for s in range(len(w.seqlens)):
        o, e = cu[s], cu[s + 1]
        L = e - o
        if L <= 0:
            continue
        nb = (L + 127) // 128
        dirs = torch.randn(hkv, ntopics, d, generator=gen, dtype=torch.float32, device=dev)
        dirs /= dirs.norm(dim=2, keepdim=True)
        topic = torch.randint(0, ntopics, (hkv, nb), generator=gen, device=dev)
        vscale = torch.exp(0.8 * torch.randn(hkv, nb, generator=gen, dtype=torch.float32, device=dev))
        blk = torch.arange(L, device=dev) // 128  # block of each token
        for hk in range(hkv):
            t_dir = dirs[hk][topic[hk][blk]]  # [L, d]
            k[o:e, hk] += a * t_dir
            q[o:e, hk * G:(hk + 1) * G] += a * t_dir[:, None, :]
            v[o:e, hk] *= vscale[hk][blk][:, None]


def _to_fp8(x: torch.Tensor):
    """Per-head scale = amax/448, values rounded to e4m3 (returned as uint8 bytes)."""
    amax = x.abs().amax(dim=(0, 2)).clamp_min(1e-12)
    scale = (amax / E4M3_MAX).to(torch.float32)
    x8 = (x / scale[None, :, None]).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return x8.view(torch.uint8), scale


def make_inputs(w: Workload, seed: int | None = None, device: str = "cpu") -> dict:
    """q [T,Hq,d], k/v [T,Hkv,d] as bf16 (or uint8 e4m3 bytes with fp32
    per-head scales q_scale/k_scale/v_scale), plus cu_seqlens int32, drawn on
    `device` with that device's generator (the CPU stream is the reference one
    the tests use; a CUDA generator gives the same distributions faster)."""
    gen = torch.Generator(device).manual_seed(w.seed if seed is None else seed)
    q, k, v = _draw(w, gen)
    out = dict(cu_seqlens=torch.tensor(w.cu_seqlens(), dtype=torch.int32, device=device))
    if w.dtype == "bf16":
        out.update(q=q.to(torch.bfloat16), k=k.to(torch.bfloat16), v=v.to(torch.bfloat16),
                   q_scale=None, k_scale=None, v_scale=None)
    elif w.dtype == "fp8":
        q8, qs = _to_fp8(q)
        k8, ks = _to_fp8(k)
        v8, vs = _to_fp8(v)
        out.update(q=q8, k=k8, v=v8, q_scale=qs, k_scale=ks, v_scale=vs)
    else:
        raise ValueError(w.dtype)
    return out


def raw_bits(t: torch.Tensor):
    """numpy view of the raw encoding: uint16 for bf16, uint8 for e4m3 bytes."""
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).numpy().view("uint16")
    if t.dtype == torch.uint8:
        return t.contiguous().numpy()
    raise TypeError(t.dtype)
