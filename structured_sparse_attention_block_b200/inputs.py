"""Seeded synthetic inputs for the CoWA workloads.

This module only draws random tensors and names workload sizes; it holds
none of the operator's arithmetic.  Tests hand host copies of the same
tensors to the CPU oracle, and the bench times the library on them.

Recipe: Q, K, V and dO are drawn N(0, 1) in fp32 from a generator seeded
with ``seed`` in the order Q, K, V, dO, then rounded to bf16.  Small
workloads draw on the CPU (``torch.Generator``) so every machine produces
the same bits; large ones draw on the device with a seeded CUDA generator,
chunk by chunk, to bound the fp32 temporaries.

Workloads stand in for the pages' settings (none needs a dataset): the 8K
associative-recall scale (d_model 512), a 14B-like model at 32K context, the
128K operator benchmark, and 128K decoding.  The window widths W are the
printed defaults ceil((Lk - N) / Hkv) for each shape.
"""
import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Lq: int
    Lk: int
    Hq: int
    Hkv: int
    d: int
    quad: tuple  # (S, N, G, W)
    kind: str    # "train" or "decode"

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 512, 512, 4, 2, 64, (16, 64, 0, 224), "train"),
    "recall8k": Workload("recall8k", 4, 8192, 8192, 8, 4, 64, (64, 1024, 0, 1792), "train"),
    "llm14b_32k": Workload("llm14b_32k", 1, 32768, 32768, 40, 8, 128, (128, 4096, 0, 3584), "train"),
    "op128k": Workload("op128k", 1, 131072, 131072, 32, 8, 128, (128, 8192, 0, 15360), "train"),
    "decode128k": Workload("decode128k", 16, 1, 131072, 32, 8, 128, (128, 8192, 0, 15360), "decode"),
}

_CPU_LIMIT = 1 << 24  # elements: draw on the CPU below this size


def _randn(shape, gen, device, dtype=torch.bfloat16):
    n = math.prod(shape)
    if gen.device.type == "cpu":
        return torch.randn(shape, generator=gen, dtype=torch.float32).to(dtype).to(device)
    out = torch.empty(n, dtype=dtype, device=device)
    chunk = 1 << 26
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        out[s:e] = torch.randn(e - s, generator=gen, dtype=torch.float32, device=device).to(dtype)
    return out.view(shape)


def generator(numel: int, device, seed: int) -> torch.Generator:
    dev = torch.device(device)
    if numel <= _CPU_LIMIT or dev.type != "cuda":
        g = torch.Generator(device="cpu")
    else:
        g = torch.Generator(device=dev)
    g.manual_seed(seed)
    return g


def training_inputs(B, Lq, Lk, Hq, Hkv, d, device="cuda", seed=0, with_dout=True):
    """(q, k, v, dout) bf16 in [B, L, H, d], N(0,1) before rounding."""
    total = B * (Lq * Hq * 2 + Lk * Hkv * 2) * d
    g = generator(total, device, seed)
    q = _randn((B, Lq, Hq, d), g, device)
    k = _randn((B, Lk, Hkv, d), g, device)
    v = _randn((B, Lk, Hkv, d), g, device)
    dout = _randn((B, Lq, Hq, d), g, device) if with_dout else None
    return q, k, v, dout


def decode_inputs(B, Lcap, Hq, Hkv, d, device="cuda", seed=0, seqlens=None):
    """(q [B,1,Hq,d], k_cache, v_cache [B,Lcap,Hkv,d], seqlens int32 [B])."""
    total = B * (Hq + 2 * Lcap * Hkv) * d
    g = generator(total, device, seed)
    q = _randn((B, 1, Hq, d), g, device)
    kc = _randn((B, Lcap, Hkv, d), g, device)
    vc = _randn((B, Lcap, Hkv, d), g, device)
    if seqlens is None:
        seqlens = [Lcap] * B
    sl = torch.tensor(seqlens, dtype=torch.int32, device=device)
    return q, kc, vc, sl


def workload_inputs(wl: Workload, device="cuda", seed=0):
    if wl.kind == "decode":
        return decode_inputs(wl.B, wl.Lk, wl.Hq, wl.Hkv, wl.d, device, seed)
    return training_inputs(wl.B, wl.Lq, wl.Lk, wl.Hq, wl.Hkv, wl.d, device, seed)


def bf16_bits(t: torch.Tensor):
    """Host numpy uint16 view of a bf16 tensor (the oracle's bf16 input form)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
