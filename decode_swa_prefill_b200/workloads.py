"""Seeded synthetic workloads: shapes and input generators only.

This module holds no attention arithmetic.  It is the one piece shared by the
tests (CUDA path vs oracle) and the benchmark: every tensor is drawn on the CPU
from a seeded torch.Generator, i.i.d. N(0,1) in fp32, then rounded to the
workload dtype (round-to-nearest-even for bf16), so both sides see identical
values.

Shapes follow the models the pages name (TinyMistral-248M with W=32 and GQA
32/8; Mistral 7B with W=4096; Longformer with a symmetric W=512 window and a
few global tokens).  No weights or datasets are involved: the values are
random.
"""
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str              # "prefill" | "prefill_global" | "decode" | "prefill_chunk"
    B: int
    T: int                 # sequence length (prefill), ring size W (decode), chunk length (chunk)
    Hq: int
    Hkv: int
    d: int
    W: int
    dtype: torch.dtype
    seed: int
    g: int = 0             # global tokens per sequence (prefill_global)
    pos_lo: int = 0        # decode / chunk: positions drawn from [pos_lo, pos_hi)
    pos_hi: int = 0
    notes: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return self.d ** -0.5


TOY = Workload("toy_causal_T16_W4_d64_f32", "prefill", B=1, T=16, Hq=1, Hkv=1, d=64, W=4,
               dtype=torch.float32, seed=0)
TINYMISTRAL = Workload("tinymistral_prefill_B4_T2048_h32x8_d32_W32", "prefill", B=4, T=2048,
                       Hq=32, Hkv=8, d=32, W=32, dtype=torch.bfloat16, seed=1)
MISTRAL_PREFILL = Workload("mistral7b_prefill_B1_T32768_h32x8_d128_W4096", "prefill", B=1,
                           T=32768, Hq=32, Hkv=8, d=128, W=4096, dtype=torch.bfloat16, seed=2)
MISTRAL_DECODE = Workload("mistral7b_decode_B64_h32x8_d128_W4096", "decode", B=64, T=4096,
                          Hq=32, Hkv=8, d=128, W=4096, dtype=torch.bfloat16, seed=3,
                          pos_lo=4096, pos_hi=131072)
LONGFORMER = Workload("longformer_prefill_B8_T4096_h12_d64_W512_g16", "prefill_global", B=8,
                      T=4096, Hq=12, Hkv=12, d=64, W=512, dtype=torch.bfloat16, seed=4, g=16)

# serving-path continuation: a 4096-token chunk of each of 4 sequences whose
# earlier tokens are in full W=4096 rings (Mistral-7B shapes)
MISTRAL_CHUNK = Workload("mistral7b_chunk_B4_n4096_h32x8_d128_W4096", "prefill_chunk", B=4, T=4096,
                         Hq=32, Hkv=8, d=128, W=4096, dtype=torch.bfloat16, seed=5,
                         pos_lo=4096, pos_hi=131072)

ALL = [TOY, TINYMISTRAL, MISTRAL_PREFILL, MISTRAL_DECODE, LONGFORMER, MISTRAL_CHUNK]


def varlen_lengths(n, total, seed, min_len=1):
    """n sequence lengths summing to `total`, drawn from a seeded uniform
    split (each at least min_len)."""
    g = _gen(seed + 3000)
    cuts = torch.sort(torch.randperm(total - n * min_len + n - 1, generator=g)[:n - 1]).values
    edges = torch.cat([torch.tensor([-1]), cuts, torch.tensor([total - n * min_len + n - 1])])
    return [int(x) - 1 + min_len for x in (edges[1:] - edges[:-1])]


def _gen(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(seed)


def randn(shape, dtype, gen):
    """fp32 N(0,1) on CPU, then rounded to dtype."""
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(dtype)


def prefill_inputs(B, T, Hq, Hkv, d, dtype, seed):
    """q [B,T,Hq,d], k/v [B,T,Hkv,d] (CPU tensors)."""
    g = _gen(seed)
    q = randn((B, T, Hq, d), dtype, g)
    k = randn((B, T, Hkv, d), dtype, g)
    v = randn((B, T, Hkv, d), dtype, g)
    return q, k, v


def global_positions(B, T, g, seed):
    """[B,g] int32: g distinct positions per sequence, sorted ascending."""
    gen = _gen(seed + 1000)
    rows = [torch.sort(torch.randperm(T, generator=gen)[:g]).values for _ in range(B)]
    if g == 0:
        return torch.zeros((B, 0), dtype=torch.int32)
    return torch.stack(rows).to(torch.int32)


def decode_inputs(B, Hq, Hkv, d, W, dtype, seed, pos_lo, pos_hi):
    """q [B,Hq,d], rings k/v [B,Hkv,W,d], pos [B] int32 in [pos_lo, pos_hi),
    and the new token's k/v [B,1,Hkv,d] to append at pos before decoding."""
    g = _gen(seed)
    q = randn((B, Hq, d), dtype, g)
    kc = randn((B, Hkv, W, d), dtype, g)
    vc = randn((B, Hkv, W, d), dtype, g)
    k_new = randn((B, 1, Hkv, d), dtype, g)
    v_new = randn((B, 1, Hkv, d), dtype, g)
    pos = torch.randint(pos_lo, pos_hi, (B,), generator=g, dtype=torch.int64).to(torch.int32)
    return q, kc, vc, k_new, v_new, pos


def chunk_inputs(B, n, Hq, Hkv, d, W, dtype, seed):
    """A chunk q [B,n,Hq,d], k/v [B,n,Hkv,d] and rings k/v [B,Hkv,W,d] whose
    every slot is filled (slots a short sequence has not reached yet hold
    values too, which a correct reader ignores)."""
    g = _gen(seed)
    q = randn((B, n, Hq, d), dtype, g)
    k = randn((B, n, Hkv, d), dtype, g)
    v = randn((B, n, Hkv, d), dtype, g)
    kc = randn((B, Hkv, W, d), dtype, g)
    vc = randn((B, Hkv, W, d), dtype, g)
    return q, k, v, kc, vc


def make(w: Workload):
    """Inputs of a named workload as a dict of CPU tensors."""
    if w.kind == "prefill":
        q, k, v = prefill_inputs(w.B, w.T, w.Hq, w.Hkv, w.d, w.dtype, w.seed)
        return {"q": q, "k": k, "v": v}
    if w.kind == "prefill_global":
        q, k, v = prefill_inputs(w.B, w.T, w.Hq, w.Hkv, w.d, w.dtype, w.seed)
        return {"q": q, "k": k, "v": v, "global_idx": global_positions(w.B, w.T, w.g, w.seed)}
    if w.kind == "decode":
        q, kc, vc, kn, vn, pos = decode_inputs(w.B, w.Hq, w.Hkv, w.d, w.W, w.dtype, w.seed,
                                               w.pos_lo, w.pos_hi)
        return {"q": q, "k_cache": kc, "v_cache": vc, "k_new": kn, "v_new": vn, "pos": pos}
    if w.kind == "prefill_chunk":
        q, k, v, kc, vc = chunk_inputs(w.B, w.T, w.Hq, w.Hkv, w.d, w.W, w.dtype, w.seed)
        pos = torch.randint(w.pos_lo, w.pos_hi, (w.B,), generator=_gen(w.seed + 2000),
                            dtype=torch.int64).to(torch.int32)
        return {"q": q, "k": k, "v": v, "k_cache": kc, "v_cache": vc, "pos": pos}
    raise ValueError(w.kind)
