"""Seeded synthetic inputs and named workloads.

This module holds no attention arithmetic: it only draws random bf16 tensors from a seed, in a
fixed order, so that the CUDA path and the CPU oracle are fed the same bytes. Both sides import it;
nothing else is shared between them.

Recipe (every workload): a CPU ``torch.Generator`` seeded with the workload's seed draws fp32
N(0, 1) values for Q, then K, then V, each rounded to bf16 (round-to-nearest-even). The long-context
workload then draws, per (batch, kv head), ``round(1% * Skv)`` distinct key indices and multiplies
those K rows by 8 (exact in bf16), so that the running max of the online softmax jumps late in the
sweep. ``scale`` is ``1/sqrt(D)`` rounded to fp32.

The shapes follow the pages' own examples: a Llama-3-8B-like layer with 32 query heads sharing 8
key/value heads at head dim 128 ("05 · Tích vô hướng, Softmax và toán của Attention", §4), a 4096
token context for decode (same page, §3-§4), and a 512-token prompt followed by 256 new tokens for
the cached case ("Bộ 06 · Bên trong model", Q2).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Skv: int
    D: int
    causal: bool
    seed: int
    outlier_frac: float = 0.0  # fraction of K rows per (b, kv head) multiplied by outlier_gain
    outlier_gain: float = 8.0

    @property
    def scale(self) -> float:
        return float(torch.tensor(1.0 / math.sqrt(self.D), dtype=torch.float32))

    @property
    def offset(self) -> int:
        return self.Skv - self.Sq

    def visible_pairs_per_head(self) -> int:
        """Number of (query, key) pairs the mask leaves visible in one head."""
        if not self.causal:
            return self.Sq * self.Skv
        return self.Sq * self.offset + self.Sq * (self.Sq + 1) // 2

    def flops(self) -> int:
        """Algorithmic FLOPs: 2*D for the score and 2*D for the PV product per visible pair."""
        return 4 * self.D * self.B * self.Hq * self.visible_pairs_per_head()

    def io_bytes(self) -> int:
        """Bytes read/written once: Q, K, V, O in bf16 and LSE in fp32."""
        q = self.B * self.Hq * self.Sq * self.D * 2
        kv = 2 * self.B * self.Hkv * self.Skv * self.D * 2
        return q + kv + q + self.B * self.Hq * self.Sq * 4

    def kv_bytes(self) -> int:
        return 2 * self.B * self.Hkv * self.Skv * self.D * 2

    def config(self) -> dict:
        return {
            "workload": self.name, "B": self.B, "Hq": self.Hq, "Hkv": self.Hkv, "Sq": self.Sq,
            "Skv": self.Skv, "D": self.D, "causal": self.causal, "seed": self.seed,
            "outlier_frac": self.outlier_frac,
        }


# The five workloads, seed 1000 + index.
TINY_PREFILL = Workload("tiny_causal_prefill_b1_h2_s64_d32", 1, 2, 2, 64, 64, 32, True, 1000)
PREFILL_8B = Workload("causal_prefill_8b_layer_b1_hq32_hkv8_s4096_d128", 1, 32, 8, 4096, 4096, 128, True, 1001)
DECODE_GQA = Workload("gqa_decode_b16_hq32_hkv8_skv4096_d128", 16, 32, 8, 1, 4096, 128, True, 1002)
CHUNKED_PREFILL = Workload("chunked_prefill_b8_hq32_hkv8_sq256_skv768_d128", 8, 32, 8, 256, 768, 128, True, 1003)
LONG_PREFILL = Workload("long_causal_prefill_b1_hq32_hkv8_s32768_d128_outliers", 1, 32, 8, 32768, 32768, 128, True,
                        1004, outlier_frac=0.01)

WORKLOADS = {w.name: w for w in (TINY_PREFILL, PREFILL_8B, DECODE_GQA, CHUNKED_PREFILL, LONG_PREFILL)}
SHORT_NAMES = {"tiny": TINY_PREFILL, "prefill": PREFILL_8B, "decode": DECODE_GQA,
               "chunked": CHUNKED_PREFILL, "long": LONG_PREFILL}


def custom(B, Hq, Hkv, Sq, Skv, D, causal=True, seed=0, outlier_frac=0.0, name=None) -> Workload:
    name = name or f"custom_b{B}_hq{Hq}_hkv{Hkv}_sq{Sq}_skv{Skv}_d{D}_{'c' if causal else 'nc'}"
    return Workload(name, B, Hq, Hkv, Sq, Skv, D, causal, seed, outlier_frac)


def generate(w: Workload):
    """Return host (CPU) bf16 tensors q [B,Hq,Sq,D], k and v [B,Hkv,Skv,D] for workload ``w``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    q = torch.randn((w.B, w.Hq, w.Sq, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((w.B, w.Hkv, w.Skv, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn((w.B, w.Hkv, w.Skv, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    if w.outlier_frac > 0.0:
        n_out = int(round(w.outlier_frac * w.Skv))
        gain = torch.tensor(w.outlier_gain, dtype=torch.bfloat16)
        for b in range(w.B):
            for h in range(w.Hkv):
                idx = torch.randperm(w.Skv, generator=g)[:n_out]
                k[b, h, idx, :] = k[b, h, idx, :] * gain
    return q, k, v


def generate_fp8(w: Workload):
    """An e4m3 K/V cache for workload ``w``: ``(q, k8, v8, k_scale, v_scale)``.

    q is drawn as by :func:`generate` (the same bytes); k and v too, then each (kv head, channel)
    gets the coefficient max|x| / 448 over every batch entry and key (1 where that is 0), and the
    codes are x / coefficient converted to e4m3 by torch (round to nearest even). k8, v8: uint8
    [B, Hkv, Skv, D]; k_scale, v_scale: fp32 [Hkv, D]. This is input preparation for a quantised
    cache, not part of the attention it feeds.
    """
    q, k, v = generate(w)

    def quantise(x):
        amax = x.float().abs().amax(dim=(0, 2))  # [Hkv, D]
        coef = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax)).to(torch.float32)
        codes = (x.float() / coef[None, :, None, :]).to(torch.float8_e4m3fn).view(torch.uint8)
        return codes.contiguous(), coef.contiguous()

    k8, k_scale = quantise(k)
    v8, v_scale = quantise(v)
    return q, k8, v8, k_scale, v_scale


def sample_rows(w: Workload, every: int = 64, seed: int = 7) -> torch.Tensor:
    """Deterministic sample of flat row ids ``(b*Hq + h)*Sq + i`` covering every (b, h):
    every ``every``-th row plus the first row, the row at the cache offset and the last row."""
    rows = []
    for b in range(w.B):
        for h in range(w.Hq):
            base = (b * w.Hq + h) * w.Sq
            picks = set(range(0, w.Sq, every)) | {0, w.Sq - 1, min(max(w.offset, 0), w.Sq - 1)}
            rows.extend(base + i for i in sorted(picks))
    return torch.tensor(rows, dtype=torch.int64)


def paged_cache(k: torch.Tensor, v: torch.Tensor, lens, page_size: int, seed: int):
    """Scatter each sequence's first lens[b] rows of a dense cache k, v [B, Hkv, cap, D] into pages
    of `page_size` slots in a seeded random order: ``(k_pages, v_pages, block_table)`` with pages
    [num_pages, Hkv, page_size, D] (unused slots zero) and an int32 table [B, ceil(cap / page_size)]
    whose unused entries point past the last page. Layout preparation for a paged cache only."""
    B, Hkv, cap, D = k.shape
    per_seq = -(-cap // page_size)
    num_pages = B * per_seq
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(seed))
    table = torch.full((B, per_seq), num_pages, dtype=torch.int32)
    kp = torch.zeros((num_pages, Hkv, page_size, D), dtype=k.dtype)
    vp = torch.zeros_like(kp)
    nxt = 0
    for b in range(B):
        for n in range(-(-min(int(lens[b]), cap) // page_size)):
            pg = int(perm[nxt])
            nxt += 1
            table[b, n] = pg
            lo, hi = n * page_size, min((n + 1) * page_size, int(lens[b]))
            kp[pg, :, :hi - lo] = k[b, :, lo:hi]
            vp[pg, :, :hi - lo] = v[b, :, lo:hi]
    return kp, vp, table


# Chunked prefill over a paged cache with per-sequence lengths: the chunked-prefill shape (8
# sequences, 256 new tokens each, 32 query / 8 kv heads, D 128) with cache lengths drawn uniformly
# from [256, 1024] (seed 1005), in pages of 64 keys.
PAGED_CHUNKED = Workload("paged_chunked_prefill_b8_hq32_hkv8_sq256_skv256to1024_page64", 8, 32, 8, 256, 1024, 128,
                         True, 1005)
PAGED_CHUNKED_PAGE = 64


def paged_chunked_lengths():
    g = torch.Generator().manual_seed(PAGED_CHUNKED.seed)
    return [int(x) for x in torch.randint(256, 1025, (PAGED_CHUNKED.B,), generator=g)]


def paged_visible_pairs(Sq: int, lens, causal: bool = True) -> int:
    """Visible (query, key) pairs per head summed over sequences: Sq new queries over len_b keys."""
    total = 0
    for L in lens:
        if not causal:
            total += Sq * L
            continue
        off = L - Sq
        if off >= 0:
            total += Sq * off + Sq * (Sq + 1) // 2
        else:  # rows i < -off see no key
            n = L
            total += n * (n + 1) // 2
    return total
