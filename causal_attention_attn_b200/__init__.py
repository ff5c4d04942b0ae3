"""Fused causal scaled-dot-product attention for B200 (sm_100a).

The compute lives in ``libattn_b200.so`` (hand-written CUDA, C ABI declared in ``include/attn.h``).
``causal_attention_attn_b200.attn`` is the thin ctypes binding; importing this package does not
load the library, so the seeded-input module can be used on machines without the build.
"""

__version__ = "0.7.0"


def __getattr__(name):
    if name in ("attn_fwd", "attn_fwd_host", "attn_decode_paged", "attn_prefill_paged", "attn_bwd", "attn_decode_fp8",
                "attn_prefill_fp8",
                "attn_decode_paged_fp8", "attn_lse_merge", "AttnError", "library_path", "load_library"):
        from . import attn as _attn

        return getattr(_attn, name)
    raise AttributeError(name)
