"""Seeded synthetic inputs for the attention block: shapes, seeds and generators only.

Both the CUDA path's tests/bench and the fp64 oracle's tests draw their inputs
here, so that both sides see the same bytes. This module does none of the
block's arithmetic: it draws N(0, 1) fp32 numbers from a seeded CPU generator
and rounds them to bf16.

The shapes follow the nanochat d20 model (head_dim 128, 2048-token context,
"SSSL" short/long layers; nanochat User Guide, 4 "The One Dial You Control" and
13 "base_train full flag list"), a GQA variant, a long-context variant, a
KV-cache decode batch and a chunked-prefill batch over ragged cache lengths.
The pages train on text corpora; these synthetic tensors stand in for the
activations that reach the attention block.
"""
import math

import torch

ROPE_BASE = 10000.0
EPS = 1e-6

CONFIGS = {
    # name: B, T, Hq, Hkv, D, windows (one entry per layer), seed
    "tiny": dict(B=1, T=256, Hq=4, Hkv=2, D=64, windows=(128,), seed=0),
    "d20": dict(B=8, T=2048, Hq=10, Hkv=10, D=128, windows=(1024, 2048), seed=1),
    "gqa": dict(B=8, T=2048, Hq=16, Hkv=4, D=128, windows=(512,), seed=2),
    "long": dict(B=2, T=8192, Hq=16, Hkv=8, D=128, windows=(2048, -1), seed=3),
}

DECODE = dict(B=32, Hq=10, Hkv=10, D=128, Tmax=2176, window=1024,
              len_lo=512, len_hi=2048, seed=4)

# chunked prefill: a 512-token chunk per sequence on top of cache lengths U[0, 1536]
PREFILL = dict(B=8, Hq=10, Hkv=10, D=128, T=512, Tmax=2048, window=1024,
               len_lo=0, len_hi=1536, seed=5)


def default_scale(D):
    return 1.0 / math.sqrt(D)


def training_inputs(B, T, Hq, Hkv, D, seed):
    """q, k, v, dO as bf16 CPU tensors in BTHD layout, drawn in that order."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn((B, T, Hq, D), generator=g, dtype=torch.float32)
    k = torch.randn((B, T, Hkv, D), generator=g, dtype=torch.float32)
    v = torch.randn((B, T, Hkv, D), generator=g, dtype=torch.float32)
    do = torch.randn((B, T, Hq, D), generator=g, dtype=torch.float32)
    return tuple(t.to(torch.bfloat16) for t in (q, k, v, do))


def config_inputs(name):
    c = CONFIGS[name]
    return training_inputs(c["B"], c["T"], c["Hq"], c["Hkv"], c["D"], c["seed"])


def decode_inputs(B, Hq, Hkv, D, Tmax, len_lo, len_hi, seed, **_):
    """Cache lengths and raw (pre-prologue) tensors for one decode step.

    Returns lengths int32 (B,), raw k cache (B, Tmax, Hkv, D), v cache,
    raw q (B, 1, Hq, D), raw k_new and v_new (B, 1, Hkv, D); all bf16.
    The k cache and the query still have to go through the prologue (at
    positions 0..Tmax-1 and at lengths[b] respectively) to become the
    "entries after RoPE + QK-norm" of the decode workload.
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    lengths = torch.randint(len_lo, len_hi + 1, (B,), generator=g, dtype=torch.int64)
    kc = torch.randn((B, Tmax, Hkv, D), generator=g, dtype=torch.float32)
    vc = torch.randn((B, Tmax, Hkv, D), generator=g, dtype=torch.float32)
    q = torch.randn((B, 1, Hq, D), generator=g, dtype=torch.float32)
    kn = torch.randn((B, 1, Hkv, D), generator=g, dtype=torch.float32)
    vn = torch.randn((B, 1, Hkv, D), generator=g, dtype=torch.float32)
    bf = torch.bfloat16
    return (lengths.to(torch.int32), kc.to(bf), vc.to(bf), q.to(bf), kn.to(bf), vn.to(bf))


def prefill_inputs(B, Hq, Hkv, D, T, Tmax, len_lo, len_hi, seed, **_):
    """Cache lengths and raw (pre-prologue) tensors for one chunked-prefill step.

    Returns lengths int32 (B,), raw k cache (B, Tmax, Hkv, D), v cache, raw q
    (B, T, Hq, D), raw k_new and v_new (B, T, Hkv, D); all bf16. The k cache goes
    through the prologue at positions 0..Tmax-1; q and k_new at lengths[b] + t.
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    lengths = torch.randint(len_lo, len_hi + 1, (B,), generator=g, dtype=torch.int64)
    kc = torch.randn((B, Tmax, Hkv, D), generator=g, dtype=torch.float32)
    vc = torch.randn((B, Tmax, Hkv, D), generator=g, dtype=torch.float32)
    q = torch.randn((B, T, Hq, D), generator=g, dtype=torch.float32)
    kn = torch.randn((B, T, Hkv, D), generator=g, dtype=torch.float32)
    vn = torch.randn((B, T, Hkv, D), generator=g, dtype=torch.float32)
    bf = torch.bfloat16
    return (lengths.to(torch.int32), kc.to(bf), vc.to(bf), q.to(bf), kn.to(bf), vn.to(bf))


def prefill_pairs(lengths, T, window):
    """Visible (query, key) pairs of one head over a prefill chunk: row t of
    sequence b sits at position lengths[b] + t and sees min(position, W) + 1 keys."""
    n = 0
    for L in lengths:
        for t in range(T):
            p = L + t
            n += (p if window < 0 else min(p, window)) + 1
    return n


def visible_pairs(T, window):
    """Visible (query, key) pairs of one head: sum over i of min(i, W) + 1."""
    if window < 0 or window >= T - 1:
        return T * (T + 1) // 2
    W = window
    # rows i <= W see i + 1 keys; rows i > W see W + 1 keys
    return (W + 1) * (W + 2) // 2 + (T - W - 1) * (W + 1)
