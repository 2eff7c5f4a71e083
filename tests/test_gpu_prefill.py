"""GPU parity of attn_prefill (a chunk of new tokens against a KV cache) with the oracle.

Ragged cache lengths, chunk lengths that are not tile multiples, windows
inside and beyond the chunk, GQA, D = 64 and 128, with and without the
in-place append. Cache rows past each chunk hold NaN and must never reach the
output. The oracle runs on the exact bf16 q_hat / k_hat the GPU prologue
produced, so the check isolates the attention kernel.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import LSE_MAX_ABS, check_out, f64, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cswa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import causal_sliding_window_attn_b200 as m
    m.lib()
    assert m.lib().attn_device_supported() == 1, "not an sm_100 device"
    return m


def _inputs(cswa, B, T, Tmax, Hq, Hkv, D, pos, seed):
    g = torch.Generator().manual_seed(seed)
    kraw = torch.randn((B, Tmax, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn((B, Tmax, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    qraw = torch.randn((B, T, Hq, D), generator=g).to(torch.bfloat16).cuda()
    knraw = torch.randn((B, T, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn((B, T, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    _, kc = cswa.attn_rope_qknorm(None, kraw)
    posd = torch.tensor(pos, dtype=torch.int32).cuda()
    q, kn = cswa.attn_rope_qknorm(qraw, knraw, pos=posd)
    return q, kc, vc, kn, vn, posd


def _prefill_case(cswa, B, T, Tmax, Hq, Hkv, D, W, pos, seed, append=True, want_lse=True):
    q, kc, vc, kn, vn, posd = _inputs(cswa, B, T, Tmax, Hq, Hkv, D, pos, seed)
    # rows past each chunk hold NaN: they must never be read
    for b, p in enumerate(pos):
        kc[b, p + (0 if append else T):] = float("nan")
        vc[b, p + (0 if append else T):] = float("nan")
        if not append:
            kc[b, p:p + T] = kn[b]
            vc[b, p:p + T] = vn[b]
    kc_before, vc_before = kc.clone(), vc.clone()
    scale = workloads.default_scale(D)
    o, lse = cswa.attn_prefill(q, kc, vc, posd, W, k_new=kn if append else None, v_new=vn if append else None,
                               lse=None if want_lse else False)
    torch.cuda.synchronize()
    assert cswa.attn_get_status() == 0
    o_ref, lse_ref, _, _ = oracle.prefill(f64(q), np.nan_to_num(f64(kc_before)), np.nan_to_num(f64(vc_before)),
                                          np.array(pos), W, scale, k_new=f64(kn) if append else None,
                                          v_new=f64(vn) if append else None)
    check_out("prefill o", f64(o), o_ref)
    if want_lse:
        assert max_abs(f64(lse), lse_ref) <= LSE_MAX_ABS
    else:
        assert lse is None
    # the append is a byte copy, and nothing else in the caches changed
    mask = torch.ones(B, Tmax, dtype=torch.bool)
    for b, p in enumerate(pos):
        if append:
            assert torch.equal(kc[b, p:p + T], kn[b]) and torch.equal(vc[b, p:p + T], vn[b])
        mask[b, p:p + T] = False
    m = mask.cuda()
    assert torch.equal(kc[m].nan_to_num(7.0), kc_before[m].nan_to_num(7.0))
    assert torch.equal(vc[m].nan_to_num(7.0), vc_before[m].nan_to_num(7.0))
    return o, lse


CASES = [
    # B, T, Tmax, Hq, Hkv, D, window, pos
    (3, 300, 1100, 4, 2, 128, 300, [0, 129, 800]),     # ragged chunk, the last one ends at Tmax
    (2, 256, 1000, 2, 2, 128, -1, [5, 640]),           # full causal, chunk of two whole tiles
    (2, 200, 600, 2, 1, 128, 0, [0, 333]),             # self only
    (2, 385, 900, 4, 4, 128, 128, [1, 515]),           # one row past three tiles, window of one tile
    (2, 1, 300, 8, 2, 64, 100, [0, 77]),               # one-token chunk, G = 4, D = 64
    (1, 517, 2000, 6, 3, 64, 1023, [1483]),            # window shorter than the cache
    (2, 640, 640, 2, 1, 128, 2000, [0, 0]),            # window beyond every position: plain causal
    (2, 300, 70000, 4, 2, 128, -1, [69700, 40000]),    # long caches, full causal: ~545 key tiles
    (1, 200, 70000, 2, 1, 64, 8000, [65000]),          # long cache, window of 63 tiles
]


def _ids(c):
    return "B{}_T{}_Tmax{}_Hq{}_Hkv{}_D{}_W{}".format(*c[:7])


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_prefill_matches_oracle(cswa, case):
    B, T, Tmax, Hq, Hkv, D, W, pos = case
    _prefill_case(cswa, B, T, Tmax, Hq, Hkv, D, W, pos, seed=T + Tmax)


def test_prefill_without_append_and_lse(cswa):
    _prefill_case(cswa, 2, 300, 1200, 4, 2, 128, 400, [129, 900], seed=31, append=False, want_lse=False)


def test_prefill_chunks_equal_forward(cswa):
    """A sequence fed in chunks of 200, 1 and 499 tokens gives attn_fwd's rows."""
    B, T, Hq, Hkv, D, W = 2, 700, 4, 2, 128, 250
    q, k, v, _ = workloads.training_inputs(B, T, Hq, Hkv, D, seed=32)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    qh, kh = cswa.attn_rope_qknorm(q, k)
    o_full, lse_full = cswa.attn_fwd(qh, kh, v, W)
    kc = torch.full((B, T, Hkv, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = kc.clone()
    for c0, c1 in ((0, 200), (200, 201), (201, 700)):
        pos = torch.full((B,), c0, dtype=torch.int32, device="cuda")
        o, lse = cswa.attn_prefill(qh[:, c0:c1].contiguous(), kc, vc, pos, W, k_new=kh[:, c0:c1].contiguous(),
                                   v_new=v[:, c0:c1].contiguous())
        assert max_abs(f64(o), f64(o_full[:, c0:c1])) <= 1e-2
        assert max_abs(f64(lse), f64(lse_full[:, :, c0:c1])) <= 1e-3
    assert cswa.attn_get_status() == 0
    assert torch.equal(kc, kh) and torch.equal(vc, v)


def test_prefill_bad_position_is_reported(cswa):
    """pos[b] + T past the cache: that sequence is neither appended nor computed."""
    B, T, Tmax, H, D = 2, 40, 64, 2, 128
    q = torch.randn((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((B, Tmax, H, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kn = torch.ones((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    pos = torch.tensor([3, Tmax - T + 1], dtype=torch.int32, device="cuda")
    o = torch.full_like(q, 5.0)
    cswa.attn_prefill(q, kc, vc, pos, -1, k_new=kn, v_new=kn, o=o)
    assert cswa.attn_get_status() == 5  # ATTN_ERR_DEVICE
    assert torch.isfinite(o[0].float()).all() and not (o[0].float() == 5.0).all()
    assert (o[1].float() == 5.0).all()          # untouched
    assert (kc[1].float() == 0).all()           # not appended
    assert cswa.attn_get_status() == 0  # cleared
