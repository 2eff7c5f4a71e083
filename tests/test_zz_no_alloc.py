"""attn_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers of this library cannot hand it a workspace -- code inside a
framework whose allocator it cannot reach, a serving loop that must not
allocate once started, or a host program that links only the C ABI. For them
attn_decode_noalloc keeps the split-K partials in a fixed 4 MiB scratch array
that the library holds in device memory. These checks call it through the C
ABI and compare it with attn_decode (which takes a workspace) on two calls in
a row, the second with different inputs so the reused scratch still holds the
first call's partials. This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import workloads
from tests.parity import LSE_MAX_ABS, check_out, f64, max_abs

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 4 * 1024 * 1024
INVALID_ARG = 1


def _inputs(cswa, B, Tmax, Hq, Hkv, D, pos, seed):
    g = torch.Generator().manual_seed(seed)
    kraw = torch.randn((B, Tmax, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn((B, Tmax, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    qraw = torch.randn((B, 1, Hq, D), generator=g).to(torch.bfloat16).cuda()
    knraw = torch.randn((B, 1, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn((B, 1, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    posd = torch.tensor(pos, dtype=torch.int32).cuda()
    _, kc = cswa.attn_rope_qknorm(None, kraw)
    q, kn = cswa.attn_rope_qknorm(qraw, knraw, pos=posd)
    return q, kc, vc, kn, vn, posd


def _noalloc(L, q, kc, vc, kn, vn, posd, o, lse, Tmax, Hkv, W, scale):
    B, _, Hq, D = q.shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return L.attn_decode_noalloc(p(q), p(kc), p(vc), p(kn), p(vn), p(posd), p(o), p(lse), B, Tmax, Hq, Hkv, D, W,
                                 ctypes.c_float(scale), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_decode_matches_workspace_decode():
    import causal_sliding_window_attn_b200 as cswa
    L = cswa.lib()
    B, Tmax, Hq, Hkv, D, W = 6, 700, 8, 2, 128, 300
    scale = workloads.default_scale(D)
    for call, (pos, seed) in enumerate((([0, 150, 699, 37, 400, 301], 31), ([650, 5, 299, 300, 1, 512], 32))):
        q, kc, vc, kn, vn, posd = _inputs(cswa, B, Tmax, Hq, Hkv, D, pos, seed)
        kc2, vc2 = kc.clone(), vc.clone()
        o_ref, lse_ref = cswa.attn_decode(q, kc, vc, posd, W, scale, k_new=kn, v_new=vn)
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        assert _noalloc(L, q, kc2, vc2, kn, vn, posd, o, lse, Tmax, Hkv, W, scale) == 0
        torch.cuda.synchronize()
        assert cswa.attn_get_status() == 0
        check_out(f"o (call {call})", f64(o), f64(o_ref))
        assert max_abs(f64(lse), f64(lse_ref)) <= LSE_MAX_ABS
        assert torch.equal(kc2, kc) and torch.equal(vc2, vc)   # same in-place append


def test_noalloc_decode_rejects_calls_beyond_its_scratch():
    import causal_sliding_window_attn_b200 as cswa
    L = cswa.lib()
    B, Tmax, Hq, Hkv, D, W = 64, 1100, 16, 16, 128, 1024    # 64*16*9*130*4 bytes > 4 MiB
    assert cswa.attn_decode_workspace_bytes(B, Hq, D, Tmax, W) > SCRATCH_BYTES
    q = torch.zeros((B, 1, Hq, D), dtype=torch.bfloat16).cuda()
    kc = torch.zeros((B, Tmax, Hkv, D), dtype=torch.bfloat16).cuda()
    posd = torch.zeros(B, dtype=torch.int32).cuda()
    o = torch.full_like(q, 7.0)
    lse = torch.full((B, Hq), 7.0).cuda()
    assert _noalloc(L, q, kc, kc, kc[:, :1].contiguous(), kc[:, :1].contiguous(), posd, o, lse, Tmax, Hkv, W,
                    0.1) == INVALID_ARG
    torch.cuda.synchronize()
    assert bool((o.float() == 7.0).all()) and bool((lse == 7.0).all())   # nothing was enqueued
