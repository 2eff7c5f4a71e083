"""The kernels' bounded waits: a wait that runs out is reported, and the GPU stays usable.

attn_debug_set_wait_limit shortens the limit of the pipeline waits (a tile copy, a
tensor-core product, another warp's results) to a few nanoseconds, so that ordinary
waits inside attn_fwd / attn_bwd / attn_prefill give up: nothing faults, traps or hangs.
A CTA that gives up still waits (with the default limit) for the copies and products it
issued itself, frees its tensor memory and exits. The test checks that
attn_get_status() reports ATTN_ERR_TIMEOUT, and that calls made afterwards with the
default limit are correct against the fp64 oracle, which they could not be if tensor
memory had been left allocated or copies left in flight.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import LSE_MAX_ABS, check_grad, check_out, f64, max_abs

pytestmark = pytest.mark.gpu

ATTN_ERR_TIMEOUT = 4


@pytest.fixture(scope="module")
def cswa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import causal_sliding_window_attn_b200 as m
    m.lib()
    return m


def test_short_wait_limit_is_reported_then_calls_recover(cswa):
    B, T, Hq, Hkv, D, W = 2, 1024, 4, 2, 128, 300
    scale = workloads.default_scale(D)
    q, k, v, do = (t.cuda() for t in workloads.training_inputs(B, T, Hq, Hkv, D, seed=41))
    assert cswa.attn_get_status() == 0
    try:
        cswa.attn_debug_set_wait_limit(1)  # 1 ns: any wait not met at its first try gives up
        cswa.attn_fwd(q, k, v, W, scale)
        assert cswa.attn_get_status() == ATTN_ERR_TIMEOUT
        o, lse = torch.zeros_like(q), torch.zeros((B, Hq, T), device="cuda")
        cswa.attn_bwd(q, k, v, o, do, lse, W, scale)
        assert cswa.attn_get_status() == ATTN_ERR_TIMEOUT
        pos = torch.tensor([100, 0], dtype=torch.int32, device="cuda")
        kc = torch.zeros((B, 2048, Hkv, D), dtype=torch.bfloat16, device="cuda")
        cswa.attn_prefill(q[:, :512].contiguous(), kc, kc.clone(), pos, W, scale, k_new=k[:, :512].contiguous(),
                          v_new=v[:, :512].contiguous())
        assert cswa.attn_get_status() == ATTN_ERR_TIMEOUT
    finally:
        cswa.attn_debug_set_wait_limit(0)
    assert cswa.attn_get_status() == 0  # cleared by the reads above

    # the default limit again: the same calls are correct
    o, lse = cswa.attn_fwd(q, k, v, W, scale)
    dq, dk, dv = cswa.attn_bwd(q, k, v, o, do, lse, W, scale)
    torch.cuda.synchronize()
    assert cswa.attn_get_status() == 0
    qf, kf, vf, dof = f64(q), f64(k), f64(v), f64(do)
    o_ref, lse_ref = oracle.attention_fwd(qf, kf, vf, W, scale)
    check_out("o after a timed-out call", f64(o), o_ref)
    assert max_abs(f64(lse), lse_ref) <= LSE_MAX_ABS
    dq_ref, dk_ref, dv_ref = oracle.attention_bwd(qf, kf, vf, dof, W, scale)
    check_grad("dq", f64(dq), dq_ref)
    check_grad("dk", f64(dk), dk_ref)
    check_grad("dv", f64(dv), dv_ref)
    assert np.isfinite(f64(dq)).all()


def test_wait_limit_above_default_is_rejected(cswa):
    with pytest.raises(cswa.AttnError):
        cswa.attn_debug_set_wait_limit(3_000_000_000)
