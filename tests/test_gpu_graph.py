"""The C-ABI calls captured in a CUDA graph and replayed: the same results as eager calls.

A graph freezes every launch's arguments, so this checks that nothing a call needs is
decided on the host per call: the backward's work-item counters are reset on the device
by its first kernel, and the decode merge's arrival counters start from zero again for a
replay of the same call (same tag). bench.py times the training step this way.
"""
import pytest
import torch

import workloads
from tests.parity import EPS, ROPE_BASE

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cswa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import causal_sliding_window_attn_b200 as m
    m.lib()
    assert m.lib().attn_device_supported() == 1, "not an sm_100 device"
    return m


@pytest.mark.parametrize("B,T,Hq,Hkv,D,W", [(2, 700, 4, 2, 128, 200), (1, 300, 6, 3, 64, -1)])
def test_training_step_replay_matches_eager(cswa, B, T, Hq, Hkv, D, W):
    scale = workloads.default_scale(D)
    q, k, v, do = (t.cuda() for t in workloads.training_inputs(B, T, Hq, Hkv, D, seed=41 + T))
    bufs = dict(qh=torch.empty_like(q), kh=torch.empty_like(k), o=torch.empty_like(q),
                lse=torch.empty((B, Hq, T), device="cuda", dtype=torch.float32),
                dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                ws=torch.empty(cswa.attn_block_bwd_workspace_bytes(B, T, Hq, Hkv, D, W), device="cuda",
                               dtype=torch.uint8))

    def step():
        cswa.attn_rope_qknorm(q, k, bufs["qh"], bufs["kh"], rope_base=ROPE_BASE, eps=EPS)
        cswa.attn_fwd(bufs["qh"], bufs["kh"], v, W, scale, o=bufs["o"], lse=bufs["lse"])
        cswa.attn_block_bwd(q, k, bufs["qh"], bufs["kh"], v, bufs["o"], do, bufs["lse"], W, scale, dq=bufs["dq"],
                            dk=bufs["dk"], dv=bufs["dv"], workspace=bufs["ws"], rope_base=ROPE_BASE, eps=EPS)

    step()
    torch.cuda.synchronize()
    assert cswa.attn_get_status() == 0
    names = ("qh", "kh", "o", "lse", "dq", "dk", "dv")
    eager = {n: bufs[n].clone() for n in names}

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(3):
        for n in names:
            bufs[n].zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert cswa.attn_get_status() == 0
        for n in names:
            assert torch.equal(bufs[n], eager[n]), n


def test_decode_replay_matches_eager(cswa):
    B, Tmax, Hq, Hkv, D, W = 4, 900, 8, 2, 128, 300
    g = torch.Generator().manual_seed(43)
    kraw = torch.randn((B, Tmax, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn((B, Tmax, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    qraw = torch.randn((B, 1, Hq, D), generator=g).to(torch.bfloat16).cuda()
    knraw = torch.randn((B, 1, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn((B, 1, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    pos = torch.tensor([899, 0, 431, 640], dtype=torch.int32).cuda()
    _, kc = cswa.attn_rope_qknorm(None, kraw)
    qd, kn = cswa.attn_rope_qknorm(qraw, knraw, pos=pos)
    o = torch.empty_like(qd)
    lse = torch.empty((B, Hq), device="cuda", dtype=torch.float32)
    ws = torch.randint(0, 256, (cswa.attn_decode_workspace_bytes(B, Hq, D, Tmax, W),), dtype=torch.uint8,
                       device="cuda")

    def call():
        # the append writes the same k_new / v_new rows each time: replays see the same caches
        cswa.attn_decode(qd, kc, vc, pos, W, k_new=kn, v_new=vn, o=o, lse=lse, workspace=ws)

    call()
    torch.cuda.synchronize()
    assert cswa.attn_get_status() == 0
    o_ref, lse_ref = o.clone(), lse.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for _ in range(4):
        o.zero_()
        lse.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert cswa.attn_get_status() == 0
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
