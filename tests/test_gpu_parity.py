"""GPU parity: every call of the C ABI against the fp64 oracle, element by element.

Small cases span several 128-row tiles and a ragged tail; three levels each:
  kernel-only  the oracle's attention run on the exact bf16 q_hat / k_hat the GPU
               prologue produced (isolates the attention kernels)
  e2e-bf16     the oracle's own fp64 prologue from the raw bf16 q, k, its outputs
               rounded to bf16 as the pages' bf16 model stores them, then the
               oracle's attention
  e2e-fp64     the oracle's own fp64 prologue and attention with no bf16 step
The first two are held to the output bar (max-abs 1e-2, relative L2 5e-3); the
third to max-abs 2e-2 (see tests/parity.py for why).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import (E2E_MAX_ABS, EPS, LSE_MAX_ABS, ROPE_BASE, check_bf16, check_grad, check_out, f64,
                          max_abs, record, run_block)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cswa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import causal_sliding_window_attn_b200 as m
    m.lib()
    assert m.lib().attn_device_supported() == 1, "not an sm_100 device"
    return m


CASES = [
    # B, T, Hq, Hkv, D, window
    (1, 256, 4, 2, 64, 128),     # the tiny correctness configuration
    (2, 700, 4, 2, 128, 200),    # ragged tail, window not a tile multiple
    (1, 300, 2, 2, 128, -1),     # full causal, ragged
    (1, 513, 4, 4, 128, 256),    # window = 2 tiles, one row past a tile
    (1, 129, 3, 1, 64, 0),       # self only, G = 3
    (2, 1, 2, 1, 128, -1),       # T = 1
    (1, 640, 8, 2, 128, 1000),   # window >= T: plain causal
    (1, 384, 2, 1, 128, 127),    # window one short of a tile
    (1, 300, 16, 1, 128, 100),   # G = 16: one KV head walked by 16 query heads per key tile
]


def _ids(c):
    return "B{}_T{}_Hq{}_Hkv{}_D{}_W{}".format(*c)


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_block_matches_oracle(cswa, case):
    B, T, Hq, Hkv, D, W = case
    scale = workloads.default_scale(D)
    q, k, v, do = workloads.training_inputs(B, T, Hq, Hkv, D, seed=100 + T)
    g = run_block(cswa, q, k, v, do, W, scale)
    pos = oracle.row_positions(B, T)
    qf, kf, vf, dof = f64(q), f64(k), f64(v), f64(do)

    # prologue
    qh_ref = oracle.prologue(qf, pos, ROPE_BASE, EPS)
    kh_ref = oracle.prologue(kf, pos, ROPE_BASE, EPS)
    check_bf16("q_hat", f64(g["qh"]), qh_ref)
    check_bf16("k_hat", f64(g["kh"]), kh_ref)

    # forward, kernel-only
    qh, kh = f64(g["qh"]), f64(g["kh"])
    o_ref, lse_ref = oracle.attention_fwd(qh, kh, vf, W, scale)
    tid = _ids(case)
    ma, rl = check_out("o (kernel)", f64(g["o"]), o_ref)
    record(tid, "kernel-only", max_abs=ma, rel_l2=rl, max_abs_o=float(np.max(np.abs(o_ref))))
    assert max_abs(f64(g["lse"]), lse_ref) <= LSE_MAX_ABS
    # forward, end-to-end with the pages' bf16 activations between prologue and attention
    o_b16, _ = oracle.attention_fwd(oracle.round_bf16(qh_ref), oracle.round_bf16(kh_ref), vf, W, scale)
    ma, rl = check_out("o (end-to-end, bf16 q_hat/k_hat)", f64(g["o"]), o_b16)
    record(tid, "e2e-bf16", max_abs=ma, rel_l2=rl, max_abs_o=float(np.max(np.abs(o_b16))))
    # forward, end-to-end in fp64 throughout
    o_e2e, _ = oracle.attention_fwd(qh_ref, kh_ref, vf, W, scale)
    ma, rl = check_out("o (end-to-end)", f64(g["o"]), o_e2e, max_abs_tol=E2E_MAX_ABS)
    record(tid, "e2e-fp64", max_abs=ma, rel_l2=rl, max_abs_o=float(np.max(np.abs(o_e2e))))

    # backward, kernel-only
    dq_ref, dk_ref, dv_ref = oracle.attention_bwd(qh, kh, vf, dof, W, scale)
    check_grad("dq_hat", f64(g["dqh"]), dq_ref)
    check_grad("dk_hat", f64(g["dkh"]), dk_ref)
    check_grad("dv", f64(g["dv"]), dv_ref)
    # backward through the prologue, end-to-end from the raw inputs
    dqe, dke, dve = oracle.attention_bwd(qh_ref, kh_ref, vf, dof, W, scale)
    dq_e2e, dk_e2e = oracle.prologue_bwd(qf, dqe, pos, ROPE_BASE, EPS), oracle.prologue_bwd(kf, dke, pos, ROPE_BASE, EPS)
    check_grad("dq (end-to-end)", f64(g["dq"]), dq_e2e)
    check_grad("dk (end-to-end)", f64(g["dk"]), dk_e2e)
    check_grad("dv (end-to-end)", f64(g["dv"]), dve)
    # the block backward: the prologue backward fused into the kernels' epilogues
    record(tid, "block-bwd", dq_rel_l2=check_grad("dq (attn_block_bwd)", f64(g["dq_f"]), dq_e2e),
           dk_rel_l2=check_grad("dk (attn_block_bwd)", f64(g["dk_f"]), dk_e2e),
           dv_rel_l2=check_grad("dv (attn_block_bwd)", f64(g["dv_f"]), dve))


def test_prologue_positions_and_inplace(cswa):
    """Per-row position offsets (decode / chunked prefill) and in-place operation."""
    B, T, Hq, Hkv, D = 3, 5, 4, 2, 128
    q, k, _, dy = workloads.training_inputs(B, T, Hq, Hkv, D, seed=7)
    pos = torch.tensor([0, 777, 8000], dtype=torch.int32)
    qd, kd, dyd = q.cuda(), k.cuda(), dy.cuda()
    qh, kh = cswa.attn_rope_qknorm(qd, kd, pos=pos.cuda())
    positions = oracle.row_positions(B, T, pos.numpy())
    check_bf16("q_hat", f64(qh), oracle.prologue(f64(q), positions, ROPE_BASE, EPS))
    check_bf16("k_hat", f64(kh), oracle.prologue(f64(k), positions, ROPE_BASE, EPS))
    q2 = qd.clone()
    cswa.attn_rope_qknorm(q2, None, q_out=q2, pos=pos.cuda())
    assert torch.equal(q2, qh)
    dq, _ = cswa.attn_rope_qknorm_bwd(qd, None, dyd, None, pos=pos.cuda())
    check_grad("dq", f64(dq), oracle.prologue_bwd(f64(q), f64(dy), positions, ROPE_BASE, EPS))


@pytest.mark.parametrize("B,T,Hq,Hkv,D", [(3, 3333, 4, 2, 128), (2, 4801, 6, 3, 64)])
def test_prologue_large_calls(cswa, B, T, Hq, Hkv, D):
    """Large calls (thousands of blocks, a partial last block of positions) with
    position offsets: q and k together, q alone, k alone and in place, all against the
    oracle."""
    q, k, _, _ = workloads.training_inputs(B, T, Hq, Hkv, D, seed=11)
    pos = torch.tensor([5, 1234, 40000][:B], dtype=torch.int32)
    qd, kd = q.cuda(), k.cuda()
    positions = oracle.row_positions(B, T, pos.numpy())
    qh, kh = cswa.attn_rope_qknorm(qd, kd, pos=pos.cuda())
    check_bf16("q_hat", f64(qh), oracle.prologue(f64(q), positions, ROPE_BASE, EPS))
    check_bf16("k_hat", f64(kh), oracle.prologue(f64(k), positions, ROPE_BASE, EPS))
    qa, _ = cswa.attn_rope_qknorm(qd, None, pos=pos.cuda())
    _, ka = cswa.attn_rope_qknorm(None, kd, pos=pos.cuda())
    assert torch.equal(qa, qh) and torch.equal(ka, kh)
    k2 = kd.clone()
    cswa.attn_rope_qknorm(None, k2, k_out=k2, pos=pos.cuda())
    assert torch.equal(k2, kh)


def test_prologue_wide_positions(cswa):
    """Positions with many head rows (160 q heads and 40 k heads): the block's row to
    (operand, position) mapping over long row ranges, against the oracle."""
    B, T, Hq, Hkv, D = 1, 40, 160, 40, 128
    q, k, _, _ = workloads.training_inputs(B, T, Hq, Hkv, D, seed=12)
    qh, kh = cswa.attn_rope_qknorm(q.cuda(), k.cuda())
    positions = oracle.row_positions(B, T, None)
    check_bf16("q_hat", f64(qh), oracle.prologue(f64(q), positions, ROPE_BASE, EPS))
    check_bf16("k_hat", f64(kh), oracle.prologue(f64(k), positions, ROPE_BASE, EPS))


def test_window_ge_T_is_causal_on_gpu(cswa):
    B, T, Hq, Hkv, D = 1, 400, 2, 1, 128
    q, k, v, _ = workloads.training_inputs(B, T, Hq, Hkv, D, seed=11)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    ref, lref = cswa.attn_fwd(q, k, v, -1)
    for W in (T - 1, T, 5000):
        o, l = cswa.attn_fwd(q, k, v, W)
        assert torch.equal(o, ref) and torch.equal(l, lref)
    o, _ = cswa.attn_fwd(q, k, v, T - 2)
    assert not torch.equal(o, ref)


def test_gqa_matches_repeated_kv_on_gpu(cswa):
    B, T, Hkv, G, D = 1, 300, 2, 4, 128
    q, k, v, do = workloads.training_inputs(B, T, Hkv * G, Hkv, D, seed=12)
    q, k, v, do = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    kr, vr = k.repeat_interleave(G, dim=2).contiguous(), v.repeat_interleave(G, dim=2).contiguous()
    o, l = cswa.attn_fwd(q, k, v, 100)
    om, lm = cswa.attn_fwd(q, kr, vr, 100)
    assert torch.equal(o, om) and torch.equal(l, lm)
    dq, dk, dv = cswa.attn_bwd(q, k, v, o, do, l, 100)
    dqm, dkm, dvm = cswa.attn_bwd(q, kr, vr, om, do, lm, 100)
    check_grad("dq", f64(dq), f64(dqm), 2e-3)
    check_grad("dk", f64(dk), f64(dkm).reshape(B, T, Hkv, G, D).sum(3), 5e-3)
    check_grad("dv", f64(dv), f64(dvm).reshape(B, T, Hkv, G, D).sum(3), 5e-3)


@pytest.mark.parametrize("B,T,Hq,Hkv,D,W", [(2, 700, 4, 2, 128, 200), (3, 300, 6, 3, 64, -1)])
def test_bwd_in_passes_matches_one_pass(cswa, B, T, Hq, Hkv, D, W):
    """A workspace below attn_bwd_workspace_bytes runs the backward in passes over the
    (batch, KV head) blocks; every gradient must equal the one-pass result bit for bit
    (each key tile's dK/dV and each query tile's dQ are computed the same way), down to
    one block per pass, and the one-pass result is checked against the oracle elsewhere.
    The workspaces start out filled with garbage."""
    scale = workloads.default_scale(D)
    q, k, v, do = (t.cuda() for t in workloads.training_inputs(B, T, Hq, Hkv, D, seed=31 + T))
    qh, kh = cswa.attn_rope_qknorm(q, k, rope_base=ROPE_BASE, eps=EPS)
    o, lse = cswa.attn_fwd(qh, kh, v, W, scale)
    full = cswa.attn_bwd_workspace_bytes(B, T, Hq, Hkv, D, W)
    least = cswa.attn_bwd_workspace_min_bytes(B, T, Hq, Hkv, D, W)
    assert 0 < least < full
    ref = cswa.attn_bwd(qh, kh, v, o, do, lse, W, scale)
    ref_f = cswa.attn_block_bwd(q, k, qh, kh, v, o, do, lse, W, scale, rope_base=ROPE_BASE, eps=EPS)
    per_block = (full - least) // (B * Hkv - 1)
    for nbytes in (least, least + per_block, least + 2 * per_block + 1000, full - 256):
        ws = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, device="cuda")
        got = cswa.attn_bwd(qh, kh, v, o, do, lse, W, scale, workspace=ws)
        ws.random_(0, 256)
        got_f = cswa.attn_block_bwd(q, k, qh, kh, v, o, do, lse, W, scale, workspace=ws, rope_base=ROPE_BASE,
                                    eps=EPS)
        torch.cuda.synchronize()
        assert cswa.attn_get_status() == 0
        for a, b in zip(got + got_f, ref + ref_f):
            assert torch.equal(a, b), nbytes
    small = torch.empty(least - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError):
        cswa.attn_bwd(qh, kh, v, o, do, lse, W, scale, workspace=small)


def test_T1_W0_return_v(cswa):
    B, T, Hq, Hkv, D = 2, 200, 4, 2, 64
    q, k, v, _ = workloads.training_inputs(B, T, Hq, Hkv, D, seed=13)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    o, _ = cswa.attn_fwd(q, k, v, 0)
    assert torch.equal(o, v.repeat_interleave(2, dim=2))
    o, _ = cswa.attn_fwd(q[:, :1].contiguous(), k[:, :1].contiguous(), v[:, :1].contiguous(), -1)
    assert torch.equal(o, v[:, :1].repeat_interleave(2, dim=2))


def _decode_case(cswa, B, Tmax, Hq, Hkv, D, W, pos, seed, append):
    g = torch.Generator().manual_seed(seed)
    kraw = torch.randn((B, Tmax, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn((B, Tmax, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    qraw = torch.randn((B, 1, Hq, D), generator=g).to(torch.bfloat16).cuda()
    knraw = torch.randn((B, 1, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn((B, 1, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    _, kc = cswa.attn_rope_qknorm(None, kraw)
    posd = torch.tensor(pos, dtype=torch.int32).cuda()
    qd, kn = cswa.attn_rope_qknorm(qraw, knraw, pos=posd)
    # slots past each sequence's position hold NaN: they must never be read
    for b, p in enumerate(pos):
        kc[b, p + (1 if not append else 0):] = float("nan")
        vc[b, p + (1 if not append else 0):] = float("nan")
    if not append:
        for b, p in enumerate(pos):
            kc[b, p] = kn[b, 0]
            vc[b, p] = vn[b, 0]
    kc_before, vc_before = kc.clone(), vc.clone()
    o, lse = cswa.attn_decode(qd, kc, vc, posd, W, k_new=kn if append else None, v_new=vn if append else None)
    torch.cuda.synchronize()
    assert cswa.attn_get_status() == 0
    o_ref, lse_ref, kc_ref, vc_ref = oracle.decode(f64(qd), np.nan_to_num(f64(kc_before)),
                                                   np.nan_to_num(f64(vc_before)), np.array(pos), W,
                                                   workloads.default_scale(D),
                                                   k_new=f64(kn) if append else None,
                                                   v_new=f64(vn) if append else None)
    check_out("decode o", f64(o), o_ref)
    assert max_abs(f64(lse), lse_ref) <= LSE_MAX_ABS
    if append:
        for b, p in enumerate(pos):
            assert torch.equal(kc[b, p], kn[b, 0]) and torch.equal(vc[b, p], vn[b, 0])
        # nothing else in the caches changed
        mask = torch.ones(B, Tmax, dtype=torch.bool)
        for b, p in enumerate(pos):
            mask[b, p] = False
        assert torch.equal(kc[mask.cuda()].nan_to_num(7.0), kc_before[mask.cuda()].nan_to_num(7.0))
    return o


@pytest.mark.parametrize("append", [True, False])
@pytest.mark.parametrize("W", [100, -1, 0])
def test_decode_small(cswa, W, append):
    _decode_case(cswa, 4, 300, 4, 2, 128, W, [0, 150, 299, 37], seed=21, append=append)


def test_decode_d64_gqa8(cswa):
    _decode_case(cswa, 2, 700, 8, 1, 64, 300, [650, 5], seed=22, append=True)


@pytest.mark.parametrize("Hq,Hkv,D", [(16, 1, 128), (32, 2, 64), (12, 1, 128)])
def test_decode_wide_groups(cswa, Hq, Hkv, D):
    """Groups of more than 8 query heads per KV head (sub-groups of 8 in one CTA)."""
    _decode_case(cswa, 3, 900, Hq, Hkv, D, 700, [899, 0, 431], seed=24, append=True)


@pytest.mark.parametrize("W", [-1, 20000])
def test_decode_long_cache(cswa, W):
    """Up to 547 chunks of one sequence merged (more than the merging CTA takes in one
    round of weights), next to a short sequence in the same batch."""
    _decode_case(cswa, 3, 70000, 4, 2, 128, W, [69999, 40000, 130], seed=25, append=True)


def test_decode_repeated_calls_share_a_workspace(cswa):
    """The arrival counters in the workspace are tagged per call: a workspace reused
    across calls (and one that starts out holding garbage) gives the same results."""
    B, Tmax, Hq, Hkv, D, W = 4, 600, 4, 2, 128, 256
    g = torch.Generator().manual_seed(25)
    q = torch.randn((B, 1, Hq, D), generator=g).to(torch.bfloat16).cuda()
    kc = torch.randn((B, Tmax, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn((B, Tmax, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    pos = torch.tensor([599, 10, 300, 128], dtype=torch.int32).cuda()
    ws = torch.randint(0, 255, (cswa.attn_decode_workspace_bytes(B, Hq, D, Tmax, W),), dtype=torch.uint8).cuda()
    ref, lref = cswa.attn_decode(q, kc, vc, pos, W)
    for _ in range(3):
        o, l = cswa.attn_decode(q, kc, vc, pos, W, workspace=ws)
        torch.cuda.synchronize()
        assert cswa.attn_get_status() == 0
        assert torch.equal(o, ref) and torch.equal(l, lref)


def test_decode_equals_forward_row(cswa):
    """Decode at position p equals row p of attn_fwd on the same sequence."""
    B, T, Hq, Hkv, D, W = 1, 520, 4, 2, 128, 200
    q, k, v, _ = workloads.training_inputs(B, T, Hq, Hkv, D, seed=23)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    qh, kh = cswa.attn_rope_qknorm(q, k)
    o, lse = cswa.attn_fwd(qh, kh, v, W)
    for p in (0, 127, 128, 519):
        posd = torch.tensor([p], dtype=torch.int32).cuda()
        od, ld = cswa.attn_decode(qh[:, p:p + 1].contiguous(), kh.clone(), v.clone(), posd, W)
        assert max_abs(f64(od[0, 0]), f64(o[0, p])) <= 1e-2
        assert max_abs(f64(ld[0]), f64(lse[0, :, p])) <= 1e-3


def test_decode_bad_position_is_reported(cswa):
    B, Tmax, H, D = 2, 64, 2, 128
    q = torch.zeros((B, 1, H, D), dtype=torch.bfloat16).cuda()
    kc = torch.zeros((B, Tmax, H, D), dtype=torch.bfloat16).cuda()
    pos = torch.tensor([3, Tmax], dtype=torch.int32).cuda()
    o, lse = cswa.attn_decode(q, kc, kc.clone(), pos, -1)
    assert cswa.attn_get_status() == 5  # ATTN_ERR_DEVICE
    assert torch.isnan(o[1].float()).all() and torch.isfinite(o[0].float()).all()
    assert cswa.attn_get_status() == 0  # cleared
