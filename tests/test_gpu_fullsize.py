"""GPU parity at the full workload sizes, in the launch configuration bench.py times.

The oracle cannot expand every row at these sizes, so it checks sampled
outputs it can compute one by one: whole query rows of o / lse / dq (rows at
tile edges, window edges and the ends, plus random ones) for every batch and
head, and dk / dv at clusters of keys (every query row that sees them is
expanded). The prologue and its backward are checked on a batch slice. The
decode and chunked-prefill workloads are checked on every (or sampled) row.
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
    return m


def sample_rows(T, W, seed):
    fixed = {0, 1, 127, 128, 129, T // 2 - 1, T // 2, T - 129, T - 128, T - 2, T - 1}
    if W >= 0:
        fixed |= {W - 1, W, W + 1, W + 127, W + 128}
    rng = np.random.default_rng(seed)
    rows = fixed | set(rng.integers(0, T, 16).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < T))


@pytest.mark.parametrize("name,W", [("d20", 1024), ("d20", 2048), ("gqa", 512), ("long", 2048), ("long", -1)])
def test_fullsize_sampled(cswa, name, W):
    c = workloads.CONFIGS[name]
    B, T, Hq, Hkv, D = c["B"], c["T"], c["Hq"], c["Hkv"], c["D"]
    _sampled_check(cswa, name, B, T, Hq, Hkv, D, W, workloads.config_inputs(name))


# the longest sequences: 512 and 256 query tiles per head, window and full causal, both head dims
LONG_CASES = [(1, 65536, 2, 1, 128, 8192), (1, 32768, 4, 2, 64, -1)]


@pytest.mark.parametrize("case", LONG_CASES, ids=lambda c: "B{}_T{}_Hq{}_Hkv{}_D{}_W{}".format(*c))
def test_long_sequence_sampled(cswa, case):
    B, T, Hq, Hkv, D, W = case
    # dk/dv at keys near the end only: a key near the start is seen by W or more query rows,
    # each of which the oracle expands over the whole sequence
    _sampled_check(cswa, f"T{T}", B, T, Hq, Hkv, D, W, workloads.training_inputs(B, T, Hq, Hkv, D, seed=T + 7),
                   early_keys=False)


def _sampled_check(cswa, name, B, T, Hq, Hkv, D, W, inputs, early_keys=True):
    scale = workloads.default_scale(D)
    q, k, v, do = inputs
    g = run_block(cswa, q, k, v, do, W, scale)
    qh, kh = f64(g["qh"]), f64(g["kh"])
    vf, dof = f64(v), f64(do)

    rows = sample_rows(T, W, seed=T + W)
    o_gpu = f64(g["o"])[:, rows]
    o_ref, lse_ref = oracle.attention_fwd(qh, kh, vf, W, scale, rows=rows)
    ma, rl = check_out(f"{name} o rows", o_gpu, o_ref)
    tid = f"fullsize {name} W={W} ({len(rows)} rows x B x Hq)"
    record(tid, "kernel-only", max_abs=ma, rel_l2=rl, max_abs_o=float(np.max(np.abs(o_ref))))
    assert max_abs(f64(g["lse"])[:, :, rows], lse_ref) <= LSE_MAX_ABS

    # end to end on the same rows: the oracle's own prologue of the raw q, k
    pos_all = oracle.row_positions(B, T)
    qh_e, kh_e = oracle.prologue(f64(q), pos_all, ROPE_BASE, EPS), oracle.prologue(f64(k), pos_all, ROPE_BASE, EPS)
    o_b16, _ = oracle.attention_fwd(oracle.round_bf16(qh_e), oracle.round_bf16(kh_e), vf, W, scale, rows=rows)
    ma, rl = check_out(f"{name} o rows (end-to-end, bf16 q_hat/k_hat)", o_gpu, o_b16)
    record(tid, "e2e-bf16", max_abs=ma, rel_l2=rl, max_abs_o=float(np.max(np.abs(o_b16))))
    o_e2e, _ = oracle.attention_fwd(qh_e, kh_e, vf, W, scale, rows=rows)
    ma, rl = check_out(f"{name} o rows (end-to-end)", o_gpu, o_e2e, max_abs_tol=E2E_MAX_ABS)
    record(tid, "e2e-fp64", max_abs=ma, rel_l2=rl, max_abs_o=float(np.max(np.abs(o_e2e))))
    del qh_e, kh_e

    bs = [0, B - 1] if B > 1 else [0]
    dq_ref = oracle.attention_bwd_rows(qh[bs], kh[bs], vf[bs], dof[bs], W, scale, rows)
    check_grad(f"{name} dq_hat rows", f64(g["dqh"])[bs][:, rows], dq_ref)

    clusters = [np.arange(T - 12, T)]
    clusters.append(np.arange(100, 104) if W >= 0 and early_keys else np.arange(T - 300, T - 296))
    for keys in clusters:
        dk_ref, dv_ref = oracle.attention_bwd_keys(qh[:1], kh[:1], vf[:1], dof[:1], W, scale, keys)
        check_grad(f"{name} dk_hat keys {keys[0]}..", f64(g["dkh"])[:1, keys], dk_ref)
        check_grad(f"{name} dv keys {keys[0]}..", f64(g["dv"])[:1, keys], dv_ref)

    # prologue forward and backward on one batch row
    pos = oracle.row_positions(1, T)
    check_bf16("q_hat", qh[:1], oracle.prologue(f64(q[:1]), pos, ROPE_BASE, EPS))
    check_bf16("k_hat", kh[:1], oracle.prologue(f64(k[:1]), pos, ROPE_BASE, EPS))
    check_grad("dq (prologue bwd)", f64(g["dq"][:1]), oracle.prologue_bwd(f64(q[:1]), f64(g["dqh"][:1]), pos,
                                                                           ROPE_BASE, EPS))
    check_grad("dk (prologue bwd)", f64(g["dk"][:1]), oracle.prologue_bwd(f64(k[:1]), f64(g["dkh"][:1]), pos,
                                                                           ROPE_BASE, EPS))
    # attn_block_bwd (prologue backward fused) against the oracle's prologue backward of the
    # GPU's own attention gradients on the same batch row; dv must equal attn_bwd's closely
    check_grad("dq (attn_block_bwd)", f64(g["dq_f"][:1]), oracle.prologue_bwd(f64(q[:1]), f64(g["dqh"][:1]), pos,
                                                                               ROPE_BASE, EPS))
    check_grad("dk (attn_block_bwd)", f64(g["dk_f"][:1]), oracle.prologue_bwd(f64(k[:1]), f64(g["dkh"][:1]), pos,
                                                                               ROPE_BASE, EPS))
    check_grad("dv (attn_block_bwd)", f64(g["dv_f"]), f64(g["dv"]), 2e-3)


def test_fullsize_decode(cswa):
    c = workloads.DECODE
    B, Hq, Hkv, D, Tmax, W = c["B"], c["Hq"], c["Hkv"], c["D"], c["Tmax"], c["window"]
    lengths, kraw, vc, qraw, knraw, vn = workloads.decode_inputs(**c)
    kraw, vc, qraw, knraw, vn = (t.cuda() for t in (kraw, vc, qraw, knraw, vn))
    pos = lengths.cuda()
    _, kc = cswa.attn_rope_qknorm(None, kraw)
    qd, kn = cswa.attn_rope_qknorm(qraw, knraw, pos=pos)
    kc0, vc0 = kc.clone(), vc.clone()
    o, lse = cswa.attn_decode(qd, kc, vc, pos, W, k_new=kn, v_new=vn)
    torch.cuda.synchronize()
    assert cswa.attn_get_status() == 0
    o_ref, lse_ref, _, _ = oracle.decode(f64(qd), f64(kc0), f64(vc0), lengths.numpy(), W,
                                         workloads.default_scale(D), k_new=f64(kn), v_new=f64(vn))
    ma, rl = check_out("decode o", f64(o), o_ref)
    record("fullsize decode", "kernel-only", max_abs=ma, rel_l2=rl, max_abs_o=float(np.max(np.abs(o_ref))))
    assert max_abs(f64(lse), lse_ref) <= LSE_MAX_ABS
    # end-to-end: the oracle's own prologue of the raw cache and query
    L = lengths.numpy()
    kc_e2e = oracle.prologue(f64(kraw), oracle.row_positions(B, Tmax), ROPE_BASE, EPS)
    q_e2e = oracle.prologue(f64(qraw), oracle.row_positions(B, 1, L), ROPE_BASE, EPS)
    kn_e2e = oracle.prologue(f64(knraw), oracle.row_positions(B, 1, L), ROPE_BASE, EPS)
    o_e2e, _, _, _ = oracle.decode(q_e2e, kc_e2e, f64(vc0), L, W, workloads.default_scale(D), k_new=kn_e2e,
                                   v_new=f64(vn))
    ma, rl = check_out("decode o (end-to-end)", f64(o), o_e2e, max_abs_tol=E2E_MAX_ABS)
    record("fullsize decode", "e2e-fp64", max_abs=ma, rel_l2=rl, max_abs_o=float(np.max(np.abs(o_e2e))))
    r16 = oracle.round_bf16
    o_b16, _, _, _ = oracle.decode(r16(q_e2e), r16(kc_e2e), f64(vc0), L, W, workloads.default_scale(D),
                                   k_new=r16(kn_e2e), v_new=f64(vn))
    ma, rl = check_out("decode o (end-to-end, bf16 q_hat/k_hat)", f64(o), o_b16)
    record("fullsize decode", "e2e-bf16", max_abs=ma, rel_l2=rl, max_abs_o=float(np.max(np.abs(o_b16))))


def test_fullsize_prefill(cswa):
    """The chunked-prefill workload: 8 sequences, a 512-token chunk each on top of
    cache lengths U[0, 1536], window 1024; sampled chunk rows of every head."""
    c = workloads.PREFILL
    B, Hq, Hkv, D, T, Tmax, W = c["B"], c["Hq"], c["Hkv"], c["D"], c["T"], c["Tmax"], c["window"]
    lengths, kraw, vc, qraw, knraw, vn = workloads.prefill_inputs(**c)
    kraw, vc, qraw, knraw, vn = (t.cuda() for t in (kraw, vc, qraw, knraw, vn))
    pos = lengths.cuda()
    _, kc = cswa.attn_rope_qknorm(None, kraw)
    q, kn = cswa.attn_rope_qknorm(qraw, knraw, pos=pos)
    kc0, vc0 = kc.clone(), vc.clone()
    o, lse = cswa.attn_prefill(q, kc, vc, pos, W, k_new=kn, v_new=vn)
    torch.cuda.synchronize()
    assert cswa.attn_get_status() == 0
    rows = np.array(sorted({0, 1, 127, 128, 255, 256, 383, 384, 510, 511} |
                           set(np.random.default_rng(7).integers(0, T, 12).tolist())))
    o_ref, lse_ref, _, _ = oracle.prefill(f64(q), f64(kc0), f64(vc0), lengths.numpy(), W,
                                          workloads.default_scale(D), k_new=f64(kn), v_new=f64(vn), rows=rows)
    check_out("prefill o rows", f64(o)[:, rows], o_ref)
    assert max_abs(f64(lse)[:, :, rows], lse_ref) <= LSE_MAX_ABS
