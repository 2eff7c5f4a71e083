"""Pins for the fp64 oracle: it is checked against things other than itself.

  * a hand-worked two-token example (tests/golden/two_token_worked_example.json)
  * a pure-Python brute force on tiny shapes (tests/brute.py)
  * central finite differences of the whole block (prologue + attention)
  * complex-number rotation (numpy complex exp) for RoPE
  * closed forms and invariants: window >= T-1 is full causal, GQA equals MHA
    with repeated KV heads, T = 1 and W = 0 return v, q = 0 gives the windowed
    prefix mean of v with lse = ln(n), sum_j dK_j = 0, sum_j dV_j = sum_i dO_i
  * torch's scaled_dot_product_attention and its autograd, in float64 on the CPU
  * decode at position p equals row p of the forward pass
  * chunked prefill against a cache equals the same rows of one forward pass,
    and a one-token chunk equals a decode step
  * the per-layer window rule on hand-computed cases; a replicated batch-1 cache
    decodes every sample exactly as the batch-1 cache does
  * bf16 rounding: hand-computed ties and near-ties, and torch's own float32 ->
    bfloat16 conversion on random float32 values
  * e4m3 rounding: hand-computed ties, subnormals and saturation, and torch's own
    float32 -> float8_e4m3fn conversion on random in-range float32 values; the
    tensorwise scale maps the absolute maximum to 448
The last test plants plausible mistakes in the oracle and shows a pin fails.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import oracle.attention as oa
import workloads
from tests import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def allclose(a, b, tol):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= tol, f"max abs err {err} > {tol}"


# ---------------------------------------------------------------- checks
# Each check raises AssertionError on failure; the planted-mistake test at the
# bottom reuses them to show that they catch specific errors.

def check_golden():
    g = json.load(open(os.path.join(GOLDEN, "two_token_worked_example.json")))
    i = g["inputs"]
    q = np.array(i["q_raw"])[None, :, None, :]
    k = np.array(i["k_raw"])[None, :, None, :]
    v = np.array(i["v"])[None, :, None, :]
    pos = oracle.row_positions(1, 2)
    qh = oracle.prologue(q, pos, i["rope_base"], i["eps"])
    kh = oracle.prologue(k, pos, i["rope_base"], i["eps"])
    e = g["expected"]
    allclose(qh[0, :, 0, :], e["q_hat"], 1e-12)
    allclose(kh[0, :, 0, :], e["k_hat"], 1e-12)
    o, lse = oracle.attention_fwd(qh, kh, v, i["window"], i["scale"])
    allclose(o[0, :, 0, :], e["o"], 1e-12)
    allclose(lse[0, 0, :], e["lse"], 1e-12)


def check_brute(W, G, seed=0):
    B, T, Hkv, D = 2, 9, 2, 8
    Hq = Hkv * G
    q, k = rnd((B, T, Hq, D), seed), rnd((B, T, Hkv, D), seed + 1)
    v, do = rnd((B, T, Hkv, D), seed + 2), rnd((B, T, Hq, D), seed + 3)
    offs = np.array([0, 5])
    pos = oracle.row_positions(B, T, offs)
    qh = oracle.prologue(q, pos, 10000.0, 1e-6)
    kh = oracle.prologue(k, pos, 10000.0, 1e-6)
    allclose(qh, brute.prologue(q, 10000.0, 1e-6, offs), 1e-12)
    allclose(kh, brute.prologue(k, 10000.0, 1e-6, offs), 1e-12)
    scale = 0.37
    o, lse = oracle.attention_fwd(qh, kh, v, W, scale)
    bo, blse = brute.attention(qh, kh, v, W, scale)
    allclose(o, bo, 1e-12)
    allclose(lse, blse, 1e-12)
    dq, dk, dv = oracle.attention_bwd(qh, kh, v, do, W, scale)
    bq, bk, bv = brute.attention_grads(qh, kh, v, do, W, scale)
    allclose(dq, bq, 1e-12)
    allclose(dk, bk, 1e-12)
    allclose(dv, bv, 1e-12)


def _block_loss(q, k, v, do, W, scale, pos, base, eps):
    qh = oracle.prologue(q, pos, base, eps)
    kh = oracle.prologue(k, pos, base, eps)
    o, _ = oracle.attention_fwd(qh, kh, v, W, scale)
    return float(np.sum(do * o))


def check_finite_differences(W=2, seed=3):
    B, T, Hq, Hkv, D = 1, 6, 4, 2, 4
    base, eps, scale = 10000.0, 1e-6, 0.8
    q, k = rnd((B, T, Hq, D), seed), rnd((B, T, Hkv, D), seed + 1)
    v, do = rnd((B, T, Hkv, D), seed + 2), rnd((B, T, Hq, D), seed + 3)
    pos = oracle.row_positions(B, T, [3])
    qh = oracle.prologue(q, pos, base, eps)
    kh = oracle.prologue(k, pos, base, eps)
    dqh, dkh, dv = oracle.attention_bwd(qh, kh, v, do, W, scale)
    dq = oracle.prologue_bwd(q, dqh, pos, base, eps)
    dk = oracle.prologue_bwd(k, dkh, pos, base, eps)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = dict(q=q, k=k, v=v)
            args[name] = xp
            lp = _block_loss(args["q"], args["k"], args["v"], do, W, scale, pos, base, eps)
            args[name] = xm
            lm = _block_loss(args["q"], args["k"], args["v"], do, W, scale, pos, base, eps)
            fd[idx] = (lp - lm) / (2 * h)
        rel = np.linalg.norm(fd - g) / np.linalg.norm(g)
        assert rel <= 1e-6, f"d{name}: finite-difference rel err {rel}"


def check_rope_complex(seed=4):
    """Half-split RoPE is z_j * exp(i phi_j) with z_j = x_j + i x_{j+D/2}."""
    B, T, H, D = 2, 7, 3, 16
    x = rnd((B, T, H, D), seed)
    pos = oracle.row_positions(B, T, [0, 1000])
    y = oracle.rope(x, pos, 10000.0)
    z = x[..., : D // 2] + 1j * x[..., D // 2:]
    j = np.arange(D // 2)
    phi = pos[:, :, None, None] * (10000.0 ** (-2.0 * j / D))
    w = z * np.exp(1j * phi)
    allclose(y[..., : D // 2], w.real, 1e-12)
    allclose(y[..., D // 2:], w.imag, 1e-12)


def check_window_full_causal(seed=5):
    B, T, Hq, Hkv, D = 1, 12, 2, 1, 8
    q, k, v = rnd((B, T, Hq, D), seed), rnd((B, T, Hkv, D), seed + 1), rnd((B, T, Hkv, D), seed + 2)
    ref, lref = oracle.attention_fwd(q, k, v, -1, 0.5)
    for W in (T - 1, T, 10 * T):
        o, l = oracle.attention_fwd(q, k, v, W, 0.5)
        allclose(o, ref, 0.0)
        allclose(l, lref, 0.0)
    o, _ = oracle.attention_fwd(q, k, v, T - 2, 0.5)
    assert np.max(np.abs(o - ref)) > 1e-6, "W = T-2 must drop the (T-1, 0) pair"
    # with q = 0 every visible key weighs the same, so lse = ln(#keys) = ln(W + 1) once i >= W
    _, l0 = oracle.attention_fwd(np.zeros_like(q), k, v, 3, 0.5)
    allclose(l0[0, 0, 3:], np.full(T - 3, math.log(4)), 1e-12)


def check_gqa_repeat(seed=6):
    B, T, Hkv, G, D = 2, 10, 2, 3, 8
    Hq = Hkv * G
    q, k = rnd((B, T, Hq, D), seed), rnd((B, T, Hkv, D), seed + 1)
    v, do = rnd((B, T, Hkv, D), seed + 2), rnd((B, T, Hq, D), seed + 3)
    kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    W = 4
    o, l = oracle.attention_fwd(q, k, v, W, 0.3)
    om, lm = oracle.attention_fwd(q, kr, vr, W, 0.3)
    allclose(o, om, 1e-13)
    allclose(l, lm, 1e-13)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, W, 0.3)
    dqm, dkm, dvm = oracle.attention_bwd(q, kr, vr, do, W, 0.3)
    allclose(dq, dqm, 1e-13)
    allclose(dk, dkm.reshape(B, T, Hkv, G, D).sum(3), 1e-12)
    allclose(dv, dvm.reshape(B, T, Hkv, G, D).sum(3), 1e-12)


def check_special_cases(seed=7):
    B, T, Hq, Hkv, D = 2, 9, 4, 2, 8
    q, k, v = rnd((B, T, Hq, D), seed), rnd((B, T, Hkv, D), seed + 1), rnd((B, T, Hkv, D), seed + 2)
    vq = np.repeat(v, 2, axis=2)
    o, l = oracle.attention_fwd(q, k, v, 0, 0.7)            # W = 0: self only
    allclose(o, vq, 1e-14)
    o, l = oracle.attention_fwd(q[:, :1], k[:, :1], v[:, :1], -1, 0.7)   # T = 1
    allclose(o, vq[:, :1], 1e-14)
    for W in (-1, 3):                                      # q = 0: uniform weights
        o, l = oracle.attention_fwd(np.zeros_like(q), k, v, W, 0.7)
        for i in range(T):
            lo = 0 if W < 0 else max(0, i - W)
            allclose(o[:, i], vq[:, lo:i + 1].mean(axis=1), 1e-13)
            allclose(l[:, :, i], np.full((B, Hq), math.log(i + 1 - lo)), 1e-13)
    # identical keys: scores are constant along each row, so dq must vanish
    ksame = np.broadcast_to(k[:, :1], k.shape).copy()
    dq, _, _ = oracle.attention_bwd(q, ksame, v, rnd((B, T, Hq, D), 9), 3, 0.7)
    allclose(dq, np.zeros_like(dq), 1e-12)


def check_bwd_invariants(seed=8):
    B, T, Hkv, G, D = 2, 11, 2, 2, 8
    Hq = Hkv * G
    q, k = rnd((B, T, Hq, D), seed), rnd((B, T, Hkv, D), seed + 1)
    v, do = rnd((B, T, Hkv, D), seed + 2), rnd((B, T, Hq, D), seed + 3)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, 3, 0.6)
    # rows of P sum to one  =>  sum_j dV_j = sum over the group's heads of sum_i dO_i
    allclose(dv.sum(axis=1), do.reshape(B, T, Hkv, G, D).sum(axis=(1, 3)), 1e-12)
    # rows of dS sum to zero  =>  sum_j dK_j = 0
    allclose(dk.sum(axis=1), np.zeros((B, Hkv, D)), 1e-12)


def check_sdpa(seed=9):
    """torch's scaled_dot_product_attention (float64, CPU) and its autograd."""
    B, T, Hkv, G, D = 2, 13, 2, 2, 16
    Hq = Hkv * G
    q, k = rnd((B, T, Hq, D), seed), rnd((B, T, Hkv, D), seed + 1)
    v, do = rnd((B, T, Hkv, D), seed + 2), rnd((B, T, Hq, D), seed + 3)
    for W in (-1, 0, 4):
        i = torch.arange(T)
        mask = (i[None, :] <= i[:, None])
        if W >= 0:
            mask &= (i[:, None] - i[None, :]) <= W
        tq, tk, tv = (torch.tensor(a).transpose(1, 2).requires_grad_(True) for a in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(
            tq, tk, tv, attn_mask=mask, scale=0.45, enable_gqa=True)
        o.backward(torch.tensor(do).transpose(1, 2))
        ro, _ = oracle.attention_fwd(q, k, v, W, 0.45)
        allclose(ro, o.detach().transpose(1, 2).numpy(), 1e-12)
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, W, 0.45)
        allclose(dq, tq.grad.transpose(1, 2).numpy(), 1e-12)
        allclose(dk, tk.grad.transpose(1, 2).numpy(), 1e-12)
        allclose(dv, tv.grad.transpose(1, 2).numpy(), 1e-12)


def check_decode_row(seed=10):
    B, Tmax, Hq, Hkv, D = 3, 20, 4, 2, 8
    kc, vc = rnd((B, Tmax, Hkv, D), seed), rnd((B, Tmax, Hkv, D), seed + 1)
    qall = rnd((B, Tmax, Hq, D), seed + 2)
    pos = np.array([0, 7, 19])
    for W in (-1, 3):
        o_full, l_full = oracle.attention_fwd(qall, kc, vc, W, 0.5)
        qd = np.stack([qall[b, pos[b]] for b in range(B)])[:, None]
        o, l, _, _ = oracle.decode(qd, kc, vc, pos, W, 0.5,
                                   k_new=kc[np.arange(B), pos][:, None],
                                   v_new=vc[np.arange(B), pos][:, None])
        for b in range(B):
            allclose(o[b, 0], o_full[b, pos[b]], 1e-13)
            allclose(l[b], l_full[b, :, pos[b]], 1e-13)


def check_prefill_chunks(seed=12):
    """Chunked prefill against a cache equals the rows of one forward pass.

    (a) one sequence per batch entry fed in chunks of 5, 1, 7 and 11 tokens,
    each chunk appending to caches that start out NaN; (b) ragged cache
    lengths: sequence b holds its first pos[b] keys and NaN after them.
    """
    B, Tmax, Hq, Hkv, D = 3, 24, 4, 2, 8
    qall, kall = rnd((B, Tmax, Hq, D), seed), rnd((B, Tmax, Hkv, D), seed + 1)
    vall = rnd((B, Tmax, Hkv, D), seed + 2)
    for W in (-1, 0, 3, 9):
        o_full, l_full = oracle.attention_fwd(qall, kall, vall, W, 0.5)
        kc = np.full((B, Tmax, Hkv, D), np.nan)
        vc = np.full((B, Tmax, Hkv, D), np.nan)
        bounds = [0, 5, 6, 13, 24]
        for c0, c1 in zip(bounds[:-1], bounds[1:]):
            pos = np.full(B, c0)
            o, l, kc, vc = oracle.prefill(qall[:, c0:c1], kc, vc, pos, W, 0.5,
                                          k_new=kall[:, c0:c1], v_new=vall[:, c0:c1])
            allclose(o, o_full[:, c0:c1], 1e-13)
            allclose(l, l_full[:, :, c0:c1], 1e-13)
        allclose(kc, kall, 0.0)
        allclose(vc, vall, 0.0)
        pos = np.array([0, 3, 13])
        Tc = 6
        kc = np.full((B, Tmax, Hkv, D), np.nan)
        vc = np.full((B, Tmax, Hkv, D), np.nan)
        for b in range(B):
            kc[b, :pos[b]] = kall[b, :pos[b]]
            vc[b, :pos[b]] = vall[b, :pos[b]]
        qc = np.stack([qall[b, pos[b]:pos[b] + Tc] for b in range(B)])
        kn = np.stack([kall[b, pos[b]:pos[b] + Tc] for b in range(B)])
        vn = np.stack([vall[b, pos[b]:pos[b] + Tc] for b in range(B)])
        o, l, _, _ = oracle.prefill(qc, kc, vc, pos, W, 0.5, k_new=kn, v_new=vn)
        o2, l2, _, _ = oracle.prefill(qc, kc, vc, pos, W, 0.5, k_new=kn, v_new=vn, rows=[5, 0, 2])
        for b in range(B):
            allclose(o[b], o_full[b, pos[b]:pos[b] + Tc], 1e-13)
            allclose(l[b], l_full[b, :, pos[b]:pos[b] + Tc], 1e-13)
            allclose(o2[b], o_full[b, pos[b] + np.array([5, 0, 2])], 1e-13)


def check_prefill_one_token_is_decode(seed=13):
    """A one-token chunk is a decode step (a separately written routine)."""
    B, Tmax, Hq, Hkv, D = 3, 20, 6, 3, 8
    kc, vc = rnd((B, Tmax, Hkv, D), seed), rnd((B, Tmax, Hkv, D), seed + 1)
    q, kn, vn = rnd((B, 1, Hq, D), seed + 2), rnd((B, 1, Hkv, D), seed + 3), rnd((B, 1, Hkv, D), seed + 4)
    pos = np.array([0, 11, 19])
    for W in (-1, 4):
        o, l, kc1, vc1 = oracle.prefill(q, kc, vc, pos, W, 0.7, k_new=kn, v_new=vn)
        od, ld, kc2, vc2 = oracle.decode(q, kc, vc, pos, W, 0.7, k_new=kn, v_new=vn)
        allclose(o, od, 1e-13)
        allclose(l[:, :, 0], ld, 1e-13)
        allclose(kc1, kc2, 0.0)
        allclose(vc1, vc2, 0.0)


def check_layer_windows():
    """The window rule as the nanochat guide states it, on hand-computed cases:
    the pattern is tiled over the layers, L is the full context, S a quarter of it
    rounded up to a 128 tile, and the last layer is L whatever the pattern says."""
    w = oracle.layer_windows(20, 2048)                       # d20, default SSSL
    assert w == [-1 if (l % 4 == 3 or l == 19) else 512 for l in range(20)]
    assert oracle.layer_windows(6, 2048, "L") == [-1] * 6
    assert oracle.layer_windows(5, 2048, "S") == [512, 512, 512, 512, -1]
    assert oracle.layer_windows(1, 2048, "S") == [-1]
    assert oracle.layer_windows(3, 2048, "SL") == [512, -1, -1]
    assert oracle.layer_windows(4, 1000, "S")[0] == 256       # 250 -> 256
    assert oracle.layer_windows(4, 4096, "S")[0] == 1024
    assert oracle.layer_windows(4, 129, "S")[0] == 128        # 33 -> 128
    assert oracle.layer_windows(4, 2048, "S", short_window=1024)[:3] == [1024] * 3
    for T in (1, 127, 128, 511, 512, 513, 2048, 8191):
        s = oracle.layer_windows(2, T, "S")[0]
        assert s % 128 == 0 and s >= T / 4 and s < T / 4 + 128
    for bad in ("", "SX", "s"):
        with pytest.raises(ValueError):
            oracle.layer_windows(4, 2048, bad)


def check_kv_replicate(seed=14):
    """A batch-1 prefill cache copied to N rows: every sample then decodes exactly as
    it would against the batch-1 cache, and rows past the prompt keep their contents."""
    L, Tsrc, Tmax, H, D, N, rows = 2, 12, 16, 2, 8, 3, 9
    ks, vs = rnd((L, 1, Tsrc, H, D), seed), rnd((L, 1, Tsrc, H, D), seed + 1)
    kd0, vd0 = rnd((L, N, Tmax, H, D), seed + 2), rnd((L, N, Tmax, H, D), seed + 3)
    kd, vd = oracle.kv_replicate(ks, vs, kd0, vd0, rows)
    allclose(kd[:, :, rows:], kd0[:, :, rows:], 0.0)
    allclose(vd[:, :, rows:], vd0[:, :, rows:], 0.0)
    q = rnd((N, 1, 4, D), seed + 4)
    kn, vn = rnd((N, 1, H, D), seed + 5), rnd((N, 1, H, D), seed + 6)
    pos = np.full(N, rows)
    for l in range(L):
        o, lse, _, _ = oracle.decode(q, kd[l], vd[l], pos, 5, 0.3, k_new=kn, v_new=vn)
        for n in range(N):
            o1, l1, _, _ = oracle.decode(q[n:n + 1], ks[l], vs[l], pos[:1], 5, 0.3, k_new=kn[n:n + 1],
                                         v_new=vn[n:n + 1])
            allclose(o[n], o1[0], 1e-13)
            allclose(lse[n], l1[0], 1e-13)


# ---------------------------------------------------------------- tests
def test_golden_two_token():
    check_golden()


@pytest.mark.parametrize("W", [-1, 0, 1, 3])
@pytest.mark.parametrize("G", [1, 2])
def test_brute_force(W, G):
    check_brute(W, G)


@pytest.mark.parametrize("W", [-1, 2])
def test_finite_differences(W):
    check_finite_differences(W)


def test_rope_is_complex_rotation():
    check_rope_complex()


def test_rope_and_norm_closed_forms():
    x = rnd((2, 5, 3, 32), 11)
    p0 = np.zeros((2, 5), np.int64)
    allclose(oracle.rope(x, p0, 10000.0), x, 0.0)                       # p = 0 is identity
    pos = oracle.row_positions(2, 5, [3, 900])
    y = oracle.rope(x, pos, 10000.0)
    allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), 1e-12)   # orthogonal
    allclose(oracle.rope_transpose(y, pos, 10000.0), x, 1e-12)          # transpose inverts
    # relative position: <R_p a, R_s b> depends only on p - s
    a, b = x[0, 0, 0], x[1, 1, 1]
    def rot(vec, p):
        return oracle.rope(vec[None, None, None], np.array([[p]]), 10000.0)[0, 0, 0]
    allclose(rot(a, 5) @ rot(b, 2), rot(a, 103) @ rot(b, 100), 1e-12)
    # norm: unit RMS up to eps, scale invariance, exact eps term, commutes with rope
    n = oracle.rms_norm(x, 0.0)
    allclose(np.sqrt(np.mean(n * n, -1)), np.ones(n.shape[:-1]), 1e-12)
    allclose(oracle.rms_norm(7.5 * x, 0.0), n, 1e-12)
    u = x / np.sqrt(np.mean(x * x, -1, keepdims=True))                 # mean(u^2) = 1
    allclose(oracle.rms_norm(u, 0.5), u / math.sqrt(1.5), 1e-12)
    allclose(oracle.rope(oracle.rms_norm(x, 1e-6), pos, 1e4),
             oracle.rms_norm(oracle.rope(x, pos, 1e4), 1e-6), 1e-12)
    allclose(oracle.rms_norm(np.zeros((1, 1, 1, 8)), 1e-6), np.zeros((1, 1, 1, 8)), 0.0)


def test_window_ge_T_is_full_causal():
    check_window_full_causal()


def test_gqa_equals_mha_with_repeated_kv():
    check_gqa_repeat()


def test_special_cases():
    check_special_cases()


def test_backward_invariants():
    check_bwd_invariants()


def test_matches_torch_sdpa_fp64():
    check_sdpa()


def test_decode_equals_forward_row():
    check_decode_row()


def test_layer_windows():
    check_layer_windows()


def test_kv_replicate():
    check_kv_replicate()


def test_prefill_chunks_equal_forward_rows():
    check_prefill_chunks()


def test_prefill_one_token_is_decode():
    check_prefill_one_token_is_decode()


def test_sampled_backward_matches_full():
    B, T, Hq, Hkv, D = 2, 40, 4, 2, 8
    q, k = rnd((B, T, Hq, D), 12), rnd((B, T, Hkv, D), 13)
    v, do = rnd((B, T, Hkv, D), 14), rnd((B, T, Hq, D), 15)
    for W in (-1, 6):
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, W, 0.4)
        rows = np.array([0, 5, 17, 39])
        allclose(oracle.attention_bwd_rows(q, k, v, do, W, 0.4, rows), dq[:, rows], 1e-12)
        sk, sv = oracle.attention_bwd_keys(q, k, v, do, W, 0.4, rows)
        allclose(sk, dk[:, rows], 1e-12)
        allclose(sv, dv[:, rows], 1e-12)
        o, l = oracle.attention_fwd(q, k, v, W, 0.4)
        so, sl = oracle.attention_fwd(q, k, v, W, 0.4, rows=rows)
        allclose(so, o[:, rows], 1e-13)
        allclose(sl, l[:, :, rows], 1e-13)


def test_visible_pair_count():
    for T, W in ((256, 128), (2048, 1024), (2048, 2048), (2048, 512), (8192, 2048), (8192, -1), (5, 0), (1, -1)):
        assert workloads.visible_pairs(T, W) == oracle.useful_pairs(T, W)


def check_round_bf16_hand():
    """Hand-computed bf16 roundings. Near 1 the bf16 spacing is 2**-7, so 1 + 2**-8 is a
    tie (to the even neighbour 1), 1 + 3 * 2**-8 a tie (to 1 + 2**-6, whose last
    mantissa bit is 0), and 1 + 2**-8 + 2**-20 just above a tie (up to 1 + 2**-7)."""
    cases = [(1 + 2.0 ** -8, 1.0), (1 + 3 * 2.0 ** -8, 1 + 2.0 ** -6), (1 + 2.0 ** -8 + 2.0 ** -20, 1 + 2.0 ** -7),
             (-(1 + 2.0 ** -8 + 2.0 ** -20), -(1 + 2.0 ** -7)), (3.0, 3.0), (0.1, 0.10009765625),
             (255.5, 256.0), (2.0 ** -100 * 1.00390625, 2.0 ** -100), (0.0, 0.0)]
    x = np.array([c[0] for c in cases])
    allclose(oracle.round_bf16(x), [c[1] for c in cases], 0.0)


def check_round_bf16_torch():
    """On float32 inputs a single round-to-nearest-even to bf16 is what torch's
    float32 -> bfloat16 conversion does: both must agree bit for bit."""
    x = torch.from_numpy(rnd(100000, 31) * np.exp(rnd(100000, 32) * 4)).to(torch.float32)
    ref = x.to(torch.bfloat16).to(torch.float64).numpy()
    allclose(oracle.round_bf16(x.to(torch.float64).numpy()), ref, 0.0)


def test_round_bf16():
    check_round_bf16_hand()
    check_round_bf16_torch()
    y = oracle.round_bf16(rnd(1000, 33))
    allclose(oracle.round_bf16(y), y, 0.0)  # idempotent


def check_round_e4m3_hand():
    """Hand-computed e4m3 roundings. Near 1 the spacing is 2**-3: 1.0625 is a tie (to
    1, even mantissa), 1.1875 a tie (to 1.25), 1.9375 a tie that carries into the next
    binade (2). The top binade [256, 448] has spacing 32: 464 is a tie (to 448), and
    values past 448 saturate. Subnormals are k * 2**-9: 2**-10 is a tie (to 0),
    3 * 2**-10 a tie (to 2**-8), 2**-6 - 2**-10 = 7.5 * 2**-9 a tie up to the smallest
    normal 2**-6."""
    cases = [(1.0625, 1.0), (1.1875, 1.25), (1.9375, 2.0), (-1.0625, -1.0), (448.0, 448.0), (464.0, 448.0),
             (480.0, 448.0), (1e6, 448.0), (-500.0, -448.0), (2.0 ** -10, 0.0), (3 * 2.0 ** -10, 2.0 ** -8),
             (2.0 ** -9, 2.0 ** -9), (2.0 ** -6 - 2.0 ** -10, 2.0 ** -6), (0.1, 0.1015625), (5.0, 5.0),
             (5.2, 5.0), (5.3, 5.5), (0.0, 0.0)]
    x = np.array([c[0] for c in cases])
    allclose(oracle.round_e4m3(x), [c[1] for c in cases], 0.0)


def check_round_e4m3_torch():
    """On in-range float32 inputs a single round-to-nearest-even to e4m3 is what torch's
    float32 -> float8_e4m3fn conversion does: both must agree bit for bit."""
    r = (rnd(100000, 41) * np.exp(rnd(100000, 42) * 3)).astype(np.float32)
    r = r[np.abs(r) < 440]
    ref = torch.from_numpy(r).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    allclose(oracle.round_e4m3(r.astype(np.float64)), ref, 0.0)


def test_round_e4m3():
    check_round_e4m3_hand()
    check_round_e4m3_torch()
    y = oracle.round_e4m3(rnd(5000, 43) * 30)
    allclose(oracle.round_e4m3(y), y, 0.0)                       # idempotent
    assert len(np.unique(np.abs(y))) <= 127                       # at most the 127 non-negative finite values


def test_quantize_e4m3_tensorwise():
    x = rnd((4, 33, 2, 16), 44)
    codes, s = oracle.quantize_e4m3_tensorwise(x)
    assert np.max(np.abs(codes)) == oracle.E4M3_MAX              # the absolute maximum maps to 448
    assert s == float(np.float32(448) / np.float32(np.max(np.abs(np.float32(x)))))
    deq = codes / s
    normal = np.abs(x) * s >= 2.0 ** -6
    # a normal e4m3 value is within half a spacing (2**-4 relative) of its input
    assert np.all(np.abs(deq - x)[normal] <= 2.0 ** -4 * np.abs(x)[normal] * (1 + 1e-6))
    assert np.all(np.abs(deq - x)[~normal] <= 2.0 ** -10 / s * (1 + 1e-6))
    z_codes, z_s = oracle.quantize_e4m3_tensorwise(np.zeros(8))
    assert z_s == 1.0 and not np.any(z_codes)


# ---------------------------------------------------------------- planted mistakes
def _rope_wrong_sign(x, positions, base):
    return oa.rope_transpose(x, positions, base)


def _rope_interleaved(x, positions, base):
    """Pairs (2j, 2j+1) instead of (j, j + D/2)."""
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    phi = oa.rope_angles(positions, D, base)[:, :, None, :]
    c, s = np.cos(phi), np.sin(phi)
    y = np.empty_like(x)
    y[..., 0::2] = x[..., 0::2] * c - x[..., 1::2] * s
    y[..., 1::2] = x[..., 0::2] * s + x[..., 1::2] * c
    return y


def _visible_off_by_one(i, j, window):
    i, j = np.asarray(i), np.asarray(j)
    ok = j <= i
    if window >= 0:
        ok = ok & ((i - j) < window)
    return ok


def _group_modulo(q, k):
    return q.shape[2] // k.shape[2]


def _row_grads_no_delta(q, k, v, dout, b, h, G, window, scale, rows):
    P, _ = oa._probabilities(q, k, b, h, G, window, scale, rows)
    dP = dout[b, rows, h, :] @ v[b, :, h // G, :].T
    return P, P * dP


def _prologue_bwd_no_projection(x, dy, positions, base, eps):
    x = np.asarray(x, np.float64)
    r = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return oa.rope_transpose(dy, positions, base) / r


@pytest.mark.parametrize("name,attr,bad,check", [
    ("rope rotates the wrong way", "rope", _rope_wrong_sign, check_rope_complex),
    ("rope pairs interleaved", "rope", _rope_interleaved, check_rope_complex),
    ("window holds W keys, not W+1", "visible", _visible_off_by_one, check_window_full_causal),
    ("softmax backward drops Delta", "_row_grads", _row_grads_no_delta, check_sdpa),
    ("prologue backward drops the norm projection", "prologue_bwd", _prologue_bwd_no_projection,
     check_finite_differences),
])
def test_pins_catch_planted_mistakes(monkeypatch, name, attr, bad, check):
    monkeypatch.setattr(oa, attr, bad)
    monkeypatch.setattr(oracle, attr, bad, raising=False)
    with pytest.raises(AssertionError):
        check()


def test_pins_catch_truncating_bf16_rounding(monkeypatch):
    """Rounding toward zero instead of to nearest must fail the hand-computed cases."""
    def truncate(x):
        m, e = np.frexp(np.asarray(x, np.float64))
        return np.ldexp(np.trunc(m * 256.0) / 256.0, e)
    monkeypatch.setattr(oracle, "round_bf16", truncate)
    with pytest.raises(AssertionError):
        check_round_bf16_hand()
    with pytest.raises(AssertionError):
        check_round_bf16_torch()


@pytest.mark.parametrize("bad", ["truncate", "four_bits"])
def test_pins_catch_wrong_e4m3_rounding(monkeypatch, bad):
    """Rounding toward zero, or keeping one mantissa bit too many, must fail the pins."""
    def wrong(x):
        x = np.asarray(x, np.float64)
        a = np.abs(x)
        _, e = np.frexp(a)
        if bad == "truncate":
            q = np.maximum(e - 4, -9).astype(np.float64)
            r = np.floor(a / np.exp2(q)) * np.exp2(q)
        else:
            q = np.maximum(e - 5, -10).astype(np.float64)
            r = np.round(a / np.exp2(q)) * np.exp2(q)
        return np.copysign(np.minimum(r, 448.0), x)
    monkeypatch.setattr(oracle, "round_e4m3", wrong)
    with pytest.raises(AssertionError):
        check_round_e4m3_hand()
    with pytest.raises(AssertionError):
        check_round_e4m3_torch()


def test_pins_catch_prefill_ignoring_the_cache(monkeypatch):
    """A chunk that attends only to its own keys (the cache left out) must fail."""
    def prefill_chunk_only(q, kcache, vcache, pos, window, scale, k_new=None, v_new=None, rows=None):
        o, lse = oa.attention_fwd(q, k_new, v_new, window, scale, rows)
        return o, lse, kcache, vcache
    monkeypatch.setattr(oracle, "prefill", prefill_chunk_only)
    with pytest.raises(AssertionError):
        check_prefill_chunks()


def test_pins_catch_prefill_positions_off_by_one(monkeypatch):
    """Chunk row t must sit at pos + t; pos + t - 1 breaks the one-token == decode pin."""
    real = oa.prefill
    def shifted(q, kcache, vcache, pos, window, scale, k_new=None, v_new=None, rows=None):
        o, lse, kc, vc = real(q, kcache, vcache, np.maximum(np.asarray(pos) - 1, 0), window, scale, k_new, v_new, rows)
        return o, lse, kc, vc
    monkeypatch.setattr(oracle, "prefill", shifted)
    with pytest.raises(AssertionError):
        check_prefill_one_token_is_decode()


def test_pins_catch_layer_windows_without_a_final_full_layer(monkeypatch):
    """The last layer must be L whatever the pattern says."""
    def tiled_only(n_layer, seq_len, pattern="SSSL", short_window=None):
        s = short_window or -(-(-(-seq_len // 4)) // 128) * 128
        return [-1 if pattern[l % len(pattern)] == "L" else s for l in range(n_layer)]
    monkeypatch.setattr(oracle, "layer_windows", tiled_only)
    with pytest.raises(AssertionError):
        check_layer_windows()


def test_pins_catch_wrong_gqa_mapping(monkeypatch):
    """Query head h must read KV head h // G; reading h % Hkv breaks GQA == repeated MHA."""
    def probs_modulo(q, k, b, h, G, window, scale, rows):
        T = k.shape[1]
        Hkv = k.shape[2]
        S = scale * (q[b, rows, h, :] @ k[b, :, h % Hkv, :].T)
        S = np.where(oa.visible(rows[:, None], np.arange(T)[None, :], window), S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        E = np.exp(S - m)
        return E / E.sum(axis=1, keepdims=True), (m + np.log(E.sum(axis=1, keepdims=True)))[:, 0]
    monkeypatch.setattr(oa, "_probabilities", probs_modulo)
    with pytest.raises(AssertionError):
        check_gqa_repeat()
