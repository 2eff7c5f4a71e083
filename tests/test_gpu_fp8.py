"""GPU parity of the fp8 path: tensorwise e4m3 quantization and the e4m3 forward.

Quantization decides integer codes, so it is checked bit for bit against the
oracle's quantize_e4m3_tensorwise (scale and products in fp32 on both sides).
The forward rounds P to e4m3 (scaled by 2^8) before the P V product, relative to
the running maximum of the tiles seen so far, so no two implementations round P
alike; it is checked against the oracle's exact attention on the same e4m3
operands with the bound that rounding implies: each P_ij moves by at most 2^-4 of
itself (half a spacing of e4m3's 4 significant bits), hence
    |o_i - o_ref_i| <= 2^-4 * sum_j P_ij |v_j| / l_i  + bf16 output rounding,
element by element (the first term is the oracle's attention of |v|), and its
relative L2 error stays below 3e-2 (one rounding of P measures about 2e-2 here).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import LSE_MAX_ABS, f64, max_abs, record, rel_l2

pytestmark = pytest.mark.gpu

FP8_REL_L2 = 3e-2


@pytest.fixture(scope="module")
def cswa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import causal_sliding_window_attn_b200 as m
    m.lib()
    return m


def codes_of(x8):
    """e4m3 codes (uint8) as float64 values (torch decodes the byte format)."""
    return x8.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


@pytest.mark.parametrize("kind", ["normal", "outlier", "tiny", "zeros"])
def test_quantize_matches_oracle_bit_for_bit(cswa, kind):
    g = torch.Generator().manual_seed(51)
    x = torch.randn((3, 257, 4, 32), generator=g)
    if kind == "outlier":
        x[1, 7, 2, 5] = 900.0
    elif kind == "tiny":
        x = x * 1e-30
    elif kind == "zeros":
        x = torch.zeros_like(x)
    x = x.to(torch.bfloat16)
    x8, d = cswa.attn_quantize_fp8(x.cuda())
    torch.cuda.synchronize()
    codes_ref, s_ref = oracle.quantize_e4m3_tensorwise(f64(x))
    np.testing.assert_array_equal(codes_of(x8), codes_ref)
    amax = float(np.max(np.abs(f64(x))))
    want = np.float32(amax) / np.float32(448) if amax > 0 else np.float32(1)
    assert float(d.item()) == float(want)


def _fp8_case(cswa, B, T, Hq, Hkv, W, seed, rows=None):
    D = 128
    scale = workloads.default_scale(D)
    q, k, v, _ = workloads.training_inputs(B, T, Hq, Hkv, D, seed)
    qh, kh = cswa.attn_rope_qknorm(q.cuda(), k.cuda())
    desc = torch.empty(3, device="cuda", dtype=torch.float32)
    q8, _ = cswa.attn_quantize_fp8(qh, descale=desc[0:1])
    k8, _ = cswa.attn_quantize_fp8(kh, descale=desc[1:2])
    v8, _ = cswa.attn_quantize_fp8(v.cuda(), descale=desc[2:3])
    o, lse = cswa.attn_fwd_fp8(q8, k8, v8, desc, W, scale)
    torch.cuda.synchronize()
    assert cswa.attn_get_status() == 0
    d = desc.cpu().numpy().astype(np.float64)
    qd, kd, vd = codes_of(q8) * d[0], codes_of(k8) * d[1], codes_of(v8) * d[2]
    o_ref, lse_ref = oracle.attention_fwd(qd, kd, vd, W, scale, rows=rows)
    o_abs, _ = oracle.attention_fwd(qd, kd, np.abs(vd), W, scale, rows=rows)
    og = f64(o) if rows is None else f64(o)[:, rows]
    lg = f64(lse) if rows is None else f64(lse)[:, :, rows]
    assert np.all(np.isfinite(og))
    bound = 2.0 ** -4 * o_abs + 2.0 ** -8 * np.abs(o_ref) + 2e-3
    err = np.abs(og - o_ref)
    assert np.all(err <= bound), f"{int((err > bound).sum())} outputs beyond the e4m3 bound, worst {err.max():.3e}"
    rl = rel_l2(og, o_ref)
    assert rl <= FP8_REL_L2, f"rel-L2 {rl:.3e}"
    assert max_abs(lg, lse_ref) <= LSE_MAX_ABS
    # the error of the whole fp8 path against bf16-free attention of the unquantized
    # operands (reported, not held to a bar: the pages give none for fp8)
    o_full, _ = oracle.attention_fwd(f64(qh), f64(kh), f64(v), W, scale, rows=rows)
    record(f"fp8 B{B}_T{T}_Hq{Hq}_Hkv{Hkv}_W{W}", "fp8-vs-e4m3-operands", max_abs=float(err.max()), rel_l2=rl,
           rel_l2_vs_unquantized=rel_l2(og, o_full))


@pytest.mark.parametrize("B,T,Hq,Hkv,W", [(1, 256, 2, 1, 128), (2, 700, 4, 2, 200), (1, 513, 2, 2, -1),
                                          (1, 129, 3, 1, 0), (2, 1, 2, 1, -1)])
def test_fp8_forward_small(cswa, B, T, Hq, Hkv, W):
    _fp8_case(cswa, B, T, Hq, Hkv, W, seed=60 + T)


def test_fp8_forward_fullsize_d20(cswa):
    """The d20 layer (B=8, T=2048, H=10, window 1024), sampled rows of every head."""
    c = workloads.CONFIGS["d20"]
    rows = np.array(sorted({0, 1, 127, 128, 1023, 1024, 1025, 2047} |
                           set(np.random.default_rng(5).integers(0, 2048, 12).tolist())))
    _fp8_case(cswa, c["B"], c["T"], c["Hq"], c["Hkv"], 1024, seed=c["seed"], rows=rows)
