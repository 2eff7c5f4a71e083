"""GPU checks of the layer-stack helpers against the oracle: the batch-1 -> N cache
replication (byte copies, so compared exactly) and nanochat's generation flow over a
small stack: a batch-1 prefill of the prompt in every layer with the layer's window,
the cache expanded to N samples, then one decode step per sample and layer."""
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
    return m


@pytest.mark.parametrize("n_layers,rows,Tsrc,N,Tmax,Hkv,D", [
    (2, 300, 512, 5, 700, 2, 128),     # N not a power of two
    (3, 1, 8, 1, 16, 4, 64),           # one sample, one row
    (4, 1024, 2048, 8, 2048, 10, 128),  # d20 shapes: 8 samples of a 1024-token prompt
])
def test_kv_replicate_is_exact(cswa, n_layers, rows, Tsrc, N, Tmax, Hkv, D):
    g = torch.Generator().manual_seed(rows + N)
    ks = torch.randn((n_layers, 1, Tsrc, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    vs = torch.randn((n_layers, 1, Tsrc, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    kd = torch.randn((n_layers, N, Tmax, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    vd = torch.full((n_layers, N, Tmax, Hkv, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    kd0, vd0 = kd.clone(), vd.clone()
    cswa.attn_kv_replicate(ks, vs, kd, vd, rows)
    torch.cuda.synchronize()
    bits = lambda t: t.view(torch.int16).cpu().numpy()  # noqa: E731  (bf16 compared as raw bits)
    k_ref, v_ref = oracle.kv_replicate(bits(ks), bits(vs), bits(kd0), bits(vd0), rows)
    assert np.array_equal(bits(kd), k_ref)
    assert np.array_equal(bits(vd), v_ref)


def test_generation_flow_over_a_stack(cswa):
    """Prompt prefilled once at batch 1 in each of 3 layers (pattern "SL": windows
    short, full, full), caches expanded to 4 samples, one decode step per sample."""
    n_layers, P0, Tmax, Hq, Hkv, D, N = 3, 300, 640, 4, 2, 128, 4
    scale = workloads.default_scale(D)
    windows = cswa.layer_windows(n_layers, Tmax, "SL")
    assert windows == oracle.layer_windows(n_layers, Tmax, "SL") == [256, -1, -1]
    g = torch.Generator().manual_seed(41)
    rnd = lambda *s: torch.randn(s, generator=g).to(torch.bfloat16).cuda()  # noqa: E731
    kc1 = torch.full((n_layers, 1, Tmax, Hkv, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc1 = kc1.clone()
    kcN = torch.full((n_layers, N, Tmax, Hkv, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    vcN = kcN.clone()
    pos1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    posN = torch.full((N,), P0, dtype=torch.int32, device="cuda")
    prompt, decoded = [], []
    for l in range(n_layers):
        q, k = cswa.attn_rope_qknorm(rnd(1, P0, Hq, D), rnd(1, P0, Hkv, D), pos=pos1)
        v = rnd(1, P0, Hkv, D)
        o, lse = cswa.attn_prefill(q, kc1[l], vc1[l], pos1, windows[l], scale, k_new=k, v_new=v)
        prompt.append((q, k, v, o, lse))
    cswa.attn_kv_replicate(kc1, vc1, kcN, vcN, P0)
    for l in range(n_layers):
        qd, kd = cswa.attn_rope_qknorm(rnd(N, 1, Hq, D), rnd(N, 1, Hkv, D), pos=posN)
        vd = rnd(N, 1, Hkv, D)
        od, ld = cswa.attn_decode(qd, kcN[l], vcN[l], posN, windows[l], scale, k_new=kd, v_new=vd)
        decoded.append((qd, kd, vd, od, ld))
    torch.cuda.synchronize()
    assert cswa.attn_get_status() == 0
    for l in range(n_layers):
        q, k, v, o, lse = prompt[l]
        empty = np.zeros((1, Tmax, Hkv, D))
        o_ref, lse_ref, kc_ref, vc_ref = oracle.prefill(f64(q), empty, empty, [0], windows[l], scale,
                                                        k_new=f64(k), v_new=f64(v))
        check_out(f"layer {l} prompt o", f64(o), o_ref)
        assert max_abs(f64(lse), lse_ref) <= LSE_MAX_ABS
        qd, kd, vd, od, ld = decoded[l]
        kN, vN = oracle.kv_replicate(kc_ref[None], vc_ref[None], np.zeros((1, N, Tmax, Hkv, D)),
                                     np.zeros((1, N, Tmax, Hkv, D)), P0)
        od_ref, ld_ref, _, _ = oracle.decode(f64(qd), kN[0], vN[0], np.full(N, P0), windows[l], scale,
                                             k_new=f64(kd), v_new=f64(vd))
        check_out(f"layer {l} decode o", f64(od), od_ref)
        assert max_abs(f64(ld), ld_ref) <= LSE_MAX_ABS
