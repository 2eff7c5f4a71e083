"""Shared helpers for the GPU parity tests: tolerances, error metrics, GPU runners.

Tolerances (outputs: max-abs 1e-2 and relative L2 5e-3; gradients dQ/dK/dV:
relative L2 1e-2) are the acceptance bar for the attention block; lse gets
1e-3 absolute.
"""
import json
import os

import numpy as np
import torch

OUT_MAX_ABS = 1e-2
OUT_REL_L2 = 5e-3
GRAD_REL_L2 = 1e-2
LSE_MAX_ABS = 1e-3
# Three parity levels for the attention output:
#   kernel-only   oracle attention on the GPU's own bf16 q_hat, k_hat: the bar above.
#   e2e-bf16      oracle prologue in fp64, its q_hat, k_hat rounded to bf16 (the pages keep
#                 activations in bf16), oracle attention in fp64: the bar above.
#   e2e-fp64      oracle prologue and attention in fp64 with no bf16 step. This also
#                 measures the bf16 storage of q_hat, k_hat: a relative perturbation of up to
#                 2^-9 per element moves each score by ~ scale * sqrt(D) * 2^-9, and o by that
#                 times |v - o|, which reaches ~1e-2 on rows with few visible keys. Any bf16
#                 tensor-core path carries it. Its max-abs bar is 2e-2, a departure from the
#                 1e-2 output bar; its relative L2 bar stays 5e-3.
E2E_MAX_ABS = 2e-2
# bf16 outputs of elementwise kernels: round-to-nearest gives at most half an
# ulp, i.e. 2^-9 relative; 2^-8 leaves room for the fp32 arithmetic before it.
BF16_REL = 2.0 ** -8
ROPE_BASE = 10000.0
EPS = 1e-6


# Measured errors, printed in pytest's terminal summary (and written as JSON to
# $CSWA_PARITY_LOG when that is set) so that every run reports what it saw.
RECORDS = []


def record(test, level, **values):
    RECORDS.append(dict(test=test, level=level, **{k: (round(float(v), 6) if isinstance(v, float) else v)
                                                   for k, v in values.items()}))


def dump_records():
    path = os.environ.get("CSWA_PARITY_LOG")
    if path and RECORDS:
        os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
        with open(path, "w") as f:
            json.dump(RECORDS, f, indent=1)


def f64(t):
    """bf16/fp32 tensor -> float64 numpy (exact widening)."""
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def rel_l2(a, ref):
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-300))


def max_abs(a, ref):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(ref, np.float64))))


def check_out(name, a, ref, max_abs_tol=OUT_MAX_ABS, rel_tol=OUT_REL_L2):
    ma, rl = max_abs(a, ref), rel_l2(a, ref)
    assert np.all(np.isfinite(a)), f"{name}: non-finite values"
    assert ma <= max_abs_tol and rl <= rel_tol, f"{name}: max-abs {ma:.3e} rel-L2 {rl:.3e} (max|ref| {np.max(np.abs(ref)):.2f})"
    return ma, rl


def check_bf16(name, a, ref, abs_tol=1e-3, rel_tol=OUT_REL_L2):
    """Elementwise: |a - ref| <= 2^-8 |ref| + abs_tol, and relative L2 <= rel_tol."""
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    assert np.all(np.isfinite(a)), f"{name}: non-finite values"
    bad = np.abs(a - ref) > BF16_REL * np.abs(ref) + abs_tol
    assert not bad.any(), f"{name}: {int(bad.sum())} elements beyond bf16 rounding, worst {np.max(np.abs(a - ref)):.3e}"
    rl = rel_l2(a, ref)
    assert rl <= rel_tol, f"{name}: rel-L2 {rl:.3e}"
    return rl


def check_grad(name, a, ref, rel_tol=GRAD_REL_L2):
    """Relative L2 <= rel_tol; a reference that is zero up to rounding (e.g. dq
    when every row sees a single key) is checked in absolute terms instead."""
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    assert np.all(np.isfinite(a)), f"{name}: non-finite values"
    if np.linalg.norm(ref) <= 1e-9 * np.sqrt(ref.size):
        ma = float(np.max(np.abs(a))) if a.size else 0.0
        assert ma <= 1e-3, f"{name}: reference is zero, max-abs {ma:.3e}"
        return ma
    rl = rel_l2(a, ref)
    assert rl <= rel_tol, f"{name}: rel-L2 {rl:.3e}"
    return rl


def run_block(cswa, q, k, v, do, window, scale):
    """prologue -> fwd -> bwd -> prologue bwd on the GPU, and the same backward through
    attn_block_bwd (prologue backward fused: dq_f, dk_f, dv_f); a dict of CUDA tensors."""
    q, k, v, do = (t.cuda() for t in (q, k, v, do))
    qh, kh = cswa.attn_rope_qknorm(q, k, rope_base=ROPE_BASE, eps=EPS)
    o, lse = cswa.attn_fwd(qh, kh, v, window, scale)
    dqh, dkh, dv = cswa.attn_bwd(qh, kh, v, o, do, lse, window, scale)
    dq, dk = cswa.attn_rope_qknorm_bwd(q, k, dqh, dkh, rope_base=ROPE_BASE, eps=EPS)
    dq_f, dk_f, dv_f = cswa.attn_block_bwd(q, k, qh, kh, v, o, do, lse, window, scale, rope_base=ROPE_BASE, eps=EPS)
    torch.cuda.synchronize()
    assert cswa.attn_get_status() == 0
    return dict(qh=qh, kh=kh, o=o, lse=lse, dqh=dqh, dkh=dkh, dv=dv, dq=dq, dk=dk, dq_f=dq_f, dk_f=dk_f, dv_f=dv_f)
