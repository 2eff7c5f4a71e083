"""fp64 CPU oracle: the causal sliding-window GQA attention block, from its definition.

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only the tests, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU legs (``cpu_baseline``, ``--impl reference``) use it.

Sources (page title, section):
  [AG3] nanochat Admin & Developer Guide, 3 "The GPT Model (Internals)":
        rotary embeddings instead of learned positions; queries and keys are
        RMS-normalised with no learnable weight; grouped-query attention with
        n_kv_head <= n_head; a per-layer sliding window handed to flash
        attention as a (left, right) pair ("Sliding-window attention"): a
        pattern of S (a quarter of the context, rounded up to a 128 tile) and
        L (full context) tiled over the layers, the last layer always L.
  [AG5] nanochat Admin & Developer Guide, 5 "Precision: Explicit dtype & FP8":
        the FP8 path scales each tensor by one factor (tensorwise, dynamic) and
        keeps forward tensors in float8 e4m3.
  [AG6] nanochat Admin & Developer Guide, 6 "Attention: FA3 with SDPA Fallback":
        GQA through enable_gqa; single-token decode slices the KV window; FA3
        runs in bf16 or fp8.
  [AG7] nanochat Admin & Developer Guide, 7 "KV cache": (B, T, H, D) caches,
        int32 per-row positions, appended in place; a batch-1 prefill cache
        copied into a batch-N decode cache (one row per sample).
  [NG8] nanoGPT Administrator & Developer Guide, 8 "CausalSelfAttention":
        the manual path -- q k^T scaled by 1/sqrt(d), a triangular mask,
        softmax, then a product with v.
  [NG6] nanoGPT Administrator & Developer Guide, 6 "MFU": attention costs
        12*H*Q*T FLOPs per token, i.e. forward 4*D per visible pair and
        backward twice that.

Readings where the pages are silent or disagree:
  * RoPE pairs dimension j with j + D/2 ("half split") and rotates by +phi,
    phi = p * base**(-2j/D). The base is an argument (10000 in every config;
    [AG3] prints 100000 for nanochat itself).
  * The RMS-norm epsilon is an argument (default 1e-6), added under the root.
  * The norm runs before the rotation. The two commute exactly, because the
    rotation is orthogonal and so leaves the RMS unchanged.
  * window W >= 0: key j is visible from query i iff 0 <= i - j <= W, the
    (left=W, right=0) pair of [AG3]; W < 0: plain causal.
  * GQA: query head h reads KV head h // (Hq / Hkv) (contiguous groups, which
    is what repeating each KV head Hq/Hkv times means).
  * lse is the natural-log log-sum-exp of the scaled scores, shape (B, Hq, T).
  * The 1.2 QK gain of [AG3] is folded into ``scale``.
  * The short window is a quarter of the context rounded up to a multiple of
    128 (2048 -> 512); the example printed beside that rule (2048 -> 768) does
    not follow from it and is not used.

Everything is float64 numpy. Query rows are independent by definition, so the
functions can be asked for a subset of rows; nothing else is blocked, fused or
reordered.
"""
import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# Prologue: QK RMS-norm and rotary embedding  [AG3]
# --------------------------------------------------------------------------
def rms_norm(x, eps):
    """x / sqrt(mean(x**2) + eps) over the last (head) dimension; no weight [AG3]."""
    x = _f64(x)
    r = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x / r


def rope_frequencies(D, base):
    """omega_j = base**(-2j/D) for j = 0 .. D/2-1 (reading of [AG3])."""
    j = np.arange(D // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * j / D)


def row_positions(B, T, pos=None):
    """Position of row (b, t): t, plus pos[b] when per-row offsets are given [AG7]."""
    t = np.arange(T, dtype=np.int64)[None, :]
    if pos is None:
        return np.broadcast_to(t, (B, T)).copy()
    return t + np.asarray(pos, dtype=np.int64).reshape(B, 1)


def rope_angles(positions, D, base):
    """phi[b, t, j] = position(b, t) * omega_j."""
    return np.asarray(positions, dtype=np.float64)[..., None] * rope_frequencies(D, base)


def _cos_sin(positions, D, base):
    phi = rope_angles(positions, D, base)[:, :, None, :]  # (B, T, 1, D/2)
    return np.cos(phi), np.sin(phi)


def rope(x, positions, base):
    """Rotate each (j, j + D/2) pair of x (B, T, H, D) by +phi [AG3]."""
    x = _f64(x)
    h = x.shape[-1] // 2
    c, s = _cos_sin(positions, x.shape[-1], base)
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def rope_transpose(y, positions, base):
    """The transpose (= inverse) of ``rope``: rotate each pair by -phi."""
    y = _f64(y)
    h = y.shape[-1] // 2
    c, s = _cos_sin(positions, y.shape[-1], base)
    y1, y2 = y[..., :h], y[..., h:]
    return np.concatenate([y1 * c + y2 * s, -y1 * s + y2 * c], axis=-1)


def prologue(x, positions, base, eps):
    """RoPE(RMSNorm(x)): the fused prologue applied to q and to k [AG3]."""
    return rope(rms_norm(x, eps), positions, base)


def round_bf16(x):
    """Round to the nearest bfloat16 value, ties to even.

    The pages keep the model's activations in bf16 ([AG6]: FA3 and its fallback
    run in bf16), so the prologue's outputs reach the attention as bf16 values.
    A bf16 number has 8 significant bits: with x = m * 2**e and 0.5 <= |m| < 1,
    the rounded value is round_half_even(m * 2**8) * 2**(e - 8). Only the normal
    range is handled (no value here is below 2**-126 in magnitude or overflows).
    """
    x = _f64(x)
    m, e = np.frexp(x)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def prologue_bwd(x, dy, positions, base, eps):
    """Gradient of sum(dy * prologue(x)) with respect to x.

    With r = sqrt(mean(x**2) + eps), xh = x / r and g = rope_transpose(dy):
    d xh_i / d x_j = (delta_ij - xh_i xh_j / D) / r, so
    dx = (g - xh * (g . xh) / D) / r.
    """
    x = _f64(x)
    D = x.shape[-1]
    r = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    xh = x / r
    g = rope_transpose(dy, positions, base)
    return (g - xh * np.sum(g * xh, axis=-1, keepdims=True) / D) / r


# --------------------------------------------------------------------------
# Attention  [AG3, AG6, NG8]
# --------------------------------------------------------------------------
def visible(i, j, window):
    """Key j is visible from query i iff j <= i and, for window >= 0, i - j <= window."""
    i = np.asarray(i)
    j = np.asarray(j)
    ok = j <= i
    if window >= 0:
        ok = ok & ((i - j) <= window)
    return ok


def useful_pairs(T, window):
    """Number of visible (i, j) pairs of one head, counted on the mask itself."""
    i = np.arange(T)
    return int(np.count_nonzero(visible(i[:, None], i[None, :], window)))


def _group(q, k):
    Hq, Hkv = q.shape[2], k.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return Hq // Hkv


def _probabilities(q, k, b, h, G, window, scale, rows):
    """Softmax probabilities P (R, T) and lse (R,) of query rows ``rows``, head h."""
    T = k.shape[1]
    Q = q[b, rows, h, :]
    K = k[b, :, h // G, :]
    S = scale * (Q @ K.T)
    S = np.where(visible(rows[:, None], np.arange(T)[None, :], window), S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    l = E.sum(axis=1, keepdims=True)
    return E / l, (m + np.log(l))[:, 0]


def attention_fwd(q, k, v, window, scale, rows=None):
    """o = softmax(scale * q k^T + mask) v and lse, for all rows or a subset.

    q (B, T, Hq, D), k and v (B, T, Hkv, D). Returns o (B, R, Hq, D) and
    lse (B, Hq, R) for the R requested query rows (all T by default).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hq, D = q.shape
    G = _group(q, k)
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    o = np.empty((B, len(rows), Hq, D))
    lse = np.empty((B, Hq, len(rows)))
    for b in range(B):
        for h in range(Hq):
            P, l = _probabilities(q, k, b, h, G, window, scale, rows)
            o[b, :, h, :] = P @ v[b, :, h // G, :]
            lse[b, h, :] = l
    return o, lse


def _row_grads(q, k, v, dout, b, h, G, window, scale, rows):
    """P and dS = P * (dP - Delta) for query rows ``rows`` of head h.

    dP = dO V^T, Delta_i = dO_i . o_i: the softmax backward of [NG8]'s manual path.
    """
    P, _ = _probabilities(q, k, b, h, G, window, scale, rows)
    V = v[b, :, h // G, :]
    dO = dout[b, rows, h, :]
    o = P @ V
    dP = dO @ V.T
    delta = np.sum(dO * o, axis=1, keepdims=True)
    return P, P * (dP - delta)


def attention_bwd(q, k, v, dout, window, scale):
    """Gradients (dq, dk, dv) of sum(dout * o) with respect to q, k and v.

    dV = P^T dO, dQ = scale dS K, dK = scale dS^T Q; the KV gradients of a
    group are summed over its Hq/Hkv query heads.
    """
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, T, Hq, D = q.shape
    G = _group(q, k)
    rows = np.arange(T)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            P, dS = _row_grads(q, k, v, dout, b, h, G, window, scale, rows)
            dq[b, :, h, :] = scale * (dS @ k[b, :, kv, :])
            dk[b, :, kv, :] += scale * (dS.T @ q[b, :, h, :])
            dv[b, :, kv, :] += P.T @ dout[b, :, h, :]
    return dq, dk, dv


def attention_bwd_rows(q, k, v, dout, window, scale, rows):
    """dq for the query rows ``rows`` only: (B, R, Hq, D)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, T, Hq, D = q.shape
    G = _group(q, k)
    rows = np.asarray(rows, dtype=np.int64)
    dq = np.empty((B, len(rows), Hq, D))
    for b in range(B):
        for h in range(Hq):
            _, dS = _row_grads(q, k, v, dout, b, h, G, window, scale, rows)
            dq[b, :, h, :] = scale * (dS @ k[b, :, h // G, :])
    return dq


def attention_bwd_keys(q, k, v, dout, window, scale, keys, batches=None):
    """dk, dv at the key rows ``keys`` only: (nb, R, Hkv, D) each.

    Each needs every query row that sees one of the keys, so the rows
    [min(keys), min(T-1, max(keys) + window)] are expanded in full.
    """
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    G = _group(q, k)
    keys = np.asarray(keys, dtype=np.int64)
    batches = list(range(B)) if batches is None else list(batches)
    hi = T - 1 if window < 0 else min(T - 1, int(keys.max()) + window)
    rows = np.arange(int(keys.min()), hi + 1)
    dk = np.zeros((len(batches), len(keys), Hkv, D))
    dv = np.zeros((len(batches), len(keys), Hkv, D))
    for n, b in enumerate(batches):
        for h in range(Hq):
            kv = h // G
            P, dS = _row_grads(q, k, v, dout, b, h, G, window, scale, rows)
            dk[n, :, kv, :] += scale * (dS[:, keys].T @ q[b, rows, h, :])
            dv[n, :, kv, :] += P[:, keys].T @ dout[b, rows, h, :]
    return dk, dv


# --------------------------------------------------------------------------
# Single-token decode against a KV cache  [AG6, AG7]
# --------------------------------------------------------------------------
def decode(q, kcache, vcache, pos, window, scale, k_new=None, v_new=None):
    """One new query token per sequence against its cache.

    q (B, 1, Hq, D); caches (B, Tmax, Hkv, D); pos (B,) = the number of
    entries already in each cache, which is also the new token's position.
    When k_new / v_new (B, 1, Hkv, D) are given they are first written into
    the caches at pos[b] [AG7]. The token then attends to the keys
    [max(0, pos - window), pos] of its own cache [AG6].
    Returns o (B, 1, Hq, D), lse (B, Hq) and the updated caches.
    """
    q = _f64(q)
    kc = _f64(kcache).copy()
    vc = _f64(vcache).copy()
    B, _, Hq, D = q.shape
    G = _group(q, kc)
    pos = np.asarray(pos, dtype=np.int64)
    if k_new is not None:
        for b in range(B):
            kc[b, pos[b]] = _f64(k_new)[b, 0]
            vc[b, pos[b]] = _f64(v_new)[b, 0]
    o = np.empty((B, 1, Hq, D))
    lse = np.empty((B, Hq))
    for b in range(B):
        p = int(pos[b])
        lo = 0 if window < 0 else max(0, p - window)
        for h in range(Hq):
            K = kc[b, lo:p + 1, h // G, :]
            V = vc[b, lo:p + 1, h // G, :]
            s = scale * (K @ q[b, 0, h, :])
            m = s.max()
            e = np.exp(s - m)
            l = e.sum()
            o[b, 0, h, :] = (e @ V) / l
            lse[b, h] = m + np.log(l)
    return o, lse, kc, vc


# --------------------------------------------------------------------------
# Chunked prefill against a KV cache  [AG6, AG7]
# --------------------------------------------------------------------------
def prefill(q, kcache, vcache, pos, window, scale, k_new=None, v_new=None, rows=None):
    """A chunk of Tc new query tokens per sequence against its cache.

    q (B, Tc, Hq, D); caches (B, Tmax, Hkv, D); pos (B,) = the number of
    entries already in each cache, so chunk row t of sequence b sits at
    position pos[b] + t. When k_new / v_new (B, Tc, Hkv, D) are given they are
    first written into the caches at rows pos[b] .. pos[b] + Tc - 1 [AG7].
    Row t then attends to the keys [max(0, p - window), p] of its own cache,
    p = pos[b] + t: the training mask of ``visible`` in absolute positions
    [AG3, AG6]. Cache rows past p are never read.
    Returns o (B, R, Hq, D), lse (B, Hq, R) for the R requested chunk rows
    (all Tc by default) and the updated caches.
    """
    q = _f64(q)
    kc = _f64(kcache).copy()
    vc = _f64(vcache).copy()
    B, Tc, Hq, D = q.shape
    G = _group(q, kc)
    pos = np.asarray(pos, dtype=np.int64)
    if k_new is not None:
        kn, vn = _f64(k_new), _f64(v_new)
        for b in range(B):
            kc[b, pos[b]:pos[b] + Tc] = kn[b]
            vc[b, pos[b]:pos[b] + Tc] = vn[b]
    rows = np.arange(Tc) if rows is None else np.asarray(rows, dtype=np.int64)
    o = np.empty((B, len(rows), Hq, D))
    lse = np.empty((B, Hq, len(rows)))
    for b in range(B):
        p_rows = pos[b] + rows              # absolute positions of the requested rows
        n_keys = int(p_rows.max()) + 1      # keys 0 .. the last row's position
        j = np.arange(n_keys)
        mask = visible(p_rows[:, None], j[None, :], window)
        for h in range(Hq):
            K = kc[b, :n_keys, h // G, :]
            V = vc[b, :n_keys, h // G, :]
            S = scale * (q[b, rows, h, :] @ K.T)
            # masked entries are set, not added: NaN in an unused cache row stays out
            S = np.where(mask, S, -np.inf)
            m = S.max(axis=1, keepdims=True)
            E = np.where(mask, np.exp(S - m), 0.0)
            l = E.sum(axis=1, keepdims=True)
            o[b, :, h, :] = (E / l) @ np.where(mask.any(axis=0)[:, None], V, 0.0)
            lse[b, h, :] = (m + np.log(l))[:, 0]
    return o, lse, kc, vc


# --------------------------------------------------------------------------
# FP8 operands: e4m3 rounding and tensorwise scaling  [AG5, AG6]
# --------------------------------------------------------------------------
E4M3_MAX = 448.0


def round_e4m3(x):
    """Round to the nearest float8 e4m3 ("fn": finite-only) value, ties to even,
    saturating at +-448 [AG5: forward tensors in float8_e4m3fn].

    e4m3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits. A normal value
    in [2**e, 2**(e+1)) (e >= -6) has 4 significant bits, so its spacing is
    2**(e-3); below 2**-6 the values are the subnormals k * 2**-9 (k = 0..7). The
    largest finite value is 448 = 1.75 * 2**8; rounding saturates there instead
    of overflowing (there is no infinity).
    """
    x = _f64(x)
    a = np.abs(x)
    _, e = np.frexp(a)                 # a = m * 2**e with 0.5 <= m < 1: leading bit 2**(e-1)
    q = np.maximum(e - 4, -9).astype(np.float64)   # spacing exponent: 3 bits below the leading one
    r = np.minimum(np.round(a / np.exp2(q)) * np.exp2(q), E4M3_MAX)   # np.round: half to even
    return np.copysign(r, x)


def quantize_e4m3_tensorwise(x):
    """Tensorwise dynamic scaling to e4m3 [AG5: the FP8 recipe scales each tensor by
    one factor from its absolute maximum]: s = 448 / amax(|x|) and codes =
    round_e4m3(x * s), the scale and the product taken in float32 as the device
    computes them (a quantised code is decided in the kernel's precision). amax = 0
    gives s = 1. Returns (codes as float64 values, s); the dequantized tensor is
    codes / s."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    s = np.float32(1) if amax == 0 else np.float32(E4M3_MAX) / amax
    codes = round_e4m3((x32 * s).astype(np.float64))
    return codes, float(s)


# --------------------------------------------------------------------------
# Layer stack: per-layer windows and batch-1 -> N cache replication  [AG3, AG7]
# --------------------------------------------------------------------------
def layer_windows(n_layer, seq_len, pattern="SSSL", short_window=None):
    """Window of every layer: ``pattern`` tiled over the layers, 'L' = the full
    context (returned as -1, unbounded), 'S' = a quarter of the context rounded
    up to a whole 128-row tile (or ``short_window`` when given); the last layer
    is always 'L' whatever the pattern says [AG3]."""
    if not pattern or any(c not in "SL" for c in pattern) or n_layer < 1 or seq_len < 1:
        raise ValueError("bad pattern or sizes")
    if short_window is None or short_window <= 0:
        quarter = -(-seq_len // 4)                  # ceil(seq_len / 4)
        short_window = -(-quarter // 128) * 128     # up to a multiple of 128
    out = []
    for layer in range(n_layer):
        c = "L" if layer == n_layer - 1 else pattern[layer % len(pattern)]
        out.append(-1 if c == "L" else short_window)
    return out


def kv_replicate(k_src, v_src, k_dst, v_dst, rows):
    """Copies rows [0, rows) of a batch-1 cache (n_layers, 1, Tsrc, H, D) into every
    batch row of a batch-N cache (n_layers, N, Tmax, H, D) [AG7: a batch-1 prefill
    is expanded across the samples]; the other rows of the destination are kept."""
    k_out, v_out = np.array(k_dst, copy=True), np.array(v_dst, copy=True)
    for n in range(k_out.shape[1]):
        k_out[:, n, :rows] = np.asarray(k_src)[:, 0, :rows]
        v_out[:, n, :rows] = np.asarray(v_src)[:, 0, :rows]
    return k_out, v_out
