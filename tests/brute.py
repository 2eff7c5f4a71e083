"""Pure-Python brute force of the attention block, for tiny shapes only.

A second, deliberately different transcription of the same definitions as the
oracle (scalar loops, the math module, no numpy), used to pin the oracle. It
shares no code with it.

Definitions (nanochat Admin & Developer Guide, 3 "The GPT Model (Internals)";
nanoGPT Administrator & Developer Guide, 8 "CausalSelfAttention"):
  norm:  x / sqrt(mean(x^2) + eps)
  rope:  pair (j, j + D/2) rotated by p * base^(-2j/D)
  attn:  softmax over the visible keys of scale * <q_i, k_j>, times v
"""
import math


def to_list(a):
    return a.tolist() if hasattr(a, "tolist") else a


def norm_row(x, eps):
    ms = sum(t * t for t in x) / len(x)
    r = math.sqrt(ms + eps)
    return [t / r for t in x]


def rope_row(x, p, base):
    D = len(x)
    h = D // 2
    out = [0.0] * D
    for j in range(h):
        ang = p * base ** (-2.0 * j / D)
        c, s = math.cos(ang), math.sin(ang)
        out[j] = x[j] * c - x[j + h] * s
        out[j + h] = x[j] * s + x[j + h] * c
    return out


def prologue(x, base, eps, offsets=None):
    """x: nested list [B][T][H][D]; position of (b, t) = t + offsets[b]."""
    x = to_list(x)
    out = []
    for b, xb in enumerate(x):
        off = 0 if offsets is None else int(offsets[b])
        out.append([[rope_row(norm_row(row, eps), t + off, base) for row in xt]
                    for t, xt in enumerate(xb)])
    return out


def _sees(i, j, W):
    return j <= i and (W < 0 or i - j <= W)


def attention(q, k, v, W, scale):
    """Returns o [B][T][Hq][D] and lse [B][Hq][T]."""
    q, k, v = to_list(q), to_list(k), to_list(v)
    B, T, Hq, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k[0][0])
    G = Hq // Hkv
    o = [[[[0.0] * D for _ in range(Hq)] for _ in range(T)] for _ in range(B)]
    lse = [[[0.0] * T for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for i in range(T):
                js = [j for j in range(T) if _sees(i, j, W)]
                s = [scale * sum(q[b][i][h][d] * k[b][j][g][d] for d in range(D)) for j in js]
                m = max(s)
                e = [math.exp(t - m) for t in s]
                z = sum(e)
                for d in range(D):
                    o[b][i][h][d] = sum(e[n] * v[b][j][g][d] for n, j in enumerate(js)) / z
                lse[b][h][i] = m + math.log(z)
    return o, lse


def attention_grads(q, k, v, do, W, scale):
    """Gradients of sum(do * o) by the chain rule through every scalar."""
    q, k, v, do = to_list(q), to_list(k), to_list(v), to_list(do)
    B, T, Hq, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k[0][0])
    G = Hq // Hkv
    z4 = lambda H: [[[[0.0] * D for _ in range(H)] for _ in range(T)] for _ in range(B)]
    dq, dk, dv = z4(Hq), z4(Hkv), z4(Hkv)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for i in range(T):
                js = [j for j in range(T) if _sees(i, j, W)]
                s = [scale * sum(q[b][i][h][d] * k[b][j][g][d] for d in range(D)) for j in js]
                m = max(s)
                e = [math.exp(t - m) for t in s]
                z = sum(e)
                p = [t / z for t in e]
                # dL/dp_n = <do_i, v_j>;  dL/ds_n = p_n (dL/dp_n - sum_m p_m dL/dp_m)
                gp = [sum(do[b][i][h][d] * v[b][j][g][d] for d in range(D)) for j in js]
                avg = sum(p[n] * gp[n] for n in range(len(js)))
                for n, j in enumerate(js):
                    gs = p[n] * (gp[n] - avg)
                    for d in range(D):
                        dv[b][j][g][d] += p[n] * do[b][i][h][d]
                        dq[b][i][h][d] += scale * gs * k[b][j][g][d]
                        dk[b][j][g][d] += scale * gs * q[b][i][h][d]
    return dq, dk, dv
