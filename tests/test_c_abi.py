"""CPU-side checks of the C ABI: the library builds, loads without a GPU, exports
every entry point include/cswa_attn.h declares, sizes workspaces, and rejects
bad arguments before touching the device (so none of these calls needs a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cswa_attn.h")

INVALID, UNSUPPORTED = 1, 2


@pytest.fixture(scope="module")
def L():
    from causal_sliding_window_attn_b200 import build
    build.build()
    import causal_sliding_window_attn_b200 as m
    return m.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_symbols_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), f"{n} declared in cswa_attn.h but not exported"


def test_status_strings(L):
    for s in range(6):
        assert L.attn_status_string(s)
    assert b"unknown" in L.attn_status_string(99)


def test_bwd_workspace_size(L):
    # -lse/scale and -Delta row pairs (fp32-sized, padded to 128-row tiles) + one 32 KB
    # dS^T tile per (key tile, query tile) pair inside the window + the work counters
    B, T, Hq, Hkv, D = 8, 2048, 10, 10, 128
    rows = B * Hq * 2048 * 4
    # window 1024: key tile n sees min(16 - n, 9) query tiles -> 7*9 + (9+8+...+1) = 108
    assert L.attn_bwd_workspace_bytes(B, T, Hq, Hkv, D, 1024) == 2 * rows + B * Hq * 108 * 32768 + 256
    # no window: the 16*17/2 = 136 tiles of the lower triangle; window >= T - 1 is the same
    full = 2 * rows + B * Hq * 136 * 32768 + 256
    assert L.attn_bwd_workspace_bytes(B, T, Hq, Hkv, D, -1) == full
    assert L.attn_bwd_workspace_bytes(B, T, Hq, Hkv, D, 2048) == full
    # the block backward needs no more (its rotary angles are computed in the kernels)
    assert L.attn_block_bwd_workspace_bytes(B, T, Hq, Hkv, D, -1) == full
    # the least workspace holds one (batch, KV head) block's tiles (G = 1 here; G = 4 and
    # 70 tiles at W = 512 below); workspaces between it and the full size run in passes
    assert L.attn_bwd_workspace_min_bytes(B, T, Hq, Hkv, D, 1024) == 2 * rows + 256 + 108 * 32768
    assert L.attn_bwd_workspace_min_bytes(8, 2048, 16, 4, 128, 512) == 2 * 8 * 16 * 2048 * 4 + 256 + 4 * 70 * 32768
    # ragged T pads the per-row arrays to whole 128-row tiles; window 0 keeps the diagonal only
    assert L.attn_bwd_workspace_bytes(1, 130, 2, 1, 64, 0) == 2 * 2048 + 2 * 2 * 32768 + 256
    assert L.attn_block_bwd_workspace_bytes(1, 3, 1, 1, 64, -1) == 2 * 512 + 32768 + 256
    assert L.attn_bwd_workspace_bytes(1, 16, 3, 2, 128, -1) == 0     # Hq % Hkv != 0
    assert L.attn_bwd_workspace_bytes(1, 16, 2, 2, 96, -1) == 0      # head dim


def test_decode_workspace_size(L):
    # fp32 partials (B, Hq, chunks, D + 2) rounded up to 256 bytes, then an 8-byte
    # arrival counter per (sequence, head); 1025 visible keys at most -> 9 chunks of 128
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert L.attn_decode_workspace_bytes(32, 10, 128, 2176, 1024) == up(32 * 10 * 9 * 130 * 4) + 32 * 10 * 8
    assert L.attn_decode_workspace_bytes(2, 4, 64, 300, -1) == up(2 * 4 * 3 * 66 * 4) + 2 * 4 * 8


P = ctypes.c_void_p(0x10000)      # a 16-byte aligned stand-in; never dereferenced
MIS = ctypes.c_void_p(0x10008)    # misaligned stand-in


def test_fwd_rejects_bad_args(L):
    ok = [P, P, P, P, P, 1, 128, 4, 2, 128, 64, ctypes.c_float(0.1), None]
    def call(**ch):
        a = list(ok)
        for i, v in ch.items():
            a[int(i[1:])] = v
        return L.attn_fwd(*a)
    assert call(a9=96) == UNSUPPORTED                 # head dim
    assert call(a8=3) == INVALID                      # Hq % Hkv
    assert call(a5=0) == INVALID                      # B
    assert call(a6=0) == INVALID                      # T
    assert call(a11=ctypes.c_float(0.0)) == INVALID   # scale
    assert call(a11=ctypes.c_float(float("nan"))) == INVALID
    assert call(a0=None) == INVALID                   # null q
    assert call(a3=MIS) == INVALID                    # misaligned o


def test_bwd_rejects_bad_args(L):
    ws = L.attn_bwd_workspace_bytes(1, 128, 4, 2, 128, 64)
    base = [P] * 9 + [P, ws, 1, 128, 4, 2, 128, 64, ctypes.c_float(0.1), None]
    def call(i, v):
        a = list(base)
        a[i] = v
        return L.attn_bwd(*a)
    # a byte less than one (batch, KV head) block's share (less than the full size runs in passes)
    assert call(10, L.attn_bwd_workspace_min_bytes(1, 128, 4, 2, 128, 64) - 1) == INVALID
    assert call(9, ctypes.c_void_p(0x10010)) == INVALID  # workspace not 256-aligned
    assert call(6, None) == INVALID                   # null dq
    assert call(15, 96) == UNSUPPORTED                # head dim


def test_block_bwd_rejects_bad_args(L):
    ws = L.attn_block_bwd_workspace_bytes(1, 128, 4, 2, 128, 64)
    f = ctypes.c_float
    base = [P] * 11 + [P, ws, 1, 128, 4, 2, 128, 64, f(0.1), f(1e4), f(1e-6), None]
    def call(i, v):
        a = list(base)
        a[i] = v
        return L.attn_block_bwd(*a)
    assert call(12, L.attn_bwd_workspace_min_bytes(1, 128, 4, 2, 128, 64) - 1) == INVALID  # too small
    assert call(0, None) == INVALID                   # null raw q
    assert call(1, MIS) == INVALID                    # misaligned raw k
    assert call(20, f(1.0)) == INVALID                # rope base
    assert call(21, f(-1.0)) == INVALID               # eps
    assert call(17, 96) == UNSUPPORTED                # head dim


def test_rope_rejects_bad_args(L):
    f = ctypes.c_float
    assert L.attn_rope_qknorm(None, None, None, None, None, 1, 4, 2, 2, 128, f(1e4), f(1e-6), None) == INVALID
    assert L.attn_rope_qknorm(P, None, P, None, None, 1, 4, 2, 2, 128, f(1.0), f(1e-6), None) == INVALID
    assert L.attn_rope_qknorm(P, None, P, None, None, 1, 4, 2, 2, 128, f(1e4), f(-1.0), None) == INVALID
    assert L.attn_rope_qknorm(P, None, MIS, None, None, 1, 4, 2, 2, 128, f(1e4), f(1e-6), None) == INVALID
    assert L.attn_rope_qknorm(P, P, P, P, None, 1, 4, 2, 2, 32, f(1e4), f(1e-6), None) == UNSUPPORTED
    # head counts above 65535 (the kernel's per-block row index must stay exact in float)
    assert L.attn_rope_qknorm(P, None, P, None, None, 1, 4, 131072, 1, 128, f(1e4), f(1e-6), None) == INVALID
    assert L.attn_rope_qknorm(None, P, None, P, None, 1, 4, 1, 65536, 128, f(1e4), f(1e-6), None) == INVALID
    assert L.attn_rope_qknorm_bwd(P, None, P, None, P, None, None, 1, 4, 70000, 1, 128, f(1e4), f(1e-6),
                                  None) == INVALID


def test_decode_rejects_bad_args(L):
    ws = L.attn_decode_workspace_bytes(2, 4, 128, 64, -1)
    base = [P, P, P, None, None, P, P, P, 2, 64, 4, 2, 128, -1, ctypes.c_float(0.1), P, ws, None]
    def call(i, v):
        a = list(base)
        a[i] = v
        return L.attn_decode(*a)
    assert call(16, ws - 4) == INVALID
    assert call(3, P) == INVALID                      # k_new without v_new
    assert call(10, 5) == INVALID                     # Hq % Hkv


def test_prefill_rejects_bad_args(L):
    # q, kcache, vcache, k_new, v_new, pos, o, lse, B, T, Tmax, Hq, Hkv, D, window, scale, stream
    base = [P, P, P, P, P, P, P, P, 2, 100, 300, 4, 2, 128, -1, ctypes.c_float(0.1), None]
    def call(i, v):
        a = list(base)
        a[i] = v
        return L.attn_prefill(*a)
    assert call(9, 301) == INVALID                    # chunk longer than the cache
    assert call(3, None) == INVALID                   # v_new without k_new
    assert call(5, None) == INVALID                   # null pos
    assert call(5, ctypes.c_void_p(0x10002)) == INVALID  # pos not 4-byte aligned
    assert call(1, MIS) == INVALID                    # misaligned k cache
    assert call(12, 3) == INVALID                     # Hq % Hkv
    assert call(15, ctypes.c_float(-1.0)) == INVALID  # scale
    assert call(13, 96) == UNSUPPORTED                # head dim


def test_layer_window_rule_on_cpu(L):
    """attn_layer_window is host-only: checked here against the oracle's rule."""
    import oracle
    import causal_sliding_window_attn_b200 as m
    for n_layer, T, pat, sw in ((20, 2048, "SSSL", 0), (12, 1000, "SL", 0), (5, 2048, "S", 1024), (1, 64, "S", 0),
                                (7, 8192, "LSS", 0), (9, 129, "SSSSL", 0)):
        assert m.layer_windows(n_layer, T, pat, sw) == oracle.layer_windows(n_layer, T, pat, sw or None)
    assert L.attn_layer_window(b"SSSL", 0, 20, 2048, 0) == 512
    assert L.attn_layer_window(b"SXSL", 0, 20, 2048, 0) == -2
    assert L.attn_layer_window(b"", 0, 20, 2048, 0) == -2
    assert L.attn_layer_window(None, 0, 20, 2048, 0) == -2
    assert L.attn_layer_window(b"SSSL", 20, 20, 2048, 0) == -2
    assert L.attn_layer_window(b"SSSL", -1, 20, 2048, 0) == -2


def test_kv_replicate_rejects_bad_args(L):
    A, B2, C, E = (ctypes.c_void_p(x) for x in (0x100000, 0x200000, 0x300000, 0x400000))
    # k_src, v_src, k_dst, v_dst, n_layers, rows, Tmax_src, N, Tmax, Hkv, D, stream
    base = [A, B2, C, E, 2, 8, 16, 3, 32, 2, 64, None]
    def call(i, v):
        a = list(base)
        a[i] = v
        return L.attn_kv_replicate(*a)
    assert call(5, 17) == INVALID                      # more rows than the source holds
    assert call(8, 4) == INVALID                       # more rows than the destination holds
    assert call(0, None) == INVALID
    assert call(7, 0) == INVALID                       # no samples
    assert call(3, ctypes.c_void_p(0x300010)) == INVALID  # v_dst overlaps k_dst
    assert call(5, 0) == 0                             # nothing to copy: ok, nothing enqueued


def test_size_limits_rejected_before_launch(L):
    """Calls past the kernels' limits come back before anything is enqueued."""
    f = ctypes.c_float(0.1)
    # decode: more than 4096 chunks of 128 keys in view (an unbounded window over 600k rows)
    Tmax = 600_000
    ws = L.attn_decode_workspace_bytes(1, 1, 128, Tmax, -1)
    assert ws > 0
    assert L.attn_decode(P, P, P, None, None, P, P, P, 1, Tmax, 1, 1, 128, -1, f, P, ws, None) == UNSUPPORTED
    # backward: one (batch, KV head) block's stored dS^T tiles beyond 2^31 rows
    # (G * tiles * 128: 256 * 131328 * 128)
    B, T, Hq, Hkv = 1, 65536, 256, 1
    ws = L.attn_bwd_workspace_bytes(B, T, Hq, Hkv, 128, -1)
    big = ctypes.c_void_p(0x100000000)
    assert ws > 0
    assert L.attn_bwd(*([P] * 9), big, ws, B, T, Hq, Hkv, 128, -1, f, None) == UNSUPPORTED
    # grid limits: 65535 sequences or query heads at most
    assert L.attn_fwd(P, P, P, P, P, 65536, 16, 1, 1, 128, -1, f, None) == INVALID
    assert L.attn_fwd(P, P, P, P, P, 1, 16, 65536, 1, 128, -1, f, None) == INVALID
    assert L.attn_prefill(P, P, P, None, None, P, P, P, 65536, 16, 32, 1, 1, 128, -1, f, None) == INVALID
    # empty inputs
    assert L.attn_fwd(P, P, P, P, P, 1, 0, 1, 1, 128, -1, f, None) == INVALID
    assert L.attn_prefill(P, P, P, None, None, P, P, P, 1, 0, 32, 1, 1, 128, -1, f, None) == INVALID
    assert L.attn_decode(P, P, P, None, None, P, P, P, 0, 64, 1, 1, 128, -1, f, P, 1 << 20, None) == INVALID


def test_wait_limit_hook_rejects_limits_above_the_default(L):
    # checked before anything touches the device
    assert L.attn_debug_set_wait_limit(3_000_000_000, None) == INVALID


def test_fp8_entry_points_reject_bad_args(L):
    f = ctypes.c_float(0.1)
    assert L.attn_quantize_fp8_workspace_bytes(1024) == 4096
    assert L.attn_quantize_fp8_workspace_bytes(12) == 0               # not a multiple of 8
    ws = L.attn_quantize_fp8_workspace_bytes(64)
    assert L.attn_quantize_fp8(P, 60, P, P, P, ws, None) == INVALID   # n % 8
    assert L.attn_quantize_fp8(None, 64, P, P, P, ws, None) == INVALID
    assert L.attn_quantize_fp8(MIS, 64, P, P, P, ws, None) == INVALID  # x misaligned
    assert L.attn_quantize_fp8(P, 64, P, P, P, ws - 4, None) == INVALID
    # q8, k8, v8, descale, o, lse, B, T, Hq, Hkv, D, window, scale, stream
    assert L.attn_fwd_fp8(P, P, P, P, P, P, 1, 128, 2, 1, 64, -1, f, None) == UNSUPPORTED   # D = 64
    assert L.attn_fwd_fp8(P, P, P, None, P, P, 1, 128, 2, 1, 128, -1, f, None) == INVALID  # no descale
    assert L.attn_fwd_fp8(P, P, P, P, P, P, 1, 128, 3, 2, 128, -1, f, None) == INVALID     # Hq % Hkv
    assert L.attn_fwd_fp8(MIS, P, P, P, P, P, 1, 128, 2, 1, 128, -1, f, None) == INVALID   # misaligned
