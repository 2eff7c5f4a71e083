"""Python binding of libcswa_attn.so: causal sliding-window GQA attention for B200.

Argument marshalling only. Every step runs in the CUDA library's kernels; torch
supplies device memory (outputs and workspaces are torch tensors) and the
current CUDA stream. The functions carry the C ABI's names (include/cswa_attn.h):

    attn_rope_qknorm      fused QK RMS-norm + RoPE prologue
    attn_rope_qknorm_bwd  its backward
    attn_fwd              attention forward -> (o, lse)
    attn_bwd              attention backward -> (dq, dk, dv)
    attn_block_bwd        the block's backward, prologue included -> (dq, dk, dv) w.r.t. raw q, k
    attn_quantize_fp8     tensorwise e4m3 quantization -> (codes, dequantization factor)
    attn_fwd_fp8          attention forward on e4m3 operands -> (o, lse)
    attn_decode           single-token decode against a KV cache -> (o, lse)
    attn_prefill          a chunk of new tokens against a KV cache -> (o, lse)
    attn_layer_window     the window of one layer of a stack (pattern such as "SSSL")
    attn_kv_replicate     a batch-1 prefill cache copied to N sample rows

Tensors are bf16 CUDA tensors in BTHD layout (B, T, H, D), contiguous. There is
no fallback: without the built library (or off an sm_100 GPU) every call raises.
"""
import ctypes
import math
import os

import torch

__all__ = [
    "AttnError", "lib", "attn_rope_qknorm", "attn_rope_qknorm_bwd", "attn_fwd", "attn_bwd",
    "attn_bwd_workspace_bytes", "attn_bwd_workspace_min_bytes", "attn_block_bwd", "attn_block_bwd_workspace_bytes", "attn_quantize_fp8",
    "attn_fwd_fp8", "attn_decode", "attn_decode_workspace_bytes", "attn_prefill", "attn_layer_window",
    "layer_windows", "attn_kv_replicate", "attn_get_status", "attn_debug_set_wait_limit",
    "attn_status_string", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcswa_attn.so")
ATTN_OK = 0
_STATUS = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_LAUNCH",
           4: "ATTN_ERR_TIMEOUT", 5: "ATTN_ERR_DEVICE"}

_lib = None
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "attn_rope_qknorm": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _f, _vp]),
    "attn_rope_qknorm_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _f, _vp]),
    "attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "attn_bwd_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "attn_bwd_workspace_min_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "attn_bwd": (_i, [_vp] * 9 + [_vp, _sz, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "attn_block_bwd_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "attn_block_bwd": (_i, [_vp] * 12 + [_sz, _i, _i, _i, _i, _i, _i, _f, _f, _f, _vp]),
    "attn_quantize_fp8_workspace_bytes": (_sz, [ctypes.c_longlong]),
    "attn_quantize_fp8": (_i, [_vp, ctypes.c_longlong, _vp, _vp, _vp, _sz, _vp]),
    "attn_fwd_fp8": (_i, [_vp] * 6 + [_i] * 6 + [_f, _vp]),
    "attn_decode_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "attn_decode": (_i, [_vp] * 8 + [_i, _i, _i, _i, _i, _i, _f, _vp, _sz, _vp]),
    "attn_decode_noalloc": (_i, [_vp] * 8 + [_i, _i, _i, _i, _i, _i, _f, _vp]),
    "attn_prefill": (_i, [_vp] * 8 + [_i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "attn_layer_window": (_i, [ctypes.c_char_p, _i, _i, _i, _i]),
    "attn_kv_replicate": (_i, [_vp] * 4 + [_i] * 7 + [_vp]),
    "attn_get_status": (_i, [_vp]),
    "attn_debug_set_wait_limit": (_i, [ctypes.c_ulonglong, _vp]),
    "attn_status_string": (ctypes.c_char_p, [_i]),
    "attn_device_supported": (_i, []),
}


class AttnError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {_STATUS.get(status, status)} ({attn_status_string(status)})")


def lib():
    """Loads libcswa_attn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m causal_sliding_window_attn_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def attn_status_string(status):
    return lib().attn_status_string(int(status)).decode()


def _check(fn, status):
    if status != ATTN_OK:
        raise AttnError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _bf16(name, t, ndim=4):
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == ndim
            and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous {ndim}-d bf16 CUDA tensor")
    return t


def _default_scale(D, scale):
    return 1.0 / math.sqrt(D) if scale is None else float(scale)


def attn_rope_qknorm(q, k, q_out=None, k_out=None, pos=None, rope_base=10000.0, eps=1e-6, stream=None):
    """Prologue: RoPE(RMSNorm(x)) for q (B,T,Hq,D) and k (B,T,Hkv,D); either may be None."""
    ref = q if q is not None else k
    B, T, _, D = _bf16("q/k", ref).shape
    Hq = q.shape[2] if q is not None else 1
    Hkv = k.shape[2] if k is not None else 1
    if q is not None:
        _bf16("q", q)
        q_out = torch.empty_like(q) if q_out is None else _bf16("q_out", q_out)
    if k is not None:
        _bf16("k", k)
        k_out = torch.empty_like(k) if k_out is None else _bf16("k_out", k_out)
    _check("attn_rope_qknorm", lib().attn_rope_qknorm(
        _ptr(q), _ptr(k), _ptr(q_out) if q is not None else None, _ptr(k_out) if k is not None else None,
        _ptr(pos), B, T, Hq, Hkv, D, float(rope_base), float(eps), _stream(stream)))
    return q_out, k_out


def attn_rope_qknorm_bwd(q, k, dq_hat, dk_hat, dq=None, dk=None, pos=None, rope_base=10000.0, eps=1e-6,
                         stream=None):
    """Backward of the prologue: gradients w.r.t. the raw q and k."""
    ref = q if q is not None else k
    B, T, _, D = _bf16("q/k", ref).shape
    Hq = q.shape[2] if q is not None else 1
    Hkv = k.shape[2] if k is not None else 1
    if q is not None:
        _bf16("dq_hat", dq_hat)
        dq = torch.empty_like(q) if dq is None else _bf16("dq", dq)
    if k is not None:
        _bf16("dk_hat", dk_hat)
        dk = torch.empty_like(k) if dk is None else _bf16("dk", dk)
    _check("attn_rope_qknorm_bwd", lib().attn_rope_qknorm_bwd(
        _ptr(q), _ptr(k), _ptr(dq_hat) if q is not None else None, _ptr(dk_hat) if k is not None else None,
        _ptr(dq) if q is not None else None, _ptr(dk) if k is not None else None, _ptr(pos),
        B, T, Hq, Hkv, D, float(rope_base), float(eps), _stream(stream)))
    return dq, dk


def attn_fwd(q, k, v, window=-1, scale=None, o=None, lse=None, stream=None):
    """o, lse = causal sliding-window GQA attention of q (B,T,Hq,D) over k, v (B,T,Hkv,D)."""
    B, T, Hq, D = _bf16("q", q).shape
    Hkv = _bf16("k", k).shape[2]
    _bf16("v", v)
    o = torch.empty_like(q) if o is None else _bf16("o", o)
    lse = torch.empty((B, Hq, T), device=q.device, dtype=torch.float32) if lse is None else lse
    _check("attn_fwd", lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, T, Hq, Hkv, D,
                                      int(window), _default_scale(D, scale), _stream(stream)))
    return o, lse


def attn_quantize_fp8(x, x8=None, descale=None, workspace=None, stream=None):
    """x8 (uint8 e4m3 codes, x's shape), descale (1 float on the device): tensorwise e4m3
    quantization of the bf16 CUDA tensor x; x ~ x8 * descale."""
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous()):
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    n = x.numel()
    x8 = torch.empty(x.shape, device=x.device, dtype=torch.uint8) if x8 is None else x8
    descale = torch.empty(1, device=x.device, dtype=torch.float32) if descale is None else descale
    nbytes = int(lib().attn_quantize_fp8_workspace_bytes(n))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 4), device=x.device, dtype=torch.uint8)
    _check("attn_quantize_fp8", lib().attn_quantize_fp8(
        _ptr(x), n, _ptr(x8), _ptr(descale), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return x8, descale


def attn_fwd_fp8(q8, k8, v8, descale, window=-1, scale=None, o=None, lse=None, stream=None):
    """o (bf16), lse of attention on e4m3 codes q8 (B,T,Hq,128), k8, v8 (B,T,Hkv,128); descale
    holds the three dequantization factors (q, k, v) as a float32 CUDA tensor."""
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.uint8 and t.dim() == 4
                and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous 4-d uint8 CUDA tensor of e4m3 codes")
    if not (descale.is_cuda and descale.dtype == torch.float32 and descale.numel() >= 3 and descale.is_contiguous()):
        raise ValueError("descale must hold 3 float32 values on the device")
    B, T, Hq, D = q8.shape
    Hkv = k8.shape[2]
    o = torch.empty((B, T, Hq, D), device=q8.device, dtype=torch.bfloat16) if o is None else _bf16("o", o)
    lse = torch.empty((B, Hq, T), device=q8.device, dtype=torch.float32) if lse is None else lse
    _check("attn_fwd_fp8", lib().attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(descale), _ptr(o), _ptr(lse), B, T,
                                              Hq, Hkv, D, int(window), _default_scale(D, scale), _stream(stream)))
    return o, lse


def attn_bwd_workspace_bytes(B, T, Hq, Hkv, D, window=-1):
    return int(lib().attn_bwd_workspace_bytes(B, T, Hq, Hkv, D, int(window)))


def attn_bwd_workspace_min_bytes(B, T, Hq, Hkv, D, window=-1):
    return int(lib().attn_bwd_workspace_min_bytes(B, T, Hq, Hkv, D, int(window)))


def attn_bwd(q, k, v, o, dout, lse, window=-1, scale=None, dq=None, dk=None, dv=None, workspace=None,
             stream=None):
    """dq, dk, dv of sum(dout * o) for o = attn_fwd(q, k, v). A workspace smaller than
    attn_bwd_workspace_bytes (down to attn_bwd_workspace_min_bytes) runs in passes."""
    B, T, Hq, D = _bf16("q", q).shape
    Hkv = _bf16("k", k).shape[2]
    for name, t in (("v", v), ("o", o), ("dout", dout)):
        _bf16(name, t)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nbytes = attn_bwd_workspace_bytes(B, T, Hq, Hkv, D, window)
    if workspace is None:
        workspace = torch.empty(nbytes, device=q.device, dtype=torch.uint8)
    _check("attn_bwd", lib().attn_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(workspace), workspace.numel() * workspace.element_size(), B, T, Hq, Hkv, D, int(window),
        _default_scale(D, scale), _stream(stream)))
    return dq, dk, dv


def attn_block_bwd_workspace_bytes(B, T, Hq, Hkv, D, window=-1):
    return int(lib().attn_block_bwd_workspace_bytes(B, T, Hq, Hkv, D, int(window)))


def attn_block_bwd(q, k, q_hat, k_hat, v, o, dout, lse, window=-1, scale=None, dq=None, dk=None, dv=None,
                   workspace=None, rope_base=10000.0, eps=1e-6, stream=None):
    """dq, dk (w.r.t. the raw q, k of the prologue) and dv of sum(dout * o) for
    o = attn_fwd(*attn_rope_qknorm(q, k), v): attn_bwd with the prologue backward fused."""
    B, T, Hq, D = _bf16("q", q).shape
    Hkv = _bf16("k", k).shape[2]
    for name, t in (("q_hat", q_hat), ("k_hat", k_hat), ("v", v), ("o", o), ("dout", dout)):
        _bf16(name, t)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nbytes = attn_block_bwd_workspace_bytes(B, T, Hq, Hkv, D, window)
    if workspace is None:
        workspace = torch.empty(nbytes, device=q.device, dtype=torch.uint8)
    _check("attn_block_bwd", lib().attn_block_bwd(
        _ptr(q), _ptr(k), _ptr(q_hat), _ptr(k_hat), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(), B, T, Hq, Hkv, D, int(window),
        _default_scale(D, scale), float(rope_base), float(eps), _stream(stream)))
    return dq, dk, dv


def attn_decode_workspace_bytes(B, Hq, D, Tmax, window):
    return int(lib().attn_decode_workspace_bytes(B, Hq, D, Tmax, window))


def attn_decode(q, kcache, vcache, pos, window=-1, scale=None, k_new=None, v_new=None, o=None, lse=None,
                workspace=None, stream=None):
    """o (B,1,Hq,D), lse (B,Hq) for one new token per sequence; appends k_new/v_new in place."""
    B, _, Hq, D = _bf16("q", q).shape
    _, Tmax, Hkv, _ = _bf16("kcache", kcache).shape
    _bf16("vcache", vcache)
    if not (pos.is_cuda and pos.dtype == torch.int32 and pos.numel() == B):
        raise ValueError("pos must be an int32 CUDA tensor of B entries")
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, Hq), device=q.device, dtype=torch.float32) if lse is None else lse
    nbytes = attn_decode_workspace_bytes(B, Hq, D, Tmax, window)
    if workspace is None:
        workspace = torch.empty(nbytes, device=q.device, dtype=torch.uint8)
    _check("attn_decode", lib().attn_decode(
        _ptr(q), _ptr(kcache), _ptr(vcache), _ptr(k_new), _ptr(v_new), _ptr(pos), _ptr(o), _ptr(lse),
        B, Tmax, Hq, Hkv, D, int(window), _default_scale(D, scale), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return o, lse


def attn_prefill(q, kcache, vcache, pos, window=-1, scale=None, k_new=None, v_new=None, o=None, lse=None,
                 stream=None):
    """o (B,T,Hq,D), lse (B,Hq,T) for a chunk of T tokens per sequence at positions pos[b] + t.

    Appends k_new / v_new (B,T,Hkv,D) into the caches at pos[b] first, in place.
    Pass lse=False to skip the lse output.
    """
    B, T, Hq, D = _bf16("q", q).shape
    _, Tmax, Hkv, _ = _bf16("kcache", kcache).shape
    _bf16("vcache", vcache)
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    if k_new is not None:
        _bf16("k_new", k_new)
        _bf16("v_new", v_new)
    if not (pos.is_cuda and pos.dtype == torch.int32 and pos.numel() == B):
        raise ValueError("pos must be an int32 CUDA tensor of B entries")
    o = torch.empty_like(q) if o is None else _bf16("o", o)
    if lse is None:
        lse = torch.empty((B, Hq, T), device=q.device, dtype=torch.float32)
    lse_t = None if lse is False else lse
    _check("attn_prefill", lib().attn_prefill(
        _ptr(q), _ptr(kcache), _ptr(vcache), _ptr(k_new), _ptr(v_new), _ptr(pos), _ptr(o), _ptr(lse_t),
        B, T, Tmax, Hq, Hkv, D, int(window), _default_scale(D, scale), _stream(stream)))
    return o, lse_t


def attn_layer_window(pattern, layer, n_layer, seq_len, short_window=0):
    """Window of one layer: -1 (full context) for L and for the last layer, else the
    short window (a quarter of seq_len up to a 128 multiple unless short_window > 0)."""
    w = int(lib().attn_layer_window(pattern.encode(), int(layer), int(n_layer), int(seq_len), int(short_window)))
    if w < -1:
        raise ValueError(f"bad window pattern {pattern!r} or sizes (layer {layer} of {n_layer}, seq_len {seq_len})")
    return w


def layer_windows(n_layer, seq_len, pattern="SSSL", short_window=0):
    """The windows of every layer of an n_layer stack."""
    return [attn_layer_window(pattern, l, n_layer, seq_len, short_window) for l in range(n_layer)]


def attn_kv_replicate(k_src, v_src, k_dst, v_dst, rows, stream=None):
    """Copies rows [0, rows) of the batch-1 caches (n_layers, 1, Tsrc, Hkv, D) into every
    sample row of (n_layers, N, Tmax, Hkv, D), in place."""
    L1, one, Tsrc, Hkv, D = _bf16("k_src", k_src, 5).shape
    L2, N, Tmax, Hkv2, D2 = _bf16("k_dst", k_dst, 5).shape
    if one != 1 or (L1, Hkv, D) != (L2, Hkv2, D2) or v_src.shape != k_src.shape or v_dst.shape != k_dst.shape:
        raise ValueError("k_src/v_src must be (n_layers, 1, Tsrc, Hkv, D), k_dst/v_dst (n_layers, N, Tmax, Hkv, D)")
    _bf16("v_src", v_src, 5)
    _bf16("v_dst", v_dst, 5)
    _check("attn_kv_replicate", lib().attn_kv_replicate(
        _ptr(k_src), _ptr(v_src), _ptr(k_dst), _ptr(v_dst), L1, int(rows), Tsrc, N, Tmax, Hkv, D, _stream(stream)))
    return k_dst, v_dst


def attn_debug_set_wait_limit(ns, stream=None):
    """Test hook: limit (ns) of the kernels' pipeline waits for later launches; 0 = default (2 s)."""
    _check("attn_debug_set_wait_limit", lib().attn_debug_set_wait_limit(int(ns), _stream(stream)))


def attn_get_status(stream=None):
    """Synchronises the stream and returns (then clears) the device status word."""
    return int(lib().attn_get_status(_stream(stream)))
