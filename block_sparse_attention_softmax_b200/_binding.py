"""ctypes binding of libsa.so (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsa.so")
_HEADER = os.path.join(os.path.dirname(_HERE), "include", "sa.h")
_lib = None

c_int, c_double, c_size_t, c_void_p = ctypes.c_int, ctypes.c_double, ctypes.c_size_t, ctypes.c_void_p

_SIGNATURES = {
    "sa_version": (c_int, []),
    "sa_status_string": (ctypes.c_char_p, [c_int]),
    "sa_last_error": (ctypes.c_char_p, []),
    "sa_device_status": (c_int, [c_void_p]),
    "sa_pool_blocks": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                               c_void_p, c_void_p, c_void_p]),
    "sa_build_mask_workspace_size": (c_size_t, [c_int] * 6),
    "sa_build_mask_launches": (c_int, [c_int] * 6),
    "sa_build_mask": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                              c_double, c_double, c_double, c_void_p, c_void_p, c_void_p,
                              c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "sa_build_mask_noalloc": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                      c_double, c_double, c_double, c_void_p, c_void_p, c_void_p,
                                      c_void_p]),
    "sa_sparse_attn_workspace_size": (c_size_t, [c_int] * 7),
    "sa_sparse_attn_fwd": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                   c_int, c_int, c_void_p, c_void_p, c_void_p, c_double,
                                   c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "sa_sparse_attn_blend_fwd": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                         c_int, c_int, c_void_p, c_void_p, c_void_p, c_double,
                                         c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                         c_void_p]),
    "sa_quantize_fp8": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "sa_sparse_attn_fp8_fwd": (c_int, [c_void_p] * 6 + [c_int] * 6 + [c_void_p, c_void_p, c_void_p, c_double,
                                                                    c_void_p, c_void_p, c_void_p, c_void_p,
                                                                    c_void_p, c_size_t, c_void_p]),
    "sa_dense_attn_fwd": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                  c_int, c_double, c_void_p, c_void_p, c_void_p]),
    "sa_linear_workspace_size": (c_size_t, [c_int] * 4),
    "sa_linear_branch": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "sa_blend_workspace_size": (c_size_t, [c_int] * 4),
    "sa_blend": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                         c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
    "sa_trip_pool": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                             c_void_p, c_void_p, c_void_p]),
    "sa_tile_heatmap": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                c_double, c_void_p, c_int, c_void_p, c_void_p, c_void_p]),
    "sa_select_mask": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_double, c_double,
                               c_void_p, c_void_p, c_void_p, c_void_p]),
    "sa_tile_permutation": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "sa_permute_tokens": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p]),
    "sa_sparse_attn_bwd_workspace_size": (c_size_t, [c_int] * 6),
    "sa_sparse_attn_bwd": (c_int, [c_void_p] * 6 + [c_int] * 6 + [c_void_p, c_void_p, c_double, c_void_p, c_void_p,
                                                                c_void_p, c_void_p, c_size_t, c_void_p]),
    "sa_linear_bwd_workspace_size": (c_size_t, [c_int] * 4),
    "sa_linear_bwd": (c_int, [c_void_p] * 6 + [c_int] * 5 + [c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                                              c_void_p]),
    "sa_blend_bwd_workspace_size": (c_size_t, [c_int] * 4),
    "sa_blend_bwd": (c_int, [c_void_p] * 4 + [c_int] * 4 + [c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                                            c_void_p]),
    "sa_diag_set_device_status": (c_int, [c_int]),
    "sa_diag_set_wait_limit": (c_int, [ctypes.c_longlong]),
    "sa_diag_wait_timeout": (c_int, [c_void_p, c_void_p]),
    "sa_diag_exp2": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_void_p]),
}


class SAError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} failed: {status} {msg}")
        self.status = status


def lib_path() -> str:
    return _LIB_PATH


def header_symbols() -> list[str]:
    """Entry points declared in include/sa.h."""
    with open(_HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(sa_\w+)\(", text, re.M)))


def load():
    """Load libsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "python -m block_sparse_attention_softmax_b200.build")
        lib = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _lib = lib
    return _lib


def _call(name, *args):
    lib = load()
    rc = getattr(lib, name)(*args)
    if rc != 0:
        raise SAError(name, lib.sa_status_string(rc).decode(), lib.sa_last_error().decode())
    return rc


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream(device):
    return c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _expect(name, t, shape, dtypes):
    """Checks what the C ABI cannot see behind a raw pointer: the tensor's
    shape, element type and layout. Returns the tensor."""
    if t is None:
        raise ValueError(f"{name} is required")
    if not isinstance(dtypes, tuple):
        dtypes = (dtypes,)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {' or '.join(map(str, dtypes))}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: libsa takes contiguous tensors")
    return t


def _on_device(device, **tensors):
    """Every given tensor is a CUDA tensor on `device`."""
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name}: libsa takes CUDA tensors")
        if t.device != device:
            raise ValueError(f"{name} is on {t.device}, the other operands on {device}")


def _qkv(q, *others, names=("q", "k", "v")):
    """[B, H, N, d] bf16 operands of one shape; returns (B, H, N, d)."""
    if q is None or q.dim() != 4:
        raise ValueError(f"{names[0]} must be a [B, H, N, d] tensor")
    for name, t in zip(names, (q,) + others):
        _expect(name, t, q.shape, torch.bfloat16)
    return tuple(q.shape)


def _workspace(nbytes, device, given=None):
    """The caller's workspace when it is a large enough contiguous uint8
    tensor on `device`, else a new one."""
    if given is not None:
        _expect("workspace", given, given.shape, torch.uint8)
        _on_device(device, workspace=given)
        if given.numel() >= nbytes:
            return given
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def sa_version() -> int:
    return load().sa_version()


def sa_status_string(status: int) -> str:
    return load().sa_status_string(status).decode()


def sa_device_status(device=None):
    device = device or torch.device("cuda", torch.cuda.current_device())
    _call("sa_device_status", _stream(device))


def sa_diag_set_device_status(code: int):
    _call("sa_diag_set_device_status", int(code))


def sa_diag_set_wait_limit(cycles: int):
    """Bound of every device-side wait, in SM cycles (<= 0 restores the default)."""
    _call("sa_diag_set_wait_limit", int(cycles))


def sa_diag_wait_timeout(device=None):
    """Runs one bounded wait that nothing completes; returns (completed, abort flag)."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    out = torch.full((2,), -1, dtype=torch.int32, device=device)
    _call("sa_diag_wait_timeout", _ptr(out), _stream(device))
    return tuple(int(t) for t in out.cpu())


def sa_diag_exp2(x):
    """(FMA-pipe polynomial 2^x, ex2.approx 2^x) of a float32 CUDA tensor."""
    _expect("x", x, x.shape, torch.float32)
    _on_device(x.device, x=x)
    yp, ym = torch.empty_like(x), torch.empty_like(x)
    _call("sa_diag_exp2", _ptr(x), _ptr(yp), _ptr(ym), x.numel(), _stream(x.device))
    return yp, ym


def sa_pool_blocks(q, k, bq, bk):
    B, H, N, d = _qkv(q, k)
    _on_device(q.device, q=q, k=k)
    nqb, nkb = -(-N // bq), -(-N // bk)
    qp = torch.empty(B, H, nqb, d, dtype=torch.float32, device=q.device)
    kp = torch.empty(B, H, nkb, d, dtype=torch.float32, device=q.device)
    _call("sa_pool_blocks", _ptr(q), _ptr(k), B, H, N, d, bq, bk, _ptr(qp), _ptr(kp), _stream(q.device))
    return qp, kp


def sa_build_mask(q, k, bq, bk, topk, topp, scale=0.0, want_mask=False, want_pools=False,
                  workspace=None):
    B, H, N, d = _qkv(q, k)
    dev = q.device
    _on_device(dev, q=q, k=k)
    nqb, nkb = -(-N // bq), -(-N // bk)
    kv_idx = torch.empty(B, H, nqb, nkb, dtype=torch.int32, device=dev)
    kv_cnt = torch.empty(B, H, nqb, dtype=torch.int32, device=dev)
    mask = torch.empty(B, H, nqb, nkb, dtype=torch.uint8, device=dev) if want_mask else None
    qp = torch.empty(B, H, nqb, d, dtype=torch.float32, device=dev) if want_pools else None
    kp = torch.empty(B, H, nkb, d, dtype=torch.float32, device=dev) if want_pools else None
    ws = _workspace(load().sa_build_mask_workspace_size(B, H, N, d, bq, bk), dev, workspace)
    _call("sa_build_mask", _ptr(q), _ptr(k), B, H, N, d, bq, bk, float(topk), float(topp),
          float(scale), _ptr(kv_idx), _ptr(kv_cnt), _ptr(mask), _ptr(qp), _ptr(kp), _ptr(ws),
          ws.numel(), _stream(dev))
    out = {"kv_idx": kv_idx, "kv_cnt": kv_cnt}
    if want_mask:
        out["mask"] = mask
    if want_pools:
        out["q_pool"], out["k_pool"] = qp, kp
    return out


def sa_sparse_attn_fwd(q, k, v, bq, bk, kv_idx=None, kv_cnt=None, ext_mask=None, scale=0.0,
                       want_lse=False, out=None, workspace=None, o_l=None, alpha=None):
    """Sparse attention; with o_l and alpha (sa_sparse_attn_blend_fwd) the
    epilogue also blends O = alpha * O_s + (1 - alpha) * O_l."""
    B, H, N, d = _qkv(q, k, v)
    if (o_l is None) != (alpha is None):
        raise ValueError("o_l and alpha go together")
    if o_l is not None:
        _expect("o_l", o_l, q.shape, torch.bfloat16)
        _expect("alpha", alpha, (H, d), torch.float32)
        if out is not None and out.data_ptr() == o_l.data_ptr():
            raise ValueError("out must not alias o_l")
    nqb, nkb = -(-N // bq), -(-N // bk)
    if kv_idx is not None:
        _expect("kv_idx", kv_idx, (B, H, nqb, nkb), torch.int32)
    if kv_cnt is not None:
        _expect("kv_cnt", kv_cnt, (B, H, nqb), torch.int32)
    if ext_mask is not None:
        _expect("ext_mask", ext_mask, (B, H, nqb, nkb), (torch.uint8, torch.bool))
    if out is not None:
        _expect("out", out, q.shape, torch.bfloat16)
    dev = q.device
    _on_device(dev, q=q, k=k, v=v, kv_idx=kv_idx, kv_cnt=kv_cnt, ext_mask=ext_mask, out=out,
               o_l=o_l, alpha=alpha)
    o = out if out is not None else torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev) if want_lse else None
    need = load().sa_sparse_attn_workspace_size(B, H, N, d, bq, bk, int(ext_mask is not None))
    ws = _workspace(need, dev, workspace) if need else None
    common = (_ptr(q), _ptr(k), _ptr(v), B, H, N, d, bq, bk, _ptr(kv_idx), _ptr(kv_cnt),
              _ptr(ext_mask), float(scale))
    tail = (_ptr(lse), _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev))
    if o_l is None:
        _call("sa_sparse_attn_fwd", *common, _ptr(o), *tail)
    else:
        _call("sa_sparse_attn_blend_fwd", *common, _ptr(o_l), _ptr(alpha), _ptr(o), *tail)
    return (o, lse) if want_lse else o


_FP8 = (torch.float8_e4m3fn, torch.uint8)


def sa_quantize_fp8(x, out=None, scale_out=None):
    """Per-(batch, head) E4M3 quantisation of a [B, H, N, d] bf16 tensor:
    returns (codes [B, H, N, d] float8_e4m3fn, scale [B, H] fp32) with
    x ~ codes * scale."""
    B, H, N, d = _qkv(x, names=("x",))
    dev = x.device
    x8 = out if out is not None else torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=dev)
    _expect("out", x8, x.shape, _FP8)
    sc = scale_out if scale_out is not None else torch.empty(B, H, dtype=torch.float32, device=dev)
    _expect("scale_out", sc, (B, H), torch.float32)
    _on_device(dev, x=x, out=x8, scale_out=sc)
    _call("sa_quantize_fp8", _ptr(x), B, H, N, d, _ptr(x8), _ptr(sc), _stream(dev))
    return x8, sc


def sa_sparse_attn_fp8_fwd(q8, k8, v8, q_scale, k_scale, v_scale, bq, bk, kv_idx=None, kv_cnt=None,
                           ext_mask=None, scale=0.0, want_lse=False, out=None, workspace=None, o_l=None,
                           alpha=None):
    """Sparse attention on E4M3 inputs (codes as float8_e4m3fn or uint8, one
    fp32 scale per (batch, head) each, as sa_quantize_fp8 returns them); with
    o_l and alpha the epilogue also blends the linear branch. d = 128."""
    if q8 is None or q8.dim() != 4:
        raise ValueError("q8 must be a [B, H, N, d] tensor")
    B, H, N, d = q8.shape
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _expect(name, t, q8.shape, _FP8)
    for name, t in (("q_scale", q_scale), ("k_scale", k_scale), ("v_scale", v_scale)):
        _expect(name, t, (B, H), torch.float32)
    if (o_l is None) != (alpha is None):
        raise ValueError("o_l and alpha go together")
    if o_l is not None:
        _expect("o_l", o_l, q8.shape, torch.bfloat16)
        _expect("alpha", alpha, (H, d), torch.float32)
    nqb, nkb = -(-N // bq), -(-N // bk)
    if kv_idx is not None:
        _expect("kv_idx", kv_idx, (B, H, nqb, nkb), torch.int32)
    if kv_cnt is not None:
        _expect("kv_cnt", kv_cnt, (B, H, nqb), torch.int32)
    if ext_mask is not None:
        _expect("ext_mask", ext_mask, (B, H, nqb, nkb), (torch.uint8, torch.bool))
    if out is not None:
        _expect("out", out, q8.shape, torch.bfloat16)
        if o_l is not None and out.data_ptr() == o_l.data_ptr():
            raise ValueError("out must not alias o_l")
    dev = q8.device
    _on_device(dev, q8=q8, k8=k8, v8=v8, q_scale=q_scale, k_scale=k_scale, v_scale=v_scale, kv_idx=kv_idx,
               kv_cnt=kv_cnt, ext_mask=ext_mask, out=out, o_l=o_l, alpha=alpha)
    o = out if out is not None else torch.empty(q8.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev) if want_lse else None
    need = load().sa_sparse_attn_workspace_size(B, H, N, d, bq, bk, int(ext_mask is not None))
    ws = _workspace(need, dev, workspace) if need else None
    _call("sa_sparse_attn_fp8_fwd", _ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
          B, H, N, d, bq, bk, _ptr(kv_idx), _ptr(kv_cnt), _ptr(ext_mask), float(scale), _ptr(o_l), _ptr(alpha),
          _ptr(o), _ptr(lse), _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev))
    return (o, lse) if want_lse else o


def sa_dense_attn_fwd(q, k, v, bq=128, scale=0.0, want_lse=False, out=None):
    B, H, N, d = _qkv(q, k, v)
    if out is not None:
        _expect("out", out, q.shape, torch.bfloat16)
    _on_device(q.device, q=q, k=k, v=v, out=out)
    o = out if out is not None else torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device) if want_lse else None
    _call("sa_dense_attn_fwd", _ptr(q), _ptr(k), _ptr(v), B, H, N, d, bq, float(scale), _ptr(o),
          _ptr(lse), _stream(q.device))
    return (o, lse) if want_lse else o


def sa_linear_branch(q, k, v, want_ol=False, workspace=None, out_ol=None):
    if want_ol:
        B, H, N, d = _qkv(q, k, v)
    else:
        B, H, N, d = _qkv(k, v, names=("k", "v"))
        q = None            # read only for O_l
    dev = k.device
    _on_device(dev, q=q, k=k, v=v)
    S = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    z = torch.empty(B, H, d, dtype=torch.float32, device=dev)
    if out_ol is not None:
        _expect("out_ol", out_ol, k.shape, torch.bfloat16)
        _on_device(dev, out_ol=out_ol)
    o_l = (out_ol if out_ol is not None else torch.empty_like(k)) if want_ol else None
    ws = _workspace(load().sa_linear_workspace_size(B, H, N, d), dev, workspace)
    _call("sa_linear_branch", _ptr(q), _ptr(k), _ptr(v), B, H, N, d, _ptr(S), _ptr(z), _ptr(o_l),
          _ptr(ws), ws.numel(), _stream(dev))
    return (S, z, o_l) if want_ol else (S, z)


def sa_blend(o_s, q, kv_state, ksum, alpha, out=None, workspace=None):
    B, H, N, d = _qkv(o_s, q, names=("o_s", "q"))
    _expect("kv_state", kv_state, (B, H, d, d), torch.float32)
    _expect("ksum", ksum, (B, H, d), torch.float32)
    _expect("alpha", alpha, (H, d), torch.float32)
    if out is not None:
        _expect("out", out, o_s.shape, torch.bfloat16)
    dev = q.device
    _on_device(dev, o_s=o_s, q=q, kv_state=kv_state, ksum=ksum, alpha=alpha, out=out)
    o = out if out is not None else torch.empty_like(o_s)
    need = load().sa_blend_workspace_size(B, H, N, d)
    ws = _workspace(need, dev, workspace) if need else None
    _call("sa_blend", _ptr(o_s), _ptr(q), _ptr(kv_state), _ptr(ksum), _ptr(alpha), B, H, N, d,
          _ptr(o), _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev))
    return o


def sa_trip_pool(q, k, bq, bk):
    """TripPool descriptors [mean | max | min] of the query and key blocks."""
    B, H, N, d = _qkv(q, k, names=("q", "k"))
    _on_device(q.device, q=q, k=k)
    qd = torch.empty(B, H, -(-N // bq), 3 * d, dtype=torch.float32, device=q.device)
    kd = torch.empty(B, H, -(-N // bk), 3 * d, dtype=torch.float32, device=q.device)
    _call("sa_trip_pool", _ptr(q), _ptr(k), B, H, N, d, bq, bk, _ptr(qd), _ptr(kd), _stream(q.device))
    return qd, kd


def sa_tile_heatmap(q, k, bq, bk=64, scale=0.0, rows=None, want_lse=False, out=None):
    """Max-pooled full-attention heatmap (natural log) of every (query block,
    key block) tile; with `rows` (int32 query-block rows) only those rows are
    evaluated and the others of `out` are left as they were."""
    B, H, N, d = _qkv(q, k, names=("q", "k"))
    nqb, nkb = -(-N // bq), -(-N // bk)
    if rows is not None:
        if rows.dtype != torch.int32 or rows.dim() != 1 or not rows.is_contiguous():
            raise ValueError("rows: contiguous 1-D int32 tensor of query-block rows")
    if out is not None:
        _expect("out", out, (B, H, nqb, nkb), torch.float32)
    dev = q.device
    _on_device(dev, q=q, k=k, rows=rows, out=out)
    heat = out if out is not None else torch.full((B, H, nqb, nkb), float("nan"), dtype=torch.float32, device=dev)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev) if want_lse else None
    _call("sa_tile_heatmap", _ptr(q), _ptr(k), B, H, N, d, bq, bk, float(scale), _ptr(rows),
          0 if rows is None else rows.numel(), _ptr(heat), _ptr(lse), _stream(dev))
    return (heat, lse) if want_lse else heat


def sa_select_mask(scores, topk, topp, want_mask=False):
    """Hybrid Top-k ∪ Top-p selection from given block scores [B, H, n_qb, n_kb]."""
    if scores.dim() != 4:
        raise ValueError("scores must be [B, H, n_qb, n_kb]")
    B, H, nqb, nkb = scores.shape
    _expect("scores", scores, scores.shape, torch.float32)
    dev = scores.device
    _on_device(dev, scores=scores)
    kv_idx = torch.empty(B, H, nqb, nkb, dtype=torch.int32, device=dev)
    kv_cnt = torch.empty(B, H, nqb, dtype=torch.int32, device=dev)
    mask = torch.empty(B, H, nqb, nkb, dtype=torch.uint8, device=dev) if want_mask else None
    _call("sa_select_mask", _ptr(scores), B, H, nqb, nkb, float(topk), float(topp), _ptr(kv_idx),
          _ptr(kv_cnt), _ptr(mask), _stream(dev))
    out = {"kv_idx": kv_idx, "kv_cnt": kv_cnt}
    if want_mask:
        out["mask"] = mask
    return out


def sa_tile_permutation(grid, tiles, device=None):
    """[H, N] int32 tile-major token orders of a (T, Hh, W) grid, one tiling
    (p_t, p_h, p_w) per head."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    T, Hh, W = (int(g) for g in grid)
    flat = [int(v) for tile in tiles for v in tile]
    H = len(flat) // 3
    if H * 3 != len(flat) or H == 0:
        raise ValueError("tiles: one (p_t, p_h, p_w) triple per head")
    perm = torch.empty(H, T * Hh * W, dtype=torch.int32, device=device)
    arr = (ctypes.c_int32 * len(flat))(*flat)
    _call("sa_tile_permutation", H, T, Hh, W, ctypes.cast(arr, c_void_p), _ptr(perm), _stream(device))
    return perm


def sa_permute_tokens(x, perm, inverse=False, out=None):
    """Rows of x [B, H, N, d] in each head's order (or back, with inverse)."""
    B, H, N, d = _qkv(x, names=("x",))
    _expect("perm", perm, (H, N), torch.int32)
    if out is not None:
        _expect("out", out, x.shape, torch.bfloat16)
    _on_device(x.device, x=x, perm=perm, out=out)
    y = out if out is not None else torch.empty_like(x)
    _call("sa_permute_tokens", _ptr(x), _ptr(perm), B, H, N, d, int(bool(inverse)), _ptr(y), _stream(x.device))
    return y


def sa_sparse_attn_bwd(q, k, v, o, lse, dout, bq, bk, kv_idx, kv_cnt, scale=0.0):
    """(dq, dk, dv) fp32 of the sparse attention for the upstream gradient dout."""
    B, H, N, d = _qkv(q, k, v, o, dout, names=("q", "k", "v", "o", "dout"))
    nqb, nkb = -(-N // bq), -(-N // bk)
    _expect("lse", lse, (B, H, N), torch.float32)
    _expect("kv_idx", kv_idx, (B, H, nqb, nkb), torch.int32)
    _expect("kv_cnt", kv_cnt, (B, H, nqb), torch.int32)
    dev = q.device
    _on_device(dev, q=q, k=k, v=v, o=o, lse=lse, dout=dout, kv_idx=kv_idx, kv_cnt=kv_cnt)
    dq, dk, dv = (torch.empty(B, H, N, d, dtype=torch.float32, device=dev) for _ in range(3))
    ws = _workspace(load().sa_sparse_attn_bwd_workspace_size(B, H, N, d, bq, bk), dev)
    _call("sa_sparse_attn_bwd", _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), B, H, N, d, bq, bk,
          _ptr(kv_idx), _ptr(kv_cnt), float(scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(), _stream(dev))
    return dq, dk, dv


def sa_linear_bwd(q, k, v, kv_state, ksum, dout_l, grads=None):
    """(dq, dk, dv) fp32 of the linear branch; with grads=(dq, dk, dv) it adds into them."""
    B, H, N, d = _qkv(q, k, v, dout_l, names=("q", "k", "v", "dout_l"))
    _expect("kv_state", kv_state, (B, H, d, d), torch.float32)
    _expect("ksum", ksum, (B, H, d), torch.float32)
    dev = q.device
    _on_device(dev, q=q, k=k, v=v, kv_state=kv_state, ksum=ksum, dout_l=dout_l)
    if grads is None:
        grads = tuple(torch.empty(B, H, N, d, dtype=torch.float32, device=dev) for _ in range(3))
        acc = 0
    else:
        for name, t in zip(("dq", "dk", "dv"), grads):
            _expect(name, t, (B, H, N, d), torch.float32)
        acc = 1
    ws = _workspace(load().sa_linear_bwd_workspace_size(B, H, N, d), dev)
    _call("sa_linear_bwd", _ptr(q), _ptr(k), _ptr(v), _ptr(kv_state), _ptr(ksum), _ptr(dout_l), B, H, N, d, acc,
          *(_ptr(t) for t in grads), _ptr(ws), ws.numel(), _stream(dev))
    return grads


def sa_blend_bwd(o_s, o_l, alpha, dout):
    """(do_s, do_l, dalpha) of O = alpha * o_s + (1 - alpha) * o_l."""
    B, H, N, d = _qkv(o_s, o_l, dout, names=("o_s", "o_l", "dout"))
    _expect("alpha", alpha, (H, d), torch.float32)
    dev = o_s.device
    _on_device(dev, o_s=o_s, o_l=o_l, alpha=alpha, dout=dout)
    do_s, do_l = torch.empty_like(o_s), torch.empty_like(o_s)
    da = torch.empty(H, d, dtype=torch.float32, device=dev)
    ws = _workspace(load().sa_blend_bwd_workspace_size(B, H, N, d), dev)
    _call("sa_blend_bwd", _ptr(o_s), _ptr(o_l), _ptr(alpha), _ptr(dout), B, H, N, d, _ptr(do_s), _ptr(do_l),
          _ptr(da), _ptr(ws), ws.numel(), _stream(dev))
    return do_s, do_l, da


def _path_on_device(q, k, v, bq, bk, topk, topp, alpha, scale, out=None):
    m = sa_build_mask(q, k, bq, bk, topk, topp, scale)
    if alpha is None:
        return sa_sparse_attn_fwd(q, k, v, bq, bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"], scale=scale, out=out)
    # linear branch first, then the sparse attention blends it in its epilogue
    _, _, o_l = sa_linear_branch(q, k, v, want_ol=True)
    return sa_sparse_attn_fwd(q, k, v, bq, bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"], scale=scale,
                              out=out, o_l=o_l, alpha=alpha)


def block_sparse_attention(q, k, v, bq=128, bk=64, topk=0.05, topp=0.9, alpha=None, scale=0.0,
                           device=None, out=None, chunks=8, perm=None):
    """Whole path: mask, sparse attention and (when alpha is given) the linear
    branch blended in. Device tensors stay on the device. Host tensors are
    copied in, and the result is copied back into `out` (a pinned host tensor
    is allocated when out is None). Every head is independent, so with host
    tensors the heads are split into up to `chunks` groups that go through a
    three-stream pipeline: the copy in of group c + 1, the path on group c and
    the copy out of group c - 1 overlap. Pinned host tensors make the copies
    asynchronous. With `perm` ([H, N] int32 device orders, e.g. from
    sa_tile_permutation; device tensors only) the tokens are gathered into
    each head's order, the path runs on the permuted sequence and the output
    is scattered back."""
    if perm is not None:
        if not q.is_cuda:
            raise ValueError("perm: the permuted path takes device tensors")
        qp, kp, vp = (sa_permute_tokens(t, perm) for t in (q, k, v))
        op = _path_on_device(qp, kp, vp, bq, bk, topk, topp, alpha, scale)
        return sa_permute_tokens(op, perm, inverse=True, out=out)
    if q.is_cuda:
        return _path_on_device(q, k, v, bq, bk, topk, topp, alpha, scale, out)
    B, H, N, d = _qkv(q, k, v)
    for name, t in (("k", k), ("v", v), ("out", out)):
        if t is not None and t.is_cuda:
            raise ValueError(f"{name} is a CUDA tensor while q is on the host")
    if alpha is not None:
        _expect("alpha", alpha, (H, d), torch.float32)
    if out is not None:
        _expect("out", out, q.shape, torch.bfloat16)
    device = device or torch.device("cuda", torch.cuda.current_device())
    BH = B * H
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    qh, kh, vh, oh = (t.reshape(BH, N, d) for t in (q, k, v, out))
    dq, dk, dv = (torch.empty((BH, N, d), dtype=t.dtype, device=device) for t in (q, k, v))
    do = torch.empty((BH, N, d), dtype=q.dtype, device=device)
    if alpha is not None:
        # alpha row of each flattened (batch, head)
        alpha_d = alpha.to(device)[torch.arange(BH, device=device) % H].contiguous()
    n = max(1, min(int(chunks), BH))
    per = (BH + n - 1) // n
    caller = torch.cuda.current_stream(device)
    s_in, s_run, s_out = (torch.cuda.Stream(device) for _ in range(3))
    for s in (s_in, s_run, s_out):
        s.wait_stream(caller)
    for c in range(n):
        i0, i1 = c * per, min(BH, (c + 1) * per)
        if i0 >= i1:
            break
        with torch.cuda.stream(s_in):
            for dst, src in ((dq, qh), (dk, kh), (dv, vh)):
                dst[i0:i1].copy_(src[i0:i1], non_blocking=True)
        s_run.wait_stream(s_in)
        with torch.cuda.stream(s_run):
            view = lambda t: t[i0:i1].view(1, i1 - i0, N, d)
            _path_on_device(view(dq), view(dk), view(dv), bq, bk, topk, topp,
                            None if alpha is None else alpha_d[i0:i1], scale, out=view(do))
        s_out.wait_stream(s_run)
        with torch.cuda.stream(s_out):
            oh[i0:i1].copy_(do[i0:i1], non_blocking=True)
    # the device buffers were used on the side streams; keep the allocator from
    # handing them out again before those streams are done with them
    for t in (dq, dk, dv, do):
        t.record_stream(s_in)
        t.record_stream(s_run)
        t.record_stream(s_out)
    caller.wait_stream(s_out)
    caller.synchronize()
    return out
