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
    "sa_dense_attn_fwd": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                  c_int, c_double, c_void_p, c_void_p, c_void_p]),
    "sa_linear_workspace_size": (c_size_t, [c_int] * 4),
    "sa_linear_branch": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "sa_blend_workspace_size": (c_size_t, [c_int] * 4),
    "sa_blend": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                         c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
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


def _check_qkv(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("libsa takes CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("libsa takes contiguous tensors")
    return ts[0].shape


def _workspace(nbytes, device):
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def sa_version() -> int:
    return load().sa_version()


def sa_status_string(status: int) -> str:
    return load().sa_status_string(status).decode()


def sa_device_status(device=None):
    device = device or torch.device("cuda", torch.cuda.current_device())
    _call("sa_device_status", _stream(device))


def sa_pool_blocks(q, k, bq, bk):
    B, H, N, d = _check_qkv(q, k)
    nqb, nkb = -(-N // bq), -(-N // bk)
    qp = torch.empty(B, H, nqb, d, dtype=torch.float32, device=q.device)
    kp = torch.empty(B, H, nkb, d, dtype=torch.float32, device=q.device)
    _call("sa_pool_blocks", _ptr(q), _ptr(k), B, H, N, d, bq, bk, _ptr(qp), _ptr(kp), _stream(q.device))
    return qp, kp


def sa_build_mask(q, k, bq, bk, topk, topp, scale=0.0, want_mask=False, want_pools=False,
                  workspace=None):
    B, H, N, d = _check_qkv(q, k)
    nqb, nkb = -(-N // bq), -(-N // bk)
    dev = q.device
    kv_idx = torch.empty(B, H, nqb, nkb, dtype=torch.int32, device=dev)
    kv_cnt = torch.empty(B, H, nqb, dtype=torch.int32, device=dev)
    mask = torch.empty(B, H, nqb, nkb, dtype=torch.uint8, device=dev) if want_mask else None
    qp = torch.empty(B, H, nqb, d, dtype=torch.float32, device=dev) if want_pools else None
    kp = torch.empty(B, H, nkb, d, dtype=torch.float32, device=dev) if want_pools else None
    need = load().sa_build_mask_workspace_size(B, H, N, d, bq, bk)
    ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
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
                       want_lse=False, out=None, workspace=None):
    B, H, N, d = _check_qkv(q, k, v)
    dev = q.device
    o = out if out is not None else torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev) if want_lse else None
    need = load().sa_sparse_attn_workspace_size(B, H, N, d, bq, bk, int(ext_mask is not None))
    ws = None
    if need:
        ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
    _call("sa_sparse_attn_fwd", _ptr(q), _ptr(k), _ptr(v), B, H, N, d, bq, bk, _ptr(kv_idx),
          _ptr(kv_cnt), _ptr(ext_mask), float(scale), _ptr(o), _ptr(lse), _ptr(ws),
          0 if ws is None else ws.numel(), _stream(dev))
    return (o, lse) if want_lse else o


def sa_dense_attn_fwd(q, k, v, bq=128, scale=0.0, want_lse=False, out=None):
    B, H, N, d = _check_qkv(q, k, v)
    o = out if out is not None else torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device) if want_lse else None
    _call("sa_dense_attn_fwd", _ptr(q), _ptr(k), _ptr(v), B, H, N, d, bq, float(scale), _ptr(o),
          _ptr(lse), _stream(q.device))
    return (o, lse) if want_lse else o


def sa_linear_branch(q, k, v, want_ol=False, workspace=None):
    B, H, N, d = _check_qkv(k, v)
    dev = k.device
    S = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    z = torch.empty(B, H, d, dtype=torch.float32, device=dev)
    o_l = torch.empty_like(k) if want_ol else None
    need = load().sa_linear_workspace_size(B, H, N, d)
    ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
    _call("sa_linear_branch", _ptr(q), _ptr(k), _ptr(v), B, H, N, d, _ptr(S), _ptr(z), _ptr(o_l),
          _ptr(ws), ws.numel(), _stream(dev))
    return (S, z, o_l) if want_ol else (S, z)


def sa_blend(o_s, q, kv_state, ksum, alpha, out=None, workspace=None):
    B, H, N, d = _check_qkv(o_s, q, kv_state, ksum, alpha)
    dev = q.device
    o = out if out is not None else torch.empty_like(o_s)
    need = load().sa_blend_workspace_size(B, H, N, d)
    ws = None
    if need:
        ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
    _call("sa_blend", _ptr(o_s), _ptr(q), _ptr(kv_state), _ptr(ksum), _ptr(alpha), B, H, N, d,
          _ptr(o), _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev))
    return o


def _path_on_device(q, k, v, bq, bk, topk, topp, alpha, scale, out=None):
    m = sa_build_mask(q, k, bq, bk, topk, topp, scale)
    o = sa_sparse_attn_fwd(q, k, v, bq, bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"], scale=scale, out=out)
    if alpha is not None:
        S, z = sa_linear_branch(q, k, v)
        o = sa_blend(o, q, S, z, alpha, out=o)
    return o


def block_sparse_attention(q, k, v, bq=128, bk=64, topk=0.05, topp=0.9, alpha=None, scale=0.0,
                           device=None, out=None, chunks=8):
    """Whole path: mask, sparse attention and (when alpha is given) the linear
    branch blended in. Device tensors stay on the device. Host tensors are
    copied in, and the result is copied back into `out` (a pinned host tensor
    is allocated when out is None). Every head is independent, so with host
    tensors the heads are split into up to `chunks` groups that go through a
    three-stream pipeline: the copy in of group c + 1, the path on group c and
    the copy out of group c - 1 overlap. Pinned host tensors make the copies
    asynchronous."""
    if q.is_cuda:
        return _path_on_device(q, k, v, bq, bk, topk, topp, alpha, scale, out)
    device = device or torch.device("cuda", torch.cuda.current_device())
    B, H, N, d = q.shape
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
