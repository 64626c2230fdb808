"""sa_build_mask_noalloc: the mask builder for callers that may not allocate
device memory when they call in (its scratch is a fixed array inside the
library). Called through the C ABI and checked against sa_build_mask on the
same inputs, on two calls in a row that reuse the shared scratch.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from block_sparse_attention_softmax_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def _noalloc(lib, q, k, bq, bk, topk, topp, with_mask):
    B, H, N, d = q.shape
    nqb, nkb = -(-N // bq), -(-N // bk)
    idx = torch.full((B, H, nqb, nkb), -7, dtype=torch.int32, device=q.device)
    cnt = torch.full((B, H, nqb), -7, dtype=torch.int32, device=q.device)
    mask = torch.full((B, H, nqb, nkb), 9, dtype=torch.uint8, device=q.device) if with_mask else None
    stream = P(torch.cuda.current_stream().cuda_stream)
    rc = lib.sa_build_mask_noalloc(P(q.data_ptr()), P(k.data_ptr()), B, H, N, d, bq, bk,
                                   float(topk), float(topp), 0.0, P(idx.data_ptr()),
                                   P(cnt.data_ptr()), P(mask.data_ptr()) if with_mask else None,
                                   stream)
    assert rc == 0, lib.sa_last_error().decode()
    return idx, cnt, mask


def _same_lists(ref, idx, cnt):
    assert torch.equal(ref["kv_cnt"], cnt)
    nkb = idx.shape[-1]
    keep = torch.arange(nkb, device=idx.device) < cnt.unsqueeze(-1)
    assert torch.equal(torch.where(keep, ref["kv_idx"], 0), torch.where(keep, idx, 0))


def test_noalloc_matches_workspace_mask_builder_on_two_calls(cuda_lib):
    sa = cuda_lib
    lib = sa.load()
    dev = torch.device("cuda", 0)
    # call 1: the tiny workload; call 2: a larger one that reuses (and
    # overwrites) the scratch left by call 1
    for name, with_mask in (("tiny", True), ("wan13b_480p", False)):
        wl = WORKLOADS[name]
        x = make_inputs(wl, dev)
        q, k = x["q"], x["k"]
        idx, cnt, mask = _noalloc(lib, q, k, wl.bq, wl.bk, wl.topk, wl.topp, with_mask)
        ref = sa.sa_build_mask(q, k, wl.bq, wl.bk, wl.topk, wl.topp, want_mask=with_mask)
        torch.cuda.synchronize()
        _same_lists(ref, idx, cnt)
        if with_mask:
            assert torch.equal(ref["mask"], mask)
    sa.sa_device_status(dev)


def test_noalloc_rejects_problems_above_the_fixed_scratch(cuda_lib):
    lib = cuda_lib.load()
    wl = WORKLOADS["wan14b_720p"]    # ~121 MB of scratch
    fake = P(0x1000)                 # never dereferenced: the size check comes first
    rc = lib.sa_build_mask_noalloc(fake, fake, wl.B, wl.H, wl.N, wl.d, wl.bq, wl.bk, wl.topk,
                                   wl.topp, 0.0, fake, fake, None, None)
    assert rc == -2
    assert b"fixed scratch" in lib.sa_last_error()


def test_noalloc_call_allocates_no_device_memory(cuda_lib):
    """After a first call (which looks up the fixed scratch), a further call
    with its outputs already allocated leaves the device's free memory as it
    was: the entry point draws on no allocator."""
    sa = cuda_lib
    lib = sa.load()
    dev = torch.device("cuda", 0)
    wl = WORKLOADS["wan13b_480p"]
    x = make_inputs(wl, dev)
    q, k = x["q"], x["k"]
    B, H, N, d = q.shape
    nqb, nkb = -(-N // wl.bq), -(-N // wl.bk)
    idx = torch.empty((B, H, nqb, nkb), dtype=torch.int32, device=dev)
    cnt = torch.empty((B, H, nqb), dtype=torch.int32, device=dev)
    stream = P(torch.cuda.current_stream().cuda_stream)
    args = (P(q.data_ptr()), P(k.data_ptr()), B, H, N, d, wl.bq, wl.bk, float(wl.topk), float(wl.topp),
            0.0, P(idx.data_ptr()), P(cnt.data_ptr()), None, stream)
    assert lib.sa_build_mask_noalloc(*args) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info(dev)
    assert lib.sa_build_mask_noalloc(*args) == 0, lib.sa_last_error().decode()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(dev)
    assert free0 == free1
    sa.sa_device_status(dev)


def test_noalloc_candidate_builder_on_the_shared_array(cuda_lib, monkeypatch):
    """The candidate builder (forced on shapes the size rule would send to the
    score-matrix builder) keeps its per-row statistics, candidate counts and
    hand-back state in the same fixed array; two calls in a row against
    sa_build_mask under the same setting."""
    sa = cuda_lib
    lib = sa.load()
    dev = torch.device("cuda", 0)
    monkeypatch.setenv("SA_MASK_BUILDER", "candidates")
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, dev)
    for q, k in ((x["q"], x["k"]), ((x["q"].float() * 3).to(torch.bfloat16), x["k"])):
        idx, cnt, mask = _noalloc(lib, q, k, wl.bq, wl.bk, wl.topk, wl.topp, True)
        ref = sa.sa_build_mask(q, k, wl.bq, wl.bk, wl.topk, wl.topp, want_mask=True)
        torch.cuda.synchronize()
        _same_lists(ref, idx, cnt)
        assert torch.equal(ref["mask"], mask)
    sa.sa_device_status(dev)
