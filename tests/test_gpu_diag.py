"""GPU checks of the error-reporting path and of the softmax's FMA-pipe
exponential, through the diagnostic entry points of the C ABI. Nothing here
faults or hangs the GPU: the timeout comes from a bounded wait on a barrier
that nothing arrives at, with a shortened limit, and the kernel returns."""
import numpy as np
import pytest
import torch

from block_sparse_attention_softmax_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _status_code(sa):
    try:
        sa.sa_device_status()
        return "SA_OK"
    except sa.SAError as e:
        return str(e).split()[2]


def test_device_status_reports_and_clears(cuda_lib):
    sa = cuda_lib
    assert _status_code(sa) == "SA_OK"
    sa.sa_diag_set_device_status(5)
    assert _status_code(sa) == "SA_ERR_DEVICE_TIMEOUT"
    assert _status_code(sa) == "SA_OK"                      # the read cleared it


def test_bounded_wait_runs_out_and_the_context_stays_usable(cuda_lib):
    sa = cuda_lib
    assert _status_code(sa) == "SA_OK"
    try:
        sa.sa_diag_set_wait_limit(200000)                   # ~0.1 ms
        done, abort = sa.sa_diag_wait_timeout()
    finally:
        sa.sa_diag_set_wait_limit(0)                        # back to the default bound
    assert (done, abort) == (0, 1)
    assert _status_code(sa) == "SA_ERR_DEVICE_TIMEOUT"
    assert _status_code(sa) == "SA_OK"
    # the library's kernels still run and report no error afterwards
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, "cpu")
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    m = sa.sa_build_mask(q, k, wl.bq, wl.bk, wl.topk, wl.topp)
    o = sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"])
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert _status_code(sa) == "SA_OK"


def test_fma_pipe_exp2_accuracy(cuda_lib):
    """The polynomial 2^x (magic-number rounding, cubic on [-1/2, 1/2]) against
    fp64 exp2 over [-130, 8], the range the softmax feeds it (its inputs are
    at most 8 above the running max): relative error <= 7.6e-5 from -125 up;
    below the clamp at -126 a value in [0, 2^-124]. ex2.approx for reference."""
    sa = cuda_lib
    xs = np.concatenate([np.linspace(-130.0, 8.0, 4_000_001),
                         np.arange(-130, 9, dtype=np.float64),            # integers
                         np.arange(-130, 8, dtype=np.float64) + 0.5,      # rounding ties
                         np.random.default_rng(0).uniform(-30, 8, 1_000_000)]).astype(np.float32)
    x = torch.from_numpy(xs).to(DEV)
    yp, ym = sa.sa_diag_exp2(x)
    torch.cuda.synchronize()
    yp, ym = yp.cpu().numpy().astype(np.float64), ym.cpu().numpy().astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    hi = xs >= -125.0
    rel = np.abs(yp[hi] - ref[hi]) / ref[hi]
    print(f"poly max rel err {rel.max():.3e}; ex2.approx {np.max(np.abs(ym[hi] - ref[hi]) / ref[hi]):.3e}")
    assert rel.max() <= 7.6e-5
    lo = xs < -125.0
    assert (yp[lo] >= 0).all() and (yp[lo] <= 2.0 ** -124).all()
    assert np.isfinite(yp).all()


def test_attention_wait_runs_out_on_the_tiny_workload(cuda_lib):
    """With the wait bound lowered to 100 cycles the attention kernel's waits
    for data run out: every role stops, the producers wait for the TMA loads
    they issued and the MMA threads for their MMAs, the two softmax warps of
    each pair stop at the same barrier, and the kernel returns. The status
    reports the timeout once; with the default bound restored the same call
    matches the oracle."""
    import oracle
    from gpu_helpers import assert_close
    sa = cuda_lib
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, "cpu")
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    m = sa.sa_build_mask(q, k, wl.bq, wl.bk, wl.topk, wl.topp, want_mask=True)
    torch.cuda.synchronize()
    assert _status_code(sa) == "SA_OK"
    try:
        sa.sa_diag_set_wait_limit(100)
        sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"])
        torch.cuda.synchronize()
    finally:
        sa.sa_diag_set_wait_limit(0)
    assert _status_code(sa) == "SA_ERR_DEVICE_TIMEOUT"
    assert _status_code(sa) == "SA_OK"
    o = sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"])
    torch.cuda.synchronize()
    assert _status_code(sa) == "SA_OK"
    f64 = oracle.as_f64
    for h in range(wl.H):
        ro, _ = oracle.masked_attention(f64(x["q"][0, h]), f64(x["k"][0, h]), f64(x["v"][0, h]),
                                        m["mask"][0, h].cpu().numpy().astype(bool), wl.bq, wl.bk)
        assert_close(o[0, h].float().cpu().numpy(), ro, f"O head {h} after the timeout")
