"""The allocation-free forward, la2_fwd_noalloc, against la2_fwd.

la2_fwd_noalloc serves callers that cannot allocate device memory when they
call (inside CUDA-graph capture, under a framework that owns all allocations):
its scratch, the per-segment states used when few sequences are cut into
segments, is an array built into the library instead of a caller workspace.
Here it is called through the C ABI twice in a row, on inputs that do need the
scratch, and each result is compared with la2_fwd's (which uses a workspace the
caller provides): within the bf16 tolerance of the parity tests, and bit for
bit, since both run the same kernels on the same launch plan.  This file is
collected last on purpose, and it runs the same alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from causal_linear_attention_la2_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def la2mod():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_linear_attention_la2_b200 import build, la2
    build.build()
    la2.load()
    return la2


def _rel_err(a: torch.Tensor, b: torch.Tensor) -> float:
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.max(np.abs(a - b)) / np.sqrt(np.mean(b * b)))


def _two_calls(la2, B, H, T, d, e):
    dev = torch.device("cuda")
    need = la2.la2_workspace_bytes(B, H, T, d, e, 128, la2.LA2_DTYPE_BF16, 0)
    assert need > 0, "this shape must use the scratch (few sequences cut into segments)"
    stream = torch.cuda.current_stream().cuda_stream
    for seed in (101, 202):  # second call: different data, the scratch holds the first call's
        x = I.make_inputs(B, H, T, d, e, "bf16", seed=seed)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        lam = x["lam"].to(dev)
        ref = la2.la2_fwd(q, k, v, lam)
        out = torch.full((B, H, T, e), float("nan"), dtype=torch.float32, device=dev)
        st = la2.la2_fwd_noalloc_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), lam.data_ptr(),
                                     out.data_ptr(), B, H, T, d, e, 128, la2.LA2_DTYPE_BF16, stream)
        assert st == la2.LA2_OK, la2.la2_status_str(st)
        torch.cuda.synchronize()
        assert la2.la2_device_status(reset=True) == 0
        assert torch.isfinite(out).all()
        assert _rel_err(out, ref) <= TOL_BF16
        # the same kernels on the same plan: the results must be identical bit for bit
        assert torch.equal(out, ref)


@pytest.mark.parametrize("B,H,T,d,e", [(1, 2, 4100, 128, 128), (1, 3, 2000, 64, 64)])
def test_noalloc_forward_matches_la2_fwd_on_two_calls(la2mod, B, H, T, d, e):
    _two_calls(la2mod, B, H, T, d, e)


def test_noalloc_forward_balanced_schedule_uses_the_last_slot(la2mod):
    """The balanced schedule at d = e = 128 with two sequences of 296 tiles:
    148 CTAs of 4 tiles, so the state pre-pass fills scratch slots 0 .. 146
    (all but the one at the sequence boundary), the largest need the built-in
    array is sized for."""
    la2 = la2mod
    B, H, T = 1, 2, 296 * 128
    prev = la2.la2_set_schedule("balanced")
    try:
        plan = la2.la2_plan_info(B, H, T, 128, 128)
        assert plan[0]["schedule"] == "balanced" and plan[0]["ctas"] == 148
        assert plan[0]["prepass_ctas"] == 147
        _two_calls(la2, B, H, T, 128, 128)
    finally:
        la2.la2_set_schedule(prev)
