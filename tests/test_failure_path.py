"""The bounded-wait failure path of the bf16 scan kernel, made to run out on
purpose without faulting, trapping or hanging the GPU.

la2_selftest_timeout launches the real forward kernel with its producer first
waiting on a device flag that nothing sets, bounded by a short limit.  The wait
runs out before any load; the kernel must record LA2_ERR_TIMEOUT with the
wait's site in the device status word, every role must leave through the abort
flag (the issuers still commit their final barrier, TMEM is freed), and the
next ordinary calls must run and match the oracle.
"""
import numpy as np
import pytest
import torch

from causal_linear_attention_la2_b200 import inputs as I

pytestmark = pytest.mark.gpu

SITE_HOLD = 90


@pytest.fixture(scope="module")
def la2mod():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_linear_attention_la2_b200 import build, la2
    build.build()
    la2.load()
    return la2


def _rel(gpu, ref):
    gpu = gpu.detach().double().cpu().numpy()
    return float(np.max(np.abs(gpu - ref)) / np.sqrt(np.mean(ref * ref)))


@pytest.mark.parametrize("d,e", [(128, 128), (64, 64), (128, 64)])
def test_wait_runs_out_reports_timeout_and_gpu_keeps_working(la2mod, oracle_mod, d, e):
    la2 = la2mod
    dev = torch.device("cuda")
    assert la2.la2_device_status(reset=True) == 0
    x = I.make_inputs(1, 1, 200, d, e, "bf16", seed=31)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    lam = x["lam"].to(dev)
    out = torch.full((1, 1, 200, e), 7.0, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    st = la2.la2_selftest_timeout_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), lam.data_ptr(),
                                      out.data_ptr(), 200, d, e, 20000, stream)
    assert st == la2.LA2_OK, la2.la2_status_str(st)
    torch.cuda.synchronize()
    code = la2.la2_device_status(reset=True)
    assert code & 0xFF == la2.LA2_ERR_TIMEOUT, hex(code)
    assert code >> 8 == SITE_HOLD, hex(code)
    assert torch.all(out == 7.0), "the aborted kernel must not write its output"
    # the context is intact: ordinary calls run and are correct
    assert la2.la2_device_status(reset=True) == 0
    o = la2.la2_fwd(q, k, v, lam)
    torch.cuda.synchronize()
    assert la2.la2_device_status(reset=True) == 0
    ref = oracle_mod.forward(x["q"], x["k"], x["v"], x["lam"].numpy().astype(np.float64))
    assert _rel(o, ref) <= 2e-2

