"""The [B, T, H, D] layout (la2_fwd_ex / la2_bwd_ex with LA2_LAYOUT_BTHD)
against the [B, H, T, D] path and the fp64 oracle, through the C ABI.

The same tiles are computed in the same order whichever layout the tensors
have, so the results must equal the [B, H, T, D] results bit for bit; they are
also checked against the oracle with the bar of the other parity tests.
"""
import numpy as np
import pytest
import torch

from causal_linear_attention_la2_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}


@pytest.fixture(scope="module")
def la2mod():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_linear_attention_la2_b200 import build, la2
    build.build()
    la2.load()
    return la2


def _err(gpu, ref):
    gpu = gpu.detach().float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(gpu - ref))) / max(rms, 1e-300)


def _bthd(t):
    return t.transpose(1, 2).contiguous()


@pytest.mark.parametrize("dtype,T,d,e", [("bf16", 300, 64, 64), ("bf16", 129, 128, 128),
                                         ("bf16", 1000, 64, 128), ("bf16", 777, 128, 64),
                                         ("bf16", 4000, 64, 64), ("f32", 300, 64, 37)])
def test_bthd_equals_bhtd_and_oracle(la2mod, oracle_mod, dtype, T, d, e):
    dev = torch.device("cuda")
    B, H = (1, 2) if T >= 4000 else (2, 3)  # T = 4000 with two sequences: segmented
    x = I.make_inputs(B, H, T, d, e, dtype, seed=T + d)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    lam = x["lam"].to(dev)
    init = torch.randn(B, H, d, e, generator=torch.Generator().manual_seed(1)).to(dev)
    o, fin = la2mod.la2_fwd_ex(q, k, v, lam, "bhtd", init_state=init, want_final=True)
    g = la2mod.la2_bwd_ex(q, k, v, lam, do, "bhtd")
    ob, finb = la2mod.la2_fwd_ex(_bthd(q), _bthd(k), _bthd(v), lam, "bthd", init_state=init,
                                 want_final=True)
    gb = la2mod.la2_bwd_ex(_bthd(q), _bthd(k), _bthd(v), lam, _bthd(do), "bthd")
    torch.cuda.synchronize()
    assert la2mod.la2_device_status(reset=True) == 0
    assert torch.equal(ob, _bthd(o)) and torch.equal(finb, fin)
    for a, b in zip(gb, g):
        assert torch.equal(a, _bthd(b))
    lam64 = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :], (B, H))
    ro, rs = oracle_mod.forward_state(x["q"], x["k"], x["v"], lam64, init.cpu().numpy())
    rg = oracle_mod.backward(x["q"], x["k"], x["v"], lam64, x["do"])
    assert _err(o, ro) <= TOL[dtype] and _err(fin, rs) <= TOL[dtype]
    for a, r in zip(g, rg):
        assert _err(a, r) <= TOL[dtype]


def test_unknown_layout_is_rejected(la2mod):
    from causal_linear_attention_la2_b200.la2 import LA2_ERR_INVALID_ARG
    lib = la2mod.load()
    st = lib.la2_fwd_ex(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 0, 0, 1, 1, 8, 64, 64, 128, 1,
                        0, 7, 0, 0, 0)
    assert st == LA2_ERR_INVALID_ARG
