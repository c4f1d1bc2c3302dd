"""GPU parity of la2_dlambda (the gradient in the decay) against the fp64
oracle's dlambda, summed over the batch, through the C ABI.

The result is one scalar per head: max|gpu - oracle| / rms(oracle over heads)
<= 2e-2 for bf16 inputs and 1e-5 for fp32 inputs, with and without carried
states, on ragged lengths around the 32-row sub-tile, every (d, e) shape class,
few-sequence shapes cut into segments, both layouts, decays from 2^-20 to 1,
and the full-size TNL-15B and long-context workloads.
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


def _state(B, H, d, e, seed, scale=0.5):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(B, H, d, e, generator=g, dtype=torch.float32) * scale


def _gpu(la2mod, x, s0=None, g=None, layout="bhtd"):
    dev = torch.device("cuda")
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    if layout == "bthd":
        q, k, v, do = (t.transpose(1, 2).contiguous() for t in (q, k, v, do))
    lam = x["lam"].to(dev)
    out = torch.full(lam.shape, float("nan"), device=dev)
    la2mod.la2_dlambda(q, k, v, lam, do, None if s0 is None else s0.to(dev),
                       None if g is None else g.to(dev), layout, d_decay=out)
    torch.cuda.synchronize()
    assert la2mod.la2_device_status(reset=True) == 0
    return out.cpu().double().numpy()


def _ref(oracle_mod, x, s0=None, g=None):
    B, H = x["q"].shape[:2]
    lam = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :], (B, H))
    per = oracle_mod.dlambda(x["q"], x["k"], x["v"], lam, x["do"],
                             None if s0 is None else s0.numpy().astype(np.float64),
                             None if g is None else g.numpy().astype(np.float64))
    return per.sum(axis=0)


def _check(la2mod, oracle_mod, x, tol, s0=None, g=None, layout="bhtd"):
    got = _gpu(la2mod, x, s0, g, layout)
    want = _ref(oracle_mod, x, s0, g)
    assert np.all(np.isfinite(got))
    if not np.any(want):  # no pair s < t and no state: exactly zero
        assert not np.any(got), got
        return 0.0
    err = float(np.max(np.abs(got - want)) / np.sqrt(np.mean(want * want)))
    assert err <= tol, (err, got, want)
    return err


@pytest.mark.parametrize("T", [1, 2, 31, 32, 33, 300, 1000])
@pytest.mark.parametrize("dtype,d,e", [("bf16", 128, 128), ("bf16", 64, 64), ("bf16", 64, 128),
                                       ("f32", 64, 64), ("f32", 3, 5), ("f32", 100, 37)])
def test_dlambda_shapes(la2mod, oracle_mod, T, dtype, d, e):
    x = I.make_inputs(2, 3, T, d, e, dtype, seed=T + d + 7 * e)
    _check(la2mod, oracle_mod, x, TOL[dtype])


@pytest.mark.parametrize("dtype,d,e", [("bf16", 128, 128), ("f32", 64, 32)])
def test_dlambda_with_states(la2mod, oracle_mod, dtype, d, e):
    x = I.make_inputs(2, 4, 517, d, e, dtype, seed=3)
    s0, g = _state(2, 4, d, e, 1), _state(2, 4, d, e, 2)
    _check(la2mod, oracle_mod, x, TOL[dtype], s0, g)
    _check(la2mod, oracle_mod, x, TOL[dtype], s0, None)
    _check(la2mod, oracle_mod, x, TOL[dtype], None, g)


@pytest.mark.parametrize("T", [4000, 4100, 9999])
def test_dlambda_segmented(la2mod, oracle_mod, T):
    """One or two sequences: each cut into up to 32 segments with a pre-pass."""
    x = I.make_inputs(1, 2, T, 128, 128, "bf16", seed=T)
    _check(la2mod, oracle_mod, x, TOL["bf16"], _state(1, 2, 128, 128, 4), _state(1, 2, 128, 128, 5))
    xf = I.make_inputs(1, 1, T, 32, 16, "f32", seed=T)
    _check(la2mod, oracle_mod, xf, TOL["f32"])


def test_dlambda_decays(la2mod, oracle_mod):
    x = I.make_inputs(2, 5, 700, 64, 64, "bf16", seed=11)
    x["lam"] = torch.tensor([2.0 ** -20, 0.3, 0.9, 0.999, 1.0], dtype=torch.float32)
    _check(la2mod, oracle_mod, x, TOL["bf16"])


def test_dlambda_layouts_agree_bitwise_and_repeat(la2mod, oracle_mod):
    x = I.make_inputs(2, 3, 333, 128, 64, "bf16", seed=12)
    a = _gpu(la2mod, x)
    b = _gpu(la2mod, x, layout="bthd")
    c = _gpu(la2mod, x)
    assert np.array_equal(a, b) and np.array_equal(a, c)


def test_dlambda_empty_is_zero(la2mod):
    dev = torch.device("cuda")
    q = torch.zeros(2, 3, 0, 64, dtype=torch.bfloat16, device=dev)
    lam = torch.full((3,), 0.9, device=dev)
    out = la2mod.la2_dlambda(q, q, q, lam, q, d_decay=torch.full((3,), 5.0, device=dev))
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0


@pytest.mark.parametrize("name", ["tnl15b", "long"])
def test_dlambda_full_size(la2mod, oracle_mod, name):
    w = I.WORKLOADS[name]
    x = I.make_workload_inputs(w, seed=0)
    _check(la2mod, oracle_mod, x, TOL[w.dtype])
