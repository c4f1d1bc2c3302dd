"""GPU parity of the two ways the bf16 kernels spread their work over CTAs
(la2_set_schedule), through the C ABI, against the fp64 oracle.

The balanced schedule lays the (sequence, role) units' tiles end to end and
gives every CTA the same run of them: a CTA then processes the end of one unit
and the start of the next, and segments start inside a unit with the state the
pre-pass hands them.  The shapes below make CTAs that run up to four pieces,
pieces of one tile, ragged last tiles in both scan directions, every (d, e), a
carried initial and final state, and the [B, T, H, D] layout.  Bar: the
parity tests' max|gpu - oracle| / rms(oracle) <= 2e-2 for bf16 inputs; the two
schedules also agree with each other far inside it.
"""
import numpy as np
import pytest
import torch

from causal_linear_attention_la2_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module")
def la2mod():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_linear_attention_la2_b200 import build, la2
    build.build()
    la2.load()
    return la2


@pytest.fixture
def schedule(la2mod, request):
    prev = la2mod.la2_set_schedule(request.param)
    yield request.param
    la2mod.la2_set_schedule(prev)


def _err(gpu, ref):
    gpu = gpu.detach().float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(gpu - ref))) / max(rms, 1e-300)


def _run(la2mod, x, init=None, layout="bhtd"):
    dev = torch.device("cuda")
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    lam = x["lam"].to(dev)
    if layout == "bthd":
        q, k, v, do = (t.transpose(1, 2).contiguous() for t in (q, k, v, do))
    B, H = x["q"].shape[:2]
    d, e = q.shape[-1], v.shape[-1]
    o, fin = la2mod.la2_fwd_ex(q, k, v, lam, layout=layout,
                               init_state=None if init is None else init.to(dev),
                               final_state=torch.full((B, H, d, e), float("nan"), device=dev))
    dq, dk, dv = la2mod.la2_bwd_ex(q, k, v, lam, do, layout=layout)
    torch.cuda.synchronize()
    assert la2mod.la2_device_status(reset=True) == 0
    outs = (o, dq, dk, dv)
    if layout == "bthd":
        outs = tuple(t.transpose(1, 2) for t in outs)
    return outs, fin


def _oracle(oracle_mod, x, init=None):
    B, H = x["q"].shape[:2]
    lam = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :], (B, H))
    s0 = None if init is None else init.numpy().astype(np.float64)
    ro, rs = oracle_mod.forward_state(x["q"], x["k"], x["v"], lam, s0)
    rdq, rdk, rdv = oracle_mod.backward(x["q"], x["k"], x["v"], lam, x["do"])
    return (ro, rdq, rdk, rdv), rs


# (B, H, T): units = B H (forward) and 3 B H (backward); tiles per unit ceil(T / 128)
SHAPES = [
    (1, 5, 2500),    # forward one tile per CTA; backward runs of 3 tiles over 20-tile units
    (4, 25, 300),    # 3-tile units, runs of 1 (forward) and 7 tiles (backward): up to 4 pieces
    (2, 3, 3000),    # 24-tile units
    (1, 1, 129),     # one unit of 2 tiles, the second holding one position
    (3, 50, 1000),   # 150 and 450 units of 8 tiles
]


@pytest.mark.parametrize("schedule", ["balanced", "uniform"], indirect=True)
@pytest.mark.parametrize("B,H,T", SHAPES)
@pytest.mark.parametrize("d,e", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_schedule_parity(la2mod, oracle_mod, schedule, B, H, T, d, e):
    if (d, e) != (64, 64) and B * H > 40:
        pytest.skip("one (d, e) covers the large unit counts")
    x = I.make_inputs(B, H, T, d, e, "bf16", seed=B * 1000 + H * 10 + T + d + e)
    g = torch.Generator().manual_seed(T)
    init = torch.randn(B, H, d, e, generator=g, dtype=torch.float32) * 0.5
    outs, fin = _run(la2mod, x, init)
    refs, rs = _oracle(oracle_mod, x, init)
    errs = {n: _err(o, r) for n, o, r in zip(("o", "dq", "dk", "dv"), outs, refs)}
    errs["final_state"] = _err(fin, rs)
    for n, o in zip(("o", "dq", "dk", "dv"), outs):
        assert torch.isfinite(o.float()).all(), n
    assert max(errs.values()) <= TOL, errs


@pytest.mark.parametrize("schedule", ["balanced"], indirect=True)
def test_balanced_bthd_layout(la2mod, oracle_mod, schedule):
    x = I.make_inputs(2, 6, 1500, 64, 64, "bf16", seed=77)
    outs, fin = _run(la2mod, x, None, layout="bthd")
    refs, rs = _oracle(oracle_mod, x, None)
    errs = [_err(o, r) for o, r in zip(outs, refs)] + [_err(fin, rs)]
    assert max(errs) <= TOL, errs


def test_balanced_and_uniform_agree(la2mod):
    x = I.make_inputs(2, 7, 2000, 128, 128, "bf16", seed=88)
    res = {}
    for sched in ("uniform", "balanced"):
        prev = la2mod.la2_set_schedule(sched)
        try:
            res[sched] = _run(la2mod, x)
        finally:
            la2mod.la2_set_schedule(prev)
    for a, b in zip(res["uniform"][0] + (res["uniform"][1],), res["balanced"][0] + (res["balanced"][1],)):
        a, b = a.float(), b.float()
        rms = a.pow(2).mean().sqrt()
        assert ((a - b).abs().max() / rms).item() < 2e-3


@pytest.mark.parametrize("schedule", ["balanced"], indirect=True)
@pytest.mark.parametrize("name", ["tnl15b", "sweep_T131072_blk128"])
def test_balanced_full_size_sampled_sequences(la2mod, oracle_mod, schedule, name):
    """The full-size workloads under the balanced schedule (148 CTAs, runs of
    26 to 665 tiles, pieces cut inside units), checked on whole sampled
    sequences: the first, a middle and the last (b, h)."""
    w = I.WORKLOADS[name]
    x = I.make_workload_inputs(w, seed=0)
    dev = torch.device("cuda")
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    lam = x["lam"].to(dev)
    o = la2mod.la2_fwd(q, k, v, lam)
    dq, dk, dv = la2mod.la2_bwd(q, k, v, lam, do)
    torch.cuda.synchronize()
    assert la2mod.la2_device_status(reset=True) == 0
    bi = np.array([0, w.B // 2, w.B - 1])
    hi = np.array([0, w.H // 2, w.H - 1])
    tb, th = torch.from_numpy(bi), torch.from_numpy(hi)
    sub = {n: x[n][tb, th] for n in ("q", "k", "v", "do")}
    lam_s = x["lam"].numpy().astype(np.float64)[hi]
    ro = oracle_mod.forward(sub["q"], sub["k"], sub["v"], lam_s)
    rdq, rdk, rdv = oracle_mod.backward(sub["q"], sub["k"], sub["v"], lam_s, sub["do"])
    errs = [_err(t[tb.to(dev), th.to(dev)], r) for t, r in zip((o, dq, dk, dv), (ro, rdq, rdk, rdv))]
    assert max(errs) <= TOL, errs
