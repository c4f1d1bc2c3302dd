"""GPU parity of la2_bwd_state (backward with carried states) against the fp64
oracle's backward_state, through the C ABI.

L = sum dout * out + <G, S_{T-1}> for the forward from S0: dq, dk, dv and dS0
are compared element by element with the bar of the other parity tests
(max|gpu - oracle| / rms(oracle) <= 2e-2 for bf16 inputs, 1e-5 for fp32), on
ragged lengths, every (d, e), segmented few-sequence shapes under both
schedules, the fp32 path at every block size and both layouts; a sequence
trained in two pieces gives the whole sequence's gradients.
"""
import numpy as np
import pytest
import torch

from causal_linear_attention_la2_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}
NAMES = ("dq", "dk", "dv", "dS0")


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


def _state(B, H, d, e, seed, scale=0.5):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(B, H, d, e, generator=g, dtype=torch.float32) * scale


def _gpu(la2mod, x, s0, g, block=128, layout="bhtd"):
    dev = torch.device("cuda")
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    lam = x["lam"].to(dev)
    if layout == "bthd":
        q, k, v, do = (t.transpose(1, 2).contiguous() for t in (q, k, v, do))
    outs = [torch.full(t.shape, float("nan"), device=dev) for t in (q, k, v)]
    B, H = x["q"].shape[:2]
    d, e = x["q"].shape[-1], x["v"].shape[-1]
    ds0 = torch.full((B, H, d, e), float("nan"), device=dev)
    res = la2mod.la2_bwd_state(q, k, v, lam, do, None if s0 is None else s0.to(dev),
                               None if g is None else g.to(dev), layout, *outs, d_init_state=ds0,
                               block=block)
    torch.cuda.synchronize()
    assert la2mod.la2_device_status(reset=True) == 0
    res = list(res)
    if layout == "bthd":
        res[:3] = [t.transpose(1, 2) for t in res[:3]]
    return res


def _ref(oracle_mod, x, s0, g):
    B, H = x["q"].shape[:2]
    lam = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :], (B, H))
    return oracle_mod.backward_state(x["q"], x["k"], x["v"], lam, x["do"],
                                     None if s0 is None else s0.numpy().astype(np.float64),
                                     None if g is None else g.numpy().astype(np.float64))


def _check(la2mod, oracle_mod, x, s0, g, tol, block=128, layout="bhtd"):
    got = _gpu(la2mod, x, s0, g, block, layout)
    want = _ref(oracle_mod, x, s0, g)
    errs = {n: _err(a, b) for n, a, b in zip(NAMES, got, want)}
    for n, a in zip(NAMES, got):
        assert torch.isfinite(a).all(), n
    assert all(v <= tol for v in errs.values()), errs
    return errs


@pytest.mark.parametrize("T", [1, 100, 128, 129, 300, 1000])
@pytest.mark.parametrize("d,e", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_bf16_bwd_state(la2mod, oracle_mod, T, d, e):
    x = I.make_inputs(2, 3, T, d, e, "bf16", seed=T + 5 * d + e)
    _check(la2mod, oracle_mod, x, _state(2, 3, d, e, T), _state(2, 3, d, e, T + 1), TOL["bf16"])


@pytest.mark.parametrize("which", ["s0", "g"])
def test_bf16_bwd_one_state_only(la2mod, oracle_mod, which):
    x = I.make_inputs(1, 4, 333, 128, 128, "bf16", seed=12)
    s = _state(1, 4, 128, 128, 7)
    _check(la2mod, oracle_mod, x, s if which == "s0" else None, s if which == "g" else None,
           TOL["bf16"])


@pytest.mark.parametrize("schedule", ["uniform", "balanced"])
@pytest.mark.parametrize("T,d,e", [(4000, 64, 64), (4100, 128, 128), (2000, 128, 64), (2000, 64, 128)])
def test_bf16_bwd_state_segmented(la2mod, oracle_mod, schedule, T, d, e):
    """Few sequences: every role is cut into segments (the first of a reverse
    role holds the sequence's last, ragged tile, where G enters)."""
    x = I.make_inputs(1, 2, T, d, e, "bf16", seed=T + d)
    prev = la2mod.la2_set_schedule(schedule)
    try:
        _check(la2mod, oracle_mod, x, _state(1, 2, d, e, 1), _state(1, 2, d, e, 2), TOL["bf16"])
    finally:
        la2mod.la2_set_schedule(prev)


@pytest.mark.parametrize("block", [64, 128, 256])
@pytest.mark.parametrize("T,d,e", [(1, 64, 64), (300, 100, 37), (517, 3, 5)])
def test_f32_bwd_state(la2mod, oracle_mod, block, T, d, e):
    x = I.make_inputs(2, 2, T, d, e, "f32", seed=T + d)
    _check(la2mod, oracle_mod, x, _state(2, 2, d, e, d), _state(2, 2, d, e, e), TOL["f32"], block)


@pytest.mark.parametrize("dtype,d,e", [("bf16", 64, 64), ("bf16", 128, 128), ("f32", 64, 32)])
def test_bthd_layout_bwd_state(la2mod, oracle_mod, dtype, d, e):
    x = I.make_inputs(2, 3, 300, d, e, dtype, seed=4)
    s0, g = _state(2, 3, d, e, 5), _state(2, 3, d, e, 6)
    a = _gpu(la2mod, x, s0, g, layout="bhtd")
    b = _gpu(la2mod, x, s0, g, layout="bthd")
    for n, u, w in zip(NAMES, a, b):
        assert torch.equal(u, w), n
    _check(la2mod, oracle_mod, x, s0, g, TOL[dtype], layout="bthd")


@pytest.mark.parametrize("dtype,d,e", [("bf16", 64, 64), ("bf16", 128, 128), ("f32", 64, 64)])
@pytest.mark.parametrize("cut", [128, 200])
def test_two_pieces_equal_whole(la2mod, oracle_mod, dtype, d, e, cut):
    """Train [0, T) as two pieces on the GPU: forward of piece 1 from S0 gives
    S_mid; the backward of piece 2 from S_mid with G gives dS_mid; the backward
    of piece 1 from S0 with dS_mid as its incoming gradient gives dS0.  Against
    the oracle's gradients of the whole sequence."""
    T = 777
    dev = torch.device("cuda")
    x = I.make_inputs(2, 4, T, d, e, dtype, seed=cut + d)
    s0, g = _state(2, 4, d, e, 8), _state(2, 4, d, e, 9)
    part = [{n: x[n][:, :, sl].contiguous() for n in ("q", "k", "v", "do")}
            for sl in (slice(0, cut), slice(cut, T))]
    for p_ in part:
        p_["lam"] = x["lam"]
    lam = x["lam"].to(dev)
    _, smid = la2mod.la2_fwd_state(*(part[0][n].to(dev) for n in ("q", "k", "v")), lam,
                                   s0.to(dev))
    dq2, dk2, dv2, dsmid = _gpu(la2mod, part[1], smid.cpu(), g)
    dq1, dk1, dv1, ds0 = _gpu(la2mod, part[0], s0, dsmid.cpu())
    want = _ref(oracle_mod, x, s0, g)
    got = (torch.cat([dq1, dq2], 2), torch.cat([dk1, dk2], 2), torch.cat([dv1, dv2], 2), ds0)
    errs = {n: _err(a, b) for n, a, b in zip(NAMES, got, want)}
    assert all(v <= TOL[dtype] for v in errs.values()), errs


def test_zero_length_passes_the_gradient_through(la2mod):
    dev = torch.device("cuda")
    B, H, d, e = 2, 3, 64, 64
    q = torch.zeros(B, H, 0, d, dtype=torch.bfloat16, device=dev)
    v = torch.zeros(B, H, 0, e, dtype=torch.bfloat16, device=dev)
    lam = torch.full((H,), 0.9, device=dev)
    g = _state(B, H, d, e, seed=3).to(dev)
    *_, ds0 = la2mod.la2_bwd_state(q, q, v, lam, v, None, g)
    torch.cuda.synchronize()
    assert torch.equal(ds0, g)
    *_, ds00 = la2mod.la2_bwd_state(q, q, v, lam, v, None, None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(ds00) == 0


@pytest.mark.parametrize("d,e", [(64, 64), (128, 128)])
def test_no_states_match_la2_bwd_bitwise(la2mod, d, e):
    dev = torch.device("cuda")
    x = I.make_inputs(2, 3, 555, d, e, "bf16", seed=9)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    lam = x["lam"].to(dev)
    a = la2mod.la2_bwd(q, k, v, lam, do)
    b = la2mod.la2_bwd_state(q, k, v, lam, do, want_d_init=False)
    torch.cuda.synchronize()
    assert b[3] is None
    for u, w in zip(a, b[:3]):
        assert torch.equal(u, w)


# ------------------------------------- bf16 with T_B = 64 and 256 (la2_scan_blk)

@pytest.mark.parametrize("block", [64, 256])
@pytest.mark.parametrize("T", [1, 63, 65, 128, 129, 255, 257, 700])
@pytest.mark.parametrize("d,e", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_bf16_other_blocks_bwd_state(la2mod, oracle_mod, block, T, d, e):
    """S0 read transposed by the dq scan, G entering at position T-1 in the dk
    and dv scans' first (ragged) block, dS0 from the dv scan's final state."""
    x = I.make_inputs(2, 3, T, d, e, "bf16", seed=T + 5 * d + e + block)
    errs = _check(la2mod, oracle_mod, x, _state(2, 3, d, e, T), _state(2, 3, d, e, T + 1), TOL["bf16"],
                  block)
    assert max(errs.values()) < 1e-3, errs


@pytest.mark.parametrize("block", [64, 256])
@pytest.mark.parametrize("which", ["s0", "g"])
def test_other_blocks_bwd_one_state_only(la2mod, oracle_mod, block, which):
    x = I.make_inputs(1, 4, 333, 128, 128, "bf16", seed=13 + block)
    s = _state(1, 4, 128, 128, 8)
    _check(la2mod, oracle_mod, x, s if which == "s0" else None, s if which == "g" else None,
           TOL["bf16"], block)


@pytest.mark.parametrize("block", [64, 256])
def test_other_blocks_bwd_pieces_equal_whole(la2mod, oracle_mod, block):
    """The backward of the second piece from the carried S0 and the incoming G,
    then of the first piece with the second's dS0 as its G: the whole
    sequence's gradients."""
    T, cut = 600, 257
    x = I.make_inputs(1, 3, T, 128, 128, "bf16", seed=50 + block)
    lam64 = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :], (1, 3))
    part = [{n: x[n][:, :, a:b].contiguous() for n in ("q", "k", "v", "do")} for a, b in ((0, cut), (cut, T))]
    for pc in part:
        pc["lam"] = x["lam"]
    _, s1 = oracle_mod.forward_state(part[0]["q"], part[0]["k"], part[0]["v"], lam64, None)
    g2 = _gpu(la2mod, part[1], torch.from_numpy(s1).float(), None, block)
    g1 = _gpu(la2mod, part[0], None, g2[3].cpu(), block)
    want = _ref(oracle_mod, x, None, None)
    for i, n in enumerate(NAMES[:3]):
        got = torch.cat([g1[i], g2[i]], dim=2)
        assert _err(got, want[i]) < 1e-3, n
