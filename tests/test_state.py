"""GPU parity of la2_fwd_state (forward with a carried state) against the
fp64 oracle's forward_state, through the C ABI.

Outputs and final states are compared element by element with the bar of the
other parity tests (max|gpu - oracle| / rms(oracle) <= 2e-2 for bf16 inputs,
1e-5 for fp32), on ragged lengths, every (d, e), segmented few-sequence
shapes, and across pieces: running a sequence in two calls, the second from the
first's final state, gives the one-call result.
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


def _init_state(B, H, d, e, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(B, H, d, e, generator=g, dtype=torch.float32) * 0.5


def _run(la2mod, x, init, block=128):
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    lam = x["lam"].to(dev)
    B, H, T, d = q.shape
    e = v.shape[-1]
    out = torch.full((B, H, T, e), float("nan"), device=dev)
    fin = torch.full((B, H, d, e), float("nan"), device=dev)
    la2mod.la2_fwd_state(q, k, v, lam, None if init is None else init.to(dev), out=out,
                         final_state=fin, block=block)
    torch.cuda.synchronize()
    assert la2mod.la2_device_status(reset=True) == 0
    return out, fin


def _ref(oracle_mod, x, init):
    B, H = x["q"].shape[:2]
    lam = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :], (B, H))
    s0 = None if init is None else init.numpy().astype(np.float64)
    return oracle_mod.forward_state(x["q"], x["k"], x["v"], lam, s0)


@pytest.mark.parametrize("T", [1, 100, 128, 129, 300, 1000])
@pytest.mark.parametrize("d,e", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_bf16_state_in_out(la2mod, oracle_mod, T, d, e):
    x = I.make_inputs(2, 3, T, d, e, "bf16", seed=T + 3 * d + e)
    init = _init_state(2, 3, d, e, seed=T)
    out, fin = _run(la2mod, x, init)
    ro, rs = _ref(oracle_mod, x, init)
    eo, es = _err(out, ro), _err(fin, rs)
    assert torch.isfinite(out).all() and torch.isfinite(fin).all()
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)


@pytest.mark.parametrize("T,d,e", [(4000, 64, 64), (4100, 128, 128), (2000, 128, 64)])
def test_bf16_state_segmented(la2mod, oracle_mod, T, d, e):
    """One or two sequences: cut into segments, the first starting from init."""
    x = I.make_inputs(1, 2, T, d, e, "bf16", seed=T)
    init = _init_state(1, 2, d, e, seed=1)
    out, fin = _run(la2mod, x, init)
    ro, rs = _ref(oracle_mod, x, init)
    assert _err(out, ro) <= TOL["bf16"] and _err(fin, rs) <= TOL["bf16"]


@pytest.mark.parametrize("block", [64, 128, 256])
@pytest.mark.parametrize("T,d,e", [(1, 64, 64), (300, 100, 37), (517, 3, 5)])
def test_f32_state_in_out(la2mod, oracle_mod, block, T, d, e):
    x = I.make_inputs(2, 2, T, d, e, "f32", seed=T + d)
    init = _init_state(2, 2, d, e, seed=d)
    out, fin = _run(la2mod, x, init, block=block)
    ro, rs = _ref(oracle_mod, x, init)
    assert _err(out, ro) <= TOL["f32"] and _err(fin, rs) <= TOL["f32"]


@pytest.mark.parametrize("dtype,d,e", [("bf16", 64, 64), ("bf16", 128, 128), ("f32", 64, 64)])
@pytest.mark.parametrize("cut", [128, 200])
def test_pieces_equal_whole(la2mod, oracle_mod, dtype, d, e, cut):
    """[0, cut) and then [cut, T) from the carried state, against the oracle
    over [0, T) in one piece."""
    T = 777
    x = I.make_inputs(2, 4, T, d, e, dtype, seed=cut)
    first = {n: x[n][:, :, :cut].contiguous() for n in ("q", "k", "v")}
    second = {n: x[n][:, :, cut:].contiguous() for n in ("q", "k", "v")}
    first["lam"] = second["lam"] = x["lam"]
    o1, s1 = _run(la2mod, first, None)
    o2, s2 = _run(la2mod, second, s1.cpu())
    ro, rs = _ref(oracle_mod, x, None)
    assert _err(torch.cat([o1, o2], dim=2), ro) <= TOL[dtype]
    assert _err(s2, rs) <= TOL[dtype]


def test_zero_length_copies_the_state(la2mod):
    dev = torch.device("cuda")
    B, H, d, e = 2, 3, 64, 64
    q = torch.zeros(B, H, 0, d, dtype=torch.bfloat16, device=dev)
    v = torch.zeros(B, H, 0, e, dtype=torch.bfloat16, device=dev)
    lam = torch.full((H,), 0.9, device=dev)
    init = _init_state(B, H, d, e, seed=3).to(dev)
    out, fin = la2mod.la2_fwd_state(q, q, v, lam, init)
    torch.cuda.synchronize()
    assert torch.equal(fin, init)
    _, fin0 = la2mod.la2_fwd_state(q, q, v, lam, None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(fin0) == 0


def test_no_init_matches_la2_fwd(la2mod):
    dev = torch.device("cuda")
    x = I.make_inputs(2, 3, 555, 128, 128, "bf16", seed=9)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    lam = x["lam"].to(dev)
    a = la2mod.la2_fwd(q, k, v, lam)
    b, _ = la2mod.la2_fwd_state(q, k, v, lam, None)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ------------------------------------- bf16 with T_B = 64 and 256 (la2_scan_blk)

@pytest.mark.parametrize("block", [64, 256])
@pytest.mark.parametrize("T", [1, 63, 65, 128, 129, 255, 257, 700])
@pytest.mark.parametrize("d,e", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_bf16_other_blocks_state_in_out(la2mod, oracle_mod, block, T, d, e):
    """The phase-serial kernel from init_state, the final state from its last
    block's true row count (every T mod block case), fp32 state in registers."""
    x = I.make_inputs(2, 3, T, d, e, "bf16", seed=T + 3 * d + e + block)
    init = _init_state(2, 3, d, e, seed=T + block)
    out, fin = _run(la2mod, x, init, block=block)
    ro, rs = _ref(oracle_mod, x, init)
    eo, es = _err(out, ro), _err(fin, rs)
    assert torch.isfinite(out).all() and torch.isfinite(fin).all()
    assert eo < 1e-3 and es < 1e-3, (eo, es)  # hi + lo operands, fp32 state


@pytest.mark.parametrize("block", [64, 256])
@pytest.mark.parametrize("cut", [100, 256])
def test_other_blocks_pieces_equal_whole(la2mod, oracle_mod, block, cut):
    T = 777
    x = I.make_inputs(2, 4, T, 128, 128, "bf16", seed=cut + block)
    first = {n: x[n][:, :, :cut].contiguous() for n in ("q", "k", "v")}
    second = {n: x[n][:, :, cut:].contiguous() for n in ("q", "k", "v")}
    first["lam"] = second["lam"] = x["lam"]
    o1, s1 = _run(la2mod, first, None, block=block)
    o2, s2 = _run(la2mod, second, s1.cpu(), block=block)
    ro, rs = _ref(oracle_mod, x, None)
    assert _err(torch.cat([o1, o2], dim=2), ro) < 1e-3
    assert _err(s2, rs) < 1e-3


@pytest.mark.parametrize("block", [64, 256])
def test_other_blocks_state_decays(la2mod, oracle_mod, block):
    """lambda from 2^-20 to 1 in one launch, with a state in and out."""
    x = I.make_inputs(1, 7, 333, 128, 128, "bf16", seed=40 + block)
    x["lam"] = torch.tensor([2.0 ** -20, 0.3, 0.8, 0.9, 0.99, 0.999, 1.0], dtype=torch.float32)
    init = _init_state(1, 7, 128, 128, seed=41)
    out, fin = _run(la2mod, x, init, block=block)
    ro, rs = _ref(oracle_mod, x, init)
    assert _err(out, ro) <= TOL["bf16"] and _err(fin, rs) <= TOL["bf16"]
