"""GPU parity of the normalised form (la2_fwd_norm, la2_bwd_norm) against the
fp64 oracle's forward_norm and backward_norm, through the C ABI.

The denominator q_t . z_t needs positive features to stay away from zero, so
the inputs are the recipe's draws with q and k replaced by their absolute
values (a positive feature map applied before the call).  y, den, dq, dk and dv
are compared element by element with the bar of the other parity tests:
max|gpu - oracle| / scale <= 2e-2 for bf16 inputs, 1e-5 for fp32, on ragged
lengths, every (d, e), chunked few-sequence shapes, both layouts and the
full-size TNL-15B shape.

The scale is rms(oracle) for y and den.  dv's rows scale like 1/den_t (its
row s sums dy_t / den_t over t >= s), largest at the first positions, so its
error is taken row by row against the row's rms.  dq and dk are each the sum of
two parts that nearly cancel where y depends weakly on q or k (T = 1 makes y =
v exactly, so dq = dk = 0): the numerator's term and the denominator's,
dden_t z_t for dq and sum_{t>=s} lambda^(t-s) dden_t q_t for dk.  Any
arithmetic that forms the parts to a relative precision p gets their sum to
p times the parts' size, not p times the sum's; so their scale is the size of
the two parts, computed here from the oracle's y and den in fp64, position by
position (the parts scale like 1/den_t, largest at the first positions): the
error of row t is divided by the rms over that row of the two parts.
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


def _inputs(B, H, T, d, e, dtype, seed, decay="tnl"):
    x = I.make_inputs(B, H, T, d, e, dtype, seed=seed, decay=decay)
    x["q"], x["k"] = x["q"].abs(), x["k"].abs()
    return x


def _err(gpu, ref):
    gpu = gpu.detach().double().cpu().numpy()
    return float(np.max(np.abs(gpu - ref)) / np.sqrt(np.mean(ref * ref)))


def _run(la2mod, x, layout="bhtd", block=128):
    dev = torch.device("cuda")
    q, k, v, dy = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    if layout == "bthd":
        q, k, v, dy = (t.transpose(1, 2).contiguous() for t in (q, k, v, dy))
    lam = x["lam"].to(dev)
    y, den = la2mod.la2_fwd_norm(q, k, v, lam, layout, block=block)
    dq, dk, dv = la2mod.la2_bwd_norm(q, k, v, lam, y, den, dy, layout, block=block)
    torch.cuda.synchronize()
    assert la2mod.la2_device_status(reset=True) == 0
    outs = [y, dq, dk, dv]
    if layout == "bthd":
        outs = [t.transpose(1, 2) for t in outs]
    return outs[0], den, outs[1], outs[2], outs[3]


def _den_parts(xs, ls, y, den, dq, dk):
    """(rms of dq's two parts, rms of dk's two parts), fp64, from the oracle."""
    q, k, dy = (xs[n].double().numpy().reshape(-1, xs[n].shape[-2], xs[n].shape[-1])
                for n in ("q", "k", "do"))
    lam = np.asarray(ls, dtype=np.float64).reshape(-1)
    yv = y.reshape(q.shape[0], q.shape[1], -1)
    dn = den.reshape(q.shape[0], q.shape[1])
    dden = -np.sum(dy * yv, axis=-1) / dn
    T = q.shape[1]
    z = np.zeros((q.shape[0], q.shape[2]))
    r = np.zeros_like(z)
    pq = np.empty_like(q)
    pk = np.empty_like(k)
    for t in range(T):
        z = lam[:, None] * z + k[:, t]
        pq[:, t] = dden[:, t, None] * z
    for t in range(T - 1, -1, -1):
        r = lam[:, None] * r + dden[:, t, None] * q[:, t]
        pk[:, t] = r
    dqf, dkf = dq.reshape(pq.shape), dk.reshape(pk.shape)
    sq = np.sqrt(np.mean(pq ** 2 + (dqf - pq) ** 2, axis=-1, keepdims=True))
    sk = np.sqrt(np.mean(pk ** 2 + (dkf - pk) ** 2, axis=-1, keepdims=True))
    return sq.reshape(dq.shape[:-1] + (1,)), sk.reshape(dk.shape[:-1] + (1,))


def _check(la2mod, oracle_mod, x, tol, layout="bhtd", block=128, heads=None):
    got = _run(la2mod, x, layout, block)
    B, H = x["q"].shape[:2]
    lam = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :], (B, H))
    xs, ls = x, lam
    if heads is not None:
        bi, hi = (torch.from_numpy(np.asarray(z)) for z in heads)
        xs = {n: x[n][bi, hi] for n in ("q", "k", "v", "do")}
        ls = lam[np.asarray(heads[0]), np.asarray(heads[1])]
        got = tuple(t[bi.cuda(), hi.cuda()] for t in got)
    y, den = oracle_mod.forward_norm(xs["q"], xs["k"], xs["v"], ls)
    grads = oracle_mod.backward_norm(xs["q"], xs["k"], xs["v"], ls, xs["do"])
    sq, sk = _den_parts(xs, ls, y, den, grads[0], grads[1])
    refs = (y, den) + grads
    sv = np.sqrt(np.mean(grads[2] ** 2, axis=-1, keepdims=True))
    scales = [None, None, sq, sk, sv]
    errs = {}
    for n, g, r, sc in zip(("y", "den", "dq", "dk", "dv"), got, refs, scales):
        gg = g.detach().double().cpu().numpy()
        if sc is None:
            errs[n] = float(np.max(np.abs(gg - r)) / np.sqrt(np.mean(r * r)))
        else:  # per row: the row's largest error over the size of its two parts
            errs[n] = float(np.max(np.max(np.abs(gg - r), axis=-1, keepdims=True) / sc))
    assert all(torch.isfinite(g).all() for g in got)
    assert all(v <= tol for v in errs.values()), errs
    return errs


@pytest.mark.parametrize("T", [1, 31, 129, 300, 1000])
@pytest.mark.parametrize("d,e", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_norm_bf16(la2mod, oracle_mod, T, d, e):
    _check(la2mod, oracle_mod, _inputs(2, 3, T, d, e, "bf16", seed=T + d + e), TOL["bf16"])


@pytest.mark.parametrize("block", [64, 128, 256])
@pytest.mark.parametrize("T,d,e", [(1, 16, 8), (300, 100, 37), (517, 64, 64)])
def test_norm_f32(la2mod, oracle_mod, block, T, d, e):
    _check(la2mod, oracle_mod, _inputs(2, 2, T, d, e, "f32", seed=T + d), TOL["f32"], block=block)


@pytest.mark.parametrize("T,d,e", [(4100, 128, 128), (3000, 64, 64)])
def test_norm_chunked_few_sequences(la2mod, oracle_mod, T, d, e):
    """One or two sequences: the scans are cut into chunks (and la2_fwd /
    la2_bwd into segments)."""
    _check(la2mod, oracle_mod, _inputs(1, 2, T, d, e, "bf16", seed=T), TOL["bf16"])


def test_norm_decays(la2mod, oracle_mod):
    x = _inputs(1, 5, 700, 64, 64, "bf16", seed=3)
    x["lam"] = torch.tensor([2.0 ** -20, 0.3, 0.9, 0.999, 1.0], dtype=torch.float32)
    _check(la2mod, oracle_mod, x, TOL["bf16"])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_norm_bthd_layout(la2mod, oracle_mod, dtype):
    x = _inputs(2, 3, 333, 64, 64, dtype, seed=8)
    a = _run(la2mod, x)
    b = _run(la2mod, x, layout="bthd")
    for u, w in zip(a, b):
        assert torch.equal(u, w)
    _check(la2mod, oracle_mod, x, TOL[dtype], layout="bthd")


def test_norm_full_size_15b(la2mod, oracle_mod):
    w = I.WORKLOADS["tnl15b"]
    x = _inputs(w.B, w.H, w.T, w.d, w.e, w.dtype, seed=0)
    _check(la2mod, oracle_mod, x, TOL[w.dtype], heads=([0, 1, 1], [0, 20, 39]))


# ------------------------------------- bf16 with T_B = 64 and 256 (la2_scan_blk)

@pytest.mark.parametrize("block", [64, 256])
@pytest.mark.parametrize("T", [1, 65, 129, 257, 700])
@pytest.mark.parametrize("d,e", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_norm_bf16_other_blocks(la2mod, oracle_mod, block, T, d, e):
    """The numerator scans of the phase-serial kernel, the backward's dk and dv
    with the factor 1 / den on the summed position."""
    _check(la2mod, oracle_mod, _inputs(2, 3, T, d, e, "bf16", seed=T + d + e + block), TOL["bf16"],
           block=block)


@pytest.mark.parametrize("block", [64, 256])
def test_norm_other_blocks_decays(la2mod, oracle_mod, block):
    x = _inputs(1, 5, 700, 128, 128, "bf16", seed=4 + block)
    x["lam"] = torch.tensor([2.0 ** -20, 0.3, 0.9, 0.999, 1.0], dtype=torch.float32)
    _check(la2mod, oracle_mod, x, TOL["bf16"], block=block)
