"""bf16 outputs (out_dtype=torch.bfloat16 in la2_fwd_ex, la2_bwd_ex and
la2_bwd_state) on the GPU, through the C ABI.

Each bf16 output is the kernel's fp32 result rounded to nearest even once, in
the output epilogue, so two things must hold:

- bit for bit, it is the fp32-output call's result rounded by torch (the same
  kernel, plan and arithmetic; only the store differs);
- against the fp64 oracle, element by element,
      |got - exact| <= 2e-2 rms(exact) (1 + 2^-8) + 2^-8 |exact|:
  the fp32 result y is within 2e-2 rms(exact) of exact (the bar of the fp32
  outputs), and rounding y to bf16 (8 significant bits) moves it by at most
  2^-8 |y| <= 2^-8 (|exact| + 2e-2 rms(exact)).
"""
import numpy as np
import pytest
import torch

from causal_linear_attention_la2_b200 import inputs as I

pytestmark = pytest.mark.gpu

TAU = 2e-2
U = 2.0 ** -8


@pytest.fixture(scope="module")
def la2mod():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_linear_attention_la2_b200 import build, la2
    build.build()
    la2.load()
    return la2


def _bound_ratio(got, ref):
    """max over elements of |got - ref| / (tau rms(ref) (1 + u) + u |ref|)."""
    g = got.detach().float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    allow = TAU * rms * (1.0 + U) + U * np.abs(ref)
    return float(np.max(np.abs(g - ref) / np.maximum(allow, 1e-300)))


def _run(la2mod, x, block=128, layout="bhtd", out_dtype=torch.bfloat16):
    dev = torch.device("cuda")
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    lam = x["lam"].to(dev)
    o = la2mod.la2_fwd_ex(q, k, v, lam, layout, block=block, out_dtype=out_dtype)
    g = la2mod.la2_bwd_ex(q, k, v, lam, do, layout, block=block, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert la2mod.la2_device_status(reset=True) == 0
    return (o,) + tuple(g)


def _check(la2mod, oracle_mod, x, block=128, heads=None):
    got = _run(la2mod, x, block)
    f32 = _run(la2mod, x, block, out_dtype=torch.float32)
    for n, a, b in zip(("o", "dq", "dk", "dv"), got, f32):
        assert a.dtype == torch.bfloat16
        assert torch.equal(a, b.to(torch.bfloat16)), f"{n}: bf16 output != rounded fp32 output"
    B, H = x["q"].shape[:2]
    lam = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :], (B, H))
    if heads is None:
        qs, ks, vs, ds, ls = x["q"], x["k"], x["v"], x["do"], lam
    else:
        bi, hi = (np.asarray(z, dtype=np.int64) for z in heads)
        tb, th = torch.from_numpy(bi), torch.from_numpy(hi)
        qs, ks, vs, ds = (x[n][tb, th] for n in ("q", "k", "v", "do"))
        ls = lam[bi, hi]
        got = tuple(t[tb.cuda(), th.cuda()] for t in got)
    refs = (oracle_mod.forward(qs, ks, vs, ls),) + tuple(oracle_mod.backward(qs, ks, vs, ls, ds))
    ratios = {n: _bound_ratio(g, r) for n, g, r in zip(("o", "dq", "dk", "dv"), got, refs)}
    assert all(r <= 1.0 for r in ratios.values()), ratios
    return ratios


@pytest.mark.parametrize("block", [128, 64, 256])
@pytest.mark.parametrize("T", [1, 129, 700])
@pytest.mark.parametrize("d,e", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_bf16_outputs_small(la2mod, oracle_mod, block, T, d, e):
    x = I.make_inputs(2, 3, T, d, e, "bf16", seed=7 * T + d + 3 * e + block)
    _check(la2mod, oracle_mod, x, block)


@pytest.mark.parametrize("B,H,T,d,e", [(1, 2, 3000, 128, 128), (1, 3, 2500, 64, 64)])
@pytest.mark.parametrize("schedule", ["uniform", "balanced"])
def test_bf16_outputs_segmented(la2mod, oracle_mod, B, H, T, d, e, schedule):
    prev = la2mod.la2_set_schedule(schedule)
    try:
        _check(la2mod, oracle_mod, I.make_inputs(B, H, T, d, e, "bf16", seed=T + d), 128)
    finally:
        la2mod.la2_set_schedule(prev)


@pytest.mark.parametrize("block", [128, 256])
def test_bf16_outputs_bthd_layout(la2mod, block):
    x = I.make_inputs(2, 3, 333, 128, 64, "bf16", seed=31)
    a = _run(la2mod, x, block)
    xt = {n: x[n].transpose(1, 2).contiguous() for n in ("q", "k", "v", "do")}
    xt["lam"] = x["lam"]
    b = _run(la2mod, xt, block, layout="bthd")
    for u, w in zip(a, b):
        assert torch.equal(u, w.transpose(1, 2))


def test_bf16_outputs_with_states(la2mod, oracle_mod):
    """la2_bwd_state with S0 and G and bf16 dq, dk, dv; the states stay fp32."""
    dev = torch.device("cuda")
    x = I.make_inputs(2, 2, 600, 128, 128, "bf16", seed=33)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    lam = x["lam"].to(dev)
    g = torch.Generator().manual_seed(34)
    s0 = torch.randn(2, 2, 128, 128, generator=g) * 0.5
    gs = torch.randn(2, 2, 128, 128, generator=g) * 0.5
    o, fin = la2mod.la2_fwd_ex(q, k, v, lam, init_state=s0.to(dev), want_final=True,
                               out_dtype=torch.bfloat16)
    o32, fin32 = la2mod.la2_fwd_ex(q, k, v, lam, init_state=s0.to(dev), want_final=True)
    r = la2mod.la2_bwd_state(q, k, v, lam, do, s0.to(dev), gs.to(dev), out_dtype=torch.bfloat16)
    r32 = la2mod.la2_bwd_state(q, k, v, lam, do, s0.to(dev), gs.to(dev))
    torch.cuda.synchronize()
    assert la2mod.la2_device_status(reset=True) == 0
    assert fin.dtype == torch.float32 and r[3].dtype == torch.float32
    assert torch.equal(o, o32.to(torch.bfloat16)) and torch.equal(fin, fin32)
    for a, b in zip(r[:3], r32[:3]):
        assert torch.equal(a, b.to(torch.bfloat16))
    assert torch.equal(r[3], r32[3])
    lam64 = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :], (2, 2))
    ro, _ = oracle_mod.forward_state(x["q"], x["k"], x["v"], lam64, s0.double().numpy())
    refs = oracle_mod.backward_state(x["q"], x["k"], x["v"], lam64, x["do"], s0.double().numpy(),
                                     gs.double().numpy())
    assert _bound_ratio(o, ro) <= 1.0
    for a, ref in zip(r[:3], refs[:3]):
        assert _bound_ratio(a, ref) <= 1.0


def test_bf16_outputs_do_not_write_past_their_end(la2mod):
    dev = torch.device("cuda")
    x = I.make_inputs(1, 2, 333, 128, 64, "bf16", seed=36)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    lam = x["lam"].to(dev)
    guard = 4096
    bufs = {n: torch.full((t.numel() + guard,), 7.0, dtype=torch.bfloat16, device=dev)
            for n, t in (("o", v), ("dq", q), ("dk", k), ("dv", v))}
    view = {n: b[:-guard].view((1, 2, 333, -1)) for n, b in bufs.items()}
    la2mod.la2_fwd_ex(q, k, v, lam, out=view["o"], out_dtype=torch.bfloat16)
    la2mod.la2_bwd_ex(q, k, v, lam, do, dq=view["dq"], dk=view["dk"], dv=view["dv"],
                      out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    for b in bufs.values():
        assert torch.all(b[-guard:] == 7.0)


def test_fp32_inputs_with_bf16_outputs_are_unsupported(la2mod):
    from causal_linear_attention_la2_b200.la2 import LA2Error, LA2_ERR_UNSUPPORTED
    x = I.make_inputs(1, 1, 64, 64, 64, "f32", seed=1)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    with pytest.raises(LA2Error) as ei:
        la2mod.la2_fwd_ex(q, k, v, x["lam"].to(dev), out_dtype=torch.bfloat16)
    assert ei.value.status == LA2_ERR_UNSUPPORTED


@pytest.mark.parametrize("name", ["tnl15b", "sweep_T131072_blk128", "tnl400m"])
def test_bf16_outputs_full_size_sampled(la2mod, oracle_mod, name):
    """The benchmark's workloads: whole tensors bitwise against the rounded fp32
    outputs, sampled sequences against the oracle."""
    w = I.WORKLOADS[name]
    x = I.make_workload_inputs(w, seed=0)
    bi = np.array([0, w.B // 2, w.B - 1])
    hi = np.array([0, w.H // 2, w.H - 1])
    _check(la2mod, oracle_mod, x, w.block, heads=(bi, hi))
