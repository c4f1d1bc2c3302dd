"""GPU parity of la2_decode (one recurrent step per token) against the fp64
oracle, through the C ABI: single steps from random states, and generation
after a prompt, where la2_fwd_state's final state is advanced token by token
and every output is compared with the oracle run over prompt + continuation.
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


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,e", [(64, 64), (128, 128), (64, 128), (3, 5), (100, 300)])
def test_one_step(la2mod, oracle_mod, dtype, d, e):
    dev = torch.device("cuda")
    B, H = 3, 5
    x = I.make_inputs(B, H, 1, d, e, dtype, seed=d + e)
    q, k, v = (x[n][:, :, 0].contiguous() for n in ("q", "k", "v"))
    g = torch.Generator().manual_seed(e)
    s0 = torch.randn(B, H, d, e, generator=g)
    state = s0.to(dev)
    out = la2mod.la2_decode(q.to(dev), k.to(dev), v.to(dev), x["lam"].to(dev), state)
    torch.cuda.synchronize()
    lam = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :], (B, H))
    ro, rs = oracle_mod.decode_step(q, k, v, lam, s0.numpy().astype(np.float64))
    # fp32 arithmetic on the state either way: bf16 only rounds the inputs
    assert _err(out, ro) <= 1e-5 and _err(state, rs) <= 1e-5


@pytest.mark.parametrize("dtype,d,e", [("bf16", 128, 128), ("bf16", 64, 64), ("f32", 64, 64)])
def test_generation_after_prompt(la2mod, oracle_mod, dtype, d, e):
    """Prompt of 300 tokens by la2_fwd_state, then 40 decode steps."""
    dev = torch.device("cuda")
    B, H, P, G = 2, 4, 300, 40
    x = I.make_inputs(B, H, P + G, d, e, dtype, seed=7)
    lam = x["lam"].to(dev)
    prompt = {n: x[n][:, :, :P].contiguous().to(dev) for n in ("q", "k", "v")}
    _, state = la2mod.la2_fwd_state(prompt["q"], prompt["k"], prompt["v"], lam, None)
    outs = []
    for t in range(P, P + G):
        q, k, v = (x[n][:, :, t].contiguous().to(dev) for n in ("q", "k", "v"))
        outs.append(la2mod.la2_decode(q, k, v, lam, state))
    torch.cuda.synchronize()
    assert la2mod.la2_device_status(reset=True) == 0
    lam64 = np.broadcast_to(x["lam"].numpy().astype(np.float64)[None, :], (B, H))
    ro, rs = oracle_mod.forward_state(x["q"], x["k"], x["v"], lam64)
    assert _err(torch.stack(outs, dim=2), ro[:, :, P:]) <= TOL[dtype]
    assert _err(state, rs) <= TOL[dtype]


def test_decode_rejects_bad_arguments(la2mod):
    dev = torch.device("cuda")
    q = torch.zeros(1, 1, 8, device=dev)
    st = torch.zeros(1, 1, 8, 8, device=dev)
    lam = torch.ones(1, device=dev)
    from causal_linear_attention_la2_b200.la2 import LA2_ERR_INVALID_ARG, LA2_OK
    assert la2mod.la2_decode_raw(q.data_ptr(), q.data_ptr(), q.data_ptr(), lam.data_ptr(),
                                 st.data_ptr(), 0, 1, 1, 8, 8, 0) == LA2_ERR_INVALID_ARG
    assert la2mod.la2_decode_raw(0, 0, 0, 0, 0, 0, 0, 1, 8, 8, 0) == LA2_OK  # empty
