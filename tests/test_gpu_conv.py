"""GPU conv1d+SiLU against the CPU oracle (element by element)."""
import numpy as np
import pytest
import torch

import mamba_selective_state_causal_b200 as ssd
import oracle
from parity_util import TOL, host, rel_l2

pytestmark = pytest.mark.gpu


def _run(b, L, cch, dtype, with_tail, with_bias, seed=0, strided=False):
    g = torch.Generator().manual_seed(seed)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    u = torch.randn(b, L, cch, generator=g).to(tdt)
    w = (torch.rand(cch, 4, generator=g) - 0.5)
    bias = torch.randn(cch, generator=g) * 0.3 if with_bias else None
    tail = torch.randn(b, 3, cch, generator=g).to(tdt) if with_tail else None
    dev = "cuda"
    if strided:   # u and v as column slices of wider rows
        ub = torch.zeros(b, L, cch + 16, dtype=tdt)
        ub[:, :, 8:8 + cch] = u
        ud = ub.to(dev)[:, :, 8:8 + cch]
        vd = torch.empty(b, L, cch + 32, dtype=tdt, device=dev)[:, :, 16:16 + cch]
    else:
        ud = u.to(dev)
        vd = None
    tout = torch.empty(b, 3, cch, dtype=tdt, device=dev)
    v, _ = ssd.conv_forward(ud, w.to(dev), None if bias is None else bias.to(dev),
                            None if tail is None else tail.to(dev), tout, v=vd)
    ssd.sync_status()
    ref_v, ref_t = oracle.conv(u.float().numpy(), w.numpy(), None if bias is None else bias.numpy(),
                               None if tail is None else tail.float().numpy(),
                               io_round="bf16" if dtype == "bf16" else "f32")
    return host(v), host(tout), ref_v, ref_t


@pytest.mark.parametrize("b,L,cch,dtype,tail,bias,strided", [
    (1, 256, 64, "f32", False, False, False),       # tiny fp32 workload shape
    (2, 1000, 2304, "bf16", True, True, False),     # 0.3B channel count, ragged L
    (1, 16384, 2304, "bf16", False, False, False),  # 0.3B L=16k
    (3, 77, 96, "f32", True, True, True),
    (2, 130, 4352, "bf16", True, False, True),      # 1.3B channel count
    (1, 1, 64, "bf16", True, True, False),          # L < 3: tail from tail_in
    (1, 2, 64, "f32", True, False, False),
    (1, 3, 64, "bf16", False, True, False),
    (1, 65, 5376, "bf16", True, True, False),       # 2.7B channel count, one token past a block
])
def test_conv_matches_oracle(b, L, cch, dtype, tail, bias, strided):
    v, tout, rv, rt = _run(b, L, cch, dtype, tail, bias, strided=strided)
    assert rel_l2(v, rv) <= TOL[dtype]
    if dtype == "bf16":
        # fp32 sum of 5 terms (|w| <= 0.5, |u| ~ 1: error well under 1e-5 absolute)
        # then one RNE rounding on each side: at most one bf16 ulp (<= 2^-7 |v|) apart
        bound = np.abs(rv) * 2.0 ** -7 + 1e-5
        assert np.all(np.abs(v - rv) <= bound), float(np.max(np.abs(v - rv) - bound))
    else:
        assert np.max(np.abs(v - rv)) <= 1e-5 * max(1.0, np.max(np.abs(rv)))
    np.testing.assert_array_equal(tout, rt)


def test_conv_tail_may_alias_tail_in():
    g = torch.Generator().manual_seed(3)
    b, L, cch = 2, 2, 64
    u = torch.randn(b, L, cch, generator=g).to(torch.bfloat16)
    tail = torch.randn(b, 3, cch, generator=g).to(torch.bfloat16)
    w = torch.rand(cch, 4, generator=g) - 0.5
    td = tail.cuda()
    v, _ = ssd.conv_forward(u.cuda(), w.cuda(), None, td, td)
    ssd.sync_status()
    ref_v, ref_t = oracle.conv(u.float().numpy(), w.numpy(), None, tail.float().numpy(), io_round="bf16")
    np.testing.assert_array_equal(host(td), ref_t)
    assert rel_l2(host(v), ref_v) < 1e-2


def test_conv_empty_sequence_keeps_tail():
    b, cch = 1, 64
    tail = torch.randn(b, 3, cch).to(torch.bfloat16).cuda()
    tout = torch.empty_like(tail)
    u = torch.empty(b, 0, cch, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(cch, 4, device="cuda")
    ssd.conv_forward(u, w, None, tail, tout)
    ssd.sync_status()
    assert torch.equal(tout, tail)
