"""Host side of ssd_gated_rmsnorm_forward: argument checks (no GPU needed)."""
import pytest


@pytest.fixture(scope="module")
def ssd():
    import __graft_entry__
    __graft_entry__.build()
    import mamba_selective_state_causal_b200 as pkg
    return pkg


BASE = dict(y=0x10000, yrs=2048, z=0x20000, zrs=2048, w=0x30000, eps=1e-5, group=0, out=0x40000,
            ors=2048, rows=16, d=2048, dtype=1)


@pytest.mark.parametrize("change,code", [
    (dict(dtype=4), 5),
    (dict(d=2047, yrs=2047, zrs=2047, ors=2047), 2),
    (dict(d=16384, yrs=16384, zrs=16384, ors=16384), 2),
    (dict(group=100), 2),
    (dict(group=24), 2),
    (dict(eps=-1.0), 2),
    (dict(rows=-1), 2),
    (dict(y=None), 1),
    (dict(w=None), 1),
    (dict(zrs=1024), 4),
    (dict(y=0x10002), 3),
    (dict(zrs=2052), 3),
    (dict(w=0x30004), 3),
])
def test_norm_rejects_bad_arguments(ssd, change, code):
    a = dict(BASE)
    a.update(change)
    rc = ssd.lib().ssd_gated_rmsnorm_forward(a["y"], a["yrs"], a["z"], a["zrs"], a["w"], a["eps"], a["group"],
                                             a["out"], a["ors"], a["rows"], a["d"], a["dtype"], None)
    assert rc == code, (rc, ssd.lib().ssd_last_error_string())


def test_norm_no_rows_is_a_no_op(ssd):
    a = dict(BASE, rows=0, y=None, z=None, out=None)
    assert ssd.lib().ssd_gated_rmsnorm_forward(a["y"], a["yrs"], a["z"], a["zrs"], a["w"], a["eps"], a["group"],
                                               a["out"], a["ors"], a["rows"], a["d"], a["dtype"], None) == 0
