"""The allocation-free decode entry point, tested last.

akv_decode_static is for callers that cannot allocate device memory at decode time: it
runs the same decode step as akv_decode on a fixed scratch array inside the library
instead of a caller-provided workspace.  This test calls it through the C ABI twice in a
row and checks each result against akv_decode on the same inputs; it also checks that a
step too large for the fixed scratch is refused.  It must pass alone in a fresh process
and after the other tests (the scratch keeps whatever the previous call left).
"""
import numpy as np
import pytest

from kv_cache_tiering_b200 import synth

pytestmark = pytest.mark.gpu

TOL_O = 2e-3
TOL_LSE = 1e-3


@pytest.fixture(scope="module")
def mods():
    from kv_cache_tiering_b200 import build
    build.build()
    from kv_cache_tiering_b200 import akv, workloads
    return akv, workloads


def _compare(akv, w, cuda):
    import torch
    st = w.step
    B, Hq, Hkv, d = st.B, st.Hq, st.Hkv, st.d
    for call in range(2):
        st.decode(w.q)  # the existing entry point, caller-provided workspace
        o_ref, l_ref = st.o.clone(), st.lse.clone()
        o = torch.full((B, Hq, d), float("nan"), device=cuda)
        lse = torch.full((B, Hq), float("nan"), device=cuda)
        akv.akv_decode_static(w.q, B, Hq, Hkv, d, st.scale, st.tiers, st.split_tokens, o, lse)
        torch.cuda.synchronize()
        assert float((o - o_ref).abs().max().item()) <= TOL_O, call
        assert float((lse - l_ref).abs().max().item()) <= TOL_LSE, call


def test_static_decode_matches_workspace_decode_exact(mods, cuda):
    akv, workloads = mods
    wl = synth.Workload("static-exact", B=3, Hq=32, Hkv=8, d=128, split_tokens=512, extra={"T": 2600})
    _compare(akv, workloads.ExactResident(wl, cuda), cuda)


def test_static_decode_matches_workspace_decode_hybrid(mods, cuda):
    akv, workloads = mods
    wl = synth.Workload("static-hybrid", B=2, Hq=32, Hkv=8, d=128, split_tokens=256,
                        extra={"T": 3001, "window": 1000})
    _compare(akv, workloads.HybridResident(wl, cuda), cuda)


def test_static_decode_refuses_steps_beyond_its_scratch(mods, cuda):
    import torch
    akv, workloads = mods
    wl = synth.Workload("static-big", B=2, Hq=32, Hkv=8, d=128, split_tokens=16, extra={"T": 4096})
    w = workloads.ExactResident(wl, cuda)
    st = w.step
    assert akv.akv_decode_workspace_size(st.B, st.Hq, st.Hkv, st.d, st.tiers, st.split_tokens) > (8 << 20)
    o = torch.empty((st.B, st.Hq, st.d), device=cuda)
    lse = torch.empty((st.B, st.Hq), device=cuda)
    with pytest.raises(akv.AkvError) as e:
        akv.akv_decode_static(w.q, st.B, st.Hq, st.Hkv, st.d, st.scale, st.tiers, st.split_tokens, o, lse)
    assert e.value.status == akv.AKV_ERR_BUDGET
