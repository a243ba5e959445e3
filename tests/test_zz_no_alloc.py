"""The allocation-free decode entry point, tested last.

akv_decode_static is for callers that cannot allocate device memory when they decode -- a
plugin whose process memory pool belongs to another framework, or a serving loop that has
frozen allocation so that nothing can block on the allocator.  It runs the same launches
as akv_decode on a fixed scratch array inside the library instead of a caller-provided
workspace, so its results must equal akv_decode's bit for bit.  The tests call it through
the C ABI twice in a row (the scratch keeps whatever the previous call left), on the
default stream and on a stream of their own, check that a call after the warm-up call
takes no device memory, and that a step too large for the fixed scratch is refused.  They
must pass alone in a fresh process and after the other tests.
"""
import pytest

from kv_cache_tiering_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    from kv_cache_tiering_b200 import build
    build.build()
    from kv_cache_tiering_b200 import akv, workloads
    return akv, workloads


def _bits(t):
    import torch
    return t.view(torch.int32)


def _compare(akv, w, cuda, stream=None):
    """Two calls in a row of akv_decode_static against akv_decode on the same stream."""
    import torch
    st = w.step
    B, Hq, Hkv, d = st.B, st.Hq, st.Hkv, st.d
    s = torch.cuda.current_stream() if stream is None else stream
    s.wait_stream(torch.cuda.current_stream())  # the workload was built on the current stream
    for call in range(2):
        with torch.cuda.stream(s):
            o = torch.full((B, Hq, d), float("nan"), device=cuda)
            lse = torch.full((B, Hq), float("nan"), device=cuda)
            st.decode(w.q, stream=s)  # the existing entry point, caller-provided workspace
            o_ref, l_ref = st.o.clone(), st.lse.clone()
            akv.akv_decode_static(w.q, B, Hq, Hkv, d, st.scale, st.tiers, st.split_tokens, o, lse, stream=s)
        s.synchronize()
        assert torch.equal(_bits(o), _bits(o_ref)), call
        assert torch.equal(_bits(lse), _bits(l_ref)), call


def test_static_decode_matches_workspace_decode_exact(mods, cuda):
    akv, workloads = mods
    wl = synth.Workload("static-exact", B=3, Hq=32, Hkv=8, d=128, split_tokens=512, extra={"T": 2600})
    _compare(akv, workloads.ExactResident(wl, cuda), cuda)


def test_static_decode_matches_workspace_decode_hybrid(mods, cuda):
    akv, workloads = mods
    wl = synth.Workload("static-hybrid", B=2, Hq=32, Hkv=8, d=128, split_tokens=256,
                        extra={"T": 3001, "window": 1000})
    _compare(akv, workloads.HybridResident(wl, cuda), cuda)


def test_static_decode_on_a_stream_of_its_own(mods, cuda):
    import torch
    akv, workloads = mods
    wl = synth.Workload("static-stream", B=2, Hq=16, Hkv=2, d=64, split_tokens=128,
                        extra={"T": 1500, "window": 500})
    _compare(akv, workloads.HybridResident(wl, cuda), cuda, stream=torch.cuda.Stream(cuda))


def test_static_decode_takes_no_device_memory_after_warm_up(mods, cuda):
    import torch
    akv, workloads = mods
    wl = synth.Workload("static-mem", B=2, Hq=32, Hkv=8, d=128, split_tokens=256, extra={"T": 2000, "window": 700})
    w = workloads.HybridResident(wl, cuda)
    st = w.step
    o = torch.empty((st.B, st.Hq, st.d), device=cuda)
    lse = torch.empty((st.B, st.Hq), device=cuda)
    args = (w.q, st.B, st.Hq, st.Hkv, st.d, st.scale, st.tiers, st.split_tokens, o, lse)
    akv.akv_decode_static(*args)  # warm-up: loads the module and looks up the scratch
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info(cuda)
    akv.akv_decode_static(*args)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(cuda)
    assert free1 == free0


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
