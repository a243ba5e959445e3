"""GPU tests of the staging ring: staged decode equals the fully resident decode bit for
bit, matches the float64 oracle, writes appended rows back to the host copy, and the
ring's refusals (not pinned, a buffer still in use) leave the buffer untouched."""
import numpy as np
import pytest

from kv_cache_tiering_b200 import synth
from oracle import akv_oracle as ora

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    from kv_cache_tiering_b200 import build
    build.build()
    from kv_cache_tiering_b200 import akv, workloads
    return akv, workloads


def _wl(T, layers=2, chunk=4096):
    return synth.Workload("staged-small", B=1, Hq=32, Hkv=8, d=128, split_tokens=512,
                          extra={"T": T, "layers": layers, "chunk": chunk})


@pytest.mark.parametrize("T", [9192, 8192, 100])
def test_staged_equals_resident_bitwise_and_oracle(mods, cuda, T):
    import torch
    akv, workloads = mods
    wl = _wl(T)
    staged = workloads.StagedDecode(wl, cuda, max_steps=4)
    resident = workloads.StagedDecode(wl, cuda, max_steps=4, resident=True)
    for step in range(2):
        q, new = staged.inputs(step)
        staged.step(q, new)
        resident.step(q, new)
        torch.cuda.synchronize()
        assert torch.equal(staged.o, resident.o) and torch.equal(staged.lse, resident.lse)
        n_split = -(-(T + step + 1) // wl.split_tokens)
        assert torch.equal(staged.o_part[:n_split], resident.o_part[:n_split])
        assert int(staged.err.item()) == 0
    # appended rows were written back to the host copies
    for layer in range(wl.extra["layers"]):
        for step in range(2):
            k_new, v_new = synth.new_token(wl, layer, step)
            row = staged.host[layer][T + step].numpy().view(np.uint16)
            assert np.array_equal(row[0], k_new) and np.array_equal(row[1], v_new)
            assert torch.equal(staged.host[layer][T + step], resident.host[layer][T + step])
    # oracle: layer 1 after step 1 (history T + 2 tokens)
    layer = 1
    k, v = synth.history_token_major(wl, layer, T)
    k_all = np.concatenate([k, np.stack([synth.new_token(wl, layer, s)[0] for s in range(2)])])
    v_all = np.concatenate([v, np.stack([synth.new_token(wl, layer, s)[1] for s in range(2)])])
    q1 = synth.queries(wl, layer=layer, step=1, B=1)[0]
    tiers = [(ora.bf16_bits_to_f64(k_all.transpose(1, 0, 2)), ora.bf16_bits_to_f64(v_all.transpose(1, 0, 2)))]
    _, _, (o_ref, l_ref) = ora.decode_sequence(ora.bf16_bits_to_f64(q1), tiers, wl.scale, wl.split_tokens)
    assert np.max(np.abs(staged.o[layer].cpu().numpy() - o_ref)) <= 2e-3
    assert np.max(np.abs(staged.lse[layer].cpu().numpy() - l_ref)) <= 1e-3
    staged.close()


@pytest.mark.parametrize("T,W", [(9003, 1000), (4700, 4096)])
def test_staged_hybrid_equals_resident_bitwise_and_oracle(mods, cuda, T, W):
    """Compact history staged from pinned host memory (a partial last block and a partial
    last chunk when T - W = 8003; a single short chunk when T - W = 604), window resident."""
    import torch
    akv, workloads = mods
    wl = synth.Workload("staged-hybrid-small", B=1, Hq=32, Hkv=8, d=128, split_tokens=512, extra={})
    kw = dict(layers=2, T=T, W=W, chunk=4096, max_steps=3, source="host")
    staged = workloads.StagedHybridDecode(wl, cuda, **kw)
    resident = workloads.StagedHybridDecode(wl, cuda, resident=True, **kw)
    Tc = T - W
    assert staged.h2d_bytes == 0
    for step in range(2):
        q, new = staged.inputs(step)
        staged.step(q, new)
        resident.step(q, new)
        torch.cuda.synchronize()
        assert torch.equal(staged.o, resident.o) and torch.equal(staged.lse, resident.lse)
        assert int(staged.err.item()) == 0
    # every step stages the whole compact part: ceil(Tc / 16) block rows of 2 x 8 x 1056 bytes per layer
    assert staged.h2d_bytes == 2 * 2 * (-(-Tc // 16)) * 2 * 8 * 1056
    # oracle: layer 1 after step 1 -- compact tokens [0, Tc) encoded, window [Tc, T) + 2 appended
    layer = 1
    k, v = staged.k_bits[layer], staged.v_bits[layer]                     # [T, Hkv, d]
    kh = np.zeros((8, Tc, 128))
    vh = np.zeros((8, Tc, 128))
    for h in range(8):
        ek, ev = ora.encode(k[:Tc, h]), ora.encode(v[:Tc, h])
        kh[h] = ora.dequantize(ek.codes, ek.scale_bits)
        vh[h] = ora.dequantize(ev.codes, ev.scale_bits)
    k_new = np.stack([synth.new_token(wl, layer, s)[0] for s in range(2)])
    v_new = np.stack([synth.new_token(wl, layer, s)[1] for s in range(2)])
    kwin = np.concatenate([k[Tc:], k_new]).transpose(1, 0, 2)
    vwin = np.concatenate([v[Tc:], v_new]).transpose(1, 0, 2)
    tiers = [(kh, vh), (ora.bf16_bits_to_f64(kwin), ora.bf16_bits_to_f64(vwin))]
    q1 = synth.queries(wl, layer=layer, step=1, B=1)[0]
    _, _, (o_ref, l_ref) = ora.decode_sequence(ora.bf16_bits_to_f64(q1), tiers, wl.scale, wl.split_tokens)
    assert np.max(np.abs(staged.o[layer].cpu().numpy() - o_ref)) <= 2e-3
    assert np.max(np.abs(staged.lse[layer].cpu().numpy() - l_ref)) <= 1e-3
    staged.close()


def test_suspend_and_resume_continue_bit_identically(mods, cuda, tmp_path):
    """A context suspended after two steps and resumed from its checkpoint produces the same
    bits on its next steps as a run that never stopped."""
    import torch
    akv, workloads = mods
    wl = _wl(5000)
    path = str(tmp_path / "ctx.ckpt")
    ref = workloads.StagedDecode(wl, cuda, max_steps=6)
    run = workloads.StagedDecode(wl, cuda, max_steps=6)
    for step in range(2):
        ref.step(*ref.inputs(step))
        run.step(*run.inputs(step))
    run.suspend(path)
    run.close()
    del run
    meta, sizes = akv.checkpoint_info(path)
    assert meta[5] == 2 and len(sizes) == wl.extra["layers"]
    res = workloads.StagedDecode.resume(path, wl, cuda)
    assert res.steps_done == 2
    for step in range(2, 4):
        q, new = ref.inputs(step)
        ref.step(q, new)
        res.step(q, new)
        torch.cuda.synchronize()
        assert torch.equal(ref.o, res.o) and torch.equal(ref.lse, res.lse)
    rows = ref.T + ref.steps_done  # the history both runs have written
    assert res.steps_done == ref.steps_done
    for layer in range(wl.extra["layers"]):
        assert torch.equal(ref.host[layer][:rows], res.host[layer][:rows])
    ref.close()
    res.close()


def test_stager_refuses_pageable_memory(mods, cuda):
    import torch
    akv, _ = mods
    region = torch.empty(1 << 20, dtype=torch.uint8, device=cuda)
    st = akv.Stager(region, region.numel(), 2)
    pageable = np.zeros(4096, dtype=np.uint8)
    with pytest.raises(akv.AkvError) as e:
        st.stage_chunk(pageable, 4096)
    assert e.value.status == akv.AKV_ERR_NOT_PINNED
    st.destroy()


def test_stager_waits_for_consumers_and_times_out(mods, cuda):
    """A buffer whose consumer has not finished is not reused: with a host wait limit the
    call returns AKV_ERR_TIMEOUT and copies nothing; once the consumer is done it works."""
    import torch
    akv, _ = mods
    region = torch.zeros(2 * 4096, dtype=torch.uint8, device=cuda)
    st = akv.Stager(region, region.numel(), 2)
    src = [torch.full((4096,), i + 1, dtype=torch.uint8).pin_memory() for i in range(3)]
    copy_s, cons_s = torch.cuda.Stream(cuda), torch.cuda.Stream(cuda)
    b0, p0 = st.stage_chunk(src[0], 4096, copy_s, timeout_ms=1000)
    st.use(b0, cons_s)
    with torch.cuda.stream(cons_s):
        torch.cuda._sleep(int(2e9))  # a bounded busy consumer (about a second)
    st.release(b0, cons_s)
    b1, p1 = st.stage_chunk(src[1], 4096, copy_s, timeout_ms=1000)
    assert b1 != b0
    with pytest.raises(akv.AkvError) as e:
        st.stage_chunk(src[2], 4096, copy_s, timeout_ms=20)  # buffer b0 is still in use
    assert e.value.status == akv.AKV_ERR_TIMEOUT
    cons_s.synchronize()
    copy_s.synchronize()
    assert torch.all(region[:4096] == 1)  # untouched by the refused call
    b2, p2 = st.stage_chunk(src[2], 4096, copy_s, timeout_ms=1000)
    assert b2 == b0
    copy_s.synchronize()
    assert torch.all(region[:4096] == 3) and torch.all(region[4096:] == 2)
    st.destroy()
