"""GPU parity at the sizes where the method runs: the CUDA path through the C ABI against
the float64 oracle on large launches.

  * Compact launches with several items per warp.  The compact kernel gives every warp an
    equal contiguous range of (split, KV head) items, so a launch with more items than
    warps (148 SMs x 16 warps at G <= 4, x 8 at G = 8) runs the loader's move to the next
    item, the query reload for a new (sequence, head) and the per-item epilogue.
  * The ragged paged hybrid batch at full size: batch 64, lengths uniform on
    [1024, 65536], Student-t keys, newest 1024 tokens exact.
  * The staged 128k history at full length: 131072 tokens per layer staged in 4096-token
    chunks, bit-identical to the resident run over appended steps, and the oracle.

Tolerances: codes and scales bit-exact; max |dO| <= 2e-3, |dLSE| <= 1e-3 (float32
accumulation from BF16 inputs; the compact tier against the oracle on the same dequantised
values).  The oracle runs in a spawned process pool (tests/oracle_jobs.py) on input bits
drawn by kv_cache_tiering_b200.synth.
"""
import numpy as np
import pytest

from kv_cache_tiering_b200 import synth
from oracle import akv_oracle as ora

import oracle_jobs

pytestmark = pytest.mark.gpu

TOL_O = 2e-3
TOL_LSE = 1e-3


@pytest.fixture(scope="module")
def mods():
    from kv_cache_tiering_b200 import build
    build.build()
    from kv_cache_tiering_b200 import akv, workloads
    return akv, workloads


@pytest.fixture(scope="module")
def jobs():
    with oracle_jobs.pool() as p:
        yield p


def _lse_diff(l, l_ref):
    both = np.isneginf(l) & np.isneginf(l_ref)
    return float(np.max(np.where(both, 0.0, np.abs(np.where(both, 0.0, l) - np.where(both, 0.0, l_ref))),
                        initial=0.0))


def _check_head(step, b, h, G, result, tiers=(0, 1)):
    """Partials of every tier and the merged output of sequence b, query heads of KV head h."""
    partials, _merged, direct = result
    sel = slice(h * G, (h + 1) * G)
    worst = [0.0, 0.0]
    for ti in tiers:
        base, n = step.tier_slots(ti, b)
        o_ref, l_ref = partials[ti]
        assert n == o_ref.shape[0], (b, h, ti, n, o_ref.shape)
        if n == 0:
            continue
        o = step.o_part[base:base + n, sel].cpu().numpy().astype(np.float64)
        l = step.lse_part[base:base + n, sel].cpu().numpy().astype(np.float64)
        do, dl = float(np.max(np.abs(o - o_ref))), _lse_diff(l, l_ref)
        assert do <= TOL_O and dl <= TOL_LSE, (b, h, ti, do, dl)
        worst = [max(worst[0], do), max(worst[1], dl)]
    o = step.o[b, sel].cpu().numpy().astype(np.float64)
    l = step.lse[b, sel].cpu().numpy().astype(np.float64)
    do, dl = float(np.max(np.abs(o - direct[0]))), _lse_diff(l, direct[1])
    assert do <= TOL_O and dl <= TOL_LSE, (b, h, "merged", do, dl)
    return worst


# ----------------------------------------------------------------------------------
# compact launches with several items per warp
# ----------------------------------------------------------------------------------


@pytest.mark.parametrize("B,Hq,Hkv", [(8, 32, 8), (4, 32, 4)])
def test_compact_launch_with_several_items_per_warp(mods, cuda, jobs, B, Hq, Hkv):
    """40960 tokens per sequence, the newest 2048 exact: 76 compact splits per (sequence,
    head), 4864 items at G = 4 (2368 warps) and 1216 at G = 8 (1184 warps).  Every KV head
    of the first and the last sequence and one KV head of every other sequence are checked
    against the oracle (codes bit-exact, partials of both tiers, merged output)."""
    import torch
    akv, workloads = mods
    G = Hq // Hkv
    wl = synth.Workload(f"multi-item-g{G}", B=B, Hq=Hq, Hkv=Hkv, d=128, split_tokens=512,
                        extra={"T": 40960, "window": 2048})
    w = workloads.HybridResident(wl, cuda)
    Tc = w.T - w.W
    n_items = B * Hkv * (-(-Tc // wl.split_tokens))
    warps = torch.cuda.get_device_properties(cuda).multi_processor_count * (16 if G <= 4 else 8)
    assert n_items > warps, (n_items, warps)
    w.step.step(w.q, akv.AKV_VARIANT_MMA)
    torch.cuda.synchronize()
    assert int(w.enc_err.item()) == 0 and int(w.step.err.item()) == 0
    heads = [(b, h) for b in (0, B - 1) for h in range(Hkv)] + [(b, (3 * b) % Hkv) for b in range(1, B - 1)]
    futs = {(b, h): jobs.submit(oracle_jobs.hybrid_head, w.q_bits[b, h * G:(h + 1) * G], w.k_bits[b, h],
                                w.v_bits[b, h], Tc, wl.scale, wl.split_tokens) for b, h in heads}
    kc, vc = w.kc.cpu().numpy(), w.vc.cpu().numpy()
    for (b, h), f in futs.items():
        (kb, vb), result = f.result()
        assert np.array_equal(kc[b, h], kb) and np.array_equal(vc[b, h], vb), (b, h)
        _check_head(w.step, b, h, G, result)


# ----------------------------------------------------------------------------------
# ragged paged hybrid batch at full size
# ----------------------------------------------------------------------------------


def test_ragged_paged_hybrid_full_size(mods, cuda, jobs):
    """Batch 64, lengths U[1024, 65536], 16-token pages through seeded permutations,
    Student-t keys, newest 1024 exact: the launch the bench times.  One KV head of every
    sequence, and every KV head of the shortest and the longest sequence, against the
    oracle: code pages bit-exact, partials of both tiers, merged output."""
    import torch
    akv, workloads = mods
    wl = synth.WORKLOADS["ragged"]
    w = workloads.RaggedPaged(wl, cuda, generator="torch")
    assert w.B == 64
    w.step.step(w.q, akv.AKV_VARIANT_AUTO)
    torch.cuda.synchronize()
    assert int(w.enc_err.item()) == 0 and int(w.step.err.item()) == 0
    G = wl.Hq // wl.Hkv
    lens = w.lens
    shortest, longest = int(np.argmin(lens)), int(np.argmax(lens))
    futs = {}
    for b in range(w.B):
        L, c = int(lens[b]), int(w.cp_len[b])
        k, v = synth.torch_sequence_kv(wl, b, L, "student_t", device=cuda)
        k = k.cpu().numpy().view(np.uint16)
        v = v.cpu().numpy().view(np.uint16)
        heads = range(wl.Hkv) if b in (shortest, longest) else [b % wl.Hkv]
        for h in heads:
            futs[(b, h)] = jobs.submit(oracle_jobs.hybrid_head, w.q_bits[b, h * G:(h + 1) * G], k[h].copy(),
                                       v[h].copy(), c, wl.scale, wl.split_tokens)
    cp_k, cp_v = w.cp_k.cpu().numpy(), w.cp_v.cpu().numpy()
    table = w.cp_table_np
    for (b, h), f in futs.items():
        (kb, vb), result = f.result()
        n_pages = -(-int(w.cp_len[b]) // 16)
        if n_pages:
            rows = table[b, :n_pages]
            assert np.array_equal(cp_k[rows, h], kb) and np.array_equal(cp_v[rows, h], vb), (b, h)
        _check_head(w.step, b, h, G, result)


# ----------------------------------------------------------------------------------
# staged 128k history at full length
# ----------------------------------------------------------------------------------


def test_staged_full_length_equals_resident_and_oracle(mods, cuda, jobs):
    """131072 BF16 tokens per layer, 2 layers, 4096-token chunks through a 2-buffer ring
    (32 chunks per layer, 33 once a token is appended): two appended steps staged equal
    the resident run bit for bit, and layer 1 after the second step matches the oracle."""
    import torch
    akv, workloads = mods
    base = synth.WORKLOADS["staged"]
    wl = synth.Workload(base.name, base.B, base.Hq, base.Hkv, base.d, base.split_tokens,
                        extra=dict(base.extra, layers=2))
    T = wl.extra["T"]
    staged = workloads.StagedDecode(wl, cuda, max_steps=4)
    copies = []
    for h in staged.host:  # the resident run gets its own copy of the same host history
        c = torch.empty_like(h).pin_memory()
        c.copy_(h)
        copies.append(c)
    resident = workloads.StagedDecode(wl, cuda, max_steps=4, resident=True, host_layers=copies)
    for step in range(2):
        q, new = staged.inputs(step)
        staged.step(q, new)
        resident.step(q, new)
        torch.cuda.synchronize()
        n_split = -(-(T + step + 1) // wl.split_tokens)
        assert torch.equal(staged.o_part[:n_split], resident.o_part[:n_split]), step
        assert torch.equal(staged.lse_part[:n_split], resident.lse_part[:n_split]), step
        assert torch.equal(staged.o, resident.o) and torch.equal(staged.lse, resident.lse), step
        assert int(staged.err.item()) == 0
    layer = 1
    k, v = synth.history_token_major(wl, layer, T)
    k_new = np.stack([synth.new_token(wl, layer, s)[0] for s in range(2)])
    v_new = np.stack([synth.new_token(wl, layer, s)[1] for s in range(2)])
    k_all = np.concatenate([k, k_new])
    v_all = np.concatenate([v, v_new])
    del k, v
    q1 = synth.queries(wl, layer=layer, step=1, B=1)[0]
    G = wl.Hq // wl.Hkv
    futs = {h: jobs.submit(oracle_jobs.exact_head, q1[h * G:(h + 1) * G], np.ascontiguousarray(k_all[:, h]),
                           np.ascontiguousarray(v_all[:, h]), wl.scale, wl.split_tokens) for h in range(wl.Hkv)}
    o = staged.o[layer].cpu().numpy().astype(np.float64)
    l = staged.lse[layer].cpu().numpy().astype(np.float64)
    for h, f in futs.items():
        _partials, _merged, (o_ref, l_ref) = f.result()
        sel = slice(h * G, (h + 1) * G)
        assert np.max(np.abs(o[sel] - o_ref)) <= TOL_O, h
        assert np.max(np.abs(l[sel] - l_ref)) <= TOL_LSE, h
    staged.close()
