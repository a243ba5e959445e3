"""Window aging on the GPU: tokens that leave the exact window are encoded into the compact
tier during decode.  After the steps, every code page equals the oracle's encoding of the
grown history bit for bit (keys and values), and the step's output matches the oracle over
the compact prefix plus the remaining window."""
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


@pytest.mark.parametrize("lens,W,steps", [([100, 257, 1000], 64, 40), ([64, 79, 600], 48, 21)])
def test_window_aging_codes_and_output(mods, cuda, lens, W, steps):
    import torch
    akv, workloads = mods
    wl = synth.Workload("aging-small", B=len(lens), Hq=32, Hkv=8, d=128, split_tokens=512, extra={})
    st = workloads.AgingHybrid(wl, cuda, lens, W, max_steps=steps + 2, source="host")
    c0 = st.c.copy()
    new_k, new_v = [], []
    for s in range(steps):
        q, kn, vn = st.inputs(s)
        st.step(q, kn, vn)
        new_k.append(kn.cpu().numpy().view(np.uint16))
        new_v.append(vn.cpu().numpy().view(np.uint16))
    torch.cuda.synchronize()
    assert int(st.err.item()) == 0
    assert np.all(st.c > c0) and st.aged_blocks == int(((st.c - c0) // 16).sum())
    assert np.all(st.win >= W) and np.all(st.win < W + 16)
    cp_k, cp_v = st.cp_k.cpu().numpy(), st.cp_v.cpu().numpy()
    q_last = q.cpu().numpy().view(np.uint16)
    for b in range(len(lens)):
        k_all = np.concatenate([st.k_hist[b], np.stack([x[b] for x in new_k], axis=1)], axis=1)  # [Hkv, L+steps, d]
        v_all = np.concatenate([st.v_hist[b], np.stack([x[b] for x in new_v], axis=1)], axis=1)
        c = int(st.c[b])
        pages = st.cp_table_np[b, :c // 16]
        kh = np.zeros((8, c, 128))
        vh = np.zeros((8, c, 128))
        for h in range(8):
            ek, ev = ora.encode(k_all[h, :c]), ora.encode(v_all[h, :c])
            assert np.array_equal(cp_k[pages, h], ora.pack_blocks(ek.codes, ek.scale_bits))
            assert np.array_equal(cp_v[pages, h], ora.pack_value_blocks(ev.codes, ev.scale_bits))
            kh[h] = ora.dequantize(ek.codes, ek.scale_bits)
            vh[h] = ora.dequantize(ev.codes, ev.scale_bits)
        tiers = [(kh, vh), (ora.bf16_bits_to_f64(k_all[:, c:]), ora.bf16_bits_to_f64(v_all[:, c:]))]
        _, (o_ref, l_ref), _ = ora.decode_sequence(ora.bf16_bits_to_f64(q_last[b]), tiers, wl.scale, wl.split_tokens)
        assert np.max(np.abs(st.o[b].cpu().numpy() - o_ref)) <= 2e-3
        assert np.max(np.abs(st.lse[b].cpu().numpy() - l_ref)) <= 1e-3


def test_append_tokens_contiguous_paged_and_bounds(mods, cuda):
    import torch
    akv, _ = mods
    B, H, d, T = 3, 8, 128, 40
    gen = synth.stream(0, "test-append")
    new_k = synth.normal_bf16(gen, (B, H, d))
    new_v = synth.normal_bf16(gen, (B, H, d))
    nk, nv = torch.from_numpy(new_k.view(np.int16)).to(cuda), torch.from_numpy(new_v.view(np.int16)).to(cuda)
    err = torch.zeros(1, dtype=torch.int32, device=cuda)
    # contiguous head-major [B, H, T, d]; sequence 1 skipped
    k = torch.zeros((B, H, T, d), dtype=torch.int16, device=cuda)
    v = torch.zeros_like(k)
    tier = akv.Tier(akv.AKV_TIER_BF16, k, v, lens=[0] * B, stride_seq=H * T * d, stride_head=T * d, stride_token=d)
    akv.akv_append_tokens(tier, [5, -1, 39], B, H, d, nk, nv, err)
    torch.cuda.synchronize()
    kk, vv = k.cpu().numpy().view(np.uint16), v.cpu().numpy().view(np.uint16)
    assert np.array_equal(kk[0, :, 5], new_k[0]) and np.array_equal(vv[2, :, 39], new_v[2])
    assert np.count_nonzero(kk[1]) == 0 and np.count_nonzero(kk[0, :, :5]) == 0
    assert int(err.item()) == 0
    # paged pool [P, H, 16, d]: position 17 -> logical page 1, row 1; sequence 2's page id is out of the pool
    P = 4
    pk = torch.zeros((P, H, 16, d), dtype=torch.int16, device=cuda)
    pv = torch.zeros_like(pk)
    table = torch.tensor([[3, 1], [0, 2], [7, 9]], dtype=torch.int32, device=cuda)
    tier = akv.Tier(akv.AKV_TIER_BF16, pk, pv, lens=[0] * B, paged=True, page_table=table, page_table_stride=2,
                    n_pages=P, stride_seq=H * 16 * d, stride_head=16 * d, stride_token=d)
    akv.akv_append_tokens(tier, [17, 2, 20], B, H, d, nk, nv, err)
    torch.cuda.synchronize()
    pkk = pk.cpu().numpy().view(np.uint16)
    assert np.array_equal(pkk[1, :, 1], new_k[0]) and np.array_equal(pkk[0, :, 2], new_k[1])
    assert np.count_nonzero(pkk[2]) == 0 and np.count_nonzero(pkk[3]) == 0   # nothing written for sequence 2
    assert int(err.item()) & akv.AKV_EFLAG_BOUNDS


def test_aging_step_at_hybrid_shape_equals_separate_calls(mods, cuda):
    """At the hybrid shape (batch 4 x 32768, W = 2048) the two tiers share the GPU, and a step
    that ages no page runs its append on the window's stream just before the window's launch,
    beside the compact tier.  After every step the same attention and merge, enqueued as
    separate calls on the state the step left (the appended token included), give the step's
    output bit for bit.  20 steps include one aging step (the window reaches W + 16 at step
    16)."""
    import torch
    akv, workloads = mods
    base = synth.WORKLOADS["hybrid"]
    wl = synth.Workload("aging-hybrid-shape", base.B, base.Hq, base.Hkv, base.d, base.split_tokens, seed=base.seed,
                        extra=dict(base.extra))
    T, W = wl.extra["T"], wl.extra["window"]
    steps = 20
    st = workloads.AgingHybrid(wl, cuda, [T] * wl.B, W, max_steps=steps + 2, source="torch")
    aged0 = st.aged_blocks
    for s in range(steps):
        q, kn, vn = st.inputs(s)
        st.step(q, kn, vn)
        torch.cuda.synchronize()
        compact = akv.Tier(akv.AKV_TIER_CODES4, st.cp_k, st.cp_v, lens=st.c.astype(np.int32), paged=True,
                           page_table=st.cp_table, page_table_stride=st.cp_table_np.shape[1], n_pages=st.n_cp,
                           **st.cp_strides)
        ref = workloads.DecodeStep(st.B, wl.Hq, wl.Hkv, wl.d, wl.split_tokens, wl.scale,
                                   [compact, st._exact_tier(lens=st.win.astype(np.int32))], cuda)
        ref.step(q)
        torch.cuda.synchronize()
        assert torch.equal(ref.o, st.o) and torch.equal(ref.lse, st.lse), s
        assert int(st.err.item()) == 0 and int(ref.err.item()) == 0
    assert st.aged_blocks - aged0 == wl.B
