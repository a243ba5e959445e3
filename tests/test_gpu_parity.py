"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Codes and scales bit-exact; max |dO| <= 2e-3 and |dLSE| <= 1e-3 for attention (float32
accumulation from BF16 inputs; the compact tier is compared on the same dequantised
values); bit-identical repeat runs."""
import math

import numpy as np
import pytest

from kv_cache_tiering_b200 import synth
from oracle import akv_oracle as ora

pytestmark = pytest.mark.gpu

TOL_O = 2e-3
TOL_LSE = 1e-3
VARIANTS = ["simt", "mma"]


@pytest.fixture(scope="module")
def akv():
    from kv_cache_tiering_b200 import build
    build.build()
    from kv_cache_tiering_b200 import akv as mod
    return mod


@pytest.fixture(scope="module")
def wlmod():
    from kv_cache_tiering_b200 import workloads
    return workloads


def variant_id(akv, name):
    return {"simt": akv.AKV_VARIANT_SIMT, "mma": akv.AKV_VARIANT_MMA, "auto": akv.AKV_VARIANT_AUTO}[name]


def f64(bits):
    return ora.bf16_bits_to_f64(bits)


def check_partials(step, tier_idx, b, oracle_partials, hq_sel=None):
    """Compare GPU partial slots of (tier, sequence) with the oracle's (O [S, Hq, d], LSE [S, Hq])."""
    o_ref, l_ref = oracle_partials
    base, n = step.tier_slots(tier_idx, b)
    assert n == o_ref.shape[0]
    if n == 0:
        return 0.0, 0.0
    o = step.o_part[base:base + n].cpu().numpy().astype(np.float64)
    l = step.lse_part[base:base + n].cpu().numpy().astype(np.float64)
    if hq_sel is not None:
        o, l, o_ref, l_ref = o[:, hq_sel], l[:, hq_sel], o_ref[:, hq_sel], l_ref[:, hq_sel]
    do, dl = float(np.max(np.abs(o - o_ref))), float(np.max(np.abs(l - l_ref)))
    assert do <= TOL_O, (tier_idx, b, do)
    assert dl <= TOL_LSE, (tier_idx, b, dl)
    return do, dl


def lse_diff(l, l_ref):
    """|dLSE| with -inf == -inf counted as no difference."""
    both = np.isneginf(l) & np.isneginf(l_ref)
    return float(np.max(np.where(both, 0.0, np.abs(np.where(both, 0.0, l) - np.where(both, 0.0, l_ref)))))


def check_merged(step, b, ref, hq_sel=None):
    o_ref, l_ref = ref
    o = step.o[b].cpu().numpy().astype(np.float64)
    l = step.lse[b].cpu().numpy().astype(np.float64)
    if hq_sel is not None:
        o, l, o_ref, l_ref = o[hq_sel], l[hq_sel], o_ref[hq_sel], l_ref[hq_sel]
    do, dl = float(np.max(np.abs(o - o_ref))), lse_diff(l, l_ref)
    assert do <= TOL_O, (b, do)
    assert dl <= TOL_LSE, (b, dl)


# ----------------------------------------------------------------------------------
# encode
# ----------------------------------------------------------------------------------


def _encode_case(akv, wlmod, cuda, x_bits, d, paged, signs=0):
    """Encode one (sequence, head) stream of n vectors [n, d] on the GPU; return its blocks."""
    import torch
    n = x_bits.shape[0]
    nb = -(-n // 16)
    bb = akv.codes4_block_bytes(d)
    src_k = wlmod.to_dev_bits(x_bits, cuda)
    src_v = wlmod.to_dev_bits(x_bits[::-1].copy(), cuda)
    err = torch.zeros(1, dtype=torch.int32, device=cuda)
    src = akv.Tier(akv.AKV_TIER_BF16, src_k, src_v, lens=[n], stride_seq=0, stride_head=0, stride_token=d)
    if paged:
        perm = np.random.default_rng(n).permutation(nb + 3).astype(np.int32)
        table = torch.from_numpy(perm[:nb].copy()).to(cuda)
        kc = torch.full((nb + 3, bb), 0xAB, dtype=torch.uint8, device=cuda)
        vc = torch.full((nb + 3, bb), 0xAB, dtype=torch.uint8, device=cuda)
        dst = akv.Tier(akv.AKV_TIER_CODES4, kc, vc, lens=[n], paged=True, page_table=table, page_table_stride=nb,
                       n_pages=nb + 3, stride_seq=1, stride_head=0, rotation_signs=signs)
    else:
        kc = torch.full((nb, bb), 0xAB, dtype=torch.uint8, device=cuda)
        vc = torch.full((nb, bb), 0xAB, dtype=torch.uint8, device=cuda)
        dst = akv.Tier(akv.AKV_TIER_CODES4, kc, vc, lens=[n], stride_seq=0, stride_head=0, stride_token=1,
                       rotation_signs=signs)
    akv.akv_encode_history(src, dst, 1, 1, d, err)
    torch.cuda.synchronize()
    kb, vb = kc.cpu().numpy(), vc.cpu().numpy()
    if paged:
        kb, vb = kb[perm[:nb]], vb[perm[:nb]]
    return kb, vb, int(err.item())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("paged", [False, True])
def test_encode_bit_exact(akv, wlmod, cuda, d, paged):
    gen = synth.stream(0, "test-encode", d, int(paged))
    n = 16 * 37 + 5  # ragged: a partial last block
    x = np.concatenate([synth.normal_bf16(gen, (n // 2, d)),
                        synth.student_t_bf16(gen, (n - n // 2 - 3, d), 3.0),
                        np.zeros((1, d), np.uint16),                       # zero vector
                        synth.f32_to_bf16_bits(np.full((1, d), 1e-30, np.float32)),  # tiny norm
                        synth.f32_to_bf16_bits(np.full((1, d), 3.0, np.float32))])  # exact ties possible
    kb, vb, err = _encode_case(akv, wlmod, cuda, x, d, paged)
    assert err == 0
    for blocks, xs, pack in ((kb, x, ora.pack_blocks), (vb, x[::-1], ora.pack_value_blocks)):
        enc = ora.encode(xs)
        want = pack(enc.codes, enc.scale_bits)
        assert np.array_equal(blocks, want)


@pytest.mark.parametrize("d", [64, 128])
def test_encode_bit_exact_with_rotation_signs(akv, wlmod, cuda, d):
    gen = synth.stream(0, "test-encode-signs", d)
    x = np.concatenate([synth.normal_bf16(gen, (40, d)), synth.student_t_bf16(gen, (9, d), 3.0)])
    bits = synth.rotation_sign_bits(0, d, "test-encode")
    kb, vb, err = _encode_case(akv, wlmod, cuda, x, d, False, signs=bits)
    assert err == 0
    ek, ev = ora.encode(x, bits), ora.encode(x[::-1], bits)
    assert np.array_equal(kb, ora.pack_blocks(ek.codes, ek.scale_bits))
    assert np.array_equal(vb, ora.pack_value_blocks(ev.codes, ev.scale_bits))
    assert not np.array_equal(ek.codes, ora.encode(x).codes)  # the signs change the codes


def test_encode_refusals_flag_and_zero_encode(akv, wlmod, cuda):
    d = 128
    gen = synth.stream(0, "test-encode-refuse")
    x = synth.normal_bf16(gen, (32, d))
    x[3, 7] = 0x7F80                                          # +inf
    x[9, 0] = 0x7FC0                                          # NaN
    x[20] = synth.f32_to_bf16_bits(np.full(d, 6000.0, np.float32))  # norm overflows binary16
    kb, vb, err = _encode_case(akv, wlmod, cuda, x, d, False)
    assert err & akv.AKV_EFLAG_NONFINITE and err & akv.AKV_EFLAG_RANGE
    enc = ora.encode(x)
    assert enc.nonfinite[3] and enc.nonfinite[9] and enc.overflow[20]
    assert np.array_equal(kb, ora.pack_blocks(enc.codes, enc.scale_bits))
    ev = ora.encode(x[::-1])
    assert np.array_equal(vb, ora.pack_value_blocks(ev.codes, ev.scale_bits))


# ----------------------------------------------------------------------------------
# exact tier
# ----------------------------------------------------------------------------------


def _oracle_exact(wl, q_bits, k_bits, v_bits, lens, split):
    out = []
    for b in range(q_bits.shape[0]):
        T = int(lens[b])
        tiers = [(f64(k_bits[b][:, :T]), f64(v_bits[b][:, :T]))]
        out.append(ora.decode_sequence(f64(q_bits[b]), tiers, wl.scale, split))
    return out


@pytest.mark.parametrize("variant", VARIANTS)
def test_tiny_exact(akv, wlmod, cuda, variant):
    import torch
    wl = synth.WORKLOADS["tiny"]
    w = wlmod.ExactResident(wl, cuda)
    w.step.step(w.q, variant_id(akv, variant))
    torch.cuda.synchronize()
    ref = _oracle_exact(wl, w.q_bits, w.k_bits, w.v_bits, [w.T], wl.split_tokens)[0]
    check_partials(w.step, 0, 0, ref[0][0])
    check_merged(w.step, 0, ref[2])
    check_merged(w.step, 0, ref[1])
    assert w.step.n_slots == 4 and int(w.step.err.item()) == 0


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("G,d", [(4, 128), (8, 128), (2, 64), (1, 128)])
def test_exact_ragged_lengths(akv, wlmod, cuda, variant, G, d):
    """Ragged lengths (tails of every size, a 1-token split, an empty sequence), several
    tiles per split, token-major and head-major strides."""
    import torch
    Hkv = 2
    wl = synth.Workload("exact-ragged", B=5, Hq=Hkv * G, Hkv=Hkv, d=d, split_tokens=128)
    T = 700
    lens = np.array([700, 513, 129, 0, 1], np.int32)
    gen = synth.stream(0, "exact-ragged", G, d)
    q_bits = synth.normal_bf16(gen, (wl.B, wl.Hq, d))
    # token-major storage [B, T, Hkv, d]
    k_tm = synth.normal_bf16(gen, (wl.B, T, Hkv, d))
    v_tm = synth.normal_bf16(gen, (wl.B, T, Hkv, d))
    q = wlmod.to_dev_bits(q_bits, cuda)
    k = wlmod.to_dev_bits(k_tm, cuda)
    v = wlmod.to_dev_bits(v_tm, cuda)
    tier = akv.Tier(akv.AKV_TIER_BF16, k, v, lens=lens, stride_seq=T * Hkv * d, stride_head=d, stride_token=Hkv * d)
    step = wlmod.DecodeStep(wl.B, wl.Hq, Hkv, d, wl.split_tokens, wl.scale, [tier], cuda)
    step.step(q, variant_id(akv, variant))
    torch.cuda.synchronize()
    k_hm = np.ascontiguousarray(k_tm.transpose(0, 2, 1, 3))
    v_hm = np.ascontiguousarray(v_tm.transpose(0, 2, 1, 3))
    refs = _oracle_exact(wl, q_bits, k_hm, v_hm, lens, wl.split_tokens)
    for b in range(wl.B):
        check_partials(step, 0, b, refs[b][0][0])
        check_merged(step, b, refs[b][2])
    assert np.all(step.lse[3].cpu().numpy() == -np.inf) and np.all(step.o[3].cpu().numpy() == 0)


@pytest.mark.parametrize("variant", VARIANTS)
def test_exact_gqa_full_size(akv, wlmod, cuda, variant):
    """Batch 8, 32/8 heads, d 128, 8192 tokens, 512-token splits: every output checked."""
    import torch
    wl = synth.WORKLOADS["exact"]
    w = wlmod.ExactResident(wl, cuda)
    w.step.step(w.q, variant_id(akv, variant))
    torch.cuda.synchronize()
    refs = _oracle_exact(wl, w.q_bits, w.k_bits, w.v_bits, [w.T] * w.B, wl.split_tokens)
    for b in range(w.B):
        check_partials(w.step, 0, b, refs[b][0][0])
        check_merged(w.step, b, refs[b][2])
    # determinism: a second run is bit-identical
    o1, l1 = w.step.o.clone(), w.step.lse.clone()
    w.step.step(w.q, variant_id(akv, variant))
    torch.cuda.synchronize()
    assert torch.equal(o1, w.step.o) and torch.equal(l1, w.step.lse)


# ----------------------------------------------------------------------------------
# compact and hybrid tiers
# ----------------------------------------------------------------------------------


def _oracle_hybrid(wl, w, b, heads=None):
    """Oracle for sequence b of a HybridResident: encode the old part, dequantise, attend."""
    bits = getattr(w, "rotation_signs", 0)
    Tc = w.T - w.W
    kk = w.k_bits[b]
    vv = w.v_bits[b]
    H = wl.Hkv
    kh = np.zeros((H, Tc, wl.d))
    vh = np.zeros((H, Tc, wl.d))
    codes = []
    for h in range(H):
        ek = ora.encode(kk[h, :Tc], bits)
        ev = ora.encode(vv[h, :Tc], bits)
        kh[h] = ora.dequantize(ek.codes, ek.scale_bits, bits)
        vh[h] = ora.dequantize(ev.codes, ev.scale_bits, bits)
        codes.append((ora.pack_blocks(ek.codes, ek.scale_bits), ora.pack_value_blocks(ev.codes, ev.scale_bits)))
    tiers = [(kh, vh), (f64(kk[:, Tc:]), f64(vv[:, Tc:]))]
    return ora.decode_sequence(f64(w.q_bits[b]), tiers, wl.scale, wl.split_tokens), codes


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("T,W,d,G", [(3001, 1000, 128, 4), (1100, 300, 64, 8), (2000, 0, 128, 1),
                                     (1500, 200, 64, 1), (1700, 300, 128, 2), (900, 100, 64, 2),
                                     (1200, 400, 128, 8)])
def test_hybrid_small(akv, wlmod, cuda, variant, T, W, d, G):
    """Every (d, G) the compact kernel is built for: its per-head lane groups hold 2 to 32
    coordinates per lane (G = 1 at d = 64 up to G = 8 at d = 128)."""
    import torch
    wl = synth.Workload("hybrid-small", B=2, Hq=2 * G, Hkv=2, d=d, split_tokens=256, extra={"T": T, "window": W})
    w = wlmod.HybridResident(wl, cuda)
    w.step.step(w.q, variant_id(akv, variant))
    torch.cuda.synchronize()
    assert int(w.enc_err.item()) == 0
    kc, vc = w.kc.cpu().numpy(), w.vc.cpu().numpy()
    for b in range(w.B):
        (partials, merged, direct), codes = _oracle_hybrid(wl, w, b)
        for h in range(wl.Hkv):
            assert np.array_equal(kc[b, h], codes[h][0]) and np.array_equal(vc[b, h], codes[h][1])
        check_partials(w.step, 0, b, partials[0])
        check_partials(w.step, 1, b, partials[1])
        check_merged(w.step, b, direct)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("T,W,d,G", [(2600, 600, 128, 4), (1100, 300, 64, 8)])
def test_hybrid_rotation_signs(akv, wlmod, cuda, variant, T, W, d, G):
    """A randomised-sign rotation: codes, partials and merged output against the oracle."""
    import torch
    wl = synth.Workload("hybrid-signs", B=2, Hq=2 * G, Hkv=2, d=d, split_tokens=256, extra={"T": T, "window": W})
    w = wlmod.HybridResident(wl, cuda, rotation_signs=synth.rotation_sign_bits(1, d))
    w.step.step(w.q, variant_id(akv, variant))
    torch.cuda.synchronize()
    assert int(w.enc_err.item()) == 0
    kc, vc = w.kc.cpu().numpy(), w.vc.cpu().numpy()
    for b in range(w.B):
        (partials, merged, direct), codes = _oracle_hybrid(wl, w, b)
        for h in range(wl.Hkv):
            assert np.array_equal(kc[b, h], codes[h][0]) and np.array_equal(vc[b, h], codes[h][1])
        check_partials(w.step, 0, b, partials[0])
        check_merged(w.step, b, direct)


@pytest.mark.parametrize("variant", VARIANTS)
def test_hybrid_full_size_sampled(akv, wlmod, cuda, variant):
    """Batch 4, 32 768 tokens (newest 2048 exact, 30 720 compact), 32/8 heads: the full
    launch runs; codes of two KV heads per sequence and the outputs of their query
    heads are checked against the oracle."""
    import torch
    wl = synth.WORKLOADS["hybrid"]
    w = wlmod.HybridResident(wl, cuda)
    w.step.step(w.q, variant_id(akv, variant))
    torch.cuda.synchronize()
    assert int(w.enc_err.item()) == 0
    G = wl.Hq // wl.Hkv
    Tc = w.T - w.W
    kc, vc = w.kc.cpu().numpy(), w.vc.cpu().numpy()
    for b in range(w.B):
        for h in (b % wl.Hkv, (b + 5) % wl.Hkv):
            ek = ora.encode(w.k_bits[b, h, :Tc])
            ev = ora.encode(w.v_bits[b, h, :Tc])
            assert np.array_equal(kc[b, h], ora.pack_blocks(ek.codes, ek.scale_bits))
            assert np.array_equal(vc[b, h], ora.pack_value_blocks(ev.codes, ev.scale_bits))
            kh = ora.dequantize(ek.codes, ek.scale_bits)[None]
            vh = ora.dequantize(ev.codes, ev.scale_bits)[None]
            qh = f64(w.q_bits[b, h * G:(h + 1) * G])
            tiers = [(kh, vh), (f64(w.k_bits[b, h:h + 1, Tc:]), f64(w.v_bits[b, h:h + 1, Tc:]))]
            partials, merged, direct = ora.decode_sequence(qh, tiers, wl.scale, wl.split_tokens)
            sel = slice(h * G, (h + 1) * G)
            for ti in range(2):
                base, n = w.step.tier_slots(ti, b)
                o = w.step.o_part[base:base + n, sel].cpu().numpy()
                l = w.step.lse_part[base:base + n, sel].cpu().numpy()
                assert np.max(np.abs(o - partials[ti][0])) <= TOL_O
                assert np.max(np.abs(l - partials[ti][1])) <= TOL_LSE
            assert np.max(np.abs(w.step.o[b, sel].cpu().numpy() - direct[0])) <= TOL_O
            assert np.max(np.abs(w.step.lse[b, sel].cpu().numpy() - direct[1])) <= TOL_LSE


@pytest.mark.parametrize("variant", VARIANTS)
def test_ragged_paged_hybrid_small(akv, wlmod, cuda, variant):
    """Ragged batch, 16-token pages through permuted page tables, Student-t keys, newest
    window exact and the rest compact; lengths below, at and above the window."""
    import torch
    wl = synth.Workload("ragged-small", B=6, Hq=32, Hkv=8, d=128, split_tokens=512,
                        extra={"window": 1024, "nu": 3.0})
    lens = np.array([1024, 1023, 1025, 3000, 17, 5000], np.int32)
    w = wlmod.RaggedPaged(wl, cuda, lens=lens)
    w.step.step(w.q, variant_id(akv, variant))
    torch.cuda.synchronize()
    assert int(w.enc_err.item()) == 0 and int(w.step.err.item()) == 0
    for b in range(w.B):
        k, v = synth.history_head_major(wl, b, int(lens[b]), key_dist="student_t")
        c = int(w.cp_len[b])
        kh = np.zeros((wl.Hkv, c, wl.d))
        vh = np.zeros((wl.Hkv, c, wl.d))
        for h in range(wl.Hkv):
            if c:
                ek, ev = ora.encode(k[h, :c]), ora.encode(v[h, :c])
                kh[h] = ora.dequantize(ek.codes, ek.scale_bits)
                vh[h] = ora.dequantize(ev.codes, ev.scale_bits)
        tiers = [(kh, vh), (f64(k[:, c:]), f64(v[:, c:]))]
        partials, merged, direct = ora.decode_sequence(f64(w.q_bits[b]), tiers, wl.scale, wl.split_tokens)
        check_partials(w.step, 0, b, partials[0])
        check_partials(w.step, 1, b, partials[1])
        check_merged(w.step, b, direct)


def test_bad_page_id_sets_bounds_flag(akv, wlmod, cuda):
    import torch
    d, H = 128, 2
    pool = torch.zeros((4, H, 16, d), dtype=torch.int16, device=cuda)
    table = torch.tensor([[0, 7]], dtype=torch.int32, device=cuda)  # page 7 is outside the pool
    tier = akv.Tier(akv.AKV_TIER_BF16, pool, pool, lens=[32], paged=True, page_table=table, page_table_stride=2,
                    n_pages=4, stride_seq=H * 16 * d, stride_head=16 * d, stride_token=d)
    q = torch.zeros((1, 8, d), dtype=torch.int16, device=cuda)
    step = wlmod.DecodeStep(1, 8, H, d, 16, 0.1, [tier], cuda)
    step.step(q)
    torch.cuda.synchronize()
    assert int(step.err.item()) & akv.AKV_EFLAG_BOUNDS
    assert akv.error_word_status(int(step.err.item())) == akv.AKV_ERR_BOUNDS


def test_merge_special_values(akv, cuda):
    """Empty partials (-inf) are ignored; a sequence without partials gives O = 0, LSE = -inf."""
    import torch
    Hq, d = 2, 64
    gen = np.random.default_rng(3)
    o_part = gen.standard_normal((5, Hq, d)).astype(np.float32)
    lse_part = gen.standard_normal((5, Hq)).astype(np.float32)
    lse_part[1, :] = -np.inf
    o_d = torch.from_numpy(o_part).to(cuda)
    l_d = torch.from_numpy(lse_part).to(cuda)
    o = torch.empty((3, Hq, d), device=cuda)
    lse = torch.empty((3, Hq), device=cuda)
    akv.akv_merge_lse(o_d, l_d, 5, [0, 3, 0], [3, 2, 0], 3, Hq, d, o, lse)
    torch.cuda.synchronize()
    for b, (a, n) in enumerate([(0, 3), (3, 2)]):
        for h in range(Hq):
            ro, rl = ora.merge_lse(o_part[a:a + n, h].astype(np.float64), lse_part[a:a + n, h].astype(np.float64))
            assert np.max(np.abs(o[b, h].cpu().numpy() - ro)) < 1e-5
            assert abs(lse[b, h].item() - rl) < 1e-5
    assert torch.all(o[2] == 0) and torch.all(lse[2] == -math.inf)


# ----------------------------------------------------------------------------------
# one-call decode (akv_decode: every tier's attention launch and the merge launch)
# ----------------------------------------------------------------------------------


def _fused_check(akv, step, q, refs_direct):
    """akv_decode plans the standard slot layout itself and runs the same launches as
    akv_decode_attend + akv_merge_lse: the same bits, and the oracle's values."""
    import torch
    o_sep, l_sep = step.o.clone(), step.lse.clone()
    step.o.fill_(float("nan"))
    step.lse.fill_(float("nan"))
    step.decode(q)
    torch.cuda.synchronize()
    assert torch.equal(step.o.view(torch.int32), o_sep.view(torch.int32))
    assert torch.equal(step.lse.view(torch.int32), l_sep.view(torch.int32))
    for b, ref in enumerate(refs_direct):
        check_merged(step, b, ref)
    o1, l1 = step.o.clone(), step.lse.clone()
    step.decode(q)  # a second call on the same workspace gives the same bits
    torch.cuda.synchronize()
    assert torch.equal(o1, step.o) and torch.equal(l1, step.lse)


def test_fused_decode_exact_full_size(akv, wlmod, cuda):
    import torch
    wl = synth.WORKLOADS["exact"]
    w = wlmod.ExactResident(wl, cuda)
    w.step.step(w.q)
    torch.cuda.synchronize()
    refs = [r[2] for r in _oracle_exact(wl, w.q_bits, w.k_bits, w.v_bits, [w.T] * w.B, wl.split_tokens)]
    _fused_check(akv, w.step, w.q, refs)


def test_fused_decode_ragged_paged_hybrid(akv, wlmod, cuda):
    """The one-call decode of a ragged paged hybrid batch, one sequence with no compact
    tokens."""
    import torch
    wl = synth.Workload("ragged-fused", B=5, Hq=32, Hkv=8, d=128, split_tokens=512,
                        extra={"window": 1024, "nu": 3.0})
    lens = np.array([700, 1024, 3000, 1500, 4100], np.int32)
    w = wlmod.RaggedPaged(wl, cuda, lens=lens)
    w.step.step(w.q)
    torch.cuda.synchronize()
    refs = []
    for b in range(w.B):
        k, v = synth.history_head_major(wl, b, int(lens[b]), key_dist="student_t")
        c = int(w.cp_len[b])
        kh = np.zeros((wl.Hkv, c, wl.d))
        vh = np.zeros((wl.Hkv, c, wl.d))
        for h in range(wl.Hkv):
            if c:
                ek, ev = ora.encode(k[h, :c]), ora.encode(v[h, :c])
                kh[h] = ora.dequantize(ek.codes, ek.scale_bits)
                vh[h] = ora.dequantize(ev.codes, ev.scale_bits)
        tiers = [(kh, vh), (f64(k[:, c:]), f64(v[:, c:]))]
        refs.append(ora.decode_sequence(f64(w.q_bits[b]), tiers, wl.scale, wl.split_tokens)[2])
    _fused_check(akv, w.step, w.q, refs)


def test_fused_decode_refuses_small_workspace(akv, wlmod, cuda):
    wl = synth.WORKLOADS["tiny"]
    w = wlmod.ExactResident(wl, cuda)
    with pytest.raises(akv.AkvError) as e:
        akv.akv_decode(w.q, w.B, wl.Hq, wl.Hkv, wl.d, wl.scale, w.step.tiers, wl.split_tokens, w.step.workspace,
                       w.step.ws_bytes - 256, w.step.o, w.step.lse)
    assert e.value.status == akv.AKV_ERR_BUDGET


@pytest.mark.parametrize("which", ["hybrid", "ragged"])
def test_side_by_side_tiers_match_serial(akv, wlmod, cuda, which):
    """One call over both tiers runs the compact and BF16 launches side by side on disjoint
    SMs; its partials and merged outputs are the same bits as the two tiers launched one
    after the other with full grids."""
    import torch
    if which == "hybrid":
        w = wlmod.HybridResident(synth.WORKLOADS["hybrid"], cuda)
    else:
        wl = synth.Workload("ragged-side", B=12, Hq=32, Hkv=8, d=128, split_tokens=512,
                            extra={"window": 1024, "nu": 3.0})
        lens = np.array([700, 1024, 1025, 3000, 17, 5000, 9000, 2047, 1, 4096, 12000, 1500], np.int32)
        w = wlmod.RaggedPaged(wl, cuda, lens=lens)
    step = w.step
    runs = []
    for serial in (False, True, False):
        step.o_part.fill_(float("nan"))
        step.lse_part.fill_(float("nan"))
        if serial:
            for i in range(len(step.tiers)):
                step.attend_tier(i, w.q)
            step.merge()
        else:
            step.step(w.q)
        torch.cuda.synchronize()
        assert int(step.err.item()) == 0
        runs.append([t.clone() for t in (step.o_part, step.lse_part, step.o, step.lse)])
    for a, b in zip(runs[0], runs[1]):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    for a, b in zip(runs[0], runs[2]):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("G,d", [(4, 128), (8, 64)])
def test_hybrid_step_replays_from_cuda_graph(akv, wlmod, cuda, G, d):
    """A decode step (the two tiers side by side, then the merge) captured into a CUDA graph
    and replayed gives the same bits as the step run eagerly: the library's fork onto its
    side stream and the join back are recorded as graph dependencies."""
    import torch
    wl = synth.Workload("hybrid-graph", B=3, Hq=8 * G, Hkv=8, d=d, split_tokens=512,
                        extra={"T": 9000, "window": 2048})
    w = wlmod.HybridResident(wl, cuda)
    step = w.step
    outs = (step.o, step.lse, step.o_part, step.lse_part)
    s = torch.cuda.Stream(cuda)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step.step(w.q)  # eager; also creates the library's per-device state before capture
    s.synchronize()
    assert int(step.err.item()) == 0
    ref = [t.clone() for t in outs]
    for t in outs:
        t.fill_(float("nan"))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step.step(w.q)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        assert int(step.err.item()) == 0
        for a, b in zip(ref, outs):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    del g


@pytest.mark.parametrize("flags", [0, 1])
@pytest.mark.parametrize("which", ["hybrid", "exact", "ragged"])
def test_decode_host_matches_device_step(akv, wlmod, cuda, which, flags):
    """akv_decode_host with the query and the results in page-locked host memory (flags 0:
    the GPU reads and writes the host arrays itself; AKV_HOST_COPY_ENGINE: copy-engine
    transfers) gives the bits of the device-memory step (akv_decode_attend + akv_merge_lse);
    two calls in a row with alternating output buffers agree."""
    import torch
    if which == "hybrid":
        w = wlmod.HybridResident(synth.WORKLOADS["hybrid"], cuda)
    elif which == "exact":
        w = wlmod.ExactResident(synth.WORKLOADS["exact"], cuda, B=3, T=3000)
    else:
        wl = synth.Workload("ragged-host", B=5, Hq=32, Hkv=8, d=128, split_tokens=512,
                            extra={"window": 1024, "nu": 3.0})
        w = wlmod.RaggedPaged(wl, cuda, lens=np.array([700, 1024, 3000, 17, 4100], np.int32))
    step = w.step
    step.step(w.q)
    torch.cuda.synchronize()
    ref_o, ref_lse = step.o.cpu(), step.lse.cpu()
    q_host = torch.from_numpy(w.q_bits.view(np.int16)).pin_memory()
    outs = [(torch.full(step.o.shape, float("nan")).pin_memory(), torch.full(step.lse.shape, float("nan")).pin_memory())
            for _ in range(2)]
    for o_h, l_h in outs:
        step.decode_host(q_host, o_h, l_h, flags)
    torch.cuda.synchronize()
    assert int(step.err.item()) == 0
    for o_h, l_h in outs:
        assert torch.equal(o_h.view(torch.int32), ref_o.view(torch.int32))
        assert torch.equal(l_h.view(torch.int32), ref_lse.view(torch.int32))


@pytest.mark.parametrize("variant", ["simt", "mma"])
def test_hybrid_more_sequences_than_one_launch(akv, wlmod, cuda, variant):
    """300 sequences: each tier takes two launches (256 sequences at most per launch), so a
    step makes four attention launches.  Sampled sequences match the oracle, and
    akv_decode_host (its query copy enqueued before the first of the four) gives the step's
    bits."""
    import torch
    wl = synth.Workload("hybrid-many", B=300, Hq=8, Hkv=2, d=64, split_tokens=64, extra={"T": 150, "window": 50})
    w = wlmod.HybridResident(wl, cuda)
    step = w.step
    step.step(w.q, variant_id(akv, variant))
    torch.cuda.synchronize()
    assert int(w.enc_err.item()) == 0 and int(step.err.item()) == 0
    for b in (0, 1, 255, 256, 299):
        (partials, merged, direct), _ = _oracle_hybrid(wl, w, b)
        check_partials(step, 0, b, partials[0])
        check_partials(step, 1, b, partials[1])
        check_merged(step, b, direct)
    q_host = torch.from_numpy(w.q_bits.view(np.int16)).pin_memory()
    o_h = torch.full(step.o.shape, float("nan")).pin_memory()
    l_h = torch.full(step.lse.shape, float("nan")).pin_memory()
    step.decode_host(q_host, o_h, l_h, 0, variant_id(akv, variant))
    torch.cuda.synchronize()
    assert torch.equal(o_h.view(torch.int32), step.o.cpu().view(torch.int32))
    assert torch.equal(l_h.view(torch.int32), step.lse.cpu().view(torch.int32))
