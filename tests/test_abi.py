"""CPU tests of the C ABI: the library loads, exports every symbol include/akv.h declares,
and its host-side logic (slot planner, argument validation, centroid table) behaves.
No call here reaches the GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def akv():
    from kv_cache_tiering_b200 import build
    build.build()
    from kv_cache_tiering_b200 import akv as mod
    return mod


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(akv_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(akv):
    syms = declared_symbols()
    assert len(syms) >= 15
    for name in syms:
        assert hasattr(akv.lib, name), name
        assert ctypes.cast(getattr(akv.lib, name), ctypes.c_void_p).value
    assert set(akv.EXPORTED) <= set(syms)


def test_abi_version_and_status_strings(akv):
    assert akv.abi_version() == 2
    assert akv.status_string(0) == "ok"
    assert akv.status_string(-9) == "page id out of bounds"
    assert akv.status_string(-10) == "kernel launch configuration defect"
    assert akv.error_word_status(akv.AKV_EFLAG_INTERNAL | akv.AKV_EFLAG_TIMEOUT) == akv.AKV_ERR_INTERNAL
    assert akv.error_word_status(0) == 0
    assert akv.error_word_status(akv.AKV_EFLAG_RANGE) == akv.AKV_ERR_RANGE
    assert akv.error_word_status(akv.AKV_EFLAG_RANGE | akv.AKV_EFLAG_BOUNDS) == akv.AKV_ERR_BOUNDS


def test_library_table_equals_oracle_table(akv):
    """The library solves for the Lloyd-Max table with Max's sequential construction; the
    oracle with Lloyd's iteration.  The binary16 tables must agree bit for bit."""
    from oracle import lloyd_max
    assert np.array_equal(akv.centroids_f16(), lloyd_max.centroids_f16_bits())


def test_plan_slots(akv):
    bases, seq_base, seq_n, n = akv.plan_slots([[100, 0, 1024], [30, 5, 0]], 64)
    assert bases[0].tolist() == [0, 3, 4] and bases[1].tolist() == [2, 3, 20]
    assert seq_base.tolist() == [0, 3, 4] and seq_n.tolist() == [3, 1, 16] and n == 20
    with pytest.raises(akv.AkvError) as e:
        akv.plan_slots([[-1]], 64)
    assert e.value.status == akv.AKV_ERR_INVALID


def _tier(akv, **kw):
    base = dict(kind=akv.AKV_TIER_BF16, k=0x1000, v=0x2000, lens=[32], slot_base=[0], stride_seq=0,
                stride_head=4096, stride_token=128)
    base.update(kw)
    return akv.Tier(**base)


@pytest.mark.parametrize("args,status", [
    (dict(d=96), -2),                 # unsupported head dim
    (dict(Hq=12, Hkv=4), -2),         # G = 3
    (dict(Hq=10, Hkv=4), -1),         # Hq not a multiple
    (dict(split_tokens=500), -2),     # not a multiple of 16
    (dict(split_tokens=2048), -2),    # too large
    (dict(n_slots=1), -1),            # slots beyond n_slots (32 tokens / 16 = 2 splits)
    (dict(tier=dict(lens=[-3])), -1),
    (dict(tier=dict(k=0x1001)), -1),  # misaligned
    (dict(tier=dict(stride_token=100)), -1),
    (dict(tier=dict(paged=True, page_table=None, n_pages=4)), -1),
    (dict(tier=dict(paged=True, page_table=0x3000, n_pages=4, page_table_stride=1)), -1),
    (dict(q=0x1002), -1),
    (dict(variant=7), -1),
])
def test_attend_refuses_before_launch(akv, args, status):
    kw = dict(q=0x4000, B=1, Hq=8, Hkv=2, d=128, split_tokens=16, n_slots=4, variant=0)
    tier_kw = args.pop("tier", {})
    kw.update(args)
    t = _tier(akv, **tier_kw)
    with pytest.raises(akv.AkvError) as e:
        akv.akv_decode_attend(kw["q"], kw["B"], kw["Hq"], kw["Hkv"], kw["d"], 0.1, [t], kw["split_tokens"],
                              0x5000, 0x6000, kw["n_slots"], kw["variant"], None, 0)
    assert e.value.status == status
    assert akv.lib.akv_last_error()


def test_empty_work_is_a_no_op(akv):
    t = _tier(akv, lens=[0], k=0, v=0)
    akv.akv_decode_attend(0, 1, 8, 2, 128, 0.1, [t], 16, 0, 0, 0, 0, None, 0)
    akv.akv_merge_lse(0, 0, 0, [0], [0], 0, 8, 128, 0, 0, 0)


def test_merge_and_encode_refusals(akv):
    with pytest.raises(akv.AkvError) as e:
        akv.akv_merge_lse(0x1000, 0x2000, 4, [2], [3], 1, 8, 128, 0x3000, 0x4000, 0)
    assert e.value.status == akv.AKV_ERR_INVALID
    with pytest.raises(akv.AkvError) as e:
        akv.akv_merge_lse(0x1000, 0x2000, 4, [0], [3], 1, 8, 80, 0x3000, 0x4000, 0)
    assert e.value.status == akv.AKV_ERR_UNSUPPORTED
    src = _tier(akv)
    dst = _tier(akv, kind=akv.AKV_TIER_CODES4, stride_head=2, stride_token=1)
    with pytest.raises(akv.AkvError) as e:
        akv.akv_encode_history(dst, dst, 1, 2, 128)
    assert e.value.status == akv.AKV_ERR_INVALID
    with pytest.raises(akv.AkvError) as e:
        akv.akv_encode_history(src, dst, 1, 2, 32)
    assert e.value.status == akv.AKV_ERR_UNSUPPORTED


def test_stager_host_refusals(akv):
    with pytest.raises(akv.AkvError) as e:
        akv.Stager(0x1000, 1 << 20, 0)
    assert e.value.status == akv.AKV_ERR_INVALID
    with pytest.raises(akv.AkvError) as e:
        akv.Stager(0x1001, 1 << 20, 2)
    assert e.value.status == akv.AKV_ERR_INVALID
    st = akv.Stager(0x100000, 1 << 20, 2)  # host bookkeeping only; nothing is touched
    buf = np.zeros(1 << 20, dtype=np.uint8)
    with pytest.raises(akv.AkvError) as e:
        st.stage_chunk(buf, (1 << 19) + 1)
    assert e.value.status == akv.AKV_ERR_BUDGET
    with pytest.raises(akv.AkvError) as e:
        st.use(5)
    assert e.value.status == akv.AKV_ERR_INVALID
    st.destroy()


def test_tier_array_keeps_its_host_arrays(akv):
    """A marshalled tier list stays valid after its Tier objects are marshalled again
    (each marshalling makes fresh host int32 copies)."""
    import ctypes
    t = akv.Tier(akv.AKV_TIER_BF16, 0x1000, 0x2000, lens=[5, 0, 17], slot_base=[0, 1, 1],
                 stride_seq=64, stride_head=0, stride_token=8)
    ta = akv.TierArray([t])
    for _ in range(3):
        t.c()  # replaces the Tier's own kept arrays
    import gc
    gc.collect()
    lens = ctypes.cast(ta.arr[0].lens, ctypes.POINTER(ctypes.c_int32))
    slots = ctypes.cast(ta.arr[0].slot_base, ctypes.POINTER(ctypes.c_int32))
    assert [lens[i] for i in range(3)] == [5, 0, 17] and [slots[i] for i in range(3)] == [0, 1, 1]
    assert ta.n == 1 and akv.TierArray(ta.tiers).n == 1


def test_append_tokens_refusals(akv):
    import ctypes
    t = akv.Tier(akv.AKV_TIER_CODES4, 0x1000, 0x2000, lens=[0])
    with pytest.raises(akv.AkvError) as e:
        akv.akv_append_tokens(t, [0], 1, 8, 128, 0x3000, 0x4000)
    assert e.value.status == akv.AKV_ERR_INVALID
    t = akv.Tier(akv.AKV_TIER_BF16, 0x1000, 0x2000, lens=[0], stride_seq=1024, stride_head=128, stride_token=8)
    with pytest.raises(akv.AkvError) as e:
        akv.akv_append_tokens(t, [3], 1, 8, 96, 0x3000, 0x4000)
    assert e.value.status == akv.AKV_ERR_UNSUPPORTED
    with pytest.raises(akv.AkvError) as e:
        akv.akv_append_tokens(t, [3], 1, 8, 128, 0x3008, 0x4000)  # misaligned rows
    assert e.value.status == akv.AKV_ERR_INVALID
    akv.akv_append_tokens(t, [-1, -5], 2, 8, 128, 0x3000, 0x4000)  # nothing to write: no launch
    assert akv.lib.akv_append_tokens(ctypes.byref(t.c()), None, 1, 8, 128, None, None, None, None) == akv.AKV_ERR_INVALID


def test_decode_workspace_size_is_the_documented_layout(akv):
    """akv_decode's workspace holds the LSE partials, then the O partials, each rounded up to
    256 bytes; the slots are the akv_plan_slots layout of the tiers."""
    up = lambda x: -(-x // 256) * 256
    tiers = [_tier(akv, lens=[100, 0, 1024]), _tier(akv, kind=akv.AKV_TIER_CODES4, lens=[30, 5, 0],
                                                      stride_head=2, stride_token=1)]
    _, _, _, n_slots = akv.plan_slots([[100, 0, 1024], [30, 5, 0]], 64)
    for Hq, Hkv, d in ((8, 2, 128), (32, 8, 64)):
        got = akv.akv_decode_workspace_size(3, Hq, Hkv, d, tiers, 64)
        assert got == up(n_slots * Hq * 4) + up(n_slots * Hq * d * 4)


def test_decode_host_refusals(akv):
    """akv_decode_host checks its workspace, its flags and its host arrays before any launch;
    arrays that are not page-locked (here plain numpy memory) are AKV_ERR_NOT_PINNED."""
    t = _tier(akv, lens=[64])
    B, Hq, Hkv, d = 1, 8, 2, 128
    need = akv.akv_decode_host_workspace_size(B, Hq, Hkv, d, [t], 16)
    up = lambda x: -(-x // 256) * 256
    slots = 64 // 16
    assert need == up(B * Hq * d * 2) + up(B * Hq * d * 4) + up(B * Hq * 4) + up(slots * Hq * 4) + up(slots * Hq * d * 4)
    q = np.zeros((B, Hq, d), np.uint16)
    o = np.zeros((B, Hq, d), np.float32)
    lse = np.zeros((B, Hq), np.float32)
    ws = 0x100000

    def call(**kw):
        a = dict(q=q, d=d, ws=ws, ws_bytes=need, flags=0)
        a.update(kw)
        with pytest.raises(akv.AkvError) as e:
            akv.akv_decode_host(a["q"], B, Hq, Hkv, a["d"], 0.1, [t], 16, a["ws"], a["ws_bytes"], o, lse, a["flags"])
        assert akv.lib.akv_last_error()
        return e.value.status

    assert call(flags=2) == akv.AKV_ERR_INVALID
    assert call(d=96) == akv.AKV_ERR_UNSUPPORTED
    assert call(ws=0x100010) == akv.AKV_ERR_INVALID
    assert call(ws_bytes=need - 256) == akv.AKV_ERR_BUDGET
    assert call() == akv.AKV_ERR_NOT_PINNED
    akv.akv_decode_host(q, 0, Hq, Hkv, d, 0.1, [_tier(akv, lens=[])], 16, ws, need, o, lse)  # B = 0: nothing


def test_header_is_plain_c():
    """include/akv.h is a C header: it compiles as C11 with strict warnings."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = '#include "akv.h"\nint main(void) { akv_tier t; (void)t; return akv_abi_version() > 0 ? 0 : 1; }\n'
    r = subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only", "-x", "c", "-",
                        "-I", os.path.join(root, "include")], input=src, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_staged_decode_refusals(akv):
    """akv_staged_decode validates before it stages or launches anything."""
    st = akv.Stager(0x100000, 1 << 20, 2)  # host bookkeeping only
    host = np.zeros(4096, dtype=np.uint8)
    common = dict(q=0x1000, Hq=32, Hkv=8, d=128, softmax_scale=0.1, split_tokens=512, o_part=0x2000,
                  lse_part=0x3000, n_slots=64, o=0x4000, lse=0x5000)

    def call(**kw):
        args = dict(common, kind=akv.AKV_TIER_BF16, host=host, n_tokens=100, chunk_tokens=4096, new_row=None,
                    window=None)
        args.update(kw)
        with pytest.raises(akv.AkvError) as e:
            akv.akv_staged_decode(st, **args)
        return e.value.status

    assert call(kind=7) == akv.AKV_ERR_INVALID                      # unknown history kind
    assert call(chunk_tokens=1000) == akv.AKV_ERR_INVALID           # not a multiple of the split
    assert call(d=96) == akv.AKV_ERR_UNSUPPORTED
    assert call(Hq=12) == akv.AKV_ERR_INVALID                       # not a multiple of Hkv
    assert call(kind=akv.AKV_TIER_CODES4, new_row=0x6000) == akv.AKV_ERR_INVALID  # compact histories take no row
    assert call(n_slots=0) == akv.AKV_ERR_BUDGET                    # 1 split needed
    assert call(n_tokens=-1) == akv.AKV_ERR_INVALID
    assert call(o=None) == akv.AKV_ERR_INVALID
    bad_window = akv.Tier(akv.AKV_TIER_CODES4, 0x1000, 0x2000, lens=[16])
    assert call(window=bad_window) == akv.AKV_ERR_INVALID          # the window is exact BF16
    st.destroy()


def test_aging_create_refusals(akv):
    """akv_aging_create checks the description on the host; nothing touches the device."""
    B, H, d, W = 2, 8, 128, 64
    R = W // 16 + 2
    win = akv.Tier(akv.AKV_TIER_BF16, 0x10000, 0x20000, lens=[0] * B, paged=True, page_table=0x30000,
                   page_table_stride=R, n_pages=B * R, stride_seq=H * 16 * d, stride_head=16 * d, stride_token=d)
    cmp = akv.Tier(akv.AKV_TIER_CODES4, 0x40000, 0x50000, lens=[0] * B, paged=True, page_table=0x60000,
                   page_table_stride=8, n_pages=16, stride_seq=H, stride_head=1)
    good = dict(B=B, Hq=32, Hkv=H, d=d, split_tokens=512, softmax_scale=0.1, window_tokens=W, ring_pages=R,
                window=win, compact=cmp, compact_len=[32, 0], window_len=[W, W + 5], ring_head=[0, 1],
                page_lists=[[3, 4, 5], [6]], lists_dev=0x70000, o_part=0x80000, lse_part=0x90000, n_slots=64)

    def refused(**kw):
        args = dict(good)
        args.update(kw)
        with pytest.raises(akv.AkvError) as e:
            akv.Aging(**args)
        return e.value.status

    ctx = akv.Aging(**good)
    c, w, r, aged = ctx.state()
    assert list(c) == [32, 0] and list(w) == [W, W + 5] and list(r) == [0, 1] and aged == 0
    ctx.destroy()
    assert refused(window_tokens=40) == akv.AKV_ERR_INVALID          # not a multiple of 16
    assert refused(ring_pages=R - 1) == akv.AKV_ERR_INVALID          # the ring cannot hold W + 16 tokens
    assert refused(window_len=[W - 1, W]) == akv.AKV_ERR_INVALID     # a window below W
    assert refused(compact_len=[40, 0]) == akv.AKV_ERR_INVALID       # not a whole code page
    assert refused(page_lists=[[3], [6]]) == akv.AKV_ERR_INVALID     # fewer pages than the compact tokens use
    assert refused(ring_head=[0, R]) == akv.AKV_ERR_INVALID
    assert refused(d=80) == akv.AKV_ERR_UNSUPPORTED
    assert refused(window=cmp) == akv.AKV_ERR_INVALID


def test_paged_code_pool_keeps_a_pages_key_and_value_blocks_adjacent(akv):
    """The paged compact pool of the ragged and aging workloads: [P][Hkv][2][block], the value
    block of (page, head) right after its key block, strides in blocks (2 Hkv per page, 2 per
    head); a tier over it passes the library's checks."""
    import torch
    from kv_cache_tiering_b200 import workloads
    P, H, d = 5, 8, 128
    bb = akv.codes4_block_bytes(d)
    assert bb == 1056
    pool, k, v, s_seq, s_head = workloads.code_page_pool(P, H, d, "cpu")
    assert tuple(pool.shape) == (P, H, 2, bb) and (s_seq, s_head) == (2 * H, 2)
    assert v.data_ptr() - k.data_ptr() == bb
    # block (page p, head h) of K starts at (p * s_seq + h * s_head) blocks
    for p, h in [(0, 0), (3, 5), (4, 7)]:
        assert k[p, h].data_ptr() - pool.data_ptr() == (p * s_seq + h * s_head) * bb
        assert v[p, h].data_ptr() - k[p, h].data_ptr() == bb
    tier = akv.Tier(akv.AKV_TIER_CODES4, 0x100000, 0x100000 + bb, lens=[60], paged=True, page_table=0x200000,
                    page_table_stride=4, n_pages=P, stride_seq=s_seq, stride_head=s_head)
    assert akv.akv_decode_workspace_size(1, 32, H, d, [tier], 512) > 0
