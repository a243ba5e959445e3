"""ctypes binding of libakv (``include/akv.h``): argument marshalling only.

Every computation runs in the CUDA library; this module converts torch tensors to
device pointers, numpy/int sequences to host int32 arrays and torch streams to
``cudaStream_t`` handles, and raises ``AkvError`` for a negative status.  There is no
fallback: importing this module fails loudly when ``lib/libakv.so`` is missing.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libakv.so")

AKV_OK = 0
AKV_ERR_INVALID = -1
AKV_ERR_UNSUPPORTED = -2
AKV_ERR_CUDA = -3
AKV_ERR_NOT_PINNED = -4
AKV_ERR_BUDGET = -5
AKV_ERR_TIMEOUT = -6
AKV_ERR_NONFINITE = -7
AKV_ERR_RANGE = -8
AKV_ERR_BOUNDS = -9
AKV_ERR_INTERNAL = -10

AKV_EFLAG_NONFINITE = 0x1
AKV_EFLAG_RANGE = 0x2
AKV_EFLAG_BOUNDS = 0x4
AKV_EFLAG_TIMEOUT = 0x8
AKV_EFLAG_INTERNAL = 0x10

AKV_TIER_BF16 = 0
AKV_TIER_CODES4 = 1
AKV_VARIANT_AUTO = 0
AKV_VARIANT_SIMT = 1
AKV_VARIANT_MMA = 2
AKV_HOST_COPY_ENGINE = 0x1
PAGE_TOKENS = 16


def codes4_block_bytes(d: int) -> int:
    return 16 * (d // 2) + 32


class AkvError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"akv status {status}: {message}")
        self.status = status


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libakv.so not built ({_LIB_PATH}); run `python -m kv_cache_tiering_b200.build`")
    return ctypes.CDLL(_LIB_PATH)


lib = _load()

_p = ctypes.c_void_p
_i32p = ctypes.POINTER(ctypes.c_int32)


class AkvTierC(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32),
        ("paged", ctypes.c_int32),
        ("k", _p),
        ("v", _p),
        ("page_table", _p),
        ("page_table_stride", ctypes.c_int64),
        ("n_pages", ctypes.c_int64),
        ("stride_seq", ctypes.c_int64),
        ("stride_head", ctypes.c_int64),
        ("stride_token", ctypes.c_int64),
        ("lens", _p),
        ("slot_base", _p),
        ("rotation_signs", ctypes.c_uint32 * 4),
    ]


class AkvStagedHistoryC(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32),
        ("chunk_tokens", ctypes.c_int32),
        ("host", _p),
        ("n_tokens", ctypes.c_int64),
        ("rotation_signs", ctypes.c_uint32 * 4),
    ]


class AkvAgingDescC(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32),
        ("split_tokens", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("window_tokens", ctypes.c_int32),
        ("ring_pages", ctypes.c_int32),
        ("window", AkvTierC),
        ("compact", AkvTierC),
        ("compact_len", _p),
        ("window_len", _p),
        ("ring_head", _p),
        ("page_lists", ctypes.POINTER(_p)),
        ("page_list_len", _p),
        ("lists_dev", _p),
        ("o_part", _p),
        ("lse_part", _p),
        ("n_slots", ctypes.c_int64),
    ]


def _sig(name, res, *args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("akv_abi_version", ctypes.c_int)
_sig("akv_last_error", ctypes.c_char_p)
_sig("akv_status_string", ctypes.c_char_p, ctypes.c_int)
_sig("akv_error_word_status", ctypes.c_int, ctypes.c_int32)
_sig("akv_centroids_f16", None, ctypes.POINTER(ctypes.c_uint16))
_sig("akv_plan_slots", ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(_p), ctypes.c_int,
     ctypes.POINTER(_p), _p, _p, ctypes.POINTER(ctypes.c_int64))
_sig("akv_encode_history", ctypes.c_int, ctypes.POINTER(AkvTierC), ctypes.POINTER(AkvTierC), ctypes.c_int,
     ctypes.c_int, ctypes.c_int, _p, _p)
_sig("akv_decode_attend", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
     ctypes.POINTER(AkvTierC), ctypes.c_int, ctypes.c_int, _p, _p, ctypes.c_int64, ctypes.c_int, _p, _p)
_sig("akv_merge_lse", ctypes.c_int, _p, _p, ctypes.c_int64, _p, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _p, _p,
     _p)
_sig("akv_decode_workspace_size", ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
     ctypes.POINTER(AkvTierC), ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t))
_sig("akv_decode", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
     ctypes.POINTER(AkvTierC), ctypes.c_int, ctypes.c_int, _p, ctypes.c_size_t, _p, _p, ctypes.c_int, _p, _p)
_sig("akv_decode_host_workspace_size", ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
     ctypes.POINTER(AkvTierC), ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t))
_sig("akv_decode_host", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
     ctypes.POINTER(AkvTierC), ctypes.c_int, ctypes.c_int, _p, ctypes.c_size_t, _p, _p, ctypes.c_int, ctypes.c_int,
     _p, _p)
_sig("akv_append_tokens", ctypes.c_int, ctypes.POINTER(AkvTierC), _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _p,
     _p, _p, _p)
_sig("akv_checkpoint_write", ctypes.c_int, ctypes.c_char_p, ctypes.POINTER(ctypes.c_uint64), ctypes.c_int,
     ctypes.POINTER(_p), ctypes.POINTER(ctypes.c_uint64), ctypes.c_int)
_sig("akv_checkpoint_info", ctypes.c_int, ctypes.c_char_p, ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_int),
     ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_int))
_sig("akv_checkpoint_read", ctypes.c_int, ctypes.c_char_p, ctypes.POINTER(_p), ctypes.POINTER(ctypes.c_uint64),
     ctypes.c_int)
_sig("akv_decode_static", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
     ctypes.POINTER(AkvTierC), ctypes.c_int, ctypes.c_int, _p, _p, ctypes.c_int, _p, _p)
_sig("akv_stager_create", ctypes.c_int, _p, ctypes.c_size_t, ctypes.c_int, ctypes.POINTER(_p))
_sig("akv_stage_chunk", ctypes.c_int, _p, _p, ctypes.c_size_t, _p, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
     ctypes.POINTER(_p))
_sig("akv_stager_use", ctypes.c_int, _p, ctypes.c_int, _p)
_sig("akv_stager_release", ctypes.c_int, _p, ctypes.c_int, _p)
_sig("akv_stage_writeback", ctypes.c_int, _p, ctypes.c_int, ctypes.c_size_t, _p, ctypes.c_size_t, _p)
_sig("akv_stager_destroy", ctypes.c_int, _p)
_sig("akv_staged_decode", ctypes.c_int, _p, ctypes.POINTER(AkvStagedHistoryC), _p, ctypes.c_int, ctypes.c_int,
     ctypes.c_int, ctypes.c_float, ctypes.c_int, _p, ctypes.POINTER(AkvTierC), _p, _p, ctypes.c_int64, _p, _p,
     ctypes.c_int, _p, _p, _p)
_sig("akv_aging_create", ctypes.c_int, ctypes.POINTER(AkvAgingDescC), ctypes.POINTER(_p))
_sig("akv_aging_step", ctypes.c_int, _p, _p, _p, _p, _p, _p, ctypes.c_int, _p, _p)
_sig("akv_aging_state", ctypes.c_int, _p, _p, _p, _p, ctypes.POINTER(ctypes.c_int64))
_sig("akv_aging_destroy", ctypes.c_int, _p)

EXPORTED = [
    "akv_abi_version", "akv_last_error", "akv_status_string", "akv_error_word_status", "akv_centroids_f16",
    "akv_plan_slots", "akv_encode_history", "akv_decode_attend", "akv_merge_lse", "akv_decode_workspace_size",
    "akv_decode", "akv_decode_host_workspace_size", "akv_decode_host", "akv_stager_create",
    "akv_stage_chunk", "akv_stager_use", "akv_stager_release", "akv_stage_writeback", "akv_stager_destroy",
    "akv_staged_decode", "akv_aging_create", "akv_aging_step", "akv_aging_state", "akv_aging_destroy",
]


def _check(status: int) -> int:
    if status < 0:
        raise AkvError(status, lib.akv_last_error().decode(errors="replace"))
    return status


def _ptr(x) -> int | None:
    """Device or host address of a torch tensor / numpy array / int (None -> NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)}")


def _stream(s) -> int | None:
    if s is None:
        try:
            import torch
            return torch.cuda.current_stream().cuda_stream
        except Exception:
            return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _host_i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


@dataclass
class Tier:
    """One tier (see ``akv_tier`` in include/akv.h).  k, v, page_table: device tensors or
    addresses; lens, slot_base: host sequences (kept alive by this object)."""
    kind: int
    k: object
    v: object
    lens: object
    slot_base: object = None
    stride_seq: int = 0
    stride_head: int = 0
    stride_token: int = 0
    paged: bool = False
    page_table: object = None
    page_table_stride: int = 0
    n_pages: int = 0
    rotation_signs: int = 0  # CODES4: bit i negates coordinate i before the rotation
    _keep: list = field(default_factory=list, repr=False)

    def c(self) -> AkvTierC:
        lens = _host_i32(self.lens)
        slots = _host_i32(self.slot_base) if self.slot_base is not None else None
        self._keep = [lens, slots]
        signs = (ctypes.c_uint32 * 4)(*[(int(self.rotation_signs) >> (32 * i)) & 0xFFFFFFFF for i in range(4)])
        return AkvTierC(self.kind, 1 if self.paged else 0, _ptr(self.k), _ptr(self.v), _ptr(self.page_table),
                        self.page_table_stride, self.n_pages, self.stride_seq, self.stride_head,
                        self.stride_token, lens.ctypes.data, None if slots is None else slots.ctypes.data, signs)


class TierArray:
    """A tier list marshalled once for repeated calls.  Holds its own references to the
    tiers' host arrays, so later changes to the Tier objects do not affect it; build a new
    one when the tiers change."""

    def __init__(self, tiers):
        self.tiers = list(tiers)
        cs = [t.c() for t in self.tiers]
        self._keep = [t._keep for t in self.tiers]
        self.arr = (AkvTierC * max(1, len(cs)))(*cs)
        self.n = len(cs)


def _tier_array(tiers) -> TierArray:
    return tiers if isinstance(tiers, TierArray) else TierArray(tiers)


def abi_version() -> int:
    return lib.akv_abi_version()


def status_string(status: int) -> str:
    return lib.akv_status_string(status).decode()


def error_word_status(word: int) -> int:
    return lib.akv_error_word_status(int(word))


def centroids_f16() -> np.ndarray:
    out = (ctypes.c_uint16 * 16)()
    lib.akv_centroids_f16(out)
    return np.frombuffer(out, dtype=np.uint16).copy()


def plan_slots(tier_lens, split_tokens: int):
    """Standard slot layout.  Returns (tier_slot_base list, seq_slot_base, seq_n_slots, n_slots)."""
    lens = [_host_i32(t) for t in tier_lens]
    B = lens[0].size if lens else 0
    bases = [np.zeros(B, dtype=np.int32) for _ in lens]
    seq_base = np.zeros(B, dtype=np.int32)
    seq_n = np.zeros(B, dtype=np.int32)
    n = ctypes.c_int64(0)
    lp = (_p * max(1, len(lens)))(*[a.ctypes.data for a in lens])
    bp = (_p * max(1, len(bases)))(*[a.ctypes.data for a in bases])
    _check(lib.akv_plan_slots(B, len(lens), lp, split_tokens, bp, seq_base.ctypes.data, seq_n.ctypes.data,
                              ctypes.byref(n)))
    return bases, seq_base, seq_n, n.value


def akv_append_tokens(tier, pos, B: int, Hkv: int, d: int, new_k, new_v, err_word=None, stream=None) -> None:
    """Write row b of new_k / new_v ([B][Hkv][d] bf16, device) to token pos[b] of a BF16 tier
    (a Tier, or a one-tier TierArray marshalled once)."""
    if isinstance(tier, TierArray):
        arg = tier.arr
    else:
        t = tier.c()
        arg = ctypes.byref(t)
    p = _host_i32(pos)
    _check(lib.akv_append_tokens(arg, p.ctypes.data, B, Hkv, d, _ptr(new_k), _ptr(new_v), _ptr(err_word),
                                 _stream(stream)))


def akv_encode_history(src: Tier, dst: Tier, B: int, Hkv: int, d: int, err_word=None, stream=None) -> None:
    s, t = src.c(), dst.c()
    _check(lib.akv_encode_history(ctypes.byref(s), ctypes.byref(t), B, Hkv, d, _ptr(err_word), _stream(stream)))


def akv_decode_attend(q, B: int, Hq: int, Hkv: int, d: int, softmax_scale: float, tiers, split_tokens: int,
                      o_part, lse_part, n_slots: int, variant: int = AKV_VARIANT_AUTO, err_word=None,
                      stream=None) -> None:
    ta = _tier_array(tiers)
    _check(lib.akv_decode_attend(_ptr(q), B, Hq, Hkv, d, float(softmax_scale), ta.arr, ta.n, split_tokens,
                                 _ptr(o_part), _ptr(lse_part), int(n_slots), variant, _ptr(err_word),
                                 _stream(stream)))


def akv_merge_lse(o_part, lse_part, n_slots: int, seq_slot_base, seq_n_slots, B: int, Hq: int, d: int, o, lse,
                  stream=None) -> None:
    base = _host_i32(seq_slot_base)
    cnt = _host_i32(seq_n_slots)
    _check(lib.akv_merge_lse(_ptr(o_part), _ptr(lse_part), int(n_slots), base.ctypes.data, cnt.ctypes.data, B, Hq,
                             d, _ptr(o), _ptr(lse), _stream(stream)))


def akv_decode_workspace_size(B: int, Hq: int, Hkv: int, d: int, tiers, split_tokens: int) -> int:
    ta = _tier_array(tiers)
    n = ctypes.c_size_t(0)
    _check(lib.akv_decode_workspace_size(B, Hq, Hkv, d, ta.arr, ta.n, split_tokens, ctypes.byref(n)))
    return n.value


def akv_decode(q, B: int, Hq: int, Hkv: int, d: int, softmax_scale: float, tiers, split_tokens: int, workspace,
               workspace_bytes: int, o, lse, variant: int = AKV_VARIANT_AUTO, err_word=None, stream=None) -> None:
    ta = _tier_array(tiers)
    _check(lib.akv_decode(_ptr(q), B, Hq, Hkv, d, float(softmax_scale), ta.arr, ta.n, split_tokens, _ptr(workspace),
                          int(workspace_bytes), _ptr(o), _ptr(lse), variant, _ptr(err_word), _stream(stream)))


def akv_decode_host_workspace_size(B: int, Hq: int, Hkv: int, d: int, tiers, split_tokens: int) -> int:
    ta = _tier_array(tiers)
    n = ctypes.c_size_t(0)
    _check(lib.akv_decode_host_workspace_size(B, Hq, Hkv, d, ta.arr, ta.n, split_tokens, ctypes.byref(n)))
    return n.value


def akv_decode_host(q_host, B: int, Hq: int, Hkv: int, d: int, softmax_scale: float, tiers, split_tokens: int,
                    workspace, workspace_bytes: int, o_host, lse_host, flags: int = 0,
                    variant: int = AKV_VARIANT_AUTO, err_word=None, stream=None) -> None:
    """One decode step with q_host, o_host and lse_host in page-locked host memory."""
    ta = _tier_array(tiers)
    _check(lib.akv_decode_host(_ptr(q_host), B, Hq, Hkv, d, float(softmax_scale), ta.arr, ta.n, split_tokens,
                               _ptr(workspace), int(workspace_bytes), _ptr(o_host), _ptr(lse_host), flags, variant,
                               _ptr(err_word), _stream(stream)))


def akv_decode_static(q, B: int, Hq: int, Hkv: int, d: int, softmax_scale: float, tiers, split_tokens: int, o, lse,
                      variant: int = AKV_VARIANT_AUTO, err_word=None, stream=None) -> None:
    """akv_decode on the library's own fixed scratch, for callers that cannot allocate
    device memory when they decode; see include/akv.h for its limits."""
    ta = _tier_array(tiers)
    _check(lib.akv_decode_static(_ptr(q), B, Hq, Hkv, d, float(softmax_scale), ta.arr, ta.n, split_tokens, _ptr(o),
                                 _ptr(lse), variant, _ptr(err_word), _stream(stream)))


def checkpoint_write(path: str, meta, spans) -> None:
    """Write a context checkpoint: `meta` uint64 values, `spans` (host address, bytes) pairs."""
    meta = list(meta)
    m = (ctypes.c_uint64 * max(1, len(meta)))(*meta)
    ptrs = (_p * max(1, len(spans)))(*[_ptr(a) for a, _ in spans])
    sizes = (ctypes.c_uint64 * max(1, len(spans)))(*[int(n) for _, n in spans])
    _check(lib.akv_checkpoint_write(os.fsencode(path), m, len(meta), ptrs, sizes, len(spans)))


def checkpoint_info(path: str):
    """(meta values, span sizes) of a checkpoint file."""
    nm, ns = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.akv_checkpoint_info(os.fsencode(path), None, ctypes.byref(nm), None, ctypes.byref(ns)))
    m = (ctypes.c_uint64 * max(1, nm.value))()
    z = (ctypes.c_uint64 * max(1, ns.value))()
    _check(lib.akv_checkpoint_info(os.fsencode(path), m, ctypes.byref(nm), z, ctypes.byref(ns)))
    return [int(m[i]) for i in range(nm.value)], [int(z[i]) for i in range(ns.value)]


def checkpoint_read(path: str, spans) -> None:
    """Read a checkpoint's spans into (host address, bytes) buffers of the recorded sizes."""
    ptrs = (_p * max(1, len(spans)))(*[_ptr(a) for a, _ in spans])
    sizes = (ctypes.c_uint64 * max(1, len(spans)))(*[int(n) for _, n in spans])
    _check(lib.akv_checkpoint_read(os.fsencode(path), ptrs, sizes, len(spans)))


class Stager:
    """Owner of an ``akv_stager`` over a caller-owned device region."""

    def __init__(self, dev_region, region_bytes: int, n_buffers: int):
        h = _p()
        _check(lib.akv_stager_create(_ptr(dev_region), region_bytes, n_buffers, ctypes.byref(h)))
        self._h = h
        self._region = dev_region  # keep the region alive

    def stage_chunk(self, pinned_src, nbytes: int, copy_stream=None, timeout_ms: int = -1):
        idx = ctypes.c_int(-1)
        ptr = _p()
        _check(lib.akv_stage_chunk(self._h, _ptr(pinned_src), nbytes, _stream(copy_stream), timeout_ms,
                                   ctypes.byref(idx), ctypes.byref(ptr)))
        return idx.value, ptr.value

    def use(self, buf: int, consumer_stream=None) -> None:
        _check(lib.akv_stager_use(self._h, buf, _stream(consumer_stream)))

    def release(self, buf: int, consumer_stream=None) -> None:
        _check(lib.akv_stager_release(self._h, buf, _stream(consumer_stream)))

    def writeback(self, buf: int, offset: int, pinned_dst, nbytes: int, stream=None) -> None:
        _check(lib.akv_stage_writeback(self._h, buf, offset, _ptr(pinned_dst), nbytes, _stream(stream)))

    def destroy(self) -> None:
        if self._h:
            h, self._h = self._h, None
            _check(lib.akv_stager_destroy(h))

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def _signs_c(bits: int):
    return (ctypes.c_uint32 * 4)(*[(int(bits) >> (32 * i)) & 0xFFFFFFFF for i in range(4)])


def akv_staged_decode(stager: "Stager", kind: int, host, n_tokens: int, chunk_tokens: int, q, Hq: int, Hkv: int,
                      d: int, softmax_scale: float, split_tokens: int, new_row, window, o_part, lse_part,
                      n_slots: int, o, lse, variant: int = AKV_VARIANT_AUTO, err_word=None, copy_stream=None,
                      compute_stream=None, rotation_signs: int = 0) -> None:
    """One staged decode step of one layer (see akv_staged_decode in include/akv.h)."""
    h = AkvStagedHistoryC(kind, chunk_tokens, _ptr(host), n_tokens, _signs_c(rotation_signs))
    w = None
    if window is not None:
        wa = _tier_array([window])
        w = wa.arr
    _check(lib.akv_staged_decode(stager._h, ctypes.byref(h), _ptr(q), Hq, Hkv, d, float(softmax_scale), split_tokens,
                                 _ptr(new_row), w, _ptr(o_part), _ptr(lse_part), int(n_slots), _ptr(o), _ptr(lse),
                                 variant, _ptr(err_word), _stream(copy_stream), _stream(compute_stream)))


class Aging:
    """Owner of an ``akv_aging`` context (see include/akv.h): a live hybrid batch whose exact
    window ages into the compact tier, one akv_aging_step call per decode step."""

    def __init__(self, B: int, Hq: int, Hkv: int, d: int, split_tokens: int, softmax_scale: float,
                 window_tokens: int, ring_pages: int, window: Tier, compact: Tier, compact_len, window_len,
                 ring_head, page_lists, lists_dev, o_part, lse_part, n_slots: int):
        lists = [_host_i32(x) for x in page_lists]
        lens = [_host_i32(x) for x in (compact_len, window_len, ring_head)]
        list_len = _host_i32([len(x) for x in lists])
        ptrs = (_p * max(1, B))(*[x.ctypes.data for x in lists])
        wc, cc = window.c(), compact.c()
        self._keep = [lists, lens, list_len, ptrs, window._keep, compact._keep]
        desc = AkvAgingDescC(B, Hq, Hkv, d, split_tokens, float(softmax_scale), window_tokens, ring_pages, wc, cc,
                             lens[0].ctypes.data, lens[1].ctypes.data, lens[2].ctypes.data, ptrs,
                             list_len.ctypes.data, _ptr(lists_dev), _ptr(o_part), _ptr(lse_part), int(n_slots))
        h = _p()
        _check(lib.akv_aging_create(ctypes.byref(desc), ctypes.byref(h)))
        self._h = h
        self.B = B

    def step(self, q, k_new, v_new, o, lse, variant: int = AKV_VARIANT_AUTO, err_word=None, stream=None) -> None:
        _check(lib.akv_aging_step(self._h, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(o), _ptr(lse), variant,
                                  _ptr(err_word), _stream(stream)))

    def state(self):
        """(compact lengths, window lengths, ring heads, pages aged so far)."""
        c, w, r = (np.zeros(self.B, np.int32) for _ in range(3))
        aged = ctypes.c_int64(0)
        _check(lib.akv_aging_state(self._h, c.ctypes.data, w.ctypes.data, r.ctypes.data, ctypes.byref(aged)))
        return c, w, r, aged.value

    def destroy(self) -> None:
        if self._h:
            h, self._h = self._h, None
            _check(lib.akv_aging_destroy(h))

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass
