"""Oracle work of the full-size GPU parity tests, run in spawned worker processes.

Test infrastructure: every function here calls only ``oracle/`` on seeded input bits that
the caller drew from ``kv_cache_tiering_b200.synth``; nothing comes from the CUDA path.
The pool uses the ``spawn`` start method, so it is safe to start after the test process
has initialised CUDA (a forked child of a CUDA process can hang).
"""
from __future__ import annotations

import multiprocessing
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np

from oracle import akv_oracle as ora


def _init_worker():
    # one BLAS thread per worker: the pool itself provides the parallelism
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def pool(max_workers: int | None = None) -> ProcessPoolExecutor:
    n = max_workers or max(1, min(16, os.cpu_count() or 1))
    return ProcessPoolExecutor(max_workers=n, mp_context=multiprocessing.get_context("spawn"),
                               initializer=_init_worker)


def hybrid_head(q_bits, k_bits, v_bits, n_compact: int, scale: float, split_tokens: int, sign_bits: int = 0):
    """One KV head of one sequence: tokens [0, n_compact) compact, the rest exact BF16.

    q_bits: bf16 bits [G, d] (the head's query group); k_bits, v_bits: bf16 bits [T, d].
    Returns (key blocks, value blocks) of the compact part as the oracle packs them, and
    decode_sequence's (partials, merged, direct) with the G query heads over one KV head."""
    c = int(n_compact)
    d = k_bits.shape[1]
    tiers = []
    blocks = (None, None)
    if c > 0:
        ek, ev = ora.encode(k_bits[:c], sign_bits), ora.encode(v_bits[:c], sign_bits)
        blocks = (ora.pack_blocks(ek.codes, ek.scale_bits), ora.pack_value_blocks(ev.codes, ev.scale_bits))
        tiers.append((ora.dequantize(ek.codes, ek.scale_bits, sign_bits)[None],
                      ora.dequantize(ev.codes, ev.scale_bits, sign_bits)[None]))
    else:
        tiers.append((np.zeros((1, 0, d)), np.zeros((1, 0, d))))
    tiers.append((ora.bf16_bits_to_f64(k_bits[c:])[None], ora.bf16_bits_to_f64(v_bits[c:])[None]))
    result = ora.decode_sequence(ora.bf16_bits_to_f64(q_bits), tiers, scale, split_tokens)
    return blocks, result


def exact_head(q_bits, k_bits, v_bits, scale: float, split_tokens: int):
    """One KV head, every token exact BF16: decode_sequence's (partials, merged, direct)."""
    tiers = [(ora.bf16_bits_to_f64(k_bits)[None], ora.bf16_bits_to_f64(v_bits)[None])]
    return ora.decode_sequence(ora.bf16_bits_to_f64(q_bits), tiers, scale, split_tokens)
