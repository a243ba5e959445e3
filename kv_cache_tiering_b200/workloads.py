"""Device-resident decode workloads driven through the C ABI.

Each class uploads one seeded synthetic workload (``synth``) into device memory in the
layout the library reads, plans the split slots, and runs one decode step -- every
tier's split attention followed by the merge -- on a given stream.  Torch provides the
device memory and streams only.
"""
from __future__ import annotations

import numpy as np
import torch

from . import akv, synth


def to_dev_bits(bits: np.ndarray, device) -> torch.Tensor:
    """uint16 bit patterns -> device int16 tensor holding the same bits."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device)


def tier_lens_slots(tiers):
    return [t.lens for t in tiers]


class DecodeStep:
    """Partials, outputs and the slot plan shared by every workload."""

    def __init__(self, B: int, Hq: int, Hkv: int, d: int, split_tokens: int, scale: float, tiers, device):
        self.B, self.Hq, self.Hkv, self.d = B, Hq, Hkv, d
        self.split_tokens, self.scale = split_tokens, scale
        self.tiers = tiers
        bases, self.seq_slot_base, self.seq_n_slots, self.n_slots = akv.plan_slots([t.lens for t in tiers], split_tokens)
        for t, b in zip(tiers, bases):
            t.slot_base = b
        self.o_part = torch.empty((max(1, self.n_slots), Hq, d), dtype=torch.float32, device=device)
        self.lse_part = torch.empty((max(1, self.n_slots), Hq), dtype=torch.float32, device=device)
        self.o = torch.empty((B, Hq, d), dtype=torch.float32, device=device)
        self.lse = torch.empty((B, Hq), dtype=torch.float32, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        # the tier list marshalled once for every call of the step
        self.tiers_c = akv.TierArray(tiers)
        self.tier_c = [akv.TierArray([t]) for t in tiers]
        self.ws_bytes = akv.akv_decode_workspace_size(B, Hq, Hkv, d, self.tiers_c, split_tokens)
        self.workspace = torch.zeros(max(256, self.ws_bytes), dtype=torch.uint8, device=device)

    def decode_host(self, q_host, o_host, lse_host, flags=0, variant=akv.AKV_VARIANT_AUTO, stream=None):
        """The whole step with the query and the results in page-locked host memory."""
        if getattr(self, "host_ws", None) is None:
            self.host_ws_bytes = akv.akv_decode_host_workspace_size(self.B, self.Hq, self.Hkv, self.d, self.tiers_c,
                                                                    self.split_tokens)
            self.host_ws = torch.empty(max(256, self.host_ws_bytes), dtype=torch.uint8, device=self.o.device)
        akv.akv_decode_host(q_host, self.B, self.Hq, self.Hkv, self.d, self.scale, self.tiers_c, self.split_tokens,
                            self.host_ws, self.host_ws_bytes, o_host, lse_host, flags, variant, self.err, stream)

    def decode(self, q, variant=akv.AKV_VARIANT_AUTO, stream=None):
        """The whole step in one call (split attention with the merge fused in)."""
        akv.akv_decode(q, self.B, self.Hq, self.Hkv, self.d, self.scale, self.tiers_c, self.split_tokens, self.workspace,
                       self.ws_bytes, self.o, self.lse, variant, self.err, stream)

    def attend(self, q, variant=akv.AKV_VARIANT_AUTO, stream=None):
        akv.akv_decode_attend(q, self.B, self.Hq, self.Hkv, self.d, self.scale, self.tiers_c, self.split_tokens,
                              self.o_part, self.lse_part, self.n_slots, variant, self.err, stream)

    def attend_tier(self, i: int, q, variant=akv.AKV_VARIANT_AUTO, stream=None):
        """Tier i alone: the same launch ``attend`` makes for it, into the same slots."""
        akv.akv_decode_attend(q, self.B, self.Hq, self.Hkv, self.d, self.scale, self.tier_c[i], self.split_tokens,
                              self.o_part, self.lse_part, self.n_slots, variant, self.err, stream)

    def merge(self, stream=None):
        akv.akv_merge_lse(self.o_part, self.lse_part, self.n_slots, self.seq_slot_base, self.seq_n_slots, self.B,
                          self.Hq, self.d, self.o, self.lse, stream)

    def step(self, q, variant=akv.AKV_VARIANT_AUTO, stream=None):
        self.attend(q, variant, stream)
        self.merge(stream)

    def tier_slots(self, i: int, b: int):
        """Slot range of tier i, sequence b."""
        t = self.tiers[i]
        n = -(-int(t.lens[b]) // self.split_tokens)
        return int(t.slot_base[b]), n


class ExactResident:
    """Exact BF16 tier, contiguous head-major [B, Hkv, T, d] (the tiny and exact GQA workloads)."""

    def __init__(self, wl: synth.Workload, device, B: int | None = None, T: int | None = None):
        self.wl = wl
        B = wl.B if B is None else B
        T = wl.extra["T"] if T is None else T
        self.B, self.T = B, T
        self.q_bits = synth.queries(wl, B=B)
        ks, vs = [], []
        for b in range(B):
            k, v = synth.history_head_major(wl, b, T)
            ks.append(k)
            vs.append(v)
        self.k_bits = np.stack(ks)
        self.v_bits = np.stack(vs)
        self.q = to_dev_bits(self.q_bits, device)
        self.k = to_dev_bits(self.k_bits, device)
        self.v = to_dev_bits(self.v_bits, device)
        d, H = wl.d, wl.Hkv
        tier = akv.Tier(akv.AKV_TIER_BF16, self.k, self.v, lens=np.full(B, T, np.int32),
                        stride_seq=H * T * d, stride_head=T * d, stride_token=d)
        self.step = DecodeStep(B, wl.Hq, H, d, wl.split_tokens, wl.scale, [tier], device)

    def kv_bytes(self) -> int:
        return 2 * self.B * self.wl.Hkv * self.T * self.wl.d * 2

    def tier_bytes(self) -> list[int]:
        return [self.kv_bytes()]


class HybridResident:
    """Hybrid tiers of one batch: tokens [0, T - W) compact (contiguous code blocks
    [B, Hkv, (T - W)/16]), tokens [T - W, T) exact BF16 (a view of the head-major history)."""

    def __init__(self, wl: synth.Workload, device, B: int | None = None, T: int | None = None, W: int | None = None,
                 rotation_signs: int = 0):
        self.wl = wl
        B = wl.B if B is None else B
        T = wl.extra["T"] if T is None else T
        W = wl.extra["window"] if W is None else W
        self.rotation_signs = rotation_signs
        self.B, self.T, self.W = B, T, W
        d, H = wl.d, wl.Hkv
        self.q_bits = synth.queries(wl, B=B)
        ks, vs = [], []
        for b in range(B):
            k, v = synth.history_head_major(wl, b, T)
            ks.append(k)
            vs.append(v)
        self.k_bits = np.stack(ks)
        self.v_bits = np.stack(vs)
        self.q = to_dev_bits(self.q_bits, device)
        self.k = to_dev_bits(self.k_bits, device)
        self.v = to_dev_bits(self.v_bits, device)
        Tc = T - W
        nb = -(-Tc // 16)
        bb = akv.codes4_block_bytes(d)
        self.kc = torch.empty((B, H, nb, bb), dtype=torch.uint8, device=device)
        self.vc = torch.empty((B, H, nb, bb), dtype=torch.uint8, device=device)
        src = akv.Tier(akv.AKV_TIER_BF16, self.k, self.v, lens=np.full(B, Tc, np.int32),
                       stride_seq=H * T * d, stride_head=T * d, stride_token=d)
        self.codes_tier = akv.Tier(akv.AKV_TIER_CODES4, self.kc, self.vc, lens=np.full(B, Tc, np.int32),
                                   stride_seq=H * nb, stride_head=nb, stride_token=1, rotation_signs=rotation_signs)
        self.enc_err = torch.zeros(1, dtype=torch.int32, device=device)
        akv.akv_encode_history(src, self.codes_tier, B, H, d, self.enc_err)
        off = Tc * d * 2  # bytes: the window starts at token Tc of every (b, h) stream
        exact = akv.Tier(akv.AKV_TIER_BF16, self.k.data_ptr() + off, self.v.data_ptr() + off,
                         lens=np.full(B, W, np.int32), stride_seq=H * T * d, stride_head=T * d, stride_token=d)
        self.step = DecodeStep(B, wl.Hq, H, d, wl.split_tokens, wl.scale, [self.codes_tier, exact], device)

    def kv_bytes(self) -> int:
        return sum(self.tier_bytes())

    def tier_bytes(self) -> list[int]:
        """Bytes each tier's launch must read: K and V codes + fp16 norms, then BF16 K and V."""
        d, H = self.wl.d, self.wl.Hkv
        Tc = self.T - self.W
        return [self.B * H * 2 * Tc * (d // 2 + 2), self.B * H * 2 * self.W * d * 2]


def code_page_pool(n_pages: int, H: int, d: int, device, zero: bool = False):
    """Paged compact pool ``[P][Hkv][2][block]``: the key block and the value block of one
    (page, KV head) sit side by side, so a 16-token step reads one 2 x 1056-byte span.  DRAM
    serves whole 128-byte lines; a 1056-byte block read alone at a random page always spans 9
    lines (96 B more than it holds), a 2112-byte span 17 (64 B more).
    Returns (pool, key view, value view, stride_seq, stride_head), the strides in blocks."""
    bb = akv.codes4_block_bytes(d)
    alloc = torch.zeros if zero else torch.empty
    pool = alloc((n_pages, H, 2, bb), dtype=torch.uint8, device=device)
    return pool, pool[:, :, 0], pool[:, :, 1], 2 * H, 2


class RaggedPaged:
    """Ragged paged hybrid batch: per-sequence lengths, 16-token pages drawn from two pools
    through seeded random page permutations; the newest W tokens exact (BF16 pool
    [P, Hkv, 16, d]), the rest compact (code-block pool [P, Hkv])."""

    def __init__(self, wl: synth.Workload, device, B: int | None = None, lens=None, W: int | None = None,
                 key_dist: str = "student_t", generator: str = "numpy"):
        self.wl = wl
        B = wl.B if B is None else B
        W = wl.extra["window"] if W is None else W
        lens = synth.ragged_lengths(wl, B) if lens is None else np.asarray(lens, np.int32)
        self.B, self.W, self.lens = B, W, lens
        d, H = wl.d, wl.Hkv
        self.q_bits = synth.queries(wl, B=B)
        self.q = to_dev_bits(self.q_bits, device)
        ex_len = np.minimum(lens, W).astype(np.int32)
        cp_len = (lens - ex_len).astype(np.int32)
        ex_pages = -(-ex_len // 16)
        cp_pages = -(-cp_len // 16)
        self.ex_table_np = synth.page_tables(ex_pages, synth.page_permutation(wl, "exact", int(ex_pages.sum())))
        self.cp_table_np = synth.page_tables(cp_pages, synth.page_permutation(wl, "codes", max(1, int(cp_pages.sum()))))
        n_ex, n_cp = int(ex_pages.sum()), max(1, int(cp_pages.sum()))
        self.ex_k = torch.zeros((n_ex, H, 16, d), dtype=torch.int16, device=device)
        self.ex_v = torch.zeros((n_ex, H, 16, d), dtype=torch.int16, device=device)
        self.cp_pool, self.cp_k, self.cp_v, cs, ch = code_page_pool(n_cp, H, d, device)
        self.cp_strides = dict(stride_seq=cs, stride_head=ch)
        self.ex_table = torch.from_numpy(self.ex_table_np).to(device)
        self.cp_table = torch.from_numpy(self.cp_table_np).to(device)
        self.enc_err = torch.zeros(1, dtype=torch.int32, device=device)
        self.codes_tier = akv.Tier(akv.AKV_TIER_CODES4, self.cp_k, self.cp_v, lens=cp_len, paged=True,
                                   page_table=self.cp_table, page_table_stride=self.cp_table_np.shape[1],
                                   n_pages=n_cp, **self.cp_strides)
        self.exact_tier = akv.Tier(akv.AKV_TIER_BF16, self.ex_k, self.ex_v, lens=ex_len, paged=True,
                                   page_table=self.ex_table, page_table_stride=self.ex_table_np.shape[1],
                                   n_pages=n_ex, stride_seq=H * 16 * d, stride_head=16 * d, stride_token=d)
        self.key_dist = key_dist
        self.ex_len, self.cp_len = ex_len, cp_len
        self.step = None
        if generator == "torch":
            self._fill_on_device(wl, device, lens, ex_len, cp_len, n_cp)
            self.step = DecodeStep(B, wl.Hq, H, d, wl.split_tokens, wl.scale, [self.codes_tier, self.exact_tier],
                                   device)
            return
        ex_pool_k = np.zeros((n_ex, H, 16, d), np.uint16)
        ex_pool_v = np.zeros((n_ex, H, 16, d), np.uint16)
        for b in range(B):
            k, v = synth.history_head_major(wl, b, int(lens[b]), key_dist=key_dist)
            c = int(cp_len[b])
            synth.scatter_pages(k[:, c:], self.ex_table_np[b], ex_pool_k)
            synth.scatter_pages(v[:, c:], self.ex_table_np[b], ex_pool_v)
            if c > 0:
                # encode the compact part of this sequence into its pages of the code pool
                ks = to_dev_bits(np.ascontiguousarray(k[:, :c]), device)
                vs = to_dev_bits(np.ascontiguousarray(v[:, :c]), device)
                src = akv.Tier(akv.AKV_TIER_BF16, ks, vs, lens=[c], stride_seq=0, stride_head=c * d, stride_token=d)
                row = self.cp_table[b:b + 1]
                dst = akv.Tier(akv.AKV_TIER_CODES4, self.cp_k, self.cp_v, lens=[c], paged=True, page_table=row,
                               page_table_stride=self.cp_table_np.shape[1], n_pages=n_cp, **self.cp_strides)
                akv.akv_encode_history(src, dst, 1, H, d, self.enc_err)
                torch.cuda.current_stream().synchronize()
                del ks, vs
        self.ex_k.copy_(torch.from_numpy(ex_pool_k.view(np.int16)))
        self.ex_v.copy_(torch.from_numpy(ex_pool_v.view(np.int16)))
        self.ex_len, self.cp_len = ex_len, cp_len
        self.step = DecodeStep(B, wl.Hq, H, d, wl.split_tokens, wl.scale, [self.codes_tier, self.exact_tier], device)

    def _fill_on_device(self, wl, device, lens, ex_len, cp_len, n_cp):
        """Full-size fill: draw each sequence on the device (seeded torch generators), encode
        its compact part through the library and scatter its exact part into the page pool."""
        d, H = wl.d, wl.Hkv
        for b in range(self.B):
            L, c = int(lens[b]), int(cp_len[b])
            k, v = synth.torch_sequence_kv(wl, b, L, self.key_dist, device=device)
            if c > 0:
                src = akv.Tier(akv.AKV_TIER_BF16, k, v, lens=[c], stride_seq=0, stride_head=L * d, stride_token=d)
                dst = akv.Tier(akv.AKV_TIER_CODES4, self.cp_k, self.cp_v, lens=[c], paged=True,
                               page_table=self.cp_table[b:b + 1], page_table_stride=self.cp_table_np.shape[1],
                               n_pages=n_cp, **self.cp_strides)
                akv.akv_encode_history(src, dst, 1, H, d, self.enc_err)
            e = int(ex_len[b])
            pages = -(-e // 16)
            ex_k = torch.zeros((H, pages * 16, d), dtype=torch.int16, device=device)
            ex_v = torch.zeros((H, pages * 16, d), dtype=torch.int16, device=device)
            ex_k[:, :e] = k[:, c:]
            ex_v[:, :e] = v[:, c:]
            rows = self.ex_table[b, :pages].long()
            self.ex_k[rows] = ex_k.view(H, pages, 16, d).permute(1, 0, 2, 3)
            self.ex_v[rows] = ex_v.view(H, pages, 16, d).permute(1, 0, 2, 3)
        torch.cuda.synchronize(device)

    def kv_bytes(self) -> int:
        return sum(self.tier_bytes())

    def tier_bytes(self) -> list[int]:
        """Bytes each tier's launch must read: compact pages' codes + norms, then BF16 pages."""
        d, H = self.wl.d, self.wl.Hkv
        return [int(H * 2 * self.cp_len.sum() * (d // 2 + 2)), int(H * 2 * self.ex_len.sum() * d * 2)]


class StagedDecode:
    """Host-authoritative history staged through a bounded device ring.

    Each layer's history lives in pinned host memory as rows [token][K|V][Hkv][d], so any
    run of tokens is one contiguous span.  A decode step, per layer: every 4096-token chunk
    is copied into the next ring buffer (akv_stage_chunk on the copy stream), the new
    token's K/V is appended into the chunk that holds its position, the chunk's splits are
    attended on the compute stream, the new row is written back to the host copy, and the
    buffer is released; the layer's split partials are then merged.  ``resident=True``
    keeps the same chunks in device memory instead and issues the same attend calls, which
    is the comparison run for bit-identity."""

    def __init__(self, wl: synth.Workload, device, layers: int | None = None, T: int | None = None,
                 chunk: int | None = None, max_steps: int = 8, n_buffers: int = 2, resident: bool = False,
                 host_layers=None, source: str = "host"):
        self.wl, self.device, self.resident = wl, device, resident
        self.L = wl.extra["layers"] if layers is None else layers
        self.T = wl.extra["T"] if T is None else T
        self.chunk = wl.extra["chunk"] if chunk is None else chunk
        H, d = wl.Hkv, wl.d
        self.row_elems = 2 * H * d
        self.row_bytes = 2 * self.row_elems
        cap = self.T + max_steps
        self.cap = -(-cap // self.chunk) * self.chunk
        if host_layers is None:
            # source "host": numpy streams (the oracle can redraw any layer); "torch": seeded
            # device generators, for full-size runs that need no oracle
            host_layers = []
            for layer in range(self.L):
                h = torch.empty((self.cap, 2, H, d), dtype=torch.int16).pin_memory()
                if source == "torch":
                    g = synth.torch_generator(wl.seed, wl.name, "staged", layer, device=device)
                    rows = torch.empty((self.T, 2, H, d), dtype=torch.int16, device=device)
                    rows[:, 0] = synth.torch_normal_bf16(g, (self.T, H, d), device)
                    rows[:, 1] = synth.torch_normal_bf16(g, (self.T, H, d), device)
                    h[: self.T].copy_(rows)
                    del rows
                else:
                    k, v = synth.history_token_major(wl, layer, self.T)
                    h[: self.T, 0] = torch.from_numpy(k.view(np.int16))
                    h[: self.T, 1] = torch.from_numpy(v.view(np.int16))
                h[self.T:].zero_()  # rows the appended tokens will take (a reused pinned block holds old data)
                host_layers.append(h)
        self.host = host_layers
        self.copy_stream = torch.cuda.Stream(device)
        self.compute_stream = torch.cuda.Stream(device)
        if resident:
            self.dev_layers = [h.to(device) for h in self.host]
        else:
            self.region = torch.empty(n_buffers * self.chunk * self.row_bytes, dtype=torch.uint8, device=device)
            self.stager = akv.Stager(self.region, self.region.numel(), n_buffers)
        n_slots = -(-self.cap // wl.split_tokens)
        self.o_part = torch.empty((n_slots, wl.Hq, d), dtype=torch.float32, device=device)
        self.lse_part = torch.empty((n_slots, wl.Hq), dtype=torch.float32, device=device)
        self.o = torch.empty((self.L, wl.Hq, d), dtype=torch.float32, device=device)
        self.lse = torch.empty((self.L, wl.Hq), dtype=torch.float32, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.steps_done = 0
        self.h2d_bytes = 0

    def inputs(self, step: int):
        """Device q [L][Hq][d] and new rows [L][2][Hkv][d] of decode step ``step``."""
        q = np.stack([synth.queries(self.wl, layer=l, step=step, B=1)[0] for l in range(self.L)])
        new = np.stack([np.stack(synth.new_token(self.wl, l, step)) for l in range(self.L)])
        return to_dev_bits(q, self.device), to_dev_bits(new, self.device)

    def step(self, q, new_rows, variant=akv.AKV_VARIANT_AUTO, timeout_ms: int = -1):
        """One decode step over all layers; q [L][Hq][d], new_rows [L][2][Hkv][d] (device).
        Staged: one akv_staged_decode call per layer.  Resident: the same attention calls over
        the same chunks in device memory (the bit-identity comparison run)."""
        if not self.resident:
            self._step_staged(q, new_rows, variant)
            return
        wl, H, d = self.wl, self.wl.Hkv, self.wl.d
        pos = self.T + self.steps_done          # position of the appended token
        n_tok = pos + 1
        cs = self.compute_stream
        n_chunks = -(-n_tok // self.chunk)
        n_split = -(-n_tok // wl.split_tokens)
        per_chunk = self.chunk // wl.split_tokens
        rb = self.row_bytes
        cs.wait_stream(torch.cuda.current_stream(self.device))  # the step's inputs
        for layer in range(self.L):
            new_row = new_rows[layer].reshape(-1).view(torch.uint8)
            store = self.dev_layers[layer].view(torch.uint8).reshape(-1)
            for c in range(n_chunks):
                tok0 = c * self.chunk
                ntc = min(self.chunk, n_tok - tok0)
                appends = tok0 <= pos < tok0 + self.chunk
                off = tok0 * rb
                base = store.data_ptr() + off
                with torch.cuda.stream(cs):
                    if appends:  # the new token's row goes into the chunk that holds its position
                        store[off + (pos - tok0) * rb: off + (pos - tok0 + 1) * rb].copy_(new_row)
                    tier = akv.Tier(akv.AKV_TIER_BF16, base, base + H * d * 2, lens=[ntc],
                                    slot_base=[c * per_chunk], stride_seq=0, stride_head=d, stride_token=2 * H * d)
                    akv.akv_decode_attend(q[layer], 1, wl.Hq, H, d, wl.scale, [tier], wl.split_tokens, self.o_part,
                                          self.lse_part, self.o_part.shape[0], variant, self.err, cs)
                    if appends:  # write the new row back to the host copy
                        self.host[layer][pos].view(torch.uint8).reshape(-1).copy_(
                            store[off + (pos - tok0) * rb: off + (pos - tok0 + 1) * rb], non_blocking=True)
            akv.akv_merge_lse(self.o_part, self.lse_part, self.o_part.shape[0], [0], [n_split], 1, wl.Hq, d,
                              self.o[layer:layer + 1], self.lse[layer:layer + 1], cs)
        torch.cuda.current_stream(self.device).wait_stream(cs)  # the results, for the caller's stream
        self.steps_done += 1

    def _step_staged(self, q, new_rows, variant):
        wl, H, d = self.wl, self.wl.Hkv, self.wl.d
        pos = self.T + self.steps_done
        cs = self.compute_stream
        cs.wait_stream(torch.cuda.current_stream(self.device))  # the step's inputs
        for layer in range(self.L):
            akv.akv_staged_decode(self.stager, akv.AKV_TIER_BF16, self.host[layer], pos, self.chunk, q[layer], wl.Hq,
                                  H, d, wl.scale, wl.split_tokens, new_rows[layer], None, self.o_part, self.lse_part,
                                  self.o_part.shape[0], self.o[layer:layer + 1], self.lse[layer:layer + 1], variant,
                                  self.err, self.copy_stream, cs)
            self.h2d_bytes += pos * self.row_bytes
        torch.cuda.current_stream(self.device).wait_stream(cs)  # the results, for the caller's stream
        self.steps_done += 1

    def suspend(self, path: str) -> None:
        """Checkpoint the context: every layer's pinned history (the authoritative copy) and
        the step count.  Device state is a working set rebuilt on resume."""
        torch.cuda.synchronize(self.device)  # write-backs of the last step have landed
        wl = self.wl
        meta = [1, self.L, self.T, self.cap, self.chunk, self.steps_done, wl.Hkv, wl.d, wl.seed]
        akv.checkpoint_write(path, meta, [(h.data_ptr(), h.numel() * h.element_size()) for h in self.host])

    @classmethod
    def resume(cls, path: str, wl: synth.Workload, device, n_buffers: int = 2, resident: bool = False):
        """Rebuild a suspended context from its checkpoint, ready for its next step."""
        meta, sizes = akv.checkpoint_info(path)
        kind, L, T, cap, chunk, steps, hkv, d, _seed = meta
        if kind != 1 or hkv != wl.Hkv or d != wl.d:
            raise ValueError("checkpoint does not hold a staged BF16 context of this shape")
        host = [torch.empty((cap, 2, hkv, d), dtype=torch.int16).pin_memory() for _ in range(L)]
        akv.checkpoint_read(path, [(h.data_ptr(), n) for h, n in zip(host, sizes)])
        st = cls(wl, device, layers=L, T=T, chunk=chunk, max_steps=cap - T, n_buffers=n_buffers, resident=resident,
                 host_layers=host)
        st.steps_done = steps
        return st

    def close(self):
        if not self.resident:
            self.stager.destroy()


class StagedHybridDecode:
    """The hybrid tier with its compact part staged from the host.

    Per layer, tokens [0, Tc) live as compact blocks in pinned host memory, Tc = T - W, and
    tokens [Tc, T + steps) stay BF16 on the device (the exact window, which the appended
    tokens join).  Host layout of a layer: block rows [Tc/16][K | V][Hkv][block bytes] -- a
    row holds the 16-token key blocks of every head, then the value blocks -- so a run of
    consecutive tokens is one contiguous span, about a quarter of its BF16 size.

    A decode step, per layer: the new token's row is appended to the window; every chunk of
    the compact part is staged through the ring (akv_stage_chunk on the copy stream) and
    attended as a CODES4 tier into its own split slots; the window is attended from device
    memory; the partials are merged.  ``resident=True`` keeps the same compact rows in device
    memory and issues the same attend calls (the bit-identity comparison).  The compact
    codes are written by the library's encoder from a seeded BF16 history."""

    def __init__(self, wl: synth.Workload, device, layers: int, T: int, W: int, chunk: int, max_steps: int = 8,
                 n_buffers: int = 2, resident: bool = False, source: str = "torch"):
        assert chunk % wl.split_tokens == 0 and chunk % 16 == 0 and 0 < W <= T
        self.wl, self.device, self.resident = wl, device, resident
        self.L, self.T, self.W, self.chunk = layers, T, W, chunk
        H, d = wl.Hkv, wl.d
        self.Tc = T - W
        self.bb = akv.codes4_block_bytes(d)
        self.crow = 2 * H * self.bb                  # bytes of one 16-token block row
        self.nrows = -(-self.Tc // 16)
        self.wrow = 2 * H * d * 2                    # bytes of one BF16 window row
        self.wcap = W + max_steps
        self.host, self.win = [], []
        self.k_bits, self.v_bits = [], []            # host copies of the BF16 history (source="host")
        for layer in range(layers):
            if source == "host":
                kk, vv = synth.history_token_major(wl, layer, T)     # [T, Hkv, d]
                self.k_bits.append(kk)
                self.v_bits.append(vv)
                k_dev = to_dev_bits(np.ascontiguousarray(kk.transpose(1, 0, 2)), device)
                v_dev = to_dev_bits(np.ascontiguousarray(vv.transpose(1, 0, 2)), device)
            else:
                g = synth.torch_generator(wl.seed, wl.name, "staged-hybrid", layer, device=device)
                k_dev = synth.torch_normal_bf16(g, (H, T, d), device)
                v_dev = synth.torch_normal_bf16(g, (H, T, d), device)
            codes = torch.empty(max(1, self.nrows) * self.crow, dtype=torch.uint8, device=device)
            if self.Tc > 0:
                src = akv.Tier(akv.AKV_TIER_BF16, k_dev, v_dev, lens=[self.Tc], stride_seq=0, stride_head=T * d,
                               stride_token=d)
                dst = akv.Tier(akv.AKV_TIER_CODES4, codes, codes.data_ptr() + H * self.bb, lens=[self.Tc],
                               stride_seq=0, stride_head=1, stride_token=2 * H)
                enc_err = torch.zeros(1, dtype=torch.int32, device=device)
                akv.akv_encode_history(src, dst, 1, H, d, enc_err)
            win = torch.zeros((self.wcap, 2, H, d), dtype=torch.int16, device=device)
            win[:W, 0] = k_dev[:, self.Tc:T].transpose(0, 1)
            win[:W, 1] = v_dev[:, self.Tc:T].transpose(0, 1)
            self.win.append(win)
            self.host.append(codes if resident else codes.cpu().pin_memory())
            del k_dev, v_dev
        torch.cuda.synchronize(device)
        self.copy_stream = torch.cuda.Stream(device)
        self.compute_stream = torch.cuda.Stream(device)
        if not resident:
            rows = -(-min(chunk, max(16, self.Tc)) // 16)          # block rows of the largest chunk
            per_buf = -(-(rows * self.crow) // 256) * 256
            self.region = torch.empty(n_buffers * per_buf, dtype=torch.uint8, device=device)
            self.stager = akv.Stager(self.region, self.region.numel(), n_buffers)
        self.n_cslots = -(-self.Tc // wl.split_tokens)
        n_slots = self.n_cslots + -(-self.wcap // wl.split_tokens)
        self.o_part = torch.empty((n_slots, wl.Hq, d), dtype=torch.float32, device=device)
        self.lse_part = torch.empty((n_slots, wl.Hq), dtype=torch.float32, device=device)
        self.o = torch.empty((layers, wl.Hq, d), dtype=torch.float32, device=device)
        self.lse = torch.empty((layers, wl.Hq), dtype=torch.float32, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.steps_done = 0
        self.h2d_bytes = 0

    def inputs(self, step: int):
        """Device q [L][Hq][d] and new rows [L][2][Hkv][d] of decode step ``step``."""
        q = np.stack([synth.queries(self.wl, layer=l, step=step, B=1)[0] for l in range(self.L)])
        new = np.stack([np.stack(synth.new_token(self.wl, l, step)) for l in range(self.L)])
        return to_dev_bits(q, self.device), to_dev_bits(new, self.device)

    def step(self, q, new_rows, variant=akv.AKV_VARIANT_AUTO, timeout_ms: int = -1):
        """One decode step over all layers; q [L][Hq][d], new_rows [L][2][Hkv][d] (device).
        Staged: the new row joins the device window, then one akv_staged_decode call per layer
        stages and attends the compact history, attends the window and merges.  Resident: the
        same attention calls over the compact rows in device memory (the comparison run)."""
        wl, H, d = self.wl, self.wl.Hkv, self.wl.d
        cs = self.compute_stream
        nw = self.W + self.steps_done + 1           # window tokens including the appended one
        per_chunk = self.chunk // wl.split_tokens
        n_wsplit = -(-nw // wl.split_tokens)
        n_chunks = -(-self.Tc // self.chunk)
        cs.wait_stream(torch.cuda.current_stream(self.device))  # the step's inputs
        for layer in range(self.L):
            win = self.win[layer]
            with torch.cuda.stream(cs):
                win[nw - 1].copy_(new_rows[layer])
            wb = win.data_ptr()
            wtier = akv.Tier(akv.AKV_TIER_BF16, wb, wb + H * d * 2, lens=[nw], slot_base=[self.n_cslots],
                             stride_seq=0, stride_head=d, stride_token=2 * H * d)
            if not self.resident:
                akv.akv_staged_decode(self.stager, akv.AKV_TIER_CODES4, self.host[layer], self.Tc, self.chunk,
                                      q[layer], wl.Hq, H, d, wl.scale, wl.split_tokens, None, wtier, self.o_part,
                                      self.lse_part, self.o_part.shape[0], self.o[layer:layer + 1],
                                      self.lse[layer:layer + 1], variant, self.err, self.copy_stream, cs)
                self.h2d_bytes += self.nrows * self.crow
                continue
            for c in range(n_chunks):
                tok0 = c * self.chunk
                ntc = min(self.chunk, self.Tc - tok0)
                base = self.host[layer].data_ptr() + (tok0 // 16) * self.crow
                tier = akv.Tier(akv.AKV_TIER_CODES4, base, base + H * self.bb, lens=[ntc], slot_base=[c * per_chunk],
                                stride_seq=0, stride_head=1, stride_token=2 * H)
                akv.akv_decode_attend(q[layer], 1, wl.Hq, H, d, wl.scale, [tier], wl.split_tokens, self.o_part,
                                      self.lse_part, self.o_part.shape[0], variant, self.err, cs)
            akv.akv_decode_attend(q[layer], 1, wl.Hq, H, d, wl.scale, [wtier], wl.split_tokens, self.o_part,
                                  self.lse_part, self.o_part.shape[0], variant, self.err, cs)
            akv.akv_merge_lse(self.o_part, self.lse_part, self.o_part.shape[0], [0], [self.n_cslots + n_wsplit], 1,
                              wl.Hq, d, self.o[layer:layer + 1], self.lse[layer:layer + 1], cs)
        torch.cuda.current_stream(self.device).wait_stream(cs)  # the results, for the caller's stream
        self.steps_done += 1

    def close(self):
        if not self.resident:
            self.stager.destroy()


class AgingHybrid:
    """A live hybrid batch whose exact window ages into the compact tier during decode.

    Sequence b starts with c_b = 16 floor((L_b - W) / 16) compact tokens and L_b - c_b in
    [W, W + 16) exact ones.  The exact window is a ring of R = W/16 + 2 pages of 16 BF16
    tokens per sequence (pool [B R, Hkv, 16, d]); the compact history is a growing list of
    code pages drawn from a seeded permutation of the code pool ([P, Hkv] blocks).  A decode
    step appends each sequence's new token to its window; a window that reaches W + 16 tokens
    has its oldest page encoded into the sequence's next code page (one akv_encode_history
    call over every aging sequence) and that ring page leaves the window.  Then both tiers
    are attended and merged.  Page tables live on the device; only entries that change are
    written."""

    def __init__(self, wl: synth.Workload, device, lens, W: int, max_steps: int, key_dist: str = "normal",
                 source: str = "host"):
        lens = np.asarray(lens, np.int64)
        assert W % 16 == 0 and W > 0 and np.all(lens >= W)
        H, d = wl.Hkv, wl.d
        self.wl, self.device, self.B, self.W = wl, device, len(lens), W
        self.bb = akv.codes4_block_bytes(d)
        self.c = ((lens - W) // 16 * 16).astype(np.int64)       # compact tokens
        self.win = (lens - self.c).astype(np.int64)              # exact tokens, in [W, W + 16)
        self.R = W // 16 + 2
        self.ring0 = np.zeros(self.B, np.int64)                  # ring page of the window's first page
        cap = self.c // 16 + max_steps // 16 + 2
        self.n_cp = int(cap.sum())
        perm = synth.page_permutation(wl, "aging-codes", self.n_cp)
        offs = np.concatenate([[0], np.cumsum(cap)])
        self.owned = [perm[offs[b]:offs[b + 1]] for b in range(self.B)]
        self.cp_table_np = np.full((self.B, int(cap.max())), -1, np.int32)
        for b in range(self.B):
            n = int(self.c[b] // 16)
            self.cp_table_np[b, :n] = self.owned[b][:n]
        self.ex_table_np = np.array([[b * self.R + j for j in range(self.R)] for b in range(self.B)], np.int32)
        self.ex_k = torch.zeros((self.B * self.R, H, 16, d), dtype=torch.int16, device=device)
        self.ex_v = torch.zeros_like(self.ex_k)
        self.cp_pool, self.cp_k, self.cp_v, cs, ch = code_page_pool(self.n_cp, H, d, device, zero=True)
        self.cp_strides = dict(stride_seq=cs, stride_head=ch)
        self.cp_table = torch.from_numpy(self.cp_table_np).to(device)
        self.ex_table = torch.from_numpy(self.ex_table_np).to(device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.k_hist, self.v_hist = [], []                        # host BF16 history (source="host")
        for b in range(self.B):
            L, c = int(lens[b]), int(self.c[b])
            if source == "host":
                k, v = synth.history_head_major(wl, b, L, key_dist=key_dist)
                self.k_hist.append(k)
                self.v_hist.append(v)
                kd, vd = to_dev_bits(k, device), to_dev_bits(v, device)
            else:
                g = synth.torch_generator(wl.seed, wl.name, "aging", b, device=device)
                kd = synth.torch_student_t3_bf16(g, (H, L, d), device) if key_dist == "student_t" \
                    else synth.torch_normal_bf16(g, (H, L, d), device)
                vd = synth.torch_normal_bf16(g, (H, L, d), device)
            if c > 0:
                src = akv.Tier(akv.AKV_TIER_BF16, kd, vd, lens=[c], stride_seq=0, stride_head=L * d, stride_token=d)
                dst = akv.Tier(akv.AKV_TIER_CODES4, self.cp_k, self.cp_v, lens=[c], paged=True,
                               page_table=self.cp_table[b:b + 1], page_table_stride=self.cp_table_np.shape[1],
                               n_pages=self.n_cp, **self.cp_strides)
                akv.akv_encode_history(src, dst, 1, H, d, self.err)
            w = L - c
            pages = -(-w // 16)
            ek = torch.zeros((H, pages * 16, d), dtype=torch.int16, device=device)
            ev = torch.zeros_like(ek)
            ek[:, :w] = kd[:, c:]
            ev[:, :w] = vd[:, c:]
            self.ex_k[b * self.R:b * self.R + pages] = ek.view(H, pages, 16, d).permute(1, 0, 2, 3)
            self.ex_v[b * self.R:b * self.R + pages] = ev.view(H, pages, 16, d).permute(1, 0, 2, 3)
        torch.cuda.synchronize(device)
        max_slots = int(sum(-(-(int(l) + max_steps) // wl.split_tokens) + 2 for l in lens))
        self.o_part = torch.empty((max_slots, wl.Hq, d), dtype=torch.float32, device=device)
        self.lse_part = torch.empty((max_slots, wl.Hq), dtype=torch.float32, device=device)
        self.o = torch.empty((self.B, wl.Hq, d), dtype=torch.float32, device=device)
        self.lse = torch.empty((self.B, wl.Hq), dtype=torch.float32, device=device)
        self.q = to_dev_bits(synth.queries(wl, B=self.B), device)
        self._enc_dev = torch.empty((self.B, 2), dtype=torch.int32, device=device)
        self.steps_done = 0
        # the step runs in the library: one akv_aging_step call appends, ages full window
        # pages into the compact tier, attends both tiers and merges
        self.ctx = akv.Aging(self.B, wl.Hq, H, d, wl.split_tokens, wl.scale, W, self.R, self._exact_tier(),
                             akv.Tier(akv.AKV_TIER_CODES4, self.cp_k, self.cp_v, lens=self.c.astype(np.int32),
                                      paged=True, page_table=self.cp_table,
                                      page_table_stride=self.cp_table_np.shape[1], n_pages=self.n_cp,
                                      **self.cp_strides),
                             self.c.astype(np.int32), self.win.astype(np.int32), self.ring0.astype(np.int32),
                             self.owned, self._enc_dev, self.o_part, self.lse_part, self.o_part.shape[0])
        self._aged0 = int(self.c.sum() // 16)
        self.aged_blocks = 0

    def _state(self):
        c, w, r, _ = self.ctx.state()
        self.c, self.win, self.ring0 = c.astype(np.int64), w.astype(np.int64), r.astype(np.int64)
        n_pages = self.c // 16
        for b in range(self.B):
            self.cp_table_np[b, :n_pages[b]] = self.owned[b][:n_pages[b]]
        self.aged_blocks = int(n_pages.sum()) - self._aged0

    def inputs(self, step: int):
        """Device q [B][Hq][d] and new K, V rows [B][Hkv][d] of decode step ``step``."""
        wl = self.wl
        q = synth.queries(wl, step=step + 1, B=self.B)
        kn = np.stack([synth.new_token(wl, 0, step, b)[0] for b in range(self.B)])
        vn = np.stack([synth.new_token(wl, 0, step, b)[1] for b in range(self.B)])
        return to_dev_bits(q, self.device), to_dev_bits(kn, self.device), to_dev_bits(vn, self.device)

    def _exact_tier(self, lens=None, slot_base=None):
        H, d = self.wl.Hkv, self.wl.d
        return akv.Tier(akv.AKV_TIER_BF16, self.ex_k, self.ex_v, lens=self.win if lens is None else lens,
                        slot_base=slot_base, paged=True, page_table=self.ex_table, page_table_stride=self.R,
                        n_pages=self.B * self.R, stride_seq=H * 16 * d, stride_head=16 * d, stride_token=d)

    def step(self, q, k_new, v_new, variant=akv.AKV_VARIANT_AUTO, stream=None, sync_state: bool = True):
        """Append one token per sequence, age full window pages, attend both tiers, merge:
        one akv_aging_step call.  sync_state=False skips reading the lengths back."""
        self.ctx.step(q, k_new, v_new, self.o, self.lse, variant, self.err, stream)
        self.steps_done += 1
        if sync_state:
            self._state()
