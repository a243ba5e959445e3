"""Float64 CPU oracle for tiered single-token decode attention.

TEST INFRASTRUCTURE ONLY.  Plain, slow, obviously correct numpy code that states what
the GPU path must compute.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it.  It shares no code with the CUDA library
(``kv_cache_tiering_b200``) and imports nothing from it; the two meet only on the
seeded inputs of ``kv_cache_tiering_b200.synth``.

Sources (web pages, cited by title and section):
  * "Context beyond VRAM" (coreyjames.ai), sections "My approach" and "What I built":
    pinned host memory holds each context's attention history, a bounded device
    staging region holds what the step needs; an exact BF16 tier; a hybrid tier that
    keeps recent context exact and older history in a compact form the GPU reads
    directly, the two merged "with exact attention arithmetic".
  * "Bringing a serving stack up on new silicon", section "What I built": the
    attention path must emit the per-split attention statistic (log-sum-exp) that the
    memory layer needs to merge partial results.
  * "QuantForge V2 Walkthrough", section 1 "Triton Fused Kernels": codes map to
    centroids times a scale, and because the Hadamard rotation preserves dot products
    the query is rotated instead of inverse-rotating the compressed keys.
The pages give no formulas.  The compact form is fixed by the hybrid-tier workload:
Walsh-Hadamard-rotated vectors (d = 128, normalised), an fp16 per-token-per-head scale
equal to the L2 norm, and 4-bit codes into the 16-level Lloyd-Max table for N(0,1)
applied to the rotated coordinates times sqrt(d).

Readings where the pages are silent (the plainest reading the rest supports):
  * Hadamard order: Sylvester (natural) order, H_1 = [1], H_2n = [[H, H], [H, -H]];
    no random signs.  The unnormalised transform z = H x is computed by butterflies
    h = 1, 2, ..., d/2, each mapping (a, b) -> (a + b, a - b).
  * Scale: s = binary16(sqrt(ss)) with ss the sum of squares in float64 by pairwise
    halving (adjacent pairs, then adjacent pairs of pairs, ...); the stored binary16 s
    (not the exact norm) is used inside quantisation.
  * Code of coordinate i: the number of boundaries b_j = (c_j + c_{j+1}) / 2 with
    z_i > s * b_j (strict), so ties go to the lower level and a zero coordinate gets
    code 7.  s == 0 gives all codes 7.  Every s * b_j is exact in float64.
  * Packing (the pages fix no storage layout): byte k of a key code row holds code 2k
    in its low nibble and code 2k+1 in its high nibble.  A 16-token key block stores
    the 16 code rows (token order) followed by the 16 binary16 scales (little-endian);
    unused slots of a partial block hold the zero-vector encoding (codes 7, scale 0).
    A value block stores the same codes by token pairs instead -- byte k of pair row r
    holds code k of token 2r (low nibble) and of token 2r + 1 (high nibble) -- with the
    d bytes of pair row r cut into 8 units of d/8 bytes and unit u stored at position
    u XOR w(r), w(r) = 2 (r mod 4) for d = 128 and 4 (floor(r / 2) mod 2) for d = 64;
    then the 16 scales as for keys.  (This is the order the tensor-core product reads.)
  * Dequantisation: y_i = s * c[code_i] / sqrt(d) in the rotated domain,
    x_hat = H y / sqrt(d) in the original domain.
  * Rotation signs (the pages only name "Hadamard vs QR" trade-offs): an optional
    randomised rotation flips the signs of the coordinates whose bits are set before the
    transform, z = H (s . x), and the inverse applies them after, x_hat = s . (H y) / sqrt(d).
    With no bits set both reduce to the plain transform.  H S is still orthogonal up to
    the factor d, so the query is rotated the same way and dot products are preserved.
  * Softmax scale sigma is applied inside; LSE is the natural log of sum exp(scores);
    GQA head h reads KV head floor(h / G); an empty token range gives O = 0,
    LSE = -inf; splits of ``split_tokens`` tokens are aligned to the start of their
    tier, the last split may be partial.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from .lloyd_max import centroids_f16

# ----------------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------------


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of bfloat16 bit patterns (uint16) as float64."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of IEEE binary16 bit patterns (uint16) as float64."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def f64_to_f16_bits(x) -> np.ndarray:
    """Round float64 to IEEE binary16, round-to-nearest-even, one rounding (numpy)."""
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


# ----------------------------------------------------------------------------------
# rotation, scale, codes
# ----------------------------------------------------------------------------------


def fwht(x) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform z = H_d x along the last axis (float64).

    H_d is the Sylvester matrix; butterfly stage h (h = 1, 2, 4, ..., d/2) maps the
    pair (z[j], z[j + h]), for every j whose bit h is clear, to (a + b, a - b)."""
    z = np.array(x, dtype=np.float64, copy=True)
    lead, d = z.shape[:-1], z.shape[-1]
    if d & (d - 1):
        raise ValueError("Hadamard size must be a power of two")
    h = 1
    while h < d:
        blocks = z.reshape(*lead, d // (2 * h), 2, h)
        a, b = blocks[..., 0, :], blocks[..., 1, :]
        z = np.stack([a + b, a - b], axis=-2).reshape(*lead, d)
        h *= 2
    return z


def pairwise_sum_of_squares(x) -> np.ndarray:
    """sum_i x_i^2 along the last axis in float64, by pairwise halving:
    adjacent elements first, then adjacent pairs of pairs, and so on."""
    s = np.asarray(x, dtype=np.float64) ** 2
    while s.shape[-1] > 1:
        s = s[..., 0::2] + s[..., 1::2]
    return s[..., 0]


def scale_f16_bits(x) -> np.ndarray:
    """Per-vector scale: binary16 of the L2 norm (pairwise float64 sum, sqrt, one rounding)."""
    return f64_to_f16_bits(np.sqrt(pairwise_sum_of_squares(x)))


def code_boundaries() -> np.ndarray:
    """The 15 decision boundaries of the binary16 table: midpoints of neighbours (exact)."""
    c = centroids_f16()
    return (c[:-1] + c[1:]) / 2.0


@dataclass
class Encoded:
    codes: np.ndarray        # uint8 [n, d], one code (0..15) per coordinate
    scale_bits: np.ndarray   # uint16 [n], binary16 scale
    nonfinite: np.ndarray    # bool [n]: some input coordinate is inf or NaN
    overflow: np.ndarray     # bool [n]: the norm rounds to binary16 infinity


def sign_vector(sign_bits: int, d: int) -> np.ndarray:
    """s_i = -1 where bit i of sign_bits is set, else +1 (float64 [d])."""
    return np.array([-1.0 if (sign_bits >> i) & 1 else 1.0 for i in range(d)])


def rotate(x, sign_bits: int = 0) -> np.ndarray:
    """H (s . x), unnormalised, along the last axis."""
    x = np.asarray(x, dtype=np.float64)
    return fwht(x * sign_vector(sign_bits, x.shape[-1]))


def encode(x_bits, sign_bits: int = 0) -> Encoded:
    """Rotate, scale and quantise BF16 vectors x_bits uint16 [n, d].

    z = H (s . x) (unnormalised; s = +1 everywhere when sign_bits = 0), s = binary16(||x||),
    code_i = #{j : z_i > s * b_j}.
    A vector with a non-finite coordinate, or whose norm rounds to binary16 infinity,
    is refused: it is flagged and written as the zero-vector encoding (codes 7, scale 0).
    """
    x = bf16_bits_to_f64(np.atleast_2d(x_bits))
    n, d = x.shape
    nonfinite = ~np.all(np.isfinite(x), axis=1)
    xs = np.where(np.isfinite(x), x, 0.0)
    z = rotate(xs, sign_bits)
    s_bits = scale_f16_bits(xs)
    s = f16_bits_to_f64(s_bits)
    overflow = np.isinf(s)
    b = code_boundaries()
    codes = np.zeros((n, d), dtype=np.uint8)
    with np.errstate(invalid="ignore"):  # inf * 0 for refused rows, overwritten below
        for j in range(b.size):  # count boundaries strictly below each coordinate
            codes += (z > (s[:, None] * b[j])).astype(np.uint8)
    codes[s == 0.0] = 7
    refused = nonfinite | overflow  # written as the zero-vector encoding
    codes[refused] = 7
    s_bits = np.where(refused, np.uint16(0), s_bits).astype(np.uint16)
    return Encoded(codes=codes, scale_bits=s_bits, nonfinite=nonfinite, overflow=overflow)


def pack_codes(codes) -> np.ndarray:
    """Two codes per byte: code 2k in the low nibble, code 2k+1 in the high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


BLOCK_TOKENS = 16


def block_bytes(d: int) -> int:
    """Bytes of one 16-token block: 16 code rows of d/2 bytes, then 16 binary16 scales."""
    return BLOCK_TOKENS * (d // 2) + 2 * BLOCK_TOKENS


def pack_blocks(codes, scale_bits) -> np.ndarray:
    """Lay out the codes uint8 [T, d] and scales uint16 [T] of one (sequence, KV head)
    token stream as ceil(T / 16) blocks, uint8 [n_blocks, block_bytes(d)]."""
    codes = np.asarray(codes, dtype=np.uint8)
    scale_bits = np.asarray(scale_bits, dtype=np.uint16)
    t, d = codes.shape
    nb = -(-t // BLOCK_TOKENS)
    full_codes = np.full((nb * BLOCK_TOKENS, d), 7, dtype=np.uint8)
    full_codes[:t] = codes
    full_scales = np.zeros(nb * BLOCK_TOKENS, dtype=np.uint16)
    full_scales[:t] = scale_bits
    rows = pack_codes(full_codes).reshape(nb, BLOCK_TOKENS * (d // 2))
    sc = full_scales.reshape(nb, BLOCK_TOKENS).astype("<u2").view(np.uint8)
    return np.concatenate([rows, sc], axis=1)


def value_unit_swizzle(r: int, d: int) -> int:
    """w(r): the position XOR of the units of value pair row r (8 units of d/8 bytes)."""
    if d == 128:
        return 2 * (r % 4)
    if d == 64:
        return 4 * ((r // 2) % 2)
    raise ValueError("value blocks are defined for d = 64 and d = 128")


def pack_value_blocks(codes, scale_bits) -> np.ndarray:
    """Value-block layout of the codes uint8 [T, d] and scales uint16 [T] of one
    (sequence, KV head) stream: uint8 [ceil(T / 16), block_bytes(d)]."""
    codes = np.asarray(codes, dtype=np.uint8)
    scale_bits = np.asarray(scale_bits, dtype=np.uint16)
    t, d = codes.shape
    nb = -(-t // BLOCK_TOKENS)
    full_codes = np.full((nb * BLOCK_TOKENS, d), 7, dtype=np.uint8)
    full_codes[:t] = codes
    full_scales = np.zeros(nb * BLOCK_TOKENS, dtype=np.uint16)
    full_scales[:t] = scale_bits
    unit = d // 8
    out = np.zeros((nb, block_bytes(d)), dtype=np.uint8)
    for n in range(nb):
        blk = full_codes[n * BLOCK_TOKENS:(n + 1) * BLOCK_TOKENS]
        for r in range(BLOCK_TOKENS // 2):
            pair = (blk[2 * r] | (blk[2 * r + 1] << 4)).astype(np.uint8)  # byte k: dim k of both tokens
            w = value_unit_swizzle(r, d)
            for u in range(8):
                dst = r * d + (u ^ w) * unit
                out[n, dst:dst + unit] = pair[u * unit:(u + 1) * unit]
        out[n, BLOCK_TOKENS * (d // 2):] = full_scales[n * BLOCK_TOKENS:(n + 1) * BLOCK_TOKENS].astype("<u2").view(np.uint8)
    return out


def unpack_value_blocks(blocks, n_tokens: int, d: int):
    """Inverse of pack_value_blocks: codes uint8 [n_tokens, d], scales uint16 [n_tokens]."""
    blocks = np.asarray(blocks, dtype=np.uint8)
    nb = blocks.shape[0]
    unit = d // 8
    codes = np.empty((nb * BLOCK_TOKENS, d), dtype=np.uint8)
    for n in range(nb):
        for r in range(BLOCK_TOKENS // 2):
            w = value_unit_swizzle(r, d)
            pair = np.empty(d, dtype=np.uint8)
            for u in range(8):
                src = r * d + (u ^ w) * unit
                pair[u * unit:(u + 1) * unit] = blocks[n, src:src + unit]
            codes[n * BLOCK_TOKENS + 2 * r] = pair & 0x0F
            codes[n * BLOCK_TOKENS + 2 * r + 1] = pair >> 4
    sc = np.ascontiguousarray(blocks[:, BLOCK_TOKENS * (d // 2):]).view("<u2").reshape(-1)
    return codes[:n_tokens], sc[:n_tokens].astype(np.uint16)


def unpack_blocks(blocks, n_tokens: int, d: int):
    """Inverse of pack_blocks: codes uint8 [n_tokens, d], scales uint16 [n_tokens]."""
    blocks = np.asarray(blocks, dtype=np.uint8)
    nb = blocks.shape[0]
    rows = blocks[:, : BLOCK_TOKENS * (d // 2)].reshape(nb * BLOCK_TOKENS, d // 2)
    sc = np.ascontiguousarray(blocks[:, BLOCK_TOKENS * (d // 2):]).view("<u2").reshape(-1)
    return unpack_codes(rows)[:n_tokens], sc[:n_tokens].astype(np.uint16)


def dequantize_rotated(codes, scale_bits) -> np.ndarray:
    """y_i = s * c[code_i] / sqrt(d): the vector in the rotated, normalised basis."""
    codes = np.asarray(codes)
    d = codes.shape[-1]
    c = centroids_f16()
    s = f16_bits_to_f64(scale_bits)
    return s[..., None] * c[codes] / math.sqrt(d)


def dequantize(codes, scale_bits, sign_bits: int = 0) -> np.ndarray:
    """x_hat = s . (H y) / sqrt(d): the reconstructed vector in the original basis."""
    y = dequantize_rotated(codes, scale_bits)
    return fwht(y) / math.sqrt(y.shape[-1]) * sign_vector(sign_bits, y.shape[-1])


# ----------------------------------------------------------------------------------
# attention, splits, merge
# ----------------------------------------------------------------------------------


def attend(q, k, v, scale: float):
    """Softmax attention of one query q [d] over keys k [T, d] and values v [T, d].

    scores_t = scale * q . k_t;  O = sum_t softmax(scores)_t v_t;  LSE = ln sum_t exp(scores_t).
    T = 0 gives O = 0 and LSE = -inf."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if k.shape[0] == 0:
        return np.zeros(v.shape[-1]), -math.inf
    s = scale * (k @ q)
    m = float(np.max(s))
    w = np.exp(s - m)
    ell = float(np.sum(w))
    return (w @ v) / ell, m + math.log(ell)


def split_ranges(n_tokens: int, split_tokens: int):
    """Half-open token ranges of the splits of one tier: [0, S), [S, 2S), ..., the last partial."""
    return [(a, min(a + split_tokens, n_tokens)) for a in range(0, n_tokens, split_tokens)]


def merge_lse(o_parts, lse_parts):
    """Exact merge of split partials (O_s, LSE_s), s = 0..S-1 in order.

    M = max_s LSE_s, w_s = exp(LSE_s - M), L = sum_s w_s, O = sum_s w_s O_s / L,
    LSE = M + ln L.  No finite partial (S = 0 or all -inf) gives O = 0, LSE = -inf."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    d = o_parts.shape[-1]
    if lse_parts.size == 0 or not np.any(np.isfinite(lse_parts)):
        return np.zeros(d), -math.inf
    m = float(np.max(lse_parts))
    w = np.exp(lse_parts - m)
    big_l = float(np.sum(w))
    return (w @ o_parts) / big_l, m + math.log(big_l)


def gqa_kv_head(h: int, hq: int, hkv: int) -> int:
    """KV head read by query head h: contiguous groups of G = hq / hkv query heads."""
    return h // (hq // hkv)


def split_partials(q, k, v, scale: float, split_tokens: int):
    """Per-split (O_s, LSE_s) of one query over one tier's token stream k, v [T, d]."""
    outs = [attend(q, k[a:b], v[a:b], scale) for a, b in split_ranges(k.shape[0], split_tokens)]
    if not outs:
        return np.zeros((0, v.shape[-1])), np.zeros(0)
    return np.stack([o for o, _ in outs]), np.array([l for _, l in outs])


def decode_sequence(q, tiers, scale: float, split_tokens: int):
    """One decode step of one sequence.

    q: float64 [Hq, d].  tiers: list of (k, v), each float64 [Hkv, T_tier, d], in
    history order (older tier first).  Returns
      partials: list over tiers of (O [S_tier, Hq, d], LSE [S_tier, Hq]),
      merged:   (O [Hq, d], LSE [Hq]) from merge_lse over all partials in tier order,
      direct:   (O [Hq, d], LSE [Hq]) from attend over the concatenated history."""
    q = np.asarray(q, dtype=np.float64)
    hq, d = q.shape
    hkv = tiers[0][0].shape[0]
    partials = []
    for k, v in tiers:
        n_split = len(split_ranges(k.shape[1], split_tokens))
        o = np.zeros((n_split, hq, d))
        lse = np.zeros((n_split, hq))
        for h in range(hq):
            kh = gqa_kv_head(h, hq, hkv)
            o_h, l_h = split_partials(q[h], k[kh], v[kh], scale, split_tokens)
            o[:, h, :] = o_h
            lse[:, h] = l_h
        partials.append((o, lse))
    all_o = np.concatenate([p[0] for p in partials], axis=0)
    all_l = np.concatenate([p[1] for p in partials], axis=0)
    m_o = np.zeros((hq, d))
    m_l = np.zeros(hq)
    d_o = np.zeros((hq, d))
    d_l = np.zeros(hq)
    k_all = np.concatenate([t[0] for t in tiers], axis=1)
    v_all = np.concatenate([t[1] for t in tiers], axis=1)
    for h in range(hq):
        m_o[h], m_l[h] = merge_lse(all_o[:, h, :], all_l[:, h])
        kh = gqa_kv_head(h, hq, hkv)
        d_o[h], d_l[h] = attend(q[h], k_all[kh], v_all[kh], scale)
    return partials, (m_o, m_l), (d_o, d_l)
