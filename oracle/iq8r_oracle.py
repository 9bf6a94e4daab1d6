"""IQ8R oracle -- TEST INFRASTRUCTURE ONLY.

A plain, slow, CPU restatement of the IQ8R rotated W8A8 linear layer, written
to check the CUDA library against. Only the tests, the package's ``smoke()``
and the CPU-baseline leg of ``bench.py`` may import it; the library never
does, and the two share no code.

What it follows (the pages are model cards of the "radiance" engine):

* "Qwen3.8-27B IQ8R + DFlash2 -- radiance container", table row "Weights":
  the trunk linears hold int8 codes in -127..127 with one u8 scale for every
  row and 256-wide block of K, below one bf16 scale per row; every 128 of K
  is first rotated by a Hadamard transform that is not normalised. The
  lm_head holds int8 codes with one bf16 scale for every row and 128-wide
  block of K.
* same page, table row "Activations": the activations are int8 too, in the
  same rotated domain (W8A8).
* same page, "How this file was made", the recipe rules
  ``codes=i8 group=256 scale=u8 scale2=bf16 block2=1x* transform=fwht128
  clamp=sym`` (trunk) and ``codes=i8 group=128 scale=bf16 clamp=sym``
  (lm_head).
* "Qwen3.8-Flash-Next, IQR-V4 -- radiance container", row "Routed experts":
  the rotation is a 128-point Walsh-Hadamard transform.

Where the pages are silent the oracle writes down a stated definition (the
library follows it exactly):

* fp32 transform order: radix-2 butterflies, h = 1, 2, 4, ..., 64, each
  (a, b) -> (a + b, a - b) with round-to-nearest-even, no fused ops;
* activation scale: one per token (row), a = amax / 127, codes
  rint(x' * (127 / amax)) clamped to +-127; a row whose amax is below 2^-64
  is first multiplied by 2^64 (exact), so that 127 / amax stays finite;
* trunk scales: step d[n, g] = float(s2[n]) * s1[n, g]; s2 = bf16 of
  R[n] / (127 * 255) rounded up, s1 = min(255, ceil(A[n, g] / (127 * s2)));
* lm_head scale: s[n, g] = bf16 of A[n, g] / 127 rounded up;
* rounding: round-half-to-even wherever a value is rounded to nearest;
* the factor 1/128 (H H = 128 I) is applied to the output.

Also written here: ``pack_search`` (the recipes' rule=search: least-error
scales among the RTN scale and the 15 below it, for all three formats),
``pack_cb4`` / ``decode_cb4`` (the drafter's 16-level codebook: nearest level
under s = bf16 of A / 127 rounded up, ties to the larger level) and
``rescore`` (the layer at a list of candidate rows).

Parity unpinned: the choice of the scale rules above (per-token activation
scale, the s2/s1 composition, the lm_head scale rule, the search window and
its error measure, the codebook's scale and tie rule) and of the butterfly
order. They are stated definitions, not facts the pages fix; the tests pin
everything that follows from them.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "GROUP_TRUNK",
    "GROUP_HEAD",
    "CODE_MAX",
    "SUB_MAX",
    "bf16_to_f32",
    "f32_to_bf16_exact",
    "bf16_round_up",
    "bf16_round_nearest",
    "hadamard128",
    "fwht128_f32",
    "fwht128_f64",
    "act_quant",
    "pack",
    "pack_search",
    "pack_cb4",
    "decode_cb4",
    "CB4_TABLE",
    "SEARCH_WINDOW",
    "packed_sizes",
    "partials",
    "linear",
    "linear_bf16",
    "rescore",
]

GROUP_TRUNK = 256  # trunk: a u8 sub-scale for every (row, 256-wide block of K) (IQ8R page, "Weights")
GROUP_HEAD = 128   # lm_head: a bf16 scale for every (row, 128-wide block of K) (IQ8R page, "Weights")
CODE_MAX = 127     # codes in -127..127, clamp=sym (IQ8R page, "Weights" and recipe)
SUB_MAX = 255      # largest u8 sub-scale (recipe: scale=u8)
ROT = 128          # fwht128: the rotation acts on each 128 of K
# Rows whose rotated absmax is below ACT_TINY are quantised after an exact
# multiplication by ACT_PRESCALE (see act_quant).
ACT_TINY = np.float32(2.0 ** -64)
ACT_PRESCALE = np.float32(2.0 ** 64)
# The drafter's 16-level integer codebook (IQ8R page, "How this file was
# made": the dflash recipe lines, table=-127;-97;...;97;127, group=128
# scale=bf16 transform=fwht128): index i (4 bits) stands for CB4_TABLE[i].
CB4_TABLE = np.array([-127, -97, -75, -58, -43, -30, -18, -6, 6, 18, 30, 43, 58, 75, 97, 127], dtype=np.int64)


# ---------------------------------------------------------------- bf16 helpers

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact widening)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_exact(v: np.ndarray) -> np.ndarray:
    """float32 values that are already bf16-representable -> bit patterns."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("value is not representable in bf16")
    return (u >> np.uint32(16)).astype(np.uint16)


_BF16_MIN_NORMAL = 2.0 ** -126
_BF16_SUB_EXP = 133  # bf16 subnormal spacing is 2**-133 (7 stored mantissa bits)


def bf16_round_up(v: np.ndarray) -> np.ndarray:
    """Smallest bf16 value >= v, for finite v >= 0. Returns float32 values.

    Written from the format: a normal bf16 carries 8 significant bits, so a
    value m * 2**e (m in [0.5, 1)) rounds up to ceil(m * 2**8) * 2**(e - 8);
    below 2**-126 the grid is the subnormal one, multiples of 2**-133.
    """
    x = np.asarray(v, dtype=np.float64)
    if np.any(x < 0) or not np.all(np.isfinite(x)):
        raise ValueError("bf16_round_up expects finite non-negative input")
    m, e = np.frexp(x)
    normal = np.ldexp(np.ceil(np.ldexp(m, 8)), e - 8)
    sub = np.ldexp(np.ceil(np.ldexp(x, _BF16_SUB_EXP)), -_BF16_SUB_EXP)
    r = np.where(x >= _BF16_MIN_NORMAL, normal, sub)
    with np.errstate(over="ignore"):
        return r.astype(np.float32)


def bf16_round_nearest(v: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16, nearest with ties to even; bit patterns.

    Same grid as ``bf16_round_up``; ``np.rint`` rounds halves to even.
    Values past the largest bf16 (and its half-ulp) become +-inf.
    """
    x = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(x)
    normal = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    sub = np.ldexp(np.rint(np.ldexp(x, _BF16_SUB_EXP)), -_BF16_SUB_EXP)
    r = np.where(np.abs(x) >= _BF16_MIN_NORMAL, normal, sub)
    with np.errstate(over="ignore"):
        r32 = r.astype(np.float32)  # exact, or +-inf past the bf16 range
    return (np.ascontiguousarray(r32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ----------------------------------------------------------------- transform

def hadamard128() -> np.ndarray:
    """The 128x128 unnormalised Hadamard matrix, natural (Sylvester) order.

    H[i][j] = (-1) ** popcount(i & j): the rotation of the IQ8R page
    ("Weights"), a Hadamard transform without normalisation, which the
    Flash-Next page ("Routed experts") names a 128-point Walsh-Hadamard
    rotation. No 1/sqrt(128) factor.
    """
    i = np.arange(ROT)
    a = i[:, None] & i[None, :]
    pc = np.zeros_like(a)
    for bit in range(7):
        pc += (a >> bit) & 1
    return np.where(pc % 2 == 0, 1, -1).astype(np.int64)


def fwht128_f32(v: np.ndarray) -> np.ndarray:
    """fwht128 of each consecutive 128 of the last axis, in float32.

    Stated definition of the fp32 arithmetic (the pages give none): radix-2
    butterflies in place, stage h = 1, 2, 4, ..., 64 in that order; for every
    index i with (i & h) == 0 the pair (v[i], v[i+h]) becomes
    (v[i] + v[i+h], v[i] - v[i+h]), each an IEEE float32 add or subtract.
    Within a stage the butterflies are independent, so doing them together
    changes no rounding.
    """
    v = np.asarray(v, dtype=np.float32)
    if v.shape[-1] % ROT:
        raise ValueError("last axis must be a multiple of 128")
    x = v.reshape(-1, ROT).copy()
    h = 1
    while h < ROT:
        y = x.reshape(x.shape[0], ROT // (2 * h), 2, h)
        lo = y[:, :, 0, :].copy()
        hi = y[:, :, 1, :].copy()
        y[:, :, 0, :] = lo + hi
        y[:, :, 1, :] = lo - hi
        h *= 2
    return x.reshape(v.shape)


def fwht128_f64(v: np.ndarray) -> np.ndarray:
    """fwht128 in float64 as the matrix product with ``hadamard128()``."""
    v = np.asarray(v, dtype=np.float64)
    if v.shape[-1] % ROT:
        raise ValueError("last axis must be a multiple of 128")
    H = hadamard128().astype(np.float64)
    return (v.reshape(-1, ROT) @ H.T).reshape(v.shape)


# ------------------------------------------------------------ activations

def act_quant(x_bits: np.ndarray, rotate: bool = True):
    """Rotate and quantise activations to int8, one scale per token.

    The activations are int8 in the weights' rotated domain, W8A8 (IQ8R page,
    "Activations"). The granularity is not given; the stated definition is per token (row):

      x' = fwht128(x) in float32 (or x itself when ``rotate`` is false),
      amax = max |x'|, a = amax / 127 (float32 divide),
      c = 2^64 if amax < 2^-64 else 1 (a power of two: x' c and amax c are exact),
      inv = 127 / (amax c) (float32 divide),
      q = clamp(rint((x' c) * inv), -127, 127).

    For every row whose 127 / amax is a finite float32 the factor c changes
    no code: (x' c) * (127 / (amax c)) is the same real number as
    x' * (127 / amax), so it rounds the same way. It only defines the rows
    with amax < 127 / FLT_MAX (about 3.7e-37), where 127 / amax overflows.
    A row with amax == 0 gives a = 0 and all-zero codes. Rows whose x' is not
    finite (non-finite inputs, or a transform that overflows float32) are
    outside the definition.
    Returns (q int8 [M, K], a float32 [M]).
    """
    x = bf16_to_f32(x_bits)
    if x.ndim != 2:
        raise ValueError("x must be [M, K]")
    xr = fwht128_f32(x) if rotate else x.copy()
    amax = np.max(np.abs(xr), axis=1) if xr.shape[1] else np.zeros(xr.shape[0], np.float32)
    q = np.zeros(xr.shape, dtype=np.int8)
    a = np.zeros(xr.shape[0], dtype=np.float32)
    nz = amax > 0
    if np.any(nz):
        c = np.where(amax[nz] < ACT_TINY, ACT_PRESCALE, np.float32(1.0)).astype(np.float32)
        inv = np.float32(CODE_MAX) / (amax[nz] * c)
        t = (xr[nz] * c[:, None]) * inv[:, None]
        q[nz] = np.clip(np.rint(t), -CODE_MAX, CODE_MAX).astype(np.int8)
        a[nz] = amax[nz] / np.float32(CODE_MAX)
    return q, a


# ---------------------------------------------------------------- weights

def packed_sizes(fmt: str, n: int, k: int):
    """Byte sizes of (codes, sub-scales, scales) for a packed [n, k] weight."""
    if fmt == "g256":
        return n * k, n * (k // GROUP_TRUNK), 2 * n
    if fmt == "g128":
        return n * k, 0, 2 * n * (k // GROUP_HEAD)
    if fmt == "cb4":
        return n * k // 2, 0, 2 * n * (k // GROUP_HEAD)
    raise ValueError(fmt)


def pack(w_bits: np.ndarray, fmt: str = "g256", rotate: bool = True):
    """Round-to-nearest packing of a bf16 weight [N, K] (the recipe's ``rtn``).

    Trunk, ``fmt="g256"`` (recipe ``codes=i8 group=256 scale=u8 scale2=bf16
    block2=1x* transform=fwht128 clamp=sym``). Stated composition d = s2*s1:

      W' = fwht128(W) in float32,
      A[n, g] = max |W'| over the 256-block g,  R[n] = max_g A[n, g],
      s2[n] = bf16 of float32(R / 32385) rounded up (32385 = 127 * 255),
      s1[n, g] = min(255, ceil(A / (127 * s2))) (float32 divide), 0 if s2 = 0,
      codes = clamp(rint(W' / (s2 * s1)), -127, 127) (float32 divide),
      0 where s2 * s1 = 0.

    lm_head, ``fmt="g128"`` (recipe ``codes=i8 group=128 scale=bf16
    clamp=sym``): s[n, g] = bf16 of float32(A / 127) rounded up over each
    128-block; codes = clamp(rint(W' / s), -127, 127), 0 where s = 0.

    Returns (codes int8 [N, K], sub uint8 [N, K/256] or None,
    scale bf16 bits: [N] for g256, [N, K/128] for g128).
    """
    w = bf16_to_f32(w_bits)
    if w.ndim != 2:
        raise ValueError("w must be [N, K]")
    n, k = w.shape
    wr = fwht128_f32(w) if rotate else w.copy()
    if fmt == "g256":
        if k % GROUP_TRUNK:
            raise ValueError("K must be a multiple of 256")
        ng = k // GROUP_TRUNK
        blocks = wr.reshape(n, ng, GROUP_TRUNK)
        A = np.max(np.abs(blocks), axis=2)                       # float32 [n, ng]
        R = np.max(A, axis=1)                                   # float32 [n]
        s2 = bf16_round_up(R / np.float32(CODE_MAX * SUB_MAX))  # float32 [n]
        den = np.float32(CODE_MAX) * s2                         # exact (8 x 7 bits)
        s1 = np.zeros((n, ng), dtype=np.float32)
        ok = s2 > 0
        if np.any(ok):
            s1[ok] = np.minimum(np.float32(SUB_MAX), np.ceil(A[ok] / den[ok, None]))
        d = s2[:, None] * s1                                    # exact (8 x 8 bits)
        codes = np.zeros((n, ng, GROUP_TRUNK), dtype=np.int8)
        dz = d > 0
        if np.any(dz):
            t = blocks[dz] / d[dz][:, None]
            codes[dz] = np.clip(np.rint(t), -CODE_MAX, CODE_MAX).astype(np.int8)
        return codes.reshape(n, k), s1.astype(np.uint8), f32_to_bf16_exact(s2)
    if fmt == "g128":
        if k % GROUP_HEAD:
            raise ValueError("K must be a multiple of 128")
        ng = k // GROUP_HEAD
        blocks = wr.reshape(n, ng, GROUP_HEAD)
        A = np.max(np.abs(blocks), axis=2)
        s = bf16_round_up(A / np.float32(CODE_MAX))             # float32 [n, ng]
        codes = np.zeros((n, ng, GROUP_HEAD), dtype=np.int8)
        sz = s > 0
        if np.any(sz):
            t = blocks[sz] / s[sz][:, None]
            codes[sz] = np.clip(np.rint(t), -CODE_MAX, CODE_MAX).astype(np.int8)
        return codes.reshape(n, k), None, f32_to_bf16_exact(s)
    raise ValueError(fmt)


def pack_cb4(w_bits: np.ndarray, rotate: bool = True):
    """The drafter's codebook format: 4-bit indices into CB4_TABLE with a
    bf16 scale per (row, 128 of K), in the rotated domain (the dflash recipe
    lines: ``rtn table=... group=128 scale=bf16 transform=fwht128``).

    Stated reading: s = bf16 of A / 127 rounded up (A the group's max |w'|,
    so the end levels +-127 cover every value), and each value takes the
    level nearest to w' / s (float32 divide), ties going to the larger level;
    a group with s = 0 takes index 8 (level +6, contributing 0). Two indices a
    byte, the even K position in the low nibble.

    Returns (packed uint8 [N, K/2], scale bf16 bits [N, K/128]).
    """
    w = bf16_to_f32(w_bits)
    n, k = w.shape
    if k % GROUP_HEAD:
        raise ValueError("K must be a multiple of 128")
    wr = fwht128_f32(w) if rotate else w.copy()
    ng = k // GROUP_HEAD
    blocks = wr.reshape(n, ng, GROUP_HEAD)
    A = np.max(np.abs(blocks), axis=2)
    s = bf16_round_up(A / np.float32(CODE_MAX))
    idx = np.full((n, ng, GROUP_HEAD), 8, dtype=np.uint8)
    sz = s > 0
    if np.any(sz):
        idx[sz] = _cb4_indices(blocks[sz], s[sz])
    return _cb4_nibbles(idx.reshape(n, k)), f32_to_bf16_exact(s)


def _cb4_indices(blocks: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Index of the level nearest to w' / s for each value of blocks
    [..., G] at scales s [...] (> 0): float32 quotient, float64 distances,
    ties to the larger level."""
    t = (blocks / s[..., None]).astype(np.float64)
    dist = np.abs(t[..., None] - CB4_TABLE.astype(np.float64))  # [..., G, 16]
    # least distance, ties to the larger level: search from the top index down
    return (15 - np.argmin(dist[..., ::-1], axis=-1)).astype(np.uint8)


def _cb4_nibbles(idx: np.ndarray) -> np.ndarray:
    """Indices [N, K] -> bytes [N, K/2], the even K position in the low nibble."""
    return (idx[:, 0::2] | (idx[:, 1::2] << 4)).astype(np.uint8)


def decode_cb4(packed: np.ndarray) -> np.ndarray:
    """The codebook values of packed indices: int8 [N, K]."""
    p = np.asarray(packed, dtype=np.uint8)
    idx = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    idx[:, 0::2] = p & 0x0F
    idx[:, 1::2] = p >> 4
    return CB4_TABLE[idx].astype(np.int8)


SEARCH_WINDOW = 16  # scale candidates tried by pack_search: the RTN scale and the 15 below it


def _group_sse(blocks: np.ndarray, d: np.ndarray) -> np.ndarray:
    """Squared reconstruction error of each group, sum over k in order.

    blocks: float32 [..., G] rotated weights; d: float32 [...] steps (> 0).
    Codes are the packer's (float32 divide, rint, clamp to +-127); each error
    term is (w' - code * d) squared in float64 and the terms are added left
    to right (a cumulative sum), the order the C++ packer uses.
    """
    q = np.clip(np.rint(blocks / d[..., None]), -CODE_MAX, CODE_MAX)
    e = blocks.astype(np.float64) - q.astype(np.float64) * d[..., None].astype(np.float64)
    return np.cumsum(e * e, axis=-1)[..., -1]


def _cb4_sse(blocks: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Squared reconstruction error of each codebook group at scale s (> 0):
    (w' - level * s) squared in float64, the levels those of
    ``_cb4_indices``, the terms added left to right."""
    lv = CB4_TABLE[_cb4_indices(blocks, s)].astype(np.float64)
    e = blocks.astype(np.float64) - lv * s[..., None].astype(np.float64)
    return np.cumsum(e * e, axis=-1)[..., -1]


def pack_search(w_bits: np.ndarray, fmt: str = "g256", rotate: bool = True, window: int = SEARCH_WINDOW):
    """The recipes' ``rule=search``: per group, the scale with least
    reconstruction error. "Qwen3.8-Flash-Next, IQR-V4 -- radiance
    container", row "Trunk", picks one scale per 128 columns by a search for
    the least error; the IQ8R recipe lines carry ``rule=search``, the trunk's
    and the drafter's codebook lines alike.

    Stated reading: start from the RTN scale of ``pack`` (the smallest that
    clips nothing) and try it and the ``window - 1`` next smaller ones --
    trunk: s1, s1 - 1, ... (s1 >= 1) under the unchanged row scale s2;
    lm_head and codebook: s and the next smaller bf16 values (> 0). Smaller
    steps clip the group's largest values but refine the rest. The error of a
    candidate is the sum of (w' - value * step)**2 over the group, the value
    the code (``_group_sse``) or the nearest level (``_cb4_sse``); the least
    wins, ties go to the larger scale. Same returns as ``pack`` (for "cb4":
    packed indices, None, scales).
    """
    if fmt == "cb4":
        return _pack_search_cb4(w_bits, rotate, window)
    codes, sub, scale = pack(w_bits, fmt, rotate)
    w = bf16_to_f32(w_bits)
    n, k = w.shape
    wr = fwht128_f32(w) if rotate else w.copy()
    if fmt == "g256":
        ng = k // GROUP_TRUNK
        s2 = bf16_to_f32(scale)
        sub = sub.copy()
        codes = codes.reshape(n, ng, GROUP_TRUNK).copy()
        for r0 in range(0, n, 256):  # rows in chunks: the candidates' errors take memory
            r1 = min(n, r0 + 256)
            blocks = wr[r0:r1].reshape(r1 - r0, ng, GROUP_TRUNK)
            s1_rtn = sub[r0:r1].astype(np.float32)
            best = np.full((r1 - r0, ng), np.inf)
            best_s1 = s1_rtn.copy()
            for i in range(window):
                s1 = s1_rtn - np.float32(i)
                ok = (s1 >= 1) & (s2[r0:r1, None] > 0)
                d = np.where(ok, s2[r0:r1, None] * s1, np.float32(1))
                sse = _group_sse(blocks, d)
                better = ok & (sse < best)
                best = np.where(better, sse, best)
                best_s1 = np.where(better, s1, best_s1)
            sub[r0:r1] = best_s1.astype(np.uint8)
            d = s2[r0:r1, None] * best_s1
            dz = d > 0
            q = np.zeros(blocks.shape, np.int8)
            if np.any(dz):
                q[dz] = np.clip(np.rint(blocks[dz] / d[dz][:, None]), -CODE_MAX, CODE_MAX).astype(np.int8)
            codes[r0:r1] = q
        return codes.reshape(n, k), sub, scale
    if fmt == "g128":
        ng = k // GROUP_HEAD
        scale = scale.copy()
        codes = codes.reshape(n, ng, GROUP_HEAD).copy()
        for r0 in range(0, n, 256):
            r1 = min(n, r0 + 256)
            blocks = wr[r0:r1].reshape(r1 - r0, ng, GROUP_HEAD)
            b_rtn = scale[r0:r1].astype(np.int64)
            best = np.full((r1 - r0, ng), np.inf)
            best_b = b_rtn.copy()
            for i in range(window):
                b = b_rtn - i
                ok = (b_rtn > 0) & (b >= 1)  # positive bf16 bit patterns: one step down is the next smaller value
                s = bf16_to_f32(np.where(ok, b, 0x3F80).astype(np.uint16))
                sse = _group_sse(blocks, s)
                better = ok & (sse < best)
                best = np.where(better, sse, best)
                best_b = np.where(better, b, best_b)
            scale[r0:r1] = best_b.astype(np.uint16)
            s = bf16_to_f32(scale[r0:r1])
            sz = s > 0
            q = np.zeros(blocks.shape, np.int8)
            if np.any(sz):
                q[sz] = np.clip(np.rint(blocks[sz] / s[sz][:, None]), -CODE_MAX, CODE_MAX).astype(np.int8)
            codes[r0:r1] = q
        return codes.reshape(n, k), None, scale
    raise ValueError(fmt)


def _pack_search_cb4(w_bits: np.ndarray, rotate: bool, window: int):
    """``pack_search`` for the codebook format: the bf16 scale candidates of
    the lm_head, scored by ``_cb4_sse``; the indices are those of the chosen
    scale."""
    _, scale = pack_cb4(w_bits, rotate)
    w = bf16_to_f32(w_bits)
    n, k = w.shape
    wr = fwht128_f32(w) if rotate else w.copy()
    ng = k // GROUP_HEAD
    scale = scale.copy()
    idx = np.full((n, ng, GROUP_HEAD), 8, dtype=np.uint8)
    for r0 in range(0, n, 64):  # rows in chunks: the level distances take memory
        r1 = min(n, r0 + 64)
        blocks = wr[r0:r1].reshape(r1 - r0, ng, GROUP_HEAD)
        b_rtn = scale[r0:r1].astype(np.int64)
        best = np.full((r1 - r0, ng), np.inf)
        best_b = b_rtn.copy()
        for i in range(window):
            b = b_rtn - i
            ok = (b_rtn > 0) & (b >= 1)  # positive bf16 bit patterns: one step down is the next smaller value
            s = bf16_to_f32(np.where(ok, b, 0x3F80).astype(np.uint16))
            sse = _cb4_sse(blocks, s)
            better = ok & (sse < best)
            best = np.where(better, sse, best)
            best_b = np.where(better, b, best_b)
        scale[r0:r1] = best_b.astype(np.uint16)
        s = bf16_to_f32(scale[r0:r1])
        sz = s > 0
        if np.any(sz):
            sub_idx = idx[r0:r1]
            sub_idx[sz] = _cb4_indices(blocks[sz], s[sz])
    return _cb4_nibbles(idx.reshape(n, k)), None, scale


# ------------------------------------------------------------------ linear

def partials(xq: np.ndarray, codes: np.ndarray, group: int) -> np.ndarray:
    """P[m, n, g] = sum over block g of xq[m, k] * codes[n, k], exact int64.

    Each block product is a float64 matrix product of small integers: every
    term is below 2**14 and every block sum below 2**22 in magnitude, so the
    float64 result is the exact integer whatever the summation order.
    """
    xq = np.asarray(xq)
    codes = np.asarray(codes)
    m, k = xq.shape
    n, k2 = codes.shape
    if k != k2 or k % group:
        raise ValueError("shape mismatch")
    ng = k // group
    out = np.empty((m, n, ng), dtype=np.int64)
    for g in range(ng):
        xs = xq[:, g * group:(g + 1) * group].astype(np.float64)
        ws = codes[:, g * group:(g + 1) * group].astype(np.float64)
        out[:, :, g] = np.rint(xs @ ws.T).astype(np.int64)
    return out


def linear(xq: np.ndarray, a: np.ndarray, fmt: str, codes: np.ndarray,
           sub: np.ndarray | None, scale_bits: np.ndarray, rotated: bool = True) -> np.ndarray:
    """The layer output in float64 before its bf16 rounding, y64 [M, N].

    Trunk: y = a[m] * s2[n] * S[m, n] / 128, S = sum_g s1[n, g] * P[m, n, g]
    (S exact in int64). lm_head: y = a[m] / 128 * sum_g s[n, g] * P[m, n, g]
    in float64: each term is exact (8 significant bits of the bf16 scale
    times an integer below 2^22), the sum of the K/128 terms is rounded, with
    a relative error of order (K/128) 2^-53, far below any tolerance used.
    The 1/128 undoes H H = 128 I and is dropped when the weight was packed
    unrotated.
    """
    a64 = np.asarray(a, dtype=np.float32).astype(np.float64)
    if fmt == "g256":
        P = partials(xq, codes, GROUP_TRUNK)
        S = np.einsum("mng,ng->mn", P, np.asarray(sub).astype(np.int64))
        s2 = bf16_to_f32(scale_bits).astype(np.float64)
        y = a64[:, None] * s2[None, :] * S.astype(np.float64)
    elif fmt in ("g128", "cb4"):
        # cb4: codes are the packed indices; their values are the codebook's
        vals = decode_cb4(codes) if fmt == "cb4" else codes
        P = partials(xq, vals, GROUP_HEAD)
        s = bf16_to_f32(scale_bits).astype(np.float64)
        y = a64[:, None] * np.einsum("mng,ng->mn", P.astype(np.float64), s)
    else:
        raise ValueError(fmt)
    if rotated:
        y = y / 128.0
    return y


def rescore(xq: np.ndarray, a: np.ndarray, fmt: str, codes: np.ndarray, sub: np.ndarray | None,
            scale_bits: np.ndarray, cand: np.ndarray, rotated: bool = True) -> np.ndarray:
    """Candidate rescoring in float64, out64 [M, C]: the layer output of each
    token at its C candidate weight rows, out[t, j] = y[t, cand[t, j]].

    "Qwen3.8-27B IQ8R + DFlash2 -- radiance container", row "Speculator": the
    drafter's 2-bit head proposes 32 candidates that are rescored against
    the model's own head. Written per (token, candidate) pair with its own
    int64 dot products (not a gather from ``linear``), so that the tests can
    pin one against the other.
    """
    xq = np.asarray(xq, dtype=np.int64)
    cand = np.asarray(cand, dtype=np.int64)
    m, c = cand.shape
    k = xq.shape[1]
    g = GROUP_TRUNK if fmt == "g256" else GROUP_HEAD
    ng = k // g
    out = np.zeros((m, c), np.float64)
    for t in range(m):
        a64 = float(np.float32(a[t]))
        for j in range(c):
            r = int(cand[t, j])
            w = np.asarray(codes[r], dtype=np.int64)
            # P over each block of the row: exact integer dot products
            P = (xq[t].reshape(ng, g) * w.reshape(ng, g)).sum(axis=1)
            if fmt == "g256":
                S = int((P * np.asarray(sub[r], dtype=np.int64)).sum())
                v = a64 * float(bf16_to_f32(np.asarray([scale_bits[r]]))[0]) * float(S)
            else:
                s = bf16_to_f32(np.asarray(scale_bits[r])).astype(np.float64)
                v = a64 * float((P.astype(np.float64) * s).sum())
            out[t, j] = v / 128.0 if rotated else v
    return out


def linear_bf16(y64: np.ndarray) -> np.ndarray:
    """bf16 output bits: y64 rounded to nearest, ties to even."""
    return bf16_round_nearest(y64)
