"""Oracle of the sparse (low-bit scan + top-delta) decode (TEST INFRASTRUCTURE ONLY).

Follows "Faster Than Flash: Exploiting Attention Sparsity for Efficient
Long-Context Decoding" (scifaro.com, abstract): a scan over low-bit keys
selects the blocks of the history that matter, by a top-delta rule that each
unit of work applies on its own (no global synchronisation), and exact
attention then runs over the selected blocks only.  The page gives no more
detail; the readings below are the plainest that fit it.

- Low-bit keys: per 64-token block of one (sequence, KV head),
  sk = max |K| / 127 (1 for an all-zero block) and k8 = rint(K / sk), int8.
  Rows at or past the sequence's length take no part and get k8 = 0.
- Low-bit query: per query head, sq = max |q| / 127 (1 when q = 0) and
  q8 = rint(q / sq).
- Scan: the approximate logit of token j for head g is
  s = ((scale * sq_g) * sk_B) * (q8_g . k8_j), the dot product exact in
  integers and every product rounded to fp32, in that order.
- Top-delta, per split of the dense decode (cut as there: T = ceil(L / 64)
  blocks into S = min(num_splits, T) splits, split s holding blocks
  [floor(s T / S), floor((s + 1) T / S))): M_g is the largest block maximum
  of head g in the split; a block is kept when some head of its group has a
  block maximum >= M_g - delta (fp32).
- Attention: exact, in fp64, over the tokens of the kept blocks of all
  splits, for every query head of the group.

Every floating-point step that decides which blocks are kept is done in
fp32 exactly as written, so that it is reproducible (select_blocks).  The
same rule is also given straight from its definition, with the logits and
the threshold in fp64 (select_blocks_exact): the codes and scales are the
same fp32 decisions, but no product is rounded to fp32.  The two agree on
every block whose decision lies farther from its threshold than the fp32
roundings can move it.  The attention over the kept tokens uses the fp64
oracle.
"""
from __future__ import annotations

import numpy as np

import oracle

BLOCK = 64


def _bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _lengths(seqlens, B: int, L: int) -> np.ndarray:
    if seqlens is None:
        return np.full(B, L, dtype=np.int64)
    return np.clip(np.asarray(seqlens, dtype=np.int64), 0, L)


def quantize_keys(k: np.ndarray, seqlens=None):
    """k [B, Hkv, L, D] bf16 bits (head-major, contiguous).

    Returns (k8 [B, Hkv, L, D] int8, sk [B, Hkv, ceil(L/64)] float32)."""
    B, Hkv, L, D = k.shape
    nblk = -(-L // BLOCK)
    n = _lengths(seqlens, B, L)
    kf = _bf16_to_f32(k).reshape(B, Hkv, L, D).copy()
    valid = np.arange(L)[None, :] < n[:, None]                      # [B, L]
    kf[~np.broadcast_to(valid[:, None, :, None], kf.shape)] = 0.0
    pad = nblk * BLOCK - L
    kp = np.concatenate([kf, np.zeros((B, Hkv, pad, D), np.float32)], axis=2)
    kp = kp.reshape(B, Hkv, nblk, BLOCK, D)
    amax = np.abs(kp).max(axis=(3, 4))                              # [B, Hkv, nblk]
    sk = np.where(amax > 0, amax / np.float32(127.0), np.float32(1.0)).astype(np.float32)
    k8 = np.clip(np.rint(kp / sk[..., None, None]), -127, 127).astype(np.int8)
    return k8.reshape(B, Hkv, nblk * BLOCK, D)[:, :, :L], sk


def quantize_query(q: np.ndarray):
    """q [..., D] bf16 bits -> (q8 [..., D] int8, sq [...] float32), per row."""
    qf = _bf16_to_f32(q)
    amax = np.abs(qf).max(axis=-1)
    sq = np.where(amax > 0, amax / np.float32(127.0), np.float32(1.0)).astype(np.float32)
    q8 = np.clip(np.rint(qf / sq[..., None]), -127, 127).astype(np.int8)
    return q8, sq


def split_blocks(max_len: int, num_splits: int):
    """Block ranges [b0, b1) of the splits: T = ceil(max_len / 64) blocks cut
    into S = min(num_splits, T) splits (one when T = 0), split s holding
    blocks [floor(s T / S), floor((s + 1) T / S))."""
    T = -(-max_len // BLOCK)
    S = min(num_splits, T) if T > 0 else 1
    return [(s * T // S, (s + 1) * T // S) for s in range(S)]


def select_blocks(q, k8, sk, scale: float, delta: float, num_splits: int, seqlens=None):
    """Kept-block mask [B, Hkv, nblk] (bool) of the top-delta rule.

    q [B, Hq, D] bf16 bits; k8, sk from quantize_keys."""
    B, Hkv, L, D = k8.shape
    Hq = q.shape[1]
    G = Hq // Hkv
    nblk = sk.shape[2]
    n = _lengths(seqlens, B, L)
    q8, sq = quantize_query(q)                                      # [B, Hq, D], [B, Hq]
    scale32 = np.float32(scale)
    delta32 = np.float32(delta)
    splits = split_blocks(L, num_splits)
    kept = np.zeros((B, Hkv, nblk), dtype=bool)
    for b in range(B):
        for h in range(Hkv):
            nb = -(-int(n[b]) // BLOCK)
            if nb == 0:
                continue
            qg = q8[b, h * G:(h + 1) * G].astype(np.int32)          # [G, D]
            kb = k8[b, h, :nb * BLOCK].astype(np.int32)
            dots = kb @ qg.T                                        # [tokens, G], exact
            qs = (scale32 * sq[b, h * G:(h + 1) * G]).astype(np.float32)       # [G]
            tok_blk = np.arange(dots.shape[0]) // BLOCK
            s = (qs[None, :] * sk[b, h, tok_blk][:, None]).astype(np.float32)
            s = (s * dots.astype(np.float32)).astype(np.float32)    # [tokens, G]
            s[np.arange(dots.shape[0]) >= n[b]] = -np.inf
            bmax = np.full((nb, G), -np.inf, dtype=np.float32)
            np.maximum.at(bmax, tok_blk, s)
            for s0, s1 in splits:                                   # the splits
                if s0 >= nb:
                    break
                s1 = min(nb, s1)
                M = bmax[s0:s1].max(axis=0)                         # [G]
                thr = (M - delta32).astype(np.float32)
                kept[b, h, s0:s1] = (bmax[s0:s1] >= thr[None, :]).any(axis=1)
    return kept


def block_maxima_exact(q, k8, sk, scale: float, seqlens=None):
    """Block maxima of the scan's logits from their definition, in fp64.

    For each (b, kv head) an array [nb, G] (nb = blocks holding tokens):
    max over the block's valid tokens j of scale * sq_g * sk_B * (q8_g . k8_j),
    with scale the fp32 value passed, the codes and scales of quantize_query
    and quantize_keys, the dot product exact in integers and the product of
    the four factors taken in fp64 (no rounding to fp32).  Returns a dict
    {(b, h): array}."""
    B, Hkv, L, D = k8.shape
    Hq = q.shape[1]
    G = Hq // Hkv
    n = _lengths(seqlens, B, L)
    q8, sq = quantize_query(q)
    sc = float(np.float32(scale))
    out = {}
    for b in range(B):
        nt = int(n[b])
        nb = -(-nt // BLOCK)
        for h in range(Hkv):
            qg = q8[b, h * G:(h + 1) * G].astype(np.int64)                 # [G, D]
            dots = k8[b, h, :nt].astype(np.int64) @ qg.T                    # [nt, G], exact
            factor = sc * sq[b, h * G:(h + 1) * G].astype(np.float64)       # [G]
            blk = np.arange(nt) // BLOCK
            logit = factor[None, :] * sk[b, h, blk].astype(np.float64)[:, None] * dots
            padded = np.full((nb * BLOCK, G), -np.inf)
            padded[:nt] = logit
            out[(b, h)] = padded.reshape(nb, BLOCK, G).max(axis=1)
    return out


def select_blocks_exact(q, k8, sk, scale: float, delta: float, num_splits: int, seqlens=None):
    """The top-delta rule on block_maxima_exact, in fp64, with the fp32 value
    of delta that the library receives.

    Returns (kept, certain), both [B, Hkv, nblk] bool.  For head g, block i
    of a split is kept when bmax_i >= M - delta, M the split's largest block
    maximum; since delta >= 0 this is bmax_i >= M_other - delta with M_other
    the largest maximum of the split's OTHER blocks (-inf when it has none).
    A decision is certain when no rounding of the scan to fp32 can flip it:
    for some head bmax_i - (M_other - delta) > eps, or for every head
    (M_other - delta) - bmax_i > eps, with
    eps = 2^-21 (|bmax_i| + |M_other| + |delta| + |M_other - delta|).
    Three fp32 roundings of each logit product and one of the subtraction move
    the compared values by at most 7 * 2^-24 times those magnitudes, which is
    below eps.  delta = +inf keeps every block, surely."""
    B, Hkv, L, D = k8.shape
    nblk = sk.shape[2]
    d = float(np.float32(delta))
    maxima = block_maxima_exact(q, k8, sk, scale, seqlens)
    kept = np.zeros((B, Hkv, nblk), dtype=bool)
    certain = np.zeros((B, Hkv, nblk), dtype=bool)
    for (b, h), bm in maxima.items():
        nb = bm.shape[0]
        if np.isinf(d):
            kept[b, h, :nb] = certain[b, h, :nb] = True
            continue
        for s0, s1 in split_blocks(L, num_splits):
            if s0 >= nb:
                break
            s1 = min(nb, s1)
            part = bm[s0:s1]                                                # [blocks, G]
            n_blk = part.shape[0]
            top = np.argmax(part, axis=0)                                   # [G]
            m1 = part.max(axis=0)
            second = np.full_like(m1, -np.inf)
            if n_blk > 1:
                rest = part.copy()
                rest[top, np.arange(part.shape[1])] = -np.inf
                second = rest.max(axis=0)
            other = np.where(np.arange(n_blk)[:, None] == top[None, :], second[None, :],
                             m1[None, :])                                   # M_other [blocks, G]
            thr = other - d
            with np.errstate(invalid="ignore"):
                gap = np.where(np.isneginf(other), np.inf, part - thr)
                eps = 2.0 ** -21 * (np.abs(part) + np.abs(other) + abs(d) + np.abs(thr))
                eps = np.where(np.isneginf(other), 0.0, eps)
            kept[b, h, s0:s1] = (gap >= 0).any(axis=1)
            certain[b, h, s0:s1] = (gap > eps).any(axis=1) | (-gap > eps).all(axis=1)
    return kept, certain


def sparse_decode(q, k, v, scale: float, delta: float, num_splits: int, seqlens=None,
                  groups=None, k8=None, sk=None):
    """fp64 attention over the kept blocks.

    q [B, Hq, D], k/v [B, Hkv, L, D] bf16 bits.  Returns (out [B, Hq, D],
    lse [B, Hq], kept [B, Hkv, nblk]); rows not in `groups` (iterable of
    (b, kv_head)) are NaN."""
    B, Hkv, L, D = k.shape
    Hq = q.shape[1]
    G = Hq // Hkv
    if k8 is None:
        k8, sk = quantize_keys(k, seqlens)
    kept = select_blocks(q, k8, sk, scale, delta, num_splits, seqlens)
    n = _lengths(seqlens, B, L)
    out = np.full((B, Hq, D), np.nan)
    lse = np.full((B, Hq), np.nan)
    if groups is None:
        groups = [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in groups:
        tok = np.arange(int(n[b]))
        tok = tok[kept[b, h, tok // BLOCK]]
        o, l = oracle.attend(q[b, h * G:(h + 1) * G], np.ascontiguousarray(k[b, h, tok]),
                             np.ascontiguousarray(v[b, h, tok]), scale)
        out[b, h * G:(h + 1) * G] = o
        lse[b, h * G:(h + 1) * G] = l
    return out, lse, kept
