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
- Top-delta, per split of the dense decode (chunking as there): M_g is the
  largest block maximum of head g in the split; a block is kept when some
  head of its group has a block maximum >= M_g - delta (fp32).
- Attention: exact, in fp64, over the tokens of the kept blocks of all
  splits, for every query head of the group.

Every floating-point step that decides which blocks are kept is done in
fp32 exactly as written, so that it is reproducible.  The attention over
the kept tokens uses the fp64 oracle.
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


def chunk_for(max_len: int, num_splits: int) -> int:
    per = -(-max_len // num_splits)
    c = -(-per // BLOCK) * BLOCK
    return max(c, BLOCK)


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
    chunk = chunk_for(L, num_splits)
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
            for s0 in range(0, nb, chunk // BLOCK):                 # the splits
                s1 = min(nb, s0 + chunk // BLOCK)
                M = bmax[s0:s1].max(axis=0)                         # [G]
                thr = (M - delta32).astype(np.float32)
                kept[b, h, s0:s1] = (bmax[s0:s1] >= thr[None, :]).any(axis=1)
    return kept


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
