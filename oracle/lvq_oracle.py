"""LoopVQ oracle: a plain, slow fp64 CPU implementation of the hot path.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
baseline leg of bench.py may import or run this module.  It shares no code
with the CUDA library (sub_bit_kv_b200/csrc): no headers, helpers, tables or
constants; neither imports the other.

Everything is numpy float64.  bf16 inputs are widened exactly (every bf16
value is an fp64 value).  Loops follow the definitions on the pages; numpy
broadcasting is used only where it is the definition written out (a sum of
squares, a dot product).

Sources (pages on LoopVQ, "LoopVQ: Sub 1-bit KV Cache Quantization for Looped
Transformers", Cheong and Yoo):
  [summary]  LoopVQ summary page (onedev.kr), sections "how it differs"
             (loop-axis joint vector, nearest entry, per-step share, pre-RoPE
             keys), "premises and limits" (8-token pages, bf16 sink and recent
             tokens, one index row per block, split attention merged with
             logsumexp, prefill/decode encoding).
  [article]  LoopVQ news article (rit.work), section "one code describes
             several loop steps" and "when LoopVQ changes the deployment plan".
  [abstract] LoopVQ abstract page (weekinpapers.com), Abstract.

Readings of points the pages leave open (each restated in the function that
uses it):
  * group g covers the contiguous channels [g*c, (g+1)*c);
  * inside a joint vector, element s*c + e is step s of the block, channel e
    of the group (step-major);
  * distance is unweighted squared L2 on the raw bf16 values; ties go to the
    lowest index;
  * RoPE is rotate-half: channel i pairs with i + d/2, angle pos * base^(-2i/d);
  * scores are scaled by 1/sqrt(d); natural-base softmax; no mask beyond ctx;
  * absolute positions: sink tokens 0..S-1, coded token n at S + n, recent
    tokens after the coded ones; the query is the newest token (position
    ctx - 1) and attends to itself;
  * split j of L coded tokens covers [j*chunk, min(L, (j+1)*chunk)) with
    chunk = ceil(L / n_splits) rounded up to a multiple of 32; the bf16 tokens
    form one more partial.
"""
from __future__ import annotations

import math

import numpy as np

ENTRIES = 256          # 8-bit codes, K = 256 [summary, "premises and limits": experiments]
NEAR_TIE_REL = 1e-6    # relative top-2 gap under which two entries count as tied


def geometry(head_dim: int, T: int, Tc: int, G: int):
    """c = G/Tc channels per step, n_g = d/c groups per step, T/Tc blocks.

    [summary, "how it differs"]: the T loop steps are cut into contiguous
    blocks of Tc steps, Tc must divide both T and G, and one code covers
    c = G/Tc channels of each of the block's Tc steps.
    """
    if Tc <= 0 or T % Tc or G % Tc:
        raise ValueError("Tc must divide T and G")
    c = G // Tc
    if head_dim % c:
        raise ValueError("c = G/Tc must divide head_dim")
    return c, head_dim // c, T // Tc


def bits_per_element(head_dim: int, T: int, Tc: int, G: int, code_bits: int = 8) -> float:
    """Code bits per cached element: one code per (block, group) over Tc*d channels-steps.

    [summary, "how it differs"]: the shared index keeps the cost at b/G bits
    per element.  Counted here from the layout, not from the formula: a token
    of one head stores n_blk * n_g codes for its T * d elements.
    """
    c, n_g, n_blk = geometry(head_dim, T, Tc, G)
    return code_bits * n_blk * n_g / (T * head_dim)


def joint_vectors(x: np.ndarray, Tc: int, G: int) -> np.ndarray:
    """Loop-axis joint vectors of one of K or V.

    x: [T][N][H][d] (pre-RoPE for keys).  Returns X: [n_blk][N][H][n_g][G] with
    X[b][n][h][g][s*c + e] = x[b*Tc + s][n][h][g*c + e].

    [summary, "how it differs"]: one code covers c channels of each of the Tc
    steps of a block; [article, "one code describes several loop steps"]:
    channels of several consecutive steps are gathered into one vector.
    """
    T, N, H, d = x.shape
    c, n_g, n_blk = geometry(d, T, Tc, G)
    X = np.empty((n_blk, N, H, n_g, G), dtype=np.float64)
    for b in range(n_blk):
        for s in range(Tc):
            step = b * Tc + s
            for g in range(n_g):
                X[b, :, :, g, s * c:(s + 1) * c] = x[step, :, :, g * c:(g + 1) * c]
    return X


def nearest_entry(X: np.ndarray, C: np.ndarray, chunk: int = 4096):
    """Brute-force nearest codebook entry in fp64.

    X: [M][G], C: [256][G].  Returns (idx [M] int64, d1 [M], d2 [M]) where
    d_k = sum_j (X_j - C_kj)^2, idx is the smallest k attaining min_k d_k, d1 is
    that minimum and d2 the second-smallest d_k (equal to d1 when the minimum
    is attained twice).

    [summary, "how it differs"]: the joint vector is encoded as its single
    nearest codebook entry.  Ties go to the lowest index (the argmin below
    returns the first minimum).
    """
    M = X.shape[0]
    idx = np.empty(M, dtype=np.int64)
    d1 = np.empty(M, dtype=np.float64)
    d2 = np.empty(M, dtype=np.float64)
    for m0 in range(0, M, chunk):
        xs = X[m0:m0 + chunk]
        D = ((xs[:, None, :] - C[None, :, :]) ** 2).sum(axis=2)
        k = D.argmin(axis=1)
        idx[m0:m0 + chunk] = k
        d1[m0:m0 + chunk] = D[np.arange(xs.shape[0]), k]
        d2[m0:m0 + chunk] = np.partition(D, 1, axis=1)[:, 1]
    return idx, d1, d2


def near_tie(d1: np.ndarray, d2: np.ndarray) -> np.ndarray:
    """True where the top-2 gap is within 1e-6 relative (d1 = 0: only an exact duplicate)."""
    return (d2 - d1) <= NEAR_TIE_REL * d1


def encode(x: np.ndarray, cb: np.ndarray, Tc: int, G: int):
    """Encode one of K or V of one layer.

    x: [T][N][H][d]; cb: [n_blk][H][n_g][256][G] (one codebook per block,
    head and group).  Returns (codes [n_blk][N][H][n_g] uint8, d1, d2 of the
    same shape).

    [summary, "premises and limits"]: encoding needs all Tc steps of a block,
    and a quantized page stores one index row per block.  One codebook set per
    block is this oracle's reading for Tc < T (the pages give "model-specific
    codebooks" only).
    """
    T, N, H, d = x.shape
    c, n_g, n_blk = geometry(d, T, Tc, G)
    X = joint_vectors(x, Tc, G)
    codes = np.empty((n_blk, N, H, n_g), dtype=np.uint8)
    d1 = np.empty((n_blk, N, H, n_g))
    d2 = np.empty((n_blk, N, H, n_g))
    for b in range(n_blk):
        for h in range(H):
            for g in range(n_g):
                k, a1, a2 = nearest_entry(X[b, :, h, g, :], cb[b, h, g])
                codes[b, :, h, g] = k.astype(np.uint8)
                d1[b, :, h, g] = a1
                d2[b, :, h, g] = a2
    return codes, d1, d2


def dequant_step(codes: np.ndarray, cb: np.ndarray, t: int, Tc: int, G: int) -> np.ndarray:
    """Step-t reconstruction from codes.

    codes: [n_blk][N][H][n_g]; cb: [n_blk][H][n_g][256][G].  Returns
    [N][H][d] with x_hat[n][h][g*c + e] = cb[b][h][g][codes[b][n][h][g]][s*c + e],
    b = t // Tc, s = t % Tc.

    [summary, "how it differs"]: each loop step restores only its own share of
    the entry; [summary, "premises and limits"]: the attention reads only the
    step-t slice of the codebook.
    """
    n_blk, N, H, n_g = codes.shape
    c = G // Tc
    b, s = t // Tc, t % Tc
    out = np.empty((N, H, n_g * c), dtype=np.float64)
    for h in range(H):
        for g in range(n_g):
            entries = cb[b, h, g][codes[b, :, h, g].astype(np.int64)]     # [N][G]
            out[:, h, g * c:(g + 1) * c] = entries[:, s * c:(s + 1) * c]
    return out


def rope(x: np.ndarray, pos, base: float = 10000.0) -> np.ndarray:
    """Rotate-half rotary embedding in fp64.

    x: [..., d]; pos broadcastable to x.shape[:-1].  For i < d/2 the pair
    (x_i, x_{i+d/2}) is rotated by angle pos * base^(-2i/d):
      y_i       = x_i cos - x_{i+d/2} sin
      y_{i+d/2} = x_{i+d/2} cos + x_i sin

    [summary, "how it differs"]: keys are quantized before RoPE and RoPE is
    applied to the reconstructed keys inside attention.  The pairing and the
    base are this oracle's reading (the pages name neither).
    """
    d = x.shape[-1]
    half = d // 2
    i = np.arange(half, dtype=np.float64)
    theta = np.power(float(base), -2.0 * i / d)
    phi = np.asarray(pos, dtype=np.float64)[..., None] * theta
    cos, sin = np.cos(phi), np.sin(phi)
    lo, hi = x[..., :half], x[..., half:]
    return np.concatenate([lo * cos - hi * sin, hi * cos + lo * sin], axis=-1)


def softmax_attention(q_rot: np.ndarray, k_rot: np.ndarray, v: np.ndarray):
    """One query over n keys: s_n = q.k_n / sqrt(d), p = softmax(s), out = sum p_n v_n.

    Returns (out [d], lse) with lse = ln sum_n exp(s_n), computed max-shifted.
    With no keys, out is all zeros and lse = -inf.
    """
    n, d = k_rot.shape
    if n == 0:
        return np.zeros(v.shape[1]), -math.inf
    s = k_rot @ q_rot / math.sqrt(d)
    m = s.max()
    e = np.exp(s - m)
    z = e.sum()
    return (e @ v) / z, m + math.log(z)


def split_ranges(L: int, n_splits: int):
    """Split j covers [j*chunk, min(L, (j+1)*chunk)), chunk = ceil(L/n_splits) up to a multiple of 32.

    [summary, "premises and limits"]: quantized tokens are split as in
    Flash-Decoding and merged by logsumexp.  The chunk rule is this oracle's
    reading; splits past the end are empty.
    """
    chunk = -(-L // n_splits) if L > 0 else 0
    chunk = -(-chunk // 32) * 32
    out = []
    for j in range(n_splits):
        a = min(L, j * chunk)
        out.append((a, min(L, a + chunk) if chunk else a))
    return out


def lse_merge(partials):
    """Merge (out_j, lse_j) partials: LSE = ln sum_j e^{lse_j}, out = sum_j e^{lse_j - LSE} out_j."""
    lses = np.array([p[1] for p in partials], dtype=np.float64)
    if np.all(np.isneginf(lses)):
        return np.zeros_like(partials[0][0]), -math.inf
    m = lses.max()
    w = np.exp(lses - m)
    tot = w.sum()
    out = sum(wj * p[0] for wj, p in zip(w, partials) if wj > 0) / tot
    return out, m + math.log(tot)


def decode_attention(q, t, Tc, G, sink_k, sink_v, codes_k, codes_v, cb_k, cb_v,
                     ring_k, ring_v, base=10000.0, n_splits=None):
    """Decode attention of one query head at loop step t over a coded cache.

    q: [d] pre-RoPE query (its position is the newest one, ctx - 1).
    sink_k/sink_v: [S][d] step-t bf16 sink tokens at positions 0..S-1.
    codes_k/codes_v: [n_blk][L][n_g] codes of the L coded tokens (positions
      S..S+L-1) of this head; cb_k/cb_v: [n_blk][n_g][256][G] its codebooks.
    ring_k/ring_v: [R][d] step-t bf16 recent tokens at positions S+L..S+L+R-1.

    Returns (out [d], lse, split_lse) where out/lse are the unsplit softmax
    attention over all S + L + R tokens and, when n_splits is given,
    split_lse[j] is the LSE over coded split j (split_ranges) and
    split_lse[n_splits] the LSE over the bf16 tokens.

    [summary, "premises and limits"]: the first (sink) and the recent tokens
    stay bf16, the rest are code indices; the attention kernel reads only the
    step-t codebook slice, splits the quantized tokens Flash-Decoding style and
    merges with logsumexp.  [article, "when LoopVQ changes the deployment
    plan"]: keys and values are restored from the tables and combined with the
    uncompressed part.  Split-and-merge reaches the unsplit result exactly (up
    to rounding), so the unsplit softmax is the definition computed here.
    """
    d = q.shape[0]
    S = sink_k.shape[0]
    L = codes_k.shape[1]
    R = ring_k.shape[0]
    ctx = S + L + R
    q_rot = rope(q[None, :], np.array([ctx - 1]), base)[0]

    k_hat = dequant_step(codes_k[:, :, None, :], cb_k[:, None], t, Tc, G)[:, 0, :]
    v_hat = dequant_step(codes_v[:, :, None, :], cb_v[:, None], t, Tc, G)[:, 0, :]
    pos_sink = np.arange(S)
    pos_coded = S + np.arange(L)
    pos_ring = S + L + np.arange(R)

    keys = np.concatenate([rope(sink_k, pos_sink, base), rope(k_hat, pos_coded, base),
                           rope(ring_k, pos_ring, base)], axis=0)
    vals = np.concatenate([sink_v, v_hat, ring_v], axis=0)
    out, lse = softmax_attention(q_rot, keys, vals)
    if n_splits is None:
        return out, lse, None

    split_lse = []
    for (a, b) in split_ranges(L, n_splits):
        _, l_j = softmax_attention(q_rot, rope(k_hat[a:b], pos_coded[a:b], base), v_hat[a:b])
        split_lse.append(l_j)
    bf_k = np.concatenate([rope(sink_k, pos_sink, base), rope(ring_k, pos_ring, base)], axis=0)
    bf_v = np.concatenate([sink_v, ring_v], axis=0)
    split_lse.append(softmax_attention(q_rot, bf_k, bf_v)[1])
    return out, lse, np.array(split_lse)


def page_encode(recent_k: np.ndarray, recent_v: np.ndarray, cb_k: np.ndarray, cb_v: np.ndarray,
                Tc: int, G: int, page: int = 8):
    """Encode the oldest page of the recent window.

    recent_k/recent_v: [T][R][H][d] recent tokens of one layer, oldest first
    (R >= page).  Returns (codes_k, codes_v), each [n_blk][page][H][n_g].

    [summary, "premises and limits"]: during decoding new tokens are written
    to the recent window and every 8 tokens the oldest page is quantized across
    all layers and loop steps.  The codes are those prefill would give the same
    tokens: the same nearest-entry encoding.
    """
    ck, _, _ = encode(recent_k[:, :page], cb_k, Tc, G)
    cv, _, _ = encode(recent_v[:, :page], cb_v, Tc, G)
    return ck, cv


# ------------------------------------------------------------------ codebook construction

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), returned as fp64.

    bf16 keeps 8 significant bits and fp32's exponent range (normal values from
    2^-126, subnormal steps of 2^-133).  The rounding is done once, from fp64,
    by scaling each value so that one bf16 step is 1 and rounding to the
    nearest integer with ties to even (numpy's rint); values past the largest
    finite bf16 become infinite.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    _, e = np.frexp(x[nz])                       # |x| = m * 2^e, m in [0.5, 1)
    step_exp = np.maximum(e - 8, -133)           # exponent of one bf16 step at |x|
    r = np.rint(np.ldexp(x[nz], -step_exp))      # ties to even
    out[nz] = np.ldexp(r, step_exp)
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    big = np.abs(out) > np.ldexp(255.0, 120)     # largest finite bf16 = (2 - 2^-7) * 2^127
    out[big] = np.sign(out[big]) * np.inf
    return out


def kmeans_update(X: np.ndarray, codes: np.ndarray, C: np.ndarray):
    """Update step of one plain k-means (Lloyd) iteration.

    X: [M][G] joint vectors, codes: [M] their nearest entries, C: [256][G] the
    current entries.  Returns (C_new [256][G] fp64, counts [256]): entry k moves
    to the mean of the vectors coded k; an entry no vector chose keeps its value.

    [summary, "how it differs"]: codebooks are initialised by k-means over joint
    vectors (Fisher-weighted there; the weights need a model's gradients, so this
    is the unweighted form).  [summary, "premises and limits"]: k-means over the
    calibration tokens is the first calibration stage.  The pages leave empty
    entries open; keeping them is the plainest reading.
    """
    C_new = np.array(C, dtype=np.float64, copy=True)
    counts = np.zeros(C.shape[0], dtype=np.int64)
    for k in range(C.shape[0]):
        members = X[codes == k]
        counts[k] = members.shape[0]
        if counts[k] > 0:
            C_new[k] = members.sum(axis=0) / counts[k]
    return C_new, counts


def kmeans_step(X: np.ndarray, C: np.ndarray):
    """One Lloyd iteration with bf16 entries: assignment by nearest entry (lowest
    index on ties), then the update step, the new entries rounded to bf16 as the
    codebooks are stored.  Returns (codes, C_new, counts)."""
    codes, _, _ = nearest_entry(X, C)
    C_new, counts = kmeans_update(X, codes, C)
    return codes, round_bf16(C_new), counts
