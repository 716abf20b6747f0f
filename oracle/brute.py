"""Pure-Python and numpy restatements used to pin the C oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

* ``brute_paged_decode``: explicit Python loops over sequence, head, token and
  dimension, gathering through the block table one element at a time.  For
  tiny cases only.
* ``contiguous_attention``: textbook softmax(scale * q K^T) V on the
  un-paged, contiguous per-sequence K/V, with numpy matmul and
  ``scipy.special.softmax`` as the library steps.
* ``partition_merge``: the split-context merge of partial softmax results
  (max, exp-sum and normalised partial output per partition), i.e. the
  blocked softmax of "PagedAttention：大模型KV Cache分页管理优化实践" §5.1
  (分块Softmax算法) applied with partitions in place of blocks.
"""
from __future__ import annotations

import math

import numpy as np
import scipy.special


def _f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Bit pattern -> float64 via numpy only (independent of the C decoder)."""
    bits = np.asarray(bits)
    if bits.dtype == np.float16:
        return bits.astype(np.float64)
    bits = bits.astype(np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    # bfloat16 is the upper half of a binary32
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def brute_paged_decode(query, k_cache, v_cache, block_tables, context_lens, scale, dtype):
    """Element-by-element loops.  Returns float64 [S][Hq][D]."""
    q = _f64(query, dtype)
    kc = _f64(k_cache, dtype)
    vc = _f64(v_cache, dtype)
    s_n, hq, d_n = q.shape
    _, bs, hkv, _ = kc.shape
    group = hq // hkv
    out = np.zeros((s_n, hq, d_n))
    for s in range(s_n):
        ctx = int(context_lens[s])
        for h in range(hq):
            g = h // group
            scores = []
            for t in range(ctx):
                blk = int(block_tables[s][t // bs])
                off = t % bs
                acc = 0.0
                for d in range(d_n):
                    acc += q[s, h, d] * kc[blk, off, g, d]
                scores.append(scale * acc)
            if not scores:
                continue
            m = max(scores)
            e = [math.exp(x - m) for x in scores]
            z = sum(e)
            for t in range(ctx):
                blk = int(block_tables[s][t // bs])
                off = t % bs
                w = e[t] / z
                for d in range(d_n):
                    out[s, h, d] += w * vc[blk, off, g, d]
    return out


def contiguous_attention(query, keys, values, context_lens, scale, dtype):
    """Un-paged reference: keys/values are per-sequence lists of [ctx][Hkv][D].

    Returns float64 [S][Hq][D]."""
    q = _f64(query, dtype)
    s_n, hq, d_n = q.shape
    out = np.zeros((s_n, hq, d_n))
    for s in range(s_n):
        ctx = int(context_lens[s])
        if ctx == 0:
            continue
        k = _f64(keys[s][:ctx], dtype)          # [ctx][Hkv][D]
        v = _f64(values[s][:ctx], dtype)
        hkv = k.shape[1]
        group = hq // hkv
        k_rep = np.repeat(k, group, axis=1)     # [ctx][Hq][D], kv head h // group
        v_rep = np.repeat(v, group, axis=1)
        logits = scale * np.einsum("hd,thd->ht", q[s], k_rep)
        w = scipy.special.softmax(logits, axis=1)
        out[s] = np.einsum("ht,thd->hd", w, v_rep)
    return out


def partition_scores(x: np.ndarray, v: np.ndarray, parts: list[tuple[int, int]]):
    """Per partition p over tokens [a, b): (m_p, l_p, Ohat_p) with
    m_p = max x, l_p = sum exp(x - m_p), Ohat_p = sum exp(x - m_p) v / l_p."""
    res = []
    for a, b in parts:
        xs = x[a:b]
        m = xs.max()
        e = np.exp(xs - m)
        l = e.sum()
        res.append((m, l, (e[:, None] * v[a:b]).sum(0) / l))
    return res


def partition_merge(partials):
    """Merge partition results: M = max m_p, w_p = l_p exp(m_p - M),
    out = sum w_p Ohat_p / sum w_p."""
    M = max(m for m, _, _ in partials)
    w = np.array([l * math.exp(m - M) for m, l, _ in partials])
    o = sum(wp * oh for wp, (_, _, oh) in zip(w, partials))
    return o / w.sum()
