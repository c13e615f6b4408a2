"""Oracle for decode attention over a dequantized KV cache (float64).

Test infrastructure only (see ``oracle/__init__.py``).

``llama.cpp für Geschwindigkeit und Speicher optimieren``, section
"Flash Attention": flash attention computes attention tile by tile in fast
on-chip memory and is mathematically equivalent to standard attention, not an
approximation.  The split-KV form (partials (m, l, acc) per context slice,
then a combine) therefore reaches exactly the plain definition in exact
arithmetic, and the oracle is that definition:

  s_t = scale * <q_h, k_hat_{g,t}>,  M = max_t s_t,  p_t = exp(s_t - M),
  o_h = sum_t p_t v_hat_{g,t} / sum_t p_t,

for each batch row b and query head h, with g = floor(h / G) the KV head of
h's group, G = n_q / n_kv (consecutive grouping; the pages do not say which
grouping, this is the common one), over all ctx_len cached rows and no mask.
"""

import numpy as np


def decode_attention(q, k_hat, v_hat, scale):
    """Plain decode attention.

    q      float  [B, n_q, D]
    k_hat  float  [B, n_kv, T, D]   dequantized keys (rows 0..T-1 attended)
    v_hat  float  [B, n_kv, T, D]   dequantized values
    Returns float64 [B, n_q, D].
    """
    q = np.asarray(q, dtype=np.float64)
    k_hat = np.asarray(k_hat, dtype=np.float64)
    v_hat = np.asarray(v_hat, dtype=np.float64)
    B, n_q, D = q.shape
    n_kv = k_hat.shape[1]
    if n_q % n_kv:
        raise ValueError("n_q must be a multiple of n_kv")
    G = n_q // n_kv
    out = np.empty((B, n_q, D))
    for b in range(B):
        for h in range(n_q):
            g = h // G
            s = scale * (k_hat[b, g] @ q[b, h])
            p = np.exp(s - s.max())
            out[b, h] = (p @ v_hat[b, g]) / p.sum()
    return out


def softmax_weights(q_row, k_rows, scale):
    """Normalised attention weights of one query row (float64 [T])."""
    s = scale * (np.asarray(k_rows, np.float64) @ np.asarray(q_row, np.float64))
    p = np.exp(s - s.max())
    return p / p.sum()


def partials(q_row, k_rows, v_rows, scale, bounds):
    """Split-KV partials of one query row.

    ``bounds`` = [t_0=0, t_1, ..., t_S=T]; slice s covers rows t_s..t_{s+1}-1.
    Returns lists (m_s, l_s, acc_s) with m_s = max score in the slice,
    l_s = sum exp(s_t - m_s), acc_s = sum exp(s_t - m_s) v_t.
    """
    q_row = np.asarray(q_row, np.float64)
    ms, ls, accs = [], [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        s = scale * (np.asarray(k_rows[a:b], np.float64) @ q_row)
        m = s.max()
        p = np.exp(s - m)
        ms.append(m)
        ls.append(p.sum())
        accs.append(p @ np.asarray(v_rows[a:b], np.float64))
    return ms, ls, accs


def combine(ms, ls, accs):
    """Merge split partials: M = max m_s, w_s = exp(m_s - M),
    o = sum w_s acc_s / sum w_s l_s."""
    M = max(ms)
    w = [np.exp(m - M) for m in ms]
    num = sum(wi * a for wi, a in zip(w, accs))
    den = sum(wi * l for wi, l in zip(w, ls))
    return num / den
