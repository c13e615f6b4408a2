"""Oracle for decode attention over a dequantized KV cache (float64) -- TEST
INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

numpy marshalling around ``oracle/attention.cc``.  "llama.cpp für
Geschwindigkeit und Speicher optimieren", section "Flash Attention": flash
attention is mathematically the same as standard attention, so the split-KV
form reaches exactly the plain definition, which is the oracle:

  s_t = scale * <q_h, k_hat_{g,t}>,  M = max_t s_t,  p_t = exp(s_t - M),
  o_h = sum_t p_t v_hat_{g,t} / sum_t p_t,

for each batch row b and query head h, g = floor(h / G), G = n_q / n_kv, over
all cached rows, no mask.
"""

import numpy as np

from . import _lib


def decode_attention(q, k_hat, v_hat, scale, threads=1):
    """Plain decode attention.

    q      float  [B, n_q, D]
    k_hat  float  [B, n_kv, T, D]   dequantized keys (rows 0..T-1 attended)
    v_hat  float  [B, n_kv, T, D]   dequantized values
    threads  CPU threads over the (b, h) pairs (<= 0: all)
    Returns float64 [B, n_q, D].
    """
    qq = _lib.arr(q, np.float64)
    k = _lib.arr(k_hat, np.float64)
    v = _lib.arr(v_hat, np.float64)
    B, n_q, D = qq.shape
    n_kv, T = k.shape[1], k.shape[2]
    if n_q % n_kv:
        raise ValueError("n_q must be a multiple of n_kv")
    assert k.shape == v.shape == (B, n_kv, T, D)
    out = np.empty((B, n_q, D), np.float64)
    _lib.check(_lib.lib.orc_decode_attention(_lib.ptr(qq), _lib.ptr(k), _lib.ptr(v), B, n_q, n_kv, T, D,
                                             float(scale), _lib.ptr(out), threads), "attention")
    return out


def softmax_weights(q_row, k_rows, scale):
    """Normalised attention weights of one query row (float64 [T])."""
    q = _lib.arr(q_row, np.float64)
    k = _lib.arr(k_rows, np.float64)
    T, D = k.shape
    w = np.empty(T, np.float64)
    _lib.check(_lib.lib.orc_softmax_weights(_lib.ptr(q), _lib.ptr(k), T, D, float(scale), _lib.ptr(w)), "softmax")
    return w


def partials(q_row, k_rows, v_rows, scale, bounds):
    """Split-KV partials of one query row.

    ``bounds`` = [t_0=0, t_1, ..., t_S=T]; slice s covers rows t_s..t_{s+1}-1.
    Returns lists (m_s, l_s, acc_s) with m_s = max score in the slice,
    l_s = sum exp(s_t - m_s), acc_s = sum exp(s_t - m_s) v_t.
    """
    q = _lib.arr(q_row, np.float64)
    k = _lib.arr(k_rows, np.float64)
    v = _lib.arr(v_rows, np.float64)
    D = k.shape[1]
    b = np.asarray(bounds, dtype=np.int64)
    S = len(b) - 1
    m = np.empty(S)
    l = np.empty(S)
    acc = np.empty((S, D))
    _lib.check(_lib.lib.orc_partials(_lib.ptr(q), _lib.ptr(k), _lib.ptr(v), D, float(scale), _lib.ptr(b), S,
                                     _lib.ptr(m), _lib.ptr(l), _lib.ptr(acc)), "partials")
    return list(m), list(l), list(acc)


def combine(ms, ls, accs):
    """Merge split partials: M = max m_s, w_s = exp(m_s - M),
    o = sum w_s acc_s / sum w_s l_s."""
    m = _lib.arr(ms, np.float64)
    l = _lib.arr(ls, np.float64)
    acc = _lib.arr(np.stack([np.asarray(a, np.float64) for a in accs]), np.float64)
    S, D = acc.shape
    out = np.empty(D, np.float64)
    _lib.check(_lib.lib.orc_combine(_lib.ptr(m), _lib.ptr(l), _lib.ptr(acc), S, D, _lib.ptr(out)), "combine")
    return out


def decode_cache(k_type, v_type, k_codes, k_scales, v_codes, v_scales, q_f16, scale, seed=0, proj=None,
                 threads=1):
    """One decode over a stored cache: every row dequantized (its format's
    definition), then the plain attention above.

    k_codes  uint8 [B, n_kv, T, code_bytes(k_type)]; k_scales float16
             [B, n_kv, T, n_scales(k_type)] (the same per-row format the
             formats define); likewise v
    q_f16    float16 [B, n_q, D]
    threads  CPU threads (<= 0: all hardware threads)
    Returns float64 [B, n_q, D].
    """
    kc = _lib.arr(k_codes, np.uint8)
    vc = _lib.arr(v_codes, np.uint8)
    ks = _lib.f16_bits(_lib.arr(k_scales, np.float16))
    vs = _lib.f16_bits(_lib.arr(v_scales, np.float16))
    q = _lib.f16_bits(_lib.arr(q_f16, np.float16))
    B, n_kv, T = kc.shape[:3]
    n_q, D = q.shape[1], q.shape[2]
    p = None if proj is None else _lib.arr(proj, np.float32)
    out = np.empty((B, n_q, D), np.float64)
    _lib.check(_lib.lib.orc_decode_cache(_lib.TYPES[k_type], _lib.TYPES[v_type], B, n_q, n_kv, T, D,
                                         _lib.ptr(kc), _lib.ptr(ks), _lib.ptr(vc), _lib.ptr(vs), seed, _lib.ptr(p),
                                         _lib.ptr(q), float(scale), _lib.ptr(out), threads), "decode over a cache")
    return out


def hardware_threads():
    """Threads the host runs at once (std::thread::hardware_concurrency)."""
    return int(_lib.lib.orc_hardware_threads())
