"""Inner-product estimator, decode attention and search over quantized vectors.

[ZX] "两阶段内积量化" and [ADM] QJL paragraph: the 1-bit QJL stage on the residual makes
the inner-product estimate unbiased; [TQN] "集成到 Attention": keys and values are
stored quantized and attention estimates <q, k> with QJL.  The estimator for a key
with stored norms n_hat = fp16(||k||), r_hat = fp16(||r||), indices idx and signs s:

    est(q, k) = n_hat * ( <Pi q, c[idx]> + sqrt(pi/2)/m * r_hat * <S q, 2 s - 1> )

Reading: sqrt(pi/2)/m is the unbiasing constant, since for sigma ~ N(0, I_d)
E[ sign(<sigma, r>) <sigma, q> ] = sqrt(2/pi) <r, q> / ||r||.
"""
from __future__ import annotations

import math

import numpy as np

from .params import MODE_PROD


def prepare_query(params: dict, q: np.ndarray):
    """Rotate the queries once: (Pi q, S q) for rows of q [nq, d]."""
    q = np.asarray(q, dtype=np.float64)
    return q @ params["Pi"].T, q @ params["S"].T


def estimate_inner_products(params: dict, q: np.ndarray, code: dict) -> np.ndarray:
    """est(q_a, k_b) for all query rows a and stored keys b -> [nq, n] float64.

    ``code`` holds idx [n,d], norm [n] and, in prod mode, signs [n,m] and rnorm [n].
    In MSE mode only the first (MSE) term is present.
    """
    qt, qs = prepare_query(params, q)
    c = params["centroids"]
    mse = qt @ c[np.asarray(code["idx"])].T                      # <Pi q, c[idx]>
    est = mse
    if params["mode"] == MODE_PROD:
        m = params["m"]
        pm = 2.0 * np.asarray(code["signs"], dtype=np.float64) - 1.0
        qjl = qs @ pm.T                                          # <S q, 2 s - 1>
        est = mse + math.sqrt(math.pi / 2.0) / m * np.asarray(code["rnorm"])[None, :] * qjl
    return np.asarray(code["norm"], dtype=np.float64)[None, :] * est


def decode_attention(kparams, vparams, group_off, q, kcodes, vcodes, seq_lens, scale, channel_perm=None):
    """One decode step of attention over a quantized KV cache.

    [TQN] "集成到 Attention": k_quant / v_quant replace the cache; logits come from the
    QJL estimator, values from the MSE dequantization ("Quant / DeQuant 函数").
    Shapes: q [B, Hq, D]; kcodes[g] / vcodes[g] are dicts of arrays indexed
    [B, Hkv, T, ...] for channel group g covering channels group_off[g]..group_off[g+1].
    Query head h reads kv head h // (Hq // Hkv).  For each (b, h):
      l_t = scale * sum_g est_g(q[b,h,group g], k_{b, h_kv, t, g})      t < seq_lens[b]
      p   = softmax(l)   (float64, max subtracted)
      o   = sum_t p_t * v_hat_t,  v_hat_t[group g] = n_hat_v Pi_v^T c_v[idx_v]
    Reading: the pages do not state the softmax scale; it is an argument (1/sqrt(D)
    for standard attention).  Returns o [B, Hq, D] float64.

    channel_perm ([Hkv, D] permutations, or None for the identity): group g of kv head
    h_kv covers channels channel_perm[h_kv][group_off[g]:group_off[g+1]] instead of the
    contiguous range ([ZX] "KV缓存量化的质量表现": 2.5 / 3.5 bits per channel as two groups;
    reading: which channels get the higher bit width is the caller's choice, e.g. the
    outlier channels).
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    G = len(kparams)
    Hkv = kcodes[0]["idx"].shape[1]
    rep = Hq // Hkv
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        T = int(seq_lens[b])
        if T == 0:
            continue
        for hk in range(Hkv):
            heads = list(range(hk * rep, (hk + 1) * rep))
            logits = np.zeros((rep, T))
            vhat = np.zeros((T, D))
            perm = np.arange(D) if channel_perm is None else np.asarray(channel_perm[hk])
            for g in range(G):
                ch = perm[group_off[g]:group_off[g + 1]]          # this group's channels
                kc = {key: (None if val is None else val[b, hk, :T]) for key, val in kcodes[g].items()}
                logits += estimate_inner_products(kparams[g], q[b][np.ix_(heads, ch)], kc)
                vc = vcodes[g]
                vhat[:, ch] = (np.asarray(vc["norm"][b, hk, :T], dtype=np.float64)[:, None]
                               * (vparams[g]["centroids"][vc["idx"][b, hk, :T]] @ vparams[g]["Pi"]))
            logits *= scale
            logits -= logits.max(axis=1, keepdims=True)
            p = np.exp(logits)
            p /= p.sum(axis=1, keepdims=True)
            out[b, heads] = p @ vhat
    return out


def search_topk(params: dict, q: np.ndarray, code: dict, k: int):
    """Top-k database entries by estimated inner product ([TQN] "向量搜索中的应用",
    [ADM] vector-search paragraph: rank a quantized database by the estimate).
    Ties keep the lower id first.  Returns (scores [nq,k], ids [nq,k] int64)."""
    est = estimate_inner_products(params, q, code)
    order = np.argsort(-est, axis=1, kind="stable")[:, :k]
    return np.take_along_axis(est, order, axis=1), order.astype(np.int64)


def recall_at(ids: np.ndarray, q: np.ndarray, db: np.ndarray) -> float:
    """1@k recall: fraction of queries whose exact (float64) maximum-inner-product
    neighbour appears among the returned ids ([TQN] "1@k Recall 对比")."""
    exact = np.argmax(np.asarray(q, np.float64) @ np.asarray(db, np.float64).T, axis=1)
    return float(np.mean([exact[i] in ids[i] for i in range(len(exact))]))
