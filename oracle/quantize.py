"""Quantize / dequantize one batch of vectors (oracle side, float64).

[TQN] "Quant / DeQuant 函数": y = Pi @ x, idx = nearest centroid of each rotated
coordinate; x_hat = Pi.T @ centroids[idx].
[TQN] "PolarQuant：极坐标变换" and [ADM] PolarQuant paragraph: the vector splits into
a radius (its norm, stored once) and a direction (the unit vector that is rotated and
quantized).  Reading: radius = ||x|| stored as fp16, direction u = x / ||x||.
[ADM] two-stage pipeline and [ZX] "两阶段内积量化": the residual of the MSE stage gets a
1-bit QJL sketch sign(S r); [TQN] "残差 norm 存储": ||r|| is one fp16 scalar.
"""
from __future__ import annotations

import numpy as np

from .params import MODE_PROD


def fp16_round(a) -> np.ndarray:
    """Round to IEEE binary16, ties to even (numpy's float16 cast), back to float64."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).astype(np.float64)


def nearest_index(y: np.ndarray, boundaries: np.ndarray) -> np.ndarray:
    """idx = number of decision boundaries strictly below y (Lloyd-Max cells are the
    intervals between consecutive midpoints, so this is the nearest centroid).
    Reading: a value exactly on a boundary goes to the lower index."""
    return np.sum(y[..., None] > boundaries, axis=-1).astype(np.int64)


def quantize(params: dict, x: np.ndarray, idx_override: np.ndarray | None = None) -> dict:
    """Quantize rows of ``x`` ([n, d], any float dtype; computed in float64).

    Steps, per vector:
      n = ||x||,  norm = fp16(n)                         (radius)
      u = x / n  (unrounded n)                           (direction)
      y = Pi u;  idx_i = #{j : y_i > t_j}                (rotate, nearest centroid)
    prod mode only:
      r = u - Pi^T c[idx],  rnorm = fp16(||r||)          (residual, its norm)
      s_j = [ (S r)_j >= 0 ]                             (1-bit QJL; reading: sign(0) = +1)
    A zero vector (n = 0) stores norm = rnorm = 0, idx of y = 0 and all signs 1; its
    contribution to every estimate is then 0.

    ``idx_override`` (tests only) replaces the nearest-centroid indices, so the residual
    and sign stages can be re-run with another implementation's indices for the
    coordinates that sit on a decision boundary.
    Returns dict(idx [n,d] int64, signs [n,m] uint8 or None, norm [n], rnorm [n] or None,
    y [n,d] float64, proj [n,m] float64 or None) -- norms rounded to fp16 -- plus the
    unrounded norm_exact / rnorm_exact.
    """
    x = np.asarray(x, dtype=np.float64)
    Pi, c, t = params["Pi"], params["centroids"], params["boundaries"]
    n = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(n > 0.0, n, 1.0)
    u = x / safe[:, None]
    u[n == 0.0] = 0.0
    y = u @ Pi.T                       # y = Pi u for every row
    idx = nearest_index(y, t) if idx_override is None else np.asarray(idx_override, dtype=np.int64)
    out = dict(idx=idx, norm=fp16_round(n), norm_exact=n, y=y, signs=None, rnorm=None,
               rnorm_exact=None, proj=None)
    if params["mode"] == MODE_PROD:
        r = u - c[idx] @ Pi            # r = u - Pi^T c[idx]
        rn = np.sqrt(np.sum(r * r, axis=1))
        z = r @ params["S"].T          # z = S r
        signs = (z >= 0.0).astype(np.uint8)
        zero = n == 0.0
        rn[zero] = 0.0
        signs[zero] = 1
        out.update(rnorm=fp16_round(rn), rnorm_exact=rn, signs=signs, proj=z)
    return out


def dequantize(params: dict, idx: np.ndarray, norm: np.ndarray) -> np.ndarray:
    """x_hat = ||x|| * Pi^T c[idx]   ([TQN] "Quant / DeQuant 函数": dequant is the MSE
    reconstruction; the stored fp16 norm restores the radius)."""
    c = params["centroids"]
    return np.asarray(norm, dtype=np.float64)[:, None] * (c[np.asarray(idx)] @ params["Pi"])


def dequantize_qjl(params: dict, idx: np.ndarray, signs: np.ndarray, norm: np.ndarray,
                   rnorm: np.ndarray) -> np.ndarray:
    """QJL-augmented reconstruction of stored keys (prod mode):

        x_hat = n_hat * ( Pi^T c[idx] + sqrt(pi/2)/m * r_hat * S^T (2 s - 1) )

    [ZX] "两阶段内积量化" and [ADM] QJL paragraph give the unbiased estimate only as an
    inner product, est(q, k) = n_hat (<Pi q, c[idx]> + sqrt(pi/2)/m r_hat <S q, 2 s - 1>).
    Reading: the vector form is the one x_hat with <q, x_hat> = est(q, k) for every q
    (est is linear in q, so this x_hat exists and is unique); for consumers that need the
    key itself rather than its dot products."""
    if params["mode"] != MODE_PROD:
        raise ValueError("the QJL reconstruction needs a prod-mode context")
    c = params["centroids"]
    m = params["m"]
    pm = 2.0 * np.asarray(signs, dtype=np.float64) - 1.0
    mse = c[np.asarray(idx)] @ params["Pi"]                      # rows: Pi^T c[idx]
    qjl = (np.sqrt(np.pi / 2.0) / m) * np.asarray(rnorm, dtype=np.float64)[:, None] * (pm @ params["S"])
    return np.asarray(norm, dtype=np.float64)[:, None] * (mse + qjl)
