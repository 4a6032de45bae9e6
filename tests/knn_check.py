"""Validity of a k-nearest answer under exact distances: the check the GPU
k-nearest tests apply on top of their bit-exact comparison with the oracle's
fp32-decided selection.  The exact distances come from the oracle's knn in
double precision (the plain definition, "Kernel matrix reduction", Overview:
the argmin-type reductions)."""
import numpy as np

import oracle


def knn_valid_under_exact_distances(x, y, od, oi, K):
    """A K-nearest answer decided in fp32, checked against the plain definition
    in double precision (the oracle's knn with exact distances).

    The device computes d = sum_k (x_k - y_k)^2 in fp32 from fp32 inputs: each
    difference is rounded once, each square-and-add (an fma) once, so every
    term carries at most D + 2 roundings and, all terms being non-negative,
    |d_f32 - d| <= gamma_(D+2) d with gamma_n = n u / (1 - n u), u = 2^-24.  Hence:
    every returned fp32 distance lies within that bound of its exact value; and
    if a returned index j were farther than the exact K-th distance a_K, some
    index of an exact K-nearest set was passed over for it, so
    d(j) (1 - gamma) <= d_f32(j) <= d_f32(j') <= a_K (1 + gamma)."""
    x64 = np.asarray(x, dtype=np.float64)
    y64 = np.asarray(y, dtype=np.float64)
    od, oi = np.asarray(od), np.asarray(oi)
    B, M, D = x64.shape
    N = y64.shape[1]
    rd, ri = oracle.knn(x64, y64, K)
    kk = min(K, N)
    assert (oi[..., kk:] == -1).all() and np.isinf(od[..., kk:]).all(), "padding past N"
    idx = oi[..., :kk]
    assert (idx >= 0).all() and (idx < N).all(), "index out of range"
    srt = np.sort(idx, axis=-1)
    assert (np.diff(srt, axis=-1) != 0).all(), "repeated index in a row"
    d32 = od[..., :kk].astype(np.float64)
    # ascending, equal distances by the lower index
    step = np.diff(d32, axis=-1)
    assert (step >= 0).all(), "not ascending"
    assert ((step > 0) | (np.diff(idx, axis=-1) > 0)).all(), "tie not broken by the lower index"
    u = 2.0 ** -24
    gam = (D + 2) * u / (1 - (D + 2) * u)
    dex = np.empty((B, M, kk))
    for b in range(B):
        dex[b] = ((x64[b][:, None, :] - y64[b][idx[b]]) ** 2).sum(-1)
    assert (np.abs(d32 - dex) <= gam * dex).all(), "fp32 distance outside its rounding bound"
    assert (dex.max(-1) <= rd[..., kk - 1] * (1 + gam) / (1 - gam)).all(), "not a K-nearest set"
    # where the exact K-th and (K+1)-th distances are apart by more than the
    # rounding, the returned set is the exact one
    if K < N:
        rd1, _ = oracle.knn(x64, y64, K + 1)
        sep = rd1[..., K] * (1 - gam) > rd1[..., K - 1] * (1 + gam)
        same = (np.sort(idx, -1) == np.sort(ri[..., :kk], -1)).all(-1)
        assert same[sep].all(), "a well-separated K-nearest set differs"
