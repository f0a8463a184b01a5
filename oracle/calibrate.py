"""WUSH / WUS / Hadamard / identity block transforms from second moments (oracle).

Cites:
  * WUSH news article, paragraph 3: WUSH is built from the Cholesky factor of the
    weights (W), the SVD components (U, S) and a Hadamard matrix (H), from the
    second-order statistics of weights and activations; it is non-orthogonal and
    block-diagonal.
  * WUSH news article, paragraph 6 (deployment workflow): collect the second
    moments of weights and activations from calibration data, compute the
    transforms (Cholesky and SVD, in parallel over blocks), apply the transform
    to the input activations at inference.
  * WUSH news article, paragraph 5: WUS (no Hadamard component) is evaluated
    beside WUSH on NVFP4.
  * AI Radio episode, "The gist": a Hadamard backbone combined with a
    data-dependent second-moment component, non-orthogonal.
  * AI Radio episode, "Problem Setup and Goal": T_W and T_X are chosen so that
    q(T_W W)^T q(T_X X) approximates W^T X.

Reading (the pages print no formula). Per d_in block j of width b:
    Sigma_X = X_j X_j^T / n_calib,   Sigma_W = W_j W_j^T / d_out     (b x b)
    W' = lower Cholesky factor of Sigma_W
    W'^T Sigma_X W' = U diag(lambda) U^T,  S = diag(sqrt(lambda))
        (this is the SVD of W'^T X_j / sqrt(n) without forming it)
    T_X = Hn S^(-1/2) U^T W'^T,     T_W = T_X^(-T) = Hn S^(1/2) U^T W'^(-1)
with Hn = H_b / sqrt(b).  WUS drops Hn; "hadamard" is T_X = T_W = Hn; "identity"
is I.  The factors are listed in the order in which they act on x (W, U, S, H),
T_W^T T_X = I so the product is lossless before rounding, and the transformed
moments balance: T_X Sigma_X T_X^T = T_W Sigma_W T_W^T = Hn S Hn^T.

Conventions the pages leave open: eigenvalues in descending order; each column
of U is negated if needed so that its largest-magnitude entry is positive (ties
to the lowest index); eigenvalues are floored at 1e-12 * max(lambda); a failed
Cholesky is retried once on Sigma_W + 1e-8 * mean(diag(Sigma_W)) I.

"wush_diag" is the simplification the WUSH news article offers for costly or
constrained deployments (paragraphs 6 and 8: approximate the data-aware component
by a diagonal matrix).  Reading: the same construction run on the diagonals of
the two moments.  Then W' = diag(sqrt(sigma_w)), W'^T Sigma_X W' is diagonal, U
is the identity (no reordering), and
    T_X = Hn D,   T_W = Hn D^(-1),   D = diag((sigma_w,k / sigma_x,k)^(1/4)),
so T_W^T T_X = I still holds and the diagonal moments balance:
T_X diag(Sigma_X) T_X^T = T_W diag(Sigma_W) T_W^T = Hn diag(sqrt(sigma_x sigma_w)) Hn^T.
Each diagonal is floored at 1e-12 times its largest entry (1 if all are zero).
"""
from __future__ import annotations

import numpy as np

from ._checks import require_finite
from .transforms import normalized_hadamard

KINDS = ("identity", "hadamard", "wus", "wush", "wush_diag")


class NotPositiveDefinite(ValueError):
    pass


def block_moments(x_rows: np.ndarray, b: int) -> np.ndarray:
    """Per-block second moments (1/rows) sum_r x_j x_j^T, as [d_in/b, b, b] fp64.

    x_rows: [rows, d_in] -- calibration tokens of X, or the d_out rows of W^T.
    """
    require_finite("block_moments", x_rows)
    x = np.asarray(x_rows, dtype=np.float64)
    rows, d_in = x.shape
    xb = x.reshape(rows, d_in // b, b)
    return np.einsum("rjk,rjl->jkl", xb, xb) / rows


def _cholesky(sigma_w: np.ndarray) -> np.ndarray:
    try:
        return np.linalg.cholesky(sigma_w)
    except np.linalg.LinAlgError:
        jitter = 1e-8 * np.mean(np.diag(sigma_w))
        try:
            return np.linalg.cholesky(sigma_w + jitter * np.eye(len(sigma_w)))
        except np.linalg.LinAlgError as e:
            raise NotPositiveDefinite(str(e)) from e


def _sorted_eig(m: np.ndarray):
    """Eigenpairs of a symmetric matrix, descending, with the sign convention above."""
    lam, u = np.linalg.eigh(m)
    order = np.argsort(-lam, kind="stable")
    lam = lam[order]
    u = u[:, order].copy()
    for c in range(u.shape[1]):
        i = int(np.argmax(np.abs(u[:, c])))     # first index of the max magnitude
        if u[i, c] < 0:
            u[:, c] = -u[:, c]
    lam = np.maximum(lam, 1e-12 * max(lam[0], 0.0))
    return lam, u


def _floored_diag(sigma: np.ndarray) -> np.ndarray:
    """Diagonal of a second moment, floored at 1e-12 of its largest entry."""
    d = np.diag(np.asarray(sigma, dtype=np.float64)).copy()
    top = d.max() if d.max() > 0 else 1.0
    return np.maximum(d, 1e-12 * top)


def block_transform_pair(sigma_x: np.ndarray, sigma_w: np.ndarray, kind: str):
    """(T_X, T_W) for one b x b block from its two second moments, fp64."""
    b = sigma_x.shape[0]
    if kind == "identity":
        return np.eye(b), np.eye(b)
    hn = normalized_hadamard(b)
    if kind == "hadamard":
        return hn.copy(), hn.copy()
    if kind == "wush_diag":
        d = (_floored_diag(sigma_w) / _floored_diag(sigma_x)) ** 0.25
        return hn @ np.diag(d), hn @ np.diag(1.0 / d)
    if kind not in ("wus", "wush"):
        raise ValueError(kind)
    wp = _cholesky(sigma_w)
    m = wp.T @ sigma_x @ wp
    lam, u = _sorted_eig(m)
    s = np.sqrt(lam)
    left = hn if kind == "wush" else np.eye(b)
    t_x = left @ np.diag(s ** -0.5) @ u.T @ wp.T
    t_w = left @ np.diag(s ** 0.5) @ u.T @ np.linalg.inv(wp)
    return t_x, t_w


def transforms_from_moments(sigma_x: np.ndarray, sigma_w: np.ndarray, kind: str):
    """(T_X, T_W) as [d_in/b, b, b] fp64 from per-block moments [d_in/b, b, b]."""
    require_finite("transforms_from_moments", sigma_x, sigma_w)
    pairs = [block_transform_pair(sx, sw, kind) for sx, sw in zip(sigma_x, sigma_w)]
    return np.stack([p[0] for p in pairs]), np.stack([p[1] for p in pairs])


def calibrate(x_calib: np.ndarray, w_rows: np.ndarray, b: int, kind: str):
    """(T_X, T_W) fp64 [d_in/b, b, b] from calibration tokens [n, d_in] and W^T [d_out, d_in]."""
    return transforms_from_moments(block_moments(x_calib, b), block_moments(w_rows, b), kind)


def nvfp4_global_scale(y_rows: np.ndarray) -> np.float32:
    """Per-tensor NVFP4 scale s_g = amax / (6 * 448), returned as fp32.

    Reading: the pages name NVFP4 only; the per-tensor fp32 scale is chosen so
    that the largest calibration value maps to the largest E2M1 magnitude (6)
    times the largest UE4M3 block scale (448).  For activations it is taken once
    from the transformed calibration tokens (static), for weights from the
    transformed weight tensor itself.
    """
    require_finite("nvfp4_global_scale", y_rows)
    amax = float(np.max(np.abs(np.asarray(y_rows, dtype=np.float64))))
    return np.float32(amax / (6.0 * 448.0))


def nvfp4_dynamic_global_scale(y_rows: np.ndarray) -> np.float32:
    """Per-batch NVFP4 scale: s_g = fp32(amax / 2688) of the transformed tensor being
    quantised, or 1 when that is below 1e-30 (all-zero input: every code is 0).

    Reading: the pages name NVFP4 without its scale rule; the static calibrated
    scale (nvfp4_global_scale on calibration tokens) is the default, and this is
    the per-batch variant of the same rule.  amax is the exact maximum of the
    fp32 values and the quotient is rounded once to fp32.
    """
    require_finite("nvfp4_dynamic_global_scale", y_rows)
    amax = np.float32(np.max(np.abs(np.asarray(y_rows, dtype=np.float32)))) if np.size(y_rows) else np.float32(0)
    g = np.float32(np.float64(amax) / 2688.0)
    return g if g >= np.float32(1e-30) else np.float32(1.0)


def group_blocks(sigma_x: np.ndarray, sigma_w: np.ndarray, groups: int, iters: int = 50) -> np.ndarray:
    """Block -> group index [nb] for transform sharing (WUSH news article,
    paragraph 6: share transform matrices between similar blocks).

    Reading (the pages give no algorithm): blocks are similar when their second
    moments have a similar shape.  Each block's feature is its two moments
    divided by their traces, flattened; k-means (Lloyd) groups the features with
    centres started at blocks round(i * nb / groups), squared Euclidean distance,
    ties to the lowest group, empty groups keeping their centre, until no block
    changes group (at most ``iters`` rounds).
    """
    require_finite("group_blocks", sigma_x, sigma_w)
    nb = sigma_x.shape[0]
    if not 1 <= groups <= nb:
        raise ValueError(groups)

    def unit(s):
        tr = np.trace(s, axis1=1, axis2=2)[:, None, None]
        return s / np.where(tr > 0, tr, 1.0)

    feat = np.concatenate([unit(sigma_x).reshape(nb, -1), unit(sigma_w).reshape(nb, -1)], axis=1)
    centres = feat[[int(round(i * nb / groups)) for i in range(groups)]].copy()
    assign = np.full(nb, -1)
    for _ in range(iters):
        d = ((feat[:, None, :] - centres[None, :, :]) ** 2).sum(axis=2)
        new = np.argmin(d, axis=1)                     # first minimum: ties to the lowest group
        if np.array_equal(new, assign):
            break
        assign = new
        for g in range(groups):
            members = assign == g
            if members.any():
                centres[g] = feat[members].mean(axis=0)
    return assign


def shared_transforms(sigma_x: np.ndarray, sigma_w: np.ndarray, kind: str, groups: int):
    """(T_X [groups, b, b], T_W [groups, b, b], index [nb]) with one transform per
    group of similar blocks, computed from the group's mean moments."""
    require_finite("shared_transforms", sigma_x, sigma_w)
    index = group_blocks(sigma_x, sigma_w, groups)
    nb = sigma_x.shape[0]
    start = [int(round(g * nb / groups)) for g in range(groups)]
    # a group left empty (its start tied with an earlier group's) maps no block; its
    # transform comes from its starting block's moments
    sx = np.stack([sigma_x[index == g].mean(axis=0) if (index == g).any() else sigma_x[start[g]]
                   for g in range(groups)])
    sw = np.stack([sigma_w[index == g].mean(axis=0) if (index == g).any() else sigma_w[start[g]]
                   for g in range(groups)])
    tx, tw = transforms_from_moments(sx, sw, kind)
    return tx, tw, index
