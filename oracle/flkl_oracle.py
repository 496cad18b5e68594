"""fp64 CPU oracle of the fused linear-head + KL-divergence loss.

TEST INFRASTRUCTURE.  Only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import or run this module; the product path
(the CUDA library and its Python binding) never does, and this module imports
nothing from the product package.

What it computes is the plain definition of the loss on the "Add
FusedLinearKLDivLoss" pull-request page (Liger-Kernel mirror):

* *Summary*: the vocabulary-head projection z = X W^T (+ b) followed by
  KL(Q || P) against an explicit teacher distribution Q, where P is the
  student softmax;
* *Details*, first bullet: reductions "batchmean" / "mean" / "sum" with the
  meaning they have in torch.nn.KLDivLoss, rows dropped through
  ``shift_labels == ignore_index``, a softmax temperature T, and an ``eps``
  clamp so that a zero teacher probability contributes 0;
* *Details*, third bullet: the gradient is the log-softmax backward evaluated
  on the log-probabilities (computed with the loss, "gradient in forward");
* *Details*, fourth bullet: ``reduction="none"`` is refused;
* GRPO frozen-head page, *Summary*: dW and db are produced only when asked for;
  the loss and dX do not change when they are not.

Readings where the pages are silent (each also listed in the design notes):

1. Gradient: d loss / d z_rv = (S_r p_rv - q_rv) / (T D) with S_r = sum_v q_rv,
   the exact log-softmax backward (equal to (p - q)/(T D) when rows of Q sum
   to 1).
2. Divisor D with ignored rows: batchmean -> N_valid, mean -> N_valid * V,
   sum -> 1.  N_valid = 0 gives loss 0 and all-zero gradients.
3. Temperature divides the student logits only; no T^2 factor.
4. eps clamps only inside log q: term = q * (log max(q, eps) - log p), and an
   entry with q == 0 contributes exactly 0 (also when eps == 0).
5. The bias is added before dividing by T.
6. Only equality of a shift label with ignore_index matters.

Also here, each from its own definition (see the function docstrings): the
cross-entropy special case (one-hot teacher), the per-token selective
log-probability and its backward, and the generalized Jensen-Shannon
divergence against a teacher head.  Every function is pinned by tests that
do not restate it (library routines, closed forms, invariants, finite
differences); none is unpinned.

Everything runs in float64 on the exact input values (bf16 inputs are upcast).
Rows are processed in blocks so that no BT x V fp64 array is held; the block
size changes only summation order.
"""

from __future__ import annotations

import numpy as np

REDUCTIONS = ("batchmean", "mean", "sum")


class OracleError(ValueError):
    pass


def _as64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def valid_rows(BT, shift_labels, ignore_index):
    """Row mask: a row is kept unless its shift label equals ignore_index
    (page *Details*, first bullet).  No labels -> every row is kept."""
    if shift_labels is None:
        return np.ones(BT, dtype=bool)
    lab = np.asarray(shift_labels).astype(np.int64)
    return lab != np.int64(ignore_index)


def divisor(reduction, n_valid, V):
    """The reduction divisor D: KLDivLoss semantics restricted to kept rows
    (batchmean: per kept row; mean: per kept element; sum: none)."""
    if reduction not in REDUCTIONS:
        raise OracleError(f"reduction={reduction!r} is not supported "
                          "(the loss must be a scalar for gradient-in-forward)")
    if reduction == "batchmean":
        return float(n_valid)
    if reduction == "mean":
        return float(n_valid) * float(V)
    return 1.0


def log_softmax_rows(u):
    """Row-wise log-softmax, max-shifted: log p = u - (max u + log sum e^(u-max u))."""
    m = u.max(axis=1, keepdims=True)
    lse = m + np.log(np.exp(u - m).sum(axis=1, keepdims=True))
    return u - lse, lse[:, 0]


def kl_terms(q, logp, eps):
    """Per-element q * (log max(q, eps) - log p), with q == 0 giving exactly 0."""
    with np.errstate(divide="ignore", invalid="ignore"):
        t = q * (np.log(np.maximum(q, eps)) - logp)
    return np.where(q == 0.0, 0.0, t)


def forward_backward(X, W, b, Q, shift_labels=None, ignore_index=-100, temperature=1.0,
                     eps=1e-10, reduction="batchmean", compute_dW=True, compute_db=False,
                     dX_rows=None, dW_rows=None, row_block=256):
    """Loss and gradients of the fused linear + KL(Q||P) loss, in float64.

    X [BT,H], W [V,H], b [V] or None, Q [BT,V], shift_labels [BT] or None.
    Returns a dict with ``loss`` (float), ``dX`` ([BT,H], or the rows listed in
    ``dX_rows``), ``dW`` ([V,H] or the rows ``dW_rows``; None when frozen),
    ``db`` ([V]; None unless compute_db), ``row_loss`` [BT] (0 on ignored rows),
    ``lse`` [BT] (of u = z/T), ``n_valid`` and ``D``.
    """
    if reduction not in REDUCTIONS:
        raise OracleError(f"reduction={reduction!r} is not supported "
                          "(the loss must be a scalar for gradient-in-forward)")
    if compute_db and b is None:
        raise OracleError("compute_db needs a bias")
    BT, H = np.shape(X)
    V = np.shape(W)[0]
    T = float(temperature)
    valid = valid_rows(BT, shift_labels, ignore_index)
    n_valid = int(valid.sum())
    D = divisor(reduction, n_valid, V)
    scale = 0.0 if n_valid == 0 else 1.0 / (T * D)

    W64 = _as64(W)
    b64 = _as64(b)
    dx_sel = np.arange(BT) if dX_rows is None else np.asarray(dX_rows, dtype=np.int64)
    dw_sel = None if not compute_dW else (np.arange(V) if dW_rows is None
                                          else np.asarray(dW_rows, dtype=np.int64))
    dX = np.zeros((len(dx_sel), H))
    dW = None if dw_sel is None else np.zeros((len(dw_sel), H))
    db = np.zeros(V) if compute_db else None
    row_loss = np.zeros(BT)
    lse_all = np.zeros(BT)
    dx_pos = {int(r): i for i, r in enumerate(dx_sel)}

    for r0 in range(0, BT, row_block):
        r1 = min(BT, r0 + row_block)
        Xc = _as64(X[r0:r1])
        Qc = _as64(Q[r0:r1])
        z = Xc @ W64.T                                  # projection
        if b64 is not None:
            z += b64                                     # bias before temperature
        u = z / T                                        # temperature
        logp, lse = log_softmax_rows(u)
        lse_all[r0:r1] = lse
        vmask = valid[r0:r1]
        rl = kl_terms(Qc, logp, eps).sum(axis=1)
        row_loss[r0:r1] = np.where(vmask, rl, 0.0)
        S = Qc.sum(axis=1)
        # log-softmax backward on the log-probabilities, chain rule through 1/T
        G = (S[:, None] * np.exp(logp) - Qc) * scale
        G[~vmask] = 0.0
        rows_here = [i for i in range(r0, r1) if i in dx_pos]
        if rows_here:
            idx = np.asarray(rows_here) - r0
            dX[[dx_pos[i] for i in rows_here]] = G[idx] @ W64
        if dW is not None:
            dW += G[:, dw_sel].T @ Xc
        if db is not None:
            db += G.sum(axis=0)

    loss = 0.0 if n_valid == 0 else float(row_loss.sum() / D)
    return dict(loss=loss, dX=dX, dW=dW, db=db, row_loss=row_loss, lse=lse_all,
                n_valid=n_valid, D=D)


def forward_backward_loops(X, W, b, Q, shift_labels=None, ignore_index=-100, temperature=1.0,
                           eps=1e-10, reduction="batchmean", compute_dW=True, compute_db=False):
    """The same quantities with explicit Python loops and the math module, for
    tiny inputs only.  Written element by element from the definition, so it
    shares no vectorised step with ``forward_backward``."""
    import math
    X = [[float(v) for v in row] for row in np.asarray(X, dtype=np.float64)]
    W = [[float(v) for v in row] for row in np.asarray(W, dtype=np.float64)]
    Q = [[float(v) for v in row] for row in np.asarray(Q, dtype=np.float64)]
    bb = None if b is None else [float(v) for v in np.asarray(b, dtype=np.float64)]
    BT, H, V = len(X), len(X[0]), len(W)
    keep = [True] * BT if shift_labels is None else [int(l) != int(ignore_index) for l in shift_labels]
    nv = sum(keep)
    if reduction == "batchmean":
        D = float(nv)
    elif reduction == "mean":
        D = float(nv * V)
    elif reduction == "sum":
        D = 1.0
    else:
        raise OracleError("unsupported reduction")
    total = 0.0
    dX = [[0.0] * H for _ in range(BT)]
    dW = [[0.0] * H for _ in range(V)]
    db = [0.0] * V
    for r in range(BT):
        if not keep[r]:
            continue
        u = []
        for v in range(V):
            acc = 0.0
            for h in range(H):
                acc += X[r][h] * W[v][h]
            if bb is not None:
                acc += bb[v]
            u.append(acc / temperature)
        mx = max(u)
        se = 0.0
        for v in range(V):
            se += math.exp(u[v] - mx)
        lse = mx + math.log(se)
        S = 0.0
        for v in range(V):
            q = Q[r][v]
            S += q
            if q != 0.0:
                total += q * (math.log(max(q, eps)) - (u[v] - lse))
        for v in range(V):
            g = (S * math.exp(u[v] - lse) - Q[r][v]) / (temperature * D)
            db[v] += g
            for h in range(H):
                dX[r][h] += g * W[v][h]
                dW[v][h] += g * X[r][h]
    loss = 0.0 if nv == 0 else total / D
    if nv == 0:
        dX = [[0.0] * H for _ in range(BT)]
        dW = [[0.0] * H for _ in range(V)]
        db = [0.0] * V
    return dict(loss=loss, dX=np.array(dX), dW=np.array(dW) if compute_dW else None,
                db=np.array(db) if compute_db else None)


def ce_forward_backward(X, W, b, target, ignore_index=-100, temperature=1.0,
                        reduction="batchmean", compute_dW=True, compute_db=False,
                        dX_rows=None, dW_rows=None, row_block=256):
    """Fused linear cross-entropy, fp64: the KL loss above with a one-hot
    teacher (the cross-entropy of fused_linear_cross_entropy, named on the
    FusedLinearKLDivLoss page, *Summary*, as the source of its token-chunk
    geometry).  Written from the cross-entropy definition:

        l_r = lse(u_r) - u_{r, y_r},   u = (X W^T + b) / T,
        d loss / d z_rv = (p_rv - [v == y_r]) / (T D),

    on rows whose target differs from ignore_index (the target doubles as the
    row mask); D follows the same reductions as the KL loss (batchmean:
    N_valid, mean: N_valid * V, sum: 1).  A target outside [0, V) that is not
    ignore_index makes its row contribute nothing (no teacher mass).
    """
    if reduction not in REDUCTIONS:
        raise OracleError(f"reduction={reduction!r} is not supported")
    if compute_db and b is None:
        raise OracleError("compute_db needs a bias")
    BT, H = np.shape(X)
    V = np.shape(W)[0]
    T = float(temperature)
    tgt = np.asarray(target).astype(np.int64)
    valid = tgt != np.int64(ignore_index)
    n_valid = int(valid.sum())
    D = divisor(reduction, n_valid, V)
    scale = 0.0 if n_valid == 0 else 1.0 / (T * D)
    W64 = _as64(W)
    b64 = _as64(b)
    dx_sel = np.arange(BT) if dX_rows is None else np.asarray(dX_rows, dtype=np.int64)
    dw_sel = None if not compute_dW else (np.arange(V) if dW_rows is None
                                          else np.asarray(dW_rows, dtype=np.int64))
    dX = np.zeros((len(dx_sel), H))
    dW = None if dw_sel is None else np.zeros((len(dw_sel), H))
    db = np.zeros(V) if compute_db else None
    row_loss = np.zeros(BT)
    dx_pos = {int(r): i for i, r in enumerate(dx_sel)}
    for r0 in range(0, BT, row_block):
        r1 = min(BT, r0 + row_block)
        Xc = _as64(X[r0:r1])
        z = Xc @ W64.T
        if b64 is not None:
            z += b64
        u = z / T
        logp, lse = log_softmax_rows(u)
        y = tgt[r0:r1]
        inside = valid[r0:r1] & (y >= 0) & (y < V)
        rows = np.arange(r1 - r0)
        ycl = np.clip(y, 0, V - 1)
        rl = np.where(inside, -logp[rows, ycl], 0.0)
        row_loss[r0:r1] = rl
        G = np.exp(logp)
        G[rows[inside], ycl[inside]] -= 1.0
        G[~inside] = 0.0
        G *= scale
        here = [i for i in range(r0, r1) if i in dx_pos]
        if here:
            dX[[dx_pos[i] for i in here]] = G[np.asarray(here) - r0] @ W64
        if dW is not None:
            dW += G[:, dw_sel].T @ Xc
        if db is not None:
            db += G.sum(axis=0)
    loss = 0.0 if n_valid == 0 else float(row_loss.sum() / D)
    return dict(loss=loss, dX=dX, dW=dW, db=db, row_loss=row_loss, n_valid=n_valid, D=D)


def selective_logprob(X, W, b, target, ignore_index=-100, temperature=1.0, row_block=256):
    """Per-row log-probability of the target, fp64 (the chunked selective
    log-probability of the GRPO frozen-head page, *Summary*):

        logp_r = u_{r, y_r} - lse(u_r),   u = (X W^T + b) / T,

    0 on rows whose target is ignore_index or outside [0, V)."""
    BT = np.shape(X)[0]
    V = np.shape(W)[0]
    T = float(temperature)
    tgt = np.asarray(target).astype(np.int64)
    W64 = _as64(W)
    b64 = _as64(b)
    out = np.zeros(BT)
    for r0 in range(0, BT, row_block):
        r1 = min(BT, r0 + row_block)
        z = _as64(X[r0:r1]) @ W64.T
        if b64 is not None:
            z += b64
        logp, _ = log_softmax_rows(z / T)
        y = tgt[r0:r1]
        inside = (y != np.int64(ignore_index)) & (y >= 0) & (y < V)
        rows = np.arange(r1 - r0)
        out[r0:r1] = np.where(inside, logp[rows, np.clip(y, 0, V - 1)], 0.0)
    return out


def selective_logprob_backward(X, W, b, target, dlogp, ignore_index=-100, temperature=1.0,
                               compute_dW=True, compute_db=False, dX_rows=None, dW_rows=None,
                               row_block=256):
    """Gradients of sum_r dlogp_r * logp_r (logp of :func:`selective_logprob`)
    for given upstream gradients dlogp, fp64:

        d / d z_rv = dlogp_r ([v == y_r] - p_rv) / T,   p_r = softmax(u_r),

    zero on the rows whose logp is 0 by definition; dX = dz W, dW = dz^T X,
    db = sum over rows of dz."""
    if compute_db and b is None:
        raise OracleError("compute_db needs a bias")
    BT, H = np.shape(X)
    V = np.shape(W)[0]
    T = float(temperature)
    tgt = np.asarray(target).astype(np.int64)
    g = np.asarray(dlogp, dtype=np.float64)
    W64 = _as64(W)
    b64 = _as64(b)
    dx_sel = np.arange(BT) if dX_rows is None else np.asarray(dX_rows, dtype=np.int64)
    dw_sel = None if not compute_dW else (np.arange(V) if dW_rows is None
                                          else np.asarray(dW_rows, dtype=np.int64))
    dX = np.zeros((len(dx_sel), H))
    dW = None if dw_sel is None else np.zeros((len(dw_sel), H))
    db = np.zeros(V) if compute_db else None
    dx_pos = {int(r): i for i, r in enumerate(dx_sel)}
    for r0 in range(0, BT, row_block):
        r1 = min(BT, r0 + row_block)
        Xc = _as64(X[r0:r1])
        z = Xc @ W64.T
        if b64 is not None:
            z += b64
        logp, _ = log_softmax_rows(z / T)
        y = tgt[r0:r1]
        inside = (y != np.int64(ignore_index)) & (y >= 0) & (y < V)
        rows = np.arange(r1 - r0)
        G = -np.exp(logp)
        G[rows[inside], np.clip(y, 0, V - 1)[inside]] += 1.0
        G *= (g[r0:r1] / T)[:, None]
        G[~inside] = 0.0
        here = [i for i in range(r0, r1) if i in dx_pos]
        if here:
            dX[[dx_pos[i] for i in here]] = G[np.asarray(here) - r0] @ W64
        if dW is not None:
            dW += G[:, dw_sel].T @ Xc
        if db is not None:
            db += G.sum(axis=0)
    return dict(dX=dX, dW=dW, db=db)


def jsd_forward_backward(X, W, b, Xt, Wt, bt, shift_labels=None, ignore_index=-100,
                         temperature=1.0, beta=0.5, reduction="batchmean", compute_dW=True,
                         compute_db=False, dX_rows=None, dW_rows=None, row_block=256):
    """Fused linear Jensen-Shannon divergence, fp64.

    The FusedLinearKLDivLoss page names LigerFusedLinearJSD as the sibling
    loss whose teacher side has its own projection; it prints no formula.
    Reading used here (the generalized JSD): student P = softmax((X W^T +
    b)/T), teacher Q = softmax((Xt Wt^T + bt)/T), M = beta P + (1 - beta) Q,

        l_r = beta KL(P_r || M_r) + (1 - beta) KL(Q_r || M_r),

    with 0 log 0 = 0, rows dropped by shift_labels == ignore_index, and the
    divisors of the KL loss (batchmean: N_valid, mean: N_valid * V, sum: 1).
    Only the student gets gradients:

        d l_r / d z_rv = beta p_rv (log(p_rv / m_rv) - KL(P_r || M_r)) / T.
    """
    if reduction not in REDUCTIONS:
        raise OracleError(f"reduction={reduction!r} is not supported")
    if not (0.0 < beta < 1.0):
        raise OracleError("beta must lie in (0, 1)")
    if compute_db and b is None:
        raise OracleError("compute_db needs a bias")
    BT, H = np.shape(X)
    V = np.shape(W)[0]
    T = float(temperature)
    valid = valid_rows(BT, shift_labels, ignore_index)
    n_valid = int(valid.sum())
    D = divisor(reduction, n_valid, V)
    scale = 0.0 if n_valid == 0 else 1.0 / (T * D)
    W64, b64 = _as64(W), _as64(b)
    Wt64, bt64 = _as64(Wt), _as64(bt)
    dx_sel = np.arange(BT) if dX_rows is None else np.asarray(dX_rows, dtype=np.int64)
    dw_sel = None if not compute_dW else (np.arange(V) if dW_rows is None
                                          else np.asarray(dW_rows, dtype=np.int64))
    dX = np.zeros((len(dx_sel), H))
    dW = None if dw_sel is None else np.zeros((len(dw_sel), H))
    db = np.zeros(V) if compute_db else None
    row_loss = np.zeros(BT)
    dx_pos = {int(r): i for i, r in enumerate(dx_sel)}

    def xlogy(x, y):
        # x * log(x / y) with 0 log 0 = 0 (y > 0 wherever x > 0)
        out = np.zeros_like(x)
        nz = x > 0
        out[nz] = x[nz] * np.log(x[nz] / y[nz])
        return out

    for r0 in range(0, BT, row_block):
        r1 = min(BT, r0 + row_block)
        Xc = _as64(X[r0:r1])
        zs = Xc @ W64.T
        if b64 is not None:
            zs += b64
        zt = _as64(Xt[r0:r1]) @ Wt64.T
        if bt64 is not None:
            zt += bt64
        logp, _ = log_softmax_rows(zs / T)
        logq, _ = log_softmax_rows(zt / T)
        p, q = np.exp(logp), np.exp(logq)
        m = beta * p + (1.0 - beta) * q
        kl_pm = xlogy(p, m)
        kl_qm = xlogy(q, m)
        K = kl_pm.sum(axis=1)
        keep = valid[r0:r1]
        row_loss[r0:r1] = np.where(keep, beta * K + (1.0 - beta) * kl_qm.sum(axis=1), 0.0)
        ell = np.zeros_like(p)
        nz = p > 0
        ell[nz] = np.log(p[nz] / m[nz])
        G = beta * p * (ell - K[:, None]) * scale
        G[~keep] = 0.0
        here = [i for i in range(r0, r1) if i in dx_pos]
        if here:
            dX[[dx_pos[i] for i in here]] = G[np.asarray(here) - r0] @ W64
        if dW is not None:
            dW += G[:, dw_sel].T @ Xc
        if db is not None:
            db += G.sum(axis=0)
    loss = 0.0 if n_valid == 0 else float(row_loss.sum() / D)
    return dict(loss=loss, dX=dX, dW=dW, db=db, row_loss=row_loss, n_valid=n_valid, D=D)
