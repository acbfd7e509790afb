"""Float64 CPU oracle for RACE attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code, table or constant with the CUDA
library; both sides receive the same seeded inputs and nothing else.

What it computes, in the order the source pages give it.  Citations name the
pages by short tags:

  [JA]  "RACE Attention: 長系列トレーニングのための厳密な線形時間アテンションの技術的概要"
        (gist.science, Japanese technical overview of arXiv 2510.04008)
  [IT]  "RACE Attention: A Strictly Linear-Time Attention for Long-Sequence Training"
        (gist.science, Italian technical summary, "Sommario tecnico")
  [KO]  the same title on gist.science in Korean ("기술 요약")
  [ABS] "Replacing Softmax Similarity with a Sharpened Angular Similarity: Theory and
        Practice of Scaling To Billion-Context Attention" (arXiv abstract page)

* Kernel being estimated: sim(q, k) = (1 - arccos(q.k / |q||k|)/pi)^gamma, with the
  sharpening exponent gamma equal to the number of hyperplanes P  ([JA] §2.1,
  sim equation; [IT] §2 item 1; [JA] §3 bias-term bullet equates P with gamma).
* Soft bucketization: each query/key is projected on P random Gaussian hyperplanes
  per table and assigned softly to the R = 2^P hypercube corners  ([JA] §2.1
  "soft bucketization"; [IT] §2 item 2, softmax over the hypercube vertices;
  [KO] §2 algorithm flow, R = 2^P).  The exact soft form used here is
  phi(x) = concat_l softmax_b(<c_b, W_l^T xhat>/tau) / sqrt(L), with xhat = x/max(|x|,1e-12).
* Bucket aggregation: per table and bucket the key mass sum phi(k) and value sum
  sum phi(k) v^T  ([JA] §2.1 "bucket aggregation"; [IT] §2 sufficient statistics;
  [KO] §2 statistics aggregation).
* Reconstruction: bucket probabilities of the query times the aggregated values,
  averaged over tables and normalised: o_i = phi(q_i).S / phi(q_i).z  ([JA] §2.1
  "reconstruction"; [IT] §2 algorithm, normalised weighted mean).
* Causal mode through prefix sums over the sequence  ([JA] §2.2 "causal support";
  [IT] §3 item 3, causal and non-causal kernels).
* Differentiable end to end through the soft assignment  ([JA] §2.2
  "differentiability"; [IT] §3 item 4).  The gradient formulas below are the chain
  rule of the forward written out (no page prints them).

Readings of points the pages leave open (each is listed in the design notes):
  * temperature: the pages' beta is 1/tau;
  * zero vectors: xhat = x / max(|x|, 1e-12), so x = 0 gives a uniform softmax;
  * corner order: bit p of bucket index b set means c_bp = +1;
  * causal attention is inclusive (j <= i);
  * hard-hash tie: u_p >= 0 maps to bit 1.
"""
from __future__ import annotations

import numpy as np

EPS_NORM = 1e-12


# --------------------------------------------------------------------------- #
# building blocks
# --------------------------------------------------------------------------- #
def corners(P: int) -> np.ndarray:
    """The R = 2^P hypercube corners c_b in {-1,+1}^P as a float64 [R, P] array.

    Bit p of b set means c_bp = +1 ([KO] §2: R = 2^P buckets; ordering is a free
    choice, fixed here)."""
    R = 1 << P
    b = np.arange(R)[:, None]
    p = np.arange(P)[None, :]
    return np.where((b >> p) & 1, 1.0, -1.0)


def normalize(x: np.ndarray) -> np.ndarray:
    """xhat = x / max(|x|_2, 1e-12), row-wise over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, EPS_NORM)


def projections(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """u[n, l, p] = W_l^T xhat_n : the P random-hyperplane projections per table.

    x: [n, d]; W: [L, d, P] (plane p of table l is W[l, :, p]).  [KO] §2: each
    table projects queries and keys on P random hyperplanes."""
    xh = normalize(x)
    return np.einsum("nd,ldp->nlp", xh, np.asarray(W, dtype=np.float64))


def soft_hash(x: np.ndarray, W: np.ndarray, tau: float) -> np.ndarray:
    """p[n, l, b] = softmax_b(<c_b, u_l>/tau): soft assignment to the 2^P corners.

    Written literally: all 2^P logits, then a max-subtracted softmax ([IT] §2 item 2:
    softmax over the hypercube vertices)."""
    P = W.shape[2]
    u = projections(x, W)                               # [n, L, P]
    logits = np.einsum("nlp,rp->nlr", u, corners(P)) / float(tau)
    logits -= logits.max(axis=-1, keepdims=True)
    e = np.exp(logits)
    return e / e.sum(axis=-1, keepdims=True)


def phi(x: np.ndarray, W: np.ndarray, tau: float) -> np.ndarray:
    """Feature map phi(x) = concat_l p_l(x) / sqrt(L), shape [n, L*R]."""
    p = soft_hash(x, W, tau)
    n, L, R = p.shape
    return p.reshape(n, L * R) / np.sqrt(L)


def hard_hash(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Integer bucket ids h[n, l] of signed random projections (the tau -> 0 limit).

    Bit p is 1 when u_p >= 0.  Two vectors at angle theta collide in one table
    with probability (1 - theta/pi)^P ([JA] §2.1: the angular-kernel power equals
    the LSH collision probability)."""
    u = projections(x, W)
    bits = (u >= 0).astype(np.int64)
    return np.sum(bits << np.arange(W.shape[2])[None, None, :], axis=-1)


def hard_forward(q, k, v, W, causal):
    """The classic RACE estimator with hard hashes (the tau -> 0 limit of the soft one)
    for one head: count arrays of bucket collisions ([JA] §2.1: repeated arrays of count
    estimators, bucket aggregation; [KO] §2: L tables of P-bit buckets).

    A_ij = number of tables l with h_l(q_i) == h_l(k_j), over the attended set J(i);
    o_i = sum_j A_ij v_j / sum_j A_ij, and o_i = 0 where no key collides with q_i in any
    table (reading: the ratio is undefined there; the soft estimator never has this case).
    Returns (o [N, d], den [N] integer collision counts)."""
    v = np.asarray(v, dtype=np.float64)
    hq, hk = hard_hash(q, W), hard_hash(k, W)              # [N, L]
    A = (hq[:, None, :] == hk[None, :, :]).sum(axis=2).astype(np.float64)
    A = A * _mask(len(q), causal)
    den = A.sum(axis=1)
    num = A @ v
    o = np.where(den[:, None] > 0, num / np.maximum(den, 1.0)[:, None], 0.0)
    return o, den.astype(np.int64)


def hard_counts(x, v, W):
    """Count arrays of one head: C[l, b] = number of keys in bucket b of table l and
    S[l, b] = sum of their values ([JA] §2.1 bucket aggregation with hard hashes)."""
    h = hard_hash(x, W)
    L, R = W.shape[0], 1 << W.shape[2]
    C = np.zeros((L, R), dtype=np.int64)
    S = np.zeros((L, R, v.shape[1]))
    for l in range(L):
        np.add.at(C[l], h[:, l], 1)
        np.add.at(S[l], h[:, l], np.asarray(v, dtype=np.float64))
    return C, S


def angular_kernel(q: np.ndarray, k: np.ndarray, P: int) -> np.ndarray:
    """sim[i, j] = (1 - arccos(qhat_i . khat_j)/pi)^P  ([JA] §2.1, sim equation)."""
    c = np.clip(normalize(q) @ normalize(k).T, -1.0, 1.0)
    return (1.0 - np.arccos(c) / np.pi) ** P


def _mask(n: int, causal: bool) -> np.ndarray:
    if causal:
        return np.tril(np.ones((n, n)))
    return np.ones((n, n))


# --------------------------------------------------------------------------- #
# forward
# --------------------------------------------------------------------------- #
def direct_forward(q, k, v, W, tau, causal):
    """O(N^2) definition for one head: a_ij = phi(q_i).phi(k_j) over the attended
    set J(i) (all j, or j <= i), o_i = sum a_ij v_j / sum a_ij.

    Returns (o [N, d], den [N]) with den_i = sum_{j in J(i)} a_ij."""
    v = np.asarray(v, dtype=np.float64)
    A = phi(q, W, tau) @ phi(k, W, tau).T * _mask(len(q), causal)
    den = A.sum(axis=1)
    return (A @ v) / den[:, None], den


def forward(q, k, v, W, tau, causal, block: int = 256):
    """Same estimator as ``direct_forward`` through the RACE sketch for one head:
    the sketch S = sum phi(k_j) v_j^T and mass z = sum phi(k_j) ([JA] §2.1 bucket
    aggregation), read out by phi(q_i) and normalised ([JA] §2.1 reconstruction).
    Causal mode carries S and z as prefix sums over blocks of ``block`` tokens plus
    the masked in-block term ([JA] §2.2 causal support).

    Returns (o [N, d], den [N])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, d = v.shape
    L, _, P = W.shape
    LR = L * (1 << P)
    vv = np.concatenate([v, np.ones((N, 1))], axis=1)          # [v | 1]
    out = np.empty((N, d))
    den = np.empty(N)
    if not causal:
        Sz = np.zeros((LR, d + 1))
        for s in range(0, N, block):
            Sz += phi(k[s:s + block], W, tau).T @ vv[s:s + block]
        for s in range(0, N, block):
            nz = phi(q[s:s + block], W, tau) @ Sz
            out[s:s + block] = nz[:, :d] / nz[:, d:]
            den[s:s + block] = nz[:, d]
        return out, den
    Sz = np.zeros((LR, d + 1))                                   # prefix state
    for s in range(0, N, block):
        fq = phi(q[s:s + block], W, tau)
        fk = phi(k[s:s + block], W, tau)
        nz = fq @ Sz + np.tril(fq @ fk.T) @ vv[s:s + block]
        out[s:s + block] = nz[:, :d] / nz[:, d:]
        den[s:s + block] = nz[:, d]
        Sz += fk.T @ vv[s:s + block]
    return out, den


def exact_angular_attention(q, k, v, P, causal):
    """O(N^2) attention with the exact angular kernel (the L -> inf, tau -> 0 target)."""
    A = angular_kernel(q, k, P) * _mask(len(q), causal)
    return (A @ np.asarray(v, dtype=np.float64)) / A.sum(axis=1, keepdims=True)


# --------------------------------------------------------------------------- #
# backward
# --------------------------------------------------------------------------- #
def hash_backward(x, W, tau, dphi):
    """Chain rule from d loss/d phi(x) back to x and W for one set of vectors.

    phi = concat_l softmax(C u_l / tau)/sqrt(L), u_l = W_l^T xhat, xhat = x/max(|x|,eps).
    Steps, each the textbook derivative of the forward step above:
      gp      = dphi / sqrt(L)                                  (concat and scale)
      dlogit  = p * (gp - <p, gp>)                               (softmax Jacobian)
      du      = C^T dlogit / tau                                 (logits = C u / tau)
      dxhat   = sum_l W_l du_l ;  dW_l = xhat du_l^T             (projection)
      dx      = (dxhat - xhat (xhat.dxhat)) / |x|   if |x| > eps, else dxhat / eps.
    Returns (dx [n, d], dW [L, d, P])."""
    x = np.asarray(x, dtype=np.float64)
    L, d, P = W.shape
    R = 1 << P
    n = x.shape[0]
    p = soft_hash(x, W, tau)                                    # [n, L, R]
    gp = np.asarray(dphi, dtype=np.float64).reshape(n, L, R) / np.sqrt(L)
    dlogit = p * (gp - np.sum(p * gp, axis=-1, keepdims=True))
    du = np.einsum("nlr,rp->nlp", dlogit, corners(P)) / float(tau)
    xh = normalize(x)
    dxh = np.einsum("nlp,ldp->nd", du, np.asarray(W, dtype=np.float64))
    dW = np.einsum("nd,nlp->ldp", xh, du)
    nrm = np.sqrt(np.sum(x * x, axis=1, keepdims=True))
    big = nrm > EPS_NORM
    proj = dxh - xh * np.sum(xh * dxh, axis=1, keepdims=True)
    dx = np.where(big, proj / np.maximum(nrm, EPS_NORM), dxh / EPS_NORM)
    return dx, dW


def direct_backward(q, k, v, W, tau, causal, dout):
    """Gradient of the O(N^2) forward for one head, through the dense a_ij matrix.

    With ghat_i = g_i/den_i and c_i = ghat_i.o_i:  d a_ij = ghat_i.v_j - c_i on the
    attended set, dv = A^T ghat, dphi(q) = dA phi(k), dphi(k) = dA^T phi(q).
    Returns (dq, dk, dv, dW)."""
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(dout, dtype=np.float64)
    fq, fk = phi(q, W, tau), phi(k, W, tau)
    M = _mask(len(q), causal)
    A = fq @ fk.T * M
    den = A.sum(axis=1)
    o = (A @ v) / den[:, None]
    gh = g / den[:, None]
    c = np.sum(gh * o, axis=1)
    dA = (gh @ v.T - c[:, None]) * M
    dv = A.T @ gh
    dq, dWq = hash_backward(q, W, tau, dA @ fk)
    dk, dWk = hash_backward(k, W, tau, dA.T @ fq)
    return dq, dk, dv, dWq + dWk


def backward(q, k, v, W, tau, causal, dout, out=None, block: int = 256):
    """Gradient for one head through the sketch states (linear in N).

    With ghat_i = g_i/den_i, c_i = ghat_i.o_i and g'_i = [ghat_i, -c_i]:
      dphi(q_i) = S_i ghat_i - z_i c_i = [S_i | z_i] g'_i         (prefix states, j <= i)
      dphi(k_j) = T_j v_j - t_j,  T_j = sum_{i >= j} phi(q_i) ghat_i^T,
                                  t_j = sum_{i >= j} phi(q_i) c_i
      dv_j      = T_j^T phi(k_j)
    (non-causal: all sums run over the whole sequence), then ``hash_backward``.
    ``out`` defaults to the oracle's own forward output.
    Returns (dq, dk, dv, dW)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(dout, dtype=np.float64)
    N, d = v.shape
    L, _, P = W.shape
    LR = L * (1 << P)
    o_ref, den = forward(q, k, v, W, tau, causal, block)
    o = o_ref if out is None else np.asarray(out, dtype=np.float64)
    gh = g / den[:, None]
    gp = np.concatenate([gh, -np.sum(gh * o, axis=1, keepdims=True)], axis=1)  # g'
    vv = np.concatenate([v, np.ones((N, 1))], axis=1)
    dphq = np.empty((N, LR))
    dphk = np.empty((N, LR))
    dv = np.empty((N, d))
    if not causal:
        fq_all = [phi(q[s:s + block], W, tau) for s in range(0, N, block)]
        fk_all = [phi(k[s:s + block], W, tau) for s in range(0, N, block)]
        Sz = sum(fk.T @ vv[s:s + block] for s, fk in zip(range(0, N, block), fk_all))
        Tt = sum(fq.T @ gp[s:s + block] for s, fq in zip(range(0, N, block), fq_all))
        for s, fq, fk in zip(range(0, N, block), fq_all, fk_all):
            dphq[s:s + block] = gp[s:s + block] @ Sz.T
            dphk[s:s + block] = vv[s:s + block] @ Tt.T
            dv[s:s + block] = fk @ Tt[:, :d]
    else:
        Sz = np.zeros((LR, d + 1))
        for s in range(0, N, block):                               # forward sweep
            fq = phi(q[s:s + block], W, tau)
            fk = phi(k[s:s + block], W, tau)
            B = np.tril(gp[s:s + block] @ vv[s:s + block].T)        # g'_i.[v_j;1], j <= i
            dphq[s:s + block] = gp[s:s + block] @ Sz.T + B @ fk
            Sz += fk.T @ vv[s:s + block]
        Tt = np.zeros((LR, d + 1))
        starts = list(range(0, N, block))
        for s in reversed(starts):                                 # reverse sweep
            fq = phi(q[s:s + block], W, tau)
            fk = phi(k[s:s + block], W, tau)
            B = np.tril(gp[s:s + block] @ vv[s:s + block].T)        # rows i, cols j <= i
            A = np.tril(fq @ fk.T)
            dphk[s:s + block] = vv[s:s + block] @ Tt.T + B.T @ fq
            dv[s:s + block] = fk @ Tt[:, :d] + A.T @ gh[s:s + block]
            Tt += fq.T @ gp[s:s + block]
    dq, dWq = hash_backward(q, W, tau, dphq)
    dk, dWk = hash_backward(k, W, tau, dphk)
    return dq, dk, dv, dWq + dWk


# --------------------------------------------------------------------------- #
# multi-head wrappers: q, k, v, dout are [H, N, d]; W is shared by every head
# --------------------------------------------------------------------------- #
def forward_heads(q, k, v, W, tau, causal, block: int = 256):
    outs, dens = zip(*(forward(q[h], k[h], v[h], W, tau, causal, block)
                       for h in range(q.shape[0])))
    return np.stack(outs), np.stack(dens)


def backward_heads(q, k, v, W, tau, causal, dout, out=None, block: int = 256):
    H = q.shape[0]
    res = [backward(q[h], k[h], v[h], W, tau, causal, dout[h],
                    None if out is None else out[h], block) for h in range(H)]
    dq = np.stack([r[0] for r in res])
    dk = np.stack([r[1] for r in res])
    dv = np.stack([r[2] for r in res])
    dW = np.sum([r[3] for r in res], axis=0)
    return dq, dk, dv, dW


def partial_sums(q, k, v, W, tau, mask=None, block: int = 256):
    """Unnormalised sums of the definition over a given set of keys:
    num_i = sum_j a_ij v_j and den_i = sum_j a_ij, a_ij = phi(q_i).phi(k_j), for every
    query row q_i and every key row k_j given (mask[i, j] in {0, 1}, when given, drops
    keys).  Summing the results over a split of the keys and dividing gives o_i of
    ``direct_forward`` ([JA] §2.1 reconstruction: a weighted mean), which is what lets a
    long sequence be cut into key ranges that are summed independently.
    Returns (num [n, d], den [n])."""
    v = np.asarray(v, dtype=np.float64)
    fq = phi(q, W, tau)
    num = np.zeros((len(fq), v.shape[1]))
    den = np.zeros(len(fq))
    for s in range(0, len(k), block):
        e = min(s + block, len(k))
        A = fq @ phi(k[s:e], W, tau).T
        if mask is not None:
            A = A * np.asarray(mask)[:, s:e]
        num += A @ v[s:e]
        den += A.sum(axis=1)
    return num, den


def forward_rows(q, k, v, W, tau, causal, rows, block: int = 256):
    """Outputs o_i for selected rows ``rows`` of one head, computed one by one from
    the definition (keys limited to j <= i when causal).  Cost grows with the
    largest row when causal, with N otherwise."""
    rows = np.asarray(rows)
    v = np.asarray(v, dtype=np.float64)
    fq = phi(q[rows], W, tau)
    hi = int(rows.max()) + 1 if causal else len(k)
    num = np.zeros((len(rows), v.shape[1]))
    den = np.zeros(len(rows))
    for s in range(0, hi, block):
        e = min(s + block, hi)
        A = fq @ phi(k[s:e], W, tau).T
        if causal:
            A = A * (np.arange(s, e)[None, :] <= rows[:, None])
        num += A @ v[s:e]
        den += A.sum(axis=1)
    return num / den[:, None], den
