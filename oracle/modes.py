"""Decode outputs of one unit for every mode, fp64.

Notation: q [G, d] the decode queries of the group, K, V [L, d], s the
softmax scale, l_hj = s q_h . K_j the true logits, I the exactly-read
positions (sorted), T the tail (the rest), n_T = |T|.  Every mode returns
o [G, d].  With n_T = 0 every mode reads everything and skips its residual,
so a full budget gives dense attention exactly (the reading of the empty tail
the RESA and vAttention pages leave open).

Parity pins: tests/test_oracle_modes.py (full budget = torch
scaled_dot_product_attention; RESA delta merge = the O(L) merged-logit
softmax; RESA exact for identical keys; lambda = 0 gives drop; proxy exact for
a one-token tail and for identical keys; sampling estimator unbiased over
seeds and exact for identical tail tokens; the per-head estimator reduces
to the group estimator when every head draws the same positions, and per
head to the one-head estimator).
"""
import numpy as np


def _softmax_weighted(logits, values):
    """sum_j softmax(logits)_j values_j over the last axis of logits [G, n]."""
    m = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - m)
    return (w @ values) / w.sum(axis=1, keepdims=True)


def dense(q, k, v, scale):
    """Plain softmax attention over all L tokens: softmax(s q K^T) V."""
    return _softmax_weighted(scale * (q @ k.T), v)


def drop(q, k, v, idx, scale):
    """Sparse attention that treats the unread tail as contributing zero.
    Attention over an empty set carries no mass and returns the zero vector
    (the pages never read nothing; this is the plain reading of an empty sum)."""
    if len(idx) == 0:
        return np.zeros((q.shape[0], v.shape[1]))
    return dense(q, k[idx], v[idx], scale)


def resa(q, k, v, idx, st, scale, lam=1.0):
    """RESA output (RESA page, Method, key design 2, "Online Aggregator").

    Prior logits P_hj = s mu_Q,h . K_j + c_h with the bias
    c_h = s (q_h - mu_Q,h) . mu_K (key design 1); Z = sum_j exp(P_hj) comes
    from the prefill normaliser: Z = exp(log_z0 + c).  At decode, in the
    page's order:
      Z'    = lam (Z - sum_{j in I} exp(P_j)) + sum_{j in I} exp(l_j)
      alpha = lam Z / Z',   beta = sum_{j in I} exp(l_j) / Z'
      O     = alpha O_Est + (beta S^SA_I - alpha S_I) V_I
    with S_I = exp(P_I)/Z the prior softmax at I and S^SA_I = exp(l_I) /
    sum_I exp(l) the sparse softmax.  The page writes alpha' = lam*alpha for
    the prior weight and says lam = 0 falls back to plain sparse attention;
    that holds when lam also scales the prior mass inside Z' (as written
    above), which equals the page at lam = 1.  Exponentials are shifted by
    one common maximum (the page's log-sum-exp protection).
    """
    L = k.shape[0]
    n_t = L - len(idx)
    if n_t == 0 or (lam == 0 and len(idx) == 0):    # nothing to merge: no mass at all
        return drop(q, k, v, idx, scale)
    kI, vI = k[idx], v[idx]
    c = scale * ((q - st["mu_q"]) @ st["mu_k"])                  # [G]
    l_i = scale * (q @ kI.T)                                      # [G, |I|]
    p_i = scale * (st["mu_q"] @ kI.T) + c[:, None]                # [G, |I|]
    log_z = st["log_z0"] + c                                      # [G]
    cols = [log_z[:, None]]
    if len(idx):
        cols += [l_i.max(axis=1, keepdims=True), p_i.max(axis=1, keepdims=True)]
    m = np.concatenate(cols, axis=1).max(axis=1, keepdims=True)   # common shift
    z = np.exp(log_z[:, None] - m)                                # Z, shifted
    e_p = np.exp(p_i - m)
    e_l = np.exp(l_i - m)
    prior_mass_t = np.maximum(z[:, 0] - e_p.sum(axis=1), 0.0)     # Z - sum_I exp(P)
    z_new = lam * prior_mass_t + e_l.sum(axis=1)                  # Z'
    alpha = lam * z[:, 0] / z_new
    beta_s_sa = e_l / z_new[:, None]                              # beta * S^SA_I
    s_i = e_p / z                                                 # S_I
    return alpha[:, None] * st["o_est"] + (beta_s_sa - alpha[:, None] * s_i) @ vI


def resa_merged_logits(q, k, v, idx, st, scale, lam=1.0):
    """The naive O(L) form the RESA page starts from: replace the prior logits
    at the selected positions by the true ones and take one softmax over all
    L positions (tail logits P_j + ln lam).  Used only to cross-check resa()."""
    L = k.shape[0]
    if L == len(idx):
        return drop(q, k, v, idx, scale)
    c = scale * ((q - st["mu_q"]) @ st["mu_k"])
    logits = scale * (st["mu_q"] @ k.T) + c[:, None]
    with np.errstate(divide="ignore"):
        logits = logits + np.log(lam)
    logits[:, idx] = scale * (q @ k[idx].T)
    return _softmax_weighted(logits, v)


def proxy(q, k, v, idx, st, scale):
    """Count-aware mean proxy (OpenAttention, abstract and stage 04): the
    whole tail folds into ONE virtual token with key = tail-mean key,
    value = tail-mean value and logit zbar + ln n_T, where zbar is the
    logit of the tail-mean key (the page's garbled "zbar_b + log n_b" read
    as the mean member logit, which is linear in K).  Tail sums are the
    prefill totals minus the selected rows; the token joins the exact ones
    in one softmax."""
    L = k.shape[0]
    n_t = L - len(idx)
    if n_t == 0:
        return drop(q, k, v, idx, scale)
    kbar_t = (st["sum_k"] - k[idx].sum(axis=0)) / n_t
    vbar_t = (st["sum_v"] - v[idx].sum(axis=0)) / n_t
    z = scale * (q @ kbar_t) + np.log(n_t)                       # [G]
    logits = np.concatenate([scale * (q @ k[idx].T), z[:, None]], axis=1)
    values = np.concatenate([v[idx], vbar_t[None, :]], axis=0)
    return _softmax_weighted(logits, values)


def sample(q, k, v, idx, pos, scale):
    """vAttention estimator (Method, key design 1, paper eq. 3): exact terms
    on I with probability 1 plus the b drawn tail positions reweighted by
    n_s / b (n_s = n_T here); draws are with replacement, a position drawn
    twice counts twice.  Reweighting is folded into the logit as + ln(n_T/b)."""
    L = k.shape[0]
    n_t = L - len(idx)
    b = len(pos)
    if n_t == 0 or b == 0:
        return drop(q, k, v, idx, scale)
    lw = np.log(n_t / b)
    logits = np.concatenate([scale * (q @ k[idx].T), scale * (q @ k[pos].T) + lw], axis=1)
    values = np.concatenate([v[idx], v[pos]], axis=0)
    return _softmax_weighted(logits, values)


def sample_per_head(q, k, v, idx, pos_per_head, scale):
    """The sampling estimator with one sample per query head (the vAttention
    page samples per head): head h uses its own draws pos_per_head[h] and
    weight n_T / len(pos_per_head[h]); the exactly read set I is the group's."""
    return np.concatenate([sample(q[h:h + 1], k, v, idx, pos_per_head[h], scale) for h in range(q.shape[0])], axis=0)


def sample_num_den(q, k, v, idx, pos, scale, shift):
    """Unnormalised estimator (N_hat [G, d], D_hat [G]) with all exponentials
    taken relative to ``shift`` [G]; used by the unbiasedness pin."""
    n_t = k.shape[0] - len(idx)
    b = len(pos)
    e_i = np.exp(scale * (q @ k[idx].T) - shift[:, None])
    e_s = np.exp(scale * (q @ k[pos].T) - shift[:, None]) * (n_t / b)
    return e_i @ v[idx] + e_s @ v[pos], e_i.sum(axis=1) + e_s.sum(axis=1)


def run_mode(mode, q, k, v, idx, st, scale, pos=None, lam=1.0):
    if mode == "dense":
        return dense(q, k, v, scale)
    if mode == "drop":
        return drop(q, k, v, idx, scale)
    if mode == "resa":
        return resa(q, k, v, idx, st, scale, lam)
    if mode == "proxy":
        return proxy(q, k, v, idx, st, scale)
    if mode == "sample":
        return sample(q, k, v, idx, pos, scale)
    raise ValueError(mode)
