"""Plain fp64 CPU oracle for SAS gated block-sparse attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The product path (the CUDA library and its Python binding) never calls
it, and this module imports nothing from the product package.

Source: "SAS: Simple Attention Sparsification via End-to-End Optimization of
Context Ranking" (arXiv 2609.13141, HTML version); cited below as "SAS paper".

Every function here is the plain definition written out in numpy float64:
the biased logit matrix and the block mask are materialised in full, the row
softmax is max-subtracted, and the gradients are the textbook softmax-attention
backward. Matrix products use numpy's ``@`` (a library matmul). There is no
tiling, no online softmax and no fusion.

Conventions (the readings of the paper that the whole build uses):

* Blocks of ``block`` tokens (64 in the paper, §5.1 "Training setup").
  Query position ``t`` sits in block ``c_t = t // block`` (its current block
  B_0). Its historical blocks are ``m < c_t``. Later blocks are never attended
  (causal attention).
* The budget ``K`` counts the current block, so ``H = K - 1`` historical
  blocks are selected per query (§4.3, the attended set S = B_0 ∪ Top-K).
* The gates are shared by the query heads of one KV group. The selection is
  per (batch, KV group, position), and all of the group's heads use it.
* ``sm_scale`` multiplies q·k only; the log-gate is added unscaled
  (Appendix E, Algorithm 3).
* Top-K ties go to the lower block index; -0.0 equals +0.0.
* LSE is the natural-log log-sum-exp of the biased, scaled logits.
"""

from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf


def _f64(x):
    """Copy any array-like (numpy or CPU torch tensor) into a float64 numpy array."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy()
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------------------
# Gate normalisation: SAS paper §4.1 eq. 4 (g = phi(s), g_0 = 1) with phi = softmax,
# and §4.2 "Activation function" eq. 6: log g_m = s_m - LSE(s) over historical blocks.
# --------------------------------------------------------------------------------------
def gate_normalize(s, block: int):
    """Return logG with ``logG[..., t, m] = s[..., t, m] - logsumexp(s[..., t, :c_t])`` for m < c_t.

    Entries with ``m >= c_t`` (the current and future blocks) are -inf.
    Rows with ``c_t == 0`` have no historical block and are all -inf.

    s: [B, Hkv, T, NB] selector logits. Returns float64 of the same shape.
    """
    s = _f64(s)
    B, Hkv, T, NB = s.shape
    out = np.full(s.shape, NEG_INF)
    for t in range(T):
        c = t // block
        if c == 0:
            continue
        hist = s[:, :, t, :c]
        mx = hist.max(axis=-1, keepdims=True)
        lse = mx + np.log(np.exp(hist - mx).sum(axis=-1, keepdims=True))
        out[:, :, t, :c] = hist - lse
    return out


def gate_lse(s, block: int):
    """Return ``lse[..., t] = log sum_{m < c_t} exp(s[..., t, m])``, the normaliser of eq. 6 (SAS paper
    §4.2 "Activation function": log g = s - log sum exp over the historical blocks).

    The compact form of the gates keeps s and this per-row value instead of logG:
    ``logG[..., t, m] = s[..., t, m] - lse[..., t]`` for m < c_t. Rows with ``c_t == 0``
    have no historical block: -inf. s: [B, Hkv, T, NB]. Returns float64 [B, Hkv, T].
    """
    s = _f64(s)
    B, Hkv, T, NB = s.shape
    out = np.full((B, Hkv, T), NEG_INF)
    for t in range(T):
        c = t // block
        if c == 0:
            continue
        hist = s[:, :, t, :c]
        mx = hist.max(axis=-1)
        out[:, :, t] = mx + np.log(np.exp(hist - mx[..., None]).sum(axis=-1))
    return out


# --------------------------------------------------------------------------------------
# Selector-score gradient: SAS paper Appendix D.3 "Gradient Derivation for Training
# Scope" (the softmax backward ds_m = g_m (dg_m - sum_l g_l dg_l)) and §4.2 eq. 8.
# With the gate gradient given in log form, dLogG_l = g_l dg_l, this is
# ds_m = dLogG_m - g_m * sum_l dLogG_l over the historical blocks l < c_t.
# --------------------------------------------------------------------------------------
def gate_grad(s, dLogG, block: int):
    """Return ``ds = dL/ds`` given ``dLogG = dL/dlogG`` for ``logG = gate_normalize(s)``.

    For each row, over the historical blocks m < c_t: the Jacobian of
    log g_l = s_l - LSE(s) is d log g_l / d s_m = [l == m] - g_m, so
    ds_m = sum_l dLogG_l ([l == m] - g_m). Entries m >= c_t are 0.
    s, dLogG: [B, Hkv, T, NB]. Returns float64 of the same shape.
    """
    s = _f64(s)
    dl = _f64(dLogG)
    B, Hkv, T, NB = s.shape
    ds = np.zeros(s.shape)
    for t in range(T):
        c = min(t // block, NB)
        if c == 0:
            continue
        hist = s[:, :, t, :c]
        g = np.exp(hist - hist.max(axis=-1, keepdims=True))
        g = g / g.sum(axis=-1, keepdims=True)
        d = dl[:, :, t, :c]
        jac = np.eye(c)[None, None] - g[:, :, None, :]          # [.., l, m] = [l == m] - g_m
        ds[:, :, t, :c] = np.einsum("bgl,bglm->bgm", d, jac)
    return ds


# --------------------------------------------------------------------------------------
# Top-K as a per-query threshold: SAS paper §4.3 "Kernel Design" and Appendix E
# (a block is active when its log gate reaches the per-query threshold tau).
# Exactly H = K-1 blocks are kept; equal values are broken toward the lower index,
# which the extra index tau_idx encodes.
# --------------------------------------------------------------------------------------
def topk_threshold_row(vals, c: int, H: int):
    """Threshold for one row: the first ``H`` of blocks ``0..c-1`` ordered by (value desc, index asc).

    Returns ``(tau, tau_idx, chosen)`` where ``chosen`` is the ascending list of
    selected block indices. Rows with ``min(c, H) == 0`` select nothing and get
    ``(+inf, -1)``. Rows with ``c <= H`` select all their historical blocks and get
    ``(-inf, c-1)``.
    """
    if min(c, H) == 0:
        return math.inf, -1, []
    if c <= H:
        return -math.inf, c - 1, list(range(c))
    # A full sort: (value descending, index ascending). -0.0 and +0.0 compare equal.
    order = sorted(range(c), key=lambda m: (-float(vals[m]) + 0.0, m))
    taken = order[:H]
    tau = float(vals[taken[-1]])
    tau_idx = max(m for m in taken if float(vals[m]) == tau)
    return tau, tau_idx, sorted(taken)


def select_threshold(logG, K: int, block: int):
    """Per-(b, g, t) Top-(K-1) threshold over the historical blocks.

    logG: [B, Hkv, T, NB] (the values are used as given, e.g. a float32 tensor upcast).
    Returns ``tau`` [B,Hkv,T] float64, ``tau_idx`` [B,Hkv,T] int32 and ``sel``
    [B,Hkv,T,H] int32 (ascending block indices, padded with -1).
    """
    v = _f64(logG)
    B, Hkv, T, NB = v.shape
    H = K - 1
    tau = np.zeros((B, Hkv, T))
    tidx = np.zeros((B, Hkv, T), dtype=np.int32)
    sel = np.full((B, Hkv, T, max(H, 0)), -1, dtype=np.int32)
    for b in range(B):
        for g in range(Hkv):
            for t in range(T):
                c = min(t // block, NB)
                tv, ti, chosen = topk_threshold_row(v[b, g, t], c, H)
                tau[b, g, t] = tv
                tidx[b, g, t] = ti
                sel[b, g, t, : len(chosen)] = chosen
    return tau, tidx, sel


def selection_mask(logG, tau, tau_idx, block: int):
    """Boolean [B,Hkv,T,NB]: block m is selected for row t iff m < c_t and
    (logG > tau, or logG == tau and m <= tau_idx).  SAS paper Appendix E
    (active = log g >= tau), with the tie index making the set exactly Top-(K-1).
    """
    v = _f64(logG)
    tau = _f64(tau)[..., None]
    tidx = np.asarray(tau_idx)[..., None]
    B, Hkv, T, NB = v.shape
    m = np.arange(NB)[None, None, None, :]
    c = (np.arange(T) // block)[None, None, :, None]
    return (m < c) & ((v > tau) | ((v == tau) & (m <= tidx)))


# --------------------------------------------------------------------------------------
# The "full*" training scope of SAS paper §4.1 (Table 1, row 11): noise is added to the
# selector scores before Top-K, so the attended set is the Top-K of the noisy scores
# while the gates of the attended blocks stay those of the clean scores.
# --------------------------------------------------------------------------------------
def select_noisy(logG32, noise32, K: int, block: int):
    """Top-(K-1) of the noisy keys ``logG + noise`` and the gate tensor restricted to it.

    logG32, noise32: float32 [B, Hkv, T, NB]. The keys are formed in float32 (the
    sum decides an index, so it is taken in the kernel's precision); adding noise
    to s or to logG = s - LSE(s) ranks the blocks of a row alike. Returns
    ``logG_sel`` (float64: logG on the chosen blocks, -inf elsewhere), ``tau`` and
    ``tau_idx`` (the threshold of ``logG_sel``, which the attention calls use to
    find the chosen blocks again) and ``sel`` (ascending chosen blocks, -1 padded).
    Blocks whose gate is -inf (other documents of a packed sequence, see
    gate_normalize_varlen) are never chosen; a row with fewer finite gates than
    K-1 chooses them all and gets the threshold (least chosen gate, last chosen
    block holding it) so that no -inf block passes it.
    """
    lg = np.asarray(logG32, dtype=np.float32)
    keys = (lg + np.asarray(noise32, dtype=np.float32)).astype(np.float32)
    B, Hkv, T, NB = lg.shape
    H = K - 1
    logG_sel = np.full((B, Hkv, T, NB), -np.inf)
    tau = np.zeros((B, Hkv, T))
    tidx = np.zeros((B, Hkv, T), dtype=np.int32)
    sel = np.full((B, Hkv, T, max(H, 0)), -1, dtype=np.int32)
    for b in range(B):
        for g in range(Hkv):
            for t in range(T):
                c = min(t // block, NB)
                # A block whose gate is -inf (another document of a packed sequence) is never chosen.
                n_fin = int(np.isfinite(lg[b, g, t, :c]).sum())
                k = min(H, n_fin)
                _, _, chosen = topk_threshold_row(keys[b, g, t].astype(np.float64), c, k)
                for m in chosen:
                    logG_sel[b, g, t, m] = float(lg[b, g, t, m])
                if k == H or n_fin == c:
                    tv, ti, again = topk_threshold_row(logG_sel[b, g, t], c, H)
                    assert again == chosen
                elif k == 0:
                    tv, ti = math.inf, -1
                else:
                    # Every finite block chosen but fewer than H: the least chosen gate and the
                    # last chosen block holding it, so that no -inf block passes the threshold.
                    tv = min(float(lg[b, g, t, m]) for m in chosen)
                    ti = max(m for m in chosen if float(lg[b, g, t, m]) == tv)
                    tv = 0.0 if tv == 0.0 else tv
                tau[b, g, t] = tv
                tidx[b, g, t] = ti
                sel[b, g, t, : len(chosen)] = chosen
    return logG_sel, tau, tidx, sel


# --------------------------------------------------------------------------------------
# The biased logit matrix of SAS paper §4.3 eq. 9:
#   softmax(q K_S^T + log g_S) V_S,  S = B_0 ∪ (selected historical blocks),
# written as a dense [rows, T] bias: 0 on the causal part of the current block,
# logG on selected historical blocks, -inf everywhere else.
# --------------------------------------------------------------------------------------
def bias_rows(logG_g, mask_g, rows, T: int, block: int):
    """Dense bias for query positions ``rows`` of one (b, g): shape [len(rows), T]."""
    rows = np.asarray(rows)
    keys = np.arange(T)
    kb = keys // block                      # block of each key
    cb = (rows // block)[:, None]           # current block of each row
    own = (kb[None, :] == cb) & (keys[None, :] <= rows[:, None])
    kb_c = np.minimum(kb, logG_g.shape[-1] - 1)
    hist = (kb[None, :] < cb) & mask_g[rows][:, kb_c]
    gate = logG_g[rows][:, kb_c]
    bias = np.full((len(rows), T), NEG_INF)
    bias[hist] = gate[hist]
    bias[own] = 0.0
    return bias


def _group_of(h: int, Hq: int, Hkv: int) -> int:
    return h // (Hq // Hkv)


def forward(Q, K, V, logG, tau, tau_idx, block: int, sm_scale: float, rows=None):
    """SAS training forward, eq. 9, materialised.

    Q [B,Hq,T,d], K/V [B,Hkv,T,d], logG [B,Hkv,T,NB], tau/tau_idx [B,Hkv,T].
    Returns O [B,Hq,R,d] and LSE [B,Hq,R] (natural log) for the query positions
    ``rows`` (default: all T, R = T).
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    mask = selection_mask(logG, tau, tau_idx, block)
    lg = _f64(logG)
    O = np.zeros((B, Hq, len(rows), d))
    LSE = np.zeros((B, Hq, len(rows)))
    for b in range(B):
        for h in range(Hq):
            g = _group_of(h, Hq, Hkv)
            z = sm_scale * (Q[b, h, rows] @ K[b, g].T) + bias_rows(lg[b, g], mask[b, g], rows, T, block)
            mx = z.max(axis=1, keepdims=True)
            e = np.exp(z - mx)
            l = e.sum(axis=1, keepdims=True)
            P = e / l
            O[b, h] = P @ V[b, g]
            LSE[b, h] = (mx + np.log(l))[:, 0]
    return O, LSE


def forward_backward(Q, K, V, dO, logG, tau, tau_idx, block: int, sm_scale: float, rows=None):
    """Forward plus the gradients of L = sum(O * dO), materialised.

    Backward as in SAS paper Appendix E "Backward pass" (recompute P from the
    logits, Delta = rowsum(O * dO), dS = P * (dP - Delta)), with the block-level
    gate gradient dLogG[t, m] = sum over the group's heads and the tokens of
    block m of dS, for selected m (zero elsewhere; Appendix D.3, dg = 0 off the
    selection).  dQ = sm_scale dS K, dK = sm_scale dS^T Q, dV = P^T dO; dK and
    dV are summed over the query heads of each KV group (GQA).

    With ``rows`` given, O/LSE/dQ/dLogG are for those positions only and dK/dV
    hold the contributions of those query positions only.
    Returns dict with O, LSE, dQ, dK, dV, dLogG (dLogG is [B,Hkv,R,NB]).
    """
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    NB = _f64(logG).shape[-1]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    R = len(rows)
    mask = selection_mask(logG, tau, tau_idx, block)
    lg = _f64(logG)
    out = {
        "O": np.zeros((B, Hq, R, d)), "LSE": np.zeros((B, Hq, R)),
        "dQ": np.zeros((B, Hq, R, d)), "dK": np.zeros((B, Hkv, T, d)),
        "dV": np.zeros((B, Hkv, T, d)), "dLogG": np.zeros((B, Hkv, R, NB)),
    }
    key_block = np.arange(T) // block
    for b in range(B):
        for h in range(Hq):
            g = _group_of(h, Hq, Hkv)
            z = sm_scale * (Q[b, h, rows] @ K[b, g].T) + bias_rows(lg[b, g], mask[b, g], rows, T, block)
            mx = z.max(axis=1, keepdims=True)
            e = np.exp(z - mx)
            l = e.sum(axis=1, keepdims=True)
            P = e / l
            O = P @ V[b, g]
            dP = dO[b, h, rows] @ V[b, g].T
            delta = (dO[b, h, rows] * O).sum(axis=1, keepdims=True)
            dS = P * (dP - delta)
            out["O"][b, h] = O
            out["LSE"][b, h] = (mx + np.log(l))[:, 0]
            out["dQ"][b, h] = sm_scale * (dS @ K[b, g])
            out["dK"][b, g] += sm_scale * (dS.T @ Q[b, h, rows])
            out["dV"][b, g] += P.T @ dO[b, h, rows]
            # Per-block sums of dS over the tokens of each block.
            blk_sum = np.zeros((R, NB))
            for m in range(NB):
                cols = key_block == m
                if cols.any():
                    blk_sum[:, m] = dS[:, cols].sum(axis=1)
            out["dLogG"][b, g] += np.where(mask[b, g][rows], blk_sum, 0.0)
    return out


# --------------------------------------------------------------------------------------
# Variable-length packing (SAS paper §5.1 training on packed sequences, and the
# packing used for the long-context selector training in its appendix): several
# documents share one sequence axis. A document never sees another: it is its own
# causal sequence whose blocks start at its first token (every document starts on a
# block boundary), so the packed problem is the independent problems of its
# documents. In the packed score and gate tensors, document i's rows are its token
# range and its blocks are the columns of its own block range.
# --------------------------------------------------------------------------------------
def doc_slices(cu_seqlens, block: int):
    """(token slice, block slice) per document; cu_seqlens: ascending multiples of block from 0 to T."""
    cu = [int(x) for x in cu_seqlens]
    assert cu[0] == 0 and all(b > a for a, b in zip(cu, cu[1:])) and all(x % block == 0 for x in cu)
    return [(slice(a, b), slice(a // block, b // block)) for a, b in zip(cu, cu[1:])]


def gate_normalize_varlen(s, cu_seqlens, block: int):
    """Packed logG: each document's gate_normalize on its own rows and block columns, -inf elsewhere."""
    s = _f64(s)
    out = np.full(s.shape, -np.inf)
    for ts, bs in doc_slices(cu_seqlens, block):
        out[:, :, ts, bs] = gate_normalize(s[:, :, ts, bs], block)
    return out


def selection_mask_varlen(logG, K: int, cu_seqlens, block: int):
    """Packed boolean [B,Hkv,T,NB]: each document's Top-(K-1) selection (select_threshold on its own gates)."""
    lg = _f64(logG)
    mask = np.zeros(lg.shape, dtype=bool)
    for ts, bs in doc_slices(cu_seqlens, block):
        part = lg[:, :, ts, bs]
        tau, tidx, _ = select_threshold(part, K, block)
        mask[:, :, ts, bs] = selection_mask(part, tau, tidx, block)
    return mask


def forward_backward_varlen(Q, K, V, dO, logG, Kbudget: int, cu_seqlens, block: int, sm_scale: float):
    """forward_backward of every document on its own (its gates, its Top-(K-1)), assembled on the packed axis."""
    Q, K, V, dO, lg = _f64(Q), _f64(K), _f64(V), _f64(dO), _f64(logG)
    B, Hq, T, d = Q.shape
    Hkv, NB = K.shape[1], lg.shape[-1]
    out = {"O": np.zeros((B, Hq, T, d)), "LSE": np.zeros((B, Hq, T)), "dQ": np.zeros((B, Hq, T, d)),
           "dK": np.zeros((B, Hkv, T, d)), "dV": np.zeros((B, Hkv, T, d)), "dLogG": np.zeros((B, Hkv, T, NB))}
    for ts, bs in doc_slices(cu_seqlens, block):
        part = lg[:, :, ts, bs]
        tau, tidx, _ = select_threshold(part, Kbudget, block)
        r = forward_backward(Q[:, :, ts], K[:, :, ts], V[:, :, ts], dO[:, :, ts], part, tau, tidx, block, sm_scale)
        for k in ("O", "LSE", "dQ", "dK", "dV"):
            out[k][:, :, ts] = r[k]
        out["dLogG"][:, :, ts, bs] = r["dLogG"]
    return out


# --------------------------------------------------------------------------------------
# The same eq. 9 evaluated the gathered way: per query row, collect the attended
# token set S = B_0 ∪ selected blocks and run softmax(q K_S^T + log g_S) V_S on
# that subset only.  Used for sampled checks at full size, where the dense
# [T, T] matrix is too large.
# --------------------------------------------------------------------------------------
def attended_keys(t: int, sel_row, block: int):
    """Token indices and per-token log-gate positions for row t: own block keys
    [c*block, t] first, then the selected historical blocks in ascending order."""
    c = t // block
    own = np.arange(c * block, t + 1)
    hist_blocks = [int(m) for m in sel_row if m >= 0]
    hist = np.concatenate([np.arange(m * block, (m + 1) * block) for m in hist_blocks]) if hist_blocks else np.zeros(0, int)
    return own, hist, hist_blocks


def rows_gathered(Q, K, V, dO, logG, sel, b: int, g: int, rows, block: int, sm_scale: float):
    """Per-row O, LSE, dQ (all heads of group g) and dLogG for positions ``rows`` of (b, g).

    ``sel`` [B,Hkv,T,H] holds the selected block indices (from ``select_threshold``).
    Returns dict: O [G,R,d], LSE [G,R], dQ [G,R,d], dLogG [R,NB].
    """
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    lg = _f64(logG)
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    NB = lg.shape[-1]
    R = len(rows)
    res = {"O": np.zeros((G, R, d)), "LSE": np.zeros((G, R)), "dQ": np.zeros((G, R, d)),
           "dLogG": np.zeros((R, NB))}
    for ri, t in enumerate(rows):
        own, hist, hist_blocks = attended_keys(int(t), sel[b, g, t], block)
        idx = np.concatenate([own, hist]).astype(int)
        gate = np.concatenate([np.zeros(len(own)), np.repeat([lg[b, g, t, m] for m in hist_blocks], block)])
        Ks, Vs = K[b, g, idx], V[b, g, idx]
        for hh in range(G):
            h = g * G + hh
            z = sm_scale * (Ks @ Q[b, h, t]) + gate
            mx = z.max()
            e = np.exp(z - mx)
            p = e / e.sum()
            o = p @ Vs
            ds = p * (Vs @ dO[b, h, t] - dO[b, h, t] @ o)
            res["O"][hh, ri] = o
            res["LSE"][hh, ri] = mx + math.log(e.sum())
            res["dQ"][hh, ri] = sm_scale * (ds @ Ks)
            for k, m in enumerate(hist_blocks):
                lo = len(own) + k * block
                res["dLogG"][ri, m] += ds[lo:lo + block].sum()
    return res


def kv_block_gathered(Q, K, V, dO, logG, sel, b: int, g: int, j: int, block: int, sm_scale: float):
    """dK and dV for the keys of block j of (b, g), gathered over every query row that attends it.

    A row t attends block j if j is its current block (keys <= t) or j is selected for t.
    Returns (dK [block, d], dV [block, d]).
    """
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    lg = _f64(logG)
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    dK = np.zeros((block, d))
    dV = np.zeros((block, d))
    for t in range(j * block, T):
        row_sel = sel[b, g, t]
        if t // block != j and j not in set(int(m) for m in row_sel):
            continue
        own, hist, hist_blocks = attended_keys(t, row_sel, block)
        idx = np.concatenate([own, hist]).astype(int)
        gate = np.concatenate([np.zeros(len(own)), np.repeat([lg[b, g, t, m] for m in hist_blocks], block)])
        Ks, Vs = K[b, g, idx], V[b, g, idx]
        in_j = (idx // block) == j
        for hh in range(G):
            h = g * G + hh
            z = sm_scale * (Ks @ Q[b, h, t]) + gate
            e = np.exp(z - z.max())
            p = e / e.sum()
            o = p @ Vs
            ds = p * (Vs @ dO[b, h, t] - dO[b, h, t] @ o)
            kpos = idx[in_j] - j * block
            dK[kpos] += sm_scale * np.outer(ds[in_j], Q[b, h, t])
            dV[kpos] += np.outer(p[in_j], dO[b, h, t])
    return dK, dV


# --------------------------------------------------------------------------------------
# Decode: SAS paper §4.3 Algorithm 2 (inference step): I = Top-K(s), S = B_0 ∪ I,
# o = softmax(q K_S^T) V_S, with no gate; and §5.1 "Inference implementation"
# (per-group selection over cached blocks, GQA).
# --------------------------------------------------------------------------------------
def decode(q, Kc, Vc, seqlen, s, K: int, block: int, sm_scale: float, apply_log_gate: bool = False):
    """One decode step per sequence.

    q [B,Hq,d]; Kc/Vc [B,Hkv,Lmax,d]; seqlen [B] (the new token included, at
    position L-1); s [B,Hkv,NBmax] selector scores.  The current block is
    c = (L-1) // block; Top-(K-1) of blocks 0..c-1 by s (ties to the lower
    index) plus block c (positions c*block .. L-1) are attended.  With
    ``apply_log_gate`` the selected blocks also get log g = s - LSE(s[:c]).
    Returns (o [B,Hq,d], sel [B,Hkv,K-1] ascending, -1 padded).
    """
    q, Kc, Vc, sv = _f64(q), _f64(Kc), _f64(Vc), _f64(s)
    B, Hq, d = q.shape
    Hkv = Kc.shape[1]
    G = Hq // Hkv
    H = K - 1
    o = np.zeros((B, Hq, d))
    sel = np.full((B, Hkv, max(H, 0)), -1, dtype=np.int32)
    for b in range(B):
        L = int(seqlen[b])
        c = (L - 1) // block
        for g in range(Hkv):
            _, _, chosen = topk_threshold_row(sv[b, g], c, H)
            sel[b, g, : len(chosen)] = chosen
            own = np.arange(c * block, L)
            hist = np.concatenate([np.arange(m * block, (m + 1) * block) for m in chosen]) if chosen else np.zeros(0, int)
            idx = np.concatenate([own, hist]).astype(int)
            bias = np.zeros(len(idx))
            if apply_log_gate and c > 0:
                hs = sv[b, g, :c]
                lse = hs.max() + math.log(np.exp(hs - hs.max()).sum())
                bias[len(own):] = np.repeat([sv[b, g, m] - lse for m in chosen], block)
            for hh in range(G):
                h = g * G + hh
                z = sm_scale * (Kc[b, g, idx] @ q[b, h]) + bias
                e = np.exp(z - z.max())
                o[b, h] = (e / e.sum()) @ Vc[b, g, idx]
    return o, sel


def paged_cache(pool, page_table, block: int):
    """Logical KV cache [B, Hkv, max_pages*block, d] of a paged pool.

    pool [num_pages, Hkv, block, d] holds one block of ``block`` tokens of every
    KV head per page; page_table [B, max_pages] names, for each sequence and
    logical block m, the page holding its tokens m*block .. m*block+block-1
    (-1 for blocks the sequence does not reach; they read as zeros and are never
    attended). Plain gather, one page at a time.
    """
    pool = _f64(pool)
    num_pages, Hkv, bl, d = pool.shape
    assert bl == block
    B, max_pages = page_table.shape
    out = np.zeros((B, Hkv, max_pages * block, d))
    for b in range(B):
        for m in range(max_pages):
            pg = int(page_table[b, m])
            if pg >= 0:
                out[b, :, m * block:(m + 1) * block] = pool[pg]
    return out


def decode_paged(q, Kpool, Vpool, page_table, seqlen, s, K: int, block: int, sm_scale: float,
                 apply_log_gate: bool = False):
    """The decode step of ``decode`` over a paged KV cache (pages of one block).

    The paged layout only changes where a token's key and value are stored, not
    what is computed (§5.1 "Inference implementation": only the selected KV
    blocks are gathered), so this is ``decode`` on the logical cache that
    ``paged_cache`` rebuilds.
    """
    return decode(q, paged_cache(Kpool, page_table, block), paged_cache(Vpool, page_table, block), seqlen, s, K,
                  block, sm_scale, apply_log_gate)
