"""Plain fp64 CPU oracle for block-sparse prefill attention with block routing.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code, header,
table or constant with the CUDA library; the only thing both sides share is
the seeded input generator, which holds none of the method's arithmetic.

Every function below restates one step of the method as the source pages
describe it, in float64, with no blocking, fusion or reordering beyond what
the step itself states.  Library primitives used as steps: ``numpy`` matmul,
``numpy.lexsort`` (for the stable top-k order), ``numpy.exp`` / ``numpy.log``.

Sources (web pages; cited by title and section):

* PISA summary -- "PISA (Piecewise Sparse Attention)" blog post
  (kodorricoding.tistory.com/108):
    - section "How are candidate blocks narrowed": per block, a representative
      query and key and the SUM of the values; a per-query-block score picks
      the key blocks of the exact path (top-k by ``density``);
    - the routing table ("A,B exact with the original K/V tokens; C,D
      approximated by the block-mean key and the value sum");
    - section "Why approximating unselected blocks keeps softmax intact":
      exact terms and approximate terms go into ONE softmax accumulation, the
      0th-order term is taken around the block-mean key;
    - section "Minimal usage": ``f(q, k, v, density=0.15, block_size=64)``.
* FlashPrefill summary -- "FlashPrefill: Instantaneous Pattern Discovery and
  Thresholding for Ultra-Fast Long-Context Prefilling" (gist.science):
    - section 2.a "Block approximation": average-pooled key blocks;
    - section 2.b "Max-based dynamic thresholding":
      thresh_I = alpha * max_J Score_{I,J}, no sort.
* FlashAttention blog -- "Flash attention: IO-aware attention"
  (blog.mna-game.duckdns.org): section 1 (naive attention materialises
  S = Q K^T, softmax, times V) and section 2 (online softmax recurrence
  m <- max(m, max z), l <- l e^{m_old-m} + sum e^{z-m},
  o <- o e^{m_old-m} + sum e^{z-m} v, answer o / l).

Readings where the pages are silent:

* layout ``[B, H, N, d]``; block I = tokens [I*b, (I+1)*b); ``N % b == 0``;
* q-bar and k-bar are means, the value statistic is the plain sum;
* block score s_IJ = q-bar_I . k-bar_J / sqrt(d) (fp64 here);
* top-k: k = clamp(ceil(fl32(density * M)), 1, #candidates), where fl32 is the
  IEEE single-precision product of the float32 density and M; ties go to the
  smaller J; the kept list is ascending; in causal mode one of the k slots is
  the diagonal block (the causal mask is applied exactly, token by token, so
  the diagonal block is always on the exact path) and the other k-1 are the
  best of the blocks J < I;
* threshold: keep J iff s_IJ >= alpha * max_J' s_IJ' over the candidates,
  plus the diagonal block I, plus block 0 when ``keep_first``;
* threshold, probability reading (``route_thresh_prob``): the "attention
  score" of the rule taken as the softmax of the row's block scores, which
  makes it s_IJ >= max_J' s_IJ' + ln(alpha), same forced blocks;
* causal: candidates are J <= I; inside the diagonal block key j is visible to
  query i iff j <= i; blocks J > I contribute nothing, not even their 0th
  order term; the diagonal block never gets a 0th-order term (its pooled key
  contains future tokens): it counts only when listed, and both routers
  always list it;
* each candidate block counts once: exact if listed, else 0th-order;
* the 0th-order term of an unselected block J for query i is
  exp(a_iJ) * (b for the denominator, sum_j v_j for the numerator), with
  a_iJ = q_i . k-bar_J / sqrt(d).

* first-order term (``attention_first_order``, oracle only so far): the
  expansion of e^{q.k_j/sqrt(d)} to first order around the block-mean key;
  the pages' "global statistic H" is read as the mean over the head's blocks
  of the per-block matrices H_J = sum_j (k_j - kbar_J) v_j^T;
* FlashPrefill's fused "score then pool" block score (the token queries of
  block I against the pooled key of block J, reduced over I in one pass,
  ``token_pooled_block_scores``) is read with mean pooling, which makes it
  equal to qbar_I . kbar_J / sqrt(d) by linearity.

Parity of the approximate output to the authors' own implementation is
unpinned (no page prints a worked PISA example); the oracle is pinned to the
definitions above by the tests in ``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "pool",
    "block_scores",
    "candidate_count",
    "topk_count",
    "route_topk",
    "route_thresh",
    "route_thresh_prob",
    "attention",
    "attention_online",
    "unit_rows",
    "block_deviation_stats",
    "global_deviation_stat",
    "attention_first_order",
    "token_pooled_block_scores",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# a1. Pooling  [PISA summary, "How are candidate blocks narrowed";
#               FlashPrefill summary, 2.a "Block approximation"]
# --------------------------------------------------------------------------
def pool(q, k, v, block_size: int = 64):
    """Per-block statistics of the three inputs.

    Returns ``(qbar, kbar, vsum)``, each ``[B, H, M, d]`` float64:
    ``qbar`` and ``kbar`` are the means over the ``block_size`` tokens of a
    block, ``vsum`` is the plain sum of the value rows of the block.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    if N % block_size:
        raise ValueError("N must be a multiple of block_size")
    M = N // block_size
    qbar = q.reshape(B, H, M, block_size, d).mean(axis=3)
    kbar = k.reshape(B, H, M, block_size, d).mean(axis=3)
    vsum = v.reshape(B, H, M, block_size, d).sum(axis=3)
    return qbar, kbar, vsum


# --------------------------------------------------------------------------
# a2. Block scores  [PISA summary, "How are candidate blocks narrowed"]
# --------------------------------------------------------------------------
def block_scores(qbar, kbar):
    """s[b, h, I, J] = qbar_I . kbar_J / sqrt(d), float64, all pairs."""
    qbar, kbar = _f64(qbar), _f64(kbar)
    d = qbar.shape[-1]
    return np.matmul(qbar, np.swapaxes(kbar, -1, -2)) / math.sqrt(d)


def candidate_count(I: int, M: int, causal: bool) -> int:
    """Number of candidate key blocks of query block I (J <= I when causal)."""
    return I + 1 if causal else M


def topk_count(density: float, M: int, n_cand: int) -> int:
    """k = clamp(ceil(fl32(density * M)), 1, n_cand)  [PISA summary, usage:
    ``density`` is the ratio of the exact path]."""
    prod = np.float32(density) * np.float32(M)  # IEEE single-precision product
    k = int(math.ceil(float(prod)))
    return max(1, min(k, n_cand))


def _to_csr(lists):
    row_ptr = np.zeros(len(lists) + 1, dtype=np.int64)
    for r, lst in enumerate(lists):
        row_ptr[r + 1] = row_ptr[r] + len(lst)
    col_idx = np.concatenate([np.asarray(lst, dtype=np.int64) for lst in lists]) \
        if lists else np.zeros(0, dtype=np.int64)
    return row_ptr, col_idx


# --------------------------------------------------------------------------
# a3. Top-k routing  [PISA summary, "How are candidate blocks narrowed";
#                     usage line ``density=0.15``]
# --------------------------------------------------------------------------
def route_topk(s, density: float, causal: bool):
    """Per query block, keep the k highest-scoring candidate key blocks
    (causal: the diagonal block plus the k-1 best blocks J < I).

    ``s`` is ``[B, H, M, M]``.  Rows are ordered (b, h, I) row-major.
    Returns ``(row_ptr, col_idx)`` int64 with each row's list ascending.
    """
    s = _f64(s)
    B, H, M, _ = s.shape
    lists = []
    for b in range(B):
        for h in range(H):
            for I in range(M):
                n_cand = candidate_count(I, M, causal)
                k = topk_count(density, M, n_cand)
                if causal:
                    # the diagonal takes one slot; the rest come from J < I
                    forced, pool_n, k_rest = [I], I, k - 1
                else:
                    forced, pool_n, k_rest = [], n_cand, k
                J = np.arange(pool_n)
                vals = s[b, h, I, :pool_n]
                # primary key: score descending; secondary: J ascending
                order = np.lexsort((J, -vals))
                lists.append(np.sort(np.concatenate(
                    [J[order[:k_rest]], np.asarray(forced, dtype=np.int64)])))
    return _to_csr(lists)


# --------------------------------------------------------------------------
# a4. Threshold routing  [FlashPrefill summary, 2.b "Max-based dynamic
#                         thresholding": thresh_I = alpha * max_J Score_IJ]
# --------------------------------------------------------------------------
def route_thresh(s, alpha: float, causal: bool, keep_first: bool):
    """Keep J iff s_IJ >= alpha * max over candidates, plus the diagonal block
    I, plus block 0 when ``keep_first``.  Lists ascending."""
    s = _f64(s)
    B, H, M, _ = s.shape
    alpha = float(np.float32(alpha))
    lists = []
    for b in range(B):
        for h in range(H):
            for I in range(M):
                n_cand = candidate_count(I, M, causal)
                vals = s[b, h, I, :n_cand]
                thresh = alpha * vals.max()
                keep = vals >= thresh
                keep[min(I, n_cand - 1)] = True   # diagonal block (I < M always)
                if keep_first:
                    keep[0] = True
                lists.append(np.nonzero(keep)[0])
    return _to_csr(lists)


def route_thresh_prob(s, alpha: float, causal: bool, keep_first: bool):
    """The same max-based rule read in the probability domain (FlashPrefill
    summary, 2.b "Max-based dynamic thresholding", with the block attention
    score taken as the softmax of the row's block scores): keep J iff
    p_IJ >= alpha * max_J p_IJ, where p_IJ = e^{s_IJ} / sum over the candidates.
    The normaliser cancels in the ratio, so this is s_IJ >= max_J s_IJ + ln(alpha),
    evaluated here in that form; plus the diagonal block I, plus block 0 when
    ``keep_first``.  alpha > 0.  Lists ascending."""
    s = _f64(s)
    B, H, M, _ = s.shape
    alpha = float(np.float32(alpha))
    if not alpha > 0:
        raise ValueError("alpha must be positive")
    log_alpha = math.log(alpha)
    lists = []
    for b in range(B):
        for h in range(H):
            for I in range(M):
                n_cand = candidate_count(I, M, causal)
                vals = s[b, h, I, :n_cand]
                keep = vals >= vals.max() + log_alpha
                keep[min(I, n_cand - 1)] = True
                if keep_first:
                    keep[0] = True
                lists.append(np.nonzero(keep)[0])
    return _to_csr(lists)


def unit_rows(B: int, H: int, M: int):
    """All (b, h, I) triples in CSR row order."""
    return [(b, h, I) for b in range(B) for h in range(H) for I in range(M)]


def _unit_terms(q, k, v, kbar, vsum, sel, b, h, I, causal, block_size):
    """Logits and values of every term query block I sees.

    Returns ``(z, Vx, a, VS)``: exact logits ``z`` [b, n_exact] with masked
    entries at -inf, their value rows ``Vx`` [n_exact, d], pseudo logits
    ``a`` [b, n_unsel] of the unselected candidates and their value sums
    ``VS`` [n_unsel, d].
    """
    bs = block_size
    M = q.shape[2] // bs
    d = q.shape[3]
    tau = 1.0 / math.sqrt(d)
    n_cand = candidate_count(I, M, causal)
    sel = np.asarray(sel, dtype=np.int64)
    if sel.size:
        if sel.min() < 0 or sel.max() >= n_cand:
            raise ValueError(f"block list of row ({b},{h},{I}) leaves the candidates")
        if np.unique(sel).size != sel.size:
            raise ValueError(f"block list of row ({b},{h},{I}) repeats a block")
    Qi = q[b, h, I * bs:(I + 1) * bs]                       # [bs, d]
    tok = (sel[:, None] * bs + np.arange(bs)[None, :]).reshape(-1)
    Kx = k[b, h, tok]                                       # [n_exact, d]
    Vx = v[b, h, tok]
    z = tau * (Qi @ Kx.T)                                   # [bs, n_exact]
    if causal:
        # inside the diagonal block, key j is visible to query i iff j <= i
        qi = np.arange(bs)[:, None] + I * bs
        z = np.where(tok[None, :] <= qi, z, -np.inf)
    # 0th-order candidates: every unlisted candidate, except that a causal
    # diagonal block is never approximated
    n_pseudo = I if causal else n_cand
    unsel = np.setdiff1d(np.arange(n_pseudo), sel)
    a = tau * (Qi @ kbar[b, h, unsel].T)                    # [bs, n_unsel]
    VS = vsum[b, h, unsel]
    return z, Vx, a, VS


# --------------------------------------------------------------------------
# a5-a7. Exact + 0th-order attention, one softmax, two-pass
#   [PISA summary, routing table and "Why approximating unselected blocks
#    keeps softmax intact"; FlashAttention blog section 1 for the softmax]
# --------------------------------------------------------------------------
def attention(q, k, v, kbar, vsum, row_ptr, col_idx, causal: bool,
              block_size: int = 64, units=None):
    """PISA 0th-order output for the query blocks in ``units``.

    For query i of block I, with S_I the listed blocks and U_I the other
    candidates:
      num_i = sum_{J in S_I} sum_{j in J, visible} e^{z_ij - m_i} v_j
              + sum_{J in U_I} e^{a_iJ - m_i} vsum_J
      den_i = sum_{J in S_I} sum_{j in J, visible} e^{z_ij - m_i}
              + sum_{J in U_I} block_size * e^{a_iJ - m_i}
      out_i = num_i / den_i,  lse_i = m_i + ln den_i,
    with z_ij = q_i.k_j/sqrt(d), a_iJ = q_i.kbar_J/sqrt(d) and m_i the largest
    of all those logits (a full max first, then the sums: two passes).

    ``units`` is an iterable of (b, h, I); ``None`` means all.  Returns
    ``(out, lse)`` of shapes ``[n_units, block_size, d]`` and
    ``[n_units, block_size]`` in the order of ``units``.
    """
    q, k, v, kbar, vsum = map(_f64, (q, k, v, kbar, vsum))
    B, H, N, d = q.shape
    bs = block_size
    M = N // bs
    if units is None:
        units = unit_rows(B, H, M)
    units = list(units)
    out = np.empty((len(units), bs, d))
    lse = np.empty((len(units), bs))
    for n, (b, h, I) in enumerate(units):
        r = (b * H + h) * M + I
        sel = col_idx[row_ptr[r]:row_ptr[r + 1]]
        z, Vx, a, VS = _unit_terms(q, k, v, kbar, vsum, sel, b, h, I, causal, bs)
        # pass 1: the row maximum over every logit the query sees
        m = np.full(bs, -np.inf)
        if z.shape[1]:
            m = np.maximum(m, z.max(axis=1))
        if a.shape[1]:
            m = np.maximum(m, a.max(axis=1))
        # pass 2: numerator and denominator
        ez = np.exp(z - m[:, None])
        ea = np.exp(a - m[:, None])
        num = ez @ Vx + ea @ VS
        den = ez.sum(axis=1) + bs * ea.sum(axis=1)
        out[n] = num / den[:, None]
        lse[n] = m + np.log(den)
    return out, lse


def attention_online(q, k, v, kbar, vsum, row_ptr, col_idx, causal: bool,
                     block_size: int = 64, units=None):
    """Same output as :func:`attention`, folded one block at a time with the
    online-softmax recurrence of the FlashAttention blog (section 2): the
    exact blocks in list order, then the unselected candidates one by one,
    each as a pseudo-key of log-weight a + ln(block_size) and value
    vsum / block_size.  Used only to pin the online fold against the
    two-pass form."""
    q, k, v, kbar, vsum = map(_f64, (q, k, v, kbar, vsum))
    B, H, N, d = q.shape
    bs = block_size
    M = N // bs
    if units is None:
        units = unit_rows(B, H, M)
    units = list(units)
    out = np.empty((len(units), bs, d))
    lse = np.empty((len(units), bs))
    for n, (b, h, I) in enumerate(units):
        r = (b * H + h) * M + I
        sel = col_idx[row_ptr[r]:row_ptr[r + 1]]
        z, Vx, a, VS = _unit_terms(q, k, v, kbar, vsum, sel, b, h, I, causal, bs)
        pieces = [(z[:, j * bs:(j + 1) * bs], Vx[j * bs:(j + 1) * bs])
                  for j in range(len(sel))]
        pieces += [(a[:, u:u + 1] + math.log(bs), VS[u:u + 1] / bs)
                   for u in range(a.shape[1])]
        m = np.full(bs, -np.inf)
        l = np.zeros(bs)
        o = np.zeros((bs, d))
        for zz, vv in pieces:
            m_new = np.maximum(m, zz.max(axis=1))
            corr = np.exp(m - m_new)
            p = np.exp(zz - m_new[:, None])
            l = l * corr + p.sum(axis=1)
            o = o * corr[:, None] + p @ vv
            m = m_new
        out[n] = o / l[:, None]
        lse[n] = m + np.log(l)
    return out, lse


# --------------------------------------------------------------------------
# f-1. First-order term of the unselected blocks
#   [PISA summary, "Why approximating unselected blocks keeps softmax intact":
#    to the 0th-order term around the block-mean key a first-order
#    correction with a global statistic H is added; FAQ "Why a global
#    first-order correction?": one global statistic instead of re-reading a
#    large matrix per block]
# --------------------------------------------------------------------------
def block_deviation_stats(k, v, block_size: int = 64):
    """H_J = sum_{j in J} (k_j - kbar_J) v_j^T for every block J.

    Returns ``[B, H, M, d, d]`` float64 (rows: key features, columns: value
    features)."""
    k, v = _f64(k), _f64(v)
    B, H, N, d = k.shape
    if N % block_size:
        raise ValueError("N must be a multiple of block_size")
    M = N // block_size
    kb = k.reshape(B, H, M, block_size, d)
    vb = v.reshape(B, H, M, block_size, d)
    dev = kb - kb.mean(axis=3, keepdims=True)
    return np.einsum("bhmtk,bhmtv->bhmkv", dev, vb)


def global_deviation_stat(HJ):
    """The global statistic, read as the mean of H_J over a head's blocks:
    ``[B, H, d, d]``."""
    return _f64(HJ).mean(axis=2)


def _first_order_numerator(ea, Qi, Hs, d):
    """sum_J e^{a_iJ - m_i} (H_J^T q_i) / sqrt(d) for the query rows ``Qi``
    [b, d], the weights ``ea`` [b, n_unsel] and the statistics ``Hs``
    [n_unsel, d, d] of the unselected blocks."""
    return np.einsum("iJ,ik,Jkv->iv", ea, Qi, Hs) / math.sqrt(d)


def attention_first_order(q, k, v, kbar, vsum, row_ptr, col_idx, causal: bool, Hstat,
                          block_size: int = 64, units=None):
    """The 0th-order output of :func:`attention` with the first-order term of
    every unselected block added.

    To first order around the block-mean key,
      e^{q.k_j/sqrt(d)} ~= e^{a_J} (1 + q.(k_j - kbar_J)/sqrt(d)),
    and the deviations k_j - kbar_J sum to zero over the block, so the
    denominator term stays block_size * e^{a_J} while the numerator term
    becomes e^{a_J} (vsum_J + H_J^T q / sqrt(d)).  ``Hstat`` is either the
    per-block ``[B, H, M, d, d]`` of :func:`block_deviation_stats` (the
    expansion itself) or one ``[B, H, d, d]`` matrix per head used for every
    block (the global statistic).  Same max and shapes as :func:`attention`.
    """
    q, k, v, kbar, vsum, Hstat = map(_f64, (q, k, v, kbar, vsum, Hstat))
    B, H, N, d = q.shape
    bs = block_size
    M = N // bs
    per_block = Hstat.ndim == 5
    if units is None:
        units = unit_rows(B, H, M)
    units = list(units)
    out = np.empty((len(units), bs, d))
    lse = np.empty((len(units), bs))
    for n, (b, h, I) in enumerate(units):
        r = (b * H + h) * M + I
        sel = col_idx[row_ptr[r]:row_ptr[r + 1]]
        z, Vx, a, VS = _unit_terms(q, k, v, kbar, vsum, sel, b, h, I, causal, bs)
        n_pseudo = I if causal else candidate_count(I, M, causal)
        unsel = np.setdiff1d(np.arange(n_pseudo), np.asarray(sel, dtype=np.int64))
        m = np.full(bs, -np.inf)
        if z.shape[1]:
            m = np.maximum(m, z.max(axis=1))
        if a.shape[1]:
            m = np.maximum(m, a.max(axis=1))
        ez = np.exp(z - m[:, None])
        ea = np.exp(a - m[:, None])
        Qi = q[b, h, I * bs:(I + 1) * bs]
        Hs = Hstat[b, h, unsel] if per_block else np.broadcast_to(Hstat[b, h], (unsel.size, d, d))
        num = ez @ Vx + ea @ VS + _first_order_numerator(ea, Qi, Hs, d)
        den = ez.sum(axis=1) + bs * ea.sum(axis=1)
        out[n] = num / den[:, None]
        lse[n] = m + np.log(den)
    return out, lse


# --------------------------------------------------------------------------
# FlashPrefill's fused scoring, read with mean pooling
#   [FlashPrefill summary, 2.a "Block approximation": average-pooled keys as
#    block representatives; a fused 2D-reduction kernel replaces an explicit
#    compute-then-pool pass]
# --------------------------------------------------------------------------
def token_pooled_block_scores(q, kbar, block_size: int = 64):
    """score[b, h, I, J] = mean over the tokens i of query block I of
    q_i . kbar_J / sqrt(d): the token-level scores against the pooled keys,
    pooled over the query block."""
    q, kbar = _f64(q), _f64(kbar)
    B, H, N, d = q.shape
    M = N // block_size
    tok = np.matmul(q, np.swapaxes(kbar, -1, -2)) / math.sqrt(d)   # [B, H, N, M]
    return tok.reshape(B, H, M, block_size, kbar.shape[2]).mean(axis=3)

