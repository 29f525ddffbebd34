"""Float64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this module: only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg use it.  It shares no code with the CUDA library.

Every function here is the plain definition, written out in float64 with the
full score matrix materialised, so a reader can check it against the pages by
eye.  Sources (web pages, cited by title and section):

* "Building Flash Attention from Scratch in Pure NumPy" -- Step 1 (the naive
  reference oracle and its stable softmax), Step 2 (the online-softmax update),
  Step 4 (the backward pass: D = rowsum(dO * O) and the per-tile recompute of P
  from the saved statistics), and the architecture overview's merge identity
  for two partial softmaxes.
* "Build a FlashAttention-2 Inference Kernel from Scratch in Pure Python" --
  Step 2 (scale, then set masked scores to -inf, then softmax) and Step 3 (the
  causal mask j <= i and the sliding-window "block-sparse" restriction).
* "Build a FlashAttention Kernel with Online Softmax and KV Cache in Pure
  Python" -- Steps 2-5 (single-query decode against a cache that already holds
  the current token; naive single-query reference).
* The same two pages' "Extending It" roadmaps (distributed tensor
  parallelism; horizontal scaling with each worker holding part of the
  key/value space): the per-shard partial forward of
  :func:`attention_forward_offset`, combined with :func:`merge_partials`.
* "FlashAttention Algorithm > Worked Example" -- the n=8, d=4, block 4 trace
  (Steps 1-3) that pins :func:`online_softmax_forward` and
  :func:`attention_forward`.

Readings where the pages are silent, buggy or garbled (each one is listed in
the design notes as well):

* mask: key j is allowed for query i iff (not causal or j <= i) and
  (window <= 0 or j > i - window).  A window therefore holds exactly `window`
  keys including the query itself.  The inference-kernel page's loop keeps
  ``j >= i - sparse_window`` (one key more); the long-context workload's
  definition "i-4096 < j <= i" is followed instead.
* scale: ``scale=None`` (or <= 0) means 1/sqrt(d), as in the NumPy page's
  Step 3 keyword default.  The scale multiplies the raw scores.
* lse: natural-log logsumexp of the scaled, masked scores of a row, i.e.
  ``lse_i = m_i + ln(l_i)`` in the NumPy page's (m, l) notation.  That page's
  forward returns m and l arrays that are never written (a bug); one lse per
  row replaces them.
* fully masked row (no allowed key): O row = 0, lse = -inf, and zero gradient
  flows through it.  The pages' code would produce NaN there.
* backward: the NumPy page's Step 4 marks its dK and dQ lines as simplified
  and wrong.  The oracle uses the analytic gradient of the forward definition
  (dV = P^T dO, dP = dO V^T, dS = P * (dP - D), dQ = scale dS K,
  dK = scale dS^T Q), which is what that page says a correct version must do.
* ragged N: keys past N are excluded from the softmax, never zero-padded into
  it (the NumPy page's Step 3 pads K with zeros, which would add score-0 keys
  to every row when N is not a multiple of the block).

Parity pins: every function is checked in ``tests/test_oracle.py`` against the
worked example's printed values, closed forms, invariants, finite differences
and torch's float64 scaled_dot_product_attention.  No function here is
"parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "allowed_mask",
    "default_scale",
    "attention_scores",
    "attention_probabilities",
    "attention_forward",
    "attention_forward_rows",
    "attention_forward_offset",
    "attention_backward",
    "decode_forward",
    "merge_partials",
    "online_softmax_forward",
]


def _f64(x) -> np.ndarray:
    """Exact upcast to float64 (bf16, fp16 and fp32 values are all exact in f64)."""
    if hasattr(x, "detach"):  # a torch tensor: upcast exactly through float32/float64
        x = x.detach().to("cpu")
        import torch  # local: torch is only needed when the caller passes tensors

        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def default_scale(d: int, scale: float | None) -> float:
    """``scale=None`` (or a non-positive value) means 1/sqrt(d).

    Building Flash Attention from Scratch in Pure NumPy, Step 3: the forward's
    ``scale`` keyword defaults to 1/sqrt(d).
    """
    if scale is None or scale <= 0:
        return 1.0 / math.sqrt(d)
    return float(scale)


def allowed_mask(n_q: int, n_k: int, causal: bool, window: int,
                 q_pos: np.ndarray | None = None) -> np.ndarray:
    """Boolean [n_q, n_k]: may query i attend to key j?

    Build a FlashAttention-2 Inference Kernel from Scratch in Pure Python,
    Step 3: the causal mask forbids j > i; the block-sparse window keeps only
    recent keys.  Reading: j > i - window (exactly `window` keys with the
    query itself), as the long-context workload defines it.

    ``q_pos`` gives each query's absolute position (default 0..n_q-1), so a
    subset of rows can be evaluated on its own.
    """
    i = np.arange(n_q) if q_pos is None else np.asarray(q_pos)
    i = i[:, None]
    j = np.arange(n_k)[None, :]
    ok = np.ones((len(i), n_k), dtype=bool)
    if causal:
        ok &= j <= i
    if window > 0:
        ok &= j > i - window
    return ok


def attention_scores(q, k, scale=None, causal=False, window=0, q_pos=None):
    """Scaled, masked scores S (float64), -inf where masked.

    Building Flash Attention from Scratch in Pure NumPy, Step 1:
    scores = Q K^T / sqrt(d).  Build a FlashAttention-2 Inference Kernel from
    Scratch in Pure Python, Step 2: scale first, then masked scores -> -inf.
    Works on [..., N, d] arrays.
    """
    q = _f64(q)
    k = _f64(k)
    d = q.shape[-1]
    s = default_scale(d, scale)
    S = np.matmul(q, np.swapaxes(k, -1, -2)) * s
    ok = allowed_mask(q.shape[-2], k.shape[-2], causal, window, q_pos)
    return np.where(ok, S, -np.inf)


def _logsumexp_rows(S: np.ndarray) -> np.ndarray:
    """lse_i = max_j S_ij + ln sum_j exp(S_ij - max_j S_ij); -inf for an empty row.

    Building Flash Attention from Scratch in Pure NumPy, Step 1: the stable
    softmax subtracts the row max before exponentiating.
    """
    m = S.max(axis=-1, keepdims=True)
    empty = np.isneginf(m)
    m_safe = np.where(empty, 0.0, m)
    with np.errstate(divide="ignore"):
        lse = m_safe + np.log(np.exp(S - m_safe).sum(axis=-1, keepdims=True))
    lse = np.where(empty, -np.inf, lse)
    return lse[..., 0]


def attention_probabilities(q, k, scale=None, causal=False, window=0, q_pos=None):
    """P = softmax(S) row-wise (zero rows where nothing is allowed), and lse.

    Building Flash Attention from Scratch in Pure NumPy, Step 1 (the stable
    softmax), extended with the mask.
    """
    S = attention_scores(q, k, scale, causal, window, q_pos)
    lse = _logsumexp_rows(S)
    lse_safe = np.where(np.isneginf(lse), 0.0, lse)
    P = np.exp(S - lse_safe[..., None])  # exp(-inf) = 0 on masked entries
    return P, lse


def attention_forward(q, k, v, scale=None, causal=False, window=0):
    """O = softmax(Q K^T * scale + mask) V and the row logsumexp, in float64.

    Building Flash Attention from Scratch in Pure NumPy, Step 1 (the naive
    O(N^2) oracle: weights = stable_softmax(scores); return weights @ V).
    q, k, v: [..., N, d].  Returns (O [..., N, d], lse [..., N]).
    """
    P, lse = attention_probabilities(q, k, scale, causal, window)
    O = np.matmul(P, _f64(v))
    return O, lse


def attention_forward_rows(q, k, v, rows, scale=None, causal=False, window=0):
    """The forward for selected query rows only (each row needs every key).

    Same definition as :func:`attention_forward`, evaluated for ``rows`` of
    one head: q [N, d] (only q[rows] is read), k, v [N, d].  Used to check
    sampled outputs at sizes where the full N x N matrix is too big.
    """
    rows = np.asarray(rows)
    qs = _f64(q)[rows]
    P, lse = attention_probabilities(qs, k, scale, causal, window, q_pos=rows)
    return np.matmul(P, _f64(v)), lse


def attention_backward(q, k, v, dO, scale=None, causal=False, window=0):
    """Analytic gradient of :func:`attention_forward`: (dQ, dK, dV), float64.

    Building Flash Attention from Scratch in Pure NumPy, Step 4: D =
    rowsum(dO * O); P recomputed from the saved statistics; dV = P^T dO.  The
    page's own dK/dQ lines are declared simplified; the correct terms are the
    softmax Jacobian applied to dP = dO V^T:
        dS = P * (dP - D[:, None]),  dQ = scale * dS K,  dK = scale * dS^T Q.
    Fully masked rows have P = 0 and so contribute nothing.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    dO = _f64(dO)
    s = default_scale(q.shape[-1], scale)
    P, _ = attention_probabilities(q, k, s, causal, window)
    O = np.matmul(P, v)
    D = (dO * O).sum(axis=-1)
    dV = np.matmul(np.swapaxes(P, -1, -2), dO)
    dP = np.matmul(dO, np.swapaxes(v, -1, -2))
    dS = P * (dP - D[..., None])
    dQ = s * np.matmul(dS, k)
    dK = s * np.matmul(np.swapaxes(dS, -1, -2), q)
    return dQ, dK, dV


def decode_forward(q, kcache, vcache, seqlens, scale=None):
    """Single-token decode: each (b, h) query attends to cache rows j < seqlens[b].

    Build a FlashAttention Kernel with Online Softmax and KV Cache in Pure
    Python, Steps 4-5: the current token's key/value are already in the cache
    when it is scored, so all cached positions are allowed; the result is the
    naive single-query attention over them.
    q: [B, H, d]; kcache, vcache: [B, H, cap, d]; seqlens: [B] ints.
    Returns (o [B, H, d], lse [B, H]); a zero-length row gives o = 0,
    lse = -inf.
    """
    q = _f64(q)
    B, H, d = q.shape
    seqlens = np.asarray(seqlens).astype(np.int64).reshape(-1)
    s = default_scale(d, scale)
    o = np.zeros((B, H, d))
    lse = np.full((B, H), -np.inf)
    for b in range(B):
        n = int(seqlens[b])
        if n <= 0:
            continue
        kb = _f64(kcache[b, :, :n])  # [H, n, d]
        vb = _f64(vcache[b, :, :n])
        S = np.einsum("hd,hnd->hn", q[b], kb) * s
        lse_b = _logsumexp_rows(S)
        P = np.exp(S - lse_b[:, None])
        o[b] = np.einsum("hn,hnd->hd", P, vb)
        lse[b] = lse_b
    return o, lse


def decode_paged_forward(q, kpool, vpool, block_table, seqlens, scale=None):
    """Single-token decode against a paged cache.

    Build a FlashAttention-2 Inference Kernel from Scratch in Pure Python,
    Extending It (paged KV-cache integration), read as a block pool: key j of
    sequence b, head h is row j mod bs of physical block block_table[b][j // bs]
    of the pool.  Each sequence's keys are gathered in order and then attended
    exactly as decode_forward does (the paging moves rows, not arithmetic).
    kpool, vpool: [num_blocks, H, bs, d]; block_table: [B, max_blocks] ints;
    seqlens: [B], clamped to [0, max_blocks * bs].
    """
    kpool, vpool = _f64(kpool), _f64(vpool)
    table = np.asarray(block_table).astype(np.int64)
    _, H, bs, d = kpool.shape
    B, max_blocks = table.shape
    cap = max_blocks * bs
    n = np.clip(np.asarray(seqlens).astype(np.int64).reshape(-1), 0, cap)
    kc = np.zeros((B, H, cap, d))
    vc = np.zeros((B, H, cap, d))
    for b in range(B):
        for t in range(-(-int(n[b]) // bs)):
            kc[b, :, t * bs:(t + 1) * bs] = kpool[table[b, t]]
            vc[b, :, t * bs:(t + 1) * bs] = vpool[table[b, t]]
    return decode_forward(q, kc, vc, n, scale)


def attention_forward_offset(q, k, v, q_offset, scale=None, causal=False, window=0):
    """One key shard's partial forward, for context-parallel attention, in float64.

    Build a FlashAttention-2 Inference Kernel from Scratch in Pure Python,
    "Extending It" (distributed tensor parallelism: the attention matrix split
    across devices so the context outgrows one device's memory), and Build a
    FlashAttention Kernel with Online Softmax and KV Cache in Pure Python,
    "Extending It" (horizontal scaling: each worker holds a portion of the
    key/value space).  Reading: a worker holding a contiguous run of keys
    computes the softmax over its own keys only, with the causal and window
    masks evaluated at sequence positions -- query row i sits ``q_offset + i``
    positions after the shard's first key.  Rows that see no key of the shard
    get O = 0 and lse = -inf; the partials of all shards combine into the full
    result with :func:`merge_partials`.
    q: [..., Nq, d]; k, v: [..., Nk, d].  Returns (O [..., Nq, d], lse [..., Nq]).
    """
    q_pos = int(q_offset) + np.arange(np.asarray(q.shape)[-2])
    P, lse = attention_probabilities(q, k, scale, causal, window, q_pos=q_pos)
    return np.matmul(P, _f64(v)), lse


def merge_partials(o_parts, lse_parts):
    """Combine normalised partial results of disjoint key sets.

    Building Flash Attention from Scratch in Pure NumPy, architecture overview:
    the softmax over the union of two key sets is a re-weighting of the two
    partial softmaxes (the printed identity is garbled; restated):
        lse = ln sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.
    o_parts: [S, ..., d], lse_parts: [S, ...].  Empty parts carry lse = -inf.
    """
    o_parts = _f64(o_parts)
    lse_parts = _f64(lse_parts)
    m = lse_parts.max(axis=0)
    empty = np.isneginf(m)
    m_safe = np.where(empty, 0.0, m)
    w = np.exp(lse_parts - m_safe)
    tot = w.sum(axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        lse = np.where(empty, -np.inf, m_safe + np.log(tot))
        O = np.where(empty[..., None], 0.0,
                     (w[..., None] * o_parts).sum(axis=0) / np.where(empty, 1.0, tot)[..., None])
    return O, lse


def online_softmax_forward(q, k, v, block_q, block_k, scale=None, causal=False,
                           window=0, trace=None):
    """The tiled forward with the online softmax, one head, float64.

    Building Flash Attention from Scratch in Pure NumPy, architecture overview
    (data flow per query block) and Step 2 (online_softmax_update), in that
    page's notation: per query block, m = -inf, l = 0, O = 0; per key block,
    m_new = max(m, rowmax S), P = exp(S - m_new), l = exp(m - m_new) l +
    rowsum P, O = exp(m - m_new) O + P V; divide by l once at the end.
    FlashAttention Algorithm > Worked Example, Steps 1-3, traces the same loop.

    Masked keys (and keys past N) get score -inf; a block whose row is fully
    masked so far leaves that row's state unchanged.  Returns (O, lse) with
    lse = m + ln l.  ``trace``, if a list, receives one dict per
    (query block, key block) step with the state after the step.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    N, d = q.shape
    Nk = k.shape[0]
    s = default_scale(d, scale)
    O_all = np.zeros((N, d))
    lse_all = np.full(N, -np.inf)
    for qs in range(0, N, block_q):
        qe = min(qs + block_q, N)
        rows = np.arange(qs, qe)
        m = np.full(len(rows), -np.inf)
        l = np.zeros(len(rows))
        O = np.zeros((len(rows), d))
        for ks in range(0, Nk, block_k):
            ke = min(ks + block_k, Nk)
            S = (q[qs:qe] @ k[ks:ke].T) * s
            ok = allowed_mask(N, Nk, causal, window)[qs:qe, ks:ke]
            S = np.where(ok, S, -np.inf)
            m_new = np.maximum(m, S.max(axis=1))
            live = ~np.isneginf(m_new)           # rows with at least one allowed key so far
            m_ref = np.where(live, m_new, 0.0)   # avoids (-inf) - (-inf)
            alpha = np.where(live, np.exp(np.where(live, m, 0.0) - m_ref), 1.0)
            alpha = np.where(np.isneginf(m) & live, 0.0, alpha)
            P = np.exp(S - m_ref[:, None])
            l = alpha * l + P.sum(axis=1)
            O = alpha[:, None] * O + P @ v[ks:ke]
            m = m_new
            if trace is not None:
                trace.append(dict(q_block=qs // block_q, k_block=ks // block_k,
                                  S=S.copy(), m=m.copy(), l=l.copy(),
                                  alpha=alpha.copy(), O=O.copy()))
        live = l > 0
        O_all[qs:qe] = np.where(live[:, None], O / np.where(live, l, 1.0)[:, None], 0.0)
        with np.errstate(divide="ignore"):
            lse_all[qs:qe] = np.where(live, m + np.log(np.where(live, l, 1.0)), -np.inf)
    return O_all, lse_all
