"""Pins that tie the float64 oracle to facts outside itself.

Each ``pin_*`` takes the oracle module (or a stand-in with the same
functions) and raises AssertionError when the oracle disagrees with:

* the values the worked-example page prints (``tests/golden``),
* closed forms and special cases (N = 1, all-equal scores, causal row 0),
* invariants (rows of P sum to 1, masked weight exactly 0, shift invariance,
  gradient sums), the tiled algorithm's independence of its block size,
* torch's float64 CPU attention (forward, logsumexp and autograd),
* central finite differences of the forward.

``tests/test_oracle_mutants.py`` plants plausible mistakes in the oracle and
checks that some pin here catches each of them.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "worked_example_n8_d4.json")

MASKS = [  # (causal, window)
    (False, 0),
    (True, 0),
    (True, 5),
    (False, 7),
    (True, 1),
]


def _close_to_printed(x, printed, what):
    """|x - printed| <= half a unit of the last printed decimal (+ rounding slack)."""
    val = np.asarray(printed["value"], dtype=np.float64)
    tol = 0.5 * 10.0 ** (-printed["decimals"]) + 1e-9
    err = np.abs(np.asarray(x, dtype=np.float64) - val).max()
    assert err <= tol, f"{what}: max |diff| {err:.3g} > {tol:.3g}"


def _golden():
    with open(GOLDEN) as f:
        g = json.load(f)
    Q, K, V = (np.asarray(g[n], dtype=np.float64) for n in ("Q", "K", "V"))
    return g, Q, K, V


def pin_worked_example_tiled(o):
    """The tiled online-softmax loop reproduces the page's trace, step by step."""
    g, Q, K, V = _golden()
    p = g["printed"]
    trace = []
    O, _ = o.online_softmax_forward(Q, K, V, g["block"], g["block"], scale=g["scale"],
                                    trace=trace)
    st0 = [t for t in trace if t["q_block"] == 0 and t["k_block"] == 0][0]
    st1 = [t for t in trace if t["q_block"] == 0 and t["k_block"] == 1][0]
    _close_to_printed(st0["S"], p["scores_block0"], "scores block 0")
    _close_to_printed(st0["m"], p["running_max_after_block0"], "running max after block 0")
    _close_to_printed(st0["l"], p["running_sum_after_block0"], "running sum after block 0")
    _close_to_printed(st1["S"], p["scores_block1"], "scores block 1")
    _close_to_printed(st1["alpha"], p["rescale_factor_block1"], "rescale factors")
    _close_to_printed(st1["m"], p["final_running_max"], "final running max")
    _close_to_printed(st1["l"], p["final_running_sum"], "final running sum")
    _close_to_printed(O[:4], p["output_rows_0_3"], "output rows 0-3 (tiled)")


def pin_worked_example_naive(o):
    """The naive definition gives the page's printed outputs and consistent lse."""
    g, Q, K, V = _golden()
    p = g["printed"]
    O, lse = o.attention_forward(Q, K, V, scale=g["scale"])
    _close_to_printed(O[:4], p["output_rows_0_3"], "output rows 0-3 (naive)")
    # lse = final max + ln(final sum); the printed sum has 3 decimals.
    l_printed = np.asarray(p["final_running_sum"]["value"])
    expect = np.asarray(p["final_running_max"]["value"]) + np.log(l_printed)
    # The printed max (0.5) is exact here: it is the score of an exact match.
    tol = 0.5e-3 / l_printed.min() + 1e-9
    assert np.abs(lse[:4] - expect).max() <= tol
    # Default scale is 1/sqrt(d) = 0.5 for d = 4.
    O2, _ = o.attention_forward(Q, K, V)
    assert np.abs(O2 - O).max() < 1e-15


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def pin_probabilities(o):
    """Rows of P sum to 1, masked weights are exactly 0, all weights >= 0."""
    for causal, window in MASKS:
        q = _rand((2, 23, 6), 1)
        k = _rand((2, 23, 6), 2)
        P, lse = o.attention_probabilities(q, k, None, causal, window)
        ok = np.zeros((23, 23), dtype=bool)
        for i in range(23):
            for j in range(23):
                ok[i, j] = (not causal or j <= i) and (window <= 0 or j > i - window)
        assert np.all(P[:, ~ok] == 0.0), (causal, window)
        assert np.all(P >= 0)
        assert np.abs(P.sum(-1) - 1.0).max() < 1e-12, (causal, window)
        assert np.all(np.isfinite(lse))


def pin_special_cases(o):
    """Closed forms: N = 1; all-equal scores; causal row 0."""
    # N = 1: the only key gets all the weight; lse is its scaled score.
    q, k, v = _rand((1, 5), 3), _rand((1, 5), 4), _rand((1, 5), 5)
    O, lse = o.attention_forward(q, k, v, scale=0.3)
    assert np.abs(O - v).max() < 1e-15
    assert abs(lse[0] - 0.3 * float(q[0] @ k[0])) < 1e-14
    # q = 0: every allowed score is 0, so O_i is the mean of the allowed V rows
    # and lse_i = ln(number of allowed keys).
    N = 17
    k, v = _rand((N, 4), 6), _rand((N, 4), 7)
    for causal, window in MASKS:
        O, lse = o.attention_forward(np.zeros((N, 4)), k, v, None, causal, window)
        for i in range(N):
            js = [j for j in range(N)
                  if (not causal or j <= i) and (window <= 0 or j > i - window)]
            assert np.abs(O[i] - v[js].mean(axis=0)).max() < 1e-14, (causal, window, i)
            assert abs(lse[i] - math.log(len(js))) < 1e-14, (causal, window, i)
    # Causal row 0 sees only key 0.
    q, k, v = _rand((9, 4), 8), _rand((9, 4), 9), _rand((9, 4), 10)
    O, lse = o.attention_forward(q, k, v, 0.7, True, 0)
    assert np.abs(O[0] - v[0]).max() < 1e-15
    assert abs(lse[0] - 0.7 * float(q[0] @ k[0])) < 1e-14


def pin_shift_invariance(o):
    """Adding one vector to every key shifts each row's scores by a constant
    (O unchanged, lse moves by scale*q_i.c); adding c to every value row adds c
    to O (rows of P sum to 1)."""
    q, k, v = _rand((13, 4), 11), _rand((13, 4), 12), _rand((13, 4), 13)
    c = _rand((4,), 14)
    for causal, window in MASKS:
        O, lse = o.attention_forward(q, k, v, 0.4, causal, window)
        O2, lse2 = o.attention_forward(q, k + c, v, 0.4, causal, window)
        assert np.abs(O2 - O).max() < 1e-12
        assert np.abs(lse2 - (lse + 0.4 * q @ c)).max() < 1e-12
        O3, _ = o.attention_forward(q, k, v + c, 0.4, causal, window)
        assert np.abs(O3 - (O + c)).max() < 1e-12


def _torch_mask(N, causal, window):
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    ok = torch.ones(N, N, dtype=torch.bool)
    if causal:
        ok &= j <= i
    if window > 0:
        ok &= j > i - window
    return ok


def pin_torch_forward(o):
    """Matches torch's float64 CPU attention: output and logsumexp."""
    B, H, N, d = 2, 3, 37, 8
    q, k, v = (torch.from_numpy(_rand((B, H, N, d), s)) for s in (20, 21, 22))
    for causal, window in MASKS:
        mask = _torch_mask(N, causal, window)
        ref = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=0.2)
        additive = torch.zeros(N, N, dtype=torch.float64).masked_fill(~mask, float("-inf"))
        out, lse_ref = torch.ops.aten._scaled_dot_product_flash_attention_for_cpu(
            q, k, v, 0.0, False, attn_mask=additive, scale=0.2)
        O, lse = o.attention_forward(q.numpy(), k.numpy(), v.numpy(), 0.2, causal, window)
        assert np.abs(O - ref.numpy()).max() < 1e-12, (causal, window)
        assert np.abs(O - out.numpy()).max() < 1e-12, (causal, window)
        assert np.abs(lse - lse_ref.numpy()).max() < 1e-12, (causal, window)


def pin_block_invariance(o):
    """The tiled online softmax equals the naive definition for any block sizes,
    including blocks that do not divide N (ragged tail)."""
    N, d = 37, 6
    q, k, v = _rand((N, d), 30), _rand((N, d), 31), _rand((N, d), 32)
    for causal, window in MASKS:
        O_ref, lse_ref = o.attention_forward(q, k, v, None, causal, window)
        for bq, bk in [(1, 1), (2, 3), (4, 4), (8, 5), (16, 16), (64, 64)]:
            O, lse = o.online_softmax_forward(q, k, v, bq, bk, None, causal, window)
            assert np.abs(O - O_ref).max() < 1e-12, (causal, window, bq, bk)
            assert np.abs(lse - lse_ref).max() < 1e-12, (causal, window, bq, bk)


def pin_backward_finite_differences(o):
    """Central differences of L = sum(O * G) match the analytic gradient."""
    n, d, h = 6, 3, 1e-6
    q, k, v, G = (_rand((n, d), s) for s in (40, 41, 42, 43))
    for causal, window in [(False, 0), (True, 0), (True, 3), (False, 2)]:
        def loss(qq, kk, vv):
            O, _ = o.attention_forward(qq, kk, vv, 0.9, causal, window)
            return float((O * G).sum())

        dq, dk, dv = o.attention_backward(q, k, v, G, 0.9, causal, window)
        for X, dX, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
            num = np.zeros_like(X)
            for idx in np.ndindex(*X.shape):
                Xp = X.copy()
                Xm = X.copy()
                Xp[idx] += h
                Xm[idx] -= h
                args_p = [q, k, v]
                args_m = [q, k, v]
                args_p[which] = Xp
                args_m[which] = Xm
                num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
            rel = np.abs(num - dX).max() / max(np.abs(num).max(), 1e-30)
            assert rel < 1e-6, (causal, window, which, rel)


def pin_backward_torch(o):
    """Matches torch autograd through float64 scaled_dot_product_attention."""
    B, H, N, d = 2, 2, 19, 8
    for causal, window in MASKS:
        q, k, v, G = (torch.from_numpy(_rand((B, H, N, d), s)) for s in (50, 51, 52, 53))
        for t in (q, k, v):
            t.requires_grad_(True)
        out = F.scaled_dot_product_attention(q, k, v, attn_mask=_torch_mask(N, causal, window),
                                             scale=0.35)
        out.backward(G)
        dq, dk, dv = o.attention_backward(q.detach().numpy(), k.detach().numpy(),
                                          v.detach().numpy(), G.numpy(), 0.35, causal, window)
        assert np.abs(dq - q.grad.numpy()).max() < 1e-11, (causal, window)
        assert np.abs(dk - k.grad.numpy()).max() < 1e-11, (causal, window)
        assert np.abs(dv - v.grad.numpy()).max() < 1e-11, (causal, window)


def pin_backward_identities(o):
    """sum_j dV_j = sum_i dO_i (rows of P sum to 1) and sum_j dK_j = 0 (each row
    of dS sums to 0), per head, when no row is fully masked."""
    q, k, v, G = (_rand((2, 29, 5), s) for s in (60, 61, 62, 63))
    for causal, window in MASKS:
        dq, dk, dv = o.attention_backward(q, k, v, G, None, causal, window)
        assert np.abs(dv.sum(-2) - G.sum(-2)).max() < 1e-11, (causal, window)
        assert np.abs(dk.sum(-2)).max() < 1e-11, (causal, window)


def pin_decode(o):
    """Decode equals the last row of a causal forward over the first seqlen
    tokens (the query is the newest token, already in the cache); an empty
    cache gives o = 0, lse = -inf."""
    B, H, cap, d = 4, 2, 40, 8
    seqlens = np.array([1, 17, 40, 0])
    kc, vc = _rand((B, H, cap, d), 70), _rand((B, H, cap, d), 71)
    qtok = _rand((B, H, d), 72)
    o_dec, lse_dec = o.decode_forward(qtok, kc, vc, seqlens, 0.25)
    for b in range(B):
        n = int(seqlens[b])
        if n == 0:
            assert np.all(o_dec[b] == 0) and np.all(np.isneginf(lse_dec[b]))
            continue
        qfull = _rand((H, n, d), 73 + b)
        qfull[:, n - 1] = qtok[b]
        O, lse = o.attention_forward(qfull, kc[b, :, :n], vc[b, :, :n], 0.25, True, 0)
        assert np.abs(o_dec[b] - O[:, n - 1]).max() < 1e-12, b
        assert np.abs(lse_dec[b] - lse[:, n - 1]).max() < 1e-12, b


def pin_paged_decode(o):
    """A padded cache cut into blocks, scattered through a pool in a random order
    with the table recording where each block went, decodes exactly as the padded
    cache does; table entries past a sequence's blocks (here -1) and pool rows past
    its length (here NaN) play no part."""
    B, H, bs, d, max_blocks = 3, 2, 4, 8, 6
    cap = bs * max_blocks
    seqlens = np.array([24, 9, 1])
    kc, vc, q = _rand((B, H, cap, d), 100), _rand((B, H, cap, d), 101), _rand((B, H, d), 102)
    o_ref, lse_ref = o.decode_forward(q, kc, vc, seqlens, 0.3)
    nblk = [-(-int(n) // bs) for n in seqlens]
    perm = np.random.default_rng(103).permutation(sum(nblk))
    kpool = np.full((sum(nblk), H, bs, d), np.nan)
    vpool = np.full((sum(nblk), H, bs, d), np.nan)
    table = np.full((B, max_blocks), -1)
    i = 0
    for b in range(B):
        for t in range(nblk[b]):
            p = perm[i]
            i += 1
            table[b, t] = p
            rows = slice(t * bs, min((t + 1) * bs, int(seqlens[b])))
            kpool[p, :, :rows.stop - rows.start] = kc[b, :, rows]
            vpool[p, :, :rows.stop - rows.start] = vc[b, :, rows]
    o_pg, lse_pg = o.decode_paged_forward(q, kpool, vpool, table, seqlens, 0.3)
    assert np.abs(o_pg - o_ref).max() < 1e-14
    assert np.abs(lse_pg - lse_ref).max() < 1e-14


def pin_merge(o):
    """Merging the results of disjoint key chunks (one of them empty) gives the
    result over all keys."""
    B, H, cap, d = 2, 3, 50, 8
    seqlens = np.array([50, 50])
    kc, vc, q = _rand((B, H, cap, d), 80), _rand((B, H, cap, d), 81), _rand((B, H, d), 82)
    o_all, lse_all = o.decode_forward(q, kc, vc, seqlens, None)
    bounds = [(0, 7), (7, 7), (7, 31), (31, 50)]
    parts_o, parts_l = [], []
    for lo, hi in bounds:
        o_p, l_p = o.decode_forward(q, kc[:, :, lo:hi], vc[:, :, lo:hi],
                                    np.full(B, hi - lo), None)
        parts_o.append(o_p)
        parts_l.append(l_p)
    O, lse = o.merge_partials(np.stack(parts_o), np.stack(parts_l))
    assert np.abs(O - o_all).max() < 1e-12
    assert np.abs(lse - lse_all).max() < 1e-12


def pin_rows_subset(o):
    """Evaluating selected rows alone gives the same rows as the full forward."""
    N, d = 41, 4
    q, k, v = _rand((N, d), 90), _rand((N, d), 91), _rand((N, d), 92)
    rows = np.array([0, 5, 17, 40])
    for causal, window in MASKS:
        O, lse = o.attention_forward(q, k, v, None, causal, window)
        Or, lr = o.attention_forward_rows(q, k, v, rows, None, causal, window)
        assert np.abs(Or - O[rows]).max() < 1e-14
        assert np.abs(lr - lse[rows]).max() < 1e-14


def pin_offset_shards(o):
    """Context parallelism: cut a ragged sequence into query and key shards of
    unequal length; each query shard's partials against every key shard, with
    the offset between the shards' first positions, merge into the same rows of
    the full forward.  Shards that a query shard cannot see come back empty
    (lse = -inf) and drop out of the merge."""
    N, d = 37, 4
    q, k, v = _rand((2, N, d), 120), _rand((2, N, d), 121), _rand((2, N, d), 122)
    bounds = [(0, 10), (10, 11), (11, 23), (23, 37)]
    for causal, window in MASKS + [(True, 12), (False, 30)]:
        O, lse = o.attention_forward(q, k, v, 0.4, causal, window)
        for qlo, qhi in bounds:
            parts_o, parts_l = [], []
            for klo, khi in bounds:
                po, pl = o.attention_forward_offset(q[:, qlo:qhi], k[:, klo:khi], v[:, klo:khi],
                                                    qlo - klo, 0.4, causal, window)
                parts_o.append(po)
                parts_l.append(pl)
            Om, lm = o.merge_partials(np.stack(parts_o), np.stack(parts_l))
            assert np.abs(Om - O[:, qlo:qhi]).max() < 1e-12, (causal, window, qlo)
            assert np.abs(lm - lse[:, qlo:qhi]).max() < 1e-12, (causal, window, qlo)


def pin_offset_closed_form(o):
    """q = 0 makes every visible score 0: with query row i at position off + i,
    O_i is the mean of the V rows it sees and lse_i = ln(their count); a row
    that sees none gets O = 0 and lse = -inf.  Also checked against torch's
    float64 scaled_dot_product_attention on random inputs, with the mask built
    from positions by loops."""
    Nq, Nk, d = 6, 9, 3
    k, v = _rand((Nk, d), 123), _rand((Nk, d), 124)
    q = _rand((Nq, d), 125)
    for off in (-8, -3, 0, 4, 11, 14):
        for causal, window in MASKS:
            O, lse = o.attention_forward_offset(np.zeros((Nq, d)), k, v, off, None, causal, window)
            ok = np.zeros((Nq, Nk), dtype=bool)
            for i in range(Nq):
                p = off + i
                js = [j for j in range(Nk)
                      if (not causal or j <= p) and (window <= 0 or j > p - window)]
                ok[i, js] = True
                if js:
                    assert np.abs(O[i] - v[js].mean(axis=0)).max() < 1e-14, (off, causal, window, i)
                    assert abs(lse[i] - math.log(len(js))) < 1e-14, (off, causal, window, i)
                else:
                    assert np.all(O[i] == 0.0) and lse[i] == -np.inf, (off, causal, window, i)
            live = ok.any(axis=1)
            if not live.any():
                continue
            O, _ = o.attention_forward_offset(q, k, v, off, 0.6, causal, window)
            ref = F.scaled_dot_product_attention(
                torch.from_numpy(q[live]), torch.from_numpy(k), torch.from_numpy(v),
                attn_mask=torch.from_numpy(ok[live]), scale=0.6).numpy()
            assert np.abs(O[live] - ref).max() < 1e-12, (off, causal, window)


ALL_PINS = [
    pin_worked_example_tiled,
    pin_worked_example_naive,
    pin_probabilities,
    pin_special_cases,
    pin_shift_invariance,
    pin_torch_forward,
    pin_block_invariance,
    pin_backward_finite_differences,
    pin_backward_torch,
    pin_backward_identities,
    pin_decode,
    pin_paged_decode,
    pin_merge,
    pin_rows_subset,
    pin_offset_shards,
    pin_offset_closed_form,
]
