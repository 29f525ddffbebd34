"""Plant plausible mistakes in the oracle (on the CPU) and check the pins catch each.

A pin set that passes a wrong oracle proves nothing; every mutant below must
make at least one pin fail.  The mutants are patched into the oracle module
for the duration of one test only.
"""
import numpy as np
import pytest

import oracle.attention as om
import oracle_pins


def _fails_some_pin(monkeypatch_target=None):
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(om)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


def _mask_window_off_by_one(n_q, n_k, causal, window, q_pos=None):
    i = np.arange(n_q)[:, None] if q_pos is None else np.asarray(q_pos)[:, None]
    j = np.arange(n_k)[None, :]
    ok = np.ones((i.shape[0], n_k), dtype=bool)
    if causal:
        ok &= j <= i
    if window > 0:
        ok &= j >= i - window          # keeps window + 1 keys
    return ok


def _mask_strict_causal(n_q, n_k, causal, window, q_pos=None):
    i = np.arange(n_q)[:, None] if q_pos is None else np.asarray(q_pos)[:, None]
    j = np.arange(n_k)[None, :]
    ok = np.ones((i.shape[0], n_k), dtype=bool)
    if causal:
        ok &= j < i                    # drops the diagonal
    if window > 0:
        ok &= j > i - window
    return ok


def _scale_inverted(d, scale):
    return np.sqrt(d) if scale is None or scale <= 0 else float(scale)


def _lse_without_max(S):
    with np.errstate(divide="ignore", over="ignore"):
        m = S.max(axis=-1, keepdims=True)
        m0 = np.where(np.isneginf(m), 0.0, m)
        return np.log(np.exp(S - m0).sum(axis=-1))   # forgot "+ m"


def _backward_factory(mistake):
    def bwd(q, k, v, dO, scale=None, causal=False, window=0):
        q, k, v, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dO))
        s = om.default_scale(q.shape[-1], scale)
        P, _ = om.attention_probabilities(q, k, s, causal, window)
        O = P @ v
        D = (dO * O).sum(-1)
        dV = np.swapaxes(P, -1, -2) @ dO
        if mistake == "dv_no_transpose":
            dV = P @ dO
        dP = dO @ np.swapaxes(v, -1, -2)
        dS = P * (dP - D[..., None])
        if mistake == "no_D":
            dS = P * dP
        dQ = s * dS @ k
        dK = s * np.swapaxes(dS, -1, -2) @ q
        if mistake == "dk_no_scale":
            dK = np.swapaxes(dS, -1, -2) @ q
        if mistake == "dq_uses_v":
            dQ = s * dS @ v
        return dQ, dK, dV
    return bwd


def _online_sign_flip(q, k, v, block_q, block_k, scale=None, causal=False, window=0,
                      trace=None):
    # The rescale factor written as exp(m_new - m) instead of exp(m - m_new).
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    N, d = q.shape
    s = om.default_scale(d, scale)
    O_all = np.zeros((N, d))
    lse_all = np.zeros(N)
    for qs in range(0, N, block_q):
        qe = min(qs + block_q, N)
        m = np.full(qe - qs, -np.inf)
        l = np.zeros(qe - qs)
        O = np.zeros((qe - qs, d))
        for ks in range(0, k.shape[0], block_k):
            ke = min(ks + block_k, k.shape[0])
            S = (q[qs:qe] @ k[ks:ke].T) * s
            S = np.where(om.allowed_mask(N, k.shape[0], causal, window)[qs:qe, ks:ke], S, -np.inf)
            m_new = np.maximum(m, S.max(1))
            alpha = np.where(np.isneginf(m), 0.0, np.exp(m_new - np.where(np.isneginf(m), 0, m)))
            P = np.exp(S - m_new[:, None])
            l = alpha * l + P.sum(1)
            O = alpha[:, None] * O + P @ v[ks:ke]
            m = m_new
            if trace is not None:
                trace.append(dict(q_block=qs // block_q, k_block=ks // block_k, S=S, m=m.copy(),
                                  l=l.copy(), alpha=alpha.copy(), O=O.copy()))
        O_all[qs:qe] = O / l[:, None]
        lse_all[qs:qe] = m + np.log(l)
    return O_all, lse_all


def _decode_reads_one_extra(q, kcache, vcache, seqlens, scale=None):
    seqlens = np.minimum(np.asarray(seqlens) + 1, np.asarray(kcache).shape[2])
    return _real_decode(q, kcache, vcache, seqlens, scale)


def _merge_unweighted(o_parts, lse_parts):
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    live = ~np.isneginf(lse_parts)
    O = (o_parts * live[..., None]).sum(0) / live.sum(0)[..., None]
    with np.errstate(divide="ignore"):
        lse = np.log(np.exp(lse_parts).sum(0))
    return O, lse


_real_decode = om.decode_forward


def _paged_blocks_reversed(q, kpool, vpool, block_table, seqlens, scale=None):
    """Gathers each sequence's blocks in reverse table order."""
    kpool, vpool = np.asarray(kpool, dtype=np.float64), np.asarray(vpool, dtype=np.float64)
    table = np.asarray(block_table).astype(np.int64)
    _, H, bs, d = kpool.shape
    B, max_blocks = table.shape
    cap = max_blocks * bs
    n = np.clip(np.asarray(seqlens).astype(np.int64), 0, cap)
    kc, vc = np.zeros((B, H, cap, d)), np.zeros((B, H, cap, d))
    for b in range(B):
        nb = -(-int(n[b]) // bs)
        for t in range(nb):
            kc[b, :, t * bs:(t + 1) * bs] = kpool[table[b, nb - 1 - t]]
            vc[b, :, t * bs:(t + 1) * bs] = vpool[table[b, nb - 1 - t]]
    return _real_decode(q, kc, vc, n, scale)

def _offset_factory(mistake):
    def fwd(q, k, v, q_offset, scale=None, causal=False, window=0):
        n_q = np.asarray(q).shape[-2]
        if mistake == "sign":
            q_pos = np.arange(n_q) - q_offset       # key shard taken as ahead of the queries
        else:
            q_pos = np.arange(n_q)                  # offset ignored: every shard seen as the diagonal
        P, lse = om.attention_probabilities(q, k, scale, causal, window, q_pos=q_pos)
        return P @ np.asarray(v, dtype=np.float64), lse
    return fwd


MUTANTS = {
    "window_off_by_one": ("allowed_mask", _mask_window_off_by_one),
    "causal_drops_diagonal": ("allowed_mask", _mask_strict_causal),
    "scale_inverted": ("default_scale", _scale_inverted),
    "lse_without_max": ("_logsumexp_rows", _lse_without_max),
    "bwd_dv_no_transpose": ("attention_backward", _backward_factory("dv_no_transpose")),
    "bwd_no_D_term": ("attention_backward", _backward_factory("no_D")),
    "bwd_dk_no_scale": ("attention_backward", _backward_factory("dk_no_scale")),
    "bwd_dq_uses_v": ("attention_backward", _backward_factory("dq_uses_v")),
    "online_rescale_sign": ("online_softmax_forward", _online_sign_flip),
    "decode_reads_past_seqlen": ("decode_forward", _decode_reads_one_extra),
    "merge_unweighted": ("merge_partials", _merge_unweighted),
    "paged_blocks_reversed": ("decode_paged_forward", _paged_blocks_reversed),
    "offset_sign_flipped": ("attention_forward_offset", _offset_factory("sign")),
    "offset_ignored": ("attention_forward_offset", _offset_factory("ignored")),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(om, attr, fn)
    with np.errstate(all="ignore"):
        failed = _fails_some_pin()
    assert failed, f"no pin caught the planted mistake {name!r}"
