"""Pins of the oracle's paged heterogeneous cache (addressing only).

QbitAI / yetianai write-ups (cache layout: a fixed state cache for the window
and the uncompressed tail, block-allocated classical cache for compressed
entries); "DeepSeek V4 Architecture Tricks", "Heterogeneous KV Cache Layout"
(each classical block covers lcm(m, m') raw tokens).  Paging must change
nothing but where rows live: identity and permuted block tables give the flat
result, every entry's own block of raw tokens stays inside one classical
block, and the ring-ordered window is the chronological window.
"""

import numpy as np
import pytest

import oracle
from long_context_attention_compress_b200 import workloads as wl


def test_block_geometry():
    assert oracle.classical_block_tokens(4, 128) == 128
    assert oracle.classical_block_tokens(4, 32) == 32
    assert oracle.classical_block_tokens(6, 16) == 48
    # an entry's own tokens [i m, (i+1) m) never straddle two classical blocks
    for m, mh in ((4, 128), (4, 32), (6, 16)):
        L = oracle.classical_block_tokens(m, mh)
        for rate in (m, mh):
            for i in range(3 * L // rate + 2):
                assert (i * rate) // L == ((i + 1) * rate - 1) // L


def _paged(E, rpb, perm):
    """Scatter flat rows E [N, w] into a pool of len(perm) physical blocks: logical
    block j goes to block perm[j]."""
    N, w = E.shape
    nb = (N + rpb - 1) // rpb
    assert nb <= len(perm)
    pool = np.full((len(perm), rpb, w), 1e6)  # unused blocks and slots hold garbage
    bt = np.asarray(perm[:nb])
    for i in range(N):
        pool[bt[i // rpb], i % rpb] = E[i]
    return pool, bt


def test_paged_rows_identity_and_permuted():
    rng = np.random.default_rng(0)
    E = rng.normal(size=(100, 8))
    for perm in (np.arange(20), rng.permutation(20)):
        pool, bt = _paged(E, 32, perm)
        np.testing.assert_array_equal(oracle.paged_rows(pool, bt, np.arange(100), 32), E)
        idx = rng.integers(0, 100, size=30)
        np.testing.assert_array_equal(oracle.paged_rows(pool, bt, idx, 32), E[idx])


def test_ring_window_is_chronological():
    n_win = 8
    toks = np.arange(40)
    rows = np.stack([toks, -toks], axis=1).astype(float)
    for t in (0, 3, 7, 8, 20, 39):
        ring = np.full((n_win, 2), np.nan)
        for tau in range(t + 1):
            ring[tau % n_win] = rows[tau]
        np.testing.assert_array_equal(oracle.ring_window(ring, t, n_win), rows[max(0, t - n_win + 1):t + 1])


@pytest.mark.parametrize("with_norm", [False, True])
def test_paged_decode_equals_flat(with_norm):
    s = wl.TINY
    rng = np.random.default_rng(1)
    t = 1000
    N = (t + 1) // s.m
    E = oracle.round_bf16(rng.normal(size=(N, s.c)))
    K = oracle.round_bf16(rng.normal(size=(N, s.d_idx)))
    q, qi, w = rng.normal(size=(s.n_heads, s.c)), rng.normal(size=(s.n_idx_heads, s.d_idx)), rng.uniform(size=s.n_idx_heads)
    raw = rng.normal(size=(t + 1, s.c))
    ring = np.empty((s.n_win, s.c))
    for tau in range(t + 1):
        ring[tau % s.n_win] = raw[tau]
    nrm = oracle.QKNorm(rng.uniform(0.5, 1.5, s.c), rng.uniform(0.5, 1.5, s.c), rope_dims=s.rope_dims) \
        if with_norm else None
    L = oracle.classical_block_tokens(s.m, s.m_hca)
    perm = rng.permutation(200)
    kv_pool, bt = _paged(E, L // s.m, perm)
    k_pool, _ = _paged(K, L // s.m, perm)
    flat = oracle.csa_layer_decode(E, K, raw[t - s.n_win + 1:t + 1], q, qi, w, t, m=s.m, topk=s.topk,
                                   n_win=s.n_win, scale=s.scale, norm=nrm)
    paged = oracle.csa_layer_decode_paged(kv_pool, k_pool, bt, N, ring, q, qi, w, t, m=s.m, m_hca=s.m_hca,
                                          topk=s.topk, n_win=s.n_win, scale=s.scale, norm=nrm)
    assert paged["idx"].tolist() == flat["idx"].tolist()
    np.testing.assert_array_equal(paged["O"], flat["O"])
    # HCA: lcm / m' entry rows per block
    Nh = (t + 1) // s.m_hca
    Eh = oracle.round_bf16(rng.normal(size=(Nh, s.c)))
    h_pool, hbt = _paged(Eh, L // s.m_hca, rng.permutation(200))
    rows = np.concatenate([Eh, raw[t - s.n_win + 1:t + 1]])
    want = (oracle.mqa_attend(q, rows, s.scale) if nrm is None else
            oracle.attend_norm_rope(q, t, raw[t - s.n_win + 1:t + 1], np.arange(t - s.n_win + 1, t + 1), s.scale, nrm,
                                    rows_ready=Eh))
    got = oracle.hca_attend_decode_paged(h_pool, hbt, Nh, ring, q, t, m=s.m, m_hca=s.m_hca, n_win=s.n_win,
                                         scale=s.scale, norm=nrm)
    np.testing.assert_allclose(got, want, atol=1e-13)
