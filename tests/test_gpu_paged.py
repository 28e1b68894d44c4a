"""GPU parity of the paged heterogeneous cache (decode) against the oracle.

"DeepSeek V4 Architecture Tricks", "Heterogeneous KV Cache Layout": the
compressed ("classical") cache is allocated in blocks of lcm(m, m') = 128 raw
tokens -- 32 CSA entries with their indexer keys and one HCA entry per block --
reached through a per-request block table; "DeepSeek-V4技术报告解读", 核心创新一:
the window lives in a separate state cache (here a ring of n_win rows).  The
GPU reads its caches from pools through a shuffled block table (spare blocks
hold garbage); the oracle (csa_layer_decode_paged, hca_attend_decode_paged)
reads the same pools through the same table.  Checked: top-k sets, both
layers' outputs, and the newest HCA entry written to its pool row.
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_attention_compress_b200 import workloads as wl
from parity_util import assert_bf16_close, assert_norm_close, check_topk_row, to64

pytestmark = pytest.mark.gpu


def _pool(flat, rpb, bt, n_blocks, garbage):
    """Scatter flat rows [B, N, w] into a pool [n_blocks, rpb, w] (bf16): logical block j
    of request b goes to physical block bt[b, j]; unused rows hold `garbage`."""
    B, N, w = flat.shape
    pool = torch.full((n_blocks, rpb, w), garbage, dtype=flat.dtype)
    for b in range(B):
        nb = (N + rpb - 1) // rpb
        for j in range(nb):
            r1 = min(N, (j + 1) * rpb)
            pool[bt[b, j], :r1 - j * rpb] = flat[b, j * rpb:r1]
    return pool


def _ring(win_chrono, t, n_win):
    """Ring form of a window block whose rows are tokens t-n_win+1 .. t, oldest first:
    token tau at row tau mod n_win."""
    ring = torch.empty_like(win_chrono)
    for w in range(n_win):
        tau = t - n_win + 1 + w
        ring[tau % n_win] = win_chrono[w]
    return ring


@pytest.mark.parametrize("with_norm", [False, True])
def test_paged_hybrid_decode(with_norm):
    import long_context_attention_compress_b200 as hca
    s = wl.PRO
    B, ctx = 3, 4 * 65536 if not with_norm else 4 * 20480
    t = ctx - 1
    L = oracle.classical_block_tokens(s.m, s.m_hca)
    rpb_c, rpb_h = L // s.m, L // s.m_hca
    d = wl.hybrid_decode_inputs(s, B, ctx, seed=31)
    hb = wl.hca_decode_inputs(s, B, ctx, seed=37, with_block=True)  # HCA layer with its newest block raw
    c = d["csa"]
    N, Nh = c["E"].shape[1], hb["E_h"].shape[1]
    nblk = ctx // L
    spare = 7
    P = B * nblk + spare
    rng = np.random.default_rng(5)
    bt = torch.tensor(rng.permutation(P)[:B * nblk].reshape(B, nblk), dtype=torch.int32)
    kv_pool = _pool(c["E"], rpb_c, bt, P, 3.0)
    k_pool = _pool(c["K_I"], rpb_c, bt, P, -2.0)
    h_pool = _pool(hb["E_h"], rpb_h, bt, P, 5.0)  # row Nh-1 of every request is zero: the GPU fills it
    csa_ring = torch.stack([_ring(c["win"][b], t, s.n_win) for b in range(B)])
    hca_ring = torch.stack([_ring(hb["win"][b], t, s.n_win) for b in range(B)])
    norm_kw, nrm = {}, {}
    if with_norm:
        norm_kw = {"csa_norm": wl.norm_weights(s, seed=3).cuda(), "hca_norm": wl.norm_weights(s, seed=4).cuda()}
        nrm = {k: oracle.QKNorm(v[0].double().cpu().numpy(), v[1].double().cpu().numpy(), eps=s.norm_eps,
                                rope_dims=s.rope_dims, base=s.rope_base) for k, v in norm_kw.items()}
    gc = {"q": c["q"].cuda(), "q_idx": c["q_idx"].cuda(), "w_idx": c["w_idx"].cuda(), "E": kv_pool.cuda(),
          "K_I": k_pool.cuda(), "win": csa_ring.cuda()}
    gh = {"q": hb["q"].cuda(), "E_h": h_pool.cuda(), "win": hca_ring.cuda(), "block_cand": hb["block_cand"].cuda(),
          "block_logits": hb["block_logits"].cuda(), "bias_hca": hb["bias_hca"].cuda()}
    q_pos = torch.full((B,), t, dtype=torch.int32, device="cuda")
    idx = torch.empty((B, s.topk), dtype=torch.int32, device="cuda")
    oc = torch.empty((B, s.n_heads, s.c), dtype=torch.bfloat16, device="cuda")
    oh = torch.empty_like(oc)
    cfg = hca.make_cfg(s)
    args, keep = hca.make_decode_args(B, q_pos, csa=gc, hca=gh, csa_topk_idx=idx, csa_out=oc, hca_out=oh,
                                      **norm_kw)
    # the pools: counts of entries per request and the block table
    args.csa_N, args.hca_N = N, Nh
    btd = bt.cuda()
    args.block_table, args.bt_stride, args.n_pool_blocks = btd.data_ptr(), nblk, P
    args.csa_kv_stride = args.csa_k_stride = args.hca_kv_stride = 0
    hca.hybrid_attn_decode(cfg, args)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()

    ii = idx.cpu().numpy()
    hp = h_pool.clone()
    kvp, kp = to64(kv_pool), to64(k_pool)
    for b in range(B):
        r = oracle.csa_layer_decode_paged(kvp, kp, bt[b].numpy(), N, to64(csa_ring[b]), to64(c["q"][b]),
                                          to64(c["q_idx"][b]), c["w_idx"][b].double().numpy(), t, m=s.m,
                                          m_hca=s.m_hca, topk=s.topk, n_win=s.n_win, scale=s.scale,
                                          norm=nrm.get("csa_norm"))
        check_topk_row(ii[b], r["idx"], r["scores"], s.topk, r["n_vis"])
        assert_norm_close(to64(oc[b].cpu()), r["O"], what=f"paged csa request {b}")
        # newest HCA entry: the oracle's compression (and normalisation), in the cache's form
        new = oracle.hca_layer_decode(to64(hb["E_h"][b]), to64(hb["block_cand"][b]), to64(hb["block_logits"][b]),
                                      hb["bias_hca"].double().numpy(), to64(hb["win"][b]), to64(hb["q"][b]), t,
                                      m_hca=s.m_hca, n_win=s.n_win, scale=s.scale, norm=nrm.get("hca_norm"))
        prow = int(bt[b, (Nh - 1) // rpb_h]) * rpb_h + (Nh - 1) % rpb_h
        got_row = gh["E_h"].view(-1, s.c)[prow].cpu()
        exact = oracle.hca_compress(to64(hb["block_cand"][b]), to64(hb["block_logits"][b]),
                                    hb["bias_hca"].double().numpy(), s.m_hca)
        if with_norm:
            nh = nrm["hca_norm"]
            exact = oracle.norm_rope_rows(exact, oracle.entry_position(Nh - 1, s.m_hca), nh.kv_gamma, nh)
        assert_bf16_close(to64(got_row), exact[0], f"new HCA entry {b} in its pool row")
        # the reference pool holds the oracle's own cache form of the entry
        hp.view(-1, s.c)[prow] = torch.tensor(new["new_entry"]).bfloat16()
    hpp = to64(hp)
    for b in range(B):
        o = oracle.hca_attend_decode_paged(hpp, bt[b].numpy(), Nh, to64(hca_ring[b]), to64(hb["q"][b]), t, m=s.m,
                                           m_hca=s.m_hca, n_win=s.n_win, scale=s.scale, norm=nrm.get("hca_norm"))
        assert_norm_close(to64(oh[b].cpu()), o, what=f"paged hca request {b}")
