"""A bounded device wait that runs out: the decode indexer (tcgen05) launched with
its key producer stalled (HCA_TEST_STALL=indexer: nothing is ever loaded, and every
wait has a budget of a few thousand polls) must return on its own, record the
failure, free its tensor memory, and leave the context usable: hca_check_device
reports HCA_ERR_DEVICE_CHECK once, and the next normal call runs correctly.
The stall is a flag that nothing sets -- no fault, trap or endless loop."""


import numpy as np
import pytest
import torch

import oracle
from long_context_attention_compress_b200 import workloads as wl
from parity_util import check_topk_row, to64

pytestmark = pytest.mark.gpu


def test_stalled_indexer_wait_runs_out_and_reports(monkeypatch):
    import long_context_attention_compress_b200 as hca
    s = wl.PRO
    cfg = hca.make_cfg(s)
    d = wl.csa_decode_inputs(s, B=2, ctx=4 * 65536, seed=21)
    g = {k: v.cuda() for k, v in d.items()}
    assert hca.lib.hca_check_device() == 0, hca.last_error()  # nothing pending from earlier tests
    monkeypatch.setenv("HCA_TEST_STALL", "indexer")
    hca.csa_indexer_topk(g["q_idx"], g["w_idx"], g["K_I"], g["q_pos"], cfg, mode=hca.HCA_MODE_DECODE)
    st = hca.lib.hca_check_device()
    assert st == -5, (st, hca.last_error())   # HCA_ERR_DEVICE_CHECK
    assert hca.lib.hca_check_device() == 0    # reported once, then cleared
    monkeypatch.delenv("HCA_TEST_STALL")
    # the context is still usable: the same call without the stall is correct
    idx = hca.csa_indexer_topk(g["q_idx"], g["w_idx"], g["K_I"], g["q_pos"], cfg, mode=hca.HCA_MODE_DECODE)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    ii = idx.cpu().numpy()
    t = 4 * 65536 - 1
    for b in range(2):
        sc = oracle.indexer_scores(to64(d["q_idx"][b]), d["w_idx"][b].double().numpy(), to64(d["K_I"][b]))
        check_topk_row(ii[b], oracle.topk_select(sc, s.topk), sc, s.topk, oracle.n_visible(t, s.m, 65536))
