"""csa_indexer_topk_noalloc: the indexer + top-k for callers that cannot
allocate device memory (a plugin inside a runtime that owns all device
memory, a serving loop that forbids allocation after start-up).

It uses a built-in 16 MiB device array instead of a caller workspace.  This
test calls it through the C ABI and checks that its output equals the
regular entry point's (which gets a torch-allocated workspace) on calls in a
row -- each later call finds the earlier calls' histograms, arrival tickets,
score rows and candidate lists still in the shared array -- and that a call
needing more scratch than the array holds is refused before anything runs.
The capacity boundary is checked exactly: 5 decode requests of 262,144
entries (about 15.5 MiB of scratch) run, 6 (about 18.6 MiB) are refused.  It
lives in its own file, collected last, so a failure here comes after every
other test has run; it also passes alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

from long_context_attention_compress_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _noalloc(lib, q_idx, w_idx, k_idx, q_pos, cfg, mode, out):
    f = lib.lib.csa_indexer_topk_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int,
                  ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.POINTER(lib.LayerCfg), ctypes.c_void_p,
                  ctypes.c_void_p]
    kstride = k_idx.stride(0) if k_idx.dim() == 3 else 0
    return f(q_idx.data_ptr(), w_idx.data_ptr(), k_idx.data_ptr(), kstride, k_idx.shape[-2], q_pos.data_ptr(),
             q_idx.shape[0], mode, ctypes.byref(cfg), out.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_entry_point_twice():
    from long_context_attention_compress_b200 import _lib as lib
    s = wl.PRO
    cfg = lib.make_cfg(s)
    first = wl.csa_decode_inputs(s, B=8, ctx=4 * 65536, seed=41)  # 8 requests x 65,536 entries (histogram select)
    cases = [
        first,
        wl.csa_decode_inputs(s, B=3, ctx=4 * 100000, seed=42),   # histogram select again, other Tq and N (ragged)
        first,                                                   # the first shape once more, after the second
        wl.csa_decode_inputs(s, B=3, ctx=4 * 20000, seed=43),    # one select CTA per request, ragged
    ]
    for d in cases:
        g = {k: v.cuda() for k, v in d.items()}
        ref = lib.csa_indexer_topk(g["q_idx"], g["w_idx"], g["K_I"], g["q_pos"], cfg, mode=lib.HCA_MODE_DECODE)
        out = torch.full_like(ref, -7)
        st = _noalloc(lib, g["q_idx"], g["w_idx"], g["K_I"], g["q_pos"], cfg, lib.HCA_MODE_DECODE, out)
        assert st == 0, lib.last_error()
        torch.cuda.synchronize()
        # same kernels, same inputs: identical (deterministic) index lists
        np.testing.assert_array_equal(out.cpu().numpy(), ref.cpu().numpy())


def test_noalloc_prefill_twice():
    from long_context_attention_compress_b200 import _lib as lib
    s = wl.TINY
    cfg = lib.make_cfg(s)
    d = wl.prefill_inputs(s, T=1024, seed=43)
    K = torch.randn((256, s.d_idx), generator=torch.Generator().manual_seed(44)).bfloat16()
    g = {k: v.cuda() for k, v in d.items()}
    Kc = K.cuda()
    ref = lib.csa_indexer_topk(g["q_idx"], g["w_idx"], Kc, g["q_pos"], cfg)
    for _ in range(2):
        out = torch.full_like(ref, -7)
        assert _noalloc(lib, g["q_idx"], g["w_idx"], Kc, g["q_pos"], cfg, lib.HCA_MODE_PREFILL, out) == 0
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out.cpu().numpy(), ref.cpu().numpy())


def test_noalloc_capacity_boundary():
    """5 requests x 262,144 entries fit the 16 MiB array (and match the
    workspace entry point); 6 requests need about 18.6 MiB and are refused
    with HCA_ERR_WORKSPACE before anything is launched or written."""
    from long_context_attention_compress_b200 import _lib as lib
    sp = wl.PRO
    cp = lib.make_cfg(sp)
    N = 262144
    assert lib.workspace_size(lib.HCA_OP_INDEXER_TOPK, cp, 5, N, lib.HCA_MODE_DECODE) <= 16 << 20
    assert lib.workspace_size(lib.HCA_OP_INDEXER_TOPK, cp, 6, N, lib.HCA_MODE_DECODE) > 16 << 20
    g = torch.Generator(device="cuda").manual_seed(45)
    qi = torch.randn((5, sp.n_idx_heads, sp.d_idx), generator=g, device="cuda").bfloat16()
    wi = torch.rand((5, sp.n_idx_heads), generator=g, device="cuda")
    ki = torch.randn((5, N, sp.d_idx), generator=g, device="cuda").bfloat16()
    qp = torch.full((5,), 4 * N - 1, dtype=torch.int32, device="cuda")
    ref = lib.csa_indexer_topk(qi, wi, ki, qp, cp, mode=lib.HCA_MODE_DECODE)
    for _ in range(2):
        out = torch.full_like(ref, -7)
        assert _noalloc(lib, qi, wi, ki, qp, cp, lib.HCA_MODE_DECODE, out) == 0, lib.last_error()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out.cpu().numpy(), ref.cpu().numpy())
    del ki
    # 6 requests: refused, nothing written (the keys are never read: a small stand-in suffices)
    qi6 = torch.zeros((6, sp.n_idx_heads, sp.d_idx), dtype=torch.bfloat16, device="cuda")
    wi6 = torch.zeros((6, sp.n_idx_heads), dtype=torch.float32, device="cuda")
    ki6 = torch.zeros((6, 8, sp.d_idx), dtype=torch.bfloat16, device="cuda")
    qp6 = torch.full((6,), 4 * N - 1, dtype=torch.int32, device="cuda")
    out6 = torch.full((6, sp.topk), -7, dtype=torch.int32, device="cuda")
    f = lib.lib.csa_indexer_topk_noalloc
    st = f(qi6.data_ptr(), wi6.data_ptr(), ki6.data_ptr(), N * sp.d_idx, N, qp6.data_ptr(), 6,
           lib.HCA_MODE_DECODE, ctypes.byref(cp), out6.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == -3 and "scratch" in lib.last_error()
    torch.cuda.synchronize()
    assert int(out6.min()) == -7 and int(out6.max()) == -7
