"""GPU parity of the FP8 (E4M3) KV cache form against the oracle.

"DeepSeek V4 Architecture Tricks", "Partial RoPE 和 Attention Sink": the
rotary channels of the KV cache stay BF16, the other channels are stored in
FP8.  The quantiser must reproduce the oracle's cache form bit for bit (E4M3
codes decoded here from the format's definition, f32 group scales, BF16 rope
part).  A decode step whose CSA and HCA caches are stored in FP8 must match
the oracle run on its own dequantised cache (the GPU widens the rows it reads
to bf16 -- one more rounding, far inside the tolerance).
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_attention_compress_b200 import workloads as wl
from parity_util import assert_norm_close, check_topk_row, to64

pytestmark = pytest.mark.gpu


def e4m3_values(codes):
    """Values of E4M3 bytes from the format definition: sign bit 7, exponent bits 3-6
    (bias 7; field 0 = subnormal, value m/8 * 2^-6), mantissa bits 0-2."""
    b = np.asarray(codes, dtype=np.int64)
    s, e, m = b >> 7, (b >> 3) & 15, b & 7
    v = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1 + m / 8.0) * np.exp2(e - 7.0))
    return np.where(s == 1, -v, v), s


def _rows(rng, n, c):
    x = rng.normal(size=(n, c)) * 10.0 ** rng.uniform(-4, 3, size=(n, 1))
    x[0, :64] = 0.0                                                     # an all-zero group
    x[1, :64] = np.linspace(-448, 448, 64)                              # codes across the range
    x[2, :64] = 1.0
    x[2, 0] = 448.0 * 1.5                                               # amax far above the rest
    x[3, 64:128] = rng.normal(size=64) * 1e-30                          # tiny group
    x[4, 128:192] = -np.abs(x[4, 128:192])
    return x


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_kv_fp8_quantize_bit_exact(dtype):
    import long_context_attention_compress_b200 as hca
    s = wl.PRO
    cfg = hca.make_cfg(s)
    rng = np.random.default_rng(3)
    x = torch.tensor(_rows(rng, 400, s.c)).to(dtype)
    codes, scales, rope = hca.kv_fp8_quantize(x.cuda(), cfg)
    torch.cuda.synchronize()
    ref_codes, ref_scales, ref_rope = oracle.fp8_kv_quantize(to64(x), s.rope_dims)
    np.testing.assert_array_equal(scales.cpu().numpy().astype(np.float64), ref_scales)
    vals, sign = e4m3_values(codes.cpu().numpy())
    np.testing.assert_array_equal(vals, ref_codes)
    np.testing.assert_array_equal(sign == 1, np.signbit(ref_codes))   # the sign of zero too
    np.testing.assert_array_equal(to64(rope), ref_rope)
    assert not np.any(codes.cpu().numpy() & 0x7F == 0x7F), "no NaN codes"


def _deq(rows64, s):
    """The oracle's own FP8 cache form of float64 rows, dequantised."""
    return oracle.fp8_kv_dequantize(*oracle.fp8_kv_quantize(rows64, s.rope_dims))


def test_decode_with_fp8_caches():
    """Both layers read FP8 caches (CSA: 65,536 entries, HCA: 2,048 with the newest block
    compressed into its FP8 row), 2 requests at 262,144 tokens of context."""
    import long_context_attention_compress_b200 as hca
    s = wl.PRO
    B, ctx = 2, 4 * 65536
    t = ctx - 1
    csa = wl.csa_decode_inputs(s, B, ctx, seed=51)
    hcd = wl.hca_decode_inputs(s, B, ctx, seed=52, with_block=True)
    cfg = hca.make_cfg(s)
    c8 = hca.kv_fp8_quantize(csa["E"].cuda(), cfg)
    h8 = hca.kv_fp8_quantize(hcd["E_h"].cuda(), cfg)
    gc = {k: v.cuda() for k, v in csa.items() if k != "E"}
    gh = {k: v.cuda() for k, v in hcd.items() if k != "E_h"}
    idx = torch.empty((B, s.topk), dtype=torch.int32, device="cuda")
    oc = torch.empty((B, s.n_heads, s.c), dtype=torch.bfloat16, device="cuda")
    oh = torch.empty_like(oc)
    args, keep = hca.make_decode_args(B, gc["q_pos"], csa=gc, hca=gh, csa_topk_idx=idx, csa_out=oc, hca_out=oh,
                                      csa_kv8=c8, hca_kv8=h8)
    hca.hybrid_attn_decode(cfg, args)
    torch.cuda.synchronize()
    assert hca.lib.hca_check_device() == 0, hca.last_error()
    ii = idx.cpu().numpy()
    Nh = hcd["E_h"].shape[1]
    for b in range(B):
        E = _deq(to64(csa["E"][b]), s)
        r = oracle.csa_layer_decode(E, to64(csa["K_I"][b]), to64(csa["win"][b]), to64(csa["q"][b]),
                                    to64(csa["q_idx"][b]), csa["w_idx"][b].double().numpy(), t, m=s.m, topk=s.topk,
                                    n_win=s.n_win, scale=s.scale)
        check_topk_row(ii[b], r["idx"], r["scores"], s.topk, r["n_vis"])
        assert_norm_close(to64(oc[b].cpu()), r["O"], what=f"csa decode from FP8, request {b}")
        # HCA: entries 0..Nh-2 from the cache, the newest compressed here (exact), all in FP8 form
        new_exact = oracle.hca_compress(to64(hcd["block_cand"][b]), to64(hcd["block_logits"][b]),
                                        hcd["bias_hca"].double().numpy(), s.m_hca)
        Eh = _deq(np.concatenate([to64(hcd["E_h"][b, :Nh - 1]), new_exact]), s)
        o = oracle.mqa_attend(to64(hcd["q"][b]), np.concatenate([Eh, to64(hcd["win"][b])]), s.scale)
        assert_norm_close(to64(oh[b].cpu()), o, what=f"hca decode from FP8, request {b}")
        # the newest entry's FP8 row (quantised from the f32 compressor output): within one
        # E4M3 step of the exact entry's own form, the scales within f32 rounding
        got = oracle.fp8_kv_dequantize(e4m3_values(h8[0][b, Nh - 1].cpu().numpy())[0], h8[1][b, Nh - 1].cpu().numpy(),
                                       to64(h8[2][b, Nh - 1]))
        want = Eh[Nh - 1]
        sc = np.repeat(h8[1][b, Nh - 1].cpu().numpy().astype(np.float64), 64)
        n = s.c - s.rope_dims
        assert np.all(np.abs(got[:n] - want[:n]) <= 2.0 ** -3 * np.abs(want[:n]) + sc * 2.0 ** -8 + 1e-12)
        np.testing.assert_allclose(got[n:], want[n:], rtol=2 ** -7, atol=1e-6)
