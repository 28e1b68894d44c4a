"""ctypes binding of libhca.so (argument marshalling only).

Every function here takes torch tensors that live on the CUDA device, checks
their dtype/shape/contiguity, and passes raw device pointers, sizes and the
current CUDA stream to the C ABI declared in include/hca.h.  All arithmetic
runs in the library's kernels; there is no other implementation to fall back
to: if the library is missing, importing this module raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("HCA_LIB", os.path.join(_PKG, "libhca.so"))

HCA_MODE_PREFILL = 0
HCA_MODE_DECODE = 1
HCA_OP_INDEXER_TOPK = 1
HCA_OP_SPARSE_MQA = 2

STATUS = {0: "HCA_OK", -1: "HCA_ERR_INVALID_ARG", -2: "HCA_ERR_UNSUPPORTED", -3: "HCA_ERR_WORKSPACE",
          -4: "HCA_ERR_CUDA", -5: "HCA_ERR_DEVICE_CHECK", -6: "HCA_ERR_INJECTED"}


class HcaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libhca.so not built at {LIB_PATH}; run `python -m long_context_attention_compress_b200.build`")
lib = ctypes.CDLL(LIB_PATH)

c_int, c_ll, c_size, c_float, c_void_p = ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p


class LayerCfg(ctypes.Structure):
    _fields_ = [("c", c_int), ("m", c_int), ("m_hca", c_int), ("topk", c_int), ("n_idx_heads", c_int),
                ("d_idx", c_int), ("n_heads", c_int), ("n_win", c_int), ("scale", c_float),
                ("rope_dims", c_int), ("rope_base", c_float), ("norm_eps", c_float)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("B", c_int), ("q_pos", c_void_p),
                ("csa_q", c_void_p), ("csa_q_idx", c_void_p), ("csa_w_idx", c_void_p), ("csa_kv", c_void_p),
                ("csa_k_idx", c_void_p), ("csa_N", c_int), ("csa_kv_stride", c_ll), ("csa_k_stride", c_ll),
                ("csa_win", c_void_p), ("csa_win_stride", c_ll), ("csa_topk_idx", c_void_p), ("csa_out", c_void_p),
                ("hca_q", c_void_p), ("hca_kv", c_void_p), ("hca_N", c_int), ("hca_kv_stride", c_ll),
                ("hca_block_cand", c_void_p), ("hca_block_logits", c_void_p), ("hca_block_stride", c_ll),
                ("hca_pos_bias", c_void_p), ("hca_win", c_void_p), ("hca_win_stride", c_ll), ("hca_out", c_void_p),
                ("events", c_void_p), ("n_events", c_int), ("csa_sink", c_void_p), ("hca_sink", c_void_p),
                ("csa_norm", c_void_p), ("hca_norm", c_void_p),
                ("csa_k_codes", c_void_p), ("csa_k_scales", c_void_p), ("csa_k4_stride", c_ll),
                ("block_table", c_void_p), ("bt_stride", c_ll), ("n_pool_blocks", c_int),
                ("csa_kv8", c_void_p), ("hca_kv8", c_void_p)]


class KvFp8(ctypes.Structure):
    _fields_ = [("codes", c_void_p), ("scales", c_void_p), ("rope", c_void_p), ("ld_codes", c_ll),
                ("ld_scales", c_ll), ("ld_rope", c_ll), ("seq_rows", c_ll)]


class PrefillArgs(ctypes.Structure):
    _fields_ = [("T", c_int), ("q_pos", c_void_p), ("cand", c_void_p), ("logits", c_void_p),
                ("kidx_cand", c_void_p), ("bias_csa", c_void_p), ("q_idx", c_void_p), ("w_idx", c_void_p),
                ("q", c_void_p), ("csa_kv", c_void_p), ("csa_k_idx", c_void_p), ("topk_idx", c_void_p),
                ("csa_out", c_void_p), ("bias_hca", c_void_p), ("hca_q", c_void_p), ("hca_kv", c_void_p),
                ("hca_out", c_void_p), ("events", c_void_p), ("n_events", c_int), ("csa_sink", c_void_p),
                ("hca_sink", c_void_p), ("csa_norm", c_void_p), ("hca_norm", c_void_p)]


def _sig(name, restype, argtypes):
    f = getattr(lib, name)
    f.restype = restype
    f.argtypes = argtypes
    return f


_csa_compress = _sig("csa_compress", c_int, [c_void_p, c_int, c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int,
                                             c_void_p, c_int, c_void_p])
_hca_compress = _sig("hca_compress", c_int, [c_void_p, c_int, c_void_p, c_int, c_void_p, c_int, c_int, c_ll, c_int,
                                             c_int, c_int, c_void_p, c_int, c_ll, c_void_p])
_indexer = _sig("csa_indexer_topk", c_int, [c_void_p, c_void_p, c_void_p, c_ll, c_int, c_void_p, c_int, c_int,
                                            ctypes.POINTER(LayerCfg), c_void_p, c_void_p, c_size, c_void_p])
_mqa = _sig("sparse_mqa_attend", c_int, [c_void_p, c_void_p, c_ll, c_int, c_void_p, c_int, c_int, c_void_p, c_ll,
                                         c_void_p, c_int, c_int, ctypes.POINTER(LayerCfg), c_void_p, c_int, c_void_p,
                                         c_void_p, c_size, c_void_p])
_mxfp4_quantize = _sig("mxfp4_quantize", c_int, [c_void_p, c_int, c_ll, c_int, c_int, c_void_p, c_ll, c_void_p, c_ll,
                                                 c_void_p])
_indexer_fp4 = _sig("csa_indexer_topk_fp4", c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_ll, c_int, c_void_p,
                                                    c_int, ctypes.POINTER(LayerCfg), c_void_p, c_void_p, c_size,
                                                    c_void_p])
_kv_fp8_quantize = _sig("kv_fp8_quantize", c_int, [c_void_p, c_int, c_ll, c_ll, ctypes.POINTER(LayerCfg), c_void_p,
                                                   c_ll, c_void_p, c_ll, c_void_p, c_ll, c_void_p])
_indexer_fp4_ws = _sig("csa_indexer_topk_fp4_workspace", c_size, [ctypes.POINTER(LayerCfg), c_int, c_int])
_norm_rope = _sig("rms_norm_rope", c_int, [c_void_p, c_int, c_ll, c_ll, c_int, c_int, c_void_p, c_int, c_int,
                                          c_void_p, ctypes.POINTER(LayerCfg), c_void_p, c_ll, c_ll, c_void_p])
_decode = _sig("hybrid_attn_decode", c_int, [ctypes.POINTER(LayerCfg), ctypes.POINTER(DecodeArgs), c_void_p, c_size,
                                             c_void_p])
_decode_ws = _sig("hybrid_attn_decode_workspace", c_size, [ctypes.POINTER(LayerCfg), ctypes.POINTER(DecodeArgs)])
_prefill = _sig("hybrid_attn_prefill", c_int, [ctypes.POINTER(LayerCfg), ctypes.POINTER(PrefillArgs), c_void_p,
                                               c_size, c_void_p])
_prefill_ws = _sig("hybrid_attn_prefill_workspace", c_size, [ctypes.POINTER(LayerCfg), ctypes.POINTER(PrefillArgs)])
_ws_size = _sig("hca_workspace_size", c_size, [c_int, ctypes.POINTER(LayerCfg), c_int, c_int, c_int])
_last_error = _sig("hca_last_error", ctypes.c_char_p, [])
_version = _sig("hca_version", ctypes.c_char_p, [])
_check_device = _sig("hca_check_device", c_int, [])
_last_launches = _sig("hca_last_launch_count", c_int, [])

SIZE_MAX = (1 << (8 * ctypes.sizeof(c_size))) - 1


def version() -> str:
    return _version().decode()


def last_error() -> str:
    return _last_error().decode()


def _check(status: int):
    if status != 0:
        raise HcaError(status, last_error())


def make_cfg(shape) -> LayerCfg:
    """LayerCfg from a workloads.LayerShape (or any object with the same fields)."""
    return LayerCfg(shape.c, shape.m, shape.m_hca, shape.topk, shape.n_idx_heads, shape.d_idx, shape.n_heads,
                    shape.n_win, float(shape.scale), int(shape.rope_dims), float(shape.rope_base),
                    float(shape.norm_eps))


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    return t.data_ptr()


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _workspace(nbytes: int, ws, device):
    if nbytes == SIZE_MAX:
        raise HcaError(-2, "unsupported configuration (workspace query)")
    if nbytes == 0:
        return None, 0
    if ws is None or ws.numel() * ws.element_size() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws, ws.numel() * ws.element_size()


BF16, F32, I32 = torch.bfloat16, torch.float32, torch.int32


# ----------------------------------------------------------------------------
# entry points
# ----------------------------------------------------------------------------
def csa_compress(cand, logits, pos_bias, m, out=None, stream=None):
    """Overlapped CSA compression of [T, c] candidates -> [T // m, c] (bf16).
    ``logits``/``pos_bias`` may be wider than cand (their first c channels are used)."""
    T, c = cand.shape
    if out is None:
        out = torch.empty((T // m, c), dtype=BF16, device=cand.device)
    _check(_csa_compress(_ptr(cand, BF16, "cand"), cand.stride(0), _ptr(logits, BF16, "logits"), logits.stride(0),
                         _ptr(pos_bias, F32, "pos_bias"), pos_bias.stride(0), T, c, m, _ptr(out, BF16, "out"),
                         out.stride(0), _stream(stream)))
    return out


def hca_compress(cand, logits, pos_bias, m_hca, out=None, stream=None):
    """HCA compression of [T, c] or [B, T, c] candidates -> [(B,) T // m', c]."""
    batched = cand.dim() == 3
    c3 = cand if batched else cand.unsqueeze(0)
    l3 = logits if batched else logits.unsqueeze(0)
    B, T, c = c3.shape
    if out is None:
        out = torch.empty((B, T // m_hca, c), dtype=BF16, device=cand.device)
        ret = out if batched else out[0]
    else:
        ret = out
        out = out if out.dim() == 3 else out.unsqueeze(0)
    _check(_hca_compress(_ptr(c3, BF16, "cand"), c3.stride(1), _ptr(l3, BF16, "logits"), l3.stride(1),
                         _ptr(pos_bias, F32, "pos_bias"), pos_bias.stride(0), B, c3.stride(0), T, c, m_hca,
                         _ptr(out, BF16, "out"), out.stride(1), out.stride(0), _stream(stream)))
    return ret


def workspace_size(op, cfg: LayerCfg, Tq: int, N: int, mode: int) -> int:
    return int(_ws_size(op, ctypes.byref(cfg), Tq, N, mode))


def csa_indexer_topk(q_idx, w_idx, k_idx, q_pos, cfg: LayerCfg, mode=HCA_MODE_PREFILL, out=None, ws=None,
                     stream=None):
    """Top-k entry indices [Tq, topk] (int32, -1 padded) by lightning-indexer score.
    k_idx: [N, d_I] (prefill) or [B, N, d_I] (decode, one query per request)."""
    Tq = q_idx.shape[0]
    N = k_idx.shape[-2]
    kstride = k_idx.stride(0) if k_idx.dim() == 3 else 0
    if out is None:
        out = torch.empty((Tq, cfg.topk), dtype=I32, device=q_idx.device)
    ws, nb = _workspace(workspace_size(HCA_OP_INDEXER_TOPK, cfg, Tq, N, mode), ws, q_idx.device)
    _check(_indexer(_ptr(q_idx, BF16, "q_idx"), _ptr(w_idx, F32, "w_idx"), _ptr(k_idx, BF16, "k_idx"), kstride, N,
                    _ptr(q_pos, I32, "q_pos"), Tq, mode, ctypes.byref(cfg), _ptr(out, I32, "out"),
                    None if ws is None else ws.data_ptr(), nb, _stream(stream)))
    return out


def mxfp4_quantize(x, codes=None, scales=None, stream=None):
    """MXFP4 form of the rows of x [rows, d] (bf16 or float32; d a multiple of 32):
    returns (codes uint8 [rows, d/2], scales uint8 [rows, d/32])."""
    rows, d = x.shape
    if x.dtype not in (BF16, F32):
        raise TypeError(f"x: dtype {x.dtype}")
    if codes is None:
        codes = torch.empty((rows, d // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((rows, d // 32), dtype=torch.uint8, device=x.device)
    _check(_mxfp4_quantize(_ptr(x, None, "x"), 1 if x.dtype == F32 else 0, x.stride(0), rows, d,
                           _ptr(codes, torch.uint8, "codes"), codes.stride(0), _ptr(scales, torch.uint8, "scales"),
                           scales.stride(0), _stream(stream)))
    return codes, scales


def kv_fp8_quantize(x, cfg: LayerCfg, out=None, stream=None):
    """FP8 cache form of KV rows x [..., c] (bf16 or float32): returns (codes uint8
    [..., c - rope_dims], scales float32 [..., (c - rope_dims) / 64], rope bf16
    [..., rope_dims]); `out` may give that triple to write into."""
    c = x.shape[-1]
    rows = x.numel() // c
    n, r = c - cfg.rope_dims, cfg.rope_dims
    lead = x.shape[:-1]
    if out is None:
        out = (torch.empty(lead + (n,), dtype=torch.uint8, device=x.device),
               torch.empty(lead + (n // 64,), dtype=F32, device=x.device),
               torch.empty(lead + (r,), dtype=BF16, device=x.device))
    codes, scales, rope = out
    if x.dtype not in (BF16, F32):
        raise TypeError(f"x: dtype {x.dtype}")
    _check(_kv_fp8_quantize(_ptr(x, None, "x"), 1 if x.dtype == F32 else 0, c, rows, ctypes.byref(cfg),
                            _ptr(codes, torch.uint8, "codes"), n, _ptr(scales, F32, "scales"), n // 64,
                            _ptr(rope, BF16, "rope"), r, _stream(stream)))
    return codes, scales, rope


def make_kv_fp8(codes, scales, rope):
    """KvFp8 descriptor of an FP8 cache (codes [B, N, n], scales [B, N, n/64], rope [B, N, r])."""
    d = KvFp8()
    d.codes, d.scales, d.rope = _ptr(codes, torch.uint8, "codes"), _ptr(scales, F32, "scales"), _ptr(rope, BF16, "rope")
    d.ld_codes, d.ld_scales, d.ld_rope = codes.shape[-1], scales.shape[-1], rope.shape[-1]
    d.seq_rows = codes.shape[-2] if codes.dim() == 3 else 0
    return d


def csa_indexer_topk_fp4(q_idx, w_idx, k_codes, k_scales, q_pos, cfg: LayerCfg, out=None, ws=None, stream=None):
    """Decode indexer + top-k over MXFP4 keys (k_codes [B, N_alloc, 64] uint8, k_scales
    [B, N_alloc, 4] uint8, N = q's visible range up to N_alloc) with BF16 scores."""
    B = q_idx.shape[0]
    N = k_codes.shape[1]
    if out is None:
        out = torch.empty((B, cfg.topk), dtype=I32, device=q_idx.device)
    nb = int(_indexer_fp4_ws(ctypes.byref(cfg), B, N))
    if nb == SIZE_MAX:
        raise HcaError(-2, "csa_indexer_topk_fp4: unsupported configuration")
    ws, nb = _workspace(nb, ws, q_idx.device)
    _check(_indexer_fp4(_ptr(q_idx, BF16, "q_idx"), _ptr(w_idx, F32, "w_idx"), _ptr(k_codes, torch.uint8, "k_codes"),
                        _ptr(k_scales, torch.uint8, "k_scales"), k_codes.stride(0) // 64, N,
                        _ptr(q_pos, I32, "q_pos"), B, ctypes.byref(cfg), _ptr(out, I32, "out"),
                        None if ws is None else ws.data_ptr(), nb, _stream(stream)))
    return out


def rms_norm_rope(x, gamma, cfg: LayerCfg, pos=None, pos_add=0, pos_step=0, out=None, stream=None):
    """Q/KV RMSNorm + partial RoPE of the rows of x ([n_seq, rows_per_seq, c] or [rows, c]; bf16 or
    float32), row r of sequence s at position max((pos[s] if pos else 0) + pos_add, 0) + r*pos_step.
    Returns bf16 rows of x's shape (out may be x itself for bf16 x)."""
    x3 = x if x.dim() == 3 else x.unsqueeze(0)
    n_seq, rps, c = x3.shape
    if x.dtype not in (BF16, F32):
        raise TypeError(f"x: dtype {x.dtype}")
    if out is None:
        out = torch.empty(x.shape, dtype=BF16, device=x.device)
    o3 = out if out.dim() == 3 else out.unsqueeze(0)
    _check(_norm_rope(_ptr(x, None, "x"), 1 if x.dtype == F32 else 0, x3.stride(1), x3.stride(0), n_seq, rps,
                      _ptr(pos, I32, "pos"), int(pos_add), int(pos_step), _ptr(gamma, F32, "gamma"),
                      ctypes.byref(cfg), _ptr(out, BF16, "out"), o3.stride(1), o3.stride(0), _stream(stream)))
    return out


def sparse_mqa_attend(q, kv, win, q_pos, cfg: LayerCfg, idx=None, rate=None, mode=HCA_MODE_PREFILL, out=None,
                      ws=None, stream=None, sink=None, rotate_out=False):
    """Shared-KV MQA over selected (idx) or all visible (idx=None) entries plus the window.
    kv: [N, c] (prefill) or [B, N, c] (decode); win: raw rows [T, c] (prefill) or [B, n_win, c] (decode);
    sink: optional [H] float32 sink logits (one per head, in the denominator only);
    rotate_out: turn the last cfg.rope_dims channels of each output head back by -q_pos."""
    Tq = q.shape[0]
    N = kv.shape[-2]
    kvs = kv.stride(0) if kv.dim() == 3 else 0
    # decode: elements between request windows; prefill: the raw rows' count
    ws_stride = win.stride(0) if win.dim() == 3 else win.shape[0]
    if rate is None:
        rate = cfg.m if idx is not None else cfg.m_hca
    n_idx = idx.shape[1] if idx is not None else 0
    if out is None:
        out = torch.empty_like(q)
    ws, nb = _workspace(workspace_size(HCA_OP_SPARSE_MQA, cfg, Tq, N, mode), ws, q.device)
    _check(_mqa(_ptr(q, BF16, "q"), _ptr(kv, BF16, "kv"), kvs, N, _ptr(idx, I32, "idx"), n_idx, rate,
                _ptr(win, BF16, "win"), ws_stride, _ptr(q_pos, I32, "q_pos"), Tq, mode, ctypes.byref(cfg),
                _ptr(sink, F32, "sink"), 1 if rotate_out else 0, _ptr(out, BF16, "out"),
                None if ws is None else ws.data_ptr(), nb,
                _stream(stream)))
    return out


def _events_array(events):
    if not events:
        return None, 0, None
    handles = []
    for e in events:
        if isinstance(e, torch.cuda.Event):
            if e.cuda_event == 0:
                e.record()  # creates the event lazily
            handles.append(e.cuda_event)
        else:
            handles.append(int(e))
    arr = (c_void_p * len(handles))(*handles)
    return ctypes.cast(arr, c_void_p), len(handles), arr


def make_decode_args(B, q_pos, csa=None, hca=None, csa_topk_idx=None, csa_out=None, hca_out=None, events=None,
                     csa_sink=None, hca_sink=None, csa_norm=None, hca_norm=None, csa_k4=None, csa_kv8=None,
                     hca_kv8=None):
    """Build DecodeArgs from dicts of tensors (see workloads.csa_decode_inputs /
    hca_decode_inputs); csa_sink / hca_sink: optional [H] float32 sink logits;
    csa_norm / hca_norm: optional [2, c] float32 Q/KV normalisation weights;
    csa_k4: optional (codes uint8 [B, N_alloc, 64], scales uint8 [B, N_alloc, 4]),
    the MXFP4 indexer keys of the FP4 indexer variant (see mxfp4_quantize).
    Returns (args, keepalive)."""
    a = DecodeArgs()
    # FP8 caches: (codes, scales, rope) triples from kv_fp8_quantize
    d8 = []
    for name, t in (("csa_kv8", csa_kv8), ("hca_kv8", hca_kv8)):
        if t is not None:
            desc = make_kv_fp8(*t)
            setattr(a, name, ctypes.cast(ctypes.pointer(desc), c_void_p))
            d8.append(desc)
    if csa_k4 is not None:
        codes, scales = csa_k4
        a.csa_k_codes = _ptr(codes, torch.uint8, "csa_k4 codes")
        a.csa_k_scales = _ptr(scales, torch.uint8, "csa_k4 scales")
        a.csa_k4_stride = codes.stride(0) // 64
    a.csa_sink = _ptr(csa_sink, F32, "csa_sink")
    a.hca_sink = _ptr(hca_sink, F32, "hca_sink")
    a.csa_norm = _ptr(csa_norm, F32, "csa_norm")
    a.hca_norm = _ptr(hca_norm, F32, "hca_norm")
    a.B = B
    a.q_pos = _ptr(q_pos, I32, "q_pos")
    # every tensor the struct points at stays alive with the returned keepalive
    keep = [q_pos, csa_sink, hca_sink, csa_norm, hca_norm, csa, hca, csa_topk_idx, csa_out, hca_out, csa_k4, csa_kv8,
            hca_kv8, d8]
    if csa is not None:
        a.csa_q = _ptr(csa["q"], BF16, "csa.q")
        a.csa_q_idx = _ptr(csa["q_idx"], BF16, "csa.q_idx")
        a.csa_w_idx = _ptr(csa["w_idx"], F32, "csa.w_idx")
        E = csa.get("E")  # (not read with an FP8 cache)
        a.csa_kv = _ptr(E, BF16, "csa.E")
        a.csa_k_idx = _ptr(csa.get("K_I"), BF16, "csa.K_I")  # (not read by the FP4 variant)
        a.csa_N = E.shape[1] if E is not None else csa_kv8[0].shape[1]
        a.csa_kv_stride = E.stride(0) if E is not None else 0
        a.csa_k_stride = csa["K_I"].stride(0) if csa.get("K_I") is not None else 0
        a.csa_win = _ptr(csa["win"], BF16, "csa.win")
        a.csa_win_stride = csa["win"].stride(0)
        a.csa_topk_idx = _ptr(csa_topk_idx, I32, "csa_topk_idx")
        a.csa_out = _ptr(csa_out, BF16, "csa_out")
    if hca is not None:
        a.hca_q = _ptr(hca["q"], BF16, "hca.q")
        Eh = hca.get("E_h")  # (not read with an FP8 cache)
        a.hca_kv = _ptr(Eh, BF16, "hca.E_h")
        a.hca_N = Eh.shape[1] if Eh is not None else hca_kv8[0].shape[1]
        a.hca_kv_stride = Eh.stride(0) if Eh is not None else 0
        if hca.get("block_cand") is not None:
            a.hca_block_cand = _ptr(hca["block_cand"], BF16, "hca.block_cand")
            a.hca_block_logits = _ptr(hca["block_logits"], BF16, "hca.block_logits")
            a.hca_block_stride = hca["block_cand"].stride(0)
            a.hca_pos_bias = _ptr(hca["bias_hca"], F32, "hca.bias_hca")
        a.hca_win = _ptr(hca["win"], BF16, "hca.win")
        a.hca_win_stride = hca["win"].stride(0)
        a.hca_out = _ptr(hca_out, BF16, "hca_out")
    ev, n, arr = _events_array(events)
    a.events = ev
    a.n_events = n
    keep.append(arr)
    return a, keep


def hybrid_attn_decode_workspace(cfg: LayerCfg, args: DecodeArgs) -> int:
    return int(_decode_ws(ctypes.byref(cfg), ctypes.byref(args)))


def hybrid_attn_decode(cfg: LayerCfg, args: DecodeArgs, ws=None, stream=None, device=None):
    """Run one decode step (see include/hca.h).  ``ws`` may be a preallocated uint8 tensor."""
    need = hybrid_attn_decode_workspace(cfg, args)
    ws, nb = _workspace(need, ws, device or torch.device("cuda"))
    _check(_decode(ctypes.byref(cfg), ctypes.byref(args), None if ws is None else ws.data_ptr(), nb, _stream(stream)))
    return ws


def make_prefill_args(inp, csa_kv, csa_k_idx, topk_idx, csa_out, hca_kv=None, hca_q=None, hca_out=None,
                      events=None, csa_sink=None, hca_sink=None, csa_norm=None, hca_norm=None):
    """PrefillArgs from a workloads.prefill_inputs dict (on the device) and output tensors;
    csa_sink / hca_sink: optional [H] float32 sink logits; csa_norm / hca_norm: optional
    [2, c] float32 Q/KV normalisation weights."""
    a = PrefillArgs()
    a.csa_sink = _ptr(csa_sink, F32, "csa_sink")
    a.hca_sink = _ptr(hca_sink, F32, "hca_sink")
    a.csa_norm = _ptr(csa_norm, F32, "csa_norm")
    a.hca_norm = _ptr(hca_norm, F32, "hca_norm")
    a.T = inp["cand"].shape[0]
    a.q_pos = _ptr(inp["q_pos"], I32, "q_pos")
    a.cand = _ptr(inp["cand"], BF16, "cand")
    a.logits = _ptr(inp["logits"], BF16, "logits")
    a.kidx_cand = _ptr(inp["kidx_cand"], BF16, "kidx_cand")
    a.bias_csa = _ptr(inp["bias_csa"], F32, "bias_csa")
    a.q_idx = _ptr(inp["q_idx"], BF16, "q_idx")
    a.w_idx = _ptr(inp["w_idx"], F32, "w_idx")
    a.q = _ptr(inp["q"], BF16, "q")
    a.csa_kv = _ptr(csa_kv, BF16, "csa_kv")
    a.csa_k_idx = _ptr(csa_k_idx, BF16, "csa_k_idx")
    a.topk_idx = _ptr(topk_idx, I32, "topk_idx")
    a.csa_out = _ptr(csa_out, BF16, "csa_out")
    if hca_kv is not None:
        a.bias_hca = _ptr(inp["bias_hca"], F32, "bias_hca")
        a.hca_q = _ptr(hca_q, BF16, "hca_q")
        a.hca_kv = _ptr(hca_kv, BF16, "hca_kv")
        a.hca_out = _ptr(hca_out, BF16, "hca_out")
    ev, n, arr = _events_array(events)
    a.events = ev
    a.n_events = n
    # every tensor the struct points at stays alive with the returned keepalive
    return a, [arr, inp, csa_kv, csa_k_idx, topk_idx, csa_out, hca_kv, hca_q, hca_out, csa_sink, hca_sink, csa_norm,
               hca_norm]


def hybrid_attn_prefill_workspace(cfg: LayerCfg, args: PrefillArgs) -> int:
    return int(_prefill_ws(ctypes.byref(cfg), ctypes.byref(args)))


def hybrid_attn_prefill(cfg: LayerCfg, args: PrefillArgs, ws=None, stream=None, device=None):
    need = hybrid_attn_prefill_workspace(cfg, args)
    ws, nb = _workspace(need, ws, device or torch.device("cuda"))
    _check(_prefill(ctypes.byref(cfg), ctypes.byref(args), None if ws is None else ws.data_ptr(), nb,
                    _stream(stream)))
    return ws
