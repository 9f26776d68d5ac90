"""Python entry points of the indexer: argument marshalling onto the C ABI (include/adx.h).

Every computation runs in libadx.so's CUDA kernels; this module only checks tensor
properties, allocates outputs and workspaces with PyTorch and passes raw device pointers
and the current CUDA stream. There is no CPU or PyTorch fallback.

Tensors: q [T, H, d] bf16 or uint8 (e4m3 codes, then q_scale [T] fp32); w [T, H] fp32;
k [S, d] (prefill layout) or [T, S, d] (decode layout, with seq_len [T] int32 on the
device), bf16 or uint8 e4m3 codes with k_scale fp32 of one value per key row.
"""

import ctypes

import torch

from . import _lib as L

PAPER, WINDOW = L.ADX_BANK_PAPER, L.ADX_BANK_WINDOW


def _mode(mode):
    if isinstance(mode, str):
        return {"paper": PAPER, "window": WINDOW}[mode]
    return int(mode)


def _dtype(t):
    if t.dtype == torch.bfloat16:
        return L.ADX_BF16
    if t.dtype == torch.uint8:
        return L.ADX_E4M3
    raise TypeError(f"operand dtype {t.dtype}: expected bfloat16 or uint8 (e4m3 codes)")


def _dev(t, name, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def make_operands(q, w, k, q_scale=None, k_scale=None, q_pos0=0, seq_len=None):
    """adx_operands for these tensors (prefill layout, or decode layout when seq_len is set)."""
    _dev(q, "q"), _dev(w, "w", torch.float32), _dev(k, "k")
    _dev(q_scale, "q_scale", torch.float32), _dev(k_scale, "k_scale", torch.float32)
    _dev(seq_len, "seq_len", torch.int32)
    T, H, d = q.shape
    S = k.shape[-2]
    o = L.Operands()
    o.q_dtype, o.k_dtype = _dtype(q), _dtype(k)
    o.q, o.q_scale, o.w = q.data_ptr(), _p(q_scale), w.data_ptr()
    o.k, o.k_scale = k.data_ptr(), _p(k_scale)
    o.T, o.H, o.d, o.S = T, H, d, S
    o.q_pos0 = int(q_pos0)
    o.seq_len = _p(seq_len)
    return o


class Workspace:
    """Grow-only device workspace; its status word starts zeroed (torch.zeros)."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, nbytes):
        nbytes = max(int(nbytes), L.ADX_STATUS_BYTES)
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device or "cuda")
        return self.buf


_default_ws = {}


def _ws(ws, device):
    if ws is not None:
        return ws
    key = torch.device(device).index
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(op, ops, K=0, B=0, G=0, mode=PAPER):
    n = L.lib().adx_workspace_size(op, ctypes.byref(ops), K, B, G, _mode(mode))
    if n == 0:
        raise L.AdxError("adx_workspace_size", L.ADX_EINVAL)
    return n


def index_prefill(q, w, k, K, q_scale=None, k_scale=None, q_pos0=0, with_scores=False,
                  all_scores=False, ws=None, stream=None):
    """Flat causal indexer (Eqs. (1)-(2)). Returns (topk_idx [T, K] int32,
    topk_score [T, K] fp32 or None, scores [T, ld] fp32 or None)."""
    ops = make_operands(q, w, k, q_scale, k_scale, q_pos0)
    T, S = ops.T, ops.S
    idx = torch.empty(T, K, dtype=torch.int32, device=q.device)
    sc = torch.empty(T, K, dtype=torch.float32, device=q.device) if with_scores else None
    full, ld = None, 0
    if all_scores:
        ld = (S + 127) // 128 * 128
        full = torch.empty(T, ld, dtype=torch.float32, device=q.device)
    buf = _ws(ws, q.device).get(workspace_size(L.ADX_OP_PREFILL, ops, K))
    L.check("adx_index_prefill", L.lib().adx_index_prefill(
        ctypes.byref(ops), K, _p(idx), _p(sc), _p(full), ld, _p(buf), buf.numel(),
        _stream(stream)))
    return idx, sc, full


def index_prefill_host(q, w, k, K, q_scale=None, k_scale=None, q_pos0=0, rows_per_chunk=2048,
                       with_scores=False, out=None, ws=None, stream=None):
    """Flat causal indexer over HOST tensors (pinned for the copies to overlap the work):
    -> (topk_idx [T, K] int32, topk_score or None), host tensors, valid once `stream` (the
    current one by default) has completed. `out` may pass preallocated (pinned) outputs."""
    for name, t in (("q", q), ("w", w), ("k", k), ("q_scale", q_scale), ("k_scale", k_scale)):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous host tensor")
    T, H, d = q.shape
    o = L.Operands()
    o.q_dtype, o.k_dtype = _dtype(q), _dtype(k)
    o.q, o.q_scale, o.w = q.data_ptr(), _p(q_scale), w.data_ptr()
    o.k, o.k_scale = k.data_ptr(), _p(k_scale)
    o.T, o.H, o.d, o.S = T, H, d, k.shape[-2]
    o.q_pos0 = int(q_pos0)
    o.seq_len = None
    if out is None:
        idx = torch.empty(T, K, dtype=torch.int32).pin_memory()
        sc = torch.empty(T, K, dtype=torch.float32).pin_memory() if with_scores else None
    else:
        idx, sc = out
    need = L.lib().adx_workspace_size(L.ADX_OP_PREFILL_HOST, ctypes.byref(o), K, rows_per_chunk,
                                      0, 0)
    if need == 0:
        raise L.AdxError("adx_workspace_size", L.ADX_EINVAL)
    buf = _ws(ws, torch.device("cuda")).get(need)
    L.check("adx_index_prefill_host", L.lib().adx_index_prefill_host(
        ctypes.byref(o), K, rows_per_chunk, _p(idx), _p(sc), _p(buf), buf.numel(),
        _stream(stream)))
    return idx, sc


def index_decode(q, w, k, seq_len, K, q_scale=None, k_scale=None, with_scores=False, ws=None,
                 stream=None):
    """One decode step of the flat indexer: row t scores its own cache k[t]."""
    ops = make_operands(q, w, k, q_scale, k_scale, 0, seq_len)
    idx = torch.empty(ops.T, K, dtype=torch.int32, device=q.device)
    sc = torch.empty(ops.T, K, dtype=torch.float32, device=q.device) if with_scores else None
    buf = _ws(ws, q.device).get(workspace_size(L.ADX_OP_DECODE, ops, K))
    L.check("adx_index_decode", L.lib().adx_index_decode(
        ctypes.byref(ops), K, _p(idx), _p(sc), _p(buf), buf.numel(), _stream(stream)))
    return idx, sc


def hisa_block_keys(q, w, k, q_scale=None, k_scale=None, q_pos0=0, seq_len=None,
                    last_only=False, out=None, stream=None):
    """HISA block keys (means of 128-key blocks, bf16 for either key format) -> (kbar, None):
    [ceil(S / 128), d] (prefill) or [T, ceil(S / 128), d] (decode). `out` updates an existing
    (kbar, _) pair in place (decode steps use last_only=True)."""
    ops = make_operands(q, w, k, q_scale, k_scale, q_pos0, seq_len)
    nb = (ops.S + L.ADX_HISA_BLOCK - 1) // L.ADX_HISA_BLOCK
    shape = (nb, ops.d) if seq_len is None else (ops.T, nb, ops.d)
    if out is None:
        kbar = torch.empty(*shape, dtype=torch.bfloat16, device=k.device)
    else:
        kbar = out[0]
        _dev(kbar, "kbar", torch.bfloat16)
        if tuple(kbar.shape) != shape:
            raise ValueError(f"kbar must be {shape}")
    L.check("adx_hisa_block_keys", L.lib().adx_hisa_block_keys(
        ctypes.byref(ops), int(bool(last_only)), _p(kbar), None, _stream(stream)))
    return kbar, None


def index_hisa(q, w, k, kbar, K, n_blocks=64, q_scale=None, k_scale=None, kbar_scale=None,
               q_pos0=0, seq_len=None, with_scores=False, with_blocks=False, ws=None,
               stream=None):
    """HISA indexer (block filter, then token refinement) -> (topk_idx [T, K] int32,
    topk_score or None, blocks [T, n_blocks] int32 or None)."""
    ops = make_operands(q, w, k, q_scale, k_scale, q_pos0, seq_len)
    _dev(kbar, "kbar", torch.bfloat16)
    idx = torch.empty(ops.T, K, dtype=torch.int32, device=q.device)
    sc = torch.empty(ops.T, K, dtype=torch.float32, device=q.device) if with_scores else None
    blocks = torch.empty(ops.T, n_blocks, dtype=torch.int32, device=q.device) \
        if with_blocks else None
    need = L.lib().adx_hisa_workspace_size(ctypes.byref(ops), n_blocks, K, int(with_blocks))
    if need == 0:
        raise L.AdxError("adx_hisa_workspace_size", L.ADX_EINVAL)
    buf = _ws(ws, q.device).get(need)
    L.check("adx_index_hisa", L.lib().adx_index_hisa(
        ctypes.byref(ops), _p(kbar), None, n_blocks, K, _p(idx), _p(sc), _p(blocks),
        _p(buf), buf.numel(), _stream(stream)))
    return idx, sc, blocks


def bank_width(B, G, mode):
    return L.lib().adx_bank_width(B, G, _mode(mode))


def group_bank(qbar, wbar, k, G, B, mode, qbar_scale=None, k_scale=None, q_pos0=0,
               seq_len=None, ws=None, stream=None):
    """Shared token banks (Eq. (13)) of Ng = qbar.shape[0] groups -> bank [Ng, width] int32."""
    ops = make_operands(qbar, wbar, k, qbar_scale, k_scale, q_pos0, seq_len)
    m = _mode(mode)
    bank = torch.empty(ops.T, bank_width(B, G, m), dtype=torch.int32, device=qbar.device)
    buf = _ws(ws, qbar.device).get(workspace_size(L.ADX_OP_GROUP_BANK, ops, 0, B, G, m))
    L.check("adx_group_bank", L.lib().adx_group_bank(
        ctypes.byref(ops), G, B, m, _p(bank), _p(buf), buf.numel(), _stream(stream)))
    return bank


def bank_refine(q, w, k, bank, G, B, mode, K, q_scale=None, k_scale=None, q_pos0=0,
                seq_len=None, with_scores=False, ws=None, stream=None):
    """Query-specific refinement (Eq. (14)) -> (topk_idx [T, K], topk_score or None)."""
    ops = make_operands(q, w, k, q_scale, k_scale, q_pos0, seq_len)
    _dev(bank, "bank", torch.int32)
    m = _mode(mode)
    idx = torch.empty(ops.T, K, dtype=torch.int32, device=q.device)
    sc = torch.empty(ops.T, K, dtype=torch.float32, device=q.device) if with_scores else None
    buf = _ws(ws, q.device).get(workspace_size(L.ADX_OP_BANK_REFINE, ops, K, B, G, m))
    L.check("adx_bank_refine", L.lib().adx_bank_refine(
        ctypes.byref(ops), G, B, m, _p(bank), K, _p(idx), _p(sc), _p(buf), buf.numel(),
        _stream(stream)))
    return idx, sc


def pack_bank_keys(q, w, k, bank, G, B, k_scale=None, seq_len=None, out=None, stream=None):
    """Contiguous copy of the decode banks' key rows (decode layout, PAPER banks) ->
    (bank_keys [T, W, d] in the key format, bank_kscale [T, W] fp32 or None), W = B + G - 1.
    `out` reuses an existing pair."""
    ops = make_operands(q, w, k, None, k_scale, 0, seq_len)
    _dev(bank, "bank", torch.int32)
    W = B + G - 1
    if out is None:
        keys = torch.empty(ops.T, W, ops.d, dtype=k.dtype, device=k.device)
        ks = torch.empty(ops.T, W, dtype=torch.float32, device=k.device) \
            if k.dtype == torch.uint8 else None
    else:
        keys, ks = out
    L.check("adx_pack_bank_keys", L.lib().adx_pack_bank_keys(
        ctypes.byref(ops), G, B, _p(bank), _p(keys), _p(ks), _stream(stream)))
    return keys, ks


def bank_refine_packed(q, w, k, bank, bank_keys, bank_kscale, G, B, K, k_scale=None,
                       seq_len=None, with_scores=False, ws=None, stream=None):
    """Decode refinement (Eq. (14)) over a packed bank (pack_bank_keys) -> (topk_idx [T, K],
    topk_score or None); the post-anchor slots of bank_keys are refreshed in place."""
    ops = make_operands(q, w, k, None, k_scale, 0, seq_len)
    _dev(bank, "bank", torch.int32), _dev(bank_keys, "bank_keys")
    _dev(bank_kscale, "bank_kscale", torch.float32)
    idx = torch.empty(ops.T, K, dtype=torch.int32, device=q.device)
    sc = torch.empty(ops.T, K, dtype=torch.float32, device=q.device) if with_scores else None
    buf = _ws(ws, q.device).get(workspace_size(L.ADX_OP_BANK_REFINE_PACKED, ops, K, B, G, PAPER))
    L.check("adx_bank_refine_packed", L.lib().adx_bank_refine_packed(
        ctypes.byref(ops), G, B, _p(bank), _p(bank_keys), _p(bank_kscale), K, _p(idx), _p(sc),
        _p(buf), buf.numel(), _stream(stream)))
    return idx, sc


def index_mtp(q, w, k, seq_len, qbar, wbar, m, G, P, K, q_scale=None, k_scale=None,
              qbar_scale=None, with_scores=False, with_banks=False, ws=None, stream=None):
    """MTP target verification: Bs = len(seq_len) windows of m queries (q [Bs*m, H, d]) against
    their own caches k [Bs, S, d], with group queries qbar [Bs*m/G, H_g, d]
    -> (topk_idx [Bs*m, K], topk_score or None, candidate rows [Bs*m/G, P+m-1] or None)."""
    full = make_operands(q, w, k, q_scale, k_scale, 0, seq_len)
    _dev(qbar, "qbar"), _dev(wbar, "wbar", torch.float32)
    _dev(qbar_scale, "qbar_scale", torch.float32)
    grp = L.Operands()
    grp.q_dtype, grp.k_dtype = _dtype(qbar), full.k_dtype
    grp.q, grp.q_scale, grp.w = qbar.data_ptr(), _p(qbar_scale), wbar.data_ptr()
    grp.T, grp.H, grp.d = qbar.shape
    idx = torch.empty(full.T, K, dtype=torch.int32, device=q.device)
    sc = torch.empty(full.T, K, dtype=torch.float32, device=q.device) if with_scores else None
    banks = (torch.empty(grp.T, P + m - 1, dtype=torch.int32, device=q.device)
             if with_banks else None)
    need = L.lib().adx_mtp_workspace_size(ctypes.byref(full), ctypes.byref(grp), m, G, P, K)
    if need == 0:
        raise L.AdxError("adx_mtp_workspace_size", L.ADX_EINVAL)
    buf = _ws(ws, q.device).get(need)
    L.check("adx_index_mtp", L.lib().adx_index_mtp(
        ctypes.byref(full), ctypes.byref(grp), m, G, P, K, _p(idx), _p(sc), _p(banks), _p(buf),
        buf.numel(), _stream(stream)))
    return idx, sc, banks


def group_query_mean(q, w, G, Hg, q_scale=None, stream=None):
    """Mean-pooled group queries (the PIVOT proxy): q [T, H, d] bf16 or e4m3, w [T, H]
    -> (qbar [T // G, Hg, d] bf16, wbar [T // G, Hg] fp32)."""
    _dev(q, "q"), _dev(w, "w", torch.float32), _dev(q_scale, "q_scale", torch.float32)
    T, H, d = q.shape
    qbar = torch.empty(T // G, Hg, d, dtype=torch.bfloat16, device=q.device)
    wbar = torch.empty(T // G, Hg, dtype=torch.float32, device=q.device)
    L.check("adx_group_query_mean", L.lib().adx_group_query_mean(
        _dtype(q), q.data_ptr(), _p(q_scale), w.data_ptr(), T, H, d, G, Hg, qbar.data_ptr(),
        wbar.data_ptr(), _stream(stream)))
    return qbar, wbar


def group_indexer_queries(cq, h, w_pool, w_q, w_g, G, H_S, d, q_pos0=0, rope_dim=64,
                          rope_base=10000.0, ws=None, stream=None):
    """The group indexer of Eqs. (6)-(7): cq [T, d_c], h [T, d_h] and the weights (bf16, [out,
    in]) -> (qbar [T // G, H_S, d] bf16, wbar [T // G, H_S] fp32)."""
    for name, t in (("cq", cq), ("h", h), ("w_pool", w_pool), ("w_q", w_q), ("w_g", w_g)):
        _dev(t, name, torch.bfloat16)
    gi = L.GroupIndexer()
    gi.cq, gi.h, gi.w_pool, gi.w_q, gi.w_g = (t.data_ptr() for t in (cq, h, w_pool, w_q, w_g))
    gi.T, gi.d_c = cq.shape
    gi.d_h = h.shape[1]
    gi.H_S, gi.d, gi.rope_dim, gi.rope_base, gi.q_pos0 = H_S, d, rope_dim, rope_base, int(q_pos0)
    need = L.lib().adx_group_indexer_workspace_size(ctypes.byref(gi), G)
    if need == 0:
        raise L.AdxError("adx_group_indexer_workspace_size", L.ADX_EINVAL)
    buf = _ws(ws, cq.device).get(need)
    ng = gi.T // G
    qbar = torch.empty(ng, H_S, d, dtype=torch.bfloat16, device=cq.device)
    wbar = torch.empty(ng, H_S, dtype=torch.float32, device=cq.device)
    L.check("adx_group_indexer_queries", L.lib().adx_group_indexer_queries(
        ctypes.byref(gi), G, _p(qbar), _p(wbar), _p(buf), buf.numel(), _stream(stream)))
    return qbar, wbar


def read_device_status(ws=None, device=None, stream=None):
    """Synchronises and returns (and clears) the device status of a workspace (0 = ok)."""
    w = _ws(ws, device or torch.device("cuda"))
    if w.buf is None:
        return L.ADX_OK
    return L.lib().adx_read_device_status(_p(w.buf), _stream(stream))
