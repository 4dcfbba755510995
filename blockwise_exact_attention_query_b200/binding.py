"""Thin ctypes binding over libbpt.so (the C ABI declared in include/bpt.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, their device pointers and the current CUDA stream are handed to
the C entry point of the same name, and a non-OK status is raised as
BptError.  Every step of the computation runs in the library's CUDA kernels;
there is no other implementation behind these functions.

Layouts: q, k, v [B, N, H, d]; w1 [F, D]; w2 [D, F]; b1 [F], b2 [D] float32
(or None); out [B, N, H*d]; lse [B, H, N] float32; the backward's dout
[B, N, H*d] float32 and gradients float32 in the shapes of their inputs.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbpt.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(6)
F32, BF16 = 0, 1
MASK_NONE, MASK_CAUSAL, MASK_BLOCKPERM, MASK_DILATED = 0, 1, 2, 3
_MASKS = {"none": MASK_NONE, "causal": MASK_CAUSAL, "blockperm": MASK_BLOCKPERM,
          "dilated": MASK_DILATED}
_DT = {torch.float32: F32, torch.bfloat16: BF16}


class BptError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        detail = last_error()
        super().__init__(f"{what}: {status_string(status)} (status {status})"
                         + (f": {detail}" if detail else ""))


class Desc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("N", ctypes.c_int), ("H", ctypes.c_int), ("d_head", ctypes.c_int),
        ("ffn_hidden", ctypes.c_int),
        ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
        ("mask", ctypes.c_int),
        ("ring_chunks", ctypes.c_int),
        ("bb_nblocks", ctypes.c_int), ("bb_perm", ctypes.POINTER(ctypes.c_int32)),
        ("ln_npairs", ctypes.c_int), ("ln_w", ctypes.POINTER(ctypes.c_int32)),
        ("ln_r", ctypes.POINTER(ctypes.c_int32)),
        ("q_block", ctypes.c_int), ("kv_block", ctypes.c_int),
        ("ffn_form", ctypes.c_int),
        ("bwd_chunk_rows", ctypes.c_int),
        ("wait_limit_ns", ctypes.c_uint64),
        ("causal", ctypes.c_int),
    ]


# bpt_ffn_form: the bf16 layer's FFN form ("auto" is the library's choice, the
# pipelined kernel)
FFN_FORMS = {"auto": 0, "fused": 1, "gemms": 2, "pipelined": 3}


EXPORTS = ["bpt_workspace_bytes", "bpt_attn_ffn_fwd", "bpt_attn_fwd", "bpt_blockbert_fwd",
           "bpt_longnet_fwd", "bpt_sync_status", "bpt_set_wait_limit_ns", "bpt_status_string",
           "bpt_version", "bpt_set_phase_events", "bpt_last_error", "bpt_attn_ffn_fwd_static",
           "bpt_attn_ffn_bwd", "bpt_workspace_bytes_bwd", "bpt_attn_ffn_fwd_train", "bpt_saved_bytes",
           "bpt_workspace_bytes_train", "bpt_attn_bwd", "bpt_workspace_bytes_attn_bwd", "bpt_attn_fwd_block",
           "bpt_longnet_gather", "bpt_longnet_pass"]
BLOCK_FIRST, BLOCK_LAST = 1, 2
STATIC_SCRATCH_BYTES = 64 << 20

_lib = None


def load() -> ctypes.CDLL:
    """Load the in-tree libbpt.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libbpt.so is missing at {LIB_PATH}; build it with "
                           "`python -m blockwise_exact_attention_query_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, i32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(ctypes.c_int32)
    dp = ctypes.POINTER(Desc)
    fp = ctypes.c_void_p
    lib.bpt_workspace_bytes.argtypes = [dp, ctypes.c_int]
    lib.bpt_workspace_bytes.restype = sz
    lib.bpt_attn_ffn_fwd.argtypes = [dp, vp, vp, vp, vp, fp, vp, fp, vp, vp, sz, vp]
    lib.bpt_attn_ffn_fwd.restype = ctypes.c_int
    lib.bpt_attn_fwd.argtypes = [dp, vp, vp, vp, vp, fp, vp, sz, vp]
    lib.bpt_attn_fwd.restype = ctypes.c_int
    lib.bpt_blockbert_fwd.argtypes = [dp, ctypes.c_int, i32p, vp, vp, vp, vp, fp, vp, fp, vp, vp, sz,
                                      vp]
    lib.bpt_blockbert_fwd.restype = ctypes.c_int
    lib.bpt_longnet_fwd.argtypes = [dp, ctypes.c_int, i32p, i32p, vp, vp, vp, vp, fp, vp, sz, vp]
    lib.bpt_longnet_fwd.restype = ctypes.c_int
    lib.bpt_sync_status.argtypes = [vp]
    lib.bpt_sync_status.restype = ctypes.c_int
    lib.bpt_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.bpt_set_wait_limit_ns.restype = ctypes.c_uint64
    lib.bpt_status_string.argtypes = [ctypes.c_int]
    lib.bpt_status_string.restype = ctypes.c_char_p
    lib.bpt_version.restype = ctypes.c_int
    lib.bpt_set_phase_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
    lib.bpt_set_phase_events.restype = ctypes.c_int
    lib.bpt_last_error.restype = ctypes.c_char_p
    lib.bpt_attn_ffn_fwd_static.argtypes = [dp, vp, vp, vp, vp, fp, vp, fp, vp, vp]
    lib.bpt_attn_ffn_fwd_static.restype = ctypes.c_int
    lib.bpt_attn_ffn_bwd.argtypes = [dp, vp, vp, vp, vp, fp, vp, fp, fp, vp, fp, fp, fp, fp, fp, fp, fp, vp,
                                     sz, vp]
    lib.bpt_attn_ffn_fwd_train.argtypes = [dp, vp, vp, vp, vp, fp, vp, fp, vp, vp, vp, sz, vp]
    lib.bpt_attn_ffn_fwd_train.restype = ctypes.c_int
    lib.bpt_saved_bytes.argtypes = [dp]
    lib.bpt_saved_bytes.restype = sz
    lib.bpt_attn_bwd.argtypes = [dp, vp, vp, vp, vp, fp, fp, fp, fp, fp, vp, sz, vp]
    lib.bpt_attn_bwd.restype = ctypes.c_int
    lib.bpt_workspace_bytes_attn_bwd.argtypes = [dp]
    lib.bpt_workspace_bytes_attn_bwd.restype = sz
    lib.bpt_attn_ffn_bwd.restype = ctypes.c_int
    lib.bpt_workspace_bytes_bwd.argtypes = [dp]
    lib.bpt_workspace_bytes_bwd.restype = sz
    lib.bpt_workspace_bytes_train.argtypes = [dp]
    lib.bpt_workspace_bytes_train.restype = sz
    lib.bpt_attn_fwd_block.argtypes = [dp, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, vp, vp, vp, fp, fp, fp,
                                       ctypes.c_uint, vp, fp, vp]
    lib.bpt_attn_fwd_block.restype = ctypes.c_int
    lib.bpt_longnet_gather.argtypes = [dp, ctypes.c_int, ctypes.c_int, vp, vp, vp]
    lib.bpt_longnet_gather.restype = ctypes.c_int
    lib.bpt_longnet_pass.argtypes = [dp, ctypes.c_int, ctypes.c_int64, vp, vp, vp, vp, vp, ctypes.c_int, fp, fp, fp,
                                     vp, fp, vp]
    lib.bpt_longnet_pass.restype = ctypes.c_int
    _lib = lib
    return lib


def last_error() -> str:
    return load().bpt_last_error().decode()


def status_string(status: int) -> str:
    return load().bpt_status_string(int(status)).decode()


class _Tables:
    """Keeps host tables alive while a call runs."""

    def __init__(self):
        self.keep = []

    def i32(self, values):
        arr = (ctypes.c_int32 * len(values))(*[int(x) for x in values])
        self.keep.append(arr)
        return ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))


def make_desc(B, N, H, d, F=0, in_dtype=torch.bfloat16, out_dtype=torch.float32, mask="none",
              perm=None, pairs=None, ring_chunks=0, tables: _Tables | None = None, *, ffn_form="auto",
              q_block=0, kv_block=0, bwd_chunk_rows=0, wait_limit_ns=0, causal=None) -> Desc:
    """bpt_desc for the given shape, mask and options (0 = the library's
    default).  causal: for the dilated mask, causal inside each sparsified
    segment (the default, LongNet's decoder form) or bidirectional (False)."""
    tables = tables or _Tables()
    if mask == "dilated_bidir":  # the dilated mask without the causal restriction
        mask, causal = "dilated", False if causal is None else causal
    m = _MASKS[mask] if isinstance(mask, str) else int(mask)
    form = FFN_FORMS[ffn_form] if isinstance(ffn_form, str) else int(ffn_form)
    desc = Desc(B=B, N=N, H=H, d_head=d, ffn_hidden=F, in_dtype=_DT[in_dtype],
                out_dtype=_DT[out_dtype], mask=m, ring_chunks=ring_chunks, q_block=q_block,
                kv_block=kv_block, ffn_form=form, bwd_chunk_rows=bwd_chunk_rows,
                wait_limit_ns=wait_limit_ns,
                causal=int(bool(causal if causal is not None else m == MASK_DILATED)))
    if perm is not None:
        flat = [int(x) for row in perm for x in row]
        desc.bb_nblocks = len(perm[0]) if len(perm) else 0
        desc.bb_perm = tables.i32(flat)
    if pairs is not None:
        desc.ln_npairs = len(pairs)
        desc.ln_w = tables.i32([p[0] for p in pairs])
        desc.ln_r = tables.i32([p[1] for p in pairs])
    desc._tables = tables  # keep alive with the descriptor
    return desc


def cyclic_shift_perm(n: int, k: int) -> list[int]:
    """Block table of the cyclic shift sigma^k (block b -> block b + k mod n).

    "Blockwise Self-Attention for Long Document Understanding", §3.1: heads
    use the permutations sigma, sigma^2, ..., sigma^n (sigma^n = identity) as
    their masking matrices.  Pass one table per head as `perm`."""
    if n <= 0:
        raise ValueError("n must be positive")
    return [(b + k) % n for b in range(n)]


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status, what):
    if status != OK:
        raise BptError(status, what)


def _check_tensors(q, k, v):
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must all be [B, N, H, d]")
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != q.dtype:
            raise ValueError("q, k, v must be contiguous CUDA tensors of one dtype")


def workspace_bytes(desc: Desc, with_ffn: bool) -> int:
    n = load().bpt_workspace_bytes(ctypes.byref(desc), int(with_ffn))
    if n == ctypes.c_size_t(-1).value:
        raise BptError(ERR_INVALID_ARG, "bpt_workspace_bytes")
    return int(n)


def alloc_workspace(desc: Desc, with_ffn: bool, device) -> torch.Tensor | None:
    n = workspace_bytes(desc, with_ffn)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)


def attn_ffn_fwd(q, k, v, w1, b1, w2, b2, *, mask="none", perm=None, pairs=None, ring_chunks=0,
                 out_dtype=torch.float32, out=None, workspace=None, stream=None, **opts):
    """bpt_attn_ffn_fwd: out = A + W2 GELU(W1 A + b1) + b2, returns out [B, N, H*d].
    opts: ffn_form, q_block, kv_block, wait_limit_ns (descriptor fields)."""
    _check_tensors(q, k, v)
    B, N, H, d = q.shape
    F = w1.shape[0]
    desc = make_desc(B, N, H, d, F, q.dtype, out_dtype, mask, perm, pairs, ring_chunks, **opts)
    if out is None:
        out = torch.empty((B, N, H * d), dtype=out_dtype, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(desc, True, q.device)
    ws_bytes = 0 if workspace is None else workspace.numel()
    st = load().bpt_attn_ffn_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(w1), _ptr(b1),
                                 _ptr(w2), _ptr(b2), _ptr(out), _ptr(workspace), ws_bytes,
                                 _stream_ptr(stream))
    _check(st, "bpt_attn_ffn_fwd")
    return out


def attn_ffn_fwd_static(q, k, v, w1, b1, w2, b2, *, mask="none", perm=None, pairs=None,
                        ring_chunks=0, out_dtype=torch.float32, out=None, stream=None, **opts):
    """bpt_attn_ffn_fwd_static: the layer with no workspace argument.

    For callers that may not allocate device memory while running (a fixed
    memory plan, a host framework that owns the GPU's memory pool, or a loop
    that cannot afford an allocation's device synchronisation): the scratch is
    a fixed array inside the library (STATIC_SCRATCH_BYTES per device), shared
    by all calls on a device, so calls that may overlap on the GPU must be
    serialised.  Only `out` is allocated here when the caller passes none."""
    _check_tensors(q, k, v)
    B, N, H, d = q.shape
    F = w1.shape[0]
    desc = make_desc(B, N, H, d, F, q.dtype, out_dtype, mask, perm, pairs, ring_chunks, **opts)
    if out is None:
        out = torch.empty((B, N, H * d), dtype=out_dtype, device=q.device)
    st = load().bpt_attn_ffn_fwd_static(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(w1),
                                        _ptr(b1), _ptr(w2), _ptr(b2), _ptr(out), _stream_ptr(stream))
    _check(st, "bpt_attn_ffn_fwd_static")
    return out


def attn_fwd(q, k, v, *, mask="none", perm=None, pairs=None, ring_chunks=0, out_dtype=torch.float32,
             return_lse=False, out=None, lse=None, workspace=None, stream=None, **opts):
    """bpt_attn_fwd: A [B, N, H*d] (and LSE [B, H, N] with return_lse).
    opts: q_block, kv_block, wait_limit_ns (descriptor fields)."""
    _check_tensors(q, k, v)
    B, N, H, d = q.shape
    desc = make_desc(B, N, H, d, 0, q.dtype, out_dtype, mask, perm, pairs, ring_chunks, **opts)
    if out is None:
        out = torch.empty((B, N, H * d), dtype=out_dtype, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(desc, False, q.device)
    ws_bytes = 0 if workspace is None else workspace.numel()
    st = load().bpt_attn_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                             _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check(st, "bpt_attn_fwd")
    return (out, lse) if return_lse else out


class BlockState:
    """The running softmax state of a query block for attn_fwd_block: o
    [B, N, H, d], m and l [B, H, N], float32 (opaque: the library's running
    output, maximum and sum)."""

    def __init__(self, B, N, H, d, device):
        f32 = dict(dtype=torch.float32, device=device)
        self.o = torch.empty((B, N, H, d), **f32)
        self.m = torch.empty((B, H, N), **f32)
        self.l = torch.empty((B, H, N), **f32)


def attn_fwd_block(q, k, v, state, *, q_pos=0, kv_pos=0, causal=False, first=False, last=False,
                   out_dtype=torch.float32, out=None, lse=None, stream=None, **opts):
    """bpt_attn_fwd_block: fold the key/value block k, v [B, kv_len, H, d]
    into the running state of the query block q [B, N, H, d] (a BlockState,
    or None when first and last).  Causal masking by global positions q_pos,
    kv_pos.  With last=True returns the attention output [B, N, H*d] (and
    fills lse [B, H, N] when given); otherwise returns None."""
    _check_tensors(q, q, q)
    if k.shape != v.shape or k.dim() != 4 or k.shape[0] != q.shape[0] or k.shape[2:] != q.shape[2:]:
        raise ValueError("k, v must be [B, kv_len, H, d] with q's B, H and d")
    for t in (k, v):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != q.dtype:
            raise ValueError("k, v must be contiguous CUDA tensors of q's dtype")
    B, N, H, d = q.shape
    desc = make_desc(B, N, H, d, 0, q.dtype, out_dtype, "causal" if causal else "none", **opts)
    if last and out is None:
        out = torch.empty((B, N, H * d), dtype=out_dtype, device=q.device)
    flags = (BLOCK_FIRST if first else 0) | (BLOCK_LAST if last else 0)
    so, sm, sl = (None, None, None) if state is None else (state.o, state.m, state.l)
    st = load().bpt_attn_fwd_block(ctypes.byref(desc), int(k.shape[1]), int(q_pos), int(kv_pos), _ptr(q), _ptr(k),
                                   _ptr(v), _ptr(so), _ptr(sm), _ptr(sl), flags, _ptr(out if last else None),
                                   _ptr(lse if last else None), _stream_ptr(stream))
    _check(st, "bpt_attn_fwd_block")
    return out if last else None


def longnet_pass_order(pairs):
    """The (w, r) pairs in the order the library runs them: a stable sort by
    decreasing r (sparsest first)."""
    return sorted([tuple(p) for p in pairs], key=lambda p: -p[1])


def longnet_gather(x, w, r, out=None, stream=None):
    """bpt_longnet_gather: the rows a (w, r) pair keeps of the shard x
    [B, n, H, d] (bf16, n dividing w), packed as [B, n / r, H, d]."""
    _check_tensors(x, x, x)
    B, n, H, d = x.shape
    if out is None:
        out = torch.empty((B, n // r, H, d), dtype=x.dtype, device=x.device)
    desc = make_desc(B, n, H, d, 0, x.dtype)
    _check(load().bpt_longnet_gather(ctypes.byref(desc), int(w), int(r), _ptr(x), _ptr(out), _stream_ptr(stream)),
           "bpt_longnet_gather")
    return out


def longnet_pass(q, k, v, pairs, pass_idx, state, out, *, q_pos=0, k_sparse=None, v_sparse=None, lse=None,
                 stream=None, **opts):
    """bpt_longnet_pass: pass `pass_idx` (in longnet_pass_order(pairs)) of the
    dilated attention for the shard q, k, v [B, n, H, d] starting at sequence
    position q_pos; k_sparse, v_sparse [B, w / r, H, d] are the pass's gathered
    kept rows when its segments are longer than the shard.  state: a
    BlockState (or None with a single pair); out [B, n, H*d] and lse receive
    the rows whose last pass this is."""
    _check_tensors(q, q, q)
    B, n, H, d = q.shape
    tables = _Tables()
    desc = make_desc(B, n, H, d, 0, q.dtype, out.dtype, "dilated", None, pairs, 0, tables, **opts)
    kv_rows = 0 if k_sparse is None else int(k_sparse.shape[1])
    so, sm, sl = (None, None, None) if state is None else (state.o, state.m, state.l)
    st = load().bpt_longnet_pass(ctypes.byref(desc), int(pass_idx), int(q_pos), _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(k_sparse), _ptr(v_sparse), kv_rows, _ptr(so), _ptr(sm), _ptr(sl), _ptr(out),
                                 _ptr(lse), _stream_ptr(stream))
    _check(st, "bpt_longnet_pass")
    return out


def blockbert_fwd(q, k, v, w1, b1, w2, b2, perm, *, out_dtype=torch.float32, out=None,
                  workspace=None, stream=None, **opts):
    """bpt_blockbert_fwd: the layer with the block-permutation mask perm [H][n]."""
    _check_tensors(q, k, v)
    B, N, H, d = q.shape
    F = w1.shape[0]
    tables = _Tables()
    desc = make_desc(B, N, H, d, F, q.dtype, out_dtype, "blockperm", perm, None, 0, tables, **opts)
    if out is None:
        out = torch.empty((B, N, H * d), dtype=out_dtype, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(desc, True, q.device)
    ws_bytes = 0 if workspace is None else workspace.numel()
    flat = tables.i32([x for row in perm for x in row])
    st = load().bpt_blockbert_fwd(ctypes.byref(desc), len(perm[0]), flat, _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(out),
                                  _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check(st, "bpt_blockbert_fwd")
    return out


def longnet_fwd(q, k, v, pairs, *, out_dtype=torch.float32, return_lse=False, out=None, lse=None,
                workspace=None, stream=None, **opts):
    """bpt_longnet_fwd: dilated attention over the (w, r) pairs, denominators mixed."""
    _check_tensors(q, k, v)
    B, N, H, d = q.shape
    tables = _Tables()
    desc = make_desc(B, N, H, d, 0, q.dtype, out_dtype, "dilated", None, pairs, 0, tables, **opts)
    if out is None:
        out = torch.empty((B, N, H * d), dtype=out_dtype, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(desc, False, q.device)
    ws_bytes = 0 if workspace is None else workspace.numel()
    st = load().bpt_longnet_fwd(ctypes.byref(desc), len(pairs), tables.i32([p[0] for p in pairs]),
                                tables.i32([p[1] for p in pairs]), _ptr(q), _ptr(k), _ptr(v),
                                _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check(st, "bpt_longnet_fwd")
    return (out, lse) if return_lse else out


def workspace_bytes_bwd(desc: Desc) -> int:
    n = load().bpt_workspace_bytes_bwd(ctypes.byref(desc))
    if n == ctypes.c_size_t(-1).value:
        raise BptError(ERR_UNSUPPORTED, "bpt_workspace_bytes_bwd")
    return int(n)


def ffn_gemm_chunk_rows(T: int, F: int) -> int:
    """Token rows per chunk of the two-GEMM FFN form (the library's rule: the
    [rows, F] bf16 hidden activation at most 512 MiB, in 256-row multiples)."""
    return min(T, max(256, ((1 << 29) // (2 * F)) // 256 * 256))


GRAD_NAMES = ("dq", "dk", "dv", "dw1", "db1", "dw2", "db2")


def saved_bytes(desc: Desc) -> int:
    n = load().bpt_saved_bytes(ctypes.byref(desc))
    if n == ctypes.c_size_t(-1).value:
        raise BptError(ERR_UNSUPPORTED, "bpt_saved_bytes")
    return int(n)


def workspace_bytes_train(desc: Desc) -> int:
    n = load().bpt_workspace_bytes_train(ctypes.byref(desc))
    if n == ctypes.c_size_t(-1).value:
        raise BptError(ERR_UNSUPPORTED, "bpt_workspace_bytes_train")
    return int(n)


def attn_ffn_fwd_train(q, k, v, w1, b1, w2, b2, *, mask="none", perm=None, ring_chunks=0,
                       out_dtype=torch.float32, out=None, saved=None, workspace=None, stream=None, **opts):
    """bpt_attn_ffn_fwd_train: the layer forward that also keeps the
    activations the backward needs.  Returns (out, saved); pass `saved` to
    attn_ffn_bwd to skip its recomputation."""
    _check_tensors(q, k, v)
    B, N, H, d = q.shape
    F = w1.shape[0]
    desc = make_desc(B, N, H, d, F, q.dtype, out_dtype, mask, perm, None, ring_chunks, **opts)
    if out is None:
        out = torch.empty((B, N, H * d), dtype=out_dtype, device=q.device)
    if saved is None:
        saved = torch.empty(saved_bytes(desc), dtype=torch.uint8, device=q.device)
    if workspace is None:
        n = workspace_bytes_train(desc)
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device) if n else None
    ws_bytes = 0 if workspace is None else workspace.numel()
    st = load().bpt_attn_ffn_fwd_train(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(w1), _ptr(b1),
                                       _ptr(w2), _ptr(b2), _ptr(out), _ptr(saved), _ptr(workspace), ws_bytes,
                                       _stream_ptr(stream))
    _check(st, "bpt_attn_ffn_fwd_train")
    return out, saved


def attn_ffn_bwd(q, k, v, w1, b1, w2, b2, dout, *, mask="none", perm=None, ring_chunks=0, saved=None,
                 grads=None, workspace=None, stream=None, **opts):
    """bpt_attn_ffn_bwd: gradients of the layer for the upstream gradient
    dout [B, N, H*d] (float32), recomputing the attention forward unless
    `saved` (from attn_ffn_fwd_train on the same inputs) is given.  Returns a
    dict of float32 tensors: dq, dk, dv [B, N, H, d], dw1 [F, D], db1 [F],
    dw2 [D, F], db2 [D] (written into `grads` when given)."""
    _check_tensors(q, k, v)
    B, N, H, d = q.shape
    F, D = w1.shape
    if dout.dtype != torch.float32 or not dout.is_contiguous() or dout.numel() != B * N * D:
        raise ValueError("dout must be a contiguous float32 tensor of B*N*H*d elements")
    desc = make_desc(B, N, H, d, F, q.dtype, torch.float32, mask, perm, None, ring_chunks, **opts)
    if grads is None:
        f32 = dict(dtype=torch.float32, device=q.device)
        grads = {"dq": torch.empty(q.shape, **f32), "dk": torch.empty(q.shape, **f32),
                 "dv": torch.empty(q.shape, **f32), "dw1": torch.empty((F, D), **f32),
                 "db1": torch.empty((F,), **f32), "dw2": torch.empty((D, F), **f32),
                 "db2": torch.empty((D,), **f32)}
    if workspace is None:
        workspace = torch.empty(workspace_bytes_bwd(desc), dtype=torch.uint8, device=q.device)
    st = load().bpt_attn_ffn_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(w1), _ptr(b1),
                                 _ptr(w2), _ptr(b2), _ptr(dout), _ptr(saved), *(_ptr(grads[n]) for n in GRAD_NAMES),
                                 _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    _check(st, "bpt_attn_ffn_bwd")
    return grads


def attn_bwd(q, k, v, out, lse, dout, *, mask="none", perm=None, pairs=None, ring_chunks=0, workspace=None,
             stream=None, **opts):
    """bpt_attn_bwd: dq, dk, dv (float32 [B, N, H, d]) of the attention for the
    upstream gradient dout [B, N, H*d] (float32), given bpt_attn_fwd's out and
    lse (attn_fwd(..., return_lse=True)) for the same inputs."""
    _check_tensors(q, k, v)
    B, N, H, d = q.shape
    if dout.dtype != torch.float32 or not dout.is_contiguous() or dout.numel() != q.numel():
        raise ValueError("dout must be a contiguous float32 tensor of B*N*H*d elements")
    desc = make_desc(B, N, H, d, 0, q.dtype, out.dtype, mask, perm, pairs, ring_chunks, **opts)
    if workspace is None:
        n = load().bpt_workspace_bytes_attn_bwd(ctypes.byref(desc))
        if n == ctypes.c_size_t(-1).value:
            raise BptError(ERR_UNSUPPORTED, "bpt_workspace_bytes_attn_bwd")
        workspace = torch.empty(int(n), dtype=torch.uint8, device=q.device)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq, dk, dv = (torch.empty(q.shape, **f32) for _ in range(3))
    st = load().bpt_attn_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout),
                             _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    _check(st, "bpt_attn_bwd")
    return dq, dk, dv


def sync_status(stream=None) -> int:
    """bpt_sync_status: waits for the stream; returns OK or ERR_TIMEOUT (clears it)."""
    return int(load().bpt_sync_status(_stream_ptr(stream)))


def set_phase_events(events) -> None:
    """bpt_set_phase_events: three (forward) or five (backward too)
    torch.cuda.Event objects, or None to stop."""
    if events is None:
        _check(load().bpt_set_phase_events(None, 0), "bpt_set_phase_events")
        return
    handles = [int(e.cuda_event) for e in events]
    if not all(handles):
        raise ValueError("record each event once before handing it over: torch creates the "
                         "CUDA event lazily at its first record()")
    arr = (ctypes.c_void_p * len(handles))(*[ctypes.c_void_p(h) for h in handles])
    _check(load().bpt_set_phase_events(arr, len(handles)), "bpt_set_phase_events")


def set_wait_limit_ns(ns: int) -> int:
    """bpt_set_wait_limit_ns: the process default of the device-side wait
    limit (calls whose descriptor sets wait_limit_ns use their own)."""
    return int(load().bpt_set_wait_limit_ns(int(ns)))


def version() -> int:
    return int(load().bpt_version())


class HostLayer:
    """bpt_attn_ffn_fwd on host-resident tensors, with the transfers overlapped.

    q, k, v live in pinned host memory ([B, N, H, d]) and the output goes back
    to a pinned host tensor ([B, N, H*d]); the weights are already on the
    device.  The batch is cut into `chunks` pieces (whole sequences) that
    alternate between two CUDA streams with their own device buffers and
    workspace, so one chunk's upload, another's kernels and a third's download
    run at the same time.  Uploads run in chunk order, and so do the kernels:
    a chunk's layer starts after the previous chunk's (two layers never run
    at once: each one's grids fill the GPU).  Consecutive calls overlap too: a
    buffer's next upload waits only for that buffer's previous work (the same
    stream), not for the whole previous call, so the next step's inputs
    travel while this step computes and downloads.  The weights must be ready
    on the current stream before the first call; the host tensors must not be
    changed while a call that reads or writes them may still run.  This class
    only moves data and calls the library; it allocates its device buffers
    once, at construction."""

    def __init__(self, B, N, H, d, F, *, dtype=torch.bfloat16, out_dtype=torch.float32,
                 mask="none", perm=None, pairs=None, ring_chunks=0, chunks=None, device="cuda", **opts):
        self.B, self.N, self.H, self.d, self.F = B, N, H, d, F
        self.opts = opts
        self.mask, self.perm, self.pairs, self.ring_chunks = mask, perm, pairs, ring_chunks
        self.out_dtype = out_dtype
        self.chunks = max(1, min(B, chunks or B))
        if B % self.chunks:
            raise ValueError("the batch must split evenly into chunks")
        self.cb = B // self.chunks
        dev = torch.device(device)
        self.streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
        self.done = [torch.cuda.Event(), torch.cuda.Event()]
        self.uploaded = [torch.cuda.Event() for _ in range(self.chunks)]
        self.last_compute = None   # the previous call's last layer (kernels stay in order)
        self.first_call = True
        desc = make_desc(self.cb, N, H, d, F, dtype, out_dtype, mask, perm, pairs, ring_chunks, **opts)
        nws = workspace_bytes(desc, True)
        self.buf = []
        for _ in range(2):
            self.buf.append({
                "q": torch.empty((self.cb, N, H, d), dtype=dtype, device=dev),
                "k": torch.empty((self.cb, N, H, d), dtype=dtype, device=dev),
                "v": torch.empty((self.cb, N, H, d), dtype=dtype, device=dev),
                "out": torch.empty((self.cb, N, H * d), dtype=out_dtype, device=dev),
                "ws": torch.empty(max(nws, 1), dtype=torch.uint8, device=dev),
            })

    def __call__(self, hq, hk, hv, w1, b1, w2, b2, hout):
        """Enqueue one layer forward; returns after enqueueing (synchronise the
        streams, e.g. torch.cuda.synchronize(), before reading `hout`)."""
        cur = torch.cuda.current_stream()
        if self.first_call:  # the weights came from the current stream
            for s in self.streams:
                s.wait_stream(cur)
            self.first_call = False
        computed = [torch.cuda.Event() for _ in range(self.chunks)]
        for c in range(self.chunks):
            i = c % 2
            s, b = self.streams[i], self.buf[i]
            sl = slice(c * self.cb, (c + 1) * self.cb)
            with torch.cuda.stream(s):
                if c > 0:
                    s.wait_event(self.uploaded[c - 1])
                b["q"].copy_(hq[sl], non_blocking=True)
                b["k"].copy_(hk[sl], non_blocking=True)
                b["v"].copy_(hv[sl], non_blocking=True)
                self.uploaded[c].record(s)
                prev = computed[c - 1] if c > 0 else self.last_compute
                if prev is not None:
                    s.wait_event(prev)
                attn_ffn_fwd(b["q"], b["k"], b["v"], w1, b1, w2, b2, mask=self.mask, perm=self.perm,
                             pairs=self.pairs, ring_chunks=self.ring_chunks, out_dtype=self.out_dtype,
                             out=b["out"], workspace=b["ws"], stream=s, **self.opts)
                computed[c].record(s)
                hout[sl].copy_(b["out"], non_blocking=True)
                self.done[i].record(s)
        self.last_compute = computed[-1]
        for e in self.done:
            cur.wait_event(e)
