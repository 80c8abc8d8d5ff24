"""Thin ctypes binding of libbbattn.so (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of the method: tensors are checked for device, dtype and
contiguity, their data pointers and sizes are passed through, and a non-OK
status raises BBError.  The library is loaded on first use; if it is missing
the call raises (there is no fallback of any kind).
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbbattn.so")

BB_OK = 0
BB_ERR_WORKSPACE = -4
BB_ERR_TIMEOUT = -5
BB_ERR_BAD_TABLE = -6
BB_F32 = 0
BB_BF16 = 1
STATUS = {0: "BB_OK", -1: "BB_ERR_INVALID", -2: "BB_ERR_UNSUPPORTED",
          -3: "BB_ERR_CUDA", -4: "BB_ERR_WORKSPACE", -5: "BB_ERR_TIMEOUT",
          -6: "BB_ERR_BAD_TABLE"}


class BBError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} "
                         f"({bb_status_str(code)})")


class bb_attn_desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int),
                ("d", ctypes.c_int), ("block_size", ctypes.c_int),
                ("r", ctypes.c_int), ("dtype", ctypes.c_int),
                ("scale", ctypes.c_float), ("mask_value", ctypes.c_float),
                ("dropout", ctypes.c_float), ("dropout_seed", ctypes.c_uint64),
                ("mask_queries", ctypes.c_int), ("grad_fp32", ctypes.c_int),
                ("dropout_bits", ctypes.c_void_p)]


_lib = None
_P = ctypes.c_void_p


def lib():
    """The loaded library (raises OSError if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} is missing: build it with "
                          "`python -m block_sparse_long_bwd_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.bb_abi_version.restype = ctypes.c_int
        L.bb_status_str.argtypes = [ctypes.c_int]
        L.bb_status_str.restype = ctypes.c_char_p
        L.bb_rand_attn_build.argtypes = [ctypes.c_uint64, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, _P]
        L.bb_rand_attn_build.restype = ctypes.c_int
        L.bb_rand_attn_build_ex.argtypes = [ctypes.c_uint64] + [
            ctypes.c_int] * 5 + [_P]
        L.bb_rand_attn_build_ex.restype = ctypes.c_int
        L.bb_attn_workspace_size.argtypes = [
            ctypes.POINTER(bb_attn_desc), ctypes.c_int,
            ctypes.POINTER(ctypes.c_size_t)]
        L.bb_attn_workspace_size.restype = ctypes.c_int
        L.bb_attn_dropout_bits_size.argtypes = [
            ctypes.POINTER(bb_attn_desc), ctypes.POINTER(ctypes.c_size_t)]
        L.bb_attn_dropout_bits_size.restype = ctypes.c_int
        L.bb_attn_fwd.argtypes = [ctypes.POINTER(bb_attn_desc)] + [_P] * 8 + [
            ctypes.c_size_t, _P]
        L.bb_attn_fwd.restype = ctypes.c_int
        L.bb_attn_bwd.argtypes = [ctypes.POINTER(bb_attn_desc)] + [_P] * 12 + [
            ctypes.c_size_t, _P]
        L.bb_attn_bwd.restype = ctypes.c_int
        L.bb_attn_launch_count.argtypes = [ctypes.POINTER(bb_attn_desc),
                                           ctypes.c_int,
                                           ctypes.POINTER(ctypes.c_int)]
        L.bb_attn_launch_count.restype = ctypes.c_int
        L.bb_attn_launch_name.argtypes = [ctypes.POINTER(bb_attn_desc),
                                          ctypes.c_int, ctypes.c_int,
                                          ctypes.POINTER(ctypes.c_char_p)]
        L.bb_attn_launch_name.restype = ctypes.c_int
        L.bb_attn_fwd_events.argtypes = (
            [ctypes.POINTER(bb_attn_desc)] + [_P] * 8
            + [ctypes.c_size_t, _P, ctypes.POINTER(_P), ctypes.c_int])
        L.bb_attn_fwd_events.restype = ctypes.c_int
        L.bb_attn_bwd_events.argtypes = (
            [ctypes.POINTER(bb_attn_desc)] + [_P] * 12
            + [ctypes.c_size_t, _P, ctypes.POINTER(_P), ctypes.c_int])
        L.bb_attn_bwd_events.restype = ctypes.c_int
        L.bb_attn_fwd_noalloc.argtypes = [ctypes.POINTER(bb_attn_desc)] + [
            _P] * 8
        L.bb_attn_fwd_noalloc.restype = ctypes.c_int
        L.bb_qkv_proj.argtypes = [ctypes.c_int] * 4 + [_P] * 7 + [ctypes.c_size_t, _P]
        L.bb_qkv_proj.restype = ctypes.c_int
        L.bb_out_proj.argtypes = [ctypes.c_int] * 4 + [_P] * 5 + [ctypes.c_size_t, _P]
        L.bb_out_proj.restype = ctypes.c_int
        L.bb_attn_noalloc_status.argtypes = [_P]
        L.bb_attn_noalloc_status.restype = ctypes.c_int
        L.bb_attn_check_status.argtypes = [_P, _P]
        L.bb_attn_check_status.restype = ctypes.c_int
        L.bb_debug_wait_probe.argtypes = [_P, ctypes.c_size_t, ctypes.c_int,
                                          _P]
        L.bb_debug_wait_probe.restype = ctypes.c_int
        _lib = L
    return _lib


def bb_status_str(code):
    return lib().bb_status_str(int(code)).decode()


def bb_abi_version():
    return lib().bb_abi_version()


def make_desc(B, H, L, d, block_size, r, dtype, scale=0.0, mask_value=0.0,
              dropout=0.0, dropout_seed=0, mask_queries=0, grad_fp32=0,
              dropout_bits=None):
    """dropout_bits: None or a contiguous CUDA uint8 tensor of
    bb_attn_dropout_bits_size bytes (the forward's keep decisions for the
    backward); the descriptor holds its address, not a reference."""
    if isinstance(dtype, torch.dtype):
        dtype = {torch.float32: BB_F32, torch.bfloat16: BB_BF16}[dtype]
    if dropout_bits is not None:
        _cuda_tensor(dropout_bits, "dropout_bits", torch.uint8)
    return bb_attn_desc(B, H, L, d, block_size, r, dtype, scale, mask_value,
                        dropout, dropout_seed & ((1 << 64) - 1),
                        int(mask_queries), int(grad_fp32), _ptr(dropout_bits))


def bb_attn_dropout_bits_size(desc):
    n = ctypes.c_size_t(0)
    _check(lib().bb_attn_dropout_bits_size(ctypes.byref(desc),
                                           ctypes.byref(n)),
           "bb_attn_dropout_bits_size")
    return n.value


def grad_dtype(desc):
    """torch dtype of dq, dk, dv for `desc` (fp32 when grad_fp32 is set or
    the I/O dtype is fp32, else bf16)."""
    if desc.grad_fp32 or desc.dtype == BB_F32:
        return torch.float32
    return torch.bfloat16


def _check(code, what):
    if code != BB_OK:
        raise BBError(code, what)


def bb_rand_attn_build(seed, heads, num_blocks, r):
    """int32 CPU tensor [heads, num_blocks, r] (see include/bb_attn.h)."""
    out = torch.empty((heads, num_blocks, r), dtype=torch.int32)
    _check(lib().bb_rand_attn_build(seed, heads, num_blocks, r,
                                    out.data_ptr() if out.numel() else None),
           "bb_rand_attn_build")
    return out


def bb_rand_attn_build_ex(seed, heads, num_blocks, r, max_blocks=0,
                          last_block=0):
    """int32 CPU tensor [heads, num_blocks, r] drawn for a table of
    max_blocks blocks with random ids capped below last_block (see
    include/bb_attn.h)."""
    out = torch.empty((heads, num_blocks, r), dtype=torch.int32)
    _check(lib().bb_rand_attn_build_ex(seed, heads, num_blocks, r, max_blocks,
                                       last_block,
                                       out.data_ptr() if out.numel() else None),
           "bb_rand_attn_build_ex")
    return out


def bb_attn_workspace_size(desc, pass_):
    n = ctypes.c_size_t(0)
    _check(lib().bb_attn_workspace_size(ctypes.byref(desc), pass_,
                                        ctypes.byref(n)),
           "bb_attn_workspace_size")
    return n.value


def bb_attn_launch_count(desc, pass_):
    n = ctypes.c_int(0)
    _check(lib().bb_attn_launch_count(ctypes.byref(desc), pass_,
                                      ctypes.byref(n)),
           "bb_attn_launch_count")
    return n.value


def bb_attn_launch_name(desc, pass_, index):
    s = ctypes.c_char_p()
    _check(lib().bb_attn_launch_name(ctypes.byref(desc), pass_, index,
                                     ctypes.byref(s)),
           "bb_attn_launch_name")
    return s.value.decode()


def _event_array(events):
    """ctypes array of raw cudaEvent_t handles of recorded torch events."""
    arr = (_P * len(events))()
    for i, e in enumerate(events):
        arr[i] = e.cuda_event
    return arr, len(events)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _cuda_tensor(t, name, dtype=None):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")


def desc_for(q, block_size, r, scale=0.0, mask_value=0.0, dropout=0.0,
             dropout_seed=0):
    B, H, L, d = q.shape
    return make_desc(B, H, L, d, block_size, r, q.dtype, scale, mask_value,
                     dropout, dropout_seed)


def bb_attn_fwd(desc, q, k, v, key_mask, rand_idx, out, lse, workspace,
                stream=None, events=None):
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        _cuda_tensor(t, name, q.dtype)
    _cuda_tensor(lse, "lse", torch.float32)
    _cuda_tensor(workspace, "workspace")
    if key_mask is not None:
        _cuda_tensor(key_mask, "key_mask", torch.uint8)
    if rand_idx is not None:
        _cuda_tensor(rand_idx, "rand_idx", torch.int32)
    args = (ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(key_mask),
            _ptr(rand_idx), _ptr(out), _ptr(lse), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if events is None:
        _check(lib().bb_attn_fwd(*args), "bb_attn_fwd")
    else:
        arr, n = _event_array(events)
        _check(lib().bb_attn_fwd_events(*args, arr, n), "bb_attn_fwd_events")


def bb_attn_fwd_noalloc(desc, q, k, v, key_mask, rand_idx, out, lse,
                        stream=None):
    """Forward using the library's built-in scratch instead of a workspace
    (for callers that cannot allocate; see include/bb_attn.h)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        _cuda_tensor(t, name, q.dtype)
    _cuda_tensor(lse, "lse", torch.float32)
    if key_mask is not None:
        _cuda_tensor(key_mask, "key_mask", torch.uint8)
    if rand_idx is not None:
        _cuda_tensor(rand_idx, "rand_idx", torch.int32)
    _check(lib().bb_attn_fwd_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k),
                                     _ptr(v), _ptr(key_mask), _ptr(rand_idx),
                                     _ptr(out), _ptr(lse),
                                     _stream_ptr(stream)),
           "bb_attn_fwd_noalloc")


def bb_attn_bwd(desc, q, k, v, out, lse, dout, key_mask, rand_idx, dq, dk, dv,
                workspace, stream=None, events=None):
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out),
                    ("dout", dout)):
        _cuda_tensor(t, name, q.dtype)
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _cuda_tensor(t, name, grad_dtype(desc))
    _cuda_tensor(lse, "lse", torch.float32)
    _cuda_tensor(workspace, "workspace")
    if key_mask is not None:
        _cuda_tensor(key_mask, "key_mask", torch.uint8)
    if rand_idx is not None:
        _cuda_tensor(rand_idx, "rand_idx", torch.int32)
    args = (ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
            _ptr(lse), _ptr(dout), _ptr(key_mask), _ptr(rand_idx), _ptr(dq),
            _ptr(dk), _ptr(dv), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if events is None:
        _check(lib().bb_attn_bwd(*args), "bb_attn_bwd")
    else:
        arr, n = _event_array(events)
        _check(lib().bb_attn_bwd_events(*args, arr, n), "bb_attn_bwd_events")


def bb_qkv_proj(x, w_qkv, b_qkv, H, workspace, q=None, k=None, v=None, stream=None):
    """Fused Q/K/V projection (see include/bb_attn.h): x [B, L, hidden] bf16,
    w_qkv [3*H*64, hidden] bf16, b_qkv [3*H*64] fp32 or None; returns q, k, v
    [B, H, L, 64] bf16."""
    B, L, hidden = x.shape
    _cuda_tensor(x, "x", torch.bfloat16)
    _cuda_tensor(w_qkv, "w_qkv", torch.bfloat16)
    if b_qkv is not None:
        _cuda_tensor(b_qkv, "b_qkv", torch.float32)
    _cuda_tensor(workspace, "workspace")
    out = []
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t is None:
            t = torch.empty((B, H, L, 64), dtype=torch.bfloat16, device=x.device)
        _cuda_tensor(t, name, torch.bfloat16)
        out.append(t)
    _check(lib().bb_qkv_proj(B, L, hidden, H, _ptr(x), _ptr(w_qkv), _ptr(b_qkv),
                             _ptr(out[0]), _ptr(out[1]), _ptr(out[2]), _ptr(workspace),
                             workspace.numel() * workspace.element_size(),
                             _stream_ptr(stream)), "bb_qkv_proj")
    return tuple(out)


def bb_out_proj(o, w_o, b_o, workspace, out=None, stream=None):
    """Output projection (see include/bb_attn.h): o [B, H, L, 64] bf16,
    w_o [hidden, H*64] bf16, b_o [hidden] fp32 or None; returns out
    [B, L, hidden] bf16."""
    B, H, L, d = o.shape
    hidden = w_o.shape[0]
    _cuda_tensor(o, "o", torch.bfloat16)
    _cuda_tensor(w_o, "w_o", torch.bfloat16)
    if b_o is not None:
        _cuda_tensor(b_o, "b_o", torch.float32)
    _cuda_tensor(workspace, "workspace")
    if out is None:
        out = torch.empty((B, L, hidden), dtype=torch.bfloat16, device=o.device)
    _cuda_tensor(out, "out", torch.bfloat16)
    _check(lib().bb_out_proj(B, L, H, hidden, _ptr(o), _ptr(w_o), _ptr(b_o), _ptr(out),
                             _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _stream_ptr(stream)), "bb_out_proj")
    return out


def bb_attn_noalloc_status(stream=None):
    """Status word the last bb_attn_fwd_noalloc left in the built-in
    scratch (waits for the stream)."""
    return lib().bb_attn_noalloc_status(_stream_ptr(stream))


def bb_attn_check_status(workspace, stream=None):
    return lib().bb_attn_check_status(_ptr(workspace), _stream_ptr(stream))


def make_table(seed, H, L, block_size, r, max_rand_mask_length=0,
               last_idx=0):
    """Random block table [H, L // block_size, r] (int32, CPU) for a call of
    length L.  max_rand_mask_length, last_idx: the pages' layer options in
    tokens (0 = off), converted to blocks by floor division; seed is the
    layer index there."""
    nb = L // block_size
    if max_rand_mask_length or last_idx:
        return bb_rand_attn_build_ex(seed, H, nb, r,
                                     max_rand_mask_length // block_size,
                                     last_idx // block_size)
    return bb_rand_attn_build(seed, H, nb, r)


def bb_debug_wait_probe(workspace, armed, stream=None):
    """Failure-detection self-test (see include/bb_attn.h): armed, a device
    wait runs out and leaves BB_ERR_TIMEOUT in the workspace's status word;
    read it with bb_attn_check_status."""
    _cuda_tensor(workspace, "workspace")
    _check(lib().bb_debug_wait_probe(
        _ptr(workspace), workspace.numel() * workspace.element_size(),
        int(armed), _stream_ptr(stream)), "bb_debug_wait_probe")


class Attention:
    """Convenience wrapper holding the table and workspaces for one shape.

    Allocation (workspace, outputs) happens here, with torch, outside the
    library; every call below goes straight to the C entry points."""

    def __init__(self, B, H, L, block_size, r, dtype, d=64, seed=0,
                 device="cuda", scale=0.0, mask_value=0.0, dropout=0.0,
                 dropout_seed=0, max_rand_mask_length=0, last_idx=0,
                 mask_queries=0, grad_fp32=0, keep_dropout_bits=True):
        """max_rand_mask_length, last_idx (tokens; 0 = off): the pages'
        layer options for the random table (drawn for the maximum length,
        random blocks before token last_idx); seed: the layer index there.
        grad_fp32: the backward writes dq, dk, dv as fp32.
        keep_dropout_bits: with dropout, hold a keep-bit buffer that the
        forward fills and the backward reads (same results, fewer draws);
        False makes every pass draw its decisions."""
        self.desc = make_desc(B, H, L, d, block_size, r, dtype, scale,
                              mask_value, dropout, dropout_seed, mask_queries,
                              grad_fp32)
        self.dropout_bits = None
        nbits = bb_attn_dropout_bits_size(self.desc) if keep_dropout_bits else 0
        if nbits:
            self.dropout_bits = torch.empty(nbits, dtype=torch.uint8,
                                            device=device)
            self.desc.dropout_bits = _ptr(self.dropout_bits)
        self.dtype = dtype
        self.table_host = make_table(seed, H, L, block_size, r,
                                     max_rand_mask_length, last_idx)
        self.table = self.table_host.to(device)
        self.ws_fwd = torch.empty(bb_attn_workspace_size(self.desc, 0),
                                  dtype=torch.uint8, device=device)
        self.ws_bwd = torch.empty(bb_attn_workspace_size(self.desc, 1),
                                  dtype=torch.uint8, device=device)

    def forward(self, q, k, v, key_mask=None, out=None, lse=None,
                stream=None, events=None):
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty(q.shape[:3], dtype=torch.float32,
                              device=q.device)
        bb_attn_fwd(self.desc, q, k, v, key_mask, self.table, out, lse,
                    self.ws_fwd, stream, events)
        return out, lse

    def backward(self, q, k, v, out, lse, dout, key_mask=None, dq=None,
                 dk=None, dv=None, stream=None, events=None):
        gd = grad_dtype(self.desc)
        dq = torch.empty_like(q, dtype=gd) if dq is None else dq
        dk = torch.empty_like(k, dtype=gd) if dk is None else dk
        dv = torch.empty_like(v, dtype=gd) if dv is None else dv
        bb_attn_bwd(self.desc, q, k, v, out, lse, dout, key_mask, self.table,
                    dq, dk, dv, self.ws_bwd, stream, events)
        return dq, dk, dv
