"""ctypes declarations of libcompactattn.so and tensor marshalling."""
import ctypes
import os

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libcompactattn.so")

CA_OK = 0
CA_ERR_ARG = -1
CA_ERR_ALIGN = -2
CA_ERR_DTYPE = -3
CA_ERR_LAUNCH = -4
CA_ERR_BOUNDS = -5
CA_ERR_TIMEOUT = -6
CA_ERR_WORKSPACE = -7
CA_DTYPE_BF16 = 0
CA_DTYPE_FP32 = 1

_c_int, _c_size, _vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p

# name -> (restype, argtypes); every symbol include/compactattn.h declares
EXPORTS = {
    "ca_build_tables": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "ca_build_tables_batched": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp,
                                         _vp]),
    "ca_build_tables_bits": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "ca_workspace_size": (_c_size, [_c_int] * 9),
    "ca_chunk_attention": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _vp, _vp, _vp, _c_int, _c_int,
                                    _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _c_size,
                                    _c_int, _vp, _vp]),
    "ca_chunk_attention_noalloc": (_c_int, [_vp, _vp, _vp, _c_int, _vp, _vp, _vp, _c_int, _c_int,
                                            _c_int, _c_int, _c_int, _c_int, _vp, _vp, _c_int,
                                            _vp, _vp]),
    "ca_noalloc_scratch_bytes": (_c_size, []),
    "ca_workspace_size_varlen": (_c_size, [_c_int] * 10),
    "ca_workspace_size_masked": (_c_size, [_c_int] * 9),
    "ca_workspace_size_fp8": (_c_size, [_c_int] * 8),
    "ca_chunk_attention_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp, _vp, _c_int,
                                        _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp,
                                        _c_size, _c_int, _vp, _vp]),
    "ca_chunk_attention_masked": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _vp, _vp, _c_int, _c_int,
                                           _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp,
                                           _vp, _c_size, _c_int, _vp, _vp]),
    "ca_chunk_attention_varlen": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp,
                                           _vp, _c_int, _vp, _vp, _vp, _vp, _c_int, _c_int,
                                           _c_int, _c_int, _vp, _vp, _vp, _c_size, _c_int, _vp,
                                           _vp]),
    "ca_append_kv": (_c_int, [_vp, _vp, _c_int, _vp, _vp, _c_int, _vp, _c_int, _c_int, _c_int,
                              _c_int, _c_int, _vp, _vp]),
    "ca_check": (_c_int, [_vp, _vp]),
    "ca_wait_probe": (_c_int, [_vp, _c_int, _vp]),
    "ca_last_error": (_c_int, [ctypes.c_char_p, _c_size]),
    "ca_version": (_c_int, []),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python block_sparse_chunked_b200/_build.py` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    L = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in EXPORTS.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


lib = _load()


class CompactAttnError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"[{code}] {msg}")
        self.code = code


def last_error():
    buf = ctypes.create_string_buffer(1024)
    lib.ca_last_error(buf, 1024)
    return buf.value.decode(errors="replace")


def _ok(rc):
    if rc != CA_OK:
        raise CompactAttnError(rc, last_error())


def version():
    return lib.ca_version()


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _need_cuda(name, t, dtypes=None, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def _out(name, t, like_device, dtype, numel):
    """A caller-provided output buffer: CUDA, contiguous, of the given dtype,
    on the inputs' device and large enough (the kernels write numel elements)."""
    _need_cuda(name, t, (dtype,))
    if t.device != like_device:
        raise ValueError(f"{name} is on {t.device}, the inputs on {like_device}")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements, {numel} needed")
    return t


def _same_device(dev, **tensors):
    """Every given tensor (None skipped) must live on `dev`: the kernels run on
    that device and take raw pointers."""
    for name, t in tensors.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the call runs on {dev}")


def _errp(err_flag, dev=None):
    """Pointer to the caller's device error word (int32 CUDA tensor on `dev`), or None."""
    if err_flag is None:
        return None
    _need_cuda("err_flag", err_flag, (torch.int32,))
    if dev is not None:
        _same_device(dev, err_flag=err_flag)
    if err_flag.numel() < 1:
        raise ValueError("err_flag must hold one int32")
    return _ptr(err_flag)


def _workspace(ws, nbytes, device):
    """The caller's workspace if it is a contiguous CUDA tensor on `device` with at
    least nbytes bytes, else a fresh uint8 buffer (None when nbytes is 0)."""
    if nbytes == 0:
        return None
    if (ws is not None and isinstance(ws, torch.Tensor) and ws.is_cuda and ws.is_contiguous()
            and ws.device == device and ws.numel() * ws.element_size() >= nbytes):
        return ws
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def build_tables_batched(masks, Hkv, tables=None, counts=None):
    """masks uint8/bool [nb, Hq, nQblk, nKblk] -> tables int32 [nb, Hkv, nKblk], counts [nb, Hkv]."""
    _need_cuda("masks", masks, (torch.uint8, torch.bool), 4)
    nb, Hq, nQ, nK = masks.shape
    if tables is None:
        tables = torch.empty(nb, Hkv, nK, dtype=torch.int32, device=masks.device)
    if counts is None:
        counts = torch.empty(nb, Hkv, dtype=torch.int32, device=masks.device)
    _out("tables", tables, masks.device, torch.int32, nb * Hkv * nK)
    _out("counts", counts, masks.device, torch.int32, nb * Hkv)
    with torch.cuda.device(masks.device):
        _ok(lib.ca_build_tables_batched(_ptr(masks), nb, Hq, Hkv, nQ, nK, _ptr(tables),
                                        _ptr(counts), _stream()))
    return tables, counts


def build_tables(mask, Hkv, tables=None, counts=None):
    """mask uint8/bool [Hq, nQblk, nKblk] -> (tables int32 [Hkv, nKblk], counts int32 [Hkv])."""
    _need_cuda("mask", mask, (torch.uint8, torch.bool), 3)
    Hq, nQ, nK = mask.shape
    if tables is None:
        tables = torch.empty(Hkv, nK, dtype=torch.int32, device=mask.device)
    if counts is None:
        counts = torch.empty(Hkv, dtype=torch.int32, device=mask.device)
    _out("tables", tables, mask.device, torch.int32, Hkv * nK)
    _out("counts", counts, mask.device, torch.int32, Hkv)
    with torch.cuda.device(mask.device):
        _ok(lib.ca_build_tables(_ptr(mask), Hq, Hkv, nQ, nK, _ptr(tables), _ptr(counts),
                                _stream()))
    return tables, counts


def build_tables_bits(mask_bits, Hkv, nKblk, tables=None, counts=None):
    """Bit-packed masks int32/uint32 [nb, Hq, nQblk, ceil(nKblk/32)] (bit j of word w selects
    block 32w + j) -> tables int32 [nb, Hkv, nKblk], counts int32 [nb, Hkv]."""
    _need_cuda("mask_bits", mask_bits, (torch.int32, torch.uint32), 4)
    nb, Hq, nQ, W = mask_bits.shape
    if W != (nKblk + 31) // 32:
        raise ValueError(f"mask_bits has {W} words per row, nKblk={nKblk} needs {(nKblk + 31) // 32}")
    if tables is None:
        tables = torch.empty(nb, Hkv, nKblk, dtype=torch.int32, device=mask_bits.device)
    if counts is None:
        counts = torch.empty(nb, Hkv, dtype=torch.int32, device=mask_bits.device)
    _out("tables", tables, mask_bits.device, torch.int32, nb * Hkv * nKblk)
    _out("counts", counts, mask_bits.device, torch.int32, nb * Hkv)
    with torch.cuda.device(mask_bits.device):
        _ok(lib.ca_build_tables_bits(_ptr(mask_bits), nb, Hq, Hkv, nQ, nKblk, _ptr(tables),
                                     _ptr(counts), _stream()))
    return tables, counts


_DT = {torch.bfloat16: CA_DTYPE_BF16, torch.float32: CA_DTYPE_FP32}


def workspace_size(dtype, Hq, Hkv, head_dim, block, chunk_len, prefix_len, num_pages, n_splits=0):
    code = _DT[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    n = lib.ca_workspace_size(code, Hq, Hkv, head_dim, block, chunk_len, prefix_len, num_pages,
                              n_splits)
    if n == ctypes.c_size_t(-1).value:
        raise CompactAttnError(CA_ERR_ARG, "invalid shapes for ca_workspace_size")
    return n


def chunk_attention(Q, K_pages, V_pages, page_table, tables, counts, prefix_len, n_splits=0,
                    err_flag=None, out=None, lse=None, workspace=None):
    """Chunk attention over the group tables' blocks of a paged KV cache.

    Q [L, Hq, d]; K_pages/V_pages [num_pages, Hkv, B, d] (bf16 or fp32, same
    dtype); page_table int32 [nKblk]; tables int32 [Hkv, nKblk]; counts int32
    [Hkv].  Returns O [L, Hq, d] (dtype of Q) and LSE float32 [Hq, L].
    """
    _need_cuda("Q", Q, tuple(_DT), 3)
    _need_cuda("K_pages", K_pages, (Q.dtype,), 4)
    _need_cuda("V_pages", V_pages, (Q.dtype,), 4)
    _need_cuda("page_table", page_table, (torch.int32,), 1)
    _need_cuda("tables", tables, (torch.int32,), 2)
    _need_cuda("counts", counts, (torch.int32,), 1)
    _same_device(Q.device, K_pages=K_pages, V_pages=V_pages, page_table=page_table,
                 tables=tables, counts=counts)
    if K_pages.shape != V_pages.shape:
        raise ValueError("K_pages and V_pages must have the same shape")
    L, Hq, d = Q.shape
    num_pages, Hkv, B, d2 = K_pages.shape
    if d2 != d:
        raise ValueError("head_dim of Q and of the pages differ")
    nK = -(-(prefix_len + L) // B) if B else 0
    if page_table.numel() < nK or tables.shape[0] != Hkv or tables.shape[1] < nK \
            or counts.numel() < Hkv:
        raise ValueError("page_table / tables / counts are smaller than the chunk needs")
    code = _DT[Q.dtype]
    if out is None:
        out = torch.empty_like(Q)
    _out("out", out, Q.device, Q.dtype, Q.numel())
    if lse is None:
        lse = torch.empty(Hq, L, dtype=torch.float32, device=Q.device)
    _out("lse", lse, Q.device, torch.float32, Hq * L)
    ws_n = workspace_size(code, Hq, Hkv, d, B, L, prefix_len, num_pages, n_splits)
    workspace = _workspace(workspace, ws_n, Q.device)
    with torch.cuda.device(Q.device):
        _ok(lib.ca_chunk_attention(
            _ptr(Q), _ptr(K_pages), _ptr(V_pages), code, num_pages, _ptr(page_table),
            _ptr(tables), _ptr(counts), Hq, Hkv, d, B, L, prefix_len, _ptr(out), _ptr(lse),
            _ptr(workspace) if ws_n else None, ws_n, n_splits, _errp(err_flag, Q.device),
            _stream()))
    return out, lse


def chunk_attention_fp8(Q, K8, V8, K_scale, V_scale, page_table, tables, counts, prefix_len,
                        n_splits=0, err_flag=None, out=None, lse=None, workspace=None):
    """Chunk attention over an E4M3 paged cache: K8/V8 uint8 [num_pages, Hkv, B, d],
    K_scale/V_scale float32 [num_pages, Hkv]; Q bf16 [L, Hq, d].  Returns O (bf16)
    and LSE float32 [Hq, L]."""
    _need_cuda("Q", Q, (torch.bfloat16,), 3)
    _need_cuda("K8", K8, (torch.uint8,), 4)
    _need_cuda("V8", V8, (torch.uint8,), 4)
    _need_cuda("K_scale", K_scale, (torch.float32,), 2)
    _need_cuda("V_scale", V_scale, (torch.float32,), 2)
    _need_cuda("page_table", page_table, (torch.int32,), 1)
    _need_cuda("tables", tables, (torch.int32,), 2)
    _need_cuda("counts", counts, (torch.int32,), 1)
    _same_device(Q.device, K8=K8, V8=V8, K_scale=K_scale, V_scale=V_scale,
                 page_table=page_table, tables=tables, counts=counts)
    L, Hq, d = Q.shape
    num_pages, Hkv, B, d2 = K8.shape
    nK = -(-(prefix_len + L) // B)
    if (V8.shape != K8.shape or d2 != d or tuple(K_scale.shape) != (num_pages, Hkv)
            or tuple(V_scale.shape) != (num_pages, Hkv) or page_table.numel() < nK
            or tables.shape[0] != Hkv or tables.shape[1] < nK or counts.numel() < Hkv):
        raise ValueError("inconsistent shapes for chunk_attention_fp8")
    if out is None:
        out = torch.empty_like(Q)
    _out("out", out, Q.device, Q.dtype, Q.numel())
    if lse is None:
        lse = torch.empty(Hq, L, dtype=torch.float32, device=Q.device)
    _out("lse", lse, Q.device, torch.float32, Hq * L)
    ws_n = lib.ca_workspace_size_fp8(Hq, Hkv, d, B, L, prefix_len, num_pages, n_splits)
    if ws_n == ctypes.c_size_t(-1).value:
        raise CompactAttnError(CA_ERR_ARG, "invalid shapes for ca_workspace_size_fp8")
    workspace = _workspace(workspace, ws_n, Q.device)
    with torch.cuda.device(Q.device):
        _ok(lib.ca_chunk_attention_fp8(
            _ptr(Q), _ptr(K8), _ptr(V8), _ptr(K_scale), _ptr(V_scale), num_pages,
            _ptr(page_table), _ptr(tables), _ptr(counts), Hq, Hkv, d, B, L, prefix_len,
            _ptr(out), _ptr(lse), _ptr(workspace), ws_n, n_splits, _errp(err_flag, Q.device),
            _stream()))
    return out, lse


def chunk_attention_masked(Q, K_pages, V_pages, page_table, mask_bits, prefix_len, n_splits=0,
                           err_flag=None, out=None, lse=None, tables_out=None, counts_out=None,
                           workspace=None):
    """Attention with the table builder fused in: mask_bits int32/uint32
    [Hq, nQblk, ceil(nKblk/32)] instead of tables.  Optionally writes the
    tables to tables_out [Hkv, nKblk] / counts_out [Hkv].  Returns O and LSE."""
    _need_cuda("Q", Q, tuple(_DT), 3)
    _need_cuda("K_pages", K_pages, (Q.dtype,), 4)
    _need_cuda("V_pages", V_pages, (Q.dtype,), 4)
    _need_cuda("page_table", page_table, (torch.int32,), 1)
    _need_cuda("mask_bits", mask_bits, (torch.int32, torch.uint32), 3)
    _same_device(Q.device, K_pages=K_pages, V_pages=V_pages, page_table=page_table,
                 mask_bits=mask_bits, tables_out=tables_out, counts_out=counts_out)
    if K_pages.shape != V_pages.shape:
        raise ValueError("K_pages and V_pages must have the same shape")
    L, Hq, d = Q.shape
    num_pages, Hkv, B, d2 = K_pages.shape
    nK = -(-(prefix_len + L) // B)
    if d2 != d or tuple(mask_bits.shape) != (Hq, -(-L // B), (nK + 31) // 32) \
            or page_table.numel() < nK:
        raise ValueError("mask_bits / page_table do not match the chunk")
    for name, t, n in (("tables_out", tables_out, Hkv * nK), ("counts_out", counts_out, Hkv)):
        if t is not None:
            _need_cuda(name, t, (torch.int32,))
            if t.numel() < n:
                raise ValueError(f"{name} is too small")
    code = _DT[Q.dtype]
    if out is None:
        out = torch.empty_like(Q)
    _out("out", out, Q.device, Q.dtype, Q.numel())
    if lse is None:
        lse = torch.empty(Hq, L, dtype=torch.float32, device=Q.device)
    _out("lse", lse, Q.device, torch.float32, Hq * L)
    ws_n = lib.ca_workspace_size_masked(code, Hq, Hkv, d, B, L, prefix_len, num_pages, n_splits)
    if ws_n == ctypes.c_size_t(-1).value:
        raise CompactAttnError(CA_ERR_ARG, "invalid shapes for ca_workspace_size_masked")
    workspace = _workspace(workspace, ws_n, Q.device)
    with torch.cuda.device(Q.device):
        _ok(lib.ca_chunk_attention_masked(
            _ptr(Q), _ptr(K_pages), _ptr(V_pages), code, num_pages, _ptr(page_table),
            _ptr(mask_bits), Hq, Hkv, d, B, L, prefix_len, _ptr(tables_out), _ptr(counts_out),
            _ptr(out), _ptr(lse), _ptr(workspace) if ws_n else None, ws_n, n_splits,
            _errp(err_flag, Q.device), _stream()))
    return out, lse


def chunk_attention_varlen(Q, K_pages, V_pages, cu_q, prefix_len, page_table, cu_pages, tables,
                           counts, max_kv_len, n_splits=1, err_flag=None, out=None, lse=None,
                           workspace=None):
    """Chunk attention for a batch of sequences over one page pool.

    Q [total_q, Hq, d]; cu_q int32 [S+1] (row offsets); prefix_len int32 [S];
    page_table int32 (concatenated, sequence s from cu_pages[s]); cu_pages int32
    [S+1]; tables int32 (flat: sequence s's [Hkv, nKblk_s] from Hkv*cu_pages[s]);
    counts int32 [S, Hkv]; max_kv_len >= every P_s + L_s.  All on the device.
    Returns O [total_q, Hq, d] and LSE float32 [Hq, total_q].
    """
    _need_cuda("Q", Q, tuple(_DT), 3)
    _need_cuda("K_pages", K_pages, (Q.dtype,), 4)
    _need_cuda("V_pages", V_pages, (Q.dtype,), 4)
    for name, t in (("cu_q", cu_q), ("prefix_len", prefix_len), ("page_table", page_table),
                    ("cu_pages", cu_pages), ("tables", tables), ("counts", counts)):
        _need_cuda(name, t, (torch.int32,))
    _same_device(Q.device, K_pages=K_pages, V_pages=V_pages, cu_q=cu_q, prefix_len=prefix_len,
                 page_table=page_table, cu_pages=cu_pages, tables=tables, counts=counts)
    if K_pages.shape != V_pages.shape:
        raise ValueError("K_pages and V_pages must have the same shape")
    total_q, Hq, d = Q.shape
    num_pages, Hkv, B, d2 = K_pages.shape
    S = prefix_len.numel()
    if d2 != d or cu_q.numel() != S + 1 or cu_pages.numel() != S + 1 or counts.numel() < S * Hkv:
        raise ValueError("inconsistent batch arrays")
    code = _DT[Q.dtype]
    if out is None:
        out = torch.empty_like(Q)
    _out("out", out, Q.device, Q.dtype, Q.numel())
    if lse is None:
        lse = torch.empty(Hq, total_q, dtype=torch.float32, device=Q.device)
    _out("lse", lse, Q.device, torch.float32, Hq * total_q)
    ws_n = lib.ca_workspace_size_varlen(code, Hq, Hkv, d, B, S, total_q, max_kv_len, num_pages,
                                        n_splits)
    if ws_n == ctypes.c_size_t(-1).value:
        raise CompactAttnError(CA_ERR_ARG, "invalid shapes for ca_workspace_size_varlen")
    workspace = _workspace(workspace, ws_n, Q.device)
    with torch.cuda.device(Q.device):
        _ok(lib.ca_chunk_attention_varlen(
            _ptr(Q), _ptr(K_pages), _ptr(V_pages), code, num_pages, S, total_q, _ptr(cu_q),
            _ptr(prefix_len), max_kv_len, _ptr(page_table), _ptr(cu_pages), _ptr(tables),
            _ptr(counts), Hq, Hkv, d, B, _ptr(out), _ptr(lse), _ptr(workspace), ws_n, n_splits,
            _errp(err_flag, Q.device), _stream()))
    return out, lse


def append_kv(K_new, V_new, K_pages, V_pages, page_table, prefix_len, err_flag=None):
    """Write the chunk's K_new/V_new [L, Hkv, d] into their pages (in place)."""
    _need_cuda("K_new", K_new, tuple(_DT), 3)
    _need_cuda("V_new", V_new, (K_new.dtype,), 3)
    _need_cuda("K_pages", K_pages, (K_new.dtype,), 4)
    _need_cuda("V_pages", V_pages, (K_new.dtype,), 4)
    _need_cuda("page_table", page_table, (torch.int32,), 1)
    L, Hkv, d = K_new.shape
    num_pages, Hkv2, B, d2 = K_pages.shape
    if V_new.shape != K_new.shape or V_pages.shape != K_pages.shape or Hkv2 != Hkv or d2 != d:
        raise ValueError("append_kv: inconsistent shapes")
    dev = K_new.device
    _same_device(dev, V_new=V_new, K_pages=K_pages, V_pages=V_pages, page_table=page_table)
    with torch.cuda.device(dev):
        _ok(lib.ca_append_kv(_ptr(K_new), _ptr(V_new), _DT[K_new.dtype], _ptr(K_pages),
                             _ptr(V_pages), num_pages, _ptr(page_table), Hkv, d, B, prefix_len, L,
                             _errp(err_flag, dev), _stream()))


def check(err_flag):
    """Synchronise, read and clear the device error word; raise on a device error."""
    if err_flag is None:
        raise ValueError("check: err_flag is required")
    p = _errp(err_flag)
    with torch.cuda.device(err_flag.device):
        _ok(lib.ca_check(p, _stream()))


def wait_probe(err_flag, limit_us):
    if err_flag is None:
        raise ValueError("wait_probe: err_flag is required")
    p = _errp(err_flag)
    with torch.cuda.device(err_flag.device):
        _ok(lib.ca_wait_probe(p, int(limit_us), _stream()))
