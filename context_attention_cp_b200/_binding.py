"""ctypes marshalling between torch tensors and the libcpattn C ABI (include/cpattn.h)."""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# CP_LIBRARY=debug selects the bounds-checking build (libcpattn_debug.so); a path
# selects a variant built with `build --define ... --out PATH`
_choice = os.environ.get("CP_LIBRARY", "")
lib_path = (os.path.join(_HERE, "libcpattn_debug.so") if _choice == "debug"
            else os.path.abspath(_choice) if _choice else os.path.join(_HERE, "libcpattn.so"))

CP_BF16, CP_FP32 = 0, 1
LAYOUTS = {"contiguous": 0, "zigzag": 1, "striped": 2}
MODES = {"fused": 0, "stepwise": 1, "stepwise_epi": 2}
STATUS = {0: "CP_OK", 1: "CP_ERR_INVALID_ARG", 2: "CP_ERR_UNSUPPORTED", 3: "CP_ERR_SHAPE",
          4: "CP_ERR_CUDA", 5: "CP_ERR_TIMEOUT", 6: "CP_ERR_BOUNDS"}


class CPError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("%s: %s" % (STATUS.get(code, code), msg))
        self.code = code


class CpTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class CpRange(ctypes.Structure):
    _fields_ = [("nseg", ctypes.c_int32), ("reserved", ctypes.c_int32), ("start", ctypes.c_int64 * 2),
                ("len", ctypes.c_int64 * 2), ("stride", ctypes.c_int64)]


class CpPeerHandle(ctypes.Structure):
    _fields_ = [("ipc", ctypes.c_uint8 * 64), ("offset", ctypes.c_uint64), ("bytes", ctypes.c_uint64)]


_T = ctypes.POINTER(CpTensor)
_R = ctypes.POINTER(CpRange)
_i32, _i64, _vp, _f32, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t

_SIGNATURES = {
    "cp_block_attn_fwd": (_i32, [_T, _T, _T, _R, _R, _i32, _f32, _T, _T, _i32, _vp]),
    "cp_lse_merge": (_i32, [_T, _T, _T, _T, _T, _vp]),
    "cp_block_attn_bwd": (_i32, [_T, _T, _T, _T, _T, _T, _R, _R, _i32, _f32, _T, _T, _T, _vp, _sz, _vp]),
    "cp_block_bwd_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "cp_ring_attn_fwd": (_i32, [_i32, _i32, _i32, _T, _T, _T, _f32, _T, _T, _i32, _vp, _sz, _vp]),
    "cp_ring_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i64, _i64, _i64, _i64]),
    "cp_ring_attn_bwd": (_i32, [_i32, _i32, _i32, _T, _T, _T, _T, _T, _T, _f32, _T, _T, _T, _vp, _sz, _vp]),
    "cp_ring_bwd_workspace_bytes": (_sz, [_i32, _i32, _i32, _i64, _i64, _i64, _i64]),
    "cp_allgather_attn_fwd": (_i32, [_i32, _i32, _i32, _T, _T, _T, ctypes.POINTER(ctypes.c_int64), _i32, _f32, _T, _T,
                                     _vp, _sz, _vp]),
    "cp_allgather_workspace_bytes": (_sz, [_i32, _i32, _i64, _i64, _i64, _i64, _i32]),
    "cp_ulysses_all_to_all": (_i32, [_i32, _i32, _T, _T, _vp]),
    "cp_allgather_attn_bwd": (_i32, [_i32, _i32, _i32, _T, _T, _T, _T, _T, _T, ctypes.POINTER(ctypes.c_int64), _i32,
                                     _f32, _T, _T, _T, _vp, _sz, _vp]),
    "cp_allgather_bwd_workspace_bytes": (_sz, [_i32, _i32, _i64, _i64, _i64, _i64, _i64, _i32]),
    "cp_ulysses_attn_fwd": (_i32, [_i32, _i32, _T, _T, _T, _f32, _T, _T, _vp, _sz, _vp]),
    "cp_ulysses_workspace_bytes": (_sz, [_i32, _i32, _i64, _i64, _i64, _i64, _i64]),
    "cp_ulysses_attn_bwd": (_i32, [_i32, _i32, _T, _T, _T, _T, _T, _T, _f32, _T, _T, _T, _vp, _sz, _vp]),
    "cp_ulysses_bwd_workspace_bytes": (_sz, [_i32, _i32, _i64, _i64, _i64, _i64, _i64]),
    "cp_usp_attn_fwd": (_i32, [_i32, _i32, _i32, _i32, _T, _T, _T, _f32, _T, _T, _vp, _sz, _vp]),
    "cp_usp_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i64, _i64, _i64, _i64, _i64]),
    "cp_usp_attn_bwd": (_i32, [_i32, _i32, _i32, _i32, _T, _T, _T, _T, _T, _T, _f32, _T, _T, _T, _vp, _sz, _vp]),
    "cp_usp_bwd_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i64, _i64, _i64, _i64, _i64]),
    "cp_layout_permute": (_i32, [_i32, _i32, _i32, _T, _T, _i32, _vp]),
    "cp_layout_range": (_i32, [_i32, _i32, _i64, _i32, _R]),
    "cp_tile_classes": (_i32, [_R, _i64, _R, _i64, _i32, _i32, _i32, ctypes.POINTER(ctypes.c_int8)]),
    "cp_stream_check": (_i32, [_vp]),
    "cp_selftest_wait_timeout": (_i32, [ctypes.c_uint64, _vp]),
    "cp_ring_attn_fwd_static_scratch": (_i32, [_i32, _i32, _i32, _T, _T, _T, _f32, _T, _T, _vp]),
    "cp_peer_export": (_i32, [_vp, ctypes.POINTER(CpPeerHandle)]),
    "cp_peer_import": (_i32, [ctypes.POINTER(CpPeerHandle), ctypes.POINTER(ctypes.c_void_p)]),
    "cp_peer_close": (_i32, [ctypes.POINTER(CpPeerHandle)]),
    "cp_peer_copy": (_i32, [_vp, _vp, _sz, _vp]),
    "cp_status_string": (ctypes.c_char_p, [_i32]),
    "cp_last_error": (ctypes.c_char_p, []),
    "cp_abi_version": (_i32, []),
}

_lib = None


def lib():
    """The loaded libcpattn.so; raises ImportError if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise ImportError("libcpattn.so is not built; run python -m context_attention_cp_b200.build")
        handle = ctypes.CDLL(lib_path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(code):
    if code != 0:
        msg = lib().cp_last_error().decode(errors="replace")
        raise CPError(code, msg)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return CP_BF16
    if t.dtype == torch.float32:
        return CP_FP32
    raise TypeError("unsupported dtype %s" % t.dtype)


def _tensor(t, as4d=None):
    """cp_tensor view of a CUDA tensor; 3-D lse tensors [b, H, s] become [b, H, s, 1]."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    shape, stride = list(t.shape), list(t.stride())
    if t.dim() == 3:
        shape, stride = shape + [1], stride + [1]
    if len(shape) != 4:
        raise ValueError("expected a 4-D token tensor or a 3-D lse tensor, got %s" % (tuple(t.shape),))
    ct = CpTensor()
    ct.data = t.data_ptr()
    ct.dtype = _dtype_code(t)
    for i in range(4):
        ct.shape[i] = shape[i]
        ct.stride[i] = stride[i]
    return ct


def _ref(x):
    return ctypes.byref(x) if x is not None else None


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _scale(scale):
    """The softmax scale for the C ABI: None asks the library for 1/sqrt(d) (0.0)."""
    return 0.0 if scale is None else float(scale)


def _range(r):
    """(starts, lens, stride) -> cp_range."""
    starts, lens, stride = r
    cr = CpRange()
    cr.nseg = len(starts)
    for i, (s, n) in enumerate(zip(starts, lens)):
        cr.start[i] = s
        cr.len[i] = n
    cr.stride = stride
    return cr


def layout_range(layout, N, S, rank):
    """Positions of rank `rank`'s tokens as (starts, lens, stride)."""
    cr = CpRange()
    _check(lib().cp_layout_range(LAYOUTS[layout], N, S, rank, ctypes.byref(cr)))
    return tuple(cr.start[: cr.nseg]), tuple(cr.len[: cr.nseg]), cr.stride


def tile_classes(q_range, q_len, kv_range, kv_len, causal, tile_q=128, tile_k=128):
    """Per-tile classes (0 skip, 1 full, 2 partial) as a list of lists."""
    n_qt = -(-q_len // tile_q)
    n_kt = -(-kv_len // tile_k)
    buf = (ctypes.c_int8 * max(1, n_qt * n_kt))()
    qr, kr = _range(q_range), _range(kv_range)
    _check(lib().cp_tile_classes(ctypes.byref(qr), q_len, ctypes.byref(kr), kv_len, int(bool(causal)),
                                 tile_q, tile_k, buf))
    return [[buf[i * n_kt + j] for j in range(n_kt)] for i in range(n_qt)]


def block_attn_fwd(q, k, v, q_range, kv_range, causal, scale, o, lse, accumulate=False):
    """One block partial (accumulate=False) or its fused merge into fp32 (o, lse)."""
    qr, kr = _range(q_range), _range(kv_range)
    tq, tk, tv, to, tl = _tensor(q), _tensor(k), _tensor(v), _tensor(o), _tensor(lse)
    _check(lib().cp_block_attn_fwd(_ref(tq), _ref(tk), _ref(tv), ctypes.byref(qr), ctypes.byref(kr),
                                   int(bool(causal)), _scale(scale), _ref(to), _ref(tl), int(bool(accumulate)),
                                   _stream()))
    return o, lse


def block_attn_bwd(q, k, v, o, lse, do, q_range, kv_range, causal, scale, dq_acc, dk_acc, dv_acc, workspace=None):
    """Adds one (query block, key block) pair's gradient shares into the fp32
    accumulators dq_acc, dk_acc, dv_acc; lse and o are the rows' global forward
    results."""
    import torch
    b, sq, Hq, _ = q.shape
    need = lib().cp_block_bwd_workspace_bytes(b, sq, Hq)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    qr, kr = _range(q_range), _range(kv_range)
    ts = [_tensor(t) for t in (q, k, v, o, lse, do, dq_acc, dk_acc, dv_acc)]
    _check(lib().cp_block_attn_bwd(*[_ref(t) for t in ts[:6]], ctypes.byref(qr), ctypes.byref(kr), int(bool(causal)),
                                   _scale(scale), *[_ref(t) for t in ts[6:]], ctypes.c_void_p(workspace.data_ptr()), need,
                                   _stream()))
    return dq_acc, dk_acc, dv_acc


def lse_merge(o_acc, lse_acc, o_b, lse_b, o_out=None):
    ta, tla, tb, tlb, tout = _tensor(o_acc), _tensor(lse_acc), _tensor(o_b), _tensor(lse_b), _tensor(o_out)
    _check(lib().cp_lse_merge(_ref(ta), _ref(tla), _ref(tb), _ref(tlb), _ref(tout), _stream()))
    return (o_out if o_out is not None else o_acc), lse_acc


def ring_workspace_bytes(layout, N, mode, dtype_code, b, S, Hq, d):
    return lib().cp_ring_workspace_bytes(LAYOUTS[layout], N, MODES[mode], dtype_code, b, S, Hq, d)


def ring_attn_fwd(q, k, v, layout, N, causal, scale=None, o=None, lse=None, mode="fused", workspace=None):
    """Ring attention over N virtual ranks; q/k/v/o/lse in rank-major order."""
    import torch
    b, S, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((b, Hq, S), dtype=torch.float32, device=q.device)
    need = ring_workspace_bytes(layout, N, mode, _dtype_code(q), b, S, Hq, d)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = ctypes.c_void_p(workspace.data_ptr()) if (need and workspace is not None) else None
    tq, tk, tv, to, tl = _tensor(q), _tensor(k), _tensor(v), _tensor(o), _tensor(lse)
    _check(lib().cp_ring_attn_fwd(LAYOUTS[layout], N, int(bool(causal)), _ref(tq), _ref(tk), _ref(tv),
                                  _scale(scale), _ref(to), _ref(tl), MODES[mode], ws_ptr, need, _stream()))
    return o, lse


def ring_bwd_workspace_bytes(layout, N, dtype_code, b, S, Hq, d):
    return lib().cp_ring_bwd_workspace_bytes(LAYOUTS[layout], N, dtype_code, b, S, Hq, d)


def ring_attn_bwd(q, k, v, o, lse, do, layout, N, causal, scale=None, dq=None, dk=None, dv=None, workspace=None):
    """Gradients (dq, dk, dv) of ring attention; every tensor in rank-major order,
    o and lse the forward's results for the same arguments."""
    import torch
    b, S, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = ring_bwd_workspace_bytes(layout, N, _dtype_code(q), b, S, Hq, d)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ts = [_tensor(t) for t in (q, k, v, o, lse, do, dq, dk, dv)]
    _check(lib().cp_ring_attn_bwd(LAYOUTS[layout], N, int(bool(causal)), *[_ref(t) for t in ts[:6]], _scale(scale),
                                  *[_ref(t) for t in ts[6:]], ctypes.c_void_p(workspace.data_ptr()), need,
                                  _stream()))
    return dq, dk, dv


def allgather_workspace_bytes(N, dtype_code, b, S, Hkv, d, n_docs):
    return lib().cp_allgather_workspace_bytes(N, dtype_code, b, S, Hkv, d, n_docs)


def allgather_attn_fwd(q, k, v, layout, N, causal, doc_starts=None, scale=None, o=None, lse=None, workspace=None):
    """All-Gather context parallelism: every rank's Q against the gathered K/V, with an
    optional document mask (doc_starts: first positions, starting with 0).  q/k/v/o/lse
    in rank-major order."""
    import torch
    b, S, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    docs = [0] if doc_starts is None else [int(x) for x in doc_starts]
    arr = (ctypes.c_int64 * len(docs))(*docs)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((b, Hq, S), dtype=torch.float32, device=q.device)
    need = allgather_workspace_bytes(N, _dtype_code(q), b, S, k.shape[2], d, len(docs))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    tq, tk, tv, to, tl = _tensor(q), _tensor(k), _tensor(v), _tensor(o), _tensor(lse)
    _check(lib().cp_allgather_attn_fwd(LAYOUTS[layout], N, int(bool(causal)), _ref(tq), _ref(tk), _ref(tv), arr,
                                       len(docs), _scale(scale), _ref(to), _ref(tl),
                                       ctypes.c_void_p(workspace.data_ptr()), need, _stream()))
    return o, lse


def allgather_attn_bwd(q, k, v, o, lse, do, layout, N, causal, doc_starts=None, scale=None, dq=None, dk=None, dv=None,
                       workspace=None):
    """Gradients of All-Gather CP with the document mask; rank-major tensors."""
    import torch
    b, S, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    docs = [0] if doc_starts is None else [int(x) for x in doc_starts]
    arr = (ctypes.c_int64 * len(docs))(*docs)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = lib().cp_allgather_bwd_workspace_bytes(N, _dtype_code(q), b, S, Hq, k.shape[2], d, len(docs))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ts = [_tensor(t) for t in (q, k, v, o, lse, do, dq, dk, dv)]
    _check(lib().cp_allgather_attn_bwd(LAYOUTS[layout], N, int(bool(causal)), *[_ref(t) for t in ts[:6]], arr,
                                       len(docs), _scale(scale), *[_ref(t) for t in ts[6:]],
                                       ctypes.c_void_p(workspace.data_ptr()), need, _stream()))
    return dq, dk, dv


def ulysses_all_to_all(x, P, inverse=False, out=None):
    """Sequence-sharded [b, S, H, d] -> head-sharded [P*b, S, H/P, d] (inverse: back)."""
    import torch
    x = x.contiguous()
    if inverse:
        Pb, S, hp, d = x.shape
        out = torch.empty((Pb // P, S, hp * P, d), dtype=x.dtype, device=x.device) if out is None else out
        _check(lib().cp_ulysses_all_to_all(P, 1, _ref(_tensor(out)), _ref(_tensor(x)), _stream()))
    else:
        b, S, H, d = x.shape
        out = torch.empty((P * b, S, H // P, d), dtype=x.dtype, device=x.device) if out is None else out
        _check(lib().cp_ulysses_all_to_all(P, 0, _ref(_tensor(x)), _ref(_tensor(out)), _stream()))
    return out


def ulysses_workspace_bytes(P, dtype_code, b, S, Hq, Hkv, d):
    return lib().cp_ulysses_workspace_bytes(P, dtype_code, b, S, Hq, Hkv, d)


def ulysses_attn_fwd(q, k, v, P, causal, scale=None, o=None, lse=None, workspace=None):
    """Ulysses attention over P virtual ranks; q/k/v/o in original order."""
    import torch
    b, S, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((b, Hq, S), dtype=torch.float32, device=q.device) if lse is None else lse
    need = ulysses_workspace_bytes(P, _dtype_code(q), b, S, Hq, k.shape[2], d)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ts = [_tensor(t) for t in (q, k, v, o, lse)]
    _check(lib().cp_ulysses_attn_fwd(P, int(bool(causal)), _ref(ts[0]), _ref(ts[1]), _ref(ts[2]), _scale(scale),
                                     _ref(ts[3]), _ref(ts[4]), ctypes.c_void_p(workspace.data_ptr()), need, _stream()))
    return o, lse


def ulysses_attn_bwd(q, k, v, o, lse, do, P, causal, scale=None, dq=None, dk=None, dv=None, workspace=None):
    """Gradients of Ulysses attention; every tensor in original order."""
    import torch
    b, S, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = lib().cp_ulysses_bwd_workspace_bytes(P, _dtype_code(q), b, S, Hq, k.shape[2], d)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ts = [_tensor(t) for t in (q, k, v, o, lse, do, dq, dk, dv)]
    _check(lib().cp_ulysses_attn_bwd(P, int(bool(causal)), *[_ref(t) for t in ts[:6]], _scale(scale),
                                     *[_ref(t) for t in ts[6:]], ctypes.c_void_p(workspace.data_ptr()), need,
                                     _stream()))
    return dq, dk, dv


def usp_workspace_bytes(layout, N, P, dtype_code, b, S, Hq, Hkv, d):
    return lib().cp_usp_workspace_bytes(LAYOUTS[layout], N, P, dtype_code, b, S, Hq, Hkv, d)


def usp_attn_fwd(q, k, v, layout, N, P, causal, scale=None, o=None, lse=None, workspace=None):
    """USP: Ulysses over P inside each of N ring groups, the ring across them; q/k/v/o
    in the ring's rank-major order for (layout, N)."""
    import torch
    b, S, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((b, Hq, S), dtype=torch.float32, device=q.device) if lse is None else lse
    need = usp_workspace_bytes(layout, N, P, _dtype_code(q), b, S, Hq, k.shape[2], d)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ts = [_tensor(t) for t in (q, k, v, o, lse)]
    _check(lib().cp_usp_attn_fwd(LAYOUTS[layout], N, P, int(bool(causal)), _ref(ts[0]), _ref(ts[1]), _ref(ts[2]),
                                 _scale(scale), _ref(ts[3]), _ref(ts[4]), ctypes.c_void_p(workspace.data_ptr()), need,
                                 _stream()))
    return o, lse


def usp_attn_bwd(q, k, v, o, lse, do, layout, N, P, causal, scale=None, dq=None, dk=None, dv=None, workspace=None):
    """Gradients of USP attention; every tensor in the ring's rank-major order."""
    import torch
    b, S, Hq, d = q.shape
    if scale is None:
        scale = 0.0  # the library's default: 1/sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = lib().cp_usp_bwd_workspace_bytes(LAYOUTS[layout], N, P, _dtype_code(q), b, S, Hq, k.shape[2], d)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ts = [_tensor(t) for t in (q, k, v, o, lse, do, dq, dk, dv)]
    _check(lib().cp_usp_attn_bwd(LAYOUTS[layout], N, P, int(bool(causal)), *[_ref(t) for t in ts[:6]], _scale(scale),
                                 *[_ref(t) for t in ts[6:]], ctypes.c_void_p(workspace.data_ptr()), need, _stream()))
    return dq, dk, dv


def ring_attn_fwd_static_scratch(q, k, v, layout, N, causal, scale, o, lse):
    """Stepwise ring that takes its workspace from the library's static device
    scratch, for callers that cannot allocate; o and lse are caller-allocated."""
    tq, tk, tv, to, tl = _tensor(q), _tensor(k), _tensor(v), _tensor(o), _tensor(lse)
    _check(lib().cp_ring_attn_fwd_static_scratch(LAYOUTS[layout], N, int(bool(causal)), _ref(tq), _ref(tk),
                                                 _ref(tv), _scale(scale), _ref(to), _ref(tl), _stream()))
    return o, lse


def layout_permute(x, layout, N, seq_axis=1, inverse=False, out=None):
    """Forward: rank-major copy of x.  Inverse: x is rank-major; returns original order."""
    import torch
    x = x.contiguous()
    if out is None:
        out = torch.empty_like(x)
    if x.dim() == 3 and seq_axis == 2:
        x4, o4 = x.unsqueeze(-1), out.unsqueeze(-1)
    else:
        x4, o4 = x, out
    tx, to = _tensor(x4), _tensor(o4)
    if inverse:
        # the ABI writes the original-order tensor (its `x`) from the ranked one
        _check(lib().cp_layout_permute(LAYOUTS[layout], N, seq_axis, _ref(to), _ref(tx), 1, _stream()))
    else:
        _check(lib().cp_layout_permute(LAYOUTS[layout], N, seq_axis, _ref(tx), _ref(to), 0, _stream()))
    return out


def selftest_wait_timeout(limit_ns=20_000_000):
    """Launch the bounded-wait self-test kernel (its wait is made to expire)."""
    _check(lib().cp_selftest_wait_timeout(int(limit_ns), _stream()))


def stream_check():
    """Synchronise the current stream and raise if a kernel reported a device-side error."""
    _check(lib().cp_stream_check(_stream()))


# ------------------------------------------------------------ other ranks' blocks

def peer_export(t):
    """The handle of CUDA tensor t's memory for other processes, as bytes
    (cp_peer_export); t must stay allocated while any peer has it mapped."""
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("peer blocks must be contiguous CUDA tensors")
    h = CpPeerHandle()
    _check(lib().cp_peer_export(ctypes.c_void_p(t.data_ptr()), ctypes.byref(h)))
    return bytes(h)


class _DeviceArray:
    """A device address seen through the CUDA array interface (zero copy)."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (ptr, False),
                                         "version": 3, "strides": None}


def peer_import(handle, shape, dtype):
    """Maps another process's block (handle bytes from peer_export) on the current
    device (cp_peer_import) and returns a contiguous tensor of `shape` and `dtype`
    over it, without a copy."""
    import torch
    if dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("unsupported dtype %s" % dtype)
    h = CpPeerHandle.from_buffer_copy(handle)
    nbytes = torch.Size(shape).numel() * torch.empty((), dtype=dtype).element_size()
    if nbytes > h.bytes:
        raise ValueError("the peer block holds %d bytes, %d asked for" % (h.bytes, nbytes))
    ptr = ctypes.c_void_p()
    _check(lib().cp_peer_import(ctypes.byref(h), ctypes.byref(ptr)))
    try:
        # no device argument: the tensor stays on the device that holds the memory (a
        # device argument naming another one would copy)
        if dtype == torch.bfloat16:
            return torch.as_tensor(_DeviceArray(ptr.value, shape, "<i2")).view(torch.bfloat16)
        return torch.as_tensor(_DeviceArray(ptr.value, shape, "<f4"))
    except Exception:
        lib().cp_peer_close(ctypes.byref(h))  # the mapping made above is not handed out
        raise


def peer_close(handle):
    """Drops one mapping made by peer_import (cp_peer_close)."""
    h = CpPeerHandle.from_buffer_copy(handle)
    _check(lib().cp_peer_close(ctypes.byref(h)))


def peer_copy(dst, src):
    """Copies contiguous tensor src (for example a block from peer_import) into dst, on
    the current stream, with the copy engines (cp_peer_copy)."""
    if not (dst.is_contiguous() and src.is_contiguous()) or dst.dtype != src.dtype or dst.shape != src.shape:
        raise ValueError("peer_copy needs contiguous tensors of one shape and dtype")
    nbytes = dst.numel() * dst.element_size()
    _check(lib().cp_peer_copy(ctypes.c_void_p(dst.data_ptr()), ctypes.c_void_p(src.data_ptr()), nbytes, _stream()))
    return dst
