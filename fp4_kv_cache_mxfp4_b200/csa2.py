"""Python binding of libcsa2 (include/csa2.h): argument marshalling only.

Every function takes torch CUDA tensors, passes their device pointers and
the current CUDA stream to the C ABI and raises ``Csa2Error`` on a non-zero
status.  All computation happens in the library's CUDA kernels; there is no
fallback: if libcsa2.so is missing, ``load()`` raises.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")

FULL, REINDEX, REINDEX_POOL, REUSE = 0, 1, 2, 3
WS_INDEX, WS_ATTN, WS_GROUP, WS_STACK = 1, 2, 3, 4
GROUP_INPUTS_READY, GROUP_SERIAL = 1, 2
FMT_BF16, FMT_FP8, FMT_MXFP4, FMT_NVFP4 = 0, 1, 2, 3
ENTRY_BYTES = 288

_c_i32, _c_i64, _c_f32, _c_p = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p


class Csa2Error(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class IndexArgs(ctypes.Structure):
    _fields_ = [("mode", _c_i32), ("B", _c_i32), ("Q", _c_i32), ("K", _c_i32), ("N", _c_i64),
                ("qI", _c_p), ("w", _c_p), ("kI", _c_p), ("n_vis", _c_p), ("idx", _c_p), ("scores", _c_p),
                ("hsi_blocks", _c_i32), ("hsi_block", _c_i32), ("pool_out", _c_p), ("pool_in", _c_p),
                ("k_format", _c_i32)]


class AttnArgs(ctypes.Structure):
    _fields_ = [("B", _c_i32), ("Q", _c_i32), ("K", _c_i32), ("W", _c_i32), ("N", _c_i64),
                ("q", _c_p), ("kv_fp4", _c_p), ("idx", _c_p), ("swa", _c_p),
                ("swa_rows", _c_i32), ("swa_step", _c_i32), ("scale", _c_f32),
                ("out", _c_p), ("lse", _c_p), ("swa_format", _c_i32), ("swa_scale", _c_p), ("q_format", _c_i32)]


class Layer(ctypes.Structure):
    _fields_ = [("mode", _c_i32), ("qI", _c_p), ("w", _c_p), ("q", _c_p), ("swa", _c_p),
                ("out", _c_p), ("lse", _c_p), ("idx", _c_p), ("scores", _c_p), ("swa_scale", _c_p)]


class GroupArgs(ctypes.Structure):
    _fields_ = [("B", _c_i32), ("Q", _c_i32), ("K", _c_i32), ("W", _c_i32), ("N", _c_i64),
                ("n_vis", _c_p), ("kI", _c_p), ("kv_fp4", _c_p), ("kv_new", _c_p), ("n_new", _c_i64),
                ("new_rows", _c_p), ("swa_rows", _c_i32), ("swa_step", _c_i32),
                ("hsi_blocks", _c_i32), ("hsi_block", _c_i32), ("pool", _c_p), ("scale", _c_f32),
                ("n_layers", _c_i32), ("layers", ctypes.POINTER(Layer)), ("pool_in", _c_p), ("flags", _c_i32),
                ("swa_format", _c_i32), ("index_k_format", _c_i32), ("q_format", _c_i32)]


class CompressArgs(ctypes.Structure):
    _fields_ = [("x", _c_p), ("n_entries", _c_i64), ("ld_x", _c_i64), ("r", _c_i32), ("w", _c_p),
                ("w_stride", _c_i64), ("cos", _c_p), ("sin", _c_p), ("kv_fp4", _c_p), ("dst_rows", _c_p),
                ("row_offset", _c_i64)]


class StackArgs(ctypes.Structure):
    _fields_ = [("n_groups", _c_i32), ("groups", ctypes.POINTER(GroupArgs))]


class Copy(ctypes.Structure):
    _fields_ = [("dst", _c_p), ("src", _c_p), ("bytes", ctypes.c_size_t), ("layer", _c_i32)]


class Io(ctypes.Structure):
    _fields_ = [("in_", ctypes.POINTER(Copy)), ("n_in", _c_i32), ("out", ctypes.POINTER(Copy)), ("n_out", _c_i32)]


_lib = None


def load(path=LIB_PATH):
    """Load libcsa2.so (built by ``python -m fp4_kv_cache_mxfp4_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"libcsa2.so not found at {path}; build it with "
                      f"`python -m fp4_kv_cache_mxfp4_b200.build`")
    lib = ctypes.CDLL(path)
    lib.csa2_quantize_kv_fp4.argtypes = [_c_p, _c_i64, _c_i64, _c_p, _c_p, _c_i64, _c_p]
    lib.csa2_quantize_window_fp8.argtypes = [_c_p, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_i64, _c_p]
    lib.csa2_quantize_index_k_mxfp4.argtypes = [_c_p, _c_i64, _c_i64, _c_p, _c_p, _c_i64, _c_p]
    lib.csa2_compress_rope_quantize_kv_fp4.argtypes = [ctypes.POINTER(CompressArgs), _c_p]
    lib.csa2_index_score_topk.argtypes = [ctypes.POINTER(IndexArgs), _c_p, ctypes.c_size_t, _c_p]
    lib.csa2_index_score_topk_noalloc.argtypes = [ctypes.POINTER(IndexArgs), _c_p]
    lib.csa2_sparse_attn.argtypes = [ctypes.POINTER(AttnArgs), _c_p, ctypes.c_size_t, _c_p]
    lib.csa2_group_decode.argtypes = [ctypes.POINTER(GroupArgs), _c_p, ctypes.c_size_t, _c_p]
    lib.csa2_stack_decode.argtypes = [ctypes.POINTER(StackArgs), _c_p, ctypes.c_size_t, _c_p]
    lib.csa2_group_decode_io.argtypes = [ctypes.POINTER(GroupArgs), ctypes.POINTER(Io), _c_p, ctypes.c_size_t, _c_p]
    lib.csa2_stack_decode_io.argtypes = [ctypes.POINTER(StackArgs), ctypes.POINTER(Io), _c_p, ctypes.c_size_t, _c_p]
    lib.csa2_noalloc_scratch_bytes.argtypes = []
    lib.csa2_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.csa2_workspace_size.argtypes = [_c_p, _c_i32]
    lib.csa2_workspace_size.restype = ctypes.c_size_t
    lib.csa2_device_status.argtypes = [ctypes.POINTER(_c_i32), _c_p]
    lib.csa2_status_string.argtypes = [_c_i32]
    lib.csa2_status_string.restype = ctypes.c_char_p
    lib.csa2_version.restype = _c_i32
    lib.csa2_cuda_error_string.argtypes = []
    lib.csa2_cuda_error_string.restype = ctypes.c_char_p
    lib.csa2_trace_begin.argtypes = [_c_i32]
    lib.csa2_trace_get.argtypes = [_c_i32, ctypes.POINTER(_c_i32), ctypes.POINTER(_c_f32)]
    lib.csa2_trace_count.restype = _c_i32
    lib.csa2_kernel_name.argtypes = [_c_i32]
    lib.csa2_kernel_name.restype = ctypes.c_char_p
    for name in ("csa2_quantize_kv_fp4", "csa2_quantize_window_fp8", "csa2_quantize_index_k_mxfp4",
                 "csa2_compress_rope_quantize_kv_fp4",
                 "csa2_index_score_topk", "csa2_index_score_topk_noalloc", "csa2_sparse_attn",
                 "csa2_group_decode", "csa2_stack_decode", "csa2_group_decode_io", "csa2_stack_decode_io",
                 "csa2_device_status", "csa2_trace_begin", "csa2_trace_stop",
                 "csa2_trace_end", "csa2_trace_get"):
        getattr(lib, name).restype = _c_i32
    _lib = lib
    return lib


def status_string(status):
    return load().csa2_status_string(int(status)).decode()


def version():
    return int(load().csa2_version())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status, what):
    if status != 0:
        if status == 5:                     # CSA2_ERR_CUDA
            what = f"{what} ({cuda_error_string()})"
        raise Csa2Error(status, what)


def cuda_error_string():
    """The CUDA runtime's description of the last failure behind a CUDA status."""
    return load().csa2_cuda_error_string().decode()


# ---------------------------------------------------------------------------
# The four calls of the C ABI
# ---------------------------------------------------------------------------

def csa2_quantize_kv_fp4(x, kv_fp4, dst_rows=None, row_offset=0, stream=None):
    """x bf16 [n, >=512] (row stride = x.stride(0)), kv_fp4 uint8 [rows, 288],
    dst_rows optional int64 [n]."""
    n = x.shape[0]
    _check(load().csa2_quantize_kv_fp4(_ptr(x), n, x.stride(0) if n else 512, _ptr(kv_fp4), _ptr(dst_rows),
                                       row_offset, _stream(stream)), "csa2_quantize_kv_fp4")


def csa2_quantize_window_fp8(x, codes, scales, dst_rows=None, row_offset=0, stream=None):
    """x bf16 [n, >=512], codes uint8 [rows, 512], scales float32 [rows],
    dst_rows optional int64 [n]."""
    n = x.shape[0]
    _check(load().csa2_quantize_window_fp8(_ptr(x), n, x.stride(0) if n else 512, _ptr(codes), _ptr(scales),
                                           _ptr(dst_rows), row_offset, _stream(stream)), "csa2_quantize_window_fp8")


def csa2_quantize_index_k_mxfp4(x, out, dst_rows=None, row_offset=0, stream=None):
    """x bf16 [n, >=128], out uint8 [rows, 68], dst_rows optional int64 [n]."""
    n = x.shape[0]
    _check(load().csa2_quantize_index_k_mxfp4(_ptr(x), n, x.stride(0) if n else 128, _ptr(out), _ptr(dst_rows),
                                              row_offset, _stream(stream)), "csa2_quantize_index_k_mxfp4")


def csa2_compress_rope_quantize_kv_fp4(x, r, w, cos, sin, kv_fp4, dst_rows=None, row_offset=0, stream=None):
    """x bf16 [n*r, >=512] tokens, w float32 [1 or n, r, 512] weights, cos/sin
    float32 [n, 32], kv_fp4 uint8 [rows, 288], dst_rows optional int64 [n]."""
    n = x.shape[0] // r
    a = CompressArgs(x=_ptr(x), n_entries=n, ld_x=x.stride(0) if n else 512, r=r, w=_ptr(w),
                     w_stride=0 if w.shape[0] == 1 else r * 512, cos=_ptr(cos), sin=_ptr(sin), kv_fp4=_ptr(kv_fp4),
                     dst_rows=_ptr(dst_rows), row_offset=row_offset)
    _check(load().csa2_compress_rope_quantize_kv_fp4(ctypes.byref(a), _stream(stream)),
           "csa2_compress_rope_quantize_kv_fp4")


def index_args(mode, qI, w, kI, n_vis, idx, scores=None, hsi_blocks=0, hsi_block=8, pool_out=None, pool_in=None):
    """Build csa2_index_args from tensors: qI [B,Q,32,128], w [B,Q,32],
    kI bf16 [B,N,128] (or uint8 [B,N,68] MXFP4 entries), n_vis int32 [B,Q],
    idx int32 [B,Q,K]."""
    B, Q = qI.shape[0], qI.shape[1]
    mx = kI.dtype == torch.uint8
    a = IndexArgs(mode=mode, B=B, Q=Q, K=idx.shape[-1], N=kI.shape[1],
                  qI=_ptr(qI), w=_ptr(w), kI=_ptr(kI), n_vis=_ptr(n_vis), idx=_ptr(idx), scores=_ptr(scores),
                  hsi_blocks=hsi_blocks, hsi_block=hsi_block, pool_out=_ptr(pool_out), pool_in=_ptr(pool_in),
                  k_format=FMT_MXFP4 if mx else FMT_BF16)
    a._tensors = (qI, w, kI, n_vis, idx, scores, pool_out, pool_in)     # the struct holds raw pointers
    return a


def csa2_index_score_topk(args, ws, stream=None):
    _check(load().csa2_index_score_topk(ctypes.byref(args), _ptr(ws), ws.numel() * ws.element_size(),
                                        _stream(stream)), "csa2_index_score_topk")


def csa2_index_score_topk_noalloc(args, stream=None):
    """csa2_index_score_topk on the library's fixed scratch array (no
    workspace argument; for callers that cannot allocate device memory)."""
    _check(load().csa2_index_score_topk_noalloc(ctypes.byref(args), _stream(stream)),
           "csa2_index_score_topk_noalloc")


def noalloc_scratch_bytes():
    """Size of the library's fixed scratch array behind the no-allocation
    index call, as compiled into libcsa2.so."""
    return int(load().csa2_noalloc_scratch_bytes())


def attn_args(q, kv_fp4, idx, swa, out, lse=None, W=128, swa_step=0, scale=0.0, swa_scale=None):
    """q bf16 [B,Q,64,512] (or uint8 [B,Q,64,288] FP4 rows: quantised Q),
    kv_fp4 uint8 [B,N,288], idx int32 [B,Q,K], swa bf16 [B,rows,512] (or
    uint8 E4M3 codes [B,rows,512] with swa_scale float32 [B,rows]), out bf16
    [B,Q,64,512], lse f32 [B,Q,64]."""
    B, Q = q.shape[0], q.shape[1]
    a = AttnArgs(B=B, Q=Q, K=idx.shape[-1] if idx is not None else 0, W=W, N=kv_fp4.shape[1],
                 q=_ptr(q), kv_fp4=_ptr(kv_fp4), idx=_ptr(idx), swa=_ptr(swa),
                 swa_rows=swa.shape[1] if swa is not None else 0, swa_step=swa_step, scale=scale,
                 out=_ptr(out), lse=_ptr(lse), swa_format=FMT_FP8 if swa_scale is not None else FMT_BF16,
                 swa_scale=_ptr(swa_scale), q_format=FMT_NVFP4 if q.dtype == torch.uint8 else FMT_BF16)
    a._tensors = (q, kv_fp4, idx, swa, out, lse, swa_scale)     # the struct holds raw pointers
    return a


def csa2_sparse_attn(args, ws, stream=None):
    _check(load().csa2_sparse_attn(ctypes.byref(args), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)), "csa2_sparse_attn")


def group_args(B, Q, K, W, N, n_vis, kI, kv_fp4, layers, kv_new=None, new_rows=None, swa_rows=128, swa_step=0,
               hsi_blocks=0, hsi_block=8, pool=None, scale=0.0, pool_in=None, flags=0, swa_format=0, q_format=0):
    """``layers`` is a list of dicts with keys mode, qI, w, q, swa, out, lse,
    idx, scores (tensors or None).  ``pool_in`` is an HSI pool built by an
    earlier group; ``flags`` a combination of GROUP_INPUTS_READY and
    GROUP_SERIAL; ``q_format`` FMT_NVFP4 for quantised attention Q;
    ``swa_format`` FMT_FP8 when every layer's swa holds E4M3
    codes with a ``swa_scale`` tensor.  The returned struct keeps its layer
    array alive."""
    arr = (Layer * len(layers))()
    for i, L in enumerate(layers):
        arr[i] = Layer(mode=L["mode"], qI=_ptr(L.get("qI")), w=_ptr(L.get("w")), q=_ptr(L["q"]),
                       swa=_ptr(L["swa"]), out=_ptr(L["out"]), lse=_ptr(L.get("lse")),
                       idx=_ptr(L.get("idx")), scores=_ptr(L.get("scores")), swa_scale=_ptr(L.get("swa_scale")))
    g = GroupArgs(B=B, Q=Q, K=K, W=W, N=N, n_vis=_ptr(n_vis), kI=_ptr(kI), kv_fp4=_ptr(kv_fp4),
                  kv_new=_ptr(kv_new), n_new=0 if kv_new is None else kv_new.shape[0], new_rows=_ptr(new_rows),
                  swa_rows=swa_rows, swa_step=swa_step, hsi_blocks=hsi_blocks, hsi_block=hsi_block,
                  pool=_ptr(pool), scale=scale, n_layers=len(layers),
                  layers=ctypes.cast(arr, ctypes.POINTER(Layer)), pool_in=_ptr(pool_in), flags=flags,
                  swa_format=swa_format, index_k_format=FMT_MXFP4 if kI.dtype == torch.uint8 else FMT_BF16,
                  q_format=q_format)
    g._layer_array = arr
    # the structs hold raw pointers: keep every tensor alive with them
    g._tensors = (n_vis, kI, kv_fp4, kv_new, new_rows, pool, pool_in, [dict(L) for L in layers])
    return g


def stack_args(groups):
    """csa2_stack_args over a list of group_args structs (kept alive)."""
    arr = (GroupArgs * len(groups))()
    for i, g in enumerate(groups):
        arr[i] = g
    s = StackArgs(n_groups=len(groups), groups=ctypes.cast(arr, ctypes.POINTER(GroupArgs)))
    s._group_array = arr
    s._groups = list(groups)
    return s


def csa2_stack_decode(args, ws, stream=None):
    _check(load().csa2_stack_decode(ctypes.byref(args), _ptr(ws), ws.numel() * ws.element_size(),
                                    _stream(stream)), "csa2_stack_decode")


def csa2_group_decode(args, ws, stream=None):
    _check(load().csa2_group_decode(ctypes.byref(args), _ptr(ws), ws.numel() * ws.element_size(),
                                    _stream(stream)), "csa2_group_decode")


def io_args(copies_in, copies_out):
    """csa2_io over two lists of (dst, src, bytes, layer) tuples (addresses
    as ints), each in non-decreasing layer order; the arrays are kept alive
    by the returned struct."""
    def arr(cs):
        a = (Copy * max(len(cs), 1))()
        for i, (dst, src, n, layer) in enumerate(cs):
            a[i] = Copy(dst=dst, src=src, bytes=n, layer=layer)
        return a
    ai, ao = arr(copies_in), arr(copies_out)
    io = Io(in_=ctypes.cast(ai, ctypes.POINTER(Copy)), n_in=len(copies_in),
            out=ctypes.cast(ao, ctypes.POINTER(Copy)), n_out=len(copies_out))
    io._arrays = (ai, ao)
    return io


def csa2_group_decode_io(args, io, ws, stream=None):
    _check(load().csa2_group_decode_io(ctypes.byref(args), ctypes.byref(io), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)), "csa2_group_decode_io")


def csa2_stack_decode_io(args, io, ws, stream=None):
    _check(load().csa2_stack_decode_io(ctypes.byref(args), ctypes.byref(io), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)), "csa2_stack_decode_io")


def csa2_workspace_size(args, which):
    return int(load().csa2_workspace_size(ctypes.byref(args), which))


def csa2_device_status(stream=None):
    code = _c_i32(0)
    st = load().csa2_device_status(ctypes.byref(code), _stream(stream))
    return int(st), int(code.value)


def workspace(args, which, device="cuda"):
    """A workspace tensor of the size the call needs (PyTorch owns the
    memory; its contents do not matter)."""
    n = csa2_workspace_size(args, which)
    if n == 0:
        raise Csa2Error(2, "csa2_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------
# Launch tracing
# ---------------------------------------------------------------------------

def csa2_trace_begin(max_launches):
    _check(load().csa2_trace_begin(max_launches), "csa2_trace_begin")


def csa2_trace_stop():
    _check(load().csa2_trace_stop(), "csa2_trace_stop")


def csa2_trace_end():
    _check(load().csa2_trace_end(), "csa2_trace_end")


def csa2_trace_records():
    """[(kernel name, ms), ...] of the traced launches (waits for them)."""
    lib = load()
    out = []
    for i in range(lib.csa2_trace_count()):
        k, ms = _c_i32(0), _c_f32(0.0)
        _check(lib.csa2_trace_get(i, ctypes.byref(k), ctypes.byref(ms)), "csa2_trace_get")
        out.append((lib.csa2_kernel_name(k.value).decode(), float(ms.value)))
    return out
