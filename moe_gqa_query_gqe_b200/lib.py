"""ctypes binding of libgqe (include/gqe.h): same entry-point names, argument
marshalling only. Tensors are torch tensors on the current CUDA device; the
binding passes their data pointers and the current stream's handle. Every step
of the computation runs in the library's CUDA kernels: there is no fallback,
and loading fails loudly when the shared library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgqe.so")

GQE_OK = 0
STATUS = {0: "GQE_OK", -1: "GQE_ERR_INVALID_ARG", -2: "GQE_ERR_UNSUPPORTED", -3: "GQE_ERR_WORKSPACE",
          -4: "GQE_ERR_CUDA", -5: "GQE_ERR_TIMEOUT", -6: "GQE_ERR_NO_DEVICE",
          -7: "GQE_ERR_DEVICE_CHECK"}
OP_ROUTE, OP_QPROJ, OP_ATTN, OP_COMBINE, OP_FORWARD, OP_DENSE, OP_FORWARD_HOST, OP_DECODE, OP_FORWARD_VARIANT = \
    1, 2, 3, 4, 5, 6, 7, 8, 9
COMBINE_SLOT, COMBINE_HARD, COMBINE_WEIGHTED, COMBINE_GLOBAL_SLOT, COMBINE_NO_SHARED = 0, 1, 2, 3, 4
# selected-query path of gqe_forward_variant, or'ed into the mode (enum gqe_qproj_path)
QPROJ_AUTO, QPROJ_GATHER, QPROJ_DENSE = 0, 0x100, 0x200

# every symbol include/gqe.h declares
EXPORTS = ("gqe_workspace_bytes", "gqe_validate_dims", "gqe_route", "gqe_route_noalloc", "gqe_qproj", "gqe_attn", "gqe_combine",
           "gqe_forward", "gqe_forward_variant", "gqe_forward_host", "gqe_decode", "gqa_dense_forward", "gqe_check_error", "gqe_status_string", "gqe_last_cuda_error",
           "gqe_selftest_wait_timeout", "gqe_version")


class GqeDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "T", "D", "G", "M", "k", "dh")]


class GqeError(RuntimeError):
    def __init__(self, fn: str, code: int, detail: str = ""):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({code}){': ' + detail if detail else ''}")
        self.code = code


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgqe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} is missing: build it with `python -m moe_gqa_query_gqe_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz, i32p, f32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
    dp = ctypes.POINTER(GqeDims)
    sig = {
        "gqe_workspace_bytes": (sz, [dp, ctypes.c_int]),
        "gqe_validate_dims": (ctypes.c_int, [dp]),
        "gqe_route": (ctypes.c_int, [dp, vp, vp, f32p, i32p, f32p, f32p, i32p, i32p, i32p, vp, sz, vp]),
        "gqe_route_noalloc": (ctypes.c_int, [dp, vp, vp, f32p, i32p, f32p, f32p, i32p, i32p, i32p, vp]),
        "gqe_qproj": (ctypes.c_int, [dp, vp, vp, vp, vp, i32p, i32p, i32p, vp, vp, vp, vp, sz, vp]),
        "gqe_attn": (ctypes.c_int, [dp, vp, vp, vp, vp, vp, sz, vp]),
        "gqe_combine": (ctypes.c_int, [dp, vp, f32p, vp, vp, vp, sz, vp]),
        "gqe_forward": (ctypes.c_int, [dp, vp, vp, vp, vp, vp, f32p, vp, vp, vp, sz, vp]),
        "gqe_decode": (ctypes.c_int, [dp, i32p, vp, vp, vp, vp, vp, f32p, vp, vp, vp, vp, i32p, f32p, vp, sz, vp]),
        "gqe_forward_variant": (ctypes.c_int, [dp, ctypes.c_int, vp, vp, vp, vp, vp, f32p, vp, vp, vp, sz, vp]),
        "gqe_forward_host": (ctypes.c_int, [dp, vp, vp, vp, vp, vp, f32p, vp, vp, vp, sz, vp]),
        "gqa_dense_forward": (ctypes.c_int, [dp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "gqe_check_error": (ctypes.c_int, [vp]),
        "gqe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "gqe_last_cuda_error": (ctypes.c_char_p, []),
        "gqe_selftest_wait_timeout": (ctypes.c_int, [vp]),
        "gqe_version": (ctypes.c_int, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def dims_struct(d) -> GqeDims:
    if isinstance(d, GqeDims):
        return d
    get = (lambda n: d[n]) if isinstance(d, dict) else (lambda n: getattr(d, n))
    return GqeDims(*(int(get(n)) for n in ("B", "T", "D", "G", "M", "k", "dh")))


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _call(name: str, *args) -> None:
    code = getattr(load(), name)(*args)
    if code != GQE_OK:
        detail = load().gqe_last_cuda_error().decode() if code == -4 else ""
        raise GqeError(name, code, detail)


def workspace_bytes(dims, op: int) -> int:
    return int(load().gqe_workspace_bytes(ctypes.byref(dims_struct(dims)), op))


def validate_dims(dims) -> int:
    return int(load().gqe_validate_dims(ctypes.byref(dims_struct(dims))))


def workspace(dims, op: int, device=None) -> torch.Tensor:
    """A device buffer of gqe_workspace_bytes(dims, op) bytes (>= 1 byte)."""
    n = max(1, workspace_bytes(dims, op))
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def gqe_route(dims, x, Wr, br, sel, w, margin, seg_off, seg_tok, row_map, ws, stream=None) -> None:
    _call("gqe_route", ctypes.byref(dims_struct(dims)), _ptr(x), _ptr(Wr), _ptr(br), _ptr(sel), _ptr(w),
          _ptr(margin), _ptr(seg_off), _ptr(seg_tok), _ptr(row_map), _ptr(ws),
          ws.numel() if ws is not None else 0, _stream(stream))


def gqe_route_noalloc(dims, x, Wr, br, sel, w, margin, seg_off, seg_tok, row_map, stream=None) -> None:
    """gqe_route with its scratch in the library's fixed device array (for
    callers that cannot allocate device memory); same outputs."""
    _call("gqe_route_noalloc", ctypes.byref(dims_struct(dims)), _ptr(x), _ptr(Wr), _ptr(br), _ptr(sel), _ptr(w),
          _ptr(margin), _ptr(seg_off), _ptr(seg_tok), _ptr(row_map), _stream(stream))


def gqe_qproj(dims, x, Wq, Wk, Wv, sel, seg_off, seg_tok, Q, K, V, ws=None, stream=None) -> None:
    _call("gqe_qproj", ctypes.byref(dims_struct(dims)), _ptr(x), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(sel),
          _ptr(seg_off), _ptr(seg_tok), _ptr(Q), _ptr(K), _ptr(V), _ptr(ws),
          ws.numel() if ws is not None else 0, _stream(stream))


def gqe_attn(dims, Q, K, V, O, ws=None, stream=None) -> None:
    _call("gqe_attn", ctypes.byref(dims_struct(dims)), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(ws),
          ws.numel() if ws is not None else 0, _stream(stream))


def gqe_combine(dims, O, w, Wo, y, ws, stream=None) -> None:
    _call("gqe_combine", ctypes.byref(dims_struct(dims)), _ptr(O), _ptr(w), _ptr(Wo), _ptr(y), _ptr(ws),
          ws.numel() if ws is not None else 0, _stream(stream))


def gqe_forward(dims, x, Wq, Wk, Wv, Wr, br, Wo, y, ws, stream=None) -> None:
    _call("gqe_forward", ctypes.byref(dims_struct(dims)), _ptr(x), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(Wr),
          _ptr(br), _ptr(Wo), _ptr(y), _ptr(ws), ws.numel(), _stream(stream))


def gqe_forward_variant(dims, mode, x, Wq, Wk, Wv, Wr, br, Wo, y, ws, stream=None) -> None:
    """gqe_forward with the output construction `mode` (COMBINE_SLOT, _HARD,
    _WEIGHTED, _GLOBAL_SLOT, _NO_SHARED), optionally or'ed with a selected-query
    path (QPROJ_AUTO, QPROJ_GATHER, QPROJ_DENSE). Wo has (G*k + G + 1),
    (G*k + 1), (G*k + 1), (G*k + 2) or (G*k + G) blocks of 64 rows
    respectively."""
    _call("gqe_forward_variant", ctypes.byref(dims_struct(dims)), int(mode), _ptr(x), _ptr(Wq), _ptr(Wk), _ptr(Wv),
          _ptr(Wr), _ptr(br), _ptr(Wo), _ptr(y), _ptr(ws), ws.numel(), _stream(stream))


def gqe_decode(dims, cache_len, x_new, Wq, Wk, Wv, Wr, br, Wo, K_cache, V_cache, y, sel, w, ws, stream=None) -> None:
    """One generation step (dims.T = cache capacity); K_cache/V_cache row
    cache_len[b] of each sequence is written with the new token's K/V."""
    _call("gqe_decode", ctypes.byref(dims_struct(dims)), _ptr(cache_len), _ptr(x_new), _ptr(Wq), _ptr(Wk), _ptr(Wv),
          _ptr(Wr), _ptr(br), _ptr(Wo), _ptr(K_cache), _ptr(V_cache), _ptr(y), _ptr(sel), _ptr(w), _ptr(ws),
          ws.numel(), _stream(stream))


def gqe_forward_host(dims, x_host, Wq, Wk, Wv, Wr, br, Wo, y_host, ws, stream=None) -> None:
    _call("gqe_forward_host", ctypes.byref(dims_struct(dims)), _ptr(x_host), _ptr(Wq), _ptr(Wk), _ptr(Wv),
          _ptr(Wr), _ptr(br), _ptr(Wo), _ptr(y_host), _ptr(ws), ws.numel(), _stream(stream))


def gqa_dense_forward(dims, x, Wq, Wk, Wv, Wo_dense, y, ws, stream=None) -> None:
    _call("gqa_dense_forward", ctypes.byref(dims_struct(dims)), _ptr(x), _ptr(Wq), _ptr(Wk), _ptr(Wv),
          _ptr(Wo_dense), _ptr(y), _ptr(ws), ws.numel(), _stream(stream))


def gqe_check_error(stream=None) -> int:
    return int(load().gqe_check_error(_stream(stream)))


def gqe_selftest_wait_timeout(stream=None) -> None:
    """Enqueue the bounded-wait self-test: the next gqe_check_error returns
    GQE_ERR_TIMEOUT (-5) after about 2 s."""
    _call("gqe_selftest_wait_timeout", _stream(stream))


def gqe_status_string(code: int) -> str:
    return load().gqe_status_string(code).decode()


def gqe_version() -> int:
    return int(load().gqe_version())


# ---- forward-pass views of the workspace (argument marshalling only) -------

def _align(v: int) -> int:
    return (v + 255) & ~255


def forward_views(dims, ws: torch.Tensor) -> dict:
    """Typed views of the intermediates gqe_forward leaves in its workspace
    (same carving order as the library: sel, w, margin, seg_off, seg_tok,
    row_map, route counts x2, Q, K, V, O, A). seg_off, seg_tok and row_map are
    written only when the forward gathers the selected queries (M > 2k);
    for M <= 2k it projects every routed head and keeps the selected rows,
    without segment lists."""
    d = dims_struct(dims)
    N = d.B * d.T
    nch = (d.T + 127) // 128
    Ha = d.G * d.k + 1
    spec = [("sel", torch.int32, (N, d.G, d.k)), ("w", torch.float32, (N, d.G, d.k)),
            ("margin", torch.float32, (N, d.G)), ("seg_off", torch.int32, (d.B * d.G * d.M + 1,)),
            ("seg_tok", torch.int32, (N * d.G * d.k,)), ("row_map", torch.int32, (N, d.G, d.k)),
            ("_counts", torch.int32, (d.B * nch * d.G * d.M,)), ("_chunk_base", torch.int32, (d.B * nch * d.G * d.M,)),
            ("Q", torch.bfloat16, (N, Ha, 64)), ("K", torch.bfloat16, (N, d.G, 64)),
            ("V", torch.bfloat16, (N, d.G, 64)), ("O", torch.bfloat16, (N, Ha, 64)),
            ("A", torch.bfloat16, (N if d.k > 1 else 0, (d.G * d.k + d.G + 1) * 64))]
    out, off = {}, 0
    for name, dt, shape in spec:
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dt).element_size()
        out[name] = ws[off:off + nbytes].view(dt).view(shape)
        off = _align(off + nbytes)
    return out
