"""ctypes binding of ``libdmuon.so`` (the C ABI in ``include/dmuon.h``).

Argument marshalling only: torch tensors are turned into device pointers,
shapes into an int64 array and the current torch stream into a cudaStream_t.
Every step of the computation runs in the library's CUDA kernels.  If the
library is missing this module raises on import: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from pathlib import Path

LIB_PATH = Path(os.environ.get("DMUON_LIB", Path(__file__).resolve().parent / "libdmuon.so"))

DMUON_OK = 0
DMUON_ERR_INVALID = -1
DMUON_ERR_DTYPE = -2
DMUON_ERR_CUDA = -3
DMUON_ERR_OOM = -4
DMUON_ERR_DEVICE_TIMEOUT = -5

DMUON_BF16 = 0
DMUON_F32 = 1

VARIANTS = {"auto": 0, "direct": 1, "gram": 2, "batched": 3}
KIND_TC_GEMM, KIND_EW, KIND_SIMT_GEMM, KIND_OTHER, KIND_TC_GEMM_PAIR = 0, 1, 2, 3, 4

# every entry point include/dmuon.h declares
EXPORTS = (
    "dmuon_options_init", "dmuon_step", "dmuon_step_ex", "dmuon_compute_update",
    "dmuon_gemm_bf16", "dmuon_cache_save", "dmuon_cache_load", "dmuon_cache_clear",
    "dmuon_cache_size", "dmuon_cache_entry", "dmuon_set_workspace", "dmuon_workspace_size",
    "dmuon_timing_enable", "dmuon_timing_reset", "dmuon_timing_get", "dmuon_launch_count",
    "dmuon_last_error", "dmuon_version", "dmuon_compute_update_noalloc", "dmuon_step_host_io",
    "dmuon_selftest_wait", "dmuon_adamw_step", "dmuon_debug_io_order", "dmuon_debug_groups",
)


class DmuonError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"dmuon error {code}: {msg}")
        self.code = code


class Options(ctypes.Structure):
    _fields_ = [
        ("param_dtype", ctypes.c_int), ("grad_dtype", ctypes.c_int), ("mom_dtype", ctypes.c_int),
        ("eps", ctypes.c_float), ("nesterov", ctypes.c_int), ("variant", ctypes.c_int),
        ("ns_a", ctypes.c_float), ("ns_b", ctypes.c_float), ("ns_c", ctypes.c_float),
    ]


def _load() -> ctypes.CDLL:
    if not LIB_PATH.exists():
        raise ImportError(f"{LIB_PATH} not found: build it with `python -m newton_schulz_normalise_b200.build`")
    lib = ctypes.CDLL(str(LIB_PATH))
    P, I, F, I64, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int64, ctypes.c_size_t
    PP = ctypes.POINTER(ctypes.c_void_p)
    PI64 = ctypes.POINTER(ctypes.c_int64)
    PI = ctypes.POINTER(ctypes.c_int)
    PD = ctypes.POINTER(ctypes.c_double)
    sig = {
        "dmuon_options_init": (None, [ctypes.POINTER(Options)]),
        "dmuon_step": (I, [PP, PP, PP, PI64, I, F, F, F, I, P]),
        "dmuon_step_ex": (I, [PP, PP, PP, PI64, I, F, F, F, I, ctypes.POINTER(Options), P]),
        "dmuon_compute_update": (I, [PP, PP, PI64, I, F, I, ctypes.POINTER(Options), PP, P]),
        "dmuon_gemm_bf16": (I, [P, I64, I64, P, I64, I64, I, P, I64, I64, P, I64, I64, I, I, I, I, F, F, I, I, P]),
        "dmuon_cache_save": (I, [ctypes.c_char_p]),
        "dmuon_cache_load": (I, [ctypes.c_char_p]),
        "dmuon_cache_clear": (None, []),
        "dmuon_cache_size": (I, []),
        "dmuon_cache_entry": (I, [I, ctypes.c_char_p, S]),
        "dmuon_set_workspace": (I, [P, S]),
        "dmuon_workspace_size": (I, [PI64, I, I, ctypes.POINTER(S)]),
        "dmuon_timing_enable": (None, [I]),
        "dmuon_timing_reset": (None, []),
        "dmuon_timing_get": (I, [I, PI64, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double),
                                 ctypes.POINTER(ctypes.c_double)]),
        "dmuon_launch_count": (I64, []),
        "dmuon_last_error": (ctypes.c_char_p, []),
        "dmuon_version": (I, []),
        "dmuon_compute_update_noalloc": (I, [P, P, I64, I64, F, I, ctypes.POINTER(Options), P, P]),
        "dmuon_step_host_io": (I, [PP, PP, PP, PP, PI64, I, F, F, F, I, ctypes.POINTER(Options), P]),
        "dmuon_selftest_wait": (I, [I, P]),
        "dmuon_adamw_step": (I, [PP, PP, PP, PP, PI64, I, F, F, F, F, F, I64, I, P]),
        "dmuon_debug_io_order": (I, [PI, PI, PD, PD, PI, I, I, PI, I]),
        "dmuon_debug_groups": (I, [PI64, I, I, I, PI64, I, PI]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def last_error() -> str:
    return lib.dmuon_last_error().decode()


def _check(rc: int):
    if rc != DMUON_OK:
        raise DmuonError(rc, last_error())
    return rc


def _ptrs_of(tensors):
    return (ctypes.c_void_p * max(len(tensors), 1))(*[t.data_ptr() if t is not None else None for t in tensors])


def _shapes_of(tensors):
    flat = []
    for i, t in enumerate(tensors):
        shape = t.shape
        if len(shape) != 2 or not t.is_contiguous():
            raise ValueError(f"matrix {i}: expected a contiguous 2-D tensor, got {tuple(shape)}")
        flat += shape
    return (ctypes.c_int64 * max(len(flat), 1))(*flat)


class TensorList:
    """A list of tensors marshalled once: the pointer array, the (rows, cols)
    pairs and the dtype code, for a loop that passes the same tensors on
    every step.  It holds references to the tensors; their storage must not
    be reallocated while it is in use.  Any entry point that takes a list of
    tensors takes a TensorList as well."""
    __slots__ = ("tensors", "ptrs", "shapes", "dtype")

    def __init__(self, tensors):
        self.tensors = list(tensors)
        self.ptrs = _ptrs_of(self.tensors)
        # (rows, cols) pairs when every tensor is a contiguous matrix (the Muon
        # entry points need them); AdamW lists of any rank leave them unset
        mats = all(t is not None and t.dim() == 2 and t.is_contiguous() for t in self.tensors)
        self.shapes = _shapes_of(self.tensors) if self.tensors and mats else None
        self.dtype = _dtype_code(self.tensors[0]) if self.tensors and self.tensors[0] is not None else DMUON_BF16

    def __len__(self):
        return len(self.tensors)

    def __getitem__(self, i):
        return self.tensors[i]

    def __iter__(self):
        return iter(self.tensors)


def _ptrs(tensors):
    return tensors.ptrs if isinstance(tensors, TensorList) else _ptrs_of(tensors)


def _shapes(tensors):
    if isinstance(tensors, TensorList) and tensors.shapes is not None:
        return tensors.shapes
    return _shapes_of(tensors)


def _list_dtype(tensors) -> int:
    if isinstance(tensors, TensorList):
        return tensors.dtype
    return _dtype_code(tensors[0]) if len(tensors) else DMUON_BF16


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return DMUON_BF16
    if t.dtype == torch.float32:
        return DMUON_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def options(param_dtype=DMUON_BF16, grad_dtype=DMUON_BF16, eps=None, nesterov=None, variant="auto",
            coeffs=None) -> Options:
    o = Options()
    lib.dmuon_options_init(ctypes.byref(o))
    o.param_dtype, o.grad_dtype = param_dtype, grad_dtype
    if eps is not None:
        o.eps = eps
    if nesterov is not None:
        o.nesterov = int(nesterov)
    o.variant = VARIANTS[variant] if isinstance(variant, str) else int(variant)
    if coeffs is not None:
        o.ns_a, o.ns_b, o.ns_c = coeffs
    return o


def dmuon_step(params, grads, momenta, lr, wd, mu, ns_steps=5, stream=None):
    """In-place Muon step over lists of bf16 params/grads and fp32 momenta."""
    n = len(params)
    assert len(grads) == n and len(momenta) == n
    return _check(lib.dmuon_step(_ptrs(params), _ptrs(grads), _ptrs(momenta), _shapes(params), n,
                                 lr, wd, mu, ns_steps, _stream(stream)))


def dmuon_step_ex(params, grads, momenta, lr, wd, mu, ns_steps=5, opts: Options | None = None, stream=None,
                  **kw):
    """In-place Muon step with explicit options (dtypes taken from the tensors)."""
    n = len(params)
    assert len(grads) == n and len(momenta) == n
    if opts is None:
        opts = options(_list_dtype(params), _list_dtype(grads), **kw)
    return _check(lib.dmuon_step_ex(_ptrs(params), _ptrs(grads), _ptrs(momenta), _shapes(grads), n,
                                    lr, wd, mu, ns_steps, ctypes.byref(opts), _stream(stream)))


def dmuon_step_host_io(params, grads_host, momenta, lr, wd, mu, ns_steps=5, params_host_out=None,
                       opts: Options | None = None, stream=None, **kw):
    """Muon step with host-memory gradients (pinned CPU tensors) and an
    optional host copy of the updated parameters; copies overlap compute."""
    n = len(params)
    assert len(grads_host) == n and len(momenta) == n
    if params_host_out is not None:
        assert len(params_host_out) == n
    if opts is None:
        opts = options(_list_dtype(params), _list_dtype(grads_host), **kw)
    out = _ptrs(params_host_out) if params_host_out is not None else None
    return _check(lib.dmuon_step_host_io(_ptrs(params), _ptrs(grads_host), _ptrs(momenta), out, _shapes(params),
                                         n, lr, wd, mu, ns_steps, ctypes.byref(opts), _stream(stream)))


def dmuon_compute_update(grads, momenta, out, mu, ns_steps=5, opts: Options | None = None, stream=None, **kw):
    """Momentum update + orthogonalised update O (fp32) into ``out`` tensors."""
    n = len(grads)
    assert len(momenta) == n and len(out) == n
    if opts is None:
        dt = _list_dtype(grads)
        opts = options(dt, dt, **kw)
    return _check(lib.dmuon_compute_update(_ptrs(grads), _ptrs(momenta), _shapes(grads), n, mu, ns_steps,
                                           ctypes.byref(opts), _ptrs(out), _stream(stream)))


def dmuon_compute_update_noalloc(grad, momentum, out, mu, ns_steps=5, opts: Options | None = None,
                                 stream=None, **kw):
    """dmuon_compute_update for one matrix with the library's static scratch
    (no device allocation)."""
    if grad.dim() != 2 or not grad.is_contiguous():
        raise ValueError("expected a contiguous 2-D gradient")
    if opts is None:
        dt = _dtype_code(grad)
        opts = options(dt, dt, **kw)
    rows, cols = grad.shape
    return _check(lib.dmuon_compute_update_noalloc(grad.data_ptr(), momentum.data_ptr(), rows, cols, mu,
                                                   ns_steps, ctypes.byref(opts), out.data_ptr(),
                                                   _stream(stream)))


def dmuon_adamw_step(params, grads, exp_avg, exp_avg_sq, lr, beta1, beta2, eps, wd, step, stream=None):
    """One AdamW step over lists of tensors (any shapes, contiguous): bf16 or
    fp32 params and grads (one dtype for the call), fp32 moment buffers."""
    n = len(params)
    assert len(grads) == n and len(exp_avg) == n and len(exp_avg_sq) == n
    for group in (params, grads, exp_avg, exp_avg_sq):
        for t in group:
            if not t.is_contiguous():
                raise ValueError("AdamW tensors must be contiguous")
    numels = (ctypes.c_int64 * max(n, 1))(*[t.numel() for t in params])
    return _check(lib.dmuon_adamw_step(_ptrs(params), _ptrs(grads), _ptrs(exp_avg), _ptrs(exp_avg_sq), numels, n,
                                       lr, beta1, beta2, eps, wd, int(step), _list_dtype(params),
                                       _stream(stream)))


def dmuon_gemm_bf16(A, B, D, alpha=1.0, beta=0.0, C=None, b_kmajor=True, tile=0, sym=False, stream=None):
    """D = alpha * A @ op(B) + beta * C on 2-D or 3-D (batched) bf16 tensors.
    tile: 128 / 256 (one CTA per 128 x tile), 512 (CTA pair per 256 x 256)."""
    def geom(t):
        if t.dim() == 2:
            return 1, t.shape[0], t.shape[1], t.stride(0), t.shape[0] * t.stride(0)
        return t.shape[0], t.shape[1], t.shape[2], t.stride(1), t.stride(0)
    batch, M, K, lda, sa = geom(A)
    _, b0, b1, ldb, sb = geom(B)
    N = b0 if b_kmajor else b1
    _, _, _, ldd, sd = geom(D)
    ldc = sc = 0
    if C is not None:
        _, _, _, ldc, sc = geom(C)
    return _check(lib.dmuon_gemm_bf16(A.data_ptr(), lda, sa, B.data_ptr(), ldb, sb, int(b_kmajor),
                                      C.data_ptr() if C is not None else None, ldc, sc,
                                      D.data_ptr(), ldd, sd, M, N, K, batch, alpha, beta, tile, int(sym),
                                      _stream(stream)))


def dmuon_cache_save(path: str):
    return _check(lib.dmuon_cache_save(str(path).encode()))


def dmuon_cache_load(path: str):
    return _check(lib.dmuon_cache_load(str(path).encode()))


def dmuon_cache_clear():
    lib.dmuon_cache_clear()


def dmuon_cache_entries():
    out = []
    buf = ctypes.create_string_buffer(256)
    for i in range(lib.dmuon_cache_size()):
        _check(lib.dmuon_cache_entry(i, buf, 256))
        out.append(buf.value.decode())
    return out


def dmuon_set_workspace(tensor_or_none):
    if tensor_or_none is None:
        return _check(lib.dmuon_set_workspace(None, 0))
    t = tensor_or_none
    return _check(lib.dmuon_set_workspace(t.data_ptr(), t.numel() * t.element_size()))


def dmuon_workspace_size(shapes, param_dtype=DMUON_BF16) -> int:
    arr = (ctypes.c_int64 * max(2 * len(shapes), 1))()
    for i, (r, c) in enumerate(shapes):
        arr[2 * i], arr[2 * i + 1] = r, c
    out = ctypes.c_size_t(0)
    _check(lib.dmuon_workspace_size(arr, len(shapes), param_dtype, ctypes.byref(out)))
    return out.value


def dmuon_timing_enable(on: bool = True):
    lib.dmuon_timing_enable(int(on))


def dmuon_timing_reset():
    lib.dmuon_timing_reset()


def dmuon_timing_get(kind: int):
    n = ctypes.c_int64(0)
    ms, fl, by = ctypes.c_double(0), ctypes.c_double(0), ctypes.c_double(0)
    _check(lib.dmuon_timing_get(kind, ctypes.byref(n), ctypes.byref(ms), ctypes.byref(fl), ctypes.byref(by)))
    return {"launches": n.value, "ms": ms.value, "flops": fl.value, "bytes": by.value}


def dmuon_selftest_wait(limit_ms: int = 50, stream=None) -> int:
    """Runs the bounded-wait self-test; returns the raw status (DMUON_ERR_DEVICE_TIMEOUT
    when the device-side timeout path works)."""
    return lib.dmuon_selftest_wait(limit_ms, _stream(stream))


def dmuon_debug_groups(shapes, param_dtype=DMUON_BF16, grads_host=False):
    """The shape groups a step forms (host logic only): a list of dicts with
    m, n, count, ntall, chunk, iter_f32 and the member matrix indices."""
    n = len(shapes)
    arr = (ctypes.c_int64 * max(2 * n, 1))(*[v for s in shapes for v in s])
    ng = lib.dmuon_debug_groups(arr, n, param_dtype, int(grads_host), None, 0, None)
    _check(min(ng, 0))
    out = (ctypes.c_int64 * max(6 * ng, 1))()
    members = (ctypes.c_int * max(n, 1))()
    _check(min(lib.dmuon_debug_groups(arr, n, param_dtype, int(grads_host), out, ng, members), 0))
    res, pos = [], 0
    for g in range(ng):
        m, nn, cnt, ntall, chunk, xf = out[6 * g:6 * g + 6]
        res.append({"m": m, "n": nn, "count": cnt, "ntall": ntall, "chunk": chunk, "iter_f32": bool(xf),
                    "members": list(members[pos:pos + cnt])})
        pos += cnt
    return res


def dmuon_debug_io_order(groups, cached: bool):
    """The chunk issue order of a step (host logic only): ``groups`` is a list
    of (count, chunk, cost_ms, bytes_per_matrix, sm_copy) in issue order;
    returns a list of (group, first matrix, matrices)."""
    n = len(groups)
    ints = lambda xs: (ctypes.c_int * max(n, 1))(*xs)  # noqa: E731
    dbls = lambda xs: (ctypes.c_double * max(n, 1))(*xs)  # noqa: E731
    args = (ints([g[0] for g in groups]), ints([g[1] for g in groups]), dbls([g[2] for g in groups]),
            dbls([g[3] for g in groups]), ints([int(bool(g[4])) for g in groups]))
    total = lib.dmuon_debug_io_order(*args, n, int(cached), None, 0)
    _check(min(total, 0))
    out = (ctypes.c_int * max(3 * total, 1))()
    _check(min(lib.dmuon_debug_io_order(*args, n, int(cached), out, total), 0))
    return [(out[3 * i], out[3 * i + 1], out[3 * i + 2]) for i in range(total)]


def dmuon_launch_count() -> int:
    return lib.dmuon_launch_count()


def dmuon_version() -> int:
    return lib.dmuon_version()
