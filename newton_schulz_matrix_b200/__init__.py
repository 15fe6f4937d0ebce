"""Python binding of libmuon (include/muon.h): the Muon optimizer step and
batched Newton-Schulz orthogonalisation on NVIDIA B200.

This module only marshals arguments: it turns torch tensors into device
pointers, groups, hyper-parameter structs and the current CUDA stream, and calls
the C ABI through ctypes.  Every step of the computation runs in the library's
CUDA kernels.  There is no fallback: if ``libmuon.so`` is missing or no CUDA
device is present, the calls raise.

Build the library with ``python -m newton_schulz_matrix_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence

import torch

__all__ = [
    "BF16", "FP16", "FP32", "STANDARD", "GRAM", "GRAM_STABILIZED", "QUINTIC", "CUBIC",
    "MuonError", "load_library", "library_path", "muon_step", "muon_ns_batched",
    "muon_workspace_size", "muon_workspace_min", "muon_ns_workspace_size", "muon_ns_flops",
    "muon_status_string", "muon_profile_begin", "muon_profile_end", "MuonStep", "StreamedMuonStep",
    "plan_slices", "muon_ns_batched_noalloc",
    "NOALLOC_SCRATCH_BYTES", "EXPORTED_SYMBOLS",
]

BF16, FP16, FP32 = 0, 1, 2
STANDARD, GRAM, GRAM_STABILIZED = 0, 1, 2
_MODE_NAMES = {"standard": STANDARD, "gram": GRAM, "gram_stabilized": GRAM_STABILIZED}
_DT_NAMES = {"bf16": BF16, "fp16": FP16, "fp32": FP32}
QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)
EXPORTED_SYMBOLS = (
    "muon_workspace_size", "muon_workspace_min", "muon_step", "muon_ns_workspace_size",
    "muon_ns_batched", "muon_ns_flops", "muon_status_string", "muon_profile_begin", "muon_profile_end",
    "muon_ns_batched_noalloc",
)
NOALLOC_SCRATCH_BYTES = 64 << 20

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


class MuonError(RuntimeError):
    pass


class _NSParams(ctypes.Structure):
    _fields_ = [("iters", ctypes.c_int), ("coeffs", ctypes.POINTER(ctypes.c_float)), ("mode", ctypes.c_int),
                ("restart_after", ctypes.c_int), ("eps", ctypes.c_float), ("compute_dtype", ctypes.c_int),
                ("gram_dtype", ctypes.c_int), ("restart_every", ctypes.c_int)]


class _Group(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int), ("cols", ctypes.c_int), ("count", ctypes.c_int),
                ("w_dtype", ctypes.c_int), ("g_dtype", ctypes.c_int),
                ("W", ctypes.POINTER(ctypes.c_void_p)), ("G", ctypes.POINTER(ctypes.c_void_p)),
                ("M", ctypes.POINTER(ctypes.c_void_p))]


class _HParams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("momentum", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("scale_coef", ctypes.c_float), ("nesterov", ctypes.c_int), ("ns", _NSParams)]


class _ProfEntry(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_char_p), ("launches", ctypes.c_int), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("exec_flops", ctypes.c_double), ("bytes", ctypes.c_double)]


def library_path() -> str:
    return os.environ.get("MUON_LIBRARY", os.path.join(_HERE, "libmuon.so"))


def load_library() -> ctypes.CDLL:
    """Load libmuon.so (raises if it has not been built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise MuonError(f"{path} is missing: build it with `python -m newton_schulz_matrix_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.muon_workspace_size.argtypes = [ctypes.POINTER(_Group), ctypes.c_int, ctypes.POINTER(_HParams)]
    lib.muon_workspace_size.restype = ctypes.c_size_t
    lib.muon_workspace_min.argtypes = [ctypes.POINTER(_Group), ctypes.c_int, ctypes.POINTER(_HParams)]
    lib.muon_workspace_min.restype = ctypes.c_size_t
    lib.muon_step.argtypes = [ctypes.POINTER(_Group), ctypes.c_int, ctypes.POINTER(_HParams), P, ctypes.c_size_t,
                              P, P]
    lib.muon_step.restype = ctypes.c_int
    lib.muon_ns_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(_NSParams)]
    lib.muon_ns_workspace_size.restype = ctypes.c_size_t
    lib.muon_ns_batched.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.POINTER(_NSParams), P, ctypes.c_size_t, P, P]
    lib.muon_ns_batched.restype = ctypes.c_int
    lib.muon_ns_flops.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(_NSParams)]
    lib.muon_ns_flops.restype = ctypes.c_double
    lib.muon_ns_batched_noalloc.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, ctypes.POINTER(_NSParams), P, P]
    lib.muon_ns_batched_noalloc.restype = ctypes.c_int
    lib.muon_profile_begin.argtypes = []
    lib.muon_profile_begin.restype = ctypes.c_int
    lib.muon_profile_end.argtypes = [ctypes.POINTER(_ProfEntry), ctypes.c_int]
    lib.muon_profile_end.restype = ctypes.c_int
    lib.muon_status_string.argtypes = [ctypes.c_int]
    lib.muon_status_string.restype = ctypes.c_char_p
    _LIB = lib
    return lib


# ---------------------------------------------------------------------------
# argument marshalling
# ---------------------------------------------------------------------------
def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return BF16
    if t == torch.float16:
        return FP16
    if t == torch.float32:
        return FP32
    raise MuonError(f"unsupported dtype {t}")


def _code(v, names) -> int:
    return names[v] if isinstance(v, str) else int(v)


def _ns_params(coeffs, mode, restart_after, eps, compute_dtype, gram_dtype, restart_every=0):
    flat = [float(x) for abc in coeffs for x in abc]
    arr = (ctypes.c_float * len(flat))(*flat)
    p = _NSParams(len(flat) // 3, ctypes.cast(arr, ctypes.POINTER(ctypes.c_float)), _code(mode, _MODE_NAMES),
                  int(restart_after), float(eps), _code(compute_dtype, _DT_NAMES), _code(gram_dtype, _DT_NAMES),
                  int(restart_every))
    return p, arr


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check_cuda(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise MuonError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise MuonError(f"{name} must be contiguous (row-major)")
    if t.dim() != 2:
        raise MuonError(f"{name} must be 2-D")


def _raise(rc: int, what: str):
    if rc != 0:
        raise MuonError(f"{what} failed: {rc} ({muon_status_string(rc)})")


def _build_groups(params, grads, moms):
    """Group tensors by (shape, W dtype, G dtype) in first-appearance order."""
    keys = []
    index = {}
    for i, (w, g, m) in enumerate(zip(params, grads, moms)):
        _check_cuda(w, "param"); _check_cuda(g, "grad"); _check_cuda(m, "momentum")
        if w.shape != g.shape or w.shape != m.shape:
            raise MuonError("param, grad and momentum shapes differ")
        if m.dtype != torch.float32:
            raise MuonError("momentum buffers must be float32")
        k = (tuple(w.shape), _dtype_code(w.dtype), _dtype_code(g.dtype))
        if k not in index:
            index[k] = len(keys)
            keys.append((k, []))
        keys[index[k]][1].append(i)
    groups = (_Group * len(keys))()
    keep = []
    order = []
    for gi, ((shape, wdt, gdt), idx) in enumerate(keys):
        n = len(idx)
        W = (ctypes.c_void_p * n)(*[params[i].data_ptr() for i in idx])
        G = (ctypes.c_void_p * n)(*[grads[i].data_ptr() for i in idx])
        M = (ctypes.c_void_p * n)(*[moms[i].data_ptr() for i in idx])
        keep += [W, G, M]
        groups[gi] = _Group(shape[0], shape[1], n, wdt, gdt, W, G, M)
        order += idx
    return groups, len(keys), keep, order


def _hparams(lr, momentum, weight_decay, scale_coef, nesterov, ns):
    return _HParams(float(lr), float(momentum), float(weight_decay), float(scale_coef), int(bool(nesterov)), ns)


# ---------------------------------------------------------------------------
# public API (same names as the C ABI)
# ---------------------------------------------------------------------------
def muon_status_string(code: int) -> str:
    return load_library().muon_status_string(int(code)).decode()


def muon_ns_flops(rows: int, cols: int, coeffs=(QUINTIC,) * 5, mode="standard", restart_after=2,
                  restart_every=0) -> float:
    ns, _arr = _ns_params(coeffs, mode, restart_after, 1e-7, BF16, FP16, restart_every)
    return load_library().muon_ns_flops(rows, cols, ctypes.byref(ns))


def _step_args(params, grads, moms, lr, momentum, nesterov, weight_decay, scale_coef, eps, coeffs, mode,
               restart_after, compute_dtype, gram_dtype, restart_every=0):
    if not (len(params) == len(grads) == len(moms)) or len(params) == 0:
        raise MuonError("params, grads and moms must be non-empty lists of equal length")
    groups, ng, keep, order = _build_groups(params, grads, moms)
    ns, arr = _ns_params(coeffs, mode, restart_after, eps, compute_dtype, gram_dtype, restart_every)
    hp = _hparams(lr, momentum, weight_decay, scale_coef, nesterov, ns)
    return groups, ng, hp, (keep, arr), order


_STEP_DEFAULTS = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.1, scale_coef=0.2, eps=1e-7,
                      coeffs=(QUINTIC,) * 5, mode="standard", restart_after=2, compute_dtype="fp16",
                      gram_dtype="fp16", restart_every=0)


def muon_workspace_size(params, grads, moms, **hp) -> int:
    a = dict(_STEP_DEFAULTS, **hp)
    groups, ng, h, _keep, _ = _step_args(params, grads, moms, **a)
    return int(load_library().muon_workspace_size(groups, ng, ctypes.byref(h)))


def muon_workspace_min(params, grads, moms, **hp) -> int:
    a = dict(_STEP_DEFAULTS, **hp)
    groups, ng, h, _keep, _ = _step_args(params, grads, moms, **a)
    return int(load_library().muon_workspace_min(groups, ng, ctypes.byref(h)))


def muon_step(params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor], moms: Sequence[torch.Tensor], *,
              workspace: torch.Tensor | None = None, status: torch.Tensor | None = None, stream=None,
              **hp) -> torch.Tensor | None:
    """One Muon step, in place on ``params`` and ``moms``.

    Keyword hyper-parameters (defaults: lr 0.02, momentum 0.95, nesterov True,
    weight_decay 0.1, scale_coef 0.2, eps 1e-7, five quintic iterations,
    mode "standard", restart_after 2, restart_every 0, compute_dtype "fp16",
    gram_dtype "fp16").
    ``compute_dtype`` is the storage type of the chain between the products
    (W and G keep their own types): "fp16" stores X0 = U / (||U|| + eps) and
    every product in binary16, "bf16" stores the raw U and the products in
    bfloat16 (8 x coarser), "fp32" runs 3xTF32 products.
    ``workspace`` is a CUDA uint8 tensor (allocated when None); ``status``, if
    given, is an int32 CUDA tensor with one word per parameter (in the order of
    ``params``) and receives the MUON_STATUS_* bits.
    """
    lib = load_library()
    a = dict(_STEP_DEFAULTS, **hp)
    groups, ng, h, keep, order = _step_args(params, grads, moms, **a)
    need = int(lib.muon_workspace_size(groups, ng, ctypes.byref(h)))
    if need == 0:
        raise MuonError("invalid arguments (workspace query returned 0)")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=params[0].device)
    st_grouped = None
    if status is not None:
        st_grouped = torch.empty(len(order), dtype=torch.int32, device=params[0].device)
    rc = lib.muon_step(groups, ng, ctypes.byref(h), ctypes.c_void_p(workspace.data_ptr()),
                       ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                       ctypes.c_void_p(st_grouped.data_ptr() if st_grouped is not None else 0),
                       ctypes.c_void_p(_stream_handle(stream)))
    _raise(rc, "muon_step")
    if status is not None:
        status[torch.tensor(order, device=status.device)] = st_grouped
    return status


def muon_ns_workspace_size(count: int, rows: int, cols: int, coeffs=(QUINTIC,) * 5, mode="standard",
                           restart_after=2, eps=1e-7, compute_dtype="fp16", gram_dtype="fp16",
                           restart_every=0) -> int:
    ns, _arr = _ns_params(coeffs, mode, restart_after, eps, compute_dtype, gram_dtype, restart_every)
    return int(load_library().muon_ns_workspace_size(count, rows, cols, ctypes.byref(ns)))


def muon_ns_batched(X: Sequence[torch.Tensor], *, coeffs=(QUINTIC,) * 5, mode="standard", restart_after=2,
                    eps=1e-7, compute_dtype=None, gram_dtype="fp16", workspace: torch.Tensor | None = None,
                    status: torch.Tensor | None = None, stream=None, restart_every=0) -> None:
    """Orthogonalise same-shape matrices in place (result has each input's shape).

    ``compute_dtype`` is the storage type of the chain: None picks "fp32" for
    fp32 inputs and "fp16" otherwise; "bf16" is also accepted.  fp32 chains run
    3xTF32 tensor-core products when the short side is at least 256, and a
    single fused launch per call for matrices small enough for one block's
    shared memory.  ``gram_dtype`` is the 16-bit type of the Gram chains.
    ``status``, if given, is an int32 CUDA tensor with one word per matrix.
    ``restart_every`` > 0 repeats the stabilised form's restart every that many
    iterations after ``restart_after``.
    """
    lib = load_library()
    if len(X) == 0:
        return
    for t in X:
        _check_cuda(t, "X")
        if t.shape != X[0].shape or t.dtype != X[0].dtype:
            raise MuonError("all matrices must share shape and dtype")
    rows, cols = X[0].shape
    dt = _dtype_code(X[0].dtype)
    if compute_dtype is None:
        compute_dtype = "fp32" if dt == FP32 else "fp16"
    ns, arr = _ns_params(coeffs, mode, restart_after, eps, compute_dtype, gram_dtype, restart_every)
    need = int(lib.muon_ns_workspace_size(len(X), rows, cols, ctypes.byref(ns)))
    if need == 0:
        raise MuonError("invalid arguments (workspace query returned 0)")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=X[0].device)
    ptrs = (ctypes.c_void_p * len(X))(*[t.data_ptr() for t in X])
    rc = lib.muon_ns_batched(ptrs, len(X), rows, cols, dt, ctypes.byref(ns), ctypes.c_void_p(workspace.data_ptr()),
                             ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                             ctypes.c_void_p(status.data_ptr() if status is not None else 0),
                             ctypes.c_void_p(_stream_handle(stream)))
    _raise(rc, "muon_ns_batched")


def muon_profile_begin() -> None:
    """Start bracketing every library launch with CUDA events (tracing aid)."""
    _raise(load_library().muon_profile_begin(), "muon_profile_begin")


def muon_profile_end() -> list[dict]:
    """Stop profiling; per kernel kind: launches, device ms, algorithmic FLOPs,
    executed FLOPs (whole tensor-core tiles, triangles only for symmetric
    products, three MMAs per 3xTF32 product) and algorithmic bytes."""
    rows = (_ProfEntry * 16)()
    n = load_library().muon_profile_end(rows, 16)
    if n < 0:
        _raise(n, "muon_profile_end")
    return [dict(kernel=r.kernel.decode(), launches=r.launches, ms=r.ms, flops=r.flops, exec_flops=r.exec_flops,
                 bytes=r.bytes) for r in rows[:n]]


class MuonStep:
    """A prepared Muon step over a fixed set of tensors.

    Builds the C structs (groups, hyper-parameters) and the workspace once, so
    each call is a single C-ABI call with no per-step marshalling.  The tensors
    must stay alive and keep their storage for the object's lifetime.
    """

    def __init__(self, params, grads, moms, *, workspace_bytes: int | None = None,
                 workspace: torch.Tensor | None = None, **hp):
        self._lib = load_library()
        a = dict(_STEP_DEFAULTS, **hp)
        self.hp = a
        self._groups, self._ng, self._h, self._keep, self.order = _step_args(params, grads, moms, **a)
        full = int(self._lib.muon_workspace_size(self._groups, self._ng, ctypes.byref(self._h)))
        lo = int(self._lib.muon_workspace_min(self._groups, self._ng, ctypes.byref(self._h)))
        if full == 0:
            raise MuonError("invalid arguments (workspace query returned 0)")
        self.workspace_needed = (lo, full)
        if workspace is not None:
            if workspace.numel() * workspace.element_size() < lo:
                raise MuonError(f"workspace of {workspace.numel()} bytes is below the minimum {lo}")
            self.workspace = workspace
        else:
            size = full if workspace_bytes is None else max(lo, min(full, int(workspace_bytes)))
            self.workspace = torch.empty(size, dtype=torch.uint8, device=params[0].device)
        self.status = torch.zeros(len(self.order), dtype=torch.int32, device=params[0].device)
        self.count = len(self.order)

    def __call__(self, stream=None) -> None:
        rc = self._lib.muon_step(self._groups, self._ng, ctypes.byref(self._h),
                                 ctypes.c_void_p(self.workspace.data_ptr()), ctypes.c_size_t(self.workspace.numel()),
                                 ctypes.c_void_p(self.status.data_ptr()), ctypes.c_void_p(_stream_handle(stream)))
        _raise(rc, "muon_step")

    def capture(self, stream=None) -> "torch.cuda.CUDAGraph":
        """Record one step into a CUDA graph and return it; ``graph.replay()``
        then runs the whole launch chain with one launch call.  The step is run
        once eagerly first (one-time kernel set-up happens outside the capture),
        so each capture advances the optimizer state by one step.  Inputs are
        read from the same tensors at replay: update G in place between replays."""
        side = torch.cuda.Stream(device=self.workspace.device) if stream is None else stream
        side.wait_stream(torch.cuda.current_stream(self.workspace.device))
        with torch.cuda.stream(side):
            self(stream=side)
        torch.cuda.current_stream(self.workspace.device).wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            self(stream=side)
        return g

    def status_in_param_order(self) -> torch.Tensor:
        out = torch.empty_like(self.status)
        out[torch.tensor(self.order, device=out.device)] = self.status
        return out


def muon_ns_batched_noalloc(X: Sequence[torch.Tensor], *, coeffs=(QUINTIC,) * 5, mode="standard", restart_after=2,
                            eps=1e-7, compute_dtype=None, gram_dtype="fp16", status: torch.Tensor | None = None,
                            stream=None, restart_every=0) -> None:
    """muon_ns_batched with the library's fixed device scratch instead of a
    workspace: for callers that cannot allocate device memory at this point
    (their allocator owns the GPU, or allocation is forbidden after start-up).
    Matrices whose one-matrix workspace exceeds NOALLOC_SCRATCH_BYTES are
    rejected.  Calls share the scratch: do not let two of them overlap on the
    GPU.  The first call on a device must come before any stream capture."""
    lib = load_library()
    if len(X) == 0:
        return
    for t in X:
        _check_cuda(t, "X")
        if t.shape != X[0].shape or t.dtype != X[0].dtype:
            raise MuonError("all matrices must share shape and dtype")
    rows, cols = X[0].shape
    dt = _dtype_code(X[0].dtype)
    if compute_dtype is None:
        compute_dtype = "fp32" if dt == FP32 else "fp16"
    ns, arr = _ns_params(coeffs, mode, restart_after, eps, compute_dtype, gram_dtype, restart_every)
    ptrs = (ctypes.c_void_p * len(X))(*[t.data_ptr() for t in X])
    rc = lib.muon_ns_batched_noalloc(ptrs, len(X), rows, cols, dt, ctypes.byref(ns),
                                     ctypes.c_void_p(status.data_ptr() if status is not None else 0),
                                     ctypes.c_void_p(_stream_handle(stream)))
    _raise(rc, "muon_ns_batched_noalloc")


def plan_slices(shapes, nbytes, slice_bytes):
    """Slices of the streamed step: lists of tensor indices, at most
    ``slice_bytes`` each (a larger tensor gets a slice of its own), taken in
    order of decreasing short side (ties by index), so that the slices with
    the most orthogonalisation work per byte come first."""
    order = sorted(range(len(shapes)), key=lambda i: (-min(shapes[i][-2:]), i))
    slices, cur, acc = [], [], 0
    for i in order:
        if cur and acc + nbytes[i] > slice_bytes:
            slices.append(cur)
            cur, acc = [], 0
        cur.append(i)
        acc += nbytes[i]
    if cur:
        slices.append(cur)
    return slices


class StreamedMuonStep:
    """A Muon step fed from and returned to pinned host memory, with the PCIe
    copies overlapped with the orthogonalisation.

    The parameters are cut into slices (at most ``slice_bytes`` of gradients
    each), taken in order of decreasing short side: the orthogonalisation's
    work per byte grows with it, so the first slices give the next slices'
    copies the most compute to hide behind, and the last slices, whose
    copies cannot be hidden, are the cheapest.  Per slice, one stream copies the
    gradients host -> device, the compute stream runs the fused step on the
    slice, and a third stream copies the updated weights device -> host, so
    slice k's step runs while slice k+1's gradients arrive and slice k-1's
    weights leave.  Every slice shares one workspace (the steps are serialised
    on the compute stream).  Across calls, a slice's gradient buffer is not
    overwritten before the previous step has read it, nor its weights updated
    before the previous copy-out has read them.  The caller's current stream
    waits for the whole step at the end of each call.
    """

    def __init__(self, params, grads, moms, host_grads, host_params, *, slice_bytes: int = 512 << 20,
                 workspace_bytes: int | None = None, **hp):
        if not (len(params) == len(grads) == len(moms) == len(host_grads) == len(host_params)):
            raise MuonError("params, grads, moms and their host copies must have equal lengths")
        for h in list(host_grads) + list(host_params):
            if h.is_cuda or not h.is_pinned():
                raise MuonError("host buffers must be pinned CPU tensors")
        dev = params[0].device
        self.params, self.grads = list(params), list(grads)
        self.host_grads, self.host_params = list(host_grads), list(host_params)
        self.slices = plan_slices([tuple(g.shape) for g in self.grads],
                                  [g.numel() * g.element_size() for g in self.grads], slice_bytes)
        self.steps = [MuonStep([self.params[i] for i in idx], [self.grads[i] for i in idx],
                               [moms[i] for i in idx], workspace=None, workspace_bytes=1, **hp)
                      for idx in self.slices]
        need = max(st.workspace_needed[1] for st in self.steps)
        if workspace_bytes is not None:
            need = max(max(st.workspace_needed[0] for st in self.steps), min(need, int(workspace_bytes)))
        self.workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        for st in self.steps:
            st.workspace = self.workspace
        self.h2d = torch.cuda.Stream(device=dev)
        self.compute = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        n = len(self.slices)
        self._computed = [None] * n   # event: slice's step finished (its gradients are read)
        self._copied_out = [None] * n  # event: slice's weights are on the host

    def __call__(self) -> None:
        caller = torch.cuda.current_stream(self.workspace.device)
        for s in (self.h2d, self.compute, self.d2h):
            s.wait_stream(caller)
        done = []
        for k, idx in enumerate(self.slices):
            with torch.cuda.stream(self.h2d):
                if self._computed[k] is not None:
                    self.h2d.wait_event(self._computed[k])
                for i in idx:
                    self.grads[i].copy_(self.host_grads[i], non_blocking=True)
                arrived = torch.cuda.Event()
                arrived.record(self.h2d)
            self.compute.wait_event(arrived)
            if self._copied_out[k] is not None:
                self.compute.wait_event(self._copied_out[k])
            self.steps[k](stream=self.compute)
            ev = torch.cuda.Event()
            ev.record(self.compute)
            self._computed[k] = ev
            with torch.cuda.stream(self.d2h):
                self.d2h.wait_event(ev)
                for i in idx:
                    self.host_params[i].copy_(self.params[i], non_blocking=True)
                out = torch.cuda.Event()
                out.record(self.d2h)
            self._copied_out[k] = out
            done.append(out)
        for ev in done:
            caller.wait_event(ev)

    @property
    def status(self) -> torch.Tensor:
        return torch.cat([st.status_in_param_order() for st in self.steps])
