"""Thin ctypes binding over libdomino (declared in ``include/domino.h``).

Argument marshalling only: every step of the head runs in the library's CUDA kernels.  PyTorch
provides device memory and the current stream.  If ``libdomino.so`` is missing or cannot be
loaded, every call raises -- there is no CPU fallback.

Names follow the C ABI without the ``domino_`` prefix: ``draft_greedy``, ``teacher_forced``,
``accept_len``, ``workspace_bytes``, ``accept_workspace_bytes``, ``status_string``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdomino.so")

OK = 0
ERR_INVALID_ARGUMENT = -1
ERR_UNSUPPORTED = -2
ERR_CUDA = -3
ERR_WORKSPACE = -4
ERR_SCRATCH_LIMIT = -5
NOALLOC_SCRATCH_BYTES = 1024 * 1024
STATUS_DEVICE_TIMEOUT = 1
STATUS_BAD_TOKEN = 2

DTYPE_F32 = 0
DTYPE_BF16 = 1
_TORCH_DTYPE = {DTYPE_F32: torch.float32, DTYPE_BF16: torch.bfloat16}

EXPORTS = ("domino_workspace_bytes", "domino_draft_greedy", "domino_teacher_forced",
           "domino_accept_workspace_bytes", "domino_accept_len", "domino_status_string",
           "domino_abi_version", "domino_debug_set_spin_limit", "domino_launch_count",
           "domino_greedy_plan", "domino_teacher_forced_plan", "domino_draft_greedy_noalloc", "domino_debug_set_trace",
           "domino_embed_proj_bytes", "domino_project_embeddings", "domino_arena_bytes",
           "domino_pack_weights", "domino_set_l2_persistence", "domino_debug_gemm",
           "domino_debug_read_passes", "domino_teacher_forced_ex", "domino_accept_sample_workspace_bytes",
           "domino_accept_sample")


class DominoError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "L", "d", "Hs", "r", "V", "dtype")]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("embed", "W_ih", "W_hh", "b_ih", "b_hh", "W1", "W2", "embed_proj")]


_lib = None


def lib(path: str = LIB_PATH) -> ctypes.CDLL:
    """Open libdomino once; raise if it is absent (no fallback path exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"libdomino not built ({path} missing): run python -m draft_block_causal_b200.build")
        L = ctypes.CDLL(path)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
        L.domino_workspace_bytes.argtypes = [ctypes.POINTER(Shape)]
        L.domino_workspace_bytes.restype = sz
        L.domino_draft_greedy.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, vp, vp, vp, vp, vp,
                                          vp, sz, vp, vp]
        L.domino_draft_greedy.restype = ctypes.c_int
        L.domino_teacher_forced.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, vp, vp, vp, vp, vp,
                                            vp, sz, vp, vp]
        L.domino_teacher_forced.restype = ctypes.c_int
        L.domino_accept_workspace_bytes.argtypes = [i32, i32]
        L.domino_accept_workspace_bytes.restype = sz
        L.domino_accept_len.argtypes = [i32, i32, i32, vp, vp, vp, vp, sz, vp, vp]
        L.domino_accept_len.restype = ctypes.c_int
        L.domino_status_string.argtypes = [ctypes.c_int]
        L.domino_status_string.restype = ctypes.c_char_p
        L.domino_abi_version.argtypes = []
        L.domino_abi_version.restype = i32
        L.domino_debug_set_spin_limit.argtypes = [ctypes.c_uint64]
        L.domino_debug_set_spin_limit.restype = ctypes.c_int
        L.domino_launch_count.argtypes = []
        L.domino_launch_count.restype = ctypes.c_uint64
        L.domino_draft_greedy_noalloc.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, vp, vp, vp,
                                                  vp, vp, vp, vp]
        L.domino_draft_greedy_noalloc.restype = ctypes.c_int
        L.domino_embed_proj_bytes.argtypes = [ctypes.POINTER(Shape)]
        L.domino_embed_proj_bytes.restype = sz
        L.domino_project_embeddings.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, vp, vp]
        L.domino_project_embeddings.restype = ctypes.c_int
        L.domino_debug_set_trace.argtypes = [vp, i32]
        L.domino_debug_set_trace.restype = ctypes.c_int
        L.domino_greedy_plan.argtypes = [ctypes.POINTER(Shape)]
        L.domino_greedy_plan.restype = ctypes.c_char_p
        L.domino_teacher_forced_plan.argtypes = [ctypes.POINTER(Shape)]
        L.domino_teacher_forced_plan.restype = ctypes.c_char_p
        L.domino_arena_bytes.argtypes = [ctypes.POINTER(Shape)]
        L.domino_arena_bytes.restype = sz
        L.domino_pack_weights.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, sz,
                                          ctypes.POINTER(Weights), vp]
        L.domino_pack_weights.restype = ctypes.c_int
        L.domino_set_l2_persistence.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, ctypes.c_float]
        L.domino_set_l2_persistence.restype = ctypes.c_int
        L.domino_debug_gemm.argtypes = [vp, vp, i32, i32, i32, i32, vp, ctypes.c_int64, i32, i32, i32, vp, vp]
        L.domino_debug_gemm.restype = ctypes.c_int
        L.domino_teacher_forced_ex.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(Weights), vp, vp, vp, vp, vp,
                                               i32, vp, vp, sz, vp, vp]
        L.domino_teacher_forced_ex.restype = ctypes.c_int
        L.domino_debug_read_passes.argtypes = [vp, sz, i32, vp]
        L.domino_debug_read_passes.restype = ctypes.c_int
        L.domino_accept_sample_workspace_bytes.argtypes = [i32, i32, i32]
        L.domino_accept_sample_workspace_bytes.restype = sz
        L.domino_accept_sample.argtypes = [i32, i32, i32, vp, vp, vp, ctypes.c_float, vp, vp, vp, vp, sz, vp, vp]
        L.domino_accept_sample.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().domino_status_string(int(code)).decode()


def abi_version() -> int:
    return int(lib().domino_abi_version())


def launch_count() -> int:
    """Kernels the library has enqueued in this process so far."""
    return int(lib().domino_launch_count())


def greedy_plan(shape: Shape) -> str:
    """Which kernels draft_greedy runs for this shape."""
    return lib().domino_greedy_plan(ctypes.byref(shape)).decode()


def teacher_forced_plan(shape: Shape) -> str:
    """Which kernels teacher_forced runs for this shape (weights without the projection table)."""
    return lib().domino_teacher_forced_plan(ctypes.byref(shape)).decode()


def set_trace(buf) -> None:
    """Profiling hook: a CUDA int64 tensor receives SM-clock stamps of the fused kernel's phases
    (CTA 0); None turns it off.  Layout in include/domino.h (domino_debug_set_trace)."""
    if buf is None:
        _check(lib().domino_debug_set_trace(None, 0), "domino_debug_set_trace")
    else:
        _check(lib().domino_debug_set_trace(ctypes.c_void_p(buf.data_ptr()), buf.numel()), "domino_debug_set_trace")


def set_spin_limit(limit: int) -> None:
    """Test hook: iteration limit of the library's bounded device waits (0 = default)."""
    lib().domino_debug_set_spin_limit(int(limit))


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise DominoError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    """The caller's stream (default: the current stream of `device`), which must belong to `device`."""
    if device.type != "cuda":
        raise ValueError(f"the call's tensors must be on a CUDA device, not {device}")
    s = torch.cuda.current_stream(device) if stream is None else stream
    if s.device != device:
        raise ValueError(f"stream is on {s.device}, the call's tensors on {device}")
    return ctypes.c_void_p(s.cuda_stream)


def _launch(device, fn, *args):
    """Call a library entry point with `device` current: the library queries and launches on the
    current device, which must be the one that holds the call's memory."""
    if torch.cuda.current_device() == device.index:
        return fn(*args)
    with torch.cuda.device(device):
        return fn(*args)


def _expect(t, name: str, shape, dtype, device) -> None:
    """The library sees only a pointer: check here that a tensor has the exact shape, dtype,
    contiguity and device the call reads or writes, so that no kernel touches memory outside it."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if t.shape != shape:  # torch.Size compares equal to a tuple of ints
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(int(x) for x in shape)}")
    if t.dtype is not dtype and not (isinstance(dtype, tuple) and t.dtype in dtype):
        dts = dtype if isinstance(dtype, tuple) else (dtype,)
        raise ValueError(f"{name} has dtype {t.dtype}, expected {' or '.join(str(d) for d in dts)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _expect_status(status, device) -> None:
    if status is not None:
        if not isinstance(status, torch.Tensor) or status.dtype != torch.int32 or status.numel() < 1:
            raise ValueError("status must be an int32 tensor with at least one element")
        if status.device != device:
            raise ValueError(f"status is on {status.device}, expected {device}")


def _expect_workspace(ws, device) -> None:
    if not isinstance(ws, torch.Tensor) or ws.dtype != torch.uint8 or ws.dim() != 1 or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous 1-D uint8 tensor (see alloc_workspace)")
    if ws.device != device:
        raise ValueError(f"workspace is on {ws.device}, expected {device}")


@dataclass
class HeadWeights:
    """Device-resident head weights (all one storage type, fp32 or bf16).

    embed [V, d], W_ih [3Hs, d], W_hh [3Hs, Hs], b_ih [3Hs], b_hh [3Hs], W1 [r, d+Hs], W2 [V, r].
    """
    embed: torch.Tensor
    W_ih: torch.Tensor
    W_hh: torch.Tensor
    b_ih: torch.Tensor
    b_hh: torch.Tensor
    W1: torch.Tensor
    W2: torch.Tensor
    embed_proj: "torch.Tensor | None" = None  # [V, 3Hs] fp32 from project_embeddings, optional

    @property
    def dtype_code(self) -> int:
        if self.W2.dtype == torch.float32:
            return DTYPE_F32
        if self.W2.dtype == torch.bfloat16:
            return DTYPE_BF16
        raise TypeError(f"unsupported weight dtype {self.W2.dtype}")

    def dims(self):
        V, d = self.embed.shape
        Hs = self.W_hh.shape[1]
        r = self.W2.shape[1]
        return d, Hs, r, V

    def check(self) -> None:
        """Every weight has the shape the dimensions of embed, W_hh and W2 imply, the storage type
        of W2, and the device of W2."""
        d, Hs, r, V = self.dims()
        dev = self.W2.device
        want = {"embed": (V, d), "W_ih": (3 * Hs, d), "W_hh": (3 * Hs, Hs), "b_ih": (3 * Hs,), "b_hh": (3 * Hs,),
                "W1": (r, d + Hs), "W2": (V, r)}
        for n, shp in want.items():
            _expect(getattr(self, n), f"weight {n}", shp, self.W2.dtype, dev)
        if self.embed_proj is not None:
            _expect(self.embed_proj, "embed_proj", (V, 3 * Hs), torch.float32, dev)

    def __post_init__(self):
        self.check()
        object.__setattr__(self, "_checked", True)

    def __setattr__(self, name, value):
        # a replaced weight is checked against the others at once (every call relies on it); a
        # rejected one leaves the previous value in place
        old = self.__dict__.get(name)
        object.__setattr__(self, name, value)
        if self.__dict__.get("_checked"):
            try:
                self.check()
            except Exception:
                object.__setattr__(self, name, old)
                raise

    def c_struct(self) -> Weights:
        for n in ("embed", "W_ih", "W_hh", "b_ih", "b_hh", "W1", "W2"):
            if not getattr(self, n).is_cuda:
                raise ValueError(f"weight {n} must be a CUDA tensor")
        xp = self.embed_proj
        ptrs = [self.__dict__[n].data_ptr() for n in ("embed", "W_ih", "W_hh", "b_ih", "b_hh", "W1", "W2")]
        return Weights(*ptrs, xp.data_ptr() if xp is not None else None)


def _check_head_inputs(w: HeadWeights, base_logits, hidden, S0):
    """The inputs every head call reads; returns (B, L, device)."""
    d, Hs, r, V = w.dims()
    dev = w.W2.device
    if not isinstance(base_logits, torch.Tensor) or base_logits.dim() != 3:
        raise ValueError("base_logits must be a [B, L, V] tensor")
    B, L = int(base_logits.shape[0]), int(base_logits.shape[1])
    _expect(base_logits, "base_logits", (B, L, V), w.W2.dtype, dev)
    _expect(hidden, "hidden", (B, L, d), w.W2.dtype, dev)
    _expect(S0, "S0", (B, Hs), torch.float32, dev)
    return B, L, dev


def make_shape(w: HeadWeights, B: int, L: int) -> Shape:
    d, Hs, r, V = w.dims()
    return Shape(int(B), int(L), int(d), int(Hs), int(r), int(V), w.dtype_code)


def workspace_bytes(w: HeadWeights, B: int, L: int) -> int:
    n = int(lib().domino_workspace_bytes(ctypes.byref(make_shape(w, B, L))))
    if n == 0:
        raise DominoError(ERR_INVALID_ARGUMENT, "domino_workspace_bytes")
    return n


def project_embeddings(w: HeadWeights, out=None, status=None, stream=None) -> torch.Tensor:
    """The GRU input projection of every embedding row, [V, 3Hs] fp32 (domino_project_embeddings).
    Assign the result to ``w.embed_proj`` to have every entry point gather it per token."""
    d, Hs, r, V = w.dims()
    if out is None:
        out = torch.empty((V, 3 * Hs), dtype=torch.float32, device=w.W2.device)
    _expect(out, "out", (V, 3 * Hs), torch.float32, w.W2.device)
    _expect_status(status, w.W2.device)
    sh = make_shape(w, 1, 1)
    ws = w.c_struct()
    dev = w.W2.device
    rc = _launch(dev, lib().domino_project_embeddings, ctypes.byref(sh), ctypes.byref(ws), _ptr(out), _ptr(status),
                 _stream(stream, dev))
    _check(rc, "domino_project_embeddings")
    return out


def arena_bytes(w: HeadWeights) -> int:
    n = int(lib().domino_arena_bytes(ctypes.byref(make_shape(w, 1, 1))))
    if n == 0:
        raise DominoError(ERR_INVALID_ARGUMENT, "domino_arena_bytes")
    return n


def pack_weights(w: HeadWeights, stream=None) -> HeadWeights:
    """Copy W2, W1, W_hh, W_ih, b_ih, b_hh into one contiguous arena (domino_pack_weights) and return
    HeadWeights whose tensors are views of it (embed and embed_proj are shared with ``w``)."""
    nbytes = arena_bytes(w)
    arena = torch.empty(nbytes, dtype=torch.uint8, device=w.W2.device)
    sh = make_shape(w, 1, 1)
    src = w.c_struct()
    out = Weights()
    rc = _launch(w.W2.device, lib().domino_pack_weights, ctypes.byref(sh), ctypes.byref(src),
                 ctypes.c_void_p(arena.data_ptr()), nbytes, ctypes.byref(out), _stream(stream, w.W2.device))
    _check(rc, "domino_pack_weights")
    dt = w.W2.dtype
    es = torch.empty((), dtype=dt).element_size()

    def view(name):
        t = getattr(w, name)
        off = getattr(out, name) - arena.data_ptr()
        return arena[off:off + t.numel() * es].view(dt).view(t.shape)

    return HeadWeights(embed=w.embed, W_ih=view("W_ih"), W_hh=view("W_hh"), b_ih=view("b_ih"), b_hh=view("b_hh"),
                       W1=view("W1"), W2=view("W2"), embed_proj=w.embed_proj)


def set_l2_persistence(w: HeadWeights, stream, hit_ratio: float = 1.0) -> None:
    """Opt-in L2 residency of packed weights for kernels on ``stream`` (domino_set_l2_persistence);
    ``hit_ratio=0`` clears it and restores the context's persisting-L2 set-aside."""
    sh = make_shape(w, 1, 1)
    ws = w.c_struct()
    rc = _launch(w.W2.device, lib().domino_set_l2_persistence, ctypes.byref(sh), ctypes.byref(ws),
                 _stream(stream, w.W2.device), float(hit_ratio))
    _check(rc, "domino_set_l2_persistence")


def debug_gemm(A, B, out=None, trans=False, a_kwrap=0, bn=0, ks=0, status=None, stream=None) -> torch.Tensor:
    """The tensor-core GEMM engine on its own (domino_debug_gemm): fp32 A[:, k mod K'] . B^T for bf16
    A [M, K'] and B [N, K]; [M, N], or [N, M] when ``trans``.  bn/ks force a plan (0, 0: automatic)."""
    M, N, K = A.shape[0], B.shape[0], B.shape[1]
    _expect(A, "A", (M, int(a_kwrap) or K), torch.bfloat16, A.device)
    _expect(B, "B", (N, K), torch.bfloat16, A.device)
    if out is None:
        out = torch.empty((N, M) if trans else (M, N), dtype=torch.float32, device=A.device)
    _expect(out, "out", (N, M) if trans else (M, N), torch.float32, A.device)
    _expect_status(status, A.device)
    rc = _launch(A.device, lib().domino_debug_gemm, _ptr(A), _ptr(B), M, N, K, int(a_kwrap), _ptr(out), out.shape[1],
                 int(bool(trans)), int(bn), int(ks), _ptr(status), _stream(stream, A.device))
    _check(rc, "domino_debug_gemm")
    return out


def debug_read_passes(buf, passes: int, stream=None) -> None:
    """Re-read a device buffer `passes` times in one launch (domino_debug_read_passes)."""
    rc = _launch(buf.device, lib().domino_debug_read_passes, _ptr(buf), buf.numel() * buf.element_size(), int(passes),
                 _stream(stream, buf.device))
    _check(rc, "domino_debug_read_passes")


def accept_workspace_bytes(B: int, L: int) -> int:
    return int(lib().domino_accept_workspace_bytes(int(B), int(L)))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    # torch's caching allocator hands out 512-byte aligned blocks
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device or "cuda")


def _check_greedy_outputs(tokens_out, logits_out, states_out, B, L, Hs, V, dev) -> None:
    _expect(tokens_out, "tokens_out", (B, L), torch.int32, dev)
    if logits_out is not None:
        _expect(logits_out, "logits_out", (B, L, V), torch.float32, dev)
    if states_out is not None:
        _expect(states_out, "states_out", (B, L, Hs), torch.float32, dev)


def draft_greedy(w: HeadWeights, base_logits, hidden, S0, tokens_out=None, logits_out=None, states_out=None,
                 workspace=None, status=None, stream=None):
    """Greedy drafting (``domino_draft_greedy``); returns (tokens, logits or None, states or None).

    base_logits [B, L, V] and hidden [B, L, d] in the weights' storage type, S0 [B, Hs] fp32.
    Pass ``logits_out=True`` / ``states_out=True`` to have them allocated, or tensors to fill.
    """
    B, L, dev = _check_head_inputs(w, base_logits, hidden, S0)
    d, Hs, r, V = w.dims()
    if tokens_out is None:
        tokens_out = torch.empty((B, L), dtype=torch.int32, device=dev)
    if logits_out is True:
        logits_out = torch.empty((B, L, V), dtype=torch.float32, device=dev)
    if states_out is True:
        states_out = torch.empty((B, L, Hs), dtype=torch.float32, device=dev)
    if logits_out is False:
        logits_out = None
    if states_out is False:
        states_out = None
    _check_greedy_outputs(tokens_out, logits_out, states_out, B, L, Hs, V, dev)
    _expect_status(status, dev)
    sh = make_shape(w, B, L)
    if workspace is None:
        workspace = alloc_workspace(workspace_bytes(w, B, L), dev)
    _expect_workspace(workspace, dev)
    ws = w.c_struct()
    rc = _launch(dev, lib().domino_draft_greedy, ctypes.byref(sh), ctypes.byref(ws), _ptr(base_logits), _ptr(hidden),
                 _ptr(S0), _ptr(tokens_out), _ptr(logits_out), _ptr(states_out), _ptr(workspace), workspace.numel(),
                 _ptr(status), _stream(stream, dev))
    _check(rc, "domino_draft_greedy")
    return tokens_out, logits_out, states_out


def draft_greedy_noalloc(w: HeadWeights, base_logits, hidden, S0, tokens_out=None, logits_out=None,
                         states_out=None, status=None, stream=None):
    """Greedy drafting with no workspace (``domino_draft_greedy_noalloc``).

    For callers that cannot allocate device memory at call time: the scratch is a fixed array
    inside the library (NOALLOC_SCRATCH_BYTES per device).  Calls that overlap on the GPU share
    that array and race -- keep them on one stream.  Pass preallocated output tensors to keep the
    whole call free of allocations; ``logits_out=True`` / ``states_out=True`` allocate them here.
    """
    B, L, dev = _check_head_inputs(w, base_logits, hidden, S0)
    d, Hs, r, V = w.dims()
    if tokens_out is None:
        tokens_out = torch.empty((B, L), dtype=torch.int32, device=dev)
    if logits_out is True:
        logits_out = torch.empty((B, L, V), dtype=torch.float32, device=dev)
    if states_out is True:
        states_out = torch.empty((B, L, Hs), dtype=torch.float32, device=dev)
    logits_out = None if logits_out is False else logits_out
    states_out = None if states_out is False else states_out
    _check_greedy_outputs(tokens_out, logits_out, states_out, B, L, Hs, V, dev)
    _expect_status(status, dev)
    sh = make_shape(w, B, L)
    ws = w.c_struct()
    rc = _launch(dev, lib().domino_draft_greedy_noalloc, ctypes.byref(sh), ctypes.byref(ws), _ptr(base_logits),
                 _ptr(hidden), _ptr(S0), _ptr(tokens_out), _ptr(logits_out), _ptr(states_out), _ptr(status),
                 _stream(stream, dev))
    _check(rc, "domino_draft_greedy_noalloc")
    return tokens_out, logits_out, states_out


def teacher_forced(w: HeadWeights, base_logits, hidden, S0, tokens, logits_out=None, states_out=None,
                   workspace=None, status=None, stream=None, logits_dtype=torch.float32):
    """Teacher-forced logits (``domino_teacher_forced``, or ``domino_teacher_forced_ex`` for bf16
    logits: ``logits_dtype=torch.bfloat16``); returns (logits, states or None)."""
    B, L, dev = _check_head_inputs(w, base_logits, hidden, S0)
    d, Hs, r, V = w.dims()
    _expect(tokens, "tokens", (B, L), torch.int32, dev)
    if logits_out is None:
        logits_out = torch.empty((B, L, V), dtype=logits_dtype, device=dev)
    _expect(logits_out, "logits_out", (B, L, V), (torch.float32, torch.bfloat16), dev)
    if states_out is True:
        states_out = torch.empty((B, L, Hs), dtype=torch.float32, device=dev)
    if states_out is False:
        states_out = None
    if states_out is not None:
        _expect(states_out, "states_out", (B, L, Hs), torch.float32, dev)
    _expect_status(status, dev)
    sh = make_shape(w, B, L)
    if workspace is None:
        workspace = alloc_workspace(workspace_bytes(w, B, L), dev)
    _expect_workspace(workspace, dev)
    ws = w.c_struct()
    if logits_out.dtype == torch.float32:
        rc = _launch(dev, lib().domino_teacher_forced, ctypes.byref(sh), ctypes.byref(ws), _ptr(base_logits),
                     _ptr(hidden), _ptr(S0), _ptr(tokens), _ptr(logits_out), _ptr(states_out), _ptr(workspace),
                     workspace.numel(), _ptr(status), _stream(stream, dev))
        _check(rc, "domino_teacher_forced")
    else:
        rc = _launch(dev, lib().domino_teacher_forced_ex, ctypes.byref(sh), ctypes.byref(ws), _ptr(base_logits),
                     _ptr(hidden), _ptr(S0), _ptr(tokens), _ptr(logits_out), DTYPE_BF16, _ptr(states_out),
                     _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream, dev))
        _check(rc, "domino_teacher_forced_ex")
    return logits_out, states_out


def accept_len(draft_tokens, target_logits, accept_out=None, workspace=None, status=None, stream=None):
    """Greedy accept length per row (``domino_accept_len``)."""
    if not isinstance(target_logits, torch.Tensor) or target_logits.dim() != 3:
        raise ValueError("target_logits must be a [B, L, V] tensor")
    B, L, V = (int(x) for x in target_logits.shape)
    dev = target_logits.device
    _expect(target_logits, "target_logits", (B, L, V), torch.float32, dev)
    _expect(draft_tokens, "draft_tokens", (B, L), torch.int32, dev)
    if accept_out is None:
        accept_out = torch.empty((B,), dtype=torch.int32, device=dev)
    _expect(accept_out, "accept_out", (B,), torch.int32, dev)
    _expect_status(status, dev)
    if workspace is None:
        workspace = alloc_workspace(accept_workspace_bytes(B, L), dev)
    _expect_workspace(workspace, dev)
    rc = _launch(dev, lib().domino_accept_len, B, L, V, _ptr(draft_tokens), _ptr(target_logits), _ptr(accept_out),
                 _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream, dev))
    _check(rc, "domino_accept_len")
    return accept_out


def accept_sample(draft_tokens, target_logits, temperature: float, uniforms, draft_logits=None, accept_out=None,
                  next_out=None, workspace=None, status=None, stream=None):
    """Sampled verification (``domino_accept_sample``): returns (accept lengths [B], replacement
    tokens [B], -1 where every position was accepted).  ``draft_logits`` None means a greedy draft
    (one-hot draft distribution); ``uniforms`` [B, L + 1] fp32 are the caller's random draws."""
    if not isinstance(target_logits, torch.Tensor) or target_logits.dim() != 3:
        raise ValueError("target_logits must be a [B, L, V] tensor")
    B, L, V = (int(x) for x in target_logits.shape)
    dev = target_logits.device
    _expect(target_logits, "target_logits", (B, L, V), torch.float32, dev)
    if draft_logits is not None:
        _expect(draft_logits, "draft_logits", (B, L, V), torch.float32, dev)
    _expect(draft_tokens, "draft_tokens", (B, L), torch.int32, dev)
    _expect(uniforms, "uniforms", (B, L + 1), torch.float32, dev)
    if accept_out is None:
        accept_out = torch.empty((B,), dtype=torch.int32, device=dev)
    if next_out is None:
        next_out = torch.empty((B,), dtype=torch.int32, device=dev)
    _expect(accept_out, "accept_out", (B,), torch.int32, dev)
    _expect(next_out, "next_out", (B,), torch.int32, dev)
    _expect_status(status, dev)
    if workspace is None:
        n = int(lib().domino_accept_sample_workspace_bytes(B, L, V))
        if n == 0:
            raise DominoError(ERR_INVALID_ARGUMENT, "domino_accept_sample_workspace_bytes")
        workspace = alloc_workspace(n, dev)
    _expect_workspace(workspace, dev)
    rc = _launch(dev, lib().domino_accept_sample, B, L, V, _ptr(draft_tokens), _ptr(draft_logits),
                 _ptr(target_logits), float(temperature), _ptr(uniforms), _ptr(accept_out), _ptr(next_out),
                 _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream, dev))
    _check(rc, "domino_accept_sample")
    return accept_out, next_out


def to_device_weights(host: dict, dtype_code: int, device="cuda") -> HeadWeights:
    """Move generator arrays (fp32, or bf16 bit patterns in uint16) to device tensors."""
    def cv(a):
        t = torch.from_numpy(a)
        if dtype_code == DTYPE_BF16:
            t = t.view(torch.int16).view(torch.bfloat16) if t.dtype == torch.uint16 else t
        return t.to(device, non_blocking=False).contiguous()
    return HeadWeights(**{k: cv(host[k]) for k in ("embed", "W_ih", "W_hh", "b_ih", "b_hh", "W1", "W2")})


def to_device(a, dtype_code: int, device="cuda") -> torch.Tensor:
    """One generator array to the device; uint16 arrays are bf16 bit patterns."""
    t = torch.from_numpy(a)
    if t.dtype == torch.uint16:
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.to(device).contiguous()
