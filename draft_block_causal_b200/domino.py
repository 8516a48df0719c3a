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
           "domino_greedy_plan", "domino_draft_greedy_noalloc", "domino_debug_set_trace",
           "domino_embed_proj_bytes", "domino_project_embeddings", "domino_arena_bytes",
           "domino_pack_weights", "domino_set_l2_persistence", "domino_debug_gemm",
           "domino_debug_read_passes", "domino_teacher_forced_ex")


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


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


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

    def c_struct(self) -> Weights:
        for n in ("embed", "W_ih", "W_hh", "b_ih", "b_hh", "W1", "W2"):
            t = getattr(self, n)
            if not t.is_contiguous() or t.dtype != self.W2.dtype or not t.is_cuda:
                raise ValueError(f"weight {n} must be a contiguous CUDA tensor of dtype {self.W2.dtype}")
        xp = self.embed_proj
        if xp is not None and (xp.dtype != torch.float32 or not xp.is_contiguous() or not xp.is_cuda):
            raise ValueError("embed_proj must be a contiguous CUDA float32 tensor [V, 3Hs]")
        ptrs = [self.__dict__[n].data_ptr() for n in ("embed", "W_ih", "W_hh", "b_ih", "b_hh", "W1", "W2")]
        return Weights(*ptrs, xp.data_ptr() if xp is not None else None)


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
    sh = make_shape(w, 1, 1)
    ws = w.c_struct()
    rc = lib().domino_project_embeddings(ctypes.byref(sh), ctypes.byref(ws), _ptr(out), _ptr(status), _stream(stream))
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
    rc = lib().domino_pack_weights(ctypes.byref(sh), ctypes.byref(src), ctypes.c_void_p(arena.data_ptr()),
                                   nbytes, ctypes.byref(out), _stream(stream))
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
    rc = lib().domino_set_l2_persistence(ctypes.byref(sh), ctypes.byref(ws), _stream(stream), float(hit_ratio))
    _check(rc, "domino_set_l2_persistence")


def debug_gemm(A, B, out=None, trans=False, a_kwrap=0, bn=0, ks=0, status=None, stream=None) -> torch.Tensor:
    """The tensor-core GEMM engine on its own (domino_debug_gemm): fp32 A[:, k mod K'] . B^T for bf16
    A [M, K'] and B [N, K]; [M, N], or [N, M] when ``trans``.  bn/ks force a plan (0, 0: automatic)."""
    M, N, K = A.shape[0], B.shape[0], B.shape[1]
    if out is None:
        out = torch.empty((N, M) if trans else (M, N), dtype=torch.float32, device=A.device)
    rc = lib().domino_debug_gemm(_ptr(A), _ptr(B), M, N, K, int(a_kwrap), _ptr(out), out.shape[1], int(bool(trans)),
                                 int(bn), int(ks), _ptr(status), _stream(stream))
    _check(rc, "domino_debug_gemm")
    return out


def debug_read_passes(buf, passes: int, stream=None) -> None:
    """Re-read a device buffer `passes` times in one launch (domino_debug_read_passes)."""
    rc = lib().domino_debug_read_passes(_ptr(buf), buf.numel() * buf.element_size(), int(passes), _stream(stream))
    _check(rc, "domino_debug_read_passes")


def accept_workspace_bytes(B: int, L: int) -> int:
    return int(lib().domino_accept_workspace_bytes(int(B), int(L)))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    # torch's caching allocator hands out 512-byte aligned blocks
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device or "cuda")


def draft_greedy(w: HeadWeights, base_logits, hidden, S0, tokens_out=None, logits_out=None, states_out=None,
                 workspace=None, status=None, stream=None):
    """Greedy drafting (``domino_draft_greedy``); returns (tokens, logits or None, states or None).

    base_logits [B, L, V] and hidden [B, L, d] in the weights' storage type, S0 [B, Hs] fp32.
    Pass ``logits_out=True`` / ``states_out=True`` to have them allocated, or tensors to fill.
    """
    B, L, V = base_logits.shape
    dev = base_logits.device
    if tokens_out is None:
        tokens_out = torch.empty((B, L), dtype=torch.int32, device=dev)
    if logits_out is True:
        logits_out = torch.empty((B, L, V), dtype=torch.float32, device=dev)
    if states_out is True:
        states_out = torch.empty((B, L, w.W_hh.shape[1]), dtype=torch.float32, device=dev)
    if logits_out is False:
        logits_out = None
    if states_out is False:
        states_out = None
    sh = make_shape(w, B, L)
    if workspace is None:
        workspace = alloc_workspace(workspace_bytes(w, B, L), dev)
    ws = w.c_struct()
    rc = lib().domino_draft_greedy(ctypes.byref(sh), ctypes.byref(ws), _ptr(base_logits), _ptr(hidden), _ptr(S0),
                                   _ptr(tokens_out), _ptr(logits_out), _ptr(states_out), _ptr(workspace),
                                   workspace.numel(), _ptr(status), _stream(stream))
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
    B, L, V = base_logits.shape
    dev = base_logits.device
    if tokens_out is None:
        tokens_out = torch.empty((B, L), dtype=torch.int32, device=dev)
    if logits_out is True:
        logits_out = torch.empty((B, L, V), dtype=torch.float32, device=dev)
    if states_out is True:
        states_out = torch.empty((B, L, w.W_hh.shape[1]), dtype=torch.float32, device=dev)
    logits_out = None if logits_out is False else logits_out
    states_out = None if states_out is False else states_out
    sh = make_shape(w, B, L)
    ws = w.c_struct()
    rc = lib().domino_draft_greedy_noalloc(ctypes.byref(sh), ctypes.byref(ws), _ptr(base_logits), _ptr(hidden),
                                           _ptr(S0), _ptr(tokens_out), _ptr(logits_out), _ptr(states_out),
                                           _ptr(status), _stream(stream))
    _check(rc, "domino_draft_greedy_noalloc")
    return tokens_out, logits_out, states_out


def teacher_forced(w: HeadWeights, base_logits, hidden, S0, tokens, logits_out=None, states_out=None,
                   workspace=None, status=None, stream=None, logits_dtype=torch.float32):
    """Teacher-forced logits (``domino_teacher_forced``, or ``domino_teacher_forced_ex`` for bf16
    logits: ``logits_dtype=torch.bfloat16``); returns (logits, states or None)."""
    B, L, V = base_logits.shape
    dev = base_logits.device
    if logits_out is None:
        logits_out = torch.empty((B, L, V), dtype=logits_dtype, device=dev)
    if logits_out.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("logits_out must be float32 or bfloat16")
    if states_out is True:
        states_out = torch.empty((B, L, w.W_hh.shape[1]), dtype=torch.float32, device=dev)
    if states_out is False:
        states_out = None
    sh = make_shape(w, B, L)
    if workspace is None:
        workspace = alloc_workspace(workspace_bytes(w, B, L), dev)
    ws = w.c_struct()
    if logits_out.dtype == torch.float32:
        rc = lib().domino_teacher_forced(ctypes.byref(sh), ctypes.byref(ws), _ptr(base_logits), _ptr(hidden),
                                         _ptr(S0), _ptr(tokens), _ptr(logits_out), _ptr(states_out),
                                         _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
        _check(rc, "domino_teacher_forced")
    else:
        rc = lib().domino_teacher_forced_ex(ctypes.byref(sh), ctypes.byref(ws), _ptr(base_logits), _ptr(hidden),
                                            _ptr(S0), _ptr(tokens), _ptr(logits_out), DTYPE_BF16, _ptr(states_out),
                                            _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
        _check(rc, "domino_teacher_forced_ex")
    return logits_out, states_out


def accept_len(draft_tokens, target_logits, accept_out=None, workspace=None, status=None, stream=None):
    """Greedy accept length per row (``domino_accept_len``)."""
    B, L, V = target_logits.shape
    dev = target_logits.device
    if accept_out is None:
        accept_out = torch.empty((B,), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(accept_workspace_bytes(B, L), dev)
    rc = lib().domino_accept_len(B, L, V, _ptr(draft_tokens), _ptr(target_logits), _ptr(accept_out),
                                 _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
    _check(rc, "domino_accept_len")
    return accept_out


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
