"""Python binding of libslra.so (the C ABI in include/slra.h): argument marshalling only.

Every step of the forward pass runs in the library's CUDA kernels; this module only fills the
problem struct, hands device pointers (torch tensors' storage) and the current torch stream to the
C entry points, and raises on a non-zero status.  If the library cannot be loaded the calls raise:
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libslra.so")

OK = 0
ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_RANGE, \
    ERR_NO_DEVICE, ERR_SCRATCH_LIMIT = range(1, 10)
OUT_F32, OUT_BF16 = 0, 1
BRANCH_SPARSE, BRANCH_LOWRANK, BRANCH_BOTH = 1, 2, 3
DEBUG_UNSATISFIED_WAIT, DEBUG_SERIAL_BRANCHES = 1, 2
ABI_VERSION = 8
DTYPE_BF16, DTYPE_F32 = 0, 1
ACT_RELU, ACT_SILU, ACT_IDENTITY, ACT_TANH = 0, 1, 2, 3
FUSION_SUM, FUSION_GATED = 0, 1

# Every symbol include/slra.h declares.
EXPORTS = ("slra_abi_version", "slra_status_string", "slra_problem_init", "slra_validate", "slra_keep_count",
           "slra_projection_elems", "slra_workspace_bytes", "slra_attn_fwd", "slra_attn_fwd_ex", "slra_sparse_fwd",
           "slra_lowrank_fwd", "slra_get_device_status", "slra_bwd_workspace_bytes", "slra_attn_bwd",
           "slra_workspace_layout", "slra_host_io_bytes", "slra_host_pipeline_groups",
           "slra_attn_fwd_host",
           "slra_select_blocks", "slra_lowrank_summary", "slra_device_status", "slra_lowrank_summary_noalloc",
           "slra_noalloc_device_status", "slra_attn_fwd_train", "slra_attn_bwd_saved")


class SlraError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


class _Problem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("heads", ctypes.c_int64), ("head_dim", ctypes.c_int64),
                ("T", ctypes.c_int64), ("H", ctypes.c_int64), ("W", ctypes.c_int64),
                ("block", ctypes.c_int64), ("keep_frac", ctypes.c_double), ("rank", ctypes.c_int64),
                ("theta", ctypes.c_double), ("out_dtype", ctypes.c_int32), ("branches", ctypes.c_int32),
                ("pos_offset", ctypes.c_int64 * 3), ("rope_split", ctypes.c_int64 * 3),
                ("wait_timeout_ns", ctypes.c_uint64), ("debug_flags", ctypes.c_uint32),
                ("stage_events", ctypes.c_void_p * 7), ("activation", ctypes.c_int32),
                ("lowrank_norope", ctypes.c_int32), ("proj_separate", ctypes.c_int32),
                ("proj_per_head", ctypes.c_int32), ("fusion", ctypes.c_int32), ("gate_bias", ctypes.c_float),
                ("gate_w", ctypes.c_void_p), ("lowrank_rope_inside", ctypes.c_int32),
                ("q_strides", ctypes.c_int64 * 3), ("k_strides", ctypes.c_int64 * 3),
                ("v_strides", ctypes.c_int64 * 3), ("out_strides", ctypes.c_int64 * 3),
                ("dgate_w", ctypes.c_void_p), ("dgate_b", ctypes.c_void_p)]


class _Tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("B", ctypes.c_int64), ("L", ctypes.c_int64),
                ("Hh", ctypes.c_int64), ("D", ctypes.c_int64), ("sB", ctypes.c_int64), ("sL", ctypes.c_int64),
                ("sH", ctypes.c_int64)]


class _Mat(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("D", ctypes.c_int64), ("R", ctypes.c_int64)]


class _Layout(ctypes.Structure):
    _fields_ = [("total_bytes", ctypes.c_size_t), ("L", ctypes.c_int64), ("nb", ctypes.c_int64),
                ("keep", ctypes.c_int64), ("nsplit", ctypes.c_int64)] + \
               [(n, ctypes.c_size_t) for n in ("status", "rope_table", "qh", "kh", "vh", "qbar", "kbar", "idx",
                                               "tie", "s_part", "z_part", "S", "z")]


_lib = None


def lib():
    """Load libslra.so (raises if it is missing: the CUDA path has no substitute)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m sparse_rank_hybrid_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.slra_abi_version.restype = ctypes.c_int
        if L.slra_abi_version() != ABI_VERSION:  # the structs below mirror this version of include/slra.h
            raise RuntimeError(f"{LIB_PATH} has ABI {L.slra_abi_version()}, this binding expects {ABI_VERSION}")
        P, S = ctypes.c_void_p, ctypes.c_size_t
        PP = ctypes.POINTER(_Problem)
        L.slra_abi_version.restype = ctypes.c_int
        L.slra_status_string.restype = ctypes.c_char_p
        L.slra_status_string.argtypes = [ctypes.c_int]
        L.slra_problem_init.argtypes = [PP] + [ctypes.c_int64] * 7 + [ctypes.c_double, ctypes.c_int64]
        L.slra_validate.argtypes = [PP]
        L.slra_keep_count.restype = ctypes.c_int64
        L.slra_keep_count.argtypes = [PP]
        L.slra_projection_elems.restype = ctypes.c_int64
        L.slra_projection_elems.argtypes = [PP]
        L.slra_workspace_layout.argtypes = [PP, ctypes.POINTER(_Layout)]
        L.slra_attn_fwd_ex.argtypes = [PP, P, P, P, P, P, P, S, P]
        PT, PM, I64, C = ctypes.POINTER(_Tensor), ctypes.POINTER(_Mat), ctypes.c_int64, ctypes.c_int
        L.slra_workspace_bytes.restype = S
        L.slra_workspace_bytes.argtypes = [I64] * 7 + [ctypes.c_float, I64]
        L.slra_attn_fwd.argtypes = [PT, PT, PT, PM, C, C, C, C, ctypes.c_float, C, PT, P]
        L.slra_sparse_fwd.argtypes = [PT, PT, PT, C, C, C, C, ctypes.c_float, PT, P, S, P]
        L.slra_lowrank_fwd.argtypes = [PT, PT, PT, PM, C, C, C, C, PT, P, P, P, S, P]
        L.slra_get_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
        L.slra_bwd_workspace_bytes.restype = S
        L.slra_bwd_workspace_bytes.argtypes = [PP]
        L.slra_attn_bwd.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, S, P]
        L.slra_attn_bwd_saved.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, S, P]
        L.slra_attn_fwd_train.argtypes = [PP, P, P, P, P, P, P, S, P]
        L.slra_host_io_bytes.restype = S
        L.slra_host_io_bytes.argtypes = [PP]
        L.slra_host_pipeline_groups.restype = ctypes.c_int64
        L.slra_host_pipeline_groups.argtypes = [PP, S, S]
        L.slra_attn_fwd_host.argtypes = [PP, P, P, P, P, P, P, S, P, S, P]
        L.slra_select_blocks.argtypes = [PP, P, P, P, P, S, P]
        L.slra_lowrank_summary.argtypes = [PP, P, P, P, P, S, P]
        L.slra_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
        L.slra_lowrank_summary_noalloc.argtypes = [PP, P, P, P, P, P, P]
        L.slra_noalloc_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
        for name in ("slra_problem_init", "slra_validate", "slra_workspace_layout", "slra_attn_fwd",
                     "slra_attn_fwd_ex", "slra_sparse_fwd", "slra_lowrank_fwd", "slra_get_device_status",
                     "slra_attn_bwd", "slra_attn_bwd_saved", "slra_attn_fwd_train",
                     "slra_attn_fwd_host", "slra_select_blocks", "slra_lowrank_summary", "slra_device_status",
                     "slra_lowrank_summary_noalloc", "slra_noalloc_device_status"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().slra_status_string(int(s)).decode()


def _check(s: int, where: str):
    if s != OK:
        raise SlraError(s, where)


@dataclass
class Problem:
    batch: int
    heads: int
    head_dim: int
    T: int
    H: int
    W: int
    block: int
    keep_frac: float
    rank: int
    theta: float = 1e4
    out_dtype: int = OUT_F32
    branches: int = BRANCH_BOTH
    pos_offset: tuple = (0, 0, 0)
    rope_split: tuple = (0, 0, 0)
    wait_timeout_ns: int = 2_000_000_000
    debug_flags: int = 0
    stage_events: tuple = (None,) * 7  # raw cudaEvent_t handles (ints) or None, see slra_problem
    activation: int = 0                # ACT_* map of the low-rank features
    lowrank_norope: int = 0            # 1: no RoPE in the low-rank branch
    proj_separate: int = 0             # 1: separate query / key projections Pq, Pk
    proj_per_head: int = 0             # 1: one projection (pair) per head
    fusion: int = 0                    # FUSION_SUM or FUSION_GATED
    gate_bias: float = 0.0             # bg of the gated fusion
    gate_w: object = None              # Wg of the gated fusion: CUDA fp32 tensor [head_dim] (or None)
    lowrank_rope_inside: int = 0       # 1: the low-rank RoPE before the activation
    q_strides: tuple = (0, 0, 0)       # (sB, sL, sH) element strides; all 0 = contiguous [B, L, Hh, D]
    k_strides: tuple = (0, 0, 0)
    v_strides: tuple = (0, 0, 0)
    out_strides: tuple = (0, 0, 0)
    dgate_w: object = None             # backward, gated: output CUDA fp32 tensor [head_dim] (d loss / d Wg)
    dgate_b: object = None             # backward, gated: output CUDA fp32 tensor [1] (d loss / d bg)

    @property
    def L(self) -> int:
        return self.T * self.H * self.W

    @classmethod
    def from_workload(cls, w, **kw) -> "Problem":
        return cls(w.batch, w.heads, w.head_dim, w.T, w.H, w.W, w.block, w.keep_frac, w.rank, **kw)

    def c(self) -> _Problem:
        p = _Problem()
        _check(lib().slra_problem_init(ctypes.byref(p), self.batch, self.heads, self.head_dim, self.T, self.H,
                                       self.W, self.block, float(self.keep_frac), self.rank), "slra_problem_init")
        p.theta = float(self.theta)
        p.out_dtype = int(self.out_dtype)
        p.branches = int(self.branches)
        p.pos_offset[:] = [int(x) for x in self.pos_offset]
        p.rope_split[:] = [int(x) for x in self.rope_split]
        p.wait_timeout_ns = int(self.wait_timeout_ns)
        p.debug_flags = int(self.debug_flags)
        for i, e in enumerate(self.stage_events):
            p.stage_events[i] = e
        p.activation = int(self.activation)
        p.lowrank_norope = int(self.lowrank_norope)
        p.proj_separate = int(self.proj_separate)
        p.proj_per_head = int(self.proj_per_head)
        p.fusion = int(self.fusion)
        p.gate_bias = float(self.gate_bias)
        p.lowrank_rope_inside = int(self.lowrank_rope_inside)
        for name in ("q_strides", "k_strides", "v_strides", "out_strides"):
            getattr(p, name)[:] = [int(x) for x in getattr(self, name)]
        if self.gate_w is not None:
            t = self.gate_w
            torch = _torch()
            if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (self.head_dim,):
                raise ValueError(f"gate_w: expected a contiguous CUDA fp32 tensor of shape ({self.head_dim},)")
            p.gate_w = int(t.data_ptr())
        for name, n in (("dgate_w", self.head_dim), ("dgate_b", 1)):
            t = getattr(self, name)
            if t is not None:
                torch = _torch()
                if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or t.numel() != n:
                    raise ValueError(f"{name}: expected a contiguous CUDA fp32 tensor of {n} elements")
                setattr(p, name, int(t.data_ptr()))
        return p

    @property
    def projection_shape(self) -> tuple:
        """Shape of the projection argument A: [D, rank] by default, else
        [1 + proj_separate, proj_per_head ? heads : 1, D, rank] (query projections first)."""
        if not self.proj_separate and not self.proj_per_head:
            return (self.head_dim, self.rank)
        return (1 + int(self.proj_separate), self.heads if self.proj_per_head else 1, self.head_dim, self.rank)


@dataclass
class Layout:
    total_bytes: int
    L: int
    nb: int
    keep: int
    nsplit: int
    offsets: dict = field(default_factory=dict)


def validate(prob: Problem) -> int:
    return int(lib().slra_validate(ctypes.byref(prob.c())))


def keep_count(prob: Problem) -> int:
    return int(lib().slra_keep_count(ctypes.byref(prob.c())))


def projection_elems(prob: Problem) -> int:
    return int(lib().slra_projection_elems(ctypes.byref(prob.c())))


def layout(prob: Problem) -> Layout:
    lay = _Layout()
    _check(lib().slra_workspace_layout(ctypes.byref(prob.c()), ctypes.byref(lay)), "slra_workspace_layout")
    offs = {n: int(getattr(lay, n)) for n, _ in _Layout._fields_[5:]}
    return Layout(int(lay.total_bytes), int(lay.L), int(lay.nb), int(lay.keep), int(lay.nsplit), offs)


# ------------------------------------------------------------------------------- torch helpers
def _torch():
    import torch
    return torch


def _ptr(t) -> int:
    return int(t.data_ptr())


def _stream_handle(stream) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def alloc_workspace(prob: Problem, device="cuda"):
    torch = _torch()
    return torch.empty(layout(prob).total_bytes, dtype=torch.uint8, device=device)


def _check_bf16(name, t, shape):
    torch = _torch()
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected contiguous CUDA bf16 tensor of shape {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


def _row_strides(name, t, shape, dtype):
    """(sB, sL, sH) element strides of a [B, L, Hh, D] CUDA tensor whose last dimension is contiguous;
    (0, 0, 0) when the whole tensor is contiguous."""
    if t.dtype != dtype or not t.is_cuda or tuple(t.shape) != tuple(shape) or t.stride(3) != 1:
        raise ValueError(f"{name}: expected a CUDA {dtype} tensor of shape {tuple(shape)} with a contiguous last "
                         f"dimension, got {t.dtype} {tuple(t.shape)} strides {t.stride()} on {t.device}")
    return (0, 0, 0) if t.is_contiguous() else (t.stride(0), t.stride(1), t.stride(2))


def attn_fwd(prob: Problem, q, k, v, A, out=None, workspace=None, stream=None, alloc_workspace_in_library=False):
    """Full forward pass through slra_attn_fwd_ex.  q, k, v: CUDA bf16 [B, L, Hh, D] with a contiguous
    last dimension (any other strides, e.g. views of a fused QKV tensor); A: CUDA bf16 of
    prob.projection_shape.  Returns (out, workspace); out is fp32 or bf16 [B, L, Hh, D] as
    prob.out_dtype (a given out may be strided too).  alloc_workspace_in_library=True passes a NULL
    workspace (the library allocates it on the stream) and returns None for it."""
    import dataclasses
    torch = _torch()
    shp = (prob.batch, prob.L, prob.heads, prob.head_dim)
    odt = torch.float32 if prob.out_dtype == OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty(shp, dtype=odt, device=q.device)
    strides = {f"{n}_strides": _row_strides(n, t, shp, dt) for n, t, dt in
               (("q", q, torch.bfloat16), ("k", k, torch.bfloat16), ("v", v, torch.bfloat16), ("out", out, odt))}
    if prob.branches & BRANCH_LOWRANK or A is not None:
        _check_bf16("A", A, prob.projection_shape)
    p = dataclasses.replace(prob, **strides)
    if workspace is None and not alloc_workspace_in_library:
        workspace = alloc_workspace(p, q.device)
    ws_ptr, ws_n = (0, 0) if workspace is None else (_ptr(workspace), workspace.numel())
    _check(lib().slra_attn_fwd_ex(ctypes.byref(p.c()), _ptr(q), _ptr(k), _ptr(v), 0 if A is None else _ptr(A),
                                  _ptr(out), ws_ptr or None, ws_n, _stream_handle(stream)), "slra_attn_fwd_ex")
    return out, workspace


def _tensor(t, dtype_code) -> _Tensor:
    """Descriptor of a [B, L, Hh, D] CUDA tensor (strides in elements; the last dimension contiguous)."""
    if t.dim() != 4 or t.stride(3) != 1 or not t.is_cuda:
        raise ValueError("expected a CUDA [B, L, Hh, D] tensor with a contiguous last dimension")
    return _Tensor(_ptr(t), dtype_code, *t.shape, t.stride(0), t.stride(1), t.stride(2))


def _dtype_code(t) -> int:
    torch = _torch()
    return {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}[t.dtype]


def workspace_bytes(batch, heads, head_dim, T, H, W, block, keep_frac, rank) -> int:
    return int(lib().slra_workspace_bytes(batch, heads, head_dim, T, H, W, block, float(keep_frac), rank))


def attn_fwd_tensors(q, k, v, A, T, H, W, block, keep_frac, rank, out, stream=None):
    """slra_attn_fwd: the forward pass from tensor descriptors (strides taken from the tensors), the
    workspace allocated by the library on the stream."""
    a = _Mat(_ptr(A), DTYPE_BF16 if A.dtype == _torch().bfloat16 else DTYPE_F32, A.shape[0], A.shape[1])
    tq, tk, tv, to = (_tensor(t, _dtype_code(t)) for t in (q, k, v, out))
    _check(lib().slra_attn_fwd(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), ctypes.byref(a), T, H, W,
                               block, float(keep_frac), rank, ctypes.byref(to), _stream_handle(stream)),
           "slra_attn_fwd")
    return out


def sparse_fwd(q, k, v, T, H, W, block, keep_frac, out, workspace=None, stream=None):
    """slra_sparse_fwd: the sparse branch alone into out (workspace None = allocated by the library)."""
    tq, tk, tv, to = (_tensor(t, _dtype_code(t)) for t in (q, k, v, out))
    ws_ptr, ws_n = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel())
    _check(lib().slra_sparse_fwd(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), T, H, W, block,
                                 float(keep_frac), ctypes.byref(to), ws_ptr, ws_n, _stream_handle(stream)),
           "slra_sparse_fwd")
    return out


def lowrank_fwd(q, k, v, A, T, H, W, rank, out, S=None, z=None, workspace=None, stream=None):
    """slra_lowrank_fwd: the low-rank branch alone into out; S, z (fp32 CUDA) receive the summary."""
    a = _Mat(_ptr(A), DTYPE_BF16, A.shape[0], A.shape[1])
    tq, tk, tv, to = (_tensor(t, _dtype_code(t)) for t in (q, k, v, out))
    ws_ptr, ws_n = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel())
    _check(lib().slra_lowrank_fwd(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), ctypes.byref(a), T, H, W,
                                  rank, ctypes.byref(to), None if S is None else _ptr(S),
                                  None if z is None else _ptr(z), ws_ptr, ws_n, _stream_handle(stream)),
           "slra_lowrank_fwd")
    return out


def bwd_workspace_bytes(prob: Problem) -> int:
    return int(lib().slra_bwd_workspace_bytes(ctypes.byref(prob.c())))


def attn_fwd_train(prob: Problem, q, k, v, A, out=None, workspace=None, stream=None):
    """Forward pass for training (slra_attn_fwd_train): out as attn_fwd gives it, and the workspace
    (backward-sized, allocated when None) keeps what attn_bwd_saved needs.  Returns (out, workspace)."""
    import dataclasses
    torch = _torch()
    shp = (prob.batch, prob.L, prob.heads, prob.head_dim)
    strides = {f"{n}_strides": _row_strides(n, t, shp, torch.bfloat16) for n, t in (("q", q), ("k", k), ("v", v))}
    p = dataclasses.replace(prob, **strides)
    if A is not None:
        _check_bf16("A", A, prob.projection_shape)
    if out is None:
        out = torch.empty(shp, dtype=torch.float32 if prob.out_dtype == OUT_F32 else torch.bfloat16, device=q.device)
    if workspace is None:
        n = bwd_workspace_bytes(p)
        if n == 0:
            raise SlraError(ERR_UNSUPPORTED, "slra_bwd_workspace_bytes")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    _check(lib().slra_attn_fwd_train(ctypes.byref(p.c()), _ptr(q), _ptr(k), _ptr(v), None if A is None else _ptr(A),
                                     _ptr(out), _ptr(workspace), workspace.numel(), _stream_handle(stream)),
           "slra_attn_fwd_train")
    return out, workspace


def attn_bwd_saved(prob: Problem, q, k, v, A, dout, workspace, grads=None, stream=None):
    """Backward pass from attn_fwd_train's workspace (slra_attn_bwd_saved): as attn_bwd, without the
    recompute.  Returns (dq, dk, dv, dA, workspace)."""
    return attn_bwd(prob, q, k, v, A, dout, grads=grads, workspace=workspace, stream=stream, _saved=True)


def attn_bwd(prob: Problem, q, k, v, A, dout, grads=None, workspace=None, stream=None, _saved=False):
    """Backward pass (slra_attn_bwd): gradients of sum(dout * out) for q, k, v (fp32 [B, L, Hh, D]) and the
    projection(s) A (fp32, prob.projection_shape).  dout: contiguous CUDA fp32 [B, L, Hh, D].  q, k, v may be
    strided views.  With the gated fusion, prob.dgate_w and prob.dgate_b receive the gate parameters'
    gradients.  Returns (dq, dk, dv, dA, workspace)."""
    import dataclasses
    torch = _torch()
    shp = (prob.batch, prob.L, prob.heads, prob.head_dim)
    strides = {f"{n}_strides": _row_strides(n, t, shp, torch.bfloat16) for n, t in (("q", q), ("k", k), ("v", v))}
    p = dataclasses.replace(prob, **strides)
    if dout.dtype != torch.float32 or not dout.is_cuda or not dout.is_contiguous() or tuple(dout.shape) != shp:
        raise ValueError(f"dout: expected a contiguous CUDA fp32 tensor of shape {shp}")
    if A is not None:
        _check_bf16("A", A, prob.projection_shape)
    if grads is None:
        grads = tuple(torch.empty(shp, dtype=torch.float32, device=q.device) for _ in range(3)) + \
            (torch.empty(prob.projection_shape, dtype=torch.float32, device=q.device),)
    dq, dk, dv, dA = grads
    if workspace is None:
        n = bwd_workspace_bytes(p)
        if n == 0:
            raise SlraError(ERR_UNSUPPORTED, "slra_bwd_workspace_bytes")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    fn = "slra_attn_bwd_saved" if _saved else "slra_attn_bwd"
    _check(getattr(lib(), fn)(ctypes.byref(p.c()), _ptr(q), _ptr(k), _ptr(v), None if A is None else _ptr(A),
                              _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dA), _ptr(workspace),
                              workspace.numel(), _stream_handle(stream)), fn)
    return dq, dk, dv, dA, workspace


def get_device_status(stream=None) -> int:
    """Read and clear the device status of the calls whose workspace the library allocated."""
    st = ctypes.c_int32(-1)
    _check(lib().slra_get_device_status(_stream_handle(stream), ctypes.byref(st)), "slra_get_device_status")
    return int(st.value)


def host_io_bytes(prob: Problem) -> int:
    return int(lib().slra_host_io_bytes(ctypes.byref(prob.c())))


def host_pipeline_groups(prob: Problem, io_bytes: int, workspace_bytes: int) -> int:
    """Head groups the host entry point pipelines for these buffer sizes (1: none)."""
    return int(lib().slra_host_pipeline_groups(ctypes.byref(prob.c()), io_bytes, workspace_bytes))


def attn_fwd_host(prob: Problem, q_host, k_host, v_host, A_host, out_host, io, workspace, stream=None):
    """Forward pass on host buffers (pinned CPU tensors): copies in, computes, copies out, synchronizes."""
    if A_host.numel() != projection_elems(prob):
        raise ValueError(f"A_host: expected {projection_elems(prob)} elements, got {A_host.numel()}")
    _check(lib().slra_attn_fwd_host(ctypes.byref(prob.c()), _ptr(q_host), _ptr(k_host), _ptr(v_host),
                                    _ptr(A_host), _ptr(out_host), _ptr(io), io.numel(), _ptr(workspace),
                                    workspace.numel(), _stream_handle(stream)), "slra_attn_fwd_host")
    return out_host


def select_blocks(prob: Problem, q, k, v, workspace=None, stream=None):
    if workspace is None:
        workspace = alloc_workspace(prob, q.device)
    _check(lib().slra_select_blocks(ctypes.byref(prob.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(workspace),
                                    workspace.numel(), _stream_handle(stream)), "slra_select_blocks")
    return workspace


def lowrank_summary(prob: Problem, k, v, A, workspace=None, stream=None):
    _check_bf16("A", A, prob.projection_shape)
    if workspace is None:
        workspace = alloc_workspace(prob, k.device)
    _check(lib().slra_lowrank_summary(ctypes.byref(prob.c()), _ptr(k), _ptr(v), _ptr(A), _ptr(workspace),
                                      workspace.numel(), _stream_handle(stream)), "slra_lowrank_summary")
    return workspace


def lowrank_summary_noalloc(prob: Problem, k, v, A, S, z, stream=None):
    """Low-rank summary into caller tensors S [B*Hh, rank, D] and z [B*Hh, rank] (fp32, CUDA) without
    any allocation: the library's fixed scratch array is used instead of a workspace."""
    _check_bf16("A", A, prob.projection_shape)
    _check(lib().slra_lowrank_summary_noalloc(ctypes.byref(prob.c()), _ptr(k), _ptr(v), _ptr(A), _ptr(S), _ptr(z),
                                              _stream_handle(stream)), "slra_lowrank_summary_noalloc")
    return S, z


def noalloc_device_status(stream=None) -> int:
    """Read and clear the device status of the no-allocation summary on the current device."""
    st = ctypes.c_int32(-1)
    _check(lib().slra_noalloc_device_status(_stream_handle(stream), ctypes.byref(st)), "slra_noalloc_device_status")
    return int(st.value)


def device_status(workspace, stream=None) -> int:
    st = ctypes.c_int32(-1)
    _check(lib().slra_device_status(_ptr(workspace), _stream_handle(stream), ctypes.byref(st)),
           "slra_device_status")
    return int(st.value)


def ws_view(prob: Problem, workspace, name: str):
    """A typed view of one intermediate inside a workspace (see slra_ws_layout)."""
    torch = _torch()
    lay = layout(prob)
    BH, nb, D, R, k = prob.batch * prob.heads, lay.nb, prob.head_dim, prob.rank, lay.keep
    spec = {"qh": (torch.float16, (BH, nb * prob.block, D)), "kh": (torch.float16, (BH, nb * prob.block, D)),
            "vh": (torch.float16, (BH, nb * prob.block, D)), "qbar": (torch.float64, (BH, nb, D)),
            "kbar": (torch.float64, (BH, nb, D)), "idx": (torch.int32, (BH, nb, k)),
            "tie": (torch.uint8, (BH, nb)), "S": (torch.float32, (BH, R, D)), "z": (torch.float32, (BH, R))}
    dt, shape = spec[name]
    off = lay.offsets[name]
    n = 1
    for s in shape:
        n *= s
    nbytes = n * torch.empty(0, dtype=dt).element_size()
    return workspace[off:off + nbytes].view(dt).view(shape)
