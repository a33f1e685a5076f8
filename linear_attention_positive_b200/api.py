"""ctypes binding of libfavor.so (C ABI in include/favor.h): argument marshalling only.

Every computation runs in the library's kernels; PyTorch provides device memory and streams.
The library is loaded on first use; if it is missing this raises ``FavorError`` (there is no CPU
fallback).
"""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfavor.so")

FAVOR_OK = 0
FAVOR_ERR_INVALID_ARG = 1
FAVOR_ERR_UNSUPPORTED = 2
FAVOR_ERR_CUDA = 3
FAVOR_ERR_TIMEOUT = 4
FAVOR_ERR_WORKSPACE = 5
FAVOR_F32 = 0
FAVOR_BF16 = 1

# Exported entry points, in the order include/favor.h declares them.
EXPORTS = (
    "favor_draw_features",
    "favor_workspace_size",
    "favor_ctx_size",
    "favor_fwd",
    "favor_bwd",
    "favor_sync_status",
    "favor_status_string",
    "favor_sp_state_size",
    "favor_sp_workspace_size",
    "favor_sp_state",
    "favor_sp_output",
    "favor_decode_state_size",
    "favor_decode_step",
    "favor_selftest_bounded_wait",
    "favor_fwd_static_scratch",
)


class FavorError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        msg = status_string(status) if _LIB is not None else f"status {status}"
        super().__init__(f"{what}: {msg}" if what else msg)


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int), ("d", ctypes.c_int),
                ("m", ctypes.c_int), ("dtype", ctypes.c_int)]


FAVOR_MAX_STAGES = 24


FAVOR_MAP_POSITIVE = 0
FAVOR_MAP_RELU = 1
FAVOR_MAP_TRIG = 2


class Opts(ctypes.Structure):
    _fields_ = [("split_tiles", ctypes.c_int), ("exp_poly_pct", ctypes.c_int), ("feature_map", ctypes.c_int),
                ("reserved", ctypes.c_int * 5), ("stage_events", ctypes.POINTER(ctypes.c_void_p))]


_LIB = None


def library():
    """The loaded libfavor.so (ctypes.CDLL) with argument types declared."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise FavorError(FAVOR_ERR_CUDA, f"{LIB_PATH} is not built (run linear_attention_positive_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
    SP, OP = ctypes.POINTER(Shape), ctypes.POINTER(Opts)
    lib.favor_draw_features.argtypes = [U64, I, I, ctypes.POINTER(ctypes.c_double)]
    lib.favor_draw_features.restype = I
    lib.favor_workspace_size.argtypes = [SP, I, I, OP]
    lib.favor_workspace_size.restype = Z
    lib.favor_ctx_size.argtypes = [SP, I]
    lib.favor_ctx_size.restype = Z
    lib.favor_fwd.argtypes = [SP, P, P, P, P, I, P, P, P, Z, OP, P]
    lib.favor_fwd.restype = I
    lib.favor_bwd.argtypes = [SP, P, P, P, P, P, P, P, I, P, P, P, P, Z, OP, P]
    lib.favor_bwd.restype = I
    lib.favor_sync_status.argtypes = [P]
    lib.favor_sync_status.restype = I
    lib.favor_status_string.argtypes = [I]
    lib.favor_status_string.restype = ctypes.c_char_p
    lib.favor_sp_state_size.argtypes = [SP]
    lib.favor_sp_state_size.restype = Z
    lib.favor_sp_workspace_size.argtypes = [SP]
    lib.favor_sp_workspace_size.restype = Z
    lib.favor_sp_state.argtypes = [SP, P, P, P, P, P, Z, P]
    lib.favor_sp_state.restype = I
    lib.favor_sp_output.argtypes = [SP, P, P, P, P, P, Z, P]
    lib.favor_sp_output.restype = I
    lib.favor_decode_state_size.argtypes = [SP]
    lib.favor_decode_state_size.restype = Z
    lib.favor_decode_step.argtypes = [SP, P, P, P, P, P, P, P]
    lib.favor_decode_step.restype = I
    lib.favor_selftest_bounded_wait.argtypes = [ctypes.c_uint, P]
    lib.favor_selftest_bounded_wait.restype = I
    lib.favor_fwd_static_scratch.argtypes = [SP, P, P, P, P, P, P]
    lib.favor_fwd_static_scratch.restype = I
    _LIB = lib
    return lib


def status_string(status):
    return library().favor_status_string(int(status)).decode()


def _check(status, what):
    if status != FAVOR_OK:
        raise FavorError(status, what)


def make_shape(B, H, L, d, m, dtype):
    return Shape(B, H, L, d, m, dtype)


def make_opts(split_tiles=0, exp_poly_pct=0, stage_events=None, feature_map=FAVOR_MAP_POSITIVE):
    """Options struct. ``stage_events``: optional list of 2*FAVOR_MAX_STAGES torch.cuda.Event
    (enable_timing=True, already recorded once so their handles exist) or None entries."""
    o = Opts(split_tiles, exp_poly_pct, feature_map, (ctypes.c_int * 5)(), None)
    if stage_events is not None:
        arr = (ctypes.c_void_p * (2 * FAVOR_MAX_STAGES))()
        for i, ev in enumerate(stage_events[: 2 * FAVOR_MAX_STAGES]):
            arr[i] = ev.cuda_event if ev is not None else None
        o._events_keepalive = arr
        o.stage_events = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    return o


def draw_features(seed, m, d):
    """Block-orthogonal random features W (m x d, float64), drawn on the host by the library."""
    out = np.empty((m, d), dtype=np.float64)
    st = library().favor_draw_features(ctypes.c_uint64(seed & (2**64 - 1)), int(m), int(d),
                                       out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    _check(st, "favor_draw_features")
    return out


def _torch():
    import torch
    return torch


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return FAVOR_BF16
    if t.dtype == torch.float32:
        return FAVOR_F32
    raise FavorError(FAVOR_ERR_INVALID_ARG, f"unsupported dtype {t.dtype}")


def _shape_of(Q, W):
    B, H, L, d = Q.shape
    return make_shape(B, H, L, d, W.shape[0], _dtype_code(Q))


def workspace_size(shape, causal=False, backward=False, opts=None):
    return library().favor_workspace_size(ctypes.byref(shape), int(causal), int(backward),
                                          ctypes.byref(opts) if opts is not None else None)


def ctx_size(shape, causal=False):
    return library().favor_ctx_size(ctypes.byref(shape), int(causal))


def _stream_ptr(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _alloc_bytes(n, device):
    torch = _torch()
    return torch.empty(max(int(n), 256), dtype=torch.uint8, device=device)


def _check_inputs(tensors, dtype_like):
    for t in tensors:
        if not t.is_cuda or not t.is_contiguous():
            raise FavorError(FAVOR_ERR_INVALID_ARG, "tensors must be contiguous CUDA tensors")
        if t.dtype != dtype_like.dtype:
            raise FavorError(FAVOR_ERR_INVALID_ARG, "Q, K, V, W (and dout) must share one dtype")


def fwd(Q, K, V, W, causal=False, out=None, ctx=None, workspace=None, opts=None, stream=None):
    """FAVOR+ forward through favor_fwd. Q, K, V: [B,H,L,d] bf16 or fp32 CUDA tensors; W: [m,d] in
    the same dtype. Returns the fp32 output (and fills ``ctx`` when given)."""
    torch = _torch()
    _check_inputs((Q, K, V, W), Q)
    shape = _shape_of(Q, W)
    if out is None:
        out = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
    if workspace is None:
        ws_n = workspace_size(shape, causal, False, opts)
        if ws_n == 0:
            raise FavorError(FAVOR_ERR_UNSUPPORTED, "favor_workspace_size")
        workspace = _alloc_bytes(ws_n, Q.device)
    st = library().favor_fwd(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(W), int(causal), _ptr(out),
                             _ptr(ctx), _ptr(workspace), workspace.numel(),
                             ctypes.byref(opts) if opts is not None else None, _stream_ptr(stream))
    _check(st, "favor_fwd")
    return out


def bwd(Q, K, V, W, out, dout, ctx=None, causal=False, workspace=None, opts=None, stream=None):
    """Gradients (dQ, dK, dV) (fp32) of sum(dout * out) through favor_bwd, W fixed."""
    torch = _torch()
    _check_inputs((Q, K, V, W, dout), Q)
    shape = _shape_of(Q, W)
    dQ, dK, dV = (torch.empty(Q.shape, dtype=torch.float32, device=Q.device) for _ in range(3))
    if workspace is None:
        ws_n = workspace_size(shape, causal, True, opts)
        if ws_n == 0:
            raise FavorError(FAVOR_ERR_UNSUPPORTED, "favor_workspace_size")
        workspace = _alloc_bytes(ws_n, Q.device)
    st = library().favor_bwd(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(W), _ptr(out), _ptr(dout),
                             _ptr(ctx), int(causal), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(workspace),
                             workspace.numel(), ctypes.byref(opts) if opts is not None else None,
                             _stream_ptr(stream))
    _check(st, "favor_bwd")
    return dQ, dK, dV


def bwd_into(Q, K, V, W, out, dout, dQ, dK, dV, ctx=None, causal=False, workspace=None, opts=None, stream=None):
    """favor_bwd writing into caller-provided fp32 gradient tensors (no allocation when a workspace
    is given)."""
    _check_inputs((Q, K, V, W, dout), Q)
    shape = _shape_of(Q, W)
    if workspace is None:
        ws_n = workspace_size(shape, causal, True, opts)
        if ws_n == 0:
            raise FavorError(FAVOR_ERR_UNSUPPORTED, "favor_workspace_size")
        workspace = _alloc_bytes(ws_n, Q.device)
    st = library().favor_bwd(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(W), _ptr(out), _ptr(dout),
                             _ptr(ctx), int(causal), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(workspace),
                             workspace.numel(), ctypes.byref(opts) if opts is not None else None,
                             _stream_ptr(stream))
    _check(st, "favor_bwd")
    return dQ, dK, dV


def sync_status(stream=None):
    """Synchronise the stream and return (and clear) the device status word."""
    return library().favor_sync_status(_stream_ptr(stream))


def sp_state(K, V, W, state=None, workspace=None, stream=None):
    """Partial state [B*H, m, d+64] (fp32) of this run of keys through favor_sp_state."""
    torch = _torch()
    _check_inputs((K, V, W), K)
    shape = _shape_of(K, W)
    lib = library()
    if state is None:
        state = torch.empty(lib.favor_sp_state_size(ctypes.byref(shape)) // 4, dtype=torch.float32, device=K.device)
    if workspace is None:
        workspace = _alloc_bytes(lib.favor_sp_workspace_size(ctypes.byref(shape)), K.device)
    st = lib.favor_sp_state(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(W), _ptr(state), _ptr(workspace),
                            workspace.numel(), _stream_ptr(stream))
    _check(st, "favor_sp_state")
    return state


def sp_output(Q, W, state, out=None, workspace=None, stream=None):
    """Outputs of this run of queries against a total state, through favor_sp_output."""
    torch = _torch()
    _check_inputs((Q, W), Q)
    shape = _shape_of(Q, W)
    lib = library()
    if out is None:
        out = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
    if workspace is None:
        workspace = _alloc_bytes(lib.favor_sp_workspace_size(ctypes.byref(shape)), Q.device)
    st = lib.favor_sp_output(ctypes.byref(shape), _ptr(Q), _ptr(W), _ptr(state), _ptr(out), _ptr(workspace),
                             workspace.numel(), _stream_ptr(stream))
    _check(st, "favor_sp_output")
    return out


def sp_forward(Q, K, V, W, group=None, state_fn=None, output_fn=None):
    """Sequence-parallel bidirectional forward: this rank holds a contiguous run of every head's
    tokens; its partial key state is summed over the ranks of ``group`` (one all-reduce) and its
    queries are answered from the total. ``state_fn`` / ``output_fn`` default to sp_state /
    sp_output (tests substitute host stand-ins to exercise the exchange without a GPU)."""
    import torch.distributed as dist

    state = (state_fn or sp_state)(K, V, W)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(state, op=dist.ReduceOp.SUM, group=group)
    return (output_fn or sp_output)(Q, W, state)


def decode_state(B, H, d, m, device):
    """A zero (empty) carried state for favor_decode_step."""
    torch = _torch()
    n = library().favor_decode_state_size(ctypes.byref(make_shape(B, H, 1, d, m, FAVOR_F32)))
    if n == 0:
        raise FavorError(FAVOR_ERR_UNSUPPORTED, "favor_decode_state_size")
    return torch.zeros(n // 4, dtype=torch.float32, device=device)


def decode_step(q, k, v, W, state, out=None, stream=None):
    """One token per head through favor_decode_step. q, k, v: [B,H,d] (bf16 or fp32); state from
    decode_state(), updated in place. Returns the fp32 output [B,H,d]."""
    torch = _torch()
    _check_inputs((q, k, v, W), q)
    B, H, d = q.shape
    shape = make_shape(B, H, 1, d, W.shape[0], _dtype_code(q))
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    st = library().favor_decode_step(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(state),
                                     _ptr(out), _stream_ptr(stream))
    _check(st, "favor_decode_step")
    return out


def selftest_bounded_wait(limit_us, stream=None):
    """Launches the library's bounded-wait self-test (a wait that nothing ends, given up after
    limit_us); the next sync_status() reports FAVOR_ERR_TIMEOUT."""
    _check(library().favor_selftest_bounded_wait(int(limit_us), _stream_ptr(stream)), "favor_selftest_bounded_wait")


STATIC_SCRATCH_BYTES = 32 << 20


def fwd_static_scratch(Q, K, V, W, out=None, stream=None):
    """Bidirectional bf16 forward through favor_fwd_static_scratch: no workspace is passed, the
    library uses its own fixed device array (for callers that cannot allocate device memory)."""
    torch = _torch()
    _check_inputs((Q, K, V, W), Q)
    shape = _shape_of(Q, W)
    if out is None:
        out = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
    st = library().favor_fwd_static_scratch(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(W), _ptr(out),
                                            _stream_ptr(stream))
    _check(st, "favor_fwd_static_scratch")
    return out
