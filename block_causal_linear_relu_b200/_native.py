"""ctypes binding of libsvlinattn.so: argument marshalling only, every step runs in the library.

Functions carry the C entry points' names. Tensors are torch CUDA tensors (PyTorch supplies device
memory and streams); outputs and the workspace are allocated here when the caller gives none.
There is no fallback: if the shared library is missing or the device is not a B200 the call
raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsvlinattn.so")
_lib = None
_lock = threading.Lock()

SV_OK, SV_ERR_INVALID_ARG, SV_ERR_UNSUPPORTED, SV_ERR_CUDA, SV_ERR_TIMEOUT = range(5)
SV_BF16, SV_F32 = 0, 1
SV_OP_LINATTN_FWD, SV_OP_BLOCK_STATE_UPDATE, SV_OP_BLOCK_CAUSAL_ATTN, SV_OP_CACHE_STEP = range(4)

#: every symbol include/svlinattn.h declares
EXPORTS = (
    "sv_workspace_bytes", "sv_workspace_init", "sv_device_status", "sv_workspace_set_mirror", "sv_linattn_fwd",
    "sv_block_state_update", "sv_block_causal_attn", "sv_cache_step", "sv_cache_step_noalloc",
    "sv_cache_step_noalloc_status", "sv_temporal_conv", "sv_temporal_conv_step", "sv_qkv_projection",
    "sv_out_projection", "sv_rope3d_table_bytes", "sv_rope3d_table", "sv_block_causal_attn_rope", "sv_profile_events",
    "sv_last_error", "sv_selftest_wait_timeout", "sv_version",
)


class SvRope3d(ctypes.Structure):
    """The C descriptor sv_rope3d (include/svlinattn.h)."""

    _fields_ = [("table", ctypes.c_void_p), ("frames", ctypes.c_int), ("height", ctypes.c_int),
                ("width", ctypes.c_int), ("D", ctypes.c_int), ("pairs_t", ctypes.c_int), ("pairs_h", ctypes.c_int),
                ("pairs_w", ctypes.c_int), ("frame0", ctypes.c_int)]


class SvError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"sv status {status}: {msg}")
        self.status = status


def lib_path() -> str:
    return _LIB_PATH


def load() -> ctypes.CDLL:
    """Load libsvlinattn.so (built in-tree by block_causal_linear_relu_b200.build)."""
    global _lib
    if _lib is not None:  # loaded: no lock on the per-call path
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with `python -m block_causal_linear_relu_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, sz, i, f, u32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float, ctypes.POINTER(ctypes.c_uint32)
        lib.sv_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
        lib.sv_workspace_bytes.restype = sz
        lib.sv_workspace_init.argtypes = [vp, sz, vp]
        lib.sv_workspace_init.restype = i
        lib.sv_device_status.argtypes = [vp, vp, u32p]
        lib.sv_device_status.restype = i
        lib.sv_workspace_set_mirror.argtypes = [vp, sz, vp, vp]
        lib.sv_workspace_set_mirror.restype = i
        lib.sv_linattn_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
        lib.sv_linattn_fwd.restype = i
        lib.sv_block_state_update.argtypes = [vp, vp, i, i, i, i, i, vp, vp, vp, sz, vp]
        lib.sv_block_state_update.restype = i
        lib.sv_block_causal_attn.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, vp, vp, vp, vp, vp, sz, vp]
        lib.sv_block_causal_attn.restype = i
        lib.sv_cache_step.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, vp, vp, i, vp, sz, vp]
        lib.sv_cache_step.restype = i
        lib.sv_cache_step_noalloc.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, vp, vp, i, vp]
        lib.sv_cache_step_noalloc.restype = i
        lib.sv_cache_step_noalloc_status.argtypes = [vp, u32p]
        lib.sv_cache_step_noalloc_status.restype = i
        lib.sv_temporal_conv.argtypes = [vp, vp, i, i, i, i, i, vp, vp, i, vp]
        lib.sv_temporal_conv.restype = i
        lib.sv_temporal_conv_step.argtypes = [vp, vp, i, i, i, i, vp, vp, vp, i, i, vp]
        lib.sv_temporal_conv_step.restype = i
        lib.sv_qkv_projection.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, vp, sz, vp]
        lib.sv_qkv_projection.restype = i
        lib.sv_out_projection.argtypes = [vp, vp, vp, i, i, i, i, i, vp, sz, vp]
        lib.sv_out_projection.restype = i
        lib.sv_rope3d_table_bytes.argtypes = [i, i, i, i]
        lib.sv_rope3d_table_bytes.restype = sz
        lib.sv_rope3d_table.argtypes = [vp, sz, i, i, i, i, i, i, i, f, vp]
        lib.sv_rope3d_table.restype = i
        lib.sv_block_causal_attn_rope.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, vp, vp, vp, vp,
                                                  ctypes.POINTER(SvRope3d), vp, sz, vp]
        lib.sv_block_causal_attn_rope.restype = i
        lib.sv_profile_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), i]
        lib.sv_profile_events.restype = i
        lib.sv_last_error.argtypes = []
        lib.sv_last_error.restype = ctypes.c_char_p
        lib.sv_selftest_wait_timeout.argtypes = [vp, sz, vp]
        lib.sv_selftest_wait_timeout.restype = i
        lib.sv_version.argtypes = []
        lib.sv_version.restype = i
        _lib = lib
        return lib


def _check(status: int):
    if status != SV_OK:
        raise SvError(status, load().sv_last_error().decode())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SV_BF16
    if t.dtype == torch.float32:
        return SV_F32
    raise TypeError(f"unsupported dtype {t.dtype}: bfloat16 or float32 expected")


def _ptr(t):
    # plain ints (and None) convert to the c_void_p parameters without a ctypes object per call
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _qkv(*ts):
    """Checks q, k, v (and o) in one pass; returns their shape [B, H, N, D]."""
    ref = ts[0]
    shape, dtype, device = ref.shape, ref.dtype, ref.device
    if not ref.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if len(shape) != 4:
        raise ValueError("q, k, v, o must share shape [B, H, N, D], dtype and device")
    for t in ts:
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, H, N, D]")
        if t is not ref and (t.shape != shape or t.dtype != dtype or t.device != device):
            raise ValueError("q, k, v, o must share shape [B, H, N, D], dtype and device")
    return shape


def workspace_bytes(op: int, B: int, H: int, N: int, D: int, block_len: int, dtype: int, device=None) -> int:
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        n = load().sv_workspace_bytes(op, B, H, N, D, block_len, dtype)
    if n == 0:
        raise SvError(SV_ERR_INVALID_ARG, load().sv_last_error().decode())
    return int(n)


class Workspace:
    """Caller-owned device scratch: a 256-byte aligned view into a torch uint8 buffer.

    A page-locked host word is registered as the workspace's status mirror: a kernel whose bounded
    wait expires writes its status code there as well, so every later call of this binding on the
    workspace raises SvError(SV_ERR_TIMEOUT) before it launches anything (``check``), without a
    synchronisation per call. ``status`` synchronises, reads and clears the device word.
    """

    def __init__(self, nbytes: int, device, stream=None):
        self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.view = self.buf[off:off + nbytes]
        self.nbytes = nbytes
        self._ptr = self.view.data_ptr()
        self._mirror = torch.zeros(1, dtype=torch.int32).pin_memory()
        self._mirror_np = self._mirror.numpy()
        lib = load()
        with torch.cuda.device(self.buf.device):
            _check(lib.sv_workspace_init(self._ptr, nbytes, _stream(stream)))
            _check(lib.sv_workspace_set_mirror(self._ptr, nbytes, self._mirror.data_ptr(), _stream(stream)))

    @property
    def ptr(self):
        return self._ptr

    def status(self, stream=None) -> int:
        """Synchronise, return the device status word (0 = no timeout) and clear it (and the mirror)."""
        code = ctypes.c_uint32(0)
        st = load().sv_device_status(self.ptr, _stream(stream), ctypes.byref(code))
        if st not in (SV_OK, SV_ERR_TIMEOUT):
            _check(st)
        self._mirror_np[0] = 0
        return int(code.value)

    def check(self, stream=None):
        """Raise SvError(SV_ERR_TIMEOUT) if a kernel has reported a timeout on this workspace since the
        last check (reads the host mirror: no synchronisation unless a timeout was reported)."""
        if self._mirror_np[0] != 0:
            code = self.status(stream)
            raise SvError(SV_ERR_TIMEOUT, f"a kernel's bounded wait expired on this workspace "
                                          f"(status word 0x{code:08x}); its output was not written")


def sv_selftest_wait_timeout(ws: Workspace, stream=None):
    """Launch the bounded-wait self-test on `ws` (its status word is raised about 2 s later; read it
    with ws.status())."""
    _check(load().sv_selftest_wait_timeout(ws.ptr, ws.nbytes, _stream(stream)))


def make_workspace(op: int, q_like: torch.Tensor, block_len: int | None = None, stream=None) -> Workspace:
    B, H, N, D = q_like.shape
    n = workspace_bytes(op, B, H, N, D, block_len if block_len is not None else N, _dt(q_like), q_like.device)
    return Workspace(n, q_like.device, stream)


_default_ws = {}


def _ws(ws, op, q_like, block_len, stream):
    """The caller's workspace, else one kept per (device, stream, op, sizes), so that calls without
    an explicit workspace reuse it (calls on one stream are ordered) and see its reported timeouts."""
    if ws is None:
        B, H, N, D = q_like.shape
        key = (q_like.device.index, _stream(stream), op, B, H, N, D, block_len, q_like.dtype)
        ws = _default_ws.get(key)
        if ws is None:
            ws = _default_ws[key] = make_workspace(op, q_like, block_len, stream)
    ws.check(stream)
    return ws


def sv_linattn_fwd(q, k, v, o=None, eps: float = 1e-6, ws: Workspace | None = None, stream=None):
    """Bidirectional ReLU linear attention; returns o."""
    o = torch.empty_like(q) if o is None else o
    B, H, N, D = _qkv(q, k, v, o)
    ws = _ws(ws, SV_OP_LINATTN_FWD, q, None, stream)
    _check(load().sv_linattn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, D, _dt(q), eps, ws.ptr, ws.nbytes,
                                 _stream(stream)))
    return o


def sv_block_causal_attn(q, k, v, block_len: int, o=None, eps: float = 1e-6, S_in=None, z_in=None, S_out=None,
                         z_out=None, ws: Workspace | None = None, stream=None):
    """Block-causal prefill; returns o (S_out/z_out are written in place when given)."""
    o = torch.empty_like(q) if o is None else o
    B, H, N, D = _qkv(q, k, v, o)
    for t in (S_in, z_in, S_out, z_out):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous() or t.device != q.device):
            raise ValueError("S/z must be contiguous float32 tensors on q's device")
    ws = _ws(ws, SV_OP_BLOCK_CAUSAL_ATTN, q, block_len, stream)
    _check(load().sv_block_causal_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, D, int(block_len), _dt(q), eps,
                                       _ptr(S_in), _ptr(z_in), _ptr(S_out), _ptr(z_out), ws.ptr, ws.nbytes,
                                       _stream(stream)))
    return o


def sv_cache_step(q, k, v, S, z, commit: bool = True, o=None, eps: float = 1e-6, ws: Workspace | None = None,
                  stream=None):
    """One streaming block against the fp32 cache (S [B,H,D,D], z [B,H,D]); returns o."""
    o = torch.empty_like(q) if o is None else o
    B, H, N, D = _qkv(q, k, v, o)
    if S.dtype != torch.float32 or z.dtype != torch.float32 or tuple(S.shape) != (B, H, D, D) or tuple(z.shape) != (B, H, D):
        raise ValueError("cache must be float32 S [B,H,D,D] and z [B,H,D]")
    ws = _ws(ws, SV_OP_CACHE_STEP, q, None, stream)
    _check(load().sv_cache_step(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, D, _dt(q), eps, _ptr(S), _ptr(z),
                                1 if commit else 0, ws.ptr, ws.nbytes, _stream(stream)))
    return o


def sv_cache_step_noalloc(q, k, v, S, z, commit: bool = True, o=None, eps: float = 1e-6, stream=None):
    """sv_cache_step with the library's static scratch instead of a workspace (see the header)."""
    o = torch.empty_like(q) if o is None else o
    B, H, N, D = _qkv(q, k, v, o)
    if S.dtype != torch.float32 or z.dtype != torch.float32 or tuple(S.shape) != (B, H, D, D) or tuple(z.shape) != (B, H, D):
        raise ValueError("cache must be float32 S [B,H,D,D] and z [B,H,D]")
    _check(load().sv_cache_step_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, D, _dt(q), eps, _ptr(S),
                                        _ptr(z), 1 if commit else 0, _stream(stream)))
    return o


def sv_cache_step_noalloc_status(stream=None) -> int:
    """Synchronise and return (then clear) the status word of sv_cache_step_noalloc's static scratch
    on the current device (0 = no timeout)."""
    code = ctypes.c_uint32(0)
    st = load().sv_cache_step_noalloc_status(_stream(stream), ctypes.byref(code))
    if st not in (SV_OK, SV_ERR_TIMEOUT):
        _check(st)
    return int(code.value)


def sv_profile_events(events):
    """Install (list of 4 torch.cuda.Event, already recorded once) or clear (None) the timing hook."""
    if events is None:
        _check(load().sv_profile_events(None, 0))
        return
    arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(load().sv_profile_events(arr, 4))


def sv_block_state_update(k, v, S, z, ws: Workspace | None = None, stream=None):
    """S += ReLU(K)^T V, z += sum ReLU(k), in place."""
    B, H, N, D = _qkv(k, v)
    if S.dtype != torch.float32 or z.dtype != torch.float32 or tuple(S.shape) != (B, H, D, D) or tuple(z.shape) != (B, H, D):
        raise ValueError("cache must be float32 S [B,H,D,D] and z [B,H,D]")
    ws = _ws(ws, SV_OP_BLOCK_STATE_UPDATE, k, None, stream)
    _check(load().sv_block_state_update(_ptr(k), _ptr(v), B, H, N, D, _dt(k), _ptr(S), _ptr(z), ws.ptr, ws.nbytes,
                                        _stream(stream)))
    return S, z


def _conv_args(x, w, bias):
    if not x.is_cuda or x.dim() != 4 or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor [B, T, S, C]")
    C = x.shape[3]
    if w.dtype != torch.float32 or tuple(w.shape) != (C, 3) or not w.is_contiguous() or w.device != x.device:
        raise ValueError("w must be a contiguous float32 [C, 3] tensor on x's device")
    if bias is not None and (bias.dtype != torch.float32 or tuple(bias.shape) != (C,) or bias.device != x.device):
        raise ValueError("bias must be a float32 [C] tensor on x's device")


def sv_temporal_conv(x, w, frames_per_block: int, bias=None, y=None, stream=None):
    """Block-causal temporal convolution over x [B, T, S, C] (kernel width 3); returns y."""
    _conv_args(x, w, bias)
    y = torch.empty_like(x) if y is None else y
    B, T, S, C = x.shape
    _check(load().sv_temporal_conv(_ptr(x), _ptr(y), B, T, S, C, int(frames_per_block), _ptr(w), _ptr(bias), _dt(x),
                                   _stream(stream)))
    return y


def sv_temporal_conv_step(x, w, carry, commit: bool = True, bias=None, y=None, stream=None):
    """One block x [B, T, S, C] of a stream with the previous block's last frame in carry [B, S, C]
    (zeros before the first block); carry takes x's last frame if commit. Returns y."""
    _conv_args(x, w, bias)
    B, T, S, C = x.shape
    if carry.dtype != x.dtype or tuple(carry.shape) != (B, S, C) or not carry.is_contiguous():
        raise ValueError("carry must be a contiguous [B, S, C] tensor of x's dtype")
    y = torch.empty_like(x) if y is None else y
    _check(load().sv_temporal_conv_step(_ptr(x), _ptr(y), B, T, S, C, _ptr(w), _ptr(bias), _ptr(carry),
                                        1 if commit else 0, _dt(x), _stream(stream)))
    return y


_proj_ws = {}


def _proj_workspace(device, stream):
    key = (device.index, _stream(stream))
    ws = _proj_ws.get(key)
    if ws is None:
        ws = _proj_ws[key] = Workspace(256, device, stream)
    ws.check(stream)
    return ws


def sv_qkv_projection(x, w_qkv, H: int, D: int, q=None, k=None, v=None, ws: Workspace | None = None, stream=None):
    """x [B, N, C] bf16, w_qkv [3*H*D, C] bf16 -> (ReLU(q), ReLU(k), v), each [B, H, N, D] bf16."""
    if not x.is_cuda or x.dim() != 3 or x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("x must be a contiguous bfloat16 CUDA tensor [B, N, C]")
    B, N, C = x.shape
    if tuple(w_qkv.shape) != (3 * H * D, C) or w_qkv.dtype != torch.bfloat16 or not w_qkv.is_contiguous():
        raise ValueError("w_qkv must be a contiguous bfloat16 [3*H*D, C] tensor")
    q, k, v = (torch.empty(B, H, N, D, dtype=torch.bfloat16, device=x.device) if t is None else t for t in (q, k, v))
    ws = ws if ws is not None else _proj_workspace(x.device, stream)
    _check(load().sv_qkv_projection(_ptr(x), _ptr(w_qkv), _ptr(q), _ptr(k), _ptr(v), B, N, C, H, D, ws.ptr, ws.nbytes,
                                    _stream(stream)))
    return q, k, v


def sv_out_projection(o, w_o, y=None, ws: Workspace | None = None, stream=None):
    """o [B, H, N, D] bf16, w_o [C_out, H*D] bf16 -> y [B, N, C_out] bf16."""
    if not o.is_cuda or o.dim() != 4 or o.dtype != torch.bfloat16 or not o.is_contiguous():
        raise ValueError("o must be a contiguous bfloat16 CUDA tensor [B, H, N, D]")
    B, H, N, D = o.shape
    if w_o.dim() != 2 or w_o.shape[1] != H * D or w_o.dtype != torch.bfloat16 or not w_o.is_contiguous():
        raise ValueError("w_o must be a contiguous bfloat16 [C_out, H*D] tensor")
    C_out = w_o.shape[0]
    y = torch.empty(B, N, C_out, dtype=torch.bfloat16, device=o.device) if y is None else y
    ws = ws if ws is not None else _proj_workspace(o.device, stream)
    _check(load().sv_out_projection(_ptr(o), _ptr(w_o), _ptr(y), B, N, H, D, C_out, ws.ptr, ws.nbytes, _stream(stream)))
    return y


def rope_pairs(D: int):
    """A split of the D/2 rotation pairs over (frame, row, column): row and column get D // 6 pairs
    each, the frame axis the rest (22, 21, 21 for D = 128)."""
    ph = D // 6
    return (D // 2 - 2 * ph, ph, ph)


def sv_rope3d_table_bytes(frames: int, height: int, width: int, D: int) -> int:
    n = load().sv_rope3d_table_bytes(frames, height, width, D)
    if n == 0:
        raise SvError(SV_ERR_INVALID_ARG, load().sv_last_error().decode())
    return n


class Rope3dTable:
    """The device (cos, sin) table of the 3D rotary embedding for one grid and feature split, built
    by sv_rope3d_table; `desc(frame0)` gives the sv_rope3d descriptor of a call."""

    def __init__(self, frames: int, height: int, width: int, D: int, pairs, base: float = 10000.0, device=None,
                 stream=None):
        pt, ph, pw = (int(p) for p in pairs)
        nbytes = sv_rope3d_table_bytes(frames, height, width, D)
        self.table = torch.empty(nbytes // 4, dtype=torch.float32, device=device or torch.device("cuda"))
        self.frames, self.height, self.width, self.D, self.pairs = frames, height, width, D, (pt, ph, pw)
        _check(load().sv_rope3d_table(self.table.data_ptr(), nbytes, frames, height, width, D, pt, ph, pw, base,
                                      _stream(stream)))

    def desc(self, frame0: int = 0) -> SvRope3d:
        pt, ph, pw = self.pairs
        return SvRope3d(self.table.data_ptr(), self.frames, self.height, self.width, self.D, pt, ph, pw, int(frame0))


def sv_rope3d_table(frames: int, height: int, width: int, D: int, pairs, base: float = 10000.0, device=None,
                    stream=None) -> Rope3dTable:
    return Rope3dTable(frames, height, width, D, pairs, base, device, stream)


def sv_block_causal_attn_rope(q, k, v, block_len: int, rope: Rope3dTable, frame0: int = 0, o=None, eps: float = 1e-6,
                              S_in=None, z_in=None, S_out=None, z_out=None, ws: Workspace | None = None, stream=None):
    """sv_block_causal_attn with the 3D rotary embedding of the numerator; returns o."""
    o = torch.empty_like(q) if o is None else o
    B, H, N, D = _qkv(q, k, v, o)
    for t in (S_in, z_in, S_out, z_out):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous() or t.device != q.device):
            raise ValueError("S/z must be contiguous float32 tensors on q's device")
    if rope.table.device != q.device:
        raise ValueError("the rope table must live on q's device")
    ws = _ws(ws, SV_OP_BLOCK_CAUSAL_ATTN, q, block_len, stream)
    d = rope.desc(frame0)
    _check(load().sv_block_causal_attn_rope(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, D, int(block_len), _dt(q),
                                            eps, _ptr(S_in), _ptr(z_in), _ptr(S_out), _ptr(z_out), ctypes.byref(d),
                                            ws.ptr, ws.nbytes, _stream(stream)))
    return o
